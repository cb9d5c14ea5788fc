"""Plain float64 CPU oracle for the KronQ per-linear-layer quantization path.

TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only the tests under ``tests/``, the
``smoke()`` check in ``__graft_entry__.py`` and the CPU-baseline leg of
``bench.py`` may import or run this module.  It shares no code with the CUDA
library (no kernels, helpers, tables or constants) and imports nothing from it.

Every function follows one step of the method as the source pages state it and
is written to be checked by eye: NumPy float64, library primitives (matmul,
inv, cholesky, kron) as single steps, no fusion and no reordering beyond what
the method itself prescribes.  Sources, cited by page and section:

[ABS]     KronQ paper page (Hugging Face papers 2607.07964): Abstract, and the
          authors' reply in its Community thread (one backward pass for H_G,
          reused across bit-widths; W2/W3/W4 per-channel settings).
[REV]     Paper review "KronQ: LLM Quantization via Kronecker-Factored
          Hessian" (romaanj.github.io/reviews/kronq): sections Background,
          Prior limitations, Goal, Method, Comparison, Limitations, and the
          research-thread essay "Where this paper sits".
[HZ]      "A Unified Hessian-Guided Framework for Post-Training Quantization"
          (hub.valency.io/works/W_r72x54u6): Background (quantization scales;
          transformations), Appendix A.1 (trace form of the Kronecker-weighted
          norm; rounding-noise model), Table 5 discussion (GPTQ rounding only
          sees the first Kronecker factor).

Where the pages leave a step open, the reading taken is named in the docstring
(R1..R11) and listed in the design notes of the repository.

Parity status: every function below is pinned by tests in ``tests/`` against
closed forms, brute force, textbook reductions or library routines.  The method
as a whole is not pinned against KronQ's own released outputs: the pages print
no per-layer values to compare with.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

__all__ = [
    "covariance", "covariance_accumulate", "sensitivity", "sylvester_hadamard",
    "rht_matrix", "rotate", "biip", "damp_and_dead", "chol_inv",
    "chol_inv_reversed", "fit_grid", "quantize_codes", "dequantize",
    "QuantResult", "quantize_layer", "kron_loss", "gptq_loss",
    "allocate_bits", "budget_units", "quantize_linear",
    "pack_codes", "unpack_codes", "dequantize_layer", "reverted_apply",
    "balance_permutation", "permutation_matrix", "hg_blockwise", "hg_lowrank", "block_rht_matrix",
    "blockwise_kron_loss", "weight_cv", "act_order_permutation", "quantize_layer_act_order",
]


# ---------------------------------------------------------------------------
# a1/a2. Covariance accumulation  ([REV] Background; [ABS] authors' reply)
# ---------------------------------------------------------------------------

def covariance(A, alpha=None, chunk=16384):
    """H = alpha * A^T A for tokens-by-channels A (default alpha = 1/n).

    [REV] Background: H_X is the input-activation covariance and H_G the
    output-gradient covariance, H_G = E[g g^T] ([REV] research thread).  With
    tokens as rows, E[x x^T] over n tokens is A^T A / n (reading: mean
    normalisation; GPTQ's factor 2 is dropped, the solver is scale free).
    The sum runs over token chunks in float64.
    """
    A = np.asarray(A)
    n, d = A.shape
    if alpha is None:
        alpha = 1.0 / n if n else 0.0
    H = np.zeros((d, d), dtype=np.float64)
    for t0 in range(0, n, chunk):
        a = A[t0:t0 + chunk].astype(np.float64)
        H += a.T @ a
    return H * float(alpha)


def covariance_accumulate(C, A, alpha):
    """C + alpha * A^T A: the streaming form used over successive token chunks."""
    return np.asarray(C, dtype=np.float64) + covariance(A, alpha)


# ---------------------------------------------------------------------------
# a3. Trace sensitivity  ([REV] Method (2); [ABS] Abstract (2))
# ---------------------------------------------------------------------------

def sensitivity(H_X, H_G):
    """(tr H_X, tr H_G, tr H_G * tr H_X).

    [REV] Method (2): the sublayer sensitivity is the product of the two traces;
    tr H_X alone is the H_X-only metric of the ablation ([REV] Comparison).
    """
    tX = float(np.trace(np.asarray(H_X, dtype=np.float64)))
    tG = float(np.trace(np.asarray(H_G, dtype=np.float64)))
    return tX, tG, tX * tG


# ---------------------------------------------------------------------------
# a4/a5. Randomised Hadamard rotations (bidirectional incoherence processing)
# ---------------------------------------------------------------------------

def sylvester_hadamard(p):
    """Unnormalised +-1 Walsh-Hadamard matrix of order p = 2^k, built by the
    Sylvester doubling H_{2p} = [[H_p, H_p], [H_p, -H_p]]."""
    if p < 1 or p & (p - 1):
        raise ValueError("Hadamard order must be a power of two")
    H = np.ones((1, 1), dtype=np.float64)
    while H.shape[0] < p:
        H = np.block([[H, H], [H, -H]])
    return H


def rht_matrix(n, log2_p, signs, Qm=None):
    """Dense T = (Q_m kron H_p / sqrt(p)) . diag(signs), n = m * 2^log2_p.

    [REV] Method (1) and [ABS] (1): an input-side random rotation extended to
    the output side; [HZ] Background (Transformations): orthogonal transforms
    mixing channels through randomised Hadamard transforms.  Reading R1/R8:
    both sides use this randomised Hadamard form; when n is not a power of two
    the odd factor m is mixed by a seeded orthogonal m x m matrix Q_m (identity
    when Qm is None, which requires m == 1).  Index convention: element
    a * p + b is (row a of Q_m, row b of H_p).
    """
    p = 1 << int(log2_p)
    if n % p:
        raise ValueError("n must be a multiple of 2^log2_p")
    m = n // p
    if Qm is None:
        if m != 1:
            raise ValueError("Qm is required when n is not a power of two")
        Q = np.ones((1, 1))
    else:
        Q = np.asarray(Qm, dtype=np.float64).reshape(m, m)
    Hp = sylvester_hadamard(p) / math.sqrt(p)
    s = np.asarray(signs, dtype=np.float64).reshape(n)
    return np.kron(Q, Hp) * s[None, :]


def rotate(M, axis, T, inverse=False):
    """Apply T (or T^T when inverse) along one axis of M.

    axis 'rows': M <- T . M  (T acts on the row index; each column transformed)
    axis 'cols': M <- M . T^T (T acts on the column index; each row transformed)
    """
    M = np.asarray(M, dtype=np.float64)
    Tm = np.asarray(T, dtype=np.float64)
    if inverse:
        Tm = Tm.T
    if axis == "rows":
        return Tm @ M
    if axis == "cols":
        return M @ Tm.T
    raise ValueError("axis must be 'rows' or 'cols'")


def biip(W, H_X, H_G, T_in, T_out):
    """Bidirectional incoherence processing of one layer y = W x.

    x' = U x with U = T_in, and the output side rotated by V = T_out:
    W' = V W U^T, H_X' = U H_X U^T, H_G' = V H_G V^T ([REV] Method (1);
    [HZ] Background: (X T)(T^-1 W) = Z, written here for y = W x).  The
    full-precision output is preserved: V^T W' U x = W x.
    """
    W = np.asarray(W, dtype=np.float64)
    Wp = rotate(rotate(W, "cols", T_in), "rows", T_out)
    HXp = rotate(rotate(H_X, "cols", T_in), "rows", T_in)
    HGp = rotate(rotate(H_G, "cols", T_out), "rows", T_out)
    return Wp, HXp, HGp


# ---------------------------------------------------------------------------
# a6. Damping, dead columns, Cholesky factor of the inverse (GPTQ solver set-up)
# ---------------------------------------------------------------------------

def damp_and_dead(H, damp_frac=0.01):
    """Dead columns get unit curvature, then lambda = damp * mean(diag) is added.

    Reading R6 (GPTQ convention): a column j with H[j, j] == 0 carries no
    signal; its diagonal is set to 1 (and its weights are zeroed in the
    solver).  The damping lambda = damp_frac * mean(diag H) is taken after that
    replacement and added to every diagonal entry.  H is symmetric by
    definition; a computed H can differ from its transpose by rounding, so the
    upper triangle is taken as the definition (mirrored onto the lower).
    """
    H = np.asarray(H, dtype=np.float64)
    H = np.triu(H) + np.triu(H, 1).T
    dead = np.diag(H) == 0
    idx = np.flatnonzero(dead)
    H[idx, idx] = 1.0
    lam = float(damp_frac) * float(np.mean(np.diag(H)))
    H[np.diag_indices_from(H)] += lam
    return H, dead, lam


def chol_inv(H, damp_frac=0.01):
    """Upper U_c with U_c^T U_c = (H_damped)^-1, via inv then Cholesky.

    [REV] Prior limitations / research thread: GPTQ solves the column-wise OBS
    update with H_X as the Hessian proxy; the solver needs the rows of the
    upper Cholesky factor of the damped inverse.  Raises
    numpy.linalg.LinAlgError when the damped matrix is not positive definite.
    """
    Hd, dead, lam = damp_and_dead(H, damp_frac)
    Hinv = np.linalg.inv(Hd)
    Hinv = 0.5 * (Hinv + Hinv.T)
    L = np.linalg.cholesky(Hinv)
    return L.T.copy(), dead, lam


def chol_inv_reversed(H, damp_frac=0.01):
    """The same U_c by a second route: H_damped = R R^T with R upper, U_c = R^-1.

    R comes from the ordinary lower Cholesky factor of the index-reversed
    matrix (J H J = L L^T gives R = J L J); then U_c^T U_c = R^-T R^-1 =
    (R R^T)^-1.  Used only to cross-check chol_inv.
    """
    Hd, dead, lam = damp_and_dead(H, damp_frac)
    L = np.linalg.cholesky(Hd[::-1, ::-1])
    R = L[::-1, ::-1]
    n = Hd.shape[0]
    Uc = np.linalg.solve(R, np.eye(n))
    return np.triu(Uc), dead, lam


# ---------------------------------------------------------------------------
# a7. Asymmetric min/max grid  (reading R2, R3)
# ---------------------------------------------------------------------------

def fit_grid(xmin, xmax, bits):
    """Per-row scale and zero of a b-bit asymmetric grid, in float32.

    [REV] Comparison: a plain uniform per-channel grid; [HZ] Background: a grid
    step s and a shift.  Reading R2: n_levels = 2^b - 1, scale = (max - min) /
    n_levels, zero = rint(-min / scale); a degenerate range (scale not > 0)
    uses scale = 1 and zero = rint(-min).  These quantities decide integers, so
    they are taken in the kernels' precision, IEEE float32 with
    round-half-to-even, in the same operation order.
    """
    xmin = np.asarray(xmin, dtype=np.float32)
    xmax = np.asarray(xmax, dtype=np.float32)
    nl = np.float32(2 ** int(bits) - 1)
    with np.errstate(divide="ignore", invalid="ignore", over="ignore"):
        scale = (xmax - xmin) / nl
        ok = scale > np.float32(0)
        scale = np.where(ok, scale, np.float32(1)).astype(np.float32)
        zero = np.where(ok, np.rint(-xmin / scale), np.rint(-xmin)).astype(np.float32)
    return scale, zero


def quantize_codes(w, scale, zero, bits):
    """Pre-rounding value v = w / scale + zero and code clamp(rint(v), 0, 2^b-1)."""
    nl = 2 ** int(bits) - 1
    v = np.asarray(w, dtype=np.float64) / np.float64(scale) + np.float64(zero)
    return v, np.clip(np.rint(v), 0, nl)


def dequantize(q, scale, zero):
    """w_hat = scale * (q - zero)."""
    return np.float64(scale) * (np.asarray(q, dtype=np.float64) - np.float64(zero))


# ---------------------------------------------------------------------------
# a8/a9. Blocked column-wise OBS solver (GPTQ; H_G cancels, Proposition 1)
# ---------------------------------------------------------------------------

@dataclasses.dataclass
class QuantResult:
    codes: np.ndarray        # uint8 [d_out, d_in]
    scales: np.ndarray       # float32 [d_out, n_groups]
    zeros: np.ndarray        # float32 [d_out, n_groups]
    W_hat: np.ndarray        # float64 [d_out, d_in], rotated coordinates
    V: np.ndarray            # float64 [d_out, d_in], pre-rounding values
    excused: int = 0         # codes adopted from force_codes under the excusal rule
    mismatches: list = dataclasses.field(default_factory=list)   # (row, col, v, ours, theirs)
    zero_excused: int = 0
    zero_mismatches: list = dataclasses.field(default_factory=list)
    snapshots: dict = dataclasses.field(default_factory=dict)    # col -> current W


def _excuse(ours, theirs, v, bits, tol):
    """Which disagreeing integer decisions are excused: v lies within tol of a
    rounding boundary k + 1/2 and the other side chose one of the two codes
    adjacent to that boundary (after clamping)."""
    nl = 2 ** int(bits) - 1
    fl = np.floor(v)
    near = np.abs(v - (fl + 0.5)) <= tol
    adj = (theirs == np.clip(fl, 0, nl)) | (theirs == np.clip(fl + 1, 0, nl))
    return (ours != theirs) & near & adj


def quantize_layer(W, Uc, bits, group=0, block=128, dead=None,
                   force_codes=None, force_zeros=None, excuse_tol=1e-5,
                   snapshot_cols=()):
    """GPTQ-style blocked OBS quantization of rotated weights W (rows = outputs).

    [REV] Goal / Method (1): the solver stays exactly the H_X-only column-wise
    OBS update; H_G cancels from it (Proposition 1; [HZ] Table 5 discussion).
    For each block [i, i+B) and each column j in it:
      q = Q(W[:, j]);  e = (W[:, j] - w_hat) / U_c[j, j];
      W[:, j+1:i+B] -= e U_c[j, j+1:i+B];  E[:, j-i] = e;
    and after the block W[:, i+B:] -= E U_c[i:i+B, i+B:].
    Grids (reading R2): per-channel (group == 0) fitted once on the initial
    rows; with groups, fitted on the current values when the group's first
    column is reached (group must divide block, so those values are current).
    Dead columns (reading R6) are zeroed first.  Natural column order (R11).

    force_codes / force_zeros: another implementation's decisions.  Where
    ours differ and the pre-rounding value lies within excuse_tol (grid-step
    units) of a rounding boundary, theirs are adopted so one excused flip does
    not cascade; all other disagreements are recorded in ``mismatches``.
    snapshot_cols: record the true current W (pending lazy updates applied)
    right after each listed column has been processed.
    """
    W = np.array(W, dtype=np.float64, copy=True)
    Uc = np.asarray(Uc, dtype=np.float64)
    d_out, d_in = W.shape
    bits = int(bits)
    nl = 2 ** bits - 1
    if group and block % group:
        raise ValueError("group must divide block")
    if dead is not None:
        W[:, np.asarray(dead, dtype=bool)] = 0.0
    n_groups = 1 if not group else -(-d_in // group)
    scales = np.zeros((d_out, n_groups), dtype=np.float32)
    zeros = np.zeros((d_out, n_groups), dtype=np.float32)
    codes = np.zeros((d_out, d_in), dtype=np.uint8)
    W_hat = np.zeros((d_out, d_in), dtype=np.float64)
    V = np.zeros((d_out, d_in), dtype=np.float64)
    res = QuantResult(codes, scales, zeros, W_hat, V)
    snap = set(int(c) for c in snapshot_cols)

    if not group:
        scales[:, 0], zeros[:, 0] = fit_grid(W.min(axis=1), W.max(axis=1), bits)

    for i in range(0, d_in, block):
        e_ = min(i + block, d_in)
        E = np.zeros((d_out, e_ - i), dtype=np.float64)
        for j in range(i, e_):
            g = 0 if not group else j // group
            if group and j % group == 0:
                seg = W[:, j:min(j + group, d_in)]
                xmin = seg.min(axis=1).astype(np.float32)
                xmax = seg.max(axis=1).astype(np.float32)
                sc, zr = fit_grid(xmin, xmax, bits)
                if force_zeros is not None:
                    theirs = np.asarray(force_zeros, dtype=np.float32)[:, g]
                    with np.errstate(divide="ignore", invalid="ignore"):
                        zv = np.where(sc > 0, -xmin.astype(np.float64) / sc.astype(np.float64),
                                      -xmin.astype(np.float64))
                    ok = (zr != theirs) & (np.abs(zv - (np.floor(zv) + 0.5)) <= excuse_tol) \
                        & ((theirs == np.floor(zv)) | (theirs == np.floor(zv) + 1))
                    zr = np.where(ok, theirs, zr).astype(np.float32)
                    res.zero_excused += int(ok.sum())
                    for r in np.flatnonzero((zr != theirs) & ~ok):
                        res.zero_mismatches.append((int(r), int(g), float(zv[r]), float(zr[r]),
                                                    float(theirs[r])))
                scales[:, g], zeros[:, g] = sc, zr
            sc = scales[:, g].astype(np.float64)
            zr = zeros[:, g].astype(np.float64)
            v = W[:, j] / sc + zr
            q = np.clip(np.rint(v), 0, nl)
            if force_codes is not None:
                theirs = np.asarray(force_codes)[:, j].astype(np.float64)
                ok = _excuse(q, theirs, v, bits, excuse_tol)
                q = np.where(ok, theirs, q)
                res.excused += int(ok.sum())
                for r in np.flatnonzero(q != theirs):
                    res.mismatches.append((int(r), int(j), float(v[r]), int(q[r]), int(theirs[r])))
            w_hat = sc * (q - zr)
            e = (W[:, j] - w_hat) / Uc[j, j]
            W[:, j + 1:e_] -= np.outer(e, Uc[j, j + 1:e_])
            E[:, j - i] = e
            codes[:, j] = q.astype(np.uint8)
            W_hat[:, j] = w_hat
            V[:, j] = v
            if j in snap:
                cur = W.copy()
                cur[:, e_:] -= E[:, :j - i + 1] @ Uc[i:j + 1, e_:]
                res.snapshots[j] = cur
        W[:, e_:] -= E @ Uc[i:e_, e_:]
    return res


# ---------------------------------------------------------------------------
# a10. Kronecker loss  ([REV] Background; [HZ] Appendix A.1 trace form)
# ---------------------------------------------------------------------------

def kron_loss(W, W_hat, H_X, H_G=None):
    """L = tr(dW H_X dW^T H_G) with dW = W - W_hat (H_G None means identity).

    [REV] Background: H ~ H_X kron H_G; [HZ] Appendix A.1: a Kronecker-weighted
    norm equals a trace of this form.  Reading R5: the undamped H's are used.
    """
    D = np.asarray(W, dtype=np.float64) - np.asarray(W_hat, dtype=np.float64)
    A = (D @ np.asarray(H_X, dtype=np.float64)) @ D.T
    if H_G is None:
        return float(np.trace(A))
    return float(np.trace(A @ np.asarray(H_G, dtype=np.float64)))


def gptq_loss(W, W_hat, H_X):
    """The H_X-only objective tr(dW H_X dW^T) (the H_G = I special case)."""
    return kron_loss(W, W_hat, H_X, None)


# ---------------------------------------------------------------------------
# a11. Sublayer bit allocation from the trace sensitivity  (reading R4)
# ---------------------------------------------------------------------------

def budget_units(n_params, avg_bits, lowest):
    """Integer budget floor(sum(n) * (avg - lowest)) in bit*parameter units.

    A relative 1e-12 is added before the floor so that a decimal average such
    as 2.4, which float64 cannot hold exactly, does not lose a unit.
    """
    total = float(np.sum(np.asarray(n_params, dtype=np.int64)))
    return int(math.floor(total * (float(avg_bits) - lowest) * (1.0 + 1e-12)))


def allocate_bits(sens, n_params, choices=(2, 3, 4), avg_bits=3.0):
    """Greedy "upgrade ordering" driven by the sensitivity score.

    [REV] Method (2) and Comparison (Table 6 ablation): sublayers are upgraded
    in the order of their score.  Reading R4: every sublayer starts at the
    lowest choice; the budget is sum(n_params) * (avg_bits - lowest) (an
    integer, see budget_units); sublayers
    are visited by descending score (ties: lower index first) and each takes
    the highest choice whose extra cost n_params * (b - lowest) still fits.
    """
    s = np.asarray(sens, dtype=np.float64)
    n = np.asarray(n_params, dtype=np.int64)
    ch = sorted(int(c) for c in choices)
    lo = ch[0]
    bits = np.full(s.shape[0], lo, dtype=np.int64)
    budget = budget_units(n, avg_bits, lo)
    order = sorted(range(s.shape[0]), key=lambda k: (-s[k], k))
    for k in order:
        for c in reversed(ch):
            cost = int(n[k]) * (c - lo)
            if c > lo and cost <= budget:
                bits[k] = c
                budget -= cost
                break
    return bits


# ---------------------------------------------------------------------------
# Whole layer, composed in the method's order
# ---------------------------------------------------------------------------

def quantize_linear(W, X, G, T_in, T_out, bits, group=0, block=128, damp_frac=0.01):
    """Covariances -> sensitivity -> BiIP -> damped Cholesky of the inverse ->
    blocked OBS -> Kronecker loss, all in float64 from the same inputs.

    Pinned as a whole (tests/test_oracle_linear_pins.py) by quantities formed
    by other routes: the loss against the sample double sum
    (1/N^2) sum_{t,s} (g_t^T dW x_s)^2 with dW = W - V^T W_hat' U in original
    coordinates, the factor against the residual of the rotated covariance
    formed by loops, the rotated weights by function preservation, and a
    dead-column case."""
    H_X = covariance(X)
    H_G = covariance(G)
    sens = sensitivity(H_X, H_G)
    Wp, HXp, HGp = biip(W, H_X, H_G, T_in, T_out)
    Uc, dead, lam = chol_inv(HXp, damp_frac)
    q = quantize_layer(Wp, Uc, bits, group, block, dead)
    return {
        "H_X": H_X, "H_G": H_G, "sens": sens, "Wp": Wp, "H_Xp": HXp, "H_Gp": HGp,
        "Uc": Uc, "dead": dead, "lam": lam, "quant": q,
        "loss": kron_loss(Wp, q.W_hat, HXp, HGp), "loss_gptq": gptq_loss(Wp, q.W_hat, HXp),
    }


# ---------------------------------------------------------------------------
# Inference side: packed codes and the online reversion of U and V
# ---------------------------------------------------------------------------

def pack_codes(codes, bits):
    """The codes of a [rows, cols] layer packed `bits` bits each into uint32.

    [REV] Limitations (third limitation): inference runs from the low-bit
    weights and reverts the orthogonal transforms online; the pages give no
    storage format.  Reading R15: each row is padded with zero codes to a
    multiple of 32; the 32 codes of group g of a row fill `bits` consecutive
    32-bit words (row r, words g*bits .. g*bits + bits - 1), code k of the
    group at bits bits*k .. bits*k + bits - 1 of the group's little-endian
    bit stream (word w of the group holds stream bits 32w .. 32w + 31).
    Returns uint32 [rows, ceil(cols / 32) * bits].
    """
    codes = np.asarray(codes)
    if codes.ndim != 2:
        raise ValueError("codes must be [rows, cols]")
    bits = int(bits)
    if not 1 <= bits <= 8:
        raise ValueError("bits must be 1..8")
    if codes.size and (codes.min() < 0 or codes.max() >= (1 << bits)):
        raise ValueError("a code does not fit in the bit-width")
    rows, cols = codes.shape
    groups = -(-cols // 32)
    out = np.zeros((rows, groups * bits), dtype=np.uint32)
    c = np.arange(cols)
    r = np.arange(rows)[:, None]
    q = codes.astype(np.uint32)
    for t in range(bits):                      # bit t of every code
        pos = bits * (c % 32) + t              # its place in the group's stream
        word = (c // 32) * bits + pos // 32
        one = ((q >> np.uint32(t)) & np.uint32(1)) << (pos % 32).astype(np.uint32)
        np.bitwise_or.at(out, (np.broadcast_to(r, q.shape), np.broadcast_to(word, q.shape)), one)
    return out


def unpack_codes(packed, bits, cols):
    """Inverse of pack_codes: uint8 codes [rows, cols] (the padding dropped)."""
    packed = np.asarray(packed, dtype=np.uint32)
    bits = int(bits)
    rows = packed.shape[0]
    if packed.shape[1] != -(-cols // 32) * bits:
        raise ValueError("packed width does not match cols and bits")
    c = np.arange(cols)
    codes = np.zeros((rows, cols), dtype=np.uint32)
    for t in range(bits):
        pos = bits * (c % 32) + t
        word = (c // 32) * bits + pos // 32
        bit = (packed[:, word] >> (pos % 32).astype(np.uint32)) & np.uint32(1)
        codes |= bit << np.uint32(t)
    return codes.astype(np.uint8)


def dequantize_layer(codes, scales, zeros, group=0):
    """W_hat[r, c] = scale[r, g] * (code[r, c] - zero[r, g]), g = 0 per channel
    or c // group for grouped grids (the solver's grid layout)."""
    codes = np.asarray(codes, dtype=np.float64)
    scales = np.asarray(scales, dtype=np.float64)
    zeros = np.asarray(zeros, dtype=np.float64)
    rows, cols = codes.shape
    g = np.zeros(cols, dtype=np.int64) if not group else np.arange(cols) // int(group)
    return scales.reshape(rows, -1)[:, g] * (codes - zeros.reshape(rows, -1)[:, g])


def reverted_apply(packed, scales, zeros, bits, group, T_in, T_out, x):
    """y = V^T (W_hat' (U x)) for x [d_in] or [d_in, B]: the quantized layer in
    the rotated basis applied between the forward input rotation U = T_in and
    the reverted output rotation V^T = T_out^T.

    [REV] Method (1): W' = V W U^T, so V^T W' U = W and the layer keeps its
    function; Limitations (third limitation): at inference U and V are
    reverted online, Theta(d_in log d_in + d_out log d_out) per layer with the
    fast transform (applied here as dense float64 matrices).
    """
    T_in = np.asarray(T_in, dtype=np.float64)
    T_out = np.asarray(T_out, dtype=np.float64)
    codes = unpack_codes(packed, bits, T_in.shape[0])
    W_hat = dequantize_layer(codes, scales, zeros, group)
    xr = T_in @ np.asarray(x, dtype=np.float64)
    return T_out.T @ (W_hat @ xr)


# ---------------------------------------------------------------------------
# Output side without the full d_out x d_out H_G (next-step row: blockwise and
# low-rank H_G), and an output rotation informed by H_G
# ---------------------------------------------------------------------------
# [REV] Limitations (second limitation): BiIP holds H_G as a full
# d_out x d_out matrix, a transient peak of memory; the research thread's
# "Sparks" list asks how much of the output-side flattening survives low-rank
# or blockwise approximations of H_G.  [ABS] Abstract (1): the output-side
# rotation extends the input-side one "using the gradient covariance".
# Readings taken here (listed with the others in the design notes):
#   * blockwise H_G: only its k x k diagonal blocks are kept (memory d_out k);
#     the output rotation is then block diagonal, the same randomised
#     Hadamard T_k in every block, so that V H_G V^T stays block diagonal and
#     is formed block by block;
#   * low-rank H_G: its best rank-r approximation (top r eigenpairs);
#   * the H_G-informed factor: a permutation P_G of the output channels from
#     diag(H_G) ahead of the Hadamard, V = T P_G.  Channels are ranked by
#     descending diag(H_G) (ties: lower index) and dealt round-robin to the
#     d_out / k blocks, so every block receives the same share of large and
#     small gradient energy before the Hadamard mixes within it.

def balance_permutation(diag_hg, k):
    """perm with new channel i = old channel perm[i]: the channel of rank q
    (descending diag(H_G), ties by lower index) goes to block q mod nb,
    position q div nb, nb = d / k blocks of k channels."""
    d = np.asarray(diag_hg).shape[0]
    k = int(k)
    if k < 1 or d % k:
        raise ValueError("k must divide the number of channels")
    nb = d // k
    order = sorted(range(d), key=lambda j: (-float(diag_hg[j]), j))
    perm = np.empty(d, dtype=np.int64)
    for q, old in enumerate(order):
        perm[(q % nb) * k + q // nb] = old
    return perm


def permutation_matrix(perm):
    """P with (P x)[i] = x[perm[i]]."""
    d = len(perm)
    P = np.zeros((d, d))
    P[np.arange(d), np.asarray(perm)] = 1.0
    return P


def hg_blockwise(H_G, k):
    """H_G with everything outside its k x k diagonal blocks set to zero."""
    H = np.asarray(H_G, dtype=np.float64)
    d = H.shape[0]
    if d % int(k):
        raise ValueError("k must divide d")
    out = np.zeros_like(H)
    for b in range(0, d, int(k)):
        out[b:b + k, b:b + k] = H[b:b + k, b:b + k]
    return out


def hg_lowrank(H_G, r):
    """Best rank-r approximation of the symmetric H_G: sum of its r largest
    eigenpairs lambda_i q_i q_i^T (library eigensolver as one step)."""
    H = np.asarray(H_G, dtype=np.float64)
    w, Q = np.linalg.eigh(0.5 * (H + H.T))
    idx = np.argsort(w)[::-1][:int(r)]
    return (Q[:, idx] * w[idx][None, :]) @ Q[:, idx].T


def block_rht_matrix(n, k, log2_p, signs, Qm=None):
    """Block diagonal I_{n/k} kron T_k with T_k = rht_matrix(k, log2_p, signs, Qm)."""
    if n % k:
        raise ValueError("k must divide n")
    return np.kron(np.eye(n // k), rht_matrix(k, log2_p, signs, Qm))


def blockwise_kron_loss(W, W_hat, H_X, HG_blocks):
    """sum_b tr(dW_b H_X dW_b^T H_G,b) over the row blocks dW_b of dW = W - W_hat
    with the k x k blocks HG_blocks[b] (array [nb, k, k]): the Kronecker loss
    of the block-diagonal H_G they form."""
    D = np.asarray(W, dtype=np.float64) - np.asarray(W_hat, dtype=np.float64)
    Hb = np.asarray(HG_blocks, dtype=np.float64)
    nb, k, _ = Hb.shape
    s = 0.0
    for b in range(nb):
        Db = D[b * k:(b + 1) * k]
        s += float(np.trace(Db @ np.asarray(H_X, dtype=np.float64) @ Db.T @ Hb[b]))
    return s


def weight_cv(W, axis):
    """Coefficient of variation (std / mean) of the L2 norms of W's rows
    (axis 'out': one norm per output channel) or columns (axis 'in'): the
    flattening diagnostic of [REV] Method (1) (weight-magnitude variance
    across input and output dimensions)."""
    W = np.asarray(W, dtype=np.float64)
    norms = np.linalg.norm(W, axis=1 if axis == "out" else 0)
    return float(np.std(norms) / np.mean(norms))


# ---------------------------------------------------------------------------
# Act-order: columns quantized in descending order of the Hessian diagonal
# ---------------------------------------------------------------------------
# "A Unified Hessian-Guided Framework for Post-Training Quantization",
# block-LDL rounding section: like GPTQ, the blocks are sorted before the
# solve so that those with the larger Fisher traces are quantized first.  For
# the column-wise solver here a column's trace is its diagonal entry of
# H_X'.  Reading: ties go to the lower index; the solve runs on the permuted
# W and H, and its dequantized weights and codes are returned in the original
# column order; a grouped grid then covers consecutive columns of the
# quantization order (group g = original columns perm[g*group:(g+1)*group]).

def act_order_permutation(H):
    """perm[q] = the column of rank q by descending H[j, j] (ties: lower j)."""
    d = np.asarray(H).diagonal()
    return np.array(sorted(range(len(d)), key=lambda j: (-float(d[j]), j)), dtype=np.int64)


def quantize_layer_act_order(W, H, bits, group=0, block=128, damp_frac=0.01):
    """Blocked OBS in act-order: permute W's columns and H's rows and columns
    by act_order_permutation(H), take the damped Cholesky factor of the
    permuted H, solve, and scatter codes and W_hat back to the original
    column order.  Returns (QuantResult in the original order with the
    solver's grid arrays, perm, Uc of the permuted H)."""
    W = np.asarray(W, dtype=np.float64)
    H = np.asarray(H, dtype=np.float64)
    perm = act_order_permutation(H)
    Hp = H[np.ix_(perm, perm)]
    Uc, dead, _ = chol_inv(Hp, damp_frac)
    q = quantize_layer(W[:, perm], Uc, bits, group, block, dead)
    codes = np.empty_like(q.codes)
    W_hat = np.empty_like(q.W_hat)
    V = np.empty_like(q.V)
    codes[:, perm] = q.codes
    W_hat[:, perm] = q.W_hat
    V[:, perm] = q.V
    return QuantResult(codes, q.scales, q.zeros, W_hat, V), perm, Uc
