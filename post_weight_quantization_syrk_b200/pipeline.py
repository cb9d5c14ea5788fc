"""One linear layer through the whole KronQ path, driven through the C ABI.

Order of the steps (KronQ paper page, Abstract; KronQ review, Method):
  H_X, H_G (covariance SYRKs) -> sensitivity -> BiIP rotations of W, H_X, H_G
  -> damped Cholesky factor of the inverse of H_X' (once per layer)
  -> for each bit-width: blocked OBS quantization + Kronecker loss.
H_G is computed once and reused across bit-widths, as the authors' reply on
the paper page describes.  All buffers are allocated once per layer shape
(torch provides device memory and the stream); every computation is a kq_*
call into libkronq.so.
"""
from __future__ import annotations

import dataclasses

import torch

from . import _lib as K


@dataclasses.dataclass
class BitResult:
    bits: int
    group: int
    codes: torch.Tensor
    scales: torch.Tensor
    zeros: torch.Tensor
    W_hat: torch.Tensor
    loss: torch.Tensor      # fp64[1] device
    # act-order: the solve's outputs in quantization order, and that order
    # (codes and W_hat above are in the original column order; a grouped
    # grid's group g covers original columns perm[g * group:(g + 1) * group])
    codes_q: torch.Tensor = None
    W_hat_q: torch.Tensor = None
    perm: torch.Tensor = None


class LayerQuantizer:
    """Device buffers for one (d_out, d_in) layer and the calls that fill them."""

    def __init__(self, d_out, d_in, device="cuda", block=128, gemm_mode=K.KQ_GEMM_FP32, full_hg=True,
                 act_order=False):
        self.d_out, self.d_in, self.block, self.gemm_mode = d_out, d_in, block, gemm_mode
        self.act_order = act_order
        dev = torch.device(device)
        self.device = dev
        f32 = dict(dtype=torch.float32, device=dev)
        self.H_X = torch.empty((d_in, d_in), **f32)
        self.H_G = torch.empty((d_out, d_out), **f32) if full_hg else None
        self.perm = None
        self.Wp = torch.empty((d_out, d_in), **f32)
        self.Uc = torch.empty((d_in, d_in), **f32)
        self.dead = torch.zeros(d_in, dtype=torch.uint8, device=dev)
        self.sens = torch.zeros(3, dtype=torch.float64, device=dev)
        self.info = K.new_info(dev)
        self._ws = K.workspace(256, dev)
        self._ws_bytes = 256
        if act_order:
            # the solve's column order (descending diag H_X'), its inverse, and
            # W' and H_X' permuted into it
            self.perm_in = torch.empty(d_in, dtype=torch.int64, device=dev)
            self.inv_in = torch.empty(d_in, dtype=torch.int64, device=dev)
            self.Hq = torch.empty((d_in, d_in), **f32)
            self.Wq = torch.empty((d_out, d_in), **f32)

    def workspace(self, nbytes):
        """One scratch buffer shared by the calls (they run in stream order)."""
        if nbytes > self._ws_bytes:
            self._ws = K.workspace(nbytes, self.device)
            self._ws_bytes = nbytes
        return self._ws

    def alloc_result(self, bits, group, solve_out=None):
        """Buffers of one setting; `solve_out` (d_out x d_in fp32), if given,
        becomes the buffer the solve writes W_hat into."""
        ng = 1 if not group else -(-self.d_in // group)
        dev = self.device
        q = self.act_order
        r = BitResult(bits, group,
                      torch.empty((self.d_out, self.d_in), dtype=torch.uint8, device=dev),
                      torch.empty((self.d_out, ng), dtype=torch.float32, device=dev),
                      torch.empty((self.d_out, ng), dtype=torch.float32, device=dev),
                      solve_out if solve_out is not None and not q else
                      torch.empty((self.d_out, self.d_in), dtype=torch.float32, device=dev),
                      torch.zeros(1, dtype=torch.float64, device=dev))
        if q:
            r.codes_q = torch.empty_like(r.codes)
            r.W_hat_q = solve_out if solve_out is not None else torch.empty_like(r.W_hat)
            r.perm = self.perm_in
        return r

    def alloc_results(self, settings):
        """Buffers of several settings, the W_hat the solve writes stacked in
        one [count, d_out, d_in] tensor: kq_quantize_layer_multi then solves
        the settings as one problem (their rows are independent chains that
        share U_c)."""
        stack = torch.empty((len(settings), self.d_out, self.d_in), dtype=torch.float32, device=self.device)
        return [self.alloc_result(b, g, stack[i]) for i, (b, g) in enumerate(settings)]

    # -- steps -----------------------------------------------------------
    def statistics(self, X, G, n_total=None, accumulate=False, stream=None):
        """H_X (+)= X^T X / N, H_G (+)= G^T G / N; sensitivity of the result."""
        n_total = X.shape[0] if n_total is None else n_total
        alpha = 1.0 / n_total if n_total else 0.0
        ws = self.workspace(max(K.kq_accum_cov_workspace_size(X.shape[0], self.d_in),
                                K.kq_accum_cov_workspace_size(G.shape[0], self.d_out)))
        K.kq_accum_cov(X, self.H_X, alpha, accumulate, ws, self.info, stream)
        K.kq_accum_cov(G, self.H_G, alpha, accumulate, ws, self.info, stream)

    def sensitivity(self, stream=None):
        K.kq_sensitivity(self.H_X, self.H_G, self.sens, stream)

    def hg_permutation(self, G, k, n_total=None, stream=None):
        """The H_G-informed factor P_G of the output rotation V = T P_G:
        output channels ranked by descending gradient energy diag(H_G)
        (ties: lower index) and dealt round-robin to d_out / k blocks
        (kq_channel_energy, kq_balance_permutation).  rotate() then applies
        P_G before T."""
        n_total = G.shape[0] if n_total is None else n_total
        energy = torch.empty(self.d_out, dtype=torch.float32, device=self.device)
        K.kq_channel_energy(G, energy, 1.0 / n_total, None, self.info, stream)
        self.perm = torch.empty(self.d_out, dtype=torch.int64, device=self.device)
        K.kq_balance_permutation(energy, k, self.perm, stream)

    def rotate(self, W, T_in: K.RHT, T_out: K.RHT, stream=None):
        """W' = V W U^T, H_X' = U H_X U^T, H_G' = V H_G V^T (in the layer's
        buffers), V = T_out, or T_out P_G after hg_permutation()."""
        if self.perm is not None:
            K.kq_gather(W, self.Wp, self.perm, None, self.info, stream)
            tmp = torch.empty_like(self.H_G)
            K.kq_gather(self.H_G, tmp, self.perm, self.perm, self.info, stream)
            self.H_G.copy_(tmp)
            del tmp
        else:
            self.Wp.copy_(W)
        K.kq_rotate(self.Wp, K.KQ_AXIS_COLS, T_in, False, stream)
        K.kq_rotate(self.Wp, K.KQ_AXIS_ROWS, T_out, False, stream)
        K.kq_rotate(self.H_X, K.KQ_AXIS_COLS, T_in, False, stream)
        K.kq_rotate(self.H_X, K.KQ_AXIS_ROWS, T_in, False, stream)
        K.kq_rotate(self.H_G, K.KQ_AXIS_COLS, T_out, False, stream)
        K.kq_rotate(self.H_G, K.KQ_AXIS_ROWS, T_out, False, stream)

    def factor(self, damp_frac=0.01, stream=None):
        """Damped Cholesky factor of the inverse of H_X' (of the act-order
        permuted H_X' when act_order; dead flags then in that order)."""
        ws = self.workspace(K.kq_chol_inv_workspace_size(self.d_in))
        H = self.H_X
        if self.act_order:
            K.kq_act_order_permutation(self.H_X, self.perm_in, stream)
            K.kq_gather(self.H_X, self.Hq, self.perm_in, self.perm_in, self.info, stream)
            # inverse permutation (index bookkeeping): inv[perm[i]] = i
            self.inv_in.scatter_(0, self.perm_in, torch.arange(self.d_in, dtype=torch.int64, device=self.device))
            H = self.Hq
        K.kq_chol_inv(H, damp_frac, self.Uc, self.dead, ws, self.info, stream)

    def _solve_input(self, stream=None):
        """W' as the solver sees it: in act-order, its columns permuted."""
        if not self.act_order:
            return self.Wp
        K.kq_gather(self.Wp, self.Wq, None, self.perm_in, self.info, stream)
        return self.Wq

    def _unpermute(self, r: BitResult, stream=None):
        if self.act_order:
            K.kq_gather(r.codes_q, r.codes, None, self.inv_in, self.info, stream)
            K.kq_gather(r.W_hat_q, r.W_hat, None, self.inv_in, self.info, stream)

    def quantize(self, res: BitResult, stream=None):
        ws = self.workspace(K.kq_quantize_layer_workspace_size(self.d_out, self.d_in, self.block))
        Win = self._solve_input(stream)
        codes, W_hat = (res.codes_q, res.W_hat_q) if self.act_order else (res.codes, res.W_hat)
        K.kq_quantize_layer(Win, self.Uc, self.dead, res.bits, res.group, codes, res.scales, res.zeros,
                            W_hat, self.block, self.gemm_mode, ws, self.info, stream)
        self._unpermute(res, stream)

    def loss(self, res: BitResult, stream=None):
        ws = self.workspace(K.kq_kron_loss_workspace_size(self.d_out, self.d_in))
        K.kq_kron_loss(self.Wp, res.W_hat, self.H_X, self.H_G, res.loss, ws, stream)

    def quantize_all(self, results, stream=None):
        """Every setting of `results` in one call: the factor's operand split is
        shared, and up to four settings are solved as one stacked problem
        (results from alloc_results) or else side by side."""
        ws = self.workspace(K.kq_quantize_layer_multi_workspace_size(self.d_out, self.d_in, self.block, len(results)))
        Win = self._solve_input(stream)
        q = self.act_order
        K.kq_quantize_layer_multi(Win, self.Uc, self.dead, [(r.bits, r.group) for r in results],
                                  [r.codes_q if q else r.codes for r in results], [r.scales for r in results],
                                  [r.zeros for r in results], [r.W_hat_q if q else r.W_hat for r in results],
                                  self.block, self.gemm_mode, ws, self.info, stream)
        for r in results:
            self._unpermute(r, stream)

    def loss_all(self, results, stream=None):
        """Every result's Kronecker loss in one call (the split of the smaller Hessian is shared)."""
        ws = self.workspace(K.kq_kron_loss_workspace_size(self.d_out, self.d_in))
        K.kq_kron_loss_multi(self.Wp, [r.W_hat for r in results], self.H_X, self.H_G, [r.loss for r in results], ws,
                             stream)

    def run(self, W, X, G, T_in, T_out, settings, damp_frac=0.01, results=None, stream=None):
        """The whole path; settings = [(bits, group), ...].  Asynchronous."""
        self.statistics(X, G, stream=stream)
        self.sensitivity(stream)
        self.rotate(W, T_in, T_out, stream)
        self.factor(damp_frac, stream)
        if results is None:
            results = self.alloc_results(settings)
        self.quantize_all(results, stream)
        self.loss_all(results, stream)
        return results

    def check(self, where="kronq"):
        K.check_info(self.info, where)


class BlockwiseLayerQuantizer(LayerQuantizer):
    """One layer whose output side never forms the full d_out x d_out H_G.

    KronQ review, Limitations (second limitation: BiIP holds the full H_G, a
    transient peak of memory) and the research thread's "Sparks" (blockwise
    H_G); KronQ paper page, Abstract (1) (the output rotation uses the
    gradient covariance).  Only the k x k diagonal blocks of H_G are formed
    (kq_accum_cov_blocks: d_out k floats), the output rotation is block
    diagonal, V = (I kron T_k) P_G, so that V H_G V^T stays block diagonal
    and is rotated block by block, and the loss is that of the block-diagonal
    H_G (kq_kron_loss_blocks).  With balanced=True, P_G is the permutation
    dealing output channels to blocks by descending gradient energy
    (kq_channel_energy, kq_balance_permutation): it needs a transient
    column-permuted copy of G (kq_gather); balanced=False takes P_G = I.
    The input side and the solver are those of LayerQuantizer.
    """

    def __init__(self, d_out, d_in, k, balanced=True, device="cuda", block=128, gemm_mode=K.KQ_GEMM_FP32):
        if d_out % k or k % 256:
            raise ValueError("k must be a multiple of 256 dividing d_out")
        self.k, self.balanced = k, balanced
        super().__init__(d_out, d_in, device, block, gemm_mode, full_hg=False)   # H_G never formed
        dev = self.device
        self.H_Gb = torch.empty((d_out, k), dtype=torch.float32, device=dev)
        self.energy = torch.empty(d_out, dtype=torch.float32, device=dev)
        self.perm = torch.arange(d_out, dtype=torch.int64, device=dev)

    def statistics(self, X, G, n_total=None, accumulate=False, stream=None):
        if accumulate:
            raise ValueError("the blockwise output side takes all calibration tokens in one call")
        n_total = X.shape[0] if n_total is None else n_total
        alpha = 1.0 / n_total if n_total else 0.0
        ws = self.workspace(max(K.kq_accum_cov_workspace_size(X.shape[0], self.d_in),
                                K.kq_accum_cov_blocks_workspace_size(G.shape[0], self.d_out, self.k)))
        K.kq_accum_cov(X, self.H_X, alpha, False, ws, self.info, stream)
        if self.balanced:
            K.kq_channel_energy(G, self.energy, alpha, None, self.info, stream)
            K.kq_balance_permutation(self.energy, self.k, self.perm, stream)
            Gp = torch.empty_like(G)                           # transient, the size of G
            K.kq_gather(G, Gp, None, self.perm, self.info, stream)
            K.kq_accum_cov_blocks(Gp, self.k, self.H_Gb, alpha, False, ws, self.info, stream)
            del Gp
        else:
            K.kq_accum_cov_blocks(G, self.k, self.H_Gb, alpha, False, ws, self.info, stream)

    def sensitivity(self, stream=None):
        K.kq_sensitivity_blocks(self.H_X, self.H_Gb, self.sens, stream)

    def rotate(self, W, T_in: K.RHT, T_k: K.RHT, stream=None):
        """W' = (I kron T_k) P_G W U^T, H_X' = U H_X U^T, each H_G block T_k B T_k^T."""
        k = self.k
        if self.balanced:
            K.kq_gather(W, self.Wp, self.perm, None, self.info, stream)
        else:
            self.Wp.copy_(W)
        K.kq_rotate(self.Wp, K.KQ_AXIS_COLS, T_in, False, stream)
        for b in range(self.d_out // k):
            K.kq_rotate(self.Wp[b * k:(b + 1) * k], K.KQ_AXIS_ROWS, T_k, False, stream)
        K.kq_rotate(self.H_X, K.KQ_AXIS_COLS, T_in, False, stream)
        K.kq_rotate(self.H_X, K.KQ_AXIS_ROWS, T_in, False, stream)
        for b in range(self.d_out // k):
            Hb = self.H_Gb[b * k:(b + 1) * k]
            K.kq_rotate(Hb, K.KQ_AXIS_COLS, T_k, False, stream)
            K.kq_rotate(Hb, K.KQ_AXIS_ROWS, T_k, False, stream)

    def loss(self, res: BitResult, stream=None):
        ws = self.workspace(K.kq_kron_loss_blocks_workspace_size(self.d_out, self.d_in, self.k))
        K.kq_kron_loss_blocks(self.Wp, res.W_hat, self.H_X, self.H_Gb, res.loss, ws, stream)

    def loss_all(self, results, stream=None):
        for r in results:
            self.loss(r, stream)

    def unrotate_output(self, M, T_k: K.RHT, out, stream=None):
        """out = P_G^T (I kron T_k)^T M for M [d_out, cols] (M is overwritten):
        takes rotated output rows back to the original channel order."""
        k = self.k
        for b in range(self.d_out // k):
            K.kq_rotate(M[b * k:(b + 1) * k], K.KQ_AXIS_ROWS, T_k, True, stream)
        if self.balanced:
            inv = torch.empty_like(self.perm)
            inv.scatter_(0, self.perm, torch.arange(self.d_out, dtype=torch.int64, device=self.device))
            K.kq_gather(M, out, inv, None, self.info, stream)
        else:
            out.copy_(M)


def quantize_from_host(lq: LayerQuantizer, host_layers, T_in, T_out, settings, results, host_outputs,
                       damp_frac=0.01):
    """Run the whole path over a sequence of layers of one shape whose inputs
    live in pinned host memory, overlapping transfers with compute.

    host_layers[i] = (W, X, G) pinned CPU tensors; host_outputs[i][k] =
    (codes, scales, zeros, loss) pinned CPU tensors for settings[k].  Layer
    i+1's inputs are copied host->device on a separate stream into the other
    of two device buffer sets while layer i is quantized on the current
    stream; layer i's results are copied back on the current stream right
    after it (device->host, the other PCIe direction).  A buffer set is
    refilled only after the layer that used it has finished.  Asynchronous:
    the caller synchronises the current stream before reading host_outputs.
    """
    dev = lq.device
    comp = torch.cuda.current_stream(dev)
    copy = torch.cuda.Stream(device=dev)
    first = host_layers[0]
    bufs = [tuple(torch.empty(t.shape, dtype=t.dtype, device=dev) for t in first) for _ in range(2)]
    copied = [torch.cuda.Event() for _ in range(2)]
    freed = [torch.cuda.Event() for _ in range(2)]
    start = torch.cuda.Event()
    start.record(comp)
    copy.wait_event(start)

    def issue_copy(i):
        slot = i % 2
        with torch.cuda.stream(copy):
            if i >= 2:
                copy.wait_event(freed[slot])
            for d, h in zip(bufs[slot], host_layers[i]):
                d.copy_(h, non_blocking=True)
            copied[slot].record(copy)

    issue_copy(0)
    for i in range(len(host_layers)):
        if i + 1 < len(host_layers):
            issue_copy(i + 1)
        slot = i % 2
        comp.wait_event(copied[slot])
        W, X, G = bufs[slot]
        lq.run(W, X, G, T_in, T_out, settings, damp_frac=damp_frac, results=results)
        freed[slot].record(comp)
        for r, o in zip(results, host_outputs[i]):
            o[0].copy_(r.codes, non_blocking=True)
            o[1].copy_(r.scales, non_blocking=True)
            o[2].copy_(r.zeros, non_blocking=True)
            o[3].copy_(r.loss, non_blocking=True)
    # the device buffers were last used on `comp`; keep them alive until then
    for b in bufs:
        for t in b:
            t.record_stream(comp)
    return results
