/*
 * kronq.h - C ABI of the KronQ per-linear-layer quantization path on B200.
 *
 * The path (one linear layer y = W x, W [d_out, d_in] row-major):
 *   1. H_X = X^T X / N and H_G = G^T G / N from bf16 calibration activations
 *      X [N, d_in] and output gradients G [N, d_out]        -> kq_accum_cov
 *   2. sensitivity tr(H_X), tr(H_G), tr(H_G) tr(H_X)          -> kq_sensitivity
 *   3. bidirectional incoherence processing: W' = V W U^T,
 *      H_X' = U H_X U^T, H_G' = V H_G V^T with randomised
 *      Hadamard rotations U (input side) and V (output side) -> kq_rotate
 *   4. damping, dead columns and the upper Cholesky factor of
 *      the damped inverse of H_X'                            -> kq_chol_inv
 *   5. blocked column-wise OBS (GPTQ) quantization of W' on a
 *      b-bit asymmetric grid                                  -> kq_quantize_layer
 *   6. Kronecker loss tr(dW H_X' dW^T H_G')                   -> kq_kron_loss
 *   7. sublayer bit allocation from the sensitivities (host)  -> kq_allocate_bits
 *
 * Sources (page title and section):
 *   - KronQ paper page (Hugging Face papers 2607.07964), Abstract: H ~ H_X kron
 *     H_G; bidirectional incoherence processing; trace sensitivity for
 *     mixed precision.  Authors' reply (Community thread): H_G from one
 *     backward pass, reused across bit-widths.
 *   - Paper review "KronQ: LLM Quantization via Kronecker-Factored Hessian"
 *     (romaanj.github.io/reviews/kronq), sections Background, Prior
 *     limitations, Goal, Method, Comparison, Limitations.
 *   - "A Unified Hessian-Guided Framework for Post-Training Quantization"
 *     (hub.valency.io/works/W_r72x54u6), Background (grid step and shift;
 *     transformations), Appendix A.1 (trace form of the Kronecker norm).
 *
 * Conventions for every entry point:
 *   - Matrices are row-major with an explicit leading dimension (elements).
 *   - Every pointer is CALLER-OWNED DEVICE memory unless stated otherwise;
 *     the library allocates and frees nothing.  Scratch memory is sized by the
 *     matching kq_*_workspace_size() and passed in as (ws, ws_bytes); ws must
 *     be 256-byte aligned.
 *   - Work is enqueued on `stream` (NULL = legacy default stream) and the
 *     call returns without synchronising.  Host-side validation errors are
 *     returned synchronously and nothing is enqueued.
 *   - Device-detected errors are written to `info`, a caller-owned device
 *     int32 that the library never clears: the first error sticks (code in
 *     bits 24..31, an index in bits 0..23, see KQ_INFO_*).  Zero it before a
 *     chain of calls and read it after the stream has synchronised.
 *   - Every device wait is bounded; on expiry the kernel records
 *     KQ_ERR_TIMEOUT in `info` and returns.
 *   - The library is stateless apart from a thread-local last-error string
 *     and is safe to call from several host threads.  No C++ exception
 *     crosses this ABI.
 */
#ifndef KRONQ_H
#define KRONQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* The same handle type as cudaStream_t. */
typedef struct CUstream_st* kq_stream_t;

typedef enum kq_status {
  KQ_OK = 0,
  KQ_ERR_INVALID_ARG = 1,       /* NULL pointer, negative size, bad enum value        */
  KQ_ERR_UNSUPPORTED_SHAPE = 2, /* a size outside the limits stated per call          */
  KQ_ERR_ALIGNMENT = 3,         /* pointer or leading dimension misaligned            */
  KQ_ERR_WORKSPACE = 4,         /* ws too small or misaligned                          */
  KQ_ERR_CUDA = 5,              /* a CUDA runtime call failed (see kq_last_error)     */
  KQ_ERR_NOT_PD = 6,            /* device: damped matrix not positive definite        */
  KQ_ERR_NONFINITE = 7,         /* device: NaN or Inf met in an input                  */
  KQ_ERR_TIMEOUT = 8            /* device: a bounded wait expired                      */
} kq_status;

#define KQ_INFO_CODE(info) ((int32_t)(((uint32_t)(info)) >> 24))
#define KQ_INFO_INDEX(info) ((int32_t)((info) & 0xFFFFFF))

enum { KQ_AXIS_ROWS = 0, KQ_AXIS_COLS = 1 };
enum { KQ_GEMM_FP32 = 0, KQ_GEMM_3XTF32 = 1 };

/* Human-readable name of a status code (static string). */
const char* kq_status_string(kq_status s);
/* Detail of the last non-OK status returned on this host thread ("" if none). */
const char* kq_last_error(void);
/* Library version, major * 10000 + minor * 100 + patch. */
int kq_version(void);
/* Number of CUDA kernel launches this library has enqueued in this process
 * (all host threads); a diagnostic for counting device work per step. */
unsigned long long kq_launch_count(void);

/* Time limit of the device waits in the tensor-core kernels (kq_accum_cov,
 * and the products inside kq_quantize_layer and kq_kron_loss): a pipeline
 * wait that has not completed after `ns` nanoseconds gives up, the kernel
 * records KQ_ERR_TIMEOUT in `info` (index = the wait's site), lets its own
 * copies and products finish (with the fixed default bound), frees its
 * tensor memory and returns.  ns == 0 makes a wait give up at the first poll
 * that finds it incomplete: a test of this failure path, whose results are
 * then garbage.  Process-wide, read by each call when it enqueues; returns
 * the previous limit.  Default KQ_WAIT_LIMIT_DEFAULT_NS (4 s). */
#define KQ_WAIT_LIMIT_DEFAULT_NS 4000000000ull
unsigned long long kq_set_wait_limit_ns(unsigned long long ns);

/* --------------------------------------------------------------------------
 * kq_accum_cov - covariance accumulation (steps a1/a2).
 *
 * Computes C = alpha * A^T A (accumulate == 0) or C += alpha * A^T A
 * (accumulate != 0), the input-activation covariance H_X = E[x x^T] or the
 * output-gradient covariance H_G = E[g g^T] (KronQ review, Background: the
 * Kronecker factors of the layer Hessian; research thread: H_G = E[g g^T]).
 * Pass alpha = 1 / N_total to obtain the mean over all calls' tokens.
 *
 *   A      bf16 bit patterns, [n, d] row-major (tokens x channels), lda >= d;
 *          lda % 8 == 0 and A 16-byte aligned (TMA requirements); may be
 *          NULL when n == 0.
 *   n      number of tokens, >= 0 (n == 0 leaves C = 0 or unchanged).
 *   d      channels, 1 <= d <= 65536.
 *   C      fp32 [d, d] row-major, ldc >= d; the full symmetric matrix is
 *          written (lower triangle computed and mirrored).
 *   ws     workspace of kq_accum_cov_workspace_size(n, d) bytes.
 *   info   device word; KQ_ERR_NONFINITE (index = row) if C gets NaN/Inf,
 *          KQ_ERR_TIMEOUT if a pipeline wait expired.
 * Tensor cores: bf16 x bf16 products accumulated in fp32.
 * ------------------------------------------------------------------------ */
size_t kq_accum_cov_workspace_size(int64_t n, int64_t d);
kq_status kq_accum_cov(const uint16_t* A, int64_t n, int64_t d, int64_t lda,
                       float* C, int64_t ldc, float alpha, int accumulate,
                       void* ws, size_t ws_bytes, int32_t* info, kq_stream_t stream);

/* kq_accum_cov_blocks - only the k x k diagonal blocks of the covariance.
 *
 * The blockwise approximation of H_G that keeps BiIP's memory at d k instead
 * of d^2 floats (KronQ review, Limitations, second limitation: the full
 * d_out x d_out H_G is a transient peak; research thread, "Sparks": blockwise
 * H_G).  Block b (rows and columns b k .. b k + k - 1 of alpha A^T A) is
 * written (or added, accumulate != 0) to rows b k .. of C, which is d x k
 * (ldc >= k): C[b k + i][j] = alpha sum_t A[t][b k + i] A[t][b k + j].
 * Same kernel and accuracy as kq_accum_cov; k a multiple of 256 dividing d.
 * Workspace: kq_accum_cov_blocks_workspace_size(n, d, k) bytes (0 when
 * the shape is unsupported). */
size_t kq_accum_cov_blocks_workspace_size(int64_t n, int64_t d, int64_t k);
kq_status kq_accum_cov_blocks(const uint16_t* A, int64_t n, int64_t d, int64_t lda, int64_t k, float* C,
                              int64_t ldc, float alpha, int accumulate, void* ws, size_t ws_bytes,
                              int32_t* info, kq_stream_t stream);

/* --------------------------------------------------------------------------
 * Output rotation informed by H_G: V = T P_G.
 *
 * KronQ paper page, Abstract (1): the output-side rotation extends the
 * input-side one "using the gradient covariance"; KronQ review, Limitations
 * (second limitation) and research thread ("Sparks"): blockwise H_G.  P_G
 * permutes the output channels: ranked by descending diag(H_G) (ties: lower
 * index), the channel of rank q goes to block q mod nb, slot q div nb, of the
 * nb = d / k blocks of a blockwise rotation, so that every block holds the
 * same share of large and small gradient energies.
 *
 * kq_channel_energy: out[j] = alpha sum_t A[t][j]^2 (the diagonal of
 *   alpha A^T A without forming it) for bf16 A [n, d] (lda >= d); fp64 sums
 *   over 64 token slices added in a fixed order; out fp32 [d] device.
 *   Workspace kq_channel_energy_workspace_size(d).  KQ_ERR_NONFINITE in info.
 * kq_balance_permutation: perm[(q % nb) k + q / nb] = channel of rank q by
 *   descending energy[j] (ties: lower j); energy fp32 [d], perm int64 [d],
 *   both device; k divides d, d <= 65536.
 * kq_gather: out[i][j] = M[row_idx[i]][col_idx[j]] (either index array may
 *   be NULL: the identity) for rows x cols matrices of 1-, 2- or 4-byte elements
 *   (ldm, ldo >= cols; out must not alias M); an index outside 0..rows-1 or
 *   0..cols-1 is skipped and reported as KQ_ERR_INVALID_ARG (index = row i).
 *   Row gather: P_G W (or P_G^T with the inverse permutation); both: P_G H
 *   P_G^T; columns of bf16 G: G P_G^T, whose covariance is P_G H_G P_G^T.
 * ------------------------------------------------------------------------ */
size_t kq_channel_energy_workspace_size(int64_t d);
kq_status kq_channel_energy(const uint16_t* A, int64_t n, int64_t d, int64_t lda, float alpha, float* out,
                            void* ws, size_t ws_bytes, int32_t* info, kq_stream_t stream);
kq_status kq_balance_permutation(const float* energy, int64_t d, int64_t k, int64_t* perm, kq_stream_t stream);
kq_status kq_gather(const void* M, int64_t ldm, int elem_bytes, const int64_t* row_idx, const int64_t* col_idx,
                    int64_t rows, int64_t cols, void* out, int64_t ldo, int32_t* info, kq_stream_t stream);

/* kq_act_order_permutation - the solver's column order by descending
 * Hessian diagonal ("A Unified Hessian-Guided Framework for Post-Training
 * Quantization", block-LDL rounding: like GPTQ, blocks with larger traces
 * are quantized first).  perm[q] = the column of rank q by descending
 * H[j][j], ties to the lower j; H fp32 [n, n] (ldh >= n), perm int64 [n],
 * both device.  The act-order solve is kq_gather of W's columns and of H's
 * rows and columns by perm, kq_chol_inv and kq_quantize_layer on those, and
 * kq_gather of W_hat and the codes back with the inverse permutation. */
kq_status kq_act_order_permutation(const float* H, int64_t n, int64_t ldh, int64_t* perm, kq_stream_t stream);

/* --------------------------------------------------------------------------
 * kq_sensitivity - trace sensitivity (step a3).
 *
 * out3[0] = tr(H_X), out3[1] = tr(H_G), out3[2] = tr(H_G) * tr(H_X), each
 * summed in fp64 (KronQ review, Method (2): the joint score tr(H_G) tr(H_X)
 * separates sublayers with identical inputs; tr(H_X) alone is the H_X-only
 * score of the Comparison section).
 *
 *   H_X  fp32 [d_in, d_in], ldhx >= d_in;  H_G fp32 [d_out, d_out], ldhg >= d_out.
 *   out3 device fp64[3].
 * ------------------------------------------------------------------------ */
kq_status kq_sensitivity(const float* H_X, int64_t d_in, int64_t ldhx,
                         const float* H_G, int64_t d_out, int64_t ldhg,
                         double* out3, kq_stream_t stream);
/* The same with H_G in the block-diagonal layout of kq_accum_cov_blocks
 * (d_out x k, block b in rows b k .., ldhgb >= k): tr(H_G) is the sum of
 * the blocks' traces. */
kq_status kq_sensitivity_blocks(const float* H_X, int64_t d_in, int64_t ldhx, const float* H_Gb,
                                int64_t d_out, int64_t k, int64_t ldhgb, double* out3, kq_stream_t stream);

/* --------------------------------------------------------------------------
 * kq_rotate - randomised Hadamard rotation (steps a4/a5, BiIP).
 *
 * T = (Q_m kron H_p / sqrt(p)) . diag(signs), n = m * p, p = 2^log2_p, with
 * H_p the Sylvester Walsh-Hadamard matrix (KronQ review, Method (1): the
 * input-side random rotation extended to the output side; Unified
 * Hessian-Guided PTQ, Background / Transformations: randomised Hadamard
 * transforms are orthogonal and preserve the layer output).  Element a*p + b
 * of a vector is (row a of Q_m, row b of H_p).
 *
 *   axis == KQ_AXIS_ROWS : M <- T . M    (T acts on the row index; T->n == rows)
 *   axis == KQ_AXIS_COLS : M <- M . T^T  (T acts on the column index; T->n == cols)
 *   inverse != 0 applies T^T instead of T.
 * In place on fp32 M [rows, cols], ld >= cols, 16-byte aligned, ld % 4 == 0.
 * Limits: 1 <= m <= 64, 0 <= log2_p <= 15, n <= 32768, and for
 * KQ_AXIS_ROWS also m * max(1, p / 128) <= 256; T->signs device
 * fp32[n] of +-1; T->Qm device fp32[m*m] row-major orthogonal, may be NULL
 * only when m == 1.  BiIP of a layer is:
 *   W:   kq_rotate(W,  KQ_AXIS_COLS, U) then kq_rotate(W, KQ_AXIS_ROWS, V)
 *   H_X: kq_rotate(HX, KQ_AXIS_COLS, U) then kq_rotate(HX, KQ_AXIS_ROWS, U)
 *   H_G: kq_rotate(HG, KQ_AXIS_COLS, V) then kq_rotate(HG, KQ_AXIS_ROWS, V)
 * ------------------------------------------------------------------------ */
typedef struct kq_rht {
  int64_t n;
  int32_t log2_p;
  int32_t m;
  const float* signs;
  const float* Qm;
} kq_rht;

kq_status kq_rotate(float* M, int64_t rows, int64_t cols, int64_t ld, int axis,
                    const kq_rht* T, int inverse, kq_stream_t stream);

/* --------------------------------------------------------------------------
 * kq_chol_inv - damping, dead columns and Cholesky factor of the inverse (a6).
 *
 * GPTQ solver set-up on H (KronQ review, Prior limitations: GPTQ's
 * column-wise OBS update uses H_X as the Hessian proxy).  A column j with
 * H[j][j] == 0 is dead: dead_mask[j] = 1 and its diagonal becomes 1.  Then
 * lambda = damp_frac * mean(diag) is added to the diagonal and the upper
 * triangular Uc with Uc^T Uc = (H + lambda I)^-1 is formed, via H = R R^T
 * (R upper) and Uc = R^-1, in fp64 throughout; Uc is written as fp32 with
 * zeros below the diagonal.
 *
 *   H         fp32 [n, n] symmetric (only the upper triangle is read), ldh >= n.
 *   Uc        fp32 [n, n], lduc >= n.   dead_mask uint8[n] or NULL.
 *   ws        kq_chol_inv_workspace_size(n) bytes.
 *   info      KQ_ERR_NOT_PD (index = column whose pivot failed),
 *             KQ_ERR_NONFINITE (index = row holding NaN/Inf).
 * Limits: 1 <= n <= 65536, 0 <= damp_frac.
 * The serial diagonal chain runs on an internal high-priority stream of the
 * library, one per (host thread, device, caller stream), forked from and
 * joined back into `stream`; calls on different caller streams (each with
 * its own workspace) run concurrently.  Blocked in 64 columns; from
 * n = 8192 on, the bulk trailing update runs once every four block steps
 * over their four panels (rank 256).  The workspace holds the padded fp64
 * matrix and its inverse (2 ld^2 doubles, ld = n rounded up to 128, + 128),
 * eight panel buffers (8 * 64 * ld doubles) and the diagonal blocks'
 * inverse factors (ceil(n/64) * 64^2 doubles).
 * ------------------------------------------------------------------------ */
size_t kq_chol_inv_workspace_size(int64_t n);
kq_status kq_chol_inv(const float* H, int64_t n, int64_t ldh, float damp_frac,
                      float* Uc, int64_t lduc, uint8_t* dead_mask,
                      void* ws, size_t ws_bytes, int32_t* info, kq_stream_t stream);

/* --------------------------------------------------------------------------
 * kq_quantize_layer - blocked column-wise OBS quantization (a7, a8, a9).
 *
 * For each block [i, i+block) and each column j in it (natural order):
 *   q = clamp(rint(w_j / scale + zero), 0, 2^bits - 1),  w_hat = scale (q - zero),
 *   e = (w_j - w_hat) / Uc[j][j],  W[:, j+1:i+block] -= e Uc[j, j+1:i+block];
 * after the block W[:, i+block:] -= E Uc[i:i+block, i+block:] (the lazy
 * trailing update).  H_G does not enter: it cancels from the update (KronQ
 * review, Method (1), Proposition 1).  Grid: asymmetric min/max, scale =
 * (max - min) / (2^bits - 1), zero = rint(-min / scale) (degenerate range:
 * scale 1, zero rint(-min)); per output channel (group == 0, fitted on the
 * initial rows) or per `group` columns (fitted on the current values when the
 * group's first column is reached).  Dead columns (dead_mask[j] != 0) are
 * zeroed first.  Arithmetic is fp32: v = fma(w_j, 1/scale, zero) with the
 * reciprocal rounded once per grid, q = clamp(rint(v)) (rint half-to-even),
 * w_hat = scale (q - zero), e = (w_j - w_hat) * (1 / Uc[j][j]).  A code can
 * therefore differ from one computed with true division only where v lies
 * within about 1e-6 grid steps of a rounding boundary.
 *
 *   W        fp32 [d_out, d_in] rotated weights, ldw >= d_in (read only).
 *   Uc       fp32 [d_in, d_in] from kq_chol_inv, lduc >= d_in.
 *   bits     2..8.   group 0 or a divisor of block that is a multiple of 32.
 *   block    128 (the only block size built).
 *   gemm_mode trailing-update precision: KQ_GEMM_FP32 (SIMT fp32) or
 *            KQ_GEMM_3XTF32 (tcgen05 tensor cores, operands split into tf32 +
 *            remainder, fp32-level accuracy).
 *   codes    uint8 [d_out, d_in], ldq >= d_in; 4-byte aligned, ldq % 4 == 0.
 *   scales, zeros  fp32 [d_out, n_groups], n_groups = 1 or ceil(d_in / group).
 *   W_hat    fp32 [d_out, d_in] dequantized weights (rotated coordinates),
 *            ldwh >= d_in; also used as the running copy of W.
 *   ws       kq_quantize_layer_workspace_size(d_out, d_in, block) bytes.
 *   info     KQ_ERR_NONFINITE (index = row) if W holds NaN/Inf.
 * Limits: 1 <= d_out, 1 <= d_in <= 65536.
 * ------------------------------------------------------------------------ */
size_t kq_quantize_layer_workspace_size(int64_t d_out, int64_t d_in, int block);
kq_status kq_quantize_layer(const float* W, int64_t d_out, int64_t d_in, int64_t ldw,
                            const float* Uc, int64_t lduc, const uint8_t* dead_mask,
                            int bits, int group, int block, int gemm_mode,
                            uint8_t* codes, int64_t ldq, float* scales, float* zeros,
                            float* W_hat, int64_t ldwh,
                            void* ws, size_t ws_bytes, int32_t* info, kq_stream_t stream);

/* kq_quantize_layer_multi - kq_quantize_layer for `count` settings of one
 * layer (the same W, Uc and dead mask; bit-width bits[i] and group group[i]
 * into codes[i], scales[i], zeros[i], W_hat[i]).  The 3xTF32 operand split
 * of Uc is formed once for all settings (KronQ paper page, authors' reply:
 * one set of statistics serves every bit-width).  Stacked outputs: in
 * 3xTF32 mode, when W_hat[i] == W_hat[0] + i * d_out * ldwh for every i
 * (one [count, d_out, ldwh] buffer), up to 4 settings are solved as ONE
 * problem of count * d_out rows (the rows are independent chains that share
 * Uc): each in-block launch covers every setting's rows, each trailing
 * update is one product with M = count * d_out, and the per-channel grids
 * come from one pass over W; settings beyond 4 form further such solves.
 * Otherwise, with a workspace of
 * kq_quantize_layer_multi_workspace_size(d_out, d_in, block, count) bytes
 * up to 4 settings are solved side by side: setting i runs on lane i % 4,
 * lane 0 being `stream` and the others internal streams of the library
 * (created on the first such call of each host thread on each device)
 * forked from and joined back into `stream` by events, so all the work is
 * still ordered on `stream` as one call.  With a smaller workspace of at
 * least kq_quantize_layer_workspace_size bytes the settings run one after
 * the other on `stream` (stacked outputs: one stacked solve per setting).
 * The results are the same in every form, bit for bit.
 * The pointer arrays are HOST arrays of device pointers, read during the
 * call; no two settings may share an output buffer.  Errors as
 * kq_quantize_layer; count >= 1; every setting is validated before any
 * work is enqueued. */
size_t kq_quantize_layer_multi_workspace_size(int64_t d_out, int64_t d_in, int block, int count);
kq_status kq_quantize_layer_multi(const float* W, int64_t d_out, int64_t d_in, int64_t ldw,
                                  const float* Uc, int64_t lduc, const uint8_t* dead_mask,
                                  int count, const int* bits, const int* group, int block, int gemm_mode,
                                  uint8_t* const* codes, int64_t ldq, float* const* scales,
                                  float* const* zeros, float* const* W_hat, int64_t ldwh,
                                  void* ws, size_t ws_bytes, int32_t* info, kq_stream_t stream);

/* kq_solver_timing - diagnostic timing of the solver's kernel classes.
 *
 * kq_solver_timing(1, NULL) makes this host thread's following
 * kq_quantize_layer / kq_quantize_layer_multi calls record a pair of CUDA
 * events around each launch of the grid fit, the in-block recursion and the
 * trailing update (on the stream it goes to); kq_solver_timing(0, out)
 * synchronises those events, writes the summed times and counts to `out`
 * (may be NULL) and stops recording.  The events sit between launches that
 * would otherwise overlap (programmatic dependent launches), so a recorded
 * solve runs slightly slower than an unrecorded one: use it to split a
 * solve's time by kernel class, not to time the solve.  Host memory. */
typedef struct kq_solver_times {
  double grid_ms, inblock_ms, update_ms;               /* summed event intervals per class */
  long long grid_launches, inblock_launches, update_launches;
  double update_flops;   /* algorithmic flops of the trailing updates: sum of 2 M N K */
  double inblock_bytes;  /* algorithmic bytes of the in-block launches: W slab read, W_hat slab,
                            codes and errors written (4 + 4 + 1 + 4 bytes per weight, the
                            errors 8 when kept as a tf32 split for the tensor cores) */
} kq_solver_times;
kq_status kq_solver_timing(int enable, kq_solver_times* out);

/* --------------------------------------------------------------------------
 * kq_kron_loss - Kronecker loss (a10).
 *
 * loss = tr(dW H_X dW^T H_G), dW = W - W_hat (KronQ review, Background: the
 * layer Hessian H ~ H_X kron H_G; Unified Hessian-Guided PTQ, Appendix A.1:
 * the Kronecker-weighted norm as a trace).  H_G == NULL means the identity
 * (the H_X-only GPTQ objective).  Evaluated as the Frobenius product of the
 * larger Hessian H2 with P = D H1^T D^T, H1 the smaller Hessian and D = dW or
 * dW^T (P = dW^T dW when H_G == NULL), P formed only in its upper block
 * triangle: d_out d_in (min + max/2) multiply-adds.  Products on the tensor
 * cores in 3xTF32 (fp32-level accuracy), elementwise products and sums in
 * fp64.
 *
 *   W, W_hat fp32 [d_out, d_in];  H_X fp32 [d_in, d_in];  H_G fp32 [d_out, d_out].
 *   H_X, H_G symmetric (as covariances are): of the larger one only the
 *            256 x 256 blocks on and above the block diagonal are read, and
 *            the result is the loss of the symmetric matrix they define.
 *   loss     device fp64[1].
 *   ws       kq_kron_loss_workspace_size(d_out, d_in) bytes.
 * ------------------------------------------------------------------------ */
size_t kq_kron_loss_workspace_size(int64_t d_out, int64_t d_in);
kq_status kq_kron_loss(const float* W, int64_t ldw, const float* W_hat, int64_t ldwh,
                       int64_t d_out, int64_t d_in,
                       const float* H_X, int64_t ldhx, const float* H_G, int64_t ldhg,
                       double* loss, void* ws, size_t ws_bytes, kq_stream_t stream);

/* kq_kron_loss_multi - kq_kron_loss of `count` dequantized layers W_hat[i]
 * against one W, H_X and H_G (loss[i], device fp64), run one after the other
 * on `stream`; the 3xTF32 operand split of the smaller Hessian is formed once.  The
 * pointer arrays are HOST arrays of device pointers, read during the call.
 * Workspace: kq_kron_loss_workspace_size.  Errors as kq_kron_loss; count >= 1. */
kq_status kq_kron_loss_multi(const float* W, int64_t ldw, int count, const float* const* W_hat,
                             int64_t ldwh, int64_t d_out, int64_t d_in,
                             const float* H_X, int64_t ldhx, const float* H_G, int64_t ldhg,
                             double* const* loss, void* ws, size_t ws_bytes, kq_stream_t stream);

/* kq_kron_loss_blocks - the Kronecker loss with the blockwise H_G of
 * kq_accum_cov_blocks: sum over the row blocks b of
 * tr(dW_b H_X dW_b^T H_G,b), dW_b = rows b k .. b k + k - 1 of W - W_hat and
 * H_G,b = rows b k .. of H_Gb (d_out x k, ldhgb >= k): the loss of the
 * block-diagonal matrix the blocks form (KronQ review, Limitations, second
 * limitation; research thread, "Sparks": blockwise H_G).  Each block as
 * kq_kron_loss (3xTF32 products, same symmetry reading), the partials of all
 * blocks summed in one fixed order.  k divides d_out.  Workspace
 * kq_kron_loss_blocks_workspace_size(d_out, d_in, k). */
size_t kq_kron_loss_blocks_workspace_size(int64_t d_out, int64_t d_in, int64_t k);
kq_status kq_kron_loss_blocks(const float* W, int64_t ldw, const float* W_hat, int64_t ldwh, int64_t d_out,
                              int64_t d_in, const float* H_X, int64_t ldhx, const float* H_Gb, int64_t k,
                              int64_t ldhgb, double* loss, void* ws, size_t ws_bytes, kq_stream_t stream);

/* --------------------------------------------------------------------------
 * kq_kron_loss_noalloc - kq_kron_loss without a caller workspace.
 *
 * The paper has no counterpart to this entry point; it exists for callers
 * that cannot allocate device memory: code embedded in a host application
 * that owns every device allocation through its own pool, or a latency-bound
 * loop where the implicit synchronisation of cudaMalloc/cudaFree is not
 * acceptable.  It computes the same loss with an fp32 CUDA-core kernel that
 * forms one 64 x 64 tile of dW H_X and of H_G^T dW per CTA and sums their
 * elementwise product, which is tr(dW H_X dW^T H_G) exactly for any H_X and
 * H_G (all of both read, no symmetry assumed), and keeps the per-tile partial sums in a
 * fixed array inside the library (static device memory: KQ_KRON_LOSS_NOALLOC_MAX_TILES fp64
 * values, 512 KiB, held by every GPU that loads the library until the
 * process exits).  It calls no cudaMalloc, cudaFree or allocating routine.
 *
 *   Arguments as kq_kron_loss, without ws/ws_bytes.
 *   Limit: ceil(d_out / 64) * ceil(d_in / 64) <= KQ_KRON_LOSS_NOALLOC_MAX_TILES
 *          (e.g. 8192 x 28672 fits) and ceil(d_out / 64) <= 65535; larger
 *          layers get KQ_ERR_UNSUPPORTED_SHAPE.
 *   The stream must belong to the current device.  The first call on a
 *   device looks up the array's device address (cudaGetSymbolAddress) with
 *   that device current; make that first call before any stream capture.
 *   All calls on a device share the one array and it keeps the last call's
 *   contents (nothing in it needs clearing: each call overwrites the slots
 *   it reads).  Calls whose work overlaps on the GPU (other streams, other
 *   host threads) race on the array: serialise them.
 * ------------------------------------------------------------------------ */
#define KQ_KRON_LOSS_NOALLOC_MAX_TILES 65536
kq_status kq_kron_loss_noalloc(const float* W, int64_t ldw, const float* W_hat, int64_t ldwh,
                               int64_t d_out, int64_t d_in,
                               const float* H_X, int64_t ldhx, const float* H_G, int64_t ldhg,
                               double* loss, kq_stream_t stream);

/* --------------------------------------------------------------------------
 * kq_allocate_bits - sublayer bit allocation (a11).  HOST memory, synchronous.
 *
 * Greedy upgrade ordering by the trace sensitivity (KronQ review, Method (2)
 * and Comparison / Table 6 ablation).  Every sublayer starts at the lowest
 * choice; the integer budget is floor(sum(n_params) * (avg_bits - lowest)
 * * (1 + 1e-12)) in bit*parameter units; sublayers are visited by descending
 * score (ties: lower index first) and each takes the highest choice whose
 * extra cost n_params[k] * (b - lowest) still fits the remaining budget.
 *
 *   sens[n_layers], n_params[n_layers] (> 0), choices[n_choices] distinct,
 *   in 1..16; bits_out[n_layers].  All host pointers.
 * ------------------------------------------------------------------------ */
kq_status kq_allocate_bits(const double* sens, const int64_t* n_params, int n_layers,
                           const int* choices, int n_choices, double avg_bits,
                           int* bits_out);

/* --------------------------------------------------------------------------
 * Inference side: packed codes and the matvec with U and V reverted online.
 *
 * KronQ review, Limitations (third limitation): at inference the orthogonal
 * transforms U and V are reverted online, Theta(d_in log d_in + d_out log
 * d_out) per layer; Method (1): W' = V W U^T, so V^T W_hat' U stands for the
 * layer.  The pages give no packed format; this one: each row padded with
 * zero codes to a multiple of 32, the 32 codes of a group in `bits`
 * consecutive 32-bit words (row r, words g*bits .. g*bits + bits - 1), code
 * k of the group at bits bits*k .. bits*k + bits - 1 of the group's
 * little-endian bit stream.
 *
 * kq_pack_codes: uint8 codes [rows, cols] (ldq >= cols) -> uint32 packed
 *   [rows, ceil(cols/32) * bits] (ldp >= that), 1 <= bits <= 8.  A code that
 *   does not fit in `bits` is masked and reported in `info`
 *   (KQ_ERR_INVALID_ARG, index = row).
 * kq_reverted_matvec: Y[b, :] = V^T (W_hat' (U X[b, :])) for b < batch
 *   (1..8), W_hat'[r, c] = scales[r, g] (code[r, c] - zeros[r, g]) with
 *   g = 0 (group == 0, scales/zeros [d_out, 1]) or c / group (group a
 *   multiple of 32, [d_out, ceil(d_in/group)]), i.e. the layout
 *   kq_quantize_layer writes.  T_in (order d_in) / T_out (order d_out) as
 *   for kq_rotate; NULL means the identity (the plain dequantized matvec).
 *   X fp32 [batch, d_in] (ldx >= d_in), Y fp32 [batch, d_out] (ldy >=
 *   d_out; 16-byte aligned with ldy % 4 == 0 when T_out is given);
 *   d_in <= 2^24 (KQ_ERR_UNSUPPORTED_SHAPE above).
 *   ws: kq_reverted_matvec_workspace_size(d_in, batch) bytes (U x is formed
 *   there; without T_in an X that is 16-byte aligned with ldx % 4 == 0 is
 *   read in place).  Kernels: for bits in {2, 3, 4, 8} a row-tiled matvec
 *   (x staged per chunk in shared memory and read once per CTA, the next
 *   chunk's x and packed words in flight while one is summed, each code
 *   decoded once for all vectors); other widths one warp per row.
 * ------------------------------------------------------------------------ */
kq_status kq_pack_codes(const uint8_t* codes, int64_t rows, int64_t cols, int64_t ldq, int bits,
                        uint32_t* packed, int64_t ldp, int32_t* info, kq_stream_t stream);
size_t kq_reverted_matvec_workspace_size(int64_t d_in, int batch);
kq_status kq_reverted_matvec(const uint32_t* packed, int64_t d_out, int64_t d_in, int64_t ldp, int bits,
                             const float* scales, const float* zeros, int group,
                             const kq_rht* T_in, const kq_rht* T_out,
                             const float* X, int64_t ldx, int batch, float* Y, int64_t ldy,
                             void* ws, size_t ws_bytes, kq_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* KRONQ_H */
