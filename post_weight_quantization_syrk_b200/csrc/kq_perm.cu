// Output-channel permutation informed by H_G, and the gathers that apply it.
//
// KronQ paper page (Hugging Face papers 2607.07964), Abstract (1): the
// output-side rotation extends the input-side random rotation "using the
// gradient covariance"; KronQ review (romaanj.github.io/reviews/kronq),
// Limitations (second limitation) and research thread ("Sparks"): a
// blockwise H_G instead of the full d_out x d_out matrix.  Here the output
// rotation may be V = T P_G with P_G a permutation of the output channels
// from diag(H_G): channels ranked by descending gradient energy (ties: lower
// index) are dealt round-robin to the d / k blocks of a blockwise rotation,
// so that every block receives the same share of large and small energies.
//
//   kq_channel_energy:      e[j] = alpha sum_t A[t][j]^2 (= diag(alpha A^T A)),
//                           fp64 partial sums over token slices, added in a
//                           fixed order;
//   kq_balance_permutation: perm[(q % nb) k + q / nb] = the channel of rank q,
//                           the rank found by counting (deterministic);
//   kq_act_order_permutation: perm[q] = the column of rank q by descending
//                           H[j][j] (ties: lower j), the solver's act-order;
//   kq_gather:              out[i][j] = M[r(i)][c(j)] for 1-, 2- or 4-byte elements.
#include <algorithm>

#include "kq_internal.cuh"

namespace {

constexpr int kEnergySlices = 64;    // token slices of the energy sum

// partial[s][j] = sum over tokens t of slice s of A[t][j]^2 (fp64).
__global__ void __launch_bounds__(256) energy_partial_kernel(const uint16_t* __restrict__ A, int64_t n, int64_t d,
                                                             int64_t lda, double* __restrict__ partial) {
  const int64_t j = (int64_t)blockIdx.x * 256 + threadIdx.x;
  const int s = blockIdx.y;
  const int64_t t0 = n * s / kEnergySlices, t1 = n * (s + 1) / kEnergySlices;
  if (j >= d) return;
  double acc = 0.0;
  for (int64_t t = t0; t < t1; ++t) {
    const float v = __uint_as_float((uint32_t)A[t * lda + j] << 16);   // bf16 -> fp32
    acc += (double)v * (double)v;
  }
  partial[(int64_t)s * d + j] = acc;
}

__global__ void __launch_bounds__(256) energy_sum_kernel(const double* __restrict__ partial, int64_t d, float alpha,
                                                         float* __restrict__ out, int32_t* info) {
  const int64_t j = (int64_t)blockIdx.x * 256 + threadIdx.x;
  if (j >= d) return;
  double acc = 0.0;
  for (int s = 0; s < kEnergySlices; ++s) acc += partial[(int64_t)s * d + j];
  const float v = (float)(acc * (double)alpha);
  if (!isfinite(v)) kq::report(info, KQ_ERR_NONFINITE, j);
  out[j] = v;
}

// rank[j] = #{i : e[i] > e[j] or (e[i] == e[j] and i < j)} with e[j] at
// e[j * stride]; one thread per channel, the values streamed through shared
// memory in tiles.  Then perm[(rank % nb) k + rank / nb] = j (k == d: the
// plain descending order).
__global__ void __launch_bounds__(256) balance_perm_kernel(const float* __restrict__ e, int64_t stride, int64_t d,
                                                           int64_t k, int64_t* __restrict__ perm) {
  __shared__ float tile[1024];
  const int64_t j = (int64_t)blockIdx.x * 256 + threadIdx.x;
  const float ej = (j < d) ? e[j * stride] : 0.f;
  int64_t rank = 0;
  for (int64_t i0 = 0; i0 < d; i0 += 1024) {
    for (int u = threadIdx.x; u < 1024; u += 256) tile[u] = (i0 + u < d) ? e[(i0 + u) * stride] : 0.f;
    __syncthreads();
    const int lim = (int)std::min<int64_t>(1024, d - i0);
    for (int u = 0; u < lim; ++u) {
      const float ei = tile[u];
      const int64_t i = i0 + u;
      rank += (ei > ej || (ei == ej && i < j)) ? 1 : 0;
    }
    __syncthreads();
  }
  if (j < d) {
    const int64_t nb = d / k;
    perm[(rank % nb) * k + rank / nb] = j;
  }
}

template <typename T>
__global__ void __launch_bounds__(256) gather_kernel(const T* __restrict__ M, int64_t ldm,
                                                     const int64_t* __restrict__ ridx, const int64_t* __restrict__ cidx,
                                                     int64_t rows, int64_t cols, T* __restrict__ out, int64_t ldo,
                                                     int32_t* info) {
  for (int64_t i = blockIdx.y; i < rows; i += gridDim.y) {
    const int64_t src_row = ridx ? ridx[i] : i;
    if (src_row < 0 || src_row >= rows) {   // an index outside the matrix: reported, not read
      if (threadIdx.x == 0 && blockIdx.x == 0) kq::report(info, KQ_ERR_INVALID_ARG, i);
      continue;
    }
    const T* src = M + src_row * ldm;
    for (int64_t j = (int64_t)blockIdx.x * 256 + threadIdx.x; j < cols; j += (int64_t)gridDim.x * 256) {
      const int64_t c = cidx ? cidx[j] : j;
      if (c < 0 || c >= cols) {
        kq::report(info, KQ_ERR_INVALID_ARG, i);
        continue;
      }
      out[i * ldo + j] = src[c];
    }
  }
}

}  // namespace

extern "C" size_t kq_channel_energy_workspace_size(int64_t d) {
  if (d < 1) return 0;
  return kq::align_up((size_t)kEnergySlices * d * sizeof(double), 256);
}

extern "C" kq_status kq_channel_energy(const uint16_t* A, int64_t n, int64_t d, int64_t lda, float alpha, float* out,
                                       void* ws, size_t ws_bytes, int32_t* info, kq_stream_t stream) {
  if ((!A && n > 0) || !out || !info) return kq::fail(KQ_ERR_INVALID_ARG, "kq_channel_energy: NULL pointer");
  if (n < 0 || d < 1 || d > 65536) return kq::fail(KQ_ERR_UNSUPPORTED_SHAPE, "kq_channel_energy: sizes");
  if (lda < d) return kq::fail(KQ_ERR_INVALID_ARG, "kq_channel_energy: lda < d");
  if (!isfinite(alpha)) return kq::fail(KQ_ERR_INVALID_ARG, "kq_channel_energy: alpha not finite");
  if (!ws || !kq::aligned(ws, 256) || ws_bytes < kq_channel_energy_workspace_size(d))
    return kq::fail(KQ_ERR_WORKSPACE, "kq_channel_energy: workspace too small or not 256-byte aligned");
  cudaStream_t st = (cudaStream_t)stream;
  double* partial = static_cast<double*>(ws);
  const unsigned gx = (unsigned)kq::cdiv(d, 256);
  energy_partial_kernel<<<dim3(gx, kEnergySlices), 256, 0, st>>>(A, n, d, lda, partial);
  KQ_TRY(kq::launch_check("kq_channel_energy"));
  energy_sum_kernel<<<gx, 256, 0, st>>>(partial, d, alpha, out, info);
  KQ_TRY(kq::launch_check("kq_channel_energy sum"));
  kq::clear_error();
  return KQ_OK;
}

extern "C" kq_status kq_balance_permutation(const float* energy, int64_t d, int64_t k, int64_t* perm,
                                            kq_stream_t stream) {
  if (!energy || !perm) return kq::fail(KQ_ERR_INVALID_ARG, "kq_balance_permutation: NULL pointer");
  if (d < 1 || d > 65536 || k < 1 || d % k)
    return kq::fail(KQ_ERR_UNSUPPORTED_SHAPE, "kq_balance_permutation: need 1 <= d <= 65536 and k dividing d");
  cudaStream_t st = (cudaStream_t)stream;
  balance_perm_kernel<<<(unsigned)kq::cdiv(d, 256), 256, 0, st>>>(energy, 1, d, k, perm);
  KQ_TRY(kq::launch_check("kq_balance_permutation"));
  kq::clear_error();
  return KQ_OK;
}

extern "C" kq_status kq_act_order_permutation(const float* H, int64_t n, int64_t ldh, int64_t* perm,
                                              kq_stream_t stream) {
  if (!H || !perm) return kq::fail(KQ_ERR_INVALID_ARG, "kq_act_order_permutation: NULL pointer");
  if (n < 1 || n > 65536) return kq::fail(KQ_ERR_UNSUPPORTED_SHAPE, "kq_act_order_permutation: n outside 1..65536");
  if (ldh < n) return kq::fail(KQ_ERR_INVALID_ARG, "kq_act_order_permutation: ldh < n");
  cudaStream_t st = (cudaStream_t)stream;
  balance_perm_kernel<<<(unsigned)kq::cdiv(n, 256), 256, 0, st>>>(H, ldh + 1, n, n, perm);
  KQ_TRY(kq::launch_check("kq_act_order_permutation"));
  kq::clear_error();
  return KQ_OK;
}

extern "C" kq_status kq_gather(const void* M, int64_t ldm, int elem_bytes, const int64_t* row_idx,
                               const int64_t* col_idx, int64_t rows, int64_t cols, void* out, int64_t ldo,
                               int32_t* info, kq_stream_t stream) {
  if (!M || !out || !info) return kq::fail(KQ_ERR_INVALID_ARG, "kq_gather: NULL pointer");
  if (rows < 0 || cols < 0 || ldm < cols || ldo < cols) return kq::fail(KQ_ERR_INVALID_ARG, "kq_gather: sizes");
  if (elem_bytes != 1 && elem_bytes != 2 && elem_bytes != 4)
    return kq::fail(KQ_ERR_INVALID_ARG, "kq_gather: elem_bytes must be 1, 2 or 4");
  if (rows == 0 || cols == 0) return KQ_OK;
  if (M == out) return kq::fail(KQ_ERR_INVALID_ARG, "kq_gather: out must not alias M");
  cudaStream_t st = (cudaStream_t)stream;
  const unsigned gx = (unsigned)std::min<int64_t>(kq::cdiv(cols, 256), 64);
  const unsigned gy = (unsigned)std::min<int64_t>(rows, 65535);
  if (elem_bytes == 4)
    gather_kernel<uint32_t><<<dim3(gx, gy), 256, 0, st>>>(static_cast<const uint32_t*>(M), ldm, row_idx,
                                                                       col_idx, rows, cols,
                                                                       static_cast<uint32_t*>(out), ldo, info);
  else if (elem_bytes == 1)
    gather_kernel<uint8_t><<<dim3(gx, gy), 256, 0, st>>>(static_cast<const uint8_t*>(M), ldm, row_idx, col_idx, rows,
                                                         cols, static_cast<uint8_t*>(out), ldo, info);
  else
    gather_kernel<uint16_t><<<dim3(gx, gy), 256, 0, st>>>(static_cast<const uint16_t*>(M), ldm, row_idx,
                                                                       col_idx, rows, cols,
                                                                       static_cast<uint16_t*>(out), ldo, info);
  KQ_TRY(kq::launch_check("kq_gather"));
  kq::clear_error();
  return KQ_OK;
}
