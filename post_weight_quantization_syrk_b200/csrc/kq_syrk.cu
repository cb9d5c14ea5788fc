// kq_accum_cov: C (+)= alpha * A^T A from bf16 tokens-by-channels A (a1/a2).
//
// KronQ review (romaanj.github.io/reviews/kronq), Background: H_X (input
// activations) and H_G (output gradients, E[g g^T] per the research thread)
// are the two Kronecker factors of the layer Hessian.
//
// Lower-triangle 64x64 tiles only; each tile is mirrored on write-out.
#include "kq_internal.cuh"

#include <cuda_bf16.h>

namespace {

constexpr int T = 64, TK = 32;

__device__ __forceinline__ void tri_index(int64_t l, int64_t* ti, int64_t* tj) {
  int64_t t = (int64_t)((sqrt(8.0 * (double)l + 1.0) - 1.0) * 0.5);
  while (t * (t + 1) / 2 > l) --t;
  while ((t + 1) * (t + 2) / 2 <= l) ++t;
  *ti = t;
  *tj = l - t * (t + 1) / 2;
}

__global__ void __launch_bounds__(256) syrk_simt_kernel(const __nv_bfloat16* __restrict__ A, int64_t n, int64_t d,
                                                        int64_t lda, float* __restrict__ C, int64_t ldc, float alpha,
                                                        int accumulate, int32_t* info) {
  __shared__ __align__(16) float As[TK][T];
  __shared__ __align__(16) float Bs[TK][T];
  int64_t ti, tj;
  tri_index(blockIdx.x, &ti, &tj);
  const int64_t i0 = ti * T, j0 = tj * T;
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
  for (int64_t t0 = 0; t0 < n; t0 += TK) {
    for (int idx = threadIdx.x; idx < TK * T; idx += 256) {
      int c = idx % T, k = idx / T;
      bool kin = t0 + k < n;
      As[k][c] = (kin && i0 + c < d) ? __bfloat162float(A[(t0 + k) * lda + i0 + c]) : 0.f;
      Bs[k][c] = (kin && j0 + c < d) ? __bfloat162float(A[(t0 + k) * lda + j0 + c]) : 0.f;
    }
    __syncthreads();
#pragma unroll 8
    for (int k = 0; k < TK; ++k) {
      float4 a = *reinterpret_cast<const float4*>(&As[k][ty * 4]);
      float4 b = *reinterpret_cast<const float4*>(&Bs[k][tx * 4]);
      float av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t gi = i0 + ty * 4 + i;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int64_t gj = j0 + tx * 4 + j;
      if (gi >= d || gj >= d || gj > gi) continue;
      float v = alpha * acc[i][j];
      if (accumulate) v += C[gi * ldc + gj];
      if (!isfinite(v)) kq::report(info, KQ_ERR_NONFINITE, gi);
      C[gi * ldc + gj] = v;
      C[gj * ldc + gi] = v;
    }
  }
}

}  // namespace

extern "C" size_t kq_accum_cov_workspace_size(int64_t n, int64_t d) {
  (void)n;
  (void)d;
  return 0;
}

extern "C" kq_status kq_accum_cov(const uint16_t* A, int64_t n, int64_t d, int64_t lda, float* C, int64_t ldc,
                                  float alpha, int accumulate, void* ws, size_t ws_bytes, int32_t* info,
                                  kq_stream_t stream) {
  (void)ws;
  (void)ws_bytes;
  if ((!A && n > 0) || !C || !info) return kq::fail(KQ_ERR_INVALID_ARG, "kq_accum_cov: NULL pointer");
  if (n < 0 || d < 1 || d > 65536) return kq::fail(KQ_ERR_UNSUPPORTED_SHAPE, "kq_accum_cov: need n >= 0, 1 <= d <= 65536");
  if (lda < d || ldc < d) return kq::fail(KQ_ERR_INVALID_ARG, "kq_accum_cov: leading dimension too small");
  if ((n > 0 && !kq::aligned(A, 16)) || (lda & 7)) return kq::fail(KQ_ERR_ALIGNMENT, "kq_accum_cov: A 16-byte aligned, lda % 8 == 0");
  if (!isfinite(alpha)) return kq::fail(KQ_ERR_INVALID_ARG, "kq_accum_cov: alpha not finite");
  cudaStream_t st = (cudaStream_t)stream;
  const int64_t nt = kq::cdiv(d, T);
  syrk_simt_kernel<<<(unsigned)(nt * (nt + 1) / 2), 256, 0, st>>>(reinterpret_cast<const __nv_bfloat16*>(A), n, d,
                                                                 lda, C, ldc, alpha, accumulate, info);
  KQ_TRY(kq::launch_check("kq_accum_cov"));
  kq::clear_error();
  return KQ_OK;
}
