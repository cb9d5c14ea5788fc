// kq_sensitivity: tr(H_X), tr(H_G) and their product in fp64 (step a3).
//
// KronQ review (romaanj.github.io/reviews/kronq), Method (2): the sublayer
// score tr(H_G) tr(H_X).  Only the two diagonals are read (4 (d_in + d_out)
// bytes), so one CTA with a fixed-order tree reduction suffices.
#include "kq_internal.cuh"

namespace {

constexpr int kThreads = 512;

// H_G's diagonal entry i at HG[i * ldg + i % kg]: kg = dg for the whole
// matrix, kg = k for the block-diagonal d x k layout (block b in rows b k ..).
__global__ void __launch_bounds__(kThreads) trace_kernel(const float* __restrict__ HX, int64_t dx, int64_t ldx,
                                                          const float* __restrict__ HG, int64_t dg, int64_t ldg,
                                                          int64_t kg, double* __restrict__ out3) {
  __shared__ double sx[kThreads];
  __shared__ double sg[kThreads];
  double ax = 0.0, ag = 0.0;
  for (int64_t i = threadIdx.x; i < dx; i += kThreads) ax += (double)HX[i * ldx + i];
  for (int64_t i = threadIdx.x; i < dg; i += kThreads) ag += (double)HG[i * ldg + i % kg];
  sx[threadIdx.x] = ax;
  sg[threadIdx.x] = ag;
  __syncthreads();
  for (int s = kThreads / 2; s > 0; s >>= 1) {
    if (threadIdx.x < s) {
      sx[threadIdx.x] += sx[threadIdx.x + s];
      sg[threadIdx.x] += sg[threadIdx.x + s];
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    out3[0] = sx[0];
    out3[1] = sg[0];
    out3[2] = sx[0] * sg[0];
  }
}

}  // namespace

extern "C" kq_status kq_sensitivity(const float* H_X, int64_t d_in, int64_t ldhx, const float* H_G,
                                    int64_t d_out, int64_t ldhg, double* out3, kq_stream_t stream) {
  if (!H_X || !H_G || !out3) return kq::fail(KQ_ERR_INVALID_ARG, "kq_sensitivity: NULL pointer");
  if (d_in < 1 || d_out < 1) return kq::fail(KQ_ERR_INVALID_ARG, "kq_sensitivity: sizes must be >= 1");
  if (ldhx < d_in || ldhg < d_out) return kq::fail(KQ_ERR_INVALID_ARG, "kq_sensitivity: leading dimension too small");
  trace_kernel<<<1, kThreads, 0, (cudaStream_t)stream>>>(H_X, d_in, ldhx, H_G, d_out, ldhg, d_out, out3);
  KQ_TRY(kq::launch_check("kq_sensitivity"));
  kq::clear_error();
  return KQ_OK;
}

extern "C" kq_status kq_sensitivity_blocks(const float* H_X, int64_t d_in, int64_t ldhx, const float* H_Gb,
                                           int64_t d_out, int64_t k, int64_t ldhgb, double* out3, kq_stream_t stream) {
  if (!H_X || !H_Gb || !out3) return kq::fail(KQ_ERR_INVALID_ARG, "kq_sensitivity_blocks: NULL pointer");
  if (d_in < 1 || d_out < 1 || k < 1 || d_out % k)
    return kq::fail(KQ_ERR_INVALID_ARG, "kq_sensitivity_blocks: sizes must be >= 1 and k must divide d_out");
  if (ldhx < d_in || ldhgb < k) return kq::fail(KQ_ERR_INVALID_ARG, "kq_sensitivity_blocks: leading dimension too small");
  trace_kernel<<<1, kThreads, 0, (cudaStream_t)stream>>>(H_X, d_in, ldhx, H_Gb, d_out, ldhgb, k, out3);
  KQ_TRY(kq::launch_check("kq_sensitivity_blocks"));
  kq::clear_error();
  return KQ_OK;
}
