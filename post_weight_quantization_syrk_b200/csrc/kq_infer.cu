// Inference side of a quantized layer: packed low-bit codes, and the matvec
// with the BiIP rotations reverted online, y = V^T (W_hat' (U x)).
//
// KronQ review (romaanj.github.io/reviews/kronq), Limitations (third
// limitation): at inference the orthogonal transforms U and V are reverted
// online, Theta(d_in log d_in + d_out log d_out) per layer; Method (1):
// W' = V W U^T, so V^T W_hat' U stands for the layer.  The pages give no
// packed format; the one used here: each row padded with zero codes to a
// multiple of 32, the 32 codes of a group in `bits` consecutive 32-bit
// words, code k at bits bits*k .. bits*k + bits - 1 of the group's
// little-endian bit stream.
#include <algorithm>

#include "kq_internal.cuh"

namespace {

constexpr int kMaxBatch = 8;

// One thread per (row, group of 32 codes): the group's codes gathered into
// B words.  Codes that do not fit in B bits are reported and masked.
template <int B>
__global__ void __launch_bounds__(256) pack_kernel(const uint8_t* __restrict__ codes, int64_t rows, int64_t cols,
                                                   int64_t ldq, uint32_t* __restrict__ packed, int64_t ldp,
                                                   int64_t groups, int32_t* info) {
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= rows * groups) return;
  const int64_t r = idx / groups, g = idx % groups;
  const uint8_t* src = codes + r * ldq + 32 * g;
  const int n = (int)std::min<int64_t>(32, cols - 32 * g);
  uint32_t q[32];
  if (n == 32 && (reinterpret_cast<uintptr_t>(src) & 15) == 0) {
    const uint4 a = reinterpret_cast<const uint4*>(src)[0], b = reinterpret_cast<const uint4*>(src)[1];
    const uint32_t v[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
    for (int k = 0; k < 32; ++k) q[k] = (v[k >> 2] >> (8 * (k & 3))) & 0xffu;
  } else {
#pragma unroll
    for (int k = 0; k < 32; ++k) q[k] = k < n ? src[k] : 0u;
  }
  constexpr uint32_t mask = (1u << B) - 1u;
  uint32_t w[B];
#pragma unroll
  for (int i = 0; i < B; ++i) w[i] = 0;
  bool bad = false;
#pragma unroll
  for (int k = 0; k < 32; ++k) {
    bad |= (q[k] & ~mask) != 0;
    const uint32_t c = q[k] & mask;
    const int pos = B * k, wi = pos >> 5, sh = pos & 31;
    w[wi] |= c << sh;
    if (sh + B > 32) w[wi + 1] |= c >> (32 - sh);
  }
  if (bad) kq::report(info, KQ_ERR_INVALID_ARG, r);
  uint32_t* dst = packed + r * ldp + g * B;
#pragma unroll
  for (int i = 0; i < B; ++i) dst[i] = w[i];
}

// Code k (a compile-time index after unrolling) of a group from its B words.
template <int B>
__device__ __forceinline__ float code_at(const uint32_t (&w)[B], int k) {
  const int pos = B * k, wi = pos >> 5, sh = pos & 31;
  uint32_t c = w[wi] >> sh;
  if (sh + B > 32) c |= w[wi + 1] << (32 - sh);
  return (float)(c & ((1u << B) - 1u));
}

// yr[b, r] = sum_c scale[r, g(c)] (code[r, c] - zero[r, g(c)]) x[b, c].
// One warp per row; lane l takes the 32-code chunks l, l + 32, ...; per chunk
// sum_k code_k x_k and sum_k x_k, then one fma with the chunk's grid (every
// chunk lies in one grid group: groups are multiples of 32 columns).  The
// packed weights stream once; x stays in L1/L2.
template <int B>
__global__ void __launch_bounds__(256) packed_matvec_kernel(const uint32_t* __restrict__ packed, int64_t ldp,
                                                            int64_t d_out, int64_t d_in,
                                                            const float* __restrict__ scales,
                                                            const float* __restrict__ zeros, int64_t ng, int group,
                                                            const float* __restrict__ X, int64_t ldx, int batch,
                                                            float* __restrict__ Y, int64_t ldy) {
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int64_t r = (int64_t)blockIdx.x * 8 + warp;
  if (r >= d_out) return;
  const int64_t chunks = (d_in + 31) / 32;
  const uint32_t* prow = packed + r * ldp;
  float acc[kMaxBatch];
#pragma unroll
  for (int b = 0; b < kMaxBatch; ++b) acc[b] = 0.f;
  for (int64_t ch = lane; ch < chunks; ch += 32) {
    uint32_t w[B];
#pragma unroll
    for (int i = 0; i < B; ++i) w[i] = prow[ch * B + i];
    const int64_t gi = group ? (32 * ch) / group : 0;
    const float s = scales[r * ng + gi], z = zeros[r * ng + gi];
    const int64_t c0 = 32 * ch;
    const bool full = c0 + 32 <= d_in;
#pragma unroll
    for (int b = 0; b < kMaxBatch; ++b) {
      if (b < batch) {
        const float* xb = X + b * ldx + c0;
        float dot = 0.f, sx = 0.f;
        if (full) {
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const float4 x4 = reinterpret_cast<const float4*>(xb)[j];
            dot = fmaf(code_at<B>(w, 4 * j), x4.x, dot);
            dot = fmaf(code_at<B>(w, 4 * j + 1), x4.y, dot);
            dot = fmaf(code_at<B>(w, 4 * j + 2), x4.z, dot);
            dot = fmaf(code_at<B>(w, 4 * j + 3), x4.w, dot);
            sx += (x4.x + x4.y) + (x4.z + x4.w);
          }
        } else {
#pragma unroll
          for (int k = 0; k < 32; ++k) {
            const float xv = (c0 + k < d_in) ? xb[k] : 0.f;
            dot = fmaf(code_at<B>(w, k), xv, dot);
            sx += xv;
          }
        }
        acc[b] = fmaf(s, fmaf(-z, sx, dot), acc[b]);
      }
    }
  }
#pragma unroll
  for (int b = 0; b < kMaxBatch; ++b) {
    if (b < batch) {
      float v = acc[b];
      for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      if (lane == 0) Y[b * ldy + r] = v;
    }
  }
}

template <int B>
kq_status launch_pack(const uint8_t* codes, int64_t rows, int64_t cols, int64_t ldq, uint32_t* packed, int64_t ldp,
                      int32_t* info, cudaStream_t st) {
  const int64_t groups = (cols + 31) / 32, n = rows * groups;
  pack_kernel<B><<<(unsigned)kq::cdiv(n, 256), 256, 0, st>>>(codes, rows, cols, ldq, packed, ldp, groups, info);
  return kq::launch_check("kq_pack_codes");
}

template <int B>
kq_status launch_matvec(const uint32_t* packed, int64_t ldp, int64_t d_out, int64_t d_in, const float* scales,
                        const float* zeros, int64_t ng, int group, const float* X, int64_t ldx, int batch, float* Y,
                        int64_t ldy, cudaStream_t st) {
  packed_matvec_kernel<B><<<(unsigned)kq::cdiv(d_out, 8), 256, 0, st>>>(packed, ldp, d_out, d_in, scales, zeros, ng,
                                                                       group, X, ldx, batch, Y, ldy);
  return kq::launch_check("kq_reverted_matvec");
}

size_t x_bytes(int64_t d_in, int batch) { return kq::align_up((size_t)batch * ((d_in + 3) / 4 * 4) * 4, 256); }

}  // namespace

extern "C" kq_status kq_pack_codes(const uint8_t* codes, int64_t rows, int64_t cols, int64_t ldq, int bits,
                                   uint32_t* packed, int64_t ldp, int32_t* info, kq_stream_t stream) {
  if (!codes || !packed || !info) return kq::fail(KQ_ERR_INVALID_ARG, "kq_pack_codes: NULL pointer");
  if (rows < 1 || cols < 1) return kq::fail(KQ_ERR_INVALID_ARG, "kq_pack_codes: sizes must be >= 1");
  if (bits < 1 || bits > 8) return kq::fail(KQ_ERR_INVALID_ARG, "kq_pack_codes: bits outside 1..8");
  if (ldq < cols || ldp < (cols + 31) / 32 * bits)
    return kq::fail(KQ_ERR_INVALID_ARG, "kq_pack_codes: leading dimension too small");
  if (kq::cdiv(rows * ((cols + 31) / 32), 256) > 0x7fffffff)
    return kq::fail(KQ_ERR_UNSUPPORTED_SHAPE, "kq_pack_codes: too large");
  cudaStream_t st = (cudaStream_t)stream;
  switch (bits) {
    case 1: return launch_pack<1>(codes, rows, cols, ldq, packed, ldp, info, st);
    case 2: return launch_pack<2>(codes, rows, cols, ldq, packed, ldp, info, st);
    case 3: return launch_pack<3>(codes, rows, cols, ldq, packed, ldp, info, st);
    case 4: return launch_pack<4>(codes, rows, cols, ldq, packed, ldp, info, st);
    case 5: return launch_pack<5>(codes, rows, cols, ldq, packed, ldp, info, st);
    case 6: return launch_pack<6>(codes, rows, cols, ldq, packed, ldp, info, st);
    case 7: return launch_pack<7>(codes, rows, cols, ldq, packed, ldp, info, st);
    default: return launch_pack<8>(codes, rows, cols, ldq, packed, ldp, info, st);
  }
}

extern "C" size_t kq_reverted_matvec_workspace_size(int64_t d_in, int batch) {
  if (d_in < 1 || batch < 1) return 0;
  return x_bytes(d_in, batch);
}

extern "C" kq_status kq_reverted_matvec(const uint32_t* packed, int64_t d_out, int64_t d_in, int64_t ldp, int bits,
                                        const float* scales, const float* zeros, int group, const kq_rht* T_in,
                                        const kq_rht* T_out, const float* X, int64_t ldx, int batch, float* Y,
                                        int64_t ldy, void* ws, size_t ws_bytes, kq_stream_t stream) {
  if (!packed || !scales || !zeros || !X || !Y) return kq::fail(KQ_ERR_INVALID_ARG, "kq_reverted_matvec: NULL pointer");
  if (d_out < 1 || d_in < 1) return kq::fail(KQ_ERR_INVALID_ARG, "kq_reverted_matvec: sizes must be >= 1");
  if (bits < 1 || bits > 8) return kq::fail(KQ_ERR_INVALID_ARG, "kq_reverted_matvec: bits outside 1..8");
  if (batch < 1 || batch > kMaxBatch) return kq::fail(KQ_ERR_UNSUPPORTED_SHAPE, "kq_reverted_matvec: batch outside 1..8");
  if (group < 0 || (group % 32)) return kq::fail(KQ_ERR_UNSUPPORTED_SHAPE, "kq_reverted_matvec: group must be 0 or a multiple of 32");
  if (ldp < (d_in + 31) / 32 * bits || ldx < d_in || ldy < d_out)
    return kq::fail(KQ_ERR_INVALID_ARG, "kq_reverted_matvec: leading dimension too small");
  if ((T_in && T_in->n != d_in) || (T_out && T_out->n != d_out))
    return kq::fail(KQ_ERR_INVALID_ARG, "kq_reverted_matvec: rotation order does not match the layer");
  if (T_out && (!kq::aligned(Y, 16) || (ldy & 3)))
    return kq::fail(KQ_ERR_ALIGNMENT, "kq_reverted_matvec: Y needs 16-byte alignment and ldy %% 4 == 0");
  if (!ws || !kq::aligned(ws, 256) || ws_bytes < kq_reverted_matvec_workspace_size(d_in, batch))
    return kq::fail(KQ_ERR_WORKSPACE, "kq_reverted_matvec: workspace too small or not 256-byte aligned");
  cudaStream_t st = (cudaStream_t)stream;
  // x' = U x for every vector of the batch, in the workspace (leading dimension a multiple of 4)
  const int64_t ldr = (d_in + 3) / 4 * 4;
  float* Xr = static_cast<float*>(ws);
  KQ_TRY(kq::cuda_check(cudaMemcpy2DAsync(Xr, ldr * 4, X, ldx * 4, d_in * 4, batch, cudaMemcpyDeviceToDevice, st),
                        "kq_reverted_matvec: copy of X"));
  if (T_in) KQ_TRY(kq_rotate(Xr, batch, d_in, ldr, KQ_AXIS_COLS, T_in, 0, stream));
  const int64_t ng = group ? (d_in + group - 1) / group : 1;
  kq_status s;
  switch (bits) {
    case 1: s = launch_matvec<1>(packed, ldp, d_out, d_in, scales, zeros, ng, group, Xr, ldr, batch, Y, ldy, st); break;
    case 2: s = launch_matvec<2>(packed, ldp, d_out, d_in, scales, zeros, ng, group, Xr, ldr, batch, Y, ldy, st); break;
    case 3: s = launch_matvec<3>(packed, ldp, d_out, d_in, scales, zeros, ng, group, Xr, ldr, batch, Y, ldy, st); break;
    case 4: s = launch_matvec<4>(packed, ldp, d_out, d_in, scales, zeros, ng, group, Xr, ldr, batch, Y, ldy, st); break;
    case 5: s = launch_matvec<5>(packed, ldp, d_out, d_in, scales, zeros, ng, group, Xr, ldr, batch, Y, ldy, st); break;
    case 6: s = launch_matvec<6>(packed, ldp, d_out, d_in, scales, zeros, ng, group, Xr, ldr, batch, Y, ldy, st); break;
    case 7: s = launch_matvec<7>(packed, ldp, d_out, d_in, scales, zeros, ng, group, Xr, ldr, batch, Y, ldy, st); break;
    default: s = launch_matvec<8>(packed, ldp, d_out, d_in, scales, zeros, ng, group, Xr, ldr, batch, Y, ldy, st); break;
  }
  KQ_TRY(s);
  // y = V^T y' in place
  if (T_out) KQ_TRY(kq_rotate(Y, batch, d_out, ldy, KQ_AXIS_COLS, T_out, 1, stream));
  kq::clear_error();
  return KQ_OK;
}
