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

// Row-tiled packed matvec for B in {2, 3, 4, 8} (eight codes of a lane lie
// in two words) and NB >= batch vectors: a CTA of WARPS warps takes WARPS R rows; x
// is staged per chunk of 512 to 2048 columns in shared memory (the more
// vectors, the shorter the chunk), so it is read once per CTA
// instead of once per row, in two buffers: the next chunk's x (asynchronous
// copies) and packed words are in flight while this chunk is summed; lane l
// takes columns 8 l .. 8 l + 7 of every 256-column tile, whose codes sit at
// bit 8 B (l % 4) of group 8 t + l / 4
// (words w0 = g B + 8 B (l % 4) / 32 and w0 + 1, never past the group's B
// words), so a warp's word loads for one row are contiguous.  Per tile the
// lane's x values serve all R rows, and each row's eight codes are decoded
// once for all the vectors, as code - zero (exact: the code ORed into the
// mantissa of 2^23, minus 2^23 + zero, the zero being integer-valued and
// the code below 2^8), so y = scale * sum (code - zero) x.  X must be
// 16-byte aligned with ldx % 4 == 0 (the call's staged copy of x is).
template <int B, int R, int NB, int WARPS>
__global__ void __launch_bounds__(WARPS * 32) packed_matvec_rows_kernel(const uint32_t* __restrict__ packed, int64_t ldp,
                                                                 int64_t d_out, int64_t d_in,
                                                                 const float* __restrict__ scales,
                                                                 const float* __restrict__ zeros, int64_t ng,
                                                                 int group, const float* __restrict__ X, int64_t ldx,
                                                                 int batch, float* __restrict__ Y, int64_t ldy) {
  static_assert(B == 2 || B == 3 || B == 4 || B == 8, "two words cover a lane's 8 codes only for these widths");
  // columns per tile; tiles per chunk: as many as keep the two x buffers at 32 KB
  constexpr int TILE = 256, CHUNK = NB <= 2 ? 8 : (NB <= 4 ? 4 : 2);
  constexpr int CW = TILE * CHUNK;       // columns per chunk
  __shared__ __align__(16) float xs[2][NB][CW];
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int64_t r0 = (int64_t)blockIdx.x * (WARPS * R) + warp * R;
  const int64_t tiles = (d_in + TILE - 1) / TILE;
  const int64_t chunks = (tiles + CHUNK - 1) / CHUNK;
  const int din = (int)d_in;   // column and word indices within a row fit in 32 bits (d_in <= 2^24)
  constexpr uint32_t mask = (1u << B) - 1u;
  const int sbit = 8 * B * (lane % 4), s0 = sbit & 31;
  const bool two = s0 + 8 * B > 32;

  // chunk ch of x into buffer ch & 1: 16-byte asynchronous copies, zero past d_in
  auto stage_x = [&](int ch) {
    for (int idx = threadIdx.x; idx < batch * (CW / 4); idx += WARPS * 32) {
      const int b = idx / (CW / 4), c4 = 4 * (idx % (CW / 4));
      const int col = CW * ch + c4;
      const int nbytes = col < din ? 4 * (din - col < 4 ? din - col : 4) : 0;
      const float* src = nbytes ? X + b * ldx + col : X;
      const uint32_t dst = static_cast<uint32_t>(__cvta_generic_to_shared(&xs[ch & 1][b][c4]));
      asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(nbytes) : "memory");
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };
  // the lane's words of chunk ch for the warp's R rows
  // the warp's rows (a row past d_out reads row 0 and is never stored)
  const uint32_t* prow[R];
#pragma unroll
  for (int q = 0; q < R; ++q) prow[q] = packed + (r0 + q < d_out ? r0 + q : 0) * ldp;
  auto load_words = [&](int ch, uint32_t (&lo)[CHUNK][R], uint32_t (&hi)[CHUNK][R]) {
    const int cfirst = CW * ch + 8 * lane;
    if (cfirst + CW - TILE < din) {   // every tile of the chunk holds this lane's columns
#pragma unroll
      for (int u = 0; u < CHUNK; ++u) {
        const int w0 = (8 * (CHUNK * ch + u) + lane / 4) * B + sbit / 32;
#pragma unroll
        for (int q = 0; q < R; ++q) {
          lo[u][q] = prow[q][w0];
          hi[u][q] = two ? prow[q][w0 + 1] : 0u;
        }
      }
    } else {
#pragma unroll
      for (int u = 0; u < CHUNK; ++u) {
        const int w0 = (8 * (CHUNK * ch + u) + lane / 4) * B + sbit / 32;
        const bool ok = cfirst + TILE * u < din;
#pragma unroll
        for (int q = 0; q < R; ++q) {
          lo[u][q] = ok ? prow[q][w0] : 0u;
          hi[u][q] = (ok && two) ? prow[q][w0 + 1] : 0u;
        }
      }
    }
  };

  float acc[R][NB];
#pragma unroll
  for (int q = 0; q < R; ++q)
#pragma unroll
    for (int b = 0; b < NB; ++b) acc[q][b] = 0.f;
  // per-channel grids: each row's scale and zero, read once
  constexpr float kTwo23 = 8388608.f;
  float row_s[R], row_z[R];
#pragma unroll
  for (int q = 0; q < R; ++q) {
    const bool ok = !group && r0 + q < d_out;
    row_s[q] = ok ? scales[(r0 + q) * ng] : 0.f;
    row_z[q] = ok ? zeros[(r0 + q) * ng] : 0.f;
  }

  uint32_t lo[CHUNK][R], hi[CHUNK][R], nlo[CHUNK][R], nhi[CHUNK][R];
  stage_x(0);
  load_words(0, lo, hi);
  for (int ch = 0; ch < (int)chunks; ++ch) {
    const bool more = ch + 1 < chunks;
    if (more) {
      stage_x(ch + 1);            // its buffer was last read before the barrier that ended chunk ch - 1
      load_words(ch + 1, nlo, nhi);
      asm volatile("cp.async.wait_group 1;" ::: "memory");
    } else {
      asm volatile("cp.async.wait_group 0;" ::: "memory");
    }
    __syncthreads();              // chunk ch of x is staged for every thread
    const float(*xc)[CW] = xs[ch & 1];
#pragma unroll
    for (int u = 0; u < CHUNK; ++u) {
      const int c0 = CW * ch + TILE * u + 8 * lane;
      if (c0 >= din) continue;
      const int gi = group ? c0 / group : 0;
      float x8[NB][8];
#pragma unroll
      for (int b = 0; b < NB; ++b) {
        const float4 xa = *reinterpret_cast<const float4*>(&xc[b][TILE * u + 8 * lane]);
        const float4 xb = *reinterpret_cast<const float4*>(&xc[b][TILE * u + 8 * lane + 4]);
        x8[b][0] = xa.x; x8[b][1] = xa.y; x8[b][2] = xa.z; x8[b][3] = xa.w;
        x8[b][4] = xb.x; x8[b][5] = xb.y; x8[b][6] = xb.z; x8[b][7] = xb.w;
      }
#pragma unroll
      for (int q = 0; q < R; ++q) {
        const int64_t r = r0 + q;
        if (r >= d_out) continue;
        const float sc = group ? scales[r * ng + gi] : row_s[q];
        const float zb = kTwo23 + (group ? zeros[r * ng + gi] : row_z[q]);
        // code - zero, exactly: the code ORed into the mantissa of 2^23, minus 2^23 + zero
        float c8[8];
        if constexpr (B == 8) {
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            c8[k] = __uint_as_float(((lo[u][q] >> (8 * k)) & 0xffu) | 0x4B000000u) - zb;
            c8[k + 4] = __uint_as_float(((hi[u][q] >> (8 * k)) & 0xffu) | 0x4B000000u) - zb;
          }
        } else {
          const uint32_t w = __funnelshift_r(lo[u][q], hi[u][q], s0);   // the 8 B <= 32 bits of the lane's codes
#pragma unroll
          for (int k = 0; k < 8; ++k) c8[k] = __uint_as_float(((w >> (B * k)) & mask) | 0x4B000000u) - zb;
        }
#pragma unroll
        for (int b = 0; b < NB; ++b) {
          if (b < batch) {
            float dot = 0.f;
#pragma unroll
            for (int k = 0; k < 8; ++k) dot = fmaf(c8[k], x8[b][k], dot);
            acc[q][b] = fmaf(sc, dot, acc[q][b]);
          }
        }
      }
    }
    __syncthreads();              // buffer ch & 1 may be refilled (chunk ch + 2)
    if (more) {
#pragma unroll
      for (int u = 0; u < CHUNK; ++u)
#pragma unroll
        for (int q = 0; q < R; ++q) {
          lo[u][q] = nlo[u][q];
          hi[u][q] = nhi[u][q];
        }
    }
  }
#pragma unroll
  for (int q = 0; q < R; ++q) {
    const int64_t r = r0 + q;
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      if (b < batch) {
        float v = acc[q][b];
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (lane == 0 && r < d_out) Y[b * ldy + r] = v;
      }
    }
  }
}

template <int B, int R, int WARPS>
void launch_rows(const uint32_t* packed, int64_t ldp, int64_t d_out, int64_t d_in, const float* scales,
                 const float* zeros, int64_t ng, int group, const float* X, int64_t ldx, int batch, float* Y,
                 int64_t ldy, cudaStream_t st) {
  const dim3 grid((unsigned)kq::cdiv(d_out, WARPS * R)), block(WARPS * 32);
  if (batch == 1)
    packed_matvec_rows_kernel<B, R, 1, WARPS><<<grid, block, 0, st>>>(packed, ldp, d_out, d_in, scales, zeros, ng,
                                                                    group, X, ldx, batch, Y, ldy);
  else if (batch == 2)
    packed_matvec_rows_kernel<B, R, 2, WARPS><<<grid, block, 0, st>>>(packed, ldp, d_out, d_in, scales, zeros, ng,
                                                                    group, X, ldx, batch, Y, ldy);
  else if (batch <= 4)
    packed_matvec_rows_kernel<B, R, 4, WARPS><<<grid, block, 0, st>>>(packed, ldp, d_out, d_in, scales, zeros, ng,
                                                                    group, X, ldx, batch, Y, ldy);
  else
    packed_matvec_rows_kernel<B, R, 8, WARPS><<<grid, block, 0, st>>>(packed, ldp, d_out, d_in, scales, zeros, ng,
                                                                    group, X, ldx, batch, Y, ldy);
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
  if constexpr (B == 2 || B == 3 || B == 4 || B == 8) {
    // rows per warp: as many as keep about one CTA per SM or more busy
    // One or two vectors: CTAs of 4 warps and one row per warp, so that the
    // rows spread evenly over the SMs in one wave.  More vectors: 8 warps of
    // 2 or 4 rows, each x value read from shared memory serving more rows.
    constexpr int64_t kSms = 148;
    if (batch <= 2)
      launch_rows<B, 1, 4>(packed, ldp, d_out, d_in, scales, zeros, ng, group, X, ldx, batch, Y, ldy, st);
    else if (d_out >= 2 * 8 * 4 * kSms)
      launch_rows<B, 4, 8>(packed, ldp, d_out, d_in, scales, zeros, ng, group, X, ldx, batch, Y, ldy, st);
    else
      launch_rows<B, 2, 8>(packed, ldp, d_out, d_in, scales, zeros, ng, group, X, ldx, batch, Y, ldy, st);
  } else {
    packed_matvec_kernel<B><<<(unsigned)kq::cdiv(d_out, 8), 256, 0, st>>>(packed, ldp, d_out, d_in, scales, zeros, ng,
                                                                         group, X, ldx, batch, Y, ldy);
  }
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
  if (d_in > (1 << 24)) return kq::fail(KQ_ERR_UNSUPPORTED_SHAPE, "kq_reverted_matvec: d_in above 2^24");
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
  // x' = U x for every vector of the batch, in the workspace (leading
  // dimension a multiple of 4); without U, x itself when it is aligned so
  int64_t ldr = (d_in + 3) / 4 * 4;
  const float* Xr = X;
  if (T_in || !kq::aligned(X, 16) || (ldx & 3)) {
    float* Xw = static_cast<float*>(ws);
    KQ_TRY(kq::cuda_check(cudaMemcpy2DAsync(Xw, ldr * 4, X, ldx * 4, d_in * 4, batch, cudaMemcpyDeviceToDevice, st),
                          "kq_reverted_matvec: copy of X"));
    if (T_in) KQ_TRY(kq_rotate(Xw, batch, d_in, ldr, KQ_AXIS_COLS, T_in, 0, stream));
    Xr = Xw;
  } else {
    ldr = ldx;
  }
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
