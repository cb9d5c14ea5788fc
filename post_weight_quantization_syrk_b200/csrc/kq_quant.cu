// kq_quantize_layer: blocked column-wise OBS (GPTQ) quantization on an
// asymmetric min/max grid (steps a7, a8, a9).
//
// KronQ review (romaanj.github.io/reviews/kronq), Goal and Method (1): the
// solver stays the H_X-only column-wise OBS update (H_G cancels from it,
// Proposition 1).  For each block of 128 columns:
//   in-block recursion (latency bound, 128 dependent steps): one thread owns
//     one output row; the rows of a CTA keep their 128-column slab in shared
//     memory and the block's Uc rows (transposed) beside it; columns are taken
//     in sub-blocks of 32 held in registers, and the rest of the block is
//     brought up to date with the sub-block's 32 errors at once (same
//     left-to-right order of the subtractions as column by column);
//   lazy trailing update W[:, end:] -= E Uc[blk, end:] (a dense GEMM).
// W_hat doubles as the running copy of W: column j of W_hat is overwritten by
// its dequantized value once the column has been quantized.
//
// Grid (asymmetric min/max): scale = (max - min) / (2^b - 1),
// zero = rint(-min / scale); degenerate range: scale 1, zero rint(-min).
// Codes q = clamp(rint(w / scale + zero), 0, 2^b - 1).  IEEE fp32 throughout
// (true division, round half to even).
#include <algorithm>

#include "kq_internal.cuh"

namespace {

constexpr int BLK = 128;      // solver block
constexpr int SUB = 32;       // register sub-block
constexpr int RPC = 32;       // rows (threads) per CTA in the in-block kernel
constexpr int UT_LD = 132;    // padded row of the transposed Uc block
constexpr int WS_LD = 129;    // padded row of the W slab

__device__ __forceinline__ void fit_grid(float mn, float mx, float nl, float* scale, float* zero) {
  float s = (mx - mn) / nl;
  if (s > 0.f) {
    *scale = s;
    *zero = rintf(-mn / s);
  } else {
    *scale = 1.f;
    *zero = rintf(-mn);
  }
}

__device__ __forceinline__ float load_w(const float* __restrict__ src, int64_t ld, int64_t r, int64_t c,
                                        const uint8_t* __restrict__ dead) {
  if (dead && dead[c]) return 0.f;
  return src[r * ld + c];
}

// Per-channel grid from the initial rotated rows (dead columns as zeros).
// One warp per row.
__global__ void grid_rows_kernel(const float* __restrict__ W, int64_t ldw, int64_t d_out, int64_t d_in,
                                 const uint8_t* __restrict__ dead, float nl, float* __restrict__ scales,
                                 float* __restrict__ zeros, int32_t* info) {
  const int64_t r = (int64_t)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  if (r >= d_out) return;
  float mn = INFINITY, mx = -INFINITY;
  bool finite = true;
  for (int64_t c = lane; c < d_in; c += 32) {
    float v = load_w(W, ldw, r, c, dead);
    finite &= isfinite(v);
    mn = fminf(mn, v);
    mx = fmaxf(mx, v);
  }
  for (int o = 16; o > 0; o >>= 1) {
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  }
  finite = __all_sync(0xffffffffu, finite);
  if (lane == 0) {
    if (!finite) kq::report(info, KQ_ERR_NONFINITE, r);
    float s, z;
    fit_grid(mn, mx, nl, &s, &z);
    scales[r] = s;
    zeros[r] = z;
  }
}

struct InblockArgs {
  const float* src;  // W for the first block, W_hat afterwards
  int64_t ld_src;
  float* W_hat;
  int64_t ldwh;
  const float* Uc;
  int64_t lduc;
  const uint8_t* dead;  // applied only when src is W
  int64_t d_out, d_in, i0;
  int bw;      // block width (<= 128)
  int group;   // 0 = per channel
  float nl;
  float* scales;
  float* zeros;
  int64_t n_groups;
  uint8_t* codes;
  int64_t ldq;
  float* ET;   // [128, d_out]: the block's errors, transposed
  int32_t* info;
};

__global__ void __launch_bounds__(RPC) inblock_kernel(InblockArgs a) {
  extern __shared__ float sm[];
  float* UT = sm;                        // [128][UT_LD], UT[k][j] = Uc[i0+j][i0+k]
  float* Ws = UT + BLK * UT_LD;          // [RPC][WS_LD] slab, later W_hat
  float* Es = Ws + RPC * WS_LD;          // [RPC][WS_LD] errors
  uint8_t* Qs = reinterpret_cast<uint8_t*>(Es + RPC * WS_LD);  // [RPC][BLK]
  const int t = threadIdx.x;
  const int64_t row0 = (int64_t)blockIdx.x * RPC;
  const int bw = a.bw;
  const int64_t i0 = a.i0;

  for (int idx = t; idx < BLK * BLK; idx += RPC) {
    int j = idx / BLK, k = idx % BLK;
    UT[k * UT_LD + j] = (k >= j && j < bw && k < bw) ? a.Uc[(i0 + j) * a.lduc + i0 + k] : 0.f;
  }
  for (int idx = t; idx < RPC * BLK; idx += RPC) {
    int r = idx / BLK, c = idx % BLK;
    float v = 0.f;
    if (row0 + r < a.d_out && c < bw) {
      v = load_w(a.src, a.ld_src, row0 + r, i0 + c, a.dead);
      if (!isfinite(v)) kq::report(a.info, KQ_ERR_NONFINITE, row0 + r);
    }
    Ws[r * WS_LD + c] = v;
  }
  __syncthreads();

  const int64_t r = row0 + t;
  float scale = 1.f, zero = 0.f;
  if (!a.group && r < a.d_out) {
    scale = a.scales[r * a.n_groups];
    zero = a.zeros[r * a.n_groups];
  }
  float* wrow = Ws + t * WS_LD;
  float* erow = Es + t * WS_LD;
  for (int s0 = 0; s0 < bw; s0 += SUB) {
    float w[SUB], e[SUB];
#pragma unroll
    for (int jj = 0; jj < SUB; ++jj) {
      w[jj] = (s0 + jj < bw) ? wrow[s0 + jj] : 0.f;
      e[jj] = 0.f;
    }
#pragma unroll
    for (int jj = 0; jj < SUB; ++jj) {
      const int j = s0 + jj;
      if (j < bw) {
        if (a.group && ((i0 + j) % a.group) == 0) {
          // Group grid on the current values of the group's columns; they are
          // all in this block and up to date (group divides the block, and
          // groups start on sub-block boundaries, so w[] == wrow here).
          const int64_t lim = a.d_in - i0;
          const int gend = (int)((int64_t)(j + a.group) < lim ? (int64_t)(j + a.group) : lim);
          float mn = INFINITY, mx = -INFINITY;
          for (int c = j; c < gend; ++c) {
            mn = fminf(mn, wrow[c]);
            mx = fmaxf(mx, wrow[c]);
          }
          fit_grid(mn, mx, a.nl, &scale, &zero);
          if (r < a.d_out) {
            const int64_t g = (i0 + j) / a.group;
            a.scales[r * a.n_groups + g] = scale;
            a.zeros[r * a.n_groups + g] = zero;
          }
        }
        const float v = w[jj] / scale + zero;
        const float q = fminf(fmaxf(rintf(v), 0.f), a.nl);
        const float wh = scale * (q - zero);
        const float ej = (w[jj] - wh) / UT[j * UT_LD + j];
        e[jj] = ej;
#pragma unroll
        for (int kk = jj + 1; kk < SUB; ++kk) w[kk] = fmaf(-ej, UT[(s0 + kk) * UT_LD + j], w[kk]);
        wrow[j] = wh;
        erow[j] = ej;
        Qs[t * BLK + j] = (uint8_t)q;
      }
    }
    // bring the rest of the block up to date with this sub-block's errors
    for (int k = s0 + SUB; k < bw; ++k) {
      float acc = wrow[k];
      const float4* u4 = reinterpret_cast<const float4*>(UT + k * UT_LD + s0);
#pragma unroll
      for (int q4 = 0; q4 < SUB / 4; ++q4) {
        float4 u = u4[q4];
        acc = fmaf(-e[4 * q4 + 0], u.x, acc);
        acc = fmaf(-e[4 * q4 + 1], u.y, acc);
        acc = fmaf(-e[4 * q4 + 2], u.z, acc);
        acc = fmaf(-e[4 * q4 + 3], u.w, acc);
      }
      wrow[k] = acc;
    }
  }
  __syncthreads();
  // coalesced write-back of codes and W_hat (row-major) and of E^T ([128][d_out])
  for (int idx = t; idx < RPC * BLK; idx += RPC) {
    int rr = idx / BLK, c = idx % BLK;
    int64_t row = row0 + rr;
    if (row >= a.d_out || c >= bw) continue;
    a.W_hat[row * a.ldwh + i0 + c] = Ws[rr * WS_LD + c];
    a.codes[row * a.ldq + i0 + c] = Qs[rr * BLK + c];
  }
  for (int idx = t; idx < RPC * BLK; idx += RPC) {
    int c = idx / RPC, rr = idx % RPC;
    int64_t row = row0 + rr;
    if (row >= a.d_out || c >= bw) continue;
    a.ET[(int64_t)c * a.d_out + row] = Es[rr * WS_LD + c];
  }
}

// Lazy trailing update, fp32 SIMT: dst[:, c0..] = src[:, c0..] - E Uc[i0:i0+bw, c0..].
// 128x128 output tile per CTA, 256 threads, 8x8 each, K in chunks of 32.
constexpr int TM = 128, TN = 128, TK = 32;
__global__ void __launch_bounds__(256) trailing_fp32_kernel(const float* __restrict__ src, int64_t ld_src,
                                                            float* __restrict__ dst, int64_t ld_dst,
                                                            const float* __restrict__ ET, const float* __restrict__ Uc,
                                                            int64_t lduc, const uint8_t* __restrict__ dead,
                                                            int64_t d_out, int64_t d_in, int64_t i0, int bw,
                                                            int64_t cstart) {
  __shared__ __align__(16) float As[TK][TM];  // As[k][r] = E[r0+r][k0+k] = ET[k0+k][r0+r]
  __shared__ __align__(16) float Bs[TK][TN];  // Bs[k][c] = Uc[i0+k0+k][c0+c]
  const int64_t r0 = (int64_t)blockIdx.y * TM;
  const int64_t c0 = cstart + (int64_t)blockIdx.x * TN;
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  float acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;
  for (int k0 = 0; k0 < bw; k0 += TK) {
    for (int idx = threadIdx.x; idx < TK * TM; idx += 256) {
      int rr = idx % TM, k = idx / TM;
      As[k][rr] = (r0 + rr < d_out && k0 + k < bw) ? ET[(int64_t)(k0 + k) * d_out + r0 + rr] : 0.f;
    }
    for (int idx = threadIdx.x; idx < TK * TN; idx += 256) {
      int cc = idx % TN, k = idx / TN;
      Bs[k][cc] = (c0 + cc < d_in && k0 + k < bw) ? Uc[(i0 + k0 + k) * lduc + c0 + cc] : 0.f;
    }
    __syncthreads();
#pragma unroll 4
    for (int k = 0; k < TK; ++k) {
      float av[8], bv[8];
      float4 a0 = *reinterpret_cast<const float4*>(&As[k][ty * 4]);
      float4 a1 = *reinterpret_cast<const float4*>(&As[k][64 + ty * 4]);
      float4 b0 = *reinterpret_cast<const float4*>(&Bs[k][tx * 4]);
      float4 b1 = *reinterpret_cast<const float4*>(&Bs[k][64 + tx * 4]);
      av[0] = a0.x; av[1] = a0.y; av[2] = a0.z; av[3] = a0.w;
      av[4] = a1.x; av[5] = a1.y; av[6] = a1.z; av[7] = a1.w;
      bv[0] = b0.x; bv[1] = b0.y; bv[2] = b0.z; bv[3] = b0.w;
      bv[4] = b1.x; bv[5] = b1.y; bv[6] = b1.z; bv[7] = b1.w;
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int64_t row = r0 + (i < 4 ? ty * 4 + i : 64 + ty * 4 + i - 4);
    if (row >= d_out) continue;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int64_t col = c0 + h * 64 + tx * 4;
      if (!dead && col + 3 < d_in) {
        float4 v = *reinterpret_cast<const float4*>(src + row * ld_src + col);
        v.x -= acc[i][4 * h + 0];
        v.y -= acc[i][4 * h + 1];
        v.z -= acc[i][4 * h + 2];
        v.w -= acc[i][4 * h + 3];
        *reinterpret_cast<float4*>(dst + row * ld_dst + col) = v;
      } else {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          if (col + j >= d_in) continue;
          dst[row * ld_dst + col + j] = load_w(src, ld_src, row, col + j, dead) - acc[i][4 * h + j];
        }
      }
    }
  }
}

}  // namespace

extern "C" size_t kq_quantize_layer_workspace_size(int64_t d_out, int64_t d_in, int block) {
  (void)d_in;
  (void)block;
  if (d_out < 1) return 0;
  return kq::align_up((size_t)d_out * BLK * sizeof(float), 256);  // E^T [128][d_out]
}

extern "C" kq_status kq_quantize_layer(const float* W, int64_t d_out, int64_t d_in, int64_t ldw, const float* Uc,
                                       int64_t lduc, const uint8_t* dead_mask, int bits, int group, int block,
                                       int gemm_mode, uint8_t* codes, int64_t ldq, float* scales, float* zeros,
                                       float* W_hat, int64_t ldwh, void* ws, size_t ws_bytes, int32_t* info,
                                       kq_stream_t stream) {
  if (!W || !Uc || !codes || !scales || !zeros || !W_hat || !info)
    return kq::fail(KQ_ERR_INVALID_ARG, "kq_quantize_layer: NULL pointer");
  if (d_out < 1 || d_in < 1 || d_in > 65536) return kq::fail(KQ_ERR_UNSUPPORTED_SHAPE, "kq_quantize_layer: sizes");
  if (d_out > (int64_t)0x7fffffff / 2) return kq::fail(KQ_ERR_UNSUPPORTED_SHAPE, "kq_quantize_layer: d_out too large");
  if (ldw < d_in || lduc < d_in || ldq < d_in || ldwh < d_in)
    return kq::fail(KQ_ERR_INVALID_ARG, "kq_quantize_layer: leading dimension too small");
  if (bits < 2 || bits > 8) return kq::fail(KQ_ERR_INVALID_ARG, "kq_quantize_layer: bits outside 2..8");
  if (block != BLK) return kq::fail(KQ_ERR_UNSUPPORTED_SHAPE, "kq_quantize_layer: only block = 128 is built");
  if (group < 0 || (group && (group % SUB || BLK % group)))
    return kq::fail(KQ_ERR_UNSUPPORTED_SHAPE, "kq_quantize_layer: group must be 0 or a multiple of 32 dividing 128");
  if (gemm_mode != KQ_GEMM_FP32)
    return kq::fail(KQ_ERR_UNSUPPORTED_SHAPE, "kq_quantize_layer: only KQ_GEMM_FP32 is built");
  if (W == W_hat) return kq::fail(KQ_ERR_INVALID_ARG, "kq_quantize_layer: W and W_hat must not alias");
  if (!kq::aligned(W, 16) || !kq::aligned(W_hat, 16) || !kq::aligned(Uc, 16) || (ldw & 3) || (ldwh & 3) || (lduc & 3))
    return kq::fail(KQ_ERR_ALIGNMENT, "kq_quantize_layer: W, W_hat, Uc need 16-byte alignment and ld % 4 == 0");
  if (!ws || !kq::aligned(ws, 256) || ws_bytes < kq_quantize_layer_workspace_size(d_out, d_in, block))
    return kq::fail(KQ_ERR_WORKSPACE, "kq_quantize_layer: workspace too small or not 256-byte aligned");
  cudaStream_t st = (cudaStream_t)stream;
  float* ET = static_cast<float*>(ws);
  const float nl = (float)((1 << bits) - 1);
  const int64_t n_groups = group ? kq::cdiv(d_in, group) : 1;

  if (!group) {
    grid_rows_kernel<<<(unsigned)kq::cdiv(d_out, 8), 256, 0, st>>>(W, ldw, d_out, d_in, dead_mask, nl, scales, zeros,
                                                                   info);
    KQ_TRY(kq::launch_check("kq_quantize_layer grid"));
  }
  const size_t smem = (size_t)BLK * UT_LD * sizeof(float) + 2 * (size_t)RPC * WS_LD * sizeof(float) + RPC * BLK;
  KQ_TRY(kq::cuda_check(cudaFuncSetAttribute(inblock_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem),
                        "kq_quantize_layer: smem attribute"));
  for (int64_t i0 = 0; i0 < d_in; i0 += BLK) {
    const int bw = (int)std::min<int64_t>(BLK, d_in - i0);
    const bool first = (i0 == 0);
    InblockArgs a;
    a.src = first ? W : W_hat;
    a.ld_src = first ? ldw : ldwh;
    a.W_hat = W_hat;
    a.ldwh = ldwh;
    a.Uc = Uc;
    a.lduc = lduc;
    a.dead = first ? dead_mask : nullptr;
    a.d_out = d_out;
    a.d_in = d_in;
    a.i0 = i0;
    a.bw = bw;
    a.group = group;
    a.nl = nl;
    a.scales = scales;
    a.zeros = zeros;
    a.n_groups = n_groups;
    a.codes = codes;
    a.ldq = ldq;
    a.ET = ET;
    a.info = info;
    inblock_kernel<<<(unsigned)kq::cdiv(d_out, RPC), RPC, smem, st>>>(a);
    KQ_TRY(kq::launch_check("kq_quantize_layer inblock"));
    const int64_t cstart = i0 + bw;
    if (cstart < d_in) {
      dim3 grid((unsigned)kq::cdiv(d_in - cstart, TN), (unsigned)kq::cdiv(d_out, TM));
      trailing_fp32_kernel<<<grid, 256, 0, st>>>(first ? W : W_hat, first ? ldw : ldwh, W_hat, ldwh, ET, Uc, lduc,
                                                first ? dead_mask : nullptr, d_out, d_in, i0, bw, cstart);
      KQ_TRY(kq::launch_check("kq_quantize_layer trailing"));
    }
  }
  kq::clear_error();
  return KQ_OK;
}
