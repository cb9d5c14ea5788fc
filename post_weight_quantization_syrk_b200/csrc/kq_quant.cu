// kq_quantize_layer: blocked column-wise OBS (GPTQ) quantization on an
// asymmetric min/max grid (steps a7, a8, a9).
//
// KronQ review (romaanj.github.io/reviews/kronq), Goal and Method (1): the
// solver stays the H_X-only column-wise OBS update (H_G cancels from it,
// Proposition 1).  For each block of 128 columns:
//   in-block recursion (latency bound, 128 dependent steps): eight lanes
//     share one output row, each holding 16 of the block's columns in
//     registers; the column's owner quantizes it and broadcasts its error by
//     warp shuffle, and every lane applies the rank-1 update to its own
//     columns with the block's Uc rows read from shared memory.  The
//     subtractions into each column happen in the same left-to-right order
//     as column by column;
//   lazy trailing update W[:, end:] -= E Uc[blk, end:] (a dense GEMM): fp32
//     SIMT (KQ_GEMM_FP32) or 3xTF32 on the tcgen05 tensor cores
//     (KQ_GEMM_3XTF32, the block's errors split into tf32 + remainder as they
//     are written, Uc split once per call).
// W_hat doubles as the running copy of W: column j of W_hat is overwritten by
// its dequantized value once the column has been quantized.
//
// Grid (asymmetric min/max): scale = (max - min) / (2^b - 1),
// zero = rint(-min / scale); degenerate range: scale 1, zero rint(-min).
// Codes q = clamp(rint(v), 0, 2^b - 1) with v = fma(w, 1/scale, zero) in fp32
// (round half to even); errors e = (w - w_hat) * (1/Uc[j][j]).  The grid
// itself (scale, zero) uses IEEE fp32 division.
#include <algorithm>
#include <cstdint>
#include <vector>

#include "kq_gemm.cuh"
#include "kq_internal.cuh"

namespace {

constexpr int BLK = 128;      // solver block

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

// The per-channel settings of a stacked solve: each fits its grid to the
// same row minimum and maximum.
struct GridSets {
  int count;
  float nl[4];
  float* scales[4];
  float* zeros[4];
};

// Per-channel grid from the initial rotated rows (dead columns as zeros),
// for every per-channel setting of the solve from one read of W.  One warp
// per row.
__global__ void grid_rows_kernel(const float* __restrict__ W, int64_t ldw, int64_t d_out, int64_t d_in,
                                 const uint8_t* __restrict__ dead, GridSets gs, int32_t* info) {
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
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      if (i >= gs.count) break;
      float sc, z;
      fit_grid(mn, mx, gs.nl[i], &sc, &z);
      gs.scales[i][r] = sc;
      gs.zeros[i][r] = z;
    }
  }
}

// Most settings of one layer solved as one stacked problem: their rows are
// independent chains that share Uc, so setting s's rows follow setting
// s - 1's in W_hat and in the errors, and every launch of the solve covers
// all of them.
constexpr int kMaxStack = 4;

// The outputs and grid of one setting.
struct SetArgs {
  uint8_t* codes;
  float* scales;
  float* zeros;
  int64_t n_groups;
  int group;   // 0 = per channel
  float nl;    // 2^bits - 1
};

struct InblockArgs {
  const float* src;  // W for the first block, W_hat afterwards
  int64_t ld_src;
  int64_t src_set;   // setting s reads its rows at src + s * src_set (0: all read W)
  float* W_hat;
  int64_t ldwh;
  int64_t wh_set;    // setting s's rows of W_hat start at W_hat + s * wh_set
  const float* Uc;
  int64_t lduc;
  const uint8_t* dead;  // applied only when src is W
  int64_t d_out, d_in, i0;
  int bw;      // block width (<= 128)
  int64_t ldq;
  float* ET;   // [128, d_out]: the block's errors, transposed (fp32 SIMT trailing update; one setting)
  float* Eb;   // tf32 part of the errors (3xTF32 trailing update), or NULL:
  float* Es;   // row r of setting s, column c of the block at [(s d_out + r) * ldE + e_col0 + c]; remainder
  int64_t ldE, e_col0;
  int32_t* info;
  SetArgs set[kMaxStack];   // setting s = blockIdx.y
};

// LPR lanes share a row (LPR = 8 or 4): lane L of a row group owns the
// 128 / LPR columns 4 LPR m + 4 L + t (t in 0..3, m in 0..32/LPR - 1), kept
// in registers.  Column j is quantized by its owner, whose error e_j reaches
// the row's other lanes by one warp shuffle; every lane then updates its own
// columns right of j.  This interleaved ownership makes each lane's float4
// reads of Uc row j hit distinct shared-memory banks (the row groups of a
// warp read the same row: broadcast).  Fewer lanes per row mean fewer warps
// repeating the per-column quantisation and shuffle (the latency-bound part)
// for the same multiply-adds.
// Threads per CTA of the in-block kernel (4 rows per warp): 224 (28 rows)
// below kStackedRows rows, so that 4096 rows make 147 CTAs on 147 SMs
// (measured 1.46 -> 1.38 ms for one attn4096 solve); 256 (32 rows) for
// larger stacked solves, where 441 CTAs of 28 rows measured slower than 384
// of 32 (1.30 against 1.05 ms for the 32 in-block launches of three
// attn4096 settings).
constexpr int kStackedRows = 2 * 148 * 32;
constexpr int IB_SMEM = BLK * BLK * 4 + BLK * 4;

template <int LPR>
__device__ __forceinline__ int col_of(int L, int r) { return 4 * LPR * (r >> 2) + 4 * L + (r & 3); }

template <int LPR, int IB_THREADS>
__global__ void __launch_bounds__(IB_THREADS) inblock_kernel(InblockArgs a) {
  constexpr int IB_ROWS = IB_THREADS / LPR;   // rows per CTA
  constexpr int NR = BLK / LPR;               // columns (registers) per lane
  constexpr int MB = NR / 4;                  // register blocks of 4 columns
  constexpr int SPAN = 4 * LPR;               // columns per register block over the row group
  extern __shared__ float sm[];
  float* Us = sm;                 // [128][128]: Uc[i0 + j][i0 + k]
  float* inv_d = sm + BLK * BLK;  // 1 / Uc[i0 + j][i0 + j]
  const int t = threadIdx.x;
  const int lane = t & 31, L = lane & (LPR - 1);
  const int64_t row = (int64_t)blockIdx.x * IB_ROWS + t / LPR;   // row of the setting
  const bool row_ok = row < a.d_out;
  const int bw = a.bw;
  const int64_t i0 = a.i0;
  // this CTA's setting (uniform over the CTA, so its control flow is too)
  const int s = blockIdx.y;
  const SetArgs S = s == 0 ? a.set[0] : s == 1 ? a.set[1] : s == 2 ? a.set[2] : a.set[3];
  const float* __restrict__ src = a.src + s * a.src_set;
  float* __restrict__ W_hat = a.W_hat + s * a.wh_set;
  const int64_t erow = s * a.d_out + row;   // row of the stacked errors
  kq::pdl_trigger();

  // the block of Uc: 16 asynchronous 16-byte copies per thread, all in
  // flight while the row is loaded (bytes past the block are zero-filled).
  // No kernel of the solve writes Uc, so the copies may start before the
  // previous kernel (a trailing update) has finished.
#pragma unroll
  for (int u = 0; u < (BLK * (BLK / 4) + IB_THREADS - 1) / IB_THREADS; ++u) {
    const int idx = t + IB_THREADS * u;
    if (idx >= BLK * (BLK / 4)) break;
    const int j = idx / (BLK / 4), k = 4 * (idx % (BLK / 4));
    // chunks wholly below the diagonal (k + 3 < j) are zero-filled: only the
    // upper triangle of Uc is the factor
    const int nbytes = (j < bw && k + 3 >= j) ? 4 * max(0, min(4, bw - k)) : 0;
    const float* g = nbytes ? a.Uc + (i0 + j) * a.lduc + i0 + k : a.Uc + i0 * a.lduc + i0;
    const uint32_t dst = static_cast<uint32_t>(__cvta_generic_to_shared(Us + j * BLK + k));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(g), "r"(nbytes) : "memory");
  }
  asm volatile("cp.async.commit_group;" ::: "memory");
  kq::pdl_wait();

  // this lane's columns of the row
  float w[NR];
#pragma unroll
  for (int m = 0; m < MB; ++m) {
    const int c = SPAN * m + 4 * L;
    float v[4] = {0.f, 0.f, 0.f, 0.f};
    if (row_ok) {
      if (c + 3 < bw && !a.dead) {
        const float4 q = *reinterpret_cast<const float4*>(src + row * a.ld_src + i0 + c);
        v[0] = q.x; v[1] = q.y; v[2] = q.z; v[3] = q.w;
      } else {
        for (int e = 0; e < 4; ++e)
          if (c + e < bw) v[e] = load_w(src, a.ld_src, row, i0 + c + e, a.dead);
      }
      if (!(isfinite(v[0]) && isfinite(v[1]) && isfinite(v[2]) && isfinite(v[3])))
        kq::report(a.info, KQ_ERR_NONFINITE, row);
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) w[4 * m + e] = v[e];
  }
  asm volatile("cp.async.wait_group 0;" ::: "memory");
  __syncthreads();
  // ... and in the chunk holding the diagonal, the entries left of it are
  // cleared, so that the column updates below can run unpredicated
  if (t < BLK) {
    for (int k = t & ~3; k < t; ++k) Us[t * BLK + k] = 0.f;
  }
  __syncthreads();
  if (t < BLK) inv_d[t] = (t < bw) ? 1.f / Us[t * BLK + t] : 0.f;
  __syncthreads();

  float scale = 1.f, zero = 0.f;
  if (!S.group && row_ok) {
    scale = S.scales[row * S.n_groups];
    zero = S.zeros[row * S.n_groups];
  }
  float inv_scale = 1.f / scale;
  float qv[NR], ev[NR];
  const int gbase = lane & ~(LPR - 1);

#pragma unroll
  for (int m = 0; m < MB; ++m) {
#pragma unroll 1
    for (int Lo = 0; Lo < LPR; ++Lo) {
#pragma unroll
      for (int tt = 0; tt < 4; ++tt) {
        const int j = SPAN * m + 4 * Lo + tt;   // column quantized in this step
        if (j >= bw) break;
        if (S.group && tt == 0 && ((i0 + j) % S.group) == 0) {
          // group grid on the current values of columns [j, j + group): every
          // lane folds its own columns in range, then the row's lanes meet
          const int64_t lim = a.d_in - i0;
          const int gend = (int)((int64_t)(j + S.group) < lim ? (int64_t)(j + S.group) : lim);
          float mn = INFINITY, mx = -INFINITY;
#pragma unroll
          for (int r = 0; r < NR; ++r) {
            const int c = col_of<LPR>(L, r);
            if (c >= j && c < gend) {
              mn = fminf(mn, w[r]);
              mx = fmaxf(mx, w[r]);
            }
          }
#pragma unroll
          for (int o = 1; o < LPR; o <<= 1) {
            mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
          }
          fit_grid(mn, mx, S.nl, &scale, &zero);
          inv_scale = 1.f / scale;
          if (row_ok && L == 0) {
            const int64_t g = (i0 + j) / S.group;
            S.scales[row * S.n_groups + g] = scale;
            S.zeros[row * S.n_groups + g] = zero;
          }
        }
        // every lane runs the owner's arithmetic on its own register 4m+tt;
        // only the owner's (L == Lo) result is kept and broadcast
        const int r = 4 * m + tt;
        const float x = w[r];
        const float v = fmaf(x, inv_scale, zero);
        const float q = fminf(fmaxf(rintf(v), 0.f), S.nl);
        const float wh = scale * (q - zero);
        const float e_own = (x - wh) * inv_d[j];
        const float e = __shfl_sync(0xffffffffu, e_own, gbase + Lo);
        // columns left of j see Uc[j][c] = 0 (cleared above), so the update
        // runs over all of this lane's columns; column j itself is then set
        // to its final dequantized value by its owner
        // register blocks m2 < m hold columns left of SPAN m <= j: final, skipped
        const float4* urow = reinterpret_cast<const float4*>(Us + j * BLK);
#pragma unroll
        for (int m2 = m; m2 < MB; ++m2) {
          const float4 u = urow[LPR * m2 + L];
          const float uu[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
          for (int t2 = 0; t2 < 4; ++t2) w[4 * m2 + t2] = fmaf(-e, uu[t2], w[4 * m2 + t2]);
        }
        if (L == Lo) {
          qv[r] = q;
          w[r] = wh;   // the column is final: keep its dequantized value
          ev[r] = e_own;
        }
      }
    }
  }

  if (!row_ok) return;
  // this lane's columns: W_hat, codes, and the errors for the trailing update
#pragma unroll
  for (int m = 0; m < MB; ++m) {
    const int c = SPAN * m + 4 * L;
    if (c + 3 < bw) {
      *reinterpret_cast<float4*>(W_hat + row * a.ldwh + i0 + c) = make_float4(w[4 * m], w[4 * m + 1], w[4 * m + 2],
                                                                             w[4 * m + 3]);
      uchar4 qq = make_uchar4((unsigned char)qv[4 * m], (unsigned char)qv[4 * m + 1], (unsigned char)qv[4 * m + 2],
                              (unsigned char)qv[4 * m + 3]);
      *reinterpret_cast<uchar4*>(S.codes + row * a.ldq + i0 + c) = qq;
    } else {
      for (int e = 0; e < 4; ++e)
        if (c + e < bw) {
          W_hat[row * a.ldwh + i0 + c + e] = w[4 * m + e];
          S.codes[row * a.ldq + i0 + c + e] = (uint8_t)qv[4 * m + e];
        }
    }
    if (a.Eb) {
      float b[4], sm4[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float ee = (c + e < bw) ? ev[4 * m + e] : 0.f;
        uint32_t bits;
        asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(bits) : "f"(ee));
        b[e] = __uint_as_float(bits);
        sm4[e] = ee - b[e];
      }
      *reinterpret_cast<float4*>(a.Eb + erow * a.ldE + a.e_col0 + c) = make_float4(b[0], b[1], b[2], b[3]);
      *reinterpret_cast<float4*>(a.Es + erow * a.ldE + a.e_col0 + c) = make_float4(sm4[0], sm4[1], sm4[2], sm4[3]);
    } else {
      for (int e = 0; e < 4; ++e)
        if (c + e < bw) a.ET[(int64_t)(c + e) * a.d_out + row] = ev[4 * m + e];
    }
  }
}

// Lanes per row of the in-block recursion.
constexpr int kLanesPerRow = 8;

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

namespace {

// Diagnostic timing (kq_solver_timing): event pairs around each launch,
// recorded per host thread while enabled.
enum TimedClass { kClassGrid = 0, kClassInblock = 1, kClassUpdate = 2 };
struct TimedLaunch {
  int cls;
  cudaEvent_t a, b;
  double flops, bytes;
};
struct SolverTiming {
  bool on = false;
  std::vector<TimedLaunch> recs;
  std::vector<cudaEvent_t> pool;
};
thread_local SolverTiming g_timing;

kq_status timing_event(cudaEvent_t* e) {
  if (!g_timing.pool.empty()) {
    *e = g_timing.pool.back();
    g_timing.pool.pop_back();
    return KQ_OK;
  }
  return kq::cuda_check(cudaEventCreate(e), "kq_solver_timing: event");
}

// Runs `launch` (a kq_status-returning callable) between two recorded events
// when timing is on; otherwise just runs it.
template <typename F>
kq_status timed(int cls, double flops, double bytes, cudaStream_t st, F&& launch) {
  if (!g_timing.on) return launch();
  TimedLaunch r{cls, nullptr, nullptr, flops, bytes};
  KQ_TRY(timing_event(&r.a));
  KQ_TRY(timing_event(&r.b));
  KQ_TRY(kq::cuda_check(cudaEventRecord(r.a, st), "kq_solver_timing: record"));
  const kq_status s = launch();
  KQ_TRY(kq::cuda_check(cudaEventRecord(r.b, st), "kq_solver_timing: record"));
  g_timing.recs.push_back(r);
  return s;
}

// Outer block of the two-level lazy update (3xTF32 path): after each
// 128-column block only the rest of its outer block is updated; after each
// outer block one GEMM with K = OUTER updates all columns to its right.
constexpr int OUTER = 1024;

// Workspace: per lane (one setting being solved at a time) the errors (E^T
// of one block for the fp32 path, or E of one outer block split in two for
// 3xTF32), then, shared by the lanes, Uc^T split in two (3xTF32 only: the
// tensor-core product reads its B operand transposed).
struct QuantWs {
  float *ET, *Eb, *Es, *Ub, *Us;
  int64_t ldu;
};

// Most settings kq_quantize_layer_multi solves side by side (when their
// outputs are not stacked); the workspace size serves both forms.
constexpr int kMaxLanes = 4;
static_assert(kMaxLanes == kMaxStack, "one workspace size for lanes and stacks");

size_t quant_layout(int64_t d_out, int64_t d_in, int lanes, int lane, QuantWs* w, void* base) {
  const int64_t ldu = (d_in + 3) / 4 * 4;
  const size_t se = kq::align_up((size_t)d_out * OUTER * sizeof(float), 256);
  const size_t su = kq::align_up((size_t)d_in * ldu * sizeof(float), 256);
  if (w && base) {
    char* b = static_cast<char*>(base);
    w->ET = reinterpret_cast<float*>(b + 2 * se * lane);
    w->Eb = w->ET;
    w->Es = reinterpret_cast<float*>(b + 2 * se * lane + se);
    w->Ub = reinterpret_cast<float*>(b + 2 * se * lanes);
    w->Us = reinterpret_cast<float*>(b + 2 * se * lanes + su);
    w->ldu = ldu;
  }
  return 2 * se * lanes + 2 * su;
}

// The workspace of a stacked solve of `count` settings: their errors as one
// [count d_out, OUTER] matrix (tf32 part, then remainder), then the split of
// Uc^T; the same size as `count` lanes side by side.
size_t stack_layout(int64_t d_out, int64_t d_in, int count, QuantWs* w, void* base) {
  const int64_t ldu = (d_in + 3) / 4 * 4;
  const size_t se = kq::align_up((size_t)d_out * OUTER * sizeof(float), 256);
  const size_t su = kq::align_up((size_t)d_in * ldu * sizeof(float), 256);
  if (w && base) {
    char* b = static_cast<char*>(base);
    w->ET = reinterpret_cast<float*>(b);
    w->Eb = w->ET;
    w->Es = reinterpret_cast<float*>(b + se * count);
    w->Ub = reinterpret_cast<float*>(b + 2 * se * count);
    w->Us = reinterpret_cast<float*>(b + 2 * se * count + su);
    w->ldu = ldu;
  }
  return 2 * se * count + 2 * su;
}

}  // namespace

extern "C" size_t kq_quantize_layer_workspace_size(int64_t d_out, int64_t d_in, int block) {
  (void)block;
  if (d_out < 1 || d_in < 1) return 0;
  return quant_layout(d_out, d_in, 1, 0, nullptr, nullptr);
}

extern "C" size_t kq_quantize_layer_multi_workspace_size(int64_t d_out, int64_t d_in, int block, int count) {
  (void)block;
  if (d_out < 1 || d_in < 1 || count < 1) return 0;
  return quant_layout(d_out, d_in, std::min(count, kMaxLanes), 0, nullptr, nullptr);
}

namespace {

// Host-side checks of one setting (nothing is enqueued).
kq_status check_args(const float* W, int64_t d_out, int64_t d_in, int64_t ldw, const float* Uc, int64_t lduc, int bits,
                     int group, int block, int gemm_mode, const uint8_t* codes, int64_t ldq, const float* scales,
                     const float* zeros, const float* W_hat, int64_t ldwh, const int32_t* info) {
  if (!W || !Uc || !codes || !scales || !zeros || !W_hat || !info)
    return kq::fail(KQ_ERR_INVALID_ARG, "kq_quantize_layer: NULL pointer");
  if (d_out < 1 || d_in < 1 || d_in > 65536) return kq::fail(KQ_ERR_UNSUPPORTED_SHAPE, "kq_quantize_layer: sizes");
  if (d_out > (int64_t)0x7fffffff / 2) return kq::fail(KQ_ERR_UNSUPPORTED_SHAPE, "kq_quantize_layer: d_out too large");
  if (ldw < d_in || lduc < d_in || ldq < d_in || ldwh < d_in)
    return kq::fail(KQ_ERR_INVALID_ARG, "kq_quantize_layer: leading dimension too small");
  if (bits < 2 || bits > 8) return kq::fail(KQ_ERR_INVALID_ARG, "kq_quantize_layer: bits outside 2..8");
  if (block != BLK) return kq::fail(KQ_ERR_UNSUPPORTED_SHAPE, "kq_quantize_layer: only block = 128 is built");
  if (group < 0 || (group && (group % 32 || BLK % group)))
    return kq::fail(KQ_ERR_UNSUPPORTED_SHAPE, "kq_quantize_layer: group must be 0 or a multiple of 32 dividing 128");
  if (gemm_mode != KQ_GEMM_FP32 && gemm_mode != KQ_GEMM_3XTF32)
    return kq::fail(KQ_ERR_INVALID_ARG, "kq_quantize_layer: gemm_mode must be KQ_GEMM_FP32 or KQ_GEMM_3XTF32");
  if (W == W_hat) return kq::fail(KQ_ERR_INVALID_ARG, "kq_quantize_layer: W and W_hat must not alias");
  if (!kq::aligned(W, 16) || !kq::aligned(W_hat, 16) || !kq::aligned(Uc, 16) || (ldw & 3) || (ldwh & 3) || (lduc & 3))
    return kq::fail(KQ_ERR_ALIGNMENT, "kq_quantize_layer: W, W_hat, Uc need 16-byte alignment and ld %% 4 == 0");
  // the in-block kernel stores four codes at a time
  if (!kq::aligned(codes, 4) || (ldq & 3))
    return kq::fail(KQ_ERR_ALIGNMENT, "kq_quantize_layer: codes need 4-byte alignment and ldq %% 4 == 0");
  return KQ_OK;
}

// One setting as the caller passes it.
struct SetOut {
  int bits, group;
  uint8_t* codes;
  float* scales;
  float* zeros;
};

// Enqueues `count` (<= kMaxStack) checked settings on `st` as one stacked
// solve: setting i's rows of W_hat start at W_hat + i d_out ldwh, its
// errors at row i d_out of the workspace's E, and every launch covers all
// the settings (M = count d_out in the trailing updates, whose first
// super-block reads W for every setting).  The tf32 split of Uc^T (3xTF32
// mode) is formed here unless `split_uc` is false (then it is already in the
// workspace).  The fp32 SIMT mode solves one setting per call (count == 1).
kq_status enqueue_stacked(const float* W, int64_t d_out, int64_t d_in, int64_t ldw, const float* Uc, int64_t lduc,
                          const uint8_t* dead_mask, int count, const SetOut* so, int gemm_mode, int64_t ldq,
                          float* W_hat, int64_t ldwh, const QuantWs& w, int32_t* info, cudaStream_t st,
                          bool split_uc) {
  const bool tc = (gemm_mode == KQ_GEMM_3XTF32);
  if (count < 1 || count > kMaxStack || (!tc && count != 1))
    return kq::fail(KQ_ERR_INVALID_ARG, "kq_quantize_layer: a stacked solve of %d settings", count);
  if (tc && split_uc) KQ_TRY(kq::split_tf32(Uc, lduc, nullptr, 0, d_in, d_in, w.Ub, w.Us, w.ldu, true, st));
  const int64_t M = count * d_out;
  const int64_t wh_set = d_out * ldwh;

  SetArgs sets[kMaxStack] = {};
  GridSets gs = {};
  for (int i = 0; i < count; ++i) {
    sets[i].codes = so[i].codes;
    sets[i].scales = so[i].scales;
    sets[i].zeros = so[i].zeros;
    sets[i].group = so[i].group;
    sets[i].n_groups = so[i].group ? kq::cdiv(d_in, so[i].group) : 1;
    sets[i].nl = (float)((1 << so[i].bits) - 1);
    if (!so[i].group) {
      gs.nl[gs.count] = sets[i].nl;
      gs.scales[gs.count] = so[i].scales;
      gs.zeros[gs.count] = so[i].zeros;
      ++gs.count;
    }
  }
  if (gs.count) {
    KQ_TRY(timed(kClassGrid, 0.0, 4.0 * d_out * d_in, st, [&]() -> kq_status {
      grid_rows_kernel<<<(unsigned)kq::cdiv(d_out, 8), 256, 0, st>>>(W, ldw, d_out, d_in, dead_mask, gs, info);
      return kq::launch_check("kq_quantize_layer grid");
    }));
  }
  const bool stacked_rows = M >= kStackedRows;
  auto ib_kernel = stacked_rows ? inblock_kernel<kLanesPerRow, 256> : inblock_kernel<kLanesPerRow, 224>;
  const int ib_threads = stacked_rows ? 256 : 224;
  KQ_TRY(kq::cuda_check(cudaFuncSetAttribute(ib_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, IB_SMEM),
                        "kq_quantize_layer: smem attribute"));
  auto inblock = [&](int64_t i0, int64_t o0) -> kq_status {
    const int bw = (int)std::min<int64_t>(BLK, d_in - i0);
    const bool first = (i0 == 0);
    InblockArgs a = {};
    a.src = first ? W : W_hat;
    a.ld_src = first ? ldw : ldwh;
    a.src_set = first ? 0 : wh_set;
    a.W_hat = W_hat;
    a.ldwh = ldwh;
    a.wh_set = wh_set;
    a.Uc = Uc;
    a.lduc = lduc;
    a.dead = first ? dead_mask : nullptr;
    a.d_out = d_out;
    a.d_in = d_in;
    a.i0 = i0;
    a.bw = bw;
    a.ldq = ldq;
    a.ET = w.ET;
    a.Eb = tc ? w.Eb : nullptr;
    a.Es = tc ? w.Es : nullptr;
    a.ldE = OUTER;
    a.e_col0 = i0 - o0;
    a.info = info;
    for (int i = 0; i < count; ++i) a.set[i] = sets[i];
    // after the first block the previous kernel is this solve's own trailing
    // update, so the launch may overlap its tail (tensor-core mode)
    return timed(kClassInblock, 0.0, (double)M * bw * (tc ? 17.0 : 13.0), st, [&]() {
      return kq::launch_ex("kq_quantize_layer inblock", tc && i0 > 0, ib_kernel,
                           dim3((unsigned)kq::cdiv(d_out, ib_threads / kLanesPerRow), (unsigned)count),
                           dim3(ib_threads), IB_SMEM, st, a);
    });
  };
  // W_hat[:, c0:c0+N] = src[:, c0:c0+N] - E[:, e0:e0+K] Uc[k0:k0+K, c0:c0+N] over
  // the stacked rows; the source is W (dead columns as zeros, row r of every
  // setting reading W's row r mod d_out) while those columns are untouched.
  auto update = [&](int64_t c0, int64_t N, int64_t e0, int64_t k0, int64_t K, bool from_w) -> kq_status {
    kq::Gemm3xTF32 g;
    g.M = M;
    g.N = N;
    g.K = K;
    g.a_big = w.Eb;
    g.a_small = w.Es;
    g.lda = OUTER;
    g.a_col0 = e0;
    g.bt_big = w.Ub;         // Uc^T: (k, n) of Uc[k0:, c0:] at Ut[c0 + n][k0 + k]
    g.bt_small = w.Us;
    g.ldbt = w.ldu;
    g.bt_row0 = c0;
    g.bt_col0 = k0;
    g.epilogue = kq::kEpiSubtract;
    g.C = W_hat + c0;
    g.ldc = ldwh;
    g.src = (from_w ? W : W_hat) + c0;
    g.ld_src = from_w ? ldw : ldwh;
    g.src_rows = from_w ? d_out : 0;
    g.dead = from_w && dead_mask ? dead_mask + c0 : nullptr;
    g.info = info;
    g.pdl = true;   // always follows this solve's in-block kernel
    // with stacked settings the next in-block kernel may be scheduled early
    // (it copies its block of Uc, which no kernel of the solve writes, while
    // this product drains; measured 2.72 -> 2.67 ms for three attn4096 solves)
    g.trigger_early = count > 1;
    return timed(kClassUpdate, 2.0 * M * N * K, 0.0, st, [&]() { return kq::gemm_3xtf32(g, st); });
  };
  if (!tc) {
    for (int64_t i0 = 0; i0 < d_in; i0 += BLK) {
      const int bw = (int)std::min<int64_t>(BLK, d_in - i0);
      const bool first = (i0 == 0);
      KQ_TRY(inblock(i0, i0));
      const int64_t cstart = i0 + bw;
      if (cstart < d_in) {
        dim3 grid((unsigned)kq::cdiv(d_in - cstart, TN), (unsigned)kq::cdiv(d_out, TM));
        KQ_TRY(timed(kClassUpdate, 2.0 * d_out * bw * (d_in - cstart), 0.0, st, [&]() -> kq_status {
          trailing_fp32_kernel<<<grid, 256, 0, st>>>(first ? W : W_hat, first ? ldw : ldwh, W_hat, ldwh, w.ET, Uc,
                                                    lduc, first ? dead_mask : nullptr, d_out, d_in, i0, bw, cstart);
          return kq::launch_check("kq_quantize_layer trailing");
        }));
      }
    }
  } else {
    for (int64_t o0 = 0; o0 < d_in; o0 += OUTER) {
      const int64_t o1 = std::min<int64_t>(o0 + OUTER, d_in);
      for (int64_t i0 = o0; i0 < o1; i0 += BLK) {
        const int64_t bw = std::min<int64_t>(BLK, d_in - i0);
        KQ_TRY(inblock(i0, o0));
        if (i0 + bw < o1) KQ_TRY(update(i0 + bw, o1 - (i0 + bw), i0 - o0, i0, bw, i0 == 0));
      }
      if (o1 < d_in) KQ_TRY(update(o1, d_in - o1, 0, o0, o1 - o0, o0 == 0));
    }
  }
  kq::clear_error();
  return KQ_OK;
}

}  // namespace

namespace {

// Streams and events for solving settings side by side: created on first
// use by each host thread for each device, kept for the thread's lifetime.
struct Lanes {
  int device = -1;
  cudaStream_t s[kMaxLanes - 1] = {};
  cudaEvent_t fork = nullptr;
  cudaEvent_t join[kMaxLanes - 1] = {};
};

kq_status side_lanes(Lanes** out) {
  thread_local Lanes cache[16];
  int dev = 0;
  KQ_TRY(kq::cuda_check(cudaGetDevice(&dev), "kq_quantize_layer_multi: cudaGetDevice"));
  Lanes* l = nullptr;
  for (auto& c : cache)
    if (c.device == dev) l = &c;
  if (!l) {
    for (auto& c : cache)
      if (c.device < 0) {
        l = &c;
        break;
      }
    if (!l) return kq::fail(KQ_ERR_UNSUPPORTED_SHAPE, "kq_quantize_layer_multi: more than 16 devices");
    for (auto& st : l->s)
      KQ_TRY(kq::cuda_check(cudaStreamCreateWithFlags(&st, cudaStreamNonBlocking), "kq_quantize_layer_multi: stream"));
    KQ_TRY(kq::cuda_check(cudaEventCreateWithFlags(&l->fork, cudaEventDisableTiming), "kq_quantize_layer_multi: event"));
    for (auto& e : l->join)
      KQ_TRY(kq::cuda_check(cudaEventCreateWithFlags(&e, cudaEventDisableTiming), "kq_quantize_layer_multi: event"));
    l->device = dev;
  }
  *out = l;
  return KQ_OK;
}

}  // namespace

extern "C" kq_status kq_quantize_layer(const float* W, int64_t d_out, int64_t d_in, int64_t ldw, const float* Uc,
                                       int64_t lduc, const uint8_t* dead_mask, int bits, int group, int block,
                                       int gemm_mode, uint8_t* codes, int64_t ldq, float* scales, float* zeros,
                                       float* W_hat, int64_t ldwh, void* ws, size_t ws_bytes, int32_t* info,
                                       kq_stream_t stream) {
  KQ_TRY(check_args(W, d_out, d_in, ldw, Uc, lduc, bits, group, block, gemm_mode, codes, ldq, scales, zeros, W_hat,
                    ldwh, info));
  if (!ws || !kq::aligned(ws, 256) || ws_bytes < kq_quantize_layer_workspace_size(d_out, d_in, block))
    return kq::fail(KQ_ERR_WORKSPACE, "kq_quantize_layer: workspace too small or not 256-byte aligned");
  QuantWs w;
  stack_layout(d_out, d_in, 1, &w, ws);
  const SetOut so = {bits, group, codes, scales, zeros};
  return enqueue_stacked(W, d_out, d_in, ldw, Uc, lduc, dead_mask, 1, &so, gemm_mode, ldq, W_hat, ldwh, w, info,
                         (cudaStream_t)stream, true);
}

extern "C" kq_status kq_quantize_layer_multi(const float* W, int64_t d_out, int64_t d_in, int64_t ldw,
                                             const float* Uc, int64_t lduc, const uint8_t* dead_mask, int count,
                                             const int* bits, const int* group, int block, int gemm_mode,
                                             uint8_t* const* codes, int64_t ldq, float* const* scales,
                                             float* const* zeros, float* const* W_hat, int64_t ldwh, void* ws,
                                             size_t ws_bytes, int32_t* info, kq_stream_t stream) {
  if (count < 1 || !bits || !group || !codes || !scales || !zeros || !W_hat)
    return kq::fail(KQ_ERR_INVALID_ARG, "kq_quantize_layer_multi: count < 1 or NULL array");
  // every setting is checked before any work is enqueued
  for (int i = 0; i < count; ++i) {
    KQ_TRY(check_args(W, d_out, d_in, ldw, Uc, lduc, bits[i], group[i], block, gemm_mode, codes[i], ldq, scales[i],
                      zeros[i], W_hat[i], ldwh, info));
    for (int j = 0; j < i; ++j)
      if (codes[j] == codes[i] || scales[j] == scales[i] || zeros[j] == zeros[i] || W_hat[j] == W_hat[i])
        return kq::fail(KQ_ERR_INVALID_ARG, "kq_quantize_layer_multi: settings %d and %d share an output", j, i);
  }
  if (!ws || !kq::aligned(ws, 256))
    return kq::fail(KQ_ERR_WORKSPACE, "kq_quantize_layer_multi: workspace NULL or not 256-byte aligned");
  cudaStream_t st = (cudaStream_t)stream;
  std::vector<SetOut> so(count);
  for (int i = 0; i < count; ++i) so[i] = SetOut{bits[i], group[i], codes[i], scales[i], zeros[i]};
  // Stacked when the settings' W_hat buffers follow one another (setting i
  // at W_hat[0] + i d_out ldwh) and the trailing updates run on the tensor
  // cores: up to kMaxStack settings per solve, every launch covering all
  // of them.
  bool stacked = gemm_mode == KQ_GEMM_3XTF32 && (int64_t)std::min(count, kMaxStack) * d_out <= INT32_MAX;
  for (int i = 1; i < count && stacked; ++i) stacked = (W_hat[i] == W_hat[0] + (int64_t)i * d_out * ldwh);
  if (stacked) {
    int per = std::min(count, kMaxStack);
    while (per > 1 && ws_bytes < stack_layout(d_out, d_in, per, nullptr, nullptr)) --per;
    if (ws_bytes < stack_layout(d_out, d_in, per, nullptr, nullptr))
      return kq::fail(KQ_ERR_WORKSPACE, "kq_quantize_layer_multi: workspace too small");
    QuantWs sw;
    stack_layout(d_out, d_in, per, &sw, ws);
    for (int i0 = 0; i0 < count; i0 += per)
      KQ_TRY(enqueue_stacked(W, d_out, d_in, ldw, Uc, lduc, dead_mask, std::min(per, count - i0), so.data() + i0,
                             gemm_mode, ldq, W_hat[i0], ldwh, sw, info, st, i0 == 0));
    return KQ_OK;
  }
  // otherwise side by side when the workspace holds a lane per setting (up
  // to kMaxLanes), else one after the other in a single lane
  int lanes = std::min(count, kMaxLanes);
  if (ws_bytes < quant_layout(d_out, d_in, lanes, 0, nullptr, nullptr)) lanes = 1;
  if (ws_bytes < quant_layout(d_out, d_in, lanes, 0, nullptr, nullptr))
    return kq::fail(KQ_ERR_WORKSPACE, "kq_quantize_layer_multi: workspace too small");
  QuantWs w[kMaxLanes];
  for (int l = 0; l < lanes; ++l) quant_layout(d_out, d_in, lanes, l, &w[l], ws);
  if (lanes == 1) {
    for (int i = 0; i < count; ++i)
      KQ_TRY(enqueue_stacked(W, d_out, d_in, ldw, Uc, lduc, dead_mask, 1, &so[i], gemm_mode, ldq, W_hat[i], ldwh, w[0],
                             info, st, i == 0));
    return KQ_OK;
  }
  Lanes* L = nullptr;
  KQ_TRY(side_lanes(&L));
  // the shared split of Uc^T on the caller's stream, then the fork
  if (gemm_mode == KQ_GEMM_3XTF32)
    KQ_TRY(kq::split_tf32(Uc, lduc, nullptr, 0, d_in, d_in, w[0].Ub, w[0].Us, w[0].ldu, true, st));
  KQ_TRY(kq::cuda_check(cudaEventRecord(L->fork, st), "kq_quantize_layer_multi: record"));
  for (int l = 1; l < lanes; ++l)
    KQ_TRY(kq::cuda_check(cudaStreamWaitEvent(L->s[l - 1], L->fork, 0), "kq_quantize_layer_multi: wait"));
  kq_status first = KQ_OK;
  for (int i = 0; i < count && first == KQ_OK; ++i) {
    const int l = i % lanes;
    first = enqueue_stacked(W, d_out, d_in, ldw, Uc, lduc, dead_mask, 1, &so[i], gemm_mode, ldq, W_hat[i], ldwh, w[l],
                            info, l ? L->s[l - 1] : st, false);
  }
  // the join is enqueued even after a failed launch, so that the caller's
  // stream is ordered after everything that did get enqueued
  for (int l = 1; l < lanes; ++l) {
    cudaError_t e = cudaEventRecord(L->join[l - 1], L->s[l - 1]);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(st, L->join[l - 1], 0);
    if (e != cudaSuccess && first == KQ_OK) first = kq::cuda_check(e, "kq_quantize_layer_multi: join");
  }
  if (first != KQ_OK) return first;
  kq::clear_error();
  return KQ_OK;
}

extern "C" kq_status kq_solver_timing(int enable, kq_solver_times* out) {
  if (enable) {
    g_timing.on = true;
    return KQ_OK;
  }
  g_timing.on = false;
  kq_solver_times t = {};
  kq_status st = KQ_OK;
  for (const TimedLaunch& r : g_timing.recs) {
    float ms = 0.f;
    if (st == KQ_OK) {
      st = kq::cuda_check(cudaEventSynchronize(r.b), "kq_solver_timing: synchronize");
      if (st == KQ_OK) st = kq::cuda_check(cudaEventElapsedTime(&ms, r.a, r.b), "kq_solver_timing: elapsed");
    }
    if (r.cls == kClassGrid) {
      t.grid_ms += ms;
      ++t.grid_launches;
    } else if (r.cls == kClassInblock) {
      t.inblock_ms += ms;
      ++t.inblock_launches;
      t.inblock_bytes += r.bytes;
    } else {
      t.update_ms += ms;
      ++t.update_launches;
      t.update_flops += r.flops;
    }
    g_timing.pool.push_back(r.a);
    g_timing.pool.push_back(r.b);
  }
  g_timing.recs.clear();
  if (out) *out = t;
  if (st == KQ_OK) kq::clear_error();
  return st;
}
