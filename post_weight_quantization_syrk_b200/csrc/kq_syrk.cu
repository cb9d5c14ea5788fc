// kq_accum_cov: C (+)= alpha * A^T A from bf16 tokens-by-channels A (a1/a2).
//
// KronQ review (romaanj.github.io/reviews/kronq), Background: H_X (input
// activations) and H_G (output gradients, E[g g^T] per the research thread)
// are the two Kronecker factors of the layer Hessian.
//
// B200 design (tcgen05 + TMEM + TMA):
//  * Output tiles are 256x256 blocks of the lower triangle (diagonal blocks
//    are computed whole, only their lower half is written).  A tile is two
//    M=128 x N=256 bf16 MMAs per 16 tokens, accumulating in fp32 in TMEM: the
//    two accumulators fill all 512 TMEM columns of the SM.
//  * X is [tokens, channels] row-major, so both MMA operands are MN-major:
//    TMA copies boxes of 64 tokens x 64 channels (128-byte rows, 128-byte
//    swizzle) and the shared-memory descriptors walk 64-channel atoms with the
//    leading offset and 8-token groups with the stride offset.  A diagonal tile
//    loads its channels once and uses them for both operands.
//  * One persistent CTA per SM walks work units (tile, token split); the
//    splits of one tile are far apart in the walk while tiles sharing a token
//    range run side by side, so X streams through L2 about once per wave.
//  * Warp roles: warp 0 issues TMA (3-stage ring of 64 KB stages guarded by
//    mbarriers), warp 1 allocates TMEM and one of its threads issues the
//    MMAs, warps 2-5 drain TMEM with tcgen05.ld and write C (or an fp32
//    partial tile when the tokens are split; a second kernel then sums the
//    splits in a fixed order, so results do not depend on scheduling).
//  * Every mbarrier wait is bounded by a time limit; on expiry the kernel
//    records KQ_ERR_TIMEOUT, lets its own copies and MMAs drain (again
//    bounded), frees TMEM and returns.
#include <cuda.h>
#include <cuda_bf16.h>

#include <algorithm>
#include <cmath>

#include "kq_tc.cuh"

namespace {

constexpr int TILE = 256;                 // output tile (rows and columns)
constexpr int BK = 64;                    // tokens per pipeline stage
constexpr int STAGES = 3;
constexpr int BOX_BYTES = 64 * 64 * 2;    // one TMA box: 64 tokens x 64 channels bf16
constexpr int OPER_BYTES = 4 * BOX_BYTES; // 256 channels x 64 tokens
constexpr int STAGE_BYTES = 2 * OPER_BYTES;
constexpr int THREADS = 192;
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 /*align*/ + 256 /*barriers*/;
constexpr int ASSUMED_SMS = 148;          // the B200's SM count, used to size splits

// Instruction descriptor, kind::f16: D fp32, A/B bf16, both MN-major, M=128, N=256.
constexpr uint32_t IDESC = kq::tc::idesc(kq::tc::kFmtBF16, 1, 1, 128, 256);

struct Params {
  int64_t n, d;
  int T;            // tiles per dimension
  int num_tiles;    // T (T + 1) / 2
  int splits;       // token splits per tile
  int kb_per_split; // 64-token blocks per split
  int kblocks;      // total 64-token blocks
  int num_units;    // num_tiles * splits
  float alpha;
  int accumulate;
  float* C;
  int64_t ldc;
  int c_vec;        // C rows 16-byte aligned (C aligned, ldc % 4 == 0)
  float* partial;   // [splits][num_tiles][256][256] when splits > 1
  int kt;           // block-diagonal mode: tiles per diagonal block side (0: whole lower triangle)
  int tiles_per_block;  // kt (kt + 1) / 2
  int64_t blk;      // block-diagonal mode: block size k = 256 kt; C is [d, k], block b in rows b k ..
  int32_t* info;
  unsigned long long wait_ns;   // limit of each pipeline wait (kq_set_wait_limit_ns)
};

using namespace kq::tc;

// Shared-memory descriptor of an MN-major 128-byte-swizzled operand: the
// leading offset steps to the next 64-channel TMA box, the stride offset to
// the next 8 tokens (8 rows of 128 bytes).
__device__ __forceinline__ uint64_t operand_desc(uint32_t addr) {
  return smem_desc(addr, BOX_BYTES, 1024, kSwizzle128);
}

__device__ __forceinline__ void tri_index(int64_t l, int* ti, int* tj) {
  int64_t t = (int64_t)((sqrt(8.0 * (double)l + 1.0) - 1.0) * 0.5);
  while (t * (t + 1) / 2 > l) --t;
  while ((t + 1) * (t + 2) / 2 <= l) ++t;
  *ti = (int)t;
  *tj = (int)(l - t * (t + 1) / 2);
}

// Tile number -> (tile row, tile column): the lower triangle of the whole
// matrix, or (block-diagonal mode) the lower triangles of the diagonal
// blocks one after the other.
__device__ __forceinline__ void tile_coords(const Params& p, int l, int* ti, int* tj) {
  if (p.kt) {
    const int b = l / p.tiles_per_block;
    tri_index(l % p.tiles_per_block, ti, tj);
    *ti += b * p.kt;
    *tj += b * p.kt;
  } else {
    tri_index(l, ti, tj);
  }
}

// Column of element (row gi, column gj <= gi of the same block) in C: the
// block-diagonal mode stores each block's rows from column 0.
__device__ __forceinline__ int64_t c_col(const Params& p, int64_t gi, int64_t gj) {
  return p.kt ? gj - (gi / p.blk) * p.blk : gj;
}

// unit -> (tile, split); units of the same split are adjacent.
__device__ __forceinline__ void unit_coords(const Params& p, int u, int* ti, int* tj, int* split) {
  *split = u / p.num_tiles;
  tile_coords(p, u % p.num_tiles, ti, tj);
}

// ------------------------------------------------------------------ kernel

__global__ void __launch_bounds__(THREADS, 1) syrk_tc_kernel(const __grid_constant__ CUtensorMap tmap, Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES);
  // bars[0..S): full, [S..2S): empty, [2S]: acc full, [2S+1]: acc empty, [2S+2]: mma drained
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 3);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const uint32_t full0 = smem_u32(bars), empty0 = smem_u32(bars + STAGES);
  const uint32_t accfull = smem_u32(bars + 2 * STAGES), accempty = smem_u32(bars + 2 * STAGES + 1);
  const uint32_t drained = smem_u32(bars + 2 * STAGES + 2);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, 1);
    }
    mbar_init(accfull, 1);
    mbar_init(accempty, 128);
    mbar_init(drained, 1);
    *abort_flag = 0;
    mbar_init_fence();
    prefetch_map(&tmap);
  }
  if (warp == 1) tmem_alloc<512>(smem_u32(tmem_slot));
  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ---------------- TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued_phase[STAGES];
      bool issued[STAGES];
      for (int s = 0; s < STAGES; ++s) issued[s] = false;
      bool ok = true;
      for (int u = blockIdx.x; u < p.num_units && ok; u += gridDim.x) {
        int ti, tj, sp;
        unit_coords(p, u, &ti, &tj, &sp);
        const int kb0 = sp * p.kb_per_split;
        const int kb1 = min(p.kblocks, kb0 + p.kb_per_split);
        const bool diag = (ti == tj);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(empty0 + 8 * stage, phase ^ 1u, abort_flag, p.info, 1, p.wait_ns)) {
            ok = false;
            break;
          }
          const uint32_t fb = full0 + 8 * stage;
          mbar_arrive_expect_tx(fb, diag ? OPER_BYTES : STAGE_BYTES);
          const uint32_t sa = smem_u32(smem + stage * STAGE_BYTES);
          const int y = kb * BK;
#pragma unroll
          for (int q = 0; q < 4; ++q) tma_load_2d(sa + q * BOX_BYTES, &tmap, ti * TILE + 64 * q, y, fb);
          if (!diag) {
#pragma unroll
            for (int q = 0; q < 4; ++q) tma_load_2d(sa + OPER_BYTES + q * BOX_BYTES, &tmap, tj * TILE + 64 * q, y, fb);
          }
          issued[stage] = true;
          issued_phase[stage] = phase;
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {
        // let this CTA's own copies land before the CTA can exit
        for (int s = 0; s < STAGES; ++s)
          if (issued[s]) mbar_drain(full0 + 8 * s, issued_phase[s]);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool ok = true, any = false;
      for (int u = blockIdx.x; u < p.num_units && ok; u += gridDim.x) {
        int ti, tj, sp;
        unit_coords(p, u, &ti, &tj, &sp);
        const int kb0 = sp * p.kb_per_split;
        const int kb1 = min(p.kblocks, kb0 + p.kb_per_split);
        const bool diag = (ti == tj);
        if (!mbar_wait(accempty, acc_phase ^ 1u, abort_flag, p.info, 2, p.wait_ns)) {
          ok = false;
          break;
        }
        fence_after();
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(full0 + 8 * stage, phase, abort_flag, p.info, 3, p.wait_ns)) {
            ok = false;
            break;
          }
          fence_after();
          const uint32_t sa = smem_u32(smem + stage * STAGE_BYTES);
          const uint32_t sb = diag ? sa : sa + OPER_BYTES;
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {
            const uint32_t acc = (kb > kb0 || k > 0) ? 1u : 0u;
            const uint64_t db = operand_desc(sb + k * 2048);
            mma_f16<IDESC>(tmem, operand_desc(sa + k * 2048), db, acc);                    // rows 0..127
            mma_f16<IDESC>(tmem + 256, operand_desc(sa + 2 * BOX_BYTES + k * 2048), db, acc);  // rows 128..255
          }
          any = true;
          mma_commit(empty0 + 8 * stage);   // stage is free once these MMAs have read it
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        mma_commit(accfull);               // accumulators complete for this unit
        acc_phase ^= 1u;
      }
      if (any) {
        // every MMA this thread issued has completed before TMEM is released
        mma_commit(drained);
        mbar_drain(drained, 0);
      }
    }
  } else {
    // ---------------- epilogue: warps 2..5 drain TMEM lanes 32*(warp%4) ..
    const int wq = warp & 3;
    const int row_in_half = 32 * wq + lane;
    uint32_t acc_phase = 0;
    for (int u = blockIdx.x; u < p.num_units; u += gridDim.x) {
      int ti, tj, sp;
      unit_coords(p, u, &ti, &tj, &sp);
      // one lane waits, the warp follows: every lane leaves together on abort
      bool ready = true;
      if (lane == 0) ready = mbar_wait(accfull, acc_phase, abort_flag, p.info, 4, p.wait_ns);
      if (!__shfl_sync(0xffffffffu, ready ? 1 : 0, 0)) break;
      __syncwarp();
      fence_after();
      const int64_t i0 = (int64_t)ti * TILE, j0 = (int64_t)tj * TILE;
      const bool diag = (ti == tj);
#pragma unroll 1
      for (int half = 0; half < 2; ++half) {
        const int r = half * 128 + row_in_half;
        const int64_t gi = i0 + r;
#pragma unroll 1
        for (int c0 = 0; c0 < TILE; c0 += 16) {
          float v[16];
          tmem_ld16(tmem + ((uint32_t)(32 * wq) << 16) + (uint32_t)(half * 256 + c0), v);
          if (p.splits > 1) {
            float* dst = p.partial + (((int64_t)sp * p.num_tiles + (u % p.num_tiles)) * TILE + r) * TILE + c0;
#pragma unroll
            for (int q = 0; q < 16; q += 4)
              *reinterpret_cast<float4*>(dst + q) = make_float4(v[q], v[q + 1], v[q + 2], v[q + 3]);
          } else if (gi < p.d && (!diag || c0 <= r)) {
#pragma unroll
            for (int q = 0; q < 16; ++q) {
              const int64_t gj = j0 + c0 + q;
              if (gj >= p.d || gj > gi) continue;
              float val = p.alpha * v[q];
              if (p.accumulate) val += p.C[gi * p.ldc + c_col(p, gi, gj)];
              if (!isfinite(val)) kq::report(p.info, KQ_ERR_NONFINITE, gi);
              p.C[gi * p.ldc + c_col(p, gi, gj)] = val;
              p.C[gj * p.ldc + c_col(p, gj, gi)] = val;
            }
          }
        }
      }
      fence_before();
      mbar_arrive(accempty);
      acc_phase ^= 1u;
    }
  }

  fence_before();
  __syncthreads();
  if (warp == 1) {
    fence_after();
    tmem_dealloc<512>(tmem);
  }
}

// Sum the token splits of every lower tile in split order (s = 0, then
// s += split 0, 1, ... in fp32), apply alpha (and the old C when
// accumulating), write the lower element and its mirror.  One CTA per
// (tile, 32-row band); per 128-column half each of the 8 warps owns 4 rows
// and each lane 4 adjacent columns, so the partials stream in as float4
// loads, the four rows' loads of two splits in flight together; the mirror
// goes through a shared-memory transpose so both writes are coalesced.
__global__ void __launch_bounds__(256) split_reduce_kernel(Params p) {
  __shared__ float t[32][129];
  const int tile = blockIdx.x / 8;
  const int band = blockIdx.x % 8;  // 32-row band within the 256-row tile
  int ti, tj;
  tile_coords(p, tile, &ti, &tj);
  const int64_t i0 = (int64_t)ti * TILE + band * 32, j0 = (int64_t)tj * TILE;
  const int lane = threadIdx.x % 32, warp = threadIdx.x / 32;
  const int64_t split_stride = (int64_t)p.num_tiles * TILE * TILE;
  for (int h = 0; h < 2; ++h) {
    const int cl = h * 128 + 4 * lane;   // first of this lane's 4 columns in the tile
    const float* src = p.partial + ((int64_t)tile * TILE + band * 32 + warp) * TILE + cl;
    float acc[4][4];
#pragma unroll
    for (int k = 0; k < 4; ++k)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[k][e] = 0.f;
    int sp = 0;
    for (; sp + 1 < p.splits; sp += 2) {
      float4 v0[4], v1[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) v0[k] = *reinterpret_cast<const float4*>(src + sp * split_stride + 8 * k * TILE);
#pragma unroll
      for (int k = 0; k < 4; ++k)
        v1[k] = *reinterpret_cast<const float4*>(src + (sp + 1) * split_stride + 8 * k * TILE);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        acc[k][0] += v0[k].x;
        acc[k][1] += v0[k].y;
        acc[k][2] += v0[k].z;
        acc[k][3] += v0[k].w;
        acc[k][0] += v1[k].x;
        acc[k][1] += v1[k].y;
        acc[k][2] += v1[k].z;
        acc[k][3] += v1[k].w;
      }
    }
    if (sp < p.splits) {
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float4 v = *reinterpret_cast<const float4*>(src + sp * split_stride + 8 * k * TILE);
        acc[k][0] += v.x;
        acc[k][1] += v.y;
        acc[k][2] += v.z;
        acc[k][3] += v.w;
      }
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int rr = warp + 8 * k;
      const int64_t gi = i0 + rr, gj = j0 + cl;
      float v[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) v[e] = p.alpha * acc[k][e];
      if (gi < p.d) {
        float* c = p.C + gi * p.ldc + c_col(p, gi, gj);
        if (p.c_vec && gj + 3 < p.d && gj + 3 <= gi) {
          if (p.accumulate) {
            const float4 o = *reinterpret_cast<const float4*>(c);
            v[0] += o.x;
            v[1] += o.y;
            v[2] += o.z;
            v[3] += o.w;
          }
          if (!(isfinite(v[0]) && isfinite(v[1]) && isfinite(v[2]) && isfinite(v[3])))
            kq::report(p.info, KQ_ERR_NONFINITE, gi);
          *reinterpret_cast<float4*>(c) = make_float4(v[0], v[1], v[2], v[3]);
        } else {
#pragma unroll
          for (int e = 0; e < 4; ++e)
            if (gj + e < p.d && gj + e <= gi) {
              if (p.accumulate) v[e] += c[e];
              if (!isfinite(v[e])) kq::report(p.info, KQ_ERR_NONFINITE, gi);
              c[e] = v[e];
            }
        }
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) t[rr][4 * lane + e] = v[e];
    }
    __syncthreads();
    // mirror: row j0 + h * 128 + c, columns i0 .. i0 + 31 (one per lane)
    for (int c = warp; c < 128; c += 8) {
      const int64_t gj2 = j0 + h * 128 + c, gi2 = i0 + lane;
      if (gi2 < p.d && gj2 < p.d && gj2 < gi2) p.C[gj2 * p.ldc + c_col(p, gj2, gi2)] = t[lane][c];
    }
    __syncthreads();
  }
}

__global__ void scale_or_zero_kernel(float* C, int64_t d, int64_t cols, int64_t ldc, int accumulate) {
  // n == 0: C = 0 (overwrite) or unchanged (accumulate); C is d x cols
  if (accumulate) return;
  for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < d * cols;
       idx += (int64_t)gridDim.x * blockDim.x)
    C[(idx / cols) * ldc + idx % cols] = 0.f;
}

// ------------------------------------------------------------------ host

struct Plan {
  int T, num_tiles, kblocks, splits, kb_per_split, num_units;
};

// At most this many 64-token blocks accumulate in one TMEM accumulator.
// The tensor core's fp32 accumulation loses a small systematic amount per
// MMA (measured on B200 for bf16 inputs: the diagonal of a covariance comes
// out low by about 4e-9 x the tokens in one accumulation chain: 4.8e-5 at
// 12288 tokens, 1.1e-4 at 24576), so long token ranges are split and the
// splits summed in fp32 in a fixed order.
constexpr int kMaxKbPerSplit = 192;   // 12288 tokens

// Token splits per tile: minimise (waves / splits) x full-tile MMA time plus
// the partial-tile round trip through HBM, with waves counted on 148 SMs,
// subject to the chain-length cap above.
Plan make_plan(int64_t n, int64_t d, int64_t blk = 0) {
  Plan pl;
  pl.T = (int)kq::cdiv(d, TILE);
  pl.num_tiles = pl.T * (pl.T + 1) / 2;
  if (blk) {   // block-diagonal mode: d / blk blocks of (blk / 256)^2 / 2 tiles
    const int kt = (int)(blk / TILE);
    pl.num_tiles = (int)(d / blk) * (kt * (kt + 1) / 2);
  }
  pl.kblocks = (int)kq::cdiv(n, BK);
  const double tile_s = 2.0 * TILE * TILE * (double)n / (1.4e15 / ASSUMED_SMS);
  double best = 1e300;
  int best_s = 1;
  const int smin = std::max(1, (int)kq::cdiv(pl.kblocks, kMaxKbPerSplit));
  const int smax = std::max(smin, std::min(16, std::max(1, pl.kblocks)));
  for (int s = smin; s <= smax; ++s) {
    const int per = (int)kq::cdiv(pl.kblocks, s);
    const int s_eff = (int)kq::cdiv(pl.kblocks, per);
    if (s_eff != s) continue;
    const double units = (double)pl.num_tiles * s;
    const double waves = std::ceil(units / ASSUMED_SMS);
    double t = waves * tile_s / s;
    if (s > 1) t += units * TILE * TILE * 8.0 / 6.4e12;
    if (t < best * 0.995) {
      best = t;
      best_s = s;
    }
  }
  pl.splits = best_s;
  pl.kb_per_split = (int)kq::cdiv(pl.kblocks, best_s);
  pl.num_units = pl.num_tiles * best_s;
  return pl;
}

}  // namespace

namespace {

size_t accum_ws_size(int64_t n, int64_t d, int64_t blk) {
  if (n <= 0 || d < 1) return 0;
  Plan pl = make_plan(n, d, blk);
  if (pl.splits == 1) return 0;
  return kq::align_up((size_t)pl.num_units * TILE * TILE * sizeof(float), 256);
}

// C (+)= alpha A^T A: the whole symmetric matrix (blk == 0) or only its
// blk x blk diagonal blocks (blk a multiple of 256 dividing d), C then being
// d x blk with block b in rows b blk .. b blk + blk - 1.
kq_status accum_cov_impl(const char* name, const uint16_t* A, int64_t n, int64_t d, int64_t lda, float* C,
                         int64_t ldc, float alpha, int accumulate, void* ws, size_t ws_bytes, int32_t* info,
                         kq_stream_t stream, int64_t blk) {
  const int64_t cols = blk ? blk : d;
  if ((!A && n > 0) || !C || !info) return kq::fail(KQ_ERR_INVALID_ARG, "%s: NULL pointer", name);
  if (n < 0 || d < 1 || d > 65536) return kq::fail(KQ_ERR_UNSUPPORTED_SHAPE, "%s: need n >= 0, 1 <= d <= 65536", name);
  if (n > ((int64_t)1 << 31) - BK) return kq::fail(KQ_ERR_UNSUPPORTED_SHAPE, "%s: n above 2^31 - 64", name);
  if (lda < d || ldc < cols) return kq::fail(KQ_ERR_INVALID_ARG, "%s: leading dimension too small", name);
  if ((n > 0 && !kq::aligned(A, 16)) || (lda & 7))
    return kq::fail(KQ_ERR_ALIGNMENT, "%s: A 16-byte aligned, lda %% 8 == 0", name);
  if (!isfinite(alpha)) return kq::fail(KQ_ERR_INVALID_ARG, "%s: alpha not finite", name);
  cudaStream_t st = (cudaStream_t)stream;
  if (n == 0) {
    scale_or_zero_kernel<<<256, 256, 0, st>>>(C, d, cols, ldc, accumulate);
    KQ_TRY(kq::launch_check(name));
    kq::clear_error();
    return KQ_OK;
  }
  Plan pl = make_plan(n, d, blk);
  const size_t need = accum_ws_size(n, d, blk);
  if (need && (!ws || !kq::aligned(ws, 256) || ws_bytes < need))
    return kq::fail(KQ_ERR_WORKSPACE, "%s: workspace of %zu bytes needed", name, need);

  CUtensorMap tmap;
  KQ_TRY(make_map_2d(&tmap, A, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, d, n, lda, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B));

  Params p;
  p.n = n;
  p.d = d;
  p.T = pl.T;
  p.num_tiles = pl.num_tiles;
  p.splits = pl.splits;
  p.kb_per_split = pl.kb_per_split;
  p.kblocks = pl.kblocks;
  p.num_units = pl.num_units;
  p.alpha = alpha;
  p.accumulate = accumulate ? 1 : 0;
  p.C = C;
  p.ldc = ldc;
  p.c_vec = (kq::aligned(C, 16) && !(ldc & 3)) ? 1 : 0;
  p.partial = static_cast<float*>(ws);
  p.kt = blk ? (int)(blk / TILE) : 0;
  p.tiles_per_block = p.kt * (p.kt + 1) / 2;
  p.blk = blk;
  p.info = info;
  p.wait_ns = kq::wait_limit_ns();

  int dev = 0, sms = ASSUMED_SMS;
  KQ_TRY(kq::cuda_check(cudaGetDevice(&dev), "kq_accum_cov: cudaGetDevice"));
  KQ_TRY(kq::cuda_check(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev), "kq_accum_cov: SM count"));
  KQ_TRY(kq::cuda_check(cudaFuncSetAttribute(syrk_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES),
                        "kq_accum_cov: smem attribute"));
  const int grid = std::min(pl.num_units, sms);
  syrk_tc_kernel<<<grid, THREADS, SMEM_BYTES, st>>>(tmap, p);
  KQ_TRY(kq::launch_check(name));
  if (pl.splits > 1) {
    split_reduce_kernel<<<pl.num_tiles * 8, 256, 0, st>>>(p);
    KQ_TRY(kq::launch_check(name));
  }
  kq::clear_error();
  return KQ_OK;
}

}  // namespace

extern "C" size_t kq_accum_cov_workspace_size(int64_t n, int64_t d) { return accum_ws_size(n, d, 0); }

extern "C" kq_status kq_accum_cov(const uint16_t* A, int64_t n, int64_t d, int64_t lda, float* C, int64_t ldc,
                                  float alpha, int accumulate, void* ws, size_t ws_bytes, int32_t* info,
                                  kq_stream_t stream) {
  return accum_cov_impl("kq_accum_cov", A, n, d, lda, C, ldc, alpha, accumulate, ws, ws_bytes, info, stream, 0);
}

extern "C" size_t kq_accum_cov_blocks_workspace_size(int64_t n, int64_t d, int64_t k) {
  if (k < 256 || k % 256 || d % k) return 0;
  return accum_ws_size(n, d, k);
}

extern "C" kq_status kq_accum_cov_blocks(const uint16_t* A, int64_t n, int64_t d, int64_t lda, int64_t k, float* C,
                                         int64_t ldc, float alpha, int accumulate, void* ws, size_t ws_bytes,
                                         int32_t* info, kq_stream_t stream) {
  if (k < 256 || k % 256 || d % k)
    return kq::fail(KQ_ERR_UNSUPPORTED_SHAPE, "kq_accum_cov_blocks: k must be a multiple of 256 dividing d");
  return accum_cov_impl("kq_accum_cov_blocks", A, n, d, lda, C, ldc, alpha, accumulate, ws, ws_bytes, info, stream,
                        k);
}
