// 3xTF32 GEMM on tcgen05 tensor cores, with TMA-fed operands and TMEM
// accumulators (internal; see kq_gemm.cuh).
//
// fp32 accuracy at tensor-core speed: each fp32 operand x is split into its
// tf32 rounding b = tf32(x) and the remainder s = x - b (exact in fp32), and
// A B ~ Ab Bb + Ab Bs + As Bb: the dropped As Bs term and the tf32 reading of
// the remainders are ~2^-22 relative.  The products the path needs (dW H1^T
// and its product with dW^T for the Kronecker loss, E Uc for the solver's
// trailing update) lose up to ~60x to cancellation, which rules out plain
// TF32 or bf16 there.
//
// Structure (same as the covariance SYRK): persistent CTAs, one per SM, walk
// the output tiles in one of two shapes chosen per launch: wide tiles of
// 256 x 256 (two M=128 x N=256 accumulators, all 512 TMEM columns), or
// narrow tiles of 128 x 256 with two accumulators used in turn, so that the
// epilogue of one tile overlaps the MMAs of the next (for products with few
// tiles or a short K, where the wide tile's un-overlapped epilogue and the
// last partial wave dominate).  Warp 0 streams 16-deep K slices of A and B (both
// K-major, 64-byte swizzle; tcgen05 kind::tf32 produced no result with an
// MN-major operand on B200 when measured, so callers pass B transposed), big
// and small parts, through a ring of 3 stages (wide tiles, 64 KB each) or 4
// stages (narrow tiles, 48 KB each); one thread of warp 1 issues 12
// tcgen05.mma kind::tf32 per stage; warps 2-9 run the epilogue from TMEM.
// Waits are time-bounded.
#include <cuda.h>

#include <algorithm>

#include "kq_gemm.cuh"
#include "kq_tc.cuh"

namespace kq {
namespace {

using namespace kq::tc;

constexpr int BM = 256, BN = 256, BKF = 16;         // tile rows, cols, K per stage (fp32)
constexpr int A_BYTES = BM * BKF * 4;               // 16 KB per part
constexpr int B_BYTES = BN * BKF * 4;               // 16 KB per part
constexpr int STAGE_BYTES = 2 * A_BYTES + 2 * B_BYTES;   // wide tiles: 3 stages of 64 KB
constexpr int STAGES = 3;
constexpr int NARROW_STAGE_BYTES = A_BYTES + 2 * B_BYTES; // narrow tiles: 4 stages of 48 KB
constexpr int NARROW_STAGES = 4;
constexpr int MAX_STAGES = 4;
static_assert(NARROW_STAGES * NARROW_STAGE_BYTES <= STAGES * STAGE_BYTES, "ring size");
constexpr int THREADS = 320;                        // warp 0 TMA, warp 1 MMA, warps 2-9 epilogue
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 + 256;
constexpr int kMaxSms = 148;   // SMs of a B200

struct Params {
  int64_t M, N, K;
  int wide;   // 1: 256 x 256 tiles, 0: 128 x 256 tiles
  int upper;  // 1: upper block triangle only (M == N), off-diagonal partials doubled
  int tiles_m, tiles_n, num_tiles, kblocks;
  int a_x0, a_y0, b_x0, b_y0;   // tensor-map coordinates of A(0,0) and B(0,0)
  int epilogue;
  float* C;
  float* C_small;
  int64_t ldc;
  const float* src;
  int64_t ld_src;
  int64_t src_rows;
  int trigger_early;
  const uint8_t* dead;
  int dead_vec;    // `dead` 4-byte aligned: the mask read 4 columns at a time
  const float* other;
  int64_t ld_other;
  int other_vec;   // `other` rows can be read as float4 (16-byte aligned rows)
  double* partial;
  int32_t* info;
  unsigned long long wait_ns;   // limit of each pipeline wait (kq_set_wait_limit_ns)
};

// Operand layout in shared memory (K-major): one 16 (k) x 256 TMA box per
// part and stage, rows of 16 fp32 = 64 B with the 64-byte swizzle; 8-row
// groups 512 B apart; a 128-row half starts 8 KB on; the second 8-deep K step
// of the slice starts 32 B on.
__device__ __forceinline__ uint64_t desc_op(uint32_t addr) { return smem_desc(addr, 16, 512, kSwizzle64); }

struct Maps {
  CUtensorMap ab, as, bb, bs;
};

// Tile t -> (row tile, column tile).  Row tile tm holds tiles_n - rb(tm)
// tiles, rb(tm) = 0, or in the upper block triangle the 256-column block of
// its first row; tiles are numbered row by row.  A role visits its tiles in
// increasing t, so the walk resumes where the last call stopped.
struct TileWalk {
  int tm = 0, base = 0;
  __device__ __forceinline__ void at(const Params& p, int bm, int t, int& tm_out, int& tn_out, int& rb_out) {
    for (;;) {
      const int rb = p.upper ? (tm * bm) / BN : 0;
      const int cnt = p.tiles_n - rb;
      if (t < base + cnt || tm + 1 >= p.tiles_m) {
        tm_out = tm;
        tn_out = rb + (t - base);
        rb_out = rb;
        return;
      }
      base += cnt;
      ++tm;
    }
  }
};

__device__ __forceinline__ float tf32_round(float x) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
  return __uint_as_float(r);
}

__global__ void __launch_bounds__(THREADS, 1) gemm_kernel(const __grid_constant__ Maps maps, Params p) {
  constexpr uint32_t IDESC = idesc(kFmtTF32, /*A K-major*/ 0, /*B K-major*/ 0, 128, 256);
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  // ring: wide tiles 3 stages of 64 KB, narrow tiles 4 stages of 48 KB
  const int nstages = p.wide ? STAGES : NARROW_STAGES;
  const int sbytes = p.wide ? STAGE_BYTES : NARROW_STAGE_BYTES;
  const int apart = p.wide ? A_BYTES : A_BYTES / 2;   // bytes of one A part in a stage
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * MAX_STAGES + 5);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const uint32_t full0 = smem_u32(bars), empty0 = smem_u32(bars + MAX_STAGES);
  const uint32_t accfull0 = smem_u32(bars + 2 * MAX_STAGES), accempty0 = smem_u32(bars + 2 * MAX_STAGES + 2);
  const uint32_t drained = smem_u32(bars + 2 * MAX_STAGES + 4);
  const int bm = p.wide ? 256 : 128;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

  if (threadIdx.x == 0) {
    for (int s = 0; s < MAX_STAGES; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(accfull0 + 8 * b, 1);
      mbar_init(accempty0 + 8 * b, 256);
    }
    mbar_init(drained, 1);
    *abort_flag = 0;
    mbar_init_fence();
    prefetch_map(&maps.ab);
    prefetch_map(&maps.as);
    prefetch_map(&maps.bb);
    prefetch_map(&maps.bs);
  }
  if (warp == 1) tmem_alloc<512>(smem_u32(tmem_slot));
  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tmem = *tmem_slot;
  // set-up done: from here on global memory that earlier kernels may write.
  // No early trigger: the solver's in-block kernel that follows fits three
  // CTAs per SM and would pile onto the SMs this grid leaves idle (measured
  // 17 % slower at d_out = 4096); it starts as these CTAs exit instead.
  pdl_wait();
  if (p.trigger_early) pdl_trigger();

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued_phase[MAX_STAGES];
      bool issued[MAX_STAGES] = {false, false, false, false};
      bool ok = true;
      TileWalk walk;
      for (int t = blockIdx.x; t < p.num_tiles && ok; t += gridDim.x) {
        int tm, tn, rb;
        walk.at(p, bm, t, tm, tn, rb);
        const int m0 = tm * bm, n0 = tn * BN;
        for (int kb = 0; kb < p.kblocks; ++kb) {
          if (!mbar_wait(empty0 + 8 * stage, phase ^ 1u, abort_flag, p.info, 11, p.wait_ns)) {
            ok = false;
            break;
          }
          const uint32_t fb = full0 + 8 * stage;
          mbar_arrive_expect_tx(fb, sbytes);
          const uint32_t s0 = smem_u32(smem + stage * sbytes);
          const int k0 = kb * BKF;
          // A boxes are 128 rows; a wide tile takes two per part
          for (int h = 0; h <= p.wide; ++h) {
            tma_load_2d(s0 + h * (A_BYTES / 2), &maps.ab, p.a_x0 + k0, p.a_y0 + m0 + 128 * h, fb);
            tma_load_2d(s0 + apart + h * (A_BYTES / 2), &maps.as, p.a_x0 + k0, p.a_y0 + m0 + 128 * h, fb);
          }
          tma_load_2d(s0 + 2 * apart, &maps.bb, p.b_x0 + k0, p.b_y0 + n0, fb);
          tma_load_2d(s0 + 2 * apart + B_BYTES, &maps.bs, p.b_x0 + k0, p.b_y0 + n0, fb);
          issued[stage] = true;
          issued_phase[stage] = phase;
          if (++stage == nstages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok)
        for (int s = 0; s < nstages; ++s)
          if (issued[s]) mbar_drain(full0 + 8 * s, issued_phase[s]);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0, acc_bits = 0;   // bit b: phase of accumulator b
      bool ok = true, any = false;
      int local = 0;
      for (int t = blockIdx.x; t < p.num_tiles && ok; t += gridDim.x, ++local) {
        const int buf = p.wide ? 0 : (local & 1);
        if (!mbar_wait(accempty0 + 8 * buf, ((acc_bits >> buf) & 1u) ^ 1u, abort_flag, p.info, 12, p.wait_ns)) break;
        fence_after();
        for (int kb = 0; kb < p.kblocks; ++kb) {
          if (!mbar_wait(full0 + 8 * stage, phase, abort_flag, p.info, 13, p.wait_ns)) {
            ok = false;
            break;
          }
          fence_after();
          const uint32_t s0 = smem_u32(smem + stage * sbytes);
          const uint32_t ab = s0, as = s0 + apart, bb = s0 + 2 * apart, bs = bb + B_BYTES;
#pragma unroll
          for (int ks = 0; ks < BKF / 8; ++ks) {
            const uint64_t dbb = desc_op(bb + ks * 32), dbs = desc_op(bs + ks * 32);
            for (int h = 0; h <= p.wide; ++h) {
              const uint32_t d = tmem + 256 * (h + buf);
              const uint32_t first = (kb == 0 && ks == 0) ? 0u : 1u;
              const uint64_t dab = desc_op(ab + h * (A_BYTES / 2) + ks * 32);
              const uint64_t das = desc_op(as + h * (A_BYTES / 2) + ks * 32);
              mma_tf32<IDESC>(d, dab, dbs, first);   // big x small
              mma_tf32<IDESC>(d, das, dbb, 1u);      // small x big
              mma_tf32<IDESC>(d, dab, dbb, 1u);      // big x big
            }
          }
          any = true;
          mma_commit(empty0 + 8 * stage);
          if (++stage == nstages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        mma_commit(accfull0 + 8 * buf);
        acc_bits ^= 1u << buf;
      }
      if (any) {
        mma_commit(drained);
        mbar_drain(drained, 0);
      }
    }
  } else {
    // Epilogue: 8 warps; warp w reads TMEM lanes 32 (w % 4) .. (the rows it
    // may access) for one 128-column half of each accumulator.  Source
    // operands (src / other) for 64 columns are fetched before they are
    // needed, so each thread keeps 16 float4 loads in flight.
    const int e = warp - 2;
    const int wq = warp & 3;
    const int cbase = (e >> 2) * 128;
    uint32_t acc_bits = 0;   // bit b: phase of accumulator b
    int local = 0;
    TileWalk walk;
    for (int t = blockIdx.x; t < p.num_tiles; t += gridDim.x, ++local) {
      const int buf = p.wide ? 0 : (local & 1);
      int tm, tn, rb;
      walk.at(p, bm, t, tm, tn, rb);
      const int64_t m0 = (int64_t)tm * bm, n0 = (int64_t)tn * BN;
      // one lane waits, the warp follows: every lane leaves together on abort
      bool ready = true;
      if (lane == 0) ready = mbar_wait(accfull0 + 8 * buf, (acc_bits >> buf) & 1u, abort_flag, p.info, 14, p.wait_ns);
      if (!__shfl_sync(0xffffffffu, ready ? 1 : 0, 0)) break;
      __syncwarp();
      fence_after();
      double dot = 0.0;
#pragma unroll 1
      for (int h = 0; h <= p.wide; ++h) {
        const int64_t gi = m0 + h * 128 + 32 * wq + lane;
        const bool row_ok = gi < p.M;
        const int64_t si = p.src_rows ? gi % p.src_rows : gi;   // source row
#pragma unroll 1
        for (int g0 = 0; g0 < 128; g0 += 64) {
          const int64_t gj0 = n0 + cbase + g0;
          const bool any = row_ok && gj0 < p.N;
          const bool fast = any && gj0 + 64 <= p.N && !(p.epilogue == kEpiSubtract && p.dead && !p.dead_vec) &&
                            !(p.epilogue == kEpiDot && !p.other_vec);
          float pre[64];
          if (fast && (p.epilogue == kEpiDot || p.epilogue == kEpiSubtract)) {
            const float* sp = (p.epilogue == kEpiDot ? p.other + gi * p.ld_other : p.src + si * p.ld_src) + gj0;
#pragma unroll
            for (int q = 0; q < 64; q += 4) {
              const float4 w = *reinterpret_cast<const float4*>(sp + q);
              pre[q] = w.x;
              pre[q + 1] = w.y;
              pre[q + 2] = w.z;
              pre[q + 3] = w.w;
            }
            if (p.epilogue == kEpiSubtract && p.dead) {
              // dead source columns read as zero; the same 64 flags for every lane
              const uint32_t* dm = reinterpret_cast<const uint32_t*>(p.dead + gj0);
#pragma unroll
              for (int q = 0; q < 16; ++q) {
                const uint32_t m = dm[q];
#pragma unroll
                for (int u = 0; u < 4; ++u) pre[4 * q + u] = ((m >> (8 * u)) & 0xffu) ? 0.f : pre[4 * q + u];
              }
            }
          }
#pragma unroll
          for (int cc = 0; cc < 64; cc += 16) {
            float v[16];
            tmem_ld16(tmem + ((uint32_t)(32 * wq) << 16) + (uint32_t)(256 * (h + buf) + cbase + g0 + cc), v);
            if (!any) continue;
            const int64_t gj = gj0 + cc;
            if (fast) {
              if (p.epilogue == kEpiDot) {
#pragma unroll
                for (int q = 0; q < 16; ++q) dot += (double)v[q] * (double)pre[cc + q];
              } else if (p.epilogue == kEpiStoreSplit) {
                float* c = p.C + gi * p.ldc + gj;
                float* cs = p.C_small + gi * p.ldc + gj;
#pragma unroll
                for (int q = 0; q < 16; q += 4) {
                  float b[4], r[4];
#pragma unroll
                  for (int u = 0; u < 4; ++u) {
                    b[u] = tf32_round(v[q + u]);
                    r[u] = v[q + u] - b[u];
                  }
                  *reinterpret_cast<float4*>(c + q) = make_float4(b[0], b[1], b[2], b[3]);
                  *reinterpret_cast<float4*>(cs + q) = make_float4(r[0], r[1], r[2], r[3]);
                }
              } else {
                float* c = p.C + gi * p.ldc + gj;
#pragma unroll
                for (int q = 0; q < 16; q += 4) {
                  float4 o;
                  if (p.epilogue == kEpiSubtract)
                    o = make_float4(pre[cc + q] - v[q], pre[cc + q + 1] - v[q + 1], pre[cc + q + 2] - v[q + 2],
                                    pre[cc + q + 3] - v[q + 3]);
                  else
                    o = make_float4(v[q], v[q + 1], v[q + 2], v[q + 3]);
                  *reinterpret_cast<float4*>(c + q) = o;
                }
              }
            } else {
              for (int q = 0; q < 16 && gj + q < p.N; ++q) {
                const int64_t j = gj + q;
                if (p.epilogue == kEpiDot) {
                  dot += (double)v[q] * (double)p.other[gi * p.ld_other + j];
                } else if (p.epilogue == kEpiSubtract) {
                  const float sv = (p.dead && p.dead[j]) ? 0.f : p.src[si * p.ld_src + j];
                  p.C[gi * p.ldc + j] = sv - v[q];
                } else if (p.epilogue == kEpiStoreSplit) {
                  const float b = tf32_round(v[q]);
                  p.C[gi * p.ldc + j] = b;
                  p.C_small[gi * p.ldc + j] = v[q] - b;
                } else {
                  p.C[gi * p.ldc + j] = v[q];
                }
              }
            }
          }
        }
      }
      fence_before();
      mbar_arrive(accempty0 + 8 * buf);
      if (p.epilogue == kEpiDot) {
        // fixed-order reduction within the warp (xor butterfly); one partial
        // per (tile, epilogue warp), summed later in index order
        for (int o = 16; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
        if (p.upper && tn > rb) dot *= 2.0;   // stands for the mirror tile below the diagonal
        if (lane == 0) p.partial[8 * (int64_t)t + e] = dot;
      }
      acc_bits ^= 1u << buf;
    }
  }

  fence_before();
  __syncthreads();
  if (warp == 1) {
    fence_after();
    tmem_dealloc<512>(tmem);
  }
}

// big = tf32(x - y), small = (x - y) - big at (r, c), or at (c, r) when
// transposing (through a 32 x 32 shared-memory tile so both sides coalesce).
__global__ void __launch_bounds__(256) split_kernel(const float* __restrict__ x, int64_t ldx,
                                                    const float* __restrict__ y, int64_t ldy, int64_t rows,
                                                    int64_t cols, float* __restrict__ big, float* __restrict__ small,
                                                    int64_t ldo, int transpose) {
  __shared__ float tb[32][33];
  __shared__ float ts[32][33];
  const int64_t tiles_c = (cols + 31) / 32;
  const int64_t r0 = (int64_t)(blockIdx.x / tiles_c) * 32, c0 = (int64_t)(blockIdx.x % tiles_c) * 32;
  const int tx = threadIdx.x % 32, ty = threadIdx.x / 32;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int64_t r = r0 + ty + 8 * k, c = c0 + tx;
    if (r < rows && c < cols) {
      float v = x[r * ldx + c];
      if (y) v -= y[r * ldy + c];
      const float b = tf32_round(v);
      if (transpose) {
        tb[ty + 8 * k][tx] = b;
        ts[ty + 8 * k][tx] = v - b;
      } else {
        big[r * ldo + c] = b;
        small[r * ldo + c] = v - b;
      }
    }
  }
  if (!transpose) return;
  __syncthreads();
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int64_t c = c0 + ty + 8 * k, r = r0 + tx;   // output row c, column r
    if (r < rows && c < cols) {
      big[c * ldo + r] = tb[tx][ty + 8 * k];
      small[c * ldo + r] = ts[tx][ty + 8 * k];
    }
  }
}

}  // namespace

// Wide tiles when they fill two waves, or when K is long enough that the
// un-overlapped epilogue is a small share of a tile (measured on B200: the
// 4096^3 products of the loss run 15 % faster wide, the solver's K <= 1024
// updates 20 % faster narrow).
namespace {

// Tiles of an M x N product with bm-row tiles; the same count as TileWalk.
int64_t tile_count(int64_t M, int64_t N, int bm, bool upper) {
  const int64_t tm = cdiv(M, bm), tn = cdiv(N, BN);
  if (!upper) return tm * tn;
  int64_t c = 0;
  for (int64_t r = 0; r < tm; ++r) c += tn - (r * bm) / BN;
  return c;
}

bool gemm_wide(int64_t M, int64_t N, int64_t K, bool upper) {
  return tile_count(M, N, BM, upper) >= 2 * kMaxSms || K >= 2048;
}

}  // namespace

int64_t gemm_tiles(int64_t M, int64_t N, int64_t K, bool upper) {
  return tile_count(M, N, gemm_wide(M, N, K, upper) ? BM : BM / 2, upper);
}

int64_t gemm_tiles_max(int64_t M, int64_t N, bool upper) { return tile_count(M, N, BM / 2, upper); }

kq_status split_tf32(const float* x, int64_t ldx, const float* y, int64_t ldy, int64_t rows, int64_t cols, float* big,
                     float* small, int64_t ldo, bool transpose, cudaStream_t st) {
  if (rows <= 0 || cols <= 0) return KQ_OK;
  const int64_t blocks = cdiv(rows, 32) * cdiv(cols, 32);
  if (blocks > 0x7fffffff) return fail(KQ_ERR_UNSUPPORTED_SHAPE, "split_tf32: too large");
  split_kernel<<<(unsigned)blocks, 256, 0, st>>>(x, ldx, y, ldy, rows, cols, big, small, ldo, transpose ? 1 : 0);
  return launch_check("split_tf32");
}

kq_status gemm_3xtf32(const Gemm3xTF32& g, cudaStream_t st) {
  if (g.M <= 0 || g.N <= 0 || g.K <= 0) return KQ_OK;
  const void* ptrs[] = {g.a_big, g.a_small, g.bt_big, g.bt_small};
  for (const void* q : ptrs)
    if (!q || !aligned(q, 16)) return fail(KQ_ERR_ALIGNMENT, "gemm: operands must be 16-byte aligned");
  if ((g.lda & 3) || (g.ldbt & 3) || (g.a_col0 & 3) || (g.bt_col0 & 3))
    return fail(KQ_ERR_ALIGNMENT, "gemm: leading dimensions and column offsets must be multiples of 4");
  const int64_t big = (int64_t)1 << 31;
  if (g.a_row0 + g.M >= big || g.a_col0 + g.K >= big || g.bt_row0 + g.N >= big || g.bt_col0 + g.K >= big)
    return fail(KQ_ERR_UNSUPPORTED_SHAPE, "gemm: coordinates beyond 2^31");
  // Tensor maps end exactly at the used region, so every read past M, N or K
  // (ragged tiles, a K tail) is filled with zeros by the TMA unit.
  Maps maps;
  auto map_op = [&](CUtensorMap* m, const float* base, int64_t ld, int64_t row0, int64_t col0, int64_t rows,
                    int box_rows) -> kq_status {
    return tc::make_map_2d(m, base, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, col0 + g.K, row0 + rows, ld, BKF, box_rows,
                           CU_TENSOR_MAP_SWIZZLE_64B);
  };
  KQ_TRY(map_op(&maps.ab, g.a_big, g.lda, g.a_row0, g.a_col0, g.M, 128));
  KQ_TRY(map_op(&maps.as, g.a_small, g.lda, g.a_row0, g.a_col0, g.M, 128));
  KQ_TRY(map_op(&maps.bb, g.bt_big, g.ldbt, g.bt_row0, g.bt_col0, g.N, BN));
  KQ_TRY(map_op(&maps.bs, g.bt_small, g.ldbt, g.bt_row0, g.bt_col0, g.N, BN));
  Params p;
  p.M = g.M;
  p.N = g.N;
  p.K = g.K;
  p.wide = gemm_wide(g.M, g.N, g.K, g.upper) ? 1 : 0;
  p.upper = g.upper ? 1 : 0;
  p.tiles_m = (int)cdiv(g.M, p.wide ? BM : BM / 2);
  p.tiles_n = (int)cdiv(g.N, BN);
  const int64_t tiles = tile_count(g.M, g.N, p.wide ? BM : BM / 2, g.upper);
  if (tiles > 0x7fffffff) return fail(KQ_ERR_UNSUPPORTED_SHAPE, "gemm: too many tiles");
  p.num_tiles = (int)tiles;
  p.kblocks = (int)cdiv(g.K, BKF);
  p.a_x0 = (int)g.a_col0;
  p.a_y0 = (int)g.a_row0;
  p.b_x0 = (int)g.bt_col0;
  p.b_y0 = (int)g.bt_row0;
  p.epilogue = g.epilogue;
  p.C = g.C;
  p.C_small = g.C_small;
  p.ldc = g.ldc;
  p.src = g.src;
  p.ld_src = g.ld_src;
  p.src_rows = g.src_rows;
  p.trigger_early = g.trigger_early ? 1 : 0;
  p.dead = g.dead;
  p.dead_vec = (g.dead && aligned(g.dead, 4)) ? 1 : 0;
  p.other = g.other;
  p.ld_other = g.ld_other;
  p.other_vec = (g.other && aligned(g.other, 16) && !(g.ld_other & 3)) ? 1 : 0;
  p.partial = g.partial;
  p.info = g.info;
  p.wait_ns = kq::wait_limit_ns();
  if (g.upper && (g.M != g.N || g.epilogue != kEpiDot))
    return fail(KQ_ERR_INVALID_ARG, "gemm: the upper block triangle needs M == N and the dot epilogue");
  if (g.epilogue == kEpiDot) {
    if (!g.other || !g.partial) return fail(KQ_ERR_INVALID_ARG, "gemm: dot epilogue needs `other` and `partial`");
  } else {
    if (!g.C || !aligned(g.C, 16) || (g.ldc & 3)) return fail(KQ_ERR_ALIGNMENT, "gemm: C must be 16-byte aligned");
    if (g.epilogue == kEpiStoreSplit && (!g.C_small || !aligned(g.C_small, 16)))
      return fail(KQ_ERR_ALIGNMENT, "gemm: C_small must be 16-byte aligned");
    if (g.epilogue == kEpiSubtract && (!g.src || !aligned(g.src, 16) || (g.ld_src & 3)))
      return fail(KQ_ERR_ALIGNMENT, "gemm: src must be 16-byte aligned");
  }
  int dev = 0, sms = 148;
  KQ_TRY(cuda_check(cudaGetDevice(&dev), "gemm: cudaGetDevice"));
  KQ_TRY(cuda_check(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev), "gemm: SM count"));
  KQ_TRY(cuda_check(cudaFuncSetAttribute(gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES),
                    "gemm: smem attribute"));
  return launch_ex("gemm_3xtf32", g.pdl, gemm_kernel, dim3((unsigned)std::min(p.num_tiles, sms)), dim3(THREADS),
                   SMEM_BYTES, st, maps, p);
}

}  // namespace kq
