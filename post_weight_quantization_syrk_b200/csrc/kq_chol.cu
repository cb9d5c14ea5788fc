// kq_chol_inv: damping, dead columns and the upper Cholesky factor of the
// damped inverse (step a6), in fp64.
//
// GPTQ's column-wise OBS update (KronQ review, romaanj.github.io/reviews/kronq,
// Prior limitations) needs the rows of the upper triangular Uc with
// Uc^T Uc = (H + lambda I)^-1.  With J the exchange matrix, J H J = L L^T gives
// H = R R^T for the upper triangular R = J L J, hence Uc = R^-1 = J L^-1 J.
// So the work is one ordinary lower Cholesky of the index-reversed matrix and
// one lower triangular inverse: n^3/3 + n^3/3 flops, no explicit H^-1.
//
// Precision: the damped matrix can have a condition number of 1e5 and more;
// fp32 would lose most digits of Uc, so everything here is fp64 and only the
// final Uc is rounded to fp32.
//
// Blocked right-looking algorithm, panel width nb = 64, per block column k:
//   potrf:  factor the 64 x 64 diagonal block and invert its factor, in
//           registers of one CTA (4 x 4 blocks per thread, one barrier per
//           column);
//   step a: the panel below it, P = A_panel L_kk^-T, stored TRANSPOSED
//           (Pt, 64 x n, row k contiguous) so that every operand of step b
//           is read k-major; and row block k of the inverse, X_k = L_kk^-1 B_k
//           (forward substitution on B = I);
//   step b: the trailing lower-triangle update A -= P P^T and the
//           substitution update B_below -= L_below,k X_k, as 128 x 64 tiles.
// Steps a and b run on the fp64 tensor cores (mma.sync m8n8k4: on B200 the
// fp64 MMA and FMA peaks are equal, but an MMA takes its operands from
// registers, so it needs a quarter of the shared-memory reads per flop that
// an FMA tile does), with operands staged in shared memory by cp.async.
// A and X live in the workspace with leading dimension N2 = align(n, 128) +
// 128, zero-padded, so that 128-row tiles starting at any multiple of 64
// stay inside the buffers and the padding stays exactly zero.
#include <math.h>

#include <algorithm>

#include "kq_internal.cuh"

namespace {

constexpr int NB = 64;
constexpr int TB = 128;   // padding granule of the workspace matrices

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_addr(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// A = reversed H in the lower triangle (fp64), zero above it and in the
// padding (ld x ld); dead columns get diagonal 1; NaN/Inf reported.
__global__ void prep_kernel(const float* __restrict__ H, int64_t ldh, int64_t n, double* __restrict__ A, int64_t ld,
                            uint8_t* __restrict__ dead, int32_t* info) {
  const int64_t jj = (int64_t)blockIdx.x * 32 + threadIdx.x;
  for (int s = 0; s < 32; s += 8) {
    const int64_t i = (int64_t)blockIdx.y * 32 + threadIdx.y + s;
    if (i >= ld || jj >= ld) continue;
    double v = 0.0;
    if (i < n && jj <= i) {
      // upper triangle of H, read through the reversal
      v = (double)H[(n - 1 - i) * ldh + (n - 1 - jj)];
      if (!isfinite(v)) kq::report(info, KQ_ERR_NONFINITE, n - 1 - i);
      if (i == jj) {
        bool d = (v == 0.0);
        if (d) v = 1.0;
        if (dead) dead[n - 1 - i] = d ? 1 : 0;
      }
    }
    A[i * ld + jj] = v;
  }
}

// lambda = damp * mean(diag A); diag A += lambda.  One CTA, fixed-order sum.
__global__ void damp_kernel(double* __restrict__ A, int64_t n, int64_t ld, double damp, double* __restrict__ lam_out) {
  __shared__ double red[1024];
  double s = 0.0;
  for (int64_t i = threadIdx.x; i < n; i += blockDim.x) s += A[i * ld + i];
  red[threadIdx.x] = s;
  __syncthreads();
  for (int w = blockDim.x / 2; w > 0; w >>= 1) {
    if (threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
    __syncthreads();
  }
  const double lam = damp * (red[0] / (double)n);
  for (int64_t i = threadIdx.x; i < n; i += blockDim.x) A[i * ld + i] += lam;
  if (threadIdx.x == 0) *lam_out = lam;
}

__device__ __forceinline__ void dmma_acc(double& d0, double& d1, double a, double b) {
  asm volatile("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0,%1}, {%2}, {%3}, {%0,%1};"
               : "+d"(d0), "+d"(d1)
               : "d"(a), "d"(b));
}

// Factor the kb x kb diagonal block at (k0, k0) (lower Cholesky, padded to
// 64 x 64 with the identity) and write the inverse of its factor to Dinv
// (64 x 64, zero above the diagonal).  One CTA of 8 warps; the block (As) and
// the substitution R being turned into the inverse (Xs, from the identity)
// sit in shared memory.  Blocked right-looking over four 16-column leaves,
// leaf kk at p = 16 kk:
//   1. warp 0 factors the 16 x 16 diagonal leaf in registers (lane l holds
//      row l / 2, columns 8 (l % 2) ..; column j is spread through shared
//      memory within the warp, no CTA barrier) and forms its inverse Li;
//   2. the panel below it, L_ik = A_ik Li^T, and the leaf's rows of the
//      inverse, X_k = Li R_k (16 x 16 products on the fp64 tensor cores,
//      one per warp);
//   3. the trailing update A_ij -= L_ik L_jk^T (j <= i) and the substitution
//      update R_i -= L_ik X_k.
// Shared-memory strides are 4 mod 16 doubles, so the fragment loads of a
// half-warp hit distinct banks.
constexpr int SP = NB + 4;    // As, Xs row stride
constexpr int SL = 16 + 4;    // leaf inverse row stride
constexpr size_t kPotrfSmem = (size_t)(2 * NB * SP + 16 * SL + 64) * sizeof(double);

// acc (2 x 2 tiles of 8 x 8) += sign * Aop(16 x 16) Bop(16 x 16), with
// Aop(r, k) = a[r * sa + k] and Bop(k, n) = b[k * sbk + n * sbn].
__device__ __forceinline__ void mma16(double (&acc)[2][2][2], const double* a, int sa, const double* b, int sbk,
                                      int sbn, double sign, int fr, int fc) {
#pragma unroll
  for (int ks = 0; ks < 4; ++ks) {
    const int k = 4 * ks + fc;
    double av[2], bv[2];
#pragma unroll
    for (int rt = 0; rt < 2; ++rt) av[rt] = sign * a[(8 * rt + fr) * sa + k];
#pragma unroll
    for (int ct = 0; ct < 2; ++ct) bv[ct] = b[k * sbk + (8 * ct + fr) * sbn];
#pragma unroll
    for (int rt = 0; rt < 2; ++rt)
#pragma unroll
      for (int ct = 0; ct < 2; ++ct) dmma_acc(acc[rt][ct][0], acc[rt][ct][1], av[rt], bv[ct]);
  }
}

__device__ __forceinline__ void load16(double (&acc)[2][2][2], const double* c, int sc, int fr, int fc) {
#pragma unroll
  for (int rt = 0; rt < 2; ++rt)
#pragma unroll
    for (int ct = 0; ct < 2; ++ct) {
      acc[rt][ct][0] = c[(8 * rt + fr) * sc + 8 * ct + 2 * fc];
      acc[rt][ct][1] = c[(8 * rt + fr) * sc + 8 * ct + 2 * fc + 1];
    }
}

__device__ __forceinline__ void store16(const double (&acc)[2][2][2], double* c, int sc, int fr, int fc) {
#pragma unroll
  for (int rt = 0; rt < 2; ++rt)
#pragma unroll
    for (int ct = 0; ct < 2; ++ct) {
      c[(8 * rt + fr) * sc + 8 * ct + 2 * fc] = acc[rt][ct][0];
      c[(8 * rt + fr) * sc + 8 * ct + 2 * fc + 1] = acc[rt][ct][1];
    }
}

// The factorisation of one diagonal block by all 256 threads of a CTA, with
// psm at least kPotrfSmem bytes of shared memory (16-byte aligned).
__device__ __forceinline__ void potrf_block(const double* __restrict__ A, int64_t ld, int64_t n, int64_t k0, int kb,
                                            double* __restrict__ Dinv, int32_t* info, double* psm) {
  double* As = psm;              // [64][SP]
  double* Xs = psm + NB * SP;    // [64][SP]
  double* Ls = Xs + NB * SP;     // [16][SL]
  double* Cb = Ls + 16 * SL;     // leaf broadcast: column j, two buffers of 16
  double* Rb = Cb + 32;          // leaf broadcast: row j of R, two buffers of 16
  const int t = threadIdx.x, warp = t / 32, lane = t % 32;
  const int fr = lane / 4, fc = lane % 4;
  {
    // all 16 loads of a thread in flight before any is used
    double v[16];
#pragma unroll
    for (int u = 0; u < 16; ++u) {
      const int idx = t + 256 * u, i = idx / NB, c = idx % NB;
      v[u] = (i < kb && c <= i) ? A[(k0 + i) * ld + k0 + c] : 0.0;
    }
#pragma unroll
    for (int u = 0; u < 16; ++u) {
      const int idx = t + 256 * u, i = idx / NB, c = idx % NB;
      As[i * SP + c] = (i >= kb && i == c) ? 1.0 : v[u];
      Xs[i * SP + c] = (i == c) ? 1.0 : 0.0;
    }
  }
  __syncthreads();
#pragma unroll 1
  for (int kk = 0; kk < 4; ++kk) {
    const int p = 16 * kk;
    if (warp == 0) {
      // ---- leaf: rows p.., lane holds row r = lane / 2, columns 8 h ..;
      // per column j the lanes holding column j and row j of R publish them
      // to shared memory (double buffered by the parity of j) and the warp
      // reads them back after __syncwarp: cheaper than 64-bit shuffles.
      const int r = lane >> 1, h = lane & 1;
      double a[8], x[8];
#pragma unroll
      for (int m = 0; m < 8; ++m) {
        a[m] = As[(p + r) * SP + p + 8 * h + m];
        x[m] = (r == 8 * h + m) ? 1.0 : 0.0;
      }
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const int reg = j & 7, hj = j >> 3, b = j & 1;
        double* colj = Cb + 16 * b;
        double* rowj = Rb + 16 * b;
        if (h == hj) colj[r] = a[reg];
        if (r == j) {
          double2* dst = reinterpret_cast<double2*>(rowj + 8 * h);
#pragma unroll
          for (int m = 0; m < 4; ++m) dst[m] = make_double2(x[2 * m], x[2 * m + 1]);
        }
        __syncwarp();
        double d = colj[j];
        const double av = colj[r];
        double cj[8], rj[8];
        const double2* cs = reinterpret_cast<const double2*>(colj + 8 * h);
        const double2* rsrc = reinterpret_cast<const double2*>(rowj + 8 * h);
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          const double2 c2 = cs[m], r2 = rsrc[m];
          cj[2 * m] = c2.x;
          cj[2 * m + 1] = c2.y;
          rj[2 * m] = r2.x;
          rj[2 * m + 1] = r2.y;
        }
        if (!(d > 0.0) || !isfinite(d)) {
          if (lane == 0) kq::report(info, KQ_ERR_NOT_PD, n - 1 - (k0 + p + j));
          d = 1.0;
        }
        const double rs = rsqrt(d);
        const double f = (r > j) ? (av * rs) * rs : 0.0;
#pragma unroll
        for (int m = 0; m < 8; ++m) {
          a[m] = fma(-f, cj[m], a[m]);
          x[m] = fma(-f, rj[m], x[m]);
        }
        if (r == j)
#pragma unroll
          for (int m = 0; m < 8; ++m) x[m] *= rs;
      }
#pragma unroll
      for (int m = 0; m < 8; ++m) Ls[r * SL + 8 * h + m] = x[m];
    }
    __syncthreads();
    // ---- panel L_ik = A_ik Li^T (i > kk) and X_k = Li R_k (column blocks <= kk)
    {
      const int nitems = (3 - kk) + (kk + 1);
      for (int it = warp; it < nitems; it += 8) {
        double acc[2][2][2] = {};
        if (it < 3 - kk) {
          const int i = kk + 1 + it;
          mma16(acc, As + 16 * i * SP + p, SP, Ls, 1, SL, 1.0, fr, fc);
          __syncwarp();
          store16(acc, As + 16 * i * SP + p, SP, fr, fc);
        } else {
          const int cb = it - (3 - kk);
          mma16(acc, Ls, SL, Xs + p * SP + 16 * cb, SP, 1, 1.0, fr, fc);
          __syncwarp();
          store16(acc, Xs + p * SP + 16 * cb, SP, fr, fc);
        }
      }
    }
    __syncthreads();
    // ---- trailing: A_ij -= L_ik L_jk^T (kk < j <= i), R_i -= L_ik X_k
    {
      const int m3 = 3 - kk;
      const int nchol = m3 * (m3 + 1) / 2;
      const int nitems = nchol + m3 * (kk + 1);
      for (int it = warp; it < nitems; it += 8) {
        double acc[2][2][2];
        if (it < nchol) {
          int i = 0, jb = 0, l = it;   // lower pairs (i, jb) of the m3 x m3 trailing blocks
          while (l > i) { l -= i + 1; ++i; }
          jb = l;
          const int bi = kk + 1 + i, bj = kk + 1 + jb;
          double* c = As + 16 * bi * SP + 16 * bj;
          load16(acc, c, SP, fr, fc);
          mma16(acc, As + 16 * bi * SP + p, SP, As + 16 * bj * SP + p, 1, SP, -1.0, fr, fc);
          store16(acc, c, SP, fr, fc);
        } else {
          const int q = it - nchol, bi = kk + 1 + q / (kk + 1), cb = q % (kk + 1);
          double* c = Xs + 16 * bi * SP + 16 * cb;
          load16(acc, c, SP, fr, fc);
          mma16(acc, As + 16 * bi * SP + p, SP, Xs + p * SP + 16 * cb, SP, 1, -1.0, fr, fc);
          store16(acc, c, SP, fr, fc);
        }
      }
    }
    __syncthreads();
  }
  kq::pdl_trigger();   // the panel step may be scheduled now; it waits for this grid's stores
  for (int idx = t; idx < NB * NB; idx += 256) Dinv[idx] = Xs[(idx / NB) * SP + idx % NB];
}

__global__ void __launch_bounds__(256) potrf_kernel(const double* __restrict__ A, int64_t ld, int64_t n, int64_t k0,
                                                    int kb, double* __restrict__ Dinv, int32_t* info) {
  extern __shared__ __align__(16) double psm[];
  kq::pdl_wait();   // the block was last updated by the previous kernel of the chain
  potrf_block(A, ld, n, k0, kb, Dinv, info, psm);
}


// Shared-memory row strides (doubles) of the fp64 MMA operands: a stride of
// 4 mod 16 puts the 16 (row, k) pairs of a half-warp's fragment load in
// distinct banks.
constexpr int SD = NB + 4;        // Dinv, [c][k]
constexpr int SPK = NB + 4;       // panel rows, [x][k]
constexpr int SXK = 128 + 4;      // inverse rows, [k][x]
constexpr size_t kStepASmem = (size_t)(NB * SD + 128 * SPK) * sizeof(double);   // 102 KB

// One launch per block step k (after the diagonal factorisation); every CTA
// forms a 64 x 128 tile of C'(c, x) = sum_k Dinv_k[c][k] B'(k, x) with the
// fp64 tensor cores (mma.sync m8n8k4, 8 warps of 32 x 32):
//   CTAs [0, tp):  the panel, transposed: B'(k, x) = A[r0 + x][k0 + k] for the
//                  128 rows from r0 = k0 + 64 + 128 blk, written to
//                  Pt[c][r0 + x] (P = A_panel Dinv_k^T);
//   CTAs after:    row block k of the inverse, forward substitution
//                  X_k = Dinv_k B_k on the 128 columns from c0, in place.
// Operands are staged with cp.async; K = 64 in one stage.
__global__ void __launch_bounds__(256) step_a_kernel(const double* __restrict__ A, double* __restrict__ X,
                                                     double* __restrict__ Pt, int64_t ld, int64_t k0, int64_t tp,
                                                     const double* __restrict__ Dinv) {
  extern __shared__ __align__(16) double sm[];
  double* Ds = sm;              // [64][SD]
  double* Bs = sm + NB * SD;    // panel [128][SPK] or inverse rows [64][SXK]
  const int t = threadIdx.x;
  const bool panel = (int64_t)blockIdx.x < tp;
  const int64_t r0 = k0 + NB + (int64_t)blockIdx.x * 128;
  const int64_t c0 = ((int64_t)blockIdx.x - tp) * 128;
  kq::pdl_wait();   // Dinv comes from the diagonal factorisation just before
#pragma unroll
  for (int u = 0; u < 8; ++u) {   // Dinv: 64 rows x 32 chunks
    const int id = u * 256 + t, row = id / 32, cc = id % 32;
    cp_async16(Ds + row * SD + 2 * cc, Dinv + row * NB + 2 * cc);
  }
  if (panel) {
#pragma unroll
    for (int u = 0; u < 16; ++u) {   // 128 rows x 32 chunks
      const int id = u * 256 + t, x = id / 32, cc = id % 32;
      cp_async16(Bs + x * SPK + 2 * cc, A + (r0 + x) * ld + k0 + 2 * cc);
    }
  } else {
#pragma unroll
    for (int u = 0; u < 16; ++u) {   // 64 rows x 64 chunks
      const int id = u * 256 + t, k = id / 64, cc = id % 64;
      cp_async16(Bs + k * SXK + 2 * cc, X + (k0 + k) * ld + c0 + 2 * cc);
    }
  }
  cp_commit();
  const int warp = t / 32, lane = t % 32;
  const int wc = warp / 4, wx = warp % 4;
  const int fr = lane / 4, fc = lane % 4;
  double acc[4][4][2];
#pragma unroll
  for (int rt = 0; rt < 4; ++rt)
#pragma unroll
    for (int ct = 0; ct < 4; ++ct) acc[rt][ct][0] = acc[rt][ct][1] = 0.0;
  cp_wait<0>();
  __syncthreads();
#pragma unroll 4
  for (int ks = 0; ks < NB / 4; ++ks) {
    const int k = 4 * ks + fc;
    double a[4], b[4];
#pragma unroll
    for (int rt = 0; rt < 4; ++rt) a[rt] = Ds[(32 * wc + 8 * rt + fr) * SD + k];
    if (panel) {
#pragma unroll
      for (int ct = 0; ct < 4; ++ct) b[ct] = Bs[(32 * wx + 8 * ct + fr) * SPK + k];
    } else {
#pragma unroll
      for (int ct = 0; ct < 4; ++ct) b[ct] = Bs[k * SXK + 32 * wx + 8 * ct + fr];
    }
#pragma unroll
    for (int rt = 0; rt < 4; ++rt)
#pragma unroll
      for (int ct = 0; ct < 4; ++ct) dmma_acc(acc[rt][ct][0], acc[rt][ct][1], a[rt], b[ct]);
  }
  double* out = panel ? Pt + r0 : X + k0 * ld + c0;
#pragma unroll
  for (int rt = 0; rt < 4; ++rt)
#pragma unroll
    for (int ct = 0; ct < 4; ++ct)
      *reinterpret_cast<double2*>(out + (32 * wc + 8 * rt + fr) * ld + 32 * wx + 8 * ct + 2 * fc) =
          make_double2(acc[rt][ct][0], acc[rt][ct][1]);
}

// Lower-triangle tiles of 128 rows x 64 columns: row block ti holds column
// blocks 0 .. 2 ti + 1, so block ti starts at linear index ti (ti + 1).
__device__ __forceinline__ void rect_index(int64_t l, int64_t* ti, int64_t* tj) {
  int64_t t = (int64_t)((sqrt(4.0 * (double)l + 1.0) - 1.0) * 0.5);
  while (t * (t + 1) > l) --t;
  while ((t + 1) * (t + 2) <= l) ++t;
  *ti = t;
  *tj = l - t * (t + 1);
}

// Trailing update after block step k (after step a), with base = k0 + 64
// the first trailing row, T = n - base and tr = ceil(T / 128); 128 x 64
// output tiles of
//   the Cholesky update A -= P P^T: row tile ti holds column tiles
//     0 .. 2 ti + 1, the ones that meet the lower triangle (tiles on the
//     diagonal also touch entries above it, which are never read);
//   the substitution update of the rows below, X[r][c] -= sum_k L[r][k]
//     X_k[k][c], c < base: row tiles 0 .. tr-1, column tiles 0 .. base/64-1.
// `part` selects the tiles (so that the next block's dependencies can be
// updated ahead of the rest):
//   kAll:  every tile;
//   kNext: Cholesky column tile 0 (column block k+1, every row) and the
//          substitution row tile 0 (rows base .. base+127);
//   kRest: the others.
// Both operands are k-major rows (Pt rows, X_k rows), staged in shared memory
// by cp.async in four 16-deep groups; the output tile is read into the fp64
// MMA accumulators at the start and written back at the end.  256 threads,
// 8 warps of 32 x 32, two CTAs per SM so that one CTA's loads overlap the
// other's arithmetic.
enum StepBPart { kAll = 0, kNext = 1, kRest = 2 };

// Block steps per bulk update (D, K = 64 D) by order: the bulk update of
// the large orders is bound by its passes over the trailing matrix, which D
// divides; at n = 4096 the diagonal chain bounds the factorisation (3.24 ms
// at D = 1, 3.37 at D = 2, 3.45 at D = 4).  Measured on one B200:
// n = 11008 42.4 / 37.2 / 35.4 ms and n = 28672 581 (D = 2) / 537 ms
// (D = 4).
constexpr int64_t kMultiStepMinN = 8192;
constexpr int kMaxSteps = 4;
int bulk_steps(int64_t n) { return n >= kMultiStepMinN ? kMaxSteps : 1; }

// CTAs of a launch: kNext covers `ncols` Cholesky column tiles and `xtiles`
// substitution row tiles; kRest the Cholesky tiles right of column tile 0
// and `xtiles` substitution row tiles.
int64_t step_b_ctas(int64_t tr, int64_t xcols, int part, int ncols, int64_t xtiles) {
  if (part == kNext) return tr * ncols + xtiles * xcols;
  if (part == kRest) return tr * tr + xtiles * xcols;
  return tr * (tr + 1) + tr * xcols;
}

constexpr int TBM = 128, TBN = 64;
constexpr int SA = TBM + 4, SB = TBN + 4;   // padded k-row strides (doubles)
constexpr size_t kStepBSmem = (size_t)NB * (SA + SB) * sizeof(double);   // 102 KB


// With Dnext != NULL (kNext launches), CTA 0 (row tile 0 of column block
// k+1, which holds the next diagonal block) goes on, once its tile is
// stored, to factor that diagonal block and write its inverse factor to
// Dnext: the next block step's diagonal factorisation without a launch of
// its own.
// Depth: the update is over `kdepth` (64 D) panel rows, Pt rows 0 ..
// kdepth - 1 from `Pt` and the inverse rows from X row xk0 (D > 1: the bulk
// update of D block steps at once, their panels in adjacent buffers).  A
// kNext launch covers `ncols` Cholesky column tiles and the first `xrows`
// substitution rows from `base` (ceil(xrows / 128) row tiles, the last one
// stored in part); a kRest launch's substitution tiles start at row
// base + xoff.
__global__ void __launch_bounds__(256, 2) step_b_kernel(double* __restrict__ A, double* __restrict__ X,
                                                       const double* __restrict__ Pt, int64_t ld, int64_t k0,
                                                       int64_t tr, int part, int64_t n, double* __restrict__ Dnext,
                                                       int32_t* info, int kdepth, int64_t xk0, int ncols, int xrows,
                                                       int64_t xoff) {
  extern __shared__ __align__(16) double sm[];
  double* As = sm;               // [64][SA]
  double* Bs = sm + NB * SA;     // [64][SB]
  const int64_t base = k0 + NB;
  const int64_t xcols = base / TBN;
  const int64_t bid = blockIdx.x;
  int64_t ti = -1, tj = 0, xrow0 = 0, cb = 0;   // Cholesky tile (ti, tj), or substitution tile (rows xrow0.., cb)
  int store_rows = TBM;
  if (part == kNext) {
    if (bid < tr * ncols) {
      ti = bid % tr;
      tj = bid / tr;
    } else {
      const int64_t x = bid - tr * ncols, rt = x / xcols;
      cb = x % xcols;
      xrow0 = base + rt * TBM;
      store_rows = (int)std::min<int64_t>(TBM, xrows - rt * TBM);
    }
  } else if (part == kRest) {
    if (bid < tr * tr) {
      int64_t q = (int64_t)sqrt((double)bid);
      while (q * q > bid) --q;
      while ((q + 1) * (q + 1) <= bid) ++q;
      ti = q;
      tj = bid - q * q + 1;
    } else {
      xrow0 = base + xoff + ((bid - tr * tr) / xcols) * TBM;
      cb = (bid - tr * tr) % xcols;
    }
  } else {
    if (bid < tr * (tr + 1)) rect_index(bid, &ti, &tj);
    else {
      xrow0 = base + ((bid - tr * (tr + 1)) / xcols) * TBM;
      cb = (bid - tr * (tr + 1)) % xcols;
    }
  }
  double* C;
  const double* opA;
  const double* opB;
  if (ti >= 0) {
    C = A + (base + ti * TBM) * ld + base + tj * TBN;
    opA = Pt + base + ti * TBM;
    opB = Pt + base + tj * TBN;
  } else {
    C = X + xrow0 * ld + cb * TBN;
    opA = Pt + xrow0;
    opB = X + xk0 * ld + cb * TBN;
  }
  const int t = threadIdx.x;
  const int warp = t / 32, lane = t % 32;
  const int wm = warp / 2, wn = warp % 2;
  const int fr = lane / 4, fc = lane % 4;
  kq::pdl_wait();
  // operands of the 64-deep half h of the update, in four 16-deep groups
  auto stage = [&](int h) {
#pragma unroll
    for (int g = 0; g < 4; ++g) {
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int id = u * 256 + t;
        const int kk = 16 * g + id / 64, cc = id % 64;
        cp_async16(As + kk * SA + 2 * cc, opA + (64 * h + kk) * ld + 2 * cc);
      }
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int id = u * 256 + t;
        const int kk = 16 * g + id / 32, cc = id % 32;
        cp_async16(Bs + kk * SB + 2 * cc, opB + (64 * h + kk) * ld + 2 * cc);
      }
      cp_commit();
    }
  };
  stage(0);
  double acc[4][4][2];
#pragma unroll
  for (int rt = 0; rt < 4; ++rt)
#pragma unroll
    for (int ct = 0; ct < 4; ++ct) {
      const double2 v =
          *reinterpret_cast<const double2*>(C + (32 * wm + 8 * rt + fr) * ld + 32 * wn + 8 * ct + 2 * fc);
      acc[rt][ct][0] = v.x;
      acc[rt][ct][1] = v.y;
    }
#pragma unroll 1
  for (int h = 0; h < kdepth / NB; ++h) {
    if (h > 0) {
      __syncthreads();   // every warp is done with the previous half's operands
      stage(h);
    }
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      if (g == 0) cp_wait<3>();
      else if (g == 1) cp_wait<2>();
      else if (g == 2) cp_wait<1>();
      else cp_wait<0>();
      __syncthreads();
#pragma unroll
      for (int ks = 0; ks < 4; ++ks) {
        const int k = 16 * g + 4 * ks + fc;
        double a[4], b[4];
#pragma unroll
        for (int rt = 0; rt < 4; ++rt) a[rt] = -As[k * SA + 32 * wm + 8 * rt + fr];
#pragma unroll
        for (int ct = 0; ct < 4; ++ct) b[ct] = Bs[k * SB + 32 * wn + 8 * ct + fr];
#pragma unroll
        for (int rt = 0; rt < 4; ++rt)
#pragma unroll
          for (int ct = 0; ct < 4; ++ct) dmma_acc(acc[rt][ct][0], acc[rt][ct][1], a[rt], b[ct]);
      }
    }
  }
  // a substitution tile of a kNext launch may store only its first rows
  // (warps 0-3 hold rows 0-63)
  if (32 * wm < store_rows) {
#pragma unroll
    for (int rt = 0; rt < 4; ++rt)
#pragma unroll
      for (int ct = 0; ct < 4; ++ct)
        *reinterpret_cast<double2*>(C + (32 * wm + 8 * rt + fr) * ld + 32 * wn + 8 * ct + 2 * fc) =
            make_double2(acc[rt][ct][0], acc[rt][ct][1]);
  }
  if (Dnext && bid == 0) {
    __syncthreads();   // the tile's stores are visible to the whole CTA; the operand smem is free
    potrf_block(A, ld, n, base, (int)(n - base < NB ? n - base : NB), Dnext, info, sm);
  }
}


// X = identity on the first n rows and columns, zero elsewhere (ld x ld).
__global__ void identity_kernel(double* __restrict__ X, int64_t n, int64_t ld) {
  const int64_t total = ld * ld;
  for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
       idx += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = idx / ld, c = idx % ld;
    X[idx] = (r == c && r < n) ? 1.0 : 0.0;
  }
}

// Uc[i][j] = X[n-1-i][n-1-j] for j >= i, 0 below the diagonal.
__global__ void output_kernel(const double* __restrict__ X, int64_t n, int64_t ld, float* __restrict__ Uc,
                              int64_t lduc) {
  const int64_t i = blockIdx.x;
  for (int64_t j = threadIdx.x; j < n; j += blockDim.x) {
    Uc[i * lduc + j] = (j >= i) ? (float)X[(n - 1 - i) * ld + (n - 1 - j)] : 0.f;
  }
}

struct CholWs {
  double* A;
  double* X;
  double* Pt;
  double* Dinv;
  double* lam;
  int64_t ld;
};

// The look-ahead needs a second stream and a few events per (device, caller
// stream), so that factorisations enqueued on different caller streams keep
// their chains apart and run concurrently; created on first use by each host
// thread and kept for its lifetime.
struct LookAhead {
  int device = -1;
  cudaStream_t caller = nullptr;
  cudaStream_t s1 = nullptr;
  cudaEvent_t ev[4] = {};
};

kq_status look_ahead(cudaStream_t caller, LookAhead** out) {
  thread_local LookAhead cache[32];
  int dev = 0;
  KQ_TRY(kq::cuda_check(cudaGetDevice(&dev), "kq_chol_inv: cudaGetDevice"));
  LookAhead* la = nullptr;
  for (auto& c : cache)
    if (c.device == dev && c.caller == caller) la = &c;
  if (!la) {
    for (auto& c : cache)
      if (c.device < 0) {
        la = &c;
        break;
      }
    if (!la) return kq::fail(KQ_ERR_UNSUPPORTED_SHAPE, "kq_chol_inv: more than 32 (device, stream) pairs");
    la->caller = caller;
    int least = 0, greatest = 0;
    KQ_TRY(kq::cuda_check(cudaDeviceGetStreamPriorityRange(&least, &greatest), "kq_chol_inv: priority range"));
    KQ_TRY(kq::cuda_check(cudaStreamCreateWithPriority(&la->s1, cudaStreamNonBlocking, greatest),
                          "kq_chol_inv: stream"));
    for (auto& e : la->ev) KQ_TRY(kq::cuda_check(cudaEventCreateWithFlags(&e, cudaEventDisableTiming), "kq_chol_inv: event"));
    la->device = dev;
  }
  *out = la;
  return KQ_OK;
}

int64_t padded_ld(int64_t n) { return (int64_t)kq::align_up((size_t)n, TB) + TB; }

size_t ws_layout(int64_t n, CholWs* w, void* base) {
  const int64_t nblk = kq::cdiv(n, NB);
  const int64_t ld = padded_ld(n);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off = kq::align_up(off + bytes, 256);
    return o;
  };
  size_t oA = take((size_t)ld * ld * sizeof(double));
  size_t oX = take((size_t)ld * ld * sizeof(double));
  size_t oP = take((size_t)2 * kMaxSteps * NB * ld * sizeof(double));   // 2 D panel buffers
  size_t oD = take((size_t)nblk * NB * NB * sizeof(double));
  size_t oL = take(sizeof(double));
  if (w && base) {
    char* b = static_cast<char*>(base);
    w->A = reinterpret_cast<double*>(b + oA);
    w->X = reinterpret_cast<double*>(b + oX);
    w->Pt = reinterpret_cast<double*>(b + oP);
    w->Dinv = reinterpret_cast<double*>(b + oD);
    w->lam = reinterpret_cast<double*>(b + oL);
    w->ld = ld;
  }
  return off;
}

}  // namespace

extern "C" size_t kq_chol_inv_workspace_size(int64_t n) {
  if (n < 1) return 0;
  return ws_layout(n, nullptr, nullptr);
}

extern "C" kq_status kq_chol_inv(const float* H, int64_t n, int64_t ldh, float damp_frac, float* Uc, int64_t lduc,
                                 uint8_t* dead_mask, void* ws, size_t ws_bytes, int32_t* info, kq_stream_t stream) {
  if (!H || !Uc || !info) return kq::fail(KQ_ERR_INVALID_ARG, "kq_chol_inv: NULL pointer");
  if (n < 1 || n > 65536) return kq::fail(KQ_ERR_UNSUPPORTED_SHAPE, "kq_chol_inv: n outside 1..65536");
  if (ldh < n || lduc < n) return kq::fail(KQ_ERR_INVALID_ARG, "kq_chol_inv: leading dimension too small");
  if (!(damp_frac >= 0.f) || !isfinite(damp_frac)) return kq::fail(KQ_ERR_INVALID_ARG, "kq_chol_inv: damp_frac");
  if (!ws || !kq::aligned(ws, 256) || ws_bytes < kq_chol_inv_workspace_size(n))
    return kq::fail(KQ_ERR_WORKSPACE, "kq_chol_inv: workspace too small or not 256-byte aligned");
  cudaStream_t st = (cudaStream_t)stream;
  CholWs w;
  ws_layout(n, &w, ws);
  const int64_t ld = w.ld;
  static_assert(kStepASmem <= 227 * 1024 && 2 * (kStepBSmem + 1024) <= 228 * 1024, "smem");
  static_assert(kPotrfSmem <= kStepBSmem, "the fused diagonal factorisation reuses step b's shared memory");
  KQ_TRY(kq::cuda_check(cudaFuncSetAttribute(potrf_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kPotrfSmem), "attr"));
  KQ_TRY(kq::cuda_check(cudaFuncSetAttribute(step_a_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kStepASmem), "attr"));
  KQ_TRY(kq::cuda_check(cudaFuncSetAttribute(step_b_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kStepBSmem), "attr"));

  const unsigned nt = (unsigned)kq::cdiv(ld, 32);
  prep_kernel<<<dim3(nt, nt), dim3(32, 8), 0, st>>>(H, ldh, n, w.A, ld, dead_mask, info);
  KQ_TRY(kq::launch_check("kq_chol_inv prep"));
  damp_kernel<<<1, 1024, 0, st>>>(w.A, n, ld, (double)damp_frac, w.lam);
  KQ_TRY(kq::launch_check("kq_chol_inv damp"));
  identity_kernel<<<1184, 256, 0, st>>>(w.X, n, ld);
  KQ_TRY(kq::launch_check("kq_chol_inv identity"));
  KQ_TRY(kq::cuda_check(cudaMemsetAsync(w.Pt, 0, (size_t)2 * kMaxSteps * NB * ld * sizeof(double), st),
                        "kq_chol_inv memset"));

  // Cholesky of the reversed matrix and the inverse of its factor, formed
  // together.  Block step k: factor diagonal block k (potrf), form its panel
  // and the k-th block row of the inverse (step a), then the trailing update
  // (step b).  Look-ahead: the chain potrf -> step a -> update of what block
  // k+1 needs (step b, kNext) runs on a high-priority stream s1, while the
  // rest of the trailing update (kRest) runs on the caller's stream; kNext of
  // step k+1 waits for kRest of step k (both update column block k+2), and
  // the transposed panel alternates between two buffers.
  LookAhead* la = nullptr;
  KQ_TRY(look_ahead(st, &la));
  cudaStream_t s1 = la->s1;
  cudaEvent_t ev_fork = la->ev[0], ev_a = la->ev[1], ev_rest[2] = {la->ev[2], la->ev[3]};
  KQ_TRY(kq::cuda_check(cudaEventRecord(ev_fork, st), "kq_chol_inv: record"));
  KQ_TRY(kq::cuda_check(cudaStreamWaitEvent(s1, ev_fork, 0), "kq_chol_inv: wait"));
  const int64_t nblk = kq::cdiv(n, NB);
  // Bulk updates of D block steps (D = bulk_steps(n)): the steps form groups
  // [g0, g0 + D); step k's kNext updates column blocks k+1 .. g0+D and their
  // substitution rows (D = 1: column block k+1 and the rows of blocks k+1,
  // k+2), so the diagonal chain never waits for a bulk update inside the
  // group; the group's last step's kRest applies the group's D panels
  // (K = 64 D) to the column blocks and substitution rows beyond.  Every
  // (panel, block) pair is updated exactly once, before the block is
  // factored or read as a panel.  The panels of two groups alternate in 2 D
  // buffers, so a group's panels stay until its kRest has read them (the
  // next group's first kNext waits for that kRest, and every later panel
  // step follows that kNext on the chain's stream).
  const int D = bulk_steps(n);
  bool rest_pending = false;   // a kRest that the next kNext must wait for
  int pending_ev = 0;
  for (int64_t b = 0; b < nblk; ++b) {
    const int64_t k0 = b * NB;
    const int kb = (int)std::min<int64_t>(NB, n - k0);
    double* Dk = w.Dinv + b * NB * NB;
    double* Pt = w.Pt + (b % (2 * D)) * NB * ld;
    const int p = (int)(b % D);   // position in the group
    // The chain potrf -> step a -> kNext -> step a ... runs as programmatic
    // dependents on s1: each kernel is scheduled while its predecessor
    // finishes and waits for it (griddepcontrol.wait) before reading.
    // Block 0's diagonal factorisation has a launch of its own; every later
    // one is done by the previous step's kNext launch (its CTA 0).
    if (b == 0)
      KQ_TRY(kq::launch_ex("kq_chol_inv potrf", false, potrf_kernel, dim3(1), dim3(256), kPotrfSmem, s1, w.A, ld, n,
                           k0, kb, Dk, info));
    const int64_t tp = kq::cdiv(n - k0 - kb, 128);   // > 0 only when kb == 64
    const int64_t xt = kq::cdiv(k0 + kb, 128);
    KQ_TRY(kq::launch_ex("kq_chol_inv step a", b > 0, step_a_kernel, dim3((unsigned)(tp + xt)), dim3(256), kStepASmem,
                         s1, w.A, w.X, Pt, ld, k0, tp, Dk));
    if (tp > 0) {
      const int64_t base = k0 + NB;
      const int64_t tr = kq::cdiv(n - base, TBM), xcols = base / TBN;
      const bool do_rest = (p == D - 1);
      if (do_rest) {
        // the group's D panels (D = 1: this step's alone)
        const int64_t g0 = b - (D - 1);
        const double* Pr = w.Pt + (g0 % (2 * D)) * NB * ld;
        const int64_t xoff = D == 1 ? TBM : NB;
        const int64_t xtiles = std::max<int64_t>(0, kq::cdiv(n - base - xoff, TBM));
        KQ_TRY(kq::cuda_check(cudaEventRecord(ev_a, s1), "kq_chol_inv: record"));
        KQ_TRY(kq::cuda_check(cudaStreamWaitEvent(st, ev_a, 0), "kq_chol_inv: wait"));
        step_b_kernel<<<(unsigned)step_b_ctas(tr, xcols, kRest, 1, xtiles), 256, kStepBSmem, st>>>(
            w.A, w.X, Pr, ld, k0, tr, kRest, n, nullptr, info, D * NB, g0 * NB, 1, TBM, xoff);
        KQ_TRY(kq::launch_check("kq_chol_inv step b"));
        KQ_TRY(kq::cuda_check(cudaEventRecord(ev_rest[b & 1], st), "kq_chol_inv: record"));
      }
      if (rest_pending) {
        KQ_TRY(kq::cuda_check(cudaStreamWaitEvent(s1, ev_rest[pending_ev], 0), "kq_chol_inv: wait"));
        rest_pending = false;
      }
      // column blocks b+1 .. g0+D (those that exist) and their substitution rows
      const int64_t ahead = D == 1 ? 1 : D - p;
      const int ncols = (int)std::min<int64_t>(ahead, kq::cdiv(n - base, NB));
      const int64_t xrows = D == 1 ? TBM : std::min<int64_t>(ahead * NB, n - base);
      const int64_t nxt = kq::cdiv(xrows, TBM);
      step_b_kernel<<<(unsigned)step_b_ctas(tr, xcols, kNext, ncols, nxt), 256, kStepBSmem, s1>>>(
          w.A, w.X, Pt, ld, k0, tr, kNext, n, w.Dinv + (b + 1) * NB * NB, info, NB, k0, ncols, (int)xrows, 0);
      KQ_TRY(kq::launch_check("kq_chol_inv step b"));
      if (do_rest) {
        rest_pending = true;
        pending_ev = (int)(b & 1);
      }
    }
  }
  KQ_TRY(kq::cuda_check(cudaEventRecord(ev_fork, s1), "kq_chol_inv: record"));
  KQ_TRY(kq::cuda_check(cudaStreamWaitEvent(st, ev_fork, 0), "kq_chol_inv: wait"));
  output_kernel<<<(unsigned)n, 256, 0, st>>>(w.X, n, ld, Uc, lduc);
  KQ_TRY(kq::launch_check("kq_chol_inv output"));
  kq::clear_error();
  return KQ_OK;
}
