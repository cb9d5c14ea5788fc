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
// Blocked right-looking algorithms over nb = 64 tiles:
//   per block column k: factor + invert the diagonal block (1 CTA); then one
//   launch for the panel X = A_panel L_kk^-T (GEMM with the inverted block)
//   and row block k of the inverse, X_k = L_kk^-1 B_k (forward substitution
//   on B = I); then one launch for the trailing lower-triangle update
//   A -= P P^T and the substitution update B_below -= L_below,k X_k.
#include <math.h>

#include <algorithm>

#include "kq_internal.cuh"

namespace {

constexpr int NB = 64;
constexpr int kPad = NB + 1;
constexpr int kGemmThreads = 256;
constexpr size_t kGemmSmem = 2 * NB * kPad * sizeof(double);

__device__ __forceinline__ int64_t dmin64(int64_t a, int64_t b) { return a < b ? a : b; }

// S[k * kPad + x] = G[x * s_x + k * s_k] for x < xv, k < kv, else 0.
__device__ __forceinline__ void load_tile(double* S, const double* __restrict__ G, int64_t s_x, int64_t s_k, int xv,
                                          int kv) {
  if (s_k == 1) {
    for (int idx = threadIdx.x; idx < NB * NB; idx += blockDim.x) {
      int k = idx % NB, x = idx / NB;
      S[k * kPad + x] = (x < xv && k < kv) ? G[x * s_x + k] : 0.0;
    }
  } else {
    for (int idx = threadIdx.x; idx < NB * NB; idx += blockDim.x) {
      int x = idx % NB, k = idx / NB;
      S[k * kPad + x] = (x < xv && k < kv) ? G[x * s_x + k * s_k] : 0.0;
    }
  }
}

// C[r][c] = alpha * sum_k A(r,k) B(k,c) + beta * C[r][c] for r < rv, c < cv, on a
// 64x64 tile.  A(r,k) = Ag[r*sar + k*sak], B(k,c) = Bg[c*sbc + k*sbk].
// 256 threads, 4x4 outputs each at rows ty + 16 i, cols tx + 16 j.
__device__ void gemm_tile(double* smem, const double* Ag, int64_t sar, int64_t sak, const double* Bg, int64_t sbc,
                          int64_t sbk, int kv, double* C, int64_t ldc, int rv, int cv, double alpha, double beta) {
  double* As = smem;
  double* Bs = smem + NB * kPad;
  load_tile(As, Ag, sar, sak, rv, kv);
  load_tile(Bs, Bg, sbc, sbk, cv, kv);
  __syncthreads();
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  double acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.0;
#pragma unroll 4
  for (int k = 0; k < NB; ++k) {
    double a[4], b[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) a[i] = As[k * kPad + ty + 16 * i];
#pragma unroll
    for (int j = 0; j < 4; ++j) b[j] = Bs[k * kPad + tx + 16 * j];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[i][j] = fma(a[i], b[j], acc[i][j]);
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    int r = ty + 16 * i;
    if (r >= rv) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      int c = tx + 16 * j;
      if (c >= cv) continue;
      double* p = C + (int64_t)r * ldc + c;
      *p = alpha * acc[i][j] + (beta != 0.0 ? beta * *p : 0.0);
    }
  }
}

// A (lower part) = reversed H (fp64); dead columns get diagonal 1; NaN/Inf reported.
__global__ void prep_kernel(const float* __restrict__ H, int64_t ldh, int64_t n, double* __restrict__ A,
                            uint8_t* __restrict__ dead, int32_t* info) {
  const int64_t ii = (int64_t)blockIdx.y * 32 + threadIdx.y;
  const int64_t jj = (int64_t)blockIdx.x * 32 + threadIdx.x;
  if ((int64_t)blockIdx.x > (int64_t)blockIdx.y) return;
  for (int s = 0; s < 32; s += 8) {
    int64_t i = ii + s;
    if (i >= n || jj >= n || jj > i) continue;
    double v = (double)H[(n - 1 - i) * ldh + (n - 1 - jj)];
    if (!isfinite(v)) kq::report(info, KQ_ERR_NONFINITE, n - 1 - i);
    if (i == jj) {
      bool d = (v == 0.0);
      if (d) v = 1.0;
      if (dead) dead[n - 1 - i] = d ? 1 : 0;
    }
    A[i * n + jj] = v;
  }
}

// lambda = damp * mean(diag A); diag A += lambda.  One CTA, fixed-order sum.
__global__ void damp_kernel(double* __restrict__ A, int64_t n, double damp, double* __restrict__ lam_out) {
  __shared__ double red[1024];
  double s = 0.0;
  for (int64_t i = threadIdx.x; i < n; i += blockDim.x) s += A[i * n + i];
  red[threadIdx.x] = s;
  __syncthreads();
  for (int w = blockDim.x / 2; w > 0; w >>= 1) {
    if (threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
    __syncthreads();
  }
  const double lam = damp * (red[0] / (double)n);
  for (int64_t i = threadIdx.x; i < n; i += blockDim.x) A[i * n + i] += lam;
  if (threadIdx.x == 0) *lam_out = lam;
}

// Factor the kb x kb diagonal block at (k0, k0) in place (lower Cholesky) and
// write its lower-triangular inverse, padded to 64 x 64 with the identity, to
// Dinv.  256 threads: four per row (Cholesky, left-looking by columns, the
// dot products split four ways) or four per column (inverse, forward
// substitution with split dot products).  Two block barriers per column.
__global__ void __launch_bounds__(256) potrf_kernel(double* __restrict__ A, int64_t n, int64_t k0, int kb,
                                                    double* __restrict__ Dinv, int32_t* info) {
  extern __shared__ double psm[];
  double (*a)[kPad] = reinterpret_cast<double (*)[kPad]>(psm);
  double (*inv)[kPad] = reinterpret_cast<double (*)[kPad]>(psm + NB * kPad);
  __shared__ double rdiag[NB];
  __shared__ double diag0[NB];   // the block's diagonal before factorisation (read-only below)
  const int t = threadIdx.x, g = t >> 2, part = t & 3;
  for (int idx = t; idx < NB * NB; idx += blockDim.x) {
    int i = idx / NB, j = idx % NB;
    double v;
    if (i < kb && j < kb) v = (j <= i) ? A[(k0 + i) * n + k0 + j] : 0.0;
    else v = (i == j) ? 1.0 : 0.0;
    a[i][j] = v;
    if (i == j) diag0[i] = v;
  }
  __syncthreads();
  // Column j: every 4-thread group forms its own row's dot product and the
  // pivot row's (same operands, same order, so every group holds the same
  // pivot), scales by 1/sqrt(pivot) and the column is final after one barrier.
  for (int j = 0; j < NB; ++j) {
    const int i = g;
    double s = 0.0, sp = 0.0;
    for (int l = part; l < j; l += 4) {
      sp = fma(a[j][l], a[j][l], sp);
      if (i > j) s = fma(a[i][l], a[j][l], s);
    }
    s += __shfl_xor_sync(0xffffffffu, s, 1);
    s += __shfl_xor_sync(0xffffffffu, s, 2);
    sp += __shfl_xor_sync(0xffffffffu, sp, 1);
    sp += __shfl_xor_sync(0xffffffffu, sp, 2);
    double d = diag0[j] - sp;
    if (!(d > 0.0) || !isfinite(d)) {
      if (i == j && part == 0) kq::report(info, KQ_ERR_NOT_PD, n - 1 - (k0 + j));
      d = 1.0;
    }
    const double rs = rsqrt(d);
    if (part == 0) {
      if (i == j) a[j][j] = d * rs;
      else if (i > j) a[i][j] = (a[i][j] - s) * rs;
    }
    __syncthreads();
  }
  if (t < NB) rdiag[t] = 1.0 / a[t][t];
  __syncthreads();
  {
    const int c = g;
    for (int i = 0; i < NB; ++i) {
      double s = 0.0;
      if (i > c)
        for (int l = c + part; l < i; l += 4) s = fma(a[i][l], inv[l][c], s);
      s += __shfl_xor_sync(0xffffffffu, s, 1);
      s += __shfl_xor_sync(0xffffffffu, s, 2);
      if (part == 0) inv[i][c] = (i < c) ? 0.0 : (i == c ? rdiag[c] : -s * rdiag[i]);
      __syncwarp();
    }
  }
  __syncthreads();
  for (int idx = t; idx < NB * NB; idx += blockDim.x) {
    int i = idx / NB, j = idx % NB;
    Dinv[idx] = inv[i][j];
    if (i < kb && j < kb && j <= i) A[(k0 + i) * n + k0 + j] = a[i][j];
  }
}

__device__ __forceinline__ void tri_index(int64_t l, int64_t* ti, int64_t* tj) {
  int64_t t = (int64_t)((sqrt(8.0 * (double)l + 1.0) - 1.0) * 0.5);
  while (t * (t + 1) / 2 > l) --t;
  while ((t + 1) * (t + 2) / 2 <= l) ++t;
  *ti = t;
  *tj = l - t * (t + 1) / 2;
}

// One launch per block step k (after the diagonal factorisation):
//   CTAs [0, tr):     panel rows below the block, X = A_panel Dinv_k^T;
//   CTAs [tr, ...):   forward substitution, X_k = Dinv_k B_k for column
//                     blocks 0..k of the inverse being formed in B.
__global__ void __launch_bounds__(kGemmThreads) step_a_kernel(double* __restrict__ A, double* __restrict__ X,
                                                             int64_t n, int64_t k0, int kb, int64_t tr,
                                                             const double* __restrict__ Dinv) {
  extern __shared__ double smem[];
  if ((int64_t)blockIdx.x < tr) {
    const int64_t r0 = k0 + kb + (int64_t)blockIdx.x * NB;
    const int rv = (int)dmin64(NB, n - r0);
    double* P = A + r0 * n + k0;
    // A(r,k) = P[r*n + k];  B(k,c) = Dinv[c][k]
    gemm_tile(smem, P, n, 1, Dinv, NB, 1, kb, P, n, rv, kb, 1.0, 0.0);
  } else {
    const int64_t c0 = ((int64_t)blockIdx.x - tr) * NB;
    const int cv = (int)dmin64(NB, n - c0);
    double* T = X + k0 * n + c0;
    // A(r,k) = Dinv[r*64 + k];  B(k,c) = T[k*n + c]
    gemm_tile(smem, Dinv, NB, 1, T, 1, n, kb, T, n, kb, cv, 1.0, 0.0);
  }
}

// One launch per block step k (after step_a):
//   CTAs [0, tr(tr+1)/2):  Cholesky trailing update of the lower tiles,
//                          A[ti][tj] -= P_ti P_tj^T;
//   CTAs after:            substitution update of the rows below,
//                          B[r][c] -= L[r][k] X_k[c] for column blocks c <= k.
__global__ void __launch_bounds__(kGemmThreads) step_b_kernel(double* __restrict__ A, double* __restrict__ X,
                                                             int64_t n, int64_t k0, int kb, int64_t tr,
                                                             int64_t kblocks) {
  extern __shared__ double smem[];
  const int64_t ntri = tr * (tr + 1) / 2;
  const int64_t base = k0 + kb;
  if ((int64_t)blockIdx.x < ntri) {
    int64_t ti, tj;
    tri_index(blockIdx.x, &ti, &tj);
    const int64_t r0 = base + ti * NB, c0 = base + tj * NB;
    const int rv = (int)dmin64(NB, n - r0), cv = (int)dmin64(NB, n - c0);
    gemm_tile(smem, A + r0 * n + k0, n, 1, A + c0 * n + k0, n, 1, kb, A + r0 * n + c0, n, rv, cv, -1.0, 1.0);
  } else {
    const int64_t idx = (int64_t)blockIdx.x - ntri;
    const int64_t cb = idx % kblocks, rb = idx / kblocks;
    const int64_t c0 = cb * NB, r0 = base + rb * NB;
    const int cv = (int)dmin64(NB, n - c0), rv = (int)dmin64(NB, n - r0);
    // A(r,k) = L[(r0+r)*n + k0 + k];  B(k,c) = X[(k0+k)*n + c0 + c]
    gemm_tile(smem, A + r0 * n + k0, n, 1, X + k0 * n + c0, 1, n, kb, X + r0 * n + c0, n, rv, cv, -1.0, 1.0);
  }
}

__global__ void identity_kernel(double* __restrict__ X, int64_t n) {
  int64_t total = n * n;
  for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
       idx += (int64_t)gridDim.x * blockDim.x)
    X[idx] = (idx / n == idx % n) ? 1.0 : 0.0;
}

// Uc[i][j] = X[n-1-i][n-1-j] for j >= i, 0 below the diagonal.
__global__ void output_kernel(const double* __restrict__ X, int64_t n, float* __restrict__ Uc, int64_t lduc) {
  const int64_t i = blockIdx.x;
  for (int64_t j = threadIdx.x; j < n; j += blockDim.x) {
    Uc[i * lduc + j] = (j >= i) ? (float)X[(n - 1 - i) * n + (n - 1 - j)] : 0.f;
  }
}

struct CholWs {
  double* A;
  double* X;
  double* Dinv;
  double* lam;
};

size_t ws_layout(int64_t n, CholWs* w, void* base) {
  const int64_t nblk = kq::cdiv(n, NB);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off = kq::align_up(off + bytes, 256);
    return o;
  };
  size_t oA = take((size_t)n * n * sizeof(double));
  size_t oX = take((size_t)n * n * sizeof(double));
  size_t oD = take((size_t)nblk * NB * NB * sizeof(double));
  size_t oL = take(sizeof(double));
  if (w && base) {
    char* b = static_cast<char*>(base);
    w->A = reinterpret_cast<double*>(b + oA);
    w->X = reinterpret_cast<double*>(b + oX);
    w->Dinv = reinterpret_cast<double*>(b + oD);
    w->lam = reinterpret_cast<double*>(b + oL);
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
  static_assert(kGemmSmem <= 227 * 1024, "smem");
  KQ_TRY(kq::cuda_check(cudaFuncSetAttribute(potrf_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kGemmSmem), "attr"));
  KQ_TRY(kq::cuda_check(cudaFuncSetAttribute(step_a_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kGemmSmem), "attr"));
  KQ_TRY(kq::cuda_check(cudaFuncSetAttribute(step_b_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kGemmSmem), "attr"));

  const unsigned nt = (unsigned)kq::cdiv(n, 32);
  prep_kernel<<<dim3(nt, nt), dim3(32, 8), 0, st>>>(H, ldh, n, w.A, dead_mask, info);
  KQ_TRY(kq::launch_check("kq_chol_inv prep"));
  damp_kernel<<<1, 1024, 0, st>>>(w.A, n, (double)damp_frac, w.lam);
  KQ_TRY(kq::launch_check("kq_chol_inv damp"));
  identity_kernel<<<1024, 256, 0, st>>>(w.X, n);
  KQ_TRY(kq::launch_check("kq_chol_inv identity"));

  // Cholesky of the reversed matrix and the inverse of its factor, formed
  // together: step k factors diagonal block k, then (a) its panel and the
  // k-th block row of the inverse, then (b) the trailing Cholesky update and
  // the substitution update of the inverse's rows below.
  const int64_t nblk = kq::cdiv(n, NB);
  for (int64_t b = 0; b < nblk; ++b) {
    const int64_t k0 = b * NB;
    const int kb = (int)std::min<int64_t>(NB, n - k0);
    double* Dk = w.Dinv + b * NB * NB;
    potrf_kernel<<<1, 256, kGemmSmem, st>>>(w.A, n, k0, kb, Dk, info);
    KQ_TRY(kq::launch_check("kq_chol_inv potrf"));
    const int64_t tr = kq::cdiv(n - k0 - kb, NB);
    step_a_kernel<<<(unsigned)(tr + b + 1), kGemmThreads, kGemmSmem, st>>>(w.A, w.X, n, k0, kb, tr, Dk);
    KQ_TRY(kq::launch_check("kq_chol_inv step a"));
    if (tr > 0) {
      step_b_kernel<<<(unsigned)(tr * (tr + 1) / 2 + tr * (b + 1)), kGemmThreads, kGemmSmem, st>>>(w.A, w.X, n, k0,
                                                                                                   kb, tr, b + 1);
      KQ_TRY(kq::launch_check("kq_chol_inv step b"));
    }
  }
  output_kernel<<<(unsigned)n, 256, 0, st>>>(w.X, n, Uc, lduc);
  KQ_TRY(kq::launch_check("kq_chol_inv output"));
  kq::clear_error();
  return KQ_OK;
}
