// kq_rotate: randomised Hadamard rotations of bidirectional incoherence
// processing (steps a4/a5).
//
// KronQ review (romaanj.github.io/reviews/kronq), Method (1): the input-side
// random rotation is extended to the output side; Unified Hessian-Guided PTQ
// (hub.valency.io/works/W_r72x54u6), Background / Transformations: randomised
// Hadamard transforms are orthogonal channel mixes that keep the layer output.
//
// T = (Q_m kron H_p / sqrt(p)) diag(s), n = m p.  The transform is HBM bound
// (8 bytes per element per pass), so the kernels stage a whole vector (row
// transform) or a strided tile of vectors (column transform) in shared memory,
// run the Walsh-Hadamard butterflies there, and touch HBM once per pass with
// coalesced 128-byte rows.
//
//  * KQ_AXIS_COLS (M <- M T^T, each row transformed): one CTA per row, the row
//    lives in shared memory (n <= 32768 floats).
//  * KQ_AXIS_ROWS (M <- T M, each column transformed): H_p = H_p1 kron H_p2 is
//    split into two passes over 32-column strips.  Pass "inner" applies H_p2 to
//    groups of p2 consecutive rows (plus signs and the 1/sqrt(p) scale); pass
//    "outer" applies H_p1 and Q_m to the m*p1 rows that share one inner index
//    (stride p2).  Each pass reads and writes M once.
#include "kq_internal.cuh"

namespace {

constexpr int kMaxM = 64;
constexpr int kMaxRowN = 32768;
constexpr int kStrip = 32;           // columns per tile in the column transform
constexpr int kMaxP2Log = 9;         // p2 <= 512
constexpr int kMaxOuterRows = 1024;  // m * p1 <= 1024

// In-smem butterflies over blocks of `len` contiguous elements (len = 2^k)
// of a vector of `n` elements, all threads of the CTA cooperating.
__device__ __forceinline__ void fwht_smem(float* x, int n, int len) {
  for (int h = 1; h < len; h <<= 1) {
    for (int idx = threadIdx.x; idx < n / 2; idx += blockDim.x) {
      int i = (idx / h) * (2 * h) + (idx % h);
      float a = x[i], b = x[i + h];
      x[i] = a + b;
      x[i + h] = a - b;
    }
    __syncthreads();
  }
}

// Mix the m blocks of p elements with Q (or Q^T): x[a*p+b] <- sum_a' Q[a][a'] x[a'*p+b].
__device__ __forceinline__ void qmix_smem(float* x, int p, int m, const float* Qs, bool transpose) {
  float tmp[kMaxM];
  for (int b = threadIdx.x; b < p; b += blockDim.x) {
    for (int a = 0; a < m; ++a) tmp[a] = x[a * p + b];
    for (int a = 0; a < m; ++a) {
      float acc = 0.f;
      for (int c = 0; c < m; ++c) acc = fmaf(transpose ? Qs[c * m + a] : Qs[a * m + c], tmp[c], acc);
      x[a * p + b] = acc;
    }
  }
  __syncthreads();
}

// Row transform: M[r, :] <- T M[r, :] (or T^T).  One CTA per row.
__global__ void __launch_bounds__(512) rotate_rows_kernel(float* __restrict__ M, int64_t ld, int n, int log2_p, int m,
                                                          const float* __restrict__ signs,
                                                          const float* __restrict__ Qm, int inverse, float scale) {
  extern __shared__ float sm[];
  float* x = sm;
  float* Qs = sm + n;
  const int p = 1 << log2_p;
  float* row = M + (int64_t)blockIdx.x * ld;
  if (m > 1)
    for (int i = threadIdx.x; i < m * m; i += blockDim.x) Qs[i] = Qm[i];
  if ((n & 3) == 0) {
    const float4* src = reinterpret_cast<const float4*>(row);
    const float4* sg = reinterpret_cast<const float4*>(signs);
    for (int i = threadIdx.x; i < n / 4; i += blockDim.x) {
      float4 v = src[i];
      if (!inverse) {
        float4 s = sg[i];
        v.x *= s.x; v.y *= s.y; v.z *= s.z; v.w *= s.w;
      }
      reinterpret_cast<float4*>(x)[i] = v;
    }
  } else {
    for (int i = threadIdx.x; i < n; i += blockDim.x) x[i] = inverse ? row[i] : row[i] * signs[i];
  }
  __syncthreads();
  if (inverse && m > 1) qmix_smem(x, p, m, Qs, true);
  fwht_smem(x, n, p);
  if (!inverse && m > 1) qmix_smem(x, p, m, Qs, false);
  if ((n & 3) == 0) {
    float4* dst = reinterpret_cast<float4*>(row);
    const float4* sg = reinterpret_cast<const float4*>(signs);
    for (int i = threadIdx.x; i < n / 4; i += blockDim.x) {
      float4 v = reinterpret_cast<float4*>(x)[i];
      v.x *= scale; v.y *= scale; v.z *= scale; v.w *= scale;
      if (inverse) {
        float4 s = sg[i];
        v.x *= s.x; v.y *= s.y; v.z *= s.z; v.w *= s.w;
      }
      dst[i] = v;
    }
  } else {
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
      float v = x[i] * scale;
      row[i] = inverse ? v * signs[i] : v;
    }
  }
}

// Column transform, inner pass: for the group of p2 consecutive rows starting
// at blockIdx.y * p2 and the strip of columns at blockIdx.x * 32, apply signs
// (forward: before), H_p2 along the rows, the 1/sqrt(p) scale, and (inverse:
// after) the signs.
__global__ void __launch_bounds__(256) rotate_cols_inner_kernel(float* __restrict__ M, int64_t ld, int64_t cols,
                                                                int p2, const float* __restrict__ signs, int inverse,
                                                                float scale) {
  extern __shared__ float t[];  // [p2][kStrip]
  const int64_t r0 = (int64_t)blockIdx.y * p2;
  const int64_t c0 = (int64_t)blockIdx.x * kStrip;
  const int c = threadIdx.x % kStrip;
  const int rs = threadIdx.x / kStrip;
  const int rstep = blockDim.x / kStrip;
  const bool cok = c0 + c < cols;
  for (int r = rs; r < p2; r += rstep) {
    float v = cok ? M[(r0 + r) * ld + c0 + c] : 0.f;
    if (!inverse) v *= signs[r0 + r];
    t[r * kStrip + c] = v;
  }
  __syncthreads();
  for (int h = 1; h < p2; h <<= 1) {
    for (int idx = rs; idx < p2 / 2; idx += rstep) {
      int i = (idx / h) * (2 * h) + (idx % h);
      float a = t[i * kStrip + c], b = t[(i + h) * kStrip + c];
      t[i * kStrip + c] = a + b;
      t[(i + h) * kStrip + c] = a - b;
    }
    __syncthreads();
  }
  if (cok) {
    for (int r = rs; r < p2; r += rstep) {
      float v = t[r * kStrip + c] * scale;
      if (inverse) v *= signs[r0 + r];
      M[(r0 + r) * ld + c0 + c] = v;
    }
  }
}

// Column transform, outer pass: rows a*p + b1*p2 + b2 (a < m, b1 < p1) for
// b2 = blockIdx.y, strip blockIdx.x.  Applies H_p1 over b1 and Q_m over a
// (Q_m^T first when inverse; the two commute, they act on different factors).
__global__ void __launch_bounds__(256) rotate_cols_outer_kernel(float* __restrict__ M, int64_t ld, int64_t cols,
                                                                int p, int p1, int p2, int m,
                                                                const float* __restrict__ Qm, int inverse) {
  extern __shared__ float sm[];
  float* Qs = sm;                   // [m*m]
  float* t = sm + kMaxM * kMaxM;    // [m*p1][kStrip]
  const int R = m * p1;
  const int b2 = blockIdx.y;
  const int64_t c0 = (int64_t)blockIdx.x * kStrip;
  const int c = threadIdx.x % kStrip;
  const int rs = threadIdx.x / kStrip;
  const int rstep = blockDim.x / kStrip;
  const bool cok = c0 + c < cols;
  if (m > 1)
    for (int i = threadIdx.x; i < m * m; i += blockDim.x) Qs[i] = Qm[i];
  for (int r = rs; r < R; r += rstep) {
    int a = r / p1, b1 = r % p1;
    int64_t row = (int64_t)a * p + (int64_t)b1 * p2 + b2;
    t[r * kStrip + c] = cok ? M[row * ld + c0 + c] : 0.f;
  }
  __syncthreads();
  // H_p1 over b1 within each a-block (rows a*p1 .. a*p1 + p1 - 1 of the tile)
  for (int h = 1; h < p1; h <<= 1) {
    for (int idx = rs; idx < R / 2; idx += rstep) {
      int i = (idx / h) * (2 * h) + (idx % h);
      float a0 = t[i * kStrip + c], b0 = t[(i + h) * kStrip + c];
      t[i * kStrip + c] = a0 + b0;
      t[(i + h) * kStrip + c] = a0 - b0;
    }
    __syncthreads();
  }
  if (m > 1) {
    float tmp[kMaxM];
    for (int b1 = rs; b1 < p1; b1 += rstep) {
      for (int a = 0; a < m; ++a) tmp[a] = t[(a * p1 + b1) * kStrip + c];
      for (int a = 0; a < m; ++a) {
        float acc = 0.f;
        for (int q = 0; q < m; ++q) acc = fmaf(inverse ? Qs[q * m + a] : Qs[a * m + q], tmp[q], acc);
        t[(a * p1 + b1) * kStrip + c] = acc;
      }
    }
    __syncthreads();
  }
  if (cok) {
    for (int r = rs; r < R; r += rstep) {
      int a = r / p1, b1 = r % p1;
      int64_t row = (int64_t)a * p + (int64_t)b1 * p2 + b2;
      M[row * ld + c0 + c] = t[r * kStrip + c];
    }
  }
}

}  // namespace

extern "C" kq_status kq_rotate(float* M, int64_t rows, int64_t cols, int64_t ld, int axis, const kq_rht* T,
                               int inverse, kq_stream_t stream) {
  if (!M || !T || !T->signs) return kq::fail(KQ_ERR_INVALID_ARG, "kq_rotate: NULL pointer");
  if (rows < 0 || cols < 0 || ld < cols) return kq::fail(KQ_ERR_INVALID_ARG, "kq_rotate: bad sizes");
  if (axis != KQ_AXIS_ROWS && axis != KQ_AXIS_COLS) return kq::fail(KQ_ERR_INVALID_ARG, "kq_rotate: bad axis");
  const int64_t n = T->n;
  const int m = T->m, lp = T->log2_p;
  if (lp < 0 || lp > 15 || m < 1 || m > kMaxM || n != (int64_t)m << lp)
    return kq::fail(KQ_ERR_UNSUPPORTED_SHAPE, "kq_rotate: need n = m * 2^log2_p with 1 <= m <= 64, log2_p <= 15");
  if (m > 1 && !T->Qm) return kq::fail(KQ_ERR_INVALID_ARG, "kq_rotate: Qm is NULL with m > 1");
  if (n != (axis == KQ_AXIS_ROWS ? rows : cols))
    return kq::fail(KQ_ERR_INVALID_ARG, "kq_rotate: T->n does not match the rotated dimension");
  if (!kq::aligned(M, 16) || (ld & 3) || !kq::aligned(T->signs, 16))
    return kq::fail(KQ_ERR_ALIGNMENT, "kq_rotate: M and signs must be 16-byte aligned and ld % 4 == 0");
  if (rows == 0 || cols == 0) return KQ_OK;
  cudaStream_t st = (cudaStream_t)stream;
  const int p = 1 << lp;
  const float scale = (float)(1.0 / sqrt((double)p));
  if (axis == KQ_AXIS_COLS) {
    if (n > kMaxRowN) return kq::fail(KQ_ERR_UNSUPPORTED_SHAPE, "kq_rotate: row length above 32768");
    if (rows > 0x7fffffff) return kq::fail(KQ_ERR_UNSUPPORTED_SHAPE, "kq_rotate: too many rows");
    size_t smem = (size_t)(n + (m > 1 ? m * m : 0)) * sizeof(float);
    KQ_TRY(kq::cuda_check(cudaFuncSetAttribute(rotate_rows_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               (int)smem), "kq_rotate: smem attribute"));
    rotate_rows_kernel<<<(unsigned)rows, 512, smem, st>>>(M, ld, (int)n, lp, m, T->signs, T->Qm, inverse, scale);
    KQ_TRY(kq::launch_check("kq_rotate rows"));
  } else {
    const int lp2 = lp < kMaxP2Log ? lp : kMaxP2Log;
    const int p2 = 1 << lp2, p1 = 1 << (lp - lp2);
    if ((int64_t)m * p1 > kMaxOuterRows)
      return kq::fail(KQ_ERR_UNSUPPORTED_SHAPE, "kq_rotate: m * p / 512 above 1024");
    const unsigned strips = (unsigned)kq::cdiv(cols, kStrip);
    const bool outer = (m > 1 || p1 > 1);
    size_t smem_in = (size_t)p2 * kStrip * sizeof(float);
    size_t smem_out = (size_t)(kMaxM * kMaxM + m * p1 * kStrip) * sizeof(float);
    KQ_TRY(kq::cuda_check(cudaFuncSetAttribute(rotate_cols_inner_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               (int)smem_in), "kq_rotate: smem attribute"));
    KQ_TRY(kq::cuda_check(cudaFuncSetAttribute(rotate_cols_outer_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               (int)smem_out), "kq_rotate: smem attribute"));
    dim3 gin(strips, (unsigned)(n / p2)), gout(strips, (unsigned)p2);
    if (!inverse) {
      rotate_cols_inner_kernel<<<gin, 256, smem_in, st>>>(M, ld, cols, p2, T->signs, 0, scale);
      KQ_TRY(kq::launch_check("kq_rotate cols inner"));
      if (outer) {
        rotate_cols_outer_kernel<<<gout, 256, smem_out, st>>>(M, ld, cols, p, p1, p2, m, T->Qm, 0);
        KQ_TRY(kq::launch_check("kq_rotate cols outer"));
      }
    } else {
      if (outer) {
        rotate_cols_outer_kernel<<<gout, 256, smem_out, st>>>(M, ld, cols, p, p1, p2, m, T->Qm, 1);
        KQ_TRY(kq::launch_check("kq_rotate cols outer"));
      }
      rotate_cols_inner_kernel<<<gin, 256, smem_in, st>>>(M, ld, cols, p2, T->signs, 1, scale);
      KQ_TRY(kq::launch_check("kq_rotate cols inner"));
    }
  }
  kq::clear_error();
  return KQ_OK;
}
