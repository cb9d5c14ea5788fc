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
// run the Walsh-Hadamard butterflies there (radix-16 passes in registers),
// and touch HBM once per pass with coalesced float4 accesses.
//
//  * KQ_AXIS_COLS (M <- M T^T, each row transformed): one CTA per row, the row
//    lives in shared memory (n <= 32768 floats).
//  * KQ_AXIS_ROWS (M <- T M, each column transformed): H_p = H_p1 kron H_p2 is
//    split into two passes over 128-column strips (512-byte row runs).  Pass "inner" applies H_p2 to
//    groups of p2 consecutive rows (plus signs and the 1/sqrt(p) scale); pass
//    "outer" applies H_p1 and Q_m to the m*p1 rows that share one inner index
//    (stride p2).  Each pass reads and writes M once.
#include "kq_internal.cuh"

namespace {

constexpr int kMaxM = 64;
constexpr int kMaxRowN = 32768;
constexpr int kStrip = 128;          // columns per tile in the column transform (512-byte row runs)
constexpr int kMaxP2Log = 7;         // inner pass: p2 <= 128 rows
constexpr int kMaxOuterRows = 256;   // outer pass: m * p1 <= 256 rows

// Shared-memory position of element i of a row: one spare float after every
// 16, so a thread reading 16 consecutive elements, and a warp reading 32
// such runs, meets no bank conflict.
__device__ __forceinline__ int pad16(int i) { return i + (i >> 4); }

// Butterflies over index bits [lo, lo + g) of 2^g register-held elements
// (g <= 4; predicated for g < 4).
__device__ __forceinline__ void fwht_regs(float (&r)[16], int g) {
#pragma unroll
  for (int s = 0; s < 4; ++s) {
    if (s >= g) break;
    const int h = 1 << s;
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      if ((e & h) || e + h >= (1 << g)) continue;
      const float a = r[e], b = r[e + h];
      r[e] = a + b;
      r[e + h] = a - b;
    }
  }
}

// In-place Q_m mix of S strands of m <= 64 values in shared memory:
// element q of strand s at buf[addr(q, s)] becomes sum_c Q[q][c] x_s[c]
// (Q^T when transposing).  A register-tiled small product: thread t owns the
// output rows of group t / 64 (ceil(m / 4) rows) for the four strands
// t % 64 + 64 j of each 256-strand chunk, so every Q value it reads from
// shared memory (a warp-wide broadcast) feeds four FMAs and every strand
// value feeds up to 16.  Must be called by all 256 threads; ends with a
// barrier.
template <typename Addr>
__device__ void qmix_tile(float* buf, const float* Qs, int m, int S, bool transpose, Addr addr) {
  const int t = threadIdx.x, bb = t & 63, ag = t >> 6;
  const int am = (m + 3) >> 2, a0 = ag * am;
  for (int chunk = 0; chunk < S; chunk += 256) {
    float acc[16][4];
#pragma unroll
    for (int i = 0; i < 16; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
    for (int c = 0; c < m; ++c) {
      float xv[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int sj = chunk + bb + 64 * j;
        xv[j] = (sj < S) ? buf[addr(c, sj)] : 0.f;
      }
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        if (i < am && a0 + i < m) {
          const float q = transpose ? Qs[c * m + a0 + i] : Qs[(a0 + i) * m + c];
#pragma unroll
          for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(q, xv[j], acc[i][j]);
        }
      }
    }
    __syncthreads();   // every read of this chunk is done
#pragma unroll
    for (int i = 0; i < 16; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int sj = chunk + bb + 64 * j;
        if (i < am && a0 + i < m && sj < S) buf[addr(a0 + i, sj)] = acc[i][j];
      }
    __syncthreads();
  }
}

// Walsh-Hadamard butterflies over bits [0, k) of the element index of nvec
// vectors held in shared memory, in passes over 4-bit groups of the index:
// each thread gathers the 16 elements of one group into registers, runs the
// butterflies there and scatters them back (index arithmetic by shifts and
// masks only).
//   ROW layout:  element i of vector v at pad16(v * 2^k + i)
//   TILE layout: element i of vector v (v = column + 128 * block) at
//                ((v >> 7) * 2^k + i) * 128 + (v & 127)
template <bool ROW>
__device__ void fwht_passes(float* x, int k, int nvec) {
  for (int lo = 0; lo < k; lo += 4) {
    const int g = min(4, k - lo);
    const int rest_bits = k - g;
    const int groups = nvec << rest_bits;
    for (int grp = threadIdx.x; grp < groups; grp += blockDim.x) {
      int v, rest;
      if (ROW) {
        v = grp >> rest_bits;
        rest = grp & ((1 << rest_bits) - 1);
      } else {
        v = (grp & 127) | ((grp >> (7 + rest_bits)) << 7);
        rest = (grp >> 7) & ((1 << rest_bits) - 1);
      }
      const int base = ((rest >> lo) << (lo + g)) | (rest & ((1 << lo) - 1));
      float r[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        if (e >= (1 << g)) break;
        const int i = base | (e << lo);
        r[e] = ROW ? x[pad16((v << k) + i)] : x[(((v >> 7) << k) + i) * 128 + (v & 127)];
      }
      fwht_regs(r, g);
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        if (e >= (1 << g)) break;
        const int i = base | (e << lo);
        if (ROW) x[pad16((v << k) + i)] = r[e];
        else x[(((v >> 7) << k) + i) * 128 + (v & 127)] = r[e];
      }
    }
    __syncthreads();
  }
}

// Row transform: M[r, :] <- T M[r, :] (or T^T).  One CTA per row; the row
// lives in shared memory in the padded layout.
__global__ void __launch_bounds__(256) rotate_rows_kernel(float* __restrict__ M, int64_t ld, int n, int log2_p, int m,
                                                          const float* __restrict__ signs,
                                                          const float* __restrict__ Qm, int inverse, float scale) {
  extern __shared__ float sm[];
  float* x = sm;
  float* Qs = sm + pad16(n) + 4;
  const int p = 1 << log2_p;
  float* row = M + (int64_t)blockIdx.x * ld;
  if (m > 1)
    for (int i = threadIdx.x; i < m * m; i += blockDim.x) Qs[i] = Qm[i];
  if ((n & 3) == 0) {
    // eight float4 loads of the row (and of the signs) in flight per thread
    const int n4 = n / 4;
    for (int b4 = 0; b4 < n4; b4 += 8 * 256) {
      float4 v[8], sg[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int i4 = b4 + threadIdx.x + 256 * u;
        if (i4 < n4) {
          v[u] = reinterpret_cast<const float4*>(row)[i4];
          sg[u] = inverse ? make_float4(1.f, 1.f, 1.f, 1.f) : reinterpret_cast<const float4*>(signs)[i4];
        }
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int i4 = b4 + threadIdx.x + 256 * u;
        if (i4 < n4) {
          const int i = 4 * i4;
          x[pad16(i)] = v[u].x * sg[u].x;
          x[pad16(i + 1)] = v[u].y * sg[u].y;
          x[pad16(i + 2)] = v[u].z * sg[u].z;
          x[pad16(i + 3)] = v[u].w * sg[u].w;
        }
      }
    }
  } else {
    for (int i = threadIdx.x; i < n; i += blockDim.x) x[pad16(i)] = inverse ? row[i] : row[i] * signs[i];
  }
  __syncthreads();
  auto qmix = [&](bool transpose) {
    qmix_tile(x, Qs, m, p, transpose, [&](int q, int b) { return pad16(q * p + b); });
  };
  if (inverse && m > 1) qmix(true);
  fwht_passes<true>(x, log2_p, m);
  if (!inverse && m > 1) qmix(false);
  if ((n & 3) == 0) {
    for (int i4 = threadIdx.x; i4 < n / 4; i4 += blockDim.x) {
      const int i = 4 * i4;
      float4 v = make_float4(x[pad16(i)] * scale, x[pad16(i + 1)] * scale, x[pad16(i + 2)] * scale,
                             x[pad16(i + 3)] * scale);
      if (inverse) {
        const float4 sg = reinterpret_cast<const float4*>(signs)[i4];
        v.x *= sg.x; v.y *= sg.y; v.z *= sg.z; v.w *= sg.w;
      }
      reinterpret_cast<float4*>(row)[i4] = v;
    }
  } else {
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
      const float v = x[pad16(i)] * scale;
      row[i] = inverse ? v * signs[i] : v;
    }
  }
}

// Column transform, inner pass: for the group of p2 consecutive rows starting
// at blockIdx.y * p2 and the strip of columns at blockIdx.x * 32, apply signs
// (forward: before), H_p2 along the rows, the 1/sqrt(p) scale, and (inverse:
// after) the signs.
__global__ void __launch_bounds__(256) rotate_cols_inner_kernel(float* __restrict__ M, int64_t ld, int64_t cols,
                                                                int log2_p2, const float* __restrict__ signs,
                                                                int inverse, float scale) {
  extern __shared__ float t[];  // [p2][128]
  const int p2 = 1 << log2_p2;
  const int64_t r0 = (int64_t)blockIdx.y * p2;
  const int64_t c0 = (int64_t)blockIdx.x * kStrip;
  const int c4 = 4 * (threadIdx.x % (kStrip / 4));   // this thread's 4 columns
  const int rs = threadIdx.x / (kStrip / 4);
  const int rstep = blockDim.x / (kStrip / 4);
  const bool full = c0 + c4 + 3 < cols;
  for (int rb = rs; rb < p2; rb += 8 * rstep) {   // eight row loads in flight per thread
    float4 v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int r = rb + u * rstep;
      v[u] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (r < p2) {
        const float* src = M + (r0 + r) * ld + c0 + c4;
        if (full) {
          v[u] = *reinterpret_cast<const float4*>(src);
        } else {
          if (c0 + c4 + 0 < cols) v[u].x = src[0];
          if (c0 + c4 + 1 < cols) v[u].y = src[1];
          if (c0 + c4 + 2 < cols) v[u].z = src[2];
        }
      }
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int r = rb + u * rstep;
      if (r < p2) {
        const float sg = inverse ? 1.f : signs[r0 + r];
        *reinterpret_cast<float4*>(t + r * kStrip + c4) =
            make_float4(v[u].x * sg, v[u].y * sg, v[u].z * sg, v[u].w * sg);
      }
    }
  }
  __syncthreads();
  fwht_passes<false>(t, log2_p2, kStrip);
  for (int r = rs; r < p2; r += rstep) {
    float4 v = *reinterpret_cast<const float4*>(t + r * kStrip + c4);
    const float f = inverse ? scale * signs[r0 + r] : scale;
    v.x *= f; v.y *= f; v.z *= f; v.w *= f;
    float* dst = M + (r0 + r) * ld + c0 + c4;
    if (full) {
      *reinterpret_cast<float4*>(dst) = v;
    } else {
      if (c0 + c4 + 0 < cols) dst[0] = v.x;
      if (c0 + c4 + 1 < cols) dst[1] = v.y;
      if (c0 + c4 + 2 < cols) dst[2] = v.z;
    }
  }
}

// Column transform, outer pass: rows a*p + b1*p2 + b2 (a < m, b1 < p1) for
// b2 = blockIdx.y, strip blockIdx.x.  Applies H_p1 over b1 and Q_m over a
// (Q_m^T first when inverse; the two commute, they act on different factors).
__global__ void __launch_bounds__(256) rotate_cols_outer_kernel(float* __restrict__ M, int64_t ld, int64_t cols,
                                                                int p, int log2_p1, int p2, int m,
                                                                const float* __restrict__ Qm, int inverse) {
  extern __shared__ float sm[];
  float* Qs = sm;                   // [m*m]
  float* t = sm + ((m * m + 3) & ~3);  // [m*p1][128]
  const int p1 = 1 << log2_p1;
  const int R = m * p1;
  const int b2 = blockIdx.y;
  const int64_t c0 = (int64_t)blockIdx.x * kStrip;
  const int c4 = 4 * (threadIdx.x % (kStrip / 4));
  const int rs = threadIdx.x / (kStrip / 4);
  const int rstep = blockDim.x / (kStrip / 4);
  const bool full = c0 + c4 + 3 < cols;
  if (m > 1)
    for (int i = threadIdx.x; i < m * m; i += blockDim.x) Qs[i] = Qm[i];
  for (int rb = rs; rb < R; rb += 8 * rstep) {   // eight row loads in flight per thread
    float4 v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int r = rb + u * rstep;
      v[u] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (r < R) {
        const int a = r >> log2_p1, b1 = r & (p1 - 1);
        const float* src = M + ((int64_t)a * p + (int64_t)b1 * p2 + b2) * ld + c0 + c4;
        if (full) {
          v[u] = *reinterpret_cast<const float4*>(src);
        } else {
          if (c0 + c4 + 0 < cols) v[u].x = src[0];
          if (c0 + c4 + 1 < cols) v[u].y = src[1];
          if (c0 + c4 + 2 < cols) v[u].z = src[2];
        }
      }
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int r = rb + u * rstep;
      if (r < R) *reinterpret_cast<float4*>(t + r * kStrip + c4) = v[u];
    }
  }
  __syncthreads();
  auto qmix = [&](bool transpose) {
    // strand s = (b1, c) with b1 = s / 128, c = s % 128
    qmix_tile(t, Qs, m, p1 * kStrip, transpose, [&](int q, int s) { return (q * p1 + (s >> 7)) * kStrip + (s & 127); });
  };
  if (m > 1 && inverse) qmix(true);
  fwht_passes<false>(t, log2_p1, kStrip * m);
  if (m > 1 && !inverse) qmix(false);
  for (int r = rs; r < R; r += rstep) {
    const int a = r >> log2_p1, b1 = r & (p1 - 1);
    const float4 v = *reinterpret_cast<const float4*>(t + r * kStrip + c4);
    float* dst = M + ((int64_t)a * p + (int64_t)b1 * p2 + b2) * ld + c0 + c4;
    if (full) {
      *reinterpret_cast<float4*>(dst) = v;
    } else {
      if (c0 + c4 + 0 < cols) dst[0] = v.x;
      if (c0 + c4 + 1 < cols) dst[1] = v.y;
      if (c0 + c4 + 2 < cols) dst[2] = v.z;
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
    return kq::fail(KQ_ERR_ALIGNMENT, "kq_rotate: M and signs must be 16-byte aligned and ld %% 4 == 0");
  if (rows == 0 || cols == 0) return KQ_OK;
  cudaStream_t st = (cudaStream_t)stream;
  const int p = 1 << lp;
  const float scale = (float)(1.0 / sqrt((double)p));
  if (axis == KQ_AXIS_COLS) {
    if (n > kMaxRowN) return kq::fail(KQ_ERR_UNSUPPORTED_SHAPE, "kq_rotate: row length above 32768");
    if (rows > 0x7fffffff) return kq::fail(KQ_ERR_UNSUPPORTED_SHAPE, "kq_rotate: too many rows");
    size_t smem = (size_t)(n + n / 16 + 4 + (m > 1 ? m * m : 0)) * sizeof(float);
    KQ_TRY(kq::cuda_check(cudaFuncSetAttribute(rotate_rows_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               (int)smem), "kq_rotate: smem attribute"));
    rotate_rows_kernel<<<(unsigned)rows, 256, smem, st>>>(M, ld, (int)n, lp, m, T->signs, T->Qm, inverse, scale);
    KQ_TRY(kq::launch_check("kq_rotate rows"));
  } else {
    const int lp2 = lp < kMaxP2Log ? lp : kMaxP2Log;
    const int p2 = 1 << lp2, p1 = 1 << (lp - lp2);
    if ((int64_t)m * p1 > kMaxOuterRows)
      return kq::fail(KQ_ERR_UNSUPPORTED_SHAPE, "kq_rotate: m * p / 128 above 256");
    const unsigned strips = (unsigned)kq::cdiv(cols, kStrip);
    const bool outer = (m > 1 || p1 > 1);
    size_t smem_in = (size_t)p2 * kStrip * sizeof(float);
    size_t smem_out = (size_t)(((m * m + 3) & ~3) + m * p1 * kStrip) * sizeof(float);
    KQ_TRY(kq::cuda_check(cudaFuncSetAttribute(rotate_cols_inner_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               (int)smem_in), "kq_rotate: smem attribute"));
    KQ_TRY(kq::cuda_check(cudaFuncSetAttribute(rotate_cols_outer_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               (int)smem_out), "kq_rotate: smem attribute"));
    dim3 gin(strips, (unsigned)(n / p2)), gout(strips, (unsigned)p2);
    if (!inverse) {
      rotate_cols_inner_kernel<<<gin, 256, smem_in, st>>>(M, ld, cols, lp2, T->signs, 0, scale);
      KQ_TRY(kq::launch_check("kq_rotate cols inner"));
      if (outer) {
        rotate_cols_outer_kernel<<<gout, 256, smem_out, st>>>(M, ld, cols, p, lp - lp2, p2, m, T->Qm, 0);
        KQ_TRY(kq::launch_check("kq_rotate cols outer"));
      }
    } else {
      if (outer) {
        rotate_cols_outer_kernel<<<gout, 256, smem_out, st>>>(M, ld, cols, p, lp - lp2, p2, m, T->Qm, 1);
        KQ_TRY(kq::launch_check("kq_rotate cols outer"));
      }
      rotate_cols_inner_kernel<<<gin, 256, smem_in, st>>>(M, ld, cols, lp2, T->signs, 1, scale);
      KQ_TRY(kq::launch_check("kq_rotate cols inner"));
    }
  }
  kq::clear_error();
  return KQ_OK;
}
