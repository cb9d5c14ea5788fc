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


// ===========================================================================
// Fast paths.  The kernels above are kept for the shapes these do not cover.
//
//  * rows_fast<K> (KQ_AXIS_COLS, p = 2^K with 4 <= K <= 12): one CTA per row;
//    every thread holds 16 consecutive elements of the row ("a chunk") in
//    registers.  The Hadamard butterflies over index bits 0..3 run in
//    registers, bits 4..8 across the lanes of a warp by shuffles (a warp's
//    32 chunks are 512 consecutive elements), and the at most three bits
//    9..K-1 in one shared-memory stage.  Q_m (m > 1) is a register-tiled
//    product in shared memory.  No index arithmetic beyond shifts by
//    compile-time amounts.
//  * cols_inner_fast<K2> / cols_outer_fast<K1> (KQ_AXIS_ROWS): the same two
//    passes as above over 128-column strips, with the butterflies along rows
//    done on float4 column quads (one 16-byte shared access moves four
//    columns) and the Q_m mix register-tiled.
// ===========================================================================

// Padded shared-memory position of element e of a row: 4 spare floats after
// every 32.  The 16-byte accesses of a quarter warp to 8 consecutive chunks,
// and 32 consecutive elements, then fall in distinct banks.
__device__ __forceinline__ int padq(int e) { return e + ((e >> 5) << 2); }

// Radix-2 butterflies over bits [0, G) of 2^G register-held values.
template <int G, int N>
__device__ __forceinline__ void bfly_regs(float (&r)[N]) {
#pragma unroll
  for (int s = 0; s < G; ++s) {
#pragma unroll
    for (int e = 0; e < (1 << G); ++e) {
      if (e & (1 << s)) continue;
      const float a = r[e], b = r[e + (1 << s)];
      r[e] = a + b;
      r[e + (1 << s)] = a - b;
    }
  }
}

// Butterflies over lane bits [0, LB) for 16 register values of each lane.
template <int LB>
__device__ __forceinline__ void bfly_lanes(float (&r)[16]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int s = 0; s < LB; ++s) {
    const float sg = (lane & (1 << s)) ? -1.f : 1.f;   // upper partner: a - b = other - mine
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      const float o = __shfl_xor_sync(0xffffffffu, r[e], 1 << s);
      r[e] = fmaf(r[e], sg, o);
    }
  }
}

// In-place Q_m mix of the strands of an m-row array in shared memory:
// element (a, s) at x[addr(a, s)], s < S, with addr(a, s + 1..3) the three
// floats after addr(a, s) for s % 4 == 0 and addr 16-byte aligned there.
// y(a, s) = sum_c QT[c * qs + a] x(c, s); QT holds rows a >= m as zeros.
// Work items are (4 rows) x (4 consecutive strands); each thread keeps up to
// four items' 4 x 4 accumulators, so strands go in slices of at most
// 1024 / ceil(m / 4) quads.  Called by all 256 threads; ends with a barrier.
template <typename Addr>
__device__ void qmix_quads(float* x, const float* QT, int qs, int m, int S, Addr addr) {
  const int t = threadIdx.x;
  const int rbn = (m + 3) >> 2;
  const int slice_q = max(1, 1024 / rbn);
  for (int q0 = 0; q0 < S / 4; q0 += slice_q) {
    const int nq = min(slice_q, S / 4 - q0);
    const int items = nq * rbn;
    float acc[4][4][4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int it = t + 256 * k;
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[k][i][j] = 0.f;
      if (it < items) {
        const int rb = it / nq, b0 = 4 * (q0 + it % nq);
        const float* qcol = QT + 4 * rb;
        for (int c = 0; c < m; ++c) {
          const float4 xv = *reinterpret_cast<const float4*>(x + addr(c, b0));
          const float4 qv = *reinterpret_cast<const float4*>(qcol + c * qs);
          const float xa[4] = {xv.x, xv.y, xv.z, xv.w}, qa[4] = {qv.x, qv.y, qv.z, qv.w};
#pragma unroll
          for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) acc[k][i][j] = fmaf(qa[i], xa[j], acc[k][i][j]);
        }
      }
    }
    __syncthreads();   // every read of this slice is done
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int it = t + 256 * k;
      if (it < items) {
        const int rb = it / nq, b0 = 4 * (q0 + it % nq);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int a = 4 * rb + i;
          if (a < m)
            *reinterpret_cast<float4*>(x + addr(a, b0)) = make_float4(acc[k][i][0], acc[k][i][1], acc[k][i][2], acc[k][i][3]);
        }
      }
    }
    __syncthreads();
  }
}

// QT[c * qs + a] = Q[a][c] (forward) or Q[c][a] (transpose), rows a in
// [m, qs) zero; qs = m rounded up to 4.
__device__ __forceinline__ void load_qt(float* QT, const float* Qm, int m, int qs, bool transpose) {
  for (int i = threadIdx.x; i < m * qs; i += blockDim.x) {
    const int c = i / qs, a = i % qs;
    QT[i] = (a < m) ? (transpose ? Qm[c * m + a] : Qm[a * m + c]) : 0.f;
  }
}

template <int K, bool QM>
__global__ void __launch_bounds__(256) rows_fast(float* __restrict__ M, int64_t ld, int m,
                                                 const float* __restrict__ signs, const float* __restrict__ Qm,
                                                 int inverse, float scale) {
  constexpr int P = 1 << K;
  constexpr int LB = (K - 4) < 5 ? (K - 4) : 5;   // lane bits inside a vector
  constexpr int SB = K > 9 ? K - 9 : 0;           // bits left for shared memory (<= 3)
  extern __shared__ __align__(16) float smf[];
  const int n = m * P, nch = n >> 4;
  const int qs = (m + 3) & ~3;
  float* QT = smf;
  float* x = smf + (m > 1 ? m * qs : 0);
  float* row = M + (int64_t)blockIdx.x * ld;
  const int t = threadIdx.x;
  constexpr bool staged = (SB > 0) || QM;   // QM: m > 1
  if constexpr (QM) load_qt(QT, Qm, m, qs, inverse != 0);

  auto load_chunk = [&](int c, float (&r)[16], bool apply_signs) {
    if (c < nch) {
      const float4* src = reinterpret_cast<const float4*>(row + 16 * c);
      float4 v[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) v[q] = src[q];
      if (apply_signs) {
        const float4* sg = reinterpret_cast<const float4*>(signs + 16 * c);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float4 g = sg[q];
          v[q].x *= g.x; v[q].y *= g.y; v[q].z *= g.z; v[q].w *= g.w;
        }
      }
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        r[4 * q] = v[q].x; r[4 * q + 1] = v[q].y; r[4 * q + 2] = v[q].z; r[4 * q + 3] = v[q].w;
      }
    } else {
#pragma unroll
      for (int e = 0; e < 16; ++e) r[e] = 0.f;
    }
  };
  auto to_smem = [&](int c, const float (&r)[16]) {
    if (c < nch) {
#pragma unroll
      for (int q = 0; q < 4; ++q)
        *reinterpret_cast<float4*>(x + padq(16 * c + 4 * q)) = make_float4(r[4 * q], r[4 * q + 1], r[4 * q + 2], r[4 * q + 3]);
    }
  };
  auto from_smem = [&](int c, float (&r)[16]) {
    if (c < nch) {
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float4 v = *reinterpret_cast<const float4*>(x + padq(16 * c + 4 * q));
        r[4 * q] = v.x; r[4 * q + 1] = v.y; r[4 * q + 2] = v.z; r[4 * q + 3] = v.w;
      }
    } else {
#pragma unroll
      for (int e = 0; e < 16; ++e) r[e] = 0.f;
    }
  };
  auto store_chunk = [&](int c, const float (&r)[16]) {
    if (c >= nch) return;
    float4* dst = reinterpret_cast<float4*>(row + 16 * c);
    float4 v[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) v[q] = make_float4(r[4 * q] * scale, r[4 * q + 1] * scale, r[4 * q + 2] * scale, r[4 * q + 3] * scale);
    if (inverse) {
      const float4* sg = reinterpret_cast<const float4*>(signs + 16 * c);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float4 g = sg[q];
        v[q].x *= g.x; v[q].y *= g.y; v[q].z *= g.z; v[q].w *= g.w;
      }
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) dst[q] = v[q];
  };
  // butterflies over in-vector bits 9 .. K-1, in shared memory: groups of
  // 2^SB elements a P + j 512 + l (j < 2^SB) for every vector a and l < 512
  auto smem_stage = [&]() {
    if constexpr (SB > 0) {
      for (int g = t; g < m * 512; g += 256) {
        const int base = (g >> 9) * P + (g & 511);
        float r[1 << SB];
#pragma unroll
        for (int j = 0; j < (1 << SB); ++j) r[j] = x[padq(base + 512 * j)];
        bfly_regs<SB>(r);
#pragma unroll
        for (int j = 0; j < (1 << SB); ++j) x[padq(base + 512 * j)] = r[j];
      }
    }
  };
  auto addr = [&](int a, int s) { return padq(a * P + s); };
  const int iters = (nch + 255) >> 8;
  float r[16];
  if (!inverse) {
    for (int i = 0; i < iters; ++i) {
      const int c = t + 256 * i;
      load_chunk(c, r, true);
      bfly_regs<4>(r);
      bfly_lanes<LB>(r);
      if constexpr (staged) to_smem(c, r);
      else store_chunk(c, r);
    }
    if constexpr (staged) {
      __syncthreads();
      if constexpr (SB > 0) {
        smem_stage();
        __syncthreads();
      }
      if constexpr (QM) qmix_quads(x, QT, qs, m, P, addr);
      for (int i = 0; i < iters; ++i) {
        const int c = t + 256 * i;
        from_smem(c, r);
        store_chunk(c, r);
      }
    }
  } else {
    if constexpr (QM) {
      for (int i = 0; i < iters; ++i) {
        const int c = t + 256 * i;
        load_chunk(c, r, false);
        to_smem(c, r);
      }
      __syncthreads();
      qmix_quads(x, QT, qs, m, P, addr);
    }
    for (int i = 0; i < iters; ++i) {
      const int c = t + 256 * i;
      if constexpr (QM) from_smem(c, r);
      else load_chunk(c, r, false);
      bfly_regs<4>(r);
      bfly_lanes<LB>(r);
      if constexpr (SB > 0) to_smem(c, r);
      else store_chunk(c, r);
    }
    if constexpr (SB > 0) {
      __syncthreads();
      smem_stage();
      __syncthreads();
      for (int i = 0; i < iters; ++i) {
        const int c = t + 256 * i;
        from_smem(c, r);
        store_chunk(c, r);
      }
    }
  }
}

size_t rows_fast_smem(int m, int K) {
  const int n = m << K;
  const int qs = (m + 3) & ~3;
  const bool staged = (K > 9) || (m > 1);
  return (size_t)((m > 1 ? m * qs : 0) + (staged ? n + (n >> 3) : 0)) * sizeof(float);
}

// One row-group of the column transform in shared memory: tile[r][128]
// (row r of the group, the strip's 128 columns).  Butterflies along rows
// over bits [LO, LO + G) of the row index, on float4 column quads: item =
// (column quad, the other row bits).
template <int KR, int LO, int G>
__device__ __forceinline__ void rows_bfly_pass(float* tile, int nsets) {
  // nsets independent sets of 2^KR rows (set s at rows s << KR)
  constexpr int REST = KR - G;
  const int items = 32 * (nsets << REST);
  for (int it = threadIdx.x; it < items; it += 256) {
    const int cq = it & 31, rest = it >> 5;
    const int set = rest >> REST, rr = rest & ((1 << REST) - 1);
    const int base = (set << KR) | ((rr >> LO) << (LO + G)) | (rr & ((1 << LO) - 1));
    float4 v[1 << G];
#pragma unroll
    for (int e = 0; e < (1 << G); ++e) v[e] = *reinterpret_cast<const float4*>(tile + (base | (e << LO)) * kStrip + 4 * cq);
#pragma unroll
    for (int s = 0; s < G; ++s) {
#pragma unroll
      for (int e = 0; e < (1 << G); ++e) {
        if (e & (1 << s)) continue;
        const float4 a = v[e], b = v[e + (1 << s)];
        v[e] = make_float4(a.x + b.x, a.y + b.y, a.z + b.z, a.w + b.w);
        v[e + (1 << s)] = make_float4(a.x - b.x, a.y - b.y, a.z - b.z, a.w - b.w);
      }
    }
#pragma unroll
    for (int e = 0; e < (1 << G); ++e) *reinterpret_cast<float4*>(tile + (base | (e << LO)) * kStrip + 4 * cq) = v[e];
  }
}

// Butterflies over all KR (<= 8) row bits of nsets sets: bits 0..3, then 4..KR-1.
template <int KR>
__device__ __forceinline__ void rows_fwht(float* tile, int nsets) {
  static_assert(KR <= 8, "two radix-16 passes at most");
  if constexpr (KR >= 4) {
    rows_bfly_pass<KR, 0, 4>(tile, nsets);
    __syncthreads();
    if constexpr (KR > 4) {
      rows_bfly_pass<KR, 4, KR - 4>(tile, nsets);
      __syncthreads();
    }
  } else if constexpr (KR > 0) {
    rows_bfly_pass<KR, 0, KR>(tile, nsets);
    __syncthreads();
  }
}

// Row r of the strip tile from/to global memory (ragged last strip by scalars).
__device__ __forceinline__ float4 strip_load(const float* src, int64_t c, int64_t cols) {
  if (c + 3 < cols) return *reinterpret_cast<const float4*>(src);
  float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
  if (c + 0 < cols) v.x = src[0];
  if (c + 1 < cols) v.y = src[1];
  if (c + 2 < cols) v.z = src[2];
  return v;
}
__device__ __forceinline__ void strip_store(float* dst, int64_t c, int64_t cols, float4 v) {
  if (c + 3 < cols) {
    *reinterpret_cast<float4*>(dst) = v;
    return;
  }
  if (c + 0 < cols) dst[0] = v.x;
  if (c + 1 < cols) dst[1] = v.y;
  if (c + 2 < cols) dst[2] = v.z;
}

// Inner pass: rows r0 .. r0 + 2^K2 - 1 (r0 = blockIdx.y 2^K2), one strip:
// signs (forward: first), H_{2^K2} along the rows, the 1/sqrt(p) scale,
// signs (inverse: last).
template <int K2>
__global__ void __launch_bounds__(256) cols_inner_fast(float* __restrict__ M, int64_t ld, int64_t cols,
                                                       const float* __restrict__ signs, int inverse, float scale) {
  constexpr int P2 = 1 << K2;
  extern __shared__ __align__(16) float tile[];   // [P2][128]
  const int64_t r0 = (int64_t)blockIdx.y * P2;
  const int64_t c0 = (int64_t)blockIdx.x * kStrip;
  const int cq = threadIdx.x & 31, rg = threadIdx.x >> 5;
  const int64_t c = c0 + 4 * cq;
  constexpr int PER = (P2 + 7) / 8;
  float4 v[PER];
#pragma unroll
  for (int u = 0; u < PER; ++u) {
    const int r = rg + 8 * u;
    if (r < P2) v[u] = strip_load(M + (r0 + r) * ld + c, c, cols);
  }
#pragma unroll
  for (int u = 0; u < PER; ++u) {
    const int r = rg + 8 * u;
    if (r < P2) {
      const float g = inverse ? 1.f : signs[r0 + r];
      *reinterpret_cast<float4*>(tile + r * kStrip + 4 * cq) = make_float4(v[u].x * g, v[u].y * g, v[u].z * g, v[u].w * g);
    }
  }
  __syncthreads();
  rows_fwht<K2>(tile, 1);
#pragma unroll
  for (int u = 0; u < PER; ++u) {
    const int r = rg + 8 * u;
    if (r < P2) {
      const float f = inverse ? scale * signs[r0 + r] : scale;
      const float4 w = *reinterpret_cast<const float4*>(tile + r * kStrip + 4 * cq);
      strip_store(M + (r0 + r) * ld + c, c, cols, make_float4(w.x * f, w.y * f, w.z * f, w.w * f));
    }
  }
}

// Outer pass: rows a p + b1 p2 + b2 (a < m, b1 < 2^K1) for b2 = blockIdx.y,
// one strip; tile row a 2^K1 + b1.  H_{2^K1} over b1 and Q_m over a (Q_m^T
// first when inverse; they act on different factors and commute).
template <int K1, bool QM>
__global__ void __launch_bounds__(256) cols_outer_fast(float* __restrict__ M, int64_t ld, int64_t cols, int p,
                                                       int p2, int m, const float* __restrict__ Qm, int inverse) {
  constexpr int P1 = 1 << K1;
  extern __shared__ __align__(16) float smo[];
  const int qs = (m + 3) & ~3;
  float* QT = smo;
  float* tile = smo + (m > 1 ? m * qs : 0);   // [m * P1][128]
  const int R = m * P1;
  const int b2 = blockIdx.y;
  const int64_t c0 = (int64_t)blockIdx.x * kStrip;
  const int cq = threadIdx.x & 31, rg = threadIdx.x >> 5;
  const int64_t c = c0 + 4 * cq;
  if constexpr (QM) load_qt(QT, Qm, m, qs, inverse != 0);
  for (int rb = rg; rb < R; rb += 64) {   // eight loads in flight per thread
    float4 v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int r = rb + 8 * u;
      if (r < R) v[u] = strip_load(M + ((int64_t)(r >> K1) * p + (int64_t)(r & (P1 - 1)) * p2 + b2) * ld + c, c, cols);
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int r = rb + 8 * u;
      if (r < R) *reinterpret_cast<float4*>(tile + r * kStrip + 4 * cq) = v[u];
    }
  }
  __syncthreads();
  // strand s = (b1, column) of row a at tile[(a P1 + b1) 128 + column]
  auto addr = [&](int a, int s) { return a * (P1 * kStrip) + s; };
  if constexpr (QM) {
    if (inverse) qmix_quads(tile, QT, qs, m, P1 * kStrip, addr);
  }
  rows_fwht<K1>(tile, m);
  if constexpr (QM) {
    if (!inverse) qmix_quads(tile, QT, qs, m, P1 * kStrip, addr);
  }
  for (int r = rg; r < R; r += 8) {
    const float4 w = *reinterpret_cast<const float4*>(tile + r * kStrip + 4 * cq);
    strip_store(M + ((int64_t)(r >> K1) * p + (int64_t)(r & (P1 - 1)) * p2 + b2) * ld + c, c, cols, w);
  }
}

template <int K>
kq_status launch_rows_fast(float* M, int64_t rows, int64_t ld, int m, const float* signs, const float* Qm, int inverse,
                           float scale, cudaStream_t st) {
  const size_t smem = rows_fast_smem(m, K);
  if (m > 1) {
    KQ_TRY(kq::cuda_check(cudaFuncSetAttribute(rows_fast<K, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               (int)smem), "kq_rotate: smem attribute"));
    rows_fast<K, true><<<(unsigned)rows, 256, smem, st>>>(M, ld, m, signs, Qm, inverse, scale);
  } else {
    KQ_TRY(kq::cuda_check(cudaFuncSetAttribute(rows_fast<K, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               (int)smem), "kq_rotate: smem attribute"));
    rows_fast<K, false><<<(unsigned)rows, 256, smem, st>>>(M, ld, m, signs, Qm, inverse, scale);
  }
  return kq::launch_check("kq_rotate rows");
}

kq_status rows_fast_dispatch(int K, float* M, int64_t rows, int64_t ld, int m, const float* signs, const float* Qm,
                             int inverse, float scale, cudaStream_t st) {
  switch (K) {
    case 4: return launch_rows_fast<4>(M, rows, ld, m, signs, Qm, inverse, scale, st);
    case 5: return launch_rows_fast<5>(M, rows, ld, m, signs, Qm, inverse, scale, st);
    case 6: return launch_rows_fast<6>(M, rows, ld, m, signs, Qm, inverse, scale, st);
    case 7: return launch_rows_fast<7>(M, rows, ld, m, signs, Qm, inverse, scale, st);
    case 8: return launch_rows_fast<8>(M, rows, ld, m, signs, Qm, inverse, scale, st);
    case 9: return launch_rows_fast<9>(M, rows, ld, m, signs, Qm, inverse, scale, st);
    case 10: return launch_rows_fast<10>(M, rows, ld, m, signs, Qm, inverse, scale, st);
    case 11: return launch_rows_fast<11>(M, rows, ld, m, signs, Qm, inverse, scale, st);
    case 12: return launch_rows_fast<12>(M, rows, ld, m, signs, Qm, inverse, scale, st);
  }
  return kq::fail(KQ_ERR_UNSUPPORTED_SHAPE, "kq_rotate: no fast row kernel for log2_p = %d", K);
}

template <int K2>
kq_status launch_inner(float* M, int64_t ld, int64_t cols, unsigned strips, unsigned groups, const float* signs,
                       int inverse, float scale, cudaStream_t st) {
  const size_t smem = (size_t)(1 << K2) * kStrip * sizeof(float);
  KQ_TRY(kq::cuda_check(cudaFuncSetAttribute(cols_inner_fast<K2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)smem), "kq_rotate: smem attribute"));
  cols_inner_fast<K2><<<dim3(strips, groups), 256, smem, st>>>(M, ld, cols, signs, inverse, scale);
  return kq::launch_check("kq_rotate cols inner");
}

kq_status inner_dispatch(int K2, float* M, int64_t ld, int64_t cols, unsigned strips, unsigned groups,
                         const float* signs, int inverse, float scale, cudaStream_t st) {
  switch (K2) {
    case 0: return launch_inner<0>(M, ld, cols, strips, groups, signs, inverse, scale, st);
    case 1: return launch_inner<1>(M, ld, cols, strips, groups, signs, inverse, scale, st);
    case 2: return launch_inner<2>(M, ld, cols, strips, groups, signs, inverse, scale, st);
    case 3: return launch_inner<3>(M, ld, cols, strips, groups, signs, inverse, scale, st);
    case 4: return launch_inner<4>(M, ld, cols, strips, groups, signs, inverse, scale, st);
    case 5: return launch_inner<5>(M, ld, cols, strips, groups, signs, inverse, scale, st);
    case 6: return launch_inner<6>(M, ld, cols, strips, groups, signs, inverse, scale, st);
    case 7: return launch_inner<7>(M, ld, cols, strips, groups, signs, inverse, scale, st);
  }
  return kq::fail(KQ_ERR_UNSUPPORTED_SHAPE, "kq_rotate: inner pass over %d row bits", K2);
}

template <int K1>
kq_status launch_outer(float* M, int64_t ld, int64_t cols, unsigned strips, unsigned groups, int p, int p2, int m,
                       const float* Qm, int inverse, cudaStream_t st) {
  const int qs = (m + 3) & ~3;
  const size_t smem = (size_t)((m > 1 ? m * qs : 0) + m * (1 << K1) * kStrip) * sizeof(float);
  if (m > 1) {
    KQ_TRY(kq::cuda_check(cudaFuncSetAttribute(cols_outer_fast<K1, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               (int)smem), "kq_rotate: smem attribute"));
    cols_outer_fast<K1, true><<<dim3(strips, groups), 256, smem, st>>>(M, ld, cols, p, p2, m, Qm, inverse);
  } else {
    KQ_TRY(kq::cuda_check(cudaFuncSetAttribute(cols_outer_fast<K1, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               (int)smem), "kq_rotate: smem attribute"));
    cols_outer_fast<K1, false><<<dim3(strips, groups), 256, smem, st>>>(M, ld, cols, p, p2, m, Qm, inverse);
  }
  return kq::launch_check("kq_rotate cols outer");
}

kq_status outer_dispatch(int K1, float* M, int64_t ld, int64_t cols, unsigned strips, unsigned groups, int p, int p2,
                         int m, const float* Qm, int inverse, cudaStream_t st) {
  switch (K1) {
    case 0: return launch_outer<0>(M, ld, cols, strips, groups, p, p2, m, Qm, inverse, st);
    case 1: return launch_outer<1>(M, ld, cols, strips, groups, p, p2, m, Qm, inverse, st);
    case 2: return launch_outer<2>(M, ld, cols, strips, groups, p, p2, m, Qm, inverse, st);
    case 3: return launch_outer<3>(M, ld, cols, strips, groups, p, p2, m, Qm, inverse, st);
    case 4: return launch_outer<4>(M, ld, cols, strips, groups, p, p2, m, Qm, inverse, st);
    case 5: return launch_outer<5>(M, ld, cols, strips, groups, p, p2, m, Qm, inverse, st);
    case 6: return launch_outer<6>(M, ld, cols, strips, groups, p, p2, m, Qm, inverse, st);
    case 7: return launch_outer<7>(M, ld, cols, strips, groups, p, p2, m, Qm, inverse, st);
    case 8: return launch_outer<8>(M, ld, cols, strips, groups, p, p2, m, Qm, inverse, st);
  }
  return kq::fail(KQ_ERR_UNSUPPORTED_SHAPE, "kq_rotate: outer pass over %d row bits", K1);
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
    if (lp >= 4 && lp <= 12) {
      KQ_TRY(rows_fast_dispatch(lp, M, rows, ld, m, T->signs, T->Qm, inverse, scale, st));
      kq::clear_error();
      return KQ_OK;
    }
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
    if (n / p2 > 65535 || p2 > 65535) return kq::fail(KQ_ERR_UNSUPPORTED_SHAPE, "kq_rotate: grid too large");
    if (!inverse) {
      KQ_TRY(inner_dispatch(lp2, M, ld, cols, strips, (unsigned)(n / p2), T->signs, 0, scale, st));
      if (outer) KQ_TRY(outer_dispatch(lp - lp2, M, ld, cols, strips, (unsigned)p2, p, p2, m, T->Qm, 0, st));
    } else {
      if (outer) KQ_TRY(outer_dispatch(lp - lp2, M, ld, cols, strips, (unsigned)p2, p, p2, m, T->Qm, 1, st));
      KQ_TRY(inner_dispatch(lp2, M, ld, cols, strips, (unsigned)(n / p2), T->signs, 1, scale, st));
    }
    kq::clear_error();
    return KQ_OK;
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
