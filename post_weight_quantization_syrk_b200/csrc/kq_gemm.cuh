// fp32-accurate GEMM on the tcgen05 tensor cores (3xTF32), internal to the
// library: used by the Kronecker loss and the solver's lazy trailing update.
#pragma once

#include "kq_internal.cuh"

namespace kq {

// Epilogues: C = AB;  partial[tile] = sum_ij (AB)_ij other_ij;  C = src - AB;
// C = tf32(AB), C_small = AB - tf32(AB) (the product stored ready to be the
// A operand of another 3xTF32 product).
enum GemmEpilogue { kEpiStore = 0, kEpiDot = 1, kEpiSubtract = 2, kEpiStoreSplit = 3 };

// C[M, N] = A[M, K] B[K, N], each operand given as a tf32 "big" part and an
// fp32 remainder "small" (see split_tf32), as AB ~ Ab Bb + Ab Bs + As Bb
// with fp32 accumulation in TMEM.  Both operands are read K-major (the
// layout tcgen05 kind::tf32 takes): A as stored, B through its transpose Bt:
//   (m, k) of A at a[(a_row0 + m) * lda + a_col0 + k]
//   (k, n) of B at bt[(bt_row0 + n) * ldbt + bt_col0 + k]
// All base pointers 16-byte aligned; leading dimensions and column offsets
// multiples of 4.
struct Gemm3xTF32 {
  int64_t M = 0, N = 0, K = 0;
  const float* a_big = nullptr;
  const float* a_small = nullptr;
  int64_t lda = 0, a_row0 = 0, a_col0 = 0;
  const float* bt_big = nullptr;
  const float* bt_small = nullptr;
  int64_t ldbt = 0, bt_row0 = 0, bt_col0 = 0;
  int epilogue = kEpiStore;
  // Upper block triangle (M == N, dot epilogue only): only the tiles whose
  // 256-column block is at or right of the 256-row block holding their rows
  // are formed, and the partials of tiles off the 256 x 256 block diagonal
  // are doubled: for a symmetric AB, the dot over the whole matrix when
  // `other` is symmetric too.
  bool upper = false;
  float* C = nullptr;              // (m, n) at C[m * ldc + n]      (store, subtract, split: tf32 part)
  float* C_small = nullptr;        // (m, n) at C_small[m * ldc + n] (split: remainder)
  int64_t ldc = 0;
  const float* src = nullptr;      // (m, n) at src[m * ld_src + n] (subtract)
  int64_t ld_src = 0;
  int64_t src_rows = 0;            // > 0: row m of the source is row m % src_rows (stacked
                                   // problems that share one source)
  const uint8_t* dead = nullptr;   // subtract: src column n reads as 0 when dead[n]
  const float* other = nullptr;    // (m, n) at other[m * ld_other + n] (dot)
  int64_t ld_other = 0;
  double* partial = nullptr;       // dot: 8 fp64 per output tile (one per epilogue warp)
  int32_t* info = nullptr;
  // Launched as a programmatic dependent of the previous kernel on the
  // stream, which must be a kernel of the same call (see pdl_wait).
  bool pdl = false;
  // Let the next kernel on the stream be scheduled as soon as this grid has
  // started (its own griddepcontrol.wait still waits for this grid's stores).
  bool trigger_early = false;
};

// Output tiles of an M x N x K product as launched (`partial` holds 8 per
// tile for kEpiDot), and the most tiles any M x N product can use.
int64_t gemm_tiles(int64_t M, int64_t N, int64_t K, bool upper = false);
int64_t gemm_tiles_max(int64_t M, int64_t N, bool upper = false);

kq_status gemm_3xtf32(const Gemm3xTF32& g, cudaStream_t st);

// big = tf32(x - y) (round to nearest), small = (x - y) - big, elementwise over
// rows x cols; y may be NULL.  Outputs have leading dimension ldo and are
// written transposed ([cols][rows]) when `transpose`.
kq_status split_tf32(const float* x, int64_t ldx, const float* y, int64_t ldy, int64_t rows, int64_t cols,
                     float* big, float* small, int64_t ldo, bool transpose, cudaStream_t st);

}  // namespace kq
