// kq_kron_loss: Kronecker loss tr(dW H_X dW^T H_G), dW = W - W_hat (a10).
//
// KronQ review (romaanj.github.io/reviews/kronq), Background: H ~ H_X kron H_G;
// Unified Hessian-Guided PTQ (hub.valency.io/works/W_r72x54u6), Appendix A.1:
// the Kronecker-weighted norm of a perturbation is a trace of this form.
// Using the symmetry of H_G, tr(dW H_X dW^T H_G) = sum_ij (dW H_X)_ij (H_G dW)_ij.
//
// kq_kron_loss runs the two products on the tensor cores in 3xTF32 (fp32
// accuracy; plain TF32 or bf16 lose too much to cancellation here): split
// dW, H_X, H_G into tf32 + remainder, A1 = dW H_X stored, then H_G dW with
// the elementwise product against A1 reduced in the GEMM epilogue to fp64
// partials, summed in a fixed order.
//
// kq_kron_loss_noalloc (below) keeps a SIMT fp32 path whose only scratch is
// one fp64 per 64x64 tile: each CTA forms one tile of both products and
// reduces their elementwise product.
#include <algorithm>
#include <mutex>

#include "kq_gemm.cuh"
#include "kq_internal.cuh"

namespace {

constexpr int T = 64, TK = 32;

// acc[4][4] += sum_k A(r,k) B(k,c) over k in [0, K), tile rows r0.., cols c0..
// A(r,k) = fa(r, k), B(k,c) = fb(k, c), both fp32 loaded through smem.
template <typename FA, typename FB>
__device__ __forceinline__ void tile_product(float (&acc)[4][4], int64_t K, FA fa, FB fb) {
  __shared__ __align__(16) float As[TK][T];
  __shared__ __align__(16) float Bs[TK][T];
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  for (int64_t k0 = 0; k0 < K; k0 += TK) {
    for (int idx = threadIdx.x; idx < TK * T; idx += 256) {
      int r = idx % T, k = idx / T;
      As[k][r] = (k0 + k < K) ? fa(r, k0 + k) : 0.f;
    }
    for (int idx = threadIdx.x; idx < TK * T; idx += 256) {
      int c = idx % T, k = idx / T;
      Bs[k][c] = (k0 + k < K) ? fb(k0 + k, c) : 0.f;
    }
    __syncthreads();
#pragma unroll 8
    for (int k = 0; k < TK; ++k) {
      float4 a = *reinterpret_cast<const float4*>(&As[k][ty * 4]);
      float4 b = *reinterpret_cast<const float4*>(&Bs[k][tx * 4]);
      float av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
    __syncthreads();
  }
}

__global__ void __launch_bounds__(256) loss_tile_kernel(const float* __restrict__ W, int64_t ldw,
                                                        const float* __restrict__ Wh, int64_t ldwh, int64_t d_out,
                                                        int64_t d_in, const float* __restrict__ HX, int64_t ldhx,
                                                        const float* __restrict__ HG, int64_t ldhg,
                                                        double* __restrict__ partial) {
  const int64_t r0 = (int64_t)blockIdx.y * T, c0 = (int64_t)blockIdx.x * T;
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  auto D = [&](int64_t r, int64_t c) -> float {
    return (r < d_out && c < d_in) ? W[r * ldw + c] - Wh[r * ldwh + c] : 0.f;
  };
  float A[4][4], B[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) A[i][j] = B[i][j] = 0.f;
  // A = dW H_X (K = d_in)
  tile_product(A, d_in, [&](int r, int64_t k) { return D(r0 + r, k); },
               [&](int64_t k, int c) { return (c0 + c < d_in) ? HX[k * ldhx + c0 + c] : 0.f; });
  if (HG) {
    // B = H_G dW (K = d_out)
    tile_product(B, d_out, [&](int r, int64_t k) { return (r0 + r < d_out) ? HG[(r0 + r) * ldhg + k] : 0.f; },
                 [&](int64_t k, int c) { return D(k, c0 + c); });
  } else {
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) B[i][j] = D(r0 + ty * 4 + i, c0 + tx * 4 + j);
  }
  double s = 0.0;
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) s += (double)A[i][j] * (double)B[i][j];
  __shared__ double red[256];
  red[threadIdx.x] = s;
  __syncthreads();
  for (int w = 128; w > 0; w >>= 1) {
    if (threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0) partial[(int64_t)blockIdx.y * gridDim.x + blockIdx.x] = red[0];
}

__global__ void sum_kernel(const double* __restrict__ partial, int64_t n, double* __restrict__ out) {
  __shared__ double red[1024];
  double s = 0.0;
  for (int64_t i = threadIdx.x; i < n; i += blockDim.x) s += partial[i];
  red[threadIdx.x] = s;
  __syncthreads();
  for (int w = blockDim.x / 2; w > 0; w >>= 1) {
    if (threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0) *out = red[0];
}

}  // namespace

namespace {

// sum_ij A1_ij (Db + Ds)_ij: the H_G = I case (dW = Db + Ds exactly).
__global__ void __launch_bounds__(256) dot_rows_kernel(const float* __restrict__ A1, const float* __restrict__ Db,
                                                       const float* __restrict__ Ds, int64_t ld, int64_t rows,
                                                       int64_t cols, double* __restrict__ partial) {
  __shared__ double red[256];
  double s = 0.0;
  for (int64_t r = blockIdx.x; r < rows; r += gridDim.x)
    for (int64_t c = threadIdx.x; c < cols; c += blockDim.x) {
      const int64_t i = r * ld + c;
      s += (double)A1[i] * (double)(Db[i] + Ds[i]);
    }
  red[threadIdx.x] = s;
  __syncthreads();
  for (int w = 128; w > 0; w >>= 1) {
    if (threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0) partial[blockIdx.x] = red[0];
}

constexpr int kDotBlocks = 1024;

// dW (as A of dW H_X), dW^T (as the transposed B of H_G dW), H_X^T, H_G, each
// split into tf32 + remainder, then A1 = dW H_X and the partial sums.
struct LossWs {
  float *Db, *Ds, *Dtb, *Dts, *Xb, *Xs, *Gb, *Gs, *A1;
  double* partial;
  int64_t ldd, ldt, ldx, ldg;
};

size_t loss_layout(int64_t d_out, int64_t d_in, LossWs* w, void* base) {
  const int64_t ldd = (d_in + 3) / 4 * 4, ldx = ldd, ldg = (d_out + 3) / 4 * 4, ldt = ldg;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off = kq::align_up(off + bytes, 256);
    return o;
  };
  const size_t sd = (size_t)d_out * ldd * 4, st_ = (size_t)d_in * ldt * 4, sx = (size_t)d_in * ldx * 4,
               sg = (size_t)d_out * ldg * 4;
  size_t oDb = take(sd), oDs = take(sd), oTb = take(st_), oTs = take(st_), oXb = take(sx), oXs = take(sx),
         oGb = take(sg), oGs = take(sg), oA = take(sd);
  const int64_t np = std::max<int64_t>(8 * kq::gemm_tiles_max(d_out, d_in), kDotBlocks);
  size_t oP = take((size_t)np * 8);
  if (w && base) {
    char* b = static_cast<char*>(base);
    w->Db = reinterpret_cast<float*>(b + oDb);
    w->Ds = reinterpret_cast<float*>(b + oDs);
    w->Dtb = reinterpret_cast<float*>(b + oTb);
    w->Dts = reinterpret_cast<float*>(b + oTs);
    w->Xb = reinterpret_cast<float*>(b + oXb);
    w->Xs = reinterpret_cast<float*>(b + oXs);
    w->Gb = reinterpret_cast<float*>(b + oGb);
    w->Gs = reinterpret_cast<float*>(b + oGs);
    w->A1 = reinterpret_cast<float*>(b + oA);
    w->partial = reinterpret_cast<double*>(b + oP);
    w->ldd = ldd;
    w->ldt = ldt;
    w->ldx = ldx;
    w->ldg = ldg;
  }
  return off;
}

}  // namespace

extern "C" size_t kq_kron_loss_workspace_size(int64_t d_out, int64_t d_in) {
  if (d_out < 1 || d_in < 1) return 0;
  return loss_layout(d_out, d_in, nullptr, nullptr);
}

namespace {

// One loss; the tf32 splits of H_X and H_G are formed here unless `split_h`
// is false (then they are already in the workspace from an earlier call).
kq_status kron_loss_impl(const float* W, int64_t ldw, const float* W_hat, int64_t ldwh, int64_t d_out, int64_t d_in,
                         const float* H_X, int64_t ldhx, const float* H_G, int64_t ldhg, double* loss, void* ws,
                         size_t ws_bytes, kq_stream_t stream, bool split_h) {
  if (!W || !W_hat || !H_X || !loss) return kq::fail(KQ_ERR_INVALID_ARG, "kq_kron_loss: NULL pointer");
  if (d_out < 1 || d_in < 1) return kq::fail(KQ_ERR_INVALID_ARG, "kq_kron_loss: sizes must be >= 1");
  if (d_out > 65536 || d_in > 65536) return kq::fail(KQ_ERR_UNSUPPORTED_SHAPE, "kq_kron_loss: sizes above 65536");
  if (ldw < d_in || ldwh < d_in || ldhx < d_in || (H_G && ldhg < d_out))
    return kq::fail(KQ_ERR_INVALID_ARG, "kq_kron_loss: leading dimension too small");
  if (!ws || !kq::aligned(ws, 256) || ws_bytes < kq_kron_loss_workspace_size(d_out, d_in))
    return kq::fail(KQ_ERR_WORKSPACE, "kq_kron_loss: workspace too small or not 256-byte aligned");
  cudaStream_t st = (cudaStream_t)stream;
  LossWs w;
  loss_layout(d_out, d_in, &w, ws);
  KQ_TRY(kq::split_tf32(W, ldw, W_hat, ldwh, d_out, d_in, w.Db, w.Ds, w.ldd, false, st));
  if (split_h) KQ_TRY(kq::split_tf32(H_X, ldhx, nullptr, 0, d_in, d_in, w.Xb, w.Xs, w.ldx, true, st));
  kq::Gemm3xTF32 g1;                 // A1 = dW H_X   (B^T = H_X^T)
  g1.M = d_out;
  g1.N = d_in;
  g1.K = d_in;
  g1.a_big = w.Db;
  g1.a_small = w.Ds;
  g1.lda = w.ldd;
  g1.bt_big = w.Xb;
  g1.bt_small = w.Xs;
  g1.ldbt = w.ldx;
  g1.epilogue = kq::kEpiStore;
  g1.C = w.A1;
  g1.ldc = w.ldd;
  KQ_TRY(kq::gemm_3xtf32(g1, st));
  int64_t np;
  if (H_G) {
    KQ_TRY(kq::split_tf32(W, ldw, W_hat, ldwh, d_out, d_in, w.Dtb, w.Dts, w.ldt, true, st));
    if (split_h) KQ_TRY(kq::split_tf32(H_G, ldhg, nullptr, 0, d_out, d_out, w.Gb, w.Gs, w.ldg, false, st));
    kq::Gemm3xTF32 g2;               // sum (H_G dW) .* A1   (B^T = dW^T)
    g2.M = d_out;
    g2.N = d_in;
    g2.K = d_out;
    g2.a_big = w.Gb;
    g2.a_small = w.Gs;
    g2.lda = w.ldg;
    g2.bt_big = w.Dtb;
    g2.bt_small = w.Dts;
    g2.ldbt = w.ldt;
    g2.epilogue = kq::kEpiDot;
    g2.other = w.A1;
    g2.ld_other = w.ldd;
    g2.partial = w.partial;
    KQ_TRY(kq::gemm_3xtf32(g2, st));
    np = 8 * kq::gemm_tiles(d_out, d_in, d_out);
  } else {
    dot_rows_kernel<<<kDotBlocks, 256, 0, st>>>(w.A1, w.Db, w.Ds, w.ldd, d_out, d_in, w.partial);
    KQ_TRY(kq::launch_check("kq_kron_loss dot"));
    np = kDotBlocks;
  }
  sum_kernel<<<1, 1024, 0, st>>>(w.partial, np, loss);
  KQ_TRY(kq::launch_check("kq_kron_loss sum"));
  kq::clear_error();
  return KQ_OK;
}

}  // namespace

extern "C" kq_status kq_kron_loss(const float* W, int64_t ldw, const float* W_hat, int64_t ldwh, int64_t d_out,
                                  int64_t d_in, const float* H_X, int64_t ldhx, const float* H_G, int64_t ldhg,
                                  double* loss, void* ws, size_t ws_bytes, kq_stream_t stream) {
  return kron_loss_impl(W, ldw, W_hat, ldwh, d_out, d_in, H_X, ldhx, H_G, ldhg, loss, ws, ws_bytes, stream, true);
}

extern "C" kq_status kq_kron_loss_multi(const float* W, int64_t ldw, int count, const float* const* W_hat,
                                        int64_t ldwh, int64_t d_out, int64_t d_in, const float* H_X, int64_t ldhx,
                                        const float* H_G, int64_t ldhg, double* const* loss, void* ws,
                                        size_t ws_bytes, kq_stream_t stream) {
  if (count < 1 || !W_hat || !loss) return kq::fail(KQ_ERR_INVALID_ARG, "kq_kron_loss_multi: count < 1 or NULL array");
  for (int i = 0; i < count; ++i)
    if (!W_hat[i] || !loss[i]) return kq::fail(KQ_ERR_INVALID_ARG, "kq_kron_loss_multi: NULL W_hat or loss entry");
  for (int i = 0; i < count; ++i)
    KQ_TRY(kron_loss_impl(W, ldw, W_hat[i], ldwh, d_out, d_in, H_X, ldhx, H_G, ldhg, loss[i], ws, ws_bytes, stream,
                          i == 0));
  return KQ_OK;
}

// ---------------------------------------------------------------------------
// kq_kron_loss_noalloc: the same loss with the per-tile partial sums kept in a
// fixed device array that belongs to this library, for callers that must not
// allocate device memory themselves (see kronq.h).
// ---------------------------------------------------------------------------
namespace {

// Per-tile partial sums, one fp64 per 64x64 tile; every GPU that loads the
// library holds this array until the process exits.
static __device__ __align__(256) double g_loss_partials[KQ_KRON_LOSS_NOALLOC_MAX_TILES];

constexpr int kMaxDevices = 64;
std::mutex g_partials_mutex;
double* g_partials_ptr[kMaxDevices] = {nullptr};

// Device address of g_loss_partials on the current device, looked up once per
// device with that device current.  A host-side use of the symbol itself
// would name a host stand-in, not device memory.
kq_status partials_address(double** out) {
  int dev = -1;
  KQ_TRY(kq::cuda_check(cudaGetDevice(&dev), "kq_kron_loss_noalloc: cudaGetDevice"));
  if (dev < 0 || dev >= kMaxDevices)
    return kq::fail(KQ_ERR_UNSUPPORTED_SHAPE, "kq_kron_loss_noalloc: device ordinal %d above %d", dev, kMaxDevices - 1);
  std::lock_guard<std::mutex> lock(g_partials_mutex);
  if (!g_partials_ptr[dev]) {
    void* p = nullptr;
    KQ_TRY(kq::cuda_check(cudaGetSymbolAddress(&p, g_loss_partials), "kq_kron_loss_noalloc: cudaGetSymbolAddress"));
    g_partials_ptr[dev] = static_cast<double*>(p);
  }
  *out = g_partials_ptr[dev];
  return KQ_OK;
}

}  // namespace

extern "C" kq_status kq_kron_loss_noalloc(const float* W, int64_t ldw, const float* W_hat, int64_t ldwh,
                                          int64_t d_out, int64_t d_in, const float* H_X, int64_t ldhx,
                                          const float* H_G, int64_t ldhg, double* loss, kq_stream_t stream) {
  if (!W || !W_hat || !H_X || !loss) return kq::fail(KQ_ERR_INVALID_ARG, "kq_kron_loss_noalloc: NULL pointer");
  if (d_out < 1 || d_in < 1) return kq::fail(KQ_ERR_INVALID_ARG, "kq_kron_loss_noalloc: sizes must be >= 1");
  if (ldw < d_in || ldwh < d_in || ldhx < d_in || (H_G && ldhg < d_out))
    return kq::fail(KQ_ERR_INVALID_ARG, "kq_kron_loss_noalloc: leading dimension too small");
  const int64_t tiles = kq::cdiv(d_out, T) * kq::cdiv(d_in, T);
  if (tiles > KQ_KRON_LOSS_NOALLOC_MAX_TILES)
    return kq::fail(KQ_ERR_UNSUPPORTED_SHAPE,
                    "kq_kron_loss_noalloc: ceil(d_out/64) * ceil(d_in/64) = %lld tiles exceeds the fixed scratch of %d "
                    "tiles; use kq_kron_loss with a caller workspace",
                    (long long)tiles, (int)KQ_KRON_LOSS_NOALLOC_MAX_TILES);
  double* partial = nullptr;
  KQ_TRY(partials_address(&partial));
  cudaStream_t st = (cudaStream_t)stream;
  dim3 grid((unsigned)kq::cdiv(d_in, T), (unsigned)kq::cdiv(d_out, T));
  // Every tile overwrites its own slot and the sum reads only those slots, so
  // nothing left in the array by an earlier call needs clearing.
  loss_tile_kernel<<<grid, 256, 0, st>>>(W, ldw, W_hat, ldwh, d_out, d_in, H_X, ldhx, H_G, ldhg, partial);
  KQ_TRY(kq::launch_check("kq_kron_loss_noalloc tiles"));
  sum_kernel<<<1, 1024, 0, st>>>(partial, tiles, loss);
  KQ_TRY(kq::launch_check("kq_kron_loss_noalloc sum"));
  kq::clear_error();
  return KQ_OK;
}
