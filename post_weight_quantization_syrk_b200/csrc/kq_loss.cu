// kq_kron_loss: Kronecker loss tr(dW H_X dW^T H_G), dW = W - W_hat (a10).
//
// KronQ review (romaanj.github.io/reviews/kronq), Background: H ~ H_X kron H_G;
// Unified Hessian-Guided PTQ (hub.valency.io/works/W_r72x54u6), Appendix A.1:
// the Kronecker-weighted norm of a perturbation is a trace of this form.
//
// kq_kron_loss writes the trace as a Frobenius product with one symmetric
// factor, taking the smaller Hessian into the product:
//   d_in <= d_out:  loss = <P, H_G>,  P = dW H_X^T dW^T      (d_out x d_out)
//   d_in >  d_out:  loss = <P, H_X>,  P = dW^T H_G^T dW      (d_in x d_in)
//   H_G = I:        loss = <P, H_X>,  P = dW^T dW
// (each is tr(dW H_X dW^T H_G) by the cyclic property and tr(M) = tr(M^T)).
// With D = dW or dW^T (n2 x n1, n1 the smaller side) and H1 the smaller
// Hessian, A1 = D H1^T is formed first (n2 n1^2 multiply-adds), then P =
// A1 D^T is formed only in its upper block triangle, each off-diagonal tile
// counting twice (P and H2 are symmetric): about n2^2 n1 / 2 more, against
// d_out d_in (d_in + d_out) for forming dW H_X and H_G dW in full.  Both
// products run on the tensor cores in 3xTF32 (fp32 accuracy; plain TF32 or
// bf16 lose too much to cancellation here); A1 leaves the first product
// already split into tf32 + remainder, and the elementwise product of P
// with H2 is reduced in the second product's epilogue to fp64 partials,
// summed in a fixed order.
//
// kq_kron_loss_noalloc (below) keeps a SIMT fp32 path whose only scratch is
// one fp64 per 64x64 tile: each CTA forms one tile of dW H_X and of
// H_G^T dW and reduces their elementwise product (exact for any H_X, H_G).
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
    // B = H_G^T dW (K = d_out): H_G read by columns, so that the sum below is
    // sum (dW H_X) .* (H_G^T dW) = tr((dW H_X)^T H_G^T dW) = tr(dW H_X dW^T H_G)
    // exactly, for any H_X and H_G (no symmetry used)
    tile_product(B, d_out, [&](int r, int64_t k) { return (r0 + r < d_out) ? HG[k * ldhg + r0 + r] : 0.f; },
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


// D = dW or dW^T (n2 x n1) and A1 = D H1^T, each as tf32 + remainder (leading
// dimension ldd); H1 likewise (leading dimension ldh); the fp64 partials of
// the upper block triangle of P.  Sized for either orientation.
struct LossWs {
  float *Db, *Ds, *Ab, *As, *Hb, *Hs;
  double* partial;
};

constexpr int64_t lead(int64_t n) { return (n + 3) / 4 * 4; }

size_t loss_layout(int64_t d_out, int64_t d_in, LossWs* w, void* base) {
  const int64_t n1 = std::min(d_out, d_in), n2 = std::max(d_out, d_in);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off = kq::align_up(off + bytes, 256);
    return o;
  };
  const size_t sd = (size_t)std::max(d_out * lead(d_in), d_in * lead(d_out)) * 4, sh = (size_t)n1 * lead(n1) * 4;
  size_t oDb = take(sd), oDs = take(sd), oAb = take(sd), oAs = take(sd), oHb = take(sh), oHs = take(sh);
  size_t oP = take((size_t)8 * kq::gemm_tiles_max(n2, n2, true) * 8);
  if (w && base) {
    char* b = static_cast<char*>(base);
    w->Db = reinterpret_cast<float*>(b + oDb);
    w->Ds = reinterpret_cast<float*>(b + oDs);
    w->Ab = reinterpret_cast<float*>(b + oAb);
    w->As = reinterpret_cast<float*>(b + oAs);
    w->Hb = reinterpret_cast<float*>(b + oHb);
    w->Hs = reinterpret_cast<float*>(b + oHs);
    w->partial = reinterpret_cast<double*>(b + oP);
  }
  return off;
}

}  // namespace

extern "C" size_t kq_kron_loss_workspace_size(int64_t d_out, int64_t d_in) {
  if (d_out < 1 || d_in < 1) return 0;
  return loss_layout(d_out, d_in, nullptr, nullptr);
}

namespace {

// The products of one loss, their fp64 partials written from `partial`
// (or the workspace's own region when NULL); *np_out = how many.  The tf32
// split of the smaller Hessian is formed here unless `split_h` is false
// (then it is already in the workspace from an earlier call with the same
// H_X, H_G and shape).
kq_status kron_loss_products(const float* W, int64_t ldw, const float* W_hat, int64_t ldwh, int64_t d_out,
                             int64_t d_in, const float* H_X, int64_t ldhx, const float* H_G, int64_t ldhg, void* ws,
                             kq_stream_t stream, bool split_h, double* partial, int64_t* np_out) {
  cudaStream_t st = (cudaStream_t)stream;
  LossWs w;
  loss_layout(d_out, d_in, &w, ws);
  if (partial) w.partial = partial;
  // orientation: the smaller Hessian goes into the product (see the top of this file)
  const bool g_first = !H_G || d_in > d_out;
  const int64_t n2 = g_first ? d_in : d_out, n1 = g_first ? d_out : d_in, ldd = lead(n1);
  const float* H1 = g_first ? H_G : H_X;
  const int64_t ld1 = g_first ? ldhg : ldhx;
  const float* H2 = g_first ? H_X : H_G;
  const int64_t ld2 = g_first ? ldhx : ldhg;
  // D = dW (rows d_out) or dW^T (rows d_in), split into tf32 + remainder
  KQ_TRY(kq::split_tf32(W, ldw, W_hat, ldwh, d_out, d_in, w.Db, w.Ds, ldd, g_first, st));
  const float *Pa_b = w.Db, *Pa_s = w.Ds;   // A operand of P = A D^T: A1, or D when H1 = I
  if (H1) {
    if (split_h) KQ_TRY(kq::split_tf32(H1, ld1, nullptr, 0, n1, n1, w.Hb, w.Hs, lead(n1), false, st));
    kq::Gemm3xTF32 g1;                 // A1 = D H1^T   (B^T = H1 as stored)
    g1.M = n2;
    g1.N = n1;
    g1.K = n1;
    g1.a_big = w.Db;
    g1.a_small = w.Ds;
    g1.lda = ldd;
    g1.bt_big = w.Hb;
    g1.bt_small = w.Hs;
    g1.ldbt = lead(n1);
    g1.epilogue = kq::kEpiStoreSplit;
    g1.C = w.Ab;
    g1.C_small = w.As;
    g1.ldc = ldd;
    KQ_TRY(kq::gemm_3xtf32(g1, st));
    Pa_b = w.Ab;
    Pa_s = w.As;
  }
  kq::Gemm3xTF32 g2;                   // sum over the upper block triangle of (A1 D^T) .* H2
  g2.M = n2;
  g2.N = n2;
  g2.K = n1;
  g2.a_big = Pa_b;
  g2.a_small = Pa_s;
  g2.lda = ldd;
  g2.bt_big = w.Db;
  g2.bt_small = w.Ds;
  g2.ldbt = ldd;
  g2.epilogue = kq::kEpiDot;
  g2.upper = true;
  g2.other = H2;
  g2.ld_other = ld2;
  g2.partial = w.partial;
  KQ_TRY(kq::gemm_3xtf32(g2, st));
  *np_out = 8 * kq::gemm_tiles(n2, n2, n1, true);
  return KQ_OK;
}

// One loss; see kron_loss_products for `split_h`.
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
  int64_t np = 0;
  KQ_TRY(kron_loss_products(W, ldw, W_hat, ldwh, d_out, d_in, H_X, ldhx, H_G, ldhg, ws, stream, split_h, nullptr,
                            &np));
  LossWs w;
  loss_layout(d_out, d_in, &w, ws);
  sum_kernel<<<1, 1024, 0, st>>>(w.partial, np, loss);
  KQ_TRY(kq::launch_check("kq_kron_loss sum"));
  kq::clear_error();
  return KQ_OK;
}

}  // namespace

// Blockwise loss: the products of every row block into one partial region
// after the per-block workspace, then one fixed-order sum.
size_t blocks_partial_offset(int64_t d_in, int64_t k) {
  return kq::align_up(loss_layout(k, d_in, nullptr, nullptr), 256);
}

extern "C" size_t kq_kron_loss_blocks_workspace_size(int64_t d_out, int64_t d_in, int64_t k) {
  if (d_out < 1 || d_in < 1 || k < 1 || d_out % k) return 0;
  const int64_t n2 = std::max(k, d_in), n1 = std::min(k, d_in);
  return blocks_partial_offset(d_in, k) + (size_t)(d_out / k) * 8 * kq::gemm_tiles(n2, n2, n1, true) * sizeof(double);
}

extern "C" kq_status kq_kron_loss_blocks(const float* W, int64_t ldw, const float* W_hat, int64_t ldwh, int64_t d_out,
                                         int64_t d_in, const float* H_X, int64_t ldhx, const float* H_Gb, int64_t k,
                                         int64_t ldhgb, double* loss, void* ws, size_t ws_bytes,
                                         kq_stream_t stream) {
  if (!W || !W_hat || !H_X || !H_Gb || !loss) return kq::fail(KQ_ERR_INVALID_ARG, "kq_kron_loss_blocks: NULL pointer");
  if (d_out < 1 || d_in < 1 || k < 1 || d_out % k)
    return kq::fail(KQ_ERR_INVALID_ARG, "kq_kron_loss_blocks: sizes must be >= 1 and k must divide d_out");
  if (d_out > 65536 || d_in > 65536) return kq::fail(KQ_ERR_UNSUPPORTED_SHAPE, "kq_kron_loss_blocks: sizes above 65536");
  if (ldw < d_in || ldwh < d_in || ldhx < d_in || ldhgb < k)
    return kq::fail(KQ_ERR_INVALID_ARG, "kq_kron_loss_blocks: leading dimension too small");
  if (!ws || !kq::aligned(ws, 256) || ws_bytes < kq_kron_loss_blocks_workspace_size(d_out, d_in, k))
    return kq::fail(KQ_ERR_WORKSPACE, "kq_kron_loss_blocks: workspace too small or not 256-byte aligned");
  cudaStream_t st = (cudaStream_t)stream;
  double* partial = reinterpret_cast<double*>(static_cast<char*>(ws) + blocks_partial_offset(d_in, k));
  int64_t total = 0;
  for (int64_t b = 0; b < d_out / k; ++b) {
    int64_t np = 0;
    // the smaller Hessian of a block is its H_G block when k < d_in: split
    // it for every block; H_X (k >= d_in) only once
    const bool split = (k < d_in) || b == 0;
    KQ_TRY(kron_loss_products(W + b * k * ldw, ldw, W_hat + b * k * ldwh, ldwh, k, d_in, H_X, ldhx, H_Gb + b * k * ldhgb,
                              ldhgb, ws, stream, split, partial + total, &np));
    total += np;
  }
  sum_kernel<<<1, 1024, 0, st>>>(partial, total, loss);
  KQ_TRY(kq::launch_check("kq_kron_loss_blocks sum"));
  kq::clear_error();
  return KQ_OK;
}

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
  if (kq::cdiv(d_out, T) > 65535)   // the tile rows are the grid's y extent
    return kq::fail(KQ_ERR_UNSUPPORTED_SHAPE, "kq_kron_loss_noalloc: ceil(d_out/64) = %lld exceeds 65535",
                    (long long)kq::cdiv(d_out, T));
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
