// Internal helpers shared by the kronq CUDA sources (not part of the ABI).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>
#include <stdio.h>

#include <utility>

#include "kronq.h"

namespace kq {

// Thread-local detail string behind kq_last_error().
void set_error(const char* fmt, ...);
void clear_error();

// Returns `s` after recording `msg`; used as `return fail(KQ_ERR_..., "...")`.
kq_status fail(kq_status s, const char* fmt, ...);

inline kq_status cuda_check(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return KQ_OK;
  return fail(KQ_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

// Counts kernel launches enqueued by this library (see kq_launch_count).
void count_launch();

// Current limit of the tensor-core kernels' device waits (kq_set_wait_limit_ns).
unsigned long long wait_limit_ns();

// Launch-error check after a kernel launch; also counts the launch.
inline kq_status launch_check(const char* what) {
  count_launch();
  return cuda_check(cudaGetLastError(), what);
}
inline kq_status launch_check_nocount(const char* what) { return cuda_check(cudaGetLastError(), what); }

#define KQ_TRY(expr)                   \
  do {                                 \
    kq_status _s = (expr);             \
    if (_s != KQ_OK) return _s;        \
  } while (0)

inline bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

inline int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Device-side sticky error: the first error wins.
__device__ __forceinline__ void report(int32_t* info, int code, int64_t index) {
  if (info == nullptr) return;
  int64_t idx = index < 0 ? 0 : (index > 0xFFFFFF ? 0xFFFFFF : index);
  int32_t v = (int32_t)(((uint32_t)code << 24) | (uint32_t)idx);
  atomicCAS(info, 0, v);
}

// Programmatic dependent launch within one call's chain of kernels.  A
// kernel launched with launch_ex(..., pdl = true) may be scheduled while its
// predecessor on the stream is still running: it does its set-up (barriers,
// TMEM, reads of data that no kernel of the chain writes), then pdl_wait(),
// which returns once the predecessor grid has completed with its writes
// visible; every other global access comes after that.  pdl_trigger() lets
// the successor be scheduled from then on (otherwise it is as each block
// exits).  Launched without the attribute, both are no-ops.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

template <typename... KArgs, typename... Args>
kq_status launch_ex(const char* what, bool pdl, void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                    cudaStream_t st, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
  count_launch();
  if (e != cudaSuccess) {
    (void)cudaGetLastError();
    return cuda_check(e, what);
  }
  return launch_check_nocount(what);
}

// Largest number of polls of a device wait before it gives up (~1 s at the
// shortest poll latency; every wait in this library is bounded).
constexpr long long kSpinLimit = 1LL << 26;

}  // namespace kq
