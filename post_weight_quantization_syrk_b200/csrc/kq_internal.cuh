// Internal helpers shared by the kronq CUDA sources (not part of the ABI).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>
#include <stdio.h>

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

// Launch-error check after a kernel launch; also counts the launch.
inline kq_status launch_check(const char* what) {
  count_launch();
  return cuda_check(cudaGetLastError(), what);
}

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

// Largest number of polls of a device wait before it gives up (~1 s at the
// shortest poll latency; every wait in this library is bounded).
constexpr long long kSpinLimit = 1LL << 26;

}  // namespace kq
