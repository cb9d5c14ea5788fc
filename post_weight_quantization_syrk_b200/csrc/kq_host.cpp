// Host-only parts of the kronq ABI: status strings, the thread-local error
// detail, the version, and the sublayer bit allocation.
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <numeric>
#include <vector>

#include "kronq.h"

namespace kq {

static thread_local char g_last_error[512] = {0};

void set_error(const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
}

void clear_error() { g_last_error[0] = 0; }

static std::atomic<unsigned long long> g_launches{0};
void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

static std::atomic<unsigned long long> g_wait_limit_ns{KQ_WAIT_LIMIT_DEFAULT_NS};
unsigned long long wait_limit_ns() { return g_wait_limit_ns.load(std::memory_order_relaxed); }

kq_status fail(kq_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
  return s;
}

}  // namespace kq

extern "C" {

const char* kq_status_string(kq_status s) {
  switch (s) {
    case KQ_OK: return "KQ_OK";
    case KQ_ERR_INVALID_ARG: return "KQ_ERR_INVALID_ARG";
    case KQ_ERR_UNSUPPORTED_SHAPE: return "KQ_ERR_UNSUPPORTED_SHAPE";
    case KQ_ERR_ALIGNMENT: return "KQ_ERR_ALIGNMENT";
    case KQ_ERR_WORKSPACE: return "KQ_ERR_WORKSPACE";
    case KQ_ERR_CUDA: return "KQ_ERR_CUDA";
    case KQ_ERR_NOT_PD: return "KQ_ERR_NOT_PD";
    case KQ_ERR_NONFINITE: return "KQ_ERR_NONFINITE";
    case KQ_ERR_TIMEOUT: return "KQ_ERR_TIMEOUT";
  }
  return "KQ_ERR_UNKNOWN";
}

const char* kq_last_error(void) { return kq::g_last_error; }

unsigned long long kq_set_wait_limit_ns(unsigned long long ns) {
  return kq::g_wait_limit_ns.exchange(ns, std::memory_order_relaxed);
}

int kq_version(void) { return 100; }  // 0.1.0

unsigned long long kq_launch_count(void) { return kq::g_launches.load(std::memory_order_relaxed); }

// Greedy upgrade ordering (see kronq.h).  Pure host code.
kq_status kq_allocate_bits(const double* sens, const int64_t* n_params, int n_layers,
                           const int* choices, int n_choices, double avg_bits,
                           int* bits_out) {
  if (n_layers < 0 || n_choices < 1) return kq::fail(KQ_ERR_INVALID_ARG, "n_layers < 0 or n_choices < 1");
  if (n_layers == 0) return KQ_OK;
  if (!sens || !n_params || !choices || !bits_out) return kq::fail(KQ_ERR_INVALID_ARG, "NULL pointer");
  std::vector<int> ch(choices, choices + n_choices);
  std::sort(ch.begin(), ch.end());
  for (int i = 0; i < n_choices; ++i) {
    if (ch[i] < 1 || ch[i] > 16) return kq::fail(KQ_ERR_INVALID_ARG, "choice %d outside 1..16", ch[i]);
    if (i && ch[i] == ch[i - 1]) return kq::fail(KQ_ERR_INVALID_ARG, "duplicate choice %d", ch[i]);
  }
  double total = 0.0;
  for (int k = 0; k < n_layers; ++k) {
    if (n_params[k] <= 0) return kq::fail(KQ_ERR_INVALID_ARG, "n_params[%d] <= 0", k);
    if (!std::isfinite(sens[k])) return kq::fail(KQ_ERR_INVALID_ARG, "sens[%d] not finite", k);
    total += (double)n_params[k];
  }
  if (!std::isfinite(avg_bits)) return kq::fail(KQ_ERR_INVALID_ARG, "avg_bits not finite");
  const int lo = ch.front();
  double b = std::floor(total * (avg_bits - (double)lo) * (1.0 + 1e-12));
  long long budget = b > 0 ? (long long)b : 0;
  std::vector<int> order(n_layers);
  std::iota(order.begin(), order.end(), 0);
  std::stable_sort(order.begin(), order.end(), [&](int a, int c) { return sens[a] > sens[c]; });
  for (int k = 0; k < n_layers; ++k) bits_out[k] = lo;
  for (int k : order) {
    for (int i = n_choices - 1; i >= 1; --i) {
      long long cost = (long long)n_params[k] * (long long)(ch[i] - lo);
      if (cost <= budget) {
        bits_out[k] = ch[i];
        budget -= cost;
        break;
      }
    }
  }
  kq::clear_error();
  return KQ_OK;
}

}  // extern "C"
