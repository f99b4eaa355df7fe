// Per-kernel timing of the library's launches with CUDA events, and a launch
// counter.  When profiling is on, every kernel launch of the library is bracketed by
// two events recorded on the launching stream; zdit_profile_end waits for them and
// aggregates elapsed time, algorithmic FLOPs and algorithmic bytes per kernel kind.
#include <cuda_runtime.h>

#include <atomic>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <vector>

#include "internal.h"

namespace zdit {

namespace {

const char* kKindNames[PROF_NUM_KINDS] = {
    "gemm_qkv_rope", "gemm_out_proj", "gemm_gate_up_swiglu", "gemm_down_proj", "gemm_embed_final",
    "attention",     "norm_modulate", "residual_norm",       "adaln_gemv",     "euler_cfg",
    "rope_table",    "misc"};

struct Rec {
  int kind;
  double flops, bytes;
  cudaEvent_t a, b;
};

struct Prof {
  std::mutex mu;
  bool on = false;
  std::vector<cudaEvent_t> pool;
  size_t used = 0;
  std::vector<Rec> recs;
  int64_t dropped = 0;
};

Prof& prof() {
  static Prof p;
  return p;
}

std::atomic<int64_t> g_launches{0};

}  // namespace

ProfScope::ProfScope(int kind, double flops, double bytes, cudaStream_t s)
    : kind_(kind), flops_(flops), bytes_(bytes), s_(s) {
  g_launches.fetch_add(1, std::memory_order_relaxed);
  Prof& p = prof();
  if (!p.on) return;
  std::lock_guard<std::mutex> g(p.mu);
  if (!p.on || p.used + 2 > p.pool.size()) {
    ++p.dropped;
    return;
  }
  a_ = p.pool[p.used++];
  b_ = p.pool[p.used++];
  cudaEventRecord(a_, s_);
  active_ = true;
}

ProfScope::~ProfScope() {
  if (!active_) return;
  Prof& p = prof();
  cudaEventRecord(b_, s_);
  std::lock_guard<std::mutex> g(p.mu);
  p.recs.push_back(Rec{kind_, flops_, bytes_, a_, b_});
}

bool profiling_on() {
  Prof& p = prof();
  std::lock_guard<std::mutex> g(p.mu);
  return p.on;
}

void add_launches(int64_t n) { g_launches.fetch_add(n, std::memory_order_relaxed); }

#ifndef ZDIT_PDL_DEFAULT
#define ZDIT_PDL_DEFAULT 1
#endif

bool pdl_enabled() {
  static const bool on = [] {
    const char* e = getenv("ZDIT_PDL");
    return e != nullptr ? e[0] != '0' : ZDIT_PDL_DEFAULT != 0;
  }();
  return on;
}

}  // namespace zdit

using namespace zdit;

extern "C" {

ZDIT_API int64_t zdit_launch_count(void) { return g_launches.load(); }

ZDIT_API zdit_status zdit_profile_begin(int32_t max_records) {
  if (max_records <= 0 || max_records > (1 << 20)) return ZDIT_ERR_INVALID_ARG;
  Prof& p = prof();
  std::lock_guard<std::mutex> g(p.mu);
  for (cudaEvent_t e : p.pool) cudaEventDestroy(e);
  p.pool.clear();
  p.recs.clear();
  p.used = 0;
  p.dropped = 0;
  for (int i = 0; i < 2 * max_records; ++i) {
    cudaEvent_t e;
    if (cudaEventCreate(&e) != cudaSuccess) {
      p.on = false;
      return ZDIT_ERR_CUDA;
    }
    p.pool.push_back(e);
  }
  p.on = true;
  return ZDIT_OK;
}

ZDIT_API zdit_status zdit_profile_end(zdit_profile_entry* entries, int32_t max_entries, int32_t* n_entries) {
  if (!entries || !n_entries || max_entries < PROF_NUM_KINDS) return ZDIT_ERR_INVALID_ARG;
  Prof& p = prof();
  std::lock_guard<std::mutex> g(p.mu);
  p.on = false;
  zdit_profile_entry agg[PROF_NUM_KINDS];
  std::memset(agg, 0, sizeof(agg));
  zdit_status st = ZDIT_OK;
  for (const Rec& r : p.recs) {
    float ms = 0.f;
    if (cudaEventSynchronize(r.b) != cudaSuccess || cudaEventElapsedTime(&ms, r.a, r.b) != cudaSuccess) {
      st = ZDIT_ERR_CUDA;
      continue;
    }
    zdit_profile_entry& e = agg[r.kind];
    e.launches += 1;
    e.total_ms += ms;
    e.flops += r.flops;
    e.bytes += r.bytes;
  }
  int n = 0;
  for (int k = 0; k < PROF_NUM_KINDS; ++k) {
    if (agg[k].launches == 0) continue;
    std::strncpy(agg[k].name, kKindNames[k], sizeof(agg[k].name) - 1);
    entries[n++] = agg[k];
  }
  *n_entries = n;
  for (cudaEvent_t e : p.pool) cudaEventDestroy(e);
  p.pool.clear();
  p.recs.clear();
  p.used = 0;
  return st;
}

}  // extern "C"
