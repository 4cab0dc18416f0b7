// Launch accounting and optional per-kind CUDA-event timing.
#include <atomic>
#include <cstring>
#include <map>
#include <mutex>
#include <string>
#include <vector>

#include <nvtx3/nvToolsExt.h>

#include "poet_internal.cuh"

namespace poet {
namespace {

std::atomic<long long> g_launches{0};
std::atomic<bool> g_trace{false};
std::atomic<double> g_ridge{216.0};  // flop per byte: measured bf16 peak over copy peak

struct Rec {
  std::string kind;
  double flop, bytes;
  cudaEvent_t e0, e1;
};

std::mutex g_mu;
std::vector<Rec> g_recs;
std::vector<cudaEvent_t> g_pool;

cudaEvent_t take_event() {
  if (!g_pool.empty()) {
    cudaEvent_t e = g_pool.back();
    g_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  cudaEventCreate(&e);
  return e;
}

}  // namespace

void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }
bool trace_on() { return g_trace.load(std::memory_order_relaxed); }

CallRange::CallRange(const char *name) { nvtxRangePushA(name); }
CallRange::~CallRange() { nvtxRangePop(); }

TraceScope::TraceScope(const char *kind, double flop, double bytes, cudaStream_t s) : st(s) {
  nvtxRangePushA(kind);
  if (!trace_on()) return;
  std::lock_guard<std::mutex> lock(g_mu);
  Rec r{kind, flop, bytes, take_event(), take_event()};
  if (!r.e0 || !r.e1) return;
  cudaEventRecord(r.e0, st);
  slot = int(g_recs.size());
  g_recs.push_back(r);
}

TraceScope::~TraceScope() {
  if (slot >= 0) {
    std::lock_guard<std::mutex> lock(g_mu);
    cudaEventRecord(g_recs[slot].e1, st);
  }
  nvtxRangePop();
}

}  // namespace poet

using namespace poet;

extern "C" {

int64_t poet_launch_count(void) { return g_launches.load(); }

poet_status poet_trace_enable(int32_t on) {
  g_trace.store(on != 0);
  return POET_OK;
}

poet_status poet_trace_set_ridge(double flop_per_byte) {
  POET_REQUIRE(flop_per_byte > 0.0, "poet_trace_set_ridge: ridge %g must be positive", flop_per_byte);
  g_ridge.store(flop_per_byte);
  return POET_OK;
}

int32_t poet_trace_read(poet_trace_row *rows, int32_t max_rows) {
  std::lock_guard<std::mutex> lock(g_mu);
  std::map<std::string, poet_trace_row> agg;
  const double ridge = g_ridge.load();
  for (auto &r : g_recs) {
    float ms = 0.f;
    if (cudaEventSynchronize(r.e1) == cudaSuccess) cudaEventElapsedTime(&ms, r.e0, r.e1);
    poet_trace_row &a = agg[r.kind];
    a.launches += 1;
    a.ms += ms;
    a.flop += r.flop;
    a.bytes += r.bytes;
    if (r.flop > 0.0 && r.flop >= ridge * r.bytes)
      a.flop_tc += r.flop;
    else
      a.bytes_hbm += r.bytes;
    g_pool.push_back(r.e0);
    g_pool.push_back(r.e1);
  }
  g_recs.clear();
  int32_t n = 0;
  for (auto &kv : agg) {
    if (!rows || n >= max_rows) break;
    rows[n] = kv.second;
    std::strncpy(rows[n].kind, kv.first.c_str(), sizeof(rows[n].kind) - 1);
    rows[n].kind[sizeof(rows[n].kind) - 1] = 0;
    ++n;
  }
  return n;
}

}  // extern "C"
