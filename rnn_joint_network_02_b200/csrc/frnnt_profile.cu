// Stage tracing: launch counts (always on) and optional CUDA-event timing.
#include <stdlib.h>
#include <string.h>

#include <vector>

#include "frnnt_internal.h"

namespace frnnt {
namespace {

struct Stage {
  char name[32];
  int launches = 0;
  int calls = 0;
  double ms = 0.0;
};

struct Pending {
  int stage;
  cudaEvent_t start, stop;
};

bool g_timing = false;
long long g_launches = 0;
std::vector<Stage> g_stages;
std::vector<Pending> g_pending;
std::vector<cudaEvent_t> g_free_events;

int stage_index(const char* name) {
  for (size_t i = 0; i < g_stages.size(); ++i)
    if (strncmp(g_stages[i].name, name, sizeof(g_stages[i].name)) == 0) return (int)i;
  Stage s;
  strncpy(s.name, name, sizeof(s.name) - 1);
  s.name[sizeof(s.name) - 1] = 0;
  g_stages.push_back(s);
  return (int)g_stages.size() - 1;
}

cudaEvent_t take_event() {
  if (!g_free_events.empty()) {
    cudaEvent_t e = g_free_events.back();
    g_free_events.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
  return e;
}

}  // namespace

void note_launch(int n) { g_launches += n; }

// ---------------------------------------------------------------- launch chaining (per host thread)
namespace {
struct Chain {
  cudaStream_t st = nullptr;
  bool active = false;   // a call is queueing on st
  bool armed = false;    // the last operation queued on st was one of the call's kernels
};
thread_local Chain t_chain;
bool chain_enabled() {
  // FRNNT_CHAIN=0 in the environment turns chaining off (every launch then
  // waits for the previous one in the plain stream order)
  static const bool on = [] {
    const char* e = getenv("FRNNT_CHAIN");
    return !(e && e[0] == '0');
  }();
  return on;
}
}  // namespace

void chain_begin(cudaStream_t st) {
  t_chain.st = st;
  t_chain.active = chain_enabled();
  t_chain.armed = false;
}
void chain_break(cudaStream_t st) {
  if (t_chain.active && st == t_chain.st) t_chain.armed = false;
}
void chain_end() { t_chain = Chain{}; }
bool chain_take(cudaStream_t st) { return t_chain.active && t_chain.armed && st == t_chain.st; }
void chain_note(cudaStream_t st) {
  if (t_chain.active && st == t_chain.st) t_chain.armed = true;
}

StageScope::StageScope(const char* name, cudaStream_t st) : st_(st), launches0_(g_launches) {
  stage_ = stage_index(name);
  if (g_timing) {
    start_ = take_event();
    if (start_) cudaEventRecord(start_, st_);
    chain_break(st_);
  }
}

StageScope::~StageScope() {
  Stage& s = g_stages[stage_];
  s.launches += (int)(g_launches - launches0_);
  s.calls += 1;
  if (g_timing && start_) {
    cudaEvent_t stop = take_event();
    if (stop) {
      cudaEventRecord(stop, st_);
      chain_break(st_);
      g_pending.push_back({stage_, (cudaEvent_t)start_, stop});
    } else {
      g_free_events.push_back((cudaEvent_t)start_);
    }
  }
}

}  // namespace frnnt

using namespace frnnt;

extern "C" FRNNT_API int frnnt_profile(int enable) {
  g_timing = enable != 0;
  return FRNNT_OK;
}

extern "C" FRNNT_API int frnnt_profile_read(frnnt_stage_stat* out, int capacity, int* count) {
  int rc = FRNNT_OK;
  for (const Pending& p : g_pending) {
    float ms = 0.f;
    if (cudaEventSynchronize(p.stop) != cudaSuccess || cudaEventElapsedTime(&ms, p.start, p.stop) != cudaSuccess)
      rc = FRNNT_ERR_CUDA;
    g_stages[p.stage].ms += ms;
    g_free_events.push_back(p.start);
    g_free_events.push_back(p.stop);
  }
  g_pending.clear();
  int n = (int)g_stages.size();
  if (count) *count = n;
  for (int i = 0; i < n && out && i < capacity; ++i) {
    memcpy(out[i].name, g_stages[i].name, sizeof(out[i].name));
    out[i].launches = g_stages[i].launches;
    out[i].calls = g_stages[i].calls;
    out[i].ms = g_stages[i].ms;
  }
  for (Stage& s : g_stages) {
    s.launches = 0;
    s.calls = 0;
    s.ms = 0.0;
  }
  return rc;
}
