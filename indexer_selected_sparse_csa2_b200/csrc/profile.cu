// Opt-in timing of the library's own kernels with CUDA events.
//
// When enabled, every launcher records one event on its launch stream just
// before and one just after its kernel; csa_profile_collect() waits for the
// recorded events and returns, per kernel name, the launch count and the
// summed event-to-event time.  Disabled by default; enabling it adds two
// event records per launch to the stream.  While the stream is being
// captured into a CUDA graph the records become external event-record nodes,
// re-recorded by every replay; csa_profile_snapshot() reads them after a
// replay without forgetting them.
#include <mutex>
#include <string>
#include <vector>

#include "common.cuh"

namespace csa {

namespace {
struct Rec {
  std::string name;
  cudaEvent_t start, stop;
};
std::mutex g_mu;
bool g_on = false;
std::vector<Rec> g_recs;
std::vector<cudaEvent_t> g_free;

cudaEvent_t take_event() {
  if (!g_free.empty()) {
    cudaEvent_t e = g_free.back();
    g_free.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  cudaEventCreate(&e);
  return e;
}
}  // namespace

ProfScope::ProfScope(cudaStream_t s, const char* name) : stream_(s), idx_(-1) {
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_on) return;
  Rec r{name, take_event(), take_event()};
  cudaStreamCaptureStatus st = cudaStreamCaptureStatusNone;
  cudaStreamIsCapturing(s, &st);
  capturing_ = st == cudaStreamCaptureStatusActive;
  if (capturing_) cudaEventRecordWithFlags(r.start, s, cudaEventRecordExternal);
  else cudaEventRecord(r.start, s);
  g_recs.push_back(r);
  idx_ = (int)g_recs.size() - 1;
}

ProfScope::~ProfScope() {
  if (idx_ < 0) return;
  std::lock_guard<std::mutex> lk(g_mu);
  if (idx_ >= (int)g_recs.size()) return;
  if (capturing_) cudaEventRecordWithFlags(g_recs[idx_].stop, stream_, cudaEventRecordExternal);
  else cudaEventRecord(g_recs[idx_].stop, stream_);
}

}  // namespace csa

using namespace csa;

extern "C" {

int32_t csa_profile_enable(int32_t on) {
  std::lock_guard<std::mutex> lk(g_mu);
  const int32_t prev = g_on ? 1 : 0;
  g_on = on != 0;
  return prev;
}

static int32_t summarize(std::vector<Rec>& recs, csa_kernel_time* out, int32_t max_entries);

int32_t csa_profile_snapshot(csa_kernel_time* out, int32_t max_entries) {
  std::vector<Rec> recs;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    recs = g_recs;
  }
  return summarize(recs, out, max_entries);
}

void csa_profile_reset(void) {
  std::lock_guard<std::mutex> lk(g_mu);
  for (Rec& r : g_recs) {
    g_free.push_back(r.start);
    g_free.push_back(r.stop);
  }
  g_recs.clear();
}

int32_t csa_profile_collect(csa_kernel_time* out, int32_t max_entries) {
  std::vector<Rec> recs;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    recs.swap(g_recs);
  }
  const int32_t n = summarize(recs, out, max_entries);
  std::lock_guard<std::mutex> lk(g_mu);
  for (Rec& r : recs) {
    g_free.push_back(r.start);
    g_free.push_back(r.stop);
  }
  return n;
}

static int32_t summarize(std::vector<Rec>& recs, csa_kernel_time* out, int32_t max_entries) {
  std::vector<std::string> names;
  std::vector<uint64_t> counts;
  std::vector<double> totals;
  for (Rec& r : recs) {
    float ms = 0.f;
    cudaEventSynchronize(r.stop);
    cudaEventElapsedTime(&ms, r.start, r.stop);
    size_t k = 0;
    while (k < names.size() && names[k] != r.name) ++k;
    if (k == names.size()) {
      names.push_back(r.name);
      counts.push_back(0);
      totals.push_back(0.0);
    }
    counts[k] += 1;
    totals[k] += ms;
  }
  const int32_t n = (int32_t)names.size();
  for (int32_t i = 0; i < n && i < max_entries && out; ++i) {
    snprintf(out[i].name, sizeof(out[i].name), "%s", names[i].c_str());
    out[i].launches = counts[i];
    out[i].total_ms = totals[i];
  }
  return n;
}

}  // extern "C"
