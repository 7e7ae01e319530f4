// Per-kernel event timing of libspa2 (spa2_timing_enable / spa2_timing_read in
// include/spa2.h). While timing is on, every kernel the library launches is
// bracketed by two CUDA events recorded on its launch stream; a read waits for
// the recorded events, sums the elapsed time per kernel and recycles them.
// Off by default: with timing off a KernelTimer does nothing.
#include <mutex>
#include <vector>

#include "common.cuh"
#include "kernels.h"

namespace spa2 {

namespace {

const char* const kNames[KID_COUNT] = {
    "pool_kernel",        // KID_POOL
    "select_kernel",      // KID_SELECT
    "logits_kernel",      // KID_LOGITS
    "csc_kernel",         // KID_CSC
    "pbar_select_kernel", // KID_PBAR_SELECT
    "v_to_f16_kernel",    // KID_V16
    "fwd_kernel",         // KID_FWD
    "bwd_pre_kernel",     // KID_BWD_PRE
    "bwd_dkdv_kernel",    // KID_BWD_DKDV
    "bwd_dq_kernel",      // KID_BWD_DQ
    "timeout_probe_kernel",  // KID_PROBE
    "tile_list_kernel",   // KID_TILES
};

struct Record {
  int kid;
  cudaEvent_t start, stop;
};

std::mutex g_mu;
bool g_on = false;
std::vector<cudaEvent_t> g_free;   // recycled events
std::vector<Record> g_recs;        // recorded, not yet read

cudaEvent_t take_event() {  // g_mu held
  if (!g_free.empty()) {
    cudaEvent_t e = g_free.back();
    g_free.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
  return e;
}

}  // namespace

KernelTimer::KernelTimer(int kid, cudaStream_t s) : slot_(-1), s_(s) {
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_on || kid < 0 || kid >= KID_COUNT) return;
  Record r{kid, take_event(), take_event()};
  if (!r.start || !r.stop || cudaEventRecord(r.start, s) != cudaSuccess) {
    if (r.start) g_free.push_back(r.start);
    if (r.stop) g_free.push_back(r.stop);
    return;
  }
  slot_ = (int)g_recs.size();
  g_recs.push_back(r);
}

KernelTimer::~KernelTimer() {
  if (slot_ < 0) return;
  std::lock_guard<std::mutex> lock(g_mu);
  if (slot_ < (int)g_recs.size()) cudaEventRecord(g_recs[slot_].stop, s_);
}

}  // namespace spa2

using namespace spa2;

extern "C" {

spa2_status spa2_timing_enable(int on) {
  std::lock_guard<std::mutex> lock(g_mu);
  g_on = on != 0;
  return SPA2_OK;
}

int spa2_kernel_count(void) { return KID_COUNT; }

const char* spa2_kernel_name(int kernel_id) {
  return (kernel_id >= 0 && kernel_id < KID_COUNT) ? kNames[kernel_id] : "unknown";
}

spa2_status spa2_timing_read(int n, int* launches, double* total_ms) {
  if (n < 0 || (n > 0 && (!launches || !total_ms))) return SPA2_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lock(g_mu);
  for (int i = 0; i < n; ++i) {
    launches[i] = 0;
    total_ms[i] = 0.0;
  }
  spa2_status st = SPA2_OK;
  for (const Record& r : g_recs) {
    float ms = 0.f;
    if (cudaEventSynchronize(r.stop) != cudaSuccess || cudaEventElapsedTime(&ms, r.start, r.stop) != cudaSuccess)
      st = SPA2_ERR_CUDA;
    else if (r.kid < n) {
      launches[r.kid] += 1;
      total_ms[r.kid] += ms;
    }
    g_free.push_back(r.start);
    g_free.push_back(r.stop);
  }
  g_recs.clear();
  return st;
}

}  // extern "C"
