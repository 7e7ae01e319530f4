// spa2_block_mask_noalloc: the block-mask computation of spa2_block_mask with
// its scratch (status word, pooled Q-bar / K-bar, per-row bit words) held in a
// fixed, file-scope device array instead of a caller-supplied workspace.
//
// Who needs it: callers that cannot hand the library a workspace at call
// time, e.g. a plain C host program that runs on a fixed memory plan with no
// device allocator of its own, or a step loop that must not call cudaMalloc
// (which synchronises the whole device) between kernels. The library never
// allocates here either: the array is part of this module's image and exists
// once per device as soon as the module is loaded on that device.
//
// Setup: on the first call on each device (with that device current), the
// address of the array on that device is looked up once with
// cudaGetSymbolAddress and cached; that lookup may load the module. Make the
// first call on each device before any stream capture begins. A
// cudaDeviceReset unloads the module on that device, so the cached address is
// stale afterwards: calls after a reset are not supported.
//
// Limits: one array per device, shared by every call on that device, so two
// calls whose executions overlap (different streams, or different host
// threads) race on it and produce garbage; calls issued one after another on
// one stream are safe. Shapes whose scratch exceeds SPA2_NOALLOC_MASK_SCRATCH_BYTES
// are refused with SPA2_ERR_WORKSPACE before anything is launched.
#include <mutex>

#include "common.cuh"

namespace spa2 {

static __device__ __align__(256) unsigned char g_mask_scratch[SPA2_NOALLOC_MASK_SCRATCH_BYTES];

static constexpr int kMaxDevices = 64;
static void* g_scratch_ptr[kMaxDevices] = {};
static std::mutex g_scratch_mu;

// Device address of g_mask_scratch on the current device, or nullptr.
static void* scratch_for_current_device() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_mask_scratch) != cudaSuccess || !p) return nullptr;
    g_scratch_ptr[dev] = p;
  }
  return g_scratch_ptr[dev];
}

}  // namespace spa2

extern "C" {

spa2_status spa2_block_mask_noalloc(const void* q, const void* k, int B, int H, int N, int d, int bq, int bkv,
                                    float k_frac, float p_frac, const spa2_mask* out, int* status,
                                    spa2_stream_t stream) {
  if (status && (reinterpret_cast<uintptr_t>(status) % 4) != 0) return SPA2_ERR_INVALID_ARG;
  // spa2_workspace_bytes returns 0 for shapes the mask op does not support;
  // spa2_block_mask then reports the precise reason.
  const size_t need = spa2_workspace_bytes(SPA2_OP_MASK, B, H, N, d, bq, bkv);
  if (need > (size_t)SPA2_NOALLOC_MASK_SCRATCH_BYTES) return SPA2_ERR_WORKSPACE;
  void* scratch = spa2::scratch_for_current_device();
  if (!scratch) return SPA2_ERR_CUDA;
  // spa2_block_mask zeroes the status word (the one scratch item that must
  // start at zero) on `stream`; every other scratch byte it reads is first
  // written by the same call.
  const spa2_status st = spa2_block_mask(q, k, B, H, N, d, bq, bkv, k_frac, p_frac, out, scratch,
                                         (size_t)SPA2_NOALLOC_MASK_SCRATCH_BYTES, stream);
  if (st != SPA2_OK || !status) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(status, scratch, 4, cudaMemcpyDeviceToDevice, s) != cudaSuccess) return SPA2_ERR_CUDA;
  return SPA2_OK;
}

}  // extern "C"
