// prefill_noalloc.cu -- gdn_chunk_prefill_noalloc: the chunked prefill with its scratch
// memory in a fixed, library-owned device array instead of a caller workspace.
//
// For callers that cannot allocate device memory: for example a plugin running inside a
// host application that owns all GPU memory through its own pool and offers no allocation
// hook, or a latency-critical loop where a cudaMalloc (and the device-wide
// synchronisation it may imply) is not acceptable. Such a caller still passes its inputs
// and outputs; only the workspace comes from here.
//
// The scratch is a file-scope __device__ array of kNoallocScratchBytes. Every GPU that
// loads this library holds that much memory until the process exits. In host code the
// array's name does not denote a device address, so its address is fetched once per
// device with cudaGetSymbolAddress (with that device current) and cached.
#include <mutex>

#include "gdn.h"
#include "launch.h"

namespace {

constexpr size_t kNoallocScratchBytes = size_t(64) << 20;   // 64 MiB

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device (set-up on first use).
cudaError_t scratch_for_current_device(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" gdn_status_t gdn_chunk_prefill_noalloc(
    const void* q, const void* k, const void* v, const float* g, const float* beta, void* o,
    gdn_dtype_t dt, int64_t T, int32_t Hk, int32_t Hv, int32_t dk, int32_t dv, int64_t qk_stride,
    int64_t v_stride, const int32_t* cu_seqlens, int32_t n_seq, const float* initial_state,
    float* final_state, float scale, int32_t qk_l2norm, gdn_stream_t stream) {
  // the scratch the path taken by these arguments needs (0 for the token-recurrent path;
  // SIZE_MAX for unsupported arguments, which the regular validation below reports)
  const size_t need = gdn::prefill_workspace_need(dt, T, cu_seqlens ? n_seq : 1, Hk, Hv, dk, dv,
                                                  qk_l2norm);
  if (need != SIZE_MAX && need > kNoallocScratchBytes)
    return gdn::set_error(GDN_ERR_WORKSPACE,
                          "chunk_prefill_noalloc: these sizes need %zu bytes of scratch, more than "
                          "the %zu-byte static array; nothing was launched (split the batch, or "
                          "use gdn_chunk_prefill with a workspace)", need, kNoallocScratchBytes);
  void* scratch = nullptr;
  const cudaError_t e = scratch_for_current_device(&scratch);
  if (e != cudaSuccess)
    return gdn::set_error(GDN_ERR_CUDA, "chunk_prefill_noalloc: scratch address: %s", cudaGetErrorString(e));
  // always hand over the scratch, so that every path clears its status word
  return gdn_chunk_prefill(q, k, v, g, beta, o, dt, T, Hk, Hv, dk, dv, qk_stride, v_stride,
                           cu_seqlens, n_seq, initial_state, final_state, scale, qk_l2norm,
                           scratch, kNoallocScratchBytes, stream);
}

extern "C" gdn_status_t gdn_prefill_noalloc_status(gdn_stream_t stream) {
  void* scratch = nullptr;
  const cudaError_t e = scratch_for_current_device(&scratch);
  if (e != cudaSuccess)
    return gdn::set_error(GDN_ERR_CUDA, "prefill_noalloc_status: scratch address: %s", cudaGetErrorString(e));
  return gdn_prefill_status(scratch, stream);
}
