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

#include "../../include/gdn.h"
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
  const size_t need = gdn_chunk_prefill_workspace_size(T, cu_seqlens ? n_seq : 1, Hk, Hv, dk, dv, dt);
  if (need == SIZE_MAX || need == 0) {
    // unsupported shapes get the regular validation and status; shapes that need no
    // scratch run the regular path directly
    return gdn_chunk_prefill(q, k, v, g, beta, o, dt, T, Hk, Hv, dk, dv, qk_stride, v_stride,
                             cu_seqlens, n_seq, initial_state, final_state, scale, qk_l2norm,
                             nullptr, 0, stream);
  }
  if (need > kNoallocScratchBytes) {
    // the regular entry point reports the size in gdn_last_error(); call it with no
    // workspace so that it fails validation without launching anything
    gdn_status_t s = gdn_chunk_prefill(q, k, v, g, beta, o, dt, T, Hk, Hv, dk, dv, qk_stride,
                                       v_stride, cu_seqlens, n_seq, initial_state, final_state,
                                       scale, qk_l2norm, nullptr, kNoallocScratchBytes, stream);
    return s == GDN_OK ? GDN_ERR_WORKSPACE : s;
  }
  void* scratch = nullptr;
  if (scratch_for_current_device(&scratch) != cudaSuccess) return GDN_ERR_CUDA;
  return gdn_chunk_prefill(q, k, v, g, beta, o, dt, T, Hk, Hv, dk, dv, qk_stride, v_stride,
                           cu_seqlens, n_seq, initial_state, final_state, scale, qk_l2norm,
                           scratch, kNoallocScratchBytes, stream);
}

extern "C" gdn_status_t gdn_prefill_noalloc_status(gdn_stream_t stream) {
  void* scratch = nullptr;
  if (scratch_for_current_device(&scratch) != cudaSuccess) return GDN_ERR_CUDA;
  return gdn_prefill_status(scratch, stream);
}
