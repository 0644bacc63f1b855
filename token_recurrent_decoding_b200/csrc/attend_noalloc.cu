// rlt_attend_noalloc: the standalone decode attention (rlt_attend) for
// callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc, or any routine that allocates: a
// serving process whose memory pool already holds the whole GPU and forbids
// further allocations, a plugin that is handed only its input and output
// buffers, or code running where an allocation would synchronise the device
// at the wrong moment. rlt_attend needs a scratch workspace (the split-KV
// partial results, the merge counters, the per-row positions); this variant
// takes it from a fixed array compiled into the library instead of from the
// caller.
//
// The scratch is a file-scope __device__ array of RLT_ATTEND_NOALLOC_BYTES.
// Every GPU that loads the library holds it until the process exits. Host
// code may not use the array's name as a device address (it is a host-side
// stand-in), so the first call on each device, with that device current,
// looks the address up with cudaGetSymbolAddress and caches it; that first
// call should come before any stream capture. All calls share the one array:
// the per-call parts that must start at zero are cleared by every call, and
// calls that overlap on the GPU race on it.
#include <mutex>

#include "../../include/rlt.h"
#include "internal.h"

static __device__ __align__(256) unsigned char g_attend_scratch[RLT_ATTEND_NOALLOC_BYTES];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_lock;
void *g_scratch[kMaxDevices] = {};

// Device address of the scratch array on the current device.
int scratch_on_current_device(void **out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return RLT_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return RLT_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> guard(g_lock);
  if (!g_scratch[dev]) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_attend_scratch) != cudaSuccess || !p) {
      cudaGetLastError();
      return RLT_ERR_CUDA;
    }
    g_scratch[dev] = p;
  }
  *out = g_scratch[dev];
  return RLT_OK;
}

}  // namespace

extern "C" RLT_API int rlt_attend_noalloc(const float *q, const void *kv,
                                          const int32_t *h_lengths, int n, int n_heads,
                                          int head_dim, int cap, int dtype, void *out,
                                          rlt_stream stream) {
  const size_t need = rlt::attend_workspace_internal(n, n_heads, head_dim, cap);
  if (need > RLT_ATTEND_NOALLOC_BYTES) return RLT_ERR_CAPACITY;
  void *scratch = nullptr;
  int rc = scratch_on_current_device(&scratch);
  if (rc != RLT_OK) return rc;
  // invalid shapes (need == 0) are rejected by the shared validation
  return rlt::attend_run_internal(q, kv, h_lengths, n, n_heads, head_dim, cap, dtype, out,
                                  scratch, RLT_ATTEND_NOALLOC_BYTES, (cudaStream_t)stream);
}
