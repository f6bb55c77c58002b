// esa_noalloc.cu -- a forward scan that allocates nothing.
//
// Some callers cannot allocate device memory where they call the scan:
// serving loops whose device-memory budget is fixed when they start, code in
// latency-critical paths where cudaMalloc may implicitly synchronise the
// whole device, and foreign-language callers that are only handed tensor
// pointers and have no device allocator of their own.  esa_scan_fwd_noalloc
// serves them: it runs the same forward scan as esa_scan_fwd, but its scratch
// (the chunk carry words) lives in the file-scope array below instead of a
// caller-provided workspace.  The caller still passes inputs and outputs.
//
// The array costs ESA_NOALLOC_SCRATCH_BYTES of device memory on every GPU on
// which this part of the library is loaded, until the process exits.
#include <cuda_runtime.h>

#include <mutex>

#include "esa.h"

namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[ESA_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
void *g_scratch_ptr[kMaxDevices] = {};

// Once per device, with that device current: resolve the device address of
// the array (in host code its name is only a host-side stand-in) and prepare
// it as a workspace (zero it, write its header).  Synchronises `stream` once.
int noalloc_scratch(void *stream, void **out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return ESA_ERR_DEVICE;
  }
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (g_scratch_ptr[dev] == nullptr) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      return ESA_ERR_LAUNCH;
    }
    int rc = esa_workspace_init(p, ESA_NOALLOC_SCRATCH_BYTES, stream);
    if (rc != ESA_OK) return rc;
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) {
      cudaGetLastError();
      return ESA_ERR_LAUNCH;
    }
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return ESA_OK;
}

}  // namespace

extern "C" int esa_scan_fwd_noalloc(const void *a, const void *v, const void *q, void *y, float *E_final,
                                    int B, int T, int H, int D, int mode, const float *E_init, int dtype,
                                    void *stream) {
  const size_t need = esa_workspace_size(B, T, H, D, dtype);
  if (need == 0) {
    // A shape the scan rejects: let the full argument check report why.
    return esa_scan_fwd(a, v, q, y, E_final, B, T, H, D, mode, E_init, dtype, nullptr, 0, stream);
  }
  if (need > ESA_NOALLOC_SCRATCH_BYTES) return ESA_ERR_NOALLOC_LIMIT;
  void *scratch = nullptr;
  const int rc = noalloc_scratch(stream, &scratch);
  if (rc != ESA_OK) return rc;
  return esa_scan_fwd(a, v, q, y, E_final, B, T, H, D, mode, E_init, dtype, scratch,
                      ESA_NOALLOC_SCRATCH_BYTES, stream);
}
