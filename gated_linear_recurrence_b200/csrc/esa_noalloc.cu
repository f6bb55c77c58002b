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
//
// Every call first runs a one-block guard kernel on the caller's stream.  It
// reads the array's header and, when the header is not initialised (the
// first call on a device) or the 32-bit call epoch is close to running out,
// clears the array and writes a fresh header.  So the array needs no
// host-side initialisation and no synchronisation, and it never reaches the
// end of its epoch range (where the scans would stop doing work).
#include <cuda_runtime.h>

#include <mutex>

#include "esa.h"
#include "esa_common.cuh"

namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[ESA_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
void *g_scratch_ptr[kMaxDevices] = {};

// Epoch from which the guard starts the array afresh.  A call advances the
// epoch by one and is always preceded by its own guard, so the epoch never
// gets past this value by more than one.
constexpr unsigned kEpochRestart = 0xFFFFFF00u;
constexpr int kGuardThreads = 1024;

// Device code may name the array directly (host code may not: there its name
// is only a host-side stand-in for the symbol).
__global__ void __launch_bounds__(kGuardThreads) esa_noalloc_guard_kernel() {
  __shared__ int restart;
  __shared__ unsigned keep;
  esa::WsHeader *hdr = reinterpret_cast<esa::WsHeader *>(g_noalloc_scratch);
  if (threadIdx.x == 0) {
    const bool ok = hdr->magic == esa::kWorkspaceMagic && hdr->epoch != 0u && hdr->epoch < kEpochRestart;
    restart = ok ? 0 : 1;
    keep = hdr->status & esa::kStatusTimeout;   // a timeout not yet read by esa_check_noalloc
  }
  __syncthreads();
  if (!restart) return;
  uint4 *p = reinterpret_cast<uint4 *>(g_noalloc_scratch);
  constexpr size_t n = ESA_NOALLOC_SCRATCH_BYTES / sizeof(uint4);
  for (size_t i = threadIdx.x; i < n; i += kGuardThreads) p[i] = make_uint4(0u, 0u, 0u, 0u);
  __syncthreads();
  if (threadIdx.x == 0) {
    hdr->status = keep;
    hdr->epoch = 1u;
    hdr->magic = esa::kWorkspaceMagic;
  }
}

// Device address of the array on the current device (looked up once per
// device, with that device current, under a lock).
int scratch_address(void **out) {
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
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return ESA_OK;
}

// The host-side argument checks of the forward scan that can fail, done here
// too so that a rejected call enqueues nothing (not even the guard).
int check_args(const void *a, const void *v, const void *q, const void *y, const float *E_final, int B, int T,
               int mode, const float *E_init) {
  if (mode != ESA_DIRECT && mode != ESA_CONTROLLED) return ESA_ERR_ARG;
  if (B > 0 && T > 0 && (!a || !v || !q || !y)) return ESA_ERR_ARG;
  for (const void *p : {a, v, q, y, static_cast<const void *>(E_final), static_cast<const void *>(E_init)})
    if (p && (reinterpret_cast<uintptr_t>(p) & 15u) != 0) return ESA_ERR_ALIGN;
  int dev = -1, major = 0, minor = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) {
    cudaGetLastError();
    return ESA_ERR_DEVICE;
  }
  return (major == 10 && minor == 0) ? ESA_OK : ESA_ERR_DEVICE;
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
  int rc = check_args(a, v, q, y, E_final, B, T, mode, E_init);
  if (rc != ESA_OK) return rc;
  void *scratch = nullptr;
  if ((rc = scratch_address(&scratch)) != ESA_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  esa_noalloc_guard_kernel<<<1, kGuardThreads, 0, st>>>();
  if (cudaGetLastError() != cudaSuccess) return ESA_ERR_LAUNCH;
  return esa_scan_fwd(a, v, q, y, E_final, B, T, H, D, mode, E_init, dtype, scratch, ESA_NOALLOC_SCRATCH_BYTES,
                      stream);
}

extern "C" int esa_check_noalloc(void *stream) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return ESA_ERR_DEVICE;
  }
  void *scratch = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    scratch = g_scratch_ptr[dev];
  }
  if (scratch == nullptr) {   // no call has used the array on this device
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) {
      cudaGetLastError();
      return ESA_ERR_LAUNCH;
    }
    return ESA_OK;
  }
  return esa_check(scratch, stream);
}

extern "C" int esa_noalloc_scratch(void **device_ptr, size_t *bytes) {
  if (!device_ptr) return ESA_ERR_ARG;
  const int rc = scratch_address(device_ptr);
  if (rc == ESA_OK && bytes) *bytes = ESA_NOALLOC_SCRATCH_BYTES;
  return rc;
}
