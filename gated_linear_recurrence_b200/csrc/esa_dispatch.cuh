// esa_dispatch.cuh -- maps runtime (dtype, mode, D) onto kernel template
// instantiations.  Internal to the library.
#pragma once

#include "esa_launch.h"

namespace esa {

// Calls f.template operator()<T, MODE, LPH, VPR, L, K>() for the runtime
// (dtype, mode, D); returns ESA_ERR_UNSUPPORTED (-3) for an unknown D.
template <typename T, int MODE, typename F>
int dispatch_d(int D, F &&f) {
  constexpr int L = sizeof(T) == 4 ? 32 : 64;
  constexpr int K = kStepsPerThread;
  switch (D) {
    case 8: return f.template operator()<T, MODE, 1, 8, L, K>();
    case 16: return f.template operator()<T, MODE, 2, 8, L, K>();
    case 32: return f.template operator()<T, MODE, 4, 8, L, K>();
    case 64: return f.template operator()<T, MODE, 8, 8, L, K>();
    case 128: return f.template operator()<T, MODE, 16, 16, L, K>();
    case 256: return f.template operator()<T, MODE, 32, 32, L, K>();
    default: return -3;
  }
}

// kFp8: also dispatch fp8 (e4m3) inputs, dtype 3 (forward scans only; the
// other kernels return ESA_ERR_UNSUPPORTED for it).
template <bool kFp8 = false, typename F>
int dispatch(int dtype, int mode, int D, F &&f) {
  if (mode != 0 && mode != 1) return -1;
  switch (dtype) {
    case 0: return mode ? dispatch_d<float, 1>(D, f) : dispatch_d<float, 0>(D, f);
    case 1: return mode ? dispatch_d<__half, 1>(D, f) : dispatch_d<__half, 0>(D, f);
    case 2: return mode ? dispatch_d<__nv_bfloat16, 1>(D, f) : dispatch_d<__nv_bfloat16, 0>(D, f);
    case 3:
      if constexpr (kFp8) return mode ? dispatch_d<__nv_fp8_e4m3, 1>(D, f) : dispatch_d<__nv_fp8_e4m3, 0>(D, f);
      else return -3;
    default: return -1;
  }
}

inline int launch_status(cudaError_t e) { return e == cudaSuccess ? 0 : -5; }

// Grid of a persistent scan kernel: as many CTAs as can be resident at once
// (occupancy x SM count), never more than there are tiles.
template <typename Kern>
int persistent_grid(Kern kern, int nthreads, size_t smem, int ntiles, int *grid) {
  int dev = 0, sms = 0, per_sm = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -5;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) !=
      cudaSuccess)
    return -5;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, nthreads, smem) != cudaSuccess) return -5;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return -5;
  if (per_sm < 1 || sms < 1) return -5;
  const long long g = static_cast<long long>(per_sm) * sms;
  *grid = static_cast<int>(g < ntiles ? g : ntiles);
  return 0;
}

}  // namespace esa
