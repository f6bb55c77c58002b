// esa_fused.cu -- instantiations and launcher of the fused projection + scan
// forward kernel (16-bit I/O, head dimension <= 64, C_in of 64, 128 or 256),
// and of its variant with the output projection (C = 64, C_in of 64 or 128).
#include "esa_dispatch.cuh"
#include "esa_fused.cuh"
#include "esa_fused_launch.h"

namespace esa {

namespace {

template <typename T, int MODE, int LPH, int CIN, bool WO>
int run_fused(const CUtensorMap &tx, const CUtensorMap &tw, const CUtensorMap *tavq, const CUtensorMap &two,
              const FusedArgs &args, cudaStream_t stream) {
  using Pl = FusedPlan<T, CIN, WO>;
  auto kern = esa_fused_fwd_kernel<T, MODE, LPH, CIN, WO>;
  const size_t smem = Pl::kBytes;
  int dev = 0, sms = 0, per_sm = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -5;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) != cudaSuccess)
    return -5;
  constexpr int kThreads = Pl::NG * Pl::NTG;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreads, smem) != cudaSuccess) return -5;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return -5;
  if (per_sm < 1 || sms < 1) return -5;
  // Every CTA must be resident at once (tiles wait on their predecessors):
  // at most one CTA per SM in total, split evenly over the channel tiles.
  const int nct = args.s.nct;
  int per_ct = (sms * per_sm) / nct;
  const int need = (args.ntiles_ct + Pl::NG - 1) / Pl::NG;
  if (per_ct > need) per_ct = need;
  if (per_ct < 1) return -5;
  kern<<<dim3(per_ct, nct), kThreads, smem, stream>>>(tx, tw, tavq[0], tavq[1], tavq[2], two, args);
  return launch_status(cudaGetLastError());
}

template <typename T, int MODE, int LPH>
int by_cin(int cin, bool wo, const CUtensorMap &tx, const CUtensorMap &tw, const CUtensorMap *tavq,
           const CUtensorMap &two, const FusedArgs &args, cudaStream_t st) {
  if (wo) {
    switch (cin) {
      case 64: return run_fused<T, MODE, LPH, 64, true>(tx, tw, tavq, two, args, st);
      case 128: return run_fused<T, MODE, LPH, 128, true>(tx, tw, tavq, two, args, st);
      default: return -3;
    }
  }
  switch (cin) {
    case 64: return run_fused<T, MODE, LPH, 64, false>(tx, tw, tavq, two, args, st);
    case 128: return run_fused<T, MODE, LPH, 128, false>(tx, tw, tavq, two, args, st);
    case 256: return run_fused<T, MODE, LPH, 256, false>(tx, tw, tavq, two, args, st);
    default: return -3;
  }
}

template <typename T, int MODE>
int by_d(int D, int cin, bool wo, const CUtensorMap &tx, const CUtensorMap &tw, const CUtensorMap *tavq,
         const CUtensorMap &two, const FusedArgs &args, cudaStream_t st) {
  switch (D) {
    case 8: return by_cin<T, MODE, 1>(cin, wo, tx, tw, tavq, two, args, st);
    case 16: return by_cin<T, MODE, 2>(cin, wo, tx, tw, tavq, two, args, st);
    case 32: return by_cin<T, MODE, 4>(cin, wo, tx, tw, tavq, two, args, st);
    case 64: return by_cin<T, MODE, 8>(cin, wo, tx, tw, tavq, two, args, st);
    default: return -3;
  }
}

}  // namespace

int launch_fused_fwd(int dtype, int mode, int D, int cin, const CUtensorMap &tx, const CUtensorMap &tw,
                     const CUtensorMap *tavq, const CUtensorMap *two, const FusedArgs &args, cudaStream_t stream) {
  if (mode != 0 && mode != 1) return -1;
  const bool wo = two != nullptr;
  const CUtensorMap &wmap = wo ? *two : tx;   // placeholder when there is no output projection
  switch (dtype) {
    case 1:
      return mode ? by_d<__half, 1>(D, cin, wo, tx, tw, tavq, wmap, args, stream)
                  : by_d<__half, 0>(D, cin, wo, tx, tw, tavq, wmap, args, stream);
    case 2:
      return mode ? by_d<__nv_bfloat16, 1>(D, cin, wo, tx, tw, tavq, wmap, args, stream)
                  : by_d<__nv_bfloat16, 0>(D, cin, wo, tx, tw, tavq, wmap, args, stream);
    default: return -3;
  }
}

}  // namespace esa
