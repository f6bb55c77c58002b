// esa_launchers.cuh -- launchers of the persistent scan kernels, templated on
// the map-only mode so that each mode is instantiated in its own translation
// unit (esa_fwd.cu / esa_bwd.cu: full scans; esa_map.cu: segment maps).
// Internal to the library.
#pragma once

#include "esa_dispatch.cuh"

namespace esa {

template <bool MAP>
struct FwdLauncher {
  const CUtensorMap &ta, &tv, &tq;
  const FwdArgs &args;
  int ntiles;
  cudaStream_t stream;

  template <typename T, int MODE, int LPH, int VPR, int L, int K>
  int operator()() const {
    constexpr int SUB = fwd_sub<T, VPR>();
    constexpr int SW = scan_segments<L * SUB / K, VPR * (L * SUB / K), VPR * 8>();
    using Cfg = TileCfg<T, LPH, VPR, L * SUB, K, SW>;
    // The host sized the tile grid with the same slots-per-tile rule.
    if (args.s.nchunks != (args.s.nslots + SUB - 1) / SUB) return -5;
    const size_t smem = FwdSmem<Cfg>::kBytes;
    auto kern = esa_scan_fwd_kernel<T, MODE, LPH, VPR, L * SUB, K, SUB, SW, MAP>;
    int grid = 0;
    const int rc = persistent_grid(kern, Cfg::NT, smem, ntiles, &grid);
    if (rc) return rc;
    kern<<<grid, Cfg::NT, smem, stream>>>(ta, tv, tq, args);
    return launch_status(cudaGetLastError());
  }
};

template <bool MAP>
struct BwdLauncher {
  const CUtensorMap &ta, &tv, &tq, &tdy;
  const BwdArgs &args;
  int ntiles;
  cudaStream_t stream;

  template <typename T, int MODE, int LPH, int VPR, int L, int K>
  int operator()() const {
    constexpr int SUB = bwd_sub<T, VPR>();
    constexpr int SW = scan_segments<L * SUB / K, VPR * (L * SUB / K), VPR * 8>();
    using Cfg = TileCfg<T, LPH, VPR, L * SUB, K, SW>;
    // The host sized the tile grid with the same slots-per-tile rule.
    if (args.s.nchunks != (args.s.nslots + SUB - 1) / SUB) return -5;
    const size_t smem = BwdSmem<Cfg>::kBytes;
    auto kern = esa_scan_bwd_kernel<T, MODE, LPH, VPR, L * SUB, K, SW, SUB, MAP>;
    int grid = 0;
    const int rc = persistent_grid(kern, Cfg::NT, smem, ntiles, &grid);
    if (rc) return rc;
    kern<<<grid, Cfg::NT, smem, stream>>>(ta, tv, tq, tdy, args);
    return launch_status(cudaGetLastError());
  }
};

}  // namespace esa
