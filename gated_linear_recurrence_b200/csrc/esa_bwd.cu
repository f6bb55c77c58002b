// esa_bwd.cu -- instantiations and launcher of the backward scan kernel.
#include "esa_dispatch.cuh"

namespace esa {

namespace {
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
    auto kern = esa_scan_bwd_kernel<T, MODE, LPH, VPR, L * SUB, K, SW, SUB>;
    int grid = 0;
    const int rc = persistent_grid(kern, Cfg::NT, smem, ntiles, &grid);
    if (rc) return rc;
    kern<<<grid, Cfg::NT, smem, stream>>>(ta, tv, tq, tdy, args);
    return launch_status(cudaGetLastError());
  }
};
}  // namespace

int launch_bwd(int dtype, int mode, int D, const CUtensorMap &ta, const CUtensorMap &tv,
               const CUtensorMap &tq, const CUtensorMap &tdy, const BwdArgs &args, int ntiles,
               cudaStream_t stream) {
  return dispatch(dtype, mode, D, BwdLauncher{ta, tv, tq, tdy, args, ntiles, stream});
}

}  // namespace esa
