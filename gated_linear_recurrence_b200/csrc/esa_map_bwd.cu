// esa_map_bwd.cu -- instantiations and launcher of the map-mode backward scan
// (reverse tile maps only: writes no gradient).
#include "esa_launchers.cuh"

namespace esa {

int launch_bwd_map(int dtype, int mode, int D, const CUtensorMap &ta, const CUtensorMap &tv,
                   const CUtensorMap &tq, const CUtensorMap &tdy, const BwdArgs &args, int ntiles,
                   cudaStream_t stream) {
  return dispatch<true>(dtype, mode, D, BwdLauncher<true>{ta, tv, tq, tdy, args, ntiles, stream});
}

}  // namespace esa
