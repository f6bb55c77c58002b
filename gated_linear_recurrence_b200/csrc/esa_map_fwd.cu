// esa_map_fwd.cu -- instantiations and launcher of the map-mode forward scan
// (tile maps only: reads a and v, writes no output).
#include "esa_launchers.cuh"

namespace esa {

int launch_fwd_map(int dtype, int mode, int D, const CUtensorMap &ta, const CUtensorMap &tv,
                   const CUtensorMap &tq, const FwdArgs &args, int ntiles, cudaStream_t stream) {
  return dispatch<true>(dtype, mode, D, FwdLauncher<true>{ta, tv, tq, args, ntiles, stream});
}

}  // namespace esa
