// esa_bwd.cu -- instantiations and launcher of the backward scan kernel.
#include "esa_launchers.cuh"

namespace esa {

int launch_bwd(int dtype, int mode, int D, const CUtensorMap &ta, const CUtensorMap &tv,
               const CUtensorMap &tq, const CUtensorMap &tdy, const BwdArgs &args, int ntiles,
               cudaStream_t stream) {
  return dispatch<true>(dtype, mode, D, BwdLauncher<false>{ta, tv, tq, tdy, args, ntiles, stream});
}

}  // namespace esa
