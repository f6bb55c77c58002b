// esa_fwd.cu -- instantiations and launcher of the forward scan kernel.
#include "esa_launchers.cuh"

namespace esa {

int launch_fwd(int dtype, int mode, int D, const CUtensorMap &ta, const CUtensorMap &tv,
               const CUtensorMap &tq, const FwdArgs &args, int ntiles, cudaStream_t stream) {
  return dispatch<true>(dtype, mode, D, FwdLauncher<false>{ta, tv, tq, args, ntiles, stream});
}

}  // namespace esa
