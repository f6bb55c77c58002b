// esa_step.cu -- instantiations and launcher of the one-token decode kernel.
#include "esa_dispatch.cuh"

namespace esa {

namespace {
struct StepLauncher {
  const void *a, *v, *q;
  float *E;
  void *y;
  long nvec;
  float inv_D;
  cudaStream_t stream;

  template <typename T, int MODE, int LPH, int VPR, int L, int K>
  int operator()() const {
    constexpr int kBlock = 256;
    const long blocks = (nvec + kBlock - 1) / kBlock;
    esa_step_kernel<T, MODE, LPH><<<static_cast<unsigned>(blocks), kBlock, 0, stream>>>(
        static_cast<const T *>(a), static_cast<const T *>(v), static_cast<const T *>(q), E,
        static_cast<typename OutOf<T>::type *>(y), nvec, inv_D);
    return launch_status(cudaGetLastError());
  }
};
}  // namespace

namespace {
__global__ void esa_ws_init_kernel(WsHeader *hdr) {
  hdr->magic = kWorkspaceMagic;
  hdr->epoch = 1u;
}
}  // namespace

int launch_ws_init(WsHeader *hdr, cudaStream_t stream) {
  esa_ws_init_kernel<<<1, 1, 0, stream>>>(hdr);
  return launch_status(cudaGetLastError());
}

int launch_step(int dtype, int mode, int D, const void *a, const void *v, const void *q, float *E,
                void *y, long nvec, float inv_D, cudaStream_t stream) {
  return dispatch<true>(dtype, mode, D, StepLauncher{a, v, q, E, y, nvec, inv_D, stream});
}

}  // namespace esa
