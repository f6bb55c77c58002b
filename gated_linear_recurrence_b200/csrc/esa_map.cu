// esa_map.cu -- segment maps of the scan, for context parallelism over time.
//
// Over a segment of time steps the recurrence of every channel is affine in
// the state that enters it, E_end = P E_start + S (P the product of the
// segment's gates, S the end state from a zero start), and so is the
// backward's carry, dE_start = P dE_end + S.  A map-mode scan kernel (the
// persistent scans with MAP = true) leaves the map of every tile of every
// chain in the workspace's agg words, at the tile's first slot; the fold
// kernel below composes a chain's tile maps in time order (latest first for
// the backward) into the map of the whole segment.  The compose kernel
// applies a sequence of segment maps to a state, which is how a time slice
// finds the state (or the gradient) at its boundary from the maps of the
// slices before (after) it.
#include "esa_dispatch.cuh"

namespace esa {

namespace {

// One CTA per chain and CT channels: thread group g of G folds a contiguous
// range of the chain's tiles (in processing order), then group 0 folds the G
// partial maps in order.  Every word must carry the tag of the map-mode call
// that ran just before on the same workspace (the epoch it advanced from);
// a missing word means that call did not finish, which is flagged.
template <int CT, int G>
__global__ void __launch_bounds__(CT *G) esa_map_fold_kernel(const ulonglong2 *__restrict__ agg, WsHeader *hdr,
                                                             ScanShape sh, int sub, int reverse,
                                                             float *__restrict__ P, float *__restrict__ S) {
  __shared__ float2 part[G][CT];
  const int c = threadIdx.x % CT, g = threadIdx.x / CT;
  const int chain = blockIdx.x;
  const unsigned tag = *reinterpret_cast<volatile unsigned *>(&hdr->epoch) - 1u;
  const int per = (sh.nchunks + G - 1) / G;
  const int k0 = min(g * per, sh.nchunks), k1 = min(k0 + per, sh.nchunks);
  const long base = static_cast<long>(chain) * sh.nslots;
  float p = 1.0f, s = 0.0f;
  bool ok = true;
#pragma unroll 8
  for (int k = k0; k < k1; ++k) {
    const int chunk = reverse ? sh.nchunks - 1 - k : k;
    const ulonglong2 w = __ldcg(&agg[(base + static_cast<long>(chunk) * sub) * CT + c]);
    ok = ok && tag_of(w.x) == tag && tag_of(w.y) == tag;
    s = __fmaf_rn(val_of(w.x), s, val_of(w.y));   // x -> P_k (p x + s) + S_k
    p = val_of(w.x) * p;
  }
  part[g][c] = make_float2(p, s);
  if (!ok) atomicOr(&hdr->status, kStatusTimeout);
  __syncthreads();
  if (g == 0) {
    float pp = 1.0f, ss = 0.0f;
#pragma unroll
    for (int j = 0; j < G; ++j) {
      const float2 m = part[j][c];
      ss = __fmaf_rn(m.x, ss, m.y);
      pp = m.x * pp;
    }
    const int cg = (chain % sh.nct) * CT + c;
    if (cg < sh.C) {
      const long at = static_cast<long>(chain / sh.nct) * sh.C + cg;
      P[at] = pp;
      S[at] = ss;
    }
  }
}

// x[i] = map_{n-1}( ... map_0(x0[i]) ) with map_j(x) = P_j x + S_j, maps in
// index order (reverse: from index n - 1 down to 0).
__global__ void __launch_bounds__(256) esa_compose_kernel(const float *__restrict__ P, const float *__restrict__ S,
                                                          int n, long count, int reverse, const float *x0,
                                                          float *x) {
  const long i = static_cast<long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= count) return;
  float e = x0 != nullptr ? x0[i] : 0.0f;
  for (int k = 0; k < n; ++k) {
    const long j = static_cast<long>(reverse ? n - 1 - k : k) * count + i;
    e = __fmaf_rn(P[j], e, S[j]);
  }
  x[i] = e;
}

template <int CT>
int fold(const Workspace &ws, const ScanShape &sh, int sub, int reverse, float *P, float *S,
         cudaStream_t stream) {
  constexpr int G = 1024 / CT;
  esa_map_fold_kernel<CT, G><<<sh.nchains, CT * G, 0, stream>>>(ws.agg, ws.hdr, sh, sub, reverse, P, S);
  return launch_status(cudaGetLastError());
}

}  // namespace

int launch_map_fold(int CT, const Workspace &ws, const ScanShape &sh, int sub, int reverse, float *P, float *S,
                    cudaStream_t stream) {
  if (sh.nchains == 0) return 0;
  switch (CT) {
    case 64: return fold<64>(ws, sh, sub, reverse, P, S, stream);
    case 128: return fold<128>(ws, sh, sub, reverse, P, S, stream);
    case 256: return fold<256>(ws, sh, sub, reverse, P, S, stream);
    default: return -3;
  }
}

int launch_compose(const float *P, const float *S, int n, long count, int reverse, const float *x0, float *x,
                   cudaStream_t stream) {
  if (count == 0) return 0;
  constexpr int kBlock = 256;
  const long blocks = (count + kBlock - 1) / kBlock;
  esa_compose_kernel<<<static_cast<unsigned>(blocks), kBlock, 0, stream>>>(P, S, n, count, reverse, x0, x);
  return launch_status(cudaGetLastError());
}

}  // namespace esa
