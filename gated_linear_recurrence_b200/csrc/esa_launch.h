// esa_launch.h -- host-side launch interface between the C ABI layer and the
// kernel instantiation units.  Internal to the library.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include "esa_kernels.cuh"

namespace esa {

// Rows per workspace slot (the backward's tile height) and channels per tile,
// as chosen for each I/O dtype and head dimension.  The workspace layout and
// the kernels both follow these.
inline int tile_rows(int dtype) { return dtype == 0 ? 32 : 64; }   // f32 : 16- and 8-bit
inline int tile_cols(int D) { return D <= 64 ? 64 : D; }
constexpr int kStepsPerThread = 4;

// Slots per forward tile: 64- and 128-channel tiles of 16-bit (and 8-bit)
// data run the forward two slots (128 rows) tall -- twice the time between
// consecutive chunks of a chain, so a tile's predecessors are further ahead
// when it looks back (128-channel tiles: one 512-thread CTA per SM; the
// forward at D = 128 took 10% less time than with 64-row tiles).
template <typename T, int VPR>
constexpr int fwd_sub() { return (sizeof(T) <= 2 && (VPR == 8 || VPR == 16)) ? 2 : 1; }
inline int fwd_slots_per_tile(int dtype, int D) {
  return (dtype != 0 && (tile_cols(D) == 64 || tile_cols(D) == 128)) ? 2 : 1;
}

// Slots per backward tile: two for 64-channel tiles of 16- and 8-bit data,
// else one.  A backward tile keeps its look-back words at its first slot (the
// end of the tile in processing order) and replays from the checkpoint of the
// slot before it.
template <typename T, int VPR>
constexpr int bwd_sub() { return (sizeof(T) <= 2 && VPR == 8) ? 2 : 1; }
inline int bwd_slots_per_tile(int dtype, int D) { return (dtype != 0 && tile_cols(D) == 64) ? 2 : 1; }

// Launch the forward / backward scan for (dtype, mode, D).  The tensor maps
// describe a, v, q (and dy) as [B][T][C] boxes of [L][CT].  Return 0 or a
// negative esa_status.
int launch_fwd(int dtype, int mode, int D, const CUtensorMap &ta, const CUtensorMap &tv,
               const CUtensorMap &tq, const FwdArgs &args, int ntiles, cudaStream_t stream);
int launch_bwd(int dtype, int mode, int D, const CUtensorMap &ta, const CUtensorMap &tv,
               const CUtensorMap &tq, const CUtensorMap &tdy, const BwdArgs &args, int ntiles,
               cudaStream_t stream);
// Map-mode scans: the same tiles, leaving each tile's (reverse) map in the
// workspace's agg words at the tile's first slot and writing no output.
int launch_fwd_map(int dtype, int mode, int D, const CUtensorMap &ta, const CUtensorMap &tv,
                   const CUtensorMap &tq, const FwdArgs &args, int ntiles, cudaStream_t stream);
int launch_bwd_map(int dtype, int mode, int D, const CUtensorMap &ta, const CUtensorMap &tv,
                   const CUtensorMap &tq, const CUtensorMap &tdy, const BwdArgs &args, int ntiles,
                   cudaStream_t stream);
// Fold the tile maps a map-mode scan just left (tiles of `sub` slots, CT
// channels) into one map per channel: P, S [B][C] float32.  reverse = 1
// composes the latest tile first (the backward's maps).
int launch_map_fold(int CT, const Workspace &ws, const ScanShape &sh, int sub, int reverse, float *P, float *S,
                    cudaStream_t stream);
// x = map_{n-1}(... map_0(x0)), map_j(x) = P[j] x + S[j] over `count` floats.
int launch_compose(const float *P, const float *S, int n, long count, int reverse, const float *x0, float *x,
                   cudaStream_t stream);
// Write the header of a freshly zeroed workspace (magic, epoch 1).
int launch_ws_init(WsHeader *hdr, cudaStream_t stream);
int launch_step(int dtype, int mode, int D, const void *a, const void *v, const void *q, float *E,
                void *y, long nvec, float inv_D, cudaStream_t stream);

}  // namespace esa
