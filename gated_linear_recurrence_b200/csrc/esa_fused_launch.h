// esa_fused_launch.h -- host-side launch interface of the fused projection +
// scan forward.  Internal to the library.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include "esa_fused.cuh"

namespace esa {

// Shapes the fused kernel takes: 16-bit I/O, channel tiles of 64 (head
// dimension <= 64), C_in of 64, 128 or 256, at most kMaxChannelTickets channel tiles.
inline bool fused_supported(int dtype, int D, int cin, int nct) {
  return (dtype == 1 || dtype == 2) && D <= 64 && (cin == 64 || cin == 128 || cin == 256) &&
         nct <= kMaxChannelTickets;
}

// Shapes the fused kernel with the output projection takes: one channel tile
// holding the whole row (C = 64), C_in of 64 or 128.
inline bool fused_out_supported(int dtype, int C, int cin) {
  return (dtype == 1 || dtype == 2) && C == 64 && (cin == 64 || cin == 128);
}

// tx: x [B][T][C_in] in boxes of [128 rows][64 elements], 128-byte swizzle;
// tw: W [3 C][C_in] in boxes of [64 rows][64 elements], 128-byte swizzle;
// tavq[3]: a, v, q [B][T][C] in boxes of [128 rows][64 channels], 128-byte
// swizzle (used only when args.a_out is set);
// two: W_O [64][64] in one box of [64 rows][64 elements], 128-byte swizzle,
// or null: with it the kernel also writes z = y W_O^T to args.z.
int launch_fused_fwd(int dtype, int mode, int D, int cin, const CUtensorMap &tx, const CUtensorMap &tw,
                     const CUtensorMap *tavq, const CUtensorMap *two, const FusedArgs &args, cudaStream_t stream);

}  // namespace esa
