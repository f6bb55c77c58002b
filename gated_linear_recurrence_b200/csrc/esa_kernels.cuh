// esa_kernels.cuh -- forward scan, backward scan and decode-step kernels of
// the ESA gated linear recurrence for sm_100a.
//
// Work decomposition (forward and backward):
//   * A "chain" is one batch row b and one tile of CT consecutive channels
//     (CT = 128, or 256 when the head dimension is 256).  Heads never straddle
//     a channel tile, so the per-head RMS readout stays inside one CTA.
//   * A chain is cut into time chunks of L steps.  One CTA processes one
//     (chain, chunk) tile; the tile's a/v/q(/dy) boxes [L x CT] are staged in
//     shared memory by TMA tensor loads (cp.async.bulk.tensor, no multicast).
//   * Inside a tile every thread owns 8 consecutive channels (one 16-byte
//     vector for 16-bit I/O) and a run of K consecutive time steps.  Pass 1
//     folds its run into an affine map x -> P x + S per channel; the runs of a
//     tile are combined by a short serial scan per channel in shared memory;
//     the tile map is then chained to earlier tiles by a single-pass
//     decoupled look-back over per-chunk flags in the workspace.  Pass 2
//     replays the run from its exact carry-in and emits the readout.
//   * The carry is always applied in chunk order, oldest first, with the same
//     fused multiply-add that the producing tile used for its own inclusive
//     state, so the result is bitwise independent of how far a look-back
//     reached: outputs are deterministic run to run.
//   * Tiles are numbered by an atomic ticket (not blockIdx) with the chain as
//     the fast index, so a tile's predecessor is always a tile whose CTA is
//     already running; every wait is bounded.
//   * The forward stores the state at every chunk end (fstate); the backward
//     replays each chunk from that checkpoint, so nothing of size T x C is
//     stored besides the outputs.
#pragma once

#include "esa_common.cuh"

namespace esa {

struct ScanShape {
  int B, T, C;          // C = H * D
  int nchunks;          // ceil(T / L)
  int nct;              // channel tiles per batch row
  int nchains;          // B * nct
  float inv_D;
};

struct FwdArgs {
  ScanShape s;
  void *y;
  float *E_final;
  const float *E_init;
  Workspace ws;
};

struct BwdArgs {
  ScanShape s;
  void *da, *dv, *dq;
  const float *dE_final;
  float *dE_init;
  const float *E_init;
  Workspace ws;
};

// Compile-time tile geometry.
template <typename T, int LPH_, int VPR_, int L_, int K_>
struct TileCfg {
  static constexpr int LPH = LPH_;                 // lanes per head = D / 8
  static constexpr int VPR = VPR_;                 // 8-channel vectors per tile row
  static constexpr int CT = VPR * 8;               // channels per tile
  static constexpr int L = L_;                     // time steps per tile
  static constexpr int K = K_;                     // time steps per thread
  static constexpr int RUNS = L / K;               // runs per vector column
  static constexpr int NT = VPR * RUNS;            // threads per CTA
  static constexpr int VW0 = LPH > 8 ? LPH : 8;
  static constexpr int VW = VW0 < VPR ? VW0 : VPR; // vectors per warp row segment
  static constexpr int RW = 32 / VW;               // runs per warp
  static constexpr int NVSEG = VPR / VW;
  static constexpr unsigned kBoxBytes = L * CT * sizeof(T);
  static_assert(L % K == 0, "K must divide L");
  static_assert(NT % 32 == 0 && NT <= 1024, "bad block size");
  static_assert(RUNS % RW == 0, "runs must fill warps");
  static_assert(CT % 32 == 0 && NT >= CT, "look-back needs CT threads");
  static_assert(RUNS * CT * sizeof(float2) <= kBoxBytes, "scan scratch must fit in the gate box");
  static_assert(VW % LPH == 0, "a head must stay inside a warp");
};

template <typename Cfg, int NBOX>
constexpr size_t scan_smem_bytes() {
  // NBOX boxes + CT floats + mbarrier + ticket, plus 128 B for alignment.
  return size_t(NBOX) * Cfg::kBoxBytes + Cfg::CT * sizeof(float) + 16 + 128;
}

__device__ __forceinline__ unsigned char *align128(unsigned char *p) {
  return reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(p) + 127) & ~uintptr_t(127));
}

// Per-thread coordinates inside a tile.
template <typename Cfg>
struct ThreadPos {
  int vec, run, ch, row0;
  __device__ __forceinline__ ThreadPos(int tid) {
    const int warp = tid >> 5, lane = tid & 31;
    const int vseg = warp % Cfg::NVSEG, rgrp = warp / Cfg::NVSEG;
    vec = vseg * Cfg::VW + lane % Cfg::VW;
    run = rgrp * Cfg::RW + lane / Cfg::VW;
    ch = vec * 8;
    row0 = run * Cfg::K;
  }
};

// Decoupled look-back for one channel (called by the first CT threads).
// `slot` is this tile; its predecessors in processing order are
// slot + dir, slot + 2 dir, ...  (dir = -1 forward in time, +1 backward).
// Returns the carry entering this tile.  The walk stops at the nearest
// predecessor whose inclusive carry is published, then applies the
// aggregates of the tiles in between oldest first.
__device__ __forceinline__ float lookback(const unsigned *flags, const float2 *agg, const float *state,
                                          long slot, int dir, int CT, int c, unsigned *abort_flag,
                                          unsigned *status) {
  long j = slot + dir;
  for (;;) {
    const unsigned f = wait_flag_bounded(&flags[j], abort_flag, status);
    if (f == kFlagIncl) break;
    if (f == 0) return 0.0f;  // gave up; status already records the timeout
    j += dir;
  }
  float E = __ldcg(&state[j * CT + c]);
  for (long m = j - dir; m != slot; m -= dir) {
    const float2 e = __ldcg(&agg[m * CT + c]);
    E = __fmaf_rn(e.x, E, e.y);
  }
  return E;
}

// ===========================================================================
// Forward scan.
// ===========================================================================
template <typename T, int MODE, int LPH, int VPR, int L, int K>
__global__ void __launch_bounds__(VPR *(L / K))
    esa_scan_fwd_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_v,
                        const __grid_constant__ CUtensorMap tm_q, const FwdArgs args) {
  using Cfg = TileCfg<T, LPH, VPR, L, K>;
  constexpr int CT = Cfg::CT, RUNS = Cfg::RUNS;

  extern __shared__ unsigned char smem_raw[];
  unsigned char *base = align128(smem_raw);
  T *a_s = reinterpret_cast<T *>(base);
  T *v_s = a_s + L * CT;
  T *q_s = v_s + L * CT;
  float *es_s = reinterpret_cast<float *>(q_s + L * CT);
  uint64_t *bar = reinterpret_cast<uint64_t *>(es_s + CT);
  int *ticket_s = reinterpret_cast<int *>(bar + 1);
  float2 *scan_s = reinterpret_cast<float2 *>(a_s);  // reused once pass 1 is done

  const int tid = threadIdx.x;
  const ScanShape &sh = args.s;
  const Workspace &ws = args.ws;

  if (tid == 0) {
    prefetch_tensormap(&tm_a);
    prefetch_tensormap(&tm_v);
    prefetch_tensormap(&tm_q);
    mbar_init(bar, 1);
    fence_mbar_init();
    fence_proxy_async_smem();
    *ticket_s = static_cast<int>(atomicAdd(&ws.fwd_hdr[1], 1u));
  }
  __syncthreads();
  const int tile = *ticket_s;
  const int chain = tile % sh.nchains;
  const int chunk = tile / sh.nchains;
  const int b = chain / sh.nct;
  const int c0 = (chain % sh.nct) * CT;
  const int t0 = chunk * L;
  const long slot = static_cast<long>(chain) * sh.nchunks + chunk;

  if (tid == 0) {
    mbar_expect_tx(bar, 3 * Cfg::kBoxBytes);
    tma_load_3d(a_s, &tm_a, c0, t0, b, bar);
    tma_load_3d(v_s, &tm_v, c0, t0, b, bar);
    tma_load_3d(q_s, &tm_q, c0, t0, b, bar);
  }

  const ThreadPos<Cfg> pos(tid);
  mbar_wait_bounded(bar, 0, ws.status);

  // ---- pass 1: gates and the run's affine map -----------------------------
  float Ar[K][8];   // direct: A_t; controlled: 1 - A_t
  float P[8], S[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) { P[j] = 1.0f; S[j] = 0.0f; }
#pragma unroll
  for (int i = 0; i < K; ++i) {
    const int r = pos.row0 + i;
    const bool valid = (t0 + r) < sh.T;
    float x[8], vv[8];
    Io<T>::load8(a_s + r * CT + pos.ch, x);
    Io<T>::load8(v_s + r * CT + pos.ch, vv);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const Gate g = gate_of(x[j]);
      if (MODE == 0) {
        Ar[i][j] = g.A;
        if (valid) { P[j] *= g.A; S[j] = __fmaf_rn(g.A, S[j], vv[j]); }
      } else {
        Ar[i][j] = g.Ac;
        if (valid) { P[j] *= g.A; S[j] = __fmaf_rn(g.Ac, vv[j] - S[j], S[j]); }
      }
    }
  }
  __syncthreads();  // the gate box is free from here on
#pragma unroll
  for (int j = 0; j < 8; ++j) scan_s[pos.run * CT + pos.ch + j] = make_float2(P[j], S[j]);
  __syncthreads();

  // ---- scan over runs, look-back, publish --------------------------------
  if (tid < CT) {
    float cp = 1.0f, cs = 0.0f;
#pragma unroll 4
    for (int r = 0; r < RUNS; ++r) {
      const float2 e = scan_s[r * CT + tid];
      scan_s[r * CT + tid] = make_float2(cp, cs);   // exclusive prefix of the runs
      cs = __fmaf_rn(e.x, cs, e.y);
      cp = cp * e.x;
    }
    const int cg = c0 + tid;
    float E_start;
    if (chunk == 0) {
      E_start = (args.E_init != nullptr && cg < sh.C) ? args.E_init[static_cast<long>(b) * sh.C + cg] : 0.0f;
    } else {
      ws.agg[slot * CT + tid] = make_float2(cp, cs);
      __threadfence();
      bar_sync_first(CT);
      if (tid == 0) st_release(&ws.fwd_flags[slot], kFlagAgg);
      E_start = lookback(ws.fwd_flags, ws.agg, ws.fstate, slot, -1, CT, tid, &ws.fwd_hdr[2], ws.status);
    }
    const float E_end = __fmaf_rn(cp, E_start, cs);
    ws.fstate[slot * CT + tid] = E_end;
    __threadfence();
    bar_sync_first(CT);
    if (tid == 0) st_release(&ws.fwd_flags[slot], kFlagIncl);
    if (chunk == sh.nchunks - 1 && args.E_final != nullptr && cg < sh.C)
      args.E_final[static_cast<long>(b) * sh.C + cg] = E_end;
    es_s[tid] = E_start;
  }
  __syncthreads();

  // ---- pass 2: exact states and the readout ------------------------------
  float E[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const float2 pe = scan_s[pos.run * CT + pos.ch + j];
    E[j] = __fmaf_rn(pe.x, es_s[pos.ch + j], pe.y);
  }
  T *yg = static_cast<T *>(args.y);
  const bool ch_ok = (c0 + pos.ch) < sh.C;
  const long gbase = (static_cast<long>(b) * sh.T + t0) * sh.C + c0 + pos.ch;
#pragma unroll
  for (int i = 0; i < K; ++i) {
    const int r = pos.row0 + i;
    const bool valid = (t0 + r) < sh.T;
    float vv[8], qq[8];
    Io<T>::load8(v_s + r * CT + pos.ch, vv);
    Io<T>::load8(q_s + r * CT + pos.ch, qq);
    float ss = 0.0f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      E[j] = (MODE == 0) ? __fmaf_rn(Ar[i][j], E[j], vv[j]) : __fmaf_rn(Ar[i][j], vv[j] - E[j], E[j]);
      ss = __fmaf_rn(E[j], E[j], ss);
    }
    ss = head_sum<LPH>(ss);
    const float rr = rsqrtf(__fmaf_rn(ss, sh.inv_D, kEps));
    float yv[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) yv[j] = qq[j] * (E[j] * rr);
    if (valid && ch_ok) Io<T>::store8(yg + gbase + static_cast<long>(r) * sh.C, yv);
  }
}

// ===========================================================================
// Backward scan.
// ===========================================================================
template <typename T>
__device__ __forceinline__ void put_ghat(T *q_slot, T *dy_slot, const float (&g)[8]) {
  if (sizeof(T) == 2) {
    reinterpret_cast<float4 *>(q_slot)[0] = make_float4(g[0], g[1], g[2], g[3]);
    reinterpret_cast<float4 *>(dy_slot)[0] = make_float4(g[4], g[5], g[6], g[7]);
  } else {
    reinterpret_cast<float4 *>(q_slot)[0] = make_float4(g[0], g[1], g[2], g[3]);
    reinterpret_cast<float4 *>(q_slot)[1] = make_float4(g[4], g[5], g[6], g[7]);
  }
}

template <typename T>
__device__ __forceinline__ void get_ghat(const T *q_slot, const T *dy_slot, float (&g)[8]) {
  float4 u, w;
  if (sizeof(T) == 2) {
    u = reinterpret_cast<const float4 *>(q_slot)[0];
    w = reinterpret_cast<const float4 *>(dy_slot)[0];
  } else {
    u = reinterpret_cast<const float4 *>(q_slot)[0];
    w = reinterpret_cast<const float4 *>(q_slot)[1];
  }
  g[0] = u.x; g[1] = u.y; g[2] = u.z; g[3] = u.w;
  g[4] = w.x; g[5] = w.y; g[6] = w.z; g[7] = w.w;
}

template <typename T, int MODE, int LPH, int VPR, int L, int K>
__global__ void __launch_bounds__(VPR *(L / K))
    esa_scan_bwd_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_v,
                        const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_dy,
                        const BwdArgs args) {
  using Cfg = TileCfg<T, LPH, VPR, L, K>;
  constexpr int CT = Cfg::CT, RUNS = Cfg::RUNS;

  extern __shared__ unsigned char smem_raw[];
  unsigned char *base = align128(smem_raw);
  T *a_s = reinterpret_cast<T *>(base);
  T *v_s = a_s + L * CT;
  T *q_s = v_s + L * CT;
  T *dy_s = q_s + L * CT;
  float *es_s = reinterpret_cast<float *>(dy_s + L * CT);
  uint64_t *bar = reinterpret_cast<uint64_t *>(es_s + CT);
  int *ticket_s = reinterpret_cast<int *>(bar + 1);
  float2 *scan_s = reinterpret_cast<float2 *>(a_s);

  const int tid = threadIdx.x;
  const ScanShape &sh = args.s;
  const Workspace &ws = args.ws;

  if (tid == 0) {
    prefetch_tensormap(&tm_a);
    prefetch_tensormap(&tm_v);
    prefetch_tensormap(&tm_q);
    prefetch_tensormap(&tm_dy);
    mbar_init(bar, 1);
    fence_mbar_init();
    fence_proxy_async_smem();
    *ticket_s = static_cast<int>(atomicAdd(&ws.bwd_hdr[1], 1u));
  }
  __syncthreads();
  const int tile = *ticket_s;
  const int chain = tile % sh.nchains;
  const int chunk = sh.nchunks - 1 - tile / sh.nchains;   // latest chunk first
  const int b = chain / sh.nct;
  const int c0 = (chain % sh.nct) * CT;
  const int t0 = chunk * L;
  const long slot = static_cast<long>(chain) * sh.nchunks + chunk;

  if (tid == 0) {
    mbar_expect_tx(bar, 4 * Cfg::kBoxBytes);
    tma_load_3d(a_s, &tm_a, c0, t0, b, bar);
    tma_load_3d(v_s, &tm_v, c0, t0, b, bar);
    tma_load_3d(q_s, &tm_q, c0, t0, b, bar);
    tma_load_3d(dy_s, &tm_dy, c0, t0, b, bar);
  }
  if (tid < CT) {   // forward state entering the chunk (checkpoint)
    const int cg = c0 + tid;
    es_s[tid] = (chunk == 0)
                    ? ((args.E_init != nullptr && cg < sh.C) ? args.E_init[static_cast<long>(b) * sh.C + cg] : 0.0f)
                    : __ldcg(&ws.fstate[(slot - 1) * CT + tid]);
  }

  const ThreadPos<Cfg> pos(tid);
  mbar_wait_bounded(bar, 0, ws.status);

  // ---- F1: gates and the run's forward map --------------------------------
  float Ar[K][8];
  float P[8], S[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) { P[j] = 1.0f; S[j] = 0.0f; }
#pragma unroll
  for (int i = 0; i < K; ++i) {
    const int r = pos.row0 + i;
    const bool valid = (t0 + r) < sh.T;
    float x[8], vv[8];
    Io<T>::load8(a_s + r * CT + pos.ch, x);
    Io<T>::load8(v_s + r * CT + pos.ch, vv);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const Gate g = gate_of(x[j]);
      if (MODE == 0) {
        Ar[i][j] = g.A;
        if (valid) { P[j] *= g.A; S[j] = __fmaf_rn(g.A, S[j], vv[j]); }
      } else {
        Ar[i][j] = g.Ac;
        if (valid) { P[j] *= g.A; S[j] = __fmaf_rn(g.Ac, vv[j] - S[j], S[j]); }
      }
    }
  }
  __syncthreads();
#pragma unroll
  for (int j = 0; j < 8; ++j) scan_s[pos.run * CT + pos.ch + j] = make_float2(P[j], S[j]);
  __syncthreads();
  if (tid < CT) {
    float cp = 1.0f, cs = 0.0f;
#pragma unroll 4
    for (int r = 0; r < RUNS; ++r) {
      const float2 e = scan_s[r * CT + tid];
      scan_s[r * CT + tid] = make_float2(cp, cs);
      cs = __fmaf_rn(e.x, cs, e.y);
      cp = cp * e.x;
    }
  }
  __syncthreads();

  // ---- F2: replay states, readout backward, dq, ghat ----------------------
  float E[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const float2 pe = scan_s[pos.run * CT + pos.ch + j];
    E[j] = __fmaf_rn(pe.x, es_s[pos.ch + j], pe.y);
  }
  float Ep[K][8];   // E_{t-1} of every row of the run
  const bool ch_ok = (c0 + pos.ch) < sh.C;
  const long gbase = (static_cast<long>(b) * sh.T + t0) * sh.C + c0 + pos.ch;
  T *dqg = static_cast<T *>(args.dq);
#pragma unroll
  for (int i = 0; i < K; ++i) {
    const int r = pos.row0 + i;
    const bool valid = (t0 + r) < sh.T;
    float vv[8], qq[8], gg[8];
    Io<T>::load8(v_s + r * CT + pos.ch, vv);
    Io<T>::load8(q_s + r * CT + pos.ch, qq);
    Io<T>::load8(dy_s + r * CT + pos.ch, gg);
    float ss = 0.0f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      Ep[i][j] = E[j];
      E[j] = (MODE == 0) ? __fmaf_rn(Ar[i][j], E[j], vv[j]) : __fmaf_rn(Ar[i][j], vv[j] - E[j], E[j]);
      ss = __fmaf_rn(E[j], E[j], ss);
    }
    ss = head_sum<LPH>(ss);
    const float rr = rsqrtf(__fmaf_rn(ss, sh.inv_D, kEps));
    float nn[8], dn[8], dqv[8];
    float dot = 0.0f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      nn[j] = E[j] * rr;
      dn[j] = gg[j] * qq[j];
      dqv[j] = gg[j] * nn[j];
      dot = __fmaf_rn(dn[j], nn[j], dot);
    }
    dot = head_sum<LPH>(dot) * sh.inv_D;
    float gh[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) gh[j] = rr * __fmaf_rn(-nn[j], dot, dn[j]);
    put_ghat<T>(q_s + r * CT + pos.ch, dy_s + r * CT + pos.ch, gh);
    if (valid && ch_ok) Io<T>::store8(dqg + gbase + static_cast<long>(r) * sh.C, dqv);
  }

  // ---- R1: the run's reverse map h -> P h + hl ---------------------------
  float hl[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) hl[j] = 0.0f;
#pragma unroll
  for (int i = K - 1; i >= 0; --i) {
    const int r = pos.row0 + i;
    if ((t0 + r) < sh.T) {
      float gh[8];
      get_ghat<T>(q_s + r * CT + pos.ch, dy_s + r * CT + pos.ch, gh);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float A = (MODE == 0) ? Ar[i][j] : 1.0f - Ar[i][j];
        hl[j] = A * (gh[j] + hl[j]);
      }
    }
  }
  __syncthreads();   // everybody is done with the forward prefixes
#pragma unroll
  for (int j = 0; j < 8; ++j) scan_s[pos.run * CT + pos.ch + j] = make_float2(P[j], hl[j]);
  __syncthreads();

  // ---- reverse scan over runs, look-back towards later chunks -------------
  if (tid < CT) {
    float cq = 1.0f, cr = 0.0f;   // run's incoming carry = cq * H_in + cr
#pragma unroll 4
    for (int r = RUNS - 1; r >= 0; --r) {
      const float2 e = scan_s[r * CT + tid];
      scan_s[r * CT + tid] = make_float2(cq, cr);
      cr = __fmaf_rn(e.x, cr, e.y);
      cq = e.x * cq;
    }
    const int cg = c0 + tid;
    float H_in;
    if (chunk == sh.nchunks - 1) {
      H_in = (args.dE_final != nullptr && cg < sh.C) ? args.dE_final[static_cast<long>(b) * sh.C + cg] : 0.0f;
    } else {
      ws.agg[slot * CT + tid] = make_float2(cq, cr);
      __threadfence();
      bar_sync_first(CT);
      if (tid == 0) st_release(&ws.bwd_flags[slot], kFlagAgg);
      H_in = lookback(ws.bwd_flags, ws.agg, ws.bstate, slot, +1, CT, tid, &ws.bwd_hdr[2], ws.status);
    }
    const float H_out = __fmaf_rn(cq, H_in, cr);
    ws.bstate[slot * CT + tid] = H_out;
    __threadfence();
    bar_sync_first(CT);
    if (tid == 0) st_release(&ws.bwd_flags[slot], kFlagIncl);
    if (chunk == 0 && args.dE_init != nullptr && cg < sh.C)
      args.dE_init[static_cast<long>(b) * sh.C + cg] = H_out;
    es_s[tid] = H_in;
  }
  __syncthreads();

  // ---- B: gradients, latest step first ------------------------------------
  float h[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const float2 qr = scan_s[pos.run * CT + pos.ch + j];
    h[j] = __fmaf_rn(qr.x, es_s[pos.ch + j], qr.y);
  }
  T *dag = static_cast<T *>(args.da);
  T *dvg = static_cast<T *>(args.dv);
#pragma unroll
  for (int i = K - 1; i >= 0; --i) {
    const int r = pos.row0 + i;
    if ((t0 + r) < sh.T) {
      float gh[8], vv[8], dav[8], dvv[8];
      get_ghat<T>(q_s + r * CT + pos.ch, dy_s + r * CT + pos.ch, gh);
      if (MODE == 1) Io<T>::load8(v_s + r * CT + pos.ch, vv);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float G = gh[j] + h[j];
        if (MODE == 0) {
          const float A = Ar[i][j];
          dvv[j] = G;
          dav[j] = G * Ep[i][j] * (A * (1.0f - A));
          h[j] = A * G;
        } else {
          const float Ac = Ar[i][j];
          const float A = 1.0f - Ac;
          dvv[j] = G * Ac;
          dav[j] = G * (Ep[i][j] - vv[j]) * (A * Ac);
          h[j] = A * G;
        }
      }
      if (ch_ok) {
        const long off = gbase + static_cast<long>(r) * sh.C;
        Io<T>::store8(dag + off, dav);
        Io<T>::store8(dvg + off, dvv);
      }
    }
  }
}

// ===========================================================================
// One-token decode step: one thread per 8 channels of one (b, h).
// ===========================================================================
template <typename T>
__device__ __forceinline__ void load8_global(const T *p, float (&x)[8]) {
  Io<T>::load8(p, x);
}

template <typename T, int MODE, int LPH>
__global__ void __launch_bounds__(256)
    esa_step_kernel(const T *__restrict__ a, const T *__restrict__ v, const T *__restrict__ q,
                    float *__restrict__ E, T *__restrict__ y, long nvec, float inv_D) {
  const long idx = static_cast<long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const bool act = idx < nvec;
  float x[8], vv[8], qq[8], e[8];
  if (act) {
    load8_global(a + idx * 8, x);
    load8_global(v + idx * 8, vv);
    load8_global(q + idx * 8, qq);
    Io<float>::load8(E + idx * 8, e);
  } else {
#pragma unroll
    for (int j = 0; j < 8; ++j) { x[j] = 0.0f; vv[j] = 0.0f; qq[j] = 0.0f; e[j] = 0.0f; }
  }
  float ss = 0.0f;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const Gate g = gate_of(x[j]);
    e[j] = (MODE == 0) ? __fmaf_rn(g.A, e[j], vv[j]) : __fmaf_rn(g.Ac, vv[j] - e[j], e[j]);
    ss = __fmaf_rn(e[j], e[j], ss);
  }
  ss = head_sum<LPH>(ss);
  const float rr = rsqrtf(__fmaf_rn(ss, inv_D, kEps));
  float yv[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) yv[j] = qq[j] * (e[j] * rr);
  if (act) {
    Io<float>::store8(E + idx * 8, e);
    Io<T>::store8(y + idx * 8, yv);
  }
}

}  // namespace esa
