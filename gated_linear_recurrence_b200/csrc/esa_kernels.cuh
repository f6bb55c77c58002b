// esa_kernels.cuh -- forward scan, backward scan and decode-step kernels of
// the ESA gated linear recurrence for sm_100a.
//
// Work decomposition (forward and backward):
//   * A "chain" is one batch row b and one tile of CT consecutive channels
//     (CT = 64, or D when the head dimension D is 128 or 256).  Heads never straddle
//     a channel tile, so the per-head RMS readout stays inside one CTA.
//   * A chain is cut into time chunks of L steps.  A tile is one (chain,
//     chunk); its a/v/q(/dy) boxes [L x CT] are staged in shared memory by TMA
//     tensor loads (cp.async.bulk.tensor, no multicast).
//   * Inside a tile every thread owns 8 consecutive channels (one 16-byte
//     vector for 16-bit I/O) and a run of K consecutive time steps.  Pass 1
//     folds its run into an affine map x -> P x + S per channel; the runs of a
//     tile are combined by a short serial scan per channel in shared memory;
//     the tile map is chained to earlier tiles by a single-pass decoupled
//     look-back: every channel publishes its chunk map and, once known, its
//     chunk-end carry as epoch-tagged 64-bit words, and reads those of its
//     four nearest predecessors in one round trip (no fences, no flags).
//     Pass 2 replays the run from its exact carry-in and emits the readout.
//   * The carry is always applied in chunk order, oldest first, with the same
//     fused multiply-add that the producing tile used for its own inclusive
//     state, so the result is bitwise independent of how far a look-back
//     reached: outputs are deterministic run to run.
//   * CTAs are persistent and software-pipelined: tiles are numbered by an
//     atomic ticket (taken one tile ahead, chain as the fast index, so a
//     tile's predecessor always belongs to a running CTA), and the TMA loads
//     of the next tile are in flight while the current one is processed.
//     The last CTA to finish resets the ticket counter and advances the
//     workspace epoch, so a call needs no separate reset launch.
//     Every wait is bounded (iteration cap, then an error status).
//   * The forward stores the state at every chunk end (incl_f); the backward
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
  int ntiles;           // nchains * nchunks
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
  static_assert(CT % 32 == 0 && NT >= CT && CT >= 64, "look-back needs CT threads");
  static_assert(RUNS * CT * sizeof(float2) <= kBoxBytes, "scan scratch must fit in the gate box");
  static_assert(VW % LPH == 0, "a head must stay inside a warp");
  static_assert(kBoxBytes % 128 == 0, "boxes must keep 128-byte alignment");
};

// Shared-memory plan of the forward kernel: two stages of {a, v, q} boxes.
template <typename Cfg>
struct FwdSmem {
  static constexpr size_t kStage = 3 * size_t(Cfg::kBoxBytes);
  static constexpr size_t kMisc = Cfg::CT * sizeof(float) + 64;
  static constexpr size_t kBytes = 2 * kStage + kMisc + 128;   // +128 for alignment
};

// Backward: two stages of {a, v} boxes plus one {q, dy} pair.
template <typename Cfg>
struct BwdSmem {
  static constexpr size_t kStage = 2 * size_t(Cfg::kBoxBytes);
  static constexpr size_t kQdy = 2 * size_t(Cfg::kBoxBytes);
  static constexpr size_t kMisc = Cfg::CT * sizeof(float) + 64;
  static constexpr size_t kBytes = 2 * kStage + kQdy + kMisc + 128;
};

__device__ __forceinline__ unsigned char *align128(unsigned char *p) {
  return reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(p) + 127) & ~uintptr_t(127));
}

// Per-thread coordinates inside a tile.
template <typename Cfg>
struct ThreadPos {
  int vec, run, ch, row0;
  __device__ __forceinline__ explicit ThreadPos(int tid) {
    const int warp = tid >> 5, lane = tid & 31;
    const int vseg = warp % Cfg::NVSEG, rgrp = warp / Cfg::NVSEG;
    vec = vseg * Cfg::VW + lane % Cfg::VW;
    run = rgrp * Cfg::RW + lane / Cfg::VW;
    ch = vec * 8;
    row0 = run * Cfg::K;
  }
};

// Run-scan scratch: float2 (map P, S) per (run, channel).  A thread's 8
// channels form a 64-byte block made of four 16-byte chunks; chunk q of vector
// `vec` is stored at position (q + vec / 2) mod 4 so that the 16-byte accesses
// of 8 consecutive vectors hit distinct banks, and the serial scan's 8-byte
// accesses by consecutive channels stay conflict-free as well.
template <int CT>
__device__ __forceinline__ int scan_pos(int run, int c) {
  const int vec = c >> 3, j = c & 7;
  const int chunk = ((j >> 1) + (vec >> 1)) & 3;
  return run * CT + vec * 8 + chunk * 2 + (j & 1);
}

template <int CT>
__device__ __forceinline__ void scan_store8(float2 *scan, int run, int ch, const float (&p)[8], const float (&s)[8]) {
  const int vec = ch >> 3;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int chunk = (q + (vec >> 1)) & 3;
    reinterpret_cast<float4 *>(scan + run * CT + ch + chunk * 2)[0] =
        make_float4(p[2 * q], s[2 * q], p[2 * q + 1], s[2 * q + 1]);
  }
}

template <int CT>
__device__ __forceinline__ void scan_load8(const float2 *scan, int run, int ch, float (&p)[8], float (&s)[8]) {
  const int vec = ch >> 3;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int chunk = (q + (vec >> 1)) & 3;
    const float4 u = reinterpret_cast<const float4 *>(scan + run * CT + ch + chunk * 2)[0];
    p[2 * q] = u.x;
    s[2 * q] = u.y;
    p[2 * q + 1] = u.z;
    s[2 * q + 1] = u.w;
  }
}

// Serial scan over the runs of one channel (threads 0..CT-1).  Replaces each
// entry by the exclusive prefix and returns the tile map (forward order:
// oldest run first; backward order: latest run first).
template <int CT, int RUNS, bool kReverse>
__device__ __forceinline__ float2 scan_runs(float2 *scan, int c) {
  float cp = 1.0f, cs = 0.0f;
#pragma unroll 4
  for (int k = 0; k < RUNS; ++k) {
    const int r = kReverse ? RUNS - 1 - k : k;
    const int at = scan_pos<CT>(r, c);
    const float2 e = scan[at];
    scan[at] = make_float2(cp, cs);
    cs = __fmaf_rn(e.x, cs, e.y);
    cp = cp * e.x;
  }
  return make_float2(cp, cs);
}

// The carry entering chunk `slot` for channel `c`: the nearest predecessor
// (distance 1, 2, ... in direction `dir`, at most `avail`) whose chunk-end
// carry carries the current tag, with the chunk maps of every tile in between
// applied oldest first -- the same fused multiply-adds those tiles used for
// their own carries, so the value does not depend on how far the search went.
// Distances 1..4 are read in one round trip; deeper searches walk one chunk
// at a time.  Bounded: gives up (returns 0, records a timeout, raises the
// abort flag) after kSpinLimit polls or when another CTA raised the flag.
__device__ __forceinline__ float carry_in(const unsigned long long *incl, const ulonglong2 *agg, long slot, int dir,
                                       int avail, int CT, int c, unsigned tag, unsigned *abort_flag,
                                       unsigned *status) {
  const long me = slot * CT + c;
  const long step = static_cast<long>(dir) * CT;
  unsigned ns = 16;
  for (unsigned it = 0; it < kSpinLimit; ++it) {
    unsigned long long iw[4];
    ulonglong2 aw[4];
#pragma unroll
    for (int d = 0; d < 4; ++d) {
      if (d < avail) {
        iw[d] = ld_relaxed_b64(&incl[me + (d + 1) * step]);
        aw[d] = ld_relaxed_v2b64(&agg[me + (d + 1) * step]);
      } else {
        iw[d] = 0ull;
        aw[d] = make_ulonglong2(0ull, 0ull);
      }
    }
    int found = -1;
    bool blocked = false;
#pragma unroll
    for (int d = 0; d < 4; ++d) {
      if (found < 0 && !blocked && d < avail) {
        if (tag_of(iw[d]) == tag) found = d;
        else if (tag_of(aw[d].x) != tag || tag_of(aw[d].y) != tag) blocked = true;
      }
    }
    if (found >= 0) {
      float E = val_of(found == 0 ? iw[0] : found == 1 ? iw[1] : found == 2 ? iw[2] : iw[3]);
#pragma unroll
      for (int d = 3; d >= 0; --d)
        if (d < found) E = __fmaf_rn(val_of(aw[d].x), E, val_of(aw[d].y));
      return E;
    }
    if (!blocked && avail > 4) {
      // Four chunk maps in a row and no carry yet: walk further back.
      int far = 4;   // distances 1..far have published maps
      for (; it < kSpinLimit; ++it) {
        const long at = me + static_cast<long>(far + 1) * step;
        const unsigned long long w = ld_relaxed_b64(&incl[at]);
        if (tag_of(w) == tag) {
          float E = val_of(w);
          for (int d = far; d >= 1; --d) {
            const ulonglong2 m = ld_relaxed_v2b64(&agg[me + static_cast<long>(d) * step]);
            E = __fmaf_rn(val_of(m.x), E, val_of(m.y));
          }
          return E;
        }
        const ulonglong2 m = ld_relaxed_v2b64(&agg[at]);
        if (tag_of(m.x) == tag && tag_of(m.y) == tag && far + 1 < avail) {
          ++far;
          continue;
        }
        if ((it & 63u) == 63u && ld_relaxed(abort_flag)) break;
        __nanosleep(ns);
        ns = ns < 256 ? ns * 2 : 256;
      }
      break;
    }
    if ((it & 63u) == 63u && ld_relaxed(abort_flag)) break;
    __nanosleep(ns);
    ns = ns < 256 ? ns * 2 : 256;
  }
  atomicOr(status, kStatusTimeout);
  atomicExch(abort_flag, 1u);
  return 0.0f;
}

// Kernel prologue shared by both scans (thread 0): read the epoch tag and
// check the workspace is initialised.  Returns the tag, or 0 if not.
__device__ __forceinline__ unsigned scan_prologue(WsHeader *hdr) {
  const unsigned long long magic = *reinterpret_cast<volatile unsigned long long *>(&hdr->magic);
  const unsigned epoch = *reinterpret_cast<volatile unsigned *>(&hdr->epoch);
  if (magic != kWorkspaceMagic || epoch == 0u) {
    atomicOr(&hdr->status, kStatusUninit);
    return 0u;
  }
  return epoch;
}

// Kernel epilogue (all threads): the last CTA to finish resets the ticket,
// done and abort words of kernel `k` and advances the epoch (an exhausted
// epoch range clears the magic, so the next call reports an uninitialised
// workspace instead of reusing tags).
__device__ __forceinline__ void scan_epilogue(WsHeader *hdr, int k, bool ran) {
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    const unsigned prev = atomicAdd(&hdr->done[k], 1u);
    if (prev == gridDim.x - 1) {
      __threadfence();
      hdr->ticket[k] = 0u;
      hdr->done[k] = 0u;
      hdr->abort[k] = 0u;
      if (ran) {
        const unsigned next = hdr->epoch + 1u;
        if (next == 0u) {
          hdr->magic = 0ull;
          hdr->epoch = 0u;
        } else {
          hdr->epoch = next;
        }
      }
      __threadfence();
    }
  }
}

// Gate of one channel in the form the recurrence uses: direct keeps A,
// controlled keeps 1 - A (no cancellation when A is close to 1).
template <int MODE>
__device__ __forceinline__ float gate_coef(const Gate &g) { return MODE == 0 ? g.A : g.Ac; }

// One step of the recurrence with the stored gate coefficient `c`.
template <int MODE>
__device__ __forceinline__ float rec_step(float c, float E, float v) {
  return MODE == 0 ? __fmaf_rn(c, E, v) : __fmaf_rn(c, v - E, E);
}

// ===========================================================================
// Forward scan (persistent).
// ===========================================================================
template <typename T, int MODE, int LPH, int VPR, int L, int K>
__global__ void __launch_bounds__(VPR *(L / K), (VPR * (L / K) <= 128) ? 4 : (VPR * (L / K) <= 256) ? 2 : 1)
    esa_scan_fwd_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_v,
                        const __grid_constant__ CUtensorMap tm_q, const FwdArgs args) {
  using Cfg = TileCfg<T, LPH, VPR, L, K>;
  using Sm = FwdSmem<Cfg>;
  constexpr int CT = Cfg::CT, RUNS = Cfg::RUNS;

  extern __shared__ unsigned char smem_raw[];
  unsigned char *base = align128(smem_raw);
  float *es_s = reinterpret_cast<float *>(base + 2 * Sm::kStage);
  uint64_t *bar = reinterpret_cast<uint64_t *>(es_s + CT);     // [2]
  int *ticket_s = reinterpret_cast<int *>(bar + 2);            // [2]
  unsigned *tag_s = reinterpret_cast<unsigned *>(ticket_s + 2);

  const int tid = threadIdx.x;
  const ScanShape &sh = args.s;
  const Workspace &ws = args.ws;
  WsHeader *hdr = ws.hdr;

  auto box = [&](int stage, int k) -> T * {
    return reinterpret_cast<T *>(base + stage * Sm::kStage + k * size_t(Cfg::kBoxBytes));
  };
  auto issue = [&](int stage, int tile) {
    const int chain = tile % sh.nchains, chunk = tile / sh.nchains;
    const int c0 = (chain % sh.nct) * CT, b = chain / sh.nct, t0 = chunk * L;
    mbar_expect_tx(&bar[stage], 3 * Cfg::kBoxBytes);
    tma_load_3d(box(stage, 0), &tm_a, c0, t0, b, &bar[stage]);
    tma_load_3d(box(stage, 1), &tm_v, c0, t0, b, &bar[stage]);
    tma_load_3d(box(stage, 2), &tm_q, c0, t0, b, &bar[stage]);
  };

  if (tid == 0) {
    prefetch_tensormap(&tm_a);
    prefetch_tensormap(&tm_v);
    prefetch_tensormap(&tm_q);
    mbar_init(&bar[0], 1);
    mbar_init(&bar[1], 1);
    fence_mbar_init();
    fence_proxy_async_smem();
    const unsigned tag = scan_prologue(hdr);
    *tag_s = tag;
    const int t0 = tag ? static_cast<int>(atomicAdd(&hdr->ticket[0], 1u)) : sh.ntiles;
    const int t1 = tag ? static_cast<int>(atomicAdd(&hdr->ticket[0], 1u)) : sh.ntiles;
    ticket_s[0] = t0;
    ticket_s[1] = t1;
    if (t0 < sh.ntiles) issue(0, t0);
    if (t1 < sh.ntiles) issue(1, t1);
  }
  __syncthreads();

  const ThreadPos<Cfg> pos(tid);
  T *yg = static_cast<T *>(args.y);
  const unsigned tag = *tag_s;
  unsigned phase = 0;   // bit s = parity of stage s

  for (int it = 0;; ++it) {
    const int s = it & 1;
    const int tile = ticket_s[s];
    if (tile >= sh.ntiles) break;
    unsigned next = 0;
    if (tid == 0) next = atomicAdd(&hdr->ticket[0], 1u);   // the tile that will refill this stage

    const int chain = tile % sh.nchains, chunk = tile / sh.nchains;
    const int b = chain / sh.nct, c0 = (chain % sh.nct) * CT, t0 = chunk * L;
    const long slot = static_cast<long>(chain) * sh.nchunks + chunk;
    const T *a_s = box(s, 0);
    const T *v_s = box(s, 1);
    const T *q_s = box(s, 2);
    float2 *scan_s = reinterpret_cast<float2 *>(box(s, 0));   // reused once pass 1 is done

    mbar_wait_bounded(&bar[s], (phase >> s) & 1u, &hdr->status);
    phase ^= 1u << s;

    // ---- pass 1: gates and the run's affine map ---------------------------
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
        Ar[i][j] = gate_coef<MODE>(g);
        if (valid) {
          P[j] *= g.A;
          S[j] = rec_step<MODE>(Ar[i][j], S[j], vv[j]);
        }
      }
    }
    __syncthreads();   // the gate box is free from here on
    scan_store8<CT>(scan_s, pos.run, pos.ch, P, S);
    __syncthreads();

    // ---- scan over runs, look-back, publish --------------------------------
    if (tid < CT) {
      const float2 tmap = scan_runs<CT, RUNS, false>(scan_s, tid);
      const int cg = c0 + tid;
      float E_start;
      const long at = slot * CT + tid;
      if (chunk == 0) {
        E_start = (args.E_init != nullptr && cg < sh.C) ? args.E_init[static_cast<long>(b) * sh.C + cg] : 0.0f;
      } else {
        st_relaxed_v2b64(&ws.agg[at], make_ulonglong2(pack_tag(tmap.x, tag), pack_tag(tmap.y, tag)));
        E_start = carry_in(ws.incl_f, ws.agg, slot, -1, chunk, CT, tid, tag, &hdr->abort[0], &hdr->status);
      }
      const float E_end = __fmaf_rn(tmap.x, E_start, tmap.y);
      st_relaxed_b64(&ws.incl_f[at], pack_tag(E_end, tag));
      if (chunk == sh.nchunks - 1 && args.E_final != nullptr && cg < sh.C)
        args.E_final[static_cast<long>(b) * sh.C + cg] = E_end;
      es_s[tid] = E_start;
    }
    __syncthreads();

    // ---- pass 2: exact states and the readout ------------------------------
    float E[8];
    {
      float pe[8], se[8];
      scan_load8<CT>(scan_s, pos.run, pos.ch, pe, se);
#pragma unroll
      for (int j = 0; j < 8; ++j) E[j] = __fmaf_rn(pe[j], es_s[pos.ch + j], se[j]);
    }
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
        E[j] = rec_step<MODE>(Ar[i][j], E[j], vv[j]);
        ss = __fmaf_rn(E[j], E[j], ss);
      }
      ss = head_sum<LPH>(ss);
      const float rr = rsqrt_approx(__fmaf_rn(ss, sh.inv_D, kEps));
      float yv[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) yv[j] = qq[j] * (E[j] * rr);
      if (valid && ch_ok) Io<T>::store8(yg + gbase + static_cast<long>(r) * sh.C, yv);
    }

    // ---- refill this stage --------------------------------------------------
    __syncthreads();   // everybody is done with stage s
    if (tid == 0) {
      ticket_s[s] = static_cast<int>(next);
      if (static_cast<int>(next) < sh.ntiles) {
        fence_proxy_async_smem();   // generic writes (scan scratch) before the async refill
        issue(s, static_cast<int>(next));
      }
    }
  }
  scan_epilogue(hdr, 0, tag != 0u);
}

// ghat (8 float32) of one thread's row, kept in that row's q and dy slots:
// 16-bit I/O splits it over both 16-byte slots; float32 I/O uses the q slot.
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

// ===========================================================================
// Backward scan (persistent).
// ===========================================================================
template <typename T, int MODE, int LPH, int VPR, int L, int K>
__global__ void __launch_bounds__(VPR *(L / K), (VPR * (L / K) <= 128) ? 4 : (VPR * (L / K) <= 256) ? 2 : 1)
    esa_scan_bwd_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_v,
                        const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_dy,
                        const BwdArgs args) {
  using Cfg = TileCfg<T, LPH, VPR, L, K>;
  using Sm = BwdSmem<Cfg>;
  constexpr int CT = Cfg::CT, RUNS = Cfg::RUNS;

  extern __shared__ unsigned char smem_raw[];
  unsigned char *base = align128(smem_raw);
  T *q_s = reinterpret_cast<T *>(base + 2 * Sm::kStage);
  T *dy_s = q_s + L * CT;
  float *es_s = reinterpret_cast<float *>(base + 2 * Sm::kStage + Sm::kQdy);
  uint64_t *bar = reinterpret_cast<uint64_t *>(es_s + CT);     // [0..1] a/v stages, [2] q/dy
  int *ticket_s = reinterpret_cast<int *>(bar + 3);            // [2]
  unsigned *tag_s = reinterpret_cast<unsigned *>(ticket_s + 2);

  const int tid = threadIdx.x;
  const ScanShape &sh = args.s;
  const Workspace &ws = args.ws;
  WsHeader *hdr = ws.hdr;

  auto box = [&](int stage, int k) -> T * {
    return reinterpret_cast<T *>(base + stage * Sm::kStage + k * size_t(Cfg::kBoxBytes));
  };
  auto coords = [&](int tile, int &c0, int &t0, int &b) {
    const int chain = tile % sh.nchains;
    const int chunk = sh.nchunks - 1 - tile / sh.nchains;   // latest chunk first
    c0 = (chain % sh.nct) * CT;
    b = chain / sh.nct;
    t0 = chunk * L;
  };
  auto issue_av = [&](int stage, int tile) {
    int c0, t0, b;
    coords(tile, c0, t0, b);
    mbar_expect_tx(&bar[stage], 2 * Cfg::kBoxBytes);
    tma_load_3d(box(stage, 0), &tm_a, c0, t0, b, &bar[stage]);
    tma_load_3d(box(stage, 1), &tm_v, c0, t0, b, &bar[stage]);
  };
  auto issue_qdy = [&](int tile) {
    int c0, t0, b;
    coords(tile, c0, t0, b);
    mbar_expect_tx(&bar[2], 2 * Cfg::kBoxBytes);
    tma_load_3d(q_s, &tm_q, c0, t0, b, &bar[2]);
    tma_load_3d(dy_s, &tm_dy, c0, t0, b, &bar[2]);
  };

  if (tid == 0) {
    prefetch_tensormap(&tm_a);
    prefetch_tensormap(&tm_v);
    prefetch_tensormap(&tm_q);
    prefetch_tensormap(&tm_dy);
    mbar_init(&bar[0], 1);
    mbar_init(&bar[1], 1);
    mbar_init(&bar[2], 1);
    fence_mbar_init();
    fence_proxy_async_smem();
    const unsigned tag = scan_prologue(hdr);
    *tag_s = tag;
    const int t0 = tag ? static_cast<int>(atomicAdd(&hdr->ticket[1], 1u)) : sh.ntiles;
    const int t1 = tag ? static_cast<int>(atomicAdd(&hdr->ticket[1], 1u)) : sh.ntiles;
    ticket_s[0] = t0;
    ticket_s[1] = t1;
    if (t0 < sh.ntiles) {
      issue_av(0, t0);
      issue_qdy(t0);
    }
    if (t1 < sh.ntiles) issue_av(1, t1);
  }
  __syncthreads();

  const ThreadPos<Cfg> pos(tid);
  T *dag = static_cast<T *>(args.da);
  T *dvg = static_cast<T *>(args.dv);
  T *dqg = static_cast<T *>(args.dq);
  const unsigned tag = *tag_s;
  unsigned phase = 0;   // bits 0..1: a/v stages, bit 2: q/dy

  for (int it = 0;; ++it) {
    const int s = it & 1;
    const int tile = ticket_s[s];
    if (tile >= sh.ntiles) break;
    unsigned next = 0;
    if (tid == 0) next = atomicAdd(&hdr->ticket[1], 1u);

    const int chain = tile % sh.nchains;
    const int chunk = sh.nchunks - 1 - tile / sh.nchains;
    const int b = chain / sh.nct, c0 = (chain % sh.nct) * CT, t0 = chunk * L;
    const long slot = static_cast<long>(chain) * sh.nchunks + chunk;
    const T *a_s = box(s, 0);
    const T *v_s = box(s, 1);
    float2 *scan_s = reinterpret_cast<float2 *>(box(s, 0));

    float E_ck = 0.0f;   // forward state entering the chunk, channel tid (checkpoint)
    if (tid < CT) {
      const int cg = c0 + tid;
      E_ck = (chunk == 0) ? ((args.E_init != nullptr && cg < sh.C) ? args.E_init[static_cast<long>(b) * sh.C + cg]
                                                                   : 0.0f)
                          : val_of(__ldcg(&ws.incl_f[(slot - 1) * CT + tid]));
    }

    mbar_wait_bounded(&bar[s], (phase >> s) & 1u, &hdr->status);
    phase ^= 1u << s;

    // ---- F1: gates and the run's forward map ------------------------------
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
        Ar[i][j] = gate_coef<MODE>(g);
        if (valid) {
          P[j] *= g.A;
          S[j] = rec_step<MODE>(Ar[i][j], S[j], vv[j]);
        }
      }
    }
    __syncthreads();
    scan_store8<CT>(scan_s, pos.run, pos.ch, P, S);
    if (tid < CT) es_s[tid] = E_ck;
    __syncthreads();
    if (tid < CT) scan_runs<CT, RUNS, false>(scan_s, tid);
    __syncthreads();

    // ---- F2: replay states, readout backward, dq, ghat ---------------------
    // ghat of each row overwrites that row's q/dy slots (only this thread
    // reads them); w keeps what da needs of the previous state.
    float w[K][8];   // direct: E_{t-1}; controlled: E_{t-1} - v_t
    {
      float E[8];
      {
        float pe[8], se[8];
        scan_load8<CT>(scan_s, pos.run, pos.ch, pe, se);
#pragma unroll
        for (int j = 0; j < 8; ++j) E[j] = __fmaf_rn(pe[j], es_s[pos.ch + j], se[j]);
      }
      mbar_wait_bounded(&bar[2], (phase >> 2) & 1u, &hdr->status);
      phase ^= 4u;
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
          w[i][j] = (MODE == 0) ? E[j] : E[j] - vv[j];
          E[j] = rec_step<MODE>(Ar[i][j], E[j], vv[j]);
          ss = __fmaf_rn(E[j], E[j], ss);
        }
        ss = head_sum<LPH>(ss);
        const float rr = rsqrt_approx(__fmaf_rn(ss, sh.inv_D, kEps));
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
        if (valid && (c0 + pos.ch) < sh.C)
          Io<T>::store8(dqg + (static_cast<long>(b) * sh.T + t0 + r) * sh.C + c0 + pos.ch, dqv);
      }
    }

    // ---- R1: the run's reverse map h -> P h + hl ----------------------------
    {
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
      __syncthreads();   // every thread has read its forward prefixes
      scan_store8<CT>(scan_s, pos.run, pos.ch, P, hl);
    }
    __syncthreads();

    // ---- reverse scan over runs, look-back towards later chunks -------------
    if (tid < CT) {
      const float2 tmap = scan_runs<CT, RUNS, true>(scan_s, tid);
      const int cg = c0 + tid;
      float H_in;
      const long at = slot * CT + tid;
      if (chunk == sh.nchunks - 1) {
        H_in = (args.dE_final != nullptr && cg < sh.C) ? args.dE_final[static_cast<long>(b) * sh.C + cg] : 0.0f;
      } else {
        st_relaxed_v2b64(&ws.agg[at], make_ulonglong2(pack_tag(tmap.x, tag), pack_tag(tmap.y, tag)));
        H_in = carry_in(ws.incl_b, ws.agg, slot, +1, sh.nchunks - 1 - chunk, CT, tid, tag, &hdr->abort[1],
                        &hdr->status);
      }
      const float H_out = __fmaf_rn(tmap.x, H_in, tmap.y);
      st_relaxed_b64(&ws.incl_b[at], pack_tag(H_out, tag));
      if (chunk == 0 && args.dE_init != nullptr && cg < sh.C)
        args.dE_init[static_cast<long>(b) * sh.C + cg] = H_out;
      es_s[tid] = H_in;
    }
    __syncthreads();

    // ---- B: total gradient G_t and da, dv, latest step first -----------------
    {
      float h[8];
      {
        float pe[8], se[8];
        scan_load8<CT>(scan_s, pos.run, pos.ch, pe, se);
#pragma unroll
        for (int j = 0; j < 8; ++j) h[j] = __fmaf_rn(pe[j], es_s[pos.ch + j], se[j]);
      }
      const bool ch_ok = (c0 + pos.ch) < sh.C;
      const long gbase = (static_cast<long>(b) * sh.T + t0) * sh.C + c0 + pos.ch;
#pragma unroll
      for (int i = K - 1; i >= 0; --i) {
        const int r = pos.row0 + i;
        if ((t0 + r) < sh.T) {
          float gh[8], dav[8], dvv[8];
          get_ghat<T>(q_s + r * CT + pos.ch, dy_s + r * CT + pos.ch, gh);
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const float G = gh[j] + h[j];
            if (MODE == 0) {
              const float A = Ar[i][j];
              dvv[j] = G;
              dav[j] = G * w[i][j] * (A * (1.0f - A));
              h[j] = A * G;
            } else {
              const float Ac = Ar[i][j];
              const float A = 1.0f - Ac;
              dvv[j] = G * Ac;
              dav[j] = G * w[i][j] * (A * Ac);
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

    // ---- refill: next tile's q/dy, and this a/v stage -------------------------
    __syncthreads();
    if (tid == 0) {
      fence_proxy_async_smem();   // generic smem writes before the async refills
      if (ticket_s[s ^ 1] < sh.ntiles) issue_qdy(ticket_s[s ^ 1]);
      ticket_s[s] = static_cast<int>(next);
      if (static_cast<int>(next) < sh.ntiles) issue_av(s, static_cast<int>(next));
    }
  }
  scan_epilogue(hdr, 1, tag != 0u);
}

// ===========================================================================
// One-token decode step: one thread per 8 channels of one (b, h).
// ===========================================================================
template <typename T, int MODE, int LPH>
__global__ void __launch_bounds__(256)
    esa_step_kernel(const T *__restrict__ a, const T *__restrict__ v, const T *__restrict__ q,
                    float *__restrict__ E, T *__restrict__ y, long nvec, float inv_D) {
  const long idx = static_cast<long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const bool act = idx < nvec;
  float x[8], vv[8], qq[8], e[8];
  if (act) {
    Io<T>::load8(a + idx * 8, x);
    Io<T>::load8(v + idx * 8, vv);
    Io<T>::load8(q + idx * 8, qq);
    Io<float>::load8(E + idx * 8, e);
  } else {
#pragma unroll
    for (int j = 0; j < 8; ++j) { x[j] = 0.0f; vv[j] = 0.0f; qq[j] = 0.0f; e[j] = 0.0f; }
  }
  float ss = 0.0f;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const Gate g = gate_of(x[j]);
    e[j] = rec_step<MODE>(gate_coef<MODE>(g), e[j], vv[j]);
    ss = __fmaf_rn(e[j], e[j], ss);
  }
  ss = head_sum<LPH>(ss);
  const float rr = rsqrt_approx(__fmaf_rn(ss, inv_D, kEps));
  float yv[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) yv[j] = qq[j] * (e[j] * rr);
  if (act) {
    Io<float>::store8(E + idx * 8, e);
    Io<T>::store8(y + idx * 8, yv);
  }
}

}  // namespace esa
