// esa_fused.cuh -- forward scan with the input projections fused in.
//
// The ESA layer computes its gate logits, values and queries by projection
// of the layer input ("entangled-state-attention 0.1.0", section "Core
// idea": a = x W_A, v = x W_V, q = x W_Q).  This kernel reads x instead of
// a, v, q: for every tile (128 time steps x 64 channels of one batch row) it
// multiplies the tile's x rows [128 x C_in] by the matching rows of the
// three weight matrices [192 x C_in] on the tensor cores (tcgen05.mma, fp32
// accumulator in tensor memory), rounds a, v, q to the I/O type -- the values
// an unfused projection would have written -- into the tile's shared-memory
// boxes, and then runs the same chunked scan, look-back and readout as the
// forward scan kernel.  HBM traffic per token is C_in + C elements instead
// of 4 C (plus the projection's own 3 C writes and C_in reads).
//
// Organisation (one CTA per SM, 512 threads; 256 for C_in = 256):
//   * The CTA serves one channel tile ct (blockIdx.y) and keeps that tile's
//     weight slice resident in shared memory (3 x 64 rows x C_in, loaded
//     once by TMA with the 128-byte swizzle the MMA reads).
//   * Two independent tile groups of 256 threads (8 warps) share the CTA;
//     each has its own x buffer, a/v/q boxes, barriers and 256 columns of
//     tensor memory, and runs its own persistent loop over tiles taken from
//     the channel tile's ticket counter (batch row fastest), so the two
//     groups hide each other's latencies as two CTAs per SM would.  With
//     C_in = 256 the weight slice (96 KB) and one group's x buffer (64 KB)
//     leave room for one group only.
//   * Per tile: one thread takes the next tile's ticket (the atomic's result
//     is used only after the read-out, so its round trip is hidden), issues
//     C_in / 16 MMAs of 128 x 192 x 16 on the tile's x rows and commits them
//     to an mbarrier; after the read-out the x buffer is refilled with the
//     next tile's rows; the group's 8 warps
//     read the accumulator (warp w: lanes 32 (w mod 4).., 96 columns) and
//     store a, v, q; then pass 1, the run scan, the look-back and pass 2 as
//     in the forward scan.  While the tile scans, the issuing thread checks
//     (without blocking) whether the next tile's x has landed and, if so,
//     starts its MMAs at once, so they run under this tile's scan.
//   * Every wait is bounded; tensor memory is freed at the end whatever
//     happened.
#pragma once

#include <type_traits>

#include "esa_kernels.cuh"
#include "esa_umma.cuh"

namespace esa {

struct FusedArgs {
  ScanShape s;          // nslots / nchunks (two slots per tile) / nct as for the forward
  int ntiles_ct;        // tiles per channel tile: B * nchunks
  void *y;
  float *E_final;
  const float *E_init;
  void *a_out, *v_out, *q_out;   // the rounded projections [B][T][C], or all null
  void *z;                       // the layer's output z = y W_O^T [B][T][64] (output-projection kernels only)
  Workspace ws;
};

template <typename T, int CIN, bool WO = false>
struct FusedPlan {
  static constexpr int L = 128, CT = 64, K = 4, SUB = 2, NTG = 256;
  static constexpr int NG = CIN <= 128 ? 2 : 1;   // tile groups per CTA
  static constexpr int KB = CIN / 64;                          // 128-byte k-blocks
  static constexpr size_t kXkb = size_t(L) * 128;             // one k-block of x: 16 KB
  static constexpr size_t kWkb = size_t(3 * CT) * 128;        // one k-block of W: 24 KB
  static constexpr size_t kX = KB * kXkb;
  static constexpr size_t kW = KB * kWkb;
  static constexpr size_t kBox = size_t(L) * CT * sizeof(T);  // one of a / v / q
  static constexpr size_t kMisc = 4096;                        // es_s, seg_s, barriers, infos
  static constexpr size_t kGroup = kX + 3 * kBox + kMisc;
  // W_O [64 out][64 in], resident with the weight slice (output-projection kernels).
  static constexpr size_t kWO = WO ? size_t(64) * 128 : 0;
  static constexpr size_t kBytes = kW + NG * kGroup + 1024 /*CTA misc*/ + kWO + 1024 /*alignment*/;
  static_assert(CIN % 64 == 0 && CIN >= 64 && CIN <= 256, "C_in of 64, 128 or 256");
  static_assert(kW % 1024 == 0 && kX % 1024 == 0 && kGroup % 1024 == 0, "swizzled tiles need 1024-byte alignment");
  static_assert(kBytes <= 227 * 1024, "shared memory");
};

// The a / v / q boxes are [128 rows][64 channels] with the eight 16-byte
// vectors of a row permuted by the row: vector j of row r sits at position
// j ^ (r mod 8).  The accumulator read-out writes 32 consecutive rows per
// warp instruction and the scan reads 4 rows x 8 vectors; both touch every
// bank once per 128 bytes.
__device__ __forceinline__ int box_vec(int j, int r) { return j ^ (r & 7); }

__device__ __forceinline__ unsigned char *smem_aligned1024(unsigned char *smem) {
  const uint32_t a = smem_u32(smem);
  return smem + (((a + 1023u) & ~1023u) - a);
}

// 32 fp32 accumulator values -> 32 I/O-type values (round to nearest even),
// packed in pairs.
template <typename T>
__device__ __forceinline__ void pack32(const uint32_t (&v)[32], uint4 (&out)[4]) {
  uint32_t *o = reinterpret_cast<uint32_t *>(out);
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const float2 f = make_float2(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
    if constexpr (sizeof(T) == 2 && std::is_same<T, __half>::value) {
      const __half2 h = __float22half2_rn(f);
      o[i] = *reinterpret_cast<const uint32_t *>(&h);
    } else {
      const __nv_bfloat162 h = __float22bfloat162_rn(f);
      o[i] = *reinterpret_cast<const uint32_t *>(&h);
    }
  }
}

template <typename T, int MODE, int LPH, int CIN, bool WO>
__global__ void __launch_bounds__(FusedPlan<T, CIN, WO>::NG * 256, 1)
    esa_fused_fwd_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                         const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_v,
                         const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_wo,
                         const FusedArgs args) {
  using Pl = FusedPlan<T, CIN, WO>;
  constexpr int L = Pl::L, CT = Pl::CT, K = Pl::K, SUB = Pl::SUB, KB = Pl::KB;
  constexpr int SW = scan_segments<L / K, Pl::NTG, CT>();
  using Cfg = TileCfg<T, LPH, 8, L, K, SW>;
  constexpr int RUNS = Cfg::RUNS, NP = Cfg::NP;
  static_assert(Cfg::NT == Pl::NTG, "a tile group is one scan block");
  static_assert(Cfg::kBoxBytes == Pl::kBox, "box size");
  constexpr uint32_t kIdesc = umma_idesc_f16(std::is_same<T, __half>::value ? 0 : 1, 128, 3 * CT);
  // Output projection: M = 128 rows of y, N = 64 outputs, into accumulator
  // columns 3 CT .. 4 CT - 1 (the projections use the first 3 CT).
  constexpr uint32_t kIdescWO = umma_idesc_f16(std::is_same<T, __half>::value ? 0 : 1, 128, 64);
  static_assert(!WO || CT == 64, "the output projection needs the whole row of y in one channel tile");

  extern __shared__ unsigned char smem_raw[];
  unsigned char *base = smem_aligned1024(smem_raw);
  const int g = threadIdx.x / Pl::NTG;        // tile group
  const int tid = threadIdx.x % Pl::NTG;      // thread within the group
  const int ct = blockIdx.y;                  // channel tile of this CTA
  const int bar_all = 1 + 2 * g, bar_scan = 2 + 2 * g;

  unsigned char *w_s = base;
  unsigned char *grp = base + Pl::kW + g * Pl::kGroup;
  unsigned char *x_s = grp;
  T *a_s = reinterpret_cast<T *>(grp + Pl::kX);
  T *v_s = a_s + L * CT;
  T *q_s = v_s + L * CT;
  unsigned char *misc = grp + Pl::kX + 3 * Pl::kBox;
  float *es_s = reinterpret_cast<float *>(misc);                          // CT floats
  float4 *seg_s = reinterpret_cast<float4 *>(misc + 256);                 // SW x NP
  uint64_t *bar = reinterpret_cast<uint64_t *>(misc + 256 + SW * NP * 16); // [0] x full, [1] mma done, [2] W_O mma done
  TileInfo *info_s = reinterpret_cast<TileInfo *>(bar + 3);               // [2]
  unsigned *tag_s = reinterpret_cast<unsigned *>(info_s + 2);
  unsigned char *cta_misc = base + Pl::kW + Pl::NG * Pl::kGroup;
  uint64_t *w_bar = reinterpret_cast<uint64_t *>(cta_misc);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(cta_misc + 8);
  unsigned char *wo_s = cta_misc + 1024;   // W_O (output-projection kernels), 1024-byte aligned

  const ScanShape &sh = args.s;
  const Workspace &ws = args.ws;
  WsHeader *hdr = ws.hdr;

  auto decode = [&](int tile) -> TileInfo {
    TileInfo t;
    t.tile = tile;
    t.pad = 0;
    if (tile >= args.ntiles_ct) {
      t.chunk = t.b = t.c0 = t.t0 = 0;
      t.slot = 0;
      return t;
    }
    t.b = tile % sh.B;
    t.chunk = tile / sh.B;
    t.c0 = ct * CT;
    t.t0 = t.chunk * L;
    const long chain = static_cast<long>(t.b) * sh.nct + ct;
    t.slot = chain * sh.nslots + static_cast<long>(t.chunk) * SUB;
    return t;
  };
  auto issue_x = [&](const TileInfo &t) {   // the group's thread 0
    mbar_expect_tx(&bar[0], static_cast<unsigned>(Pl::kX));
#pragma unroll
    for (int kb = 0; kb < KB; ++kb) tma_load_3d(x_s + kb * Pl::kXkb, &tm_x, kb * 64, t.t0, t.b, &bar[0]);
  };

  if (threadIdx.x == 0) {
    prefetch_tensormap(&tm_x);
    prefetch_tensormap(&tm_w);
    mbar_init(w_bar, 1);
  }
  if (tid == 0) {
    mbar_init(&bar[0], 1);
    mbar_init(&bar[1], 1);
    mbar_init(&bar[2], 1);
    fence_mbar_init();
  }
  if (threadIdx.x < 32) {   // warp 0 allocates the CTA's tensor memory: 256 columns per group
    tmem_alloc(tmem_slot, Pl::NG * 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const uint32_t tmem_d = tmem_base + static_cast<uint32_t>(g * 256);

  if (threadIdx.x == 0) {   // the channel tile's weight slice: rows p C + ct CT + [0, 64) of W
    mbar_expect_tx(w_bar, static_cast<unsigned>(Pl::kW + Pl::kWO));
    if constexpr (WO) tma_load_2d(wo_s, &tm_wo, 0, 0, w_bar);
#pragma unroll
    for (int kb = 0; kb < KB; ++kb)
#pragma unroll
      for (int p = 0; p < 3; ++p)
        tma_load_2d(w_s + kb * Pl::kWkb + p * (CT * 128), &tm_w, kb * 64, p * sh.C + ct * CT, w_bar);
  }
  if (tid == 0) {
    const unsigned tag = scan_prologue(hdr);
    *tag_s = tag;
    const int first = tag ? static_cast<int>(atomicAdd(&hdr->ct_ticket[ct], 1u)) : args.ntiles_ct;
    const TileInfo t = decode(first);
    info_s[0] = t;
    if (first < args.ntiles_ct) issue_x(t);
  }
  __syncthreads();

  const ThreadPos<Cfg> pos(tid);
  T *yg = static_cast<T *>(args.y);
  const unsigned tag = *tag_s;
  unsigned ph_x = 0, ph_m = 0;   // ph_x: the group's thread 0 only
  unsigned ph_o = 0;             // the output projection's barrier
  bool pre = false;              // thread 0: the current tile's MMAs were issued during the previous tile
  bool next_ok = false;          // thread 0: the next ticket is a tile
  // MMAs of the tile whose x is in the buffer (thread 0; the accumulator is free).
  auto issue_mma = [&]() {
    tc_fence_after();
    const uint32_t xa = smem_u32(x_s), wa = smem_u32(w_s);
#pragma unroll
    for (int kb = 0; kb < KB; ++kb)
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        umma_f16(tmem_d, umma_desc_sw128(xa + kb * Pl::kXkb) + 2 * kk, umma_desc_sw128(wa + kb * Pl::kWkb) + 2 * kk,
                 kIdesc, (kb | kk) != 0);
    umma_commit(&bar[1]);
  };
  // Start the next tile's MMAs as soon as its x has landed, while this tile
  // is still scanning (thread 0, after this tile's accumulator was read).
  auto try_issue_next = [&]() {
    if (tid == 0 && next_ok && !pre && mbar_test_wait(&bar[0], ph_x)) {
      ph_x ^= 1u;
      issue_mma();
      pre = true;
    }
  };

  for (int it = 0;; ++it) {
    const TileInfo ti = info_s[it & 1];
    if (ti.tile >= args.ntiles_ct) break;
    const int chunk = ti.chunk, b = ti.b, c0 = ti.c0, t0 = ti.t0;
    const long slot = ti.slot;
    const long slot_end = slot + SUB - 1;
    const bool full = t0 + L <= sh.T && c0 + CT <= sh.C;

    // ---- projections on the tensor cores -----------------------------------
    unsigned nt_raw = 0;
    if (tid == 0) {
      nt_raw = atomicAdd(&hdr->ct_ticket[ct], 1u);   // the next tile; its value is needed only after the read-out
      if (!pre) {
        if (it == 0) mbar_wait_bounded(w_bar, 0u, &hdr->status);
        mbar_wait_bounded(&bar[0], ph_x, &hdr->status);
        ph_x ^= 1u;
        issue_mma();
      }
      pre = false;
    }

    const bool lb_thread = tid >= Cfg::LB0 && tid < Cfg::LB0 + CT;
    unsigned long long early = 0ull;
    if (lb_thread && chunk > 0) early = ld_relaxed_b64(&ws.incl_f[(slot_end - SUB) * CT + (tid - Cfg::LB0)]);

    mbar_wait_bounded(&bar[1], ph_m, &hdr->status);
    ph_m ^= 1u;
    tc_fence_after();

    // ---- accumulator -> a, v, q boxes (rounded to the I/O type) ------------
    __syncwarp();   // the tensor-memory loads below are warp-collective
    {
      const int wg = tid >> 5, lane = tid & 31;
      const int quad = wg & 3;
      const int r = 32 * quad + lane;
#pragma unroll
      for (int j = 0; j < 3; ++j) {
        const int c = (wg >> 2) * 96 + 32 * j;   // accumulator column: projection c / 64, channel c % 64
        uint32_t acc[32];
        tmem_ld32(tmem_d + (static_cast<uint32_t>(32 * quad) << 16) + static_cast<uint32_t>(c), acc);
        tmem_wait_ld();
        uint4 out[4];
        pack32<T>(acc, out);
        const int p = c >> 6;
        uint4 *row = reinterpret_cast<uint4 *>((p == 0 ? a_s : p == 1 ? v_s : q_s) + r * CT);
#pragma unroll
        for (int i = 0; i < 4; ++i) row[box_vec(((c & 63) >> 3) + i, r)] = out[i];
      }
    }
    const bool store_avq = args.a_out != nullptr;
    if (store_avq) fence_proxy_async_smem();   // box writes, before the TMA store reads them
    tc_fence_before();
    named_sync(bar_all, Pl::NTG);
    if (tid == 0) {   // x has been consumed: the next tile's rows go in now
      const int nt = static_cast<int>(nt_raw);
      const TileInfo tn = decode(nt);
      info_s[(it + 1) & 1] = tn;
      next_ok = nt < args.ntiles_ct;
      if (next_ok) issue_x(tn);
    }
    // The projections themselves, when asked for: the boxes' layout is the
    // 128-byte swizzle, so one TMA store per box writes them out.
    if (store_avq && tid == 0) {
      tma_store_3d(&tm_a, c0, t0, b, a_s);
      tma_store_3d(&tm_v, c0, t0, b, v_s);
      tma_store_3d(&tm_q, c0, t0, b, q_s);
      bulk_commit();
    }

    float *scan_s = reinterpret_cast<float *>(a_s);   // reused once pass 1 is done

    auto resolve_carry = [&]() {
      const int c = tid - Cfg::LB0;
      const int cg = c0 + c;
      float E_start;
      if (chunk == 0) {
        E_start = (args.E_init != nullptr && cg < sh.C) ? args.E_init[static_cast<long>(b) * sh.C + cg] : 0.0f;
      } else if (tag_of(early) == tag) {
        E_start = val_of(early);
      } else {
        E_start = carry_in(ws.incl_f, ws.agg, slot_end * CT + c, -static_cast<long>(SUB) * CT, chunk, tag,
                           &hdr->abort[0], &hdr->status);
      }
      es_s[c] = E_start;
    };

    // ---- pass 1: gates and the run's affine map ---------------------------
    float2 Ar[K][4];
    float2 P[4], S[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) { P[q] = splat(1.0f); S[q] = splat(0.0f); }
    with_full(full, [&](auto kf) {
#pragma unroll
      for (int i = 0; i < K; ++i) {
        const int r = pos.row0 + i;
        const bool valid = decltype(kf)::value || (t0 + r) < sh.T;
        float2 x[4];
        VRow<T, MODE> vr;
        Io<T>::load8_gate(a_s + r * CT + 8 * box_vec(pos.vec, r), x);
        vr.load(v_s + r * CT + 8 * box_vec(pos.vec, r));
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const Gate2 gt = gate2(x[q]);
          Ar[i][q] = gate_coef<MODE>(gt);
          if (valid) {
            P[q] = mul2(P[q], gt.A);
            S[q] = vr.step(q, Ar[i][q], S[q]);
          }
        }
      }
    });
    // The scan scratch overwrites the a box: with the projections being
    // stored, the whole group waits until the TMA store has read it.
    if (store_avq) {
      if (tid == 0) bulk_wait_read0();
      named_sync(bar_all, Pl::NTG);
    } else if constexpr (Cfg::kWarpScratch) {
      __syncwarp();
    } else {
      named_sync(bar_all, Pl::NTG);
    }
    scan_store8<CT>(scan_s, pos.run, pos.ch, P, S);
    named_sync(bar_all, Pl::NTG);

    // ---- scan over runs, look-back, publish --------------------------------
    const int c2 = tid % NP, sg = tid / NP;
    const bool publisher = tid < Cfg::NSCAN && sg == SW - 1;
    float2 tP = splat(1.0f), tS = splat(0.0f);
    if (tid < Cfg::NSCAN) {
      float2 eP, eS;
      scan_runs<CT, RUNS, SW, false>(scan_s, seg_s, c2, sg, eP, eS, tP, tS, bar_scan);
      if (chunk > 0 && chunk < sh.nchunks - 1 && publisher) {
        const long at = slot_end * CT + 2 * c2;
        st_relaxed_v2b64(&ws.agg[at], make_ulonglong2(pack_tag(tP.x, tag), pack_tag(tS.x, tag)));
        st_relaxed_v2b64(&ws.agg[at + 1], make_ulonglong2(pack_tag(tP.y, tag), pack_tag(tS.y, tag)));
      }
      scan_runs_fold<CT, RUNS, SW, false>(scan_s, c2, sg, eP, eS);
    }
    if (lb_thread) resolve_carry();
    named_sync(bar_all, Pl::NTG);
    try_issue_next();
    if (publisher) {   // chunk-end state of the pair
      const float2 E_in = reinterpret_cast<const float2 *>(es_s)[c2];
      const float2 E_end = fma2(tP, E_in, tS);
      if (chunk * SUB + SUB - 1 < sh.nslots)
        st_relaxed_v2b64(reinterpret_cast<ulonglong2 *>(&ws.incl_f[slot_end * CT + 2 * c2]),
                         make_ulonglong2(pack_tag(E_end.x, tag), pack_tag(E_end.y, tag)));
      const int cg = c0 + 2 * c2;
      if (chunk == sh.nchunks - 1 && args.E_final != nullptr && cg < sh.C)
        *reinterpret_cast<float2 *>(&args.E_final[static_cast<long>(b) * sh.C + cg]) = E_end;
    }

    // ---- pass 2: exact states and the readout ------------------------------
    {
      float2 E[4];
      run_carry<CT>(scan_s, es_s, pos.run, pos.ch, E);
      const long gbase = (static_cast<long>(b) * sh.T + t0) * sh.C + c0 + pos.ch;
      with_full(full, [&](auto kf) {
        constexpr bool kFull = decltype(kf)::value;
        const bool ch_ok = kFull || (c0 + pos.ch) < sh.C;
#pragma unroll
        for (int i = 0; i < K; ++i) {
          const int r = pos.row0 + i;
          const bool valid = kFull || (t0 + r) < sh.T;
          float2 qq[4];
          VRow<T, MODE> vr;
          vr.load(v_s + r * CT + 8 * box_vec(pos.vec, r));
          Io<T>::load8(q_s + r * CT + 8 * box_vec(pos.vec, r), qq);
          float2 ss = splat(0.0f);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            E[q] = vr.step(q, Ar[i][q], E[q]);
            ss = fma2(E[q], E[q], ss);
          }
          const float rr = rsqrt_approx(__fmaf_rn(head_sum2<LPH>(ss), sh.inv_D, kEps));
          float2 yv[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) yv[q] = mul2(qq[q], mul2(E[q], splat(rr)));
          if (valid && ch_ok && (!WO || yg != nullptr)) Io<T>::store8(yg + gbase + static_cast<long>(r) * sh.C, yv);
          // y, rounded to the I/O type as written, in place of v (this
          // thread's own slot, already read): the output projection's operand.
          if constexpr (WO) Io<T>::store8(v_s + r * CT + 8 * box_vec(pos.vec, r), yv);
        }
      });
    }

    // ---- output projection: z = y W_O^T ("entangled-state-attention 0.1.0",
    //      "Core idea": y_t = W_O (q_t (.) Norm(E_t))) ---------------------
    if constexpr (WO) {
      fence_proxy_async_smem();   // this thread's y stores, before the tensor cores read them
      tc_fence_before();
      named_sync(bar_all, Pl::NTG);
      if (tid == 0) {
        tc_fence_after();
        const uint32_t ya = smem_u32(v_s), woa = smem_u32(wo_s);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          umma_f16(tmem_d + static_cast<uint32_t>(3 * CT), umma_desc_sw128(ya) + 2 * kk,
                   umma_desc_sw128(woa) + 2 * kk, kIdescWO, kk != 0);
        umma_commit(&bar[2]);
      }
      mbar_wait_bounded(&bar[2], ph_o, &hdr->status);
      ph_o ^= 1u;
      tc_fence_after();
      __syncwarp();   // the tensor-memory loads below are warp-collective
      {
        const int wg = tid >> 5, lane = tid & 31;
        const int quad = wg & 3, half = wg >> 2;   // rows 32 quad + lane; outputs 32 half ..
        const int r = 32 * quad + lane;
        uint32_t acc[32];
        tmem_ld32(tmem_d + (static_cast<uint32_t>(32 * quad) << 16) + static_cast<uint32_t>(3 * CT + 32 * half), acc);
        tmem_wait_ld();
        uint4 out[4];
        pack32<T>(acc, out);
        if (t0 + r < sh.T) {
          uint4 *zp = reinterpret_cast<uint4 *>(static_cast<T *>(args.z) +
                                                (static_cast<long>(b) * sh.T + t0 + r) * 64 + 32 * half);
#pragma unroll
          for (int i = 0; i < 4; ++i) zp[i] = out[i];
        }
      }
      tc_fence_before();
    }
    try_issue_next();
    named_sync(bar_all, Pl::NTG);   // boxes, scratch and carries are free for the next tile
  }

  // ---- end: free tensor memory, count the CTA out ----------------------------
  // A CTA whose groups found no tile never waited for the weight slice; its
  // copy must have landed before the CTA's shared memory goes away, and so
  // must the groups' last projection stores.
  if (threadIdx.x == 0) mbar_wait_bounded(w_bar, 0u, &hdr->status);
  if (tid == 0) bulk_wait0();
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x < 32) {
    tc_fence_after();
    tmem_dealloc(tmem_base, Pl::NG * 256);
  }
  if (threadIdx.x == 0) {
    __threadfence();
    const unsigned prev = atomicAdd(&hdr->done[0], 1u);
    if (prev == gridDim.x * gridDim.y - 1) {
      __threadfence();
      for (int i = 0; i < sh.nct; ++i) hdr->ct_ticket[i] = 0u;
      hdr->done[0] = 0u;
      hdr->abort[0] = 0u;
      if (tag != 0u) {
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

}  // namespace esa
