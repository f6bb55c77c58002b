// esa_common.cuh -- device helpers shared by the ESA scan kernels (sm_100a).
//
// Contents: I/O vector loads/stores of 8 channels, the gate sigmoid, the
// per-tile workspace view, and thin inline-PTX wrappers for mbarriers, TMA
// tensor loads and acquire/release flag accesses.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <stdint.h>

namespace esa {

constexpr float kEps = 1e-6f;          // RMS-norm epsilon (inside the square root)

// Device status bits (sticky in the workspace header until esa_check).
constexpr unsigned kStatusTimeout = 1u;    // a bounded wait gave up
constexpr unsigned kStatusUninit = 2u;     // workspace not initialised (or epochs exhausted)

// Iteration cap of every device-side wait.  With the back-off below this is
// at most a second or two, far above any legitimate wait (microseconds).
constexpr unsigned kSpinLimit = 1u << 21;

// Marks an initialised workspace header.
constexpr unsigned long long kWorkspaceMagic = 0x45534153434e3031ull;

// ---------------------------------------------------------------------------
// Workspace.  A 256-byte header followed by per-chunk carry words.  Every
// time chunk of every sequence owns one "slot":
//   slot = chain * nchunks + chunk,  chain = b * nct + ct
// and per slot and channel:
//   incl_f  (E, tag)          forward state at the chunk's end; also the
//                             checkpoint the backward replays from
//   incl_b  (H, tag)          backward carry leaving the chunk (to earlier time)
//   agg     (P, tag), (S, tag) the chunk's affine carry map x -> P x + S
// Each word packs a float32 value with the 32-bit epoch of the call that wrote
// it, and is written with one single-copy-atomic 64-bit store, so a reader
// that sees the current epoch also sees the matching value: publication needs
// no fence and a look-back needs one round trip.  The epoch advances by one
// per scan call (the kernel's last CTA does it) and is never 0; init zeroes
// every word, so no stale word can carry a current tag.
// ---------------------------------------------------------------------------
constexpr int kMaxChannelTickets = 48;   // channel tiles of the fused projection + scan

struct WsHeader {
  unsigned long long magic;   // kWorkspaceMagic once initialised
  unsigned epoch;             // tag used by the next scan call
  unsigned status;            // sticky status bits
  unsigned ticket[2];         // tile ticket counters: [0] forward, [1] backward
  unsigned done[2];           // CTAs finished, per kernel
  unsigned abort[2];          // raised by a CTA whose wait gave up
  unsigned ct_ticket[kMaxChannelTickets];   // fused forward: one ticket counter per channel tile
};
static_assert(sizeof(WsHeader) <= 256, "the workspace header is 256 bytes");

struct Workspace {
  WsHeader *hdr;
  unsigned long long *incl_f;
  unsigned long long *incl_b;
  ulonglong2 *agg;
};

__device__ __forceinline__ unsigned long long pack_tag(float v, unsigned tag) {
  return (static_cast<unsigned long long>(tag) << 32) | __float_as_uint(v);
}
__device__ __forceinline__ unsigned tag_of(unsigned long long w) { return static_cast<unsigned>(w >> 32); }
__device__ __forceinline__ float val_of(unsigned long long w) {
  return __uint_as_float(static_cast<unsigned>(w));
}

// ---------------------------------------------------------------------------
// Packed float32 pairs.  sm_100 executes FADD2 / FMUL2 / FFMA2 on two fp32
// lanes per instruction, each lane rounded to nearest exactly like the
// scalar instruction, so packing halves the float32 instruction count without
// changing a single result bit.  A thread's 8 channels are 4 pairs (2i, 2i+1).
// nvcc may still fuse a packed multiply with a packed add that consumes it
// into one FFMA2 when both sit in one basic block (it did so across the rows
// of the backward's reverse phases once their per-row branches were removed),
// so values that must agree bit for bit between two code paths -- a tile's
// published carry and the look-back's recomposition of it -- are formed with
// explicit fused multiply-adds.
// ---------------------------------------------------------------------------
__device__ __forceinline__ float2 splat(float a) { return make_float2(a, a); }

__device__ __forceinline__ float2 add2(float2 a, float2 b) { return __fadd2_rn(a, b); }
__device__ __forceinline__ float2 sub2(float2 a, float2 b) {   // a - b: b * (-1) is exact, so one rounding
  return __ffma2_rn(b, make_float2(-1.0f, -1.0f), a);
}
__device__ __forceinline__ float2 mul2(float2 a, float2 b) { return __fmul2_rn(a, b); }
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }

// ---------------------------------------------------------------------------
// I/O element traits: 8 consecutive channels per thread, as 4 float2 pairs.
// load8_gate also clamps the gate logit at -80 (in the I/O type, one packed
// min/max per pair) so that exp(-x) stays finite.
// ---------------------------------------------------------------------------
template <typename T> struct Io;

// The output type of a scan whose inputs are T: the input type itself, except
// that fp8 (e4m3) inputs produce fp16 outputs.
template <typename T> struct OutOf { using type = T; };
template <> struct OutOf<__nv_fp8_e4m3> { using type = __half; };

template <> struct Io<float> {
  static __device__ __forceinline__ void load8(const float *p, float2 (&x)[4]) {
    const float4 u = reinterpret_cast<const float4 *>(p)[0];
    const float4 w = reinterpret_cast<const float4 *>(p)[1];
    x[0] = make_float2(u.x, u.y); x[1] = make_float2(u.z, u.w);
    x[2] = make_float2(w.x, w.y); x[3] = make_float2(w.z, w.w);
  }
  static __device__ __forceinline__ void load8_gate(const float *p, float2 (&x)[4]) {
    load8(p, x);
#pragma unroll
    for (int i = 0; i < 4; ++i) x[i] = make_float2(fmaxf(x[i].x, -80.0f), fmaxf(x[i].y, -80.0f));
  }
  static __device__ __forceinline__ void store8(float *p, const float2 (&x)[4]) {
    reinterpret_cast<float4 *>(p)[0] = make_float4(x[0].x, x[0].y, x[1].x, x[1].y);
    reinterpret_cast<float4 *>(p)[1] = make_float4(x[2].x, x[2].y, x[3].x, x[3].y);
  }
};

template <> struct Io<__half> {
  static __device__ __forceinline__ void load8(const __half *p, float2 (&x)[4]) {
    const uint4 u = *reinterpret_cast<const uint4 *>(p);
    const __half2 *h = reinterpret_cast<const __half2 *>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) x[i] = __half22float2(h[i]);
  }
  static __device__ __forceinline__ void load8_gate(const __half *p, float2 (&x)[4]) {
    const uint4 u = *reinterpret_cast<const uint4 *>(p);
    const __half2 *h = reinterpret_cast<const __half2 *>(&u);
    const __half2 lo = __float2half2_rn(-80.0f);
#pragma unroll
    for (int i = 0; i < 4; ++i) x[i] = __half22float2(__hmax2(h[i], lo));
  }
  static __device__ __forceinline__ void store8(__half *p, const float2 (&x)[4]) {
    uint4 u;
    __half2 *h = reinterpret_cast<__half2 *>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) h[i] = __float22half2_rn(x[i]);
    *reinterpret_cast<uint4 *>(p) = u;
  }
};

template <> struct Io<__nv_bfloat16> {
  static __device__ __forceinline__ void load8(const __nv_bfloat16 *p, float2 (&x)[4]) {
    const uint4 u = *reinterpret_cast<const uint4 *>(p);
    const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) x[i] = __bfloat1622float2(h[i]);
  }
  static __device__ __forceinline__ void load8_gate(const __nv_bfloat16 *p, float2 (&x)[4]) {
    const uint4 u = *reinterpret_cast<const uint4 *>(p);
    const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&u);
    const __nv_bfloat162 lo = __float2bfloat162_rn(-80.0f);
#pragma unroll
    for (int i = 0; i < 4; ++i) x[i] = __bfloat1622float2(__hmax2(h[i], lo));
  }
  static __device__ __forceinline__ void store8(__nv_bfloat16 *p, const float2 (&x)[4]) {
    uint4 u;
    __nv_bfloat162 *h = reinterpret_cast<__nv_bfloat162 *>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) h[i] = __float22bfloat162_rn(x[i]);
    *reinterpret_cast<uint4 *>(p) = u;
  }
};

// fp8 e4m3 inputs (forward scans only): 8 channels = 8 bytes; each byte pair
// is widened exactly to half precision, then to float.
template <> struct Io<__nv_fp8_e4m3> {
  static __device__ __forceinline__ __half2 h2(unsigned short pair) {
    const __half2_raw r = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(pair), __NV_E4M3);
    return __half2(r);
  }
  static __device__ __forceinline__ void load8(const __nv_fp8_e4m3 *p, float2 (&x)[4]) {
    const uint2 u = *reinterpret_cast<const uint2 *>(p);
    const unsigned short *w = reinterpret_cast<const unsigned short *>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) x[i] = __half22float2(h2(w[i]));
  }
  static __device__ __forceinline__ void load8_gate(const __nv_fp8_e4m3 *p, float2 (&x)[4]) {
    const uint2 u = *reinterpret_cast<const uint2 *>(p);
    const unsigned short *w = reinterpret_cast<const unsigned short *>(&u);
    const __half2 lo = __float2half2_rn(-80.0f);
#pragma unroll
    for (int i = 0; i < 4; ++i) x[i] = __half22float2(__hmax2(h2(w[i]), lo));
  }
};

// ---------------------------------------------------------------------------
// Approximate transcendental instructions (PTX ex2/rcp/rsqrt .approx.ftz).
// ---------------------------------------------------------------------------
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float rcp_approx(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float rsqrt_approx(float x) {
  float y;
  asm("rsqrt.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// ---------------------------------------------------------------------------
// Gate of a channel pair.  With u = exp(-x) = 2^(-x log2 e) (x already
// clamped at -80 so u stays finite):
//   A = 1 / (1 + u)      (the logistic sigmoid)
//   1 - A = u * A        (no cancellation when A is close to 1)
// ---------------------------------------------------------------------------
struct Gate2 {
  float2 A;    // sigmoid(x)
  float2 Ac;   // 1 - sigmoid(x)
};

constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ Gate2 gate2(float2 x) {
  const float2 t = mul2(x, splat(-kLog2e));
  const float2 u = make_float2(ex2_approx(t.x), ex2_approx(t.y));
  const float2 d = add2(u, splat(1.0f));
  const float2 A = make_float2(rcp_approx(d.x), rcp_approx(d.y));
  return Gate2{A, mul2(u, A)};
}

// Sum over the `LPH` adjacent lanes that hold one head (LPH a power of two).
template <int LPH>
__device__ __forceinline__ float head_sum(float s) {
#pragma unroll
  for (int o = 1; o < LPH; o <<= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  return s;
}

// ---------------------------------------------------------------------------
// Inline PTX: shared-memory addresses, mbarriers, TMA tensor loads, flags.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, unsigned count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t *bar, unsigned bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

// Wait on an mbarrier phase; the hardware may suspend the thread for up to
// about a microsecond (the hint) before returning false.
__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, unsigned phase) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(phase), "r"(1000u)
      : "memory");
  return ok != 0;
}

// 3-D tiled TMA load (no multicast): box at coordinates (x, y, z) of the
// tensor map into shared memory, completing on `bar`.
__device__ __forceinline__ void tma_load_3d(void *dst, const CUtensorMap *map, int x, int y, int z,
                                            uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap *map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

__device__ __forceinline__ unsigned long long ld_relaxed_b64(const unsigned long long *p) {
  unsigned long long v;
  asm volatile("ld.relaxed.gpu.global.b64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}

// Two independent 64-bit words (each single-copy atomic on its own).
__device__ __forceinline__ ulonglong2 ld_relaxed_v2b64(const ulonglong2 *p) {
  ulonglong2 v;
  asm volatile("ld.relaxed.gpu.global.v2.b64 {%0, %1}, [%2];" : "=l"(v.x), "=l"(v.y) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void st_relaxed_b64(unsigned long long *p, unsigned long long v) {
  asm volatile("st.relaxed.gpu.global.b64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

__device__ __forceinline__ void st_relaxed_v2b64(ulonglong2 *p, ulonglong2 v) {
  asm volatile("st.relaxed.gpu.global.v2.b64 [%0], {%1, %2};" ::"l"(p), "l"(v.x), "l"(v.y) : "memory");
}

__device__ __forceinline__ unsigned ld_relaxed(const unsigned *p) {
  unsigned v;
  asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}




// Wait for the TMA transaction on `bar` (given phase parity).  Bounded: on
// giving up it records a timeout in the status word and returns false.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t *bar, unsigned phase, unsigned *status) {
  for (unsigned it = 0; it < kSpinLimit; ++it)
    if (mbar_try_wait(bar, phase)) return true;
  atomicOr(status, kStatusTimeout);
  return false;
}

}  // namespace esa
