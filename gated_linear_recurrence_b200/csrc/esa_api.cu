// esa_api.cu -- the C ABI of the ESA scan library (declared in include/esa.h).
//
// Host responsibilities: argument and alignment checks (before anything is
// enqueued), the workspace layout, TMA tensor-map encoding, the per-call
// reset of the look-back flags, and kernel dispatch on the caller's stream.
#include <cudaTypedefs.h>

#include <atomic>
#include <climits>
#include <cstdint>
#include <cstddef>
#include <cstring>
#include <mutex>

#include "esa.h"
#include "esa_fused_launch.h"
#include "esa_launch.h"

namespace {

using esa::fwd_slots_per_tile;
using esa::tile_cols;
using esa::tile_rows;

constexpr int kVersion = 100;   // 0.1.0

bool supported_d(int D) {
  return D == 8 || D == 16 || D == 32 || D == 64 || D == 128 || D == 256;
}

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

size_t elem_bytes(int dtype) { return dtype == ESA_F32 ? 4 : dtype == ESA_E4M3 ? 1 : 2; }

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Workspace layout (byte offsets from the workspace base):
//   [0, 256)     header (esa::WsHeader: magic, epoch, status, per-kernel
//                ticket / done / abort words)
//   incl_f       n * CT  u64   forward chunk-end states (epoch-tagged)
//   incl_b       n * CT  u64   backward chunk carries (epoch-tagged)
//   agg          n * CT  2*u64 chunk maps (P, S), each word epoch-tagged
// with n = B * ceil(C / CT) * ceil(T / L) slots of L rows (L = tile_rows).
// The backward's tiles are one slot tall; a forward tile may span several.
struct Layout {
  int L = 0, CT = 0, nct = 0, nslots = 0, nchains = 0;
  long long ntiles = 0;   // nchains * nslots
  size_t incl_f_off = 0, incl_b_off = 0, agg_off = 0, total = 0;
};

constexpr size_t kHeaderBytes = 256;

bool make_layout(int B, int T, int H, int D, int dtype, Layout *lo) {
  if (B < 0 || T < 0 || H < 1 || D < 1) return false;
  if (dtype < ESA_F32 || dtype > ESA_E4M3) return false;
  if (!supported_d(D)) return false;
  const long long C = static_cast<long long>(H) * D;
  if (C > INT_MAX / 2) return false;
  lo->L = tile_rows(dtype);
  lo->CT = tile_cols(D);
  lo->nct = static_cast<int>((C + lo->CT - 1) / lo->CT);
  lo->nslots = (T + lo->L - 1) / lo->L;
  const long long nchains = static_cast<long long>(B) * lo->nct;
  if (nchains > INT_MAX) return false;
  lo->nchains = static_cast<int>(nchains);
  lo->ntiles = nchains * lo->nslots;
  if (lo->ntiles > INT_MAX) return false;
  const size_t words = static_cast<size_t>(lo->ntiles) * lo->CT;
  size_t off = kHeaderBytes;
  lo->incl_f_off = off;
  off = align_up(off + words * sizeof(unsigned long long), 256);
  lo->incl_b_off = off;
  off = align_up(off + words * sizeof(unsigned long long), 256);
  lo->agg_off = off;
  off = align_up(off + words * sizeof(ulonglong2), 256);
  lo->total = off;
  return true;
}

esa::Workspace workspace_view(void *base, const Layout &lo) {
  unsigned char *p = static_cast<unsigned char *>(base);
  esa::Workspace ws;
  ws.hdr = reinterpret_cast<esa::WsHeader *>(p);
  ws.incl_f = reinterpret_cast<unsigned long long *>(p + lo.incl_f_off);
  ws.incl_b = reinterpret_cast<unsigned long long *>(p + lo.incl_b_off);
  ws.agg = reinterpret_cast<ulonglong2 *>(p + lo.agg_off);
  return ws;
}

// The current device must be compute capability 10.0 (B200, sm_100a code).
int check_device() {
  static std::atomic<int> cache[64];   // 0 unknown, 1 ok, 2 unsupported
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) {
    cudaGetLastError();
    return ESA_ERR_DEVICE;
  }
  if (dev < 64) {
    const int c = cache[dev].load(std::memory_order_relaxed);
    if (c == 1) return ESA_OK;
    if (c == 2) return ESA_ERR_DEVICE;
  }
  int major = 0, minor = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) {
    cudaGetLastError();
    return ESA_ERR_DEVICE;
  }
  const bool ok = (major == 10 && minor == 0);
  if (dev < 64) cache[dev].store(ok ? 1 : 2, std::memory_order_relaxed);
  return ok ? ESA_OK : ESA_ERR_DEVICE;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    cudaGetLastError();
  });
  return fn;
}

// [B][T][C] tensor in the I/O dtype, read in boxes of [rows][CT channels];
// consecutive tokens' rows are `ld` elements apart (ld = C: contiguous).
int make_tmap(CUtensorMap *map, const void *ptr, int dtype, int B, int T, int C, const Layout &lo, int rows,
              long long ld = 0) {
  if (ld == 0) ld = C;
  auto fn = encode_fn();
  if (fn == nullptr) return ESA_ERR_LAUNCH;
  const CUtensorMapDataType dt = dtype == ESA_F32    ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                                 : dtype == ESA_F16  ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16
                                 : dtype == ESA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                                     : CU_TENSOR_MAP_DATA_TYPE_UINT8;   // e4m3 bytes
  const cuuint64_t s = elem_bytes(dtype);
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(C), static_cast<cuuint64_t>(T),
                              static_cast<cuuint64_t>(B)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(ld) * s,
                                 static_cast<cuuint64_t>(T) * static_cast<cuuint64_t>(ld) * s};
  const cuuint32_t box[3] = {static_cast<cuuint32_t>(lo.CT), static_cast<cuuint32_t>(rows), 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  std::memset(map, 0, sizeof(*map));
  // L2 promotion of 128 bytes, the row of a 64-channel 16-bit box: 256-byte
  // promotion was 2% slower on the fwd + bwd step (interleaved A/B on B200).
  const CUresult r = fn(map, dt, 3, const_cast<void *>(ptr), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? ESA_OK : ESA_ERR_LAUNCH;
}

// A 16-bit row-major matrix of `rank` 2 or 3 dimensions (innermost first),
// read in boxes of 64 elements (128 bytes) x box_rows with the 128-byte
// swizzle the tensor-core operands use.
int make_tmap_sw128(CUtensorMap *map, const void *ptr, int dtype, int rank, const cuuint64_t *dims,
                    cuuint32_t box_rows) {
  auto fn = encode_fn();
  if (fn == nullptr) return ESA_ERR_LAUNCH;
  const CUtensorMapDataType dt = dtype == ESA_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  cuuint64_t strides[2] = {dims[0] * 2, rank > 2 ? dims[0] * dims[1] * 2 : 0};
  const cuuint32_t box[3] = {64, box_rows, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  std::memset(map, 0, sizeof(*map));
  const CUresult r = fn(map, dt, static_cast<cuuint32_t>(rank), const_cast<void *>(ptr), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? ESA_OK : ESA_ERR_LAUNCH;
}

int check_shape(int B, int T, int H, int D, int mode, int dtype) {
  if (B < 0 || T < 0 || H < 1 || D < 1) return ESA_ERR_ARG;
  if (mode != ESA_DIRECT && mode != ESA_CONTROLLED) return ESA_ERR_ARG;
  if (dtype < ESA_F32 || dtype > ESA_E4M3) return ESA_ERR_ARG;
  if (!supported_d(D)) return ESA_ERR_UNSUPPORTED;
  if (static_cast<long long>(H) * D > INT_MAX / 2) return ESA_ERR_ARG;
  return ESA_OK;
}

// Shape of a scan whose tiles span `sub` slots each.
esa::ScanShape scan_shape(int B, int T, int H, int D, const Layout &lo, int sub) {
  esa::ScanShape s;
  s.B = B;
  s.T = T;
  s.C = H * D;
  s.nslots = lo.nslots;
  s.nchunks = (lo.nslots + sub - 1) / sub;
  s.nct = lo.nct;
  s.nchains = lo.nchains;
  s.ntiles = lo.nchains * s.nchunks;   // <= lo.ntiles, checked to fit an int
  s.inv_D = 1.0f / static_cast<float>(D);
  return s;
}

int rt(cudaError_t e) {
  if (e == cudaSuccess) return ESA_OK;
  cudaGetLastError();
  return ESA_ERR_LAUNCH;
}

// A row stride of `ld` elements of `bytes` each: at least C, a whole number
// of 16-byte units (TMA strides and the kernels' 16-byte stores), and small
// enough that T rows of a batch stay addressable.
int check_ld(long long ld, int C, size_t bytes, int T) {
  if (ld < C || ld > INT_MAX) return ESA_ERR_ARG;
  if ((static_cast<unsigned long long>(ld) * bytes) % 16u != 0) return ESA_ERR_ALIGN;
  if (static_cast<long double>(ld) * bytes * (T > 0 ? T : 1) > static_cast<long double>(1ull << 40))
    return ESA_ERR_ARG;
  return ESA_OK;
}

// Element size of the gradients and y: fp8 inputs give fp16 outputs.
size_t out_bytes(int dtype) { return dtype == ESA_E4M3 ? 2 : elem_bytes(dtype); }

int scan_fwd_impl(const void *a, const void *v, const void *q, long long ld_in, void *y, float *E_final, int B,
                  int T, int H, int D, int mode, const float *E_init, int dtype, void *workspace,
                  size_t workspace_bytes, void *stream);
int scan_bwd_impl(const void *a, const void *v, const void *q, long long ld_in, const void *dy,
                  const float *dE_final, void *da, void *dv, void *dq, long long ld_grad, float *dE_init, int B,
                  int T, int H, int D, int mode, const float *E_init, int dtype, void *workspace,
                  size_t workspace_bytes, void *stream);

// The fused forward, with (out = true) or without the output projection.
int fused_impl(const void *x, const void *W, const void *W_O, void *z, void *y, float *E_final, void *a, void *v,
               void *q, int B, int T, int H, int D, int C_in, int mode, const float *E_init, int dtype,
               void *workspace, size_t workspace_bytes, void *stream, bool out = false) {
  int rc = check_shape(B, T, H, D, mode, dtype);
  if (rc) return rc;
  if (C_in < 1) return ESA_ERR_ARG;
  Layout lo;
  if (!make_layout(B, T, H, D, dtype, &lo)) return ESA_ERR_ARG;
  if (!esa::fused_supported(dtype, D, C_in, lo.nct)) return ESA_ERR_UNSUPPORTED;
  const int C = H * D;
  if (out && !esa::fused_out_supported(dtype, C, C_in)) return ESA_ERR_UNSUPPORTED;
  const bool has_tokens = B > 0 && T > 0;
  if (has_tokens && (!x || !W || (!y && !out))) return ESA_ERR_ARG;
  if ((a == nullptr) != (v == nullptr) || (a == nullptr) != (q == nullptr)) return ESA_ERR_ARG;
  for (const void *p : {x, W, W_O, static_cast<const void *>(z), static_cast<const void *>(y),
                        static_cast<const void *>(E_final), static_cast<const void *>(a),
                        static_cast<const void *>(v), static_cast<const void *>(q),
                        static_cast<const void *>(E_init), static_cast<const void *>(workspace)})
    if (p && !aligned16(p)) return ESA_ERR_ALIGN;
  if (!workspace || workspace_bytes < lo.total) return ESA_ERR_WORKSPACE;
  if ((rc = check_device())) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (B == 0) return ESA_OK;
  if (T == 0) {
    if (!E_final) return ESA_OK;
    const size_t bytes = static_cast<size_t>(B) * C * sizeof(float);
    return E_init ? rt(cudaMemcpyAsync(E_final, E_init, bytes, cudaMemcpyDeviceToDevice, st))
                  : rt(cudaMemsetAsync(E_final, 0, bytes, st));
  }
  CUtensorMap tx, tw, two;
  const cuuint64_t xdims[3] = {static_cast<cuuint64_t>(C_in), static_cast<cuuint64_t>(T), static_cast<cuuint64_t>(B)};
  const cuuint64_t wdims[2] = {static_cast<cuuint64_t>(C_in), static_cast<cuuint64_t>(3) * C};
  if ((rc = make_tmap_sw128(&tx, x, dtype, 3, xdims, 128))) return rc;
  if ((rc = make_tmap_sw128(&tw, W, dtype, 2, wdims, 64))) return rc;
  if (out) {
    const cuuint64_t odims[2] = {static_cast<cuuint64_t>(C), static_cast<cuuint64_t>(C)};   // W_O [C_out = C][C]
    if ((rc = make_tmap_sw128(&two, W_O, dtype, 2, odims, 64))) return rc;
  }
  CUtensorMap tavq[3] = {tx, tx, tx};   // placeholders when the projections are not stored
  if (a != nullptr) {
    const cuuint64_t pdims[3] = {static_cast<cuuint64_t>(C), static_cast<cuuint64_t>(T), static_cast<cuuint64_t>(B)};
    const void *outs[3] = {a, v, q};
    for (int i = 0; i < 3; ++i)
      if ((rc = make_tmap_sw128(&tavq[i], outs[i], dtype, 3, pdims, 128))) return rc;
  }
  esa::FusedArgs args;
  args.s = scan_shape(B, T, H, D, lo, 2);
  args.ntiles_ct = B * args.s.nchunks;
  args.y = y;
  args.E_final = E_final;
  args.E_init = E_init;
  args.a_out = a;
  args.v_out = v;
  args.q_out = q;
  args.z = z;
  args.ws = workspace_view(workspace, lo);
  return esa::launch_fused_fwd(dtype, mode, D, C_in, tx, tw, tavq, out ? &two : nullptr, args, st);
}

}  // namespace

extern "C" {

size_t esa_workspace_size(int B, int T, int H, int D, int dtype) {
  Layout lo;
  if (!make_layout(B, T, H, D, dtype, &lo)) return 0;
  return lo.total;
}

int esa_scan_fwd(const void *a, const void *v, const void *q, void *y, float *E_final, int B, int T,
                 int H, int D, int mode, const float *E_init, int dtype, void *workspace,
                 size_t workspace_bytes, void *stream) {
  return scan_fwd_impl(a, v, q, 0, y, E_final, B, T, H, D, mode, E_init, dtype, workspace, workspace_bytes,
                       stream);
}

int esa_scan_fwd_ld(const void *a, const void *v, const void *q, long long ld_in, void *y, float *E_final, int B,
                    int T, int H, int D, int mode, const float *E_init, int dtype, void *workspace,
                    size_t workspace_bytes, void *stream) {
  if (ld_in <= 0) return ESA_ERR_ARG;
  return scan_fwd_impl(a, v, q, ld_in, y, E_final, B, T, H, D, mode, E_init, dtype, workspace, workspace_bytes,
                       stream);
}

int esa_scan_bwd_ld(const void *a, const void *v, const void *q, long long ld_in, const void *dy,
                    const float *dE_final, void *da, void *dv, void *dq, long long ld_grad, float *dE_init, int B,
                    int T, int H, int D, int mode, const float *E_init, int dtype, void *workspace,
                    size_t workspace_bytes, void *stream) {
  if (ld_in <= 0 || ld_grad <= 0) return ESA_ERR_ARG;
  return scan_bwd_impl(a, v, q, ld_in, dy, dE_final, da, dv, dq, ld_grad, dE_init, B, T, H, D, mode, E_init,
                       dtype, workspace, workspace_bytes, stream);
}

int esa_scan_bwd(const void *a, const void *v, const void *q, const void *dy, const float *dE_final,
                 void *da, void *dv, void *dq, float *dE_init, int B, int T, int H, int D, int mode,
                 const float *E_init, int dtype, void *workspace, size_t workspace_bytes, void *stream) {
  return scan_bwd_impl(a, v, q, 0, dy, dE_final, da, dv, dq, 0, dE_init, B, T, H, D, mode, E_init, dtype,
                       workspace, workspace_bytes, stream);
}

}  // extern "C"

namespace {

// ld_in / ld_grad = 0: contiguous rows (C elements apart).
int scan_fwd_impl(const void *a, const void *v, const void *q, long long ld_in, void *y, float *E_final, int B,
                  int T, int H, int D, int mode, const float *E_init, int dtype, void *workspace,
                  size_t workspace_bytes, void *stream) {
  int rc = check_shape(B, T, H, D, mode, dtype);
  if (rc) return rc;
  if (ld_in != 0 && (rc = check_ld(ld_in, H * D, elem_bytes(dtype), T))) return rc;
  const bool has_tokens = B > 0 && T > 0;   // empty tensors may carry NULL pointers
  if (has_tokens && (!a || !v || !q || !y)) return ESA_ERR_ARG;
  for (const void *p : {a, v, q, static_cast<const void *>(y), static_cast<const void *>(E_final),
                        static_cast<const void *>(E_init), static_cast<const void *>(workspace)})
    if (p && !aligned16(p)) return ESA_ERR_ALIGN;
  Layout lo;
  if (!make_layout(B, T, H, D, dtype, &lo)) return ESA_ERR_ARG;
  if (!workspace || workspace_bytes < lo.total) return ESA_ERR_WORKSPACE;
  if ((rc = check_device())) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int C = H * D;
  if (B == 0) return ESA_OK;
  if (T == 0) {   // no tokens: the final state is the initial one
    if (!E_final) return ESA_OK;
    const size_t bytes = static_cast<size_t>(B) * C * sizeof(float);
    return E_init ? rt(cudaMemcpyAsync(E_final, E_init, bytes, cudaMemcpyDeviceToDevice, st))
                  : rt(cudaMemsetAsync(E_final, 0, bytes, st));
  }
  const int sub = fwd_slots_per_tile(dtype, D);
  CUtensorMap ta, tv, tq;
  if ((rc = make_tmap(&ta, a, dtype, B, T, C, lo, lo.L * sub, ld_in))) return rc;
  if ((rc = make_tmap(&tv, v, dtype, B, T, C, lo, lo.L * sub, ld_in))) return rc;
  if ((rc = make_tmap(&tq, q, dtype, B, T, C, lo, lo.L * sub, ld_in))) return rc;
  esa::FwdArgs args;
  args.s = scan_shape(B, T, H, D, lo, sub);
  args.y = y;
  args.E_final = E_final;
  args.E_init = E_init;
  args.ws = workspace_view(workspace, lo);
  return esa::launch_fwd(dtype, mode, D, ta, tv, tq, args, args.s.ntiles, st);
}

int scan_bwd_impl(const void *a, const void *v, const void *q, long long ld_in, const void *dy,
                  const float *dE_final, void *da, void *dv, void *dq, long long ld_grad, float *dE_init, int B,
                  int T, int H, int D, int mode, const float *E_init, int dtype, void *workspace,
                  size_t workspace_bytes, void *stream) {
  int rc = check_shape(B, T, H, D, mode, dtype);
  if (rc) return rc;
  if (ld_in != 0 && (rc = check_ld(ld_in, H * D, elem_bytes(dtype), T))) return rc;
  if (ld_grad != 0 && (rc = check_ld(ld_grad, H * D, out_bytes(dtype), T))) return rc;
  const bool has_tokens = B > 0 && T > 0;   // empty tensors may carry NULL pointers
  if (has_tokens && (!a || !v || !q || !dy || !da || !dv || !dq)) return ESA_ERR_ARG;
  for (const void *p : {a, v, q, dy, static_cast<const void *>(dE_final), static_cast<const void *>(da),
                        static_cast<const void *>(dv), static_cast<const void *>(dq),
                        static_cast<const void *>(dE_init), static_cast<const void *>(E_init),
                        static_cast<const void *>(workspace)})
    if (p && !aligned16(p)) return ESA_ERR_ALIGN;
  Layout lo;
  if (!make_layout(B, T, H, D, dtype, &lo)) return ESA_ERR_ARG;
  if (!workspace || workspace_bytes < lo.total) return ESA_ERR_WORKSPACE;
  if ((rc = check_device())) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int C = H * D;
  if (B == 0) return ESA_OK;
  if (T == 0) {   // no tokens: the gradient passes straight through
    if (!dE_init) return ESA_OK;
    const size_t bytes = static_cast<size_t>(B) * C * sizeof(float);
    return dE_final ? rt(cudaMemcpyAsync(dE_init, dE_final, bytes, cudaMemcpyDeviceToDevice, st))
                    : rt(cudaMemsetAsync(dE_init, 0, bytes, st));
  }
  const int sub = esa::bwd_slots_per_tile(dtype, D);
  CUtensorMap ta, tv, tq, tdy;
  if ((rc = make_tmap(&ta, a, dtype, B, T, C, lo, lo.L * sub, ld_in))) return rc;
  if ((rc = make_tmap(&tv, v, dtype, B, T, C, lo, lo.L * sub, ld_in))) return rc;
  if ((rc = make_tmap(&tq, q, dtype, B, T, C, lo, lo.L * sub, ld_in))) return rc;
  if ((rc = make_tmap(&tdy, dy, dtype, B, T, C, lo, lo.L * sub))) return rc;
  esa::BwdArgs args;
  args.s = scan_shape(B, T, H, D, lo, sub);
  args.da = da;
  args.dv = dv;
  args.dq = dq;
  args.ldg = ld_grad != 0 ? ld_grad : C;
  args.dE_final = dE_final;
  args.dE_init = dE_init;
  args.E_init = E_init;
  args.ws = workspace_view(workspace, lo);
  return esa::launch_bwd(dtype, mode, D, ta, tv, tq, tdy, args, args.s.ntiles, st);
}

}  // namespace

extern "C" {

int esa_scan_map(const void *a, const void *v, float *P, float *S, int B, int T, int H, int D, int mode,
                 int dtype, void *workspace, size_t workspace_bytes, void *stream) {
  int rc = check_shape(B, T, H, D, mode, dtype);
  if (rc) return rc;
  if (B > 0 && (!P || !S)) return ESA_ERR_ARG;
  if (B > 0 && T > 0 && (!a || !v)) return ESA_ERR_ARG;
  for (const void *p : {a, v, static_cast<const void *>(P), static_cast<const void *>(S),
                        static_cast<const void *>(workspace)})
    if (p && !aligned16(p)) return ESA_ERR_ALIGN;
  Layout lo;
  if (!make_layout(B, T, H, D, dtype, &lo)) return ESA_ERR_ARG;
  if (!workspace || workspace_bytes < lo.total) return ESA_ERR_WORKSPACE;
  if ((rc = check_device())) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (B == 0) return ESA_OK;
  const int C = H * D;
  const int sub = fwd_slots_per_tile(dtype, D);
  esa::FwdArgs args;
  args.s = scan_shape(B, T, H, D, lo, sub);
  args.y = nullptr;
  args.E_final = nullptr;
  args.E_init = nullptr;
  args.ws = workspace_view(workspace, lo);
  if (T > 0) {   // T = 0: no tiles, the fold writes the identity map
    CUtensorMap ta, tv;
    if ((rc = make_tmap(&ta, a, dtype, B, T, C, lo, lo.L * sub))) return rc;
    if ((rc = make_tmap(&tv, v, dtype, B, T, C, lo, lo.L * sub))) return rc;
    if ((rc = esa::launch_fwd_map(dtype, mode, D, ta, tv, ta, args, args.s.ntiles, st))) return rc;
  }
  return esa::launch_map_fold(lo.CT, args.ws, args.s, sub, 0, P, S, st);
}

int esa_scan_bwd_map(const void *a, const void *v, const void *q, const void *dy, float *P, float *S, int B,
                     int T, int H, int D, int mode, const float *E_init, int dtype, void *workspace,
                     size_t workspace_bytes, void *stream) {
  int rc = check_shape(B, T, H, D, mode, dtype);
  if (rc) return rc;
  if (B > 0 && (!P || !S)) return ESA_ERR_ARG;
  if (B > 0 && T > 0 && (!a || !v || !q || !dy)) return ESA_ERR_ARG;
  for (const void *p : {a, v, q, dy, static_cast<const void *>(P), static_cast<const void *>(S),
                        static_cast<const void *>(E_init), static_cast<const void *>(workspace)})
    if (p && !aligned16(p)) return ESA_ERR_ALIGN;
  Layout lo;
  if (!make_layout(B, T, H, D, dtype, &lo)) return ESA_ERR_ARG;
  if (!workspace || workspace_bytes < lo.total) return ESA_ERR_WORKSPACE;
  if ((rc = check_device())) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (B == 0) return ESA_OK;
  const int C = H * D;
  const int sub = esa::bwd_slots_per_tile(dtype, D);
  esa::BwdArgs args;
  args.s = scan_shape(B, T, H, D, lo, sub);
  args.da = args.dv = args.dq = nullptr;
  args.ldg = C;
  args.dE_final = nullptr;
  args.dE_init = nullptr;
  args.E_init = E_init;
  args.ws = workspace_view(workspace, lo);
  if (T > 0) {
    CUtensorMap ta, tv, tq, tdy;
    if ((rc = make_tmap(&ta, a, dtype, B, T, C, lo, lo.L * sub))) return rc;
    if ((rc = make_tmap(&tv, v, dtype, B, T, C, lo, lo.L * sub))) return rc;
    if ((rc = make_tmap(&tq, q, dtype, B, T, C, lo, lo.L * sub))) return rc;
    if ((rc = make_tmap(&tdy, dy, dtype, B, T, C, lo, lo.L * sub))) return rc;
    if ((rc = esa::launch_bwd_map(dtype, mode, D, ta, tv, tq, tdy, args, args.s.ntiles, st))) return rc;
  }
  return esa::launch_map_fold(lo.CT, args.ws, args.s, sub, 1, P, S, st);
}

int esa_compose(const float *P, const float *S, int n, long long count, int reverse, const float *x0, float *x,
                void *stream) {
  if (n < 0 || count < 0 || (reverse != 0 && reverse != 1)) return ESA_ERR_ARG;
  if (count > 0 && (!x || (n > 0 && (!P || !S)))) return ESA_ERR_ARG;
  if (static_cast<long long>(n) * count > LLONG_MAX / 8) return ESA_ERR_ARG;
  for (const void *p : {static_cast<const void *>(P), static_cast<const void *>(S), static_cast<const void *>(x0),
                        static_cast<const void *>(x)})
    if (p && !aligned16(p)) return ESA_ERR_ALIGN;
  int rc = check_device();
  if (rc) return rc;
  return esa::launch_compose(P, S, n, static_cast<long>(count), reverse, x0, x, static_cast<cudaStream_t>(stream));
}

int esa_fused_fwd(const void *x, const void *W, void *y, float *E_final, void *a, void *v, void *q, int B, int T,
                  int H, int D, int C_in, int mode, const float *E_init, int dtype, void *workspace,
                  size_t workspace_bytes, void *stream) {
  return fused_impl(x, W, nullptr, nullptr, y, E_final, a, v, q, B, T, H, D, C_in, mode, E_init, dtype, workspace,
                    workspace_bytes, stream);
}

int esa_fused_layer_fwd(const void *x, const void *W, const void *W_O, void *z, void *y, float *E_final, int B,
                        int T, int H, int D, int C_in, int mode, const float *E_init, int dtype, void *workspace,
                        size_t workspace_bytes, void *stream) {
  if (B > 0 && T > 0 && (!W_O || !z)) return ESA_ERR_ARG;
  return fused_impl(x, W, W_O ? W_O : W, z, y, E_final, nullptr, nullptr, nullptr, B, T, H, D, C_in, mode, E_init,
                    dtype, workspace, workspace_bytes, stream, true);
}

int esa_step(const void *a_t, const void *v_t, const void *q_t, float *E, void *y_t, int B, int H, int D,
             int mode, int dtype, void *stream) {
  int rc = check_shape(B, 1, H, D, mode, dtype);
  if (rc) return rc;
  if (B > 0 && (!a_t || !v_t || !q_t || !E || !y_t)) return ESA_ERR_ARG;
  for (const void *p : {a_t, v_t, q_t, static_cast<const void *>(E), static_cast<const void *>(y_t)})
    if (p && !aligned16(p)) return ESA_ERR_ALIGN;
  if ((rc = check_device())) return rc;
  if (B == 0) return ESA_OK;
  const long nvec = static_cast<long>(B) * H * D / 8;
  return esa::launch_step(dtype, mode, D, a_t, v_t, q_t, E, y_t, nvec, 1.0f / static_cast<float>(D),
                          static_cast<cudaStream_t>(stream));
}

int esa_check(void *workspace, void *stream) {
  if (!workspace) return ESA_ERR_ARG;
  if (!aligned16(workspace)) return ESA_ERR_ALIGN;
  int rc = check_device();
  if (rc) return rc;
  if ((rc = rt(cudaStreamSynchronize(static_cast<cudaStream_t>(stream))))) return rc;
  esa::WsHeader h;
  if ((rc = rt(cudaMemcpy(&h, workspace, sizeof(h), cudaMemcpyDeviceToHost)))) return rc;
  const unsigned status = h.status;
  if (status != 0) {
    unsigned char *st_word = static_cast<unsigned char *>(workspace) + offsetof(esa::WsHeader, status);
    if ((rc = rt(cudaMemset(st_word, 0, sizeof(unsigned))))) return rc;
  }
  if (h.magic != esa::kWorkspaceMagic || (status & esa::kStatusUninit)) return ESA_ERR_WORKSPACE;
  if (status & esa::kStatusTimeout) return ESA_ERR_TIMEOUT;
  return ESA_OK;
}

int esa_workspace_init(void *workspace, size_t workspace_bytes, void *stream) {
  if (!workspace) return ESA_ERR_ARG;
  if (!aligned16(workspace)) return ESA_ERR_ALIGN;
  if (workspace_bytes < kHeaderBytes) return ESA_ERR_WORKSPACE;
  int rc = check_device();
  if (rc) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if ((rc = rt(cudaMemsetAsync(workspace, 0, workspace_bytes, st)))) return rc;
  return esa::launch_ws_init(static_cast<esa::WsHeader *>(workspace), st);
}

const char *esa_strerror(int status) {
  switch (status) {
    case ESA_OK: return "ok";
    case ESA_ERR_ARG: return "invalid argument (size, mode, dtype or a required NULL pointer)";
    case ESA_ERR_ALIGN: return "a pointer is not 16-byte aligned";
    case ESA_ERR_UNSUPPORTED: return "head dimension D must be one of 8, 16, 32, 64, 128, 256";
    case ESA_ERR_WORKSPACE: return "workspace missing or smaller than esa_workspace_size()";
    case ESA_ERR_LAUNCH: return "the CUDA runtime rejected a launch, copy or tensor map";
    case ESA_ERR_TIMEOUT: return "a bounded device-side wait gave up; outputs of the call are invalid";
    case ESA_ERR_DEVICE: return "no CUDA device, or the current device is not sm_100 (B200)";
    case ESA_ERR_NOALLOC_LIMIT:
      return "esa_scan_fwd_noalloc: the shape needs more scratch than the built-in 64 MiB array";
    default: return "unknown esa status";
  }
}

int esa_version(void) { return kVersion; }

}  // extern "C"
