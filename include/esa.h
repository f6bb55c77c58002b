/*
 * esa.h -- C ABI of the B200 (sm_100a) ESA scan library.
 *
 * The library evaluates the gated linear recurrence of Entangled State
 * Attention (ESA),
 *
 *     E_t = A_t (.) E_{t-1} + B_t,      A_t = sigmoid(a_t),
 *     B_t = v_t                  (direct mode),
 *     B_t = (1 - A_t) (.) v_t    (controlled mode),
 *     y_t = q_t (.) E_t / sqrt(mean_d(E_t^2) + 1e-6)   (per-head RMS readout),
 *
 * for every (batch, head, channel), as a chunked associative prefix scan over
 * time on the GPU, together with its backward pass and the one-token decode
 * update.  Sources: the recurrence is stated in "Entangled State Attention
 * v2.1" (entangled_state_attention-2.1.0 PKG-INFO, opening section) and in
 * the "Core recurrence" panel of mlbricks-web.pages.dev/esa; the direct and
 * controlled modes and the readout y_t = W_O(q_t (.) Norm(E_t)) are in
 * "entangled-state-attention 0.1.0" (PyPI), section "Core idea".  Norm is
 * left open there and is fixed here as an RMS over the D channels of a head,
 * eps = 1e-6 inside the square root, no learned scale.  The projections
 * (x W_A, x W_V, x W_Q, W_O) are not part of this library: a, v, q are their
 * outputs (a is the gate logit, before the sigmoid) and y is q (.) Norm(E).
 *
 * Conventions shared by every entry point:
 *   - All pointers are DEVICE pointers owned by the caller; the library never
 *     allocates, frees or retains them.  Every pointer must be 16-byte
 *     aligned.  Optional pointers may be NULL where stated.
 *   - Sequence tensors (a, v, q, y, dy, da, dv, dq) are contiguous
 *     [B, T, H, D] in the I/O dtype; state tensors (E_init, E_final, E,
 *     dE_final, dE_init) are contiguous [B, H, D] in float32.  C = H * D.
 *   - dtype is one of esa_dtype; all arithmetic and the state are float32,
 *     outputs are rounded to the I/O dtype with round-to-nearest-even (fp16
 *     for ESA_E4M3 inputs).  Calls that do not take ESA_E4M3 return
 *     ESA_ERR_UNSUPPORTED for it.
 *   - D must be one of 8, 16, 32, 64, 128, 256; H >= 1; B >= 0; T >= 0.
 *   - stream is a cudaStream_t passed as void* (NULL = the legacy default
 *     stream).  Every call only enqueues work and returns; it does not
 *     synchronise.  Calls that share a workspace must be ordered (same
 *     stream, or events) and must not overlap.
 *   - Return value: ESA_OK (0) or a negative esa_status.  Argument errors are
 *     detected on the host before anything is enqueued.  A device-side
 *     failure (a bounded wait that gave up) is recorded in the workspace and
 *     reported by esa_check().
 */
#ifndef ESA_H_
#define ESA_H_

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Recurrence mode ("entangled-state-attention 0.1.0", "Direct vs controlled mode"). */
typedef enum { ESA_DIRECT = 0, ESA_CONTROLLED = 1 } esa_mode;

/* I/O element type of the sequence tensors.  ESA_E4M3: the sequence inputs
 * (a, v, q, and dy for the backward) in fp8 e4m3 (1 sign, 4 exponent,
 * 3 mantissa bits, finite, largest 448) and the sequence outputs (y, da, dv,
 * dq, y_t) in fp16; accepted by every call but esa_fused_fwd.  "Entangled State Attention v2.1" lists fp8 as an
 * experimental precision mode. */
typedef enum { ESA_F32 = 0, ESA_F16 = 1, ESA_BF16 = 2, ESA_E4M3 = 3 } esa_dtype;

typedef enum {
    ESA_OK = 0,
    ESA_ERR_ARG = -1,         /* bad size, mode, dtype or a required NULL pointer */
    ESA_ERR_ALIGN = -2,       /* a pointer is not 16-byte aligned */
    ESA_ERR_UNSUPPORTED = -3, /* head dimension D outside {8,16,32,64,128,256} */
    ESA_ERR_WORKSPACE = -4,   /* workspace NULL, too small, or not initialised (esa_workspace_init) */
    ESA_ERR_LAUNCH = -5,      /* the CUDA runtime rejected a launch or copy */
    ESA_ERR_TIMEOUT = -6,     /* a bounded device-side wait gave up (see esa_check) */
    ESA_ERR_DEVICE = -7,      /* no CUDA device, or the current device is not sm_100 */
    ESA_ERR_NOALLOC_LIMIT = -8 /* esa_scan_fwd_noalloc: the shape needs more scratch than
                                  ESA_NOALLOC_SCRATCH_BYTES */
} esa_status;

/*
 * Bytes of device workspace that esa_scan_fwd / esa_scan_bwd need for a
 * problem of this shape and dtype (0 on a bad argument).  The workspace
 * holds a 256-byte header, the float32 state at the end of every time chunk
 * of every sequence (written by the forward, read by the backward as its
 * replay checkpoints) and the per-chunk carry words of the single-pass scan,
 * each tagged with the epoch of the call that wrote it.  That is
 * 256 + 32 * B * ceil(C / CT) * CT * ceil(T / L) bytes (rounded up to 256 B
 * per array), with L = 64 time steps per chunk for 16-bit I/O and 32 for
 * float32, and CT = 64 channels per tile (CT = D when D is 128 or 256).
 */
size_t esa_workspace_size(int B, int T, int H, int D, int dtype);

/*
 * Prepare a workspace for use: zero all `workspace_bytes` and write its
 * header (enqueued on `stream`).  Call once after allocating the buffer,
 * before its first scan; the buffer can then be reused by any number of scan
 * calls of any shape whose esa_workspace_size() fits in it.  Scans advance a
 * 32-bit epoch stored in the header; after 2^32 - 1 scan calls the header is
 * invalidated and esa_check() reports ESA_ERR_WORKSPACE until the workspace
 * is initialised again.  A scan given a workspace that was never initialised
 * does no work and esa_check() reports ESA_ERR_WORKSPACE.
 */
int esa_workspace_init(void *workspace, size_t workspace_bytes, void *stream);

/*
 * Forward scan (prefill / training forward).  The stages of the scan:
 * gate sigmoid, chunk-local scan, carry between chunks, readout -- all in
 * one kernel launch, without a separate reset launch.
 *   a, v, q   [B,T,H,D] inputs: gate logits, values, queries (required).
 *   y         [B,T,H,D] output: q (.) E_t / rms(E_t) (required).
 *   E_final   [B,H,D] float32 output: E_T, the state to continue decoding
 *             from (NULL = not written).  With T = 0 it equals E_init.
 *   E_init    [B,H,D] float32 initial state E_0 (NULL = zeros).
 *   workspace device buffer of at least esa_workspace_size() bytes,
 *             initialised once with esa_workspace_init.  After the call it
 *             holds the chunk-boundary states that esa_scan_bwd needs, so
 *             run no other forward on it before the matching backward.
 * Sources: state recurrence and modes ("entangled-state-attention 0.1.0",
 * "Core idea"); prefill returning the state (mlbricks-web.pages.dev/esa,
 * Quick start: prefill returns (out, state)).
 */
int esa_scan_fwd(const void *a, const void *v, const void *q, void *y, float *E_final,
                 int B, int T, int H, int D, int mode, const float *E_init,
                 int dtype, void *workspace, size_t workspace_bytes, void *stream);

/*
 * Backward scan: gradients of  sum(dy . y) + sum(dE_final . E_final)
 * with respect to a, v, q and E_init.
 *   a, v, q, E_init  exactly the forward's inputs (E_init NULL = zeros).
 *   dy        [B,T,H,D] upstream gradient of y (required).
 *   dE_final  [B,H,D] float32 upstream gradient of E_final (NULL = zeros).
 *   da, dv, dq [B,T,H,D] outputs in the I/O dtype (required).
 *   dE_init   [B,H,D] float32 output (NULL = not written).
 *   workspace the buffer the matching esa_scan_fwd wrote, unchanged since;
 *             the chunk-boundary states in it are read, the rest is scratch.
 * The pages do not print the backward; it is the chain rule of the forward
 * (training through the layer with loss.backward(), "Entangled State
 * Attention v2.1", section 9 "Continue training a loaded model"):
 *   G_t = ghat_t + A_{t+1} G_{t+1}, G_T = ghat_T + dE_final,
 *   ghat_t = r (dn - n mean_d(dn n)), n = E r, dn = dy q, dq = dy n,
 *   direct: dv = G, da = G E_{t-1} A(1-A);
 *   controlled: dv = G (1-A), da = G (E_{t-1} - v) A(1-A);  dE_init = A_1 G_1.
 */
int esa_scan_bwd(const void *a, const void *v, const void *q, const void *dy,
                 const float *dE_final, void *da, void *dv, void *dq, float *dE_init,
                 int B, int T, int H, int D, int mode, const float *E_init,
                 int dtype, void *workspace, size_t workspace_bytes, void *stream);

/*
 * The two scans on token rows with a stride, so that a, v, q can be column
 * blocks of one projection output [B,T,ld_in] (e.g. ld_in = 3C, a at column
 * 0, v at C, q at 2C) and da, dv, dq column blocks of one gradient buffer
 * [B,T,ld_grad], which the projections' backward then multiplies in a
 * single GEMM.  Element (b, t, c) of a, v, q (and of a gradient) is at
 * ptr[(b T + t) ld + c].  y and dy stay contiguous [B,T,H,D].
 *   ld_in     row stride of a, v, q, in elements: >= C, and ld_in times the
 *             element size a multiple of 16 bytes (else ESA_ERR_ARG /
 *             ESA_ERR_ALIGN).
 *   ld_grad   row stride of da, dv, dq, in elements of the output type (fp16
 *             for ESA_E4M3): the same rules.  Their rows must not overlap.
 * Every other argument, the results and the workspace rules are those of
 * esa_scan_fwd / esa_scan_bwd, which are these calls with ld_in = ld_grad = C.
 */
int esa_scan_fwd_ld(const void *a, const void *v, const void *q, long long ld_in, void *y, float *E_final,
                    int B, int T, int H, int D, int mode, const float *E_init,
                    int dtype, void *workspace, size_t workspace_bytes, void *stream);
int esa_scan_bwd_ld(const void *a, const void *v, const void *q, long long ld_in, const void *dy,
                    const float *dE_final, void *da, void *dv, void *dq, long long ld_grad, float *dE_init,
                    int B, int T, int H, int D, int mode, const float *E_init,
                    int dtype, void *workspace, size_t workspace_bytes, void *stream);

/*
 * Forward scan that allocates nothing.  The pages have no counterpart of this
 * entry point; it exists for callers that cannot allocate device memory at
 * the point where they run the scan -- serving loops whose device-memory
 * budget is fixed at start-up, latency-critical paths where cudaMalloc may
 * implicitly synchronise the device, and foreign-language callers that are
 * only handed tensor pointers and own no device allocator.
 *
 * Same arguments and results as esa_scan_fwd, minus the workspace: the
 * scratch lives in a static device array of ESA_NOALLOC_SCRATCH_BYTES
 * (64 MiB) inside the library, which every GPU that loads this part of the
 * library holds until the process exits.
 *   - A shape whose esa_workspace_size() exceeds ESA_NOALLOC_SCRATCH_BYTES is
 *     rejected with ESA_ERR_NOALLOC_LIMIT before anything is enqueued (for
 *     example B=64, T=8192, C=128 in 16-bit I/O needs 33.6 MB and fits).
 *     Other argument errors are reported as by esa_scan_fwd, also before
 *     anything is enqueued.
 *   - The first call on a device looks up the array's device address with
 *     that device current (once per device); make that first call before any
 *     stream capture.  A cudaDeviceReset() invalidates the looked-up address:
 *     do not use this entry point on a device after resetting it.
 *   - Each call enqueues two kernels on `stream`: a one-block guard, then the
 *     scan.  The guard initialises the array the first time it is used on a
 *     device, and clears it and starts its call counter (the 32-bit epoch
 *     that tags the chunk carries) afresh every 2^32 - 256 calls, so the
 *     counter never runs out.  Those two cases take a fraction of a
 *     millisecond; otherwise the guard only reads the array's header.
 *   - All calls share the one array, which keeps the last call's contents
 *     (the carries are tagged with the call's epoch, so nothing needs clearing
 *     between calls).  Calls whose executions overlap on the GPU, from any
 *     stream or thread, race on it: order them.  The chunk-end states it holds
 *     are not kept for a backward pass.
 *   - Device-side failures (a bounded wait inside the scan that gave up) are
 *     recorded in the array and reported by esa_check_noalloc().
 */
#define ESA_NOALLOC_SCRATCH_BYTES (64u * 1024u * 1024u)
int esa_scan_fwd_noalloc(const void *a, const void *v, const void *q, void *y, float *E_final,
                         int B, int T, int H, int D, int mode, const float *E_init,
                         int dtype, void *stream);

/*
 * Status of esa_scan_fwd_noalloc on the current device (no counterpart on the
 * pages): synchronise `stream`, then read and clear the status recorded in
 * the built-in array.  Returns ESA_OK (also when no call has used the array
 * on this device yet), ESA_ERR_TIMEOUT if a bounded wait inside one of its
 * scans gave up since the last check (that call's outputs are invalid), or
 * ESA_ERR_LAUNCH if the stream reports a CUDA error.  Allocates nothing.
 */
int esa_check_noalloc(void *stream);

/*
 * Device address and size of the built-in array of esa_scan_fwd_noalloc on
 * the current device (no counterpart on the pages), for inspection and
 * tests: its first 256 bytes are the header esa_check reads, the rest the
 * chunk carries.  Looks the address up if no call has done so yet (with the
 * device current); `bytes` may be NULL.  Writing to the array other than
 * through this library's calls leaves the results of later calls undefined.
 */
int esa_noalloc_scratch(void **device_ptr, size_t *bytes);

/*
 * Segment maps, for splitting one sequence over several GPUs along time
 * (context parallelism).  mlbricks-web.pages.dev/esa, opening panel
 * "Long-context throughput": the state composition is associative, which is
 * what gives a parallel path over the full sequence; here it is applied
 * across devices.  Over the T steps of one call, every channel's state is an
 * affine function of the state entering it, and the backward's carry is an
 * affine function of the gradient leaving it:
 *     E_T      = P (.) E_0      + S_fwd,     P = prod_{t=1..T} A_t,
 *     dE_init  = P (.) dE_final + S_bwd.
 * A time slice can therefore publish (P, S) -- 2 B C floats -- and find its
 * own boundary state from the maps of the slices before it (esa_compose),
 * instead of waiting for them to finish their scans.
 *
 * esa_scan_map: the forward map of one slice.
 *   a, v      [B,T,H,D] gate logits and values (q is not needed).
 *   P, S      [B,H,D] float32 outputs: P = prod A_t, S = E_T from E_0 = 0.
 *             With T = 0: P = 1, S = 0.
 *   workspace as for esa_scan_fwd.  Only its chunk-map words are written:
 *             chunk states that an earlier esa_scan_fwd left there for its
 *             backward are kept.  Two launches (tile maps, then their fold);
 *             no output of size T.
 */
int esa_scan_map(const void *a, const void *v, float *P, float *S, int B, int T, int H, int D, int mode,
                 int dtype, void *workspace, size_t workspace_bytes, void *stream);

/*
 * esa_scan_bwd_map: the backward (reverse) map of one slice.
 *   a, v, q, dy, E_init  as for esa_scan_bwd (E_init: the slice's true
 *             initial state, NULL = zeros).
 *   P, S      [B,H,D] float32 outputs: dE_init = P (.) dE_final + S for any
 *             dE_final; P = prod A_t, S = dE_init for dE_final = 0.
 *   workspace the buffer of the matching esa_scan_fwd (same inputs, same
 *             E_init), unchanged since: its chunk states are read and kept,
 *             so esa_scan_bwd can follow on the same workspace.
 */
int esa_scan_bwd_map(const void *a, const void *v, const void *q, const void *dy, float *P, float *S, int B,
                     int T, int H, int D, int mode, const float *E_init, int dtype, void *workspace,
                     size_t workspace_bytes, void *stream);

/*
 * esa_compose: apply n segment maps in sequence to `count` values,
 *     x = map_{n-1}( ... map_0(x0) ),   map_j(x) = P_j (.) x + S_j,
 * with maps in index order (reverse = 0, forward: earliest slice first) or
 * from index n - 1 down to 0 (reverse = 1, backward: latest slice first).
 *   P, S      [n, count] float32 (may be NULL when n = 0).
 *   x0        [count] float32 start value (NULL = zeros).
 *   x         [count] float32 output; may alias x0.
 * Each value is folded with float32 fused multiply-adds in map order.
 */
int esa_compose(const float *P, const float *S, int n, long long count, int reverse, const float *x0, float *x,
                void *stream);

/*
 * Forward scan with the input projections fused in (inference / prefill of
 * the ESA layer).  "entangled-state-attention 0.1.0", section "Core idea":
 * the layer's gate logits, values and queries are projections of its input,
 * a = x W_A^T, v = x W_V^T, q = x W_Q^T; this call computes them on the
 * tensor cores tile by tile, rounds them to the I/O dtype (the values an
 * unfused projection writes) and runs the forward scan on them without
 * writing them to memory.  Results equal esa_scan_fwd on those a, v, q.
 *   x         [B,T,C_in] layer input, I/O dtype (required).
 *   W         [3C, C_in] the three projection weights stacked (rows 0..C-1:
 *             W_A, C..2C-1: W_V, 2C..3C-1: W_Q), each [out, in] as stored by
 *             a linear layer, I/O dtype (required).
 *   a, v, q   [B,T,H,D] outputs (optional, all NULL or none): the rounded
 *             projections the scan consumed.  With them written, the call
 *             is a complete training forward: esa_scan_bwd(a, v, q, ...) on
 *             the same workspace gives the scan's gradients.  Without them
 *             the call only reads x and W and writes y (inference, prefill).
 *   y, E_final, E_init, mode, workspace: as for esa_scan_fwd.
 * Supported: dtype ESA_F16 or ESA_BF16, D <= 64, C_in of 64, 128 or 256, C <= 3072;
 * other shapes return ESA_ERR_UNSUPPORTED (compute the projections
 * separately and call esa_scan_fwd).
 */
int esa_fused_fwd(const void *x, const void *W, void *y, float *E_final, void *a, void *v, void *q, int B, int T,
                  int H, int D, int C_in, int mode, const float *E_init, int dtype, void *workspace,
                  size_t workspace_bytes, void *stream);

/*
 * The ESA layer's whole forward from its input for a layer of C = H * D = 64
 * channels: the fused projections and scan of esa_fused_fwd followed by the
 * output projection ("entangled-state-attention 0.1.0", section "Core idea":
 * y_t = W_O (q_t (.) Norm(E_t))), on the tensor cores inside the same kernel.
 * Each tile's readout y, rounded to the I/O dtype as esa_fused_fwd writes it,
 * is multiplied by W_O^T with float32 accumulation and rounded to the I/O
 * dtype; with 64 channels one tile holds whole rows of y, so no partial sums
 * cross tiles.
 *   x, W      as for esa_fused_fwd.
 *   W_O       [64, 64] output weights, [out, in] as stored by a linear layer,
 *             I/O dtype (required).
 *   z         [B,T,64] output, I/O dtype (required): z = y W_O^T.
 *   y         [B,T,H,D] readout, or NULL when only z is wanted (inference);
 *             when given it equals esa_fused_fwd's y bit for bit.
 *   E_final, E_init, mode, workspace: as for esa_scan_fwd.
 * Supported: dtype ESA_F16 or ESA_BF16, C = H * D = 64, C_in of 64 or 128;
 * other shapes return ESA_ERR_UNSUPPORTED (call esa_fused_fwd and multiply by
 * W_O separately).  Pointers 16-byte aligned (ESA_ERR_ALIGN otherwise).
 */
int esa_fused_layer_fwd(const void *x, const void *W, const void *W_O, void *z, void *y, float *E_final, int B,
                        int T, int H, int D, int C_in, int mode, const float *E_init, int dtype, void *workspace,
                        size_t workspace_bytes, void *stream);

/*
 * One-token recurrent update (decode): E <- A (.) E + B in place, then
 * y_t = q_t (.) E / rms(E).
 *   a_t, v_t, q_t [B,H,D] inputs of one token; y_t [B,H,D] output (I/O dtype).
 *   E             [B,H,D] float32 state, read and overwritten.
 * Needs no workspace.  Sources: mlbricks-web.pages.dev/esa, Architecture
 * step "One-token update" and Quick start decode_step(token, state);
 * "Entangled State Attention v2.1", ESA-Lightning lightning_step.
 */
int esa_step(const void *a_t, const void *v_t, const void *q_t, float *E, void *y_t,
             int B, int H, int D, int mode, int dtype, void *stream);

/*
 * Synchronise `stream`, then read and clear the device status word in
 * `workspace`.  Returns ESA_OK; ESA_ERR_WORKSPACE if the workspace is not
 * initialised (a scan on it did nothing); ESA_ERR_TIMEOUT if a bounded wait
 * inside a scan kernel gave up since the last check (the outputs of that
 * call are then invalid); or ESA_ERR_LAUNCH if the stream reports a CUDA
 * error.
 */
int esa_check(void *workspace, void *stream);

/* Static, human-readable text for an esa_status code. */
const char *esa_strerror(int status);

/* Library version as 10000 * major + 100 * minor + patch. */
int esa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* ESA_H_ */
