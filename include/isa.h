/*
 * isa.h - C ABI of the In-context Sparse Attention (ISA) forward pass for
 * NVIDIA B200 (sm_100a).
 *
 * The method is the one of "Lightning Unified Video Editing via In-Context
 * Sparse Attention" (arXiv 2605.04569), as described in the papernotes.org
 * notes (Overall framework; Key designs 1-3) and the paperlayer.ai summary
 * (sections 2 and 3). For an in-context sequence whose first L_src tokens are
 * the source video and whose last L_ctx tokens are the context, one call runs:
 *
 *   1. pooling probe: Qc, Kc, Vc = means over blocks of b tokens;
 *      S_coarse = softmax(Qc Kc^T / sqrt(D)) over all n_q key blocks
 *      (papernotes, Key design 1; paperlayer, section 2 "Pooling Attention");
 *   2. context pre-selection: score[c] = mean over the source query blocks of
 *      S_coarse[i, n_src + c]; keep the k = ceil(alpha_s * L_ctx / b) best
 *      context blocks and gather K_new = [K_src ; kept blocks], same for V
 *      (papernotes, Key design 1; paperlayer, section 3 "Pre-Selection");
 *   3. sharpness routing: M_i = Var(softmax(Qc_i Kc_new^T / sqrt(D))); the
 *      floor(alpha_f * n_q) blocks of lowest M_i take the approximate path
 *      (papernotes, Key design 3; paperlayer, section 3 "Grouped Computation");
 *   4. exact attention over K_new / V_new for the other blocks, and block-wise
 *      0th-order Taylor attention (each K_new block stands in as its mean key
 *      with weight b and its mean value) for the flat blocks (papernotes, Key
 *      design 2);
 *   5. both outputs written back in the original token order.
 *
 * Readings where the pages are silent (they are fixed here, and the CPU
 * oracle of the test suite follows the same ones): the source tokens form
 * n_src = ceil(L_src / b) blocks from token 0 and the context tokens
 * n_ctx = ceil(L_ctx / b) blocks from token L_src, so the last block of
 * either part may be short (its mean is over its own tokens, and in the
 * Taylor path it weighs its own length instead of b); k = ceil(alpha_s * n_ctx - 1e-4) and
 * n_flat = floor(alpha_f * n_q + 1e-4), computed in double from the float
 * arguments; top-k and routing ties break by lower block index; kept blocks
 * enter K_new in ascending order after the source part.
 *
 * Layout: q, k, v and out are row-major contiguous [B, H, N, D] with
 * N = L_src + L_ctx, in the element type given by isa_dtype (bfloat16 or
 * float32); out has the same type. Device pointers must be 16-byte aligned
 * (the kernels move them with bulk and tensor copies); a misaligned one is
 * rejected with ISA_ERR_ARG before any GPU work. Sizes supported: D in {64, 128}, b in
 * {64, 128}, any positive L_src and L_ctx with n_src + n_ctx <= 2048;
 * float32 only with D = 64.
 *
 * Ownership: the caller owns every buffer passed in. The library never frees
 * caller memory and keeps no pointer after a call returns.
 *
 * Errors: a negative return code, never an exception or an abort. The
 * thread-local message of the last failure is available from
 * isa_last_error().
 */
#ifndef ISA_H
#define ISA_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define ISA_API __attribute__((visibility("default")))
#else
#define ISA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum { ISA_BF16 = 0, ISA_F32 = 1 } isa_dtype;

enum {
  ISA_OK = 0,
  ISA_ERR_ARG = -1,         /* null, aliased or misaligned pointer, non-positive size, ratio outside [0,1] or NaN */
  ISA_ERR_SHAPE = -2,       /* reserved: lengths that b does not divide are accepted (short last blocks) */
  ISA_ERR_UNSUPPORTED = -3, /* D, b, dtype or the block count outside the supported set */
  ISA_ERR_WORKSPACE = -4,   /* workspace null or smaller than isa_workspace_bytes() */
  ISA_ERR_CUDA = -5,        /* a CUDA runtime error; the message holds cudaGetErrorString() */
  ISA_ERR_TIMEOUT = -6      /* a kernel's bounded wait gave up (reported by isa_device_status) */
};

/*
 * isa_plan - block counts of a call, computed on the host only (no CUDA).
 * Writes n_q (query / key blocks), k (kept context blocks) and n_flat (Taylor
 * query blocks); any output pointer may be NULL. Returns ISA_OK or an error
 * code for invalid arguments (same checks as isa_forward_ex).
 */
ISA_API int isa_plan(int B, int H, int L_src, int L_ctx, int D, int b, float alpha_s, float alpha_f,
             int32_t* n_q, int32_t* k, int32_t* n_flat);

/*
 * isa_workspace_bytes - device workspace size that isa_forward_ex needs for
 * these sizes (0 if the arguments are invalid; the reason is in
 * isa_last_error()). The workspace holds the pooled blocks, the coarse
 * scores, the selection and routing lists and the gathered context blocks.
 */
ISA_API size_t isa_workspace_bytes(int B, int H, int L_src, int L_ctx, int D, int b, float alpha_s, isa_dtype dt);

/*
 * isa_forward_ex - the whole forward pass, enqueued on `stream`
 * (a cudaStream_t; NULL = the legacy default stream). Asynchronous: returns
 * once the kernels are enqueued. All pointers are device pointers.
 *   q, k, v      [B, H, N, D] inputs (read only, must not alias out)
 *   out          [B, H, N, D] output
 *   dbg_sel      optional int32 [B, H, k]: kept context blocks (0-based,
 *                relative to the first context block), ascending; NULL to skip
 *   dbg_route    optional int32 [B, H, n_q]: exact-path blocks ascending,
 *                then Taylor-path blocks ascending; NULL to skip
 *   workspace    device memory of at least isa_workspace_bytes(), 256-byte
 *                aligned, used as scratch; it must not be shared by calls that
 *                may run at the same time
 * The enqueue makes no device->host synchronisation and no allocation.
 */
ISA_API int isa_forward_ex(const void* q, const void* k, const void* v, int B, int H, int L_src, int L_ctx, int D, int b,
                   float alpha_s, float alpha_f, isa_dtype dt, void* out, int32_t* dbg_sel, int32_t* dbg_route,
                   void* workspace, size_t workspace_bytes, void* stream);

/*
 * isa_forward - bfloat16 convenience form: allocates its workspace with
 * cudaMallocAsync on the legacy default stream, runs isa_forward_ex, checks
 * the device status, frees the workspace and synchronises before returning.
 */
ISA_API int isa_forward(const void* q, const void* k, const void* v, int B, int H, int L_src, int L_ctx, int D, int b,
                float alpha_s, float alpha_f, void* out, int32_t* dbg_sel, int32_t* dbg_route);

/*
 * isa_forward_host - the same pass with HOST buffers (pageable or pinned):
 * copies q, k, v to the device, runs the pass, copies out (and the optional
 * dbg_sel / dbg_route, host int32) back, then synchronises. Element type as
 * given by dt. Device memory is taken inside the call from a stream-ordered
 * memory pool that belongs to the library (one per device, created on first
 * use) and given back to that pool before returning; the pool keeps the memory
 * for the next call until the process exits. The device's default pool and its
 * settings are not touched.
 */
ISA_API int isa_forward_host(const void* q, const void* k, const void* v, int B, int H, int L_src, int L_ctx, int D, int b,
                     float alpha_s, float alpha_f, isa_dtype dt, void* out, int32_t* dbg_sel, int32_t* dbg_route);

/*
 * isa_device_status - synchronises `stream`, then reads and clears the error
 * word that kernels of earlier calls with this workspace may have set.
 * Returns ISA_OK, ISA_ERR_TIMEOUT (a bounded wait in a kernel gave up) or
 * ISA_ERR_CUDA.
 */
ISA_API int isa_device_status(void* workspace, void* stream);

/*
 * isa_debug_pooled - copies intermediates of the LAST isa_forward_ex call made
 * with this workspace (stream-ordered on `stream`): qc, kc, vc as float32
 * [B, H, n_q, D], colscore float32 [B, H, n_ctx], sharp float32 [B, H, n_q].
 * Any output pointer may be NULL. The sizes must match that call.
 */
ISA_API int isa_debug_pooled(int B, int H, int L_src, int L_ctx, int D, int b, float alpha_s, isa_dtype dt,
                     const void* workspace, float* qc, float* kc, float* vc, float* colscore, float* sharp,
                     void* stream);

/*
 * isa_selftest_wait_timeout - enqueues a one-thread kernel that waits on a
 * barrier nothing will ever arrive on. Its bounded wait gives up after
 * timeout_ms (1..10000) and sets the error word of `workspace` (at least 256
 * bytes of device memory, e.g. a forward workspace), so that the next
 * isa_device_status on it returns ISA_ERR_TIMEOUT. It exercises the same
 * bounded-wait path that guards every wait of the forward kernels, without
 * faulting or hanging the GPU, and leaves the CUDA context usable.
 */
ISA_API int isa_selftest_wait_timeout(void* workspace, int timeout_ms, void* stream);

/*
 * isa_selftest_exp2 - for testing: y_poly[i] = the polynomial 2^x[i] that the
 * attention softmax computes on the FMA pipe for part of its exponentials
 * (round-to-nearest range reduction plus a cubic fitted to 2^f on [-1/2, 1/2]),
 * y_ref[i] = CUDA's exp2f(x[i]). Device pointers, n floats, enqueued on stream.
 */
ISA_API int isa_selftest_exp2(const float* x, float* y_poly, float* y_ref, int n, void* stream);

/*
 * isa_set_stage_events - for live per-kernel timing: while set, every forward
 * call made on this host thread records the 5 given CUDA events (cudaEvent_t
 * handles owned by the caller) on its stream: before the pooling kernel and
 * after the pooling, gather, routing and attention kernels. Pass NULL to stop.
 * Returns ISA_ERR_ARG unless n_events == 5 and no handle is NULL.
 */
ISA_API int isa_set_stage_events(void* const* events, int n_events);

/*
 * isa_select_context_noalloc - allocation-free form of stages 1-2 (pooling,
 * coarse scores, context top-k). The paper has no counterpart: this entry
 * point exists for callers that cannot allocate device memory, such as
 * operator plugins that a host runtime hands only their input and output
 * buffers, or serving loops that forbid cudaMalloc because it can
 * synchronise the device.
 *   q, k, v    device inputs [B, H, N, D] (as for isa_forward_ex, 16-byte aligned)
 *   sel        device int32 [B, H, k] output: kept context blocks, ascending
 *   colscore   device float32 [B, H, ceil(L_ctx / b)] output: context-block scores
 * Scratch (the block means of Q, K, V, 3 * B*H * n_q * D * 4 bytes, plus
 * small partial sums, counters and control words, each part rounded up to 256
 * bytes) lives in a fixed 32 MiB device array inside the library, which
 * every GPU that loads the library holds until the process exits. Larger sizes
 * return ISA_ERR_UNSUPPORTED before any GPU work. The first call on a device
 * looks up the array's device address (cudaGetSymbolAddress); make that first
 * call before any stream capture. The looked-up address is kept for the life of
 * the process and does not survive cudaDeviceReset: after a reset, this entry
 * point must not be called again in that process. Every call shares the one
 * array: calls whose GPU work may overlap (several streams or host threads on
 * one device) race on it and must be serialised by the caller. No allocation is
 * made. The return value covers the enqueue only; a kernel wait that gave up is
 * reported by isa_select_context_noalloc_status, which the caller must check
 * before the next call on the device (each call clears the array's error word).
 */
ISA_API int isa_select_context_noalloc(const void* q, const void* k, const void* v, int B, int H, int L_src, int L_ctx,
                                       int D, int b, float alpha_s, isa_dtype dt, int32_t* sel, float* colscore,
                                       void* stream);

/*
 * isa_select_context_noalloc_status - companion of isa_select_context_noalloc
 * (the paper has no counterpart). Synchronises `stream`, then reads and clears
 * the error word in the library's fixed scratch array on the current device.
 * Returns ISA_OK (also when no allocation-free call has run on the device),
 * ISA_ERR_TIMEOUT when a bounded wait of the last call's kernel gave up (its
 * sel and colscore are then not valid), or ISA_ERR_CUDA. Allocates nothing.
 */
ISA_API int isa_select_context_noalloc_status(void* stream);

/* Number of kernel launches one isa_forward_ex call makes for these sizes (0 if invalid). */
ISA_API int isa_launch_count(int B, int H, int L_src, int L_ctx, int D, int b, float alpha_s, float alpha_f, isa_dtype dt);

/*
 * No-sparsity ratio alpha_ns (papernotes.org, Key design 3; the notes quote
 * alpha_ns = 0.0625, i.e. 93.75 % sparsity inside the Taylor path). Inside
 * every Taylor-path query block i, the k_ns = ceil(alpha_ns * n_new - 1e-4)
 * blocks of K_new with the largest coarse scores softmax(Qc_i Kc_new^T /
 * sqrt(D)) (ties to the lower block index) are computed exactly, key by key;
 * the other blocks stay pooled with weight b (papernotes.org, Key design 2:
 * l += P^c * b, O += P^c Vc * b), and one softmax covers both kinds of terms.
 * With alpha_ns = 0 every call below equals its plain counterpart. Needs
 * bfloat16 inputs when alpha_ns > 0 (ISA_ERR_UNSUPPORTED otherwise).
 */

/* isa_plan with alpha_ns: also writes k_ns (exact key blocks per Taylor query block). */
ISA_API int isa_plan_ns(int B, int H, int L_src, int L_ctx, int D, int b, float alpha_s, float alpha_f,
                        float alpha_ns, int32_t* n_q, int32_t* k, int32_t* n_flat, int32_t* k_ns);

/* isa_workspace_bytes with alpha_ns: adds the per-query-block lists and bitmasks of exact key blocks. */
ISA_API size_t isa_workspace_bytes_ns(int B, int H, int L_src, int L_ctx, int D, int b, float alpha_s,
                                      float alpha_ns, isa_dtype dt);

/*
 * isa_forward_ns - isa_forward_ex with the no-sparsity ratio alpha_ns in [0, 1].
 * Arguments, layout, ownership and errors as for isa_forward_ex, plus:
 *   dbg_ns       optional device int32 [B, H, n_q, k_ns]: for every query block
 *                (in block order) its exactly computed K_new blocks, ascending
 *                (0-based blocks of K_new: source blocks, then kept context
 *                blocks in K_new order); written for Taylor and exact query
 *                blocks alike, used only by the Taylor ones; NULL to skip
 *   workspace    at least isa_workspace_bytes_ns() bytes
 * With alpha_ns > 0 the Taylor query blocks take one extra kernel launch.
 */
ISA_API int isa_forward_ns(const void* q, const void* k, const void* v, int B, int H, int L_src, int L_ctx, int D,
                           int b, float alpha_s, float alpha_f, float alpha_ns, isa_dtype dt, void* out,
                           int32_t* dbg_sel, int32_t* dbg_route, int32_t* dbg_ns, void* workspace,
                           size_t workspace_bytes, void* stream);

/*
 * isa_forward_host_ns - isa_forward_host with the no-sparsity ratio alpha_ns
 * (host buffers, copies inside the call, synchronous; alpha_ns as for
 * isa_forward_ns). With alpha_ns = 0 it is isa_forward_host.
 */
ISA_API int isa_forward_host_ns(const void* q, const void* k, const void* v, int B, int H, int L_src, int L_ctx,
                                int D, int b, float alpha_s, float alpha_f, float alpha_ns, isa_dtype dt, void* out,
                                int32_t* dbg_sel, int32_t* dbg_route);

/* Number of kernel launches one isa_forward_ns call makes for these sizes (0 if invalid). */
ISA_API int isa_launch_count_ns(int B, int H, int L_src, int L_ctx, int D, int b, float alpha_s, float alpha_f,
                                float alpha_ns, isa_dtype dt);

/*
 * Variable-length batches (papernotes.org, Key design 1 counts the context
 * blocks as ceil(L_ctx / b), so every element of a batch may have its own
 * lengths and its own short last blocks). Element i has L_src[i] source and
 * L_ctx[i] context tokens, N_i = L_src[i] + L_ctx[i]; every element is an
 * independent ISA pass over its H heads (its own pooling probe, top-k, routing
 * and attention).
 *
 * isa_workspace_bytes_varlen - workspace for isa_forward_varlen: the largest
 * element's isa_workspace_bytes (0 if an argument is invalid).
 */
ISA_API size_t isa_workspace_bytes_varlen(int B, int H, const int32_t* L_src, const int32_t* L_ctx, int D, int b,
                                          float alpha_s, isa_dtype dt);

/*
 * isa_forward_varlen - the pass over a batch of B elements of different lengths.
 *   L_src, L_ctx  HOST int32 arrays [B] (read during the call only); B <= 4096
 *   q, k, v, out  device, packed: element i is a contiguous row-major [H, N_i, D]
 *                 array starting at element offset H * D * (N_0 + ... + N_{i-1})
 *                 (16-byte aligned, out not overlapping the inputs)
 *   dbg_sel       optional device int32: element i's [H, k_i] kept context blocks,
 *                 packed after those of the earlier elements; NULL to skip
 *   dbg_route     optional device int32: element i's [H, n_q_i] routing, packed
 *                 likewise; NULL to skip
 *   workspace     at least isa_workspace_bytes_varlen() bytes: the elements run
 *                 one after another on `stream` and reuse it
 * Other arguments as for isa_forward_ex; errors name the failing element.
 * Asynchronous; an element's kernel timeout stays in the workspace's error word
 * for isa_device_status (later elements do not clear it).
 */
ISA_API int isa_forward_varlen(const void* q, const void* k, const void* v, int B, int H, const int32_t* L_src,
                               const int32_t* L_ctx, int D, int b, float alpha_s, float alpha_f, isa_dtype dt,
                               void* out, int32_t* dbg_sel, int32_t* dbg_route, void* workspace,
                               size_t workspace_bytes, void* stream);

/*
 * Training (trainable ISA: papernotes.org, overview and Key design 2; paperlayer.ai
 * summary, appendix H, where the kernels implement the forward and the backward
 * pass). The backward holds the forward's discrete decisions fixed (kept context
 * blocks and routing): the gradient flows through the exact path over K_new /
 * V_new, the Taylor path over the block means (a mean spreads its gradient as
 * 1/b over its block's rows) and the gather (a kept context block's rows get
 * their K_new rows' gradient; the other context rows get none). The pooling
 * probe, the top-k and the sharpness carry no gradient.
 *
 * isa_forward_train - isa_forward_ex (alpha_ns = 0) that also writes
 *   lse   device float32 [B, H, N], 16-byte aligned: for every row the natural
 *         log of its softmax denominator, sum_t exp(q . k_t / sqrt(D)) over
 *         K_new for an exact row, sum_j L_K(j) exp(q . Kc_j / sqrt(D)) over the
 *         blocks of K_new for a Taylor row (L_K = the block's length).
 * The workspace then holds the call's decisions and pooled rows; keep it, unused
 * by other calls, until isa_backward has run. Debug outputs are not offered.
 */
ISA_API int isa_forward_train(const void* q, const void* k, const void* v, int B, int H, int L_src, int L_ctx, int D,
                              int b, float alpha_s, float alpha_f, isa_dtype dt, void* out, float* lse,
                              void* workspace, size_t workspace_bytes, void* stream);

/* Scratch that isa_backward needs beyond the forward's workspace (0 if the arguments are invalid). */
ISA_API size_t isa_backward_workspace_bytes(int B, int H, int L_src, int L_ctx, int D, int b, float alpha_s,
                                            isa_dtype dt);

/*
 * isa_backward - gradients of sum(out * dout) with respect to q, k and v, enqueued on
 * `stream`. Needs bfloat16, D = 128 and lengths that b divides (else
 * ISA_ERR_UNSUPPORTED). All pointers are device pointers, 16-byte aligned.
 *   q, k, v, out, lse  the forward call's inputs and outputs (isa_forward_train)
 *   dout               [B, H, N, D] gradient of the output
 *   dq, dk, dv         [B, H, N, D] outputs (bfloat16), not overlapping the inputs
 *   fwd_workspace      the workspace of that isa_forward_train call, untouched since;
 *                      the call reads its decisions and pooled rows and uses three of
 *                      its control words as work counters, so two backward calls on one
 *                      forward workspace must not run at the same time (in stream order
 *                      they may run any number of times)
 *   bwd_workspace      at least isa_backward_workspace_bytes(), 256-byte aligned
 * Other arguments must equal the forward call's. Asynchronous, no allocation. A
 * kernel wait that gives up is reported by isa_device_status(fwd_workspace).
 */
ISA_API int isa_backward(const void* q, const void* k, const void* v, const void* out, const float* lse,
                         const void* dout, int B, int H, int L_src, int L_ctx, int D, int b, float alpha_s,
                         float alpha_f, isa_dtype dt, void* dq, void* dk, void* dv, void* fwd_workspace,
                         size_t fwd_workspace_bytes, void* bwd_workspace, size_t bwd_workspace_bytes, void* stream);

/* Message of the last failed call on this host thread ("" if none). */
ISA_API const char* isa_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* ISA_H */
