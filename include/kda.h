/*
 * kda.h -- C ABI of the B200 (sm_100a) Kimi Delta Attention (KDA) recurrence library.
 *
 * KDA is a gated delta-rule linear attention with a per-channel forget gate.  Per
 * batch element b and head h it carries a state S in R^{dk x dv} and, for each token t,
 *
 *     S_t = (I - beta_t k_t k_t^T) Diag(exp g_t) S_{t-1} + beta_t k_t v_t^T
 *     o_t = S_t^T q_t
 *
 * i.e. decay every row i of the state by exp(g_t[i]), let the decayed memory predict v_t
 * from k_t, write only the residual (scaled by beta_t) back along k_t, then read the
 * updated state with q_t.  Sources:
 *   - "Day 21" course page (ai.air7.fun/decks/k3-course-30/day-21): interview item D19
 *     (fixed-size d x d state, delta-rule residual update, per-channel decay gate),
 *     quiz Q8 (state built from k^T v products, O(1) memory), quiz Q9 (predict with the
 *     old memory, overwrite with the residual v - S k only);
 *   - Kimi K3 skill card (skillsmp.com), quick facts: the log-decay is a lower-bounded
 *     scaled sigmoid with g_min = -5, which keeps the diagonal tiles of the chunked form
 *     dense enough for tensor-core products;
 *   - podcast show-notes (scripod.com), section 2.1: chunk-recurrent form (RetNet) and
 *     gated delta rule (Gated DeltaNet), which this library's prefill follows.
 *
 * Conventions shared by every entry point
 *   - All tensor pointers are DEVICE pointers owned by the caller (except in
 *     kda_forward_chunked_host, which takes HOST buffers and a caller-owned device
 *     workspace).  The library never allocates, frees or retains caller memory.  It owns one
 *     small static device status word per device (see kda_get_device_status) and the fixed
 *     scratch array of kda_forward_chunked_host_noalloc (KDA_NOALLOC_SCRATCH_BYTES per device).
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = the legacy default
 *     stream).  A return of KDA_OK means the work was validated and enqueued.
 *   - Tensors are contiguous, row-major, with the layouts stated per function.
 *   - `dtype` applies to q, k, v, g, beta and o.  The state is always fp32.
 *   - g is the per-channel LOG-decay itself (g <= 0; the gate nonlinearity is the
 *     caller's).  There is no query scaling and no q/k normalisation inside the library.
 *   - Supported sizes: dk, dv in {64, 128}; B, H >= 1; T >= 0 (T == 0 copies S0 to S_T).
 *     Every pointer must be 16-byte aligned.
 *   - Errors: argument checks happen before anything is enqueued and return a negative
 *     kda_status; a failed launch returns KDA_ERR_CUDA.  A device-side wait that runs
 *     out (it never hangs) sets the device status word to KDA_ERR_TIMEOUT, which
 *     kda_get_device_status reports.
 */
#ifndef KDA_H_
#define KDA_H_

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

struct CUstream_st; /* == cudaStream_t's pointee; keeps this header free of CUDA includes */

/* Exported symbols (the library is built with hidden visibility by default). */
#if defined(__GNUC__)
#define KDA_API __attribute__((visibility("default")))
#else
#define KDA_API
#endif

typedef enum {
    KDA_OK = 0,
    KDA_ERR_INVALID_ARG = -1, /* null pointer, non-positive size, aliasing that is not allowed */
    KDA_ERR_UNSUPPORTED = -2, /* dtype or head size the library has no kernel for */
    KDA_ERR_MISALIGNED = -3,  /* a pointer is not 16-byte aligned */
    KDA_ERR_CUDA = -4,        /* a CUDA runtime/driver call failed (launch, attribute, ...) */
    KDA_ERR_TIMEOUT = -5      /* a device-side bounded wait gave up (reported by the status word) */
} kda_status;

typedef enum { KDA_DTYPE_BF16 = 0, KDA_DTYPE_FP32 = 1 } kda_dtype;

/* Prefill kernel selection for kda_forward_chunked_impl. */
typedef enum {
    KDA_IMPL_AUTO = 0,    /* bf16 inputs: the tcgen05 kernel (every supported head size); fp32
                             inputs: the SIMT kernel (the only fp32 kernel: bf16 tensor-core
                             operands cannot meet an fp32 accuracy bar) */
    KDA_IMPL_TCGEN05 = 1, /* chunkwise tensor-core kernel: bf16, dk and dv each 64 or 128.  It
                             always computes 128 x 128 states; a head size of 64 is embedded in
                             them with zero channels (exact), so it costs what 128 does */
    KDA_IMPL_SIMT = 2     /* token-serial fp32 CUDA-core kernel: every supported dtype and size */
} kda_impl;

/*
 * kda_forward_chunked -- prefill: run the recurrence over T tokens for every (b, h).
 *
 * Computes o_t for t = 1..T and the final state S_T, starting from S0 (the chunkwise
 * parallel form with 64-token chunks; exact up to rounding, see the header comment).
 *
 *   q, k, g : [B, T, H, dk]   dtype     (g = log-decay, per channel)
 *   v       : [B, T, H, dv]   dtype
 *   beta    : [B, T, H]       dtype     (write strength, one scalar per token and head)
 *   S0      : [B, H, dk, dv]  fp32, or NULL for a zero initial state
 *   o       : [B, T, H, dv]   dtype     output (bf16 outputs are rounded to nearest even)
 *   S_T     : [B, H, dk, dv]  fp32, or NULL when the final state is not wanted.
 *             S_T may alias S0 exactly (in-place state carry); any other overlap
 *             between outputs and inputs is not allowed.
 *   dtype   : kda_dtype.
 *
 * Kernel: KDA_IMPL_AUTO (see kda_impl): bf16 runs the chunkwise tensor-core kernel, fp32 the
 * fp32 kernel.
 *
 * Returns KDA_OK, or a negative kda_status (nothing is enqueued on error).
 */
KDA_API int kda_forward_chunked(const void* q, const void* k, const void* v, const void* g,
                        const void* beta, const float* S0, void* o, float* S_T, int B, int T,
                        int H, int dk, int dv, int dtype, struct CUstream_st* stream);

/*
 * kda_forward_chunked_impl -- kda_forward_chunked with an explicit kernel choice
 * (kda_impl).  Same arguments, layouts and semantics; returns KDA_ERR_UNSUPPORTED when
 * the requested kernel does not cover the dtype/shape.
 */
KDA_API int kda_forward_chunked_impl(const void* q, const void* k, const void* v, const void* g,
                             const void* beta, const float* S0, void* o, float* S_T, int B,
                             int T, int H, int dk, int dv, int dtype, int impl,
                             struct CUstream_st* stream);

/*
 * kda_forward_chunked_states -- kda_forward_chunked that also writes the state after every
 * `interval` tokens: the boundaries from which a prefix cache resumes the recurrence
 * (podcast show-notes (scripod.com), outline item 5.3.1 "KDA-Aware Prefix Cache Management";
 * the channel post on the K3 report (t.iss.one), online-inference paragraph: prefixes are
 * reused at 512-token boundaries).
 *
 *   S_mid    : [B, H, n_mid, dk, dv] fp32 output, n_mid = T / interval (integer division):
 *              S_mid[b][h][n] is the state after the first (n+1)*interval tokens of (b, h),
 *              the same values a kda_forward_chunked over those tokens returns as S_T.
 *              Must not overlap any other argument.  May be NULL only when n_mid == 0.
 *   interval : a positive multiple of 64 (the prefill's chunk length).
 *   impl     : kda_impl, as for kda_forward_chunked_impl.
 *
 * Every other argument, layout and rule as kda_forward_chunked; o and S_T are the values it
 * would produce.  Returns KDA_ERR_INVALID_ARG for interval <= 0, KDA_ERR_UNSUPPORTED for an
 * interval that is not a multiple of 64.
 */
KDA_API int kda_forward_chunked_states(const void* q, const void* k, const void* v, const void* g,
                               const void* beta, const float* S0, void* o, float* S_T,
                               float* S_mid, int interval, int B, int T, int H, int dk, int dv,
                               int dtype, int impl, struct CUstream_st* stream);

/*
 * kda_forward_chunked_host -- kda_forward_chunked on HOST buffers: the library copies the
 * inputs in, runs the prefill and copies o (and S_T) out.  The work is cut into segments of
 * one batch entry and at most 2048 tokens (a multiple of the 64-token chunk); the state passes
 * from one segment of a sequence to the next in device memory, so o and S_T are bitwise those
 * of kda_forward_chunked on the same values.  Copy-in of the next segment, the kernel of the
 * current one and copy-out of the previous one overlap (two internal streams, created and
 * destroyed by the call, ordered by events with `stream`).
 *
 *   q, k, v, g, beta, S0, o, S_T : layouts, dtypes and NULL rules of kda_forward_chunked, in
 *              HOST memory owned by the caller.  Page-locked memory makes the copies
 *              asynchronous; with pageable memory they are staged and the call blocks the host
 *              thread.  S_T may be S0 itself; no other output may overlap an input.  Inputs
 *              must stay unchanged, and outputs unread, until the work on `stream` completes.
 *   workspace       : DEVICE memory owned by the caller, 16-byte aligned, of at least
 *                     kda_forward_chunked_host_workspace(T, H, dk, dv, dtype) bytes; it must
 *                     not be used by anything else until the work on `stream` completes.
 *   workspace_bytes : its size.
 *   impl            : kda_impl, as for kda_forward_chunked_impl.
 *
 * Asynchronous on `stream`: everything the call enqueues comes after the work already on
 * `stream`, and work enqueued on `stream` afterwards comes after all of it (after the last
 * copy-out).  Returns KDA_OK; KDA_ERR_INVALID_ARG for a missing or too small workspace or a
 * bad size or overlap; KDA_ERR_MISALIGNED for an unaligned workspace; KDA_ERR_UNSUPPORTED as
 * kda_forward_chunked_impl (these checks happen before anything is enqueued); KDA_ERR_CUDA if
 * a stream, event, copy or launch fails part-way (work already enqueued still completes, and
 * `stream` still waits for it).
 */
KDA_API int kda_forward_chunked_host(const void* q, const void* k, const void* v, const void* g,
                             const void* beta, const float* S0, void* o, float* S_T, int B,
                             int T, int H, int dk, int dv, int dtype, void* workspace,
                             size_t workspace_bytes, int impl, struct CUstream_st* stream);

/*
 * kda_forward_chunked_host_workspace -- bytes of device workspace kda_forward_chunked_host
 * needs for sequences of T tokens with H heads (independent of B): two segments' inputs and
 * outputs plus two states.  Returns 0 for an unsupported dtype or head size, H <= 0 or T < 0.
 */
KDA_API size_t kda_forward_chunked_host_workspace(int T, int H, int dk, int dv, int dtype);

/*
 * KDA_NOALLOC_SCRATCH_BYTES -- size of the fixed device scratch array that
 * kda_forward_chunked_host_noalloc stages its work through (32 MiB).  The library reserves it
 * in the device memory of every GPU it is loaded on, when it is loaded, and holds it until the
 * process exits.
 */
#define KDA_NOALLOC_SCRATCH_BYTES ((size_t)32 << 20)

/*
 * kda_forward_chunked_host_noalloc -- kda_forward_chunked_host for callers that cannot allocate
 * device memory.  (The pages describe no such entry point: it is an interface matter of this
 * library, with no counterpart in the method.)
 *
 * Who needs it: a caller that holds only host arrays and reaches the library through a plain C
 * foreign-function interface, with no CUDA allocator of its own to create the device workspace
 * kda_forward_chunked_host asks for; or an engine whose device memory is all owned by a pool that
 * forbids allocations outside it (and in which a cudaMalloc would also synchronise the device in
 * the middle of its work).  This call allocates nothing, on the device or the host: it calls no
 * cudaMalloc, cudaFree, stream or event creation, or any other allocating routine.  Instead it
 * stages the work through one fixed scratch array of KDA_NOALLOC_SCRATCH_BYTES that the library
 * reserves when it is loaded.
 *
 *   q, k, v, g, beta, S0, o, S_T : HOST buffers, with the layouts, dtypes, NULL rules and overlap
 *              rules of kda_forward_chunked_host (S_T may be S0 itself).  Page-locked memory makes
 *              the copies asynchronous.  With pageable memory the copies are staged by the driver
 *              and the call blocks the host thread.  Inputs must stay unchanged, and outputs unread,
 *              until the work on `stream` completes.
 *   impl     : kda_impl, as for kda_forward_chunked_impl.
 *
 * Every step runs in order on `stream`: the inputs of one segment are copied in, the prefill runs
 * on them, and o (and S_T after a sequence's last segment) is copied out.  A segment is one batch
 * entry and the largest multiple of 64 tokens whose q, k, g, v, beta and o fit the scratch
 * together with one fp32 state [H, dk, dv]: 192 tokens for H = 96 and bf16 d = 128.
 * The state carried between the segments of a sequence stays in fp32 device memory, so o and S_T
 * are bitwise those of kda_forward_chunked_host and kda_forward_chunked on the same values.  There
 * is no overlap of copies with kernels: this entry point trades speed for needing no memory.
 *
 * Maximum size: the state of one batch entry plus 64 tokens of inputs and outputs (T tokens when
 * T < 64) must fit the scratch: 256-byte-rounded H*dk*dv*4 + 3*n*dk*e + 2*n*dv*e + n*e bytes, with
 * n = H * min(T, 64) and e = 2 (bf16) or 4 (fp32).  So H <= 227 at bf16 d = 128 and H <= 146 at
 * fp32 d = 128.  Larger problems return KDA_ERR_UNSUPPORTED before anything is enqueued.
 *
 * Shared scratch: the array is one per device, shared by every call on that device, and it keeps
 * the last call's contents.  Nothing in it needs to start at zero: a sequence without S0 starts
 * from the zero state inside the kernel, and every byte a segment reads is first written by that
 * same segment's copy-in.  Calls whose work overlaps on the GPU (on different streams, or on one
 * stream from different host threads without ordering) race on the scratch and give undefined
 * results: run them in order, on one stream.
 *
 * First call on a device: it looks up the device address of the scratch (cudaGetSymbolAddress,
 * with that device current) and keeps it for later calls.  Make that first call before any
 * stream capture on the device.
 *
 * Returns KDA_OK; KDA_ERR_INVALID_ARG or KDA_ERR_UNSUPPORTED (also: the problem does not fit the
 * scratch, as above) before anything is enqueued, as kda_forward_chunked_host; KDA_ERR_CUDA if the
 * scratch's address cannot be looked up, or if a copy or launch fails part-way (work already
 * enqueued on `stream` still runs).
 */
KDA_API int kda_forward_chunked_host_noalloc(const void* q, const void* k, const void* v, const void* g,
                                             const void* beta, const float* S0, void* o, float* S_T, int B,
                                             int T, int H, int dk, int dv, int dtype, int impl,
                                             struct CUstream_st* stream);

/*
 * kda_decode_step -- one token for every (b, h), state updated in place.
 *
 * Same recurrence with T = 1 (the memory-bound state read-modify-write of decoding):
 *   S <- Diag(exp g) S;  u = beta (v - S^T k);  S <- S + k u^T;  o = S^T q.
 *
 *   q, k, g : [B, H, dk]      dtype
 *   v       : [B, H, dv]      dtype
 *   beta    : [B, H]          dtype
 *   S       : [B, H, dk, dv]  fp32, read and written in place (must not be NULL)
 *   o       : [B, H, dv]      dtype output
 *
 * Returns KDA_OK or a negative kda_status (nothing is enqueued on error).
 */
KDA_API int kda_decode_step(const void* q, const void* k, const void* v, const void* g,
                    const void* beta, float* S, void* o, int B, int H, int dk, int dv,
                    int dtype, struct CUstream_st* stream);

/*
 * kda_forward_chunked_fused -- kda_forward_chunked with the gate and normalisation prologue fused
 * into the kernels' load stage, so no separate elementwise pass over q, k, g and beta is needed:
 *
 *   g    = -5 * sigmoid(z_g)           per channel (the bounded scaled-sigmoid log-decay with
 *                                      lower bound -5: Kimi K3 skill card (skillsmp.com), quick facts)
 *   beta = sigmoid(z_beta)             per token and head
 *   q, k = q_raw / |q_raw|, k_raw / |k_raw|   (L2 over the head dimension; a zero row stays zero)
 *
 * then exactly the recurrence of kda_forward_chunked.  Layouts, dtypes, sizes and rules as for
 * kda_forward_chunked_impl with (q_raw, k_raw, v, z_g, z_beta) in the places of (q, k, v, g, beta).
 * The tensor-core kernel forms sigmoid and the inverse norms with the hardware's approximate
 * exponential, reciprocal and reciprocal square root (fp32, relative error ~1e-6); the fp32
 * kernel with expf and rsqrtf.
 */
KDA_API int kda_forward_chunked_fused(const void* q_raw, const void* k_raw, const void* v, const void* z_g,
                                      const void* z_beta, const float* S0, void* o, float* S_T, int B, int T,
                                      int H, int dk, int dv, int dtype, int impl, struct CUstream_st* stream);

/*
 * kda_forward_varlen -- prefill over packed sequences of different lengths (continuous batching).
 *
 * N sequences stored back to back along the token axis (the layout a paged serving engine
 * batches prefills in; podcast show-notes (scripod.com), outline item 5.3.1, and the channel
 * post on the K3 report (t.iss.one), online-inference paragraph: one paged pool for the KDA
 * states):
 *
 *   q, k, g    : [T_total, H, dk]   dtype
 *   v          : [T_total, H, dv]   dtype
 *   beta       : [T_total, H]       dtype
 *   cu_seqlens : [N + 1] int32 DEVICE array: sequence n is tokens cu_seqlens[n] .. cu_seqlens[n+1]-1,
 *                with 0 <= cu_seqlens[0] <= cu_seqlens[1] <= ... <= cu_seqlens[N] <= T_total (so no two
 *                sequences share a token; gaps between them are allowed).  The kernels check the whole
 *                array: if it breaks any of these rules, EVERY sequence is processed as empty (S_T = S0,
 *                no o row written) and the device status word is set to KDA_ERR_INVALID_ARG.  o rows of
 *                tokens outside every range are not written.
 *   S0, S_T    : [N, H, dk, dv] fp32, S0 may be NULL (zeros), S_T may be NULL or alias S0
 *   o          : [T_total, H, dv]   dtype
 *   impl       : kda_impl.
 *
 * Every sequence gives exactly what kda_forward_chunked gives for it alone.  Returns KDA_OK
 * or a negative kda_status (nothing enqueued on error).
 */
KDA_API int kda_forward_varlen(const void* q, const void* k, const void* v, const void* g, const void* beta,
                               const int* cu_seqlens, const float* S0, void* o, float* S_T, int N,
                               int T_total, int H, int dk, int dv, int dtype, int impl,
                               struct CUstream_st* stream);

/*
 * kda_decode_step_paged -- kda_decode_step with the states in a pool indexed per sequence.
 *
 *   S_pool : [n_slots, H, dk, dv] fp32, read and written in place
 *   slots  : [B] int32 DEVICE array: sequence b uses S_pool[slots[b]]; slots[b] < 0 skips sequence
 *            b (nothing read or written, o[b] untouched).  Active slots must be distinct.  A slot
 *            >= n_slots is skipped and sets the device status word to KDA_ERR_INVALID_ARG.
 *   q, k, g, v, beta, o : as kda_decode_step (per sequence b).
 *
 * Returns KDA_OK or a negative kda_status (nothing enqueued on error).
 */
KDA_API int kda_decode_step_paged(const void* q, const void* k, const void* v, const void* g, const void* beta,
                                  float* S_pool, int n_slots, const int* slots, void* o, int B, int H,
                                  int dk, int dv, int dtype, struct CUstream_st* stream);

/*
 * kda_state_compose -- apply a segment's state map: S_out = M S_in + N for `count` heads (fp32).
 *
 * Over a segment of tokens the recurrence is affine in its initial state: S_end = M S_start + N,
 * with M = prod_t (I - beta_t k_t k_t^T) Diag(exp g_t) and N the final state from a zero start.
 * Splitting a long sequence over devices then only needs this fixed-size pair exchanged
 * (KDA context parallelism: channel post on the K3 report (t.iss.one), infrastructure
 * paragraph).  A segment's pair comes from two kda_forward_chunked calls: N with S0 = NULL,
 * M as S_T with v = 0 (dv = dk) and S0 = the identity.
 *
 *   M      : [count, dk, dk] fp32
 *   S_in   : [count, dk, dv] fp32
 *   N      : [count, dk, dv] fp32, or NULL for zero
 *   S_out  : [count, dk, dv] fp32 output; may be S_in or N itself (in place), must not
 *            overlap M or partially overlap S_in / N
 *
 * dk, dv in {64, 128}.  Returns KDA_OK or a negative kda_status (nothing enqueued on error).
 */
KDA_API int kda_state_compose(const float* M, const float* S_in, const float* N, float* S_out, int count,
                              int dk, int dv, struct CUstream_st* stream);

/*
 * kda_output_correct -- correct the outputs of a segment that was run from a zero state, once the
 * state it really starts from is known: o_out[b,t,h,:] = o_in[b,t,h,:] + S_in[b,h]^T C[b,t,h,:].
 *
 * Over a segment S_t = Phi_t S_in + S_t^0 (Phi_t = prod_{u<=t} (I - beta_u k_u k_u^T) Diag(exp g_u),
 * S_t^0 the state from a zero start), so o_t = o_t^0 + S_in^T (Phi_t^T q_t).  The correction operand
 * C_t = Phi_t^T q_t is the output of kda_forward_chunked on the same q, k, g, beta with v = 0 (dv = dk)
 * and S0 = the identity; its S_T is the segment's map M (see kda_state_compose).  This is the one
 * exchange step of KDA context parallelism (channel post on the K3 report (t.iss.one),
 * infrastructure paragraph): a rank runs its segment before its incoming state is known, then
 * applies this correction.
 *
 *   C      : [B, T, H, dk]  dtype
 *   S_in   : [B, H, dk, dv] fp32
 *   o_in   : [B, T, H, dv]  dtype (the zero-start outputs)
 *   o_out  : [B, T, H, dv]  dtype output (bf16 rounded to nearest even); may be o_in itself
 *
 * bf16 with dk = dv = 128 runs on the tensor core (S_in rounded to bf16 as the product's operand,
 * fp32 accumulation); other shapes and fp32 on CUDA cores in fp32.  T == 0 does nothing.  Returns
 * KDA_OK or a negative kda_status (nothing enqueued on error).
 */
KDA_API int kda_output_correct(const void* C, const float* S_in, const void* o_in, void* o_out, int B, int T, int H,
                               int dk, int dv, int dtype, struct CUstream_st* stream);

/*
 * kda_get_device_status -- synchronise `stream`, then return and clear the status word
 * of the current device: KDA_OK, KDA_ERR_TIMEOUT (a kernel's bounded wait gave up; its
 * outputs are then undefined), KDA_ERR_INVALID_ARG (a kernel found an out-of-range device
 * index: a sequence offset or a state slot), or KDA_ERR_CUDA if the synchronisation itself
 * failed.
 *
 * The word belongs to the DEVICE, not to a call or a stream: every kernel of the library on that
 * device, on any stream, sets the same word (the first error wins), and a read clears it.  Only
 * `stream` is synchronised, so with work on several streams a kernel still running on another one
 * may set the word after the read, and the error read may come from another stream's call.  When
 * several streams are in use, synchronise the device (cudaDeviceSynchronize) before calling this
 * to attribute an error to the work enqueued before that point.
 */
KDA_API int kda_get_device_status(struct CUstream_st* stream);

/* kda_status_string -- static, human-readable name of a kda_status value. */
KDA_API const char* kda_status_string(int status);

/* kda_version -- library version as major*10000 + minor*100 + patch. */
KDA_API int kda_version(void);

/*
 * kda_debug_set_wait_fault -- TEST HOOK for the device-side timeout path (not for production).
 *
 * The tensor-core prefill coordinates its two warp groups with mbarrier waits, each bounded
 * in wall time (2 s by default); a wait that runs out sets the status word to
 * KDA_ERR_TIMEOUT, lets every warp of the CTA leave its loop, drains the outstanding
 * tensor-core and TMA work, frees the tensor memory and returns.  Nothing traps, faults or
 * hangs, and the CUDA context stays usable.
 *
 *   mode 1: subsequent tcgen05 prefill launches skip the first hand-off from the operand
 *           warps to the recurrence warps, so a wait is guaranteed to run out; every wait
 *           is limited to timeout_ns (1 ms .. 10 s).  Outputs of such launches are undefined.
 *   mode 0: normal operation (the timeout_ns argument is ignored; 2 s limit).
 *
 * Process-wide setting, read at launch.  Returns KDA_OK or KDA_ERR_INVALID_ARG.
 */
KDA_API int kda_debug_set_wait_fault(int mode, unsigned long long timeout_ns);

#ifdef __cplusplus
}
#endif

#endif /* KDA_H_ */
