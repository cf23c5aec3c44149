/*
 * wkv4.h -- C ABI of the RWKV-4 WKV forward and decode step on NVIDIA B200 (sm_100a).
 *
 * The operation (per batch row b and channel c, independently):
 *   with decay w = w_c (normally -exp(time_decay_c)) and bonus u = u_c,
 *   wkv_t = ( sum_{i<t} e^{(t-1-i) w + k_i} v_i + e^{u + k_t} v_t )
 *         / ( sum_{i<t} e^{(t-1-i) w + k_i}     + e^{u + k_t}     ),
 * i.e. the RWKV-4 time-mix recurrence, carried as a per-channel fp32
 * (numerator, denominator, max) state with the max-trick: "RWKV in a
 * self-built engine: a second non-attention paradigm (WKV/RNN)", abstract,
 * Methods table ("Precision": WKV numerator/denominator/max state carried in
 * fp32) and Reproducibility / Provenance ("Implementation").  That the state
 * is first-class -- produced by one call and consumed by the next, tracked by
 * the caller -- follows "An RNN that claims to match transformers, now in
 * chatbot form" ("The interesting bit"; "Caveats").
 *
 * State layout: one fp32 buffer [3][B][C], planes (num a, den b, max p), C
 * fastest, with true numerator A = a e^p and denominator D = b e^p (natural
 * units).  The empty state is (0, 0, -1e38).  A state given on entry is the
 * state after the previous call's last token: it enters output t with weight
 * e^{t w}, so splitting T over two calls with the state carried gives the
 * result of one call (to fp32 rounding).
 *
 * Tensor layout: k, v, y are [B][T][C] row-major (C fastest) in the I/O dtype;
 * w, u are fp32 [C].  All pointers are DEVICE pointers owned by the caller;
 * the library keeps none of them after the call returns.
 *
 * Calls are asynchronous on `stream` (NULL = the legacy default stream) and
 * return a status without synchronising.  Pointers need no particular
 * alignment: misaligned or odd-C inputs take a slower element-wise path.
 * NaN / Inf inputs propagate unchecked.  Distinct calls may run concurrently
 * on different streams.
 *
 * Every kernel is launched with programmatic stream serialization: it may
 * start while the kernel before it on the stream is finishing, and touches no
 * memory before that kernel has completed (griddepcontrol.wait); it lets the
 * next kernel start at once (griddepcontrol.launch_dependents).  Ordering on
 * the stream is unchanged for ordinary launches; a caller's own kernel
 * launched with programmatic serialization right after a call must, as with
 * any such launch, wait for the grid before it (cudaGridDependencySynchronize)
 * before reading the call's outputs.
 */
#ifndef WKV4_H
#define WKV4_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define WKV4_API __attribute__((visibility("default")))
#else
#define WKV4_API
#endif

struct CUstream_st;
typedef struct CUstream_st* wkv4_stream_t; /* a cudaStream_t */

/* I/O dtype of k, v and y.  w, u and the state are always fp32. */
enum {
    WKV4_F32 = 0,
    WKV4_F16 = 1,
    WKV4_BF16 = 2
};

/* status codes (0 = success, negative = error) */
enum {
    WKV4_OK = 0,
    WKV4_ERR_ARG = -1,     /* a required pointer is NULL, or B/T/C < 0 */
    WKV4_ERR_DTYPE = -2,   /* dtype is not one of WKV4_F32/F16/BF16 */
    WKV4_ERR_ALIAS = -3,   /* y or the output state overlaps an input it must not */
    WKV4_ERR_CUDA = -4,    /* a CUDA runtime call or kernel launch failed */
    WKV4_ERR_TIMEOUT = -5, /* a bounded device-side wait ran out (see wkv4_device_error) */
    WKV4_ERR_VARIANT = -7, /* unknown kernel variant */
    WKV4_ERR_SLOT = -8     /* a decode row named a state slot outside the pool (see wkv4_device_error) */
};

/*
 * Forward over T time steps (prefill).
 *   B, T, C     batch rows, time steps, channels.  B == 0 or C == 0: no-op.
 *               T == 0: state_out <- state_in (or the empty state).
 *   w, u        [C] fp32 decay (w = -exp(time_decay), supplied by the caller)
 *               and bonus, both in natural-log units.
 *   k, v        [B][T][C] in `dtype`.
 *   state_in    [3][B][C] fp32, or NULL for the empty state.
 *   y           [B][T][C] in `dtype`, written with round-to-nearest-even.
 *               Must not overlap k, v, w, u, state_in or state_out.
 *   state_out   [3][B][C] fp32 state after the last step, or NULL.  May equal
 *               state_in exactly (in-place update); any other overlap with an
 *               input is WKV4_ERR_ALIAS.
 *   stream      CUDA stream of the call.
 *   dtype       WKV4_F32, WKV4_F16 or WKV4_BF16.
 * The call allocates no memory.  Returns WKV4_OK or an error code; a
 * device-side wait that ran out is reported by wkv4_device_error().
 */
WKV4_API int wkv4_forward(int64_t B, int64_t T, int64_t C, const float* w, const float* u,
                 const void* k, const void* v, const float* state_in, void* y,
                 float* state_out, wkv4_stream_t stream, int dtype);

/* Kernel choices of wkv4_forward_variant (for tests and tuning). */
enum {
    WKV4_KERNEL_AUTO = 0,     /* what wkv4_forward picks */
    WKV4_KERNEL_SEQ = 1,      /* channel-parallel, sequential over T, TMA-staged time tiles */
    WKV4_KERNEL_SCAN = 2,     /* chunked scan, time segments chained in a thread-block cluster */
    WKV4_KERNEL_SCAN_LDG = 3, /* the chunked scan with element-wise loads and stores */
    WKV4_KERNEL_STEP = 4      /* exact per-step max-trick, one thread per channel (any T) */
};

/* wkv4_forward with an explicit kernel choice.  SEQ and SCAN need TMA
 * alignment (16-byte aligned k, v and y, and C * sizeof(dtype) a multiple of
 * 16); when it is not met both run as SCAN_LDG.  AUTO and T == 1 run the
 * decode-step kernel; an explicit choice runs that kernel for any T >= 1.
 * Unknown variant: WKV4_ERR_VARIANT. */
WKV4_API int wkv4_forward_variant(int64_t B, int64_t T, int64_t C, const float* w, const float* u,
                         const void* k, const void* v, const float* state_in, void* y,
                         float* state_out, wkv4_stream_t stream, int dtype, int variant);

/*
 * The forward with the receptance gate of the time mix applied to its output:
 *   y = sigmoid(r) * wkv  elementwise,  sigmoid(r) = 1 / (1 + e^{-r}),
 * the gating that follows the WKV recurrence in the time mix ("RWKV in a
 * self-built engine: a second non-attention paradigm (WKV/RNN)", abstract
 * and Reproducibility / Provenance, "Implementation": time-mix gating;
 * "RWKV-4 14B", "Every architecture field": the time mix's receptance
 * matrix).  The pages name the gate but not its function; the logistic
 * sigmoid is the reading taken.  Fused into the output pass: one more
 * exponential a channel-step, no extra pass over y.
 *   r          [B][T][C] in `dtype` (the receptance), required when B, T and
 *              C are all non-zero (else WKV4_ERR_ARG).  y must not overlap r,
 *              nor may state_out (WKV4_ERR_ALIAS).
 * Every other argument, the state, the return codes and the alignment rules
 * (r takes part in them like k and v) are those of wkv4_forward; the state
 * does not depend on r.  No allocation.
 */
WKV4_API int wkv4_forward_gated(int64_t B, int64_t T, int64_t C, const float* w, const float* u,
                                const void* k, const void* v, const void* r,
                                const float* state_in, void* y, float* state_out,
                                wkv4_stream_t stream, int dtype);

/* wkv4_forward_gated with an explicit kernel choice (as wkv4_forward_variant). */
WKV4_API int wkv4_forward_gated_variant(int64_t B, int64_t T, int64_t C, const float* w,
                                        const float* u, const void* k, const void* v,
                                        const void* r, const float* state_in, void* y,
                                        float* state_out, wkv4_stream_t stream, int dtype,
                                        int variant);

/*
 * One decode step (T = 1) for B sequences, updating the state in place.
 *   w, u     [C] fp32.
 *   k, v     [B][C] in `dtype`.
 *   state    [3][B][C] fp32, read and overwritten (RNN mode: "An RNN that
 *            claims to match transformers, now in chatbot form").
 *   y        [B][C] in `dtype`; must not overlap k, v, w, u or state.
 * Equal, bit for bit, to wkv4_forward with T = 1 and state_in == state_out.
 */
WKV4_API int wkv4_decode_step(int64_t B, int64_t C, const float* w, const float* u, const void* k,
                     const void* v, float* state, void* y, wkv4_stream_t stream, int dtype);

/*
 * wkv4_decode_step with the receptance gate on its output: y = sigmoid(r) *
 * wkv (see wkv4_forward_gated).  r [B][C] in `dtype`, required; y must not
 * overlap it.  Equal, bit for bit, to wkv4_forward_gated with T = 1 and
 * state_in == state_out.
 */
WKV4_API int wkv4_decode_step_gated(int64_t B, int64_t C, const float* w, const float* u,
                                    const void* k, const void* v, const void* r, float* state,
                                    void* y, wkv4_stream_t stream, int dtype);

/*
 * One decode step (T = 1) for B sequences whose states live in a pool of S
 * slots: row b of k, v and y steps the state in slot slot_ids[b], in place.
 * The RNN state as a first-class object that the caller keeps per
 * conversation ("An RNN that claims to match transformers, now in chatbot
 * form", sections "The interesting bit" and "Caveats"), for many
 * conversations served together.
 *   w, u        [C] fp32.
 *   k, v        [B][C] in `dtype`.
 *   state_pool  [3][S][C] fp32 (planes numerator, denominator, max); the rows
 *               slot_ids[b] are read and overwritten, every other row is left
 *               as it is.
 *   slot_ids    [B] int32 in device memory, each in [0, S), all distinct
 *               (repeated ids make their rows race on one slot: undefined).
 *               A row whose id is outside [0, S) touches neither the pool
 *               nor its row of y, and sets bit 8 of the device error word
 *               (wkv4_device_error then returns WKV4_ERR_SLOT).
 *   y           [B][C] in `dtype`.
 * y must not overlap k, v, w, u, the pool or slot_ids, and the pool must not
 * overlap k, v, w, u or slot_ids: WKV4_ERR_ALIAS.  S < 0: WKV4_ERR_ARG.
 * Per row, equal bit for bit to wkv4_decode_step on that row's state.  The
 * call allocates no memory.
 */
WKV4_API int wkv4_decode_step_slots(int64_t B, int64_t C, int64_t S, const float* w, const float* u,
                                    const void* k, const void* v, float* state_pool,
                                    const int32_t* slot_ids, void* y, wkv4_stream_t stream,
                                    int dtype);

/*
 * Token shift of the RWKV-4 time mix, the step before the k, v (and r)
 * projections: each output mixes the current token's channels with the
 * previous token's ("RWKV in a self-built engine: a second non-attention
 * paradigm (WKV/RNN)", Reproducibility / Provenance, "Implementation":
 * token-shift, "mix current and previous token"), read as
 *   xk[b,t,c] = mix_k[c] x[b,t,c] + (1 - mix_k[c]) x[b,t-1,c]
 * and likewise xv (mix_v) and xr (mix_r), with x[b,-1,c] = x_prev[b,c].
 *   x            [B][T][C] in `dtype`.
 *   x_prev       [B][C] in `dtype`: the token before t = 0 (the previous
 *                call's x_last), or NULL for zeros (a sequence start).
 *   mix_k, mix_v [C] fp32; mix_r [C] fp32 or NULL (then xr is not written).
 *   xk, xv, xr   [B][T][C] in `dtype` (xr may be NULL when mix_r is).
 *   x_last       [B][C] in `dtype` or NULL: receives x[:, T-1, :] (x_prev
 *                when T == 0), the next call's x_prev.
 * Each output is x_prev + mix (x - x_prev) in fp32, rounded once to `dtype`.
 * Outputs must not overlap the inputs or one another (x_last included):
 * WKV4_ERR_ALIAS.  B, T or C < 0, B > 65535 or T > 1048560: WKV4_ERR_ARG; a
 * NULL x, mix_k, mix_v, xk, xv (or xr with mix_r given): WKV4_ERR_ARG.
 * Chained calls with x_last fed back as x_prev equal one call over the joined
 * T.  No allocation.
 */
WKV4_API int wkv4_token_shift(int64_t B, int64_t T, int64_t C, const void* x, const void* x_prev,
                              const float* mix_k, const float* mix_v, const float* mix_r,
                              void* xk, void* xv, void* xr, void* x_last, wkv4_stream_t stream,
                              int dtype);

/*
 * The state after two consecutive segments of one sequence, from the state
 * after the first and the second's own state: x (the state after the first
 * segment, or NULL for the empty state) followed by y (the state of a
 * segment of n_steps steps from the empty state), per channel
 *   A = e^{n_steps w} A_x + A_y,   D = e^{n_steps w} D_x + D_y,
 * returned as a (num, den, max) triple with the max-trick.  The state is the
 * sequence's whole history ("An RNN that claims to match transformers, now
 * in chatbot form", "The interesting bit"), so a sequence split over T --
 * across devices, each summarising its own segment from the empty state --
 * is joined by this combine: the state entering segment r is the combine of
 * the segments before it, in order.
 *   w          [C] fp32 decay (as for wkv4_forward).
 *   x, y, out  [3][B][C] fp32 (planes num, den, max).  out may be x or y
 *              itself; any other overlap (or out over w) is WKV4_ERR_ALIAS.
 * B, C or n_steps < 0, a NULL w, y or out: WKV4_ERR_ARG.  Asynchronous on
 * `stream`, no allocation.
 */
WKV4_API int wkv4_state_combine(int64_t B, int64_t C, const float* w, int64_t n_steps,
                                const float* x, const float* y, float* out,
                                wkv4_stream_t stream);

/*
 * The forward (or, with r, the gated forward) from HOST buffers: the
 * activations come from host memory and the outputs go back to it, the
 * copies overlapped with the kernels.  T is cut into chunks of chunk_steps
 * steps (0: the library's choice, about a sixteenth of the input bytes and
 * at least 16 MB of them); while the forward runs on chunk i, chunk i + 1's
 * inputs are copied in and chunk i - 1's outputs copied out, on two streams
 * of the call's own, and the chunks are forward calls chained through one
 * device state: the state after a call is the next call's initial state
 * ("An RNN that claims to match transformers, now in chatbot form", "The
 * interesting bit"), so the result is that of one wkv4_forward (or
 * wkv4_forward_gated) over the whole T, to the rounding of the fp32 state
 * at each chunk boundary.
 *   w, u         [C] fp32 DEVICE pointers (the layer's parameters).
 *   k, v         [B][T][C] in `dtype`, HOST pointers (pinned memory lets the
 *                copies overlap; pageable memory works, serialised).
 *   r            [B][T][C] in `dtype` on the host, or NULL: the ungated
 *                forward.
 *   state_in     [3][B][C] fp32 on the host, or NULL for the empty state.
 *   y            [B][T][C] in `dtype` on the host.
 *   state_out    [3][B][C] fp32 on the host, or NULL; may equal state_in.
 *   workspace    DEVICE memory of the current device, owned by the caller,
 *                at least wkv4_forward_host_workspace(B, T, C, dtype,
 *                r != NULL, chunk_steps) bytes, 16-byte aligned; it holds two
 *                chunks' k, v (r) and y and the state, and must not overlap
 *                any other argument.  Contents undefined after the call.
 *   chunk_steps  steps a chunk, or 0.
 * The call is asynchronous on `stream` like every call of the library: y and
 * state_out are complete once `stream` has reached the point after the call
 * (it waits for the call's last copy).  The library allocates no device
 * memory.  B == 0 or C == 0: no-op; T == 0: state_out <- state_in (or the
 * empty state, written through the workspace).  Returns WKV4_ERR_ARG for a
 * NULL required pointer, negative sizes or a workspace that is too small,
 * WKV4_ERR_ALIAS for overlapping outputs (as wkv4_forward), WKV4_ERR_DTYPE,
 * WKV4_ERR_CUDA; the errors of the chained forward calls pass through.
 */
WKV4_API int wkv4_forward_host(int64_t B, int64_t T, int64_t C, const float* w, const float* u,
                               const void* k, const void* v, const void* r,
                               const float* state_in, void* y, float* state_out,
                               void* workspace, size_t workspace_bytes, int64_t chunk_steps,
                               wkv4_stream_t stream, int dtype);

/* Workspace bytes wkv4_forward_host needs for these sizes (gated: r given;
 * with T == 0 the state's bytes), or 0 for B or C <= 0, T or chunk_steps < 0
 * or an unknown dtype. */
WKV4_API size_t wkv4_forward_host_workspace(int64_t B, int64_t T, int64_t C, int dtype, int gated,
                                            int64_t chunk_steps);

/*
 * Device-side error word of the current device (bit 1: a bounded wait for a
 * TMA copy ran out; bit 2: a bounded wait for a cluster peer's partial state
 * ran out; bit 8: a slot-indexed decode row named a slot outside its pool;
 * bit 16, bounds-checked builds only: an index outside its buffer).  One word
 * per device and process, shared by every stream and call.  Synchronises the
 * WHOLE device (cudaDeviceSynchronize: every stream, not only the caller's),
 * reads the word, and clears it when `reset` is non-zero -- meant for tests
 * and error paths, not for polling after every call.  Returns WKV4_OK when
 * the word is zero, WKV4_ERR_TIMEOUT when a wait ran out, else WKV4_ERR_SLOT
 * when a slot id was out of range (or an index was out of bounds), or
 * WKV4_ERR_CUDA when the read itself failed.
 */
WKV4_API int wkv4_device_error(int reset);

/* Static description of a status code. */
WKV4_API const char* wkv4_status_string(int status);

/* Library ABI version (major * 10000 + minor * 100 + patch). */
WKV4_API int wkv4_version(void);

#ifdef __cplusplus
}
#endif

#endif /* WKV4_H */
