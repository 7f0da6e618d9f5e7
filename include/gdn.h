/*
 * gdn.h -- C ABI of libgdn, the Gated-Delta-Net (GDN) linear-attention
 * recurrence on NVIDIA B200 (sm_100a).
 *
 * The operation: the "GDN (Gated-Delta-Net) linear-attention recurrence" that
 * the librediffusion PR #21 page names ("What's added"), in the streaming and
 * bidirectional forms of the flashdreams SANA-WM page ("Bidirectional
 * variant") and the causal linear-attention KV cache of the LongSANA diffusers
 * PR #12723 page ("PR feature").  The pages print no formula; the update is
 * the gated delta rule (Gated DeltaNet), per batch b and head h, with a
 * dv x dk state S:
 *
 *     S_t = a_t * S_{t-1} * (I - b_t k_t k_t^T) + b_t v_t k_t^T
 *     o_t = S_t q_t
 *
 * a_t = decay[b,h,t], b_t = beta[b,h,t].  The stored state is H = S^T, a
 * row-major [dk][dv] fp32 matrix per head.  No 1/sqrt(dk) factor is applied.
 *
 * Precondition on the gates: decay in (0, 1] (a gate), beta finite (typically
 * in [0, 1]).  The chunkwise kernels work with log2 decay: a decay below
 * 2^-120 acts as 2^-120, and decays above 1 (growth) are computed as written
 * only while every product of decays within a 64-token chunk stays a normal
 * fp32 number (checked up to 1 + 1e-3); the library does not scan the gates.
 *
 * Layouts (all row-major, contiguous, element strides implied by the sizes):
 *   q, k        [B, H, T, dk]      bf16 or fp32 (mode bit GDN_FP32)
 *   v, o        [B, H, T, dv]      same dtype as q
 *   beta, decay [B, H, T]          fp32 (see the precondition above)
 *   state_in    [B, H, dk, dv]     fp32, or NULL for a zero initial state
 *   state_out   causal: [B, H, dk, dv];  bidi: [2, B, H, dk, dv] =
 *               {forward final state, reverse final state}; or NULL to skip
 *
 * Modes (bit flags, OR-ed):
 *   GDN_CAUSAL (0) / GDN_BIDI (1): causal scan, or bidirectional
 *       o = fwd(x).o + flip_t(fwd(flip_t(x)).o), flip_t reversing q, k, v,
 *       beta and decay together along T; the reverse scan starts from zero and
 *       state_in applies to the forward scan only.
 *   GDN_BF16 (0) / GDN_FP32 (2): dtype of q, k, v and o.  The state and all
 *       accumulation are fp32 in both cases.
 *   GDN_RECURRENT (4): run the token-by-token fp32 SIMT kernel even for bf16
 *       inputs (a slower cross-check of the chunkwise tensor-core kernel).
 *
 * Ownership and asynchrony: every pointer is device memory owned by the
 * caller (except gdn_forward_host, which takes host memory).  Calls enqueue
 * work on `stream` (a cudaStream_t; NULL = the legacy default stream) and
 * return without synchronising.  Temporary workspace is taken stream-ordered
 * on `stream` from a memory pool the library keeps per device; the pool holds
 * on to what it has reserved between calls (so a loop of calls maps device
 * memory once) until gdn_workspace_release().  No other state persists
 * between calls.  state_in == state_out is allowed.  Inputs must not overlap outputs
 * otherwise.
 *
 * Errors: every call returns GDN_OK (0) or a negative code below, and records
 * a message readable with gdn_last_error() (thread-local).  All argument
 * errors are detected on the host before anything is launched.  No C++
 * exception crosses this boundary.
 */
#ifndef GDN_H_
#define GDN_H_

#ifdef __cplusplus
extern "C" {
#endif

enum gdn_mode_bits {
    GDN_CAUSAL = 0,
    GDN_BIDI = 1,
    GDN_BF16 = 0,
    GDN_FP32 = 2,
    GDN_RECURRENT = 4
};

enum gdn_status {
    GDN_OK = 0,
    GDN_ERR_INVALID_ARG = -1,    /* NULL required pointer, B/H/T/n_chunks <= 0, bad mode bits */
    GDN_ERR_UNSUPPORTED = -2,    /* shape/dtype combination the kernels do not implement      */
    GDN_ERR_MISALIGNED = -3,     /* a pointer not 16-byte aligned                              */
    GDN_ERR_CUDA = -4,           /* a CUDA runtime/driver call or kernel launch failed         */
    GDN_ERR_DEVICE_TIMEOUT = -5  /* a bounded device-side wait gave up (gdn_device_status)     */
};

/*
 * gdn_forward -- one causal or bidirectional pass over T tokens.
 *
 * Supported shapes:
 *   bf16 (chunkwise tensor-core kernel): dk = 128, dv in {64, 128}.
 *   fp32, or any dtype with GDN_RECURRENT: dk, dv multiples of 32, <= 128.
 * T >= 1 of any value (a ragged last chunk is handled).  B*H <= 65535.
 *
 * Kernels whose CTAs wait for one another (the pooled chunkwise kernel used
 * for dk = dv = 128, and bidirectional single-CTA launches that fit on the
 * GPU's SMs) are launched cooperatively: CUDA starts them only with every CTA
 * resident, so work on other streams delays them but cannot starve them.
 * Every such wait is bounded (4 s); one that runs out sets the device error
 * word (GDN_ERR_DEVICE_TIMEOUT from gdn_device_status) and the kernel
 * returns: no hang, no silent result.
 */
int gdn_forward(const void *q, const void *k, const void *v,
                const float *beta, const float *decay,
                const float *state_in, float *state_out, void *o,
                int B, int H, int T, int dk, int dv, int mode, void *stream);

/*
 * gdn_rollout -- n_chunks consecutive causal chunks of Tc tokens, the final
 * state of chunk c being the initial state of chunk c+1 (the streaming
 * linear-attention cache).  Equal to n_chunks gdn_forward(GDN_CAUSAL) calls
 * with the state threaded between them.
 *   q, k [n_chunks, B, H, Tc, dk]; v, o [n_chunks, B, H, Tc, dv];
 *   beta, decay [n_chunks, B, H, Tc]; state_in/state_out [B, H, dk, dv] (NULL
 *   allowed); chunk_states NULL or [n_chunks, B, H, dk, dv]: the state after
 *   each chunk.  GDN_BIDI is rejected (GDN_ERR_UNSUPPORTED).
 */
int gdn_rollout(const void *q, const void *k, const void *v,
                const float *beta, const float *decay,
                const float *state_in, float *state_out, float *chunk_states,
                void *o, int B, int H, int n_chunks, int Tc, int dk, int dv,
                int mode, void *stream);

/*
 * gdn_forward_host -- gdn_forward on HOST buffers (same layouts).  Copies the
 * inputs to the device, runs gdn_forward, copies o (and state_out if given)
 * back, and synchronises `stream` before returning.  Device buffers come
 * stream-ordered from the library's workspace pool and go back to it in the
 * same call.  Pinned host memory gives asynchronous copies; pageable memory
 * works but is slower.
 */
int gdn_forward_host(const void *q, const void *k, const void *v,
                     const float *beta, const float *decay,
                     const float *state_in, float *state_out, void *o,
                     int B, int H, int T, int dk, int dv, int mode, void *stream);

/*
 * gdn_forward_host_async -- gdn_forward_host without the final synchronise:
 * the copies in, the kernels and the copies out are enqueued on `stream` and
 * the call returns.  The caller keeps the host buffers alive and untouched
 * (inputs unchanged, outputs unread) until `stream` has passed the call, e.g.
 * by synchronising it or waiting on an event recorded after the call.  With
 * pinned host memory, calls on two streams overlap one call's copies with the
 * other's kernels: the streaming loop of a video pipeline, where chunk i+1 is
 * uploaded while chunk i runs and downloads.  The kernels of host-buffer
 * calls on one device run one after another whatever their streams (each
 * takes every SM; in call order the copies of one overlap the kernel of the
 * other).  Errors of
 * the enqueued copies and kernels surface at the caller's synchronise;
 * argument errors are returned as for gdn_forward.
 */
int gdn_forward_host_async(const void *q, const void *k, const void *v,
                           const float *beta, const float *decay,
                           const float *state_in, float *state_out, void *o,
                           int B, int H, int T, int dk, int dv, int mode, void *stream);

/*
 * gdn_forward_noalloc -- gdn_forward that allocates no device memory.
 *
 * The pages describe no counterpart: this entry point exists for callers
 * that cannot allocate device memory while they run this library -- plugins hosted
 * by a framework that owns all device memory (media and real-time video
 * pipelines, inference engines with a fixed memory plan) and streaming loops
 * that must never wait on an allocator mid-run.  gdn_forward takes its only
 * workspace (the bidirectional arrival counters) stream-ordered; this variant
 * uses a fixed 1 MiB static device array instead, which every device that
 * loads the library holds until the process exits.
 *
 * Same arguments and layouts as gdn_forward; the caller still provides every
 * input and output buffer.  Limits: bf16 chunkwise kernel only (dk = 128,
 * dv in {64, 128}; GDN_FP32 and GDN_RECURRENT return GDN_ERR_UNSUPPORTED);
 * a bidirectional call needs B*H*ceil(T/64)*(dv/64) <= 262144 counters, and a
 * larger one returns GDN_ERR_UNSUPPORTED with the sizes in gdn_last_error()
 * before anything is launched.  Causal calls need no scratch.
 *
 * The first call on a device looks up the array's device address (and may
 * load the library's device code): make that first call before any stream
 * capture.  All calls share the one array; the library clears the counters a
 * call uses before its kernel runs, so back-to-back calls on one stream are
 * fine, but bidirectional calls that overlap on the GPU (other streams, other
 * threads) race on it: they give wrong results, or a wait on a counter runs
 * out and gdn_device_status reports GDN_ERR_DEVICE_TIMEOUT.  Never allocates,
 * frees or calls an allocating library routine.
 */
int gdn_forward_noalloc(const void *q, const void *k, const void *v,
                        const float *beta, const float *decay,
                        const float *state_in, float *state_out, void *o,
                        int B, int H, int T, int dk, int dv, int mode, void *stream);

/*
 * gdn_forward_segmented -- causal gdn_forward with each head's sequence split
 * along time into segments that run in parallel (the segment-parallel scan
 * for streaming calls with few heads: flashdreams SANA-WM page, chunk-causal
 * streaming, where the per-chunk latency is what matters, and LongSANA's
 * causal KV cache).
 *
 * Same arguments, layouts and results as gdn_forward with mode GDN_CAUSAL
 * (bf16 inputs, dk = 128, dv in {64, 128}), up to rounding: the state is
 * affine in its initial value, so each segment's transition
 * P = prod a_t (I - b_t k_t k_t^T) and its zero-start final state L are
 * computed in parallel, the states entering the segments follow from
 * E_{p+1} = P_p E_p + L_p (fp32), and the segments are rerun from them.
 * `n_segments` is the requested number of segments (>= 1); segments are whole
 * 64-token chunks (the last may be shorter), and with fewer than three the
 * call is a plain gdn_forward.  Costs about three times the arithmetic of one
 * scan for a chain about 3/n_segments as long; worth it when B*H*2*(dv/64)
 * CTAs leave most of the GPU idle.  Workspace (stream-ordered): about
 * 4 B*H*n_segments*dk*dv*4 + 2 B*H*n_segments*dk*dk*4 + 4 B*H*T*dk bytes.
 * Errors: as gdn_forward; GDN_BIDI, GDN_FP32 or GDN_RECURRENT return
 * GDN_ERR_UNSUPPORTED, n_segments < 1 returns GDN_ERR_INVALID_ARG.
 */
int gdn_forward_segmented(const void *q, const void *k, const void *v,
                          const float *beta, const float *decay,
                          const float *state_in, float *state_out, void *o,
                          int B, int H, int T, int dk, int dv, int n_segments, int mode,
                          void *stream);

/*
 * gdn_forward_blockcausal -- the frame-block causal read-out: every token of a
 * frame sees its whole frame and every earlier one (the LongSANA page, "PR
 * feature": a causal linear-attention KV cache carried across video frames).
 * The state runs token by token exactly as in gdn_forward; token t of block f
 * (tokens [f*block, (f+1)*block) of a head) is read out with the state after
 * the whole block:  o_t = H_{(f+1)*block-1}^T q_t.  state_out is the final
 * state, as in gdn_forward.
 *
 * Arguments and layouts as gdn_forward (bf16 inputs, dk = 128, dv in {64, 128},
 * mode GDN_CAUSAL); `block` is the frame length in tokens and T must be a
 * multiple of it.  The blocks' zero-start states and transitions are computed
 * in parallel (B*H*T/block independent blocks), the state after every block
 * follows from an fp32 combine, and a read-out pass forms o.  Workspace
 * (stream-ordered): about B*H*(T/block)*(3*dk*dv + 2*dk*dk)*4 + B*H*T*(4*dk + 8)
 * bytes.  Errors: as gdn_forward; block < 1 or T not a multiple of block
 * return GDN_ERR_INVALID_ARG; GDN_BIDI, GDN_FP32 or GDN_RECURRENT, or
 * B*H*T/block > 65535, return GDN_ERR_UNSUPPORTED.
 */
int gdn_forward_blockcausal(const void *q, const void *k, const void *v,
                            const float *beta, const float *decay,
                            const float *state_in, float *state_out, void *o,
                            int B, int H, int T, int dk, int dv, int block, int mode,
                            void *stream);

/*
 * gdn_forward_normalized -- the normalised read-out with a z state next to the
 * kv state (the librediffusion PR #21 review names state_kv and state_z of its
 * bidirectional kernel; the pages give no formula, so this is a reading).  z
 * runs the same gated delta recurrence driven by a constant value of 1,
 *     z_t = a_t (I - b_t k_t k_t^T) z_{t-1} + b_t k_t,
 * and o_t = (S_t q_t) / (z_t . q_t + eps).  GDN_BIDI sums the numerators and
 * the denominators of the two scan directions, then divides.
 *
 * Arguments as gdn_forward (bf16 inputs, dk = 128, dv in {64, 128}), plus
 * state_z_in [B,H,dk] fp32 (NULL: zero; forward scan only), state_z_out
 * [B,H,dk] (GDN_BIDI: [2,B,H,dk]) or NULL, and eps.  The denominators come from
 * a second chunkwise pass over a 64-wide value of ones (beside the first on a
 * second stream for causal calls, after it for bidirectional ones); both
 * passes write bf16, so numerator and denominator are each rounded to bf16
 * before the division.  Workspace (stream-ordered): about B*H*T*256 +
 * B*H*dk*768 bytes.  Errors: as gdn_forward; GDN_FP32 or GDN_RECURRENT return
 * GDN_ERR_UNSUPPORTED; a misaligned state_z pointer GDN_ERR_MISALIGNED.
 */
int gdn_forward_normalized(const void *q, const void *k, const void *v,
                           const float *beta, const float *decay,
                           const float *state_in, const float *state_z_in,
                           float *state_out, float *state_z_out, void *o,
                           int B, int H, int T, int dk, int dv, float eps, int mode,
                           void *stream);

/*
 * gdn_forward_fp8 -- gdn_forward with fp8 (E4M3) q, k, v and one fp32 scale
 * per (batch, head) for each (the flashdreams SANA-WM page, "Developer
 * Details": FP8 inference on sm_90 and newer): the inputs are
 * x = x_scale[b][h] * decode(x8), o is bf16.
 *   q8, k8 [B,H,T,dk], v8 [B,H,T,dv]: E4M3 codes (one byte each);
 *   q_scale, k_scale, v_scale [B,H] fp32;
 *   beta, decay, state_in, state_out, o and mode as gdn_forward (o bf16;
 *   GDN_CAUSAL or GDN_BIDI).
 * dk = 128, dv in {64, 128}.  This version dequantises into bf16 workspace
 * copies (stream-ordered, 2*B*H*T*(2*dk + dv) bytes) and runs the bf16
 * chunkwise kernel on them: fp8 inputs are accepted, their bandwidth is not
 * yet saved.  Errors: as gdn_forward; a NULL scale returns
 * GDN_ERR_INVALID_ARG; GDN_FP32 or GDN_RECURRENT, GDN_ERR_UNSUPPORTED.
 */
int gdn_forward_fp8(const void *q8, const void *k8, const void *v8,
                    const float *q_scale, const float *k_scale, const float *v_scale,
                    const float *beta, const float *decay,
                    const float *state_in, float *state_out, void *o,
                    int B, int H, int T, int dk, int dv, int mode, void *stream);

/*
 * gdn_device_status -- synchronises `stream` and reports (and clears) the
 * library's device-side error word: GDN_OK, or GDN_ERR_DEVICE_TIMEOUT if a
 * bounded wait inside a kernel gave up since the last call, or GDN_ERR_CUDA.
 */
int gdn_device_status(void *stream);

/* Message for the last non-zero return on this thread ("" if none). */
const char *gdn_last_error(void);

/* ABI version: major * 10000 + minor * 100 + patch. */
int gdn_version(void);

/*
 * gdn_workspace_release -- returns to the driver the device memory that the
 * library's workspace pool on `device` holds in reserve (all of it once every
 * call on that device has completed: synchronise first).  Later calls reserve
 * again as they need.  GDN_OK also when the pool was never used;
 * GDN_ERR_INVALID_ARG for a device index outside [0, 64); GDN_ERR_CUDA if the
 * driver refuses.
 *
 * gdn_workspace_reserved -- writes to *bytes the device memory that pool now
 * reserves (0 if never used).  GDN_ERR_INVALID_ARG for a NULL `bytes` or a bad
 * device index.
 */
int gdn_workspace_release(int device);
int gdn_workspace_reserved(int device, unsigned long long *bytes);

/*
 * gdn_kernel_launches -- number of CUDA kernels this library has launched in
 * this process (all devices, all threads).  For launch accounting in
 * benchmarks and tests; reading it has no side effects.
 */
long long gdn_kernel_launches(void);

#ifdef __cplusplus
}
#endif

#endif /* GDN_H_ */
