/*
 * attn.h -- C ABI of libattn.so: multi-head causal scaled dot-product
 * self-attention, forward and backward, on NVIDIA B200 (sm_100a).
 *
 * What it computes (per head, rows i and columns j of a T x T tile):
 *
 *   S_ij = scale * <q_i, k_j>  for j <= i, -inf above the diagonal
 *   P    = row softmax of S,  O = P V,  lse_i = ln sum_{j<=i} exp(S_ij)
 *
 * "How Andrej Karpathy built GPT from 200 lines of code" (rdly.ru summary of
 * the "Let's build GPT" video): section "Implementing the attention heads
 * (Query, Key, Value)" -- affinities are the dot product of a token's query
 * with the keys of the tokens up to it [1:06:16], divided by the square root
 * of the head size [1:17:18], used to aggregate the values [1:10:15], several
 * heads in parallel [1:22:27]; section "Self-Attention: the mathematical
 * trick" -- the upper triangle is set to -inf before the softmax so a token
 * cannot look into the future [55:20].  Dropout is 0 ("Model Architecture
 * Nanogpt" skill card, Workflow 2 config), so there is no dropout argument.
 * The backward pass is the exact derivative of the forward (the pages give no
 * formula for it): dV = P^T dO, dS = P o (dO V^T - Delta), Delta_i =
 * <dO_i, O_i>, dQ = scale dS K, dK = scale dS^T Q.
 *
 * Common rules for every entry point:
 *
 *  - Layout: q, k, v, o, dO, dq, dk, dv are [B, H, T, D] contiguous row-major
 *    (D fastest); lse is [B, H, T] contiguous float32.
 *  - All pointers are device pointers owned by the caller.  The library
 *    allocates no device memory, never synchronises the stream and only
 *    enqueues work on `stream` (NULL = the legacy default stream).
 *  - Stream order is the ordinary one.  The bf16 kernels are launched with
 *    programmatic stream serialisation, so a kernel's set-up may overlap the
 *    end of the work before it in the stream.  But each kernel waits for that
 *    work to complete before it reads or writes any memory, so work enqueued
 *    earlier (a producer of q, k, v, a reader of the workspace) is fully
 *    ordered before it.  The calls may be captured into CUDA graphs (after
 *    one call outside the capture on the device).
 *  - bf16 entry points take __nv_bfloat16 data through `void *`; every tensor
 *    pointer must be 16-byte aligned (TMA requirement).  float32 entry points
 *    need 4-byte alignment.
 *  - `scale` is normally 1/sqrt(D); any finite positive value is accepted.
 *  - Argument errors are reported before anything is launched; a failed
 *    launch is reported as ATTN_ERR_CUDA.  Faults inside a kernel surface
 *    asynchronously at the caller's next synchronisation.  Every internal wait
 *    of the kernels is bounded: a wait that runs out records a flag that
 *    attn_device_error() returns as ATTN_ERR_TIMEOUT.
 *  - The plain entry points compute the decoder's causal attention; the _ex
 *    entry points also take an attn_options (the mask) and, for bf16,
 *    strides.
 *  - Calls are thread-safe; tensor descriptors travel as kernel parameters.
 *    Calls that write the same output buffers race like any CUDA work.
 */
#ifndef ATTN_H
#define ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* The CUDA runtime's own stream handle type (an opaque pointer). */
typedef struct CUstream_st *cudaStream_t;

typedef enum {
    ATTN_OK = 0,
    ATTN_ERR_NULL = -1,          /* a required pointer is NULL                      */
    ATTN_ERR_SHAPE = -2,         /* B, H or T < 1, or B*H*T*D overflows             */
    ATTN_ERR_UNSUPPORTED_D = -3, /* head_dim outside the supported set              */
    ATTN_ERR_ALIGN = -4,         /* a pointer misses its required alignment         */
    ATTN_ERR_CUDA = -5,          /* a CUDA runtime/driver call or launch failed     */
    ATTN_ERR_TIMEOUT = -6,       /* a bounded in-kernel wait ran out                */
    ATTN_ERR_WORKSPACE = -7,     /* workspace NULL or smaller than required         */
    ATTN_ERR_DEVICE = -8,        /* current device is not sm_100 (B200 class)       */
    ATTN_ERR_SCALE = -9,         /* scale is not finite and positive                */
    ATTN_ERR_OPTION = -10,       /* an attn_options field holds an unsupported value */
    ATTN_ERR_DEVICE_CHECK = -11  /* a device-side bounds check failed (the debug
                                    build, libattn_debug.so, only)               */
} attn_status;

/* Human-readable name of a status code (static string, never NULL). */
const char *attn_status_string(int status);

/* ---------------- bf16 path: tcgen05 tensor cores + TMA ------------------ */

/* Forward.  q, k, v: bf16 inputs; o: bf16 output; lse: float32 output, the
 * natural-log log-sum-exp of each row's scaled, masked scores (needed by
 * attn_bwd).  D must be 32, 64 or 128.  Any T >= 1. */
int attn_fwd(const void *q, const void *k, const void *v, void *o, float *lse,
             int B, int H, int T, int D, float scale, cudaStream_t stream);

/* Bytes of device workspace attn_bwd needs: a float32 dQ accumulator
 * [B,H,T,D], then -lse * log2(e) and -Delta_i = -<dO_i, O_i> (with dropout,
 * divided by the keep scale), each [B*H] rows of T rounded up to a multiple
 * of 128 floats; each part 256-byte aligned.  0 on a bad shape or
 * unsupported D. */
size_t attn_bwd_workspace_bytes(int B, int H, int T, int D);

/* Backward.  q, k, v, o, lse: as given to / returned by attn_fwd; dO: bf16
 * upstream gradient; dq, dk, dv: bf16 outputs (fully overwritten).
 * workspace: caller-owned device scratch of at least
 * attn_bwd_workspace_bytes(B,H,T,D) bytes, 256-byte aligned; its contents on
 * entry do not matter and are clobbered.  D must be 32, 64 or 128. */
int attn_bwd(const void *q, const void *k, const void *v, const void *o, const float *lse,
             const void *dO, void *dq, void *dk, void *dv,
             int B, int H, int T, int D, float scale,
             void *workspace, size_t workspace_bytes, cudaStream_t stream);

/* Backward without caller-supplied workspace (no counterpart in the pages:
 * it exists for the library's users, not for the method).
 *
 * For callers that cannot allocate device memory: C hosts without a device
 * allocator, plug-ins in a framework that owns all device memory through its
 * own pool and forbids cudaMalloc, and latency-critical loops where a
 * cudaMalloc (which may synchronise the device) is not acceptable.  Same
 * arguments, result and errors as attn_bwd minus the workspace: the scratch
 * comes from a fixed array of ATTN_NOALLOC_SCRATCH_BYTES built into the
 * library, which every GPU that loads the library holds until exit.  The call
 * allocates nothing.
 *  - Shapes whose attn_bwd_workspace_bytes() exceeds the array (e.g. more than
 *    about 16 M (B*H*T*D) elements at D=64) return ATTN_ERR_WORKSPACE.
 *  - The first call on each device looks up the array's device address (with
 *    that device current); make that first call before any stream capture.
 *  - All calls on a device share the array; calls that overlap on the GPU
 *    (other streams or host threads on the same device) race and must be
 *    serialised by the caller.  Each call clears what must start at zero. */
#define ATTN_NOALLOC_SCRATCH_BYTES (64u * 1024u * 1024u)
int attn_bwd_noalloc(const void *q, const void *k, const void *v, const void *o,
                     const float *lse, const void *dO, void *dq, void *dk, void *dv,
                     int B, int H, int T, int D, float scale, cudaStream_t stream);

/* ---------------- bf16 path on strided views --------------------------- */

/* Element strides of one [B, H, T, D] operand: from one batch to the next, one
 * head to the next and one token to the next; the D stride is 1.  A
 * contiguous tensor has {H*T*D, T*D, D}.  In nanoGPT's CausalSelfAttention
 * ("nanoGPT — 架构与原理", section 7 code map, and the component table of
 * section 2.2) q, k and v are slices of one c_attn projection [B, T, 3*H*D]
 * and the attention output feeds c_proj as [B, T, H*D]; with strides the
 * kernels read and write those layouts directly, with no transposes:
 *   q: {T*3*H*D, D, 3*H*D} at offset 0, k: the same at offset H*D, v at 2*H*D;
 *   o: {T*H*D, D, H*D}. */
typedef struct {
    int64_t b, h, t;
} attn_strides;

/* attn_fwd on strided views.  strides[0..3] describe q, k, v, o.  Every
 * stride must be a positive multiple of 8 elements (16 bytes), else
 * ATTN_ERR_ALIGN; NULL strides give ATTN_ERR_NULL.  lse stays [B, H, T]
 * contiguous.  Output rows must not overlap one another.  Other rules as
 * attn_fwd. */
int attn_fwd_strided(const void *q, const void *k, const void *v, void *o, float *lse,
                     int B, int H, int T, int D, float scale, const attn_strides *strides,
                     cudaStream_t stream);

/* attn_bwd on strided views.  strides[0..7] describe q, k, v, o, dO, dq, dk,
 * dv (dq/dk/dv may be slices of one [B, T, 3*H*D] buffer for the c_attn
 * backward).  Same stride rules as attn_fwd_strided; workspace as attn_bwd. */
int attn_bwd_strided(const void *q, const void *k, const void *v, const void *o,
                     const float *lse, const void *dO, void *dq, void *dk, void *dv,
                     int B, int H, int T, int D, float scale, const attn_strides *strides,
                     void *workspace, size_t workspace_bytes, cudaStream_t stream);

/* ---------------- options: the mask and attention dropout --------------- */

/* Options of the _ex entry points.  A NULL options pointer means the
 * defaults, which are the decoder's attention computed by attn_fwd/attn_bwd
 * (causal, no dropout).
 *
 * causal: 1 (default) masks key j for query i when j > i -- the -inf upper
 *   triangle that keeps a decoder token from seeing later tokens ("How Andrej
 *   Karpathy built GPT from 200 lines of code", section "Self-Attention: the
 *   mathematical trick" [55:20]).  0 drops the mask: every query attends to
 *   all T keys (the encoder-style attention that the same passage contrasts
 *   with the decoder's), lse_i = ln sum_{j<T} exp(S_ij), and the backward
 *   sums over all i and j.  Any other value gives ATTN_ERR_OPTION.
 *
 * dropout_p, dropout_seed, dropout_offset: attention dropout on the weights
 *   after the softmax, before they meet the values.  The pages train with a
 *   dropout rate ("GPT da zero", table "Come funziona": 0.1) without saying
 *   where in attention it acts; here it is the plain reading, weights zeroed
 *   at random and the kept ones rescaled.  Element (i, j) of head b*H + h is
 *   kept iff 16-bit lane (j mod 8) of Philox4x32-10 (Salmon et al., "Parallel
 *   Random Numbers: As Easy as 1, 2, 3", SC 2011) at counter
 *   (i, j / 8, b*H + h, dropout_offset) under key (low, high word of
 *   dropout_seed) is >= t = floor(dropout_p * 65536 + 1/2); lane e is bits
 *   16 (e mod 2) .. +15 of output word e / 2.  Kept weights are scaled by
 *   65536 / (65536 - t), so p acts rounded to a multiple of 1/65536.
 *   lse stays the log-sum-exp of the undropped scores.  Pass the same seed
 *   and offset to the backward; use a new offset (or seed) per call that
 *   needs a fresh mask (each layer, each step).  0 <= dropout_p < 1 with
 *   t < 65536, else ATTN_ERR_OPTION; t = 0 (p < 1/131072) is no dropout.
 *
 * dropout_mask, dropout_mask_bytes: optional device buffer of at least
 *   attn_dropout_mask_bytes(B,H,T) bytes that keeps the drawn mask, so that
 *   neither the forward's softmax nor the backward runs the generator (its
 *   ten rounds per eight weights otherwise cost each of them about as much
 *   as the attention itself).  With dropout on and dropout_mask != NULL,
 *   attn_fwd_ex first draws the keep bits of every weight the kernels visit
 *   into the buffer (one extra kernel on the same stream) and its attention
 *   kernel loads them; attn_bwd_ex loads them instead of drawing them.  The
 *   buffer must then hold what the forward of the same shape and options
 *   stored (the results equal those of drawing the mask in the kernels).
 *   Layout, for the curious: byte (query i, key group g = j / 8) of head
 *   b*H + h is at ((b*H + h) * Tp + i) * Tp/8 + g with Tp = T rounded up to a
 *   multiple of 128, bit e = key 8 g + e, 1 = kept.  The buffer must be
 *   16-byte aligned (ATTN_ERR_ALIGN otherwise); one smaller than required
 *   gives ATTN_ERR_OPTION.  The float32 entry points and calls without
 *   dropout ignore the two fields.  NULL / 0 (the default): the backward
 *   draws the mask again.
 *
 * reserved: must be 0 (ATTN_ERR_OPTION otherwise). */
typedef struct {
    int32_t causal;
    float dropout_p;
    uint64_t dropout_seed;
    uint32_t dropout_offset;
    uint32_t reserved;
    void *dropout_mask;
    size_t dropout_mask_bytes;
} attn_options;

/* Bytes of a kept dropout mask for a [B, H, T] attention (see attn_options);
 * 0 on a bad shape. */
size_t attn_dropout_mask_bytes(int B, int H, int T);

/* attn_fwd with options, on strided views.  strides: NULL for contiguous
 * [B, H, T, D] tensors, else strides[0..3] for q, k, v, o under the rules of
 * attn_fwd_strided.  opts: NULL for the defaults.  Other rules as attn_fwd. */
int attn_fwd_ex(const void *q, const void *k, const void *v, void *o, float *lse,
                int B, int H, int T, int D, float scale, const attn_strides *strides,
                const attn_options *opts, cudaStream_t stream);

/* attn_bwd with options, on strided views.  strides: NULL for contiguous
 * tensors, else strides[0..7] as attn_bwd_strided.  opts must describe the
 * same attention the forward computed (lse depends on it).  Workspace as
 * attn_bwd (attn_bwd_workspace_bytes). */
int attn_bwd_ex(const void *q, const void *k, const void *v, const void *o,
                const float *lse, const void *dO, void *dq, void *dk, void *dv,
                int B, int H, int T, int D, float scale, const attn_strides *strides,
                const attn_options *opts, void *workspace, size_t workspace_bytes,
                cudaStream_t stream);

/* ---------------- decode: new tokens against kept keys and values ------- */

/* Text generation appends one token at a time and each new token attends to
 * every earlier token and to itself ("nanoGPT — 架构与原理", section 5
 * "边界与局限": nanoGPT's generate has no KV cache and recomputes the whole
 * forward per token).  With the keys and values of all Tk tokens kept, the
 * Tq newest tokens need only their rows of the causal attention:
 *
 *   query r (0 <= r < Tq) is the token at position Tk - Tq + r and attends to
 *   keys 0 .. Tk - Tq + r;  o_r = softmax(scale q_r K^T) V over those keys,
 *   lse_r = ln sum_j exp(scale q_r . k_j) over the same keys.
 *
 * q: bf16 [B, H, Tq, D]; k, v: bf16 [B, H, Tk, D] (the kept keys/values, e.g.
 * the first Tk rows of a cache of larger capacity); o: bf16 [B, H, Tq, D];
 * lse: float32 [B, H, Tq] contiguous.  1 <= Tq <= ATTN_DECODE_MAX_QUERIES and
 * Tq <= Tk (else ATTN_ERR_SHAPE); D 32 or 64.  strides: NULL for contiguous
 * tensors (a cache of capacity Tmax is {H*Tmax*D, Tmax*D, D}), else
 * strides[0..3] for q, k, v, o under the rules of attn_fwd_strided.  Forward
 * only (generation does not differentiate), no dropout, one kernel launch, no
 * workspace.  Other rules as attn_fwd. */
#define ATTN_DECODE_MAX_QUERIES 16
int attn_decode(const void *q, const void *k, const void *v, void *o, float *lse,
                int B, int H, int Tq, int Tk, int D, float scale, const attn_strides *strides,
                cudaStream_t stream);

/* ---------------- float32 path: CUDA cores, IEEE expf -------------------- */

/* Forward in float32 (all tensors float32).  1 <= D <= 128. */
int attn_fwd_f32(const float *q, const float *k, const float *v, float *o, float *lse,
                 int B, int H, int T, int D, float scale, cudaStream_t stream);

/* Bytes of device workspace attn_bwd_f32 needs (Delta [B,H,T], float32). */
size_t attn_bwd_f32_workspace_bytes(int B, int H, int T, int D);

/* Backward in float32.  Same arguments as attn_bwd with float32 tensors. */
int attn_bwd_f32(const float *q, const float *k, const float *v, const float *o,
                 const float *lse, const float *dO, float *dq, float *dk, float *dv,
                 int B, int H, int T, int D, float scale,
                 void *workspace, size_t workspace_bytes, cudaStream_t stream);

/* attn_fwd_f32 / attn_bwd_f32 with options (NULL = defaults); contiguous
 * tensors only.  Workspace as attn_bwd_f32. */
int attn_fwd_f32_ex(const float *q, const float *k, const float *v, float *o, float *lse,
                    int B, int H, int T, int D, float scale, const attn_options *opts,
                    cudaStream_t stream);
int attn_bwd_f32_ex(const float *q, const float *k, const float *v, const float *o,
                    const float *lse, const float *dO, float *dq, float *dk, float *dv,
                    int B, int H, int T, int D, float scale, const attn_options *opts,
                    void *workspace, size_t workspace_bytes, cudaStream_t stream);

/* ---------------- diagnostics ------------------------------------------- */

/* Synchronises `stream`, then reads and clears the current device's
 * in-kernel error flag.  Returns ATTN_OK, ATTN_ERR_TIMEOUT (a bounded wait
 * ran out since the last call), ATTN_ERR_DEVICE_CHECK (the debug build
 * libattn_debug.so only: a kernel's bounds check on a tile coordinate, TMEM
 * column or shared-memory offset failed; the kernel records it and carries
 * on) or ATTN_ERR_CUDA (the sync itself failed, or a kernel found its dynamic
 * shared memory placed too far from a 1024-byte boundary for its tile layout
 * and left without computing). */
int attn_device_error(cudaStream_t stream);

/* Failure-path self test: enqueues one thread that waits on an in-kernel
 * barrier nothing ever completes, gives up after `polls` polls (1 .. 2^22)
 * and sets the error flag, as any timed-out wait in the attention kernels
 * does.  A following attn_device_error() then returns ATTN_ERR_TIMEOUT.
 * Faults nothing and never hangs. */
int attn_selftest_wait_timeout(uint32_t polls, cudaStream_t stream);

/* Self test of the device-side bounds checks: enqueues one kernel that runs
 * a single check that cannot hold and touches no memory.  In the debug build
 * (libattn_debug.so) a following attn_device_error() returns
 * ATTN_ERR_DEVICE_CHECK; the release build compiles the check away, and it
 * returns ATTN_OK. */
int attn_selftest_device_check(cudaStream_t stream);

/* Number of kernels the most recent successful call on this host thread
 * enqueued (for launch accounting). */
int attn_last_launch_count(void);

/* Timing hook: arms the next forward or backward call made on this host
 * thread to record `start` just before and `end` just after enqueueing its
 * main kernel (the forward kernel, or the backward's tile kernel), on the
 * call's stream.  Both are cudaEvent_t handles owned by the caller; the call
 * consumes the arming whether or not it succeeds.  Pass NULLs to disarm. */
typedef struct CUevent_st *cudaEvent_t;
int attn_profile_next_call(cudaEvent_t start, cudaEvent_t end);

/* Library ABI version: 1. */
int attn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* ATTN_H */
