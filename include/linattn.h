/*
 * linattn — kernelised causal linear attention read as a fast-weight update,
 * for NVIDIA B200 (sm_100a).  C ABI of liblinattn.so.
 *
 * The operation (sources by page title and section):
 *   [FW]  "attention is also an FFN" fast-weight article (kwkr.cn/news/587576)
 *   [LN]  linear-attention note (tqpw.cn/news/561043)
 *   [BSA] "Beyond self-attention: what comes after the Transformer"
 *         (datadaily.news, section on linear attention)
 *
 *   phi(x) = elu(x) + 1  (x + 1 for x > 0, exp(x) otherwise; ELU alpha = 1)
 *                        [FW] §4.1, [LN] §4.1, [BSA] linear-attention code
 *   S_i = lambda S_{i-1} + phi(k_i) v_i^T     [FW] §2.1 (recurrence), §3.2 (decay)
 *   z_i = lambda z_{i-1} + phi(k_i)           [FW] §4.2 (normaliser, decayed)
 *   y_i = phi(q_i)^T S_i / (phi(q_i)^T z_i + eps)   [FW] §4.2, [LN] §3
 *
 * Conventions shared by every entry point
 *   - Layouts are contiguous row-major: q, k [B, H, N, dk]; v, out
 *     [B, H, N, dv]; S [B, H, dk, dv] (S[k][v], the [FW] §2.1 / [LN] §3
 *     orientation); z [B, H, dk].  Decode uses N = 1 and drops that axis.
 *   - q, k, v and out share one element type (dims.dtype); S, z, KV and ksum
 *     are always fp32 ([FW] §4.1: the accumulated state must stay fp32).
 *   - q and k are passed raw: phi is applied inside the library (dims.phi =
 *     LINATTN_PHI_ELU1), or they are feature vectors already
 *     (LINATTN_PHI_IDENTITY; the backward then returns gradients with respect
 *     to those features).  Any 1/sqrt(d) scaling is part of the caller's
 *     data, not of the operation.
 *   - lambda points to H fp32 values in device memory (one decay per head),
 *     or is NULL for lambda = 1 (no decay).  Values are used as given; the
 *     method assumes 0 <= lambda <= 1 ([FW] §3.2).  lambda = 0 is allowed
 *     (each token then sees only itself: lambda^0 = 1).
 *   - eps >= 0 is added to the denominator ([FW] §4.2, [LN] §4.1 1e-6).
 *   - Every pointer is a device pointer, 16-byte aligned.  The caller owns
 *     every buffer.  The library keeps no per-call state and never
 *     synchronises; it allocates no memory, except that linattn_bwd_causal
 *     takes its tensor-core workspace as a stream-ordered allocation on
 *     `stream` (linattn_bwd_causal_ws takes the caller's instead).  Work is
 *     queued on `stream` (NULL: the legacy default stream).  Inputs must not
 *     alias outputs.
 *   - Supported sizes: dk and dv in {16, 32, 64, 128}; B, H, N >= 0 with
 *     B*H*N*max(dk,dv) < 2^31.  dtype LINATTN_BF16 or LINATTN_F32.
 *
 * Errors
 *   Arguments are checked on the host before anything is queued; a bad call
 *   returns LINATTN_ERR_INVALID / LINATTN_ERR_UNSUPPORTED and touches nothing.
 *   LINATTN_ERR_CUDA means a launch was refused (cudaGetLastError).  Faults
 *   inside a kernel surface at the caller's next synchronisation.  Kernels
 *   never trap: a bounded wait that runs out records a flag readable with
 *   linattn_device_status().  No C++ exception crosses this interface.
 */
#ifndef LINATTN_H
#define LINATTN_H

#if defined(__GNUC__)
#define LINATTN_API __attribute__((visibility("default")))
#else
#define LINATTN_API
#endif

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t. */
typedef struct CUstream_st *linattn_stream_t;

typedef enum { LINATTN_BF16 = 0, LINATTN_F32 = 1 } linattn_dtype;

/* Feature map the attention calls apply to q and k. */
typedef enum {
    LINATTN_PHI_ELU1 = 0,     /* phi(x) = elu(x) + 1, elementwise (the default) */
    LINATTN_PHI_IDENTITY = 1  /* q and k already hold feature vectors of length dk, e.g. the
                                 random features of linattn_performer_features; they may be
                                 negative, so the denominator may be too */
} linattn_phi;

typedef struct {
    int B;      /* batch */
    int H;      /* heads */
    int N;      /* tokens per sequence (ignored by linattn_decode_step) */
    int dk;     /* key / feature dimension */
    int dv;     /* value dimension */
    int dtype;  /* linattn_dtype of q, k, v and out */
    int phi;    /* linattn_phi; zero-initialised dims mean elu + 1 */
} linattn_dims;

enum {
    LINATTN_OK = 0,
    LINATTN_ERR_INVALID = 1,     /* NULL, negative, misaligned or aliased argument */
    LINATTN_ERR_UNSUPPORTED = 2, /* dk, dv, dtype or size outside the supported set */
    LINATTN_ERR_CUDA = 3,        /* the CUDA runtime refused a launch */
    LINATTN_ERR_DEVICE = 4       /* a kernel recorded a device-side error flag */
};

/*
 * Causal (prefill / training) forward, chunk-parallel
 * ([FW] §3.1 triangular-mask form, §4.1 and §5.2 blockwise accumulation;
 *  recurrence [FW] §2.1, §3.2, §4.2).
 *   q, k   [B, H, N, dk]  dtype      v [B, H, N, dv] dtype
 *   lambda [H] fp32 or NULL          eps >= 0
 *   out    [B, H, N, dv]  dtype      y_i for every token (token i included)
 *   S_final [B, H, dk, dv] fp32 or NULL   state after the last token
 *   z_final [B, H, dk]     fp32 or NULL   normaliser after the last token
 * The starting state is zero ([FW] §4.1 init_state, [LN] §6 init_state).
 * N = 0 writes zero S_final / z_final and nothing else.
 * Kernels: bf16 with dk and dv in {64, 128} runs on the tensor cores (bf16
 * operands, fp32 accumulators and state), one CTA per (b, h) with the whole
 * dv; everything else runs on CUDA cores in fp32 arithmetic.  Both are cut
 * into sequence segments when there are too few heads to fill the GPU and
 * the caller supplies a workspace (linattn_fwd_causal_ws).
 */
LINATTN_API int linattn_fwd_causal(const linattn_dims *dims, const void *q, const void *k,
                       const void *v, const float *lambda, float eps, void *out,
                       float *S_final, float *z_final, linattn_stream_t stream);

/*
 * The same forward continued from a given state: the recurrence of
 * linattn_fwd_causal with S_0 = S_init, z_0 = z_init instead of zero
 * ([FW] §4.1: the fast weights persist across calls; §6: a non-zero
 * initial state), so that
 *   y_i = phi(q_i)^T S_i / (phi(q_i)^T z_i + eps),
 *   S_i = lambda^i S_init + sum_{j<=i} lambda^(i-j) phi(k_j) v_j^T,
 *   z_i = lambda^i z_init + sum_{j<=i} lambda^(i-j) phi(k_j).
 * A prefill of N1 tokens followed by this call on the next N2 tokens with
 * the prefill's S_final / z_final gives the same y, S_final, z_final as one
 * call on N1 + N2 tokens.
 *   S_init [B, H, dk, dv] fp32, z_init [B, H, dk] fp32: both NULL (a zero
 *   state, exactly linattn_fwd_causal) or both device pointers, 16-byte
 *   aligned, owned by the caller, only read, and not overlapping out,
 *   S_final or z_final (LINATTN_ERR_INVALID otherwise; to update a state in
 *   place, alternate two buffers).
 * N = 0 copies S_init / z_init to S_final / z_final.
 */
LINATTN_API int linattn_fwd_causal_from(const linattn_dims *dims, const void *q, const void *k,
                       const void *v, const float *lambda, float eps,
                       const float *S_init, const float *z_init, void *out,
                       float *S_final, float *z_final, linattn_stream_t stream);

/*
 * Segment-parallel causal forward (the "parallel scan" alternative to one
 * sequential pass, [FW] §4.1 note and §5.2, one level above the chunks).  When
 * there are too few (b, h) to fill the GPU, each sequence is cut into G
 * segments: every segment's own final state is computed from zero, the
 * segments' starting states follow from one short scan over them
 * (carry_{g+1} = lambda^len_g carry_g + dS_g), and all segments then run at
 * once.  The result is the recurrence of linattn_fwd_causal_from, up to fp32
 * summation order.
 *
 * linattn_fwd_causal_workspace: the bytes of workspace the segmented form
 *   needs for these dims on this device (0: the single pass is used; also for
 *   invalid dims): B*H*G*(dk*dv + dk)*4 bytes for G segments.  G is chosen so
 *   that B*H*G is about the number of SMs; with B*H above a third of them the
 *   single pass is used.  On the tensor-core path the segment states come from
 *   a tensor-core state pass that reads k and v of every segment but the last
 *   once more.
 * linattn_fwd_causal_ws: linattn_fwd_causal_from with a caller-owned device
 *   workspace (16-byte aligned, overlapping no other argument, contents
 *   irrelevant and overwritten); with workspace_bytes below the size above,
 *   or workspace = NULL, it runs the single pass.
 */
LINATTN_API size_t linattn_fwd_causal_workspace(const linattn_dims *dims);
LINATTN_API int linattn_fwd_causal_ws(const linattn_dims *dims, const void *q, const void *k,
                       const void *v, const float *lambda, float eps,
                       const float *S_init, const float *z_init, void *out,
                       float *S_final, float *z_final, void *workspace,
                       size_t workspace_bytes, linattn_stream_t stream);

/*
 * Kernel family choice, for tests and benchmarks that run the same call on
 * two kernel families (not part of the method; the default is AUTO and
 * nothing needs to call this).  Process-wide; set it only while no call of
 * the library is being made from another thread.
 *   op:       LINATTN_OP_CAUSAL (both causal forwards), LINATTN_OP_GLOBAL,
 *             LINATTN_OP_PERFORMER (linattn_performer_features),
 *             LINATTN_OP_BACKWARD (linattn_bwd_causal)
 *   kernel:   LINATTN_KERNEL_AUTO (the library's choice),
 *             LINATTN_KERNEL_CUDA_CORES (the fp32 CUDA-core kernels),
 *             LINATTN_KERNEL_TC_PAIRED (causal only: the tensor-core kernel
 *             with two CTAs per head, each owning 64 columns of dv; bf16,
 *             dk in {64, 128}, dv a multiple of 64; never segmented)
 *   segments: causal tensor-core path only: 0 lets the library choose G,
 *             G >= 1 asks for at most G segments per sequence (used when the
 *             call has a large enough workspace)
 * Returns LINATTN_ERR_INVALID for an unknown op or kernel, a kernel the op
 * does not have, or segments outside 0..64.
 */
enum { LINATTN_OP_CAUSAL = 0, LINATTN_OP_GLOBAL = 1, LINATTN_OP_PERFORMER = 2,
       LINATTN_OP_BACKWARD = 3 };
enum { LINATTN_KERNEL_AUTO = 0, LINATTN_KERNEL_CUDA_CORES = 1, LINATTN_KERNEL_TC_PAIRED = 2 };
LINATTN_API int linattn_set_kernel_choice(int op, int kernel, int segments);

/*
 * linattn_fwd_causal (zero starting state) for callers that cannot allocate
 * device memory themselves (no cudaMalloc: a host that hands out only fixed
 * buffers, or code that runs where an allocation could block or fail): the
 * segmented form takes its workspace from a 16 MB device array the library
 * holds for every device it is loaded on (until the process exits), and the
 * call falls back to the single pass when the workspace it needs is larger.
 * The paper has no counterpart of this entry point.  It allocates nothing.
 * The array's device address is looked up with cudaGetSymbolAddress on the
 * first call on a device (and again if the device's context has changed), so
 * make that first call before any stream capture.  The array is shared by
 * all calls of this entry point on one device and keeps the last call's
 * contents; calls that overlap on the GPU race on it, so order them (one
 * stream, or streams ordered by events).  It is the only memory the library
 * owns.  Arguments and errors as linattn_fwd_causal.
 */
LINATTN_API int linattn_fwd_causal_noalloc(const linattn_dims *dims, const void *q, const void *k,
                       const void *v, const float *lambda, float eps, void *out,
                       float *S_final, float *z_final, linattn_stream_t stream);

/*
 * State-only causal pass: the fast weights a sequence leaves behind, without
 * its outputs ([FW] §2.1 and §3.2 recurrence, §4.2 normaliser, from a zero
 * start):
 *   S = sum_j lambda^(N-1-j) phi(k_j) v_j^T      z = sum_j lambda^(N-1-j) phi(k_j)
 *   k [B, H, N, dk] dtype, v [B, H, N, dv] dtype, lambda [H] fp32 or NULL
 *   S [B, H, dk, dv] fp32, z [B, H, dk] fp32     written (N = 0: zeros)
 * Equal to the S_final / z_final of linattn_fwd_causal up to fp32 summation
 * order; it reads k and v only.  Its use: the state each segment of a
 * sequence split across devices hands on (see linattn_combine_states).
 * bf16 with dk and dv in {64, 128} runs on the tensor cores, the rest on CUDA
 * cores.  S and z must not overlap k, v or each other.
 */
LINATTN_API int linattn_causal_state(const linattn_dims *dims, const void *k, const void *v,
                       const float *lambda, float *S, float *z, linattn_stream_t stream);

/*
 * Scan of segment states into starting states: the step that joins the
 * segments of the "parallel scan" form ([FW] §4.1 note and §5.2: blocks
 * computed in parallel, the state carried across them).  A sequence is cut
 * into G consecutive segments of dims->N tokens each (the last may be
 * shorter: its length does not enter); dS [G, B, H, dk, dv] and
 * dz [G, B, H, dk] (fp32, slot-major) hold each segment's own final state from
 * zero (linattn_causal_state on that segment).  On return slot g holds the
 * state at the start of segment g:
 *   carry_0 = (S_init, z_init), or zero when both are NULL
 *   carry_{g+1} = lambda^N carry_g + dS_g      (and likewise for z)
 * so that linattn_fwd_causal_from on segment g from slot g continues the
 * whole sequence.  dims.dtype, dims.phi are ignored; 0 <= G <= 64.  S_init,
 * z_init must not overlap dS or dz.
 */
LINATTN_API int linattn_combine_states(const linattn_dims *dims, int G, const float *lambda,
                       const float *S_init, const float *z_init, float *dS, float *dz,
                       linattn_stream_t stream);

/*
 * Backward of linattn_fwd_causal (zero starting state): the gradients of
 * L = sum over all (b, h, i) of dy_i . y_i ([FW] §3.1 and §4.1 train the
 * chunked forward; the gradients follow from the recurrence of [FW] §2.1,
 * §3.2, §4.2 by the chain rule, with phi'(x) = 1 for x > 0 and e^x otherwise).
 *   q, k, v, lambda, eps, dims: as given to the forward
 *   dy      [B, H, N, dv] dtype     upstream gradient of out
 *   dq, dk  [B, H, N, dk] dtype     written
 *   dv      [B, H, N, dv] dtype     written
 *   dlambda [H] fp32 or NULL        written (summed over the batch); with
 *                                   lambda = NULL it is the gradient at 1
 * Every output must overlap no input and no other output.  The forward is
 * recomputed inside (nothing from it is needed).  bf16 with dk = dv = 128
 * runs on the tensor cores (bf16 operands, fp32 accumulation, chunks of 128
 * tokens: a forward pass for dq, a pass for dlambda when it is wanted, a
 * reverse pass for dk and dv); every other shape, fp32, and the CUDA-core
 * choice of linattn_set_kernel_choice(LINATTN_OP_BACKWARD, ...) use fp32
 * arithmetic on CUDA cores.  dlambda is a sum of per-(b, h) fp32 atomics, so
 * its last bits may vary from run to run; dq, dk, dv do not.  The
 * tensor-core passes keep two fp32 numbers per token between them (and, when
 * the forward pass is split, each head's state at the split point) in a
 * stream-ordered allocation made inside the call; if that allocation fails
 * the numbers live in the first 8 bytes of each token's dk row, which is
 * overwritten afterwards.  Either way dk must not be read before the call
 * completes.
 */
LINATTN_API int linattn_bwd_causal(const linattn_dims *dims, const void *q, const void *k,
                       const void *v, const float *lambda, float eps, const void *dy,
                       void *dq, void *dk, void *dv, float *dlambda,
                       linattn_stream_t stream);

/*
 * linattn_bwd_causal_workspace: the bytes of workspace with which
 * linattn_bwd_causal_ws runs its fastest form (0 when the call takes the
 * CUDA-core kernel, which needs none): per-token den, dden (8 bytes per
 * token) and, when the forward pass is split in two halves per head, the
 * state at the split point of every head (66,576 bytes per head).
 *
 * linattn_bwd_causal_ws: linattn_bwd_causal with a caller-owned device
 * workspace instead of a stream-ordered allocation inside the call.
 *   workspace, workspace_bytes: 16-byte aligned, overlapping no input or
 *     output; used from launch to completion of the call on `stream`.  With
 *     fewer bytes than the query returns but at least 8 per token the call
 *     runs unsplit; with fewer than that (or NULL, 0) the per-token numbers
 *     live in the dk rows and the passes run in order (nothing is allocated).
 *   Everything else as linattn_bwd_causal.  NULL with nonzero bytes:
 *   LINATTN_ERR_INVALID.
 */
LINATTN_API size_t linattn_bwd_causal_workspace(const linattn_dims *dims);
LINATTN_API int linattn_bwd_causal_ws(const linattn_dims *dims, const void *q, const void *k,
                       const void *v, const float *lambda, float eps, const void *dy,
                       void *dq, void *dk, void *dv, float *dlambda, void *workspace,
                       size_t workspace_bytes, linattn_stream_t stream);

/*
 * Global (non-causal) forward ([LN] §3 after the sum swap and §6 forward;
 * [BSA] linear-attention code, here with eps):
 *   KV = sum_n phi(k_n) v_n^T, ksum = sum_n phi(k_n),
 *   y_i = phi(q_i)^T KV / (phi(q_i)^T ksum + eps).  No decay: the sum has no order.
 *   out  [B, H, N, dv] dtype
 *   KV   [B, H, dk, dv] fp32, required (written)
 *   ksum [B, H, dk]     fp32, required (written)
 */
LINATTN_API int linattn_fwd_global(const linattn_dims *dims, const void *q, const void *k,
                       const void *v, float eps, void *out, float *KV, float *ksum,
                       linattn_stream_t stream);

/*
 * Cross form of the global forward: the d->N queries of one sequence attend
 * to the Nk keys / values of another ([LN] §6: the multi-head module's target
 * and source lengths; §3 with the sums over the source):
 *   KV = sum_{n<Nk} phi(k_n) v_n^T,  ksum = sum_{n<Nk} phi(k_n),
 *   y_i = phi(q_i)^T KV / (phi(q_i)^T ksum + eps),   i < d->N.
 *   q [B, H, d->N, dk], out [B, H, d->N, dv], k [B, H, Nk, dk], v [B, H, Nk, dv]
 *   dtype; KV, ksum as linattn_fwd_global (written).  Nk = 0 gives KV = 0,
 *   ksum = 0 and y = 0.  linattn_fwd_global is this call with Nk = d->N.
 */
LINATTN_API int linattn_fwd_global_cross(const linattn_dims *dims, int Nk, const void *q,
                       const void *k, const void *v, float eps, void *out, float *KV,
                       float *ksum, linattn_stream_t stream);

/*
 * The global / cross forward with a key padding mask ([LN] §6: the module's
 * forward takes key_padding_mask and its example leaves it out; read here in
 * the usual sense: a key marked as padding is not attended to, so it enters
 * neither sum):
 *   KV = sum_{n<Nk, mask[b][n] = 0} phi(k_n) v_n^T,   ksum likewise,
 *   y_i = phi(q_i)^T KV / (phi(q_i)^T ksum + eps).
 *   key_padding_mask [B, Nk] bytes, nonzero = padding (one row per sequence,
 *   shared by its heads), device memory, not overlapping out, KV or ksum; NULL
 *   means no padding (exactly linattn_fwd_global_cross).  A sequence whose
 *   keys are all padding gets KV = 0, ksum = 0 and y = 0.  Other arguments as
 *   linattn_fwd_global_cross.
 */
LINATTN_API int linattn_fwd_global_masked(const linattn_dims *dims, int Nk, const void *q,
                       const void *k, const void *v, const unsigned char *key_padding_mask,
                       float eps, void *out, float *KV, float *ksum, linattn_stream_t stream);

/*
 * One decode step for every (b, h) ([FW] §4.1 forward_step, §3.1 constant
 * d x d cache; [LN] §5 O(1) per token, §6 forward_autoregressive):
 *   S <- lambda S + phi(k) v^T;  z <- lambda z + phi(k);
 *   out = phi(q)^T S / (phi(q)^T z + eps)       (updated state, token included)
 *   q, k [B, H, dk] dtype    v [B, H, dv] dtype    out [B, H, dv] dtype
 *   S [B, H, dk, dv] fp32 and z [B, H, dk] fp32 are read and updated in place.
 * dims->N is ignored.  A state produced by linattn_fwd_causal (S_final,
 * z_final) continues exactly where the prefill stopped.
 */
LINATTN_API int linattn_decode_step(const linattn_dims *dims, const void *q, const void *k,
                        const void *v, const float *lambda, float eps, float *S,
                        float *z, void *out, linattn_stream_t stream);

/* Static English text for a status code (never NULL). */
/*
 * Performer random features ([LN] §4.2), the feature map to pair with
 * dims.phi = LINATTN_PHI_IDENTITY.  For every row x of x:
 *   out = g(x) / sqrt(m) [cos(omega_1.x) .. cos(omega_m.x), sin(omega_1.x) .. sin(omega_m.x)]
 *   kernel LINATTN_PERFORMER_SOFTMAX:  g(x) = exp(|x|^2 / 2)   (h = 1; phi(x).phi(y)
 *                                      is an unbiased estimate of exp(x.y))
 *   kernel LINATTN_PERFORMER_GAUSSIAN: g(x) = 1   (h(x) = exp(-|x|^2/2), the note's example;
 *                                      the estimate is of exp(-|x-y|^2 / 2))
 *   x     [rows, d]   dtype   e.g. q or k of shape [B, H, N, d] with rows = B*H*N
 *   omega [m, d]      dtype   the projection, drawn by the caller ([LN] §4.2: rows from
 *                             N(0, I_d), optionally orthogonalised, one fixed seed shared by
 *                             every process); the library draws no random numbers
 *   out   [rows, 2m]  dtype   the m cosines, then the m sines
 * d in {16, 32, 64, 128}; m in {8, 16, 32, 64}, so 2m is a supported dk of the attention
 * calls; rows >= 0 with rows * max(d, 2m) < 2^31.  bf16 forms omega.x from the bf16 values
 * with fp32 accumulation (tensor cores when d is 64 or 128 and m is 32 or 64) and rounds
 * the features to bf16; fp32 computes in fp32.  With the softmax kernel g grows as
 * exp(|x|^2 / 2) and overflows to inf for |x|^2 above about 177: keep x small (Performer
 * scales q and k by d^-1/4 before the map).  out must not overlap x or omega; with rows = 0
 * nothing is read or written and the pointers may be NULL.
 */
enum { LINATTN_PERFORMER_SOFTMAX = 0, LINATTN_PERFORMER_GAUSSIAN = 1 };
LINATTN_API int linattn_performer_features(long long rows, int d, int m, int kernel, int dtype,
                                           const void *x, const void *omega, void *out,
                                           linattn_stream_t stream);

LINATTN_API const char *linattn_status_string(int status);

/*
 * Synchronises `stream`, then returns the device-side error word of the
 * current device (0 = no kernel recorded an error; bit 0: a bounded wait
 * ran out).  clear != 0 resets the word afterwards.  Returns -1 if CUDA
 * itself reports an error.
 */
LINATTN_API int linattn_device_status(int clear, linattn_stream_t stream);

/* Library version, major * 10000 + minor * 100 + patch. */
LINATTN_API int linattn_version(void);

#ifdef __cplusplus
}
#endif
#endif /* LINATTN_H */
