/*
 * retnet.h -- C interface of the B200 (sm_100a) RetNet multi-scale retention library
 * (libretnet.so).
 *
 * What it computes.  Retention as defined in "阅读笔记：RetNet" (mzeromiko blog, reading
 * notes on arXiv 2307.08621):
 *   - §2.2 Recurrent Mode:   S_n = gamma S_{n-1} + K_n^T V_n,  o_n = Q_n S_n
 *   - §2.3 Parallel Mode:    O = (Q K^T (.) D) V,  D_nm = gamma^(n-m) for n >= m, else 0,
 *                            Q = (X W_Q) (.) Theta, K = (X W_K) (.) conj(Theta), Theta_n = e^{in.theta}
 *   - §2.4 Chunkwise Recurrent Mode: per chunk i of B tokens,
 *                            R_i = K_[i]^T (V_[i] (.) zeta) + gamma^B R_{i-1},  zeta_r = gamma^(B-1-r)
 *                            O_[i] = (Q_[i] K_[i]^T (.) D) V_[i] + (Q_[i] R_{i-1}) (.) xi,  xi_r = gamma^(r+1)
 *   - §三.2 MSR: per-head gamma, Y = GroupNorm_h(heads), out = swish(G) (.) Y
 *   - §三.3 Normalization: QK^T / sqrt(d), D~ (rows of D divided by the root of their sum),
 *                          R~ (rows of the score matrix divided by max(|row sum|, 1))
 *
 * Readings where the page is silent (the library and its tests follow these):
 *   - xPos on real tensors: elements (2j, 2j+1) of a head vector are one complex number;
 *     q and k of the token at absolute position p are both turned by the angle p*theta[j].
 *     Their real dot product is then Re[(q e^{in.theta})(k e^{im.theta})^dagger], a function
 *     of n-m only.
 *   - Positions are 0-based absolute: token t of a call is at p = pos0 + t.  D~ divides row p
 *     by c_p = sqrt(sum_{j=0..p} gamma^j), the number of decayed tokens seen so far.
 *   - Chunk rows r are 0-based: xi_r = gamma^(r+1), zeta_r = gamma^(b'-1-r) with b' the
 *     chunk's actual length (the tail chunk may be shorter than B).
 *   - The recurrent step updates the state with token n before reading it (D_nn = 1).
 *   - GroupNorm: groups are heads, biased variance over d_v, eps inside the root, unit affine;
 *     swish(g) = g * sigmoid(g).
 *
 * Layout ("BLHD", dense, row-major, no strides):
 *   q, k : [batch][seqlen][heads][d_k]     v, o : [batch][seqlen][heads][d_v]
 *   state: [batch][heads][d_k][d_v] fp32   z    : [batch][heads][d_k] fp32 (key-sum state)
 *   MSR y, g, out: [tokens][heads][d_v]
 *
 * Ownership and memory.  The caller owns every buffer.  Tensor arguments (q, k, v, o, state,
 * z, y, g, out) are DEVICE pointers on the current CUDA device.  gamma and theta are HOST
 * pointers, read before the call returns (their values travel to the kernels as launch
 * parameters).  The library allocates no device memory, frees nothing, and keeps no
 * per-call state.
 *
 * Asynchrony.  Every compute call enqueues its kernels on `stream` (a cudaStream_t; NULL is
 * the legacy default stream) and returns without synchronising.  Outputs are valid once the
 * stream reaches that point.
 *
 * Errors.  Arguments are checked on the host before any launch; a bad argument returns a
 * status and enqueues nothing.  A failed launch returns RETNET_ERR_CUDA.  No exception
 * crosses this interface and no kernel traps.  Devices other than sm_100 return
 * RETNET_ERR_UNSUPPORTED.
 *
 * Precision.  fp32 inputs are computed in fp32 on the CUDA cores.  bf16 inputs of the
 * chunkwise call, for the shapes listed at retnet_retention_chunkwise, run on the tensor
 * cores (tcgen05) with fp16 operands and fp32 accumulation: bf16 q, k, v convert to fp16
 * exactly, the rotated q, k, the masked scores and the chunk state are rounded to fp16 once
 * each.  fp16 has three more mantissa bits than bf16 and a smaller range, so finite results
 * need |q|, |k|, |v| < 32768, |q.k| / sqrt(d_k) < 65504 and state entries below
 * 65504 * sqrt(d_k); the kernels count every rounding outside that range
 * (retnet_fp16_range_errors), so a call that left it is detected rather than silent.
 * RETNET_F_PRECISE (and R~, and the fused MSR call) carries each rounded operand as two fp16
 * numbers, hi = fp16(x) and lo = fp16(x - hi), and sums the hi*hi, lo*hi and hi*lo products:
 * about 22 significant bits per operand, at about twice the tensor-core work; the results
 * then agree with an fp64 evaluation to about 1e-5 of their rms.
 */
#ifndef RETNET_H
#define RETNET_H

#include <stddef.h>
#include <stdint.h>

/* Exported symbols of libretnet.so (the library is built with hidden default visibility). */
#if defined(__GNUC__)
#define RETNET_API __attribute__((visibility("default")))
#else
#define RETNET_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    RETNET_OK = 0,
    RETNET_ERR_NULL_PTR = 1,    /* a required pointer is NULL */
    RETNET_ERR_BAD_SHAPE = 2,   /* a size is <= 0 (or < 0 where 0 is allowed), or over a limit */
    RETNET_ERR_BAD_DTYPE = 3,   /* dtype value not in retnet_dtype_t, or combination unsupported */
    RETNET_ERR_BAD_PARAM = 4,   /* gamma not in (0,1), chunk <= 0, odd d_k with XPOS, eps < 0,
                                   negative position, unknown flag bits, non-finite theta */
    RETNET_ERR_UNSUPPORTED = 5, /* e.g. NORM_R on a step call without z, or not an sm_100 device */
    RETNET_ERR_CUDA = 6         /* a CUDA runtime/driver call or a launch failed */
} retnet_status_t;

typedef enum { RETNET_F32 = 0, RETNET_BF16 = 1 } retnet_dtype_t;

/* Normalisation / position flags (bitwise OR). */
enum {
    RETNET_F_XPOS = 1u,         /* xPos rotation of q and k (§2.3 Theta) */
    RETNET_F_SCALE_SQRT_D = 2u, /* QK^T / sqrt(d_k) (§三.3) */
    RETNET_F_NORM_D = 4u,       /* D~ row normalisation (§三.3) */
    RETNET_F_NORM_R = 8u,       /* R~ normalisation by max(|row sum|, 1) (§三.3) */
    RETNET_F_PRECISE = 16u      /* tensor-core kernel with split fp16 operands (see Precision) */
};

typedef struct {
    int64_t batch, seqlen, heads, d_k, d_v;
} retnet_dims_t;

/* Limits checked on the host (RETNET_ERR_BAD_SHAPE beyond them). */
#define RETNET_MAX_HEADS 256
#define RETNET_MAX_DK 512
#define RETNET_MAX_DV 1024

/*
 * Parallel form (§2.3 with §三.3): o = ((Q K^T) * s (.) D~) V / max(|row sum|, 1), the flags
 * choosing which factors apply.  A fresh sequence whose first token sits at absolute
 * position pos0 >= 0 (pos0 moves the rotation and the D~ row counts; no earlier tokens
 * contribute).  q, k, v: in_dtype; o: out_dtype.  gamma: host float[heads] in (0,1);
 * theta: host float[d_k/2] (may be NULL without RETNET_F_XPOS).  seqlen may be 0 (no work).
 * Kernels: bf16 inputs without RETNET_F_NORM_R, on the shapes the tensor-core chunkwise kernel
 * takes (see retnet_retention_chunkwise), run on the tensor cores: a sequence of up to 512
 * tokens as one masked tile of 64, 128, 256 or 512 rows (the O(seqlen^2) product itself), a
 * longer one in 512-token chunks (the same sum re-associated, §2.4).  Other calls run the fp32
 * CUDA-core kernel, O(seqlen^2) per (batch, head).
 */
RETNET_API retnet_status_t retnet_retention_parallel(const void* q, const void* k, const void* v, void* o,
                                          retnet_dims_t dims, retnet_dtype_t in_dtype,
                                          retnet_dtype_t out_dtype, const float* gamma,
                                          const float* theta, int64_t pos0, uint32_t flags,
                                          void* stream);

/*
 * Chunkwise recurrent form (§2.4) with chunk length `chunk` (> 0); the result equals the
 * parallel form's up to rounding, and continues from a carried state.
 *   state_in : device fp32 [batch][heads][d_k][d_v], the state S before the first token
 *              (the recurrent S_{pos0-1}); NULL means zeros.
 *   state_out: device fp32, same shape; receives the state after the last token; may be NULL;
 *              may alias state_in.
 *   z_in/z_out: device fp32 [batch][heads][d_k], the key-sum state (gamma z + k) that the
 *              R~ row sum needs across calls; read/written only with RETNET_F_NORM_R; NULL
 *              means zeros / not written.
 * Kernels: bf16 q, k, v without RETNET_F_NORM_R, with d_k in {64, 128, 256}, d_v a multiple
 * of 64, chunk in {64, 128, 256, 512}, 16-byte aligned tensors and gamma^T >= 2^-12 for every
 * head (T = 64, or 128 when d_k <= 128 and chunk >= 128: the sub-block the kernel scales its
 * fp16 operands within) run on the tcgen05 tensor-core kernel; every other case runs on the
 * fp32 CUDA-core kernel.  retnet_chunkwise_kernel reports which one a call takes.
 */
RETNET_API retnet_status_t retnet_retention_chunkwise(const void* q, const void* k, const void* v, void* o,
                                           retnet_dims_t dims, retnet_dtype_t in_dtype,
                                           retnet_dtype_t out_dtype, const float* gamma,
                                           const float* theta, int64_t pos0, uint32_t flags,
                                           int64_t chunk, const float* state_in, float* state_out,
                                           const float* z_in, float* z_out, void* stream);

/*
 * retnet_retention_chunkwise with a caller-owned device workspace.  The result is the same
 * function of the same arguments (§2.4 read as a scan over chunks: R_i = gamma^B R_{i-1} +
 * K_[i]^T (V_[i] (.) zeta) is associative, so the chunks may be cut into consecutive segments
 * whose own states are combined by R = gamma^len R + W).  When the tensor-core kernel runs
 * with fewer (batch, head, d_v slice) units than SMs, it cuts the sequence into up to four
 * segments: a first launch computes the states of the earlier segments (cut again into
 * sub-segments, up to six states) in parallel, a second produces every segment's outputs
 * starting from state_in carried over the earlier sub-segments.  Without a workspace the same split runs as one launch in which each later segment
 * first replays the earlier chunks' state.
 *   workspace: device memory, 16-byte aligned, workspace_bytes long, not overlapping any other
 *              argument; its contents on entry are irrelevant and are overwritten.  It holds,
 *              with RETNET_F_NORM_R, first the R~ row factors (fp32 [batch][seqlen][heads])
 *              and the key-sum pass's segment values (fp32 [batch * heads][64][d_k]), each
 *              rounded up to 256 bytes: §三.3's R~ then runs on the tensor-core kernel, a key-
 *              sum pass over q and k before it, z_in/z_out carried by that pass; without the
 *              room R~ runs on the CUDA-core kernel; then either the sub-segment states
 *              (fp32, one is batch * heads * d_k * d_v * 4 bytes; fewer than one means no
 *              split of this kind) or, for chunks of several 64-row sub-blocks without a
 *              split, fp16 copies of q, k, v that a conversion pre-pass writes once.
 *              retnet_chunkwise_workspace_size gives the size that allows all of it.  The
 *              workspace is in use until the call's work on `stream` completes; two calls
 *              sharing one workspace must be ordered on the device.
 * Other arguments, errors and kernels as retnet_retention_chunkwise; a misaligned workspace
 * is RETNET_ERR_BAD_PARAM.
 */
RETNET_API retnet_status_t retnet_retention_chunkwise_ws(const void* q, const void* k, const void* v, void* o,
                                              retnet_dims_t dims, retnet_dtype_t in_dtype,
                                              retnet_dtype_t out_dtype, const float* gamma,
                                              const float* theta, int64_t pos0, uint32_t flags,
                                              int64_t chunk, const float* state_in, float* state_out,
                                              const float* z_in, float* z_out, void* workspace,
                                              size_t workspace_bytes, void* stream);

/*
 * Sequence sharding (§2.4 read as an associative scan over chunks; sequence-parallel use
 * across GPUs).  The state a sequence leaves behind from a zero start,
 *   W = sum_t gamma^(L-1-t) rot_{pos0+t}(k_t)^T v_t      -> state_out [batch][heads][d_k][d_v] fp32,
 * without outputs (q is not needed).  A shard of a longer sequence starting at position pos0
 * contributes W; the state after it is gamma^L R_before + W (retnet_state_advance).  Runs the
 * tensor-core state pass: the shapes and dtypes of the tensor-core chunkwise kernel (bf16,
 * no RETNET_F_NORM_R), else RETNET_ERR_UNSUPPORTED.  k, v as for retnet_retention_chunkwise.
 */
RETNET_API retnet_status_t retnet_chunkwise_segment_state(const void* k, const void* v, retnet_dims_t dims,
                                               retnet_dtype_t in_dtype, const float* gamma,
                                               const float* theta, int64_t pos0, uint32_t flags,
                                               int64_t chunk, float* state_out, void* stream);

/*
 * state <- gamma_h^len * state + w, in place, for fp32 [batch][heads][d_k][d_v] states (the
 * combination step of a sequence split into shards: R after a shard of len tokens whose own
 * state is w).  gamma: host float[heads]; gamma^len is taken in fp64.  state and w 16-byte
 * aligned, d_k * d_v a multiple of 4; they may not overlap unless equal.
 */
RETNET_API retnet_status_t retnet_state_advance(float* state, const float* w, int64_t batch, int64_t heads,
                                     int64_t d_k, int64_t d_v, const float* gamma, int64_t len,
                                     void* stream);

/*
 * Allocation-free variant of retnet_retention_chunkwise_ws.  The pages have no counterpart:
 * it is the same computation with the segment states kept in a static device array of
 * RETNET_STATIC_SCRATCH_BYTES inside the library (one per device), for callers that cannot
 * allocate device memory -- hosts that link only this C library and have no device
 * allocator, or code that must not allocate on its hot path (cudaMalloc / cudaFree
 * synchronise the device).  The library allocates nothing for it.
 *   Limits: a call whose single segment state, batch * heads * d_k * d_v * 4 bytes, exceeds
 *   RETNET_STATIC_SCRATCH_BYTES returns RETNET_ERR_UNSUPPORTED (use the _ws form with a
 *   workspace of retnet_chunkwise_workspace_size bytes instead); smaller calls use as many
 *   segment states as fit.
 *   Zeroing: nothing in the scratch has to start at zero; every call overwrites what it reads.
 *   Concurrency: the scratch is shared by every call on a device, so calls whose work
 *   overlaps on the GPU (two streams, two host threads) race on it and give wrong results;
 *   order them on the device.
 *   R~: with RETNET_F_NORM_R the row factors and the key-sum values (the front region that
 *   retnet_chunkwise_workspace_size describes) take the front of the scratch when they fit,
 *   and R~ then runs on the tensor-core kernel; when they do not fit, the call runs on the
 *   fp32 CUDA-core kernel (retnet_chunkwise_launches with RETNET_STATIC_SCRATCH_BYTES tells).
 *   Set-up: every call looks up the scratch's address in the current device's context (a
 *   host-side CUDA symbol query, nothing cached, so a device reset leaves no stale address);
 *   the first call on a device may load the library's module there, so make it outside any
 *   stream capture.
 * Other arguments, results and errors as retnet_retention_chunkwise.
 */
#define RETNET_STATIC_SCRATCH_BYTES (16u << 20)
RETNET_API retnet_status_t retnet_retention_chunkwise_static(const void* q, const void* k, const void* v, void* o,
                                                  retnet_dims_t dims, retnet_dtype_t in_dtype,
                                                  retnet_dtype_t out_dtype, const float* gamma,
                                                  const float* theta, int64_t pos0, uint32_t flags,
                                                  int64_t chunk, const float* state_in, float* state_out,
                                                  const float* z_in, float* z_out, void* stream);

/*
 * Workspace size (bytes) that lets retnet_retention_chunkwise_ws use all its forms for these
 * dimensions, with a256(x) = x rounded up to a multiple of 256:
 *   a256(4 * batch * seqlen * heads)                        (R~ row factors)
 *   + a256(4 * batch * heads * d_k * 64)                     (R~ key-sum segment values)
 *   + max(6 * batch * heads * d_k * d_v * 4,                 (six sub-segment states)
 *         4 * a256(2 * batch * seqlen * heads * d_k) + a256(2 * batch * seqlen * heads * d_v),
 *                                                            (fp16 copies of q, k (hi and lo), v)
 *         2 * a256(2 * batch * seqlen * heads * d_k) + a256(2 * batch * seqlen * heads * d_v)
 *         + P)                                               (fp16 copies, then the P tiles)
 *   with P = a256(batch * heads * ceil(seqlen / 512) * 36 * 64 * 64 * 2) for d_k = 256, else 0
 *   (the masked score tiles that the P pass computes once per head, for chunks of 128 to 512).
 * Host-only; no device access.  RETNET_ERR_NULL_PTR without `bytes`, RETNET_ERR_BAD_SHAPE for
 * negative sizes.
 */
RETNET_API retnet_status_t retnet_chunkwise_workspace_size(retnet_dims_t dims, size_t* bytes);

/*
 * One recurrent decode step (§2.2) for a whole batch: for the token at absolute position
 * pos >= 0, S <- gamma S + k^T v in place, then o = (q S) * s / c_pos / max(|s/c_pos q.z|, 1)
 * as the flags ask (z <- gamma z + k in place with RETNET_F_NORM_R, which requires z).
 *   q, k: [batch][heads][d_k] in_dtype;  v: [batch][heads][d_v] in_dtype;
 *   o: [batch][heads][d_v] out_dtype;  state: device fp32 [batch][heads][d_k][d_v], in/out.
 * The state is read once and written once per call (the call is HBM-bound).  o must not
 * overlap the state.
 */
RETNET_API retnet_status_t retnet_retention_step(const void* q, const void* k, const void* v, void* o,
                                      int64_t batch, int64_t heads, int64_t d_k, int64_t d_v,
                                      retnet_dtype_t in_dtype, retnet_dtype_t out_dtype,
                                      float* state, float* z, const float* gamma,
                                      const float* theta, int64_t pos, uint32_t flags,
                                      void* stream);

/*
 * MSR epilogue (§三.2): for every (token, head) row of d_v values of y, GroupNorm with the
 * biased variance and eps >= 0 inside the root, unit affine, then multiply by swish(g).
 *   y, g: [tokens][heads][d_v] in_dtype;  out: same shape, out_dtype (may alias y when the
 *   dtypes match).  tokens may be 0.  d_v must be a multiple of 8 and <= RETNET_MAX_DV.
 */
RETNET_API retnet_status_t retnet_msr_epilogue(const void* y, const void* g, void* out, int64_t tokens,
                                    int64_t heads, int64_t d_v, float eps, retnet_dtype_t in_dtype,
                                    retnet_dtype_t out_dtype, void* stream);

/*
 * Chunkwise retention with the MSR epilogue (§三.2) fused into the tensor-core kernel:
 *   out = swish(g) (.) GroupNorm_h(o),  o the output retnet_retention_chunkwise_ws would write,
 * with the GroupNorm of retnet_msr_epilogue (per (token, head) row of d_v values, biased
 * variance, eps >= 0 inside the root, unit affine).  The retention output itself is never
 * written to memory: the d_v / 64 CTAs of a (batch, head) form one thread-block cluster and
 * pool each row's statistics in distributed shared memory.
 *   q, k, v, state_in, state_out, gamma, theta, pos0, flags, chunk, workspace: as for
 *   retnet_retention_chunkwise_ws (the workspace only feeds the conversion pre-pass of chunks
 *   of several sub-blocks; sequences are never split into segments here).
 *   g:   gate [batch][seqlen][heads][d_v] in_dtype, 16-byte aligned;
 *   out: [batch][seqlen][heads][d_v] out_dtype, must not overlap q, k, v or g.
 * Handled: what the tensor-core kernel handles (retnet_chunkwise_kernel == 1: bf16 inputs,
 * d_k in {64, 128, 256}, no RETNET_F_NORM_R, ...) with d_v in {64, 128, 192, 256}.
 * Anything else returns RETNET_ERR_UNSUPPORTED without touching the device; run
 * retnet_retention_chunkwise_ws then retnet_msr_epilogue for those.  seqlen == 0 copies
 * state_in to state_out (or clears it) as the other chunkwise entry points do.
 */
RETNET_API retnet_status_t retnet_msr_chunkwise(const void* q, const void* k, const void* v, const void* g,
                                     void* out, retnet_dims_t dims, retnet_dtype_t in_dtype,
                                     retnet_dtype_t out_dtype, const float* gamma, const float* theta,
                                     int64_t pos0, uint32_t flags, int64_t chunk, float eps,
                                     const float* state_in, float* state_out, void* workspace,
                                     size_t workspace_bytes, void* stream);

/*
 * Gradient of the retention forward, for training (§2.4: training runs the chunkwise form,
 * whose outputs are those of the parallel form §2.3, so this is the derivative of that
 * definition).  With q~, k~ the xPos-rotated rows, f_n the row factor of §三.3 and S0 =
 * state_in (the state before the first token, as for retnet_retention_chunkwise):
 *   O_n = f_n [ sum_{m<=n} gamma^(n-m) (q~_n . k~_m) v_m + gamma^(n+1) q~_n S0 ],
 * and for a loss with gradient dout = dL/dO:
 *   dq, dk: [batch][seqlen][heads][d_k] fp32;  dv: [batch][seqlen][heads][d_v] fp32;
 *   dstate: [batch][heads][d_k][d_v] fp32, dL/dS0 (may be NULL: not computed).
 *   q, k, v, dout in in_dtype (dout laid out as v); state_in fp32 or NULL (zeros).
 *   workspace: device memory, 16-byte aligned: retnet_backward_workspace_size bytes for either
 *   path (at least 2 * 4 * batch * seqlen * heads * d_k for the CUDA-core path).
 * Paths: bf16 inputs with d_k and d_v in {64, 128, 256} and a workspace of
 * retnet_backward_workspace_size bytes run on the tensor cores: each gradient sum has the shape
 * of a retention output (dq: query dO, key v, value k~; dk: read backwards, query v, key dO,
 * value f q~; dv: backwards, query k, key q, value f dO), so three runs of the chunkwise kernel
 * compute them: k~, f q~ and f dO, which are not bf16 numbers, go in as fp16 value rows (one
 * rounding to 11 significant bits; max|err|/rms <= 1e-2), counted by retnet_fp16_range_errors
 * where they leave the fp16 range.  Every other call runs on fp32 CUDA cores, O(seqlen^2) per
 * (batch, head).
 * d_k, d_v <= 256 and seqlen <= 524280, else RETNET_ERR_UNSUPPORTED; RETNET_F_NORM_R (R~, a
 * division by a function of q and k) is RETNET_ERR_UNSUPPORTED.  Outputs do not alias inputs.
 */
RETNET_API retnet_status_t retnet_retention_backward(const void* q, const void* k, const void* v,
                                          const void* dout, float* dq, float* dk, float* dv,
                                          retnet_dims_t dims, retnet_dtype_t in_dtype,
                                          const float* gamma, const float* theta, int64_t pos0,
                                          uint32_t flags, const float* state_in, float* dstate,
                                          void* workspace, size_t workspace_bytes, void* stream);

/*
 * Workspace bytes that let retnet_retention_backward take the tensor-core path where it
 * applies (bf16 and fp16 operands of the three chunkwise runs, their fp32 outputs, S0^T and the
 * runs' segment states); at least 2 * 4 * batch * seqlen * heads * d_k, what the CUDA-core path
 * needs.
 */
RETNET_API retnet_status_t retnet_backward_workspace_size(retnet_dims_t dims, size_t* bytes);

/*
 * Which path retnet_retention_backward takes for these arguments with a workspace of
 * workspace_bytes (host-only; assumes 16-byte aligned buffers): 1 = tensor cores (three runs of
 * the chunkwise forward kernel), 0 = fp32 CUDA cores, negative = the negated status.
 */
RETNET_API int retnet_backward_kernel(retnet_dims_t dims, retnet_dtype_t in_dtype, uint32_t flags,
                                      const float* gamma, size_t workspace_bytes);

/*
 * Kernel launches retnet_retention_backward makes for these arguments (with_state: state_in
 * given; with_dstate: dstate requested); negative = the negated status.  Reads the device's SM
 * count on the tensor-core path; no device memory is touched.
 */
RETNET_API int retnet_backward_launches(retnet_dims_t dims, retnet_dtype_t in_dtype, uint32_t flags,
                                        const float* gamma, size_t workspace_bytes, int with_state,
                                        int with_dstate);

/*
 * Which kernel retnet_retention_chunkwise runs for these arguments (host-only decision, no
 * device access): 1 = the tcgen05 tensor-core kernel, 0 = the fp32 CUDA-core kernel,
 * negative = the arguments would be rejected (the negated status).  Device pointers that
 * are not 16-byte aligned also send a call to the CUDA-core kernel; this query assumes
 * aligned buffers.  gamma: host float[heads].
 */
RETNET_API int retnet_chunkwise_kernel(retnet_dims_t dims, retnet_dtype_t in_dtype, uint32_t flags, int64_t chunk,
                                       const float* gamma);

/*
 * Kernel launches retnet_retention_chunkwise_ws makes for these arguments on the current
 * device (workspace_bytes = 0: retnet_retention_chunkwise): 0 without tokens; else 1, or 2
 * when a pre-pass runs first (the two-pass sequence segments' state pass, or the conversion
 * pre-pass), plus, with RETNET_F_NORM_R on the tensor-core path, the key-sum pass (1 launch,
 * or 2 when it cuts the sequence into segments); negative = the negated status the call would
 * return.  Reads the device's SM count; no device memory is touched.  gamma: host
 * float[heads].  Assumes 16-byte aligned buffers, as retnet_chunkwise_kernel does.
 */
RETNET_API int retnet_chunkwise_launches(retnet_dims_t dims, retnet_dtype_t in_dtype, uint32_t flags, int64_t chunk,
                                         const float* gamma, size_t workspace_bytes);

/*
 * Kernel launches retnet_msr_chunkwise makes for these arguments on the current device: 0
 * without tokens, 1 (the fused kernel), 2 (conversion pre-pass + fused kernel, for chunks of
 * several sub-blocks when workspace_bytes covers the fp16 copies); negative = the negated
 * status the call would return (-RETNET_ERR_UNSUPPORTED for shapes it does not handle).
 * Same assumptions as retnet_chunkwise_launches.
 */
RETNET_API int retnet_msr_chunkwise_launches(retnet_dims_t dims, retnet_dtype_t in_dtype, uint32_t flags,
                                             int64_t chunk, const float* gamma, size_t workspace_bytes);

/*
 * Number of bounded waits that gave up inside the tensor-core kernel since the last clear
 * (a kernel that hits one abandons its output, releases what it holds and returns rather
 * than hang).  Synchronises with the device.  With clear != 0 the count is reset to 0.
 * Returns RETNET_OK or RETNET_ERR_CUDA; *count receives the value before any clear.
 */
RETNET_API retnet_status_t retnet_debug_wait_timeouts(unsigned int* count, int clear);

/*
 * Testing aid for the bounded waits above: sets, for the tensor-core kernels of the current
 * device, how many SM clock cycles a wait for another role's progress may last before it gives
 * up (cycles > 0, at least 100), or restores the default of 4e9 cycles (about 2 s; cycles <= 0).
 * With a small budget waits give up: the kernel then stops its work, waits with the full budget
 * for the TMA copies and MMAs it already issued, frees its tensor memory and returns; the
 * outputs of such a call are undefined and retnet_debug_wait_timeouts counts the give-ups.
 * Not for production calls.  Synchronises with the device.  RETNET_OK, RETNET_ERR_BAD_PARAM
 * (0 < cycles < 100) or RETNET_ERR_CUDA.
 */
RETNET_API retnet_status_t retnet_debug_set_wait_budget(long long cycles);

/*
 * Count of device threads that, since the last clear, rounded a tensor-core operand outside
 * the fp16 range (a magnitude of 65520 or more becomes inf; a NaN counts too): the scaled,
 * rotated q and k, v, the masked scores or the fp16 state copy (see Precision), and the fp16
 * value rows of the gradient's runs (retnet_retention_backward).  A call whose
 * bf16 inputs leave that range produces non-finite outputs on the tensor-core kernel and
 * raises this count; the fp32 CUDA-core kernel (fp32 inputs) has no such limit.  Synchronises
 * with the device; with clear != 0 the count is reset to 0.  Returns RETNET_OK or
 * RETNET_ERR_CUDA; *count receives the value before any clear.
 */
RETNET_API retnet_status_t retnet_fp16_range_errors(unsigned int* count, int clear);

/* Static, NUL-terminated description of a status code (never NULL). */
RETNET_API const char* retnet_status_string(retnet_status_t status);

/* Library version as major*10000 + minor*100 + patch. */
RETNET_API int retnet_version(void);

#ifdef __cplusplus
}
#endif

#endif /* RETNET_H */
