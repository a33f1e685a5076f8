/*
 * favor.h -- C ABI of libfavor.so, the FAVOR+ attention hot path for NVIDIA B200 (sm_100a).
 *
 * FAVOR+ ("Fast Attention Via Positive Orthogonal Random Features", the attention of the
 * Performer, "Rethinking Attention with Performers", arXiv 2009.14794) replaces the L x L
 * softmax attention matrix A(i,j) = K(q_i, k_j) by random features phi with
 * K(x, y) = E[phi(x)^T phi(y)] ("Fast Attention Via Positive Orthogonal Random Features",
 * codewithpapers.app/method/favor, the FA-part equations), and evaluates
 *
 *     out = D^-1 (Q' ((K')^T V)),   D = diag(Q' ((K')^T 1_L)),   Q' = phi(Q), K' = phi(K),
 *
 * in time linear in L. This library uses the positive map phi(x) = exp(W x - |x|^2/2) / sqrt(m)
 * with block-orthogonal Gaussian W (m x d), a causal (masked, j <= i) variant by prefix sums
 * ("Random Features for Efficient Attention Approximation", thesis abstract: masked
 * self-attention), and the backward pass with W held fixed.
 *
 * Conventions for every call:
 *   - Tensors are contiguous row-major [B, H, L, d] (d innermost); W is row-major [m, d].
 *   - Device pointers are CUDA global-memory pointers owned by the caller; the library never
 *     frees or retains them. Host pointers are marked "host".
 *   - Q and K are used as given: any d^-1/4 scaling belongs to the caller.
 *   - Outputs and gradients are fp32. With bf16 inputs a bf16 output would by itself exceed a
 *     2e-2 * RMS(out) max-error budget (outputs are averages whose largest entries are ~10x
 *     their RMS), so the output precision is fixed at fp32.
 *   - Calls that take a stream are asynchronous on that stream (a cudaStream_t passed as
 *     void*; NULL is the legacy default stream). Argument errors are reported before any launch.
 *     Device-side conditions (a bounded wait that ran out) are recorded in a device status word
 *     read by favor_sync_status().
 *   - No call allocates device memory. favor_fwd and favor_bwd take their scratch from the
 *     caller's workspace; favor_fwd_static_scratch takes it from the library's own fixed array
 *     (FAVOR_STATIC_SCRATCH_BYTES, a __device__ variable every GPU that loads the library holds).
 *   - Nothing aborts, throws or prints; every call returns a favor_status.
 */
#ifndef FAVOR_H
#define FAVOR_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define FAVOR_API __attribute__((visibility("default")))
#else
#define FAVOR_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    FAVOR_OK = 0,
    FAVOR_ERR_INVALID_ARG = 1,  /* null pointer, non-positive or inconsistent size         */
    FAVOR_ERR_UNSUPPORTED = 2,  /* valid arguments outside what the kernels implement       */
    FAVOR_ERR_CUDA = 3,         /* a CUDA runtime/driver call failed (launch, tensor map)   */
    FAVOR_ERR_TIMEOUT = 4,      /* a device-side bounded wait gave up (see favor_sync_status) */
    FAVOR_ERR_WORKSPACE = 5     /* workspace or ctx pointer null or smaller than required   */
} favor_status;

typedef enum {
    FAVOR_F32 = 0,   /* fp32 Q, K, V, W, dO: CUDA-core fp32 path                           */
    FAVOR_BF16 = 1   /* bf16 Q, K, V, W, dO: tcgen05 tensor-core path, fp32 accumulation   */
} favor_dtype;

/* Problem shape. L >= 1; d in {64, 128}; m a multiple of 16 (fp32 path: 16..512;
 * bf16 path: 64..256, multiple of 64). */
typedef struct {
    int B, H, L, d, m;
    favor_dtype dtype;
} favor_shape;

/* Most kernel launches one call makes (the length of a stage_events array is 2x this). */
#define FAVOR_MAX_STAGES 24

/* Tuning knobs; pass NULL for defaults. Zero fields take their defaults too.
 *   split_tiles : 128-token tiles per causal segment (the unit of the causal key-side reduction
 *                 and of the chunked scan; default 8); the bidirectional path spreads its key
 *                 tiles over the SMs by itself
 *   exp_poly_pct: percent (1..100) of feature exponentials evaluated by the FMA-pipe
 *                 polynomial instead of the MUFU ex2 unit (bf16 path), in every kernel; a
 *                 negative value puts all of them on MUFU; 0 takes each kernel's default (a
 *                 quarter in the d = 64 query output kernel, none elsewhere)
 *   feature_map : the random-feature map (bf16 bidirectional forward only; other calls refuse a
 *                 non-default map with FAVOR_ERR_UNSUPPORTED):
 *                 FAVOR_MAP_POSITIVE (0, default): phi(x) = exp(Wx - |x|^2/2)/sqrt(m), FAVOR+;
 *                 FAVOR_MAP_RELU: phi(x) = max(Wx, 0)/sqrt(m), generalised (kernelizable)
 *                 attention with the degree-1 arc-cosine kernel ("Rethinking Attention with
 *                 Performers", abstract: attention mechanisms beyond softmax);
 *                 FAVOR_MAP_TRIG: phi(x) = exp(|x|^2/2)/sqrt(m) [sin(Wx), cos(Wx)] (2m features),
 *                 the trigonometric softmax features of FAVOR ("Random Features for Efficient
 *                 Attention Approximation", thesis abstract: FAVOR to FAVOR+). Its normaliser can
 *                 be negative or near zero on large-norm inputs; exp(|k|^2/2) must stay in fp32
 *                 range (|k|^2 < 170).
 *   stage_events: NULL, or 2 * FAVOR_MAX_STAGES caller-created cudaEvent_t handles (as void*);
 *                 the call records events[2k] before and events[2k+1] after its k-th kernel
 *                 launch on the call's stream (NULL entries are skipped). For timing. */
#define FAVOR_MAP_POSITIVE 0
#define FAVOR_MAP_RELU 1
#define FAVOR_MAP_TRIG 2
typedef struct {
    int split_tiles;
    int exp_poly_pct;
    int feature_map;
    int reserved[5];
    void **stage_events;
} favor_opts;

/*
 * favor_draw_features -- draw the block-orthogonal random feature matrix W (host only).
 *
 * Positive *orthogonal* random features ("Rethinking Attention with Performers" abstract; the
 * summary page's limitations: orthogonality holds within blocks of at most d rows). W has
 * ceil(m/d) independent blocks; block b is a d x d Gaussian matrix from Philox4x64-10 keyed by
 * (seed, 0), counter (n/4, b, 0, 0), Box-Muller pairs; its rows are orthonormalised by modified
 * Gram-Schmidt with one re-orthogonalisation pass, then each row i is scaled by an independent
 * chi(d) norm sqrt(sum of d squared Gaussians from counter (n/4, b, 1, 0)). The last block is
 * truncated to its first rows. Every step is one IEEE double operation in a fixed order, so the
 * result is reproducible bit for bit.
 *
 *   seed   : any 64-bit value
 *   m, d   : W is m x d; 1 <= m, 1 <= d <= 1024
 *   W_host : host, caller-owned, m*d doubles, row-major; written on FAVOR_OK only
 * Returns FAVOR_ERR_INVALID_ARG on a null pointer or bad size.
 */
FAVOR_API favor_status favor_draw_features(uint64_t seed, int m, int d, double *W_host);

/*
 * favor_workspace_size -- bytes of device workspace favor_fwd (backward = 0) or favor_bwd
 * (backward = 1) needs for this shape, causal flag and options (NULL = defaults).
 * Returns 0 for an invalid or unsupported shape.
 */
FAVOR_API size_t favor_workspace_size(const favor_shape *shape, int causal, int backward, const favor_opts *opts);

/*
 * favor_ctx_size -- bytes of the forward-to-backward context (per-head key stabiliser,
 * per-key norms and the fp32 state (K')^T [V | 1_L]). Returns 0 for an invalid shape.
 */
FAVOR_API size_t favor_ctx_size(const favor_shape *shape, int causal);

/*
 * favor_fwd -- FAVOR+ forward: out = D^-1 (Q' ((K')^T V)) (causal = 0, the bidirectional
 * FA-part) or out_i = phi(q_i)^T S_i / phi(q_i)^T z_i with prefix sums S_i, z_i over j <= i
 * (causal = 1).
 *
 *   shape        : host pointer
 *   Q, K, V      : device, [B,H,L,d] in shape->dtype
 *   W            : device, [m,d] in shape->dtype (the caller rounds the fp64 draw)
 *   causal       : 0 or 1
 *   out          : device, fp32 [B,H,L,d]; fully written
 *   ctx          : device, favor_ctx_size bytes, or NULL when no backward will follow (the bf16
 *                  forward writes the per-head key reference, and the causal path the per-key
 *                  -|k|^2/2, into it)
 *   workspace    : device, >= favor_workspace_size(shape, causal, 0, opts) bytes, 256-B aligned
 *   stream       : cudaStream_t as void*
 * Numerics: query features are stabilised by their row maximum. Key features, bidirectional: each
 * persistent CTA keeps a per-feature stabiliser over its run of key tiles, and the runs are brought
 * to one per-(batch, head) reference before the state is used; causal: the per-(batch, head)
 * maximum key logit. All of them cancel exactly in D^-1. Inputs Q, K, V, W, out must be 16-byte
 * aligned.
 */
FAVOR_API favor_status favor_fwd(const favor_shape *shape, const void *Q, const void *K, const void *V,
                       const void *W, int causal, float *out, void *ctx, void *workspace,
                       size_t ws_bytes, const favor_opts *opts, void *stream);

/*
 * favor_bwd -- gradients of sum(dout * out) with respect to Q, K, V, with W fixed.
 * (Derived by the chain rule from the forward definition; the pages print no backward.)
 *
 *   Q, K, V, W   : as passed to favor_fwd
 *   out          : device, fp32 [B,H,L,d], the forward output (validated, not read: the kernels
 *                  recompute out_i at the precision of the gradient passes)
 *   dout         : device, [B,H,L,d] in shape->dtype, upstream gradient
 *   ctx          : bf16: device, required, the context favor_fwd wrote for the same inputs and
 *                  mask; the backward reads the per-head key reference from it (the largest key
 *                  stabiliser of the forward), which keeps its key features below 2^19.
 *                  fp32: not read (may be NULL); the fp32 kernels recompute everything.
 *   dQ, dK, dV   : device, fp32 [B,H,L,d]; fully written
 *   workspace    : device, >= favor_workspace_size(shape, causal, 1, opts) bytes
 * bf16 arithmetic: every operand computed on the way (phi(Q), phi(K), the state, [g | s], the
 * query-side sums, phi * dphi) is a pair of bf16 values hi + lo, and each product is three tcgen05
 * MMAs (two where one side is an exact bf16 input), accumulated in fp32: the gradients' largest
 * entries are 50-90x their RMS, beyond what single 16-bit operands resolve within 2e-2 x RMS.
 * Returns FAVOR_ERR_WORKSPACE for a missing (bf16) context or short workspace, FAVOR_ERR_UNSUPPORTED
 * for a feature map other than the positive one or an unsupported shape (bf16 causal: d = 64).
 */
FAVOR_API favor_status favor_bwd(const favor_shape *shape, const void *Q, const void *K, const void *V,
                       const void *W, const float *out, const void *dout, const void *ctx,
                       int causal, float *dQ, float *dK, float *dV, void *workspace,
                       size_t ws_bytes, const favor_opts *opts, void *stream);

/*
 * favor_sync_status -- synchronise the stream, then return and clear the device status word
 * (FAVOR_ERR_TIMEOUT if a bounded wait inside a kernel gave up since the last call;
 * FAVOR_ERR_UNSUPPORTED if a bf16 forward met a V entry of magnitude 2^23 or more, or a non-finite
 * one: the values reach the fp16 tensor-core operands scaled by at most 2^-7 per key tile (the
 * causal path scales each 1024-key segment further, by 2^-b, b as needed), and such outputs are not
 * valid), or
 * FAVOR_ERR_CUDA if the stream reports an error.
 */
FAVOR_API favor_status favor_sync_status(void *stream);

/*
 * favor_decode_state_size -- bytes of the carried state of favor_decode_step for shape's B*H
 * heads (shape->L is ignored here): per head (d*m + 2*m) fp32. Returns 0 for an unsupported shape
 * (d in {64, 128}; m a multiple of 32, at most 256).
 */
FAVOR_API size_t favor_decode_state_size(const favor_shape *shape);

/*
 * favor_decode_step -- the masked FA-part advanced by one token per head: the prefix-sum
 * recurrence S_t = S_{t-1} + phi(k_t) v_t^T, z_t = z_{t-1} + phi(k_t),
 * out_t = phi(q_t)^T S_t / phi(q_t)^T z_t ("Random Features for Efficient Attention
 * Approximation", abstract: masked self-attention; the causal form of the FA-part equations on
 * "Fast Attention Via Positive Orthogonal Random Features", codewithpapers.app/method/favor).
 * Feeding tokens 0..t one call at a time gives the rows of favor_fwd(..., causal = 1).
 *
 *   shape        : host pointer; L must be 1 (one token per head per call); B, H, d, m, dtype
 *   q, k, v      : device, [B,H,d] in shape->dtype (this token's query, key and value)
 *   W            : device, [m,d] in shape->dtype
 *   state        : device, favor_decode_state_size(shape) bytes, read and updated in place. Per
 *                  head (b*H + h): S'[c][r] (d x m), z'[r] (m), D[r] (m), fp32, with
 *                  sum_j exp(u_r(k_j)) v_j[c] = exp(D[r]) S'[c][r] and
 *                  sum_j exp(u_r(k_j)) = exp(D[r]) z'[r], u_r(x) = w_r.x - |x|^2/2. An all-zero
 *                  buffer is the empty state (a feature with z'[r] = 0 holds no token).
 *   out          : device, fp32 [B,H,d]; fully written
 *   stream       : cudaStream_t as void*
 * All pointers 16-byte aligned. Arithmetic is fp32 for either dtype. Returns FAVOR_ERR_INVALID_ARG
 * (null or misaligned pointer, L != 1), FAVOR_ERR_UNSUPPORTED (d not 64/128, m not a multiple of
 * 32 up to 256), FAVOR_ERR_CUDA (launch failure).
 */
FAVOR_API favor_status favor_decode_step(const favor_shape *shape, const void *q, const void *k, const void *v,
                                         const void *W, float *state, float *out, void *stream);

/*
 * Sequence-parallel bidirectional forward (bf16). The keys of one sequence may be spread over
 * several calls -- one per rank, each holding a contiguous run of every head's tokens: the FA-part
 * needs only the sums (K')^T V and (K')^T 1_L over all keys ("Fast Attention Via Positive
 * Orthogonal Random Features", codewithpapers.app/method/favor, the FA-part equations), and sums
 * over disjoint runs add. favor_sp_state writes a run's partial [S | z]; the caller adds the
 * partial states of all runs (an all-reduce SUM across ranks); favor_sp_output then gives the
 * outputs of any run of queries from the total.
 *
 * Every partial state is taken against the same per-feature offsets c_r = |w_r|^2/2 - 40 (natural
 * log units), fixed by W alone: since u_r(k) = w_r.k - |k|^2/2 <= |w_r|^2/2 for every key, the key
 * features exp(u_r(k) - c_r) never exceed e^40, and partial states from different calls add
 * directly. Operands are carried as bf16 hi + lo pairs (fp32 accumulation), as in the backward.
 *
 * State layout (device, fp32, favor_sp_state_size bytes): [B*H][m][d + 64]; column c < d holds
 * sum_j exp(u_r(k_j) - c_r) v_j[c], column d the same sum of 1, the other columns zero.
 */
FAVOR_API size_t favor_sp_state_size(const favor_shape *shape);
/* favor_sp_workspace_size -- device workspace bytes of either call for this (local) shape; 0 if
 * unsupported (bf16; d in {64, 128}; m in {128, 256}). */
FAVOR_API size_t favor_sp_workspace_size(const favor_shape *shape);
/*
 * favor_sp_state -- partial state of the keys K, V (device, [B,H,L,d] bf16, L = this run's length)
 * with W ([m,d] bf16): state (device, fp32, favor_sp_state_size bytes) is fully written.
 * Returns FAVOR_ERR_INVALID_ARG (null or misaligned pointer, bad size), FAVOR_ERR_UNSUPPORTED,
 * FAVOR_ERR_WORKSPACE, FAVOR_ERR_CUDA.
 */
FAVOR_API favor_status favor_sp_state(const favor_shape *shape, const void *K, const void *V, const void *W,
                                      float *state, void *workspace, size_t ws_bytes, void *stream);
/*
 * favor_sp_output -- out_i = phi(q_i)^T S / phi(q_i)^T z for the queries Q (device, [B,H,L,d] bf16,
 * L = this run's length) against state (device, fp32: the sum of the partial states of all key
 * runs); out (device, fp32 [B,H,L,d]) is fully written. Errors as favor_sp_state.
 */
FAVOR_API favor_status favor_sp_output(const favor_shape *shape, const void *Q, const void *W, const float *state,
                                       float *out, void *workspace, size_t ws_bytes, void *stream);

/* favor_status_string -- static, never-NULL description of a status code. */
FAVOR_API const char *favor_status_string(favor_status status);

/*
 * favor_selftest_bounded_wait -- exercises the bounded device-side wait every kernel uses (the
 * pages have no counterpart: this is a diagnostic of the library's failure reporting). One CTA
 * waits on a shared-memory barrier that nothing arrives on, through the same bounded wait, with a
 * limit of limit_us microseconds; the wait gives up, records FAVOR_ERR_TIMEOUT in the device status
 * word, the CTA frees its tensor memory and returns. No copy or MMA is in flight, the context stays
 * usable, and the next favor_sync_status(stream) returns FAVOR_ERR_TIMEOUT (and clears it).
 *
 *   limit_us : 1 .. 1000000
 *   stream   : cudaStream_t as void*
 * Returns FAVOR_ERR_INVALID_ARG for a limit outside that range, FAVOR_ERR_CUDA if the launch fails.
 */
FAVOR_API favor_status favor_selftest_bounded_wait(unsigned int limit_us, void *stream);

/* Size of the library's own fixed scratch array used by favor_fwd_static_scratch (32 MiB). */
#define FAVOR_STATIC_SCRATCH_BYTES (32u << 20)

/*
 * favor_fwd_static_scratch -- bidirectional bf16 forward that allocates nothing and takes no
 * workspace. (The paper has no counterpart: this is an interface for callers that cannot
 * allocate device memory -- code running inside another allocator's callback, where a nested
 * cudaMalloc would recurse, or in a process whose device memory is fully reserved by a
 * framework's caching allocator.)
 *
 * Computes exactly what favor_fwd(shape, Q, K, V, W, causal = 0, out, ctx = NULL, ...) computes,
 * with the same kernels; the scratch comes from a fixed array of FAVOR_STATIC_SCRATCH_BYTES in
 * the library's device memory, which every GPU that loads the library holds until process exit.
 *
 *   shape        : host pointer; dtype must be FAVOR_BF16
 *   Q, K, V, W   : device, as for favor_fwd (16-byte aligned)
 *   out          : device, fp32 [B,H,L,d]; fully written
 *   stream       : cudaStream_t as void*
 * Returns FAVOR_ERR_WORKSPACE when favor_workspace_size(shape, 0, 0, NULL) exceeds
 * FAVOR_STATIC_SCRATCH_BYTES, FAVOR_ERR_UNSUPPORTED for fp32 or unsupported shapes.
 *
 * The first call on a device (with that device current) looks up the array's device address
 * with cudaGetSymbolAddress; make that first call before any stream capture. Every call on a
 * device shares the one array: calls that overlap on the GPU (different streams, no ordering
 * between them) race on it. No part of the array has to start at zero; each call overwrites
 * everything it reads. Calls no cudaMalloc, cudaFree or allocating library routine. The device
 * address is cached per device for the life of the process: a cudaDeviceReset between calls is not
 * supported.
 */
FAVOR_API favor_status favor_fwd_static_scratch(const favor_shape *shape, const void *Q, const void *K,
                                                const void *V, const void *W, float *out, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* FAVOR_H */
