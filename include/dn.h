/*
 * dn.h -- C ABI of the B200 (sm_100a) causal delta-rule layer.
 *
 * The layer keeps, per sequence b and head h, a state S of d_k x d_v fp32
 * values (row i = key channel, column j = value channel) and for every token
 * t runs
 *
 *     forget   S~  = decay_t(S)          (none | exp(g_t) S | Diag(exp(g_t)) S)
 *     predict  p   = S~^T k_t
 *     correct  e   = beta_t (v_t - p)
 *     write    S   = S~ + k_t e^T
 *     read     o_t = S^T (scale q_t)     (after the write)
 *
 * i.e. S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T
 * with alpha_t = exp(g_t) (decay first; for a scalar alpha this is
 * alpha_t (I - beta_t k_t k_t^T) S_{t-1} + beta_t k_t v_t^T).  Sources: "Linear attention and Gated DeltaNet"
 * (inference.shantanugoel.com, ch. 28), sections "Correct: the delta rule",
 * "Gated DeltaNet" and "The recurrent form" (the contract: q, k [B,H,T,Dk]
 * already L2-normalised, v [B,H,T,Dv], g and beta [B,H,T], optional initial
 * state [B,H,Dk,Dv], returning o and the final state); section "The chunked
 * form" (same contract and result, computed chunk by chunk); D2L 12.5
 * "DeltaNet", slides "One rule, two readings" and "Gating: the modern cell";
 * and "A walk through of the DeltaNet family of linear attention variants"
 * (selinyilmaz.dev), its KDA update with a per-key-channel decay.
 *
 * Conventions for every entry point
 *   - All tensor pointers are DEVICE pointers owned by the caller.  The
 *     library keeps no state between calls except a per-device status word
 *     read by dn_device_status(), and allocates no device memory except the
 *     tensor-core prefill's workspace when the caller passes none (a
 *     stream-ordered cudaMallocAsync / cudaFreeAsync pair on the call's
 *     stream; see dn_chunk_fwd_workspace_size).
 *   - Every layout is dense row-major (C order) with the shapes given.
 *   - Calls are asynchronous on `cuda_stream` (a cudaStream_t; NULL = the
 *     legacy default stream).  Inputs must stay valid until the work ends.
 *   - The return value is a dn_status.  Nothing throws or aborts across the
 *     ABI.  On DN_ERR_INVALID / DN_ERR_UNSUPPORTED nothing was launched and
 *     no output was touched; dn_last_error() gives the reason.
 *   - beta is not clamped (values in (0, 2) give the negative-eigenvalue
 *     transitions of D2L 12.5, "The reflection hiding in the delta rule").
 *     g is the log-decay (alpha = exp(g)); g <= 0 is expected but not
 *     enforced.  k is not normalised by the library, except by the *_gdn
 *     entry points, which take raw q and k and normalise both.
 *   - Pointers to q, k, v, o, S0, S_T and S must be 16-byte aligned, as must a
 *     per-key g; beta and a scalar g 4-byte aligned.
 */
#ifndef DN_H
#define DN_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define DN_API __attribute__((visibility("default")))
#else
#define DN_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    DN_OK = 0,
    DN_ERR_INVALID = 1,      /* null required pointer, bad size, misalignment, aliasing */
    DN_ERR_UNSUPPORTED = 2,  /* valid request this library does not implement */
    DN_ERR_CUDA = 3,         /* a CUDA call or kernel launch failed */
    DN_ERR_TIMEOUT = 4       /* a bounded device wait gave up (see dn_device_status) */
} dn_status;

typedef enum { DN_F32 = 0, DN_BF16 = 1 } dn_dtype;   /* storage type of q, k, v and o */

typedef enum {
    DN_GATE_NONE = 0,     /* DeltaNet: alpha = 1, g must be NULL            */
    DN_GATE_SCALAR = 1,   /* Gated DeltaNet: g [B,H,T] (decode: [B,H])       */
    DN_GATE_PER_KEY = 2   /* KDA: g [B,H,T,d_k] (decode: [B,H,d_k])          */
} dn_gate;

typedef enum {
    DN_PATH_AUTO = 0,     /* tensor-core path when it supports the request, else SIMT */
    DN_PATH_SIMT = 1,     /* fp32 CUDA-core chunk kernel: any chunk 1..64          */
    DN_PATH_TC = 2,       /* tcgen05 chunk kernels: bf16, chunk 64, d_k = d_v = 128, any gate */
    /* Self-test of the failure path: the tensor-core kernels run with their input
     * loads withheld, so every bounded wait inside them expires (about two seconds);
     * nothing is written to o or S_T, dn_device_status() then returns
     * DN_ERR_TIMEOUT, and the CUDA context stays usable. */
    DN_PATH_TC_STALL_TEST = 3
} dn_path;

/*
 * dn_chunk_fwd -- chunked prefill ("The chunked form", ch. 28).
 *
 *   q     [B,H,T,d_k]  dtype   queries (multiplied by `scale` inside)
 *   k     [B,H,T,d_k]  dtype   keys
 *   v     [B,H,T,d_v]  dtype   values
 *   beta  [B,H,T]      fp32    write strengths
 *   g     NULL | [B,H,T] | [B,H,T,d_k]  fp32 log-decay, per `gate`
 *   S0    NULL (zero state) | [B,H,d_k,d_v] fp32, read only
 *   o     [B,H,T,d_v]  dtype   output, o_t read after token t's write
 *   S_T   NULL (not written) | [B,H,d_k,d_v] fp32 final state; may equal S0
 *         exactly (in-place continuation), must not partly overlap it
 *   chunk tokens per chunk; the result does not depend on it beyond rounding
 *         (the last chunk may be partial: it equals zero padding with g = 0,
 *         beta = 0).  SIMT path: 1..64; tensor-core path: 64.
 *   d_k, d_v in {64, 128}.  B, H, T >= 0 (T = 0 writes S_T = S0 or zeros).
 *
 * o must not overlap any input.  Returns DN_ERR_UNSUPPORTED for a d or chunk
 * outside the ranges above (or a DN_PATH_TC request the tensor-core kernels
 * do not cover).  The kernels are chosen as by DN_PATH_AUTO; a workspace the
 * tensor-core path needs is allocated and freed stream-ordered on
 * `cuda_stream` (pass one to dn_chunk_fwd_ex to avoid that).
 */
DN_API int dn_chunk_fwd(const void* q, const void* k, const void* v,
                 const float* beta, const float* g, const float* S0,
                 void* o, float* S_T,
                 int B, int T, int H, int d_k, int d_v, int chunk, float scale,
                 dn_dtype dtype, dn_gate gate, void* cuda_stream);

/*
 * dn_chunk_fwd_workspace_size -- bytes of device workspace that dn_chunk_fwd_ex
 * uses for this request on `path` (0 when the chosen kernels need none).  The
 * tensor-core path computes W = T diag(beta e^G) K, u = T diag(beta) V and the
 * intra-chunk attention P of every chunk ("Training it: the WY trick", D2L
 * 12.5; "The chunked form", ch. 28) in a kernel that runs over all chunks at
 * once, then streams them into the sequential state pass: 40.25 KiB (W, u, P and,
 * for the layer prologue's output rows, 1 / ||q|| of each position) and a 4-byte
 * ready flag per (b, h, chunk), and a 4-byte tile counter, i.e. with
 * n = B * H * ceil(T / 64) chunks, n * 41216 + (4 (n + 1) rounded up to a
 * multiple of 256) bytes.  With the per-key
 * gate (KDA: "A walk through of the DeltaNet family of linear attention
 * variants") each chunk also keeps q and k with their decays applied and the
 * chunk's decay per key channel: 72.75 KiB per chunk, n * 74496 + (4 (n + 1)
 * rounded up to a multiple of 256) bytes.  Its gram splits the decays around one
 * reference position per 16-token block, so the tensor-core result is exact up
 * to rounding while no key channel decays by more than e^-80 over 8
 * consecutive tokens (the SIMT path has no such bound).  Sizes are checked as
 * in dn_chunk_fwd_ex; *bytes is written on DN_OK only.
 */
DN_API int dn_chunk_fwd_workspace_size(int B, int T, int H, int d_k, int d_v, int chunk,
                                       dn_dtype dtype, dn_gate gate, dn_path path, size_t* bytes);

/*
 * dn_chunk_fwd with an explicit kernel choice and workspace.
 *   workspace        NULL: when the kernels need one, the call allocates it
 *                    stream-ordered on `cuda_stream` and frees it there;
 *                    otherwise a device buffer of at least
 *                    dn_chunk_fwd_workspace_size() bytes, 256-byte aligned,
 *                    overlapping no argument.  Its contents are scratch
 *                    (overwritten; nothing needs initialising) and it must not
 *                    be used by other work until this call's work has ended.
 *   workspace_bytes  its size (ignored when workspace is NULL).
 */
DN_API int dn_chunk_fwd_ex(const void* q, const void* k, const void* v,
                    const float* beta, const float* g, const float* S0,
                    void* o, float* S_T,
                    int B, int T, int H, int d_k, int d_v, int chunk, float scale,
                    dn_dtype dtype, dn_gate gate, dn_path path,
                    void* workspace, size_t workspace_bytes, void* cuda_stream);

/*
 * dn_chunk_fwd_snapshots -- dn_chunk_fwd_ex that also writes the state at
 * chunk boundaries.  An engine keeps such snapshots to roll a request back
 * after rejected speculative tokens and to cache prefixes at block boundaries
 * ("Linear attention and Gated DeltaNet", ch. 28, "The state a request
 * carries").
 *   snaps  NULL (no snapshots, as dn_chunk_fwd_ex) or [B,H,n_snap,d_k,d_v]
 *          fp32, 16-byte aligned, overlapping no other argument, with
 *          n_snap = floor(T / (every * chunk)): snapshot s is the state after
 *          the first (s + 1) * every * chunk tokens of each (b, h), the value
 *          S_T would have for that prefix.  A partial last chunk has none.
 *   every  chunks between snapshots, >= 1 (DN_ERR_INVALID otherwise).
 * Everything else is as for dn_chunk_fwd_ex.  On the tensor-core path each
 * snapshot costs one extra write of 64 KiB per head.
 */
DN_API int dn_chunk_fwd_snapshots(const void* q, const void* k, const void* v,
                                  const float* beta, const float* g, const float* S0,
                                  void* o, float* S_T, float* snaps, int every,
                                  int B, int T, int H, int d_k, int d_v, int chunk, float scale,
                                  dn_dtype dtype, dn_gate gate, dn_path path,
                                  void* workspace, size_t workspace_bytes, void* cuda_stream);

/*
 * dn_chunk_fwd_gdn -- the Gated DeltaNet prefill with the layer's prologue
 * fused into the kernels ("Linear attention and Gated DeltaNet", ch. 28, "The
 * full layer", steps 4 and 5): the rule runs on
 *   q / max(||q||, 1e-12), k / max(||k||, 1e-12)  (norms over d_k, per token),
 *   beta = sigmoid(b),  g = -exp(A_log[h]) * softplus(a + dt_bias[h])
 * (softplus(x) = log(1 + e^x)), as dn_chunk_fwd with the scalar gate on these.
 *   q, k  [B,H,T,d_k] bf16, raw (not normalised);  v [B,H,T,d_v] bf16
 *   b, a  [B,H,T] fp32 raw write-strength and decay inputs, 4-byte aligned
 *   A_log, dt_bias  [H] fp32 per head, 4-byte aligned, required
 *   S0, o, S_T, scale, workspace, workspace_bytes, cuda_stream as dn_chunk_fwd_ex
 * Tensor-core path only: d_k = d_v = 128 (chunk 64); DN_ERR_UNSUPPORTED
 * otherwise.  The workspace is the scalar gate's (dn_chunk_fwd_workspace_size
 * with DN_BF16, DN_GATE_SCALAR, DN_PATH_TC).
 */
DN_API int dn_chunk_fwd_gdn(const void* q, const void* k, const void* v, const float* b, const float* a,
                            const float* A_log, const float* dt_bias, const float* S0, void* o, float* S_T,
                            int B, int T, int H, int d_k, int d_v, float scale,
                            void* workspace, size_t workspace_bytes, void* cuda_stream);

/* Flags of the *_gdn_ex entry points. */
enum {
    /* beta = 2 sigmoid(b), in (0, 2): the write-strength gate of D2L 12.5, "The
     * reflection hiding in the delta rule", whose transitions I - beta k k^T reach
     * the eigenvalue 1 - beta < 0 (allow_neg_eigval) */
    DN_GDN_BETA_2SIGMOID = 1,
    /* the *_gdn_ex entry points with z: the gated RMSNorm's gate is sigmoid(z) instead of SiLU(z) */
    DN_GDN_NORM_SIGMOID = 2
};

/*
 * dn_chunk_fwd_gdn_ex -- dn_chunk_fwd_gdn on either kernel path, with flags.
 * Same prologue and arguments as dn_chunk_fwd_gdn, plus
 *   chunk, dtype, path   as dn_chunk_fwd_ex: the tensor-core kernels (bf16,
 *         d_k = d_v = 128, chunk 64) or the fp32 CUDA-core kernel (fp32 or bf16
 *         tokens, d in {64, 128}, chunk 1..64), which normalises q and k and
 *         derives beta and g in the same way
 *   flags DN_GDN_BETA_2SIGMOID: beta = 2 sigmoid(b); DN_GDN_NORM_SIGMOID: the
 *         norm's gate is sigmoid(z), else SiLU(z); other bits return DN_ERR_INVALID
 *   z, norm_weight, eps   NULL, NULL, 0: o is the rule's read-out [B,H,T,d_v].
 *         Else the layer's gated RMSNorm (ch. 28, "The full layer", step 7) runs
 *         on the output rows inside the kernels (tensor-core path only):
 *         z [B,T,H,d_v] dtype (token-major, 16-byte aligned), norm_weight [d_v]
 *         fp32 shared by every head, eps in (0, 1], and o receives
 *         y = norm_weight * o / sqrt(mean(o^2) + eps) * act(z) token-major
 *         [B,T,H,d_v], the layout of z (the mean over each head's d_v channels)
 * The workspace is dn_chunk_fwd_workspace_size's for the scalar gate and the
 * chosen path (zero on the CUDA-core path).
 */
DN_API int dn_chunk_fwd_gdn_ex(const void* q, const void* k, const void* v, const float* b, const float* a,
                               const float* A_log, const float* dt_bias, const float* S0, void* o, float* S_T,
                               int B, int T, int H, int d_k, int d_v, int chunk, float scale, dn_dtype dtype,
                               dn_path path, int flags, const void* z, const float* norm_weight, float eps,
                               void* workspace, size_t workspace_bytes, void* cuda_stream);

/*
 * dn_chunk_fwd_noalloc -- dn_chunk_fwd for callers that cannot allocate device
 * memory (a process that reserved the device's memory for its own pools, a
 * framework whose allocator must see every byte, or a latency-critical loop
 * that cannot afford an allocation or its implicit synchronisation).  The
 * pages have no counterpart: it is a deployment variant of dn_chunk_fwd.
 *
 * Same arguments, kernel choice and results as dn_chunk_fwd.  The tensor-core
 * path's scratch workspace (dn_chunk_fwd_workspace_size bytes) comes from a
 * fixed area of DN_NOALLOC_SCRATCH_BYTES compiled into the library; no call
 * allocates or frees memory.
 *   - The area exists once per device, created when the library's code is
 *     loaded there, and is held until the process exits.
 *   - Every call looks up the area's address (cudaGetSymbolAddress, with the
 *     call's device current) and keeps nothing: after a cudaDeviceReset the
 *     library's code is loaded again and the area may have moved.
 *   - Capacity: a (b, h, chunk) tile takes 41,216 bytes with no gate or the
 *     scalar gate (about 1628 tiles fit, e.g. B*H = 12 at T = 8192) and
 *     74,496 bytes with the per-key gate (about 900 tiles, e.g. B*H = 7 at
 *     T = 8192), plus 4 bytes of ready flag per tile.
 *   - A request needing more scratch than the area returns DN_ERR_UNSUPPORTED
 *     (dn_last_error() gives both sizes) before any device work.
 *   - Every call on a device shares the area and it keeps the last call's
 *     contents.  Nothing in it needs clearing (each call writes every byte it
 *     reads), but calls whose GPU work overlaps (other streams, other host
 *     threads) race on it: order them on one stream, or use dn_chunk_fwd_ex
 *     with separate workspaces.
 */
#define DN_NOALLOC_SCRATCH_BYTES ((size_t)64 << 20)   /* 64 MiB */

DN_API int dn_chunk_fwd_noalloc(const void* q, const void* k, const void* v,
                                const float* beta, const float* g, const float* S0,
                                void* o, float* S_T,
                                int B, int T, int H, int d_k, int d_v, int chunk, float scale,
                                dn_dtype dtype, dn_gate gate, void* cuda_stream);

/*
 * dn_chunk_fwd_gva -- the chunked prefill with grouped value heads ("Linear
 * attention and Gated DeltaNet", ch. 28, "The full layer", step 3: the
 * layer projects fewer key heads than value heads, and each key head's q and
 * k serve a group of value heads).
 *
 *   q, k      [B,H_k,T,d_k] dtype   H_k key heads
 *   v, o      [B,H,T,d_v]   dtype   H value heads, H a multiple of H_k
 *   beta      [B,H,T] fp32;  g NULL | [B,H,T] fp32 (per value head)
 *   S0, S_T   [B,H,d_k,d_v] fp32 (per value head), as for dn_chunk_fwd
 *   workspace as for dn_chunk_fwd_ex, dn_chunk_fwd_workspace_size(B, T, H, ...)
 *             bytes (value heads); NULL allocates it stream-ordered
 *
 * Value head h of batch row b runs the rule of dn_chunk_fwd on q[b, h / R],
 * k[b, h / R] with R = H / H_k, and its own v, beta, g and state.  The
 * tensor-core kernels load each key head's tiles by its row, so no repeated
 * copy of q and k is formed.  Tensor-core path only: bf16, d_k = d_v = 128,
 * chunk 64, gate DN_GATE_NONE or DN_GATE_SCALAR; other requests return
 * DN_ERR_UNSUPPORTED.  H % H_k != 0 returns DN_ERR_INVALID.
 */
DN_API int dn_chunk_fwd_gva(const void* q, const void* k, const void* v, const float* beta, const float* g,
                            const float* S0, void* o, float* S_T, int B, int T, int H_k, int H, int d_k,
                            int d_v, float scale, dn_dtype dtype, dn_gate gate, void* workspace,
                            size_t workspace_bytes, void* cuda_stream);

/*
 * dn_chunk_fwd_varlen -- the chunked prefill of a packed batch ("Linear
 * attention and Gated DeltaNet", ch. 28, "The state a request carries": each
 * request carries its own fixed-size state).  N sequences of different lengths
 * share one time axis; sequence s holds tokens cu_seqlens[s] ..
 * cu_seqlens[s + 1] - 1 and runs the rule of dn_chunk_fwd from its own S0[s]
 * to its own S_T[s], chunked from its own first token.
 *
 *   q, k        [H,T,d_k] dtype;  v, o [H,T,d_v] dtype  (B = 1, T tokens in all)
 *   beta        [H,T] fp32;  g NULL | [H,T] fp32 (DN_GATE_NONE or DN_GATE_SCALAR)
 *   S0, S_T     NULL | [N,H,d_k,d_v] fp32, as for dn_chunk_fwd
 *   cu_seqlens  DEVICE int32 [N + 1], non-decreasing from 0 to T; N >= 1;
 *               empty sequences are allowed (their S_T is S0, or zeros)
 *   workspace   dn_chunk_fwd_varlen_workspace_size bytes, 256-byte aligned, or
 *               NULL (allocated stream-ordered on cuda_stream)
 *
 * Tensor-core path: bf16, d_k = d_v = 128 (chunk 64); else DN_ERR_UNSUPPORTED.
 * The kernels read cu_seqlens on the device (no host synchronisation): one
 * small kernel builds the chunk tables in the workspace, then the WY kernel
 * covers every chunk and the state pass every (sequence, head).  If
 * cu_seqlens does not rise from 0 to T, nothing is computed (o is left as it
 * was, S_T = S0) and the next dn_device_status() returns DN_ERR_INVALID.
 */
DN_API int dn_chunk_fwd_varlen(const void* q, const void* k, const void* v, const float* beta, const float* g,
                               const float* S0, void* o, float* S_T, const int* cu_seqlens, int N, int T,
                               int H, int d_k, int d_v, float scale, dn_dtype dtype, dn_gate gate,
                               void* workspace, size_t workspace_bytes, void* cuda_stream);

/* Bytes of workspace dn_chunk_fwd_varlen needs for N sequences of T tokens in all
 * (it depends on N and T only, not on the lengths). */
DN_API int dn_chunk_fwd_varlen_workspace_size(int N, int T, int H, int d_k, int d_v, dn_dtype dtype,
                                              dn_gate gate, size_t* bytes);

/*
 * dn_decode_step_gva -- dn_decode_step with grouped value heads (ch. 28,
 * "The full layer", step 3).  q, k [B,H_k,d_k]; v, o [B,H,d_v]; beta [B,H];
 * g NULL | [B,H] | [B,H,d_k]; S [B,H,d_k,d_v] in place.  Value head h reads
 * q and k of key head h / (H / H_k).  Every gate, dtype and d of
 * dn_decode_step.  H % H_k != 0 returns DN_ERR_INVALID.
 */
DN_API int dn_decode_step_gva(const void* q, const void* k, const void* v, const float* beta, const float* g,
                              float* S, void* o, int B, int H_k, int H, int d_k, int d_v, float scale,
                              dn_dtype dtype, dn_gate gate, void* cuda_stream);

/*
 * dn_chunk_fwd_general -- the generalised delta rule of RWKV-7 ("DeltaNet:
 * Memory That Edits", D2L 12.5, "The generalized delta rule"), chunked:
 *
 *     S_t = (diag(w_t) - (a_t * kappa_t) kappa_t^T) S_{t-1} + k_t v_t^T
 *     o_t = S_t^T (scale q_t)        (read after the write, as for dn_chunk_fwd)
 *
 * with w_t = exp(w_log_t) a per-key-channel decay, kappa_t the removal key, a_t
 * a per-channel removal rate and k_t the write key (k_t need not equal
 * kappa_t; w = 1, kappa = k', a = beta, k = beta k' is DeltaNet).
 *
 *   q, kappa, k  [B,H,T,d_k] dtype;  v [B,H,T,d_v] dtype
 *   w_log, a     [B,H,T,d_k] fp32 (w_log <= 0 expected, not enforced; kappa is
 *                used as given, not normalised)
 *   S0, S_T      NULL | [B,H,d_k,d_v] fp32, as for dn_chunk_fwd
 *   o            [B,H,T,d_v] dtype
 *   d_k, d_v in {64, 128}; chunk 1..32 (the result does not depend on it
 *   beyond rounding)
 *
 * fp32 arithmetic on the CUDA cores (fp32 or bf16 storage): the page gives the
 * recurrence only, and its chunkwise form (pairwise per-channel decays inside
 * the sums) runs here as derived from it.  Same aliasing and error rules as
 * dn_chunk_fwd.
 */
DN_API int dn_chunk_fwd_general(const void* q, const float* w_log, const void* kappa, const float* a,
                                const void* k, const void* v, const float* S0, void* o, float* S_T,
                                int B, int T, int H, int d_k, int d_v, int chunk, float scale, dn_dtype dtype,
                                void* cuda_stream);

/*
 * dn_decode_step -- one recurrent step ("The recurrent form", ch. 28; KDA's
 * recurrence in "A walk through of the DeltaNet family").
 *
 *   q, k  [B,H,d_k] dtype;  v [B,H,d_v] dtype;  beta [B,H] fp32
 *   g     NULL | [B,H] | [B,H,d_k] fp32 per `gate`
 *   S     [B,H,d_k,d_v] fp32, updated in place
 *   o     [B,H,d_v] dtype, must not overlap any other argument
 *   d_k, d_v in {64, 128}; B, H >= 0.
 */
DN_API int dn_decode_step(const void* q, const void* k, const void* v,
                   const float* beta, const float* g, float* S, void* o,
                   int B, int H, int d_k, int d_v, float scale,
                   dn_dtype dtype, dn_gate gate, void* cuda_stream);

/*
 * dn_decode_step_gdn -- dn_decode_step with the Gated DeltaNet layer's
 * prologue ("Linear attention and Gated DeltaNet", ch. 28, "The full layer",
 * steps 4 and 5) fused into the kernel: the step runs on
 *   q / max(||q||, 1e-12), k / max(||k||, 1e-12),
 *   beta = sigmoid(b), g = -exp(A_log[h]) * softplus(a + dt_bias[h])
 * as dn_decode_step with the scalar gate on these.
 *   q, k [B,H,d_k] raw; v [B,H,d_v]; b, a [B,H] fp32 raw; A_log, dt_bias [H]
 *   fp32 (required, 4-byte aligned); S, o, d_k, d_v, scale, dtype as dn_decode_step.
 */
DN_API int dn_decode_step_gdn(const void* q, const void* k, const void* v, const float* b, const float* a,
                              const float* A_log, const float* dt_bias, float* S, void* o,
                              int B, int H, int d_k, int d_v, float scale, dn_dtype dtype, void* cuda_stream);

/*
 * dn_decode_step_gdn_ex -- dn_decode_step_gdn with flags and, optionally, the
 * layer's gated RMSNorm fused into the step ("Linear attention and Gated
 * DeltaNet", ch. 28, "The full layer", step 7, RMSNormGated):
 *   flags        DN_GDN_BETA_2SIGMOID: beta = 2 sigmoid(b);
 *                DN_GDN_NORM_SIGMOID: the norm's gate is sigmoid(z), else SiLU(z);
 *                other bits return DN_ERR_INVALID
 *   z            NULL (o is the rule's read-out) | [B,H,d_v] dtype: then
 *                o = norm_weight * o / sqrt(mean(o^2) + eps) * act(z), the mean
 *                over the d_v channels of each head's row
 *   norm_weight  [d_v] fp32, shared by every head (required with z)
 *   eps          in (0, 1] (required with z; the page uses 1e-6)
 * z and norm_weight must be 16-byte aligned and must not overlap o or S.
 */
DN_API int dn_decode_step_gdn_ex(const void* q, const void* k, const void* v, const float* b, const float* a,
                                 const float* A_log, const float* dt_bias, float* S, void* o,
                                 int B, int H, int d_k, int d_v, float scale, dn_dtype dtype, int flags,
                                 const void* z, const float* norm_weight, float eps, void* cuda_stream);

/*
 * dn_causal_conv1d -- step 2 of the Gated DeltaNet layer ("Linear attention
 * and Gated DeltaNet", ch. 28, "The full layer", causal_conv1d): a depthwise
 * causal convolution over time, one length-K filter per channel, then SiLU,
 * carrying the previous K-1 inputs as its state.  With joined = the K-1 state
 * rows followed by the T rows of x,
 *   y[t][c] = act( sum_{j<K} weight[c][j] * joined[t + j][c] ),
 * so weight[c][K-1] multiplies the current input; the new state is the last
 * K-1 rows of joined.  fp32 arithmetic, one rounding at each store.
 *
 *   x          [B, T, ld_x] dtype, token-major; channels 0..C-1 of each row
 *              are used (ld_x >= C: x may be a column slice of a wider
 *              projection output, e.g. the q, k or v part)
 *   weight     [C, K] fp32
 *   state_in   [B, K-1, C] dtype, oldest row first, or NULL (zeros)
 *   y          [B, C / head_dim, T, head_dim] dtype: head-major, the layout
 *              dn_chunk_fwd and dn_decode_step read (head_dim = C gives
 *              [B, T, C])
 *   state_out  [B, K-1, C] dtype, or NULL.  It may be state_in itself when
 *              T <= 16 (a decode step); otherwise it must not overlap it.
 *   1 <= K <= 4; head_dim divides C; activation 1 = SiLU, 0 = none.  With
 *   T = 0 only the state moves (x and y may be NULL).
 *   Returns DN_ERR_INVALID on bad sizes, overlaps (y with any input, state_out
 *   with x, weight or y) or misalignment (x, y and the states 2-byte (bf16) or
 *   4-byte (f32) aligned, weight 4-byte); the kernel uses 8-byte accesses
 *   when every pointer, ld_x, C and head_dim allow them.
 */
DN_API int dn_causal_conv1d(const void* x, int ld_x, const float* weight, const void* state_in,
                            void* y, void* state_out, int B, int T, int C, int K, int head_dim,
                            int activation, dn_dtype dtype, void* cuda_stream);

/*
 * dn_rms_norm_gated -- step 7 of the Gated DeltaNet layer ("Linear attention
 * and Gated DeltaNet", ch. 28, RMSNormGated): each head's output row divided
 * by its root mean square, times a per-channel weight and a gate of z,
 *   y = weight * x / sqrt(mean(x^2) + eps) * act(z),  act = SiLU or sigmoid,
 * in fp32 with one rounding at the store.
 *
 *   x       [B, H, T, D] dtype if x_head_major (the layout dn_chunk_fwd writes
 *           o in; a decode step's o [B, H, D] is either layout with T = 1),
 *           else [B, T, H, D]
 *   z       [B, T, H, D] dtype;  y [B, T, H, D] dtype (token-major, the
 *           output projection's layout), must not overlap x, z or weight
 *   weight  [D] fp32, shared by every head
 *   D in {64, 128, 256}; eps >= 0 and finite; activation 1 = SiLU, 0 = sigmoid.
 *   x, z, y 16-byte aligned, weight 4-byte.
 */
DN_API int dn_rms_norm_gated(const void* x, const void* z, const float* weight, void* y,
                             int B, int T, int H, int D, float eps, int x_head_major,
                             int activation, dn_dtype dtype, void* cuda_stream);

/*
 * dn_device_status -- synchronise `cuda_stream`, then read and clear the
 * status word of the current device.  Returns DN_ERR_TIMEOUT if a kernel of
 * this library launched since the previous call gave up on a bounded wait
 * (its outputs are then unspecified), DN_ERR_CUDA if the synchronisation
 * failed, else DN_OK.
 */
DN_API int dn_device_status(void* cuda_stream);

/* Static description of a status code. */
DN_API const char* dn_status_str(int status);

/* Reason for the last non-DN_OK return on the calling thread ("" if none). */
DN_API const char* dn_last_error(void);

/* ABI version, (major << 16) | minor.  2.2: the per-key gate on the tensor-core path;
 * 2.3: dn_chunk_fwd_snapshots; 2.4: dn_chunk_fwd_gdn; 2.5: dn_decode_step_gdn;
 * 2.6: dn_causal_conv1d, dn_rms_norm_gated; 2.7: dn_chunk_fwd_gva, dn_decode_step_gva,
 * dn_chunk_fwd_gdn_ex, dn_decode_step_gdn_ex (the CUDA-core prologue and the 2 sigmoid gate),
 * dn_chunk_fwd_varlen, dn_chunk_fwd_varlen_workspace_size, dn_chunk_fwd_general; 2.8: 256 more
 * workspace bytes per tensor-core chunk (1 / ||q|| of its positions, for the layer prologue). */
DN_API int dn_version(void);

/*
 * dn_kernel_launches -- number of CUDA kernels this library has launched in
 * this process, over all threads and devices (monotonic; counted when the
 * launch call succeeds, not when the kernel ends).  Memsets and copies on the
 * caller's stream are not kernels of this library and are not counted.  The
 * difference of two reads brackets the kernels a region of calls issued.
 */
DN_API unsigned long long dn_kernel_launches(void);

#ifdef __cplusplus
}
#endif

#endif /* DN_H */
