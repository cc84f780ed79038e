/*
 * flint_attn.h - C ABI of the B200 (sm_100a) sink-aware GQA attention of the
 * Flint hybrid-attention MoE decoder: forward, its gradient, and a decode step.
 *
 * The operation is the core of FlintAttention.forward (NeMo AutoModel API
 * page "nemo_automodel.components.models.flint.layers", FlintAttention.forward:
 * "full-sequence causal attention with a zero-value sink category"), from the
 * projected Q/K/V up to the input of o_proj:
 *
 *   1. per-head RMSNorm on Q and K in weight form, x / sqrt(mean(x^2) + eps) * w
 *      (HF discussion #26 on RecursiveSI/flint: plain RMSNorm, not 1+w;
 *      FlintConfig.rms_norm_eps = 1e-6; model page, "Model Architecture":
 *      query/key normalisation precedes RoPE);
 *   2. on sliding layers only, NeoX RoPE over all 128 channels, channel i
 *      rotated against channel i+64 at the token's document-local position
 *      (FlintAttention._apply_rope; FlintConfig: sliding layers rotate all
 *      head channels);
 *   3. causal attention of 32 query heads over 4 key/value heads (query head h
 *      reads KV head h/8), logits scaled by 1/sqrt(128), full or restricted to
 *      a window that counts the current token (513 = current + 512 preceding;
 *      model page "Model Architecture", FlintConfig.sliding_window);
 *   4. one learned FP32 sink per query head acting as an extra softmax column
 *      with zero value, in natural-logit units and not scaled by 1/sqrt(d)
 *      (HF discussion #26, learned-sink semantics and item 5;
 *      _FlintSinkParameters.forward returns unscaled sink logits);
 *   5. padded queries and keys are excluded, the sink stays valid, so a padded
 *      query's output is zero and its LSE equals the sink
 *      (FlintAttention.forward, attention_mask).
 *
 * Memory: every pointer argument except the host-side `stream` handle is a
 * DEVICE pointer owned by the caller.  The library never allocates; the call
 * is asynchronous on `stream` (a cudaStream_t; NULL = legacy default stream).
 * Argument errors are detected on the host before any launch and return a
 * status without touching the GPU.  Errors that can only be seen on the
 * device (an ill-formed cu_seqlens or padding mask, a timed-out wait inside a
 * kernel) are recorded in the workspace and read back with
 * flint_attn_device_status().
 */
#ifndef FLINT_ATTN_H_
#define FLINT_ATTN_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define FLINT_API __attribute__((visibility("default")))
#else
#define FLINT_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    FLINT_OK = 0,
    FLINT_ERR_INVALID_ARG = 1,  /* bad pointer, size, alignment or flag */
    FLINT_ERR_UNSUPPORTED = 2,  /* well-formed but outside what the kernels do
                                   (non-trailing padding mask, no sm_100 GPU) */
    FLINT_ERR_CUDA = 3,         /* a CUDA runtime/driver call failed */
    FLINT_ERR_TIMEOUT = 4,      /* a bounded wait inside a kernel ran out */
    FLINT_ERR_WORKSPACE = 5     /* workspace missing, misaligned or too small */
} flint_status_t;

#define FLINT_HQ 32      /* query heads            */
#define FLINT_HKV 4      /* key/value heads        */
#define FLINT_HEAD_DIM 128
#define FLINT_MAX_TOKENS (1 << 24)

/* ABI revision of this header (bumped on any signature change). */
FLINT_API int32_t flint_attn_abi_version(void);

/*
 * Bytes of device workspace flint_attn_fwd needs for T tokens split into
 * `num_segments` documents or batch rows (1 for a single sequence).  The
 * workspace holds the normalised/rotated keys (FP16, 1 KiB per token), the
 * work plan and a status word.  Returns 0 for invalid sizes.
 */
FLINT_API size_t flint_attn_workspace_bytes(int32_t T, int32_t num_segments);

/*
 * Sink-aware GQA attention forward.
 *
 *  q          bf16 [T,32,128] contiguous: projected queries, before q_norm.
 *  k, v       bf16 [T,4,128] contiguous: projected keys (before k_norm), values.
 *             q, k, v and out must be 16-byte aligned.  K and V must be finite
 *             at every token, padded ones included.
 *  q_norm_w   fp32 [128] q_norm weight, shared by all query heads.
 *  k_norm_w   fp32 [128] k_norm weight, shared by all key heads.
 *  sinks      fp32 [32] sink logits in natural-log units (may be +-inf).
 *  pos_ids    int32 [T] document-local positions used by RoPE; NULL means the
 *             index of the token within its document / batch row.  Ignored
 *             when use_rope == 0.
 *  cu_seqlens int32 [num_docs+1] packed-THD document boundaries: cu[0] = 0,
 *             non-decreasing, cu[num_docs] <= T; tokens >= cu[num_docs] are
 *             padding.  NULL when not packed.
 *  pad_mask   uint8 [batch, seqlen], 1 = valid token, 0 = padding; every row
 *             must be ones followed by zeros (trailing padding), otherwise the
 *             device status becomes FLINT_ERR_UNSUPPORTED and no output is
 *             produced.  NULL when unpadded.  At most one of cu_seqlens and
 *             pad_mask may be non-NULL; with neither, q is one sequence.
 *  batch, seqlen  shape of pad_mask (batch * seqlen == T); ignored otherwise.
 *  T          total tokens, 0 <= T <= FLINT_MAX_TOKENS (T == 0: no-op).
 *  window     0 for full causal attention; W > 0 keeps keys j with
 *             i - W < j <= i (W = 513 on Flint's sliding layers).
 *  use_rope   1 on sliding layers, 0 on full layers.
 *  rope_theta RoPE base (> 1), e.g. 10000.
 *  eps        RMSNorm epsilon (> 0), 1e-6 for Flint.
 *  out        bf16 [T,4096]: out[t, h*128 + c], the o_proj input.  Rows of
 *             padded tokens are written as +0.0.  On sliding layers
 *             (window > 0) the call also uses out as scratch: the preparation
 *             kernel leaves each valid token's normalised FP16 queries in its
 *             rows and the attention kernel overwrites them with the result;
 *             on full layers the attention kernel prepares the queries on
 *             tile load.  Either way out may be q itself (each query row is
 *             read before anything is written over it); it must not overlap
 *             k, v, lse or the workspace.
 *  lse        fp32 [32,T] natural-log sum of exponentials including the sink
 *             (lse[h*T + t]); padded tokens get sinks[h].  May be NULL.
 *  workspace  device buffer of at least flint_attn_workspace_bytes(T, n)
 *             bytes, 256-byte aligned, where n = num_docs, batch or 1.
 *             Must not be shared by calls that may overlap on the GPU.
 *  stream     cudaStream_t as void*.
 *
 * Returns FLINT_OK once the kernels are enqueued.
 */
FLINT_API flint_status_t flint_attn_fwd(const void* q, const void* k, const void* v,
                              const float* q_norm_w, const float* k_norm_w,
                              const float* sinks, const int32_t* pos_ids,
                              const int32_t* cu_seqlens, int32_t num_docs,
                              const uint8_t* pad_mask, int32_t batch, int32_t seqlen,
                              int32_t T, int32_t window, int32_t use_rope,
                              float rope_theta, float eps,
                              void* out, float* lse,
                              void* workspace, size_t workspace_bytes,
                              void* stream);

/*
 * The two stages flint_attn_fwd enqueues, exposed so a caller (or a profiler)
 * can time them apart.  flint_attn_prepare runs the preparation kernel: the
 * work plan, the normalised/rotated FP16 keys in the workspace, the outputs
 * of padded query tokens and, on sliding layers, the normalised/rotated FP16
 * queries in the rows of out (intermediate values, not a result).
 * flint_attn_attend runs the attention kernel on a workspace and an out that
 * flint_attn_prepare filled with the same arguments; calling it with other
 * arguments, or after out was modified in between, is undefined.  Both take
 * the arguments of flint_attn_fwd and validate them the same way.
 */
FLINT_API flint_status_t flint_attn_prepare(const void* q, const void* k, const void* v,
                              const float* q_norm_w, const float* k_norm_w,
                              const float* sinks, const int32_t* pos_ids,
                              const int32_t* cu_seqlens, int32_t num_docs,
                              const uint8_t* pad_mask, int32_t batch, int32_t seqlen,
                              int32_t T, int32_t window, int32_t use_rope,
                              float rope_theta, float eps,
                              void* out, float* lse,
                              void* workspace, size_t workspace_bytes,
                              void* stream);
FLINT_API flint_status_t flint_attn_attend(const void* q, const void* k, const void* v,
                              const float* q_norm_w, const float* k_norm_w,
                              const float* sinks, const int32_t* pos_ids,
                              const int32_t* cu_seqlens, int32_t num_docs,
                              const uint8_t* pad_mask, int32_t batch, int32_t seqlen,
                              int32_t T, int32_t window, int32_t use_rope,
                              float rope_theta, float eps,
                              void* out, float* lse,
                              void* workspace, size_t workspace_bytes,
                              void* stream);

/*
 * The forward on a slice of the KV heads: the unit of work of head-split
 * context parallelism ("flint" model page, "Parallelism and backends": TE
 * context parallelism splits the attention heads over the CP group, which
 * both head counts must divide, so the 4 KV heads permit CP2 or CP4).  Each
 * rank holds the whole sequence for kv_heads KV heads and their 8 * kv_heads
 * query heads (after an all-to-all from sequence shards) and runs this call.
 *
 *  kv_heads   1, 2 or 4 (4: the same as flint_attn_fwd).
 *  q          bf16 [T, 8 kv_heads, 128];  k, v  bf16 [T, kv_heads, 128].
 *  sinks      fp32 [8 kv_heads]: the slice's sinks.
 *  out        bf16 [T, 8 kv_heads x 128];  lse  fp32 [8 kv_heads, T] or NULL.
 *  workspace  flint_attn_workspace_bytes(T, n) bytes, as for flint_attn_fwd.
 *  Every other argument, and the error behaviour, as for flint_attn_fwd.
 */
FLINT_API flint_status_t flint_attn_fwd_heads(const void* q, const void* k, const void* v,
                              const float* q_norm_w, const float* k_norm_w,
                              const float* sinks, const int32_t* pos_ids,
                              const int32_t* cu_seqlens, int32_t num_docs,
                              const uint8_t* pad_mask, int32_t batch, int32_t seqlen,
                              int32_t T, int32_t kv_heads, int32_t window, int32_t use_rope,
                              float rope_theta, float eps,
                              void* out, float* lse,
                              void* workspace, size_t workspace_bytes,
                              void* stream);

/*
 * The FP16 attention-compute policy ("flint" model page, "Numerical
 * comparison": attention_compute_dtype fp16 casts the normalised, rotated
 * Q/K/V to FP16 at the attention boundary of an FP32 model and restores FP32
 * before the output projection; the pages measure it closest to the FP32
 * reference).  The same operation as flint_attn_fwd on FP32 projections:
 * q~, k~ are normalised and rotated in FP32 and cast to FP16, v is cast to
 * FP16, the probabilities multiply v in FP16 with FP32 accumulation, and the
 * result is written in FP16 (exact in FP32, restoring it is a widening).
 *
 *  q          fp32 [T,32,128]; k, v fp32 [T,4,128] (16-byte aligned).
 *  out        fp16 [T,4096].
 *  workspace  at least flint_attn_fp16_workspace_bytes(T, n) bytes: the
 *             forward's workspace plus the FP16 queries (8 KiB per token)
 *             and values (1 KiB per token).
 *  Every other argument, and the error behaviour, as for flint_attn_fwd.
 */
FLINT_API size_t flint_attn_fp16_workspace_bytes(int32_t T, int32_t num_segments);
FLINT_API flint_status_t flint_attn_fwd_fp16(const float* q, const float* k, const float* v,
                              const float* q_norm_w, const float* k_norm_w,
                              const float* sinks, const int32_t* pos_ids,
                              const int32_t* cu_seqlens, int32_t num_docs,
                              const uint8_t* pad_mask, int32_t batch, int32_t seqlen,
                              int32_t T, int32_t window, int32_t use_rope,
                              float rope_theta, float eps,
                              void* out, float* lse,
                              void* workspace, size_t workspace_bytes,
                              void* stream);

/*
 * Synchronises `stream`, then returns the status the kernels of the last
 * flint_attn_fwd or flint_attn_decode on `workspace` recorded (FLINT_OK,
 * FLINT_ERR_INVALID_ARG for an ill-formed cu_seqlens or a decode window that
 * does not fit its cache, FLINT_ERR_UNSUPPORTED for a non-trailing mask,
 * FLINT_ERR_TIMEOUT), or FLINT_ERR_CUDA if synchronising failed.
 */
FLINT_API flint_status_t flint_attn_device_status(const void* workspace, void* stream);

/*
 * Size in bytes of the scratch array behind flint_attn_fwd_static: 16 MiB,
 * enough for about 16,000 tokens (1 KiB of normalised keys per token plus the
 * work plan).
 */
#define FLINT_STATIC_SCRATCH_BYTES (16u << 20)

/*
 * flint_attn_fwd_static - the same forward as flint_attn_fwd, for callers
 * that cannot allocate device memory when they run the layer (an allocator
 * that must not be re-entered from a callback, a memory budget fixed up front,
 * a host that only hands out its own buffers).  The pages have no counterpart
 * of this entry point; it exists for those callers.
 *
 * Arguments are those of flint_attn_fwd without workspace and
 * workspace_bytes; the caller still provides inputs and outputs.  The
 * kernels' scratch (work plan, normalised keys) lives in a file-scope device
 * array of FLINT_STATIC_SCRATCH_BYTES that every GPU loading the library
 * keeps until the process exits.  No cudaMalloc, cudaFree or allocating
 * library call is made.
 *  - A problem whose scratch would exceed FLINT_STATIC_SCRATCH_BYTES
 *    (flint_attn_workspace_bytes(T, n) larger than it) is rejected with
 *    FLINT_ERR_WORKSPACE before any launch.
 *  - Every call looks up the array's device address (cudaGetSymbolAddress)
 *    with the calling thread's current device, so the address always belongs
 *    to the current context, also after a device reset.  The first call on a
 *    device may load the library's device code there; make that first call
 *    before any stream capture.
 *  - Every call shares the one array and it keeps the last call's contents
 *    (the kernels initialise what they read); calls that may overlap on the
 *    GPU race on it, so serialise them (one stream, or events).
 *  - Errors only the device can see (ill-formed cu_seqlens, non-trailing
 *    mask, a timed-out wait) are recorded in the array's status word; read
 *    it with flint_attn_fwd_static_status.
 */
FLINT_API flint_status_t flint_attn_fwd_static(const void* q, const void* k, const void* v,
                              const float* q_norm_w, const float* k_norm_w,
                              const float* sinks, const int32_t* pos_ids,
                              const int32_t* cu_seqlens, int32_t num_docs,
                              const uint8_t* pad_mask, int32_t batch, int32_t seqlen,
                              int32_t T, int32_t window, int32_t use_rope,
                              float rope_theta, float eps,
                              void* out, float* lse,
                              void* stream);

/*
 * Synchronises `stream`, then returns the status recorded by the kernels of
 * the last flint_attn_fwd_static call that launched any (FLINT_OK,
 * FLINT_ERR_INVALID_ARG for an ill-formed cu_seqlens, FLINT_ERR_UNSUPPORTED
 * for a non-trailing mask, FLINT_ERR_TIMEOUT), or FLINT_ERR_CUDA if
 * synchronising or reading failed.  Calls rejected on the host and T == 0
 * launch nothing and leave the word as it was.  Copies one word from the
 * device to the host; allocates nothing.  Like the array itself, it is
 * shared: read it before the next flint_attn_fwd_static call is enqueued.
 */
FLINT_API flint_status_t flint_attn_fwd_static_status(void* stream);

/* Largest batch of one decode step (sequences per call). */
#define FLINT_MAX_DECODE_BATCH 65535

/*
 * One decode step: a new token per sequence attends to the keys and values
 * cached for its earlier positions (FlintAttention.forward on the NeMo
 * AutoModel "flint.layers" API page, applied to the last position only; the
 * "flint" model page notes that the KV cache must honour the per-layer
 * window sizes).  Sequence b's new token sits at position p = cache_len[b]:
 * its queries and key get the prologue (per-head RMSNorm in weight form,
 * then NeoX RoPE at p when use_rope), it attends to positions
 * max(0, p - window + 1) .. p (window > 0, the window counting the token
 * itself) or 0 .. p (window == 0) plus the learned sink, and the step
 * appends it to the cache.
 *
 *  q          bf16 [B,32,128]: the new tokens' projected queries, before q_norm.
 *  k, v       bf16 [B,4,128]: their projected keys (before k_norm) and values.
 *  q_norm_w, k_norm_w, sinks   as for flint_attn_fwd.
 *  k_cache    bf16 [B,4,cap,128], head-major: normalised, rotated keys of
 *             earlier positions; position j of sequence b, KV head g lives in
 *             k_cache[b][g][j mod cap], so a cache of capacity >= window is a
 *             ring on sliding layers, and each head's slots are consecutive
 *             256-byte rows.  The keys are assumed normalised with k_norm_w
 *             (|k~|_2 <= sqrt(128) max|k_norm_w|, as the step itself writes
 *             them): the tensor-core path starts its softmax from the bound
 *             this gives on every logit.
 *  v_cache    bf16 [B,4,cap,128]: values, same slots.
 *             The step writes the new token's key (normalised, rotated,
 *             rounded to BF16) and value into slot p mod cap.  The window
 *             must fit the cache (p - lo + 1 <= cap); otherwise the device
 *             status becomes FLINT_ERR_INVALID_ARG and that sequence's output
 *             is undefined.
 *  cache_len  int32 [B]: positions already cached = position of the new token,
 *             0 <= cache_len[b] < FLINT_MAX_TOKENS (else the device status
 *             becomes FLINT_ERR_INVALID_ARG).
 *  B          sequences, 0 <= B <= FLINT_MAX_DECODE_BATCH (0: no-op).
 *  cap        cache capacity in positions, >= 1.
 *  window     0 for a full layer, W > 0 for a sliding layer.
 *  use_rope, rope_theta, eps   as for flint_attn_fwd.
 *  out        bf16 [B,4096]: out[b, h*128 + c].
 *  lse        fp32 [32,B] natural-log sum of exponentials including the sink;
 *             may be NULL.
 *  workspace  device buffer of at least flint_attn_decode_workspace_bytes(B,
 *             cap, window) bytes, 256-byte aligned; holds the device status
 *             (read with flint_attn_device_status) and the split partials.
 *  stream     cudaStream_t as void*.
 *
 * When the logit bound 16.45 max|q_norm_w| max|k_norm_w| (log2 units) is at
 * most 48, a tensor-core kernel streams the cache in tiles of 128 slots:
 * scores from BF16 keys and queries split into BF16 high and low parts
 * (FP32 accumulation), probabilities 2^(s - bound) in BF16 for the value
 * product; splits of up to 8 tiles per (sequence, KV head), the last split
 * to finish folding them with the sink.  Otherwise queries, keys and scores
 * are computed in FP32 on CUDA cores over splits of 256 positions, folded
 * the same way.  One call launches a small kernel that resets the status
 * and counters in the workspace, then both kernels (each a programmatic
 * dependent of the launch before it); the one not taken returns at once.
 */
FLINT_API size_t flint_attn_decode_workspace_bytes(int32_t B, int32_t cap, int32_t window);
FLINT_API flint_status_t flint_attn_decode(const void* q, const void* k, const void* v,
                              const float* q_norm_w, const float* k_norm_w,
                              const float* sinks, void* k_cache, void* v_cache,
                              const int32_t* cache_len, int32_t B, int32_t cap,
                              int32_t window, int32_t use_rope, float rope_theta,
                              float eps, void* out, float* lse,
                              void* workspace, size_t workspace_bytes, void* stream);

/*
 * Gradient of flint_attn_fwd.  The "flint" model page (NeMo AutoModel,
 * "Parallelism and backends") makes every head's sink a trainable FP32
 * parameter whose adjoint needs care; the call computes the exact derivative
 * of the forward defined above for a loss that depends on `out` (lse receives
 * no gradient):
 *
 *   D_i = dO_i . out_i,  P_ij = exp(s_ij - lse_i),  dS_ij = P_ij (dO_i . v_j - D_i)
 *   dv_j = sum P_ij dO_i,  dq~_i = sum_j dS_ij k~_j / sqrt(128),
 *   dk~_j = sum dS_ij q~_i / sqrt(128),  dsink_h = -sum_i exp(sink_h - lse_i) D_i
 *
 * (sums over the query heads of a KV head where the operand is shared), then
 * back through RoPE (rotation by -p) and the RMSNorm in weight form, which
 * also gives the norm weights' gradients.
 *
 *  q, k, v, q_norm_w, k_norm_w, sinks, pos_ids, cu_seqlens, num_docs,
 *  pad_mask, batch, seqlen, T, window, use_rope, rope_theta, eps
 *             the forward's arguments, unchanged (same rules).
 *  out        bf16 [T,4096]: the forward's result for these arguments.
 *  lse        fp32 [32,T]: the forward's log-sum-exp (required here).
 *  dout       bf16 [T,4096]: gradient of the loss with respect to out.
 *  dq         fp32 [T,32,128]: gradient with respect to q (pre-norm).
 *  dk, dv     fp32 [T,4,128]: gradients with respect to k (pre-norm) and v.
 *  dq_norm_w, dk_norm_w   fp32 [128];  dsinks  fp32 [32].
 *             Every gradient is overwritten, not accumulated; padded tokens
 *             get zero rows.  q, k, v, out and dout must be 16-byte aligned,
 *             dq, dk and dv too; no output may overlap an input, another
 *             output or the workspace.
 *  workspace  device buffer of at least flint_attn_bwd_workspace_bytes(T)
 *             bytes (about 9.3 KiB per token), 256-byte aligned; holds the
 *             device status (flint_attn_device_status: FLINT_ERR_INVALID_ARG
 *             for an ill-formed cu_seqlens, FLINT_ERR_UNSUPPORTED for a
 *             non-trailing mask, FLINT_ERR_TIMEOUT), per-token document
 *             bounds, D, the FP16 operands q~ and k~ and per-CTA partial sums.
 *  stream     cudaStream_t as void*.
 *
 * T == 0 sets dq_norm_w, dk_norm_w and dsinks to zero and does nothing else.
 * The products run on the tensor cores (tcgen05; q~, k~ and dS in FP16, v,
 * dout and P in BF16, FP32 accumulation), the RoPE and RMSNorm adjoints on
 * CUDA cores in FP32; every sum has a fixed order, so repeated calls give
 * identical bits.
 */
FLINT_API size_t flint_attn_bwd_workspace_bytes(int32_t T);
FLINT_API flint_status_t flint_attn_bwd(const void* q, const void* k, const void* v,
                           const float* q_norm_w, const float* k_norm_w,
                           const float* sinks, const int32_t* pos_ids,
                           const int32_t* cu_seqlens, int32_t num_docs,
                           const uint8_t* pad_mask, int32_t batch, int32_t seqlen,
                           int32_t T, int32_t window, int32_t use_rope,
                           float rope_theta, float eps, const void* out,
                           const float* lse, const void* dout, float* dq, float* dk,
                           float* dv, float* dq_norm_w, float* dk_norm_w,
                           float* dsinks, void* workspace, size_t workspace_bytes,
                           void* stream);

/* Largest hidden size of the projection entry points. */
#define FLINT_MAX_HIDDEN 65536

/*
 * The projections around the attention core: FlintAttention.forward (NeMo
 * AutoModel "flint.layers" API page) maps hidden states x [T, hidden] to
 * q = x W_q^T, k = x W_k^T, v = x W_v^T (bias-free: FlintConfig
 * attention_bias = False), runs the attention above on them and returns
 * y = a W_o^T.  Weights use the PyTorch Linear layout [out, in], BF16; q, k
 * and v are head-major (column h*128 + c).  Products accumulate in FP32 on
 * the tensor cores (tcgen05) and are rounded to BF16 once.
 *
 * flint_qkv_proj: the fused projection.
 *  x          bf16 [T, hidden], hidden a multiple of 64 in [64, FLINT_MAX_HIDDEN].
 *  w_qkv      bf16 [5120, hidden]: W_q (rows 0..4095), W_k (4096..4607) and
 *             W_v (4608..5119) stacked.
 *  q          bf16 [T, 32, 128]; k, v bf16 [T, 4, 128]: the projections,
 *             as flint_attn_fwd takes them.
 *  All pointers are device pointers, 16-byte aligned; no output may overlap
 *  an input.  T == 0 is a no-op.  Asynchronous on `stream`.
 *
 * flint_o_proj: y = attn_out W_o^T.
 *  attn_out   bf16 [T, 4096] (flint_attn_fwd's out);  w_o bf16 [hidden, 4096];
 *  y          bf16 [T, hidden].
 *
 * Bounded waits inside these two kernels cannot report a timeout (there is
 * no workspace); flint_attn_layer_fwd records one in its workspace status.
 */
FLINT_API flint_status_t flint_qkv_proj(const void* x, const void* w_qkv, int32_t T, int32_t hidden,
                              void* q, void* k, void* v, void* stream);
FLINT_API flint_status_t flint_o_proj(const void* attn_out, const void* w_o, int32_t T,
                              int32_t hidden, void* y, void* stream);

/*
 * The whole attention layer: flint_qkv_proj, the attention forward, then
 * flint_o_proj, with the key prologue fused into the projection: its
 * epilogue writes the normalised, rotated FP16 keys the attention kernel
 * reads straight into the workspace (FlintAttention.forward; model page
 * "Model Architecture": query/key normalisation precedes RoPE), so the
 * preparation kernel only plans the work and writes padded rows, and the
 * attention kernel normalises and rotates the queries on tile load.
 *
 *  x, w_qkv, w_o, hidden      as for flint_qkv_proj / flint_o_proj.
 *  q_norm_w ... eps           as for flint_attn_fwd.
 *  q, k, v    bf16 outputs: the raw projections (kept for the backward).
 *  attn_out   bf16 [T, 4096]: the attention output (o_proj's input).
 *  y          bf16 [T, hidden]: the layer's output.
 *  lse        fp32 [32, T] or NULL.
 *  workspace  at least flint_attn_workspace_bytes(T, n) bytes, as for
 *             flint_attn_fwd; read its status with flint_attn_device_status.
 */
FLINT_API flint_status_t flint_attn_layer_fwd(const void* x, const void* w_qkv, const void* w_o,
                              const float* q_norm_w, const float* k_norm_w,
                              const float* sinks, const int32_t* pos_ids,
                              const int32_t* cu_seqlens, int32_t num_docs,
                              const uint8_t* pad_mask, int32_t batch, int32_t seqlen,
                              int32_t T, int32_t hidden, int32_t window, int32_t use_rope,
                              float rope_theta, float eps, void* q, void* k, void* v,
                              void* attn_out, void* y, float* lse,
                              void* workspace, size_t workspace_bytes, void* stream);

/* Text of the last error raised on the calling host thread ("" if none). */
FLINT_API const char* flint_attn_last_error(void);

/* Fixed name of a status code. */
FLINT_API const char* flint_attn_status_string(flint_status_t status);

#ifdef __cplusplus
}
#endif
#endif /* FLINT_ATTN_H_ */
