/*
 * sage.h -- C ABI of the B200 (sm_100a) SageAttention-style quantized
 * attention library (libsage_b200.so).
 *
 * What it computes.  Attention O = softmax(Q K^T / sqrt(D) + mask) V for bf16
 * Q, K, V, approximated the SageAttention way: Q and K quantized to INT8 per
 * block of 64 tokens (K after subtracting its per-channel mean over tokens),
 * V cast to FP8 e4m3 with a per-channel scale, Q K^T on INT8 tensor cores,
 * softmax taken online in fp32, P quantized to FP8 e4m3 and P V on FP8 tensor
 * cores with fp32 accumulation.
 *   - "SageAttention: low-bit quantized attention, plug-and-play in place of
 *     FlashAttention" -- Crossing podcast show notes (wav.pub), section
 *     "硬件上明明有更快的计算单元"; English notes (elsewhere.news), same section.
 *   - Per-block 8-bit quantization because per-tensor and per-channel scales
 *     are stretched by outliers -- "Vidu S1" technical digest
 *     (zhao9797.github.io), section "Infra", linear-layer quantization bullet.
 *   - 8-bit block-wise quantization on INT8 tensor cores -- reportify.cn
 *     TurboDiffusion notes, "W8A8线性层量化" bullet.
 *   - Streaming generation attends over a KV cache of earlier frames, which is
 *     what the block-causal mask expresses -- "Vidu S1" digest, section
 *     "Infra", sliding-window decoding paragraph.
 * The pages print neither the block sizes nor the rounding rules; the values
 * used here (64-token INT8 blocks, absmax/127 with round-half-to-even, K mean
 * over all tokens, e4m3 V with absmax/448 per channel, P scale 2^8, KV tiles of
 * 128) are this library's readings and are documented with each call.
 *
 * Conventions shared by every call.
 *   - Memory: the library never allocates device memory.  The caller owns
 *     every buffer (inputs, outputs, workspace).  All pointers named "device"
 *     must be device-accessible addresses on the current CUDA device and
 *     16-byte aligned.
 *   - Streams: `stream` is a cudaStream_t passed as void* (NULL = legacy
 *     default stream).  All device work is enqueued asynchronously on it; no
 *     call synchronizes except sage_sync_status.
 *   - Errors: argument errors are detected on the host before anything is
 *     enqueued and return SAGE_ERR_INVALID_ARG or SAGE_ERR_UNSUPPORTED.
 *     A failed launch returns SAGE_ERR_CUDA.  Every wait inside a kernel is
 *     bounded; a wait that runs out records SAGE_ERR_TIMEOUT in a device-side
 *     status word and the kernel returns early with its outputs undefined;
 *     sage_sync_status reports and clears it.  No call throws or aborts.
 *   - Layouts are row-major.  Padded token counts: N_pad = ceil(N/64)*64.
 */
#ifndef SAGE_B200_H
#define SAGE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define SAGE_ABI_VERSION 1

typedef enum {
    SAGE_OK = 0,
    SAGE_ERR_INVALID_ARG = 1, /* null/misaligned pointer, bad size or mask   */
    SAGE_ERR_UNSUPPORTED = 2, /* valid request the library does not support */
    SAGE_ERR_CUDA = 3,        /* a CUDA launch or runtime call failed         */
    SAGE_ERR_TIMEOUT = 4      /* a bounded device-side wait ran out           */
} sage_status;

typedef enum {
    SAGE_MASK_NONE = 0,
    /* key j visible to query i iff j <= i + (Nkv - Nq): queries are the
     * newest Nq tokens of the Nkv-token cache (bottom-right alignment). */
    SAGE_MASK_CAUSAL = 1,
    /* block-causal over blocks of mask_block tokens (one latent frame in a
     * streaming video step): key j visible to query i iff
     * floor(j / mask_block) <= floor((i + Nkv - Nq) / mask_block). */
    SAGE_MASK_BLOCK_CAUSAL = 2
    /* The sliding window with a persistent reference context has its own
     * call, sage_attn_fwd_window, because it takes three parameters; it is
     * not a sage_mask value, and the mask-taking calls reject any other. */
} sage_mask;

/* Problem shape.  Inputs are [B, H, Nq, D] (Q) and [B, H, Nkv, D] (K, V).
 * Supported: B, H, Nq, Nkv >= 1; D in {64, 128}; B*H <= 65535. */
typedef struct {
    int B, H, Nq, Nkv, D;
} sage_shape;

/* The quantized operands produced by sage_quant_qk and read by
 * sage_attn_fwd.  All device pointers, caller-allocated, 16-byte aligned:
 *   q_i8    int8  [B, H, Nq_pad,  D]  Q codes; rows >= Nq are 0
 *   q_scale f32   [B, H, Nq_pad/64]   per-block Q scale (absmax/127)
 *   k_i8    int8  [B, H, Nkv_pad, D]  codes of K - k_mean; rows >= Nkv are 0
 *   k_scale f32   [B, H, Nkv_pad/64]  per-block K scale
 *   k_mean  f32   [B, H, D]           per-channel mean of K over all Nkv tokens
 *   v_f8    e4m3  [B, H, Nkv_pad, D]  V codes, token-major like k_i8:
 *                                     byte ((b*H+h)*Nkv_pad + n)*D + d;
 *                                     tokens n >= Nkv are 0
 *   v_scale f32   [B, H, D]           per-channel V scale (absmax/448)
 * Dequantization: q = q_i8 * q_scale[n/64]; k = k_i8 * k_scale[n/64] + k_mean;
 * v = e4m3_value(v_f8) * v_scale[d]. */
typedef struct {
    int8_t *q_i8;
    float *q_scale;
    int8_t *k_i8;
    float *k_scale;
    float *k_mean;
    uint8_t *v_f8;
    float *v_scale;
} sage_qkv_quant;

/* Byte sizes of the seven sage_qkv_quant buffers, in struct order
 * (q_i8, q_scale, k_i8, k_scale, k_mean, v_f8, v_scale).
 * Returns SAGE_ERR_INVALID_ARG for a null pointer or an invalid shape. */
sage_status sage_quant_buffer_bytes(const sage_shape *shape, size_t sizes[7]);

/* Device workspace sage_quant_qk needs for `shape` (bytes; 0 on an invalid
 * shape).  It holds per-64-token-block fp64 K channel sums and V channel
 * maxima, and the V inverse scales: B*H*ceil(Nkv/64)*D*12 + B*H*D*4 bytes.
 * Its contents never need initialising. */
size_t sage_quant_workspace_bytes(const sage_shape *shape);

/* Quantize Q, K and V (all device, bf16, contiguous [B,H,N,D]).
 *
 * This is the quantization half of low-bit quantized attention: Q and K to
 * 8-bit codes with per-block scales, so that Q K^T runs on INT8 tensor cores
 * (reportify.cn TurboDiffusion notes, "混合注意力加速" and "W8A8线性层量化"
 * bullets: SageAttention is 8-bit block-wise quantized attention on INT8
 * tensor cores; "Vidu S1" digest, section "Infra": per-block scales because
 * per-tensor and per-channel scales are stretched by outliers).  The block
 * size, rounding, K smoothing and the e4m3 V are this library's readings.
 *
 *   Q: per (b, h, 64-token block): a = max|Q| over the block, q_scale = a/127,
 *      q_i8 = clamp(round_half_even(Q * fp32(127/a)), -127, 127); a = 0 gives
 *      scale 0 and codes 0.
 *   K: k_mean[d] = fp32(S/Nkv) with S the fp64 sum of K[:, d] taken as
 *      ascending 64-token block sums (each summed in ascending token order)
 *      added in ascending block order; then the block quantization above on
 *      fp32(K - k_mean).
 *   V: per channel, a = max|V[:, d]| over all tokens, v_scale = a/448,
 *      v_f8 = e4m3_rne_satfinite(V * fp32(448/a)).
 * All fp32 operations are single IEEE operations rounded to nearest-even, so
 * the outputs are reproducible bit for bit.
 *
 * `out` points to caller-allocated buffers sized by sage_quant_buffer_bytes;
 * `workspace` to at least sage_quant_workspace_bytes(shape) device bytes
 * (contents need not be initialised; they are overwritten).
 * Enqueues three kernels on `stream`: the statistics of every 64-token
 * block (and the Q codes), the per-head K mean and V scales, then the K and
 * V codes.  Returns SAGE_OK or an error (above). */
sage_status sage_quant_qk(const void *q_bf16, const void *k_bf16, const void *v_bf16,
                          const sage_shape *shape, const sage_qkv_quant *out,
                          void *workspace, size_t workspace_bytes, void *stream);

/* sage_quant_qk with rotary position embedding applied to Q and K first.
 *
 * The pages cache features before RoPE and apply RoPE at their current,
 * re-based positions whenever the streaming window slides ("Vidu S1" digest,
 * Infra, RoPE Repositioning).  This call fuses that rotation into the
 * quantizer, so the cache can stay un-rotated in bf16.
 *
 *   Rotation: for every (b, h), token n and channel pair (2p, 2p+1), p < D/2,
 *     with c = cos[n][p], s = sin[n][p] from the tables below:
 *       x'[2p]   = fma(x[2p], c, -fp32(x[2p+1] * s))
 *       x'[2p+1] = fma(x[2p], s,  fp32(x[2p+1] * c))
 *     (each product and fma rounded once to fp32; the result is not rounded
 *     to bf16).  Per-pair angles cover 1D and multi-axis (frame / height /
 *     width) RoPE alike.
 *   Then exactly the steps of sage_quant_qk on Q' and K' (the K mean is that
 *   of the rotated keys); V is not rotated.
 *
 *   q_cos, q_sin: device f32 [Nq, D/2]; k_cos, k_sin: device f32 [Nkv, D/2];
 *     row n holds token n's values; shared by every batch entry and head;
 *     read only; 16-byte aligned.
 *   Other arguments and outputs: as for sage_quant_qk.
 *
 * Errors: SAGE_ERR_INVALID_ARG for a null or misaligned table and for every
 * case sage_quant_qk rejects; SAGE_ERR_UNSUPPORTED for Nq or Nkv above
 * 65535 * 64 = 4194240 tokens; SAGE_ERR_CUDA if a launch fails. */
sage_status sage_quant_qk_rope(const void *q_bf16, const void *k_bf16, const void *v_bf16,
                               const sage_shape *shape, const float *q_cos,
                               const float *q_sin, const float *k_cos, const float *k_sin,
                               const sage_qkv_quant *out, void *workspace,
                               size_t workspace_bytes, void *stream);

/* Device workspace sage_quant_qk_equalized needs for `shape` (bytes; 0 on an
 * invalid shape): sage_quant_workspace_bytes(shape) + B*H*D*4*(ceil(Nq/64) +
 * 2*ceil(Nkv/64) + 2).  Its contents never need initialising. */
size_t sage_quant_equalized_workspace_bytes(const sage_shape *shape);

/* Channel-equalised quantization: a labelled accuracy variant of
 * sage_quant_qk, outside the pages' recipe (which sage_quant_qk computes).
 *
 * The pages present 8-bit attention as nearly lossless for video models
 * (reportify.cn TurboDiffusion notes, "几乎无损"); with per-block INT8 codes a
 * K channel that carries outliers sets the scale of every K block it lives in,
 * and the INT8 error of Q K^T then dominates.  This variant, before the
 * per-block INT8 codes, multiplies channel d of Q by 2^e[d] and divides
 * channel d of the smoothed key fp32(K - mu) by 2^e[d] (each one fp32
 * multiplication), which leaves every score unchanged in exact arithmetic:
 *   aq = max_n |Q[n,d]|, ak = max_n |fp32(K[n,d] - mu[d])| (per b, h, d),
 *   e = floor((floor(log2 ak) - floor(log2 aq)) / 2) clamped to [-32, 32],
 *   e = 0 when aq or ak is 0.
 * The K mean, the V codes and scales, and the layout of every output are
 * those of sage_quant_qk; sage_attn_fwd and the other attention calls take
 * the result unchanged.  Q is read twice (its channel maxima, then its codes).
 *
 *   q_bf16 ... out, stream  as for sage_quant_qk (no rotation)
 *   eq_exp                  NULL, or device int8 [B, H, D]: receives e
 *   workspace               at least sage_quant_equalized_workspace_bytes
 * Enqueues three kernels.  Errors as sage_quant_qk. */
sage_status sage_quant_qk_equalized(const void *q_bf16, const void *k_bf16, const void *v_bf16,
                                    const sage_shape *shape, const sage_qkv_quant *out,
                                    int8_t *eq_exp, void *workspace, size_t workspace_bytes,
                                    void *stream);

/* The keys a sliding-window step attends to (the union over its query rows
 * of the keys sage_attn_fwd_window lets them see): the reference context
 * [0, *n_sink) and the window [*lo, *hi) of the cache of `shape` (queries are
 * its newest Nq tokens).  *lo - *n_sink is a whole number of frames.
 * Errors: SAGE_ERR_INVALID_ARG for a bad shape, a null output, frame or win
 * below 1, sink below 0, or Nkv < Nq. */
sage_status sage_window_keys(const sage_shape *shape, int frame, int win, int sink, int *n_sink,
                             int *lo, int *hi);

/* Windowed quantization of the streaming cache: sage_quant_qk (or, with the
 * four angle tables, sage_quant_qk_rope) over only the keys a sliding-window
 * step attends to.
 *
 * The pages' streaming decoder attends, at every step, to the persistent
 * reference context and a fixed-length window of the cache ("Vidu S1"
 * digest, section "Infra", sliding-window decoding paragraph), and keeps the
 * cache before RoPE, re-applying RoPE at the current positions (RoPE
 * Repositioning bullet).  Reading: the step's K mean and V channel scales are
 * those of the keys it attends to, and only those keys are quantized.
 *
 *   q_bf16                 device bf16 [B, H, Nq, D]: the step's queries
 *   k_cache, v_cache       device bf16 [B, H, Nkv, D]: the whole cache
 *   cache_shape            B, H, Nq, Nkv (the cache's length), D
 *   frame, win, sink       the window of sage_attn_fwd_window
 *   q_cos ... k_sin        NULL (no rotation) or all four tables of
 *                          sage_quant_qk_rope: q_* [Nq, D/2], k_* [Nkv', D/2]
 *                          for the gathered keys' current positions
 *   out, workspace         sized for the gathered shape (B, H, Nq, Nkv', D),
 *                          Nkv' = n_sink + hi - lo of sage_window_keys
 * Key r of the result is cache key r for r < n_sink and cache key
 * r + (lo - n_sink) after, i.e. the reference context then the window, in
 * cache order.  sage_attn_fwd_window with the same (frame, win, sink) on the
 * result gives every query row the same keys as on the whole cache.
 * Errors: as sage_quant_qk / sage_quant_qk_rope on the gathered shape, plus
 * SAGE_ERR_INVALID_ARG for bad window parameters or only some angle tables. */
sage_status sage_quant_qk_window(const void *q_bf16, const void *k_cache, const void *v_cache,
                                 const sage_shape *cache_shape, int frame, int win, int sink,
                                 const float *q_cos, const float *q_sin, const float *k_cos,
                                 const float *k_sin, const sage_qkv_quant *out, void *workspace,
                                 size_t workspace_bytes, void *stream);

/* Size of the fixed device scratch array sage_quant_qk_noalloc uses: 16 MiB
 * on every GPU that loads the library, held until the process exits. */
#define SAGE_NOALLOC_SCRATCH_BYTES ((size_t)16 << 20)

/* sage_quant_qk for callers that cannot allocate device memory.
 *
 * The pages describe no such call; it exists for callers that are handed only
 * their input and output buffers and are not allowed to allocate -- for
 * example code running inside a memory pool that has been sized and locked in
 * advance, a real-time loop that must not enter the allocator, or a plugin of
 * a host framework that owns all device memory.  Such callers cannot supply
 * the workspace sage_quant_qk needs, so this variant keeps it in one fixed,
 * library-owned device array of SAGE_NOALLOC_SCRATCH_BYTES.  It computes
 * exactly what sage_quant_qk computes (same kernels, same results) and calls
 * no allocation routine.
 *
 *   q_bf16, k_bf16, v_bf16, shape, out, stream: as for sage_quant_qk.
 *
 * Errors: SAGE_ERR_INVALID_ARG for a bad shape or pointer;
 * SAGE_ERR_UNSUPPORTED if sage_quant_workspace_bytes(shape) exceeds
 * SAGE_NOALLOC_SCRATCH_BYTES (e.g. B1 H24 Nkv26520 D128 fits, B1 H40 Nkv75600
 * D128 does not) -- nothing is enqueued then; SAGE_ERR_CUDA if a launch
 * fails.
 *
 * Sharing: all calls on a device use the same array, which keeps whatever
 * the last call left in it.  Nothing in it needs to start at zero (each call
 * writes every cell it later reads), but two calls whose work can overlap on
 * the GPU (e.g. on two streams with no ordering between them) race on it and
 * give undefined results; order such calls on one stream.
 * Set-up: the first call on a device looks up the array's device address
 * (cudaGetSymbolAddress, with that device current).  Make that first call
 * before any stream capture.  It sets up only this array: the attention and
 * GEMM calls do their own one-time set-up on their first call, so a program
 * that captures those calls needs one eager call of each before capturing. */
sage_status sage_quant_qk_noalloc(const void *q_bf16, const void *k_bf16, const void *v_bf16,
                                  const sage_shape *shape, const sage_qkv_quant *out,
                                  void *stream);

/* Fused quantized attention over the output of sage_quant_qk.
 *
 * SageAttention-style low-bit attention, the plug-and-play replacement of
 * FlashAttention that moves both matmuls onto 8-bit tensor cores (Crossing
 * podcast show notes, section "硬件上明明有更快的计算单元"; reportify.cn
 * TurboDiffusion notes, "混合注意力加速" bullet).  The arithmetic below is
 * this library's reading of it; every step is one IEEE fp32 operation
 * rounded to nearest-even unless stated.
 *
 * Per query row i (row limit lim_i from `mask`, see sage_mask), over KV tiles
 * of 128 keys in ascending order (only tiles holding a visible key):
 *   S    = q_i8 . k_i8 (exact int32 on the INT8 tensor cores)
 *   c    = fp32(fp32(q_scale * C0) * k_scale[j/64]), C0 = fp32(log2(e)/sqrt(D))
 *   m    = max(m, max_j fp32(S*c))   (running max in the log2 domain)
 *   y    = exp2(fma(S, c, fp32(8 - m)))  (= 2^8 p: the fixed P scale 2^8 is
 *          folded into the exponent argument; exp2 is the hardware
 *          approximation, relative error below 2^-21)
 *   l    = l*alpha + sum_j y   (fp32, from y before quantization)
 *   P    = e4m3(y) (round to nearest even; y <= 2^8 (1 + 2^-21) never
 *          saturates); O_acc = O_acc*alpha + P . v_f8 (FP8 tensor cores,
 *          fp32 accumulation), alpha = exp2(m_old - m_new) (exactly 1 when
 *          the maximum did not move, 0 before the first tile)
 *   O    = O_acc * (v_scale[d] * (1 / l)), rounded to bf16 (l is in units of
 *          2^8 p, so the 2^8 cancels).
 *   lse  = (m + log2(l) - 8) * ln 2.
 * Softmax invariance makes the K-mean subtraction exact in real arithmetic.
 *
 *   mask        a sage_mask value; CAUSAL and BLOCK_CAUSAL need Nkv >= Nq
 *   mask_block  block length for SAGE_MASK_BLOCK_CAUSAL (>= 1), else ignored
 *   o_bf16      device bf16 [B, H, Nq, D] output (required)
 *   o_f32       device f32  [B, H, Nq, D] output before bf16 rounding, or NULL
 *   lse         device f32  [B, H, Nq] natural-log log-sum-exp of the
 *               dequantized scaled scores, or NULL
 * One kernel launch on `stream`. */
sage_status sage_attn_fwd(const sage_qkv_quant *qkv, const sage_shape *shape, int mask,
                          int mask_block, void *o_bf16, float *o_f32, float *lse, void *stream);

/* sage_attn_fwd with block-sparse skipping: tiles of 128 query rows x 128
 * keys that `block_mask` switches off are not computed (neither Q K^T nor
 * P V nor the softmax visits them).  This is the skipping that the sparse
 * layers stacked on quantized attention rely on (TurboDiffusion notes,
 * hybrid-attention bullet: SageAttention combined with sparse-linear
 * attention); how the mask is predicted is not given by the pages and is
 * the caller's business.
 *   block_mask  device uint8 [B, H, ceil(Nq/128), ceil(Nkv/128)], row-major;
 *               key j is visible to query i iff `mask` allows it AND
 *               block_mask[b][h][i/128][j/128] != 0.  Read only.
 * The tile order of the online softmax is unchanged (ascending over the
 * visited tiles), so an all-ones mask gives exactly sage_attn_fwd's result.
 * A query row that sees no key at all gets O = 0 (bf16 and f32) and
 * lse = -inf.
 * Errors: as sage_attn_fwd, plus SAGE_ERR_INVALID_ARG for a NULL block_mask
 * and SAGE_ERR_UNSUPPORTED for more than 6144 KV tiles (786432 keys). */
sage_status sage_attn_fwd_block_sparse(const sage_qkv_quant *qkv, const sage_shape *shape,
                                       int mask, int mask_block, const uint8_t *block_mask,
                                       void *o_bf16, float *o_f32, float *lse, void *stream);

/* Device workspace sage_attn_fwd_split needs (bytes): kv_splits * B * H *
 * ceil(Nq/128)*128 * (D + 2) * 4; 0 for kv_splits = 1 or an invalid
 * argument (kv_splits outside 1..16, bad shape). */
size_t sage_attn_split_workspace_bytes(const sage_shape *shape, int kv_splits);

/* sage_attn_fwd in split-KV form, for shapes with few query tiles (e.g. one
 * streaming frame against a long cache), where one CTA per 128-query tile
 * leaves most of the GPU idle.
 *
 * The KV tiles that a query tile visits under `mask` ([0, nk), nk from its
 * last row) are cut into kv_splits contiguous ranges [floor(s nk / S),
 * floor((s+1) nk / S)).  Each range runs the online softmax of sage_attn_fwd
 * on its own CTA, giving an unnormalized O_s with running max m_s and sum l_s;
 * a second kernel merges them in ascending s:
 *   m = max_s m_s,  a_s = exp2(m_s - m) (0 for a range that saw no key),
 *   O = sum_s a_s O_s,  l = sum_s a_s l_s,  o = O * v_scale / l,
 * lse as for sage_attn_fwd.  P is quantized relative to each range's own
 * running max, so results differ from sage_attn_fwd by rounding only.
 * kv_splits = 1 is sage_attn_fwd itself (no workspace needed).
 *
 *   kv_splits: 1..16.  workspace: device, 16-byte aligned, at least
 *   sage_attn_split_workspace_bytes(shape, kv_splits) bytes (contents need
 *   not be initialised).  Other arguments: as for sage_attn_fwd.
 * Enqueues two kernels on `stream`.
 * Errors: as sage_attn_fwd, plus SAGE_ERR_INVALID_ARG for kv_splits outside
 * 1..16 or a missing, misaligned or too small workspace. */
sage_status sage_attn_fwd_split(const sage_qkv_quant *qkv, const sage_shape *shape, int mask,
                                int mask_block, int kv_splits, void *workspace,
                                size_t workspace_bytes, void *o_bf16, float *o_f32, float *lse,
                                void *stream);

/* sage_attn_fwd under a sliding window with a persistent reference context:
 * the attention of streaming generation, where every step attends to a
 * fixed-length window made of the reference context (tokens taken once
 * from the first frame and the first generated state, kept for the whole
 * stream, in the role of a sink token), the cached history frames inside
 * the window and the frame being denoised (Vidu S1 digest, section "Infra",
 * sliding-window decoding paragraph).
 *
 * Key layout read: the reference context at positions [0, sink_tokens),
 * then frames of frame_len tokens.  Queries are the newest Nq of the Nkv
 * positions (query i sits at g = i + Nkv - Nq).  A query with g >= sink_tokens
 * in frame f = (g - sink_tokens) / frame_len sees the whole reference
 * context and frames f - window_frames + 1 .. f (its own frame in full);
 * a query inside the reference context sees the reference context only.
 * With sink_tokens = 0 and a window of at least Nkv / frame_len + 1 frames
 * this is SAGE_MASK_BLOCK_CAUSAL with mask_block = frame_len, bit for bit.
 *
 * Only tiles holding a visible key are computed: a query tile visits the
 * reference context's tiles and then, past a gap it never touches, the
 * window's; the online softmax runs over that sequence in ascending order.
 * kv_splits > 1 cuts the sequence into ranges and merges them as
 * sage_attn_fwd_split does (workspace: sage_attn_split_workspace_bytes);
 * kv_splits = 1 needs no workspace (pass NULL, 0).
 *
 *   frame_len >= 1, window_frames >= 1, sink_tokens >= 0 (values above Nkv
 *   act as Nkv).  Other arguments: as for sage_attn_fwd_split.
 * Enqueues one kernel (kv_splits = 1) or two on `stream`.
 * Errors: SAGE_ERR_INVALID_ARG for Nkv < Nq, a parameter out of range, or a
 * missing, misaligned or too small workspace when kv_splits > 1; otherwise
 * as sage_attn_fwd. */
sage_status sage_attn_fwd_window(const sage_qkv_quant *qkv, const sage_shape *shape,
                                 int frame_len, int window_frames, int sink_tokens,
                                 int kv_splits, void *workspace, size_t workspace_bytes,
                                 void *o_bf16, float *o_f32, float *lse, void *stream);

/* Debug: run the attention kernel's load + INT8 MMA path on selected tiles
 * and copy the int32 score tile it leaves in tensor memory to `out`.
 *   tiles  host int array of n_tiles triples (bh, qt, kt): head index b*H+h,
 *          query tile (rows qt*128 .. qt*128+127), KV tile (keys kt*128 ..)
 *   out    device int32 [n_tiles, 128, 128]: out[t][r][c] = S of query row
 *          qt*128+r and key kt*128+c (rows/keys past the padded ends read
 *          as zero codes).
 * Tiles outside the shape give SAGE_ERR_INVALID_ARG.  n_tiles <= 65535. */
sage_status sage_debug_qk_int32(const sage_qkv_quant *qkv, const sage_shape *shape,
                                const int *tiles, int n_tiles, int32_t *out, void *stream);

/* Debug: launch one CTA that waits on a shared-memory barrier nothing ever
 * arrives at, with a budget of `budget_cycles` SM clock cycles (1 .. 2^40).
 * The wait gives up, records SAGE_ERR_TIMEOUT in the status word and the
 * kernel returns.  Exercises the bounded-wait path every kernel uses. */
sage_status sage_debug_timeout_probe(long long budget_cycles, void *stream);

/* Debug: y[i] = e4m3 code of x[i] (round to nearest even, saturating to
 * +-448, NaN to NaN), computed with the conversion instruction the kernels
 * use for V and P.  x: device f32 [n], y: device uint8 [n]. */
sage_status sage_debug_e4m3(const float *x, uint8_t *y, size_t n, void *stream);

/* Debug: y[i] = 2^x[i] as the attention kernel's softmax computes it (the
 * hardware approximate base-2 exponential, subnormal results flushed to
 * zero).  x, y: device f32 [n]. */
sage_status sage_debug_exp2(const float *x, float *y, size_t n, void *stream);

/* Synchronize `stream`, then return and clear the device-side status word:
 * SAGE_ERR_TIMEOUT if any kernel's bounded wait ran out since the last call,
 * SAGE_ERR_CUDA if the synchronization failed, else SAGE_OK. */
sage_status sage_sync_status(void *stream);

/* ------------------------------------------------------------------------
 * Per-block W8A8 linear layer: Y = X W^T with INT8 activations and weights
 * (Vidu S1 digest, section "Infra": per-block W8A8 for the linear layers,
 * because per-tensor and per-channel scales are stretched by outliers;
 * TurboDiffusion notes, W8A8 bullet: 8-bit block-wise quantization on INT8
 * tensor cores).  Blocks are 128 channels wide along the reduction dim K:
 * one activation scale per token and 128-channel group, one weight scale per
 * 128 x 128 block; symmetric absmax/127, codes round-half-to-even, an
 * all-zero block gets scale 0.  Requirements: K and N multiples of 128,
 * 1 <= M <= 65535 * 128; all pointers device pointers, caller-allocated,
 * 16-byte aligned (scale arrays 4-byte aligned).  Asynchronous on `stream`;
 * errors as for the attention calls.
 * ---------------------------------------------------------------------- */

/* X bf16 [M, K] -> xq int8 [M, K], sx f32 [M, K/128]:
 *   a = max |x| over (m, channels 128g .. 128g+127), sx = a/127,
 *   xq = clamp(rne(x * fp32(127/a)), -127, 127). */
sage_status sage_w8a8_quant_act(const void *x_bf16, long long M, long long K, int8_t *xq,
                                float *sx, void *stream);

/* W bf16 [N, K] -> wq int8 [N, K], sw f32 [N/128, K/128], one scale per
 * 128 x 128 block, same rule as above. */
sage_status sage_w8a8_quant_weight(const void *w_bf16, long long N, long long K, int8_t *wq,
                                   float *sw, void *stream);

/* Y = dequant(X) dequant(W)^T on the INT8 tensor cores: for each output
 * element, each 128-channel group's integer product P_g = sum xq*wq is exact
 * (int32) and is promoted into an fp32 running sum in ascending group order,
 *   y = fmaf((float)P_g, fp32(sx[m][g] * sw[n/128][g]), y),
 * and Y = bf16(y) (round-half-to-even).
 *   y_bf16  device bf16 [M, N] (required)
 *   y_f32   device f32 [M, N] (y before rounding) or NULL
 * One kernel launch (persistent: one CTA per SM loops over the 128 x 128
 * output tiles, column tiles fastest). */
sage_status sage_w8a8_gemm(const int8_t *xq, const float *sx, const int8_t *wq, const float *sw,
                           long long M, long long N, long long K, void *y_bf16, float *y_f32,
                           void *stream);

/* sage_w8a8_gemm for the projection that produces attention's Q, with Q's
 * quantization fused into the GEMM epilogue (the fusion "into the producing
 * GEMM's epilogue" of the pages' kernel-fusion bullet, for the one operand
 * whose quantization needs no statistic over all tokens).
 *
 * Y [M, N] = X W^T as sage_w8a8_gemm computes it, read as Q of one batch
 * entry: M tokens, N/128 heads of D = 128 (column c of head h is column
 * 128 h + c of Y).  The epilogue rounds Y to bf16 and quantizes it exactly as
 * sage_quant_qk quantizes Q: per head and 64-token block, a = max|Q| over the
 * block, q_scale = a/127, q_i8 = clamp(round_half_even(Q * fp32(127/a)),
 * -127, 127); a = 0 gives scale 0 and codes 0; tokens M..M_pad-1 get code 0.
 * So q_i8 and q_scale equal sage_quant_qk's Q output for that bf16 Q, bit for
 * bit, without the bf16 round trip of Q through memory.
 *
 *   q_i8: device int8 [N/128][M_pad][128], M_pad = M rounded up to 64 (the
 *     layout of one batch entry of sage_qkv_quant.q_i8), 16-byte aligned.
 *   q_scale: device f32 [N/128][M_pad/64], 4-byte aligned.
 *   y_bf16: the bf16 Y as well, or NULL.
 *   Other arguments: as for sage_w8a8_gemm (N a multiple of 128).
 * Errors: as sage_w8a8_gemm, plus SAGE_ERR_INVALID_ARG for a null or
 * misaligned q_i8 or q_scale. */
sage_status sage_w8a8_gemm_q(const int8_t *xq, const float *sx, const int8_t *wq,
                             const float *sw, long long M, long long N, long long K,
                             void *y_bf16, int8_t *q_i8, float *q_scale, void *stream);

/* Static description of a status code (never NULL). */
const char *sage_status_string(sage_status status);

/* Hardware ceilings: microbenchmarks of the rates the kernels' rooflines rest
 * on.  One kernel launch on `stream`, whose blocks are all resident at once
 * (one wave); block i writes the SM clock cycles of its timed loop to
 * cycles[i].  On return (before the kernel has run) *blocks, *blocks_per_sm
 * and *ops_per_block describe the launch, so that
 *   rate per SM per clock = ops_per_block * blocks_per_sm / cycles[i]
 *   whole-GPU rate        = ops_per_block * blocks / (the launch's duration).
 *   kind 0  exp2 unit (ex2.approx.f32): iters rounds of 8 dependent chains
 *           per thread; an operation is one exp2 result.
 *   kind 1  packed fp32x2 fma: an operation is one fma lane.
 *   kind 2  fp32 pair -> e4m3x2 conversion (satfinite): an operation is one
 *           conversion instruction (two values).
 *   kind 3  device memory copy of scratch's first half into its second half
 *           (16-byte vectors); an operation is one byte read or written.
 *           scratch: device, 16-byte aligned, at least 1 MiB; iters unused.
 *   kind 4  tcgen05 kind::i8 MMA (M 128, N n, K 32, int32 accumulator in
 *           tensor memory), one CTA per SM, one issuing thread, iters groups
 *           of 4 MMAs; an operation is one multiply or add (2 M N K per MMA).
 *   kind 5  the same with kind::f8f6f4, e4m3 operands, fp32 accumulator.
 *   iters: 1 .. 2^24 (kinds 0-2, 4, 5); n: 64, 128 or 256 (kinds 4, 5).
 *   cycles: device int64, 8-byte aligned, at least 8 x (number of SMs)
 *   entries.  The MMA kinds' completion wait is bounded: a timeout is
 *   reported by sage_sync_status.
 * Errors: SAGE_ERR_INVALID_ARG for an unknown kind or an argument out of
 * range, SAGE_ERR_CUDA if the launch fails. */
sage_status sage_ceiling(int kind, int iters, int n, void *scratch, size_t scratch_bytes,
                         long long *cycles, int *blocks, int *blocks_per_sm,
                         double *ops_per_block, void *stream);

/* SAGE_ABI_VERSION of the loaded library. */
int sage_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SAGE_B200_H */
