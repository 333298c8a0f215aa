/*
 * sage_oracle.c -- plain, slow CPU reference for SageAttention-style
 * quantized attention (INT8 per-block Q/K with K mean-smoothing, FP8 e4m3
 * per-channel V, FP8 P, fp32 online softmax).
 *
 * TEST INFRASTRUCTURE.  Only the test-suite, the smoke check and the
 * benchmark's CPU-baseline / reference arm may load this library.  The GPU
 * product path never calls it and shares no code, header or table with it.
 *
 * Sources of the method:
 *   - "Vidu S1: A Real-Time Interactive Video Generation Model" digest
 *     (zhao9797.github.io), section "Infra": SageAttention is the attention
 *     accelerator; per-block 8-bit quantization is chosen because per-tensor
 *     and per-channel scales are stretched by outliers.
 *   - reportify.cn TurboDiffusion notes: SageAttention is low-bit quantized
 *     attention; 8-bit block-wise quantization runs on INT8 tensor cores.
 *   - The finer recipe (64-token INT8 blocks with absmax/127 and
 *     round-half-to-even, K mean-smoothing over tokens, e4m3 V with a
 *     per-channel absmax/448 scale, FP8 P, fp32 online softmax with exp2) is
 *     not printed on the pages; the readings taken here are listed in the
 *     design notes and restated next to each function below.
 *
 * Build: plain C11, no FMA contraction (-ffp-contract=off), no fast-math, so
 * that every float expression below is one IEEE binary32 operation rounded
 * to nearest-even (x86-64 SSE: FLT_EVAL_METHOD == 0).
 *
 * Parity status of each exported function (what pins it in the tests):
 *   orc_e4m3_encode / decode : OCP OFP8 E4M3 special points + brute-force
 *                              nearest-even search + torch float8 cast.
 *   orc_quant_head           : quantizer invariants, numpy mean for mu.
 *   orc_quant_head_eq        : the exponent rule restated with numpy frexp;
 *                              dequantized scores within the INT8 bound of
 *                              Q (K - mu)^T; balanced channels reproduce
 *                              orc_quant_head bit for bit; accuracy against
 *                              fp64 attention on outlier channels.
 *   orc_qk_int32             : numpy int64 brute force.
 *   orc_attn_rows (identity) : textbook softmax attention to 1e-12.
 *   orc_attn_rows (quant)    : closed forms (Q = 0, single visible key);
 *                              plain fp64 attention over the dequantized
 *                              operands within the rigorous bound of P's
 *                              e4m3 rounding, lse to 1e-5; the error bound
 *                              against fp64 attention.
 *   rounding slack           : exp2 results moved to the edges of their
 *                              uncertainty interval (orc_attn_rows_pert)
 *                              stay within it and, pushed per channel to
 *                              the extreme codes, span it exactly.
 *   orc_attn_fp64_rows       : textbook softmax attention (torch) to 1e-12.
 *   orc_attn_rows_bs / _identity_bs (block mask): identity mode against
 *                              textbook softmax attention under the combined
 *                              row and block mask to 1e-12; an all-ones mask
 *                              reproduces the dense result bit for bit; rows
 *                              that see no key give O = 0, lse = -inf.
 *   orc_attn_rows_win / _identity_win / orc_attn_fp64_rows_win (sliding
 *                              window + reference context): identity mode
 *                              against textbook attention over the gathered
 *                              visible keys to 1e-12; sink = 0 with a window
 *                              wider than the cache reproduces the
 *                              block-causal result bit for bit; brute-force
 *                              visibility on small grids.
 *   orc_w8a8_quant_act / _weight : quantizer invariants (max code 127, half-
 *                              step reconstruction, zero groups, RNE ties,
 *                              block shapes).
 *   orc_w8a8_gemm_rows       : exact integer product on unit scales (numpy
 *                              int64), fp64 blockwise definition within the
 *                              fp32 accumulation bound.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_BLK 64 /* Q/K quantization block: 64 tokens */

/* Compile-time switches used only by the test-suite, which builds separate
 * copies of this library with them to show that its pins catch plausible
 * mistakes (the product build defines neither):
 *   ORC_PLANT = 1  the K scale of key j taken from block j / 128, not j / 64
 *             = 2  l summed from the decoded e4m3 codes instead of from y
 *             = 3  the slack not rescaled by alpha when the running max moves
 *             = 4  the slack gap measured in code units instead of values
 *             = 5  the slack not divided by l
 *             = 6  equalisation: the smoothed K multiplied by 2^e, not divided
 *             = 7  equalisation: e = ilogb(ak) - ilogb(aq), not half of it
 *   ORC_PSCALE_UNFOLDED  the other admissible reading of the 2^8 P scale:
 *             y = 2^8 * fp32(exp2(fmaf(S, c, -m))) instead of
 *             y = fp32(exp2(fmaf(S, c, fp32(8 - m)))) */
#ifndef ORC_PLANT
#define ORC_PLANT 0
#endif

enum {
    ORC_MASK_NONE = 0,
    ORC_MASK_CAUSAL = 1,
    ORC_MASK_BLOCK_CAUSAL = 2,
    ORC_MASK_SLIDING_WINDOW = 3
};

/* ------------------------------------------------------------------ */
/* bf16                                                               */
/* ------------------------------------------------------------------ */

static float bf16_to_f32(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* ------------------------------------------------------------------ */
/* FP8 E4M3 (OCP OFP8): 1 sign bit, 4 exponent bits with bias 7,       */
/* 3 mantissa bits.  Exponent field 0 holds subnormals m/8 * 2^-6.     */
/* No infinities; S.1111.111 is NaN, so the largest finite is          */
/* 1.75 * 2^8 = 448.                                                   */
/* ------------------------------------------------------------------ */

double orc_e4m3_decode(uint8_t c)
{
    int s = c >> 7, e = (c >> 3) & 15, m = c & 7;
    double v;
    if (e == 15 && m == 7)
        return NAN;
    if (e == 0)
        v = ldexp((double)m / 8.0, -6);
    else
        v = ldexp(1.0 + (double)m / 8.0, e - 7);
    return s ? -v : v;
}

/* Round a non-negative finite double to e4m3 with round-to-nearest-even and
 * saturation to the largest finite value (the "satfinite" convention). */
static uint8_t e4m3_encode_abs(double a)
{
    int e2, E;
    double quantum, n, r, v;
    if (a >= 448.0)
        return 0x7E;
    if (a == 0.0)
        return 0x00;
    frexp(a, &e2);      /* a = f * 2^e2, f in [0.5, 1) */
    E = e2 - 1;         /* a in [2^E, 2^(E+1)) */
    if (E < -6)
        E = -6;         /* subnormal range shares the 2^-9 quantum */
    quantum = ldexp(1.0, E - 3);
    n = a / quantum;    /* exact: power-of-two division */
    r = nearbyint(n);   /* ties to even on the integer = on the mantissa */
    v = r * quantum;
    if (v == 0.0)
        return 0x00;
    if (v >= 448.0)
        return 0x7E;
    /* encode the representable value v */
    frexp(v, &e2);
    E = e2 - 1;
    if (E < -6) {       /* subnormal: v = m/8 * 2^-6 */
        int m = (int)(v / ldexp(1.0, -9));
        return (uint8_t)m;
    } else {
        int m = (int)((v / ldexp(1.0, E) - 1.0) * 8.0);
        return (uint8_t)(((E + 7) << 3) | m);
    }
}

static uint8_t e4m3_encode_d(double x)
{
    if (isnan(x))
        return 0x7F;
    if (signbit(x))
        return (uint8_t)(0x80 | e4m3_encode_abs(-x));
    return e4m3_encode_abs(x);
}

uint8_t orc_e4m3_encode(float x) { return e4m3_encode_d((double)x); }

void orc_e4m3_encode_n(const float *x, long n, uint8_t *out)
{
    for (long i = 0; i < n; i++)
        out[i] = orc_e4m3_encode(x[i]);
}

/* ------------------------------------------------------------------ */
/* Quantization                                                        */
/* ------------------------------------------------------------------ */

/* Symmetric per-block INT8 over blocks of 64 rows of an [n, D] matrix:
 * a = max |x| over the block's valid rows, scale = a/127, inv = 127/a,
 * q = clamp(round_half_even(x * inv), -127, 127).  An all-zero block gets
 * scale 0 and q = 0; rows past n (padding up to the next multiple of 64)
 * are 0.  Reading: no zero point, -128 unused, multiply by the rounded
 * inverse rather than divide per element. */
static void quant_blocks_i8(const float *x, long n, int D, int8_t *q, float *scale)
{
    long nblk = (n + ORC_BLK - 1) / ORC_BLK;
    for (long b = 0; b < nblk; b++) {
        long r0 = b * ORC_BLK, r1 = r0 + ORC_BLK;
        long rv = r1 < n ? r1 : n;
        float a = 0.0f;
        for (long r = r0; r < rv; r++)
            for (int d = 0; d < D; d++) {
                float t = fabsf(x[r * D + d]);
                if (t > a)
                    a = t;
            }
        memset(q + r0 * D, 0, (size_t)(ORC_BLK * D));
        if (a == 0.0f) {
            scale[b] = 0.0f;
            continue;
        }
        scale[b] = a / 127.0f;
        float inv = 127.0f / a;
        for (long r = r0; r < rv; r++)
            for (int d = 0; d < D; d++) {
                float y = x[r * D + d] * inv;
                float t = nearbyintf(y);
                if (t > 127.0f)
                    t = 127.0f;
                if (t < -127.0f)
                    t = -127.0f;
                q[r * D + d] = (int8_t)t;
            }
    }
}

/* Rotary position embedding of the rows of an [n, D] fp32 matrix, in place
 * (the pages' RoPE: features are cached before RoPE and rotated at their
 * current positions, "Vidu S1" digest, Infra, RoPE Repositioning).
 * Reading: channel pairs (2p, 2p+1), p < D/2, are rotated as one complex
 * number by the angle whose cosine and sine the caller supplies per row and
 * pair (cs, sn: [n, D/2] fp32), which covers 1D and multi-axis (frame,
 * height, width) RoPE alike:
 *   x'[2p]   = fma(x[2p], c, -fp32(x[2p+1] * s))
 *   x'[2p+1] = fma(x[2p], s,  fp32(x[2p+1] * c))
 * each product and each fma rounded once to fp32; the result is not rounded
 * to bf16 before quantization. */
static void rope_rows(float *x, long n, int D, const float *cs, const float *sn)
{
    const int P = D / 2;
    for (long r = 0; r < n; r++)
        for (int p = 0; p < P; p++) {
            float x0 = x[r * D + 2 * p], x1 = x[r * D + 2 * p + 1];
            float c = cs[r * P + p], s = sn[r * P + p];
            float t = x1 * s;
            float u = x1 * c;
            x[r * D + 2 * p] = fmaf(x0, c, -t);
            x[r * D + 2 * p + 1] = fmaf(x0, s, u);
        }
}

/* Quantize one (batch, head): Q [nq, D], K [nkv, D], V [nkv, D] as bf16 bits.
 *
 * Outputs (caller-allocated):
 *   q8 [ceil(nq/64)*64, D] int8, qs [ceil(nq/64)]
 *   k8 [ceil(nkv/64)*64, D] int8, ks [ceil(nkv/64)], mu [D]
 *   v8 [nkv, D] e4m3 codes (logical token-major order), vs [D]
 *
 * K mean-smoothing: mu[d] = fp32(sum_n K[n,d] / nkv) where the sum is taken
 * in fp64 in a fixed order: each 64-token block summed in ascending token
 * order, then the block sums added in ascending block order.  The smoothed
 * key ks = fp32(K - mu) is what gets block-quantized.  Q is not smoothed.
 *
 * V: per channel d over all nkv tokens, a = max |V[:,d]|, vs = a/448,
 * inv = 448/a, v8 = e4m3_rne_satfinite(V * inv); a == 0 gives vs = 0, v8 = 0.
 *
 * With rotation tables (q_cos, q_sin: [nq, D/2]; k_cos, k_sin: [nkv, D/2];
 * all four or none), Q and K are first rotated by rope_rows and everything
 * above applies to the rotated values (the K mean included); V is not
 * rotated.
 */
/* floor(a / 2) for any int a. */
static int floor_half(int a)
{
    return a >= 0 ? a / 2 : -((1 - a) / 2);
}

/* Channel equalisation of Q [nq, D] and the smoothed K [nkv, D], in place
 * (a labelled accuracy variant, not the pages' recipe; the pages' per-block
 * INT8 recipe is the default).  The scores sum_d Q[i,d] K[j,d] are unchanged
 * in exact arithmetic when channel d of Q is multiplied and channel d of K
 * divided by the same power of two.  With aq = max_n |Q[n,d]| and
 * ak = max_n |K[n,d]|, the exponent is e = floor((ilogb(ak) - ilogb(aq)) / 2),
 * clamped to [-ORC_EQ_MAX, ORC_EQ_MAX] (0 when either maximum is 0); after
 * Q 2^e and K 2^-e the two channel maxima lie within a factor (1/2, 4) of each
 * other, so a K channel with outliers no longer sets the scale of every K
 * block alone.  Each product is one fp32 multiplication (exact unless it
 * leaves the normal range). */
#define ORC_EQ_MAX 32
static void equalise_channels(float *xq, long nq, float *xk, long nkv, int D, int8_t *eq_exp)
{
    for (int d = 0; d < D; d++) {
        float aq = 0.0f, ak = 0.0f;
        for (long n = 0; n < nq; n++)
            if (fabsf(xq[n * D + d]) > aq)
                aq = fabsf(xq[n * D + d]);
        for (long n = 0; n < nkv; n++)
            if (fabsf(xk[n * D + d]) > ak)
                ak = fabsf(xk[n * D + d]);
        int e = 0;
        if (aq > 0.0f && ak > 0.0f) {
#if ORC_PLANT == 7
            e = ilogbf(ak) - ilogbf(aq);
#else
            e = floor_half(ilogbf(ak) - ilogbf(aq));
#endif
            if (e > ORC_EQ_MAX)
                e = ORC_EQ_MAX;
            if (e < -ORC_EQ_MAX)
                e = -ORC_EQ_MAX;
        }
        eq_exp[d] = (int8_t)e;
#if ORC_PLANT == 6
        const float up = ldexpf(1.0f, e), down = ldexpf(1.0f, e);
#else
        const float up = ldexpf(1.0f, e), down = ldexpf(1.0f, -e);
#endif
        for (long n = 0; n < nq; n++)
            xq[n * D + d] = xq[n * D + d] * up;
        for (long n = 0; n < nkv; n++)
            xk[n * D + d] = xk[n * D + d] * down;
    }
}

static int quant_head_impl(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                           long nq, long nkv, int D,
                           const float *q_cos, const float *q_sin,
                           const float *k_cos, const float *k_sin,
                           int8_t *q8, float *qs, int8_t *k8, float *ks, float *mu,
                           uint8_t *v8, float *vs, int8_t *eq_exp)
{
    float *x = (float *)malloc(sizeof(float) * (size_t)((nq > nkv ? nq : nkv) * D));
    float *xq = eq_exp ? (float *)malloc(sizeof(float) * (size_t)(nq * D)) : NULL;
    if (!x || (eq_exp && !xq)) {
        free(x);
        free(xq);
        return 1;
    }
    /* Q (quantized at once, or kept for the equalisation) */
    for (long i = 0; i < nq * D; i++)
        x[i] = bf16_to_f32(q[i]);
    if (q_cos)
        rope_rows(x, nq, D, q_cos, q_sin);
    if (eq_exp)
        memcpy(xq, x, sizeof(float) * (size_t)(nq * D));
    else
        quant_blocks_i8(x, nq, D, q8, qs);
    /* K (rotated), then its channel mean in the canonical fp64 order */
    for (long i = 0; i < nkv * D; i++)
        x[i] = bf16_to_f32(k[i]);
    if (k_cos)
        rope_rows(x, nkv, D, k_cos, k_sin);
    long nblk = (nkv + ORC_BLK - 1) / ORC_BLK;
    for (int d = 0; d < D; d++) {
        double total = 0.0;
        for (long b = 0; b < nblk; b++) {
            double s = 0.0;
            long r1 = (b + 1) * ORC_BLK < nkv ? (b + 1) * ORC_BLK : nkv;
            for (long r = b * ORC_BLK; r < r1; r++)
                s += (double)x[r * D + d];
            total += s;
        }
        mu[d] = (float)(total / (double)nkv);
    }
    /* smoothed K, then block quantization */
    for (long r = 0; r < nkv; r++)
        for (int d = 0; d < D; d++)
            x[r * D + d] = x[r * D + d] - mu[d];
    if (eq_exp) {
        equalise_channels(xq, nq, x, nkv, D, eq_exp);
        quant_blocks_i8(xq, nq, D, q8, qs);
        free(xq);
    }
    quant_blocks_i8(x, nkv, D, k8, ks);
    /* V per channel */
    for (int d = 0; d < D; d++) {
        float a = 0.0f;
        for (long r = 0; r < nkv; r++) {
            float t = fabsf(bf16_to_f32(v[r * D + d]));
            if (t > a)
                a = t;
        }
        if (a == 0.0f) {
            vs[d] = 0.0f;
            for (long r = 0; r < nkv; r++)
                v8[r * D + d] = 0;
            continue;
        }
        vs[d] = a / 448.0f;
        float inv = 448.0f / a;
        for (long r = 0; r < nkv; r++)
            v8[r * D + d] = orc_e4m3_encode(bf16_to_f32(v[r * D + d]) * inv);
    }
    free(x);
    return 0;
}

int orc_quant_head(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                   long nq, long nkv, int D,
                   int8_t *q8, float *qs, int8_t *k8, float *ks, float *mu,
                   uint8_t *v8, float *vs)
{
    return quant_head_impl(q, k, v, nq, nkv, D, NULL, NULL, NULL, NULL,
                           q8, qs, k8, ks, mu, v8, vs, NULL);
}

/* The channel-equalised variant (equalise_channels); eq_exp [D] receives the
 * exponents e. */
int orc_quant_head_eq(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                      long nq, long nkv, int D,
                      int8_t *q8, float *qs, int8_t *k8, float *ks, float *mu,
                      uint8_t *v8, float *vs, int8_t *eq_exp)
{
    if (!eq_exp)
        return 2;
    return quant_head_impl(q, k, v, nq, nkv, D, NULL, NULL, NULL, NULL,
                           q8, qs, k8, ks, mu, v8, vs, eq_exp);
}

int orc_quant_head_rope(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                        long nq, long nkv, int D,
                        const float *q_cos, const float *q_sin,
                        const float *k_cos, const float *k_sin,
                        int8_t *q8, float *qs, int8_t *k8, float *ks, float *mu,
                        uint8_t *v8, float *vs)
{
    if (!q_cos || !q_sin || !k_cos || !k_sin)
        return 2;
    return quant_head_impl(q, k, v, nq, nkv, D, q_cos, q_sin, k_cos, k_sin,
                           q8, qs, k8, ks, mu, v8, vs, NULL);
}

/* Exact integer scores S[i,j] = sum_d q8[i,d] * k8[j,d] for rows i0..i0+ni-1
 * and keys j0..j0+nj-1 (brute force in int64, stored as int32). */
void orc_qk_int32(const int8_t *q8, const int8_t *k8, int D,
                  long i0, long ni, long j0, long nj, int32_t *out)
{
    for (long a = 0; a < ni; a++)
        for (long b = 0; b < nj; b++) {
            int64_t s = 0;
            for (int d = 0; d < D; d++)
                s += (int64_t)q8[(i0 + a) * D + d] * (int64_t)k8[(j0 + b) * D + d];
            out[a * nj + b] = (int32_t)s;
        }
}

/* ------------------------------------------------------------------ */
/* Masks                                                               */
/* ------------------------------------------------------------------ */

/* Keys j < limit are visible to query row i.  Queries are the newest nq
 * tokens of a cache of nkv (bottom-right alignment: query i sits at cache
 * position g = i + nkv - nq).
 *   none          : limit = nkv
 *   causal        : limit = g + 1
 *   block-causal  : every key of the query's own block (of mb tokens) and of
 *                   all earlier blocks: limit = min(nkv, (g/mb + 1) * mb). */
long orc_row_limit(long i, long nq, long nkv, int mask, long mb)
{
    long g = i + (nkv - nq);
    long lim;
    switch (mask) {
    case ORC_MASK_CAUSAL:
        lim = g + 1;
        break;
    case ORC_MASK_BLOCK_CAUSAL:
        lim = (g / mb + 1) * mb;
        break;
    default:
        lim = nkv;
    }
    return lim < nkv ? lim : nkv;
}

/* The keys visible to query row i, as the union [0, sink_end) u [lo, hi).
 * For the none / causal / block-causal masks: sink_end = 0, lo = 0 and
 * hi = orc_row_limit.
 *
 * Sliding window with a persistent reference context (Vidu S1 digest,
 * section "Infra", the sliding-window decoding paragraph): every step
 * attends to a fixed-length window made of (1) the reference context, the
 * tokens taken once from the first frame and the first generated state and
 * kept for the whole stream (the role of a sink token), (2) the cached
 * history states inside the window, (3) the state being denoised.  Reading
 * taken: the cache holds the reference context at positions [0, sink) and
 * then frames of mb tokens; a query at position g >= sink belongs to frame
 * f = (g - sink) / mb and sees the whole reference context plus frames
 * f - win + 1 .. f (its own frame in full, as the block-causal mask does);
 * a query inside the reference context sees the reference context only.
 * With sink = 0 and win >= the number of frames this is the block-causal
 * mask with block mb. */
static void orc_row_window(long i, long nq, long nkv, int mask, long mb, long win, long sink,
                           long *sink_end, long *lo, long *hi)
{
    *sink_end = 0;
    *lo = 0;
    if (mask != ORC_MASK_SLIDING_WINDOW) {
        *hi = orc_row_limit(i, nq, nkv, mask, mb);
        return;
    }
    const long g = i + (nkv - nq);
    const long s0 = sink < nkv ? sink : nkv;
    if (g < s0) {
        *hi = s0;
        return;
    }
    const long f = (g - s0) / mb;
    const long end = s0 + (f + 1) * mb;
    const long first = f - win + 1 > 0 ? f - win + 1 : 0;
    *sink_end = s0;
    *lo = s0 + first * mb;
    *hi = end < nkv ? end : nkv;
}

static int key_visible(long j, long sink_end, long lo, long hi)
{
    return j < sink_end || (j >= lo && j < hi);
}

/* ------------------------------------------------------------------ */
/* Attention, one query row at a time                                  */
/* ------------------------------------------------------------------ */

typedef struct {
    int identity; /* 1: quantizers replaced by identity, arithmetic in fp64 */
    long nq, nkv;
    int D, mask;
    long mb, tkv;
    double eps; /* relative exp2 uncertainty used for the rounding slack */
    /* quantized operands (identity == 0) */
    const int8_t *q8;
    const float *qs;
    const int8_t *k8;
    const float *ks;
    const uint8_t *v8; /* [nkv, D] */
    const float *vs;
    /* full-precision operands (identity == 1), [n, D] doubles */
    const double *qd, *kd, *vd;
    /* rows and outputs */
    const long *rows;
    long nrows;
    double *o;     /* [nrows, D] */
    double *slack; /* [nrows, D] or NULL */
    double *lse;   /* [nrows] natural-log log-sum-exp, or NULL */
    /* block-sparse skipping (NULL: dense): KV tile t (keys t*tkv ..) is
     * visited by query row i only if bmask[(i / bq) * n_kt + t] != 0 */
    const uint8_t *bmask;
    long bq, n_kt;
    /* split-KV form (see attend_row): number of KV ranges, <= 1 for none;
     * bq is then the query tile height */
    int splits;
    /* sliding-window mask (mask == ORC_MASK_SLIDING_WINDOW): frames of mb
     * tokens, win frames per window, sink reference-context tokens */
    long win, sink;
    /* test hook (NULL: off): pert[i * nkv + j] = +1 replaces the exp2 result
     * y of query row i and key j by the largest fp32 value <= y (1 +
     * pert_eps), -1 by the smallest fp32 value >= y (1 - pert_eps): the
     * extreme results of an exp2 whose relative error is up to pert_eps, the
     * uncertainty that the rounding slack is meant to cover */
    const int8_t *pert;
    double pert_eps;
    /* tile columns >= poly_from take the software exp2 (orc_exp2_poly) */
    int poly_from;
} attn_job;

static float exp2_f32(float x) { return (float)exp2((double)x); }

/* Software exp2: the recipe's exp2 for the tile columns >= poly_from (a
 * reading: the target specification says only "exp2 in registers"; the
 * device evaluates this share of the exponentials on its fma units instead
 * of the exp2 unit, and both sides then agree bit for bit).
 * Cody-Waite style reduction x = j + f with j = round-half-even(x) (adding
 * and subtracting 1.5 * 2^23) and |f| <= 1/2, a degree-3 polynomial for 2^f
 * fitted here (minimax relative error on [-1/2, 1/2]; 2^-13.7 including its
 * fp32 Horner evaluation), and 2^j applied by adding j to the exponent field
 * of the polynomial's bits.  x is first raised to -125 so that the exponent
 * field stays normal (a masked key's -inf gives 2^-125 * p(0), whose e4m3
 * code is 0).  Each step is one fp32 operation rounded to nearest-even or an
 * integer add. */
#define ORC_EXP2_C0 0x3f7ffb49u /* 0.999928057 */
#define ORC_EXP2_C1 0x3f31798du /* 0.693260968 */
#define ORC_EXP2_C2 0x3e786f0du /* 0.242611125 */
#define ORC_EXP2_C3 0x3d61fbb0u /* 0.0551716685 */

static float f32_of(uint32_t b)
{
    float f;
    memcpy(&f, &b, 4);
    return f;
}

float orc_exp2_poly(float x)
{
    const float magic = 12582912.0f; /* 1.5 * 2^23 */
    const float xc = x > -125.0f ? x : -125.0f;
    const float t = xc + magic;
    const float jf = t - magic;
    const float f = xc - jf;
    const float p = fmaf(fmaf(fmaf(f32_of(ORC_EXP2_C3), f, f32_of(ORC_EXP2_C2)), f,
                              f32_of(ORC_EXP2_C1)),
                         f, f32_of(ORC_EXP2_C0));
    uint32_t pb, tb;
    memcpy(&pb, &p, 4);
    memcpy(&tb, &t, 4);
    return f32_of(pb + (tb << 23)); /* (t's bits << 23) = j << 23 modulo 2^32 */
}

void orc_exp2_poly_n(const float *x, long n, float *y)
{
    for (long i = 0; i < n; i++)
        y[i] = orc_exp2_poly(x[i]);
}

/* The first tile column (0 .. tkv) whose exponentials use orc_exp2_poly; the
 * recipe's value is ORC_EXP2_POLY_FROM (tkv or more: none).  The setter is
 * for the tests that pin the polynomial's effect; set it before a call, not
 * during one. */
#ifndef ORC_EXP2_POLY_FROM
#define ORC_EXP2_POLY_FROM 128
#endif
static int g_poly_from = ORC_EXP2_POLY_FROM;
void orc_set_exp2_poly_from(int c) { g_poly_from = c; }
int orc_get_exp2_poly_from(void) { return g_poly_from; }


/* Width, in units of y = p*2^8, of the set of e4m3 codes that an fp32 value
 * within relative distance eps of y can round to; zero when that set is one
 * code.  The device's y is an fp32 value, so its admissible values are the
 * fp32 numbers in [y (1 - eps), y (1 + eps)]: the smallest of them is the
 * lower end rounded up to fp32, the largest the upper end rounded down
 * (y (1 +- eps) itself is exact in double for the eps used here). */
static float f32_at_least(double a)
{
    float f = (float)a;
    return (double)f < a ? nextafterf(f, INFINITY) : f;
}

static float f32_at_most(double b)
{
    float f = (float)b;
    return (double)f > b ? nextafterf(f, -INFINITY) : f;
}

static double e4m3_flip_gap(double y, double eps)
{
    uint8_t lo = e4m3_encode_d((double)f32_at_least(y * (1.0 - eps)));
    uint8_t hi = e4m3_encode_d((double)f32_at_most(y * (1.0 + eps)));
    if (lo == hi)
        return 0.0;
#if ORC_PLANT == 4
    return fabs((double)hi - (double)lo);
#endif
    return fabs(orc_e4m3_decode(hi) - orc_e4m3_decode(lo));
}

/* One query row i with the flash-style online softmax over KV tiles of
 * width tkv, visiting tiles in ascending order, only those holding a
 * visible key.  Per tile k (scores in the log2 domain):
 *   m_k   = max(m_{k-1}, max_j t_ij)                  (m_{-1} = -inf)
 *   alpha = 0 if m_{k-1} = -inf else exp2(m_{k-1} - m_k)
 *   p_ij  = exp2(t_ij - m_k)
 *   l     = l * alpha + sum_j p_ij
 *   O     = O * alpha + sum_j w_ij V_j
 * and finally O / l.
 *
 * Quantized mode (the same-quantization result):
 *   C0    = fp32(log2(e) / sqrt(D))             (fp64, rounded once)
 *   sqC   = fp32(sq[i/64] * C0); c_ij = fp32(sqC * sk[j/64])
 *   S_ij  = sum_d q8 k8 (exact integer)
 *   t_ij  = fp32(fp32(S_ij) * c_ij)             (for the max)
 *   P is quantized with the fixed scale 2^8, folded into the exponent:
 *   y_ij  = fp32(exp2(fmaf(fp32(S_ij), c_ij, fp32(8 - m_k))))   (~ 256 p_ij)
 *   l is accumulated in fp32 from y (before quantization),
 *   w_ij  = e4m3(y_ij), V_j = e4m3 code values,
 *   O     = O_acc * vs[d] / l;  lse = (m + log2(l) - 8) * ln 2.
 * Identity mode: t_ij = (q_i . k_j) * log2(e)/sqrt(D), w = p, all fp64.
 */
/* Online softmax of query row i over the KV tiles tl[0 .. nt) (ascending),
 * keys [0, se) u [lo, hi) only; a tile without a visible key leaves the row
 * unchanged and is passed over.  On return o holds the unnormalized sum of
 * P.V in the units of the final running maximum (m, or mf and lf in
 * quantized mode), sl its rounding slack.  o and sl start at zero. */
typedef struct {
    double *o, *sl;
    double m, l;
    float mf, lf;
} attn_part;

static void attend_range(const attn_job *J, long i, long se, long lo, long hi, const long *tl,
                         long nt, attn_part *P, double *acc, double *sacc, int32_t *S, float *c,
                         double *t, long *js)
{
    const int D = J->D;
    const long tkv = J->tkv;
    double *o = P->o;
    double *sl = P->sl;
    const double C64 = 1.4426950408889634 / sqrt((double)D); /* log2(e)/sqrt(D) */
    const float C0 = (float)C64;
    float sqC = 0.0f;
    if (!J->identity)
        sqC = J->qs[i / ORC_BLK] * C0;
    double m = -INFINITY, l = 0.0;
    float mf = -INFINITY, lf = 0.0f;
    for (int d = 0; d < D; d++) {
        o[d] = 0.0;
        if (sl)
            sl[d] = 0.0;
    }

    for (long ti = 0; ti < nt; ti++) {
        const long j0 = tl[ti] * tkv;
        if (J->bmask && !J->bmask[(i / J->bq) * J->n_kt + tl[ti]])
            continue; /* tile switched off by the block mask */
        long nj = 0; /* visible keys of this tile, ascending */
        for (long j = j0; j < j0 + tkv && j < J->nkv; j++)
            if (key_visible(j, se, lo, hi))
                js[nj++] = j;
        if (nj == 0)
            continue;
        /* scores */
        for (long jj = 0; jj < nj; jj++) {
            long j = js[jj];
            if (J->identity) {
                double s = 0.0;
                for (int d = 0; d < D; d++)
                    s += J->qd[i * D + d] * J->kd[j * D + d];
                t[jj] = s * C64;
            } else {
                int64_t s = 0;
                for (int d = 0; d < D; d++)
                    s += (int64_t)J->q8[i * D + d] * (int64_t)J->k8[j * D + d];
                S[jj] = (int32_t)s;
#if ORC_PLANT == 1
                c[jj] = sqC * J->ks[j / 128];
#else
                c[jj] = sqC * J->ks[j / ORC_BLK];
#endif
                t[jj] = (double)((float)S[jj] * c[jj]);
            }
        }
        /* running max and rescale factor */
        double tmax = -INFINITY;
        for (long jj = 0; jj < nj; jj++)
            if (t[jj] > tmax)
                tmax = t[jj];
        double alpha;
        if (J->identity) {
            double mn = m > tmax ? m : tmax;
            alpha = (m == -INFINITY) ? 0.0 : exp2(m - mn);
            m = mn;
        } else {
            float mn = mf > (float)tmax ? mf : (float)tmax;
            alpha = (mf == -INFINITY) ? 0.0 : (double)exp2_f32(mf - mn);
            mf = mn;
        }
        /* probabilities (scaled by 2^8 in quantized mode) and the P.V contribution */
        const float nm8 = 8.0f - mf;
        for (int d = 0; d < D; d++) {
            acc[d] = 0.0;
            sacc[d] = 0.0;
        }
        double rowsum = 0.0;
        float rowsum_f = 0.0f;
        for (long jj = 0; jj < nj; jj++) {
            long j = js[jj];
            if (J->identity) {
                double p = exp2(t[jj] - m);
                rowsum += p;
                for (int d = 0; d < D; d++)
                    acc[d] += p * J->vd[j * D + d];
            } else {
#ifdef ORC_PSCALE_UNFOLDED
                (void)nm8;
                const int poly = 0;
                float y = 256.0f * exp2_f32(fmaf((float)S[jj], c[jj], -mf));
#else
                float x = fmaf((float)S[jj], c[jj], nm8);
                const int poly = (j % tkv) >= J->poly_from;
                float y = poly ? orc_exp2_poly(x) : exp2_f32(x);
#endif
                /* the software exp2 is reproduced exactly: it has neither an
                 * uncertainty (test hook) nor a slack */
                if (!poly && J->pert && J->pert[i * J->nkv + j] > 0)
                    y = f32_at_most((double)y * (1.0 + J->pert_eps));
                else if (!poly && J->pert && J->pert[i * J->nkv + j] < 0)
                    y = f32_at_least((double)y * (1.0 - J->pert_eps));
                double w = orc_e4m3_decode(orc_e4m3_encode(y));
#if ORC_PLANT == 2
                rowsum_f += (float)w;
#else
                rowsum_f += y;
#endif
                double gap = (sl && !poly) ? e4m3_flip_gap((double)y, J->eps) : 0.0;
                for (int d = 0; d < D; d++) {
                    double vv = orc_e4m3_decode(J->v8[j * D + d]);
                    acc[d] += w * vv;
                    if (gap != 0.0)
                        sacc[d] += gap * fabs(vv);
                }
            }
        }
        for (int d = 0; d < D; d++) {
            o[d] = o[d] * alpha + acc[d];
#if ORC_PLANT == 3
            if (sl)
                sl[d] = sl[d] + sacc[d];
#else
            if (sl)
                sl[d] = sl[d] * alpha + sacc[d];
#endif
        }
        if (J->identity)
            l = l * alpha + rowsum;
        else
            lf = lf * (float)alpha + rowsum_f;
    }
    P->m = m;
    P->l = l;
    P->mf = mf;
    P->lf = lf;
}

/* One query row.  Without KV splits: one online softmax over all the row's
 * tiles.  With J->splits = S > 1 (the split-KV form of the device kernel):
 * the KV tiles of the row's query tile (bq rows), i.e. the tiles holding a
 * key visible to at least one of its rows, ascending, nk of them, are cut
 * into S contiguous ranges of that sequence [floor(s nk / S),
 * floor((s+1) nk / S)); each range runs its own online softmax; the partial
 * results are merged with m = max_s m_s, a_s = exp2(m_s - m) (0 for an empty
 * range), O = sum_s a_s O_s and l = sum_s a_s l_s (fp32, ascending s, each
 * product and sum rounded once), then normalized as without splits. */
static void attend_row(const attn_job *J, long r)
{
    const long i = J->rows[r];
    const int D = J->D;
    long se, lo, hi;
    orc_row_window(i, J->nq, J->nkv, J->mask, J->mb, J->win, J->sink, &se, &lo, &hi);
    const long tkv = J->tkv;
    const long n_all = (J->nkv + tkv - 1) / tkv;
    long *tl = (long *)malloc(sizeof(long) * (size_t)(n_all > 0 ? n_all : 1));
    long *js = (long *)malloc(sizeof(long) * (size_t)tkv);
    double *o = J->o + r * D;
    double *sl = J->slack ? J->slack + r * D : NULL;
    double *acc = (double *)calloc((size_t)D, sizeof(double));
    double *sacc = (double *)calloc((size_t)D, sizeof(double));
    int32_t *S = (int32_t *)malloc(sizeof(int32_t) * (size_t)tkv);
    float *c = (float *)malloc(sizeof(float) * (size_t)tkv);
    double *t = (double *)malloc(sizeof(double) * (size_t)tkv);

    double m = -INFINITY, l = 0.0;
    float mf = -INFINITY, lf = 0.0f;
    const int nsplit = J->splits > 1 ? J->splits : 1;
    if (nsplit == 1) {
        attn_part P = {o, sl, 0, 0, 0, 0};
        long nt = 0;
        for (long tt = 0; tt * tkv < hi; tt++)
            tl[nt++] = tt;
        attend_range(J, i, se, lo, hi, tl, nt, &P, acc, sacc, S, c, t, js);
        m = P.m;
        l = P.l;
        mf = P.mf;
        lf = P.lf;
    } else {
        /* the query tile's KV tiles, by brute force over its rows */
        const long q0 = (i / J->bq) * J->bq;
        const long q1 = q0 + J->bq < J->nq ? q0 + J->bq : J->nq;
        long nk = 0;
        for (long tt = 0; tt < n_all; tt++) {
            const long a = tt * tkv, b = a + tkv;
            for (long rr = q0; rr < q1; rr++) {
                long se2, lo2, hi2;
                orc_row_window(rr, J->nq, J->nkv, J->mask, J->mb, J->win, J->sink, &se2, &lo2,
                               &hi2);
                if (a < se2 || (a < hi2 && lo2 < b && lo2 < hi2)) {
                    tl[nk++] = tt;
                    break;
                }
            }
        }
        double *po = (double *)calloc((size_t)D * nsplit, sizeof(double));
        double *ps = (double *)calloc((size_t)D * nsplit, sizeof(double));
        attn_part *parts = (attn_part *)calloc((size_t)nsplit, sizeof(attn_part));
        for (int sp = 0; sp < nsplit; sp++) {
            parts[sp].o = po + (size_t)sp * D;
            parts[sp].sl = sl ? ps + (size_t)sp * D : NULL;
            const long b0 = nk * sp / nsplit, b1 = nk * (sp + 1) / nsplit;
            attend_range(J, i, se, lo, hi, tl + b0, b1 - b0, &parts[sp], acc, sacc, S, c, t, js);
        }
        for (int d = 0; d < D; d++) {
            o[d] = 0.0;
            if (sl)
                sl[d] = 0.0;
        }
        if (J->identity) {
            for (int sp = 0; sp < nsplit; sp++)
                if (parts[sp].m > m)
                    m = parts[sp].m;
            for (int sp = 0; sp < nsplit; sp++) {
                double a = parts[sp].m == -INFINITY ? 0.0 : exp2(parts[sp].m - m);
                for (int d = 0; d < D; d++)
                    o[d] += a * parts[sp].o[d];
                l += a * parts[sp].l;
            }
        } else {
            for (int sp = 0; sp < nsplit; sp++)
                if (parts[sp].mf > mf)
                    mf = parts[sp].mf;
            for (int sp = 0; sp < nsplit; sp++) {
                float a = parts[sp].mf == -INFINITY ? 0.0f : exp2_f32(parts[sp].mf - mf);
                for (int d = 0; d < D; d++) {
                    o[d] += (double)a * parts[sp].o[d];
                    if (sl)
                        sl[d] += (double)a * parts[sp].sl[d];
                }
                lf = lf + a * parts[sp].lf;
            }
        }
        free(po);
        free(ps);
        free(parts);
    }
    /* output; a row that sees no key at all (possible only with a block
     * mask) has no softmax: O = 0 and lse = -inf by definition */
    if ((J->identity && l == 0.0) || (!J->identity && lf == 0.0f)) {
        for (int d = 0; d < D; d++) {
            o[d] = 0.0;
            if (sl)
                sl[d] = 0.0;
        }
        if (J->lse)
            J->lse[r] = -INFINITY;
    } else if (J->identity) {
        for (int d = 0; d < D; d++)
            o[d] = o[d] / l;
        if (J->lse)
            J->lse[r] = (m + log2(l)) * 0.6931471805599453;
    } else {
        for (int d = 0; d < D; d++) {
            double f = (double)J->vs[d] / (double)lf;
            o[d] = o[d] * f;
#if ORC_PLANT == 5
            if (sl)
                sl[d] = sl[d] * (double)J->vs[d];
#else
            if (sl)
                sl[d] = sl[d] * f;
#endif
        }
        if (J->lse)
            J->lse[r] = ((double)mf + log2((double)lf) - 8.0) * 0.6931471805599453;
    }
    free(acc);
    free(sacc);
    free(S);
    free(c);
    free(t);
    free(tl);
    free(js);
}

/* ------------------------------------------------------------------ */
/* Thread fan-out over rows (rows are independent)                     */
/* ------------------------------------------------------------------ */

typedef struct {
    const void *job;
    void (*fn)(const void *, long);
    long r0, r1;
} span;

static void *span_run(void *arg)
{
    span *s = (span *)arg;
    for (long r = s->r0; r < s->r1; r++)
        s->fn(s->job, r);
    return NULL;
}

static void for_rows(const void *job, void (*fn)(const void *, long), long nrows, int nthreads)
{
    if (nthreads < 1)
        nthreads = 1;
    if (nthreads > nrows)
        nthreads = (int)(nrows > 0 ? nrows : 1);
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)nthreads);
    span *sp = (span *)malloc(sizeof(span) * (size_t)nthreads);
    long per = (nrows + nthreads - 1) / nthreads;
    for (int t = 0; t < nthreads; t++) {
        sp[t].job = job;
        sp[t].fn = fn;
        sp[t].r0 = t * per < nrows ? t * per : nrows;
        sp[t].r1 = (t + 1) * per < nrows ? (t + 1) * per : nrows;
        if (t == 0)
            continue;
        pthread_create(&th[t], NULL, span_run, &sp[t]);
    }
    span_run(&sp[0]);
    for (int t = 1; t < nthreads; t++)
        pthread_join(th[t], NULL);
    free(th);
    free(sp);
}

static void attend_row_cb(const void *job, long r) { attend_row((const attn_job *)job, r); }

/* Same-quantization attention for the given query rows of one head.
 * q8/qs/k8/ks/v8/vs as produced by orc_quant_head (v8 token-major [nkv, D]).
 * o, slack: [nrows, D] doubles; lse: [nrows] or NULL; slack may be NULL.
 * eps: relative uncertainty of the device exp2 (plus one fp32 rounding) used
 * to mark e4m3 rounding decisions of p*256 that may go either way. */
int orc_attn_rows_bs(const int8_t *q8, const float *qs, const int8_t *k8, const float *ks,
                     const uint8_t *v8, const float *vs, long nq, long nkv, int D,
                     int mask, long mb, long tkv, double eps,
                     const uint8_t *bmask, long bq, long n_kt,
                     const long *rows, long nrows, double *o, double *slack, double *lse,
                     int nthreads)
{
    if (bmask && (bq <= 0 || n_kt < (nkv + tkv - 1) / tkv))
        return 1;
    if (tkv <= 0 || nq <= 0 || nkv <= 0 || D <= 0)
        return 1;
    if ((mask == ORC_MASK_CAUSAL || mask == ORC_MASK_BLOCK_CAUSAL) && nkv < nq)
        return 1;
    if (mask == ORC_MASK_BLOCK_CAUSAL && mb <= 0)
        return 1;
    attn_job J = {0};
    J.identity = 0;
    J.nq = nq;
    J.nkv = nkv;
    J.D = D;
    J.mask = mask;
    J.mb = mb;
    J.tkv = tkv;
    J.poly_from = g_poly_from;
    J.eps = eps;
    J.q8 = q8;
    J.qs = qs;
    J.k8 = k8;
    J.ks = ks;
    J.v8 = v8;
    J.vs = vs;
    J.rows = rows;
    J.nrows = nrows;
    J.o = o;
    J.slack = slack;
    J.lse = lse;
    J.bmask = bmask;
    J.bq = bq;
    J.n_kt = n_kt;
    if (slack)
        memset(slack, 0, sizeof(double) * (size_t)(nrows * D));
    for_rows(&J, attend_row_cb, nrows, nthreads);
    return 0;
}

/* The same tiled online-softmax loop with the quantizers replaced by
 * identity and all arithmetic in fp64 (q, k, v: [n, D] doubles). */
int orc_attn_rows_identity_bs(const double *q, const double *k, const double *v,
                              long nq, long nkv, int D, int mask, long mb, long tkv,
                              const uint8_t *bmask, long bq, long n_kt,
                              const long *rows, long nrows, double *o, double *lse,
                              int nthreads)
{
    if (bmask && (bq <= 0 || n_kt < (nkv + tkv - 1) / tkv))
        return 1;
    if (tkv <= 0 || nq <= 0 || nkv <= 0 || D <= 0)
        return 1;
    if ((mask == ORC_MASK_CAUSAL || mask == ORC_MASK_BLOCK_CAUSAL) && nkv < nq)
        return 1;
    if (mask == ORC_MASK_BLOCK_CAUSAL && mb <= 0)
        return 1;
    attn_job J = {0};
    J.identity = 1;
    J.nq = nq;
    J.nkv = nkv;
    J.D = D;
    J.mask = mask;
    J.mb = mb;
    J.tkv = tkv;
    J.poly_from = g_poly_from;
    J.qd = q;
    J.kd = k;
    J.vd = v;
    J.rows = rows;
    J.nrows = nrows;
    J.o = o;
    J.lse = lse;
    J.bmask = bmask;
    J.bq = bq;
    J.n_kt = n_kt;
    for_rows(&J, attend_row_cb, nrows, nthreads);
    return 0;
}

/* Dense forms (no block mask). */
/* Split-KV forms (attend_row): the KV tiles of each 128-query tile (bq rows)
 * in `splits` contiguous ranges, each with its own online softmax, merged. */
int orc_attn_rows_split(const int8_t *q8, const float *qs, const int8_t *k8, const float *ks,
                        const uint8_t *v8, const float *vs, long nq, long nkv, int D,
                        int mask, long mb, long tkv, double eps, int splits, long bq,
                        const long *rows, long nrows, double *o, double *slack, double *lse,
                        int nthreads)
{
    if (tkv <= 0 || nq <= 0 || nkv <= 0 || D <= 0 || splits < 1 || bq <= 0)
        return 1;
    if ((mask == ORC_MASK_CAUSAL || mask == ORC_MASK_BLOCK_CAUSAL) && nkv < nq)
        return 1;
    if (mask == ORC_MASK_BLOCK_CAUSAL && mb <= 0)
        return 1;
    attn_job J = {0};
    J.identity = 0;
    J.nq = nq;
    J.nkv = nkv;
    J.D = D;
    J.mask = mask;
    J.mb = mb;
    J.tkv = tkv;
    J.poly_from = g_poly_from;
    J.eps = eps;
    J.q8 = q8;
    J.qs = qs;
    J.k8 = k8;
    J.ks = ks;
    J.v8 = v8;
    J.vs = vs;
    J.rows = rows;
    J.nrows = nrows;
    J.o = o;
    J.slack = slack;
    J.lse = lse;
    J.bq = bq;
    J.splits = splits;
    if (slack)
        memset(slack, 0, sizeof(double) * (size_t)(nrows * D));
    for_rows(&J, attend_row_cb, nrows, nthreads);
    return 0;
}

int orc_attn_rows_identity_split(const double *q, const double *k, const double *v,
                                 long nq, long nkv, int D, int mask, long mb, long tkv,
                                 int splits, long bq, const long *rows, long nrows, double *o,
                                 double *lse, int nthreads)
{
    if (tkv <= 0 || nq <= 0 || nkv <= 0 || D <= 0 || splits < 1 || bq <= 0)
        return 1;
    if ((mask == ORC_MASK_CAUSAL || mask == ORC_MASK_BLOCK_CAUSAL) && nkv < nq)
        return 1;
    if (mask == ORC_MASK_BLOCK_CAUSAL && mb <= 0)
        return 1;
    attn_job J = {0};
    J.identity = 1;
    J.nq = nq;
    J.nkv = nkv;
    J.D = D;
    J.mask = mask;
    J.mb = mb;
    J.tkv = tkv;
    J.poly_from = g_poly_from;
    J.qd = q;
    J.kd = k;
    J.vd = v;
    J.rows = rows;
    J.nrows = nrows;
    J.o = o;
    J.lse = lse;
    J.bq = bq;
    J.splits = splits;
    for_rows(&J, attend_row_cb, nrows, nthreads);
    return 0;
}

int orc_attn_rows(const int8_t *q8, const float *qs, const int8_t *k8, const float *ks,
                  const uint8_t *v8, const float *vs, long nq, long nkv, int D,
                  int mask, long mb, long tkv, double eps,
                  const long *rows, long nrows, double *o, double *slack, double *lse,
                  int nthreads)
{
    return orc_attn_rows_bs(q8, qs, k8, ks, v8, vs, nq, nkv, D, mask, mb, tkv, eps, NULL, 0, 0,
                            rows, nrows, o, slack, lse, nthreads);
}

/* orc_attn_rows with the exp2 perturbation hook (test-suite only): pert is
 * int8 [nq, nkv] of -1, 0, +1, see attn_job.pert. */
int orc_attn_rows_pert(const int8_t *q8, const float *qs, const int8_t *k8, const float *ks,
                       const uint8_t *v8, const float *vs, long nq, long nkv, int D,
                       int mask, long mb, long tkv, double eps, const int8_t *pert,
                       double pert_eps, const long *rows, long nrows, double *o, double *slack,
                       double *lse, int nthreads)
{
    if (tkv <= 0 || nq <= 0 || nkv <= 0 || D <= 0 || !pert)
        return 1;
    if ((mask == ORC_MASK_CAUSAL || mask == ORC_MASK_BLOCK_CAUSAL) && nkv < nq)
        return 1;
    if (mask == ORC_MASK_BLOCK_CAUSAL && mb <= 0)
        return 1;
    attn_job J = {0};
    J.nq = nq;
    J.nkv = nkv;
    J.D = D;
    J.mask = mask;
    J.mb = mb;
    J.tkv = tkv;
    J.poly_from = g_poly_from;
    J.eps = eps;
    J.q8 = q8;
    J.qs = qs;
    J.k8 = k8;
    J.ks = ks;
    J.v8 = v8;
    J.vs = vs;
    J.rows = rows;
    J.nrows = nrows;
    J.o = o;
    J.slack = slack;
    J.lse = lse;
    J.pert = pert;
    J.pert_eps = pert_eps;
    if (slack)
        memset(slack, 0, sizeof(double) * (size_t)(nrows * D));
    for_rows(&J, attend_row_cb, nrows, nthreads);
    return 0;
}

int orc_attn_rows_identity(const double *q, const double *k, const double *v,
                           long nq, long nkv, int D, int mask, long mb, long tkv,
                           const long *rows, long nrows, double *o, double *lse,
                           int nthreads)
{
    return orc_attn_rows_identity_bs(q, k, v, nq, nkv, D, mask, mb, tkv, NULL, 0, 0, rows, nrows,
                                     o, lse, nthreads);
}

/* ------------------------------------------------------------------ */
/* Full-precision attention: the plain definition                       */
/* O_i = sum_j softmax_j(q_i . k_j / sqrt(D) over visible j) v_j, fp64 */
/* from the bf16 inputs.                                               */
/* ------------------------------------------------------------------ */

typedef struct {
    const uint16_t *q, *k, *v;
    long nq, nkv;
    int D, mask;
    long mb;
    const long *rows;
    double *o;
    long win, sink; /* sliding-window mask only */
} fp64_job;

static void fp64_row(const void *job, long r)
{
    const fp64_job *J = (const fp64_job *)job;
    const int D = J->D;
    const long i = J->rows[r];
    long se, lo, lim;
    orc_row_window(i, J->nq, J->nkv, J->mask, J->mb, J->win, J->sink, &se, &lo, &lim);
    double *s = (double *)malloc(sizeof(double) * (size_t)lim);
    double *qi = (double *)malloc(sizeof(double) * (size_t)D);
    double *o = J->o + r * D;
    const double scale = 1.0 / sqrt((double)D);
    for (int d = 0; d < D; d++)
        qi[d] = (double)bf16_to_f32(J->q[i * D + d]);
    double mx = -INFINITY;
    for (long j = 0; j < lim; j++) {
        if (!key_visible(j, se, lo, lim))
            continue;
        double a = 0.0;
        for (int d = 0; d < D; d++)
            a += qi[d] * (double)bf16_to_f32(J->k[j * D + d]);
        s[j] = a * scale;
        if (s[j] > mx)
            mx = s[j];
    }
    double den = 0.0;
    for (int d = 0; d < D; d++)
        o[d] = 0.0;
    for (long j = 0; j < lim; j++) {
        if (!key_visible(j, se, lo, lim))
            continue;
        double p = exp(s[j] - mx);
        den += p;
        for (int d = 0; d < D; d++)
            o[d] += p * (double)bf16_to_f32(J->v[j * D + d]);
    }
    for (int d = 0; d < D; d++)
        o[d] /= den;
    free(s);
    free(qi);
}

int orc_attn_fp64_rows(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                       long nq, long nkv, int D, int mask, long mb,
                       const long *rows, long nrows, double *o, int nthreads)
{
    if (nq <= 0 || nkv <= 0 || D <= 0)
        return 1;
    if ((mask == ORC_MASK_CAUSAL || mask == ORC_MASK_BLOCK_CAUSAL) && nkv < nq)
        return 1;
    if (mask == ORC_MASK_BLOCK_CAUSAL && mb <= 0)
        return 1;
    fp64_job J = {q, k, v, nq, nkv, D, mask, mb, rows, o, 0, 0};
    for_rows(&J, fp64_row, nrows, nthreads);
    return 0;
}

/* ------------------------------------------------------------------ */
/* Sliding-window forms (orc_row_window): frames of mb tokens, win      */
/* frames per window, sink reference-context tokens.                    */
/* ------------------------------------------------------------------ */

static int window_ok(long nq, long nkv, int D, long mb, long win, long sink)
{
    return nq > 0 && nkv >= nq && D > 0 && mb > 0 && win > 0 && sink >= 0;
}

int orc_attn_fp64_rows_win(const uint16_t *q, const uint16_t *k, const uint16_t *v, long nq,
                           long nkv, int D, long mb, long win, long sink, const long *rows,
                           long nrows, double *o, int nthreads)
{
    if (!window_ok(nq, nkv, D, mb, win, sink))
        return 1;
    fp64_job J = {q, k, v, nq, nkv, D, ORC_MASK_SLIDING_WINDOW, mb, rows, o, win, sink};
    for_rows(&J, fp64_row, nrows, nthreads);
    return 0;
}

/* Same-quantization attention under the sliding-window mask; splits > 1 is
 * the split-KV form over the query tile's KV tiles (bq query rows). */
int orc_attn_rows_win(const int8_t *q8, const float *qs, const int8_t *k8, const float *ks,
                      const uint8_t *v8, const float *vs, long nq, long nkv, int D, long mb,
                      long win, long sink, long tkv, double eps, int splits, long bq,
                      const long *rows, long nrows, double *o, double *slack, double *lse,
                      int nthreads)
{
    if (!window_ok(nq, nkv, D, mb, win, sink) || tkv <= 0 || splits < 1 || bq <= 0)
        return 1;
    attn_job J = {0};
    J.identity = 0;
    J.nq = nq;
    J.nkv = nkv;
    J.D = D;
    J.mask = ORC_MASK_SLIDING_WINDOW;
    J.mb = mb;
    J.win = win;
    J.sink = sink;
    J.tkv = tkv;
    J.poly_from = g_poly_from;
    J.eps = eps;
    J.q8 = q8;
    J.qs = qs;
    J.k8 = k8;
    J.ks = ks;
    J.v8 = v8;
    J.vs = vs;
    J.rows = rows;
    J.nrows = nrows;
    J.o = o;
    J.slack = slack;
    J.lse = lse;
    J.bq = bq;
    J.splits = splits;
    if (slack)
        memset(slack, 0, sizeof(double) * (size_t)(nrows * D));
    for_rows(&J, attend_row_cb, nrows, nthreads);
    return 0;
}

int orc_attn_rows_identity_win(const double *q, const double *k, const double *v, long nq,
                               long nkv, int D, long mb, long win, long sink, long tkv,
                               int splits, long bq, const long *rows, long nrows, double *o,
                               double *lse, int nthreads)
{
    if (!window_ok(nq, nkv, D, mb, win, sink) || tkv <= 0 || splits < 1 || bq <= 0)
        return 1;
    attn_job J = {0};
    J.identity = 1;
    J.nq = nq;
    J.nkv = nkv;
    J.D = D;
    J.mask = ORC_MASK_SLIDING_WINDOW;
    J.mb = mb;
    J.win = win;
    J.sink = sink;
    J.tkv = tkv;
    J.poly_from = g_poly_from;
    J.qd = q;
    J.kd = k;
    J.vd = v;
    J.rows = rows;
    J.nrows = nrows;
    J.o = o;
    J.lse = lse;
    J.bq = bq;
    J.splits = splits;
    for_rows(&J, attend_row_cb, nrows, nthreads);
    return 0;
}

/* The visible-key description of one row (for the tests): out[0..2] =
 * sink_end, lo, hi. */
void orc_row_window_export(long i, long nq, long nkv, int mask, long mb, long win, long sink,
                           long *out)
{
    orc_row_window(i, nq, nkv, mask, mb, win, sink, &out[0], &out[1], &out[2]);
}

/* ------------------------------------------------------------------ */
/* Per-block W8A8 linear layer (Y = X W^T with INT8 operands)          */
/* ------------------------------------------------------------------ */
/* The pages quantize the linear layers to 8-bit weights and activations
 * per block, on INT8 tensor cores, because per-tensor and per-channel
 * scales are stretched by outliers (Vidu S1 digest, "Infra"; TurboDiffusion
 * notes, W8A8 bullet).  Readings taken here: blocks are 128 channels wide
 * along the reduction dimension K; an activation block is one token x 128
 * channels, a weight block 128 output channels x 128 channels; both are
 * symmetric absmax/127 with round-half-to-even, as the attention quantizer.
 * Each 128-channel group is reduced exactly in integers and promoted into an
 * fp32 running sum, group by group in ascending order:
 *   y = fmaf((float)P_g, fp32(sx[m,g] * sw[n/128,g]), y),
 * and Y is y rounded to bf16 (round-half-to-even). */

#define ORC_W8A8_G 128

static void quant_group_i8(const float *x, long n, int8_t *q, float *scale)
{
    float a = 0.0f;
    for (long i = 0; i < n; i++) {
        float t = fabsf(x[i]);
        if (t > a)
            a = t;
    }
    if (a == 0.0f) {
        *scale = 0.0f;
        memset(q, 0, (size_t)n);
        return;
    }
    *scale = a / 127.0f;
    float inv = 127.0f / a;
    for (long i = 0; i < n; i++) {
        float t = nearbyintf(x[i] * inv);
        if (t > 127.0f)
            t = 127.0f;
        if (t < -127.0f)
            t = -127.0f;
        q[i] = (int8_t)t;
    }
}

/* X [M, K] bf16 bits, K a multiple of 128 -> xq [M, K] int8, sx [M, K/128]. */
int orc_w8a8_quant_act(const uint16_t *x, long M, long K, int8_t *xq, float *sx)
{
    if (M <= 0 || K <= 0 || K % ORC_W8A8_G)
        return 1;
    const long G = K / ORC_W8A8_G;
    float buf[ORC_W8A8_G];
    for (long m = 0; m < M; m++)
        for (long g = 0; g < G; g++) {
            for (int c = 0; c < ORC_W8A8_G; c++)
                buf[c] = bf16_to_f32(x[m * K + g * ORC_W8A8_G + c]);
            quant_group_i8(buf, ORC_W8A8_G, xq + m * K + g * ORC_W8A8_G, sx + m * G + g);
        }
    return 0;
}

/* W [N, K] bf16 bits, N and K multiples of 128 -> wq [N, K] int8,
 * sw [N/128, K/128] (one scale per 128 x 128 block). */
int orc_w8a8_quant_weight(const uint16_t *w, long N, long K, int8_t *wq, float *sw)
{
    if (N <= 0 || K <= 0 || N % ORC_W8A8_G || K % ORC_W8A8_G)
        return 1;
    const long G = K / ORC_W8A8_G, NB = N / ORC_W8A8_G;
    float *blk = (float *)malloc(sizeof(float) * ORC_W8A8_G * ORC_W8A8_G);
    int8_t *qb = (int8_t *)malloc(ORC_W8A8_G * ORC_W8A8_G);
    if (!blk || !qb) {
        free(blk);
        free(qb);
        return 1;
    }
    for (long nb = 0; nb < NB; nb++)
        for (long g = 0; g < G; g++) {
            for (int r = 0; r < ORC_W8A8_G; r++)
                for (int c = 0; c < ORC_W8A8_G; c++)
                    blk[r * ORC_W8A8_G + c] =
                        bf16_to_f32(w[(nb * ORC_W8A8_G + r) * K + g * ORC_W8A8_G + c]);
            quant_group_i8(blk, (long)ORC_W8A8_G * ORC_W8A8_G, qb, sw + nb * G + g);
            for (int r = 0; r < ORC_W8A8_G; r++)
                memcpy(wq + (nb * ORC_W8A8_G + r) * K + g * ORC_W8A8_G, qb + r * ORC_W8A8_G,
                       ORC_W8A8_G);
        }
    free(blk);
    free(qb);
    return 0;
}

typedef struct {
    const int8_t *xq, *wq;
    const float *sx, *sw;
    long N, K;
    const long *rows;
    float *y;
} w8a8_job;

static void w8a8_row(const void *job, long r)
{
    const w8a8_job *J = (const w8a8_job *)job;
    const long m = J->rows[r], K = J->K, G = K / ORC_W8A8_G;
    for (long n = 0; n < J->N; n++) {
        float y = 0.0f;
        for (long g = 0; g < G; g++) {
            int64_t p = 0;
            for (int c = 0; c < ORC_W8A8_G; c++)
                p += (int64_t)J->xq[m * K + g * ORC_W8A8_G + c] *
                     (int64_t)J->wq[n * K + g * ORC_W8A8_G + c];
            const float s = J->sx[m * G + g] * J->sw[(n / ORC_W8A8_G) * G + g];
            y = fmaf((float)p, s, y);
        }
        J->y[r * J->N + n] = y;
    }
}

/* Rows `rows` of Y = (dequantized X)(dequantized W)^T by the promotion rule
 * above: y [nrows, N] fp32 (round to bf16 for the layer's output). */
int orc_w8a8_gemm_rows(const int8_t *xq, const float *sx, const int8_t *wq, const float *sw,
                       long M, long N, long K, const long *rows, long nrows, float *y,
                       int nthreads)
{
    if (M <= 0 || N <= 0 || K <= 0 || K % ORC_W8A8_G || N % ORC_W8A8_G)
        return 1;
    for (long r = 0; r < nrows; r++)
        if (rows[r] < 0 || rows[r] >= M)
            return 1;
    w8a8_job J = {xq, wq, sx, sw, N, K, rows, y};
    for_rows(&J, w8a8_row, nrows, nthreads);
    return 0;
}
