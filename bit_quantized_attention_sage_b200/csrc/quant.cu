// quant.cu -- sage_quant_qk: per-block INT8 quantization of Q and of the
// mean-smoothed K, and per-channel FP8 e4m3 quantization of V.
//
// SageAttention's quantizer (low-bit attention, "Vidu S1" digest section
// "Infra" and the TurboDiffusion notes on 8-bit block-wise quantization):
// 64-token blocks, symmetric absmax/127 INT8 codes with round-half-to-even,
// K smoothed by its per-channel mean over all tokens, V cast to e4m3 with a
// per-channel absmax/448 scale.
//
// Three stream-ordered kernels (the K mean and the V maxima span all tokens
// of a head, so the K and V codes need a second pass):
//   pass1    one CTA per (head, 64-token block): Q block codes + scale; fp64
//            per-channel sums of the K block in ascending token order; V
//            block per-channel maxima.
//   finalize one CTA per (head, 8 channels): ascending sum of the block
//            sums -> k_mean; max of the block maxima -> v_scale, 448/absmax.
//   pass2    one CTA per (head, 64-token block): K - mean block codes + scale;
//            V codes, token-major like the K codes ([B,H,Nkv_pad,D]).
// Memory traffic: 16-byte vectorised bf16 loads; every fp32 operation is an
// explicit IEEE round-to-nearest intrinsic so the codes match a plain CPU
// implementation bit for bit.
//
// Rotary variant (sage_quant_qk_rope; the digest's RoPE Repositioning: the
// cache holds features before RoPE, which is applied at their current
// positions): Q and K are rotated in fp32 as they are loaded, channel pair
// (2p, 2p+1) of token n by the caller's cos/sin[n][p], and quantized as
// above; the K mean is that of the rotated keys.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "quant.cuh"
#include "sm100.cuh"

namespace sage {

namespace {

// Programmatic dependent launch.  finalize and pass 2 are launched with
// programmatic stream serialization, so their CTAs may be scheduled while
// the previous kernel's last CTAs still run; grid_dep_wait holds them until
// that grid has completed and its writes are visible.  grid_dep_trigger lets
// the next kernel launch once every CTA of this grid has passed it.
__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_dep_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

constexpr int kBlk = 64;
constexpr int kThreads = 256;

__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ void unpack8(const uint4& u, float (&x)[8]) {
  x[0] = bf16lo(u.x); x[1] = bf16hi(u.x);
  x[2] = bf16lo(u.y); x[3] = bf16hi(u.y);
  x[4] = bf16lo(u.z); x[5] = bf16hi(u.z);
  x[6] = bf16lo(u.w); x[7] = bf16hi(u.w);
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Max over the CTA (kThreads threads); every thread gets the result.
__device__ __forceinline__ float block_max(float v, float* red) {
  v = warp_max(v);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  __syncthreads();  // `red` may still be read by a previous call
  if (l == 0) red[w] = v;
  __syncthreads();
  float r = red[0];
#pragma unroll
  for (int i = 1; i < kThreads / 32; i++) r = fmaxf(r, red[i]);
  return r;
}

// Pair rotation (x0, x1) -> (x0 c - x1 s, x0 s + x1 c): each product and
// each fma rounded once.
__device__ __forceinline__ void rot_pair(float& x0, float& x1, float c, float s) {
  const float t = __fmul_rn(x1, s), u = __fmul_rn(x1, c);
  const float r0 = __fmaf_rn(x0, c, -t), r1 = __fmaf_rn(x0, s, u);
  x0 = r0;
  x1 = r1;
}

// The cos / sin of the 4 channel pairs of one 8-channel chunk (channels
// col..col+7 of token `tok`; tables [N][D/2], 16-byte aligned rows).
template <int D>
__device__ __forceinline__ void rope_load(const float* cs, const float* sn, int tok, int col,
                                          float4& c, float4& s) {
  const size_t o = static_cast<size_t>(tok) * (D / 2) + col / 2;
  c = __ldg(reinterpret_cast<const float4*>(cs + o));
  s = __ldg(reinterpret_cast<const float4*>(sn + o));
}

__device__ __forceinline__ void rope_apply(float (&x)[8], const float4& c, const float4& s) {
  rot_pair(x[0], x[1], c.x, s.x);
  rot_pair(x[2], x[3], c.y, s.y);
  rot_pair(x[4], x[5], c.z, s.z);
  rot_pair(x[6], x[7], c.w, s.w);
}

// The 16-byte chunk `chunk` (row-major over the block's D / 8 chunks per row)
// of K / V block `blk` of head `bh`, through the gather map.
template <int D>
__device__ __forceinline__ const uint4* kv_chunk(const uint16_t* src, const QuantArgs& a, int bh,
                                                 int blk, int chunk) {
  constexpr int kChunksPerRow = D / 8;
  const int row = blk * kBlk + chunk / kChunksPerRow;
  const int srow = row < a.kv_split ? row : row + a.kv_gap;
  return reinterpret_cast<const uint4*>(src + (static_cast<size_t>(bh) * a.Nkv_src + srow) * D) +
         chunk % kChunksPerRow;
}

// The INT8 code clamp(rne(x * inv), -127, 127) of one value, as the low byte
// of the returned word.  With |x| <= a (the block absmax) and inv =
// fp32(127 / a), |fp32(x * inv)| <= 127 (1 + 2^-24)^2 < 127.5, so the clamp
// never acts and rne(y) is taken by adding 1.5 * 2^23: for |y| < 2^22 the
// fp32 sum rounds y to the nearest integer, ties to even (the ulp there is
// 1 and 1.5 * 2^23 is even), and its low byte is the two's-complement code.
__device__ __forceinline__ uint32_t q_i8_word(float x, float inv) {
  return __float_as_uint(__fadd_rn(__fmul_rn(x, inv), 12582912.0f));
}

// clamp(rne(x * inv), -127, 127) by the conversion unit: used when inv is
// infinite (a block absmax below 127 / FLT_MAX), where the sum above is not.
__device__ __forceinline__ int8_t q_i8(float x, float inv) {
  int q = __float2int_rn(__fmul_rn(x, inv));
  q = q > 127 ? 127 : (q < -127 ? -127 : q);
  return static_cast<int8_t>(q);
}

// Low bytes of four words -> one packed word (first word in the low byte).
__device__ __forceinline__ uint32_t pack_low_bytes(uint32_t w0, uint32_t w1, uint32_t w2, uint32_t w3) {
  return __byte_perm(__byte_perm(w0, w1, 0x0040u), __byte_perm(w2, w3, 0x0040u), 0x5410u);
}

// Quantize the 64 x D block held as `ch` 16-byte chunks per thread (x[c][8],
// chunk index c*kThreads + tid), write codes and the block scale.  Rows >=
// `valid` are written as zero and excluded from the max.
template <int D, int CH>
__device__ __forceinline__ void quant_block_store(float (&x)[CH][8], int valid, int8_t* codes,
                                                  float* scale_out, float* red) {
  constexpr int kChunksPerRow = D / 8;
  float a = 0.0f;
#pragma unroll
  for (int c = 0; c < CH; c++) {
    const int chunk = c * kThreads + threadIdx.x;
    const int row = chunk / kChunksPerRow;
    if (row < valid) {
#pragma unroll
      for (int e = 0; e < 8; e++) a = fmaxf(a, fabsf(x[c][e]));
    }
  }
  a = block_max(a, red);
  const float scale = (a == 0.0f) ? 0.0f : __fdiv_rn(a, 127.0f);
  const float inv = (a == 0.0f) ? 0.0f : __fdiv_rn(127.0f, a);
#pragma unroll
  for (int c = 0; c < CH; c++) {
    const int chunk = c * kThreads + threadIdx.x;
    const int row = chunk / kChunksPerRow;
    const int col = (chunk % kChunksPerRow) * 8;
    uint32_t lo = 0, hi = 0;
    if (row < valid && a != 0.0f) {
      if (inv != INFINITY) {
        uint32_t w[8];
#pragma unroll
        for (int e = 0; e < 8; e++) w[e] = q_i8_word(x[c][e], inv);
        lo = pack_low_bytes(w[0], w[1], w[2], w[3]);
        hi = pack_low_bytes(w[4], w[5], w[6], w[7]);
      } else {
#pragma unroll
        for (int e = 0; e < 4; e++) {
          lo |= static_cast<uint32_t>(static_cast<uint8_t>(q_i8(x[c][e], inv))) << (8 * e);
          hi |= static_cast<uint32_t>(static_cast<uint8_t>(q_i8(x[c][e + 4], inv))) << (8 * e);
        }
      }
    }
    *reinterpret_cast<uint2*>(codes + static_cast<size_t>(row) * D + col) = make_uint2(lo, hi);
  }
  if (threadIdx.x == 0) *scale_out = scale;
}

// Channel maxima of |x| over the valid rows of a 64 x D bf16 block staged in
// shared memory (thread t < D: channel t).
template <int D>
__device__ __forceinline__ float channel_absmax(const uint16_t* blk, int valid, int t) {
  float m = 0.0f;
  for (int r = 0; r < valid; r++)
    m = fmaxf(m, fabsf(__uint_as_float(static_cast<uint32_t>(blk[r * D + t]) << 16)));
  return m;
}

// pass 1.  EQ (channel equalisation): the Q codes wait for the per-channel
// factors, so a Q block only records its channel maxima here, and a K block
// also its channel maxima and minima.
template <int D, bool ROPE, bool EQ>
__global__ void __launch_bounds__(kThreads) k_quant_pass1(QuantArgs a) {
  grid_dep_trigger();
  constexpr int kChunksPerRow = D / 8;
  constexpr int CH = kBlk * kChunksPerRow / kThreads;  // chunks per thread
  __shared__ float red[kThreads / 32];
  // staging of one 64-token block: bf16 K then bf16 V; or (rotary variant)
  // bf16 V, then the rotated K in fp32
  __shared__ __align__(16) uint32_t stage[kBlk * D];
  uint16_t* ks = reinterpret_cast<uint16_t*>(stage);
  uint16_t* vsm = ks + kBlk * D;

  // rotary variant: heads run fastest, so that the CTAs in flight share the
  // table rows of their tokens through L2
  const int blk = ROPE ? blockIdx.y : blockIdx.x;
  const int bh = ROPE ? blockIdx.x : blockIdx.y;
  const int nqb = (a.Nq + kBlk - 1) / kBlk;
  const int nkb = (a.Nkv + kBlk - 1) / kBlk;

  if (EQ && blk < nqb) {  // Q block: channel maxima of |Q|
    // Thread t holds the 8 channels of group t mod (D/8) in CH rows; the
    // lanes of a warp that share a group combine by shuffles, the warps
    // through shared memory (rows past `valid` read as 0, which no maximum
    // of magnitudes can exceed).
    const int valid = min(kBlk, a.Nq - blk * kBlk);
    const uint4* src = reinterpret_cast<const uint4*>(
        a.q + (static_cast<size_t>(bh) * a.Nq + static_cast<size_t>(blk) * kBlk) * D);
    float mx[8];
#pragma unroll
    for (int e = 0; e < 8; e++) mx[e] = 0.0f;
#pragma unroll
    for (int c = 0; c < CH; c++) {
      const int chunk = c * kThreads + threadIdx.x;
      float x[8];
      unpack8(chunk / kChunksPerRow < valid ? __ldg(src + chunk) : make_uint4(0, 0, 0, 0), x);
#pragma unroll
      for (int e = 0; e < 8; e++) mx[e] = fmaxf(mx[e], fabsf(x[e]));
    }
#pragma unroll
    for (int o = kChunksPerRow; o < 32; o <<= 1)
#pragma unroll
      for (int e = 0; e < 8; e++) mx[e] = fmaxf(mx[e], __shfl_xor_sync(0xffffffffu, mx[e], o));
    float* red8 = reinterpret_cast<float*>(stage);  // [warp][channel]
    const int lane = threadIdx.x & 31, wp = threadIdx.x >> 5;
    if (lane < kChunksPerRow) {
#pragma unroll
      for (int e = 0; e < 8; e++) red8[wp * D + lane * 8 + e] = mx[e];
    }
    __syncthreads();
    if (threadIdx.x < D) {
      float m = red8[threadIdx.x];
#pragma unroll
      for (int w2 = 1; w2 < kThreads / 32; w2++) m = fmaxf(m, red8[w2 * D + threadIdx.x]);
      a.ws_qmax[(static_cast<size_t>(bh) * nqb + blk) * D + threadIdx.x] = m;
    }
    __syncthreads();  // the staging area is reused by the K / V block
  } else if (blk < nqb) {  // Q block: codes and scale
    const int valid = min(kBlk, a.Nq - blk * kBlk);
    const uint4* src = reinterpret_cast<const uint4*>(
        a.q + (static_cast<size_t>(bh) * a.Nq + static_cast<size_t>(blk) * kBlk) * D);
    float x[CH][8];
    uint4 u[CH];
    float4 rc[ROPE ? CH : 1], rs[ROPE ? CH : 1];  // all loads first, then the math
#pragma unroll
    for (int c = 0; c < CH; c++) {
      const int chunk = c * kThreads + threadIdx.x;
      const int row = chunk / kChunksPerRow;
      u[c] = make_uint4(0, 0, 0, 0);
      if (row < valid) u[c] = __ldg(src + chunk);
      if constexpr (ROPE) {
        rc[c] = rs[c] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
        if (row < valid)
          rope_load<D>(a.q_cos, a.q_sin, blk * kBlk + row, (chunk % kChunksPerRow) * 8, rc[c], rs[c]);
      }
    }
#pragma unroll
    for (int c = 0; c < CH; c++) {
      unpack8(u[c], x[c]);
      if constexpr (ROPE) rope_apply(x[c], rc[c], rs[c]);
    }
    int8_t* codes = a.q_i8 + (static_cast<size_t>(bh) * nqb + blk) * kBlk * D;
    quant_block_store<D, CH>(x, valid, codes, a.q_scale + static_cast<size_t>(bh) * nqb + blk,
                             red);
  }

  if (blk < nkb && ROPE) {  // V block maxima, then sums of the rotated K block
    const int valid = min(kBlk, a.Nkv - blk * kBlk);
    const size_t ws = (static_cast<size_t>(bh) * nkb + blk) * D;
    const int t = threadIdx.x;
    // every load of the block first: K chunks and their angles (kept in
    // registers), V chunks (staged)
    uint4 ku[CH];
    float4 kc[CH], ksn[CH];
#pragma unroll
    for (int c = 0; c < CH; c++) {
      const int chunk = c * kThreads + threadIdx.x;
      const int row = chunk / kChunksPerRow;
      if (row < valid) {
        ku[c] = __ldg(kv_chunk<D>(a.k, a, bh, blk, chunk));
        rope_load<D>(a.k_cos, a.k_sin, blk * kBlk + row, (chunk % kChunksPerRow) * 8, kc[c], ksn[c]);
      }
    }
#pragma unroll
    for (int c = 0; c < CH; c++) {
      const int chunk = c * kThreads + threadIdx.x;
      if (chunk / kChunksPerRow < valid)
        reinterpret_cast<uint4*>(ks)[chunk] = __ldg(kv_chunk<D>(a.v, a, bh, blk, chunk));
    }
    __syncthreads();
    if (t >= D && t < 2 * D) {  // max |V| of channel t - D
      const int d = t - D;
      float m = 0.0f;
      for (int r = 0; r < valid; r++)
        m = fmaxf(m, fabsf(__uint_as_float(static_cast<uint32_t>(ks[r * D + d]) << 16)));
      a.ws_vmax[ws + d] = m;
    }
    __syncthreads();  // V is read; the rotated K overwrites the staging area
    float* kf = reinterpret_cast<float*>(stage);
#pragma unroll
    for (int c = 0; c < CH; c++) {
      const int chunk = c * kThreads + threadIdx.x;
      const int row = chunk / kChunksPerRow;
      if (row < valid) {
        float x[8];
        unpack8(ku[c], x);
        rope_apply(x, kc[c], ksn[c]);
        reinterpret_cast<float4*>(kf)[2 * chunk] = make_float4(x[0], x[1], x[2], x[3]);
        reinterpret_cast<float4*>(kf)[2 * chunk + 1] = make_float4(x[4], x[5], x[6], x[7]);
      }
    }
    __syncthreads();
    if (t < D) {  // fp64 sum of channel t, ascending token order
      double s = 0.0;
      for (int r = 0; r < valid; r++) s = __dadd_rn(s, static_cast<double>(kf[r * D + t]));
      a.ws_ksum[ws + t] = s;
    }
  } else if (blk < nkb) {  // K block sums and V block maxima
    const int valid = min(kBlk, a.Nkv - blk * kBlk);
#pragma unroll
    for (int c = 0; c < CH; c++) {
      const int chunk = c * kThreads + threadIdx.x;
      const int row = chunk / kChunksPerRow;
      if (row < valid) {
        reinterpret_cast<uint4*>(ks)[chunk] = __ldg(kv_chunk<D>(a.k, a, bh, blk, chunk));
        reinterpret_cast<uint4*>(vsm)[chunk] = __ldg(kv_chunk<D>(a.v, a, bh, blk, chunk));
      }
    }
    __syncthreads();
    const size_t ws = (static_cast<size_t>(bh) * nkb + blk) * D;
    const int t = threadIdx.x;
    if (t < D) {  // fp64 sum of channel t, ascending token order
      double s = 0.0;
      float mx = -INFINITY, mn = INFINITY;
      for (int r = 0; r < valid; r++) {
        const float x = __uint_as_float(static_cast<uint32_t>(ks[r * D + t]) << 16);
        s = __dadd_rn(s, static_cast<double>(x));
        if (EQ) {
          mx = fmaxf(mx, x);
          mn = fminf(mn, x);
        }
      }
      a.ws_ksum[ws + t] = s;
      if (EQ) {
        a.ws_kmax[ws + t] = mx;
        a.ws_kmin[ws + t] = mn;
      }
    } else if (t < 2 * D) {  // max |V| of channel t - D
      a.ws_vmax[ws + t - D] = channel_absmax<D>(vsm, valid, t - D);
    }
  }
}

// floor(log2 x) of a finite x > 0 (normal or subnormal), from its bits.
__device__ __forceinline__ int floor_log2(float x) {
  const uint32_t b = __float_as_uint(x);
  const int ef = static_cast<int>((b >> 23) & 0xFF);
  return ef ? ef - 127 : (31 - __clz(static_cast<int>(b & 0x7FFFFF))) - 149;
}

constexpr int kEqMax = 32;  // |e| limit of the channel equalisation

// Channel equalisation exponent of channel d (finalize, EQ): aq = max |Q|,
// ak = max |fp32(K - mu)|, which, fp32 subtraction being monotone, is the
// larger of |fp32(kmax - mu)| and |fp32(kmin - mu)|; e = floor((floor(log2
// ak) - floor(log2 aq)) / 2) in [-kEqMax, kEqMax], 0 if either is 0.
__device__ __forceinline__ int eq_exponent(float aq, float kmax, float kmin, float mu) {
  const float ak = fmaxf(fabsf(__fsub_rn(kmax, mu)), fabsf(__fsub_rn(kmin, mu)));
  if (!(aq > 0.0f) || !(ak > 0.0f)) return 0;
  const int t = floor_log2(ak) - floor_log2(aq);
  const int e = t >= 0 ? t / 2 : -((1 - t) / 2);
  return e > kEqMax ? kEqMax : (e < -kEqMax ? -kEqMax : e);
}

// One CTA per (head, 8 channels).  The fp64 block sums of a channel must be
// added one after the other in ascending block order (the canonical order
// that makes the mean reproducible): the CTA stages up to 512 block sums
// per channel in shared memory with loads spread over all its threads, then
// one thread per channel adds them in order (shared-memory reads issued
// eight ahead of the additions, so that the chain of fp64 additions is the
// only serial part).  The V block maxima and the equalisation maxima are
// order-free: every thread reduces the blocks it loaded, then the CTA
// combines its 32 partial maxima per channel.
constexpr int kFinCh = 8;                      // channels per CTA
constexpr int kFinRows = kThreads / kFinCh;    // 32 threads per channel
constexpr int kFinChunk = 512;                 // blocks per staged chunk

__global__ void __launch_bounds__(kThreads) k_quant_finalize(QuantArgs a) {
  grid_dep_wait();
  grid_dep_trigger();
  __shared__ double part[kFinChunk][kFinCh];   // 32 KB
  __shared__ float red[4][kFinRows][kFinCh];   // V max; K max, K min, |Q| max (equalisation)
  const int D = a.D;
  const int bh = blockIdx.y;
  const int d0 = blockIdx.x * kFinCh;
  const int nkb = (a.Nkv + kBlk - 1) / kBlk;
  const int ch = threadIdx.x % kFinCh;         // channel d0 + ch
  const int rl = threadIdx.x / kFinCh;         // 0 .. 31
  const bool eq = a.eq;
  double total = 0.0;
  float m = 0.0f, kmx = -INFINITY, kmn = INFINITY, qmx = 0.0f;
  for (int b0 = 0; b0 < nkb; b0 += kFinChunk) {
    const int nb = min(kFinChunk, nkb - b0);
    for (int r = rl; r < nb; r += kFinRows) {
      const size_t w = (static_cast<size_t>(bh) * nkb + b0 + r) * D + d0 + ch;
      part[r][ch] = a.ws_ksum[w];
      m = fmaxf(m, a.ws_vmax[w]);
      if (eq) {
        kmx = fmaxf(kmx, a.ws_kmax[w]);
        kmn = fminf(kmn, a.ws_kmin[w]);
      }
    }
    __syncthreads();
    if (threadIdx.x < kFinCh) {
      int r = 0;
      for (; r + 8 <= nb; r += 8) {
        double v[8];
#pragma unroll
        for (int e = 0; e < 8; e++) v[e] = part[r + e][threadIdx.x];
#pragma unroll
        for (int e = 0; e < 8; e++) total = __dadd_rn(total, v[e]);
      }
      for (; r < nb; r++) total = __dadd_rn(total, part[r][threadIdx.x]);
    }
    __syncthreads();
  }
  if (eq) {
    const int nqb = (a.Nq + kBlk - 1) / kBlk;
    for (int r = rl; r < nqb; r += kFinRows)
      qmx = fmaxf(qmx, a.ws_qmax[(static_cast<size_t>(bh) * nqb + r) * D + d0 + ch]);
    red[1][rl][ch] = kmx;
    red[2][rl][ch] = kmn;
    red[3][rl][ch] = qmx;
  }
  red[0][rl][ch] = m;
  __syncthreads();
  if (threadIdx.x < kFinCh) {  // rl = 0, ch = threadIdx.x
    for (int g = 1; g < kFinRows; g++) m = fmaxf(m, red[0][g][threadIdx.x]);
    const int idx = bh * D + d0 + threadIdx.x;
    const float mu = __double2float_rn(__ddiv_rn(total, static_cast<double>(a.Nkv)));
    a.k_mean[idx] = mu;
    a.v_scale[idx] = (m == 0.0f) ? 0.0f : __fdiv_rn(m, 448.0f);
    a.ws_vinv[idx] = (m == 0.0f) ? 0.0f : __fdiv_rn(448.0f, m);
    if (eq) {
      for (int g = 1; g < kFinRows; g++) {
        kmx = fmaxf(kmx, red[1][g][threadIdx.x]);
        kmn = fminf(kmn, red[2][g][threadIdx.x]);
        qmx = fmaxf(qmx, red[3][g][threadIdx.x]);
      }
      const int e = eq_exponent(qmx, kmx, kmn, mu);
      a.ws_eq_up[idx] = __uint_as_float(static_cast<uint32_t>(127 + e) << 23);    // 2^e
      a.ws_eq_down[idx] = __uint_as_float(static_cast<uint32_t>(127 - e) << 23);  // 2^-e
      if (a.eq_exp) a.eq_exp[idx] = static_cast<int8_t>(e);
    }
  }
}

// pass 2.  EQ: the grid also covers the Q blocks, whose codes are taken
// here from Q * 2^e; the smoothed K is multiplied by 2^-e before its codes.
template <int D, bool ROPE, bool EQ>
__global__ void __launch_bounds__(kThreads) k_quant_pass2(QuantArgs a) {
  grid_dep_wait();
  constexpr int kChunksPerRow = D / 8;
  constexpr int CH = kBlk * kChunksPerRow / kThreads;
  __shared__ float red[kThreads / 32];

  const int blk = ROPE ? blockIdx.y : blockIdx.x;  // as in pass 1
  const int bh = ROPE ? blockIdx.x : blockIdx.y;
  const int nkb = (a.Nkv + kBlk - 1) / kBlk;
  const int nkv_pad = nkb * kBlk;
  if constexpr (EQ) {
    const int nqb = (a.Nq + kBlk - 1) / kBlk;
    if (blk < nqb) {  // Q * 2^e: block codes and scale
      const int qvalid = min(kBlk, a.Nq - blk * kBlk);
      const uint4* src = reinterpret_cast<const uint4*>(
          a.q + (static_cast<size_t>(bh) * a.Nq + static_cast<size_t>(blk) * kBlk) * D);
      const float* up = a.ws_eq_up + static_cast<size_t>(bh) * D;
      float x[CH][8];
#pragma unroll
      for (int c = 0; c < CH; c++) {
        const int chunk = c * kThreads + threadIdx.x;
        const int col = (chunk % kChunksPerRow) * 8;
        unpack8(chunk / kChunksPerRow < qvalid ? __ldg(src + chunk) : make_uint4(0, 0, 0, 0), x[c]);
#pragma unroll
        for (int e = 0; e < 8; e++) x[c][e] = __fmul_rn(x[c][e], __ldg(up + col + e));
      }
      quant_block_store<D, CH>(x, qvalid, a.q_i8 + (static_cast<size_t>(bh) * nqb + blk) * kBlk * D,
                               a.q_scale + static_cast<size_t>(bh) * nqb + blk, red);
    }
    if (blk >= nkb) return;  // uniform over the CTA
  }
  const int valid = min(kBlk, a.Nkv - blk * kBlk);
  // The V loads are issued first, together with the K loads, so that the
  // whole 64-token block of K and V is in flight at once.  Chunk c*256 + t
  // (8 channels of one token) belongs to thread t, as for K.
  uint4 vu[CH];
#pragma unroll
  for (int c = 0; c < CH; c++) {
    const int chunk = c * kThreads + threadIdx.x;
    vu[c] = chunk / kChunksPerRow < valid ? __ldg(kv_chunk<D>(a.v, a, bh, blk, chunk))
                                          : make_uint4(0, 0, 0, 0);
  }

  {  // K - mean, block codes and scale
    const float* mu = a.k_mean + static_cast<size_t>(bh) * D;
    float x[CH][8];
    uint4 u[CH];
    float4 rc[ROPE ? CH : 1], rs[ROPE ? CH : 1];  // all loads first, then the math
#pragma unroll
    for (int c = 0; c < CH; c++) {
      const int chunk = c * kThreads + threadIdx.x;
      const int row = chunk / kChunksPerRow;
      u[c] = make_uint4(0, 0, 0, 0);
      if (row < valid) u[c] = __ldg(kv_chunk<D>(a.k, a, bh, blk, chunk));
      if constexpr (ROPE) {
        rc[c] = rs[c] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
        if (row < valid)
          rope_load<D>(a.k_cos, a.k_sin, blk * kBlk + row, (chunk % kChunksPerRow) * 8, rc[c], rs[c]);
      }
    }
#pragma unroll
    for (int c = 0; c < CH; c++) {
      const int col = ((c * kThreads + threadIdx.x) % kChunksPerRow) * 8;
      unpack8(u[c], x[c]);
      if constexpr (ROPE) rope_apply(x[c], rc[c], rs[c]);
#pragma unroll
      for (int e = 0; e < 8; e++) x[c][e] = __fsub_rn(x[c][e], __ldg(mu + col + e));
      if constexpr (EQ) {
        const float* down = a.ws_eq_down + static_cast<size_t>(bh) * D;
#pragma unroll
        for (int e = 0; e < 8; e++) x[c][e] = __fmul_rn(x[c][e], __ldg(down + col + e));
      }
    }
    int8_t* codes = a.k_i8 + (static_cast<size_t>(bh) * nkb + blk) * kBlk * D;
    quant_block_store<D, CH>(x, valid, codes, a.k_scale + static_cast<size_t>(bh) * nkb + blk,
                             red);
  }

  {  // V codes, token-major like K: [BH][Nkv_pad][D] (the attention kernel
     // reads V tiles as MN-major tensor-core operands, so no transpose)
    const float* inv = a.ws_vinv + static_cast<size_t>(bh) * D;
    uint8_t* dst = a.v_f8 + (static_cast<size_t>(bh) * nkv_pad + static_cast<size_t>(blk) * kBlk) * D;
#pragma unroll
    for (int c = 0; c < CH; c++) {
      const int chunk = c * kThreads + threadIdx.x;
      const int row = chunk / kChunksPerRow;
      const int col = (chunk % kChunksPerRow) * 8;
      float x[8];
      unpack8(vu[c], x);
      uint32_t w[2];
#pragma unroll
      for (int h = 0; h < 2; h++) {
        uint32_t b4 = 0;
#pragma unroll
        for (int e = 0; e < 4; e += 2) {
          const int d = col + h * 4 + e;
          const float i0 = __ldg(inv + d), i1 = __ldg(inv + d + 1);
          uint32_t pr = cvt_e4m3x2(__fmul_rn(x[h * 4 + e], i0), __fmul_rn(x[h * 4 + e + 1], i1));
          if (i0 == 0.0f) pr &= 0xFF00u;  // zero channel
          if (i1 == 0.0f) pr &= 0x00FFu;
          b4 |= pr << (8 * e);
        }
        w[h] = row < valid ? b4 : 0u;  // padding tokens are 0
      }
      *reinterpret_cast<uint2*>(dst + static_cast<size_t>(row) * D + col) = make_uint2(w[0], w[1]);
    }
  }
}


}  // namespace

// a launch of `kernel` that may begin before the previous kernel of the
// stream has finished (the kernel waits for it in grid_dep_wait)
template <typename Kernel>
cudaError_t launch_after(Kernel kernel, dim3 grid, cudaStream_t stream, const QuantArgs& a) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, a);
}

cudaError_t launch_quant(const QuantArgs& a, cudaStream_t stream) {
  const int nqb = (a.Nq + kBlk - 1) / kBlk;
  const int nkb = (a.Nkv + kBlk - 1) / kBlk;
  dim3 g1(nqb > nkb ? nqb : nkb, a.BH);
  dim3 g2(nkb, a.BH);
  dim3 gf(a.D / kFinCh, a.BH);
  const bool rope = a.q_cos != nullptr;
  const dim3 r1(a.BH, g1.x), r2(a.BH, g2.x);  // rotary variant: heads fastest
  if (rope && g1.x > 65535) return cudaErrorInvalidConfiguration;
  if (rope && a.eq) return cudaErrorInvalidValue;  // not offered together
  cudaError_t e = cudaSuccess;
  if (a.D == 128) {
    if (rope) k_quant_pass1<128, true, false><<<r1, kThreads, 0, stream>>>(a);
    else if (a.eq) k_quant_pass1<128, false, true><<<g1, kThreads, 0, stream>>>(a);
    else k_quant_pass1<128, false, false><<<g1, kThreads, 0, stream>>>(a);
    e = cudaGetLastError();
    if (e == cudaSuccess) e = launch_after(k_quant_finalize, gf, stream, a);
    if (e == cudaSuccess)
      e = rope   ? launch_after(k_quant_pass2<128, true, false>, r2, stream, a)
          : a.eq ? launch_after(k_quant_pass2<128, false, true>, g1, stream, a)
                 : launch_after(k_quant_pass2<128, false, false>, g2, stream, a);
  } else {
    if (rope) k_quant_pass1<64, true, false><<<r1, kThreads, 0, stream>>>(a);
    else if (a.eq) k_quant_pass1<64, false, true><<<g1, kThreads, 0, stream>>>(a);
    else k_quant_pass1<64, false, false><<<g1, kThreads, 0, stream>>>(a);
    e = cudaGetLastError();
    if (e == cudaSuccess) e = launch_after(k_quant_finalize, gf, stream, a);
    if (e == cudaSuccess)
      e = rope   ? launch_after(k_quant_pass2<64, true, false>, r2, stream, a)
          : a.eq ? launch_after(k_quant_pass2<64, false, true>, g1, stream, a)
                 : launch_after(k_quant_pass2<64, false, false>, g2, stream, a);
  }
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace sage
