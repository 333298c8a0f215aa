// attn.cu -- sage_attn_fwd: fused SageAttention-style quantized attention
// for sm_100a.
//
// The method (low-bit quantized attention that keeps FlashAttention's
// streaming structure but runs its matmuls on 8-bit tensor cores; "Vidu S1"
// digest section "Infra", TurboDiffusion notes): Q K^T on INT8 tensor cores
// from per-block INT8 codes, an fp32 online softmax in the log2 domain, P
// quantized to FP8 e4m3 with a fixed 2^8 scale and P V on FP8 tensor cores
// with fp32 accumulation.
//
// One CTA owns 128 query rows of one (batch, head) and streams the visible
// KV tiles of 128 keys.  Warp roles (256 threads, two CTAs per SM; launched
// at 128 registers per thread, then warpgroup 0 drops to 32 and warpgroup 1
// rises to 224: 128 x 32 + 128 x 224 = 256 x 128):
//   warp 0      TMA producer: the Q tile once, then K and V^T tiles through
//               a two-stage shared-memory ring (128-byte swizzle).
//   warp 1      allocates 256 TMEM columns (S: 128 x 128 int32, O: 128 x D
//               fp32) and one elected thread issues every tcgen05.mma:
//               S = Q K^T (kind::i8) for tile k+1 while the softmax warps
//               work on tile k, then O (+)= P V^T (kind::f8f6f4).
//   warps 2-3   idle.
//   warps 4-7   softmax: thread t of the warpgroup owns query row t (TMEM
//               lane t).  The S columns are seeded with the integer bit
//               pattern of 1.5 * 2^23 before every Q K^T, so the int32 MMA
//               leaves 0x4B400000 + S, which read as an fp32 is exactly
//               12582912 + S: no int-to-float conversion per score.  Per
//               tile: load the score row, re-seed the columns, take the
//               masked max per 64-key scale group with 3-input maxima,
//               update the running max, y = exp2(fma(S, c, 8 - m)) (P scaled
//               by 2^8) with packed fp32x2 arithmetic, row sum, e4m3(y) into
//               the swizzled shared-memory P tile, and rescale the O row in
//               TMEM when the max moved.  Epilogue: O * v_scale / l -> bf16
//               (and optional fp32 O, lse).
// Every wait is bounded (see WaitCtx); on a timeout the CTA drains its
// in-flight copies and MMAs, frees TMEM and returns.
#include "attn.cuh"
#include "sm100.cuh"

#include <cfloat>
#include <climits>

namespace sage {

namespace {

constexpr int BM = kAttnBM;
constexpr int BN = kAttnBN;
constexpr int NK = 3;              // K stages; stage k%NK also holds P of tile k
constexpr int NV = 2;              // V stages
constexpr int kThreads = 256;      // 8 warps: warpgroup 0 = roles, 1 = softmax
constexpr int kLaunchRegs = 128;   // registers per thread at launch (2 CTAs per SM)
constexpr int kRegsRoles = 32;     // registers per thread of warpgroup 0
constexpr int kRegsSoftmax = 224;  // registers per thread of warpgroup 1
static_assert(128 * kRegsRoles + 128 * kRegsSoftmax == kThreads * kLaunchRegs,
              "register shares must add up to the launch allocation");
constexpr int kTmemCols = 256;
constexpr uint32_t kFull = 0xffffffffu;
// Seed of the S accumulator: the int32 bit pattern of 1.5 * 2^23.  For
// |S| < 2^22 the word 0x4B400000 + S is the fp32 value 12582912 + S.
constexpr uint32_t kBiasBits = 0x4B400000u;
constexpr float kBias = 12582912.0f;

// wait-site codes for the status word (kernel 1 = attention)
enum : int {
  kSiteProdKEmpty = 0x10101, kSiteProdVEmpty, kSiteMmaQ, kSiteMmaK, kSiteMmaSFree,
  kSiteMmaV, kSiteMmaP, kSiteSmS, kSiteSmO, kSiteSmEpi, kSiteDrain
};

// Bytes of one K stage: the int8 K tile [128 keys][D], and after Q K^T of
// that tile has completed, the e4m3 P tile [128 rows][128 keys] (128-byte
// swizzle) that P V reads.
template <int D>
constexpr int kStageBytes = (BN * D > BM * BN) ? BN * D : BM * BN;

template <int D>
struct alignas(1024) Smem {
  uint8_t q[BM * D];              // int8 Q tile [128 rows][D]
  uint8_t k[NK][kStageBytes<D>];  // K tile, then P tile, of tile k in stage k % NK
  uint8_t v[NV][D * BN];          // e4m3 V^T tiles [D][128 keys]
  uint64_t q_full;
  uint64_t k_full[NK], k_empty[NK];
  uint64_t v_full[NV], v_empty[NV];
  uint64_t s_full, s_free, p_full, o_ready, drain;
  uint32_t tmem_base;
  int abort;
};

__host__ __device__ inline size_t smem_bytes_for(int D) {
  return (D == 128 ? sizeof(Smem<128>) : sizeof(Smem<64>)) + 1024;  // + alignment slack
}

// A wait taken by all 32 threads of a warp that reports success only if it
// succeeded for every lane, so that the warp never splits before the
// warp-collective tcgen05.ld / tcgen05.st that follow.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, const WaitCtx& w,
                                          int site) {
  return __all_sync(kFull, mbar_wait(bar, parity, w, site));
}

// First key index that query row i (global row) may NOT see.
__device__ __forceinline__ int row_limit(int i, const AttnParams& p) {
  const int g = i + (p.Nkv - p.Nq);
  int lim = p.Nkv;
  if (p.mask == 1) lim = g + 1;
  else if (p.mask == 2) lim = (g / p.mask_block + 1) * p.mask_block;
  return lim < p.Nkv ? lim : p.Nkv;
}

// Bounded wait that ignores the abort flag: used while draining copies and
// MMAs that were already issued, so that the CTA never frees shared memory
// or TMEM under an operation in flight.
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity, const WaitCtx& w) {
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > w.budget) {
      record_timeout(w.status, kSiteDrain);
      return;
    }
  }
}

template <int D, bool DUMP>
__device__ __forceinline__ void producer(Smem<D>& s, const AttnMaps& maps, int bh, int qt,
                                         int kt0, int nk, const WaitCtx& w) {
  tma_prefetch_desc(&maps.q);
  tma_prefetch_desc(&maps.k);
  tma_prefetch_desc(&maps.v);
  mbar_arrive_expect_tx(&s.q_full, BM * D);
  tma_load_3d(s.q, &maps.q, &s.q_full, 0, qt * BM, bh);
  int k_issued = 0, v_issued = 0;
  for (int it = 0; it < nk; it++) {
    const int kt = kt0 + it;
    {  // K stage it % NK is free once P V of tile it - NK has read its P
      const int st = it % NK;
      if (it >= NK && !mbar_wait(&s.k_empty[st], ((it / NK) & 1) ^ 1, w, kSiteProdKEmpty)) break;
      mbar_arrive_expect_tx(&s.k_full[st], BN * D);
      tma_load_3d(s.k[st], &maps.k, &s.k_full[st], 0, kt * BN, bh);
      k_issued++;
    }
    if (DUMP) continue;
    {
      const int st = it % NV;
      if (it >= NV && !mbar_wait(&s.v_empty[st], ((it / NV) & 1) ^ 1, w, kSiteProdVEmpty)) break;
      mbar_arrive_expect_tx(&s.v_full[st], D * BN);
      tma_load_3d(s.v[st], &maps.v, &s.v_full[st], kt * BN, 0, bh);
      v_issued++;
    }
  }
  // Drain: every issued load must have landed before the CTA may exit.  A
  // load is only issued once the previous load of its stage was consumed, so
  // only the last NK (NV) loads can still be in flight.
  drain_wait(&s.q_full, 0, w);
  for (int it = (k_issued > NK ? k_issued - NK : 0); it < k_issued; it++)
    drain_wait(&s.k_full[it % NK], (it / NK) & 1, w);
  for (int it = (v_issued > NV ? v_issued - NV : 0); it < v_issued; it++)
    drain_wait(&s.v_full[it % NV], (it / NV) & 1, w);
}

template <int D, bool DUMP>
__device__ __forceinline__ void mma_issuer(Smem<D>& s, uint32_t tmem_S, uint32_t tmem_O, int nk,
                                           const WaitCtx& w) {
  constexpr uint32_t idesc_qk = idesc_i8_s32(BM, BN);
  constexpr uint32_t idesc_pv = idesc_e4m3_f32(BM, D);
  const uint32_t q_addr = smem_u32(s.q);
  bool ok = mbar_wait(&s.q_full, 0, w, kSiteMmaQ);
  for (int it = 0; ok && it <= nk; it++) {
    if (it < nk) {  // S = Q K^T for tile it
      const int st = it % NK;
      if (!mbar_wait(&s.k_full[st], (it / NK) & 1, w, kSiteMmaK)) break;
      // the softmax warps have read S of the previous tile and re-seeded it
      if (!mbar_wait(&s.s_free, it & 1, w, kSiteMmaSFree)) break;
      tc_fence_after();
      const uint32_t k_addr = smem_u32(s.k[st]);
#pragma unroll
      for (int kk = 0; kk < D / 32; kk++)
        mma_i8_ss(tmem_S, smem_desc_kmajor(q_addr + kk * 32, D),
                  smem_desc_kmajor(k_addr + kk * 32, D), idesc_qk, 1u);
      mma_commit(&s.s_full);
    }
    if (!DUMP && it > 0) {  // O (+)= P V^T for tile it - 1; P sits in its K stage
      const int j = it - 1;
      const int stv = j % NV;
      if (!mbar_wait(&s.v_full[stv], (j / NV) & 1, w, kSiteMmaV)) break;
      if (!mbar_wait(&s.p_full, j & 1, w, kSiteMmaP)) break;
      tc_fence_after();
      const uint32_t p_addr = smem_u32(s.k[j % NK]);
      const uint32_t v_addr = smem_u32(s.v[stv]);
#pragma unroll
      for (int kk = 0; kk < BN / 32; kk++)
        mma_f8_ss(tmem_O, smem_desc_kmajor(p_addr + kk * 32, BN),
                  smem_desc_kmajor(v_addr + kk * 32, BN), idesc_pv, (j > 0 || kk > 0));
      mma_commit(&s.k_empty[j % NK]);
      mma_commit(&s.v_empty[stv]);
      mma_commit(&s.o_ready);
    }
    if (DUMP && it < nk) mma_commit(&s.k_empty[it % NK]);
  }
  // Drain: all MMAs issued by this thread complete before TMEM is freed.
  mma_commit(&s.drain);
  drain_wait(&s.drain, 0, w);
}

// Seed the warp's 32 rows of the S columns with kBiasBits (asynchronous
// TMEM store; see release_scores).
__device__ __forceinline__ void seed_scores(uint32_t tS) { tmem_fill128_nowait(tS, kBiasBits); }

// Wait for the seed to land and tell the MMA issuer that S may be written.
__device__ __forceinline__ void release_scores(uint64_t* s_free, int lane) {
  tmem_wait_st();
  tc_fence_before();
  __syncwarp();
  if (lane == 0) mbar_arrive(s_free);
}

// Max of 64 biased scores (all > 0), 3-input maxima in four chains.
__device__ __forceinline__ float max64(const float* v) {
  float a = fmax3(v[0], v[1], v[2]), b = fmax3(v[3], v[4], v[5]);
  float c = fmax3(v[6], v[7], v[8]), d = fmax3(v[9], v[10], v[11]);
#pragma unroll
  for (int j = 12; j < 60; j += 8) {
    a = fmax3(a, v[j], v[j + 1]);
    b = fmax3(b, v[j + 2], v[j + 3]);
    c = fmax3(c, v[j + 4], v[j + 5]);
    d = fmax3(d, v[j + 6], v[j + 7]);
  }
  a = fmax3(a, v[60], v[61]);
  b = fmax3(b, v[62], v[63]);
  return fmax3(a, b, fmaxf(c, d));
}

// Softmax / correction / epilogue for one query row per thread.
template <int D>
__device__ __forceinline__ void softmax_rows(Smem<D>& s, const AttnParams& p, uint32_t tmem_S,
                                             uint32_t tmem_O, int bh, int qt, int nk,
                                             const WaitCtx& w) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int quad = warp & 3;               // TMEM lane quadrant of this warp
  const int r = quad * 32 + lane;          // row within the tile
  const int i = qt * BM + r;               // query row
  const bool valid = i < p.Nq;
  const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
  const uint32_t tS = tmem_S + lane_off, tO = tmem_O + lane_off;
  const int lim = valid ? row_limit(i, p) : 0;
  const float sqC = valid ? __fmul_rn(__ldg(p.q_scale + static_cast<size_t>(bh) * p.nq_blocks + i / 64), p.c0)
                          : 0.0f;
  const float* ksc = p.k_scale + static_cast<size_t>(bh) * p.nkv_blocks;

  seed_scores(tS);  // S seed for the first tile
  release_scores(&s.s_free, lane);

  // K scales of the tile's two 64-key groups, loaded one tile ahead
  float skn0 = __ldg(ksc), skn1 = p.nkv_blocks > 1 ? __ldg(ksc + 1) : 0.0f;
  float m = -INFINITY, l = 0.0f;
  bool ok = true;
  for (int it = 0; it < nk; it++) {
    const int j0 = it * BN;
    const float c0 = __fmul_rn(sqC, skn0), c1 = __fmul_rn(sqC, skn1);
    {
      const int g0 = 2 * it + 2, g1 = 2 * it + 3;
      skn0 = g0 < p.nkv_blocks ? __ldg(ksc + g0) : 0.0f;
      skn1 = g1 < p.nkv_blocks ? __ldg(ksc + g1) : 0.0f;
    }
    if (!warp_wait(&s.s_full, it & 1, w, kSiteSmS)) { ok = false; break; }
    tc_fence_after();
    float sv[128];  // 12582912 + S, exact
    tmem_ld128(tS, *reinterpret_cast<uint32_t(*)[128]>(&sv[0]));
    seed_scores(tS);  // S seed for the next tile; released after the max

    const int nvis = min(max(lim - j0, 0), BN);  // visible keys of this tile
    const bool full = __all_sync(kFull, nvis == BN);
    if (!full) {
      // masked keys: 0 is below every seeded score, and their p is forced to 0
#pragma unroll
      for (int j = 0; j < 128; j++) sv[j] = j < nvis ? sv[j] : 0.0f;
    }
    // max_j fp32(S_j * c) = fp32(max_j S_j * c) for c >= 0 (rounding is monotone)
    const float mb0 = max64(sv), mb1 = max64(sv + 64);
    const float t0 = mb0 > 0.0f ? __fmul_rn(__fsub_rn(mb0, kBias), c0) : -INFINITY;
    const float t1 = mb1 > 0.0f ? __fmul_rn(__fsub_rn(mb1, kBias), c1) : -INFINITY;
    const float m_new = fmax3(m, t0, t1);
    const float alpha = (m == -INFINITY) ? 0.0f
                        : (m == m_new)   ? 1.0f
                                         : ex2_approx(__fsub_rn(m, m_new));
    const float nm8 = __fsub_rn(8.0f, m_new);  // P scale 2^8 folded into the exponent
    release_scores(&s.s_free, lane);

    // P of this tile goes into its K stage (Q K^T of the tile has completed)
    uint8_t* prow = s.k[it % NK] + r * BN;

    const float2 nb2 = make_float2(-kBias, -kBias);
    const float2 nm2 = make_float2(nm8, nm8);
    float2 rs = make_float2(0.0f, 0.0f);
#pragma unroll
    for (int c = 0; c < 8; c++) {  // 16-key chunks
      const float2 cc = c < 4 ? make_float2(c0, c0) : make_float2(c1, c1);
      uint32_t pk[4];
#pragma unroll
      for (int q4 = 0; q4 < 4; q4++) {
        const int j = c * 16 + q4 * 4;
        float2 xa = __ffma2_rn(__fadd2_rn(make_float2(sv[j], sv[j + 1]), nb2), cc, nm2);
        float2 xb = __ffma2_rn(__fadd2_rn(make_float2(sv[j + 2], sv[j + 3]), nb2), cc, nm2);
        if (!full) {
          xa.x = j < nvis ? xa.x : -INFINITY;
          xa.y = j + 1 < nvis ? xa.y : -INFINITY;
          xb.x = j + 2 < nvis ? xb.x : -INFINITY;
          xb.y = j + 3 < nvis ? xb.y : -INFINITY;
        }
        const float2 ya = make_float2(ex2_approx(xa.x), ex2_approx(xa.y));
        const float2 yb = make_float2(ex2_approx(xb.x), ex2_approx(xb.y));
        rs = __fadd2_rn(rs, ya);
        rs = __fadd2_rn(rs, yb);
        pk[q4] = __byte_perm(cvt_e4m3x2(ya.x, ya.y), cvt_e4m3x2(yb.x, yb.y), 0x5410);
      }
      *reinterpret_cast<uint4*>(prow + ((c ^ (r & 7)) << 4)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
    }
    fence_proxy_async_smem();

    // P V of the previous tile must be complete before O may be rescaled (and
    // before the next P V is issued, which waits for this warp's arrival)
    if (it > 0 && !warp_wait(&s.o_ready, (it - 1) & 1, w, kSiteSmO)) { ok = false; break; }
    tc_fence_after();
    // rescale the O row when the running max moved (never before the first P V)
    if (it > 0 && __any_sync(kFull, alpha != 1.0f)) {
      if constexpr (D == 128) {
        uint32_t o[128];
        tmem_ld128(tO, o);
#pragma unroll
        for (int e = 0; e < 128; e++) o[e] = __float_as_uint(__fmul_rn(__uint_as_float(o[e]), alpha));
        tmem_st128_nowait(tO, o);
        tmem_wait_st();
      } else {
        uint32_t o[64];
        tmem_ld64(tO, o);
#pragma unroll
        for (int e = 0; e < 64; e++) o[e] = __float_as_uint(__fmul_rn(__uint_as_float(o[e]), alpha));
        tmem_st32(tO, *reinterpret_cast<uint32_t(*)[32]>(&o[0]));
        tmem_st32(tO + 32, *reinterpret_cast<uint32_t(*)[32]>(&o[32]));
      }
    }
    l = __fadd_rn(__fmul_rn(l, alpha), __fadd_rn(rs.x, rs.y));
    m = m_new;
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&s.p_full);
  }

  if (!ok || nk == 0) return;
  if (!warp_wait(&s.o_ready, (nk - 1) & 1, w, kSiteSmEpi)) return;
  tc_fence_after();
  const float inv = __frcp_rn(l);  // l is in units of 2^8 p
  const float* vsc = p.v_scale + static_cast<size_t>(bh) * D;
  const size_t orow = (static_cast<size_t>(bh) * p.Nq + (valid ? i : 0)) * D;
#pragma unroll 1
  for (int c = 0; c < D; c += 32) {
    uint32_t o[32];
    tmem_ld32(tO + c, o);
    if (!valid) continue;
    float f[32];
#pragma unroll
    for (int e = 0; e < 32; e++) f[e] = __uint_as_float(o[e]) * (__ldg(vsc + c + e) * inv);
    uint32_t b[16];
#pragma unroll
    for (int e = 0; e < 16; e++) {
      __nv_bfloat162 h = __floats2bfloat162_rn(f[2 * e], f[2 * e + 1]);
      b[e] = *reinterpret_cast<uint32_t*>(&h);
    }
    uint4* dst = reinterpret_cast<uint4*>(p.o + orow + c);
#pragma unroll
    for (int e = 0; e < 4; e++) dst[e] = make_uint4(b[4 * e], b[4 * e + 1], b[4 * e + 2], b[4 * e + 3]);
    if (p.o_f32) {
      float4* d32 = reinterpret_cast<float4*>(p.o_f32 + orow + c);
#pragma unroll
      for (int e = 0; e < 8; e++) d32[e] = make_float4(f[4 * e], f[4 * e + 1], f[4 * e + 2], f[4 * e + 3]);
    }
  }
  if (valid && p.lse)
    p.lse[static_cast<size_t>(bh) * p.Nq + i] = (m + log2f(l) - 8.0f) * 0.69314718055994531f;
}

// Score dump (debug): copy the int32 S tile from TMEM to global memory (the
// accumulator seed removed).
template <int D>
__device__ __forceinline__ void dump_rows(Smem<D>& s, const AttnParams& p, uint32_t tmem_S,
                                          const WaitCtx& w) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int quad = warp & 3;
  const int r = quad * 32 + lane;
  const uint32_t tS = tmem_S + (static_cast<uint32_t>(quad * 32) << 16);
  seed_scores(tS);
  release_scores(&s.s_free, lane);
  if (!warp_wait(&s.s_full, 0, w, kSiteSmS)) return;
  tc_fence_after();
#pragma unroll 1
  for (int c = 0; c < BN; c += 32) {
    uint32_t v[32];
    tmem_ld32(tS + c, v);
#pragma unroll
    for (int e = 0; e < 32; e++) v[e] -= kBiasBits;
    uint4* dst = reinterpret_cast<uint4*>(p.dbg_out + static_cast<size_t>(r) * BN + c);
#pragma unroll
    for (int e = 0; e < 8; e++) dst[e] = make_uint4(v[4 * e], v[4 * e + 1], v[4 * e + 2], v[4 * e + 3]);
  }
}

template <int D, bool DUMP>
__global__ void __launch_bounds__(kThreads, 2)
    k_attn(const __grid_constant__ AttnMaps maps, const AttnParams p) {
  extern __shared__ uint8_t smem_raw[];
  Smem<D>& s = *reinterpret_cast<Smem<D>*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qt = DUMP ? p.dbg_qt : static_cast<int>(blockIdx.x);
  const int bh = DUMP ? p.dbg_bh : static_cast<int>(blockIdx.y);

  // KV tiles this CTA visits: those holding a key visible to its last valid
  // row (the masks' limits grow with the row index).
  int kt0 = 0, nk;
  if (DUMP) {
    kt0 = p.dbg_kt;
    nk = 1;
  } else {
    const int last = min(p.Nq - 1, qt * BM + BM - 1);
    nk = (row_limit(last, p) + BN - 1) / BN;
  }

  if (threadIdx.x == 0) {
    mbar_init(&s.q_full, 1);
    for (int i = 0; i < NK; i++) {
      mbar_init(&s.k_full[i], 1);
      mbar_init(&s.k_empty[i], 1);
    }
    for (int i = 0; i < NV; i++) {
      mbar_init(&s.v_full[i], 1);
      mbar_init(&s.v_empty[i], 1);
    }
    mbar_init(&s.s_full, 1);
    mbar_init(&s.s_free, 4);
    mbar_init(&s.p_full, 4);
    mbar_init(&s.o_ready, 1);
    mbar_init(&s.drain, 1);
    s.abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&s.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s.tmem_base;
  const uint32_t tmem_S = tmem;        // columns [0, 128): int32 scores
  const uint32_t tmem_O = tmem + 128;  // columns [128, 128 + D): fp32 output
  const WaitCtx w{p.budget, p.status, &s.abort};

  if (warp < 4) {
    regs_dec<kRegsRoles>();
    if (warp == 0) {
      if (lane == 0) producer<D, DUMP>(s, maps, bh, qt, kt0, nk, w);
    } else if (warp == 1) {
      if (lane == 0) mma_issuer<D, DUMP>(s, tmem_S, tmem_O, nk, w);
    }
  } else {
    regs_inc<kRegsSoftmax>();
    if (DUMP) dump_rows<D>(s, p, tmem_S, w);
    else softmax_rows<D>(s, p, tmem_S, tmem_O, bh, qt, nk, w);
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace

size_t attn_smem_bytes(int D) { return smem_bytes_for(D); }

// One-time per-device setup: dynamic shared memory size, and a check that
// the compiled kernels were built with exactly kLaunchRegs registers per
// thread.  The warpgroups' setmaxnreg shares add up to that launch
// allocation; a different allocation could leave the increase waiting, so
// such a build is refused here instead of launched.
template <int D, bool DUMP>
cudaError_t prepare_one() {
  cudaError_t e = cudaFuncSetAttribute(k_attn<D, DUMP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem_bytes_for(D)));
  if (e != cudaSuccess) return e;
  cudaFuncAttributes attr;
  e = cudaFuncGetAttributes(&attr, k_attn<D, DUMP>);
  if (e != cudaSuccess) return e;
  return attr.numRegs == kLaunchRegs ? cudaSuccess : cudaErrorInvalidDeviceFunction;
}

cudaError_t attn_prepare(int D) {
  cudaError_t e;
  if (D == 128) {
    e = prepare_one<128, false>();
    if (e == cudaSuccess) e = prepare_one<128, true>();
  } else {
    e = prepare_one<64, false>();
    if (e == cudaSuccess) e = prepare_one<64, true>();
  }
  return e;
}

cudaError_t launch_attn(const AttnMaps& maps, const AttnParams& p, cudaStream_t stream) {
  dim3 grid((p.Nq + BM - 1) / BM, p.BH);
  if (p.D == 128)
    k_attn<128, false><<<grid, kThreads, smem_bytes_for(128), stream>>>(maps, p);
  else
    k_attn<64, false><<<grid, kThreads, smem_bytes_for(64), stream>>>(maps, p);
  return cudaGetLastError();
}

cudaError_t launch_attn_dump(const AttnMaps& maps, const AttnParams& p, cudaStream_t stream) {
  if (p.D == 128)
    k_attn<128, true><<<1, kThreads, smem_bytes_for(128), stream>>>(maps, p);
  else
    k_attn<64, true><<<1, kThreads, smem_bytes_for(64), stream>>>(maps, p);
  return cudaGetLastError();
}

}  // namespace sage
