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
// One CTA per SM owns two 128-row query tiles (A and B) of one (batch, head)
// and streams the visible KV tiles of 128 keys.  512 threads, launched at
// 128 registers each and re-split per warpgroup with setmaxnreg (the shares
// add up to at most the launch allocation):
//   WG0  (56 regs)  warp 0: TMA producer of both Q tiles (once) and of K
//                   through a 4-stage shared-memory ring; warp 2: producer of
//                   V^T through its own 4-stage ring (separate threads, so a
//                   full V ring never holds back K loads).  Tiles further
//                   ahead are prefetched into L2, since the CTAs of a head
//                   run in step and would otherwise all wait for the same
//                   DRAM fetch.
//                   warp 1: owns all 512 TMEM columns (S_A, S_B: 128 x 128
//                   int32; O_A, O_B: 128 x D fp32); one elected thread
//                   issues every tcgen05.mma: S_X = Q_X K^T (kind::i8),
//                   O_X (+)= P_X V^T (kind::f8f6f4).
//   WG1, WG2 (184)  softmax of tile A and tile B: thread t owns query row t
//                   (TMEM lane t).  The S columns are seeded with the bit
//                   pattern of 1.5 * 2^23 before every Q K^T, so the int32
//                   accumulator reads as the fp32 value 12582912 + S: no
//                   conversion per score.  Per KV tile: load S, re-seed,
//                   masked max per 64-key scale group (3-input maxima),
//                   running max, rescale factor alpha to the correction
//                   warps, then -- taking turns with the other softmax
//                   warpgroup so that one warpgroup's exp2-heavy phase runs
//                   while the other does its loads and maxima --
//                   y = exp2(fma(S, c, 8 - m)) (P scale 2^8) with packed
//                   fp32x2 arithmetic, row sum, e4m3(y) into the
//                   128-byte-swizzled shared-memory P tile of its query tile.
//   WG3  (80 regs)  correction and epilogue: rescales O_X in TMEM by alpha
//                   when a row's max moved (between P V of consecutive
//                   tiles), and finally writes O * v_scale / l as bf16 (plus
//                   optional fp32 O and lse).
// Every wait is bounded (see WaitCtx); on a timeout the CTA drains its
// in-flight copies and MMAs, frees TMEM and returns.  Every mbarrier is
// waited by one role only and can never run two phases ahead of its waiter
// (double-buffered signals use one barrier per buffer).
#include "attn.cuh"
#include "sm100.cuh"

#include <cfloat>
#include <climits>

namespace sage {

namespace {

constexpr int BM = kAttnBM;        // rows per query tile
constexpr int BN = kAttnBN;        // keys per KV tile
constexpr int NQT = 2;             // query tiles per CTA
constexpr int NK = 4;              // K stages
constexpr int NV = 4;              // V stages
constexpr int kPrefetch = 6;       // KV tiles prefetched into L2 ahead of the loads
constexpr int kThreads = 512;      // 16 warps = 4 warpgroups
constexpr int kLaunchRegs = 128;   // registers per thread at launch (1 CTA per SM)
constexpr int kRegsRoles = 56;     // WG0
constexpr int kRegsSoftmax = 184;  // WG1, WG2
constexpr int kRegsCorr = 80;      // WG3
static_assert(128 * kRegsRoles + 256 * kRegsSoftmax + 128 * kRegsCorr <= kThreads * kLaunchRegs,
              "register shares must fit in the launch allocation");
constexpr int kTmemCols = 512;
constexpr uint32_t kFull = 0xffffffffu;
// Seed of the S accumulator: the int32 bit pattern of 1.5 * 2^23.  For
// |S| < 2^22 the word 0x4B400000 + S is the fp32 value 12582912 + S.
constexpr uint32_t kBiasBits = 0x4B400000u;
constexpr float kBias = 12582912.0f;

// wait-site codes for the status word (kernel 1 = attention)
enum : int {
  kSiteProdKEmpty = 0x10101, kSiteProdVEmpty, kSiteMmaQ, kSiteMmaK, kSiteMmaSFree,
  kSiteMmaV, kSiteMmaP, kSiteMmaCorr, kSiteSmS, kSiteSmPFree, kSiteSmTurn, kSiteCorrAlpha,
  kSiteCorrO, kSiteEpiO, kSiteEpiFin, kSiteDrain
};

template <int D>
struct alignas(1024) Smem {
  uint8_t q[NQT][BM * D];        // int8 Q tiles [128 rows][D]
  uint8_t k[NK][BN * D];         // int8 K tiles [128 keys][D]
  uint8_t v[NV][D * BN];         // e4m3 V^T tiles [D][128 keys]
  uint8_t p[NQT][BM * BN];       // e4m3 P tiles [128 rows][128 keys], 128-byte swizzle
  float alpha[NQT][2][BM];       // rescale factor per row and tile parity
  float fin_m[NQT][BM];          // final running max per row
  float fin_l[NQT][BM];          // final row sum (units of 2^8 p)
  uint64_t q_full;
  uint64_t k_full[NK], k_empty[NK];
  uint64_t v_full[NV], v_empty[NV];
  uint64_t s_full[NQT], s_free[NQT];
  uint64_t p_full[NQT], p_free[NQT];
  uint64_t alpha_full[NQT][2], corr_done[NQT], o_done[NQT];
  uint64_t turn[NQT], fin_ready[NQT];
  uint64_t drain;
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

// Warp-level arrival: the warp's prior work is ordered before lane 0 arrives.
__device__ __forceinline__ void warp_arrive(uint64_t* bar, int lane) {
  __syncwarp();
  if (lane == 0) mbar_arrive(bar);
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
  while (!mbar_try_wait_sleep(bar, parity, kSleepHintNs)) {
    if (clock64() - t0 > w.budget) {
      record_timeout(w.status, kSiteDrain);
      return;
    }
  }
}

// ------------------------------------------------------------------ producer

// K producer (and both Q tiles) when load_k, else the V producer.
template <int D, bool DUMP>
__device__ __forceinline__ void producer(Smem<D>& s, const AttnMaps& maps, int bh, int q0,
                                         int kt0, int nk, bool load_k, const WaitCtx& w) {
  constexpr int nqt = DUMP ? 1 : NQT;
  int issued = 0;
  if (load_k) {
    tma_prefetch_desc(&maps.q);
    tma_prefetch_desc(&maps.k);
    mbar_arrive_expect_tx(&s.q_full, nqt * BM * D);
    for (int x = 0; x < nqt; x++) tma_load_3d(s.q[x], &maps.q, &s.q_full, 0, q0 + x * BM, bh);
    if (!DUMP)
      for (int it = 0; it < kPrefetch && it < nk; it++)
        tma_prefetch_l2_3d(&maps.k, 0, (kt0 + it) * BN, bh);
    for (int it = 0; it < nk; it++) {
      const int kt = kt0 + it, st = it % NK;
      if (!DUMP && it + kPrefetch < nk) tma_prefetch_l2_3d(&maps.k, 0, (kt + kPrefetch) * BN, bh);
      if (it >= NK && !mbar_wait(&s.k_empty[st], ((it / NK) & 1) ^ 1, w, kSiteProdKEmpty)) break;
      mbar_arrive_expect_tx(&s.k_full[st], BN * D);
      tma_load_3d(s.k[st], &maps.k, &s.k_full[st], 0, kt * BN, bh);
      issued++;
    }
  } else {
    tma_prefetch_desc(&maps.v);
    for (int it = 0; it < kPrefetch && it < nk; it++)
      tma_prefetch_l2_3d(&maps.v, (kt0 + it) * BN, 0, bh);
    for (int it = 0; it < nk; it++) {
      const int kt = kt0 + it, st = it % NV;
      if (it + kPrefetch < nk) tma_prefetch_l2_3d(&maps.v, (kt + kPrefetch) * BN, 0, bh);
      if (it >= NV && !mbar_wait(&s.v_empty[st], ((it / NV) & 1) ^ 1, w, kSiteProdVEmpty)) break;
      mbar_arrive_expect_tx(&s.v_full[st], D * BN);
      tma_load_3d(s.v[st], &maps.v, &s.v_full[st], kt * BN, 0, bh);
      issued++;
    }
  }
  // Drain: every issued load must have landed before the CTA may exit.  A
  // load is only issued once the previous load of its stage was consumed, so
  // only the last NK (NV) loads can still be in flight.
  const int ns = load_k ? NK : NV;
  if (load_k) drain_wait(&s.q_full, 0, w);
  for (int it = (issued > ns ? issued - ns : 0); it < issued; it++)
    drain_wait(load_k ? &s.k_full[it % NK] : &s.v_full[it % NV], (it / ns) & 1, w);
}

// ------------------------------------------------------------------ MMA issuer

template <int D, bool DUMP>
__device__ __forceinline__ void mma_issuer(Smem<D>& s, uint32_t tmem, int nk, const WaitCtx& w) {
  constexpr uint32_t idesc_qk = idesc_i8_s32(BM, BN);
  constexpr uint32_t idesc_pv = idesc_e4m3_f32(BM, D);
  constexpr int nqt = DUMP ? 1 : NQT;
  bool ok = mbar_wait(&s.q_full, 0, w, kSiteMmaQ);
  for (int it = 0; ok && it <= nk; it++) {
    if (it < nk) {  // S_X = Q_X K^T for tile it
      const int st = it % NK;
      if (!mbar_wait(&s.k_full[st], (it / NK) & 1, w, kSiteMmaK)) break;
      const uint32_t k_addr = smem_u32(s.k[st]);
      for (int x = 0; x < nqt; x++) {
        // softmax X has read S_X of the previous tile and re-seeded it
        if (!mbar_wait(&s.s_free[x], it & 1, w, kSiteMmaSFree)) { ok = false; break; }
        tc_fence_after();
        const uint32_t q_addr = smem_u32(s.q[x]);
#pragma unroll
        for (int kk = 0; kk < D / 32; kk++)
          mma_i8_ss(tmem + x * BN, smem_desc_kmajor(q_addr + kk * 32, D),
                    smem_desc_kmajor(k_addr + kk * 32, D), idesc_qk, 1u);
        mma_commit(&s.s_full[x]);
      }
      if (!ok) break;
      mma_commit(&s.k_empty[st]);
    }
    if (!DUMP && it > 0) {  // O_X (+)= P_X V^T for tile it - 1
      const int j = it - 1;
      const int stv = j % NV;
      if (!mbar_wait(&s.v_full[stv], (j / NV) & 1, w, kSiteMmaV)) break;
      const uint32_t v_addr = smem_u32(s.v[stv]);
      for (int x = 0; x < NQT; x++) {
        if (!mbar_wait(&s.p_full[x], j & 1, w, kSiteMmaP) ||
            !mbar_wait(&s.corr_done[x], j & 1, w, kSiteMmaCorr)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t p_addr = smem_u32(s.p[x]);
#pragma unroll
        for (int kk = 0; kk < BN / 32; kk++)
          mma_f8_ss(tmem + 2 * BN + x * BN, smem_desc_kmajor(p_addr + kk * 32, BN),
                    smem_desc_kmajor(v_addr + kk * 32, BN), idesc_pv, (j > 0 || kk > 0));
        mma_commit(&s.p_free[x]);
        mma_commit(&s.o_done[x]);
      }
      if (!ok) break;
      mma_commit(&s.v_empty[stv]);
    }
  }
  // Drain: all MMAs issued by this thread complete before TMEM is freed.
  mma_commit(&s.drain);
  drain_wait(&s.drain, 0, w);
}

// ------------------------------------------------------------------ softmax

// Seed the warp's 32 rows of the S columns with kBiasBits (asynchronous
// TMEM store; see release_scores).
__device__ __forceinline__ void seed_scores(uint32_t tS) { tmem_fill128_nowait(tS, kBiasBits); }

// Wait for the seed to land and tell the MMA issuer that S may be written.
__device__ __forceinline__ void release_scores(uint64_t* s_free, int lane) {
  tmem_wait_st();
  tc_fence_before();
  warp_arrive(s_free, lane);
}

// Max of 32 biased scores (all > 0), 3-input maxima in two chains.
__device__ __forceinline__ float max32(const uint32_t (&v)[32]) {
  float a = fmax3(__uint_as_float(v[0]), __uint_as_float(v[1]), __uint_as_float(v[2]));
  float b = fmax3(__uint_as_float(v[3]), __uint_as_float(v[4]), __uint_as_float(v[5]));
#pragma unroll
  for (int j = 6; j < 30; j += 4) {
    a = fmax3(a, __uint_as_float(v[j]), __uint_as_float(v[j + 1]));
    b = fmax3(b, __uint_as_float(v[j + 2]), __uint_as_float(v[j + 3]));
  }
  return fmax3(a, b, fmaxf(__uint_as_float(v[30]), __uint_as_float(v[31])));
}

// Keys at or past `nvis` (masked) read as 0, below every seeded score.
__device__ __forceinline__ void mask_chunk(uint32_t (&v)[32], int j0, int nvis) {
#pragma unroll
  for (int e = 0; e < 32; e++) v[e] = (j0 + e < nvis) ? v[e] : 0u;
}

// Online softmax of query tile X (0 = A, 1 = B), one row per thread.  The
// score row is read from TMEM in 32-column chunks (double-buffered), once
// for the maximum and once for the exponentials, so that few registers are
// live at any time.
template <int D>
__device__ __forceinline__ void softmax_rows(Smem<D>& s, const AttnParams& p, uint32_t tmem,
                                             int X, int bh, int q0, int nk, const WaitCtx& w) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int quad = warp & 3;               // TMEM lane quadrant of this warp
  const int r = quad * 32 + lane;          // row within the tile
  const int i = q0 + X * BM + r;           // query row
  const bool valid = i < p.Nq;
  const uint32_t tS = tmem + (static_cast<uint32_t>(quad * 32) << 16) + X * BN;
  const int lim = valid ? row_limit(i, p) : 0;
  const float sqC = valid ? __fmul_rn(__ldg(p.q_scale + static_cast<size_t>(bh) * p.nq_blocks + i / 64), p.c0)
                          : 0.0f;
  const float* ksc = p.k_scale + static_cast<size_t>(bh) * p.nkv_blocks;

  seed_scores(tS);  // S seed for the first tile
  release_scores(&s.s_free[X], lane);
  if (X == 1) warp_arrive(&s.turn[0], lane);  // tile A takes the first turn

  // K scales of a tile's two 64-key groups, loaded one tile ahead (blocks
  // past the end read as 0)
  float sk0 = __ldg(ksc), sk1 = p.nkv_blocks > 1 ? __ldg(ksc + 1) : 0.0f;
  float m = -INFINITY, l = 0.0f;
  for (int it = 0; it < nk; it++) {
    const int j0 = it * BN;
    const int pb = it & 1;
    const float c0 = __fmul_rn(sqC, sk0), c1 = __fmul_rn(sqC, sk1);
    {
      const int g0 = 2 * it + 2, g1 = 2 * it + 3;
      sk0 = g0 < p.nkv_blocks ? __ldg(ksc + g0) : 0.0f;
      sk1 = g1 < p.nkv_blocks ? __ldg(ksc + g1) : 0.0f;
    }
    if (!warp_wait(&s.s_full[X], it & 1, w, kSiteSmS)) return;
    tc_fence_after();
    const int nvis = min(max(lim - j0, 0), BN);  // visible keys of this tile
    const bool full = __all_sync(kFull, nvis == BN);

    // ---- maximum per 64-key scale group (biased scores; 0 = all masked)
    float mb[2];
    {
      uint32_t b0[32], b1[32];
      tmem_ld32_async(tS, b0);
#pragma unroll
      for (int c = 0; c < 4; c++) {
        uint32_t (&cur)[32] = (c & 1) ? b1 : b0;
        uint32_t (&nxt)[32] = (c & 1) ? b0 : b1;
        tmem_wait_ld(cur);
        if (c < 3) tmem_ld32_async(tS + 32 * (c + 1), nxt);
        if (!full) mask_chunk(cur, 32 * c, nvis);
        const float cm = max32(cur);
        if (c & 1) mb[c >> 1] = fmaxf(mb[c >> 1], cm);
        else mb[c >> 1] = cm;
      }
    }
    // max_j fp32(S_j * c) = fp32(max_j S_j * c) for c >= 0 (rounding is monotone)
    const float t0 = mb[0] > 0.0f ? __fmul_rn(__fsub_rn(mb[0], kBias), c0) : -INFINITY;
    const float t1 = mb[1] > 0.0f ? __fmul_rn(__fsub_rn(mb[1], kBias), c1) : -INFINITY;
    const float m_new = fmax3(m, t0, t1);
    const float alpha = (m == -INFINITY) ? 0.0f
                        : (m == m_new)   ? 1.0f
                                         : ex2_approx(__fsub_rn(m, m_new));
    const float nm8 = __fsub_rn(8.0f, m_new);  // P scale 2^8 folded into the exponent
    s.alpha[X][pb][r] = alpha;
    warp_arrive(&s.alpha_full[X][pb], lane);

    // the P tile is free once P V of the previous tile has read it; then
    // wait for this warpgroup's turn at the exp2 phase
    if (it >= 1 && !warp_wait(&s.p_free[X], (it - 1) & 1, w, kSiteSmPFree)) return;
    if (!warp_wait(&s.turn[X], it & 1, w, kSiteSmTurn)) return;

    // ---- y = 2^(S c + 8 - m), row sum, e4m3 codes into the swizzled P tile
    uint8_t* prow = s.p[X] + r * BN;
    const float2 nb2 = make_float2(-kBias, -kBias);
    const float2 nm2 = make_float2(nm8, nm8);
    float2 acc[2] = {make_float2(0.0f, 0.0f), make_float2(0.0f, 0.0f)};
    {
      uint32_t b0[32], b1[32];
      tmem_ld32_async(tS, b0);
#pragma unroll
      for (int c = 0; c < 4; c++) {
        uint32_t (&cur)[32] = (c & 1) ? b1 : b0;
        uint32_t (&nxt)[32] = (c & 1) ? b0 : b1;
        tmem_wait_ld(cur);
        if (c < 3) tmem_ld32_async(tS + 32 * (c + 1), nxt);
        const float2 cc = c < 2 ? make_float2(c0, c0) : make_float2(c1, c1);
        float y[32];
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          const float2 x = __ffma2_rn(
              __fadd2_rn(make_float2(__uint_as_float(cur[e]), __uint_as_float(cur[e + 1])), nb2), cc, nm2);
          y[e] = x.x;
          y[e + 1] = x.y;
        }
        if (!full) {
#pragma unroll
          for (int e = 0; e < 32; e++) y[e] = (32 * c + e < nvis) ? y[e] : -INFINITY;
        }
#pragma unroll
        for (int e = 0; e < 32; e++) y[e] = ex2_approx(y[e]);
#pragma unroll
        for (int e = 0; e < 32; e += 4) {
          acc[0] = __fadd2_rn(acc[0], make_float2(y[e], y[e + 1]));
          acc[1] = __fadd2_rn(acc[1], make_float2(y[e + 2], y[e + 3]));
        }
#pragma unroll
        for (int h = 0; h < 2; h++) {  // two 16-key chunks of the P row
          uint32_t pk[4];
#pragma unroll
          for (int q4 = 0; q4 < 4; q4++) {
            const int e = h * 16 + q4 * 4;
            pk[q4] = __byte_perm(cvt_e4m3x2(y[e], y[e + 1]), cvt_e4m3x2(y[e + 2], y[e + 3]), 0x5410);
          }
          const int chunk = 2 * c + h;
          *reinterpret_cast<uint4*>(prow + ((chunk ^ (r & 7)) << 4)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        }
      }
    }
    seed_scores(tS);  // S seed for the next tile
    fence_proxy_async_smem();
    release_scores(&s.s_free[X], lane);
    __syncwarp();
    if (lane == 0) {
      mbar_arrive(&s.turn[X ^ 1]);   // the other warpgroup's turn
      mbar_arrive(&s.p_full[X]);
    }
    const float2 a2 = __fadd2_rn(acc[0], acc[1]);
    l = __fadd_rn(__fmul_rn(l, alpha), __fadd_rn(a2.x, a2.y));
    m = m_new;
  }
  s.fin_m[X][r] = m;
  s.fin_l[X][r] = l;
  warp_arrive(&s.fin_ready[X], lane);
}

// ------------------------------------------------------------------ correction + epilogue

template <int D>
__device__ __forceinline__ void rescale_row(uint32_t tO, float alpha) {
  // 32-column pieces keep the register footprint small
#pragma unroll 1
  for (int c = 0; c < D; c += 32) {
    uint32_t o[32];
    tmem_ld32(tO + c, o);
#pragma unroll
    for (int e = 0; e < 32; e += 2) {
      const float2 v = __fmul2_rn(make_float2(__uint_as_float(o[e]), __uint_as_float(o[e + 1])),
                                  make_float2(alpha, alpha));
      o[e] = __float_as_uint(v.x);
      o[e + 1] = __float_as_uint(v.y);
    }
    tmem_st32(tO + c, o);
  }
}

template <int D>
__device__ __forceinline__ void correction_rows(Smem<D>& s, const AttnParams& p, uint32_t tmem,
                                                int bh, int q0, int nk, const WaitCtx& w) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int quad = warp & 3;
  const int r = quad * 32 + lane;
  const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
  for (int it = 0; it < nk; it++) {
    const int pb = it & 1;
    for (int x = 0; x < NQT; x++) {
      if (!warp_wait(&s.alpha_full[x][pb], (it >> 1) & 1, w, kSiteCorrAlpha)) return;
      const float alpha = s.alpha[x][pb][r];
      if (it > 0) {
        // P V of the previous tile must have completed before O is rescaled
        if (!warp_wait(&s.o_done[x], (it - 1) & 1, w, kSiteCorrO)) return;
        tc_fence_after();
        if (__any_sync(kFull, alpha != 1.0f))
          rescale_row<D>(tmem + lane_off + 2 * BN + x * BN, alpha);
      }
      tc_fence_before();
      warp_arrive(&s.corr_done[x], lane);
    }
  }
  // epilogue: O_X * v_scale / l -> bf16 (and fp32 O, lse)
  const float* vsc = p.v_scale + static_cast<size_t>(bh) * D;
  for (int x = 0; x < NQT; x++) {
    if (!warp_wait(&s.o_done[x], (nk - 1) & 1, w, kSiteEpiO)) return;
    if (!warp_wait(&s.fin_ready[x], 0, w, kSiteEpiFin)) return;
    tc_fence_after();
    const int i = q0 + x * BM + r;
    const bool valid = i < p.Nq;
    const float l = s.fin_l[x][r], m = s.fin_m[x][r];
    const float inv = __frcp_rn(l);  // l is in units of 2^8 p
    const size_t orow = (static_cast<size_t>(bh) * p.Nq + (valid ? i : 0)) * D;
    const uint32_t tO = tmem + lane_off + 2 * BN + x * BN;
#pragma unroll 1
    for (int c = 0; c < D; c += 32) {
      uint32_t o[32];
      tmem_ld32(tO + c, o);
      if (!valid) continue;
#pragma unroll
      for (int e = 0; e < 32; e++)
        o[e] = __float_as_uint(__uint_as_float(o[e]) * (__ldg(vsc + c + e) * inv));
      if (p.o_f32) {
        float4* d32 = reinterpret_cast<float4*>(p.o_f32 + orow + c);
#pragma unroll
        for (int e = 0; e < 8; e++)
          d32[e] = make_float4(__uint_as_float(o[4 * e]), __uint_as_float(o[4 * e + 1]),
                               __uint_as_float(o[4 * e + 2]), __uint_as_float(o[4 * e + 3]));
      }
#pragma unroll
      for (int e = 0; e < 16; e++) {
        __nv_bfloat162 h = __floats2bfloat162_rn(__uint_as_float(o[2 * e]), __uint_as_float(o[2 * e + 1]));
        o[e] = *reinterpret_cast<uint32_t*>(&h);
      }
      uint4* dst = reinterpret_cast<uint4*>(p.o + orow + c);
#pragma unroll
      for (int e = 0; e < 4; e++) dst[e] = make_uint4(o[4 * e], o[4 * e + 1], o[4 * e + 2], o[4 * e + 3]);
    }
    if (valid && p.lse)
      p.lse[static_cast<size_t>(bh) * p.Nq + i] = (m + log2f(l) - 8.0f) * 0.69314718055994531f;
  }
}

// Score dump (debug): copy the int32 S tile of query tile A from TMEM to
// global memory (the accumulator seed removed).
template <int D>
__device__ __forceinline__ void dump_rows(Smem<D>& s, const AttnParams& p, uint32_t tmem,
                                          const WaitCtx& w) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int quad = warp & 3;
  const int r = quad * 32 + lane;
  const uint32_t tS = tmem + (static_cast<uint32_t>(quad * 32) << 16);
  seed_scores(tS);
  release_scores(&s.s_free[0], lane);
  if (!warp_wait(&s.s_full[0], 0, w, kSiteSmS)) return;
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

// ------------------------------------------------------------------ kernel

template <int D, bool DUMP>
__global__ void __launch_bounds__(kThreads, 1)
    k_attn(const __grid_constant__ AttnMaps maps, const AttnParams p) {
  extern __shared__ uint8_t smem_raw[];
  Smem<D>& s = *reinterpret_cast<Smem<D>*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = DUMP ? p.dbg_bh : static_cast<int>(blockIdx.y);
  // first query row of the CTA (DUMP: the requested 128-row tile)
  const int q0 = DUMP ? p.dbg_qt * BM : static_cast<int>(blockIdx.x) * NQT * BM;

  // KV tiles this CTA visits: those holding a key visible to its last valid
  // row (the masks' limits grow with the row index).
  int kt0 = 0, nk;
  if (DUMP) {
    kt0 = p.dbg_kt;
    nk = 1;
  } else {
    const int last = min(p.Nq - 1, q0 + NQT * BM - 1);
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
    for (int x = 0; x < NQT; x++) {
      mbar_init(&s.s_full[x], 1);
      mbar_init(&s.s_free[x], 4);
      mbar_init(&s.p_full[x], 4);
      mbar_init(&s.p_free[x], 1);
      for (int b = 0; b < 2; b++) mbar_init(&s.alpha_full[x][b], 4);
      mbar_init(&s.corr_done[x], 4);
      mbar_init(&s.o_done[x], 1);
      mbar_init(&s.turn[x], 4);
      mbar_init(&s.fin_ready[x], 4);
    }
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
  const uint32_t tmem = s.tmem_base;  // S_A, S_B at columns 0, 128; O_A, O_B at 256, 384
  const WaitCtx w{p.budget, p.status, &s.abort};

  const int wg = warp >> 2;
  if (wg == 0) {
    regs_dec<kRegsRoles>();
    if (warp == 0) {
      if (lane == 0) producer<D, DUMP>(s, maps, bh, q0, kt0, nk, true, w);
    } else if (warp == 1) {
      if (lane == 0) mma_issuer<D, DUMP>(s, tmem, nk, w);
    } else if (warp == 2 && !DUMP) {
      if (lane == 0) producer<D, DUMP>(s, maps, bh, q0, kt0, nk, false, w);
    }
  } else if (wg <= NQT) {
    regs_inc<kRegsSoftmax>();
    if (DUMP) {
      if (wg == 1) dump_rows<D>(s, p, tmem, w);
    } else {
      softmax_rows<D>(s, p, tmem, wg - 1, bh, q0, nk, w);
    }
  } else {
    regs_dec<kRegsCorr>();
    if (!DUMP) correction_rows<D>(s, p, tmem, bh, q0, nk, w);
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// One-time per-device setup: dynamic shared memory size, and a check that
// the compiled kernels were built with exactly kLaunchRegs registers per
// thread.  The warpgroups' setmaxnreg shares add up to that launch
// allocation; a different allocation could leave an increase waiting, so
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

}  // namespace

size_t attn_smem_bytes(int D) { return smem_bytes_for(D); }

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
  dim3 grid((p.Nq + NQT * BM - 1) / (NQT * BM), p.BH);
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
