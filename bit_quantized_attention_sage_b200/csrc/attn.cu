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
// KV tiles of 128 keys.  Warp roles (192 threads, two CTAs per SM):
//   warp 0      TMA producer: the Q tile once, then K and V tiles through
//               a two-stage shared-memory ring (128-byte swizzle; V tiles
//               are [keys][D], used as MN-major operands).
//               The e4m3 P tile is double-buffered: the softmax of tile k
//               writes P(k) while P V of tile k-1 may still read P(k-1).
//   warp 1      allocates 256 TMEM columns (S: 128 x 128 int32, O: 128 x D
//               fp32) and one elected thread issues every tcgen05.mma:
//               S = Q K^T (kind::i8) for tile k+1 while the softmax warps
//               work on tile k, then O (+)= P V (kind::f8f6f4).
//   warps 2-5   softmax: thread t of the warpgroup owns query row t (TMEM
//               lane t).  The S accumulator columns are seeded with the bit
//               pattern 0x4B400000 before each Q K^T, so the int32 result
//               0x4B400000 + S reads as the fp32 value 1.5*2^23 + S exactly
//               (no conversion unit, no integer add).  Per tile: load the
//               score row from TMEM, take the masked max per 64-key scale
//               group with a tree of 3-input maxima, update the running max,
//               re-seed the row, y = exp2(fma(S, c, 8 - m)) (P scale 2^8 folded
//               into the exponent) with packed fp32x2 arithmetic, row sum,
//               e4m3(y) into the swizzled shared-memory P buffer of the
//               tile's parity, then (once P V of the previous tile has
//               completed) rescale the O row in TMEM when the max moved.
//               Epilogue: O * v_scale / l -> bf16 (and optional fp32 O, lse).
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
constexpr int NS = 2;              // K/V pipeline stages
constexpr int kThreads = 192;      // 6 warps
constexpr int kTmemCols = 256;
constexpr int kMaxTileWords = kAttnMaxKvTiles / 32;  // block-sparse tile bitmap
constexpr uint32_t kFull = 0xffffffffu;
// The S accumulator is seeded with the bit pattern of 1.5 * 2^23; for
// |S| < 2^22 the int32 sum 0x4B400000 + S reads as the fp32 value
// 1.5 * 2^23 + S exactly (|S| <= 128 * 128 * D < 2^22 for D <= 128).
constexpr uint32_t kBiasBits = 0x4B400000u;
constexpr float kBias = 12582912.0f;
constexpr uint32_t kNegInfBits = 0xFF800000u;
// KV-tile columns >= kPolyFrom take the software exp2 (exp2_poly2), the rest
// the exp2 unit
#ifndef SAGE_POLY_FROM
#define SAGE_POLY_FROM 128
#endif
constexpr int kPolyFrom = SAGE_POLY_FROM;

// wait-site codes for the status word (kernel 1 = attention)
enum : int {
  kSiteProdKEmpty = 0x10101, kSiteProdVEmpty, kSiteMmaQ, kSiteMmaK, kSiteMmaSFree,
  kSiteMmaV, kSiteMmaP, kSiteSmS, kSiteSmO, kSiteSmEpi, kSiteDrain, kSiteSmemAlign
};

// The keys query row i sees: [0, sink_end) and [lo, hi).  Queries are the
// newest Nq positions of the Nkv keys (position g = i + Nkv - Nq).
//   none / causal / block-causal: sink_end = lo = 0; hi = Nkv, g + 1, or the
//     end of g's block of mask_block keys.
//   sliding window: sink_end = sink, the reference context, for every row;
//     for g >= sink, [lo, hi) = frames f - win + 1 .. f of
//     f = (g - sink) / mask_block (frames of mask_block keys after the
//     reference context); a query inside the reference context has the
//     empty window lo = hi = sink, i.e. sees the reference context only.
// lo and hi never decrease with g, and hi(g) >= lo(g + 1): the rows of a
// query tile together see [0, sink_end) and one contiguous key range.
struct RowKeys {
  int sink_end, lo, hi;
};

__device__ __forceinline__ RowKeys row_keys(int i, const AttnParams& p) {
  const int g = i + (p.Nkv - p.Nq);
  RowKeys r{0, 0, p.Nkv};
  if (p.mask == 1) {
    r.hi = g + 1;
  } else if (p.mask == 2) {
    r.hi = (g / p.mask_block + 1) * p.mask_block;
  } else if (p.mask == kMaskSlidingWindow) {
    r.sink_end = p.sink;
    if (g < p.sink) {
      r.lo = r.hi = p.sink;
    } else {
      const int f = (g - p.sink) / p.mask_block;
      r.lo = p.sink + max(f - p.win + 1, 0) * p.mask_block;
      r.hi = p.sink + (f + 1) * p.mask_block;
    }
  }
  r.hi = min(r.hi, p.Nkv);
  return r;
}

// The KV tiles of a query tile form the sequence [0, ns) then [ns + gap, ...):
// a gap of tiles that no row sees lies between the reference context and the
// window (sliding-window mask only; gap = 0 otherwise).
struct TileGap {
  int ns, gap;
  __device__ __forceinline__ int tile(int idx) const { return idx < ns ? idx : idx + gap; }
};

template <int D>
struct alignas(1024) Smem {
  uint8_t q[BM * D];         // int8 Q tile [128 rows][D]
  uint8_t k[NS][BN * D];     // int8 K tiles [128 keys][D]
  uint8_t v[NS][BN * D];     // e4m3 V tiles [128 keys][D] (MN-major operand)
  uint8_t p[2][BM * BN];     // e4m3 P tiles [parity][128 rows][128 keys], 128-byte swizzle
  uint64_t q_full;
  uint64_t k_full[NS], k_empty[NS];
  uint64_t v_full[NS], v_empty[NS];
  uint64_t s_full, s_free, p_full, o_ready, drain;
  uint32_t tmem_base;
  int abort;
  // block-sparse mode: bit t set = KV tile t is visited by this CTA
  uint32_t tile_bits[kMaxTileWords];
};

// Exactly the struct: two D = 128 CTAs fill the SM's 228 KB (2 x (113 KB +
// 1 KB reserved)), so there is no room for alignment slack.  The dynamic
// shared-memory window is 1024-byte aligned (the kernel checks this).
__host__ __device__ inline size_t smem_bytes_for(int D) {
  return D == 128 ? sizeof(Smem<128>) : sizeof(Smem<64>);
}
static_assert(sizeof(Smem<128>) <= 115712, "two CTAs per SM must fit in 228 KB");

// A wait taken by all 32 threads of a warp that reports success only if it
// succeeded for every lane, so that the warp never splits before the
// warp-collective tcgen05.ld / tcgen05.st that follow.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, const WaitCtx& w,
                                          int site) {
  return __all_sync(kFull, mbar_wait(bar, parity, w, site));
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

// The KV tiles a CTA visits, in ascending order: entries kt0, kt0 + 1, ... of
// the tile sequence (dense) or the set bits of the CTA's tile bitmap
// (block-sparse).  next() must be
// called at most as many times as there are tiles.
template <bool SPARSE>
struct TileSeq {
  const uint32_t* bits;
  int w;
  uint32_t cur;
  TileGap tg;
  __device__ __forceinline__ TileSeq(const uint32_t* b, int kt0, TileGap g)
      : bits(b), w(SPARSE ? 0 : kt0), cur(SPARSE ? b[0] : 0u), tg(g) {}
  __device__ __forceinline__ int next() {
    if constexpr (!SPARSE) {
      return tg.tile(w++);
    } else {
      while (cur == 0u) cur = bits[++w];
      const int t = w * 32 + __ffs(static_cast<int>(cur)) - 1;
      cur &= cur - 1u;
      return t;
    }
  }
};

template <int D, bool DUMP, bool SPARSE>
__device__ __forceinline__ void producer(Smem<D>& s, const AttnMaps& maps, int bh, int qt,
                                         int kt0, int nk, TileGap tg, const WaitCtx& w) {
  tma_prefetch_desc(&maps.q);
  tma_prefetch_desc(&maps.k);
  tma_prefetch_desc(&maps.v);
  mbar_arrive_expect_tx(&s.q_full, BM * D);
  tma_load_3d(s.q, &maps.q, &s.q_full, 0, qt * BM, bh);
  int k_issued = 0, v_issued = 0;
  TileSeq<SPARSE> seq(s.tile_bits, kt0, tg);
  for (int it = 0; it < nk; it++) {
    const int st = it % NS;
    const uint32_t ph = (it / NS) & 1;
    const int kt = seq.next();
    if (it >= NS && !mbar_wait(&s.k_empty[st], ph ^ 1, w, kSiteProdKEmpty)) break;
    mbar_arrive_expect_tx(&s.k_full[st], BN * D);
    tma_load_3d(s.k[st], &maps.k, &s.k_full[st], 0, kt * BN, bh);
    k_issued++;
    if (DUMP) continue;
    if (it >= NS && !mbar_wait(&s.v_empty[st], ph ^ 1, w, kSiteProdVEmpty)) break;
    mbar_arrive_expect_tx(&s.v_full[st], D * BN);
    tma_load_3d(s.v[st], &maps.v, &s.v_full[st], 0, kt * BN, bh);
    v_issued++;
  }
  // Drain: every issued load must have landed before the CTA may exit.  A
  // load is only issued once the previous load of its stage was consumed, so
  // only the last NS loads of each kind can still be in flight.
  drain_wait(&s.q_full, 0, w);
  for (int it = (k_issued > NS ? k_issued - NS : 0); it < k_issued; it++)
    drain_wait(&s.k_full[it % NS], (it / NS) & 1, w);
  for (int it = (v_issued > NS ? v_issued - NS : 0); it < v_issued; it++)
    drain_wait(&s.v_full[it % NS], (it / NS) & 1, w);
}

template <int D, bool DUMP>
__device__ __forceinline__ void mma_issuer(Smem<D>& s, uint32_t tmem_S, uint32_t tmem_O, int nk,
                                           const WaitCtx& w) {
  constexpr uint32_t idesc_qk = idesc_i8_s32(BM, BN);
  // P V: B = V tile stored [keys][D], i.e. N-contiguous (MN-major)
  constexpr uint32_t idesc_pv = idesc_e4m3_f32(BM, D) | kIdescBMajorMN;
  const uint32_t q_addr = smem_u32(s.q);
  const uint32_t p_addr0 = smem_u32(s.p[0]);
  bool ok = mbar_wait(&s.q_full, 0, w, kSiteMmaQ);
  for (int it = 0; ok && it <= nk; it++) {
    if (it < nk) {  // S = Q K^T for tile it
      const int st = it % NS;
      const uint32_t ph = (it / NS) & 1;
      if (!mbar_wait(&s.k_full[st], ph, w, kSiteMmaK)) break;
      // the softmax warps have read S of the previous tile and re-seeded it
      // (score dumps are not seeded and hold one tile only)
      if (!DUMP && !mbar_wait(&s.s_free, it & 1, w, kSiteMmaSFree)) break;
      tc_fence_after();
      const uint32_t k_addr = smem_u32(s.k[st]);
#pragma unroll
      for (int kk = 0; kk < D / 32; kk++)
        mma_i8_ss(tmem_S, smem_desc_kmajor(q_addr + kk * 32, D),
                  smem_desc_kmajor(k_addr + kk * 32, D), idesc_qk, DUMP ? kk > 0 : 1);
      mma_commit(&s.k_empty[st]);
      mma_commit(&s.s_full);
    }
    if (!DUMP && it > 0) {  // O (+)= P V for tile it - 1
      const int j = it - 1;
      const int st = j % NS;
      const uint32_t ph = (j / NS) & 1;
      if (!mbar_wait(&s.v_full[st], ph, w, kSiteMmaV)) break;
      if (!mbar_wait(&s.p_full, j & 1, w, kSiteMmaP)) break;
      tc_fence_after();
      const uint32_t v_addr = smem_u32(s.v[st]);
      const uint32_t p_addr = p_addr0 + static_cast<uint32_t>(j & 1) * (BM * BN);
#pragma unroll
      for (int kk = 0; kk < BN / 32; kk++)
        mma_f8_ss(tmem_O, smem_desc_kmajor(p_addr + kk * 32, BN),
                  smem_desc_mnmajor(v_addr + kk * 32 * D, D), idesc_pv, (j > 0 || kk > 0));
      mma_commit(&s.v_empty[st]);
      mma_commit(&s.o_ready);
    }
  }
  // Drain: all MMAs issued by this thread complete before TMEM is freed.
  mma_commit(&s.drain);
  drain_wait(&s.drain, 0, w);
}

// Scale of K block g of a head; blocks past the end read as 0.
__device__ __forceinline__ float k_block_scale(const float* ksc, int g, int nblocks) {
  return g < nblocks ? __ldg(ksc + g) : 0.0f;
}

// O row (this thread's TMEM lane) *= alpha: one TMEM round trip, packed
// fp32x2 multiplies.
template <int D>
__device__ __forceinline__ void rescale_row(uint32_t tO, float alpha) {
  const float2 al2 = make_float2(alpha, alpha);
  if constexpr (D == 128) {
    uint32_t o[128];
    tmem_ld128(tO, o);
#pragma unroll
    for (int e = 0; e < 128; e += 2) {
      const float2 v = __fmul2_rn(make_float2(__uint_as_float(o[e]), __uint_as_float(o[e + 1])), al2);
      o[e] = __float_as_uint(v.x);
      o[e + 1] = __float_as_uint(v.y);
    }
    tmem_st128_nowait(tO, o);
  } else {
    uint32_t o[64];
    tmem_ld64(tO, o);
#pragma unroll
    for (int e = 0; e < 64; e += 2) {
      const float2 v = __fmul2_rn(make_float2(__uint_as_float(o[e]), __uint_as_float(o[e + 1])), al2);
      o[e] = __float_as_uint(v.x);
      o[e + 1] = __float_as_uint(v.y);
    }
    tmem_st64_nowait(tO, o);
  }
  tmem_wait_st();
}

// Softmax / correction / epilogue for one query row per thread.
template <int D, bool SPARSE, bool SPLIT, bool WIN>
__device__ __forceinline__ void softmax_rows(Smem<D>& s, const AttnParams& p, uint32_t tmem_S,
                                             uint32_t tmem_O, int bh, int qt, int kt0, int nk,
                                             TileGap tg, const WaitCtx& w) {
  const int kt_base = SPLIT ? kt0 : 0;  // first entry of the tile sequence (dense: 0)
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int quad = warp & 3;               // TMEM lane quadrant of this warp
  const int r = quad * 32 + lane;          // row within the tile
  const int i = qt * BM + r;               // query row
  const bool valid = i < p.Nq;
  // visible keys of this row: [0, p.sink) and [rk.lo, rk.hi) (sliding
  // window), or [0, lim) (the prefix masks).  Rows past Nq are never
  // stored; they see no key, or the reference context alone (all their
  // scores are 0: their Q codes are zero).
  RowKeys rk{0, 0, 0};
  int lim = 0;
  if (valid) {
    if constexpr (WIN) rk = row_keys(i, p);
    else lim = row_keys(i, p).hi;
  }
  const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
  const uint32_t tS = tmem_S + lane_off, tO = tmem_O + lane_off;
  const float sqC = valid ? __fmul_rn(__ldg(p.q_scale + static_cast<size_t>(bh) * p.nq_blocks + i / 64), p.c0)
                          : 0.0f;
  const float* ksc = p.k_scale + static_cast<size_t>(bh) * p.nkv_blocks;
  uint8_t* prow0 = s.p[0] + r * BN;

  TileSeq<SPARSE> seq(s.tile_bits, 0, tg);
  // KV tile of this iteration
  int kt = (SPARSE && nk > 0) ? seq.next() : (WIN ? tg.tile(kt_base) : kt_base);
  float ks0 = k_block_scale(ksc, 2 * kt, p.nkv_blocks);
  float ks1 = k_block_scale(ksc, 2 * kt + 1, p.nkv_blocks);
  float m = -INFINITY, l = 0.0f;
  bool ok = true;
  // seed the S row for the first tile (the MMA issuer waits for it)
  tmem_fill128_nowait(tS, kBiasBits);
  tmem_wait_st();
  tc_fence_before();
  __syncwarp();
  if (lane == 0) mbar_arrive(&s.s_free);
  for (int it = 0; it < nk; it++) {
    if constexpr (!SPARSE) kt = WIN ? tg.tile(kt_base + it) : kt_base + it;
    const int j0 = kt * BN;
    if (!warp_wait(&s.s_full, it & 1, w, kSiteSmS)) { ok = false; break; }
    tc_fence_after();
    uint32_t sv[128];  // 0x4B400000 + S: the fp32 value 1.5 * 2^23 + S
    tmem_ld128(tS, sv);
    const bool more = it + 1 < nk;

    // scale of each 64-key group of the tile; the next tile's K scales are
    // loaded now so that their latency is hidden behind this tile
    const float c0 = __fmul_rn(sqC, ks0), c1 = __fmul_rn(sqC, ks1);
    const int kt_next = (SPARSE && more) ? seq.next()
                        : WIN            ? tg.tile(kt_base + it + 1)
                                         : kt + 1;
    ks0 = k_block_scale(ksc, 2 * kt_next, p.nkv_blocks);
    ks1 = k_block_scale(ksc, 2 * kt_next + 1, p.nkv_blocks);
    // masked keys read as -inf: below every seeded score (> 2^23) in the
    // max, and exp2 of their argument is exactly 0 (see ce0, ce1, nm8)
    if constexpr (WIN) {
      // visible keys of this tile: [0, na) (reference context) and [nb, nc)
      const int na = min(max(p.sink - j0, 0), BN);
      const int nb = min(max(rk.lo - j0, 0), BN);
      const int nc = min(max(rk.hi - j0, 0), BN);
      if (!__all_sync(kFull, na == BN || (nb == 0 && nc == BN))) {
        const uint32_t nbc = static_cast<uint32_t>(nc - nb);  // nb <= nc
#pragma unroll
        for (int j = 0; j < BN; j++)
          sv[j] = (j < na || static_cast<uint32_t>(j - nb) < nbc) ? sv[j] : kNegInfBits;
      }
    } else {
      const int nvis = min(max(lim - j0, 0), BN);  // visible keys of this tile
      if (!__all_sync(kFull, nvis == BN)) {
#pragma unroll
        for (int j = 0; j < BN; j++) sv[j] = j < nvis ? sv[j] : kNegInfBits;
      }
    }
    // masked max per 64-key group on the seeded values, a tree of 3-input
    // maxima (monotone in S; for c >= 0, max_j fp32(S_j c) = fp32(max_j S_j c))
    float mg[2];
#pragma unroll
    for (int g = 0; g < 2; g++) {
      float t[8];
#pragma unroll
      for (int a = 0; a < 8; a++) {
        const int j = g * 64 + a * 8;
        t[a] = fmax3(__uint_as_float(sv[j]), __uint_as_float(sv[j + 1]), __uint_as_float(sv[j + 2]));
      }
#pragma unroll
      for (int a = 0; a < 8; a++) {
        const int j = g * 64 + a * 8;
        t[a] = fmax3(t[a], __uint_as_float(sv[j + 3]), __uint_as_float(sv[j + 4]));
        t[a] = fmax3(t[a], __uint_as_float(sv[j + 5]), __uint_as_float(sv[j + 6]));
        t[a] = fmaxf(t[a], __uint_as_float(sv[j + 7]));
      }
      mg[g] = fmax3(fmax3(t[0], t[1], t[2]), fmax3(t[3], t[4], t[5]), fmaxf(t[6], t[7]));
    }
    const float t0 = mg[0] < 8388608.0f ? -INFINITY : __fmul_rn(__fsub_rn(mg[0], kBias), c0);
    const float t1 = mg[1] < 8388608.0f ? -INFINITY : __fmul_rn(__fsub_rn(mg[1], kBias), c1);
    const float m_new = fmaxf(m, fmaxf(t0, t1));
    const float alpha = (m == -INFINITY) ? 0.0f
                        : (m == m_new)   ? 1.0f
                                         : ex2_approx(__fsub_rn(m, m_new));
    // P scale 2^8 folded into the exponent; a row with no visible key so far
    // (m_new = -inf) keeps every argument at -inf
    const float nm8 = m_new == -INFINITY ? 0.0f : __fsub_rn(8.0f, m_new);
    // exp arguments fma(S, c, nm8) with c replaced by FLT_MIN where c = 0:
    // identical for visible keys (c = 0 gives nm8 either way: |S| FLT_MIN is
    // far below half an ulp of nm8) and -inf for masked keys (-inf * c must
    // not be -inf * 0 = NaN)
    const float ce0 = c0 > 0.0f ? c0 : FLT_MIN, ce1 = c1 > 0.0f ? c1 : FLT_MIN;

    // re-seed S for the next tile (issued here, just before its wait: placed
    // ahead of the maximum it measured 2.8 % slower)
    if (more) tmem_fill128_x8_nowait(tS, kBiasBits);
    // the seed has landed; the MMA issuer may now write S of the next tile
    if (more) tmem_wait_st();
    tc_fence_before();
    __syncwarp();
    if (more && lane == 0) mbar_arrive(&s.s_free);

    // P buffer it & 1 was last read by P V of tile it - 2, which completed
    // before this thread's previous iteration passed its o_ready wait
    uint8_t* prow = prow0 + (it & 1) * (BM * BN);
    float2 acc[2] = {make_float2(0.0f, 0.0f), make_float2(0.0f, 0.0f)};
    const float2 nm2 = make_float2(nm8, nm8);
    const float2 nb2 = make_float2(-kBias, -kBias);
#pragma unroll
    for (int c = 0; c < 8; c++) {  // 16-key chunks
      uint32_t pk[4];
      const float2 cc = c < 4 ? make_float2(ce0, ce0) : make_float2(ce1, ce1);
#pragma unroll
      for (int q4 = 0; q4 < 4; q4++) {
        const int j = c * 16 + q4 * 4;
        float y[4];
#pragma unroll
        for (int e = 0; e < 4; e += 2) {
          const float2 sf = __fadd2_rn(make_float2(__uint_as_float(sv[j + e]), __uint_as_float(sv[j + e + 1])), nb2);
          float2 x = __ffma2_rn(sf, cc, nm2);
          if (c * 16 >= kPolyFrom) x = exp2_poly2(x);  // columns of the software exp2
          y[e] = x.x; y[e + 1] = x.y;
        }
        if (c * 16 < kPolyFrom) {
#pragma unroll
          for (int e = 0; e < 4; e++) y[e] = ex2_approx(y[e]);
        }
        acc[q4 & 1] = __fadd2_rn(acc[q4 & 1], make_float2(y[0], y[1]));
        acc[q4 & 1] = __fadd2_rn(acc[q4 & 1], make_float2(y[2], y[3]));
        pk[q4] = cvt_e4m3x4(y[0], y[1], y[2], y[3]);
      }
      *reinterpret_cast<uint4*>(prow + ((c ^ (r & 7)) << 4)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
    }
    const float2 a2 = __fadd2_rn(acc[0], acc[1]);
    const float rs = __fadd_rn(a2.x, a2.y);
    fence_proxy_async_smem();

    // O holds the sum through tile it - 1 once that tile's P V has completed;
    // rescale the O row when the running max moved (never before the first P V)
    if (it > 0 && !warp_wait(&s.o_ready, (it - 1) & 1, w, kSiteSmO)) { ok = false; break; }
    // the tcgen05 fences order the rescale's TMEM accesses after the P V it
    // waited for and before the next P V; a tile without a rescale touches
    // no TMEM here and needs neither
    if (it > 0 && __any_sync(kFull, alpha != 1.0f)) {
      tc_fence_after();
      rescale_row<D>(tO, alpha);
      tc_fence_before();
    }
    l = __fadd_rn(__fmul_rn(l, alpha), rs);
    m = m_new;
    kt = kt_next;
    __syncwarp();
    if (lane == 0) mbar_arrive(&s.p_full);
  }

  if (!ok) return;
  if constexpr (SPLIT) {  // this range's partial result: the raw O sum, m, l
    const size_t rows_pad = static_cast<size_t>(p.n_qt) * BM;
    const size_t prow = (static_cast<size_t>(blockIdx.z) * p.BH + bh) * rows_pad +
                        static_cast<size_t>(qt) * BM + r;
    float4* po = reinterpret_cast<float4*>(p.part_o + prow * D);
    if (nk == 0) {  // an empty range (fewer tiles than ranges): nothing seen
#pragma unroll 1
      for (int e = 0; e < D / 4; e++) po[e] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
      p.part_ml[prow * 2] = -INFINITY;
      p.part_ml[prow * 2 + 1] = 0.0f;
      return;
    }
    if (!warp_wait(&s.o_ready, (nk - 1) & 1, w, kSiteSmEpi)) return;
    tc_fence_after();
#pragma unroll 1
    for (int c = 0; c < D; c += 32) {
      uint32_t o[32];
      tmem_ld32(tO + c, o);
#pragma unroll
      for (int e = 0; e < 8; e++)
        po[c / 4 + e] = make_float4(__uint_as_float(o[4 * e]), __uint_as_float(o[4 * e + 1]),
                                    __uint_as_float(o[4 * e + 2]), __uint_as_float(o[4 * e + 3]));
    }
    p.part_ml[prow * 2] = m;
    p.part_ml[prow * 2 + 1] = l;
    return;
  }
  const float* vsc = p.v_scale + static_cast<size_t>(bh) * D;
  const size_t orow = (static_cast<size_t>(bh) * p.Nq + (valid ? i : 0)) * D;
  if (SPARSE && nk == 0) {  // no tile at all for this CTA; O = 0, lse = -inf
    if (valid) {
      uint4* dst = reinterpret_cast<uint4*>(p.o + orow);
#pragma unroll 1
      for (int e = 0; e < D / 8; e++) dst[e] = make_uint4(0u, 0u, 0u, 0u);
      if (p.o_f32) {
        float4* d32 = reinterpret_cast<float4*>(p.o_f32 + orow);
#pragma unroll 1
        for (int e = 0; e < D / 4; e++) d32[e] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
      }
      if (p.lse) p.lse[static_cast<size_t>(bh) * p.Nq + i] = -INFINITY;
    }
    return;
  }
  if (!warp_wait(&s.o_ready, (nk - 1) & 1, w, kSiteSmEpi)) return;
  tc_fence_after();
  // a row that saw no key (possible only with a block mask) has l = 0:
  // O = 0 (its O_acc row is 0) and lse = -inf
  const bool seen = !SPARSE || l > 0.0f;
  const float inv = seen ? __frcp_rn(l) : 0.0f;  // l is in units of 2^8 p
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
    p.lse[static_cast<size_t>(bh) * p.Nq + i] =
        seen ? (m + log2f(l) - 8.0f) * 0.69314718055994531f : -INFINITY;
}

// Score dump (debug): copy the int32 S tile from TMEM to global memory.
template <int D>
__device__ __forceinline__ void dump_rows(Smem<D>& s, const AttnParams& p, uint32_t tmem_S,
                                          const WaitCtx& w) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int quad = warp & 3;
  const int r = quad * 32 + lane;
  if (!warp_wait(&s.s_full, 0, w, kSiteSmS)) return;
  tc_fence_after();
  const uint32_t tS = tmem_S + (static_cast<uint32_t>(quad * 32) << 16);
#pragma unroll 1
  for (int c = 0; c < BN; c += 32) {
    uint32_t v[32];
    tmem_ld32(tS + c, v);
    uint4* dst = reinterpret_cast<uint4*>(p.dbg_out + static_cast<size_t>(r) * BN + c);
#pragma unroll
    for (int e = 0; e < 8; e++) dst[e] = make_uint4(v[4 * e], v[4 * e + 1], v[4 * e + 2], v[4 * e + 3]);
  }
  tc_fence_before();
  __syncwarp();
  if (lane == 0) mbar_arrive(&s.s_free);
}

template <int D, bool DUMP, bool SPARSE, bool SPLIT, bool WIN>
__device__ __forceinline__ void attn_body(const AttnMaps& maps, const AttnParams& p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // 128-byte swizzled TMA tiles and the MMA descriptors need 1024-byte
  // aligned tiles; refuse (before any barrier, copy or TMEM use) otherwise.
  if (smem_u32(smem_raw) & 1023u) {
    if (threadIdx.x == 0 && atomicCAS(p.status, 0, 3 /* SAGE_ERR_CUDA */) == 0)
      atomicExch(p.status + 1, kSiteSmemAlign);
    return;
  }
  Smem<D>& s = *reinterpret_cast<Smem<D>*>(smem_raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // masked shapes: the query tiles' work grows with their index, so the
  // heaviest are dispatched first and the last wave holds the lightest
  const int qt = DUMP ? p.dbg_qt
                      : static_cast<int>(p.mask != 0 ? gridDim.x - 1 - blockIdx.x : blockIdx.x);
  const int bh = DUMP ? p.dbg_bh : static_cast<int>(blockIdx.y);

  // KV tiles this CTA visits: those holding a key visible to one of its
  // rows, i.e. the reference context's tiles [0, ns) and the tiles of
  // [lo(first row), hi(last row)) -- one run unless a gap separates them.
  int kt0 = 0, nk;
  TileGap tg{0, 0};
  if (DUMP) {
    kt0 = p.dbg_kt;
    nk = 1;
  } else {
    const int last = min(p.Nq - 1, qt * BM + BM - 1);
    nk = (row_keys(last, p).hi + BN - 1) / BN;
    tg.ns = nk;
    if (WIN) {
      const int ts = (p.sink + BN - 1) / BN;
      const int t_lo = row_keys(qt * BM, p).lo / BN;
      if (t_lo > ts) {
        tg.ns = ts;
        tg.gap = t_lo - ts;
        nk -= tg.gap;
      }
    }
    if constexpr (SPLIT) {  // range blockIdx.z of p.splits contiguous ranges
      const int sp = static_cast<int>(blockIdx.z);
      kt0 = nk * sp / p.splits;
      nk = nk * (sp + 1) / p.splits - kt0;
    }
  }
  if constexpr (SPARSE) {
    // bitmap of the tiles below nk that the block mask switches on (one
    // ballot per 32 tiles); nk becomes their count after the barrier below
    const uint8_t* row = p.bmask + (static_cast<size_t>(bh) * p.n_qt + qt) * p.n_kt;
    const int nwords = (nk + 31) / 32;
    for (int wd = warp; wd < nwords; wd += kThreads / 32) {
      const int t = wd * 32 + lane;
      const uint32_t b = __ballot_sync(kFull, t < nk && row[t] != 0);
      if (lane == 0) s.tile_bits[wd] = b;
    }
  }

  if (threadIdx.x == 0) {
    mbar_init(&s.q_full, 1);
    for (int i = 0; i < NS; i++) {
      mbar_init(&s.k_full[i], 1);
      mbar_init(&s.k_empty[i], 1);
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
  if constexpr (SPARSE) {
    const int nwords = (nk + 31) / 32;
    int cnt = 0;
    for (int wd = 0; wd < nwords; wd++) cnt += __popc(s.tile_bits[wd]);
    nk = cnt;
  }
  const uint32_t tmem = s.tmem_base;
  const uint32_t tmem_S = tmem;        // columns [0, 128): int32 scores
  const uint32_t tmem_O = tmem + 128;  // columns [128, 128 + D): fp32 output
  const WaitCtx w{p.budget, p.status, &s.abort};

  if (warp == 0) {
    if (lane == 0) producer<D, DUMP, SPARSE>(s, maps, bh, qt, kt0, nk, tg, w);
  } else if (warp == 1) {
    if (lane == 0) mma_issuer<D, DUMP>(s, tmem_S, tmem_O, nk, w);
  } else {
    if (DUMP) dump_rows<D>(s, p, tmem_S, w);
    else softmax_rows<D, SPARSE, SPLIT, WIN>(s, p, tmem_S, tmem_O, bh, qt, kt0, nk, tg, w);
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <int D, bool DUMP, bool SPARSE>
__global__ void __launch_bounds__(kThreads, 2)
    k_attn(const __grid_constant__ AttnMaps maps, const AttnParams p) {
  attn_body<D, DUMP, SPARSE, false, false>(maps, p);
}

// Split-KV: CTA (qt, bh, range) over its range of the query tile's KV tiles;
// writes partial results for k_attn_merge.
template <int D>
__global__ void __launch_bounds__(kThreads, 2)
    k_attn_split(const __grid_constant__ AttnMaps maps, const AttnParams p) {
  attn_body<D, false, false, true, false>(maps, p);
}

// Sliding window with a reference context (mask kMaskSlidingWindow): the
// query tile's tiles are the reference context's and the window's, with the
// gap between them skipped; SPLIT as k_attn_split.
template <int D, bool SPLIT>
__global__ void __launch_bounds__(kThreads, 2)
    k_attn_win(const __grid_constant__ AttnMaps maps, const AttnParams p) {
  attn_body<D, false, false, SPLIT, true>(maps, p);
}

// Merge of the split-KV partials, 8 rows per 128-thread CTA, thread t: row
// t / 16, channels 8 (t % 16) .. + 7 (D = 128; D = 64 uses the first 8
// threads of each row).  m = max_s m_s, a_s = exp2(m_s - m) (0 for a range
// that saw no key), O = sum_s a_s O_s, l = sum_s a_s l_s in ascending s, each
// product and sum rounded once; then O vs / l as in the unsplit epilogue.
template <int D>
__global__ void __launch_bounds__(128) k_attn_merge(const AttnParams p) {
  const int bh = blockIdx.y;
  const int r = blockIdx.x * 8 + (threadIdx.x >> 4);  // row of the head
  const int c8 = (threadIdx.x & 15) * 8;
  if (r >= p.Nq || c8 >= D) return;
  const size_t rows_pad = static_cast<size_t>(p.n_qt) * BM;
  const size_t stride_s = static_cast<size_t>(p.BH) * rows_pad;  // rows per range
  const size_t row = static_cast<size_t>(bh) * rows_pad + r;
  float m = -INFINITY;
  for (int sp = 0; sp < p.splits; sp++) m = fmaxf(m, p.part_ml[(sp * stride_s + row) * 2]);
  float l = 0.0f;
  float o[8] = {0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f};
  for (int sp = 0; sp < p.splits; sp++) {
    const float ms = p.part_ml[(sp * stride_s + row) * 2];
    const float ls = p.part_ml[(sp * stride_s + row) * 2 + 1];
    const float a = ms == -INFINITY ? 0.0f : ex2_approx(__fsub_rn(ms, m));
    const float4* src = reinterpret_cast<const float4*>(p.part_o + (sp * stride_s + row) * D + c8);
    const float4 u = src[0], v = src[1];
    const float x[8] = {u.x, u.y, u.z, u.w, v.x, v.y, v.z, v.w};
#pragma unroll
    for (int e = 0; e < 8; e++) o[e] = __fmaf_rn(a, x[e], o[e]);
    l = __fadd_rn(l, __fmul_rn(a, ls));
  }
  const bool seen = l > 0.0f;
  const float inv = seen ? __frcp_rn(l) : 0.0f;
  const float* vsc = p.v_scale + static_cast<size_t>(bh) * D + c8;
  float f[8];
#pragma unroll
  for (int e = 0; e < 8; e++) f[e] = o[e] * (__ldg(vsc + e) * inv);
  uint32_t b[4];
#pragma unroll
  for (int e = 0; e < 4; e++) {
    __nv_bfloat162 h = __floats2bfloat162_rn(f[2 * e], f[2 * e + 1]);
    b[e] = *reinterpret_cast<uint32_t*>(&h);
  }
  const size_t orow = (static_cast<size_t>(bh) * p.Nq + r) * D + c8;
  *reinterpret_cast<uint4*>(p.o + orow) = make_uint4(b[0], b[1], b[2], b[3]);
  if (p.o_f32) {
    float4* d32 = reinterpret_cast<float4*>(p.o_f32 + orow);
    d32[0] = make_float4(f[0], f[1], f[2], f[3]);
    d32[1] = make_float4(f[4], f[5], f[6], f[7]);
  }
  if (p.lse && c8 == 0)
    p.lse[static_cast<size_t>(bh) * p.Nq + r] =
        seen ? (m + log2f(l) - 8.0f) * 0.69314718055994531f : -INFINITY;
}


}  // namespace

size_t attn_smem_bytes(int D) { return smem_bytes_for(D); }

namespace {
template <int D, bool DUMP, bool SPARSE>
cudaError_t prepare_one() {
  return cudaFuncSetAttribute(k_attn<D, DUMP, SPARSE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              static_cast<int>(smem_bytes_for(D)));
}
template <int D>
cudaError_t prepare_split() {
  cudaError_t e = cudaFuncSetAttribute(k_attn_split<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem_bytes_for(D)));
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(k_attn_win<D, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem_bytes_for(D)));
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(k_attn_win<D, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem_bytes_for(D)));
  return e;
}
}  // namespace

cudaError_t attn_prepare(int D) {
  cudaError_t e;
  if (D == 128) {
    e = prepare_one<128, false, false>();
    if (e == cudaSuccess) e = prepare_one<128, true, false>();
    if (e == cudaSuccess) e = prepare_one<128, false, true>();
    if (e == cudaSuccess) e = prepare_split<128>();
  } else {
    e = prepare_one<64, false, false>();
    if (e == cudaSuccess) e = prepare_one<64, true, false>();
    if (e == cudaSuccess) e = prepare_one<64, false, true>();
    if (e == cudaSuccess) e = prepare_split<64>();
  }
  return e;
}

cudaError_t launch_attn(const AttnMaps& maps, const AttnParams& p, cudaStream_t stream) {
  dim3 grid((p.Nq + BM - 1) / BM, p.BH);
  const bool sparse = p.bmask != nullptr;
  if (p.mask == kMaskSlidingWindow) {  // never block-sparse
    const size_t sm = smem_bytes_for(p.D);
    if (p.splits > 1) {
      grid.z = p.splits;
      if (p.D == 128) k_attn_win<128, true><<<grid, kThreads, sm, stream>>>(maps, p);
      else k_attn_win<64, true><<<grid, kThreads, sm, stream>>>(maps, p);
    } else {
      if (p.D == 128) k_attn_win<128, false><<<grid, kThreads, sm, stream>>>(maps, p);
      else k_attn_win<64, false><<<grid, kThreads, sm, stream>>>(maps, p);
    }
    return cudaGetLastError();
  }
  if (p.splits > 1) {  // split-KV partials; launch_attn_merge combines them
    grid.z = p.splits;
    if (p.D == 128) k_attn_split<128><<<grid, kThreads, smem_bytes_for(128), stream>>>(maps, p);
    else k_attn_split<64><<<grid, kThreads, smem_bytes_for(64), stream>>>(maps, p);
    return cudaGetLastError();
  }
  if (p.D == 128) {
    if (sparse) k_attn<128, false, true><<<grid, kThreads, smem_bytes_for(128), stream>>>(maps, p);
    else k_attn<128, false, false><<<grid, kThreads, smem_bytes_for(128), stream>>>(maps, p);
  } else {
    if (sparse) k_attn<64, false, true><<<grid, kThreads, smem_bytes_for(64), stream>>>(maps, p);
    else k_attn<64, false, false><<<grid, kThreads, smem_bytes_for(64), stream>>>(maps, p);
  }
  return cudaGetLastError();
}

cudaError_t launch_attn_dump(const AttnMaps& maps, const AttnParams& p, cudaStream_t stream) {
  if (p.D == 128)
    k_attn<128, true, false><<<1, kThreads, smem_bytes_for(128), stream>>>(maps, p);
  else
    k_attn<64, true, false><<<1, kThreads, smem_bytes_for(64), stream>>>(maps, p);
  return cudaGetLastError();
}

cudaError_t launch_attn_merge(const AttnParams& p, cudaStream_t stream) {
  dim3 grid((p.Nq + 7) / 8, p.BH);
  if (p.D == 128) k_attn_merge<128><<<grid, 128, 0, stream>>>(p);
  else k_attn_merge<64><<<grid, 128, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace sage
