// w8a8.cu -- per-block W8A8 linear layer on sm_100a: Y = X W^T with INT8
// activations and weights (the 8-bit block-wise linear-layer quantization of
// the "Vidu S1" digest, section "Infra", and the TurboDiffusion notes' W8A8
// bullet: per-block scales because per-tensor and per-channel scales are
// stretched by outliers; the products run on INT8 tensor cores).
//
// Quantization (symmetric absmax/127, round-half-to-even, like the attention
// quantizer): one activation scale per token and 128-channel group, one
// weight scale per 128 x 128 block.
//
// GEMM: persistent, one CTA per SM looping over 128 x 128 output tiles (one
// weight block wide), 352 threads:
//   warp 0      TMA producer: the X and W tiles of two 128-channel groups per
//               step through a 3-stage shared-memory ring (128-byte swizzle).
//   warps 1-2   two MMA-issuing threads, alternating steps (warp 1 also
//               allocates 512 TMEM columns: four int32 accumulators of
//               128 x 128, one pair per step in flight).  Per group: one
//               kind::f16 MMA of a broadcast 128-byte tile (rows
//               [2048, 1024, 1024, 0, ...] read twice along K = 16: every
//               product sum is 2 (2^22 + 2^20 + 2^20) = 1.5 * 2^23) writes the
//               bit pattern 0x4B400000 into the accumulator; four
//               tcgen05.mma kind::i8 (K = 32 steps) add the group's exact
//               integer product P, so that it reads back as the fp32 value
//               1.5 * 2^23 + P.
//   warps 3-10  promotion: column part c (0-1) of lane quadrant q owns
//               output rows 32 q .. 32 q + 31 and columns 64 c .. 64 c + 63
//               (two warps per SM sub-partition).  Per step: load the pair's
//               scores, release the pair as soon as both groups are in
//               registers, and fold them into y = fma(P, sx * sw, y) in fp32
//               registers (packed fp32x2), in ascending group order.  At the
//               end: y -> bf16 (and optional fp32) rows.
// Every wait is bounded; on a timeout the CTA drains what it issued, frees
// TMEM and returns.
#include "w8a8.cuh"
#include "sm100.cuh"

#include <cuda_bf16.h>

namespace sage {

namespace {

constexpr int G = kW8a8Group;
constexpr int BM = kW8a8BM;
constexpr int BN = kW8a8BN;
constexpr int GPS = 2;           // 128-channel groups per pipeline step
constexpr int NS = 3;            // shared-memory stages (one step each)
constexpr int NACC = 4;          // TMEM accumulators (NACC / GPS steps in flight)
constexpr int NPAIR = NACC / GPS;
constexpr int kPromWarps = 8;    // two per lane quadrant, 64 columns each
constexpr int kPromCols = BN / (kPromWarps / 4);
constexpr int kIssuers = 2;      // MMA-issuing threads, alternating steps
constexpr int kFirstProm = 1 + kIssuers;  // warp index of the first promotion warp
constexpr int kThreads = 32 * (kFirstProm + kPromWarps);
constexpr int kTmemCols = 512;
constexpr uint32_t kFull = 0xffffffffu;
constexpr float kBias = 12582912.0f;  // 1.5 * 2^23, the accumulator seed

enum : int {
  kSiteProdEmpty = 0x20101, kSiteMmaFull, kSiteMmaAccFree, kSitePromFull, kSiteDrain,
  kSiteSmemAlign
};

// ---------------------------------------------------------------- quantizers

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ uint32_t q_i8x4(float a, float b, float c, float d, float inv) {
  auto q1 = [inv](float x) {
    int q = __float2int_rn(__fmul_rn(x, inv));
    q = q > 127 ? 127 : (q < -127 ? -127 : q);
    return static_cast<uint32_t>(static_cast<uint8_t>(static_cast<int8_t>(q)));
  };
  return q1(a) | (q1(b) << 8) | (q1(c) << 16) | (q1(d) << 24);
}

// One (token, 128-channel group) per 16 consecutive threads, 8 channels each.
__global__ void __launch_bounds__(256) k_w8a8_quant_act(const uint16_t* __restrict__ x, int M,
                                                         int K, int8_t* __restrict__ xq,
                                                         float* __restrict__ sx) {
  const int ngroups = K / G;
  const long long gid = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 4;
  const int sub = threadIdx.x & 15;
  const bool live = gid < static_cast<long long>(M) * ngroups;
  const long long m = live ? gid / ngroups : 0;
  const int g = live ? static_cast<int>(gid % ngroups) : 0;
  const size_t off = static_cast<size_t>(m) * K + static_cast<size_t>(g) * G + sub * 8;
  uint4 u = make_uint4(0, 0, 0, 0);
  if (live) u = __ldg(reinterpret_cast<const uint4*>(x + off));
  const float v[8] = {bf16_lo(u.x), bf16_hi(u.x), bf16_lo(u.y), bf16_hi(u.y),
                      bf16_lo(u.z), bf16_hi(u.z), bf16_lo(u.w), bf16_hi(u.w)};
  float a = 0.0f;
#pragma unroll
  for (int e = 0; e < 8; e++) a = fmaxf(a, fabsf(v[e]));
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(kFull, a, o));
  if (!live) return;
  const float inv = a == 0.0f ? 0.0f : __fdiv_rn(127.0f, a);
  if (sub == 0) sx[static_cast<size_t>(m) * ngroups + g] = a == 0.0f ? 0.0f : __fdiv_rn(a, 127.0f);
  *reinterpret_cast<uint2*>(xq + off) =
      make_uint2(q_i8x4(v[0], v[1], v[2], v[3], inv), q_i8x4(v[4], v[5], v[6], v[7], inv));
}

// One 128 x 128 weight block per CTA (256 threads, 8 chunks of 8 each).
__global__ void __launch_bounds__(256) k_w8a8_quant_weight(const uint16_t* __restrict__ w, int N,
                                                            int K, int8_t* __restrict__ wq,
                                                            float* __restrict__ sw) {
  __shared__ float red[8];
  const int ngroups = K / G;
  const int g = blockIdx.x, nb = blockIdx.y;
  constexpr int kChunks = G * G / 8 / 256;  // 8 chunks of 8 channels per thread
  float v[kChunks][8];
  float a = 0.0f;
#pragma unroll
  for (int c = 0; c < kChunks; c++) {
    const int chunk = c * 256 + threadIdx.x;
    const int r = chunk / (G / 8), col = (chunk % (G / 8)) * 8;
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(
        w + static_cast<size_t>(nb * BN + r) * K + static_cast<size_t>(g) * G + col));
    v[c][0] = bf16_lo(u.x); v[c][1] = bf16_hi(u.x); v[c][2] = bf16_lo(u.y); v[c][3] = bf16_hi(u.y);
    v[c][4] = bf16_lo(u.z); v[c][5] = bf16_hi(u.z); v[c][6] = bf16_lo(u.w); v[c][7] = bf16_hi(u.w);
#pragma unroll
    for (int e = 0; e < 8; e++) a = fmaxf(a, fabsf(v[c][e]));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(kFull, a, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = a;
  __syncthreads();
  a = red[0];
#pragma unroll
  for (int i = 1; i < 8; i++) a = fmaxf(a, red[i]);
  const float inv = a == 0.0f ? 0.0f : __fdiv_rn(127.0f, a);
  if (threadIdx.x == 0) sw[static_cast<size_t>(nb) * ngroups + g] = a == 0.0f ? 0.0f : __fdiv_rn(a, 127.0f);
#pragma unroll
  for (int c = 0; c < kChunks; c++) {
    const int chunk = c * 256 + threadIdx.x;
    const int r = chunk / (G / 8), col = (chunk % (G / 8)) * 8;
    *reinterpret_cast<uint2*>(wq + static_cast<size_t>(nb * BN + r) * K +
                              static_cast<size_t>(g) * G + col) =
        make_uint2(q_i8x4(v[c][0], v[c][1], v[c][2], v[c][3], inv),
                   q_i8x4(v[c][4], v[c][5], v[c][6], v[c][7], inv));
  }
}

// ---------------------------------------------------------------- GEMM

struct alignas(1024) GemmSmem {
  uint8_t x[NS][GPS][BM * G];  // int8 X tiles [group][128 rows][128 channels]
  uint8_t w[NS][GPS][BN * G];  // int8 W tiles [group][128 out channels][128 channels]
  // bf16 Y tile staging for the TMA store, one buffer per column part:
  // [128 rows][64 columns], 128-byte swizzled like the tensor map
  uint8_t ystage[kPromWarps / 4][BM * kPromCols * 2];
  float qmax[4][kPromWarps / 4];  // attention-Q mode: |Q| maxima per (quadrant, column part)
  uint8_t seed[128];           // f16 broadcast tile of the accumulator seed MMA
  uint64_t full[NS], empty[NS];
  uint64_t acc_full[NPAIR], acc_free[NPAIR];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};
static_assert(sizeof(GemmSmem) <= 227 * 1024, "shared memory of one CTA");

// TMA store of one 2-D tile from this CTA's shared memory, and the
// bulk-group bookkeeping of the issuing thread.
__device__ __forceinline__ void tma_store_2d(const void* map, const void* src, int x, int y) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.tile.bulk_group [%0, {%2, %3}], [%1];"
               ::"l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(src)), "r"(x), "r"(y)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// every committed store has finished reading shared memory / has completed
__device__ __forceinline__ void bulk_wait_read_all() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// Named barrier of `n` threads; the _or form returns, to every thread, whether
// `pred` held for any of them.
__device__ __forceinline__ void bar_sync_n(int id, int n) {
  asm volatile("barrier.cta.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}
__device__ __forceinline__ bool bar_or_n(int id, int n, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "barrier.cta.red.or.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(pred)), "r"(id), "r"(n)
      : "memory");
  return r != 0;
}

__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, const WaitCtx& w,
                                          int site) {
  return __all_sync(kFull, mbar_wait(bar, parity, w, site));
}

__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity, const WaitCtx& w) {
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > w.budget) {
      record_timeout(w.status, kSiteDrain);
      return;
    }
  }
}

// The output tiles of one CTA: t = blockIdx.x, blockIdx.x + gridDim.x, ...
// (one CTA per SM, persistent).  Column tiles run fastest, so that the CTAs
// in flight share their X rows (read once from HBM, then from L2) and sweep
// all of W (L2-resident).  Pipeline steps are numbered across the CTA's
// tiles (step J = tile i * nsteps + step j of the tile), so the stage ring
// and the accumulator pairs run on from one tile into the next.
struct TileSched {
  int ntn, ntiles, nsteps;
  __device__ __forceinline__ TileSched(const W8a8Params& p)
      : ntn(p.N / BN), ntiles(((p.M + BM - 1) / BM) * (p.N / BN)),
        nsteps((p.K / G + GPS - 1) / GPS) {}
  __device__ __forceinline__ int count() const {
    const int b = static_cast<int>(blockIdx.x), g = static_cast<int>(gridDim.x);
    return b < ntiles ? (ntiles - 1 - b) / g + 1 : 0;
  }
  __device__ __forceinline__ int tile(int i) const {
    return static_cast<int>(blockIdx.x) + i * static_cast<int>(gridDim.x);
  }
  __device__ __forceinline__ int m0(int i) const { return (tile(i) / ntn) * BM; }
  __device__ __forceinline__ int n0(int i) const { return (tile(i) % ntn) * BN; }
  __device__ __forceinline__ int total() const { return count() * nsteps; }
};

__device__ __forceinline__ void gemm_producer(GemmSmem& s, const W8a8Maps& maps,
                                              const TileSched& ts, int ngroups, const WaitCtx& w) {
  tma_prefetch_desc(&maps.x);
  tma_prefetch_desc(&maps.w);
  const int ntile = ts.count();
  int J = 0;  // pipeline step of the CTA
  for (int i = 0; i < ntile; i++) {
    const int m0 = ts.m0(i), n0 = ts.n0(i);
    bool ok = true;
    for (int j = 0; j < ts.nsteps; j++, J++) {
      const int st = J % NS;
      if (J >= NS && !mbar_wait(&s.empty[st], ((J / NS) & 1) ^ 1, w, kSiteProdEmpty)) {
        ok = false;
        break;
      }
      const int ng = min(GPS, ngroups - j * GPS);  // groups of this step
      mbar_arrive_expect_tx(&s.full[st], ng * (BM + BN) * G);
      for (int q = 0; q < ng; q++) {
        const int g = j * GPS + q;
        tma_load_3d(s.x[st][q], &maps.x, &s.full[st], g * G, m0, 0);
        tma_load_3d(s.w[st][q], &maps.w, &s.full[st], g * G, n0, 0);
      }
    }
    if (!ok) break;
  }
  // every issued load must land before the CTA exits (only the last NS can
  // still be in flight)
  for (int k = (J > NS ? J - NS : 0); k < J; k++) drain_wait(&s.full[k % NS], (k / NS) & 1, w);
}

// One thread per issuer: steps who, who + kIssuers, ...
__device__ __forceinline__ void gemm_mma(GemmSmem& s, uint32_t tmem, const TileSched& ts,
                                         int ngroups, const WaitCtx& w, int who) {
  constexpr uint32_t idesc = idesc_i8_s32(BM, BN);
  const int total = ts.total();
  const uint64_t seed = smem_desc_bcast(smem_u32(s.seed));
  // step J = who, who + kIssuers, ...; j = J mod nsteps kept without divisions
  int j = who;
  while (j >= ts.nsteps) j -= ts.nsteps;
  for (int J = who; J < total; J += kIssuers) {
    const int st = J % NS, pr = J % NPAIR;
    if (!mbar_wait(&s.full[st], (J / NS) & 1, w, kSiteMmaFull)) break;
    // the promotion warps have loaded this accumulator pair's previous step
    // (the first use waits for their initial release)
    if (!mbar_wait(&s.acc_free[pr], (J / NPAIR) & 1, w, kSiteMmaAccFree)) break;
    tc_fence_after();
    const int ng = min(GPS, ngroups - j * GPS);
    for (int q = 0; q < ng; q++) {
      const uint32_t xa = smem_u32(s.x[st][q]), wa = smem_u32(s.w[st][q]);
      const uint32_t acc = tmem + (pr * GPS + q) * BN;
      // seed: D = A B with A = B = the broadcast tile, 1.5 * 2^23 in every cell
      // (the f16 kind's instruction descriptor has the same fields as e4m3's)
      mma_f16_ss(acc, seed, seed, idesc_e4m3_f32(BM, BN), 0);
#pragma unroll
      for (int kk = 0; kk < G / 32; kk++)
        mma_i8_ss(acc, smem_desc_kmajor(xa + kk * 32, G), smem_desc_kmajor(wa + kk * 32, G), idesc,
                  1);
    }
    mma_commit(&s.empty[st]);
    mma_commit(&s.acc_full[pr]);
    j += kIssuers;
    while (j >= ts.nsteps) j -= ts.nsteps;
  }
  mma_commit(&s.drain);
  drain_wait(&s.drain, 0, w);
}

// A promotion warp's kPromCols accumulator columns.
template <int C>
__device__ __forceinline__ void load_cols(uint32_t taddr, uint32_t (&v)[C]) {
  if constexpr (C == 64) tmem_ld64(taddr, v);
  else tmem_ld32(taddr, v);
}

// Promotion warps: rows 32 q + lane, columns kPromCols * c .. + kPromCols - 1
// of each tile (q = lane quadrant, c = column part).
__device__ __forceinline__ void gemm_promote(GemmSmem& s, const W8a8Maps& maps, const W8a8Params& p,
                                             uint32_t tmem, const TileSched& ts, int ngroups,
                                             const WaitCtx& w) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int quad = warp & 3, part = (warp - kFirstProm) >> 2;
  // the first warp of a column part issues its TMA stores
  const bool storer = ((warp - kFirstProm) & 3) == 0 && lane == 0;
  const int bar_id = 1 + part;  // named barrier of the part's 4 warps (0 is __syncthreads)
  const bool qout = p.q_i8 != nullptr;  // attention-Q epilogue (barrier 3: all promotion warps)
  uint8_t* stg = s.ystage[part];
  const int r = quad * 32 + lane;
  const uint32_t tl = tmem + (static_cast<uint32_t>(quad * 32) << 16) + part * kPromCols;
  const float2 nb2 = make_float2(-kBias, -kBias);
  const int ntile = ts.count(), total = ts.total();

  // release every accumulator pair for its first step (the issuers seed
  // the accumulators themselves)
  tc_fence_before();
  __syncwarp();
  if (lane == 0)
    for (int pr = 0; pr < NPAIR; pr++) mbar_arrive(&s.acc_free[pr]);

  bool ok = true;
  int J = 0;
  for (int i = 0; i < ntile; i++) {
    const int m0 = ts.m0(i), m = m0 + r, n0 = ts.n0(i);
    const bool valid = m < p.M;
    const float* sxr = p.sx + static_cast<size_t>(valid ? m : 0) * ngroups;
    const float* swr = p.sw + static_cast<size_t>(n0 / BN) * ngroups;
    float2 y[kPromCols / 2];
#pragma unroll
    for (int e = 0; e < kPromCols / 2; e++) y[e] = make_float2(0.0f, 0.0f);
    float sxn = valid ? __ldg(sxr) : 0.0f, swn = __ldg(swr);
    for (int j = 0; j < ts.nsteps; j++, J++) {
      const int pr = J % NPAIR;
      if (!warp_wait(&s.acc_full[pr], (J / NPAIR) & 1, w, kSitePromFull)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const bool reuse = J + NPAIR < total;  // a later step fills this pair again
      const int ng = min(GPS, ngroups - j * GPS);
      for (int q = 0; q < ng; q++) {
        const int g = j * GPS + q;
        const uint32_t acc = tl + (pr * GPS + q) * BN;
        const float sc = __fmul_rn(sxn, swn);  // fp32(sx[m, g] * sw[n / 128, g])
        if (g + 1 < ngroups) {
          sxn = valid ? __ldg(sxr + g + 1) : 0.0f;
          swn = __ldg(swr + g + 1);
        }
        uint32_t v[kPromCols];  // 0x4B400000 + P
        load_cols(acc, v);
        if (q == ng - 1) {  // the pair is in registers: release it
          tc_fence_before();
          __syncwarp();
          if (reuse && lane == 0) mbar_arrive(&s.acc_free[pr]);
        }
        const float2 sc2 = make_float2(sc, sc);
#pragma unroll
        for (int e = 0; e < kPromCols / 2; e++) {
          const float2 pf = __fadd2_rn(make_float2(__uint_as_float(v[2 * e]), __uint_as_float(v[2 * e + 1])), nb2);
          y[e] = __ffma2_rn(pf, sc2, y[e]);
        }
      }
    }
    if (qout) {
      // attention-Q epilogue: every promotion warp leaves together after a
      // timeout anywhere (one 256-thread barrier for both column parts)
      if (storer) bulk_wait_read_all();
      if (bar_or_n(3, 32 * kPromWarps, !ok || *w.abort != 0)) break;
      float yb[kPromCols];  // Q = bf16(y) as floats
#pragma unroll
      for (int e = 0; e < kPromCols / 2; e++) {
        __nv_bfloat162 h2 = __floats2bfloat162_rn(y[e].x, y[e].y);
        yb[2 * e] = __low2float(h2);
        yb[2 * e + 1] = __high2float(h2);
      }
      if (p.y) {
        uint8_t* row = stg + r * (kPromCols * 2);
#pragma unroll
        for (int c = 0; c < kPromCols / 8; c++) {
          uint32_t pk[4];
#pragma unroll
          for (int e = 0; e < 4; e++) {
            __nv_bfloat162 h2 = __floats2bfloat162_rn(yb[8 * c + 2 * e], yb[8 * c + 2 * e + 1]);
            pk[e] = *reinterpret_cast<uint32_t*>(&h2);
          }
          *reinterpret_cast<uint4*>(row + ((c ^ (r & 7)) << 4)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        }
        fence_proxy_async_smem();
      }
      float a = 0.0f;  // |Q| max of this thread's valid values
      if (valid) {
#pragma unroll
        for (int e = 0; e < kPromCols; e += 2) a = fmax3(a, fabsf(yb[e]), fabsf(yb[e + 1]));
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(kFull, a, o));
      if (lane == 0) s.qmax[quad][part] = a;
      bar_sync_n(3, 32 * kPromWarps);
      if (storer && p.y) {
        tma_store_2d(&maps.y, stg, n0 + part * kPromCols, m0);
        bulk_commit();
      }
      // 64-token block b = rows 64 b .. 64 b + 63 of the tile: quadrants 2b, 2b + 1
      const int qb = quad >> 1;
      a = fmaxf(fmaxf(s.qmax[2 * qb][0], s.qmax[2 * qb][1]),
                fmaxf(s.qmax[2 * qb + 1][0], s.qmax[2 * qb + 1][1]));
      const float scale = (a == 0.0f) ? 0.0f : __fdiv_rn(a, 127.0f);
      const float inv = (a == 0.0f) ? 0.0f : __fdiv_rn(127.0f, a);
      const int mpad = (p.M + 63) / 64 * 64;
      const int head = n0 / BN;
      if (m < mpad) {  // rows past M within the padding get zero codes
        // code = round_half_even(Q * inv), |Q inv| <= 127 (1 + 2^-22), so no
        // clamp is needed; adding 1.5 * 2^23 rounds it into the low byte of
        // the fp32 bit pattern (0x4B400000 + code), which is packed directly
        // (the product is rounded on its own, as in the plain quantizer: the
        // scalar intrinsics are never contracted into an fma)
        uint32_t pk[kPromCols / 4];
#pragma unroll
        for (int c = 0; c < kPromCols / 4; c++) {
          uint32_t t[4];
#pragma unroll
          for (int e = 0; e < 4; e++)
            t[e] = __float_as_uint(__fadd_rn(__fmul_rn(yb[4 * c + e], inv), kBias));
          const uint32_t lo = __byte_perm(t[0], t[1], 0x0040);
          const uint32_t hi = __byte_perm(t[2], t[3], 0x0040);
          pk[c] = (valid && a != 0.0f) ? __byte_perm(lo, hi, 0x5410) : 0u;
        }
        uint4* dst = reinterpret_cast<uint4*>(p.q_i8 + (static_cast<size_t>(head) * mpad + m) * BN +
                                              part * kPromCols);
#pragma unroll
        for (int c = 0; c < kPromCols / 16; c++)
          dst[c] = make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
        if (part == 0 && (quad & 1) == 0 && lane == 0)
          p.q_scale[static_cast<size_t>(head) * (mpad / 64) + m / 64] = scale;
      }
      if (valid && p.y_f32) {
        float4* d32 = reinterpret_cast<float4*>(p.y_f32 + static_cast<size_t>(m) * p.N + n0 +
                                                part * kPromCols);
#pragma unroll
        for (int e = 0; e < kPromCols / 4; e++)
          d32[e] = make_float4(y[2 * e].x, y[2 * e].y, y[2 * e + 1].x, y[2 * e + 1].y);
      }
      continue;
    }
    // epilogue of this tile (the issuers already run the next tile's steps):
    // bf16 rows into the part's staging buffer, then one TMA store of the
    // 128 x 64 tile (rows past M are clipped by the tensor map)
    if (storer) bulk_wait_read_all();  // the previous tile's store has read the buffer
    bar_sync_n(bar_id, 128);
    if (ok) {
      uint8_t* row = stg + r * (kPromCols * 2);
#pragma unroll
      for (int c = 0; c < kPromCols / 8; c++) {  // 16-byte chunk c of the row, swizzled
        uint32_t pk[4];
#pragma unroll
        for (int e = 0; e < 4; e++) {
          __nv_bfloat162 h2 = __floats2bfloat162_rn(y[4 * c + e].x, y[4 * c + e].y);
          pk[e] = *reinterpret_cast<uint32_t*>(&h2);
        }
        *reinterpret_cast<uint4*>(row + ((c ^ (r & 7)) << 4)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
      }
    }
    fence_proxy_async_smem();
    // every warp of the part leaves together after a timeout anywhere
    if (bar_or_n(bar_id, 128, !ok || *w.abort != 0)) break;
    if (storer) {
      tma_store_2d(&maps.y, stg, n0 + part * kPromCols, m0);
      bulk_commit();
    }
    if (valid && p.y_f32) {
      float4* d32 = reinterpret_cast<float4*>(p.y_f32 + static_cast<size_t>(m) * p.N + n0 +
                                              part * kPromCols);
#pragma unroll
      for (int e = 0; e < kPromCols / 4; e++)
        d32[e] = make_float4(y[2 * e].x, y[2 * e].y, y[2 * e + 1].x, y[2 * e + 1].y);
    }
  }
  if (storer) bulk_wait_all();  // the stores are complete before the CTA exits
}

__global__ void __launch_bounds__(kThreads, 1)
    k_w8a8_gemm(const __grid_constant__ W8a8Maps maps, const W8a8Params p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if (smem_u32(smem_raw) & 1023u) {
    if (threadIdx.x == 0 && atomicCAS(p.status, 0, 3 /* SAGE_ERR_CUDA */) == 0)
      atomicExch(p.status + 1, kSiteSmemAlign);
    return;
  }
  GemmSmem& s = *reinterpret_cast<GemmSmem*>(smem_raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ngroups = p.K / G;
  const TileSched ts(p);
  if (threadIdx.x == 0) {
    for (int i = 0; i < NS; i++) {
      mbar_init(&s.full[i], 1);
      mbar_init(&s.empty[i], 1);
    }
    for (int i = 0; i < NPAIR; i++) {
      mbar_init(&s.acc_full[i], 1);
      mbar_init(&s.acc_free[i], kPromWarps);
    }
    mbar_init(&s.drain, kIssuers);
    s.abort = 0;
    fence_mbar_init();
  }
  if (threadIdx.x < 32) {  // seed tile: 8 rows of f16 [2048, 1024, 1024, 0, 0, 0, 0, 0]
    const uint32_t wv = (threadIdx.x & 3) == 0 ? 0x64006800u : (threadIdx.x & 3) == 1 ? 0x6400u : 0u;
    reinterpret_cast<uint32_t*>(s.seed)[threadIdx.x] = wv;
    fence_proxy_async_smem();
  }
  if (warp == 1) {
    tmem_alloc(&s.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s.tmem_base;
  const WaitCtx w{p.budget, p.status, &s.abort};
  if (warp == 0) {
    if (lane == 0) gemm_producer(s, maps, ts, ngroups, w);
  } else if (warp < kFirstProm) {
    if (lane == 0) gemm_mma(s, tmem, ts, ngroups, w, warp - 1);
  } else {
    gemm_promote(s, maps, p, tmem, ts, ngroups, w);
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

cudaError_t w8a8_prepare() {
  return cudaFuncSetAttribute(k_w8a8_gemm, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              static_cast<int>(sizeof(GemmSmem)));
}

cudaError_t launch_w8a8_quant_act(const uint16_t* x, int M, int K, int8_t* xq, float* sx,
                                  cudaStream_t stream) {
  const long long threads = static_cast<long long>(M) * (K / G) * 16;
  const unsigned blocks = static_cast<unsigned>((threads + 255) / 256);
  k_w8a8_quant_act<<<blocks, 256, 0, stream>>>(x, M, K, xq, sx);
  return cudaGetLastError();
}

cudaError_t launch_w8a8_quant_weight(const uint16_t* w, int N, int K, int8_t* wq, float* sw,
                                     cudaStream_t stream) {
  k_w8a8_quant_weight<<<dim3(K / G, N / BN), 256, 0, stream>>>(w, N, K, wq, sw);
  return cudaGetLastError();
}

cudaError_t launch_w8a8_gemm(const W8a8Maps& maps, const W8a8Params& p, cudaStream_t stream) {
  // one CTA per SM (the CTAs loop over the output tiles)
  static int sms[64] = {0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (sms[dev] == 0) {
    e = cudaDeviceGetAttribute(&sms[dev], cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
  }
  const long long ntiles = static_cast<long long>((p.M + BM - 1) / BM) * (p.N / BN);
  const int grid = static_cast<int>(ntiles < sms[dev] ? ntiles : sms[dev]);
  // the pipeline step counters of one CTA are ints
  const long long steps = (ntiles + grid - 1) / grid * ((p.K / G + GPS - 1) / GPS);
  if (steps > (1ll << 31) - 1) return cudaErrorInvalidValue;
  k_w8a8_gemm<<<grid, kThreads, sizeof(GemmSmem), stream>>>(maps, p);
  return cudaGetLastError();
}

}  // namespace sage
