// ceilings.cu -- microbenchmarks of the hardware rates that the kernels'
// rooflines rest on: the exp2 unit (MUFU), packed fp32x2 fma, the fp32 ->
// e4m3x2 conversion, an HBM copy, and the 5th-generation tensor core's
// kind::i8 and kind::f8f6f4 MMA throughput.
//
// Every kernel runs exactly one wave (its blocks are all co-resident) and
// each block records the SM clock cycles it spent (clock64 around its timed
// loop), so the host can state a rate per SM per clock that does not depend
// on the clock the GPU ran at; the caller's CUDA events give the whole-GPU
// rate at that clock.
#include <cuda_runtime.h>

#include <cstdint>

#include "ceilings.cuh"
#include "sm100.cuh"

namespace sage {
namespace {

constexpr int kCeilThreads = 256;
constexpr int kChains = 8;  // independent dependency chains per thread
enum : int { kSiteCeilMma = 0x30101 };

// written only when a never-true test passes: keeps the timed loops alive
__device__ float g_ceil_sink;

// exp2: x <- ex2(x) - 1.5 keeps every chain in (-1.5, 0.5].
__global__ void __launch_bounds__(kCeilThreads) k_ceil_ex2(int iters, long long* cycles) {
  float x[kChains];
#pragma unroll
  for (int e = 0; e < kChains; e++) x[e] = -1.0f + 1e-3f * static_cast<float>(threadIdx.x + e);
  __syncthreads();
  const long long t0 = clock64();
  // empty volatile statements pin the loop between the two clock reads: the
  // chains count as redefined after the first and as used before the second
#pragma unroll
  for (int e = 0; e < kChains; e++) asm volatile("" : "+f"(x[e]));
  for (int i = 0; i < iters; i++) {
#pragma unroll
    for (int e = 0; e < kChains; e++) x[e] = __fadd_rn(ex2_approx(x[e]), -1.5f);
  }
#pragma unroll
  for (int e = 0; e < kChains; e++) asm volatile("" ::"f"(x[e]));
  __syncthreads();
  const long long t1 = clock64();
  float acc = 0.0f;
#pragma unroll
  for (int e = 0; e < kChains; e++) acc += x[e];
  if (acc == 1234.5f) g_ceil_sink = acc;  // keeps the loop alive; never true
  if (threadIdx.x == 0) cycles[blockIdx.x] = t1 - t0;
}

// packed fp32x2 fma: x <- fma(x, 0.999, 1e-3) per lane pair, bounded.
__global__ void __launch_bounds__(kCeilThreads) k_ceil_ffma2(int iters, long long* cycles) {
  float2 x[kChains];
#pragma unroll
  for (int e = 0; e < kChains; e++)
    x[e] = make_float2(1e-3f * static_cast<float>(threadIdx.x + e), 0.5f);
  const float2 a = make_float2(0.999f, 0.999f), b = make_float2(1e-3f, 1e-3f);
  __syncthreads();
  const long long t0 = clock64();
#pragma unroll
  for (int e = 0; e < kChains; e++) asm volatile("" : "+f"(x[e].x), "+f"(x[e].y));
  for (int i = 0; i < iters; i++) {
#pragma unroll
    for (int e = 0; e < kChains; e++) x[e] = __ffma2_rn(x[e], a, b);
  }
#pragma unroll
  for (int e = 0; e < kChains; e++) asm volatile("" ::"f"(x[e].x), "f"(x[e].y));
  __syncthreads();
  const long long t1 = clock64();
  float acc = 0.0f;
#pragma unroll
  for (int e = 0; e < kChains; e++) acc += x[e].x + x[e].y;
  if (acc == 1234.5f) g_ceil_sink = acc;
  if (threadIdx.x == 0) cycles[blockIdx.x] = t1 - t0;
}

// fp32 pair -> e4m3x2 conversion; the codes are folded into an integer
// checksum and the inputs advance by one fp32 add per conversion.
__global__ void __launch_bounds__(kCeilThreads) k_ceil_cvt(int iters, long long* cycles) {
  float x[kChains];
  uint32_t h[kChains];
#pragma unroll
  for (int e = 0; e < kChains; e++) {
    x[e] = 1e-2f * static_cast<float>(threadIdx.x + e);
    h[e] = 0u;
  }
  __syncthreads();
  const long long t0 = clock64();
#pragma unroll
  for (int e = 0; e < kChains; e++) asm volatile("" : "+f"(x[e]), "+r"(h[e]));
  for (int i = 0; i < iters; i++) {
#pragma unroll
    for (int e = 0; e < kChains; e++) {
      h[e] ^= cvt_e4m3x2(x[e], -x[e]);
      x[e] = __fadd_rn(x[e], 0.25f);
    }
  }
#pragma unroll
  for (int e = 0; e < kChains; e++) asm volatile("" ::"r"(h[e]));
  __syncthreads();
  const long long t1 = clock64();
  uint32_t acc = 0u;
#pragma unroll
  for (int e = 0; e < kChains; e++) acc ^= h[e];
  if (acc == 0x12345678u) g_ceil_sink = static_cast<float>(acc);
  if (threadIdx.x == 0) cycles[blockIdx.x] = t1 - t0;
}

// HBM copy: 16-byte vector loads and stores, grid-stride over n16 vectors
// from src to dst (two halves of the scratch buffer).
__global__ void __launch_bounds__(kCeilThreads) k_ceil_copy(const uint4* __restrict__ src,
                                                             uint4* __restrict__ dst, size_t n16,
                                                             long long* cycles) {
  __syncthreads();
  const long long t0 = clock64();
  const size_t stride = static_cast<size_t>(gridDim.x) * kCeilThreads;
  size_t i = static_cast<size_t>(blockIdx.x) * kCeilThreads + threadIdx.x;
  for (; i + 3 * stride < n16; i += 4 * stride) {
    const uint4 a = src[i], b = src[i + stride], c = src[i + 2 * stride], d = src[i + 3 * stride];
    dst[i] = a;
    dst[i + stride] = b;
    dst[i + 2 * stride] = c;
    dst[i + 3 * stride] = d;
  }
  for (; i < n16; i += stride) dst[i] = src[i];
  asm volatile("" ::: "memory");
  __syncthreads();
  const long long t1 = clock64();
  if (threadIdx.x == 0) cycles[blockIdx.x] = t1 - t0;
}

// tcgen05 MMA rate: one CTA per SM (its shared-memory request keeps a second
// one off the SM); one thread issues `iters` groups of four K = 32 MMAs
// (M = 128, N = n, one 128-byte K row per operand row) into one TMEM
// accumulator, commits once and waits (bounded) for completion.  The
// operand tiles hold finite arbitrary codes.
struct CeilSmem {
  alignas(1024) uint8_t a[128 * 128];
  alignas(1024) uint8_t b[256 * 128];
  uint64_t done;
  uint32_t tmem_base;
  int abort;
};

template <bool F8>
__global__ void __launch_bounds__(128, 1) k_ceil_mma(int n, int iters, long long budget,
                                                     int* status, long long* cycles) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  CeilSmem& s = *reinterpret_cast<CeilSmem*>(smem_raw);
  if (smem_u32(smem_raw) & 1023u) {  // descriptors need 1024-byte aligned tiles
    if (threadIdx.x == 0) cycles[blockIdx.x] = -1;
    return;
  }
  const int warp = threadIdx.x >> 5;
  for (int i = threadIdx.x; i < 128 * 128; i += blockDim.x)
    s.a[i] = static_cast<uint8_t>((i * 37u + 11u) & 0x77u);  // e4m3: finite; i8: any
  for (int i = threadIdx.x; i < n * 128; i += blockDim.x)
    s.b[i] = static_cast<uint8_t>((i * 53u + 5u) & 0x77u);
  if (threadIdx.x == 0) {
    mbar_init(&s.done, 1);
    s.abort = 0;
    fence_mbar_init();
  }
  fence_proxy_async_smem();  // the generic-proxy writes above, for the tensor core
  if (warp == 0) {
    tmem_alloc(&s.tmem_base, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s.tmem_base;
  if (threadIdx.x == 0) {
    const WaitCtx w{budget, status, &s.abort};
    const uint32_t idesc = F8 ? idesc_e4m3_f32(128, n) : idesc_i8_s32(128, n);
    const uint32_t a0 = smem_u32(s.a), b0 = smem_u32(s.b);
    const long long t0 = clock64();
    for (int i = 0; i < iters; i++) {
#pragma unroll
      for (int kk = 0; kk < 4; kk++) {
        const uint64_t da = smem_desc_kmajor(a0 + kk * 32, 128);
        const uint64_t db = smem_desc_kmajor(b0 + kk * 32, 128);
        if (F8) mma_f8_ss(tmem, da, db, idesc, (i | kk) != 0);
        else mma_i8_ss(tmem, da, db, idesc, (i | kk) != 0);
      }
    }
    mma_commit(&s.done);
    if (!mbar_wait(&s.done, 0, w, kSiteCeilMma)) {
      // completion not seen within the budget: keep TMEM until the MMAs are
      // done (a second bounded wait), then report through the status word
      const long long d0 = clock64();
      while (!mbar_try_wait(&s.done, 0) && clock64() - d0 < budget) {
      }
    }
    cycles[blockIdx.x] = clock64() - t0;
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

}  // namespace

size_t ceiling_mma_smem_bytes() {
  // sizeof(CeilSmem) + 1024 alignment slack, raised so that one CTA fills
  // the SM's shared memory (one CTA per SM)
  return 160 * 1024;
}

cudaError_t launch_ceiling(const CeilingArgs& a, CeilingInfo* info, cudaStream_t stream) {
  int sms = 0, dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  const double thr = static_cast<double>(kCeilThreads);
  // Blocks per SM: as many as are co-resident (the occupancy calculator, for
  // the kernel's own register use), so that every block's clock64 span
  // covers the whole launch and ops_per_block x blocks_per_sm / cycles is a
  // per-SM rate.  Launching more blocks than are resident runs several waves,
  // each block spans only its own wave and that ratio over-counts the rate
  // by the number of waves.
  int per_sm = 0;
  const void* fn = a.kind == kCeilEx2     ? reinterpret_cast<const void*>(k_ceil_ex2)
                   : a.kind == kCeilFfma2 ? reinterpret_cast<const void*>(k_ceil_ffma2)
                   : a.kind == kCeilCvt   ? reinterpret_cast<const void*>(k_ceil_cvt)
                                          : reinterpret_cast<const void*>(k_ceil_copy);
  if (a.kind <= kCeilCopy) {
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, kCeilThreads, 0);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    per_sm = per_sm > 8 ? 8 : per_sm;  // the caller's cycles buffer holds 8 per SM
  }
  switch (a.kind) {
    case kCeilEx2:
    case kCeilFfma2:
    case kCeilCvt: {
      info->blocks = sms * per_sm;
      info->blocks_per_sm = per_sm;
      // results per block: ex2 = one exp2; ffma2 = two lanes of fma; cvt = one
      // e4m3x2 conversion (two values)
      const double per_iter = a.kind == kCeilFfma2 ? 2.0 * kChains : kChains;
      info->ops_per_block = thr * per_iter * a.iters;
      if (a.kind == kCeilEx2)
        k_ceil_ex2<<<info->blocks, kCeilThreads, 0, stream>>>(a.iters, a.cycles);
      else if (a.kind == kCeilFfma2)
        k_ceil_ffma2<<<info->blocks, kCeilThreads, 0, stream>>>(a.iters, a.cycles);
      else
        k_ceil_cvt<<<info->blocks, kCeilThreads, 0, stream>>>(a.iters, a.cycles);
      return cudaGetLastError();
    }
    case kCeilCopy: {
      info->blocks = sms * per_sm;
      info->blocks_per_sm = per_sm;
      const size_t n16 = a.scratch_bytes / 2 / 16;
      info->ops_per_block = 2.0 * 16.0 * static_cast<double>(n16) / info->blocks;  // bytes moved
      const uint4* src = static_cast<const uint4*>(a.scratch);
      uint4* dst = static_cast<uint4*>(a.scratch) + n16;
      k_ceil_copy<<<info->blocks, kCeilThreads, 0, stream>>>(src, dst, n16, a.cycles);
      return cudaGetLastError();
    }
    case kCeilMmaI8:
    case kCeilMmaF8: {
      info->blocks = sms;
      info->blocks_per_sm = 1;
      info->ops_per_block = 2.0 * 128.0 * a.n * 128.0 * a.iters;  // 4 MMAs of K = 32 per iter
      const int sm = static_cast<int>(ceiling_mma_smem_bytes());
      if (a.kind == kCeilMmaI8) {
        e = cudaFuncSetAttribute(k_ceil_mma<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, sm);
        if (e != cudaSuccess) return e;
        k_ceil_mma<false><<<sms, 128, sm, stream>>>(a.n, a.iters, a.budget, a.status, a.cycles);
      } else {
        e = cudaFuncSetAttribute(k_ceil_mma<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, sm);
        if (e != cudaSuccess) return e;
        k_ceil_mma<true><<<sms, 128, sm, stream>>>(a.n, a.iters, a.budget, a.status, a.cycles);
      }
      return cudaGetLastError();
    }
    default:
      return cudaErrorInvalidValue;
  }
}

}  // namespace sage
