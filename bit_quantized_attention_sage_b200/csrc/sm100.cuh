// sm100.cuh -- hand-written inline-PTX wrappers for the sm_100a features the
// kernels use: mbarriers with bounded waits, TMA tile loads, and the 5th
// generation tensor core (tcgen05: TMEM allocation, MMA, commit, TMEM
// loads/stores).  Written from the PTX ISA descriptions of these
// instructions.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace sage {

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// Bounded-wait context of a CTA.  `status` points to the library's device
// status word pair {code, site}: code 0 = ok, else a sage_status value (first
// writer wins); site says where the first failed wait was.  `abort` is a
// shared-memory flag that tells the CTA's other roles to stop waiting.
struct WaitCtx {
  long long budget;  // SM clock cycles per wait
  int* status;
  volatile int* abort;
};

__device__ __forceinline__ void record_timeout(int* status, int site) {
  if (atomicCAS(status, 0, 4 /* SAGE_ERR_TIMEOUT */) == 0) atomicExch(status + 1, site);
}

// ---------------------------------------------------------------- mbarrier

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(
                   smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Same test, but a thread whose phase is not complete is suspended in
// hardware until the phase completes or about `hint_ns` nanoseconds pass, so
// waiting warps do not take issue slots from the warps doing the work.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t* bar, uint32_t parity,
                                                    uint32_t hint_ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(hint_ns)
      : "memory");
  return ok != 0;
}

constexpr uint32_t kSleepHintNs = 200000;  // 0.2 ms per suspended try

// Bounded wait for the phase with the given parity to complete.  Gives up
// after w.budget SM clock cycles or as soon as *w.abort becomes non-zero
// (another role of the CTA gave up first).  Returns false if it gave up; a
// wait that runs out its own budget records SAGE_ERR_TIMEOUT with `site`.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, const WaitCtx& w,
                                          int site) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (true) {
    if (mbar_try_wait_sleep(bar, parity, kSleepHintNs)) return true;
    if (*w.abort) return false;
    if (clock64() - t0 > w.budget) {
      record_timeout(w.status, site);
      *w.abort = 1;
      return false;
    }
  }
}

// ---------------------------------------------------------------- TMA

__device__ __forceinline__ void tma_prefetch_desc(const void* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// 3-D tiled TMA load of one box into shared memory; completion is signalled
// as transaction bytes on `bar`.  Coordinates are element offsets, x
// innermost.  The box lands in this CTA's own shared memory only.
__device__ __forceinline__ void tma_load_3d(void* dst, const void* map, uint64_t* bar, int x,
                                            int y, int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z)
      : "memory");
}

// Prefetch one 3-D tile into L2 (no shared memory involved; coordinates
// outside the tensor are ignored).
__device__ __forceinline__ void tma_prefetch_l2_3d(const void* map, int x, int y, int z) {
  asm volatile("cp.async.bulk.prefetch.tensor.3d.L2.global.tile [%0, {%1, %2, %3}];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(x), "r"(y), "r"(z)
               : "memory");
}

// Make this thread's generic-proxy shared-memory writes visible to the async
// proxy (the tensor core reads operands through it).
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---------------------------------------------------------------- tcgen05

// Allocate `ncols` (power of two >= 32) TMEM columns; the whole warp must
// call it.  The TMEM address is written to *dst (shared memory).
__device__ __forceinline__ void tmem_alloc(uint32_t* dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(dst)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T with 8-bit signed integer operands and an
// int32 accumulator (kind::i8).  `accumulate` = 0 overwrites D.
__device__ __forceinline__ void mma_i8_ss(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Same with FP8/FP6/FP4 operands (here e4m3 x e4m3) and an fp32 accumulator.
__device__ __forceinline__ void mma_f8_ss(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Same with f16 operands (kind::f16, both A and B f16) and an fp32
// accumulator.
__device__ __forceinline__ void mma_f16_ss(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                           uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Shared-memory matrix descriptor with no swizzle and both byte offsets 0:
// every 8-row group and both 8-element K halves of a K = 16 f16 operand read
// the same 8 x 16-byte core matrix at saddr (a 128-byte broadcast tile).
__device__ __forceinline__ uint64_t smem_desc_bcast(uint32_t saddr) {
  return (uint64_t((saddr >> 4) & 0x3FFFu)) | (1ull << 46);
}
// Arrive once on `bar` when every MMA this thread issued so far has completed.
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}

// Instruction descriptor (kinds f16/tf32/f8f6f4/i8), dense, both operands
// K-major:  bits 4-5 accumulator format (1 = f32, 2 = s32), 7-9 A format,
// 10-12 B format (kind::i8: 1 = signed; kind::f8f6f4: 0 = e4m3),
// 17-22 N >> 3, 24-28 M >> 4.
__host__ __device__ constexpr uint32_t idesc_i8_s32(int M, int N) {
  return (2u << 4) | (1u << 7) | (1u << 10) | (uint32_t(N >> 3) << 17) |
         (uint32_t(M >> 4) << 24);
}
__host__ __device__ constexpr uint32_t idesc_e4m3_f32(int M, int N) {
  return (1u << 4) | (0u << 7) | (0u << 10) | (uint32_t(N >> 3) << 17) |
         (uint32_t(M >> 4) << 24);
}

// Instruction-descriptor bit 16: operand B is MN-major (N contiguous in
// shared memory) instead of K-major.  Valid for 8-bit (e4m3, e5m2, int8),
// 16-bit and tf32 operands.
constexpr uint32_t kIdescBMajorMN = 1u << 16;

// Shared-memory matrix descriptor for a K-major operand tile written by TMA
// with 128-byte (layout 2) or 64-byte (layout 4) swizzling: start address
// >> 4 in bits 0-13, leading byte offset (unused for swizzled K-major, 16 B)
// in 16-29, stride byte offset (distance between 8-row groups) >> 4 in
// 32-45, descriptor version 1 in 46-47, swizzle mode in 61-63.  The tile base
// must be aligned to the swizzle atom (8 rows x row bytes).
__device__ __forceinline__ uint64_t smem_desc_kmajor(uint32_t saddr, uint32_t row_bytes) {
  const uint64_t layout = (row_bytes == 128) ? 2ull : 4ull;
  const uint64_t sbo = (8ull * row_bytes) >> 4;
  return (uint64_t((saddr >> 4) & 0x3FFFu)) | (1ull << 16) | (sbo << 32) | (1ull << 46) |
         (layout << 61);
}

// Shared-memory matrix descriptor for an MN-major 8-bit operand tile written
// by TMA with 128-byte (N = 128 bytes per K row, layout 2) or 64-byte (N = 64
// bytes, layout 4) swizzling: the swizzle atom spans the whole N extent, so
// the leading byte offset (stride between atoms along N) is unused (16 B),
// and the stride byte offset is the distance between groups of 8 K rows.
// `saddr` is the first K row of the slice and must be atom aligned (8 rows).
__device__ __forceinline__ uint64_t smem_desc_mnmajor(uint32_t saddr, uint32_t row_bytes) {
  const uint64_t layout = (row_bytes == 128) ? 2ull : 4ull;
  const uint64_t sbo = (8ull * row_bytes) >> 4;
  return (uint64_t((saddr >> 4) & 0x3FFFu)) | (1ull << 16) | (sbo << 32) | (1ull << 46) |
         (layout << 61);
}

// TMEM loads: lane quadrant of the calling warp (32 lanes), `n` consecutive
// 32-bit columns per thread, followed by tcgen05.wait::ld inside the same asm
// statement so that no consumer of the registers can be scheduled before the
// data has arrived.
#define SAGE_R8(i) "=r"(r[i + 0]), "=r"(r[i + 1]), "=r"(r[i + 2]), "=r"(r[i + 3]), \
                   "=r"(r[i + 4]), "=r"(r[i + 5]), "=r"(r[i + 6]), "=r"(r[i + 7])

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : SAGE_R8(0), SAGE_R8(8), SAGE_R8(16), SAGE_R8(24)
      : "r"(taddr)
      : "memory");
}

__device__ __forceinline__ void tmem_ld64(uint32_t taddr, uint32_t (&r)[64]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x64.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,"
      "%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,"
      "%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%64];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : SAGE_R8(0), SAGE_R8(8), SAGE_R8(16), SAGE_R8(24), SAGE_R8(32), SAGE_R8(40),
        SAGE_R8(48), SAGE_R8(56)
      : "r"(taddr)
      : "memory");
}
#undef SAGE_R8

#define SAGE_W8(i) "r"(r[i + 0]), "r"(r[i + 1]), "r"(r[i + 2]), "r"(r[i + 3]), \
                   "r"(r[i + 4]), "r"(r[i + 5]), "r"(r[i + 6]), "r"(r[i + 7])
// TMEM store of 32 columns for the warp's lane quadrant, then wait::st.
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};\n\t"
      "tcgen05.wait::st.sync.aligned;" ::"r"(taddr),
      SAGE_W8(0), SAGE_W8(8), SAGE_W8(16), SAGE_W8(24)
      : "memory");
}
#undef SAGE_W8

// 128 consecutive 32-bit columns of the warp's lane quadrant: two x64 loads
// issued back to back and one wait::ld (a single TMEM round trip).
__device__ __forceinline__ void tmem_ld128(uint32_t taddr, uint32_t (&r)[128]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x64.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%128];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x64.b32 {%64,%65,%66,%67,%68,%69,%70,%71,%72,%73,%74,%75,%76,%77,%78,%79,%80,%81,%82,%83,%84,%85,%86,%87,%88,%89,%90,%91,%92,%93,%94,%95,%96,%97,%98,%99,%100,%101,%102,%103,%104,%105,%106,%107,%108,%109,%110,%111,%112,%113,%114,%115,%116,%117,%118,%119,%120,%121,%122,%123,%124,%125,%126,%127}, [%129];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]), "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]), "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]), "=r"(r[48]), "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]), "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63]), "=r"(r[64]), "=r"(r[65]), "=r"(r[66]), "=r"(r[67]), "=r"(r[68]), "=r"(r[69]), "=r"(r[70]), "=r"(r[71]), "=r"(r[72]), "=r"(r[73]), "=r"(r[74]), "=r"(r[75]), "=r"(r[76]), "=r"(r[77]), "=r"(r[78]), "=r"(r[79]), "=r"(r[80]), "=r"(r[81]), "=r"(r[82]), "=r"(r[83]), "=r"(r[84]), "=r"(r[85]), "=r"(r[86]), "=r"(r[87]), "=r"(r[88]), "=r"(r[89]), "=r"(r[90]), "=r"(r[91]), "=r"(r[92]), "=r"(r[93]), "=r"(r[94]), "=r"(r[95]), "=r"(r[96]), "=r"(r[97]), "=r"(r[98]), "=r"(r[99]), "=r"(r[100]), "=r"(r[101]), "=r"(r[102]), "=r"(r[103]), "=r"(r[104]), "=r"(r[105]), "=r"(r[106]), "=r"(r[107]), "=r"(r[108]), "=r"(r[109]), "=r"(r[110]), "=r"(r[111]), "=r"(r[112]), "=r"(r[113]), "=r"(r[114]), "=r"(r[115]), "=r"(r[116]), "=r"(r[117]), "=r"(r[118]), "=r"(r[119]), "=r"(r[120]), "=r"(r[121]), "=r"(r[122]), "=r"(r[123]), "=r"(r[124]), "=r"(r[125]), "=r"(r[126]), "=r"(r[127])
      : "r"(taddr), "r"(taddr + 64u)
      : "memory");
}

// Store 128 columns (two x64 stores) without waiting; the caller issues
// tmem_wait_st() before the values may be read by the tensor core.
__device__ __forceinline__ void tmem_st128_nowait(uint32_t taddr, const uint32_t (&r)[128]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x64.b32 [%128], {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63};\n\t"
      "tcgen05.st.sync.aligned.32x32b.x64.b32 [%129], {%64,%65,%66,%67,%68,%69,%70,%71,%72,%73,%74,%75,%76,%77,%78,%79,%80,%81,%82,%83,%84,%85,%86,%87,%88,%89,%90,%91,%92,%93,%94,%95,%96,%97,%98,%99,%100,%101,%102,%103,%104,%105,%106,%107,%108,%109,%110,%111,%112,%113,%114,%115,%116,%117,%118,%119,%120,%121,%122,%123,%124,%125,%126,%127};" ::"r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31]), "r"(r[32]), "r"(r[33]), "r"(r[34]), "r"(r[35]), "r"(r[36]), "r"(r[37]), "r"(r[38]), "r"(r[39]), "r"(r[40]), "r"(r[41]), "r"(r[42]), "r"(r[43]), "r"(r[44]), "r"(r[45]), "r"(r[46]), "r"(r[47]), "r"(r[48]), "r"(r[49]), "r"(r[50]), "r"(r[51]), "r"(r[52]), "r"(r[53]), "r"(r[54]), "r"(r[55]), "r"(r[56]), "r"(r[57]), "r"(r[58]), "r"(r[59]), "r"(r[60]), "r"(r[61]), "r"(r[62]), "r"(r[63]), "r"(r[64]), "r"(r[65]), "r"(r[66]), "r"(r[67]), "r"(r[68]), "r"(r[69]), "r"(r[70]), "r"(r[71]), "r"(r[72]), "r"(r[73]), "r"(r[74]), "r"(r[75]), "r"(r[76]), "r"(r[77]), "r"(r[78]), "r"(r[79]), "r"(r[80]), "r"(r[81]), "r"(r[82]), "r"(r[83]), "r"(r[84]), "r"(r[85]), "r"(r[86]), "r"(r[87]), "r"(r[88]), "r"(r[89]), "r"(r[90]), "r"(r[91]), "r"(r[92]), "r"(r[93]), "r"(r[94]), "r"(r[95]), "r"(r[96]), "r"(r[97]), "r"(r[98]), "r"(r[99]), "r"(r[100]), "r"(r[101]), "r"(r[102]), "r"(r[103]), "r"(r[104]), "r"(r[105]), "r"(r[106]), "r"(r[107]), "r"(r[108]), "r"(r[109]), "r"(r[110]), "r"(r[111]), "r"(r[112]), "r"(r[113]), "r"(r[114]), "r"(r[115]), "r"(r[116]), "r"(r[117]), "r"(r[118]), "r"(r[119]), "r"(r[120]), "r"(r[121]), "r"(r[122]), "r"(r[123]), "r"(r[124]), "r"(r[125]), "r"(r[126]), "r"(r[127]),
      "r"(taddr), "r"(taddr + 64u)
      : "memory");
}

// Store 64 columns (one x64 store) without waiting; the caller issues
// tmem_wait_st() before the values may be read by the tensor core.
__device__ __forceinline__ void tmem_st64_nowait(uint32_t taddr, const uint32_t (&r)[64]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x64.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63,%64};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31]), "r"(r[32]), "r"(r[33]), "r"(r[34]), "r"(r[35]), "r"(r[36]), "r"(r[37]), "r"(r[38]), "r"(r[39]), "r"(r[40]), "r"(r[41]), "r"(r[42]), "r"(r[43]), "r"(r[44]), "r"(r[45]), "r"(r[46]), "r"(r[47]), "r"(r[48]), "r"(r[49]), "r"(r[50]), "r"(r[51]), "r"(r[52]), "r"(r[53]), "r"(r[54]), "r"(r[55]), "r"(r[56]), "r"(r[57]), "r"(r[58]), "r"(r[59]), "r"(r[60]), "r"(r[61]), "r"(r[62]), "r"(r[63])
      : "memory");
}

// Fill 32 columns with one value as four x8 stores, without waiting.
__device__ __forceinline__ void tmem_fill32_x8_nowait(uint32_t taddr, uint32_t v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0+0], {%1,%1,%1,%1,%1,%1,%1,%1};\n\t"
      "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0+8], {%1,%1,%1,%1,%1,%1,%1,%1};\n\t"
      "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0+16], {%1,%1,%1,%1,%1,%1,%1,%1};\n\t"
      "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0+24], {%1,%1,%1,%1,%1,%1,%1,%1};\n\t" ::"r"(taddr), "r"(v)
      : "memory");
}

// Fill 128 columns with one value as sixteen x8 stores, without waiting
// (a store reads a run of consecutive registers, so narrow stores need only
// eight copies of the value).
__device__ __forceinline__ void tmem_fill128_x8_nowait(uint32_t taddr, uint32_t v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0+0], {%1,%1,%1,%1,%1,%1,%1,%1};\n\t"
      "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0+8], {%1,%1,%1,%1,%1,%1,%1,%1};\n\t"
      "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0+16], {%1,%1,%1,%1,%1,%1,%1,%1};\n\t"
      "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0+24], {%1,%1,%1,%1,%1,%1,%1,%1};\n\t"
      "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0+32], {%1,%1,%1,%1,%1,%1,%1,%1};\n\t"
      "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0+40], {%1,%1,%1,%1,%1,%1,%1,%1};\n\t"
      "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0+48], {%1,%1,%1,%1,%1,%1,%1,%1};\n\t"
      "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0+56], {%1,%1,%1,%1,%1,%1,%1,%1};\n\t"
      "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0+64], {%1,%1,%1,%1,%1,%1,%1,%1};\n\t"
      "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0+72], {%1,%1,%1,%1,%1,%1,%1,%1};\n\t"
      "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0+80], {%1,%1,%1,%1,%1,%1,%1,%1};\n\t"
      "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0+88], {%1,%1,%1,%1,%1,%1,%1,%1};\n\t"
      "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0+96], {%1,%1,%1,%1,%1,%1,%1,%1};\n\t"
      "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0+104], {%1,%1,%1,%1,%1,%1,%1,%1};\n\t"
      "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0+112], {%1,%1,%1,%1,%1,%1,%1,%1};\n\t"
      "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0+120], {%1,%1,%1,%1,%1,%1,%1,%1};\n\t" ::"r"(taddr), "r"(v)
      : "memory");
}

// Fill 128 columns with one value (four x32 stores), without waiting.
__device__ __forceinline__ void tmem_fill128_nowait(uint32_t taddr, uint32_t v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%4,%4,%4,%4,%4,%4,%4,%4,%4,%4,%4,%4,%4,%4,%4,%4,%4,%4,%4,%4,%4,%4,%4,%4,%4,%4,%4,%4,%4,%4,%4,%4};\n\t"
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%1], {%4,%4,%4,%4,%4,%4,%4,%4,%4,%4,%4,%4,%4,%4,%4,%4,%4,%4,%4,%4,%4,%4,%4,%4,%4,%4,%4,%4,%4,%4,%4,%4};\n\t"
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%2], {%4,%4,%4,%4,%4,%4,%4,%4,%4,%4,%4,%4,%4,%4,%4,%4,%4,%4,%4,%4,%4,%4,%4,%4,%4,%4,%4,%4,%4,%4,%4,%4};\n\t"
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%3], {%4,%4,%4,%4,%4,%4,%4,%4,%4,%4,%4,%4,%4,%4,%4,%4,%4,%4,%4,%4,%4,%4,%4,%4,%4,%4,%4,%4,%4,%4,%4,%4};" ::"r"(taddr),
      "r"(taddr + 32u), "r"(taddr + 64u), "r"(taddr + 96u), "r"(v)
      : "memory");
}

__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// ---------------------------------------------------------------- math

// Three-input fp32 maximum (one instruction on sm_100).
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// Hardware base-2 exponential (MUFU), subnormal results flushed to zero.
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// The recipe's software exp2 of two arguments, evaluated on the fma pipes
// (the exp2 unit gives 16 results per clock per SM, half of what the 8-bit
// tensor core consumes at D = 128, so a share of the exponentials is taken
// off it).  Cody-Waite style reduction x = j + f with j = round-half-even(x)
// (adding and subtracting 1.5 * 2^23) and |f| <= 1/2; a degree-3 polynomial
// for 2^f whose coefficients were fitted for this library (minimax relative
// error on [-1/2, 1/2], 2^-13.7 including the fp32 Horner evaluation); 2^j
// added to the exponent field of the polynomial's bits.  x is first raised to
// -125 so that the exponent stays normal (a masked key's -inf gives
// 2^-125 p(0), whose e4m3 code is 0).  Every step is one fp32 operation
// rounded to nearest-even or an integer add, so a CPU evaluation of the same
// steps gives the same bits.
__device__ __forceinline__ float2 exp2_poly2(float2 x) {
  const float2 magic = make_float2(12582912.0f, 12582912.0f);  // 1.5 * 2^23
  const float2 nmagic = make_float2(-12582912.0f, -12582912.0f);
  const float2 neg1 = make_float2(-1.0f, -1.0f);
  const float2 c0 = make_float2(__uint_as_float(0x3f7ffb49u), __uint_as_float(0x3f7ffb49u));
  const float2 c1 = make_float2(__uint_as_float(0x3f31798du), __uint_as_float(0x3f31798du));
  const float2 c2 = make_float2(__uint_as_float(0x3e786f0du), __uint_as_float(0x3e786f0du));
  const float2 c3 = make_float2(__uint_as_float(0x3d61fbb0u), __uint_as_float(0x3d61fbb0u));
  const float2 xc = make_float2(fmaxf(x.x, -125.0f), fmaxf(x.y, -125.0f));
  const float2 t = __fadd2_rn(xc, magic);     // magic + j
  const float2 jf = __fadd2_rn(t, nmagic);    // j
  const float2 f = __ffma2_rn(jf, neg1, xc);  // xc - j, exact
  float2 p = __ffma2_rn(c3, f, c2);
  p = __ffma2_rn(p, f, c1);
  p = __ffma2_rn(p, f, c0);
  return make_float2(__uint_as_float(__float_as_uint(p.x) + (__float_as_uint(t.x) << 23)),
                     __uint_as_float(__float_as_uint(p.y) + (__float_as_uint(t.y) << 23)));
}

// Four fp32 values to four e4m3 codes packed in one word, a in bits 0-7, b in
// 8-15, c in 16-23, d in 24-31 (round to nearest even, saturating to +-448):
// two pair conversions whose 16-bit results are joined in the same
// statement, so no separate byte permute is needed.
__device__ __forceinline__ uint32_t cvt_e4m3x4(float a, float b, float c, float d) {
  uint32_t r;
  asm("{\n\t.reg .b16 lo, hi;\n\t"
      "cvt.rn.satfinite.e4m3x2.f32 lo, %2, %1;\n\t"
      "cvt.rn.satfinite.e4m3x2.f32 hi, %4, %3;\n\t"
      "mov.b32 %0, {lo, hi};\n\t}"
      : "=r"(r)
      : "f"(a), "f"(b), "f"(c), "f"(d));
  return r;
}

// Two fp32 values to two e4m3 codes (round to nearest even, saturating to
// +-448): `lo` lands in bits 0-7, `hi` in bits 8-15.
__device__ __forceinline__ uint32_t cvt_e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

}  // namespace sage
