// noalloc.cu -- sage_quant_qk_noalloc: the quantizer for callers that cannot
// allocate device memory.
//
// sage_quant_qk needs a caller-provided scratch workspace (fp64 K block sums,
// V block maxima, V inverse scales).  Some callers cannot provide one: code
// running where cudaMalloc is not allowed or not wanted, e.g. inside a
// region whose allocations are fixed in advance (a memory pool that has been
// sized and locked, a real-time loop that must not call into the allocator),
// or a plugin that receives only its input and output buffers from a host
// framework.  This entry point keeps that scratch in a fixed, file-scope
// device array instead, so the call itself allocates nothing.
//
// Limits and sharing rules (also in include/sage.h):
//   * the scratch is kSageNoallocScratchBytes (16 MiB); shapes whose
//     workspace (sage_quant_workspace_bytes) is larger are rejected with
//     SAGE_ERR_UNSUPPORTED before anything is enqueued;
//   * every GPU that loads the library holds this array until the process
//     exits;
//   * all calls on a device share the one array and it keeps the last call's
//     contents; nothing in it needs to start at zero (every cell the kernels
//     read is written earlier in the same call), but calls whose kernels
//     overlap on the GPU (different streams, no ordering between them) race
//     on it and give undefined results;
//   * the first call on a device looks up the array's device address
//     (cudaGetSymbolAddress, with that device current); make that first call
//     before any stream capture.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "quant.cuh"
#include "sage.h"

#define SAGE_EXPORT extern "C" __attribute__((visibility("default")))

namespace sage {
namespace {

constexpr size_t kSageNoallocScratchBytes = SAGE_NOALLOC_SCRATCH_BYTES;

// The scratch itself.  Host code must not pass `g_noalloc_scratch` to a
// kernel: on the host that name is only a stand-in for the symbol, not a
// device address.  The address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kSageNoallocScratchBytes];

constexpr int kMaxDevices = 64;

// Device address of g_noalloc_scratch per device, once looked up.
std::mutex g_scratch_mu;
unsigned char* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch on the current device; nullptr if the lookup
// failed.  Only a successful lookup is kept: a failure (which may be an
// unrelated error left by an earlier launch) is retried on the next call.
unsigned char* scratch_address() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) == cudaSuccess)
      g_scratch_ptr[dev] = static_cast<unsigned char*>(p);
  }
  return g_scratch_ptr[dev];
}

inline bool aligned16(const void* p) { return p && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace sage

using namespace sage;

SAGE_EXPORT sage_status sage_quant_qk_noalloc(const void* q_bf16, const void* k_bf16,
                                              const void* v_bf16, const sage_shape* shape,
                                              const sage_qkv_quant* out, void* stream) {
  const size_t need = sage_quant_workspace_bytes(shape);  // 0 for an invalid shape
  if (need == 0 || !out) return SAGE_ERR_INVALID_ARG;
  if (!aligned16(q_bf16) || !aligned16(k_bf16) || !aligned16(v_bf16)) return SAGE_ERR_INVALID_ARG;
  if (!aligned16(out->q_i8) || !aligned16(out->q_scale) || !aligned16(out->k_i8) ||
      !aligned16(out->k_scale) || !aligned16(out->k_mean) || !aligned16(out->v_f8) ||
      !aligned16(out->v_scale))
    return SAGE_ERR_INVALID_ARG;
  if (need > kSageNoallocScratchBytes) return SAGE_ERR_UNSUPPORTED;
  unsigned char* ws = scratch_address();
  if (!ws) return SAGE_ERR_CUDA;
  QuantArgs a{};
  a.q = static_cast<const uint16_t*>(q_bf16);
  a.k = static_cast<const uint16_t*>(k_bf16);
  a.v = static_cast<const uint16_t*>(v_bf16);
  a.BH = shape->B * shape->H;
  a.Nq = shape->Nq;
  a.Nkv = shape->Nkv;
  a.D = shape->D;
  a.q_i8 = out->q_i8;
  a.q_scale = out->q_scale;
  a.k_i8 = out->k_i8;
  a.k_scale = out->k_scale;
  a.k_mean = out->k_mean;
  a.v_f8 = out->v_f8;
  a.v_scale = out->v_scale;
  // same workspace layout as sage_quant_qk: fp64 K block sums, then f32 V
  // block maxima, then f32 V inverse scales
  const size_t cells = static_cast<size_t>(a.BH) * ((static_cast<size_t>(a.Nkv) + 63) / 64) * a.D;
  a.ws_ksum = reinterpret_cast<double*>(ws);
  a.ws_vmax = reinterpret_cast<float*>(ws + cells * 8);
  a.ws_vinv = reinterpret_cast<float*>(ws + cells * 12);
  a.Nkv_src = a.Nkv;
  a.kv_split = a.Nkv;
  a.kv_gap = 0;
  return launch_quant(a, static_cast<cudaStream_t>(stream)) == cudaSuccess ? SAGE_OK
                                                                           : SAGE_ERR_CUDA;
}
