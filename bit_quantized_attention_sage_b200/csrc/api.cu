// api.cu -- the C ABI declared in include/sage.h: argument validation, TMA
// descriptor encoding, kernel launches and the device status word.
//
// Nothing here allocates device memory: every buffer comes from the caller.
// No exception crosses the ABI; errors are returned as sage_status codes.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <mutex>

#include "attn.cuh"
#include "ceilings.cuh"
#include "quant.cuh"
#include "sage.h"
#include "w8a8.cuh"
#include "sm100.cuh"

#define SAGE_EXPORT extern "C" __attribute__((visibility("default")))

namespace sage {
namespace {

// {code, site} -- see WaitCtx.  One copy per device that loads the library.
__device__ int g_status[2];

constexpr long long kWaitBudget = 1ll << 31;  // ~1 s of SM clock per wait
constexpr int kMaxDevices = 64;

struct DeviceState {
  bool ready = false;     // set-up succeeded on this device
  int* status = nullptr;  // device address of g_status
};
DeviceState g_dev[kMaxDevices];
std::mutex g_dev_mu;

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static std::once_flag once;
  static EncodeTiledFn fn = nullptr;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// Per-device one-time setup: the status word's device address and the
// kernels' shared-memory attributes.  Only a complete, successful set-up is
// kept; after a failure (which may be an unrelated error left by an earlier
// launch) the next call tries again.
DeviceState* device_state() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  DeviceState& d = g_dev[dev];
  std::lock_guard<std::mutex> lock(g_dev_mu);
  if (!d.ready) {
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_status);
    if (e == cudaSuccess) e = attn_prepare(128);
    if (e == cudaSuccess) e = attn_prepare(64);
    if (e == cudaSuccess) e = w8a8_prepare();
    if (e != cudaSuccess) return nullptr;
    d.status = static_cast<int*>(p);
    d.ready = true;
  }
  return &d;
}

inline bool aligned16(const void* p) { return p && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline size_t pad64(int n) { return (static_cast<size_t>(n) + 63) / 64 * 64; }

bool shape_ok(const sage_shape* s) {
  if (!s) return false;
  if (s->B < 1 || s->H < 1 || s->Nq < 1 || s->Nkv < 1) return false;
  if (s->D != 64 && s->D != 128) return false;
  if (static_cast<long long>(s->B) * s->H > 65535) return false;
  if (s->Nq > (1 << 30) || s->Nkv > (1 << 30)) return false;
  return true;
}

void buffer_bytes(const sage_shape* s, size_t sz[7]) {
  const size_t bh = static_cast<size_t>(s->B) * s->H, D = s->D;
  sz[0] = bh * pad64(s->Nq) * D;         // q_i8
  sz[1] = bh * (pad64(s->Nq) / 64) * 4;  // q_scale
  sz[2] = bh * pad64(s->Nkv) * D;        // k_i8
  sz[3] = bh * (pad64(s->Nkv) / 64) * 4; // k_scale
  sz[4] = bh * D * 4;                    // k_mean
  sz[5] = bh * D * pad64(s->Nkv);        // v_f8
  sz[6] = bh * D * 4;                    // v_scale
}

size_t workspace_bytes(const sage_shape* s) {
  const size_t bh = static_cast<size_t>(s->B) * s->H, D = s->D;
  return bh * (pad64(s->Nkv) / 64) * D * 12 + bh * D * 4;
}

// sage_quant_qk_equalized: the base workspace, then the per-block channel
// maxima of |Q| and maxima and minima of K, then the factors 2^e and 2^-e.
size_t eq_workspace_bytes(const sage_shape* s) {
  const size_t bh = static_cast<size_t>(s->B) * s->H, D = s->D;
  return workspace_bytes(s) +
         bh * D * 4 * (pad64(s->Nq) / 64 + 2 * (pad64(s->Nkv) / 64) + 2);
}

bool qkv_ok(const sage_qkv_quant* q) {
  return q && aligned16(q->q_i8) && aligned16(q->q_scale) && aligned16(q->k_i8) &&
         aligned16(q->k_scale) && aligned16(q->k_mean) && aligned16(q->v_f8) &&
         aligned16(q->v_scale);
}

// 3-D tiled map over a contiguous uint8 array [d2][d1][d0] with a
// box0 x box1 x 1 box.
bool encode_u8_3d(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
                  uint32_t box0, uint32_t box1, CUtensorMapSwizzle sw) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {d0, d1, d2};
  const cuuint64_t strides[2] = {d0, d0 * d1};
  const cuuint32_t box[3] = {box0, box1, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// bf16 [rows][cols] matrix, row-major, box0 columns x box1 rows.
bool encode_bf16_2d(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows,
                    uint32_t box0, uint32_t box1, CUtensorMapSwizzle sw) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * 2};
  const cuuint32_t box[2] = {box0, box1};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_NONE,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_maps(const sage_qkv_quant* q, const sage_shape* s, AttnMaps* m) {
  const uint64_t bh = static_cast<uint64_t>(s->B) * s->H, D = s->D;
  const CUtensorMapSwizzle swqk =
      D == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  return encode_u8_3d(&m->q, q->q_i8, D, pad64(s->Nq), bh, static_cast<uint32_t>(D), kAttnBM,
                      swqk) &&
         encode_u8_3d(&m->k, q->k_i8, D, pad64(s->Nkv), bh, static_cast<uint32_t>(D), kAttnBN,
                      swqk) &&
         encode_u8_3d(&m->v, q->v_f8, D, pad64(s->Nkv), bh, static_cast<uint32_t>(D), kAttnBN,
                      swqk);
}

AttnParams base_params(const sage_qkv_quant* q, const sage_shape* s, const DeviceState* d) {
  AttnParams p{};
  p.BH = s->B * s->H;
  p.Nq = s->Nq;
  p.Nkv = s->Nkv;
  p.D = s->D;
  p.nq_blocks = static_cast<int>(pad64(s->Nq) / 64);
  p.nkv_blocks = static_cast<int>(pad64(s->Nkv) / 64);
  p.q_scale = q->q_scale;
  p.k_scale = q->k_scale;
  p.v_scale = q->v_scale;
  // fp32(log2(e) / sqrt(D)), the log2-domain softmax scale, rounded once
  p.c0 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(s->D)));
  p.budget = kWaitBudget;
  p.status = d->status;
  return p;
}

__global__ void k_timeout_probe(long long budget, int* status) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x != 0) return;
  mbar_init(&bar, 1);
  abort_flag = 0;
  fence_mbar_init();
  const WaitCtx w{budget, status, &abort_flag};
  // Nothing arrives on `bar`: the bounded wait must give up and report.
  (void)mbar_wait(&bar, 0, w, 0x7F001);
}

// Debug: the same e4m3 conversion and exp2 the kernels use, elementwise.
__global__ void k_e4m3(const float* x, uint8_t* y, size_t n) {
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<size_t>(gridDim.x) * blockDim.x)
    y[i] = static_cast<uint8_t>(cvt_e4m3x2(x[i], 0.0f) & 0xFF);
}

__global__ void k_exp2(const float* x, float* y, size_t n) {
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<size_t>(gridDim.x) * blockDim.x)
    y[i] = ex2_approx(x[i]);
}

}  // namespace
}  // namespace sage

using namespace sage;

SAGE_EXPORT int sage_abi_version(void) { return SAGE_ABI_VERSION; }

// ---------------------------------------------------------------- W8A8 linear layer

namespace {
bool w8a8_dims_ok(long long M, long long N, long long K) {
  return M >= 1 && N >= kW8a8BN && K >= kW8a8Group && N % kW8a8BN == 0 && K % kW8a8Group == 0 &&
         M <= (1ll << 31) - 1 && N <= (1 << 24) && K <= (1 << 24) &&
         ((M + kW8a8BM - 1) / kW8a8BM) * (N / kW8a8BN) <= (1ll << 31) - 1;
}
}  // namespace

SAGE_EXPORT sage_status sage_w8a8_quant_act(const void* x_bf16, long long M, long long K,
                                            int8_t* xq, float* sx, void* stream) {
  if (!w8a8_dims_ok(M, kW8a8BN, K) || !aligned16(x_bf16) || !aligned16(xq) || !sx ||
      (reinterpret_cast<uintptr_t>(sx) & 3u))
    return SAGE_ERR_INVALID_ARG;
  if (!device_state()) return SAGE_ERR_CUDA;
  return launch_w8a8_quant_act(static_cast<const uint16_t*>(x_bf16), static_cast<int>(M),
                               static_cast<int>(K), xq, sx,
                               static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? SAGE_OK
             : SAGE_ERR_CUDA;
}

SAGE_EXPORT sage_status sage_w8a8_quant_weight(const void* w_bf16, long long N, long long K,
                                               int8_t* wq, float* sw, void* stream) {
  if (!w8a8_dims_ok(1, N, K) || !aligned16(w_bf16) || !aligned16(wq) || !sw ||
      (reinterpret_cast<uintptr_t>(sw) & 3u))
    return SAGE_ERR_INVALID_ARG;
  if (!device_state()) return SAGE_ERR_CUDA;
  return launch_w8a8_quant_weight(static_cast<const uint16_t*>(w_bf16), static_cast<int>(N),
                                  static_cast<int>(K), wq, sw,
                                  static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? SAGE_OK
             : SAGE_ERR_CUDA;
}

namespace {
sage_status w8a8_gemm_common(const int8_t* xq, const float* sx, const int8_t* wq, const float* sw,
                             long long M, long long N, long long K, void* y_bf16, float* y_f32,
                             int8_t* q_i8, float* q_scale, void* stream) {
  DeviceState* d = device_state();
  if (!d) return SAGE_ERR_CUDA;
  W8a8Maps maps{};
  if (!encode_u8_3d(&maps.x, xq, K, M, 1, kW8a8Group, kW8a8BM, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_u8_3d(&maps.w, wq, K, N, 1, kW8a8Group, kW8a8BN, CU_TENSOR_MAP_SWIZZLE_128B) ||
      (y_bf16 && !encode_bf16_2d(&maps.y, y_bf16, N, M, 64, kW8a8BM, CU_TENSOR_MAP_SWIZZLE_128B)))
    return SAGE_ERR_CUDA;
  W8a8Params p{};
  p.M = static_cast<int>(M);
  p.N = static_cast<int>(N);
  p.K = static_cast<int>(K);
  p.sx = sx;
  p.sw = sw;
  p.y = static_cast<uint16_t*>(y_bf16);
  p.y_f32 = y_f32;
  p.q_i8 = q_i8;
  p.q_scale = q_scale;
  p.budget = kWaitBudget;
  p.status = d->status;
  return launch_w8a8_gemm(maps, p, static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? SAGE_OK
             : SAGE_ERR_CUDA;
}
}  // namespace

SAGE_EXPORT sage_status sage_w8a8_gemm(const int8_t* xq, const float* sx, const int8_t* wq,
                                       const float* sw, long long M, long long N, long long K,
                                       void* y_bf16, float* y_f32, void* stream) {
  if (!w8a8_dims_ok(M, N, K) || !aligned16(xq) || !aligned16(wq) || !aligned16(y_bf16) || !sx ||
      !sw || (y_f32 && !aligned16(y_f32)))
    return SAGE_ERR_INVALID_ARG;
  return w8a8_gemm_common(xq, sx, wq, sw, M, N, K, y_bf16, y_f32, nullptr, nullptr, stream);
}

SAGE_EXPORT sage_status sage_w8a8_gemm_q(const int8_t* xq, const float* sx, const int8_t* wq,
                                         const float* sw, long long M, long long N, long long K,
                                         void* y_bf16, int8_t* q_i8, float* q_scale,
                                         void* stream) {
  if (!w8a8_dims_ok(M, N, K) || !aligned16(xq) || !aligned16(wq) || !sx || !sw ||
      !aligned16(q_i8) || !q_scale || (reinterpret_cast<uintptr_t>(q_scale) & 3u) ||
      (y_bf16 && !aligned16(y_bf16)))
    return SAGE_ERR_INVALID_ARG;
  return w8a8_gemm_common(xq, sx, wq, sw, M, N, K, y_bf16, nullptr, q_i8, q_scale, stream);
}

SAGE_EXPORT const char* sage_status_string(sage_status st) {
  switch (st) {
    case SAGE_OK: return "ok";
    case SAGE_ERR_INVALID_ARG: return "invalid argument";
    case SAGE_ERR_UNSUPPORTED: return "unsupported";
    case SAGE_ERR_CUDA: return "CUDA error";
    case SAGE_ERR_TIMEOUT: return "device wait timed out";
  }
  return "unknown status";
}

SAGE_EXPORT sage_status sage_quant_buffer_bytes(const sage_shape* shape, size_t sizes[7]) {
  if (!shape_ok(shape) || !sizes) return SAGE_ERR_INVALID_ARG;
  buffer_bytes(shape, sizes);
  return SAGE_OK;
}

SAGE_EXPORT size_t sage_quant_workspace_bytes(const sage_shape* shape) {
  return shape_ok(shape) ? workspace_bytes(shape) : 0;
}

namespace {
// The keys a sliding-window step over a cache of `shape` attends to (the
// union over its query rows): [0, *n_sink) and [*lo, *hi), *lo >= *n_sink.
// The same row windows as the attention kernel's (queries are the newest Nq
// of the Nkv tokens).
void window_key_ranges(const sage_shape* s, int frame, int win, int sink, int* n_sink, int* lo,
                       int* hi) {
  const long long off = static_cast<long long>(s->Nkv) - s->Nq;
  const long long se = std::min<long long>(sink, s->Nkv);
  auto row = [&](long long g, long long* l, long long* h) {
    if (g < se) {
      *l = *h = se;
      return;
    }
    const long long f = (g - se) / frame;
    *l = se + std::max<long long>(f - win + 1, 0) * frame;
    *h = std::min<long long>(se + (f + 1) * frame, s->Nkv);
  };
  long long l0, h0, l1, h1;
  row(off, &l0, &h0);
  row(off + s->Nq - 1, &l1, &h1);
  *n_sink = static_cast<int>(se);
  *lo = static_cast<int>(std::max(l0, se));
  *hi = static_cast<int>(std::max(h1, std::max(l0, se)));
}

sage_status quant_common(const void* q_bf16, const void* k_bf16, const void* v_bf16,
                         const sage_shape* shape, const float* const rope[4],
                         const sage_qkv_quant* out, void* workspace, size_t ws_bytes,
                         void* stream, int nkv_src = -1, int kv_split = -1, int kv_gap = 0,
                         bool eq = false, int8_t* eq_exp = nullptr) {
  if (!shape_ok(shape) || !qkv_ok(out)) return SAGE_ERR_INVALID_ARG;
  if (!aligned16(q_bf16) || !aligned16(k_bf16) || !aligned16(v_bf16) || !aligned16(workspace))
    return SAGE_ERR_INVALID_ARG;
  if (ws_bytes < (eq ? eq_workspace_bytes(shape) : workspace_bytes(shape)))
    return SAGE_ERR_INVALID_ARG;
  if (rope)
    for (int i = 0; i < 4; i++)
      if (!aligned16(rope[i])) return SAGE_ERR_INVALID_ARG;
  if (!device_state()) return SAGE_ERR_CUDA;
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
  const size_t cells = static_cast<size_t>(a.BH) * (pad64(a.Nkv) / 64) * a.D;
  a.ws_ksum = static_cast<double*>(workspace);
  a.ws_vmax = reinterpret_cast<float*>(static_cast<char*>(workspace) + cells * 8);
  a.ws_vinv = reinterpret_cast<float*>(static_cast<char*>(workspace) + cells * 12);
  a.Nkv_src = nkv_src < 0 ? a.Nkv : nkv_src;
  a.kv_split = kv_split < 0 ? a.Nkv : kv_split;
  a.kv_gap = kv_gap;
  if (eq) {
    const size_t qcells = static_cast<size_t>(a.BH) * (pad64(a.Nq) / 64) * a.D;
    float* x = reinterpret_cast<float*>(static_cast<char*>(workspace) + workspace_bytes(shape));
    a.eq = true;
    a.ws_qmax = x;
    a.ws_kmax = x + qcells;
    a.ws_kmin = x + qcells + cells;
    a.ws_eq_up = x + qcells + 2 * cells;
    a.ws_eq_down = a.ws_eq_up + static_cast<size_t>(a.BH) * a.D;
    a.eq_exp = eq_exp;
  }
  if (rope) {
    a.q_cos = rope[0];
    a.q_sin = rope[1];
    a.k_cos = rope[2];
    a.k_sin = rope[3];
  }
  return launch_quant(a, static_cast<cudaStream_t>(stream)) == cudaSuccess ? SAGE_OK
                                                                           : SAGE_ERR_CUDA;
}
}  // namespace

SAGE_EXPORT sage_status sage_quant_qk(const void* q_bf16, const void* k_bf16, const void* v_bf16,
                                      const sage_shape* shape, const sage_qkv_quant* out,
                                      void* workspace, size_t ws_bytes, void* stream) {
  return quant_common(q_bf16, k_bf16, v_bf16, shape, nullptr, out, workspace, ws_bytes, stream);
}

SAGE_EXPORT size_t sage_quant_equalized_workspace_bytes(const sage_shape* shape) {
  return shape_ok(shape) ? eq_workspace_bytes(shape) : 0;
}

SAGE_EXPORT sage_status sage_quant_qk_equalized(const void* q_bf16, const void* k_bf16,
                                                const void* v_bf16, const sage_shape* shape,
                                                const sage_qkv_quant* out, int8_t* eq_exp,
                                                void* workspace, size_t ws_bytes, void* stream) {
  return quant_common(q_bf16, k_bf16, v_bf16, shape, nullptr, out, workspace, ws_bytes, stream, -1,
                      -1, 0, true, eq_exp);
}

SAGE_EXPORT sage_status sage_window_keys(const sage_shape* shape, int frame, int win, int sink,
                                         int* n_sink, int* lo, int* hi) {
  if (!shape_ok(shape) || !n_sink || !lo || !hi || frame < 1 || win < 1 || sink < 0 ||
      shape->Nkv < shape->Nq)
    return SAGE_ERR_INVALID_ARG;
  window_key_ranges(shape, frame, win, sink, n_sink, lo, hi);
  return SAGE_OK;
}

SAGE_EXPORT sage_status sage_quant_qk_window(const void* q_bf16, const void* k_cache,
                                             const void* v_cache, const sage_shape* cache_shape,
                                             int frame, int win, int sink, const float* q_cos,
                                             const float* q_sin, const float* k_cos,
                                             const float* k_sin, const sage_qkv_quant* out,
                                             void* workspace, size_t ws_bytes, void* stream) {
  if (!shape_ok(cache_shape) || frame < 1 || win < 1 || sink < 0 ||
      cache_shape->Nkv < cache_shape->Nq)
    return SAGE_ERR_INVALID_ARG;
  const int nrope = (q_cos != nullptr) + (q_sin != nullptr) + (k_cos != nullptr) + (k_sin != nullptr);
  if (nrope != 0 && nrope != 4) return SAGE_ERR_INVALID_ARG;
  int n_sink = 0, lo = 0, hi = 0;
  window_key_ranges(cache_shape, frame, win, sink, &n_sink, &lo, &hi);
  sage_shape g = *cache_shape;
  g.Nkv = n_sink + (hi - lo);
  if (g.Nkv < g.Nq) return SAGE_ERR_INVALID_ARG;
  const float* rope[4] = {q_cos, q_sin, k_cos, k_sin};
  return quant_common(q_bf16, k_cache, v_cache, &g, nrope ? rope : nullptr, out, workspace,
                      ws_bytes, stream, cache_shape->Nkv, n_sink, lo - n_sink);
}

SAGE_EXPORT sage_status sage_quant_qk_rope(const void* q_bf16, const void* k_bf16,
                                           const void* v_bf16, const sage_shape* shape,
                                           const float* q_cos, const float* q_sin,
                                           const float* k_cos, const float* k_sin,
                                           const sage_qkv_quant* out, void* workspace,
                                           size_t ws_bytes, void* stream) {
  const float* const rope[4] = {q_cos, q_sin, k_cos, k_sin};
  // the rotary kernels put the 64-token blocks on the grid's y dimension
  if (shape && shape_ok(shape) && (pad64(shape->Nq) / 64 > 65535 || pad64(shape->Nkv) / 64 > 65535))
    return SAGE_ERR_UNSUPPORTED;
  return quant_common(q_bf16, k_bf16, v_bf16, shape, rope, out, workspace, ws_bytes, stream);
}

namespace {
size_t split_ws_bytes(const sage_shape* s, int splits) {
  const size_t rows = static_cast<size_t>(s->B) * s->H * ((s->Nq + kAttnBM - 1) / kAttnBM) *
                      kAttnBM;
  return static_cast<size_t>(splits) * rows * (static_cast<size_t>(s->D) + 2) * 4;
}

// The sliding-window parameters (mask == kMaskSlidingWindow only).
struct WindowSpec {
  int frame, win, sink;
};

sage_status attn_common(const sage_qkv_quant* qkv, const sage_shape* shape, int mask,
                        int mask_block, const uint8_t* block_mask, void* o_bf16, float* o_f32,
                        float* lse, void* stream, int splits = 1, void* workspace = nullptr,
                        size_t ws_bytes = 0, WindowSpec ws = WindowSpec{1, 1, 0}) {
  if (!shape_ok(shape) || !qkv_ok(qkv) || !aligned16(o_bf16)) return SAGE_ERR_INVALID_ARG;
  if (o_f32 && !aligned16(o_f32)) return SAGE_ERR_INVALID_ARG;
  if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) return SAGE_ERR_INVALID_ARG;
  if (mask < SAGE_MASK_NONE || mask > kMaskSlidingWindow) return SAGE_ERR_INVALID_ARG;
  if (mask != SAGE_MASK_NONE && shape->Nkv < shape->Nq) return SAGE_ERR_INVALID_ARG;
  if (mask == SAGE_MASK_BLOCK_CAUSAL && mask_block < 1) return SAGE_ERR_INVALID_ARG;
  if (mask == kMaskSlidingWindow && (block_mask || ws.frame < 1 || ws.win < 1 || ws.sink < 0))
    return SAGE_ERR_INVALID_ARG;
  DeviceState* d = device_state();
  if (!d) return SAGE_ERR_CUDA;
  AttnMaps maps;
  if (!make_maps(qkv, shape, &maps)) return SAGE_ERR_CUDA;
  AttnParams p = base_params(qkv, shape, d);
  p.mask = mask;
  p.mask_block = mask == SAGE_MASK_BLOCK_CAUSAL ? mask_block : 1;
  if (mask == kMaskSlidingWindow) {
    // frames, windows or a reference context longer than the keys act as if
    // they were Nkv long; clamping keeps the kernel's key arithmetic in int
    p.mask_block = std::min(ws.frame, shape->Nkv);
    p.win = std::min(ws.win, shape->Nkv);
    p.sink = std::min(ws.sink, shape->Nkv);
  }
  p.o = static_cast<__nv_bfloat16*>(o_bf16);
  p.o_f32 = o_f32;
  p.lse = lse;
  p.bmask = block_mask;
  p.n_qt = (shape->Nq + kAttnBM - 1) / kAttnBM;
  p.n_kt = (shape->Nkv + kAttnBN - 1) / kAttnBN;
  if (splits > 1) {
    const size_t rows = static_cast<size_t>(p.BH) * p.n_qt * kAttnBM;
    p.splits = splits;
    p.part_o = static_cast<float*>(workspace);
    p.part_ml = reinterpret_cast<float*>(static_cast<char*>(workspace) +
                                         static_cast<size_t>(splits) * rows * shape->D * 4);
    if (launch_attn(maps, p, static_cast<cudaStream_t>(stream)) != cudaSuccess)
      return SAGE_ERR_CUDA;
    return launch_attn_merge(p, static_cast<cudaStream_t>(stream)) == cudaSuccess ? SAGE_OK
                                                                                 : SAGE_ERR_CUDA;
  }
  return launch_attn(maps, p, static_cast<cudaStream_t>(stream)) == cudaSuccess ? SAGE_OK
                                                                                : SAGE_ERR_CUDA;
}

bool public_mask(int mask) { return mask >= SAGE_MASK_NONE && mask <= SAGE_MASK_BLOCK_CAUSAL; }
}  // namespace

SAGE_EXPORT sage_status sage_attn_fwd(const sage_qkv_quant* qkv, const sage_shape* shape, int mask,
                                      int mask_block, void* o_bf16, float* o_f32, float* lse,
                                      void* stream) {
  if (!public_mask(mask)) return SAGE_ERR_INVALID_ARG;
  return attn_common(qkv, shape, mask, mask_block, nullptr, o_bf16, o_f32, lse, stream);
}

SAGE_EXPORT size_t sage_attn_split_workspace_bytes(const sage_shape* shape, int kv_splits) {
  if (!shape_ok(shape) || kv_splits < 1 || kv_splits > kAttnMaxSplits) return 0;
  return kv_splits == 1 ? 0 : split_ws_bytes(shape, kv_splits);
}

SAGE_EXPORT sage_status sage_attn_fwd_split(const sage_qkv_quant* qkv, const sage_shape* shape,
                                            int mask, int mask_block, int kv_splits,
                                            void* workspace, size_t workspace_bytes,
                                            void* o_bf16, float* o_f32, float* lse,
                                            void* stream) {
  if (!shape_ok(shape) || kv_splits < 1 || kv_splits > kAttnMaxSplits || !public_mask(mask))
    return SAGE_ERR_INVALID_ARG;
  if (kv_splits == 1)
    return attn_common(qkv, shape, mask, mask_block, nullptr, o_bf16, o_f32, lse, stream);
  if (!aligned16(workspace) || workspace_bytes < split_ws_bytes(shape, kv_splits))
    return SAGE_ERR_INVALID_ARG;
  return attn_common(qkv, shape, mask, mask_block, nullptr, o_bf16, o_f32, lse, stream,
                     kv_splits, workspace, workspace_bytes);
}

SAGE_EXPORT sage_status sage_attn_fwd_block_sparse(const sage_qkv_quant* qkv,
                                                   const sage_shape* shape, int mask,
                                                   int mask_block, const uint8_t* block_mask,
                                                   void* o_bf16, float* o_f32, float* lse,
                                                   void* stream) {
  if (!block_mask || !shape_ok(shape) || !public_mask(mask)) return SAGE_ERR_INVALID_ARG;
  if ((shape->Nkv + kAttnBN - 1) / kAttnBN > kAttnMaxKvTiles) return SAGE_ERR_UNSUPPORTED;
  return attn_common(qkv, shape, mask, mask_block, block_mask, o_bf16, o_f32, lse, stream);
}

SAGE_EXPORT sage_status sage_attn_fwd_window(const sage_qkv_quant* qkv, const sage_shape* shape,
                                             int frame_len, int window_frames, int sink_tokens,
                                             int kv_splits, void* workspace,
                                             size_t workspace_bytes, void* o_bf16, float* o_f32,
                                             float* lse, void* stream) {
  if (!shape_ok(shape) || kv_splits < 1 || kv_splits > kAttnMaxSplits)
    return SAGE_ERR_INVALID_ARG;
  const WindowSpec ws{frame_len, window_frames, sink_tokens};
  if (kv_splits == 1)
    return attn_common(qkv, shape, kMaskSlidingWindow, 0, nullptr, o_bf16, o_f32, lse, stream, 1,
                       nullptr, 0, ws);
  if (!aligned16(workspace) || workspace_bytes < split_ws_bytes(shape, kv_splits))
    return SAGE_ERR_INVALID_ARG;
  return attn_common(qkv, shape, kMaskSlidingWindow, 0, nullptr, o_bf16, o_f32, lse, stream,
                     kv_splits, workspace, workspace_bytes, ws);
}

SAGE_EXPORT sage_status sage_debug_qk_int32(const sage_qkv_quant* qkv, const sage_shape* shape,
                                            const int* tiles, int n_tiles, int32_t* out,
                                            void* stream) {
  if (!shape_ok(shape) || !qkv_ok(qkv) || !aligned16(out) || !tiles) return SAGE_ERR_INVALID_ARG;
  if (n_tiles < 0 || n_tiles > 65535) return SAGE_ERR_INVALID_ARG;
  const int bh = shape->B * shape->H;
  const int nqt = static_cast<int>((pad64(shape->Nq) + kAttnBM - 1) / kAttnBM);
  const int nkt = static_cast<int>((pad64(shape->Nkv) + kAttnBN - 1) / kAttnBN);
  for (int t = 0; t < n_tiles; t++) {
    const int* tt = tiles + 3 * t;
    if (tt[0] < 0 || tt[0] >= bh || tt[1] < 0 || tt[1] >= nqt || tt[2] < 0 || tt[2] >= nkt)
      return SAGE_ERR_INVALID_ARG;
  }
  DeviceState* d = device_state();
  if (!d) return SAGE_ERR_CUDA;
  AttnMaps maps;
  if (!make_maps(qkv, shape, &maps)) return SAGE_ERR_CUDA;
  AttnParams p = base_params(qkv, shape, d);
  p.mask_block = 1;
  for (int t = 0; t < n_tiles; t++) {
    p.dbg_bh = tiles[3 * t];
    p.dbg_qt = tiles[3 * t + 1];
    p.dbg_kt = tiles[3 * t + 2];
    p.dbg_out = out + static_cast<size_t>(t) * kAttnBM * kAttnBN;
    if (launch_attn_dump(maps, p, static_cast<cudaStream_t>(stream)) != cudaSuccess)
      return SAGE_ERR_CUDA;
  }
  return SAGE_OK;
}

SAGE_EXPORT sage_status sage_debug_timeout_probe(long long budget_cycles, void* stream) {
  if (budget_cycles < 1 || budget_cycles > (1ll << 40)) return SAGE_ERR_INVALID_ARG;
  DeviceState* d = device_state();
  if (!d) return SAGE_ERR_CUDA;
  k_timeout_probe<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(budget_cycles, d->status);
  return cudaGetLastError() == cudaSuccess ? SAGE_OK : SAGE_ERR_CUDA;
}

SAGE_EXPORT sage_status sage_debug_e4m3(const float* x, uint8_t* y, size_t n, void* stream) {
  if (!x || !y) return SAGE_ERR_INVALID_ARG;
  if (n == 0) return SAGE_OK;
  k_e4m3<<<1184, 256, 0, static_cast<cudaStream_t>(stream)>>>(x, y, n);
  return cudaGetLastError() == cudaSuccess ? SAGE_OK : SAGE_ERR_CUDA;
}

SAGE_EXPORT sage_status sage_debug_exp2(const float* x, float* y, size_t n, void* stream) {
  if (!x || !y) return SAGE_ERR_INVALID_ARG;
  if (n == 0) return SAGE_OK;
  k_exp2<<<1184, 256, 0, static_cast<cudaStream_t>(stream)>>>(x, y, n);
  return cudaGetLastError() == cudaSuccess ? SAGE_OK : SAGE_ERR_CUDA;
}

SAGE_EXPORT sage_status sage_ceiling(int kind, int iters, int n, void* scratch,
                                     size_t scratch_bytes, long long* cycles, int* blocks,
                                     int* blocks_per_sm, double* ops_per_block, void* stream) {
  if (!cycles || (reinterpret_cast<uintptr_t>(cycles) & 7u) || !blocks || !blocks_per_sm ||
      !ops_per_block)
    return SAGE_ERR_INVALID_ARG;
  if (kind < kCeilEx2 || kind > kCeilMmaF8) return SAGE_ERR_INVALID_ARG;
  if (kind == kCeilCopy) {
    if (!aligned16(scratch) || scratch_bytes < (1u << 20)) return SAGE_ERR_INVALID_ARG;
  } else if (iters < 1 || iters > (1 << 24)) {
    return SAGE_ERR_INVALID_ARG;
  }
  if ((kind == kCeilMmaI8 || kind == kCeilMmaF8) && n != 64 && n != 128 && n != 256)
    return SAGE_ERR_INVALID_ARG;
  DeviceState* d = device_state();
  if (!d) return SAGE_ERR_CUDA;
  CeilingArgs a{kind, iters, n, scratch, scratch_bytes, cycles, kWaitBudget, d->status};
  CeilingInfo info{};
  if (launch_ceiling(a, &info, static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return SAGE_ERR_CUDA;
  *blocks = info.blocks;
  *blocks_per_sm = info.blocks_per_sm;
  *ops_per_block = info.ops_per_block;
  return SAGE_OK;
}

SAGE_EXPORT sage_status sage_sync_status(void* stream) {
  DeviceState* d = device_state();
  if (!d) return SAGE_ERR_CUDA;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return SAGE_ERR_CUDA;
  int h[2] = {0, 0};
  if (cudaMemcpy(h, d->status, sizeof h, cudaMemcpyDeviceToHost) != cudaSuccess)
    return SAGE_ERR_CUDA;
  if (h[0] != 0) {
    const int z[2] = {0, 0};
    if (cudaMemcpy(d->status, z, sizeof z, cudaMemcpyHostToDevice) != cudaSuccess)
      return SAGE_ERR_CUDA;
    return static_cast<sage_status>(h[0]);
  }
  return SAGE_OK;
}
