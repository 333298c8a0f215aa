// w8a8.cuh -- launch interface of the per-block W8A8 linear layer kernels
// (activation / weight quantization and the INT8 tensor-core GEMM with
// per-group fp32 promotion).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

namespace sage {

constexpr int kW8a8Group = 128;  // channels per quantization group along K
constexpr int kW8a8BM = 128;     // output rows per GEMM tile
constexpr int kW8a8BN = 128;     // output columns per GEMM tile (one weight block)

struct W8a8Params {
  int M, N, K;            // Y [M, N] = X [M, K] W [N, K]^T; N, K multiples of 128
  const float* sx;        // [M, K/128]
  const float* sw;        // [N/128, K/128]
  uint16_t* y;            // bf16 bits [M, N], or null when q_i8 is set
  float* y_f32;           // [M, N] or null
  // attention-Q output (null: none): Y read as Q of N/128 heads of D = 128
  // (column tile = head), rounded to bf16 and quantized like sage_quant_qk's
  // Q: int8 [N/128][M_pad][128] codes, per-64-token-block scales
  // [N/128][M_pad/64], M_pad = M rounded up to 64
  int8_t* q_i8;
  float* q_scale;
  long long budget;       // per-wait budget, SM cycles
  int* status;            // device status word pair
};

struct W8a8Maps {
  CUtensorMap x;  // int8 [M][K], box 128 x 128
  CUtensorMap w;  // int8 [N][K], box 128 x 128
  CUtensorMap y;  // bf16 [M][N], box 64 columns x 128 rows, 128-byte swizzle (stores)
};

cudaError_t w8a8_prepare();
cudaError_t launch_w8a8_quant_act(const uint16_t* x, int M, int K, int8_t* xq, float* sx,
                                  cudaStream_t stream);
cudaError_t launch_w8a8_quant_weight(const uint16_t* w, int N, int K, int8_t* wq, float* sw,
                                     cudaStream_t stream);
cudaError_t launch_w8a8_gemm(const W8a8Maps& maps, const W8a8Params& p, cudaStream_t stream);

}  // namespace sage
