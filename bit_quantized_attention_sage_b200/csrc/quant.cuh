// quant.cuh -- launch interface of the quantization kernels (sage_quant_qk).
#pragma once

#include <cuda_runtime.h>

#include <cstdint>

namespace sage {

struct QuantArgs {
  const uint16_t* q;  // bf16 bits [BH, Nq, D]
  const uint16_t* k;  // bf16 bits [BH, Nkv, D]
  const uint16_t* v;  // bf16 bits [BH, Nkv, D]
  int BH, Nq, Nkv, D;
  int8_t* q_i8;
  float* q_scale;
  int8_t* k_i8;
  float* k_scale;
  float* k_mean;
  uint8_t* v_f8;
  float* v_scale;
  double* ws_ksum;  // [BH, nkb, D] fp64 per-block K channel sums
  float* ws_vmax;   // [BH, nkb, D] per-block V channel maxima
  float* ws_vinv;   // [BH, D] 448 / channel absmax (0 for an all-zero channel)
  // rotation tables [Nq, D/2] / [Nkv, D/2] (cos, sin per token and channel
  // pair), shared by all (b, h); all four null: no rotation
  const float* q_cos;
  const float* q_sin;
  const float* k_cos;
  const float* k_sin;
  // K / V rows: gathered row r (r < Nkv) is input row r if r < kv_split,
  // else r + kv_gap, of Nkv_src rows per head (no gather: Nkv_src = Nkv,
  // kv_split = Nkv, kv_gap = 0)
  int Nkv_src, kv_split, kv_gap;
  // channel equalisation (sage_quant_qk_equalized; false: the recipe as is):
  // per-block channel maxima of |Q| [BH, nqb, D], maxima and minima of K
  // [BH, nkb, D], the per-channel factors 2^e and 2^-e [BH, D], and the
  // optional exponent output e [BH, D]
  bool eq;
  float* ws_qmax;
  float* ws_kmax;
  float* ws_kmin;
  float* ws_eq_up;
  float* ws_eq_down;
  int8_t* eq_exp;
};

cudaError_t launch_quant(const QuantArgs& a, cudaStream_t stream);

}  // namespace sage
