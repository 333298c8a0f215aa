// attn.cuh -- launch interface of the fused quantized-attention kernel
// (sage_attn_fwd) and of its score-dump debug variant.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

namespace sage {

constexpr int kAttnBM = 128;  // query rows per CTA (tcgen05 M)
constexpr int kAttnBN = 128;  // keys per KV tile
// block-sparse mode: at most this many KV tiles (786432 keys) per head
constexpr int kAttnMaxKvTiles = 6144;

struct AttnParams {
  int BH, Nq, Nkv, D;
  int mask, mask_block;
  int nq_blocks, nkv_blocks;  // ceil(N / 64)
  const float* q_scale;       // [BH, nq_blocks]
  const float* k_scale;       // [BH, nkv_blocks]
  const float* v_scale;       // [BH, D]
  __nv_bfloat16* o;           // [BH, Nq, D]
  float* o_f32;               // [BH, Nq, D] or null
  float* lse;                 // [BH, Nq] or null
  float c0;                   // fp32(log2(e) / sqrt(D))
  long long budget;           // per-wait budget, SM cycles
  int* status;                // device status word pair
  // block-sparse mode (null: dense): uint8 [BH][n_qt][n_kt], tile (qt, kt)
  // visited only if non-zero
  const uint8_t* bmask;
  int n_qt, n_kt;
  // score-dump mode (debug): a single tile (bh, qt, kt), int32 [128, 128]
  int dbg_bh, dbg_qt, dbg_kt;
  int32_t* dbg_out;
};

struct AttnMaps {
  CUtensorMap q;  // int8 [BH][Nq_pad][D], box D x 128
  CUtensorMap k;  // int8 [BH][Nkv_pad][D], box D x 128
  CUtensorMap v;  // e4m3 [BH][Nkv_pad][D], box D x 128
};

size_t attn_smem_bytes(int D);
cudaError_t attn_prepare(int D);  // one-time function attributes
cudaError_t launch_attn(const AttnMaps& maps, const AttnParams& p, cudaStream_t stream);
cudaError_t launch_attn_dump(const AttnMaps& maps, const AttnParams& p, cudaStream_t stream);

}  // namespace sage
