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
// split-KV mode: at most this many KV ranges per query tile
constexpr int kAttnMaxSplits = 16;

// mask ids: 0 none, 1 causal, 2 block-causal (block mask_block), 3 sliding
// window with a reference context (frames of mask_block tokens after `sink`
// reference tokens, `win` frames per window)
constexpr int kMaskSlidingWindow = 3;

struct AttnParams {
  int BH, Nq, Nkv, D;
  int mask, mask_block;
  int win, sink;              // sliding-window mask only (sink <= Nkv, mask_block <= Nkv)
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
  // split-KV mode (splits > 1): the KV tiles of each query tile in `splits`
  // ranges, one CTA each (grid z); every CTA writes its unnormalized O and
  // its running max and sum, which launch_attn_merge combines
  int splits;
  float* part_o;   // [splits][BH][n_qt * 128][D] fp32
  float* part_ml;  // [splits][BH][n_qt * 128][2]: m (log2 units), l
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
// the merge of a split-KV launch (same params): O, optional fp32 O and lse
cudaError_t launch_attn_merge(const AttnParams& p, cudaStream_t stream);

}  // namespace sage
