// ceilings.cuh -- launch interface of the hardware-ceiling microbenchmarks
// (sage_ceiling).
#pragma once

#include <cuda_runtime.h>

#include <cstddef>

namespace sage {

enum : int {
  kCeilEx2 = 0,    // exp2 unit: ex2.approx.f32 results
  kCeilFfma2 = 1,  // packed fp32x2 fma lanes
  kCeilCvt = 2,    // fp32 pair -> e4m3x2 conversions
  kCeilCopy = 3,   // device memory copy: bytes read + written
  kCeilMmaI8 = 4,  // tcgen05 kind::i8 MMA, M 128, N n, K 32: 2 M N K operations each
  kCeilMmaF8 = 5,  // tcgen05 kind::f8f6f4 (e4m3) MMA, same shape
};

struct CeilingArgs {
  int kind;
  int iters;        // timed loop trip count (not used by the copy)
  int n;            // MMA N (64, 128 or 256)
  void* scratch;    // copy: source and destination halves
  size_t scratch_bytes;
  long long* cycles;  // device, one entry per block
  long long budget;   // bounded-wait budget (SM cycles)
  int* status;        // device status word pair
};

struct CeilingInfo {
  int blocks, blocks_per_sm;
  double ops_per_block;
};

size_t ceiling_mma_smem_bytes();
cudaError_t launch_ceiling(const CeilingArgs& a, CeilingInfo* info, cudaStream_t stream);

}  // namespace sage
