// K-CVT: fp32 -> bf16 (round to nearest, ties to even) over a flat array.
//
// Serves the sharded step's fp32 gradient reduction: the gradients of a
// bucket are reduce-scattered in fp32 (so an 8-way sum accumulates in fp32),
// and the owner rounds its summed segment once to the bf16 gradient the Muon
// step reads.  Eight elements per thread and iteration (two 16-byte loads,
// one 16-byte store) when both arrays are 16-byte aligned; scalar otherwise
// and for the tail.  Grid-stride, HBM-bound: 6 bytes per element.
//
// Context: PR #1893 "Record: L_ParallelResiduals_UNetSkips_DepthRecur_Muon_
// 1.0901", table "Architecture and training stack", row "Train context"
// (8-way data-parallel training); the pages print no reduction scheme.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

namespace muonb200 {

constexpr int kCvtThreads = 256;

__global__ void __launch_bounds__(kCvtThreads)
f32_to_bf16_kernel(uint16_t* __restrict__ dst, const float* __restrict__ src, long long n,
                   int vec) {
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  const long long tid = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  long long done = 0;
  if (vec) {
    const long long n8 = n / 8;
    for (long long i = tid; i < n8; i += stride) {
      const float4 a = __ldcs(reinterpret_cast<const float4*>(src) + 2 * i);
      const float4 b = __ldcs(reinterpret_cast<const float4*>(src) + 2 * i + 1);
      __nv_bfloat162 h[4] = {__floats2bfloat162_rn(a.x, a.y), __floats2bfloat162_rn(a.z, a.w),
                             __floats2bfloat162_rn(b.x, b.y), __floats2bfloat162_rn(b.z, b.w)};
      __stcs(reinterpret_cast<uint4*>(dst) + i, *reinterpret_cast<uint4*>(h));
    }
    done = n8 * 8;
  }
  for (long long i = done + tid; i < n; i += stride) {
    const __nv_bfloat16 v = __float2bfloat16_rn(src[i]);
    dst[i] = *reinterpret_cast<const uint16_t*>(&v);
  }
}

}  // namespace muonb200
