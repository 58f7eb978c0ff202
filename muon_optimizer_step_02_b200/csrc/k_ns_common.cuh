// Pieces shared by the Newton-Schulz tensor-core kernels: thread layout
// and the epilogue's row loader.
#pragma once

#include <cuda_bf16.h>

#include "muon_types.cuh"
#include "sm100_ptx.cuh"

namespace muonb200 {

constexpr int kEpiWarps = 8;                 // two per TMEM lane quadrant
constexpr int kNsThreads = 64 + 32 * kEpiWarps;



// 32 consecutive bf16 of one row -> fp32 (zeros beyond `limit` columns).
__device__ __forceinline__ void load_row32_bf16(const __nv_bfloat16* src,
                                                int col0, int limit,
                                                float (&v)[32]) {
  if (col0 + 32 <= limit) {
    const uint4* p = reinterpret_cast<const uint4*>(src + col0);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint4 raw = p[q];
      const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        v[8 * q + 2 * i] = __uint_as_float(w[i] << 16);
        v[8 * q + 2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
      }
    }
  } else {
#pragma unroll
    for (int e = 0; e < 32; ++e)
      v[e] = (col0 + e < limit) ? __bfloat162float(src[col0 + e]) : 0.f;
  }
}


}  // namespace muonb200
