// Pieces shared by the Newton-Schulz tensor-core kernels: thread layout,
// failure reporting, the Frobenius scale, and the epilogue's row, mirror and
// bf16 conversion helpers.
#pragma once

#include <cuda_bf16.h>

#include "muon_types.cuh"
#include "sm100_ptx.cuh"

namespace muonb200 {

constexpr int kEpiWarps = 8;                 // two per TMEM lane quadrant
constexpr int kNsThreads = 64 + 32 * kEpiWarps;
constexpr int kXposeLd = 34;                 // bf16 per row of a 32x32 block


__device__ __forceinline__ void record_failure(int32_t* err, int32_t code,
                                               volatile int* abort_flag) {
  atomicCAS(err, 0, code);
  *abort_flag = 1;
}

__device__ __forceinline__ float frob_scale(const MatDev* md,
                                            const float* __restrict__ partials,
                                            float eps) {
  float sum = 0.f;
  for (int i = 0; i < md->part_count; ++i) sum += partials[md->part_first + i];
  return 1.f / (sqrtf(sum) + eps);
}

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

// 32 fp32 -> bf16 into one row (only columns below `limit`).
__device__ __forceinline__ void store_row32_bf16(__nv_bfloat16* dst, int col0,
                                                 int limit,
                                                 const float (&v)[32]) {
  if (col0 + 32 <= limit) {
    uint4* p = reinterpret_cast<uint4*>(dst + col0);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      __nv_bfloat162 h[4];
#pragma unroll
      for (int i = 0; i < 4; ++i)
        h[i] = __floats2bfloat162_rn(v[8 * q + 2 * i], v[8 * q + 2 * i + 1]);
      p[q] = *reinterpret_cast<uint4*>(h);
    }
  } else {
#pragma unroll
    for (int e = 0; e < 32; ++e)
      if (col0 + e < limit) dst[col0 + e] = __float2bfloat16_rn(v[e]);
  }
}

// The mirrored 32 x 32 block: lane l holds row (row0 + l), columns
// col0..col0+31; the block is transposed through `buf` (per warp, 32 rows of
// kXposeLd bf16) and lane l then writes row (col0 + l) of the mirror,
// columns row0..row0+31, as four 16-byte stores.
__device__ __forceinline__ void store_mirror32_bf16(__nv_bfloat16* base, int ld,
                                                    int row0, int col0,
                                                    int limit, int lane,
                                                    __nv_bfloat16* buf,
                                                    const float (&v)[32]) {
  __nv_bfloat162* wrow = reinterpret_cast<__nv_bfloat162*>(buf + lane * kXposeLd);
#pragma unroll
  for (int i = 0; i < 16; ++i)
    wrow[i] = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
  __syncwarp();
  const int mrow = col0 + lane;
  if (mrow < limit) {
    __nv_bfloat16* dst = base + static_cast<size_t>(mrow) * ld + row0;
    if (row0 + 32 <= limit) {
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        __align__(16) __nv_bfloat16 h[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) h[k] = buf[(8 * q + k) * kXposeLd + lane];
        reinterpret_cast<uint4*>(dst)[q] = *reinterpret_cast<uint4*>(h);
      }
    } else {
      for (int k = 0; k < 32 && row0 + k < limit; ++k)
        dst[k] = buf[k * kXposeLd + lane];
    }
  }
  __syncwarp();
}

}  // namespace muonb200
