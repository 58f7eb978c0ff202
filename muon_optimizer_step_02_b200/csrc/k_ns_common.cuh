// Pieces shared by the Newton-Schulz tensor-core kernels: thread layout
// and the epilogue's row loader.
#pragma once

#include <cuda_bf16.h>

#include "muon_types.cuh"
#include "sm100_ptx.cuh"

namespace muonb200 {

constexpr int kEpiWarps = 12;                // three per TMEM lane quadrant
constexpr int kEpiPerQuad = kEpiWarps / 4;
// Warpgroup 0: producer warp, MMA warp, completion-signal warp, one idle
// warp; warpgroups 1 to 3: the epilogue warps.
constexpr int kEpiWarp0 = 4;                 // first epilogue warp
constexpr int kNsThreads = 32 * (kEpiWarp0 + kEpiWarps);
// Register split after set-up (setmaxnreg): the launch gives every thread
// kNsRegsLaunch registers (512 threads x 128 = the SM's 65,536); warpgroup
// 0 returns all but kNsRegsControl and the three epilogue warpgroups take
// them, 128 x 56 + 384 x 152 = 65,536: the sum never exceeds what the block
// was launched with, so the increase cannot wait.
constexpr int kNsRegsLaunch = 128;
constexpr int kNsRegsControl = 56;
constexpr int kNsRegsEpilogue = 152;
static_assert(128 * kNsRegsControl + 32 * kEpiWarps * kNsRegsEpilogue <=
                  kNsThreads * kNsRegsLaunch,
              "register split exceeds the launch allocation");
static_assert(kEpiWarps % 4 == 0 && 32 * kEpiWarps % 128 == 0,
              "epilogue warps fill whole warpgroups, the same number per quadrant");



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

// Row segment src[col0 .. col0 + 32) of a bf16 row as raw bf16 pairs (zeros
// at and beyond `limit`); unpack_row32_bf16 widens it.
__device__ __forceinline__ void load_row32_bf16_raw(const __nv_bfloat16* src,
                                                    int col0, int limit,
                                                    uint4 (&r)[4]) {
  if (col0 + 32 <= limit) {
    const uint4* p = reinterpret_cast<const uint4*>(src + col0);
#pragma unroll
    for (int q = 0; q < 4; ++q) r[q] = p[q];
  } else {
    const uint16_t* h = reinterpret_cast<const uint16_t*>(src);
    uint32_t w[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const uint32_t lo = col0 + 2 * i < limit ? h[col0 + 2 * i] : 0u;
      const uint32_t hi = col0 + 2 * i + 1 < limit ? h[col0 + 2 * i + 1] : 0u;
      w[i] = lo | (hi << 16);
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) r[q] = make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
  }
}

__device__ __forceinline__ void unpack_row32_bf16(const uint4 (&r)[4], float (&v)[32]) {
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint32_t w[4] = {r[q].x, r[q].y, r[q].z, r[q].w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[8 * q + 2 * i] = __uint_as_float(w[i] << 16);
      v[8 * q + 2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
  }
}

}  // namespace muonb200
