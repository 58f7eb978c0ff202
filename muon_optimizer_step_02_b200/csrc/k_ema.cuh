// K-EMA: E <- d E + (1 - d) P over many parameter tensors in one launch.
//
// The tensors form one flat space of 4-element units; each thread walks it
// with a grid stride, finds its first tensor by binary search in the segment
// table and then advances a cursor (units only increase), so a warp almost
// always works inside one tensor.  16-byte aligned tensors
// move as float4 (128-bit loads/stores); tails and unaligned tensors use
// scalar accesses.
//
// Source: PR #1893 "Record: L_ParallelResiduals_UNetSkips_DepthRecur_Muon_
// 1.0901", table "Architecture and training stack", row "EMA" (decay 0.9965);
// PR #1584 "Record: Improved Parallel Residuals + Systems Optimization",
// section "Summary" (batched EMA).
#pragma once

#include <cstdint>

namespace muonb200 {

constexpr int kEmaMaxSegs = 320;  // 10 KB of kernel parameters
constexpr int kEmaThreads = 256;

struct EmaSeg {
  float* e;
  const float* p;
  long long numel;
  long long ubeg;  // first unit of this tensor in the flat unit space
};

struct EmaParams {
  EmaSeg seg[kEmaMaxSegs];
  long long total_units;
  float d;
  float one_minus_d;
  int32_t n_seg;
};

__global__ void __launch_bounds__(kEmaThreads)
ema_update_kernel(const __grid_constant__ EmaParams p) {
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  const long long u0 = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  // last segment with ubeg <= u0
  int lo = 0, hi = p.n_seg - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (p.seg[mid].ubeg <= u0) lo = mid; else hi = mid - 1;
  }
  int cur = lo;
  for (long long u = u0; u < p.total_units; u += stride) {
    while (cur + 1 < p.n_seg && u >= p.seg[cur + 1].ubeg) ++cur;
    float* e = p.seg[cur].e;
    const float* q = p.seg[cur].p;
    const long long numel = p.seg[cur].numel;
    const long long i0 = (u - p.seg[cur].ubeg) * 4;
    const bool vec = ((reinterpret_cast<uintptr_t>(e) |
                       reinterpret_cast<uintptr_t>(q)) & 15u) == 0;
    if (vec && i0 + 4 <= numel) {
      float4 ev = __ldcs(reinterpret_cast<const float4*>(e + i0));
      const float4 pv = __ldcs(reinterpret_cast<const float4*>(q + i0));
      ev.x = fmaf(p.d, ev.x, p.one_minus_d * pv.x);
      ev.y = fmaf(p.d, ev.y, p.one_minus_d * pv.y);
      ev.z = fmaf(p.d, ev.z, p.one_minus_d * pv.z);
      ev.w = fmaf(p.d, ev.w, p.one_minus_d * pv.w);
      __stcs(reinterpret_cast<float4*>(e + i0), ev);
    } else {
      for (int k = 0; k < 4; ++k) {
        const long long i = i0 + k;
        if (i < numel) e[i] = fmaf(p.d, e[i], p.one_minus_d * q[i]);
      }
    }
  }
}

}  // namespace muonb200
