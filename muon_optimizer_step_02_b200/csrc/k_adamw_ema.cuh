// K-ADAMW-EMA: the AdamW step of the non-matrix parameters (embeddings,
// vectors, scalars) and the EMA of their updated values in one HBM pass:
//
//   M' = b1 M + (1 - b1) G
//   V' = b2 V + (1 - b2) G^2
//   P' = P (1 - lr wd) - lr (M' bc1) / (sqrt(V' bc2) + eps),
//        bc1 = 1 / (1 - b1^t), bc2 = 1 / (1 - b2^t)   (t = 1 for the first step)
//   E' = d E + (1 - d) P'
//
// Many tensors in one launch: the same flat space of 4-element units and
// segment table as the EMA kernel (binary search for the first segment, then
// a forward cursor).  Tensors whose five arrays are 16-byte aligned move as
// float4; the rest use scalar accesses.  Per element: P, M, V, E read and
// written, G read: 36 bytes.
//
// The step count t comes from the host, or from a device counter (the number
// of steps taken, t = counter + 1), which the host call advances afterwards
// with adamw_step_advance_kernel so that a captured graph serves every step.
//
// Source: PR #1893 "Record: L_ParallelResiduals_UNetSkips_DepthRecur_Muon_
// 1.0901", table "Architecture and training stack", rows "Optimizer" (AdamW
// on embeddings/scalars) and "EMA" (decay 0.9965).  The page gives no AdamW
// setting; the update is AdamW's published definition (decoupled weight
// decay, bias-corrected moments).
#pragma once

#include <cstdint>

namespace muonb200 {

constexpr int kAdamMaxSegs = 480;   // 480 x 56 bytes: 27 KB of kernel parameters (limit 32 KB)
constexpr int kAdamThreads = 256;

struct AdamSeg {
  float* p;
  const float* g;
  float* m;
  float* v;
  float* e;          // null: no EMA for this tensor
  long long numel;
  long long ubeg;    // first unit of this tensor in the flat unit space
};

struct AdamParams {
  AdamSeg seg[kAdamMaxSegs];
  long long total_units;
  const int32_t* step_dev;   // steps taken so far (t = *step_dev + 1), or null
  int32_t step;              // t when step_dev is null (>= 1)
  float lr, b1, b2, eps, wd, d;
  int32_t n_seg;
};

__device__ __forceinline__ void adamw_ema_one(float& p, float g, float& m, float& v,
                                              float* e, float omb1, float omb2, float bc1,
                                              float bc2, float decay_p, const AdamParams& a) {
  m = fmaf(a.b1, m, omb1 * g);
  v = fmaf(a.b2, v, omb2 * g * g);
  const float upd = (m * bc1) / (sqrtf(v * bc2) + a.eps);
  p = fmaf(p, decay_p, -a.lr * upd);
  if (e) *e = fmaf(a.d, *e, (1.f - a.d) * p);
}

__global__ void __launch_bounds__(kAdamThreads)
adamw_ema_kernel(const __grid_constant__ AdamParams a) {
  const int t = a.step_dev ? *a.step_dev + 1 : a.step;
  const float omb1 = 1.f - a.b1, omb2 = 1.f - a.b2;
  const float bc1 = 1.f / (1.f - powf(a.b1, static_cast<float>(t)));
  const float bc2 = 1.f / (1.f - powf(a.b2, static_cast<float>(t)));
  const float decay_p = 1.f - a.lr * a.wd;
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  const long long u0 = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  int lo = 0, hi = a.n_seg - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (a.seg[mid].ubeg <= u0) lo = mid; else hi = mid - 1;
  }
  int cur = lo;
  for (long long u = u0; u < a.total_units; u += stride) {
    while (cur + 1 < a.n_seg && u >= a.seg[cur + 1].ubeg) ++cur;
    const AdamSeg& s = a.seg[cur];
    const long long i0 = (u - s.ubeg) * 4;
    const bool vec = ((reinterpret_cast<uintptr_t>(s.p) | reinterpret_cast<uintptr_t>(s.g) |
                       reinterpret_cast<uintptr_t>(s.m) | reinterpret_cast<uintptr_t>(s.v) |
                       reinterpret_cast<uintptr_t>(s.e)) & 15u) == 0;
    if (vec && i0 + 4 <= s.numel) {
      float4 pv = __ldcs(reinterpret_cast<const float4*>(s.p + i0));
      const float4 gv = __ldcs(reinterpret_cast<const float4*>(s.g + i0));
      float4 mv = __ldcs(reinterpret_cast<const float4*>(s.m + i0));
      float4 vv = __ldcs(reinterpret_cast<const float4*>(s.v + i0));
      float4 ev = make_float4(0.f, 0.f, 0.f, 0.f);
      if (s.e) ev = __ldcs(reinterpret_cast<const float4*>(s.e + i0));
      float* ep = s.e ? &ev.x : nullptr;
      adamw_ema_one(pv.x, gv.x, mv.x, vv.x, ep, omb1, omb2, bc1, bc2, decay_p, a);
      adamw_ema_one(pv.y, gv.y, mv.y, vv.y, ep ? &ev.y : nullptr, omb1, omb2, bc1, bc2,
                    decay_p, a);
      adamw_ema_one(pv.z, gv.z, mv.z, vv.z, ep ? &ev.z : nullptr, omb1, omb2, bc1, bc2,
                    decay_p, a);
      adamw_ema_one(pv.w, gv.w, mv.w, vv.w, ep ? &ev.w : nullptr, omb1, omb2, bc1, bc2,
                    decay_p, a);
      __stcs(reinterpret_cast<float4*>(s.p + i0), pv);
      __stcs(reinterpret_cast<float4*>(s.m + i0), mv);
      __stcs(reinterpret_cast<float4*>(s.v + i0), vv);
      if (s.e) __stcs(reinterpret_cast<float4*>(s.e + i0), ev);
    } else {
      for (int k = 0; k < 4; ++k) {
        const long long i = i0 + k;
        if (i < s.numel)
          adamw_ema_one(s.p[i], s.g[i], s.m[i], s.v[i], s.e ? s.e + i : nullptr, omb1, omb2,
                        bc1, bc2, decay_p, a);
      }
    }
  }
}

// Advances a device step counter by one (after every launch of a call).
__global__ void adamw_step_advance_kernel(int32_t* step_dev) { *step_dev += 1; }

}  // namespace muonb200
