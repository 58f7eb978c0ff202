// The three tensor-core products of one Newton-Schulz step, as one persistent
// warp-specialised tcgen05 kernel over a tile list that spans every matrix of
// the batch (grouped launch):
//
//   gram  A  = s^2 X X^T             (upper tile pairs only; mirrored store)
//   poly  B' = a I + b A + c A A     (A symmetric, so A A = A A^T: same kernel)
//   apply X <- s B' X                (last step: W <- W (1 - lr wd) - lr scale O)
//
// X <- a X + B X is evaluated as (a I + B) X: one product, and the bf16 copy
// of B' carries the sum a + B on its diagonal instead of the cancelling pair.
//
// s = 1 / (||X~||_F + eps_frob) on the first step (the Frobenius
// normalisation folded into the products), 1 afterwards.
//
// Roles (192 threads): warp 0 issues TMA loads into a ring of shared-memory
// stages; warp 1 owns TMEM and issues tcgen05.mma (M = 128, N = BN, K = 16)
// from one thread; warps 2-5 drain the double-buffered TMEM accumulator and
// run the fused epilogue.  Every wait is bounded (see mbar_wait_bounded).
//
// Source of the step: PR #1396 "Record: Combined 3-Layer Recurrence +
// Parallel Residuals + Polar Express + Brotli", table "Techniques Combined",
// row "Polar Express Newton-Schulz" (per-step coefficients); PR #1584
// "Record: Improved Parallel Residuals + Systems Optimization", section
// "Summary" (fused Muon kernel).
#pragma once

#include <cuda_bf16.h>

#include "muon_types.cuh"
#include "sm100_ptx.cuh"

namespace muonb200 {

template <int BN, bool kBmn, int kStages>
struct NsCfg {
  static constexpr int kABytes = kTileM * kTileK * 2;
  static constexpr int kBBytes = BN * kTileK * 2;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kTmemCols = 2 * BN;
  static constexpr int kNumBars = 2 * kStages + 5;
  static constexpr size_t kSmemBytes =
      1024 + static_cast<size_t>(kStages) * kStageBytes + kNumBars * 8 + 16;
  static_assert(kTmemCols == 256 || kTmemCols == 512, "TMEM columns");
  static_assert(kSmemBytes <= 227 * 1024, "shared memory");
};

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

// Column `row` of the mirrored tile: element (row, col0+e) goes to
// (col0+e, row).  Lanes hold consecutive rows, so each store is coalesced
// across the warp.
__device__ __forceinline__ void store_col32_bf16(__nv_bfloat16* base, int ld,
                                                 int row, int col0, int limit,
                                                 const float (&v)[32]) {
#pragma unroll
  for (int e = 0; e < 32; ++e)
    if (col0 + e < limit)
      base[static_cast<size_t>(col0 + e) * ld + row] = __float2bfloat16_rn(v[e]);
}

template <int BN, bool kBmn, int kStages>
__global__ void __launch_bounds__(192, 1)
ns_gemm_kernel(const __grid_constant__ NsParams p) {
  using Cfg = NsCfg<BN, kBmn, kStages>;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kStages * Cfg::kStageBytes);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + Cfg::kNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const uint32_t smem0 = smem_addr(smem);
  auto sA = [&](int s) { return smem0 + s * Cfg::kStageBytes; };
  auto sB = [&](int s) { return smem0 + s * Cfg::kStageBytes + Cfg::kABytes; };
  auto full_bar = [&](int s) { return smem_addr(bars + s); };
  auto empty_bar = [&](int s) { return smem_addr(bars + kStages + s); };
  auto tfull_bar = [&](int a) { return smem_addr(bars + 2 * kStages + a); };
  auto tempty_bar = [&](int a) { return smem_addr(bars + 2 * kStages + 2 + a); };
  const uint32_t drain_bar = smem_addr(bars + 2 * kStages + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull_bar(a), 1);
      mbar_init(tempty_bar(a), 128);
    }
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_addr(tmem_slot), Cfg::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int it = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < p.n_tiles; t += gridDim.x) {
        const NsTile tl = p.tiles[t];
        const MatDev* md = p.mats + tl.mat;
        const CUtensorMap* tm_a;
        const CUtensorMap* tm_b;
        if (p.mode == kModeGram) {
          tm_a = &md->tm_xk[p.src];
          tm_b = tm_a;
        } else if (p.mode == kModePoly) {
          tm_a = &md->tm_a;
          tm_b = tm_a;
        } else {
          tm_a = &md->tm_b;
          tm_b = &md->tm_xn[p.src];
        }
        if (p.fresh) {
          tensormap_acquire(tm_a);
          if (tm_b != tm_a) tensormap_acquire(tm_b);
        }
        const int ay = tl.ti * kTileM;
        for (int kb = 0; kb < tl.kt; ++kb, ++it) {
          const int s = it % kStages;
          const uint32_t ph = (it / kStages) & 1;
          if (!mbar_wait_bounded(empty_bar(s), ph ^ 1u, abort_flag)) {
            record_failure(p.err, kErrTimeoutProducer, abort_flag);
            ok = false;
            break;
          }
          if (p.fault == 1 && blockIdx.x == 0 && it == 0) continue;  // test hook
          mbar_arrive_expect_tx(full_bar(s), Cfg::kStageBytes);
          tma_load_2d(sA(s), tm_a, full_bar(s), kb * kTileK, ay);
          if (!kBmn) {
            tma_load_2d(sB(s), tm_b, full_bar(s), kb * kTileK, tl.tj * BN);
          } else {
#pragma unroll
            for (int c = 0; c < BN / 64; ++c)
              tma_load_2d(sB(s) + c * (64 * kTileK * 2), tm_b, full_bar(s),
                          tl.tj * BN + c * 64, kb * kTileK);
          }
        }
      }
      if (!ok) {
        // Let every copy this thread started land before the block exits:
        // the last kStages iterations before the failed one were issued.
        volatile int never = 0;
        for (int j = (it > kStages ? it - kStages : 0); j < it; ++j)
          mbar_wait_bounded(full_bar(j % kStages), (j / kStages) & 1, &never,
                            10ull * 1000ull * 1000ull);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(BN, kBmn);
      int it = 0, lt = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < p.n_tiles; t += gridDim.x, ++lt) {
        const NsTile tl = p.tiles[t];
        const int acc = lt & 1;
        const uint32_t aph = (lt >> 1) & 1;
        if (!mbar_wait_bounded(tempty_bar(acc), aph ^ 1u, abort_flag)) {
          record_failure(p.err, kErrTimeoutMma, abort_flag);
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        for (int kb = 0; kb < tl.kt; ++kb, ++it) {
          const int s = it % kStages;
          const uint32_t ph = (it / kStages) & 1;
          if (!mbar_wait_bounded(full_bar(s), ph, abort_flag)) {
            record_failure(p.err, kErrTimeoutMma, abort_flag);
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < kTileK / 16; ++kk) {
            const uint64_t adesc = smem_desc_sw128(sA(s) + kk * 32, 16, 1024);
            const uint64_t bdesc =
                kBmn ? smem_desc_sw128(sB(s) + kk * 2048, 64 * kTileK * 2, 1024)
                     : smem_desc_sw128(sB(s) + kk * 32, 16, 1024);
            umma_bf16(d_tmem, adesc, bdesc, idesc, (kb | kk) != 0 ? 1u : 0u);
          }
          umma_commit(empty_bar(s));
        }
        if (!ok) break;
        umma_commit(tfull_bar(acc));
      }
      // Drain: every MMA this thread issued completes before TMEM is freed.
      umma_commit(drain_bar);
      volatile int never = 0;
      mbar_wait_bounded(drain_bar, 0, &never, 10ull * 1000ull * 1000ull);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int quad = warp & 3;             // TMEM lane quadrant of this warp
    const int r_in = quad * 32 + lane;     // accumulator row of this thread
    int lt = 0;
    for (int t = blockIdx.x; t < p.n_tiles; t += gridDim.x, ++lt) {
      const NsTile tl = p.tiles[t];
      const MatDev* md = p.mats + tl.mat;
      const int acc = lt & 1;
      const uint32_t aph = (lt >> 1) & 1;
      if (!mbar_wait_bounded(tfull_bar(acc), aph, abort_flag)) {
        record_failure(p.err, kErrTimeoutEpilogue, abort_flag);
        break;
      }
      tc_fence_after();
      const uint32_t tbase = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) +
                             static_cast<uint32_t>(acc * BN);
      const int row = tl.ti * kTileM + r_in;
      const int m = md->m;
      const bool row_ok = row < m;
      const float s = p.first ? frob_scale(md, p.partials, p.eps_frob) : 1.f;

      if (p.mode == kModeGram || p.mode == kModePoly) {
        __nv_bfloat16* outp = (p.mode == kModeGram) ? md->a : md->b;
        const bool mirror = tl.ti != tl.tj;
#pragma unroll 1
        for (int cc = 0; cc < BN / 32; ++cc) {
          float v[32];
          tmem_load_32cols(tbase + cc * 32, v);
          const int col0 = tl.tj * BN + cc * 32;
          if (p.mode == kModeGram) {
            const float s2 = s * s;
#pragma unroll
            for (int e = 0; e < 32; ++e) v[e] *= s2;
          } else if (row_ok) {
            float av[32];
            load_row32_bf16(md->a + static_cast<size_t>(row) * md->lda, col0, m, av);
#pragma unroll
            for (int e = 0; e < 32; ++e) v[e] = fmaf(p.b, av[e], p.c * v[e]);
            if (!mirror && (r_in >> 5) == cc) {  // this row's diagonal element
              const int d = r_in & 31;
#pragma unroll
              for (int e = 0; e < 32; ++e)
                if (e == d) v[e] += p.a;
            }
          }
          if (row_ok) {
            store_row32_bf16(outp + static_cast<size_t>(row) * md->lda, col0, m, v);
            if (mirror) store_col32_bf16(outp, md->lda, row, col0, m, v);
          }
        }
      } else {
        const int n = md->n;
        __nv_bfloat16* xd = md->x[p.src ^ 1] + static_cast<size_t>(row) * md->ldx;
        const float decay = 1.f - p.lr * p.wd;
        const float step = p.lr * md->update_scale;
#pragma unroll 1
        for (int cc = 0; cc < BN / 32; ++cc) {
          float v[32];
          tmem_load_32cols(tbase + cc * 32, v);
          const int col0 = tl.tj * BN + cc * 32;
          if (!row_ok || col0 >= n) continue;
          if (p.first) {
#pragma unroll
            for (int e = 0; e < 32; ++e) v[e] *= s;
          }
          if (!p.last) {
            store_row32_bf16(xd, col0, n, v);
          } else if (!md->transposed) {
            // O (rows x cols) = X: this thread owns a contiguous row segment.
            float* w = md->w + static_cast<size_t>(row) * n;
            float* o = md->out ? md->out + static_cast<size_t>(row) * n : nullptr;
            if (col0 + 32 <= n && (n & 3) == 0) {
#pragma unroll
              for (int q = 0; q < 8; ++q) {
                float4 wv = *reinterpret_cast<const float4*>(w + col0 + 4 * q);
                wv.x = fmaf(wv.x, decay, -step * v[4 * q + 0]);
                wv.y = fmaf(wv.y, decay, -step * v[4 * q + 1]);
                wv.z = fmaf(wv.z, decay, -step * v[4 * q + 2]);
                wv.w = fmaf(wv.w, decay, -step * v[4 * q + 3]);
                *reinterpret_cast<float4*>(w + col0 + 4 * q) = wv;
                if (o)
                  *reinterpret_cast<float4*>(o + col0 + 4 * q) =
                      make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
              }
            } else {
#pragma unroll
              for (int e = 0; e < 32; ++e) {
                if (col0 + e < n) {
                  w[col0 + e] = fmaf(w[col0 + e], decay, -step * v[e]);
                  if (o) o[col0 + e] = v[e];
                }
              }
            }
          } else {
            // O = X^T: W is n x m; element (row, col) of X lands at
            // W[col][row], consecutive across the warp's lanes.
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              const int col = col0 + e;
              if (col < n) {
                const size_t off = static_cast<size_t>(col) * m + row;
                md->w[off] = fmaf(md->w[off], decay, -step * v[e]);
                if (md->out) md->out[off] = v[e];
              }
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(tempty_bar(acc));
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem_base, Cfg::kTmemCols);
  }
}

}  // namespace muonb200
