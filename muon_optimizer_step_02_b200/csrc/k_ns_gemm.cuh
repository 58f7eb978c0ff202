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
// Roles (320 threads): warp 0 issues TMA loads into a ring of shared-memory
// stages; warp 1 owns TMEM and issues tcgen05.mma (M = 128, N = BN, K = 16)
// from one thread; warps 2-9 drain the double-buffered TMEM accumulator and
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

constexpr int kEpiWarps = 8;                 // two per TMEM lane quadrant
constexpr int kNsThreads = 64 + 32 * kEpiWarps;
constexpr int kXposeLd = 34;                 // bf16 per row of a 32x32 block

template <int BN, bool kBmn, int kStages>
struct NsCfg {
  static constexpr int kABytes = kTileM * kTileK * 2;
  static constexpr int kBBytes = BN * kTileK * 2;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kTmemCols = 2 * BN;
  static constexpr int kNumBars = 2 * kStages + 5;
  // per epilogue warp: a 32 x 32 bf16 block for the mirrored store
  static constexpr int kXposeBytes = kBmn ? 0 : kEpiWarps * 32 * kXposeLd * 2;
  static constexpr size_t kSmemBytes = 1024 +
      static_cast<size_t>(kStages) * kStageBytes + kXposeBytes +
      kNumBars * 8 + 16;
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

template <int BN, bool kBmn, int kStages>
__global__ void __launch_bounds__(kNsThreads, 1)
ns_gemm_kernel(const __grid_constant__ NsParams p) {
  using Cfg = NsCfg<BN, kBmn, kStages>;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  __nv_bfloat16* xpose =
      reinterpret_cast<__nv_bfloat16*>(smem + kStages * Cfg::kStageBytes);
  uint64_t* bars = reinterpret_cast<uint64_t*>(
      smem + kStages * Cfg::kStageBytes + Cfg::kXposeBytes);
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
      mbar_init(tempty_bar(a), 32 * kEpiWarps);
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
    // Eight warps: two per TMEM lane quadrant, splitting a tile's 32-column
    // chunks between them.  Inputs of a chunk (A for poly, W for the update)
    // are loaded before the accumulator so their latency overlaps.
    const int ew = warp - 2;
    const int quad = warp & 3;             // TMEM lane quadrant of this warp
    const int half = ew >> 2;              // chunk parity handled by this warp
    const int r_in = quad * 32 + lane;     // accumulator row of this thread
    __nv_bfloat16* xbuf = xpose + ew * 32 * kXposeLd;
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
      const int row0 = tl.ti * kTileM + quad * 32;
      const int row = row0 + lane;
      const int m = md->m;
      const bool row_ok = row < m;
      const float s = p.first ? frob_scale(md, p.partials, p.eps_frob) : 1.f;

      if (p.mode == kModeGram || p.mode == kModePoly) {
        __nv_bfloat16* outp = (p.mode == kModeGram) ? md->a : md->b;
        const bool mirror = tl.ti != tl.tj;
#pragma unroll 1
        for (int cc = half; cc < BN / 32; cc += 2) {
          const int col0 = tl.tj * BN + cc * 32;
          float av[32];
          if (p.mode == kModePoly && row_ok)
            load_row32_bf16(md->a + static_cast<size_t>(row) * md->lda, col0, m, av);
          float v[32];
          tmem_load_32cols(tbase + cc * 32, v);
          if (p.mode == kModeGram) {
            const float s2 = s * s;
#pragma unroll
            for (int e = 0; e < 32; ++e) v[e] *= s2;
          } else if (row_ok) {
#pragma unroll
            for (int e = 0; e < 32; ++e) v[e] = fmaf(p.b, av[e], p.c * v[e]);
            if (!mirror && (r_in >> 5) == cc) {  // this row's diagonal element
              const int d = r_in & 31;
#pragma unroll
              for (int e = 0; e < 32; ++e)
                if (e == d) v[e] += p.a;
            }
          }
          if (row_ok)
            store_row32_bf16(outp + static_cast<size_t>(row) * md->lda, col0, m, v);
          if (mirror)
            store_mirror32_bf16(outp, md->lda, row0, col0, m, lane, xbuf, v);
        }
      } else {
        const int n = md->n;
        __nv_bfloat16* xd = md->x[p.src ^ 1] + static_cast<size_t>(row) * md->ldx;
        const float decay = 1.f - p.lr * p.wd;
        const float step = p.lr * md->update_scale;
        const bool tr = md->transposed != 0;
#pragma unroll 1
        for (int cc = half; cc < BN / 32; cc += 2) {
          const int col0 = tl.tj * BN + cc * 32;
          const bool live = row_ok && col0 < n;
          // W (and only W) is read in the last step: all 32 loads first.
          float wv[32];
          float* w_row = nullptr;
          const bool wvec = !tr && col0 + 32 <= n && (n & 3) == 0;
          if (p.last && live) {
            if (!tr) {
              w_row = md->w + static_cast<size_t>(row) * n + col0;
              if (wvec) {
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                  const float4 w4 = reinterpret_cast<const float4*>(w_row)[q];
                  wv[4 * q] = w4.x; wv[4 * q + 1] = w4.y;
                  wv[4 * q + 2] = w4.z; wv[4 * q + 3] = w4.w;
                }
              } else {
#pragma unroll
                for (int e = 0; e < 32; ++e) wv[e] = col0 + e < n ? w_row[e] : 0.f;
              }
            } else {
#pragma unroll
              for (int e = 0; e < 32; ++e)
                wv[e] = col0 + e < n
                            ? md->w[static_cast<size_t>(col0 + e) * m + row] : 0.f;
            }
          }
          float v[32];
          tmem_load_32cols(tbase + cc * 32, v);
          if (!live) continue;
          if (p.first) {
#pragma unroll
            for (int e = 0; e < 32; ++e) v[e] *= s;
          }
          if (!p.last) {
            store_row32_bf16(xd, col0, n, v);
            continue;
          }
#pragma unroll
          for (int e = 0; e < 32; ++e) wv[e] = fmaf(wv[e], decay, -step * v[e]);
          if (!tr) {
            float* o = md->out ? md->out + static_cast<size_t>(row) * n + col0 : nullptr;
            if (wvec) {
#pragma unroll
              for (int q = 0; q < 8; ++q) {
                reinterpret_cast<float4*>(w_row)[q] =
                    make_float4(wv[4 * q], wv[4 * q + 1], wv[4 * q + 2], wv[4 * q + 3]);
                if (o)
                  reinterpret_cast<float4*>(o)[q] =
                      make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
              }
            } else {
#pragma unroll
              for (int e = 0; e < 32; ++e)
                if (col0 + e < n) {
                  w_row[e] = wv[e];
                  if (o) o[e] = v[e];
                }
            }
          } else {
            // O = X^T: element (row, col) of X lands at W[col][row];
            // consecutive lanes write consecutive addresses.
#pragma unroll
            for (int e = 0; e < 32; ++e)
              if (col0 + e < n) {
                const size_t off = static_cast<size_t>(col0 + e) * m + row;
                md->w[off] = wv[e];
                if (md->out) md->out[off] = v[e];
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
