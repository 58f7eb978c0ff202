// K-PRO: the elementwise front of the Muon step, one HBM pass per matrix.
//
// Per stored row of every matrix:  M' = mu M + G;  U = G + mu M' (Nesterov);
// r = ||U||;  X~ = U / (r + eps_row) (MuonEq-R);  X~ is written in bf16 in the
// working orientation (transposed through shared memory when rows > cols);
// the Frobenius partial sum of X~ over the work item goes to `partials`.
//
// Every work item writes its Frobenius partial sum to its own slot; the
// scale s = 1 / (||X~||_F + eps_frob) of each matrix is summed from them by
// muon_frob_scale_kernel (one warp per matrix, a fixed order).
//
// Sources: PR #1893 "Record: L_ParallelResiduals_UNetSkips_DepthRecur_Muon_
// 1.0901", table "Architecture and training stack", row "Optimizer" (Muon,
// momentum 0.99); PR #1396 "Record: Combined 3-Layer Recurrence + Parallel
// Residuals + Polar Express + Brotli", table "Techniques Combined", row
// "MuonEq-R" (row-norm before NS).
#pragma once

#include <cuda_bf16.h>

#include "muon_types.cuh"
#include "sm100_ptx.cuh"

namespace muonb200 {

__device__ __forceinline__ float warp_allreduce_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ void prefetch_l2(const void* p) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

__device__ __forceinline__ float bf16_bits_to_float(uint16_t b) {
  return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

// Element e of chunk ch for this lane: contiguous 8-element groups on the
// vector path, lane-strided elements otherwise.
__device__ __forceinline__ int chunk_pos(bool vec, int ch, int lane, int e) {
  return vec ? ch * 256 + lane * 8 + e : ch * 256 + e * 32 + lane;
}

__device__ __forceinline__ void load_g_m(const uint16_t* __restrict__ g,
                                         const float* __restrict__ mo,
                                         bool vec, int ch, int lane, int cols,
                                         float (&gv)[8], float (&mv)[8]) {
  if (vec) {
    const int p0 = ch * 256 + lane * 8;
    if (p0 < cols) {
      const uint4 graw = *reinterpret_cast<const uint4*>(g + p0);
      const float4 m0 = *reinterpret_cast<const float4*>(mo + p0);
      const float4 m1 = *reinterpret_cast<const float4*>(mo + p0 + 4);
      const uint32_t gw[4] = {graw.x, graw.y, graw.z, graw.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        gv[2 * i] = __uint_as_float(gw[i] << 16);
        gv[2 * i + 1] = __uint_as_float(gw[i] & 0xFFFF0000u);
      }
      mv[0] = m0.x; mv[1] = m0.y; mv[2] = m0.z; mv[3] = m0.w;
      mv[4] = m1.x; mv[5] = m1.y; mv[6] = m1.z; mv[7] = m1.w;
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) gv[e] = mv[e] = 0.f;
    }
  } else {
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int p = chunk_pos(false, ch, lane, e);
      gv[e] = p < cols ? bf16_bits_to_float(g[p]) : 0.f;
      mv[e] = p < cols ? mo[p] : 0.f;
    }
  }
}

__device__ __forceinline__ void store_m(float* __restrict__ mo, bool vec,
                                        int ch, int lane, int cols,
                                        const float (&mv)[8]) {
  if (vec) {
    const int p0 = ch * 256 + lane * 8;
    if (p0 < cols) {
      // default caching: pass 2 re-reads M' from L2
      *reinterpret_cast<float4*>(mo + p0) = make_float4(mv[0], mv[1], mv[2], mv[3]);
      *reinterpret_cast<float4*>(mo + p0 + 4) = make_float4(mv[4], mv[5], mv[6], mv[7]);
    }
  } else {
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int p = chunk_pos(false, ch, lane, e);
      if (p < cols) mo[p] = mv[e];
    }
  }
}

// Writes 8 normalised values of one stored row: straight into X (row-major)
// or into the shared staging tile for the transposed write-out.
__device__ __forceinline__ void emit_x(__nv_bfloat16* __restrict__ xrow,
                                       __nv_bfloat16* __restrict__ srow,
                                       bool transposed, bool vec, int ch,
                                       int lane, int cols,
                                       const float (&x)[8]) {
  if (vec) {
    const int p0 = ch * 256 + lane * 8;
    if (p0 >= cols) return;
    __nv_bfloat162 h[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(x[2 * i], x[2 * i + 1]);
    if (!transposed) {
      *reinterpret_cast<uint4*>(xrow + p0) = *reinterpret_cast<uint4*>(h);
    } else {
      // staging rows are (cols + 2) elements: 4-byte aligned only
#pragma unroll
      for (int i = 0; i < 4; ++i)
        *reinterpret_cast<__nv_bfloat162*>(srow + p0 + 2 * i) = h[i];
    }
  } else {
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int p = chunk_pos(false, ch, lane, e);
      if (p < cols) {
        const __nv_bfloat16 v = __float2bfloat16_rn(x[e]);
        if (!transposed) xrow[p] = v; else srow[p] = v;
      }
    }
  }
}

// Loads of one chunk kept raw: G as 8 packed bf16, M as 8 floats.
struct ChunkRaw {
  uint4 g;
  float4 m0, m1;
};

__device__ __forceinline__ void load_chunk_vec(const uint16_t* __restrict__ g,
                                               const float* __restrict__ mo,
                                               int p0, ChunkRaw& c) {
  c.g = *reinterpret_cast<const uint4*>(g + p0);
  c.m0 = *reinterpret_cast<const float4*>(mo + p0);
  c.m1 = *reinterpret_cast<const float4*>(mo + p0 + 4);
}

__device__ __forceinline__ void unpack_chunk(const ChunkRaw& c, float (&gv)[8],
                                             float (&mv)[8]) {
  const uint32_t gw[4] = {c.g.x, c.g.y, c.g.z, c.g.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    gv[2 * i] = __uint_as_float(gw[i] << 16);
    gv[2 * i + 1] = __uint_as_float(gw[i] & 0xFFFF0000u);
  }
  mv[0] = c.m0.x; mv[1] = c.m0.y; mv[2] = c.m0.z; mv[3] = c.m0.w;
  mv[4] = c.m1.x; mv[5] = c.m1.y; mv[6] = c.m1.z; mv[7] = c.m1.w;
}

// Two variants, one launch each, over disjoint parts of the item list:
//
// kOnePass (rows of up to kProOneWarps * 1024 elements, cols a multiple of 8;
// every matrix of the 11L/16L/24L stacks): a row is spread over wpr warps of
// 1024 elements each (four 8-element chunks per lane, all requested at once),
// U stays in registers between the row-norm reduction and the write of X~,
// and the row norm is summed across the row's warps in shared memory.  G and M
// are read once: 12 bytes of HBM per element.
//
// two-pass (longer or unaligned rows): one warp per stored row and no
// register copy of it.  Pass 1 streams G and M (kProBatch chunks of 8
// elements per lane in flight), writes M' and sums U^2; pass 2 re-reads G and
// the M' it just wrote (from L2 while the item is small enough), rebuilds U
// and writes the normalised row.
//
// The variants are separate kernels because the one-pass register budget
// (128 per thread at two blocks per SM) leaves no room for the other path's
// live values, and the two-pass variant keeps three blocks per SM.  Both are
// persistent: as many blocks as fit on the GPU at once, block b taking items
// b, b + grid, ... of its part of the list (items listed largest first), so
// that no partial last wave of blocks trails the pass and no counter has to
// be reset before it.
template <bool kOnePass>
__global__ void __launch_bounds__(kProThreads, kOnePass ? 2 : 3)
muon_prologue_kernel(const MatDev* __restrict__ mats,
                     const ProItem* __restrict__ items, int n_items, HyperDev h,
                     float* __restrict__ partials, int32_t* __restrict__ zero, int n_zero,
                     int prefetch, int write_lr, int32_t* err, int n_mats, int n_parts) {
  extern __shared__ __align__(16) unsigned char pro_smem[];
  __shared__ float warp_sums[kProThreads / 32];
  __shared__ float row_sums[2][kProThreads / 32];

  // The Newton-Schulz kernel launched next may get its CTAs resident as
  // soon as this grid's blocks leave their SMs (it needs a whole SM's shared
  // memory); it waits for this grid to complete before it reads anything
  // written here.
  grid_launch_dependents();
  // A scheduled step's learning rate, for the Newton-Schulz kernel (which
  // advances the step counter once every block here has read it).
  if (write_lr && h.step && blockIdx.x == 0 && threadIdx.x == 0)
    *h.lr_slot = linear_ramp(h.lr_v0, h.lr_v1, h.lr_t0, h.lr_t1, *h.step);

  // The step's Newton-Schulz completion counters start at zero: the previous
  // step's Newton-Schulz kernel finished before this launch, and this step's
  // starts after it.
  for (int i = blockIdx.x * kProThreads + threadIdx.x; i < n_zero; i += gridDim.x * kProThreads)
    zero[i] = 0;

  for (int idx = blockIdx.x; idx < n_items; idx += gridDim.x) {
    __syncthreads();   // the previous item's staging and sums are consumed
    const ProItem it = items[idx];
    if constexpr (kDeviceChecks) {
      // Device-checked build: an item outside its matrix (or with a partial
      // slot past the table) is skipped and recorded.
      const bool valid = it.mat >= 0 && it.mat < n_mats && it.nrows > 0 && it.row0 >= 0 &&
                         it.row0 + it.nrows <= mats[it.mat].rows && it.part >= 0 &&
                         it.part < n_parts;
      if (!valid) {
        if (threadIdx.x == 0) record_check_failure(err, kErrCheckPrologue, idx);
        continue;
      }
    }
    const MatDev& md = mats[it.mat];
    const int cols = md.cols;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const bool vec = (cols & 7) == 0;
    const bool tr = md.transposed != 0;
    const int sld = cols + 2;  // staging row stride (elements)
    __nv_bfloat16* stage = reinterpret_cast<__nv_bfloat16*>(pro_smem);
    const int nch = (cols + 255) / 256;
    const float mu = h.step ? linear_ramp(h.mu_v0, h.mu_v1, h.mu_t0, h.mu_t1, *h.step) : h.mu;

    float fro = 0.f;
    if constexpr (kOnePass) {
      // warps per row: 1, 2, 4 or 8
      const int wpr = pro_warps_per_row(cols);
      const int rpp = (kProThreads / 32) / wpr;   // rows per pass of the block
      const int rg = warp / wpr, wi = warp - rg * wpr;
      for (int r0 = 0, pass = 0; r0 < it.nrows; r0 += rpp, ++pass) {
        const int r = r0 + rg;
        const bool act = r < it.nrows;
        const int row = it.row0 + (act ? r : 0);
        const size_t base = static_cast<size_t>(row) * cols;
        const uint16_t* __restrict__ g = md.g + base;
        float* __restrict__ mo = md.mom + base;
        __nv_bfloat16* xrow = tr ? nullptr : md.x[0] + static_cast<size_t>(row) * md.ldx;
        __nv_bfloat16* srow = tr ? stage + r * sld : nullptr;
        ChunkRaw raw[4];
  #pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int p0 = (wi * 4 + j) * 256 + lane * 8;
          if (act && p0 < cols) load_chunk_vec(g, mo, p0, raw[j]);
        }
        // The next pass's row of this warp goes into L2 while this one is
        // processed (when the host asks for it): one prefetch per 128-byte
        // line of G (every 8th lane) and of M (every 4th lane).
        if (prefetch && r + rpp < it.nrows) {
          const size_t nbase = static_cast<size_t>(it.row0 + r + rpp) * cols;
  #pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int p0 = (wi * 4 + j) * 256 + lane * 8;
            if (p0 < cols) {
              if ((lane & 7) == 0) prefetch_l2(md.g + nbase + p0);
              if ((lane & 3) == 0) prefetch_l2(md.mom + nbase + p0);
            }
          }
        }
        float u[4][8];
        float ss = 0.f;
  #pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int p0 = (wi * 4 + j) * 256 + lane * 8;
          if (act && p0 < cols) {
            float gv[8], mv[8];
            unpack_chunk(raw[j], gv, mv);
  #pragma unroll
            for (int e = 0; e < 8; ++e) {
              const float mn = fmaf(mu, mv[e], gv[e]);
              u[j][e] = h.nesterov ? fmaf(mu, mn, gv[e]) : mn;
              mv[e] = mn;
              ss = fmaf(u[j][e], u[j][e], ss);
            }
            store_m(mo, true, wi * 4 + j, lane, cols, mv);
          }
        }
        ss = warp_allreduce_sum(ss);
        if (wpr > 1) {
          // one barrier per pass; the two buffers alternate, so a buffer is
          // rewritten only after every warp passed the next pass's barrier
          if (lane == 0) row_sums[pass & 1][warp] = ss;
          __syncthreads();
          float t = 0.f;
          for (int w = 0; w < wpr; ++w) t += row_sums[pass & 1][rg * wpr + w];
          ss = t;
        }
        const float inv = h.eq_r ? 1.f / (sqrtf(ss) + h.eps_row) : 1.f;
        if (act && wi == 0) fro += ss * inv * inv;
  #pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int p0 = (wi * 4 + j) * 256 + lane * 8;
          if (act && p0 < cols) {
            float x[8];
  #pragma unroll
            for (int e = 0; e < 8; ++e) x[e] = u[j][e] * inv;
            emit_x(xrow, srow, tr, true, wi * 4 + j, lane, cols, x);
          }
        }
      }
    } else {
      for (int r = warp; r < it.nrows; r += kProThreads / 32) {
        const int row = it.row0 + r;
        const size_t base = static_cast<size_t>(row) * cols;
        const uint16_t* __restrict__ g = md.g + base;
        float* __restrict__ mo = md.mom + base;
        __nv_bfloat16* xrow = tr ? nullptr : md.x[0] + static_cast<size_t>(row) * md.ldx;
        __nv_bfloat16* srow = tr ? stage + r * sld : nullptr;

        // Pass 1: M' = mu M + G (stored), U = G + mu M', sum of U^2.
        float ss = 0.f;
        for (int c0 = 0; c0 < nch; c0 += kProBatch) {
          if (vec) {
            ChunkRaw raw[kProBatch];
    #pragma unroll
            for (int b = 0; b < kProBatch; ++b) {
              const int p0 = (c0 + b) * 256 + lane * 8;
              if (c0 + b < nch && p0 < cols) load_chunk_vec(g, mo, p0, raw[b]);
            }
    #pragma unroll
            for (int b = 0; b < kProBatch; ++b) {
              const int p0 = (c0 + b) * 256 + lane * 8;
              if (c0 + b < nch && p0 < cols) {
                float gv[8], mv[8];
                unpack_chunk(raw[b], gv, mv);
    #pragma unroll
                for (int e = 0; e < 8; ++e) {
                  const float mn = fmaf(mu, mv[e], gv[e]);
                  const float u = h.nesterov ? fmaf(mu, mn, gv[e]) : mn;
                  mv[e] = mn;
                  ss = fmaf(u, u, ss);
                }
                store_m(mo, true, c0 + b, lane, cols, mv);
              }
            }
          } else {
            for (int b = 0; b < kProBatch && c0 + b < nch; ++b) {
              float gv[8], mv[8];
              load_g_m(g, mo, false, c0 + b, lane, cols, gv, mv);
    #pragma unroll
              for (int e = 0; e < 8; ++e) {
                const float mn = fmaf(mu, mv[e], gv[e]);
                const float u = h.nesterov ? fmaf(mu, mn, gv[e]) : mn;
                mv[e] = mn;
                ss = fmaf(u, u, ss);
              }
              store_m(mo, false, c0 + b, lane, cols, mv);
            }
          }
        }
        ss = warp_allreduce_sum(ss);
        const float inv = h.eq_r ? 1.f / (sqrtf(ss) + h.eps_row) : 1.f;
        fro += ss * inv * inv;
        __syncwarp();  // this lane's M' stores precede its own re-reads below

        // Pass 2: U again from G and M', normalised, bf16.
        for (int c0 = 0; c0 < nch; c0 += kProBatch) {
          if (vec) {
            ChunkRaw raw[kProBatch];
    #pragma unroll
            for (int b = 0; b < kProBatch; ++b) {
              const int p0 = (c0 + b) * 256 + lane * 8;
              if (c0 + b < nch && p0 < cols) load_chunk_vec(g, mo, p0, raw[b]);
            }
    #pragma unroll
            for (int b = 0; b < kProBatch; ++b) {
              const int p0 = (c0 + b) * 256 + lane * 8;
              if (c0 + b < nch && p0 < cols) {
                float gv[8], mv[8], x[8];
                unpack_chunk(raw[b], gv, mv);
    #pragma unroll
                for (int e = 0; e < 8; ++e) {
                  const float u = h.nesterov ? fmaf(mu, mv[e], gv[e]) : mv[e];
                  x[e] = u * inv;
                }
                emit_x(xrow, srow, tr, true, c0 + b, lane, cols, x);
              }
            }
          } else {
            for (int b = 0; b < kProBatch && c0 + b < nch; ++b) {
              float gv[8], mv[8], x[8];
              load_g_m(g, mo, false, c0 + b, lane, cols, gv, mv);
    #pragma unroll
              for (int e = 0; e < 8; ++e) {
                const float u = h.nesterov ? fmaf(mu, mv[e], gv[e]) : mv[e];
                x[e] = u * inv;
              }
              emit_x(xrow, srow, tr, false, c0 + b, lane, cols, x);
            }
          }
        }
      }
    }

    if (lane == 0) warp_sums[warp] = fro;
    __syncthreads();
    if (threadIdx.x == 0) {
      float s = 0.f;
  #pragma unroll
      for (int w = 0; w < kProThreads / 32; ++w) s += warp_sums[w];
      partials[it.part] = s;   // summed per matrix by muon_frob_scale_kernel
    }

    if (tr) {
      // X[c][row0 + r] = stage[r][c]: 8 stored rows -> one 16-byte store.
      const int ngrp = (it.nrows + 7) / 8;
      __nv_bfloat16* xbase = md.x[0];
      for (int idx = threadIdx.x; idx < cols * ngrp; idx += kProThreads) {
        const int c = idx / ngrp;
        const int grp = idx - c * ngrp;
        const int r0 = grp * 8;
        __nv_bfloat16* dst = xbase + static_cast<size_t>(c) * md.ldx + it.row0 + r0;
        if (r0 + 8 <= it.nrows && ((it.row0 + r0) & 7) == 0) {
          __align__(16) __nv_bfloat16 v[8];
  #pragma unroll
          for (int k = 0; k < 8; ++k) v[k] = stage[(r0 + k) * sld + c];
          *reinterpret_cast<uint4*>(dst) = *reinterpret_cast<uint4*>(v);
        } else {
          for (int k = 0; k < 8 && r0 + k < it.nrows; ++k)
            dst[k] = stage[(r0 + k) * sld + c];
        }
      }
    }
  }
}

// The Frobenius scale s = 1 / (||X~||_F + eps_frob) of every matrix from its
// prologue partials, for the step without Newton-Schulz iterations (the
// Newton-Schulz kernel sums the partials itself, in the same order): one
// warp per matrix, lane l adds slots l, l + 32, ... and the warp's butterfly
// adds the lanes, the same order on every run.
//
// With a schedule, thread 0 of block 0 also resolves the step's learning
// rate into *lr_slot and advances the step counter: every prologue block has
// read the counter by now, and the later kernels of the step read the slot.
__global__ void __launch_bounds__(256)
muon_frob_scale_kernel(const MatDev* __restrict__ mats, int n_mats,
                       const float* __restrict__ partials, HyperDev h,
                       float* __restrict__ mat_scale) {
  if (h.step && blockIdx.x == 0 && threadIdx.x == 0) {
    const int32_t t = *h.step;
    *h.lr_slot = linear_ramp(h.lr_v0, h.lr_v1, h.lr_t0, h.lr_t1, t);
    *h.step = t + 1;
  }
  const int mat = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (mat >= n_mats) return;
  const MatDev& md = mats[mat];
  float s = 0.f;
  for (int i = lane; i < md.part_count; i += 32) s += partials[md.part_first + i];
  s = warp_allreduce_sum(s);
  if (lane == 0) mat_scale[mat] = 1.f / (sqrtf(s) + h.eps_frob);
}

// ns_steps == 0: O = s X~ straight from the prologue's output, then the
// decoupled decay and scaled update.  One block per prologue work item.
__global__ void __launch_bounds__(kProThreads)
muon_final_noiter_kernel(const MatDev* __restrict__ mats,
                         const ProItem* __restrict__ items,
                         const float* __restrict__ mat_scale, float lr_host,
                         const float* __restrict__ lr_dev, float wd) {
  const ProItem it = items[blockIdx.x];
  const MatDev& md = mats[it.mat];
  const float s = mat_scale[it.mat];
  const float lr = lr_dev ? *lr_dev : lr_host;
  const float decay = 1.f - lr * wd;
  const float step = lr * md.update_scale;
  const int cols = md.cols;
  const int total = it.nrows * cols;
  for (int idx = threadIdx.x; idx < total; idx += kProThreads) {
    const int r = it.row0 + idx / cols;
    const int c = idx - (idx / cols) * cols;
    const size_t xo = md.transposed
                          ? static_cast<size_t>(c) * md.ldx + r
                          : static_cast<size_t>(r) * md.ldx + c;
    const float o = s * __bfloat162float(md.x[0][xo]);
    const size_t wo = static_cast<size_t>(r) * cols + c;
    md.w[wo] = fmaf(md.w[wo], decay, -step * o);
    if (md.out) md.out[wo] = o;
  }
}

}  // namespace muonb200
