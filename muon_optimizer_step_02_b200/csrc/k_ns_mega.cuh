// All K Newton-Schulz steps of every matrix in one persistent launch on CTA
// pairs (tcgen05.mma.cta_group::2, 256 x 256 tiles).
//
// The work list (built on the host by schedule.h) holds the gram, poly and
// apply pair tiles of every step of every matrix.  Cluster c takes items c,
// c + C, c + 2C, ... in that order.  An item waits (in its producer, before
// loading) until the phase it reads is complete for its matrix:
//   gram(k)  reads X_k   <- every apply(k-1) tile of the matrix (k > 0)
//   poly(k)  reads A     <- every gram(k) tile of the matrix
//   apply(k) reads B', X <- every poly(k) tile of the matrix
// Completion is counted per (matrix, step, phase) in global memory: each CTA
// adds 1 after its half of a tile is stored (release), producers spin with
// acquire loads (bounded).  Every dependency precedes its dependants in the
// list and every cluster walks the list in order, so with all clusters
// resident the schedule cannot deadlock.  Different matrices overlap freely,
// and a tile's epilogue overlaps the next item's loads and MMAs.
//
// Per item:
//   gram  A  = s^2 X X^T   (upper pair tiles only: a consumer reads a block
//                          below the diagonal as the transpose of the stored
//                          block above it)
//   poly  B' = a I + b A + c A A   (A symmetric, so A A = A A^T; upper tiles)
//   apply X <- s B' X      (last step: W <- W (1 - lr wd) - lr scale O)
// X <- a X + B X is evaluated as (a I + B) X: one product, and the bf16 copy
// of B' holds a + B on its diagonal instead of the cancelling pair.
// s = 1 / (||X~||_F + eps_frob) in step 0 (the Frobenius normalisation folded
// into the first products), 1 afterwards.
//
// Roles (512 threads per CTA, four warpgroups): warp 0 issues TMA loads
// (.cta_group::2, no multicast) into a 5-stage ring, counting both CTAs'
// bytes on the leader's barrier; warp 1 of the leader issues the pair MMAs
// from one thread and frees stages / hands over accumulators with multicast
// tcgen05.commit; warp 2 publishes completed items; warp 3 idles; warps 4-15
// (warpgroups 1 to 3, three warps per TMEM lane quadrant, each taking every
// third 32-column block of the tile) drain that CTA's 128 TMEM lanes and run
// the fused epilogue.  After set-up warpgroup 0 gives its registers to the
// epilogue warpgroups (setmaxnreg), which then hold their blocks without
// spilling.  All waits are bounded: a failure raises both CTAs' abort flags
// and the global error word, and every CTA still meets the final cluster
// barrier before TMEM is freed.
//
// Source of the step: PR #1396 "Record: Combined 3-Layer Recurrence +
// Parallel Residuals + Polar Express + Brotli", table "Techniques Combined",
// row "Polar Express Newton-Schulz"; PR #1584 "Record: Improved Parallel
// Residuals + Systems Optimization", section "Summary" (fused Muon kernel).
#pragma once

#include <cuda_bf16.h>

#include "k_ns_common.cuh"
#include "muon_types.cuh"
#include "schedule.h"
#include "sm100_ptx.cuh"

namespace muonb200 {

constexpr int kMegaMaxSteps = 16;
constexpr int kMegaStages = 5;

struct MegaParams {
  const MatDev* mats;
  const SchedItem* items; // the schedule (host-built list, see schedule.h)
  const float* partials;  // the prologue's Frobenius partial sums
  int32_t* step_inc;      // scheduled step counter to advance, or null
  int32_t* err;           // error word, then the index of a failed check
  int32_t* done;          // [mat][step][phase] completion counts, zeroed
  int32_t n_items;
  int32_t n_mats;
  int32_t steps;
  int32_t fault, fresh;
  float a[kMegaMaxSteps], b[kMegaMaxSteps], c[kMegaMaxSteps];
  float lr, wd, eps_frob;
  const float* lr_dev;    // scheduled learning rate of the step, or null (use lr)
};

// Shared memory: the operand ring (per stage 16 KB of A rows + 16 KB of B
// columns), then per epilogue warp a 4 KB staging block (a 32 x 32 bf16
// output block, or the 32 x 32 fp32 block of the weight update), then the
// barriers.
struct MegaCfg {
  static constexpr int kABytes = 128 * kTileK * 2;
  static constexpr int kBBytes = (kPairTile / 2) * kTileK * 2;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr uint32_t kTxBytes = 2u * kStageBytes;   // both CTAs
  static constexpr int kTmemCols = 2 * kPairTile;
  static constexpr int kOutBlockElems = 32 * 32;
  static constexpr int kOutStageBytes = kEpiWarps * 2 * kOutBlockElems * 2;
  static constexpr int kEpiBars = 4;   // completion hand-off ring
  static constexpr int kNumBars = 2 * kMegaStages + 5 + kEpiBars;
  static constexpr size_t kSmemBytes = 1024 +
      static_cast<size_t>(kMegaStages) * kStageBytes + kOutStageBytes +
      kNumBars * 8 + 16;
  static_assert(kSmemBytes <= 227 * 1024, "shared memory");
};
constexpr size_t kMegaSmemBytes = MegaCfg::kSmemBytes;

// Spins (acquire) until *ctr >= target.  Gives up on the CTA's abort flag,
// on a non-zero global error word (another CTA failed) or after the limit.
__device__ __forceinline__ bool wait_count(const int32_t* ctr, int32_t target,
                                           volatile int* abort_flag,
                                           const int32_t* err) {
  if (ld_acquire_gpu(ctr) >= target) return true;
  const uint64_t t0 = global_timer_ns();
  for (uint32_t i = 1;; ++i) {
    if (ld_acquire_gpu(ctr) >= target) return true;
    if ((i & 15u) == 0) {
      if (*abort_flag) return false;
      if (*reinterpret_cast<const volatile int32_t*>(err) != 0) return false;
      if (global_timer_ns() - t0 > kWaitLimitNs) return false;
    }
    __nanosleep(64);
  }
}

// s = 1 / (||X~||_F + eps) of a matrix from its prologue partials: lane l
// adds slots l, l + 32, ..., then the warp's butterfly adds the lanes -- a
// fixed order, the same in every warp and on every run.
__device__ __forceinline__ float frob_scale(const float* partials, const MatDev* md,
                                            int lane, float eps) {
  float s = 0.f;
  for (int i = lane; i < md->part_count; i += 32) s += partials[md->part_first + i];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  return 1.f / (sqrtf(s) + eps);
}

struct MegaItem {
  NsTile tl;
  int mode;
  int k;
  int dep_target;   // completion count of the phase it reads (0: none)
};

// The raw 16-byte record of list position g (zeros past the end), read with
// one vector load.  Each role loads the record of its next item while it
// works on the current one, so no item starts with a global-memory round
// trip for its own description.
__device__ __forceinline__ uint4 load_item_raw(const MegaParams& p, int g) {
  if (g >= p.n_items) return make_uint4(0u, 0u, 0u, 0u);
  return __ldg(reinterpret_cast<const uint4*>(p.items) + g);
}

__device__ __forceinline__ MegaItem unpack_item(const uint4 r) {
  MegaItem it;
  it.tl.mat = static_cast<uint16_t>(r.x & 0xFFFFu);
  it.tl.ti = static_cast<uint16_t>(r.x >> 16);
  it.tl.tj = static_cast<uint16_t>(r.y & 0xFFFFu);
  it.tl.kt = static_cast<uint16_t>(r.y >> 16);
  it.mode = static_cast<int>(r.z & 0xFFu);
  it.k = static_cast<int>((r.z >> 8) & 0xFFu);
  it.dep_target = static_cast<int>(r.w);
  return it;
}

__device__ __forceinline__ int32_t* done_counter(const MegaParams& p, int mat,
                                                 int k, int mode) {
  return p.done + (static_cast<size_t>(mat) * p.steps + k) * 3 + mode;
}

// The completion counter of the phase an item reads (it.dep_target counts
// its tiles); nullptr if it has no in-kernel dependency (the gram of step 0
// reads the prologue's X).
__device__ __forceinline__ const int32_t* dep_counter(const MegaParams& p,
                                                      const MegaItem& it) {
  if (it.dep_target == 0) return nullptr;
  if (it.mode == kModeGram) return done_counter(p, it.tl.mat, it.k - 1, kModeApply);
  return done_counter(p, it.tl.mat, it.k, it.mode == kModePoly ? kModeGram : kModePoly);
}

// The fp32 weight update of the last step works on 32 x 32 blocks of the
// working orientation (W itself, or W^T for transposed matrices), rows
// row0 .. row0 + 32, columns col0 .. col0 + 32.  Full blocks of row-major W
// with 16-byte rows are "coalesced": lane L holds rows row0 + 4 i + L / 8
// (i = 0..7), columns col0 + 4 (L % 8) .. + 4, so each warp access covers
// four whole 128-byte rows; O reaches that layout through the warp's shared
// staging block.  Other blocks keep the accumulator's layout (lane = row).
__device__ __forceinline__ bool w_block_coalesced(const MatDev* md, int row0, int col0) {
  return !md->transposed && (md->n & 3) == 0 && col0 + 32 <= md->n &&
         row0 + 32 <= md->m && (reinterpret_cast<uintptr_t>(md->w) & 15u) == 0 &&
         (reinterpret_cast<uintptr_t>(md->out) & 15u) == 0;
}

// W of the block into wv (zeros outside the matrix).
__device__ __forceinline__ void load_w_block(const MatDev* md, int row0, int col0,
                                             int lane, float (&wv)[32]) {
  const int m = md->m, n = md->n;
  const float* __restrict__ w = md->w;
  if (w_block_coalesced(md, row0, col0)) {
    const float* base = w + static_cast<size_t>(row0 + (lane >> 3)) * n + col0 + 4 * (lane & 7);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float4 w4 = *reinterpret_cast<const float4*>(base + static_cast<size_t>(4 * i) * n);
      wv[4 * i] = w4.x; wv[4 * i + 1] = w4.y; wv[4 * i + 2] = w4.z; wv[4 * i + 3] = w4.w;
    }
    return;
  }
  const int row = row0 + lane;
  if (row >= m || col0 >= n) {
#pragma unroll
    for (int e = 0; e < 32; ++e) wv[e] = 0.f;
    return;
  }
  if (!md->transposed) {
    const float* w_row = w + static_cast<size_t>(row) * n + col0;
#pragma unroll
    for (int e = 0; e < 32; ++e) wv[e] = col0 + e < n ? w_row[e] : 0.f;
  } else {
#pragma unroll
    for (int e = 0; e < 32; ++e)
      wv[e] = col0 + e < n ? w[static_cast<size_t>(col0 + e) * m + row] : 0.f;
  }
}

// W <- W decay - step O on the block of load_w_block: wv holds its W, v the
// accumulator row of this lane (O); O also goes to the optional update
// output.  `stage` is the warp's 32 x 32 fp32 shared staging block.
// Device-checked build: a weight store outside the rows x cols matrix is
// skipped and its offset recorded.
__device__ __forceinline__ bool w_store_ok(const MatDev* md, size_t off, int width,
                                           int32_t* err) {
  if constexpr (!kDeviceChecks) {
    return true;
  } else {
    if (off + width <= static_cast<size_t>(md->rows) * md->cols) return true;
    record_check_failure(err, kErrCheckStore, static_cast<int32_t>(off));
    return false;
  }
}

__device__ __forceinline__ void store_w_block(const MatDev* md, int row0, int col0,
                                              int lane, float decay, float step,
                                              const float (&wv)[32], const float (&v)[32],
                                              float* stage, int32_t* err) {
  const int m = md->m, n = md->n;
  float* __restrict__ w = md->w;
  float* __restrict__ out = md->out;
  if (w_block_coalesced(md, row0, col0)) {
    // O row `lane` into the stage, 16-byte chunks XOR-swizzled by row so
    // that both the row-wise writes and the transposed reads are free of
    // bank conflicts.
#pragma unroll
    for (int q = 0; q < 8; ++q)
      *reinterpret_cast<float4*>(stage + lane * 32 + 4 * (q ^ (lane & 7))) =
          make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
    __syncwarp();
    const int c = lane & 7;
    const size_t g0 = static_cast<size_t>(row0 + (lane >> 3)) * n + col0 + 4 * c;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int rr = 4 * i + (lane >> 3);
      const float4 o4 = *reinterpret_cast<const float4*>(stage + rr * 32 + 4 * (c ^ (rr & 7)));
      const size_t g = g0 + static_cast<size_t>(4 * i) * n;
      if (!w_store_ok(md, g, 4, err)) continue;
      *reinterpret_cast<float4*>(w + g) =
          make_float4(fmaf(wv[4 * i], decay, -step * o4.x),
                      fmaf(wv[4 * i + 1], decay, -step * o4.y),
                      fmaf(wv[4 * i + 2], decay, -step * o4.z),
                      fmaf(wv[4 * i + 3], decay, -step * o4.w));
      if (out) *reinterpret_cast<float4*>(out + g) = o4;
    }
    __syncwarp();
    return;
  }
  const int row = row0 + lane;
  if (row >= m || col0 >= n) return;
  if (!md->transposed) {
    const size_t g = static_cast<size_t>(row) * n + col0;
#pragma unroll
    for (int e = 0; e < 32; ++e)
      if (col0 + e < n && w_store_ok(md, g + e, 1, err)) {
        w[g + e] = fmaf(wv[e], decay, -step * v[e]);
        if (out) out[g + e] = v[e];
      }
  } else {
#pragma unroll
    for (int e = 0; e < 32; ++e)
      if (col0 + e < n) {
        const size_t off = static_cast<size_t>(col0 + e) * m + row;
        if (!w_store_ok(md, off, 1, err)) continue;
        w[off] = fmaf(wv[e], decay, -step * v[e]);
        if (out) out[off] = v[e];
      }
  }
}

__global__ void __launch_bounds__(kNsThreads, 1)
ns_mega_pair_kernel(const __grid_constant__ MegaParams p) {
  using Cfg = MegaCfg;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  __nv_bfloat16* out_stage =
      reinterpret_cast<__nv_bfloat16*>(smem + kMegaStages * Cfg::kStageBytes);
  uint64_t* bars = reinterpret_cast<uint64_t*>(
      smem + kMegaStages * Cfg::kStageBytes + Cfg::kOutStageBytes);
  // bars: full[S], empty[S], tfull[2], tempty[2], drain, epi[kEpiBars]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + Cfg::kNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  // items whose completion the signal warp has published
  volatile int* sig_count = reinterpret_cast<volatile int*>(tmem_slot + 2);
  constexpr int S = kMegaStages;

  const uint32_t smem0 = smem_addr(smem);
  auto sA = [&](int s) { return smem0 + s * Cfg::kStageBytes; };
  auto sB = [&](int s) { return smem0 + s * Cfg::kStageBytes + Cfg::kABytes; };
  auto full_bar = [&](int s) { return smem_addr(bars + s); };
  auto empty_bar = [&](int s) { return smem_addr(bars + S + s); };
  auto tfull_bar = [&](int a) { return smem_addr(bars + 2 * S + a); };
  auto tempty_bar = [&](int a) { return smem_addr(bars + 2 * S + 2 + a); };
  const uint32_t drain_bar = smem_addr(bars + 2 * S + 4);
  auto epi_bar = [&](int a) { return smem_addr(bars + 2 * S + 5 + a); };

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1;
  const int npairs = gridDim.x >> 1;
  const int total = p.n_items;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull_bar(a), 1);
      mbar_init(tempty_bar(a), 2 * kEpiWarps);
    }
    for (int a = 0; a < Cfg::kEpiBars; ++a) mbar_init(epi_bar(a), kEpiWarps);
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    *sig_count = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_addr(tmem_slot), Cfg::kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // The kernel is launched as a programmatic dependent of the prologue: the
  // set-up above overlaps the prologue's last blocks; everything below reads
  // what the prologue wrote (X~, the Frobenius partials, the zeroed
  // counters, the scheduled learning rate), so every thread waits for it to
  // complete here.  (It lets no kernel after it start early: measured on the
  // 11L step, EMA blocks waiting resident beside this kernel cost it 15-30
  // us.)
  grid_dependency_wait();
  // The prologue has read the scheduled step number; advance it once.
  if (p.step_inc != nullptr && blockIdx.x == 0 && threadIdx.x == 0) *p.step_inc += 1;
  const uint32_t peer_abort = mapa_shared(smem_addr(const_cast<int*>(abort_flag)), rank ^ 1u);
  const uint32_t leader_full0 = mapa_shared(full_bar(0), 0);
  auto fail = [&](int32_t code) {
    atomicCAS(p.err, 0, code);
    *abort_flag = 1;
    st_shared_cluster_u32(peer_abort, 1u);
  };
  // Device-checked build: an item outside its matrix's tile grid (or with
  // the wrong K extent or dependency target) is never touched; its list
  // position is recorded and the kernel aborts like a failed wait.
  auto item_ok = [&](const MegaItem& it, int g) -> bool {
    if constexpr (!kDeviceChecks) {
      return true;
    } else {
      bool valid = it.tl.mat < p.n_mats;
      if (valid) {
        const MatDev* md = p.mats + it.tl.mat;
        valid = sched_item_valid(it.mode, it.k, it.tl.ti, it.tl.tj, it.tl.kt,
                                 it.dep_target, md->m, md->n, p.steps);
      }
      if (!valid) {
        record_check_failure(p.err, kErrCheckItem, g);
        *abort_flag = 1;
        st_shared_cluster_u32(peer_abort, 1u);
      }
      return valid;
    }
  };

  if (warp < kEpiWarp0) {
  // Warpgroup 0 keeps few registers; the epilogue warpgroups take the rest.
  // (The change sits at the top of each warpgroup's branch, so that the
  // compiler gives each branch its own register budget.)
  regs_decrease<kNsRegsControl>();
  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int it = 0;
      bool ok = true;
      uint4 nx = load_item_raw(p, pair);
      for (int g = pair; ok && g < total; g += npairs) {
        const MegaItem item = unpack_item(nx);
        nx = load_item_raw(p, g + npairs);
        if (!item_ok(item, g)) {
          ok = false;
          break;
        }
        const NsTile tl = item.tl;
        const MatDev* md = p.mats + tl.mat;
        const int src = item.k & 1;
        // A and B' hold their upper 256-blocks only: a K block of the A
        // operand (or of the polynomial's B operand) that falls below the
        // diagonal is loaded from the stored block above it as an MN-major
        // box (tm_an / tm_bn), and the MMA reads that K block transposed.
        const CUtensorMap* tm_a;
        const CUtensorMap* tm_b;
        const CUtensorMap* tm_an = nullptr;   // MN-major map of the A operand
        if (item.mode == kModeGram) {
          tm_a = &md->tm_xk[src];
          tm_b = tm_a;
        } else if (item.mode == kModePoly) {
          tm_a = &md->tm_a;
          tm_b = tm_a;
          tm_an = &md->tm_an;
        } else {
          tm_a = &md->tm_b;
          tm_b = &md->tm_xn[src];
          tm_an = &md->tm_bn;
        }
        if (p.fresh) {
          tensormap_acquire(tm_a);
          if (tm_b != tm_a) tensormap_acquire(tm_b);
          if (tm_an != nullptr) tensormap_acquire(tm_an);
        }
        const int32_t* dep = dep_counter(p, item);
        if (dep != nullptr) {
          if (!wait_count(dep, item.dep_target, abort_flag, p.err)) {
            fail(kErrTimeoutProducer);
            ok = false;
            break;
          }
          fence_proxy_async_global();   // generic stores of other CTAs -> TMA reads
        }
        const int arow = tl.ti * kPairTile + static_cast<int>(rank) * 128;
        const int bcol = tl.tj * kPairTile + static_cast<int>(rank) * 128;
        // Diagonal tiles of X X^T and A A: this CTA's half of the B operand
        // is the same 128 rows as its half of A, loaded once.
        const bool same = item.mode != kModeApply && tl.ti == tl.tj;
        for (int kb = 0; kb < tl.kt; ++kb, ++it) {
          const int s = it % S;
          const uint32_t ph = (it / S) & 1;
          if (!mbar_wait_bounded(empty_bar(s), ph ^ 1u, abort_flag)) {
            fail(kErrTimeoutProducer);
            ok = false;
            break;
          }
          if (p.fault == 1 && pair == 0 && it == 0 && leader) continue;  // test hook
          if (leader)
            mbar_arrive_expect_tx(full_bar(s), same ? 2u * Cfg::kABytes : Cfg::kTxBytes);
          const uint32_t lfull = leader_full0 + 8u * s;
          const int kblk = kb * kTileK / kPairTile;   // 256-block column of this K block
          // (an MN-major half is two 64-column boxes, the second 8 KB on)
          if (tm_an != nullptr && kblk < tl.ti) {
            tma_load_2d_pair(sA(s), tm_an, lfull, arow, kb * kTileK);
            tma_load_2d_pair(sA(s) + 64 * kTileK * 2, tm_an, lfull, arow + 64, kb * kTileK);
          } else {
            tma_load_2d_pair(sA(s), tm_a, lfull, kb * kTileK, arow);
          }
          if (item.mode == kModeGram) {
            if (!same) tma_load_2d_pair(sB(s), tm_b, lfull, kb * kTileK, bcol);
          } else if (item.mode == kModePoly) {
            if (!same) {
              if (kblk < tl.tj) {
                tma_load_2d_pair(sB(s), tm_an, lfull, bcol, kb * kTileK);
                tma_load_2d_pair(sB(s) + 64 * kTileK * 2, tm_an, lfull, bcol + 64,
                                 kb * kTileK);
              } else {
                tma_load_2d_pair(sB(s), tm_b, lfull, kb * kTileK, bcol);
              }
            }
          } else {
            tma_load_2d_pair(sB(s), tm_b, lfull, bcol, kb * kTileK);
            tma_load_2d_pair(sB(s) + 64 * kTileK * 2, tm_b, lfull, bcol + 64,
                             kb * kTileK);
          }
        }
      }
      if (!ok) {
        volatile int never = 0;
        if (leader)
          for (int j = (it > S ? it - S : 0); j < it; ++j)
            mbar_wait_bounded(full_bar(j % S), (j / S) & 1, &never,
                              10ull * 1000ull * 1000ull);
        const uint64_t t0 = global_timer_ns();
        while (global_timer_ns() - t0 < 20000ull) {
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && leader) {

      int it = 0, lt = 0;
      bool ok = true;
      uint4 nx = load_item_raw(p, pair);
      for (int g = pair; ok && g < total; g += npairs, ++lt) {
        const MegaItem item = unpack_item(nx);
        nx = load_item_raw(p, g + npairs);
        if (!item_ok(item, g)) break;
        const bool apply = item.mode == kModeApply;
        const bool same = !apply && item.tl.ti == item.tl.tj;   // B half = A half
        const int acc = lt & 1;
        const uint32_t aph = (lt >> 1) & 1;
        if (!mbar_wait_bounded(tempty_bar(acc), aph ^ 1u, abort_flag)) {
          fail(kErrTimeoutMma);
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * kPairTile;
        for (int kb = 0; kb < item.tl.kt; ++kb, ++it) {
          const int s = it % S;
          const uint32_t ph = (it / S) & 1;
          if (!mbar_wait_bounded(full_bar(s), ph, abort_flag)) {
            fail(kErrTimeoutMma);
            ok = false;
            break;
          }
          tc_fence_after();
          // Operand major-ness of this K block (see the producer): X in the
          // apply, and blocks of A or B' below the diagonal, are MN-major.
          const int kblk = kb * kTileK / kPairTile;
          const bool amn = item.mode != kModeGram && kblk < item.tl.ti;
          const bool bmn = apply || (item.mode == kModePoly && kblk < item.tl.tj);
          const uint32_t idesc = idesc_bf16_f32_pair(kPairTile, bmn, amn);
#pragma unroll
          for (int kk = 0; kk < kTileK / 16; ++kk) {
            const uint64_t adesc =
                amn ? smem_desc_sw128(sA(s) + kk * 2048, 64 * kTileK * 2, 1024)
                    : smem_desc_sw128(sA(s) + kk * 32, 16, 1024);
            const uint32_t bbase = same ? sA(s) : sB(s);
            const uint64_t bdesc =
                bmn ? smem_desc_sw128(bbase + kk * 2048, 64 * kTileK * 2, 1024)
                    : smem_desc_sw128(bbase + kk * 32, 16, 1024);
            umma_bf16_pair(d_tmem, adesc, bdesc, idesc, (kb | kk) != 0 ? 1u : 0u);
          }
          umma_commit_pair_mc(empty_bar(s), 0x3);
        }
        if (!ok) break;
        umma_commit_pair_mc(tfull_bar(acc), 0x3);
      }
      umma_commit_pair_mc(drain_bar, 0x1);
      volatile int never = 0;
      mbar_wait_bounded(drain_bar, 0, &never, 10ull * 1000ull * 1000ull);
    }
  } else if (warp == 2) {
    // ------------------------------------------------------------ signal
    // Publishes each item once all epilogue warps of this CTA have stored
    // it: gpu-scope fence, then a release add on the item's phase counter.
    if (lane == 0) {
      int lt = 0;
      uint4 nx = load_item_raw(p, pair);
      for (int g = pair; g < total; g += npairs, ++lt) {
        const MegaItem item = unpack_item(nx);
        nx = load_item_raw(p, g + npairs);
        if (!item_ok(item, g)) break;
        if (!mbar_wait_bounded(epi_bar(lt % Cfg::kEpiBars), (lt / Cfg::kEpiBars) & 1,
                               abort_flag)) {
          fail(kErrTimeoutEpilogue);
          break;
        }
        // release at gpu scope, cumulative over the stores the barrier
        // made visible to this thread
        red_release_gpu_add(done_counter(p, item.tl.mat, item.k, item.mode), 1);
        *sig_count = lt + 1;
      }
    }
  }
  } else {
    regs_increase<kNsRegsEpilogue>();
    // ------------------------------------------------------------ epilogue
    const int ew = warp - kEpiWarp0;
    const int quad = warp & 3;   // the TMEM lane quadrant this warp may read
    // this warp's 32-column blocks of the tile: cc = third, third + 3, ...
    const int third = ew >> 2;
    const int nb = (kPairTile / 32 - third + kEpiPerQuad - 1) / kEpiPerQuad;
    const int r_pair = static_cast<int>(rank) * 128 + quad * 32 + lane;
    // This warp's 4 KB staging area: a 32 x 32 bf16 output block, or the
    // fp32 block of the weight update.
    __nv_bfloat16* stg_d = out_stage + ew * 2 * Cfg::kOutBlockElems;
    float* stage_f32 = reinterpret_cast<float*>(stg_d);
    // Stores v (lane = row) as bf16 at rows row0_ .., columns col0_ .. of
    // dst (leading dimension ld; rows below max_r, 8-column chunks starting
    // below max_c, which ld covers).  The block goes through shared
    // memory so that every global store instruction writes eight whole
    // 64-byte row segments; the 16-byte chunks of a staged row are
    // XOR-swizzled by (row / 2) % 4, which keeps both the row writes and the
    // segment reads free of bank conflicts.
    auto put_block = [&](__nv_bfloat16* dst, int ld, int rows_alloc, int max_r, int max_c,
                         int row0_, int col0_, const float (&v)[32]) {
      uint4* srow = reinterpret_cast<uint4*>(stg_d) + lane * 4;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        __nv_bfloat162 h[4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
          h[i] = __floats2bfloat162_rn(v[8 * q + 2 * i], v[8 * q + 2 * i + 1]);
        srow[q ^ ((lane >> 1) & 3)] = *reinterpret_cast<uint4*>(h);
      }
      __syncwarp();
      const int c = lane & 3;
      // Device-checked build: every 8-element piece stays inside its row of
      // the buffer (rows_alloc rows of ld elements), else it is skipped and
      // the row recorded.
      auto store_ok = [&](int gr, int gc) -> bool {
        if constexpr (!kDeviceChecks) {
          return true;
        } else {
          if (gr >= 0 && gr < rows_alloc && gc >= 0 && gc + 8 <= ld) return true;
          record_check_failure(p.err, kErrCheckStore, gr);
          return false;
        }
      };
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int rr = 8 * i + (lane >> 2);
        const uint4 val = reinterpret_cast<const uint4*>(stg_d)[rr * 4 + (c ^ ((rr >> 1) & 3))];
        const int gr = row0_ + rr, gc = col0_ + 8 * c;
        if (gr < max_r && gc < max_c && store_ok(gr, gc))
          *reinterpret_cast<uint4*>(dst + static_cast<size_t>(gr) * ld + gc) = val;
      }
      __syncwarp();   // staging free for the next block
    };
    const uint32_t leader_tempty0 = mapa_shared(tempty_bar(0), 0);
    // Called after this warp's last accumulator read of an item: the leader
    // may start the item after next in this accumulator while this one is
    // still being stored.
    auto release_acc = [&](int acc_) {
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (leader) mbar_arrive_relaxed(tempty_bar(acc_));
        else mbar_arrive_cluster_relaxed(leader_tempty0 + 8u * acc_);
      }
    };
    int lt = 0;
    uint4 nx = load_item_raw(p, pair);
    for (int g = pair; g < total; g += npairs, ++lt) {
      const MegaItem item = unpack_item(nx);
      nx = load_item_raw(p, g + npairs);
      if (!item_ok(item, g)) break;
      const NsTile tl = item.tl;
      const MatDev* md = p.mats + tl.mat;
      const int acc = lt & 1;
      const uint32_t aph = (lt >> 1) & 1;
      const int row0 = tl.ti * kPairTile + static_cast<int>(rank) * 128 + quad * 32;
      const int row = row0 + lane;
      const int m = md->m;
      const bool row_ok = row < m;
      const bool first = item.k == 0;
      const bool last = item.k == p.steps - 1;
      const int colw = tl.tj * kPairTile + third * 32;   // this warp's first block
      // Inputs that do not depend on the accumulator are requested before
      // waiting for it: the last step's W blocks, the poly's rows of A.
      float wa[32], wb[32];
      uint4 ar[2][4];
      // The first step's products carry the Frobenius scale (gram s^2, apply
      // s), summed from the partials while the tensor cores run.
      const float s = first && item.mode != kModePoly
                          ? frob_scale(p.partials, md, lane, p.eps_frob) : 1.f;
      if (item.mode == kModeApply && last) {
        load_w_block(md, row0, colw, lane, wa);
      } else if (item.mode == kModePoly) {
        // The generic reads of A need the gram stores of other CTAs.
        if (lane == 0) {
          if (!wait_count(done_counter(p, tl.mat, item.k, kModeGram), item.dep_target,
                          abort_flag, p.err))
            fail(kErrTimeoutEpilogue);
        }
        __syncwarp();
        // this lane's row of A under the first two blocks (the third is
        // requested once the first has been used)
        if (row_ok) {
          const __nv_bfloat16* arow = md->a + static_cast<size_t>(row) * md->lda;
#pragma unroll
          for (int j = 0; j < 2; ++j)
            load_row32_bf16_raw(arow, colw + 32 * kEpiPerQuad * j, m, ar[j]);
        }
      }
      if (!mbar_wait_bounded(tfull_bar(acc), aph, abort_flag)) {
        fail(kErrTimeoutEpilogue);
        break;
      }
      tc_fence_after();
      const uint32_t tbase = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) +
                             static_cast<uint32_t>(acc * kPairTile);

      if (item.mode == kModeGram || item.mode == kModePoly) {
        const bool diag_tile = tl.ti == tl.tj;
        const bool poly = item.mode == kModePoly;
        // gram: s^2 X X^T;  poly: a I + b A + c A A (A A from the accumulator)
        const float mul = poly ? p.c[item.k] : s * s;
        const float pb = p.b[item.k];
        const float pa = p.a[item.k];
        // Block j (columns colw + 96 j) with this lane's A row in `cur`.
        auto block = [&](int j, const uint4 (&cur)[4]) {
          const int cc = third + kEpiPerQuad * j;
          const int col0 = colw + 32 * kEpiPerQuad * j;
          float v[32];
          tmem_load_32cols(tbase + cc * 32, v);
          if (j == nb - 1) release_acc(acc);
          if (poly) {
            float av[32];
            unpack_row32_bf16(cur, av);
#pragma unroll
            for (int e = 0; e < 32; ++e) v[e] = row_ok ? fmaf(pb, av[e], mul * v[e]) : 0.f;
            if (diag_tile && (r_pair >> 5) == cc) {
              const int d = r_pair & 31;
#pragma unroll
              for (int e = 0; e < 32; ++e)
                if (e == d) v[e] += pa;
            }
          } else {
#pragma unroll
            for (int e = 0; e < 32; ++e) v[e] *= mul;
          }
          put_block(poly ? md->b : md->a, md->lda, m, m, m, row0, col0, v);
        };
        block(0, ar[0]);
        if (poly && nb > 2 && row_ok)
          load_row32_bf16_raw(md->a + static_cast<size_t>(row) * md->lda,
                              colw + 2 * 32 * kEpiPerQuad, m, ar[0]);
        block(1, ar[1]);
        if (nb > 2) block(2, ar[0]);
      } else if (!last) {
#pragma unroll 1
        for (int cc = third; cc < kPairTile / 32; cc += kEpiPerQuad) {
          const int col0 = tl.tj * kPairTile + cc * 32;
          float v[32];
          tmem_load_32cols(tbase + cc * 32, v);
          if (cc + kEpiPerQuad >= kPairTile / 32) release_acc(acc);
          if (first) {
#pragma unroll
            for (int e = 0; e < 32; ++e) v[e] *= s;
          }
          put_block(md->x[(item.k & 1) ^ 1], md->ldx, m, m, md->n, row0, col0, v);
        }
      } else {
        // W <- W (1 - lr wd) - lr scale O over this warp's two or three
        // blocks; each block's W is already in registers when it is stored
        // (loaded one block ahead, the first before the accumulator was
        // ready: two blocks ahead do not fit the 152-register budget).
        const float lr = p.lr_dev ? *p.lr_dev : p.lr;
        const float decay = 1.f - lr * p.wd;
        const float step = lr * md->update_scale;
        auto block = [&](int j, float (&wv)[32]) {
          float v[32];
          tmem_load_32cols(tbase + (third + kEpiPerQuad * j) * 32, v);
          if (j == nb - 1) release_acc(acc);
          if (first) {
#pragma unroll
            for (int e = 0; e < 32; ++e) v[e] *= s;
          }
          store_w_block(md, row0, colw + 32 * kEpiPerQuad * j, lane, decay, step, wv, v,
                        stage_f32, p.err);
          if (j + 1 < nb) load_w_block(md, row0, colw + 32 * kEpiPerQuad * (j + 1), lane, wv);
        };
        block(0, wa);
        block(1, wa);
        if (nb > 2) block(2, wa);
      }
      // Hand the item to the signal warp (the arrival releases this warp's
      // stores to it).  Its barrier slot was last used four items ago; that
      // item must have been published first, or the slot's phases would run
      // ahead of the signal warp.
      __syncwarp();
      bool ok = true;
      if (lane == 0) {
        if (lt >= Cfg::kEpiBars) {
          const uint64_t t0 = global_timer_ns();
          while (*sig_count < lt - Cfg::kEpiBars + 1) {
            if (*abort_flag || global_timer_ns() - t0 > kWaitLimitNs) {
              fail(kErrTimeoutEpilogue);
              ok = false;
              break;
            }
            __nanosleep(32);
          }
        }
        if (ok) mbar_arrive(epi_bar(lt % Cfg::kEpiBars));
      }
      if (!__shfl_sync(0xffffffffu, ok ? 1 : 0, 0)) break;
    }
  }

  tc_fence_before();
  __syncthreads();
  __syncwarp();
  cluster_sync_all();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc_pair(tmem_base, Cfg::kTmemCols);
  }
}

}  // namespace muonb200
