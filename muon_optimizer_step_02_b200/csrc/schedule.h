// Host-side schedule of the persistent Newton-Schulz kernel.
//
// The kernel runs a list of items (pair tiles of gram / poly / apply of every
// step and matrix); cluster c executes list positions c, c + C, c + 2C, ...
// in order and waits in-kernel until the phase an item reads is complete.
// The order decides how often clusters stall, not correctness; every
// dependency must precede its dependants (the kernel's deadlock-freedom
// condition).  The order built here is phase-major: for each step the gram
// tiles of all matrices, then the poly tiles, then the apply tiles, each
// phase longest first (matrix order among equals).  A simulation of the
// clusters under a simple cost model (tensor cycles per 64-deep K block plus
// a fixed cost per item) gives its makespan; a greedy ready-first list
// scheduler was tried under the same model and came out worse, because with
// a fixed round-robin assignment an idle wait cannot be handed to another
// cluster.  Uses only caller-provided arrays: no allocation.
#pragma once

#include <cstdint>

#include "muon_types.cuh"

namespace muonb200 {

struct SchedMatrix {
  int m, n;          // working shape
  int t2;            // 256-row blocks of m
  int tn;            // 256-column blocks of n
};

struct SchedGroup {
  int mat, k, mode;
  int size;          // tiles in this (matrix, step, phase)
  int placed;
  double done;       // simulated finish of the last placed tile
  int dep;           // group whose completion this one reads, or -1
};

inline int sched_group_index(int mat, int k, int mode, int steps) {
  return (mat * steps + k) * 3 + mode;
}

inline int sched_ceil_div(int a, int b) { return (a + b - 1) / b; }

// Whether a work item lies inside its matrix's tile grid and carries the
// K-block count and dependency target of its phase: m x n working shape
// (m <= n), `steps` Newton-Schulz steps.  The device-checked build of the
// tensor-core kernel calls it on every item it decodes, before any access.
__host__ __device__ inline bool sched_item_valid(int mode, int k, int ti, int tj, int kt,
                                                 int dep_target, int m, int n, int steps) {
  if (mode < 0 || mode > 2 || k < 0 || k >= steps || m < 1 || n < m) return false;
  const int t2 = (m + kPairTile - 1) / kPairTile, tn = (n + kPairTile - 1) / kPairTile;
  if (ti < 0 || ti >= t2) return false;
  if (mode == kModeApply ? (tj < 0 || tj >= tn) : (tj < ti || tj >= t2)) return false;
  if (kt != (mode == kModeGram ? (n + kTileK - 1) / kTileK : (m + kTileK - 1) / kTileK))
    return false;
  const int sym = t2 * (t2 + 1) / 2, app = t2 * tn;
  const int want = mode == kModeGram ? (k == 0 ? 0 : 2 * app) : 2 * sym;
  return dep_target == want;
}

// Item cost in tensor-core cycles of one CTA pair (256 x 256 x 64 per K
// block) plus a fixed per-item cost; the last step's apply also moves W.
inline double sched_cost(const SchedMatrix& mm, int mode, int k, int steps) {
  const int kt = mode == kModeGram ? sched_ceil_div(mm.n, kTileK)
                                   : sched_ceil_div(mm.m, kTileK);
  double c = 512.0 * kt + 3000.0;
  if (mode == kModeApply && k == steps - 1) c += 12000.0;
  return c;
}

// Tile `idx` of a group: upper pair blocks for gram/poly, all blocks for apply.
inline void sched_tile(const SchedMatrix& mm, int mode, int idx, int& ti, int& tj) {
  if (mode == kModeApply) {
    ti = idx / mm.tn;
    tj = idx % mm.tn;
    return;
  }
  int i = 0;
  while (idx >= mm.t2 - i) {
    idx -= mm.t2 - i;
    ++i;
  }
  ti = i;
  tj = i + idx;
}

// Order of the list: matrices form groups of consecutive plan entries whose
// working buffers (X ping and pong, A, B') add up to about group_bytes; the
// 3K phases of group g start `lag` phase slots after those of group g - 1.
// Slot t holds phase t - lag g of every group g for which that phase exists,
// older groups first, each phase's matrices longest first and each matrix's
// tiles consecutive.  lag = 0 (or one group) is the phase-major order; a lag
// keeps only the buffers of the groups in flight live at a time (so that
// they can stay in L2) and spreads the last step's weight updates, which
// move W, over the launch instead of leaving them all for its end.
struct SchedPolicy {
  double group_bytes;  // target working-buffer bytes of one group
  int lag;             // phase slots between the starts of consecutive groups
};

// Working-buffer bytes of one matrix in the workspace (bf16 X ping and pong,
// A and B').
inline double sched_matrix_bytes(const SchedMatrix& mm) {
  return 2.0 * (2.0 * mm.m * mm.n + 2.0 * mm.m * mm.m);
}

// Returns the number of items written to `out` (capacity `cap`), or -1.
// `groups` needs n_mats * steps * 3 entries, `order` (scratch) 2 * n_mats
// + 1 ints, `cl_time` `clusters` doubles (the simulated finish time of each
// cluster).
inline long long build_schedule(const SchedMatrix* mats, int n_mats, int steps,
                                int clusters, SchedPolicy pol, SchedItem* out,
                                long long cap, SchedGroup* groups, int* order,
                                double* cl_time) {
  long long total = 0;
  for (int i = 0; i < n_mats; ++i)
    for (int k = 0; k < steps; ++k)
      for (int mode = 0; mode < 3; ++mode) {
        SchedGroup& g = groups[sched_group_index(i, k, mode, steps)];
        g.mat = i;
        g.k = k;
        g.mode = mode;
        g.size = mode == kModeApply ? mats[i].t2 * mats[i].tn
                                    : mats[i].t2 * (mats[i].t2 + 1) / 2;
        g.placed = 0;
        g.done = 0.0;
        g.dep = mode == kModeGram ? (k == 0 ? -1 : sched_group_index(i, k - 1, kModeApply, steps))
                                  : sched_group_index(i, k, mode - 1, steps);
        total += g.size;
      }
  if (total > cap) return -1;
  for (int c = 0; c < clusters; ++c) cl_time[c] = 0.0;

  // wave groups: first matrix of group w in gstart[w], gstart[n_groups] = n_mats
  int* gstart = order + n_mats;
  int n_groups = 0;
  {
    double acc = 0.0;
    gstart[0] = 0;
    for (int i = 0; i < n_mats; ++i) {
      acc += sched_matrix_bytes(mats[i]);
      if (acc >= pol.group_bytes && i + 1 < n_mats) {
        gstart[++n_groups] = i + 1;
        acc = 0.0;
      }
    }
    gstart[++n_groups] = n_mats;
  }
  const int lag = pol.lag > 0 ? pol.lag : 0;
  const int n_phases = 3 * steps;
  const int n_slots = n_phases + lag * (n_groups - 1);

  long long pos = 0;
  for (int t = 0; t < n_slots; ++t)
    for (int w = 0; w < n_groups; ++w) {
      const int q = lag == 0 ? t : t - lag * w;
      if (q < 0 || q >= n_phases) continue;
      if (lag == 0 && w > 0) continue;   // phase-major: one pass over all matrices
      const int k = q / 3, mode = q % 3;
      const int lo = lag == 0 ? 0 : gstart[w], hi = lag == 0 ? n_mats : gstart[w + 1];
      // matrices of this phase, longest item first (insertion sort, stable)
      for (int i = lo; i < hi; ++i) {
        int j = i - lo;
        const double ci = sched_cost(mats[i], mode, k, steps);
        while (j > 0 && sched_cost(mats[order[j - 1]], mode, k, steps) < ci) {
          order[j] = order[j - 1];
          --j;
        }
        order[j] = i;
      }
      // all tiles of one matrix consecutively, so that each matrix's phase
      // completes as early as possible
      for (int x = 0; x < hi - lo; ++x) {
        const int mi = order[x];
        SchedGroup& g = groups[sched_group_index(mi, k, mode, steps)];
        const SchedMatrix& mm = mats[mi];
        const double dep_t = g.dep < 0 ? 0.0 : groups[g.dep].done;
        const double cost = sched_cost(mm, mode, k, steps);
        for (int tt = 0; tt < g.size; ++tt) {
          int ti = 0, tj = 0;
          sched_tile(mm, mode, tt, ti, tj);
          SchedItem& it = out[pos];
          it.mat = static_cast<uint16_t>(mi);
          it.ti = static_cast<uint16_t>(ti);
          it.tj = static_cast<uint16_t>(tj);
          it.kt = static_cast<uint16_t>(mode == kModeGram ? sched_ceil_div(mm.n, kTileK)
                                                           : sched_ceil_div(mm.m, kTileK));
          it.mode = static_cast<uint8_t>(mode);
          it.k = static_cast<uint8_t>(k);
          it.pad = 0;
          it.dep_target = g.dep < 0 ? 0 : 2 * groups[g.dep].size;
          // simulation: in-order execution on cluster pos % clusters
          const int c = static_cast<int>(pos % clusters);
          const double start = cl_time[c] > dep_t ? cl_time[c] : dep_t;
          cl_time[c] = start + cost;
          g.placed += 1;
          if (cl_time[c] > g.done) g.done = cl_time[c];
          ++pos;
        }
      }
    }
  return pos;
}

// The order the library uses: phase-major (lag 0).  Measured on B200 with the
// 11L x 512d set (66 matrices, K = 5; outputs bit-identical across orders),
// Newton-Schulz kernel time per launch: phase-major 0.402 ms; waves of one
// layer (15 MB) with lags of 1, 2, 3 phases 0.510, 0.597, 0.737 ms; two
// layers (31 MB) with lags 3 and 6 0.566 and 0.720 ms; 8 MB groups, lag 2,
// 0.745 ms.  Keeping fewer matrices in flight lets their buffers stay in L2
// but exposes each matrix's 15-phase dependency chain, which costs more.
inline SchedPolicy default_policy() { return SchedPolicy{0.0, 0}; }

}  // namespace muonb200
