// C ABI of the batched Muon step and the batched EMA (include/muon_b200.h):
// argument validation, the plan (shapes -> workspace layout, prologue work
// items and the Newton-Schulz schedule, built once), TMA descriptor
// encoding, and the launch sequence on the caller's stream:
//
//   counter reset (memset) -> prologue -> all Newton-Schulz steps (one
//   persistent CTA-pair kernel)                      or, with 0 steps,
//   counter reset -> prologue -> finisher
//
// No device memory is allocated after muon_plan_create.
#include <cuda.h>
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <new>
#include <vector>

#include "muon_b200.h"


#include "k_adamw_ema.cuh"
#include "k_convert.cuh"
#include "k_ema.cuh"
#include "k_ns_mega.cuh"
#include "k_prologue.cuh"
#include "muon_types.cuh"
#include "schedule.h"

using namespace muonb200;

namespace {

constexpr int kMaxNsSteps = 16;
constexpr int kMaxMats = 4096;
constexpr int kMaxLaunchesPerStep = 3;   // timed segments of one step
constexpr int kTimingSlots = 64;
constexpr size_t kProSmemCap = 48 * 1024;   // staging of the transposed write

inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Every device allocation of the library goes through dev_alloc, which counts
// successful ones (muon_device_allocation_count).
std::atomic<long long> g_device_allocations{0};

cudaError_t dev_alloc(void** p, size_t bytes) {
  const cudaError_t e = cudaMalloc(p, bytes);
  if (e == cudaSuccess) g_device_allocations.fetch_add(1, std::memory_order_relaxed);
  return e;
}
inline int ceil_div(int a, int b) { return (a + b - 1) / b; }

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t,
                                  void*, const cuuint64_t*, const cuuint64_t*,
                                  const cuuint32_t*, const cuuint32_t*,
                                  CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000,
                                         cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// bf16 matrix of `rows` x `cols` elements with leading dimension `ld`,
// boxes of box_cols x box_rows, 128-byte swizzle (the tensor-core operand
// layout in shared memory).
bool encode_bf16_2d(CUtensorMap* tm, void* base, int rows, int cols, int ld,
                    int box_cols, int box_rows) {
  EncodeTiledFn fn = get_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols),
                        static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld) * 2};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(box_cols),
                       static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  return fn(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Per-matrix geometry and its place in the workspace.
struct Geom {
  int rows, cols, m, n, ldx, lda, transposed;
  size_t x_off[2], a_off, b_off;
  int part_first, part_count;
  int t2, tn;                      // 256-blocks of m and of n
  int n_sym_tiles, n_apply_tiles;  // pair tiles per phase
};

// Stored rows per prologue work item.  A transposed item is staged in shared
// memory whole: up to kProSmemCap in the two-pass kernel (three blocks per
// SM), up to kProTransBufCap in the one-pass kernel (two blocks per SM).
int pro_rows_per_item(int rows, int cols) {
  if (rows <= cols) return kProRows;
  const size_t cap = pro_one_pass(cols) ? kProTransBufCap : kProSmemCap;
  const size_t per_row = static_cast<size_t>(cols + 2) * 2;
  int rt = static_cast<int>(std::min<size_t>(kProRows, cap / per_row));
  if (rt >= 8) rt &= ~7;
  return std::max(rt, 1);
}

// Shared memory of one transposed staging buffer of the matrix (0 when the
// matrix is not transposed).
size_t pro_trans_bytes(int rows, int cols) {
  if (rows <= cols) return 0;
  return static_cast<size_t>(pro_rows_per_item(rows, cols)) * (cols + 2) * 2;
}

// Shape checks, geometry, and the workspace offsets of X ping/pong, A, B'.
muon_status_t layout_matrix(int rows, int cols, Geom& g, size_t& off) {
  if (rows < 1 || cols < 1) return MUON_ERR_INVALID_ARG;
  // tile coordinates are 16-bit; keep every dimension well inside
  if (rows > (1 << 20) || cols > (1 << 20) ||
      static_cast<long long>(rows) * cols > (1ll << 31) - 1)
    return MUON_ERR_UNSUPPORTED;
  g.rows = rows;
  g.cols = cols;
  g.transposed = rows > cols;
  g.m = std::min(rows, cols);
  g.n = std::max(rows, cols);
  g.ldx = static_cast<int>(align_up(g.n, 8));
  g.lda = static_cast<int>(align_up(g.m, 8));
  for (int b = 0; b < 2; ++b) {
    g.x_off[b] = off;
    off = align_up(off + static_cast<size_t>(g.m) * g.ldx * 2, 1024);
  }
  g.a_off = off;
  off = align_up(off + static_cast<size_t>(g.m) * g.lda * 2, 1024);
  g.b_off = off;
  off = align_up(off + static_cast<size_t>(g.m) * g.lda * 2, 1024);
  g.t2 = ceil_div(g.m, kPairTile);
  g.tn = ceil_div(g.n, kPairTile);
  g.n_sym_tiles = g.t2 * (g.t2 + 1) / 2;
  g.n_apply_tiles = g.t2 * g.tn;
  return MUON_OK;
}

// Counters of one step: one completion count per (matrix, step, phase),
// zeroed by the prologue.
int counters_for(int n_mats, int steps) { return n_mats * 3 * std::max(steps, 1); }

// Prologue work items, each with its partial-sum slot (the matrix's items
// keep consecutive slots): the one-pass items first, then the two-pass ones,
// each part listed largest first for its persistent kernel (ties in slot
// order).  Returns the number of one-pass items.  std::sort: no allocation.
int order_prologue_items(ProItem* items, int n, const Geom* geom) {
  std::sort(items, items + n, [geom](const ProItem& a, const ProItem& b) {
    const bool oa = pro_one_pass(geom[a.mat].cols), ob = pro_one_pass(geom[b.mat].cols);
    if (oa != ob) return oa;
    const long long wa = static_cast<long long>(a.nrows) * geom[a.mat].cols;
    const long long wb = static_cast<long long>(b.nrows) * geom[b.mat].cols;
    return wa != wb ? wa > wb : a.part < b.part;
  });
  int n_one = 0;
  while (n_one < n && pro_one_pass(geom[items[n_one].mat].cols)) ++n_one;
  return n_one;
}

// Blocks of a persistent prologue kernel: all resident at once, at most one
// per item (0 when there are no items).
template <bool kOnePass>
int prologue_grid(int n_items, size_t pro_smem) {
  if (n_items <= 0) return 0;
  int dev = 0, sms = 0, per_sm = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, muon_prologue_kernel<kOnePass>,
                                                    kProThreads, pro_smem) != cudaSuccess) {
    cudaGetLastError();
    return -1;
  }
  return std::max(1, std::min(n_items, sms * std::max(per_sm, 1)));
}

// Dynamic shared memory of the one-pass prologue: the staging buffer of its
// largest transposed item (0 when no one-pass matrix is transposed).
size_t one_pass_smem(const Geom* geom, int n_mats) {
  size_t tb = 0;
  for (int i = 0; i < n_mats; ++i)
    if (pro_one_pass(geom[i].cols))
      tb = std::max(tb, pro_trans_bytes(geom[i].rows, geom[i].cols));
  return tb;
}

// Whether the one-pass prologue prefetches each warp's next row into L2.
// Measured on B200: the prefetch shortens the pass by 3-6% while the
// one-pass matrices hold up to ~32M elements (the 11L stack), and lengthens
// it by 2-13% at 100M (24L MLP matrices), where the loads alone keep HBM
// busy; the cut-off sits between the two.
constexpr size_t kProPrefetchMaxElems = size_t(48) << 20;

int one_pass_prefetch(const Geom* geom, int n_mats) {
  size_t elems = 0;
  for (int i = 0; i < n_mats; ++i)
    if (pro_one_pass(geom[i].cols))
      elems += static_cast<size_t>(geom[i].rows) * geom[i].cols;
  return elems <= kProPrefetchMaxElems ? 1 : 0;
}

struct TimingSlot {
  cudaEvent_t ev[kMaxLaunchesPerStep + 1];
  int kind[kMaxLaunchesPerStep];
  int n = 0;
  bool pending = false;
};

bool finite(float v) { return std::isfinite(v); }
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

struct muon_plan {
  int device = 0;
  int num_sms = 148;
  int n_mats = 0;
  int max_ns = 0;
  std::vector<Geom> geom;
  std::vector<ProItem> items;
  size_t ws_bytes = 0;
  size_t part_off = 0;
  size_t scale_off = 0;
  size_t counter_off = 0;
  size_t lr_slot_off = 0;
  size_t pro_smem = 0;
  int n_one = 0;       // one-pass prologue items (listed first)
  size_t pro_smem_one = 0;    // dynamic shared memory of the one-pass prologue
  int pro_grid[2] = {0, 0};   // blocks of the one-pass and two-pass prologues
  int pro_prefetch = 0;       // one-pass prologue prefetches the next row
  int max_clusters = 0;

  // Newton-Schulz schedule for `sched_steps` steps (rebuilt when the step
  // count of a call changes)
  std::vector<SchedMatrix> smats;
  std::vector<SchedItem> sched;
  std::vector<SchedGroup> sgroups;
  std::vector<int> sorder;
  std::vector<double> scl;
  int sched_steps = -1;
  long long sched_len = 0;
  long long sched_cap = 0;

  // device table: [MatDev x n_mats][ProItem][SchedItem x cap][err]
  void* d_block = nullptr;
  MatDev* d_mats = nullptr;
  ProItem* d_items = nullptr;
  SchedItem* d_sched = nullptr;
  int32_t* d_err = nullptr;

  std::vector<MatDev> h_mats;     // what the device table holds now
  bool h_valid = false;
  void* enc_ws = nullptr;         // workspace the tensor maps were encoded for

  int fault = 0;
  bool timing = false;
  std::vector<TimingSlot> slots;
  int slot_head = 0;
  double kind_ms[MUON_KIND_COUNT] = {};
  long long kind_launches[MUON_KIND_COUNT] = {};
};

namespace {

void harvest(muon_plan* plan, TimingSlot& s) {
  if (!s.pending) return;
  cudaEventSynchronize(s.ev[s.n]);
  for (int i = 0; i < s.n; ++i) {
    float ms = 0.f;
    if (cudaEventElapsedTime(&ms, s.ev[i], s.ev[i + 1]) == cudaSuccess) {
      plan->kind_ms[s.kind[i]] += ms;
      plan->kind_launches[s.kind[i]] += 1;
    }
  }
  s.pending = false;
}

// CUDA events on the launching stream around each launch of one call.
struct Recorder {
  muon_plan* plan;
  cudaStream_t stream;
  TimingSlot* slot = nullptr;
  Recorder(muon_plan* p, cudaStream_t s) : plan(p), stream(s) {
    if (!plan->timing) return;
    slot = &plan->slots[plan->slot_head];
    plan->slot_head = (plan->slot_head + 1) % kTimingSlots;
    harvest(plan, *slot);
    slot->n = 0;
    cudaEventRecord(slot->ev[0], stream);
  }
  void after(int kind) {
    if (!slot) return;
    slot->kind[slot->n] = kind;
    cudaEventRecord(slot->ev[slot->n + 1], stream);
    slot->n += 1;
  }
  void finish() {
    if (slot && slot->n > 0) slot->pending = true;
  }
};

// Everything the launch sequence needs: where the device tables are.
struct LaunchTables {
  const MatDev* mats;
  const ProItem* items;
  int n_items;
  int n_one;          // one-pass prologue items (the first n_one of `items`)
  const SchedItem* sched;
  long long n_sched;
  int32_t* err;
  size_t pro_smem;      // two-pass prologue
  size_t pro_smem_one;  // one-pass prologue
  int pro_grid[2];      // blocks of the one-pass and two-pass prologues
  int clusters;       // clusters the schedule was built for (all resident)
  int pro_prefetch;     // one-pass prologue prefetches the next row into L2
};

// Scratch of one step inside the workspace.
struct StepScratch {
  float* partials;    // one per prologue item
  float* mat_scale;   // one per matrix
  int32_t* counters;  // done: n_mats * K * 3, zeroed by the prologue
  int n_counters;
  int n_mats;
  float* lr_slot;     // the scheduled learning rate of the step (or null)
};

muon_status_t validate_hyper(const muon_hyper_t* hyper, const float* ns_coeffs,
                             int32_t ns_steps, int32_t max_ns) {
  if (!hyper) return MUON_ERR_INVALID_ARG;
  if (ns_steps < 0 || ns_steps > max_ns) return MUON_ERR_UNSUPPORTED;
  if (ns_steps > 0 && !ns_coeffs) return MUON_ERR_INVALID_ARG;
  for (int k = 0; k < 3 * ns_steps; ++k)
    if (!finite(ns_coeffs[k])) return MUON_ERR_INVALID_ARG;
  const muon_hyper_t& h = *hyper;
  if (!finite(h.momentum) || !finite(h.lr) || !finite(h.weight_decay) ||
      !finite(h.eps_row) || !finite(h.eps_frob) || h.eps_row < 0.f ||
      h.eps_frob < 0.f || (h.nesterov != 0 && h.nesterov != 1) ||
      (h.eq_r != 0 && h.eq_r != 1))
    return MUON_ERR_INVALID_ARG;
  return MUON_OK;
}

muon_status_t validate_matrix(const muon_matrix_t& mt, const Geom& g) {
  if (mt.rows != g.rows || mt.cols != g.cols) return MUON_ERR_UNSUPPORTED;
  if (!mt.w || !mt.momentum || !mt.grad_bf16) return MUON_ERR_INVALID_ARG;
  if (!finite(mt.update_scale)) return MUON_ERR_INVALID_ARG;
  if (!aligned16(mt.w) || !aligned16(mt.momentum) || !aligned16(mt.grad_bf16) ||
      (mt.update_out && !aligned16(mt.update_out)))
    return MUON_ERR_ALIGNMENT;
  return MUON_OK;
}

// Workspace-dependent part of a matrix record: buffer pointers, tensor maps,
// geometry.
bool fill_workspace_fields(MatDev& d, const Geom& g, char* ws) {
  std::memset(&d, 0, sizeof(MatDev));
  for (int b = 0; b < 2; ++b) {
    d.x[b] = reinterpret_cast<__nv_bfloat16*>(ws + g.x_off[b]);
    if (!encode_bf16_2d(&d.tm_xk[b], d.x[b], g.m, g.n, g.ldx, kTileK, kTileM) ||
        !encode_bf16_2d(&d.tm_xn[b], d.x[b], g.m, g.n, g.ldx, 64, kTileK))
      return false;
  }
  d.a = reinterpret_cast<__nv_bfloat16*>(ws + g.a_off);
  d.b = reinterpret_cast<__nv_bfloat16*>(ws + g.b_off);
  if (!encode_bf16_2d(&d.tm_a, d.a, g.m, g.m, g.lda, kTileK, kTileM) ||
      !encode_bf16_2d(&d.tm_b, d.b, g.m, g.m, g.lda, kTileK, kTileM) ||
      !encode_bf16_2d(&d.tm_an, d.a, g.m, g.m, g.lda, 64, kTileK) ||
      !encode_bf16_2d(&d.tm_bn, d.b, g.m, g.m, g.lda, 64, kTileK))
    return false;
  d.rows = g.rows;
  d.cols = g.cols;
  d.m = g.m;
  d.n = g.n;
  d.ldx = g.ldx;
  d.lda = g.lda;
  d.transposed = g.transposed;
  d.part_first = g.part_first;
  d.part_count = g.part_count;
  d.n_sym_tiles = g.n_sym_tiles;
  d.n_apply_tiles = g.n_apply_tiles;
  return true;
}

// Caller-pointer part of a matrix record; returns true if it changed.
bool fill_caller_fields(MatDev& d, const muon_matrix_t& mt) {
  if (d.w == mt.w && d.mom == mt.momentum && d.g == mt.grad_bf16 &&
      d.out == mt.update_out &&
      std::memcmp(&d.update_scale, &mt.update_scale, sizeof(float)) == 0)
    return false;
  d.w = mt.w;
  d.mom = mt.momentum;
  d.g = mt.grad_bf16;
  d.out = mt.update_out;
  d.update_scale = mt.update_scale;
  return true;
}

// The dynamic shared memory limit of a kernel (cudaFuncAttributeMax-
// DynamicSharedMemorySize) is a per-device, process-wide setting.  Plans of
// different shapes need different prologue staging sizes, so the limit is
// only ever raised: each kernel keeps, per device, the largest value set so
// far (under a mutex), and a plan needing less leaves it alone.  Lowering it
// would make the launches of an earlier plan that needs more fail.
constexpr int kMaxDevices = 64;
struct SmemLimits {
  size_t ns = 0, pro_two = 0, pro_one = 0;
};
std::mutex g_smem_mutex;
SmemLimits g_smem_limits[kMaxDevices];

bool raise_smem_limit(const void* fn, size_t& cur, size_t want) {
  if (want <= cur) return true;
  if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(want)) != cudaSuccess)
    return false;
  cur = want;
  return true;
}

// (a limit is set whenever there is dynamic shared memory: static plus
// dynamic above 48 KB needs the opt-in even when the dynamic part alone is
// below it)
bool set_kernel_attributes(size_t pro_smem, size_t pro_smem_one) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return false;
  std::lock_guard<std::mutex> lock(g_smem_mutex);
  SmemLimits& lim = g_smem_limits[dev];
  return raise_smem_limit(reinterpret_cast<const void*>(ns_mega_pair_kernel), lim.ns,
                          kMegaSmemBytes) &&
         raise_smem_limit(reinterpret_cast<const void*>(muon_prologue_kernel<false>),
                          lim.pro_two, pro_smem) &&
         raise_smem_limit(reinterpret_cast<const void*>(muon_prologue_kernel<true>),
                          lim.pro_one, pro_smem_one);
}

// Launch configuration of the tensor-core kernel: clusters of two CTAs and,
// with `pdl`, programmatic stream serialization (the kernel may start while
// the prologue before it finishes; it waits for it in-kernel).  attr needs
// two entries.
cudaLaunchConfig_t pair_launch_config(int clusters, cudaStream_t st,
                                      cudaLaunchAttribute* attr, bool pdl) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * clusters);
  cfg.blockDim = dim3(kNsThreads);
  cfg.dynamicSmemBytes = kMegaSmemBytes;
  cfg.stream = st;
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 2 : 1;
  return cfg;
}

// Clusters of two that can be resident at once (the persistent schedule
// relies on every launched cluster being resident); 0 on failure.
int query_max_clusters() {
  if (!set_kernel_attributes(0, 0)) {
    cudaGetLastError();
    return 0;
  }
  cudaLaunchAttribute attr[2];
  cudaLaunchConfig_t cfg = pair_launch_config(1, nullptr, attr, false);
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, ns_mega_pair_kernel, &cfg) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  return n;
}

void fill_sched_matrix(SchedMatrix& s, const Geom& g) {
  s.m = g.m;
  s.n = g.n;
  s.t2 = g.t2;
  s.tn = g.tn;
}

// prologue (which also zeroes the step's counters) -> Newton-Schulz, a
// programmatic dependent of the prologue that sums the Frobenius partials
// itself; or, with 0 steps, prologue -> Frobenius scale -> finisher.  Each
// launch is checked as it
// is made: if the runtime refuses one, nothing after it is enqueued (a later
// kernel would otherwise run on partials and counters the refused one never
// wrote) and MUON_ERR_CUDA is returned; the launches before it have run.
muon_status_t enqueue_step(const LaunchTables& t, const muon_hyper_t& h,
                  const muon_schedule_t* sched, int32_t* step_dev,
                  const float* ns_coeffs, int32_t ns_steps, const StepScratch& sc,
                  int fault, bool fresh, cudaStream_t st, Recorder* rec) {
  HyperDev hd{};
  hd.mu = h.momentum;
  hd.lr = h.lr;
  hd.wd = h.weight_decay;
  hd.eps_row = h.eps_row;
  hd.eps_frob = h.eps_frob;
  hd.nesterov = h.nesterov;
  hd.eq_r = h.eq_r;
  const float* lr_dev = nullptr;
  if (sched) {
    hd.step = step_dev;
    hd.lr_slot = sc.lr_slot;
    hd.mu_v0 = sched->momentum.v0;
    hd.mu_v1 = sched->momentum.v1;
    hd.mu_t0 = sched->momentum.t0;
    hd.mu_t1 = sched->momentum.t1;
    hd.lr_v0 = sched->lr.v0;
    hd.lr_v1 = sched->lr.v1;
    hd.lr_t0 = sched->lr.t0;
    hd.lr_t1 = sched->lr.t1;
    lr_dev = sc.lr_slot;
  }
  int32_t* done = sc.counters;
  auto launched = [] { return cudaGetLastError() == cudaSuccess; };
  nvtxRangePushA("muon.prologue");
  // The first prologue launch resolves a scheduled learning rate for the
  // Newton-Schulz kernel (with 0 steps the scale kernel does).
  const int lr_by_prologue = ns_steps > 0 ? 1 : 0;
  if (t.n_one > 0)
    muon_prologue_kernel<true><<<static_cast<unsigned>(t.pro_grid[0]), kProThreads,
                                 t.pro_smem_one, st>>>(t.mats, t.items, t.n_one, hd,
                                                       sc.partials, sc.counters,
                                                       sc.n_counters, t.pro_prefetch,
                                                       lr_by_prologue, t.err, sc.n_mats,
                                                       t.n_items);
  bool ok = launched();
  if (ok && t.n_items > t.n_one) {
    muon_prologue_kernel<false><<<static_cast<unsigned>(t.pro_grid[1]), kProThreads,
                                  t.pro_smem, st>>>(
        t.mats, t.items + t.n_one, t.n_items - t.n_one, hd, sc.partials, sc.counters,
        sc.n_counters, 0, t.n_one > 0 ? 0 : lr_by_prologue, t.err, sc.n_mats, t.n_items);
    ok = launched();
  }
  nvtxRangePop();
  if (!ok) return MUON_ERR_CUDA;
  if (rec) rec->after(MUON_KIND_PROLOGUE);

  if (ns_steps == 0) {
    nvtxRangePushA("muon.frobenius_scale");
    muon_frob_scale_kernel<<<static_cast<unsigned>((sc.n_mats + 7) / 8), 256, 0, st>>>(
        t.mats, sc.n_mats, sc.partials, hd, sc.mat_scale);
    nvtxRangePop();
    if (!launched()) return MUON_ERR_CUDA;
    if (rec) rec->after(MUON_KIND_SCALE);
    muon_final_noiter_kernel<<<static_cast<unsigned>(t.n_items), kProThreads, 0,
                               st>>>(t.mats, t.items, sc.mat_scale, h.lr, lr_dev,
                                     h.weight_decay);
    if (!launched()) return MUON_ERR_CUDA;
    if (rec) rec->after(MUON_KIND_FINAL);
    return MUON_OK;
  }
  MegaParams p{};
  p.mats = t.mats;
  p.items = t.sched;
  p.partials = sc.partials;
  p.step_inc = sched ? step_dev : nullptr;
  p.err = t.err;
  p.done = done;
  p.n_items = static_cast<int32_t>(t.n_sched);
  p.n_mats = sc.n_mats;
  p.steps = ns_steps;
  p.fault = fault;
  p.fresh = fresh ? 1 : 0;
  for (int k = 0; k < ns_steps; ++k) {
    p.a[k] = ns_coeffs[3 * k + 0];
    p.b[k] = ns_coeffs[3 * k + 1];
    p.c[k] = ns_coeffs[3 * k + 2];
  }
  p.lr = h.lr;
  p.lr_dev = lr_dev;
  p.wd = h.weight_decay;
  p.eps_frob = h.eps_frob;
  cudaLaunchAttribute attr[2];
  cudaLaunchConfig_t cfg = pair_launch_config(t.clusters, st, attr, true);
  // test hook 2: more dynamic shared memory than the kernel was set up for,
  // so that the runtime refuses the launch (no kernel runs)
  if (fault == 2) cfg.dynamicSmemBytes = kMegaSmemBytes + 64 * 1024;
  nvtxRangePushA("muon.newton_schulz");
  const cudaError_t e = cudaLaunchKernelEx(&cfg, ns_mega_pair_kernel, p);
  nvtxRangePop();
  cudaGetLastError();
  if (e != cudaSuccess) return MUON_ERR_CUDA;
  if (rec) rec->after(MUON_KIND_NS);
  return MUON_OK;
}

}  // namespace

extern "C" {

int32_t muon_abi_version(void) { return 101; }

int64_t muon_device_allocation_count(void) {
  return g_device_allocations.load(std::memory_order_relaxed);
}

const char* muon_status_string(muon_status_t s) {
  switch (s) {
    case MUON_OK: return "ok";
    case MUON_ERR_INVALID_ARG: return "invalid argument";
    case MUON_ERR_UNSUPPORTED: return "unsupported shape or step count";
    case MUON_ERR_ALIGNMENT: return "device pointer not 16-byte aligned";
    case MUON_ERR_CUDA: return "CUDA error";
    case MUON_ERR_TIMEOUT: return "device-side wait timed out";
    case MUON_ERR_WORKSPACE: return "workspace missing, too small or misaligned";
    case MUON_ERR_DEVICE_CHECK: return "device-side bounds check failed";
  }
  return "unknown status";
}

int32_t muon_step_launches(int32_t ns_steps) {
  // one prologue kernel (which also zeroes the step's counters), then one
  // Newton-Schulz launch for all steps; with 0 steps the Frobenius scale
  // kernel and the finisher; no memset
  return ns_steps < 0 ? 0 : (ns_steps > 0 ? 2 : 3);
}

int32_t muon_plan_step_launches(const muon_plan_t* plan, int32_t ns_steps) {
  if (!plan || ns_steps < 0) return 0;
  const int n_items = static_cast<int>(plan->items.size());
  return (plan->n_one > 0 ? 1 : 0) + (n_items > plan->n_one ? 1 : 0) +
         (ns_steps > 0 ? 1 : 2);
}

int32_t ema_update_launches(int32_t n_tensors) {
  return n_tensors <= 0 ? 0 : (n_tensors + kEmaMaxSegs - 1) / kEmaMaxSegs;
}

int32_t adamw_ema_launches(int32_t n_tensors, int32_t with_step_dev) {
  if (n_tensors < 0) return 0;
  return (n_tensors + kAdamMaxSegs - 1) / kAdamMaxSegs + (with_step_dev ? 1 : 0);
}

muon_status_t muon_plan_create(const int32_t* rows, const int32_t* cols,
                               int32_t n_mats, int32_t max_ns_steps,
                               muon_plan_t** out) {
  if (!out) return MUON_ERR_INVALID_ARG;
  *out = nullptr;
  if (!rows || !cols || n_mats < 1 || n_mats > kMaxMats) return MUON_ERR_INVALID_ARG;
  if (max_ns_steps < 0 || max_ns_steps > kMaxNsSteps) return MUON_ERR_UNSUPPORTED;
  for (int i = 0; i < n_mats; ++i) {
    Geom g;
    size_t scratch = 0;
    const muon_status_t vs = layout_matrix(rows[i], cols[i], g, scratch);
    if (vs != MUON_OK) return vs;
  }

  muon_plan* plan = new (std::nothrow) muon_plan();
  if (!plan) return MUON_ERR_INVALID_ARG;
  plan->n_mats = n_mats;
  plan->max_ns = max_ns_steps;

  // Geometry, workspace layout, prologue work items.
  size_t off = 0;
  long long per_step_items = 0;
  plan->geom.resize(n_mats);
  plan->smats.resize(n_mats);
  for (int i = 0; i < n_mats; ++i) {
    Geom& g = plan->geom[i];
    layout_matrix(rows[i], cols[i], g, off);
    const int rt = pro_rows_per_item(g.rows, g.cols);
    g.part_first = static_cast<int>(plan->items.size());
    for (int r0 = 0; r0 < g.rows; r0 += rt)
      plan->items.push_back(ProItem{i, r0, std::min(rt, g.rows - r0),
                                    static_cast<int32_t>(plan->items.size())});
    g.part_count = static_cast<int>(plan->items.size()) - g.part_first;
    if (g.transposed && !pro_one_pass(g.cols))
      plan->pro_smem = std::max(plan->pro_smem,
                                static_cast<size_t>(rt) * (g.cols + 2) * 2);
    fill_sched_matrix(plan->smats[i], g);
    per_step_items += 2 * g.n_sym_tiles + g.n_apply_tiles;
  }
  plan->sched_cap = per_step_items * std::max(max_ns_steps, 1);
  plan->n_one = order_prologue_items(plan->items.data(),
                                     static_cast<int>(plan->items.size()),
                                     plan->geom.data());
  if (plan->items.size() > 0x7FFFFFFF || plan->sched_cap > 0x7FFFFFFF) {
    delete plan;
    return MUON_ERR_UNSUPPORTED;
  }
  plan->part_off = off;
  off = align_up(off + plan->items.size() * sizeof(float), 1024);
  plan->scale_off = off;
  off = align_up(off + static_cast<size_t>(n_mats) * sizeof(float), 1024);
  plan->counter_off = off;
  off = align_up(off + static_cast<size_t>(counters_for(n_mats, max_ns_steps)) *
                           sizeof(int32_t), 1024);
  plan->lr_slot_off = off;   // the scheduled learning rate of a step
  off = align_up(off + sizeof(float), 1024);
  plan->ws_bytes = off;

  if (cudaGetDevice(&plan->device) != cudaSuccess ||
      cudaDeviceGetAttribute(&plan->num_sms, cudaDevAttrMultiProcessorCount,
                             plan->device) != cudaSuccess) {
    cudaGetLastError();
    delete plan;
    return MUON_ERR_CUDA;
  }
  plan->max_clusters = query_max_clusters();

  // Device table.
  size_t t_off = 0;
  const size_t mats_off = t_off;
  t_off = align_up(t_off + sizeof(MatDev) * n_mats, 256);
  const size_t items_off = t_off;
  t_off = align_up(t_off + sizeof(ProItem) * plan->items.size(), 256);
  const size_t sched_off = t_off;
  t_off = align_up(t_off + sizeof(SchedItem) * plan->sched_cap, 256);
  const size_t err_off = t_off;
  t_off += 256;
  const int n_two = static_cast<int>(plan->items.size()) - plan->n_one;
  plan->pro_smem_one = one_pass_smem(plan->geom.data(), n_mats);
  plan->pro_prefetch = one_pass_prefetch(plan->geom.data(), n_mats);
  if (plan->max_clusters <= 0 ||
      !set_kernel_attributes(plan->pro_smem, plan->pro_smem_one) ||
      (plan->pro_grid[0] = prologue_grid<true>(plan->n_one, plan->pro_smem_one)) < 0 ||
      (plan->pro_grid[1] = prologue_grid<false>(n_two, plan->pro_smem)) < 0 ||
      dev_alloc(&plan->d_block, t_off) != cudaSuccess) {
    cudaGetLastError();
    delete plan;
    return MUON_ERR_CUDA;
  }
  char* base = static_cast<char*>(plan->d_block);
  plan->d_mats = reinterpret_cast<MatDev*>(base + mats_off);
  plan->d_items = reinterpret_cast<ProItem*>(base + items_off);
  plan->d_sched = reinterpret_cast<SchedItem*>(base + sched_off);
  plan->d_err = reinterpret_cast<int32_t*>(base + err_off);
  const bool ok =
      cudaMemcpy(plan->d_items, plan->items.data(), sizeof(ProItem) * plan->items.size(),
                 cudaMemcpyHostToDevice) == cudaSuccess &&
      cudaMemset(plan->d_err, 0, sizeof(int32_t)) == cudaSuccess;
  if (!ok) {
    cudaGetLastError();
    cudaFree(plan->d_block);
    delete plan;
    return MUON_ERR_CUDA;
  }
  plan->h_mats.resize(n_mats);
  plan->sched.resize(plan->sched_cap);
  plan->sgroups.resize(static_cast<size_t>(n_mats) * std::max(max_ns_steps, 1) * 3);
  plan->sorder.resize(2 * static_cast<size_t>(n_mats) + 1);
  plan->scl.resize(plan->max_clusters);
  *out = plan;
  return MUON_OK;
}

size_t muon_plan_workspace_bytes(const muon_plan_t* plan) {
  return plan ? plan->ws_bytes : 0;
}

void muon_plan_destroy(muon_plan_t* plan) {
  if (!plan) return;
  cudaDeviceSynchronize();
  for (auto& s : plan->slots)
    for (auto& e : s.ev)
      if (e) cudaEventDestroy(e);
  if (plan->d_block) cudaFree(plan->d_block);
  delete plan;
}

muon_status_t muon_plan_set_fault(muon_plan_t* plan, int32_t fault) {
  if (!plan || fault < 0 || fault > 3) return MUON_ERR_INVALID_ARG;
  // fault 3 hands the kernel an invalid work item: only a build that checks
  // every item before touching memory may receive one
  if (fault == 3 && !kDeviceChecks) return MUON_ERR_UNSUPPORTED;
  plan->fault = fault;
  plan->sched_steps = -1;   // the next call uploads the list anew
  return MUON_OK;
}

int32_t muon_device_checks(void) { return kDeviceChecks ? 1 : 0; }

muon_status_t muon_plan_set_timing(muon_plan_t* plan, int32_t enable) {
  if (!plan) return MUON_ERR_INVALID_ARG;
  if (enable && plan->slots.empty()) {
    plan->slots.resize(kTimingSlots);
    for (auto& s : plan->slots)
      for (auto& e : s.ev) {
        e = nullptr;
        if (cudaEventCreate(&e) != cudaSuccess) return MUON_ERR_CUDA;
      }
  }
  plan->timing = enable != 0;
  return MUON_OK;
}

muon_status_t muon_plan_timing_read(muon_plan_t* plan, int32_t* launches,
                                    double* ms, int32_t n_kinds) {
  if (!plan || n_kinds < 0) return MUON_ERR_INVALID_ARG;
  // Harvest in issue order: oldest slot first.
  for (int k = 0; k < static_cast<int>(plan->slots.size()); ++k)
    harvest(plan, plan->slots[(plan->slot_head + k) % plan->slots.size()]);
  for (int k = 0; k < n_kinds && k < MUON_KIND_COUNT; ++k) {
    if (launches) launches[k] = static_cast<int32_t>(plan->kind_launches[k]);
    if (ms) ms[k] = plan->kind_ms[k];
  }
  for (int k = 0; k < MUON_KIND_COUNT; ++k) {
    plan->kind_ms[k] = 0.0;
    plan->kind_launches[k] = 0;
  }
  return MUON_OK;
}

muon_status_t muon_get_last_error(muon_plan_t* plan, muon_stream_t stream) {
  if (!plan) return MUON_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return MUON_ERR_CUDA;
  int32_t word = 0;
  if (cudaMemcpy(&word, plan->d_err, sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess)
    return MUON_ERR_CUDA;
  if (word != 0) {
    cudaMemset(plan->d_err, 0, 2 * sizeof(int32_t));
    cudaDeviceSynchronize();
    return (word & 0xF00) == 0x200 ? MUON_ERR_DEVICE_CHECK : MUON_ERR_TIMEOUT;
  }
  if (cudaGetLastError() != cudaSuccess) return MUON_ERR_CUDA;
  return MUON_OK;
}

}  // extern "C"

namespace {

bool finite_ramp(const muon_ramp_t& r) { return finite(r.v0) && finite(r.v1); }

// The plain and the scheduled step (sched non-null).
muon_status_t step_impl(muon_plan_t* plan, const muon_matrix_t* mats,
                        const muon_hyper_t* hyper, const muon_schedule_t* sched,
                        int32_t* step_dev, const float* ns_coeffs, int32_t ns_steps,
                        void* workspace, size_t workspace_bytes, muon_stream_t stream) {
  // ---- validation (host, before anything is enqueued)
  if (!plan || !mats) return MUON_ERR_INVALID_ARG;
  muon_status_t vs = validate_hyper(hyper, ns_coeffs, ns_steps, plan->max_ns);
  if (vs != MUON_OK) return vs;
  if (sched) {
    if (!step_dev || !finite_ramp(sched->momentum) || !finite_ramp(sched->lr) ||
        sched->momentum.v0 < 0.f || sched->momentum.v0 >= 1.f ||
        sched->momentum.v1 < 0.f || sched->momentum.v1 >= 1.f)
      return MUON_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(step_dev) & 3u) != 0) return MUON_ERR_ALIGNMENT;
  }
  if (!workspace || workspace_bytes < plan->ws_bytes) return MUON_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return MUON_ERR_WORKSPACE;
  for (int i = 0; i < plan->n_mats; ++i) {
    vs = validate_matrix(mats[i], plan->geom[i]);
    if (vs != MUON_OK) return vs;
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);

  // ---- per-matrix device table and schedule (uploaded only on change)
  char* ws = static_cast<char*>(workspace);
  std::vector<MatDev>& hm = plan->h_mats;
  if (plan->enc_ws != workspace) {
    for (int i = 0; i < plan->n_mats; ++i)
      if (!fill_workspace_fields(hm[i], plan->geom[i], ws)) {
        plan->enc_ws = nullptr;
        plan->h_valid = false;
        return MUON_ERR_CUDA;
      }
    plan->enc_ws = workspace;
    plan->h_valid = false;
  }
  bool changed = !plan->h_valid;
  for (int i = 0; i < plan->n_mats; ++i)
    changed |= fill_caller_fields(hm[i], mats[i]);
  const bool resched = ns_steps > 0 && ns_steps != plan->sched_steps;
  if (changed || resched) {
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    // The host copy of the table already holds this call's pointers: until a
    // call uploads it, the device copy is stale.
    if (changed) plan->h_valid = false;
    if (cudaStreamIsCapturing(st, &cap) != cudaSuccess) return MUON_ERR_CUDA;
    // A host-to-device table copy cannot be captured from pageable memory:
    // run one call with the same buffers and step count before capturing.
    if (cap != cudaStreamCaptureStatusNone) return MUON_ERR_UNSUPPORTED;
  }
  if (changed) {
    // Pageable source: the call returns once the bytes are staged, so the
    // host table may change right after; the copy is ordered on `st` after
    // every earlier kernel of this plan.
    if (cudaMemcpyAsync(plan->d_mats, hm.data(), sizeof(MatDev) * plan->n_mats,
                        cudaMemcpyHostToDevice, st) != cudaSuccess) {
      plan->h_valid = false;
      return MUON_ERR_CUDA;
    }
    plan->h_valid = true;
  }
  if (resched) {
    const long long n = build_schedule(plan->smats.data(), plan->n_mats, ns_steps,
                                       plan->max_clusters, default_policy(),
                                       plan->sched.data(),
                                       plan->sched_cap, plan->sgroups.data(),
                                       plan->sorder.data(), plan->scl.data());
    if (n < 0) return MUON_ERR_UNSUPPORTED;
    // test hook 3 (device-checked build only): the last item of the list gets
    // a tile row past its matrix; the kernel must catch it before any access
    SchedItem saved = plan->sched[n - 1];
    if (plan->fault == 3) plan->sched[n - 1].ti = static_cast<uint16_t>(0xFFFF);
    const cudaError_t ce = cudaMemcpyAsync(plan->d_sched, plan->sched.data(),
                                           sizeof(SchedItem) * n, cudaMemcpyHostToDevice, st);
    plan->sched[n - 1] = saved;
    if (plan->fault == 3) plan->sched_steps = -1;   // (re-uploaded clean later)
    if (ce != cudaSuccess) {
      plan->sched_steps = -1;
      return MUON_ERR_CUDA;
    }
    if (plan->fault != 3) plan->sched_steps = ns_steps;
    plan->sched_len = n;
  }

  // ---- launches
  LaunchTables t{plan->d_mats, plan->d_items, static_cast<int>(plan->items.size()),
                 plan->n_one, plan->d_sched, plan->sched_len, plan->d_err, plan->pro_smem,
                 plan->pro_smem_one, {plan->pro_grid[0], plan->pro_grid[1]},
                 plan->max_clusters, plan->pro_prefetch};
  StepScratch sc{reinterpret_cast<float*>(ws + plan->part_off),
                 reinterpret_cast<float*>(ws + plan->scale_off),
                 reinterpret_cast<int32_t*>(ws + plan->counter_off),
                 counters_for(plan->n_mats, ns_steps), plan->n_mats,
                 reinterpret_cast<float*>(ws + plan->lr_slot_off)};
  Recorder rec(plan, st);
  const muon_status_t es = enqueue_step(t, *hyper, sched, step_dev, ns_coeffs, ns_steps,
                                        sc, plan->fault, changed, st,
                                        plan->timing ? &rec : nullptr);
  rec.finish();
  if (es != MUON_OK) return es;
  if (cudaGetLastError() != cudaSuccess) return MUON_ERR_CUDA;
  return MUON_OK;
}

}  // namespace

extern "C" {

muon_status_t muon_plan_error_async(const muon_plan_t* plan, int32_t* host_word,
                                    muon_stream_t stream) {
  if (!plan || !host_word) return MUON_ERR_INVALID_ARG;
  if (cudaMemcpyAsync(host_word, plan->d_err, sizeof(int32_t), cudaMemcpyDeviceToHost,
                      static_cast<cudaStream_t>(stream)) != cudaSuccess) {
    cudaGetLastError();
    return MUON_ERR_CUDA;
  }
  return MUON_OK;
}

muon_status_t muon_step_batched(muon_plan_t* plan, const muon_matrix_t* mats,
                                const muon_hyper_t* hyper,
                                const float* ns_coeffs, int32_t ns_steps,
                                void* workspace, size_t workspace_bytes,
                                muon_stream_t stream) {
  return step_impl(plan, mats, hyper, nullptr, nullptr, ns_coeffs, ns_steps, workspace,
                   workspace_bytes, stream);
}

muon_status_t muon_step_batched_sched(muon_plan_t* plan, const muon_matrix_t* mats,
                                      const muon_hyper_t* hyper,
                                      const muon_schedule_t* sched, int32_t* step_dev,
                                      const float* ns_coeffs, int32_t ns_steps,
                                      void* workspace, size_t workspace_bytes,
                                      muon_stream_t stream) {
  if (!sched) return MUON_ERR_INVALID_ARG;
  return step_impl(plan, mats, hyper, sched, step_dev, ns_coeffs, ns_steps, workspace,
                   workspace_bytes, stream);
}

muon_status_t ema_update_batched(float* const* ema, const float* const* params,
                                 const int64_t* numel, int32_t n_tensors,
                                 float decay, muon_stream_t stream) {
  if (n_tensors < 0) return MUON_ERR_INVALID_ARG;
  if (n_tensors == 0) return MUON_OK;
  if (!ema || !params || !numel || !finite(decay)) return MUON_ERR_INVALID_ARG;
  for (int i = 0; i < n_tensors; ++i) {
    if (numel[i] < 0) return MUON_ERR_INVALID_ARG;
    if (numel[i] == 0) continue;
    if (!ema[i] || !params[i]) return MUON_ERR_INVALID_ARG;
    if (((reinterpret_cast<uintptr_t>(ema[i]) |
          reinterpret_cast<uintptr_t>(params[i])) & 3u) != 0)
      return MUON_ERR_ALIGNMENT;
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int sms = 148;
  {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return MUON_ERR_CUDA;
  }
  const double omd = 1.0 - static_cast<double>(decay);
  for (int first = 0; first < n_tensors; first += kEmaMaxSegs) {
    EmaParams p{};
    p.d = decay;
    p.one_minus_d = static_cast<float>(omd);
    long long units = 0;
    int ns = 0;
    for (int i = first; i < std::min(n_tensors, first + kEmaMaxSegs); ++i, ++ns) {
      p.seg[ns].e = ema[i];
      p.seg[ns].p = params[i];
      p.seg[ns].numel = numel[i];
      p.seg[ns].ubeg = units;
      units += (numel[i] + 3) / 4;
    }
    p.n_seg = ns;
    p.total_units = units;
    if (units == 0) continue;
    const long long want = (units + kEmaThreads - 1) / kEmaThreads;
    const unsigned grid = static_cast<unsigned>(std::min<long long>(want, 8ll * sms));
    nvtxRangePushA("muon.ema");
    ema_update_kernel<<<grid, kEmaThreads, 0, st>>>(p);
    nvtxRangePop();
  }
  if (cudaGetLastError() != cudaSuccess) return MUON_ERR_CUDA;
  return MUON_OK;
}

muon_status_t muon_f32_to_bf16(uint16_t* dst, const float* src, int64_t n,
                               muon_stream_t stream) {
  if (n < 0) return MUON_ERR_INVALID_ARG;
  if (n == 0) return MUON_OK;
  if (!dst || !src) return MUON_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(dst) & 1u) || (reinterpret_cast<uintptr_t>(src) & 3u))
    return MUON_ERR_ALIGNMENT;
  const int vec = ((reinterpret_cast<uintptr_t>(dst) | reinterpret_cast<uintptr_t>(src)) &
                   15u) == 0 ? 1 : 0;
  int sms = 148;
  {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return MUON_ERR_CUDA;
  }
  const long long per_thread = vec ? 8 : 1;
  const long long want = (n / per_thread + kCvtThreads - 1) / kCvtThreads;
  const unsigned grid =
      static_cast<unsigned>(std::max(1ll, std::min<long long>(want, 8ll * sms)));
  f32_to_bf16_kernel<<<grid, kCvtThreads, 0, static_cast<cudaStream_t>(stream)>>>(
      dst, src, n, vec);
  if (cudaGetLastError() != cudaSuccess) return MUON_ERR_CUDA;
  return MUON_OK;
}

muon_status_t adamw_ema_batched(const adamw_tensor_t* tensors, int32_t n_tensors,
                                const adamw_hyper_t* hyper, int32_t step,
                                int32_t* step_dev, float ema_decay, muon_stream_t stream) {
  if (n_tensors < 0 || !hyper || !finite(ema_decay)) return MUON_ERR_INVALID_ARG;
  if (n_tensors > 0 && !tensors) return MUON_ERR_INVALID_ARG;
  const adamw_hyper_t& h = *hyper;
  if (!finite(h.lr) || !finite(h.weight_decay) || !finite(h.eps) || h.eps < 0.f ||
      !(h.beta1 >= 0.f && h.beta1 < 1.f) || !(h.beta2 >= 0.f && h.beta2 < 1.f))
    return MUON_ERR_INVALID_ARG;
  if (!step_dev && step < 1) return MUON_ERR_INVALID_ARG;
  if (step_dev && (reinterpret_cast<uintptr_t>(step_dev) & 3u) != 0) return MUON_ERR_ALIGNMENT;
  for (int i = 0; i < n_tensors; ++i) {
    const adamw_tensor_t& x = tensors[i];
    if (x.numel < 0) return MUON_ERR_INVALID_ARG;
    if (x.numel == 0) continue;
    if (!x.param || !x.grad || !x.exp_avg || !x.exp_avg_sq) return MUON_ERR_INVALID_ARG;
    if (((reinterpret_cast<uintptr_t>(x.param) | reinterpret_cast<uintptr_t>(x.grad) |
          reinterpret_cast<uintptr_t>(x.exp_avg) | reinterpret_cast<uintptr_t>(x.exp_avg_sq) |
          reinterpret_cast<uintptr_t>(x.ema)) & 3u) != 0)
      return MUON_ERR_ALIGNMENT;
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int sms = 148;
  {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return MUON_ERR_CUDA;
  }
  for (int first = 0; first < n_tensors; first += kAdamMaxSegs) {
    AdamParams a{};
    a.step_dev = step_dev;
    a.step = step;
    a.lr = h.lr;
    a.b1 = h.beta1;
    a.b2 = h.beta2;
    a.eps = h.eps;
    a.wd = h.weight_decay;
    a.d = ema_decay;
    long long units = 0;
    int ns = 0;
    for (int i = first; i < std::min(n_tensors, first + kAdamMaxSegs); ++i, ++ns) {
      const adamw_tensor_t& x = tensors[i];
      a.seg[ns] = AdamSeg{x.param, x.grad, x.exp_avg, x.exp_avg_sq, x.ema, x.numel, units};
      units += (x.numel + 3) / 4;
    }
    a.n_seg = ns;
    a.total_units = units;
    // (launched even when empty, so that the launch count is fixed)
    const long long want = std::max(1ll, (units + kAdamThreads - 1) / kAdamThreads);
    const unsigned grid = static_cast<unsigned>(std::min<long long>(want, 8ll * sms));
    nvtxRangePushA("muon.adamw_ema");
    adamw_ema_kernel<<<grid, kAdamThreads, 0, st>>>(a);
    nvtxRangePop();
  }
  if (step_dev) adamw_step_advance_kernel<<<1, 1, 0, st>>>(step_dev);
  if (cudaGetLastError() != cudaSuccess) return MUON_ERR_CUDA;
  return MUON_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// muon_step_batched_noalloc: the batched step for callers that cannot
// allocate device memory.
//
// All of the step's scratch (the per-matrix records with their TMA
// descriptors, the work items and the schedule, the error word, and the
// working matrices X, A, B', the norm partials and the counters) lives in one
// file-scope device array, g_noalloc_scratch, of MUON_NOALLOC_SCRATCH_BYTES.
// The CUDA runtime reserves it on every device where this library's kernels
// are loaded, for the life of the process.  Host code must not pass the
// array's name to a kernel (in host code it names a host-side stand-in); the
// device address comes from cudaGetSymbolAddress, looked up once per device
// with that device current, on the first call made on that device.  The host
// side uses fixed-size static tables only.
// ---------------------------------------------------------------------------
namespace {

static __device__ __align__(256) unsigned char
    g_noalloc_scratch[MUON_NOALLOC_SCRATCH_BYTES];

constexpr int kNoAllocMaxDevices = 64;
constexpr int kNoAllocMaxItems = 8192;
constexpr int kNoAllocMaxSched = 65536;
constexpr int kNoAllocMaxClusters = 1024;
constexpr int kNoAllocMaxGroups = MUON_NOALLOC_MAX_MATS * kMaxNsSteps * 3;

// Device address of g_noalloc_scratch per device (filled on first use).
void* g_noalloc_dev_ptr[kNoAllocMaxDevices] = {};
int g_noalloc_clusters[kNoAllocMaxDevices] = {};
std::mutex g_noalloc_mutex;

// Host-side staging of the tables (fixed capacity; guarded by the mutex).
Geom g_na_geom[MUON_NOALLOC_MAX_MATS];
MatDev g_na_mats[MUON_NOALLOC_MAX_MATS];
ProItem g_na_items[kNoAllocMaxItems];
SchedMatrix g_na_smats[MUON_NOALLOC_MAX_MATS];
SchedItem g_na_sched[kNoAllocMaxSched];
SchedGroup g_na_groups[kNoAllocMaxGroups];
int g_na_order[2 * MUON_NOALLOC_MAX_MATS + 1];
double g_na_cltime[kNoAllocMaxClusters];

// Test hook of the allocation-free path (muon_noalloc_set_fault).
int g_noalloc_fault = 0;

// Set-up of the current device, once per device, with g_noalloc_mutex held:
// the device address of g_noalloc_scratch (cudaGetSymbolAddress, with this
// device current) and the cluster count of the tensor-core kernel.  *dev
// receives the current device.
muon_status_t noalloc_setup(int& dev) {
  if (cudaGetDevice(&dev) != cudaSuccess) return MUON_ERR_CUDA;
  if (dev < 0 || dev >= kNoAllocMaxDevices) return MUON_ERR_UNSUPPORTED;
  if (g_noalloc_dev_ptr[dev]) return MUON_OK;
  void* ptr = nullptr;
  if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || !ptr) {
    cudaGetLastError();
    return MUON_ERR_CUDA;
  }
  const int clusters = query_max_clusters();
  if (clusters <= 0 || clusters > kNoAllocMaxClusters) {
    cudaGetLastError();
    return MUON_ERR_CUDA;
  }
  g_noalloc_clusters[dev] = clusters;
  g_noalloc_dev_ptr[dev] = ptr;
  return MUON_OK;
}

}  // namespace

extern "C" {

muon_status_t muon_step_batched_noalloc(const muon_matrix_t* mats,
                                        int32_t n_mats,
                                        const muon_hyper_t* hyper,
                                        const float* ns_coeffs,
                                        int32_t ns_steps,
                                        muon_stream_t stream) {
  if (!mats || n_mats < 1) return MUON_ERR_INVALID_ARG;
  if (n_mats > MUON_NOALLOC_MAX_MATS) return MUON_ERR_UNSUPPORTED;
  muon_status_t vs = validate_hyper(hyper, ns_coeffs, ns_steps, kMaxNsSteps);
  if (vs != MUON_OK) return vs;

  std::lock_guard<std::mutex> lock(g_noalloc_mutex);

  // Geometry and work items into the fixed host tables.
  size_t off = 0;
  int n_items = 0;
  size_t pro_smem = 0;
  for (int i = 0; i < n_mats; ++i) {
    Geom& g = g_na_geom[i];
    vs = layout_matrix(mats[i].rows, mats[i].cols, g, off);
    if (vs != MUON_OK) return vs;
    vs = validate_matrix(mats[i], g);
    if (vs != MUON_OK) return vs;
    const int rt = pro_rows_per_item(g.rows, g.cols);
    g.part_first = n_items;
    for (int r0 = 0; r0 < g.rows; r0 += rt) {
      if (n_items >= kNoAllocMaxItems) return MUON_ERR_UNSUPPORTED;
      g_na_items[n_items] = ProItem{i, r0, std::min(rt, g.rows - r0), n_items};
      ++n_items;
    }
    g.part_count = n_items - g.part_first;
    if (g.transposed && !pro_one_pass(g.cols))
      pro_smem = std::max(pro_smem, static_cast<size_t>(rt) * (g.cols + 2) * 2);
    fill_sched_matrix(g_na_smats[i], g);
  }
  const int n_one = order_prologue_items(g_na_items, n_items, g_na_geom);
  const size_t part_off = off;
  off = align_up(off + static_cast<size_t>(n_items) * sizeof(float), 1024);
  const size_t scale_off = off;
  off = align_up(off + static_cast<size_t>(n_mats) * sizeof(float), 1024);
  const size_t counter_off = off;
  const int n_counters = counters_for(n_mats, ns_steps);
  off = align_up(off + static_cast<size_t>(n_counters) * sizeof(int32_t), 1024);
  const size_t ws_bytes = off;

  // Device address of the array on the current device (once per device).
  int dev = 0;
  vs = noalloc_setup(dev);
  if (vs != MUON_OK) return vs;
  const int clusters = g_noalloc_clusters[dev];
  long long n_sched = 0;
  if (ns_steps > 0) {
    n_sched = build_schedule(g_na_smats, n_mats, ns_steps, clusters, default_policy(),
                             g_na_sched,
                             kNoAllocMaxSched, g_na_groups, g_na_order, g_na_cltime);
    if (n_sched < 0) return MUON_ERR_UNSUPPORTED;
  }

  // Layout of the device array: [error word][tables][workspace].
  size_t t_off = 256;
  const size_t mats_off = t_off;
  t_off = align_up(t_off + sizeof(MatDev) * n_mats, 256);
  const size_t items_off = t_off;
  t_off = align_up(t_off + sizeof(ProItem) * n_items, 256);
  const size_t sched_off = t_off;
  t_off = align_up(t_off + sizeof(SchedItem) * n_sched, 1024);
  const size_t ws_off = t_off;
  if (ws_off + ws_bytes > MUON_NOALLOC_SCRATCH_BYTES) return MUON_ERR_WORKSPACE;

  const size_t pro_smem_one = one_pass_smem(g_na_geom, n_mats);
  if (!set_kernel_attributes(pro_smem, pro_smem_one)) {
    cudaGetLastError();
    return MUON_ERR_CUDA;
  }
  const int pro_grid_one = prologue_grid<true>(n_one, pro_smem_one);
  const int pro_grid_two = prologue_grid<false>(n_items - n_one, pro_smem);
  if (pro_grid_one < 0 || pro_grid_two < 0) return MUON_ERR_CUDA;
  char* base = static_cast<char*>(g_noalloc_dev_ptr[dev]);
  char* ws = base + ws_off;
  for (int i = 0; i < n_mats; ++i) {
    if (!fill_workspace_fields(g_na_mats[i], g_na_geom[i], ws)) return MUON_ERR_CUDA;
    fill_caller_fields(g_na_mats[i], mats[i]);
  }

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // The array keeps the previous call's contents: the error word must start
  // at zero (the counters are reset by the step itself); everything else is
  // written before it is read.
  if (cudaMemsetAsync(base, 0, sizeof(int32_t), st) != cudaSuccess ||
      cudaMemcpyAsync(base + mats_off, g_na_mats, sizeof(MatDev) * n_mats,
                      cudaMemcpyHostToDevice, st) != cudaSuccess ||
      cudaMemcpyAsync(base + items_off, g_na_items, sizeof(ProItem) * n_items,
                      cudaMemcpyHostToDevice, st) != cudaSuccess ||
      (n_sched > 0 &&
       cudaMemcpyAsync(base + sched_off, g_na_sched, sizeof(SchedItem) * n_sched,
                       cudaMemcpyHostToDevice, st) != cudaSuccess)) {
    cudaGetLastError();
    return MUON_ERR_CUDA;
  }

  LaunchTables t{reinterpret_cast<const MatDev*>(base + mats_off),
                 reinterpret_cast<const ProItem*>(base + items_off), n_items, n_one,
                 reinterpret_cast<const SchedItem*>(base + sched_off), n_sched,
                 reinterpret_cast<int32_t*>(base), pro_smem, pro_smem_one,
                 {pro_grid_one, pro_grid_two}, clusters,
                 one_pass_prefetch(g_na_geom, n_mats)};
  StepScratch sc{reinterpret_cast<float*>(ws + part_off),
                 reinterpret_cast<float*>(ws + scale_off),
                 reinterpret_cast<int32_t*>(ws + counter_off), n_counters, n_mats,
                 nullptr};
  const muon_status_t es = enqueue_step(t, *hyper, nullptr, nullptr, ns_coeffs, ns_steps,
                                        sc, g_noalloc_fault, true, st, nullptr);
  if (es != MUON_OK) return es;
  if (cudaGetLastError() != cudaSuccess) return MUON_ERR_CUDA;
  return MUON_OK;
}

muon_status_t muon_noalloc_error_async(int32_t* host_word, muon_stream_t stream) {
  if (!host_word) return MUON_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  int dev = 0;
  const muon_status_t vs = noalloc_setup(dev);
  if (vs != MUON_OK) return vs;
  // word 0 of the array; the next allocation-free call clears it
  if (cudaMemcpyAsync(host_word, g_noalloc_dev_ptr[dev], sizeof(int32_t),
                      cudaMemcpyDeviceToHost,
                      static_cast<cudaStream_t>(stream)) != cudaSuccess) {
    cudaGetLastError();
    return MUON_ERR_CUDA;
  }
  return MUON_OK;
}

muon_status_t muon_noalloc_set_fault(int32_t fault) {
  if (fault < 0 || fault > 2) return MUON_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  g_noalloc_fault = fault;
  return MUON_OK;
}

}  // extern "C"
