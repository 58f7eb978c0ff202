// Device-side tables shared by the host launcher and the kernels.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

namespace muonb200 {

constexpr int kTileM = 128;       // rows of a tile held by one CTA (TMEM lanes)
constexpr int kTileK = 64;        // K per pipeline stage (one 128-B swizzle row)
constexpr int kPairTile = 256;    // CTA-pair tile: 256 rows (128 per CTA) x 256 cols
constexpr int kProRows = 32;      // rows per prologue work item
constexpr int kProThreads = 256;  // 8 warps
constexpr int kProBatch = 2;      // row chunks (of 256 elements) in flight per warp
constexpr int kProOneWarps = 8;   // one-pass rows: up to 8 warps x 1024 elements

// Stored rows that the one-pass prologue takes: a multiple of 8 elements (one
// 16-byte load of G per chunk) and at most kProOneWarps * 1024 elements.
__host__ __device__ constexpr bool pro_one_pass(int cols) {
  return (cols & 7) == 0 && cols <= kProOneWarps * 1024;
}

// One-pass prologue: a row of up to 1024 elements per warp, longer rows
// over wpr = 2, 4 or 8 warps (1024 elements each).
__host__ __device__ constexpr int pro_warps_per_row(int cols) {
  return cols <= 1024 ? 1 : cols <= 2048 ? 2 : cols <= 4096 ? 4 : 8;
}
// One staging buffer of a transposed one-pass item (32 rows of up to 1024
// elements, 16 of up to 2048).
constexpr int kProTransBufCap = 65 * 1024;

// Per-matrix record.  Tensor maps first (64-byte aligned), pointers after.
struct alignas(64) MatDev {
  CUtensorMap tm_xk[2];  // X ping/pong as a K-major operand, box 64 x 128
  CUtensorMap tm_xn[2];  // X ping/pong as an MN-major operand, box 64 x 64
  CUtensorMap tm_a;      // A = X X^T (m x m), box 64 x 128
  CUtensorMap tm_b;      // B = b A + c A A (m x m), box 64 x 128
  CUtensorMap tm_an;     // A as an MN-major operand, box 64 x 64
  CUtensorMap tm_bn;     // B as an MN-major operand, box 64 x 64
  __nv_bfloat16* x[2];   // m x ldx each
  __nv_bfloat16* a;      // m x lda
  __nv_bfloat16* b;      // m x lda
  float* w;              // rows x cols (caller)
  float* mom;            // rows x cols (caller)
  const uint16_t* g;     // rows x cols bf16 bits (caller)
  float* out;            // rows x cols or null (caller)
  int32_t rows, cols;    // stored shape
  int32_t m, n;          // working shape, m <= n
  int32_t ldx, lda;      // leading dimensions (elements) of X and A/B
  int32_t transposed;    // rows > cols
  int32_t part_first;    // first prologue partial of this matrix
  int32_t part_count;    // number of prologue partials
  int32_t n_sym_tiles;   // 256 x 256 pair tiles of A (and of B'), upper blocks
  int32_t n_apply_tiles; // 256 x 256 pair tiles of X
  float update_scale;
};

// A prologue work item: up to kProRows stored rows of one matrix.
struct ProItem {
  int32_t mat;
  int32_t row0;
  int32_t nrows;
  int32_t part;          // slot of this item's Frobenius partial sum
};

// A tile of one tensor-core phase.
struct NsTile {
  uint16_t mat;
  uint16_t ti;   // tile row (128 rows)
  uint16_t tj;   // tile column (128 or 256 columns)
  uint16_t kt;   // number of 64-wide K blocks
};

// One item of the persistent Newton-Schulz schedule: a pair tile of one
// phase (gram, poly, apply) of one step of one matrix.  16 bytes, read with
// one vector load.
struct alignas(16) SchedItem {
  uint16_t mat;
  uint16_t ti;    // pair-tile row (256 rows)
  uint16_t tj;    // pair-tile column (256 columns)
  uint16_t kt;    // number of 64-wide K blocks
  uint8_t mode;   // kModeGram / kModePoly / kModeApply
  uint8_t k;      // Newton-Schulz step
  uint16_t pad;
  int32_t dep_target;  // completion count of the phase the item reads (two
                       // per tile, one from each CTA); 0: no dependency
};
static_assert(sizeof(SchedItem) == 16, "SchedItem is one 16-byte load");

struct HyperDev {
  float mu, lr, wd, eps_row, eps_frob;
  int32_t nesterov, eq_r;
  // Scheduled momentum and learning rate (when `step` is not null): the
  // values at step *step of two linear ramps.  The Frobenius scale kernel
  // writes the step's learning rate to *lr_slot for the Newton-Schulz or
  // finishing kernel and advances *step.
  int32_t* step;
  float* lr_slot;
  float mu_v0, mu_v1, lr_v0, lr_v1;
  int32_t mu_t0, mu_t1, lr_t0, lr_t1;
};

// A value moving linearly from v0 at step t0 to v1 at step t1, holding its
// end values outside [t0, t1] (t1 <= t0: v0 before t1, v1 from t1 on).
__host__ __device__ inline float linear_ramp(float v0, float v1, int32_t t0, int32_t t1,
                                             int32_t t) {
  if (t1 <= t0) return t >= t1 ? v1 : v0;
  float f = static_cast<float>(t - t0) / static_cast<float>(t1 - t0);
  f = f < 0.f ? 0.f : (f > 1.f ? 1.f : f);
  return v0 + (v1 - v0) * f;
}

enum NsMode : int32_t { kModeGram = 0, kModePoly = 1, kModeApply = 2 };


// Error word values (device -> host).
constexpr int32_t kErrTimeoutProducer = 0x101;
constexpr int32_t kErrTimeoutMma = 0x102;
constexpr int32_t kErrTimeoutEpilogue = 0x103;
// Device-checked build (MUON_DEVICE_CHECKS): a Newton-Schulz work item
// outside its matrix's tile grid, a store outside its buffer, a prologue work
// item outside its matrix.  The word after the error word receives the
// offending list position, row or item index.
constexpr int32_t kErrCheckItem = 0x201;
constexpr int32_t kErrCheckStore = 0x202;
constexpr int32_t kErrCheckPrologue = 0x203;

#ifdef MUON_DEVICE_CHECKS
constexpr bool kDeviceChecks = true;
#else
constexpr bool kDeviceChecks = false;
#endif

#ifdef __CUDACC__
// Records the first failed device check (code, then its index).
__device__ __forceinline__ void record_check_failure(int32_t* err, int32_t code,
                                                     int32_t index) {
  if (atomicCAS(err, 0, code) == 0) atomicExch(err + 1, index);
}
#endif

}  // namespace muonb200
