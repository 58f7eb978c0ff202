// Geometry of the CTA-pair (tcgen05.mma.cta_group::2) Newton-Schulz tiles:
// 256 x 256 tiles, 128 rows of A and 128 columns of B staged per CTA, so
// every byte a CTA loads feeds twice the tensor work of a single-CTA
// 128 x 128 tile; shared-memory and L2 traffic per FLOP halve.
#pragma once

#include <cuda_bf16.h>

#include "k_ns_common.cuh"
#include "muon_types.cuh"
#include "sm100_ptx.cuh"

namespace muonb200 {

constexpr int kPairTile = 256;   // pair tile rows (128 per CTA) and columns

template <bool kBmn, int kStages>
struct PairCfg {
  static constexpr int kABytes = 128 * kTileK * 2;              // own 128 rows
  static constexpr int kBBytes = (kPairTile / 2) * kTileK * 2;  // own N half
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr uint32_t kTxBytes = 2u * kStageBytes;        // both CTAs
  static constexpr int kTmemCols = 2 * kPairTile;
  static constexpr int kNumBars = 2 * kStages + 5;
  static constexpr int kXposeBytes = kBmn ? 0 : kEpiWarps * 32 * kXposeLd * 2;
  static constexpr size_t kSmemBytes = 1024 +
      static_cast<size_t>(kStages) * kStageBytes + kXposeBytes +
      kNumBars * 8 + 16;
  static_assert(kSmemBytes <= 227 * 1024, "shared memory");
};

}  // namespace muonb200
