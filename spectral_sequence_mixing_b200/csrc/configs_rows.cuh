// configs_rows.cuh -- the long-row kernels' instances: transform sizes,
// cluster shapes and resident-CTA targets.
#pragma once

#include "bigconv.cuh"

namespace ccv {

// One row per CTA in clusters of 8 channels (N = 4096 or 8192), or one row
// per 8-CTA cluster (N = 131072: R0 = 16, mirror pairs of k0 per CTA).
template <typename IO> using BigM = BigCfg<16, 16, 16, 1, 1, 256, IO>;   // N = 4096,   L <= 2048
template <typename IO> using BigL = BigCfg<32, 16, 16, 1, 1, 256, IO>;   // N = 8192,   L <= 4096
template <typename IO> using BigX = BigCfg<16, 32, 16, 16, 8, 512, IO>;  // N = 131072, L <= 65536
constexpr int kMinbBigM = 2, kMinbBigL = 2, kMinbBigX = 1;

}  // namespace ccv
