// configs_fused.cuh -- the fused kernel's instances: size classes, tile
// shapes and resident-CTA targets (the launch bounds' minimum blocks per SM).
#pragma once

#include "fftconv_fused.cuh"

namespace ccv {

// Tiles of ROWS channels x whole rows, N = 2 N2^2.
template <typename IO> using CfgS = FusedCfg<16, 8, IO>;  // N = 512,  L <= 256
template <typename IO> using CfgM = FusedCfg<32, 4, IO>;  // N = 2048, L <= 1024
constexpr int kMinbS = 4;
constexpr int kMinbM = 2;

}  // namespace ccv
