// configs.cuh -- the kernel instances the library launches: transform size
// classes, tile shapes and resident-CTA targets (the launch bounds' minimum
// blocks per SM).  Everything that decides a kernel's device code is in the
// .cuh files; api.cu holds host code and the storage of the twiddle tables.
#pragma once

#include "bigconv.cuh"
#include "fftconv_fused.cuh"

namespace ccv {

// Fused kernel: tiles of ROWS channels x whole rows, N = 2 N2^2.
template <typename IO> using CfgS = FusedCfg<16, 8, IO>;  // N = 512,  L <= 256
template <typename IO> using CfgM = FusedCfg<32, 4, IO>;  // N = 2048, L <= 1024
constexpr int kMinbS = 4;
constexpr int kMinbM = 2;

// Long rows: one row per CTA in clusters of 8 channels (N = 8192), or one
// row per 8-CTA cluster (N = 131072).
template <typename IO> using BigL = BigCfg<32, 16, 16, 1, 1, 256, IO>;   // N = 8192,   L <= 4096
template <typename IO> using BigX = BigCfg<8, 32, 32, 16, 8, 512, IO>;   // N = 131072, L <= 65536
constexpr int kMinbBigL = 2, kMinbBigX = 1;

}  // namespace ccv
