// configs.cuh -- the kernel instances the library launches.  Everything that
// decides a kernel's device code is in the .cuh files; api.cu holds host code
// and the storage of the twiddle tables.
#pragma once

#include "configs_fused.cuh"
#include "configs_rows.cuh"
