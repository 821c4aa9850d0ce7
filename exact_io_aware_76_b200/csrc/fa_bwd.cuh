// fa_bwd.cuh -- backward kernels (placeholder until the recomputation backward lands).
#pragma once
#include "sm100.cuh"
