#pragma once
#include "sm100.cuh"
static int fattn_bwd_launch(const void*, const void*, const void*, const void*, const float*,
                            const void*, void*, void*, void*, int, int, int, bool, float, void*,
                            uint64_t, cudaStream_t) { return 2; }
