// Router GEMM + score function on the tensor cores (tcgen05, bf16 inputs, fp32 TMEM
// accumulators; the score function runs in the epilogue).
#pragma once
#include "nmoe_internal.cuh"

namespace nmoe {

bool router_sm100_supported(const Shape& s);

cudaError_t launch_router_sm100(const void* x, const void* W_r, const Shape& s,
                                nmoe_score_fn fn, const float* bias, float* scores,
                                float* scores_t, unsigned* err, cudaStream_t st);

}  // namespace nmoe
