// Internal declarations shared by the CUDA translation units of libnmoe.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "nmoe.h"

namespace nmoe {

// Bits of the per-device error word (see nmoe_get_last_error).
constexpr unsigned kErrDeviceCheck = 1u;
constexpr unsigned kErrTimeout = 2u;

__host__ __device__ inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }
template <typename T> __device__ __forceinline__ T from_f32(float v);
template <> __device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) {
  return __float2bfloat16_rn(v);
}

// Shapes of one layer call, already validated on the host.
struct Shape {
  int T;         // tokens
  int d;         // model dim
  int E;         // experts
  int F;         // expert hidden dim
  int C;         // capacity per segment
  int n_seg;     // segments
  int S;         // tokens per segment = T / n_seg
  int Ce;        // entries per expert = n_seg * C
};

// Launchers. Each returns the launch status (cudaGetLastError after the launch).
cudaError_t launch_router_simt(const void* x, const void* W_r, const Shape& s, nmoe_dtype dt,
                               nmoe_score_fn fn, const float* bias, float* scores,
                               float* scores_t, cudaStream_t st);

cudaError_t launch_select(const float* scores_t, const Shape& s, int32_t* idx, float* gate,
                          unsigned* err, cudaStream_t st);

// combine == NMOE_COMBINE_NORMALIZED rewrites gate[] in place to
// route_scale * gate / (sum of the token's gates).
cudaError_t launch_csr(const int32_t* idx, const Shape& s, int32_t* tok_ptr, int32_t* tok_ent,
                       float* gate, nmoe_combine combine, float route_scale, unsigned* err,
                       cudaStream_t st);

// CUDA-core expert GEMMs. dt is the type of x and the weights; h_f32 / y_f32 select
// fp32 (else dt) for the H and Y intermediates.
cudaError_t launch_gemm1_simt(const void* x, const int32_t* idx, const void* W1, const void* W3,
                              const Shape& s, nmoe_dtype dt, bool h_f32, void* H,
                              cudaStream_t st);

cudaError_t launch_gemm2_simt(const void* H, const float* gate, const void* W2, const Shape& s,
                              nmoe_dtype dt, bool h_f32, bool y_f32, void* Y, cudaStream_t st);

// out[t] = sum of Y rows listed for t; Y is fp32 if y_f32 (else bf16), out fp32 if out_f32.
cudaError_t launch_combine(const void* Y, const int32_t* tok_ptr, const int32_t* tok_ent,
                           const Shape& s, bool y_f32, bool out_f32, void* out, int sm_count,
                           cudaStream_t st);

}  // namespace nmoe
