// Deterministic weighted combine.
//
// NucleusMoE-Image walkthrough, section 6.2: the weighted outputs of the routed experts
// are added back onto their tokens (the page uses scatter_add, whose order of additions
// is not fixed). Here every token gathers its own contributions instead:
//   out[t, :] = sum over j in [tok_ptr[t], tok_ptr[t+1]) of Y[tok_ent[j], :]
// in ascending expert order (the order tok_ent lists them), accumulated in fp32 and
// rounded once to the output type. The combine weight was applied to Y by the down-
// projection epilogue. A token no expert chose gets an exact zero row.
//
// One warp per token; each lane moves 16-byte vectors and keeps several rows in flight.
#include "nmoe_internal.cuh"

namespace nmoe {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kVecPerLane = 4;   // 16-byte vectors a lane accumulates at once

__device__ __forceinline__ void unpack_add(float* acc, const uint4& v, __nv_bfloat16*) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 f = __bfloat1622float2(h[i]);
    acc[2 * i] += f.x;
    acc[2 * i + 1] += f.y;
  }
}
__device__ __forceinline__ void unpack_add(float* acc, const uint4& v, float*) {
  acc[0] += __uint_as_float(v.x);
  acc[1] += __uint_as_float(v.y);
  acc[2] += __uint_as_float(v.z);
  acc[3] += __uint_as_float(v.w);
}
__device__ __forceinline__ uint4 pack(const float* acc, __nv_bfloat16*) {
  uint4 v;
  __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&v);
#pragma unroll
  for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(acc[2 * i], acc[2 * i + 1]);
  return v;
}
__device__ __forceinline__ uint4 pack(const float* acc, float*) {
  return make_uint4(__float_as_uint(acc[0]), __float_as_uint(acc[1]), __float_as_uint(acc[2]),
                    __float_as_uint(acc[3]));
}

// Each lane owns 8 consecutive columns per vector slot: one 16-byte load of bf16 Y or
// two of fp32 Y, and one 16-byte store of bf16 out or two of fp32 out.
template <typename TY, typename TO>
__global__ void __launch_bounds__(kThreads)
combine_kernel(const TY* __restrict__ Y, const int32_t* __restrict__ tok_ptr,
               const int32_t* __restrict__ tok_ent, int Tn, int d, TO* __restrict__ out) {
  constexpr int W = 8;  // columns per lane per vector slot
  const int lane = threadIdx.x & 31;
  const int ngrp = d / W;  // d is a multiple of 8 (checked on the host)
  for (int t = blockIdx.x * kWarps + (threadIdx.x >> 5); t < Tn; t += gridDim.x * kWarps) {
    const int beg = tok_ptr[t], end = tok_ptr[t + 1];
    for (int c0 = 0; c0 < ngrp; c0 += 32 * kVecPerLane) {
      float acc[kVecPerLane][W];
#pragma unroll
      for (int v = 0; v < kVecPerLane; ++v)
#pragma unroll
        for (int i = 0; i < W; ++i) acc[v][i] = 0.f;
      for (int j = beg; j < end; ++j) {
        const TY* src = Y + (int64_t)tok_ent[j] * d;
        uint4 r[kVecPerLane][sizeof(TY) / 2];
#pragma unroll
        for (int v = 0; v < kVecPerLane; ++v) {
          const int c = c0 + v * 32 + lane;
#pragma unroll
          for (int h = 0; h < (int)sizeof(TY) / 2; ++h)
            r[v][h] = c < ngrp ? __ldg(reinterpret_cast<const uint4*>(src + (int64_t)c * W) + h)
                               : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int v = 0; v < kVecPerLane; ++v)
#pragma unroll
          for (int h = 0; h < (int)sizeof(TY) / 2; ++h)
            unpack_add(acc[v] + h * (16 / sizeof(TY)), r[v][h], (TY*)nullptr);
      }
#pragma unroll
      for (int v = 0; v < kVecPerLane; ++v) {
        const int c = c0 + v * 32 + lane;
        if (c < ngrp) {
          uint4* dst = reinterpret_cast<uint4*>(out + (int64_t)t * d + (int64_t)c * W);
#pragma unroll
          for (int h = 0; h < (int)sizeof(TO) / 2; ++h)
            dst[h] = pack(acc[v] + h * (16 / sizeof(TO)), (TO*)nullptr);
        }
      }
    }
  }
}

}  // namespace

cudaError_t launch_combine(const void* Y, const int32_t* tok_ptr, const int32_t* tok_ent,
                           const Shape& s, bool y_f32, bool out_f32, void* out, int sm_count,
                           cudaStream_t st) {
  using bf = __nv_bfloat16;
  int64_t blocks = ceil_div(s.T, kWarps);
  int64_t cap = (int64_t)sm_count * 8;
  dim3 grid((unsigned)(blocks < cap ? blocks : cap));
  if (s.d % 8 != 0) return cudaErrorInvalidValue;
  if (y_f32 && out_f32)
    combine_kernel<float, float><<<grid, kThreads, 0, st>>>((const float*)Y, tok_ptr, tok_ent,
                                                            s.T, s.d, (float*)out);
  else if (y_f32)
    combine_kernel<float, bf><<<grid, kThreads, 0, st>>>((const float*)Y, tok_ptr, tok_ent, s.T,
                                                         s.d, (bf*)out);
  else if (out_f32)
    combine_kernel<bf, float><<<grid, kThreads, 0, st>>>((const bf*)Y, tok_ptr, tok_ent, s.T,
                                                         s.d, (float*)out);
  else
    combine_kernel<bf, bf><<<grid, kThreads, 0, st>>>((const bf*)Y, tok_ptr, tok_ent, s.T, s.d,
                                                      (bf*)out);
  return cudaGetLastError();
}

}  // namespace nmoe
