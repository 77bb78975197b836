// Grouped expert GEMMs on the CUDA cores (fp32 FFMA, fp32 accumulation).
//
// The exact-fp32 path of the packed SwiGLU experts (NucleusMoE-Image walkthrough,
// section 6: fused gate/up projection, then the down projection, "two grouped matmuls"):
//   gemm1: H[e, s, :] = silu(x[idx[e,s]] W1_e) * (x[idx[e,s]] W3_e)
//   gemm2: Y[ent_pos[e*Ce + s], :] = gate[e, s] * (H[e, s, :] W2_e)
// The rows of expert e are gathered straight from x through idx; there is no permuted
// copy of the tokens. Used for fp32 inputs; bf16 inputs take the tcgen05 kernels.
#include "nmoe_internal.cuh"

namespace nmoe {
namespace {

constexpr int kBM = 64, kBN = 64, kBK = 16, kThreads = 256;

__device__ __forceinline__ float silu_f32(float g) { return g / (1.f + expf(-g)); }

template <typename T, typename TH>
__global__ void __launch_bounds__(kThreads)
gemm1_simt_kernel(const T* __restrict__ x, const int32_t* __restrict__ idx,
                  const T* __restrict__ W1, const T* __restrict__ W3, int d, int F, int Ce,
                  TH* __restrict__ H) {
  __shared__ float As[kBK][kBM + 4];
  __shared__ float Bg[kBK][kBN + 4];
  __shared__ float Bu[kBK][kBN + 4];
  __shared__ int rows[kBM];
  pdl_launch_dependents();
  pdl_wait();
  const int e = blockIdx.z, m0 = blockIdx.y * kBM, n0 = blockIdx.x * kBN;
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  // NULL idx: identity row map (the shared expert)
  if (tid < kBM)
    rows[tid] = (m0 + tid < Ce) ? (idx ? idx[(int64_t)e * Ce + m0 + tid] : m0 + tid) : -1;
  __syncthreads();
  const T* w1 = W1 + (int64_t)e * d * F;
  const T* w3 = W3 + (int64_t)e * d * F;
  float ag[4][4] = {}, au[4][4] = {};
  for (int k0 = 0; k0 < d; k0 += kBK) {
#pragma unroll
    for (int j = 0; j < kBM * kBK / kThreads; ++j) {
      int i = tid + j * kThreads;
      int r = i / kBK, kk = i % kBK, k = k0 + kk;
      As[kk][r] = (rows[r] >= 0 && k < d) ? to_f32(x[(int64_t)rows[r] * d + k]) : 0.f;
    }
#pragma unroll
    for (int j = 0; j < kBK * kBN / kThreads; ++j) {
      int i = tid + j * kThreads;
      int kk = i / kBN, n = i % kBN, k = k0 + kk;
      bool ok = k < d && n0 + n < F;
      Bg[kk][n] = ok ? to_f32(w1[(int64_t)k * F + n0 + n]) : 0.f;
      Bu[kk][n] = ok ? to_f32(w3[(int64_t)k * F + n0 + n]) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < kBK; ++kk) {
      float a[4], bg[4], bu[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) { bg[j] = Bg[kk][tx * 4 + j]; bu[j] = Bu[kk][tx * 4 + j]; }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          ag[i][j] = fmaf(a[i], bg[j], ag[i][j]);
          au[i][j] = fmaf(a[i], bu[j], au[i][j]);
        }
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    int s = m0 + ty * 4 + i;
    if (s >= Ce) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      int f = n0 + tx * 4 + j;
      if (f < F) H[((int64_t)e * Ce + s) * F + f] = from_f32<TH>(silu_f32(ag[i][j]) * au[i][j]);
    }
  }
}

template <typename T, typename TH, typename TY>
__global__ void __launch_bounds__(kThreads)
gemm2_simt_kernel(const TH* __restrict__ H, const float* __restrict__ gate,
                  const T* __restrict__ W2, const int32_t* __restrict__ ent_pos, int d, int F,
                  int Ce, TY* __restrict__ Y) {
  __shared__ float As[kBK][kBM + 4];
  __shared__ float Bs[kBK][kBN + 4];
  pdl_launch_dependents();
  pdl_wait();
  const int e = blockIdx.z, m0 = blockIdx.y * kBM, n0 = blockIdx.x * kBN;
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const TH* h = H + (int64_t)e * Ce * F;
  const T* w2 = W2 + (int64_t)e * F * d;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < F; k0 += kBK) {
#pragma unroll
    for (int j = 0; j < kBM * kBK / kThreads; ++j) {
      int i = tid + j * kThreads;
      int r = i / kBK, kk = i % kBK, k = k0 + kk;
      As[kk][r] = (m0 + r < Ce && k < F) ? to_f32(h[(int64_t)(m0 + r) * F + k]) : 0.f;
    }
#pragma unroll
    for (int j = 0; j < kBK * kBN / kThreads; ++j) {
      int i = tid + j * kThreads;
      int kk = i / kBN, n = i % kBN, k = k0 + kk;
      Bs[kk][n] = (k < F && n0 + n < d) ? to_f32(w2[(int64_t)k * d + n0 + n]) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < kBK; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = Bs[kk][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    int s = m0 + ty * 4 + i;
    if (s >= Ce) continue;
    float w = gate ? gate[(int64_t)e * Ce + s] : 1.f;  // NULL gate: weight 1
    const int64_t yrow = ent_pos[(int64_t)e * Ce + s];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      int n = n0 + tx * 4 + j;
      if (n < d) Y[yrow * d + n] = from_f32<TY>(w * acc[i][j]);
    }
  }
}

}  // namespace

cudaError_t launch_gemm1_simt(const void* x, const int32_t* idx, const void* W1, const void* W3,
                              const Shape& s, nmoe_dtype dt, bool h_f32, void* H,
                              cudaStream_t st) {
  using bf = __nv_bfloat16;
  dim3 grid((unsigned)ceil_div(s.F, kBN), (unsigned)ceil_div(s.Ce, kBM), (unsigned)s.E);
  if (dt == NMOE_F32)
    return launch_kernel(gemm1_simt_kernel<float, float>, grid, dim3(kThreads), 0, st, s.pdl, 1, 
        (const float*)x, idx, (const float*)W1, (const float*)W3, s.d, s.F, s.Ce, (float*)H);
  else if (h_f32)
    return launch_kernel(gemm1_simt_kernel<bf, float>, grid, dim3(kThreads), 0, st, s.pdl, 1, 
        (const bf*)x, idx, (const bf*)W1, (const bf*)W3, s.d, s.F, s.Ce, (float*)H);
  else
    return launch_kernel(gemm1_simt_kernel<bf, bf>, grid, dim3(kThreads), 0, st, s.pdl, 1, 
        (const bf*)x, idx, (const bf*)W1, (const bf*)W3, s.d, s.F, s.Ce, (bf*)H);
}

cudaError_t launch_gemm2_simt(const void* H, const float* gate, const void* W2,
                              const int32_t* ent_pos, const Shape& s, nmoe_dtype dt, bool h_f32,
                              bool y_f32, void* Y, cudaStream_t st) {
  using bf = __nv_bfloat16;
  dim3 grid((unsigned)ceil_div(s.d, kBN), (unsigned)ceil_div(s.Ce, kBM), (unsigned)s.E);
  if (dt == NMOE_F32)
    return launch_kernel(gemm2_simt_kernel<float, float, float>, grid, dim3(kThreads), 0, st, s.pdl, 1, 
        (const float*)H, gate, (const float*)W2, ent_pos, s.d, s.F, s.Ce, (float*)Y);
  else if (h_f32 && y_f32)
    return launch_kernel(gemm2_simt_kernel<bf, float, float>, grid, dim3(kThreads), 0, st, s.pdl, 1, 
        (const float*)H, gate, (const bf*)W2, ent_pos, s.d, s.F, s.Ce, (float*)Y);
  else if (!h_f32 && !y_f32)
    return launch_kernel(gemm2_simt_kernel<bf, bf, bf>, grid, dim3(kThreads), 0, st, s.pdl, 1, 
        (const bf*)H, gate, (const bf*)W2, ent_pos, s.d, s.F, s.Ce, (bf*)Y);
  return cudaErrorInvalidValue;
}

}  // namespace nmoe
