// Router GEMM + score function on the CUDA cores (fp32 FFMA).
//
// logits[t, e] = sum_k x[t, k] W_r[k, e] (+ bias[segment(t), e]); scores = softmax over
// the experts of each token (or sigmoid), written token-major [T, E] and expert-major
// [E, T]. (NucleusMoE-Image walkthrough, section 6.2: gate Linear, then softmax or
// sigmoid, viewed per expert.) Each 32-long k-chunk is summed with fp32 FMAs and the
// chunk sums are added in fp64; the score function runs in fp64 and each score is
// rounded once to fp32, so scores stay within 1e-5 relative of an fp64 reference even
// for logits of magnitude ~30.
//
// One block owns 32 tokens and every expert (E <= 256). Used for fp32 inputs and for
// bf16 shapes the tensor-core router does not take.
#include "nmoe_internal.cuh"

namespace nmoe {
namespace {

constexpr int kBM = 32;       // tokens per block
constexpr int kBK = 32;       // k per stage
constexpr int kThreads = 256; // 8 column groups x 32 rows
constexpr int kMaxE = 256;

template <typename T>
__global__ void __launch_bounds__(kThreads)
router_simt_kernel(const T* __restrict__ x, const T* __restrict__ W_r, int Tn, int d, int E,
                   int S, int score_fn, const float* __restrict__ bias,
                   float* __restrict__ scores, float* __restrict__ scores_t) {
  pdl_launch_dependents();
  pdl_wait();
  extern __shared__ double smem_d[];
  double* lg = smem_d;                                // [kBM][E + 1] logits / scores
  float* xs = reinterpret_cast<float*>(lg + kBM * (E + 1));  // [kBM][kBK + 1]
  float* ws = xs + kBM * (kBK + 1);                   // [kBK][E]
  const int tid = threadIdx.x;
  const int t0 = blockIdx.x * kBM;
  const int r = tid >> 3;                  // row 0..31
  const int cg = tid & 7;                  // expert group: experts cg, cg+8, ...

  double acc[kMaxE / 8];
#pragma unroll
  for (int j = 0; j < kMaxE / 8; ++j) acc[j] = 0.0;

  for (int k0 = 0; k0 < d; k0 += kBK) {
    for (int i = tid; i < kBM * kBK; i += kThreads) {
      int rr = i / kBK, kk = i % kBK;
      int t = t0 + rr, k = k0 + kk;
      xs[rr * (kBK + 1) + kk] = (t < Tn && k < d) ? to_f32(x[(int64_t)t * d + k]) : 0.f;
    }
    for (int i = tid; i < kBK * E; i += kThreads) {
      int kk = i / E, e = i % E;
      int k = k0 + kk;
      ws[kk * E + e] = (k < d) ? to_f32(W_r[(int64_t)k * E + e]) : 0.f;
    }
    __syncthreads();
    float part[kMaxE / 8];
#pragma unroll
    for (int j = 0; j < kMaxE / 8; ++j) part[j] = 0.f;
#pragma unroll 4
    for (int kk = 0; kk < kBK; ++kk) {
      float a = xs[r * (kBK + 1) + kk];
#pragma unroll
      for (int j = 0; j < kMaxE / 8; ++j) {
        int e = cg + 8 * j;
        if (e < E) part[j] = fmaf(a, ws[kk * E + e], part[j]);
      }
    }
#pragma unroll
    for (int j = 0; j < kMaxE / 8; ++j) acc[j] += (double)part[j];
    __syncthreads();
  }

  // logits to shared memory (plus the per-segment bias)
  {
    int t = t0 + r;
#pragma unroll
    for (int j = 0; j < kMaxE / 8; ++j) {
      int e = cg + 8 * j;
      if (e < E) {
        double v = acc[j];
        if (bias != nullptr && t < Tn) v += (double)bias[(int64_t)(t / S) * E + e];
        lg[r * (E + 1) + e] = v;
      }
    }
  }
  __syncthreads();

  // score function: one warp per token row
  const int warp = tid >> 5, lane = tid & 31;
  for (int rr = warp; rr < kBM; rr += kThreads / 32) {
    double* row = lg + rr * (E + 1);
    if (score_fn == NMOE_SCORE_SOFTMAX) {
      double m = -INFINITY;
      for (int e = lane; e < E; e += 32) m = fmax(m, row[e]);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) m = fmax(m, __shfl_xor_sync(0xffffffffu, m, o));
      double z = 0.0;
      for (int e = lane; e < E; e += 32) {
        double v = exp(row[e] - m);
        row[e] = v;
        z += v;
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
      for (int e = lane; e < E; e += 32) row[e] = row[e] / z;
    } else {
      for (int e = lane; e < E; e += 32) row[e] = 1.0 / (1.0 + exp(-row[e]));
    }
  }
  __syncthreads();

  // token-major scores: rows of E contiguous floats
  if (scores != nullptr) {
    for (int i = tid; i < kBM * E; i += kThreads) {
      int rr = i / E, e = i % E;
      int t = t0 + rr;
      if (t < Tn) scores[(int64_t)t * E + e] = (float)lg[rr * (E + 1) + e];
    }
  }
  // expert-major scores: for each expert, 32 consecutive tokens
  if (scores_t != nullptr) {
    for (int i = tid; i < kBM * E; i += kThreads) {
      int e = i / kBM, rr = i % kBM;
      int t = t0 + rr;
      if (t < Tn) scores_t[(int64_t)e * Tn + t] = (float)lg[rr * (E + 1) + e];
    }
  }
}

}  // namespace

cudaError_t launch_router_simt(const void* x, const void* W_r, const Shape& s, nmoe_dtype dt,
                               nmoe_score_fn fn, const float* bias, float* scores,
                               float* scores_t, cudaStream_t st) {
  size_t smem = sizeof(double) * (size_t)kBM * (s.E + 1) +
                sizeof(float) * (size_t)(kBM * (kBK + 1) + kBK * s.E);
  dim3 grid((unsigned)ceil_div(s.T, kBM));
  if (dt == NMOE_F32)
    return launch_kernel(router_simt_kernel<float>, grid, dim3(kThreads), smem, st, s.pdl, 1,
                         (const float*)x, (const float*)W_r, s.T, s.d, s.E, s.S, (int)fn, bias,
                         scores, scores_t);
  return launch_kernel(router_simt_kernel<__nv_bfloat16>, grid, dim3(kThreads), smem, st, s.pdl,
                       1, (const __nv_bfloat16*)x, (const __nv_bfloat16*)W_r, s.T, s.d, s.E, s.S,
                       (int)fn, bias, scores, scores_t);
}

}  // namespace nmoe
