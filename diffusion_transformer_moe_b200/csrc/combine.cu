// Deterministic weighted combine.
//
// NucleusMoE-Image walkthrough, section 6.2: the weighted outputs of the routed experts
// are added back onto their tokens (the page uses scatter_add, whose order of additions
// is not fixed). Here the down projection has already written every weighted expert
// output at its token-major position, so the combine is a segmented sum of contiguous
// rows:
//   out[t, :] = sum over r in [tok_ptr[t], tok_ptr[t+1]) of Y[r, :]
// in ascending expert order (the order of the token lists), accumulated in fp32 and
// rounded once to the output type. A token no expert chose gets an exact zero row.
//
// With the surrounding block's residual (section 6.3 of the walkthrough: the modulation
// gates go through clamp(-2, 2) and tanh), each stored sum becomes
//   out[t, :] = residual[t, :] + tanh(clamp(gate2[t / S, :], -2, 2)) * sum,
// in fp32 before the one rounding.
//
// Each CTA owns a contiguous token range, whose rows of Y form one contiguous span, and a
// slice of at most kMaxGroups 16-byte column groups; every thread owns one column group and
// walks the span row by row, adding into the current token's sum and storing it when the
// row index crosses the token's end: the memory access pattern of a plain copy, with no
// synchronisation between warps. Two walks are built. The register walk keeps eight loads
// in flight per thread. The ring walk (plain sum only) queues each thread's own 16-byte
// piece of the next kRing rows with cp.async into a private column of a shared-memory
// ring (a thread reads back only what it copied, so no barrier is needed), and does not
// fetch the rows of single-entry tokens at all. Measured on one B200: alone, the register
// walk streams faster (18.4 against 20.5 µs for 8192 one-row tokens of 8 KB, 152 against
// 177 µs for 32768 four-row tokens of 6 KB); inside the layer, the ring walk of short spans
// wins (the 1024 px layer 205.0 -> 198.7 µs): its rows of single-entry tokens cost
// nothing, and its shared-memory footprint matches the expert GEMMs' before it, so the SMs
// keep their shared-memory configuration across that boundary. Short spans (at most
// kRingRowsPerCta rows per CTA on average) take the ring walk, longer ones the register
// walk.
//
// When the down projection has already written the output row of every token that a
// single expert chose (its sum is that one term, rounded once), such a token's row of Y
// was never written: the ring does not fetch it (a bitmap of the CTA's span marks those
// rows), the walk adds whatever its slot holds into a sum that is then dropped, and the
// token costs neither a read nor a write here.
//
// Right after the tensor-core down GEMM (`early`), a CTA reads its token pointers and
// builds that bitmap before its programmatic-launch wait: that GEMM lets this kernel start
// only after its own wait, so the token lists, written before it, are already complete
// (1024 px layer: -1 µs per step, interleaved A/B in both orders, outputs bit-identical).
#include "nmoe_internal.cuh"
#include "sm100_ptx.cuh"

namespace nmoe {
namespace {

constexpr int kAhead = 8;                 // rows loaded per round
constexpr int kMaxTokPerCta = 2048;
constexpr int kMaxGroups = 512;           // column groups (threads) per CTA

template <typename T> struct Vec;        // 16 bytes of T, unpacked to fp32
template <> struct Vec<float> {
  static constexpr int N = 4;
  __device__ static void add(float* a, const uint4& v) {
    a[0] += __uint_as_float(v.x); a[1] += __uint_as_float(v.y);
    a[2] += __uint_as_float(v.z); a[3] += __uint_as_float(v.w);
  }
};
template <> struct Vec<__nv_bfloat16> {
  static constexpr int N = 8;
  __device__ static void add(float* a, const uint4& v) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[i]));
      a[2 * i] += f.x;
      a[2 * i + 1] += f.y;
    }
  }
};

template <int N>
__device__ __forceinline__ void store_out(float* dst, const float* a) {
#pragma unroll
  for (int i = 0; i < N; i += 4)
    *reinterpret_cast<float4*>(dst + i) = make_float4(a[i], a[i + 1], a[i + 2], a[i + 3]);
}
template <int N>
__device__ __forceinline__ void store_out(__nv_bfloat16* dst, const float* a) {
#pragma unroll
  for (int i = 0; i < N; i += 4) {
    __nv_bfloat162 h0 = __floats2bfloat162_rn(a[i], a[i + 1]);
    __nv_bfloat162 h1 = __floats2bfloat162_rn(a[i + 2], a[i + 3]);
    uint2 v;
    v.x = *reinterpret_cast<uint32_t*>(&h0);
    v.y = *reinterpret_cast<uint32_t*>(&h1);
    *reinterpret_cast<uint2*>(dst + i) = v;
  }
}

// n residual values (of x's type) from p, as fp32
template <int N>
__device__ __forceinline__ void load_res(const void* p, bool bf16, float* r) {
  if (bf16) {
    const __nv_bfloat162* h = static_cast<const __nv_bfloat162*>(p);
#pragma unroll
    for (int i = 0; i < N / 2; ++i) {
      const float2 f = __bfloat1622float2(h[i]);
      r[2 * i] = f.x;
      r[2 * i + 1] = f.y;
    }
  } else {
    const float4* f = static_cast<const float4*>(p);
#pragma unroll
    for (int i = 0; i < N / 4; ++i) {
      const float4 v = f[i];
      r[4 * i] = v.x; r[4 * i + 1] = v.y; r[4 * i + 2] = v.z; r[4 * i + 3] = v.w;
    }
  }
}

// residual + tanh(clamp(gate, -2, 2)) * sum, on the N columns of one group
template <int N>
struct Gated {
  const void* res;     // NULL: plain sum
  bool res_bf16;
  const float* gate2;  // [n_seg, d] or NULL (gate 1)
  int d, S, col;
  int seg = -1;
  float g[N];
  __device__ __forceinline__ void apply(int t, float* acc) {
    if (res == nullptr) return;
    if (gate2 != nullptr && t / S != seg) {
      seg = t / S;
#pragma unroll
      for (int i = 0; i < N; ++i)
        g[i] = tanhf(fminf(fmaxf(gate2[(int64_t)seg * d + col + i], -2.f), 2.f));
    }
    float r[N];
    const size_t esz = res_bf16 ? 2 : 4;
    load_res<N>(static_cast<const char*>(res) + ((int64_t)t * d + col) * esz, res_bf16, r);
#pragma unroll
    for (int i = 0; i < N; ++i) acc[i] = r[i] + (gate2 != nullptr ? g[i] : 1.f) * acc[i];
  }
};

// One CTA: tokens [t0, t1) (blockIdx.x), column groups of blockIdx.y. RES: the block's
// gated residual is applied to each stored sum (its gate and residual registers make that
// variant one CTA per SM; the plain sum fits two).
template <typename TY, typename TO, bool RES>
__global__ void __launch_bounds__(kMaxGroups, RES ? 1 : 2)
combine_kernel(const TY* __restrict__ Y, const int32_t* __restrict__ tok_ptr, int Tn, int d,
               int tok_per_cta, TO* __restrict__ out, const void* __restrict__ residual,
               int res_bf16, const float* __restrict__ gate2, int S, int64_t y_rows,
               int skip_single, int early, unsigned* __restrict__ err) {
  constexpr int N = Vec<TY>::N;          // columns per 16-byte group
  pdl_launch_dependents();
  __shared__ int s_ptr[kMaxTokPerCta + 1];
  const int t0 = min(Tn, (int)blockIdx.x * tok_per_cta), t1 = min(Tn, t0 + tok_per_cta);
  if (!early) pdl_wait();
  for (int i = threadIdx.x; i <= t1 - t0; i += blockDim.x) s_ptr[i] = tok_ptr[t0 + i];
  __syncthreads();
  if (early) pdl_wait();  // Y (and the direct output rows) are complete
  if (t0 >= t1) return;
  if (kDebugChecks) {
    // debug build: every span must run forwards and inside Y, else nothing is read
    bool bad = false;
    for (int i = threadIdx.x; i <= t1 - t0; i += blockDim.x)
      bad |= s_ptr[i] < 0 || s_ptr[i] > y_rows || (i > 0 && s_ptr[i] < s_ptr[i - 1]);
    if (__syncthreads_or(bad)) {
      if (threadIdx.x == 0) atomicOr(err, kErrDeviceCheck);
      return;
    }
  }
  const int grp = blockIdx.y * blockDim.x + threadIdx.x;
  if (grp >= d / N) return;
  const int r0 = s_ptr[0], r1 = s_ptr[t1 - t0];
  const int col = grp * N;
  const int64_t stride = d / N;          // 16-byte groups per row
  [[maybe_unused]] Gated<N> gt{residual, res_bf16 != 0, gate2, d, S, col};
  const uint4* src = reinterpret_cast<const uint4*>(Y) + grp;
  float acc[N];
#pragma unroll
  for (int i = 0; i < N; ++i) acc[i] = 0.f;
  // token t's sum is complete: store it (unless the down projection already did)
  auto finish = [&](int t) {
    const int i = t - t0;
    if (!(skip_single && s_ptr[i + 1] - s_ptr[i] == 1)) {
      if (RES) gt.apply(t, acc);
      store_out<N>(out + (int64_t)t * d + col, acc);
    }
#pragma unroll
    for (int k = 0; k < N; ++k) acc[k] = 0.f;
  };
  int t = t0;                            // token whose sum is being built
  int tend = s_ptr[1];                   // its rows end here
  for (int r = r0; r < r1; r += kAhead) {
    uint4 v[kAhead];
#pragma unroll
    for (int k = 0; k < kAhead; ++k)
      v[k] = r + k < r1 ? __ldg(src + (int64_t)(r + k) * stride) : make_uint4(0, 0, 0, 0);
#pragma unroll
    for (int k = 0; k < kAhead; ++k) {
      if (r + k < r1) {
        while (r + k >= tend) {          // token t is complete (or had no rows)
          finish(t);
          ++t;
          tend = s_ptr[t - t0 + 1];
        }
        Vec<TY>::add(acc, v[k]);
      }
    }
  }
  for (; t < t1; ++t) finish(t);         // the last token and any empty ones after it
}

constexpr int kRing = 12;            // rows each thread has in flight (16 bytes of each)
constexpr int kRingRowsPerCta = 96;  // longest average span that takes the ring walk
constexpr int kSkipWords = 256;      // spans up to 8192 rows get the skip bitmap

// The plain sum (no residual): tokens [t0, t1) of blockIdx.x, column groups of
// blockIdx.y, two CTAs per SM.
template <typename TY, typename TO>
__global__ void __launch_bounds__(kMaxGroups, 2)
combine_ring_kernel(const TY* __restrict__ Y, const int32_t* __restrict__ tok_ptr, int Tn,
                    int d, int tok_per_cta, TO* __restrict__ out, int64_t y_rows,
                    int skip_single, int early, unsigned* __restrict__ err) {
  constexpr int N = Vec<TY>::N;
  pdl_launch_dependents();
  __shared__ int s_ptr[kMaxTokPerCta + 1];
  __shared__ uint32_t s_live[kSkipWords];  // bit r - r0: row r is fetched
  extern __shared__ uint4 s_ring[];        // [kRing][blockDim.x]
  const int t0 = min(Tn, (int)blockIdx.x * tok_per_cta), t1 = min(Tn, t0 + tok_per_cta);
  if (!early) pdl_wait();
  for (int i = threadIdx.x; i <= t1 - t0; i += blockDim.x) s_ptr[i] = tok_ptr[t0 + i];
  __syncthreads();
  if (t0 >= t1) return;
  if (kDebugChecks) {
    // debug build: every span must run forwards and inside Y, else nothing is read
    bool bad = false;
    for (int i = threadIdx.x; i <= t1 - t0; i += blockDim.x)
      bad |= s_ptr[i] < 0 || s_ptr[i] > y_rows || (i > 0 && s_ptr[i] < s_ptr[i - 1]);
    if (__syncthreads_or(bad)) {
      if (threadIdx.x == 0) atomicOr(err, kErrDeviceCheck);
      return;
    }
  }
  const int r0 = s_ptr[0], r1 = s_ptr[t1 - t0];
  // rows of single-entry tokens are not fetched (their rows of Y were never written)
  const bool skip = skip_single && r1 - r0 <= 32 * kSkipWords;
  if (skip) {
    for (int w = threadIdx.x; w < kSkipWords; w += blockDim.x) s_live[w] = ~0u;
    __syncthreads();
    for (int i = threadIdx.x; i < t1 - t0; i += blockDim.x)
      if (s_ptr[i + 1] - s_ptr[i] == 1) {
        const int r = s_ptr[i] - r0;
        atomicAnd(&s_live[r >> 5], ~(1u << (r & 31)));
      }
    __syncthreads();
  }
  if (early) pdl_wait();  // Y is complete
  const int grp = blockIdx.y * blockDim.x + threadIdx.x;
  if (grp >= d / N) return;
  const int col = grp * N;
  const int64_t stride = d / N;          // 16-byte groups per row
  const uint4* src = reinterpret_cast<const uint4*>(Y) + grp;
  uint4* ring = s_ring + threadIdx.x;    // this thread's column of the ring
  const int nt = blockDim.x;
  auto fetch = [&](int r, int slot) {
    if (r < r1 && (!skip || ((s_live[(r - r0) >> 5] >> ((r - r0) & 31)) & 1u)))
      ptx::cp_async16(ring + slot * nt, src + (int64_t)r * stride);
    ptx::cp_async_commit();              // one group per row, empty or not
  };
  for (int k = 0; k < kRing; ++k) fetch(r0 + k, k);
  float acc[N];
#pragma unroll
  for (int i = 0; i < N; ++i) acc[i] = 0.f;
  // token t's sum is complete: store it (unless the down projection already did)
  auto finish = [&](int t) {
    const int i = t - t0;
    if (!(skip_single && s_ptr[i + 1] - s_ptr[i] == 1))
      store_out<N>(out + (int64_t)t * d + col, acc);
#pragma unroll
    for (int k = 0; k < N; ++k) acc[k] = 0.f;
  };
  int t = t0;                            // token whose sum is being built
  int tend = s_ptr[1];                   // its rows end here
  int slot = 0;
  for (int r = r0; r < r1; ++r) {
    ptx::cp_async_wait<kRing - 1>();     // row r's group is complete (groups complete in order)
    const uint4 v = ring[slot * nt];
    while (r >= tend) {                  // token t is complete (or had no rows)
      finish(t);
      ++t;
      tend = s_ptr[t - t0 + 1];
    }
    Vec<TY>::add(acc, v);                // v is in registers before its slot is refilled
    fetch(r + kRing, slot);
    if (++slot == kRing) slot = 0;
  }
  ptx::cp_async_wait<0>();               // no copy is still writing when the CTA exits
  for (; t < t1; ++t) finish(t);         // the last token and any empty ones after it
}

template <typename TY, typename TO>
cudaError_t launch_typed(const void* Y, const int32_t* tok_ptr, const Shape& s, void* out,
                         const void* residual, bool res_bf16, const float* gate2,
                         bool skip_single, unsigned* err, int sm_count, cudaStream_t st) {
  constexpr int N = Vec<TY>::N;
  const int ngroups = s.d / N;
  // column slices of at most kMaxGroups groups, as even as possible
  const int slices = (int)ceil_div(ngroups, kMaxGroups);
  int threads = (int)ceil_div(ceil_div(ngroups, slices), 32) * 32;
  // two CTAs per SM, each a contiguous token range
  int ranges = (2 * sm_count + slices - 1) / slices;
  if (ranges > s.T) ranges = s.T;
  int per = (int)ceil_div(s.T, ranges);
  if (per > kMaxTokPerCta) per = kMaxTokPerCta;
  ranges = (int)ceil_div(s.T, per);
  const dim3 grid((unsigned)ranges, (unsigned)slices);
  if (residual != nullptr)
    return launch_kernel(combine_kernel<TY, TO, true>, grid, dim3(threads), 0, st, s.pdl, 1,
                         (const TY*)Y, tok_ptr, s.T, s.d, per, (TO*)out, residual,
                         (int)res_bf16, gate2, s.S, s.y_rows, (int)skip_single,
                         (int)s.after_gemm2, err);
  if (s.y_rows <= (int64_t)kRingRowsPerCta * ranges)
    return launch_kernel(combine_ring_kernel<TY, TO>, grid, dim3(threads),
                         (size_t)kRing * threads * 16, st, s.pdl, 1, (const TY*)Y, tok_ptr,
                         s.T, s.d, per, (TO*)out, s.y_rows, (int)skip_single,
                         (int)s.after_gemm2, err);
  return launch_kernel(combine_kernel<TY, TO, false>, grid, dim3(threads), 0, st, s.pdl, 1,
                       (const TY*)Y, tok_ptr, s.T, s.d, per, (TO*)out, residual,
                       (int)res_bf16, gate2, s.S, s.y_rows, (int)skip_single,
                       (int)s.after_gemm2, err);
}

}  // namespace

cudaError_t launch_combine(const void* Y, const int32_t* tok_ptr, const Shape& s, bool y_f32,
                           bool out_f32, void* out, const void* residual, bool res_bf16,
                           const float* gate2, bool skip_single, unsigned* err, int sm_count,
                           cudaStream_t st) {
  using bf = __nv_bfloat16;
  if (s.d % 8 != 0) return cudaErrorInvalidValue;
  auto go = [&](auto launch) {
    return launch(Y, tok_ptr, s, out, residual, res_bf16, gate2, skip_single, err, sm_count,
                  st);
  };
  if (y_f32 && out_f32) return go(launch_typed<float, float>);
  if (y_f32) return go(launch_typed<float, bf>);
  if (out_f32) return go(launch_typed<bf, float>);
  return go(launch_typed<bf, bf>);
}

}  // namespace nmoe
