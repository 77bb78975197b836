// Expert-choice top-C selection and the token -> (expert, slot) lists.
//
// NucleusMoE-Image walkthrough, section 6.2: every expert takes its top `capacity`
// tokens along the token axis, so each expert receives exactly that many tokens. The
// page leaves ties open; here the key is (fp32 score, -token index), so a tie goes to
// the lower token index, and the chosen tokens are written in ascending token order.
//
// select_kernel: one CTA per (expert, segment). Scores are non-negative floats, so their
// bit patterns order like unsigned integers. The CTA finds the exact C-th largest key
// with an MSB-first radix select (four 8-bit digits; warp-aggregated shared-memory
// histograms built with __match_any_sync), then compacts in token order: every key
// above the threshold, plus the first (C - #above) keys equal to it.
//
// csr_kernel: one CTA per 32 consecutive tokens. Because each expert's list is sorted,
// the number of entries that belong to tokens before t0 is sum_e lower_bound(idx[e], t0),
// so every CTA finds its output offset with E binary searches: no global scan, no
// atomics, and every output element has exactly one writer. It also records, for every
// (expert, slot), its position in that token-major order (ent_pos), where the down-
// projection writes the row so that the combine reads each token's rows contiguously.
#include "nmoe_internal.cuh"

namespace nmoe {
namespace {

constexpr int kSelThreads = 1024;
constexpr int kSelWarps = kSelThreads / 32;
// Rows up to this many keys are staged in shared memory; longer rows are read from
// global memory (L2) on every pass.
constexpr int kSelMaxCached = 48 * 1024;

__device__ __forceinline__ uint32_t load_key(const uint32_t* p) { return *p; }

// Exclusive block scan of two counters at once; returns the block totals.
__device__ __forceinline__ void block_scan2(int a, int b, int* ex_a, int* ex_b, int* tot_a,
                                            int* tot_b, int* sh /* 2 * kSelWarps + 2 */) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int ia = a, ib = b;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int va = __shfl_up_sync(0xffffffffu, ia, o);
    int vb = __shfl_up_sync(0xffffffffu, ib, o);
    if (lane >= o) { ia += va; ib += vb; }
  }
  if (lane == 31) { sh[warp] = ia; sh[kSelWarps + warp] = ib; }
  __syncthreads();
  if (warp == 0) {
    int wa = lane < kSelWarps ? sh[lane] : 0;
    int wb = lane < kSelWarps ? sh[kSelWarps + lane] : 0;
    int sa = wa, sb = wb;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int va = __shfl_up_sync(0xffffffffu, sa, o);
      int vb = __shfl_up_sync(0xffffffffu, sb, o);
      if (lane >= o) { sa += va; sb += vb; }
    }
    if (lane < kSelWarps) { sh[lane] = sa - wa; sh[kSelWarps + lane] = sb - wb; }
    if (lane == kSelWarps - 1) { sh[2 * kSelWarps] = sa; sh[2 * kSelWarps + 1] = sb; }
  }
  __syncthreads();
  *ex_a = sh[warp] + ia - a;
  *ex_b = sh[kSelWarps + warp] + ib - b;
  *tot_a = sh[2 * kSelWarps];
  *tot_b = sh[2 * kSelWarps + 1];
  __syncthreads();
}

__global__ void __launch_bounds__(kSelThreads)
select_kernel(const float* __restrict__ scores_t, int64_t Tn, int S, int C, int Ce,
              int cached, int32_t* __restrict__ idx, float* __restrict__ gate,
              unsigned* __restrict__ err) {
  pdl_launch_dependents();
  pdl_wait();
  extern __shared__ uint32_t s_keys[];
  __shared__ unsigned s_hist[256];
  __shared__ int s_scan[2 * kSelWarps + 2];
  __shared__ unsigned s_digit, s_above, s_bad;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int e = blockIdx.x, g = blockIdx.y;
  const uint32_t* row =
      reinterpret_cast<const uint32_t*>(scores_t + (int64_t)e * Tn + (int64_t)g * S);

  if (tid == 0) s_bad = 0;
  __syncthreads();
  const uint32_t* keys = row;
  {
    // Non-negative finite scores only: sign bit clear and below +inf.
    unsigned bad = 0;
    if (cached) {
      for (int i = tid; i < S; i += kSelThreads) {
        uint32_t k = row[i];
        bad |= (k >= 0x7f800000u);
        s_keys[i] = k;
      }
      keys = s_keys;
    } else {
      for (int i = tid; i < S; i += kSelThreads) bad |= (row[i] >= 0x7f800000u);
    }
    if (__any_sync(0xffffffffu, bad) && lane == 0) atomicOr(&s_bad, 1u);
  }
  __syncthreads();
  if (s_bad) {
    if (tid == 0) atomicOr(err, kErrDeviceCheck);
  }

  // MSB-first radix select of the C-th largest key.
  uint32_t prefix = 0, pmask = 0;
  int k = C;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = tid; i < 256; i += kSelThreads) s_hist[i] = 0;
    __syncthreads();
    for (int i0 = 0; i0 < S; i0 += kSelThreads) {
      int i = i0 + tid;
      uint32_t key = i < S ? load_key(keys + i) : 0u;
      bool in = (i < S) && ((key & pmask) == prefix);
      unsigned digit = in ? ((key >> shift) & 255u) : 256u;
      unsigned peers = __match_any_sync(0xffffffffu, digit);
      if (in && lane == __ffs(peers) - 1) atomicAdd(&s_hist[digit], (unsigned)__popc(peers));
    }
    __syncthreads();
    if (warp == 0) {
      // lane L owns bins [8L, 8L+8); count of keys with a larger digit than each bin
      unsigned c[8], mine = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) { c[j] = s_hist[lane * 8 + j]; mine += c[j]; }
      // inclusive suffix sum over lanes (higher lanes hold higher digits)
      unsigned suf = mine;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        unsigned v = __shfl_down_sync(0xffffffffu, suf, o);
        if (lane + o < 32) suf += v;
      }
      unsigned above = suf - mine;  // keys in bins owned by higher lanes
#pragma unroll
      for (int j = 7; j >= 0; --j) {
        if (above < (unsigned)k && above + c[j] >= (unsigned)k) {
          s_digit = (unsigned)(lane * 8 + j);
          s_above = above;
        }
        above += c[j];
      }
    }
    __syncthreads();
    k -= (int)s_above;
    prefix |= s_digit << shift;
    pmask |= 255u << shift;
    __syncthreads();
  }
  const uint32_t thr = prefix;  // the C-th largest key; take k keys equal to it

  // Ordered compaction: thread tid owns a contiguous run of keys.
  const int per = (S + kSelThreads - 1) / kSelThreads;
  const int b0 = min(S, tid * per), b1 = min(S, b0 + per);
  int n_gt = 0, n_eq = 0;
  for (int i = b0; i < b1; ++i) {
    uint32_t key = load_key(keys + i);
    n_gt += key > thr;
    n_eq += key == thr;
  }
  int ex_gt, ex_eq, tot_gt, tot_eq;
  block_scan2(n_gt, n_eq, &ex_gt, &ex_eq, &tot_gt, &tot_eq, s_scan);
  int eq_seen = ex_eq;
  int pos = ex_gt + min(ex_eq, k);
  int32_t* out_idx = idx + (int64_t)e * Ce + (int64_t)g * C;
  float* out_gate = gate + (int64_t)e * Ce + (int64_t)g * C;
  for (int i = b0; i < b1; ++i) {
    uint32_t key = load_key(keys + i);
    bool take = key > thr;
    if (key == thr) { take = eq_seen < k; ++eq_seen; }
    if (take) {
      out_idx[pos] = g * S + i;
      out_gate[pos] = __uint_as_float(key);
      ++pos;
    }
  }
  if (tid == 0 && tot_gt + min(tot_eq, k) != C) atomicOr(err, kErrDeviceCheck);
}

constexpr int kCsrTok = 32;
constexpr int kCsrThreads = 256;

__device__ __forceinline__ int lower_bound_i32(const int32_t* a, int n, int v) {
  int lo = 0, hi = n;
  while (lo < hi) {
    int mid = (lo + hi) >> 1;
    if (a[mid] < v) lo = mid + 1; else hi = mid;
  }
  return lo;
}

__global__ void __launch_bounds__(kCsrThreads)
csr_kernel(const int32_t* __restrict__ idx, int Tn, int E, int Ce, int32_t* __restrict__ tok_ptr,
           int32_t* __restrict__ tok_ent, int32_t* __restrict__ ent_pos, float* __restrict__ gate,
           int normalize, float route_scale, unsigned* __restrict__ err) {
  pdl_launch_dependents();
  pdl_wait();
  extern __shared__ int s_slot[];  // [kCsrTok][E]: slot of (token, expert) or -1
  __shared__ int s_lo[256], s_hi[256];
  __shared__ int s_base_part[kCsrThreads / 32];
  __shared__ int s_cnt[kCsrTok], s_off[kCsrTok];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int t0 = blockIdx.x * kCsrTok;
  const int t1 = min(Tn, t0 + kCsrTok);

  for (int i = tid; i < kCsrTok * E; i += kCsrThreads) s_slot[i] = -1;
  int part = 0;
  for (int e = tid; e < E; e += kCsrThreads) {
    const int32_t* row = idx + (int64_t)e * Ce;
    int lo = lower_bound_i32(row, Ce, t0);
    int hi = lower_bound_i32(row, Ce, t1);
    s_lo[e] = lo;
    s_hi[e] = hi;
    part += lo;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
  if (lane == 0) s_base_part[warp] = part;
  __syncthreads();
  int base = 0;
#pragma unroll
  for (int w = 0; w < kCsrThreads / 32; ++w) base += s_base_part[w];

  // scatter this block's entries into the (token, expert) slot map
  for (int e = warp; e < E; e += kCsrThreads / 32) {
    const int32_t* row = idx + (int64_t)e * Ce;
    for (int s = s_lo[e] + lane; s < s_hi[e]; s += 32) {
      int t = row[s];
      if (t >= t0 && t < t1) s_slot[(t - t0) * E + e] = s;
      else atomicOr(err, kErrDeviceCheck);
    }
  }
  __syncthreads();

  // per-token counts and their exclusive scan (one warp: kCsrTok == 32)
  if (warp == 0) {
    int c = 0;
    if (t0 + lane < t1)
      for (int e = 0; e < E; ++e) c += s_slot[lane * E + e] >= 0;
    int inc = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int v = __shfl_up_sync(0xffffffffu, inc, o);
      if (lane >= o) inc += v;
    }
    s_cnt[lane] = c;
    s_off[lane] = inc - c;
    if (t0 + lane < t1) tok_ptr[t0 + lane] = base + inc - c;
    if (t0 + lane == Tn - 1) tok_ptr[Tn] = base + inc;
  }
  __syncthreads();

  // entries of each token in ascending expert order: one warp per token
  for (int r = warp; r < t1 - t0; r += kCsrThreads / 32) {
    int out = base + s_off[r];
    const int* srow = s_slot + r * E;
    for (int e0 = 0; e0 < E; e0 += 32) {
      int e = e0 + lane;
      int sl = e < E ? srow[e] : -1;
      unsigned m = __ballot_sync(0xffffffffu, sl >= 0);
      if (sl >= 0) {
        const int at = out + __popc(m & ((1u << lane) - 1u));
        tok_ent[at] = e * Ce + sl;
        if (ent_pos != nullptr) ent_pos[e * Ce + sl] = at;
      }
      out += __popc(m);
    }
    if (normalize) {
      __syncwarp();
      // fixed order: ascending expert, fp32
      float tot = 0.f;
      int beg = base + s_off[r], n = s_cnt[r];
      for (int j = 0; j < n; ++j) tot += gate[tok_ent[beg + j]];
      __syncwarp();  // every lane has read the raw gates before any is overwritten
      for (int j = lane; j < n; j += 32) {
        int v = tok_ent[beg + j];
        gate[v] = route_scale * (gate[v] / tot);
      }
    }
  }
}

}  // namespace

cudaError_t launch_select(const float* scores_t, const Shape& s, int32_t* idx, float* gate,
                          unsigned* err, cudaStream_t st) {
  int cached = s.S <= kSelMaxCached;
  size_t smem = cached ? sizeof(uint32_t) * (size_t)s.S : 0;
  dim3 grid((unsigned)s.E, (unsigned)s.n_seg);
  return launch_kernel(select_kernel, grid, dim3(kSelThreads), smem, st, s.pdl, 1, scores_t,
                       (int64_t)s.T, s.S, s.C, s.Ce, cached, idx, gate, err);
}

cudaError_t launch_csr(const int32_t* idx, const Shape& s, int32_t* tok_ptr, int32_t* tok_ent,
                       int32_t* ent_pos, float* gate, nmoe_combine combine, float route_scale,
                       unsigned* err, cudaStream_t st) {
  size_t smem = sizeof(int) * (size_t)kCsrTok * s.E;
  dim3 grid((unsigned)ceil_div(s.T, kCsrTok));
  return launch_kernel(csr_kernel, grid, dim3(kCsrThreads), smem, st, s.pdl, 1, idx, s.T, s.E,
                       s.Ce, tok_ptr, tok_ent, ent_pos, gate,
                       (int)(combine == NMOE_COMBINE_NORMALIZED), route_scale, err);
}

}  // namespace nmoe
