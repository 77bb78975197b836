// Expert-choice top-C selection and the token -> (expert, slot) lists.
//
// NucleusMoE-Image walkthrough, section 6.2: every expert takes its top `capacity`
// tokens along the token axis, so each expert receives exactly that many tokens. The
// page leaves ties open; here the key is (fp32 score, -token index), so a tie goes to
// the lower token index, and the chosen tokens are written in ascending token order.
//
// select_kernel: one CTA per (expert, segment). Scores are non-negative floats, so their
// bit patterns order like unsigned integers. The CTA stages its row of keys in shared
// memory with 16-byte loads and finds the exact C-th largest key with an MSB-first radix
// select over three digits (bits 31..20, 19..8, 7..0; shared-memory histograms). The
// first digit splits fp32 scores into bins an eighth of an octave wide, so the bin
// holding the threshold is a small share of the row: its keys are copied to a candidate
// list and the last two digits are counted over that list alone (a list of at most
// kRankMax keys is instead ranked directly, each key against all). The same sweep that
// lists the candidates records, 32 tokens to a word, which keys lie in a higher bin;
// once the threshold is known only the candidates' bits are added (above it, or equal
// to it); a block-wide scan over the words' popcounts then gives every chosen key (each key
// above the threshold, plus the first C - #above keys equal to it) its position in
// ascending token order, and, for every block of kBlockTok tokens, how many of the
// expert's entries come before the block (the boundary table).
//
// csr_kernel: one CTA per kBlockTok consecutive tokens runs csr_block (csr_block.cuh)
// from the boundary table; the standalone selection call, which has no scratch for the
// table, searches each expert's ascending token list instead. On the tensor-core path
// of the whole layer the same blocks are built inside the gate/up GEMM instead.
#include "csr_block.cuh"
#include "nmoe_internal.cuh"

namespace nmoe {
namespace {

constexpr int kSelThreads = 1024;
constexpr int kSelWarps = kSelThreads / 32;
// Rows up to this many keys are staged in shared memory; longer rows are read from
// global memory (L2) on every pass.
constexpr int kSelMaxCached = 40 * 1024;
constexpr int kBins = 4096;     // 12-bit digits; thread t owns bins [4t, 4t + 4)
constexpr int kCandMax = 4096;  // capacity of the candidate list
constexpr int kRankMax = 256;   // candidate lists up to this long are ranked directly
static_assert(kBins == 4 * kSelThreads, "four histogram bins per thread");

constexpr int kBlockTok = 32;   // tokens per CSR block (one warp lane per token)
static_assert(kBlockTok == 32, "one bitmap word per CSR block");

__device__ __forceinline__ unsigned lanemask_lt() {
  unsigned m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

// Bit k of the low byte of b moved to bit 4k (the other bits cleared).
__device__ __forceinline__ uint32_t spread4(uint32_t b) {
  b = (b | (b << 12)) & 0x000F000Fu;
  b = (b | (b << 6)) & 0x03030303u;
  return (b | (b << 3)) & 0x11111111u;
}

__device__ __forceinline__ unsigned is_bad(uint32_t key) {
  return key >= 0x7f800000u;  // negative, +inf or NaN
}

// Adds to hist[] the digit (key >> shift) & dmask of every key in src[0, n) whose bits
// under pmask equal prefix: one shared-memory atomic per key. The loop is bound by
// instruction issue, not by address conflicts: grouping equal digits first (with
// __match_any_sync, or a ballot on the first lane's digit) costs more than the
// conflicts it saves, even on rows full of equal scores.
__device__ __forceinline__ void histogram(const uint32_t* src, int n, uint32_t pmask,
                                          uint32_t prefix, int shift, uint32_t dmask,
                                          unsigned* hist) {
  for (int i = threadIdx.x; i < n; i += kSelThreads) {
    const uint32_t key = src[i];
    if ((key & pmask) == prefix) atomicAdd(&hist[(key >> shift) & dmask], 1u);
  }
}

// Exclusive block scan of two counters at once; returns the block totals.
__device__ __forceinline__ void block_scan2(int a, int b, int* ex_a, int* ex_b, int* tot_a,
                                            int* tot_b, int* sh /* 2 * kSelWarps + 2 */) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int ia = a, ib = b;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int va = __shfl_up_sync(0xffffffffu, ia, o);
    const int vb = __shfl_up_sync(0xffffffffu, ib, o);
    if (lane >= o) {
      ia += va;
      ib += vb;
    }
  }
  if (lane == 31) {
    sh[warp] = ia;
    sh[kSelWarps + warp] = ib;
  }
  __syncthreads();
  int wa = sh[lane], wb = sh[kSelWarps + lane];  // kSelWarps == 32
  int sa = wa, sb = wb;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int va = __shfl_up_sync(0xffffffffu, sa, o);
    const int vb = __shfl_up_sync(0xffffffffu, sb, o);
    if (lane >= o) {
      sa += va;
      sb += vb;
    }
  }
  *ex_a = __shfl_sync(0xffffffffu, sa - wa, warp) + ia - a;
  *ex_b = __shfl_sync(0xffffffffu, sb - wb, warp) + ib - b;
  *tot_a = __shfl_sync(0xffffffffu, sa, 31);
  *tot_b = __shfl_sync(0xffffffffu, sb, 31);
}

// The bin d that holds the k-th largest of the counted keys (bins in descending order):
// res[0] = d, res[1] = number of counted keys in higher bins, res[2] = hist[d]. Exactly
// one thread writes res; the caller synchronises before reading it.
__device__ __forceinline__ void find_digit(const unsigned* hist, unsigned k, unsigned* wsum,
                                           unsigned* res) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint4 c = reinterpret_cast<const uint4*>(hist)[tid];
  const unsigned mine = c.x + c.y + c.z + c.w;
  unsigned suf = mine;  // bins of this lane and the higher lanes of the warp
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned v = __shfl_down_sync(0xffffffffu, suf, o);
    if (lane + o < 32) suf += v;
  }
  if (lane == 0) wsum[warp] = suf;
  __syncthreads();
  unsigned wsuf = wsum[lane];  // then: warps lane .. 31
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned v = __shfl_down_sync(0xffffffffu, wsuf, o);
    if (lane + o < 32) wsuf += v;
  }
  const unsigned higher_warps = __shfl_sync(0xffffffffu, wsuf, (warp + 1) & 31);
  unsigned above = (warp == kSelWarps - 1 ? 0u : higher_warps) + (suf - mine);
  const unsigned cnt[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
  for (int j = 3; j >= 0; --j) {
    if (above < k && above + cnt[j] >= k) {
      res[0] = (unsigned)(4 * tid + j);
      res[1] = above;
      res[2] = cnt[j];
    }
    above += cnt[j];
  }
}

// MIN_CTAS = 2 (32 registers a thread, no spills) fits two CTAs on an SM, for calls with
// more rows than SMs (the model default shape's 128 experts x 2 segments run in one wave,
// not two: its selection 22.6 -> 19.2 us traced, interleaved A/B); with fewer rows the
// one-CTA build (more registers) runs.
template <int MIN_CTAS>
__global__ void __launch_bounds__(kSelThreads, MIN_CTAS)
select_kernel(const float* __restrict__ scores_t, int64_t Tn, int S, int C, int Ce, int E,
              int cached, int32_t* __restrict__ idx, float* __restrict__ gate,
              int32_t* __restrict__ bnd, unsigned* __restrict__ err) {
  pdl_launch_dependents();
  // dynamic: [keys, cached ? S (rounded up to 4) : 0][gt words, nw4][eq words, nw4]
  //          [the candidates' positions in the row, kCandMax]
  extern __shared__ __align__(16) uint32_t s_dyn[];
  __shared__ __align__(16) unsigned s_hist[kBins];
  __shared__ uint32_t s_cand[kCandMax];
  __shared__ unsigned s_wsum[kSelWarps];
  __shared__ int s_scan[2 * kSelWarps];
  __shared__ unsigned s_res[3];
  __shared__ unsigned s_ncand;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int e = blockIdx.x, g = blockIdx.y;
  const int nw = (S + 31) >> 5, nw4 = (nw + 3) & ~3;
  uint32_t* s_keys = s_dyn;
  uint32_t* s_gtw = s_dyn + (cached ? ((S + 3) & ~3) : 0);
  uint32_t* s_eqw = s_gtw + nw4;
  int32_t* s_cidx = reinterpret_cast<int32_t*>(s_eqw + nw4);

  reinterpret_cast<uint4*>(s_hist)[tid] = make_uint4(0u, 0u, 0u, 0u);
  if (tid == 0) s_ncand = 0;
  __syncthreads();  // the histogram is zero before the row's first digit is counted
  pdl_wait();

  const uint32_t* row =
      reinterpret_cast<const uint32_t*>(scores_t + (int64_t)e * Tn + (int64_t)g * S);
  const uint32_t* keys = row;
  // Non-negative finite scores only: sign bit clear and below +inf. The first digit's
  // histogram (bits 31..20) is counted as the row is read, with no pass of its own.
  unsigned bad = 0;
  if (cached) {
    int head = 0;
    if ((reinterpret_cast<uintptr_t>(row) & 15u) == 0) {
      const int n4 = S >> 2;
      const uint4* r4 = reinterpret_cast<const uint4*>(row);
      uint4* k4 = reinterpret_cast<uint4*>(s_keys);
#pragma unroll 4
      for (int i = tid; i < n4; i += kSelThreads) {
        const uint4 v = r4[i];
        bad |= is_bad(v.x) | is_bad(v.y) | is_bad(v.z) | is_bad(v.w);
        k4[i] = v;
        atomicAdd(&s_hist[v.x >> 20], 1u);
        atomicAdd(&s_hist[v.y >> 20], 1u);
        atomicAdd(&s_hist[v.z >> 20], 1u);
        atomicAdd(&s_hist[v.w >> 20], 1u);
      }
      head = 4 * n4;
    }
#pragma unroll 4
    for (int i = head + tid; i < S; i += kSelThreads) {
      const uint32_t v = row[i];
      bad |= is_bad(v);
      s_keys[i] = v;
      atomicAdd(&s_hist[v >> 20], 1u);
    }
    keys = s_keys;
  } else {
#pragma unroll 4
    for (int i = tid; i < S; i += kSelThreads) {
      const uint32_t v = row[i];
      bad |= is_bad(v);
      atomicAdd(&s_hist[v >> 20], 1u);
    }
  }
  if (__syncthreads_or((int)bad) && tid == 0) atomicOr(err, kErrDeviceCheck);

  // MSB-first radix select of the C-th largest key.
  const uint32_t* src = keys;
  int n = S;
  uint32_t prefix = 0, pmask = 0;
  int k = C;
  bool ranked = false;
  bool collected = false;  // candidates listed, and the bitmap words above their bin set
#pragma unroll 1
  for (int pass = 0; pass < 3 && !ranked; ++pass) {
    const int shift = pass == 0 ? 20 : (pass == 1 ? 8 : 0);
    const uint32_t dmask = pass == 2 ? 0xffu : 0xfffu;
    if (pass > 0) {  // the first digit was counted while the row was read
      histogram(src, n, pmask, prefix, shift, dmask, s_hist);
      __syncthreads();
    }
    find_digit(s_hist, (unsigned)k, s_wsum, s_res);
    __syncthreads();
    prefix |= s_res[0] << shift;
    pmask |= dmask << shift;
    k -= (int)s_res[1];
    const int nbin = (int)s_res[2];
    reinterpret_cast<uint4*>(s_hist)[tid] = make_uint4(0u, 0u, 0u, 0u);
    if (pass == 0 && nbin <= kCandMax) {
      // Keys of the threshold's bin, with their positions (their order is irrelevant
      // to the histograms), and, 32 keys to a word, which keys lie in a higher bin:
      // those are above the threshold whatever it is (the equal words start empty).
      if (cached) {
        // four keys per lane: a warp sweeps 128 consecutive keys (four words) per step
        for (int c0 = 128 * warp; c0 < S; c0 += 128 * kSelWarps) {
          const int i = c0 + 4 * lane;
          const uint4 v = *reinterpret_cast<const uint4*>(keys + i);
          const uint32_t kv[4] = {v.x, v.y, v.z, v.w};
          unsigned a[4];
          int nin = 0;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const bool live = i + j < S;
            a[j] = __ballot_sync(0xffffffffu, live && (kv[j] & pmask) > prefix);
            nin += live && (kv[j] & pmask) == prefix;
          }
          if (lane < 4) {  // word lane: keys c0 + 32 lane .. + 31 = lanes 8 lane .. + 7
            const int w = (c0 >> 5) + lane;
            if (w < nw) {
              uint32_t word = 0;
#pragma unroll
              for (int j = 0; j < 4; ++j) word |= spread4((a[j] >> (8 * lane)) & 0xffu) << j;
              s_gtw[w] = word;
              s_eqw[w] = 0u;
            }
          }
          // this lane's candidates go to consecutive slots after the warp's earlier lanes'
          int before = nin;
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const int t = __shfl_up_sync(0xffffffffu, before, o);
            if (lane >= o) before += t;
          }
          const int total = __shfl_sync(0xffffffffu, before, 31);
          before -= nin;
          if (total > 0) {
            unsigned base = 0;
            if (lane == 0) base = atomicAdd(&s_ncand, (unsigned)total);
            unsigned at = __shfl_sync(0xffffffffu, base, 0) + (unsigned)before;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              if (i + j < S && (kv[j] & pmask) == prefix) {
                if (at < (unsigned)kCandMax) {
                  s_cand[at] = kv[j];
                  s_cidx[at] = i + j;
                }
                ++at;
              }
            }
          }
        }
      } else for (int i0 = 0; i0 < S; i0 += kSelThreads) {
        const int i = i0 + tid;
        const uint32_t key = i < S ? keys[i] : 0u;
        const bool in = i < S && (key & pmask) == prefix;
        const unsigned above = __ballot_sync(0xffffffffu, i < S && (key & pmask) > prefix);
        const int w = (i0 >> 5) + warp;
        if (lane == 0 && w < nw) {
          s_gtw[w] = above;
          s_eqw[w] = 0u;
        }
        const unsigned b = __ballot_sync(0xffffffffu, in);
        if (b != 0u) {
          unsigned base = 0;
          if (lane == 0) base = atomicAdd(&s_ncand, (unsigned)__popc(b));
          base = __shfl_sync(0xffffffffu, base, 0);
          const unsigned at = base + (unsigned)__popc(b & lanemask_lt());
          if (in && at < (unsigned)kCandMax) {
            s_cand[at] = key;
            s_cidx[at] = i;
          }
        }
      }
      src = s_cand;
      n = nbin;
      collected = true;
      if (nbin <= kRankMax) {
        // Few candidates: rank them directly instead of two more digits. The k-th
        // largest candidate c has #{> c} < k <= #{>= c}; equal candidates agree. Four
        // threads per candidate each count a quarter of the others.
        static_assert(kSelThreads == 4 * kRankMax, "four counters per candidate");
        __syncthreads();
        const int ci = tid % kRankMax, q = tid / kRankMax;
        int gt = 0, ge = 0;
        if (ci < nbin) {
          const uint32_t c = s_cand[ci];
          for (int j = q; j < nbin; j += 4) {
            const uint32_t o = s_cand[j];
            gt += o > c;
            ge += o >= c;
          }
        }
        int2* part = reinterpret_cast<int2*>(s_hist);  // free: no histogram follows
        part[q * kRankMax + ci] = make_int2(gt, ge);
        __syncthreads();
        if (q == 0 && ci < nbin) {
#pragma unroll
          for (int r = 1; r < 4; ++r) {
            const int2 v = part[r * kRankMax + ci];
            gt += v.x;
            ge += v.y;
          }
          if (gt < k && k <= ge) {
            s_res[0] = s_cand[ci];
            s_res[1] = (unsigned)gt;
          }
        }
        __syncthreads();
        prefix = s_res[0];
        k -= (int)s_res[1];
        ranked = true;
      }
    }
    __syncthreads();
  }
  const uint32_t thr = prefix;  // the C-th largest key; take k keys equal to it

  // Word w of the bitmaps covers keys [32w, 32w + 32): bit b set if key 32w + b is
  // above (gt) or equal to (eq) the threshold. With a candidate list, only the
  // candidates' bits are left to set; otherwise one sweep of the row sets them all.
  if (collected) {
    for (int j = tid; j < n; j += kSelThreads) {
      const uint32_t key = s_cand[j];
      const int i = s_cidx[j];
      if (key > thr) atomicOr(&s_gtw[i >> 5], 1u << (i & 31));
      else if (key == thr) atomicOr(&s_eqw[i >> 5], 1u << (i & 31));
    }
  } else {
    for (int w = warp; w < nw; w += kSelWarps) {
      const int i = 32 * w + lane;
      const uint32_t key = i < S ? keys[i] : 0u;
      const unsigned gw = __ballot_sync(0xffffffffu, i < S && key > thr);
      const unsigned qw = __ballot_sync(0xffffffffu, i < S && key == thr);
      if (lane == 0) {
        s_gtw[w] = gw;
        s_eqw[w] = qw;
      }
    }
  }
  __syncthreads();

  // Thread tid owns words [w0, w1); a scan of their popcounts places every chosen key.
  const int wpt = (nw + kSelThreads - 1) / kSelThreads;
  const int w0 = min(nw, tid * wpt), w1 = min(nw, w0 + wpt);
  int n_gt = 0, n_eq = 0;
  for (int w = w0; w < w1; ++w) {
    n_gt += __popc(s_gtw[w]);
    n_eq += __popc(s_eqw[w]);
  }
  int gt_run, eq_run, tot_gt, tot_eq;
  block_scan2(n_gt, n_eq, &gt_run, &eq_run, &tot_gt, &tot_eq, s_scan);

  const int tok0 = g * S;
  // the bit of each word whose token starts a CSR block
  const int rb = (kBlockTok - tok0 % kBlockTok) % kBlockTok;
  int32_t* out_idx = idx + (int64_t)e * Ce + (int64_t)g * C;
  float* out_gate = gate + (int64_t)e * Ce + (int64_t)g * C;
  for (int w = w0; w < w1; ++w) {
    const uint32_t gw = s_gtw[w], qw = s_eqw[w];
    if (bnd != nullptr && 32 * w + rb < S) {
      const uint32_t m = (1u << rb) - 1u;
      const int before = gt_run + __popc(gw & m) + min(eq_run + __popc(qw & m), k);
      bnd[(int64_t)((tok0 + 32 * w + rb) / kBlockTok) * E + e] = g * C + before;
    }
    for (uint32_t bits = gw | qw; bits != 0u; bits &= bits - 1u) {
      const int b = __ffs(bits) - 1;
      const uint32_t m = (1u << b) - 1u;
      const int gt_before = gt_run + __popc(gw & m);
      const int eq_before = eq_run + __popc(qw & m);
      const int pos = gt_before + min(eq_before, k);
      if ((((gw >> b) & 1u) != 0u || eq_before < k) && pos < C) {
        out_idx[pos] = tok0 + 32 * w + b;
        out_gate[pos] = __uint_as_float(keys[32 * w + b]);
      }
    }
    gt_run += __popc(gw);
    eq_run += __popc(qw);
  }
  if (tid == 0) {
    if (bnd != nullptr && g == (int)gridDim.y - 1)
      bnd[((Tn + kBlockTok - 1) / kBlockTok) * E + e] = Ce;
    if (tot_gt + min(tot_eq, k) != C) atomicOr(err, kErrDeviceCheck);
  }
}

static_assert(kBlockTok == kCsrBlockTok, "the boundary table is per CSR block");

__global__ void __launch_bounds__(kCsrThreads) csr_kernel(const CsrArgs a) {
  pdl_launch_dependents();
  extern __shared__ __align__(16) uint8_t s_csr[];
  pdl_wait();
  csr_block(blockIdx.x, a, s_csr, threadIdx.x, []() { __syncthreads(); });
}

}  // namespace

size_t select_bound_entries(const Shape& s) {
  return ((size_t)ceil_div(s.T, kBlockTok) + 1) * (size_t)s.E;
}

cudaError_t launch_select(const float* scores_t, const Shape& s, int32_t* idx, float* gate,
                          int32_t* bnd, unsigned* err, int sm_count, cudaStream_t st) {
  if (s.S > kSelectMaxRow) return cudaErrorInvalidValue;
  const int cached = s.S <= kSelMaxCached;
  const size_t nw4 = (size_t)((ceil_div(s.S, 32) + 3) & ~3);
  const size_t smem = sizeof(uint32_t) * ((cached ? (size_t)((s.S + 3) & ~3) : 0) + 2 * nw4 +
                                          (size_t)kCandMax);
  dim3 grid((unsigned)s.E, (unsigned)s.n_seg);
  const bool two = (int64_t)s.E * s.n_seg > sm_count;
  return launch_kernel(two ? select_kernel<2> : select_kernel<1>, grid, dim3(kSelThreads), smem,
                       st, s.pdl, 1, scores_t,
                       (int64_t)s.T, s.S, s.C, s.Ce, s.E, cached, idx, gate, bnd, err);
}

cudaError_t launch_csr(const int32_t* idx, const int32_t* bnd, const Shape& s, bool shared,
                       int32_t* tok_ptr, int32_t* tok_ent, int32_t* ent_pos, float* gate,
                       nmoe_combine combine, float route_scale, bool direct, unsigned* err,
                       cudaStream_t st) {
  const CsrArgs a = csr_args(idx, bnd, s, shared, tok_ptr, tok_ent, ent_pos, gate, combine,
                             route_scale, direct, err);
  dim3 grid((unsigned)ceil_div(s.T, kBlockTok));
  return launch_kernel(csr_kernel, grid, dim3(kCsrThreads), csr_smem_bytes(s.E), st, s.pdl, 1,
                       a);
}

CsrArgs csr_args(const int32_t* idx, const int32_t* bnd, const Shape& s, bool shared,
                 int32_t* tok_ptr, int32_t* tok_ent, int32_t* ent_pos, float* gate,
                 nmoe_combine combine, float route_scale, bool direct, unsigned* err) {
  CsrArgs a;
  a.idx = idx; a.bnd = bnd; a.T = s.T; a.E = s.E; a.Ce = s.Ce; a.shared = shared ? 1 : 0;
  a.tok_ptr = tok_ptr; a.tok_ent = tok_ent; a.ent_pos = ent_pos; a.gate = gate;
  a.normalize = combine == NMOE_COMBINE_NORMALIZED ? 1 : 0;
  a.route_scale = route_scale; a.direct = direct ? 1 : 0; a.err = err;
  return a;
}

}  // namespace nmoe
