// One block of the token -> (expert, slot) lists, for kCsrBlockTok consecutive tokens,
// built by kCsrThreads threads. Used by the CSR kernel (one block per CTA) and by the
// gate/up GEMM's epilogue warps, which build the lists while their first tile's
// accumulator is still being filled.
//
// For every expert, the selection's boundary table gives the slot range [lo, lo + cnt)
// of its entries inside the block, and the sum of the lo's is the block's offset in the
// token-major order (without the table: binary searches of each expert's ascending
// token list). Entries are scattered into a (token x expert) slot map in shared memory,
// one per thread, and each token's list is written in ascending expert order, with each
// entry's token-major position (ent_pos), where the down projection writes its row.
// With a shared expert every token's span starts with one more entry, its shared row.
// NORMALIZED combine weights are rewritten in place from the fp32 sum of the token's
// gates in ascending expert order. With `direct`, the one entry of a token that a single
// expert chose gets ent_pos = -(t + 1): the down projection writes that row straight to
// the output (a sum of one term is that term, rounded once), and the combine skips it.
#pragma once

#include "nmoe_internal.cuh"

namespace nmoe {

constexpr int kCsrBlockTok = 32;   // tokens per block (one warp lane per token)
constexpr int kCsrThreads = 256;   // threads per block (one per expert: E <= 256)
constexpr int kCsrWarps = kCsrThreads / 32;

struct CsrArgs {
  const int32_t* idx;   // [E, Ce] chosen tokens, ascending per expert
  const int32_t* bnd;   // boundary table [ceil(T/32) + 1, E], or NULL (search idx)
  int T, E, Ce;
  int shared;           // nonzero: one shared-expert entry first in every token's span
  int32_t* tok_ptr;     // [T + 1]
  int32_t* tok_ent;     // [E*Ce (+ T)]
  int32_t* ent_pos;     // [E*Ce] or NULL
  float* gate;          // [E, Ce]
  int normalize;
  float route_scale;
  int direct;           // single-entry tokens: ent_pos = -(t + 1), written by gemm2
  unsigned* err;
};

struct CsrShared {
  int lo[256], beg[256];
  int wlo[kCsrWarps], wcnt[kCsrWarps];
  int cnt[kCsrBlockTok], off[kCsrBlockTok];
};

// shared memory a block needs: CsrShared, then the [kCsrBlockTok][E] int slot map
__host__ __device__ constexpr size_t csr_smem_bytes(int E) {
  return ((sizeof(CsrShared) + 15) / 16) * 16 + sizeof(int) * kCsrBlockTok * (size_t)E;
}

namespace csr_detail {

__device__ __forceinline__ unsigned lanemask_lt() {
  unsigned m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

__device__ __forceinline__ int lower_bound_i32(const int32_t* a, int n, int v) {
  int lo = 0, hi = n;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (a[mid] < v) lo = mid + 1; else hi = mid;
  }
  return lo;
}

}  // namespace csr_detail

// Builds block `blk`. tid in [0, kCsrThreads); sync() is a barrier over exactly those
// threads. `smem` holds csr_smem_bytes(E) bytes; it is free again when this returns.
template <typename Sync>
__device__ __forceinline__ void csr_block(int blk, const CsrArgs& a, uint8_t* smem, int tid,
                                          Sync sync) {
  using namespace csr_detail;
  CsrShared& sh = *reinterpret_cast<CsrShared*>(smem);
  int* s_slot = reinterpret_cast<int*>(smem + ((sizeof(CsrShared) + 15) / 16) * 16);
  const int lane = tid & 31, warp = tid >> 5;
  const int E = a.E, Ce = a.Ce;
  const int t0 = blk * kCsrBlockTok;
  const int t1 = min(a.T, t0 + kCsrBlockTok);

  for (int i = tid; i < kCsrBlockTok * E; i += kCsrThreads) s_slot[i] = -1;
  if (tid < kCsrBlockTok) sh.cnt[tid] = 0;

  // slot range [lo, lo + cnt) of expert `tid` inside the block
  int lo = 0, cnt = 0;
  if (tid < E) {
    if (a.bnd != nullptr) {
      lo = a.bnd[(int64_t)blk * E + tid];
      cnt = a.bnd[(int64_t)(blk + 1) * E + tid] - lo;
    } else {
      const int32_t* row = a.idx + (int64_t)tid * Ce;
      lo = lower_bound_i32(row, Ce, t0);
      cnt = lower_bound_i32(row, Ce, t1) - lo;
    }
    if (lo < 0 || cnt < 0 || lo + cnt > Ce) {  // not a table the selection wrote
      atomicOr(a.err, kErrDeviceCheck);
      lo = 0;
      cnt = 0;
    }
    sh.lo[tid] = lo;
  }
  // exclusive scan of cnt over the experts; sum of lo = entries before the block
  int inc = cnt, part = lo;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += v;
    part += __shfl_xor_sync(0xffffffffu, part, o);
  }
  if (lane == 31) sh.wcnt[warp] = inc;
  if (lane == 0) sh.wlo[warp] = part;
  sync();
  int base = 0, total = 0, before = 0;
#pragma unroll
  for (int w = 0; w < kCsrWarps; ++w) {
    base += sh.wlo[w];
    total += sh.wcnt[w];
    if (w < warp) before += sh.wcnt[w];
  }
  if (tid < E) sh.beg[tid] = before + inc - cnt;
  base += a.shared * t0;  // with a shared expert, one more entry for every earlier token
  sync();

  // scatter the block's entries into the (token, expert) slot map, one per thread
  for (int j = tid; j < total; j += kCsrThreads) {
    int lo_e = 0, hi_e = E - 1;  // last expert whose first flat entry is <= j
    while (lo_e < hi_e) {
      const int mid = (lo_e + hi_e + 1) >> 1;
      if (sh.beg[mid] <= j) lo_e = mid; else hi_e = mid - 1;
    }
    const int sl = sh.lo[lo_e] + (j - sh.beg[lo_e]);
    const int t = a.idx[(int64_t)lo_e * Ce + sl];
    if (t >= t0 && t < t1) {
      s_slot[(t - t0) * E + lo_e] = sl;
      atomicAdd(&sh.cnt[t - t0], 1);
    } else {
      atomicOr(a.err, kErrDeviceCheck);
    }
  }
  sync();

  // per-token offsets (one warp: kCsrBlockTok == 32)
  if (warp == 0) {
    const int c = sh.cnt[lane];
    int incl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    sh.off[lane] = incl - c + a.shared * lane;   // start of the token's span
    if (t0 + lane < t1) a.tok_ptr[t0 + lane] = base + sh.off[lane];
    if (t0 + lane == a.T - 1) a.tok_ptr[a.T] = base + incl + a.shared * (lane + 1);
  }
  sync();

  // entries of each token in ascending expert order: one warp per token
  const unsigned lt = lanemask_lt();
  for (int r = warp; r < t1 - t0; r += kCsrWarps) {
    int out = base + sh.off[r];
    if (a.shared) {  // the shared-expert row comes first
      if (lane == 0) a.tok_ent[out] = E * Ce + t0 + r;
      ++out;
    }
    const int* srow = s_slot + r * E;
    float tot = 0.f;  // the token's gates summed in ascending expert order, fp32
    for (int e0 = 0; e0 < E; e0 += 32) {
      const int e = e0 + lane;
      const int sl = e < E ? srow[e] : -1;
      const unsigned m = __ballot_sync(0xffffffffu, sl >= 0);
      if (sl >= 0) {
        const int at = out + __popc(m & lt);
        a.tok_ent[at] = e * Ce + sl;
        if (a.ent_pos != nullptr)
          a.ent_pos[e * Ce + sl] = (a.direct && sh.cnt[r] == 1) ? -(t0 + r + 1) : at;
      }
      if (a.normalize) {
        const float v = sl >= 0 ? a.gate[(int64_t)e * Ce + sl] : 0.f;
        for (unsigned mm = m; mm != 0u; mm &= mm - 1u)
          tot += __shfl_sync(0xffffffffu, v, __ffs(mm) - 1);
      }
      out += __popc(m);
    }
    if (a.normalize) {
      // every entry belongs to one token, so this lane alone reads and rewrites it
      for (int e0 = 0; e0 < E; e0 += 32) {
        const int e = e0 + lane;
        const int sl = e < E ? srow[e] : -1;
        if (sl >= 0) {
          float* gp = a.gate + (int64_t)e * Ce + sl;
          *gp = a.route_scale * (*gp / tot);
        }
      }
    }
  }
  sync();  // the slot map and offsets are read before anyone reuses the memory
}

}  // namespace nmoe
