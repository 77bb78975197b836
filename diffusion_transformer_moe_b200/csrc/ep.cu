// Expert-parallel pieces: the row lists one rank owes another, row gather/scatter, and
// the combine of a token range.
//
// Every list is padded to a capacity the host knows in advance (a rank's experts own
// (e_end - e_begin) * Ce entries, so no list can be longer), with -1 rows that the copies
// skip: the exchange moves fixed-size buffers, and no count has to come back to the host
// before the next launch.
//
// With experts split into contiguous ranges, one per rank, every rank computes the same
// routing and token lists, runs the expert GEMMs for its own range (each row landing at
// its token-major position in Y), and the owner of a token range needs exactly the rows
// of its tokens that each other rank computed: ep_rows_kernel lists them, in ascending
// row order, from the token lists alone, so sender and receiver agree without exchanging
// counts. The rows travel packed (rows_copy_kernel gathers before the all-to-all and
// scatters after it), and the owner's combine of its range then equals one GPU's.
#include "nmoe_internal.cuh"

namespace nmoe {
namespace {

constexpr int kRowsThreads = 1024;

// One CTA: ordered compaction of the rows [tok_ptr[t_begin], tok_ptr[t_end]) whose entry
// e*Ce + slot has e in [e_begin, e_end), into rows[0 .. count); rows[count .. capacity)
// are set to -1 (padding the copies below skip). A list longer than `capacity` keeps its
// first `capacity` rows and sets the error word; *count is the full length either way.
__global__ void __launch_bounds__(kRowsThreads)
ep_rows_kernel(const int32_t* __restrict__ tok_ptr, const int32_t* __restrict__ tok_ent,
               int E, int Ce, int t_begin, int t_end, int e_begin, int e_end,
               int32_t* __restrict__ rows, int capacity, int32_t* __restrict__ count,
               unsigned* __restrict__ err) {
  __shared__ int s_warp[kRowsThreads / 32];
  __shared__ int s_base;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int r0 = tok_ptr[t_begin], r1 = tok_ptr[t_end];
  if (kDebugChecks && (r0 < 0 || r1 < r0 || r1 > E * Ce)) {
    // debug build: a span outside the token lists is reported and nothing is listed
    if (tid == 0) atomicOr(err, kErrDeviceCheck);
    r0 = r1 = 0;
  }
  if (tid == 0) s_base = 0;
  __syncthreads();
  for (int c0 = r0; c0 < r1; c0 += kRowsThreads) {
    const int r = c0 + tid;
    bool keep = false;
    if (r < r1) {
      const int v = tok_ent[r];
      keep = v >= 0 && v < E * Ce && v / Ce >= e_begin && v / Ce < e_end;
    }
    const unsigned b = __ballot_sync(0xffffffffu, keep);
    if (lane == 0) s_warp[warp] = __popc(b);
    __syncthreads();
    int before = s_base, total = 0;
    for (int w = 0; w < kRowsThreads / 32; ++w) {
      if (w < warp) before += s_warp[w];
      total += s_warp[w];
    }
    const int at = before + __popc(b & ((1u << lane) - 1u));
    if (keep && at < capacity) rows[at] = r;
    __syncthreads();
    if (tid == 0) s_base += total;
    __syncthreads();
  }
  const int n = s_base;
  for (int i = n + tid; i < capacity; i += kRowsThreads) rows[i] = -1;
  if (tid == 0) {
    *count = n;
    if (n > capacity) atomicOr(err, kErrDeviceCheck);
  }
}

// dst[i] = src[rows[i]] (GATHER; a zero row where rows[i] < 0) or dst[rows[i]] = src[i]
// (nothing where rows[i] < 0), rows of `chunks` 16-byte units. One warp per row: lane l
// moves the units l, l + 32, ..., issuing up to kCopyUnroll loads before its stores, so a
// 4 KB row (d = 2048 bf16) is one round of eight 16-byte loads per lane and an SM keeps
// ~128 KB of reads in flight at four CTAs.
constexpr int kCopyThreads = 256;
constexpr int kCopyUnroll = 8;

template <bool GATHER>
__global__ void __launch_bounds__(kCopyThreads)
rows_copy_kernel(const uint4* __restrict__ src, const int32_t* __restrict__ rows, int64_t n,
                 int chunks, uint4* __restrict__ dst) {
  const int lane = threadIdx.x & 31;
  const int64_t wpc = kCopyThreads / 32;
  const int64_t nwarps = (int64_t)gridDim.x * wpc;
  for (int64_t i = blockIdx.x * wpc + (threadIdx.x >> 5); i < n; i += nwarps) {
    const int64_t r = rows[i];
    if (!GATHER && r < 0) continue;
    const uint4* s = GATHER ? src + (r >= 0 ? r : 0) * chunks : src + i * chunks;
    uint4* d = GATHER ? dst + i * chunks : dst + r * chunks;
    const bool zero = GATHER && r < 0;
    for (int c0 = 0; c0 < chunks; c0 += 32 * kCopyUnroll) {
      uint4 v[kCopyUnroll];
#pragma unroll
      for (int u = 0; u < kCopyUnroll; ++u) {
        const int c = c0 + 32 * u + lane;
        v[u] = (c < chunks && !zero) ? s[c] : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int u = 0; u < kCopyUnroll; ++u) {
        const int c = c0 + 32 * u + lane;
        if (c < chunks) d[c] = v[u];
      }
    }
  }
}

}  // namespace

cudaError_t launch_ep_rows(const int32_t* tok_ptr, const int32_t* tok_ent, int E, int Ce,
                           int t_begin, int t_end, int e_begin, int e_end, int32_t* rows,
                           int capacity, int32_t* count, unsigned* err, cudaStream_t st) {
  ep_rows_kernel<<<1, kRowsThreads, 0, st>>>(tok_ptr, tok_ent, E, Ce, t_begin, t_end, e_begin,
                                              e_end, rows, capacity, count, err);
  return cudaGetLastError();
}

cudaError_t launch_rows_copy(const void* src, const int32_t* rows, int64_t n, int64_t row_bytes,
                             void* dst, bool gather, int sm_count, cudaStream_t st) {
  if (n == 0) return cudaSuccess;
  const int chunks = (int)(row_bytes / 16);
  constexpr int64_t kRowsPerCta = kCopyThreads / 32;
  int64_t grid = (n + kRowsPerCta - 1) / kRowsPerCta;
  if (grid > 4 * (int64_t)sm_count) grid = 4 * (int64_t)sm_count;
  if (gather)
    rows_copy_kernel<true><<<(unsigned)grid, kCopyThreads, 0, st>>>(
        static_cast<const uint4*>(src), rows, n, chunks, static_cast<uint4*>(dst));
  else
    rows_copy_kernel<false><<<(unsigned)grid, kCopyThreads, 0, st>>>(
        static_cast<const uint4*>(src), rows, n, chunks, static_cast<uint4*>(dst));
  return cudaGetLastError();
}

}  // namespace nmoe
