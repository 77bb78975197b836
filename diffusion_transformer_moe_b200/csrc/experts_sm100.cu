// Grouped SwiGLU expert GEMMs on the 5th-generation tensor cores.
//
// The packed SwiGLU experts of the NucleusMoE-Image walkthrough (section 6: fused
// gate/up projection of shape (experts, hidden, 2 * moe_intermediate_dim), then the down
// projection; "only two grouped matmuls at runtime"; the grouped path wants each
// expert's tokens as one contiguous block). Expert choice makes every block exactly
// Ce = n_segments * C rows, so both GEMMs have static shapes:
//
//   gemm1: H[e, s, :] = silu(x[idx[e,s]] W1_e) * (x[idx[e,s]] W3_e)
//   gemm2: Y[ent_pos[e*Ce + s], :] = gate[e, s] * (H[e, s, :] W2_e)
//
// (Y rows land in token-major order, so the combine reads each token's rows
// contiguously.)
//
// Instead of permuting tokens into per-expert blocks, gemm1 gathers the 128 rows of its
// A tile straight from x. Two ways are built: four producer warps issuing 16-byte
// cp.async copies into the 128-byte-swizzled tile (default), or TMA tile::gather4 (32
// copies of 4 rows per k-block). On B200 the gather4 form caps gemm1 at about half the
// HBM rate (measured: 201 us against 109 us for the same bytes as plain tiles at
// T = 8192, d = 2048, E = 64, F = 1024), so cp.async is the default.
//
// Intermediate precision. With SPLIT (the default), H is stored as a pair of bf16
// arrays hi = bf16(h), lo = bf16(h - hi) (about 16 significant bits), gemm2 runs both
// halves against the same W2 tile into one fp32 accumulator, and Y is stored in fp32.
// Without SPLIT, H and Y are single bf16 arrays (the usual bf16 MoE numerics), which
// moves ~10% fewer bytes but lets large-magnitude tokens drift by ~0.1-0.2 absolute.
//
// One persistent CTA per SM walks tiles (expert, 128-row block, N block) in a static
// round-robin. Warp roles: warp 0 issues the TMA copies (weights, and A unless cp.async
// gathers it), warp 1 allocates TMEM and one of its threads issues tcgen05.mma into a
// double-buffered accumulator (2 x 256 fp32 columns), the cp.async warps (gemm1) fill
// the A tiles, and eight epilogue warps (two per TMEM lane quarter) drain a finished
// accumulator with tcgen05.ld while the next tile's MMAs run. Tile: M = 128 rows,
// K = 64 per stage, N = 256 accumulator columns (gemm1: 128 gate + 128 up columns of F;
// gemm2: 256 columns of d). A is K-major, B (the weights, [E, K, N] with N contiguous)
// is MN-major; both use the 128-byte swizzle. Every wait is bounded; a wait that runs
// out sets the device error word and the kernel drains its copies and MMAs, frees TMEM
// and returns.
//
// Larger experts take two variants:
// * 1024 or more rows per expert: each gate/up work item covers two 128-row blocks that
//   share every weight tile (MT = 2). Both accumulators then belong to one item, so they
//   are not double-buffered across items.
// * 256 or more rows per expert: the down projection runs on 2-CTA clusters
//   (pair_gemm2_kernel). One tcgen05.mma.cta_group::2 covers M = 256 rows, and each CTA
//   stages its own 128 H rows and half of the W2 tile.
// Both down GEMMs issue griddepcontrol.launch_dependents only after their own wait, so the
// combine after them may read the token lists early.
#include <cudaTypedefs.h>

#include <mutex>
#include <utility>
#include <vector>

#include "csr_block.cuh"
#include "experts_sm100.cuh"
#include "sm100_ptx.cuh"

namespace nmoe {
namespace {

using namespace ptx;

constexpr int kBM = 128;
constexpr int kBK = 64;
constexpr int kABytes = kBM * kBK * 2;          // 16 KB per A tile
constexpr int kBBoxBytes = 64 * kBK * 2;        // 8 KB: 64 N x 64 K
constexpr int kBBytes = 4 * kBBoxBytes;         // 32 KB: N = 256
constexpr int kAccCols = 256;
constexpr int kTmemCols = 2 * kAccCols;
constexpr uint64_t kDrainNs = 20000000ull;      // 20 ms per drain wait after an abort

enum { kGemm1 = 0, kGemm2 = 1 };
enum { kGatherLsu = 0, kGatherTma4 = 1 };       // how gemm1 fetches its token rows

// MT: 128-row blocks of one expert per work item (2 only for gemm1 with the cp.async
// gather): each k-block's weight tile then feeds two MMAs, one per row block, into the two
// TMEM accumulators, so the ring moves a third fewer bytes per output; the accumulators
// are no longer double-buffered across items.
template <int MODE, bool SPLIT, int GATHER, int MT = 1>
struct Cfg {
  static_assert(MT == 1 || (MT == 2 && MODE == kGemm1 && GATHER == kGatherLsu),
                "two row blocks per item only for the cp.async-gathered gate/up GEMM");
  static constexpr bool kLsuA = MODE == kGemm1 && GATHER == kGatherLsu;
  static constexpr int kATiles = (MODE == kGemm2 && SPLIT) ? 2 : 1;  // H hi and lo
  static constexpr int kAStageBytes = (MT == 2 ? 2 : kATiles) * kABytes;
  static constexpr int kStageBytes = kAStageBytes + kBBytes;
  static constexpr int kStages = MT == 2 ? 3 : ((MODE == kGemm2 && SPLIT) ? 3 : 4);
  static constexpr size_t kRingBytes = (size_t)kStages * kStageBytes;
  static constexpr int kAWarps = kLsuA ? 4 : 0;          // cp.async gather warps
  static constexpr int kEpiWarps = 8;                    // two per TMEM lane quarter
  static constexpr int kEpiWarp0 = 2 + kAWarps;
  static constexpr int kThreads = 32 * (2 + kAWarps + kEpiWarps);
  static constexpr int kFullCount = 1 + 32 * kAWarps;    // TMA arrive + one per gather thread
  // staging block per epilogue warp: gemm2, 32 rows x 128 bytes of Y (32 fp32 with SPLIT,
  // else 64 bf16); gemm1, 32 rows x 32 bf16 of H (and as much again for H lo)
  static constexpr int kEpiStage =
      MODE == kGemm2 ? 32 * 128 : (SPLIT ? 2 * 32 * 64 : 32 * 64);
  static constexpr size_t kSmem = kRingBytes + kEpiWarps * kEpiStage + 1024;
  static_assert(kSmem <= 232448, "dynamic shared memory beyond the 227 KB a CTA may use");
};

struct Params {
  int Ce;          // rows per expert
  int K;           // reduction length (d for gemm1, F for gemm2)
  int N;           // output row length (F for gemm1, d for gemm2)
  int tiles_m, tiles_n, num_tiles;
  // Work items: tiles [0, num_full) whole, then every remaining tile as two items, each
  // half of its N range (so a last, partial wave of tiles runs on twice the SMs).
  int num_full, num_items;
  const int32_t* idx;    // gemm1: chosen tokens [E, Ce]
  const float* gate;     // gemm2: combine weights [E, Ce]
  const int32_t* ent_pos;  // gemm2: Y row of entry e*Ce + s (token-major order)
  void* out;             // gemm1: H (hi) [E*Ce, F] bf16; gemm2: Y [E*Ce, d] (fp32 if SPLIT)
  void* out_lo;          // gemm1 with SPLIT: H lo [E*Ce, F] bf16
  // gemm1: csr_blocks > 0 builds the token lists' blocks in the epilogue warps before
  // the first tile's accumulator is ready (their staging memory is free until then)
  CsrArgs csr;
  int csr_blocks;
  unsigned* err;
  uint64_t wait_ns;      // budget of each pipeline wait
  int rows_x;            // gemm1: rows of x (debug checks of the gathered indices)
  int64_t rows_y;        // gemm2: rows of Y (debug checks of ent_pos)
  // gemm2: a row whose position is -(t + 1) is token t's only entry; it goes straight to
  // row t of out_direct (the layer output, fp32 if out_direct_f32, else bf16), rounded
  // once, instead of to Y
  void* out_direct;
  int out_direct_f32;
};

// Debug build: a gathered token index must lie in x; otherwise the error word is set and
// row 0 is read instead (nothing outside x is touched).
__device__ __forceinline__ int checked_row(int t, const Params& p) {
  if (kDebugChecks && (t < 0 || t >= p.rows_x)) {
    atomicOr(p.err, kErrDeviceCheck);
    return 0;
  }
  return t;
}

// silu(g) = g * sigmoid(g) = g / (1 + e^-g) with the fast exp and the fast divide
// (each within a few ulp of fp32, far below the hi/lo split's 16 bits). g is a finite
// GEMM output; very negative g gives 0 and g -> +inf gives g.
__device__ __forceinline__ float silu_f32(float g) {
  return __fdividef(g, 1.f + __expf(-g));
}

// Work item -> tile: expert, first row, first column of its N range, and whether it
// covers half of the tile's N range. n_per_tile: gemm1 128 columns of F (gate and up
// each), gemm2 256 columns of d.
struct Tile {
  int e, m0, n0;
  bool half;
};
__device__ __forceinline__ Tile tile_of(int item, const Params& p, int n_per_tile) {
  int t = item, part = -1;
  if (item >= p.num_full) {
    t = p.num_full + ((item - p.num_full) >> 1);
    part = (item - p.num_full) & 1;
  }
  Tile r;
  r.e = t / (p.tiles_m * p.tiles_n);
  const int rem = t % (p.tiles_m * p.tiles_n);
  r.m0 = (rem / p.tiles_n) * kBM;
  r.n0 = (rem % p.tiles_n) * n_per_tile;
  r.half = part >= 0;
  if (r.half) r.n0 += part * (n_per_tile / 2);
  return r;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

// lo half of the (hi, lo) split: bf16(v - bf16(v)), for two values
__device__ __forceinline__ uint32_t pack_lo_bf16x2(float a, float b, uint32_t hi) {
  __nv_bfloat162 h = *reinterpret_cast<__nv_bfloat162*>(&hi);
  float2 f = __bfloat1622float2(h);
  return pack_bf16x2(a - f.x, b - f.y);
}

template <int MODE, bool SPLIT, int GATHER, int MT>
__global__ void __launch_bounds__(Cfg<MODE, SPLIT, GATHER, MT>::kThreads, 1)
grouped_gemm_kernel(const __grid_constant__ CUtensorMap map_a,
                    const __grid_constant__ CUtensorMap map_a2,
                    const __grid_constant__ CUtensorMap map_b0,
                    const __grid_constant__ CUtensorMap map_b1, const __nv_bfloat16* x,
                    const Params p) {
  using C = Cfg<MODE, SPLIT, GATHER, MT>;
  constexpr int kStages = C::kStages;
  if (MODE != kGemm2) pdl_launch_dependents();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ __align__(8) uint64_t full_bar[kStages], empty_bar[kStages];
  __shared__ __align__(8) uint64_t tfull_bar[2], tempty_bar[2], drain_bar;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nk = (p.K + kBK - 1) / kBK;
  constexpr int n_per_tile = MODE == kGemm1 ? 128 : 256;
  // stage s: A tile(s) at s * kStageBytes, B boxes after them
  auto a_tile = [&](int s, int which) { return smem + s * C::kStageBytes + which * kABytes; };
  auto b_tile = [&](int s) { return smem + s * C::kStageBytes + C::kAStageBytes; };
  uint8_t* const epi_smem = smem + C::kRingBytes;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&full_bar[i], C::kFullCount);
      mbar_init(&empty_bar[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull_bar[i], 1);
      mbar_init(&tempty_bar[i], C::kEpiWarps);
    }
    mbar_init(&drain_bar, 1);
    abort_flag = 0;
    fence_mbar_init();
    if (!C::kLsuA) prefetch_tensormap(&map_a);
    if (C::kATiles == 2) prefetch_tensormap(&map_a2);
    prefetch_tensormap(&map_b0);
    if (MODE == kGemm1) prefetch_tensormap(&map_b1);
  }
  if (warp == 1) tmem_alloc(&tmem_base_sh, kTmemCols);
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = tmem_base_sh;
  volatile int* abort_v = &abort_flag;
  pdl_wait();  // the previous kernel's outputs (idx, x or H, gate) are complete
  // the down GEMM lets the next kernel start only now: everything before it is complete
  if (MODE == kGemm2) pdl_launch_dependents();

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    // Every weight tile is read exactly once per call: its copies are marked evict-first,
    // so that the weight stream (hundreds of MB) does not push out of L2 the token rows,
    // H and Y that this kernel and the next one read again.
    const uint64_t wpol = l2_policy_evict_first();
    int stage = 0;
    uint32_t phase = 0;
    uint32_t issued_mask = 0, issued_par = 0;  // per stage: ever issued / parity of last issue
    for (int item = blockIdx.x; item < p.num_items; item += gridDim.x) {
      const Tile tl = tile_of(item, p, n_per_tile);
      const int e = tl.e, m0 = tl.m0, n0 = tl.n0;
      const int nbox = tl.half ? 2 : 4;  // 64-column boxes of B
      const uint32_t b_bytes = (uint32_t)(nbox * kBBoxBytes);
      int r0 = 0, r1 = 0, r2 = 0, r3 = 0;
      if (MODE == kGemm1 && !C::kLsuA) {
        const int32_t* ir = p.idx + (int64_t)e * p.Ce;  // NULL idx: identity (shared)
        const int s = m0 + 4 * lane;
        r0 = checked_row(s + 0 < p.Ce ? (p.idx ? ir[s + 0] : s + 0) : 0, p);
        r1 = checked_row(s + 1 < p.Ce ? (p.idx ? ir[s + 1] : s + 1) : 0, p);
        r2 = checked_row(s + 2 < p.Ce ? (p.idx ? ir[s + 2] : s + 2) : 0, p);
        r3 = checked_row(s + 3 < p.Ce ? (p.idx ? ir[s + 3] : s + 3) : 0, p);
      }
      bool ok = true;
      for (int kb = 0; kb < nk; ++kb) {
        int w = 1;
        if (lane == 0) w = mbar_wait(&empty_bar[stage], phase ^ 1, abort_v, p.wait_ns);
        ok = __shfl_sync(0xffffffffu, w, 0) != 0;
        if (!ok) break;
        if (lane == 0)
          mbar_arrive_expect_tx(&full_bar[stage],
                                C::kLsuA ? b_bytes : C::kAStageBytes + b_bytes);
        __syncwarp();
        const int k0 = kb * kBK;
        uint8_t* b_dst = b_tile(stage);
        if (MODE == kGemm1) {
          if (!C::kLsuA)
            tma_gather4(a_tile(stage, 0) + lane * 512, &map_a, &full_bar[stage], k0, r0, r1,
                        r2, r3);
          // boxes: gate columns, then up columns (two of each, or one of each for a half)
          if (lane < nbox) {
            const int per = nbox / 2;
            const CUtensorMap* mb = lane < per ? &map_b0 : &map_b1;
            tma_load_3d_hint(b_dst + lane * kBBoxBytes, mb, &full_bar[stage],
                             n0 + 64 * (lane % per), k0, e, wpol);
          }
        } else {
          if (lane == 0)
            tma_load_2d(a_tile(stage, 0), &map_a, &full_bar[stage], k0, e * p.Ce + m0);
          if (C::kATiles == 2 && lane == 1)
            tma_load_2d(a_tile(stage, 1), &map_a2, &full_bar[stage], k0, e * p.Ce + m0);
          if (lane < nbox)
            tma_load_3d_hint(b_dst + lane * kBBoxBytes, &map_b0, &full_bar[stage],
                             n0 + 64 * lane, k0, e, wpol);
        }
        issued_mask |= 1u << stage;
        issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
        if (++stage == kStages) { stage = 0; phase ^= 1; }
      }
      if (!ok) break;
    }
    if (*abort_v && lane == 0) {
      // let every copy this CTA issued land before the CTA can exit
      int dummy = 0;
      for (int s = 0; s < kStages; ++s)
        if (issued_mask & (1u << s))
          mbar_wait(&full_bar[s], (issued_par >> s) & 1u, &dummy, kDrainNs);
    }
    __syncwarp();
  } else if (C::kLsuA && warp >= 2 && warp < 2 + C::kAWarps) {
    // ---------------- cp.async gather of the token rows (gemm1) ----------------
    // Warp pw owns tile rows [32 pw, 32 pw + 32); per instruction each group of eight
    // lanes copies one row's 128-byte k-slice (eight 16-byte pieces), and the piece c of
    // row r lands at r * 128 + ((c ^ (r % 8)) * 16): the 128-byte swizzle TMA would apply.
    // Each thread's copies arrive on the stage's full barrier by themselves when they
    // land (cp.async.mbarrier.arrive.noinc), so the warp never waits for its own data.
    const int pw = warp - 2;
    const int sub = lane >> 3, c = lane & 7;
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    for (int item = blockIdx.x; item < p.num_items && ok; item += gridDim.x) {
      const Tile tl = tile_of(item, p, n_per_tile);
      const int e = tl.e, m0 = MT * tl.m0;  // tile_of counts blocks of kBM rows
      const __nv_bfloat16* src[MT][8];
      uint32_t dst_off[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int r = pw * 32 + i * 4 + sub;
        dst_off[i] = r * 128 + ((c ^ (r & 7)) << 4);
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
          const int s = m0 + mt * kBM + r;
          const int t =
              checked_row(s < p.Ce ? (p.idx ? p.idx[(int64_t)e * p.Ce + s] : s) : 0, p);
          src[mt][i] = x + (int64_t)t * p.K + c * 8;
        }
      }
      for (int kb = 0; kb < nk; ++kb) {
        int w = 1;
        if (lane == 0) w = mbar_wait(&empty_bar[stage], phase ^ 1, abort_v, p.wait_ns);
        if (__shfl_sync(0xffffffffu, w, 0) == 0) { ok = false; break; }
        const int k0 = kb * kBK;
        if (k0 + c * 8 < p.K) {
#pragma unroll
          for (int mt = 0; mt < MT; ++mt)
#pragma unroll
            for (int i = 0; i < 8; ++i)
              cp_async16(a_tile(stage, mt) + dst_off[i], src[mt][i] + k0);
          cp_async_arrive_noinc(&full_bar[stage]);
        } else {  // beyond d: zeros, as the TMA path's out-of-bounds fill
#pragma unroll
          for (int mt = 0; mt < MT; ++mt)
#pragma unroll
            for (int i = 0; i < 8; ++i)
              *reinterpret_cast<uint4*>(a_tile(stage, mt) + dst_off[i]) = make_uint4(0, 0, 0, 0);
          fence_proxy_async_smem();
          mbar_arrive(&full_bar[stage]);
        }
        if (++stage == kStages) { stage = 0; phase ^= 1; }
      }
    }
    cp_async_wait<0>();  // no copy may still be writing when the CTA exits
  } else if (warp == 1) {
    // ---------------- MMA issuer (one thread) ----------------
    if (lane == 0) {
      constexpr uint32_t idesc_full = idesc_bf16(kBM, 256, 1);
      constexpr uint32_t idesc_half = idesc_bf16(kBM, 128, 1);
      // MT == 1: items alternate between the two accumulators; MT == 2: every item uses
      // both (accumulator mt holds row block mt) and their barriers flip once per item
      int stage = 0, acc = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool ok = true;
      for (int item = blockIdx.x; item < p.num_items && ok; item += gridDim.x) {
        const uint32_t idesc = tile_of(item, p, n_per_tile).half ? idesc_half : idesc_full;
        for (int kb = 0; kb < nk; ++kb) {
          if (!(ok = mbar_wait(&full_bar[stage], phase, abort_v, p.wait_ns))) break;
          tc_fence_after();
          if (C::kLsuA) fence_proxy_async_smem();  // cp.async writes -> tensor-core reads
          const uint32_t b_addr = smem_u32(b_tile(stage));
#pragma unroll
          for (int mt = 0; mt < MT; ++mt) {
            const int a = MT == 1 ? acc : mt;
            if (kb == 0) {
              // the accumulator's previous contents have been read out
              if (!(ok = mbar_wait(&tempty_bar[a], acc_phase ^ 1, abort_v, p.wait_ns))) break;
              tc_fence_after();
            }
            const uint32_t d_tmem = tmem_base + a * kAccCols;
#pragma unroll
            for (int kk = 0; kk < kBK / 16; ++kk) {
              const uint64_t bd = sdesc_sw128(b_addr + kk * 2048, kBBoxBytes, 1024);
#pragma unroll
              for (int h = 0; h < (MT == 2 ? 1 : C::kATiles); ++h) {
                const uint64_t ad =
                    sdesc_sw128(smem_u32(a_tile(stage, MT == 2 ? mt : h)) + kk * 32, 16, 1024);
                mma_bf16(d_tmem, ad, bd, idesc, (kb | kk | h) != 0);
              }
            }
          }
          if (!ok) break;
          mma_commit(&empty_bar[stage]);
          if (++stage == kStages) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) mma_commit(&tfull_bar[MT == 1 ? acc : mt]);
        if (MT == 2) {
          acc_phase ^= 1;
        } else if (++acc == 2) {
          acc = 0;
          acc_phase ^= 1;
        }
      }
      // every MMA issued above has completed once drain_bar flips
      mma_commit(&drain_bar);
      int dummy = 0;
      mbar_wait(&drain_bar, 0, &dummy, kDrainNs);
    }
    __syncwarp();  // the warp reconverges before the block barrier and the TMEM release
  } else if (warp >= C::kEpiWarp0) {
    // ---------------- epilogue: eight warps, two per TMEM lane quarter ----------------
    if (MODE == kGemm1 && p.csr_blocks > 0) {
      static_assert(C::kEpiWarps * 32 == kCsrThreads, "one CSR block per epilogue");
      uint8_t* cs = epi_smem;
      const int et = threadIdx.x - 32 * C::kEpiWarp0;
      for (int blk = blockIdx.x; blk < p.csr_blocks; blk += gridDim.x)
        csr_block(blk, p.csr, cs, et, []() { asm volatile("bar.sync 1, 256;" ::: "memory"); });
    }
    const int q = warp & 3;                         // TMEM lane quarter this warp may access
    const int half = (warp - C::kEpiWarp0) >> 2;    // which half of the columns
    const int row = q * 32 + lane;                  // accumulator row = tile row
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int item = blockIdx.x; item < p.num_items; item += gridDim.x) {
      const Tile tl = tile_of(item, p, n_per_tile);
      const int e = tl.e, n0 = tl.n0;
      // accumulator columns this warp drains: [c_lo, c_lo + c_n) (gemm1: gate columns,
      // the matching up columns sit `up` further on)
      const int acc_n = tl.half ? 128 : 256;
      const int up = acc_n / 2;
      const int c_n = MODE == kGemm1 ? acc_n / 4 : acc_n / 2;
      const int c_lo = half * c_n;
      bool stop = false;
#pragma unroll 1
      for (int mt = 0; mt < MT; ++mt) {  // the item's row blocks, one accumulator each
      const int a = MT == 1 ? acc : mt;
      const int m0 = MT * tl.m0 + mt * kBM;  // tile_of counts blocks of kBM rows
      int w = 1;
      if (lane == 0) w = mbar_wait(&tfull_bar[a], acc_phase, abort_v, p.wait_ns);
      if (__shfl_sync(0xffffffffu, w, 0) == 0) { stop = true; break; }
      tc_fence_after();
      const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + a * kAccCols;
      const int s = m0 + row;
      bool valid = s < p.Ce;
      const int64_t ent = (int64_t)e * p.Ce + (valid ? s : 0);
      int64_t pos = MODE == kGemm2 ? (int64_t)p.ent_pos[ent] : ent;
      if (kDebugChecks && MODE == kGemm2 && valid &&
          (pos >= p.rows_y ||
           (pos < 0 && (p.out_direct == nullptr || -pos - 1 >= (int64_t)p.rows_x)))) {
        // debug build: a row position outside Y (or the output) is reported and its
        // store skipped
        atomicOr(p.err, kErrDeviceCheck);
        valid = false;
        pos = 0;
      }
      const bool direct = MODE == kGemm2 && pos < 0;   // the token's only entry
      const int64_t orow = (direct ? -pos - 1 : pos) * p.N;
      if (MODE == kGemm1) {
        // staging blocks of this warp, 32 rows x 64 bytes each (H, then H lo): 16-byte
        // chunk c of row r at r * 64 + (c ^ ((r / 2) % 4)) * 16
        uint8_t* sh = epi_smem + (warp - C::kEpiWarp0) * C::kEpiStage;
        uint8_t* sl = sh + 32 * 64;
        const int sw = (lane >> 1) & 3;
#pragma unroll 1
        for (int j0 = c_lo; j0 < c_lo + c_n; j0 += 32) {
          uint32_t g[32], u[32];
          tmem_ld32(taddr + j0, g);
          tmem_ld32(taddr + up + j0, u);
          tmem_ld_wait();
          float h[32];
#pragma unroll
          for (int i = 0; i < 32; ++i)
            h[i] = silu_f32(__uint_as_float(g[i])) * __uint_as_float(u[i]);
          uint32_t ph[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) ph[i] = pack_bf16x2(h[2 * i], h[2 * i + 1]);
          // this row's 32 values into the staging blocks ...
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            const int off = lane * 64 + ((v ^ sw) << 4);
            *reinterpret_cast<uint4*>(sh + off) =
                make_uint4(ph[4 * v], ph[4 * v + 1], ph[4 * v + 2], ph[4 * v + 3]);
            if (SPLIT) {
              uint4 l;
              l.x = pack_lo_bf16x2(h[8 * v + 0], h[8 * v + 1], ph[4 * v + 0]);
              l.y = pack_lo_bf16x2(h[8 * v + 2], h[8 * v + 3], ph[4 * v + 1]);
              l.z = pack_lo_bf16x2(h[8 * v + 4], h[8 * v + 5], ph[4 * v + 2]);
              l.w = pack_lo_bf16x2(h[8 * v + 6], h[8 * v + 7], ph[4 * v + 3]);
              *reinterpret_cast<uint4*>(sl + off) = l;
            }
          }
          __syncwarp();
          // ... then out 8 rows per store, 64 contiguous bytes per row
          const int c = lane & 3;
          const int f = n0 + j0 + 8 * c;
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int r = 8 * i + (lane >> 2);
            const int64_t ro = __shfl_sync(0xffffffffu, orow, r);
            const int rv = __shfl_sync(0xffffffffu, (int)valid, r);
            const int off = r * 64 + ((c ^ ((r >> 1) & 3)) << 4);
            if (rv && f < p.N) {
              *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out) + ro + f) =
                  *reinterpret_cast<const uint4*>(sh + off);
              if (SPLIT)
                *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out_lo) + ro + f) =
                    *reinterpret_cast<const uint4*>(sl + off);
            }
          }
          __syncwarp();  // the blocks are read before the next chunk overwrites them
        }
      } else {
        const float gw = valid ? (p.gate ? p.gate[(int64_t)e * p.Ce + s] : 1.f) : 0.f;
        // staging block of this warp: 16-byte chunk c of row r at r * 128 + (c ^ (r % 8)) * 16
        float* sb = reinterpret_cast<float*>(epi_smem +
                                             (warp - C::kEpiWarp0) * C::kEpiStage);
        // columns per round: 32 fp32 (SPLIT) or 64 bf16, 128 bytes of the row either way
        constexpr int kStep = SPLIT ? 32 : 64;
#pragma unroll 1
        for (int j0 = c_lo; j0 < c_lo + c_n; j0 += kStep) {
          uint32_t y[32];
          tmem_ld32(taddr + j0, y);
          tmem_ld_wait();
          if (SPLIT) {
            // Each thread holds one row's 32 values; written straight out, one warp store
            // would touch 32 rows. Through the staging block, a store covers 4 rows with
            // 128 contiguous bytes each.
#pragma unroll
            for (int c = 0; c < 8; ++c)
              *reinterpret_cast<float4*>(sb + lane * 32 + ((c ^ (lane & 7)) << 2)) = make_float4(
                  gw * __uint_as_float(y[4 * c]), gw * __uint_as_float(y[4 * c + 1]),
                  gw * __uint_as_float(y[4 * c + 2]), gw * __uint_as_float(y[4 * c + 3]));
            __syncwarp();
            const int c = lane & 7;
            const int col = n0 + j0 + 4 * c;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const int r = 4 * i + (lane >> 3);
              const int64_t ro = __shfl_sync(0xffffffffu, orow, r);
              const int rv = __shfl_sync(0xffffffffu, (int)valid, r);
              const int rd = __shfl_sync(0xffffffffu, (int)direct, r);
              float4 v = *reinterpret_cast<const float4*>(sb + r * 32 + ((c ^ (r & 7)) << 2));
              if (rv && col < p.N) {
                if (!rd) {
                  *reinterpret_cast<float4*>(static_cast<float*>(p.out) + ro + col) = v;
                } else {
                  // the combine's sum of one term: 0 + y (a -0 becomes +0), rounded once
                  v = make_float4(v.x + 0.f, v.y + 0.f, v.z + 0.f, v.w + 0.f);
                  if (p.out_direct_f32)
                    *reinterpret_cast<float4*>(static_cast<float*>(p.out_direct) + ro + col) = v;
                  else
                    *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(p.out_direct) + ro +
                                              col) =
                        make_uint2(pack_bf16x2(v.x, v.y), pack_bf16x2(v.z, v.w));
                }
              }
            }
            __syncwarp();  // the block is read before the next chunk overwrites it
          } else {
            // 64 columns: this round's 32 and the next 32, as bf16 (one rounding each)
            uint32_t h[32];
#pragma unroll
            for (int i = 0; i < 16; ++i)
              h[i] = pack_bf16x2(gw * __uint_as_float(y[2 * i]),
                                 gw * __uint_as_float(y[2 * i + 1]));
            tmem_ld32(taddr + j0 + 32, y);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 16; ++i)
              h[16 + i] = pack_bf16x2(gw * __uint_as_float(y[2 * i]),
                                      gw * __uint_as_float(y[2 * i + 1]));
            // Each thread holds one row's 128 bytes; through the staging block a store
            // covers 4 rows with 128 contiguous bytes each (instead of 32 rows x 16 bytes).
            uint8_t* sh = reinterpret_cast<uint8_t*>(sb);
#pragma unroll
            for (int c = 0; c < 8; ++c)
              *reinterpret_cast<uint4*>(sh + lane * 128 + ((c ^ (lane & 7)) << 4)) =
                  make_uint4(h[4 * c], h[4 * c + 1], h[4 * c + 2], h[4 * c + 3]);
            __syncwarp();
            const int c = lane & 7;
            const int col = n0 + j0 + 8 * c;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const int r = 4 * i + (lane >> 3);
              const int64_t ro = __shfl_sync(0xffffffffu, orow, r);
              const int rv = __shfl_sync(0xffffffffu, (int)valid, r);
              const int rd = __shfl_sync(0xffffffffu, (int)direct, r);
              const uint4 v = *reinterpret_cast<const uint4*>(sh + r * 128 + ((c ^ (r & 7)) << 4));
              if (!rv || col >= p.N) continue;
              if (!rd) {
                *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out) + ro + col) = v;
                continue;
              }
              // the combine's sum of one bf16 term: 0 + float(bf16(y)), rounded once
              const uint32_t w[4] = {v.x, v.y, v.z, v.w};
              float f[8];
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                const float2 t =
                    __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[k]));
                f[2 * k] = t.x + 0.f;
                f[2 * k + 1] = t.y + 0.f;
              }
              if (p.out_direct_f32) {
                float* o = static_cast<float*>(p.out_direct) + ro + col;
                *reinterpret_cast<float4*>(o) = make_float4(f[0], f[1], f[2], f[3]);
                *reinterpret_cast<float4*>(o + 4) = make_float4(f[4], f[5], f[6], f[7]);
              } else {
                *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out_direct) + ro +
                                          col) =
                    make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]),
                               pack_bf16x2(f[4], f[5]), pack_bf16x2(f[6], f[7]));
              }
            }
            __syncwarp();  // the block is read before the next round overwrites it
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty_bar[a]);
      }
      if (stop) break;
      if (MT == 2) {
        acc_phase ^= 1;
      } else if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1;
      }
    }
  }

  __syncthreads();
  if (threadIdx.x == 0 && abort_flag) atomicOr(p.err, kErrTimeout);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

// ---- the down projection on CTA pairs (long expert blocks) -------------------------------
//
// With at least 256 rows per expert, gemm2 runs on pairs of CTAs (a 2-CTA cluster): one
// tcgen05.mma.cta_group::2 per k-step (two with SPLIT: H hi, then H lo, into one
// accumulator) covers 256 rows of one expert (128 from each CTA's shared memory) x N = 256
// columns of d, and each CTA stages only half of the W2 tile (128 columns). Per CTA and
// k-block the ring takes 16 KB of H (32 KB with SPLIT) and 16 KB of W2 instead of 16 (32) +
// 32 KB for the same MMA work: six stages fit (four with SPLIT). Each CTA's TMEM receives
// its own 128 rows for all 256 columns, and its epilogue is the one-CTA kernel's.
//
// Barriers: the ring's full barriers live in the leader (rank 0): both CTAs' copies
// complete on them (cta_group::2) and the leader's producer alone arrives, announcing both
// CTAs' bytes (the other CTA's copies may land first: the phase cannot complete while that
// arrival is missing). The empty and accumulator-full barriers live in each CTA (the
// leader's MMA thread commits to both); the accumulator-empty barriers in the leader (all
// sixteen epilogue warps of the pair arrive). Every wait is bounded.
constexpr int kPairBBytes = 2 * kBBoxBytes;                      // 128 columns x 64 K
constexpr int kPairEpiWarps = 8;
constexpr int kPairThreads = 32 * (2 + kPairEpiWarps);
constexpr int kPairEpiStage = 32 * 128;

template <bool SPLIT>
struct PairCfg {
  static constexpr int kATiles = SPLIT ? 2 : 1;                  // H hi (and H lo)
  static constexpr int kAStageBytes = kATiles * kABytes;         // 128 rows x 64 K each
  static constexpr int kStageBytes = kAStageBytes + kPairBBytes;
  static constexpr int kStages = SPLIT ? 4 : 6;
  static constexpr size_t kSmem =
      (size_t)kStages * kStageBytes + kPairEpiWarps * kPairEpiStage + 1024;
  static_assert(kSmem <= 232448, "dynamic shared memory beyond the 227 KB a CTA may use");
};

template <bool SPLIT>
__global__ void __launch_bounds__(kPairThreads, 1)
pair_gemm2_kernel(const __grid_constant__ CUtensorMap map_h,
                  const __grid_constant__ CUtensorMap map_hlo,
                  const __grid_constant__ CUtensorMap map_w, const Params p) {
  using PC = PairCfg<SPLIT>;
  constexpr int kPairStages = PC::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ __align__(8) uint64_t full_bar[kPairStages], empty_bar[kPairStages];
  __shared__ __align__(8) uint64_t tfull_bar[2], tempty_bar[2], drain_bar;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();  // 0: the leader, which issues the MMAs
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const int nk = (p.K + kBK - 1) / kBK;
  auto a_tile = [&](int st, int h) { return smem + st * PC::kStageBytes + h * kABytes; };
  auto b_tile = [&](int st) { return smem + st * PC::kStageBytes + PC::kAStageBytes; };
  uint8_t* const epi_smem = smem + (size_t)kPairStages * PC::kStageBytes;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kPairStages; ++i) {
      mbar_init(&full_bar[i], 1);  // the leader's producer, with both CTAs' bytes
      mbar_init(&empty_bar[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull_bar[i], 1);
      mbar_init(&tempty_bar[i], 2 * kPairEpiWarps);
    }
    mbar_init(&drain_bar, 1);
    abort_flag = 0;
    fence_mbar_init();
    prefetch_tensormap(&map_h);
    if (SPLIT) prefetch_tensormap(&map_hlo);
    prefetch_tensormap(&map_w);
  }
  if (warp == 1) tmem_alloc_pair(&tmem_base_sh, kTmemCols);
  tc_fence_before();
  cluster_sync_all();  // both CTAs' barriers are initialised and the TMEM is allocated
  tc_fence_after();
  const uint32_t tmem_base = tmem_base_sh;
  volatile int* abort_v = &abort_flag;
  pdl_wait();  // the previous kernel's outputs (H, gate, ent_pos) are complete
  pdl_launch_dependents();  // after the wait, as in the one-CTA down GEMM

  if (warp == 0) {
    // ---------------- TMA producer (both CTAs) ----------------
    const uint64_t wpol = l2_policy_evict_first();
    int stage = 0;
    uint32_t phase = 0;
    for (int item = pair; item < p.num_items; item += npairs) {
      const Tile tl = tile_of(item, p, 256);
      const int nbox = tl.half ? 1 : 2;  // 64-column boxes of this CTA's half of the W2 tile
      const uint32_t bytes = (uint32_t)(PC::kAStageBytes + nbox * kBBoxBytes);
      // tile_of counts row blocks of kBM; a pair item spans two of them
      const int hrow = tl.e * p.Ce + 2 * tl.m0 + (int)rank * kBM;
      const int col0 = tl.n0 + (int)rank * nbox * 64;
      bool ok = true;
      for (int kb = 0; kb < nk; ++kb) {
        int w = 1;
        if (lane == 0) w = mbar_wait(&empty_bar[stage], phase ^ 1, abort_v, p.wait_ns);
        ok = __shfl_sync(0xffffffffu, w, 0) != 0;
        if (!ok) break;
        const uint32_t fb = mapa_shared(&full_bar[stage], 0);
        if (lane == 0 && rank == 0) mbar_arrive_expect_tx(&full_bar[stage], 2 * bytes);
        __syncwarp();
        const int k0 = kb * kBK;
        if (lane == 0) tma_load_2d_pair(a_tile(stage, 0), &map_h, fb, k0, hrow);
        if (SPLIT && lane == 3) tma_load_2d_pair(a_tile(stage, 1), &map_hlo, fb, k0, hrow);
        if (lane >= 1 && lane <= nbox)
          tma_load_3d_pair(b_tile(stage) + (lane - 1) * kBBoxBytes, &map_w, fb,
                           col0 + 64 * (lane - 1), k0, tl.e, wpol);
        if (++stage == kPairStages) { stage = 0; phase ^= 1; }
      }
      if (!ok) break;
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------- MMA issuer (the leader's one thread) ----------------
    if (rank == 0 && lane == 0) {
      constexpr uint32_t idesc_full = idesc_bf16(256, 256, 1);  // B (W2) MN-major
      constexpr uint32_t idesc_half = idesc_bf16(256, 128, 1);
      int stage = 0, acc = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool ok = true;
      for (int item = pair; item < p.num_items && ok; item += npairs) {
        const uint32_t idesc = tile_of(item, p, 256).half ? idesc_half : idesc_full;
        if (!(ok = mbar_wait(&tempty_bar[acc], acc_phase ^ 1, abort_v, p.wait_ns))) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * kAccCols;
        for (int kb = 0; kb < nk; ++kb) {
          if (!(ok = mbar_wait(&full_bar[stage], phase, abort_v, p.wait_ns))) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk) {
            const uint64_t bd = sdesc_sw128(smem_u32(b_tile(stage)) + kk * 2048, kBBoxBytes, 1024);
#pragma unroll
            for (int h = 0; h < PC::kATiles; ++h) {
              const uint64_t ad = sdesc_sw128(smem_u32(a_tile(stage, h)) + kk * 32, 16, 1024);
              mma_bf16_pair(d_tmem, ad, bd, idesc, (kb | kk | h) != 0);
            }
          }
          mma_commit_pair(mapa_shared(&empty_bar[stage], 0));
          mma_commit_pair(mapa_shared(&empty_bar[stage], 1));
          if (++stage == kPairStages) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        mma_commit_pair(mapa_shared(&tfull_bar[acc], 0));
        mma_commit_pair(mapa_shared(&tfull_bar[acc], 1));
        if (++acc == 2) { acc = 0; acc_phase ^= 1; }
      }
      // every MMA issued above has completed once drain_bar flips
      mma_commit_pair(mapa_shared(&drain_bar, 0));
      int dummy = 0;
      mbar_wait(&drain_bar, 0, &dummy, kDrainNs);
    }
    __syncwarp();
  } else {
    // ---------------- epilogue: eight warps per CTA, two per TMEM lane quarter ----------
    // This CTA's 128 rows of the item, every column; the one-CTA kernel's paths.
    const int q = warp & 3;
    const int half = (warp - 2) >> 2;
    const int row = q * 32 + lane;
    uint8_t* sh = epi_smem + (warp - 2) * kPairEpiStage;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int item = pair; item < p.num_items; item += npairs) {
      const Tile tl = tile_of(item, p, 256);
      const int acc_n = tl.half ? 128 : 256;
      const int c_n = acc_n / 2;
      const int c_lo = half * c_n;
      int w = 1;
      if (lane == 0) w = mbar_wait(&tfull_bar[acc], acc_phase, abort_v, p.wait_ns);
      if (__shfl_sync(0xffffffffu, w, 0) == 0) break;
      tc_fence_after();
      const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + acc * kAccCols;
      const int s = 2 * tl.m0 + (int)rank * kBM + row;   // item rows: 2 * m0 + [0, 256)
      bool valid = s < p.Ce;
      const int64_t ent = (int64_t)tl.e * p.Ce + (valid ? s : 0);
      int64_t pos = p.ent_pos[ent];
      if (kDebugChecks && valid &&
          (pos >= p.rows_y ||
           (pos < 0 && (p.out_direct == nullptr || -pos - 1 >= (int64_t)p.rows_x)))) {
        atomicOr(p.err, kErrDeviceCheck);
        valid = false;
        pos = 0;
      }
      const bool direct = pos < 0;   // the token's only entry
      const int64_t orow = (direct ? -pos - 1 : pos) * p.N;
      const float gw = valid ? (p.gate ? p.gate[ent] : 1.f) : 0.f;
      constexpr int kStep = SPLIT ? 32 : 64;  // columns per round: 128 bytes of the row
#pragma unroll 1
      for (int j0 = c_lo; j0 < c_lo + c_n; j0 += kStep) {
        uint32_t y[32], h[32];
        tmem_ld32(taddr + j0, y);
        tmem_ld_wait();
        if constexpr (SPLIT) {
          // fp32 Y: 32 columns per round through the staging block, 4 rows x 128 bytes per
          // store
          float* sb = reinterpret_cast<float*>(sh);
#pragma unroll
          for (int c = 0; c < 8; ++c)
            *reinterpret_cast<float4*>(sb + lane * 32 + ((c ^ (lane & 7)) << 2)) = make_float4(
                gw * __uint_as_float(y[4 * c]), gw * __uint_as_float(y[4 * c + 1]),
                gw * __uint_as_float(y[4 * c + 2]), gw * __uint_as_float(y[4 * c + 3]));
          __syncwarp();
          const int c = lane & 7;
          const int col = tl.n0 + j0 + 4 * c;
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int r = 4 * i + (lane >> 3);
            const int64_t ro = __shfl_sync(0xffffffffu, orow, r);
            const int rv = __shfl_sync(0xffffffffu, (int)valid, r);
            const int rd = __shfl_sync(0xffffffffu, (int)direct, r);
            float4 v = *reinterpret_cast<const float4*>(sb + r * 32 + ((c ^ (r & 7)) << 2));
            if (!rv || col >= p.N) continue;
            if (!rd) {
              *reinterpret_cast<float4*>(static_cast<float*>(p.out) + ro + col) = v;
              continue;
            }
            // the combine's sum of one term: 0 + y (a -0 becomes +0), rounded once
            v = make_float4(v.x + 0.f, v.y + 0.f, v.z + 0.f, v.w + 0.f);
            if (p.out_direct_f32)
              *reinterpret_cast<float4*>(static_cast<float*>(p.out_direct) + ro + col) = v;
            else
              *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(p.out_direct) + ro + col) =
                  make_uint2(pack_bf16x2(v.x, v.y), pack_bf16x2(v.z, v.w));
          }
          __syncwarp();  // the block is read before the next round overwrites it
        } else {
#pragma unroll
        for (int i = 0; i < 16; ++i)
          h[i] = pack_bf16x2(gw * __uint_as_float(y[2 * i]), gw * __uint_as_float(y[2 * i + 1]));
        tmem_ld32(taddr + j0 + 32, y);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 16; ++i)
          h[16 + i] =
              pack_bf16x2(gw * __uint_as_float(y[2 * i]), gw * __uint_as_float(y[2 * i + 1]));
#pragma unroll
        for (int c = 0; c < 8; ++c)
          *reinterpret_cast<uint4*>(sh + lane * 128 + ((c ^ (lane & 7)) << 4)) =
              make_uint4(h[4 * c], h[4 * c + 1], h[4 * c + 2], h[4 * c + 3]);
        __syncwarp();
        const int c = lane & 7;
        const int col = tl.n0 + j0 + 8 * c;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int r = 4 * i + (lane >> 3);
          const int64_t ro = __shfl_sync(0xffffffffu, orow, r);
          const int rv = __shfl_sync(0xffffffffu, (int)valid, r);
          const int rd = __shfl_sync(0xffffffffu, (int)direct, r);
          const uint4 v = *reinterpret_cast<const uint4*>(sh + r * 128 + ((c ^ (r & 7)) << 4));
          if (!rv || col >= p.N) continue;
          if (!rd) {
            *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out) + ro + col) = v;
            continue;
          }
          // the combine's sum of one bf16 term: 0 + float(bf16(y)), rounded once
          const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
          float f[8];
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const float2 t = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&wv[k]));
            f[2 * k] = t.x + 0.f;
            f[2 * k + 1] = t.y + 0.f;
          }
          if (p.out_direct_f32) {
            float* o = static_cast<float*>(p.out_direct) + ro + col;
            *reinterpret_cast<float4*>(o) = make_float4(f[0], f[1], f[2], f[3]);
            *reinterpret_cast<float4*>(o + 4) = make_float4(f[4], f[5], f[6], f[7]);
          } else {
            *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out_direct) + ro + col) =
                make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]),
                           pack_bf16x2(f[4], f[5]), pack_bf16x2(f[6], f[7]));
          }
        }
        __syncwarp();  // the block is read before the next round overwrites it
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(mapa_shared(&tempty_bar[acc], 0));
      if (++acc == 2) { acc = 0; acc_phase ^= 1; }
    }
  }

  __syncthreads();
  if (*abort_v) {
    // a wait ran out: give the copies this CTA issued (which complete on the leader's
    // barriers, out of this CTA's sight) time to land before the pair's final barrier
    const uint64_t t0 = globaltimer_ns();
    while ((int64_t)(globaltimer_ns() - t0) < 1000000) {
    }
  }
  cluster_sync_all();  // the other CTA no longer touches this CTA's barriers or TMEM
  if (threadIdx.x == 0 && abort_flag) atomicOr(p.err, kErrTimeout);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, kTmemCols);
  }
}

// ---- host side ----------------------------------------------------------------------------

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(tensor_map_encoder());
}

// bf16 tensor map with 128-byte swizzle. dims/box are innermost first; strides are the
// byte strides of dims 1.. (rank - 1 entries).
bool make_map(CUtensorMap* m, const void* base, int rank, const uint64_t* dims,
              const uint64_t* strides, const uint32_t* box) {
  auto fn = encode_fn();
  if (!fn) return false;
  uint32_t elem[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (cuuint32_t)rank, const_cast<void*>(base),
                  dims, strides, box, elem, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Weights [E, K, N] bf16, N contiguous: boxes of 64 N x 64 K of one expert.
bool weight_map(CUtensorMap* m, const void* W, int E, int K, int N) {
  uint64_t dims[3] = {(uint64_t)N, (uint64_t)K, (uint64_t)E};
  uint64_t strides[2] = {(uint64_t)N * 2, (uint64_t)K * N * 2};
  uint32_t box[3] = {64, 64, 1};
  return make_map(m, W, 3, dims, strides, box);
}

// Rows of a [rows, cols] bf16 matrix, boxes of box_rows x 64 columns.
bool rows_map(CUtensorMap* m, const void* base, int64_t rows, int cols, uint32_t box_rows) {
  uint64_t dims[2] = {(uint64_t)cols, (uint64_t)rows};
  uint64_t strides[1] = {(uint64_t)cols * 2};
  uint32_t box[2] = {64, box_rows};
  return make_map(m, base, 2, dims, strides, box);
}

// With one persistent CTA per SM, the last wave of tiles is partial. When it fills at
// most half of the SMs, its tiles run as two half-width items each, so that wave takes
// half as long on up to twice the SMs.
void split_tail(Params& p, int sm_count) {
  const int r = p.num_tiles % sm_count;
  p.num_full = p.num_tiles;
  if (r > 0 && 2 * r <= sm_count) p.num_full = p.num_tiles - r;
  p.num_items = p.num_full + 2 * (p.num_tiles - p.num_full);
}

template <int MODE, bool SPLIT, int GATHER, int MT = 1>
cudaError_t launch(const CUtensorMap& a, const CUtensorMap& a2, const CUtensorMap& b0,
                   const CUtensorMap& b1, const __nv_bfloat16* x, const Params& p,
                   int sm_count, cudaStream_t st, bool pdl) {
  using C = Cfg<MODE, SPLIT, GATHER, MT>;
  const int grid = p.num_items < sm_count ? p.num_items : sm_count;
  return launch_kernel(grouped_gemm_kernel<MODE, SPLIT, GATHER, MT>, dim3(grid),
                       dim3(C::kThreads), C::kSmem, st, pdl, 1, a, a2, b0, b1, x, p);
}

}  // namespace

bool experts_sm100_supported(const Shape& s) {
  return s.d >= 64 && s.F >= 64 && (int64_t)s.E * s.Ce >= kBM && s.d % 8 == 0 &&
         s.F % 8 == 0 && encode_fn() != nullptr;
}

bool gemm1_sm100_fuses_csr(const Shape& s, bool split) {
  const size_t room = split ? Cfg<kGemm1, true, kGatherLsu>::kEpiWarps *
                                  (size_t)Cfg<kGemm1, true, kGatherLsu>::kEpiStage
                            : Cfg<kGemm1, false, kGatherLsu>::kEpiWarps *
                                  (size_t)Cfg<kGemm1, false, kGatherLsu>::kEpiStage;
  return csr_smem_bytes(s.E) <= room;
}

cudaError_t launch_gemm1_sm100(const void* x, const int32_t* idx, const void* W1,
                               const void* W3, const Shape& s, bool split, bool tma_gather,
                               void* H_hi, void* H_lo, const CsrArgs* csr, unsigned* err,
                               int sm_count, cudaStream_t st) {
  CUtensorMap ma, mb0, mb1;
  if (!rows_map(&ma, x, s.T, s.d, 1) || !weight_map(&mb0, W1, s.E, s.d, s.F) ||
      !weight_map(&mb1, W3, s.E, s.d, s.F))
    return cudaErrorInvalidValue;
  // Two row blocks per item (the cp.async gather only) for experts of at least 1024 rows.
  // Measured interleaved on one B200: batch-4 (Ce = 2048) layer -3.7%; the model default
  // (Ce = 512) unchanged within noise; 512 px (Ce = 256, half as many items: 1.7 waves
  // without a split tail) +6%. Weight-streaming tiles also lose the accumulators' double
  // buffering across items.
  const int mt = (!tma_gather && s.Ce >= 8 * kBM) ? 2 : 1;
  Params p;
  p.Ce = s.Ce; p.K = s.d; p.N = s.F;
  p.tiles_m = (int)ceil_div(s.Ce, mt * kBM);
  p.tiles_n = (int)ceil_div(s.F, 128);
  p.num_tiles = s.E * p.tiles_m * p.tiles_n;
  split_tail(p, sm_count);
  p.idx = idx; p.gate = nullptr; p.ent_pos = nullptr; p.out = H_hi; p.out_lo = H_lo;
  p.out_direct = nullptr; p.out_direct_f32 = 0;
  p.csr_blocks = 0;
  if (csr != nullptr) {
    if (!gemm1_sm100_fuses_csr(s, split)) return cudaErrorInvalidValue;
    p.csr = *csr;
    p.csr_blocks = (int)ceil_div(s.T, kCsrBlockTok);
  }
  p.err = err;
  p.wait_ns = s.wait_ns;
  p.rows_x = s.T;
  p.rows_y = s.y_rows;
  const __nv_bfloat16* xb = static_cast<const __nv_bfloat16*>(x);
  if (tma_gather)
    return split ? launch<kGemm1, true, kGatherTma4>(ma, ma, mb0, mb1, xb, p, sm_count, st, s.pdl)
                 : launch<kGemm1, false, kGatherTma4>(ma, ma, mb0, mb1, xb, p, sm_count, st, s.pdl);
  if (mt == 2)
    return split ? launch<kGemm1, true, kGatherLsu, 2>(ma, ma, mb0, mb1, xb, p, sm_count, st, s.pdl)
                 : launch<kGemm1, false, kGatherLsu, 2>(ma, ma, mb0, mb1, xb, p, sm_count, st, s.pdl);
  return split ? launch<kGemm1, true, kGatherLsu>(ma, ma, mb0, mb1, xb, p, sm_count, st, s.pdl)
               : launch<kGemm1, false, kGatherLsu>(ma, ma, mb0, mb1, xb, p, sm_count, st, s.pdl);
}

namespace {

// Pairs of SMs that can hold one pair CTA each at the same time (a pair's two CTAs sit on
// one TPC): what the occupancy calculator reports for 2-CTA clusters of the pair kernel.
template <bool SPLIT>
int pair_slots(int sm_count) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  static std::mutex mu;
  static std::vector<std::pair<int, int>> cache;  // (device, slots)
  std::lock_guard<std::mutex> lk(mu);
  for (const auto& c : cache)
    if (c.first == dev) return c.second;
  int n = 0;
  if (set_smem_limit(reinterpret_cast<const void*>(pair_gemm2_kernel<SPLIT>),
                     PairCfg<SPLIT>::kSmem) == cudaSuccess) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(sm_count & ~1));
    cfg.blockDim = dim3(kPairThreads);
    cfg.dynamicSmemBytes = PairCfg<SPLIT>::kSmem;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeClusterDimension;
    attr.val.clusterDim.x = 2;
    attr.val.clusterDim.y = 1;
    attr.val.clusterDim.z = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    if (cudaOccupancyMaxActiveClusters(&n, pair_gemm2_kernel<SPLIT>, &cfg) != cudaSuccess) {
      cudaGetLastError();  // no pair slots: the one-CTA kernel runs instead
      n = 0;
    }
  } else {
    cudaGetLastError();
  }
  cache.emplace_back(dev, n);
  return n;
}

int pair_slots(bool split, int sm_count) {
  return split ? pair_slots<true>(sm_count) : pair_slots<false>(sm_count);
}

cudaError_t launch_gemm2_pair(const void* H, const void* H_lo, bool split, const float* gate,
                              const int32_t* ent_pos, const void* W2, const Shape& s, void* Y,
                              void* out_direct, bool out_direct_f32, unsigned* err, int npairs,
                              cudaStream_t st) {
  CUtensorMap mh, mhl, mw;
  const int64_t rows = (int64_t)s.E * s.Ce;
  if (!rows_map(&mh, H, rows, s.F, kBM) || !weight_map(&mw, W2, s.E, s.F, s.d))
    return cudaErrorInvalidValue;
  if (split && !rows_map(&mhl, H_lo, rows, s.F, kBM)) return cudaErrorInvalidValue;
  if (!split) mhl = mh;
  Params p;
  p.Ce = s.Ce; p.K = s.F; p.N = s.d;
  p.tiles_m = (int)ceil_div(s.Ce, 2 * kBM);
  p.tiles_n = (int)ceil_div(s.d, 256);
  p.num_tiles = s.E * p.tiles_m * p.tiles_n;
  split_tail(p, npairs);
  p.idx = nullptr; p.gate = gate; p.ent_pos = ent_pos; p.out = Y; p.out_lo = nullptr;
  p.out_direct = out_direct; p.out_direct_f32 = out_direct_f32 ? 1 : 0;
  p.csr_blocks = 0;
  p.err = err;
  p.wait_ns = s.wait_ns;
  p.rows_x = s.T;
  p.rows_y = s.y_rows;
  const int pairs = p.num_items < npairs ? p.num_items : npairs;
  if (split)
    return launch_kernel(pair_gemm2_kernel<true>, dim3((unsigned)(2 * pairs)),
                         dim3(kPairThreads), PairCfg<true>::kSmem, st, s.pdl, 2, mh, mhl, mw, p);
  return launch_kernel(pair_gemm2_kernel<false>, dim3((unsigned)(2 * pairs)),
                       dim3(kPairThreads), PairCfg<false>::kSmem, st, s.pdl, 2, mh, mhl, mw, p);
}

cudaError_t launch_gemm2_one_cta(const void* H_hi, const void* H_lo, const float* gate,
                                 const int32_t* ent_pos, const void* W2, const Shape& s,
                                 bool split, void* Y, void* out_direct, bool out_direct_f32,
                                 unsigned* err, int sm_count, cudaStream_t st) {
  CUtensorMap ma, ma2, mb;
  const int64_t rows = (int64_t)s.E * s.Ce;
  if (!rows_map(&ma, H_hi, rows, s.F, kBM) || !weight_map(&mb, W2, s.E, s.F, s.d))
    return cudaErrorInvalidValue;
  if (split && !rows_map(&ma2, H_lo, rows, s.F, kBM)) return cudaErrorInvalidValue;
  if (!split) ma2 = ma;
  Params p;
  p.Ce = s.Ce; p.K = s.F; p.N = s.d;
  p.tiles_m = (int)ceil_div(s.Ce, kBM);
  p.tiles_n = (int)ceil_div(s.d, 256);
  p.num_tiles = s.E * p.tiles_m * p.tiles_n;
  split_tail(p, sm_count);
  p.idx = nullptr; p.gate = gate; p.ent_pos = ent_pos; p.out = Y; p.out_lo = nullptr;
  p.out_direct = out_direct; p.out_direct_f32 = out_direct_f32 ? 1 : 0;
  p.csr_blocks = 0;
  p.err = err;
  p.wait_ns = s.wait_ns;
  p.rows_x = s.T;
  p.rows_y = s.y_rows;
  return split ? launch<kGemm2, true, kGatherLsu>(ma, ma2, mb, mb, nullptr, p, sm_count, st, s.pdl)
               : launch<kGemm2, false, kGatherLsu>(ma, ma2, mb, mb, nullptr, p, sm_count, st, s.pdl);
}

}  // namespace

bool gemm2_sm100_uses_pairs(const Shape& s, bool split, int sm_count) {
  return s.Ce >= 2 * kBM && s.d % 64 == 0 && pair_slots(split, sm_count) > 0;
}

cudaError_t launch_gemm2_sm100(const void* H_hi, const void* H_lo, const float* gate,
                               const int32_t* ent_pos, const void* W2, const Shape& s, bool split,
                               void* Y, void* out_direct, bool out_direct_f32, unsigned* err,
                               int sm_count, cudaStream_t st) {
  if (gemm2_sm100_uses_pairs(s, split, sm_count))
    return launch_gemm2_pair(H_hi, H_lo, split, gate, ent_pos, W2, s, Y, out_direct,
                             out_direct_f32, err, pair_slots(split, sm_count), st);
  return launch_gemm2_one_cta(H_hi, H_lo, gate, ent_pos, W2, s, split, Y, out_direct,
                              out_direct_f32, err, sm_count, st);
}

}  // namespace nmoe
