// Router GEMM + score function on the tensor cores, for bf16 inputs.
//
// NucleusMoE-Image walkthrough, section 6.2: gate = Linear(hidden, experts, no bias),
// scored by softmax (or sigmoid), then viewed per expert. logits[t, e] = x[t, :] W_r[:, e].
//
// Precision: the scores must match an fp64 reference to 1e-5 relative, and with
// LogNormal-scaled tokens the logits reach |l| ~ 30, where a single fp32 accumulator
// over d = 2048 drifts by more than that (tensor-core accumulation also truncates). So
// the MMAs accumulate only one 128-long k-chunk (two k-blocks) per TMEM slice, and the
// epilogue warps read every chunk back with tcgen05.ld (two chunks per round trip) and
// add it to Kahan-compensated fp32 running sums. (Modelled on the 1024 px workload with
// round-toward-zero accumulation, 128-long chunks keep the scores within ~3e-6 of fp64,
// 256-long ones ~8e-6; 64-long ones took twice the read-back round trips.) From there
// each logit is an unevaluated pair of fp32 numbers h + l, and the score function works
// on the pairs: two-sum for every shift, exp(h + l) = exp(h) (1 + l), compensated sums,
// one fp32 division (relative error a few 1e-7).
//
// Each 128-token tile is split along d between the two CTAs of a cluster (so T = 8192
// fills 128 SMs, not 64). In each CTA, warp 0 streams x and W_r tiles with TMA into a
// 6-stage ring; warp 1 (one thread) issues tcgen05.mma (M = 128, N = E rounded up to
// 64, K = 16) into a ring of TMEM chunk buffers; 4*G epilogue warps (G = ceil(E/CW))
// each own 32 tokens x CW experts. Then each CTA sends its sums for the partner's half
// of the tokens to the partner's shared memory (distributed shared memory, no global
// traffic), and all its epilogue warps finish the score function and both score layouts
// for its 64 tokens. Every wait is bounded.
#include <cudaTypedefs.h>

#include <cooperative_groups.h>

#include "router_sm100.cuh"
#include "sm100_ptx.cuh"

namespace cg = cooperative_groups;

namespace nmoe {
namespace {

using namespace ptx;

constexpr int kBM = 128;
constexpr int kBK = 64;
constexpr int kStages = 6;
constexpr int kABytes = kBM * kBK * 2;     // 16 KB
constexpr int kBBoxBytes = 64 * kBK * 2;   // 8 KB: 64 experts x 64 k
constexpr int kMaxE = 128;
constexpr int kSplit = 2;   // CTAs per token tile (one cluster), each owning half of d
constexpr int kChunkKB = 2; // k-blocks accumulated per TMEM chunk slice (128-long chunks)
constexpr uint64_t kDrainNs = 20000000ull;  // 20 ms per drain wait after an abort

struct Params {
  int T, d, E, S;
  int epad;         // N of the MMA: E rounded up to 64
  int nbox;         // epad / 64
  int nbuf;         // TMEM chunk buffers of epad columns (even)
  int score_fn;
  const float* bias;
  float* scores;
  float* scores_t;
  unsigned* err;
  uint64_t wait_ns;  // budget of each pipeline wait
};

// a + b = s + e exactly (Knuth's two-sum; no operation here may be contracted or
// reassociated, which nvcc does not do to plain adds).
__device__ __forceinline__ void two_sum(float a, float b, float& s, float& e) {
  s = a + b;
  const float bb = s - a;
  e = (a - (s - bb)) + (b - bb);
}

// Each epilogue thread owns CW experts (16 up to E = 64, else 32) of one token row;
// G = ceil(E / CW) column groups, so the epilogue has 4 G warps (one per TMEM lane
// quarter and group).
template <int G, int CW>
__global__ void __launch_bounds__(64 + 128 * G, 1)
router_sm100_kernel(const __grid_constant__ CUtensorMap map_x,
                    const __grid_constant__ CUtensorMap map_w, const Params p) {
  pdl_launch_dependents();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int b_bytes = p.nbox * kBBoxBytes;
  uint8_t* sA = smem;
  uint8_t* sB = smem + kStages * kABytes;
  __shared__ __align__(8) uint64_t full_bar[kStages], empty_bar[kStages];
  __shared__ __align__(8) uint64_t tfull_bar[8], tempty_bar[8], drain_bar;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = (int)cluster.block_rank();
  const int nk_all = (p.d + kBK - 1) / kBK;
  const int kb0 = rank == 0 ? 0 : (nk_all + 1) / 2;
  const int nk = rank == 0 ? (nk_all + 1) / 2 : nk_all - (nk_all + 1) / 2;
  const int nch = (nk + kChunkKB - 1) / kChunkKB;  // chunk slices this CTA fills
  const int t0 = (blockIdx.x / kSplit) * kBM;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) { mbar_init(&full_bar[i], 1); mbar_init(&empty_bar[i], 1); }
    for (int i = 0; i < p.nbuf; ++i) { mbar_init(&tfull_bar[i], 1); mbar_init(&tempty_bar[i], 4 * G); }
    mbar_init(&drain_bar, 1);
    abort_flag = 0;
    fence_mbar_init();
    prefetch_tensormap(&map_x);
    prefetch_tensormap(&map_w);
  }
  if (warp == 2) tmem_alloc(&tmem_base_sh, 512);
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = tmem_base_sh;
  volatile int* abort_v = &abort_flag;
  pdl_wait();  // x, W_r and the bias are complete; earlier readers of the outputs are done

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0, issued_mask = 0, issued_par = 0;
      for (int kb = 0; kb < nk; ++kb) {
        if (!mbar_wait(&empty_bar[stage], phase ^ 1, abort_v, p.wait_ns)) break;
        mbar_arrive_expect_tx(&full_bar[stage], kABytes + b_bytes);
        const int k0 = (kb0 + kb) * kBK;
        tma_load_2d(sA + stage * kABytes, &map_x, &full_bar[stage], k0, t0);
        for (int j = 0; j < p.nbox; ++j)
          tma_load_2d(sB + stage * b_bytes + j * kBBoxBytes, &map_w, &full_bar[stage], 64 * j,
                      k0);
        issued_mask |= 1u << stage;
        issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
        if (++stage == kStages) { stage = 0; phase ^= 1; }
      }
      if (*abort_v) {
        int dummy = 0;
        for (int s = 0; s < kStages; ++s)
          if (issued_mask & (1u << s))
            mbar_wait(&full_bar[s], (issued_par >> s) & 1u, &dummy, kDrainNs);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16(kBM, p.epad, 1);
      int stage = 0, buf = 0;
      uint32_t phase = 0, buf_phase = 0;
      for (int kb = 0; kb < nk; ++kb) {
        const bool first = kb % kChunkKB == 0;
        const bool last = kb % kChunkKB == kChunkKB - 1 || kb == nk - 1;
        if (first && !mbar_wait(&tempty_bar[buf], buf_phase ^ 1, abort_v, p.wait_ns)) break;
        if (!mbar_wait(&full_bar[stage], phase, abort_v, p.wait_ns)) break;
        tc_fence_after();
        const uint32_t a_addr = smem_u32(sA + stage * kABytes);
        const uint32_t b_addr = smem_u32(sB + stage * b_bytes);
        const uint32_t d0 = tmem_base + buf * p.epad;
#pragma unroll
        for (int kk = 0; kk < kBK / 16; ++kk) {
          const uint64_t ad = sdesc_sw128(a_addr + kk * 32, 16, 1024);
          const uint64_t bd = sdesc_sw128(b_addr + kk * 2048, kBBoxBytes, 1024);
          // one chunk slice per kChunkKB k-blocks, restarted at the chunk's first MMA
          mma_bf16(d0, ad, bd, idesc, !(first && kk == 0));
        }
        mma_commit(&empty_bar[stage]);
        if (++stage == kStages) { stage = 0; phase ^= 1; }
        if (last) {
          mma_commit(&tfull_bar[buf]);
          if (++buf == p.nbuf) { buf = 0; buf_phase ^= 1; }
        }
      }
      mma_commit(&drain_bar);
      int dummy = 0;
      mbar_wait(&drain_bar, 0, &dummy, kDrainNs);
    }
  } else {
    // ---------------- epilogue: 32 tokens x CW experts per warp ----------------
    const int q = warp & 3;
    const int g = (warp - 2) >> 2;
    const int row = q * 32 + lane;
    const int e0 = g * CW;
    // Kahan-compensated fp32 sums of the chunk sums: hi accumulates, lo keeps
    // what each addition rounded away (error ~2 ulp of the total, however many chunks);
    // hi + lo is taken in fp64 once at the end.
    float hi[CW], lo[CW];
#pragma unroll
    for (int j = 0; j < CW; ++j) { hi[j] = 0.f; lo[j] = 0.f; }
    int buf = 0;
    uint32_t buf_phase = 0;
    bool ok = true;
    // two chunk slices per TMEM-load round trip
    for (int ch = 0; ch < nch; ch += 2) {
      const bool two = ch + 1 < nch;
      int w = 1;
      if (lane == 0) {
        w = mbar_wait(&tfull_bar[buf], buf_phase, abort_v, p.wait_ns);
        if (w && two) w = mbar_wait(&tfull_bar[buf + 1], buf_phase, abort_v, p.wait_ns);
      }
      if (__shfl_sync(0xffffffffu, w, 0) == 0) { ok = false; break; }
      tc_fence_after();
      const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + buf * p.epad + e0;
#pragma unroll
      for (int h = 0; h < CW / 16; ++h) {
        uint32_t c0[16], c1[16];
        tmem_ld16(taddr + h * 16, c0);
        if (two) tmem_ld16(taddr + p.epad + h * 16, c1);
        tmem_ld_wait();
        if (h == CW / 16 - 1) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) {
            mbar_arrive(&tempty_bar[buf]);
            if (two) mbar_arrive(&tempty_bar[buf + 1]);
          }
        }
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          // the round's two chunk sums (one rounding), then Kahan
          const float c = two ? __uint_as_float(c0[j]) + __uint_as_float(c1[j])
                              : __uint_as_float(c0[j]);
          const float y = c - lo[h * 16 + j];
          const float t = hi[h * 16 + j] + y;
          lo[h * 16 + j] = (t - hi[h * 16 + j]) - y;
          hi[h * 16 + j] = t;
        }
      }
      buf += 2;
      if (buf >= p.nbuf) { buf -= p.nbuf; buf_phase ^= 1; }
    }
    // Each logit as an unevaluated fp32 pair h + l (l below half an ulp of h): the
    // compensated sum hi - lo, renormalised.
    // Each logit as an unevaluated fp32 pair h + l (l below half an ulp of h), from the
    // compensated sum hi - lo. Tokens 0..63 of the tile are finished by the first CTA,
    // 64..127 by the second. Every thread puts its half-d pairs where the finishing CTA
    // reads them, laid out [expert][64 tokens]: its own rows in `own`, the partner's rows
    // in the partner's `xch` (distributed shared memory). The first cluster barrier has
    // left both stage rings idle for this.
    const bool mine = (q >> 1) == rank;
    float2* xch = reinterpret_cast<float2*>(smem);
    float2* own = xch + (size_t)kMaxE * 64;
    float* red_m = reinterpret_cast<float*>(own + (size_t)kMaxE * 64);  // [2G][64]
    float2* red_z = reinterpret_cast<float2*>(red_m + 8 * 64);          // [2G][64]
    cluster.sync();                         // (1) every ring is idle
    {
      float2* dst = mine ? own : cluster.map_shared_rank(xch, rank ^ 1);
      const int r64 = row & 63;
#pragma unroll
      for (int j = 0; j < CW; ++j) {
        float s_, e_;
        two_sum(hi[j], -lo[j], s_, e_);
        if (e0 + j < p.E) dst[(e0 + j) * 64 + r64] = make_float2(s_, e_);
      }
    }
    cluster.sync();                         // (2) the partner's sums have landed
    // All 4G epilogue warps finish this CTA's 64 tokens: thread et takes token et % 64
    // and the kEpc experts of group et / 64 (2G groups).
    constexpr int kEpc = CW / 2;
    const int nthr = 128 * G;
    const int et = threadIdx.x - 64;
    const int tk = et & 63, grp = et >> 6;
    const int eb = grp * kEpc;
    const int t = t0 + rank * 64 + tk;
    const bool live = t < p.T;
    const float* b = (p.bias != nullptr && live) ? p.bias + (int64_t)(t / p.S) * p.E : nullptr;
    float h[kEpc], l[kEpc], pr[kEpc];
#pragma unroll
    for (int j = 0; j < kEpc; ++j) {
      h[j] = 0.f;
      l[j] = 0.f;
      const int e = eb + j;
      if (e < p.E) {
        const float2 u = own[e * 64 + tk], v = xch[e * 64 + tk];
        float s_, e_;
        two_sum(u.x, v.x, s_, e_);
        two_sum(s_, e_ + (u.y + v.y), h[j], l[j]);
        if (b) {
          two_sum(h[j], b[e], s_, e_);
          two_sum(s_, e_ + l[j], h[j], l[j]);
        }
      }
    }
    if (p.score_fn == NMOE_SCORE_SOFTMAX) {
      // shift by the largest high part; exp(h - m + l) = exp(d) (1 + t) with d + t =
      // h - m + l exactly up to t's rounding (|t| < 1e-6, so the dropped t^2 is far
      // below fp32)
      float m = -INFINITY;
#pragma unroll
      for (int j = 0; j < kEpc; ++j)
        if (eb + j < p.E) m = fmaxf(m, h[j]);
      red_m[grp * 64 + tk] = m;
      asm volatile("bar.sync 1, %0;" ::"r"(nthr) : "memory");
      for (int k = 0; k < 2 * G; ++k) m = fmaxf(m, red_m[k * 64 + tk]);
      bool deep = false;                     // some argument below -80
      float zs = 0.f, zc = 0.f;              // compensated sum of the exponentials
#pragma unroll
      for (int j = 0; j < kEpc; ++j) {
        float dd, tt;                        // exp argument: dd + tt
        two_sum(h[j], -m, dd, tt);
        tt += l[j];
        const bool live_e = eb + j < p.E;
        deep |= live_e && dd < -80.f;
        pr[j] = live_e ? expf(dd) * (1.f + tt) : 0.f;
      }
      // below e^-80 the fp32 exponential leaves the normal range: fp64 there (rare, and
      // kept out of the loop above so that it costs nothing otherwise)
      if (__any_sync(0xffffffffu, deep)) {
        for (int j = 0; j < kEpc; ++j) {
          float dd, tt;
          two_sum(h[j], -m, dd, tt);
          if (eb + j < p.E && dd < -80.f) pr[j] = (float)exp((double)dd + (double)(tt + l[j]));
        }
      }
#pragma unroll
      for (int j = 0; j < kEpc; ++j) {
        float s_, e_;
        two_sum(zs, pr[j], s_, e_);
        zs = s_;
        zc += e_;
      }
      red_z[grp * 64 + tk] = make_float2(zs, zc);
      asm volatile("bar.sync 1, %0;" ::"r"(nthr) : "memory");
      zs = 0.f;
      zc = 0.f;
      for (int k = 0; k < 2 * G; ++k) {
        const float2 v = red_z[k * 64 + tk];
        float s_, e_;
        two_sum(zs, v.x, s_, e_);
        zs = s_;
        zc += e_ + v.y;
      }
      const float rz = 1.f / (zs + zc);      // one division; each score 1 ulp from e / z
#pragma unroll
      for (int j = 0; j < kEpc; ++j) pr[j] *= rz;
    } else {
      // 1 / (1 + exp(-(h + l))), exp(-(h + l)) = exp(-h) (1 - l)
      bool deep = false;
#pragma unroll
      for (int j = 0; j < kEpc; ++j) {
        deep |= fabsf(h[j]) > 80.f;
        pr[j] = 1.f / (1.f + expf(-h[j]) * (1.f - l[j]));
      }
      if (__any_sync(0xffffffffu, deep)) {
        for (int j = 0; j < kEpc; ++j)
          if (fabsf(h[j]) > 80.f)
            pr[j] = (float)(1.0 / (1.0 + exp(-((double)h[j] + (double)l[j]))));
      }
    }
    if (ok && live && eb < p.E) {
      float* srow = p.scores + (int64_t)t * p.E + eb;
      if ((p.E & 3) == 0 && eb + kEpc <= p.E) {
#pragma unroll
        for (int j = 0; j < kEpc; j += 4)
          *reinterpret_cast<float4*>(srow + j) =
              make_float4(pr[j], pr[j + 1], pr[j + 2], pr[j + 3]);
      } else {
        for (int j = 0; j < kEpc; ++j)
          if (eb + j < p.E) srow[j] = pr[j];
      }
#pragma unroll
      for (int j = 0; j < kEpc; ++j)
        if (eb + j < p.E) p.scores_t[(int64_t)(eb + j) * p.T + t] = pr[j];
    }
  }
  if (warp < 2) {
    // the producer and MMA warps take part in the two cluster barriers as well
    __syncwarp();
    cluster.sync();
    cluster.sync();
  }

  __syncthreads();
  if (threadIdx.x == 0 && abort_flag) atomicOr(p.err, kErrTimeout);
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(tensor_map_encoder());
}

bool map_2d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint32_t box_in,
            uint32_t box_out) {
  auto fn = encode_fn();
  if (!fn) return false;
  uint64_t dims[2] = {inner, outer};
  uint64_t strides[1] = {inner * 2};
  uint32_t box[2] = {box_in, box_out};
  uint32_t elem[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
            elem, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

}  // namespace

bool router_sm100_supported(const Shape& s) {
  return s.E >= 1 && s.E <= kMaxE && s.T >= kBM && s.d >= kBK && s.d % 8 == 0 &&
         encode_fn() != nullptr;
}

cudaError_t launch_router_sm100(const void* x, const void* W_r, const Shape& s,
                                nmoe_score_fn fn, const float* bias, float* scores,
                                float* scores_t, unsigned* err, cudaStream_t st) {
  Params p;
  p.T = s.T; p.d = s.d; p.E = s.E; p.S = s.S;
  p.epad = (int)ceil_div(s.E, 64) * 64;
  p.nbox = p.epad / 64;
  p.nbuf = 512 / p.epad;   // one epad-wide chunk slice per k-block: 8 (E <= 64) or 4
  if (p.nbuf > 8) p.nbuf = 8;
  p.score_fn = (int)fn;
  p.bias = bias; p.scores = scores; p.scores_t = scores_t; p.err = err;
  p.wait_ns = s.wait_ns;
  CUtensorMap mx, mw;
  if (!map_2d(&mx, x, (uint64_t)s.d, (uint64_t)s.T, 64, kBM) ||
      !map_2d(&mw, W_r, (uint64_t)s.E, (uint64_t)s.d, 64, 64))
    // a shape the tensor maps cannot describe: the CUDA-core router computes the same
    return launch_router_simt(x, W_r, s, NMOE_BF16, fn, bias, scores, scores_t, st);
  size_t smem = (size_t)kStages * (kABytes + p.nbox * kBBoxBytes);
  // the tail reuses the ring: two [kMaxE][64] arrays of (h, l) pairs, then [8][64] maxima
  // and [8][64] (sum, error) pairs
  const size_t red = 2 * sizeof(float2) * 64 * kMaxE + sizeof(float) * 8 * 64 +
                     sizeof(float2) * 8 * 64;
  smem = (smem > red ? smem : red) + 1024;
  // 16 experts per thread up to E = 64 (up to 16 epilogue warps), 32 beyond
  const int CW = s.E <= 64 ? 16 : 32;
  const int G = (int)ceil_div(s.E, CW);
  auto k = CW == 16 ? (G == 1 ? router_sm100_kernel<1, 16>
                     : G == 2 ? router_sm100_kernel<2, 16>
                     : G == 3 ? router_sm100_kernel<3, 16>
                              : router_sm100_kernel<4, 16>)
                    : (G == 3 ? router_sm100_kernel<3, 32> : router_sm100_kernel<4, 32>);
  return launch_kernel(k, dim3((unsigned)(ceil_div(s.T, kBM) * kSplit)), dim3(64 + 128 * G), smem,
                       st, s.pdl, kSplit, mx, mw, p);
}

}  // namespace nmoe
