// C ABI of libnmoe: argument checks, workspace layout, stage launches.
//
// Every entry point validates its arguments on the host before it touches CUDA, so a
// rejected call enqueues nothing. The layer's steps run in this library's kernels in
// launch order router -> select -> csr -> gemm1 -> gemm2 -> combine, all on the
// caller's stream, with no host synchronisation (every shape is fixed by (T, E, C):
// expert choice gives each expert exactly C tokens per segment).
#include <math.h>
#include <mutex>
#include <new>
#include <vector>

#include "csr_block.cuh"
#include "nmoe_internal.cuh"
#include "experts_sm100.cuh"
#include "router_sm100.cuh"

// Per-device error word: kernels OR kErr* bits into it; nmoe_get_last_error reads and
// clears it. Host code reaches it through cudaGetSymbolAddress.
__device__ unsigned nmoe_g_err_word;

namespace {

using nmoe::Shape;

struct DevState {
  bool ready = false;
  bool ok = false;
  int sm_count = 0;
  unsigned* err = nullptr;
};

std::mutex g_mu;
constexpr int kMaxDevices = 64;
DevState g_dev[kMaxDevices];

nmoe_status dev_state(DevState** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return NMOE_ERR_NO_DEVICE;
  }
  std::lock_guard<std::mutex> lk(g_mu);
  DevState& s = g_dev[dev];
  if (!s.ready) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
      cudaGetLastError();
      return NMOE_ERR_CUDA;
    }
    s.ok = (major == 10 && minor == 0);
    s.sm_count = sms;
    if (s.ok) {
      void* p = nullptr;
      if (cudaGetSymbolAddress(&p, nmoe_g_err_word) != cudaSuccess) {
        cudaGetLastError();
        return NMOE_ERR_CUDA;
      }
      s.err = static_cast<unsigned*>(p);
    }
    s.ready = true;
  }
  if (!s.ok) return NMOE_ERR_NO_DEVICE;
  *out = &s;
  return NMOE_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
size_t align256(size_t v) { return (v + 255) & ~size_t(255); }
size_t esize(nmoe_dtype dt) { return dt == NMOE_F32 ? 4 : 2; }

nmoe_options default_options() {
  nmoe_options o;
  nmoe_options_init(&o);
  return o;
}

// Sizes and enums shared by every entry point.
nmoe_status check_shape(int64_t T, int64_t d, int64_t E, int64_t F, int64_t C, int64_t n_seg,
                        nmoe_dtype dt, bool need_dF) {
  if (dt != NMOE_BF16 && dt != NMOE_F32) return NMOE_ERR_INVALID_ARG;
  if (T < 1 || T >= (int64_t(1) << 31)) return NMOE_ERR_INVALID_ARG;
  if (E < 1 || E > 256) return NMOE_ERR_INVALID_ARG;
  if (n_seg < 1 || n_seg > 65535 || T % n_seg != 0) return NMOE_ERR_INVALID_ARG;
  if (C < 1 || C > T / n_seg) return NMOE_ERR_INVALID_ARG;
  if (T / n_seg > nmoe::kSelectMaxRow) return NMOE_ERR_UNSUPPORTED;
  if (E * n_seg * C >= (int64_t(1) << 31)) return NMOE_ERR_INVALID_ARG;
  if (need_dF) {
    if (d < 1 || F < 1) return NMOE_ERR_INVALID_ARG;
    if (d % 8 != 0 || F % 8 != 0) return NMOE_ERR_UNSUPPORTED;
    if (d >= (int64_t(1) << 31) || F >= (int64_t(1) << 31)) return NMOE_ERR_INVALID_ARG;
  }
  return NMOE_OK;
}

Shape make_shape(int64_t T, int64_t d, int64_t E, int64_t F, int64_t C, int64_t n_seg) {
  Shape s;
  s.T = (int)T; s.d = (int)d; s.E = (int)E; s.F = (int)F; s.C = (int)C;
  s.n_seg = (int)n_seg; s.S = (int)(T / n_seg); s.Ce = (int)(n_seg * C);
  s.pdl = true;
  s.wait_ns = nmoe::kDefaultWaitNs;
  s.y_rows = (int64_t)s.E * s.Ce;
  return s;
}

// Bytes per element of the H and Y intermediates: fp32 layers and SPLIT bf16 layers
// use 4 (fp32, or a bf16 hi/lo pair), BF16 intermediates use 2.
size_t inter_size(nmoe_dtype dt, const nmoe_options& o) {
  return (dt == NMOE_F32 || o.intermediate == NMOE_INTERMEDIATE_SPLIT) ? 4 : 2;
}
size_t out_size(nmoe_dtype dt, const nmoe_options& o) {
  return (dt == NMOE_F32 || o.out_f32) ? 4 : 2;
}

struct Layout {
  size_t scores, scores_t, idx, gate, bnd, tok_ptr, tok_ent, ent_pos, H, Hs, Y, xin, xr, xout,
      total;
};

Layout make_layout(const Shape& s, nmoe_dtype dt, const nmoe_options& o) {
  Layout L;
  size_t off = 0;
  const size_t is = inter_size(dt, o);
  const size_t none = ~size_t(0);
  auto take = [&](size_t bytes) { size_t at = off; off = align256(off + bytes); return at; };
  L.scores = o.scores_out ? none : take(sizeof(float) * (size_t)s.T * s.E);
  L.scores_t = take(sizeof(float) * (size_t)s.T * s.E);
  L.idx = o.idx_out ? none : take(sizeof(int32_t) * (size_t)s.E * s.Ce);
  L.gate = take(sizeof(float) * (size_t)s.E * s.Ce);
  L.bnd = take(sizeof(int32_t) * nmoe::select_bound_entries(s));
  // with a shared expert every token has one more entry (and Y row): its shared row
  const size_t shared_rows = o.shared_w1 ? (size_t)s.T : 0;
  L.tok_ptr = take(sizeof(int32_t) * ((size_t)s.T + 1));
  L.tok_ent = take(sizeof(int32_t) * ((size_t)s.E * s.Ce + shared_rows));
  L.ent_pos = take(sizeof(int32_t) * (size_t)s.E * s.Ce);
  L.H = take(is * (size_t)s.E * s.Ce * s.F);
  L.Hs = o.shared_w1 ? take(is * (size_t)s.T * (size_t)o.shared_f) : none;
  L.Y = take(is * ((size_t)s.E * s.Ce + shared_rows) * s.d);
  L.xin = o.host_io ? take(esize(dt) * (size_t)s.T * s.d) : none;
  L.xr = o.host_io && o.router_x ? take(esize(dt) * (size_t)s.T * s.d) : none;
  L.xout = o.host_io ? take(out_size(dt, o) * (size_t)s.T * s.d) : none;
  L.total = off;
  return L;
}

nmoe_status options_ok(const nmoe_options& o) {
  if (o.score_fn != NMOE_SCORE_SOFTMAX && o.score_fn != NMOE_SCORE_SIGMOID)
    return NMOE_ERR_INVALID_ARG;
  if (o.combine != NMOE_COMBINE_RAW && o.combine != NMOE_COMBINE_NORMALIZED)
    return NMOE_ERR_INVALID_ARG;
  if (!isfinite(o.route_scale)) return NMOE_ERR_INVALID_ARG;
  if (o.router_bias && (reinterpret_cast<uintptr_t>(o.router_bias) & 3u))
    return NMOE_ERR_INVALID_ARG;
  if (o.scores_out && !aligned16(o.scores_out)) return NMOE_ERR_INVALID_ARG;
  if (o.idx_out && !aligned16(o.idx_out)) return NMOE_ERR_INVALID_ARG;
  if (o.workspace && (reinterpret_cast<uintptr_t>(o.workspace) & 255u))
    return NMOE_ERR_INVALID_ARG;
  if (o.intermediate != NMOE_INTERMEDIATE_SPLIT && o.intermediate != NMOE_INTERMEDIATE_BF16)
    return NMOE_ERR_INVALID_ARG;
  const int n_shared = (o.shared_w1 != nullptr) + (o.shared_w3 != nullptr) +
                       (o.shared_w2 != nullptr);
  if (n_shared != 0 && n_shared != 3) return NMOE_ERR_INVALID_ARG;
  if (n_shared == 3) {
    if (!aligned16(o.shared_w1) || !aligned16(o.shared_w3) || !aligned16(o.shared_w2))
      return NMOE_ERR_INVALID_ARG;
    if (o.shared_f < 1 || o.shared_f >= (int64_t(1) << 31)) return NMOE_ERR_INVALID_ARG;
    if (o.shared_f % 8 != 0) return NMOE_ERR_UNSUPPORTED;
  }
  if (o.gate2 && !o.residual) return NMOE_ERR_INVALID_ARG;
  const bool ep = o.expert_end > o.expert_begin || o.skip_combine;
  if (ep && (n_shared != 0 || o.residual != nullptr)) return NMOE_ERR_INVALID_ARG;
  if (o.expert_begin < 0 || o.expert_end < 0) return NMOE_ERR_INVALID_ARG;
  if (o.skip_combine && (o.workspace == nullptr || o.host_io)) return NMOE_ERR_INVALID_ARG;
  // a rank's partial rows are only a layer output after the exchange
  if (o.expert_end > o.expert_begin && !o.skip_combine) return NMOE_ERR_INVALID_ARG;
  if (o.residual && !aligned16(o.residual)) return NMOE_ERR_INVALID_ARG;
  if (o.gate2 && !aligned16(o.gate2)) return NMOE_ERR_INVALID_ARG;
  if (o.router_x && !o.host_io && !aligned16(o.router_x)) return NMOE_ERR_INVALID_ARG;
  return NMOE_OK;
}

}  // namespace

struct nmoe_trace {
  int max_calls = 0;
  int n = 0;
  std::vector<cudaEvent_t> ev;  // (NMOE_N_STAGES + 1) per call
};

namespace {

cudaEvent_t* trace_slot(nmoe_trace* tr) {
  if (!tr || tr->n >= tr->max_calls) return nullptr;
  return &tr->ev[(size_t)tr->n++ * (NMOE_N_STAGES + 1)];
}

nmoe_status forward_impl(const void* x, const void* W_r, const void* W1, const void* W3,
                         const void* W2, int64_t T, int64_t d, int64_t E, int64_t F, int64_t C,
                         void* out, cudaStream_t st, const nmoe_options& o) {
  nmoe_status v = check_shape(T, d, E, F, C, o.n_segments, o.dtype, true);
  if (v != NMOE_OK) return v;
  if ((v = options_ok(o)) != NMOE_OK) return v;
  // with skip_combine the call writes no output, and out may be NULL
  if (!x || !W_r || !W1 || !W3 || !W2 || (!out && !o.skip_combine))
    return NMOE_ERR_INVALID_ARG;
  if (!aligned16(W_r) || !aligned16(W1) || !aligned16(W3) || !aligned16(W2))
    return NMOE_ERR_INVALID_ARG;
  if (!o.host_io && (!aligned16(x) || (out && !aligned16(out)))) return NMOE_ERR_INVALID_ARG;
  if (x == out) return NMOE_ERR_INVALID_ARG;
  if (o.residual != nullptr && o.residual == out) return NMOE_ERR_INVALID_ARG;
  if (o.router_x != nullptr && o.router_x == out) return NMOE_ERR_INVALID_ARG;

  DevState* ds = nullptr;
  if ((v = dev_state(&ds)) != NMOE_OK) return v;
  Shape s = make_shape(T, d, E, F, C, o.n_segments);
  if (s.Ce > 65535 * 64) return NMOE_ERR_UNSUPPORTED;
  const bool has_shared = o.shared_w1 != nullptr;
  // the experts this call runs (all, or one rank's range under expert parallelism)
  const int e_lo = o.expert_end > o.expert_begin ? (int)o.expert_begin : 0;
  const int e_hi = o.expert_end > o.expert_begin ? (int)o.expert_end : (int)E;
  if (e_hi > E) return NMOE_ERR_INVALID_ARG;
  if (has_shared && (int64_t)s.E * s.Ce + s.T >= (int64_t(1) << 31)) return NMOE_ERR_INVALID_ARG;
  // per-stage events sit between the launches, so traced calls run without overlap
  s.pdl = o.trace == nullptr;
  if (o.wait_budget_ns != 0) s.wait_ns = o.wait_budget_ns;
  if (has_shared) s.y_rows += s.T;
  const Layout L = make_layout(s, o.dtype, o);

  char* ws = static_cast<char*>(o.workspace);
  bool own = false;
  if (!ws) {
    if (cudaMallocAsync(reinterpret_cast<void**>(&ws), L.total, st) != cudaSuccess) {
      cudaGetLastError();
      return NMOE_ERR_WORKSPACE;
    }
    own = true;
  } else if (o.workspace_bytes < L.total) {
    return NMOE_ERR_WORKSPACE;
  }

  float* scores = o.scores_out ? o.scores_out : reinterpret_cast<float*>(ws + L.scores);
  float* scores_t = reinterpret_cast<float*>(ws + L.scores_t);
  int32_t* idx = o.idx_out ? o.idx_out : reinterpret_cast<int32_t*>(ws + L.idx);
  float* gate = reinterpret_cast<float*>(ws + L.gate);
  int32_t* bnd = reinterpret_cast<int32_t*>(ws + L.bnd);
  int32_t* tok_ptr = reinterpret_cast<int32_t*>(ws + L.tok_ptr);
  int32_t* tok_ent = reinterpret_cast<int32_t*>(ws + L.tok_ent);
  int32_t* ent_pos = reinterpret_cast<int32_t*>(ws + L.ent_pos);
  void* H = ws + L.H;
  void* Y = ws + L.Y;
  // the shared expert: one "expert" over all T tokens in token order (identity row map,
  // weight 1), whose row of Y for token t is the first of t's span (tok_ptr[t])
  Shape sh = s;
  sh.E = 1; sh.F = (int)o.shared_f; sh.C = s.T; sh.n_seg = 1; sh.S = s.T; sh.Ce = s.T;
  void* Hs = has_shared ? static_cast<void*>(ws + L.Hs) : nullptr;
  void* Hs_lo = has_shared ? static_cast<void*>(ws + L.Hs + sizeof(uint16_t) * (size_t)s.T *
                                                               (size_t)o.shared_f)
                           : nullptr;
  const size_t xbytes = esize(o.dtype) * (size_t)s.T * s.d;
  const size_t obytes = out_size(o.dtype, o) * (size_t)s.T * s.d;
  const bool f32 = o.dtype == NMOE_F32;
  const bool split = !f32 && o.intermediate == NMOE_INTERMEDIATE_SPLIT;
  const bool y_f32 = f32 || split;
  const bool out_f32 = f32 || o.out_f32;

  const void* xd = x;
  const void* xrd = o.router_x ? o.router_x : x;  // what the router scores
  void* outd = out;
  cudaError_t e = cudaSuccess;
  if (o.host_io) {
    xd = ws + L.xin;
    outd = ws + L.xout;
    e = cudaMemcpyAsync(ws + L.xin, x, xbytes, cudaMemcpyHostToDevice, st);
    xrd = xd;
    if (o.router_x && e == cudaSuccess) {
      xrd = ws + L.xr;
      e = cudaMemcpyAsync(ws + L.xr, o.router_x, xbytes, cudaMemcpyHostToDevice, st);
    }
  }
  cudaEvent_t* ev = trace_slot(o.trace);
  auto mark = [&](int i) {
    if (ev && e == cudaSuccess) e = cudaEventRecord(ev[i], st);
  };
  mark(0);
  if (e == cudaSuccess) {
    if (o.dtype == NMOE_BF16 && nmoe::router_sm100_supported(s))
      e = nmoe::launch_router_sm100(xrd, W_r, s, o.score_fn, o.router_bias, scores, scores_t,
                                    ds->err, st);
    else
      e = nmoe::launch_router_simt(xrd, W_r, s, o.dtype, o.score_fn, o.router_bias, scores,
                                   scores_t, st);
  }
  mark(1);
  if (e == cudaSuccess)
    e = nmoe::launch_select(scores_t, s, idx, gate, bnd, ds->err, ds->sm_count, st);
  mark(2);
  // the expert GEMMs cover experts [e_lo, e_hi): their slice of idx, gate and ent_pos
  Shape sl = s;
  sl.E = e_hi - e_lo;
  const int64_t eoff = (int64_t)e_lo * s.Ce;
  const bool run_experts = sl.E > 0;
  const bool tc = !f32 && run_experts && nmoe::experts_sm100_supported(sl);
  // On the tensor-core path the gate/up GEMM's epilogue warps build the token lists
  // while their first accumulators fill (no CSR launch); otherwise the CSR kernel does.
  const bool fuse_csr = tc && nmoe::gemm1_sm100_fuses_csr(s, split);
  // A token that a single expert chose: its output is that expert's weighted row rounded
  // once, so the tensor-core down projection writes it straight to out and the combine
  // skips it (its row of Y is never written or read). Only for the plain layer output:
  // no shared expert, no residual, all experts on this GPU, combined here.
  const bool direct = tc && !has_shared && o.residual == nullptr && !o.skip_combine &&
                      e_lo == 0 && e_hi == (int)E;
  const nmoe::CsrArgs csr = nmoe::csr_args(idx, bnd, s, has_shared, tok_ptr, tok_ent, ent_pos,
                                           gate, o.combine, o.route_scale, direct, ds->err);
  if (e == cudaSuccess && !fuse_csr)
    e = nmoe::launch_csr(idx, bnd, s, has_shared, tok_ptr, tok_ent, ent_pos, gate, o.combine,
                         o.route_scale, direct, ds->err, st);
  mark(3);
  const bool tc_sh = has_shared && !f32 && nmoe::experts_sm100_supported(sh);
  if (has_shared && e == cudaSuccess)
    e = tc_sh ? nmoe::launch_gemm1_sm100(xd, nullptr, o.shared_w1, o.shared_w3, sh, split,
                                         false, Hs, Hs_lo, nullptr, ds->err, ds->sm_count, st)
              : nmoe::launch_gemm1_simt(xd, nullptr, o.shared_w1, o.shared_w3, sh, o.dtype,
                                        split, Hs, st);
  // SPLIT on the tensor cores: H_hi then H_lo, each [E*Ce, F] bf16; on the CUDA cores
  // (shapes the tcgen05 kernels do not take) H is one fp32 array of the same size.
  void* H_lo = static_cast<char*>(H) + sizeof(uint16_t) * (size_t)s.E * s.Ce * s.F;
  if (e == cudaSuccess && run_experts)
    e = tc ? nmoe::launch_gemm1_sm100(xd, idx + eoff, W1, W3, sl, split, o.tma_gather != 0, H,
                                      H_lo, fuse_csr ? &csr : nullptr, ds->err, ds->sm_count,
                                      st)
           : nmoe::launch_gemm1_simt(xd, idx + eoff, W1, W3, sl, o.dtype, split, H, st);
  mark(4);
  if (has_shared && e == cudaSuccess)
    e = tc_sh ? nmoe::launch_gemm2_sm100(Hs, Hs_lo, nullptr, tok_ptr, o.shared_w2, sh, split,
                                         Y, nullptr, false, ds->err, ds->sm_count, st)
              : nmoe::launch_gemm2_simt(Hs, nullptr, o.shared_w2, tok_ptr, sh, o.dtype, split,
                                        y_f32, Y, st);
  if (e == cudaSuccess && run_experts)
    e = tc ? nmoe::launch_gemm2_sm100(H, H_lo, gate + eoff, ent_pos + eoff, W2, sl, split, Y,
                                      direct ? outd : nullptr, out_f32, ds->err, ds->sm_count,
                                      st)
           : nmoe::launch_gemm2_simt(H, gate + eoff, W2, ent_pos + eoff, sl, o.dtype, split,
                                     y_f32, Y, st);
  mark(5);
  // the tensor-core down GEMM signals the combine only after its own wait (see
  // nmoe_internal.cuh), so the combine may read the token lists before its wait
  s.after_gemm2 = s.pdl && tc && run_experts;
  if (e == cudaSuccess && !o.skip_combine)
    e = nmoe::launch_combine(Y, tok_ptr, s, y_f32, out_f32, outd, o.residual, !f32, o.gate2,
                             direct, ds->err, ds->sm_count, st);
  mark(6);
  if (o.host_io && e == cudaSuccess)
    e = cudaMemcpyAsync(out, outd, obytes, cudaMemcpyDeviceToHost, st);
  if (own) {
    cudaError_t f = cudaFreeAsync(ws, st);
    if (e == cudaSuccess) e = f;
  }
  if (e != cudaSuccess) {
    cudaGetLastError();
    return NMOE_ERR_CUDA;
  }
  return NMOE_OK;
}

}  // namespace

extern "C" {

void nmoe_options_init(nmoe_options* o) {
  if (!o) return;
  o->dtype = NMOE_BF16;
  o->score_fn = NMOE_SCORE_SOFTMAX;
  o->combine = NMOE_COMBINE_RAW;
  o->route_scale = 1.0f;
  o->n_segments = 1;
  o->router_bias = nullptr;
  o->workspace = nullptr;
  o->workspace_bytes = 0;
  o->scores_out = nullptr;
  o->idx_out = nullptr;
  o->host_io = 0;
  o->trace = nullptr;
  o->intermediate = NMOE_INTERMEDIATE_SPLIT;
  o->out_f32 = 0;
  o->tma_gather = 0;
  o->shared_w1 = nullptr;
  o->shared_w3 = nullptr;
  o->shared_w2 = nullptr;
  o->shared_f = 0;
  o->residual = nullptr;
  o->gate2 = nullptr;
  o->expert_begin = 0;
  o->expert_end = 0;
  o->skip_combine = 0;
  o->router_x = nullptr;
  o->wait_budget_ns = 0;
}

nmoe_status nmoe_router(const void* x, const void* W_r, int64_t T, int64_t d, int64_t E,
                        nmoe_dtype dtype, nmoe_score_fn score_fn, const float* router_bias,
                        int64_t n_segments, float* scores, float* scores_t,
                        nmoe_stream_t stream) {
  nmoe_status v = check_shape(T, d, E, 1, 1, n_segments, dtype, false);
  if (v != NMOE_OK) return v;
  if (d < 1 || d >= (int64_t(1) << 31)) return NMOE_ERR_INVALID_ARG;
  if (d % 8 != 0) return NMOE_ERR_UNSUPPORTED;
  if (score_fn != NMOE_SCORE_SOFTMAX && score_fn != NMOE_SCORE_SIGMOID)
    return NMOE_ERR_INVALID_ARG;
  if (!x || !W_r || (!scores && !scores_t)) return NMOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(W_r)) return NMOE_ERR_INVALID_ARG;
  if ((scores && !aligned16(scores)) || (scores_t && !aligned16(scores_t)))
    return NMOE_ERR_INVALID_ARG;
  if (router_bias && (reinterpret_cast<uintptr_t>(router_bias) & 3u)) return NMOE_ERR_INVALID_ARG;
  DevState* ds = nullptr;
  if ((v = dev_state(&ds)) != NMOE_OK) return v;
  const Shape s = make_shape(T, d, E, 8, 1, n_segments);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (dtype == NMOE_BF16 && nmoe::router_sm100_supported(s) && scores && scores_t)
    e = nmoe::launch_router_sm100(x, W_r, s, score_fn, router_bias, scores, scores_t, ds->err,
                                  st);
  else
    e = nmoe::launch_router_simt(x, W_r, s, dtype, score_fn, router_bias, scores, scores_t, st);
  if (e != cudaSuccess) { cudaGetLastError(); return NMOE_ERR_CUDA; }
  return NMOE_OK;
}

nmoe_status nmoe_select(const float* scores_t, int64_t T, int64_t E, int64_t C,
                        int64_t n_segments, int32_t* idx, float* gate, int32_t* tok_ptr,
                        int32_t* tok_ent, nmoe_stream_t stream) {
  nmoe_status v = check_shape(T, 8, E, 8, C, n_segments, NMOE_F32, false);
  if (v != NMOE_OK) return v;
  if (!scores_t || !idx || !gate) return NMOE_ERR_INVALID_ARG;
  if ((tok_ptr == nullptr) != (tok_ent == nullptr)) return NMOE_ERR_INVALID_ARG;
  if (!aligned16(scores_t) || !aligned16(idx) || !aligned16(gate)) return NMOE_ERR_INVALID_ARG;
  if (tok_ptr && (!aligned16(tok_ptr) || !aligned16(tok_ent))) return NMOE_ERR_INVALID_ARG;
  DevState* ds = nullptr;
  if ((v = dev_state(&ds)) != NMOE_OK) return v;
  const Shape s = make_shape(T, 8, E, 8, C, n_segments);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // no scratch here: the CSR build searches idx instead of reading a boundary table
  cudaError_t e = nmoe::launch_select(scores_t, s, idx, gate, nullptr, ds->err, ds->sm_count, st);
  if (e == cudaSuccess && tok_ptr)
    e = nmoe::launch_csr(idx, nullptr, s, false, tok_ptr, tok_ent, nullptr, gate,
                         NMOE_COMBINE_RAW, 1.f, false, ds->err, st);
  if (e != cudaSuccess) { cudaGetLastError(); return NMOE_ERR_CUDA; }
  return NMOE_OK;
}

nmoe_status nmoe_forward(const void* x, const void* W_r, const void* W1, const void* W3,
                         const void* W2, int64_t T, int64_t d, int64_t E, int64_t F,
                         int64_t C, void* out, nmoe_stream_t stream) {
  return forward_impl(x, W_r, W1, W3, W2, T, d, E, F, C, out,
                      static_cast<cudaStream_t>(stream), default_options());
}

nmoe_status nmoe_forward_ex(const void* x, const void* W_r, const void* W1, const void* W3,
                            const void* W2, int64_t T, int64_t d, int64_t E, int64_t F,
                            int64_t C, void* out, nmoe_stream_t stream,
                            const nmoe_options* opts) {
  return forward_impl(x, W_r, W1, W3, W2, T, d, E, F, C, out,
                      static_cast<cudaStream_t>(stream), opts ? *opts : default_options());
}

nmoe_status nmoe_workspace_offsets(int64_t T, int64_t d, int64_t E, int64_t F, int64_t C,
                                   const nmoe_options* opts, size_t* y_offset,
                                   size_t* tok_ptr_offset, size_t* tok_ent_offset) {
  const nmoe_options o = opts ? *opts : default_options();
  if (check_shape(T, d, E, F, C, o.n_segments, o.dtype, true) != NMOE_OK)
    return NMOE_ERR_INVALID_ARG;
  const Layout L = make_layout(make_shape(T, d, E, F, C, o.n_segments), o.dtype, o);
  if (y_offset) *y_offset = L.Y;
  if (tok_ptr_offset) *tok_ptr_offset = L.tok_ptr;
  if (tok_ent_offset) *tok_ent_offset = L.tok_ent;
  return NMOE_OK;
}

nmoe_status nmoe_ep_rows(const int32_t* tok_ptr, const int32_t* tok_ent, int64_t T, int64_t E,
                         int64_t Ce, int64_t t_begin, int64_t t_end, int64_t e_begin,
                         int64_t e_end, int32_t* rows, int64_t capacity, int32_t* count,
                         nmoe_stream_t stream) {
  if (!tok_ptr || !tok_ent || !count) return NMOE_ERR_INVALID_ARG;
  if (T < 1 || E < 1 || Ce < 1 || E * Ce >= (int64_t(1) << 31)) return NMOE_ERR_INVALID_ARG;
  if (t_begin < 0 || t_end < t_begin || t_end > T) return NMOE_ERR_INVALID_ARG;
  if (e_begin < 0 || e_end < e_begin || e_end > E) return NMOE_ERR_INVALID_ARG;
  if (capacity < 0 || capacity >= (int64_t(1) << 31) || (capacity > 0 && !rows))
    return NMOE_ERR_INVALID_ARG;
  DevState* ds = nullptr;
  nmoe_status v = dev_state(&ds);
  if (v != NMOE_OK) return v;
  if (nmoe::launch_ep_rows(tok_ptr, tok_ent, (int)E, (int)Ce, (int)t_begin, (int)t_end,
                           (int)e_begin, (int)e_end, rows, (int)capacity, count, ds->err,
                           static_cast<cudaStream_t>(stream)) != cudaSuccess) {
    cudaGetLastError();
    return NMOE_ERR_CUDA;
  }
  return NMOE_OK;
}

namespace {
nmoe_status rows_copy(const void* src, const int32_t* rows, int64_t n, int64_t row_bytes,
                      void* dst, bool gather, nmoe_stream_t stream) {
  if (n < 0 || row_bytes < 16 || row_bytes % 16 != 0 || row_bytes / 16 > INT32_MAX)
    return NMOE_ERR_INVALID_ARG;
  if (n > 0 && (!src || !rows || !dst || !aligned16(src) || !aligned16(dst)))
    return NMOE_ERR_INVALID_ARG;
  DevState* ds = nullptr;
  nmoe_status v = dev_state(&ds);
  if (v != NMOE_OK) return v;
  if (nmoe::launch_rows_copy(src, rows, n, row_bytes, dst, gather, ds->sm_count,
                             static_cast<cudaStream_t>(stream)) != cudaSuccess) {
    cudaGetLastError();
    return NMOE_ERR_CUDA;
  }
  return NMOE_OK;
}
}  // namespace

nmoe_status nmoe_rows_gather(const void* src, const int32_t* rows, int64_t n, int64_t row_bytes,
                             void* dst, nmoe_stream_t stream) {
  return rows_copy(src, rows, n, row_bytes, dst, true, stream);
}

nmoe_status nmoe_rows_scatter(const void* src, const int32_t* rows, int64_t n,
                              int64_t row_bytes, void* dst, nmoe_stream_t stream) {
  return rows_copy(src, rows, n, row_bytes, dst, false, stream);
}

nmoe_status nmoe_combine_tokens(const void* Y, const int32_t* tok_ptr, int64_t T, int64_t d,
                                int64_t t_begin, int64_t t_end, nmoe_dtype y_dtype,
                                nmoe_dtype out_dtype, void* out, nmoe_stream_t stream) {
  if (!Y || !tok_ptr || !out) return NMOE_ERR_INVALID_ARG;
  if (T < 1 || T >= (int64_t(1) << 31) || d < 8 || d >= (int64_t(1) << 31))
    return NMOE_ERR_INVALID_ARG;
  if (d % 8 != 0) return NMOE_ERR_UNSUPPORTED;
  if (t_begin < 0 || t_end < t_begin || t_end > T) return NMOE_ERR_INVALID_ARG;
  if ((y_dtype != NMOE_F32 && y_dtype != NMOE_BF16) ||
      (out_dtype != NMOE_F32 && out_dtype != NMOE_BF16))
    return NMOE_ERR_INVALID_ARG;
  if (!aligned16(Y) || !aligned16(out)) return NMOE_ERR_INVALID_ARG;
  if (t_end == t_begin) return NMOE_OK;
  DevState* ds = nullptr;
  nmoe_status v = dev_state(&ds);
  if (v != NMOE_OK) return v;
  // the token range as a layer of its own: its tok_ptr entries, its output rows
  Shape s = make_shape(t_end - t_begin, d, 1, 8, 1, 1);
  s.pdl = false;
  s.y_rows = int64_t(1) << 40;  // Y's row count is not passed: only the order is checked
  if (nmoe::launch_combine(Y, tok_ptr + t_begin, s, y_dtype == NMOE_F32,
                           out_dtype == NMOE_F32, out, nullptr, false, nullptr, false, ds->err,
                           ds->sm_count, static_cast<cudaStream_t>(stream)) != cudaSuccess) {
    cudaGetLastError();
    return NMOE_ERR_CUDA;
  }
  return NMOE_OK;
}

int nmoe_kernels_per_call(int64_t T, int64_t d, int64_t E, int64_t F, int64_t C,
                          const nmoe_options* opts) {
  const nmoe_options o = opts ? *opts : default_options();
  if (check_shape(T, d, E, F, C, o.n_segments, o.dtype, true) != NMOE_OK) return 0;
  const Shape s = make_shape(T, d, E, F, C, o.n_segments);
  const bool f32 = o.dtype == NMOE_F32;
  const bool split = !f32 && o.intermediate == NMOE_INTERMEDIATE_SPLIT;
  Shape sl = s;
  if (o.expert_end > o.expert_begin) sl.E = (int)(o.expert_end - o.expert_begin);
  const bool run_experts = sl.E > 0;
  const bool tc = !f32 && run_experts && nmoe::experts_sm100_supported(sl);
  const bool fuse_csr = tc && nmoe::gemm1_sm100_fuses_csr(s, split);
  // router, select, (CSR), gate/up, down, (combine); two more for a shared expert
  return 2 + (fuse_csr ? 0 : 1) + (run_experts ? 2 : 0) + (o.skip_combine ? 0 : 1) +
         (o.shared_w1 != nullptr ? 2 : 0);
}

size_t nmoe_workspace_size(int64_t T, int64_t d, int64_t E, int64_t F, int64_t C,
                           const nmoe_options* opts) {
  const nmoe_options o = opts ? *opts : default_options();
  if (check_shape(T, d, E, F, C, o.n_segments, o.dtype, true) != NMOE_OK) return 0;
  return make_layout(make_shape(T, d, E, F, C, o.n_segments), o.dtype, o).total;
}

nmoe_status nmoe_get_last_error(nmoe_stream_t stream) {
  DevState* ds = nullptr;
  nmoe_status v = dev_state(&ds);
  if (v != NMOE_OK) return v;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) {
    cudaGetLastError();
    return NMOE_ERR_CUDA;
  }
  unsigned word = 0;
  if (cudaMemcpy(&word, ds->err, sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess) {
    cudaGetLastError();
    return NMOE_ERR_CUDA;
  }
  if (word != 0 && cudaMemset(ds->err, 0, sizeof(unsigned)) != cudaSuccess) {
    cudaGetLastError();
    return NMOE_ERR_CUDA;
  }
  if (word & nmoe::kErrTimeout) return NMOE_ERR_TIMEOUT;
  if (word & nmoe::kErrDeviceCheck) return NMOE_ERR_DEVICE_CHECK;
  return NMOE_OK;
}

const char* nmoe_status_str(nmoe_status s) {
  switch (s) {
    case NMOE_OK: return "ok";
    case NMOE_ERR_INVALID_ARG: return "invalid argument";
    case NMOE_ERR_UNSUPPORTED: return "unsupported size or option";
    case NMOE_ERR_WORKSPACE: return "workspace too small or allocation failed";
    case NMOE_ERR_CUDA: return "CUDA error";
    case NMOE_ERR_TIMEOUT: return "device-side wait timed out";
    case NMOE_ERR_DEVICE_CHECK: return "device-side check failed";
    case NMOE_ERR_NO_DEVICE: return "no sm_100 device is current";
  }
  return "unknown status";
}

nmoe_status nmoe_trace_create(int max_calls, nmoe_trace** out) {
  if (!out || max_calls < 1) return NMOE_ERR_INVALID_ARG;
  nmoe_trace* tr = new (std::nothrow) nmoe_trace();
  if (!tr) return NMOE_ERR_WORKSPACE;
  tr->max_calls = max_calls;
  tr->ev.assign((size_t)max_calls * (NMOE_N_STAGES + 1), nullptr);
  for (auto& e : tr->ev) {
    if (cudaEventCreate(&e) != cudaSuccess) {
      cudaGetLastError();
      nmoe_trace_destroy(tr);
      return NMOE_ERR_CUDA;
    }
  }
  *out = tr;
  return NMOE_OK;
}

nmoe_status nmoe_trace_read(nmoe_trace* tr, double* stage_ms, int* n_calls) {
  if (!tr || !stage_ms) return NMOE_ERR_INVALID_ARG;
  for (int i = 0; i < NMOE_N_STAGES; ++i) stage_ms[i] = 0.0;
  for (int c = 0; c < tr->n; ++c) {
    cudaEvent_t* ev = &tr->ev[(size_t)c * (NMOE_N_STAGES + 1)];
    if (cudaEventSynchronize(ev[NMOE_N_STAGES]) != cudaSuccess) {
      cudaGetLastError();
      return NMOE_ERR_CUDA;
    }
    for (int i = 0; i < NMOE_N_STAGES; ++i) {
      float ms = 0.f;
      if (cudaEventElapsedTime(&ms, ev[i], ev[i + 1]) != cudaSuccess) {
        cudaGetLastError();
        return NMOE_ERR_CUDA;
      }
      stage_ms[i] += ms;
    }
  }
  if (n_calls) *n_calls = tr->n;
  return NMOE_OK;
}

nmoe_status nmoe_trace_reset(nmoe_trace* tr) {
  if (!tr) return NMOE_ERR_INVALID_ARG;
  tr->n = 0;
  return NMOE_OK;
}

void nmoe_trace_destroy(nmoe_trace* tr) {
  if (!tr) return;
  for (auto& e : tr->ev)
    if (e) cudaEventDestroy(e);
  delete tr;
}

const char* nmoe_stage_name(int stage) {
  static const char* names[NMOE_N_STAGES] = {"router", "select", "csr", "gemm1_swiglu",
                                             "gemm2_scale", "combine"};
  return (stage >= 0 && stage < NMOE_N_STAGES) ? names[stage] : "unknown";
}

const char* nmoe_build_info(void) {
  return "nmoe sm_100a: router tcgen05(bf16)/simt(fp32); select radix; token lists in the "
         "gate/up GEMM's epilogue warps (own kernel when too many experts); experts tcgen05 with "
         "cp.async row gather (TMA gather4 option) and TMA weights (bf16)/simt(fp32); "
         "combine fixed-order"
#ifdef NMOE_DEBUG
         "; debug checks (gathered indices, row positions, token-list spans)"
#endif
      ;
}

}  // extern "C"
