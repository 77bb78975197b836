// Internal declarations shared by the CUDA translation units of libnmoe.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include <utility>

#include "nmoe.h"

namespace nmoe {

// Bits of the per-device error word (see nmoe_get_last_error).
constexpr unsigned kErrDeviceCheck = 1u;
constexpr unsigned kErrTimeout = 2u;

// The debug build (-DNMOE_DEBUG, libnmoe_debug.so) adds index and span checks to the
// kernels: a gathered token index outside x, a down-projection row position outside Y,
// a token-list span that runs backwards or outside Y. A failed check sets
// kErrDeviceCheck and skips the access it guards (no trap); the release build compiles
// the checks out.
#ifdef NMOE_DEBUG
constexpr bool kDebugChecks = true;
#else
constexpr bool kDebugChecks = false;
#endif

__host__ __device__ inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }
template <typename T> __device__ __forceinline__ T from_f32(float v);
template <> __device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) {
  return __float2bfloat16_rn(v);
}

// Programmatic dependent launch. Every kernel of the layer lets the next kernel on the
// stream start its prologue early (launch_dependents, issued by every thread at entry)
// and waits for the previous grid's memory (wait) before its first global access. The
// tensor-core down GEMM is the exception: it issues launch_dependents only after its own
// wait, so the kernel after it starts only once every earlier kernel of the call (and
// whatever ran before the call) has completed, and may read their outputs before its own
// wait (the combine reads its token lists there).
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Raises a kernel's dynamic shared-memory limit on the current device to at least
// `bytes`, once per (kernel, device, larger size). The default limit counts the
// kernel's static shared memory against the same 48 KB, so every launch with dynamic
// shared memory goes through here, not only those asking for more than 48 KB.
cudaError_t set_smem_limit(const void* kernel, size_t bytes);

// The driver's cuTensorMapEncodeTiled (cast to its PFN type by the caller), or NULL when the
// driver does not provide it; looked up once per process, safe from several host threads.
void* tensor_map_encoder();

// Launch with programmatic stream serialization (pdl) and an optional 1-D cluster.
template <typename... KArgs, typename... Args>
cudaError_t launch_kernel(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                          cudaStream_t st, bool pdl, unsigned cluster_x, Args&&... args) {
  if (smem > 0) {
    cudaError_t e = set_smem_limit(reinterpret_cast<const void*>(kernel), smem);
    if (e != cudaSuccess) return e;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  unsigned n = 0;
  if (pdl) {
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
  }
  if (cluster_x > 1) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = cluster_x;
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

// Shapes of one layer call, already validated on the host.
struct Shape {
  int T;         // tokens
  int d;         // model dim
  int E;         // experts
  int F;         // expert hidden dim
  int C;         // capacity per segment
  int n_seg;     // segments
  int S;         // tokens per segment = T / n_seg
  int Ce;        // entries per expert = n_seg * C
  bool pdl;      // launch with programmatic dependent launch
  uint64_t wait_ns;  // budget of each bounded device-side wait (nmoe_options)
  int64_t y_rows;    // rows of the layer's Y (all experts' entries, plus the shared rows)
  // The previous launch on the stream is the tensor-core down GEMM with programmatic
  // dependent launch (it signals its dependents only after its own wait).
  bool after_gemm2 = false;
};

// Budget of a device-side wait when the caller sets none: far beyond any wait of a
// healthy call (the longest are a few microseconds).
constexpr uint64_t kDefaultWaitNs = 2000000000ull;

// Launchers. Each returns the launch status (cudaGetLastError after the launch).
cudaError_t launch_router_simt(const void* x, const void* W_r, const Shape& s, nmoe_dtype dt,
                               nmoe_score_fn fn, const float* bias, float* scores,
                               float* scores_t, cudaStream_t st);

// Longest segment (tokens per expert row) the selection takes: its per-row bitmaps live
// in shared memory.
constexpr int kSelectMaxRow = 1 << 19;

// bnd (may be NULL) receives the block boundary table the CSR build reads: for every
// block of 32 tokens b and expert e, bnd[b*E + e] = number of e's entries whose token
// comes before the block; select_bound_entries(s) int32 entries.
size_t select_bound_entries(const Shape& s);
cudaError_t launch_select(const float* scores_t, const Shape& s, int32_t* idx, float* gate,
                          int32_t* bnd, unsigned* err, int sm_count, cudaStream_t st);

// bnd: the table launch_select wrote, or NULL to search idx instead.
// combine == NMOE_COMBINE_NORMALIZED rewrites gate[] in place to
// route_scale * gate / (sum of the token's gates). ent_pos (may be NULL) receives, for
// each entry e*Ce + slot, its index in the token-major order of tok_ent, or with
// `direct` -(t + 1) for the one entry of a token t that a single expert chose. With
// `shared`, every token's span starts with one more entry, its shared-expert row
// (tok_ent value E*Ce + t), so tok_ptr[T] = E*Ce + T.
cudaError_t launch_csr(const int32_t* idx, const int32_t* bnd, const Shape& s, bool shared,
                       int32_t* tok_ptr, int32_t* tok_ent, int32_t* ent_pos, float* gate,
                       nmoe_combine combine, float route_scale, bool direct, unsigned* err,
                       cudaStream_t st);
// The same arguments, for a kernel that builds the lists itself (csr_block.cuh).
struct CsrArgs;
CsrArgs csr_args(const int32_t* idx, const int32_t* bnd, const Shape& s, bool shared,
                 int32_t* tok_ptr, int32_t* tok_ent, int32_t* ent_pos, float* gate,
                 nmoe_combine combine, float route_scale, bool direct, unsigned* err);

// CUDA-core expert GEMMs. dt is the type of x and the weights; h_f32 / y_f32 select
// fp32 (else dt) for the H and Y intermediates.
// idx NULL: row s of the single expert is token s (the shared expert).
cudaError_t launch_gemm1_simt(const void* x, const int32_t* idx, const void* W1, const void* W3,
                              const Shape& s, nmoe_dtype dt, bool h_f32, void* H,
                              cudaStream_t st);

// Row e*Ce + s of the product goes to Y row ent_pos[e*Ce + s] (token-major order);
// gate NULL: weight 1.
cudaError_t launch_gemm2_simt(const void* H, const float* gate, const void* W2,
                              const int32_t* ent_pos, const Shape& s, nmoe_dtype dt, bool h_f32,
                              bool y_f32, void* Y, cudaStream_t st);

// out[t] = sum of Y rows tok_ptr[t] .. tok_ptr[t+1]-1 (token-major Y, ascending expert);
// Y is fp32 if y_f32 (else bf16), out fp32 if out_f32.
// With residual (x's dtype: bf16 if res_bf16, else fp32), out[t] = residual[t] +
// tanh(clamp(gate2[t / S], -2, 2)) * (that sum), gate2 NULL meaning a gate of 1.
// skip_single: tokens with exactly one row were written by the down projection (their
// rows of Y were never written): neither read nor stored here.
cudaError_t launch_combine(const void* Y, const int32_t* tok_ptr, const Shape& s, bool y_f32,
                           bool out_f32, void* out, const void* residual, bool res_bf16,
                           const float* gate2, bool skip_single, unsigned* err, int sm_count,
                           cudaStream_t st);

// Expert parallelism (ep.cu): rows[0 .. *count) = the token-major rows of tokens
// [t_begin, t_end) whose expert is in [e_begin, e_end), ascending, then -1 up to
// `capacity`; row gather/scatter (rows < 0 are skipped).
cudaError_t launch_ep_rows(const int32_t* tok_ptr, const int32_t* tok_ent, int E, int Ce,
                           int t_begin, int t_end, int e_begin, int e_end, int32_t* rows,
                           int capacity, int32_t* count, unsigned* err, cudaStream_t st);
cudaError_t launch_rows_copy(const void* src, const int32_t* rows, int64_t n, int64_t row_bytes,
                             void* dst, bool gather, int sm_count, cudaStream_t st);

}  // namespace nmoe
