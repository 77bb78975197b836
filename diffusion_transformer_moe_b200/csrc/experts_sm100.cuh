// Grouped SwiGLU expert GEMMs on the 5th-generation tensor cores (tcgen05 + TMEM + TMA).
#pragma once
#include "nmoe_internal.cuh"

namespace nmoe {

// True when the tcgen05 kernels cover this shape (bf16 only).
bool experts_sm100_supported(const Shape& s);

// H[e, s, :] = silu(x[idx[e,s]] W1_e) * (x[idx[e,s]] W3_e), the rows gathered from x by
// cp.async (default) or by TMA tile::gather4 (tma_gather).
// split: H is written as bf16 hi = bf16(h) to H_hi and lo = bf16(h - hi) to H_lo;
// otherwise only H_hi (bf16(h)) is written.
// idx NULL: row s of the single expert is token s (the shared expert); gate NULL in
// gemm2: weight 1. csr (may be NULL; only if gemm1_sm100_fuses_csr) also builds the
// token lists inside the gate/up GEMM, in place of the CSR kernel.
struct CsrArgs;
bool gemm1_sm100_fuses_csr(const Shape& s, bool split);
cudaError_t launch_gemm1_sm100(const void* x, const int32_t* idx, const void* W1,
                               const void* W3, const Shape& s, bool split, bool tma_gather,
                               void* H_hi, void* H_lo, const CsrArgs* csr, unsigned* err,
                               int sm_count, cudaStream_t st);

// True when launch_gemm2_sm100 runs this shape on CTA pairs (at least 256 rows per expert,
// d a multiple of 64, and 2-CTA clusters of the pair kernel fit).
bool gemm2_sm100_uses_pairs(const Shape& s, bool split, int sm_count);

// Row e*Ce + s of H W2_e, times gate[e, s], goes to Y row ent_pos[e*Ce + s]; a
// negative position -(t + 1) sends it instead to row t of out_direct (fp32 if
// out_direct_f32, else bf16), rounded once (the token's only entry).
cudaError_t launch_gemm2_sm100(const void* H_hi, const void* H_lo, const float* gate,
                               const int32_t* ent_pos, const void* W2, const Shape& s,
                               bool split, void* Y, void* out_direct, bool out_direct_f32,
                               unsigned* err, int sm_count, cudaStream_t st);

}  // namespace nmoe
