/*
 * nmoe.h — C ABI of the expert-choice MoE feed-forward layer for NVIDIA B200 (sm_100a).
 *
 * The layer is the MoE FFN of NucleusMoE-Image's single-stream DiT block, described in
 * "Diffusers 中 NucleusMoE-Image 文生图流水线：单流 DiT + MoE 专家层 + Qwen3-VL 文本编码的
 * 全链路解析" (trdm.cn), section 6.2 ("expert-choice routing + shared expert") and the
 * packed SwiGLU experts of section 6:
 *   1. a gate Linear scores every token against every expert (softmax over the experts
 *      of a token by default, sigmoid as an option);
 *   2. every expert chooses its own top-C tokens (expert choice, so each expert gets
 *      exactly C tokens; ties go to the lower token index);
 *   3. every expert runs its SwiGLU FFN y = (silu(x W1_e) * (x W3_e)) W2_e on its rows;
 *   4. each token sums the weighted outputs of the experts that chose it, in ascending
 *      expert order (a fixed, atomic-free order); a token no expert chose outputs 0.
 *
 * Conventions for every entry point
 *   - Pointers are DEVICE pointers unless stated otherwise; all arrays are dense,
 *     row-major and 16-byte aligned. The caller owns every buffer; the library keeps
 *     no pointer after a call returns.
 *   - Work is enqueued asynchronously on `stream` (a cudaStream_t; NULL = legacy default
 *     stream). Inputs must stay valid, and outputs untouched, until the stream has
 *     passed the call. Outputs must not alias inputs.
 *   - Argument checks run on the host before anything is enqueued; on failure nothing
 *     is enqueued and the status says why. Faults found on the device (the debug
 *     checks, a bounded wait that ran out) are recorded in a per-device error word and
 *     reported by nmoe_get_last_error().
 *   - No CPU fallback exists: every step runs in this library's CUDA kernels.
 *   - Sizes: 1 <= E <= 256, 1 <= C <= T / n_segments, T < 2^31, E * n_segments * C
 *     < 2^31, d and F multiples of 8 (else NMOE_ERR_INVALID_ARG or, for the multiples,
 *     NMOE_ERR_UNSUPPORTED). T / n_segments <= 2^19 tokens per segment
 *     (NMOE_ERR_UNSUPPORTED above: the selection keeps a segment's bitmaps on chip).
 */
#ifndef NMOE_H_
#define NMOE_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define NMOE_API __attribute__((visibility("default")))
#else
#define NMOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  NMOE_OK = 0,
  NMOE_ERR_INVALID_ARG = 1,   /* a size, pointer or alignment the ABI forbids */
  NMOE_ERR_UNSUPPORTED = 2,   /* valid request the library does not implement */
  NMOE_ERR_WORKSPACE = 3,     /* caller workspace too small, or allocation failed */
  NMOE_ERR_CUDA = 4,          /* a CUDA runtime call or kernel launch failed */
  NMOE_ERR_TIMEOUT = 5,       /* a bounded device-side wait ran out */
  NMOE_ERR_DEVICE_CHECK = 6,  /* a device-side check failed (NaN score, bad index) */
  NMOE_ERR_NO_DEVICE = 7      /* no sm_100 device is current */
} nmoe_status;

typedef enum { NMOE_BF16 = 0, NMOE_F32 = 1 } nmoe_dtype;

/* Score function (section 6.2: "sigmoid (optional) or softmax"). */
typedef enum { NMOE_SCORE_SOFTMAX = 0, NMOE_SCORE_SIGMOID = 1 } nmoe_score_fn;

/* Combine weight (section 6.2): RAW = the token's score for the expert; NORMALIZED =
 * route_scale * score / (sum of the token's scores over the experts that chose it). */
typedef enum { NMOE_COMBINE_RAW = 0, NMOE_COMBINE_NORMALIZED = 1 } nmoe_combine;

/* Storage of the two intermediates of bf16 layers, H = SwiGLU(x W1, x W3) [E, C, F]
 * and Y = gate * (H W2) [E, C, d]:
 *   SPLIT (default): H is kept as two bf16 arrays hi = bf16(h), lo = bf16(h - hi)
 *     (~16 significant bits; the down projection runs both halves into one fp32
 *     accumulator) and Y in fp32, so that before the final rounding the output stays
 *     within 5e-2 absolute of the exact result even for tokens whose outputs reach
 *     |y| ~ 100;
 *   BF16: H and Y in plain bf16, as a bf16 framework would store them; ~10% fewer
 *     bytes at d = 2048, F = 1024, but large-magnitude tokens drift by ~0.1-0.2.
 * fp32 layers keep both intermediates in fp32. */
typedef enum { NMOE_INTERMEDIATE_SPLIT = 0, NMOE_INTERMEDIATE_BF16 = 1 } nmoe_intermediate;

/* A cudaStream_t, passed as an opaque pointer so this header needs no CUDA header. */
typedef void* nmoe_stream_t;

/* Stages of the layer, in launch order (for nmoe_trace). */
enum {
  NMOE_STAGE_ROUTER = 0,   /* router GEMM + score function */
  NMOE_STAGE_SELECT = 1,   /* per-expert top-C */
  NMOE_STAGE_CSR = 2,      /* token -> (expert, slot) lists */
  NMOE_STAGE_GEMM1 = 3,    /* gathered rows x [W1|W3] + SwiGLU */
  NMOE_STAGE_GEMM2 = 4,    /* H x W2, scaled by the combine weight */
  NMOE_STAGE_COMBINE = 5,  /* per-token fixed-order sum */
  NMOE_N_STAGES = 6
};

/* Opaque per-stage timer: CUDA events recorded around each stage of nmoe_forward_ex. */
typedef struct nmoe_trace nmoe_trace;

typedef struct nmoe_options {
  nmoe_dtype dtype;          /* type of x, W_*, out (and of the H, Y intermediates) */
  nmoe_score_fn score_fn;    /* default NMOE_SCORE_SOFTMAX */
  nmoe_combine combine;      /* default NMOE_COMBINE_RAW */
  float route_scale;         /* NORMALIZED only (the page's default is 2.5) */
  int64_t n_segments;        /* >= 1: tokens form n_segments equal groups (samples);
                                every expert takes C tokens from each group */
  const float* router_bias;  /* NULL, or device fp32 [n_segments, E] added to the
                                logits of every token of a group (the page's timestep
                                half of cat([timestep, hidden]) @ W_gate) */
  void* workspace;           /* NULL: allocated stream-ordered per call; else device
                                memory of >= nmoe_workspace_size() bytes, 256-B aligned */
  size_t workspace_bytes;
  float* scores_out;         /* NULL, or device fp32 [T, E]: the router scores */
  int32_t* idx_out;          /* NULL, or device int32 [E, n_segments*C]: chosen tokens */
  int host_io;               /* nonzero: x is a HOST pointer and out a HOST pointer
                                (pinned memory recommended); the call copies x in and
                                out back on `stream`; weights stay on the device */
  nmoe_trace* trace;         /* NULL, or a timer to record per-stage events into */
  nmoe_intermediate intermediate;  /* bf16 layers: storage of H and Y (default SPLIT) */
  int out_f32;               /* nonzero: out is fp32 even when dtype is bf16 */
  int tma_gather;            /* nonzero: the gate/up GEMM fetches its token rows with TMA
                                tile::gather4 instead of cp.async (about 2x slower on
                                B200; kept for comparison) */
  /* Shared expert (section 6.2: one SwiGLU feed-forward that every token goes through;
   * the routed, weighted outputs are added onto its output). All NULL: none. Otherwise
   * device arrays in `dtype`: shared_w1, shared_w3 [d, shared_f], shared_w2
   * [shared_f, d], row-major, 16-byte aligned; shared_f a multiple of 8 (else
   * NMOE_ERR_UNSUPPORTED). The page does not give the width; the caller does. */
  const void* shared_w1;
  const void* shared_w3;
  const void* shared_w2;
  int64_t shared_f;
  /* Gated residual of the surrounding block (section 6.3: the modulation gates are
   * clamped to [-2, 2] and passed through tanh). NULL: out = the layer output. Else a
   * device array [T, d] in `dtype` (it may be x; it must not overlap out), and
   *   out = residual + tanh(clamp(gate2[segment], -2, 2)) * (layer output),
   * with gate2 NULL (a gate of 1) or device fp32 [n_segments, d], 16-byte aligned. */
  const void* residual;
  const float* gate2;
  /* Expert parallelism (no counterpart on the pages; an exact sharding of the layer over
   * GPUs, one rank per contiguous range of experts). expert_end > expert_begin: the
   * expert GEMMs run for experts [expert_begin, expert_end) only, W1, W3 and W2 then
   * holding just those experts ([expert_end - expert_begin, ...]); the router, selection
   * and token lists still cover all E experts and every token. skip_combine: the call
   * stops after the down projection and leaves its rows (token-major positions, see
   * nmoe_workspace_offsets) in the workspace, which the caller must then provide; the
   * nmoe_ep_rows / nmoe_rows_gather / nmoe_rows_scatter / nmoe_combine_tokens calls
   * finish the layer. Not combinable with a shared expert or residual. */
  int64_t expert_begin;
  int64_t expert_end;
  int skip_combine;
  /* Separate router input (section 6.2: the gate reads the unmodulated hidden states,
   * concatenated with the timestep, while the experts transform the block's modulated
   * input). NULL: the router scores x. Else [T, d] in `dtype`, 16-byte aligned, not
   * overlapping out: the router scores router_x and the experts still gather their rows
   * from x (with router_bias carrying the timestep half, this is the page's gate
   * exactly). With host_io it is a HOST pointer, copied in like x. */
  const void* router_x;
  /* Longest time, in nanoseconds, that any single device-side wait of the tensor-core
   * kernels (a pipeline barrier between their copy, MMA and epilogue roles) may take
   * before the kernel gives up: it then stops issuing work, lets its copies and MMAs in
   * flight finish, frees its tensor memory, returns, and sets the error word that
   * nmoe_get_last_error() reports as NMOE_ERR_TIMEOUT; the call's outputs are then
   * undefined. 0 = the default of 2 s, far beyond any wait of a healthy call. A tiny
   * value makes a wait give up on purpose (the failure path is tested that way). */
  uint64_t wait_budget_ns;
} nmoe_options;

/* Fills `o` with the defaults: bf16, softmax, raw combine, route_scale 1, one segment,
 * no bias, internal workspace, no extra outputs, device I/O, no trace, SPLIT
 * intermediates, out in the input dtype, no shared expert or residual, all experts, the
 * router scoring x, the default wait budget. */
NMOE_API void nmoe_options_init(nmoe_options* o);

/* Router (section 6.2 "gate = Linear(..., num_experts, bias=False)", then softmax over
 * the experts of each token, or sigmoid).
 *   x [T, d] (dtype), W_r [d, E] (dtype), router_bias NULL or fp32 [n_segments, E].
 *   scores [T, E] fp32 and scores_t [E, T] fp32 (the same values, expert-major; either
 *   may be NULL but not both). Logits accumulate in fp32. */
NMOE_API nmoe_status nmoe_router(const void* x, const void* W_r, int64_t T, int64_t d, int64_t E,
                        nmoe_dtype dtype, nmoe_score_fn score_fn, const float* router_bias,
                        int64_t n_segments, float* scores, float* scores_t,
                        nmoe_stream_t stream);

/* Expert-choice selection (section 6.2: each expert takes its top `capacity` tokens)
 * and the token lists the combine needs.
 *   scores_t [E, T] fp32 (non-negative: softmax or sigmoid output).
 *   Within each of the n_segments groups of T/n_segments tokens, expert e keeps the C
 *   tokens with the largest (score, -token) key; ties go to the lower token index.
 *   idx  [E, Ce] int32, Ce = n_segments*C: chosen tokens, ascending;
 *   gate [E, Ce] fp32: the chosen token's score for the expert;
 *   tok_ptr [T+1] int32, tok_ent [E*Ce] int32: CSR of the inverse map — token t's
 *   entries are tok_ent[tok_ptr[t] .. tok_ptr[t+1]), each e*Ce + slot, ascending e.
 *   tok_ptr / tok_ent may both be NULL to skip the CSR. */
NMOE_API nmoe_status nmoe_select(const float* scores_t, int64_t T, int64_t E, int64_t C,
                        int64_t n_segments, int32_t* idx, float* gate, int32_t* tok_ptr,
                        int32_t* tok_ent, nmoe_stream_t stream);

/* The whole layer, bf16, defaults (softmax, flat token axis, raw score weights):
 *   x [T, d], W_r [d, E], W1 [E, d, F] (gate), W3 [E, d, F] (up), W2 [E, F, d],
 *   out [T, d], all bf16 (the page's gate_up_proj (E, d, 2F) split at F into W1 | W3).
 * Scratch is allocated stream-ordered (cudaMallocAsync) for the call. */
NMOE_API nmoe_status nmoe_forward(const void* x, const void* W_r, const void* W1, const void* W3,
                         const void* W2, int64_t T, int64_t d, int64_t E, int64_t F,
                         int64_t C, void* out, nmoe_stream_t stream);

/* The whole layer with options (NULL = defaults). Same arguments as nmoe_forward. */
NMOE_API nmoe_status nmoe_forward_ex(const void* x, const void* W_r, const void* W1, const void* W3,
                            const void* W2, int64_t T, int64_t d, int64_t E, int64_t F,
                            int64_t C, void* out, nmoe_stream_t stream,
                            const nmoe_options* opts);

/* Bytes of workspace nmoe_forward_ex needs for these sizes and options (0 on invalid
 * sizes). */
NMOE_API size_t nmoe_workspace_size(int64_t T, int64_t d, int64_t E, int64_t F, int64_t C,
                           const nmoe_options* opts);

/* Byte offsets, inside a workspace laid out for these sizes and options, of Y
 * [E*Ce, d] (fp32 for fp32 layers and SPLIT intermediates, else bf16; row r is the r-th
 * entry in token-major order), tok_ptr [T + 1] int32 and tok_ent [E*Ce] int32 (entry r
 * = e*Ce + slot). NMOE_ERR_INVALID_ARG for invalid sizes. Pure host logic. */
NMOE_API nmoe_status nmoe_workspace_offsets(int64_t T, int64_t d, int64_t E, int64_t F,
                                            int64_t C, const nmoe_options* opts,
                                            size_t* y_offset, size_t* tok_ptr_offset,
                                            size_t* tok_ent_offset);

/* Expert parallelism: the token-major rows of tokens [t_begin, t_end) whose expert lies
 * in [e_begin, e_end), ascending, into rows[0 .. n) (device int32), and -1 into
 * rows[n .. capacity), with n written to *count (device int32). The capacity is known
 * on the host in advance: (e_end - e_begin) * Ce can never be exceeded, so buffers of
 * that many rows let ranks exchange fixed-size buffers without reading any count back
 * to the host. A list longer than `capacity` keeps its first `capacity` rows and sets
 * the error word (NMOE_ERR_DEVICE_CHECK). tok_ptr and tok_ent as left in the workspace
 * (nmoe_workspace_offsets); Ce = n_segments * C. */
NMOE_API nmoe_status nmoe_ep_rows(const int32_t* tok_ptr, const int32_t* tok_ent, int64_t T,
                                  int64_t E, int64_t Ce, int64_t t_begin, int64_t t_end,
                                  int64_t e_begin, int64_t e_end, int32_t* rows,
                                  int64_t capacity, int32_t* count, nmoe_stream_t stream);

/* dst[i, :] = src[rows[i], :] (gather; a zero row where rows[i] < 0) / dst[rows[i], :] =
 * src[i, :] (scatter; nothing where rows[i] < 0) for i < n: rows of row_bytes bytes (a
 * positive multiple of 16), 16-byte aligned device arrays; rows device int32. Ownership
 * stays with the caller; rows[i] must index a row of src (gather) or dst (scatter); any
 * other rows[i] >= 0 is an error the library cannot detect.
 *
 * With src = x and rows = the chosen tokens idx [E, Ce] (flattened), the gather is the
 * grouped-matmul path's "permute the tokens into contiguous per-expert blocks" step
 * (NucleusMoE-Image walkthrough, section 6): dst holds each expert's Ce rows as one
 * block. The layer itself never runs it (the gate/up GEMM reads the chosen rows of x
 * straight into its A tiles); it stands alone for expert parallelism and to measure
 * that copy's bandwidth. */
NMOE_API nmoe_status nmoe_rows_gather(const void* src, const int32_t* rows, int64_t n,
                                      int64_t row_bytes, void* dst, nmoe_stream_t stream);
NMOE_API nmoe_status nmoe_rows_scatter(const void* src, const int32_t* rows, int64_t n,
                                       int64_t row_bytes, void* dst, nmoe_stream_t stream);

/* The combine alone for tokens [t_begin, t_end): out[t - t_begin, :] = sum of Y rows
 * tok_ptr[t] .. tok_ptr[t+1]-1 in order, fp32, rounded once (0 for a token without
 * rows). Y in y_dtype (NMOE_F32 or NMOE_BF16), out in out_dtype, d a multiple of 8. */
NMOE_API nmoe_status nmoe_combine_tokens(const void* Y, const int32_t* tok_ptr, int64_t T,
                                         int64_t d, int64_t t_begin, int64_t t_end,
                                         nmoe_dtype y_dtype, nmoe_dtype out_dtype, void* out,
                                         nmoe_stream_t stream);

/* Number of kernels one nmoe_forward_ex call with these sizes and options launches
 * (0 for invalid sizes): the router, the selection, the token lists (inside the gate/up
 * GEMM on the tensor-core path, else a kernel of their own), the gate/up and down GEMMs
 * (twice with a shared expert) and the combine. Pure host logic; no device access. */
NMOE_API int nmoe_kernels_per_call(int64_t T, int64_t d, int64_t E, int64_t F, int64_t C,
                                   const nmoe_options* opts);

/* Waits for `stream`, then returns and clears the current device's error word
 * (NMOE_OK, NMOE_ERR_TIMEOUT or NMOE_ERR_DEVICE_CHECK), or NMOE_ERR_CUDA if the stream
 * itself reported an error. */
NMOE_API nmoe_status nmoe_get_last_error(nmoe_stream_t stream);

/* Static description of a status code. */
NMOE_API const char* nmoe_status_str(nmoe_status s);

/* Per-stage timer. nmoe_trace_create makes room for `max_calls` traced calls on the
 * current device. nmoe_trace_read waits for the recorded events and writes the summed
 * milliseconds of each stage over all recorded calls to stage_ms[NMOE_N_STAGES] and the
 * number of calls to *n_calls; nmoe_trace_reset forgets them. */
NMOE_API nmoe_status nmoe_trace_create(int max_calls, nmoe_trace** out);
NMOE_API nmoe_status nmoe_trace_read(nmoe_trace* tr, double* stage_ms, int* n_calls);
NMOE_API nmoe_status nmoe_trace_reset(nmoe_trace* tr);
NMOE_API void nmoe_trace_destroy(nmoe_trace* tr);
NMOE_API const char* nmoe_stage_name(int stage);

/* The whole layer, like nmoe_forward (bf16, default options), for callers that cannot
 * allocate device memory while they run it: code under a memory manager that owns all
 * of the device's memory (a caching allocator, a pre-partitioned arena), real-time
 * paths that must not enter the CUDA allocator, or hosts that forbid allocation after
 * start-up. The pages describe no such entry point; it exists for those callers.
 *   - Scratch lives in one fixed array of NMOE_NOALLOC_SCRATCH_BYTES (128 MiB) in device
 *     memory, reserved on every device that loads this library and held until the
 *     process exits. The call makes no cudaMalloc, cudaFree or other allocation.
 *   - Sizes whose scratch (nmoe_workspace_size with default options) exceeds that
 *     capacity are rejected with NMOE_ERR_WORKSPACE before anything is enqueued
 *     (T = 8192, d = 2048, E = 64, F = 1024, C = 128 needs ~100 MiB and fits).
 *   - The first call on a device looks the array's address up on that device; make
 *     that first call before any stream capture.
 *   - All calls on a device share the one array and it keeps the last call's
 *     contents (nothing in it needs to start at zero). Calls whose work overlaps on the
 *     GPU (other streams, or concurrent host threads) race on it: order them.
 * Arguments, layouts, ownership and the other errors are those of nmoe_forward. */
#define NMOE_NOALLOC_SCRATCH_BYTES ((size_t)128 << 20)
NMOE_API nmoe_status nmoe_forward_noalloc(const void* x, const void* W_r, const void* W1,
                                          const void* W3, const void* W2, int64_t T,
                                          int64_t d, int64_t E, int64_t F, int64_t C,
                                          void* out, nmoe_stream_t stream);

/* Build identification: a static string (architecture, kernel variants). */
NMOE_API const char* nmoe_build_info(void);

#ifdef __cplusplus
}
#endif

#endif /* NMOE_H_ */
