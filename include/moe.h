/*
 * moe.h -- C ABI of the B200 (sm_100a) MoE-layer forward library (libmoe.so).
 *
 * One MoE layer forward, as the grouped-GEMM pages state it:
 *   p = softmax(W_r x_t);  S_t = top-k(p);
 *   y_t = E_shared(x_t) + sum_{i in S_t} p_i E_i(x_t)
 *     ("MegaMoE math model -> DeepGEMM source walk-through", §2.1)
 * computed by the six-step data flow of "Dense GEMM -> GroupedGEMM -> TP MoE"
 * §2.2: router scores, top-k, per-expert histogram + prefix sum, scatter into
 * expert-contiguous order, grouped GEMMs (up with SiLU gate, then down), and
 * gather * gate weight + sum.  E_i(x) = W2[i] (silu(W1[i][0:I] x) * W1[i][I:2I] x).
 *
 * Conventions shared by every entry point
 *   - Pointers are DEVICE pointers owned by the caller, except where a
 *     parameter says "host".  The library never allocates device memory.
 *   - All matrices are row-major.  Weights are "K-major": W1[e] is [2I, d],
 *     W2[e] is [d, I] (contraction dimension contiguous), experts stacked
 *     contiguously (W1[e] = W1 + e*2I*d elements).
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Calls only
 *     enqueue work on it: they neither synchronise nor copy between host and
 *     device, except moe_read_device_status and moe_forward_host, which say so.
 *   - Argument and shape errors are detected on the host before anything is
 *     launched and returned as MOE_ERR_INVALID / MOE_ERR_UNSUPPORTED /
 *     MOE_ERR_WORKSPACE.  Errors only a kernel can see (bad device offsets,
 *     a pipeline wait that timed out, an expert id out of range) are written
 *     to a status word at the start of the caller's workspace; read it with
 *     moe_read_device_status after the work has run.
 *   - Inputs must be finite; NaN/Inf propagate unspecified.
 *   - Workspaces must be 256-byte aligned.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MOE_ABI_VERSION 2

typedef enum moe_status {
  MOE_OK = 0,
  MOE_ERR_INVALID = -1,      /* null pointer, bad size, k > E, ...                  */
  MOE_ERR_UNSUPPORTED = -2,  /* valid but not implemented (e.g. N % 128 != 0)       */
  MOE_ERR_WORKSPACE = -3,    /* workspace smaller than the *_workspace_size result  */
  MOE_ERR_CUDA = -4,         /* a CUDA runtime / driver call failed                 */
  MOE_ERR_BAD_OFFSETS = -5,  /* device offsets not monotone / not starting at 0 / past rows */
  MOE_ERR_TIMEOUT = -6       /* a kernel pipeline wait exceeded its time limit      */
} moe_status;

/* MOE_E4M3: E4M3 codes with fp32 scales s = amax/448, one per 128 elements
 * along K (activations) or per 128x128 block (weights); a GEMM promotes each
 * 128-wide K block's partial product by its scales ("MegaMoE ..." §2.3, §5.1).
 * MOE_MXE4M3: the same codes and groups with power-of-two scales, the
 * smallest 2^p (p in [-127, 127]) with 448 * 2^p >= amax, still stored as
 * fp32 values; a GEMM hands them to the tensor core as UE8M0 block scales
 * (tcgen05.mma kind::mxf8f6f4), which applies them itself. */
typedef enum moe_dtype { MOE_F32 = 0, MOE_F16 = 1, MOE_BF16 = 2, MOE_E4M3 = 3, MOE_MXE4M3 = 4 } moe_dtype;

typedef enum moe_epilogue {
  MOE_EPI_NONE = 0,      /* C = A B^T                                                   */
  MOE_EPI_SILU_GATE = 1  /* B holds 2N rows per group [gate; up]: C = silu(A Bg^T) * (A Bu^T) */
} moe_epilogue;

/* One layer's shape.  x_dtype: MOE_F32 | MOE_BF16.  router_dtype (W_r):
 * MOE_F32 | MOE_BF16 (an fp32 router needs fp32 x).  expert_dtype: MOE_BF16 |
 * MOE_E4M3 (the expert GEMMs run in E4M3 with fp32 scales) | MOE_MXE4M3
 * (E4M3 with power-of-two scales the tensor core applies).  out_dtype:
 * MOE_F32 | MOE_BF16.  shared_inter is 0 (no shared expert) or equal to inter.
 * d and inter are multiples of 128 (E4M3 / MX experts: d a multiple of 256).
 * renormalize = 0 weights each expert by its softmax value p_i (MegaMoE §2.1);
 * 1 divides by the sum over the selected experts (route_tokens in
 * Dense GEMM -> GroupedGEMM -> TP MoE §4.2).
 * capacity = 0: no limit; > 0: each expert takes at most `capacity` of the
 * batch's (token, slot) pairs, the first ones in token order, and a pair
 * over it adds nothing to its token's output (the token keeps the shared
 * expert and its other experts, weights unchanged).  This is the capacity
 * factor of Dense GEMM -> GroupedGEMM -> TP MoE §5.1 (tokens over an
 * expert's capacity take a fallback path) and DeepSeek MoE architecture
 * overview §3.2 (a bound on one expert's share of a forward's tokens);
 * capacity = ceil(factor * T * k / E) for a capacity factor `factor`.
 * flags: MOE_FLAG_GATHER_A makes the up GEMM gather its A rows through
 * row_to_token in the load (moe_grouped_gemm_gather) whenever it runs on a
 * single-CTA kernel, so the expert-ordered copy of x is not written; the
 * result is identical.  It is off by default: on the fine-grained layer the
 * gathered load (32 tile::gather4 per 128-row tile and k-step) measured
 * slower than writing and re-reading the copy. */
#define MOE_FLAG_GATHER_A 1
typedef struct moe_config {
  int T, d, E, k, inter, shared_inter;
  int x_dtype, router_dtype, expert_dtype, out_dtype;
  int renormalize;
  int capacity;
  int flags;
} moe_config;

/* Human-readable name of a status code (static string). */
const char* moe_status_string(int status);

/* Description of the last CUDA runtime / driver failure on this host thread
 * (the call that made an entry point return MOE_ERR_CUDA); static storage. */
const char* moe_last_error_string(void);

/* Multiprocessor count and compute capability of the current device; returns
 * MOE_ERR_UNSUPPORTED when it is not an sm_100 part. */
int moe_device_info(int* num_sms, int* cc_major, int* cc_minor);

/* Synchronises `stream`, then copies the device status word at the start of
 * workspace `ws` into *status (MOE_OK or a negative moe_status). */
int moe_read_device_status(const void* ws, void* stream, int* status);

/* ---------------------------------------------------------------- router
 * Router scores, softmax over all E experts and top-k ("MegaMoE ..." §2.1:
 * p_i = Softmax(W_r x_t)_i; "Dense GEMM -> GroupedGEMM -> TP MoE" §4.2
 * route_tokens: F.linear -> softmax -> topk).
 *   x        [T, d]  x_dtype (MOE_F32 | MOE_BF16)
 *   W_r      [E, d]  w_dtype (MOE_F32 | MOE_BF16)
 *   bias     [E] fp32 added to the logits before the softmax, or NULL
 *   logits_out [T, E] fp32, or NULL (the logits every later step depends on)
 *   topk_idx [T, k] int32: selected experts, descending logit, ties -> lower index
 *            (-0 and +0 are equal logits)
 *   topk_w   [T, k] fp32: p of the selected experts (renormalised if asked)
 *   ws       scratch of moe_router_workspace_size(T, E) bytes (status word + logits)
 * 1 <= k <= min(E, 32), E <= 1024, d % 8 == 0; x and W_r 16-byte aligned.
 * bf16 x and W_r with E <= 256 and k <= 8 run as one launch (tensor-core
 * logits, K split over a thread-block cluster, softmax and top-k on chip);
 * the logits are then summed over the K slices in a fixed order, so they do
 * not vary from run to run. */
size_t moe_router_workspace_size(int T, int E);
int moe_router_topk(const void* x, int x_dtype, const void* W_r, int w_dtype, const float* bias, int T,
                    int d, int E, int k, int renormalize, float* logits_out, int32_t* topk_idx,
                    float* topk_w, void* ws, size_t ws_bytes, void* stream);

/* Softmax + top-k of precomputed logits (the router's second half; also the
 * router-only microbenchmark).  logits [N, E] in dtype MOE_F16 | MOE_F32 |
 * MOE_BF16; outputs as for moe_router_topk.  E <= 1024, 1 <= k <= min(E, 32). */
int moe_topk_logits(const void* logits, int dtype, int N, int E, int k, int renormalize,
                    int32_t* topk_idx, float* topk_w, void* stream);

/* ---------------------------------------------------------------- permute
 * Steps 3-4 of "Dense GEMM -> GroupedGEMM -> TP MoE" §2.2: per-expert
 * histogram, exclusive prefix sum (expert sizes stay on the device, §2.3)
 * and the scatter of tokens into expert-contiguous order.  Inside an
 * expert's segment rows follow ascending token id, so the plan is
 * deterministic.  With append_shared the T tokens are appended as rows
 * R..R+T-1 (R = T*k), the shared expert's group.
 *   x            [T, d] x_dtype (MOE_F32 | MOE_BF16)
 *   topk_idx     [T, k] int32 in [0, E), distinct within a token
 *   xp_dtype     MOE_BF16 (x rounded to bf16) | MOE_E4M3 (quantised once per
 *                token per 128 columns: s = amax/448, q = e4m3_rn_satfinite(x/s))
 *                | MOE_MXE4M3 (the same with power-of-two s, see moe_dtype)
 *   xp           [R', d] (R' = R + T if append_shared else R)
 *   xp_scales    [d/128][R'] fp32 (K-block-major: scale of row r, block b at
 *                b*R' + r) when xp_dtype is MOE_E4M3 / MOE_MXE4M3, else NULL
 *   counts       [E] int32; offsets [E+1] (+1 with append_shared): offsets[e]
 *                = sum of counts before e, offsets[E] = R, offsets[E+1] = R+T
 *   row_to_token [R'] int32;  token_to_row [T, k] int32
 *   ws           moe_permute_workspace_size(T, E) bytes (status + per-block counts)
 * T * (k + 1) <= 2^30 (rows are int32 indices), else MOE_ERR_UNSUPPORTED.
 * Out-of-range or repeated expert ids set MOE_ERR_INVALID in the status word
 * and leave the outputs unspecified. */
size_t moe_permute_workspace_size(int T, int E);
int moe_permute(const void* x, int x_dtype, const int32_t* topk_idx, int T, int d, int E, int k,
                int append_shared, int xp_dtype, void* xp, float* xp_scales, int32_t* counts,
                int32_t* offsets, int32_t* row_to_token, int32_t* token_to_row, void* ws, size_t ws_bytes,
                void* stream);

/* moe_permute with a capacity limit (capacity = 0: none): each expert keeps
 * its first `capacity` (token, slot) pairs in token order, as moe_config's
 * capacity describes.  A pair over its expert's capacity gets no row
 * (token_to_row = -1); counts[e] are the kept rows, offsets their exclusive
 * scan, offsets[E] the kept total R_kept, and with append_shared the shared
 * expert's rows are R_kept .. R_kept+T-1 (offsets[E+1] = R_kept + T).  Rows
 * from there up to R' - 1 belong to no token (row_to_token = -1).  The
 * buffers keep moe_permute's sizes (R' = T*k (+ T) rows).  The pairs with
 * token_to_row = -1 are the overflow: a caller may send them to another
 * path (moe_combine_plan skips them).  capacity < 0: MOE_ERR_INVALID. */
int moe_permute_capacity(const void* x, int x_dtype, const int32_t* topk_idx, int T, int d, int E, int k,
                         int append_shared, int capacity, int xp_dtype, void* xp, float* xp_scales,
                         int32_t* counts, int32_t* offsets, int32_t* row_to_token, int32_t* token_to_row,
                         void* ws, size_t ws_bytes, void* stream);

/* Allocation-free variant of moe_permute, for callers that cannot give the
 * library any device memory of its own: a plugin whose host runtime owns all
 * allocations and offers no workspace, or a serving loop whose memory plan
 * is fixed at start-up and allows no allocation afterwards.  The source
 * pages have no counterpart; the operation and the arguments are those of
 * moe_permute, minus `ws`.
 *   Scratch (status word + per-block expert counts) lives in a 1 MiB + 256 B
 *   array of static device memory inside the library, which every GPU that
 *   loads the library keeps until the process exits.  Limit:
 *   ceil(T / 32) * E <= 262144 (e.g. T <= 32768 at E = 256, T <= 65536 at
 *   E = 128) and T * (k + 1) <= 2^30; larger calls return
 *   MOE_ERR_UNSUPPORTED before launching.
 *   The first call in each CUDA context looks up the array's device address
 *   in that context (with it current) and caches it under the context's
 *   unique id, so a caller's own context, or the new primary context after
 *   cudaDeviceReset, gets its own lookup.  Make the first call of a context
 *   before any stream capture begins.
 *   All calls on a device share the one array and leave their contents
 *   there; each call clears the status word and rewrites every count it
 *   reads.  Calls whose kernels overlap on the GPU (e.g. on two streams)
 *   race on it: order them.  There is no status read-back: invalid expert
 *   ids are skipped (nothing out of bounds is written) and leave the outputs
 *   unspecified; use moe_permute + moe_read_device_status to detect them.
 * Never calls cudaMalloc / cudaFree or any allocating routine. */
int moe_permute_noalloc(const void* x, int x_dtype, const int32_t* topk_idx, int T, int d, int E, int k,
                        int append_shared, int xp_dtype, void* xp, float* xp_scales, int32_t* counts,
                        int32_t* offsets, int32_t* row_to_token, int32_t* token_to_row, void* stream);

/* ---------------------------------------------------------------- grouped GEMM
 * One persistent launch computes, for every group g (an expert) with rows
 * offsets[g] .. offsets[g+1]-1 of A:
 *     C[rows_g, :] = A[rows_g, :] * B[g]^T            (MOE_EPI_NONE)
 *     C[rows_g, :] = silu(A Bg^T) * (A Bu^T)           (MOE_EPI_SILU_GATE)
 * ("MegaMoE ..." §4.3: one launch, many problems with variable M_i and
 * shared N, K; "Dense GEMM -> GroupedGEMM -> TP MoE" §2.3: the
 * grouped_gemm(A_ptrs, B_ptrs, C_ptrs, expert_sizes, N, K, workspace, stream)
 * call, with the pointer arrays replaced by base + device offsets.)
 *   A        [rows, K] ab_dtype (MOE_BF16 | MOE_E4M3 | MOE_MXE4M3), row-major
 *   A_scales [K/128][rows] fp32 (E4M3 / MX only, else NULL)
 *   B        [G, Nb, K] ab_dtype, K-major, Nb = N (NONE) or 2N (SILU_GATE:
 *            rows 0..N-1 gate, N..2N-1 up)
 *   B_scales [G][Nb/128][K/128] fp32 (E4M3 / MX only, else NULL)
 *   offsets  [G+1] int32 DEVICE array, offsets[0] = 0, non-decreasing,
 *            offsets[G] <= rows; checked on the device (MOE_ERR_BAD_OFFSETS,
 *            nothing written)
 *   C        [rows, N] c_dtype: MOE_BF16 | MOE_F32 (NONE, bf16 inputs) or
 *            MOE_BF16 | ab_dtype's E4M3 kind (SILU_GATE); rows outside every group untouched
 *   C_scales [N/128][rows] fp32 when C is E4M3 (per row per 128 columns)
 *   ws       moe_grouped_gemm_workspace_size() bytes (status word)
 * MOE_MXE4M3 operands: the power-of-two scales go to the tensor core as
 * UE8M0 block scales (tcgen05.mma kind::mxf8f6f4), which applies them
 * itself; an MX C gets power-of-two scales.  Same shape rules as E4M3.
 * E4M3 operands: the scales vary along K, so each 128-wide K block's partial
 * product is scaled by sa[row, kb] * sb[n/128, kb] and accumulated in fp32
 * ("MegaMoE ..." §5.1); an E4M3 C is quantised per row per 128 columns
 * (s = amax/448, q = e4m3_rn_satfinite(c/s)) like the permute's activations.
 * Supported: bf16: K % 64 == 0, N % 128 == 0 (SILU_GATE) or N % 64 == 0
 * (NONE); E4M3: K % 128 == 0, N % 128 == 0 (SILU_GATE, C bf16 or E4M3) or
 * N % 256 == 0 (NONE, C bf16); G <= 1024. */
size_t moe_grouped_gemm_workspace_size(void);
/* The kernel a grouped GEMM of this shape runs on, as a short description
 * (host arithmetic only, no device needed; num_sms <= 0 means 148).
 * extra_groups = 1 counts the shared expert moe_forward appends as a group. */
const char* moe_grouped_gemm_plan(int G, int extra_groups, int rows, int N, int K, int ab_dtype, int epilogue,
                                  int c_dtype, int num_sms);
int moe_grouped_gemm(const void* A, const float* A_scales, const void* B, const float* B_scales,
                     const int32_t* offsets, int G, int rows, int N, int K, int ab_dtype, int epilogue,
                     void* C, int c_dtype, float* C_scales, void* ws, size_t ws_bytes, void* stream);

/* moe_grouped_gemm whose A rows are gathered in the load: row r of the
 * grouped problem (r < rows, in offsets order) is row A_rows[r] of the
 * source A [A_src_rows, K] (an entry < 0 or >= A_src_rows reads row 0 and
 * must belong to no group's valid rows), so an expert-contiguous copy of the
 * tokens never has to be written ("Dense GEMM -> GroupedGEMM -> TP MoE"
 * §2.2 names steps 3-4, prefix sum and scatter, as hotspots; here the
 * scatter folds into the GEMM's TMA loads, tile::gather4).  A_rows is a
 * DEVICE int32 array of `rows` entries (moe_permute's row_to_token);
 * A_scales, for E4M3 / MX operands, is [K/128][A_src_rows].  Everything else
 * as moe_grouped_gemm.  The shapes the CTA-pair and swap-AB kernels would
 * take run on the single-CTA kernels here; an fp32 C is MOE_ERR_UNSUPPORTED. */
int moe_grouped_gemm_gather(const void* A, const float* A_scales, int A_src_rows, const int32_t* A_rows,
                            const void* B, const float* B_scales, const int32_t* offsets, int G, int rows, int N,
                            int K, int ab_dtype, int epilogue, void* C, int c_dtype, float* C_scales, void* ws,
                            size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------- failure detection
 * Self-test of the grouped GEMM's failure path (no counterpart on the source
 * pages): launches the bf16 grouped-GEMM kernel on one CTA over a small
 * problem carved from `ws` (four tiles), whose epilogue first waits on a
 * barrier that no thread ever arrives at.  That wait gives up after
 * wait_limit_ns (1e6 .. 2e9); the kernel then raises its abort flag, the
 * producer waits for the copies it has in flight, the MMA issuer drains its
 * MMAs, TMEM is released and the kernel returns, leaving MOE_ERR_TIMEOUT in
 * the status word at the start of ws (read it with moe_read_device_status).
 * No fault, trap or unbounded wait is involved; the context stays usable.
 * ws: moe_selftest_workspace_size() bytes, 256-byte aligned. */
size_t moe_selftest_workspace_size(void);
int moe_selftest_stalled_pipeline(void* ws, size_t ws_bytes, unsigned long long wait_limit_ns, void* stream);

/* ---------------------------------------------------------------- combine
 * Step 6 of "Dense GEMM -> GroupedGEMM -> TP MoE" §2.2 and the sum of
 * "MegaMoE ..." §2.1:
 *   out[t] = Y[R + t] (if has_shared) + sum_{j<k} topk_w[t,j] * Y[token_to_row[t,j]]
 * accumulated in fp32 in that order.
 *   Y [R', d] MOE_BF16;  token_to_row [T, k];  topk_w [T, k] fp32
 *   out [T, d] out_dtype (MOE_BF16 | MOE_F32).  d % 8 == 0. */
int moe_combine(const void* Y, const int32_t* token_to_row, const float* topk_w, int has_shared, int T,
                int d, int k, void* out, int out_dtype, void* stream);

/* moe_combine over a plan from moe_permute_capacity: the shared expert's row
 * of token t is offsets[E] + t (offsets: the permute's DEVICE array), and a
 * slot with token_to_row[t, j] < 0 (its pair overflowed an expert's
 * capacity) adds nothing.  Otherwise as moe_combine. */
int moe_combine_plan(const void* Y, const int32_t* token_to_row, const float* topk_w, const int32_t* offsets, int E,
                     int has_shared, int T, int d, int k, void* out, int out_dtype, void* stream);

/* ---------------------------------------------------------------- FP8 weights
 * Quantise bf16 weights W [G, N, K] per 128x128 block ("MegaMoE ..." §2.3,
 * §5.1): s = amax(block)/448 (1 if the block is zero), Wq = e4m3_rn_satfinite(W/s).
 *   Wq [G, N, K] uint8 (E4M3 codes);  scales [G][N/128][K/128] fp32.
 * N % 128 == 0, K % 128 == 0. */
int moe_quantize_weights_fp8(const void* W, int G, int N, int K, uint8_t* Wq, float* scales, void* stream);

/* As moe_quantize_weights_fp8, with power-of-two block scales (MOE_MXE4M3):
 * s = the smallest 2^p with 448 * 2^p >= amax(block), p in [-127, 127]
 * (1 if the block is zero); w / s is exact, then rounded to E4M3. */
int moe_quantize_weights_mx(const void* W, int G, int N, int K, uint8_t* Wq, float* scales, void* stream);

/* ---------------------------------------------------------------- whole layer
 * moe_forward runs the whole layer: router, permute, up grouped GEMM with the
 * SiLU-gate epilogue, down grouped GEMM, combine.  The shared expert (if
 * cfg->shared_inter) is one more group of the grouped GEMMs.
 *   x [T, d] cfg->x_dtype;  W_r [E, d] cfg->router_dtype;  router_bias [E] or NULL
 *   BF16 experts: W1 [E, 2I, d], W2 [E, d, I] bf16, *_scales NULL
 *   E4M3 experts: W1/W2 as moe_quantize_weights_fp8 output with their scales
 *   MX experts:   W1/W2 as moe_quantize_weights_mx output with their scales
 *   W1_shared [2I, d], W2_shared [d, I] (+ scales) or NULL
 *   out [T, d] cfg->out_dtype;  counts_out [E] int32 (rows each expert took:
 *       its tokens, or at most cfg->capacity of them) or NULL
 *   ws  moe_workspace_size(cfg) bytes: status, routing, permutation plan and
 *       the intermediates Xp [R', d], H [R', I], Y [R', d].
 * No host synchronisation and no host<->device copy: the call can be
 * captured in a CUDA graph. */
size_t moe_workspace_size(const moe_config* cfg);
int moe_forward(const moe_config* cfg, const void* x, const void* W_r, const float* router_bias,
                const void* W1, const float* W1_scales, const void* W2, const float* W2_scales,
                const void* W1_shared, const float* W1s_scales, const void* W2_shared,
                const float* W2s_scales, void* out, int32_t* counts_out, void* ws, size_t ws_bytes,
                void* stream);

/* As moe_forward, and also records stage_events[0..5] (cudaEvent_t handles
 * the caller created) on `stream`: [0] before the router, [1] before the
 * permute, [2] before the up GEMM, [3] before the down GEMM, [4] before the
 * combine and [5] after it, so that the caller can time each kernel of the
 * layer as it runs inside the whole forward.  A NULL array or handle is
 * MOE_ERR_INVALID; with T == 0 no event is recorded. */
int moe_forward_marked(const moe_config* cfg, const void* x, const void* W_r, const float* router_bias,
                       const void* W1, const float* W1_scales, const void* W2, const float* W2_scales,
                       const void* W1_shared, const float* W1s_scales, const void* W2_shared,
                       const float* W2s_scales, void* out, int32_t* counts_out, void* ws, size_t ws_bytes,
                       void* const* stage_events, void* stream);

/* How many kernels one moe_forward of this shape launches (host arithmetic
 * only, no device needed): the router (1 when it runs fused, else 2), the
 * permute's 3, the 2 grouped GEMMs and the combine; 0 for T = 0, -1 for an
 * invalid config.  (Status-word resets are memsets, not kernels.) */
int moe_forward_launches(const moe_config* cfg);

/* As moe_forward, but x_host and out_host are HOST buffers (page-locked for
 * the copies to overlap): x is copied into the workspace, the layer runs,
 * and out is copied back, all on `stream`.  The call returns without
 * synchronising; out_host is valid once the stream has drained.
 * ws: moe_workspace_size(cfg) + moe_host_staging_size(cfg) bytes. */
size_t moe_host_staging_size(const moe_config* cfg);
int moe_forward_host(const moe_config* cfg, const void* x_host, const void* W_r, const float* router_bias,
                     const void* W1, const float* W1_scales, const void* W2, const float* W2_scales,
                     const void* W1_shared, const float* W1s_scales, const void* W2_shared,
                     const float* W2s_scales, void* out_host, void* ws, size_t ws_bytes, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
