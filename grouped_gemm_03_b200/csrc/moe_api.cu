// The C ABI (include/moe.h): argument validation, workspace layout and the
// composition of the kernels into the layer forward.  Nothing here computes;
// every step of the path runs in the kernels of the other translation units.
#include <cstdio>
#include <cstring>

#include "common.cuh"

namespace moe {

namespace {
thread_local char g_last_error[256] = "no error";
}

int record_cuda_error(cudaError_t e, const char* where) {
  snprintf(g_last_error, sizeof(g_last_error), "%s: %s (%d)", where, cudaGetErrorString(e), static_cast<int>(e));
  return MOE_ERR_CUDA;
}

int num_sms() {
  static int cached[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (!cached[dev]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cached[dev] = n;
  }
  return cached[dev];
}

namespace {

inline cudaStream_t as_stream(void* s) { return static_cast<cudaStream_t>(s); }

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

size_t dtype_bytes(int dt) {
  switch (dt) {
    case MOE_F32: return 4;
    case MOE_F16: return 2;
    case MOE_BF16: return 2;
    case MOE_E4M3: return 1;
    case MOE_MXE4M3: return 1;
    default: return 0;
  }
}

struct FwdLayout {
  size_t status, idx, w, logits, base, counts, offsets, r2t, t2r, xp, xps, h, hs, y, total;
};

FwdLayout fwd_layout(const moe_config& c) {
  FwdLayout L{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align_up(off + (bytes ? bytes : 1), 1024);
    return o;
  };
  const size_t T = c.T, k = c.k, E = c.E, d = c.d, I = c.inter;
  const size_t R = T * k, Rp = R + (c.shared_inter ? T : 0);
  const bool fp8 = is_e4m3(c.expert_dtype);
  const size_t eb = fp8 ? 1 : 2;
  L.status = take(256);
  L.idx = take(T * k * 4);
  L.w = take(T * k * 4);
  L.logits = take(kRouterMaxSplit * T * static_cast<size_t>(router_padded_experts(c.E)) * 4);
  L.base = take(static_cast<size_t>(permute_blocks(c.T)) * E * 4);
  L.counts = take(E * 4);
  L.offsets = take((E + 2) * 4);
  L.r2t = take(Rp * 4);
  L.t2r = take(T * k * 4);
  L.xp = take(Rp * d * eb);
  L.xps = fp8 ? take(d / 128 * Rp * 4) : 0;
  L.h = take(Rp * I * eb);
  L.hs = fp8 ? take(I / 128 * Rp * 4) : 0;
  L.y = take(Rp * d * 2);
  L.total = off;
  return L;
}

int check_config(const moe_config* c) {
  if (!c) return MOE_ERR_INVALID;
  if (c->T < 0 || c->d <= 0 || c->E <= 0 || c->k <= 0 || c->inter <= 0) return MOE_ERR_INVALID;
  if (c->k > c->E || c->k > kMaxTopK) return MOE_ERR_INVALID;
  if (c->E > kMaxExperts || c->E + 1 > kMaxGroups) return MOE_ERR_UNSUPPORTED;
  if (c->shared_inter != 0 && c->shared_inter != c->inter) return MOE_ERR_UNSUPPORTED;
  if (c->x_dtype != MOE_F32 && c->x_dtype != MOE_BF16) return MOE_ERR_INVALID;
  if (c->router_dtype != MOE_F32 && c->router_dtype != MOE_BF16) return MOE_ERR_INVALID;
  if (c->expert_dtype != MOE_BF16 && !is_e4m3(c->expert_dtype)) return MOE_ERR_INVALID;
  if (c->out_dtype != MOE_F32 && c->out_dtype != MOE_BF16) return MOE_ERR_INVALID;
  if (c->d % 128 != 0 || c->inter % 128 != 0) return MOE_ERR_UNSUPPORTED;
  if (is_e4m3(c->expert_dtype) && c->d % 256 != 0) return MOE_ERR_UNSUPPORTED;
  if (c->capacity < 0) return MOE_ERR_INVALID;
  if (c->flags & ~MOE_FLAG_GATHER_A) return MOE_ERR_INVALID;
  const long long rows = static_cast<long long>(c->T) * (c->k + 1);
  if (rows * c->d > (1ll << 40) || rows > kMaxPermuteRows) return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" {

const char* moe_status_string(int s) {
  switch (s) {
    case MOE_OK: return "MOE_OK";
    case MOE_ERR_INVALID: return "MOE_ERR_INVALID: invalid argument";
    case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED: valid but unsupported shape or type";
    case MOE_ERR_WORKSPACE: return "MOE_ERR_WORKSPACE: workspace too small or misaligned";
    case MOE_ERR_CUDA: return "MOE_ERR_CUDA: CUDA call failed";
    case MOE_ERR_BAD_OFFSETS: return "MOE_ERR_BAD_OFFSETS: group offsets not monotone from 0 within rows";
    case MOE_ERR_TIMEOUT: return "MOE_ERR_TIMEOUT: kernel pipeline wait timed out";
    default: return "unknown moe status";
  }
}

const char* moe_last_error_string(void) { return g_last_error; }

int moe_device_info(int* num_sms_out, int* cc_major, int* cc_minor) {
  int dev = 0, maj = 0, min_ = 0;
  MOE_CUDA_CHECK(cudaGetDevice(&dev));
  MOE_CUDA_CHECK(cudaDeviceGetAttribute(&maj, cudaDevAttrComputeCapabilityMajor, dev));
  MOE_CUDA_CHECK(cudaDeviceGetAttribute(&min_, cudaDevAttrComputeCapabilityMinor, dev));
  if (num_sms_out) *num_sms_out = num_sms();
  if (cc_major) *cc_major = maj;
  if (cc_minor) *cc_minor = min_;
  return maj == 10 ? MOE_OK : MOE_ERR_UNSUPPORTED;
}

int moe_read_device_status(const void* ws, void* stream, int* status) {
  if (!ws || !status) return MOE_ERR_INVALID;
  MOE_CUDA_CHECK(cudaStreamSynchronize(as_stream(stream)));
  int v = 0;
  MOE_CUDA_CHECK(cudaMemcpy(&v, ws, sizeof(int), cudaMemcpyDeviceToHost));
  *status = v;
  return MOE_OK;
}

// ------------------------------------------------------------------ router
size_t moe_router_workspace_size(int T, int E) {
  return 256 + align_up(static_cast<size_t>(kRouterMaxSplit) * (T > 0 ? T : 0) *
                            static_cast<size_t>(E > 0 ? router_padded_experts(E) : 0) * 4,
                        256);
}

int moe_router_topk(const void* x, int x_dtype, const void* W_r, int w_dtype, const float* bias, int T, int d,
                    int E, int k, int renormalize, float* logits_out, int32_t* topk_idx, float* topk_w, void* ws,
                    size_t ws_bytes, void* stream) {
  if (T < 0 || d <= 0 || E <= 0 || k <= 0 || k > E || k > kMaxTopK || E > kMaxExperts) return MOE_ERR_INVALID;
  if (d % 8 != 0) return MOE_ERR_UNSUPPORTED;
  if ((x_dtype != MOE_F32 && x_dtype != MOE_BF16) || (w_dtype != MOE_F32 && w_dtype != MOE_BF16))
    return MOE_ERR_INVALID;
  if (T > 0 && (!x || !W_r || !topk_idx || !topk_w)) return MOE_ERR_INVALID;
  if (!ws || !aligned(ws, 256)) return MOE_ERR_WORKSPACE;
  if (ws_bytes < moe_router_workspace_size(T, E)) return MOE_ERR_WORKSPACE;
  if (!aligned(x, 16) || !aligned(W_r, 16)) return MOE_ERR_INVALID;
  cudaStream_t s = as_stream(stream);
  MOE_CUDA_CHECK(cudaMemsetAsync(ws, 0, sizeof(int), s));
  return launch_router(x, x_dtype, W_r, w_dtype, bias, T, d, E, k, renormalize, logits_out, topk_idx, topk_w,
                       reinterpret_cast<float*>(static_cast<char*>(ws) + 256), static_cast<int*>(ws), s);
}

int moe_topk_logits(const void* logits, int dtype, int N, int E, int k, int renormalize, int32_t* topk_idx,
                    float* topk_w, void* stream) {
  if (N < 0 || E <= 0 || k <= 0 || k > E || k > kMaxTopK || E > kMaxExperts) return MOE_ERR_INVALID;
  if (dtype != MOE_F16 && dtype != MOE_F32 && dtype != MOE_BF16) return MOE_ERR_INVALID;
  if (N > 0 && (!logits || !topk_idx || !topk_w)) return MOE_ERR_INVALID;
  if (!aligned(logits, 16)) return MOE_ERR_INVALID;
  return launch_topk_logits(logits, dtype, N, E, k, renormalize, topk_idx, topk_w, as_stream(stream));
}

// ------------------------------------------------------------------ permute
size_t moe_permute_workspace_size(int T, int E) {
  if (T < 0 || E <= 0) return 0;
  return 256 + align_up(static_cast<size_t>(permute_blocks(T)) * E * 4, 256);
}

namespace {
int permute_impl(const void* x, int x_dtype, const int32_t* topk_idx, int T, int d, int E, int k, int append_shared,
                 int capacity, int xp_dtype, void* xp, float* xp_scales, int32_t* counts, int32_t* offsets,
                 int32_t* row_to_token, int32_t* token_to_row, void* ws, size_t ws_bytes, void* stream) {
  if (T < 0 || d <= 0 || E <= 0 || k <= 0 || k > E || k > kMaxTopK || E > kMaxExperts) return MOE_ERR_INVALID;
  if (static_cast<long long>(T) * (k + 1) > kMaxPermuteRows) return MOE_ERR_UNSUPPORTED;
  if (capacity < 0) return MOE_ERR_INVALID;
  if (x_dtype != MOE_F32 && x_dtype != MOE_BF16) return MOE_ERR_INVALID;
  if (xp_dtype != MOE_BF16 && !is_e4m3(xp_dtype)) return MOE_ERR_INVALID;
  if (d % 8 != 0 || (is_e4m3(xp_dtype) && d % 128 != 0)) return MOE_ERR_UNSUPPORTED;
  if (!counts || !offsets) return MOE_ERR_INVALID;
  if (T > 0 && (!x || !topk_idx || !xp || !row_to_token || !token_to_row)) return MOE_ERR_INVALID;
  if (T > 0 && is_e4m3(xp_dtype) && !xp_scales) return MOE_ERR_INVALID;
  if (!aligned(x, 16) || !aligned(xp, 16)) return MOE_ERR_INVALID;
  if (!ws || !aligned(ws, 256)) return MOE_ERR_WORKSPACE;
  if (ws_bytes < moe_permute_workspace_size(T, E)) return MOE_ERR_WORKSPACE;
  cudaStream_t s = as_stream(stream);
  MOE_CUDA_CHECK(cudaMemsetAsync(ws, 0, sizeof(int), s));
  PermuteArgs a;
  a.x = x;
  a.x_dtype = x_dtype;
  a.idx = topk_idx;
  a.T = T;
  a.d = d;
  a.E = E;
  a.k = k;
  a.shared = append_shared ? 1 : 0;
  a.xp_dtype = xp_dtype;
  a.xp = xp;
  a.xp_scales = xp_scales;
  a.counts = counts;
  a.offsets = offsets;
  a.row_to_token = row_to_token;
  a.token_to_row = token_to_row;
  a.block_base = reinterpret_cast<int32_t*>(static_cast<char*>(ws) + 256);
  a.status = static_cast<int*>(ws);
  a.capacity = capacity;
  return launch_permute(a, s);
}
}  // namespace

int moe_permute(const void* x, int x_dtype, const int32_t* topk_idx, int T, int d, int E, int k, int append_shared,
                int xp_dtype, void* xp, float* xp_scales, int32_t* counts, int32_t* offsets, int32_t* row_to_token,
                int32_t* token_to_row, void* ws, size_t ws_bytes, void* stream) {
  return permute_impl(x, x_dtype, topk_idx, T, d, E, k, append_shared, 0, xp_dtype, xp, xp_scales, counts, offsets,
                      row_to_token, token_to_row, ws, ws_bytes, stream);
}

int moe_permute_capacity(const void* x, int x_dtype, const int32_t* topk_idx, int T, int d, int E, int k,
                         int append_shared, int capacity, int xp_dtype, void* xp, float* xp_scales, int32_t* counts,
                         int32_t* offsets, int32_t* row_to_token, int32_t* token_to_row, void* ws, size_t ws_bytes,
                         void* stream) {
  return permute_impl(x, x_dtype, topk_idx, T, d, E, k, append_shared, capacity, xp_dtype, xp, xp_scales, counts,
                      offsets, row_to_token, token_to_row, ws, ws_bytes, stream);
}

// ------------------------------------------------------------------ grouped GEMM
size_t moe_grouped_gemm_workspace_size(void) { return 256; }

int moe_grouped_gemm(const void* A, const float* A_scales, const void* B, const float* B_scales,
                     const int32_t* offsets, int G, int rows, int N, int K, int ab_dtype, int epilogue, void* C,
                     int c_dtype, float* C_scales, void* ws, size_t ws_bytes, void* stream) {
  if (G <= 0 || rows < 0 || N <= 0 || K <= 0) return MOE_ERR_INVALID;
  if (G > kMaxGroups) return MOE_ERR_UNSUPPORTED;
  if (!A || !B || !offsets || !C) return MOE_ERR_INVALID;
  if (ab_dtype != MOE_BF16 && !is_e4m3(ab_dtype)) return MOE_ERR_INVALID;
  if (epilogue != MOE_EPI_NONE && epilogue != MOE_EPI_SILU_GATE) return MOE_ERR_INVALID;
  if (is_e4m3(ab_dtype) && (!A_scales || !B_scales)) return MOE_ERR_INVALID;
  if (is_e4m3(c_dtype) && !C_scales) return MOE_ERR_INVALID;
  if (is_e4m3(c_dtype) && c_dtype != ab_dtype) return MOE_ERR_UNSUPPORTED;  // h keeps the operands' scale kind
  if (ab_dtype == MOE_BF16 && K % 64 != 0) return MOE_ERR_UNSUPPORTED;
  if (is_e4m3(ab_dtype) && K % 128 != 0) return MOE_ERR_UNSUPPORTED;
  if (!aligned(A, 16) || !aligned(B, 16) || !aligned(C, 16)) return MOE_ERR_INVALID;
  if (!ws || !aligned(ws, 256)) return MOE_ERR_WORKSPACE;
  if (ws_bytes < moe_grouped_gemm_workspace_size()) return MOE_ERR_WORKSPACE;
  cudaStream_t s = as_stream(stream);
  MOE_CUDA_CHECK(cudaMemsetAsync(ws, 0, sizeof(int), s));
  GemmArgs a{};
  a.A = A;
  a.A_scales = A_scales;
  a.B = B;
  a.B_scales = B_scales;
  a.offsets = offsets;
  a.G = G;
  a.has_extra = 0;
  a.rows = rows;
  a.N = N;
  a.K = K;
  a.ab_dtype = ab_dtype;
  a.epilogue = epilogue;
  a.c_dtype = c_dtype;
  a.C = C;
  a.C_scales = C_scales;
  a.status = static_cast<int*>(ws);
  return launch_grouped_gemm(a, s);
}

int moe_grouped_gemm_gather(const void* A, const float* A_scales, int A_src_rows, const int32_t* A_rows,
                            const void* B, const float* B_scales, const int32_t* offsets, int G, int rows, int N,
                            int K, int ab_dtype, int epilogue, void* C, int c_dtype, float* C_scales, void* ws,
                            size_t ws_bytes, void* stream) {
  if (G <= 0 || rows < 0 || N <= 0 || K <= 0 || A_src_rows <= 0) return MOE_ERR_INVALID;
  if (G > kMaxGroups) return MOE_ERR_UNSUPPORTED;
  if (!A || !B || !offsets || !C || !A_rows) return MOE_ERR_INVALID;
  if (ab_dtype != MOE_BF16 && !is_e4m3(ab_dtype)) return MOE_ERR_INVALID;
  if (epilogue != MOE_EPI_NONE && epilogue != MOE_EPI_SILU_GATE) return MOE_ERR_INVALID;
  if (is_e4m3(ab_dtype) && (!A_scales || !B_scales)) return MOE_ERR_INVALID;
  if (is_e4m3(c_dtype) && !C_scales) return MOE_ERR_INVALID;
  if (is_e4m3(c_dtype) && c_dtype != ab_dtype) return MOE_ERR_UNSUPPORTED;
  if (ab_dtype == MOE_BF16 && K % 64 != 0) return MOE_ERR_UNSUPPORTED;
  if (is_e4m3(ab_dtype) && K % 128 != 0) return MOE_ERR_UNSUPPORTED;
  if (!aligned(A, 16) || !aligned(B, 16) || !aligned(C, 16)) return MOE_ERR_INVALID;
  if (!ws || !aligned(ws, 256)) return MOE_ERR_WORKSPACE;
  if (ws_bytes < moe_grouped_gemm_workspace_size()) return MOE_ERR_WORKSPACE;
  GemmArgs a{};
  a.A = A;
  a.A_scales = A_scales;
  a.a_rows = A_rows;
  a.a_src_rows = A_src_rows;
  a.B = B;
  a.B_scales = B_scales;
  a.offsets = offsets;
  a.G = G;
  a.rows = rows;
  a.N = N;
  a.K = K;
  a.ab_dtype = ab_dtype;
  a.epilogue = epilogue;
  a.c_dtype = c_dtype;
  a.C = C;
  a.C_scales = C_scales;
  if (!plan_takes_gathered_a(plan_grouped_gemm(a, num_sms()))) return MOE_ERR_UNSUPPORTED;
  cudaStream_t s = as_stream(stream);
  MOE_CUDA_CHECK(cudaMemsetAsync(ws, 0, sizeof(int), s));
  a.status = static_cast<int*>(ws);
  return launch_grouped_gemm(a, s);
}

// ------------------------------------------------------------------ failure-detection self-test
size_t moe_selftest_workspace_size(void) { return 1024 + (16 + 128 + 256) * 1024; }

int moe_selftest_stalled_pipeline(void* ws, size_t ws_bytes, unsigned long long wait_limit_ns, void* stream) {
  if (!ws || !aligned(ws, 256) || ws_bytes < moe_selftest_workspace_size()) return MOE_ERR_WORKSPACE;
  if (wait_limit_ns < 1000000ull || wait_limit_ns > 2000000000ull) return MOE_ERR_INVALID;
  cudaStream_t s = as_stream(stream);
  char* base = static_cast<char*>(ws);
  void* A = base + 1024;                 // [128, 64] bf16
  void* B = base + 1024 + 16 * 1024;     // [1024, 64] bf16
  void* C = base + 1024 + 144 * 1024;    // [128, 1024] bf16
  MOE_CUDA_CHECK(cudaMemsetAsync(ws, 0, 1024 + 144 * 1024, s));
  GemmArgs g{};
  g.A = A;
  g.B = B;
  g.offsets = nullptr;  // one group of 128 rows: four 256-column tiles on one CTA
  g.G = 1;
  g.rows = 128;
  g.N = 1024;
  g.K = 64;
  g.mma_n = 256;
  g.pair_tiles = -1;
  g.ab_dtype = MOE_BF16;
  g.epilogue = MOE_EPI_NONE;
  g.c_dtype = MOE_BF16;
  g.C = C;
  g.status = static_cast<int*>(ws);
  g.wait_ns = wait_limit_ns;
  g.stall = 1;
  g.grid = 1;
  return launch_grouped_gemm(g, s);
}

const char* moe_grouped_gemm_plan(int G, int extra_groups, int rows, int N, int K, int ab_dtype, int epilogue,
                                  int c_dtype, int num_sms) {
  GemmArgs a{};
  a.G = G;
  a.has_extra = extra_groups ? 1 : 0;
  a.rows = rows;
  a.N = N;
  a.K = K;
  a.ab_dtype = ab_dtype;
  a.epilogue = epilogue;
  a.c_dtype = c_dtype;
  return gemm_variant_name(plan_grouped_gemm(a, num_sms > 0 ? num_sms : 148));
}

// ------------------------------------------------------------------ combine
int moe_combine(const void* Y, const int32_t* token_to_row, const float* topk_w, int has_shared, int T, int d, int k,
                void* out, int out_dtype, void* stream) {
  if (T < 0 || d <= 0 || k <= 0 || k > kMaxTopK) return MOE_ERR_INVALID;
  if (d % 8 != 0) return MOE_ERR_UNSUPPORTED;
  if (out_dtype != MOE_F32 && out_dtype != MOE_BF16) return MOE_ERR_INVALID;
  if (T > 0 && (!Y || !token_to_row || !topk_w || !out)) return MOE_ERR_INVALID;
  if (!aligned(Y, 16) || !aligned(out, 16)) return MOE_ERR_INVALID;
  return launch_combine(Y, token_to_row, topk_w, has_shared, T, d, k, out, out_dtype, as_stream(stream));
}

int moe_combine_plan(const void* Y, const int32_t* token_to_row, const float* topk_w, const int32_t* offsets, int E,
                     int has_shared, int T, int d, int k, void* out, int out_dtype, void* stream) {
  if (T < 0 || d <= 0 || k <= 0 || k > kMaxTopK || E <= 0 || E > kMaxExperts) return MOE_ERR_INVALID;
  if (d % 8 != 0) return MOE_ERR_UNSUPPORTED;
  if (out_dtype != MOE_F32 && out_dtype != MOE_BF16) return MOE_ERR_INVALID;
  if (T > 0 && (!Y || !token_to_row || !topk_w || !out || !offsets)) return MOE_ERR_INVALID;
  if (!aligned(Y, 16) || !aligned(out, 16)) return MOE_ERR_INVALID;
  return launch_combine(Y, token_to_row, topk_w, has_shared, T, d, k, out, out_dtype, as_stream(stream),
                        T > 0 ? offsets + E : nullptr);
}

// ------------------------------------------------------------------ FP8 weights
int moe_quantize_weights_fp8(const void* W, int G, int N, int K, uint8_t* Wq, float* scales, void* stream) {
  if (G < 0 || N <= 0 || K <= 0) return MOE_ERR_INVALID;
  if (N % 128 != 0 || K % 128 != 0) return MOE_ERR_UNSUPPORTED;
  if (G > 0 && (!W || !Wq || !scales)) return MOE_ERR_INVALID;
  if (!aligned(W, 16) || !aligned(Wq, 16)) return MOE_ERR_INVALID;
  return launch_quantize_weights(W, G, N, K, Wq, scales, as_stream(stream));
}

int moe_quantize_weights_mx(const void* W, int G, int N, int K, uint8_t* Wq, float* scales, void* stream) {
  if (G < 0 || N <= 0 || K <= 0) return MOE_ERR_INVALID;
  if (N % 128 != 0 || K % 128 != 0) return MOE_ERR_UNSUPPORTED;
  if (G > 0 && (!W || !Wq || !scales)) return MOE_ERR_INVALID;
  if (!aligned(W, 16) || !aligned(Wq, 16)) return MOE_ERR_INVALID;
  return launch_quantize_weights(W, G, N, K, Wq, scales, as_stream(stream), true);
}

// ------------------------------------------------------------------ whole layer
size_t moe_workspace_size(const moe_config* cfg) {
  if (check_config(cfg) != MOE_OK) return 0;
  return fwd_layout(*cfg).total;
}

namespace {

// The layer's five stages; `marks` (or NULL) gets one event recorded before
// each stage and one after the last.
int forward_impl(const moe_config* cfg, const void* x, const void* W_r, const float* router_bias, const void* W1,
                 const float* W1_scales, const void* W2, const float* W2_scales, const void* W1_shared,
                 const float* W1s_scales, const void* W2_shared, const float* W2s_scales, void* out,
                 int32_t* counts_out, void* ws, size_t ws_bytes, void* stream, void* const* marks) {
  int st = check_config(cfg);
  if (st != MOE_OK) return st;
  const moe_config c = *cfg;
  const bool fp8 = is_e4m3(c.expert_dtype);
  const int qdt = c.expert_dtype;  // MOE_E4M3 or MOE_MXE4M3 when fp8
  const bool shared = c.shared_inter != 0;
  if (c.T > 0 && (!x || !W_r || !W1 || !W2 || !out)) return MOE_ERR_INVALID;
  if (shared && (!W1_shared || !W2_shared)) return MOE_ERR_INVALID;
  if (fp8 && (!W1_scales || !W2_scales || (shared && (!W1s_scales || !W2s_scales)))) return MOE_ERR_INVALID;
  if (!aligned(x, 16) || !aligned(W_r, 16) || !aligned(W1, 16) || !aligned(W2, 16) || !aligned(out, 16) ||
      !aligned(W1_shared, 16) || !aligned(W2_shared, 16))
    return MOE_ERR_INVALID;
  if (!ws || !aligned(ws, 256)) return MOE_ERR_WORKSPACE;
  const FwdLayout L = fwd_layout(c);
  if (ws_bytes < L.total) return MOE_ERR_WORKSPACE;
  cudaStream_t s = as_stream(stream);
  char* base = static_cast<char*>(ws);
  int* status = reinterpret_cast<int*>(base + L.status);
  int32_t* idx = reinterpret_cast<int32_t*>(base + L.idx);
  float* w = reinterpret_cast<float*>(base + L.w);
  int32_t* counts = reinterpret_cast<int32_t*>(base + L.counts);
  int32_t* offsets = reinterpret_cast<int32_t*>(base + L.offsets);
  int32_t* t2r = reinterpret_cast<int32_t*>(base + L.t2r);
  MOE_CUDA_CHECK(cudaMemsetAsync(status, 0, sizeof(int), s));
  if (c.T == 0) {
    if (counts_out) MOE_CUDA_CHECK(cudaMemsetAsync(counts_out, 0, sizeof(int32_t) * c.E, s));
    return MOE_OK;
  }
  const int T = c.T, d = c.d, E = c.E, k = c.k, I = c.inter;
  const int Rp = T * k + (shared ? T : 0);
  auto mark = [&](int i) -> int {
    if (marks) MOE_CUDA_CHECK(cudaEventRecord(static_cast<cudaEvent_t>(marks[i]), s));
    return MOE_OK;
  };

  if ((st = mark(0)) != MOE_OK) return st;
  st = launch_router(x, c.x_dtype, W_r, c.router_dtype, router_bias, T, d, E, k, c.renormalize, nullptr, idx, w,
                     reinterpret_cast<float*>(base + L.logits), status, s);
  if (st != MOE_OK) return st;
  if ((st = mark(1)) != MOE_OK) return st;

  // "Permute in the load" (MOE_FLAG_GATHER_A): when the up GEMM runs on a
  // single-CTA kernel it gathers its A rows through row_to_token
  // (tile::gather4), so the permute writes only the plan (plus, for E4M3
  // experts or fp32 x, each token's row once, quantised or cast) and the
  // expert-ordered copy of x is never made.
  GemmArgs up{};
  up.B = W1;
  up.B_extra = W1_shared;
  up.offsets = offsets;
  up.G = E;
  up.has_extra = shared ? 1 : 0;
  up.rows = Rp;
  up.N = I;
  up.K = d;
  up.ab_dtype = fp8 ? qdt : MOE_BF16;
  up.epilogue = MOE_EPI_SILU_GATE;
  up.c_dtype = fp8 ? qdt : MOE_BF16;
  up.C = base + L.h;
  up.status = status;
  const bool gather = (c.flags & MOE_FLAG_GATHER_A) && plan_takes_gathered_a(plan_grouped_gemm(up, num_sms()));
  const bool x_as_is = gather && !fp8 && c.x_dtype == MOE_BF16;  // the GEMM reads x itself

  PermuteArgs pa;
  pa.x = x;
  pa.x_dtype = c.x_dtype;
  pa.idx = idx;
  pa.T = T;
  pa.d = d;
  pa.E = E;
  pa.k = k;
  pa.shared = shared ? 1 : 0;
  pa.xp_dtype = fp8 ? qdt : MOE_BF16;
  pa.xp = base + L.xp;
  pa.xp_scales = fp8 ? reinterpret_cast<float*>(base + L.xps) : nullptr;
  pa.counts = counts;
  pa.offsets = offsets;
  pa.row_to_token = reinterpret_cast<int32_t*>(base + L.r2t);
  pa.token_to_row = t2r;
  pa.block_base = reinterpret_cast<int32_t*>(base + L.base);
  pa.status = status;
  pa.capacity = c.capacity;
  pa.gather = gather ? 1 : 0;
  st = launch_permute(pa, s);
  if (st != MOE_OK) return st;
  if ((st = mark(2)) != MOE_OK) return st;

  up.A = x_as_is ? x : base + L.xp;
  if (gather) {
    up.a_rows = pa.row_to_token;
    up.a_src_rows = T;
  }
  if (fp8) {
    up.A_scales = reinterpret_cast<const float*>(base + L.xps);
    up.B_scales = W1_scales;
    up.B_extra_scales = W1s_scales;
    up.C_scales = reinterpret_cast<float*>(base + L.hs);
  }
  st = launch_grouped_gemm(up, s);
  if (st != MOE_OK) return st;
  if ((st = mark(3)) != MOE_OK) return st;

  GemmArgs dn{};
  dn.A = base + L.h;
  dn.B = W2;
  dn.B_extra = W2_shared;
  dn.offsets = offsets;
  dn.G = E;
  dn.has_extra = shared ? 1 : 0;
  dn.rows = Rp;
  dn.N = d;
  dn.K = I;
  dn.ab_dtype = fp8 ? qdt : MOE_BF16;
  dn.epilogue = MOE_EPI_NONE;
  dn.c_dtype = MOE_BF16;
  dn.C = base + L.y;
  dn.status = status;
  if (fp8) {
    dn.A_scales = reinterpret_cast<const float*>(base + L.hs);
    dn.B_scales = W2_scales;
    dn.B_extra_scales = W2s_scales;
  }
  st = launch_grouped_gemm(dn, s);
  if (st != MOE_OK) return st;
  if ((st = mark(4)) != MOE_OK) return st;

  st = launch_combine(base + L.y, t2r, w, shared ? 1 : 0, T, d, k, out, c.out_dtype, s, offsets + E);
  if (st != MOE_OK) return st;
  if ((st = mark(5)) != MOE_OK) return st;
  if (counts_out) MOE_CUDA_CHECK(cudaMemcpyAsync(counts_out, counts, sizeof(int32_t) * E, cudaMemcpyDeviceToDevice, s));
  return MOE_OK;
}

}  // namespace

int moe_forward(const moe_config* cfg, const void* x, const void* W_r, const float* router_bias, const void* W1,
                const float* W1_scales, const void* W2, const float* W2_scales, const void* W1_shared,
                const float* W1s_scales, const void* W2_shared, const float* W2s_scales, void* out,
                int32_t* counts_out, void* ws, size_t ws_bytes, void* stream) {
  return forward_impl(cfg, x, W_r, router_bias, W1, W1_scales, W2, W2_scales, W1_shared, W1s_scales, W2_shared,
                      W2s_scales, out, counts_out, ws, ws_bytes, stream, nullptr);
}

int moe_forward_marked(const moe_config* cfg, const void* x, const void* W_r, const float* router_bias,
                       const void* W1, const float* W1_scales, const void* W2, const float* W2_scales,
                       const void* W1_shared, const float* W1s_scales, const void* W2_shared,
                       const float* W2s_scales, void* out, int32_t* counts_out, void* ws, size_t ws_bytes,
                       void* const* stage_events, void* stream) {
  if (!stage_events) return MOE_ERR_INVALID;
  for (int i = 0; i < 6; ++i)
    if (!stage_events[i]) return MOE_ERR_INVALID;
  return forward_impl(cfg, x, W_r, router_bias, W1, W1_scales, W2, W2_scales, W1_shared, W1s_scales, W2_shared,
                      W2s_scales, out, counts_out, ws, ws_bytes, stream, stage_events);
}

int moe_forward_launches(const moe_config* cfg) {
  if (check_config(cfg) != MOE_OK) return -1;
  if (cfg->T == 0) return 0;
  const int router =
      router_is_fused(cfg->x_dtype, cfg->router_dtype, cfg->T, cfg->d, cfg->E, cfg->k) ? 1 : 2;  // or logits + selection
  const int permute = permute_fuses_scan(cfg->T, cfg->E) ? 2 : 3;      // histogram, (scan,) scatter
  return router + permute + 2 /* grouped GEMMs */ + 1 /* combine */;
}

size_t moe_host_staging_size(const moe_config* cfg) {
  if (check_config(cfg) != MOE_OK) return 0;
  const size_t td = static_cast<size_t>(cfg->T) * cfg->d;
  return align_up(td * dtype_bytes(cfg->x_dtype), 1024) + align_up(td * dtype_bytes(cfg->out_dtype), 1024);
}

int moe_forward_host(const moe_config* cfg, const void* x_host, const void* W_r, const float* router_bias,
                     const void* W1, const float* W1_scales, const void* W2, const float* W2_scales,
                     const void* W1_shared, const float* W1s_scales, const void* W2_shared, const float* W2s_scales,
                     void* out_host, void* ws, size_t ws_bytes, void* stream) {
  int st = check_config(cfg);
  if (st != MOE_OK) return st;
  if (cfg->T > 0 && (!x_host || !out_host)) return MOE_ERR_INVALID;
  if (!ws || !aligned(ws, 256)) return MOE_ERR_WORKSPACE;
  const size_t fwd = moe_workspace_size(cfg);
  if (ws_bytes < fwd + moe_host_staging_size(cfg)) return MOE_ERR_WORKSPACE;
  cudaStream_t s = as_stream(stream);
  const size_t td = static_cast<size_t>(cfg->T) * cfg->d;
  char* xd = static_cast<char*>(ws) + fwd;
  char* od = xd + align_up(td * dtype_bytes(cfg->x_dtype), 1024);
  if (td) MOE_CUDA_CHECK(cudaMemcpyAsync(xd, x_host, td * dtype_bytes(cfg->x_dtype), cudaMemcpyHostToDevice, s));
  st = moe_forward(cfg, xd, W_r, router_bias, W1, W1_scales, W2, W2_scales, W1_shared, W1s_scales, W2_shared,
                   W2s_scales, od, nullptr, ws, fwd, stream);
  if (st != MOE_OK) return st;
  if (td) MOE_CUDA_CHECK(cudaMemcpyAsync(out_host, od, td * dtype_bytes(cfg->out_dtype), cudaMemcpyDeviceToHost, s));
  return MOE_OK;
}

}  // extern "C"
