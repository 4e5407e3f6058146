// Shared definitions of the library's translation units: status handling,
// small device helpers and the internal launcher interfaces the C ABI layer
// (moe_api.cu) composes.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <utility>

#include <cstdint>

#include "moe.h"

namespace moe {

constexpr int kMaxGroups = 1024;     // experts (+ shared) one grouped GEMM launch handles
constexpr int kMaxTopK = 32;
constexpr int kMaxExperts = 1024;
// Rows of a permuted buffer (T*k + T) are int32 indices in the kernels.
constexpr long long kMaxPermuteRows = 1ll << 30;
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s per pipeline wait

// Record the first device-side error in the status word (0 = OK).
__device__ __forceinline__ void set_status(int* status, int code) {
  if (status) atomicCAS(status, 0, code);
}

__device__ __forceinline__ float bf16_bits_to_float(uint16_t b) {
  return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

template <typename T>
__device__ __forceinline__ float to_f32(T v);
template <>
__device__ __forceinline__ float to_f32<float>(float v) { return v; }
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 v) { return __bfloat162float(v); }
template <>
__device__ __forceinline__ float to_f32<__half>(__half v) { return __half2float(v); }

// Two fp32 -> packed E4M3 pair (round to nearest even, saturating to +-448);
// `lo` lands in the low byte.
__device__ __forceinline__ uint16_t f32x2_to_e4m3x2(float lo, float hi) {
  return static_cast<uint16_t>(__nv_cvt_float2_to_fp8x2(make_float2(lo, hi), __NV_SATFINITE, __NV_E4M3));
}

// Scale of a quantisation group with largest magnitude amax.
//   fp32 scales:  s = amax / 448 (IEEE division), 1 for amax = 0;
//   MX (pow2):    s = 2^p with p the smallest integer such that 448 * 2^p >= amax,
//                 clamped to [-127, 127] (an 8-bit exponent carries it), 1 for amax = 0.
// With amax = (1 + m / 2^23) 2^e and 448 = 1.75 * 2^8: amax / 448 lies in
// (2^(e-9), 2^(e-8)] when 1 + m / 2^23 <= 1.75 (mantissa bits <= 0x600000),
// else in (2^(e-8), 2^(e-7)); a subnormal amax gives p below -127.
__device__ __forceinline__ int pow2_exponent(float amax) {
  const uint32_t b = __float_as_uint(amax) & 0x7fffffffu;
  const int ef = static_cast<int>(b >> 23);
  if (ef == 0) return b ? -127 : 0;
  const int p = ef - 127 - 8 + ((b & 0x7fffffu) > 0x600000u ? 1 : 0);
  return p < -127 ? -127 : p;
}
__device__ __forceinline__ float pow2_value(int p) {  // 2^p for -127 <= p <= 127
  return p >= -126 ? __uint_as_float(static_cast<uint32_t>(p + 127) << 23) : __uint_as_float(0x00400000u);
}
template <bool kPow2>
__device__ __forceinline__ float group_scale(float amax) {
  if constexpr (kPow2) {
    return amax > 0.f ? pow2_value(pow2_exponent(amax)) : 1.0f;
  } else {
    return amax > 0.f ? __fdiv_rn(amax, 448.0f) : 1.0f;
  }
}

inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }
inline bool is_e4m3(int dt) { return dt == MOE_E4M3 || dt == MOE_MXE4M3; }

// ---------------------------------------------------------------- launchers
// Each returns a moe_status; they assume arguments were validated.

constexpr int kRouterMaxSplit = 8;  // K slices of the tensor-core router
// parts: scratch of kRouterMaxSplit * T * router_padded_experts(E) fp32 (partial logits)
int launch_router(const void* x, int x_dtype, const void* W_r, int w_dtype, const float* bias, int T, int d, int E,
                  int k, int renorm, float* logits_out, int32_t* idx, float* w, float* parts, int* status,
                  cudaStream_t s);
bool router_uses_tensor_cores(int x_dtype, int w_dtype, int T, int d, int E);
// one launch (logits + softmax + top-k on chip)
bool router_is_fused(int x_dtype, int w_dtype, int T, int d, int E, int k);
// the tensor-core router (router_tc.cu): bf16 x and W_r, E <= 256, k <= 8
bool router_tc_applies(int x_dtype, int w_dtype, int d, int E, int k);
int launch_router_tc(const void* x, const void* W_r, const float* bias, int T, int d, int E, int k, int renorm,
                     float* logits_out, int32_t* idx, float* w, int* status, cudaStream_t s);
int router_padded_experts(int E);  // logits columns the tensor-core router computes
int launch_topk_logits(const void* logits, int dtype, int N, int E, int k, int renorm, int32_t* idx,
                       float* w, cudaStream_t s);

struct PermuteArgs {
  const void* x;
  int x_dtype;
  const int32_t* idx;
  int T, d, E, k, shared, xp_dtype;
  void* xp;
  float* xp_scales;
  int32_t* counts;
  int32_t* offsets;
  int32_t* row_to_token;
  int32_t* token_to_row;
  int32_t* block_base;  // scratch [nblocks * E]
  int* status;
  int capacity = 0;     // > 0: an expert keeps only its first `capacity` pairs in token order
  // 1: the grouped GEMM gathers its A rows through row_to_token, so xp is
  // [T, d] with each token's row once (cast / quantised as xp_dtype says,
  // scales [d/128][T]); with bf16 x and a bf16 xp nothing is copied at all
  int gather = 0;
  int fuse_scan = 0;  // set by launch_permute (permute_fuses_scan)
};
// The scatter computes the expert offsets and its block's bases itself from
// the histogram (no separate scan launch) when the count matrix is this small.
constexpr int kFusedScanCounts = 8192;
bool permute_fuses_scan(int T, int E);
int permute_blocks(int T);  // number of token blocks the permute kernels use
int launch_permute(const PermuteArgs& a, cudaStream_t s);

struct GemmArgs {
  const void* A;
  const float* A_scales;
  const void* B;            // [G, Nb, K]
  const float* B_scales;
  const void* B_extra;      // optional extra group (index G) with its own [Nb, K] weights
  const float* B_extra_scales;
  const int32_t* offsets;   // [G + has_extra + 1]
  const int32_t* a_rows;    // gather: A row r is row a_rows[r] of A (< 0: any row); A has a_src_rows rows
  int a_src_rows;
  int G, has_extra, rows, N, K;
  int B_rows;               // > 0: rows of B actually present (G == 1); rows past it read as zero
  int ksplit;               // > 1: fp32 partial products of K slices at C + s * rows * N (no epilogue)
  int mma_n;                // 0 = widest tile that divides N; else 64 / 128 / 256 (no-gate GEMMs)
  int pair_tiles;           // 256-row tiles on CTA pairs: 0 = by average group size, 1 = always, -1 = never
  uint64_t wait_ns;         // pipeline wait limit (0 = the default of 2 s)
  int stall;                // failure-detection self-test (see moe_selftest_stalled_pipeline)
  int grid;                 // CTAs (0 = one per SM)
  int swap_ab;              // weights on the MMA's 128-row side: 0 = for small groups, 1 = always, -1 = never
  int ab_dtype, epilogue, c_dtype;
  void* C;
  float* C_scales;
  int* status;
};
int launch_grouped_gemm(const GemmArgs& a, cudaStream_t s);
int plan_grouped_gemm(const GemmArgs& a, int sms);  // host-only choice of kernel (see gemm_variant_name)
bool plan_takes_gathered_a(int variant);            // the variant can load A rows through a_rows
const char* gemm_variant_name(int variant);

// shared_base: device int32 holding the first shared row (offsets[E] of the
// permute), or nullptr for the fixed T*k.  token_to_row entries < 0 are
// slots that overflowed an expert's capacity and are skipped.
int launch_combine(const void* Y, const int32_t* t2r, const float* w, int has_shared, int T, int d, int k,
                   void* out, int out_dtype, cudaStream_t s, const int32_t* shared_base = nullptr);
// pow2: power-of-two (MX) block scales instead of amax / 448
int launch_quantize_weights(const void* W, int G, int N, int K, uint8_t* Wq, float* scales, cudaStream_t s,
                            bool pow2 = false);

int num_sms();

}  // namespace moe

namespace moe {
// Remember the last failing CUDA call (per host thread) for moe_last_error_string.
int record_cuda_error(cudaError_t e, const char* where);
// Status of the kernel launch just made.
inline int launch_status(const char* where) {
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? MOE_OK : record_cuda_error(e, where);
}

// silu(g) = g / (1 + e^-g) with the fast reciprocal-based division (a few ulp;
// for g below about -87 the denominator overflows and the result is -0, the
// limit of the function).
__device__ __forceinline__ float silu(float g) { return __fdividef(g, 1.0f + __expf(-g)); }

// Programmatic dependent launch.  Every kernel of the library is launched so
// that it may start while the kernel before it on the stream is finishing,
// and every kernel begins with pdl_wait(), which returns once the preceding
// grid has completed and its memory is visible: no kernel touches global
// memory before that.  pdl_launch_dependents() lets the next kernel's CTAs
// be scheduled as soon as every CTA of this grid has issued it.  Both are
// no-ops for a kernel launched without the attribute.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Launch `kernel` on `s` with programmatic stream serialisation allowed.
template <typename... Params, typename... Args>
int launch_pdl(const char* where, void (*kernel)(Params...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
               Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
  return e == cudaSuccess ? MOE_OK : record_cuda_error(e, where);
}
}  // namespace moe

#define MOE_CUDA_CHECK(expr)                                            \
  do {                                                                  \
    cudaError_t _e = (expr);                                            \
    if (_e != cudaSuccess) return ::moe::record_cuda_error(_e, #expr);  \
  } while (0)
