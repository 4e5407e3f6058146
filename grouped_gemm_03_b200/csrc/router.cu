// Router: logits = x W_r^T (+ bias), softmax over all experts, top-k.
//
// "MegaMoE math model -> DeepGEMM source walk-through" §2.1 (p = Softmax(W_r x_t),
// keep the k best) and "Dense GEMM -> GroupedGEMM -> TP MoE" §4.2 (route_tokens).
// One warp owns one token: the dot products are split over the lanes along d
// and reduced with shuffles, then k rounds of a warp-wide arg-max on
// (logit descending, expert index ascending) pick the experts.  Selection
// compares logits, so equal probabilities never reorder it; the weight of a
// selected expert is its softmax value (or that value over the sum of the
// selected ones when renormalising).
#include <cfloat>
#include <climits>

#include "common.cuh"

namespace moe {
namespace {

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Softmax + top-k over the values a warp holds in registers: lane `lane`
// holds v[i] for expert ix[i] (ix = INT_MAX marks padding, v = -inf).
template <int V>
__device__ __forceinline__ void warp_select(float (&v)[V], const int (&ix)[V], int k, int renorm, int lane,
                                            int32_t* idx_out, float* w_out) {
  float m = -FLT_MAX;
#pragma unroll
  for (int i = 0; i < V; ++i) m = fmaxf(m, v[i]);
  m = warp_max(m);
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < V; ++i)
    if (ix[i] != INT_MAX) s += expf(v[i] - m);
  s = warp_sum(s);

  float my_p = 0.f;
  int my_i = 0;
  for (int j = 0; j < k; ++j) {
    float bv = -INFINITY;
    int bi = INT_MAX;
#pragma unroll
    for (int i = 0; i < V; ++i)
      if (v[i] > bv || (v[i] == bv && ix[i] < bi)) {
        bv = v[i];
        bi = ix[i];
      }
#pragma unroll
    for (int o = 16; o; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (ov > bv || (ov == bv && oi < bi)) {
        bv = ov;
        bi = oi;
      }
    }
    if (lane == j) {
      my_i = bi;
      my_p = expf(bv - m) / s;
    }
#pragma unroll
    for (int i = 0; i < V; ++i)
      if (ix[i] == bi) v[i] = -INFINITY;
  }
  if (renorm) {
    const float ps = warp_sum(lane < k ? my_p : 0.f);
    my_p = my_p / ps;
  }
  if (lane < k) {
    idx_out[lane] = my_i;
    w_out[lane] = my_p;
  }
}

// 8 consecutive elements as fp32 (16- or 32-byte vector loads).
__device__ __forceinline__ void load8(const float* p, float (&f)[8]) {
  const float4 a = __ldg(reinterpret_cast<const float4*>(p));
  const float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
  f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
  f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
}
__device__ __forceinline__ void load8(const __nv_bfloat16* p, float (&f)[8]) {
  const uint4 a = __ldg(reinterpret_cast<const uint4*>(p));
  const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}
constexpr int kRouterWarps = 8;

// Fused logits + softmax + top-k, one warp per token.
template <typename XT, typename WT, int V>
__global__ void __launch_bounds__(kRouterWarps * 32) router_simt_kernel(
    const XT* __restrict__ x, const WT* __restrict__ Wr, const float* __restrict__ bias, int T, int d, int E,
    int k, int renorm, float* __restrict__ logits_out, int32_t* __restrict__ idx_out,
    float* __restrict__ w_out) {
  extern __shared__ float s_logit[];  // [kRouterWarps][E]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float* lg = s_logit + warp * E;
  for (int t = blockIdx.x * kRouterWarps + warp; t < T; t += gridDim.x * kRouterWarps) {
    const XT* xr = x + static_cast<size_t>(t) * d;
    for (int e0 = 0; e0 < E; e0 += 8) {
      const int ne = min(8, E - e0);
      float acc[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) acc[j] = 0.f;
      for (int c = lane * 8; c < d; c += 32 * 8) {
        float xv[8];
        load8(xr + c, xv);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if (j < ne) {
            float wv[8];
            load8(Wr + static_cast<size_t>(e0 + j) * d + c, wv);
#pragma unroll
            for (int q = 0; q < 8; ++q) acc[j] = fmaf(xv[q], wv[q], acc[j]);
          }
        }
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) acc[j] = warp_sum(acc[j]);
      if (lane < ne) {
        float a = acc[0];
#pragma unroll
        for (int j = 1; j < 8; ++j)
          if (lane == j) a = acc[j];
        lg[e0 + lane] = a + (bias ? bias[e0 + lane] : 0.f);
      }
    }
    __syncwarp();
    float v[V];
    int ix[V];
#pragma unroll
    for (int i = 0; i < V; ++i) {
      const int e = lane + 32 * i;
      ix[i] = e < E ? e : INT_MAX;
      v[i] = e < E ? lg[e] : -INFINITY;
    }
    if (logits_out)
      for (int e = lane; e < E; e += 32) logits_out[static_cast<size_t>(t) * E + e] = lg[e];
    warp_select<V>(v, ix, k, renorm, lane, idx_out + static_cast<size_t>(t) * k,
                   w_out + static_cast<size_t>(t) * k);
    __syncwarp();
  }
}

// Softmax + top-k of stored logits, one warp per token; lane l holds the
// V consecutive experts l*V .. l*V+V-1.
template <typename LT, int V>
__global__ void __launch_bounds__(256) topk_logits_kernel(const LT* __restrict__ logits, int N, int E, int k,
                                                          int renorm, int32_t* __restrict__ idx_out,
                                                          float* __restrict__ w_out) {
  const int lane = threadIdx.x & 31;
  const int warps = gridDim.x * (blockDim.x >> 5);
  const bool vec = (E == 32 * V) && (V * sizeof(LT)) % 8 == 0;
  for (int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); t < N; t += warps) {
    const LT* row = logits + static_cast<size_t>(t) * E;
    float v[V];
    int ix[V];
    if (vec && V * sizeof(LT) == 8) {
      const uint2 raw = __ldg(reinterpret_cast<const uint2*>(row) + lane);
      const LT* pv = reinterpret_cast<const LT*>(&raw);
#pragma unroll
      for (int i = 0; i < V; ++i) {
        v[i] = to_f32(pv[i]);
        ix[i] = lane * V + i;
      }
    } else if (vec && V * sizeof(LT) == 16) {
      const uint4 raw = __ldg(reinterpret_cast<const uint4*>(row) + lane);
      const LT* pv = reinterpret_cast<const LT*>(&raw);
#pragma unroll
      for (int i = 0; i < V; ++i) {
        v[i] = to_f32(pv[i]);
        ix[i] = lane * V + i;
      }
    } else {
#pragma unroll
      for (int i = 0; i < V; ++i) {
        const int e = lane * V + i;
        ix[i] = e < E ? e : INT_MAX;
        v[i] = e < E ? to_f32(row[e]) : -INFINITY;
      }
    }
    warp_select<V>(v, ix, k, renorm, lane, idx_out + static_cast<size_t>(t) * k,
                   w_out + static_cast<size_t>(t) * k);
  }
}

template <typename XT, typename WT>
int router_dispatch(const void* x, const void* Wr, const float* bias, int T, int d, int E, int k, int renorm,
                    float* lo, int32_t* idx, float* w, cudaStream_t s) {
  const int blocks = min((T + kRouterWarps - 1) / kRouterWarps, num_sms() * 8);
  const size_t smem = static_cast<size_t>(kRouterWarps) * E * sizeof(float);
  const XT* xp = static_cast<const XT*>(x);
  const WT* wp = static_cast<const WT*>(Wr);
  const int v = (E + 31) / 32;
#define MOE_ROUTER_CASE(VV)                                                                                  \
  if (v <= VV) {                                                                                            \
    router_simt_kernel<XT, WT, VV><<<blocks, kRouterWarps * 32, smem, s>>>(xp, wp, bias, T, d, E, k, renorm, \
                                                                          lo, idx, w);                     \
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;                                       \
  }
  MOE_ROUTER_CASE(1)
  MOE_ROUTER_CASE(2)
  MOE_ROUTER_CASE(4)
  MOE_ROUTER_CASE(8)
  MOE_ROUTER_CASE(16)
  MOE_ROUTER_CASE(32)
#undef MOE_ROUTER_CASE
  return MOE_ERR_UNSUPPORTED;
}

template <typename LT>
int topk_dispatch(const void* logits, int N, int E, int k, int renorm, int32_t* idx, float* w, cudaStream_t s) {
  const int warps_per_block = 8;
  const int blocks = max(1, min((N + warps_per_block - 1) / warps_per_block, num_sms() * 16));
  const LT* lp = static_cast<const LT*>(logits);
  const int v = (E + 31) / 32;
#define MOE_TOPK_CASE(VV)                                                                                    \
  if (v <= VV) {                                                                                            \
    topk_logits_kernel<LT, VV><<<blocks, warps_per_block * 32, 0, s>>>(lp, N, E, k, renorm, idx, w);         \
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;                                       \
  }
  MOE_TOPK_CASE(1)
  MOE_TOPK_CASE(2)
  MOE_TOPK_CASE(4)
  MOE_TOPK_CASE(8)
  MOE_TOPK_CASE(16)
  MOE_TOPK_CASE(32)
#undef MOE_TOPK_CASE
  return MOE_ERR_UNSUPPORTED;
}

}  // namespace

int launch_router_simt(const void* x, int x_dtype, const void* W_r, int w_dtype, const float* bias, int T,
                       int d, int E, int k, int renorm, float* logits_out, int32_t* idx, float* w,
                       cudaStream_t s) {
  if (T == 0) return MOE_OK;
  if (x_dtype == MOE_BF16 && w_dtype == MOE_BF16)
    return router_dispatch<__nv_bfloat16, __nv_bfloat16>(x, W_r, bias, T, d, E, k, renorm, logits_out, idx, w, s);
  if (x_dtype == MOE_F32 && w_dtype == MOE_F32)
    return router_dispatch<float, float>(x, W_r, bias, T, d, E, k, renorm, logits_out, idx, w, s);
  if (x_dtype == MOE_F32 && w_dtype == MOE_BF16)
    return router_dispatch<float, __nv_bfloat16>(x, W_r, bias, T, d, E, k, renorm, logits_out, idx, w, s);
  if (x_dtype == MOE_BF16 && w_dtype == MOE_F32)
    return router_dispatch<__nv_bfloat16, float>(x, W_r, bias, T, d, E, k, renorm, logits_out, idx, w, s);
  return MOE_ERR_UNSUPPORTED;
}

int launch_topk_logits(const void* logits, int dtype, int N, int E, int k, int renorm, int32_t* idx, float* w,
                       cudaStream_t s) {
  if (N == 0) return MOE_OK;
  if (dtype == MOE_F16) return topk_dispatch<__half>(logits, N, E, k, renorm, idx, w, s);
  if (dtype == MOE_F32) return topk_dispatch<float>(logits, N, E, k, renorm, idx, w, s);
  if (dtype == MOE_BF16) return topk_dispatch<__nv_bfloat16>(logits, N, E, k, renorm, idx, w, s);
  return MOE_ERR_UNSUPPORTED;
}

}  // namespace moe
