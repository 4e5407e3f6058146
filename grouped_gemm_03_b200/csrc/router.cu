// Router: logits = x W_r^T (+ bias), softmax over all experts, top-k.
//
// "MegaMoE math model -> DeepGEMM source walk-through" §2.1 (p = Softmax(W_r x_t),
// keep the k best) and "Dense GEMM -> GroupedGEMM -> TP MoE" §4.2 (route_tokens).
// Two launches:
//   logits  either the grouped-GEMM kernel on the tensor cores (bf16, large
//           E and d: the logits GEMM is then near the compute ridge), split
//           along K into fp32 partial products, or a SIMT kernel that keeps
//           a block's W_r rows in shared memory (small E or d, fp32 inputs);
//   finish  one warp per token sums the partials in a fixed order, adds the
//           bias, and runs k rounds of a warp-wide arg-max on (logit
//           descending, expert index ascending) for the softmax + top-k.
// Selection compares logits, so equal probabilities never reorder it; the
// weight of a selected expert is its softmax value (or that value over the
// sum of the selected ones when renormalising).
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


// 8 consecutive elements as fp32.
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

// ------------------------------------------------------------------ SIMT logits
// Block = 16 tokens x 8 experts; each warp owns 2 tokens.  The block's W_r
// rows are staged in shared memory 32 KB at a time (2048 bf16 / 1024 fp32
// columns), so each block reads them once from L2 while x streams from HBM
// once per expert block; every lane keeps the next 8 columns of its tokens
// in flight while it multiplies the current ones.  Used when E or d is small
// (the logits are then bound by reading x) and for fp32 operands.
constexpr int kREC = 8;
constexpr int kTPW = 2;
constexpr int kRTok = 8 * kTPW;

template <typename T>
__device__ __forceinline__ void load8_any(const T* p, float (&f)[8]) {
  load8(p, f);
}

// 8 consecutive shared-memory elements as fp32.
__device__ __forceinline__ void smem8(const float* p, float (&f)[8]) {
  const float4 a = *reinterpret_cast<const float4*>(p);
  const float4 b = *(reinterpret_cast<const float4*>(p) + 1);
  f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
  f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
}
__device__ __forceinline__ void smem8(const __nv_bfloat16* p, float (&f)[8]) {
  const uint4 a = *reinterpret_cast<const uint4*>(p);
  const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}

template <typename XT, typename WT>
__global__ void __launch_bounds__(256) logits_simt_kernel(const XT* __restrict__ x, const WT* __restrict__ Wr,
                                                          int T, int d, int E, float* __restrict__ logits) {
  constexpr int DC = 32768 / (kREC * static_cast<int>(sizeof(WT)));  // columns per staged chunk
  constexpr int VPE = 16 / static_cast<int>(sizeof(WT));            // elements per 16-byte copy
  __shared__ __align__(16) WT s_w[kREC][DC];
  const int t0 = blockIdx.x * kRTok, e0 = blockIdx.y * kREC;
  const int ne = min(kREC, E - e0);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tw = t0 + warp * kTPW;
  float acc[kTPW][kREC];
#pragma unroll
  for (int i = 0; i < kTPW; ++i)
#pragma unroll
    for (int e = 0; e < kREC; ++e) acc[i][e] = 0.f;
  for (int c0 = 0; c0 < d; c0 += DC) {
    const int dc = min(DC, d - c0);
    __syncthreads();
    for (int i = threadIdx.x; i < kREC * (DC / VPE); i += blockDim.x) {
      const int e = i / (DC / VPE), c = (i % (DC / VPE)) * VPE;
      uint4 v = make_uint4(0, 0, 0, 0);
      if (e < ne && c < dc) v = __ldg(reinterpret_cast<const uint4*>(Wr + static_cast<size_t>(e0 + e) * d + c0 + c));
      *reinterpret_cast<uint4*>(&s_w[e][c]) = v;
    }
    __syncthreads();
    float xv[kTPW][8];
#pragma unroll
    for (int i = 0; i < kTPW; ++i) {
      const int c = lane * 8;
      if (tw + i < T && c < dc) {
        load8_any(x + static_cast<size_t>(tw + i) * d + c0 + c, xv[i]);
      } else {
#pragma unroll
        for (int q = 0; q < 8; ++q) xv[i][q] = 0.f;
      }
    }
    for (int c = lane * 8; c < dc; c += 256) {
      float xn[kTPW][8];
      const int cn = c + 256;
#pragma unroll
      for (int i = 0; i < kTPW; ++i) {
        if (tw + i < T && cn < dc) {
          load8_any(x + static_cast<size_t>(tw + i) * d + c0 + cn, xn[i]);
        } else {
#pragma unroll
          for (int q = 0; q < 8; ++q) xn[i][q] = 0.f;
        }
      }
#pragma unroll
      for (int e = 0; e < kREC; ++e) {
        float wv[8];
        smem8(&s_w[e][c], wv);
#pragma unroll
        for (int i = 0; i < kTPW; ++i)
#pragma unroll
          for (int q = 0; q < 8; ++q) acc[i][e] = fmaf(xv[i][q], wv[q], acc[i][e]);
      }
#pragma unroll
      for (int i = 0; i < kTPW; ++i)
#pragma unroll
        for (int q = 0; q < 8; ++q) xv[i][q] = xn[i][q];
    }
  }
  float mine = 0.f;
#pragma unroll
  for (int i = 0; i < kTPW; ++i)
#pragma unroll
    for (int e = 0; e < kREC; ++e) {
      const float v = warp_sum(acc[i][e]);
      if (lane == i * kREC + e) mine = v;
    }
  const int t = tw + lane / kREC, e = lane % kREC;
  if (lane < kTPW * kREC && t < T && e < ne) logits[static_cast<size_t>(t) * E + e0 + e] = mine;
}

// ------------------------------------------------------------------ finish
// Sum the K-slice partial logits in slice order, add the bias, optionally
// store the logits, then softmax + top-k.  One warp per token; lane l holds
// experts l*V .. l*V+V-1.
template <typename LT, int V>
__global__ void __launch_bounds__(256) finish_kernel(const LT* __restrict__ parts, int nsplit, size_t split_stride,
                                                     const float* __restrict__ bias, int N, int E, int k, int renorm,
                                                     float* __restrict__ logits_out, int32_t* __restrict__ idx_out,
                                                     float* __restrict__ w_out) {
  const int lane = threadIdx.x & 31;
  const int warps = gridDim.x * (blockDim.x >> 5);
  const bool vec = (E == 32 * V) && ((V * sizeof(LT)) % 8 == 0) && ((V * sizeof(LT)) <= 32);
  for (int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); t < N; t += warps) {
    float v[V];
    int ix[V];
#pragma unroll
    for (int i = 0; i < V; ++i) {
      v[i] = 0.f;
      ix[i] = lane * V + i < E ? lane * V + i : INT_MAX;
    }
    for (int sp = 0; sp < nsplit; ++sp) {
      const LT* row = parts + sp * split_stride + static_cast<size_t>(t) * E;
      if (vec) {
        constexpr int kWords = (V * sizeof(LT) + 7) / 8;  // 8-byte words per lane
        uint2 raw[kWords > 0 ? kWords : 1];
#pragma unroll
        for (int wd = 0; wd < kWords; ++wd) raw[wd] = __ldg(reinterpret_cast<const uint2*>(row + lane * V) + wd);
        const LT* pv = reinterpret_cast<const LT*>(raw);
#pragma unroll
        for (int i = 0; i < V; ++i) v[i] += to_f32(pv[i]);
      } else {
#pragma unroll
        for (int i = 0; i < V; ++i)
          if (ix[i] != INT_MAX) v[i] += to_f32(row[ix[i]]);
      }
    }
#pragma unroll
    for (int i = 0; i < V; ++i) {
      if (ix[i] == INT_MAX) {
        v[i] = -INFINITY;
      } else {
        if (bias) v[i] += bias[ix[i]];
        if (logits_out) logits_out[static_cast<size_t>(t) * E + ix[i]] = v[i];
      }
    }
    warp_select<V>(v, ix, k, renorm, lane, idx_out + static_cast<size_t>(t) * k,
                   w_out + static_cast<size_t>(t) * k);
  }
}

template <typename LT>
int finish_dispatch(const void* parts, int nsplit, size_t stride, const float* bias, int N, int E, int k,
                    int renorm, float* lo, int32_t* idx, float* w, cudaStream_t s) {
  const int warps_per_block = 8;
  const int blocks = max(1, min((N + warps_per_block - 1) / warps_per_block, num_sms() * 16));
  const LT* lp = static_cast<const LT*>(parts);
  const int v = (E + 31) / 32;
#define MOE_FINISH_CASE(VV)                                                                                   \
  if (v <= VV) {                                                                                             \
    finish_kernel<LT, VV><<<blocks, warps_per_block * 32, 0, s>>>(lp, nsplit, stride, bias, N, E, k, renorm, lo, \
                                                                 idx, w);                                    \
    return launch_status(__func__);                                        \
  }
  MOE_FINISH_CASE(1)
  MOE_FINISH_CASE(2)
  MOE_FINISH_CASE(4)
  MOE_FINISH_CASE(8)
  MOE_FINISH_CASE(16)
  MOE_FINISH_CASE(32)
#undef MOE_FINISH_CASE
  return MOE_ERR_UNSUPPORTED;
}

template <typename XT, typename WT>
int simt_logits(const void* x, const void* Wr, int T, int d, int E, float* logits, cudaStream_t s) {
  dim3 grid((T + kRTok - 1) / kRTok, (E + kREC - 1) / kREC);
  logits_simt_kernel<XT, WT><<<grid, 256, 0, s>>>(static_cast<const XT*>(x), static_cast<const WT*>(Wr), T, d, E,
                                                  logits);
  return launch_status(__func__);
}

}  // namespace

// Tensor-core router: x [T, d] x W_r[E, d]^T on the grouped GEMM kernel (one
// group, fp32 output), split along K so that about one tile per SM is
// in flight; the slices' partial logits are summed in slice order by the
// finish kernel, so the result does not depend on scheduling.
bool router_uses_tensor_cores(int x_dtype, int w_dtype, int T, int d, int E) {
  return x_dtype == MOE_BF16 && w_dtype == MOE_BF16 && E % 64 == 0 && d % 64 == 0 && T >= 256 && E >= 64 &&
         d >= 1024;
}

int launch_router(const void* x, int x_dtype, const void* W_r, int w_dtype, const float* bias, int T, int d, int E,
                  int k, int renorm, float* logits_out, int32_t* idx, float* w, float* parts, int* status,
                  cudaStream_t s) {
  if (T == 0) return MOE_OK;
  int nsplit = 1;
  int st;
  if (router_uses_tensor_cores(x_dtype, w_dtype, T, d, E)) {
    const int mma_n = E % 256 == 0 ? 256 : (E % 128 == 0 ? 128 : 64);
    const int tiles = (T + 127) / 128 * (E / mma_n);
    nsplit = max(1, min(kRouterMaxSplit, min(num_sms() / max(tiles, 1), d / 64 / 4)));
    GemmArgs g{};
    g.A = x;
    g.B = W_r;
    g.offsets = nullptr;  // one group: all T rows
    g.G = 1;
    g.rows = T;
    g.N = E;
    g.K = d;
    g.ksplit = nsplit;
    g.mma_n = mma_n;
    g.ab_dtype = MOE_BF16;
    g.epilogue = MOE_EPI_NONE;
    g.c_dtype = MOE_F32;
    g.C = parts;
    g.status = status;
    st = launch_grouped_gemm(g, s);
  } else if (x_dtype == MOE_BF16 && w_dtype == MOE_BF16) {
    st = simt_logits<__nv_bfloat16, __nv_bfloat16>(x, W_r, T, d, E, parts, s);
  } else if (x_dtype == MOE_F32 && w_dtype == MOE_F32) {
    st = simt_logits<float, float>(x, W_r, T, d, E, parts, s);
  } else if (x_dtype == MOE_F32 && w_dtype == MOE_BF16) {
    st = simt_logits<float, __nv_bfloat16>(x, W_r, T, d, E, parts, s);
  } else if (x_dtype == MOE_BF16 && w_dtype == MOE_F32) {
    st = simt_logits<__nv_bfloat16, float>(x, W_r, T, d, E, parts, s);
  } else {
    return MOE_ERR_UNSUPPORTED;
  }
  if (st != MOE_OK) return st;
  return finish_dispatch<float>(parts, nsplit, static_cast<size_t>(T) * E, bias, T, E, k, renorm, logits_out, idx, w,
                                s);
}

int launch_topk_logits(const void* logits, int dtype, int N, int E, int k, int renorm, int32_t* idx, float* w,
                       cudaStream_t s) {
  if (N == 0) return MOE_OK;
  if (dtype == MOE_F16) return finish_dispatch<__half>(logits, 1, 0, nullptr, N, E, k, renorm, nullptr, idx, w, s);
  if (dtype == MOE_F32) return finish_dispatch<float>(logits, 1, 0, nullptr, N, E, k, renorm, nullptr, idx, w, s);
  if (dtype == MOE_BF16)
    return finish_dispatch<__nv_bfloat16>(logits, 1, 0, nullptr, N, E, k, renorm, nullptr, idx, w, s);
  return MOE_ERR_UNSUPPORTED;
}

}  // namespace moe
