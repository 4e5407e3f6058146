// Router: logits = x W_r^T (+ bias), softmax over all experts, top-k.
//
// "MegaMoE math model -> DeepGEMM source walk-through" §2.1 (p = Softmax(W_r x_t),
// keep the k best) and "Dense GEMM -> GroupedGEMM -> TP MoE" §4.2 (route_tokens).
// bf16 x and W_r with E <= 256 and k <= 8 take the one-launch tensor-core
// router (router_tc.cu).  This file holds the other paths.  Up to 16
// experts: one launch, router_fused_kernel (below), which streams x once and
// keeps every logit on chip.  Otherwise two launches:
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
#include <type_traits>

#include "common.cuh"
#include "ptx.cuh"

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
// Block = 8 tokens x 8 experts (4 warps of 2 tokens).  The block's W_r rows
// are staged in shared memory 32 KB at a time (2048 bf16 / 1024 fp32
// columns), so each block reads them once from L2 while x streams from HBM
// once per expert block; every lane keeps the next two steps of its tokens'
// columns in flight while it multiplies the current ones.  Used when E or d is small
// (the logits are then bound by reading x) and for fp32 operands.
constexpr int kREC = 8;
constexpr int kTPW = 2;
constexpr int kRWarps = 4;
constexpr int kRTok = kRWarps * kTPW;

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
__global__ void __launch_bounds__(kRWarps * 32) logits_simt_kernel(const XT* __restrict__ x, const WT* __restrict__ Wr,
                                                          int T, int d, int E, float* __restrict__ logits) {
  pdl_wait();  // the preceding kernel on the stream is complete and visible
  pdl_launch_dependents();
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
    // three steps of 8 columns in flight per lane: current (xa), next (xb), after next (xc)
    auto fetch = [&](float (&dst)[kTPW][8], int c) {
#pragma unroll
      for (int i = 0; i < kTPW; ++i) {
        if (tw + i < T && c < dc) {
          load8_any(x + static_cast<size_t>(tw + i) * d + c0 + c, dst[i]);
        } else {
#pragma unroll
          for (int q = 0; q < 8; ++q) dst[i][q] = 0.f;
        }
      }
    };
    float xa[kTPW][8], xb[kTPW][8];
    fetch(xa, lane * 8);
    fetch(xb, lane * 8 + 256);
    for (int c = lane * 8; c < dc; c += 256) {
      float xc[kTPW][8];
      fetch(xc, c + 512);
#pragma unroll
      for (int e = 0; e < kREC; ++e) {
        float wv[8];
        smem8(&s_w[e][c], wv);
#pragma unroll
        for (int i = 0; i < kTPW; ++i)
#pragma unroll
          for (int q = 0; q < 8; ++q) acc[i][e] = fmaf(xa[i][q], wv[q], acc[i][e]);
      }
#pragma unroll
      for (int i = 0; i < kTPW; ++i)
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          xa[i][q] = xb[i][q];
          xb[i][q] = xc[i][q];
        }
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
// store the logits, then softmax + top-k.  A group of G lanes owns one token
// (each lane V consecutive experts, 16- or 32-byte loads), so a warp handles
// 32/G tokens at once; max, sum and the k arg-max rounds are reduced over the
// group with xor shuffles on (logit descending, expert index ascending).
// (logit, expert) as one 64-bit key whose unsigned order is "larger logit,
// then lower expert index": the float's bits mapped to an order-preserving
// unsigned integer in the high word, the complemented index in the low word.
__device__ __forceinline__ uint64_t sel_key(float v, int e) {
  uint32_t u = __float_as_uint(v);
  if ((u << 1) == 0u) u = 0u;  // -0 and +0 are the same logit: the lower index must win
  const uint32_t o = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
  return (static_cast<uint64_t>(o) << 32) | static_cast<uint32_t>(~static_cast<uint32_t>(e));
}
__device__ __forceinline__ float key_value(uint64_t key) {
  const uint32_t o = static_cast<uint32_t>(key >> 32);
  return __uint_as_float((o & 0x80000000u) ? (o & 0x7fffffffu) : ~o);
}
__device__ __forceinline__ int key_index(uint64_t key) {
  return static_cast<int>(~static_cast<uint32_t>(key));
}

// 16-bit logits taken as stored (no partial sums, no bias): the same order in
// one 32-bit key, 16-bit order-preserving value over the complemented index.
template <typename LT>
__device__ __forceinline__ uint32_t sel_key16(LT v, int e) {
  uint16_t u = *reinterpret_cast<const uint16_t*>(&v);
  if ((u & 0x7fffu) == 0u) u = 0u;  // -0 and +0 are the same logit: the lower index must win
  const uint16_t o = (u & 0x8000u) ? static_cast<uint16_t>(~u) : static_cast<uint16_t>(u | 0x8000u);
  return (static_cast<uint32_t>(o) << 16) | static_cast<uint32_t>(0xffffu - e);
}
template <typename LT>
__device__ __forceinline__ float key16_value(uint32_t key) {
  const uint16_t o = static_cast<uint16_t>(key >> 16);
  const uint16_t u = (o & 0x8000u) ? static_cast<uint16_t>(o & 0x7fffu) : static_cast<uint16_t>(~o);
  return to_f32(*reinterpret_cast<const LT*>(&u));
}

template <typename LT, int V, int G, bool K16>
__global__ void __launch_bounds__(256) finish_kernel(const LT* __restrict__ parts, int nsplit, size_t split_stride,
                                                     int pstride, const float* __restrict__ bias, int N, int E,
                                                     int k, int renorm, float* __restrict__ logits_out,
                                                     int32_t* __restrict__ idx_out, float* __restrict__ w_out) {
  pdl_wait();  // the preceding kernel on the stream is complete and visible
  pdl_launch_dependents();
  constexpr int TPW = 32 / G;
  constexpr int kBytes = V * static_cast<int>(sizeof(LT));
  constexpr float kLog2e = 1.4426950408889634f;
  const int lane = threadIdx.x & 31;
  const int gl = lane % G, gw = lane / G;
  const int e_base = gl * V;
  const int warps = gridDim.x * (blockDim.x >> 5);
  const int warp_id = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const bool vec = (E == G * V) && (pstride == E) && (kBytes % 16 == 0);
  for (int t0 = warp_id * TPW; t0 < N; t0 += warps * TPW) {  // warp-uniform trip count
    const int t = t0 + gw;
    const bool tok = t < N;
    float v[V];
    [[maybe_unused]] uint32_t key16[K16 ? V : 1];
#pragma unroll
    for (int i = 0; i < V; ++i) v[i] = 0.f;
    if constexpr (K16) {
      // single stored 16-bit row: keys straight from the raw values
      LT raw[V];
#pragma unroll
      for (int i = 0; i < V; ++i) raw[i] = LT();
      if (tok) {
        const LT* row = parts + static_cast<size_t>(t) * pstride;
        if (vec) {
#pragma unroll
          for (int q = 0; q < kBytes / 16; ++q)
            reinterpret_cast<uint4*>(raw)[q] = __ldg(reinterpret_cast<const uint4*>(row + e_base) + q);
        } else {
#pragma unroll
          for (int i = 0; i < V; ++i)
            if (e_base + i < E) raw[i] = row[e_base + i];
        }
      }
#pragma unroll
      for (int i = 0; i < V; ++i) {
        v[i] = to_f32(raw[i]);
        key16[i] = (tok && e_base + i < E) ? sel_key16(raw[i], e_base + i) : 0u;
      }
    } else if (tok) {
      for (int sp = 0; sp < nsplit; ++sp) {
        const LT* row = parts + sp * split_stride + static_cast<size_t>(t) * pstride;
        if (vec) {
          uint4 raw[kBytes / 16 > 0 ? kBytes / 16 : 1];
#pragma unroll
          for (int q = 0; q < kBytes / 16; ++q) raw[q] = __ldg(reinterpret_cast<const uint4*>(row + e_base) + q);
          const LT* pv = reinterpret_cast<const LT*>(raw);
#pragma unroll
          for (int i = 0; i < V; ++i) v[i] += to_f32(pv[i]);
        } else {
#pragma unroll
          for (int i = 0; i < V; ++i)
            if (e_base + i < E) v[i] += to_f32(row[e_base + i]);
        }
      }
    }
    float m = -INFINITY;
#pragma unroll
    for (int i = 0; i < V; ++i) {
      const int e = e_base + i;
      if (!tok || e >= E) {
        v[i] = -INFINITY;
      } else {
        if (bias) v[i] += bias[e];
        if (logits_out) logits_out[static_cast<size_t>(t) * E + e] = v[i];
      }
      m = fmaxf(m, v[i]);
    }
#pragma unroll
    for (int o = G / 2; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    float sum = 0.f;
#pragma unroll
    for (int i = 0; i < V; ++i)
      if (e_base + i < E) sum += exp2f((v[i] - m) * kLog2e);
#pragma unroll
    for (int o = G / 2; o; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    const float inv_sum = 1.0f / sum;
    float psum = 0.f;
    if constexpr (K16) {
      for (int r = 0; r < k; ++r) {
        uint32_t best = 0;
#pragma unroll
        for (int i = 0; i < V; ++i) best = max(best, key16[i]);
#pragma unroll
        for (int o = G / 2; o; o >>= 1) best = max(best, __shfl_xor_sync(0xffffffffu, best, o));
        const float pr = exp2f((key16_value<LT>(best) - m) * kLog2e) * inv_sum;
        psum += pr;
        if (tok && gl == 0) {
          idx_out[static_cast<size_t>(t) * k + r] = static_cast<int>(0xffffu - (best & 0xffffu));
          w_out[static_cast<size_t>(t) * k + r] = pr;
        }
#pragma unroll
        for (int i = 0; i < V; ++i) key16[i] = key16[i] == best ? 0u : key16[i];
      }
    } else {
      uint64_t key[V];
#pragma unroll
      for (int i = 0; i < V; ++i) key[i] = (e_base + i < E && tok) ? sel_key(v[i], e_base + i) : 0ull;
      for (int r = 0; r < k; ++r) {
        uint64_t best = 0;
#pragma unroll
        for (int i = 0; i < V; ++i) best = key[i] > best ? key[i] : best;
#pragma unroll
        for (int o = G / 2; o; o >>= 1) {
          const uint64_t other = __shfl_xor_sync(0xffffffffu, best, o);
          best = other > best ? other : best;
        }
        const float pr = exp2f((key_value(best) - m) * kLog2e) * inv_sum;
        psum += pr;
        if (tok && gl == 0) {
          idx_out[static_cast<size_t>(t) * k + r] = key_index(best);
          w_out[static_cast<size_t>(t) * k + r] = pr;
        }
#pragma unroll
        for (int i = 0; i < V; ++i) key[i] = key[i] == best ? 0ull : key[i];
      }
    }
    if (renorm && tok && gl == 0)
      for (int r = 0; r < k; ++r) w_out[static_cast<size_t>(t) * k + r] /= psum;
  }
}

template <typename LT, int V, int G>
int finish_launch(const void* parts, int nsplit, size_t stride, int pstride, const float* bias, int N, int E, int k,
                  int renorm, float* lo, int32_t* idx, float* w, cudaStream_t s) {
  constexpr int TPB = 8 * (32 / G);  // tokens per 256-thread block
  const int blocks = max(1, min((N + TPB - 1) / TPB, num_sms() * 32));
  const LT* pp = static_cast<const LT*>(parts);
  if (sizeof(LT) == 2 && nsplit == 1 && bias == nullptr && E <= 65535)
    return launch_pdl(__func__, finish_kernel<LT, V, G, sizeof(LT) == 2>, dim3(blocks), dim3(256), 0, s, pp, nsplit,
                      stride, pstride, bias, N, E, k, renorm, lo, idx, w);
  return launch_pdl(__func__, finish_kernel<LT, V, G, false>, dim3(blocks), dim3(256), 0, s, pp, nsplit, stride,
                    pstride, bias, N, E, k, renorm, lo, idx, w);
}

// ------------------------------------------------------------------ top-k of stored 16-bit logits
// "DeepSeek MoE architecture overview" §2.2 gives each token its own top-k
// selection.  Two threads share a token, each over alternate 16-byte chunks of
// its E logits, staged in shared memory.  A logit and its expert form one
// 32-bit key: the logit's 16-bit order-preserving image over the complemented
// index, so a larger key means "larger logit, then lower expert", and keys are
// distinct.  Each thread keeps its K largest keys sorted with a branch-free
// max/min insertion network (the lanes never diverge) along with the running
// max logit and the sum of exponentials, rescaled whenever the max grows; the
// two threads then merge their lists.  E <= 256 (the index fits 16 bits),
// E % 8 == 0, k <= K <= 8.
constexpr int kTopkList = 8;
constexpr int kTopkWarps = 4;
constexpr int kTopkRowsPerWarp = 16;

// Order-preserving images of the two 16-bit floats of a word, two at a time:
// a positive half h maps to h | 0x8000, a negative one to 0x10000 - h, so -0
// and +0 share the image 0x8000 (the +1 of the negation never carries out of
// a negative half, whose complement is at most 0x7fff).  And back, for one.
__device__ __forceinline__ uint32_t ord16x2(uint32_t w) {
  const uint32_t neg = (w >> 15) & 0x00010001u;
  return (w ^ ((neg * 0xffffu) | 0x80008000u)) + neg;
}
__device__ __forceinline__ uint32_t unord16(uint32_t o) { return (o & 0x8000u) ? (o & 0x7fffu) : (0x10000u - o); }
template <typename LT>
__device__ __forceinline__ float bits16_f32(uint32_t u) {
  const uint16_t b = static_cast<uint16_t>(u);
  return to_f32(*reinterpret_cast<const LT*>(&b));
}
template <typename LT>
__device__ __forceinline__ float2 word_f32x2(uint32_t w) {
  if constexpr (std::is_same<LT, __half>::value) {
    return __half22float2(*reinterpret_cast<const __half2*>(&w));
  } else {
    return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
  }
}
// 2^x by the SFU's approximation (relative error about 2^-22; results below
// the normal range flush to zero, far under a softmax term's tolerance)
__device__ __forceinline__ float sfu_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
// insert a key into a descending list of K distinct keys (the smallest falls off)
template <int K>
__device__ __forceinline__ void insert_key(uint32_t (&b)[K], uint32_t x) {
#pragma unroll
  for (int j = 0; j < K; ++j) {
    const uint32_t hi = max(b[j], x);
    x = min(b[j], x);
    b[j] = hi;
  }
}
// compare-exchange: the larger key to a, the smaller to b
__device__ __forceinline__ void cx(uint32_t& a, uint32_t& b) {
  const uint32_t hi = max(a, b);
  b = min(a, b);
  a = hi;
}
// Merge a descending list t of K keys into the descending list b of K (both
// distinct): the element-wise max of b and reversed t holds the K largest as
// a bitonic sequence, which half-cleaners of distance K/2 .. 1 sort.
template <int K>
__device__ __forceinline__ void merge_top(uint32_t (&b)[K], const uint32_t (&t)[K]) {
#pragma unroll
  for (int i = 0; i < K; ++i) b[i] = max(b[i], t[K - 1 - i]);
#pragma unroll
  for (int dist = K / 2; dist > 0; dist /= 2)
#pragma unroll
    for (int i = 0; i < K; ++i)
      if ((i / dist) % 2 == 0) cx(b[i], b[i + dist]);
}
// Fold a chunk of 8 distinct keys into the descending top-K list (K = 4 or 8):
// the chunk's own top K by a sorting network (two sorted halves of 4 merged
// for K = 4; Batcher's 19-comparator network for K = 8), then one merge.
// Fewer max/min per key than inserting each key (5.5 vs 7 at K = 4, 8.75 vs
// 15 at K = 8).
template <int K>
__device__ __forceinline__ void fold_chunk(uint32_t (&b)[K], uint32_t (&c)[8]) {
  static_assert(K == 4 || K == 8, "chunk networks for K = 4 and 8");
  if constexpr (K == 4) {
    uint32_t lo[4] = {c[0], c[1], c[2], c[3]}, hi[4] = {c[4], c[5], c[6], c[7]};
    cx(lo[0], lo[1]); cx(lo[2], lo[3]); cx(lo[0], lo[2]); cx(lo[1], lo[3]); cx(lo[1], lo[2]);
    cx(hi[0], hi[1]); cx(hi[2], hi[3]); cx(hi[0], hi[2]); cx(hi[1], hi[3]); cx(hi[1], hi[2]);
    merge_top<4>(lo, hi);  // the chunk's top 4, sorted
    merge_top<4>(b, lo);
  } else {
    cx(c[0], c[1]); cx(c[2], c[3]); cx(c[4], c[5]); cx(c[6], c[7]);
    cx(c[0], c[2]); cx(c[1], c[3]); cx(c[4], c[6]); cx(c[5], c[7]);
    cx(c[1], c[2]); cx(c[5], c[6]);
    cx(c[0], c[4]); cx(c[1], c[5]); cx(c[2], c[6]); cx(c[3], c[7]);
    cx(c[2], c[4]); cx(c[3], c[5]);
    cx(c[1], c[2]); cx(c[3], c[4]); cx(c[5], c[6]);
    merge_top<8>(b, c);
  }
}

template <typename LT, int K>
__global__ void __launch_bounds__(kTopkWarps * 32) topk_rows_kernel(const LT* __restrict__ logits, int N, int E, int k,
                                                                    int renorm, int32_t* __restrict__ idx_out,
                                                                    float* __restrict__ w_out) {
  pdl_wait();  // the preceding kernel on the stream is complete and visible
  pdl_launch_dependents();
  constexpr float kLog2e = 1.4426950408889634f;
  const int RB = E * 2 + 32;  // bytes per staged row: the pad spreads a warp's rows over the banks
  extern __shared__ __align__(16) uint8_t s_rows[];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int t0 = (blockIdx.x * kTopkWarps + warp) * kTopkRowsPerWarp;  // the warp's 16 tokens
  const int nrow = min(kTopkRowsPerWarp, N - t0);
  if (nrow <= 0) return;
  uint8_t* rows = s_rows + warp * kTopkRowsPerWarp * RB;
  int32_t* s_idx = reinterpret_cast<int32_t*>(s_rows + kTopkWarps * kTopkRowsPerWarp * RB) +
                   warp * kTopkRowsPerWarp * kTopkList;
  float* s_w = reinterpret_cast<float*>(s_idx + (kTopkWarps - warp) * kTopkRowsPerWarp * kTopkList) +
               warp * kTopkRowsPerWarp * kTopkList;
  // the warp's rows are contiguous: all of them in flight at once, 16 bytes a
  // copy; q / cpr as (q * ceil(2^16 / cpr)) >> 16, exact for q < 2^16 / cpr
  // (here q < 16 * cpr <= 512 and cpr <= 32)
  const int cpr = E / 8;  // 16-byte chunks per row
  const int inv_cpr = (65536 + cpr - 1) / cpr;
  const uint8_t* src = reinterpret_cast<const uint8_t*>(logits + static_cast<size_t>(t0) * E);
  for (int q = lane; q < nrow * cpr; q += 32) {
    const int r = (q * inv_cpr) >> 16;
    ptx::cp_async_16(rows + r * RB + (q - r * cpr) * 16, src + q * 16);
  }
  ptx::cp_async_wait_all();
  __syncwarp();
  const int j = lane >> 1, h = lane & 1;
  if (j >= nrow) return;
  const uint32_t pm = 3u << (2 * j);  // the token's two lanes
  const uint8_t* mine = rows + j * RB;

  uint32_t b[K];
#pragma unroll
  for (int i = 0; i < K; ++i) b[i] = 0u;  // below every key (a key's low half is at least 0xff00)
  float m = -INFINITY, sum = 0.f;
#pragma unroll 1
  for (int c = h; c < cpr; c += 2) {
    const uint4 q = *reinterpret_cast<const uint4*>(mine + c * 16);
    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
    const uint32_t base = 0xffffu - 8u * c;  // low 3 bits set: base - i == base ^ i
    if constexpr (K >= 4) {
      uint32_t kc[8];
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) {
        const uint32_t o = ord16x2(w[jj]);
        kc[2 * jj] = (o << 16) | (base ^ (2 * jj));
        kc[2 * jj + 1] = (o & 0xffff0000u) | (base ^ (2 * jj + 1));
      }
      fold_chunk<K>(b, kc);
    } else {
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) {
        const uint32_t o = ord16x2(w[jj]);
        insert_key<K>(b, (o << 16) | (base ^ (2 * jj)));
        insert_key<K>(b, (o & 0xffff0000u) | (base ^ (2 * jj + 1)));
      }
    }
    // the running max logit is the value of the largest key
    const float mn = bits16_f32<LT>(unord16(b[0] >> 16));
    const float mnl = mn * kLog2e;
    float s = sum * sfu_exp2(m * kLog2e - mnl);
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {
      const float2 f = word_f32x2<LT>(w[jj]);
      s += sfu_exp2(fmaf(f.x, kLog2e, -mnl));
      s += sfu_exp2(fmaf(f.y, kLog2e, -mnl));
    }
    sum = s;
    m = mn;
  }
  // merge the two threads' lists and sums (both lanes end with the same ones)
  uint32_t other[K];
#pragma unroll
  for (int i = 0; i < K; ++i) other[i] = __shfl_xor_sync(pm, b[i], 1);
  merge_top<K>(b, other);  // both lists are sorted: one bitonic merge
  {
    const float mo = __shfl_xor_sync(pm, m, 1), so = __shfl_xor_sync(pm, sum, 1);
    const float mn = fmaxf(m, mo);
    sum = sum * sfu_exp2((m - mn) * kLog2e) + so * sfu_exp2((mo - mn) * kLog2e);
    m = mn;
  }
  // probabilities of the picks (softmax over all E), optionally renormalised
  const float inv_sum = 1.0f / sum;
  float pr[K];
  float psum = 0.f;
#pragma unroll
  for (int r = 0; r < K; ++r) {
    if (r < k) {
      pr[r] = exp2f((bits16_f32<LT>(unord16(b[r] >> 16)) - m) * kLog2e) * inv_sum;
      psum += pr[r];
    }
  }
#pragma unroll
  for (int r = 0; r < K; ++r) {
    if (r < k && (r & 1) == h) {
      s_idx[j * k + r] = 0xffff - static_cast<int>(b[r] & 0xffffu);
      s_w[j * k + r] = renorm ? pr[r] / psum : pr[r];
    }
  }
  // the warp's k*nrow outputs are contiguous: store them coalesced
  const int live = 2 * nrow;
  __syncwarp(live == 32 ? 0xffffffffu : (1u << live) - 1u);
  for (int q = lane; q < nrow * k; q += live) {
    idx_out[static_cast<size_t>(t0) * k + q] = s_idx[q];
    w_out[static_cast<size_t>(t0) * k + q] = s_w[q];
  }
}

template <typename LT>
int topk_rows_dispatch(const void* logits, int N, int E, int k, int renorm, int32_t* idx, float* w, cudaStream_t s) {
  constexpr int kTokensPerBlock = kTopkWarps * kTopkRowsPerWarp;
  const dim3 grid((N + kTokensPerBlock - 1) / kTokensPerBlock);
  // staged rows plus the outputs: 38,912 bytes at E = 256, under the default limit
  const size_t smem = static_cast<size_t>(kTokensPerBlock) * (E * 2 + 32) +
                      static_cast<size_t>(kTokensPerBlock) * kTopkList * 8;
  const LT* l = static_cast<const LT*>(logits);
  const dim3 block(kTopkWarps * 32);
  if (k == 1) return launch_pdl("topk_rows_kernel", topk_rows_kernel<LT, 1>, grid, block, smem, s, l, N, E, k, renorm, idx, w);
  if (k == 2) return launch_pdl("topk_rows_kernel", topk_rows_kernel<LT, 2>, grid, block, smem, s, l, N, E, k, renorm, idx, w);
  if (k <= 4) return launch_pdl("topk_rows_kernel", topk_rows_kernel<LT, 4>, grid, block, smem, s, l, N, E, k, renorm, idx, w);
  return launch_pdl("topk_rows_kernel", topk_rows_kernel<LT, 8>, grid, block, smem, s, l, N, E, k, renorm, idx, w);
}

template <typename LT>
int finish_dispatch(const void* parts, int nsplit, size_t stride, int pstride, const float* bias, int N, int E, int k,
                    int renorm, float* lo, int32_t* idx, float* w, cudaStream_t s) {
#define MOE_FINISH(VV, GG) finish_launch<LT, VV, GG>(parts, nsplit, stride, pstride, bias, N, E, k, renorm, lo, idx, w, s)
  // Few experts: more lanes per token (one or two experts each), so that a
  // batch of a few thousand tokens still spreads over every SM.
  if (N >= 1024) {
    if (E <= 8) return MOE_FINISH(1, 8);
    if (E <= 16) return MOE_FINISH(1, 16);
    if (E <= 32) return MOE_FINISH(2, 16);
  } else if (E > 16 && E <= 128) {
    // few tokens: 16 lanes per token, so that a decode batch spreads over more CTAs
    if (E <= 64) return MOE_FINISH(4, 16);
    return MOE_FINISH(8, 16);
  }
  if (E <= 16) return MOE_FINISH(16, 1);
  if (E <= 32) return MOE_FINISH(16, 2);
  if (E <= 64) return MOE_FINISH(16, 4);
  if (E <= 128) return MOE_FINISH(16, 8);
  if (E <= 256) return MOE_FINISH(16, 16);
  if (E <= 512) return MOE_FINISH(16, 32);
  if (E <= 1024) return MOE_FINISH(32, 32);
#undef MOE_FINISH
  return MOE_ERR_UNSUPPORTED;
}

// ------------------------------------------------------------------ fused router (E <= 16)
// One launch: logits, softmax and top-k ("MegaMoE ..." §2.1; the fused
// logits + softmax kernel of "DeepSeek-R1 deployment on A100" §3.2 and the
// warp-level top-k of "DeepSeek MoE architecture overview" §2.2).  The
// logits of a few experts are a short dot product per token, bound by
// reading x once: a warp takes TPW = 16 / EP tokens at a time (EP = E
// rounded up to 8 or 16) and its lanes split d into 16-byte chunks, lane l
// owning chunks l, l + 32, ...; every lane accumulates the 16 (token,
// expert) partial logits in fp32 (packed FMAs on even / odd columns), the
// W_r chunk it needs coming through L1 and reused by the warp's tokens,
// with the next two chunks of x in flight.  A butterfly reduce-scatter over
// lane bits 16..2 and a final exchange with the neighbouring lane leave
// lanes 2i and 2i + 1 with the full logit of (token i / EP, expert i % EP);
// the 2 EP lanes of a token run the softmax and k rounds of an arg-max on
// packed (logit, ~index) keys, so ties go to the lower expert index.
constexpr int kFusedWarps = 8;

template <typename T>
struct Chunk8;  // 8 consecutive elements as raw 16- or 32-byte words
template <>
struct Chunk8<__nv_bfloat16> {
  uint4 w;
  __device__ __forceinline__ void load(const __nv_bfloat16* p) { w = __ldg(reinterpret_cast<const uint4*>(p)); }
  __device__ __forceinline__ void zero() { w = make_uint4(0, 0, 0, 0); }
  __device__ __forceinline__ float2 pair(int i) const {  // elements 2i, 2i+1
    const uint32_t u = i == 0 ? w.x : i == 1 ? w.y : i == 2 ? w.z : w.w;
    return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xffff0000u));
  }
};
template <>
struct Chunk8<float> {
  float4 a, b;
  __device__ __forceinline__ void load(const float* p) {
    a = __ldg(reinterpret_cast<const float4*>(p));
    b = __ldg(reinterpret_cast<const float4*>(p) + 1);
  }
  __device__ __forceinline__ void zero() { a = b = make_float4(0.f, 0.f, 0.f, 0.f); }
  __device__ __forceinline__ float2 pair(int i) const {
    return i == 0 ? make_float2(a.x, a.y) : i == 1 ? make_float2(a.z, a.w) : i == 2 ? make_float2(b.x, b.y)
                                                                                     : make_float2(b.z, b.w);
  }
};

// One level of the butterfly reduce-scatter: lanes with `bit` clear keep the
// lower half of v[0, S), the others the upper half, each adding the
// partner's copy of the half it keeps; the kept half moves to v[0, S/2).
template <int S>
__device__ __forceinline__ void rs_level(float (&v)[16], int lane, int bit) {
  const bool up = lane & bit;
#pragma unroll
  for (int i = 0; i < S / 2; ++i) {
    const float send = up ? v[i] : v[S / 2 + i];
    const float keep = up ? v[S / 2 + i] : v[i];
    v[i] = keep + __shfl_xor_sync(0xffffffffu, send, bit);
  }
}

template <typename XT, typename WT, int EP>
__global__ void __launch_bounds__(kFusedWarps * 32, 2) router_fused_kernel(const XT* __restrict__ x,
                                                                         const WT* __restrict__ Wr,
                                                                         const float* __restrict__ bias, int T, int d,
                                                                         int E, int k, int renorm,
                                                                         float* __restrict__ logits_out,
                                                                         int32_t* __restrict__ idx_out,
                                                                         float* __restrict__ w_out) {
  pdl_wait();  // the preceding kernel on the stream is complete and visible
  pdl_launch_dependents();
  static_assert(EP == 8 || EP == 16, "8 or 16 (padded) experts");
  constexpr int TPW = 16 / EP;  // tokens per warp
  constexpr int G = 2 * EP;     // lanes of one token after the reduction
  constexpr float kLog2e = 1.4426950408889634f;
  const int lane = threadIdx.x & 31;
  const int nwarps = gridDim.x * kFusedWarps;
  const int nchunk = d / 8;  // 8-element chunks per row
  for (int t0 = (blockIdx.x * kFusedWarps + (threadIdx.x >> 5)) * TPW; t0 < T; t0 += nwarps * TPW) {
    float2 acc2[16];  // (token j, expert e) at j * EP + e: running sums of even and odd columns
#pragma unroll
    for (int i = 0; i < 16; ++i) acc2[i] = make_float2(0.f, 0.f);
    auto fetch = [&](Chunk8<XT>(&dst)[TPW], int c) {
#pragma unroll
      for (int j = 0; j < TPW; ++j) {
        if (c < nchunk && t0 + j < T)
          dst[j].load(x + static_cast<size_t>(t0 + j) * d + c * 8);
        else
          dst[j].zero();
      }
    };
    // three steps of x in flight per lane: this one, the next and the one after
    Chunk8<XT> cur[TPW], nxt[TPW];
    fetch(cur, lane);
    fetch(nxt, lane + 32);
    for (int c0 = 0; c0 < nchunk; c0 += 32) {  // warp-uniform trip count
      const int c = c0 + lane;
      Chunk8<XT> after[TPW];
      fetch(after, c + 64);
#pragma unroll
      for (int e = 0; e < EP; ++e) {
        Chunk8<WT> w;
        if (c < nchunk && e < E)
          w.load(Wr + static_cast<size_t>(e) * d + c * 8);
        else
          w.zero();
#pragma unroll
        for (int j = 0; j < TPW; ++j)
#pragma unroll
          for (int i = 0; i < 4; ++i) acc2[j * EP + e] = __ffma2_rn(cur[j].pair(i), w.pair(i), acc2[j * EP + e]);
      }
#pragma unroll
      for (int j = 0; j < TPW; ++j) {
        cur[j] = nxt[j];
        nxt[j] = after[j];
      }
    }
    float acc[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) acc[i] = acc2[i].x + acc2[i].y;
    // reduce-scatter over lane bits 16, 8, 4, 2; then lanes 2i and 2i + 1 add
    // their halves: both hold partial index i = lane / 2
    rs_level<16>(acc, lane, 16);
    rs_level<8>(acc, lane, 8);
    rs_level<4>(acc, lane, 4);
    rs_level<2>(acc, lane, 2);
    const float logit = acc[0] + __shfl_xor_sync(0xffffffffu, acc[0], 1);
    const int t = t0 + (lane >> 1) / EP;
    const int e = (lane >> 1) % EP;
    const bool tok = t < T;
    const bool real = tok && e < E;
    float v = -INFINITY;
    uint64_t key = 0ull;
    if (real) {
      v = logit + (bias ? bias[e] : 0.f);
      if (logits_out && (lane & 1) == 0) logits_out[static_cast<size_t>(t) * E + e] = v;
      key = sel_key(v, e);
    }
    float m = v;
#pragma unroll
    for (int o = G / 2; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    float sum = (real && (lane & 1) == 0) ? exp2f((v - m) * kLog2e) : 0.f;  // each expert counted once
#pragma unroll
    for (int o = G / 2; o; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    const float inv_sum = 1.0f / sum;
    const bool leader = (lane % G) == 0;
    float psum = 0.f;
    for (int r = 0; r < k; ++r) {
      uint64_t best = key;
#pragma unroll
      for (int o = G / 2; o; o >>= 1) {
        const uint64_t other = __shfl_xor_sync(0xffffffffu, best, o);
        best = other > best ? other : best;
      }
      const float pr = exp2f((key_value(best) - m) * kLog2e) * inv_sum;
      psum += pr;
      if (tok && leader) {
        idx_out[static_cast<size_t>(t) * k + r] = key_index(best);
        w_out[static_cast<size_t>(t) * k + r] = pr;
      }
      key = key == best ? 0ull : key;
    }
    if (renorm && tok && leader)
      for (int r = 0; r < k; ++r) w_out[static_cast<size_t>(t) * k + r] /= psum;
  }
}

template <typename XT, typename WT, int EP>
int fused_launch(const void* x, const void* Wr, const float* bias, int T, int d, int E, int k, int renorm,
                 float* logits_out, int32_t* idx, float* w, cudaStream_t s) {
  constexpr int TPW = 16 / EP;
  const int warps_needed = (T + TPW - 1) / TPW;
  const int blocks = max(1, min((warps_needed + kFusedWarps - 1) / kFusedWarps, num_sms() * 8));
  return launch_pdl("router_fused_kernel", router_fused_kernel<XT, WT, EP>, dim3(blocks), dim3(kFusedWarps * 32), 0,
                    s, static_cast<const XT*>(x), static_cast<const WT*>(Wr), bias, T, d, E, k, renorm, logits_out,
                    idx, w);
}

template <typename XT, typename WT>
int fused_dispatch(const void* x, const void* Wr, const float* bias, int T, int d, int E, int k, int renorm,
                   float* lo, int32_t* idx, float* w, cudaStream_t s) {
  if (E <= 8) return fused_launch<XT, WT, 8>(x, Wr, bias, T, d, E, k, renorm, lo, idx, w, s);
  return fused_launch<XT, WT, 16>(x, Wr, bias, T, d, E, k, renorm, lo, idx, w, s);
}

template <typename XT, typename WT>
int simt_logits(const void* x, const void* Wr, int T, int d, int E, float* logits, cudaStream_t s) {
  dim3 grid((T + kRTok - 1) / kRTok, (E + kREC - 1) / kREC);
  return launch_pdl(__func__, logits_simt_kernel<XT, WT>, grid, dim3(kRWarps * 32), 0, s, static_cast<const XT*>(x),
                    static_cast<const WT*>(Wr), T, d, E, logits);
}

}  // namespace

// Tensor-core router: x [T, d] x W_r[E, d]^T on the grouped GEMM kernel (one
// group, fp32 output), split along K so that about one tile per SM is
// in flight; the slices' partial logits are summed in slice order by the
// finish kernel, so the result does not depend on scheduling.
bool router_uses_tensor_cores(int x_dtype, int w_dtype, int T, int d, int E) {
  return x_dtype == MOE_BF16 && w_dtype == MOE_BF16 && d % 64 == 0 && T >= 256 && d >= 512;
}

int router_padded_experts(int E) { return (E + 63) / 64 * 64; }

bool router_is_fused(int x_dtype, int w_dtype, int T, int d, int E, int k) {
  (void)T;
  return router_tc_applies(x_dtype, w_dtype, d, E, k) || E <= 16;
}

int launch_router(const void* x, int x_dtype, const void* W_r, int w_dtype, const float* bias, int T, int d, int E,
                  int k, int renorm, float* logits_out, int32_t* idx, float* w, float* parts, int* status,
                  cudaStream_t s) {
  if (T == 0) return MOE_OK;
  if (router_tc_applies(x_dtype, w_dtype, d, E, k))
    return launch_router_tc(x, W_r, bias, T, d, E, k, renorm, logits_out, idx, w, status, s);
  if (E <= 16) {
    if (x_dtype == MOE_BF16 && w_dtype == MOE_BF16)
      return fused_dispatch<__nv_bfloat16, __nv_bfloat16>(x, W_r, bias, T, d, E, k, renorm, logits_out, idx, w, s);
    if (x_dtype == MOE_F32 && w_dtype == MOE_F32)
      return fused_dispatch<float, float>(x, W_r, bias, T, d, E, k, renorm, logits_out, idx, w, s);
    if (x_dtype == MOE_F32 && w_dtype == MOE_BF16)
      return fused_dispatch<float, __nv_bfloat16>(x, W_r, bias, T, d, E, k, renorm, logits_out, idx, w, s);
    if (x_dtype == MOE_BF16 && w_dtype == MOE_F32)
      return fused_dispatch<__nv_bfloat16, float>(x, W_r, bias, T, d, E, k, renorm, logits_out, idx, w, s);
    return MOE_ERR_UNSUPPORTED;
  }
  int nsplit = 1;
  int pstride = E;
  int st;
  if (router_uses_tensor_cores(x_dtype, w_dtype, T, d, E)) {
    // N = E rounded up to 64: the weight rows past E are read as zeros (TMA
    // fill beyond the tensor) and their logits columns are ignored
    pstride = router_padded_experts(E);
    const int mma_n = pstride % 256 == 0 ? 256 : (pstride % 128 == 0 ? 128 : 64);
    const int tiles = (T + 127) / 128 * (pstride / mma_n);
    nsplit = max(1, min(kRouterMaxSplit, min(num_sms() / max(tiles, 1), d / 64 / 4)));
    GemmArgs g{};
    g.A = x;
    g.B = W_r;
    g.offsets = nullptr;  // one group: all T rows
    g.G = 1;
    g.rows = T;
    g.N = pstride;
    g.B_rows = E;
    g.K = d;
    g.ksplit = nsplit;
    g.mma_n = mma_n;
    g.pair_tiles = -1;
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
  return finish_dispatch<float>(parts, nsplit, static_cast<size_t>(T) * pstride, pstride, bias, T, E, k, renorm,
                                logits_out, idx, w, s);
}

int launch_topk_logits(const void* logits, int dtype, int N, int E, int k, int renorm, int32_t* idx, float* w,
                       cudaStream_t s) {
  if (N == 0) return MOE_OK;
  if ((dtype == MOE_F16 || dtype == MOE_BF16) && E % 8 == 0 && E <= 256 && k <= kTopkList)
    return dtype == MOE_F16 ? topk_rows_dispatch<__half>(logits, N, E, k, renorm, idx, w, s)
                            : topk_rows_dispatch<__nv_bfloat16>(logits, N, E, k, renorm, idx, w, s);
  if (dtype == MOE_F16) return finish_dispatch<__half>(logits, 1, 0, E, nullptr, N, E, k, renorm, nullptr, idx, w, s);
  if (dtype == MOE_F32) return finish_dispatch<float>(logits, 1, 0, E, nullptr, N, E, k, renorm, nullptr, idx, w, s);
  if (dtype == MOE_BF16)
    return finish_dispatch<__nv_bfloat16>(logits, 1, 0, E, nullptr, N, E, k, renorm, nullptr, idx, w, s);
  return MOE_ERR_UNSUPPORTED;
}

}  // namespace moe
