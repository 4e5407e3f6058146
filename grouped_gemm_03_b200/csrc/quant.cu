// Weight quantisation to E4M3 with one fp32 scale per 128x128 block
// ("MegaMoE ..." §2.3 / §5.1: per-block scaling of the weights).
//   s = amax(block) / 448  (1 for an all-zero block),  q = e4m3_rn_satfinite(w / s)
// or, for the MX variant, s = the smallest power of two with 448 s >= amax
// (group_scale<true>); w / s is then exact before the E4M3 rounding.
// One CTA per block; each thread owns 64 contiguous elements of one row.
#include "common.cuh"

namespace moe {
namespace {

template <bool kPow2>
__global__ void __launch_bounds__(256) quant_block_kernel(const __nv_bfloat16* __restrict__ W, int N, int K,
                                                          uint8_t* __restrict__ Wq, float* __restrict__ scales) {
  pdl_wait();  // the preceding kernel on the stream is complete and visible
  pdl_launch_dependents();
  __shared__ float s_max[8];
  const int kb = blockIdx.x, nb = blockIdx.y, g = blockIdx.z;
  const int r = threadIdx.x >> 1, half = threadIdx.x & 1;
  const size_t off = (static_cast<size_t>(g) * N + static_cast<size_t>(nb) * 128 + r) * K +
                     static_cast<size_t>(kb) * 128 + half * 64;
  const uint4* src = reinterpret_cast<const uint4*>(W + off);
  float f[64];
#pragma unroll
  for (int v = 0; v < 8; ++v) {
    const uint4 raw = __ldg(src + v);
    const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      f[8 * v + 2 * i] = __uint_as_float(w[i] << 16);
      f[8 * v + 2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
  }
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 64; ++i) amax = fmaxf(amax, fabsf(f[i]));
#pragma unroll
  for (int o = 16; o; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if ((threadIdx.x & 31) == 0) s_max[threadIdx.x >> 5] = amax;
  __syncthreads();
  amax = s_max[0];
#pragma unroll
  for (int i = 1; i < 8; ++i) amax = fmaxf(amax, s_max[i]);
  const float s = group_scale<kPow2>(amax);
  uint4* dst = reinterpret_cast<uint4*>(Wq + off);
#pragma unroll
  for (int v = 0; v < 4; ++v) {
    uint32_t q[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float* p = f + 16 * v + 4 * i;
      const uint16_t lo = f32x2_to_e4m3x2(__fdiv_rn(p[0], s), __fdiv_rn(p[1], s));
      const uint16_t hi = f32x2_to_e4m3x2(__fdiv_rn(p[2], s), __fdiv_rn(p[3], s));
      q[i] = static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
    }
    dst[v] = make_uint4(q[0], q[1], q[2], q[3]);
  }
  if (threadIdx.x == 0)
    scales[(static_cast<size_t>(g) * (N / 128) + nb) * (K / 128) + kb] = s;
}

}  // namespace

int launch_quantize_weights(const void* W, int G, int N, int K, uint8_t* Wq, float* scales, cudaStream_t s,
                            bool pow2) {
  if (G == 0) return MOE_OK;
  dim3 grid(K / 128, N / 128, G);
  const __nv_bfloat16* w = static_cast<const __nv_bfloat16*>(W);
  return pow2 ? launch_pdl(__func__, quant_block_kernel<true>, grid, dim3(256), 0, s, w, N, K, Wq, scales)
              : launch_pdl(__func__, quant_block_kernel<false>, grid, dim3(256), 0, s, w, N, K, Wq, scales);
}

}  // namespace moe
