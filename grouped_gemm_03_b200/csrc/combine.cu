// Combine: gather each token's k expert outputs back to token order, weight
// them by their gate values and sum, adding the shared expert's row
// ("Dense GEMM -> GroupedGEMM -> TP MoE" §2.2 step 6; "MegaMoE ..." §2.1).
//   out[t] = Y[R + t] + sum_{j<k} w[t, j] * Y[token_to_row[t, j]]
// fp32 accumulation in that fixed order, 16-byte loads.
#include "common.cuh"

namespace moe {
namespace {

constexpr int kCombThreads = 128;

__device__ __forceinline__ void unpack8(const uint4& r, float (&f)[8]) {
  const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}

// Grid = tokens x (d / 1024): each thread owns 8 columns of one token and
// issues the k + 1 row loads for them at once.
constexpr int kCombCols = kCombThreads * 8;

template <typename OT>
__global__ void __launch_bounds__(kCombThreads) combine_kernel(const __nv_bfloat16* __restrict__ Y,
                                                              const int32_t* __restrict__ t2r,
                                                              const float* __restrict__ w, int has_shared,
                                                              int T, int d, int k, OT* __restrict__ out) {
  __shared__ int s_row[kMaxTopK];
  __shared__ float s_w[kMaxTopK];
  const int t = blockIdx.x;
  if (threadIdx.x < k) {
    s_row[threadIdx.x] = t2r[static_cast<size_t>(t) * k + threadIdx.x];
    s_w[threadIdx.x] = w[static_cast<size_t>(t) * k + threadIdx.x];
  }
  __syncthreads();
  const int c = blockIdx.y * kCombCols + threadIdx.x * 8;
  if (c >= d) return;
  const size_t R = static_cast<size_t>(T) * k;
  float acc[8];
  if (has_shared) {
    unpack8(__ldg(reinterpret_cast<const uint4*>(Y + (R + t) * d + c)), acc);
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.f;
  }
  int j = 0;
  for (; j + 4 <= k; j += 4) {  // four rows in flight
    uint4 r[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) r[u] = __ldg(reinterpret_cast<const uint4*>(Y + static_cast<size_t>(s_row[j + u]) * d + c));
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      float f[8];
      unpack8(r[u], f);
      const float wj = s_w[j + u];
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] = fmaf(wj, f[i], acc[i]);
    }
  }
  for (; j < k; ++j) {
    float f[8];
    unpack8(__ldg(reinterpret_cast<const uint4*>(Y + static_cast<size_t>(s_row[j]) * d + c)), f);
    const float wj = s_w[j];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = fmaf(wj, f[i], acc[i]);
  }
  OT* o = out + static_cast<size_t>(t) * d + c;
  if constexpr (sizeof(OT) == 4) {
    reinterpret_cast<float4*>(o)[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
    reinterpret_cast<float4*>(o)[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
  } else {
    __nv_bfloat162 h[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(acc[2 * i], acc[2 * i + 1]);
    *reinterpret_cast<uint4*>(o) = *reinterpret_cast<uint4*>(h);
  }
}

}  // namespace

int launch_combine(const void* Y, const int32_t* t2r, const float* w, int has_shared, int T, int d, int k,
                   void* out, int out_dtype, cudaStream_t s) {
  if (T == 0) return MOE_OK;
  const __nv_bfloat16* y = static_cast<const __nv_bfloat16*>(Y);
  const dim3 grid(T, (d + kCombCols - 1) / kCombCols);
  if (out_dtype == MOE_F32)
    combine_kernel<float><<<grid, kCombThreads, 0, s>>>(y, t2r, w, has_shared, T, d, k, static_cast<float*>(out));
  else
    combine_kernel<__nv_bfloat16>
        <<<grid, kCombThreads, 0, s>>>(y, t2r, w, has_shared, T, d, k, static_cast<__nv_bfloat16*>(out));
  return launch_status(__func__);
}

}  // namespace moe
