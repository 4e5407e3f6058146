// Combine: gather each token's k expert outputs back to token order, weight
// them by their gate values and sum, adding the shared expert's row
// ("Dense GEMM -> GroupedGEMM -> TP MoE" §2.2 step 6; "MegaMoE ..." §2.1).
//   out[t] = Y[R + t] + sum_{j<k} w[t, j] * Y[token_to_row[t, j]]
// fp32 accumulation in that fixed order, 16-byte loads.  R is T*k, or the
// first shared row the permute recorded (offsets[E]) when experts have a
// capacity; a slot whose pair overflowed (token_to_row < 0) adds nothing.
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

// Grid = tokens x (d / 2048): each thread owns 16 columns (two 16-byte
// pieces) of one token and issues the loads of all k + 1 rows for them before
// it accumulates.
constexpr int kCombCols = kCombThreads * 16;

template <typename OT>
__device__ __forceinline__ void store8(OT* o, const float (&acc)[8]) {
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

template <typename OT>
__global__ void __launch_bounds__(kCombThreads) combine_kernel(const __nv_bfloat16* __restrict__ Y,
                                                              const int32_t* __restrict__ t2r,
                                                              const float* __restrict__ w, int has_shared,
                                                              int T, int d, int k, OT* __restrict__ out,
                                                              const int32_t* __restrict__ shared_base) {
  pdl_wait();  // the preceding kernel on the stream is complete and visible
  pdl_launch_dependents();
  const int t = blockIdx.x;
  const int c0 = blockIdx.y * kCombCols + threadIdx.x * 8;               // first piece
  const int c1 = c0 + kCombThreads * 8;                                   // second piece
  const bool p0 = c0 < d, p1 = c1 < d;
  if (!p0) return;
  const size_t R = shared_base ? static_cast<size_t>(__ldg(shared_base)) : static_cast<size_t>(T) * k;
  float a0[8], a1[8];
  if (has_shared) {
    const __nv_bfloat16* ys = Y + (R + t) * d;
    unpack8(__ldg(reinterpret_cast<const uint4*>(ys + c0)), a0);
    if (p1) unpack8(__ldg(reinterpret_cast<const uint4*>(ys + c1)), a1);
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) a0[i] = a1[i] = 0.f;
  }
  const int32_t* rows = t2r + static_cast<size_t>(t) * k;
  const float* ws = w + static_cast<size_t>(t) * k;
  int j = 0;
  for (; j + 4 <= k; j += 4) {  // four rows x two pieces in flight
    uint4 r0[4], r1[4];
    float wj[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int row = __ldg(rows + j + u);
      // an overflowed slot (row < 0) contributes +0 * 0: the sum is unchanged
      const __nv_bfloat16* yr = Y + static_cast<size_t>(row < 0 ? 0 : row) * d;
      wj[u] = row < 0 ? 0.f : __ldg(ws + j + u);
      r0[u] = r1[u] = make_uint4(0, 0, 0, 0);
      if (row >= 0) {
        r0[u] = __ldg(reinterpret_cast<const uint4*>(yr + c0));
        if (p1) r1[u] = __ldg(reinterpret_cast<const uint4*>(yr + c1));
      }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      float f[8];
      unpack8(r0[u], f);
#pragma unroll
      for (int i = 0; i < 8; ++i) a0[i] = fmaf(wj[u], f[i], a0[i]);
      if (p1) {
        unpack8(r1[u], f);
#pragma unroll
        for (int i = 0; i < 8; ++i) a1[i] = fmaf(wj[u], f[i], a1[i]);
      }
    }
  }
  for (; j < k; ++j) {
    const int row = __ldg(rows + j);
    if (row < 0) continue;  // overflowed its expert's capacity
    const __nv_bfloat16* yr = Y + static_cast<size_t>(row) * d;
    const float wj = __ldg(ws + j);
    float f[8];
    unpack8(__ldg(reinterpret_cast<const uint4*>(yr + c0)), f);
#pragma unroll
    for (int i = 0; i < 8; ++i) a0[i] = fmaf(wj, f[i], a0[i]);
    if (p1) {
      unpack8(__ldg(reinterpret_cast<const uint4*>(yr + c1)), f);
#pragma unroll
      for (int i = 0; i < 8; ++i) a1[i] = fmaf(wj, f[i], a1[i]);
    }
  }
  OT* o = out + static_cast<size_t>(t) * d;
  store8(o + c0, a0);
  if (p1) store8(o + c1, a1);
}

}  // namespace

int launch_combine(const void* Y, const int32_t* t2r, const float* w, int has_shared, int T, int d, int k,
                   void* out, int out_dtype, cudaStream_t s, const int32_t* shared_base) {
  if (T == 0) return MOE_OK;
  const __nv_bfloat16* y = static_cast<const __nv_bfloat16*>(Y);
  const dim3 grid(T, (d + kCombCols - 1) / kCombCols);
  if (out_dtype == MOE_F32)
    return launch_pdl(__func__, combine_kernel<float>, grid, dim3(kCombThreads), 0, s, y, t2r, w, has_shared, T, d, k,
                      static_cast<float*>(out), shared_base);
  return launch_pdl(__func__, combine_kernel<__nv_bfloat16>, grid, dim3(kCombThreads), 0, s, y, t2r, w, has_shared, T,
                    d, k, static_cast<__nv_bfloat16*>(out), shared_base);
}

}  // namespace moe
