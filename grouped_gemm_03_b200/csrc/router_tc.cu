// One-launch router on the tensor cores: logits = x W_r^T (+ bias), softmax
// over all E experts and the top-k, for bf16 x and W_r, E <= 256, k <= 8.
//
// "DeepSeek MoE architecture overview" §2.2 and "R1 on A100" §3.2 describe the
// router as the logits product followed, on chip, by the softmax and a per-token
// top-k.  Here the product is a tcgen05 GEMM with M = 128 tokens per tile and
// N = E rounded up to a power of two (at least 16; the weight rows past E come
// in as zeros from the TMA bounds fill).  K is split over a thread-block
// cluster of CS CTAs (CS <= 8) so that a few hundred tokens still spread over
// the SMs.  After the main loop each CTA pushes its 128 x N fp32 partial sums
// through distributed shared memory to the CTA that owns each row (128 / CS
// rows per CTA), into the stage buffers the main loop no longer needs; the
// owner adds the CS partials in rank order, so the logits do not depend on
// timing.  No partial sum leaves the chip.
//
// Per tile, per CTA: warp 0 issues the TMA loads (x [128 x 64] and W_r [N x 64]
// per 64-wide K block, 128-byte swizzle), warp 1 one thread issues the MMAs,
// warp 2 owns the TMEM allocation, warp 4 waits for the accumulator; then every
// warp moves a column slice of its TMEM lane quarter to the rows' owners.
// The selection gives each row P threads (N / 16, at least 4, at most threads /
// rows), each over every P-th group of 4 columns.  Each logit becomes an
// order-preserving 32-bit image (-0 taken as +0; padding columns image 0, below
// every logit); round r takes the largest (image, lower column) pair over the
// row and clears it, so of equal logits the lower expert comes first.
#include <cstdint>
#include <mutex>

#include "common.cuh"
#include "ptx.cuh"

namespace moe {

// K-major TMA map (grouped_gemm.cu): box {64 bf16, box_rows}, 128-byte swizzle
bool make_map(CUtensorMap* m, const void* base, int ebytes, uint64_t rows, uint64_t K, uint32_t box_rows);

namespace {

// threads per CTA: 256, or 512 for N >= 128, where the exchange and the
// selection have 16 to 32 times more columns per row to go through
template <int NP>
constexpr int rt_threads() { return NP >= 128 ? 512 : 256; }
constexpr int kRtBM = 128;             // tokens per tile
constexpr int kRtXBytes = kRtBM * 128;  // x tile: 128 rows x 64 bf16
constexpr int kRtMaxCluster = 8;

struct RtParams {
  const float* bias;
  int T, d, E, k, renorm;
  float* logits_out;
  int32_t* idx;
  float* w;
  int* status;
  uint64_t wait_ns;
};

template <int NP>
struct RtLayout {
  static constexpr int W_BYTES = NP * 128;
  static constexpr int STAGE = kRtXBytes + W_BYTES;
  static constexpr int STAGES = NP >= 128 ? 4 : 8;
  static constexpr int RSTRIDE = NP + 4;  // floats per received row: the pad spreads rows over the banks
  static constexpr int RECV = kRtBM * RSTRIDE * 4;
  static constexpr int AREA = STAGES * STAGE > RECV ? STAGES * STAGE : RECV;
  static constexpr int SMEM = AREA + 256 + 1024;  // + barriers, + alignment slack
  static constexpr int TMEM_COLS = NP < 32 ? 32 : NP;
  static constexpr int THREADS = rt_threads<NP>();
  static_assert(NP % 16 == 0 && NP <= 256, "MMA N");
  static_assert(SMEM <= 227 * 1024, "shared memory");
};

__device__ __forceinline__ uint32_t cluster_nctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void st_cluster_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared::cluster.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d)
               : "memory");
}
// 2^x by the SFU's approximation (relative error about 2^-22; results below the
// normal range flush to zero): the terms of the softmax denominator
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
// order-preserving image of an fp32 value, -0 taken as +0; and back
__device__ __forceinline__ uint32_t ord32(float v) {
  uint32_t u = __float_as_uint(v);
  if ((u << 1) == 0u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float unord32(uint32_t o) {
  return __uint_as_float((o & 0x80000000u) ? (o & 0x7fffffffu) : ~o);
}

template <int NP>
__global__ void __launch_bounds__(rt_threads<NP>(), 1)
    router_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                     const RtParams p) {
  using L = RtLayout<NP>;
  constexpr uint32_t IDESC = ptx::make_idesc(kRtBM, NP, 1);
  constexpr float kLog2e = 1.4426950408889634f;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sX = smem;
  uint8_t* sW = smem + L::STAGES * kRtXBytes;
  float* recv = reinterpret_cast<float*>(smem);  // after the main loop: [CS][128 / CS][RSTRIDE]
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::AREA);
  uint64_t* empty = full + L::STAGES;
  uint64_t* accb = empty + L::STAGES;
  uint64_t* drain = accb + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* s_quiet = reinterpret_cast<int*>(tmem_slot + 2);  // stays 0: drains wait on their own limit only
  volatile int* s_acc_bad = reinterpret_cast<volatile int*>(tmem_slot + 3);  // the accumulator never completed

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int CS = static_cast<int>(cluster_nctarank());
  const int rank = static_cast<int>(ptx::cluster_ctarank());
  const int m0 = static_cast<int>(blockIdx.x) / CS * kRtBM;
  const int nkb = (p.d + 63) / 64;
  const int kb0 = rank * nkb / CS, kb1 = (rank + 1) * nkb / CS;  // CS <= nkb: never empty

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < L::STAGES; ++s) {
      ptx::mbar_init(&full[s], 1);
      ptx::mbar_init(&empty[s], 1);
    }
    ptx::mbar_init(accb, 1);
    ptx::mbar_init(drain, 1);
    *abort_flag = 0;
    *s_quiet = 0;
    *s_acc_bad = 0;
    ptx::fence_mbar_init();
    ptx::prefetch_tmap(&tmX);
    ptx::prefetch_tmap(&tmW);
  }
  if (warp == 2) {
    ptx::tmem_alloc(tmem_slot, L::TMEM_COLS);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // the setup above touches only on-chip state and the kernel's own parameters,
  // so it overlaps the end of the preceding kernel; global memory waits for it
  pdl_wait();
  pdl_launch_dependents();

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ producer
      uint32_t stage = 0, phase = 0, issued = 0;
      bool ok = true;
      for (int kb = kb0; kb < kb1; ++kb) {
        if (!ptx::mbar_wait(&empty[stage], phase ^ 1, abort_flag, p.wait_ns)) {
          ok = false;
          break;
        }
        ptx::mbar_arrive_expect_tx(&full[stage], L::STAGE);
        ptx::tma_load_2d(sX + stage * kRtXBytes, &tmX, &full[stage], kb * 64, m0);
        ptx::tma_load_2d(sW + stage * L::W_BYTES, &tmW, &full[stage], kb * 64, 0);
        ++issued;
        if (++stage == L::STAGES) {
          stage = 0;
          phase ^= 1;
        }
      }
      if (!ok) {
        *abort_flag = 1;
        set_status(p.status, MOE_ERR_TIMEOUT);
        // let the copies already issued land before the buffers are reused
        const uint32_t pending = issued < static_cast<uint32_t>(L::STAGES) ? issued : L::STAGES;
        uint32_t s = stage, ph = phase;
        for (uint32_t i = 0; i < pending; ++i) {
          if (s == 0) {
            s = L::STAGES - 1;
            ph ^= 1;
          } else {
            --s;
          }
          ptx::mbar_wait(&full[s], ph, s_quiet, p.wait_ns);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------------ MMA issuer
      uint32_t stage = 0, phase = 0;
      bool ok = true;
      for (int kb = kb0; kb < kb1; ++kb) {
        if (!ptx::mbar_wait(&full[stage], phase, abort_flag, p.wait_ns)) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        const uint64_t adesc = ptx::sw128_kmajor_desc(ptx::smem_u32(sX + stage * kRtXBytes));
        const uint64_t bdesc = ptx::sw128_kmajor_desc(ptx::smem_u32(sW + stage * L::W_BYTES));
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          ptx::umma_f16(tmem_base, adesc + 2 * kk, bdesc + 2 * kk, IDESC, (kb > kb0) || (kk > 0));
        ptx::umma_commit(&empty[stage]);
        if (++stage == L::STAGES) {
          stage = 0;
          phase ^= 1;
        }
      }
      if (ok) {
        ptx::umma_commit(accb);
      } else {
        *abort_flag = 1;
        set_status(p.status, MOE_ERR_TIMEOUT);
      }
      // every MMA issued must finish before TMEM is released
      ptx::umma_commit(drain);
      ptx::mbar_wait(drain, 0, s_quiet, p.wait_ns);
    }
  } else if (warp == 4) {
    // the accumulator is complete, so this CTA's stage buffers are free
    if (!ptx::mbar_wait_warp(accb, 0, abort_flag, p.wait_ns) && lane == 0) {
      *s_acc_bad = 1;
      *abort_flag = 1;
      set_status(p.status, MOE_ERR_TIMEOUT);
    }
  }
  ptx::tc_fence_before();
  __syncwarp();
  // every CTA of the cluster is past its main loop: stage buffers may be overwritten
  ptx::cluster_sync();
  ptx::tc_fence_after();

  const int R = kRtBM / CS;  // rows each CTA of the cluster selects for
  if (!*s_acc_bad) {
    // every warp moves a column slice of its TMEM lane quarter's 32 rows:
    // row (q * 32 + lane)'s partial sums go to slot `rank` of the row's owner
    constexpr int WPQ = L::THREADS / 128;  // warps per lane quarter
    constexpr int CPW = NP / WPQ;          // columns per warp: 8 to 64
    const int q = warp & 3, c0 = (warp >> 2) * CPW;
    const int row = q * 32 + lane;
    const int owner = row / R, lr = row % R;
    const uint32_t dst =
        ptx::map_to_rank(ptx::smem_u32(recv + static_cast<size_t>(rank * R + lr) * L::RSTRIDE + c0), owner);
    const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + c0;
    uint32_t r[CPW];
    if constexpr (CPW == 8) {
      ptx::tmem_ld_32x32b_x8(taddr, *reinterpret_cast<uint32_t(*)[8]>(r));
    } else if constexpr (CPW == 16) {
      ptx::tmem_ld_32x32b_x16(taddr, *reinterpret_cast<uint32_t(*)[16]>(r));
    } else {
#pragma unroll
      for (int c = 0; c < CPW; c += 32) ptx::tmem_ld_32x32b_x32(taddr + c, *reinterpret_cast<uint32_t(*)[32]>(r + c));
    }
    ptx::tmem_ld_wait();
#pragma unroll
    for (int j = 0; j < CPW / 4; ++j) st_cluster_v4(dst + 16 * j, r[4 * j], r[4 * j + 1], r[4 * j + 2], r[4 * j + 3]);
  }
  ptx::tc_fence_before();
  __syncwarp();
  // every partial sum has landed in its owner's shared memory
  ptx::cluster_sync();
  ptx::tc_fence_after();
  if (warp == 2) ptx::tmem_dealloc(tmem_base, L::TMEM_COLS);

  // ---------------------------------------------------------------- selection
  // P threads per row (a power of two, P * R <= threads): N / 16, at least 4
  // (one warp alone would run a row's whole chain with nothing to hide its
  // latency); each takes every P-th group of 4 columns.  Threads past the R
  // rows have nothing left to do.
  constexpr int PN = NP / 16 < 4 ? 4 : NP / 16;
  const int P = PN < L::THREADS / R ? PN : L::THREADS / R;
  const int lr = threadIdx.x / P, pp = threadIdx.x % P;
  const unsigned live = __ballot_sync(0xffffffffu, lr < R);
  if (lr >= R) return;
  const unsigned gmask = live;  // the lanes of whole rows: every P-group is inside it
  const int t = m0 + rank * R + lr;
  const bool tok = t < p.T;
  float* row0 = recv + static_cast<size_t>(lr) * L::RSTRIDE;  // slot 0's row, rewritten as images
  uint32_t* img = reinterpret_cast<uint32_t*>(row0);
  const size_t slot_stride = static_cast<size_t>(R) * L::RSTRIDE;
  constexpr int NCH = NP / 4;
  const int E = p.E;
  // pass A: the logits (partials added in rank order, then the bias), their
  // images in place, the running max and sum of exp(l - max)
  float m = -INFINITY, sum = 0.f;
  for (int c = pp; c < NCH; c += P) {
    float4 v = *reinterpret_cast<const float4*>(row0 + 4 * c);
    for (int s = 1; s < CS; ++s) {
      const float4 u = *reinterpret_cast<const float4*>(row0 + s * slot_stride + 4 * c);
      v.x += u.x;
      v.y += u.y;
      v.z += u.z;
      v.w += u.w;
    }
    float l[4] = {v.x, v.y, v.z, v.w};
    uint32_t o[4];
    float mc = -INFINITY;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int col = 4 * c + i;
      if (col < E) {
        l[i] += p.bias ? __ldg(p.bias + col) : 0.f;
        if (p.logits_out && tok) p.logits_out[static_cast<size_t>(t) * E + col] = l[i];
        o[i] = ord32(l[i]);
        mc = fmaxf(mc, l[i]);
      } else {
        o[i] = 0u;
        l[i] = -INFINITY;
      }
    }
    *reinterpret_cast<uint4*>(img + 4 * c) = make_uint4(o[0], o[1], o[2], o[3]);
    const float mn = fmaxf(m, mc);
    if (mn != -INFINITY) {  // a chunk of padding columns alone adds nothing
      float sc = sum * fast_exp2((m - mn) * kLog2e);
#pragma unroll
      for (int i = 0; i < 4; ++i) sc += fast_exp2((l[i] - mn) * kLog2e);
      sum = sc;
      m = mn;
    }
  }
  for (int off = 1; off < P; off <<= 1) {
    const float mo = __shfl_xor_sync(gmask, m, off), so = __shfl_xor_sync(gmask, sum, off);
    const float mn = fmaxf(m, mo);
    if (mn != -INFINITY) {  // (a thread may hold only padding columns)
      sum = sum * fast_exp2((m - mn) * kLog2e) + so * fast_exp2((mo - mn) * kLog2e);
      m = mn;
    }
  }
  const float inv_sum = 1.0f / sum;
  // k rounds: the largest (image, lower column) pair of the row, then cleared;
  // a 4-way tree per chunk keeps the dependent chain one step per chunk.  The
  // loop stays rolled (this code runs once per CTA: its size is fetch time)
  // and each pick is stored as it is found.
  int32_t* idx_row = p.idx + static_cast<size_t>(t) * p.k;
  float* w_row = p.w + static_cast<size_t>(t) * p.k;
  const bool writer = tok && pp == 0;
  float psum = 0.f;
#pragma unroll 1
  for (int r = 0; r < p.k; ++r) {
    uint32_t bi = 0u;
    int bc = NP;
#pragma unroll 1
    for (int c = pp; c < NCH; c += P) {
      const uint4 o = *reinterpret_cast<const uint4*>(img + 4 * c);
      const bool s1 = o.y > o.x, s3 = o.w > o.z;
      const uint32_t i01 = s1 ? o.y : o.x, i23 = s3 ? o.w : o.z;
      const bool s23 = i23 > i01;
      const uint32_t ic = s23 ? i23 : i01;
      const int cc = 4 * c + (s23 ? (s3 ? 3 : 2) : (s1 ? 1 : 0));
      if (ic > bi) {
        bi = ic;
        bc = cc;
      }
    }
#pragma unroll 1
    for (int off = 1; off < P; off <<= 1) {
      const uint32_t oi = __shfl_xor_sync(gmask, bi, off);
      const int oc = __shfl_xor_sync(gmask, bc, off);
      if (oi > bi || (oi == bi && oc < bc)) {
        bi = oi;
        bc = oc;
      }
    }
    if (bc < NP && (bc >> 2) % P == pp) img[bc] = 0u;  // the owning thread clears the pick
    const float pr = fast_exp2((unord32(bi) - m) * kLog2e) * inv_sum;
    psum += pr;
    if (writer) {
      idx_row[r] = bc;
      w_row[r] = pr;
    }
  }
  if (writer && p.renorm) {
#pragma unroll 1
    for (int r = 0; r < p.k; ++r) w_row[r] /= psum;  // a division: a lone pick renormalises to exactly 1
  }
}

// Cluster size: the largest power of two <= 8 that keeps every CTA resident at
// once (tiles * CS <= SMs) and gives each CTA at least one K block.
int router_tc_cluster(int T, int d) {
  const int mtiles = (T + kRtBM - 1) / kRtBM;
  const int nkb = (d + 63) / 64;
  int cs = kRtMaxCluster;
  while (cs > 1 && (mtiles * cs > num_sms() || cs > nkb)) cs >>= 1;
  return cs;
}

template <int NP>
int router_tc_launch(const void* x, const void* W_r, const float* bias, int T, int d, int E, int k, int renorm,
                     float* logits_out, int32_t* idx, float* w, int* status, cudaStream_t s) {
  using L = RtLayout<NP>;
  static bool attr_set[64] = {};
  static std::mutex mu;
  int dev = 0;
  MOE_CUDA_CHECK(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return MOE_ERR_UNSUPPORTED;
  {
    std::lock_guard<std::mutex> g(mu);
    if (!attr_set[dev]) {
      MOE_CUDA_CHECK(cudaFuncSetAttribute(router_tc_kernel<NP>, cudaFuncAttributeMaxDynamicSharedMemorySize, L::SMEM));
      attr_set[dev] = true;
    }
  }
  CUtensorMap mX, mW;
  if (!make_map(&mX, x, 2, static_cast<uint64_t>(T), static_cast<uint64_t>(d), kRtBM)) return MOE_ERR_CUDA;
  if (!make_map(&mW, W_r, 2, static_cast<uint64_t>(E), static_cast<uint64_t>(d), NP)) return MOE_ERR_CUDA;
  const int cs = router_tc_cluster(T, d);
  const int mtiles = (T + kRtBM - 1) / kRtBM;
  RtParams prm{bias, T, d, E, k, renorm, logits_out, idx, w, status, kWaitLimitNs};
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = cs;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.gridDim = dim3(mtiles * cs);
  cfg.blockDim = dim3(L::THREADS);
  cfg.dynamicSmemBytes = L::SMEM;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, router_tc_kernel<NP>, mX, mW, prm);
  return e == cudaSuccess ? MOE_OK : record_cuda_error(e, "router_tc_kernel");
}

}  // namespace

bool router_tc_applies(int x_dtype, int w_dtype, int d, int E, int k) {
  return x_dtype == MOE_BF16 && w_dtype == MOE_BF16 && E <= 256 && k <= 8 && d % 8 == 0;
}

int launch_router_tc(const void* x, const void* W_r, const float* bias, int T, int d, int E, int k, int renorm,
                     float* logits_out, int32_t* idx, float* w, int* status, cudaStream_t s) {
  if (T == 0) return MOE_OK;
  if (E <= 16) return router_tc_launch<16>(x, W_r, bias, T, d, E, k, renorm, logits_out, idx, w, status, s);
  if (E <= 32) return router_tc_launch<32>(x, W_r, bias, T, d, E, k, renorm, logits_out, idx, w, status, s);
  if (E <= 64) return router_tc_launch<64>(x, W_r, bias, T, d, E, k, renorm, logits_out, idx, w, status, s);
  if (E <= 128) return router_tc_launch<128>(x, W_r, bias, T, d, E, k, renorm, logits_out, idx, w, status, s);
  return router_tc_launch<256>(x, W_r, bias, T, d, E, k, renorm, logits_out, idx, w, status, s);
}

}  // namespace moe
