// Permute: per-expert histogram, exclusive prefix sum and scatter of tokens
// into expert-contiguous order ("Dense GEMM -> GroupedGEMM -> TP MoE" §2.2
// steps 3-4, §4.2 compute_expert_offsets; "MegaMoE ..." §4.3 same-expert
// tokens contiguous in memory).
//
// Three launches, no atomics deciding any position, so the plan is
// bit-identical run to run:
//   hist    block b counts, per expert, the (token, slot) pairs of its 32
//           tokens (shared-memory histogram) -> cnt[b][e];
//   scan    one CTA turns cnt into absolute row bases base[b][e] =
//           offsets[e] + sum_{b' < b} cnt[b'][e], plus counts / offsets;
//   scatter block b ranks its pairs by token order inside the block and
//           copies each token's row to its k destinations (and, for the
//           shared expert, to row offsets[E] + t), casting to bf16 or
//           quantising to E4M3 with one scale per 128 columns on the way.
// With a capacity C ("Dense GEMM -> GroupedGEMM -> TP MoE" §5.1: a capacity
// factor caps each expert's tokens, the rest take a fallback path) an expert
// keeps its first C pairs in token order: the scan counts min(n_e, C) rows
// per expert, and a pair whose rank in its expert reaches C gets no row
// (token_to_row = -1); the shared expert's rows follow the kept rows.
#include <mutex>

#include "common.cuh"

namespace moe {
namespace {

constexpr int kTokPerBlock = 32;
constexpr int kPermThreads = 256;

__global__ void __launch_bounds__(kPermThreads) hist_kernel(const int32_t* __restrict__ idx, int T, int E, int k,
                                                            int32_t* __restrict__ cnt, int* status) {
  pdl_wait();  // the preceding kernel on the stream is complete and visible
  pdl_launch_dependents();
  extern __shared__ int s_cnt[];
  const int b = blockIdx.x;
  const int t0 = b * kTokPerBlock;
  const int nt = min(kTokPerBlock, T - t0);
  for (int e = threadIdx.x; e < E; e += blockDim.x) s_cnt[e] = 0;
  __syncthreads();
  for (int p = threadIdx.x; p < nt * k; p += blockDim.x) {
    const size_t g = static_cast<size_t>(t0) * k + p;
    const int e = idx[g];
    bool ok = e >= 0 && e < E;
    const int j = p % k;
    for (int jj = 0; jj < j && ok; ++jj) ok = idx[g - j + jj] != e;  // distinct within a token
    if (ok)
      atomicAdd(&s_cnt[e], 1);
    else
      set_status(status, MOE_ERR_INVALID);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) cnt[static_cast<size_t>(b) * E + e] = s_cnt[e];
}

// Single CTA of 1024 threads: thread (e, c) owns expert e and a contiguous
// chunk c of the token blocks; the tpe (<= 32) threads of one expert are
// consecutive lanes of one warp, so the chunk prefix is a segmented shuffle
// scan.  Counts are read and rewritten 8 blocks at a time so that the loads
// of a batch are in flight together.
constexpr int kScanBatch = 8;

__global__ void __launch_bounds__(1024) scan_kernel(int32_t* __restrict__ base, int nblk, int E, int T,
                                                    int shared, int capacity, int32_t* __restrict__ counts,
                                                    int32_t* __restrict__ offsets) {
  pdl_wait();  // the preceding kernel on the stream is complete and visible
  pdl_launch_dependents();
  __shared__ int s_tot[1024];
  __shared__ int s_off[1024];
  __shared__ int s_warp[32];
  int tpe = 1;  // threads per expert (power of two <= 32, tpe * E <= 1024)
  while (tpe < 32 && tpe * 2 * E <= 1024 && tpe * 2 <= nblk) tpe *= 2;
  const int chunk = (nblk + tpe - 1) / tpe;
  const int e = threadIdx.x / tpe, c = threadIdx.x % tpe;
  const bool active = e < E;
  const int b0 = c * chunk, b1 = min(nblk, b0 + chunk);
  // up to 32 blocks per thread (E >= 32 with up to 1024 token blocks, or fewer
  // experts): the counts stay in registers, one round trip to read them all
  const bool held = chunk <= 32;
  int held_v[32];
  int local = 0;
  if (active && held) {
#pragma unroll
    for (int u = 0; u < 32; ++u) held_v[u] = b0 + u < b1 ? base[static_cast<size_t>(b0 + u) * E + e] : 0;
#pragma unroll
    for (int u = 0; u < 32; ++u) local += held_v[u];
  } else if (active) {
    for (int b = b0; b < b1; b += kScanBatch) {
      int v[kScanBatch];
#pragma unroll
      for (int u = 0; u < kScanBatch; ++u) v[u] = b + u < b1 ? base[static_cast<size_t>(b + u) * E + e] : 0;
#pragma unroll
      for (int u = 0; u < kScanBatch; ++u) local += v[u];
    }
  }
  // inclusive scan of the chunk sums over the expert's tpe lanes (every lane takes part)
  int incl_c = local;
  for (int o = 1; o < tpe; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl_c, o);
    if (c >= o) incl_c += y;
  }
  const int chunk_pre = incl_c - local;
  if (active && c == tpe - 1) s_tot[e] = incl_c;  // the expert's total
  __syncthreads();
  // exclusive scan of s_tot[0..E) by the whole block (one value per thread)
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  // rows an expert keeps: all of its pairs, or the first `capacity` of them
  const int mine = threadIdx.x < E ? (capacity > 0 ? min(s_tot[threadIdx.x], capacity) : s_tot[threadIdx.x]) : 0;
  int incl = mine;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) s_warp[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int w = s_warp[lane];
    int wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += y;
    }
    s_warp[lane] = wi - w;
  }
  __syncthreads();
  const int excl = incl - mine + s_warp[warp];
  if (threadIdx.x < E) {
    s_off[threadIdx.x] = excl;
    counts[threadIdx.x] = mine;
    offsets[threadIdx.x] = excl;
  }
  if (threadIdx.x == E - 1) {  // E <= 1024 = blockDim.x
    // the kept rows end where the last expert's do; the shared rows follow them
    const int used = excl + mine;
    offsets[E] = used;
    if (shared) offsets[E + 1] = used + T;
  }
  __syncthreads();
  if (active && held) {
    int run = s_off[e] + chunk_pre;
#pragma unroll
    for (int u = 0; u < 32; ++u) {
      if (b0 + u < b1) base[static_cast<size_t>(b0 + u) * E + e] = run;
      run += held_v[u];
    }
  } else if (active) {
    int run = s_off[e] + chunk_pre;
    for (int b = b0; b < b1; b += kScanBatch) {
      int v[kScanBatch];
#pragma unroll
      for (int u = 0; u < kScanBatch; ++u) v[u] = b + u < b1 ? base[static_cast<size_t>(b + u) * E + e] : 0;
#pragma unroll
      for (int u = 0; u < kScanBatch; ++u) {
        if (b + u < b1) base[static_cast<size_t>(b + u) * E + e] = run;
        run += v[u];
      }
    }
  }
}

__device__ __forceinline__ void load_row8(const float* p, float (&f)[8]) {
  const float4 a = *reinterpret_cast<const float4*>(p);
  const float4 b = *(reinterpret_cast<const float4*>(p) + 1);
  f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
  f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
}

// Columns of x one scatter block copies: the grid is (token blocks) x (d /
// kScatterCols) so that even a few hundred tokens keep every SM busy.
constexpr int kScatterCols = 512;

template <typename XT, bool kFp8, bool kPow2 = false>
__global__ void __launch_bounds__(kPermThreads) scatter_kernel(PermuteArgs a) {
  pdl_wait();  // the preceding kernel on the stream is complete and visible
  pdl_launch_dependents();
  __shared__ int s_idx[kTokPerBlock * kMaxTopK];
  __shared__ int s_row[kTokPerBlock * (kMaxTopK + 1)];
  const int b = blockIdx.x;
  const int t0 = b * kTokPerBlock;
  const int nt = min(kTokPerBlock, a.T - t0);
  const int k = a.k, E = a.E;
  const int R = a.T * k;
  const int rows_total = R + (a.shared ? a.T : 0);
  // destinations per token: its k rows (and shared row), or with gather its own row once
  const int nd = a.gather ? 1 : k + (a.shared ? 1 : 0);
  const int xp_rows = a.gather ? a.T : rows_total;  // leading dimension of xp_scales
  const bool writer = blockIdx.y == 0;   // one column block writes the index maps
  __shared__ int s_used;  // rows the experts keep: the shared rows start there
  // small count matrices: this block reduces the histogram itself (no scan launch)
  __shared__ int s_tot[kMaxExperts];      // rows each expert keeps
  __shared__ int s_pre[kMaxExperts];      // pairs of each expert in the blocks before this one
  __shared__ int s_offx[kMaxExperts + 1];  // exclusive scan of s_tot
  __shared__ int s_wsum[kPermThreads / 32];
  __shared__ int s_rank[kTokPerBlock * kMaxTopK];  // pair p's rank among the block's earlier pairs of its expert
  __shared__ int s_cnt[kMaxExperts];               // pairs per expert ranked so far
  const bool fused = a.fuse_scan;
  for (int p = threadIdx.x; p < nt * k; p += blockDim.x) s_idx[p] = a.idx[static_cast<size_t>(t0) * k + p];
  for (int e = threadIdx.x; e < E; e += blockDim.x) s_cnt[e] = 0;
  if (fused) {
    // the histogram is cnt[b'][e] at b' * E + e.  P parts per expert each sum
    // every P-th block (no atomics, a fixed order); P = 1 when E >= threads
    const int nblk = gridDim.x;
    const int P = E < static_cast<int>(blockDim.x) ? static_cast<int>(blockDim.x) / E : 1;
    if (P > 1) {
      int* s_part_tot = s_rank;  // [P][E] <= threads entries (free until the ranks are taken)
      int* s_part_pre = s_rank + blockDim.x;
      const int e = threadIdx.x % E, part = threadIdx.x / E;
      if (part < P) {
        int tot = 0, pre = 0;
        for (int b2 = part; b2 < nblk; b2 += P) {
          const int c = a.block_base[static_cast<size_t>(b2) * E + e];
          tot += c;
          pre += b2 < b ? c : 0;
        }
        s_part_tot[part * E + e] = tot;
        s_part_pre[part * E + e] = pre;
      }
      __syncthreads();
      for (int e2 = threadIdx.x; e2 < E; e2 += blockDim.x) {
        int tot = 0, pre = 0;
        for (int q = 0; q < P; ++q) {
          tot += s_part_tot[q * E + e2];
          pre += s_part_pre[q * E + e2];
        }
        s_tot[e2] = tot;
        s_pre[e2] = pre;
      }
    } else {
      for (int e2 = threadIdx.x; e2 < E; e2 += blockDim.x) {
        int tot = 0, pre = 0;
#pragma unroll 4
        for (int b2 = 0; b2 < nblk; ++b2) {
          const int c = a.block_base[static_cast<size_t>(b2) * E + e2];
          tot += c;
          pre += b2 < b ? c : 0;
        }
        s_tot[e2] = tot;
        s_pre[e2] = pre;
      }
    }
    __syncthreads();
    // kept rows per expert, then their exclusive scan (each thread 4 consecutive experts)
    int v[4], loc = 0;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int e = 4 * threadIdx.x + u;
      v[u] = e < E ? (a.capacity > 0 ? min(s_tot[e], a.capacity) : s_tot[e]) : 0;
      loc += v[u];
    }
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int incl = loc;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane == 31) s_wsum[warp] = incl;
    __syncthreads();
    int wpre = 0;
    for (int w = 0; w < warp; ++w) wpre += s_wsum[w];
    int run = wpre + incl - loc;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int e = 4 * threadIdx.x + u;
      if (e < E) {
        s_offx[e] = run;
        if (b == 0 && writer) {
          a.counts[e] = v[u];
          a.offsets[e] = run;
        }
      }
      run += v[u];
    }
    if (threadIdx.x == blockDim.x - 1) {
      s_offx[E] = run;  // the last thread's running sum is the total
      s_used = run;
      if (b == 0 && writer) {
        a.offsets[E] = run;
        if (a.shared) a.offsets[E + 1] = run + a.T;
      }
    }
  } else if (threadIdx.x == 0) {
    s_used = a.offsets[E];
  }
  __syncthreads();
  if (threadIdx.x < 32) {
    // ranks in pair order (token order: a token's experts are distinct), 32
    // pairs at a time: lanes holding the same expert find each other with a
    // match; the highest of them advances the expert's count
    const int lane = threadIdx.x;
    for (int p0 = 0; p0 < nt * k; p0 += 32) {
      const int p = p0 + lane;
      const bool in = p < nt * k;
      const int e = in ? s_idx[p] : -1;
      const bool valid = in && e >= 0 && e < E;
      const unsigned m = __match_any_sync(0xffffffffu, valid ? e : -2 - lane);
      const int prior = valid ? s_cnt[e] : 0;
      __syncwarp();
      if (valid && (m >> lane) == 1u) s_cnt[e] = prior + __popc(m);
      __syncwarp();
      if (in) s_rank[p] = prior + __popc(m & ((1u << lane) - 1u));
    }
  }
  __syncthreads();
  for (int p = threadIdx.x; p < nt * k; p += blockDim.x) {
    const int tl = p / k, j = p % k;
    const int e = s_idx[p];
    int row = 0;
    if (e >= 0 && e < E) {
      const int rank = s_rank[p];
      const int off_e = fused ? s_offx[e] : a.offsets[e];
      row = (fused ? off_e + s_pre[e] : a.block_base[static_cast<size_t>(b) * E + e]) + rank;
      // past the expert's capacity: the pair overflows and gets no row
      if (a.capacity > 0 && row - off_e >= a.capacity) row = -1;
      if (row >= R) row = 0;  // only reachable with invalid ids (status already set)
    }
    if (!a.gather) s_row[tl * nd + j] = row;
    if (writer) {
      a.token_to_row[static_cast<size_t>(t0 + tl) * k + j] = row;
      if (row >= 0) a.row_to_token[row] = t0 + tl;
    }
  }
  if (a.shared)
    for (int tl = threadIdx.x; tl < nt; tl += blockDim.x) {
      if (!a.gather) s_row[tl * nd + k] = s_used + t0 + tl;
      if (writer) a.row_to_token[s_used + t0 + tl] = t0 + tl;
    }
  if (a.gather)
    for (int tl = threadIdx.x; tl < nt; tl += blockDim.x) s_row[tl] = t0 + tl;
  if (writer && a.capacity > 0) {  // rows left unused by the overflowing pairs belong to no token
    const int end = s_used + (a.shared ? a.T : 0);
    for (int r = end + b * blockDim.x + threadIdx.x; r < rows_total; r += gridDim.x * blockDim.x)
      a.row_to_token[r] = -1;
  }
  __syncthreads();

  if (a.gather && !kFp8 && sizeof(XT) == 2) return;  // the GEMM reads x itself: no copy
  const int d = a.d;
  const int cbeg = blockIdx.y * kScatterCols;
  const int cw = min(kScatterCols, d - cbeg);
  const XT* x = static_cast<const XT*>(a.x);
  if constexpr (!kFp8) {
    // bf16 destination: 8 elements (16 bytes) per item, 4 items in flight per thread
    constexpr int U = 4;
    __nv_bfloat16* xp = static_cast<__nv_bfloat16*>(a.xp);
    const int nvec = cw / 8;
    const int items = nt * nvec;
    // a full column block has 64 vectors per token: shift and mask instead of dividing
    const bool pow2 = nvec == kScatterCols / 8;
    constexpr int kVecShift = 6;
    static_assert(kScatterCols / 8 == 1 << kVecShift, "vectors per full column block");
    for (int base = threadIdx.x; base < items; base += U * blockDim.x) {
      uint4 v[U];
      int tl[U], c[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int it = base + u * blockDim.x;
        const int q = pow2 ? it >> kVecShift : it / nvec;
        const int rmd = pow2 ? it & ((1 << kVecShift) - 1) : it - q * nvec;
        tl[u] = it < items ? q : -1;
        c[u] = it < items ? cbeg + rmd * 8 : 0;
        if (tl[u] < 0) continue;
        const XT* src = x + static_cast<size_t>(t0 + tl[u]) * d + c[u];
        if constexpr (sizeof(XT) == 2) {
          v[u] = *reinterpret_cast<const uint4*>(src);
        } else {
          float f[8];
          load_row8(reinterpret_cast<const float*>(src), f);
          __nv_bfloat162 h[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
          v[u] = *reinterpret_cast<uint4*>(h);
        }
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        if (tl[u] < 0) continue;
        for (int j = 0; j < nd; ++j) {
          const int row = s_row[tl[u] * nd + j];
          if (row >= 0) *reinterpret_cast<uint4*>(xp + static_cast<size_t>(row) * d + c[u]) = v[u];
        }
      }
    }
  } else {
    // E4M3 destination: 16 threads quantise one 128-column group of one token
    uint8_t* xp = static_cast<uint8_t*>(a.xp);
    const int ngrp = cw / 128;
    const int sub = threadIdx.x & 15;
    const int half = (threadIdx.x >> 4) & 1;
    const int total = nt * ngrp;
    // warp-uniform trip count: both half-warps run every iteration (the
    // shuffles below name all 32 lanes), the idle half on dummy data
    for (int base = (threadIdx.x >> 5) * 2; base < total; base += (blockDim.x >> 5) * 2) {
      const int it = base + half;
      const bool act = it < total;
      const int tl = act ? it / ngrp : 0, gi = act ? cbeg / 128 + it % ngrp : 0;
      const int c = gi * 128 + sub * 8;
      float f[8];
      const XT* src = x + static_cast<size_t>(t0 + tl) * d + c;
      if (!act) {
#pragma unroll
        for (int i = 0; i < 8; ++i) f[i] = 0.f;
      } else if constexpr (sizeof(XT) == 2) {
        const uint4 raw = *reinterpret_cast<const uint4*>(src);
        const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          f[2 * i] = __uint_as_float(w[i] << 16);
          f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
        }
      } else {
        load_row8(reinterpret_cast<const float*>(src), f);
        // experts consume x rounded to bf16
#pragma unroll
        for (int i = 0; i < 8; ++i) f[i] = __bfloat162float(__float2bfloat16_rn(f[i]));
      }
      float amax = 0.f;
#pragma unroll
      for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(f[i]));
#pragma unroll
      for (int o = 8; o; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
      const float s = group_scale<kPow2>(amax);
      uint32_t q[2];
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const uint16_t lo = f32x2_to_e4m3x2(__fdiv_rn(f[4 * i], s), __fdiv_rn(f[4 * i + 1], s));
        const uint16_t hi = f32x2_to_e4m3x2(__fdiv_rn(f[4 * i + 2], s), __fdiv_rn(f[4 * i + 3], s));
        q[i] = static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
      }
      const uint2 qv = make_uint2(q[0], q[1]);
      if (!act) continue;
      for (int j = 0; j < nd; ++j) {
        const int row = s_row[tl * nd + j];
        if (row < 0) continue;  // overflowed its expert's capacity
        *reinterpret_cast<uint2*>(xp + static_cast<size_t>(row) * d + c) = qv;
        if (sub == 0) a.xp_scales[static_cast<size_t>(gi) * xp_rows + row] = s;
      }
    }
  }
}

}  // namespace

int permute_blocks(int T) { return (T + kTokPerBlock - 1) / kTokPerBlock; }

bool permute_fuses_scan(int T, int E) {
  return static_cast<long long>(permute_blocks(T)) * E <= kFusedScanCounts;
}

int launch_permute(const PermuteArgs& a, cudaStream_t s) {
  const int nblk = permute_blocks(a.T);
  if (a.T == 0) {
    // no tokens: counts are zero and every offset is zero
    MOE_CUDA_CHECK(cudaMemsetAsync(a.counts, 0, sizeof(int32_t) * a.E, s));
    MOE_CUDA_CHECK(cudaMemsetAsync(a.offsets, 0, sizeof(int32_t) * (a.E + 1 + (a.shared ? 1 : 0)), s));
    return MOE_OK;
  }
  int st = launch_pdl("hist_kernel", hist_kernel, dim3(nblk), dim3(kPermThreads), sizeof(int) * a.E, s, a.idx, a.T,
                      a.E, a.k, a.block_base, a.status);
  if (st != MOE_OK) return st;
  PermuteArgs b = a;
  b.fuse_scan = permute_fuses_scan(a.T, a.E) ? 1 : 0;
  if (!b.fuse_scan) {
    st = launch_pdl("scan_kernel", scan_kernel, dim3(1), dim3(1024), 0, s, a.block_base, nblk, a.E, a.T, a.shared,
                    a.capacity, a.counts, a.offsets);
    if (st != MOE_OK) return st;
  }
  const bool fp8 = is_e4m3(a.xp_dtype);
  const bool mx = a.xp_dtype == MOE_MXE4M3;
  const bool copies = !(a.gather && !fp8 && a.x_dtype == MOE_BF16);
  const dim3 grid(nblk, copies ? (a.d + kScatterCols - 1) / kScatterCols : 1);
  const dim3 block(kPermThreads);
  if (a.x_dtype == MOE_BF16) {
    if (!fp8) return launch_pdl("scatter_kernel", scatter_kernel<__nv_bfloat16, false>, grid, block, 0, s, b);
    return mx ? launch_pdl("scatter_kernel", scatter_kernel<__nv_bfloat16, true, true>, grid, block, 0, s, b)
              : launch_pdl("scatter_kernel", scatter_kernel<__nv_bfloat16, true>, grid, block, 0, s, b);
  }
  if (!fp8) return launch_pdl("scatter_kernel", scatter_kernel<float, false>, grid, block, 0, s, b);
  return mx ? launch_pdl("scatter_kernel", scatter_kernel<float, true, true>, grid, block, 0, s, b)
            : launch_pdl("scatter_kernel", scatter_kernel<float, true>, grid, block, 0, s, b);
}

}  // namespace moe

// ---------------------------------------------------------------------------
// Allocation-free permute (moe_permute_noalloc).
//
// Some callers cannot hand this library a workspace: a plugin whose host
// runtime owns all device memory and offers none, or a serving loop whose
// memory plan is frozen at start-up and allows no allocation afterwards.
// For them the permute's scratch (the status word and the per-block expert
// counts) lives in this file-scope device array instead of a caller
// workspace.  Every GPU that loads the library keeps the array (1 MiB + 256
// bytes) until the process exits; all calls on a device share it, so calls
// whose kernels overlap on the GPU (two streams, say) race on it and must be
// ordered by the caller.  A call rewrites every count it reads and clears
// the status word first, so what a previous call left there does not matter.
namespace moe {
namespace {

constexpr int kNoAllocStatusWords = 64;          // status word, padded to 256 bytes
constexpr size_t kNoAllocCountWords = 262144;    // per-block expert counts (1 MiB of int32)

static __device__ __align__(256) int32_t g_permute_scratch[kNoAllocStatusWords + kNoAllocCountWords];

// The device address of a __device__ array belongs to the CUDA context the
// module is loaded in, not to a device ordinal: a caller may drive the
// library from a context of its own, and a context destroyed by
// cudaDeviceReset is replaced by a new one with the module loaded afresh.
// So the address is cached per context, keyed by the context's unique id
// (cuCtxGetId: never reused within the process, unlike a CUcontext handle).
using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

struct ScratchEntry {
  unsigned long long ctx_id;
  int32_t* ptr;
};
std::mutex g_scratch_mu;
ScratchEntry g_scratch_cache[64] = {};
int g_scratch_used = 0;
int g_scratch_next = 0;  // next entry to replace once the table is full

template <typename Fn>
Fn driver_entry(const char* name) {
  void* f = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint(name, &f, cudaEnableDefault, &q) != cudaSuccess || q != cudaDriverEntryPointSuccess)
    return nullptr;
  return reinterpret_cast<Fn>(f);
}

// Device address of g_permute_scratch in the current context.  In host code
// the array's name is only a host-side stand-in, so it must never be passed
// to a kernel; the address is looked up once per context, with that context
// current, and cached.
int noalloc_scratch(int32_t** out) {
  static const CtxGetCurrentFn get_ctx = driver_entry<CtxGetCurrentFn>("cuCtxGetCurrent");
  static const CtxGetIdFn get_id = driver_entry<CtxGetIdFn>("cuCtxGetId");
  if (!get_ctx || !get_id) return record_cuda_error(cudaErrorNotSupported, "cuCtxGetCurrent / cuCtxGetId");
  CUcontext ctx = nullptr;
  if (get_ctx(&ctx) != CUDA_SUCCESS) return record_cuda_error(cudaErrorDeviceUninitialized, "cuCtxGetCurrent");
  void* fresh = nullptr;
  if (ctx == nullptr) {
    // no context is current on this thread yet: the runtime binds the
    // current device's primary context on its first call, this lookup
    const cudaError_t e = cudaGetSymbolAddress(&fresh, g_permute_scratch);
    if (e != cudaSuccess) return record_cuda_error(e, "cudaGetSymbolAddress(g_permute_scratch)");
    if (get_ctx(&ctx) != CUDA_SUCCESS || ctx == nullptr)
      return record_cuda_error(cudaErrorDeviceUninitialized, "no current CUDA context for moe_permute_noalloc");
  }
  unsigned long long id = 0;
  if (get_id(ctx, &id) != CUDA_SUCCESS) return record_cuda_error(cudaErrorDeviceUninitialized, "cuCtxGetId");
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  for (int i = 0; i < g_scratch_used; ++i)
    if (g_scratch_cache[i].ctx_id == id) {
      *out = g_scratch_cache[i].ptr;
      return MOE_OK;
    }
  void* p = fresh;
  if (p == nullptr) {
    const cudaError_t e = cudaGetSymbolAddress(&p, g_permute_scratch);
    if (e != cudaSuccess) return record_cuda_error(e, "cudaGetSymbolAddress(g_permute_scratch)");
  }
  if (p == nullptr) return record_cuda_error(cudaErrorInvalidSymbol, "cudaGetSymbolAddress(g_permute_scratch)");
  // a bounded table: once full, the oldest entry is replaced
  int slot;
  if (g_scratch_used < 64) {
    slot = g_scratch_used++;
  } else {
    slot = g_scratch_next;
    g_scratch_next = (g_scratch_next + 1) % 64;
  }
  g_scratch_cache[slot] = {id, static_cast<int32_t*>(p)};
  *out = static_cast<int32_t*>(p);
  return MOE_OK;
}

}  // namespace
}  // namespace moe

extern "C" int moe_permute_noalloc(const void* x, int x_dtype, const int32_t* topk_idx, int T, int d, int E, int k,
                                   int append_shared, int xp_dtype, void* xp, float* xp_scales, int32_t* counts,
                                   int32_t* offsets, int32_t* row_to_token, int32_t* token_to_row, void* stream) {
  using namespace moe;
  if (T < 0 || d <= 0 || E <= 0 || k <= 0 || k > E || k > kMaxTopK || E > kMaxExperts) return MOE_ERR_INVALID;
  if (static_cast<long long>(T) * (k + 1) > kMaxPermuteRows) return MOE_ERR_UNSUPPORTED;
  if (static_cast<size_t>(permute_blocks(T)) * static_cast<size_t>(E) > kNoAllocCountWords)
    return MOE_ERR_UNSUPPORTED;  // beyond the built-in scratch: use moe_permute with a workspace
  if (x_dtype != MOE_F32 && x_dtype != MOE_BF16) return MOE_ERR_INVALID;
  if (xp_dtype != MOE_BF16 && !is_e4m3(xp_dtype)) return MOE_ERR_INVALID;
  if (d % 8 != 0 || (is_e4m3(xp_dtype) && d % 128 != 0)) return MOE_ERR_UNSUPPORTED;
  if (!counts || !offsets) return MOE_ERR_INVALID;
  if (T > 0 && (!x || !topk_idx || !xp || !row_to_token || !token_to_row)) return MOE_ERR_INVALID;
  if (T > 0 && is_e4m3(xp_dtype) && !xp_scales) return MOE_ERR_INVALID;
  if (reinterpret_cast<uintptr_t>(x) % 16 || reinterpret_cast<uintptr_t>(xp) % 16) return MOE_ERR_INVALID;
  int32_t* scratch = nullptr;
  const int st = noalloc_scratch(&scratch);
  if (st != MOE_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(scratch, 0, sizeof(int32_t), s) != cudaSuccess) return MOE_ERR_CUDA;
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
  a.block_base = scratch + kNoAllocStatusWords;
  a.status = scratch;
  return launch_permute(a, s);
}
