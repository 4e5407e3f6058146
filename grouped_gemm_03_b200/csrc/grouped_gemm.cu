// Persistent grouped GEMM on the 5th-generation tensor cores (tcgen05 + TMEM).
//
// "MegaMoE ..." §4.3: one launch computes many GEMM problems that share N and
// K but have their own M_i; tokens of one expert are contiguous, so problem
// g is rows offsets[g] .. offsets[g+1]-1 of one A matrix.  "Dense GEMM ->
// GroupedGEMM -> TP MoE" §2.3 gives the call shape; its pointer arrays become
// base + offset arithmetic done on the device (its §4.3 / §5.4 note that
// host-built pointer arrays raced), and the expert sizes never leave the GPU.
//
// Structure (one CTA per SM, persistent, 6 warps):
//   warp 0      TMA producer: A tile [128 x 128 B] and B tile [N_mma x 128 B]
//               per k-step into an S-stage shared-memory ring (mbarrier
//               full/empty pairs, 128-byte swizzle);
//   warp 1      allocates TMEM, one thread issues tcgen05.mma 128 x N_mma x 16
//               into one of two TMEM accumulators and commits stage / tile
//               completion to mbarriers;
//   warps 2-5   epilogue: tcgen05.ld the accumulator (thread = row), apply the
//               SiLU gate or a plain cast, store the row segment with 16-byte
//               stores predicated on the row belonging to the group
//               ("MegaMoE ..." §5.3 tail rows), then release the accumulator.
// The two accumulators let the epilogue of tile i overlap the main loop of
// tile i+1 ("MegaMoE ..." §5.2 double buffering, here in TMEM).
//
// Tiles: the scheduler enumerates, group by group, ceil(M_g / 128) m-blocks x
// (N / N_out) n-blocks, m-blocks of one n-block adjacent so that CTAs running
// at the same time share the weight tile through L2.  An expert with no rows
// contributes no tile and its weights are never read.  CTA c takes tiles
// c, c + gridDim.x, ...  A tile that runs past its group's last row reads the
// next group's rows (or TMA zero fill past the end of A); those rows are
// computed and discarded, never stored.
//
// SiLU-gate epilogue: per k-step the B tile is [gate rows n0..n0+127 ; up rows
// N+n0..N+n0+127], so one 128 x 256 MMA produces gate and up side by side in
// TMEM and the epilogue writes h = silu(g) * u for 128 output columns.
//
// Variants, chosen on the host from the shapes alone (plan_grouped_gemm):
//   gg_bf16_kernel       the structure above (128-row tiles, N_mma 64..256);
//   gg_bf16_pair_kernel  CTA pairs sharing 256-row tiles (large groups);
//   gg_bf16_swap_kernel  weights on the MMA's 128-row side, tokens on the
//                        32-wide side (groups of a few tokens);
//   gg_fp8_kernel        E4M3 operands, scales applied per 128-wide K block.
// Every kernel begins with the programmatic-dependent-launch wait (common.cuh).
#include <cstdio>
#include <mutex>

#include "common.cuh"
#include "ptx.cuh"

namespace moe {
namespace {

constexpr int BM = 128;
constexpr int kThreads = 192;
constexpr int kSmemBudget = 220 * 1024;

// Shared memory of the single-CTA bf16 kernel.  With bf16 output and no
// gate, each of the four epilogue warps stages its 32 rows in two 4 KB boxes
// (32 rows x 64 columns, 128-byte swizzled) for bulk tensor stores, at OUTB;
// that takes one operand stage, which the gated kernel (half the output
// columns) measured better kept.
template <int MMA_N, bool kStageOut>
struct Tile {
  static constexpr int A_BYTES = BM * 128;
  static constexpr int B_BYTES = MMA_N * 128;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int TABLE_BYTES = 2 * (kMaxGroups + 2) * 4;
  // one 4 KiB box buffer per epilogue warp: with it, four operand stages of
  // 48 KiB still fit (two buffers would leave three)
  static constexpr int OUT_WARP = kStageOut ? 4096 : 0;
  static constexpr int STAGES_RAW = (kSmemBudget - 2048 - TABLE_BYTES - 512 - 4 * OUT_WARP) / STAGE_BYTES;
  static constexpr int STAGES = STAGES_RAW > 8 ? 8 : STAGES_RAW;
  static constexpr int TMEM_COLS = 2 * MMA_N;
  static constexpr int OUTB = (STAGES * STAGE_BYTES + 512 + TABLE_BYTES + 1023) / 1024 * 1024;
  static constexpr int SMEM = 1024 + OUTB + 4 * OUT_WARP;
};

struct Params {
  const int32_t* offsets;
  int G_total;  // groups, including the extra one
  int G_main;   // groups whose weights come from tmB; group G_main (if any) uses tmBx
  int N, K, rows;
  int ksplit;          // K is split into this many slices (fp32 partial outputs, no gate)
  size_t split_stride; // elements between the partial outputs of consecutive slices
  void* C;
  int* status;
  // E4M3 operands only
  const float* A_scales;   // [K/128][rows]
  const float* B_scales;   // [G_main][Nb/128][K/128]
  const float* Bx_scales;  // [Nb/128][K/128] of the extra group
  float* C_scales;         // [N/128][rows] when C is E4M3
  uint64_t wait_ns;        // limit of every pipeline wait
  int stall;               // self-test: the epilogue first waits on a barrier no thread arrives at
  // gathered A ("permute in the load"): A row r of the grouped problem is row
  // a_rows[r] of the a_src_rows-row tensor tmA maps (box one row high); < 0: any row
  const int32_t* a_rows;
  int a_src_rows;
};

// Source rows of the 4 A rows lane `lane` gathers for the tile starting at
// row a_row: rows past the problem or without a token read row 0 (never stored).
__device__ __forceinline__ void gather_rows(const Params& p, int a_row, int lane, int (&tok)[4]) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = a_row + 4 * lane + i;
    const int v = r < p.rows ? __ldg(p.a_rows + r) : 0;
    tok[i] = (v < 0 || v >= p.a_src_rows) ? 0 : v;
  }
}

// Source row of A row r (gathered or not), for per-row A scales.
__device__ __forceinline__ int a_source_row(const Params& p, int r) {
  if (!p.a_rows) return r;
  const int v = r < p.rows ? __ldg(p.a_rows + r) : 0;
  return (v < 0 || v >= p.a_src_rows) ? 0 : v;
}

struct TileCoord {
  int g, mb, nb, ks, m_g;
};

// Largest g in [0, G) with tile_start[g] <= tile.
__device__ __forceinline__ int find_group(const int* tile_start, int G, int tile) {
  int lo = 0, hi = G - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (tile_start[mid] <= tile)
      lo = mid;
    else
      hi = mid - 1;
  }
  return lo;
}

// Tile t of group g: m-block fastest, then n-block, then K slice.
__device__ __forceinline__ TileCoord decode_tile(const int* s_tile, const int* s_off, int G, int nt, int tile) {
  TileCoord c;
  c.g = find_group(s_tile, G, tile);
  c.m_g = s_off[c.g + 1] - s_off[c.g];
  const int mt = (c.m_g + BM - 1) / BM;
  const int tl = tile - s_tile[c.g];
  const int q = tl / mt;
  c.mb = tl % mt;
  c.ks = q / nt;
  c.nb = q % nt;
  return c;
}

template <int MMA_N, int EPI, int OUT>
__global__ void __launch_bounds__(kThreads, 1)
    gg_bf16_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ CUtensorMap tmBx, const __grid_constant__ CUtensorMap tmC, const Params p) {
  pdl_wait();  // the preceding kernel on the stream is complete and visible
  pdl_launch_dependents();
  using L = Tile<MMA_N, OUT == 0 && EPI == 0>;
  constexpr int OUT_COLS = EPI ? MMA_N / 2 : MMA_N;
  constexpr uint32_t IDESC = ptx::make_idesc(BM, MMA_N, 1);
  // 64-row MMA of a group's short last tile: its rows 16j + i (i < 16) land in
  // TMEM lane 32j + i, the first half of each 32-lane quarter
  constexpr uint32_t IDESC64 = ptx::make_idesc(64, MMA_N, 1);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + L::STAGES * L::A_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(sB + L::STAGES * L::B_BYTES);
  uint64_t* empty = full + L::STAGES;
  uint64_t* tfull = empty + L::STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint64_t* never = drain + 1;  // self-test only: initialised, never arrived at
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(never + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* s_bad = reinterpret_cast<int*>(tmem_slot + 2);
  int* s_off = reinterpret_cast<int*>(smem + L::STAGES * L::STAGE_BYTES + 512);
  int* s_tile = s_off + kMaxGroups + 2;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = p.G_total;
  const int nt = p.N / OUT_COLS;
  const int ntk = nt * p.ksplit;  // tiles per m-block

  // ---- group tables: row offsets and the exclusive prefix of tile counts
  if (warp == 0) {
    // no offsets array: a single group spanning every row of A
    for (int g = lane; g <= G; g += 32) s_off[g] = p.offsets ? p.offsets[g] : (g == 0 ? 0 : p.rows);
    __syncwarp();
    const int per = (G + 31) / 32;
    const int g0 = min(G, lane * per), g1 = min(G, g0 + per);
    int bad = 0, mine = 0;
    for (int g = g0; g < g1; ++g) {
      const int m = s_off[g + 1] - s_off[g];
      if (m < 0) bad = 1;
      mine += (max(m, 0) + BM - 1) / BM * ntk;
    }
    int incl = mine;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    int run = incl - mine;
    for (int g = g0; g < g1; ++g) {
      s_tile[g] = run;
      run += (max(s_off[g + 1] - s_off[g], 0) + BM - 1) / BM * ntk;
    }
    if (lane == 31) s_tile[G] = incl;
    if (lane == 0 && (s_off[0] != 0 || s_off[G] > p.rows)) bad = 1;
    bad = __any_sync(0xffffffffu, bad);
    if (lane == 0) {
      *s_bad = bad;
      *abort_flag = 0;
      if (bad && blockIdx.x == 0) set_status(p.status, MOE_ERR_BAD_OFFSETS);
    }
  }
  __syncthreads();
  if (*s_bad) return;  // uniform: nothing loaded, nothing allocated

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < L::STAGES; ++s) {
      ptx::mbar_init(&full[s], 1);
      ptx::mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      ptx::mbar_init(&tfull[a], 1);
      ptx::mbar_init(&tempty[a], 128);
    }
    ptx::mbar_init(drain, 1);
    ptx::mbar_init(never, 1);
    ptx::fence_mbar_init();
    ptx::prefetch_tmap(&tmA);
    ptx::prefetch_tmap(&tmB);
    ptx::prefetch_tmap(&tmBx);
  }
  if (warp == 1) {
    ptx::tmem_alloc(tmem_slot, L::TMEM_COLS);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int total = s_tile[G];
  const int nk = p.K / 64;

  if (warp == 0 && p.a_rows) {
    // -------------------------------------------------------------- producer, gathered A
    // lane l brings A rows 4l..4l+3 of the tile (one tile::gather4 each k-step);
    // lane 0 also waits for the stage and loads B
    uint32_t stage = 0, phase = 0, issued = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
      const TileCoord tc = decode_tile(s_tile, s_off, G, nt, tile);
      const int g = tc.g, nb = tc.nb;
      int tok[4];
      gather_rows(p, s_off[g] + tc.mb * BM, lane, tok);
      const bool extra = g >= p.G_main;
      const CUtensorMap* mB = extra ? &tmBx : &tmB;
      const int gb = extra ? 0 : g;
      const int kb0 = tc.ks * nk / p.ksplit, kb1 = (tc.ks + 1) * nk / p.ksplit;
      for (int kb = kb0; kb < kb1; ++kb) {
        int go = 1;
        if (lane == 0) {
          go = ptx::mbar_wait(&empty[stage], phase ^ 1, abort_flag, p.wait_ns);
          if (go) ptx::mbar_arrive_expect_tx(&full[stage], L::STAGE_BYTES);
        }
        if (!__shfl_sync(0xffffffffu, go, 0)) {
          ok = false;
          break;
        }
        ptx::tma_gather4(sA + stage * L::A_BYTES + lane * 512, &tmA, &full[stage], kb * 64, tok[0], tok[1], tok[2],
                         tok[3]);
        if (lane == 0) {
          if (EPI) {
            const int brow = gb * 2 * p.N + nb * (MMA_N / 2);
            ptx::tma_load_2d(sB + stage * L::B_BYTES, mB, &full[stage], kb * 64, brow);
            ptx::tma_load_2d(sB + stage * L::B_BYTES + (MMA_N / 2) * 128, mB, &full[stage], kb * 64, brow + p.N);
          } else {
            ptx::tma_load_2d(sB + stage * L::B_BYTES, mB, &full[stage], kb * 64, gb * p.N + nb * MMA_N);
          }
        }
        ++issued;
        if (++stage == L::STAGES) {
          stage = 0;
          phase ^= 1;
        }
      }
    }
    if (!ok && lane == 0) {
      *abort_flag = 1;
      set_status(p.status, MOE_ERR_TIMEOUT);
      const uint32_t pending = issued < static_cast<uint32_t>(L::STAGES) ? issued : L::STAGES;
      uint32_t s2 = stage, ph = phase;
      for (uint32_t i = 0; i < pending; ++i) {
        if (s2 == 0) {
          s2 = L::STAGES - 1;
          ph ^= 1;
        } else {
          --s2;
        }
        ptx::mbar_wait(&full[s2], ph, reinterpret_cast<volatile int*>(s_bad), p.wait_ns);
      }
    }
  } else if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ producer
      uint32_t stage = 0, phase = 0;
      uint32_t issued = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
        const TileCoord tc = decode_tile(s_tile, s_off, G, nt, tile);
        const int g = tc.g, nb = tc.nb;
        const int a_row = s_off[g] + tc.mb * BM;
        const bool extra = g >= p.G_main;
        const CUtensorMap* mB = extra ? &tmBx : &tmB;
        const int gb = extra ? 0 : g;
        const int kb0 = tc.ks * nk / p.ksplit, kb1 = (tc.ks + 1) * nk / p.ksplit;
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!ptx::mbar_wait(&empty[stage], phase ^ 1, abort_flag, p.wait_ns)) {
            ok = false;
            break;
          }
          ptx::mbar_arrive_expect_tx(&full[stage], L::STAGE_BYTES);
          ptx::tma_load_2d(sA + stage * L::A_BYTES, &tmA, &full[stage], kb * 64, a_row);
          if (EPI) {
            const int brow = gb * 2 * p.N + nb * (MMA_N / 2);
            ptx::tma_load_2d(sB + stage * L::B_BYTES, mB, &full[stage], kb * 64, brow);
            ptx::tma_load_2d(sB + stage * L::B_BYTES + (MMA_N / 2) * 128, mB, &full[stage], kb * 64,
                             brow + p.N);
          } else {
            ptx::tma_load_2d(sB + stage * L::B_BYTES, mB, &full[stage], kb * 64, gb * p.N + nb * MMA_N);
          }
          ++issued;
          if (++stage == L::STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      if (!ok) {
        *abort_flag = 1;
        set_status(p.status, MOE_ERR_TIMEOUT);
        // let the copies already issued land before the CTA exits
        const uint32_t pending = issued < static_cast<uint32_t>(L::STAGES) ? issued : L::STAGES;
        uint32_t s = stage, ph = phase;
        for (uint32_t i = 0; i < pending; ++i) {
          if (s == 0) {
            s = L::STAGES - 1;
            ph ^= 1;
          } else {
            --s;
          }
          ptx::mbar_wait(&full[s], ph, reinterpret_cast<volatile int*>(s_bad), p.wait_ns);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------------ MMA issuer
      uint32_t stage = 0, phase = 0;
      bool ok = true;
      int it = 0;
      for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x, ++it) {
        const int acc = it & 1;
        const uint32_t use = static_cast<uint32_t>(it >> 1);
        if (!ptx::mbar_wait(&tempty[acc], (use & 1) ^ 1, abort_flag, p.wait_ns)) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * MMA_N;
        const TileCoord tcm = decode_tile(s_tile, s_off, G, nt, tile);
        const int ks = tcm.ks;
        // a group's last tile of at most 64 rows: a 64-row MMA (half the work)
        const uint32_t idesc = tcm.m_g - tcm.mb * BM <= 64 ? IDESC64 : IDESC;
        const int kb0 = ks * nk / p.ksplit, kb1 = (ks + 1) * nk / p.ksplit;
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!ptx::mbar_wait(&full[stage], phase, abort_flag, p.wait_ns)) {
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          const uint64_t adesc = ptx::sw128_kmajor_desc(ptx::smem_u32(sA + stage * L::A_BYTES));
          const uint64_t bdesc = ptx::sw128_kmajor_desc(ptx::smem_u32(sB + stage * L::B_BYTES));
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            ptx::umma_f16(d_tmem, adesc + 2 * kk, bdesc + 2 * kk, idesc, (kb > kb0) || (kk > 0));
          ptx::umma_commit(&empty[stage]);
          if (++stage == L::STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        ptx::umma_commit(&tfull[acc]);
      }
      if (!ok) {
        *abort_flag = 1;
        set_status(p.status, MOE_ERR_TIMEOUT);
      }
      // every MMA issued must finish before TMEM is released
      ptx::umma_commit(drain);
      ptx::mbar_wait(drain, 0, reinterpret_cast<volatile int*>(s_bad), p.wait_ns);
    }
  } else {
    // -------------------------------------------------------------- epilogue
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
    int it = 0;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x, ++it) {
      const int acc = it & 1;
      const uint32_t use = static_cast<uint32_t>(it >> 1);
      const TileCoord tc = decode_tile(s_tile, s_off, G, nt, tile);
      const int g = tc.g, nb = tc.nb, m_g = tc.m_g;
      // the lane's row: q * 32 + lane, or after a 64-row MMA q * 16 + lane for lanes 0..15
      const bool half = m_g - tc.mb * BM <= 64;
      const int row_t = half ? (lane < 16 ? q * 16 + lane : BM) : q * 32 + lane;
      const int r_in = tc.mb * BM + row_t;
      const bool valid = r_in < m_g;
      const size_t grow = static_cast<size_t>(s_off[g] + r_in);
      if (p.stall && it == 0 && !ptx::mbar_wait_warp(never, 0, abort_flag, p.wait_ns)) {
        *abort_flag = 1;
        set_status(p.status, MOE_ERR_TIMEOUT);
        break;
      }
      if (!ptx::mbar_wait_warp(&tfull[acc], use & 1, abort_flag, p.wait_ns)) {
        *abort_flag = 1;
        set_status(p.status, MOE_ERR_TIMEOUT);
        break;
      }
      ptx::tc_fence_after();
      const uint32_t tacc = lane_base + acc * MMA_N;
      if constexpr (OUT == 0) {
        // bf16 output in 64-column boxes.  A warp whose 32 rows all belong to
        // the group stages each box (128-byte swizzled) in its buffer and
        // writes it with a bulk tensor store; a slice crossing the group's
        // end stores its valid rows directly.
        const int r0 = tc.mb * BM + q * 32;
        // (the gated output, half as wide, keeps the operand stage instead: direct stores)
        const bool slice_full = L::OUT_WARP > 0 && !half && r0 + 32 <= m_g;
        uint8_t* s_out = smem + L::OUTB + (warp - 2) * L::OUT_WARP;
#pragma unroll 1
        for (int b = 0; b < OUT_COLS / 64; ++b) {
          uint32_t pk[32];
#pragma unroll
          for (int h2 = 0; h2 < 2; ++h2) {
            const int c = 64 * b + 32 * h2;
            if constexpr (EPI == 1) {
              uint32_t gv[32], uv[32];
              ptx::tmem_ld_32x32b_x32(tacc + c, gv);
              ptx::tmem_ld_32x32b_x32(tacc + OUT_COLS + c, uv);
              ptx::tmem_ld_wait();
#pragma unroll
              for (int i = 0; i < 16; ++i) {
                const float h0 = silu(__uint_as_float(gv[2 * i])) * __uint_as_float(uv[2 * i]);
                const float h1 = silu(__uint_as_float(gv[2 * i + 1])) * __uint_as_float(uv[2 * i + 1]);
                const __nv_bfloat162 hb = __floats2bfloat162_rn(h0, h1);
                pk[16 * h2 + i] = *reinterpret_cast<const uint32_t*>(&hb);
              }
            } else {
              uint32_t v[32];
              ptx::tmem_ld_32x32b_x32(tacc + c, v);
              ptx::tmem_ld_wait();
#pragma unroll
              for (int i = 0; i < 16; ++i) {
                const __nv_bfloat162 hb =
                    __floats2bfloat162_rn(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
                pk[16 * h2 + i] = *reinterpret_cast<const uint32_t*>(&hb);
              }
            }
          }
          if (slice_full) {
            constexpr int kBufs = L::OUT_WARP / 4096 > 0 ? L::OUT_WARP / 4096 : 1;
            uint8_t* buf = s_out + (b % kBufs) * 4096;
            if (lane == 0) {  // the store that used this buffer has read it
              if constexpr (kBufs > 1)
                ptx::bulk_wait_read_allow1();
              else
                ptx::bulk_wait_read_all();
            }
            __syncwarp();
#pragma unroll
            for (int c = 0; c < 8; ++c)
              *reinterpret_cast<uint4*>(buf + lane * 128 + ((c ^ (lane & 7)) << 4)) =
                  make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
            ptx::fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              ptx::tma_store_2d(&tmC, buf, nb * OUT_COLS + 64 * b, s_off[g] + r0);
              ptx::bulk_commit_group();
            }
          } else if (valid) {
            uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.C) + grow * p.N + nb * OUT_COLS +
                                                  64 * b);
#pragma unroll
            for (int c = 0; c < 8; ++c) dst[c] = make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
          }
        }
      } else {
        // fp32 output (router logits, split-K partial products): direct stores
#pragma unroll 1
        for (int c = 0; c < OUT_COLS; c += 32) {
          uint32_t v[32];
          ptx::tmem_ld_32x32b_x32(tacc + c, v);
          ptx::tmem_ld_wait();
          if (valid) {
            float* C = static_cast<float*>(p.C) + tc.ks * p.split_stride + grow * p.N + nb * OUT_COLS + c;
            uint4* dst = reinterpret_cast<uint4*>(C);
#pragma unroll
            for (int i = 0; i < 8; ++i) dst[i] = make_uint4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
          }
        }
      }
      ptx::tc_fence_before();
      ptx::mbar_arrive(&tempty[acc]);
    }
    if (L::OUT_WARP > 0 && lane == 0) ptx::bulk_wait_all();  // this warp's stores are complete before the CTA exits
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem_base, L::TMEM_COLS);
  }
}

// ------------------------------------------------------------------ swap-AB bf16 kernel (small groups)
// Decode-shaped problems give each expert a handful of tokens.  Here the
// weights are the 128-row MMA operand and the tokens the narrow one:
// D[128 weight rows, NT tokens] = W_tile . X_tile^T, so a tile streams 16 KB
// of weights and only NT x 128 B of activations per k-step (the
// activation-major kernel would stream a 128-row activation tile, mostly rows
// of other experts, as many bytes as the weights).  With the SiLU gate the
// 128 weight rows are four 32-row chunks [16 gate rows; the 16 matching up
// rows], so lane l < 16 of a warp holds gate(col l) and lane l + 16 holds
// up(col l): one shuffle pairs them.  Each thread owns one output column and
// writes it for the tile's tokens.
constexpr int kSwapNT = 32;     // tokens per tile (MMA N)
constexpr int kSwapStages = 8;  // (16 KB weights + 4 KB tokens) per stage
constexpr int kSwapSmem = 1024 + kSwapStages * (16384 + kSwapNT * 128) + 512 + 2 * (kMaxGroups + 2) * 4;

template <int EPI>
__global__ void __launch_bounds__(kThreads, 1)
    gg_bf16_swap_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                        const __grid_constant__ CUtensorMap tmWx, const Params p) {
  pdl_wait();  // the preceding kernel on the stream is complete and visible
  pdl_launch_dependents();
  constexpr int NT = kSwapNT;
  constexpr int W_BYTES = 128 * 128;
  constexpr int X_BYTES = NT * 128;
  constexpr int STAGES = kSwapStages;
  constexpr int COLS = EPI ? 64 : 128;  // output columns per tile
  constexpr int TMEM_COLS = 2 * NT;
  constexpr uint32_t IDESC = ptx::make_idesc(128, NT, 1);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sW = smem;
  uint8_t* sX = smem + STAGES * W_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(sX + STAGES * X_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* s_bad = reinterpret_cast<int*>(tmem_slot + 2);
  int* s_off = reinterpret_cast<int*>(smem + STAGES * (W_BYTES + X_BYTES) + 512);
  int* s_tile = s_off + kMaxGroups + 2;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = p.G_total;
  const int nt = p.N / COLS;

  if (warp == 0) {
    for (int g = lane; g <= G; g += 32) s_off[g] = p.offsets ? p.offsets[g] : (g == 0 ? 0 : p.rows);
    __syncwarp();
    const int per = (G + 31) / 32;
    const int g0 = min(G, lane * per), g1 = min(G, g0 + per);
    int bad = 0, mine = 0;
    for (int g = g0; g < g1; ++g) {
      const int m = s_off[g + 1] - s_off[g];
      if (m < 0) bad = 1;
      mine += (max(m, 0) + NT - 1) / NT * nt;
    }
    int incl = mine;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    int run = incl - mine;
    for (int g = g0; g < g1; ++g) {
      s_tile[g] = run;
      run += (max(s_off[g + 1] - s_off[g], 0) + NT - 1) / NT * nt;
    }
    if (lane == 31) s_tile[G] = incl;
    if (lane == 0 && (s_off[0] != 0 || s_off[G] > p.rows)) bad = 1;
    bad = __any_sync(0xffffffffu, bad);
    if (lane == 0) {
      *s_bad = bad;
      *abort_flag = 0;
      if (bad && blockIdx.x == 0) set_status(p.status, MOE_ERR_BAD_OFFSETS);
    }
  }
  __syncthreads();
  if (*s_bad) return;

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < STAGES; ++s) {
      ptx::mbar_init(&full[s], 1);
      ptx::mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      ptx::mbar_init(&tfull[a], 1);
      ptx::mbar_init(&tempty[a], 128);
    }
    ptx::mbar_init(drain, 1);
    ptx::fence_mbar_init();
    ptx::prefetch_tmap(&tmX);
    ptx::prefetch_tmap(&tmW);
    ptx::prefetch_tmap(&tmWx);
  }
  if (warp == 1) {
    ptx::tmem_alloc(tmem_slot, TMEM_COLS);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int total = s_tile[G];
  const int nk = p.K / 64;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ producer
      uint32_t stage = 0, phase = 0, issued = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
        const int g = find_group(s_tile, G, tile);
        const int m_g = s_off[g + 1] - s_off[g];
        const int mt = (m_g + NT - 1) / NT;
        const int tl = tile - s_tile[g];
        const int nb = tl / mt, tb = tl % mt;
        const int x_row = s_off[g] + tb * NT;
        const bool extra = g >= p.G_main;
        const CUtensorMap* mW = extra ? &tmWx : &tmW;
        const int gb = extra ? 0 : g;
        for (int kb = 0; kb < nk; ++kb) {
          if (!ptx::mbar_wait(&empty[stage], phase ^ 1, abort_flag, kWaitLimitNs)) {
            ok = false;
            break;
          }
          ptx::mbar_arrive_expect_tx(&full[stage], W_BYTES + X_BYTES);
          uint8_t* w = sW + stage * W_BYTES;
          if (EPI) {
            // one 4-D box {64 k, 16 rows, gate/up, 4 chunks}: chunk c lands as
            // [16 gate rows; the 16 up rows of the same output columns]
            ptx::tma_load_4d(w, mW, &full[stage], kb * 64, 0, 0, (gb * 2 * p.N + nb * 64) / 16);
          } else {
            ptx::tma_load_2d(w, mW, &full[stage], kb * 64, gb * p.N + nb * 128);
          }
          ptx::tma_load_2d(sX + stage * X_BYTES, &tmX, &full[stage], kb * 64, x_row);
          ++issued;
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      if (!ok) {
        *abort_flag = 1;
        set_status(p.status, MOE_ERR_TIMEOUT);
        const uint32_t pending = issued < static_cast<uint32_t>(STAGES) ? issued : STAGES;
        uint32_t s = stage, ph = phase;
        for (uint32_t i = 0; i < pending; ++i) {
          if (s == 0) {
            s = STAGES - 1;
            ph ^= 1;
          } else {
            --s;
          }
          ptx::mbar_wait(&full[s], ph, reinterpret_cast<volatile int*>(s_bad), kWaitLimitNs);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------------ MMA issuer
      uint32_t stage = 0, phase = 0;
      bool ok = true;
      int it = 0;
      for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x, ++it) {
        const int acc = it & 1;
        const uint32_t use = static_cast<uint32_t>(it >> 1);
        if (!ptx::mbar_wait(&tempty[acc], (use & 1) ^ 1, abort_flag, kWaitLimitNs)) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * NT;
        for (int kb = 0; kb < nk; ++kb) {
          if (!ptx::mbar_wait(&full[stage], phase, abort_flag, kWaitLimitNs)) {
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          const uint64_t adesc = ptx::sw128_kmajor_desc(ptx::smem_u32(sW + stage * W_BYTES));
          const uint64_t bdesc = ptx::sw128_kmajor_desc(ptx::smem_u32(sX + stage * X_BYTES));
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            ptx::umma_f16(d_tmem, adesc + 2 * kk, bdesc + 2 * kk, IDESC, (kb | kk) != 0);
          ptx::umma_commit(&empty[stage]);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        ptx::umma_commit(&tfull[acc]);
      }
      if (!ok) {
        *abort_flag = 1;
        set_status(p.status, MOE_ERR_TIMEOUT);
      }
      ptx::umma_commit(drain);
      ptx::mbar_wait(drain, 0, reinterpret_cast<volatile int*>(s_bad), kWaitLimitNs);
    }
  } else {
    // -------------------------------------------------------------- epilogue
    const int q = warp & 3;  // TMEM lane quarter = weight rows 32q .. 32q+31
    const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
    int it = 0;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x, ++it) {
      const int acc = it & 1;
      const uint32_t use = static_cast<uint32_t>(it >> 1);
      const int g = find_group(s_tile, G, tile);
      const int m_g = s_off[g + 1] - s_off[g];
      const int mt = (m_g + NT - 1) / NT;
      const int tl = tile - s_tile[g];
      const int nb = tl / mt, tb = tl % mt;
      const int ntok = min(NT, m_g - tb * NT);  // valid tokens of this tile
      const size_t row0 = static_cast<size_t>(s_off[g] + tb * NT);
      if (!ptx::mbar_wait_warp(&tfull[acc], use & 1, abort_flag, kWaitLimitNs)) {
        *abort_flag = 1;
        set_status(p.status, MOE_ERR_TIMEOUT);
        break;
      }
      ptx::tc_fence_after();
      uint32_t v[32];
      ptx::tmem_ld_32x32b_x32(lane_base + acc * NT, v);
      ptx::tmem_ld_wait();
      ptx::tc_fence_before();
      ptx::mbar_arrive(&tempty[acc]);  // the values are in registers: release the accumulator early
      __nv_bfloat16* C = static_cast<__nv_bfloat16*>(p.C);
      if constexpr (EPI == 1) {
        // lanes 0..15: gate of column c; lanes 16..31: up of the same column
        const int col = nb * 64 + q * 16 + (lane & 15);
#pragma unroll
        for (int t = 0; t < NT; ++t) {
          const float mine = __uint_as_float(v[t]);
          const float up = __shfl_xor_sync(0xffffffffu, mine, 16);
          if (lane < 16 && t < ntok) {
            const float hval = silu(mine) * up;
            C[(row0 + t) * p.N + col] = __float2bfloat16_rn(hval);
          }
        }
      } else {
        const int col = nb * 128 + q * 32 + lane;
#pragma unroll
        for (int t = 0; t < NT; ++t)
          if (t < ntok) C[(row0 + t) * p.N + col] = __float2bfloat16_rn(__uint_as_float(v[t]));
      }
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

// ------------------------------------------------------------------ CTA-pair bf16 kernel
// For large groups (the compute-bound Mixtral-shaped layer) two SMs of a
// cluster share one 256-row tile: each CTA stages its own 128 rows of A and
// one half of the 256 B columns (with the SiLU gate: CTA 0 the gate rows, CTA 1
// the up rows), and the pair's leader issues tcgen05.mma.cta_group::2
// 256 x 256 x 16, which reads both CTAs' shared memory and accumulates each
// CTA's 128 rows in its own TMEM.  Per FLOP each SM now moves two thirds of
// the operand bytes of the single-CTA kernel.  Barriers: both CTAs' TMA loads
// count their bytes on the leader's full[stage]; the leader's commits arrive
// on empty[stage] / tfull[acc] in both CTAs; both epilogues release an
// accumulator on the leader's tempty[acc].
constexpr int kPairStages = 6;
constexpr int kPairSmem = 1024 + kPairStages * 32768 + 512 + 2 * (kMaxGroups + 2) * 4;

template <int EPI, int OUT>
__global__ void __launch_bounds__(kThreads, 1)
    gg_bf16_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                        const __grid_constant__ CUtensorMap tmBx, const __grid_constant__ CUtensorMap tmB64,
                        const __grid_constant__ CUtensorMap tmBx64, const __grid_constant__ CUtensorMap tmA64,
                        const Params p) {
  pdl_wait();  // the preceding kernel on the stream is complete and visible
  pdl_launch_dependents();
  constexpr int MMA_N = 256;
  constexpr int BM2 = 256;
  constexpr int A_BYTES = 128 * 128;
  constexpr int B_BYTES = 128 * 128;
  constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  constexpr int STAGES = kPairStages;
  constexpr int TMEM_COLS = 512;
  constexpr int OUT_COLS = EPI ? 128 : 256;
  constexpr uint32_t IDESC = ptx::make_idesc(BM2, MMA_N, 1);
  constexpr uint32_t IDESC_HALF = ptx::make_idesc(128, MMA_N, 1);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * A_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(sB + STAGES * B_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* s_bad = reinterpret_cast<int*>(tmem_slot + 2);
  int* s_off = reinterpret_cast<int*>(smem + STAGES * STAGE_BYTES + 512);
  int* s_tile = s_off + kMaxGroups + 2;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = ptx::cluster_ctarank();
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const int G = p.G_total;
  const int nt = p.N / OUT_COLS;

  if (warp == 0) {
    for (int g = lane; g <= G; g += 32) s_off[g] = p.offsets ? p.offsets[g] : (g == 0 ? 0 : p.rows);
    __syncwarp();
    const int per = (G + 31) / 32;
    const int g0 = min(G, lane * per), g1 = min(G, g0 + per);
    int bad = 0, mine = 0;
    for (int g = g0; g < g1; ++g) {
      const int m = s_off[g + 1] - s_off[g];
      if (m < 0) bad = 1;
      mine += (max(m, 0) + BM2 - 1) / BM2 * nt;
    }
    int incl = mine;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    int run = incl - mine;
    for (int g = g0; g < g1; ++g) {
      s_tile[g] = run;
      run += (max(s_off[g + 1] - s_off[g], 0) + BM2 - 1) / BM2 * nt;
    }
    if (lane == 31) s_tile[G] = incl;
    if (lane == 0 && (s_off[0] != 0 || s_off[G] > p.rows)) bad = 1;
    bad = __any_sync(0xffffffffu, bad);
    if (lane == 0) {
      *s_bad = bad;
      *abort_flag = 0;
      if (bad && blockIdx.x == 0) set_status(p.status, MOE_ERR_BAD_OFFSETS);
    }
  }
  __syncthreads();
  if (*s_bad) return;  // both CTAs of the pair read the same offsets: uniform

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < STAGES; ++s) {
      ptx::mbar_init(&full[s], 1);
      ptx::mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      ptx::mbar_init(&tfull[a], 1);
      ptx::mbar_init(&tempty[a], 256);
    }
    ptx::mbar_init(drain, 1);
    ptx::fence_mbar_init();
    ptx::prefetch_tmap(&tmA);
    ptx::prefetch_tmap(&tmB);
    ptx::prefetch_tmap(&tmBx);
  }
  if (warp == 1) {
    ptx::tmem_alloc_pair(tmem_slot, TMEM_COLS);
    ptx::tmem_relinquish_pair();
  }
  ptx::tc_fence_before();
  ptx::cluster_sync();  // barrier inits of both CTAs visible to the pair
  ptx::tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int total = s_tile[G];
  const int nk = p.K / 64;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ producer (both CTAs)
      uint32_t stage = 0, phase = 0;
      bool ok = true;
      for (int tile = pair; tile < total && ok; tile += npairs) {
        const int g = find_group(s_tile, G, tile);
        const int m_g = s_off[g + 1] - s_off[g];
        const int mt = (m_g + BM2 - 1) / BM2;
        const int tl = tile - s_tile[g];
        const int nb = tl / mt, mb = tl % mt;
        // a group's last tile with at most 128 rows runs as a 128-row pair MMA (64 rows per CTA)
        const bool half = m_g - mb * BM2 <= 128;
        const int a_row = s_off[g] + mb * BM2 + static_cast<int>(rank) * (half ? 64 : 128);
        const bool extra = g >= p.G_main;
        const CUtensorMap* mB = extra ? &tmBx : &tmB;
        const CUtensorMap* mB64 = extra ? &tmBx64 : &tmB64;
        const int gb = extra ? 0 : g;
        const int brow = EPI ? gb * 2 * p.N + static_cast<int>(rank) * p.N + nb * 128
                             : gb * p.N + nb * 256 + static_cast<int>(rank) * 128;
        // gated half tile: this CTA's 128 B rows are 64 gate rows and the 64 matching up rows, so
        // that each accumulator lane holds a row's gate and up columns side by side
        const int hrow = gb * 2 * p.N + nb * 128 + static_cast<int>(rank) * 64;
        for (int kb = 0; kb < nk; ++kb) {
          if (!ptx::mbar_wait(&empty[stage], phase ^ 1, abort_flag, kWaitLimitNs)) {
            ok = false;
            break;
          }
          const uint32_t fb = ptx::map_to_rank(ptx::smem_u32(&full[stage]), 0);
          // a half tile's MMA reads 64 A rows per CTA: load just those (64-row box)
          if (leader) ptx::mbar_arrive_expect_tx(&full[stage], half ? 2 * (A_BYTES / 2 + B_BYTES) : 2 * STAGE_BYTES);
          ptx::tma_load_2d_pair(sA + stage * A_BYTES, half ? &tmA64 : &tmA, fb, kb * 64, a_row);
          if (EPI && half) {
            ptx::tma_load_2d_pair(sB + stage * B_BYTES, mB64, fb, kb * 64, hrow);
            ptx::tma_load_2d_pair(sB + stage * B_BYTES + 64 * 128, mB64, fb, kb * 64, hrow + p.N);
          } else {
            ptx::tma_load_2d_pair(sB + stage * B_BYTES, mB, fb, kb * 64, brow);
          }
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      if (!ok) {
        *abort_flag = 1;
        set_status(p.status, MOE_ERR_TIMEOUT);
        for (int i = 0; i < 20; ++i) __nanosleep(50000);  // let copies in flight land (~1 ms)
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      // ------------------------------------------------------------ MMA issuer (leader CTA)
      uint32_t stage = 0, phase = 0;
      bool ok = true;
      int it = 0;
      for (int tile = pair; tile < total && ok; tile += npairs, ++it) {
        const int acc = it & 1;
        const uint32_t use = static_cast<uint32_t>(it >> 1);
        if (!ptx::mbar_wait(&tempty[acc], (use & 1) ^ 1, abort_flag, kWaitLimitNs)) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * MMA_N;
        const int g = find_group(s_tile, G, tile);
        const int m_g = s_off[g + 1] - s_off[g];
        const int mt = (m_g + BM2 - 1) / BM2;
        const uint32_t idesc = m_g - ((tile - s_tile[g]) % mt) * BM2 <= 128 ? IDESC_HALF : IDESC;
        for (int kb = 0; kb < nk; ++kb) {
          if (!ptx::mbar_wait(&full[stage], phase, abort_flag, kWaitLimitNs)) {
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          const uint64_t adesc = ptx::sw128_kmajor_desc(ptx::smem_u32(sA + stage * A_BYTES));
          const uint64_t bdesc = ptx::sw128_kmajor_desc(ptx::smem_u32(sB + stage * B_BYTES));
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            ptx::umma_f16_pair(d_tmem, adesc + 2 * kk, bdesc + 2 * kk, idesc, (kb | kk) != 0);
          ptx::umma_commit_pair_both(&empty[stage]);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        ptx::umma_commit_pair_both(&tfull[acc]);
      }
      if (!ok) {
        *abort_flag = 1;
        set_status(p.status, MOE_ERR_TIMEOUT);
      }
      ptx::umma_commit_pair_both(drain);
      ptx::mbar_wait(drain, 0, reinterpret_cast<volatile int*>(s_bad), kWaitLimitNs);
    }
  } else {
    // -------------------------------------------------------------- epilogue (both CTAs)
    const int q = warp & 3;
    const int row_t = q * 32 + lane;
    const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
    int it = 0;
    for (int tile = pair; tile < total; tile += npairs, ++it) {
      const int acc = it & 1;
      const uint32_t use = static_cast<uint32_t>(it >> 1);
      const int g = find_group(s_tile, G, tile);
      const int m_g = s_off[g + 1] - s_off[g];
      const int mt = (m_g + BM2 - 1) / BM2;
      const int tl = tile - s_tile[g];
      const int nb = tl / mt, mb = tl % mt;
      // Half tile (128-row pair MMA): each CTA holds 64 rows; lanes 0-63 carry the first 128
      // columns of the MMA's 256 and lanes 64-127 the last 128, both at accumulator columns 0-127.
      const bool half = m_g - mb * BM2 <= 128;
      const int lrow = half ? (row_t & 63) : row_t;
      const int hsel = half ? (row_t >> 6) : 0;
      const int r_in = mb * BM2 + static_cast<int>(rank) * (half ? 64 : 128) + lrow;
      const bool valid = r_in < m_g;
      const size_t grow = static_cast<size_t>(s_off[g] + r_in);
      if (!ptx::mbar_wait_warp(&tfull[acc], use & 1, abort_flag, kWaitLimitNs)) {
        *abort_flag = 1;
        set_status(p.status, MOE_ERR_TIMEOUT);
        break;
      }
      ptx::tc_fence_after();
      const uint32_t tacc = lane_base + acc * MMA_N;
      // output columns of this lane: in a half tile each lane has half of them (with the gate:
      // gate at accumulator columns [0, 64), up at [64, 128)), in a full tile all
      const int ncols = half ? OUT_COLS / 2 : OUT_COLS;
      const int col0 = nb * OUT_COLS + hsel * ncols;
      if constexpr (EPI == 1) {
        __nv_bfloat16* C = static_cast<__nv_bfloat16*>(p.C) + grow * p.N + col0;
#pragma unroll 1
        for (int c = 0; c < ncols; c += 32) {
          uint32_t gv[32], uv[32];
          ptx::tmem_ld_32x32b_x32(tacc + c, gv);
          ptx::tmem_ld_32x32b_x32(tacc + ncols + c, uv);
          ptx::tmem_ld_wait();
          if (valid) {
            uint32_t packed[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const float g0 = __uint_as_float(gv[2 * i]), g1 = __uint_as_float(gv[2 * i + 1]);
              const float h0 = silu(g0) * __uint_as_float(uv[2 * i]);
              const float h1 = silu(g1) * __uint_as_float(uv[2 * i + 1]);
              const __nv_bfloat162 hb = __floats2bfloat162_rn(h0, h1);
              packed[i] = *reinterpret_cast<const uint32_t*>(&hb);
            }
            uint4* dst = reinterpret_cast<uint4*>(C + c);
#pragma unroll
            for (int v = 0; v < 4; ++v)
              dst[v] = make_uint4(packed[4 * v], packed[4 * v + 1], packed[4 * v + 2], packed[4 * v + 3]);
          }
        }
      } else {
#pragma unroll 1
        for (int c = 0; c < ncols; c += 32) {
          uint32_t v[32];
          ptx::tmem_ld_32x32b_x32(tacc + c, v);
          ptx::tmem_ld_wait();
          if (valid) {
            if constexpr (OUT == 1) {
              uint4* dst = reinterpret_cast<uint4*>(static_cast<float*>(p.C) + grow * p.N + col0 + c);
#pragma unroll
              for (int i = 0; i < 8; ++i) dst[i] = make_uint4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
            } else {
              uint32_t packed[16];
#pragma unroll
              for (int i = 0; i < 16; ++i) {
                const __nv_bfloat162 hb =
                    __floats2bfloat162_rn(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
                packed[i] = *reinterpret_cast<const uint32_t*>(&hb);
              }
              uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.C) + grow * p.N + col0 + c);
#pragma unroll
              for (int i = 0; i < 4; ++i)
                dst[i] = make_uint4(packed[4 * i], packed[4 * i + 1], packed[4 * i + 2], packed[4 * i + 3]);
            }
          }
        }
      }
      ptx::tc_fence_before();
      ptx::mbar_arrive_cluster(ptx::map_to_rank(ptx::smem_u32(&tempty[acc]), 0));
    }
  }

  ptx::tc_fence_before();
  ptx::cluster_sync();  // neither CTA leaves while the pair still uses its memory
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc_pair(tmem_base, TMEM_COLS);
  }
}

// ------------------------------------------------------------------ FP8 (E4M3) kernel
// Same persistent structure; operands are E4M3 with fp32 scales that vary
// along K ("MegaMoE ..." §2.3 / §5.1: 1x128 per token, 128x128 per weight
// block), so one K block of 128 is one pipeline stage and the scales are
// applied per K block ("promotion"): the MMA warp writes each block's partial
// product A_kb B_kb^T into one of two TMEM buffers (kind::f8f6f4, 128 x 256
// x 32 per instruction) and sixteen epilogue warps fold it into fp32
// registers,
//     acc[m][n] += partial[m][n] * sa[m, kb] * sb[n/128, kb],
// while the MMA fills the other buffer.  Epilogue thread = one row and a
// quarter c of the tile's 256 columns (64 accumulators, so four warps share
// each TMEM lane quarter and hide each other's load latency): with the SiLU
// gate, quarter c owns gate columns [32c, 32c+32) and the matching up
// columns, so silu(g)*u stays in-thread; the E4M3 output (per row per 128
// columns) exchanges the four quarters' amax through shared memory under an
// mbarrier.
constexpr int kThreadsF8 = 576;  // producer, MMA issuer, 16 epilogue warps

// Shared memory of the FP8 kernel, as offsets from the 1024-byte aligned base.
// Without the gate, each epilogue warp stages its 32 output rows (32 x 128 B
// of bf16) for one bulk tensor store, which takes the room of one operand
// stage; the gated kernels store their narrower rows directly.
template <int EPI, int OUT>
struct F8Smem {
  static constexpr int A_BYTES = BM * 128;
  static constexpr int B_BYTES = 256 * 128;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr bool STAGE_OUT = EPI == 0;
  static constexpr int OUT_WARP = STAGE_OUT ? 4096 : 0;
  static constexpr int STAGES = STAGE_OUT ? 3 : 4;
  static constexpr int TMEM_COLS = 512;
  static constexpr int OUTB = STAGES * STAGE_BYTES;              // output staging
  static constexpr int BARS = OUTB + 16 * OUT_WARP;              // barriers and flags
  static constexpr int TABLES = BARS + 512;                      // group offsets and tile prefix
  static constexpr int AMAX = TABLES + 2 * (kMaxGroups + 2) * 4;  // [2 parity][4 quarters][128 rows]
  static constexpr int SMEM = AMAX + 2 * 4 * 128 * 4 + 1024;     // + alignment slack
  static_assert(SMEM <= 227 * 1024, "shared memory budget");
};

template <int EPI, int OUT>  // EPI 1: SiLU gate (OUT 0 bf16 / 2 e4m3); EPI 0: OUT 0 bf16
__global__ void __launch_bounds__(kThreadsF8, 1)
    gg_fp8_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                  const __grid_constant__ CUtensorMap tmBx, const __grid_constant__ CUtensorMap tmC,
                  const Params p) {
  pdl_wait();  // the preceding kernel on the stream is complete and visible
  pdl_launch_dependents();
  constexpr int MMA_N = 256;
  using L = F8Smem<EPI, OUT>;
  constexpr int OUT_COLS = EPI ? 128 : 256;
  constexpr uint32_t IDESC = ptx::make_idesc(BM, MMA_N, 0);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + L::STAGES * L::A_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::BARS);
  uint64_t* empty = full + L::STAGES;
  uint64_t* pfull = empty + L::STAGES;
  uint64_t* pempty = pfull + 2;
  uint64_t* xchg = pempty + 2;
  uint64_t* drain = xchg + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* s_bad = reinterpret_cast<int*>(tmem_slot + 2);
  int* s_off = reinterpret_cast<int*>(smem + L::TABLES);
  int* s_tile = s_off + kMaxGroups + 2;
  float* s_amax = reinterpret_cast<float*>(smem + L::AMAX);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = p.G_total;
  const int nt = p.N / OUT_COLS;

  if (warp == 0) {
    for (int g = lane; g <= G; g += 32) s_off[g] = p.offsets ? p.offsets[g] : (g == 0 ? 0 : p.rows);
    __syncwarp();
    const int per = (G + 31) / 32;
    const int g0 = min(G, lane * per), g1 = min(G, g0 + per);
    int bad = 0, mine = 0;
    for (int g = g0; g < g1; ++g) {
      const int m = s_off[g + 1] - s_off[g];
      if (m < 0) bad = 1;
      mine += (max(m, 0) + BM - 1) / BM * nt;
    }
    int incl = mine;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    int run = incl - mine;
    for (int g = g0; g < g1; ++g) {
      s_tile[g] = run;
      run += (max(s_off[g + 1] - s_off[g], 0) + BM - 1) / BM * nt;
    }
    if (lane == 31) s_tile[G] = incl;
    if (lane == 0 && (s_off[0] != 0 || s_off[G] > p.rows)) bad = 1;
    bad = __any_sync(0xffffffffu, bad);
    if (lane == 0) {
      *s_bad = bad;
      *abort_flag = 0;
      if (bad && blockIdx.x == 0) set_status(p.status, MOE_ERR_BAD_OFFSETS);
    }
  }
  __syncthreads();
  if (*s_bad) return;

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < L::STAGES; ++s) {
      ptx::mbar_init(&full[s], 1);
      ptx::mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      ptx::mbar_init(&pfull[a], 1);
      ptx::mbar_init(&pempty[a], 16);  // one arrival per epilogue warp
    }
    ptx::mbar_init(xchg, 16);
    ptx::mbar_init(drain, 1);
    ptx::fence_mbar_init();
    ptx::prefetch_tmap(&tmA);
    ptx::prefetch_tmap(&tmB);
    ptx::prefetch_tmap(&tmBx);
  }
  if (warp == 1) {
    ptx::tmem_alloc(tmem_slot, L::TMEM_COLS);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int total = s_tile[G];
  const int nk = p.K / 128;

  if (warp == 0 && p.a_rows) {
    // -------------------------------------------------------------- producer, gathered A
    // lane l brings A rows 4l..4l+3 of the tile (one tile::gather4 each k-step);
    // lane 0 also waits for the stage and loads B
    uint32_t stage = 0, phase = 0, issued = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
      const TileCoord tc = decode_tile(s_tile, s_off, G, nt, tile);
      const int g = tc.g, nb = tc.nb;
      int tok[4];
      gather_rows(p, s_off[g] + tc.mb * BM, lane, tok);
      const bool extra = g >= p.G_main;
      const CUtensorMap* mB = extra ? &tmBx : &tmB;
      const int gb = extra ? 0 : g;
      for (int kb = 0; kb < nk; ++kb) {
        int go = 1;
        if (lane == 0) {
          go = ptx::mbar_wait(&empty[stage], phase ^ 1, abort_flag, kWaitLimitNs);
          if (go) ptx::mbar_arrive_expect_tx(&full[stage], L::A_BYTES + L::B_BYTES);
        }
        if (!__shfl_sync(0xffffffffu, go, 0)) {
          ok = false;
          break;
        }
        ptx::tma_gather4(sA + stage * L::A_BYTES + lane * 512, &tmA, &full[stage], kb * 128, tok[0], tok[1], tok[2],
                         tok[3]);
        if (lane == 0) {
          if (EPI) {
            const int brow = gb * 2 * p.N + nb * 128;
            ptx::tma_load_2d(sB + stage * L::B_BYTES, mB, &full[stage], kb * 128, brow);
            ptx::tma_load_2d(sB + stage * L::B_BYTES + 128 * 128, mB, &full[stage], kb * 128, brow + p.N);
          } else {
            ptx::tma_load_2d(sB + stage * L::B_BYTES, mB, &full[stage], kb * 128, gb * p.N + nb * 256);
          }
        }
        ++issued;
        if (++stage == L::STAGES) {
          stage = 0;
          phase ^= 1;
        }
      }
    }
    if (!ok && lane == 0) {
      *abort_flag = 1;
      set_status(p.status, MOE_ERR_TIMEOUT);
      const uint32_t pending = issued < static_cast<uint32_t>(L::STAGES) ? issued : L::STAGES;
      uint32_t s2 = stage, ph = phase;
      for (uint32_t i = 0; i < pending; ++i) {
        if (s2 == 0) {
          s2 = L::STAGES - 1;
          ph ^= 1;
        } else {
          --s2;
        }
        ptx::mbar_wait(&full[s2], ph, reinterpret_cast<volatile int*>(s_bad), kWaitLimitNs);
      }
    }
  } else if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ producer
      uint32_t stage = 0, phase = 0, issued = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
        const TileCoord tc = decode_tile(s_tile, s_off, G, nt, tile);
        const int g = tc.g, nb = tc.nb;
        const int a_row = s_off[g] + tc.mb * BM;
        const bool extra = g >= p.G_main;
        const CUtensorMap* mB = extra ? &tmBx : &tmB;
        const int gb = extra ? 0 : g;
        for (int kb = 0; kb < nk; ++kb) {
          if (!ptx::mbar_wait(&empty[stage], phase ^ 1, abort_flag, kWaitLimitNs)) {
            ok = false;
            break;
          }
          ptx::mbar_arrive_expect_tx(&full[stage], L::STAGE_BYTES);
          ptx::tma_load_2d(sA + stage * L::A_BYTES, &tmA, &full[stage], kb * 128, a_row);
          if (EPI) {
            const int brow = gb * 2 * p.N + nb * 128;
            ptx::tma_load_2d(sB + stage * L::B_BYTES, mB, &full[stage], kb * 128, brow);
            ptx::tma_load_2d(sB + stage * L::B_BYTES + 128 * 128, mB, &full[stage], kb * 128, brow + p.N);
          } else {
            ptx::tma_load_2d(sB + stage * L::B_BYTES, mB, &full[stage], kb * 128, gb * p.N + nb * 256);
          }
          ++issued;
          if (++stage == L::STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      if (!ok) {
        *abort_flag = 1;
        set_status(p.status, MOE_ERR_TIMEOUT);
        const uint32_t pending = issued < static_cast<uint32_t>(L::STAGES) ? issued : L::STAGES;
        uint32_t s2 = stage, ph = phase;
        for (uint32_t i = 0; i < pending; ++i) {
          if (s2 == 0) {
            s2 = L::STAGES - 1;
            ph ^= 1;
          } else {
            --s2;
          }
          ptx::mbar_wait(&full[s2], ph, reinterpret_cast<volatile int*>(s_bad), kWaitLimitNs);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------------ MMA issuer
      uint32_t stage = 0, phase = 0;
      uint32_t pb = 0, puse = 0;  // partial buffer and how many times the pair was cycled
      bool ok = true;
      for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
        for (int kb = 0; kb < nk; ++kb) {
          if (!ptx::mbar_wait(&pempty[pb], (puse & 1) ^ 1, abort_flag, kWaitLimitNs) ||
              !ptx::mbar_wait(&full[stage], phase, abort_flag, kWaitLimitNs)) {
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          const uint32_t d_tmem = tmem_base + pb * MMA_N;
          const uint64_t adesc = ptx::sw128_kmajor_desc(ptx::smem_u32(sA + stage * L::A_BYTES));
          const uint64_t bdesc = ptx::sw128_kmajor_desc(ptx::smem_u32(sB + stage * L::B_BYTES));
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) ptx::umma_f8(d_tmem, adesc + 2 * kk, bdesc + 2 * kk, IDESC, kk > 0);
          ptx::umma_commit(&empty[stage]);
          ptx::umma_commit(&pfull[pb]);
          if (++stage == L::STAGES) {
            stage = 0;
            phase ^= 1;
          }
          pb ^= 1;
          if (pb == 0) ++puse;
        }
      }
      if (!ok) {
        *abort_flag = 1;
        set_status(p.status, MOE_ERR_TIMEOUT);
      }
      ptx::umma_commit(drain);
      ptx::mbar_wait(drain, 0, reinterpret_cast<volatile int*>(s_bad), kWaitLimitNs);
    }
  } else {
    // -------------------------------------------------------------- epilogue (16 warps)
    const int q = warp & 3;           // TMEM lane quarter this warp may access
    const int cq = (warp - 2) >> 2;   // column quarter
    const int row_t = q * 32 + lane;
    const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
    // TMEM columns of this thread's two 32-column pieces: (gate, up) or one 64-column range
    const int c_lo = EPI ? 32 * cq : 64 * cq;
    const int c_hi = EPI ? 128 + 32 * cq : 64 * cq + 32;
    const int nbk = p.K / 128;
    uint32_t pb = 0, puse = 0;
    int it = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x, ++it) {
      const TileCoord tc = decode_tile(s_tile, s_off, G, nt, tile);
      const int g = tc.g, nb = tc.nb;
      const int r_in = tc.mb * BM + row_t;
      const bool valid = r_in < tc.m_g;
      const size_t grow = static_cast<size_t>(s_off[g] + r_in);
      // weight-block scales of the thread's two column pieces: (gate, up) blocks, or one block of 128 columns
      const float* bsc = g >= p.G_main ? p.Bx_scales
                                       : p.B_scales + static_cast<size_t>(g) * ((EPI ? 2 : 1) * p.N / 128) * nbk;
      const float* sb_lo_p = bsc + static_cast<size_t>(EPI ? nb : 2 * nb + (cq >> 1)) * nbk;
      const float* sb_hi_p = bsc + static_cast<size_t>(EPI ? p.N / 128 + nb : 2 * nb + (cq >> 1)) * nbk;
      // fp32 accumulators as pairs for the packed FMA: acc[i] holds columns 2i, 2i+1 of the thread's 64
      float2 acc[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) acc[i] = make_float2(0.f, 0.f);
      // Scales are fetched ahead of use so that no K block waits on a global
      // load: the row's sa[kb] through a 2-deep register queue, the two
      // weight-block scales one K block ahead (the same address in every lane).
      const float* sa_p = p.A_scales + a_source_row(p, static_cast<int>(grow));
      const size_t rstride = static_cast<size_t>(p.a_rows ? p.a_src_rows : p.rows);
      float sa0 = valid ? __ldg(sa_p) : 0.f;
      float sa1 = (valid && 1 < nbk) ? __ldg(sa_p + rstride) : 0.f;
      sa_p += 2 * rstride;
      float sbl = __ldg(sb_lo_p), sbh = __ldg(sb_hi_p);
      for (int kb = 0; kb < nbk; ++kb) {
        const float m_lo = sa0 * sbl;
        const float m_hi = sa0 * sbh;
        sa0 = sa1;
        sa1 = (valid && kb + 2 < nbk) ? __ldg(sa_p) : 0.f;
        sa_p += rstride;
        if (kb + 1 < nbk) {
          sbl = __ldg(sb_lo_p + kb + 1);
          sbh = __ldg(sb_hi_p + kb + 1);
        }
        if (!ptx::mbar_wait_warp(&pfull[pb], puse & 1, abort_flag, kWaitLimitNs)) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        const uint32_t t0 = lane_base + pb * MMA_N;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          uint32_t v[8];
          ptx::tmem_ld_32x32b_x8(t0 + (j < 4 ? c_lo : c_hi) + (j & 3) * 8, v);
          ptx::tmem_ld_wait();
          const float m = j < 4 ? m_lo : m_hi;
          const float2 m2 = make_float2(m, m);
#pragma unroll
          for (int i = 0; i < 4; ++i)
            acc[4 * j + i] =
                __ffma2_rn(make_float2(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1])), m2, acc[4 * j + i]);
        }
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&pempty[pb]);
        pb ^= 1;
        if (pb == 0) ++puse;
      }
      if (!ok) break;
      // Output.  A warp whose 32 rows all belong to the group stages them in
      // its shared-memory buffer and writes them with one bulk tensor store
      // (full 128-byte lines); a slice that crosses the group's end stores
      // its valid rows one by one, so the next group's rows are never touched.
      const int r0 = tc.mb * BM + q * 32;
      const bool slice_full = L::STAGE_OUT && r0 + 32 <= tc.m_g;
      uint8_t* s_out = smem + L::OUTB + (warp - 2) * L::OUT_WARP;
      if (slice_full) {
        if (lane == 0) ptx::bulk_wait_read_all();  // the previous tile's store has read the buffer
        __syncwarp();
      }
      if constexpr (EPI == 1) {
        // columns 0..31 of the thread are gate, 32..63 the matching up columns;
        // h = silu(gate) * up replaces the gate half in place
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float2 gt = acc[i], up = acc[16 + i];
          acc[i].x = silu(gt.x) * up.x;
          acc[i].y = silu(gt.y) * up.y;
        }

        if constexpr (OUT == 2) {
          float amax = 0.f;
#pragma unroll
          for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fmaxf(fabsf(acc[i].x), fabsf(acc[i].y)));
          float* xa = s_amax + (it & 1) * 512;
          xa[cq * 128 + row_t] = amax;
          __syncwarp();
          if (lane == 0) ptx::mbar_arrive(xchg);
          if (!ptx::mbar_wait_warp(xchg, it & 1, abort_flag, kWaitLimitNs)) {
            ok = false;
            break;
          }
          amax = fmaxf(fmaxf(xa[row_t], xa[128 + row_t]), fmaxf(xa[256 + row_t], xa[384 + row_t]));
          const float sc = amax > 0.f ? __fdiv_rn(amax, 448.0f) : 1.0f;
          uint32_t qw[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const uint16_t lo = f32x2_to_e4m3x2(__fdiv_rn(acc[2 * i].x, sc), __fdiv_rn(acc[2 * i].y, sc));
            const uint16_t hi = f32x2_to_e4m3x2(__fdiv_rn(acc[2 * i + 1].x, sc), __fdiv_rn(acc[2 * i + 1].y, sc));
            qw[i] = static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
          }
          if (valid && cq == 0) p.C_scales[static_cast<size_t>(nb) * p.rows + grow] = sc;
          if (slice_full) {  // 32 rows x 32 B, row-major
            uint4* d = reinterpret_cast<uint4*>(s_out + lane * 32);
            d[0] = make_uint4(qw[0], qw[1], qw[2], qw[3]);
            d[1] = make_uint4(qw[4], qw[5], qw[6], qw[7]);
          } else if (valid) {
            uint4* dst = reinterpret_cast<uint4*>(static_cast<uint8_t*>(p.C) + grow * p.N + nb * 128 + cq * 32);
            dst[0] = make_uint4(qw[0], qw[1], qw[2], qw[3]);
            dst[1] = make_uint4(qw[4], qw[5], qw[6], qw[7]);
          }
        } else {
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const __nv_bfloat162 hb = __floats2bfloat162_rn(acc[i].x, acc[i].y);
            pk[i] = *reinterpret_cast<const uint32_t*>(&hb);
          }
          uint4* dst = slice_full ? reinterpret_cast<uint4*>(s_out + lane * 64)  // 32 rows x 64 B, row-major
                                  : reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.C) + grow * p.N +
                                                             nb * 128 + cq * 32);
          if (slice_full || valid) {
#pragma unroll
            for (int v = 0; v < 4; ++v) dst[v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
          }
        }
      } else {
        uint32_t pk[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const __nv_bfloat162 hb = __floats2bfloat162_rn(acc[i].x, acc[i].y);
          pk[i] = *reinterpret_cast<const uint32_t*>(&hb);
        }
        if (slice_full) {
          // 32 rows x 128 B in the 128-byte swizzled layout of the store map:
          // 16-byte chunk c of row r sits at chunk c ^ (r % 8)
#pragma unroll
          for (int c = 0; c < 8; ++c)
            *reinterpret_cast<uint4*>(s_out + lane * 128 + ((c ^ (lane & 7)) << 4)) =
                make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
        } else if (valid) {
          uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.C) + grow * p.N + nb * 256 + cq * 64);
#pragma unroll
          for (int c = 0; c < 8; ++c) dst[c] = make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
        }
      }
      if (slice_full) {
        ptx::fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          const int x = EPI ? nb * 128 + cq * 32 : nb * 256 + cq * 64;
          ptx::tma_store_2d(&tmC, s_out, x, s_off[g] + r0);
          ptx::bulk_commit_group();
        }
      }
    }
    if (lane == 0) ptx::bulk_wait_all();  // this warp's stores are complete before the CTA exits
    if (!ok) {
      *abort_flag = 1;
      set_status(p.status, MOE_ERR_TIMEOUT);
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem_base, L::TMEM_COLS);
  }
}

// ------------------------------------------------------------------ MX FP8 (block-scaled E4M3) kernel
// E4M3 operands whose scales are powers of two ("MegaMoE ..." §2.3 / §5.1
// groups: 1x128 per token, 128x128 per weight block).  The tensor core takes
// them as UE8M0 block scales (tcgen05.mma kind::mxf8f6f4, one scale per row
// per 32 K elements), so the whole K reduction of a tile accumulates in TMEM
// with no promotion step: D = sum_k qa * qb * 2^(ea[m, k/128] + eb[n/128, k/128]).
// The four 32-wide sub-blocks of a 128-wide K block share one scale, so
// byte 0 of each scale-factor word serves every MMA of the block.
//
// Per k-step (128 K): a TMA thread loads A [128 x 128 B] and B [256 x 128 B];
// a scale-factor warp writes the step's scale factors into shared memory as
// 32 x 16-byte atoms (lane i, word c = the scale of row i + 32c, in each of
// its four bytes): one atom for A's 128 rows, two for B's 256; the MMA
// thread copies them to TMEM with tcgen05.cp (32x128b.warpx4) and issues
// four block-scaled MMAs 128 x 256 x 32.  TMEM holds one 256-column fp32
// accumulator (the scale factors take 12 columns after it), so the epilogue
// of a tile holds the next tile's MMAs back; the TMA ring keeps loading
// meanwhile.  Eight epilogue warps read the accumulator (two per TMEM lane
// quarter, each half of the columns), release it, then convert and store.
constexpr int kThreadsMX = 352;  // TMA producer, MMA issuer, 8 epilogue warps, scale-factor warp
constexpr int kMXSfWarp = 10;

template <int EPI, int OUT>
struct MXSmem {
  static constexpr int A_BYTES = BM * 128;
  static constexpr int B_BYTES = 256 * 128;
  static constexpr int SF_BYTES = 3 * 512;  // A atom, two B atoms
  static constexpr int STAGE_ALL = A_BYTES + B_BYTES + SF_BYTES;
  // output staging per epilogue warp (32 rows of its column half) for the
  // bulk tensor stores: bf16 128 columns (two 128-byte boxes), bf16 64
  // columns (one box) or E4M3 64 columns (64-byte rows)
  static constexpr int OUT_WARP = EPI == 0 ? 8192 : (OUT == 2 ? 2048 : 4096);
  static constexpr int FIXED = 512 + 2 * (kMaxGroups + 2) * 4 + 2 * 2 * 128 * 4 + 2048;  // + both alignments
  static constexpr int STAGES_FIT = (227 * 1024 - FIXED - 8 * OUT_WARP) / STAGE_ALL;
  static constexpr int STAGES = STAGES_FIT > 4 ? 4 : STAGES_FIT;
  static constexpr int SB = STAGES * A_BYTES;                   // B ring
  static constexpr int SFR = SB + STAGES * B_BYTES;             // scale-factor ring
  static constexpr int OUTB = (SFR + STAGES * SF_BYTES + 1023) / 1024 * 1024;  // output staging
  static constexpr int BARS = OUTB + 8 * OUT_WARP;              // barriers and flags
  static constexpr int TABLES = BARS + 512;                     // group offsets and tile prefix
  static constexpr int AMAX = TABLES + 2 * (kMaxGroups + 2) * 4;  // [2 parity][2 halves][128 rows]
  static constexpr int SMEM = AMAX + 2 * 2 * 128 * 4 + 1024;    // + alignment slack
  static_assert(STAGES >= 3, "pipeline depth");
  static_assert(OUTB % 1024 == 0, "128-byte swizzled staging needs 1024-byte alignment");
  static_assert(SMEM <= 227 * 1024, "shared memory budget");
};

// The UE8M0 byte of a power-of-two fp32 scale (2^-127 .. 2^127), repeated in
// the four bytes of a word.
__device__ __forceinline__ uint32_t ue8m0_word(float s) {
  return ((__float_as_uint(s) >> 23) & 0xffu) * 0x01010101u;
}

template <int EPI, int OUT>  // EPI 1: SiLU gate (OUT 0 bf16 / 2 MX e4m3); EPI 0: OUT 0 bf16
__global__ void __launch_bounds__(kThreadsMX, 1)
    gg_mx_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                 const __grid_constant__ CUtensorMap tmBx, const __grid_constant__ CUtensorMap tmC, const Params p) {
  pdl_wait();  // the preceding kernel on the stream is complete and visible
  pdl_launch_dependents();
  using L = MXSmem<EPI, OUT>;
  constexpr int MMA_N = 256;
  constexpr int OUT_COLS = EPI ? 128 : 256;
  constexpr uint32_t IDESC = ptx::make_idesc_mx(BM, MMA_N);
  constexpr uint32_t SFA_COL = 256, SFB_COL = 260;  // TMEM columns of the scale factors

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + L::SB;
  uint8_t* sSF = smem + L::SFR;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::BARS);
  uint64_t* empty = full + L::STAGES;
  uint64_t* tfull = empty + L::STAGES;
  uint64_t* tempty = tfull + 1;
  uint64_t* drain = tempty + 1;
  uint64_t* xchg = drain + 1;  // [4]: the two epilogue warps of a lane quarter swap row amax (E4M3 out)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(xchg + 4);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* s_bad = reinterpret_cast<int*>(tmem_slot + 2);
  int* s_off = reinterpret_cast<int*>(smem + L::TABLES);
  int* s_tile = s_off + kMaxGroups + 2;
  float* s_amax = reinterpret_cast<float*>(smem + L::AMAX);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = p.G_total;
  const int nt = p.N / OUT_COLS;

  if (warp == 0) {
    for (int g = lane; g <= G; g += 32) s_off[g] = p.offsets ? p.offsets[g] : (g == 0 ? 0 : p.rows);
    __syncwarp();
    const int per = (G + 31) / 32;
    const int g0 = min(G, lane * per), g1 = min(G, g0 + per);
    int bad = 0, mine = 0;
    for (int g = g0; g < g1; ++g) {
      const int m = s_off[g + 1] - s_off[g];
      if (m < 0) bad = 1;
      mine += (max(m, 0) + BM - 1) / BM * nt;
    }
    int incl = mine;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    int run = incl - mine;
    for (int g = g0; g < g1; ++g) {
      s_tile[g] = run;
      run += (max(s_off[g + 1] - s_off[g], 0) + BM - 1) / BM * nt;
    }
    if (lane == 31) s_tile[G] = incl;
    if (lane == 0 && (s_off[0] != 0 || s_off[G] > p.rows)) bad = 1;
    bad = __any_sync(0xffffffffu, bad);
    if (lane == 0) {
      *s_bad = bad;
      *abort_flag = 0;
      if (bad && blockIdx.x == 0) set_status(p.status, MOE_ERR_BAD_OFFSETS);
    }
  }
  __syncthreads();
  if (*s_bad) return;

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < L::STAGES; ++s) {
      ptx::mbar_init(&full[s], 2);  // the TMA bytes and the scale-factor warp
      ptx::mbar_init(&empty[s], 1);
    }
    ptx::mbar_init(tfull, 1);
    ptx::mbar_init(tempty, 8);  // one arrival per epilogue warp
    ptx::mbar_init(drain, 1);
    for (int i = 0; i < 4; ++i) ptx::mbar_init(&xchg[i], 2);
    ptx::fence_mbar_init();
    ptx::prefetch_tmap(&tmA);
    ptx::prefetch_tmap(&tmB);
    ptx::prefetch_tmap(&tmBx);
  }
  if (warp == 1) {
    ptx::tmem_alloc(tmem_slot, 512);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int total = s_tile[G];
  const int nk = p.K / 128;

  if (warp == 0 && p.a_rows) {
    // -------------------------------------------------------------- producer, gathered A
    // lane l brings A rows 4l..4l+3 of the tile (one tile::gather4 each k-step);
    // lane 0 also waits for the stage and loads B
    uint32_t stage = 0, phase = 0, issued = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
      const TileCoord tc = decode_tile(s_tile, s_off, G, nt, tile);
      const int g = tc.g, nb = tc.nb;
      int tok[4];
      gather_rows(p, s_off[g] + tc.mb * BM, lane, tok);
      const bool extra = g >= p.G_main;
      const CUtensorMap* mB = extra ? &tmBx : &tmB;
      const int gb = extra ? 0 : g;
      for (int kb = 0; kb < nk; ++kb) {
        int go = 1;
        if (lane == 0) {
          go = ptx::mbar_wait(&empty[stage], phase ^ 1, abort_flag, kWaitLimitNs);
          if (go) ptx::mbar_arrive_expect_tx(&full[stage], L::A_BYTES + L::B_BYTES);
        }
        if (!__shfl_sync(0xffffffffu, go, 0)) {
          ok = false;
          break;
        }
        ptx::tma_gather4(sA + stage * L::A_BYTES + lane * 512, &tmA, &full[stage], kb * 128, tok[0], tok[1], tok[2],
                         tok[3]);
        if (lane == 0) {
          if (EPI) {
            const int brow = gb * 2 * p.N + nb * 128;
            ptx::tma_load_2d(sB + stage * L::B_BYTES, mB, &full[stage], kb * 128, brow);
            ptx::tma_load_2d(sB + stage * L::B_BYTES + 128 * 128, mB, &full[stage], kb * 128, brow + p.N);
          } else {
            ptx::tma_load_2d(sB + stage * L::B_BYTES, mB, &full[stage], kb * 128, gb * p.N + nb * 256);
          }
        }
        ++issued;
        if (++stage == L::STAGES) {
          stage = 0;
          phase ^= 1;
        }
      }
    }
    if (!ok && lane == 0) {
      *abort_flag = 1;
      set_status(p.status, MOE_ERR_TIMEOUT);
      const uint32_t pending = issued < static_cast<uint32_t>(L::STAGES) ? issued : L::STAGES;
      uint32_t s2 = stage, ph = phase;
      for (uint32_t i = 0; i < pending; ++i) {
        if (s2 == 0) {
          s2 = L::STAGES - 1;
          ph ^= 1;
        } else {
          --s2;
        }
        ptx::mbar_wait(&full[s2], ph, reinterpret_cast<volatile int*>(s_bad), kWaitLimitNs);
      }
    }
  } else if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ TMA producer
      uint32_t stage = 0, phase = 0, issued = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
        const TileCoord tc = decode_tile(s_tile, s_off, G, nt, tile);
        const int g = tc.g, nb = tc.nb;
        const int a_row = s_off[g] + tc.mb * BM;
        const bool extra = g >= p.G_main;
        const CUtensorMap* mB = extra ? &tmBx : &tmB;
        const int gb = extra ? 0 : g;
        for (int kb = 0; kb < nk; ++kb) {
          if (!ptx::mbar_wait(&empty[stage], phase ^ 1, abort_flag, kWaitLimitNs)) {
            ok = false;
            break;
          }
          ptx::mbar_arrive_expect_tx(&full[stage], L::A_BYTES + L::B_BYTES);
          ptx::tma_load_2d(sA + stage * L::A_BYTES, &tmA, &full[stage], kb * 128, a_row);
          if (EPI) {
            const int brow = gb * 2 * p.N + nb * 128;
            ptx::tma_load_2d(sB + stage * L::B_BYTES, mB, &full[stage], kb * 128, brow);
            ptx::tma_load_2d(sB + stage * L::B_BYTES + 128 * 128, mB, &full[stage], kb * 128, brow + p.N);
          } else {
            ptx::tma_load_2d(sB + stage * L::B_BYTES, mB, &full[stage], kb * 128, gb * p.N + nb * 256);
          }
          ++issued;
          if (++stage == L::STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      if (!ok) {
        *abort_flag = 1;
        set_status(p.status, MOE_ERR_TIMEOUT);
        const uint32_t pending = issued < static_cast<uint32_t>(L::STAGES) ? issued : L::STAGES;
        uint32_t s2 = stage, ph = phase;
        for (uint32_t i = 0; i < pending; ++i) {
          if (s2 == 0) {
            s2 = L::STAGES - 1;
            ph ^= 1;
          } else {
            --s2;
          }
          ptx::mbar_wait(&full[s2], ph, reinterpret_cast<volatile int*>(s_bad), kWaitLimitNs);
        }
      }
    }
  } else if (warp == kMXSfWarp) {
    // -------------------------------------------------------------- scale-factor warp
    // Lane i writes word c of row i of each atom: A's scale of tile row i + 32c,
    // and B's scale of its 128-row weight block (one value per atom).
    uint32_t stage = 0, phase = 0;
    bool ok = true;
    const size_t rstride = static_cast<size_t>(p.a_rows ? p.a_src_rows : p.rows);
    for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
      const TileCoord tc = decode_tile(s_tile, s_off, G, nt, tile);
      const int g = tc.g, nb = tc.nb;
      const int a_row = s_off[g] + tc.mb * BM;
      const float* bsc = g >= p.G_main ? p.Bx_scales
                                       : p.B_scales + static_cast<size_t>(g) * ((EPI ? 2 : 1) * p.N / 128) * nk;
      const float* sb0 = bsc + static_cast<size_t>(EPI ? nb : 2 * nb) * nk;          // gate / first half
      const float* sb1 = bsc + static_cast<size_t>(EPI ? p.N / 128 + nb : 2 * nb + 1) * nk;  // up / second half
      int rowc[4];
#pragma unroll
      for (int c = 0; c < 4; ++c) rowc[c] = a_source_row(p, min(a_row + lane + 32 * c, p.rows - 1));  // past A: any
      // the scales of the next two k-steps are in flight while this one is written
      float qa[2][4] = {}, qb[2][2] = {};
      auto fetch = [&](float (&fa)[4], float (&fb)[2], int kb) {
        if (kb < nk) {
#pragma unroll
          for (int c = 0; c < 4; ++c) fa[c] = __ldg(p.A_scales + kb * rstride + rowc[c]);
          fb[0] = __ldg(sb0 + kb);
          fb[1] = __ldg(sb1 + kb);
        }
      };
      fetch(qa[0], qb[0], 0);
      fetch(qa[1], qb[1], 1);
      for (int kb = 0; kb < nk; ++kb) {
        float sa[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          sa[c] = qa[0][c];
          qa[0][c] = qa[1][c];
        }
        const float b0 = qb[0][0], b1 = qb[0][1];
        qb[0][0] = qb[1][0];
        qb[0][1] = qb[1][1];
        fetch(qa[1], qb[1], kb + 2);
        if (!ptx::mbar_wait_warp(&empty[stage], phase ^ 1, abort_flag, kWaitLimitNs)) {
          ok = false;
          break;
        }
        uint8_t* sf = sSF + stage * L::SF_BYTES;
        *reinterpret_cast<uint4*>(sf + lane * 16) =
            make_uint4(ue8m0_word(sa[0]), ue8m0_word(sa[1]), ue8m0_word(sa[2]), ue8m0_word(sa[3]));
        const uint32_t w0 = ue8m0_word(b0), w1 = ue8m0_word(b1);
        *reinterpret_cast<uint4*>(sf + 512 + lane * 16) = make_uint4(w0, w0, w0, w0);
        *reinterpret_cast<uint4*>(sf + 1024 + lane * 16) = make_uint4(w1, w1, w1, w1);
        ptx::fence_proxy_async_smem();  // visible to tcgen05.cp (async proxy)
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&full[stage]);
        if (++stage == L::STAGES) {
          stage = 0;
          phase ^= 1;
        }
      }
    }
    if (!ok && lane == 0) {
      *abort_flag = 1;
      set_status(p.status, MOE_ERR_TIMEOUT);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------------ MMA issuer
      uint32_t stage = 0, phase = 0;
      bool ok = true;
      int it = 0;
      const uint32_t sfa = tmem_base + SFA_COL, sfb = tmem_base + SFB_COL;
      for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x, ++it) {
        if (!ptx::mbar_wait(tempty, (static_cast<uint32_t>(it) & 1) ^ 1, abort_flag, kWaitLimitNs)) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        for (int kb = 0; kb < nk; ++kb) {
          if (!ptx::mbar_wait(&full[stage], phase, abort_flag, kWaitLimitNs)) {
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          const uint32_t sf = ptx::smem_u32(sSF + stage * L::SF_BYTES);
          ptx::tmem_cp_32x128b_warpx4(sfa, ptx::plain_16B_rows_desc(sf));
          ptx::tmem_cp_32x128b_warpx4(sfb, ptx::plain_16B_rows_desc(sf + 512));
          ptx::tmem_cp_32x128b_warpx4(sfb + 4, ptx::plain_16B_rows_desc(sf + 1024));
          const uint64_t adesc = ptx::sw128_kmajor_desc(ptx::smem_u32(sA + stage * L::A_BYTES));
          const uint64_t bdesc = ptx::sw128_kmajor_desc(ptx::smem_u32(sB + stage * L::B_BYTES));
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            ptx::umma_mxf8(tmem_base, adesc + 2 * kk, bdesc + 2 * kk, IDESC, sfa, sfb, (kb | kk) != 0);
          ptx::umma_commit(&empty[stage]);
          if (++stage == L::STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        ptx::umma_commit(tfull);
      }
      if (!ok) {
        *abort_flag = 1;
        set_status(p.status, MOE_ERR_TIMEOUT);
      }
      ptx::umma_commit(drain);
      ptx::mbar_wait(drain, 0, reinterpret_cast<volatile int*>(s_bad), kWaitLimitNs);
    }
  } else {
    // -------------------------------------------------------------- epilogue (warps 2..9)
    const int q = warp & 3;         // TMEM lane quarter this warp may access
    const int hf = (warp - 2) >> 2;  // which half of the tile's columns
    const int row_t = q * 32 + lane;
    const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
    int it = 0;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x, ++it) {
      const TileCoord tc = decode_tile(s_tile, s_off, G, nt, tile);
      const int g = tc.g, nb = tc.nb;
      const int r_in = tc.mb * BM + row_t;
      const bool valid = r_in < tc.m_g;
      const size_t grow = static_cast<size_t>(s_off[g] + r_in);
      if (!ptx::mbar_wait_warp(tfull, static_cast<uint32_t>(it) & 1, abort_flag, kWaitLimitNs)) {
        *abort_flag = 1;
        set_status(p.status, MOE_ERR_TIMEOUT);
        break;
      }
      ptx::tc_fence_after();
      if constexpr (EPI == 1) {
        // gate columns [64 hf, 64 hf + 64) and the matching up columns 128 + ...
        float h[64];
#pragma unroll
        for (int c = 0; c < 64; c += 32) {
          uint32_t gv[32], uv[32];
          ptx::tmem_ld_32x32b_x32(lane_base + 64 * hf + c, gv);
          ptx::tmem_ld_32x32b_x32(lane_base + 128 + 64 * hf + c, uv);
          ptx::tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) h[c + i] = silu(__uint_as_float(gv[i])) * __uint_as_float(uv[i]);
        }
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(tempty);  // the values are in registers: release the accumulator
        // A warp whose 32 rows all belong to the group stages them in shared
        // memory and writes them with a bulk tensor store; a slice crossing
        // the group's end stores its valid rows one by one.
        const bool slice_full = tc.mb * BM + q * 32 + 32 <= tc.m_g;
        uint8_t* s_out = smem + L::OUTB + (warp - 2) * L::OUT_WARP;
        if (slice_full) {
          if (lane == 0) ptx::bulk_wait_read_all();  // the previous tile's store has read the buffer
          __syncwarp();
        }
        if constexpr (OUT == 2) {
          // E4M3 with one power-of-two scale per row per 128 columns: the two halves exchange amax
          float amax = 0.f;
#pragma unroll
          for (int i = 0; i < 64; ++i) amax = fmaxf(amax, fabsf(h[i]));
          float* xa = s_amax + (it & 1) * 256;  // by tile parity: a slot is rewritten only after both read it
          xa[hf * 128 + row_t] = amax;
          __syncwarp();
          if (lane == 0) ptx::mbar_arrive(&xchg[q]);
          if (!ptx::mbar_wait_warp(&xchg[q], static_cast<uint32_t>(it) & 1, abort_flag, kWaitLimitNs)) {
            *abort_flag = 1;
            set_status(p.status, MOE_ERR_TIMEOUT);
            break;
          }
          amax = fmaxf(amax, xa[(hf ^ 1) * 128 + row_t]);
          const float sc = group_scale<true>(amax);
          uint32_t qw[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const uint16_t lo = f32x2_to_e4m3x2(__fdiv_rn(h[4 * i], sc), __fdiv_rn(h[4 * i + 1], sc));
            const uint16_t hi = f32x2_to_e4m3x2(__fdiv_rn(h[4 * i + 2], sc), __fdiv_rn(h[4 * i + 3], sc));
            qw[i] = static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
          }
          if (valid && hf == 0) p.C_scales[static_cast<size_t>(nb) * p.rows + grow] = sc;
          uint4* dst = slice_full ? reinterpret_cast<uint4*>(s_out + lane * 64)  // 32 rows x 64 B
                                  : reinterpret_cast<uint4*>(static_cast<uint8_t*>(p.C) + grow * p.N + nb * 128 +
                                                             hf * 64);
          if (slice_full || valid) {
#pragma unroll
            for (int v = 0; v < 4; ++v) dst[v] = make_uint4(qw[4 * v], qw[4 * v + 1], qw[4 * v + 2], qw[4 * v + 3]);
          }
        } else {
          uint32_t pk[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const __nv_bfloat162 hb = __floats2bfloat162_rn(h[2 * i], h[2 * i + 1]);
            pk[i] = *reinterpret_cast<const uint32_t*>(&hb);
          }
          if (slice_full) {  // 32 rows x 128 B, 16-byte chunk c of row r at chunk c ^ (r % 8)
#pragma unroll
            for (int c = 0; c < 8; ++c)
              *reinterpret_cast<uint4*>(s_out + lane * 128 + ((c ^ (lane & 7)) << 4)) =
                  make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
          } else if (valid) {
            uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.C) + grow * p.N + nb * 128 + hf * 64);
#pragma unroll
            for (int c = 0; c < 8; ++c) dst[c] = make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
          }
        }
        if (slice_full) {
          ptx::fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            ptx::tma_store_2d(&tmC, s_out, nb * 128 + hf * 64, s_off[g] + tc.mb * BM + q * 32);
            ptx::bulk_commit_group();
          }
        }
      } else {
        // columns [128 hf, 128 hf + 128) as bf16
        uint32_t pk[64];
#pragma unroll
        for (int c = 0; c < 128; c += 32) {
          uint32_t v[32];
          ptx::tmem_ld_32x32b_x32(lane_base + 128 * hf + c, v);
          ptx::tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const __nv_bfloat162 hb = __floats2bfloat162_rn(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
            pk[c / 2 + i] = *reinterpret_cast<const uint32_t*>(&hb);
          }
        }
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(tempty);
        const bool slice_full = tc.mb * BM + q * 32 + 32 <= tc.m_g;
        uint8_t* s_out = smem + L::OUTB + (warp - 2) * L::OUT_WARP;
        if (slice_full) {
          if (lane == 0) ptx::bulk_wait_read_all();  // the previous tile's stores have read the buffer
          __syncwarp();
          // two boxes of 32 rows x 64 columns (128 B), 128-byte swizzled
#pragma unroll
          for (int b = 0; b < 2; ++b)
#pragma unroll
            for (int c = 0; c < 8; ++c)
              *reinterpret_cast<uint4*>(s_out + b * 4096 + lane * 128 + ((c ^ (lane & 7)) << 4)) =
                  make_uint4(pk[32 * b + 4 * c], pk[32 * b + 4 * c + 1], pk[32 * b + 4 * c + 2],
                             pk[32 * b + 4 * c + 3]);
          ptx::fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            const int y = s_off[g] + tc.mb * BM + q * 32;
            ptx::tma_store_2d(&tmC, s_out, nb * 256 + hf * 128, y);
            ptx::tma_store_2d(&tmC, s_out + 4096, nb * 256 + hf * 128 + 64, y);
            ptx::bulk_commit_group();
          }
        } else if (valid) {
          uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.C) + grow * p.N + nb * 256 + hf * 128);
#pragma unroll
          for (int v = 0; v < 16; ++v) dst[v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
        }
      }
    }
    if (lane == 0) ptx::bulk_wait_all();  // this warp's stores are complete before the CTA exits
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem_base, 512);
  }
}

// ------------------------------------------------------------------ host side
}  // namespace

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(f);
  });
  return fn;
}

// 2-D K-major map over [rows, K] elements of `ebytes` bytes, box {128 B, box_rows}.
bool make_map(CUtensorMap* m, const void* base, int ebytes, uint64_t rows, uint64_t K, uint32_t box_rows) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) {
    record_cuda_error(cudaErrorNotSupported, "cuTensorMapEncodeTiled unavailable from the driver");
    return false;
  }
  const cuuint64_t dims[2] = {K, rows};
  const cuuint64_t strides[1] = {K * static_cast<uint64_t>(ebytes)};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(128 / ebytes), box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUtensorMapDataType dt = ebytes == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8;
  const CUresult r = enc(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                         CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    record_cuda_error(cudaErrorInvalidValue, "cuTensorMapEncodeTiled rejected the operand layout");
    return false;
  }
  return true;
}

namespace {

// 2-D map over a row-major [rows, cols] output for tiled bulk stores of
// {box_cols, box_rows} boxes (box_cols * ebytes = 128 with 128-byte swizzle).
bool make_store_map(CUtensorMap* m, void* base, int ebytes, uint64_t rows, uint64_t cols, uint32_t box_cols,
                    uint32_t box_rows, bool swizzle128) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) {
    record_cuda_error(cudaErrorNotSupported, "cuTensorMapEncodeTiled unavailable from the driver");
    return false;
  }
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * static_cast<uint64_t>(ebytes)};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUtensorMapDataType dt = ebytes == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8;
  const CUresult r = enc(m, dt, 2, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                         swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                         CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    record_cuda_error(cudaErrorInvalidValue, "cuTensorMapEncodeTiled rejected the output layout");
    return false;
  }
  return true;
}

// 4-D view of stacked [G][2N][K] bf16 gate/up weights for the swap-AB kernel:
// (k, row r of a 16-row chunk, half h = gate/up, chunk c) -> row c*16 + r + h*N.
// Chunks run over all groups' rows; only gate chunks are addressed, the up
// half adds N rows, so the outermost extent stops N rows short of the end.
bool make_gateup_map(CUtensorMap* m, const void* base, int G, int N, int K) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) {
    record_cuda_error(cudaErrorNotSupported, "cuTensorMapEncodeTiled unavailable from the driver");
    return false;
  }
  const uint64_t rowb = static_cast<uint64_t>(K) * 2;
  const cuuint64_t dims[4] = {static_cast<cuuint64_t>(K), 16, 2,
                              (static_cast<cuuint64_t>(G) * 2 * N - N) / 16};
  const cuuint64_t strides[3] = {rowb, rowb * N, rowb * 16};
  const cuuint32_t box[4] = {64, 16, 2, 4};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  const CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    record_cuda_error(cudaErrorInvalidValue, "cuTensorMapEncodeTiled rejected the gate/up layout");
    return false;
  }
  return true;
}

// The A operand's map: [rows, K] in 128-row boxes, or, when A rows are
// gathered, the source [a_src_rows, K] in one-row boxes for tile::gather4.
bool a_map(CUtensorMap* m, const GemmArgs& a, int ebytes) {
  if (a.a_rows)
    return make_map(m, a.A, ebytes, static_cast<uint64_t>(a.a_src_rows > 0 ? a.a_src_rows : 1), a.K, 1);
  return make_map(m, a.A, ebytes, static_cast<uint64_t>(a.rows > 0 ? a.rows : 1), a.K, BM);
}

template <int MMA_N, int EPI, int OUT>
int run_bf16(const GemmArgs& a, cudaStream_t s) {
  using L = Tile<MMA_N, OUT == 0 && EPI == 0>;
  static_assert(L::SMEM <= 227 * 1024, "shared memory budget");
  const int nb_rows = EPI ? 2 * a.N : a.N;
  const uint32_t box_b = EPI ? MMA_N / 2 : MMA_N;
  CUtensorMap mA, mB, mBx;
  if (!a_map(&mA, a, 2)) return MOE_ERR_CUDA;
  const uint64_t b_rows = a.B_rows > 0 ? static_cast<uint64_t>(a.B_rows)
                                       : static_cast<uint64_t>(a.G > 0 ? a.G : 1) * nb_rows;
  if (!make_map(&mB, a.B, 2, b_rows, a.K, box_b)) return MOE_ERR_CUDA;
  if (!make_map(&mBx, a.has_extra ? a.B_extra : a.B, 2, nb_rows, a.K, box_b)) return MOE_ERR_CUDA;
  // bf16 output: boxes of 32 rows x 64 columns for the epilogue's bulk tensor stores
  CUtensorMap mC = mA;
  if (L::OUT_WARP > 0 &&
      !make_store_map(&mC, a.C, 2, static_cast<uint64_t>(a.rows > 0 ? a.rows : 1), a.N, 64, 32, true))
    return MOE_ERR_CUDA;
  static bool attr_set[64] = {};
  int dev = 0;
  MOE_CUDA_CHECK(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return MOE_ERR_UNSUPPORTED;
  if (!attr_set[dev]) {
    MOE_CUDA_CHECK(cudaFuncSetAttribute(gg_bf16_kernel<MMA_N, EPI, OUT>,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize, L::SMEM));
    attr_set[dev] = true;
  }
  Params p{};
  p.offsets = a.offsets;
  p.G_total = a.G + a.has_extra;
  p.G_main = a.G;
  p.N = a.N;
  p.K = a.K;
  p.rows = a.rows;
  p.ksplit = a.ksplit > 1 ? a.ksplit : 1;
  p.split_stride = static_cast<size_t>(a.rows) * a.N;
  p.C = a.C;
  p.status = a.status;
  p.wait_ns = a.wait_ns ? a.wait_ns : kWaitLimitNs;
  p.stall = a.stall;
  p.a_rows = a.a_rows;
  p.a_src_rows = a.a_src_rows;
  return launch_pdl(__func__, gg_bf16_kernel<MMA_N, EPI, OUT>, dim3(a.grid > 0 ? a.grid : num_sms()), dim3(kThreads),
                    L::SMEM, s, mA, mB, mBx, mC, p);
}

template <int EPI>
int run_bf16_swap(const GemmArgs& a, cudaStream_t s) {
  static_assert(kSwapSmem <= 227 * 1024, "shared memory budget");
  const int nb_rows = EPI ? 2 * a.N : a.N;
  CUtensorMap mX, mW, mWx;
  if (!make_map(&mX, a.A, 2, static_cast<uint64_t>(a.rows > 0 ? a.rows : 1), a.K, kSwapNT)) return MOE_ERR_CUDA;
  const int G = a.G > 0 ? a.G : 1;
  if (EPI) {
    if (!make_gateup_map(&mW, a.B, G, a.N, a.K)) return MOE_ERR_CUDA;
    if (!make_gateup_map(&mWx, a.has_extra ? a.B_extra : a.B, 1, a.N, a.K)) return MOE_ERR_CUDA;
  } else {
    if (!make_map(&mW, a.B, 2, static_cast<uint64_t>(G) * nb_rows, a.K, 128)) return MOE_ERR_CUDA;
    if (!make_map(&mWx, a.has_extra ? a.B_extra : a.B, 2, nb_rows, a.K, 128)) return MOE_ERR_CUDA;
  }
  static bool attr_set[64] = {};
  int dev = 0;
  MOE_CUDA_CHECK(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return MOE_ERR_UNSUPPORTED;
  if (!attr_set[dev]) {
    MOE_CUDA_CHECK(
        cudaFuncSetAttribute(gg_bf16_swap_kernel<EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSwapSmem));
    attr_set[dev] = true;
  }
  Params p{};
  p.offsets = a.offsets;
  p.G_total = a.G + a.has_extra;
  p.G_main = a.G;
  p.N = a.N;
  p.K = a.K;
  p.rows = a.rows;
  p.ksplit = 1;
  p.C = a.C;
  p.status = a.status;
  return launch_pdl(__func__, gg_bf16_swap_kernel<EPI>, dim3(num_sms()), dim3(kThreads), kSwapSmem, s, mX, mW, mWx, p);
}

template <int EPI, int OUT>
int run_bf16_pair(const GemmArgs& a, cudaStream_t s) {
  static_assert(kPairSmem <= 227 * 1024, "shared memory budget");
  const int nb_rows = EPI ? 2 * a.N : a.N;
  CUtensorMap mA, mB, mBx;
  if (!make_map(&mA, a.A, 2, static_cast<uint64_t>(a.rows > 0 ? a.rows : 1), a.K, 128)) return MOE_ERR_CUDA;
  if (!make_map(&mB, a.B, 2, static_cast<uint64_t>(a.G > 0 ? a.G : 1) * nb_rows, a.K, 128)) return MOE_ERR_CUDA;
  if (!make_map(&mBx, a.has_extra ? a.B_extra : a.B, 2, nb_rows, a.K, 128)) return MOE_ERR_CUDA;
  // 64-row boxes for the gated half tiles (64 gate rows, then the 64 matching up rows)
  CUtensorMap mB64, mBx64, mA64;
  if (!make_map(&mB64, a.B, 2, static_cast<uint64_t>(a.G > 0 ? a.G : 1) * nb_rows, a.K, 64)) return MOE_ERR_CUDA;
  if (!make_map(&mBx64, a.has_extra ? a.B_extra : a.B, 2, nb_rows, a.K, 64)) return MOE_ERR_CUDA;
  // 64-row A boxes for the half tiles (64 rows per CTA)
  if (!make_map(&mA64, a.A, 2, static_cast<uint64_t>(a.rows > 0 ? a.rows : 1), a.K, 64)) return MOE_ERR_CUDA;
  static int clusters[64] = {};
  int dev = 0;
  MOE_CUDA_CHECK(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return MOE_ERR_UNSUPPORTED;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kPairSmem;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (!clusters[dev]) {
    MOE_CUDA_CHECK(cudaFuncSetAttribute(gg_bf16_pair_kernel<EPI, OUT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        kPairSmem));
    // persistent grid: as many CTA pairs as can be resident at once
    cfg.gridDim = dim3(num_sms() & ~1);
    int n = 0;
    MOE_CUDA_CHECK(cudaOccupancyMaxActiveClusters(&n, gg_bf16_pair_kernel<EPI, OUT>, &cfg));
    clusters[dev] = n > 0 ? n : 1;
  }
  cfg.gridDim = dim3(2 * clusters[dev]);
  cudaLaunchAttribute attrs[2] = {cfg.attrs[0], {}};
  attrs[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // see launch_pdl
  attrs[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attrs;
  cfg.numAttrs = 2;
  Params p{};
  p.offsets = a.offsets;
  p.G_total = a.G + a.has_extra;
  p.G_main = a.G;
  p.N = a.N;
  p.K = a.K;
  p.rows = a.rows;
  p.ksplit = 1;
  p.C = a.C;
  p.status = a.status;
  MOE_CUDA_CHECK(cudaLaunchKernelEx(&cfg, gg_bf16_pair_kernel<EPI, OUT>, mA, mB, mBx, mB64, mBx64, mA64, p));
  return MOE_OK;
}

template <int EPI, int OUT>
int run_fp8(const GemmArgs& a, cudaStream_t s) {
  constexpr int kF8Smem = F8Smem<EPI, OUT>::SMEM;
  const int nb_rows = EPI ? 2 * a.N : a.N;
  const uint32_t box_b = EPI ? 128 : 256;
  CUtensorMap mA, mB, mBx;
  if (!a_map(&mA, a, 1)) return MOE_ERR_CUDA;
  if (!make_map(&mB, a.B, 1, static_cast<uint64_t>(a.G > 0 ? a.G : 1) * nb_rows, a.K, box_b)) return MOE_ERR_CUDA;
  if (!make_map(&mBx, a.has_extra ? a.B_extra : a.B, 1, nb_rows, a.K, box_b)) return MOE_ERR_CUDA;
  // output boxes of one warp's 32 rows: 64 bf16 columns (128-byte swizzle), or 32 columns of the gated output
  CUtensorMap mC;
  const uint64_t c_rows = static_cast<uint64_t>(a.rows > 0 ? a.rows : 1);
  if (!make_store_map(&mC, a.C, OUT == 2 ? 1 : 2, c_rows, a.N, EPI ? 32 : 64, 32, !EPI)) return MOE_ERR_CUDA;
  static bool attr_set[64] = {};
  int dev = 0;
  MOE_CUDA_CHECK(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return MOE_ERR_UNSUPPORTED;
  if (!attr_set[dev]) {
    MOE_CUDA_CHECK(cudaFuncSetAttribute(gg_fp8_kernel<EPI, OUT>, cudaFuncAttributeMaxDynamicSharedMemorySize, kF8Smem));
    attr_set[dev] = true;
  }
  Params p{};
  p.offsets = a.offsets;
  p.G_total = a.G + a.has_extra;
  p.G_main = a.G;
  p.N = a.N;
  p.K = a.K;
  p.rows = a.rows;
  p.ksplit = 1;
  p.C = a.C;
  p.status = a.status;
  p.A_scales = a.A_scales;
  p.B_scales = a.B_scales;
  p.Bx_scales = a.has_extra ? a.B_extra_scales : a.B_scales;
  p.C_scales = a.C_scales;
  p.a_rows = a.a_rows;
  p.a_src_rows = a.a_src_rows;
  return launch_pdl(__func__, gg_fp8_kernel<EPI, OUT>, dim3(num_sms()), dim3(kThreadsF8), kF8Smem, s, mA, mB, mBx, mC,
                    p);
}


template <int EPI, int OUT>
int run_mx(const GemmArgs& a, cudaStream_t s) {
  constexpr int kSmem = MXSmem<EPI, OUT>::SMEM;
  const int nb_rows = EPI ? 2 * a.N : a.N;
  const uint32_t box_b = EPI ? 128 : 256;
  CUtensorMap mA, mB, mBx;
  if (!a_map(&mA, a, 1)) return MOE_ERR_CUDA;
  if (!make_map(&mB, a.B, 1, static_cast<uint64_t>(a.G > 0 ? a.G : 1) * nb_rows, a.K, box_b)) return MOE_ERR_CUDA;
  if (!make_map(&mBx, a.has_extra ? a.B_extra : a.B, 1, nb_rows, a.K, box_b)) return MOE_ERR_CUDA;
  // output boxes of one epilogue warp: 32 rows x 64 columns (bf16 128-byte swizzled, or E4M3 64-byte rows)
  CUtensorMap mC;
  const uint64_t c_rows = static_cast<uint64_t>(a.rows > 0 ? a.rows : 1);
  if (!make_store_map(&mC, a.C, OUT == 2 ? 1 : 2, c_rows, a.N, 64, 32, OUT != 2)) return MOE_ERR_CUDA;
  static bool attr_set[64] = {};
  int dev = 0;
  MOE_CUDA_CHECK(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return MOE_ERR_UNSUPPORTED;
  if (!attr_set[dev]) {
    MOE_CUDA_CHECK(cudaFuncSetAttribute(gg_mx_kernel<EPI, OUT>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem));
    attr_set[dev] = true;
  }
  Params p{};
  p.offsets = a.offsets;
  p.G_total = a.G + a.has_extra;
  p.G_main = a.G;
  p.N = a.N;
  p.K = a.K;
  p.rows = a.rows;
  p.ksplit = 1;
  p.C = a.C;
  p.status = a.status;
  p.A_scales = a.A_scales;
  p.B_scales = a.B_scales;
  p.Bx_scales = a.has_extra ? a.B_extra_scales : a.B_scales;
  p.C_scales = a.C_scales;
  p.a_rows = a.a_rows;
  p.a_src_rows = a.a_src_rows;
  return launch_pdl(__func__, gg_mx_kernel<EPI, OUT>, dim3(num_sms()), dim3(kThreadsMX), kSmem, s, mA, mB, mBx, mC,
                    p);
}

}  // namespace

// Which kernel a grouped GEMM runs on: decided on the host from shapes alone
// (the per-group row counts live on the device).
enum GemmVariant {
  kEmpty = 0, kUnsupported, kInvalid,
  kSwapGate, kSwapNone,                       // weights on the 128-row side (a few tokens per group)
  kGate64, kGate128, kPairGate,               // SiLU gate: 64 / 128 output columns per tile, CTA pairs
  kPairNone, kPairNoneF32,                    // no epilogue on CTA pairs (bf16 / fp32 out)
  kNone256, kNone128, kNone64,                // single-CTA, bf16 out
  kNone256F32, kNone128F32, kNone64F32,       // single-CTA, fp32 out (router logits, split-K)
  kFp8GateE4M3, kFp8GateBf16, kFp8None,       // E4M3 operands, per-128-K promotion
  kMxGateE4M3, kMxGateBf16, kMxNone           // E4M3 with power-of-two scales applied by the MMA
};

int plan_grouped_gemm(const GemmArgs& a, int sms) {
  const int groups = a.G + a.has_extra;
  if (groups == 0 || a.rows == 0) return kEmpty;
  if (a.ab_dtype == MOE_BF16) {
    // CTA pairs pay off when tiles of 256 rows are mostly full: large groups on average;
    // groups of a few tokens (decode) put the weights on the 128-row side instead
    // gathered A rows (tile::gather4) are loaded by the single-CTA kernels only
    const bool pairs = !a.a_rows && (a.pair_tiles > 0 || (a.pair_tiles == 0 && a.rows >= 512 * groups));
    const bool swap = !a.a_rows && (a.swap_ab > 0 || (a.swap_ab == 0 && a.rows < 32 * groups));
    if (swap && a.ksplit <= 1 && a.c_dtype == MOE_BF16) {
      if (a.epilogue == MOE_EPI_SILU_GATE && a.N % 64 == 0) return kSwapGate;
      if (a.epilogue == MOE_EPI_NONE && a.N % 128 == 0) return kSwapNone;
    }
    if (a.epilogue == MOE_EPI_SILU_GATE) {
      if (a.c_dtype != MOE_BF16 || a.N % 64 != 0 || a.ksplit > 1) return kUnsupported;
      // small problems: 64-column output tiles (64 gate + 64 up rows of B) give twice
      // the tiles when 128-column tiles would not fill two waves of the SMs
      const long long est_tiles = (static_cast<long long>(a.rows) / 128 + groups) * (a.N / 128);
      const bool narrow =
          a.mma_n == 128 || a.N % 128 != 0 || (a.mma_n == 0 && !pairs && est_tiles < 2ll * sms);
      if (narrow) return kGate64;
      return pairs ? kPairGate : kGate128;
    }
    if (a.c_dtype != MOE_F32 && a.c_dtype != MOE_BF16) return kUnsupported;
    const bool out = a.c_dtype == MOE_F32;
    if (pairs && a.ksplit <= 1 && a.N % 256 == 0 && (a.mma_n == 0 || a.mma_n == 256))
      return out ? kPairNoneF32 : kPairNone;
    if (a.ksplit > 1 && (!out || a.ksplit > a.K / 64)) return kUnsupported;
    const int want = a.mma_n;
    if ((want == 0 || want == 256) && a.N % 256 == 0) return out ? kNone256F32 : kNone256;
    if ((want == 0 || want == 128) && a.N % 128 == 0) return out ? kNone128F32 : kNone128;
    if ((want == 0 || want == 64) && a.N % 64 == 0) return out ? kNone64F32 : kNone64;
    return kUnsupported;
  }
  if (a.ab_dtype == MOE_MXE4M3) {
    if (a.ksplit > 1) return kUnsupported;
    if (a.epilogue == MOE_EPI_SILU_GATE && a.N % 128 == 0) {
      if (a.c_dtype == MOE_MXE4M3) return kMxGateE4M3;
      if (a.c_dtype == MOE_BF16) return kMxGateBf16;
      return kUnsupported;
    }
    if (a.epilogue == MOE_EPI_NONE && a.N % 256 == 0 && a.c_dtype == MOE_BF16) return kMxNone;
    return kUnsupported;
  }
  if (a.ab_dtype == MOE_E4M3) {
    if (a.ksplit > 1) return kUnsupported;
    if (a.epilogue == MOE_EPI_SILU_GATE && a.N % 128 == 0) {
      if (a.c_dtype == MOE_E4M3) return kFp8GateE4M3;
      if (a.c_dtype == MOE_BF16) return kFp8GateBf16;
      return kUnsupported;
    }
    if (a.epilogue == MOE_EPI_NONE && a.N % 256 == 0 && a.c_dtype == MOE_BF16) return kFp8None;
    return kUnsupported;
  }
  return kUnsupported;
}

bool plan_takes_gathered_a(int v) {
  return v == kGate64 || v == kGate128 || v == kNone256 || v == kNone128 || v == kNone64 || v == kFp8GateE4M3 ||
         v == kFp8GateBf16 || v == kFp8None || v == kMxGateE4M3 || v == kMxGateBf16 || v == kMxNone;
}

const char* gemm_variant_name(int v) {
  switch (v) {
    case kEmpty: return "empty";
    case kUnsupported: return "unsupported";
    case kInvalid: return "invalid";
    case kSwapGate: return "bf16 swap-ab 128x32 silu-gate";
    case kSwapNone: return "bf16 swap-ab 128x32";
    case kGate64: return "bf16 128x128 silu-gate (64 out cols)";
    case kGate128: return "bf16 128x256 silu-gate";
    case kPairGate: return "bf16 cta-pair 256x256 silu-gate";
    case kPairNone: return "bf16 cta-pair 256x256";
    case kPairNoneF32: return "bf16 cta-pair 256x256 fp32-out";
    case kNone256: return "bf16 128x256";
    case kNone128: return "bf16 128x128";
    case kNone64: return "bf16 128x64";
    case kNone256F32: return "bf16 128x256 fp32-out";
    case kNone128F32: return "bf16 128x128 fp32-out";
    case kNone64F32: return "bf16 128x64 fp32-out";
    case kFp8GateE4M3: return "e4m3 128x256 silu-gate e4m3-out";
    case kFp8GateBf16: return "e4m3 128x256 silu-gate";
    case kFp8None: return "e4m3 128x256";
    case kMxGateE4M3: return "mx-e4m3 128x256 silu-gate mx-e4m3-out";
    case kMxGateBf16: return "mx-e4m3 128x256 silu-gate";
    case kMxNone: return "mx-e4m3 128x256";
    default: return "unknown";
  }
}

int launch_grouped_gemm(const GemmArgs& a, cudaStream_t s) {
  if (is_e4m3(a.ab_dtype) && (!a.A_scales || !a.B_scales || (a.has_extra && !a.B_extra_scales)))
    return MOE_ERR_UNSUPPORTED;
  switch (plan_grouped_gemm(a, num_sms())) {
    case kEmpty: return MOE_OK;
    case kSwapGate: return run_bf16_swap<1>(a, s);
    case kSwapNone: return run_bf16_swap<0>(a, s);
    case kGate64: return run_bf16<128, 1, 0>(a, s);
    case kGate128: return run_bf16<256, 1, 0>(a, s);
    case kPairGate: return run_bf16_pair<1, 0>(a, s);
    case kPairNone: return run_bf16_pair<0, 0>(a, s);
    case kPairNoneF32: return run_bf16_pair<0, 1>(a, s);
    case kNone256: return run_bf16<256, 0, 0>(a, s);
    case kNone128: return run_bf16<128, 0, 0>(a, s);
    case kNone64: return run_bf16<64, 0, 0>(a, s);
    case kNone256F32: return run_bf16<256, 0, 1>(a, s);
    case kNone128F32: return run_bf16<128, 0, 1>(a, s);
    case kNone64F32: return run_bf16<64, 0, 1>(a, s);
    case kFp8GateE4M3: return a.C_scales ? run_fp8<1, 2>(a, s) : MOE_ERR_INVALID;
    case kFp8GateBf16: return run_fp8<1, 0>(a, s);
    case kFp8None: return run_fp8<0, 0>(a, s);
    case kMxGateE4M3: return a.C_scales ? run_mx<1, 2>(a, s) : MOE_ERR_INVALID;
    case kMxGateBf16: return run_mx<1, 0>(a, s);
    case kMxNone: return run_mx<0, 0>(a, s);
    default: return MOE_ERR_UNSUPPORTED;
  }
}

}  // namespace moe
