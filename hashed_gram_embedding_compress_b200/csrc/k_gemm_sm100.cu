// Dense bf16 contractions of the backward on CTA pairs (tcgen05, TMEM, TMA).
//
// The backward of "Conditional Memory via Scalable Lookup" section 2.3 Eq.
// (3)-(4) / section 2.4 Eq. (6) has three dense contractions besides the
// forward's own (k and v recomputed, which runs on the projection kernel):
//   dW = dkv^T e      (contraction over the rows: both operands MN-major)
//   de = dkv [W_K; W_V] (contraction over the M d + d projection rows: A
//                        K-major, B MN-major, B read from two tensors)
// This kernel computes D[m, n] (= or +=) sum_k A(m, k) B(n, k) for either
// major of A and B:
//   K-major A: stored [M, K] row-major; MN-major A: stored [K, M] row-major
//   (the same for B with N).
// A cluster of two CTAs owns a 256 x 256 tile: CTA rank r loads rows
// [128 r, 128 r + 128) of the tile's A and of its B (the pair MMA, M = 256,
// N = 256, splits B by N), and keeps the tile's 128 x 256 fp32 accumulator in
// TMEM, twice (512 columns): the epilogue of one tile overlaps the next
// tile's mainloop.  Stages of 64 K hold A and B as 128-byte-swizzled boxes;
// an MN-major operand arrives as two 64-wide boxes of 64 K rows, which is the
// canonical MN-major 128-byte-swizzle layout (8 K rows of 128 bytes per atom,
// the two 64-wide halves 8 KB apart).  The epilogue streams the accumulator
// out in 32 x 32 fp32 boxes by TMA store, or by TMA reduce-add when D
// accumulates (then K may also be split over several tiles, each adding its
// part).
// Roles (192 threads): warps 0-3 epilogue (TMEM lanes 32 w..), warp 4 TMA
// producer, warp 5 TMEM allocator and MMA issuer (on the pair's leader).
// Every wait is bounded; on expiry the CTA sets the error bit, leaves its
// loops, drains its MMAs and frees TMEM, as the projection kernels do.
#include "sm100_ptx.cuh"

namespace engram {

namespace {

using namespace sm100;

constexpr int kTileM = 256, kTileN = 256, kBK = 64;
constexpr uint32_t A_BYTES = 128 * 128;               // 128 rows x 64 bf16 of this CTA
constexpr uint32_t B_BYTES = 128 * 128;               // this CTA's 128 of the 256 N rows
constexpr uint32_t HALF_BYTES = 64 * 128;             // one 64-wide MN-major box of 64 K rows
constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES;   // 32 KB
constexpr int STAGES = 6;
constexpr int kEpiWarps = 4;
constexpr int kThreads = (kEpiWarps + 2) * 32;
constexpr int kProducerWarp = kEpiWarps, kMmaWarp = kEpiWarps + 1;
constexpr uint32_t OUT_BYTES = 32 * 32 * 4;           // one 32 x 32 fp32 box
constexpr uint32_t TMEM_COLS = 512;
constexpr int NUM_BARS = 2 * STAGES + 4 + 2;
constexpr size_t SMEM = 1024 + (size_t)STAGES * STAGE_BYTES + (size_t)kEpiWarps * 2 * OUT_BYTES +
                        8 * NUM_BARS + 16;
static_assert(SMEM <= 232448, "shared memory budget");

// Descriptor of an MN-major tile with the 128-byte swizzle: 64 MN elements
// per 128-byte row, one row per K index, 8-row atoms 1024 bytes apart along K
// (SBO) and 64-wide MN blocks `lbo` bytes apart (LBO); version 1, type 2.
__device__ __forceinline__ uint64_t sw128_mn_desc(uint32_t saddr, uint32_t lbo) {
  return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)(lbo >> 4) << 16) |
         ((uint64_t)(1024 >> 4) << 32) | ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

template <bool A_MN, bool B_MN, bool ADD>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_pair_kernel(const __grid_constant__ CUtensorMap map_a,
                     const __grid_constant__ CUtensorMap map_b0,
                     const __grid_constant__ CUtensorMap map_b1,
                     const __grid_constant__ CUtensorMap map_d, GemmArgs g) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  const uint32_t sA = smem_u32(smem);
  const uint32_t sB = sA + STAGES * A_BYTES;
  uint8_t* obuf = smem + (size_t)STAGES * STAGE_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(obuf + (size_t)kEpiWarps * 2 * OUT_BYTES);
  const uint32_t bar0 = smem_u32(bars);
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (STAGES + s); };
  auto tfull_bar = [&](int b) { return bar0 + 8u * (2 * STAGES + b); };
  auto tempty_bar = [&](int b) { return bar0 + 8u * (2 * STAGES + 2 + b); };
  const uint32_t drain_bar = bar0 + 8u * (2 * STAGES + 4);
  const uint32_t pair_bar = drain_bar + 8u;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + NUM_BARS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const bool leader = rank == 0;
  const int mt = (g.M + kTileM - 1) / kTileM, nt = (g.N + kTileN - 1) / kTileN;
  const int kb_total = (g.K + kBK - 1) / kBK;
  const int num_tiles = mt * nt * g.splits;
  const int first_tile = (int)(blockIdx.x >> 1), tile_step = (int)(gridDim.x >> 1);
  // tile -> (m block, n block, K range).  The K split is the slowest index:
  // the tiles running at one time share their K range, so each K slab of A
  // and B is read from HBM about once and then from L2 by the other tiles;
  // neighbouring tiles share their m block.
  auto tile_coords = [&](int tile, int& m_blk, int& n_blk, int& kb0, int& kb1) {
    const int split = tile / (mt * nt), mn = tile - split * (mt * nt);
    m_blk = mn / nt;
    n_blk = mn - m_blk * nt;
    kb0 = split * g.kb_per_split;
    kb1 = min(kb_total, kb0 + g.kb_per_split);
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(tfull_bar(b), 1);
      mbar_init(tempty_bar(b), 2 * kEpiWarps);  // every epilogue warp of the pair
    }
    mbar_init(drain_bar, 1);
    mbar_init(pair_bar, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == kMmaWarp) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(TMEM_COLS));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == kProducerWarp) {
    // ------------------------------------------------------ A / B producer
    if (lane == 0) {
      asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&map_a) : "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&map_b0) : "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&map_b1) : "memory");
    }
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    for (int tile = first_tile; ok && tile < num_tiles; tile += tile_step) {
      int m_blk, n_blk, kb0, kb1;
      tile_coords(tile, m_blk, n_blk, kb0, kb1);
      const int a_mn = g.a_off + m_blk * kTileM + (int)rank * 128;  // this CTA's A rows
      const int b_n = n_blk * kTileN + (int)rank * 128;             // this CTA's B rows
      for (int kb = kb0; kb < kb1; ++kb) {
        if (lane == 0) ok = wait_ready(empty_bar(stage), phase ^ 1u, abort_flag, g.err);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        if (lane == 0) {
          const uint32_t fb = peer_addr(full_bar(stage), 0);
          if (leader) mbar_expect_tx(full_bar(stage), 2 * STAGE_BYTES);
          const uint32_t a_dst = sA + stage * A_BYTES, b_dst = sB + stage * B_BYTES;
          if (A_MN) {
            tma_load_2d_pair(a_dst, &map_a, fb, a_mn, kb * kBK);
            tma_load_2d_pair(a_dst + HALF_BYTES, &map_a, fb, a_mn + 64, kb * kBK);
          } else {
            tma_load_2d_pair(a_dst, &map_a, fb, kb * kBK, a_mn);
          }
          const bool first = kb < g.kb_split;
          const CUtensorMap* mb = first ? &map_b0 : &map_b1;
          const int kk = (first ? kb : kb - g.kb_split) * kBK;
          if (B_MN) {
            tma_load_2d_pair(b_dst, mb, fb, b_n, kk);
            tma_load_2d_pair(b_dst + HALF_BYTES, mb, fb, b_n + 64, kk);
          } else {
            tma_load_2d_pair(b_dst, mb, fb, kk, b_n);
          }
        }
        __syncwarp();
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
    if (!ok && lane == 0) {
      const uint64_t t0 = globaltimer();
      while (globaltimer() - t0 < 100000ull) {
      }
    }
  } else if (warp == kMmaWarp) {
    // --------------------------------------------- MMA issuer (leader only)
    constexpr uint32_t idesc = idesc_bf16<kTileM, kTileN>() | ((uint32_t)A_MN << 15) |
                               ((uint32_t)B_MN << 16);
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    if (leader) {
      int t = 0;
      for (int tile = first_tile; ok && tile < num_tiles; tile += tile_step, ++t) {
        int m_blk, n_blk, kb0, kb1;
        tile_coords(tile, m_blk, n_blk, kb0, kb1);
        const int buf = t & 1;
        if (lane == 0) ok = wait_ready(tempty_bar(buf), ((uint32_t)(t >> 1) & 1u) ^ 1u, abort_flag, g.err);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        tc_fence_after();
        const uint32_t tacc = tmem_base + (uint32_t)(buf * kTileN);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (lane == 0) ok = wait_ready(full_bar(stage), phase, abort_flag, g.err);
          ok = __shfl_sync(0xffffffffu, ok, 0);
          if (!ok) break;
          tc_fence_after();
          if (lane == 0) {
            const uint32_t a_s = sA + stage * A_BYTES, b_s = sB + stage * B_BYTES;
#pragma unroll
            for (int k = 0; k < kBK / 16; ++k) {
              // K = 16 per MMA: 32 bytes along a K-major row, or 16 rows (2 atoms) of an
              // MN-major tile
              const uint64_t ad = A_MN ? sw128_mn_desc(a_s + k * 2048u, HALF_BYTES)
                                       : sw128_desc(a_s) + 2u * k;
              const uint64_t bd = B_MN ? sw128_mn_desc(b_s + k * 2048u, HALF_BYTES)
                                       : sw128_desc(b_s) + 2u * k;
              umma_bf16_pair(tacc, ad, bd, idesc, (kb != kb0 || k != 0) ? 1u : 0u);
            }
            umma_commit_pair_both(empty_bar(stage));
          }
          __syncwarp();
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        if (lane == 0) umma_commit_pair_both(tfull_bar(buf));
        __syncwarp();
      }
      if (lane == 0) {
        umma_commit_pair_local(drain_bar);
        wait_drain(drain_bar, 0);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    bool ok = true;
    int t = 0;
    uint8_t* st0 = obuf + warp * 2 * OUT_BYTES;
    int sbuf = 0;
    for (int tile = first_tile; ok && tile < num_tiles; tile += tile_step, ++t) {
      int m_blk, n_blk, kb0, kb1;
      tile_coords(tile, m_blk, n_blk, kb0, kb1);
      const int buf = t & 1;
      if (lane == 0) ok = wait_ready(tfull_bar(buf), (uint32_t)(t >> 1) & 1u, abort_flag, g.err);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      tc_fence_after();
      const uint32_t taddr = tmem_base + ((uint32_t)(warp * 32) << 16) + (uint32_t)(buf * kTileN);
      const int row0 = m_blk * kTileM + (int)rank * 128 + warp * 32;  // this warp's first row
      const bool rows_in = row0 < g.M;
      uint32_t va[32], vb[32];
      __syncwarp();
      tmem_ld32_async(taddr, va);
      auto chunk = [&](int q, uint32_t(&v)[32], uint32_t(&vn)[32]) {
        tmem_wait32(v);
        __syncwarp();
        if (q + 1 < kTileN / 32) {
          tmem_ld32_async(taddr + (q + 1) * 32, vn);
        } else {
          tc_fence_before();  // last TMEM read of this buffer: hand it back
          __syncwarp();
          if (lane == 0) mbar_arrive_remote(peer_addr(tempty_bar(buf), 0));
        }
        const int col = n_blk * kTileN + q * 32;
        // the staging buffer's previous store has finished reading it
        if (lane == 0) asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
        __syncwarp();
        uint8_t* st = st0 + sbuf * OUT_BYTES;
#pragma unroll
        for (int c = 0; c < 8; ++c)
          *reinterpret_cast<uint4*>(st + sw128_off(lane, c)) =
              make_uint4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
        fence_async_smem();
        __syncwarp();
        if (lane == 0) {
          if (rows_in && col < g.N) {
            if (ADD)
              tma_reduce_add_2d(&map_d, smem_u32(st), g.d_col0 + col, row0);
            else
              tma_store_2d(&map_d, smem_u32(st), g.d_col0 + col, row0);
          } else {
            asm volatile("cp.async.bulk.commit_group;" ::: "memory");
          }
        }
        sbuf ^= 1;
      };
#pragma unroll 1
      for (int q = 0; q < kTileN / 32; q += 2) {
        chunk(q, va, vb);
        chunk(q + 1, vb, va);
      }
    }
    if (lane == 0) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
  }

  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0) {
    mbar_arrive_cluster(peer_addr(pair_bar, rank ^ 1u));
    wait_drain(pair_bar, 0);
  }
  __syncthreads();
  tc_fence_after();
  if (warp == kMmaWarp)
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                 "r"(TMEM_COLS));
}

template <bool A_MN, bool B_MN, bool ADD>
cudaError_t launch_pair(const GemmMaps& maps, const GemmArgs& g, int grid, cudaStream_t stream) {
  auto kern = gemm_pair_kernel<A_MN, B_MN, ADD>;
  cudaError_t e =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t lc = {};
  lc.gridDim = dim3(grid);
  lc.blockDim = dim3(kThreads);
  lc.dynamicSmemBytes = SMEM;
  lc.stream = stream;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = 2;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  lc.attrs = at;
  lc.numAttrs = 1;
  e = cudaLaunchKernelEx(&lc, kern, maps.a, maps.b0, maps.b1, maps.d, g);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace

int gemm_pair_tiles(const GemmArgs& g) {
  return ((g.M + kTileM - 1) / kTileM) * ((g.N + kTileN - 1) / kTileN) * g.splits;
}

cudaError_t launch_gemm_pair(bool a_mn, bool b_mn, bool add, const GemmMaps& maps,
                             const GemmArgs& g, int grid, cudaStream_t stream) {
  if (g.M <= 0 || g.N <= 0 || g.K <= 0) return cudaSuccess;
  if (grid < 2 || (grid & 1) || g.splits < 1 || g.kb_per_split < 1) return cudaErrorInvalidValue;
  if (g.splits > 1 && !add) return cudaErrorInvalidValue;  // split K needs the reduce-add epilogue
  switch ((a_mn ? 4 : 0) | (b_mn ? 2 : 0) | (add ? 1 : 0)) {
    case 0: return launch_pair<false, false, false>(maps, g, grid, stream);
    case 1: return launch_pair<false, false, true>(maps, g, grid, stream);
    case 2: return launch_pair<false, true, false>(maps, g, grid, stream);
    case 3: return launch_pair<false, true, true>(maps, g, grid, stream);
    case 4: return launch_pair<true, false, false>(maps, g, grid, stream);
    case 5: return launch_pair<true, false, true>(maps, g, grid, stream);
    case 6: return launch_pair<true, true, false>(maps, g, grid, stream);
    default: return launch_pair<true, true, true>(maps, g, grid, stream);
  }
}

}  // namespace engram
