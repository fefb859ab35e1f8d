// bf16 projection + context-aware gate on CTA pairs: the large-batch path.
//
// Same computation as k_proj_gate_sm100.cu ("Conditional Memory via Scalable
// Lookup", section 2.3 Eq. (3)-(4), section 2.4 Eq. (6)); only the tiling
// differs.  A cluster of two CTAs on one TPC computes a 512 x 256 tile of
// e . W^T with tcgen05.mma.cta_group::2 (M = 256 per instruction):
//
//   CTA rank r holds rows [256 r, 256 r + 256) of the tile: it loads those
//   256 rows of e (one 256 x 64 TMA box per K step) and rows
//   [128 r, 128 r + 128) of the 256 W rows (the pair's B operand is split by
//   N), and keeps two 128 x 256 fp32 accumulators in its 512 TMEM columns
//   (tile rows 0-127 in columns 0-255, rows 128-255 in columns 256-511).
//   The leader (rank 0) issues, per 16-wide K step, two pair MMAs that share
//   B: rows 0-127 of both CTAs, then rows 128-255 of both CTAs.
//
// Each byte brought from L2 feeds 1.5x the FLOPs of a 128-row tile, which is
// what the mainloop is bound by on this part: the operand stream from L2
// into shared memory, not the tensor pipe.  TMEM holds one tile, so the
// epilogue runs between tiles; eight epilogue warps keep it short, and h is
// prefetched into a 5-slot ring during the mainloop.
//
// Roles (352 threads per CTA):
//   warps 0-7   epilogue: warp w reads TMEM lanes 32(w%4).. of accumulator
//               w/4, i.e. tile row 128(w/4) + 32(w%4) + lane;
//   warp 8      TMA producer of e and W (3 stages x 48 KB);
//   warp 9      TMEM allocator; MMA issuer on the leader;
//   warp 10     TMA producer of h sub-tiles [256 rows x 32 columns, 64-byte
//               swizzle], shared by both epilogue warpgroups; in the value
//               phase out is written over h in the slot and stored by TMA.
// Phases: 0 = keys (partial sums), 1 = values (out = h + alpha v through the
// h ring), 2 = values when out aliases h (the residual update in place): the
// epilogue stages bf16(alpha v) for 64 columns at a time and adds it into out
// with a TMA reduce-add, so h never passes through shared memory; the sum is rounded once more
// (RN(h + RN(alpha v)) instead of RN(h + alpha v)); with one branch the
// whole tile is read out of TMEM (half staged, half kept in registers) before
// the first reduce-add, so the accumulators are free again within a fraction
// of the time the reduce-adds take (bf16 operands); 3 = values for the short
// convolution (Eq. 5): v in fp32 and its sum of squares per row and tile,
// plus alpha; h is not read.
// FP8 form (section 2.4, the projections as one dense FP8 matmul): e and W
// arrive as E4M3 codes, 128 per 128-byte row of a stage (K = 32 per MMA,
// tcgen05.mma kind::f8f6f4, fp32 accumulation), and every accumulator chunk
// is multiplied by W's per-column scale as it leaves TMEM; e's per-row scale
// multiplies the row's key sums (keys) or alpha (values), or v itself (phase
// 3).  Both scales are powers of two.
// Waits are bounded as in the single-CTA kernel; the pair leaves together
// through a bounded handshake, then frees TMEM (cta_group::2).
#include "sm100_ptx.cuh"

namespace engram {

namespace {

using namespace sm100;

constexpr int kRows = 256;                           // tile rows per CTA
constexpr int kCols = 256;                           // tile columns
constexpr int ROW_BYTES = 128;                       // of K per row and stage: 64 bf16 or 128 E4M3
constexpr int kMmaPerStage = ROW_BYTES / 32;         // K = 16 bf16 or 32 E4M3 per MMA
constexpr uint32_t A_BYTES = kRows * ROW_BYTES;      // 32 KB
constexpr uint32_t B_BYTES = (kCols / 2) * ROW_BYTES;  // 16 KB: this CTA's half of B
constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES;  // 48 KB
constexpr int STAGES = 3;
constexpr int H_SLOTS = 5;
constexpr int H_COLS = 32;
constexpr uint32_t H_BYTES = kRows * H_COLS * 2;     // 16 KB
constexpr int kEpiWarps = 8;
constexpr int kThreads = (kEpiWarps + 3) * 32;       // 352
constexpr int kProducerWarp = kEpiWarps, kMmaWarp = kEpiWarps + 1, kHWarp = kEpiWarps + 2;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t W_BYTES = kCols * 4;  // the tile's columns of w_q * w_k (fp32)
constexpr int NUM_BARS = 2 * STAGES + 2 + 2 * H_SLOTS + 4;
constexpr size_t SMEM = 1024 + (size_t)STAGES * STAGE_BYTES + (size_t)H_SLOTS * H_BYTES +
                        W_BYTES + 8 * NUM_BARS + 16;
static_assert(SMEM <= 232448, "shared memory budget");
static_assert(kEpiWarps * 8192 <= H_SLOTS * H_BYTES, "per-warp store staging fits in the h ring");

// v[0..31] (fp32 bits, one accumulator chunk of 32 columns) *= sc[0..31]
// (times rs when ROW): the E4M3 operands' scales.
template <bool ROW>
__device__ __forceinline__ void dequant_chunk(uint32_t (&v)[32], const float* sc, float rs) {
  const float4* sp = reinterpret_cast<const float4*>(sc);
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    float4 s4 = __ldg(sp + c);
    if (ROW) {
      s4.x *= rs;
      s4.y *= rs;
      s4.z *= rs;
      s4.w *= rs;
    }
    const float2 a = f2_unpack(
        f2_mul(f2_pack(v[4 * c], v[4 * c + 1]), f2_pack(__float_as_uint(s4.x), __float_as_uint(s4.y))));
    const float2 b = f2_unpack(f2_mul(f2_pack(v[4 * c + 2], v[4 * c + 3]),
                                      f2_pack(__float_as_uint(s4.z), __float_as_uint(s4.w))));
    v[4 * c] = __float_as_uint(a.x);
    v[4 * c + 1] = __float_as_uint(a.y);
    v[4 * c + 2] = __float_as_uint(b.x);
    v[4 * c + 3] = __float_as_uint(b.y);
  }
}

template <int PHASE, bool F8>
__global__ void __launch_bounds__(kThreads, 1)
    proj_gate_wide_kernel(const __grid_constant__ CUtensorMap map_e,
                          const __grid_constant__ CUtensorMap map_w,
                          const __grid_constant__ CUtensorMap map_h,
                          const __grid_constant__ CUtensorMap map_out, GateArgs g) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  const uint32_t sA = smem_u32(smem);
  const uint32_t sB = sA + STAGES * A_BYTES;
  uint8_t* hbuf = smem + (size_t)STAGES * STAGE_BYTES;
  const uint32_t sH = smem_u32(hbuf);
  const float* wbuf = reinterpret_cast<const float*>(hbuf + (size_t)H_SLOTS * H_BYTES);
  const uint32_t sW = smem_u32(wbuf);
  uint64_t* bars = reinterpret_cast<uint64_t*>(hbuf + (size_t)H_SLOTS * H_BYTES + W_BYTES);
  const uint32_t bar0 = smem_u32(bars);
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (STAGES + s); };
  const uint32_t tfull_bar = bar0 + 8u * (2 * STAGES);
  const uint32_t tempty_bar = tfull_bar + 8u;
  auto hfull_bar = [&](int s) { return bar0 + 8u * (2 * STAGES + 2 + s); };
  auto hempty_bar = [&](int s) { return bar0 + 8u * (2 * STAGES + 2 + H_SLOTS + s); };
  const uint32_t wfull_bar = bar0 + 8u * (2 * STAGES + 2 + 2 * H_SLOTS);
  const uint32_t wempty_bar = wfull_bar + 8u;
  const uint32_t drain_bar = wfull_bar + 16u;
  const uint32_t pair_bar = wfull_bar + 24u;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + NUM_BARS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();  // 0 = the pair's MMA leader
  const bool leader = rank == 0;
  const int R = g.R, d = g.d, M = g.M;
  const int n_total = PHASE == 0 ? M * d : d;
  const int num_n = n_total / kCols;
  const int num_tiles = ((R + 2 * kRows - 1) / (2 * kRows)) * num_n;
  constexpr int BK = F8 ? ROW_BYTES : ROW_BYTES / 2;  // K elements per stage
  const int num_kb = (g.d_mem + BK - 1) / BK;
  const int first_tile = (int)(blockIdx.x >> 1), tile_step = (int)(gridDim.x >> 1);
  // h sub-tiles per tile: one branch in the key phase, every branch in the
  // value phase (v is shared across branches, Eq. 6); none when the value
  // phase adds into h in place
  const int nsub = PHASE >= 2 ? 0 : (kCols / H_COLS) * (PHASE == 0 ? 1 : M);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    mbar_init(tfull_bar, 1);
    mbar_init(tempty_bar, 2 * kEpiWarps);  // every epilogue warp of the pair
    for (int s = 0; s < H_SLOTS; ++s) {
      mbar_init(hfull_bar(s), 1);
      mbar_init(hempty_bar(s), kEpiWarps);  // every epilogue warp releases its rows
    }
    mbar_init(wfull_bar, 1);
    mbar_init(wempty_bar, kEpiWarps);
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
  cluster_sync_all();  // the partner's barriers are initialised before any signal
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // Programmatic dependent launch.  Key phase: e (and its scales) come from
  // the previous kernel; the producers wait for it (the e/W producer after
  // issuing the first tile's W boxes, which do not depend on it) and then let
  // the value phase launch.  Value phase: the next call's gather (which
  // writes the other e buffer) may start at once.
  if (PHASE != 0) griddep_launch_dependents();

  if (warp == kProducerWarp) {
    // ---------------------------------------------------- e / W producer
    if (lane == 0) {
      asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&map_e) : "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&map_w) : "memory");
    }
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    // key phase: the first tile's first stages of W go out before the wait
    // for the previous kernel (every stage is free at this point)
    int pre = 0;
    if (PHASE == 0 && first_tile < num_tiles) {
      pre = num_kb < STAGES ? num_kb : STAGES;
      const int b_row = (first_tile % num_n) * kCols + (int)rank * (kCols / 2);
      if (lane == 0) {
        for (int kb = 0; kb < pre; ++kb) {
          if (leader) mbar_expect_tx(full_bar(kb), 2 * STAGE_BYTES);
          tma_load_2d_pair(sB + kb * B_BYTES, &map_w, peer_addr(full_bar(kb), 0), kb * BK, b_row);
        }
      }
      __syncwarp();
    }
    if (PHASE == 0) {
      griddep_wait();
      griddep_launch_dependents();
    }
    // e (written by the gather with the same policy, read by about ten CTA
    // pairs per launch and by both launches) is kept in L2 over the streamed h
    const uint64_t e_policy = policy_evict_last();
    for (int tile = first_tile; ok && tile < num_tiles; tile += tile_step) {
      const int m_blk = tile / num_n, n_blk = tile - m_blk * num_n;
      const int a_row = m_blk * 2 * kRows + (int)rank * kRows;
      const int b_row = n_blk * kCols + (int)rank * (kCols / 2);
      for (int kb = 0; kb < num_kb; ++kb) {
        const bool early = tile == first_tile && kb < pre;  // W already on its way
        if (!early) {
          if (lane == 0) ok = wait_ready(empty_bar(stage), phase ^ 1u, abort_flag, g.err);
          ok = __shfl_sync(0xffffffffu, ok, 0);
          if (!ok) break;
        }
        if (lane == 0) {
          // the leader's full barrier counts the bytes of both CTAs
          const uint32_t fb = peer_addr(full_bar(stage), 0);
          if (!early && leader) mbar_expect_tx(full_bar(stage), 2 * STAGE_BYTES);
          tma_load_2d_pair_hint(sA + stage * A_BYTES, &map_e, fb, kb * BK, a_row, e_policy);
          if (!early) tma_load_2d_pair(sB + stage * B_BYTES, &map_w, fb, kb * BK, b_row);
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
  } else if (warp == kHWarp) {
    // -------------------------------------------------- h sub-tile producer
    if (lane == 0) asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&map_h) : "memory");
    // h may still be written by the kernel before the previous kernel
    if (PHASE == 0) griddep_wait();
    int slot = 0;
    uint32_t phase = 0;
    bool ok = true;
    uint32_t wphase = 0;
    int tix = 0;
    const int nbox = (kCols / H_COLS) * (PHASE == 0 ? 1 : M);  // h boxes of a tile
    for (int tile = first_tile; ok && tile < num_tiles; tile += tile_step, ++tix) {
      const int m_blk = tile / num_n, n0 = (tile - m_blk * num_n) * kCols;
      const int row0 = m_blk * 2 * kRows + (int)rank * kRows;
      // Bring this tile's h into L2 while its MMAs run: the boxes beyond the
      // smem ring (keys, values) or, in place with one branch, all of them
      // (the epilogue read-modify-writes h in L2), paced by the accumulator:
      // tile i once tile i-1's MMAs are done.  In place with several branches
      // the h of the tiles in flight (M x 128 KB per CTA) does not fit in L2
      // beside e, the prefetched lines were evicted before the reduce-adds
      // reached them and h came from DRAM twice: nothing is prefetched there.
      const bool prefetch = PHASE != 3 && !(PHASE == 2 && M > 1);
      if (PHASE == 2 && prefetch && tix > 0) {
        if (lane == 0) ok = wait_ready(tfull_bar, (uint32_t)(tix - 1) & 1u, abort_flag, g.err);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
      }
      if (prefetch && lane == 0 && row0 < R) {
        for (int i = PHASE == 2 ? 0 : H_SLOTS; i < nbox; ++i)
          tma_prefetch_l2_2d(&map_h, PHASE == 0 ? n0 + H_COLS * i
                                                : (i % M) * d + n0 + H_COLS * (i / M),
                             row0);
      }
      __syncwarp();
      if (PHASE == 0) {
        // the key epilogue's column weights: w_qk[n0 .. n0+256) of [M*d]
        if (lane == 0) ok = wait_ready(wempty_bar, wphase ^ 1u, abort_flag, g.err);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        if (lane == 0) {
          mbar_expect_tx(wfull_bar, W_BYTES);
          bulk_load(sW, g.w_qk + n0, W_BYTES, wfull_bar);
        }
        __syncwarp();
        wphase ^= 1u;
      }
      for (int i = 0; i < nsub; ++i) {
        // h viewed as [R, M*d]: key phase column n0 + 32 i; value phase
        // branch i % M, column n0 + 32 (i / M)
        const int x = PHASE == 0 ? n0 + H_COLS * i : (i % M) * d + n0 + H_COLS * (i / M);
        if (lane == 0) ok = wait_ready(hempty_bar(slot), phase ^ 1u, abort_flag, g.err);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        if (lane == 0) {
          mbar_expect_tx(hfull_bar(slot), H_BYTES);
          tma_load_2d(sH + slot * H_BYTES, &map_h, hfull_bar(slot), x, row0);
        }
        __syncwarp();
        if (++slot == H_SLOTS) {
          slot = 0;
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
    constexpr uint32_t idesc = F8 ? idesc_e4m3<2 * 128, kCols>() : idesc_bf16<2 * 128, kCols>();
    int stage = 0;
    uint32_t phase = 0, tphase = 0;
    bool ok = true;
    if (leader) {
      for (int tile = first_tile; ok && tile < num_tiles; tile += tile_step) {
        if (lane == 0) ok = wait_ready(tempty_bar, tphase ^ 1u, abort_flag, g.err);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        tc_fence_after();
        for (int kb = 0; kb < num_kb; ++kb) {
          if (lane == 0) ok = wait_ready(full_bar(stage), phase, abort_flag, g.err);
          ok = __shfl_sync(0xffffffffu, ok, 0);
          if (!ok) break;
          tc_fence_after();
          if (lane == 0) {
            const uint64_t a0 = sw128_desc(sA + stage * A_BYTES);
            const uint64_t a1 = sw128_desc(sA + stage * A_BYTES + A_BYTES / 2);  // rows 128-255
            const uint64_t bd = sw128_desc(sB + stage * B_BYTES);
#pragma unroll
            for (int k = 0; k < kMmaPerStage; ++k) {
              // 32 bytes of K per MMA: +2 in the descriptor's 16-byte address units
              const uint32_t accum = (kb | k) != 0;
              if (F8) {
                umma_e4m3_pair(tmem_base, a0 + 2u * k, bd + 2u * k, idesc, accum);
                umma_e4m3_pair(tmem_base + kCols, a1 + 2u * k, bd + 2u * k, idesc, accum);
              } else {
                umma_bf16_pair(tmem_base, a0 + 2u * k, bd + 2u * k, idesc, accum);
                umma_bf16_pair(tmem_base + kCols, a1 + 2u * k, bd + 2u * k, idesc, accum);
              }
            }
            umma_commit_pair_both(empty_bar(stage));  // slot free in both CTAs
          }
          __syncwarp();
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        if (lane == 0) umma_commit_pair_both(tfull_bar);  // tile complete in both CTAs
        __syncwarp();
        tphase ^= 1u;
      }
      if (lane == 0) {
        umma_commit_pair_local(drain_bar);  // arrives once every MMA above has finished
        wait_drain(drain_bar, 0);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    // the key phase's partial sums are complete (and h no longer read by it)
    if (PHASE >= 1) griddep_wait();
    const int quarter = warp & 3, half = warp >> 2;
    const int wrow0 = half * 128 + quarter * 32;  // first tile row of this warp
    const int r = wrow0 + lane;                   // tile row of this thread
    int hslot = 0;
    uint32_t hphase = 0, tphase = 0, wphase = 0;
    bool ok = true;
    const int tiles_per_branch = d / g.key_tile;
    constexpr int NQ = kCols / H_COLS;  // 32-column chunks per tile
    for (int tile = first_tile; ok && tile < num_tiles; tile += tile_step) {
      const int m_blk = tile / num_n, n_blk = tile - m_blk * num_n;
      const int row0 = m_blk * 2 * kRows + (int)rank * kRows;  // first row of this CTA
      const int row = row0 + r;
      const bool valid = row < R;
      const int n0 = n_blk * kCols;
      const float se = F8 && valid ? __ldg(g.s_row + row) : 1.f;  // e's row scale
      float al[kMaxBranches];
      if (PHASE >= 1) {
        // alpha from the key phase's per-tile partial sums (Eq. 4 / Eq. 6);
        // computed while the MMAs of this tile run
#pragma unroll
        for (int mb = 0; mb < kMaxBranches; ++mb) {
          al[mb] = 0.f;
          if (mb < M && valid) {
            if (g.alpha_in) {
              al[mb] = g.alpha_in[(int64_t)row * M + mb];
            } else {
              al[mb] = row_alpha<1>(g.partials, R, row, mb, tiles_per_branch, d, g.eps, g.inv_sqrt_d);
              if (g.alpha && n_blk == 0) g.alpha[(int64_t)row * M + mb] = al[mb];
            }
          }
        }
      }
      if (lane == 0) ok = wait_ready(tfull_bar, tphase, abort_flag, g.err);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      tc_fence_after();
      const uint32_t taddr =
          tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(half * kCols);
      // two register sets: chunk q+1 loads from TMEM while chunk q is used
      static_assert(NQ % 2 == 0, "chunks are processed in pairs");
      uint32_t va[32], vb[32];
      __syncwarp();
      tmem_ld32_async(taddr, va);
      if (PHASE == 0) {
        if (lane == 0) ok = wait_ready(wfull_bar, wphase, abort_flag, g.err);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        wphase ^= 1u;
        float skk = 0.f, shk = 0.f, shh = 0.f;
        // one 32-column chunk: v holds it (loaded), vn receives chunk q+1
        auto key_chunk = [&](int q, uint32_t(&v)[32], uint32_t(&vn)[32]) {
          tmem_wait32(v);
          __syncwarp();
          if (q + 1 < NQ) {
            tmem_ld32_async(taddr + (q + 1) * H_COLS, vn);
          } else {
            // every TMEM read of this tile is done: the accumulators are free
            // for the next tile's MMAs (the leader owns the barrier)
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_remote(peer_addr(tempty_bar, 0));
          }
          if (F8) dequant_chunk<false>(v, g.s_col + n0 + q * H_COLS, 0.f);
          if (lane == 0) ok = wait_ready(hfull_bar(hslot), hphase, abort_flag, g.err);
          ok = __shfl_sync(0xffffffffu, ok, 0);
          if (!ok) return;
          const uint8_t* hs = hbuf + hslot * H_BYTES;
          const float4* wp = reinterpret_cast<const float4*>(wbuf + q * H_COLS);
          uint4 hu[4];
          float4 wv[8];
#pragma unroll
          for (int c = 0; c < 4; ++c) hu[c] = *reinterpret_cast<const uint4*>(hs + sw64_off(r, c));
#pragma unroll
          for (int c = 0; c < 8; ++c) wv[c] = wp[c];
          // packed fp32 pairs, two accumulators per sum: four chains each
          unsigned long long akk[2] = {0ull, 0ull}, ahh[2] = {0ull, 0ull}, ahk[2] = {0ull, 0ull};
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const uint32_t hw[4] = {hu[c].x, hu[c].y, hu[c].z, hu[c].w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const int e = c * 8 + 2 * j;  // elements e, e+1 of the chunk
              const unsigned long long h2 = bf16x2_to_f2(hw[j]);
              const unsigned long long k2 = f2_pack(v[e], v[e + 1]);
              const float4 wq = wv[(c * 8 + 2 * j) / 4];
              const unsigned long long w2 =
                  (j & 1) ? f2_pack(__float_as_uint(wq.z), __float_as_uint(wq.w))
                          : f2_pack(__float_as_uint(wq.x), __float_as_uint(wq.y));
              akk[j & 1] = f2_fma(k2, k2, akk[j & 1]);
              ahh[j & 1] = f2_fma(h2, h2, ahh[j & 1]);
              ahk[j & 1] = f2_fma(f2_mul(h2, w2), k2, ahk[j & 1]);
            }
          }
          const float2 kk0 = f2_unpack(akk[0]), kk1 = f2_unpack(akk[1]);
          const float2 hh0 = f2_unpack(ahh[0]), hh1 = f2_unpack(ahh[1]);
          const float2 hk0 = f2_unpack(ahk[0]), hk1 = f2_unpack(ahk[1]);
          skk += (kk0.x + kk0.y) + (kk1.x + kk1.y);
          shh += (hh0.x + hh0.y) + (hh1.x + hh1.y);
          shk += (hk0.x + hk0.y) + (hk1.x + hk1.y);
          __syncwarp();
          if (lane == 0) mbar_arrive(hempty_bar(hslot));
          if (++hslot == H_SLOTS) {
            hslot = 0;
            hphase ^= 1u;
          }
        };
#pragma unroll 1
        for (int q = 0; ok && q < NQ; q += 2) {
          key_chunk(q, va, vb);
          if (ok) key_chunk(q + 1, vb, va);
        }
        if (!ok) break;
        // the weight buffer is free again; then the partial sums go out
        __syncwarp();
        if (lane == 0) mbar_arrive(wempty_bar);
        if (F8) {  // k = se * (the column-scaled accumulator)
          skk *= se * se;
          shk *= se;
        }
        if (valid) g.partials[(int64_t)n_blk * R + row] = make_float4(skk, shk, shh, 0.f);
      } else if (PHASE == 3) {
        // values for the short convolution (Eq. 5): v in fp32 and the row's
        // sum of v^2 over this tile; the conv kernel forms alpha v from them.
        // Each warp stages its 32 rows x 32 columns (4 KB, 128-byte swizzle)
        // in one of two buffers and stores them by TMA (map_out covers v).
        float svv = 0.f;
        uint8_t* stage0 = hbuf + warp * 8192;
        int sbuf = 0;
        auto vals_chunk = [&](int q, uint32_t(&v)[32], uint32_t(&vn)[32]) {
          tmem_wait32(v);
          __syncwarp();
          if (q + 1 < NQ) {
            tmem_ld32_async(taddr + (q + 1) * H_COLS, vn);
          } else {
            tc_fence_before();  // last TMEM read done: release the accumulators
            __syncwarp();
            if (lane == 0) mbar_arrive_remote(peer_addr(tempty_bar, 0));
          }
          if (F8) dequant_chunk<true>(v, g.s_col + n0 + q * H_COLS, se);
          unsigned long long s2[2] = {0ull, 0ull};
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            const unsigned long long v2 = f2_pack(v[e], v[e + 1]);
            s2[(e >> 1) & 1] = f2_fma(v2, v2, s2[(e >> 1) & 1]);
          }
          const float2 s0 = f2_unpack(s2[0]), s1 = f2_unpack(s2[1]);
          svv += (s0.x + s0.y) + (s1.x + s1.y);
          // the buffer's previous store has finished reading it
          if (lane == 0) asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
          __syncwarp();
          uint8_t* st = stage0 + sbuf * 4096;
#pragma unroll
          for (int c = 0; c < 8; ++c)
            *reinterpret_cast<uint4*>(st + sw128_off(lane, c)) =
                make_uint4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
          fence_async_smem();
          __syncwarp();
          if (lane == 0) {
            if (row0 + wrow0 < R)
              tma_store_2d(&map_out, smem_u32(st), n0 + q * H_COLS, row0 + wrow0);
            else
              asm volatile("cp.async.bulk.commit_group;" ::: "memory");
          }
          sbuf ^= 1;
        };
#pragma unroll 1
        for (int q = 0; q < NQ; q += 2) {
          vals_chunk(q, va, vb);
          vals_chunk(q + 1, vb, va);
        }
        if (valid) g.vv[(int64_t)n_blk * R + row] = svv;
      } else if (PHASE == 2 && !F8 && M == 1) {
        // out aliases h, one branch (bf16 operands; the E4M3 form takes the
        // general path below): the whole tile leaves TMEM before any
        // reduce-add is issued.  bf16(alpha v) of chunks 0-3 (columns 0-127)
        // is staged in the warp's two 4 KB buffers and that of chunks 4-7 kept
        // packed in registers; the accumulators are released, then the four
        // 32 x 64 reduce-adds go out (the last two once the first two have
        // read their buffers) while the next tile's MMAs run.
        uint8_t* stage0 = hbuf + warp * 8192;
        const float a = al[0];
        const unsigned long long a2 = f2_pack(__float_as_uint(a), __float_as_uint(a));
        uint32_t keep[2][32];
        // the previous tile's reduces have read the buffers
        if (lane == 0) asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
        __syncwarp();
        tmem_ld32_async(taddr + H_COLS, vb);  // chunk 1 (chunk 0 is on its way into va)
#pragma unroll
        for (int p = 0; p < NQ / 2; ++p) {
          const int q = 2 * p;
          tmem_wait32(va);
          tmem_wait32(vb);
          __syncwarp();
          uint32_t ow[32];
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const uint32_t* v = c < 4 ? va : vb;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const int e = (c & 3) * 8 + 2 * j;
              const float2 o = f2_unpack(f2_mul(a2, f2_pack(v[e], v[e + 1])));
              ow[4 * c + j] = pack2(o.x, o.y);
            }
          }
          if (g.delta && valid) {
            float4* dp = reinterpret_cast<float4*>(g.delta + (int64_t)row * d + n0 + q * H_COLS);
#pragma unroll
            for (int c = 0; c < 16; ++c) {
              const uint32_t* v = c < 8 ? va : vb;
              const int e = (c & 7) * 4;
              dp[c] = make_float4(a * __uint_as_float(v[e]), a * __uint_as_float(v[e + 1]),
                                  a * __uint_as_float(v[e + 2]), a * __uint_as_float(v[e + 3]));
            }
          }
          __syncwarp();
          if (q + 2 < NQ) {
            tmem_ld32_async(taddr + (q + 2) * H_COLS, va);
            tmem_ld32_async(taddr + (q + 3) * H_COLS, vb);
          } else {
            tc_fence_before();  // last TMEM read done: release the accumulators
            __syncwarp();
            if (lane == 0) mbar_arrive_remote(peer_addr(tempty_bar, 0));
          }
          if (p < 2) {
            uint8_t* st = stage0 + p * 4096;
#pragma unroll
            for (int c = 0; c < 8; ++c)
              *reinterpret_cast<uint4*>(st + sw128_off(lane, c)) =
                  make_uint4(ow[4 * c], ow[4 * c + 1], ow[4 * c + 2], ow[4 * c + 3]);
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) keep[p - 2][i] = ow[i];
          }
        }
        // a warp whose rows all lie past R commits empty groups instead
        const bool any = row0 + wrow0 < R;
        fence_async_smem();
        __syncwarp();
        if (lane == 0) {
#pragma unroll
          for (int b = 0; b < 2; ++b) {
            if (any)
              tma_reduce_add_2d(&map_out, smem_u32(stage0 + b * 4096), n0 + b * 2 * H_COLS,
                                row0 + wrow0);
            else
              asm volatile("cp.async.bulk.commit_group;" ::: "memory");
          }
        }
#pragma unroll
        for (int b = 0; b < 2; ++b) {
          // buffer b has been read by its first reduce (the other may be pending)
          if (lane == 0) asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
          __syncwarp();
          uint8_t* st = stage0 + b * 4096;
#pragma unroll
          for (int c = 0; c < 8; ++c)
            *reinterpret_cast<uint4*>(st + sw128_off(lane, c)) =
                make_uint4(keep[b][4 * c], keep[b][4 * c + 1], keep[b][4 * c + 2], keep[b][4 * c + 3]);
          fence_async_smem();
          __syncwarp();
          if (lane == 0) {
            if (any)
              tma_reduce_add_2d(&map_out, smem_u32(st), n0 + (2 + b) * 2 * H_COLS, row0 + wrow0);
            else
              asm volatile("cp.async.bulk.commit_group;" ::: "memory");
          }
        }
      } else if (PHASE == 2) {
        // out aliases h, several branches: add bf16(alpha_m v) into each
        // branch with TMA reduce-add, two 32-column chunks per operation (32
        // rows x 64 columns, 4 KB, 128-byte swizzle); each warp stages in one
        // of two buffers (the h ring is unused in this phase)
        uint8_t* stage0 = hbuf + warp * 8192;
        int sbuf = 0;
        __syncwarp();
        tmem_ld32_async(taddr + H_COLS, vb);  // chunk 1 (chunk 0 is on its way into va)
#pragma unroll 1
        for (int q = 0; q < NQ; q += 2) {
          tmem_wait32(va);
          tmem_wait32(vb);
          __syncwarp();
          if (F8) {
            dequant_chunk<false>(va, g.s_col + n0 + q * H_COLS, 0.f);
            dequant_chunk<false>(vb, g.s_col + n0 + (q + 1) * H_COLS, 0.f);
          }
          if (q + 2 >= NQ) {
            tc_fence_before();  // last TMEM read done: release the accumulators
            __syncwarp();
            if (lane == 0) mbar_arrive_remote(peer_addr(tempty_bar, 0));
          }
#pragma unroll 1
          for (int mb = 0; mb < M; ++mb) {
            float a = 0.f;
#pragma unroll
            for (int b = 0; b < kMaxBranches; ++b)
              if (b == mb) a = al[b];
            if (F8) a *= se;  // alpha v = (alpha se) (the column-scaled accumulator)
            const unsigned long long a2 = f2_pack(__float_as_uint(a), __float_as_uint(a));
            // the buffer's previous reduce has finished reading it
            if (lane == 0) asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
            __syncwarp();
            uint8_t* st = stage0 + sbuf * 4096;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              const uint32_t* v = c < 4 ? va : vb;
              uint32_t ow[4];
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                const int e = (c & 3) * 8 + 2 * j;
                const float2 o = f2_unpack(f2_mul(a2, f2_pack(v[e], v[e + 1])));
                ow[j] = pack2(o.x, o.y);
              }
              *reinterpret_cast<uint4*>(st + sw128_off(lane, c)) =
                  make_uint4(ow[0], ow[1], ow[2], ow[3]);
            }
            if (g.delta && valid) {
              float4* dp = reinterpret_cast<float4*>(g.delta + ((int64_t)row * M + mb) * d + n0 +
                                                     q * H_COLS);
#pragma unroll
              for (int c = 0; c < 16; ++c) {
                const uint32_t* v = c < 8 ? va : vb;
                const int e = (c & 7) * 4;
                dp[c] = make_float4(a * __uint_as_float(v[e]), a * __uint_as_float(v[e + 1]),
                                    a * __uint_as_float(v[e + 2]), a * __uint_as_float(v[e + 3]));
              }
            }
            if (mb == M - 1 && q + 2 < NQ) {
              // both register sets are staged: fetch the next two chunks now
              __syncwarp();
              tmem_ld32_async(taddr + (q + 2) * H_COLS, va);
              tmem_ld32_async(taddr + (q + 3) * H_COLS, vb);
            }
            fence_async_smem();
            __syncwarp();
            if (lane == 0) {
              if (row0 + wrow0 < R)
                tma_reduce_add_2d(&map_out, smem_u32(st), mb * d + n0 + q * H_COLS, row0 + wrow0);
              else
                asm volatile("cp.async.bulk.commit_group;" ::: "memory");
            }
            sbuf ^= 1;
          }
        }
      } else {
        int pending = -1;  // slot whose TMA store may still be reading it
        auto value_chunk = [&](int q, uint32_t(&v)[32], uint32_t(&vn)[32]) {
          tmem_wait32(v);
          __syncwarp();
          if (q + 1 < NQ) {
            tmem_ld32_async(taddr + (q + 1) * H_COLS, vn);
          } else {
            tc_fence_before();  // last TMEM read done: release the accumulators
            __syncwarp();
            if (lane == 0) mbar_arrive_remote(peer_addr(tempty_bar, 0));
          }
          if (F8) dequant_chunk<false>(v, g.s_col + n0 + q * H_COLS, 0.f);
#pragma unroll 1
          for (int mb = 0; mb < M; ++mb) {
            if (lane == 0) ok = wait_ready(hfull_bar(hslot), hphase, abort_flag, g.err);
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) return;
            uint8_t* hs = hbuf + hslot * H_BYTES;
            float a = 0.f;
#pragma unroll
            for (int b = 0; b < kMaxBranches; ++b)
              if (b == mb) a = al[b];
            if (F8) a *= se;  // alpha v = (alpha se) (the column-scaled accumulator)
            // out = h + alpha v, written over h in place, then stored by TMA
            const unsigned long long a2 = f2_pack(__float_as_uint(a), __float_as_uint(a));
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              uint4* p = reinterpret_cast<uint4*>(hs + sw64_off(r, c));
              const uint4 hu = *p;
              const uint32_t hw[4] = {hu.x, hu.y, hu.z, hu.w};
              uint32_t ow[4];
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                const int e = c * 8 + 2 * j;
                const float2 o =
                    f2_unpack(f2_fma(a2, f2_pack(v[e], v[e + 1]), bf16x2_to_f2(hw[j])));
                ow[j] = pack2(o.x, o.y);
              }
              *p = make_uint4(ow[0], ow[1], ow[2], ow[3]);
            }
            if (g.delta && valid) {
              float4* dp = reinterpret_cast<float4*>(g.delta + ((int64_t)row * M + mb) * d + n0 +
                                                     q * H_COLS);
#pragma unroll
              for (int c = 0; c < 8; ++c)
                dp[c] = make_float4(a * __uint_as_float(v[4 * c]), a * __uint_as_float(v[4 * c + 1]),
                                    a * __uint_as_float(v[4 * c + 2]),
                                    a * __uint_as_float(v[4 * c + 3]));
            }
            fence_async_smem();  // generic-proxy writes -> visible to the TMA store
            __syncwarp();
            if (lane == 0) {
              // this warp's 32 rows of the slot; rows past R are clipped, and a
              // warp whose rows all lie past R commits an empty group instead
              if (row0 + wrow0 < R)
                tma_store_2d(&map_out, sH + hslot * H_BYTES + wrow0 * (H_COLS * 2),
                             mb * d + n0 + q * H_COLS, row0 + wrow0);
              else
                asm volatile("cp.async.bulk.commit_group;" ::: "memory");
              // release the previous slot once its store has read it
              asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
              if (pending >= 0) mbar_arrive(hempty_bar(pending));
            }
            pending = hslot;
            if (++hslot == H_SLOTS) {
              hslot = 0;
              hphase ^= 1u;
            }
          }
        };
#pragma unroll 1
        for (int q = 0; ok && q < NQ; q += 2) {
          value_chunk(q, va, vb);
          if (ok) value_chunk(q + 1, vb, va);
        }
        if (!ok) break;
        __syncwarp();
        if (lane == 0) {
          asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
          if (pending >= 0) mbar_arrive(hempty_bar(pending));
        }
      }
      tphase ^= 1u;
    }
    if (PHASE >= 1 && lane == 0) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
  }

  tc_fence_before();
  __syncthreads();
  // neither CTA leaves while its partner may still read its shared memory (the
  // leader's MMAs) or signal its barriers (the follower's arrivals)
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

template <int PHASE, bool F8>
cudaError_t launch_wide(const ProjMaps& maps, const GateArgs& g, int grid, cudaStream_t stream) {
  auto kern = proj_gate_wide_kernel<PHASE, F8>;
  cudaError_t e =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t lc = {};
  lc.gridDim = dim3(grid);
  lc.blockDim = dim3(kThreads);
  lc.dynamicSmemBytes = SMEM;
  lc.stream = stream;
  cudaLaunchAttribute at[2];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = 2;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[1].val.programmaticStreamSerializationAllowed = 1;
  lc.attrs = at;
  lc.numAttrs = g.pdl ? 2 : 1;
  e = cudaLaunchKernelEx(&lc, kern, maps.e, maps.w, maps.h, maps.out, g);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_proj_gate_wide(int phase, const ProjMaps& maps, const GateArgs& g, int grid,
                                  cudaStream_t stream, bool f8) {
  if (g.R == 0) return cudaSuccess;
  if (grid < 2 || (grid & 1)) return cudaErrorInvalidValue;
  if (f8 && (!g.s_row || !g.s_col)) return cudaErrorInvalidValue;
  switch (phase * 2 + (f8 ? 1 : 0)) {
    case 0: return launch_wide<0, false>(maps, g, grid, stream);
    case 1: return launch_wide<0, true>(maps, g, grid, stream);
    case 2: return launch_wide<1, false>(maps, g, grid, stream);
    case 3: return launch_wide<1, true>(maps, g, grid, stream);
    case 4: return launch_wide<2, false>(maps, g, grid, stream);
    case 5: return launch_wide<2, true>(maps, g, grid, stream);
    case 6: return launch_wide<3, false>(maps, g, grid, stream);
    case 7: return launch_wide<3, true>(maps, g, grid, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace engram
