// bf16 projection + context-aware gate on CTA pairs with 256-row tiles and
// accumulators double-buffered in TMEM: the path for few rows and many
// columns (decode keys: 256 rows, M d = 10 240 columns).
//
// Same computation as k_proj_gate_sm100.cu ("Conditional Memory via Scalable
// Lookup", section 2.3 Eq. (3)-(4), section 2.4 Eq. (6)); only the tiling
// differs.  A cluster of two CTAs on one TPC computes a 256 x 256 tile of
// e . W^T with tcgen05.mma.cta_group::2 (M = 256, N = 256 per instruction):
// CTA rank r loads rows [128 r, 128 r + 128) of the tile's e rows and rows
// [128 r, 128 r + 128) of its 256 W rows (the pair's B operand is split by
// N), so every W row is read once per 256 rows of e and each CTA streams
// 256 rows of K per tile (single-CTA tiles of the same width stream 384).
// Each CTA's 128 x 256 fp32 accumulator fills 256 TMEM columns, so two tiles
// fit in the 512 columns and the gate epilogue of one tile overlaps the MMAs
// of the next.
//
// Roles (352 threads per CTA):
//   warps 0-7   epilogue: warp w reads TMEM lanes 32 (w % 4).. (tile row
//               32 (w % 4) + lane) and the 128 columns [128 (w / 4), +128),
//               in four 32-column chunks;
//   warp 8      TMA producer of e and W (4 stages x 32 KB);
//   warp 9      TMEM allocator; MMA issuer on the leader (rank 0);
//   warp 10     TMA producer of h sub-tiles [128 rows x 32 columns, 64-byte
//               swizzle] into a 10-slot ring, and of the key epilogue's
//               column weights w_q * w_k (double-buffered with the tiles).
// Phases: 0 = keys (partial sums per 128-column half tile), 1 = values
// (out = h + alpha v, written over h in its ring slot and stored by TMA),
// 2 = values when out aliases h (bf16(alpha v) staged per warp, 32 x 64 at a
// time, and added into out with a TMA reduce-add: RN(h + RN(alpha v))
// instead of RN(h + alpha v)).
// Every wait is bounded (kWaitLimitNs); on expiry the CTA raises its abort
// flag and kDevErrTimeout, every role leaves its loop, and the pair leaves
// together through a bounded handshake before TMEM is freed (cta_group::2).
#include "sm100_ptx.cuh"

namespace engram {

namespace {

using namespace sm100;

constexpr int kRows = 128;                           // tile rows per CTA
constexpr int kCols = 256;                           // tile columns
constexpr int kHalf = kCols / 2;                     // columns per epilogue warp
constexpr int BK = 64;
constexpr uint32_t A_BYTES = kRows * BK * 2;         // 16 KB
constexpr uint32_t B_BYTES = (kCols / 2) * BK * 2;   // 16 KB: this CTA's half of B
constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES;  // 32 KB
constexpr int STAGES = 4;
constexpr int H_SLOTS = 10;
constexpr int H_COLS = 32;
constexpr uint32_t H_BYTES = kRows * H_COLS * 2;     // 8 KB
constexpr int kEpiWarps = 8;
constexpr int kThreads = (kEpiWarps + 3) * 32;       // 352
constexpr int kProducerWarp = kEpiWarps, kMmaWarp = kEpiWarps + 1, kHWarp = kEpiWarps + 2;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t ACC_COLS = kCols;                 // one accumulator buffer
constexpr uint32_t W_BYTES = kCols * 4;              // one tile's w_q * w_k (fp32)
constexpr int NQ = kHalf / H_COLS;                   // 32-column chunks per warp and tile
constexpr int NUM_BARS = 2 * STAGES + 4 + 2 * H_SLOTS + 4 + 2;
constexpr size_t SMEM = 1024 + (size_t)STAGES * STAGE_BYTES + (size_t)H_SLOTS * H_BYTES +
                        2 * W_BYTES + 8 * NUM_BARS + 16;
static_assert(SMEM <= 232448, "shared memory budget");
static_assert(kEpiWarps * 8192 <= H_SLOTS * H_BYTES, "in-place staging fits in the h ring");
static_assert(NQ % 2 == 0, "chunks are processed in pairs");

// Column offset, within the [R, M*d] view of h, of ring entry i of a tile
// starting at column n0: entries run over (chunk j, branch mb) with j the
// slower index; chunk j covers columns 128 (j % 2) + 32 (j / 2) of the tile,
// so entries of the two column halves alternate.
__device__ __forceinline__ int h_entry_col(int i, int M, int d, int n0, bool key) {
  const int j = key ? i : i / M;
  const int mb = key ? 0 : i - j * M;
  return mb * d + n0 + kHalf * (j & 1) + H_COLS * (j >> 1);
}

template <int PHASE>
__global__ void __launch_bounds__(kThreads, 1)
    proj_gate_pair_kernel(const __grid_constant__ CUtensorMap map_e,
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
  uint64_t* bars =
      reinterpret_cast<uint64_t*>(hbuf + (size_t)H_SLOTS * H_BYTES + 2 * W_BYTES);
  const uint32_t bar0 = smem_u32(bars);
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (STAGES + s); };
  auto tfull_bar = [&](int b) { return bar0 + 8u * (2 * STAGES + b); };
  auto tempty_bar = [&](int b) { return bar0 + 8u * (2 * STAGES + 2 + b); };
  auto hfull_bar = [&](int s) { return bar0 + 8u * (2 * STAGES + 4 + s); };
  auto hempty_bar = [&](int s) { return bar0 + 8u * (2 * STAGES + 4 + H_SLOTS + s); };
  auto wfull_bar = [&](int b) { return bar0 + 8u * (2 * STAGES + 4 + 2 * H_SLOTS + b); };
  auto wempty_bar = [&](int b) { return bar0 + 8u * (2 * STAGES + 6 + 2 * H_SLOTS + b); };
  const uint32_t drain_bar = bar0 + 8u * (2 * STAGES + 8 + 2 * H_SLOTS);
  const uint32_t pair_bar = drain_bar + 8u;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + NUM_BARS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();  // 0 = the pair's MMA leader
  const bool leader = rank == 0;
  const int R = g.R, d = g.d, M = g.M;
  const int n_total = PHASE == 0 ? M * d : d;
  const int num_n = n_total / kCols;
  const int num_tiles = ((R + 2 * kRows - 1) / (2 * kRows)) * num_n;
  const int num_kb = (g.d_mem + BK - 1) / BK;
  const int first_tile = (int)(blockIdx.x >> 1), tile_step = (int)(gridDim.x >> 1);
  // h ring entries per tile: the tile's 256 columns of one branch for keys,
  // of every branch for values (v is shared across branches, Eq. 6); none
  // when the values are added into h in place
  const int nsub = PHASE == 2 ? 0 : (kCols / H_COLS) * (PHASE == 0 ? 1 : M);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(tfull_bar(b), 1);
      mbar_init(tempty_bar(b), 2 * kEpiWarps);  // every epilogue warp of the pair
      mbar_init(wfull_bar(b), 1);
      mbar_init(wempty_bar(b), kEpiWarps);
    }
    for (int s = 0; s < H_SLOTS; ++s) {
      mbar_init(hfull_bar(s), 1);
      mbar_init(hempty_bar(s), kEpiWarps / 2);  // the four warps of one column half
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
          tma_load_2d_pair(sA + stage * A_BYTES, &map_e, fb, kb * BK, a_row);
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
    // --------------------------------------------- h sub-tile and w producer
    if (lane == 0) asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&map_h) : "memory");
    // h may still be written by the kernel before the previous kernel
    if (PHASE == 0) griddep_wait();
    int slot = 0;
    uint32_t phase = 0;
    bool ok = true;
    int tix = 0;
    const int nbox = (kCols / H_COLS) * (PHASE == 0 ? 1 : M);  // h boxes of a tile
    for (int tile = first_tile; ok && tile < num_tiles; tile += tile_step, ++tix) {
      const int m_blk = tile / num_n, n0 = (tile - m_blk * num_n) * kCols;
      const int row0 = m_blk * 2 * kRows + (int)rank * kRows;
      const int b = tix & 1;
      const uint32_t use = (uint32_t)(tix >> 1);
      if (PHASE == 2) {
        // values added in place read-modify-write h in L2: bring the tile's
        // h into L2 while its MMAs run, once the previous tile's MMAs are done
        // (the ring-less phase has nothing else to pace this warp)
        if (tix > 0) {
          const int pb = (tix - 1) & 1;
          if (lane == 0)
            ok = wait_ready(tfull_bar(pb), (uint32_t)((tix - 1) >> 1) & 1u, abort_flag, g.err);
          ok = __shfl_sync(0xffffffffu, ok, 0);
          if (!ok) break;
        }
        if (lane == 0 && row0 < R)
          for (int i = 0; i < nbox; ++i)
            tma_prefetch_l2_2d(&map_h, h_entry_col(i, M, d, n0, false), row0);
        __syncwarp();
        continue;
      }
      if (lane == 0 && row0 < R)  // boxes beyond the ring (several branches)
        for (int i = H_SLOTS; i < nsub; ++i)
          tma_prefetch_l2_2d(&map_h, h_entry_col(i, M, d, n0, PHASE == 0), row0);
      if (PHASE == 0) {
        // the key epilogue's column weights: w_qk[n0 .. n0+256) of [M*d]
        if (lane == 0) ok = wait_ready(wempty_bar(b), (use & 1u) ^ 1u, abort_flag, g.err);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        if (lane == 0) {
          mbar_expect_tx(wfull_bar(b), W_BYTES);
          bulk_load(sW + b * W_BYTES, g.w_qk + n0, W_BYTES, wfull_bar(b));
        }
        __syncwarp();
      }
      for (int i = 0; i < nsub; ++i) {
        if (lane == 0) ok = wait_ready(hempty_bar(slot), phase ^ 1u, abort_flag, g.err);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        if (lane == 0) {
          mbar_expect_tx(hfull_bar(slot), H_BYTES);
          tma_load_2d(sH + slot * H_BYTES, &map_h, hfull_bar(slot),
                      h_entry_col(i, M, d, n0, PHASE == 0), row0);
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
    constexpr uint32_t idesc = idesc_bf16<2 * kRows, kCols>();
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    if (leader) {
      int tix = 0;
      for (int tile = first_tile; ok && tile < num_tiles; tile += tile_step, ++tix) {
        const int b = tix & 1;
        const uint32_t use = (uint32_t)(tix >> 1);
        if (lane == 0) ok = wait_ready(tempty_bar(b), (use & 1u) ^ 1u, abort_flag, g.err);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        tc_fence_after();
        const uint32_t acc = tmem_base + (uint32_t)b * ACC_COLS;
        for (int kb = 0; kb < num_kb; ++kb) {
          if (lane == 0) ok = wait_ready(full_bar(stage), phase, abort_flag, g.err);
          ok = __shfl_sync(0xffffffffu, ok, 0);
          if (!ok) break;
          tc_fence_after();
          if (lane == 0) {
            const uint64_t ad = sw128_desc(sA + stage * A_BYTES);
            const uint64_t bd = sw128_desc(sB + stage * B_BYTES);
#pragma unroll
            for (int k = 0; k < BK / 16; ++k)
              umma_bf16_pair(acc, ad + 2u * k, bd + 2u * k, idesc, (kb | k) != 0);
            umma_commit_pair_both(empty_bar(stage));  // slot free in both CTAs
          }
          __syncwarp();
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        if (lane == 0) umma_commit_pair_both(tfull_bar(b));  // tile complete in both CTAs
        __syncwarp();
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
    const int quarter = warp & 3, colhalf = warp >> 2;
    const int r = quarter * 32 + lane;  // tile row of this thread (within the CTA)
    uint32_t hpos = 0;                  // ring position of the tile's first entry
    bool ok = true;
    const int tiles_per_branch = d / g.key_tile;
    int pending = -1;  // phase 1: slot whose TMA store may still be reading it
    int sbuf = 0;      // phase 2: staging buffer
    int tix = 0;
    for (int tile = first_tile; ok && tile < num_tiles; tile += tile_step, ++tix) {
      const int m_blk = tile / num_n, n_blk = tile - m_blk * num_n;
      const int row0 = m_blk * 2 * kRows + (int)rank * kRows;  // first row of this CTA
      const int row = row0 + r;
      const bool valid = row < R;
      const bool rows_in = row0 + quarter * 32 < R;  // this warp has a row inside R
      const int n0 = n_blk * kCols;
      const int b = tix & 1;
      const uint32_t use = (uint32_t)(tix >> 1);
      float al[kMaxBranches];
      if (PHASE >= 1) {
        // alpha from the key phase's per-tile partial sums (Eq. 4 / Eq. 6);
        // computed while this tile's MMAs run
#pragma unroll
        for (int mb = 0; mb < kMaxBranches; ++mb) {
          al[mb] = 0.f;
          if (mb < M && valid) {
            if (g.alpha_in) {
              al[mb] = g.alpha_in[(int64_t)row * M + mb];
            } else {
              al[mb] = row_alpha<1>(g.partials, R, row, mb, tiles_per_branch, d, g.eps, g.inv_sqrt_d);
              if (g.alpha && n_blk == 0 && colhalf == 0) g.alpha[(int64_t)row * M + mb] = al[mb];
            }
          }
        }
      }
      if (lane == 0) ok = wait_ready(tfull_bar(b), use & 1u, abort_flag, g.err);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      tc_fence_after();
      const uint32_t taddr = tmem_base + ((uint32_t)(quarter * 32) << 16) +
                             (uint32_t)b * ACC_COLS + (uint32_t)(colhalf * kHalf);
      const int c0 = n0 + colhalf * kHalf;  // first column of this warp in the tile
      // two register sets: chunk q+1 loads from TMEM while chunk q is used;
      // after the last load the buffer goes back to the MMA issuer
      uint32_t va[32], vb[32];
      auto next_chunk = [&](int q, uint32_t(&v)[32], uint32_t(&vn)[32]) {
        tmem_wait32(v);
        __syncwarp();
        if (q + 1 < NQ) {
          tmem_ld32_async(taddr + (q + 1) * H_COLS, vn);
        } else {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive_remote(peer_addr(tempty_bar(b), 0));
        }
      };
      // ring slot and parity of this tile's entry i
      auto ring = [&](int i, int& slot, uint32_t& par) {
        const uint32_t pos = hpos + (uint32_t)i;
        slot = (int)(pos % H_SLOTS);
        par = (pos / H_SLOTS) & 1u;
      };
      __syncwarp();
      tmem_ld32_async(taddr, va);
      if (PHASE == 0) {
        if (lane == 0) ok = wait_ready(wfull_bar(b), use & 1u, abort_flag, g.err);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        float skk = 0.f, shk = 0.f, shh = 0.f;
        const float* wcol = wbuf + b * kCols + colhalf * kHalf;
        auto key_chunk = [&](int q, uint32_t(&v)[32], uint32_t(&vn)[32]) {
          next_chunk(q, v, vn);
          int slot;
          uint32_t par;
          ring(2 * q + colhalf, slot, par);
          if (lane == 0) ok = wait_ready(hfull_bar(slot), par, abort_flag, g.err);
          ok = __shfl_sync(0xffffffffu, ok, 0);
          if (!ok) return;
          const uint8_t* hs = hbuf + slot * H_BYTES;
          const float4* wp = reinterpret_cast<const float4*>(wcol + q * H_COLS);
          uint4 hu[4];
          float4 wv[8];
#pragma unroll
          for (int c = 0; c < 4; ++c) hu[c] = *reinterpret_cast<const uint4*>(hs + sw64_off(r, c));
#pragma unroll
          for (int c = 0; c < 8; ++c) wv[c] = wp[c];
          // packed fp32 pairs, two accumulators per sum
          unsigned long long akk[2] = {0ull, 0ull}, ahh[2] = {0ull, 0ull}, ahk[2] = {0ull, 0ull};
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const uint32_t hw[4] = {hu[c].x, hu[c].y, hu[c].z, hu[c].w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const int e = c * 8 + 2 * j;  // elements e, e+1 of the chunk
              const unsigned long long h2 = bf16x2_to_f2(hw[j]);
              const unsigned long long k2 = f2_pack(v[e], v[e + 1]);
              const float4 wq = wv[e / 4];
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
          if (lane == 0) mbar_arrive(hempty_bar(slot));
        };
#pragma unroll 1
        for (int q = 0; ok && q < NQ; q += 2) {
          key_chunk(q, va, vb);
          if (ok) key_chunk(q + 1, vb, va);
        }
        if (!ok) break;
        // the weight buffer is free again; then the partial sums go out
        __syncwarp();
        if (lane == 0) mbar_arrive(wempty_bar(b));
        if (valid)
          g.partials[(int64_t)(n_blk * 2 + colhalf) * R + row] = make_float4(skk, shk, shh, 0.f);
      } else if (PHASE == 2) {
        // out aliases h: add bf16(alpha v) into it with TMA reduce-add, two
        // 32-column chunks per operation (32 rows x 64 columns, 4 KB,
        // 128-byte swizzle); each warp stages in one of two buffers (the h
        // ring is unused in this phase)
        uint8_t* stage0 = hbuf + warp * 8192;
        __syncwarp();
        tmem_ld32_async(taddr + H_COLS, vb);  // chunk 1 (chunk 0 is on its way into va)
#pragma unroll 1
        for (int q = 0; q < NQ; q += 2) {
          tmem_wait32(va);
          tmem_wait32(vb);
          __syncwarp();
          if (q + 2 >= NQ) {
            tc_fence_before();  // last TMEM read done: release the accumulators
            __syncwarp();
            if (lane == 0) mbar_arrive_remote(peer_addr(tempty_bar(b), 0));
          }
#pragma unroll 1
          for (int mb = 0; mb < M; ++mb) {
            float a = 0.f;
#pragma unroll
            for (int bb = 0; bb < kMaxBranches; ++bb)
              if (bb == mb) a = al[bb];
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
              float4* dp = reinterpret_cast<float4*>(g.delta + ((int64_t)row * M + mb) * d + c0 +
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
              if (rows_in)
                tma_reduce_add_2d(&map_out, smem_u32(st), mb * d + c0 + q * H_COLS,
                                  row0 + quarter * 32);
              else
                asm volatile("cp.async.bulk.commit_group;" ::: "memory");
            }
            sbuf ^= 1;
          }
        }
      } else {
        auto value_chunk = [&](int q, uint32_t(&v)[32], uint32_t(&vn)[32]) {
          next_chunk(q, v, vn);
#pragma unroll 1
          for (int mb = 0; mb < M; ++mb) {
            int slot;
            uint32_t par;
            ring((2 * q + colhalf) * M + mb, slot, par);
            if (lane == 0) ok = wait_ready(hfull_bar(slot), par, abort_flag, g.err);
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) return;
            uint8_t* hs = hbuf + slot * H_BYTES;
            float a = 0.f;
#pragma unroll
            for (int bb = 0; bb < kMaxBranches; ++bb)
              if (bb == mb) a = al[bb];
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
              float4* dp = reinterpret_cast<float4*>(g.delta + ((int64_t)row * M + mb) * d + c0 +
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
              if (rows_in)
                tma_store_2d(&map_out, sH + slot * H_BYTES + quarter * 32 * (H_COLS * 2),
                             mb * d + c0 + q * H_COLS, row0 + quarter * 32);
              else
                asm volatile("cp.async.bulk.commit_group;" ::: "memory");
              // release the previous slot once its store has read it
              asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
              if (pending >= 0) mbar_arrive(hempty_bar(pending));
            }
            pending = slot;
          }
        };
#pragma unroll 1
        for (int q = 0; ok && q < NQ; q += 2) {
          value_chunk(q, va, vb);
          if (ok) value_chunk(q + 1, vb, va);
        }
        if (!ok) break;
      }
      hpos += (uint32_t)nsub;
    }
    // a loop left early may still have a TMEM load in flight
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
    if (PHASE == 1 && lane == 0) {
      asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
      if (pending >= 0 && ok) mbar_arrive(hempty_bar(pending));
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

template <int PHASE>
cudaError_t launch_pair(const ProjMaps& maps, const GateArgs& g, int grid, cudaStream_t stream) {
  auto kern = proj_gate_pair_kernel<PHASE>;
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

cudaError_t launch_proj_gate_pair(int phase, const ProjMaps& maps, const GateArgs& g, int grid,
                                  cudaStream_t stream) {
  if (g.R == 0) return cudaSuccess;
  if (grid < 2 || (grid & 1)) return cudaErrorInvalidValue;
  if (phase == 0 && g.key_tile != kHalf) return cudaErrorInvalidValue;
  switch (phase) {
    case 0: return launch_pair<0>(maps, g, grid, stream);
    case 1: return launch_pair<1>(maps, g, grid, stream);
    case 2: return launch_pair<2>(maps, g, grid, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace engram
