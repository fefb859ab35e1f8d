// Steps 5-7 of a short call (at most 256 rows, bf16) in ONE launch: the key
// and value projections, alpha and the residual update, handed between CTAs
// through global counters instead of three dependent launches.
//
// Same computation as k_proj_gate_pair_sm100.cu ("Conditional Memory via
// Scalable Lookup", section 2.3 Eq. (3)-(4), section 2.4 Eq. (6)):
//   k^(m) = W_K^(m) e,  v = W_V e,
//   alpha^(m) = sigmoid(RMSNorm(h^(m)) . RMSNorm(k^(m)) / sqrt(d)),
//   out^(m) = h^(m) + alpha^(m) v.
//
// Grid: clusters of two CTAs (tcgen05 cta_group::2 with M = 256; CTA rank r
// owns rows [128 r, 128 r + 128) of the call), one tile per cluster:
//   clusters [0, nkey)          key tiles: 256 columns [j0, j0 + 256) of
//                               branch mb (nkey = M d / 256).  The CTA loads
//                               its 128 x 256 block of h^(mb) at the start;
//                               while its MMAs run, the epilogue warps form
//                               h w_q w_k into the spare TMEM columns and the
//                               rows' sums of h^2.
//                               Epilogue: the per-row partial sums of Eq. (4)
//                               of each 128-column half tile (the arithmetic
//                               of the 256 x 256 pair kernel's key phase),
//                               stored and counted on the counter of (row
//                               half, branch); once the d / 256 key CTAs of
//                               that counter are done, alpha of its 128 rows
//                               (their partial sums added in the order of
//                               row_alpha, so alpha is bit-identical to that
//                               path); then out = h + alpha v over the staged
//                               h block, v taken from the value CTAs through
//                               global memory, stored by TMA per warp.
//   clusters [nkey, nkey+nval)  value tiles: 128 columns of v (nval = d / 128);
//                               the epilogue writes v (fp32) to a scratch laid
//                               out [2 row halves][d / 4][128 rows][4] (a key
//                               CTA's block of v is then contiguous), counts
//                               itself done on its row half's counter and
//                               leaves.
// Only the key CTAs touch h: each reads and writes its own block, so the
// in-place update (out aliasing h) needs no ordering between CTAs.  The value
// CTAs' mainloops run beside the key CTAs'; the step costs one mainloop, one
// key epilogue, one hand-off among the key CTAs of a branch, alpha, and the
// update of one 64 KB block per key CTA.
//
// Every CTA of the grid must be resident at once (key CTAs wait for each other
// and for the value CTAs): the launcher checks the cluster occupancy, and
// every wait is bounded (kWaitLimitNs; on expiry kDevErrTimeout and the CTA
// leaves).  The counters are zeroed by the last CTA to leave, so consecutive
// launches and graph replays start from zero; a later launch touches them only
// after griddepcontrol.wait, which the gather kernel in between extends to
// this launch's completion.  The launch lets its dependents (the next call's
// gather, which overwrites the e buffer the previous launch read) start only
// after its own griddepcontrol.wait, i.e. after that previous launch ended.
//
// Roles (352 threads per CTA):
//   warps 0-7   epilogue: warp w owns TMEM lanes 32 (w % 4).. (tile rows) and
//               column half w / 4 of the tile;
//   warp 8      TMA producer of e and W (4 stages x 32 KB);
//   warp 9      TMEM allocator; MMA issuer on the leader (rank 0);
//   warp 10     key CTAs: loads of the h block and its column weights
//               w_q * w_k, then (after the mainloop, into the free stage
//               buffers) of the v block once the value CTAs are done.
#include "sm100_ptx.cuh"
#include "sm100_wait.cuh"

namespace engram {

namespace {

using namespace sm100;

constexpr int kRows = 128;                             // tile rows per CTA
constexpr int kKeyCols = 256;                          // key tile columns (pair)
constexpr int kValCols = 128;                          // value tile columns (pair)
constexpr int BK = 64;
constexpr uint32_t A_BYTES = kRows * BK * 2;           // 16 KB
constexpr uint32_t KB_BYTES = (kKeyCols / 2) * BK * 2; // 16 KB: a key CTA's half of B
constexpr uint32_t VB_BYTES = (kValCols / 2) * BK * 2; // 8 KB: a value CTA's half of B
constexpr int STAGES = 4;
constexpr uint32_t STAGE_REGION = STAGES * (A_BYTES + KB_BYTES);  // 128 KB
constexpr int H_COLS = 32;
constexpr uint32_t KH_BOX = kRows * H_COLS * 2;        // 8 KB: 128 rows x 32 columns
constexpr int KH_BOXES = kKeyCols / H_COLS;            // 8
constexpr uint32_t KH_BYTES = KH_BOXES * KH_BOX;       // 64 KB
constexpr uint32_t VT_CHUNK = kRows * 16;              // 2 KB: 4 columns of v, 128 rows
constexpr int VT_CHUNKS = kKeyCols / 4;                // 64 per key tile
constexpr uint32_t W_BYTES = kKeyCols * 4;             // the key tile's w_q * w_k
constexpr int kEpiWarps = 8;
constexpr int kEpiThreads = kEpiWarps * 32;
constexpr int kThreads = kEpiThreads + 3 * 32;         // 352
constexpr int kProducerWarp = kEpiWarps, kMmaWarp = kEpiWarps + 1, kHWarp = kEpiWarps + 2;
constexpr uint32_t TMEM_COLS = 512;  // k (or v) and, in key CTAs, h w_q w_k
constexpr int NQ = (kKeyCols / 2) / H_COLS;            // 32-column chunks per key epilogue warp
constexpr int kSegBatch = 20;                          // partial-sum loads in flight per row
constexpr int NUM_BARS = 2 * STAGES + 5;
constexpr size_t SMEM = 1024 + (size_t)STAGE_REGION + KH_BYTES + W_BYTES + kRows * 4 +
                        8 * NUM_BARS + 16;
static_assert(SMEM <= 232448, "shared memory budget");
static_assert(VT_CHUNKS * VT_CHUNK <= STAGE_REGION, "a key tile's v fits the stages");
static_assert(NQ % 2 == 0, "chunks are processed in pairs");

// Counters in GateArgs::sync: [r * kMaxBranches + mb] key CTAs of row half r
// and branch mb done; [kVCount + r] value CTAs of row half r done; [kExit]
// CTAs that have left.
constexpr int kVCount = 2 * kMaxBranches, kExit = kVCount + 2;

__device__ __forceinline__ void epi_bar_sync() {
  asm volatile("bar.sync 1, %0;" ::"n"(kEpiThreads) : "memory");
}

// Count this CTA done on *p once the epilogue warps' global writes before the
// barrier are visible (barrier, then a gpu-scope fence and the increment).
__device__ __forceinline__ void epi_count_done(unsigned* p) {
  epi_bar_sync();
  if (threadIdx.x == 0) {
    __threadfence();
    atomicAdd(p, 1u);
  }
}

// alpha of one row and branch from its tpb partial sums [segment][R], loads
// in flight kSegBatch at a time (they bypass L1: other CTAs of this launch
// wrote them), added in segment order as row_alpha adds them.
__device__ __forceinline__ float fused_row_alpha(const float4* partials, int64_t R, int64_t row,
                                                 int seg0, int tpb, int d, float eps,
                                                 float inv_sqrt_d) {
  float skk = 0.f, shk = 0.f, shh = 0.f;
  for (int s0 = 0; s0 < tpb; s0 += kSegBatch) {
    float4 p[kSegBatch];
#pragma unroll
    for (int i = 0; i < kSegBatch; ++i)
      if (s0 + i < tpb) p[i] = __ldcg(partials + (int64_t)(seg0 + s0 + i) * R + row);
#pragma unroll
    for (int i = 0; i < kSegBatch; ++i)
      if (s0 + i < tpb) {
        skk += p[i].x;
        shk += p[i].y;
        shh += p[i].z;
      }
  }
  return alpha_from_sums(skk, shk, shh, d, eps, inv_sqrt_d);
}

__global__ void __launch_bounds__(kThreads, 1)
    proj_gate_fused_kernel(const __grid_constant__ CUtensorMap map_e,
                           const __grid_constant__ CUtensorMap map_wk,
                           const __grid_constant__ CUtensorMap map_wv,
                           const __grid_constant__ CUtensorMap map_h,
                           const __grid_constant__ CUtensorMap map_out, GateArgs g, int nkey) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  const uint32_t sA = smem_u32(smem);
  const uint32_t sB = sA + STAGES * A_BYTES;
  uint8_t* khbuf = smem + STAGE_REGION;
  const uint32_t sKH = smem_u32(khbuf);
  const float* wbuf = reinterpret_cast<const float*>(khbuf + KH_BYTES);
  const uint32_t sW = smem_u32(wbuf);
  float* s_alpha = reinterpret_cast<float*>(khbuf + KH_BYTES + W_BYTES);  // [128]
  uint64_t* bars = reinterpret_cast<uint64_t*>(khbuf + KH_BYTES + W_BYTES + kRows * 4);
  const uint32_t bar0 = smem_u32(bars);
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (STAGES + s); };
  const uint32_t tfull_bar = bar0 + 8u * (2 * STAGES);  // the tile's MMAs are done
  const uint32_t hfull_bar = tfull_bar + 8u;            // key: h block and w_q * w_k landed
  const uint32_t vfull_bar = tfull_bar + 16u;           // key: v block landed
  const uint32_t drain_bar = tfull_bar + 24u;
  const uint32_t pair_bar = tfull_bar + 32u;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + NUM_BARS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();  // 0 = the pair's MMA leader
  const bool leader = rank == 0;
  const int R = g.R, d = g.d, M = g.M;
  const int cl = (int)(blockIdx.x >> 1);
  const bool key = cl < nkey;
  const int num_kb = (g.d_mem + BK - 1) / BK;
  const int row0 = (int)rank * kRows;  // first row of this CTA
  // key tile: columns [n0, n0 + 256) of the [M d] key space, i.e. columns
  // [j0, j0 + 256) of branch mb (d is a multiple of 256); value tile:
  // columns [n0, n0 + 128) of v
  const int n0 = key ? cl * kKeyCols : (cl - nkey) * kValCols;
  const int mb = key ? n0 / d : 0;
  const int j0 = n0 - mb * d;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    mbar_init(tfull_bar, 1);
    mbar_init(hfull_bar, 1);
    mbar_init(vfull_bar, 1);
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

  if (warp == kProducerWarp) {
    // ---------------------------------------------------- e / W producer
    const CUtensorMap* map_w = key ? &map_wk : &map_wv;
    if (lane == 0) {
      asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&map_e) : "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)map_w) : "memory");
    }
    // the leader's full barrier counts the bytes of both CTAs
    const uint32_t tx = 2 * (A_BYTES + (key ? KB_BYTES : VB_BYTES));
    const int b_row = n0 + (int)rank * (key ? kKeyCols / 2 : kValCols / 2);
    // the first stages of W go out before the wait for the gather (W does not
    // depend on it; every stage is free at this point)
    const int pre = num_kb < STAGES ? num_kb : STAGES;
    if (lane == 0)
      for (int kb = 0; kb < pre; ++kb) {
        if (leader) mbar_expect_tx(full_bar(kb), tx);
        tma_load_2d_pair(sB + kb * KB_BYTES, map_w, peer_addr(full_bar(kb), 0), kb * BK, b_row);
      }
    __syncwarp();
    // e comes from the gather; once it has completed (and with it the launch
    // before it), the next call's gather may start
    griddep_wait();
    griddep_launch_dependents();
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    for (int kb = 0; kb < num_kb; ++kb) {
      const bool early = kb < pre;  // W already on its way
      if (!early) {
        if (lane == 0) ok = wait_ready(empty_bar(stage), phase ^ 1u, abort_flag, g.err);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
      }
      if (lane == 0) {
        const uint32_t fb = peer_addr(full_bar(stage), 0);
        if (!early && leader) mbar_expect_tx(full_bar(stage), tx);
        tma_load_2d_pair(sA + stage * A_BYTES, &map_e, fb, kb * BK, row0);
        if (!early) tma_load_2d_pair(sB + stage * KB_BYTES, map_w, fb, kb * BK, b_row);
      }
      __syncwarp();
      if (++stage == STAGES) {
        stage = 0;
        phase ^= 1u;
      }
    }
    if (!ok && lane == 0) {
      // let copies already issued land before the CTA can leave
      const uint64_t t0 = globaltimer();
      while (globaltimer() - t0 < 100000ull) {
      }
    }
  } else if (warp == kMmaWarp) {
    // --------------------------------------------- MMA issuer (leader only)
    if (leader) {
      const uint32_t idesc =
          key ? idesc_bf16<2 * kRows, kKeyCols>() : idesc_bf16<2 * kRows, kValCols>();
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      tc_fence_after();
      for (int kb = 0; kb < num_kb; ++kb) {
        if (lane == 0) ok = wait_ready(full_bar(stage), phase, abort_flag, g.err);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        tc_fence_after();
        if (lane == 0) {
          const uint64_t ad = sw128_desc(sA + stage * A_BYTES);
          const uint64_t bd = sw128_desc(sB + stage * KB_BYTES);
#pragma unroll
          for (int k = 0; k < BK / 16; ++k)
            umma_bf16_pair(tmem_base, ad + 2u * k, bd + 2u * k, idesc, (kb | k) != 0);
          umma_commit_pair_both(empty_bar(stage));  // slot free in both CTAs
        }
        __syncwarp();
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (lane == 0) {
        if (ok) umma_commit_pair_both(tfull_bar);  // the tile is complete in both CTAs
        umma_commit_pair_local(drain_bar);         // arrives once every MMA above has finished
        wait_drain(drain_bar, 0);
      }
    }
    __syncwarp();
  } else if (warp == kHWarp) {
    // ------------------------------------------- h and v loads (key CTAs)
    if (key) {
      griddep_wait();  // h may have been written by the launch before the gather
      if (lane == 0) {
        asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&map_h) : "memory");
        mbar_expect_tx(hfull_bar, KH_BYTES + W_BYTES);
        for (int b = 0; b < KH_BOXES; ++b)
          tma_load_2d(sKH + b * KH_BOX, &map_h, hfull_bar, n0 + b * H_COLS, row0);
        bulk_load(sW, g.w_qk + n0, W_BYTES, hfull_bar);
        // v of this block, into the stage buffers once every MMA of the tile
        // has completed and every value CTA of the row half has written v
        bool ok = wait_ready(tfull_bar, 0, abort_flag, g.err) &&
                  wait_count(g.sync + kVCount + rank, (unsigned)(d / kValCols), abort_flag, g.err);
        if (ok) {
          // generic-proxy writes of other CTAs, read by bulk copies
          asm volatile("fence.proxy.async.global;" ::: "memory");
          // the block is contiguous in the [2][d / 4][128][4] layout: four copies
          mbar_expect_tx(vfull_bar, VT_CHUNKS * VT_CHUNK);
          const float* src = g.vt + (int64_t)((int)rank * (d / 4) + j0 / 4) * kRows * 4;
          constexpr uint32_t kPart = VT_CHUNKS * VT_CHUNK / 4;
          for (int c = 0; c < 4; ++c)
            bulk_load(sA + c * kPart, src + (int64_t)c * (kPart / 4), kPart, vfull_bar);
          wait_drain(vfull_bar, 0);
        }
        wait_drain(hfull_bar, 0);  // no copy of this CTA is in flight when it leaves
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    // the previous launches' reads of the partial sums and of v are over
    griddep_wait();
    const int quarter = warp & 3, half = warp >> 2;
    const int r = quarter * 32 + lane;  // tile row of this thread (within the CTA)
    const int row = row0 + r;
    const bool valid = row < R;
    const bool rows_in = row0 + quarter * 32 < R;  // this warp has a row inside R
    bool ok = true;
    if (key) {
      if (lane == 0) ok = wait_ready(hfull_bar, 0, abort_flag, g.err);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      float skk = 0.f, shk = 0.f, shh = 0.f;
      // this warp's TMEM lanes: columns [0, 256) hold k, [256, 512) h w_q w_k
      const uint32_t tl = tmem_base + ((uint32_t)(quarter * 32) << 16);
      const uint32_t tk = tl + (uint32_t)(half * (kKeyCols / 2));
      const uint32_t thw = tl + (uint32_t)(kKeyCols + half * (kKeyCols / 2));
      if (ok) {
        // while the MMAs run: h w_q w_k of this row's 128 columns into TMEM,
        // and the row's sum of h^2 (both in the pair kernel's order).  Chunk
        // q: columns 128 half + 32 q of the tile, h box 4 half + q.
        const float* wcol = wbuf + half * (kKeyCols / 2);
#pragma unroll 1
        for (int q = 0; q < NQ; ++q) {
          const uint8_t* hs = khbuf + (half * NQ + q) * KH_BOX;
          const float4* wp = reinterpret_cast<const float4*>(wcol + q * H_COLS);
          uint4 hu[4];
          float4 wv[8];
#pragma unroll
          for (int c = 0; c < 4; ++c) hu[c] = *reinterpret_cast<const uint4*>(hs + sw64_off(r, c));
#pragma unroll
          for (int c = 0; c < 8; ++c) wv[c] = wp[c];
          unsigned long long ahh[2] = {0ull, 0ull};
          uint32_t hwv[32];
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const uint32_t hw[4] = {hu[c].x, hu[c].y, hu[c].z, hu[c].w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const int e = c * 8 + 2 * j;  // elements e, e+1 of the chunk
              const unsigned long long h2 = bf16x2_to_f2(hw[j]);
              const float4 wq = wv[e / 4];
              const unsigned long long w2 =
                  (j & 1) ? f2_pack(__float_as_uint(wq.z), __float_as_uint(wq.w))
                          : f2_pack(__float_as_uint(wq.x), __float_as_uint(wq.y));
              ahh[j & 1] = f2_fma(h2, h2, ahh[j & 1]);
              const float2 p = f2_unpack(f2_mul(h2, w2));
              hwv[e] = __float_as_uint(p.x);
              hwv[e + 1] = __float_as_uint(p.y);
            }
          }
          const float2 hh0 = f2_unpack(ahh[0]), hh1 = f2_unpack(ahh[1]);
          shh += (hh0.x + hh0.y) + (hh1.x + hh1.y);
          __syncwarp();
          tmem_st32(thw + q * H_COLS, hwv);
        }
        tmem_wait_st();
      }
      if (lane == 0 && ok) ok = wait_ready(tfull_bar, 0, abort_flag, g.err);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (ok) {
        tc_fence_after();
        // sum k^2 and sum (h w_q w_k) k: packed fp32 pairs, two accumulators
        // per sum, chunk sums added in order (the pair kernel's arithmetic)
        uint32_t kv[32], hv[32];
#pragma unroll 1
        for (int q = 0; q < NQ; ++q) {
          __syncwarp();
          tmem_ld32_async(tk + q * H_COLS, kv);
          tmem_ld32_async(thw + q * H_COLS, hv);
          tmem_wait32(kv);
          tmem_wait32(hv);
          unsigned long long akk[2] = {0ull, 0ull}, ahk[2] = {0ull, 0ull};
#pragma unroll
          for (int c = 0; c < 4; ++c)
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const int e = c * 8 + 2 * j;
              const unsigned long long k2 = f2_pack(kv[e], kv[e + 1]);
              akk[j & 1] = f2_fma(k2, k2, akk[j & 1]);
              ahk[j & 1] = f2_fma(f2_pack(hv[e], hv[e + 1]), k2, ahk[j & 1]);
            }
          const float2 kk0 = f2_unpack(akk[0]), kk1 = f2_unpack(akk[1]);
          const float2 hk0 = f2_unpack(ahk[0]), hk1 = f2_unpack(ahk[1]);
          skk += (kk0.x + kk0.y) + (kk1.x + kk1.y);
          shk += (hk0.x + hk0.y) + (hk1.x + hk1.y);
        }
        // segment (tile, half) of the [M d / 128][R] partial sums
        if (valid)
          g.partials[(int64_t)(cl * 2 + half) * R + row] = make_float4(skk, shk, shh, 0.f);
      }
      // count this CTA done (also after a failed wait, so that no other CTA
      // waits in vain), then wait for the key CTAs of the same branch
      unsigned* kcount = g.sync + rank * kMaxBranches + mb;
      epi_count_done(kcount);
      if (threadIdx.x == 0) wait_count(kcount, (unsigned)(d / kKeyCols), abort_flag, g.err);
      epi_bar_sync();
      ok = ok && *abort_flag == 0;
      // alpha of the CTA's 128 rows for branch mb: one row per thread of the
      // first column half; the first tile of the branch also writes it out
      if (ok && half == 0) {
        float a = 0.f;
        if (valid) {
          const int tpb = d / (kKeyCols / 2);  // partial-sum segments per branch
          a = fused_row_alpha(g.partials, R, row, mb * tpb, tpb, d, g.eps, g.inv_sqrt_d);
          if (g.alpha && j0 == 0) g.alpha[(int64_t)row * M + mb] = a;
        }
        s_alpha[r] = a;
      }
      epi_bar_sync();
      if (ok && lane == 0) ok = wait_ready(vfull_bar, 0, abort_flag, g.err);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (ok) {
        // out = h + alpha v over the staged h, chunk by chunk, each chunk
        // stored by TMA (this warp's 32 rows x 32 columns, 64-byte swizzle)
        const float a = s_alpha[r];
        const unsigned long long a2 = f2_pack(__float_as_uint(a), __float_as_uint(a));
#pragma unroll 1
        for (int q = 0; q < NQ; ++q) {
          const int cc = half * (kKeyCols / 2) + q * H_COLS;  // first column in the tile
          uint8_t* hs = khbuf + (half * NQ + q) * KH_BOX;
          const float4* vs = reinterpret_cast<const float4*>(smem) + (cc / 4) * kRows + r;
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint4* p = reinterpret_cast<uint4*>(hs + sw64_off(r, c));
            const uint4 hu = *p;
            const float4 v0 = vs[(2 * c) * kRows], v1 = vs[(2 * c + 1) * kRows];
            const float vf[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
            const uint32_t hw[4] = {hu.x, hu.y, hu.z, hu.w};
            uint32_t ow[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const float2 o = f2_unpack(f2_fma(
                  a2, f2_pack(__float_as_uint(vf[2 * j]), __float_as_uint(vf[2 * j + 1])),
                  bf16x2_to_f2(hw[j])));
              ow[j] = pack2(o.x, o.y);
            }
            *p = make_uint4(ow[0], ow[1], ow[2], ow[3]);
            if (g.delta && valid) {
              float4* dp = reinterpret_cast<float4*>(g.delta + ((int64_t)row * M + mb) * d + j0 +
                                                     cc + 8 * c);
              dp[0] = make_float4(a * v0.x, a * v0.y, a * v0.z, a * v0.w);
              dp[1] = make_float4(a * v1.x, a * v1.y, a * v1.z, a * v1.w);
            }
          }
          fence_async_smem();  // generic-proxy writes -> visible to the TMA store
          __syncwarp();
          if (lane == 0 && rows_in)
            tma_store_2d(&map_out, sKH + (half * NQ + q) * KH_BOX + quarter * 32 * (H_COLS * 2),
                         n0 + cc, row0 + quarter * 32);
        }
        if (lane == 0) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
      }
    } else {
      // v of this CTA's 128 rows and 64 columns (column half `half` of the
      // tile) into the [2][d / 4][128][4] scratch, then count this CTA done
      if (lane == 0) ok = wait_ready(tfull_bar, 0, abort_flag, g.err);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (ok) {
        tc_fence_after();
        const uint32_t taddr =
            tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(half * 64);
        uint32_t va[32], vb[32];
        __syncwarp();
        tmem_ld32_async(taddr, va);
        tmem_ld32_async(taddr + 32, vb);
        tmem_wait32(va);
        tmem_wait32(vb);
        if (valid) {
          float4* vt = reinterpret_cast<float4*>(g.vt) +
                       (int64_t)((int)rank * (d / 4) + (n0 + half * 64) / 4) * kRows + r;
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            const uint32_t* v = c < 8 ? va : vb;
            const int e = (c & 7) * 4;
            vt[(int64_t)c * kRows] =
                make_float4(__uint_as_float(v[e]), __uint_as_float(v[e + 1]),
                            __uint_as_float(v[e + 2]), __uint_as_float(v[e + 3]));
          }
        }
      }
      epi_count_done(g.sync + kVCount + rank);
    }
    // a failed wait may leave a TMEM load in flight
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
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
  // the last CTA to leave zeroes the counters for the next launch (every
  // other CTA has passed its waits by then)
  if (threadIdx.x == 0) {
    __threadfence();
    if (atomicAdd(g.sync + kExit, 1u) == gridDim.x - 1)
      for (int i = 0; i <= kExit; ++i) atomicExch(g.sync + i, 0u);
  }
}

}  // namespace

cudaError_t launch_proj_gate_fused(const FusedMaps& maps, const GateArgs& g, int nkey, int nval,
                                   cudaStream_t stream) {
  if (g.R == 0) return cudaSuccess;
  if (g.R > 2 * kRows || nkey < 1 || nval < 1 || g.M < 1 || g.M > kMaxBranches || !g.sync ||
      !g.vt || g.d % kKeyCols != 0 || nkey != g.M * g.d / kKeyCols || nval != g.d / kValCols)
    return cudaErrorInvalidValue;
  auto kern = proj_gate_fused_kernel;
  cudaError_t e =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t lc = {};
  lc.gridDim = dim3(2 * (nkey + nval));
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
  e = cudaLaunchKernelEx(&lc, kern, maps.e, maps.wk, maps.wv, maps.h, maps.out, g, nkey);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

int fused_max_clusters() {
  auto kern = proj_gate_fused_kernel;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM) !=
      cudaSuccess)
    return 0;
  cudaLaunchConfig_t lc = {};
  lc.gridDim = dim3(2);
  lc.blockDim = dim3(kThreads);
  lc.dynamicSmemBytes = SMEM;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = 2;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  lc.attrs = at;
  lc.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, kern, &lc) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  return n;
}

}  // namespace engram
