// bf16 projection + context-aware gate on clusters of two CTA pairs.
//
// Same computation as k_proj_gate_sm100.cu ("Conditional Memory via Scalable
// Lookup", section 2.3 Eq. (3)-(4), section 2.4 Eq. (6)); only the tiling and
// the operand traffic differ.
//
// A cluster of 4 CTAs = two tcgen05 CTA pairs (ranks {0,1} and {2,3}) computes
// a 512 x 256 tile of e . W^T: pair p holds rows [256 p, 256 p + 256), CTA
// rank q rows [128 q, 128 q + 128), each pair issuing
// tcgen05.mma.cta_group::2 (M = 256, N = 256, K = 16) into a 128 x 256 fp32
// accumulator per CTA.  TMEM holds two such accumulators (512 columns), so the
// gate epilogue of one tile overlaps the mainloop of the next.
//
// Both pairs need the same 256 W rows.  Pair 0 loads them from L2 (each of its
// CTAs its 128-row half) and pushes each half over the cluster's shared-memory
// network into the same stage of its twin in pair 1 (cp.async.bulk
// shared::cta -> shared::cluster; not a TMA multicast).  L2 -> SMEM operand
// traffic per output element is therefore that of a 512 x 256 tile on one
// pair, while each pair keeps double-buffered accumulators.
//
// Stage protocol (stage s, one use per round):
//   bfull[s]   this CTA's W half has landed (pair 0: its TMA; pair 1: the
//              push from rank q-2).  Armed by the CTA's producer.
//   full[s]    (pair leader) the pair's two e halves have landed (TMA bytes,
//              armed by the leader's producer) and both CTAs' W halves are
//              present (one arrival each, relayed by warp 7 from bfull[s]).
//   empty[s]   (pair 0) the pair-0 MMAs have read stage s (commit from rank
//              0) and this CTA's push has landed in its twin (the twin's
//              warp 7 arrives: a landed push has read its source).
//   p1free[s]  pair 1's MMAs have read stage s (commit from rank 2 to all four
//              CTAs): pair 1 may refill it and pair 0 may push into it again.
//
// Roles (256 threads per CTA): warps 0-3 epilogue (row 32w + lane), warp 4
// e/W producer, warp 5 TMEM allocator + MMA issuer (pair leaders), warp 6 h
// producer (64-byte-swizzled 128 x 32 sub-tiles, 8 slots, and w_q * w_k of
// the tile), warp 7 W relay and
// pusher.  Phases: 0 keys, 1 values (out = h + alpha v through the h ring),
// 2 values added into h in place (TMA reduce-add).  Every wait is bounded;
// the four CTAs leave through a bounded handshake.
#include "sm100_ptx.cuh"

namespace engram {

namespace {

using namespace sm100;

constexpr int kRows = 128;                         // tile rows per CTA
constexpr int kCols = 256;                         // tile columns
constexpr int BK = 64;
constexpr uint32_t A_BYTES = kRows * BK * 2;       // 16 KB
constexpr uint32_t B_BYTES = (kCols / 2) * BK * 2; // 16 KB: one W half
constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int STAGES = 5;
constexpr int H_COLS = 32;
constexpr uint32_t H_BYTES = kRows * H_COLS * 2;   // 8 KB
constexpr int H_SLOTS = 8;                         // one key tile's h
constexpr uint32_t W_BYTES = kCols * 4;
constexpr int kEpiWarps = 4;
constexpr int kThreads = (kEpiWarps + 4) * 32;     // 256
constexpr int kProducerWarp = 4, kMmaWarp = 5, kHWarp = 6, kRelayWarp = 7;
constexpr uint32_t TMEM_COLS = 2 * kCols;          // two accumulators
constexpr int NUM_BARS = 4 * STAGES + 4 + 2 * H_SLOTS + 4;
constexpr size_t SMEM = 1024 + (size_t)STAGES * STAGE_BYTES + (size_t)H_SLOTS * H_BYTES + W_BYTES +
                        8 * NUM_BARS + 16;
static_assert(SMEM <= 232448, "shared memory budget");
static_assert(kEpiWarps * 4096 <= H_SLOTS * H_BYTES, "in-place staging fits in the h ring");

// Bulk copy of this CTA's shared memory into another CTA of the cluster,
// completion counted on an mbarrier of the destination CTA (which is also the
// only sign that the source has been read).
__device__ __forceinline__ void push_to_peer(uint32_t dst_cluster, uint32_t src, uint32_t bytes,
                                             uint32_t bar_cluster) {
  asm volatile(
      "cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          dst_cluster),
      "r"(src), "r"(bytes), "r"(bar_cluster)
      : "memory");
}

__device__ __forceinline__ void umma_commit_mask(uint32_t bar, uint16_t mask) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], %1;" ::"r"(bar),
      "h"(mask)
      : "memory");
}

template <int PHASE>
__global__ void __launch_bounds__(kThreads, 1)
    proj_gate_quad_kernel(const __grid_constant__ CUtensorMap map_e,
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
  auto bfull_bar = [&](int s) { return bar0 + 8u * (STAGES + s); };
  auto empty_bar = [&](int s) { return bar0 + 8u * (2 * STAGES + s); };
  auto p1free_bar = [&](int s) { return bar0 + 8u * (3 * STAGES + s); };
  auto tfull_bar = [&](int a) { return bar0 + 8u * (4 * STAGES + a); };
  auto tempty_bar = [&](int a) { return bar0 + 8u * (4 * STAGES + 2 + a); };
  auto hfull_bar = [&](int s) { return bar0 + 8u * (4 * STAGES + 4 + s); };
  auto hempty_bar = [&](int s) { return bar0 + 8u * (4 * STAGES + 4 + H_SLOTS + s); };
  const uint32_t wfull_bar = bar0 + 8u * (4 * STAGES + 4 + 2 * H_SLOTS);
  const uint32_t wempty_bar = wfull_bar + 8u;
  const uint32_t drain_bar = wfull_bar + 16u;
  const uint32_t exit_bar = wfull_bar + 24u;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + NUM_BARS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t q = cluster_rank();         // 0..3
  const uint32_t pair = q >> 1;              // 0 loads W, 1 receives it
  const uint32_t lead = q & 2u;              // rank of this pair's MMA leader
  const bool leader = q == lead;
  const uint16_t pair_mask = (uint16_t)(3u << lead);
  const int R = g.R, d = g.d, M = g.M;
  const int n_total = PHASE == 0 ? M * d : d;
  const int num_n = n_total / kCols;
  const int num_tiles = ((R + 4 * kRows - 1) / (4 * kRows)) * num_n;
  const int num_kb = (g.d_mem + BK - 1) / BK;
  const int first_tile = (int)(blockIdx.x >> 2), tile_step = (int)(gridDim.x >> 2);
  const int nsub = PHASE == 2 ? 0 : (kCols / H_COLS) * (PHASE == 0 ? 1 : M);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), 3);   // leader's TMA arming + two W-half arrivals
      mbar_init(bfull_bar(s), 1);
      mbar_init(empty_bar(s), 2);  // pair-0 MMA commit + the twin's push-landed relay
      mbar_init(p1free_bar(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull_bar(a), 1);
      mbar_init(tempty_bar(a), 2 * kEpiWarps);
    }
    for (int s = 0; s < H_SLOTS; ++s) {
      mbar_init(hfull_bar(s), 1);
      mbar_init(hempty_bar(s), kEpiWarps);
    }
    mbar_init(wfull_bar, 1);
    mbar_init(wempty_bar, kEpiWarps);
    mbar_init(drain_bar, 1);
    mbar_init(exit_bar, 3);
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
  cluster_sync_all();  // every CTA's barriers are initialised before any signal
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == kProducerWarp) {
    // ---------------------------------------------------- e / W producer
    if (lane == 0) {
      asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&map_e) : "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&map_w) : "memory");
    }
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    for (int tile = first_tile; ok && tile < num_tiles; tile += tile_step) {
      const int m_blk = tile / num_n, n_blk = tile - m_blk * num_n;
      const int a_row = m_blk * 4 * kRows + (int)q * kRows;
      const int b_row = n_blk * kCols + (int)(q & 1u) * (kCols / 2);
      for (int kb = 0; kb < num_kb; ++kb) {
        if (lane == 0)
          ok = wait_ready(pair == 0 ? empty_bar(stage) : p1free_bar(stage), phase ^ 1u,
                          abort_flag, g.err);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        if (lane == 0) {
          // this CTA's W half arrives on bfull (its own TMA, or the push)
          mbar_expect_tx(bfull_bar(stage), B_BYTES);
          if (leader) mbar_expect_tx(full_bar(stage), 2 * A_BYTES);
          tma_load_2d_pair(sA + stage * A_BYTES, &map_e, peer_addr(full_bar(stage), lead), kb * BK,
                           a_row);
          if (pair == 0)
            tma_load_2d(sB + stage * B_BYTES, &map_w, bfull_bar(stage), kb * BK, b_row);
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
  } else if (warp == kRelayWarp) {
    // ------------------------------------------- W-half relay and pusher
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    for (int tile = first_tile; ok && tile < num_tiles; tile += tile_step) {
      for (int kb = 0; kb < num_kb; ++kb) {
        if (lane == 0) ok = wait_ready(bfull_bar(stage), phase, abort_flag, g.err);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        if (lane == 0) {
          mbar_arrive_cluster(peer_addr(full_bar(stage), lead));  // my W half is here
          if (pair == 0) {
            // into the twin's stage once pair 1 has finished reading it
            ok = wait_ready(p1free_bar(stage), phase ^ 1u, abort_flag, g.err);
            if (ok)
              push_to_peer(peer_addr(sB + stage * B_BYTES, q + 2), sB + stage * B_BYTES, B_BYTES,
                           peer_addr(bfull_bar(stage), q + 2));
          } else {
            // the push has landed, so it has read its source: the twin in
            // pair 0 may refill that stage (once its own MMAs are done too)
            mbar_arrive_cluster(peer_addr(empty_bar(stage), q - 2));
          }
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
  } else if (warp == kHWarp) {
    // -------------------------------------------------- h sub-tile producer
    if (lane == 0) asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&map_h) : "memory");
    int slot = 0;
    uint32_t phase = 0, wphase = 0;
    bool ok = true;
    for (int tile = first_tile; ok && tile < num_tiles; tile += tile_step) {
      const int m_blk = tile / num_n, n0 = (tile - m_blk * num_n) * kCols;
      const int row0 = m_blk * 4 * kRows + (int)q * kRows;
      if (PHASE == 2) continue;  // values added in place: h is not staged
      if (PHASE == 0) {
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
    // ------------------------------------------ MMA issuer (pair leaders)
    constexpr uint32_t idesc = idesc_bf16<2 * kRows, kCols>();
    int stage = 0, acc = 0;
    uint32_t phase = 0, acc_phase = 0;
    bool ok = true;
    if (leader) {
      for (int tile = first_tile; ok && tile < num_tiles; tile += tile_step) {
        if (lane == 0) ok = wait_ready(tempty_bar(acc), acc_phase ^ 1u, abort_flag, g.err);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * kCols);
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
              umma_bf16_pair(d_tmem, ad + 2u * k, bd + 2u * k, idesc, (kb | k) != 0);
            // pair 0 frees its own stage; pair 1 tells all four CTAs, since
            // pair 0 pushes into pair 1's stage
            if (pair == 0)
              umma_commit_mask(empty_bar(stage), (uint16_t)0x3);
            else
              umma_commit_mask(p1free_bar(stage), (uint16_t)0xF);
          }
          __syncwarp();
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        if (lane == 0) umma_commit_mask(tfull_bar(acc), pair_mask);
        __syncwarp();
        if (++acc == 2) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
      if (lane == 0) {
        umma_commit_pair_local(drain_bar);
        wait_drain(drain_bar, 0);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int wrow0 = warp * 32;  // first tile row of this warp
    const int r = wrow0 + lane;   // tile row of this thread: TMEM lane r
    int hslot = 0, acc = 0;
    uint32_t hphase = 0, acc_phase = 0, wphase = 0;
    bool ok = true;
    const int tiles_per_branch = d / g.key_tile;
    constexpr int NQ = kCols / H_COLS;
    static_assert(NQ % 2 == 0, "chunks are processed in pairs");
    for (int tile = first_tile; ok && tile < num_tiles; tile += tile_step) {
      const int m_blk = tile / num_n, n_blk = tile - m_blk * num_n;
      const int row0 = m_blk * 4 * kRows + (int)q * kRows;
      const int row = row0 + r;
      const bool valid = row < R;
      const int n0 = n_blk * kCols;
      float al[kMaxBranches];
      if (PHASE >= 1) {
#pragma unroll
        for (int mb = 0; mb < kMaxBranches; ++mb) {
          al[mb] = 0.f;
          if (mb < M && valid) {
            float skk = 0.f, shk = 0.f, shh = 0.f;
            for (int tb = mb * tiles_per_branch; tb < (mb + 1) * tiles_per_branch; ++tb) {
              const float4 p = g.partials[(int64_t)tb * R + row];
              skk += p.x;
              shk += p.y;
              shh += p.z;
            }
            const float rh = 1.0f / sqrtf(shh / (float)d + g.eps);
            const float rk = 1.0f / sqrtf(skk / (float)d + g.eps);
            al[mb] = sigmoid_f(shk * rh * rk * g.inv_sqrt_d);
            if (g.alpha && n_blk == 0) g.alpha[(int64_t)row * M + mb] = al[mb];
          }
        }
      }
      if (lane == 0) ok = wait_ready(tfull_bar(acc), acc_phase, abort_flag, g.err);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      tc_fence_after();
      const uint32_t taddr = tmem_base + ((uint32_t)wrow0 << 16) + (uint32_t)(acc * kCols);
      uint32_t va[32], vb[32];
      __syncwarp();
      tmem_ld32_async(taddr, va);
      if (PHASE == 0) {
        if (lane == 0) ok = wait_ready(wfull_bar, wphase, abort_flag, g.err);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        wphase ^= 1u;
        float skk = 0.f, shk = 0.f, shh = 0.f;
        auto key_chunk = [&](int qc, uint32_t(&v)[32], uint32_t(&vn)[32]) {
          tmem_wait32(v);
          __syncwarp();
          if (qc + 1 < NQ) tmem_ld32_async(taddr + (qc + 1) * H_COLS, vn);
          if (lane == 0) ok = wait_ready(hfull_bar(hslot), hphase, abort_flag, g.err);
          ok = __shfl_sync(0xffffffffu, ok, 0);
          if (!ok) return;
          const uint8_t* hs = hbuf + hslot * H_BYTES;
          const float4* wp = reinterpret_cast<const float4*>(wbuf + qc * H_COLS);
          uint4 hu[4];
          float4 wv[8];
#pragma unroll
          for (int c = 0; c < 4; ++c) hu[c] = *reinterpret_cast<const uint4*>(hs + sw64_off(r, c));
#pragma unroll
          for (int c = 0; c < 8; ++c) wv[c] = wp[c];
          unsigned long long akk[2] = {0ull, 0ull}, ahh[2] = {0ull, 0ull}, ahk[2] = {0ull, 0ull};
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const uint32_t hw[4] = {hu[c].x, hu[c].y, hu[c].z, hu[c].w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const int e = c * 8 + 2 * j;
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
          if (lane == 0) mbar_arrive(hempty_bar(hslot));
          if (++hslot == H_SLOTS) {
            hslot = 0;
            hphase ^= 1u;
          }
        };
#pragma unroll 1
        for (int qc = 0; ok && qc < NQ; qc += 2) {
          key_chunk(qc, va, vb);
          if (ok) key_chunk(qc + 1, vb, va);
        }
        if (!ok) break;
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive_cluster(peer_addr(tempty_bar(acc), lead));
          mbar_arrive(wempty_bar);
        }
        if (valid) g.partials[(int64_t)n_blk * R + row] = make_float4(skk, shk, shh, 0.f);
      } else if (PHASE == 2) {
        uint8_t* stage0 = hbuf + warp * 4096;
        int sbuf = 0;
        auto add_chunk = [&](int qc, uint32_t(&v)[32], uint32_t(&vn)[32]) {
          tmem_wait32(v);
          __syncwarp();
          if (qc + 1 < NQ) tmem_ld32_async(taddr + (qc + 1) * H_COLS, vn);
#pragma unroll 1
          for (int mb = 0; mb < M; ++mb) {
            float a = 0.f;
#pragma unroll
            for (int b = 0; b < kMaxBranches; ++b)
              if (b == mb) a = al[b];
            const unsigned long long a2 = f2_pack(__float_as_uint(a), __float_as_uint(a));
            if (lane == 0) asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
            __syncwarp();
            uint8_t* st = stage0 + sbuf * 2048;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              uint32_t ow[4];
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                const int e = c * 8 + 2 * j;
                const float2 o = f2_unpack(f2_mul(a2, f2_pack(v[e], v[e + 1])));
                ow[j] = pack2(o.x, o.y);
              }
              *reinterpret_cast<uint4*>(st + sw64_off(lane, c)) =
                  make_uint4(ow[0], ow[1], ow[2], ow[3]);
            }
            if (g.delta && valid) {
              float4* dp = reinterpret_cast<float4*>(g.delta + ((int64_t)row * M + mb) * d + n0 +
                                                     qc * H_COLS);
#pragma unroll
              for (int c = 0; c < 8; ++c)
                dp[c] = make_float4(a * __uint_as_float(v[4 * c]), a * __uint_as_float(v[4 * c + 1]),
                                    a * __uint_as_float(v[4 * c + 2]),
                                    a * __uint_as_float(v[4 * c + 3]));
            }
            fence_async_smem();
            __syncwarp();
            if (lane == 0) {
              if (row0 + wrow0 < R)
                tma_reduce_add_2d(&map_out, smem_u32(st), mb * d + n0 + qc * H_COLS, row0 + wrow0);
              else
                asm volatile("cp.async.bulk.commit_group;" ::: "memory");
            }
            sbuf ^= 1;
          }
        };
#pragma unroll 1
        for (int qc = 0; qc < NQ; qc += 2) {
          add_chunk(qc, va, vb);
          add_chunk(qc + 1, vb, va);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(peer_addr(tempty_bar(acc), lead));
      } else {
        int pending = -1;
        auto value_chunk = [&](int qc, uint32_t(&v)[32], uint32_t(&vn)[32]) {
          tmem_wait32(v);
          __syncwarp();
          if (qc + 1 < NQ) tmem_ld32_async(taddr + (qc + 1) * H_COLS, vn);
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
                                                     qc * H_COLS);
#pragma unroll
              for (int c = 0; c < 8; ++c)
                dp[c] = make_float4(a * __uint_as_float(v[4 * c]), a * __uint_as_float(v[4 * c + 1]),
                                    a * __uint_as_float(v[4 * c + 2]),
                                    a * __uint_as_float(v[4 * c + 3]));
            }
            fence_async_smem();
            __syncwarp();
            if (lane == 0) {
              if (row0 + wrow0 < R)
                tma_store_2d(&map_out, sH + hslot * H_BYTES + wrow0 * (H_COLS * 2),
                             mb * d + n0 + qc * H_COLS, row0 + wrow0);
              else
                asm volatile("cp.async.bulk.commit_group;" ::: "memory");
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
        for (int qc = 0; ok && qc < NQ; qc += 2) {
          value_chunk(qc, va, vb);
          if (ok) value_chunk(qc + 1, vb, va);
        }
        if (!ok) break;
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive_cluster(peer_addr(tempty_bar(acc), lead));
          asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
          if (pending >= 0) mbar_arrive(hempty_bar(pending));
        }
      }
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
    if (PHASE >= 1 && lane == 0) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
  }

  tc_fence_before();
  __syncthreads();
  // no CTA leaves while another may still read its shared memory (the pair
  // leader's MMAs, pair 0's pushes) or signal its barriers
  if (threadIdx.x == 0) {
    for (uint32_t o = 1; o < 4; ++o) mbar_arrive_cluster(peer_addr(exit_bar, (q + o) & 3u));
    wait_drain(exit_bar, 0);
  }
  __syncthreads();
  tc_fence_after();
  if (warp == kMmaWarp)
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                 "r"(TMEM_COLS));
}

template <int PHASE>
cudaError_t launch_quad(const ProjMaps& maps, const GateArgs& g, int grid, cudaStream_t stream) {
  auto kern = proj_gate_quad_kernel<PHASE>;
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
  at[0].val.clusterDim.x = 4;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  lc.attrs = at;
  lc.numAttrs = 1;
  e = cudaLaunchKernelEx(&lc, kern, maps.e, maps.w, maps.h, maps.out, g);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <int PHASE>
int quad_clusters() {
  auto kern = proj_gate_quad_kernel<PHASE>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM) !=
      cudaSuccess)
    return 0;
  cudaLaunchConfig_t lc = {};
  lc.gridDim = dim3(4);
  lc.blockDim = dim3(kThreads);
  lc.dynamicSmemBytes = SMEM;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = 4;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  lc.attrs = at;
  lc.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, kern, &lc) != cudaSuccess) return 0;
  return n;
}

}  // namespace

int quad_max_clusters() { return quad_clusters<0>(); }

cudaError_t launch_proj_gate_quad(int phase, const ProjMaps& maps, const GateArgs& g, int grid,
                                  cudaStream_t stream) {
  if (g.R == 0) return cudaSuccess;
  if (grid < 4 || (grid & 3)) return cudaErrorInvalidValue;
  switch (phase) {
    case 0: return launch_quad<0>(maps, g, grid, stream);
    case 1: return launch_quad<1>(maps, g, grid, stream);
    case 2: return launch_quad<2>(maps, g, grid, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace engram
