// bf16 projection + context-aware gate on the 5th-generation tensor cores.
//
// "Conditional Memory via Scalable Lookup", section 2.3 Eq. (3)-(4) and
// section 2.4 Eq. (6): k^(m) = W_K^(m) e, v = W_V e,
//   alpha^(m) = sigmoid(RMSNorm_q(h^(m)) . RMSNorm_k(k^(m)) / sqrt(d)),
//   out^(m)   = h^(m) + alpha^(m) v.
// The paper fuses all projections into one dense matmul (section 2.4).  Here
// both are one persistent warp-specialised GEMM kernel, launched twice:
//
//   phase 0 (keys):   N = M*d columns of [W_K^(1); ...; W_K^(M)].  The
//                     epilogue never stores k: it reduces each 128 x BN tile
//                     to per-row partial sums (sum k^2, sum h w_q w_k k,
//                     sum h^2), which decompose RMSNorm(h).RMSNorm(k) over
//                     column tiles because both norms are per-row scalars.
//   phase 1 (values): N = d columns of W_V.  The epilogue finishes alpha from
//                     the partials of every key tile of the branch and writes
//                     out = h + alpha v for each branch directly from TMEM.
//
// Per CTA (one per SM, persistent, 192 threads):
//   warp 4      TMA producer: A = e tile [128 x 64], B = W tile [BN x 64],
//               128-byte swizzle, STAGES-deep ring of smem slots;
//   warp 5      TMEM allocator and MMA issuer: tcgen05.mma.cta_group::1
//               kind::f16 (bf16 in, fp32 accumulate), M=128, N=BN, K=16,
//               accumulators double-buffered in TMEM (2*BN columns);
//   warps 0-3   epilogue: tcgen05.ld 32 columns at a time (warp w owns TMEM
//               lanes 32w..32w+31, i.e. rows of the tile), fused gate math,
//               global loads of h and stores of out.
// Every mbarrier wait is bounded (kWaitLimitNs); on expiry the kernel records
// kDevErrTimeout, every role leaves its loop, outstanding MMAs are drained and
// TMEM is freed before the CTA exits.
#include <cuda_bf16.h>

#include "engram_internal.cuh"

namespace engram {

namespace {

constexpr int BM = 128;
constexpr int BK = 64;                    // 64 bf16 = one 128-byte swizzle row
constexpr uint32_t A_BYTES = BM * BK * 2; // 16 KB
constexpr int kThreads = 224;  // 7 warps
constexpr unsigned long long kWaitLimitNs = 2000000000ull;  // 2 s

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wait for phase `parity` of `bar` to complete, for at most kWaitLimitNs.
// Returns false (and raises the CTA's abort flag) on expiry or if another role
// has already aborted.
__device__ __noinline__ bool wait_bounded(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          unsigned* err) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (globaltimer() - t0 > kWaitLimitNs) {
      *abort_flag = 1;
      atomicOr(err, kDevErrTimeout);
      return false;
    }
  }
}

// Same, ignoring the abort flag (used only to drain on the way out).
__device__ __noinline__ void wait_drain(uint32_t bar, uint32_t parity) {
  const uint64_t t0 = globaltimer();
  while (!mbar_try_wait(bar, parity))
    if (globaltimer() - t0 > kWaitLimitNs) return;
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
      "l"((uint64_t)map), "r"(bar), "r"(x), "r"(y)
      : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Shared-memory matrix descriptor for a K-major tile written by TMA with the
// 128-byte swizzle: rows of 128 bytes, 8-row atoms 1024 bytes apart (SBO),
// descriptor version 1 (sm_100), layout type 2 = SWIZZLE_128B.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
  return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)1 << 16) |
         ((uint64_t)(1024 >> 4) << 32) | ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// Instruction descriptor, kind::f16: D fp32 (bits 4-5 = 1), A and B bf16
// (bits 7-9 and 10-12 = 1), both K-major, N>>3 at bit 17, M>>4 at bit 24.
template <int M, int N>
__host__ __device__ constexpr uint32_t idesc_bf16() {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) |
         ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void umma_bf16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate));
}

__device__ __forceinline__ void umma_commit(uint32_t bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
      : "memory");
}

// --- CTA-pair (cta_group::2) forms -----------------------------------------

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// Address of the same shared-memory location in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t peer_addr(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}

__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr)
               : "memory");
}

__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                   : "memory");
}

// TMA load into this CTA's shared memory whose completion bytes are counted on
// an mbarrier that may live in either CTA of the pair (no multicast).
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap* map,
                                                 uint32_t cluster_bar, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
      "l"((uint64_t)map), "r"(cluster_bar), "r"(x), "r"(y)
      : "memory");
}

__device__ __forceinline__ void umma_bf16_pair(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                               uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate));
}

// Arrive on the mbarrier at this offset in both CTAs of the pair once every
// MMA issued so far by this thread has completed.
__device__ __forceinline__ void umma_commit_pair_both(uint32_t bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], %1;" ::"r"(bar),
      "h"((uint16_t)3)
      : "memory");
}

__device__ __forceinline__ void umma_commit_pair_local(uint32_t bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
      : "memory");
}

// 32 consecutive fp32 columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float* v) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
        "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
        "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void unpack8(const uint4& u, float* f) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

__device__ __forceinline__ uint32_t pack2(float a, float b) {
  const __nv_bfloat162 p = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&p);
}

__device__ __forceinline__ float sigmoid_f(float s) { return 1.0f / (1.0f + expf(-s)); }

__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, uint32_t src, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
          (uint64_t)map),
      "r"(src), "r"(x), "r"(y)
      : "memory");
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}

__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

constexpr int H_SLOTS = 2;                  // ring of h / out sub-tiles
constexpr uint32_t H_BYTES = BM * 64 * 2;   // one sub-tile: 128 rows x 64 bf16, 128-B swizzle

template <int BN, bool PAIR>
struct Cfg {
  // In a CTA pair each CTA holds half of the B tile (its BN/2 rows of W).
  static constexpr uint32_t B_BYTES = (PAIR ? BN / 2 : BN) * BK * 2;
  static constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int STAGES = (196608 / STAGE_BYTES) > 8 ? 8 : (196608 / STAGE_BYTES);
  static constexpr uint32_t TMEM_COLS = 2 * BN;
  static constexpr int UMMA_M = PAIR ? 2 * BM : BM;
  static constexpr int NUM_BARS = 2 * STAGES + 4 + 3 * H_SLOTS + 2;
  static constexpr uint32_t BAR_BYTES = 8 * NUM_BARS + 16;
  static constexpr size_t SMEM =
      1024 + (size_t)STAGES * STAGE_BYTES + (size_t)H_SLOTS * H_BYTES + BAR_BYTES;
  static_assert(SMEM <= 232448, "shared memory budget");
  static_assert(!PAIR || BN == 256, "CTA pairs use 256-column tiles");
};

// Byte offset of 16-byte chunk c of tile row r in a 128-byte-swizzled tile.
__device__ __forceinline__ uint32_t sw128_off(int r, int c) {
  return (uint32_t)(r * 128 + ((c ^ (r & 7)) << 4));
}

// One launch computes [R x n_total] = e [R x d_mem] . W^T with the gate
// epilogue of PHASE.  PAIR: a cluster of 2 CTAs computes 256 x 256 tiles with
// tcgen05.mma.cta_group::2 (each CTA loads 128 rows of e and 128 rows of W,
// holds the accumulator rows of its own 128 tile rows); else one CTA computes
// 128 x BN tiles.
template <int BN, int PHASE, bool PAIR>
__global__ void __launch_bounds__(kThreads, 1)
    proj_gate_kernel(const __grid_constant__ CUtensorMap map_e,
                     const __grid_constant__ CUtensorMap map_w,
                     const __grid_constant__ CUtensorMap map_h,
                     const __grid_constant__ CUtensorMap map_out, GateArgs g) {
  using C = Cfg<BN, PAIR>;
  constexpr int STAGES = C::STAGES;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  const uint32_t sA = smem_u32(smem);
  const uint32_t sB = sA + STAGES * A_BYTES;
  uint8_t* hbuf = smem + (size_t)STAGES * C::STAGE_BYTES;
  const uint32_t sH = smem_u32(hbuf);
  uint64_t* bars = reinterpret_cast<uint64_t*>(hbuf + (size_t)H_SLOTS * H_BYTES);
  const uint32_t bar0 = smem_u32(bars);
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (STAGES + s); };
  auto tfull_bar = [&](int a) { return bar0 + 8u * (2 * STAGES + a); };
  auto tempty_bar = [&](int a) { return bar0 + 8u * (2 * STAGES + 2 + a); };
  auto hfull_bar = [&](int s) { return bar0 + 8u * (2 * STAGES + 4 + s); };
  auto hempty_bar = [&](int s) { return bar0 + 8u * (2 * STAGES + 4 + H_SLOTS + s); };
  auto hdone_bar = [&](int s) { return bar0 + 8u * (2 * STAGES + 4 + 2 * H_SLOTS + s); };
  const uint32_t drain_bar = bar0 + 8u * (2 * STAGES + 4 + 3 * H_SLOTS);
  const uint32_t pair_bar = drain_bar + 8u;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::NUM_BARS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = PAIR ? cluster_rank() : 0u;  // 0 = the pair's MMA leader
  const bool leader = rank == 0;
  const int R = g.R, d = g.d, M = g.M;
  const int n_total = PHASE == 0 ? M * d : d;
  const int num_n = n_total / BN;
  const int tile_rows = PAIR ? 2 * BM : BM;  // rows of one (pair) tile
  const int num_tiles = ((R + tile_rows - 1) / tile_rows) * num_n;
  const int num_kb = (g.d_mem + BK - 1) / BK;
  const int first_tile = PAIR ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;
  const int tile_step = PAIR ? (int)(gridDim.x >> 1) : (int)gridDim.x;
  // h sub-tiles per output tile: the key phase reads one branch, the value
  // phase every branch (v is shared, Eq. 6)
  const int nsub = (BN / 64) * (PHASE == 0 ? 1 : M);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull_bar(a), 1);
      mbar_init(tempty_bar(a), PAIR ? 8 : 4);  // every epilogue warp of the pair
    }
    for (int s = 0; s < H_SLOTS; ++s) {
      mbar_init(hfull_bar(s), 1);
      mbar_init(hempty_bar(s), PHASE == 0 ? 4 : 1);
      mbar_init(hdone_bar(s), 4);
    }
    mbar_init(drain_bar, 1);
    mbar_init(pair_bar, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 5) {
    if (PAIR) {
      asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                       smem_u32(tmem_slot)),
                   "r"(C::TMEM_COLS));
      asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;");
    } else {
      asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                       smem_u32(tmem_slot)),
                   "r"(C::TMEM_COLS));
      asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
  }
  tc_fence_before();
  __syncthreads();
  // both CTAs of a pair are co-scheduled: their barriers are initialised
  // before either one signals the other
  if (PAIR) cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 4) {
    // ------------------------------------------------- e / W producer (TMA)
    if (lane == 0) {
      asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&map_e) : "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&map_w) : "memory");
    }
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    for (int tile = first_tile; ok && tile < num_tiles; tile += tile_step) {
      const int m_blk = tile / num_n, n_blk = tile - m_blk * num_n;
      const int a_row = m_blk * tile_rows + (int)rank * BM;
      const int b_row = n_blk * BN + (int)rank * (BN / 2);
      for (int kb = 0; kb < num_kb; ++kb) {
        if (lane == 0) ok = wait_bounded(empty_bar(stage), phase ^ 1u, abort_flag, g.err);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        if (lane == 0) {
          if (PAIR) {
            // the leader's full barrier counts the bytes of both CTAs
            const uint32_t fb = peer_addr(full_bar(stage), 0);
            if (leader) mbar_expect_tx(full_bar(stage), 2 * C::STAGE_BYTES);
            tma_load_2d_pair(sA + stage * A_BYTES, &map_e, fb, kb * BK, a_row);
            tma_load_2d_pair(sB + stage * C::B_BYTES, &map_w, fb, kb * BK, b_row);
          } else {
            mbar_expect_tx(full_bar(stage), C::STAGE_BYTES);
            tma_load_2d(sA + stage * A_BYTES, &map_e, full_bar(stage), kb * BK, a_row);
            tma_load_2d(sB + stage * C::B_BYTES, &map_w, full_bar(stage), kb * BK, n_blk * BN);
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
      // give any copy already issued time to land before the CTA's smem is released
      const uint64_t t0 = globaltimer();
      while (globaltimer() - t0 < 100000ull) {
      }
    }
  } else if (warp == 6) {
    // ---------------------------------------------- h sub-tile producer (TMA)
    if (lane == 0) asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&map_h) : "memory");
    int slot = 0;
    uint32_t phase = 0;
    bool ok = true;
    for (int tile = first_tile; ok && tile < num_tiles; tile += tile_step) {
      const int m_blk = tile / num_n, n0 = (tile - m_blk * num_n) * BN;
      const int row0 = m_blk * tile_rows + (int)rank * BM;
      for (int i = 0; i < nsub; ++i) {
        // columns of h viewed as [R, M*d]: key phase n0 + 64q; value phase mb*d + n0 + 64q
        const int x = PHASE == 0 ? n0 + 64 * i : (i % M) * d + n0 + 64 * (i / M);
        if (lane == 0) ok = wait_bounded(hempty_bar(slot), phase ^ 1u, abort_flag, g.err);
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
  } else if (warp == 5) {
    // ------------------------------------------- MMA issuer (pair: leader only)
    constexpr uint32_t idesc = idesc_bf16<C::UMMA_M, BN>();
    int stage = 0, acc = 0;
    uint32_t phase = 0, acc_phase = 0;
    bool ok = true;
    if (leader) {
      for (int tile = first_tile; ok && tile < num_tiles; tile += tile_step) {
        if (lane == 0) ok = wait_bounded(tempty_bar(acc), acc_phase ^ 1u, abort_flag, g.err);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
        for (int kb = 0; kb < num_kb; ++kb) {
          if (lane == 0) ok = wait_bounded(full_bar(stage), phase, abort_flag, g.err);
          ok = __shfl_sync(0xffffffffu, ok, 0);
          if (!ok) break;
          tc_fence_after();
          if (lane == 0) {
            const uint64_t ad = sw128_desc(sA + stage * A_BYTES);
            const uint64_t bd = sw128_desc(sB + stage * C::B_BYTES);
#pragma unroll
            for (int k = 0; k < BK / 16; ++k) {
              if (PAIR)
                umma_bf16_pair(d_tmem, ad + 2u * k, bd + 2u * k, idesc, (kb | k) != 0);
              else
                umma_bf16(d_tmem, ad + 2u * k, bd + 2u * k, idesc, (kb | k) != 0);
            }
            // the slot (in both CTAs of a pair) is free once these MMAs have read it
            if (PAIR)
              umma_commit_pair_both(empty_bar(stage));
            else
              umma_commit(empty_bar(stage));
          }
          __syncwarp();
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        if (lane == 0) {  // accumulator complete (in both CTAs of a pair)
          if (PAIR)
            umma_commit_pair_both(tfull_bar(acc));
          else
            umma_commit(tfull_bar(acc));
        }
        __syncwarp();
        if (++acc == 2) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
      if (lane == 0) {
        // arrives once every MMA issued above has finished
        if (PAIR)
          umma_commit_pair_local(drain_bar);
        else
          umma_commit(drain_bar);
        wait_drain(drain_bar, 0);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    // Thread (warp w, lane l) owns tile row r = 32w + l: TMEM lane r and
    // row r of every h sub-tile in shared memory.
    const int r = warp * 32 + lane;
    int acc = 0, hslot = 0;
    uint32_t acc_phase = 0, hphase = 0;
    bool ok = true;
    const int tiles_per_branch = d / g.key_tile;
    for (int tile = first_tile; ok && tile < num_tiles; tile += tile_step) {
      const int m_blk = tile / num_n, n_blk = tile - m_blk * num_n;
      const int row0 = m_blk * tile_rows + (int)rank * BM;
      const int row = row0 + r;
      const bool valid = row < R;
      const int n0 = n_blk * BN;
      float al[kMaxBranches];
      if (PHASE == 1) {
        // alpha from the key phase's per-tile partial sums (Eq. 4 / Eq. 6)
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
      if (lane == 0) ok = wait_bounded(tfull_bar(acc), acc_phase, abort_flag, g.err);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      tc_fence_after();
      const uint32_t taddr = tmem_base + ((uint32_t)(warp * 32) << 16) + (uint32_t)(acc * BN);
      float v[64];
      if (PHASE == 0) {
        const int mb = n0 / d, j0 = n0 - mb * d;
        const float* wrow = g.w_qk + (int64_t)mb * d + j0;
        float skk = 0.f, shk = 0.f, shh = 0.f;
#pragma unroll 1
        for (int q = 0; q < BN / 64; ++q) {
          __syncwarp();
          tmem_ld32(taddr + q * 64, v);
          tmem_ld32(taddr + q * 64 + 32, v + 32);
          if (lane == 0) ok = wait_bounded(hfull_bar(hslot), hphase, abort_flag, g.err);
          ok = __shfl_sync(0xffffffffu, ok, 0);
          if (!ok) break;
          const uint8_t* hs = hbuf + hslot * H_BYTES;
          const float4* wp = reinterpret_cast<const float4*>(wrow + q * 64);
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            float hf[8];
            unpack8(*reinterpret_cast<const uint4*>(hs + sw128_off(r, c)), hf);
            const float4 w0 = __ldg(wp + 2 * c), w1 = __ldg(wp + 2 * c + 1);
            const float wf[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const float k = v[c * 8 + i];
              skk = fmaf(k, k, skk);
              shh = fmaf(hf[i], hf[i], shh);
              shk = fmaf(hf[i] * wf[i], k, shk);
            }
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(hempty_bar(hslot));
          if (++hslot == H_SLOTS) {
            hslot = 0;
            hphase ^= 1u;
          }
        }
        if (!ok) break;
        if (valid) g.partials[(int64_t)n_blk * R + row] = make_float4(skk, shk, shh, 0.f);
      } else {
#pragma unroll 1
        for (int q = 0; q < BN / 64; ++q) {
          __syncwarp();
          tmem_ld32(taddr + q * 64, v);
          tmem_ld32(taddr + q * 64 + 32, v + 32);
#pragma unroll 1
          for (int mb = 0; mb < M; ++mb) {
            if (lane == 0) ok = wait_bounded(hfull_bar(hslot), hphase, abort_flag, g.err);
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) break;
            uint8_t* hs = hbuf + hslot * H_BYTES;
            float a = 0.f;
#pragma unroll
            for (int b = 0; b < kMaxBranches; ++b)
              if (b == mb) a = al[b];
            // out = h + alpha v, written over h in place, then stored by TMA
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              uint4* p = reinterpret_cast<uint4*>(hs + sw128_off(r, c));
              float hf[8], o[8];
              unpack8(*p, hf);
#pragma unroll
              for (int i = 0; i < 8; ++i) o[i] = fmaf(a, v[c * 8 + i], hf[i]);
              *p = make_uint4(pack2(o[0], o[1]), pack2(o[2], o[3]), pack2(o[4], o[5]),
                              pack2(o[6], o[7]));
            }
            if (g.delta && valid) {
              float4* dp = reinterpret_cast<float4*>(g.delta + ((int64_t)row * M + mb) * d + n0 +
                                                     q * 64);
#pragma unroll
              for (int c = 0; c < 16; ++c)
                dp[c] = make_float4(a * v[4 * c], a * v[4 * c + 1], a * v[4 * c + 2],
                                    a * v[4 * c + 3]);
            }
            fence_async_smem();  // generic-proxy writes -> visible to the TMA store
            __syncwarp();
            if (lane == 0) mbar_arrive(hdone_bar(hslot));
            if (warp == 0) {
              if (lane == 0) {
                ok = wait_bounded(hdone_bar(hslot), hphase, abort_flag, g.err);
                if (ok) {
                  if (row0 < R) {  // rows past R are clipped; a tile wholly past R stores nothing
                    tma_store_2d(&map_out, sH + hslot * H_BYTES, mb * d + n0 + q * 64, row0);
                    asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
                  }
                  mbar_arrive(hempty_bar(hslot));
                }
              }
              ok = __shfl_sync(0xffffffffu, ok, 0);
              if (!ok) break;
            }
            if (++hslot == H_SLOTS) {
              hslot = 0;
              hphase ^= 1u;
            }
          }
          if (!ok) break;
        }
        if (!ok) break;
      }
      // accumulator buffer free again (the pair's leader owns the barrier)
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (PAIR)
          mbar_arrive_cluster(peer_addr(tempty_bar(acc), 0));
        else
          mbar_arrive(tempty_bar(acc));
      }
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
    if (PHASE == 1 && warp == 0 && lane == 0)
      asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
  }

  tc_fence_before();
  __syncthreads();
  if (PAIR) {
    // neither CTA leaves while its partner may still read its shared memory
    // (the leader's MMAs) or signal its barriers (the follower's arrivals)
    if (threadIdx.x == 0) {
      mbar_arrive_cluster(peer_addr(pair_bar, rank ^ 1u));
      wait_drain(pair_bar, 0);
    }
    __syncthreads();
  }
  tc_fence_after();
  if (warp == 5) {
    if (PAIR)
      asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                   "r"(C::TMEM_COLS));
    else
      asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                   "r"(C::TMEM_COLS));
  }
}

template <int BN, int PHASE, bool PAIR>
cudaError_t launch_bn(const ProjMaps& maps, const GateArgs& g, int grid, cudaStream_t stream) {
  auto kern = proj_gate_kernel<BN, PHASE, PAIR>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)Cfg<BN, PAIR>::SMEM);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t lc = {};
  lc.gridDim = dim3(grid);
  lc.blockDim = dim3(kThreads);
  lc.dynamicSmemBytes = Cfg<BN, PAIR>::SMEM;
  lc.stream = stream;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = PAIR ? 2 : 1;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  lc.attrs = at;
  lc.numAttrs = 1;
  e = cudaLaunchKernelEx(&lc, kern, maps.e, maps.w, maps.h, maps.out, g);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace

int sm100_stages(int bn) {
  return bn == 256 ? Cfg<256, false>::STAGES
                   : bn == 128 ? Cfg<128, false>::STAGES : Cfg<64, false>::STAGES;
}

size_t sm100_smem_bytes(int bn) {
  return bn == 256 ? Cfg<256, false>::SMEM : bn == 128 ? Cfg<128, false>::SMEM : Cfg<64, false>::SMEM;
}

cudaError_t launch_proj_gate_sm100(int phase, int bn, bool pair, const ProjMaps& maps,
                                   const GateArgs& g, int grid, cudaStream_t stream) {
  if (g.R == 0) return cudaSuccess;
  if (pair) {
    if (bn != 256 || (grid & 1)) return cudaErrorInvalidValue;
    return phase == 0 ? launch_bn<256, 0, true>(maps, g, grid, stream)
                      : launch_bn<256, 1, true>(maps, g, grid, stream);
  }
  switch (bn * 2 + phase) {
    case 512: return launch_bn<256, 0, false>(maps, g, grid, stream);
    case 513: return launch_bn<256, 1, false>(maps, g, grid, stream);
    case 256: return launch_bn<128, 0, false>(maps, g, grid, stream);
    case 257: return launch_bn<128, 1, false>(maps, g, grid, stream);
    case 128: return launch_bn<64, 0, false>(maps, g, grid, stream);
    case 129: return launch_bn<64, 1, false>(maps, g, grid, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace engram
