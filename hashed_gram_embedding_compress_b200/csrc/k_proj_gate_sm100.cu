// bf16 projection + context-aware gate on the 5th-generation tensor cores:
// single-CTA 128-row tiles (64-, 128- or 256-column), for shapes too small to
// fill the GPU with the CTA-pair kernel (k_proj_gate_wide_sm100.cu).
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
//                     out = h + alpha v for each branch.
//
// Per CTA (one per SM, persistent, 224 threads):
//   warp 4      TMA producer: A = e tile [128 x 64], B = W tile [BN x 64],
//               128-byte swizzle, STAGES-deep ring of smem slots;
//   warp 5      TMEM allocator and MMA issuer: tcgen05.mma.cta_group::1
//               kind::f16 (bf16 in, fp32 accumulate), M=128, N=BN, K=16,
//               accumulators double-buffered in TMEM (2*BN columns);
//   warp 6      TMA producer of h sub-tiles [128 x 64] into a 2- or 4-slot ring;
//   warps 0-3   epilogue: tcgen05.ld 32 columns at a time (warp w owns TMEM
//               lanes 32w..32w+31, i.e. rows of the tile), fused gate math
//               against h in shared memory; the value phase writes out over h
//               in place and each warp stores its 32 rows with TMA.
// Every mbarrier wait is bounded (kWaitLimitNs); on expiry the kernel records
// kDevErrTimeout, every role leaves its loop, outstanding MMAs are drained and
// TMEM is freed before the CTA exits.
#include "sm100_ptx.cuh"

namespace engram {

namespace {

using namespace sm100;

constexpr int BM = 128;
constexpr int BK = 64;                     // 64 bf16 = one 128-byte swizzle row
constexpr uint32_t A_BYTES = BM * BK * 2;  // 16 KB
constexpr int kThreads = 224;              // 7 warps
constexpr uint32_t H_BYTES = BM * 64 * 2;  // one sub-tile: 128 rows x 64 bf16, 128-B swizzle

template <int BN>
struct Cfg {
  // ring of h / out sub-tiles: with 64-column tiles there is room to hold a
  // chunk's sub-tiles of up to four branches while the mainloop runs
  static constexpr int H_SLOTS = BN == 64 ? 4 : 2;
  static constexpr uint32_t B_BYTES = BN * BK * 2;
  static constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int STAGES = ((229376 - H_SLOTS * H_BYTES) / STAGE_BYTES) > 8
                                    ? 8
                                    : ((229376 - H_SLOTS * H_BYTES) / STAGE_BYTES);
  static constexpr uint32_t TMEM_COLS = 2 * BN;
  static constexpr int NUM_BARS = 2 * STAGES + 4 + 2 * H_SLOTS + 1;
  static constexpr uint32_t BAR_BYTES = 8 * NUM_BARS + 16;
  static constexpr size_t SMEM =
      1024 + (size_t)STAGES * STAGE_BYTES + (size_t)H_SLOTS * H_BYTES + BAR_BYTES;
  static_assert(SMEM <= 232448, "shared memory budget");
};

template <int BN, int PHASE>
__global__ void __launch_bounds__(kThreads, 1)
    proj_gate_kernel(const __grid_constant__ CUtensorMap map_e,
                     const __grid_constant__ CUtensorMap map_w,
                     const __grid_constant__ CUtensorMap map_h,
                     const __grid_constant__ CUtensorMap map_out, GateArgs g) {
  using C = Cfg<BN>;
  constexpr int STAGES = C::STAGES;
  constexpr int H_SLOTS = C::H_SLOTS;
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
  const uint32_t drain_bar = bar0 + 8u * (2 * STAGES + 4 + 2 * H_SLOTS);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::NUM_BARS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int R = g.R, d = g.d, M = g.M;
  const int n_total = PHASE == 0 ? M * d : d;
  const int num_n = n_total / BN;
  const int num_tiles = ((R + BM - 1) / BM) * num_n;
  const int num_kb = (g.d_mem + BK - 1) / BK;
  // h sub-tiles per output tile: the key phase reads one branch, the value
  // phase every branch (v is shared, Eq. 6)
  const int nsub = PHASE == 3 ? 0 : (BN / 64) * (PHASE == 0 ? 1 : M);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull_bar(a), 1);
      mbar_init(tempty_bar(a), 4);
    }
    for (int s = 0; s < H_SLOTS; ++s) {
      mbar_init(hfull_bar(s), 1);
      mbar_init(hempty_bar(s), 4);  // every epilogue warp releases its rows
    }
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 5) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(C::TMEM_COLS));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  if (PHASE == 0) {
    // e (and its scales) come from the previous kernel; once it is complete
    // the value phase may launch
    griddep_wait();
    griddep_launch_dependents();
  } else {
    // the next call's gather (which writes the other e buffer) may start
    griddep_launch_dependents();
  }

  if (warp == 4) {
    // ------------------------------------------------- e / W producer (TMA)
    if (lane == 0) {
      asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&map_e) : "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&map_w) : "memory");
    }
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x) {
      const int m_blk = tile / num_n, n_blk = tile - m_blk * num_n;
      for (int kb = 0; kb < num_kb; ++kb) {
        if (lane == 0) ok = wait_ready(empty_bar(stage), phase ^ 1u, abort_flag, g.err);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        if (lane == 0) {
          mbar_expect_tx(full_bar(stage), C::STAGE_BYTES);
          tma_load_2d(sA + stage * A_BYTES, &map_e, full_bar(stage), kb * BK, m_blk * BM);
          tma_load_2d(sB + stage * C::B_BYTES, &map_w, full_bar(stage), kb * BK, n_blk * BN);
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
    for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x) {
      const int m_blk = tile / num_n, n0 = (tile - m_blk * num_n) * BN;
      for (int i = 0; i < nsub; ++i) {
        // columns of h viewed as [R, M*d]: key phase n0 + 64q; value phase mb*d + n0 + 64q
        const int x = PHASE == 0 ? n0 + 64 * i : (i % M) * d + n0 + 64 * (i / M);
        if (lane == 0) ok = wait_ready(hempty_bar(slot), phase ^ 1u, abort_flag, g.err);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        if (lane == 0) {
          mbar_expect_tx(hfull_bar(slot), H_BYTES);
          tma_load_2d(sH + slot * H_BYTES, &map_h, hfull_bar(slot), x, m_blk * BM);
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
    // ---------------------------------------------------------- MMA issuer
    constexpr uint32_t idesc = idesc_bf16<BM, BN>();
    int stage = 0, acc = 0;
    uint32_t phase = 0, acc_phase = 0;
    bool ok = true;
    for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x) {
      if (lane == 0) ok = wait_ready(tempty_bar(acc), acc_phase ^ 1u, abort_flag, g.err);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      tc_fence_after();
      const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
      for (int kb = 0; kb < num_kb; ++kb) {
        if (lane == 0) ok = wait_ready(full_bar(stage), phase, abort_flag, g.err);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        tc_fence_after();
        if (lane == 0) {
          const uint64_t ad = sw128_desc(sA + stage * A_BYTES);
          const uint64_t bd = sw128_desc(sB + stage * C::B_BYTES);
#pragma unroll
          for (int k = 0; k < BK / 16; ++k)
            umma_bf16(d_tmem, ad + 2u * k, bd + 2u * k, idesc, (kb | k) != 0);
          umma_commit(empty_bar(stage));  // slot free once these MMAs have read it
        }
        __syncwarp();
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (!ok) break;
      if (lane == 0) umma_commit(tfull_bar(acc));  // accumulator complete
      __syncwarp();
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
    if (lane == 0) {
      umma_commit(drain_bar);  // arrives once every MMA issued above has finished
      wait_drain(drain_bar, 0);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    // the key phase's partial sums are complete (and h no longer read by it)
    if (PHASE >= 1) griddep_wait();
    // Thread (warp w, lane l) owns tile row r = 32w + l: TMEM lane r and
    // row r of every h sub-tile in shared memory.
    const int r = warp * 32 + lane;
    int pending = -1;  // value phase: slot whose TMA store (this warp's rows) may still read it
    int acc = 0, hslot = 0;
    uint32_t acc_phase = 0, hphase = 0;
    bool ok = true;
    const int tiles_per_branch = d / g.key_tile;
    for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x) {
      const int m_blk = tile / num_n, n_blk = tile - m_blk * num_n;
      const int row = m_blk * BM + r;
      const bool valid = row < R;
      const int n0 = n_blk * BN;
      float al[kMaxBranches];
      if (PHASE >= 1) {
        // alpha from the key phase's per-tile partial sums (Eq. 4 / Eq. 6)
#pragma unroll
        for (int mb = 0; mb < kMaxBranches; ++mb) {
          al[mb] = 0.f;
          if (mb < M && valid) {
            if (g.alpha_in) {
              al[mb] = g.alpha_in[(int64_t)row * M + mb];
            } else {
              al[mb] = row_alpha<1>(g.partials, R, row, mb, tiles_per_branch, d, g.eps,
                                    g.inv_sqrt_d);
              if (g.alpha && n_blk == 0) g.alpha[(int64_t)row * M + mb] = al[mb];
            }
          }
        }
      }
      if (lane == 0) ok = wait_ready(tfull_bar(acc), acc_phase, abort_flag, g.err);
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
          if (lane == 0) ok = wait_ready(hfull_bar(hslot), hphase, abort_flag, g.err);
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
      } else if (PHASE == 3) {
        // values for the short convolution (Eq. 5): v in fp32 and the row's
        // sum of v^2 over this tile
        float svv = 0.f;
#pragma unroll 1
        for (int q = 0; q < BN / 64; ++q) {
          __syncwarp();
          tmem_ld32(taddr + q * 64, v);
          tmem_ld32(taddr + q * 64 + 32, v + 32);
#pragma unroll
          for (int i = 0; i < 64; ++i) svv = fmaf(v[i], v[i], svv);
          if (valid) {
            float4* vp = reinterpret_cast<float4*>(g.vals + (int64_t)row * d + n0 + q * 64);
#pragma unroll
            for (int c = 0; c < 16; ++c)
              vp[c] = make_float4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
          }
        }
        if (valid) g.vv[(int64_t)n_blk * R + row] = svv;
      } else {
#pragma unroll 1
        for (int q = 0; q < BN / 64; ++q) {
          __syncwarp();
          tmem_ld32(taddr + q * 64, v);
          tmem_ld32(taddr + q * 64 + 32, v + 32);
#pragma unroll 1
          for (int mb = 0; mb < M; ++mb) {
            if (lane == 0) ok = wait_ready(hfull_bar(hslot), hphase, abort_flag, g.err);
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
            if (lane == 0) {
              // this warp's 32 rows of the slot (map_out has 32-row boxes;
              // rows past R are clipped, a warp with none commits an empty
              // group), then hand back the previous slot once this warp's
              // store of it has read it
              if (m_blk * BM + warp * 32 < R)
                tma_store_2d(&map_out, sH + hslot * H_BYTES + warp * 32 * 128,
                             mb * d + n0 + q * 64, m_blk * BM + warp * 32);
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
          if (!ok) break;
        }
        if (!ok) break;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tempty_bar(acc));
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
    if (PHASE == 1 && lane == 0) {
      asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
      if (pending >= 0 && ok) mbar_arrive(hempty_bar(pending));
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 5) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                 "r"(C::TMEM_COLS));
  }
}

template <int BN, int PHASE>
cudaError_t launch_bn(const ProjMaps& maps, const GateArgs& g, int grid, cudaStream_t stream) {
  auto kern = proj_gate_kernel<BN, PHASE>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)Cfg<BN>::SMEM);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t lc = {};
  lc.gridDim = dim3(grid);
  lc.blockDim = dim3(kThreads);
  lc.dynamicSmemBytes = Cfg<BN>::SMEM;
  lc.stream = stream;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  lc.attrs = at;
  lc.numAttrs = g.pdl ? 1 : 0;
  e = cudaLaunchKernelEx(&lc, kern, maps.e, maps.w, maps.h, maps.out, g);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

// One thread per (branch, row), rows fastest: the warp's loads of a tile's
// partials are one coalesced 512-byte read.  Blocks of 128 threads: a short
// call's blocks then occupy few SMs while they wait for the key launch (more,
// smaller blocks measured slower: they held SMs the value launch needed).
__global__ void __launch_bounds__(128) row_alpha_kernel(GateArgs g, float* alpha) {
  griddep_launch_dependents();  // the value launch may set up and stream its operands
  griddep_wait();               // the key launch's partial sums are complete
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (int64_t)g.R * g.M) return;
  const int mb = (int)(i / g.R);
  const int64_t row = i - (int64_t)mb * g.R;
  alpha[row * g.M + mb] = row_alpha<16>(g.partials, g.R, row, mb, g.d / g.key_tile, g.d, g.eps,
                                        g.inv_sqrt_d);
}

}  // namespace

cudaError_t launch_row_alpha(const GateArgs& g, float* alpha, cudaStream_t stream) {
  if (g.R == 0) return cudaSuccess;
  if (!alpha || g.key_tile <= 0 || g.d % g.key_tile) return cudaErrorInvalidValue;
  const int64_t n = (int64_t)g.R * g.M;
  cudaLaunchConfig_t lc = {};
  lc.gridDim = dim3((unsigned)((n + 127) / 128));
  lc.blockDim = dim3(128);
  lc.stream = stream;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  lc.attrs = at;
  lc.numAttrs = g.pdl ? 1 : 0;
  cudaError_t e = cudaLaunchKernelEx(&lc, row_alpha_kernel, g, alpha);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

int sm100_stages(int bn) {
  return bn == 256 ? Cfg<256>::STAGES : bn == 128 ? Cfg<128>::STAGES : Cfg<64>::STAGES;
}

cudaError_t launch_proj_gate_sm100(int phase, int bn, const ProjMaps& maps, const GateArgs& g,
                                   int grid, cudaStream_t stream) {
  if (g.R == 0) return cudaSuccess;
  switch (bn * 2 + phase) {
    case 512: return launch_bn<256, 0>(maps, g, grid, stream);
    case 513: return launch_bn<256, 1>(maps, g, grid, stream);
    case 256: return launch_bn<128, 0>(maps, g, grid, stream);
    case 257: return launch_bn<128, 1>(maps, g, grid, stream);
    case 128: return launch_bn<64, 0>(maps, g, grid, stream);
    case 129: return launch_bn<64, 1>(maps, g, grid, stream);
    case 515: return launch_bn<256, 3>(maps, g, grid, stream);
    case 259: return launch_bn<128, 3>(maps, g, grid, stream);
    case 131: return launch_bn<64, 3>(maps, g, grid, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace engram
