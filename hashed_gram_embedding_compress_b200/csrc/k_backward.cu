// Backward of the lookup-and-gate step (training).
//
// "Conditional Memory via Scalable Lookup", section 2.3 Eq. (3)-(4) and
// section 2.4 Eq. (6) give the forward; this file holds the hand-written
// kernels of its exact derivative apart from the dense contractions (k and v
// recomputed, the weight and memory-vector gradients), which run on the
// CTA-pair tcgen05 GEMM of k_gemm_sm100.cu, issued by the ABI layer:
//
//   per row r and branch m, with k = W_K^(m) e, v = W_V e,
//   rh = (mean(h^2) + eps)^-1/2, rk likewise, qn = h rh w_q, kn = k rk w_k,
//   s = qn . kn / sqrt(d), alpha = sigmoid(s), out = h + alpha v:
//     dalpha = dout . v,  dv += alpha dout,  ds = dalpha alpha (1 - alpha),
//     dqn = ds kn / sqrt(d),  dkn = ds qn / sqrt(d),
//     dw_q += dqn h rh,  dw_k += dkn k rk,
//     u_q = dqn w_q:  dh = dout + rh u_q - rh^3 / d h (u_q . h),
//     u_k = dkn w_k:  dk = rk u_k - rk^3 / d k (u_k . k).
//
// gate_backward_ring_kernel: a CTA of d / 8 threads per row at a time
// (grid-stride, two CTAs per SM); thread 0 streams the rows' h, dout and kv
// into a ring of three shared-memory slots with bulk copies two rows ahead,
// so the loads of the next rows overlap the reductions of the current one.
// One block reduction (of four sums) and one barrier per branch and row.
// dw_q and dw_k are summed per CTA (in registers with one branch, else in
// shared memory; each thread owns its columns) and reduced over the CTAs in a
// fixed order by dnorm_reduce_kernel (deterministic).
// gate_backward_kernel is the same arithmetic with the row in registers and
// no ring, for rows too long for three slots.
// table_grad_kernel adds the slices of de into fp32 table gradients.
#include "sm100_ptx.cuh"

namespace engram {

namespace {

constexpr int kBwThreads = 256;

__device__ __forceinline__ float load_elt(const void* p, int64_t i, bool bf16) {
  if (bf16) return __uint_as_float((uint32_t)(reinterpret_cast<const uint16_t*>(p)[i]) << 16);
  return reinterpret_cast<const float*>(p)[i];
}

// Round to nearest even (the value is finite).
__device__ __forceinline__ uint16_t bf16_rne(float x) {
  uint32_t u = __float_as_uint(x);
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

__device__ __forceinline__ void store_elt(void* p, int64_t i, float x, bool bf16) {
  if (bf16)
    reinterpret_cast<uint16_t*>(p)[i] = bf16_rne(x);
  else
    reinterpret_cast<float*>(p)[i] = x;
}

// Sum of N values over the block (256 threads); every thread gets the result.
template <int N>
__device__ __forceinline__ void block_sum(float (&x)[N], float* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int n = 0; n < N; ++n)
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x[n] += __shfl_xor_sync(0xffffffffu, x[n], o);
  __syncthreads();  // the previous reduction's readers are done with red
  if (lane == 0)
#pragma unroll
    for (int n = 0; n < N; ++n) red[warp * N + n] = x[n];
  __syncthreads();
#pragma unroll
  for (int n = 0; n < N; ++n) {
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < kBwThreads / 32; ++w) s += red[w * N + n];
    x[n] = s;
  }
}

template <int PER>
__global__ void __launch_bounds__(kBwThreads) gate_backward_kernel(GateBwArgs a) {
  extern __shared__ float sm[];
  float* red = sm;                               // [8 warps][4]
  float* s_dwq = sm + 32;                        // [M][d]: this CTA's sum of dqn h rh
  float* s_dwk = s_dwq + (int64_t)a.M * a.d;     // [M][d]
  const int d = a.d, M = a.M, tid = threadIdx.x;
  const int64_t nkv = (int64_t)(M + 1) * d;
  const float inv_d = 1.f / (float)d;
  for (int64_t i = tid; i < 2LL * M * d; i += kBwThreads) s_dwq[i] = 0.f;

  for (int64_t r = blockIdx.x; r < a.R; r += gridDim.x) {
    const float* kv = a.kv + r * nkv;
    float v[PER], dv[PER];
#pragma unroll
    for (int j = 0; j < PER; ++j) {
      const int c = tid + kBwThreads * j;
      v[j] = c < d ? kv[(int64_t)M * d + c] : 0.f;
      dv[j] = 0.f;
    }
    for (int m = 0; m < M; ++m) {
      const int64_t base = (r * M + m) * (int64_t)d;
      const float* wq = a.w_q + (int64_t)m * d;
      const float* wk = a.w_k + (int64_t)m * d;
      float h[PER], k[PER], g[PER];
      float sums[4] = {0.f, 0.f, 0.f, 0.f};  // sum h^2, sum k^2, sum (h w_q)(k w_k), dout . v
#pragma unroll
      for (int j = 0; j < PER; ++j) {
        const int c = tid + kBwThreads * j;
        h[j] = k[j] = g[j] = 0.f;
        if (c < d) {
          h[j] = load_elt(a.h, base + c, a.bf16);
          k[j] = kv[(int64_t)m * d + c];
          g[j] = load_elt(a.dout, base + c, a.bf16);
          sums[0] += h[j] * h[j];
          sums[1] += k[j] * k[j];
          sums[2] += (h[j] * wq[c]) * (k[j] * wk[c]);
          sums[3] += g[j] * v[j];
        }
      }
      block_sum(sums, red);
      const float rh = rsqrtf(sums[0] * inv_d + a.eps);
      const float rk = rsqrtf(sums[1] * inv_d + a.eps);
      const float alpha = 1.f / (1.f + __expf(-sums[2] * rh * rk * a.inv_sqrt_d));
      const float ds = sums[3] * alpha * (1.f - alpha);
      // dqn_c = ds kn_c / sqrt(d), dkn_c = ds qn_c / sqrt(d)
      const float cq = ds * rk * a.inv_sqrt_d;  // dqn_c = cq k_c w_k,c
      const float ck = ds * rh * a.inv_sqrt_d;  // dkn_c = ck h_c w_q,c
      float u[2] = {0.f, 0.f};                  // u_q . h, u_k . k
#pragma unroll
      for (int j = 0; j < PER; ++j) {
        const int c = tid + kBwThreads * j;
        if (c < d) {
          const float dqn = cq * k[j] * wk[c], dkn = ck * h[j] * wq[c];
          s_dwq[(int64_t)m * d + c] += dqn * h[j] * rh;
          s_dwk[(int64_t)m * d + c] += dkn * k[j] * rk;
          u[0] += dqn * wq[c] * h[j];
          u[1] += dkn * wk[c] * k[j];
          dv[j] += alpha * g[j];
        }
      }
      block_sum(u, red);
      const float th = rh * rh * rh * inv_d * u[0], tk = rk * rk * rk * inv_d * u[1];
#pragma unroll
      for (int j = 0; j < PER; ++j) {
        const int c = tid + kBwThreads * j;
        if (c < d) {
          const float dqn = cq * k[j] * wk[c], dkn = ck * h[j] * wq[c];
          store_elt(a.dh, base + c, g[j] + rh * dqn * wq[c] - th * h[j], a.bf16);
          store_elt(a.dkv, r * nkv + (int64_t)m * d + c, rk * dkn * wk[c] - tk * k[j], a.bf16);
        }
      }
    }
#pragma unroll
    for (int j = 0; j < PER; ++j) {
      const int c = tid + kBwThreads * j;
      if (c < d) store_elt(a.dkv, r * nkv + (int64_t)M * d + c, dv[j], a.bf16);
    }
  }
  __syncthreads();
  float* part = a.partials + (int64_t)blockIdx.x * 2 * M * d;
  for (int64_t i = tid; i < 2LL * M * d; i += kBwThreads) part[i] = s_dwq[i];
}

constexpr int kRing = 3;

// Bytes of one ring slot: h and dout rows (element size elt) and the kv row (fp32).
__host__ __device__ inline size_t ring_slot_bytes(int M, int d, int elt) {
  return (size_t)2 * M * d * elt + (size_t)(M + 1) * d * 4;
}

using u64 = unsigned long long;

// Four consecutive elements as two packed fp32 pairs: bf16 (one 8-byte load)
// or fp32 (one 16-byte load).
template <bool BF16>
__device__ __forceinline__ void load4(const void* base, int64_t i, u64& p0, u64& p1) {
  if (BF16) {
    const uint2 u = *reinterpret_cast<const uint2*>(reinterpret_cast<const uint16_t*>(base) + i);
    p0 = sm100::bf16x2_to_f2(u.x);
    p1 = sm100::bf16x2_to_f2(u.y);
  } else {
    const uint4 u = *reinterpret_cast<const uint4*>(reinterpret_cast<const float*>(base) + i);
    p0 = sm100::f2_pack(u.x, u.y);
    p1 = sm100::f2_pack(u.z, u.w);
  }
}

__device__ __forceinline__ void load4f(const float* p, u64& p0, u64& p1) {
  const uint4 u = *reinterpret_cast<const uint4*>(p);
  p0 = sm100::f2_pack(u.x, u.y);
  p1 = sm100::f2_pack(u.z, u.w);
}

__device__ __forceinline__ void ldg4f(const float* p, u64& p0, u64& p1) {
  const uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
  p0 = sm100::f2_pack(u.x, u.y);
  p1 = sm100::f2_pack(u.z, u.w);
}

template <bool BF16>
__device__ __forceinline__ void store4(void* base, int64_t i, u64 p0, u64 p1) {
  const float2 a = sm100::f2_unpack(p0), b = sm100::f2_unpack(p1);
  if (BF16) {
    *reinterpret_cast<uint2*>(reinterpret_cast<uint16_t*>(base) + i) =
        make_uint2(sm100::pack2(a.x, a.y), sm100::pack2(b.x, b.y));
  } else {
    *reinterpret_cast<float4*>(reinterpret_cast<float*>(base) + i) = make_float4(a.x, a.y, b.x, b.y);
  }
}

__device__ __forceinline__ u64 f2s(float x) {  // {x, x}
  return sm100::f2_pack(__float_as_uint(x), __float_as_uint(x));
}
__device__ __forceinline__ float f2sum(u64 p) {
  const float2 v = sm100::f2_unpack(p);
  return v.x + v.y;
}

// One CTA per row at a time.  Thread t owns columns [4t, 4t + 4) and
// [4t + 4T, 4t + 4T + 4) (T = blockDim.x = d / 8 rounded up to whole warps),
// so every shared-memory load of a warp reads consecutive words; the branch's
// h, dout, k and v stay in registers as packed fp32 pairs (fma.rn.f32x2)
// through the three passes.  The derivative is arranged to share products:
// with kw = k w_k and hw = h w_q, u_q . h = cq sum(kw hw) and u_k . k =
// ck sum(kw hw) = the first reduction's third sum times cq or ck: one block
// reduction per branch.  M1: one branch, whose weight-gradient sums stay in
// registers.
template <bool BF16, bool M1>
__global__ void __maxnreg__(96) gate_backward_ring_kernel(GateBwArgs a) {
  extern __shared__ __align__(128) unsigned char smraw[];
  const int d = a.d, M = a.M, tid = threadIdx.x, T = blockDim.x;
  const int nwarps = T >> 5;
  const int cA = 4 * tid, cB = 4 * tid + 4 * T;  // this thread's two groups of 4 columns
  const bool actA = cA < d, actB = cB < d;
  constexpr int elt = BF16 ? 2 : 4;
  const int64_t nkv = (int64_t)(M + 1) * d;
  const float inv_d = 1.f / (float)d;
  const uint32_t hb = (uint32_t)M * d * elt, kvb = (uint32_t)nkv * 4;
  const size_t slot_bytes = ring_slot_bytes(M, d, elt);
  unsigned char* ring = smraw;
  float* red = reinterpret_cast<float*>(ring + kRing * slot_bytes);   // [2][32 warps][4]
  // M > 1: the weight-gradient sums [M][d] each; one branch (sums in
  // registers): the RMSNorm weights w_q, w_k [d] each, read there every row
  float* s_dwq = red + 256;
  float* s_dwk = s_dwq + (int64_t)M * d;
  uint64_t* full = reinterpret_cast<uint64_t*>(s_dwk + (int64_t)M * d);  // [kRing]
  volatile int* flag = reinterpret_cast<volatile int*>(full + kRing);
  if (!M1) {
    for (int64_t i = tid; i < 2LL * M * d; i += T) s_dwq[i] = 0.f;
  } else {
    for (int i = tid; i < d; i += T) {
      s_dwq[i] = __ldg(a.w_q + i);
      s_dwk[i] = __ldg(a.w_k + i);
    }
  }
  if (tid == 0) {
    for (int i = 0; i < kRing; ++i) sm100::mbar_init(sm100::smem_u32(full + i), 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  // the branch's RMSNorm weights; with one branch the weight-gradient sums
  // stay in registers
  u64 WQ[4] = {0, 0, 0, 0}, WK[4] = {0, 0, 0, 0}, DQ[4] = {0, 0, 0, 0}, DK[4] = {0, 0, 0, 0};
  auto load_w = [&](int m) {
    if (M1) {  // from shared memory (two CTAs' rows and the ring leave little L1)
      if (actA) {
        load4f(s_dwq + cA, WQ[0], WQ[1]);
        load4f(s_dwk + cA, WK[0], WK[1]);
      }
      if (actB) {
        load4f(s_dwq + cB, WQ[2], WQ[3]);
        load4f(s_dwk + cB, WK[2], WK[3]);
      }
      return;
    }
    if (actA) {
      ldg4f(a.w_q + m * d + cA, WQ[0], WQ[1]);
      ldg4f(a.w_k + m * d + cA, WK[0], WK[1]);
    }
    if (actB) {
      ldg4f(a.w_q + m * d + cB, WQ[2], WQ[3]);
      ldg4f(a.w_k + m * d + cB, WK[2], WK[3]);
    }
  };
  // row i of this CTA is blockIdx.x + i gridDim.x, staged in slot i % kRing
  const int64_t n_rows = a.R > blockIdx.x ? (a.R - 1 - blockIdx.x) / gridDim.x + 1 : 0;
  int64_t issued = 0;  // rows whose copies thread 0 has issued
  auto issue_next = [&]() {
    if (issued >= n_rows) return;
    const int64_t r = blockIdx.x + issued * (int64_t)gridDim.x;
    const int slot = (int)(issued % kRing);
    const uint32_t bar = sm100::smem_u32(full + slot);
    const uint32_t dst = sm100::smem_u32(ring + slot * slot_bytes);
    sm100::mbar_expect_tx(bar, 2 * hb + kvb);
    sm100::bulk_load(dst, (const char*)a.h + r * hb, hb, bar);
    sm100::bulk_load(dst + hb, (const char*)a.dout + r * hb, hb, bar);
    sm100::bulk_load(dst + 2 * hb, a.kv + r * nkv, kvb, bar);
    ++issued;
  };
  // bounded wait for the copies of row i
  auto wait_row = [&](int64_t i) -> bool {
    const uint32_t bar = sm100::smem_u32(full + (i % kRing));
    const uint32_t par = (uint32_t)(i / kRing) & 1u;
    if (sm100::mbar_try_wait(bar, par)) return true;
    const uint64_t t0 = sm100::globaltimer();
    while (!sm100::mbar_try_wait(bar, par))
      if (sm100::globaltimer() - t0 > sm100::kWaitLimitNs) return false;
    return true;
  };
  if (tid == 0) {
    *flag = 1;
    for (int i = 0; i < kRing - 1; ++i) issue_next();
  }
  __syncthreads();
  int rb = 0;  // which half of `red` the next reduction uses
  // Sum of the four values x[0..3] over the block with one barrier, every
  // thread getting the four totals.  Within a warp the four sums share one
  // shuffle tree: after the exchanges across lane bits 4 and 3 each lane
  // carries one of the four values (v = 2 bit4 + bit3), whose sum over the
  // remaining lane bits the last three exchanges complete.  Warp w's totals go
  // to red; after the barrier lane l < nwarps takes warp l's four and the same
  // tree sums them over the warps, and four shuffles hand the totals to every
  // lane.  The halves of `red` alternate, so a reduction never overwrites
  // values still being read (a thread writes a half again only after the next
  // row's barrier, which every thread reaches after reading this half).
  auto tree4 = [](float x0, float x1, float x2, float x3, int lane) -> float {
    const bool b4 = lane & 16, b3 = lane & 8;
    float k0 = b4 ? x2 : x0, k1 = b4 ? x3 : x1;
    const float s0 = b4 ? x0 : x2, s1 = b4 ? x1 : x3;
    k0 += __shfl_xor_sync(0xffffffffu, s0, 16);
    k1 += __shfl_xor_sync(0xffffffffu, s1, 16);
    float c = b3 ? k1 : k0;
    c += __shfl_xor_sync(0xffffffffu, b3 ? k0 : k1, 8);
    c += __shfl_xor_sync(0xffffffffu, c, 4);
    c += __shfl_xor_sync(0xffffffffu, c, 2);
    c += __shfl_xor_sync(0xffffffffu, c, 1);
    return c;  // the total of value 2 bit4 + bit3 over the warp's lanes
  };
  auto bsum = [&](float* x) {
    const int lane = tid & 31, warp = tid >> 5;
    const int v = ((lane >> 4) & 1) * 2 + ((lane >> 3) & 1);
    const float c = tree4(x[0], x[1], x[2], x[3], lane);
    float* rr = red + rb * 128;
    if ((lane & 7) == 0) rr[warp * 4 + v] = c;
    __syncthreads();
    float4 q = make_float4(0.f, 0.f, 0.f, 0.f);
    if (lane < nwarps) q = reinterpret_cast<const float4*>(rr)[lane];
    const float t = tree4(q.x, q.y, q.z, q.w, lane);
    x[0] = __shfl_sync(0xffffffffu, t, 0);
    x[1] = __shfl_sync(0xffffffffu, t, 8);
    x[2] = __shfl_sync(0xffffffffu, t, 16);
    x[3] = __shfl_sync(0xffffffffu, t, 24);
    rb ^= 1;
  };
  // One barrier per row (the block reduction's).  Every thread waits for row
  // i's copies itself; after row i's barrier every thread has finished with
  // row i - 1's slot, so thread 0 then refills it with row i + kRing - 1.  A
  // timed-out wait is acted on after the barrier, by every thread alike.
  int64_t i = 0;
  for (; i < n_rows; ++i) {
    const int64_t r = blockIdx.x + i * (int64_t)gridDim.x;
    if (!wait_row(i)) {
      *flag = 0;
      atomicOr(a.err, kDevErrTimeout);
    }
    const unsigned char* slot = ring + (i % kRing) * slot_bytes;
    const void* hs = slot;
    const void* gs = slot + hb;
    const float* kv = reinterpret_cast<const float*>(slot + 2 * hb);
    u64 V[4] = {0, 0, 0, 0}, DV[4] = {0, 0, 0, 0};
    if (actA) load4f(kv + (int64_t)M * d + cA, V[0], V[1]);
    if (actB) load4f(kv + (int64_t)M * d + cB, V[2], V[3]);
    bool stop = false;
    for (int m = 0; m < M; ++m) {
      const int64_t base = (r * M + m) * (int64_t)d;
      const int sb = m * d;
      load_w(m);  // shared memory with one branch, else L1
      u64 H[4] = {0, 0, 0, 0}, G[4] = {0, 0, 0, 0}, K[4] = {0, 0, 0, 0};
      if (actA) {
        load4<BF16>(hs, sb + cA, H[0], H[1]);
        load4<BF16>(gs, sb + cA, G[0], G[1]);
        load4f(kv + sb + cA, K[0], K[1]);
      }
      if (actB) {
        load4<BF16>(hs, sb + cB, H[2], H[3]);
        load4<BF16>(gs, sb + cB, G[2], G[3]);
        load4f(kv + sb + cB, K[2], K[3]);
      }
      // sum h^2, sum k^2, sum (h w_q)(k w_k), dout . v
      u64 s0 = 0, s1 = 0, s2 = 0, s3 = 0;
#pragma unroll
      for (int p = 0; p < 4; ++p) {
        s0 = sm100::f2_fma(H[p], H[p], s0);
        s1 = sm100::f2_fma(K[p], K[p], s1);
        s2 = sm100::f2_fma(sm100::f2_mul(H[p], WQ[p]), sm100::f2_mul(K[p], WK[p]), s2);
        s3 = sm100::f2_fma(G[p], V[p], s3);
      }
      float sums[4] = {f2sum(s0), f2sum(s1), f2sum(s2), f2sum(s3)};
      bsum(sums);
      if (m == 0) {
        if (!*flag) {  // a wait timed out: leave before any store of this row
          stop = true;
          break;
        }
        if (tid == 0) issue_next();  // row i + kRing - 1, into the slot row i - 1 left
      }
      const float rh = rsqrtf(sums[0] * inv_d + a.eps);
      const float rk = rsqrtf(sums[1] * inv_d + a.eps);
      const float alpha = 1.f / (1.f + __expf(-sums[2] * rh * rk * a.inv_sqrt_d));
      const float ds = sums[3] * alpha * (1.f - alpha);
      const float cq = ds * rk * a.inv_sqrt_d;  // dqn_c = cq k_c w_k,c
      const float ck = ds * rh * a.inv_sqrt_d;  // dkn_c = ck h_c w_q,c
      // dw_q += cq rh h kw; dw_k += ck rk k hw; dv += alpha dout
      const u64 cqr = f2s(cq * rh), ckr = f2s(ck * rk), al = f2s(alpha);
      float U[1] = {f2sum(s2)};  // sum kw hw (this thread's part) is s2
      if (M1) {
#pragma unroll
        for (int p = 0; p < 4; ++p) {
          const u64 hk = sm100::f2_mul(H[p], K[p]);
          DQ[p] = sm100::f2_fma(cqr, sm100::f2_mul(hk, WK[p]), DQ[p]);
          DK[p] = sm100::f2_fma(ckr, sm100::f2_mul(hk, WQ[p]), DK[p]);
        }
      } else {
        u64 aq[4], ak[4];
        if (actA) {
          load4f(s_dwq + sb + cA, aq[0], aq[1]);
          load4f(s_dwk + sb + cA, ak[0], ak[1]);
        }
        if (actB) {
          load4f(s_dwq + sb + cB, aq[2], aq[3]);
          load4f(s_dwk + sb + cB, ak[2], ak[3]);
        }
#pragma unroll
        for (int p = 0; p < 4; ++p) {
          const u64 hk = sm100::f2_mul(H[p], K[p]);
          aq[p] = sm100::f2_fma(cqr, sm100::f2_mul(hk, WK[p]), aq[p]);
          ak[p] = sm100::f2_fma(ckr, sm100::f2_mul(hk, WQ[p]), ak[p]);
        }
        if (actA) {
          store4<false>(s_dwq, sb + cA, aq[0], aq[1]);
          store4<false>(s_dwk, sb + cA, ak[0], ak[1]);
        }
        if (actB) {
          store4<false>(s_dwq, sb + cB, aq[2], aq[3]);
          store4<false>(s_dwk, sb + cB, ak[2], ak[3]);
        }
      }
#pragma unroll
      for (int p = 0; p < 4; ++p) DV[p] = sm100::f2_fma(al, G[p], DV[p]);
      // the first reduction already summed kw hw (s2) over the block
      U[0] = sums[2];
      const float th = rh * rh * rh * inv_d * (cq * U[0]);
      const float tk = rk * rk * rk * inv_d * (ck * U[0]);
      // dh = dout + (rh cq) kw w_q - th h;  dk = (rk ck) hw w_k - tk k
      const u64 a_h = f2s(rh * cq), a_k = f2s(rk * ck), m_th = f2s(-th), m_tk = f2s(-tk);
      u64 OH[4], OK[4];
#pragma unroll
      for (int p = 0; p < 4; ++p) {
        const u64 ww = sm100::f2_mul(WQ[p], WK[p]);
        OH[p] = sm100::f2_fma(m_th, H[p], sm100::f2_fma(a_h, sm100::f2_mul(K[p], ww), G[p]));
        OK[p] = sm100::f2_fma(m_tk, K[p], sm100::f2_mul(a_k, sm100::f2_mul(H[p], ww)));
      }
      if (actA) {
        store4<BF16>(a.dh, base + cA, OH[0], OH[1]);
        store4<BF16>(a.dkv, r * nkv + sb + cA, OK[0], OK[1]);
      }
      if (actB) {
        store4<BF16>(a.dh, base + cB, OH[2], OH[3]);
        store4<BF16>(a.dkv, r * nkv + sb + cB, OK[2], OK[3]);
      }
    }
    if (stop) break;
    if (actA) store4<BF16>(a.dkv, r * nkv + (int64_t)M * d + cA, DV[0], DV[1]);
    if (actB) store4<BF16>(a.dkv, r * nkv + (int64_t)M * d + cB, DV[2], DV[3]);
  }
  __syncthreads();
  float* part = a.partials + (int64_t)blockIdx.x * 2 * M * d;
  if (M1) {
    if (actA) {
      store4<false>(part, cA, DQ[0], DQ[1]);
      store4<false>(part, d + cA, DK[0], DK[1]);
    }
    if (actB) {
      store4<false>(part, cB, DQ[2], DQ[3]);
      store4<false>(part, d + cB, DK[2], DK[3]);
    }
  } else {
    for (int64_t j = tid; j < 2LL * M * d; j += T) part[j] = s_dwq[j];
  }
  // after a timeout: the copies still in flight land before the CTA leaves
  // (each waited for a bounded time)
  if (tid == 0)
    for (int64_t k = i; k < issued; ++k) (void)wait_row(k);
}

// dnorm_q[i] += sum over CTAs b of partials[b][0][i], dnorm_k likewise, in
// a fixed order (deterministic): a block of 32 x 8 threads takes 32
// consecutive columns; thread (x, y) sums the CTAs b = y, y + 8, ... in
// order (the 32 columns of one b are one coalesced 128-byte read), then the
// 8 partial sums of a column are added in order of y.
__global__ void __launch_bounds__(256) dnorm_reduce_kernel(const float* partials, int nblocks,
                                                           int64_t n, float* dnorm_q,
                                                           float* dnorm_k) {
  __shared__ float part[8][33];
  const int x = threadIdx.x & 31, y = threadIdx.x >> 5;
  for (int64_t c0 = (int64_t)blockIdx.x * 32; c0 < 2 * n; c0 += (int64_t)gridDim.x * 32) {
    const int64_t i = c0 + x;
    float s = 0.f;
    if (i < 2 * n)
      for (int b = y; b < nblocks; b += 8) s += partials[(int64_t)b * 2 * n + i];
    part[y][x] = s;
    __syncthreads();
    if (y == 0 && i < 2 * n) {
      float t = 0.f;
#pragma unroll
      for (int k = 0; k < 8; ++k) t += part[k][x];
      if (i < n) {
        if (dnorm_q) dnorm_q[i] += t;
      } else if (dnorm_k) {
        dnorm_k[i - n] += t;
      }
    }
    __syncthreads();
  }
}

// dtab[s][idx[r][s]][c..c+3] += de[r][s d_h + c..c+3]: one thread per four
// elements of de, added by one 16-byte vector reduction in L2 (d_head is a
// multiple of 4 and the gradient rows 16-byte aligned).
__global__ void table_grad_kernel(TableGradArgs a) {
  const int32_t q_per_row = a.d_head >> 2;  // float4 per table row
  const int64_t per_row = (int64_t)a.S * q_per_row;
  const int64_t total = a.rows * per_row;
  const float4* de4 = reinterpret_cast<const float4*>(a.de);
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = i / per_row;
    const int32_t rem = (int32_t)(i - r * per_row);
    const int32_t s = rem / q_per_row, c = (rem - s * q_per_row) * 4;
    const int64_t z = a.idx[r * a.S + s];
    if (z < 0 || z >= a.primes[s]) {
      if (c == 0) atomicOr(a.err, kDevErrIndex);
      continue;
    }
    float* dst;
    if (a.shards == 1) {
      dst = a.dtables[s] + z * a.d_head;
    } else {
      // row-sharded: owner z % N at local row z / N (z < 2^31)
      const uint32_t q = (uint32_t)z / (uint32_t)a.shards;
      dst = a.dtables[s * a.shards + (int)((uint32_t)z - q * (uint32_t)a.shards)] +
            (int64_t)q * a.d_head;
    }
    const float4 v = __ldg(de4 + i);
    asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(dst + c), "f"(v.x),
                 "f"(v.y), "f"(v.z), "f"(v.w)
                 : "memory");
  }
}

int grid_cap(int64_t work, int threads) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  int64_t blocks = (work + threads - 1) / threads;
  const int64_t cap = (int64_t)sms * 16;
  if (blocks > cap) blocks = cap;
  return blocks < 1 ? 1 : (int)blocks;
}

template <int PER>
cudaError_t launch_gate_bw(const GateBwArgs& a, int grid, size_t smem, cudaStream_t stream) {
  auto kern = gate_backward_kernel<PER>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  kern<<<grid, kBwThreads, smem, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace

size_t gate_bw_smem(int M, int d) { return (32 + 2 * (size_t)M * d) * sizeof(float); }

namespace {

// Resident CTAs per SM of one instantiation (registers and shared memory).
template <int PER>
int resident(size_t smem) {
  auto kern = gate_backward_kernel<PER>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
      cudaSuccess)
    return 1;
  int n = 1;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, kBwThreads, smem) != cudaSuccess)
    return 1;
  return n < 1 ? 1 : n;
}

}  // namespace

// One CTA per resident slot on every SM (each loops over rows), at most R.
int gate_bw_grid(int M, int d, int64_t R, int elt) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const size_t rsm = gate_bw_ring_smem(M, d, elt);
  if (rsm <= 232448 && d % 8 == 0 && ((d / 8 + 31) / 32) * 32 <= 1024) {
    // the ring kernel: as many CTAs per SM as its registers and shared memory allow
    int per_sm = 1;
    const int threads = ((d / 8 + 31) / 32) * 32;
    auto occ = [&](auto kern) {
      if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)rsm) ==
              cudaSuccess &&
          cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, threads, rsm) == cudaSuccess)
        return;
      per_sm = 1;
    };
    if (elt == 2)
      occ(gate_backward_ring_kernel<true, false>);
    else
      occ(gate_backward_ring_kernel<false, false>);
    if (per_sm < 1) per_sm = 1;
    int64_t grid = (int64_t)sms * per_sm;
    if (grid > R) grid = R;
    return grid < 1 ? 1 : (int)grid;
  }
  const size_t smem = gate_bw_smem(M, d);
  const int per = (d + kBwThreads - 1) / kBwThreads;
  const int per_sm = per <= 1   ? resident<1>(smem)
                     : per <= 2 ? resident<2>(smem)
                     : per <= 4 ? resident<4>(smem)
                     : per <= 8 ? resident<8>(smem)
                     : per <= 12 ? resident<12>(smem)
                                 : resident<16>(smem);
  int64_t grid = (int64_t)sms * per_sm;
  if (grid > R) grid = R;
  return grid < 1 ? 1 : (int)grid;
}

size_t gate_bw_ring_smem(int M, int d, int elt) {
  return kRing * ring_slot_bytes(M, d, elt) + 256 * sizeof(float) + 2 * (size_t)M * d * 4 +
         kRing * 8 + 16;
}

namespace {

int ring_threads(int d) { return ((d / 8 + 31) / 32) * 32; }

template <bool BF16, bool M1>
cudaError_t launch_ring(const GateBwArgs& a, int grid, size_t smem, cudaStream_t stream) {
  auto kern = gate_backward_ring_kernel<BF16, M1>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  kern<<<grid, ring_threads(a.d), smem, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gate_backward(const GateBwArgs& a, int grid, cudaStream_t stream) {
  if (a.R == 0) return cudaSuccess;
  const size_t rsm = gate_bw_ring_smem(a.M, a.d, a.bf16 ? 2 : 4);
  if (rsm <= 232448 && a.d % 8 == 0 && ring_threads(a.d) <= 1024)
    return a.bf16 ? (a.M == 1 ? launch_ring<true, true>(a, grid, rsm, stream)
                              : launch_ring<true, false>(a, grid, rsm, stream))
                  : (a.M == 1 ? launch_ring<false, true>(a, grid, rsm, stream)
                              : launch_ring<false, false>(a, grid, rsm, stream));
  const size_t smem = gate_bw_smem(a.M, a.d);
  if (smem > 232448) return cudaErrorInvalidValue;
  const int per = (a.d + kBwThreads - 1) / kBwThreads;
  if (per <= 1) return launch_gate_bw<1>(a, grid, smem, stream);
  if (per <= 2) return launch_gate_bw<2>(a, grid, smem, stream);
  if (per <= 4) return launch_gate_bw<4>(a, grid, smem, stream);
  if (per <= 8) return launch_gate_bw<8>(a, grid, smem, stream);
  if (per <= 12) return launch_gate_bw<12>(a, grid, smem, stream);
  if (per <= 16) return launch_gate_bw<16>(a, grid, smem, stream);
  return cudaErrorInvalidValue;
}

cudaError_t launch_dnorm_reduce(const float* partials, int nblocks, int64_t n, float* dnorm_q,
                                float* dnorm_k, cudaStream_t stream) {
  if (n == 0 || (!dnorm_q && !dnorm_k)) return cudaSuccess;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  int64_t blocks = (2 * n + 31) / 32;
  if (blocks > (int64_t)sms * 8) blocks = (int64_t)sms * 8;
  dnorm_reduce_kernel<<<(unsigned)blocks, 256, 0, stream>>>(partials, nblocks, n, dnorm_q, dnorm_k);
  return cudaGetLastError();
}

cudaError_t launch_table_grad(const TableGradArgs& a, cudaStream_t stream) {
  if (a.d_head % 4) return cudaErrorInvalidValue;
  const int64_t total = a.rows * a.S * (a.d_head / 4);
  if (total == 0) return cudaSuccess;
  table_grad_kernel<<<grid_cap(total, 256), 256, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace engram
