// Short depthwise causal convolution on the gated values, and the residual
// update: "Conditional Memory via Scalable Lookup", section 2.3, Eq. (5).
//
//   V~_t^(m) = alpha_t^(m) v_t
//   Y_t^(m)[c] = SiLU( sum_i cw[c][i] RMSNorm(V~^(m))_{t - i dil}[c] ) + V~_t^(m)[c]
//   out = h + Y
//
// RMSNorm(V~_t^(m)) = v_t * s_t^(m) * norm_w with s = alpha / sqrt(alpha^2
// mean(v_t^2) + eps), so the value-phase epilogue leaves v (fp32, shared by
// the M branches) and the per-row sums of v^2 per value tile; a small kernel
// turns those into s per (position, branch), and the conv kernel needs one
// pass.  Positions before the start of a sequence contribute zero; there is
// no bias.  Kernel sizes 1-4 run as four taps with the unused ones zero.
//
// The conv kernel is persistent and works on tiles of 16 positions of one
// sequence x 128 channels: cp.async copies stage the tile's rows of v (with
// the 3 dil rows of halo before it), h, the scales and alpha in shared
// memory, two tiles deep, so the next tile's copies stream in while this one
// computes; the stages are small enough for several blocks per SM.  A thread
// takes 4 channels of 4 positions, reads the taps
// premultiplied by the norm weight from a tap-major copy (one coalesced float4
// per tap) and sums them in packed fp32 pairs; out = h + Y is stored
// straight to global memory (coalesced), Y too when asked.
#include "sm100_ptx.cuh"

#include <cuda_bf16.h>


namespace engram {

namespace {

using sm100::bf16x2_to_f2;
using sm100::f2_fma;
using sm100::f2_mul;
using sm100::f2_pack;
using sm100::f2_unpack;

constexpr int kTaps = 4;

// x sigmoid(x) = x / (1 + e^-x) with the fast exponential and the fast
// division (a few ulp of fp32, far inside the 1e-5 bound of the fp32 path; a
// denominator beyond 2^126, x below about -87, gives 0 where the true value
// is below 1e-36)
__device__ __forceinline__ float silu_f(float x) { return __fdividef(x, 1.0f + __expf(-x)); }

__device__ __forceinline__ unsigned long long f2_add(unsigned long long a, unsigned long long b) {
  unsigned long long d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

// s[row][m] = alpha / sqrt(alpha^2 mean(v_row^2) + eps)
__global__ void __launch_bounds__(256) conv_scale_kernel(ConvArgs a, float* __restrict__ s) {
  const int64_t R = (int64_t)a.B * a.T;
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= R * a.M) return;
  const int64_t row = i / a.M;
  float ss = 0.f;
  for (int k = 0; k < a.n_vtiles; ++k) ss += __ldg(a.vv + (int64_t)k * R + row);
  const float al = __ldg(a.alpha + i);
  s[i] = al * rsqrtf(al * al * (ss / (float)a.d) + a.eps);
}

// Async copies global -> shared (the LDGSTS path: no registers held while
// in flight).  With src_bytes = 0 nothing is read and the destination is
// zero-filled (rows outside the sequence).
__device__ __forceinline__ void cp_async16(void* dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(
                   (uint32_t)__cvta_generic_to_shared(dst)),
               "l"(src), "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async4(void* dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(
                   (uint32_t)__cvta_generic_to_shared(dst)),
               "l"(src), "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

constexpr int kCh = 128;                  // channels per tile
constexpr int kQuads = kCh / 4;           // threads per position (4 channels each)
constexpr int kConvBlock = 128;           // threads: 4 position groups x 32
constexpr int kGroups = kConvBlock / kQuads;

// Positions per tile: 16, fewer with several fp32 branches, so that two
// stages stay small and several blocks share an SM.
template <bool BF16, int M>
struct ConvTile {
  static constexpr int ELT = BF16 ? 2 : 4;
  static constexpr int PT = M * ELT <= 8 ? 16 : 8;
};

template <int DIL, bool BF16, int M>
struct ConvSmem {
  static constexpr int PT = ConvTile<BF16, M>::PT;
  static constexpr int H = (kTaps - 1) * DIL;
  static constexpr int NR = PT + H;                       // rows of v per tile
  static constexpr int ELT = BF16 ? 2 : 4;
  static constexpr size_t V = (size_t)NR * kCh * 4;       // v rows
  static constexpr size_t HB = (size_t)PT * M * kCh * ELT;  // h rows
  static constexpr size_t F = (size_t)M * NR * 4;         // scales
  static constexpr size_t AL = (size_t)M * PT * 4;        // alpha
  static constexpr size_t STAGE = (V + HB + F + AL + 15) / 16 * 16;
  static constexpr size_t BYTES = 2 * STAGE;
  static_assert(BYTES <= 232448, "two stages fit in shared memory");
};

// Persistent: a block takes tiles (sequence, 16 positions, 128 channels) in
// a grid stride; tile i + 1's copies are in flight while tile i computes.
template <int DIL, bool BF16, int M>
__global__ void __launch_bounds__(kConvBlock) short_conv_kernel(ConvArgs a,
                                                               const float* __restrict__ s) {
  using L = ConvSmem<DIL, BF16, M>;
  constexpr int PT = L::PT, H = L::H, NR = L::NR, ELT = L::ELT;
  extern __shared__ __align__(16) unsigned char smem[];
  const int d = a.d;
  const int T = a.T;
  const int tiles_t = (T + PT - 1) / PT;
  const int tiles_c = (d + kCh - 1) / kCh;
  const int64_t R = (int64_t)a.B * T;
  const int num_tiles = a.B * tiles_t * tiles_c;
  const int tid = threadIdx.x;

  auto stage_ptr = [&](int st) { return smem + (size_t)st * L::STAGE; };
  // issue the copies of tile `tile` into stage `st`
  auto load_tile = [&](int tile, int st) {
    unsigned char* base = stage_ptr(st);
    float4* sv = reinterpret_cast<float4*>(base);
    unsigned char* sh = base + L::V;
    float* sf = reinterpret_cast<float*>(base + L::V + L::HB);
    float* sal = reinterpret_cast<float*>(base + L::V + L::HB + L::F);
    const int tc = tile % tiles_c;
    const int rest = tile / tiles_c;
    const int tt = rest % tiles_t, b = rest / tiles_t;
    const int c0 = tc * kCh, t0 = tt * PT;
    const int64_t row_base = (int64_t)b * T;
    // v: NR rows x kQuads chunks of 16 bytes
    for (int i = tid; i < NR * kQuads; i += kConvBlock) {
      const int r = i / kQuads, q = i % kQuads;
      const int t = t0 - H + r, c = c0 + 4 * q;
      const bool in = t >= 0 && t < T && c < d;
      const float* src = in ? a.vals + (row_base + t) * d + c : a.vals;
      cp_async16(sv + i, src, in ? 16u : 0u);
    }
    // h: PT rows x M branches x (kCh * ELT / 16) chunks
    constexpr int HC = kCh * ELT / 16;
    for (int i = tid; i < PT * M * HC; i += kConvBlock) {
      const int q = i % HC, pm = i / HC;
      const int m = pm % M, p = pm / M;
      const int t = t0 + p, c = c0 + q * (16 / ELT);
      const bool in = t < T && c < d;
      const unsigned char* src =
          in ? static_cast<const unsigned char*>(a.h) + (((row_base + t) * M + m) * d + c) * ELT
             : static_cast<const unsigned char*>(a.h);
      cp_async16(sh + (size_t)i * 16, src, in ? 16u : 0u);
    }
    // scales of the NR rows and alpha of the PT outputs, per branch
    for (int i = tid; i < M * NR; i += kConvBlock) {
      const int m = i / NR, r = i % NR;
      const int t = t0 - H + r;
      const bool in = t >= 0 && t < T;
      cp_async4(sf + i, in ? s + (row_base + t) * M + m : s, in ? 4u : 0u);
    }
    for (int i = tid; i < M * PT; i += kConvBlock) {
      const int m = i / PT, p = i % PT;
      const int t = t0 + p;
      const bool in = t < T;
      cp_async4(sal + i, in ? a.alpha + (row_base + t) * M + m : a.alpha, in ? 4u : 0u);
    }
  };

  const int grp = tid / kQuads, cq = tid % kQuads;  // positions group, channel quad
  int tile = blockIdx.x, st = 0;
  if (tile < num_tiles) load_tile(tile, 0);
  cp_async_commit();
  if (tile + (int)gridDim.x < num_tiles) load_tile(tile + gridDim.x, 1);
  cp_async_commit();
  for (; tile < num_tiles; tile += gridDim.x, st ^= 1) {
    cp_async_wait<1>();  // this tile's group has landed (the next may still fly)
    __syncthreads();
    const unsigned char* base = stage_ptr(st);
    const float4* sv = reinterpret_cast<const float4*>(base);
    const unsigned char* sh = base + L::V;
    const float* sf = reinterpret_cast<const float*>(base + L::V + L::HB);
    const float* sal = reinterpret_cast<const float*>(base + L::V + L::HB + L::F);
    const int tc = tile % tiles_c;
    const int rest = tile / tiles_c;
    const int tt = rest % tiles_t, b = rest / tiles_t;
    const int c = tc * kCh + 4 * cq, t0 = tt * PT;
    const int64_t row_base = (int64_t)b * T;
    if (c < d) {
      // taps of the 4 channels times their RMSNorm weights, as packed pairs
      unsigned long long cw01[kTaps], cw23[kTaps];
#pragma unroll
      for (int k = 0; k < kTaps; ++k) {
        const float4 w = __ldg(reinterpret_cast<const float4*>(a.taps + (int64_t)k * d + c));
        cw01[k] = f2_pack(__float_as_uint(w.x), __float_as_uint(w.y));
        cw23[k] = f2_pack(__float_as_uint(w.z), __float_as_uint(w.w));
      }
#pragma unroll 2
      for (int pp = 0; pp < PT / kGroups; ++pp) {
        const int p = grp * (PT / kGroups) + pp;
        if (t0 + p >= T) break;
        const int64_t row = row_base + t0 + p;
        const float4 xt = sv[(p + H) * kQuads + cq];
#pragma unroll
        for (int m = 0; m < M; ++m) {
          unsigned long long a01 = 0ull, a23 = 0ull;
#pragma unroll
          for (int k = 0; k < kTaps; ++k) {
            const int r = p + H - k * DIL;
            const float4 xk = sv[r * kQuads + cq];
            const float fk = sf[m * NR + r];  // zero outside the sequence
            const unsigned long long f2 = f2_pack(__float_as_uint(fk), __float_as_uint(fk));
            a01 = f2_fma(cw01[k], f2_mul(f2_pack(__float_as_uint(xk.x), __float_as_uint(xk.y)), f2), a01);
            a23 = f2_fma(cw23[k], f2_mul(f2_pack(__float_as_uint(xk.z), __float_as_uint(xk.w)), f2), a23);
          }
          const float2 s01 = f2_unpack(a01), s23 = f2_unpack(a23);
          const float al = sal[m * PT + p];
          const unsigned long long al2 = f2_pack(__float_as_uint(al), __float_as_uint(al));
          const int64_t o = (row * M + m) * d + c;
          const unsigned char* hp = sh + ((size_t)(p * M + m) * kCh + 4 * cq) * ELT;
          unsigned long long y01, y23;  // Y = SiLU(conv) + alpha v, packed pairs
          if (BF16) {
            y01 = f2_fma(al2, f2_pack(__float_as_uint(xt.x), __float_as_uint(xt.y)),
                         f2_pack(__float_as_uint(silu_f(s01.x)), __float_as_uint(silu_f(s01.y))));
            y23 = f2_fma(al2, f2_pack(__float_as_uint(xt.z), __float_as_uint(xt.w)),
                         f2_pack(__float_as_uint(silu_f(s23.x)), __float_as_uint(silu_f(s23.y))));
            const uint2 hb = *reinterpret_cast<const uint2*>(hp);
            const float2 o01 = f2_unpack(f2_add(bf16x2_to_f2(hb.x), y01));
            const float2 o23 = f2_unpack(f2_add(bf16x2_to_f2(hb.y), y23));
            const __nv_bfloat162 b01 = __floats2bfloat162_rn(o01.x, o01.y);
            const __nv_bfloat162 b23 = __floats2bfloat162_rn(o23.x, o23.y);
            uint2 ob;
            ob.x = *reinterpret_cast<const uint32_t*>(&b01);
            ob.y = *reinterpret_cast<const uint32_t*>(&b23);
            *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(a.out) + o) = ob;
          } else {
            y01 = f2_fma(al2, f2_pack(__float_as_uint(xt.x), __float_as_uint(xt.y)),
                         f2_pack(__float_as_uint(silu_f(s01.x)), __float_as_uint(silu_f(s01.y))));
            y23 = f2_fma(al2, f2_pack(__float_as_uint(xt.z), __float_as_uint(xt.w)),
                         f2_pack(__float_as_uint(silu_f(s23.x)), __float_as_uint(silu_f(s23.y))));
            const float4 h4 = *reinterpret_cast<const float4*>(hp);
            const float2 o01 = f2_unpack(f2_add(f2_pack(__float_as_uint(h4.x), __float_as_uint(h4.y)), y01));
            const float2 o23 = f2_unpack(f2_add(f2_pack(__float_as_uint(h4.z), __float_as_uint(h4.w)), y23));
            *reinterpret_cast<float4*>(static_cast<float*>(a.out) + o) =
                make_float4(o01.x, o01.y, o23.x, o23.y);
          }
          if (a.delta) {
            const float2 y0 = f2_unpack(y01), y1 = f2_unpack(y23);
            *reinterpret_cast<float4*>(a.delta + o) = make_float4(y0.x, y0.y, y1.x, y1.y);
          }
        }
      }
    }
    __syncthreads();  // every thread is done with this stage
    const int next = tile + 2 * (int)gridDim.x;
    if (next < num_tiles) load_tile(next, st);
    cp_async_commit();
  }
  cp_async_wait<0>();
  (void)R;
  (void)ELT;
}

__global__ void conv_taps_kernel(const float* __restrict__ conv_w, const float* __restrict__ norm_w,
                                 int d, float* __restrict__ taps) {
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  if (c >= d) return;
#pragma unroll
  for (int k = 0; k < kTaps; ++k) taps[(int64_t)k * d + c] = conv_w[(int64_t)c * kTaps + k] * norm_w[c];
}

template <int DIL, bool BF16, int M>
cudaError_t launch_one(const ConvArgs& a, const float* s, cudaStream_t stream) {
  using L = ConvSmem<DIL, BF16, M>;
  auto kern = short_conv_kernel<DIL, BF16, M>;
  cudaError_t e =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L::BYTES);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148, per_sm = 1;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kConvBlock, L::BYTES);
  if (per_sm < 1) per_sm = 1;
  const int64_t tiles = (int64_t)a.B * ((a.T + L::PT - 1) / L::PT) * ((a.d + kCh - 1) / kCh);
  const int64_t grid = tiles < (int64_t)sms * per_sm ? tiles : (int64_t)sms * per_sm;
  kern<<<(unsigned)grid, kConvBlock, L::BYTES, stream>>>(a, s);
  return cudaGetLastError();
}

template <int DIL, bool BF16>
cudaError_t launch_typed(const ConvArgs& a, const float* s, cudaStream_t stream) {
  switch (a.M) {
    case 1: return launch_one<DIL, BF16, 1>(a, s, stream);
    case 2: return launch_one<DIL, BF16, 2>(a, s, stream);
    case 3: return launch_one<DIL, BF16, 3>(a, s, stream);
    case 4: return launch_one<DIL, BF16, 4>(a, s, stream);
    default: return cudaErrorInvalidValue;
  }
}

template <int DIL>
cudaError_t launch_dil(const ConvArgs& a, const float* s, cudaStream_t stream) {
  return a.bf16 ? launch_typed<DIL, true>(a, s, stream) : launch_typed<DIL, false>(a, s, stream);
}

}  // namespace

cudaError_t launch_conv_taps(const float* conv_w, const float* norm_w, int d, float* taps,
                             cudaStream_t stream) {
  conv_taps_kernel<<<(d + 255) / 256, 256, 0, stream>>>(conv_w, norm_w, d, taps);
  return cudaGetLastError();
}

cudaError_t launch_short_conv(const ConvArgs& a, int dilation, float* scale, cudaStream_t stream) {
  const int64_t R = (int64_t)a.B * a.T;
  if (R == 0) return cudaSuccess;
  if (a.d % 4 != 0 || a.M < 1 || a.M > kMaxBranches || a.n_vtiles < 1)
    return cudaErrorInvalidValue;
  // tile indices stay below 2^31
  if ((R / 8 + a.B) * ((a.d + kCh - 1) / kCh) >= ((int64_t)1 << 31)) return cudaErrorInvalidValue;
  conv_scale_kernel<<<(unsigned)((R * a.M + 255) / 256), 256, 0, stream>>>(a, scale);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  switch (dilation) {
    case 1: return launch_dil<1>(a, scale, stream);
    case 2: return launch_dil<2>(a, scale, stream);
    case 3: return launch_dil<3>(a, scale, stream);
    case 4: return launch_dil<4>(a, scale, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace engram
