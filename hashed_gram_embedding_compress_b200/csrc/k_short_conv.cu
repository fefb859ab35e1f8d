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
// The conv kernel gives each thread P consecutive positions of one sequence
// and 4 channels.  It issues all its loads first (the P + 3 dil rows of v the
// taps reach, their scales, alpha and h), so each thread keeps tens of
// requests in flight, and the P outputs share the tap weights and the
// overlapping rows of v.  Consecutive threads walk the channels, consecutive
// blocks the positions, so rows of v read again by the next chunk's halo are
// found in L2: HBM sees v, h and out about once each.
#include "sm100_ptx.cuh"

#include <cuda_bf16.h>

#include <type_traits>

namespace engram {

namespace {

using sm100::f2_fma;
using sm100::f2_mul;
using sm100::f2_pack;
using sm100::f2_unpack;

constexpr int kTaps = 4;
constexpr int kConvThreads = 128;

// x sigmoid(x) with the fast exponential and reciprocal (relative error a few
// ulp of fp32, far inside the 1e-5 bound of the fp32 path)
__device__ __forceinline__ float silu_f(float x) { return x * __frcp_rn(1.0f + __expf(-x)); }

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

// Positions per thread: the P outputs share their tap loads and the
// overlapping rows of v (P + 3 dil rows for P outputs), keeping the L1
// traffic per output low; fewer for several branches to bound registers.
template <int M>
struct ConvPos {
  static constexpr int P = M == 1 ? 4 : 2;
};

template <int DIL, bool BF16, int M>
__global__ void __launch_bounds__(kConvThreads) short_conv_kernel(ConvArgs a,
                                                                  const float* __restrict__ s) {
  constexpr int P = ConvPos<M>::P;
  constexpr int H = (kTaps - 1) * DIL;
  constexpr int NX = P + H;  // rows of v one thread reads
  using HVec = typename std::conditional<BF16, uint2, float4>::type;
  const int d = a.d;
  const uint32_t groups = (uint32_t)d / 4;  // channel groups of 4 per position
  const uint32_t chunks = ((uint32_t)a.T + P - 1) / P;  // position chunks per sequence
  // 32-bit index arithmetic: the launcher keeps B * chunks * d / 4 < 2^31
  const uint32_t i = blockIdx.x * kConvThreads + threadIdx.x;
  if (i >= (uint32_t)a.B * chunks * groups) return;
  const uint32_t q = i / groups;  // (sequence, chunk)
  const int c = (int)(i - q * groups) * 4;
  const uint32_t b = q / chunks;
  const int t0 = (int)(q - b * chunks) * P;  // first output position
  const int64_t row_base = (int64_t)b * a.T;

  // every load first: v rows t0 - H .. t0 + P - 1, their scales, alpha and h
  float4 x[NX];
  float f[NX][M];
#pragma unroll
  for (int j = 0; j < NX; ++j) {
    const int t = t0 - H + j;
    const bool in = t >= 0 && t < a.T;  // positions of this sequence only
    const int64_t r = row_base + t;
    x[j] = in ? __ldg(reinterpret_cast<const float4*>(a.vals + r * d + c))
              : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int m = 0; m < M; ++m) f[j][m] = in ? __ldg(s + r * M + m) : 0.f;
  }
  HVec hv[P][M];
  float al[P][M];
#pragma unroll
  for (int p = 0; p < P; ++p) {
    const bool in = t0 + p < a.T;
    const int64_t r = row_base + t0 + p;
#pragma unroll
    for (int m = 0; m < M; ++m) {
      const int64_t o = (r * M + m) * d + c;
      if (in) {
        hv[p][m] = BF16 ? *reinterpret_cast<const HVec*>(static_cast<const __nv_bfloat16*>(a.h) + o)
                        : *reinterpret_cast<const HVec*>(static_cast<const float*>(a.h) + o);
        al[p][m] = __ldg(a.alpha + r * M + m);
      } else {
        al[p][m] = 0.f;
      }
    }
  }
  // taps of the 4 channels times their RMSNorm weights: one coalesced float4
  // per tap, kept as packed fp32 pairs (channels c, c+1 and c+2, c+3)
  unsigned long long cw01[kTaps], cw23[kTaps];
#pragma unroll
  for (int k = 0; k < kTaps; ++k) {
    const float4 w = __ldg(reinterpret_cast<const float4*>(a.taps + (int64_t)k * d + c));
    cw01[k] = f2_pack(__float_as_uint(w.x), __float_as_uint(w.y));
    cw23[k] = f2_pack(__float_as_uint(w.z), __float_as_uint(w.w));
  }

#pragma unroll
  for (int p = 0; p < P; ++p) {
    if (t0 + p >= a.T) break;
    const int64_t r = row_base + t0 + p;
    const float4 xt = x[p + H];  // v at the output position
#pragma unroll
    for (int m = 0; m < M; ++m) {
      unsigned long long a01 = 0ull, a23 = 0ull;
#pragma unroll
      for (int k = 0; k < kTaps; ++k) {
        const float4 xk = x[p + H - k * DIL];
        const float fk = f[p + H - k * DIL][m];
        const unsigned long long f2 = f2_pack(__float_as_uint(fk), __float_as_uint(fk));
        a01 = f2_fma(cw01[k], f2_mul(f2_pack(__float_as_uint(xk.x), __float_as_uint(xk.y)), f2), a01);
        a23 = f2_fma(cw23[k], f2_mul(f2_pack(__float_as_uint(xk.z), __float_as_uint(xk.w)), f2), a23);
      }
      const float2 s01 = f2_unpack(a01), s23 = f2_unpack(a23);
      const float acc[4] = {s01.x, s01.y, s23.x, s23.y};
      const float a_ = al[p][m];
      const float y[4] = {silu_f(acc[0]) + a_ * xt.x, silu_f(acc[1]) + a_ * xt.y,
                          silu_f(acc[2]) + a_ * xt.z, silu_f(acc[3]) + a_ * xt.w};
      const int64_t o = (r * M + m) * d + c;
      if (BF16) {
        const uint2 hb = *reinterpret_cast<const uint2*>(&hv[p][m]);
        const float2 h01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&hb.x));
        const float2 h23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&hb.y));
        const __nv_bfloat162 o01 = __floats2bfloat162_rn(h01.x + y[0], h01.y + y[1]);
        const __nv_bfloat162 o23 = __floats2bfloat162_rn(h23.x + y[2], h23.y + y[3]);
        uint2 ob;
        ob.x = *reinterpret_cast<const uint32_t*>(&o01);
        ob.y = *reinterpret_cast<const uint32_t*>(&o23);
        *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(a.out) + o) = ob;
      } else {
        const float4 h4 = *reinterpret_cast<const float4*>(&hv[p][m]);
        *reinterpret_cast<float4*>(static_cast<float*>(a.out) + o) =
            make_float4(h4.x + y[0], h4.y + y[1], h4.z + y[2], h4.w + y[3]);
      }
      if (a.delta) *reinterpret_cast<float4*>(a.delta + o) = make_float4(y[0], y[1], y[2], y[3]);
    }
  }
}

__global__ void conv_taps_kernel(const float* __restrict__ conv_w, const float* __restrict__ norm_w,
                                 int d, float* __restrict__ taps) {
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  if (c >= d) return;
#pragma unroll
  for (int k = 0; k < kTaps; ++k) taps[(int64_t)k * d + c] = conv_w[(int64_t)c * kTaps + k] * norm_w[c];
}

template <int M>
int64_t conv_blocks(const ConvArgs& a) {
  constexpr int P = ConvPos<M>::P;
  return ((int64_t)a.B * ((a.T + P - 1) / P) * (a.d / 4) + kConvThreads - 1) / kConvThreads;
}

template <int DIL, bool BF16>
cudaError_t launch_typed(const ConvArgs& a, const float* s, cudaStream_t stream) {
  switch (a.M) {
    case 1: short_conv_kernel<DIL, BF16, 1><<<(unsigned)conv_blocks<1>(a), kConvThreads, 0, stream>>>(a, s); break;
    case 2: short_conv_kernel<DIL, BF16, 2><<<(unsigned)conv_blocks<2>(a), kConvThreads, 0, stream>>>(a, s); break;
    case 3: short_conv_kernel<DIL, BF16, 3><<<(unsigned)conv_blocks<3>(a), kConvThreads, 0, stream>>>(a, s); break;
    case 4: short_conv_kernel<DIL, BF16, 4><<<(unsigned)conv_blocks<4>(a), kConvThreads, 0, stream>>>(a, s); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
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
  // thread indices stay below 2^31 (at most one position per thread)
  if ((R + (int64_t)a.B * 8) * (a.d / 4) >= ((int64_t)1 << 31)) return cudaErrorInvalidValue;
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
