// Short depthwise causal convolution on the gated values, and the residual
// update: "Conditional Memory via Scalable Lookup", section 2.3, Eq. (5).
//
//   V~_t^(m) = alpha_t^(m) v_t
//   Y_t^(m)[c] = SiLU( sum_i cw[c][i] RMSNorm(V~^(m))_{t - i dil}[c] ) + V~_t^(m)[c]
//   out = h + Y
//
// RMSNorm(V~_t^(m)) = v_t * alpha / sqrt(alpha^2 mean(v_t^2) + eps) * norm_w,
// so the value-phase epilogue leaves v (fp32, shared by the M branches) and
// the per-row sums of v^2 per value tile, and this kernel needs one pass over
// v.  Positions before the start of a sequence contribute zero; there is no
// bias.  Kernel sizes 1-4 run as four taps with the unused ones zero.
//
// One block covers kTT consecutive positions of one sequence and 4 channels
// per thread.  A thread slides along t keeping the last 3 dil + 1 positions of
// v for its channels in registers, so each position of v is loaded once (and
// the 3 dil positions of halo before the block's first position once more).
// Per element and branch the kernel reads h and writes out once: it is bound
// by HBM bandwidth.
#include "engram_internal.cuh"

#include <cuda_bf16.h>

namespace engram {

namespace {

constexpr int kTT = 64;         // positions per block
constexpr int kConvThreads = 128;
constexpr int kTaps = 4;

__device__ __forceinline__ float silu_f(float x) { return x / (1.0f + expf(-x)); }

template <int DIL, bool BF16>
__global__ void __launch_bounds__(kConvThreads) short_conv_kernel(ConvArgs a) {
  constexpr int H = (kTaps - 1) * DIL;  // halo positions before the block's first
  constexpr int WIN = H + 1;
  constexpr int NP = kTT + H;
  __shared__ float s_al[kMaxBranches][NP];  // alpha
  __shared__ float s_sc[kMaxBranches][NP];  // alpha / sqrt(alpha^2 mean(v^2) + eps)
  const int M = a.M, d = a.d;
  const int tiles_per_seq = (a.T + kTT - 1) / kTT;
  const int b = (int)(blockIdx.x / (unsigned)tiles_per_seq);
  const int t0 = ((int)blockIdx.x - b * tiles_per_seq) * kTT;
  const int64_t row_base = (int64_t)b * a.T;
  const int64_t R = (int64_t)a.B * a.T;

  for (int i = threadIdx.x; i < NP * M; i += blockDim.x) {
    const int m = i / NP, j = i - m * NP;
    const int t = t0 - H + j;
    float al = 0.f, sc = 0.f;
    if (t >= 0 && t < a.T) {
      const int64_t row = row_base + t;
      float ss = 0.f;
      for (int k = 0; k < a.n_vtiles; ++k) ss += a.vv[(int64_t)k * R + row];
      al = a.alpha[row * M + m];
      sc = al * rsqrtf(al * al * (ss / (float)d) + a.eps);
    }
    s_al[m][j] = al;
    s_sc[m][j] = sc;
  }
  __syncthreads();

  const int c = ((int)blockIdx.y * kConvThreads + (int)threadIdx.x) * 4;
  if (c >= d) return;
  // cwn[i][k]: tap i of channel c + k times the RMSNorm weight of the channel
  float cwn[kTaps][4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const float4 w = *reinterpret_cast<const float4*>(a.conv_w + (int64_t)(c + k) * kTaps);
    const float nw = a.norm_w[c + k];
    cwn[0][k] = w.x * nw;
    cwn[1][k] = w.y * nw;
    cwn[2][k] = w.z * nw;
    cwn[3][k] = w.w * nw;
  }
  float4 win[WIN];  // win[j]: v at (current position - j) for channels c..c+3
#pragma unroll
  for (int q = 0; q < WIN; ++q) win[q] = make_float4(0.f, 0.f, 0.f, 0.f);

  for (int j = 0; j < NP; ++j) {
    const int t = t0 - H + j;
    if (t >= a.T) break;
#pragma unroll
    for (int q = WIN - 1; q > 0; --q) win[q] = win[q - 1];
    win[0] = t >= 0 ? __ldg(reinterpret_cast<const float4*>(a.vals + (row_base + t) * d + c))
                    : make_float4(0.f, 0.f, 0.f, 0.f);
    if (j < H) continue;  // halo position: no output
    const int64_t row = row_base + t;
#pragma unroll 1
    for (int m = 0; m < M; ++m) {
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int i = 0; i < kTaps; ++i) {
        const float f = s_sc[m][j - i * DIL];  // zero before the sequence start
        const float4 x = win[i * DIL];
        acc[0] = fmaf(cwn[i][0], x.x * f, acc[0]);
        acc[1] = fmaf(cwn[i][1], x.y * f, acc[1]);
        acc[2] = fmaf(cwn[i][2], x.z * f, acc[2]);
        acc[3] = fmaf(cwn[i][3], x.w * f, acc[3]);
      }
      const float al = s_al[m][j];
      const float y[4] = {silu_f(acc[0]) + al * win[0].x, silu_f(acc[1]) + al * win[0].y,
                          silu_f(acc[2]) + al * win[0].z, silu_f(acc[3]) + al * win[0].w};
      const int64_t o = (row * M + m) * d + c;
      if (BF16) {
        const uint2 hb = *reinterpret_cast<const uint2*>(static_cast<const __nv_bfloat16*>(a.h) + o);
        const float2 h01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&hb.x));
        const float2 h23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&hb.y));
        const __nv_bfloat162 o01 = __floats2bfloat162_rn(h01.x + y[0], h01.y + y[1]);
        const __nv_bfloat162 o23 = __floats2bfloat162_rn(h23.x + y[2], h23.y + y[3]);
        uint2 ob;
        ob.x = *reinterpret_cast<const uint32_t*>(&o01);
        ob.y = *reinterpret_cast<const uint32_t*>(&o23);
        *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(a.out) + o) = ob;
      } else {
        const float4 hv = *reinterpret_cast<const float4*>(static_cast<const float*>(a.h) + o);
        *reinterpret_cast<float4*>(static_cast<float*>(a.out) + o) =
            make_float4(hv.x + y[0], hv.y + y[1], hv.z + y[2], hv.w + y[3]);
      }
      if (a.delta)
        *reinterpret_cast<float4*>(a.delta + o) = make_float4(y[0], y[1], y[2], y[3]);
    }
  }
}

template <int DIL>
cudaError_t launch_dil(const ConvArgs& a, cudaStream_t stream) {
  const int tiles_per_seq = (a.T + kTT - 1) / kTT;
  dim3 grid((unsigned)(a.B * tiles_per_seq), (a.d / 4 + kConvThreads - 1) / kConvThreads);
  if (a.bf16)
    short_conv_kernel<DIL, true><<<grid, kConvThreads, 0, stream>>>(a);
  else
    short_conv_kernel<DIL, false><<<grid, kConvThreads, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_short_conv(const ConvArgs& a, int dilation, cudaStream_t stream) {
  if ((int64_t)a.B * a.T == 0) return cudaSuccess;
  if (a.d % 4 != 0 || a.M < 1 || a.M > kMaxBranches) return cudaErrorInvalidValue;
  if ((int64_t)a.B * ((a.T + kTT - 1) / kTT) > 2147483647) return cudaErrorInvalidValue;
  switch (dilation) {
    case 1: return launch_dil<1>(a, stream);
    case 2: return launch_dil<2>(a, stream);
    case 3: return launch_dil<3>(a, stream);
    case 4: return launch_dil<4>(a, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace engram
