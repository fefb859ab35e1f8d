// fp32 dense contractions of the backward for fp32 handles (SIMT FFMA).
//
// The same three contractions as k_gemm_sm100.cu (k and v recomputed, the
// weight gradients, the memory-vector gradient), for the fp32 configuration:
// TF32 tensor cores round the operands to 10 mantissa bits, which the fp32
// tolerance does not allow.  A 64 x 64 tile per CTA of 256 threads, each
// thread 4 x 4 outputs; 16-deep K slices of A and B staged in shared memory.
// Operands are addressed through element strides, so any transposition is a
// choice of strides.
#include "engram_internal.cuh"

namespace engram {

namespace {

constexpr int kT = 64, kK = 16;

__global__ void __launch_bounds__(256) gemm_f32_kernel(GemmF32Args g) {
  __shared__ float As[kK][kT + 1];
  __shared__ float Bs[kK][kT + 1];
  const int m0 = blockIdx.y * kT, n0 = blockIdx.x * kT;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < g.K; k0 += kK) {
    for (int i = threadIdx.x; i < kK * kT; i += 256) {
      const int kk = i / kT, r = i - kk * kT;
      const int k = k0 + kk;
      const int m = m0 + r, n = n0 + r;
      As[kk][r] = (k < g.K && m < g.M) ? g.A[(int64_t)m * g.a_m + (int64_t)k * g.a_k] : 0.f;
      Bs[kk][r] = (k < g.K && n < g.N) ? g.B[(int64_t)n * g.b_n + (int64_t)k * g.b_k] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < kK; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        a[i] = As[kk][ty * 4 + i];
        b[i] = Bs[kk][tx * 4 + i];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int m = m0 + ty * 4 + i;
    if (m >= g.M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tx * 4 + j;
      if (n >= g.N) continue;
      float* p = g.D + (int64_t)m * g.ldd + n;
      *p = g.add ? *p + acc[i][j] : acc[i][j];
    }
  }
}

}  // namespace

cudaError_t launch_gemm_f32(const GemmF32Args& g, cudaStream_t stream) {
  if (g.M <= 0 || g.N <= 0) return cudaSuccess;
  if ((g.M + kT - 1) / kT > 65535) return cudaErrorInvalidValue;
  const dim3 grid((g.N + kT - 1) / kT, (g.M + kT - 1) / kT);
  gemm_f32_kernel<<<grid, 256, 0, stream>>>(g);
  return cudaGetLastError();
}

}  // namespace engram
