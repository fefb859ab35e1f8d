// fp32 projection + context-aware gate (SIMT FFMA).
//
// "Conditional Memory via Scalable Lookup", section 2.3 Eq. (3)-(4) and
// section 2.4 Eq. (6).  Used when tables, weights and hidden states are fp32:
// TF32 tensor cores round the operands to 10 mantissa bits, which cannot meet
// a 1e-5 absolute bound, so this path stays on the FFMA pipe.
//
// Two launches share the structure of the bf16 tensor-core path:
//   phase 0: key tiles   k = e W_K^T, reduced per row and tile to the partial
//            sums (sum k^2, sum h (w_q w_k) k, sum h^2) of the RMSNorm-ed dot;
//   phase 1: value tiles v = e W_V^T; the epilogue finishes alpha from the
//            partials of every key tile of the branch and writes
//            out = h + alpha v (plus alpha and alpha v when requested);
//   phase 3: value tiles for the short convolution (Eq. 5): alpha, v and the
//            per-row sum of v^2 of the tile; h is not read.
#include "engram_internal.cuh"

namespace engram {

namespace {

constexpr int BM = 64, BN = kF32Tile, BK = 16;

__device__ __forceinline__ float sigmoid_f(float s) { return 1.0f / (1.0f + expf(-s)); }

template <int PHASE>
__global__ void __launch_bounds__(256) proj_gate_f32_kernel(const float* __restrict__ e,
                                                            const float* __restrict__ w,
                                                            int n_total, GateArgs g) {
  __shared__ float As[BK][BM + 4];
  __shared__ float Bs[BK][BN + 4];
  const int tid = threadIdx.x, tx = tid % 16, ty = tid / 16;
  const int m0 = blockIdx.y * BM, n0 = blockIdx.x * BN;
  const int R = g.R, dm = g.d_mem, d = g.d, M = g.M;
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;

  const int lr = tid / 4, lk = (tid % 4) * 4;
  for (int k0 = 0; k0 < dm; k0 += BK) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int k = k0 + lk + q;
      As[lk + q][lr] = (m0 + lr < R && k < dm) ? e[(int64_t)(m0 + lr) * dm + k] : 0.f;
      Bs[lk + q][lr] = (n0 + lr < n_total && k < dm) ? w[(int64_t)(n0 + lr) * dm + k] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int k = 0; k < BK; ++k) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[k][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = Bs[k][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }

  const float* h = (const float*)g.h;
  if (PHASE == 0) {
    const int mb = n0 / d, j0 = n0 - mb * d + tx * 4;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int row = m0 + ty * 4 + i;
      float skk = 0.f, shk = 0.f, shh = 0.f;
      if (row < R) {
        const float* hr = h + ((int64_t)row * M + mb) * d + j0;
        const float* wr = g.w_qk + (int64_t)mb * d + j0;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float k = acc[i][j], hv = hr[j];
          skk = fmaf(k, k, skk);
          shh = fmaf(hv, hv, shh);
          shk = fmaf(hv * wr[j], k, shk);
        }
      }
#pragma unroll
      for (int off = 8; off > 0; off >>= 1) {
        skk += __shfl_xor_sync(0xffffffffu, skk, off);
        shk += __shfl_xor_sync(0xffffffffu, shk, off);
        shh += __shfl_xor_sync(0xffffffffu, shh, off);
      }
      if (tx == 0 && row < R)
        g.partials[(int64_t)blockIdx.x * R + row] = make_float4(skk, shk, shh, 0.f);
    }
  } else if (PHASE == 3) {
    const int tiles_per_branch = d / g.key_tile;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int row = m0 + ty * 4 + i;
      float svv = 0.f;
      if (row < R) {
#pragma unroll
        for (int j = 0; j < 4; ++j) svv = fmaf(acc[i][j], acc[i][j], svv);
        *reinterpret_cast<float4*>(g.vals + (int64_t)row * d + n0 + tx * 4) =
            make_float4(acc[i][0], acc[i][1], acc[i][2], acc[i][3]);
        if (blockIdx.x == 0 && tx == 0)
          for (int mb = 0; mb < M; ++mb) {
            float skk = 0.f, shk = 0.f, shh = 0.f;
            for (int tb = mb * tiles_per_branch; tb < (mb + 1) * tiles_per_branch; ++tb) {
              const float4 p = g.partials[(int64_t)tb * R + row];
              skk += p.x;
              shk += p.y;
              shh += p.z;
            }
            const float rh = 1.0f / sqrtf(shh / (float)d + g.eps);
            const float rk = 1.0f / sqrtf(skk / (float)d + g.eps);
            g.alpha[(int64_t)row * M + mb] = sigmoid_f(shk * rh * rk * g.inv_sqrt_d);
          }
      }
#pragma unroll
      for (int off = 8; off > 0; off >>= 1) svv += __shfl_xor_sync(0xffffffffu, svv, off);
      if (tx == 0 && row < R) g.vv[(int64_t)blockIdx.x * R + row] = svv;
    }
  } else {
    const int tiles_per_branch = d / g.key_tile;
    float* out = (float*)g.out;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int row = m0 + ty * 4 + i;
      if (row >= R) continue;
      for (int mb = 0; mb < M; ++mb) {
        float skk = 0.f, shk = 0.f, shh = 0.f;
        for (int tb = mb * tiles_per_branch; tb < (mb + 1) * tiles_per_branch; ++tb) {
          const float4 p = g.partials[(int64_t)tb * R + row];
          skk += p.x;
          shk += p.y;
          shh += p.z;
        }
        const float rh = 1.0f / sqrtf(shh / (float)d + g.eps);
        const float rk = 1.0f / sqrtf(skk / (float)d + g.eps);
        const float al = sigmoid_f(shk * rh * rk * g.inv_sqrt_d);
        const int64_t base = ((int64_t)row * M + mb) * d + n0 + tx * 4;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float dl = al * acc[i][j];
          out[base + j] = h[base + j] + dl;
          if (g.delta) g.delta[base + j] = dl;
        }
        if (g.alpha && blockIdx.x == 0 && tx == 0) g.alpha[(int64_t)row * M + mb] = al;
      }
    }
  }
}

}  // namespace

cudaError_t launch_proj_gate_f32(int phase, const float* e, const float* w, const GateArgs& g,
                                 cudaStream_t stream) {
  if (g.R == 0) return cudaSuccess;
  const int n_total = phase == 0 ? g.M * g.d : g.d;
  dim3 grid(n_total / BN, (g.R + BM - 1) / BM);
  if (phase == 0)
    proj_gate_f32_kernel<0><<<grid, 256, 0, stream>>>(e, w, n_total, g);
  else if (phase == 3)
    proj_gate_f32_kernel<3><<<grid, 256, 0, stream>>>(e, w, n_total, g);
  else
    proj_gate_f32_kernel<1><<<grid, 256, 0, stream>>>(e, w, n_total, g);
  return cudaGetLastError();
}

}  // namespace engram
