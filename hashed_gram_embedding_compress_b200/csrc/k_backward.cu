// Backward of the lookup-and-gate step (training).
//
// "Conditional Memory via Scalable Lookup", section 2.3 Eq. (3)-(4) and
// section 2.4 Eq. (6) give the forward; this file holds the hand-written
// kernels of its exact derivative (the dense contractions, k and v recomputed
// and the weight and memory-vector gradients, are library GEMMs issued by the
// ABI layer):
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
// gate_backward_kernel: a CTA per row at a time (grid-stride), 256 threads,
// each holding PER elements of the row (column tid + 256 j) in registers; the
// two row reductions per branch are block reductions.  dw_q and dw_k are
// summed per CTA in shared memory (each thread owns its columns) and reduced
// over the CTAs in a fixed order by dnorm_reduce_kernel (deterministic).
// table_grad_kernel adds the slices of de into fp32 table gradients.
#include "engram_internal.cuh"

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

// dnorm_q[i] += sum over CTAs b of partials[b][0][i], dnorm_k likewise, in
// order of b (one thread per column).
__global__ void dnorm_reduce_kernel(const float* partials, int nblocks, int64_t n, float* dnorm_q,
                                    float* dnorm_k) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < 2 * n;
       i += (int64_t)gridDim.x * blockDim.x) {
    float s = 0.f;
    for (int b = 0; b < nblocks; ++b) s += partials[(int64_t)b * 2 * n + i];
    if (i < n) {
      if (dnorm_q) dnorm_q[i] += s;
    } else if (dnorm_k) {
      dnorm_k[i - n] += s;
    }
  }
}

// dtab[s][idx[r][s]][c] += de[r][s d_h + c]: one thread per element of de.
__global__ void table_grad_kernel(TableGradArgs a) {
  const int64_t per_row = (int64_t)a.S * a.d_head;
  const int64_t total = a.rows * per_row;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = i / per_row;
    const int32_t rem = (int32_t)(i - r * per_row);
    const int32_t s = rem / a.d_head, c = rem - s * a.d_head;
    const int64_t z = a.idx[r * a.S + s];
    if (z < 0 || z >= a.primes[s]) {
      if (c == 0) atomicOr(a.err, kDevErrIndex);
      continue;
    }
    atomicAdd(a.dtables[s] + z * a.d_head + c, a.de[i]);
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
int gate_bw_grid(int M, int d, int64_t R) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
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

cudaError_t launch_gate_backward(const GateBwArgs& a, int grid, cudaStream_t stream) {
  if (a.R == 0) return cudaSuccess;
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
  dnorm_reduce_kernel<<<grid_cap(2 * n, 256), 256, 0, stream>>>(partials, nblocks, n, dnorm_q,
                                                                 dnorm_k);
  return cudaGetLastError();
}

cudaError_t launch_table_grad(const TableGradArgs& a, cudaStream_t stream) {
  const int64_t total = a.rows * a.S * a.d_head;
  if (total == 0) return cudaSuccess;
  table_grad_kernel<<<grid_cap(total, 256), 256, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace engram
