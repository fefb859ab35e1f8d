// Compress + suffix n-gram + multi-head hash, and the row gather.
//
// "Conditional Memory via Scalable Lookup", section 2.2: x'_t = P(x_t);
// g_{t,n} = (x'_{t-n+1}, ..., x'_t); z_{t,n,k} = phi_{n,k}(g_{t,n}) (Eq. 1);
// e_t = concatenation of E_{n,k}[z_{t,n,k}] (Eq. 2).
//
// phi is the multiplicative-XOR form fixed by this library (see engram.h):
// x = XOR_j c[t-j] * m[s][j] in wrapping 64-bit arithmetic, z = x mod p[s].
#include "engram_internal.cuh"

namespace engram {

namespace {

constexpr int kHashThreads = 256;

// One thread per (row, slot): consecutive threads write consecutive int64, so
// the index store is coalesced; the three token reads and map lookups per
// thread hit L1/L2 (the map is at most 512 KB).
// x mod p for a 64-bit x and 2 <= p < 2^31, by Barrett reduction (P. Barrett,
// "Implementing the RSA public key encryption algorithm on a standard digital
// signal processor", CRYPTO 1986): with inv = floor((2^64 - 1) / p), the
// quotient estimate q = floor(x * inv / 2^64) is floor(x / p) or one less, so
// x - q p lies in [0, 2p) and one conditional subtraction gives the exact
// remainder.
__device__ __forceinline__ uint64_t mod_barrett(uint64_t x, uint64_t p, uint64_t inv) {
  const uint64_t q = __umul64hi(x, inv);
  uint64_t r = x - q * p;
  if (r >= p) r -= p;
  return r;
}

__global__ void __launch_bounds__(kHashThreads) hash_kernel(HashArgs a) {
  __shared__ uint64_t s_mult[kMaxTables * kMaxOrders];
  __shared__ uint64_t s_prime[kMaxTables];
  __shared__ uint64_t s_inv[kMaxTables];
  __shared__ int32_t s_order_of_slot[kMaxTables];
  const int S = a.S;
  for (int i = threadIdx.x; i < S * a.max_order; i += blockDim.x) s_mult[i] = a.mult[i];
  for (int i = threadIdx.x; i < S; i += blockDim.x) {
    const uint64_t p = (uint64_t)a.primes[i];
    s_prime[i] = p;
    s_inv[i] = 0xFFFFFFFFFFFFFFFFull / p;
    s_order_of_slot[i] = a.orders[i / a.heads];
  }
  __syncthreads();

  const int Tout = a.T - a.t_begin;
  const int64_t total = (int64_t)a.B * Tout * S;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t row = i / S;
    const int s = (int)(i - row * S);
    const int b = (int)(row / Tout);
    const int t = a.t_begin + (int)(row - (int64_t)b * Tout);
    const int n = s_order_of_slot[s];
    const int32_t* seq = a.tokens + (int64_t)b * a.T;
    uint64_t x = 0;
    for (int j = 0; j < n; ++j) {
      const int pos = t - j;
      uint32_t c = (uint32_t)a.pad;
      if (pos >= 0) {
        const int32_t tok = __ldg(seq + pos);
        if (tok >= 0 && tok < a.V) {
          c = (uint32_t)__ldg(a.map + tok);
        } else {
          atomicOr(a.err, kDevErrToken);
        }
      }
      x ^= (uint64_t)c * s_mult[s * a.max_order + j];
    }
    a.idx[i] = (int64_t)mod_barrett(x, s_prime[s], s_inv[s]);
  }
}

constexpr int kGatherThreads = 256;

__device__ __forceinline__ uint4 ld_stream_16(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// One thread per 16-byte chunk of e.  Consecutive threads cover consecutive
// chunks of one table row (a 160-byte bf16 row is 10 chunks), so each warp
// reads whole rows and writes a contiguous run of e.
__global__ void __launch_bounds__(kGatherThreads) gather_kernel(GatherArgs a) {
  __shared__ const char* s_tab[kMaxTables];
  __shared__ int64_t s_prime[kMaxTables];
  for (int i = threadIdx.x; i < a.S; i += blockDim.x) {
    s_tab[i] = (const char*)a.tables[i];
    s_prime[i] = a.primes[i];
  }
  __syncthreads();
  const int cpr = a.row_bytes >> 4;  // chunks per table row
  const int64_t total = a.rows * a.S * cpr;
  char* e = (char*)a.e;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t rs = i / cpr;
    const int c = (int)(i - rs * cpr);
    const int s = (int)(rs % a.S);
    const int64_t z = __ldg(a.idx + rs);
    uint4 v = make_uint4(0, 0, 0, 0);
    if (z >= 0 && z < s_prime[s]) {
      v = ld_stream_16(s_tab[s] + z * a.row_bytes + c * 16);
    } else if (c == 0) {
      atomicOr(a.err, kDevErrIndex);
    }
    *reinterpret_cast<uint4*>(e + rs * a.row_bytes + c * 16) = v;
  }
}

__global__ void mul_kernel(const float* x, const float* y, float* out, int64_t n) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x)
    out[i] = x[i] * y[i];
}

int grid_for(int64_t work, int threads) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  int64_t blocks = (work + threads - 1) / threads;
  const int64_t cap = (int64_t)sms * 16;
  if (blocks > cap) blocks = cap;
  return blocks < 1 ? 1 : (int)blocks;
}

}  // namespace

cudaError_t launch_hash(const HashArgs& a, cudaStream_t stream) {
  const int64_t total = (int64_t)a.B * (a.T - a.t_begin) * a.S;
  if (total == 0) return cudaSuccess;
  hash_kernel<<<grid_for(total, kHashThreads), kHashThreads, 0, stream>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_gather(const GatherArgs& a, cudaStream_t stream) {
  const int64_t total = a.rows * a.S * (a.row_bytes >> 4);
  if (total == 0) return cudaSuccess;
  gather_kernel<<<grid_for(total, kGatherThreads), kGatherThreads, 0, stream>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_mul(const float* x, const float* y, float* out, int64_t n, cudaStream_t stream) {
  if (n == 0) return cudaSuccess;
  mul_kernel<<<grid_for(n, 256), 256, 0, stream>>>(x, y, out, n);
  return cudaGetLastError();
}

}  // namespace engram
