// Compress + suffix n-gram + multi-head hash, and the row gather.
//
// "Conditional Memory via Scalable Lookup", section 2.2: x'_t = P(x_t);
// g_{t,n} = (x'_{t-n+1}, ..., x'_t); z_{t,n,k} = phi_{n,k}(g_{t,n}) (Eq. 1);
// e_t = concatenation of E_{n,k}[z_{t,n,k}] (Eq. 2).
//
// phi is the multiplicative-XOR form fixed by this library (see engram.h):
// x = XOR_j c[t-j] * m[s][j] in wrapping 64-bit arithmetic, z = x mod p[s].
#include "e4m3.cuh"
#include "engram_internal.cuh"

namespace engram {

namespace {

constexpr int kHashThreads = 256;

// One thread per (row, slot): consecutive threads write consecutive int64, so
// the index store is coalesced; the three token reads and map lookups per
// thread hit L1/L2 (the map is at most 512 KB).
// x mod p for a 64-bit x and 2 <= p < 2^31, by Barrett reduction (P. Barrett,
// "Implementing the RSA public key encryption algorithm on a standard digital
// signal processor", CRYPTO 1986): with inv = floor((2^64 - 1) / p) (computed
// once on the host when the tables are set), the
// quotient estimate q = floor(x * inv / 2^64) is floor(x / p) or one less, so
// x - q p lies in [0, 2p) and one conditional subtraction gives the exact
// remainder.
__device__ __forceinline__ uint64_t mod_barrett(uint64_t x, uint64_t p, uint64_t inv) {
  const uint64_t q = __umul64hi(x, inv);
  uint64_t r = x - q * p;
  if (r >= p) r -= p;
  return r;
}

// phi_{n,k} of the n-gram ending at position t of one sequence, for table
// slot s: all token loads are issued before the map lookups, and all map
// lookups before the products, so a thread waits on two memory round trips.
__device__ __forceinline__ uint64_t hash_slot(const HashArgs& a, const int32_t* seq, int t, int n,
                                              const uint64_t* mult, uint64_t p, uint64_t inv) {
  int32_t tok[kMaxOrders];
#pragma unroll
  for (int j = 0; j < kMaxOrders; ++j)
    tok[j] = (j < n && t - j >= 0) ? __ldg(seq + t - j) : 0;
  uint32_t c[kMaxOrders];
  bool bad = false;
#pragma unroll
  for (int j = 0; j < kMaxOrders; ++j) {
    c[j] = (uint32_t)a.pad;  // positions before the sequence start
    if (j < n && t - j >= 0) {
      if (tok[j] >= 0 && tok[j] < a.V)
        c[j] = (uint32_t)__ldg(a.map + tok[j]);
      else
        bad = true;
    }
  }
  if (bad) atomicOr(a.err, kDevErrToken);
  uint64_t x = 0;
#pragma unroll
  for (int j = 0; j < kMaxOrders; ++j)
    if (j < n) x ^= (uint64_t)c[j] * mult[j];
  return mod_barrett(x, p, inv);
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
    s_inv[i] = a.barrett[i];
    s_order_of_slot[i] = a.orders[i / a.heads];
  }
  __syncthreads();

  // 32-bit index arithmetic (the launcher keeps B * (T - t_begin) * S < 2^31):
  // 64-bit division is a long software sequence on the GPU
  const uint32_t Tout = (uint32_t)(a.T - a.t_begin);
  const uint32_t total = (uint32_t)a.B * Tout * (uint32_t)S;
  for (uint32_t i = blockIdx.x * blockDim.x + threadIdx.x; i < total; i += gridDim.x * blockDim.x) {
    const uint32_t row = i / (uint32_t)S;
    const int s = (int)(i - row * (uint32_t)S);
    const int b = (int)(row / Tout);
    const int t = a.t_begin + (int)(row - (uint32_t)b * Tout);
    a.idx[i] = (int64_t)hash_slot(a, a.tokens + (int64_t)b * a.T, t, s_order_of_slot[s],
                                  s_mult + s * a.max_order, s_prime[s], s_inv[s]);
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
// Address of row z of table s: whole tables, or row-sharded ones (owner z %
// N, local row z / N; z < 2^31).
__device__ __forceinline__ const char* row_addr(const char* const* tab, int s, uint64_t z,
                                                int shards, int64_t row_bytes) {
  if (shards == 1) return tab[s] + z * (uint64_t)row_bytes;
  const uint32_t zz = (uint32_t)z, q = zz / (uint32_t)shards;
  return tab[s * shards + (int)(zz - q * (uint32_t)shards)] + (uint64_t)q * (uint64_t)row_bytes;
}

__global__ void __launch_bounds__(kGatherThreads) gather_kernel(GatherArgs a) {
  griddep_launch_dependents();  // the key phase may set up while this runs
  __shared__ const char* s_tab[kMaxTables * kMaxShards];
  __shared__ int64_t s_prime[kMaxTables];
  for (int i = threadIdx.x; i < a.S * a.shards; i += blockDim.x) s_tab[i] = (const char*)a.tables[i];
  for (int i = threadIdx.x; i < a.S; i += blockDim.x) s_prime[i] = a.primes[i];
  __syncthreads();
  const uint32_t cpr = (uint32_t)(a.row_bytes >> 4);  // chunks per table row
  const uint32_t S = (uint32_t)a.S;
  // 32-bit index arithmetic (the launcher keeps rows * S * cpr < 2^31)
  const uint32_t total = (uint32_t)a.rows * S * cpr;
  char* e = (char*)a.e;
  for (uint32_t i = blockIdx.x * blockDim.x + threadIdx.x; i < total; i += gridDim.x * blockDim.x) {
    const uint32_t rs = i / cpr;
    const uint32_t c = i - rs * cpr;
    const uint32_t s = rs % S;
    const int64_t z = __ldg(a.idx + rs);
    uint4 v = make_uint4(0, 0, 0, 0);
    if (z >= 0 && z < s_prime[s]) {
      v = ld_stream_16(row_addr(s_tab, (int)s, (uint64_t)z, a.shards, a.row_bytes) + c * 16);
    } else if (c == 0) {
      atomicOr(a.err, kDevErrIndex);
    }
    *reinterpret_cast<uint4*>(e + (int64_t)rs * a.row_bytes + c * 16) = v;
  }
}

// Hash and gather fused: a block owns up to 256 / S consecutive output rows.  Its
// threads first compute the rows' S indices each (one per thread, as in
// hash_kernel) and keep the source row addresses in shared memory; then they
// copy the rows' table rows into e, 16 bytes per thread and load, four loads
// in flight per thread.  The block's part of e is one contiguous run, so the
// stores are coalesced, and the indices never travel through HBM.
constexpr int kFusedThreads = 256;

__global__ void __launch_bounds__(kFusedThreads) hash_gather_kernel(HashGatherArgs g) {
  griddep_launch_dependents();  // the key phase may set up while this runs
  const HashArgs& a = g.hash;
  __shared__ uint64_t s_mult[kMaxTables * kMaxOrders];
  __shared__ uint64_t s_prime[kMaxTables];
  __shared__ uint64_t s_inv[kMaxTables];
  __shared__ int32_t s_order_of_slot[kMaxTables];
  __shared__ const char* s_tab[kMaxTables * kMaxShards];
  __shared__ const char* s_src[kFusedThreads];  // source row of (row, slot)
  const int S = a.S;
  for (int i = threadIdx.x; i < S * a.max_order; i += blockDim.x) s_mult[i] = a.mult[i];
  for (int i = threadIdx.x; i < S; i += blockDim.x) {
    s_prime[i] = (uint64_t)a.primes[i];
    s_inv[i] = a.barrett[i];
    s_order_of_slot[i] = a.orders[i / a.heads];
  }
  for (int i = threadIdx.x; i < S * g.shards; i += blockDim.x) s_tab[i] = (const char*)g.tables[i];
  __syncthreads();

  const uint32_t Tout = (uint32_t)(a.T - a.t_begin);
  const uint32_t rows = (uint32_t)a.B * Tout;
  const uint32_t rb = (uint32_t)g.rows_per_block;  // <= 256 / S
  const uint32_t row0 = blockIdx.x * rb;
  const uint32_t nrows = min(rb, rows - row0);
  const uint32_t nslots = nrows * (uint32_t)S;
  if (threadIdx.x < nslots) {
    const uint32_t rl = threadIdx.x / (uint32_t)S;
    const int s = (int)(threadIdx.x - rl * (uint32_t)S);
    const uint32_t row = row0 + rl;
    const int b = (int)(row / Tout);
    const int t = a.t_begin + (int)(row - (uint32_t)b * Tout);
    const uint64_t z = hash_slot(a, a.tokens + (int64_t)b * a.T, t, s_order_of_slot[s],
                                 s_mult + s * a.max_order, s_prime[s], s_inv[s]);
    s_src[threadIdx.x] = row_addr(s_tab, s, z, g.shards, g.row_bytes);
  }
  __syncthreads();

  const uint32_t cpr = (uint32_t)(g.row_bytes >> 4);
  const uint32_t nchunks = nslots * cpr;
  // row0 * S * row_bytes < 2^31 * 16 by the launcher's bound
  uint4* dst = reinterpret_cast<uint4*>((char*)g.e + (int64_t)row0 * S * g.row_bytes);
  // e is written evict-last (the projection launches read it next, with the
  // same policy), the table rows, read once, evict-first
  uint64_t keep, once;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(keep));
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(once));
  constexpr int kInFlight = 4;
  for (uint32_t i0 = threadIdx.x; i0 < nchunks; i0 += kInFlight * kFusedThreads) {
    uint4 v[kInFlight];
#pragma unroll
    for (int k = 0; k < kInFlight; ++k) {
      const uint32_t i = i0 + k * kFusedThreads;
      if (i < nchunks) {
        const uint32_t rs = i / cpr;
        asm volatile("ld.global.nc.L1::no_allocate.L2::cache_hint.v4.u32 {%0,%1,%2,%3}, [%4], %5;"
                     : "=r"(v[k].x), "=r"(v[k].y), "=r"(v[k].z), "=r"(v[k].w)
                     : "l"(s_src[rs] + (i - rs * cpr) * 16), "l"(once));
      }
    }
#pragma unroll
    for (int k = 0; k < kInFlight; ++k) {
      const uint32_t i = i0 + k * kFusedThreads;
      if (i < nchunks)
        asm volatile("st.global.L2::cache_hint.v4.u32 [%0], {%1,%2,%3,%4}, %5;" ::"l"(dst + i),
                     "r"(v[k].x), "r"(v[k].y), "r"(v[k].z), "r"(v[k].w), "l"(keep)
                     : "memory");
    }
  }
  // the previous kernel (which this one may have overlapped) is complete
  // before this block, and so this kernel, completes
  if (threadIdx.x == 0) griddep_wait();
}

// Hash, gather and E4M3 quantisation fused (the FP8 projections): the hash
// stage is hash_gather_kernel's; then each warp takes whole rows of the block,
// loads the row's S table rows (each lane up to 8 chunks of 16 bytes, all in
// flight together), reduces the row's largest magnitude over the warp and
// writes the row's codes (half the bytes of e) and its scale.
__global__ void __launch_bounds__(kFusedThreads) hash_gather_e4m3_kernel(HashGatherArgs g) {
  griddep_launch_dependents();  // the key phase may set up while this runs
  const HashArgs& a = g.hash;
  __shared__ uint64_t s_mult[kMaxTables * kMaxOrders];
  __shared__ uint64_t s_prime[kMaxTables];
  __shared__ uint64_t s_inv[kMaxTables];
  __shared__ int32_t s_order_of_slot[kMaxTables];
  __shared__ const char* s_tab[kMaxTables * kMaxShards];
  __shared__ const char* s_src[kFusedThreads];  // source row of (row, slot)
  const int S = a.S;
  for (int i = threadIdx.x; i < S * a.max_order; i += blockDim.x) s_mult[i] = a.mult[i];
  for (int i = threadIdx.x; i < S; i += blockDim.x) {
    s_prime[i] = (uint64_t)a.primes[i];
    s_inv[i] = a.barrett[i];
    s_order_of_slot[i] = a.orders[i / a.heads];
  }
  for (int i = threadIdx.x; i < S * g.shards; i += blockDim.x) s_tab[i] = (const char*)g.tables[i];
  __syncthreads();

  const uint32_t Tout = (uint32_t)(a.T - a.t_begin);
  const uint32_t rows = (uint32_t)a.B * Tout;
  const uint32_t rb = (uint32_t)g.rows_per_block;  // <= 256 / S
  const uint32_t row0 = blockIdx.x * rb;
  const uint32_t nrows = min(rb, rows - row0);
  const uint32_t nslots = nrows * (uint32_t)S;
  if (threadIdx.x < nslots) {
    const uint32_t rl = threadIdx.x / (uint32_t)S;
    const int s = (int)(threadIdx.x - rl * (uint32_t)S);
    const uint32_t row = row0 + rl;
    const int b = (int)(row / Tout);
    const int t = a.t_begin + (int)(row - (uint32_t)b * Tout);
    const uint64_t z = hash_slot(a, a.tokens + (int64_t)b * a.T, t, s_order_of_slot[s],
                                 s_mult + s * a.max_order, s_prime[s], s_inv[s]);
    s_src[threadIdx.x] = row_addr(s_tab, s, z, g.shards, g.row_bytes);
  }
  __syncthreads();

  const int cpr = g.row_bytes >> 4;  // chunks per table row
  const int C = S * cpr;             // chunks per row of e (<= 32 * kQuantMaxChunks)
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (uint32_t rl = warp; rl < nrows; rl += kFusedThreads / 32) {
    const char* const* src = s_src + rl * S;
    auto chunk = [&](int c) {
      const int s = c / cpr;
      return ld_stream_16(src[s] + (c - s * cpr) * 16);
    };
    quant_row_warp(chunk, C, g.q + (int64_t)(row0 + rl) * C * 8, g.scale + row0 + rl, lane);
  }
  if (threadIdx.x == 0) griddep_wait();  // as in hash_gather_kernel
}

// E4M3 codes and scales of bf16 rows (the quantiser on its own: for W when
// the FP8 projections are switched on, and for e gathered by gather_kernel).
// One warp per row.
__global__ void __launch_bounds__(256) quantize_rows_kernel(const uint16_t* x, int64_t rows,
                                                            int cols, uint8_t* q, float* scale) {
  const int lane = threadIdx.x & 31;
  const int C = cols / 8;
  const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x / 32);
  for (int64_t r = (int64_t)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5); r < rows;
       r += nwarps) {
    const uint4* src = reinterpret_cast<const uint4*>(x + r * cols);
    auto chunk = [&](int c) { return ld_stream_16(src + c); };
    quant_row_warp(chunk, C, q + r * cols, scale + r, lane);
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
  if (total >= ((int64_t)1 << 31)) return cudaErrorInvalidValue;
  hash_kernel<<<grid_for(total, kHashThreads), kHashThreads, 0, stream>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_gather(const GatherArgs& a, cudaStream_t stream) {
  const int64_t total = a.rows * a.S * (a.row_bytes >> 4);
  if (total == 0) return cudaSuccess;
  if (total >= ((int64_t)1 << 31)) return cudaErrorInvalidValue;
  gather_kernel<<<grid_for(total, kGatherThreads), kGatherThreads, 0, stream>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_hash_gather(const HashGatherArgs& a, cudaStream_t stream) {
  const int64_t rows = (int64_t)a.hash.B * (a.hash.T - a.hash.t_begin);
  if (rows == 0) return cudaSuccess;
  if (a.hash.S < 1 || a.hash.S > kMaxTables) return cudaErrorInvalidValue;
  if (rows * a.hash.S * (a.row_bytes >> 4) >= ((int64_t)1 << 31)) return cudaErrorInvalidValue;
  // 256 / S rows per block, fewer when that leaves SMs idle (short calls,
  // e.g. decode): the copies of a block then take a single round
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  int64_t rb = kFusedThreads / a.hash.S;
  const int64_t fill = (rows + 2 * (int64_t)sms - 1) / (2 * (int64_t)sms);
  if (fill < rb) rb = fill < 1 ? 1 : fill;
  HashGatherArgs b = a;
  b.rows_per_block = (int32_t)rb;
  cudaLaunchConfig_t lc = {};
  lc.gridDim = dim3((unsigned)((rows + rb - 1) / rb));
  lc.blockDim = dim3(kFusedThreads);
  lc.stream = stream;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  lc.attrs = at;
  lc.numAttrs = b.pdl ? 1 : 0;
  cudaError_t e = cudaLaunchKernelEx(&lc, hash_gather_kernel, b);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t launch_hash_gather_e4m3(const HashGatherArgs& a, cudaStream_t stream) {
  const int64_t rows = (int64_t)a.hash.B * (a.hash.T - a.hash.t_begin);
  if (rows == 0) return cudaSuccess;
  if (a.hash.S < 1 || a.hash.S > kMaxTables) return cudaErrorInvalidValue;
  const int64_t chunks = (int64_t)a.hash.S * (a.row_bytes >> 4);
  if (chunks > 32 * kQuantMaxChunks || rows * chunks >= ((int64_t)1 << 31))
    return cudaErrorInvalidValue;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  int64_t rb = kFusedThreads / a.hash.S;
  const int64_t fill = (rows + 2 * (int64_t)sms - 1) / (2 * (int64_t)sms);
  if (fill < rb) rb = fill < 1 ? 1 : fill;
  HashGatherArgs b = a;
  b.rows_per_block = (int32_t)rb;
  cudaLaunchConfig_t lc = {};
  lc.gridDim = dim3((unsigned)((rows + rb - 1) / rb));
  lc.blockDim = dim3(kFusedThreads);
  lc.stream = stream;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  lc.attrs = at;
  lc.numAttrs = b.pdl ? 1 : 0;
  cudaError_t e = cudaLaunchKernelEx(&lc, hash_gather_e4m3_kernel, b);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t launch_quantize_e4m3(const void* x, int64_t rows, int cols, uint8_t* q, float* scale,
                                 cudaStream_t stream) {
  if (rows == 0) return cudaSuccess;
  if (cols < 16 || cols % 16 || cols > 8 * 32 * kQuantMaxChunks) return cudaErrorInvalidValue;
  // a warp per row, eight rows per block, at most 16 blocks per SM (grid-stride)
  quantize_rows_kernel<<<grid_for(rows * 32, 256), 256, 0, stream>>>(static_cast<const uint16_t*>(x), rows, cols, q,
                                                  scale);
  return cudaGetLastError();
}

cudaError_t launch_mul(const float* x, const float* y, float* out, int64_t n, cudaStream_t stream) {
  if (n == 0) return cudaSuccess;
  mul_kernel<<<grid_for(n, 256), 256, 0, stream>>>(x, y, out, n);
  return cudaGetLastError();
}

}  // namespace engram
