// Deterministic prefetch of host-resident table rows.
//
// "Conditional Memory via Scalable Lookup", section 2.5 and Figure 2(b): the
// retrieval indices depend only on the token sequence, so they are known
// before the layer runs; the rows are fetched asynchronously from host memory
// over PCIe and the transfer overlaps the preceding blocks' compute.  The
// paper's Table 4 run sends every retrieval over PCIe, and notes that the
// traffic scales with the active rows, not the table size.
//
// Steps 1-4 run on the prefetch stream:
//   1. clear an open-addressing set of 64-bit keys (slot s << 40 | row z);
//   2. insert every (s, z[r, s]) with atomicCAS: one key per distinct row;
//   3. number the occupied buckets: a staging slot per distinct row.  Rows
//      held in the HBM hot-row cache take slots from the back of the staging
//      buffer (count[1]), all others from the front (count[0]), with a list
//      of (s, z) per front slot and of the cache slot per back slot;
//   4. remap every index to its staging slot (a lookup, no waiting on other
//      threads: the slot numbers are final after step 3), and copy the hot
//      rows from the cache into their back slots (HBM to HBM).
// Step 5 moves the front slots' rows, each distinct row once, from pinned
// host memory into the HBM staging buffer, by one of two routes:
//   - host threads read the rows into a pinned bounce buffer and the copy
//     engines send it over PCIe in large copies (engram_host_gather.cu): no
//     SM takes part, so the transfer runs beside any compute;
//   - fetch_kernel reads them through the mapped host address (zero-copy
//     loads over PCIe, 16 bytes per load, eight in flight per thread) on a
//     capped number of CTAs.
// The forward then gathers from the staging buffer with the remapped indices.
//
// Hot-row cache (the paper's cache hierarchy over a Zipfian access pattern,
// section 2.5): engram_build_hot_cache counts the rows calibration tokens
// address (count_kernel) and keeps the most frequent ones in HBM
// (hot_insert_kernel, hot_copy_kernel).
#include "engram_internal.cuh"

namespace engram {

namespace {

constexpr unsigned long long kEmpty = 0xFFFFFFFFFFFFFFFFull;

__device__ __forceinline__ uint32_t mix_bucket(unsigned long long key, uint32_t mask) {
  // 64-bit finaliser (the SplitMix64 output mix) spreads consecutive rows
  unsigned long long z = key + 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  z ^= z >> 31;
  return (uint32_t)z & mask;
}

__global__ void clear_kernel(unsigned long long* keys, int32_t* vals, uint32_t cap,
                             unsigned long long* count) {
  for (uint32_t i = blockIdx.x * blockDim.x + threadIdx.x; i < cap; i += gridDim.x * blockDim.x) {
    keys[i] = kEmpty;
    if (vals) vals[i] = -1;
  }
  if (count && blockIdx.x == 0 && threadIdx.x < 2) count[threadIdx.x] = 0;
}

// Linear probing; the set holds at least twice as many buckets as inserted
// keys, so a probe sequence always meets an empty bucket or its key.
__global__ void insert_kernel(const int64_t* idx, int64_t n, int32_t S, unsigned long long* keys,
                              uint32_t mask) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int s = (int)(i % S);
    const unsigned long long key = ((unsigned long long)s << 40) | (unsigned long long)idx[i];
    uint32_t b = mix_bucket(key, mask);
    for (uint32_t probe = 0; probe <= mask; ++probe) {
      const unsigned long long prev = atomicCAS(keys + b, kEmpty, key);
      if (prev == kEmpty || prev == key) break;
      b = (b + 1) & mask;
    }
  }
}

// Cache slot of key in the hot-row table, or -1.
__device__ __forceinline__ int32_t hot_lookup(const unsigned long long* keys, const int32_t* slots,
                                              uint32_t mask, unsigned long long key) {
  uint32_t b = mix_bucket(key, mask);
  for (uint32_t probe = 0; probe <= mask; ++probe) {
    const unsigned long long k = keys[b];
    if (k == key) return slots[b];
    if (k == kEmpty) return -1;
    b = (b + 1) & mask;
  }
  return -1;
}

// Staging slot per distinct key: rows from the host tables count up from the
// front (count[0]; uniq = (s, z)), rows in the hot-row cache down from the
// back (count[1]; uniq = (-1, cache slot)).  At most `entries` keys exist, so
// the two ranges never meet.
__global__ void number_kernel(PrefetchArgs a) {
  for (uint32_t i = blockIdx.x * blockDim.x + threadIdx.x; i < a.cap; i += gridDim.x * blockDim.x) {
    const unsigned long long k = a.keys[i];
    if (k == kEmpty) continue;
    const int32_t hot = a.hot_keys ? hot_lookup(a.hot_keys, a.hot_slots, a.hot_cap - 1, k) : -1;
    int64_t slot;
    if (hot >= 0) {
      slot = a.rows * a.S - 1 - (int64_t)atomicAdd(a.count + 1, 1ull);
      a.uniq[slot] = make_int2(-1, hot);
    } else {
      slot = (int64_t)atomicAdd(a.count, 1ull);
      a.uniq[slot] = make_int2((int)(k >> 40), (int)(k & 0xFFFFFFFFFFull));
    }
    a.vals[i] = (int32_t)slot;
  }
}

__global__ void remap_kernel(const int64_t* idx, int64_t n, int32_t S,
                             const unsigned long long* keys, const int32_t* vals, uint32_t mask,
                             int64_t* out) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int s = (int)(i % S);
    const unsigned long long key = ((unsigned long long)s << 40) | (unsigned long long)idx[i];
    uint32_t b = mix_bucket(key, mask);
    int64_t v = -1;
    for (uint32_t probe = 0; probe <= mask; ++probe) {
      const unsigned long long k = keys[b];
      if (k == key) {
        v = vals[b];
        break;
      }
      if (k == kEmpty) break;
      b = (b + 1) & mask;
    }
    out[i] = v;  // -1 never happens for a key inserted above; the gather bounds-checks it
  }
}

__device__ __forceinline__ uint4 ld_host_16(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// The hot rows of this prefetch, copied from the cache (HBM) into their
// staging slots at the back of the buffer; one thread per 16-byte chunk.
__global__ void hot_fill_kernel(PrefetchArgs a) {
  const int cpr = a.row_bytes >> 4;
  const int64_t n_hot = (int64_t)a.count[1];
  const int64_t first = a.rows * a.S - n_hot;
  char* staging = (char*)a.staging;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n_hot * cpr;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t u = first + i / cpr;
    const int c = (int)(i % cpr);
    const int2 e = a.uniq[u];
    *reinterpret_cast<uint4*>(staging + u * a.row_bytes + c * 16) = __ldg(
        reinterpret_cast<const uint4*>((const char*)a.hot_rows + (int64_t)e.y * a.row_bytes + c * 16));
  }
}

// Zero-copy route of step 5: the front slots' rows read through the mapped
// host address.  Chunk i = 16 bytes of a row; a thread keeps eight chunks,
// gridDim x blockDim apart, in flight at once (PCIe latency is microseconds,
// so few CTAs need many loads outstanding).
__global__ void fetch_kernel(PrefetchArgs a) {
  const int cpr = a.row_bytes >> 4;
  const int64_t total = (int64_t)a.count[0] * cpr;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  char* staging = (char*)a.staging;
  constexpr int kInFlight = 8;
  for (int64_t i0 = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i0 < total;
       i0 += stride * kInFlight) {
    uint4 v[kInFlight];
#pragma unroll
    for (int k = 0; k < kInFlight; ++k) {
      const int64_t i = i0 + k * stride;
      if (i < total) {
        const int64_t u = i / cpr;
        const int c = (int)(i - u * cpr);
        const int2 sz = a.uniq[u];
        v[k] = ld_host_16((const char*)a.tables[sz.x] + (int64_t)sz.y * a.row_bytes + c * 16);
      }
    }
#pragma unroll
    for (int k = 0; k < kInFlight; ++k) {
      const int64_t i = i0 + k * stride;
      if (i < total) *reinterpret_cast<uint4*>(staging + i * 16) = v[k];
    }
  }
}

// Frequency count for the hot-row cache: insert like insert_kernel, then
// count the key's bucket.
__global__ void count_kernel(const int64_t* idx, int64_t n, int32_t S, unsigned long long* keys,
                             unsigned long long* counts, uint32_t mask) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int s = (int)(i % S);
    const unsigned long long key = ((unsigned long long)s << 40) | (unsigned long long)idx[i];
    uint32_t b = mix_bucket(key, mask);
    for (uint32_t probe = 0; probe <= mask; ++probe) {
      const unsigned long long prev = atomicCAS(keys + b, kEmpty, key);
      if (prev == kEmpty || prev == key) {
        atomicAdd(counts + b, 1ull);
        break;
      }
      b = (b + 1) & mask;
    }
  }
}

__global__ void hot_insert_kernel(const unsigned long long* list, int64_t n,
                                  unsigned long long* keys, int32_t* slots, uint32_t mask) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    const unsigned long long key = list[i];
    uint32_t b = mix_bucket(key, mask);
    for (uint32_t probe = 0; probe <= mask; ++probe) {
      const unsigned long long prev = atomicCAS(keys + b, kEmpty, key);
      if (prev == kEmpty || prev == key) {
        slots[b] = (int32_t)i;
        break;
      }
      b = (b + 1) & mask;
    }
  }
}

__global__ void hot_copy_kernel(const unsigned long long* list, int64_t n,
                                const void* const* tables, int32_t row_bytes, char* rows) {
  const int cpr = row_bytes >> 4;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n * cpr;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t u = i / cpr;
    const int c = (int)(i - u * cpr);
    const unsigned long long key = list[u];
    const int s = (int)(key >> 40);
    const int64_t z = (int64_t)(key & 0xFFFFFFFFFFull);
    *reinterpret_cast<uint4*>(rows + u * row_bytes + c * 16) =
        ld_host_16((const char*)tables[s] + z * row_bytes + c * 16);
  }
}

int blocks_for(int64_t n, int threads, int cap) {
  int64_t b = (n + threads - 1) / threads;
  if (b > cap) b = cap;
  return b < 1 ? 1 : (int)b;
}

}  // namespace

cudaError_t launch_prefetch_index(const PrefetchArgs& a, cudaStream_t stream) {
  const int n = 256;
  const int cap_blocks = a.sms * 16;
  const int64_t entries = a.rows * a.S;
  clear_kernel<<<blocks_for(a.cap, n, cap_blocks), n, 0, stream>>>(a.keys, a.vals, a.cap, a.count);
  if (entries > 0) {
    insert_kernel<<<blocks_for(entries, n, cap_blocks), n, 0, stream>>>(a.idx, entries, a.S,
                                                                       a.keys, a.cap - 1);
    number_kernel<<<blocks_for(a.cap, n, cap_blocks), n, 0, stream>>>(a);
    remap_kernel<<<blocks_for(entries, n, cap_blocks), n, 0, stream>>>(
        a.idx, entries, a.S, a.keys, a.vals, a.cap - 1, a.remapped);
    if (a.hot_keys)
      hot_fill_kernel<<<blocks_for(entries * (a.row_bytes >> 4), n, a.sms * 4), n, 0, stream>>>(a);
  }
  return cudaGetLastError();
}

cudaError_t launch_prefetch_fetch(const PrefetchArgs& a, cudaStream_t stream) {
  const int n = 256;
  const int64_t entries = a.rows * a.S;
  if (entries > 0) {
    // at most `entries` distinct rows
    const int64_t per_block = (int64_t)n * 8;
    fetch_kernel<<<blocks_for(entries * (a.row_bytes >> 4), (int)per_block, a.fetch_blocks), n, 0,
                   stream>>>(a);
  }
  return cudaGetLastError();
}

cudaError_t launch_count_rows(const int64_t* idx, int64_t n, int32_t S, unsigned long long* keys,
                              unsigned long long* counts, uint32_t cap, int sms,
                              cudaStream_t stream) {
  const int t = 256;
  clear_kernel<<<blocks_for(cap, t, sms * 16), t, 0, stream>>>(keys, nullptr, cap, nullptr);
  cudaError_t e = cudaMemsetAsync(counts, 0, (size_t)cap * sizeof(unsigned long long), stream);
  if (e != cudaSuccess) return e;
  if (n > 0) count_kernel<<<blocks_for(n, t, sms * 16), t, 0, stream>>>(idx, n, S, keys, counts, cap - 1);
  return cudaGetLastError();
}

cudaError_t launch_fill_hot_cache(const unsigned long long* list, int64_t n,
                                  unsigned long long* hot_keys, int32_t* hot_slots,
                                  uint32_t hot_cap, const void* const* tables, int32_t row_bytes,
                                  void* rows, int sms, cudaStream_t stream) {
  const int t = 256;
  clear_kernel<<<blocks_for(hot_cap, t, sms * 16), t, 0, stream>>>(hot_keys, hot_slots, hot_cap,
                                                                 nullptr);
  if (n > 0) {
    hot_insert_kernel<<<blocks_for(n, t, sms * 16), t, 0, stream>>>(list, n, hot_keys, hot_slots,
                                                                   hot_cap - 1);
    hot_copy_kernel<<<blocks_for(n * (row_bytes >> 4), t, sms * 8), t, 0, stream>>>(
        list, n, tables, row_bytes, (char*)rows);
  }
  return cudaGetLastError();
}

}  // namespace engram
