// C ABI of libengram.so (declared in include/engram.h): configuration checks,
// the handle and its scratch, tensor maps, and the launch sequence of the
// Engram forward ("Conditional Memory via Scalable Lookup", section 2).
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <new>
#include <thread>
#include <string>
#include <utility>
#include <vector>

#include "engram_handle.cuh"

using namespace engram;


namespace {

thread_local std::string g_create_error;

int fail(engram_handle* h, int code, const std::string& msg) {
  if (h)
    h->last_error = msg;
  else
    g_create_error = msg;
  return code;
}

int cuda_fail(engram_handle* h, cudaError_t e, const char* what) {
  return fail(h, e == cudaErrorMemoryAllocation ? ENGRAM_ERR_OOM : ENGRAM_ERR_CUDA,
              std::string(what) + ": " + cudaGetErrorString(e));
}

#define CK(h, call)                                       \
  do {                                                    \
    cudaError_t e__ = (call);                             \
    if (e__ != cudaSuccess) return cuda_fail(h, e__, #call); \
  } while (0)

// SplitMix64 (Steele, Lea and Flood, OOPSLA 2014): the multiplier stream.
uint64_t splitmix64(uint64_t& state) {
  state += 0x9E3779B97F4A7C15ull;
  uint64_t z = state;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

bool prime(int64_t n) {
  if (n < 2) return false;
  if (n % 2 == 0) return n == 2;
  for (int64_t f = 3; f <= n / f; f += 2)
    if (n % f == 0) return false;
  return true;
}

template <class T>
void free_dev(T*& p) {
  if (p) cudaFree((void*)p);
  p = nullptr;
}

}  // namespace

namespace engram {

// The driver's tensor-map encoder, looked up once (a function-local static:
// its initialisation is thread-safe).
static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static const PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    return (PFN_cuTensorMapEncodeTiled_v12000) nullptr;
  }();
  return fn;
}

// 2-D row-major tensor map: `rows` rows of `cols` elements of esz bytes (2:
// bf16, 4: fp32, 1: E4M3 codes), box box_cols x box_rows; the swizzle follows
// the box's row bytes (128-byte rows: 128-byte swizzle, 64-byte rows: 64-byte
// swizzle).
int make_map(engram_handle* h, CUtensorMap* m, const void* base, int64_t cols, int64_t rows,
             int box_rows, int box_cols, int esz) {
  auto fn = encode_fn();
  if (!fn) return fail(h, ENGRAM_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  const CUtensorMapDataType dt = esz == 4   ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                                 : esz == 1 ? CU_TENSOR_MAP_DATA_TYPE_UINT8
                                            : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)cols * esz};
  cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1u, 1u};
  const CUtensorMapSwizzle sw =
      box_cols * esz == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  CUresult r = fn(m, dt, 2,
                  const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(h, ENGRAM_ERR_CUDA, "cuTensorMapEncodeTiled failed");
  return ENGRAM_OK;
}

int cached_map(engram_handle* h, CUtensorMap* m, const void* base, int64_t cols, int64_t rows,
               int box_rows, int box_cols, int esz) {
  for (const auto& e : h->map_cache) {
    if (e.base == base && e.cols == cols && e.rows == rows && e.box_rows == box_rows &&
        e.box_cols == box_cols && e.esz == esz) {
      *m = e.map;
      return ENGRAM_OK;
    }
  }
  const int rc = make_map(h, m, base, cols, rows, box_rows, box_cols, esz);
  if (rc) return rc;
  auto& e = h->map_cache[h->map_cache_next];
  h->map_cache_next = (h->map_cache_next + 1) % engram_handle::kMapCache;
  e.base = base;
  e.cols = cols;
  e.rows = rows;
  e.box_rows = box_rows;
  e.box_cols = box_cols;
  e.esz = esz;
  e.map = *m;
  return ENGRAM_OK;
}

}  // namespace engram

namespace {

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

int ensure_scratch(engram_handle* h, int64_t rows) {
  if (!h->fused_sync && h->cfg.dtype == ENGRAM_BF16 && h->cfg.d_hidden % 256 == 0) {
    // the fused short-call kernel's counters (zero before its first launch,
    // zeroed again by every launch on its way out) and its v hand-off buffer
    CK(h, cudaMalloc(&h->fused_vt, (size_t)h->cfg.d_hidden * 256 * sizeof(float)));
    CK(h, cudaMalloc(&h->fused_sync, engram::kFusedSyncWords * sizeof(unsigned)));
    CK(h, cudaMemset(h->fused_sync, 0, engram::kFusedSyncWords * sizeof(unsigned)));
    CK(h, cudaDeviceSynchronize());
  }
  if (rows <= h->cap_rows) return ENGRAM_OK;
  free_dev(h->e);
  free_dev(h->e_alt);
  free_dev(h->partials);
  free_dev(h->alpha_scratch);
  h->cap_rows = 0;
  const int64_t key_tiles = (int64_t)h->cfg.branches * h->cfg.d_hidden / 64;
  CK(h, cudaMalloc(&h->alpha_scratch, (size_t)rows * h->cfg.branches * sizeof(float)));
  CK(h, cudaMalloc(&h->e, (size_t)rows * h->d_mem * h->elt));
  CK(h, cudaMalloc(&h->e_alt, (size_t)rows * h->d_mem * h->elt));
  CK(h, cudaMalloc(&h->partials, (size_t)rows * key_tiles * sizeof(float4)));
  h->cap_rows = rows;
  return ENGRAM_OK;
}

int ensure_fp8_scratch(engram_handle* h, int64_t rows) {
  if (rows <= h->fp8_cap_rows) return ENGRAM_OK;
  free_dev(h->e8);
  free_dev(h->se8);
  free_dev(h->e8_alt);
  free_dev(h->se8_alt);
  h->fp8_cap_rows = 0;
  CK(h, cudaMalloc(&h->e8, (size_t)rows * h->d_mem));
  CK(h, cudaMalloc(&h->se8, (size_t)rows * sizeof(float)));
  CK(h, cudaMalloc(&h->e8_alt, (size_t)rows * h->d_mem));
  CK(h, cudaMalloc(&h->se8_alt, (size_t)rows * sizeof(float)));
  h->fp8_cap_rows = rows;
  return ENGRAM_OK;
}

// E4M3 copy of [W_K; W_V] (one scale per row) and its tensor maps (boxes of
// 128 rows x 128 codes for the CTA-pair kernel); synchronises the device.
int quantize_weights(engram_handle* h, cudaStream_t st) {
  const int64_t M = h->cfg.branches, d = h->cfg.d_hidden, dm = h->d_mem;
  if (!h->d_w8) {
    CK(h, cudaMalloc(&h->d_w8, (size_t)(M + 1) * d * dm));
    CK(h, cudaMalloc(&h->d_sw8, (size_t)(M + 1) * d * sizeof(float)));
  }
  CK(h, launch_quantize_e4m3(h->w_k, M * d, (int)dm, h->d_w8, h->d_sw8, st));
  CK(h, launch_quantize_e4m3(h->w_v, d, (int)dm, h->d_w8 + M * d * dm, h->d_sw8 + M * d, st));
  h->launches += 2;
  CK(h, cudaDeviceSynchronize());
  int rc = make_map(h, &h->map_wk8, h->d_w8, dm, M * d, 128, 128, 1);
  if (rc) return rc;
  return make_map(h, &h->map_wv8, h->d_w8 + M * d * dm, dm, d, 128, 128, 1);
}

int ensure_conv_scratch(engram_handle* h, int64_t rows) {
  if (rows <= h->conv_cap_rows) return ENGRAM_OK;
  free_dev(h->conv_v);
  free_dev(h->conv_vv);
  free_dev(h->conv_alpha);
  free_dev(h->conv_scale);
  h->conv_cap_rows = 0;
  const int d = h->cfg.d_hidden;
  CK(h, cudaMalloc(&h->conv_v, (size_t)rows * d * sizeof(float)));
  CK(h, cudaMalloc(&h->conv_vv, (size_t)rows * (d / 64) * sizeof(float)));
  CK(h, cudaMalloc(&h->conv_alpha, (size_t)rows * h->cfg.branches * sizeof(float)));
  CK(h, cudaMalloc(&h->conv_scale, (size_t)rows * h->cfg.branches * sizeof(float)));
  h->conv_cap_rows = rows;
  return ENGRAM_OK;
}

int check_shape(engram_handle* h, int32_t B, int32_t T, int32_t t_begin) {
  if (B < 0 || T < 0) return fail(h, ENGRAM_ERR_INVALID, "B and T must be >= 0");
  if (B > 0 && T > 0 && (t_begin < 0 || t_begin >= T))
    return fail(h, ENGRAM_ERR_INVALID, "t_begin must lie in [0, T)");
  const int64_t rows = (int64_t)B * (T - t_begin);
  const int64_t per_row = (int64_t)h->S * ((h->cfg.d_head * h->elt) >> 4);  // gather chunks per row
  if (rows * per_row >= ((int64_t)1 << 31))
    return fail(h, ENGRAM_ERR_INVALID, "too many rows for one call (rows x tables x row chunks >= 2^31)");
  return ENGRAM_OK;
}

HashArgs hash_args(engram_handle* h, const int32_t* tokens, int32_t B, int32_t T, int32_t t_begin,
                   int64_t* idx) {
  HashArgs a{};
  a.tokens = tokens;
  a.map = h->d_map;
  a.mult = h->d_mult;
  a.primes = h->d_primes;
  a.barrett = h->d_barrett;
  a.idx = idx;
  a.err = h->d_err;
  a.V = h->cfg.vocab;
  a.pad = h->cfg.pad_id;
  a.B = B;
  a.T = T;
  a.t_begin = t_begin;
  a.S = h->S;
  a.heads = h->cfg.heads;
  a.num_orders = h->cfg.num_orders;
  a.max_order = h->max_order;
  for (int i = 0; i < kMaxOrders; ++i) a.orders[i] = h->cfg.orders[i];
  return a;
}

void free_host_gather(engram_handle* h) {
  delete h->hg;  // waits for its queued jobs
  h->hg = nullptr;
  for (int i = 0; i < 2; ++i) {
    if (h->h_count[i]) cudaFreeHost(h->h_count[i]);
    if (h->h_list[i]) cudaFreeHost(h->h_list[i]);
    if (h->h_bounce[i]) cudaFreeHost(h->h_bounce[i]);
    h->h_count[i] = nullptr;
    h->h_list[i] = nullptr;
    h->h_bounce[i] = nullptr;
  }
}

// Pinned buffers, copy stream, events and threads of the host-thread route
// for `entries` (row, table) lookups per prefetch.
int ensure_host_gather(engram_handle* h, int64_t entries) {
  const size_t row_bytes = (size_t)h->cfg.d_head * h->elt;
  for (int i = 0; i < 2; ++i) {
    if (!h->h_count[i])
      CK(h, cudaHostAlloc((void**)&h->h_count[i], 2 * sizeof(unsigned long long),
                          cudaHostAllocDefault));
    if (!h->h_list[i])
      CK(h, cudaHostAlloc((void**)&h->h_list[i], (size_t)entries * sizeof(int2),
                          cudaHostAllocDefault));
    if (!h->h_bounce[i])
      CK(h, cudaHostAlloc((void**)&h->h_bounce[i], (size_t)entries * row_bytes,
                          cudaHostAllocDefault));
    if (!h->ev_list[i]) CK(h, cudaEventCreateWithFlags(&h->ev_list[i], cudaEventDisableTiming));
  }
  if (!h->copy_stream) CK(h, cudaStreamCreateWithFlags(&h->copy_stream, cudaStreamNonBlocking));
  if (!h->hg) {
    int n = h->pf_workers;
    if (n <= 0) {
      const int hw = (int)std::thread::hardware_concurrency();
      n = std::max(1, std::min(8, hw / 2));
    }
    h->hg = new (std::nothrow) HostGather(h->device, n);
    if (!h->hg) return fail(h, ENGRAM_ERR_OOM, "host gather threads");
  }
  return ENGRAM_OK;
}

int ensure_prefetch_scratch(engram_handle* h, int64_t rows) {
  if (rows <= h->pf_cap_rows) {
    if (h->pf_mode == ENGRAM_PREFETCH_HOST_THREADS)
      return ensure_host_gather(h, h->pf_cap_rows * h->S);
    return ENGRAM_OK;
  }
  // growing frees the staging buffers, which a pending prefetch has filled
  if (h->n_prefetch != h->n_consumed)
    return fail(h, ENGRAM_ERR_STATE,
                "a larger batch while a prefetch is pending; engram_reserve the largest batch "
                "first, or run engram_forward first");
  // the staging buffers may still be in use by queued work
  CK(h, cudaDeviceSynchronize());
  free_host_gather(h);
  free_dev(h->d_keys);
  free_dev(h->d_vals);
  free_dev(h->d_uniq);
  free_dev(h->d_stage_bound);
  for (int i = 0; i < 2; ++i) {
    free_dev(h->d_count[i]);
    free_dev(h->d_remap[i]);
    free_dev(h->d_staging[i]);
    free_dev(h->d_stage_tables[i]);
  }
  h->pf_cap_rows = 0;
  const int64_t entries = rows * h->S;
  uint64_t cap = 1;
  while (cap < (uint64_t)(2 * entries)) cap <<= 1;
  if (cap > (1ull << 31)) return fail(h, ENGRAM_ERR_INVALID, "prefetch batch too large");
  h->set_cap = (uint32_t)cap;
  const size_t row_bytes = (size_t)h->cfg.d_head * h->elt;
  CK(h, cudaMalloc(&h->d_keys, cap * sizeof(unsigned long long)));
  CK(h, cudaMalloc(&h->d_vals, cap * sizeof(int32_t)));
  CK(h, cudaMalloc(&h->d_uniq, (size_t)entries * sizeof(int2)));
  CK(h, cudaMalloc(&h->d_stage_bound, h->S * sizeof(int64_t)));
  int64_t bound[kMaxTables];
  for (int s = 0; s < h->S; ++s) bound[s] = entries;
  CK(h, cudaMemcpy(h->d_stage_bound, bound, h->S * sizeof(int64_t), cudaMemcpyHostToDevice));
  for (int i = 0; i < 2; ++i) {
    CK(h, cudaMalloc(&h->d_count[i], 2 * sizeof(unsigned long long)));
    CK(h, cudaMemset(h->d_count[i], 0, 2 * sizeof(unsigned long long)));
    CK(h, cudaMalloc(&h->d_remap[i], (size_t)entries * sizeof(int64_t)));
    CK(h, cudaMalloc(&h->d_staging[i], (size_t)entries * row_bytes));
    CK(h, cudaMalloc(&h->d_stage_tables[i], h->S * sizeof(void*)));
    const void* ptrs[kMaxTables];
    for (int s = 0; s < h->S; ++s) ptrs[s] = h->d_staging[i];
    CK(h, cudaMemcpy(h->d_stage_tables[i], ptrs, h->S * sizeof(void*), cudaMemcpyHostToDevice));
  }
  h->pf_cap_rows = rows;
  if (h->pf_mode == ENGRAM_PREFETCH_HOST_THREADS) return ensure_host_gather(h, entries);
  return ENGRAM_OK;
}

}  // namespace

extern "C" {

size_t engram_config_size(void) { return sizeof(engram_config); }

const char* engram_last_error(const engram_handle* h) {
  return h ? h->last_error.c_str() : g_create_error.c_str();
}

int engram_create(const engram_config* cfg, engram_handle** out) {
  if (!cfg || !out) return fail(nullptr, ENGRAM_ERR_INVALID, "null argument");
  *out = nullptr;
  const engram_config& c = *cfg;
  if (c.vocab < 1 || c.cvocab < 1 || c.cvocab > c.vocab)
    return fail(nullptr, ENGRAM_ERR_INVALID, "need 1 <= cvocab <= vocab");
  if (!c.comp_map) return fail(nullptr, ENGRAM_ERR_INVALID, "comp_map is required");
  if (c.num_orders < 1 || c.num_orders > ENGRAM_MAX_ORDERS)
    return fail(nullptr, ENGRAM_ERR_INVALID, "num_orders must lie in [1, 4]");
  for (int i = 0; i < c.num_orders; ++i) {
    if (c.orders[i] < 1 || c.orders[i] > ENGRAM_MAX_ORDERS)
      return fail(nullptr, ENGRAM_ERR_INVALID, "n-gram orders must lie in [1, 4]");
    if (i > 0 && c.orders[i] <= c.orders[i - 1])
      return fail(nullptr, ENGRAM_ERR_INVALID, "n-gram orders must be strictly ascending");
  }
  if (c.heads < 1 || c.num_orders * c.heads > ENGRAM_MAX_TABLES)
    return fail(nullptr, ENGRAM_ERR_INVALID, "need 1 <= heads and orders*heads <= 64");
  if (c.dtype != ENGRAM_F32 && c.dtype != ENGRAM_BF16)
    return fail(nullptr, ENGRAM_ERR_INVALID, "dtype must be ENGRAM_F32 or ENGRAM_BF16");
  const int elt = c.dtype == ENGRAM_F32 ? 4 : 2;
  if (c.d_head < 1 || (c.d_head * elt) % 16 != 0)
    return fail(nullptr, ENGRAM_ERR_INVALID, "d_head * element size must be a multiple of 16");
  if (c.d_hidden < 64 || c.d_hidden % 64 != 0)
    return fail(nullptr, ENGRAM_ERR_INVALID, "d_hidden must be a positive multiple of 64");
  if (c.branches < 1 || c.branches > ENGRAM_MAX_BRANCHES)
    return fail(nullptr, ENGRAM_ERR_INVALID, "branches must lie in [1, 4]");
  if (!(c.eps >= 0.f) || !std::isfinite(c.eps))
    return fail(nullptr, ENGRAM_ERR_INVALID, "eps must be finite and >= 0");
  if (c.table_location != ENGRAM_DEVICE && c.table_location != ENGRAM_PINNED_HOST)
    return fail(nullptr, ENGRAM_ERR_INVALID, "bad table_location");
  if (c.pad_id < -1) return fail(nullptr, ENGRAM_ERR_INVALID, "pad_id must be >= -1");
  if (c.flags & ~(ENGRAM_FLAG_NO_CTA_PAIRS | ENGRAM_FLAG_NO_FUSED_SHORT))
    return fail(nullptr, ENGRAM_ERR_INVALID, "unknown flags");
  const int S = c.num_orders * c.heads;
  const int64_t d_mem = (int64_t)S * c.d_head;
  if (d_mem > (1 << 20)) return fail(nullptr, ENGRAM_ERR_INVALID, "d_mem too large");

  int64_t primes[kMaxTables];
  int given = 0;
  for (int s = 0; s < S; ++s) given += c.primes[s] != 0;
  if (given != 0 && given != S)
    return fail(nullptr, ENGRAM_ERR_INVALID, "give all table sizes or none");
  if (given == S) {
    for (int s = 0; s < S; ++s) {
      if (c.primes[s] < 2 || c.primes[s] >= ((int64_t)1 << 31))
        return fail(nullptr, ENGRAM_ERR_INVALID, "table sizes must lie in [2, 2^31)");
      primes[s] = c.primes[s];
    }
  } else {
    if (c.table_rows_target < 2 || c.table_rows_target >= ((int64_t)1 << 31) - 4096)
      return fail(nullptr, ENGRAM_ERR_INVALID, "table_rows_target must lie in [2, 2^31 - 4096)");
    int64_t n = c.table_rows_target;
    for (int s = 0; s < S; ++s) {
      while (!prime(n)) ++n;
      primes[s] = n++;
    }
  }
  for (int i = 0; i < c.vocab; ++i)
    if (c.comp_map[i] < 0 || c.comp_map[i] >= c.cvocab)
      return fail(nullptr, ENGRAM_ERR_INVALID, "comp_map values must lie in [0, cvocab)");

  engram_handle* h = new (std::nothrow) engram_handle();
  if (!h) return fail(nullptr, ENGRAM_ERR_OOM, "host allocation failed");
  h->cfg = c;
  h->cfg.comp_map = nullptr;
  if (h->cfg.pad_id == -1) h->cfg.pad_id = c.cvocab;
  h->S = S;
  h->elt = elt;
  h->d_mem = (int)d_mem;
  h->max_order = c.orders[c.num_orders - 1];
  for (int s = 0; s < S; ++s) h->primes[s] = primes[s];
  uint64_t st = c.hash_seed;
  for (int s = 0; s < S; ++s)
    for (int j = 0; j < h->max_order; ++j) h->mult[s * h->max_order + j] = splitmix64(st) | 1ull;

  auto bail = [&](int code) {
    g_create_error = h->last_error;
    engram_destroy(h);
    return code;
  };
  int rc;
  if ((rc = [&]() -> int {
         CK(h, cudaGetDevice(&h->device));
         CK(h, cudaDeviceGetAttribute(&h->sms, cudaDevAttrMultiProcessorCount, h->device));
         CK(h, cudaMalloc(&h->d_map, (size_t)c.vocab * sizeof(int32_t)));
         CK(h, cudaMemcpy(h->d_map, c.comp_map, (size_t)c.vocab * sizeof(int32_t),
                          cudaMemcpyHostToDevice));
         CK(h, cudaMalloc(&h->d_primes, S * sizeof(int64_t)));
         CK(h, cudaMemcpy(h->d_primes, h->primes, S * sizeof(int64_t), cudaMemcpyHostToDevice));
         uint64_t barrett[ENGRAM_MAX_TABLES];
         for (int i = 0; i < S; ++i) barrett[i] = ~0ull / (uint64_t)h->primes[i];
         CK(h, cudaMalloc(&h->d_barrett, S * sizeof(uint64_t)));
         CK(h, cudaMemcpy(h->d_barrett, barrett, S * sizeof(uint64_t), cudaMemcpyHostToDevice));
         CK(h, cudaMalloc(&h->d_mult, (size_t)S * h->max_order * sizeof(uint64_t)));
         CK(h, cudaMemcpy(h->d_mult, h->mult, (size_t)S * h->max_order * sizeof(uint64_t),
                          cudaMemcpyHostToDevice));
         CK(h, cudaMalloc(&h->d_err, sizeof(unsigned)));
         CK(h, cudaMemset(h->d_err, 0, sizeof(unsigned)));
         CK(h, cudaMalloc(&h->d_tables, (size_t)S * kMaxShards * sizeof(void*)));
         CK(h, cudaMalloc(&h->d_wqk, (size_t)c.branches * c.d_hidden * sizeof(float)));
         for (int i = 0; i < 2; ++i) {
           CK(h, cudaEventCreateWithFlags(&h->ev_ready[i], cudaEventDisableTiming));
           CK(h, cudaEventCreateWithFlags(&h->ev_consumed[i], cudaEventDisableTiming));
         }
         return ENGRAM_OK;
       }()) != ENGRAM_OK)
    return bail(rc);
  *out = h;
  return ENGRAM_OK;
}

void engram_destroy(engram_handle* h) {
  if (!h) return;
  int cur = 0;
  cudaGetDevice(&cur);
  cudaSetDevice(h->device);
  cudaDeviceSynchronize();
  free_host_gather(h);  // joins the prefetch threads
  cudaDeviceSynchronize();
  engram::free_host_io(h);
  if (h->copy_stream) cudaStreamDestroy(h->copy_stream);
  for (int i = 0; i < 2; ++i)
    if (h->ev_list[i]) cudaEventDestroy(h->ev_list[i]);
  free_dev(h->d_map);
  free_dev(h->d_primes);
  free_dev(h->d_barrett);
  free_dev(h->d_mult);
  free_dev(h->d_err);
  free_dev(h->d_tables);
  free_dev(h->d_wqk);
  free_dev(h->e);
  free_dev(h->e_alt);
  free_dev(h->partials);
  free_dev(h->alpha_scratch);
  free_dev(h->fused_sync);
  free_dev(h->fused_vt);
  free_dev(h->d_w8);
  free_dev(h->d_sw8);
  free_dev(h->bw_idx);
  free_dev(h->bw_kv);
  free_dev(h->bw_dkv);
  free_dev(h->bw_de);
  free_dev(h->bw_partials);
  free_dev(h->e8);
  free_dev(h->se8);
  free_dev(h->e8_alt);
  free_dev(h->se8_alt);
  free_dev(h->d_conv_w);
  free_dev(h->d_conv_nw);
  free_dev(h->d_conv_taps);
  free_dev(h->conv_v);
  free_dev(h->conv_vv);
  free_dev(h->conv_alpha);
  free_dev(h->conv_scale);
  free_dev(h->d_keys);
  free_dev(h->d_vals);
  free_dev(h->d_uniq);
  free_dev(h->d_stage_bound);
  free_dev(h->d_hot_keys);
  free_dev(h->d_hot_slots);
  free_dev(h->d_hot_rows);
  for (int i = 0; i < 2; ++i) {
    free_dev(h->d_count[i]);
    free_dev(h->d_remap[i]);
    free_dev(h->d_staging[i]);
    free_dev(h->d_stage_tables[i]);
    if (h->ev_ready[i]) cudaEventDestroy(h->ev_ready[i]);
    if (h->ev_consumed[i]) cudaEventDestroy(h->ev_consumed[i]);
  }
  cudaSetDevice(cur);
  delete h;
}

int engram_set_params(engram_handle* h, const void* const* tables, const void* w_k, const void* w_v,
                      const float* norm_q, const float* norm_k) {
  if (!h) return ENGRAM_ERR_INVALID;
  if (!tables || !w_k || !w_v || !norm_q || !norm_k)
    return fail(h, ENGRAM_ERR_INVALID, "null parameter pointer");
  for (int s = 0; s < h->S; ++s) {
    if (!tables[s] || !aligned16(tables[s]))
      return fail(h, ENGRAM_ERR_INVALID, "table pointers must be non-null and 16-byte aligned");
  }
  if (!aligned16(w_k) || !aligned16(w_v) || !aligned16(norm_q) || !aligned16(norm_k))
    return fail(h, ENGRAM_ERR_INVALID, "parameter pointers must be 16-byte aligned");
  if (h->cfg.table_location == ENGRAM_PINNED_HOST) {
    for (int s = 0; s < h->S; ++s) {
      cudaPointerAttributes at;
      if (cudaPointerGetAttributes(&at, tables[s]) != cudaSuccess || at.type != cudaMemoryTypeHost ||
          at.devicePointer == nullptr) {
        cudaGetLastError();
        return fail(h, ENGRAM_ERR_INVALID, "host tables must be pinned and mapped");
      }
    }
  }
  const int M = h->cfg.branches, d = h->cfg.d_hidden;
  const void* dev_tab[kMaxTables];
  for (int s = 0; s < h->S; ++s) {
    h->tables[s] = tables[s];
    dev_tab[s] = tables[s];
    if (h->cfg.table_location == ENGRAM_PINNED_HOST) {
      void* dp = nullptr;
      CK(h, cudaHostGetDevicePointer(&dp, const_cast<void*>(tables[s]), 0));
      dev_tab[s] = dp;
    }
  }
  CK(h, cudaMemcpy(h->d_tables, dev_tab, h->S * sizeof(void*), cudaMemcpyHostToDevice));
  h->shards = 1;
  CK(h, launch_mul(norm_q, norm_k, h->d_wqk, (int64_t)M * d, 0));
  CK(h, cudaDeviceSynchronize());
  h->w_k = w_k;
  h->w_v = w_v;
  h->norm_q = norm_q;
  h->norm_k = norm_k;
  if (h->cfg.dtype == ENGRAM_BF16) {
    for (int bn : {64, 128, 256}) {
      if (d % bn) continue;
      int rc = make_map(h, &h->map_wk[bn_index(bn)], w_k, h->d_mem, (int64_t)M * d, bn);
      if (rc) return rc;
      rc = make_map(h, &h->map_wv[bn_index(bn)], w_v, h->d_mem, d, bn);
      if (rc) return rc;
    }
  }
  h->have_params = true;
  if (h->fp8) return quantize_weights(h, 0);  // the new weights' E4M3 copy
  return ENGRAM_OK;
}

int engram_set_table_shards(engram_handle* h, int32_t shards, const void* const* ptrs) {
  if (!h) return ENGRAM_ERR_INVALID;
  if (!h->have_params) return fail(h, ENGRAM_ERR_STATE, "engram_set_params first");
  if (h->cfg.table_location != ENGRAM_DEVICE)
    return fail(h, ENGRAM_ERR_UNSUPPORTED, "row-sharded tables are device tables");
  if (shards < 1 || shards > kMaxShards)
    return fail(h, ENGRAM_ERR_INVALID, "shards must lie in [1, " + std::to_string(kMaxShards) + "]");
  if (!ptrs) return fail(h, ENGRAM_ERR_INVALID, "null shard array");
  for (int i = 0; i < h->S * shards; ++i) {
    if (!ptrs[i] || !aligned16(ptrs[i]))
      return fail(h, ENGRAM_ERR_INVALID, "shard pointers must be non-null and 16-byte aligned");
    cudaPointerAttributes at;
    if (cudaPointerGetAttributes(&at, ptrs[i]) != cudaSuccess || at.type != cudaMemoryTypeDevice) {
      cudaGetLastError();
      return fail(h, ENGRAM_ERR_INVALID, "shard pointers must be device memory (own or a peer's)");
    }
  }
  // the previous pointers may still be read by queued work
  CK(h, cudaDeviceSynchronize());
  CK(h, cudaMemcpy(h->d_tables, ptrs, (size_t)h->S * shards * sizeof(void*),
                   cudaMemcpyHostToDevice));
  h->shards = shards;
  return ENGRAM_OK;
}

int engram_ipc_handle(engram_handle* h, const void* ptr, void* handle) {
  if (!h) return ENGRAM_ERR_INVALID;
  if (!ptr || !handle) return fail(h, ENGRAM_ERR_INVALID, "null pointer");
  cudaIpcMemHandle_t mh;
  CK(h, cudaIpcGetMemHandle(&mh, const_cast<void*>(ptr)));
  static_assert(sizeof(mh) == ENGRAM_IPC_HANDLE_BYTES, "IPC handle size");
  std::memcpy(handle, &mh, sizeof(mh));
  return ENGRAM_OK;
}

int engram_ipc_open(engram_handle* h, const void* handle, void** ptr) {
  if (!h) return ENGRAM_ERR_INVALID;
  if (!handle || !ptr) return fail(h, ENGRAM_ERR_INVALID, "null pointer");
  cudaIpcMemHandle_t mh;
  std::memcpy(&mh, handle, sizeof(mh));
  CK(h, cudaSetDevice(h->device));
  CK(h, cudaIpcOpenMemHandle(ptr, mh, cudaIpcMemLazyEnablePeerAccess));
  return ENGRAM_OK;
}

int engram_ipc_close(engram_handle* h, void* ptr) {
  if (!h) return ENGRAM_ERR_INVALID;
  if (!ptr) return fail(h, ENGRAM_ERR_INVALID, "null pointer");
  CK(h, cudaIpcCloseMemHandle(ptr));
  return ENGRAM_OK;
}

int engram_set_fp8(engram_handle* h, int32_t enable, void* stream) {
  if (!h) return ENGRAM_ERR_INVALID;
  if (enable != 0 && enable != 1) return fail(h, ENGRAM_ERR_INVALID, "enable must be 0 or 1");
  if (!enable) {
    h->fp8 = false;
    return ENGRAM_OK;
  }
  if (!h->have_params) return fail(h, ENGRAM_ERR_STATE, "engram_set_params first");
  if (h->cfg.dtype != ENGRAM_BF16)
    return fail(h, ENGRAM_ERR_UNSUPPORTED, "FP8 projections need bf16 tables, weights and h");
  if (h->cfg.d_hidden % 256 || h->d_mem % 128 || h->d_mem > 2048)
    return fail(h, ENGRAM_ERR_UNSUPPORTED,
                "FP8 projections need d a multiple of 256 and d_mem a multiple of 128, <= 2048");
  if (h->cfg.flags & ENGRAM_FLAG_NO_CTA_PAIRS)
    return fail(h, ENGRAM_ERR_UNSUPPORTED, "FP8 projections run on CTA pairs only");
  int rc = quantize_weights(h, (cudaStream_t)stream);
  if (rc) return rc;
  h->fp8 = true;
  return ENGRAM_OK;
}

int engram_quantize_e4m3(engram_handle* h, const void* x, int64_t rows, int32_t cols, uint8_t* q,
                         float* scale, void* stream) {
  if (!h) return ENGRAM_ERR_INVALID;
  if (rows < 0 || rows > ((int64_t)1 << 31)) return fail(h, ENGRAM_ERR_INVALID, "rows out of range");
  if (cols < 16 || cols > 2048 || cols % 16)
    return fail(h, ENGRAM_ERR_INVALID, "cols must be a multiple of 16 in [16, 2048]");
  if (rows == 0) return ENGRAM_OK;
  if (!x || !q || !scale || !aligned16(x) || !aligned16(q) || ((uintptr_t)scale & 3u))
    return fail(h, ENGRAM_ERR_INVALID, "x and q must be 16-byte aligned, scale 4-byte aligned");
  CK(h, launch_quantize_e4m3(x, rows, cols, q, scale, (cudaStream_t)stream));
  h->launches += 1;
  return ENGRAM_OK;
}

int engram_set_short_conv(engram_handle* h, const float* conv_w, const float* norm_w,
                          int32_t kernel_size, int32_t dilation, void* stream) {
  if (!h) return ENGRAM_ERR_INVALID;
  if (!h->have_params) return fail(h, ENGRAM_ERR_STATE, "engram_set_params first");
  if (kernel_size == 0) {
    h->conv_W = 0;
    return ENGRAM_OK;
  }
  if (kernel_size < 1 || kernel_size > 4)
    return fail(h, ENGRAM_ERR_INVALID, "kernel_size must be 0 (off) or 1..4");
  if (dilation < 1 || dilation > 4) return fail(h, ENGRAM_ERR_INVALID, "dilation must be 1..4");
  if (!conv_w || !norm_w) return fail(h, ENGRAM_ERR_INVALID, "null conv_w or norm_w");
  const int d = h->cfg.d_hidden;
  cudaStream_t st = (cudaStream_t)stream;
  if (!h->d_conv_w) {
    CK(h, cudaMalloc(&h->d_conv_w, (size_t)d * 4 * sizeof(float)));
    CK(h, cudaMalloc(&h->d_conv_nw, (size_t)d * sizeof(float)));
    CK(h, cudaMalloc(&h->d_conv_taps, (size_t)d * 4 * sizeof(float)));
  }
  // [d][kernel_size] -> [d][4] with the unused taps zero
  CK(h, cudaMemsetAsync(h->d_conv_w, 0, (size_t)d * 4 * sizeof(float), st));
  CK(h, cudaMemcpy2DAsync(h->d_conv_w, 4 * sizeof(float), conv_w, kernel_size * sizeof(float),
                          kernel_size * sizeof(float), d, cudaMemcpyDeviceToDevice, st));
  CK(h, cudaMemcpyAsync(h->d_conv_nw, norm_w, (size_t)d * sizeof(float), cudaMemcpyDeviceToDevice,
                        st));
  CK(h, launch_conv_taps(h->d_conv_w, h->d_conv_nw, d, h->d_conv_taps, st));
  h->launches += 1;
  CK(h, cudaStreamSynchronize(st));
  h->conv_W = kernel_size;
  h->conv_dil = dilation;
  return ENGRAM_OK;
}

int engram_reserve(engram_handle* h, int64_t max_rows) {
  if (!h) return ENGRAM_ERR_INVALID;
  if (max_rows < 0 || max_rows > ((int64_t)1 << 31))
    return fail(h, ENGRAM_ERR_INVALID, "max_rows out of range");
  int rc = ensure_scratch(h, max_rows);
  if (rc) return rc;
  if (h->conv_W > 0 && (rc = ensure_conv_scratch(h, max_rows))) return rc;
  if (h->fp8 && (rc = ensure_fp8_scratch(h, max_rows))) return rc;
  if (h->cfg.table_location == ENGRAM_PINNED_HOST) return ensure_prefetch_scratch(h, max_rows);
  return ENGRAM_OK;
}

int engram_get_hash_params(const engram_handle* h, int64_t* primes, uint64_t* mult) {
  if (!h) return ENGRAM_ERR_INVALID;
  if (primes) std::memcpy(primes, h->primes, h->S * sizeof(int64_t));
  if (mult) std::memcpy(mult, h->mult, (size_t)h->S * h->max_order * sizeof(uint64_t));
  return ENGRAM_OK;
}

int engram_hash(engram_handle* h, const int32_t* tokens, int32_t B, int32_t T, int32_t t_begin,
                int64_t* idx, void* stream) {
  if (!h) return ENGRAM_ERR_INVALID;
  int rc = check_shape(h, B, T, t_begin);
  if (rc) return rc;
  if ((int64_t)B * T == 0) return ENGRAM_OK;
  if (!tokens || !idx) return fail(h, ENGRAM_ERR_INVALID, "null tokens or idx");
  CK(h, launch_hash(hash_args(h, tokens, B, T, t_begin, idx), (cudaStream_t)stream));
  h->launches += 1;
  return ENGRAM_OK;
}

int engram_gather(engram_handle* h, const int64_t* idx, int64_t rows, void* e, void* stream) {
  if (!h) return ENGRAM_ERR_INVALID;
  if (!h->have_params) return fail(h, ENGRAM_ERR_STATE, "engram_set_params first");
  if (h->cfg.table_location != ENGRAM_DEVICE)
    return fail(h, ENGRAM_ERR_UNSUPPORTED, "engram_gather reads device-resident tables only");
  if (rows < 0) return fail(h, ENGRAM_ERR_INVALID, "rows < 0");
  if (rows == 0) return ENGRAM_OK;
  if (rows * h->S * ((h->cfg.d_head * h->elt) >> 4) >= ((int64_t)1 << 31))
    return fail(h, ENGRAM_ERR_INVALID, "too many rows for one call");
  if (!idx || !e || !aligned16(e)) return fail(h, ENGRAM_ERR_INVALID, "null or misaligned buffer");
  GatherArgs g{};
  g.tables = h->d_tables;
  g.shards = h->shards;
  g.primes = h->d_primes;
  g.idx = idx;
  g.e = e;
  g.err = h->d_err;
  g.rows = rows;
  g.S = h->S;
  g.row_bytes = h->cfg.d_head * h->elt;
  CK(h, launch_gather(g, (cudaStream_t)stream));
  h->launches += 1;
  return ENGRAM_OK;
}

int engram_build_hot_cache(engram_handle* h, const int32_t* tokens, int32_t B, int32_t T,
                           int32_t t_begin, int64_t max_rows, void* stream) {
  if (!h) return ENGRAM_ERR_INVALID;
  if (h->cfg.table_location != ENGRAM_PINNED_HOST)
    return fail(h, ENGRAM_ERR_STATE, "the hot-row cache fronts ENGRAM_PINNED_HOST tables");
  if (!h->have_params) return fail(h, ENGRAM_ERR_STATE, "engram_set_params first");
  if (max_rows < 0) return fail(h, ENGRAM_ERR_INVALID, "max_rows < 0");
  int rc = check_shape(h, B, T, t_begin);
  if (rc) return rc;
  const int64_t rows = (int64_t)B * (T - t_begin);
  if (rows > 0 && !tokens) return fail(h, ENGRAM_ERR_INVALID, "null tokens");
  cudaStream_t st = (cudaStream_t)stream;
  // no prefetch may still read the old cache
  CK(h, cudaDeviceSynchronize());
  free_dev(h->d_hot_keys);
  free_dev(h->d_hot_slots);
  free_dev(h->d_hot_rows);
  h->n_hot = 0;
  h->hot_cap = 0;
  const int64_t entries = rows * h->S;
  if (max_rows == 0 || entries == 0) return ENGRAM_OK;
  uint64_t cap = 1;
  while (cap < (uint64_t)(2 * entries)) cap <<= 1;
  if (cap > (1ull << 31)) return fail(h, ENGRAM_ERR_INVALID, "calibration batch too large");
  // 1. indices of the calibration tokens, 2. how often each row is addressed
  int64_t* d_idx = nullptr;
  unsigned long long *d_keys = nullptr, *d_counts = nullptr, *d_list = nullptr;
  auto release = [&]() {
    free_dev(d_idx);
    free_dev(d_keys);
    free_dev(d_counts);
    free_dev(d_list);
  };
  auto body = [&]() -> int {
    CK(h, cudaMalloc(&d_idx, (size_t)entries * sizeof(int64_t)));
    CK(h, cudaMalloc(&d_keys, cap * sizeof(unsigned long long)));
    CK(h, cudaMalloc(&d_counts, cap * sizeof(unsigned long long)));
    CK(h, launch_hash(hash_args(h, tokens, B, T, t_begin, d_idx), st));
    CK(h, launch_count_rows(d_idx, entries, h->S, d_keys, d_counts, (uint32_t)cap, h->sms, st));
    h->launches += 3;
    std::vector<unsigned long long> keys(cap), counts(cap);
    CK(h, cudaMemcpyAsync(keys.data(), d_keys, cap * sizeof(unsigned long long),
                          cudaMemcpyDeviceToHost, st));
    CK(h, cudaMemcpyAsync(counts.data(), d_counts, cap * sizeof(unsigned long long),
                          cudaMemcpyDeviceToHost, st));
    CK(h, cudaStreamSynchronize(st));
    // 3. the max_rows most frequent rows; ties go to the lower (table, row)
    std::vector<std::pair<unsigned long long, unsigned long long>> seen;  // (count, key)
    for (uint64_t i = 0; i < cap; ++i)
      if (keys[i] != ~0ull) seen.emplace_back(counts[i], keys[i]);
    const int64_t n = std::min<int64_t>(max_rows, (int64_t)seen.size());
    auto more_frequent = [](const std::pair<unsigned long long, unsigned long long>& x,
                            const std::pair<unsigned long long, unsigned long long>& y) {
      return x.first != y.first ? x.first > y.first : x.second < y.second;
    };
    std::partial_sort(seen.begin(), seen.begin() + n, seen.end(), more_frequent);
    std::vector<unsigned long long> list((size_t)n);
    for (int64_t i = 0; i < n; ++i) list[i] = seen[i].second;
    // 4. the cache: a lookup table (slot = rank) and the rows, copied once
    uint64_t hcap = 1;
    while (hcap < (uint64_t)(2 * n)) hcap <<= 1;
    const size_t row_bytes = (size_t)h->cfg.d_head * h->elt;
    CK(h, cudaMalloc(&d_list, (size_t)n * sizeof(unsigned long long)));
    CK(h, cudaMemcpyAsync(d_list, list.data(), (size_t)n * sizeof(unsigned long long),
                          cudaMemcpyHostToDevice, st));
    CK(h, cudaMalloc(&h->d_hot_keys, hcap * sizeof(unsigned long long)));
    CK(h, cudaMalloc(&h->d_hot_slots, hcap * sizeof(int32_t)));
    CK(h, cudaMalloc(&h->d_hot_rows, (size_t)n * row_bytes));
    CK(h, launch_fill_hot_cache(d_list, n, h->d_hot_keys, h->d_hot_slots, (uint32_t)hcap,
                                (const void* const*)h->d_tables, (int32_t)row_bytes,
                                h->d_hot_rows, h->sms, st));
    h->launches += 3;
    CK(h, cudaStreamSynchronize(st));
    h->n_hot = n;
    h->hot_cap = (uint32_t)hcap;
    return ENGRAM_OK;
  };
  rc = body();
  release();
  if (rc != ENGRAM_OK) {
    free_dev(h->d_hot_keys);
    free_dev(h->d_hot_slots);
    free_dev(h->d_hot_rows);
    h->n_hot = 0;
    h->hot_cap = 0;
  }
  return rc;
}

int engram_prefetch_hot_hits(engram_handle* h, int64_t* hits) {
  if (!h || !hits) return ENGRAM_ERR_INVALID;
  *hits = 0;
  if (h->n_prefetch == 0 || !h->d_count[(h->n_prefetch - 1) & 1]) return ENGRAM_OK;
  CK(h, cudaDeviceSynchronize());
  unsigned long long v[2] = {0, 0};
  CK(h, cudaMemcpy(v, h->d_count[(h->n_prefetch - 1) & 1], sizeof(v), cudaMemcpyDeviceToHost));
  *hits = (int64_t)v[1];
  return ENGRAM_OK;
}

int engram_set_prefetch(engram_handle* h, int32_t mode, int32_t workers) {
  if (!h) return ENGRAM_ERR_INVALID;
  if (h->cfg.table_location != ENGRAM_PINNED_HOST)
    return fail(h, ENGRAM_ERR_STATE, "engram_set_prefetch needs ENGRAM_PINNED_HOST tables");
  if (mode != ENGRAM_PREFETCH_HOST_THREADS && mode != ENGRAM_PREFETCH_ZERO_COPY)
    return fail(h, ENGRAM_ERR_INVALID, "unknown prefetch mode");
  if (workers < 0 || workers > 4096) return fail(h, ENGRAM_ERR_INVALID, "workers outside [0, 4096]");
  if (h->n_prefetch != h->n_consumed)
    return fail(h, ENGRAM_ERR_STATE, "a prefetch is pending; run engram_forward first");
  // threads of the old setting finish and leave; the next prefetch starts new ones
  delete h->hg;
  h->hg = nullptr;
  h->pf_mode = mode;
  h->pf_workers = workers;
  return ENGRAM_OK;
}

int engram_prefetch_wait(engram_handle* h) {
  if (!h) return ENGRAM_ERR_INVALID;
  if (h->n_prefetch == h->n_consumed) return fail(h, ENGRAM_ERR_STATE, "no prefetch is pending");
  const int slot = (int)(h->n_consumed & 1);
  if (h->hg) {
    std::string msg;
    const cudaError_t ge = h->hg->wait_issued(slot, &msg);
    if (ge != cudaSuccess) return fail(h, ENGRAM_ERR_CUDA, "prefetch: " + msg);
  }
  CK(h, cudaEventSynchronize(h->ev_ready[slot]));
  return ENGRAM_OK;
}

int engram_prefetch(engram_handle* h, const int32_t* tokens, int32_t B, int32_t T, int32_t t_begin,
                    void* side_stream, int64_t* unique_rows) {
  if (!h) return ENGRAM_ERR_INVALID;
  if (h->cfg.table_location != ENGRAM_PINNED_HOST)
    return fail(h, ENGRAM_ERR_STATE, "engram_prefetch needs ENGRAM_PINNED_HOST tables");
  if (!h->have_params) return fail(h, ENGRAM_ERR_STATE, "engram_set_params first");
  int rc = check_shape(h, B, T, t_begin);
  if (rc) return rc;
  if (h->n_prefetch - h->n_consumed >= 2)
    return fail(h, ENGRAM_ERR_STATE, "two prefetches already pending; run engram_forward first");
  const int64_t rows = (int64_t)B * (T - t_begin);
  if (rows > 0 && !tokens) return fail(h, ENGRAM_ERR_INVALID, "null tokens");
  if ((rc = ensure_prefetch_scratch(h, rows))) return rc;
  cudaStream_t st = (cudaStream_t)side_stream;
  const int slot = (int)(h->n_prefetch & 1);
  const bool host_threads = h->pf_mode == ENGRAM_PREFETCH_HOST_THREADS;
  // the staging slot must no longer be read by the forward that used it last
  if (h->n_prefetch >= 2) CK(h, cudaStreamWaitEvent(st, h->ev_consumed[slot], 0));
  if (rows > 0) {
    // hash into this slot's index buffer; the prefetch then rewrites each
    // index in place with its staging slot
    CK(h, launch_hash(hash_args(h, tokens, B, T, t_begin, h->d_remap[slot]), st));
    h->launches += 1;
  }
  PrefetchArgs a{};
  a.idx = h->d_remap[slot];
  a.rows = rows;
  a.S = h->S;
  a.keys = h->d_keys;
  a.vals = h->d_vals;
  a.cap = h->set_cap;
  a.count = h->d_count[slot];
  a.uniq = h->d_uniq;
  a.remapped = h->d_remap[slot];
  a.tables = h->d_tables;
  a.row_bytes = h->cfg.d_head * h->elt;
  a.staging = h->d_staging[slot];
  a.sms = h->sms;
  a.fetch_blocks = h->pf_workers > 0 ? h->pf_workers : h->sms;
  if (h->n_hot > 0) {
    a.hot_keys = h->d_hot_keys;
    a.hot_slots = h->d_hot_slots;
    a.hot_cap = h->hot_cap;
    a.hot_rows = h->d_hot_rows;
  }
  CK(h, launch_prefetch_index(a, st));
  h->launches += rows > 0 ? (h->n_hot > 0 ? 5 : 4) : 1;
  if (host_threads) {
    // the row list goes to the host; reader threads gather the rows and the
    // copy engines send them (ev_ready is recorded after the last copy)
    const int64_t entries = rows * h->S;
    CK(h, cudaMemcpyAsync(h->h_count[slot], h->d_count[slot], 2 * sizeof(unsigned long long),
                          cudaMemcpyDeviceToHost, st));
    if (entries > 0)
      CK(h, cudaMemcpyAsync(h->h_list[slot], h->d_uniq, (size_t)entries * sizeof(int2),
                            cudaMemcpyDeviceToHost, st));
    CK(h, cudaEventRecord(h->ev_list[slot], st));
    HostGatherJob job;
    job.slot = slot;
    job.idx_ready = h->ev_list[slot];
    job.count = h->h_count[slot];
    job.list = h->h_list[slot];
    job.tables = h->tables;
    job.row_bytes = a.row_bytes;
    job.bounce = h->h_bounce[slot];
    job.staging = (char*)h->d_staging[slot];
    job.copy_stream = h->copy_stream;
    job.done = h->ev_ready[slot];
    h->hg->submit(job);
  } else {
    CK(h, launch_prefetch_fetch(a, st));
    h->launches += rows > 0 ? 1 : 0;
    CK(h, cudaEventRecord(h->ev_ready[slot], st));
  }
  h->pf_rows[slot] = rows;
  ++h->n_prefetch;
  if (unique_rows) {
    unsigned long long n[2] = {0, 0};
    CK(h, cudaMemcpyAsync(n, h->d_count[slot], sizeof(n), cudaMemcpyDeviceToHost, st));
    CK(h, cudaStreamSynchronize(st));
    *unique_rows = rows > 0 ? (int64_t)(n[0] + n[1]) : 0;
  }
  return ENGRAM_OK;
}

namespace {

// Whether a bf16 call of R rows takes the one-launch short-call kernel: at
// most 256 rows, d a multiple of 256, at most four branches, CTA pairs
// allowed, and all nkey + nval clusters resident at once.
bool use_fused(engram_handle* h, int64_t R, int* nkey, int* nval) {
  const int M = h->cfg.branches, d = h->cfg.d_hidden;
  if (h->cfg.dtype != ENGRAM_BF16 || R > 256 || M > engram::kMaxBranches || d % 256 != 0)
    return false;
  if (h->cfg.flags & (ENGRAM_FLAG_NO_CTA_PAIRS | ENGRAM_FLAG_NO_FUSED_SHORT)) return false;
  if (!h->fused_sync) return false;
  if (h->fused_clusters < 0) h->fused_clusters = engram::fused_max_clusters();
  *nkey = M * d / 256;
  *nval = d / 128;
  return *nkey + *nval <= h->fused_clusters;
}

}  // namespace

int engram_forward(engram_handle* h, const int32_t* tokens, const int64_t* idx, int32_t B,
                   int32_t T, int32_t t_begin, const void* hid, void* out, float* alpha,
                   float* delta, void* stream) {
  if (!h) return ENGRAM_ERR_INVALID;
  if (!h->have_params) return fail(h, ENGRAM_ERR_STATE, "engram_set_params first");
  int rc = check_shape(h, B, T, t_begin);
  if (rc) return rc;
  cudaStream_t st = (cudaStream_t)stream;
  const int64_t R = (int64_t)B * (T - t_begin);
  const bool host_tables = h->cfg.table_location == ENGRAM_PINNED_HOST;
  int slot = 0;
  if (host_tables) {
    if (h->n_prefetch == h->n_consumed)
      return fail(h, ENGRAM_ERR_STATE, "host-resident tables: call engram_prefetch first");
    slot = (int)(h->n_consumed & 1);
    if (h->pf_rows[slot] != R)
      return fail(h, ENGRAM_ERR_INVALID, "forward shape differs from the pending prefetch");
  }
  if (host_tables && h->hg) {
    // the host-thread route: its copies and ev_ready[slot] are enqueued by
    // the reader threads; wait until they are
    std::string msg;
    const cudaError_t ge = h->hg->wait_issued(slot, &msg);
    if (ge != cudaSuccess)
      return fail(h, ge == cudaErrorMemoryAllocation ? ENGRAM_ERR_OOM : ENGRAM_ERR_CUDA,
                  "prefetch: " + msg);
  }
  if (R == 0) {
    if (host_tables) {
      CK(h, cudaStreamWaitEvent(st, h->ev_ready[slot], 0));
      CK(h, cudaEventRecord(h->ev_consumed[slot], st));
      ++h->n_consumed;
    }
    return ENGRAM_OK;
  }
  if (!hid || !out || !aligned16(hid) || !aligned16(out))
    return fail(h, ENGRAM_ERR_INVALID, "h and out must be non-null and 16-byte aligned");
  if ((alpha && !aligned16(alpha)) || (delta && !aligned16(delta)))
    return fail(h, ENGRAM_ERR_INVALID, "alpha and delta must be 16-byte aligned");
  if (!idx && !tokens && !host_tables) return fail(h, ENGRAM_ERR_INVALID, "need tokens or idx");
  if (R > (int64_t)65535 * 64 && h->cfg.dtype == ENGRAM_F32)
    return fail(h, ENGRAM_ERR_INVALID, "fp32 path limited to 4194240 rows per call");
  if ((rc = ensure_scratch(h, R))) return rc;
  const bool fp8 = h->fp8;  // E4M3 operands for the projections (bf16 handles only)
  if (fp8 && (rc = ensure_fp8_scratch(h, R))) return rc;
  // this call's e buffers (alternating between calls)
  const bool flip = h->e_flip != 0;
  h->e_flip ^= 1;
  void* const E = flip ? h->e_alt : h->e;
  uint8_t* const E8 = flip ? h->e8_alt : h->e8;
  float* const SE8 = flip ? h->se8_alt : h->se8;
  const bool prof = h->prof_armed;
  h->prof_armed = false;
  auto mark = [&](int i) -> cudaError_t {
    return prof && i < h->n_prof ? cudaEventRecord(h->prof[i], st) : cudaSuccess;
  };
  // with the short convolution on: the value phase leaves v, its sums of
  // squares and alpha, and one more kernel forms out = h + Y (Eq. 5)
  const bool conv = h->conv_W > 0;
  if (conv && t_begin != 0)
    return fail(h, ENGRAM_ERR_UNSUPPORTED,
                "the short convolution needs every position of each sequence (t_begin = 0)");
  if (conv && R * (h->cfg.d_hidden / 4) >= ((int64_t)1 << 31))
    return fail(h, ENGRAM_ERR_INVALID, "too many rows for the short convolution in one call");
  if (conv && (rc = ensure_conv_scratch(h, R))) return rc;
  CK(h, mark(0));

  // steps 1-4: indices, then the gathered memory vectors e
  GatherArgs ga{};
  ga.e = E;
  ga.err = h->d_err;
  ga.rows = R;
  ga.S = h->S;
  ga.row_bytes = h->cfg.d_head * h->elt;
  if (host_tables) {
    CK(h, cudaStreamWaitEvent(st, h->ev_ready[slot], 0));
    ga.tables = h->d_stage_tables[slot];
    ga.shards = 1;
    ga.primes = h->d_stage_bound;
    ga.idx = h->d_remap[slot];
  } else {
    ga.tables = h->d_tables;
    ga.shards = h->shards;
    ga.primes = h->d_primes;
    ga.idx = idx;
  }
  if (!host_tables && !idx) {
    // indices computed and consumed on chip: one kernel for steps 1-4 (the
    // hash stage of a profiled forward is then empty)
    HashGatherArgs hg{};
    hg.hash = hash_args(h, tokens, B, T, t_begin, nullptr);
    hg.tables = h->d_tables;
    hg.shards = h->shards;
    hg.e = E;
    hg.q = E8;
    hg.scale = SE8;
    hg.row_bytes = ga.row_bytes;
    hg.pdl = 1;  // overlaps the previous call's value launch (other e buffer)
    CK(h, mark(1));
    // FP8: e leaves the gather as E4M3 codes and row scales
    CK(h, fp8 ? launch_hash_gather_e4m3(hg, st) : launch_hash_gather(hg, st));
  } else {
    CK(h, mark(1));
    CK(h, launch_gather(ga, st));
    if (fp8) {
      CK(h, launch_quantize_e4m3(E, R, h->d_mem, E8, SE8, st));
      h->launches += 1;
    }
  }
  h->launches += 1;
  CK(h, mark(2));
  if (host_tables) {
    CK(h, cudaEventRecord(h->ev_consumed[slot], st));
    ++h->n_consumed;
  }

  // steps 5-7: projections, gate, residual
  GateArgs g{};
  g.h = hid;
  g.out = out;
  g.w_qk = h->d_wqk;
  g.partials = h->partials;
  g.alpha = alpha;
  g.delta = delta;
  g.err = h->d_err;
  g.R = (int32_t)R;
  g.M = h->cfg.branches;
  g.d = h->cfg.d_hidden;
  g.d_mem = h->d_mem;
  g.eps = h->cfg.eps;
  g.inv_sqrt_d = (float)(1.0 / std::sqrt((double)h->cfg.d_hidden));
  // the key launch overlaps the gather's tail and the value launch the key's
  g.pdl = 1;
  if (conv) {
    g.vals = h->conv_v;
    g.vv = h->conv_vv;
    if (!g.alpha) g.alpha = h->conv_alpha;
  }
  // step 7 with the short convolution (Eq. 5), after the value phase left v,
  // its sums of squares per value tile and alpha
  auto short_conv = [&](int value_tile) -> int {
    ConvArgs ca{};
    ca.vals = h->conv_v;
    ca.vv = h->conv_vv;
    ca.alpha = g.alpha;
    ca.h = hid;
    ca.out = out;
    ca.delta = delta;
    ca.taps = h->d_conv_taps;
    ca.B = B;
    ca.T = T;
    ca.M = g.M;
    ca.d = g.d;
    ca.n_vtiles = g.d / value_tile;
    ca.bf16 = h->cfg.dtype == ENGRAM_BF16;
    ca.eps = g.eps;
    CK(h, launch_short_conv(ca, h->conv_dil, h->conv_scale, st));
    h->launches += 2;
    CK(h, mark(5));
    return ENGRAM_OK;
  };
  if (h->cfg.dtype == ENGRAM_F32) {
    g.key_tile = kF32Tile;
    CK(h, launch_proj_gate_f32(0, (const float*)E, (const float*)h->w_k, g, st));
    CK(h, mark(3));
    CK(h, launch_proj_gate_f32(conv ? 3 : 1, (const float*)E, (const float*)h->w_v, g, st));
    CK(h, mark(4));
    h->launches += 2;
    if (conv) return short_conv(kF32Tile);
    CK(h, mark(5));
    return ENGRAM_OK;
  }
  const int64_t hcols = (int64_t)g.M * g.d;
  int nkey = 0, nval = 0;
  if (!conv && !fp8 && use_fused(h, R, &nkey, &nval)) {
    // Short calls: keys, alpha and values in one launch, the value CTAs
    // taking alpha from the key CTAs' partial sums through counters
    FusedMaps fm;
    if ((rc = cached_map(h, &fm.e, E, h->d_mem, R, 128))) return rc;
    if ((rc = cached_map(h, &fm.h, hid, hcols, R, 128, 32))) return rc;
    if ((rc = cached_map(h, &fm.out, out, hcols, R, 32, 32))) return rc;  // per-warp boxes
    fm.wk = h->map_wk[bn_index(128)];  // each CTA of a key pair: 128 of the tile's 256 W rows
    fm.wv = h->map_wv[bn_index(64)];   // each CTA of a value pair: 64 of 128
    g.key_tile = 128;
    g.sync = h->fused_sync;
    g.vt = h->fused_vt;
    CK(h, launch_proj_gate_fused(fm, g, nkey, nval, st));
    h->launches += 1;
    CK(h, mark(3));
    CK(h, mark(4));
    CK(h, mark(5));
    return ENGRAM_OK;
  }
  // Tensor maps are built for whichever kernel each phase uses (choose_proj):
  // 512 x 256 tiles on CTA pairs when the tile count fills every pair at least
  // once, else 256 x 256 pair tiles or single-CTA 128-row tiles by cost.
  ProjMaps single, wide, pair;
  bool have_single = false, have_wide = false, have_pair = false;
  int value_tile = 0;
  if (fp8) g.s_row = SE8;
  int key_grid = 0;
  for (int phase = 0; phase < 2; ++phase) {
    const CUtensorMap* wmaps = phase == 0 ? h->map_wk : h->map_wv;
    // the E4M3 operands run on the 512 x 256 CTA-pair kernel only
    ProjChoice pc = fp8 ? wide_proj(phase, R, g.M, g.d, h->sms)
                        : choose_proj(phase, R, g.M, g.d, h->sms, h->cfg.flags, conv);
    if (phase == 0) key_grid = pc.grid;
    if (phase == 1 && pc.kind != ProjKernel::Wide && key_grid < h->sms) {
      // Short calls: the value CTAs stream their operands beside the key
      // launch, on the SMs that it and the row alpha kernel (whose blocks,
      // launched before, wait on SMs too) leave free.  A value CTA beyond
      // those would start only when a key CTA leaves and end the step late,
      // so the launch takes at most the free SMs, each then taking up to two
      // tiles (both mainloops run before alpha is ready).
      const int alpha_blocks = conv ? 0 : (int)((R * g.M + 127) / 128);
      const int free_sms = h->sms - key_grid - alpha_blocks;
      const int64_t n_total = g.d;
      const int64_t tiles = pc.kind == ProjKernel::Pair ? (R + 255) / 256 * (n_total / 256)
                                                        : (R + 127) / 128 * (n_total / pc.bn);
      const int unit = pc.kind == ProjKernel::Pair ? 2 : 1;  // CTAs per tile
      const int cap = free_sms / unit * unit;
      if (cap >= unit && pc.grid > cap && tiles * unit <= 2 * (int64_t)cap) pc.grid = cap;
    }
    if (fp8) g.s_col = h->d_sw8 + (phase == 0 ? 0 : (int64_t)g.M * g.d);
    if (phase == 0) g.key_tile = pc.key_tile;
    if (phase == 1) value_tile = pc.key_tile;
    if (phase == 1 && !conv && pc.kind != ProjKernel::Wide) {
      // short calls: alpha is formed once per row between the launches, so
      // that the value CTAs (many per row block) do not each sum the same
      // partials after the key launch completes
      float* adst = alpha ? alpha : h->alpha_scratch;
      CK(h, launch_row_alpha(g, adst, st));
      h->launches += 1;
      g.alpha_in = adst;
    }
    // values: 3 = v for the short convolution; 2 = in place (out aliases h,
    // alpha v is added into out); 1 = out = h + alpha v
    const int kphase = phase == 0 ? 0 : conv ? 3 : out == hid ? 2 : 1;
    if (pc.kind == ProjKernel::Pair) {
      if (!have_pair) {
        if ((rc = cached_map(h, &pair.e, E, h->d_mem, R, 128))) return rc;
        if ((rc = cached_map(h, &pair.h, hid, hcols, R, 128, 32))) return rc;
        if ((rc = cached_map(h, &pair.out, out, hcols, R, 32, 32))) return rc;  // per-warp boxes
        have_pair = true;
      }
      pair.w = wmaps[bn_index(pc.bn)];  // each CTA of a pair loads 128 of the tile's 256 W rows
      ProjMaps pm = pair;
      // in place: per-warp reduce-adds of 32 rows x 64 columns
      if (kphase == 2 && (rc = cached_map(h, &pm.out, out, hcols, R, 32, 64))) return rc;
      CK(h, launch_proj_gate_pair(kphase, pm, g, pc.grid, st));
    } else if (pc.kind == ProjKernel::Wide) {
      if (!have_wide) {
        if (fp8) {
          if ((rc = cached_map(h, &wide.e, E8, h->d_mem, R, 256, 128, 1))) return rc;
        } else if ((rc = cached_map(h, &wide.e, E, h->d_mem, R, 256))) {
          return rc;
        }
        if ((rc = cached_map(h, &wide.h, hid, hcols, R, 256, 32))) return rc;
        if ((rc = cached_map(h, &wide.out, out, hcols, R, 32, 32))) return rc;
        have_wide = true;
      }
      wide.w = fp8 ? (phase == 0 ? h->map_wk8 : h->map_wv8) : wmaps[bn_index(pc.bn)];
      if (kphase == 2) {
        // in place: per-warp reduce-adds of 32 rows x 64 columns
        ProjMaps wr = wide;
        if ((rc = cached_map(h, &wr.out, out, hcols, R, 32, 64))) return rc;
        CK(h, launch_proj_gate_wide(kphase, wr, g, pc.grid, st, fp8));
      } else if (kphase == 3) {
        // v leaves through per-warp TMA stores of 32 x 32 fp32 boxes
        ProjMaps wv = wide;
        if ((rc = cached_map(h, &wv.out, h->conv_v, g.d, R, 32, 32, 4))) return rc;
        CK(h, launch_proj_gate_wide(kphase, wv, g, pc.grid, st, fp8));
      } else {
        CK(h, launch_proj_gate_wide(kphase, wide, g, pc.grid, st, fp8));
      }
    } else {
      if (!have_single) {
        if ((rc = cached_map(h, &single.e, E, h->d_mem, R, 128))) return rc;
        if ((rc = cached_map(h, &single.h, hid, hcols, R, 128))) return rc;
        // the value epilogue stores per warp: 32-row boxes
        if ((rc = cached_map(h, &single.out, out, hcols, R, 32))) return rc;
        have_single = true;
      }
      single.w = wmaps[bn_index(pc.bn)];
      CK(h, launch_proj_gate_sm100(kphase == 3 ? 3 : phase, pc.bn, single, g, pc.grid, st));
    }
    CK(h, mark(3 + phase));
  }
  h->launches += 2;
  if (conv) return short_conv(value_tile);
  CK(h, mark(5));
  return ENGRAM_OK;
}

namespace {

int ensure_bw_scratch(engram_handle* h, int64_t rows, int grid) {
  const int64_t M = h->cfg.branches, d = h->cfg.d_hidden;
  if (rows > h->bw_cap_rows) {
    free_dev(h->bw_idx);
    free_dev(h->bw_kv);
    free_dev(h->bw_dkv);
    free_dev(h->bw_de);
    h->bw_cap_rows = 0;
    CK(h, cudaMalloc(&h->bw_idx, (size_t)rows * h->S * sizeof(int64_t)));
    CK(h, cudaMalloc(&h->bw_kv, (size_t)rows * (M + 1) * d * sizeof(float)));
    CK(h, cudaMalloc(&h->bw_dkv, (size_t)rows * (M + 1) * d * h->elt));
    CK(h, cudaMalloc(&h->bw_de, (size_t)rows * h->d_mem * sizeof(float)));
    h->bw_cap_rows = rows;
  }
  if (grid > h->bw_part_blocks) {
    free_dev(h->bw_partials);
    h->bw_part_blocks = 0;
    CK(h, cudaMalloc(&h->bw_partials, (size_t)grid * 2 * M * d * sizeof(float)));
    h->bw_part_blocks = grid;
  }
  return ENGRAM_OK;
}

// K splits of a reduce-add contraction: the count that fills the most of
// `rounds` rounds of CTA pairs (1-8 rounds), at least 8 K blocks per split.
void choose_splits(GemmArgs& g, int pairs) {
  const int kb_total = (g.K + 63) / 64;
  const int mn = gemm_pair_tiles(GemmArgs{g.M, g.N, g.K, 0, 0, 1, 1, 0, nullptr});
  int best = 1;
  double best_util = (double)mn / (((mn + pairs - 1) / pairs) * (double)pairs);
  for (int rounds = 1; rounds <= 8; ++rounds) {
    const int sp = std::min(std::max(1, rounds * pairs / mn), std::max(1, kb_total / 8));
    const int tiles = mn * sp;
    const double util = (double)tiles / (((tiles + pairs - 1) / pairs) * (double)pairs);
    if (util > best_util + 1e-9) {
      best_util = util;
      best = sp;
    }
  }
  g.kb_per_split = (kb_total + best - 1) / best;
  g.splits = (kb_total + g.kb_per_split - 1) / g.kb_per_split;
}

// D (=|+=) A B^T on the tensor cores; see GemmArgs.  a_mn / b_mn: the
// operand is stored MN-major ([K, rows]).
int gemm_bf16(engram_handle* h, bool a_mn, bool b_mn, bool add, const void* A, int64_t a_rows,
              int64_t a_cols, const void* B0, int64_t b0_rows, const void* B1, int64_t b1_rows,
              int64_t b_cols, float* D, int64_t d_rows, int64_t d_cols, GemmArgs g,
              cudaStream_t st) {
  GemmMaps mp;
  int rc;
  if ((rc = make_map(h, &mp.a, A, a_cols, a_rows, a_mn ? 64 : 128, 64))) return rc;
  if ((rc = make_map(h, &mp.b0, B0, b_cols, b0_rows, b_mn ? 64 : 128, 64))) return rc;
  if ((rc = make_map(h, &mp.b1, B1 ? B1 : B0, b_cols, B1 ? b1_rows : b0_rows, b_mn ? 64 : 128,
                     64)))
    return rc;
  if ((rc = make_map(h, &mp.d, D, d_cols, d_rows, 32, 32, 4))) return rc;
  g.err = h->d_err;
  const int pairs = h->sms / 2;
  if (add) {
    choose_splits(g, pairs);
  } else {
    g.splits = 1;
    g.kb_per_split = (g.K + 63) / 64;
  }
  const int tiles = gemm_pair_tiles(g);
  CK(h, launch_gemm_pair(a_mn, b_mn, add, mp, g, 2 * std::min(tiles, pairs), st));
  h->launches += 1;
  return ENGRAM_OK;
}

int gemm_f32(engram_handle* h, const float* A, int64_t a_m, int64_t a_k, const float* B,
             int64_t b_n, int64_t b_k, float* D, int64_t ldd, int M, int N, int K, bool add,
             cudaStream_t st) {
  GemmF32Args g{A, a_m, a_k, B, b_n, b_k, D, ldd, M, N, K, add};
  CK(h, launch_gemm_f32(g, st));
  h->launches += 1;
  return ENGRAM_OK;
}

}  // namespace

int engram_backward(engram_handle* h, const int32_t* tokens, const int64_t* idx, int32_t B,
                    int32_t T, int32_t t_begin, const void* hid, const void* dout, void* dhid,
                    float* dw_k, float* dw_v, float* dnorm_q, float* dnorm_k,
                    float* const* dtables, void* stream) {
  if (!h) return ENGRAM_ERR_INVALID;
  if (!h->have_params) return fail(h, ENGRAM_ERR_STATE, "engram_set_params first");
  int rc = check_shape(h, B, T, t_begin);
  if (rc) return rc;
  if (h->cfg.table_location == ENGRAM_PINNED_HOST)
    return fail(h, ENGRAM_ERR_UNSUPPORTED, "engram_backward: device-resident tables only");
  if (h->fp8 || h->conv_W > 0)
    return fail(h, ENGRAM_ERR_UNSUPPORTED,
                "engram_backward: the FP8 projections and the short convolution have no backward");
  const int M = h->cfg.branches, d = h->cfg.d_hidden, dm = h->d_mem, S = h->S;
  if (d > 4096 || gate_bw_smem(M, d) > 232448)
    return fail(h, ENGRAM_ERR_UNSUPPORTED, "engram_backward: d must be <= 4096");
  const int64_t R = (int64_t)B * (T - t_begin);
  if (R == 0) return ENGRAM_OK;
  if (R > INT32_MAX / std::max(M + 1, 1) / std::max(d, 1) || R * dm > INT32_MAX)
    return fail(h, ENGRAM_ERR_INVALID, "engram_backward: too many rows for one call");
  if (!hid || !dout || !dhid || !aligned16(hid) || !aligned16(dout) || !aligned16(dhid))
    return fail(h, ENGRAM_ERR_INVALID, "h, dout and dh must be non-null and 16-byte aligned");
  if (!idx && !tokens) return fail(h, ENGRAM_ERR_INVALID, "need tokens or idx");
  if (dtables)
    for (int s = 0; s < S * h->shards; ++s)
      if (!dtables[s] || !aligned16(dtables[s]))
        return fail(h, ENGRAM_ERR_INVALID, "table-gradient pointers must be non-null and 16-byte aligned");
  cudaStream_t st = (cudaStream_t)stream;
  const int grid = gate_bw_grid(M, d, R, h->elt);
  if ((rc = ensure_scratch(h, R))) return rc;
  if ((rc = ensure_bw_scratch(h, R, grid))) return rc;
  const bool prof = h->bprof_armed;
  h->bprof_armed = false;
  auto mark = [&](int i) -> cudaError_t {
    return prof ? cudaEventRecord(h->bprof[i], st) : cudaSuccess;
  };
  CK(h, mark(0));

  // steps 1-4 again: indices (kept for the table gradients) and e
  const int64_t* z = idx;
  if (!idx) {
    CK(h, launch_hash(hash_args(h, tokens, B, T, t_begin, h->bw_idx), st));
    h->launches += 1;
    z = h->bw_idx;
  }
  GatherArgs ga{};
  ga.tables = h->d_tables;
  ga.shards = h->shards;
  ga.primes = h->d_primes;
  ga.idx = z;
  ga.e = h->e;
  ga.err = h->d_err;
  ga.rows = R;
  ga.S = S;
  ga.row_bytes = h->cfg.d_head * h->elt;
  CK(h, launch_gather(ga, st));
  h->launches += 1;
  CK(h, mark(1));

  // k and v recomputed (Eq. 3): kv [R, (M+1) d] = e [W_K; W_V]^T
  const int nkv = (M + 1) * d;
  const bool bf16 = h->cfg.dtype == ENGRAM_BF16;
  const int Md = M * d;
  const void* dkv = h->bw_dkv;  // [R, (M + 1) d] in the handle's dtype
  if (bf16) {
    GemmArgs g{};
    g.M = (int)R;
    g.K = dm;
    g.kb_split = 1 << 30;
    g.N = Md;
    if ((rc = gemm_bf16(h, false, false, false, h->e, R, dm, h->w_k, Md, nullptr, 0, dm, h->bw_kv,
                        R, nkv, g, st)))
      return rc;
    g.N = d;
    g.d_col0 = Md;
    if ((rc = gemm_bf16(h, false, false, false, h->e, R, dm, h->w_v, d, nullptr, 0, dm, h->bw_kv,
                        R, nkv, g, st)))
      return rc;
  } else {
    const float* e32 = (const float*)h->e;
    if ((rc = gemm_f32(h, e32, dm, 1, (const float*)h->w_k, dm, 1, h->bw_kv, nkv, (int)R, Md, dm,
                       false, st)) ||
        (rc = gemm_f32(h, e32, dm, 1, (const float*)h->w_v, dm, 1, h->bw_kv + Md, nkv, (int)R, d,
                       dm, false, st)))
      return rc;
  }
  CK(h, mark(2));

  // gate and residual backward: dh, dk, dv, RMSNorm weight gradients
  GateBwArgs a{};
  a.h = hid;
  a.dout = dout;
  a.kv = h->bw_kv;
  a.w_q = h->norm_q;
  a.w_k = h->norm_k;
  a.dh = dhid;
  a.dkv = h->bw_dkv;
  a.partials = h->bw_partials;
  a.err = h->d_err;
  a.R = R;
  a.M = M;
  a.d = d;
  a.bf16 = h->cfg.dtype == ENGRAM_BF16;
  a.eps = h->cfg.eps;
  a.inv_sqrt_d = (float)(1.0 / std::sqrt((double)d));
  CK(h, launch_gate_backward(a, grid, st));
  h->launches += 1;
  if (dnorm_q || dnorm_k) {
    CK(h, launch_dnorm_reduce(h->bw_partials, grid, (int64_t)M * d, dnorm_q, dnorm_k, st));
    h->launches += 1;
  }
  CK(h, mark(3));

  // weight gradients (Eq. 3 transposed): dW_K += dk^T e, dW_V += dv^T e, a
  // contraction over the rows (both operands MN-major)
  if (bf16) {
    GemmArgs g{};
    g.N = dm;
    g.K = (int)R;
    g.kb_split = 1 << 30;
    if (dw_k) {
      g.M = Md;
      if ((rc = gemm_bf16(h, true, true, true, dkv, R, nkv, h->e, R, nullptr, 0, dm, dw_k, Md, dm,
                          g, st)))
        return rc;
    }
    if (dw_v) {
      g.M = d;
      g.a_off = Md;
      if ((rc = gemm_bf16(h, true, true, true, dkv, R, nkv, h->e, R, nullptr, 0, dm, dw_v, d, dm,
                          g, st)))
        return rc;
    }
  } else {
    const float* dkv32 = (const float*)h->bw_dkv;
    const float* e32 = (const float*)h->e;
    if (dw_k && (rc = gemm_f32(h, dkv32, 1, nkv, e32, 1, dm, dw_k, dm, Md, dm, (int)R, true, st)))
      return rc;
    if (dw_v &&
        (rc = gemm_f32(h, dkv32 + Md, 1, nkv, e32, 1, dm, dw_v, dm, d, dm, (int)R, true, st)))
      return rc;
  }
  CK(h, mark(4));

  // memory-vector gradient de = [dk dv] [W_K; W_V] (B MN-major, its K range
  // from the two weight tensors), then the table rows (Eq. 2 transposed)
  if (dtables) {
    if (bf16) {
      GemmArgs g{};
      g.M = (int)R;
      g.N = dm;
      g.K = nkv;
      g.kb_split = Md / 64;
      if ((rc = gemm_bf16(h, false, true, false, dkv, R, nkv, h->w_k, Md, h->w_v, d, dm, h->bw_de,
                          R, dm, g, st)))
        return rc;
    } else {
      const float* dkv32 = (const float*)h->bw_dkv;
      if ((rc = gemm_f32(h, dkv32, nkv, 1, (const float*)h->w_k, 1, dm, h->bw_de, dm, (int)R, dm,
                         Md, false, st)) ||
          (rc = gemm_f32(h, dkv32 + Md, nkv, 1, (const float*)h->w_v, 1, dm, h->bw_de, dm, (int)R,
                         dm, d, true, st)))
        return rc;
    }
    TableGradArgs tg{};
    tg.de = h->bw_de;
    tg.idx = z;
    tg.primes = h->d_primes;
    for (int s = 0; s < S * h->shards; ++s) tg.dtables[s] = dtables[s];
    tg.shards = h->shards;
    tg.err = h->d_err;
    tg.rows = R;
    tg.S = S;
    tg.d_head = h->cfg.d_head;
    CK(h, launch_table_grad(tg, st));
    h->launches += 1;
  }
  CK(h, mark(5));
  return ENGRAM_OK;
}

int engram_profile_next_backward(engram_handle* h, void* const* events, int32_t n_events) {
  if (!h) return ENGRAM_ERR_INVALID;
  if (!events) {
    h->bprof_armed = false;
    return ENGRAM_OK;
  }
  if (n_events != 6) return fail(h, ENGRAM_ERR_INVALID, "n_events must be 6");
  for (int i = 0; i < n_events; ++i) {
    if (!events[i]) return fail(h, ENGRAM_ERR_INVALID, "null event");
    h->bprof[i] = (cudaEvent_t)events[i];
  }
  h->bprof_armed = true;
  return ENGRAM_OK;
}

int engram_profile_next_forward(engram_handle* h, void* const* events, int32_t n_events) {
  if (!h) return ENGRAM_ERR_INVALID;
  if (!events) {
    h->prof_armed = false;
    return ENGRAM_OK;
  }
  if (n_events != 5 && n_events != 6) return fail(h, ENGRAM_ERR_INVALID, "n_events must be 5 or 6");
  for (int i = 0; i < n_events; ++i) {
    if (!events[i]) return fail(h, ENGRAM_ERR_INVALID, "null event");
    h->prof[i] = (cudaEvent_t)events[i];
  }
  h->n_prof = n_events;
  h->prof_armed = true;
  return ENGRAM_OK;
}

int64_t engram_kernel_launches(const engram_handle* h) { return h ? h->launches : -1; }

int engram_selftest_timeout(engram_handle* h, void* stream) {
  if (!h) return ENGRAM_ERR_INVALID;
  // both kinds of bounded wait: an mbarrier, then a count in global memory
  for (int which = 0; which < 2; ++which) {
    CK(h, launch_wait_timeout_selftest(h->d_err, which, (cudaStream_t)stream));
    h->launches += 1;
    const int rc = engram_check_errors(h, stream);
    if (rc != ENGRAM_ERR_TIMEOUT) return rc;  // ENGRAM_OK: the wait did not expire
  }
  return fail(h, ENGRAM_ERR_TIMEOUT, "both bounded waits expired and were reported");
}

int engram_check_errors(engram_handle* h, void* stream) {
  if (!h) return ENGRAM_ERR_INVALID;
  CK(h, cudaStreamSynchronize((cudaStream_t)stream));
  unsigned w = 0;
  CK(h, cudaMemcpy(&w, h->d_err, sizeof(w), cudaMemcpyDeviceToHost));
  CK(h, cudaMemset(h->d_err, 0, sizeof(unsigned)));
  if (w & kDevErrTimeout) return fail(h, ENGRAM_ERR_TIMEOUT, "a kernel's bounded wait expired");
  if (w & (kDevErrToken | kDevErrIndex))
    return fail(h, ENGRAM_ERR_BOUNDS,
                (w & kDevErrToken) ? "token id outside [0, vocab) replaced by the pad id"
                                   : "table index outside the table: zero row used");
  return ENGRAM_OK;
}

}  // extern "C"
