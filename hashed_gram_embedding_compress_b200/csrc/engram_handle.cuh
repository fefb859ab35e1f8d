// The handle behind the C ABI (include/engram.h): configuration, device
// copies of the hash parameters, borrowed parameters, tensor maps of the
// weights, scratch and prefetch state.  Internal to libengram.so.
#pragma once

#include <string>

#include "../../include/engram.h"
#include "engram_internal.cuh"
#include "host_gather.cuh"

struct engram_handle {
  engram_config cfg{};
  int device = 0, sms = 148;
  int S = 0, max_order = 0, d_mem = 0, elt = 4;
  int64_t primes[engram::kMaxTables] = {};
  uint64_t mult[engram::kMaxTables * engram::kMaxOrders] = {};
  std::string last_error;

  // device copies of the configuration
  int32_t* d_map = nullptr;
  int64_t* d_primes = nullptr;
  uint64_t* d_barrett = nullptr;  // floor((2^64 - 1) / p) per table, for x mod p
  uint64_t* d_mult = nullptr;
  unsigned* d_err = nullptr;

  // borrowed parameters
  bool have_params = false;
  const void* tables[engram::kMaxTables] = {};
  const void** d_tables = nullptr;  // device array of S x shards table (shard) pointers
  int shards = 1;                   // row shards per table (engram_set_table_shards)
  const void* w_k = nullptr;
  const void* w_v = nullptr;
  float* d_wqk = nullptr;           // norm_q * norm_k, [M, d]
  const float* norm_q = nullptr;    // [M, d] (borrowed; the backward needs both factors)
  const float* norm_k = nullptr;
  CUtensorMap map_wk[3], map_wv[3]; // box widths 64, 128, 256

  // short convolution (Eq. 5): off while conv_W == 0
  int conv_W = 0, conv_dil = 0;
  float* d_conv_w = nullptr;   // [d][4], taps >= conv_W zero
  float* d_conv_nw = nullptr;  // [d]
  float* d_conv_taps = nullptr;  // [4][d]: conv_w times norm_w, tap-major

  // FP8 projections (engram_set_fp8): E4M3 copy of [W_K; W_V] with one scale
  // per row, and per-row E4M3 scratch of e
  bool fp8 = false;
  uint8_t* d_w8 = nullptr;     // [(M + 1) d, d_mem]: the M d rows of W_K, then W_V
  float* d_sw8 = nullptr;      // [(M + 1) d]
  CUtensorMap map_wk8, map_wv8;
  int64_t fp8_cap_rows = 0;
  uint8_t* e8 = nullptr;       // [rows, d_mem] codes of e
  float* se8 = nullptr;        // [rows] scales of e
  uint8_t* e8_alt = nullptr;
  float* se8_alt = nullptr;

  // scratch, sized for cap_rows emitted positions.  The forward alternates
  // between two buffers of e (e, e_alt; e8/se8 and their twins for FP8), so a
  // call's gather may run while the previous call's value launch still reads
  // the other one.
  int64_t cap_rows = 0;
  void* e = nullptr;
  void* e_alt = nullptr;
  int e_flip = 0;
  float4* partials = nullptr;
  float* alpha_scratch = nullptr;  // [rows, M]: alpha formed once per row at short calls
  unsigned* fused_sync = nullptr;  // counters of the one-launch short-call kernel
  float* fused_vt = nullptr;       // its v hand-off buffer, d x 256 fp32
  int fused_clusters = -1;         // its clusters resident at once (-1: not yet asked)
  // short-convolution scratch, sized for conv_cap_rows
  int64_t conv_cap_rows = 0;
  float* conv_v = nullptr;      // [rows, d] v = W_V e
  float* conv_vv = nullptr;     // [d / 64][rows] sums of v^2 per value tile
  float* conv_alpha = nullptr;  // [rows, M] when the caller passes none
  float* conv_scale = nullptr;  // [rows, M] alpha / sqrt(alpha^2 mean(v^2) + eps)

  // host-resident tables: prefetch state, double-buffered
  int64_t pf_cap_rows = 0;
  uint32_t set_cap = 0;
  unsigned long long* d_keys = nullptr;
  int32_t* d_vals = nullptr;
  unsigned long long* d_count[2] = {nullptr, nullptr};  // [2] each: host-table rows, hot rows
  int2* d_uniq = nullptr;
  int64_t* d_remap[2] = {nullptr, nullptr};
  void* d_staging[2] = {nullptr, nullptr};
  const void** d_stage_tables[2] = {nullptr, nullptr};
  int64_t* d_stage_bound = nullptr;
  cudaEvent_t ev_ready[2] = {nullptr, nullptr};
  cudaEvent_t ev_consumed[2] = {nullptr, nullptr};
  int64_t pf_rows[2] = {0, 0};
  uint64_t n_prefetch = 0, n_consumed = 0;
  // how step 5 moves the rows (engram_set_prefetch): host threads + copy
  // engines, or zero-copy loads on a few CTAs
  int pf_mode = ENGRAM_PREFETCH_HOST_THREADS;
  int pf_workers = 0;                           // 0: the default for the mode
  engram::HostGather* hg = nullptr;             // host-thread route
  // engram_forward_host: device staging of two calls (so that one call's
  // host-to-device copies overlap the previous call's device-to-host ones),
  // the two copy streams and their events
  void* io_h[2] = {nullptr, nullptr};
  int32_t* io_tok[2] = {nullptr, nullptr};
  float* io_alpha[2] = {nullptr, nullptr};
  size_t io_h_bytes = 0, io_tok_bytes = 0, io_alpha_bytes = 0;
  cudaStream_t io_in = nullptr, io_out = nullptr;
  cudaEvent_t io_ev_in[2] = {nullptr, nullptr}, io_ev_comp[2] = {nullptr, nullptr},
              io_ev_out[2] = {nullptr, nullptr};
  int io_flip = 0;
  // engram_backward_host: h, dout and dh of two calls
  void* bio_h[2] = {nullptr, nullptr};
  void* bio_dout[2] = {nullptr, nullptr};
  void* bio_dh[2] = {nullptr, nullptr};
  int32_t* bio_tok[2] = {nullptr, nullptr};
  size_t bio_bytes = 0, bio_tok_bytes = 0;
  cudaStream_t copy_stream = nullptr;
  cudaEvent_t ev_list[2] = {nullptr, nullptr};  // the row list has reached the host
  unsigned long long* h_count[2] = {nullptr, nullptr};  // pinned [2]
  int2* h_list[2] = {nullptr, nullptr};         // pinned [rows*S]
  char* h_bounce[2] = {nullptr, nullptr};       // pinned [rows*S, row_bytes]

  // hot-row cache in HBM in front of the host tables (engram_build_hot_cache)
  int64_t n_hot = 0;
  uint32_t hot_cap = 0;
  unsigned long long* d_hot_keys = nullptr;  // [hot_cap] set of (s << 40 | z)
  int32_t* d_hot_slots = nullptr;            // [hot_cap] cache slot per bucket
  void* d_hot_rows = nullptr;                // [n_hot, row_bytes]

  // backward (engram_backward): scratch sized for bw_cap_rows
  int64_t bw_cap_rows = 0;
  int64_t* bw_idx = nullptr;       // [rows, S]
  float* bw_kv = nullptr;          // [rows, (M + 1) d]
  void* bw_dkv = nullptr;          // [rows, (M + 1) d] dtype
  float* bw_de = nullptr;          // [rows, d_mem]
  float* bw_partials = nullptr;    // [bw_part_blocks][2][M][d]
  int bw_part_blocks = 0;

  // tensor maps of the per-call operands (e, h, out), keyed by their
  // arguments: a repeated call shape encodes nothing on the host
  struct MapEntry {
    const void* base = nullptr;
    int64_t cols = 0, rows = 0;
    int box_rows = 0, box_cols = 0, esz = 0;
    CUtensorMap map;
  };
  static constexpr int kMapCache = 32;
  MapEntry map_cache[kMapCache];
  int map_cache_next = 0;

  // instrumentation
  int64_t launches = 0;
  cudaEvent_t prof[6] = {};
  int n_prof = 0;
  bool prof_armed = false;
  cudaEvent_t bprof[6] = {};  // stages of the next engram_backward
  bool bprof_armed = false;
};

namespace engram {

// 2-D row-major tensor map of `rows` rows x `cols` elements of esz bytes (2:
// bf16, 4: fp32, 1: E4M3 codes) with a box of box_cols x box_rows; a box row
// of 128 bytes gets the 128-byte swizzle, any other the 64-byte one.  On
// failure the message goes to h->last_error.
int make_map(engram_handle* h, CUtensorMap* m, const void* base, int64_t cols, int64_t rows,
             int box_rows, int box_cols = 64, int esz = 2);
// make_map through the handle's cache of recently encoded maps.
int cached_map(engram_handle* h, CUtensorMap* m, const void* base, int64_t cols, int64_t rows,
               int box_rows, int box_cols = 64, int esz = 2);

// Frees what engram_forward_host allocated (after a device synchronise).
void free_host_io(engram_handle* h);

// Index into the handle's W tensor maps (map_wk, map_wv) of a box width.
inline int bn_index(int bn) { return bn == 64 ? 0 : bn == 128 ? 1 : 2; }

}  // namespace engram
