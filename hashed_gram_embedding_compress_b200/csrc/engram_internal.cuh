// Internal interface between the C-ABI layer (engram_api.cu) and the kernels.
// Not installed; callers use include/engram.h.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/engram.h"

namespace engram {

// Bits of the handle's device error word.
constexpr unsigned kDevErrToken = 1u;    // token id outside [0, V): pad used instead
constexpr unsigned kDevErrIndex = 2u;    // table index outside [0, p): zero row used
constexpr unsigned kDevErrTimeout = 4u;  // a bounded mbarrier wait expired

constexpr int kMaxTables = 64;
constexpr int kMaxOrders = 4;
constexpr int kMaxBranches = 4;
constexpr int kMaxShards = 8;  // row shards per table (engram_set_table_shards)

#ifdef __CUDACC__
// Programmatic dependent launch: a kernel launched with the programmatic
// stream-serialization attribute may start while the previous kernel on the
// stream runs; griddep_wait() blocks until that kernel has completed and its
// memory is visible, griddep_launch_dependents() lets the next such kernel
// start.  Both are no-ops in a kernel launched without the attribute.
__device__ __forceinline__ void griddep_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
#endif

// Everything the compress+hash kernel needs (section 2.2, Eq. 1).
struct HashArgs {
  const int32_t* tokens;   // [B, T] raw ids
  const int32_t* map;      // [V] compression map
  const uint64_t* mult;    // [S, max_order] odd multipliers
  const int64_t* primes;   // [S]
  const uint64_t* barrett; // [S] floor((2^64 - 1) / primes[s])
  int64_t* idx;            // [B*(T-t_begin), S]
  unsigned* err;
  int32_t V, pad, B, T, t_begin, S, heads, num_orders, max_order;
  int32_t orders[kMaxOrders];
};

// Row gather (Eq. 2).  Tables are addressed through a device array of S pointers.
// Row-sharded tables: row z of table s lives in shard z % shards at local row
// z / shards; `tables` then holds S x shards pointers, table-major.
struct GatherArgs {
  const void* const* tables;  // device array [S x shards] of table (shard) base pointers
  int32_t shards;             // 1: whole tables
  const int64_t* primes;      // [S]
  const int64_t* idx;         // [rows, S]
  void* e;                    // [rows, S*d_head]
  unsigned* err;
  int64_t rows;
  int32_t S;
  int32_t row_bytes;          // d_head * element size, a multiple of 16
};

// Hash and gather in one pass (Eq. 1 then Eq. 2), for device-resident tables.
struct HashGatherArgs {
  HashArgs hash;              // idx is unused: the indices stay on chip
  const void* const* tables;  // device array [S x shards] of table (shard) base pointers
  int32_t shards;             // 1: whole tables
  void* e;                    // [rows, S*d_head]
  uint8_t* q;                 // E4M3 form: codes [rows, S*d_head] (bf16 tables)
  float* scale;               // E4M3 form: power-of-two scale per row
  int32_t row_bytes;          // d_head * element size, a multiple of 16
  int32_t rows_per_block;     // set by the launcher
  // 1: launch with programmatic dependent launch, so that the kernel runs
  // while the previous kernel on the stream (the previous call's value
  // launch, which reads the other e buffer) finishes; each block waits for
  // that kernel before it exits, so the next launch still sees it complete.
  int32_t pdl;
};

// Projection + gate epilogue arguments (Eq. 3, 4, 6).
struct GateArgs {
  const void* h;        // [R, M, d]
  void* out;            // [R, M, d]
  const float* w_qk;    // [M, d]: norm_q * norm_k (the two RMSNorm weights multiply)
  float4* partials;     // [num key tiles][R]: (sum k^2, sum h w_q w_k k, sum h^2, 0)
  float* alpha;         // [R, M] or null
  // [R, M] alpha already formed from the partial sums (launch_row_alpha), or
  // null: the value phase forms it itself from `partials`
  const float* alpha_in;
  float* delta;         // [R, M, d] or null
  float* vals;          // phase 3: v = W_V e, fp32 [R, d]
  float* vv;            // phase 3: sum of v^2 per value tile and row, [d / value tile][R]
  unsigned* err;
  int32_t R, M, d, d_mem;
  const float* s_row;   // FP8 operands: scale of each row of e [R] (else null)
  const float* s_col;   // FP8 operands: scale of each W row of this phase's columns
  int32_t key_tile;     // width of the key-phase tiles that wrote `partials`
  float eps;
  float inv_sqrt_d;
  // one launch for steps 5-7 of a short call (launch_proj_gate_fused): [0],
  // [1] key CTAs done per 128-row half, [2] CTAs done; zero between launches
  unsigned* sync;
  float* vt;            // fused short-call kernel: v handed to the key CTAs, [2 row halves][d / 4][128][4]
  // 1: launch with programmatic dependent launch.  The key phase then waits
  // for the previous kernel (the gather) before reading e and lets the value
  // phase start early; the value phase's epilogue waits for the key phase
  // before it reads the partial sums or writes out.
  int32_t pdl;
};

// Short convolution and residual (Eq. 5) over B sequences of T positions.
struct ConvArgs {
  const float* vals;    // [B*T, d] v = W_V e (fp32)
  const float* vv;      // [n_vtiles][B*T] sums of v^2 per value tile
  const float* alpha;   // [B*T, M]
  const void* h;        // [B*T, M, d] fp32 or bf16
  void* out;            // [B*T, M, d], may alias h
  float* delta;         // [B*T, M, d] the increment Y, or null
  const float* taps;    // [4][d]: tap i of channel c (it multiplies position
                        // t - i * dilation) times the RMSNorm weight of c
  int32_t B, T, M, d, n_vtiles, bf16;
  float eps;
};

// Backward of the gate and residual (training): see k_backward.cu.
struct GateBwArgs {
  const void* h;        // [R, M, d] fp32 or bf16
  const void* dout;     // [R, M, d] gradient of out, same dtype
  const float* kv;      // [R, (M + 1) d]: k of each branch, then v (recomputed, fp32)
  const float* w_q;     // [M, d] RMSNorm weight of the query
  const float* w_k;     // [M, d] RMSNorm weight of the key
  void* dh;             // [R, M, d] gradient of h, same dtype
  void* dkv;            // [R, (M + 1) d] dk of each branch, then dv, same dtype
  float* partials;      // [grid][2][M][d] per-CTA sums for the RMSNorm weight gradients
  unsigned* err;        // device error word (a bounded wait that expired)
  int64_t R;
  int32_t M, d;
  bool bf16;
  float eps, inv_sqrt_d;
};

// Table gradients: dtables[s][idx[r][s]] += the slot-s slice of de[r].
struct TableGradArgs {
  const float* de;               // [rows, S * d_head]
  const int64_t* idx;            // [rows, S]
  const int64_t* primes;         // [S] (indices outside a table are skipped and flagged)
  float* dtables[kMaxTables * kMaxShards];  // fp32 [rows of the shard, d_head], table-major
  unsigned* err;
  int64_t rows;
  int32_t S, d_head;
  int32_t shards;                // 1: whole tables
};

size_t gate_bw_smem(int M, int d);
size_t gate_bw_ring_smem(int M, int d, int elt);
int gate_bw_grid(int M, int d, int64_t R, int elt);
// d <= 4096 and gate_bw_smem(M, d) within the per-CTA shared memory limit.
cudaError_t launch_gate_backward(const GateBwArgs& a, int grid, cudaStream_t stream);
// dnorm_q[i] += sum_b partials[b][0][i], dnorm_k[i] += sum_b partials[b][1][i]
// over the nblocks CTAs in order (n = M d; either output may be null).
cudaError_t launch_dnorm_reduce(const float* partials, int nblocks, int64_t n, float* dnorm_q,
                                float* dnorm_k, cudaStream_t stream);
cudaError_t launch_table_grad(const TableGradArgs& a, cudaStream_t stream);

// Prefetch of host-resident rows into an HBM staging buffer (section 2.5).
struct PrefetchArgs {
  const int64_t* idx;           // [rows, S] table indices of the upcoming step
  int64_t rows;
  int32_t S;
  unsigned long long* keys;     // [cap] open-addressing set, cap a power of two >= 2*rows*S
  int32_t* vals;                // [cap] staging slot of each occupied bucket
  uint32_t cap;
  unsigned long long* count;    // [2]: distinct rows from the host tables, from the hot cache
  int2* uniq;                   // [rows*S] per staging slot: (s, z) at the front, (-1, cache
                                // slot) at the back
  int64_t* remapped;            // [rows, S] staging slot of each index
  const void* const* tables;    // device array [S] of pinned host table pointers
  int32_t row_bytes;
  void* staging;                // [rows*S, row_bytes] device
  int sms;
  int fetch_blocks;             // grid of the zero-copy fetch kernel
  // hot-row cache in HBM (null hot_keys: none): its rows are copied from HBM
  const unsigned long long* hot_keys;  // [hot_cap] open-addressing set of (s << 40 | z)
  const int32_t* hot_slots;     // [hot_cap] cache slot of each occupied bucket
  uint32_t hot_cap;             // power of two
  const void* hot_rows;         // [cached rows, row_bytes]
};

// Hot-row cache building blocks (host-resident tables).
// Count how often each (s, z) of idx [n / S, S] is addressed: keys/counts are
// an open-addressing table of cap (a power of two >= 2 n) buckets.
cudaError_t launch_count_rows(const int64_t* idx, int64_t n, int32_t S, unsigned long long* keys,
                              unsigned long long* counts, uint32_t cap, int sms,
                              cudaStream_t stream);
// Insert the n chosen keys (cache slot = list position) into the cache's
// lookup table (hot_cap buckets) and copy their rows from the host tables
// into rows [n, row_bytes].
cudaError_t launch_fill_hot_cache(const unsigned long long* list, int64_t n,
                                  unsigned long long* hot_keys, int32_t* hot_slots,
                                  uint32_t hot_cap, const void* const* tables, int32_t row_bytes,
                                  void* rows, int sms, cudaStream_t stream);

// Launchers (all asynchronous on `stream`; return the launch error).
cudaError_t launch_hash(const HashArgs& a, cudaStream_t stream);
cudaError_t launch_gather(const GatherArgs& a, cudaStream_t stream);
cudaError_t launch_hash_gather(const HashGatherArgs& a, cudaStream_t stream);
// Hash + gather + E4M3 quantisation of each row of e (FP8 projections): writes
// a.q and a.scale instead of a.e; bf16 tables, S * d_head <= 2048.
cudaError_t launch_hash_gather_e4m3(const HashGatherArgs& a, cudaStream_t stream);
// E4M3 codes q [rows, cols] and power-of-two scales [rows] of bf16 x [rows,
// cols]; 16 <= cols <= 2048, cols a multiple of 16.
cudaError_t launch_quantize_e4m3(const void* x, int64_t rows, int cols, uint8_t* q, float* scale,
                                 cudaStream_t stream);
// taps[i][c] = conv_w[c][i] * norm_w[c] for the [d][4] conv weights.
cudaError_t launch_conv_taps(const float* conv_w, const float* norm_w, int d, float* taps,
                             cudaStream_t stream);
// dilation 1..4; scale is scratch [B*T, M] fp32.  Two launches: the RMS
// scale per (position, branch), then the convolution and residual.
cudaError_t launch_short_conv(const ConvArgs& a, int dilation, float* scale, cudaStream_t stream);
// Steps 1-4 of the prefetch: distinct rows, staging slots, remapped indices,
// hot rows copied from the cache.
cudaError_t launch_prefetch_index(const PrefetchArgs& a, cudaStream_t stream);
// Step 5 by zero-copy loads: the count[0] rows of the host tables listed at
// the front of uniq, on a.fetch_blocks CTAs.
cudaError_t launch_prefetch_fetch(const PrefetchArgs& a, cudaStream_t stream);
cudaError_t launch_wait_timeout_selftest(unsigned* err, int which, cudaStream_t stream);
cudaError_t launch_mul(const float* x, const float* y, float* out, int64_t n, cudaStream_t stream);

// fp32 path (SIMT FFMA; 64-column tiles).  phase 0 = key tiles over W_K
// [M*d, d_mem], phase 1 = value tiles over W_V [d, d_mem].
constexpr int kF32Tile = 64;
cudaError_t launch_proj_gate_f32(int phase, const float* e, const float* w, const GateArgs& g,
                                 cudaStream_t stream);

// bf16 path (tcgen05 / TMEM / TMA, sm_100a).  `bn` in {64, 128, 256}.
int sm100_stages(int bn);
// Tensor maps of one launch, all bf16: e [R, d_mem] and W [N, d_mem] with the
// 128-byte swizzle, h and out viewed as [R, M*d].
//   single-CTA kernel: e box 64 x 128, W box 64 x BN, h/out box 64 x 128 (128-B swizzle)
//   CTA-pair kernel:   e box 64 x 256, W box 64 x 128, h box 32 x 256, out box 32 x 32
//                      (h and out with the 64-B swizzle)
struct ProjMaps {
  CUtensorMap e, w, h, out;
};
cudaError_t launch_proj_gate_sm100(int phase, int bn, const ProjMaps& maps, const GateArgs& g,
                                   int grid, cudaStream_t stream);
// alpha[R, M] from the key phase's partial sums (g.partials, g.key_tile):
// the value phase of a short call then reads it instead of every value CTA
// summing the same partials.  Launched between the key and value launches
// with programmatic dependent launch when g.pdl.
cudaError_t launch_row_alpha(const GateArgs& g, float* alpha, cudaStream_t stream);
// 512 x 256 tiles on CTA pairs (tcgen05 cta_group::2); grid = 2 x pairs.
// phase 0 keys, 1 values, 2 values added in place (out aliases h), 3 values
// for the short convolution.  f8: e and W are E4M3 codes (maps of uint8 with
// 128-column boxes) with the scales g.s_row and g.s_col.
cudaError_t launch_proj_gate_wide(int phase, const ProjMaps& maps, const GateArgs& g, int grid,
                                  cudaStream_t stream, bool f8 = false);

// 256 x 256 tiles on CTA pairs with two TMEM accumulators (few rows, many
// columns); grid = 2 x pairs; key tiles of 128 columns (g.key_tile must be
// 128 in phase 0).  Phases 0-2 as above.
cudaError_t launch_proj_gate_pair(int phase, const ProjMaps& maps, const GateArgs& g, int grid,
                                  cudaStream_t stream);

// Steps 5-7 of a short call (R <= 256, bf16, d a multiple of 256, M <= 4) in
// one launch of nkey = M d / 256 key clusters and nval = d / 128 value
// clusters (CTA pairs); out = h + alpha v (out may alias h); g.partials,
// g.sync (kFusedSyncWords, zeroed), g.vt (d x 256 fp32), g.alpha and g.delta
// as for the other kernels.  Every CTA must be resident at once: 2 (nkey +
// nval) CTAs at one per SM, nkey + nval <= fused_max_clusters().
constexpr int kFusedSyncWords = 16;
struct FusedMaps {
  CUtensorMap e;    // e [R, d_mem], boxes of 128 rows x 64
  CUtensorMap wk;   // W_K [M d, d_mem], boxes of 128 rows x 64
  CUtensorMap wv;   // W_V [d, d_mem], boxes of 64 rows x 64
  CUtensorMap h;    // h [R, M d], boxes of 128 rows x 32
  CUtensorMap out;  // out [R, M d], boxes of 32 rows x 32
};
cudaError_t launch_proj_gate_fused(const FusedMaps& maps, const GateArgs& g, int nkey, int nval,
                                   cudaStream_t stream);
// Clusters of the fused kernel that can be resident at once on this device (0
// if unknown).
int fused_max_clusters();

// Dense contractions of the backward (bf16 operands, fp32 accumulation):
// D[m, n] (= or +=) sum_k A(m, k) B(n, k), m < M, n < N, k < K.  A K-major A
// is stored [rows, K] (map box 64 x 128, 128-byte swizzle), an MN-major A
// [K, rows] (box 64 x 64); the same for B.  B's K range may come from two
// tensors: K blocks (of 64) below kb_split from map b0, the rest from map b1
// at K - 64 kb_split.  D is fp32 (map box 32 x 32, 128-byte swizzle), n = 0 at
// column d_col0.  With `add` the tiles reduce-add into D, and K may be split
// over `splits` tiles of kb_per_split K blocks each.
struct GemmArgs {
  int32_t M, N, K;
  int32_t a_off;          // first A row (K-major) or column (MN-major) used
  int32_t kb_split;       // K blocks read from map b0
  int32_t splits, kb_per_split;
  int32_t d_col0;
  unsigned* err;
};
struct GemmMaps {
  CUtensorMap a, b0, b1, d;
};
// Tiles of 256 x 256 (one per CTA pair and round) times the K splits.
int gemm_pair_tiles(const GemmArgs& g);
// grid = 2 x pairs (even).
cudaError_t launch_gemm_pair(bool a_mn, bool b_mn, bool add, const GemmMaps& maps,
                             const GemmArgs& g, int grid, cudaStream_t stream);

// fp32 form (SIMT FFMA, 64 x 64 tiles) with strided operands:
// D[m * ldd + n] (= or +=) sum_k A[m * a_m + k * a_k] B[n * b_n + k * b_k].
struct GemmF32Args {
  const float* A;
  int64_t a_m, a_k;
  const float* B;
  int64_t b_n, b_k;
  float* D;
  int64_t ldd;
  int32_t M, N, K;
  bool add;
};
cudaError_t launch_gemm_f32(const GemmF32Args& g, cudaStream_t stream);

// The bf16 projection kernel of one phase (0 keys, 1 values) for R rows.
enum class ProjKernel { Wide, Pair, Single };
struct ProjChoice {
  ProjKernel kind;
  int bn;        // W rows per TMA box (the tensor map of W to use)
  int grid;      // CTAs
  int key_tile;  // columns per partial-sum tile (phase 0)
};
// The kernel with the least estimated time: rounds of tiles per SM (or per
// CTA pair) x the time of one tile.  A tile's mainloop streams its operands
// from L2 at a fixed rate per SM, so its time is about the rows of K it
// streams per CTA: 512 x 256 pair tiles 256 + 128, 256 x 256 pair tiles
// 128 + 128, single-CTA 128 x N tiles 128 + N; the 512 x 256 tile holds its
// accumulators through the gate epilogue (one TMEM buffer), which adds about
// 30 % per tile, while the other two overlap it with the next tile (measured
// on B200: 13.2 us mainloop + 3.1-4.3 us epilogue per 512 x 256 tile).  Key
// tiles must not straddle branches, so their width divides d.  The value
// phase of the short convolution (phase 3) has no 256 x 256 pair variant.
// The 512 x 256 CTA-pair kernel (the only one with E4M3 operands): one CTA
// pair per tile up to every pair of SMs.  d a multiple of 256.
inline ProjChoice wide_proj(int phase, int64_t R, int M, int d, int sms) {
  const int n_total = phase == 0 ? M * d : d;
  const int pairs = sms / 2;
  const int64_t tiles = (R + 511) / 512 * (n_total / 256);
  return {ProjKernel::Wide, 128, 2 * (int)(tiles < pairs ? tiles : pairs), 256};
}

inline ProjChoice choose_proj(int phase, int64_t R, int M, int d, int sms, int flags,
                              bool conv = false) {
  const int n_total = phase == 0 ? M * d : d;
  const int pairs = sms / 2;
  const bool pairs_ok = !(flags & ENGRAM_FLAG_NO_CTA_PAIRS) && n_total % 256 == 0;
  const int64_t mblk = (R + 127) / 128;
  ProjChoice best{ProjKernel::Single, 64, 1, 64};
  int64_t best_cost = -1;
  for (int c : {256, 128, 64}) {
    if (n_total % c != 0 || d % c != 0) continue;
    const int64_t tiles = mblk * (n_total / c);
    const int64_t cost = (tiles + sms - 1) / sms * (128 + c) * 10;
    if (best_cost < 0 || cost < best_cost) {
      best_cost = cost;
      best = {ProjKernel::Single, c, (int)(tiles < sms ? tiles : sms), c};
    }
  }
  if (pairs_ok && d % 128 == 0 && !(phase == 1 && conv)) {
    const int64_t tiles = (R + 255) / 256 * (n_total / 256);
    const int64_t cost = (tiles + pairs - 1) / pairs * 256 * 10;
    const int grid = 2 * (int)(tiles < pairs ? tiles : pairs);
    if (cost < best_cost) {
      best_cost = cost;
      best = {ProjKernel::Pair, 128, grid, 128};
    }
  }
  if (pairs_ok && d % 256 == 0) {
    const int64_t tiles = (R + 511) / 512 * (n_total / 256);
    const int64_t cost = (tiles + pairs - 1) / pairs * 384 * 13;
    if (cost <= best_cost) best = wide_proj(phase, R, M, d, sms);
  }
  return best;
}

}  // namespace engram
