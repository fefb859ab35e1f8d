/*
 * engram.h -- C ABI of libengram.so: the forward lookup-and-gate step of the
 * Engram conditional-memory module on one NVIDIA B200 (sm_100a).
 *
 * Method: "Conditional Memory via Scalable Lookup: A New Axis of Sparsity for
 * Large Language Models" (DeepSeek-AI & Peking University), section 2:
 *   2.2  tokenizer compression x' = P(x), suffix n-grams g_{t,n},
 *        multi-head hashing z_{t,n,k} = phi_{n,k}(g_{t,n}) into tables of
 *        prime size (Eq. 1), concatenation e_t of the addressed rows (Eq. 2);
 *   2.3  k_t = W_K e_t, v_t = W_V e_t (Eq. 3);
 *        alpha_t = sigmoid(RMSNorm(h_t) . RMSNorm(k_t) / sqrt(d)) (Eq. 4);
 *        gated value alpha_t v_t added to the hidden state;
 *   2.4  multi-branch form: one W_K per branch, W_V shared (Eq. 6);
 *   2.5  tables offloaded to host memory, rows prefetched over PCIe
 *        because the indices depend on the tokens only (Figure 2b).
 *
 * Conventions for every call:
 *  - Return value: ENGRAM_OK (0) or one of the ENGRAM_ERR_* codes below.  No
 *    call aborts or throws; engram_last_error() gives a message for the last
 *    failure on that handle.
 *  - "device" pointers point into the memory of the device that was current
 *    at engram_create; "host" pointers are ordinary CPU memory; "pinned host"
 *    is page-locked host memory (cudaHostAlloc / cudaHostRegister).
 *  - All tensors are row-major and densely packed; shapes are given in
 *    brackets, outermost first.  Every buffer is owned by the caller and is
 *    only borrowed for the duration of the call, except the parameter
 *    pointers given to engram_set_params, which must stay valid until the
 *    handle is destroyed or new parameters are set.
 *  - `stream` is a cudaStream_t passed as void* (NULL = the legacy default
 *    stream).  Work is enqueued asynchronously on it; results are ready when
 *    the stream reaches that point.  A handle must not be used from two
 *    streams at once: its scratch buffers are shared by its calls.
 *  - Device-side range violations (a token id outside [0, V)) never lead to
 *    an out-of-bounds access: the kernel substitutes the pad id, sets a bit in
 *    the handle's device error word, and engram_check_errors() reports it.
 */
#ifndef ENGRAM_H
#define ENGRAM_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define ENGRAM_API __attribute__((visibility("default")))
#else
#define ENGRAM_API
#endif

#define ENGRAM_MAX_ORDERS 4   /* n-gram orders per module            */
#define ENGRAM_MAX_TABLES 64  /* orders x heads                      */
#define ENGRAM_MAX_BRANCHES 4 /* M of the multi-branch form (Eq. 6)  */
#define ENGRAM_MAX_SHARDS 8   /* row shards per table (engram_set_table_shards) */
#define ENGRAM_IPC_HANDLE_BYTES 64

/* element types */
#define ENGRAM_F32 0
#define ENGRAM_BF16 1

/* where the embedding tables live */
#define ENGRAM_DEVICE 0      /* HBM of the handle's device            */
#define ENGRAM_PINNED_HOST 1 /* page-locked host memory, read over PCIe */

/* config flags */
#define ENGRAM_FLAG_NO_CTA_PAIRS 1 /* bf16 projection on single-CTA tiles only */
#define ENGRAM_FLAG_NO_FUSED_SHORT 2 /* short calls: separate key, alpha and value launches */

/* how engram_prefetch moves rows from host tables (engram_set_prefetch) */
#define ENGRAM_PREFETCH_HOST_THREADS 0 /* host threads + copy engines (default) */
#define ENGRAM_PREFETCH_ZERO_COPY 1    /* device loads through the mapped address */

/* status codes */
#define ENGRAM_OK 0
#define ENGRAM_ERR_INVALID 1     /* bad argument or configuration                 */
#define ENGRAM_ERR_BOUNDS 2      /* a token id outside [0, V) was seen on device  */
#define ENGRAM_ERR_CUDA 3        /* a CUDA runtime call failed                     */
#define ENGRAM_ERR_OOM 4         /* device or pinned allocation failed             */
#define ENGRAM_ERR_TIMEOUT 5     /* a bounded device-side or prefetch wait expired */
#define ENGRAM_ERR_UNSUPPORTED 6 /* valid request the library does not implement */
#define ENGRAM_ERR_STATE 7       /* call out of order (e.g. forward before params) */

typedef struct engram_handle engram_handle;

/*
 * Module configuration (section 2.2 and Table 5 of the paper; the paper's
 * Engram-27B uses orders {2,3}, 8 heads, d_mem 1280, M = 4).
 *
 *  vocab, cvocab   V and V' of the compression map P: V -> V' (section 2.2,
 *                  "Tokenizer compression").  comp_map is a HOST int32 [vocab]
 *                  array with values in [0, cvocab); it is copied at create.
 *  pad_id          compressed id read for positions before a sequence's start;
 *                  -1 selects the default cvocab (outside the image of P, so a
 *                  padded n-gram never aliases a real one).
 *  num_orders,     the n-gram orders, ascending, each in [1, 4] (paper: {2,3}).
 *  orders
 *  heads           K hash heads per order.  Table slot s = order_index*K + k;
 *                  e_t concatenates the slots in that order (Eq. 2).
 *  primes          rows of table s.  All zero: derived as the ascending primes
 *                  >= table_rows_target, one per slot in slot order.  Non-zero
 *                  entries must all be given and be >= 2 (primality of given
 *                  sizes is not checked; the paper asks for primes).
 *  hash_seed       seed of the hash multipliers.  The pages name phi only a
 *                  "lightweight multiplicative-XOR hash"; this library fixes
 *                     x = 0; for j < n: x ^= c[t-j] * m[s][j]   (mod 2^64)
 *                     z = x mod primes[s]
 *                  with m[s][j] = SplitMix64(hash_seed) | 1 drawn for s
 *                  ascending, then j ascending, max(orders) draws per slot
 *                  (SplitMix64: Steele, Lea and Flood, OOPSLA 2014).
 *  d_head          d_h, columns of every table; d_mem = S * d_h.
 *  d_hidden        d, the backbone hidden size (also the 1/sqrt(d) scale).
 *  branches        M (1 = single stream, Eq. 4; > 1 = Eq. 6).
 *  dtype           ENGRAM_F32 or ENGRAM_BF16: type of tables, W_K, W_V, h and
 *                  out.  Accumulation is always fp32.
 *  eps             RMSNorm epsilon (the pages give none; 1e-6 is typical).
 *  table_location  ENGRAM_DEVICE or ENGRAM_PINNED_HOST.
 *  flags           0, or an OR of: ENGRAM_FLAG_NO_CTA_PAIRS to keep the bf16
 *                  projection on single-CTA 128-row tiles (by default 512 x
 *                  256 tiles on CTA pairs are used when they fill the GPU);
 *                  ENGRAM_FLAG_NO_FUSED_SHORT to run calls of at most 256 rows
 *                  as separate key, alpha and value launches (by default one
 *                  launch does all three when d is a multiple of 256, M <= 4
 *                  and its CTAs fit on the GPU at once).  All choices give the
 *                  same results up to fp32 summation order.
 */
typedef struct engram_config {
  int32_t vocab;
  int32_t cvocab;
  int32_t pad_id;
  int32_t num_orders;
  int32_t orders[ENGRAM_MAX_ORDERS];
  int32_t heads;
  int32_t d_head;
  int32_t d_hidden;
  int32_t branches;
  int32_t dtype;
  int32_t table_location;
  float eps;
  int32_t flags;
  int64_t table_rows_target;
  uint64_t hash_seed;
  int64_t primes[ENGRAM_MAX_TABLES];
  const int32_t *comp_map;
} engram_config;

/*
 * Validate `cfg`, derive primes and multipliers, copy the compression map to
 * the current device, and return a new handle in *out.  Requirements:
 * 1 <= cvocab <= vocab; 1 <= heads; num_orders * heads <= 64; d_head >= 1 with
 * d_head * element size a multiple of 16 bytes; d_hidden a multiple of 64;
 * 1 <= branches <= 4.  Errors: ENGRAM_ERR_INVALID, _OOM, _CUDA.
 */
ENGRAM_API int engram_create(const engram_config *cfg, engram_handle **out);

/* Release everything the handle owns (not the caller's buffers).  NULL is a no-op. */
ENGRAM_API void engram_destroy(engram_handle *h);

/* sizeof(engram_config) as compiled into the library (for bindings to check their layout). */
ENGRAM_API size_t engram_config_size(void);

/* Message of the last failure on `h` (or of the last failed create if h is NULL). */
ENGRAM_API const char *engram_last_error(const engram_handle *h);

/*
 * Borrow the learned parameters (section 2.2 and 2.3).
 *  tables  array of S pointers; table s is [primes[s], d_head] of dtype,
 *          device memory or pinned host memory according to table_location.
 *          Rows must start 16-byte aligned.
 *  w_k     device [M, d, d_mem] dtype: one key projection per branch (Eq. 6).
 *  w_v     device [d, d_mem] dtype: the shared value projection (Eq. 3).
 *  norm_q  device fp32 [M, d]: RMSNorm weight of the query h (Eq. 4).
 *  norm_k  device fp32 [M, d]: RMSNorm weight of the key k (Eq. 4).
 * Errors: ENGRAM_ERR_INVALID (NULL or misaligned pointer), _CUDA.
 */
ENGRAM_API int engram_set_params(engram_handle *h, const void *const *tables, const void *w_k,
                      const void *w_v, const float *norm_q, const float *norm_k);

/*
 * The short convolution of the module output (section 2.3, Eq. 5):
 *   Y = SiLU(Conv1D(RMSNorm(V~))) + V~,  out = h + Y,  V~ = alpha * v,
 * Conv1D depthwise and causal over the positions of each sequence (zero
 * before its start, no bias), kernel size W, dilation delta: tap i of channel
 * c multiplies position t - i * delta.  The paper uses W = 4, delta = the
 * largest n-gram order, zero-initialised weights (then Y = V~ exactly).  In
 * the multi-branch form the same weights act on each branch's gated values.
 *  conv_w  device fp32 [d, kernel_size] (row c holds the taps of channel c).
 *  norm_w  device fp32 [d]: RMSNorm weight (the handle's eps is used).
 *  kernel_size 1..4, or 0 to switch the convolution off again (pointers
 *          ignored); dilation 1..4.
 * The weights are copied (on `stream`, which is synchronised before the call
 * returns).  While it is on, engram_forward needs t_begin = 0 (every position
 * of each sequence is an input of the convolution) and returns
 * ENGRAM_ERR_UNSUPPORTED otherwise; its delta output receives Y; and
 * engram_project_gate_noalloc returns ENGRAM_ERR_UNSUPPORTED.  Extra scratch
 * per row: 4 d bytes of v and 4 (d / 64 + 2 M) bytes.
 * Errors: _INVALID, _STATE (engram_set_params first), _OOM, _CUDA.
 */
ENGRAM_API int engram_set_short_conv(engram_handle *h, const float *conv_w, const float *norm_w,
                                     int32_t kernel_size, int32_t dilation, void *stream);

/*
 * Row-sharded tables (section 2.5, Figure 2a: for training, the paper spreads
 * the embedding tables over the GPUs and exchanges the active rows).  Row z
 * of table s lives in shard z mod N at local row floor(z / N), so shard j of
 * table s has ceil((primes[s] - j) / N) rows of d_head elements.  Every
 * kernel that reads a table row (the forward's gather, engram_gather, the
 * backward's recomputation) and the backward's table-gradient scatter
 * address the owner's shard directly; with shards on other GPUs of the
 * node (pointers from engram_ipc_open) those are peer loads and remote
 * atomic adds over NVLink, so no request or row exchange step is needed.
 *  shards  N in [1, ENGRAM_MAX_SHARDS].
 *  ptrs    host array of S x N device pointers, table by table: ptrs[s N + j]
 *          = shard j of table s, in the handle's dtype, 16-byte aligned; own
 *          or a peer's memory.  Borrowed: must outlive the handle.
 * Replaces the tables given to engram_set_params until the next
 * engram_set_params.  Device-resident tables only (ENGRAM_ERR_UNSUPPORTED
 * otherwise).  Waits for all device work first.
 * Errors: _INVALID, _STATE (engram_set_params first), _UNSUPPORTED, _CUDA.
 */
ENGRAM_API int engram_set_table_shards(engram_handle *h, int32_t shards, const void *const *ptrs);

/*
 * CUDA inter-process handles for the shards of the other GPUs (plumbing of
 * engram_set_table_shards across processes; no counterpart in the paper).
 * engram_ipc_handle writes the ENGRAM_IPC_HANDLE_BYTES-byte handle of the
 * device allocation that starts at `ptr` (on the handle's device) into
 * `handle`; another process passes those bytes to engram_ipc_open, which maps
 * the allocation into its own device's address space (peer access enabled)
 * and returns the pointer; engram_ipc_close unmaps it.
 * Errors: _INVALID, _CUDA.
 */
ENGRAM_API int engram_ipc_handle(engram_handle *h, const void *ptr, void *handle);
ENGRAM_API int engram_ipc_open(engram_handle *h, const void *handle, void **ptr);
ENGRAM_API int engram_ipc_close(engram_handle *h, void *ptr);

/*
 * FP8 projections (section 2.4: the value projection and the M key
 * projections computed as one dense FP8 matmul).  enable = 1: every later
 * engram_forward multiplies an E4M3 form of e by an E4M3 copy of [W_K; W_V]
 * with fp32 accumulation (tcgen05.mma kind::f8f6f4); enable = 0 returns to
 * bf16 operands.  The pages give neither the format nor the scaling; here
 * each row of e (position) and each row of W (output channel) is quantised
 * as engram_quantize_e4m3 describes, and both scales multiply the fp32
 * products in the epilogue; the gate and output are unchanged.  The copy of
 * W is made now (on `stream`, then the device is synchronised) and again by
 * every engram_set_params while FP8 is on.  Needs a bf16 handle, d a multiple
 * of 256, d_mem a multiple of 128 and at most 2048, and CTA pairs (no
 * ENGRAM_FLAG_NO_CTA_PAIRS); otherwise ENGRAM_ERR_UNSUPPORTED.  While it is
 * on, engram_project_gate_noalloc returns ENGRAM_ERR_UNSUPPORTED.  Device
 * memory: (M + 1) d (d_mem + 4) bytes for W, and d_mem + 4 bytes of scratch
 * per row.  Errors: _INVALID (enable not 0 or 1), _STATE (engram_set_params
 * first), _UNSUPPORTED, _OOM, _CUDA.
 */
ENGRAM_API int engram_set_fp8(engram_handle *h, int32_t enable, void *stream);

/*
 * The quantiser of the FP8 projections, one row at a time: with amax the
 * largest magnitude in row r of x and E the smallest integer for which
 * amax <= 448 * 2^E (E = 0 when amax = 0), scale[r] = 2^E and
 * q[r, j] = E4M3(x[r, j] * 2^-E), rounded to the nearest E4M3 value with ties
 * to even and saturated at +-448 (E4M3: 1 sign bit, 4 exponent bits with bias
 * 7, 3 mantissa bits, no infinities, S.1111.111 NaN; zero keeps its sign).
 * x * 2^-E is exact, so the codes are a function of x alone.
 *  x      device bf16 [rows, cols], finite values, 16-byte aligned.
 *  q      device uint8 [rows, cols] E4M3 codes, 16-byte aligned.
 *  scale  device fp32 [rows], 4-byte aligned.
 * 16 <= cols <= 2048, cols a multiple of 16.  Enqueued on `stream`.
 * Errors: _INVALID, _CUDA.
 */
ENGRAM_API int engram_quantize_e4m3(engram_handle *h, const void *x, int64_t rows, int32_t cols,
                                    uint8_t *q, float *scale, void *stream);

/*
 * Pre-allocate the handle's device scratch for calls of up to `max_rows`
 * emitted positions (rows = B * (T - t_begin)).  Calls with more rows grow the
 * scratch themselves; reserving first keeps allocation out of timed or
 * captured regions.  Scratch per row: S int64 indices, d_mem gathered
 * elements, and 16 bytes per (row, key tile).  Errors: _INVALID, _OOM.
 */
ENGRAM_API int engram_reserve(engram_handle *h, int64_t max_rows);

/* Table sizes and multipliers in use: primes [S], mult [S, max(orders)] (host). */
ENGRAM_API int engram_get_hash_params(const engram_handle *h, int64_t *primes, uint64_t *mult);

/*
 * Steps 1-3 (section 2.2, Eq. 1): compress, form suffix n-grams (pad before
 * each sequence's start; n-grams never cross sequences) and hash.
 *  tokens  device int32 [B, T] raw ids.
 *  idx     device int64 [B*(T-t_begin), S]: row (b, t) for t >= t_begin.
 * 0 <= t_begin < T (decode: t_begin = T-1 emits only the newest position,
 * the earlier tokens being its history).  Errors: _INVALID, _CUDA.
 */
ENGRAM_API int engram_hash(engram_handle *h, const int32_t *tokens, int32_t B, int32_t T, int32_t t_begin,
                int64_t *idx, void *stream);

/*
 * Step 4 (Eq. 2): e[r, s*d_h:(s+1)*d_h] = table_s[idx[r, s]], bit-exact copy.
 *  idx  device int64 [rows, S], every entry in [0, primes[s]).
 *  e    device [rows, d_mem] dtype.
 * Indices outside a table set ENGRAM_ERR_BOUNDS in the device error word and
 * the row is filled with zeros instead.  Device-resident tables only.
 */
ENGRAM_API int engram_gather(engram_handle *h, const int64_t *idx, int64_t rows, void *e, void *stream);

/*
 * The whole forward (steps 1-7): out = h + alpha * (W_V e) per branch, with
 * alpha = sigmoid(RMSNorm_q(h) . RMSNorm_k(W_K e) / sqrt(d)) (Eq. 3, 4, 6).
 * At the paper's zero-initialised ShortConv (Eq. 5, Table 5) this equals the
 * module output added to the residual stream; with engram_set_short_conv the
 * convolution is applied (out = h + Y, Eq. 5).
 *  tokens  device int32 [B, T].
 *  idx     device int64 [rows, S] precomputed by engram_hash, or NULL to hash
 *          inside this call.
 *  hid     device [rows, M, d] dtype, rows = B*(T-t_begin).
 *  out     device [rows, M, d] dtype (may alias hid for an in-place update).
 *  alpha   device fp32 [rows, M] or NULL.
 *  delta   device fp32 [rows, M, d] or NULL: what is added to h (alpha * v,
 *          or Y with the short convolution).
 * With ENGRAM_PINNED_HOST tables, the rows must have been staged by
 * engram_prefetch for the same tokens; the call waits (on the stream) for
 * that prefetch.  Errors: _INVALID, _STATE, _OOM, _CUDA.
 */
ENGRAM_API int engram_forward(engram_handle *h, const int32_t *tokens, const int64_t *idx, int32_t B,
                   int32_t T, int32_t t_begin, const void *hid, void *out, float *alpha,
                   float *delta, void *stream);

/*
 * engram_forward from HOST buffers: the call copies tokens and h to device
 * staging owned by the handle (on an internal stream), runs engram_forward
 * there in place on `stream`, and copies the result to out (and alpha) on a
 * second internal stream; `stream` then waits for those copies, so work
 * issued on it after the call (a synchronise, an event) sees out.  The
 * handle keeps two stagings and alternates them, so the host-to-device copies
 * of one call overlap the device-to-host copies of the call before it: a loop
 * of calls moves both directions over PCIe at once.
 *  tokens  host int32 [B, T].
 *  hid     host [rows, M, d] dtype, rows = B*(T-t_begin); read by the call's
 *          copy, so it must stay unchanged until `stream` passes the call.
 *  out     host [rows, M, d] dtype (may be hid itself).
 *  alpha   host fp32 [rows, M] or NULL.
 * Host buffers should be pinned (cudaHostAlloc / cudaHostRegister); pageable
 * ones work but their copies do not overlap.  The staging grows on demand
 * (the call then waits for the handle's earlier copies).  Device-resident
 * tables, or host tables with a pending engram_prefetch of the same tokens.
 * Errors: _INVALID, _STATE, _OOM, _CUDA (those of engram_forward included).
 */
ENGRAM_API int engram_forward_host(engram_handle *h, const int32_t *tokens, int32_t B, int32_t T,
                        int32_t t_begin, const void *hid, void *out, float *alpha,
                        void *stream);

/*
 * Backward of engram_forward (training): the exact derivative of
 * out = h + alpha v (Eq. 3, 4, 6) for a loss whose gradient with respect to
 * out is dout, for the same tokens (or idx) and h.  The pages give only the
 * forward; per row and branch, with qn = RMSNorm_q(h), kn = RMSNorm_k(k):
 *   dalpha = dout . v, dv = sum over branches of alpha dout,
 *   ds = dalpha alpha (1 - alpha), dqn = ds kn / sqrt(d), dkn = ds qn / sqrt(d),
 *   dh = dout + (RMSNorm backward of dqn), dk = (RMSNorm backward of dkn),
 *   dW_K += dk e^T, dW_V += dv e^T, de = W_K^T dk + W_V^T dv,
 *   dtable_s[z_s] += the slot-s slice of de.
 * k and v are recomputed (the forward keeps neither).  bf16 handles round dk
 * and dv to bf16 for the GEMMs (fp32 accumulation), as bf16 training does;
 * fp32 handles keep fp32 throughout.
 *  tokens, idx  as engram_forward (idx NULL: hashed here).
 *  hid     device [rows, M, d] dtype: the forward's h.
 *  dout    device [rows, M, d] dtype.
 *  dhid    device [rows, M, d] dtype: written with dL/dh.
 *  dw_k    device fp32 [M, d, d_mem] or NULL, accumulated (+=); the sum over
 *          rows is split into parts added in an order that varies between
 *          runs (last-bit differences).
 *  dw_v    device fp32 [d, d_mem] or NULL, accumulated the same way.
 *  dnorm_q, dnorm_k  device fp32 [M, d] or NULL, accumulated.
 *  dtables host array of S device pointers (16-byte aligned) to fp32
 *          [primes[s], d_head] table gradients, accumulated (atomic adds: the
 *          order of additions
 *          into one row varies between runs); or NULL.  With row-sharded
 *          tables (engram_set_table_shards) it holds S x N pointers, table
 *          by table, shard j of table s's gradient having the rows of its
 *          table shard; row z's gradient is added into its owner's shard
 *          (a peer's memory when the shard lives on another GPU).
 * Device-resident tables, d <= 4096; not with the FP8 projections or the
 * short convolution on (ENGRAM_ERR_UNSUPPORTED).  Scratch per row: S int64,
 * (M + 1) d (4 + element size) bytes and 4 d_mem bytes, plus the forward's.
 * The dense contractions run on the library's own kernels on `stream`
 * (tcgen05 tensor-core tiles for bf16, FFMA tiles for fp32).  The first call
 * creates its scratch (engram_reserve does
 * not cover the backward's): make it outside any stream capture.
 * Errors: _INVALID, _STATE, _UNSUPPORTED, _OOM, _CUDA.
 */
ENGRAM_API int engram_backward(engram_handle *h, const int32_t *tokens, const int64_t *idx,
                               int32_t B, int32_t T, int32_t t_begin, const void *hid,
                               const void *dout, void *dhid, float *dw_k, float *dw_v,
                               float *dnorm_q, float *dnorm_k, float *const *dtables,
                               void *stream);

/*
 * engram_backward from HOST buffers, as engram_forward_host is to
 * engram_forward: tokens, h and dout are copied to device staging owned by
 * the handle (internal stream), the backward runs there on `stream`, and dh is
 * copied back (second internal stream); `stream` then waits for that copy.
 * Consecutive calls alternate two stagings, so one call's copies in overlap
 * the previous call's copy out.
 *  tokens, hid, dout  host, as engram_backward's device arguments; read by the
 *                     call's copies, unchanged until `stream` passes the call.
 *  dhid               host [rows, M, d] dtype.
 *  dw_k, dw_v, dnorm_q, dnorm_k, dtables  DEVICE buffers, as engram_backward.
 * Host buffers should be pinned.  Errors: those of engram_backward.
 */
ENGRAM_API int engram_backward_host(engram_handle *h, const int32_t *tokens, int32_t B, int32_t T,
                         int32_t t_begin, const void *hid, const void *dout, void *dhid,
                         float *dw_k, float *dw_v, float *dnorm_q, float *dnorm_k,
                         float *const *dtables, void *stream);

/*
 * Deterministic prefetch for host-resident tables (section 2.5, Figure 2b):
 * hash the tokens of an upcoming step, de-duplicate the addressed rows per
 * table, and copy each distinct row once from pinned host memory over PCIe
 * into a device staging buffer.  The hashing and de-duplication run on
 * `side_stream`; the copy follows the route engram_set_prefetch chose (by
 * default host threads and the copy engines, no SM involved).  The call
 * returns without waiting for the copy.  The next engram_forward with the
 * same tokens reads the staged rows; its stream waits for this prefetch
 * through an event (with the host-thread route, engram_forward first waits
 * on the host until the copies have been enqueued), so the transfer overlaps
 * whatever runs on other streams meanwhile.  At most two prefetches may be
 * pending (staging is double-buffered).  ENGRAM_PINNED_HOST handles only.
 * *unique_rows (host, may be NULL) receives the number of distinct rows once
 * the de-duplication has completed (this synchronises side_stream when
 * non-NULL).  Pinned host memory of the host-thread route: 2 x (16 + 8 +
 * d_head x element size) bytes per (row, table) of the largest batch.
 * Errors: _INVALID, _STATE (engram_set_params first; more than two pending),
 * _OOM, _CUDA.
 */
ENGRAM_API int engram_prefetch(engram_handle *h, const int32_t *tokens, int32_t B, int32_t T,
                    int32_t t_begin, void *side_stream, int64_t *unique_rows);

/*
 * Block the calling host thread until the rows of the oldest pending
 * prefetch (the one the next engram_forward reads) are in device memory.
 * Not needed for correctness (engram_forward orders itself after the
 * prefetch); for callers that time or schedule the transfer.
 * Errors: _STATE (no prefetch pending), _CUDA.
 */
ENGRAM_API int engram_prefetch_wait(engram_handle *h);

/*
 * The route of engram_prefetch's copy from the host tables (section 2.5: the
 * paper fetches the rows asynchronously over PCIe while earlier blocks
 * compute, but does not say how).
 *  mode  ENGRAM_PREFETCH_HOST_THREADS: `workers` host threads (0: up to 8,
 *        half the host's hardware threads) read the distinct rows into a
 *        pinned bounce buffer and the copy engines send it to the device in
 *        chunks of about 1 MB; no SM takes part, so the transfer runs beside
 *        any compute.  Random 160-byte reads from host DRAM set its rate.
 *        ENGRAM_PREFETCH_ZERO_COPY: a kernel of `workers` CTAs (0: one per SM)
 *        on side_stream loads the rows through the tables' mapped device
 *        address, 16 bytes per load; those CTAs occupy SMs for the whole
 *        transfer.
 * Both routes stage the same bytes, so results do not depend on the mode.
 * No prefetch may be pending (ENGRAM_ERR_STATE).  ENGRAM_PINNED_HOST handles
 * only.  Errors: _INVALID, _STATE.
 */
ENGRAM_API int engram_set_prefetch(engram_handle *h, int32_t mode, int32_t workers);

/*
 * Hot-row cache for host-resident tables (section 2.5: the accesses follow
 * the Zipfian n-gram statistics, so a small set of rows carries much of the
 * traffic).  Hashes the calibration tokens on `stream`, counts how often each
 * (table, row) is addressed, and copies the max_rows most frequent rows (ties:
 * lower table slot, then lower row) once from the host tables into HBM.
 * Every later engram_prefetch copies the distinct rows it needs from this
 * cache when they are there and over PCIe otherwise; results are unchanged.
 * max_rows = 0 drops the cache.  Waits for all device work first (no prefetch
 * may read the old cache) and synchronises `stream` before returning.
 * HBM used: max_rows x d_head x element size, plus 12 bytes x 2 max_rows of
 * lookup table, plus a temporary 16 bytes x 2 B (T - t_begin) S.
 * ENGRAM_PINNED_HOST handles only.  Errors: _INVALID, _STATE, _OOM, _CUDA.
 */
ENGRAM_API int engram_build_hot_cache(engram_handle *h, const int32_t *tokens, int32_t B,
                                      int32_t T, int32_t t_begin, int64_t max_rows, void *stream);

/*
 * Distinct rows of the most recent engram_prefetch that were copied from the
 * hot-row cache instead of over PCIe (host int64).  Waits for all device work.
 */
ENGRAM_API int engram_prefetch_hot_hits(engram_handle *h, int64_t *hits);

/*
 * Synchronise `stream`, then read and clear the handle's device error word.
 * Returns ENGRAM_OK, ENGRAM_ERR_BOUNDS (a token or index out of range was
 * replaced) or ENGRAM_ERR_TIMEOUT (a kernel's bounded wait expired and the
 * kernel returned early; its outputs are invalid).
 */
ENGRAM_API int engram_check_errors(engram_handle *h, void *stream);

/*
 * Stage timing for the NEXT engram_forward on this handle (one-shot).
 * `events` holds 5 or 6 cudaEvent_t (as void*), created by the caller with
 * timing enabled.  That forward records them on its stream at: start, after
 * hashing, after the gather, after the key-projection kernel, after the
 * value-projection kernel, and (6th) after the short convolution
 * (consecutive events coincide for a stage that does not run, e.g. hashing
 * when idx is given or when it is fused into the gather).  With 5 events the
 * convolution counts in the value stage.  NULL clears.
 */
ENGRAM_API int engram_profile_next_forward(engram_handle *h, void *const *events, int32_t n_events);

/*
 * Stage timing for the NEXT engram_backward on this handle (one-shot).
 * `events` holds 6 cudaEvent_t (as void*) created with timing enabled; that
 * call records them on its stream at: start, after hashing and the gather,
 * after k and v are recomputed, after the gate backward (and the RMSNorm
 * weight-gradient reduction), after the weight-gradient GEMMs, and after the
 * memory-vector GEMMs and the table-gradient scatter.  NULL clears.
 */
ENGRAM_API int engram_profile_next_backward(engram_handle *h, void *const *events,
                                            int32_t n_events);

/*
 * Self-test of device-side failure detection.  Launches on `stream` a one-CTA
 * kernel that waits on an mbarrier no thread ever arrives at, then one that
 * waits on a count in global memory that never reaches its target, with the
 * same bounded waits the tensor-core kernels use (limit 2 s each): each wait
 * expires, the kernel records a timeout in the device error word and returns
 * normally, and the word is read and cleared as engram_check_errors does.
 * Returns ENGRAM_ERR_TIMEOUT when both waits expired and were reported (the
 * mechanism works), ENGRAM_OK if one of them was not; the handle and the CUDA
 * context remain usable.
 */
ENGRAM_API int engram_selftest_timeout(engram_handle *h, void *stream);

/* Number of CUDA kernels this handle has launched since it was created. */
ENGRAM_API int64_t engram_kernel_launches(const engram_handle *h);

/*
 * Allocation-free projection + gate (steps 5-7 of engram_forward), for callers
 * that must not have the library allocate device memory: code that runs while
 * a CUDA graph is being captured (cudaMalloc cannot be captured and breaks the
 * capture), and hosts whose device memory must all come from their own
 * allocator or pool.  This call has no counterpart in the paper; it is the
 * same computation as engram_forward from the gathered memory vectors on.
 *  e      device [rows, d_mem] dtype: memory vectors, e.g. from engram_hash +
 *         engram_gather into the caller's own buffers.
 *  hid    device [rows, M, d] dtype.
 *  out    device [rows, M, d] dtype (may alias hid for the in-place update).
 *  alpha  device fp32 [rows, M] or NULL.
 * The only scratch, 16 bytes per (row, 64-column key tile) of partial sums, is
 * a fixed 4 MiB array in the library's device image (every GPU that loads the
 * library keeps it until the process exits), so rows may not exceed
 * 4 MiB / (16 * M * d / 64); larger calls fail with ENGRAM_ERR_INVALID and a
 * message that states the limit.  The first call on a device looks up that
 * array's device address (cudaGetSymbolAddress) with the handle's device
 * current; make that first call before any stream capture.  Every call on a
 * device shares the array and the next call overwrites it: calls whose work
 * overlaps on the GPU (other streams, other handles) race and must be
 * serialised by the caller.  Errors: _INVALID, _STATE, _CUDA.
 */
ENGRAM_API int engram_project_gate_noalloc(engram_handle *h, const void *e, int64_t rows,
                                           const void *hid, void *out, float *alpha,
                                           void *stream);

#ifdef __cplusplus
}
#endif

#endif /* ENGRAM_H */
