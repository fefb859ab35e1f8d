// engram_project_gate_noalloc: the projection + gate step for callers that
// must not have the library allocate device memory.
//
// engram_forward keeps its scratch (indices, memory vectors, per-row partial
// sums) in buffers the handle allocates on demand.  Some callers cannot allow
// that: code that runs while a CUDA graph is being captured (cudaMalloc is
// not a capturable operation and fails the capture), and hosts whose device
// memory must all come from their own allocator or pool budget.  With this
// entry point such a caller supplies every input and output itself (it can
// produce e with engram_hash and engram_gather into its own buffers), and the
// only scratch, the key phase's per-row partial sums, lives in a fixed array
// in the library's device image.
#include <cmath>
#include <mutex>
#include <string>

#include "engram_handle.cuh"

using namespace engram;

namespace {

// Size of the partial-sum array: 16 bytes per (row, 64-column key tile).
constexpr size_t kNoAllocScratchBytes = size_t(4) << 20;  // 4 MiB

}  // namespace

// Every GPU that loads the library holds this array until the process exits.
// All calls on a device share it: calls that overlap on the GPU race.
static __device__ __align__(256) unsigned char g_noalloc_partials[kNoAllocScratchBytes];

namespace {

constexpr int kMaxDevices = 256;
std::mutex g_mu;
void* g_partials_dev[kMaxDevices] = {};

int fail(engram_handle* h, int code, const std::string& msg) {
  h->last_error = msg;
  return code;
}

// Device address of the array on the current device, looked up once per
// device with that device current.  In host code the array's name is only a
// host-side stand-in, never a device address.
int partials_address(engram_handle* h, float4** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(h, ENGRAM_ERR_CUDA, cudaGetErrorString(e));
  if (dev != h->device) return fail(h, ENGRAM_ERR_INVALID, "the handle's device must be current");
  if (dev < 0 || dev >= kMaxDevices) return fail(h, ENGRAM_ERR_INVALID, "device id out of range");
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_partials_dev[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_partials);
    if (e != cudaSuccess || !p)
      return fail(h, ENGRAM_ERR_CUDA,
                  std::string("cudaGetSymbolAddress: ") + cudaGetErrorString(e));
    g_partials_dev[dev] = p;
  }
  *out = reinterpret_cast<float4*>(g_partials_dev[dev]);
  return ENGRAM_OK;
}

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

}  // namespace

extern "C" int engram_project_gate_noalloc(engram_handle* h, const void* e, int64_t rows,
                                           const void* hid, void* out, float* alpha,
                                           void* stream) {
  if (!h) return ENGRAM_ERR_INVALID;
  if (!h->have_params) return fail(h, ENGRAM_ERR_STATE, "engram_set_params first");
  if (h->fp8)
    return fail(h, ENGRAM_ERR_UNSUPPORTED,
                "engram_project_gate_noalloc: FP8 projections are on; use engram_forward");
  if (h->conv_W > 0)
    return fail(h, ENGRAM_ERR_UNSUPPORTED,
                "engram_project_gate_noalloc: the short convolution needs scratch; use engram_forward");
  const int M = h->cfg.branches, d = h->cfg.d_hidden;
  const int64_t bytes_per_row = (int64_t)(M * d / 64) * (int64_t)sizeof(float4);
  const int64_t max_rows = (int64_t)kNoAllocScratchBytes / bytes_per_row;
  if (rows < 0) return fail(h, ENGRAM_ERR_INVALID, "rows < 0");
  if (rows > max_rows)
    return fail(h, ENGRAM_ERR_INVALID,
                "engram_project_gate_noalloc: " + std::to_string(rows) + " rows exceed the " +
                    std::to_string(max_rows) + "-row limit of its fixed 4 MiB scratch (" +
                    std::to_string(bytes_per_row) + " bytes per row); use engram_forward");
  if (rows == 0) return ENGRAM_OK;
  if (!e || !hid || !out || !aligned16(e) || !aligned16(hid) || !aligned16(out) ||
      (alpha && !aligned16(alpha)))
    return fail(h, ENGRAM_ERR_INVALID, "null or misaligned buffer");
  float4* partials = nullptr;
  int rc = partials_address(h, &partials);
  if (rc) return rc;
  cudaStream_t st = (cudaStream_t)stream;
  const int R = (int)rows;

  // Every (row, key tile) entry the value phase reads is written by the key
  // phase of the same call, so the array needs no clearing between calls.
  GateArgs g{};
  g.h = hid;
  g.out = out;
  g.w_qk = h->d_wqk;
  g.partials = partials;
  g.alpha = alpha;
  g.delta = nullptr;
  g.err = h->d_err;
  g.R = R;
  g.M = M;
  g.d = d;
  g.d_mem = h->d_mem;
  g.eps = h->cfg.eps;
  g.inv_sqrt_d = (float)(1.0 / std::sqrt((double)d));
  cudaError_t ce;
  if (h->cfg.dtype == ENGRAM_F32) {
    g.key_tile = kF32Tile;
    if ((ce = launch_proj_gate_f32(0, (const float*)e, (const float*)h->w_k, g, st)) ||
        (ce = launch_proj_gate_f32(1, (const float*)e, (const float*)h->w_v, g, st)))
      return fail(h, ENGRAM_ERR_CUDA, cudaGetErrorString(ce));
    h->launches += 2;
    return ENGRAM_OK;
  }
  // the same kernel choice as engram_forward (choose_proj)
  const int64_t hcols = (int64_t)M * d;
  ProjMaps single, wide, pair;
  bool have_single = false, have_wide = false, have_pair = false;
  for (int phase = 0; phase < 2; ++phase) {
    const CUtensorMap* wmaps = phase == 0 ? h->map_wk : h->map_wv;
    const ProjChoice pc = choose_proj(phase, rows, M, d, h->sms, h->cfg.flags);
    if (phase == 0) g.key_tile = pc.key_tile;
    const int kphase = (phase == 1 && out == hid) ? 2 : phase;
    if (pc.kind == ProjKernel::Pair) {
      if (!have_pair) {
        if ((rc = make_map(h, &pair.e, e, h->d_mem, R, 128, 64)) ||
            (rc = make_map(h, &pair.h, hid, hcols, R, 128, 32)) ||
            (rc = make_map(h, &pair.out, out, hcols, R, 32, 32)))
          return rc;
        have_pair = true;
      }
      pair.w = wmaps[bn_index(pc.bn)];
      ProjMaps pm = pair;
      // in place: per-warp reduce-adds of 32 rows x 64 columns
      if (kphase == 2 && (rc = make_map(h, &pm.out, out, hcols, R, 32, 64))) return rc;
      if ((ce = launch_proj_gate_pair(kphase, pm, g, pc.grid, st)))
        return fail(h, ENGRAM_ERR_CUDA, cudaGetErrorString(ce));
    } else if (pc.kind == ProjKernel::Wide) {
      if (!have_wide) {
        if ((rc = make_map(h, &wide.e, e, h->d_mem, R, 256, 64)) ||
            (rc = make_map(h, &wide.h, hid, hcols, R, 256, 32)) ||
            (rc = make_map(h, &wide.out, out, hcols, R, 32, 32)))
          return rc;
        have_wide = true;
      }
      wide.w = wmaps[bn_index(pc.bn)];
      ProjMaps wl = wide;
      // in place: per-warp reduce-adds of 32 rows x 64 columns
      if (kphase == 2 && (rc = make_map(h, &wl.out, out, hcols, R, 32, 64))) return rc;
      if ((ce = launch_proj_gate_wide(kphase, wl, g, pc.grid, st)))
        return fail(h, ENGRAM_ERR_CUDA, cudaGetErrorString(ce));
    } else {
      if (!have_single) {
        if ((rc = make_map(h, &single.e, e, h->d_mem, R, 128, 64)) ||
            (rc = make_map(h, &single.h, hid, hcols, R, 128, 64)) ||
            (rc = make_map(h, &single.out, out, hcols, R, 32, 64)))
          return rc;
        have_single = true;
      }
      single.w = wmaps[bn_index(pc.bn)];
      if ((ce = launch_proj_gate_sm100(phase, pc.bn, single, g, pc.grid, st)))
        return fail(h, ENGRAM_ERR_CUDA, cudaGetErrorString(ce));
    }
  }
  h->launches += 2;
  return ENGRAM_OK;
}
