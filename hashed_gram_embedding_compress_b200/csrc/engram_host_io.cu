// engram_forward_host: the forward from host buffers.
//
// The call stages tokens and h in one of two device buffers with
// host-to-device copies on its own stream, runs engram_forward in place on
// that staging (on the caller's stream), and copies out (and alpha) back with
// device-to-host copies on a second stream; the caller's stream then waits for
// those copies, so everything after the call on that stream sees out.  The
// two staging buffers alternate between calls, so call i + 1's host-to-device
// copies run while call i's results travel back: over PCIe, which carries
// both directions at once, a loop of calls takes about one direction's copy
// time per call instead of both.
#include <cuda_runtime.h>

#include <cstdint>
#include <string>

#include "engram.h"
#include "engram_handle.cuh"

namespace engram {

namespace {

int io_fail(engram_handle* h, int code, const std::string& msg) {
  h->last_error = msg;
  return code;
}

#define IO_CK(h, expr)                                                              \
  do {                                                                              \
    const cudaError_t e_ = (expr);                                                  \
    if (e_ != cudaSuccess)                                                          \
      return io_fail(h, e_ == cudaErrorMemoryAllocation ? ENGRAM_ERR_OOM : ENGRAM_ERR_CUDA, \
                     std::string(#expr) + ": " + cudaGetErrorString(e_));           \
  } while (0)

// Streams and events on first use; staging at least the given sizes.  Before a
// buffer is replaced every earlier call's copies and forward have finished:
// the output stream's last copy waited for that call's forward.
int ensure_io(engram_handle* h, size_t h_bytes, size_t tok_bytes, size_t alpha_bytes) {
  if (!h->io_in) {
    IO_CK(h, cudaStreamCreateWithFlags(&h->io_in, cudaStreamNonBlocking));
    IO_CK(h, cudaStreamCreateWithFlags(&h->io_out, cudaStreamNonBlocking));
    for (int i = 0; i < 2; ++i) {
      IO_CK(h, cudaEventCreateWithFlags(&h->io_ev_in[i], cudaEventDisableTiming));
      IO_CK(h, cudaEventCreateWithFlags(&h->io_ev_comp[i], cudaEventDisableTiming));
      IO_CK(h, cudaEventCreateWithFlags(&h->io_ev_out[i], cudaEventDisableTiming));
    }
  }
  if (h_bytes > h->io_h_bytes || tok_bytes > h->io_tok_bytes || alpha_bytes > h->io_alpha_bytes) {
    IO_CK(h, cudaStreamSynchronize(h->io_in));
    IO_CK(h, cudaStreamSynchronize(h->io_out));
    for (int i = 0; i < 2; ++i) {
      if (h_bytes > h->io_h_bytes) {
        cudaFree(h->io_h[i]);
        h->io_h[i] = nullptr;
      }
      if (tok_bytes > h->io_tok_bytes) {
        cudaFree(h->io_tok[i]);
        h->io_tok[i] = nullptr;
      }
      if (alpha_bytes > h->io_alpha_bytes) {
        cudaFree(h->io_alpha[i]);
        h->io_alpha[i] = nullptr;
      }
    }
    if (h_bytes > h->io_h_bytes) {
      h->io_h_bytes = 0;
      for (int i = 0; i < 2; ++i) IO_CK(h, cudaMalloc(&h->io_h[i], h_bytes));
      h->io_h_bytes = h_bytes;
    }
    if (tok_bytes > h->io_tok_bytes) {
      h->io_tok_bytes = 0;
      for (int i = 0; i < 2; ++i) IO_CK(h, cudaMalloc(&h->io_tok[i], tok_bytes));
      h->io_tok_bytes = tok_bytes;
    }
    if (alpha_bytes > h->io_alpha_bytes) {
      h->io_alpha_bytes = 0;
      for (int i = 0; i < 2; ++i) IO_CK(h, cudaMalloc(&h->io_alpha[i], alpha_bytes));
      h->io_alpha_bytes = alpha_bytes;
    }
  }
  return ENGRAM_OK;
}

// The backward's stagings (h, dout, dh of rows x M x d; tokens), grown as
// ensure_io grows the forward's.
int ensure_bio(engram_handle* h, size_t bytes, size_t tok_bytes) {
  int rc = ensure_io(h, 0, 0, 0);  // streams and events
  if (rc) return rc;
  if (bytes > h->bio_bytes || tok_bytes > h->bio_tok_bytes) {
    IO_CK(h, cudaStreamSynchronize(h->io_in));
    IO_CK(h, cudaStreamSynchronize(h->io_out));
    if (bytes > h->bio_bytes) {
      h->bio_bytes = 0;
      for (int i = 0; i < 2; ++i) {
        for (void** b : {&h->bio_h[i], &h->bio_dout[i], &h->bio_dh[i]}) {
          cudaFree(*b);
          *b = nullptr;
          IO_CK(h, cudaMalloc(b, bytes));
        }
      }
      h->bio_bytes = bytes;
    }
    if (tok_bytes > h->bio_tok_bytes) {
      h->bio_tok_bytes = 0;
      for (int i = 0; i < 2; ++i) {
        cudaFree(h->bio_tok[i]);
        h->bio_tok[i] = nullptr;
        IO_CK(h, cudaMalloc(&h->bio_tok[i], tok_bytes));
      }
      h->bio_tok_bytes = tok_bytes;
    }
  }
  return ENGRAM_OK;
}

}  // namespace

void free_host_io(engram_handle* h) {
  for (int i = 0; i < 2; ++i) {
    for (void** b : {&h->bio_h[i], &h->bio_dout[i], &h->bio_dh[i]}) {
      cudaFree(*b);
      *b = nullptr;
    }
    cudaFree(h->bio_tok[i]);
    h->bio_tok[i] = nullptr;
  }
  h->bio_bytes = h->bio_tok_bytes = 0;
  for (int i = 0; i < 2; ++i) {
    cudaFree(h->io_h[i]);
    cudaFree(h->io_tok[i]);
    cudaFree(h->io_alpha[i]);
    h->io_h[i] = nullptr;
    h->io_tok[i] = nullptr;
    h->io_alpha[i] = nullptr;
    if (h->io_ev_in[i]) cudaEventDestroy(h->io_ev_in[i]);
    if (h->io_ev_comp[i]) cudaEventDestroy(h->io_ev_comp[i]);
    if (h->io_ev_out[i]) cudaEventDestroy(h->io_ev_out[i]);
    h->io_ev_in[i] = h->io_ev_comp[i] = h->io_ev_out[i] = nullptr;
  }
  if (h->io_in) cudaStreamDestroy(h->io_in);
  if (h->io_out) cudaStreamDestroy(h->io_out);
  h->io_in = h->io_out = nullptr;
  h->io_h_bytes = h->io_tok_bytes = h->io_alpha_bytes = 0;
}

}  // namespace engram

int engram_forward_host(engram_handle* h, const int32_t* tokens, int32_t B, int32_t T,
                        int32_t t_begin, const void* hid, void* out, float* alpha,
                        void* stream) {
  using namespace engram;
  if (!h) return ENGRAM_ERR_INVALID;
  if (!tokens || !hid || !out)
    return io_fail(h, ENGRAM_ERR_INVALID, "engram_forward_host: tokens, h and out must be non-null");
  if (B < 0 || T <= 0 || t_begin < 0 || t_begin >= T)
    return io_fail(h, ENGRAM_ERR_INVALID, "engram_forward_host: need B >= 0 and 0 <= t_begin < T");
  const int64_t R = (int64_t)B * (T - t_begin);
  if (R == 0) return ENGRAM_OK;
  const size_t h_bytes = (size_t)R * h->cfg.branches * h->cfg.d_hidden * h->elt;
  const size_t tok_bytes = (size_t)B * T * sizeof(int32_t);
  const size_t alpha_bytes = alpha ? (size_t)R * h->cfg.branches * sizeof(float) : 0;
  int rc = ensure_io(h, h_bytes, tok_bytes, alpha_bytes);
  if (rc) return rc;
  const int slot = h->io_flip;
  h->io_flip ^= 1;
  cudaStream_t st = (cudaStream_t)stream;
  // the staging of `slot` is free once the call before the previous one has
  // copied its results out (an event not yet recorded is complete)
  IO_CK(h, cudaStreamWaitEvent(h->io_in, h->io_ev_out[slot], 0));
  IO_CK(h, cudaMemcpyAsync(h->io_tok[slot], tokens, tok_bytes, cudaMemcpyHostToDevice, h->io_in));
  IO_CK(h, cudaMemcpyAsync(h->io_h[slot], hid, h_bytes, cudaMemcpyHostToDevice, h->io_in));
  IO_CK(h, cudaEventRecord(h->io_ev_in[slot], h->io_in));
  IO_CK(h, cudaStreamWaitEvent(st, h->io_ev_in[slot], 0));
  rc = engram_forward(h, h->io_tok[slot], nullptr, B, T, t_begin, h->io_h[slot], h->io_h[slot],
                      alpha ? h->io_alpha[slot] : nullptr, nullptr, stream);
  if (rc) return rc;
  IO_CK(h, cudaEventRecord(h->io_ev_comp[slot], st));
  IO_CK(h, cudaStreamWaitEvent(h->io_out, h->io_ev_comp[slot], 0));
  IO_CK(h, cudaMemcpyAsync(out, h->io_h[slot], h_bytes, cudaMemcpyDeviceToHost, h->io_out));
  if (alpha)
    IO_CK(h, cudaMemcpyAsync(alpha, h->io_alpha[slot], alpha_bytes, cudaMemcpyDeviceToHost,
                             h->io_out));
  IO_CK(h, cudaEventRecord(h->io_ev_out[slot], h->io_out));
  // work after this call on `stream` sees out (and alpha)
  IO_CK(h, cudaStreamWaitEvent(st, h->io_ev_out[slot], 0));
  return ENGRAM_OK;
}

int engram_backward_host(engram_handle* h, const int32_t* tokens, int32_t B, int32_t T,
                         int32_t t_begin, const void* hid, const void* dout, void* dhid,
                         float* dw_k, float* dw_v, float* dnorm_q, float* dnorm_k,
                         float* const* dtables, void* stream) {
  using namespace engram;
  if (!h) return ENGRAM_ERR_INVALID;
  if (!tokens || !hid || !dout || !dhid)
    return io_fail(h, ENGRAM_ERR_INVALID,
                   "engram_backward_host: tokens, h, dout and dh must be non-null");
  if (B < 0 || T <= 0 || t_begin < 0 || t_begin >= T)
    return io_fail(h, ENGRAM_ERR_INVALID, "engram_backward_host: need B >= 0 and 0 <= t_begin < T");
  const int64_t R = (int64_t)B * (T - t_begin);
  if (R == 0) return ENGRAM_OK;
  const size_t bytes = (size_t)R * h->cfg.branches * h->cfg.d_hidden * h->elt;
  const size_t tok_bytes = (size_t)B * T * sizeof(int32_t);
  int rc = ensure_bio(h, bytes, tok_bytes);
  if (rc) return rc;
  const int slot = h->io_flip;
  h->io_flip ^= 1;
  cudaStream_t st = (cudaStream_t)stream;
  IO_CK(h, cudaStreamWaitEvent(h->io_in, h->io_ev_out[slot], 0));
  IO_CK(h, cudaMemcpyAsync(h->bio_tok[slot], tokens, tok_bytes, cudaMemcpyHostToDevice, h->io_in));
  IO_CK(h, cudaMemcpyAsync(h->bio_h[slot], hid, bytes, cudaMemcpyHostToDevice, h->io_in));
  IO_CK(h, cudaMemcpyAsync(h->bio_dout[slot], dout, bytes, cudaMemcpyHostToDevice, h->io_in));
  IO_CK(h, cudaEventRecord(h->io_ev_in[slot], h->io_in));
  IO_CK(h, cudaStreamWaitEvent(st, h->io_ev_in[slot], 0));
  rc = engram_backward(h, h->bio_tok[slot], nullptr, B, T, t_begin, h->bio_h[slot],
                       h->bio_dout[slot], h->bio_dh[slot], dw_k, dw_v, dnorm_q, dnorm_k, dtables,
                       stream);
  if (rc) return rc;
  IO_CK(h, cudaEventRecord(h->io_ev_comp[slot], st));
  IO_CK(h, cudaStreamWaitEvent(h->io_out, h->io_ev_comp[slot], 0));
  IO_CK(h, cudaMemcpyAsync(dhid, h->bio_dh[slot], bytes, cudaMemcpyDeviceToHost, h->io_out));
  IO_CK(h, cudaEventRecord(h->io_ev_out[slot], h->io_out));
  // work after this call on `stream` sees dh
  IO_CK(h, cudaStreamWaitEvent(st, h->io_ev_out[slot], 0));
  return ENGRAM_OK;
}
