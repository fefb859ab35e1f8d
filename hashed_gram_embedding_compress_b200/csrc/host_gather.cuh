// Host-thread route of the offload prefetch (step 5, "Conditional Memory via
// Scalable Lookup", section 2.5 and Figure 2(b)): the distinct rows of the
// next step are read by host threads from the pinned host tables into a
// pinned bounce buffer, and the copy engines move the buffer into the HBM
// staging buffer in large copies.  No SM takes part, so the transfer runs
// beside whatever the GPU computes meanwhile.  Internal to libengram.so.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <condition_variable>
#include <deque>
#include <mutex>
#include <string>
#include <thread>
#include <vector>

namespace engram {

// One prefetch's transfer.  Every pointer stays valid until the job has
// finished (wait_issued, then the done event).
struct HostGatherJob {
  int slot = 0;                            // 0 or 1: the staging slot
  cudaEvent_t idx_ready = nullptr;         // after the copy of count and the list to the host
  const unsigned long long* count = nullptr;  // pinned: [0] rows to read
  const int2* list = nullptr;              // pinned [count[0]]: (table s, row z) per slot
  const void* const* tables = nullptr;     // host [S]: table base pointers
  int64_t row_bytes = 0;
  char* bounce = nullptr;                  // pinned [rows, row_bytes]
  char* staging = nullptr;                 // device [rows, row_bytes]
  cudaStream_t copy_stream = nullptr;
  cudaEvent_t done = nullptr;              // recorded on copy_stream after the last copy
};

class HostGather {
 public:
  // `threads` readers (>= 1) and one coordinator thread, all on `device`.
  HostGather(int device, int threads);
  // Waits for queued jobs, then joins every thread.
  ~HostGather();
  HostGather(const HostGather&) = delete;
  HostGather& operator=(const HostGather&) = delete;

  // Queue a job (first in, first out).  Returns at once.
  void submit(const HostGatherJob& job);
  // Block until every job submitted so far for `slot` has enqueued all its
  // copies and recorded its done event.  Returns the first CUDA error a job
  // met (the message in *msg), or cudaSuccess.
  cudaError_t wait_issued(int slot, std::string* msg);
  int threads() const { return (int)readers_.size(); }

 private:
  void coordinate();
  void read_rows(int worker);
  void run(const HostGatherJob& job);
  void note_error(cudaError_t e, const char* what);  // with mu_ held

  int device_;
  std::mutex mu_;
  std::condition_variable cv_;       // job queue, job completion, reader chunks
  std::deque<HostGatherJob> queue_;
  uint64_t submitted_[2] = {0, 0}, issued_[2] = {0, 0};
  bool stop_ = false, readers_stop_ = false;
  cudaError_t error_ = cudaSuccess;  // first error since the last wait_issued
  std::string error_msg_;

  // the job being read: chunks of rows handed out to the readers
  HostGatherJob cur_;
  bool have_job_ = false;
  int64_t n_rows_ = 0, chunk_rows_ = 0, n_chunks_ = 0;
  int64_t next_chunk_ = 0, chunks_done_ = 0;
  std::thread coordinator_;
  std::vector<std::thread> readers_;
};

}  // namespace engram
