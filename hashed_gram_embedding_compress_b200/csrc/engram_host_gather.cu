// Host-thread route of the offload prefetch: see host_gather.cuh.
//
// A coordinator thread takes jobs in order.  For each it waits until the
// list of distinct rows has reached host memory, then hands out chunks of
// about 1 MB of rows to the reader threads.  A reader copies its chunk's rows
// (random 160-byte reads from the pinned tables, a few rows of prefetch
// ahead) into the bounce buffer and enqueues the chunk's host-to-device copy
// at once, so the copy engines work while the other chunks are read.  When
// every chunk is enqueued the coordinator records the job's done event after
// them on the copy stream.
#include <algorithm>
#include <cstring>

#include "host_gather.cuh"

namespace engram {

namespace {

constexpr int64_t kChunkBytes = int64_t(1) << 20;
constexpr int kPrefetchAhead = 8;  // rows

}  // namespace

HostGather::HostGather(int device, int threads) : device_(device) {
  coordinator_ = std::thread([this] { coordinate(); });
  for (int i = 0; i < std::max(1, threads); ++i) readers_.emplace_back([this, i] { read_rows(i); });
}

HostGather::~HostGather() {
  {
    std::lock_guard<std::mutex> lk(mu_);
    stop_ = true;
  }
  cv_.notify_all();
  coordinator_.join();  // it finishes every queued job first
  {
    std::lock_guard<std::mutex> lk(mu_);
    readers_stop_ = true;
  }
  cv_.notify_all();
  for (auto& t : readers_) t.join();
}

void HostGather::submit(const HostGatherJob& job) {
  {
    std::lock_guard<std::mutex> lk(mu_);
    queue_.push_back(job);
    ++submitted_[job.slot & 1];
  }
  cv_.notify_all();
}

cudaError_t HostGather::wait_issued(int slot, std::string* msg) {
  std::unique_lock<std::mutex> lk(mu_);
  cv_.wait(lk, [&] { return issued_[slot & 1] == submitted_[slot & 1]; });
  if (msg) *msg = error_msg_;
  const cudaError_t e = error_;
  error_ = cudaSuccess;
  error_msg_.clear();
  return e;
}

void HostGather::note_error(cudaError_t e, const char* what) {
  // caller holds mu_
  if (e != cudaSuccess && error_ == cudaSuccess) {
    error_ = e;
    error_msg_ = std::string(what) + ": " + cudaGetErrorString(e);
  }
}

void HostGather::coordinate() {
  cudaSetDevice(device_);
  for (;;) {
    HostGatherJob job;
    {
      std::unique_lock<std::mutex> lk(mu_);
      cv_.wait(lk, [&] { return stop_ || !queue_.empty(); });
      if (queue_.empty()) return;  // stopping, and every job is done
      job = queue_.front();
      queue_.pop_front();
    }
    run(job);
    {
      std::lock_guard<std::mutex> lk(mu_);
      ++issued_[job.slot & 1];
    }
    cv_.notify_all();
  }
}

void HostGather::run(const HostGatherJob& job) {
  const cudaError_t e = cudaEventSynchronize(job.idx_ready);
  const int64_t n = e == cudaSuccess ? (int64_t)job.count[0] : 0;
  {
    std::unique_lock<std::mutex> lk(mu_);
    note_error(e, "waiting for the prefetch's row list");
    cur_ = job;
    n_rows_ = n;
    chunk_rows_ = std::max<int64_t>(1, kChunkBytes / std::max<int64_t>(1, job.row_bytes));
    n_chunks_ = (n + chunk_rows_ - 1) / chunk_rows_;
    next_chunk_ = 0;
    chunks_done_ = 0;
    have_job_ = n_chunks_ > 0;
  }
  cv_.notify_all();
  {
    std::unique_lock<std::mutex> lk(mu_);
    cv_.wait(lk, [&] { return chunks_done_ == n_chunks_; });
    have_job_ = false;
  }
  // after every chunk's copy on the copy stream (enqueued by the readers)
  const cudaError_t r = cudaEventRecord(job.done, job.copy_stream);
  std::lock_guard<std::mutex> lk(mu_);
  note_error(r, "recording the prefetch's done event");
}

void HostGather::read_rows(int) {
  cudaSetDevice(device_);
  for (;;) {
    HostGatherJob job;
    int64_t a = 0, b = 0;
    {
      std::unique_lock<std::mutex> lk(mu_);
      cv_.wait(lk, [&] { return readers_stop_ || (have_job_ && next_chunk_ < n_chunks_); });
      if (!(have_job_ && next_chunk_ < n_chunks_)) return;  // stopping
      job = cur_;
      a = next_chunk_++ * chunk_rows_;
      b = std::min(n_rows_, a + chunk_rows_);
    }
    const int64_t rb = job.row_bytes;
    for (int64_t u = a; u < b; ++u) {
      if (u + kPrefetchAhead < b) {
        const int2 q = job.list[u + kPrefetchAhead];
        const char* p = (const char*)job.tables[q.x] + (int64_t)q.y * rb;
        for (int64_t o = 0; o < rb; o += 64) __builtin_prefetch(p + o);
        __builtin_prefetch(p + rb - 1);
      }
      const int2 q = job.list[u];
      std::memcpy(job.bounce + u * rb, (const char*)job.tables[q.x] + (int64_t)q.y * rb, (size_t)rb);
    }
    const cudaError_t e = cudaMemcpyAsync(job.staging + a * rb, job.bounce + a * rb,
                                          (size_t)((b - a) * rb), cudaMemcpyHostToDevice,
                                          job.copy_stream);
    {
      std::lock_guard<std::mutex> lk(mu_);
      note_error(e, "host-to-device copy of prefetched rows");
      ++chunks_done_;
    }
    cv_.notify_all();
  }
}

}  // namespace engram
