// Disk tier of the layer stream: per-layer shard files read ahead into a ring
// of host staging buffers (Soup pages, "how layer streaming works" and the
// streaming configuration keys: `stream_source: disk` reads the frozen base
// from NVMe when host RAM cannot hold it; `stream_read_ahead` (1..8) sets how
// many layers are read ahead, each step of it one more layer of page-locked
// RAM).
//
// The reader walks the training step's layer visit order (a cyclic schedule
// set by the caller) and reads only the visits that will need a host->device
// copy: it replays the device slot ring (n_slots slots, least recently used
// first, the policy of the stream plan) over the schedule, so a visit whose
// layer is still in one of the last n_slots distinct layers visited (the
// turn-arounds of the forward and backward passes) is not read.  Each read is
// cut into chunks that a pool of I/O threads reads in parallel (queue depth
// for NVMe).  A consumer acquires the staging buffer of its next copied visit,
// enqueues the device copy from it, records the buffer's copy-done event on
// the copy stream and releases it; the buffer is refilled only after that
// event has completed.  If the consumer deviates from the schedule, visits it
// passes over are dropped (counted as skipped) and results stay correct.
#include <fcntl.h>
#include <sys/stat.h>
#include <unistd.h>

#include <algorithm>
#include <cerrno>
#include <chrono>
#include <condition_variable>
#include <cstdlib>
#include <cstring>
#include <deque>
#include <mutex>
#include <string>
#include <thread>
#include <vector>

#include "soup_internal.h"

namespace {

constexpr size_t kChunk = 8u << 20;  // bytes per I/O request
constexpr size_t kPage = 4096;       // staging buffers and O_DIRECT requests are page-aligned

enum BufState { B_FREE, B_READING, B_READY, B_HELD, B_DRAINING };

struct Buf {
  char* host = nullptr;
  cudaEvent_t done = nullptr;  // copy out of this buffer complete (pinned mode)
  BufState state = B_FREE;
  long long pos = -1;          // schedule position (unrolled) being read / held
  int layer = -1;
  int pending = 0;             // chunks still being read
  bool discard = false;        // the consumer passed this visit over
  bool err = false;
  std::string msg;
  std::chrono::steady_clock::time_point t0;
};

struct Visit {
  long long pos;
  int layer;
  int buf;  // staging buffer holding this copied visit
};

struct Job {
  int buf;
  long long pos;
  size_t off, len;
};

}  // namespace

struct soup_disk {
  int n_layers = 0;
  size_t layer_bytes = 0, buf_bytes = 0;
  std::vector<int> fds;
  std::vector<bool> direct;
  bool pinned = false;
  int device = 0;
  int n_slots = 2;
  std::vector<Buf> bufs;
  // schedule and the read cursor's replay of the slot ring
  std::vector<int> order;
  long long next_read = 0;
  std::deque<int> ring;       // last n_slots distinct layers visited, least recent first
  std::deque<Visit> window;   // copied visits read (or being read), not yet acquired, in order
  bool exhausted = false;     // a whole cycle without a copied visit: nothing to read ever
  long long force_pos = -1;   // a visit read even if the replayed ring holds its layer (resync)
  // I/O
  std::deque<Job> jobs;
  std::vector<std::thread> io;
  std::mutex mu;
  std::condition_variable cv_io, cv_ready;
  bool stop = false;
  // statistics
  long long reads = 0, skipped = 0, acquires = 0;
  unsigned long long bytes_read = 0;
  double read_ms = 0, wait_ms = 0;
};

namespace {

using soup::fail;

bool ring_has(const soup_disk* d, int layer) {
  return std::find(d->ring.begin(), d->ring.end(), layer) != d->ring.end();
}

void ring_touch(soup_disk* d, int layer) {
  auto it = std::find(d->ring.begin(), d->ring.end(), layer);
  if (it != d->ring.end()) d->ring.erase(it);
  d->ring.push_back(layer);
  while ((int)d->ring.size() > d->n_slots) d->ring.pop_front();
}

// Returns buffers whose copy-out has completed to the free list and starts
// reads into free buffers along the schedule.  Caller holds d->mu.
void pump(soup_disk* d) {
  for (auto& b : d->bufs) {
    if (b.state != B_DRAINING) continue;
    if (!b.done) {
      b.state = B_FREE;
      continue;
    }
    const cudaError_t q = cudaEventQuery(b.done);
    if (q == cudaSuccess) {
      b.state = B_FREE;
    } else if (q != cudaErrorNotReady) {
      b.state = B_FREE;  // the copy failed; the consumer sees the CUDA error on its own stream
      cudaGetLastError();
    }
  }
  if (d->order.empty() || d->exhausted) return;
  for (int bi = 0; bi < (int)d->bufs.size(); ++bi) {
    Buf& b = d->bufs[bi];
    if (b.state != B_FREE) continue;
    // advance the read cursor to the next visit that needs a copy
    const long long n = (long long)d->order.size();
    long long scanned = 0;
    int layer = -1;
    while (true) {
      const int l = d->order[d->next_read % n];
      const bool copy = !ring_has(d, l) || d->next_read == d->force_pos;
      ring_touch(d, l);
      ++d->next_read;
      if (copy) {
        layer = l;
        break;
      }
      if (++scanned >= n) {  // every layer stays resident: no copies after the first cycle
        d->exhausted = true;
        break;
      }
    }
    if (layer < 0) break;  // exhausted; the reads queued above still need the wake-up below
    b.state = B_READING;
    b.pos = d->next_read - 1;
    b.layer = layer;
    b.discard = false;
    b.err = false;
    b.msg.clear();
    b.t0 = std::chrono::steady_clock::now();
    b.pending = 0;
    for (size_t off = 0; off < d->layer_bytes; off += kChunk) {
      d->jobs.push_back(Job{bi, b.pos, off, std::min(kChunk, d->layer_bytes - off)});
      ++b.pending;
    }
    d->window.push_back(Visit{b.pos, layer, bi});
  }
  d->cv_io.notify_all();
}

bool any_draining(const soup_disk* d) {
  for (const auto& b : d->bufs)
    if (b.state == B_DRAINING) return true;
  return false;
}

// Reads [off, off + len) of layer `layer`'s shard into dst.  Returns "" or an error message.
std::string read_range(soup_disk* d, int layer, char* dst, size_t off, size_t len) {
  const int fd = d->fds[layer];
  size_t want = len;
  if (d->direct[layer]) want = (len + kPage - 1) / kPage * kPage;  // O_DIRECT: whole pages (stops at EOF)
  size_t got = 0;
  while (got < len) {
    const ssize_t r = pread(fd, dst + got, want - got, (off_t)(off + got));
    if (r < 0) {
      if (errno == EINTR) continue;
      return std::string("read failed: ") + strerror(errno);
    }
    if (r == 0) return "unexpected end of file";
    got += (size_t)r;
  }
  return "";
}

void io_main(soup_disk* d) {
  if (d->pinned) cudaSetDevice(d->device);
  std::unique_lock<std::mutex> lk(d->mu);
  while (true) {
    if (d->stop) return;
    if (d->jobs.empty()) {
      if (any_draining(d)) {
        d->cv_io.wait_for(lk, std::chrono::microseconds(200));
        pump(d);
        d->cv_ready.notify_all();
      } else {
        d->cv_io.wait(lk);
      }
      continue;
    }
    Job j = d->jobs.front();
    d->jobs.pop_front();
    Buf& b = d->bufs[j.buf];
    std::string err;
    if (!(b.discard && b.pos == j.pos)) {
      char* dst = b.host + j.off;
      const int layer = b.layer;
      lk.unlock();
      err = read_range(d, layer, dst, j.off, j.len);
      lk.lock();
    }
    if (!err.empty() && !b.err) {
      b.err = true;
      b.msg = err;
    }
    if (--b.pending == 0) {
      if (b.discard) {
        b.state = B_FREE;
        b.discard = false;
      } else {
        b.state = B_READY;
        ++d->reads;
        d->bytes_read += d->layer_bytes;
        d->read_ms += std::chrono::duration<double, std::milli>(std::chrono::steady_clock::now() - b.t0).count();
      }
      pump(d);
      d->cv_ready.notify_all();
    }
  }
}

// Drops visits the consumer passed over: window entries before index k.
void drop_before(soup_disk* d, size_t k) {
  for (size_t i = 0; i < k; ++i) {
    Buf& b = d->bufs[d->window.front().buf];
    if (b.state == B_READING) {
      b.discard = true;
    } else if (b.state == B_READY) {
      b.state = B_FREE;
    }
    ++d->skipped;
    d->window.pop_front();
  }
}

}  // namespace

extern "C" soup_status soup_disk_close(soup_disk* d) {
  if (!d) return SOUP_OK;
  {
    std::lock_guard<std::mutex> lk(d->mu);
    d->stop = true;
  }
  d->cv_io.notify_all();
  for (auto& t : d->io) t.join();
  for (auto& b : d->bufs) {
    if (b.done) {
      cudaEventSynchronize(b.done);
      cudaEventDestroy(b.done);
    }
    if (b.host) {
      if (d->pinned)
        cudaFreeHost(b.host);
      else
        free(b.host);
    }
  }
  for (int fd : d->fds)
    if (fd >= 0) close(fd);
  delete d;
  return SOUP_OK;
}

extern "C" soup_status soup_disk_open(const char* const* paths, int32_t n_layers, size_t layer_bytes,
                                      int32_t read_ahead, int32_t n_slots, int32_t io_threads, int32_t flags,
                                      soup_disk** out) {
  SOUP_CHECK(out, SOUP_ERR_INVALID_ARG, "soup_disk_open: null out");
  *out = nullptr;
  SOUP_CHECK(paths && n_layers >= 1, SOUP_ERR_INVALID_ARG, "soup_disk_open: no shard files");
  SOUP_CHECK(read_ahead >= 1 && read_ahead <= 8, SOUP_ERR_INVALID_ARG,
             "soup_disk_open: stream_read_ahead must be in [1, 8] (got %d)", read_ahead);
  SOUP_CHECK(n_slots >= 2 && n_slots <= 8, SOUP_ERR_INVALID_ARG, "soup_disk_open: n_slots must be in [2, 8]");
  SOUP_CHECK(io_threads >= 1 && io_threads <= 64, SOUP_ERR_INVALID_ARG, "soup_disk_open: io_threads in [1, 64]");
  SOUP_CHECK(layer_bytes > 0 && layer_bytes % 256 == 0, SOUP_ERR_ALIGN,
             "soup_disk_open: layer_bytes must be a positive multiple of 256");
  SOUP_CHECK((flags & ~(SOUP_DISK_PINNED | SOUP_DISK_DIRECT)) == 0, SOUP_ERR_INVALID_ARG,
             "soup_disk_open: unknown flags 0x%x", flags);
  for (int i = 0; i < n_layers; ++i)
    SOUP_CHECK(paths[i] != nullptr, SOUP_ERR_INVALID_ARG, "soup_disk_open: shard path %d is null", i);
  soup_disk* d = new soup_disk();
  auto cleanup = [&](soup_status st) {
    soup_disk_close(d);
    return st;
  };
  d->n_layers = n_layers;
  d->layer_bytes = layer_bytes;
  d->buf_bytes = (layer_bytes + kPage - 1) / kPage * kPage;
  d->pinned = (flags & SOUP_DISK_PINNED) != 0;
  d->n_slots = n_slots;
  d->fds.assign(n_layers, -1);
  d->direct.assign(n_layers, false);
  // every shard: open, size check, O_DIRECT where the file system takes it
  void* probe = nullptr;
  if ((flags & SOUP_DISK_DIRECT) && posix_memalign(&probe, kPage, kPage) != 0) probe = nullptr;
  for (int i = 0; i < n_layers; ++i) {
    int fd = -1;
    if (probe) {
      fd = open(paths[i], O_RDONLY | O_DIRECT);
      if (fd >= 0 && pread(fd, probe, kPage, 0) < 0) {
        close(fd);
        fd = -1;
      }
      d->direct[i] = fd >= 0;
    }
    if (fd < 0) fd = open(paths[i], O_RDONLY);
    if (fd < 0) {
      free(probe);
      return cleanup(fail(SOUP_ERR_IO, "soup_disk_open: %s: %s", paths[i], strerror(errno)));
    }
    d->fds[i] = fd;
    struct stat st;
    if (fstat(fd, &st) != 0 || (size_t)st.st_size != layer_bytes) {
      free(probe);
      return cleanup(fail(SOUP_ERR_SHAPE, "soup_disk_open: %s holds %lld bytes, not the layer's %zu", paths[i],
                          (long long)st.st_size, layer_bytes));
    }
  }
  free(probe);
  if (d->pinned && cudaGetDevice(&d->device) != cudaSuccess)
    return cleanup(fail(SOUP_ERR_CUDA, "soup_disk_open: no CUDA device"));
  d->bufs.resize(read_ahead);
  for (auto& b : d->bufs) {
    if (d->pinned) {
      if (cudaHostAlloc(reinterpret_cast<void**>(&b.host), d->buf_bytes, cudaHostAllocDefault) != cudaSuccess) {
        b.host = nullptr;
        return cleanup(fail(SOUP_ERR_CUDA, "soup_disk_open: cudaHostAlloc(%zu) failed", d->buf_bytes));
      }
      if (cudaEventCreateWithFlags(&b.done, cudaEventDisableTiming) != cudaSuccess) {
        b.done = nullptr;
        return cleanup(fail(SOUP_ERR_CUDA, "soup_disk_open: event creation failed"));
      }
    } else {
      void* p = nullptr;
      if (posix_memalign(&p, kPage, d->buf_bytes) != 0)
        return cleanup(fail(SOUP_ERR_IO, "soup_disk_open: out of host memory (%zu bytes)", d->buf_bytes));
      b.host = static_cast<char*>(p);
    }
  }
  for (int t = 0; t < io_threads; ++t) d->io.emplace_back(io_main, d);
  *out = d;
  return SOUP_OK;
}

extern "C" soup_status soup_disk_schedule(soup_disk* d, const int32_t* order, int32_t n) {
  SOUP_CHECK(d && order && n >= 1, SOUP_ERR_INVALID_ARG, "soup_disk_schedule: empty schedule");
  for (int i = 0; i < n; ++i)
    SOUP_CHECK(order[i] >= 0 && order[i] < d->n_layers, SOUP_ERR_INVALID_ARG,
               "soup_disk_schedule: layer %d out of range [0, %d)", order[i], d->n_layers);
  std::lock_guard<std::mutex> lk(d->mu);
  for (const auto& b : d->bufs)
    SOUP_CHECK(b.state != B_HELD, SOUP_ERR_INVALID_ARG, "soup_disk_schedule: a staging buffer is still held");
  drop_before(d, d->window.size());
  d->order.assign(order, order + n);
  d->next_read = 0;
  d->ring.clear();
  d->exhausted = false;
  pump(d);
  return SOUP_OK;
}

extern "C" soup_status soup_disk_acquire(soup_disk* d, int32_t layer, int32_t timeout_ms, const void** host,
                                         void** copy_done_event) {
  SOUP_CHECK(d && host, SOUP_ERR_INVALID_ARG, "soup_disk_acquire: null argument");
  SOUP_CHECK(layer >= 0 && layer < d->n_layers, SOUP_ERR_INVALID_ARG, "soup_disk_acquire: layer %d out of range",
             layer);
  SOUP_CHECK(timeout_ms >= 0, SOUP_ERR_INVALID_ARG, "soup_disk_acquire: negative timeout");
  const auto start = std::chrono::steady_clock::now();
  const auto deadline = start + std::chrono::milliseconds(timeout_ms);
  std::unique_lock<std::mutex> lk(d->mu);
  SOUP_CHECK(!d->order.empty(), SOUP_ERR_INVALID_ARG, "soup_disk_acquire: no schedule set");
  SOUP_CHECK(std::find(d->order.begin(), d->order.end(), layer) != d->order.end(), SOUP_ERR_INVALID_ARG,
             "soup_disk_acquire: layer %d is not in the read schedule", layer);
  for (const auto& b : d->bufs)
    SOUP_CHECK(!(b.state == B_HELD && b.layer == layer), SOUP_ERR_INVALID_ARG,
               "soup_disk_acquire: layer %d is already held", layer);
  while (true) {
    pump(d);
    size_t k = 0;
    while (k < d->window.size() && d->window[k].layer != layer) ++k;
    if (k < d->window.size()) {
      drop_before(d, k);
      Buf& b = d->bufs[d->window.front().buf];
      if (b.state == B_READY) {
        d->window.pop_front();
        d->wait_ms += std::chrono::duration<double, std::milli>(std::chrono::steady_clock::now() - start).count();
        ++d->acquires;
        if (b.err) {
          b.state = B_FREE;
          const std::string m = b.msg;
          pump(d);
          return fail(SOUP_ERR_IO, "soup_disk_acquire: layer %d: %s", layer, m.c_str());
        }
        b.state = B_HELD;
        *host = b.host;
        if (copy_done_event) *copy_done_event = b.done;
        return SOUP_OK;
      }
    } else {
      // The layer's next copied visit lies beyond every visit read so far
      // (those were passed over), or the replayed ring holds the layer where
      // the consumer's plan does not: resynchronise the read cursor on the
      // layer's next visit in the schedule and read that one next.
      drop_before(d, d->window.size());
      const long long n = (long long)d->order.size();
      long long s = 0;
      while (s < n && d->order[(d->next_read + s) % n] != layer) ++s;
      for (long long i = 0; i < s; ++i) ring_touch(d, d->order[(d->next_read + i) % n]);
      d->next_read += s;
      d->force_pos = d->next_read;
      d->exhausted = false;
      pump(d);
      // queued now: take it on the next pass; else wait for a buffer to free up
      if (!d->window.empty() && d->window.front().layer == layer) continue;
    }
    if (d->cv_ready.wait_until(lk, deadline) == std::cv_status::timeout) {
      pump(d);
      bool ready = false;
      for (const auto& v : d->window)
        if (v.layer == layer && d->bufs[v.buf].state == B_READY) ready = true;
      if (!ready)
        return fail(SOUP_ERR_TIMEOUT, "soup_disk_acquire: layer %d not read after %d ms", layer, timeout_ms);
    }
  }
}

extern "C" soup_status soup_disk_release(soup_disk* d, int32_t layer) {
  SOUP_CHECK(d, SOUP_ERR_INVALID_ARG, "soup_disk_release: null reader");
  std::lock_guard<std::mutex> lk(d->mu);
  for (auto& b : d->bufs) {
    if (b.state == B_HELD && b.layer == layer) {
      b.state = b.done ? B_DRAINING : B_FREE;
      pump(d);
      d->cv_io.notify_all();
      return SOUP_OK;
    }
  }
  return fail(SOUP_ERR_INVALID_ARG, "soup_disk_release: layer %d is not held", layer);
}

extern "C" soup_status soup_disk_stats(soup_disk* d, soup_disk_stats_t* out) {
  SOUP_CHECK(d && out, SOUP_ERR_INVALID_ARG, "soup_disk_stats: null argument");
  std::lock_guard<std::mutex> lk(d->mu);
  memset(out, 0, sizeof(*out));
  out->reads = d->reads;
  out->skipped = d->skipped;
  out->acquires = d->acquires;
  out->bytes_read = d->bytes_read;
  out->read_ms = d->read_ms;
  out->wait_ms = d->wait_ms;
  out->direct_files = (int32_t)std::count(d->direct.begin(), d->direct.end(), true);
  return SOUP_OK;
}
