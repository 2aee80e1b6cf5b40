// Layer-streaming runtime: a ring of preallocated device slots filled from
// pinned host blobs by a dedicated copy stream, with event hand-off to the
// compute stream (Soup pages, "how layer streaming works": the frozen base is
// cut into per-layer shards held in page-locked host RAM; `stream_buffers`
// (2..8, default 2) preallocated VRAM buffers; while one layer computes, a
// separate CUDA stream copies the next layer into another buffer; the
// vocab-sized embed_tokens and an untied lm_head share one slot).
//
// Slots are handed out least-recently-released first.  An item that is still
// resident in a released slot is not copied again when it is prefetched
// (e.g. the layers still in the ring when the forward pass turns into the
// backward pass); its bytes are identical, so results do not change.
#include <algorithm>
#include <chrono>
#include <cstring>
#include <thread>
#include <vector>

#include "soup_internal.h"

namespace {
// Timing events of the stream's statistics, as a fixed ring: each prefetch
// or wait records one (start, end) pair.  Before an entry is reused, its
// elapsed time is folded into a running total, so a long training run holds
// at most kTimedCap event pairs per ring however many steps it takes.
struct TimedRing {
  static constexpr size_t kCap = 256;
  std::vector<std::pair<cudaEvent_t, cudaEvent_t>> ev;
  size_t recorded = 0;     // pairs recorded since the last reset
  double folded_ms = 0.0;  // elapsed time of the pairs already overwritten
  // Next pair to record into; folds the previous lap's pair of this entry.
  soup_status next(std::pair<cudaEvent_t, cudaEvent_t>** out) {
    const size_t i = recorded % kCap;
    if (i == ev.size()) {
      cudaEvent_t a, b;
      SOUP_CUDA_TRY(cudaEventCreate(&a));
      if (cudaEventCreate(&b) != cudaSuccess) {
        cudaEventDestroy(a);
        return soup::fail(SOUP_ERR_CUDA, "timing event creation failed");
      }
      ev.emplace_back(a, b);
    } else if (recorded >= kCap) {
      // this entry holds a pair recorded since the last reset (a lap ago)
      SOUP_CUDA_TRY(cudaEventSynchronize(ev[i].second));
      float ms = 0.f;
      SOUP_CUDA_TRY(cudaEventElapsedTime(&ms, ev[i].first, ev[i].second));
      folded_ms += ms;
    }
    ++recorded;
    *out = &ev[i];
    return SOUP_OK;
  }
  // Total elapsed time of every pair recorded since the last reset (entries
  // [0, min(recorded, kCap)) hold this lap's pairs; older ones are folded).
  soup_status total_ms(double* out) const {
    double t = folded_ms;
    const size_t live = std::min(recorded, kCap);
    for (size_t i = 0; i < live; ++i) {
      SOUP_CUDA_TRY(cudaEventSynchronize(ev[i].second));
      float ms = 0.f;
      SOUP_CUDA_TRY(cudaEventElapsedTime(&ms, ev[i].first, ev[i].second));
      t += ms;
    }
    *out = t;
    return SOUP_OK;
  }
  void reset() {
    recorded = 0;
    folded_ms = 0.0;
  }
  void destroy() {
    for (auto& pr : ev) {
      cudaEventDestroy(pr.first);
      cudaEventDestroy(pr.second);
    }
    ev.clear();
  }
};
}  // namespace

struct soup_plan {
  int n_layers = 0;
  size_t layer_bytes = 0, vocab_bytes = 0;
  std::vector<const void*> host_layers;
  const void* host_embed = nullptr;
  const void* host_head = nullptr;
  int n_buffers = 0;
  int device = 0;
  char* arena = nullptr;      // n_buffers * layer_bytes + vocab_bytes
  size_t arena_bytes = 0;
  cudaStream_t copy = nullptr;
  // A second copy stream takes half of every large copy: on some hosts one
  // DMA engine moves ~35 GB/s over PCIe Gen5 while two together reach the
  // link's ~55 GB/s.  fork/join order it after `copy`'s waits and before
  // the slot's ready event.
  cudaStream_t copy2 = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
  struct Slot {
    char* dev = nullptr;
    size_t bytes = 0;
    int item = SOUP_ITEM_NONE;   // resident item
    bool pinned = false;         // prefetched and not yet released
    long long released_seq = -1; // order of the last release (LRU)
    cudaEvent_t ready = nullptr; // copy of `item` complete
    cudaEvent_t free_ = nullptr; // compute done with the previous item
    bool free_recorded = false;
  };
  std::vector<Slot> slots;      // [0, n_buffers) layer slots, [n_buffers] vocab slot
  long long seq = 0;
  // statistics
  long long copies = 0, reuses = 0;
  size_t bytes_copied = 0;
  TimedRing stall_events;  // (before wait, after wait) on the compute stream
  TimedRing copy_events;   // (start, end) of each copy on the copy stream
  bool fail_next_copy = false;
  cudaEvent_t gate = nullptr;   // test hook: the next copy waits on this event
};

namespace {

int slot_of(soup_plan* p, int item) {
  const int first = (item >= 0) ? 0 : p->n_buffers, last = (item >= 0) ? p->n_buffers : p->n_buffers + 1;
  for (int s = first; s < last; ++s)
    if (p->slots[s].item == item) return s;
  return -1;
}

soup_status check_item(soup_plan* p, int item) {
  SOUP_CHECK(p, SOUP_ERR_INVALID_ARG, "stream: null plan");
  if (item >= 0) {
    SOUP_CHECK(item < p->n_layers, SOUP_ERR_INVALID_ARG, "stream: layer %d out of range [0, %d)", item, p->n_layers);
  } else {
    SOUP_CHECK(item == SOUP_ITEM_EMBED || item == SOUP_ITEM_HEAD, SOUP_ERR_INVALID_ARG, "stream: bad item %d", item);
    SOUP_CHECK(p->vocab_bytes > 0, SOUP_ERR_INVALID_ARG, "stream: plan has no vocab slot");
    SOUP_CHECK(item == SOUP_ITEM_EMBED ? p->host_embed != nullptr : p->host_head != nullptr, SOUP_ERR_INVALID_ARG,
               "stream: no host tensor for vocab item %d", item);
  }
  return SOUP_OK;
}

}  // namespace

extern "C" soup_status soup_stream_plan(const soup_stream_desc* d, soup_plan** out) {
  using namespace soup;
  SOUP_CHECK(d && out, SOUP_ERR_INVALID_ARG, "soup_stream_plan: null argument");
  *out = nullptr;
  SOUP_CHECK(d->n_buffers >= 2 && d->n_buffers <= 8, SOUP_ERR_INVALID_ARG,
             "soup_stream_plan: stream_buffers must be in [2, 8] (got %d)", d->n_buffers);
  SOUP_CHECK(d->n_layers >= 1, SOUP_ERR_INVALID_ARG, "soup_stream_plan: no layers");
  SOUP_CHECK(d->layer_bytes > 0 && d->layer_bytes % 256 == 0, SOUP_ERR_ALIGN,
             "soup_stream_plan: layer_bytes must be a positive multiple of 256");
  SOUP_CHECK(d->vocab_bytes % 256 == 0, SOUP_ERR_ALIGN, "soup_stream_plan: vocab_bytes must be a multiple of 256");
  // host_layers == NULL: every layer copy comes from soup_stream_prefetch_from (disk tier)
  if (d->host_layers)
    for (int i = 0; i < d->n_layers; ++i)
      SOUP_CHECK(d->host_layers[i] != nullptr, SOUP_ERR_INVALID_ARG, "soup_stream_plan: host layer %d is null", i);
  const size_t arena = (size_t)d->n_buffers * d->layer_bytes + d->vocab_bytes;
  if (d->device_cap_bytes > 0) {
    const size_t need = arena + d->reserve_bytes;
    SOUP_CHECK(need <= d->device_cap_bytes, SOUP_ERR_OOM_PLAN,
               "soup_stream_plan: plan needs %zu bytes (%d slots x %zu + vocab %zu + reserve %zu) > cap %zu", need,
               d->n_buffers, d->layer_bytes, d->vocab_bytes, d->reserve_bytes, d->device_cap_bytes);
  }
  soup_plan* p = new soup_plan();
  p->n_layers = d->n_layers;
  p->layer_bytes = d->layer_bytes;
  p->vocab_bytes = d->vocab_bytes;
  if (d->host_layers)
    p->host_layers.assign(d->host_layers, d->host_layers + d->n_layers);
  else
    p->host_layers.assign(d->n_layers, nullptr);
  p->host_embed = d->host_embed;
  p->host_head = d->host_head;
  p->n_buffers = d->n_buffers;
  cudaGetDevice(&p->device);
  auto cleanup = [&](soup_status st) {
    soup_stream_plan_free(p);
    return st;
  };
  cudaError_t e = cudaMalloc(&p->arena, arena);
  if (e != cudaSuccess) return cleanup(fail(SOUP_ERR_CUDA, "soup_stream_plan: cudaMalloc(%zu): %s", arena, cudaGetErrorString(e)));
  p->arena_bytes = arena;
  e = cudaStreamCreateWithFlags(&p->copy, cudaStreamNonBlocking);
  if (e != cudaSuccess) return cleanup(fail(SOUP_ERR_CUDA, "soup_stream_plan: copy stream: %s", cudaGetErrorString(e)));
  e = cudaStreamCreateWithFlags(&p->copy2, cudaStreamNonBlocking);
  if (e != cudaSuccess) return cleanup(fail(SOUP_ERR_CUDA, "soup_stream_plan: copy stream: %s", cudaGetErrorString(e)));
  if (cudaEventCreateWithFlags(&p->fork, cudaEventDisableTiming) != cudaSuccess ||
      cudaEventCreateWithFlags(&p->join, cudaEventDisableTiming) != cudaSuccess)
    return cleanup(fail(SOUP_ERR_CUDA, "soup_stream_plan: event creation failed"));
  p->slots.resize(p->n_buffers + 1);
  for (int s = 0; s <= p->n_buffers; ++s) {
    auto& sl = p->slots[s];
    sl.dev = p->arena + (size_t)s * p->layer_bytes;
    sl.bytes = s < p->n_buffers ? p->layer_bytes : p->vocab_bytes;
    if (cudaEventCreateWithFlags(&sl.ready, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&sl.free_, cudaEventDisableTiming) != cudaSuccess)
      return cleanup(fail(SOUP_ERR_CUDA, "soup_stream_plan: event creation failed"));
  }
  *out = p;
  return SOUP_OK;
}

extern "C" soup_status soup_stream_plan_free(soup_plan* p) {
  if (!p) return SOUP_OK;
  if (p->copy) cudaStreamSynchronize(p->copy);
  if (p->copy2) cudaStreamSynchronize(p->copy2);
  if (p->fork) cudaEventDestroy(p->fork);
  if (p->join) cudaEventDestroy(p->join);
  for (auto& sl : p->slots) {
    if (sl.ready) cudaEventDestroy(sl.ready);
    if (sl.free_) cudaEventDestroy(sl.free_);
  }
  p->stall_events.destroy();
  p->copy_events.destroy();
  if (p->copy) cudaStreamDestroy(p->copy);
  if (p->copy2) cudaStreamDestroy(p->copy2);
  if (p->arena) cudaFree(p->arena);
  delete p;
  return SOUP_OK;
}

namespace {

// src_override: the host bytes of a layer (else the plan's own host copy);
// done: recorded on the copy stream after the copy (may be null).
soup_status prefetch_impl(soup_plan* p, int32_t item, const void* src_override, cudaEvent_t done) {
  using namespace soup;
  SOUP_TRY(check_item(p, item));
  int s = slot_of(p, item);
  if (s >= 0) {
    auto& sl = p->slots[s];
    SOUP_CHECK(!sl.pinned, SOUP_ERR_INVALID_ARG, "soup_stream_prefetch: item %d is already prefetched", item);
    sl.pinned = true;  // still resident: no copy
    ++p->reuses;
    return SOUP_OK;
  }
  // pick the least recently released, unpinned slot of the right kind
  if (item >= 0) {
    for (int i = 0; i < p->n_buffers; ++i) {
      const auto& sl = p->slots[i];
      if (sl.pinned) continue;
      if (s < 0 || sl.released_seq < p->slots[s].released_seq) s = i;
    }
    SOUP_CHECK(s >= 0, SOUP_ERR_INVALID_ARG,
               "soup_stream_prefetch: all %d layer slots hold items that were not released", p->n_buffers);
  } else {
    s = p->n_buffers;
    SOUP_CHECK(!p->slots[s].pinned, SOUP_ERR_INVALID_ARG,
               "soup_stream_prefetch: the vocab slot holds item %d, not released", p->slots[s].item);
  }
  auto& sl = p->slots[s];
  const void* src = src_override ? src_override
                                  : (item >= 0 ? p->host_layers[item]
                                               : (item == SOUP_ITEM_EMBED ? p->host_embed : p->host_head));
  SOUP_CHECK(src, SOUP_ERR_INVALID_ARG,
             "soup_stream_prefetch: the plan holds no host copy of layer %d (bring it with soup_stream_prefetch_from)",
             item);
  const size_t bytes = item >= 0 ? p->layer_bytes : p->vocab_bytes;
  if (p->fail_next_copy) {
    p->fail_next_copy = false;
    return fail(SOUP_ERR_CUDA, "soup_stream_prefetch: injected copy failure for item %d", item);
  }
  if (sl.free_recorded) SOUP_CUDA_TRY(cudaStreamWaitEvent(p->copy, sl.free_, 0));
  if (p->gate) {
    SOUP_CUDA_TRY(cudaStreamWaitEvent(p->copy, p->gate, 0));
    p->gate = nullptr;
  }
  std::pair<cudaEvent_t, cudaEvent_t>* cep = nullptr;
  SOUP_TRY(p->copy_events.next(&cep));
  auto& ce = *cep;
  SOUP_CUDA_TRY(cudaEventRecord(ce.first, p->copy));
  if (bytes >= (8u << 20)) {
    // second half on the second copy stream, after the same waits
    const size_t half = (bytes / 2) & ~(size_t)255;
    SOUP_CUDA_TRY(cudaEventRecord(p->fork, p->copy));
    SOUP_CUDA_TRY(cudaStreamWaitEvent(p->copy2, p->fork, 0));
    SOUP_CUDA_TRY(cudaMemcpyAsync(sl.dev, src, half, cudaMemcpyHostToDevice, p->copy));
    SOUP_CUDA_TRY(cudaMemcpyAsync(sl.dev + half, static_cast<const char*>(src) + half, bytes - half,
                                  cudaMemcpyHostToDevice, p->copy2));
    SOUP_CUDA_TRY(cudaEventRecord(p->join, p->copy2));
    SOUP_CUDA_TRY(cudaStreamWaitEvent(p->copy, p->join, 0));
  } else {
    SOUP_CUDA_TRY(cudaMemcpyAsync(sl.dev, src, bytes, cudaMemcpyHostToDevice, p->copy));
  }
  SOUP_CUDA_TRY(cudaEventRecord(sl.ready, p->copy));
  if (done) SOUP_CUDA_TRY(cudaEventRecord(done, p->copy));
  SOUP_CUDA_TRY(cudaEventRecord(ce.second, p->copy));
  sl.item = item;
  sl.pinned = true;
  ++p->copies;
  p->bytes_copied += bytes;
  return SOUP_OK;
}

}  // namespace

extern "C" soup_status soup_stream_prefetch(soup_plan* p, int32_t item) {
  return prefetch_impl(p, item, nullptr, nullptr);
}

extern "C" soup_status soup_stream_prefetch_from(soup_plan* p, int32_t layer, const void* host_src,
                                                 void* copy_done_event) {
  using namespace soup;
  SOUP_CHECK(layer >= 0 && host_src, SOUP_ERR_INVALID_ARG,
             "soup_stream_prefetch_from: needs a layer index and a host source");
  return prefetch_impl(p, layer, host_src, static_cast<cudaEvent_t>(copy_done_event));
}

extern "C" soup_status soup_stream_resident(soup_plan* p, int32_t item, int32_t* resident) {
  using namespace soup;
  SOUP_TRY(check_item(p, item));
  SOUP_CHECK(resident, SOUP_ERR_INVALID_ARG, "soup_stream_resident: null out");
  *resident = slot_of(p, item) >= 0 ? 1 : 0;
  return SOUP_OK;
}

extern "C" soup_status soup_stream_wait(soup_plan* p, int32_t item, void* compute_stream, void** slot_dev) {
  using namespace soup;
  SOUP_TRY(check_item(p, item));
  SOUP_CHECK(slot_dev, SOUP_ERR_INVALID_ARG, "soup_stream_wait: null slot_dev");
  const int s = slot_of(p, item);
  SOUP_CHECK(s >= 0 && p->slots[s].pinned, SOUP_ERR_INVALID_ARG, "soup_stream_wait: item %d was not prefetched",
             item);
  cudaStream_t cs = static_cast<cudaStream_t>(compute_stream);
  std::pair<cudaEvent_t, cudaEvent_t>* prp = nullptr;
  SOUP_TRY(p->stall_events.next(&prp));
  auto& pr = *prp;
  SOUP_CUDA_TRY(cudaEventRecord(pr.first, cs));
  SOUP_CUDA_TRY(cudaStreamWaitEvent(cs, p->slots[s].ready, 0));
  SOUP_CUDA_TRY(cudaEventRecord(pr.second, cs));
  *slot_dev = p->slots[s].dev;
  return SOUP_OK;
}

extern "C" soup_status soup_stream_wait_host(soup_plan* p, int32_t item, int32_t timeout_ms) {
  using namespace soup;
  SOUP_TRY(check_item(p, item));
  SOUP_CHECK(timeout_ms >= 0, SOUP_ERR_INVALID_ARG, "soup_stream_wait_host: negative timeout");
  const int s = slot_of(p, item);
  SOUP_CHECK(s >= 0 && p->slots[s].pinned, SOUP_ERR_INVALID_ARG, "soup_stream_wait_host: item %d was not prefetched",
             item);
  const auto deadline = std::chrono::steady_clock::now() + std::chrono::milliseconds(timeout_ms);
  while (true) {
    const cudaError_t q = cudaEventQuery(p->slots[s].ready);
    if (q == cudaSuccess) return SOUP_OK;
    if (q != cudaErrorNotReady) return fail(SOUP_ERR_CUDA, "soup_stream_wait_host: %s", cudaGetErrorString(q));
    if (std::chrono::steady_clock::now() >= deadline)
      return fail(SOUP_ERR_TIMEOUT, "soup_stream_wait_host: item %d not ready after %d ms", item, timeout_ms);
    std::this_thread::sleep_for(std::chrono::microseconds(100));
  }
}

extern "C" soup_status soup_stream_release(soup_plan* p, int32_t item, void* compute_stream) {
  using namespace soup;
  SOUP_TRY(check_item(p, item));
  const int s = slot_of(p, item);
  SOUP_CHECK(s >= 0 && p->slots[s].pinned, SOUP_ERR_INVALID_ARG, "soup_stream_release: item %d is not held", item);
  auto& sl = p->slots[s];
  SOUP_CUDA_TRY(cudaEventRecord(sl.free_, static_cast<cudaStream_t>(compute_stream)));
  sl.free_recorded = true;
  sl.pinned = false;
  sl.released_seq = p->seq++;
  return SOUP_OK;
}

extern "C" soup_status soup_stream_stats(soup_plan* p, soup_stream_stats_t* out) {
  using namespace soup;
  SOUP_CHECK(p && out, SOUP_ERR_INVALID_ARG, "soup_stream_stats: null argument");
  SOUP_CUDA_TRY(cudaStreamSynchronize(p->copy));
  memset(out, 0, sizeof(*out));
  out->copies = p->copies;
  out->reuses = p->reuses;
  out->bytes_copied = p->bytes_copied;
  out->arena_bytes = p->arena_bytes;
  double stall = 0, cms = 0;
  SOUP_TRY(p->stall_events.total_ms(&stall));
  SOUP_TRY(p->copy_events.total_ms(&cms));
  out->waits = (int64_t)p->stall_events.recorded;
  out->stall_ms = stall;
  out->copy_ms = cms;
  return SOUP_OK;
}

extern "C" soup_status soup_stream_stats_reset(soup_plan* p) {
  SOUP_CHECK(p, SOUP_ERR_INVALID_ARG, "soup_stream_stats_reset: null plan");
  SOUP_CUDA_TRY(cudaStreamSynchronize(p->copy));
  p->copies = p->reuses = 0;
  p->bytes_copied = 0;
  p->stall_events.reset();
  p->copy_events.reset();
  return SOUP_OK;
}

extern "C" soup_status soup_stream_debug_fail_next_copy(soup_plan* p) {
  SOUP_CHECK(p, SOUP_ERR_INVALID_ARG, "null plan");
  p->fail_next_copy = true;
  return SOUP_OK;
}

extern "C" soup_status soup_stream_debug_gate_next_copy(soup_plan* p, void* event) {
  SOUP_CHECK(p && event, SOUP_ERR_INVALID_ARG, "null argument");
  p->gate = static_cast<cudaEvent_t>(event);
  return SOUP_OK;
}

extern "C" void* soup_stream_copy_stream(soup_plan* p) { return p ? p->copy : nullptr; }

extern "C" int64_t soup_stream_debug_timing_events(soup_plan* p) {
  return p ? (int64_t)(2 * (p->stall_events.ev.size() + p->copy_events.ev.size())) : -1;
}
