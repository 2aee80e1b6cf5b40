// Library-wide runtime pieces: last-error strings, the device error word that
// bounded kernel waits report into, and the driver entry point used to build
// TMA tensor maps.
#include <atomic>
#include <cstdarg>
#include <cstring>
#include <mutex>
#include <vector>

#include "soup_internal.h"

namespace {
thread_local char g_last_error[1024] = "";

// Written by kernels when one of their bounded waits expires (nonzero code).
__device__ __align__(256) int g_soup_device_error = 0;

std::mutex g_mu;
soup::EncodeTiledFn g_encode = nullptr;
bool g_encode_tried = false;
std::atomic<long long> g_launches{0};

struct ProfRec {
  cudaEvent_t a, b;
  int cls;
  double flops, bytes;
};
bool g_prof = false;
int g_prof_mask = 0;
std::vector<ProfRec> g_prof_recs;
size_t g_prof_used = 0;
int g_prof_open = -1;
}  // namespace

namespace soup {

soup_status fail(soup_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
  return st;
}

void clear_error() { g_last_error[0] = 0; }

namespace {
typedef int (*CtxGetCurrentFn)(void** ctx);
CtxGetCurrentFn ctx_get_current() {
  static CtxGetCurrentFn fn = [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      f = nullptr;
    return reinterpret_cast<CtxGetCurrentFn>(f);
  }();
  return fn;
}
// Per (array, device): the context the address was looked up in, and the address.
struct SymAddr {
  void* ctx = nullptr;
  void* ptr = nullptr;
};
SymAddr g_sym[SYM_N][64];
std::mutex g_sym_mu;
}  // namespace

void* current_context() {
  void* ctx = nullptr;
  CtxGetCurrentFn get = ctx_get_current();
  return (get && get(&ctx) == 0) ? ctx : nullptr;
}

soup_status static_symbol_address(int which, const void* symbol, void** out) {
  SOUP_CHECK(which >= 0 && which < SYM_N && symbol && out, SOUP_ERR_INVALID_ARG, "static_symbol_address: bad argument");
  int dev = 0;
  SOUP_CUDA_TRY(cudaGetDevice(&dev));
  SOUP_CHECK(dev >= 0 && dev < 64, SOUP_ERR_INVALID_ARG, "device %d out of range", dev);
  void* ctx = nullptr;
  CtxGetCurrentFn get = ctx_get_current();
  const bool known_ctx = get && get(&ctx) == 0 && ctx != nullptr;
  std::lock_guard<std::mutex> lk(g_sym_mu);
  SymAddr& c = g_sym[which][dev];
  if (!known_ctx || c.ptr == nullptr || c.ctx != ctx) {
    void* p = nullptr;
    SOUP_CUDA_TRY(cudaGetSymbolAddress(&p, symbol));
    SOUP_CHECK(p != nullptr && soup_aligned(p, 256), SOUP_ERR_CUDA, "static array %d: bad device address", which);
    c.ptr = p;
    c.ctx = known_ctx ? ctx : nullptr;
  }
  *out = c.ptr;
  return SOUP_OK;
}

int* device_error_word() {
  void* p = nullptr;
  if (static_symbol_address(SYM_DEVICE_ERROR, reinterpret_cast<const void*>(&g_soup_device_error), &p) != SOUP_OK)
    return nullptr;
  return static_cast<int*>(p);
}

EncodeTiledFn encode_tiled() {
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_encode_tried) {
    g_encode_tried = true;
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<EncodeTiledFn>(fn);
  }
  return g_encode;
}

void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

bool profiling() { return g_prof; }

void profile_begin(cudaStream_t st, int cls, double flops, double bytes) {
  if (!g_prof || !(g_prof_mask & (1 << cls))) return;
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_prof_used == g_prof_recs.size()) {
    ProfRec r;
    cudaEventCreate(&r.a);
    cudaEventCreate(&r.b);
    g_prof_recs.push_back(r);
  }
  ProfRec& r = g_prof_recs[g_prof_used];
  r.cls = cls;
  r.flops = flops;
  r.bytes = bytes;
  cudaEventRecord(r.a, st);
  g_prof_open = (int)g_prof_used;
}

void profile_end(cudaStream_t st) {
  if (!g_prof) return;
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_prof_open < 0) return;
  cudaEventRecord(g_prof_recs[g_prof_open].b, st);
  g_prof_open = -1;
  ++g_prof_used;
}

int sm_count() {
  int dev = 0, n = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

}  // namespace soup

extern "C" const char* soup_last_error(void) { return g_last_error; }

extern "C" soup_status soup_device_error(int32_t* code_out) {
  if (!code_out) return soup::fail(SOUP_ERR_INVALID_ARG, "soup_device_error: null code_out");
  int* p = soup::device_error_word();
  if (!p) return soup::fail(SOUP_ERR_CUDA, "soup_device_error: no device error word");
  SOUP_CUDA_TRY(cudaDeviceSynchronize());
  int v = 0;
  SOUP_CUDA_TRY(cudaMemcpy(&v, p, sizeof(int), cudaMemcpyDeviceToHost));
  const int zero = 0;
  SOUP_CUDA_TRY(cudaMemcpy(p, &zero, sizeof(int), cudaMemcpyHostToDevice));
  *code_out = v;
  return SOUP_OK;
}

extern "C" int64_t soup_launch_count(void) { return g_launches.load(); }

extern "C" soup_status soup_profile_enable(int32_t class_mask) {
  std::lock_guard<std::mutex> lk(g_mu);
  g_prof = class_mask != 0;
  g_prof_mask = class_mask;
  g_prof_used = 0;
  g_prof_open = -1;
  return SOUP_OK;
}

extern "C" soup_status soup_profile_read(soup_gemm_profile* out, int32_t n_classes) {
  SOUP_CHECK(out && n_classes >= 1, SOUP_ERR_INVALID_ARG, "soup_profile_read: bad argument");
  std::lock_guard<std::mutex> lk(g_mu);
  for (int c = 0; c < n_classes; ++c) memset(&out[c], 0, sizeof(out[c]));
  for (size_t i = 0; i < g_prof_used; ++i) {
    const ProfRec& r = g_prof_recs[i];
    SOUP_CUDA_TRY(cudaEventSynchronize(r.b));
    float ms = 0;
    SOUP_CUDA_TRY(cudaEventElapsedTime(&ms, r.a, r.b));
    if (r.cls < n_classes) {
      out[r.cls].launches += 1;
      out[r.cls].total_ms += ms;
      out[r.cls].flops += r.flops;
      out[r.cls].bytes += r.bytes;
    }
  }
  return SOUP_OK;
}
