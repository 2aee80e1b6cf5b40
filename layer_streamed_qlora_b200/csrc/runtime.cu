// Library-wide runtime pieces: last-error strings, the device error word that
// bounded kernel waits report into, and the driver entry point used to build
// TMA tensor maps.
#include <cstdarg>
#include <cstring>
#include <mutex>

#include "soup_internal.h"

namespace {
thread_local char g_last_error[1024] = "";

// Written by kernels when one of their bounded waits expires (nonzero code).
__device__ int g_soup_device_error = 0;

int* g_err_ptr[64] = {nullptr};
std::mutex g_mu;
soup::EncodeTiledFn g_encode = nullptr;
bool g_encode_tried = false;
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

int* device_error_word() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_err_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_soup_device_error) != cudaSuccess) return nullptr;
    g_err_ptr[dev] = static_cast<int*>(p);
  }
  return g_err_ptr[dev];
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
