// Internal host-side helpers shared by the library's translation units:
// status codes, the thread-local last-error string, argument checks and the
// device error word that bounded waits in kernels report into.
#pragma once

#include <cstdint>
#include <cstdio>
#include <cuda_runtime.h>

#include "../../include/soup.h"

namespace soup {

// Records a formatted message as the calling thread's last error and returns `st`.
soup_status fail(soup_status st, const char* fmt, ...);
void clear_error();

// Device-side error word for the current device (set by kernels whose bounded
// waits expired; read by soup_device_error()).
int* device_error_word();

// Device address, on the current device, of one of the library's
// module-static __device__ arrays.  Host code may not pass such an array's
// name to a kernel (that is a host-side stand-in, not a device address), so
// it is looked up with the device current and cached together with the CUDA
// context it belongs to: a call in a new context (after cudaDeviceReset,
// say, which unloads the module and its arrays) looks it up again, and so
// does every call while the thread has no current context to compare with.
// The calling thread's current CUDA context (null when it has none or the
// driver entry point is unavailable).
void* current_context();

enum StaticSym : int { SYM_DEVICE_ERROR = 0, SYM_NOALLOC_SCRATCH = 1, SYM_SPLIT_COUNTERS = 2, SYM_N = 3 };
soup_status static_symbol_address(int which, const void* symbol, void** out);

// Bytes of module-static device arrays held by the GEMM engine (the slice
// counters of its split last round).
size_t gemm_static_device_bytes();


// cuTensorMapEncodeTiled resolved through the runtime's driver entry point.
typedef int (*EncodeTiledFn)(void* tmap, int dtype, uint32_t rank, void* gaddr,
                             const uint64_t* gdim, const uint64_t* gstride,
                             const uint32_t* box, const uint32_t* estride, int interleave,
                             int swizzle, int l2promo, int oobfill);
EncodeTiledFn encode_tiled();

int sm_count();

// Counts kernel launches made by this library (every launch site goes
// through SOUP_LAUNCH_CHECK).
void count_launch();

// Optional CUDA-event timing of kernel launches, by class, on the launching
// stream (enabled through soup_profile_enable): the GEMM classes, attention,
// and the memory-bound kernels tagged with their algorithmic bytes.
enum GemmClass : int {
  GC_NF4_FWD = 0, GC_NF4_BWD = 1, GC_BF16 = 2, GC_SKINNY = 3, GC_NF4_DUAL = 4,
  GC_ATTN = 5, GC_RMSNORM = 6, GC_SPLITK = 7, GC_ELEM = 8, GC_CE = 9, GC_ADAMW = 10, GC_N = 11
};
bool profiling();
void profile_begin(cudaStream_t st, int cls, double flops, double bytes);
void profile_end(cudaStream_t st);

}  // namespace soup

#define SOUP_CUDA_TRY(expr)                                                            \
  do {                                                                                 \
    cudaError_t e__ = (expr);                                                          \
    if (e__ != cudaSuccess)                                                            \
      return ::soup::fail(SOUP_ERR_CUDA, "%s: %s (%s:%d)", #expr, cudaGetErrorString(e__), \
                          __FILE__, __LINE__);                                         \
  } while (0)

#define SOUP_CHECK(cond, st, ...)                  \
  do {                                             \
    if (!(cond)) return ::soup::fail((st), __VA_ARGS__); \
  } while (0)

#define SOUP_TRY(expr)                   \
  do {                                   \
    soup_status s__ = (expr);            \
    if (s__ != SOUP_OK) return s__;      \
  } while (0)

#define SOUP_LAUNCH_CHECK()                                                            \
  do {                                                                                 \
    ::soup::count_launch();                                                            \
    cudaError_t e__ = cudaGetLastError();                                              \
    if (e__ != cudaSuccess)                                                            \
      return ::soup::fail(SOUP_ERR_CUDA, "kernel launch: %s (%s:%d)", cudaGetErrorString(e__), \
                          __FILE__, __LINE__);                                         \
  } while (0)

static inline bool soup_aligned(const void* p, size_t a) {
  return (reinterpret_cast<uintptr_t>(p) % a) == 0;
}
