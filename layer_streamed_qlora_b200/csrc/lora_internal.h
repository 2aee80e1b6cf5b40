// Helpers shared by the LoRA linear and decoder-layer translation units.
#pragma once

#include "gemm.h"

namespace soup {

static inline int64_t round_up8(int64_t v) { return (v + 7) / 8 * 8; }
static inline size_t align256(size_t v) { return (v + 255) / 256 * 256; }

soup_status check_weight(const soup_weight* W, const char* fn);
void set_weight_fwd(GemmDesc& g, const soup_weight* W);
void set_weight_bwd(GemmDesc& g, const soup_weight* W);
soup_status transpose_bf16(const uint16_t* in, int rows, int cols, uint16_t* out, cudaStream_t st);

}  // namespace soup
