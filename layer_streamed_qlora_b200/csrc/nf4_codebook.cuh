// The 16-level NormalFloat (NF4) codebook of QLoRA (Dettmers et al. 2023,
// section 3 and the appendix that lists the NF4 values), as fp32 bit
// patterns, ascending: index 0 = -1, index 7 = 0 exactly, index 15 = +1.
// The Soup pages name NF4 as the storage of the streamed base but do not
// print the table.
#pragma once
#include <cstdint>

namespace soup {

#define SOUP_NF4_BITS_LIST                                                                            \
  0xBF800000u, 0xBF3239B1u, 0xBF066B30u, 0xBECA32A0u, 0xBE91A24Du, 0xBE3D353Fu, 0xBDBA7871u, 0x00000000u, \
      0x3DA2FAFFu, 0x3E24CAE3u, 0x3E7C04DDu, 0x3EAD033Au, 0x3EE1A4B8u, 0x3F1007ABu, 0x3F3913B3u, 0x3F800000u

// Device copy in constant memory: a read with a warp-uniform index is one
// broadcast (a runtime index into the constexpr table below would place that
// table in local memory and rebuild it on every call).
namespace {
__constant__ uint32_t c_nf4_bits[16] = {SOUP_NF4_BITS_LIST};
}

// Values: -1, -0.6961928, -0.5250731, -0.3949175, -0.2844414, -0.1847734,
// -0.0910500, 0, 0.0795803, 0.1609302, 0.2461123, 0.3379152, 0.4407098,
// 0.5626170, 0.7229568, 1 (fp32, round to nearest).
__host__ __device__ constexpr uint32_t nf4_code_bits(int i) {
  constexpr uint32_t bits[16] = {SOUP_NF4_BITS_LIST};
  return bits[i];
}

}  // namespace soup
