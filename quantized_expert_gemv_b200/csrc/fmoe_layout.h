// fmoe_layout.h -- packed expert record geometry (host and device).
//
// One record per expert, sections 16-byte aligned:
//   [gate/up codes: I row pairs x 2 rows x H*bits/8 bytes]
//   [down codes:    I*bits/32 column blocks x H rows x one 32-bit word]
//   [gate/up scale-bias: I x 2 rows x H/64 words]
//   [down scale-bias:    I/64 groups x H rows x one word]
// Gate/up rows are stored row by row (one row pair gives g_n and u_n); the
// down matrix column block by column block, so that the codes of any run of
// 8 (4-bit) or 16 (2-bit) consecutive intermediate units for every hidden
// row are one contiguous range.  The per-row chunk order and the code
// permutation inside a word are described in include/fmoe.h.
#pragma once

#include <stddef.h>
#include <stdint.h>

#if defined(__CUDACC__)
#define FMOE_HD __host__ __device__ __forceinline__
#else
#define FMOE_HD inline
#endif

namespace fmoe {

struct RecordLayout {
  size_t gu_row_bytes;    // bytes of one gate or up row (H codes)
  size_t down_row_bytes;  // bytes of one down row's codes (I codes), spread over the column blocks
  size_t gu_codes;        // offsets of the four sections
  size_t down_codes;
  size_t gu_sb;
  size_t down_sb;
  size_t bytes;           // record size
};

FMOE_HD RecordLayout record_layout(int bits, int H, int I) {
  RecordLayout L;
  L.gu_row_bytes = (size_t)H * bits / 8;
  L.down_row_bytes = (size_t)I * bits / 8;
  L.gu_codes = 0;
  L.down_codes = L.gu_codes + (size_t)I * 2 * L.gu_row_bytes;
  L.gu_sb = L.down_codes + (size_t)H * L.down_row_bytes;
  L.down_sb = L.gu_sb + (size_t)I * 2 * (H / 64) * 4;
  L.bytes = L.down_sb + (size_t)H * (I / 64) * 4;
  return L;
}

// A row of K inputs is handled by min(32, K/64) lanes, each owning whole
// groups; so K/64 must be a power of two up to 32, or a multiple of 32.
FMOE_HD bool width_supported(int K) {
  if (K < 64 || K % 64) return false;
  const int ng = K / 64;
  if (ng >= 32) return ng % 32 == 0;
  return (ng & (ng - 1)) == 0;
}

FMOE_HD bool shape_supported(int bits, int H, int I, int group) {
  return (bits == 4 || bits == 2) && group == 64 && width_supported(H) && width_supported(I);
}

}  // namespace fmoe
