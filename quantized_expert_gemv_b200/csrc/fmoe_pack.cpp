// fmoe_pack.cpp -- host-side packer for quantised expert records.
//
// Lays out group-affine int4/int2 codes ("What is Flash-MoE?", section
// "2. FMA-optimised dequantisation kernels": weight = code * scale + bias)
// so that the device matrix-vector kernels read every weight byte exactly
// once with 16-byte, fully coalesced loads, and can turn a 32-bit word of
// codes into byte lanes with a single AND before the integer dot-product
// instructions.  The format is documented in include/fmoe.h.
#include <cstdint>
#include <cstring>
#include <thread>
#include <vector>

#include <cuda_runtime.h>

#include "fmoe.h"
#include "fmoe_layout.h"

namespace fmoe {

// 32-bit words of a packed record by byte copies: the host buffers carry no
// alignment guarantee, and a 4-byte memcpy compiles to one move.
static inline void st32(uint8_t* base, size_t word, uint32_t v) { std::memcpy(base + 4 * word, &v, 4); }
static inline uint32_t ld32(const uint8_t* base, size_t word) {
  uint32_t v;
  std::memcpy(&v, base + 4 * word, 4);
  return v;
}

static inline float bf16_bits_to_f32(uint16_t h) {
  uint32_t u = (uint32_t)h << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return f;
}

// Exact power-of-two scaling of a bf16 value; false if bits would be lost
// (a result below the normal range) or the input is not finite.
static bool bf16_scale_pow2(uint16_t h, int e, uint16_t* out) {
  uint32_t exp = (h >> 7) & 0xFFu;
  if (exp == 0xFFu) return false;
  if ((h & 0x7FFFu) == 0) {  // +-0
    *out = h;
    return true;
  }
  if (exp == 0) return false;  // subnormal input
  int ne = (int)exp + e;
  if (ne <= 0 || ne >= 0xFF) return false;
  *out = (uint16_t)((h & 0x807Fu) | ((uint32_t)ne << 7));
  return true;
}

static bool bf16_unscale_pow2(uint16_t h, int e, uint16_t* out) { return bf16_scale_pow2(h, e, out); }

// Byte offset, inside a packed row of K inputs, of the 16-byte chunk that
// holds inputs [32 * half, 32 * half + 32) of group g (4-bit), or of group g
// (2-bit, half must be 0).
static inline size_t chunk_offset(int bits, int K, int g, int half) {
  if (bits == 2) return (size_t)g * 16;
  const int ng = K / 64;
  const int seg = ng < 32 ? ng : 32;
  const int s = g / seg, gi = g % seg;
  return (size_t)s * seg * 32 + (size_t)half * seg * 16 + (size_t)gi * 16;
}

// One 32-bit word of codes for 32 / bits consecutive inputs src[0 ..):
// field per_byte * a + b (bits wide) holds input 4 b + a, so that masking the
// word leaves byte lanes that pair with consecutive inputs.
static uint32_t pack_word(int bits, const uint8_t* src) {
  const int per_byte = 8 / bits;  // 2 or 4
  uint32_t word = 0;
  for (int a = 0; a < 4; ++a)
    for (int b = 0; b < per_byte; ++b) word |= (uint32_t)src[4 * b + a] << ((per_byte * a + b) * bits);
  return word;
}

static void unpack_word(int bits, uint32_t word, uint8_t* out) {
  const int per_byte = 8 / bits;
  const uint32_t mask = (1u << bits) - 1u;
  for (int a = 0; a < 4; ++a)
    for (int b = 0; b < per_byte; ++b) out[4 * b + a] = (uint8_t)((word >> ((per_byte * a + b) * bits)) & mask);
}

// Packs one logical row (K codes) into `dst` (K * bits / 8 bytes).
static void pack_row(int bits, int K, const uint8_t* q, uint8_t* dst) {
  const int ng = K / 64;
  const int per_chunk = 128 / bits;   // inputs per 16-byte chunk: 32 or 64
  const int per_word = 32 / bits;     // inputs per 32-bit word: 8 or 16
  for (int g = 0; g < ng; ++g) {
    for (int half = 0; half < 64 / per_chunk; ++half) {
      uint32_t words[4];
      const uint8_t* src = q + (size_t)g * 64 + (size_t)half * per_chunk;
      for (int w = 0; w < 4; ++w) words[w] = pack_word(bits, src + w * per_word);
      std::memcpy(dst + chunk_offset(bits, K, g, half), words, 16);
    }
  }
}

static void unpack_row(int bits, int K, const uint8_t* src, uint8_t* q) {
  const int ng = K / 64;
  const int per_chunk = 128 / bits, per_word = 32 / bits;
  for (int g = 0; g < ng; ++g)
    for (int half = 0; half < 64 / per_chunk; ++half) {
      uint32_t words[4];
      std::memcpy(words, src + chunk_offset(bits, K, g, half), 16);
      uint8_t* out = q + (size_t)g * 64 + (size_t)half * per_chunk;
      for (int w = 0; w < 4; ++w) unpack_word(bits, words[w], out + w * per_word);
    }
}

// Packs one expert.  Returns FMOE_OK or FMOE_ERR_INVALID_ARG.
static int pack_expert(int bits, int H, int I, const uint8_t* q, const uint16_t* sc,
                       const uint16_t* bi, uint8_t* dst) {
  const RecordLayout L = record_layout(bits, H, I);
  const size_t n = (size_t)H * I, ng = n / 64;
  const uint32_t qmax = (1u << bits) - 1u;
  for (size_t i = 0; i < 3 * n; ++i)
    if (q[i] > qmax) return FMOE_ERR_INVALID_ARG;
  const int shift = bits == 4 ? -4 : -6;
  // gate/up rows interleaved: packed row 2n = gate row n, 2n + 1 = up row n
  for (int r = 0; r < I; ++r)
    for (int m = 0; m < 2; ++m) {
      pack_row(bits, H, q + m * n + (size_t)r * H, dst + L.gu_codes + (size_t)(2 * r + m) * L.gu_row_bytes);
      const size_t gpr = (size_t)H / 64;
      uint8_t* sb = dst + L.gu_sb + (size_t)(2 * r + m) * gpr * 4;
      for (size_t g = 0; g < gpr; ++g) {
        uint16_t s;
        if (!bf16_scale_pow2(sc[m * ng + (size_t)r * gpr + g], shift, &s)) return FMOE_ERR_INVALID_ARG;
        st32(sb, g, (uint32_t)s | ((uint32_t)bi[m * ng + (size_t)r * gpr + g] << 16));
      }
    }
  // down matrix, column-block major: word (nb, r) holds inputs
  // [nb * per_word, (nb + 1) * per_word) of row r; scale-bias word (g, r)
  const int per_word = 32 / bits;
  uint8_t* dw = dst + L.down_codes;
  uint8_t* dsb = dst + L.down_sb;
  const size_t gpr = (size_t)I / 64;
  for (int r = 0; r < H; ++r) {
    const uint8_t* qr = q + 2 * n + (size_t)r * I;
    for (int nb = 0; nb < I / per_word; ++nb) st32(dw, (size_t)nb * H + r, pack_word(bits, qr + (size_t)nb * per_word));
    for (size_t g = 0; g < gpr; ++g) {
      uint16_t s;
      if (!bf16_scale_pow2(sc[2 * ng + (size_t)r * gpr + g], shift, &s)) return FMOE_ERR_INVALID_ARG;
      st32(dsb, g * H + r, (uint32_t)s | ((uint32_t)bi[2 * ng + (size_t)r * gpr + g] << 16));
    }
  }
  return FMOE_OK;
}

static int unpack_expert(int bits, int H, int I, const uint8_t* src, uint8_t* q, uint16_t* sc,
                         uint16_t* bi) {
  const RecordLayout L = record_layout(bits, H, I);
  const size_t n = (size_t)H * I, ng = n / 64;
  const int shift = bits == 4 ? 4 : 6;
  for (int r = 0; r < I; ++r)
    for (int m = 0; m < 2; ++m) {
      unpack_row(bits, H, src + L.gu_codes + (size_t)(2 * r + m) * L.gu_row_bytes, q + m * n + (size_t)r * H);
      const size_t gpr = (size_t)H / 64;
      const uint8_t* sb = src + L.gu_sb + (size_t)(2 * r + m) * gpr * 4;
      for (size_t g = 0; g < gpr; ++g) {
        const uint32_t w = ld32(sb, g);
        if (!bf16_unscale_pow2((uint16_t)(w & 0xFFFFu), shift, &sc[m * ng + (size_t)r * gpr + g]))
          return FMOE_ERR_INVALID_ARG;
        bi[m * ng + (size_t)r * gpr + g] = (uint16_t)(w >> 16);
      }
    }
  const int per_word = 32 / bits;
  const uint8_t* dw = src + L.down_codes;
  const uint8_t* dsb = src + L.down_sb;
  const size_t gpr = (size_t)I / 64;
  for (int r = 0; r < H; ++r) {
    uint8_t* qr = q + 2 * n + (size_t)r * I;
    for (int nb = 0; nb < I / per_word; ++nb) unpack_word(bits, ld32(dw, (size_t)nb * H + r), qr + (size_t)nb * per_word);
    for (size_t g = 0; g < gpr; ++g) {
      const uint32_t w = ld32(dsb, g * H + r);
      if (!bf16_unscale_pow2((uint16_t)(w & 0xFFFFu), shift, &sc[2 * ng + (size_t)r * gpr + g]))
        return FMOE_ERR_INVALID_ARG;
      bi[2 * ng + (size_t)r * gpr + g] = (uint16_t)(w >> 16);
    }
  }
  return FMOE_OK;
}

// Runs fn(e) for e in [0, n) on up to hardware_concurrency threads; returns
// the first non-OK status.
template <class F>
static int parallel_experts(int n, F fn) {
  unsigned nt = std::thread::hardware_concurrency();
  if (nt == 0) nt = 1;
  if ((int)nt > n) nt = (unsigned)n;
  if (nt <= 1) {
    for (int e = 0; e < n; ++e) {
      int rc = fn(e);
      if (rc != FMOE_OK) return rc;
    }
    return FMOE_OK;
  }
  std::vector<int> rc(nt, FMOE_OK);
  std::vector<std::thread> th;
  for (unsigned t = 0; t < nt; ++t)
    th.emplace_back([&, t] {
      for (int e = (int)t; e < n; e += (int)nt) {
        int r = fn(e);
        if (r != FMOE_OK) {
          rc[t] = r;
          return;
        }
      }
    });
  for (auto& x : th) x.join();
  for (int r : rc)
    if (r != FMOE_OK) return r;
  return FMOE_OK;
}

}  // namespace fmoe

using namespace fmoe;

extern "C" size_t fmoe_packed_bytes(int bits, int n_experts, int hidden, int inter, int group) {
  if (!shape_supported(bits, hidden, inter, group) || n_experts < 0) return 0;
  return record_layout(bits, hidden, inter).bytes * (size_t)n_experts;
}

extern "C" int fmoe_pack_experts_host(const uint8_t* q, const uint16_t* scale, const uint16_t* bias,
                                      int bits, int n_experts, int hidden, int inter, int group,
                                      void* h_packed, size_t h_bytes) {
  if (!q || !scale || !bias || !h_packed || n_experts < 1) return FMOE_ERR_INVALID_ARG;
  if (!shape_supported(bits, hidden, inter, group)) return FMOE_ERR_UNSUPPORTED;
  const size_t rec = record_layout(bits, hidden, inter).bytes;
  if (h_bytes < rec * (size_t)n_experts) return FMOE_ERR_BUFFER_TOO_SMALL;
  const size_t n = (size_t)hidden * inter, ng = n / 64;
  uint8_t* out = static_cast<uint8_t*>(h_packed);
  return parallel_experts(n_experts, [&](int e) {
    return pack_expert(bits, hidden, inter, q + (size_t)e * 3 * n, scale + (size_t)e * 3 * ng,
                       bias + (size_t)e * 3 * ng, out + (size_t)e * rec);
  });
}

extern "C" int fmoe_unpack_experts_host(const void* h_packed, int bits, int n_experts, int hidden,
                                        int inter, int group, uint8_t* q, uint16_t* scale,
                                        uint16_t* bias) {
  if (!q || !scale || !bias || !h_packed || n_experts < 1) return FMOE_ERR_INVALID_ARG;
  if (!shape_supported(bits, hidden, inter, group)) return FMOE_ERR_UNSUPPORTED;
  const size_t rec = record_layout(bits, hidden, inter).bytes;
  const size_t n = (size_t)hidden * inter, ng = n / 64;
  const uint8_t* src = static_cast<const uint8_t*>(h_packed);
  return parallel_experts(n_experts, [&](int e) {
    return unpack_expert(bits, hidden, inter, src + (size_t)e * rec, q + (size_t)e * 3 * n,
                         scale + (size_t)e * 3 * ng, bias + (size_t)e * 3 * ng);
  });
}

extern "C" int fmoe_pack_experts(const uint8_t* q, const uint16_t* scale, const uint16_t* bias,
                                 int bits, int n_experts, int hidden, int inter, int group,
                                 void* d_packed, size_t d_bytes, cudaStream_t stream) {
  if (!q || !scale || !bias || !d_packed || n_experts < 1) return FMOE_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(d_packed) % 16) return FMOE_ERR_INVALID_ARG;
  if (!shape_supported(bits, hidden, inter, group)) return FMOE_ERR_UNSUPPORTED;
  const size_t rec = record_layout(bits, hidden, inter).bytes;
  if (d_bytes < rec * (size_t)n_experts) return FMOE_ERR_BUFFER_TOO_SMALL;
  const size_t n = (size_t)hidden * inter, ng = n / 64;
  // pack in chunks through two pinned staging buffers, overlapping the
  // packing of one chunk with the copy of the previous one
  const int chunk = (int)((rec * 16 <= ((size_t)256 << 20)) ? 16 : 1);
  void* stage[2] = {nullptr, nullptr};
  cudaEvent_t done[2] = {nullptr, nullptr};
  int rc = FMOE_OK;
  for (int i = 0; i < 2 && rc == FMOE_OK; ++i) {
    if (cudaMallocHost(&stage[i], rec * chunk) != cudaSuccess) rc = FMOE_ERR_CUDA;
    else if (cudaEventCreateWithFlags(&done[i], cudaEventDisableTiming) != cudaSuccess) rc = FMOE_ERR_CUDA;
  }
  bool pending[2] = {false, false};
  for (int e0 = 0, it = 0; rc == FMOE_OK && e0 < n_experts; e0 += chunk, ++it) {
    const int b = it & 1;
    const int ne = (n_experts - e0) < chunk ? (n_experts - e0) : chunk;
    if (pending[b] && cudaEventSynchronize(done[b]) != cudaSuccess) { rc = FMOE_ERR_CUDA; break; }
    rc = fmoe_pack_experts_host(q + (size_t)e0 * 3 * n, scale + (size_t)e0 * 3 * ng,
                                bias + (size_t)e0 * 3 * ng, bits, ne, hidden, inter, group,
                                stage[b], rec * chunk);
    if (rc != FMOE_OK) break;
    if (cudaMemcpyAsync(static_cast<uint8_t*>(d_packed) + (size_t)e0 * rec, stage[b], rec * ne,
                        cudaMemcpyHostToDevice, stream) != cudaSuccess ||
        cudaEventRecord(done[b], stream) != cudaSuccess) {
      rc = FMOE_ERR_CUDA;
      break;
    }
    pending[b] = true;
  }
  if (cudaStreamSynchronize(stream) != cudaSuccess && rc == FMOE_OK) rc = FMOE_ERR_CUDA;
  for (int i = 0; i < 2; ++i) {
    if (stage[i]) cudaFreeHost(stage[i]);
    if (done[i]) cudaEventDestroy(done[i]);
  }
  return rc;
}
