// fmoe_tc.cuh -- tensor-core (tcgen05) products for expert groups with many
// tokens in the T > 1 path.
//
// A group of m >= kTcMinTokens tokens turns the expert's matrix-vector
// products into a dense contraction: D[M x N] = W[M x K] X[N x K]^T with W
// the dequantised weights (w = code * scale + bias, rounded to fp16) and X
// the tokens' inputs split as x = x_hi + x_lo (two fp16 values, so the
// input keeps ~22 bits): X holds the Np hi rows, then the Np lo rows, and
// the output for token t is D[., t] + D[., Np + t].  Persistent CTAs (one
// per SM) take work units of (item of <= 32 tokens, tile of 128 weight
// rows), all N = 2 Np columns, the accumulator in tensor memory:
//   - the eight producer warps stream the tile's raw codes with 16-byte
//     cp.async into a ring of four supersteps of 4 groups (three supersteps
//     ahead), and two warps per 64-input group dequantise it into a 4-stage
//     fp16 A ring (K-major, 128-byte swizzle); the group's staged X tile
//     comes by one bulk copy into an 8-stage ring, requested four steps
//     ahead;
//   - one thread (warp 0, alone on its SM sub-partition) issues the four
//     128 x N x 16 tcgen05.mma of the group and commits them to the stage's
//     mbarrier, so dequantising the next groups overlaps the tensor cores
//     (at N <= 64 the issue rate of these small products, about 75 ns each,
//     bounds the kernel: measured per step);
//   - the epilogue (warps 0-7) reads the accumulator with tcgen05.ld (warp
//     w: tensor memory lanes 32 (w % 4) .., the token columns split between
//     warps w and w + 4), adds the hi and lo columns, and writes SwiGLU
//     outputs (gate/up) or expert outputs (down).
// Error bound per output: w is rounded once (relative 2^-12), x keeps 22
// bits, the fp32 accumulation adds at most K 2^-24 of the sum of |w x|:
// below 5e-4 of that sum at K = 4096, inside the 1e-3 tolerance.
// Source pages: "What is Flash-MoE?" (a2a-mcp.org), section "2. FMA-optimised
// dequantisation kernels" (the dequantisation w = code * scale + bias; the
// pages' kernels serve one token, the tensor-core path serves many).
#pragma once

#include <cstdint>

#include <cuda_fp16.h>

#include "fmoe.h"
#include "fmoe_batched.cuh"
#include "fmoe_device.cuh"
#include "fmoe_fused.cuh"  // mbarrier and bulk-copy primitives
#include "fmoe_layout.h"

namespace fmoe {

constexpr int kTcMinTokens = 3;   // from 3 tokens per expert the tensor-core path is faster (measured, 24-bit inputs)
constexpr int kTcMaxNp = kTcItemMax;  // tokens per tensor-core item (N = 2 Np <= 64)
constexpr int kTcThreads = 256;  // producer threads (8 warps)
// The CTA has 12 warps.  Warps are spread over the SM's four sub-partitions
// by index modulo 4; the issuing thread (warp 0) gets sub-partition 0 to
// itself (warps 4 and 8 only join the barriers and the epilogue), the eight
// producer warps sit on sub-partitions 1-3, so the MMA issue loop is not
// starved of issue slots by the dequantisation (measured: ~0.65 us per step
// when it shared a sub-partition with two producer warps).
constexpr int kTcBlock = 384;
__host__ __device__ constexpr int tc_producer_of(int warp) {  // producer index 0..7 of a warp, or -1
  return (warp & 3) == 0 || warp == 11 ? -1 : warp - 1 - warp / 4;
}
constexpr int kTcRows = 128;      // weight rows per CTA (the MMA's M)
constexpr uint32_t kTcATile = kTcRows * 64 * 2;  // fp16 A tile of one 64-input group

// ------------------------------------------------------------ primitives --
// K-major, 128-byte swizzle (layout type 2 in bits 61-63): 8-row atoms of
// 128-byte lines, SBO = 1024 bytes between atoms (LBO unused).  A K = 16
// slice at byte offset 32 j of the lines starts 32 j bytes on.
__device__ __forceinline__ uint64_t umma_desc_sw128(uint32_t saddr) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | (1ull << 16) | ((uint64_t)(1024 >> 4) << 32) | (1ull << 46) |
         (2ull << 61);
}

__device__ __forceinline__ uint64_t umma_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  // K-major, no swizzle: core matrices of 8 rows x 16 bytes; lbo = distance
  // between the two 8-element halves of a K = 16 slice, sbo = between
  // 8-row groups; bit 46: descriptor version of this architecture
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46);
}

// kind::f16 instruction descriptor: fp16 A and B, K-major, fp32 accumulator, M x N.
__device__ __forceinline__ uint32_t umma_idesc_f16(int M, int N) {
  return (1u << 4) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void umma_f16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, bool acc) {
  asm volatile(
      "{ .reg .pred p; setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p; }" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"((uint32_t)acc)
      : "memory");
}

__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// 8 consecutive fp32 columns of this thread's tensor-memory lane.
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, float* v) {
  uint32_t r[8];
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
               : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ uint32_t pack_h2(float a, float b) {
  const __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&h);
}

__host__ __device__ __forceinline__ int tc_np(int m) { return (m + 7) / 8 * 8; }

// Per staged row of the tensor-core items: the multiplier that undoes the
// row's staging scale in the epilogue, and (gate/up products) the largest
// |a| of the row, from which the down products' staging takes its scale.
struct TcScale {
  float* rscale;  // [rows]
  unsigned* amax;  // [rows], fp32 bits of max |a|
};

// ------------------------------------------------------- token staging --
// Stages the inputs of every tensor-core item in fp16 hi / lo core matrices:
// per 64-input step, rows 0 .. Np-1 the hi parts of the item's tokens, rows
// Np .. 2 Np - 1 the lo parts (zero rows past the m tokens), stored as
// [8-input chunk][8-row group][8 rows][8 inputs].  Item i's block starts at
// byte it.w * 4 K (it.w: the items' running sum of Np).
//   mode 0: token vectors src + (slot / (k + 1)) K   (normed inputs xn)
//   mode 1: slot vectors  src + slot K               (SwiGLU outputs a)
// With mode 0 the CTAs also compute gamma for the shared expert's tokens.
__global__ void __launch_bounds__(kTcThreads)
tc_stage_kernel(GroupWork w, const float* __restrict__ src, int K, int k1, int mode, uint8_t* __restrict__ dst,
                int E, const float* __restrict__ w_sg, float* __restrict__ gamma, const float* __restrict__ tscale,
                TcScale sc) {
  if ((int)blockIdx.x >= w.n_items[1]) return;
  const int4 it = w.tc[blockIdx.x];
  const int g = it.x, m = it.z, np = tc_np(m), s = blockIdx.y;
  const int* slots = w.slots + w.offset[g] + it.y;
  uint8_t* base = dst + (size_t)it.w * 4 * K + (size_t)s * (2 * np) * 128;
  // row scales: mode 0 the token's (stage_tokens_kernel), mode 1 from the
  // gate/up products' max |a| of the row; the first step's CTA records the
  // epilogue multipliers and (mode 0) clears the rows' max |a|
  if (s == 0) {
    for (int r = threadIdx.x; r < m; r += blockDim.x) {
      const float f = mode == 0 ? tscale[slots[r] / k1] : tc_row_scale(__uint_as_float(sc.amax[it.w + r]));
      sc.rscale[it.w + r] = 1.f / f;
      if (mode == 0) sc.amax[it.w + r] = 0u;
    }
  }
  for (int u = threadIdx.x; u < 2 * np * 8; u += blockDim.x) {
    const int row = u >> 3, kc = u & 7;  // 8 inputs 8 kc .. 8 kc + 7 of row `row`
    const int tok = row < np ? row : row - np;
    uint4 out = make_uint4(0u, 0u, 0u, 0u);
    if (tok < m) {
      const int slot = slots[tok];
      const float* v = src + (size_t)(mode == 0 ? slot / k1 : slot) * K + s * 64 + kc * 8;
      const float rs = mode == 0 ? tscale[slot / k1] : tc_row_scale(__uint_as_float(sc.amax[it.w + tok]));
      const float4 a = __ldg(reinterpret_cast<const float4*>(v));
      const float4 b = __ldg(reinterpret_cast<const float4*>(v + 4));
      float f[8] = {a.x * rs, a.y * rs, a.z * rs, a.w * rs, b.x * rs, b.y * rs, b.z * rs, b.w * rs};
      if (row >= np) {
#pragma unroll
        for (int i = 0; i < 8; ++i) f[i] = f[i] - __half2float(__float2half_rn(f[i]));
      }
      out = make_uint4(pack_h2(f[0], f[1]), pack_h2(f[2], f[3]), pack_h2(f[4], f[5]), pack_h2(f[6], f[7]));
    }
    *reinterpret_cast<uint4*>(base + (size_t)kc * (2 * np / 8) * 128 + (size_t)(row >> 3) * 128 + (row & 7) * 16) = out;
  }
  if (mode == 0 && g == E && gamma) {  // token i's gate in the CTA of step i % steps, all its warps
    __shared__ float s_part[kTcThreads / 32];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, steps = K / 64;
    for (int i = s; i < m; i += steps) {
      const int t = slots[i] / k1;
      const float* x = src + (size_t)t * K;
      float z = 0.f;
#pragma unroll 4
      for (int c = (int)threadIdx.x * 4; c < K; c += kTcThreads * 4) {
        const float4 wv = __ldg(reinterpret_cast<const float4*>(w_sg + c));
        const float4 v = __ldg(reinterpret_cast<const float4*>(x + c));
        z = fmaf(wv.x, v.x, z);
        z = fmaf(wv.y, v.y, z);
        z = fmaf(wv.z, v.z, z);
        z = fmaf(wv.w, v.w, z);
      }
      z = warp_sum(z);
      if (lane == 0) s_part[warp] = z;
      __syncthreads();
      if (threadIdx.x == 0) {
        float zz = 0.f;
        for (int w = 0; w < kTcThreads / 32; ++w) zz += s_part[w];
        gamma[t] = 1.f / (1.f + expf(-zz));
      }
      __syncthreads();
    }
  }
}

// ---------------------------------------------------------- dequantise --
// Codes become fp16 pairs without integer-to-float conversions: a pair of
// code fields is moved into the low mantissa bits of two fp16 values of
// exponent 2^10 (1024 + field, exact), 1024 is subtracted (exact), and one
// fused half2 multiply-add applies the group's scale and bias, so each
// weight is rounded once to fp16.  A field that sits j bits up in its half
// reads as 2^j code, so its pair takes the scale 2^-j s.
__device__ __forceinline__ uint32_t deq_pair(uint32_t fields, __half2 s2, __half2 b2) {
  const uint32_t v = fields | 0x64006400u, m = 0x64006400u;
  const __half2 q = __hsub2(*reinterpret_cast<const __half2*>(&v), *reinterpret_cast<const __half2*>(&m));
  const __half2 w = __hfma2(q, s2, b2);
  return *reinterpret_cast<const uint32_t*>(&w);
}

// 16-byte fp16 store of inputs 8 c .. 8 c + 7 of row r into the A tile:
// K-major with the 128-byte swizzle -- a row's 64 inputs are one 128-byte
// line, 8 rows an atom of 1024 bytes, and the 16-byte chunk c of row r sits
// at chunk position c ^ (r % 8) (the tile is 1024-byte aligned).
__device__ __forceinline__ void store_a8h(uint8_t* a_tile, int r, int c, uint4 h) {
  *reinterpret_cast<uint4*>(a_tile + (r >> 3) * 1024 + (r & 7) * 128 + ((c ^ (r & 7)) << 4)) = h;
}

// The eight weights of a 4-bit word (field 2a+b holds input 4b+a: byte j
// holds inputs j and 4 + j), scales s (low fields) and s / 16 (high fields).
__device__ __forceinline__ uint4 dequant_word4h(uint32_t word, __half2 s1, __half2 s16, __half2 b2) {
  const uint32_t p01 = __byte_perm(word, 0u, 0x4140), p23 = __byte_perm(word, 0u, 0x4342);
  return make_uint4(deq_pair(p01 & 0x000F000Fu, s1, b2), deq_pair(p23 & 0x000F000Fu, s1, b2),
                    deq_pair(p01 & 0x00F000F0u, s16, b2), deq_pair(p23 & 0x00F000F0u, s16, b2));
}

// The sixteen weights of a 2-bit word (field 4a+b holds input 4b+a: byte j
// holds inputs j, 4 + j, 8 + j, 12 + j), as two 8-input chunks; sc[i] = 4^-i s.
__device__ __forceinline__ void dequant_word2h(uint32_t word, const __half2 (&sc)[4], __half2 b2, uint4* lo,
                                               uint4* hi) {
  const uint32_t p01 = __byte_perm(word, 0u, 0x4140), p23 = __byte_perm(word, 0u, 0x4342);
  *lo = make_uint4(deq_pair(p01 & 0x00030003u, sc[0], b2), deq_pair(p23 & 0x00030003u, sc[0], b2),
                   deq_pair(p01 & 0x000C000Cu, sc[1], b2), deq_pair(p23 & 0x000C000Cu, sc[1], b2));
  *hi = make_uint4(deq_pair(p01 & 0x00300030u, sc[2], b2), deq_pair(p23 & 0x00300030u, sc[2], b2),
                   deq_pair(p01 & 0x00C000C0u, sc[3], b2), deq_pair(p23 & 0x00C000C0u, sc[3], b2));
}

// True scale and bias of a packed scale-bias word (the scale is stored
// pre-multiplied by 2^-4 / 2^-6).
__device__ __forceinline__ void sb_true(uint32_t sbw, int bits, float* s, float* b) {
  *s = __uint_as_float(sbw << 16) * (bits == 4 ? 16.f : 64.f);
  *b = __uint_as_float(sbw & 0xFFFF0000u);
}

// ------------------------------------------------------ raw code ring --
// The producers stream the tile's raw codes and scale-bias words into a
// shared-memory ring of four "supersteps" of SG = 4 64-groups each, three
// supersteps ahead of the one being dequantised.  A superstep's bytes
// are copied in runs that are contiguous in global memory -- a row's SG
// groups (gate/up codes: two 16 SG byte runs per row, one per half of the
// 32-byte group), or 128 rows of one column-block word (down codes) -- so
// every warp-wide cp.async covers whole 128-byte lines.  The shared-memory
// copies are laid out so that the dequantising warps (lane l: rows l,
// l + 32, l + 64, l + 96, one half of the group's inputs) read without bank
// conflicts:
//   gate/up codes  [128 rows][2 halves][SG groups][16 B], row stride 144 B
//   gate/up s-b    [128 rows][SG words], row stride 48 B, at kRawSbOff
//   down codes     [SG groups x words per group][128 rows] u32
//   down s-b       [SG][128 rows] u32, at kRawDnSbOff
constexpr int kTcStages = 4;                      // ring of A tiles
constexpr int kTcBStages = 2 * kTcStages;         // ring of token tiles: requested kTcStages steps ahead
constexpr uint32_t kTcBRing = kTcBStages * kTcMaxNp * 2 * 128;
constexpr int kTcRawBufs = 4;                     // supersteps in the raw ring
constexpr int kTcMaxSG = 4;                       // 64-groups per superstep
constexpr uint32_t kRawHalf = kTcMaxSG * 16;      // one half of a row's groups
constexpr uint32_t kRawRow = 2 * kRawHalf + 16, kRawSbRow = 48;
constexpr uint32_t kRawSbOff = 128 * kRawRow;                 // 18432
constexpr uint32_t kRawDnSbOff = 8 * kTcMaxSG * 128 * 4;     // 16384
constexpr uint32_t kTcRawBuf = kRawSbOff + 128 * kRawSbRow;  // 24576 >= kRawDnSbOff + kTcMaxSG * 512
static_assert(kTcRawBuf >= kRawDnSbOff + kTcMaxSG * 512, "raw buffer holds the down layout");

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }
// Barrier of the kTcThreads producer threads only (the issuer warp is not
// in it) that also ANDs their flags, so that all of them leave or stay.
__device__ __forceinline__ bool producer_bar_and(bool v) {
  uint32_t r;
  asm volatile(
      "{ .reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, 1, %2, p;\n\t"
      "selp.u32 %0, 1, 0, q; }"
      : "=r"(r)
      : "r"((uint32_t)v), "n"(kTcThreads)
      : "memory");
  return r != 0;
}

// Requests superstep S (64-groups S SG .. S SG + SG - 1) of tile rows
// [r0, r0 + 128) into raw buffer buf.  MODE 0: gate/up rows (packed rows:
// gate n, up n interleaved, row-major codes); MODE 1: down rows
// (column-block codes: one word per row and column block).
template <int MODE, int BITS>
__device__ __forceinline__ void tc_issue_super(const uint8_t* rec, int H, int I, int r0, int S, int SG, uint8_t* buf,
                                               int t) {
  const RecordLayout L = record_layout(BITS, H, I);
  const int g0 = S * SG;
  if (MODE == 0) {
    const int ng = H / 64;
    const int runs = BITS == 4 ? 256 : 128;  // (row, half) runs of 16 SG bytes; 2-bit groups are one 16-byte chunk
    for (int c = t; c < runs * SG; c += kTcThreads) {
      const int run = c / SG, piece = c % SG;
      const int row = BITS == 4 ? run >> 1 : run, h = BITS == 4 ? run & 1 : 0;
      const uint8_t* src = rec + L.gu_codes + (size_t)(r0 + row) * L.gu_row_bytes +
                           (BITS == 4 ? chunk_off<4>(ng, g0, h) : chunk_off<2>(ng, g0, 0)) + piece * 16;
      cp_async16(buf + row * kRawRow + h * kRawHalf + piece * 16, src);
    }
    const int spr = SG / 4;  // 16-byte pieces of a row's scale-bias words
    for (int c = t; c < 128 * spr; c += kTcThreads) {
      const int row = c / spr, piece = c % spr;
      const uint8_t* src = rec + L.gu_sb + ((size_t)(r0 + row) * ng + g0) * 4 + piece * 16;
      cp_async16(buf + kRawSbOff + row * kRawSbRow + piece * 16, src);
    }
  } else {
    constexpr int kWpg = BITS == 4 ? 8 : 4;  // column-block words per 64-group
    const uint32_t* codes = reinterpret_cast<const uint32_t*>(rec + L.down_codes);
    for (int c = t; c < kWpg * SG * 32; c += kTcThreads) {
      const int run = c >> 5, piece = c & 31;
      cp_async16(buf + run * 512 + piece * 16, codes + (size_t)(kWpg * g0 + run) * H + r0 + 4 * piece);
    }
    const uint32_t* sbw = reinterpret_cast<const uint32_t*>(rec + L.down_sb);
    for (int c = t; c < SG * 32; c += kTcThreads) {
      const int run = c >> 5, piece = c & 31;
      cp_async16(buf + kRawDnSbOff + run * 512 + piece * 16, sbw + (size_t)(g0 + run) * H + r0 + 4 * piece);
    }
  }
}

// Raw words of one thread's share of a tile step: 16 bytes of codes (up to
// four 32-bit words) and the scale-bias word.
struct TcRaw {
  uint4 c;
  uint32_t sb;
};

// Group j of the superstep in buf, row r, inputs 32 hh .. 32 hh + 31.
template <int MODE, int BITS>
__device__ __forceinline__ TcRaw tc_read_raw(const uint8_t* buf, int j, int r, int hh) {
  TcRaw w;
  if (MODE == 0) {
    w.c = *reinterpret_cast<const uint4*>(buf + r * kRawRow + (BITS == 4 ? hh * kRawHalf : 0) + j * 16);
    if (BITS == 2 && hh) w.c = make_uint4(w.c.z, w.c.w, 0u, 0u);
    w.sb = *reinterpret_cast<const uint32_t*>(buf + kRawSbOff + r * kRawSbRow + j * 4);
  } else {
    const uint32_t* wd = reinterpret_cast<const uint32_t*>(buf);
    if (BITS == 4)
      w.c = make_uint4(wd[(8 * j + 4 * hh + 0) * 128 + r], wd[(8 * j + 4 * hh + 1) * 128 + r],
                       wd[(8 * j + 4 * hh + 2) * 128 + r], wd[(8 * j + 4 * hh + 3) * 128 + r]);
    else
      w.c = make_uint4(wd[(4 * j + 2 * hh + 0) * 128 + r], wd[(4 * j + 2 * hh + 1) * 128 + r], 0u, 0u);
    w.sb = *reinterpret_cast<const uint32_t*>(buf + kRawDnSbOff + (j * 128 + r) * 4);
  }
  return w;
}

// Dequantises row r, inputs 32 hh .. 32 hh + 31 of a step into the fp16 A tile.
template <int BITS>
__device__ __forceinline__ void tc_dequant(const TcRaw& w, uint8_t* a_tile, int r, int hh) {
  float s, b;
  sb_true(w.sb, BITS, &s, &b);
  const __half2 b2 = __float2half2_rn(b);
  if (BITS == 4) {
    const __half2 s1 = __float2half2_rn(s), s16 = __float2half2_rn(s * 0.0625f);
    const uint32_t wd[4] = {w.c.x, w.c.y, w.c.z, w.c.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) store_a8h(a_tile, r, 4 * hh + q, dequant_word4h(wd[q], s1, s16, b2));
  } else {
    const __half2 sc[4] = {__float2half2_rn(s), __float2half2_rn(s * 0.25f), __float2half2_rn(s * 0.0625f),
                           __float2half2_rn(s * 0.015625f)};
    const uint32_t wd[2] = {w.c.x, w.c.y};
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      uint4 lo, hi;
      dequant_word2h(wd[q], sc, b2, &lo, &hi);
      store_a8h(a_tile, r, 4 * hh + 2 * q, lo);
      store_a8h(a_tile, r, 4 * hh + 2 * q + 1, hi);
    }
  }
}

// ------------------------------------------------------------- the GEMM --

// One work unit (item it, row tile r0) of tc_gemm_kernel.  MODE 0: gate/up
// (M = 2 I, K = H), epilogue SwiGLU -> a[slot][n].  MODE 1: down (M = H,
// K = I) -> y[slot][row].  Warps 0..7 keep three supersteps of raw codes in
// flight (see the raw code ring); warps w and w + 4 handle the steps
// s = w (mod 4) (one 64-input group each, one half of its inputs per warp,
// so four steps are in flight): once the products of step s - 4 are done,
// lane 0 of warp w requests the token tile of step s + 4 into the B stage
// that held step s - 4's (the first four steps' tiles are requested with
// them), both warps dequantise into A stage s % 4 and arrive
// on full[s % 4].  So a token tile is in flight for four steps, not on the
// critical path of its own step.  Warp 8 (one thread) only waits for
// full[s % 4] and the token tile, issues the four products and commits them
// to done[s % 4].  Completion c of an A stage's mbarriers belongs to the
// CTA's step stage + 4 c (steps counted over its work units from gb), so a
// wait's parity is ((gb + s) / 4) & 1; step s's token tile is in B stage
// (gb + s) % 8, parity ((gb + s) / 8) & 1.  Bounded
// waits: on expiry the CTA sets FMOE_STATUS_WAIT_TIMEOUT, waits (bounded)
// for its committed products and copies and leaves its work loop.
template <int MODE, int BITS>
__device__ __forceinline__ void tc_gemm_body(const ExpertSet& es, const int4 it, const uint8_t* rec, int r0, int gb,
                                             const uint8_t* __restrict__ staged, float* __restrict__ out,
                                             unsigned char* tsm, uint64_t* bar_b, uint64_t* bar_m, uint64_t* bar_f,
                                             uint32_t tmem, const int* s_slot, int* s_ok, TcScale sc) {
  const int m = it.z, np = tc_np(m), N = 2 * np;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int K = MODE == 0 ? es.H : es.I;
  const int steps = K / 64;
  const uint32_t b_bytes = (uint32_t)N * 128;  // one 64-input step of the staged tokens
  const uint8_t* bsrc = staged + (size_t)it.w * 4 * K;
  auto a_st = [&](int st) { return tsm + (size_t)st * kTcATile; };
  auto b_st = [&](int st) { return tsm + (size_t)kTcStages * kTcATile + (size_t)st * b_bytes; };
  auto raw_buf = [&](int S) { return tsm + (size_t)kTcStages * kTcATile + kTcBRing + (size_t)(S % kTcRawBufs) * kTcRawBuf; };
  // parities count the CTA's steps over all of its work units (gb: steps before this one)
  auto par = [&](int s) { return (uint32_t)(((gb + s) / kTcStages) & 1); };
  auto par_b = [&](int s) { return (uint32_t)(((gb + s) / kTcBStages) & 1); };
  auto st_b = [&](int s) { return (gb + s) % kTcBStages; };
  auto request_b = [&](int s) {
    const int st = st_b(s);
    mbar_expect_tx(&bar_b[st], b_bytes);
    bulk_g2s(b_st(st), bsrc + (size_t)s * b_bytes, b_bytes, &bar_b[st]);
  };
  const int pw = tc_producer_of(warp), pt = pw * 32 + lane;  // producer warp / thread index
  if (pw >= 0) {
    // ---- producers
    const int SG = kTcMaxSG, nsup = steps / SG;  // steps: a multiple of 4
#pragma unroll
    for (int S = 0; S < kTcRawBufs - 1; ++S) {
      if (S < nsup) tc_issue_super<MODE, BITS>(rec, es.H, es.I, r0, S, SG, raw_buf(S), pt);
      cp_async_commit();
    }
    bool ok = true;
    int b_last = -1;  // last token tile requested by this lane
#pragma unroll 1
    for (int S = 0; S < nsup; ++S) {
      cp_async_wait<kTcRawBufs - 2>();  // this thread's copies of superstep S have landed
      ok = producer_bar_and(ok);        // ... and everyone's; buffer (S + 3) % 4 is no longer read
      if (!ok) break;                   // a wait expired somewhere: every producer leaves here
      if (S + kTcRawBufs - 1 < nsup)
        tc_issue_super<MODE, BITS>(rec, es.H, es.I, r0, S + kTcRawBufs - 1, SG, raw_buf(S + kTcRawBufs - 1), pt);
      cp_async_commit();
      const uint8_t* buf = raw_buf(S);
      // warps w and w + 4 dequantise the steps s = w (mod 4), inputs
      // 32 (w / 4) .. + 31 of them, always into A stage s % 4 = w % 4
#pragma unroll 1
      for (int j = pw & 3; j < SG; j += kTcStages) {
        const int s = S * SG + j, st = s % kTcStages, hh = pw >> 2;
        if (s >= kTcStages && !mbar_wait(&bar_m[st], par(s - kTcStages))) {  // products of step s - 4 done
          ok = false;
          *s_ok = 0;
          break;
        }
        if (hh == 0 && lane == 0) {  // token tiles: this step's (the first four), and step s + 4's
          if (s < kTcStages) request_b(s);
          if (s + kTcStages < steps) request_b(s + kTcStages);
          b_last = s + kTcStages < steps ? s + kTcStages : s;
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int r = lane + 32 * i;
          tc_dequant<BITS>(tc_read_raw<MODE, BITS>(buf, j, r, hh), a_st(st), r, hh);
        }
        fence_proxy_async();  // the generic-proxy A tile is read by the tensor cores
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar_f[st]);
      }
    }
    cp_async_wait_all();  // no copy may land after the CTA is gone
    // on an early exit, the last two token tiles this lane requested may
    // still be in flight (each earlier one was waited for by the issuer)
    if (!ok && b_last >= 0) {
      (void)mbar_wait(&bar_b[st_b(b_last)], par_b(b_last));
      if (b_last >= kTcStages) (void)mbar_wait(&bar_b[st_b(b_last - kTcStages)], par_b(b_last - kTcStages));
    }
  } else if (warp == 0 && lane == 0) {
    // ---- issuer: the fewest instructions per step.  The descriptors of stage 0
    // are built once; a stage, and a K = 16 slice inside it, add constant
    // amounts to their address fields (shared addresses < 256 KB fit the
    // 14-bit field, so no carry leaves it).
    const uint32_t idesc = umma_idesc_f16(kTcRows, N);
    const uint64_t ad0 = umma_desc_sw128(smem_u32(a_st(0)));
    const uint64_t bd0 = umma_desc(smem_u32(b_st(0)), (uint32_t)(N / 8) * 128, 128);
    constexpr uint64_t kAStage = kTcATile >> 4, kASlice = 32 >> 4;
    const uint64_t b_stage = b_bytes >> 4, b_slice = (uint64_t)(2 * (N / 8) * 128) >> 4;
    int last_commit = -1;
    bool ok = true;
    for (int s = 0; s < steps; ++s) {
      const int st = s % kTcStages, sb = st_b(s);
      if (!mbar_wait(&bar_f[st], par(s)) || !mbar_wait(&bar_b[sb], par_b(s))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint64_t ad = ad0 + (uint64_t)st * kAStage, bd = bd0 + (uint64_t)sb * b_stage;
      // K = 16 slices (two 8-input chunks each)
      umma_f16(tmem, ad, bd, idesc, s > 0);
      umma_f16(tmem, ad + kASlice, bd + b_slice, idesc, true);
      umma_f16(tmem, ad + 2 * kASlice, bd + 2 * b_slice, idesc, true);
      umma_f16(tmem, ad + 3 * kASlice, bd + 3 * b_slice, idesc, true);
      umma_commit(&bar_m[st]);
      last_commit = s;
    }
    if (!ok) {
      *s_ok = 0;
      if (last_commit >= 0)  // products complete in order: the last one covers the rest
        (void)mbar_wait(&bar_m[last_commit % kTcStages], par(last_commit));
    }
  }
  __syncthreads();
  bool ok = *s_ok != 0;
  if (ok) {  // the last products
    const bool done = mbar_wait(&bar_m[(steps - 1) % kTcStages], par(steps - 1));
    ok = __syncthreads_and(done);
  } else {
    __syncthreads_and(false);
  }
  tc_fence_after();
  if (ok && warp < kTcThreads / 32) {
    // epilogue: warp w reads lanes 32 (w % 4) .. (tile rows), tokens split
    // between warps w and w + 4 in chunks of 8 columns
    const int q4 = warp & 3, half = warp >> 2;
    const int row = 32 * q4 + lane;
    const uint32_t lane_base = tmem + ((uint32_t)(32 * q4) << 16);
    const int nchunk = np / 8;
    for (int ch = half; ch < nchunk; ch += 2) {
      float hi[8], lo[8];
      tmem_ld8(lane_base + (uint32_t)(ch * 8), hi);
      tmem_ld8(lane_base + (uint32_t)(np + ch * 8), lo);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int t = ch * 8 + i;
        const float v = (hi[i] + lo[i]) * (t < m ? sc.rscale[it.w + t] : 0.f);
        if (MODE == 0) {
          const float partner = __shfl_xor_sync(0xffffffffu, v, 1);  // gate row 2n, up row 2n + 1
          if ((lane & 1) == 0 && t < m) {
            const float av = silu_mul(v, partner);
            out[(size_t)s_slot[t] * es.I + (r0 + row) / 2] = av;
            atomicMax(&sc.amax[it.w + t], __float_as_uint(fabsf(av)));
          }
        } else if (t < m) {
          out[(size_t)s_slot[t] * es.H + r0 + row] = v;
        }
      }
    }
  }
  if (!ok && tid == 0) raise_status(FMOE_STATUS_WAIT_TIMEOUT);
}

// Persistent: CTA c takes the work units c, c + gridDim.x, .. of the
// n_items[1] x (M / 128) units (item u / tiles, row tile u % tiles), so the
// grid never holds idle CTAs; tensor memory, mbarriers and rings carry over
// from unit to unit (steps % 4 == 0 keeps every ring stage in step).
template <int MODE>
__global__ void __launch_bounds__(kTcBlock, 1)
tc_gemm_kernel(ExpertSet es, GroupWork w, const uint8_t* __restrict__ staged, float* __restrict__ out, TcScale sc) {
  static_assert(tc_producer_of(1) == 0 && tc_producer_of(3) == 2 && tc_producer_of(5) == 3 &&
                    tc_producer_of(7) == 5 && tc_producer_of(9) == 6 && tc_producer_of(10) == 7 &&
                    tc_producer_of(0) < 0 && tc_producer_of(4) < 0 && tc_producer_of(8) < 0 && tc_producer_of(11) < 0,
                "producer warps");
  extern __shared__ __align__(1024) unsigned char tsm[];
  __shared__ uint64_t bar_b[kTcBStages], bar_m[kTcStages], bar_f[kTcStages];
  __shared__ uint32_t s_tmem;
  __shared__ int s_slot[kTcMaxNp];
  __shared__ int s_ok;
  const int tiles = (MODE == 0 ? 2 * es.I : es.H) / kTcRows;
  const int steps = (MODE == 0 ? es.H : es.I) / 64;
  const int units = w.n_items[1] * tiles;
  if ((int)blockIdx.x >= units) return;
  const int tid = threadIdx.x, warp = tid >> 5;
  constexpr uint32_t ncols = 2 * kTcMaxNp;  // N <= 2 kTcMaxNp fp32 columns, a power of two >= 32
  static_assert(ncols >= 32 && (ncols & (ncols - 1)) == 0, "tensor memory allocation");
  if (tid == 0) {
    s_ok = 1;
    for (int i = 0; i < kTcBStages; ++i) mbar_init(&bar_b[i], 1);
    for (int i = 0; i < kTcStages; ++i) {
      mbar_init(&bar_m[i], 1);
      mbar_init(&bar_f[i], 2);  // the two warps that dequantise a step
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&s_tmem)),
                 "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;
  int gb = 0;
  for (int u = blockIdx.x; u < units; u += gridDim.x, gb += steps) {
    const int4 it = w.tc[u / tiles];
    const int g = it.x, m = it.z, r0 = (u % tiles) * kTcRows;
    for (int i = tid; i < m; i += blockDim.x) s_slot[i] = w.slots[w.offset[g] + it.y + i];
    __syncthreads();
    int bits;
    const uint8_t* rec = group_record(es, g, &bits);
    if (bits == 4) tc_gemm_body<MODE, 4>(es, it, rec, r0, gb, staged, out, tsm, bar_b, bar_m, bar_f, tmem, s_slot, &s_ok, sc);
    else tc_gemm_body<MODE, 2>(es, it, rec, r0, gb, staged, out, tsm, bar_b, bar_m, bar_f, tmem, s_slot, &s_ok, sc);
    // the epilogue's tensor-memory reads and s_slot uses end before the next unit
    tc_fence_before();
    const bool go = __syncthreads_and(s_ok != 0);
    tc_fence_after();
    if (!go) break;
  }
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(ncols) : "memory");
  }
}

// Dynamic shared memory of tc_gemm_kernel: the A ring, the token-tile ring
// and the raw code ring.
constexpr size_t tc_smem_bytes() {
  return (size_t)kTcStages * kTcATile + kTcBRing + (size_t)kTcRawBufs * kTcRawBuf;
}


}  // namespace fmoe
