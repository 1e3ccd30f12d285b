// fmoe_device.cuh -- device building blocks shared by the expert-forward kernels.
//
// The dequantised matrix-vector product follows the factorisation the
// source pages use for their dequantisation kernel ("What is Flash-MoE?",
// section "2. FMA-optimised dequantisation kernels": (code * scale + bias) * x
// = code * (scale * x) + bias * x), applied per group of 64 inputs:
//     y_r = sum_g [ s_rg * (sum_{j in g} q_rj x_j) + b_rg * X_g ],  X_g = sum_{j in g} x_j.
// On sm_100a the inner sum runs on integer dot-product instructions over an
// input vector held in 24-bit block floating point: each group of 64 inputs
// shares one power-of-two step delta_g = 2^(e_g - 23), with e_g the smallest
// exponent such that max_j |x_j| < 2^e_g, and x_j ~ delta_g * xi_j with xi_j
// a 24-bit integer (|xi_j| < 2^23).  That is the significand width of an
// fp32 number at the group's largest magnitude: |x_j - delta_g xi_j| <=
// delta_g / 2 <= 2^-23 max_j |x_j|.  xi_j is split into a signed 16-bit high
// part and an unsigned 8-bit low part (xi = 256 hi + lo); a masked 32-bit
// word of codes supplies four byte lanes, dp2a multiplies two high parts by
// two codes and dp4a four low parts by four codes, both accumulating in
// int32 exactly.  The fp32 epilogue per group is
//     y += (s * delta) * (256 A_hi + A_lo) + b * (delta * sum xi).
#pragma once

#include <cstdint>

#include <cuda_runtime.h>

#include "fmoe_layout.h"

namespace fmoe {

// Sticky device status word (FMOE_STATUS_* bits).  Defined here: all device
// code of the library is compiled as one translation unit (fmoe_kernels.cu).
__device__ uint32_t g_status = 0;

__device__ __forceinline__ void raise_status(uint32_t bits) { atomicOr(&g_status, bits); }

// Streaming 16-byte load: read once, do not keep in L1.
__device__ __forceinline__ uint4 ld_stream(const void* p) {
  uint4 v;
  asm("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
      : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
      : "l"(p));
  return v;
}

__device__ __forceinline__ float4 ld_stream_f4(const float* p) {
  uint4 v = ld_stream(p);
  return make_float4(__uint_as_float(v.x), __uint_as_float(v.y), __uint_as_float(v.z),
                     __uint_as_float(v.w));
}

__device__ __forceinline__ uint32_t ld_stream_u32(const void* p) {
  uint32_t v;
  asm("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(v) : "l"(p));
  return v;
}

// d = c + a.lo16 * b.byte0 + a.hi16 * b.byte1  (a signed 16-bit, b unsigned 8-bit)
__device__ __forceinline__ int dp2a_lo(uint32_t a, uint32_t b, int c) {
  int d;
  asm("dp2a.lo.s32.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}
// d = c + a.lo16 * b.byte2 + a.hi16 * b.byte3
__device__ __forceinline__ int dp2a_hi(uint32_t a, uint32_t b, int c) {
  int d;
  asm("dp2a.hi.s32.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

// Byte offset of a 16-byte code chunk inside a packed row of `ng` groups:
// group g, half h (4-bit: inputs 32h .. 32h+31 of the group; 2-bit: h = 0).
template <int BITS>
__device__ __forceinline__ uint32_t chunk_off(int ng, int g, int h) {
  if (BITS == 2) return (uint32_t)g * 16u;
  // segments hold min(32, ng) groups; ng is a power of two below 32
  const int seg = ng < 32 ? ng : 32;
  const int sh = __ffs(seg) - 1;
  return (uint32_t)(((g >> sh) << (sh + 5)) + (h << (sh + 4)) + ((g & (seg - 1)) << 4));
}

// Codes of one group of one row: 32 bytes (4-bit) or 16 bytes (2-bit).
template <int BITS>
struct GroupCodes {
  uint4 c[BITS == 4 ? 2 : 1];
};

template <int BITS>
__device__ __forceinline__ GroupCodes<BITS> load_group(const uint8_t* row, int ng, int g) {
  GroupCodes<BITS> gc;
  gc.c[0] = ld_stream(row + chunk_off<BITS>(ng, g, 0));
  if (BITS == 4) gc.c[BITS == 4 ? 1 : 0] = ld_stream(row + chunk_off<BITS>(ng, g, 1));
  return gc;
}

// d = c + a.byte0 * b.byte0 + ... + a.byte3 * b.byte3  (both unsigned)
__device__ __forceinline__ int dp4a_u(uint32_t a, uint32_t b, int c) {
  int d;
  asm("dp4a.u32.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

// Exact integer dot product of codes with staged inputs, split by the input
// parts: hi = sum q * xi_hi, lo = sum q * xi_lo (each times the place value
// the masked code fields carry).
struct Acc2 {
  int hi, lo;
};

// One group of 64 inputs: xv[u] holds the high parts of inputs 8u .. 8u+7
// (int16 pairs), xl[u] their low parts (bytes, .x inputs 8u .. 8u+3, .y
// 8u+4 .. 8u+7).  Returns 16 * sum q x for 4-bit codes and 64 * sum q x for
// 2-bit codes (in both parts): the masked high fields keep their place
// value, and the packed scale carries the matching 2^-4 / 2^-6.
template <int BITS>
__device__ __forceinline__ Acc2 group_dot(const GroupCodes<BITS>& gc, const uint4* xv, const uint2* xl) {
  if (BITS == 4) {
    int hl[2] = {0, 0}, hh[2] = {0, 0}, ll = 0, lh = 0;  // two accumulators each: shorter chains
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const uint32_t w[4] = {gc.c[h].x, gc.c[h].y, gc.c[h].z, gc.c[h].w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint4 x = xv[4 * h + i];
        const uint2 xb = xl[4 * h + i];
        const uint32_t l = w[i] & 0x0F0F0F0Fu, u = w[i] & 0xF0F0F0F0u;
        hl[i & 1] = dp2a_lo(x.x, l, hl[i & 1]);
        hl[i & 1] = dp2a_hi(x.y, l, hl[i & 1]);
        hh[i & 1] = dp2a_lo(x.z, u, hh[i & 1]);
        hh[i & 1] = dp2a_hi(x.w, u, hh[i & 1]);
        ll = dp4a_u(xb.x, l, ll);
        lh = dp4a_u(xb.y, u, lh);
      }
    }
    return Acc2{16 * (hl[0] + hl[1]) + (hh[0] + hh[1]), 16 * ll + lh};
  } else {
    int a0 = 0, a1 = 0, a2 = 0, a3 = 0, b0 = 0, b1 = 0, b2 = 0, b3 = 0;
    const uint32_t w[4] = {gc.c[0].x, gc.c[0].y, gc.c[0].z, gc.c[0].w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint4 x0 = xv[2 * i], x1 = xv[2 * i + 1];
      const uint2 l0 = xl[2 * i], l1 = xl[2 * i + 1];
      const uint32_t m0 = w[i] & 0x03030303u, m1 = w[i] & 0x0C0C0C0Cu;
      const uint32_t m2 = w[i] & 0x30303030u, m3 = w[i] & 0xC0C0C0C0u;
      a0 = dp2a_lo(x0.x, m0, a0);
      a0 = dp2a_hi(x0.y, m0, a0);
      a1 = dp2a_lo(x0.z, m1, a1);
      a1 = dp2a_hi(x0.w, m1, a1);
      a2 = dp2a_lo(x1.x, m2, a2);
      a2 = dp2a_hi(x1.y, m2, a2);
      a3 = dp2a_lo(x1.z, m3, a3);
      a3 = dp2a_hi(x1.w, m3, a3);
      b0 = dp4a_u(l0.x, m0, b0);
      b1 = dp4a_u(l0.y, m1, b1);
      b2 = dp4a_u(l1.x, m2, b2);
      b3 = dp4a_u(l1.y, m3, b3);
    }
    return Acc2{64 * a0 + 16 * a1 + 4 * a2 + a3, 64 * b0 + 16 * b1 + 4 * b2 + b3};
  }
}

// One 32-bit word of 4-bit codes (8 inputs) with those inputs' parts x
// (int16 pairs) and xb (bytes).  Returns 16 * sum q x, like group_dot.
__device__ __forceinline__ Acc2 word_dot4(uint32_t w, uint4 x, uint2 xb) {
  const uint32_t l = w & 0x0F0F0F0Fu, u = w & 0xF0F0F0F0u;
  const int hl = dp2a_hi(x.y, l, dp2a_lo(x.x, l, 0));
  const int hh = dp2a_hi(x.w, u, dp2a_lo(x.z, u, 0));
  const int ll = dp4a_u(xb.x, l, 0), lh = dp4a_u(xb.y, u, 0);
  return Acc2{16 * hl + hh, 16 * ll + lh};
}

// One word of 2-bit codes (16 inputs) with the parts of inputs 0..7 (x0,
// xb0) and 8..15 (x1, xb1).  Returns 64 * sum q x.
__device__ __forceinline__ Acc2 word_dot2(uint32_t w, uint4 x0, uint4 x1, uint2 xb0, uint2 xb1) {
  const uint32_t m0 = w & 0x03030303u, m1 = w & 0x0C0C0C0Cu;
  const uint32_t m2 = w & 0x30303030u, m3 = w & 0xC0C0C0C0u;
  const int a0 = dp2a_hi(x0.y, m0, dp2a_lo(x0.x, m0, 0));
  const int a1 = dp2a_hi(x0.w, m1, dp2a_lo(x0.z, m1, 0));
  const int a2 = dp2a_hi(x1.y, m2, dp2a_lo(x1.x, m2, 0));
  const int a3 = dp2a_hi(x1.w, m3, dp2a_lo(x1.z, m3, 0));
  const int b = 64 * dp4a_u(xb0.x, m0, 0) + 16 * dp4a_u(xb0.y, m1, 0) + 4 * dp4a_u(xb1.x, m2, 0) +
                dp4a_u(xb1.y, m3, 0);
  return Acc2{64 * a0 + 16 * a1 + 4 * a2 + a3, b};
}

__device__ __forceinline__ Acc2 operator+(Acc2 a, Acc2 b) { return Acc2{a.hi + b.hi, a.lo + b.lo}; }

// The 24-bit value sum of a dot product, in fp32: 256 A_hi + A_lo.
__device__ __forceinline__ float acc_value(Acc2 a) { return fmaf(256.f, (float)a.hi, (float)a.lo); }

// fp32 epilogue of one group: y + (s * delta) * A + b * xsum, with the packed
// scale-bias word (bf16 scale in the low half, bf16 bias in the high half).
__device__ __forceinline__ float group_epilogue(float y, uint32_t sb, Acc2 A, float delta, float xsum) {
  const float s = __uint_as_float(sb << 16);
  const float b = __uint_as_float(sb & 0xFFFF0000u);
  y = fmaf(s * delta, acc_value(A), y);
  return fmaf(b, xsum, y);
}

// Power-of-two step of a group whose largest magnitude is m: delta =
// 2^(e - 23) with m < 2^e, and inv = 1 / delta (both exact).  A group whose
// largest magnitude is below 2^-104 (or zero) is staged as zeros (inv = 0,
// delta = 0): its contribution is below 2^-104 per input.
__device__ __forceinline__ void bfp_step(float m, float* inv, float* delta) {
  const uint32_t E = (__float_as_uint(m) >> 23) & 0xFFu;  // m in [2^(E-127), 2^(E-126))
  if (E >= 23u && E < 255u) {
    *inv = __uint_as_float((276u - E) << 23);   // 2^(149 - E) = 2^(23 - e), e = E - 126
    *delta = __uint_as_float((E - 22u) << 23);  // 2^(E - 149)
  } else {
    *inv = 0.f;
    *delta = 0.f;
  }
}

// The 24-bit integer of x at step 1 / inv, clamped to |xi| < 2^23.
__device__ __forceinline__ int bfp_int(float x, float inv) {
  int t = __float2int_rn(x * inv);
  return t > 8388607 ? 8388607 : (t < -8388607 ? -8388607 : t);
}

// The high (int16) and low (uint8) parts of 8 24-bit values, packed: hi as
// 4 words of int16 pairs, lo as 2 words of bytes (the order group_dot reads).
__device__ __forceinline__ void bfp_pack8(const int (&q)[8], uint4* hi, uint2* lo) {
  uint32_t h[8], l[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    h[i] = (uint32_t)(q[i] >> 8) & 0xFFFFu;
    l[i] = (uint32_t)q[i] & 0xFFu;
  }
  *hi = make_uint4(h[0] | (h[1] << 16), h[2] | (h[3] << 16), h[4] | (h[5] << 16), h[6] | (h[7] << 16));
  *lo = make_uint2(l[0] | (l[1] << 8) | (l[2] << 16) | (l[3] << 24), l[4] | (l[5] << 8) | (l[6] << 16) | (l[7] << 24));
}

// Power-of-two multiplier that brings a row whose largest magnitude is m
// into [2^13, 2^14), far inside the fp16 range of the tensor-core inputs
// (their hi / lo split then keeps ~22 bits at any magnitude); 1 for rows below 2^-113 or non-finite.
__device__ __forceinline__ float tc_row_scale(float m) {
  const uint32_t E = (__float_as_uint(m) >> 23) & 0xFFu;  // m in [2^(E-127), 2^(E-126))
  return (E >= 14u && E < 255u) ? __uint_as_float((267u - E) << 23) : 1.f;
}

// Staged input vector of one token in shared memory:
//   xs[u * ng + g] : high parts of inputs 64 g + 8 u .. 64 g + 8 u + 7
//   xl[u * ng + g] : their low parts
//   delta[g]       : step of group g
//   xsum[g]        : delta[g] * (sum of the group's 24-bit values)
struct StagedX {
  uint4* xs;
  uint2* xl;
  float* delta;
  float* xsum;
};

__host__ __device__ constexpr size_t staged_x_bytes(int K) {
  return (size_t)K * 3 + (size_t)(K / 64) * 8;
}

__device__ __forceinline__ StagedX staged_x_at(unsigned char* base, int K) {
  StagedX s;
  s.xs = reinterpret_cast<uint4*>(base);
  s.xl = reinterpret_cast<uint2*>(base + (size_t)K * 2);
  s.delta = reinterpret_cast<float*>(base + (size_t)K * 3);
  s.xsum = s.delta + K / 64;
  return s;
}

// Stages 8 inputs v[0..7] (inputs 64 g + 8 u .. +7) of a group whose 8
// threads (consecutive lanes, u = lane & 7) call this together with the same
// g; every lane of the warp must call it (the shuffles span the warp).
// Inactive lanes pass zeros and active = false.
__device__ __forceinline__ void stage_unit(const float (&v)[8], bool active, int g, int u, int ng, StagedX s) {
  float m = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) m = fmaxf(m, fabsf(v[i]));
  m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
  m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
  m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 4));
  float inv, delta;
  bfp_step(m, &inv, &delta);
  int q[8];
  int sum = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    q[i] = bfp_int(v[i], inv);
    sum += q[i];
  }
  sum += __shfl_xor_sync(0xffffffffu, sum, 1);
  sum += __shfl_xor_sync(0xffffffffu, sum, 2);
  sum += __shfl_xor_sync(0xffffffffu, sum, 4);
  if (active) {
    uint4 hi;
    uint2 lo;
    bfp_pack8(q, &hi, &lo);
    s.xs[u * ng + g] = hi;
    s.xl[u * ng + g] = lo;
    if (u == 0) {
      s.delta[g] = delta;
      s.xsum[g] = delta * (float)sum;
    }
  }
}

// Stages x[0..K) (fp32, global or shared) into `s`.  All threads of the
// block take part; 8 consecutive threads share one group.  With `cg` the
// loads bypass L1 (data written by other CTAs of a running kernel).  Caller
// syncs afterwards.
__device__ __forceinline__ void stage_x(const float* __restrict__ x, int K, StagedX s, bool cg = false) {
  const int ng = K / 64;
  const int nunits = ng * 8;
  // round the loop up to a multiple of 8 threads so that group shuffles stay converged
  for (int base = 0; base < nunits; base += blockDim.x) {
    const int idx = base + (int)threadIdx.x;  // idx = g * 8 + u
    const bool active = idx < nunits;
    const int g = idx >> 3, u = idx & 7;
    float v[8];
    if (active) {
      const float4* src = reinterpret_cast<const float4*>(x + (size_t)g * 64 + u * 8);
      const float4 a = cg ? __ldcg(src) : src[0];
      const float4 b = cg ? __ldcg(src + 1) : src[1];
      v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
      v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] = 0.f;
    }
    stage_unit(v, active, g, u, ng, s);
  }
}

// Stages nvec vectors of K inputs each (x + v * K, global, L1 bypassed) into
// staged blocks at base + v * stride.  All loads of a thread are issued
// before any of them is used (one memory round trip for up to 4 * blockDim.x
// groups-of-8).  Caller syncs afterwards.
__device__ __forceinline__ void stage_x_multi(const float* __restrict__ x, int K, int nvec,
                                              unsigned char* base, size_t stride) {
  constexpr int kMaxIt = 4;
  const int upv = K / 8;  // units of 8 inputs per vector (a multiple of 8)
  const int nunits = upv * nvec;
  for (int base_u = 0; base_u < nunits; base_u += kMaxIt * (int)blockDim.x) {
    float4 lo[kMaxIt], hi[kMaxIt];
#pragma unroll
    for (int it = 0; it < kMaxIt; ++it) {
      const int idx = base_u + it * (int)blockDim.x + (int)threadIdx.x;
      if (idx < nunits) {
        const float4* src = reinterpret_cast<const float4*>(x + (size_t)idx * 8);
        lo[it] = __ldcg(src);
        hi[it] = __ldcg(src + 1);
      } else {
        lo[it] = make_float4(0.f, 0.f, 0.f, 0.f);
        hi[it] = lo[it];
      }
    }
#pragma unroll
    for (int it = 0; it < kMaxIt; ++it) {
      if (base_u + it * (int)blockDim.x >= nunits) break;  // uniform across the block
      const int idx = base_u + it * (int)blockDim.x + (int)threadIdx.x;
      const bool active = idx < nunits;
      const int v = active ? idx / upv : 0, w = idx % upv, g = w >> 3, u = w & 7;
      const float vals[8] = {lo[it].x, lo[it].y, lo[it].z, lo[it].w, hi[it].x, hi[it].y, hi[it].z, hi[it].w};
      stage_unit(vals, active, g, u, K / 64, staged_x_at(base + (size_t)v * stride, K));
    }
  }
}

__device__ __forceinline__ void load_xv(const StagedX& s, int ng, int g, uint4* xv, uint2* xl) {
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    xv[u] = s.xs[u * ng + g];
    xl[u] = s.xl[u * ng + g];
  }
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ float silu_mul(float g, float u) { return g * u / (1.f + expf(-g)); }

}  // namespace fmoe
