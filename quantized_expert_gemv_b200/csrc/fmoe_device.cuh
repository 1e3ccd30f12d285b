// fmoe_device.cuh -- device building blocks shared by the expert-forward kernels.
//
// The dequantised matrix-vector product follows the factorisation the
// source pages use for their dequantisation kernel ("What is Flash-MoE?",
// section "2. FMA-optimised dequantisation kernels": (code * scale + bias) * x
// = code * (scale * x) + bias * x), applied per group of 64 inputs:
//     y_r = sum_g [ s_rg * (sum_{j in g} q_rj x_j) + b_rg * X_g ],  X_g = sum_{j in g} x_j.
// On sm_100a the inner sum runs on integer dot-product instructions: each
// CTA stages its input vector in shared memory as 16-bit fixed point per
// group (x_j ~ delta_g * xi_j, |xi_j| <= 32767, delta_g = max_j |x_j| / 32767),
// a masked 32-bit word of codes supplies four byte lanes, and dp2a multiplies
// two 16-bit inputs by two 8-bit codes and accumulates in int32, exactly.
// The fp32 epilogue per group is y += (s * delta) * A + b * (delta * sum xi).
// The only approximation is the rounding of x to 16 bits (|error| <=
// delta_g / 2 per input), far inside the 1e-3 relative tolerance.
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

// Integer dot product of one group's codes with its 64 staged inputs
// xv[0..7] (8 int16 each, inputs 8u .. 8u+7).  Returns 16 * sum q x for
// 4-bit codes and 64 * sum q x for 2-bit codes: the masked high fields keep
// their place value, and the packed scale carries the matching 2^-4 / 2^-6.
template <int BITS>
__device__ __forceinline__ int group_dot(const GroupCodes<BITS>& gc, const uint4* xv) {
  if (BITS == 4) {
    int lo[2] = {0, 0}, hi[2] = {0, 0};  // two accumulators each: shorter dependency chains
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const uint32_t w[4] = {gc.c[h].x, gc.c[h].y, gc.c[h].z, gc.c[h].w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint4 x = xv[4 * h + i];
        const uint32_t l = w[i] & 0x0F0F0F0Fu, u = w[i] & 0xF0F0F0F0u;
        lo[i & 1] = dp2a_lo(x.x, l, lo[i & 1]);
        lo[i & 1] = dp2a_hi(x.y, l, lo[i & 1]);
        hi[i & 1] = dp2a_lo(x.z, u, hi[i & 1]);
        hi[i & 1] = dp2a_hi(x.w, u, hi[i & 1]);
      }
    }
    return 16 * (lo[0] + lo[1]) + (hi[0] + hi[1]);
  } else {
    int a0 = 0, a1 = 0, a2 = 0, a3 = 0;
    const uint32_t w[4] = {gc.c[0].x, gc.c[0].y, gc.c[0].z, gc.c[0].w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint4 x0 = xv[2 * i], x1 = xv[2 * i + 1];
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
    }
    return 64 * a0 + 16 * a1 + 4 * a2 + a3;
  }
}

// Integer dot product of one 32-bit word of 4-bit codes (8 inputs) with its
// 8 staged inputs x (int16 pairs).  Returns 16 * sum q x, like group_dot.
__device__ __forceinline__ int word_dot4(uint32_t w, uint4 x) {
  const uint32_t l = w & 0x0F0F0F0Fu, u = w & 0xF0F0F0F0u;
  const int lo = dp2a_hi(x.y, l, dp2a_lo(x.x, l, 0));
  const int hi = dp2a_hi(x.w, u, dp2a_lo(x.z, u, 0));
  return 16 * lo + hi;
}

// One word of 2-bit codes (16 inputs) with its staged inputs x0 (inputs
// 0..7) and x1 (8..15).  Returns 64 * sum q x.
__device__ __forceinline__ int word_dot2(uint32_t w, uint4 x0, uint4 x1) {
  const uint32_t m0 = w & 0x03030303u, m1 = w & 0x0C0C0C0Cu;
  const uint32_t m2 = w & 0x30303030u, m3 = w & 0xC0C0C0C0u;
  const int a0 = dp2a_hi(x0.y, m0, dp2a_lo(x0.x, m0, 0));
  const int a1 = dp2a_hi(x0.w, m1, dp2a_lo(x0.z, m1, 0));
  const int a2 = dp2a_hi(x1.y, m2, dp2a_lo(x1.x, m2, 0));
  const int a3 = dp2a_hi(x1.w, m3, dp2a_lo(x1.z, m3, 0));
  return 64 * a0 + 16 * a1 + 4 * a2 + a3;
}

// fp32 epilogue of one group: y + (s * delta) * A + b * xsum, with the packed
// scale-bias word (bf16 scale in the low half, bf16 bias in the high half).
__device__ __forceinline__ float group_epilogue(float y, uint32_t sb, int A, float delta, float xsum) {
  const float s = __uint_as_float(sb << 16);
  const float b = __uint_as_float(sb & 0xFFFF0000u);
  y = fmaf(s * delta, (float)A, y);
  return fmaf(b, xsum, y);
}

// Staged input vector of one token in shared memory:
//   xs[u * ng + g] : 8 int16 inputs 64 g + 8 u .. 64 g + 8 u + 7
//   delta[g]       : fixed-point step of group g
//   xsum[g]        : delta[g] * (sum of the group's int16 inputs)
struct StagedX {
  uint4* xs;
  float* delta;
  float* xsum;
};

__host__ __device__ constexpr size_t staged_x_bytes(int K) {
  return (size_t)K * 2 + (size_t)(K / 64) * 8;
}

__device__ __forceinline__ StagedX staged_x_at(unsigned char* base, int K) {
  StagedX s;
  s.xs = reinterpret_cast<uint4*>(base);
  s.delta = reinterpret_cast<float*>(base + (size_t)K * 2);
  s.xsum = s.delta + K / 64;
  return s;
}

// Quantises x[0..K) (fp32, global or shared) into `s`.  All threads of the
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
    float m = 0.f;
    if (active) {
      const float4* src = reinterpret_cast<const float4*>(x + (size_t)g * 64 + u * 8);
      const float4 a = cg ? __ldcg(src) : src[0];
      const float4 b = cg ? __ldcg(src + 1) : src[1];
      v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
      v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
#pragma unroll
      for (int i = 0; i < 8; ++i) m = fmaxf(m, fabsf(v[i]));
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] = 0.f;
    }
    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 4));
    const float inv = m > 0.f ? 32767.f / m : 0.f;
    const float delta = m * (1.f / 32767.f);
    int q[8];
    int sum = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      int t = __float2int_rn(v[i] * inv);
      t = t > 32767 ? 32767 : (t < -32767 ? -32767 : t);
      q[i] = t;
      sum += t;
    }
    sum += __shfl_xor_sync(0xffffffffu, sum, 1);
    sum += __shfl_xor_sync(0xffffffffu, sum, 2);
    sum += __shfl_xor_sync(0xffffffffu, sum, 4);
    if (active) {
      uint4 pk;
      pk.x = (uint32_t)(q[0] & 0xFFFF) | ((uint32_t)q[1] << 16);
      pk.y = (uint32_t)(q[2] & 0xFFFF) | ((uint32_t)q[3] << 16);
      pk.z = (uint32_t)(q[4] & 0xFFFF) | ((uint32_t)q[5] << 16);
      pk.w = (uint32_t)(q[6] & 0xFFFF) | ((uint32_t)q[7] << 16);
      s.xs[u * ng + g] = pk;
      if (u == 0) {
        s.delta[g] = delta;
        s.xsum[g] = delta * (float)sum;
      }
    }
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
      const int v = idx / upv, w = idx % upv, g = w >> 3, u = w & 7;
      const float vals[8] = {lo[it].x, lo[it].y, lo[it].z, lo[it].w, hi[it].x, hi[it].y, hi[it].z, hi[it].w};
      float m = 0.f;
#pragma unroll
      for (int i = 0; i < 8; ++i) m = fmaxf(m, fabsf(vals[i]));
      m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
      m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
      m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 4));
      const float inv = m > 0.f ? 32767.f / m : 0.f;
      const float delta = m * (1.f / 32767.f);
      int q[8], sum = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        int t = __float2int_rn(vals[i] * inv);
        t = t > 32767 ? 32767 : (t < -32767 ? -32767 : t);
        q[i] = t;
        sum += t;
      }
      sum += __shfl_xor_sync(0xffffffffu, sum, 1);
      sum += __shfl_xor_sync(0xffffffffu, sum, 2);
      sum += __shfl_xor_sync(0xffffffffu, sum, 4);
      if (active) {
        const StagedX s = staged_x_at(base + (size_t)v * stride, K);
        const int ng = K / 64;
        uint4 pk;
        pk.x = (uint32_t)(q[0] & 0xFFFF) | ((uint32_t)q[1] << 16);
        pk.y = (uint32_t)(q[2] & 0xFFFF) | ((uint32_t)q[3] << 16);
        pk.z = (uint32_t)(q[4] & 0xFFFF) | ((uint32_t)q[5] << 16);
        pk.w = (uint32_t)(q[6] & 0xFFFF) | ((uint32_t)q[7] << 16);
        s.xs[u * ng + g] = pk;
        if (u == 0) {
          s.delta[g] = delta;
          s.xsum[g] = delta * (float)sum;
        }
      }
    }
  }
}

__device__ __forceinline__ void load_xv(const StagedX& s, int ng, int g, uint4* xv) {
#pragma unroll
  for (int u = 0; u < 8; ++u) xv[u] = s.xs[u * ng + g];
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ float silu_mul(float g, float u) { return g * u / (1.f + expf(-g)); }

}  // namespace fmoe
