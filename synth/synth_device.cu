// synth_device.cu -- device twin of synth.c: the same counter-based streams,
// evaluated on the GPU so that large workloads (tens of GB of expert codes)
// can be generated where they are used.  Shared input generation only: no
// part of the method's arithmetic is here.  The definitions (SplitMix64
// output function, stream element i = mix64(key + (i + 1) * GOLDEN), the
// uniform / Box-Muller / bf16 recipes) are those of synth.c; the tests check
// that both produce identical bytes.
#include <cstdint>

#include <cuda_runtime.h>

namespace {

constexpr uint64_t kGolden = 0x9E3779B97F4A7C15ULL;

__device__ __forceinline__ uint64_t mix64(uint64_t z) {
  z ^= z >> 30;
  z *= 0xBF58476D1CE4E5B9ULL;
  z ^= z >> 27;
  z *= 0x94D049BB133111EBULL;
  z ^= z >> 31;
  return z;
}

__device__ __forceinline__ uint64_t word_at(uint64_t key, uint64_t i) { return mix64(key + (i + 1) * kGolden); }

__device__ __forceinline__ double uniform01(uint64_t w) { return (double)(w >> 11) * 0x1.0p-53; }

__device__ __forceinline__ double normal_at(uint64_t key, uint64_t n) {
  const double u1 = __dmul_rn(__dadd_rn((double)(word_at(key, 2 * n) >> 11), 1.0), 0x1.0p-53);
  const double u2 = uniform01(word_at(key, 2 * n + 1));
  return __dmul_rn(sqrt(__dmul_rn(-2.0, log(u1))), cos(__dmul_rn(6.283185307179586476925286766559, u2)));
}

__device__ __forceinline__ uint16_t f32_to_bf16_rne(float f) {
  uint32_t u = __float_as_uint(f);
  if ((u & 0x7F800000u) == 0x7F800000u) return (uint16_t)((u >> 16) | ((u & 0xFFFFu) ? 0x40u : 0u));
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

__device__ __forceinline__ float bf16_to_f32(uint16_t h) { return __uint_as_float((uint32_t)h << 16); }

// one thread per 64-bit word of the stream: writes 64 / bits codes
__global__ void codes_kernel(uint64_t key, int bits, uint64_t n, uint8_t* out) {
  const uint64_t per = 64u / (uint64_t)bits;
  const uint64_t mask = (1ULL << bits) - 1ULL;
  const uint64_t nw = (n + per - 1) / per;
  for (uint64_t w = blockIdx.x * (uint64_t)blockDim.x + threadIdx.x; w < nw; w += (uint64_t)gridDim.x * blockDim.x) {
    const uint64_t v = word_at(key, w);
    const uint64_t e0 = w * per;
    if (e0 + per <= n && bits == 4) {
      uint32_t lo = 0, hi = 0;  // 16 codes -> 16 bytes
#pragma unroll
      for (int f = 0; f < 4; ++f) lo |= (uint32_t)((v >> (4 * f)) & 0xF) << (8 * f);
#pragma unroll
      for (int f = 0; f < 4; ++f) hi |= (uint32_t)((v >> (4 * (f + 4))) & 0xF) << (8 * f);
      uint32_t lo2 = 0, hi2 = 0;
#pragma unroll
      for (int f = 0; f < 4; ++f) lo2 |= (uint32_t)((v >> (4 * (f + 8))) & 0xF) << (8 * f);
#pragma unroll
      for (int f = 0; f < 4; ++f) hi2 |= (uint32_t)((v >> (4 * (f + 12))) & 0xF) << (8 * f);
      *reinterpret_cast<uint4*>(out + e0) = make_uint4(lo, hi, lo2, hi2);
    } else {
      for (uint64_t f = 0; f < per && e0 + f < n; ++f) out[e0 + f] = (uint8_t)((v >> (bits * f)) & mask);
    }
  }
}

__global__ void scale_bias_kernel(uint64_t key_s, uint64_t key_b, int bits, double lo, double hi, double sigma,
                                  uint64_t n, uint16_t* scale, uint16_t* bias) {
  for (uint64_t g = blockIdx.x * (uint64_t)blockDim.x + threadIdx.x; g < n; g += (uint64_t)gridDim.x * blockDim.x) {
    const double u = uniform01(word_at(key_s, g));
    const uint16_t sb = f32_to_bf16_rne((float)__dadd_rn(lo, __dmul_rn(__dsub_rn(hi, lo), u)));
    const double s = (double)bf16_to_f32(sb);
    double b;
    if (bits == 4)
      b = __dadd_rn(__dmul_rn(-8.0, s), __dmul_rn(sigma, normal_at(key_b, g)));
    else
      b = __dmul_rn(-1.5, s);
    scale[g] = sb;
    bias[g] = f32_to_bf16_rne((float)b);
  }
}

}  // namespace

extern "C" int synth_dev_codes(uint64_t key, int bits, uint64_t n, uint8_t* d_out, cudaStream_t st) {
  if (n == 0) return 0;
  if ((reinterpret_cast<uintptr_t>(d_out) & 15u) != 0) return 1;
  const uint64_t nw = (n * bits + 63) / 64;
  const unsigned blocks = (unsigned)((nw + 255) / 256 < 65535 * 8 ? (nw + 255) / 256 : 65535 * 8);
  codes_kernel<<<blocks, 256, 0, st>>>(key, bits, n, d_out);
  return cudaGetLastError() == cudaSuccess ? 0 : 3;
}

extern "C" int synth_dev_scale_bias(uint64_t key_s, uint64_t key_b, int bits, double lo, double hi, double sigma,
                                    uint64_t n, uint16_t* d_scale, uint16_t* d_bias, cudaStream_t st) {
  if (n == 0) return 0;
  const unsigned blocks = (unsigned)((n + 255) / 256 < 65535 * 8 ? (n + 255) / 256 : 65535 * 8);
  scale_bias_kernel<<<blocks, 256, 0, st>>>(key_s, key_b, bits, lo, hi, sigma, n, d_scale, d_bias);
  return cudaGetLastError() == cudaSuccess ? 0 : 3;
}
