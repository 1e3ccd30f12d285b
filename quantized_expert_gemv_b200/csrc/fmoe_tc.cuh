// fmoe_tc.cuh -- tensor-core (tcgen05) products for expert groups with many
// tokens in the T > 1 path.
//
// A group of m >= kTcMinTokens tokens turns the expert's matrix-vector
// products into a dense contraction: D[M x N] = W[M x K] X[N x K]^T with W
// the dequantised weights (w = code * scale + bias, rounded to fp16) and X
// the tokens' inputs split as x = x_hi + x_lo (two fp16 values, so the
// input keeps ~22 bits): X holds the Np hi rows, then the Np lo rows, and
// the output for token t is D[., t] + D[., Np + t].  Per CTA: a tile of 128
// weight rows, all N = 2 Np columns, the accumulator in tensor memory:
//   - all 256 threads dequantise one 64-input group of the tile into shared
//     memory (fp16, K-major core matrices of 8 rows x 16 bytes);
//   - the staged X tile of that group arrives by one bulk copy;
//   - one thread issues the four 128 x N x 16 tcgen05.mma of the group and
//     commits them to the stage's mbarrier (a ring of three stages, so
//     dequantising the next groups overlaps the tensor cores; the raw
//     weight words are loaded four groups ahead);
//   - the epilogue reads the accumulator with tcgen05.ld (warp w: tensor
//     memory lanes 32 (w % 4) ..), adds the hi and lo columns, and writes
//     SwiGLU outputs (gate/up) or expert outputs (down).
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

constexpr int kTcMinTokens = 16;  // a group this large goes to the tensor cores
constexpr int kTcMaxNp = 128;     // tokens per tensor-core item (N = 2 Np <= 256)
constexpr int kTcThreads = 256;
constexpr int kTcRows = 128;      // weight rows per CTA (the MMA's M)
constexpr uint32_t kTcATile = kTcRows * 64 * 2;  // fp16 A tile of one 64-input group

// ------------------------------------------------------------ primitives --
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
                int E, const float* __restrict__ w_sg, float* __restrict__ gamma) {
  if ((int)blockIdx.x >= w.n_items[1]) return;
  const int4 it = w.tc[blockIdx.x];
  const int g = it.x, m = it.z, np = tc_np(m), s = blockIdx.y;
  const int* slots = w.slots + w.offset[g] + it.y;
  uint8_t* base = dst + (size_t)it.w * 4 * K + (size_t)s * (2 * np) * 128;
  for (int u = threadIdx.x; u < 2 * np * 8; u += blockDim.x) {
    const int row = u >> 3, kc = u & 7;  // 8 inputs 8 kc .. 8 kc + 7 of row `row`
    const int tok = row < np ? row : row - np;
    uint4 out = make_uint4(0u, 0u, 0u, 0u);
    if (tok < m) {
      const int slot = slots[tok];
      const float* v = src + (size_t)(mode == 0 ? slot / k1 : slot) * K + s * 64 + kc * 8;
      const float4 a = __ldg(reinterpret_cast<const float4*>(v));
      const float4 b = __ldg(reinterpret_cast<const float4*>(v + 4));
      float f[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
      if (row >= np) {
#pragma unroll
        for (int i = 0; i < 8; ++i) f[i] = f[i] - __half2float(__float2half_rn(f[i]));
      }
      out = make_uint4(pack_h2(f[0], f[1]), pack_h2(f[2], f[3]), pack_h2(f[4], f[5]), pack_h2(f[6], f[7]));
    }
    *reinterpret_cast<uint4*>(base + (size_t)kc * (2 * np / 8) * 128 + (size_t)(row >> 3) * 128 + (row & 7) * 16) = out;
  }
  if (mode == 0 && g == E && gamma) {  // token i's gate in the CTA of step i % steps, one warp each
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, steps = K / 64;
    for (int i = s + steps * warp; i < m; i += steps * (kTcThreads / 32)) {
      const int t = slots[i] / k1;
      const float* x = src + (size_t)t * K;
      float z = 0.f;
      for (int c = lane * 4; c < K; c += 128) {
        const float4 wv = __ldg(reinterpret_cast<const float4*>(w_sg + c));
        const float4 v = __ldg(reinterpret_cast<const float4*>(x + c));
        z = fmaf(wv.x, v.x, z);
        z = fmaf(wv.y, v.y, z);
        z = fmaf(wv.z, v.z, z);
        z = fmaf(wv.w, v.w, z);
      }
      z = warp_sum(z);
      if (lane == 0) gamma[t] = 1.f / (1.f + expf(-z));
    }
  }
}

// ---------------------------------------------------------- dequantise --
// Four 16-byte fp16 stores of 8 weights each into the A tile: row r, inputs
// 8 c .. 8 c + 7 for c = c0 .. c0 + 3.
__device__ __forceinline__ void store_a8(uint8_t* a_tile, int r, int c, const float* w8) {
  *reinterpret_cast<uint4*>(a_tile + (size_t)c * (kTcRows / 8) * 128 + (r >> 3) * 128 + (r & 7) * 16) =
      make_uint4(pack_h2(w8[0], w8[1]), pack_h2(w8[2], w8[3]), pack_h2(w8[4], w8[5]), pack_h2(w8[6], w8[7]));
}

// Weights of inputs 0..7 of a 4-bit word (field 2a+b holds input 4b+a).
__device__ __forceinline__ void dequant_word4(uint32_t word, float s, float b, float* w8) {
#pragma unroll
  for (int i = 0; i < 8; ++i) w8[i] = fmaf((float)((word >> (4 * (2 * (i & 3) + (i >> 2)))) & 15u), s, b);
}

// Weights of inputs 0..15 of a 2-bit word (field 4a+b holds input 4b+a).
__device__ __forceinline__ void dequant_word2(uint32_t word, float s, float b, float* w16) {
#pragma unroll
  for (int i = 0; i < 16; ++i) w16[i] = fmaf((float)((word >> (2 * (4 * (i & 3) + (i >> 2)))) & 3u), s, b);
}

// True scale and bias of a packed scale-bias word (the scale is stored
// pre-multiplied by 2^-4 / 2^-6).
__device__ __forceinline__ void sb_true(uint32_t sbw, int bits, float* s, float* b) {
  *s = __uint_as_float(sbw << 16) * (bits == 4 ? 16.f : 64.f);
  *b = __uint_as_float(sbw & 0xFFFF0000u);
}

// Raw words of one thread's share of a tile step: 16 bytes of codes (up to
// four 32-bit words) and the scale-bias word.
struct TcRaw {
  uint4 c;
  uint32_t sb;
};

// Thread t's share of 64-group gi of tile rows [r0, r0 + 128): row t / 2,
// inputs 32 (t % 2) .. + 31.  MODE 0: gate/up rows (packed rows: gate n, up
// n interleaved, row-major codes); MODE 1: down rows (column-block codes).
template <int MODE, int BITS>
__device__ __forceinline__ TcRaw tc_load_raw(const uint8_t* rec, int H, int I, int r0, int gi) {
  const RecordLayout L = record_layout(BITS, H, I);
  const int t = threadIdx.x, r = t >> 1, hh = t & 1;
  TcRaw w;
  if (MODE == 0) {
    const int ng = H / 64, pr = r0 + r;
    const uint8_t* row = rec + L.gu_codes + (size_t)pr * L.gu_row_bytes;
    w.c = ld_stream(row + (BITS == 4 ? chunk_off<4>(ng, gi, hh) : chunk_off<2>(ng, gi, 0)));
    if (BITS == 2 && hh) w.c = make_uint4(w.c.z, w.c.w, 0u, 0u);
    w.sb = ld_stream_u32(reinterpret_cast<const uint32_t*>(rec + L.gu_sb) + (size_t)pr * ng + gi);
  } else {
    const int row = r0 + r;
    const uint32_t* codes = reinterpret_cast<const uint32_t*>(rec + L.down_codes) + row;
    if (BITS == 4) {  // words 8 gi + 4 hh .. + 3
      w.c.x = ld_stream_u32(codes + (size_t)(8 * gi + 4 * hh + 0) * H);
      w.c.y = ld_stream_u32(codes + (size_t)(8 * gi + 4 * hh + 1) * H);
      w.c.z = ld_stream_u32(codes + (size_t)(8 * gi + 4 * hh + 2) * H);
      w.c.w = ld_stream_u32(codes + (size_t)(8 * gi + 4 * hh + 3) * H);
    } else {  // words 4 gi + 2 hh .. + 1
      w.c.x = ld_stream_u32(codes + (size_t)(4 * gi + 2 * hh + 0) * H);
      w.c.y = ld_stream_u32(codes + (size_t)(4 * gi + 2 * hh + 1) * H);
      w.c.z = w.c.w = 0u;
    }
    w.sb = ld_stream_u32(reinterpret_cast<const uint32_t*>(rec + L.down_sb) + (size_t)gi * H + row);
  }
  return w;
}

// Dequantises a thread's share into the fp16 A tile.
template <int BITS>
__device__ __forceinline__ void tc_dequant(const TcRaw& w, uint8_t* a_tile) {
  const int t = threadIdx.x, r = t >> 1, hh = t & 1;
  float s, b;
  sb_true(w.sb, BITS, &s, &b);
  if (BITS == 4) {
    const uint32_t wd[4] = {w.c.x, w.c.y, w.c.z, w.c.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      float w8[8];
      dequant_word4(wd[q], s, b, w8);
      store_a8(a_tile, r, 4 * hh + q, w8);
    }
  } else {
    const uint32_t wd[2] = {w.c.x, w.c.y};
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      float w16[16];
      dequant_word2(wd[q], s, b, w16);
      store_a8(a_tile, r, 4 * hh + 2 * q, w16);
      store_a8(a_tile, r, 4 * hh + 2 * q + 1, w16 + 8);
    }
  }
}

// ------------------------------------------------------------- the GEMM --
constexpr int kTcStages = 3;  // shared-memory ring of A and B tiles
constexpr int kTcAhead = 4;   // steps of raw weight words held in registers ahead of use

template <int MODE, int BITS>
__device__ __forceinline__ TcRaw tc_raw_or_zero(const uint8_t* rec, int H, int I, int r0, int gi, int steps) {
  if (gi < steps) return tc_load_raw<MODE, BITS>(rec, H, I, r0, gi);
  TcRaw z;
  z.c = make_uint4(0u, 0u, 0u, 0u);
  z.sb = 0u;
  return z;
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// grid (max tensor-core items, M / 128), kTcThreads + 32 threads.  MODE 0:
// gate/up (M = 2 I, K = H), epilogue SwiGLU -> a[slot][n].  MODE 1: down
// (M = H, K = I) -> y[slot][row].  Warps 0..7 dequantise step s (one
// 64-input group) into ring stage s % 3 and arrive on full[stage]; warp 8
// (one thread) waits for the stage's A and token tile, issues the four
// products, commits them to done[stage] and requests the token tile of step
// s + 2.  Completion c of a stage's mbarriers belongs to step stage + 3 c,
// so every wait's parity is (s / 3) & 1.  Bounded waits: on expiry the CTA
// sets FMOE_STATUS_WAIT_TIMEOUT, waits (bounded) for its committed products
// and copies, frees its tensor memory and returns.
template <int MODE, int BITS>
__device__ __forceinline__ void tc_gemm_body(const ExpertSet& es, const int4 it, const uint8_t* rec,
                                             const uint8_t* __restrict__ staged, float* __restrict__ out,
                                             unsigned char* tsm, uint64_t* bar_b, uint64_t* bar_m, uint64_t* bar_f,
                                             uint32_t tmem, const int* s_slot, int* s_ok) {
  const int m = it.z, np = tc_np(m), N = 2 * np;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int K = MODE == 0 ? es.H : es.I;
  const int steps = K / 64;
  const int r0 = (int)blockIdx.y * kTcRows;
  const uint32_t b_bytes = (uint32_t)N * 128;  // one 64-input step of the staged tokens
  const uint8_t* bsrc = staged + (size_t)it.w * 4 * K;
  auto a_st = [&](int st) { return tsm + (size_t)st * kTcATile; };
  auto b_st = [&](int st) { return tsm + (size_t)kTcStages * kTcATile + (size_t)st * kTcMaxNp * 2 * 128; };
  auto par = [](int s) { return (uint32_t)((s / kTcStages) & 1); };
  if (warp < kTcThreads / 32) {
    // ---- producers: raw words of steps s .. s + 3 in four fixed register
    // sets, each refilled with step s + 4 right after its use
    TcRaw rw[kTcAhead];
#pragma unroll
    for (int i = 0; i < kTcAhead; ++i) rw[i] = tc_raw_or_zero<MODE, BITS>(rec, es.H, es.I, r0, i, steps);
    bool ok = true;
    for (int s0 = 0; s0 < steps && ok; s0 += kTcAhead) {
#pragma unroll
      for (int i = 0; i < kTcAhead; ++i) {
        const int s = s0 + i;
        if (!ok || s >= steps) break;
        const int st = s % kTcStages;
        if (s >= kTcStages && !mbar_wait(&bar_m[st], par(s - kTcStages))) {  // products of step s - 3 done
          ok = false;
          *s_ok = 0;
          break;
        }
        tc_dequant<BITS>(rw[i], a_st(st));
        rw[i] = tc_raw_or_zero<MODE, BITS>(rec, es.H, es.I, r0, s + kTcAhead, steps);
        fence_proxy_async();  // the generic-proxy A tile is read by the tensor cores
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar_f[st]);
      }
    }
  } else if (lane == 0) {
    // ---- issuer
    const uint32_t idesc = umma_idesc_f16(kTcRows, N);
    int last_commit = -1, b_issued = -1, b_waited = -1;
    auto issue_b = [&](int s) {
      const int st = s % kTcStages;
      b_issued = s;
      mbar_expect_tx(&bar_b[st], b_bytes);
      bulk_g2s(b_st(st), bsrc + (size_t)s * b_bytes, b_bytes, &bar_b[st]);
    };
    issue_b(0);
    if (steps > 1) issue_b(1);
    bool ok = true;
    for (int s = 0; s < steps; ++s) {
      const int st = s % kTcStages;
      if (!mbar_wait(&bar_f[st], par(s)) || !mbar_wait(&bar_b[st], par(s))) {
        ok = false;
        break;
      }
      b_waited = s;
      tc_fence_after();
      const uint32_t a0 = smem_u32(a_st(st)), b0 = smem_u32(b_st(st));
#pragma unroll
      for (int j = 0; j < 4; ++j) {  // K = 16 slices: two 8-input chunks each
        const uint64_t ad = umma_desc(a0 + (uint32_t)(2 * j) * (kTcRows / 8) * 128, (kTcRows / 8) * 128, 128);
        const uint64_t bd = umma_desc(b0 + (uint32_t)(2 * j) * (uint32_t)(N / 8) * 128, (uint32_t)(N / 8) * 128, 128);
        umma_f16(tmem, ad, bd, idesc, s > 0 || j > 0);
      }
      umma_commit(&bar_m[st]);
      last_commit = s;
      // token tile of step s + 2: its stage was read by the products of step s - 1
      if (s + 2 < steps) {
        if (s >= 1 && !mbar_wait(&bar_m[(s + 2) % kTcStages], par(s - 1))) {
          ok = false;
          break;
        }
        issue_b(s + 2);
      }
    }
    if (!ok) {
      *s_ok = 0;
      if (last_commit >= 0)  // products complete in order: the last one covers the rest
        (void)mbar_wait(&bar_m[last_commit % kTcStages], par(last_commit));
      for (int q = b_waited + 1; q <= b_issued; ++q)  // token tiles still in flight
        (void)mbar_wait(&bar_b[q % kTcStages], par(q));
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
        const float v = hi[i] + lo[i];
        if (MODE == 0) {
          const float partner = __shfl_xor_sync(0xffffffffu, v, 1);  // gate row 2n, up row 2n + 1
          if ((lane & 1) == 0 && t < m) out[(size_t)s_slot[t] * es.I + (r0 + row) / 2] = silu_mul(v, partner);
        } else if (t < m) {
          out[(size_t)s_slot[t] * es.H + r0 + row] = v;
        }
      }
    }
  }
  if (!ok && tid == 0) raise_status(FMOE_STATUS_WAIT_TIMEOUT);
}

template <int MODE>
__global__ void __launch_bounds__(kTcThreads + 32)
tc_gemm_kernel(ExpertSet es, GroupWork w, const uint8_t* __restrict__ staged, float* __restrict__ out) {
  extern __shared__ __align__(1024) unsigned char tsm[];
  __shared__ uint64_t bar_b[kTcStages], bar_m[kTcStages], bar_f[kTcStages];
  __shared__ uint32_t s_tmem;
  __shared__ int s_slot[kTcMaxNp];
  __shared__ int s_ok;
  if ((int)blockIdx.x >= w.n_items[1]) return;
  const int4 it = w.tc[blockIdx.x];
  const int g = it.x, m = it.z, N = 2 * tc_np(m);
  const int tid = threadIdx.x, warp = tid >> 5;
  uint32_t ncols = 32;
  while ((int)ncols < N) ncols <<= 1;
  for (int i = tid; i < m; i += blockDim.x) s_slot[i] = w.slots[w.offset[g] + it.y + i];
  if (tid == 0) {
    s_ok = 1;
    for (int i = 0; i < kTcStages; ++i) {
      mbar_init(&bar_b[i], 1);
      mbar_init(&bar_m[i], 1);
      mbar_init(&bar_f[i], kTcThreads / 32);
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
  int bits;
  const uint8_t* rec = group_record(es, g, &bits);
  if (bits == 4) tc_gemm_body<MODE, 4>(es, it, rec, staged, out, tsm, bar_b, bar_m, bar_f, tmem, s_slot, &s_ok);
  else tc_gemm_body<MODE, 2>(es, it, rec, staged, out, tsm, bar_b, bar_m, bar_f, tmem, s_slot, &s_ok);
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(ncols) : "memory");
  }
}

// Dynamic shared memory of tc_gemm_kernel: the ring of A and B tiles.
constexpr size_t tc_smem_bytes() { return kTcStages * ((size_t)kTcATile + (size_t)kTcMaxNp * 2 * 128); }

}  // namespace fmoe
