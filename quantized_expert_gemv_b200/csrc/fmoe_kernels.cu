// fmoe_kernels.cu -- sm_100a kernels and the C ABI of the quantised MoE
// expert forward (see include/fmoe.h for the contract of every entry point).
//
// Which kernels run a layer:
//   - one or two tokens (and up to fmoe_fused_max_tokens in pairs): the
//     persistent fused_stack_kernel (fmoe_fused.cuh), whole layers and
//     layer stacks in one cooperative launch;
//   - otherwise (or with fmoe_set_fused(0)), one kernel per step, in the
//     order one layer runs them:
//       router_partial_kernel  fp32 router rows x normed input, split along H
//       topk_kernel            sums the splits, warp top-k, softmax of the k
//                              selected logits, shared-expert sigmoid gate
//       gateup_kernel          dequantising gate/up products of every
//                              selected expert and the shared expert, fused
//                              SwiGLU (T = 1)
//       down_kernel            dequantising down product (T = 1)
//       combine_kernel         weighted combine + residual + shared gate,
//                              then the two-pass RMSNorm
//     with T > 1 the expert products group the slots by expert first
//     (fmoe_batched.cuh: integer-dot GEMVs; fmoe_tc.cuh: tcgen05 GEMM for
//     experts with fmoe_tc_min_tokens or more tokens);
//   - off the layer: the packer (pack_codes_kernel, pack_sb_kernel) and the
//     quantiser (quantize_groups_kernel); the host expert tier's cache
//     (fmoe_cache.cuh).
// Source pages: "What is Flash-MoE?" (a2a-mcp.org), sections "Understanding
// Mixture-of-Experts" (top-4 of 512 plus one shared expert),
// "2. FMA-optimised dequantisation kernels" and "3. Hand-tuned Metal compute
// shaders" (dequantising matrix-vector products, fused SwiGLU, MoE combine +
// residual + sigmoid gating, two-pass RMSNorm feeding the next layer).
#include <atomic>
#include <cstdint>
#include <cstring>
#include <mutex>

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "fmoe.h"
#include "fmoe_device.cuh"
#include "fmoe_fused.cuh"
#include "fmoe_layout.h"

namespace fmoe {

constexpr int kMaxK = 8;
constexpr int kMaxE = 1024;
constexpr int kRouterSplit = 4;  // router rows are split in 4 along H
constexpr int kTokChunk = 8;     // tokens per router launch
constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;

// ------------------------------------------------------------ router ----
// part[t][row][s] = sum over split s of W[row] . xn[t]; row E is the shared
// expert's gate vector (skipped when w_sg is null).  One warp per (row, split).
__global__ void __launch_bounds__(kThreads)
router_partial_kernel(const float* __restrict__ xn, const float* __restrict__ w_router,
                      const float* __restrict__ w_sg, int T, int H, int E,
                      float* __restrict__ part) {
  const int warp = (int)((blockIdx.x * blockDim.x + threadIdx.x) >> 5);
  const int lane = threadIdx.x & 31;
  if (warp >= (E + (w_sg ? 1 : 0)) * kRouterSplit) return;
  const int row = warp / kRouterSplit, sp = warp % kRouterSplit;
  const float* w = row < E ? w_router + (size_t)row * H : w_sg;
  const int hs = H / kRouterSplit, c0 = sp * hs;
  float acc[kTokChunk];
#pragma unroll
  for (int t = 0; t < kTokChunk; ++t) acc[t] = 0.f;
#pragma unroll 4
  for (int c = lane * 4; c < hs; c += 128) {
    const float4 wv = ld_stream_f4(w + c0 + c);
#pragma unroll
    for (int t = 0; t < kTokChunk; ++t) {
      if (t < T) {
        const float4 xv = __ldg(reinterpret_cast<const float4*>(xn + (size_t)t * H + c0 + c));
        acc[t] = fmaf(wv.x, xv.x, acc[t]);
        acc[t] = fmaf(wv.y, xv.y, acc[t]);
        acc[t] = fmaf(wv.z, xv.z, acc[t]);
        acc[t] = fmaf(wv.w, xv.w, acc[t]);
      }
    }
  }
#pragma unroll
  for (int t = 0; t < kTokChunk; ++t) {
    if (t < T) {
      const float v = warp_sum(acc[t]);
      if (lane == 0) part[((size_t)t * (E + 1) + row) * kRouterSplit + sp] = v;
    }
  }
}

// Orders (value, index): larger value first, NaN below every number, equal
// values (including +0 / -0) to the lower index; index < 0 marks "none".
__device__ __forceinline__ bool route_better(float av, int ai, float bv, int bi) {
  if (ai < 0) return false;
  if (bi < 0) return true;
  const bool an = isnan(av), bn = isnan(bv);
  if (an || bn) return an && bn ? ai < bi : bn;
  if (av != bv) return av > bv;
  return ai < bi;
}

// One warp per token: logits (sum of the splits, or given), top-k, softmax
// over the selected logits, and the shared gate sigmoid(z).
__global__ void __launch_bounds__(128)
topk_kernel(const float* __restrict__ part, const float* __restrict__ logits_in, int T, int E,
            int k, float* __restrict__ logits, int32_t* __restrict__ ids,
            float* __restrict__ weights, float* __restrict__ gamma) {
  __shared__ float lg[4][kMaxE];
  const int wi = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * 4 + wi;
  if (t >= T) return;
  bool nan_seen = false;
  for (int e = lane; e < E; e += 32) {
    float v;
    if (part) {
      const float* p = part + ((size_t)t * (E + 1) + e) * kRouterSplit;
      v = p[0];
#pragma unroll
      for (int s = 1; s < kRouterSplit; ++s) v += p[s];
      logits[(size_t)t * E + e] = v;
    } else {
      v = logits_in[(size_t)t * E + e];
    }
    nan_seen |= isnan(v);
    lg[wi][e] = v;
  }
  if (part && gamma && lane == 0) {
    const float* p = part + ((size_t)t * (E + 1) + E) * kRouterSplit;
    float z = p[0];
#pragma unroll
    for (int s = 1; s < kRouterSplit; ++s) z += p[s];
    gamma[t] = 1.f / (1.f + expf(-z));
  }
  if (__any_sync(0xffffffffu, nan_seen) && lane == 0) raise_status(FMOE_STATUS_NAN_LOGIT);
  __syncwarp();
  uint32_t taken = 0;  // bit i: element lane + 32 i already selected
  float selv[kMaxK];
  int seli[kMaxK];
  for (int r = 0; r < k; ++r) {
    float bv = 0.f;
    int bi = -1;
    for (int i = 0, e = lane; e < E; ++i, e += 32) {
      if (taken & (1u << i)) continue;
      const float v = lg[wi][e];
      if (route_better(v, e, bv, bi)) { bv = v; bi = e; }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (route_better(ov, oi, bv, bi)) { bv = ov; bi = oi; }
    }
    if (bi >= 0 && (bi & 31) == lane) taken |= 1u << (bi >> 5);
    selv[r] = bv;
    seli[r] = bi;
  }
  float m = -INFINITY;
  for (int r = 0; r < k; ++r)
    if (!isnan(selv[r])) m = fmaxf(m, selv[r]);
  float p[kMaxK];
  float z = 0.f;
  for (int r = 0; r < k; ++r) {
    p[r] = isnan(selv[r]) ? 0.f : expf(selv[r] - m);
    z += p[r];
  }
  if (lane < k) {
    float pv = 0.f;
    int iv = 0;
    for (int r = 0; r < k; ++r)
      if (r == lane) { pv = p[r]; iv = seli[r]; }
    ids[(size_t)t * k + lane] = iv;
    weights[(size_t)t * k + lane] = z > 0.f ? pv / z : 0.f;
  }
}

// ---------------------------------------------------------- experts ----
struct ExpertSet {
  const uint8_t* experts;  // E records
  const uint64_t* rec_table;  // when set: device address of routed record id (an expert cache's slots)
  const uint8_t* shared;   // one record
  size_t rec_bytes, shared_rec_bytes;
  int bits, shared_bits;
  int H, I, E, k;
};

// Resolves slot j of token t to a record; returns nullptr for a bad id.
__device__ __forceinline__ const uint8_t* slot_record(const ExpertSet& es, const int32_t* ids,
                                                      int t, int j, int* bits) {
  if (j == es.k) {
    *bits = es.shared_bits;
    return es.shared;
  }
  const int id = ids[(size_t)t * es.k + j];
  *bits = es.bits;
  if (id < 0 || id >= es.E) return nullptr;
  if (es.rec_table) return reinterpret_cast<const uint8_t*>(es.rec_table[id]);
  return es.experts + (size_t)id * es.rec_bytes;
}

// Gate/up rows of one record for one token: each warp owns units of
// 32 / lanes_per_row row pairs; a lane owns whole groups of both the gate and
// the up row of its pair, so the staged x it reads serves both.
template <int BITS>
__device__ __forceinline__ void gateup_rows(const uint8_t* rec, const ExpertSet& es,
                                            const StagedX& sx, float* __restrict__ a_out,
                                            int unit0, int unit1) {
  const int H = es.H;
  const int ng = H / 64;
  const int lpr = ng < 32 ? ng : 32;  // lanes per row
  const int gpl = ng / lpr;           // groups per lane
  const int ppu = 32 / lpr;           // row pairs per unit
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int ps = lane / lpr, lg = lane % lpr;
  const RecordLayout L = record_layout(BITS, H, es.I);
  const uint8_t* codes = rec + L.gu_codes;
  const uint32_t* sbw = reinterpret_cast<const uint32_t*>(rec + L.gu_sb);
  for (int u = unit0 + warp; u < unit1; u += kWarps) {
    const int n = u * ppu + ps;
    const uint8_t* rg = codes + (size_t)(2 * n) * L.gu_row_bytes;
    const uint8_t* ru = rg + L.gu_row_bytes;
    float yg = 0.f, yu = 0.f;
    for (int m = 0; m < gpl; ++m) {
      const int g = lg + m * lpr;
      const GroupCodes<BITS> cg = load_group<BITS>(rg, ng, g);
      const GroupCodes<BITS> cu = load_group<BITS>(ru, ng, g);
      const uint32_t sg = ld_stream_u32(sbw + (size_t)(2 * n) * ng + g);
      const uint32_t su = ld_stream_u32(sbw + (size_t)(2 * n + 1) * ng + g);
      uint4 xv[8];
      uint2 xl[8];
      load_xv(sx, ng, g, xv, xl);
      const float d = sx.delta[g], xs = sx.xsum[g];
      yg = group_epilogue(yg, sg, group_dot<BITS>(cg, xv, xl), d, xs);
      yu = group_epilogue(yu, su, group_dot<BITS>(cu, xv, xl), d, xs);
    }
    for (int o = lpr >> 1; o > 0; o >>= 1) {
      yg += __shfl_xor_sync(0xffffffffu, yg, o);
      yu += __shfl_xor_sync(0xffffffffu, yu, o);
    }
    if (lg == 0) a_out[n] = silu_mul(yg, yu);
  }
}

// Down product of one record for one hidden row: the column blocks of each
// 64-group of the intermediate dimension (8 words of 4-bit codes or 4 of
// 2-bit codes, one per block), accumulated exactly in int32 and scaled once
// per group.  Consecutive threads take consecutive rows, so every load of a
// warp is one contiguous 128-byte line.
template <int BITS>
__device__ __forceinline__ float down_row_cols(const uint8_t* rec, const ExpertSet& es, const StagedX& sx,
                                               int row) {
  const int H = es.H, I = es.I, ngI = I / 64;
  constexpr int kWpg = BITS == 4 ? 8 : 4;  // column blocks (words) per group
  const RecordLayout L = record_layout(BITS, H, I);
  const uint32_t* codes = reinterpret_cast<const uint32_t*>(rec + L.down_codes) + row;
  const uint32_t* sbw = reinterpret_cast<const uint32_t*>(rec + L.down_sb) + row;
  float y = 0.f;
  for (int g = 0; g < ngI; ++g) {
    uint32_t w[kWpg];
#pragma unroll
    for (int b = 0; b < kWpg; ++b) w[b] = ld_stream_u32(codes + (size_t)(g * kWpg + b) * H);
    const uint32_t sb = ld_stream_u32(sbw + (size_t)g * H);
    Acc2 acc{0, 0};
#pragma unroll
    for (int b = 0; b < kWpg; ++b) {
      if (BITS == 4) acc = acc + word_dot4(w[b], sx.xs[b * ngI + g], sx.xl[b * ngI + g]);
      else
        acc = acc + word_dot2(w[b], sx.xs[(2 * b) * ngI + g], sx.xs[(2 * b + 1) * ngI + g], sx.xl[(2 * b) * ngI + g],
                              sx.xl[(2 * b + 1) * ngI + g]);
    }
    y = group_epilogue(y, sb, acc, sx.delta[g], sx.xsum[g]);
  }
  return y;
}

__device__ __forceinline__ void unit_range(int n_units, int* u0, int* u1) {
  const int per = (n_units + (int)gridDim.x - 1) / (int)gridDim.x;
  *u0 = (int)blockIdx.x * per;
  *u1 = min(n_units, *u0 + per);
}

// grid (row blocks, T * (k + 1) slots): slot = t * (k + 1) + j, j == k the shared expert.
__global__ void __launch_bounds__(kThreads)
gateup_kernel(ExpertSet es, const float* __restrict__ xn, const int32_t* __restrict__ ids,
              float* __restrict__ a, const float* __restrict__ w_sg, float* __restrict__ gamma) {
  extern __shared__ __align__(128) unsigned char smem[];
  const int slot = blockIdx.y, t = slot / (es.k + 1), j = slot % (es.k + 1);
  int bits;
  const uint8_t* rec = slot_record(es, ids, t, j, &bits);
  const int ng = es.H / 64, lpr = ng < 32 ? ng : 32;
  int u0, u1;
  unit_range(es.I / (32 / lpr), &u0, &u1);
  float* a_out = a + (size_t)slot * es.I;
  if (!rec) {
    if (threadIdx.x == 0 && blockIdx.x == 0) raise_status(FMOE_STATUS_BAD_EXPERT_ID);
    for (int i = u0 * (32 / lpr) + (int)threadIdx.x; i < u1 * (32 / lpr); i += blockDim.x) a_out[i] = 0.f;
    return;
  }
  const StagedX sx = staged_x_at(smem, es.H);
  stage_x(xn + (size_t)t * es.H, es.H, sx);
  __syncthreads();
  if (gamma && j == es.k && blockIdx.x == 0 && threadIdx.x < 32) {
    const float* x = xn + (size_t)t * es.H;
    float z = 0.f;
    for (int c = threadIdx.x * 4; c < es.H; c += 128) {
      const float4 w = __ldg(reinterpret_cast<const float4*>(w_sg + c));
      const float4 v = __ldg(reinterpret_cast<const float4*>(x + c));
      z = fmaf(w.x, v.x, z);
      z = fmaf(w.y, v.y, z);
      z = fmaf(w.z, v.z, z);
      z = fmaf(w.w, v.w, z);
    }
    z = warp_sum(z);
    if (threadIdx.x == 0) gamma[t] = 1.f / (1.f + expf(-z));
  }
  if (bits == 4)
    gateup_rows<4>(rec, es, sx, a_out, u0, u1);
  else
    gateup_rows<2>(rec, es, sx, a_out, u0, u1);
}

// grid (H / kDownThreads, T * (k + 1) slots); one hidden row per thread.
constexpr int kDownThreads = 128;
__global__ void __launch_bounds__(kDownThreads)
down_kernel(ExpertSet es, const int32_t* __restrict__ ids, const float* __restrict__ a,
            float* __restrict__ y) {
  extern __shared__ __align__(128) unsigned char smem[];
  const int slot = blockIdx.y, t = slot / (es.k + 1), j = slot % (es.k + 1);
  int bits;
  const uint8_t* rec = slot_record(es, ids, t, j, &bits);
  const int row = (int)blockIdx.x * kDownThreads + (int)threadIdx.x;
  float* y_out = y + (size_t)slot * es.H;
  if (!rec) {
    if (row < es.H) y_out[row] = 0.f;
    return;
  }
  const StagedX sx = staged_x_at(smem, es.I);
  stage_x(a + (size_t)slot * es.I, es.I, sx);
  __syncthreads();
  if (row >= es.H) return;
  y_out[row] = bits == 4 ? down_row_cols<4>(rec, es, sx, row) : down_row_cols<2>(rec, es, sx, row);
}

}  // namespace fmoe

#include "fmoe_batched.cuh"
#include "fmoe_tc.cuh"

namespace fmoe {

// ---------------------------------------------------------- combine ----
__device__ __forceinline__ float block_sum(float v, float* red) {
  v = warp_sum(v);
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();
  if (lane == 0) red[w] = v;
  __syncthreads();
  float s = 0.f;
  for (int i = 0; i < (int)(blockDim.x >> 5); ++i) s += red[i];
  return s;
}

// One CTA per token.  With H <= 4 kCombVec kThreads (and H % 4 == 0) each
// thread keeps its h' values in registers: all of its loads go out at once
// and the norm pass reads nothing back; otherwise a strided two-pass loop.
constexpr int kCombVec = 4;
__global__ void __launch_bounds__(kThreads)
combine_kernel(const float* __restrict__ y, const float* __restrict__ weights,
               const float* __restrict__ gamma, const float* h, const float* __restrict__ norm_w,
               float eps, int k, int H, float* h_out, float* __restrict__ xn_out) {
  __shared__ float red[kWarps];
  const int t = blockIdx.x;
  const float* yt = y + (size_t)t * (k + 1) * H;
  float p[kMaxK];
#pragma unroll
  for (int j = 0; j < kMaxK; ++j) p[j] = j < k ? weights[(size_t)t * k + j] : 0.f;
  const float gm = gamma[t];
  float ss = 0.f;
  if (H % 4 == 0 && H <= 4 * kCombVec * (int)blockDim.x) {
    const int nv = H / 4;
    float4 v[kCombVec];
#pragma unroll
    for (int u = 0; u < kCombVec; ++u) {
      const int i4 = threadIdx.x + u * blockDim.x;
      if (i4 < nv) {
        float4 acc = reinterpret_cast<const float4*>(h + (size_t)t * H)[i4];
        const float4 ys = __ldcg(reinterpret_cast<const float4*>(yt + (size_t)k * H) + i4);
#pragma unroll
        for (int j = 0; j < kMaxK; ++j) {
          if (j < k) {
            const float4 yj = __ldcg(reinterpret_cast<const float4*>(yt + (size_t)j * H) + i4);
            acc.x = fmaf(p[j], yj.x, acc.x);
            acc.y = fmaf(p[j], yj.y, acc.y);
            acc.z = fmaf(p[j], yj.z, acc.z);
            acc.w = fmaf(p[j], yj.w, acc.w);
          }
        }
        acc.x = fmaf(gm, ys.x, acc.x);
        acc.y = fmaf(gm, ys.y, acc.y);
        acc.z = fmaf(gm, ys.z, acc.z);
        acc.w = fmaf(gm, ys.w, acc.w);
        v[u] = acc;
        reinterpret_cast<float4*>(h_out + (size_t)t * H)[i4] = acc;
        ss = fmaf(acc.x, acc.x, ss);
        ss = fmaf(acc.y, acc.y, ss);
        ss = fmaf(acc.z, acc.z, ss);
        ss = fmaf(acc.w, acc.w, ss);
      }
    }
    ss = block_sum(ss, red);
    const float r = 1.f / sqrtf(ss / (float)H + eps);
#pragma unroll
    for (int u = 0; u < kCombVec; ++u) {
      const int i4 = threadIdx.x + u * blockDim.x;
      if (i4 < nv) {
        const float4 nw = __ldg(reinterpret_cast<const float4*>(norm_w) + i4);
        reinterpret_cast<float4*>(xn_out + (size_t)t * H)[i4] =
            make_float4(v[u].x * r * nw.x, v[u].y * r * nw.y, v[u].z * r * nw.z, v[u].w * r * nw.w);
      }
    }
    return;
  }
  for (int i = threadIdx.x; i < H; i += blockDim.x) {
    float v = h[(size_t)t * H + i];
    for (int j = 0; j < k; ++j) v = fmaf(p[j], yt[(size_t)j * H + i], v);
    v = fmaf(gm, yt[(size_t)k * H + i], v);
    h_out[(size_t)t * H + i] = v;
    ss = fmaf(v, v, ss);
  }
  ss = block_sum(ss, red);
  const float r = 1.f / sqrtf(ss / (float)H + eps);
  for (int i = threadIdx.x; i < H; i += blockDim.x)
    xn_out[(size_t)t * H + i] = h_out[(size_t)t * H + i] * r * norm_w[i];
}

// ---------------------------------------------------------- quantiser ----
// Stored-format quantiser: fp32 weights, 64-group min/max affine codes with
// bf16 scale and bias (the offline conversion the pages' conclusion
// mentions; "What is Flash-MoE?", conclusion).  One warp per group, lane l
// holds inputs 2l, 2l+1.  Every decision in fp32 with correctly rounded
// operations: lo = min (+0 for -0), hi = max, s = (hi - lo) / (2^bits - 1),
// S = bf16(s), B = bf16(lo) (round to nearest even), q = rint((w - B) / S)
// clamped to [0, 2^bits - 1], q = 0 where S = 0.
__global__ void __launch_bounds__(256)
quantize_groups_kernel(const float* __restrict__ w, size_t n_groups, int bits, uint8_t* __restrict__ q,
                       uint16_t* __restrict__ scale, uint16_t* __restrict__ bias) {
  const int lane = threadIdx.x & 31;
  const size_t nw = ((size_t)gridDim.x * blockDim.x) >> 5;
  const float qmax = (float)((1 << bits) - 1);
  for (size_t g = ((size_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; g < n_groups; g += nw) {
    const float2 v = reinterpret_cast<const float2*>(w + g * 64)[lane];
    float lo = fminf(v.x, v.y), hi = fmaxf(v.x, v.y);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
      hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
    }
    lo = __fadd_rn(lo, 0.0f);
    const __nv_bfloat16 sb = __float2bfloat16_rn(__fdiv_rn(__fsub_rn(hi, lo), qmax));
    const __nv_bfloat16 bb = __float2bfloat16_rn(lo);
    const float S = __bfloat162float(sb), B = __bfloat162float(bb);
    auto code = [&](float x) -> uint32_t {
      if (!(S > 0.f)) return 0u;
      const float c = fminf(fmaxf(rintf(__fdiv_rn(__fsub_rn(x, B), S)), 0.f), qmax);
      return (uint32_t)c;
    };
    reinterpret_cast<uchar2*>(q + g * 64)[lane] = make_uchar2((unsigned char)code(v.x), (unsigned char)code(v.y));
    if (lane == 0) {
      scale[g] = __bfloat16_as_ushort(sb);
      bias[g] = __bfloat16_as_ushort(bb);
    }
  }
}

// ------------------------------------------------------- device packer ----
// One thread per 16-byte chunk of packed codes.  Gate/up: packed row pr of
// an expert (pr = 2n + m: logical matrix m, row n; H inputs), chunk p of the
// row.  Down: column block nb, rows 4j .. 4j + 3 (one word each).
template <int BITS>
__global__ void pack_codes_kernel(const uint8_t* __restrict__ q, int n_experts, int H, int I,
                                  uint8_t* __restrict__ out) {
  const RecordLayout L = record_layout(BITS, H, I);
  const size_t n = (size_t)H * I;
  const int gu_chunks = H * BITS / 128;
  constexpr int per_word = 32 / BITS, per_byte = 8 / BITS;
  const size_t gu_total = (size_t)2 * I * gu_chunks;
  const size_t per_expert = gu_total + (size_t)(I / per_word) * (H / 4);
  const size_t total = per_expert * n_experts;
  for (size_t c = blockIdx.x * (size_t)blockDim.x + threadIdx.x; c < total; c += (size_t)gridDim.x * blockDim.x) {
    const size_t e = c / per_expert;
    size_t r = c % per_expert;
    const uint8_t* in[4];  // the 32 / BITS inputs of each of the four words
    uint8_t* dst;
    if (r < gu_total) {
      const int pr = (int)(r / gu_chunks);
      const int p = (int)(r % gu_chunks);
      const uint8_t* src = q + e * 3 * n + (size_t)(pr & 1) * n + (size_t)(pr >> 1) * H;
      dst = out + e * L.bytes + L.gu_codes + (size_t)pr * L.gu_row_bytes + (size_t)p * 16;
      const int ng = H / 64;
      int g, h;
      if (BITS == 2) {
        g = p;
        h = 0;
      } else {
        const int seg = ng < 32 ? ng : 32;
        const int s = p / (2 * seg), rem = p % (2 * seg);
        h = rem / seg;
        g = s * seg + rem % seg;
      }
#pragma unroll
      for (int w = 0; w < 4; ++w) in[w] = src + g * 64 + h * 32 + w * per_word;  // h is 0 for 2-bit
    } else {
      r -= gu_total;
      const int nb = (int)(r / (H / 4)), row0 = (int)(r % (H / 4)) * 4;
      dst = out + e * L.bytes + L.down_codes + ((size_t)nb * H + row0) * 4;
#pragma unroll
      for (int w = 0; w < 4; ++w) in[w] = q + e * 3 * n + 2 * n + (size_t)(row0 + w) * I + (size_t)nb * per_word;
    }
    uint32_t words[4];
    bool bad = false;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      uint32_t word = 0;
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < per_byte; ++b) {
          const uint32_t v = in[w][4 * b + a];
          bad |= v >= (1u << BITS);
          word |= (v & ((1u << BITS) - 1u)) << ((per_byte * a + b) * BITS);
        }
      words[w] = word;
    }
    if (bad) {
      raise_status(FMOE_STATUS_BAD_PACK_INPUT);
      words[0] = words[1] = words[2] = words[3] = 0u;
    }
    *reinterpret_cast<uint4*>(dst) = make_uint4(words[0], words[1], words[2], words[3]);
  }
}

// One thread per scale-bias word.
__global__ void pack_sb_kernel(const uint16_t* __restrict__ scale, const uint16_t* __restrict__ bias,
                               int bits, int n_experts, int H, int I, uint8_t* __restrict__ out) {
  const RecordLayout L = record_layout(bits, H, I);
  const size_t ng = (size_t)3 * H * I / 64;
  const size_t gu = (size_t)2 * I * (H / 64);
  const int shift = bits == 4 ? 4 : 6;
  for (size_t c = blockIdx.x * (size_t)blockDim.x + threadIdx.x; c < ng * n_experts; c += (size_t)gridDim.x * blockDim.x) {
    const size_t e = c / ng, r = c % ng;
    size_t src;  // logical index within the expert
    uint32_t* dst;
    if (r < gu) {
      const size_t gpr = H / 64, pr = r / gpr, g = r % gpr;
      src = (pr & 1) * ((size_t)I * gpr) + (pr >> 1) * gpr + g;
      dst = reinterpret_cast<uint32_t*>(out + e * L.bytes + L.gu_sb) + r;
    } else {
      src = r;
      const size_t gpr = I / 64, rr = r - gu, row = rr / gpr, g = rr % gpr;
      dst = reinterpret_cast<uint32_t*>(out + e * L.bytes + L.down_sb) + g * H + row;
    }
    const uint16_t sv = scale[e * ng + src], bv = bias[e * ng + src];
    // exact scaling by 2^-shift of a bf16 value (normal, finite, no underflow)
    const uint32_t ex = (sv >> 7) & 0xFFu;
    uint16_t ps;
    bool ok = true;
    if ((sv & 0x7FFFu) == 0) ps = sv;
    else if (ex == 0 || ex == 0xFFu || (int)ex - shift <= 0) { ps = 0; ok = false; }
    else ps = (uint16_t)((sv & 0x807Fu) | ((ex - shift) << 7));
    if (!ok) raise_status(FMOE_STATUS_BAD_PACK_INPUT);
    *dst = ok ? ((uint32_t)ps | ((uint32_t)bv << 16)) : 0u;
  }
}

// ------------------------------------------------------- host helpers ----
struct WsLayout {
  size_t sync, x_logit, x_ss, x_h, x_part, grp, part, logits, ids, weights, gamma, a, y, bytes;
  size_t g_count, g_offset, g_slots, g_nitems, g_items, g_bitems, g_tc, g_xs;  // inside grp
  size_t tcx, tca;  // staged fp16 inputs of the tensor-core items (0 bytes when T < kTcMinTokens)
  size_t tsc, rsc, amax;  // their staging scales (tokens, staged rows) and rows' max |a|
};

// Upper bound of the tensor-core items' token rows (sum of tokens rounded up to 8).
static size_t tc_np_bound(int T, int k) {
  if (T < kTcMinTokens) return 0;
  return (size_t)T * (k + 1) + 8 * (size_t)group_max_tc(T, k, kTcMinTokens);
}

static inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

static WsLayout ws_layout(int H, int I, int E, int k, int T) {
  WsLayout w;
  w.sync = 0;  // grid-barrier counter, exit counter and epoch of the fused kernel
  // exchange buffers of the fused kernel (logit exchange words, fp32
  // partial outputs and h', for up to kFusedMaxNT tokens), at offsets and
  // sizes that do not depend on the shape or T: no other kernel writes there
  size_t o = 4096;
  w.x_logit = o;
  o = align_up(o + (size_t)kFusedMaxNT * kXLogitStride * 8, 256);
  w.x_ss = o;
  o = align_up(o + (size_t)kFusedMaxNT * kXSsStride * 4, 256);
  w.x_h = o;
  o = align_up(o + (size_t)kFusedMaxNT * kXHStride * 4, 256);
  w.x_part = o;
  o = align_up(o + (size_t)kFusedMaxNT * kXPartStride * 4, 256);
  // expert groups of the T > 1 path
  w.grp = o;
  w.g_count = o;
  o = align_up(o + (size_t)(E + 1) * 4, 16);
  w.g_offset = o;
  o = align_up(o + (size_t)(E + 2) * 4, 16);
  w.g_slots = o;
  o = align_up(o + (size_t)T * (k + 1) * 4, 16);
  w.g_nitems = o;
  o = align_up(o + 4 * (2 + kGrpBuckets), 16);
  w.g_items = o;
  o = align_up(o + (size_t)group_max_items(T, k, E) * 16, 16);
  w.g_bitems = o;
  o = align_up(o + (size_t)kGrpBuckets * group_max_items(T, k, E) * 16, 16);
  w.g_xs = o;  // every token's staged input (T > 1)
  o = align_up(o + (T > 1 ? (size_t)T * ((staged_x_bytes(H) + 15) & ~(size_t)15) : 0), 16);
  w.g_tc = o;
  o = align_up(o + (size_t)group_max_tc(T, k, kTcMinTokens) * 16, 256);
  w.tcx = o;
  o = align_up(o + tc_np_bound(T, k) * 4 * H, 256);
  w.tca = o;
  o = align_up(o + tc_np_bound(T, k) * 4 * I, 256);
  w.tsc = o;
  o = align_up(o + (size_t)T * 4, 256);
  w.rsc = o;
  o = align_up(o + tc_np_bound(T, k) * 4, 256);
  w.amax = o;
  o = align_up(o + tc_np_bound(T, k) * 4, 256);
  w.part = o;
  o = align_up(o + (size_t)T * (E + 1) * kRouterSplit * 4, 256);
  w.logits = o;
  o = align_up(o + (size_t)T * E * 4, 256);
  w.ids = o;
  o = align_up(o + (size_t)T * k * 4, 256);
  w.weights = o;
  o = align_up(o + (size_t)T * k * 4, 256);
  w.gamma = o;
  o = align_up(o + (size_t)T * 4, 256);
  w.a = o;
  o = align_up(o + (size_t)T * (k + 1) * I * 4, 256);
  w.y = o;
  o = align_up(o + (size_t)T * (k + 1) * H * 4, 256);
  w.bytes = o;
  return w;
}

// One layer's record of a stack trace (fmoe_stack_forward_trace): sections
// in the order of the FMOE_TRACE_* constants, each 256-byte aligned.
struct TraceLayout {
  size_t off[7];
  size_t bytes;
};

static TraceLayout trace_layout(int H, int I, int E, int k, int T) {
  const size_t sz[7] = {(size_t)T * H * 4, (size_t)T * E * 4, (size_t)T * k * 4, (size_t)T * k * 4,
                        (size_t)T * 4,     (size_t)T * (k + 1) * I * 4, (size_t)T * H * 4};
  TraceLayout t;
  size_t o = 0;
  for (int i = 0; i < 7; ++i) {
    t.off[i] = o;
    o = align_up(o + sz[i], 256);
  }
  t.bytes = o;
  return t;
}

static inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// The device ranges [a, a + na) and [b, b + nb) share no byte.  The layer and
// stack calls read h and xn and write h' and xn' over them in place, so their
// token rows must be apart (the same buffer for both would give xn' in place
// of h').
static inline bool disjoint(const void* a, size_t na, const void* b, size_t nb) {
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x + na <= y || y + nb <= x;
}
static inline bool disjoint(const void* a, const void* b, size_t bytes) { return disjoint(a, bytes, b, bytes); }

static bool desc_valid(const fmoe_layer_desc* d) {
  return d && d->hidden > 0 && d->inter > 0 && d->n_experts >= 1 && d->n_experts <= kMaxE &&
         d->top_k >= 1 && d->top_k <= kMaxK && d->top_k <= d->n_experts && d->eps >= 0.f;
}

static bool desc_supported(const fmoe_layer_desc* d) {
  return shape_supported(d->bits, d->hidden, d->inter, d->group) &&
         shape_supported(d->shared_bits, d->hidden, d->inter, d->group);
}

static int weights_check(const fmoe_layer_weights* lw) {
  if (!lw || !desc_valid(&lw->desc)) return FMOE_ERR_INVALID_ARG;
  if (!desc_supported(&lw->desc)) return FMOE_ERR_UNSUPPORTED;
  const void* ps[] = {lw->experts, lw->shared, lw->w_router, lw->w_shared_gate, lw->norm_w};
  for (const void* p : ps)
    if (!p || !aligned16(p)) return FMOE_ERR_INVALID_ARG;
  return FMOE_OK;
}

static ExpertSet expert_set(const fmoe_layer_weights* lw) {
  const fmoe_layer_desc& d = lw->desc;
  ExpertSet es;
  es.experts = static_cast<const uint8_t*>(lw->experts);
  es.rec_table = nullptr;
  es.shared = static_cast<const uint8_t*>(lw->shared);
  es.rec_bytes = record_layout(d.bits, d.hidden, d.inter).bytes;
  es.shared_rec_bytes = record_layout(d.shared_bits, d.hidden, d.inter).bytes;
  es.bits = d.bits;
  es.shared_bits = d.shared_bits;
  es.H = d.hidden;
  es.I = d.inter;
  es.E = d.n_experts;
  es.k = d.top_k;
  return es;
}

static inline int cuda_rc(cudaError_t e) { return e == cudaSuccess ? FMOE_OK : FMOE_ERR_CUDA; }

static int launch_router(const float* xn, const float* w_router, const float* w_sg, int T, int H,
                         int E, float* part, cudaStream_t st) {
  const int warps = (E + (w_sg ? 1 : 0)) * kRouterSplit;
  const int blocks = (warps + kWarps - 1) / kWarps;
  for (int t0 = 0; t0 < T; t0 += kTokChunk) {
    const int nt = T - t0 < kTokChunk ? T - t0 : kTokChunk;
    router_partial_kernel<<<blocks, kThreads, 0, st>>>(xn + (size_t)t0 * H, w_router, w_sg, nt, H, E,
                                                      part + (size_t)t0 * (E + 1) * kRouterSplit);
  }
  return cuda_rc(cudaGetLastError());
}

static int launch_topk(const float* part, const float* logits_in, int T, int E, int k, float* logits,
                       int32_t* ids, float* weights, float* gamma, cudaStream_t st) {
  topk_kernel<<<(T + 3) / 4, 128, 0, st>>>(part, logits_in, T, E, k, logits, ids, weights, gamma);
  return cuda_rc(cudaGetLastError());
}

// Tensor-core products for groups of >= kTcMinTokens tokens (a process-wide
// switch; calls from several host threads read it while one may set it).
static std::atomic<int> g_tc_enabled{1};

// Dynamic shared memory above the default 48 KB for a kernel, set once per
// device (under a lock: calls may come from several host threads).
static bool smem_optin(const void* fn, size_t bytes, int slot) {
  static size_t done[64][32];
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
  std::lock_guard<std::mutex> lock(mu);
  if (done[dev][slot] >= bytes) return true;
  if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes) != cudaSuccess) return false;
  done[dev][slot] = bytes;
  return true;
}

// Expert forward of T tokens.  With T >= 2 and a group workspace the slots
// are grouped by expert first (each expert's weights read once per step);
// otherwise one CTA column per slot.
template <int MB>
static bool grp_optin(size_t gu_smem, size_t dn_smem, int b) {
  return smem_optin(reinterpret_cast<const void*>(&gateup_group_kernel<MB>), gu_smem, 8 + b) &&
         smem_optin(reinterpret_cast<const void*>(&down_group_kernel<MB>), dn_smem, 12 + b);
}

// Small items (MB <= 4) go through the bulk-copied kernel when a row pair
// is whole warp-widths of groups (H / 64 >= 32) and its ring fits.
template <int MB>
static bool gu_bulk_ok(const ExpertSet& es) {
  if (MB > 4 || es.H / 64 < 32) return false;
  return smem_optin(reinterpret_cast<const void*>(&gateup_bulk_kernel<MB>), gu_bulk_smem(MB, es.H, 4), 16 + MB);
}

template <int MB>
static void grp_launch_gu(const ExpertSet& es, const GroupWork& gw, int b, int items, int grid, const float* xn,
                          const unsigned char* xs, float* a, const float* w_sg, float* gamma, size_t sxs,
                          cudaStream_t st) {
  if (gu_bulk_ok<MB>(es)) {
    gateup_bulk_kernel<(MB <= 4 ? MB : 4)><<<dim3(grid, gu_split(MB)), kGrpThreads, gu_bulk_smem(MB, es.H, 4), st>>>(
        es, gw, b, items, xn, xs, a, w_sg, gamma);
    return;
  }
  gateup_group_kernel<MB><<<dim3(grid, gu_split(MB)), kGrpThreads, MB * sxs, st>>>(es, gw, b, items, xn, xs, a, w_sg,
                                                                             gamma);
}

template <int MB>
static void grp_launch_dn(const ExpertSet& es, const GroupWork& gw, int b, int items, int grid, const float* a,
                          float* y, size_t sas, cudaStream_t st) {
  down_group_kernel<MB><<<dim3(grid, (es.H + kDnRows - 1) / kDnRows), kDnRows, MB * sas, st>>>(es, gw, b, items, a,
                                                                                                 y);
}

// SMs of the current device (cached per device; 148 if the query fails).
static int device_sms() {
  static int cached[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (cached[dev] == 0) {
    int n = 0;
    cached[dev] = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && n > 0 ? n : 148;
  }
  return cached[dev];
}

// Upper bound of the GEMV items of size bucket b (sizes (2^b, 2^(b+1)], the
// first bucket from 1): no more than S / (smallest size) of them, and none
// when the tensor cores take every group of that size.
static int bucket_items_bound(int b, int S, int max_items, int tc_min) {
  const int lo = b == 0 ? 1 : (1 << b) + 1;
  if (tc_min > 0 && lo >= tc_min) return 0;
  return S / lo < max_items ? S / lo : max_items;
}

static int launch_experts(const ExpertSet& es, const float* xn, const int32_t* ids, int T, float* a,
                          float* y, const float* w_sg, float* gamma, const GroupWork* gw, uint8_t* tcx,
                          uint8_t* tca, unsigned char* xs, cudaStream_t st) {
  const int slots = T * (es.k + 1);
  if (T >= 2 && gw) {
    const size_t sxs = (staged_x_bytes(es.H) + 15) & ~(size_t)15, sas = (staged_x_bytes(es.I) + 15) & ~(size_t)15;
    const size_t gu_smem = kGrpMaxM * sxs, dn_smem = kGrpMaxM * sas;
    const size_t grp_smem = (size_t)(3 * es.E + 5 + slots) * 4;
    if (xs && gu_smem <= 200 * 1024 && dn_smem <= 200 * 1024 && grp_smem <= 200 * 1024 &&
        smem_optin(reinterpret_cast<const void*>(&group_kernel), grp_smem, 4) && grp_optin<2>(2 * sxs, 2 * sas, 0) &&
        grp_optin<4>(4 * sxs, 4 * sas, 1) && grp_optin<8>(8 * sxs, 8 * sas, 2) &&
        grp_optin<16>(16 * sxs, 16 * sas, 3)) {
      const int items = group_max_items(T, es.k, es.E);
      // groups of >= kTcMinTokens tokens go to the tensor cores when the shape tiles
      const bool tc = g_tc_enabled && T >= kTcMinTokens && tcx && tca && es.H % kTcRows == 0 &&
                      (2 * es.I) % kTcRows == 0 && (es.H / 64) % 4 == 0 && (es.I / 64) % 4 == 0 &&
                      smem_optin(reinterpret_cast<const void*>(&tc_gemm_kernel<0>), tc_smem_bytes(), 2) &&
                      smem_optin(reinterpret_cast<const void*>(&tc_gemm_kernel<1>), tc_smem_bytes(), 3);
      const int max_tc = group_max_tc(T, es.k, kTcMinTokens);
      group_kernel<<<1, 1024, grp_smem, st>>>(ids, T, es.k, es.E, es.I, es.H, tc ? kTcMinTokens : 0, *gw, a, y);
      stage_tokens_kernel<<<T, kGrpThreads, 0, st>>>(xn, es.H, xs, sxs, tc ? gw->tscale : nullptr);
      // a bucket's grid covers at most the items it can hold (the kernels
      // index the bucket lists with the full stride `items`)
      int nb[kGrpBuckets];
      for (int b = 0; b < kGrpBuckets; ++b) nb[b] = bucket_items_bound(b, slots, items, tc ? kTcMinTokens : 0);
      // only items of <= 4 tokens: one launch for both of their buckets
      const bool small_only = nb[2] == 0 && nb[3] == 0 && nb[0] > 0 && nb[1] > 0 && gu_bulk_ok<2>(es) &&
                              gu_bulk_ok<4>(es) &&
                              smem_optin(reinterpret_cast<const void*>(&gateup_bulk_small_kernel),
                                         gu_bulk_smem(4, es.H, 4), 30) &&
                              smem_optin(reinterpret_cast<const void*>(&down_group_small_kernel), 4 * sas, 31);
      if (small_only) {
        gateup_bulk_small_kernel<<<dim3(nb[0] + nb[1], gu_split(4)), kGrpThreads, gu_bulk_smem(4, es.H, 4), st>>>(
            es, *gw, items, nb[0], xn, xs, a, w_sg, gamma);
      } else {
        if (nb[0]) grp_launch_gu<2>(es, *gw, 0, items, nb[0], xn, xs, a, w_sg, gamma, sxs, st);
        if (nb[1]) grp_launch_gu<4>(es, *gw, 1, items, nb[1], xn, xs, a, w_sg, gamma, sxs, st);
      }
      if (nb[2]) grp_launch_gu<8>(es, *gw, 2, items, nb[2], xn, xs, a, w_sg, gamma, sxs, st);
      if (nb[3]) grp_launch_gu<16>(es, *gw, 3, items, nb[3], xn, xs, a, w_sg, gamma, sxs, st);
      if (tc) {
        const TcScale sc{gw->rscale, gw->amax};
        tc_stage_kernel<<<dim3(max_tc, es.H / 64), kTcThreads, 0, st>>>(*gw, xn, es.H, es.k + 1, 0, tcx, es.E, w_sg,
                                                                      gamma, gw->tscale, sc);
        const int n_sm = device_sms();
        const int u0 = max_tc * (2 * es.I / kTcRows);
        tc_gemm_kernel<0><<<u0 < n_sm ? u0 : n_sm, kTcBlock, tc_smem_bytes(), st>>>(es, *gw, tcx, a, sc);
      }
      if (small_only) {
        down_group_small_kernel<<<dim3(nb[0] + nb[1], (es.H + kDnRows - 1) / kDnRows), kDnRows, 4 * sas, st>>>(
            es, *gw, items, nb[0], a, y);
      } else {
        if (nb[0]) grp_launch_dn<2>(es, *gw, 0, items, nb[0], a, y, sas, st);
        if (nb[1]) grp_launch_dn<4>(es, *gw, 1, items, nb[1], a, y, sas, st);
      }
      if (nb[2]) grp_launch_dn<8>(es, *gw, 2, items, nb[2], a, y, sas, st);
      if (nb[3]) grp_launch_dn<16>(es, *gw, 3, items, nb[3], a, y, sas, st);
      if (tc) {
        const TcScale sc{gw->rscale, gw->amax};
        tc_stage_kernel<<<dim3(max_tc, es.I / 64), kTcThreads, 0, st>>>(*gw, a, es.I, es.k + 1, 1, tca, es.E, nullptr,
                                                                      nullptr, nullptr, sc);
        const int n_sm = device_sms();
        const int u1 = max_tc * (es.H / kTcRows);
        tc_gemm_kernel<1><<<u1 < n_sm ? u1 : n_sm, kTcBlock, tc_smem_bytes(), st>>>(es, *gw, tca, y, sc);
      }
      return cuda_rc(cudaGetLastError());
    }
  }
  {
    const int ng = es.H / 64, lpr = ng < 32 ? ng : 32;
    const int units = es.I / (32 / lpr);
    int blocks = (units + 2 * kWarps - 1) / (2 * kWarps);
    const size_t smem = staged_x_bytes(es.H);
    gateup_kernel<<<dim3(blocks, slots), kThreads, smem, st>>>(es, xn, ids, a, w_sg, gamma);
  }
  {
    const int blocks = (es.H + kDownThreads - 1) / kDownThreads;
    const size_t smem = staged_x_bytes(es.I);
    down_kernel<<<dim3(blocks, slots), kDownThreads, smem, st>>>(es, ids, a, y);
  }
  return cuda_rc(cudaGetLastError());
}

static int launch_combine(const float* y, const float* weights, const float* gamma, const float* h,
                          const float* norm_w, float eps, int T, int k, int H, float* h_out,
                          float* xn_out, cudaStream_t st) {
  combine_kernel<<<T, kThreads, 0, st>>>(y, weights, gamma, h, norm_w, eps, k, H, h_out, xn_out);
  return cuda_rc(cudaGetLastError());
}

// ------------------------------------------------- persistent-kernel path --
static std::atomic<int> g_fused_enabled{1};  // process-wide, as g_tc_enabled
// Token counts up to which T > 1 runs through the persistent kernel, two
// tokens per launch (measured: a layer of T = 2 / 4 / 8 tokens takes
// 77 / 138 / 197 us on the grouped path against 31.9 / 60.3 / 124.7 us per
// layer in stack launches of token pairs; a single-layer launch costs
// ~34 us).
constexpr int kFusedTokensLayer = 4;
constexpr int kFusedTokensStack = 8;

struct FusedConfig {
  bool ok;
  int n_sm;
  FusedPlan plan;
};
struct FusedConfigs {
  FusedConfig nt[kFusedMaxNT + 1];  // by tokens per launch (index 0 unused)
};

static bool same_desc(const fmoe_layer_desc& a, const fmoe_layer_desc& b);

// Per-device cache of the last configuration (shape checks and the
// attribute / occupancy queries run once per shape, not per call).  Host
// threads that run layers of different shapes on one device share an entry,
// so it is read and replaced under a lock.
struct FusedCacheEntry {
  bool valid;
  fmoe_layer_desc desc;
  FusedConfigs fc;
};
static FusedCacheEntry g_fused_cache[64];
static std::mutex g_fused_cache_mu;

static FusedConfig fused_config_uncached(const fmoe_layer_desc& d, int dev, int nt);

// The configuration of the persistent kernel for nt tokens per launch.
static FusedConfig fused_config(const fmoe_layer_desc& d, int nt = 1) {
  int dev = 0;
  if (nt < 1 || nt > kFusedMaxNT) return FusedConfig{};
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return FusedConfig{};
  std::lock_guard<std::mutex> lock(g_fused_cache_mu);
  FusedCacheEntry& e = g_fused_cache[dev];
  if (!(e.valid && same_desc(e.desc, d))) {
    for (int n = 1; n <= kFusedMaxNT; ++n) e.fc.nt[n] = fused_config_uncached(d, dev, n);
    e.desc = d;
    e.valid = true;
  }
  return e.fc.nt[nt];
}

// The fused kernel instantiation for a pair of code widths and nt tokens per
// launch (two tokens: 4-bit codes, whose slots leave room for two tokens'
// staged inputs).
static const void* fused_kernel_for(int bits, int sbits, int nt) {
  if (nt == 2) return bits == 4 && sbits == 4 ? reinterpret_cast<const void*>(&fused_stack_kernel<4, 4, 2>) : nullptr;
  if (nt != 1) return nullptr;
  if (bits == 4 && sbits == 4) return reinterpret_cast<const void*>(&fused_stack_kernel<4, 4, 1>);
  if (bits == 2 && sbits == 4) return reinterpret_cast<const void*>(&fused_stack_kernel<2, 4, 1>);
  if (bits == 2 && sbits == 2) return reinterpret_cast<const void*>(&fused_stack_kernel<2, 2, 1>);
  if (bits == 4 && sbits == 2) return reinterpret_cast<const void*>(&fused_stack_kernel<4, 2, 1>);
  return nullptr;
}

static FusedConfig fused_config_uncached(const fmoe_layer_desc& d, int dev, int nt) {
  FusedConfig fc{};
  int n_sm = 0, optin = 0;
  if (cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return fc;
  if (cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess) return fc;
  if (n_sm < 1) return fc;
  if (n_sm > kFusedMaxCtas) n_sm = kFusedMaxCtas;  // one CTA per SM, at most kFusedMaxCtas of them
  const size_t max_dyn = optin > 2048 ? (size_t)optin - 1024 : 0;
  if (!fused_plan(d.hidden, d.inter, d.n_experts, d.top_k, d.bits, d.shared_bits, nt, n_sm, max_dyn, &fc.plan))
    return fc;
  const void* kfn = fused_kernel_for(d.bits, d.shared_bits, nt);
  if (!kfn) return fc;
  if (cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)fc.plan.total) != cudaSuccess)
    return fc;
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kfn, kFusedThreads, fc.plan.total) != cudaSuccess ||
      per_sm < 1)
    return fc;
  fc.n_sm = n_sm;
  fc.ok = true;
  return fc;
}

static bool same_desc(const fmoe_layer_desc& a, const fmoe_layer_desc& b) {
  return a.hidden == b.hidden && a.inter == b.inter && a.n_experts == b.n_experts && a.top_k == b.top_k &&
         a.bits == b.bits && a.shared_bits == b.shared_bits && a.group == b.group && a.eps == b.eps;
}

// Runs n_layers layers of nt tokens with the persistent kernel: tokens
// t .. t + nt - 1 of a T-token workspace (their rows of the logits, ids,
// weights, gamma and a intermediates; h and xn point at token t's row, the
// others follow).  Returns FMOE_ERR_UNSUPPORTED when the configuration does
// not fit it.
static int launch_fused(const fmoe_layer_weights* layers, int n_layers, float* h, float* xn, void* ws,
                        size_t ws_bytes, cudaStream_t st, int T = 1, int t = 0, int nt = 1,
                        unsigned char* trace = nullptr) {
  const fmoe_layer_desc& d = layers[0].desc;
  const FusedConfig fc = fused_config(d, nt);
  if (!fc.ok) return FMOE_ERR_UNSUPPORTED;
  const WsLayout w = ws_layout(d.hidden, d.inter, d.n_experts, d.top_k, T);
  if (ws_bytes < w.bytes || t < 0 || t + nt > T) return FMOE_ERR_BUFFER_TOO_SMALL;
  unsigned char* base = static_cast<unsigned char*>(ws);
  FusedArgs args;
  std::memset(&args, 0, sizeof(args));
  args.H = d.hidden;
  args.I = d.inter;
  args.E = d.n_experts;
  args.k = d.top_k;
  args.eps = d.eps;
  args.h = h;
  args.xn = xn;
  args.logits = reinterpret_cast<float*>(base + w.logits) + (size_t)t * d.n_experts;
  args.ids = reinterpret_cast<int32_t*>(base + w.ids) + (size_t)t * d.top_k;
  args.weights = reinterpret_cast<float*>(base + w.weights) + (size_t)t * d.top_k;
  args.gamma = reinterpret_cast<float*>(base + w.gamma) + t;
  args.a = reinterpret_cast<float*>(base + w.a) + (size_t)t * (d.top_k + 1) * d.inter;
  args.x_logit = reinterpret_cast<uint64_t*>(base + w.x_logit);
  args.x_h = reinterpret_cast<float*>(base + w.x_h);
  args.x_ss = reinterpret_cast<float*>(base + w.x_ss);
  args.x_part = reinterpret_cast<float*>(base + w.x_part);
  args.sync = reinterpret_cast<unsigned*>(base + w.sync);
  args.plan = fc.plan;
  const TraceLayout tl = trace_layout(d.hidden, d.inter, d.n_experts, d.top_k, T);
  for (int l0 = 0; l0 < n_layers; l0 += kFusedMaxLayers) {
    const int n = n_layers - l0 < kFusedMaxLayers ? n_layers - l0 : kFusedMaxLayers;
    args.n_layers = n;
    if (trace) {
      // this chunk's layers' records, token t's rows
      unsigned char* tb = trace + (size_t)l0 * tl.bytes;
      args.tr_xn = reinterpret_cast<float*>(tb + tl.off[FMOE_TRACE_XN_IN]) + (size_t)t * d.hidden;
      args.logits = reinterpret_cast<float*>(tb + tl.off[FMOE_TRACE_LOGITS]) + (size_t)t * d.n_experts;
      args.ids = reinterpret_cast<int32_t*>(tb + tl.off[FMOE_TRACE_IDS]) + (size_t)t * d.top_k;
      args.weights = reinterpret_cast<float*>(tb + tl.off[FMOE_TRACE_WEIGHTS]) + (size_t)t * d.top_k;
      args.gamma = reinterpret_cast<float*>(tb + tl.off[FMOE_TRACE_GAMMA]) + t;
      args.a = reinterpret_cast<float*>(tb + tl.off[FMOE_TRACE_A]) + (size_t)t * (d.top_k + 1) * d.inter;
      args.tr_h = reinterpret_cast<float*>(tb + tl.off[FMOE_TRACE_H_OUT]) + (size_t)t * d.hidden;
      args.lstride = tl.bytes;
    }
    for (int l = 0; l < n; ++l) {
      const fmoe_layer_weights& L = layers[l0 + l];
      args.layers[l].experts = static_cast<const uint8_t*>(L.experts);
      args.layers[l].shared = static_cast<const uint8_t*>(L.shared);
      args.layers[l].w_router = L.w_router;
      args.layers[l].w_sg = L.w_shared_gate;
      args.layers[l].norm_w = L.norm_w;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(fc.n_sm);
    cfg.blockDim = dim3(kFusedThreads);
    cfg.dynamicSmemBytes = fc.plan.total;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    void* kargs[] = {&args};
    const cudaError_t e = cudaLaunchKernelExC(&cfg, fused_kernel_for(d.bits, d.shared_bits, nt), kargs);
    if (e != cudaSuccess) return FMOE_ERR_CUDA;
  }
  return FMOE_OK;
}

// T tokens (rows of h and xn) through n_layers layers: launches of two
// tokens where the kernel supports them, one token otherwise.
// FMOE_ERR_UNSUPPORTED (nothing launched) when the one-token kernel does not
// fit the shape.
static int launch_fused_tokens(const fmoe_layer_weights* layers, int n_layers, float* h, float* xn, int T,
                               void* ws, size_t ws_bytes, cudaStream_t st, unsigned char* trace = nullptr) {
  const fmoe_layer_desc& d = layers[0].desc;
  if (!fused_config(d, 1).ok) return FMOE_ERR_UNSUPPORTED;
  const bool pairs = fused_config(d, 2).ok;
  const size_t H = (size_t)d.hidden;
  for (int t = 0; t < T;) {
    const int nt = pairs && T - t >= 2 ? 2 : 1;
    const int rc = launch_fused(layers, n_layers, h + t * H, xn + t * H, ws, ws_bytes, st, T, t, nt, trace);
    if (rc != FMOE_OK) return rc;
    t += nt;
  }
  return FMOE_OK;
}

static GroupWork group_work(unsigned char* base, const WsLayout& w) {
  GroupWork g;
  g.count = reinterpret_cast<int*>(base + w.g_count);
  g.offset = reinterpret_cast<int*>(base + w.g_offset);
  g.slots = reinterpret_cast<int*>(base + w.g_slots);
  g.n_items = reinterpret_cast<int*>(base + w.g_nitems);
  g.items = reinterpret_cast<int4*>(base + w.g_items);
  g.bitems = reinterpret_cast<int4*>(base + w.g_bitems);
  g.tc = reinterpret_cast<int4*>(base + w.g_tc);
  g.tscale = reinterpret_cast<float*>(base + w.tsc);
  g.rscale = reinterpret_cast<float*>(base + w.rsc);
  g.amax = reinterpret_cast<unsigned*>(base + w.amax);
  return g;
}

static int layer_forward_impl(const fmoe_layer_weights* lw, const float* logits_in, float* h,
                              float* xn, int T, void* ws, size_t ws_bytes, cudaStream_t st) {
  int rc = weights_check(lw);
  if (rc != FMOE_OK) return rc;
  const fmoe_layer_desc& d = lw->desc;
  if (T < 1 || !h || !xn || !ws || !aligned16(h) || !aligned16(xn) || !aligned16(ws))
    return FMOE_ERR_INVALID_ARG;
  if (!disjoint(h, xn, (size_t)T * d.hidden * 4)) return FMOE_ERR_INVALID_ARG;
  if (logits_in && !aligned16(logits_in)) return FMOE_ERR_INVALID_ARG;
  const WsLayout w = ws_layout(d.hidden, d.inter, d.n_experts, d.top_k, T);
  if (ws_bytes < w.bytes) return FMOE_ERR_BUFFER_TOO_SMALL;
  if (T <= kFusedTokensLayer && !logits_in && g_fused_enabled) {
    // a few tokens: persistent launches of two tokens (one for an odd last
    // token) are faster than the grouped path's sequence of launches
    rc = launch_fused_tokens(lw, 1, h, xn, T, ws, ws_bytes, st);
    if (rc != FMOE_ERR_UNSUPPORTED) return rc;
  }
  unsigned char* base = static_cast<unsigned char*>(ws);
  float* part = reinterpret_cast<float*>(base + w.part);
  float* logits = reinterpret_cast<float*>(base + w.logits);
  int32_t* ids = reinterpret_cast<int32_t*>(base + w.ids);
  float* weights = reinterpret_cast<float*>(base + w.weights);
  float* gamma = reinterpret_cast<float*>(base + w.gamma);
  float* a = reinterpret_cast<float*>(base + w.a);
  float* y = reinterpret_cast<float*>(base + w.y);
  const ExpertSet es = expert_set(lw);
  if (logits_in) {
    // given routing: top-k on the given logits; the shared gate is computed
    // by the gate/up kernel
    rc = cuda_rc(cudaMemcpyAsync(logits, logits_in, (size_t)T * d.n_experts * 4, cudaMemcpyDeviceToDevice, st));
    if (rc == FMOE_OK) rc = launch_topk(nullptr, logits, T, d.n_experts, d.top_k, logits, ids, weights, nullptr, st);
  } else {
    rc = launch_router(xn, lw->w_router, lw->w_shared_gate, T, d.hidden, d.n_experts, part, st);
    if (rc == FMOE_OK) rc = launch_topk(part, nullptr, T, d.n_experts, d.top_k, logits, ids, weights, gamma, st);
  }
  if (rc != FMOE_OK) return rc;
  const GroupWork gw = group_work(base, w);
  rc = launch_experts(es, xn, ids, T, a, y, lw->w_shared_gate, logits_in ? gamma : nullptr, &gw, base + w.tcx,
                      base + w.tca, T > 1 ? base + w.g_xs : nullptr, st);
  if (rc != FMOE_OK) return rc;
  return launch_combine(y, weights, gamma, h, lw->norm_w, d.eps, T, d.top_k, d.hidden, h, xn, st);
}

}  // namespace fmoe

using namespace fmoe;

extern "C" const char* fmoe_error_string(int status) {
  switch (status) {
    case FMOE_OK: return "ok";
    case FMOE_ERR_INVALID_ARG: return "invalid argument";
    case FMOE_ERR_UNSUPPORTED: return "unsupported shape or bit width";
    case FMOE_ERR_CUDA: return "CUDA runtime error";
    case FMOE_ERR_DEVICE_STATUS: return "device status word set";
    case FMOE_ERR_BUFFER_TOO_SMALL: return "buffer too small";
    default: return "unknown status";
  }
}

extern "C" int fmoe_read_status(uint32_t* status, int clear) {
  if (!status) return FMOE_ERR_INVALID_ARG;
  if (cudaDeviceSynchronize() != cudaSuccess) return FMOE_ERR_CUDA;
  if (cudaMemcpyFromSymbol(status, g_status, sizeof(uint32_t)) != cudaSuccess) return FMOE_ERR_CUDA;
  if (clear) {
    const uint32_t zero = 0;
    if (cudaMemcpyToSymbol(g_status, &zero, sizeof(uint32_t)) != cudaSuccess) return FMOE_ERR_CUDA;
  }
  return FMOE_OK;
}

extern "C" size_t fmoe_workspace_bytes(const fmoe_layer_desc* d, int T) {
  if (!desc_valid(d) || T < 1) return 0;
  return ws_layout(d->hidden, d->inter, d->n_experts, d->top_k, T).bytes;
}

extern "C" int fmoe_workspace_init(void* d_ws, size_t ws_bytes, cudaStream_t stream) {
  if (!d_ws || !aligned16(d_ws)) return FMOE_ERR_INVALID_ARG;
  return cuda_rc(cudaMemsetAsync(d_ws, 0, ws_bytes, stream));
}

extern "C" size_t fmoe_workspace_offset(const fmoe_layer_desc* d, int T, int which) {
  if (!desc_valid(d) || T < 1) return (size_t)-1;
  const WsLayout w = ws_layout(d->hidden, d->inter, d->n_experts, d->top_k, T);
  switch (which) {
    case 0: return w.logits;
    case 1: return w.ids;
    case 2: return w.weights;
    case 3: return w.gamma;
    case 4: return w.a;
    case 5: return w.y;
    default: return (size_t)-1;
  }
}

extern "C" int fmoe_route_topk(const float* d_xn, const float* d_w_router, int T, int H, int E, int k,
                               unsigned flags, float* d_logits, int32_t* d_ids, float* d_weights,
                               void* d_ws, size_t ws_bytes, cudaStream_t stream) {
  const bool given = (flags & FMOE_LOGITS_GIVEN) != 0;
  if (T < 1 || H < 64 || H % 64 || E < 1 || k < 1 || k > E) return FMOE_ERR_INVALID_ARG;
  if (k > kMaxK || E > kMaxE) return FMOE_ERR_UNSUPPORTED;
  if (!d_logits || !d_ids || !d_weights || !aligned16(d_logits) || !aligned16(d_ids) || !aligned16(d_weights))
    return FMOE_ERR_INVALID_ARG;
  if (given) return launch_topk(nullptr, d_logits, T, E, k, d_logits, d_ids, d_weights, nullptr, stream);
  if (!d_xn || !d_w_router || !d_ws || !aligned16(d_xn) || !aligned16(d_w_router) || !aligned16(d_ws))
    return FMOE_ERR_INVALID_ARG;
  const WsLayout w = ws_layout(H, 64, E, k, T);
  if (ws_bytes < w.part + (size_t)T * (E + 1) * kRouterSplit * 4) return FMOE_ERR_BUFFER_TOO_SMALL;
  float* part = reinterpret_cast<float*>(static_cast<unsigned char*>(d_ws) + w.part);
  int rc = launch_router(d_xn, d_w_router, nullptr, T, H, E, part, stream);
  if (rc != FMOE_OK) return rc;
  return launch_topk(part, nullptr, T, E, k, d_logits, d_ids, d_weights, nullptr, stream);
}

extern "C" int fmoe_expert_forward(const fmoe_layer_weights* lw, const float* d_xn, int T,
                                   const int32_t* d_ids, int k, float* d_y, float* d_gamma,
                                   void* d_ws, size_t ws_bytes, cudaStream_t stream) {
  int rc = weights_check(lw);
  if (rc != FMOE_OK) return rc;
  const fmoe_layer_desc& d = lw->desc;
  if (T < 1 || k != d.top_k) return FMOE_ERR_INVALID_ARG;
  const void* ps[] = {d_xn, d_ids, d_y, d_gamma, d_ws};
  for (const void* p : ps)
    if (!p || !aligned16(p)) return FMOE_ERR_INVALID_ARG;
  const WsLayout w = ws_layout(d.hidden, d.inter, d.n_experts, d.top_k, T);
  if (ws_bytes < w.bytes) return FMOE_ERR_BUFFER_TOO_SMALL;
  float* a = reinterpret_cast<float*>(static_cast<unsigned char*>(d_ws) + w.a);
  unsigned char* base = static_cast<unsigned char*>(d_ws);
  const GroupWork gw = group_work(base, w);
  return launch_experts(expert_set(lw), d_xn, d_ids, T, a, d_y, lw->w_shared_gate, d_gamma, &gw, base + w.tcx,
                        base + w.tca, T > 1 ? base + w.g_xs : nullptr, stream);
}

extern "C" int fmoe_combine_residual_rmsnorm(const float* d_y, const float* d_weights,
                                             const float* d_gamma, const float* d_h,
                                             const float* d_norm_w, float eps, int T, int k, int H,
                                             float* d_h_out, float* d_xn_out, cudaStream_t stream) {
  if (T < 1 || k < 1 || k > kMaxK || H < 1 || eps < 0.f) return FMOE_ERR_INVALID_ARG;
  const void* ps[] = {d_y, d_weights, d_gamma, d_h, d_norm_w, d_h_out, d_xn_out};
  for (const void* p : ps)
    if (!p || !aligned16(p)) return FMOE_ERR_INVALID_ARG;
  // h_out may be h itself (in place); otherwise the outputs share no byte
  // with each other, with h or with y
  const size_t rows = (size_t)T * H * 4, ys = (size_t)T * (k + 1) * H * 4;
  if (!disjoint(d_xn_out, d_h, rows) || !disjoint(d_xn_out, d_h_out, rows) || !disjoint(d_xn_out, rows, d_y, ys) ||
      !disjoint(d_h_out, rows, d_y, ys) || (d_h_out != d_h && !disjoint(d_h_out, d_h, rows)))
    return FMOE_ERR_INVALID_ARG;
  return launch_combine(d_y, d_weights, d_gamma, d_h, d_norm_w, eps, T, k, H, d_h_out, d_xn_out, stream);
}

extern "C" int fmoe_layer_forward(const fmoe_layer_weights* lw, float* d_h, float* d_xn, int T,
                                  void* d_ws, size_t ws_bytes, cudaStream_t stream) {
  return layer_forward_impl(lw, nullptr, d_h, d_xn, T, d_ws, ws_bytes, stream);
}

extern "C" int fmoe_layer_forward_host(const fmoe_layer_weights* lw, const float* hx_in, float* hx_out,
                                       float* d_hx, int T, void* d_ws, size_t ws_bytes, cudaStream_t stream) {
  const int rc0 = weights_check(lw);
  if (rc0 != FMOE_OK) return rc0;
  if (!hx_in || !hx_out || !d_hx || !d_ws || T < 1 || !aligned16(d_hx) || !aligned16(d_ws))
    return FMOE_ERR_INVALID_ARG;
  const int H = lw->desc.hidden;
  const WsLayout w = ws_layout(H, lw->desc.inter, lw->desc.n_experts, lw->desc.top_k, T);
  if (ws_bytes < w.bytes) return FMOE_ERR_BUFFER_TOO_SMALL;
  const size_t bytes = (size_t)2 * T * H * sizeof(float);
  if (cudaMemcpyAsync(d_hx, hx_in, bytes, cudaMemcpyHostToDevice, stream) != cudaSuccess) return FMOE_ERR_CUDA;
  const int rc = layer_forward_impl(lw, nullptr, d_hx, d_hx + (size_t)T * H, T, d_ws, ws_bytes, stream);
  if (rc != FMOE_OK) return rc;
  return cudaMemcpyAsync(hx_out, d_hx, bytes, cudaMemcpyDeviceToHost, stream) == cudaSuccess ? FMOE_OK
                                                                                            : FMOE_ERR_CUDA;
}

extern "C" int fmoe_layer_forward_logits(const fmoe_layer_weights* lw, const float* d_logits,
                                         float* d_h, float* d_xn, int T, void* d_ws,
                                         size_t ws_bytes, cudaStream_t stream) {
  if (!d_logits) return FMOE_ERR_INVALID_ARG;
  return layer_forward_impl(lw, d_logits, d_h, d_xn, T, d_ws, ws_bytes, stream);
}

extern "C" int fmoe_pack_experts_device(const uint8_t* d_q, const uint16_t* d_scale,
                                        const uint16_t* d_bias, int bits, int n_experts, int hidden,
                                        int inter, int group, void* d_packed, size_t d_bytes,
                                        cudaStream_t stream) {
  if (!d_q || !d_scale || !d_bias || !d_packed || n_experts < 1) return FMOE_ERR_INVALID_ARG;
  const void* ps[] = {d_q, d_scale, d_bias, d_packed};
  for (const void* p : ps)
    if (!aligned16(p)) return FMOE_ERR_INVALID_ARG;
  if (!shape_supported(bits, hidden, inter, group)) return FMOE_ERR_UNSUPPORTED;
  const RecordLayout L = record_layout(bits, hidden, inter);
  if (d_bytes < L.bytes * (size_t)n_experts) return FMOE_ERR_BUFFER_TOO_SMALL;
  const unsigned blocks = 148u * 16u;
  uint8_t* out = static_cast<uint8_t*>(d_packed);
  if (bits == 4)
    pack_codes_kernel<4><<<blocks, 256, 0, stream>>>(d_q, n_experts, hidden, inter, out);
  else
    pack_codes_kernel<2><<<blocks, 256, 0, stream>>>(d_q, n_experts, hidden, inter, out);
  pack_sb_kernel<<<blocks, 256, 0, stream>>>(d_scale, d_bias, bits, n_experts, hidden, inter, out);
  return cuda_rc(cudaGetLastError());
}

extern "C" int fmoe_quantize_groups(const float* d_w, size_t n_groups, int group, int bits, uint8_t* d_q,
                                    uint16_t* d_scale, uint16_t* d_bias, cudaStream_t stream) {
  if (!d_w || !d_q || !d_scale || !d_bias) return FMOE_ERR_INVALID_ARG;
  if (!aligned16(d_w) || !aligned16(d_q) || !aligned16(d_scale) || !aligned16(d_bias)) return FMOE_ERR_INVALID_ARG;
  if (group != 64 || (bits != 4 && bits != 2)) return FMOE_ERR_UNSUPPORTED;
  if (n_groups == 0) return FMOE_OK;
  const size_t warps = n_groups < (size_t)148 * 64 ? n_groups : (size_t)148 * 64;
  quantize_groups_kernel<<<(unsigned)((warps + 7) / 8), 256, 0, stream>>>(d_w, n_groups, bits, d_q, d_scale, d_bias);
  return cuda_rc(cudaGetLastError());
}

extern "C" int fmoe_fused_supported(const fmoe_layer_desc* d) {
  if (!desc_valid(d) || !desc_supported(d)) return 0;
  return fused_config(*d).ok ? 1 : 0;
}

extern "C" int fmoe_set_tensor_cores(int enable) { return g_tc_enabled.exchange(enable ? 1 : 0); }

extern "C" int fmoe_tc_min_tokens(void) { return kTcMinTokens; }

extern "C" int fmoe_fused_max_tokens(int stack) { return stack ? kFusedTokensStack : kFusedTokensLayer; }

extern "C" int fmoe_set_fused(int enable) { return g_fused_enabled.exchange(enable ? 1 : 0); }

// A stack of layers; with a trace, every layer's input xn, intermediates and
// output h' recorded in its record of the trace.
static int stack_forward_impl(const fmoe_layer_weights* layers, int n_layers, float* d_h, float* d_xn, int T,
                              void* d_ws, size_t ws_bytes, unsigned char* trace, size_t trace_bytes,
                              cudaStream_t stream) {
  if (!layers || n_layers < 1 || !desc_valid(&layers[0].desc)) return FMOE_ERR_INVALID_ARG;
  if (T >= 1 && d_h && d_xn && !disjoint(d_h, d_xn, (size_t)T * layers[0].desc.hidden * 4))
    return FMOE_ERR_INVALID_ARG;
  if (trace) {
    for (int l = 0; l < n_layers; ++l) {
      const int rc = weights_check(&layers[l]);
      if (rc != FMOE_OK) return rc;
      if (!same_desc(layers[l].desc, layers[0].desc)) return FMOE_ERR_INVALID_ARG;
    }
    const fmoe_layer_desc& d = layers[0].desc;
    if (T < 1 || !aligned16(trace)) return FMOE_ERR_INVALID_ARG;
    if (trace_bytes < (size_t)n_layers * trace_layout(d.hidden, d.inter, d.n_experts, d.top_k, T).bytes)
      return FMOE_ERR_BUFFER_TOO_SMALL;
  }
  if (T >= 1 && T <= kFusedTokensStack && g_fused_enabled) {
    bool uniform = true;
    for (int l = 0; l < n_layers; ++l) {
      const int rc = weights_check(&layers[l]);
      if (rc != FMOE_OK) return rc;
      uniform = uniform && same_desc(layers[l].desc, layers[0].desc);
    }
    if (!d_h || !d_xn || !d_ws || !aligned16(d_h) || !aligned16(d_xn) || !aligned16(d_ws))
      return FMOE_ERR_INVALID_ARG;
    if (uniform) {
      // the tokens through the whole stack, two per persistent launch; up to
      // kFusedTokensStack tokens this beats the grouped path layer by layer
      const int rc = launch_fused_tokens(layers, n_layers, d_h, d_xn, T, d_ws, ws_bytes, stream, trace);
      if (rc != FMOE_ERR_UNSUPPORTED) return rc;
    }
  }
  for (int l = 0; l < n_layers; ++l) {
    const fmoe_layer_desc& d = layers[l].desc;
    const TraceLayout tl = trace_layout(d.hidden, d.inter, d.n_experts, d.top_k, T);
    unsigned char* rec = trace ? trace + (size_t)l * tl.bytes : nullptr;
    const size_t hb = (size_t)T * d.hidden * 4;
    if (rec && cudaMemcpyAsync(rec + tl.off[FMOE_TRACE_XN_IN], d_xn, hb, cudaMemcpyDeviceToDevice, stream) !=
                   cudaSuccess)
      return FMOE_ERR_CUDA;
    const int rc = fmoe_layer_forward(&layers[l], d_h, d_xn, T, d_ws, ws_bytes, stream);
    if (rc != FMOE_OK) return rc;
    if (rec) {
      // the layer's intermediates, as it left them in the workspace
      const WsLayout w = ws_layout(d.hidden, d.inter, d.n_experts, d.top_k, T);
      const unsigned char* base = static_cast<const unsigned char*>(d_ws);
      const size_t src[5] = {w.logits, w.ids, w.weights, w.gamma, w.a};
      const size_t n[5] = {(size_t)T * d.n_experts * 4, (size_t)T * d.top_k * 4, (size_t)T * d.top_k * 4,
                           (size_t)T * 4, (size_t)T * (d.top_k + 1) * d.inter * 4};
      for (int i = 0; i < 5; ++i)
        if (cudaMemcpyAsync(rec + tl.off[FMOE_TRACE_LOGITS + i], base + src[i], n[i], cudaMemcpyDeviceToDevice,
                            stream) != cudaSuccess)
          return FMOE_ERR_CUDA;
      if (cudaMemcpyAsync(rec + tl.off[FMOE_TRACE_H_OUT], d_h, hb, cudaMemcpyDeviceToDevice, stream) != cudaSuccess)
        return FMOE_ERR_CUDA;
    }
  }
  return FMOE_OK;
}

extern "C" int fmoe_stack_forward(const fmoe_layer_weights* layers, int n_layers, float* d_h,
                                  float* d_xn, int T, void* d_ws, size_t ws_bytes,
                                  cudaStream_t stream) {
  return stack_forward_impl(layers, n_layers, d_h, d_xn, T, d_ws, ws_bytes, nullptr, 0, stream);
}

extern "C" size_t fmoe_trace_bytes(const fmoe_layer_desc* d, int T, int n_layers) {
  if (!desc_valid(d) || T < 1 || n_layers < 1) return 0;
  return (size_t)n_layers * trace_layout(d->hidden, d->inter, d->n_experts, d->top_k, T).bytes;
}

extern "C" size_t fmoe_trace_offset(const fmoe_layer_desc* d, int T, int layer, int which) {
  if (!desc_valid(d) || T < 1 || layer < 0 || which < FMOE_TRACE_XN_IN || which > FMOE_TRACE_H_OUT)
    return (size_t)-1;
  const TraceLayout tl = trace_layout(d->hidden, d->inter, d->n_experts, d->top_k, T);
  return (size_t)layer * tl.bytes + tl.off[which];
}

extern "C" int fmoe_stack_forward_trace(const fmoe_layer_weights* layers, int n_layers, float* d_h, float* d_xn,
                                        int T, void* d_ws, size_t ws_bytes, void* d_trace, size_t trace_bytes,
                                        cudaStream_t stream) {
  if (!d_trace) return FMOE_ERR_INVALID_ARG;
  return stack_forward_impl(layers, n_layers, d_h, d_xn, T, d_ws, ws_bytes, static_cast<unsigned char*>(d_trace),
                            trace_bytes, stream);
}

extern "C" int fmoe_stack_forward_host(const fmoe_layer_weights* layers, int n_layers, const float* hx_in,
                                       float* hx_out, float* d_hx, int T, void* d_ws, size_t ws_bytes,
                                       cudaStream_t stream) {
  if (!layers || n_layers < 1 || !hx_in || !hx_out || !d_hx || !d_ws || T < 1 || !aligned16(d_hx) ||
      !aligned16(d_ws))
    return FMOE_ERR_INVALID_ARG;
  for (int l = 0; l < n_layers; ++l) {
    const int rc = weights_check(&layers[l]);
    if (rc != FMOE_OK) return rc;
    if (layers[l].desc.hidden != layers[0].desc.hidden) return FMOE_ERR_INVALID_ARG;
    const fmoe_layer_desc& d = layers[l].desc;
    if (ws_bytes < ws_layout(d.hidden, d.inter, d.n_experts, d.top_k, T).bytes) return FMOE_ERR_BUFFER_TOO_SMALL;
  }
  const int H = layers[0].desc.hidden;
  const size_t bytes = (size_t)2 * T * H * sizeof(float);
  if (cudaMemcpyAsync(d_hx, hx_in, bytes, cudaMemcpyHostToDevice, stream) != cudaSuccess) return FMOE_ERR_CUDA;
  const int rc = fmoe_stack_forward(layers, n_layers, d_hx, d_hx + (size_t)T * H, T, d_ws, ws_bytes, stream);
  if (rc != FMOE_OK) return rc;
  return cudaMemcpyAsync(hx_out, d_hx, bytes, cudaMemcpyDeviceToHost, stream) == cudaSuccess ? FMOE_OK
                                                                                            : FMOE_ERR_CUDA;
}

// --------------------------------------------- fixed device scratch ----
// Workspace of fmoe_layer_forward_noalloc: one array per device, set aside
// when the module loads, so that the call itself reserves no memory.
namespace fmoe {

constexpr size_t kStaticScratchBytes = size_t(12) << 20;  // 12 MiB: T <= 17 at 4096 x 1024 x 512 experts, top-4
constexpr size_t kStaticCounterBytes = 4096;             // the counter words at the start of the layout
constexpr int kStaticMaxDevices = 64;

static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

static std::mutex g_static_scratch_mu;
static void* g_static_scratch_ptr[kStaticMaxDevices];

// Address of the current device's scratch.  The first call on a device looks
// the symbol up and zeroes its counter words on `st`; later calls only read
// the cached address.
static int static_scratch(cudaStream_t st, void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FMOE_ERR_CUDA;
  if (dev < 0 || dev >= kStaticMaxDevices) return FMOE_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_static_scratch_mu);
  if (!g_static_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || !p) return FMOE_ERR_CUDA;
    if (cudaMemsetAsync(p, 0, kStaticCounterBytes, st) != cudaSuccess) return FMOE_ERR_CUDA;
    g_static_scratch_ptr[dev] = p;
  }
  *out = g_static_scratch_ptr[dev];
  return FMOE_OK;
}

}  // namespace fmoe

extern "C" int fmoe_layer_forward_noalloc(const fmoe_layer_weights* lw, float* d_h, float* d_xn, int T,
                                          cudaStream_t stream) {
  if (!lw || !desc_valid(&lw->desc) || T < 1) return FMOE_ERR_INVALID_ARG;
  const fmoe_layer_desc& d = lw->desc;
  if (!d_h || !d_xn || !disjoint(d_h, d_xn, (size_t)T * d.hidden * 4)) return FMOE_ERR_INVALID_ARG;
  if (ws_layout(d.hidden, d.inter, d.n_experts, d.top_k, T).bytes > kStaticScratchBytes)
    return FMOE_ERR_BUFFER_TOO_SMALL;
  void* ws = nullptr;
  const int rc = static_scratch(stream, &ws);
  if (rc != FMOE_OK) return rc;
  return layer_forward_impl(lw, nullptr, d_h, d_xn, T, ws, kStaticScratchBytes, stream);
}

#include "fmoe_cache.cuh"

#ifdef FMOE_TIMELINE
// Timeline build only (see fmoe_fused.cuh): the layer to record, and the
// records of the last launch, [kFusedMaxCtas][kTimelinePoints] u64 ns.
extern "C" int fmoe_timeline_layer(int layer) {
  return cudaMemcpyToSymbol(g_fmoe_ts_layer, &layer, sizeof(int)) == cudaSuccess ? FMOE_OK : FMOE_ERR_CUDA;
}
extern "C" int fmoe_timeline_read(void* host) {
  return cudaMemcpyFromSymbol(host, g_fmoe_ts, sizeof(g_fmoe_ts)) == cudaSuccess ? FMOE_OK : FMOE_ERR_CUDA;
}
#endif
