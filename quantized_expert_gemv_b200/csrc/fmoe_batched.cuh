// fmoe_batched.cuh -- the expert forward for T > 1 tokens, grouped by expert.
//
// With T tokens and k routed experts each, the T k routed slots and the T
// shared-expert slots are sorted by expert (group_kernel, in token order
// within an expert, so every result is deterministic).  Each expert's
// weights are then read once per step for all of its tokens:
//   - groups with fewer than kTcMinTokens tokens (all groups, with the
//     tensor cores switched off), in work items of up to kGrpMaxM tokens, go
//     through the integer-dot GEMV: gate/up row pairs by bulk copy into
//     per-warp slots for items of up to 4 tokens when a row holds at least
//     32 groups (gateup_bulk_small_kernel, gateup_bulk_kernel), by direct
//     loads otherwise (gateup_group_kernel), then the down products
//     (down_group_small_kernel, down_group_kernel); one load of a weight row
//     serves every token of the item;
//   - groups with at least kTcMinTokens tokens are dense enough for the
//     tensor cores (fmoe_tc.cuh): their items are listed separately.
// Slot s = t (k + 1) + j addresses a [T][k+1][I] and y [T][k+1][H] exactly as
// on the one-kernel-per-slot path, so the combine kernel is shared.
// Source pages: "What is Flash-MoE?" (a2a-mcp.org), section "2. FMA-optimised
// dequantisation kernels" (the pages run one token at a time; grouping the
// batch by expert is this implementation's addition for T > 1).
#pragma once

#include <cstdint>

#include "fmoe.h"
#include "fmoe_device.cuh"
#include "fmoe_fused.cuh"  // mbarrier and bulk-copy primitives, lds_group
#include "fmoe_layout.h"

namespace fmoe {

constexpr int kGrpMaxM = 16;      // tokens per GEMV work item
constexpr int kGrpBuckets = 4;    // GEMV items by size: <= 2, <= 4, <= 8, <= 16 tokens
constexpr int kTcItemMax = 32;    // tokens per tensor-core work item (more CTAs, shorter products each)
constexpr int kGrpThreads = 256;
// CTAs per item over the gate/up row pairs for items of up to MB tokens:
// the larger items are bound by the integer dot products rather than by
// their weight bytes, so they are cut finer to keep every SM busy
__host__ __device__ constexpr int gu_split(int MB) { return MB <= 4 ? 16 : 4 * MB; }
constexpr int kDnRows = 128;      // hidden rows per CTA of the grouped down product

// Device lists built by group_kernel.  Group g < E is routed expert g, group
// E the shared expert.
struct GroupWork {
  int* count;   // [E + 1] slots per group
  int* offset;  // [E + 2] first slot of each group in `slots`
  int* slots;   // [T (k + 1)] slot indices, grouped, in token order
  int* n_items; // [2 + kGrpBuckets] GEMV items, tensor-core items, GEMV items per size bucket
  int4* items;  // [max_items] (group, first slot within the group, tokens, 0), by group
  int4* bitems; // [kGrpBuckets][max_items] the GEMV items of each size bucket
  int4* tc;     // [max_tc]    (group, first, tokens, running sum of the items' tokens rounded up to 8)
  float* tscale;    // [T] tensor-core staging multiplier of each token (stage_tokens_kernel)
  float* rscale;    // [staged rows] epilogue multiplier of each tensor-core row
  unsigned* amax;   // [staged rows] max |a| of each tensor-core row (gate/up epilogue)
};

__host__ __device__ constexpr int group_max_tc(int T, int k, int min_tokens) {
  return T * (k + 1) / min_tokens + T * (k + 1) / kTcItemMax + 2;
}

__host__ __device__ constexpr int grp_bucket_max(int b) { return 2 << b; }

__device__ __forceinline__ int grp_bucket(int m) { return m <= 2 ? 0 : (m <= 4 ? 1 : (m <= 8 ? 2 : 3)); }

__host__ __device__ constexpr int group_max_items(int T, int k, int E) {
  // one item per non-empty group plus one per further kGrpMaxM slots
  return (T * k < E ? T * k : E) + 1 + (T * (k + 1)) / kGrpMaxM + 1;
}

// Block-wide exclusive scan (component-wise) of v over the CTA's threads in
// thread order; returns the scan, *total the sum.  blockDim.x <= 1024, a
// multiple of 32; red: 32 int4 of shared memory.
__device__ __forceinline__ int4 block_scan4(int4 v, int4* red, int4* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  int4 x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int a = __shfl_up_sync(0xffffffffu, x.x, o), b = __shfl_up_sync(0xffffffffu, x.y, o);
    const int c = __shfl_up_sync(0xffffffffu, x.z, o), d = __shfl_up_sync(0xffffffffu, x.w, o);
    if (lane >= o) x = make_int4(x.x + a, x.y + b, x.z + c, x.w + d);
  }
  if (lane == 31) red[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int4 t = lane < nw ? red[lane] : make_int4(0, 0, 0, 0);
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int a = __shfl_up_sync(0xffffffffu, t.x, o), b = __shfl_up_sync(0xffffffffu, t.y, o);
      const int c = __shfl_up_sync(0xffffffffu, t.z, o), d = __shfl_up_sync(0xffffffffu, t.w, o);
      if (lane >= o) t = make_int4(t.x + a, t.y + b, t.z + c, t.w + d);
    }
    if (lane < nw) red[lane] = t;  // inclusive sums of the warps
  }
  __syncthreads();
  const int4 before = warp > 0 ? red[warp - 1] : make_int4(0, 0, 0, 0);
  *total = red[nw - 1];
  __syncthreads();  // red may be reused
  return make_int4(before.x + x.x - v.x, before.y + x.y - v.y, before.z + x.z - v.z, before.w + x.w - v.w);
}

// One CTA of 1024 threads.  Sorts the T (k + 1) slots by group (stable),
// builds the work items (groups with >= tc_min tokens go to the tensor-core
// list when tc_min > 0), and zeroes a / y of slots whose expert id is out of
// range.  Groups are scanned two per thread (E + 1 <= 2048).
__global__ void __launch_bounds__(1024) group_kernel(const int32_t* __restrict__ ids, int T, int k, int E, int I,
                                                     int H, int tc_min, GroupWork w, float* __restrict__ a,
                                                     float* __restrict__ y) {
  extern __shared__ int gsm[];
  __shared__ int4 s_red[32];
  int* cnt = gsm;             // [E + 1]
  int* off = cnt + (E + 1);   // [E + 2]
  int* nit = off + (E + 2);   // [E + 2]: first GEMV item of each group
  int* grp = nit + (E + 2);   // [S]: group of each slot (-1: bad id)
  const int S = T * (k + 1);
  const int tid = threadIdx.x, nt = blockDim.x;
  for (int g = tid; g <= E; g += nt) cnt[g] = 0;
  if (tid < kGrpBuckets) w.n_items[2 + tid] = 0;
  for (int s = tid; s < S; s += nt) {
    const int t = s / (k + 1), j = s % (k + 1);
    int g = E;
    if (j < k) {
      const int id = ids[(size_t)t * k + j];
      g = (id >= 0 && id < E) ? id : -1;
    }
    grp[s] = g;
  }
  __syncthreads();
  bool bad = false;
  for (int s = tid; s < S; s += nt) {
    const int g = grp[s];
    if (g >= 0) atomicAdd(&cnt[g], 1);
    else {
      bad = true;
      for (int i = 0; i < I; ++i) a[(size_t)s * I + i] = 0.f;
      for (int i = 0; i < H; ++i) y[(size_t)s * H + i] = 0.f;
    }
  }
  if (__syncthreads_or(bad) && tid == 0) raise_status(FMOE_STATUS_BAD_EXPERT_ID);
  // per group: (slots, GEMV items, tensor-core items, their rounded tokens)
  auto group_terms = [&](int g) -> int4 {
    if (g > E) return make_int4(0, 0, 0, 0);
    const int c = cnt[g];
    if (c == 0) return make_int4(0, 0, 0, 0);
    if (tc_min > 0 && c >= tc_min) {
      const int full = c / kTcItemMax, rem = c % kTcItemMax;
      return make_int4(c, 0, full + (rem > 0), full * kTcItemMax + (rem + 7) / 8 * 8);
    }
    return make_int4(c, (c + kGrpMaxM - 1) / kGrpMaxM, 0, 0);
  };
  const int g0 = 2 * tid, g1 = g0 + 1;
  const int4 v0 = group_terms(g0), v1 = group_terms(g1);
  int4 tot;
  const int4 e0 = block_scan4(make_int4(v0.x + v1.x, v0.y + v1.y, v0.z + v1.z, v0.w + v1.w), s_red, &tot);
  const int4 e1 = make_int4(e0.x + v0.x, e0.y + v0.y, e0.z + v0.z, e0.w + v0.w);
  if (g0 <= E) off[g0] = e0.x, nit[g0] = e0.y;
  if (g1 <= E) off[g1] = e1.x, nit[g1] = e1.y;
  if (tid == 0) {
    off[E + 1] = tot.x;
    nit[E + 1] = tot.y;
    w.n_items[0] = tot.y;
    w.n_items[1] = tot.z;
  }
  // tensor-core items of this thread's groups, in group order
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int g = h == 0 ? g0 : g1;
    const int4 v = h == 0 ? v0 : v1;
    const int4 e = h == 0 ? e0 : e1;
    int idx = e.z, np_sum = e.w;
    for (int f = 0; f < v.x && v.z > 0; f += kTcItemMax) {
      const int mm = min(kTcItemMax, v.x - f);
      w.tc[idx++] = make_int4(g, f, mm, np_sum);
      np_sum += (mm + 7) / 8 * 8;
    }
  }
  __syncthreads();
  const int max_items = group_max_items(T, k, E);
  for (int g = tid; g <= E + 1; g += nt) w.offset[g] = off[g];
  for (int g = tid; g <= E; g += nt) {
    w.count[g] = cnt[g];
    const int c = cnt[g];
    if (c > 0 && !(tc_min > 0 && c >= tc_min))
      for (int i = 0; i * kGrpMaxM < c; ++i) {
        const int mm = min(kGrpMaxM, c - i * kGrpMaxM), b = grp_bucket(mm);
        const int4 item = make_int4(g, i * kGrpMaxM, mm, 0);
        w.items[nit[g] + i] = item;
        // bucket order does not matter: every item writes its own slots
        w.bitems[(size_t)b * max_items + atomicAdd(&w.n_items[2 + b], 1)] = item;
      }
  }
  // stable placement: rank of s = earlier slots of the same group
  for (int s = tid; s < S; s += nt) {
    const int g = grp[s];
    if (g < 0) continue;
    int r = 0;
#pragma unroll 8
    for (int s2 = 0; s2 < s; ++s2) r += grp[s2] == g;
    w.slots[off[g] + r] = s;
  }
}

__device__ __forceinline__ const uint8_t* group_record(const ExpertSet& es, int g, int* bits) {
  if (g == es.E) {
    *bits = es.shared_bits;
    return es.shared;
  }
  *bits = es.bits;
  if (es.rec_table) return reinterpret_cast<const uint8_t*>(es.rec_table[g]);
  return es.experts + (size_t)g * es.rec_bytes;
}

// Token i's staged vector: K inputs at base + i * stride.
__device__ __forceinline__ StagedX staged_i(unsigned char* base, size_t stride, int i, int K) {
  return staged_x_at(base + (size_t)i * stride, K);
}

// Stages every token's normed input once per step (24-bit block floating
// point groups, the layout of StagedX) at xs + t * stride.  grid T.
// With tscale, also the token's power-of-two staging multiplier for the
// tensor-core products (tc_row_scale of its largest magnitude).
__global__ void __launch_bounds__(kGrpThreads)
stage_tokens_kernel(const float* __restrict__ xn, int H, unsigned char* __restrict__ xs, size_t stride,
                    float* __restrict__ tscale) {
  const float* x = xn + (size_t)blockIdx.x * H;
  stage_x(x, H, staged_x_at(xs + blockIdx.x * stride, H));
  if (tscale) {
    __shared__ float s_m[kGrpThreads / 32];
    float m = 0.f;
    for (int i = threadIdx.x; i < H; i += blockDim.x) m = fmaxf(m, fabsf(x[i]));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if ((threadIdx.x & 31) == 0) s_m[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
      for (int w = 1; w < kGrpThreads / 32; ++w) m = fmaxf(m, s_m[w]);
      tscale[blockIdx.x] = tc_row_scale(m);
    }
  }
}

// Gate/up row pairs [p0, p1) of one record for the m <= MB tokens staged at
// sxb: each warp takes PAIRS row pairs at a time (their code loads in flight
// together); a lane owns whole groups of both rows of a pair, loads their
// codes once and applies them to every token.
template <int BITS, int MB, int PAIRS>
__device__ __forceinline__ void gateup_rows_multi(const uint8_t* rec, const ExpertSet& es, unsigned char* sxb,
                                                  size_t sxs, int m, float* __restrict__ a, const int* slot_of,
                                                  int p0, int p1) {
  const int H = es.H, ng = H / 64;
  const int lpr = ng < 32 ? ng : 32, gpl = ng / lpr, ppu = 32 / lpr;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  const int ps = lane / lpr, lg = lane % lpr;
  const RecordLayout L = record_layout(BITS, H, es.I);
  const uint8_t* codes = rec + L.gu_codes;
  const uint32_t* sbw = reinterpret_cast<const uint32_t*>(rec + L.gu_sb);
  for (int u0 = p0 / ppu + warp; u0 * ppu < p1; u0 += nw * PAIRS) {
    float yg[PAIRS][MB], yu[PAIRS][MB];
#pragma unroll
    for (int q = 0; q < PAIRS; ++q)
#pragma unroll
      for (int i = 0; i < MB; ++i) yg[q][i] = yu[q][i] = 0.f;
    for (int mm = 0; mm < gpl; ++mm) {
      const int g = lg + mm * lpr;
      GroupCodes<BITS> cg[PAIRS], cu[PAIRS];
      uint32_t sg[PAIRS], su[PAIRS];
#pragma unroll
      for (int q = 0; q < PAIRS; ++q) {  // all loads of the PAIRS pairs first
        const int n = (u0 + q * nw) * ppu + ps;
        const int nn = n < p1 ? n : p1 - 1;
        const uint8_t* rg = codes + (size_t)(2 * nn) * L.gu_row_bytes;
        cg[q] = load_group<BITS>(rg, ng, g);
        cu[q] = load_group<BITS>(rg + L.gu_row_bytes, ng, g);
        sg[q] = ld_stream_u32(sbw + (size_t)(2 * nn) * ng + g);
        su[q] = ld_stream_u32(sbw + (size_t)(2 * nn + 1) * ng + g);
      }
#pragma unroll
      for (int i = 0; i < MB; ++i) {
        if (i < m) {
          const StagedX sx = staged_i(sxb, sxs, i, H);
          uint4 xv[8];
          uint2 xl[8];
          load_xv(sx, ng, g, xv, xl);
          const float d = sx.delta[g], xs = sx.xsum[g];
#pragma unroll
          for (int q = 0; q < PAIRS; ++q) {
            yg[q][i] = group_epilogue(yg[q][i], sg[q], group_dot<BITS>(cg[q], xv, xl), d, xs);
            yu[q][i] = group_epilogue(yu[q][i], su[q], group_dot<BITS>(cu[q], xv, xl), d, xs);
          }
        }
      }
    }
#pragma unroll
    for (int q = 0; q < PAIRS; ++q) {
      const int n = (u0 + q * nw) * ppu + ps;
#pragma unroll
      for (int i = 0; i < MB; ++i) {
        if (i < m) {
          float g = yg[q][i], v = yu[q][i];
          for (int o = lpr >> 1; o > 0; o >>= 1) {
            g += __shfl_xor_sync(0xffffffffu, g, o);
            v += __shfl_xor_sync(0xffffffffu, v, o);
          }
          if (lg == 0 && n < p1) a[(size_t)slot_of[i] * es.I + n] = silu_mul(g, v);
        }
      }
    }
  }
}

// grid (max items, gu_split(MB)), one size bucket of GEMV items (m <= MB).
// Item (group, first, m): the group's slots first .. first + m - 1; the
// tokens' staged inputs are copied from xs (stage_tokens_kernel).  Also
// computes gamma[t] = sigmoid(w_sg . xn[t]) for the shared expert's tokens
// when gamma is given.  Used for hidden sizes below 2048 (larger ones take
// gateup_bulk_kernel); one CTA per SM's worth of registers, so that the
// 24-bit dot products of MB tokens do not spill.
template <int MB>
__global__ void __launch_bounds__(kGrpThreads, 1)
gateup_group_kernel(ExpertSet es, GroupWork w, int bucket, int max_items, const float* __restrict__ xn,
                    const unsigned char* __restrict__ xs, float* __restrict__ a, const float* __restrict__ w_sg,
                    float* __restrict__ gamma) {
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ int s_slot[kGrpMaxM];
  if ((int)blockIdx.x >= w.n_items[2 + bucket]) return;
  const int4 it = w.bitems[(size_t)bucket * max_items + blockIdx.x];
  const int g = it.x, m = it.z, k1 = es.k + 1;
  if (threadIdx.x < m) s_slot[threadIdx.x] = w.slots[w.offset[g] + it.y + threadIdx.x];
  __syncthreads();
  const size_t sxs = (staged_x_bytes(es.H) + 15) & ~(size_t)15;
  for (int i = 0; i < m; ++i) {
    const uint4* src = reinterpret_cast<const uint4*>(xs + (size_t)(s_slot[i] / k1) * sxs);
    uint4* dst = reinterpret_cast<uint4*>(smem + (size_t)i * sxs);
    for (int j = threadIdx.x; j < (int)(sxs / 16); j += kGrpThreads) dst[j] = __ldcg(src + j);
  }
  __syncthreads();
  if (gamma && g == es.E && blockIdx.y == 0) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int i = warp; i < m; i += kGrpThreads / 32) {
      const float* x = xn + (size_t)(s_slot[i] / k1) * es.H;
      float z = 0.f;
#pragma unroll 8
      for (int c = lane * 4; c < es.H; c += 128) {
        const float4 wv = __ldg(reinterpret_cast<const float4*>(w_sg + c));
        const float4 v = __ldg(reinterpret_cast<const float4*>(x + c));
        z = fmaf(wv.x, v.x, z);
        z = fmaf(wv.y, v.y, z);
        z = fmaf(wv.z, v.z, z);
        z = fmaf(wv.w, v.w, z);
      }
      z = warp_sum(z);
      if (lane == 0) gamma[s_slot[i] / k1] = 1.f / (1.f + expf(-z));
    }
  }
  int p0, p1;
  {
    const int ng = es.H / 64, ppu = 32 / (ng < 32 ? ng : 32);  // row pairs per warp unit
    const int per = ((es.I + gu_split(MB) - 1) / gu_split(MB) + ppu - 1) / ppu * ppu;
    p0 = min(es.I, (int)blockIdx.y * per);
    p1 = min(es.I, p0 + per);
  }
  int bits;
  const uint8_t* rec = group_record(es, g, &bits);
  constexpr int kPairs = MB <= 4 ? 2 : 1;
  if (bits == 4) gateup_rows_multi<4, MB, kPairs>(rec, es, smem, sxs, m, a, s_slot, p0, p1);
  else gateup_rows_multi<2, MB, kPairs>(rec, es, smem, sxs, m, a, s_slot, p0, p1);
}

// ------------------------------------------- bulk-copied gate/up GEMV --
// For the small items (m <= 4 tokens, bound by their weight bytes): a row
// pair's codes (two contiguous rows) and scale-bias words (two contiguous
// runs) come into shared memory by two bulk copies, so the bytes in flight
// are set by shared memory, not by registers.  Warp w takes the pairs
// p0 + w, p0 + w + 8, .. of the CTA's range and owns two ring slots: while
// it works on one pair the next one is landing; its lane 0 requests the
// pair after next into the slot it has just finished.  Needs H / 64 >= 32.
constexpr int kGuBulkWarps = kGrpThreads / 32;
constexpr int kGuBulkSlots = 2 * kGuBulkWarps;

__host__ __device__ constexpr size_t gu_bulk_slot_bytes(int H, int bits) {
  return (size_t)2 * H * bits / 8 + (size_t)2 * (H / 64) * 4;  // two code rows + their scale-bias words
}

template <int MB>
__device__ __forceinline__ void gateup_bulk_body(const ExpertSet& es, const GroupWork& w, int bucket, int max_items,
                                                 int item, const float* __restrict__ xn,
                                                 const unsigned char* __restrict__ xs, float* __restrict__ a,
                                                 const float* __restrict__ w_sg, float* __restrict__ gamma) {
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ int s_slot[MB];
  __shared__ uint64_t full[kGuBulkSlots];
  if (item >= w.n_items[2 + bucket]) return;
  const int4 it = w.bitems[(size_t)bucket * max_items + item];
  const int g = it.x, m = it.z, k1 = es.k + 1;
  const int H = es.H, I = es.I, ng = H / 64;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int bits;
  const uint8_t* rec = group_record(es, g, &bits);
  const RecordLayout L = record_layout(bits, H, I);
  const size_t sxs = (staged_x_bytes(H) + 15) & ~(size_t)15;
  const uint32_t code_bytes = 2u * (uint32_t)L.gu_row_bytes, sb_bytes = 8u * (uint32_t)ng;
  const size_t slot_bytes = ((size_t)code_bytes + sb_bytes + 127) & ~(size_t)127;
  unsigned char* ring = smem + (((size_t)MB * sxs + 127) & ~(size_t)127);
  int p0, p1;
  {
    const int per = (I + gu_split(MB) - 1) / gu_split(MB);
    p0 = min(I, (int)blockIdx.y * per);
    p1 = min(I, p0 + per);
  }
  if (tid == 0) {
    for (int i = 0; i < kGuBulkSlots; ++i) mbar_init(&full[i], 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (tid < m) s_slot[tid] = w.slots[w.offset[g] + it.y + tid];
  __syncthreads();
  // pair n into slot q (lane 0 of the owning warp)
  auto request = [&](int n, int q) {
    uint8_t* dst = ring + (size_t)q * slot_bytes;
    mbar_expect_tx(&full[q], code_bytes + sb_bytes);
    bulk_g2s(dst, rec + L.gu_codes + (size_t)(2 * n) * L.gu_row_bytes, code_bytes, &full[q]);
    bulk_g2s(dst + code_bytes, rec + L.gu_sb + (size_t)(2 * n) * ng * 4, sb_bytes, &full[q]);
  };
  if (lane == 0) {
    if (p0 + warp < p1) request(p0 + warp, 2 * warp);
    if (p0 + warp + kGuBulkWarps < p1) request(p0 + warp + kGuBulkWarps, 2 * warp + 1);
  }
  // the tokens' staged inputs (and the shared expert's gates) while the first pairs land
  for (int i = 0; i < m; ++i) {
    const uint4* src = reinterpret_cast<const uint4*>(xs + (size_t)(s_slot[i] / k1) * sxs);
    uint4* dst = reinterpret_cast<uint4*>(smem + (size_t)i * sxs);
    for (int j = tid; j < (int)(sxs / 16); j += kGrpThreads) dst[j] = __ldcg(src + j);
  }
  if (gamma && g == es.E && blockIdx.y == 0) {
    for (int i = warp; i < m; i += kGuBulkWarps) {
      const float* x = xn + (size_t)(s_slot[i] / k1) * H;
      float z = 0.f;
#pragma unroll 8
      for (int c = lane * 4; c < H; c += 128) {
        const float4 wv = __ldg(reinterpret_cast<const float4*>(w_sg + c));
        const float4 v = __ldg(reinterpret_cast<const float4*>(x + c));
        z = fmaf(wv.x, v.x, z);
        z = fmaf(wv.y, v.y, z);
        z = fmaf(wv.z, v.z, z);
        z = fmaf(wv.w, v.w, z);
      }
      z = warp_sum(z);
      if (lane == 0) gamma[s_slot[i] / k1] = 1.f / (1.f + expf(-z));
    }
  }
  __syncthreads();
  bool ok = true;
  int kk = 0;
  for (int n = p0 + warp; n < p1; n += kGuBulkWarps, ++kk) {
    const int q = 2 * warp + (kk & 1);
    if (!mbar_wait(&full[q], (uint32_t)((kk >> 1) & 1))) {
      ok = false;
      break;
    }
    const uint8_t* rows = ring + (size_t)q * slot_bytes;
    const uint32_t* sbw = reinterpret_cast<const uint32_t*>(rows + code_bytes);
    float yg[MB], yu[MB];
#pragma unroll
    for (int i = 0; i < MB; ++i) yg[i] = yu[i] = 0.f;
    for (int g0 = lane; g0 < ng; g0 += 32) {
      if (bits == 4) {
        const GroupCodes<4> cg = lds_group<4>(rows, ng, g0), cu = lds_group<4>(rows + L.gu_row_bytes, ng, g0);
        const uint32_t sg = sbw[g0], su = sbw[ng + g0];
#pragma unroll
        for (int i = 0; i < MB; ++i) {
          if (i < m) {
            const StagedX sx = staged_i(smem, sxs, i, H);
            uint4 xv[8];
            uint2 xl[8];
            load_xv(sx, ng, g0, xv, xl);
            yg[i] = group_epilogue(yg[i], sg, group_dot<4>(cg, xv, xl), sx.delta[g0], sx.xsum[g0]);
            yu[i] = group_epilogue(yu[i], su, group_dot<4>(cu, xv, xl), sx.delta[g0], sx.xsum[g0]);
          }
        }
      } else {
        const GroupCodes<2> cg = lds_group<2>(rows, ng, g0), cu = lds_group<2>(rows + L.gu_row_bytes, ng, g0);
        const uint32_t sg = sbw[g0], su = sbw[ng + g0];
#pragma unroll
        for (int i = 0; i < MB; ++i) {
          if (i < m) {
            const StagedX sx = staged_i(smem, sxs, i, H);
            uint4 xv[8];
            uint2 xl[8];
            load_xv(sx, ng, g0, xv, xl);
            yg[i] = group_epilogue(yg[i], sg, group_dot<2>(cg, xv, xl), sx.delta[g0], sx.xsum[g0]);
            yu[i] = group_epilogue(yu[i], su, group_dot<2>(cu, xv, xl), sx.delta[g0], sx.xsum[g0]);
          }
        }
      }
    }
    __syncwarp();
    // the slot is read: it takes the pair after next
    if (lane == 0 && n + 2 * kGuBulkWarps < p1) {
      fence_proxy_async();
      request(n + 2 * kGuBulkWarps, q);
    }
#pragma unroll
    for (int i = 0; i < MB; ++i) {
      if (i < m) {
        const float gs = warp_sum(yg[i]), us = warp_sum(yu[i]);
        if (lane == 0) a[(size_t)s_slot[i] * I + n] = silu_mul(gs, us);
      }
    }
  }
  if (!ok) {
    // leave no copy in flight: this warp's slots still owed a completion
    if (lane == 0) {
      for (int j = 0; j < 2; ++j) {
        const int n2 = p0 + warp + (kk + j) * kGuBulkWarps;
        if (n2 < p1) (void)mbar_wait(&full[2 * warp + ((kk + j) & 1)], (uint32_t)(((kk + j) >> 1) & 1));
      }
      raise_status(FMOE_STATUS_WAIT_TIMEOUT);
    }
  }
}

// grid (max items, gu_split(MB)): one size bucket.
template <int MB>
__global__ void __launch_bounds__(kGrpThreads, 2)
gateup_bulk_kernel(ExpertSet es, GroupWork w, int bucket, int max_items, const float* __restrict__ xn,
                   const unsigned char* __restrict__ xs, float* __restrict__ a, const float* __restrict__ w_sg,
                   float* __restrict__ gamma) {
  gateup_bulk_body<MB>(es, w, bucket, max_items, (int)blockIdx.x, xn, xs, a, w_sg, gamma);
}

// grid (n0 + n1, gu_split): the items of buckets 0 (<= 2 tokens) and 1
// (<= 4 tokens) in one launch, so that neither bucket's tail idles the GPU.
__global__ void __launch_bounds__(kGrpThreads, 2)
gateup_bulk_small_kernel(ExpertSet es, GroupWork w, int max_items, int n0, const float* __restrict__ xn,
                         const unsigned char* __restrict__ xs, float* __restrict__ a,
                         const float* __restrict__ w_sg, float* __restrict__ gamma) {
  if ((int)blockIdx.x < n0) gateup_bulk_body<2>(es, w, 0, max_items, (int)blockIdx.x, xn, xs, a, w_sg, gamma);
  else gateup_bulk_body<4>(es, w, 1, max_items, (int)blockIdx.x - n0, xn, xs, a, w_sg, gamma);
}

__host__ __device__ constexpr size_t gu_bulk_smem(int MB, int H, int bits) {
  return (((size_t)MB * ((staged_x_bytes(H) + 15) & ~(size_t)15) + 127) & ~(size_t)127) +
         (size_t)kGuBulkSlots * ((gu_bulk_slot_bytes(H, bits) + 127) & ~(size_t)127);
}

// Down product of one record for one hidden row and the m tokens staged at
// sx[0..m) (their SwiGLU outputs): the group's column-block words are loaded
// once and applied to every token.
template <int BITS, int MB>
__device__ __forceinline__ void down_row_multi(const uint8_t* rec, const ExpertSet& es, unsigned char* sab,
                                               size_t sas, int m, int row, float (&yv)[MB]) {
  const int H = es.H, I = es.I, ngI = I / 64;
  constexpr int kWpg = BITS == 4 ? 8 : 4;
  const RecordLayout L = record_layout(BITS, H, I);
  const uint32_t* codes = reinterpret_cast<const uint32_t*>(rec + L.down_codes) + row;
  const uint32_t* sbw = reinterpret_cast<const uint32_t*>(rec + L.down_sb) + row;
  // unrolled so that several groups' loads are in flight per thread
#pragma unroll 4
  for (int g = 0; g < ngI; ++g) {
    uint32_t wd[kWpg];
#pragma unroll
    for (int b = 0; b < kWpg; ++b) wd[b] = ld_stream_u32(codes + (size_t)(g * kWpg + b) * H);
    const uint32_t sb = ld_stream_u32(sbw + (size_t)g * H);
#pragma unroll
    for (int i = 0; i < MB; ++i) {
      if (i < m) {
        const StagedX sx = staged_i(sab, sas, i, I);
        Acc2 acc{0, 0};
#pragma unroll
        for (int b = 0; b < kWpg; ++b) {
          if (BITS == 4) acc = acc + word_dot4(wd[b], sx.xs[b * ngI + g], sx.xl[b * ngI + g]);
          else
            acc = acc + word_dot2(wd[b], sx.xs[(2 * b) * ngI + g], sx.xs[(2 * b + 1) * ngI + g],
                                  sx.xl[(2 * b) * ngI + g], sx.xl[(2 * b + 1) * ngI + g]);
        }
        yv[i] = group_epilogue(yv[i], sb, acc, sx.delta[g], sx.xsum[g]);
      }
    }
  }
}

// Down product of one GEMV item (m <= MB tokens) for hidden rows
// blockIdx.y * kDnRows + thread; one hidden row per thread.
template <int MB>
__device__ __forceinline__ void down_group_body(const ExpertSet& es, const GroupWork& w, int bucket, int max_items,
                                                int item, const float* __restrict__ a, float* __restrict__ y) {
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ int s_slot[kGrpMaxM];
  if (item >= w.n_items[2 + bucket]) return;
  const int4 it = w.bitems[(size_t)bucket * max_items + item];
  const int g = it.x, m = it.z;
  if (threadIdx.x < m) s_slot[threadIdx.x] = w.slots[w.offset[g] + it.y + threadIdx.x];
  __syncthreads();
  const size_t sas = (staged_x_bytes(es.I) + 15) & ~(size_t)15;
  for (int i = 0; i < m; ++i) stage_x(a + (size_t)s_slot[i] * es.I, es.I, staged_i(smem, sas, i, es.I));
  __syncthreads();
  const int row = (int)blockIdx.y * kDnRows + (int)threadIdx.x;
  if (row >= es.H) return;
  float yv[MB];
#pragma unroll
  for (int i = 0; i < MB; ++i) yv[i] = 0.f;
  int bits;
  const uint8_t* rec = group_record(es, g, &bits);
  if (bits == 4) down_row_multi<4, MB>(rec, es, smem, sas, m, row, yv);
  else down_row_multi<2, MB>(rec, es, smem, sas, m, row, yv);
#pragma unroll
  for (int i = 0; i < MB; ++i)
    if (i < m) y[(size_t)s_slot[i] * es.H + row] = yv[i];
}


// grid (max items, H / kDnRows), one size bucket of GEMV items (m <= MB).
template <int MB>
__global__ void __launch_bounds__(kDnRows)
down_group_kernel(ExpertSet es, GroupWork w, int bucket, int max_items, const float* __restrict__ a,
                  float* __restrict__ y) {
  down_group_body<MB>(es, w, bucket, max_items, (int)blockIdx.x, a, y);
}

// grid (n0 + n1, H / kDnRows): buckets 0 and 1 in one launch.
__global__ void __launch_bounds__(kDnRows)
down_group_small_kernel(ExpertSet es, GroupWork w, int max_items, int n0, const float* __restrict__ a,
                        float* __restrict__ y) {
  if ((int)blockIdx.x < n0) down_group_body<2>(es, w, 0, max_items, (int)blockIdx.x, a, y);
  else down_group_body<4>(es, w, 1, max_items, (int)blockIdx.x - n0, a, y);
}

}  // namespace fmoe
