// fmoe_fused.cuh -- one persistent kernel for a stack of MoE layers, batch 1.
//
// One CTA per SM, launched cooperatively so that every CTA is resident and
// grid-wide barriers are safe.  Each layer runs in three phases separated by
// grid barriers -- the three global dependencies of the layer:
//   P1  router rows and the shared expert's gate/up rows (neither depends on
//       routing) -> logits, gamma, the shared expert's SwiGLU outputs
//   --  barrier: all logits written
//   P2  every CTA takes the top-k of the logits itself, then streams its
//       share of the routed experts' gate/up rows -> SwiGLU outputs a, while
//       the routed experts' down rows it will need are already on the way
//   --  barrier: every a written
//   P3  down rows (already in shared memory) of all k + 1 experts for this
//       CTA's slice of the hidden dimension -> y; weighted combine +
//       residual -> h', and this CTA's part of sum(h'^2)
//   --  barrier: every h' and partial sum written
// The next layer (or the epilogue) turns h' into xn' = h' r w with
// r = (sum h'^2 / H + eps)^(-1/2), every CTA for the whole vector.
// Source pages: "What is Flash-MoE?" (a2a-mcp.org), sections
// "Understanding Mixture-of-Experts", "2. FMA-optimised dequantisation
// kernels" and "3. Hand-tuned Metal compute shaders" (deferred command-buffer
// submission there plays the role the persistent kernel plays here: no host
// round trip between the steps or between layers).
//
// Weight bytes move global -> shared with cp.async.bulk (the bulk-copy
// engine), completion tracked by mbarriers; every weight byte is read from
// HBM exactly once per layer.  Every wait (mbarrier or grid barrier) is
// bounded: on expiry the CTA sets FMOE_STATUS_WAIT_TIMEOUT, waits (bounded)
// for its own copies in flight, and returns.
#pragma once

#include <cstdint>

#include "fmoe.h"
#include "fmoe_device.cuh"
#include "fmoe_layout.h"

namespace fmoe {

constexpr int kFusedThreads = 512;
constexpr int kFusedWarps = kFusedThreads / 32;
constexpr int kFusedMaxLayers = 32;
constexpr int kFusedMaxRouterRows = 8;
constexpr int kFusedMaxSharedPairs = 32;
constexpr int kFusedMaxRoutedPairs = 96;
constexpr int kFusedMaxK = 8;
constexpr int kMbRouter = 0;
constexpr int kMbSPair = kMbRouter + kFusedMaxRouterRows;
constexpr int kMbSDown = kMbSPair + kFusedMaxSharedPairs;
constexpr int kMbRPair = kMbSDown + 1;
constexpr int kMbRDown = kMbRPair + kFusedMaxRoutedPairs;
constexpr int kMbCount = kMbRDown + kFusedMaxK;
constexpr long long kWaitCycles = 4000000000LL;  // ~2 s at 2 GHz

struct FusedLayer {
  const uint8_t* experts;
  const uint8_t* shared;
  const float* w_router;
  const float* w_sg;
  const float* norm_w;
};

// Shared-memory plan (byte offsets), computed on the host.
struct FusedPlan {
  uint32_t region_a;     // P1: router rows + shared pairs; P2: routed pairs; P3: staged a
  uint32_t region_b;     // shared down rows, then routed down rows (x in fp32 during P1)
  uint32_t xf;           // fp32 x (may alias the routed part of region B)
  uint32_t xq;           // staged int16 x
  uint32_t logit;        // fp32 [E]
  uint32_t ypart;        // fp32 [(k+1)][down rows]
  uint32_t rpart;        // fp32 [router rows][slices]
  uint32_t mbar;
  uint32_t total;
};

struct FusedArgs {
  FusedLayer layers[kFusedMaxLayers];
  int n_layers;
  int H, I, E, k, bits, sbits;
  float eps;
  float* h;
  float* xn;
  float* logits;
  int32_t* ids;
  float* weights;
  float* gamma;
  float* a;        // [(k+1)][I], shared expert last
  float* y;        // [(k+1)][H]
  float* ss_part;  // [gridDim.x]
  unsigned* sync;  // [0] barrier arrivals, [1] exits
  FusedPlan plan;
};

// ------------------------------------------------------------ primitives --
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cta.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ bool mbar_try(uint64_t* bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2; selp.u32 %0, 1, 0, p; }"
      : "=r"(done)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return done != 0;
}

// Bounded wait for phase `parity` of an mbarrier to complete.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
  if (mbar_try(bar, parity)) return true;
  const long long t0 = clock64();
  while (clock64() - t0 < kWaitCycles)
    if (mbar_try(bar, parity)) return true;
  return false;
}

__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// 16-byte shared-memory load (a plain load, so the compiler may schedule it
// freely but never above an mbarrier wait, whose asm clobbers memory).
__device__ __forceinline__ uint4 lds128(const void* p) { return *reinterpret_cast<const uint4*>(p); }

__device__ __forceinline__ float ldcg_f(const float* p) { return __ldcg(p); }

// [lo, hi) share of `total` items for part `c` of `n`
__device__ __forceinline__ void share(int total, int c, int n, int* lo, int* hi) {
  *lo = (int)(((long long)total * c) / n);
  *hi = (int)(((long long)total * (c + 1)) / n);
}

// ------------------------------------------------------ GEMV from smem --
template <int BITS>
__device__ __forceinline__ GroupCodes<BITS> lds_group(const uint8_t* row, int ng, int g) {
  GroupCodes<BITS> gc;
  gc.c[0] = lds128(row + chunk_off<BITS>(ng, g, 0));
  if (BITS == 4) gc.c[BITS == 4 ? 1 : 0] = lds128(row + chunk_off<BITS>(ng, g, 1));
  return gc;
}

__device__ __forceinline__ void lds_xv(const StagedX& s, int ng, int g, uint4* xv) {
#pragma unroll
  for (int u = 0; u < 8; ++u) xv[u] = lds128(s.xs + u * ng + g);
}

// Dot products of gate and up row of a pair held in shared memory (codes of
// both rows, then their scale-bias words), one lane group per pair.
template <int BITS>
__device__ __forceinline__ void pair_dot_smem(const uint8_t* slot, int H, const StagedX& sx, int lg,
                                              int lpr, float* yg, float* yu) {
  const int ng = H / 64;
  const int rb = H * BITS / 8;
  const uint8_t* rg = slot;
  const uint8_t* ru = slot + rb;
  const uint32_t* sbg = reinterpret_cast<const uint32_t*>(slot + 2 * rb);
  const uint32_t* sbu = sbg + ng;
  float g = 0.f, u = 0.f;
  for (int gi = lg; gi < ng; gi += lpr) {
    const GroupCodes<BITS> cg = lds_group<BITS>(rg, ng, gi);
    const GroupCodes<BITS> cu = lds_group<BITS>(ru, ng, gi);
    uint4 xv[8];
    lds_xv(sx, ng, gi, xv);
    const float d = sx.delta[gi], xs = sx.xsum[gi];
    g = group_epilogue(g, sbg[gi], group_dot<BITS>(cg, xv), d, xs);
    u = group_epilogue(u, sbu[gi], group_dot<BITS>(cu, xv), d, xs);
  }
  for (int o = lpr >> 1; o > 0; o >>= 1) {
    g += __shfl_xor_sync(0xffffffffu, g, o);
    u += __shfl_xor_sync(0xffffffffu, u, o);
  }
  *yg = g;
  *yu = u;
}

// Dot product of one down row held in shared memory (codes block, scale-bias block).
template <int BITS>
__device__ __forceinline__ float row_dot_smem(const uint8_t* codes, const uint32_t* sb, int I,
                                              const StagedX& sx, int lg, int lpr) {
  const int ng = I / 64;
  float y = 0.f;
  for (int gi = lg; gi < ng; gi += lpr) {
    const GroupCodes<BITS> c = lds_group<BITS>(codes, ng, gi);
    uint4 xv[8];
    lds_xv(sx, ng, gi, xv);
    y = group_epilogue(y, sb[gi], group_dot<BITS>(c, xv), sx.delta[gi], sx.xsum[gi]);
  }
  for (int o = lpr >> 1; o > 0; o >>= 1) y += __shfl_xor_sync(0xffffffffu, y, o);
  return y;
}

// Warp-level top-k over lg[0..E) (shared memory): lane r < k returns the
// r-th selection in *id / *val.  Larger first, NaN last, ties to the lower index.
__device__ __forceinline__ void warp_topk(const float* lg, int E, int k, int* id, float* val) {
  const int lane = threadIdx.x & 31;
  uint32_t taken = 0;
  int my_id = 0;
  float my_val = 0.f;
  for (int r = 0; r < k; ++r) {
    float bv = 0.f;
    int bi = -1;
    for (int i = 0, e = lane; e < E; ++i, e += 32) {
      if (taken & (1u << i)) continue;
      const float v = lg[e];
      bool better;
      if (bi < 0) better = true;
      else {
        const bool an = isnan(v), bn = isnan(bv);
        better = (an || bn) ? (an && bn ? e < bi : bn) : (v != bv ? v > bv : e < bi);
      }
      if (better) { bv = v; bi = e; }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      bool better;
      if (oi < 0) better = false;
      else if (bi < 0) better = true;
      else {
        const bool an = isnan(ov), bn = isnan(bv);
        better = (an || bn) ? (an && bn ? oi < bi : bn) : (ov != bv ? ov > bv : oi < bi);
      }
      if (better) { bv = ov; bi = oi; }
    }
    if (bi >= 0 && (bi & 31) == lane) taken |= 1u << (bi >> 5);
    if (lane == r) { my_id = bi; my_val = bv; }
  }
  *id = my_id;
  *val = my_val;
}

// ------------------------------------------------------------ the kernel --
__global__ void __launch_bounds__(kFusedThreads, 1) fused_stack_kernel(const __grid_constant__ FusedArgs A) {
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ int s_abort;
  __shared__ int s_ids[kFusedMaxK];
  __shared__ float s_p[kFusedMaxK];
  __shared__ float s_red[kFusedWarps];
  __shared__ float s_r;

  const int c = blockIdx.x, nC = gridDim.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int H = A.H, I = A.I, E = A.E, k = A.k;
  const int ngH = H / 64, ngI = I / 64;
  const int lprH = ngH < 32 ? ngH : 32, lprI = ngI < 32 ? ngI : 32;
  const FusedPlan& P = A.plan;
  uint64_t* mbar = reinterpret_cast<uint64_t*>(smem + P.mbar);
  uint8_t* regA = smem + P.region_a;
  uint8_t* regB = smem + P.region_b;
  float* xf = reinterpret_cast<float*>(smem + P.xf);
  const StagedX sxq = staged_x_at(smem + P.xq, H);
  float* slog = reinterpret_cast<float*>(smem + P.logit);
  float* ypart = reinterpret_cast<float*>(smem + P.ypart);
  float* rpart = reinterpret_cast<float*>(smem + P.rpart);

  // static work shares of this CTA
  int r0, r1, s0, s1, q0, q1, i0, i1;
  share(E + 1, c, nC, &r0, &r1);  // router rows; row E is the shared gate vector
  share(I, c, nC, &s0, &s1);      // shared expert gate/up pairs
  share(k * I, c, nC, &q0, &q1);  // routed gate/up pairs, expert-major
  share(H, c, nC, &i0, &i1);      // hidden rows of the down products and the combine
  const int nr = r1 - r0, nsp = s1 - s0, nq = q1 - q0, nd = i1 - i0;
  const int nsl = H >= 512 ? H / 512 : 1;  // router slices per row
  const int sl_len = H / nsl;

  const RecordLayout LR = record_layout(A.bits, H, I);   // routed records
  const RecordLayout LS = record_layout(A.sbits, H, I);  // shared record
  const uint32_t pair_r = (uint32_t)(2 * LR.gu_row_bytes + 2 * ngH * 4);
  const uint32_t pair_s = (uint32_t)(2 * LS.gu_row_bytes + 2 * ngH * 4);
  const uint32_t drow_r = (uint32_t)(LR.down_row_bytes), drow_s = (uint32_t)(LS.down_row_bytes);
  // region B: shared down [codes nd*drow_s][sb nd*ngI*4], then routed down per expert
  uint8_t* sd_codes = regB;
  uint32_t* sd_sb = reinterpret_cast<uint32_t*>(regB + (size_t)nd * drow_s);
  uint8_t* rd_base = regB + (size_t)nd * (drow_s + ngI * 4);
  const size_t rd_stride = (size_t)nd * (drow_r + ngI * 4);

  if (tid == 0) {
    s_abort = 0;
    for (int i = 0; i < kMbCount; ++i) mbar_init(&mbar[i], 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();

  unsigned bar_target = 0;
  uint32_t cur_par = 0;
  // slots armed by this lane of warp 0 in the current layer (bulk copies are
  // issued by the lanes of warp 0; each lane drains its own on abort)
  uint32_t armed[(kMbCount + 31) / 32];
#pragma unroll
  for (int i = 0; i < (kMbCount + 31) / 32; ++i) armed[i] = 0;

  auto arm = [&](int slot, uint32_t bytes) {
    mbar_expect_tx(&mbar[slot], bytes);
    armed[slot >> 5] |= 1u << (slot & 31);
  };

  auto grid_sync = [&]() -> bool {
    __syncthreads();
    bar_target += (unsigned)nC;
    if (tid == 0) {
      __threadfence();
      atomicAdd(&A.sync[0], 1u);
      const long long t0 = clock64();
      bool ok = false;
      while (true) {
        const unsigned v = *reinterpret_cast<volatile unsigned*>(&A.sync[0]);
        if (v >= bar_target) { ok = true; break; }
        if (clock64() - t0 > kWaitCycles) break;
      }
      __threadfence();
      if (!ok) {
        s_abort = 1;
        raise_status(FMOE_STATUS_WAIT_TIMEOUT);
      }
    }
    __syncthreads();
    return !s_abort;
  };

  auto wait_slot = [&](int slot, uint32_t parity) -> bool {
    if (mbar_wait(&mbar[slot], parity)) return true;
    s_abort = 1;
    raise_status(FMOE_STATUS_WAIT_TIMEOUT);
    return false;
  };

  for (int l = 0; l < A.n_layers; ++l) {
    const FusedLayer& LY = A.layers[l];
    const uint32_t par = (uint32_t)(l & 1);
    cur_par = par;
    // ------------------------------------------------------------ P1 --
    if (warp == 0) {
#pragma unroll
      for (int i = 0; i < (kMbCount + 31) / 32; ++i) armed[i] = 0;
      fence_proxy_async();
      for (int r = lane; r < nr; r += 32) {
        const int row = r0 + r;
        const float* src = row < E ? LY.w_router + (size_t)row * H : LY.w_sg;
        arm(kMbRouter + r, (uint32_t)H * 4);
        bulk_g2s(regA + (size_t)r * H * 4, src, (uint32_t)H * 4, &mbar[kMbRouter + r]);
      }
      uint8_t* sp_base = regA + (size_t)nr * H * 4;
      for (int p = lane; p < nsp; p += 32) {
        const int n = s0 + p;
        uint8_t* dst = sp_base + (size_t)p * pair_s;
        arm(kMbSPair + p, pair_s);
        bulk_g2s(dst, LY.shared + LS.gu_codes + (size_t)(2 * n) * LS.gu_row_bytes,
                 (uint32_t)(2 * LS.gu_row_bytes), &mbar[kMbSPair + p]);
        bulk_g2s(dst + 2 * LS.gu_row_bytes, LY.shared + LS.gu_sb + (size_t)(2 * n) * ngH * 4,
                 (uint32_t)(2 * ngH * 4), &mbar[kMbSPair + p]);
      }
      if (nd > 0 && lane == 31) {
        arm(kMbSDown, (uint32_t)nd * (drow_s + ngI * 4));
        bulk_g2s(sd_codes, LY.shared + LS.down_codes + (size_t)i0 * drow_s, (uint32_t)nd * drow_s,
                 &mbar[kMbSDown]);
        bulk_g2s(sd_sb, LY.shared + LS.down_sb + (size_t)i0 * ngI * 4, (uint32_t)nd * ngI * 4,
                 &mbar[kMbSDown]);
      }
    }
    // x for this layer: the input (first layer) or h' r w of the previous layer
    if (l == 0) {
      for (int j = tid; j < H; j += kFusedThreads) xf[j] = ldcg_f(A.xn + j);
    } else {
      if (warp == 0) {
        float s = 0.f;
        for (int i = lane; i < nC; i += 32) s += ldcg_f(A.ss_part + i);
        s = warp_sum(s);
        if (lane == 0) s_r = 1.f / sqrtf(s / (float)H + A.eps);
      }
      __syncthreads();
      const float r = s_r;
      const float* wprev = A.layers[l - 1].norm_w;
      for (int j = tid; j < H; j += kFusedThreads) xf[j] = ldcg_f(A.h + j) * r * wprev[j];
    }
    __syncthreads();
    stage_x(xf, H, sxq);
    __syncthreads();
    // router rows: units (row, slice)
    for (int u = warp; u < nr * nsl; u += kFusedWarps) {
      const int r = u / nsl, sl = u % nsl;
      if (!wait_slot(kMbRouter + r, par)) break;
      const float* w = reinterpret_cast<const float*>(regA) + (size_t)r * H + sl * sl_len;
      const float* x = xf + sl * sl_len;
      float acc = 0.f;
      for (int cc = lane * 4; cc < sl_len; cc += 128) {
        const float4 wv = *reinterpret_cast<const float4*>(w + cc);
        const float4 xv = *reinterpret_cast<const float4*>(x + cc);
        acc = fmaf(wv.x, xv.x, acc);
        acc = fmaf(wv.y, xv.y, acc);
        acc = fmaf(wv.z, xv.z, acc);
        acc = fmaf(wv.w, xv.w, acc);
      }
      acc = warp_sum(acc);
      if (lane == 0) rpart[r * nsl + sl] = acc;
    }
    // shared expert gate/up pairs
    {
      const int ppu = 32 / lprH;  // pairs per warp unit
      const int ps = lane / lprH, lg = lane % lprH;
      const uint8_t* sp_base = regA + (size_t)nr * H * 4;
      for (int u0 = warp * ppu; u0 < nsp; u0 += kFusedWarps * ppu) {
        const int p = u0 + ps;
        bool ok = true;
        if (p < nsp) ok = wait_slot(kMbSPair + p, par);
        if (!__all_sync(0xffffffffu, ok)) break;
        float g = 0.f, uu = 0.f;
        const int pp = p < nsp ? p : nsp - 1;
        if (A.sbits == 4)
          pair_dot_smem<4>(sp_base + (size_t)pp * pair_s, H, sxq, lg, lprH, &g, &uu);
        else
          pair_dot_smem<2>(sp_base + (size_t)pp * pair_s, H, sxq, lg, lprH, &g, &uu);
        if (lg == 0 && p < nsp) A.a[(size_t)k * I + s0 + p] = silu_mul(g, uu);
      }
    }
    __syncthreads();
    if (tid < nr && !s_abort) {
      float v = rpart[tid * nsl];
      for (int sl = 1; sl < nsl; ++sl) v += rpart[tid * nsl + sl];
      const int row = r0 + tid;
      if (row < E) A.logits[row] = v;
      else A.gamma[0] = 1.f / (1.f + expf(-v));
    }
    if (s_abort || !grid_sync()) break;
    // ------------------------------------------------------------ P2 --
    if (warp == 0) {
      bool nan_seen = false;
      for (int e = lane; e < E; e += 32) {
        const float v = ldcg_f(A.logits + e);
        nan_seen |= isnan(v);
        slog[e] = v;
      }
      __syncwarp();
      int id;
      float val;
      warp_topk(slog, E, k, &id, &val);
      float m = -INFINITY;
      for (int r = 0; r < k; ++r) {
        const float vr = __shfl_sync(0xffffffffu, val, r);
        if (!isnan(vr)) m = fmaxf(m, vr);
      }
      const float pe = (lane < k && !isnan(val)) ? expf(val - m) : 0.f;
      const float z = warp_sum(pe);
      if (lane < k) {
        s_ids[lane] = id;
        s_p[lane] = z > 0.f ? pe / z : 0.f;
        if (c == 0) {
          A.ids[lane] = id;
          A.weights[lane] = s_p[lane];
        }
      }
      const bool any_nan = __any_sync(0xffffffffu, nan_seen);
      if (c == 0 && lane == 0 && any_nan) raise_status(FMOE_STATUS_NAN_LOGIT);
    }
    __syncthreads();
    if (warp == 0) {
      fence_proxy_async();
      for (int q = lane; q < nq; q += 32) {
        const int gq = q0 + q, j = gq / I, n = gq % I;
        const uint8_t* rec = LY.experts + (size_t)s_ids[j] * LR.bytes;
        uint8_t* dst = regA + (size_t)q * pair_r;
        arm(kMbRPair + q, pair_r);
        bulk_g2s(dst, rec + LR.gu_codes + (size_t)(2 * n) * LR.gu_row_bytes, (uint32_t)(2 * LR.gu_row_bytes),
                 &mbar[kMbRPair + q]);
        bulk_g2s(dst + 2 * LR.gu_row_bytes, rec + LR.gu_sb + (size_t)(2 * n) * ngH * 4, (uint32_t)(2 * ngH * 4),
                 &mbar[kMbRPair + q]);
      }
      if (nd > 0) {
        for (int j = lane; j < k; j += 32) {
          const uint8_t* rec = LY.experts + (size_t)s_ids[j] * LR.bytes;
          uint8_t* dst = rd_base + (size_t)j * rd_stride;
          arm(kMbRDown + j, (uint32_t)nd * (drow_r + ngI * 4));
          bulk_g2s(dst, rec + LR.down_codes + (size_t)i0 * drow_r, (uint32_t)nd * drow_r, &mbar[kMbRDown + j]);
          bulk_g2s(dst + (size_t)nd * drow_r, rec + LR.down_sb + (size_t)i0 * ngI * 4, (uint32_t)nd * ngI * 4,
                   &mbar[kMbRDown + j]);
        }
      }
    }
    {
      const int ppu = 32 / lprH;
      const int ps = lane / lprH, lg = lane % lprH;
      for (int u0 = warp * ppu; u0 < nq; u0 += kFusedWarps * ppu) {
        const int q = u0 + ps;
        bool ok = true;
        if (q < nq) ok = wait_slot(kMbRPair + q, par);
        if (!__all_sync(0xffffffffu, ok)) break;
        float g = 0.f, uu = 0.f;
        const int qq = q < nq ? q : nq - 1;
        if (A.bits == 4)
          pair_dot_smem<4>(regA + (size_t)qq * pair_r, H, sxq, lg, lprH, &g, &uu);
        else
          pair_dot_smem<2>(regA + (size_t)qq * pair_r, H, sxq, lg, lprH, &g, &uu);
        if (lg == 0 && q < nq) {
          const int gq = q0 + q;
          A.a[gq] = silu_mul(g, uu);  // a[j][n] with gq = j * I + n
        }
      }
    }
    if (s_abort || !grid_sync()) break;
    // ------------------------------------------------------------ P3 --
    // stage a of the k routed experts and the shared one (region A is free)
    const size_t sa_bytes = (staged_x_bytes(I) + 15) & ~(size_t)15;
    for (int j = 0; j <= k; ++j) stage_x(A.a + (size_t)j * I, I, staged_x_at(regA + j * sa_bytes, I), true);
    __syncthreads();
    if (nd > 0) {
      const int rpu = 32 / lprI;  // rows per warp unit
      const int rs = lane / lprI, lg = lane % lprI;
      const int units_per_expert = (nd + rpu - 1) / rpu;
      for (int u = warp; u < (k + 1) * units_per_expert; u += kFusedWarps) {
        const int j = u / units_per_expert, rr = (u % units_per_expert) * rpu + rs;
        const bool shared = j == k;
        bool ok = wait_slot(shared ? kMbSDown : kMbRDown + j, par);
        if (!__all_sync(0xffffffffu, ok)) break;
        const StagedX sa = staged_x_at(regA + j * sa_bytes, I);
        const int row = rr < nd ? rr : nd - 1;
        float v;
        if (shared) {
          const uint8_t* codes = sd_codes + (size_t)row * drow_s;
          const uint32_t* sb = sd_sb + (size_t)row * ngI;
          v = A.sbits == 4 ? row_dot_smem<4>(codes, sb, I, sa, lg, lprI) : row_dot_smem<2>(codes, sb, I, sa, lg, lprI);
        } else {
          const uint8_t* base = rd_base + (size_t)j * rd_stride;
          const uint8_t* codes = base + (size_t)row * drow_r;
          const uint32_t* sb = reinterpret_cast<const uint32_t*>(base + (size_t)nd * drow_r) + (size_t)row * ngI;
          v = A.bits == 4 ? row_dot_smem<4>(codes, sb, I, sa, lg, lprI) : row_dot_smem<2>(codes, sb, I, sa, lg, lprI);
        }
        if (lg == 0 && rr < nd) ypart[j * nd + rr] = v;
      }
    }
    __syncthreads();
    if (s_abort) break;
    {
      const float gm = ldcg_f(A.gamma);
      float ss = 0.f;
      for (int rr = tid; rr < nd; rr += kFusedThreads) {
        const int i = i0 + rr;
        float v = ldcg_f(A.h + i);
        for (int j = 0; j < k; ++j) v = fmaf(s_p[j], ypart[j * nd + rr], v);
        v = fmaf(gm, ypart[k * nd + rr], v);
        A.h[i] = v;
        for (int j = 0; j <= k; ++j) A.y[(size_t)j * H + i] = ypart[j * nd + rr];
        ss = fmaf(v, v, ss);
      }
      ss = warp_sum(ss);
      if (lane == 0) s_red[warp] = ss;
      __syncthreads();
      if (tid == 0) {
        float t = 0.f;
        for (int w = 0; w < kFusedWarps; ++w) t += s_red[w];
        A.ss_part[c] = t;
      }
    }
    if (!grid_sync()) break;
  }

  if (!s_abort) {
    // epilogue: xn' of the last layer for this CTA's rows
    if (warp == 0) {
      float s = 0.f;
      for (int i = lane; i < nC; i += 32) s += ldcg_f(A.ss_part + i);
      s = warp_sum(s);
      if (lane == 0) s_r = 1.f / sqrtf(s / (float)H + A.eps);
    }
    __syncthreads();
    const float r = s_r;
    const float* w = A.layers[A.n_layers - 1].norm_w;
    for (int i = i0 + tid; i < i1; i += kFusedThreads) A.xn[i] = ldcg_f(A.h + i) * r * w[i];
    __syncthreads();
    if (tid == 0) {
      __threadfence();
      const unsigned prev = atomicAdd(&A.sync[1], 1u);
      if (prev == (unsigned)nC - 1) {  // every CTA is past its last barrier
        A.sync[0] = 0;
        A.sync[1] = 0;
        __threadfence();
      }
    }
  } else if (warp == 0) {
    // drain: wait (bounded) for this lane's own copies still in flight
    for (int s = 0; s < kMbCount; ++s)
      if (armed[s >> 5] & (1u << (s & 31))) (void)mbar_wait(&mbar[s], cur_par);
  }
}

// Host-side plan: shared-memory layout for n_ctas CTAs; false if it does not fit.
inline bool fused_plan(int H, int I, int E, int k, int bits, int sbits, int n_ctas, size_t max_smem,
                       FusedPlan* out) {
  // every per-CTA block moved by cp.async.bulk and every 16-byte shared load
  // must be 16-byte aligned: a down row's scale-bias words (I/64 * 4 bytes)
  // and a pair's (2 * H/64 * 4 bytes) must come in multiples of 16 bytes
  if ((I / 64) % 4 != 0 || (H / 64) % 2 != 0) return false;
  auto cdiv = [](long long a, long long b) { return (a + b - 1) / b; };
  const long long nr = cdiv(E + 1, n_ctas), nsp = cdiv(I, n_ctas), nq = cdiv((long long)k * I, n_ctas),
                  nd = cdiv(H, n_ctas);
  if (nr > kFusedMaxRouterRows || nsp > kFusedMaxSharedPairs || nq > kFusedMaxRoutedPairs || k > kFusedMaxK)
    return false;
  const RecordLayout LR = record_layout(bits, H, I), LS = record_layout(sbits, H, I);
  const int ngH = H / 64, ngI = I / 64;
  const long long pair_r = 2 * (long long)LR.gu_row_bytes + 2 * ngH * 4;
  const long long pair_s = 2 * (long long)LS.gu_row_bytes + 2 * ngH * 4;
  const long long sa = ((long long)staged_x_bytes(I) + 15) & ~15LL;
  auto al = [](long long v) { return (v + 127) & ~127LL; };
  const long long a_p1 = nr * H * 4 + nsp * pair_s;
  const long long a_p2 = nq * pair_r;
  const long long a_p3 = (k + 1) * sa;
  long long regA = a_p1 > a_p2 ? a_p1 : a_p2;
  regA = regA > a_p3 ? regA : a_p3;
  const long long sdown = nd * ((long long)LS.down_row_bytes + ngI * 4);
  const long long rdown = k * nd * ((long long)LR.down_row_bytes + ngI * 4);
  FusedPlan p;
  long long o = 0;
  p.region_a = (uint32_t)o;
  o = al(o + regA);
  p.region_b = (uint32_t)o;
  const long long xf_bytes = (long long)(H > I ? H : I) * 4;
  if (rdown >= xf_bytes) {
    p.xf = (uint32_t)(o + sdown);  // aliases the routed down rows (P1 / P3 staging only)
    o = al(o + sdown + rdown);
  } else {
    o = al(o + sdown + rdown);
    p.xf = (uint32_t)o;
    o = al(o + xf_bytes);
  }
  p.xq = (uint32_t)o;
  o = al(o + (long long)staged_x_bytes(H));
  p.logit = (uint32_t)o;
  o = al(o + (long long)E * 4);
  p.ypart = (uint32_t)o;
  o = al(o + (k + 1) * nd * 4);
  p.rpart = (uint32_t)o;
  o = al(o + nr * (H >= 512 ? H / 512 : 1) * 4);
  p.mbar = (uint32_t)o;
  o = al(o + kMbCount * 8);
  p.total = (uint32_t)o;
  if ((size_t)o > max_smem) return false;
  *out = p;
  return true;
}

}  // namespace fmoe
