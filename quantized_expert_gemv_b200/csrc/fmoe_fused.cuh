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

#include <cuda.h>  // CUtensorMap

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
constexpr int kPairsPerChunk = 4;  // gate/up row pairs per bulk-copy chunk (one mbarrier)
constexpr int kMbRouter = 0;
constexpr int kMbSPair = kMbRouter + kFusedMaxRouterRows;
constexpr int kMbSDown = kMbSPair + kFusedMaxSharedPairs / kPairsPerChunk;
constexpr int kMbRPair = kMbSDown + 1;
constexpr int kMbRDown = kMbRPair + kFusedMaxRoutedPairs / kPairsPerChunk;
constexpr int kMbCount = kMbRDown + kFusedMaxK;
constexpr long long kWaitCycles = 4000000000LL;  // ~2 s at 2 GHz
constexpr int kSyncGroups = 2;        // first per-group publication counter in FusedArgs::sync
constexpr int kMaxGroupCounters = 1022;
constexpr int kWStage = 144;          // per-warp staged a-group: 8 uint4 + delta + xsum (+pad)
constexpr int kMaxSliceRows = 64;     // hidden rows per CTA in the down products (2 per lane)
// Down rows reach shared memory through 3-D tensor copies whose box is
// kRowPadWords wider than a row: the tensor engine zero-fills the excess, so
// consecutive rows land 16 bytes off the 128-byte bank period and lanes
// reading one row each do not collide on banks.
constexpr int kRowPadWords = 4;
enum { kTmRoutedCodes = 0, kTmRoutedSb = 1, kTmSharedCodes = 2, kTmSharedSb = 3, kTmPerLayer = 4 };

struct FusedLayer {
  const uint8_t* experts;
  const uint8_t* shared;
  const float* w_router;
  const float* w_sg;
  const float* norm_w;
};

// Shared-memory plan (byte offsets), computed on the host.
//   region A  P1: router rows, shared pairs' codes, shared pairs' scale-bias
//             P2: routed pairs' codes, routed pairs' scale-bias
//   region B  shared down rows, then routed down rows (fp32 x during P1)
//   xq        staged int16 x (P1, P2), then the staged SwiGLU outputs (P3)
struct FusedPlan {
  uint32_t region_a;
  uint32_t region_b;
  uint32_t xf;     // fp32 x (may alias the routed part of region B)
  uint32_t xq;
  uint32_t logit;  // fp32 [E]
  uint32_t cand;   // top-k candidates: fp32 [warps][k] values, int32 [warps][k] ids
  uint32_t ypart;  // fp32 [(k+1)][down rows]
  uint32_t rpart;  // fp32 [router rows][slices]
  uint32_t cons;   // inside region A, past the P1 data (free once the routed pairs are
                   // consumed): per-warp staged a-groups, then per-warp partial down
                   // sums fp32 [warps][2][kMaxSliceRows]
  uint32_t prod;   // u32 [k * I / 64]: CTAs producing each routed a-group (static)
  uint32_t mbar;
  uint32_t nd_box;     // rows of every down-row tensor copy (the largest hidden slice)
  uint32_t sd_codes, sd_sb;         // offsets of the shared expert's padded down rows
  uint32_t rd_slot;                 // offset of the first routed expert's padded down rows
  uint32_t rd_stride;               // bytes per routed expert (codes then scale-bias)
  uint32_t rd_sb;                   // offset of the scale-bias rows inside a routed slot
  uint32_t total;
};

struct alignas(64) FusedArgs {
  CUtensorMap tm[kFusedMaxLayers][kTmPerLayer];  // down rows (codes, scale-bias) of the routed / shared records
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
  unsigned* sync;  // [0] barrier arrivals, [1] exits, [kSyncGroups + g] publications of a-group g
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

// One try_wait; the thread may be suspended (up to the hint, 20 us) until the
// phase completes, so waiting warps do not compete for issue slots.
// 3-D tensor copy global -> shared (box of `map` at coordinates c0, c1, c2).
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, int c0, int c1, int c2,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], "
      "[%5];" ::"r"(smem_u32(dst)),
      "l"(map), "r"(c0), "r"(c1), "r"(c2), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ bool mbar_try(uint64_t* bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, 20000; selp.u32 %0, 1, 0, p; }"
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
__device__ __forceinline__ void pair_dot_smem(const uint8_t* codes, const uint32_t* sb, int H,
                                              const StagedX& sx, int lg, int lpr, float* yg, float* yu) {
  const int ng = H / 64;
  const int rb = H * BITS / 8;
  const uint8_t* rg = codes;
  const uint8_t* ru = codes + rb;
  const uint32_t* sbg = sb;
  const uint32_t* sbu = sb + ng;
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

// Routing key of logit v at index e: one 64-bit integer whose order is the
// selection order -- larger value first, NaN after every number, +0 and -0
// equal, then the lower index.  Key 0 never names a logit ("none").
__device__ __forceinline__ uint64_t route_key(float v, int e) {
  uint32_t k32;
  if (isnan(v)) k32 = 0u;
  else {
    const uint32_t u = __float_as_uint(v == 0.f ? 0.f : v);
    k32 = (u >> 31) ? ~u : (u | 0x80000000u);
  }
  return ((uint64_t)k32 << 32) | (uint64_t)(0xFFFFFFFFu - (uint32_t)e);
}

__device__ __forceinline__ int key_index(uint64_t key) { return (int)(0xFFFFFFFFu - (uint32_t)key); }

// Warp-wide selection of the k largest keys among the PER keys each lane
// holds (0 = empty); the r-th selected key lands in lane r.  Two redux.sync
// reductions per selection.
template <int PER>
__device__ __forceinline__ uint64_t warp_select_keys(uint64_t* key, int k) {
  const int lane = threadIdx.x & 31;
  uint64_t mine = 0;
  for (int r = 0; r < k; ++r) {
    uint64_t best = key[0];
#pragma unroll
    for (int i = 1; i < PER; ++i) best = key[i] > best ? key[i] : best;
    const uint32_t hi = __reduce_max_sync(0xffffffffu, (uint32_t)(best >> 32));
    const uint32_t lo = __reduce_max_sync(0xffffffffu, (uint32_t)(best >> 32) == hi ? (uint32_t)best : 0u);
    const uint64_t win = ((uint64_t)hi << 32) | lo;
#pragma unroll
    for (int i = 0; i < PER; ++i)
      if (key[i] == win) key[i] = 0;
    if (lane == r) mine = win;
  }
  return mine;
}

// ------------------------------------------------------------ the kernel --
template <int BITS, int SBITS>  // routed and shared code widths
__global__ void __launch_bounds__(kFusedThreads, 1) fused_stack_kernel(const __grid_constant__ FusedArgs A) {
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ int s_abort;
  __shared__ int s_ids[kFusedMaxK];
  __shared__ float s_p[kFusedMaxK];
  __shared__ float s_red[kFusedWarps];

  const int c = blockIdx.x, nC = gridDim.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int H = A.H, I = A.I, E = A.E, k = A.k;
  const int ngH = H / 64, ngI = I / 64;
  const int lprH = ngH < 32 ? ngH : 32;
  const FusedPlan& P = A.plan;
  uint64_t* mbar = reinterpret_cast<uint64_t*>(smem + P.mbar);
  uint8_t* regA = smem + P.region_a;
  uint8_t* regB = smem + P.region_b;
  float* xf = reinterpret_cast<float*>(smem + P.xf);
  unsigned char* xq_base = smem + P.xq;
  const StagedX sxq = staged_x_at(xq_base, H);
  float* slog = reinterpret_cast<float*>(smem + P.logit);
  uint64_t* cand = reinterpret_cast<uint64_t*>(smem + P.cand);  // [warps][k] routing keys
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
  const uint32_t pc_r = (uint32_t)(2 * LR.gu_row_bytes), pc_s = (uint32_t)(2 * LS.gu_row_bytes);  // pair codes
  const uint32_t psb = (uint32_t)(2 * ngH * 4);                                                     // pair scale-bias
  const uint32_t drow_r = (uint32_t)(LR.down_row_bytes), drow_s = (uint32_t)(LS.down_row_bytes);
  // region A
  uint8_t* sc_codes = regA + (size_t)nr * H * 4;
  uint8_t* sc_sb = sc_codes + (size_t)nsp * pc_s;
  uint8_t* rc_codes = regA;
  uint8_t* rc_sb = regA + (size_t)nq * pc_r;
  // region B: the shared expert's padded down rows, then the routed experts'
  // (each: codes rows of drow + 16 bytes, then scale-bias rows of (I/64 + 4) words)
  (void)regB;
  uint8_t* sd_codes = smem + P.sd_codes;
  const uint32_t* sd_sb = reinterpret_cast<const uint32_t*>(smem + P.sd_sb);
  uint8_t* rd_base = smem + P.rd_slot;
  const size_t rd_stride = P.rd_stride;
  const uint32_t rd_sb_off = P.rd_sb;
  const uint32_t prow_r = drow_r + 4 * kRowPadWords, prow_s = drow_s + 4 * kRowPadWords;  // padded code rows
  const uint32_t psbrow = (uint32_t)(ngI + kRowPadWords);                                  // padded sb row, words
  const uint32_t box_r = P.nd_box * prow_r + P.nd_box * psbrow * 4;  // bytes of one routed expert's copies
  const uint32_t box_s = P.nd_box * prow_s + P.nd_box * psbrow * 4;
  uint8_t* cons = smem + P.cons;
  float* cons_wy = reinterpret_cast<float*>(cons + kFusedWarps * kWStage);
  // number of CTAs whose pair share touches a-group gg and publish it once per
  // layer: gg < k I / 64 are the routed experts' groups (routed pairs shared
  // out over k I pairs), the next I / 64 the shared expert's (I pairs)
  auto producers = [&](int gg) -> unsigned {
    const bool routed = gg < k * ngI;
    const int T = routed ? k * I : I;
    const int first = (routed ? gg : gg - k * ngI) * 64, last = first + 63;
    const int c_lo = (int)((((long long)first + 1) * nC - 1) / T);
    const int c_hi = (int)((((long long)last + 1) * nC - 1) / T);
    unsigned cnt = 0;
    for (int cc = c_lo; cc <= c_hi; ++cc) {
      int a0, a1;
      share(T, cc, nC, &a0, &a1);
      if (a0 < a1) ++cnt;
    }
    return cnt;
  };

  // static tables: producers of each routed a-group; first/last expert of each warp's groups
  unsigned* s_prod = reinterpret_cast<unsigned*>(smem + P.prod);
  const int U = (k + 1) * ngI;                              // a-groups: k routed experts, then the shared one
  const int per_warp = (U + kFusedWarps - 1) / kFusedWarps;  // a-groups per warp in the down products
  for (int gg = tid; gg < U; gg += kFusedThreads) s_prod[gg] = producers(gg);
  if (tid == 0) {
    s_abort = 0;
    for (int i = 0; i < kMbCount; ++i) mbar_init(&mbar[i], 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();

  unsigned bar_target = 0;
  // per issuing thread (lane 0 of a warp): slots armed, by the parity of their
  // latest arming (each issuer drains its own copies on abort)
  constexpr int kMW = (kMbCount + 31) / 32;
  uint32_t armed[2][kMW];
#pragma unroll
  for (int p = 0; p < 2; ++p)
#pragma unroll
    for (int i = 0; i < kMW; ++i) armed[p][i] = 0;
  auto arm = [&](int slot, uint32_t bytes, uint32_t parity) {
    mbar_expect_tx(&mbar[slot], bytes);
    armed[parity][slot >> 5] |= 1u << (slot & 31);
    armed[parity ^ 1][slot >> 5] &= ~(1u << (slot & 31));
  };

  // split grid barrier: arrive once this CTA's results are written, do local
  // work, then wait (release/acquire on one counter, bounded spin)
  auto grid_arrive = [&]() {
    __syncthreads();
    bar_target += (unsigned)nC;
    if (tid == 0) asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(A.sync) : "memory");
  };
  auto grid_wait = [&]() -> bool {
    if (tid == 0) {
      bool ok = false;
      const long long t0 = clock64();
      while (true) {
        unsigned v;
        asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(A.sync) : "memory");
        if (v >= bar_target) { ok = true; break; }
        if (clock64() - t0 > kWaitCycles) break;
      }
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

  // bulk copies, issued by lane 0 of several warps in parallel (each issue
  // takes a few hundred cycles; spreading them keeps any one warp short) ---
  // router rows and the shared expert's gate/up pairs of layer l (region A)
  auto issue_p1 = [&](int l) {
    const FusedLayer& LY = A.layers[l];
    const uint32_t par = (uint32_t)(l & 1);
    if (lane != 0) return;
    fence_proxy_async();
    for (int r = warp; r < nr; r += kFusedWarps) {
      const int row = r0 + r;
      const float* src = row < E ? LY.w_router + (size_t)row * H : LY.w_sg;
      arm(kMbRouter + r, (uint32_t)H * 4, par);
      bulk_g2s(regA + (size_t)r * H * 4, src, (uint32_t)H * 4, &mbar[kMbRouter + r]);
    }
    const int nch = (nsp + kPairsPerChunk - 1) / kPairsPerChunk;
    for (int ch = (warp + kFusedWarps - nr % kFusedWarps) % kFusedWarps; ch < nch; ch += kFusedWarps) {
      const int pa = ch * kPairsPerChunk, pb = min(nsp, pa + kPairsPerChunk), n = s0 + pa;
      arm(kMbSPair + ch, (uint32_t)(pb - pa) * (pc_s + psb), par);
      bulk_g2s(sc_codes + (size_t)pa * pc_s, LY.shared + LS.gu_codes + (size_t)n * pc_s, (uint32_t)(pb - pa) * pc_s,
               &mbar[kMbSPair + ch]);
      bulk_g2s(sc_sb + (size_t)pa * psb, LY.shared + LS.gu_sb + (size_t)n * psb, (uint32_t)(pb - pa) * psb,
               &mbar[kMbSPair + ch]);
    }
  };
  // the shared expert's down rows of layer l (region B, shared part)
  auto issue_sdown = [&](int l) {
    if (nd > 0 && lane == 0 && warp == kFusedWarps - 1) {
      fence_proxy_async();
      arm(kMbSDown, box_s, (uint32_t)(l & 1));
      tma_load_3d(sd_codes, &A.tm[l][kTmSharedCodes], 0, i0, 0, &mbar[kMbSDown]);
      tma_load_3d(const_cast<uint32_t*>(sd_sb), &A.tm[l][kTmSharedSb], 0, i0, 0, &mbar[kMbSDown]);
    }
  };
  // the routed experts' gate/up pairs of this CTA's share and down rows of its slice
  auto issue_routed = [&](int l) {
    const FusedLayer& LY = A.layers[l];
    const uint32_t par = (uint32_t)(l & 1);
    if (lane != 0) return;
    fence_proxy_async();
    const int nch = (nq + kPairsPerChunk - 1) / kPairsPerChunk;
    for (int ch = warp; ch < nch; ch += kFusedWarps) {
      const int qa = ch * kPairsPerChunk, qb = min(nq, qa + kPairsPerChunk);
      arm(kMbRPair + ch, (uint32_t)(qb - qa) * (pc_r + psb), par);
      for (int q = qa; q < qb;) {  // runs within one expert
        const int gq = q0 + q, j = gq / I, n = gq % I;
        const int cnt = min(qb - q, I - n);
        const uint8_t* rec = LY.experts + (size_t)s_ids[j] * LR.bytes;
        bulk_g2s(rc_codes + (size_t)q * pc_r, rec + LR.gu_codes + (size_t)n * pc_r, (uint32_t)cnt * pc_r,
                 &mbar[kMbRPair + ch]);
        bulk_g2s(rc_sb + (size_t)q * psb, rec + LR.gu_sb + (size_t)n * psb, (uint32_t)cnt * psb, &mbar[kMbRPair + ch]);
        q += cnt;
      }
    }
    if (nd > 0) {
      for (int j = (warp + kFusedWarps - nch % kFusedWarps) % kFusedWarps; j < k; j += kFusedWarps) {
        uint8_t* dst = rd_base + (size_t)j * rd_stride;
        arm(kMbRDown + j, box_r, par);
        tma_load_3d(dst, &A.tm[l][kTmRoutedCodes], 0, i0, s_ids[j], &mbar[kMbRDown + j]);
        tma_load_3d(dst + rd_sb_off, &A.tm[l][kTmRoutedSb], 0, i0, s_ids[j], &mbar[kMbRDown + j]);
      }
    }
  };

  // r = (sum of the CTAs' partial sums of h'^2 / H + eps)^(-1/2), the same
  // summation order in every CTA; all threads take part
  auto norm_scale = [&]() -> float {
    float v = 0.f;
    for (int i = tid; i < nC; i += kFusedThreads) v += ldcg_f(A.ss_part + i);
    v = warp_sum(v);
    if (lane == 0) s_red[warp] = v;
    __syncthreads();
    const float t = warp_sum(lane < kFusedWarps ? s_red[lane] : 0.f);  // same order in every warp
    return 1.f / sqrtf(t / (float)H + A.eps);
  };

  if (A.n_layers > 0) {
    issue_p1(0);
    issue_sdown(0);
  }

  for (int l = 0; l < A.n_layers; ++l) {
    const uint32_t par = (uint32_t)(l & 1);
    // ------------------------------------------------------------ P1 --
    // x for this layer: the input (first layer) or h' r w of the previous layer
    if (l == 0) {
      for (int j = tid * 4; j < H; j += kFusedThreads * 4)
        *reinterpret_cast<float4*>(xf + j) = __ldcg(reinterpret_cast<const float4*>(A.xn + j));
    } else {
      constexpr int kMaxV = 4;  // float4 per thread (H <= 8192)
      float4 hv[kMaxV], wv[kMaxV];
      const float* wprev = A.layers[l - 1].norm_w;
#pragma unroll
      for (int it = 0; it < kMaxV; ++it) {
        const int j = (it * kFusedThreads + tid) * 4;
        if (j < H) {
          hv[it] = __ldcg(reinterpret_cast<const float4*>(A.h + j));
          wv[it] = __ldg(reinterpret_cast<const float4*>(wprev + j));
        }
      }
      const float r = norm_scale();
#pragma unroll
      for (int it = 0; it < kMaxV; ++it) {
        const int j = (it * kFusedThreads + tid) * 4;
        if (j < H)
          *reinterpret_cast<float4*>(xf + j) =
              make_float4(hv[it].x * r * wv[it].x, hv[it].y * r * wv[it].y, hv[it].z * r * wv[it].z,
                          hv[it].w * r * wv[it].w);
      }
    }
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
    __syncthreads();
    if (tid < nr && !s_abort) {
      float v = rpart[tid * nsl];
      for (int sl = 1; sl < nsl; ++sl) v += rpart[tid * nsl + sl];
      const int row = r0 + tid;
      if (row < E) A.logits[row] = v;
      else A.gamma[0] = 1.f / (1.f + expf(-v));
    }
    if (s_abort) break;
    grid_arrive();  // B1: logits written
    // while the other CTAs finish: quantise x, run the shared expert's gate/up pairs
    stage_x(xf, H, sxq);
    __syncthreads();
    {
      const int ppu = 32 / lprH;  // pairs per warp unit
      const int ps = lane / lprH, lg = lane % lprH;
      for (int u0 = warp * ppu; u0 < nsp; u0 += kFusedWarps * ppu) {
        const int p = u0 + ps;
        bool ok = true;
        if (p < nsp) ok = wait_slot(kMbSPair + p / kPairsPerChunk, par);
        if (!__all_sync(0xffffffffu, ok)) break;
        float g = 0.f, uu = 0.f;
        const int pp = p < nsp ? p : nsp - 1;
        const uint8_t* cp = sc_codes + (size_t)pp * pc_s;
        const uint32_t* sp = reinterpret_cast<const uint32_t*>(sc_sb + (size_t)pp * psb);
        pair_dot_smem<SBITS>(cp, sp, H, sxq, lg, lprH, &g, &uu);
        if (lg == 0 && p < nsp) A.a[(size_t)k * I + s0 + p] = silu_mul(g, uu);
      }
    }
    __syncthreads();
    // publish the shared expert's a-groups this CTA produced
    if (nsp > 0 && tid <= (s1 - 1) / 64 - s0 / 64)
      asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(A.sync + kSyncGroups + k * ngI + s0 / 64 + tid)
                   : "memory");
    if (s_abort || !grid_wait()) break;
    // ------------------------------------------------------------ P2 --
    {
      // routing: every thread keys up to two logits; per-warp top-k, then one
      // warp merges the warps' candidates
      uint64_t key[2];
      bool nan_seen = false;
      float lv[2];
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const int e = tid + i * kFusedThreads;
        lv[i] = e < E ? ldcg_f(A.logits + e) : 0.f;
      }
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const int e = tid + i * kFusedThreads;
        key[i] = 0;
        if (e < E) {
          nan_seen |= isnan(lv[i]);
          slog[e] = lv[i];
          key[i] = route_key(lv[i], e);
        }
      }
      const uint64_t wk = warp_select_keys<2>(key, k);
      if (lane < k) cand[warp * k + lane] = wk;
      nan_seen = __syncthreads_or(nan_seen);
      if (warp == 0) {
        uint64_t kk[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int idx = lane + 32 * i;
          kk[i] = idx < kFusedWarps * k ? cand[idx] : 0;
        }
        const uint64_t win = warp_select_keys<4>(kk, k);
        const int sel = lane < k ? key_index(win) : 0;
        const float val = lane < k ? slog[sel] : 0.f;
        float m = -INFINITY;
        for (int r = 0; r < k; ++r) {
          const float vr = __shfl_sync(0xffffffffu, val, r);
          if (!isnan(vr)) m = fmaxf(m, vr);
        }
        const float pe = (lane < k && !isnan(val)) ? expf(val - m) : 0.f;
        const float z = warp_sum(pe);
        if (lane < k) {
          s_ids[lane] = sel;
          s_p[lane] = z > 0.f ? pe / z : 0.f;
          if (c == 0) {
            A.ids[lane] = sel;
            A.weights[lane] = s_p[lane];
          }
        }
        if (c == 0 && lane == 0 && nan_seen) raise_status(FMOE_STATUS_NAN_LOGIT);
      }
      __syncthreads();
      issue_routed(l);
    }
    {
      const int ppu = 32 / lprH;
      const int ps = lane / lprH, lg = lane % lprH;
      for (int u0 = warp * ppu; u0 < nq; u0 += kFusedWarps * ppu) {
        const int q = u0 + ps;
        bool ok = true;
        if (q < nq) ok = wait_slot(kMbRPair + q / kPairsPerChunk, par);
        if (!__all_sync(0xffffffffu, ok)) break;
        float g = 0.f, uu = 0.f;
        const int qq = q < nq ? q : nq - 1;
        const uint8_t* cp = rc_codes + (size_t)qq * pc_r;
        const uint32_t* sp = reinterpret_cast<const uint32_t*>(rc_sb + (size_t)qq * psb);
        pair_dot_smem<BITS>(cp, sp, H, sxq, lg, lprH, &g, &uu);
        if (lg == 0 && q < nq) A.a[q0 + q] = silu_mul(g, uu);  // a[j][n], q0 + q = j * I + n
      }
    }
    __syncthreads();
    if (s_abort) break;
    // this CTA's SwiGLU outputs are written: publish them, one counter per
    // 64-wide group of a (release: the writes above are visible to whoever
    // acquires the counter)
    if (nq > 0 && tid <= (q1 - 1) / 64 - q0 / 64)
      asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(A.sync + kSyncGroups + q0 / 64 + tid) : "memory");
    // ---------------------------------------------- down products, dataflow --
    // The routed experts' down rows of this CTA's hidden slice, one a-group at
    // a time: each warp owns a contiguous run of a-groups, waits (one round of
    // polls) until the CTAs producing them have published them, loads them
    // (one round trip), then quantises each group and accumulates it, one
    // hidden row per lane.  The warps' sums are added in warp order.
    if (nd > 0) {
      constexpr int kBatch = 6;
      const int u_lo = min(U, warp * per_warp), u_hi = min(U, u_lo + per_warp);
      uint8_t* wst = cons + warp * kWStage;
      const uint4* wxs = reinterpret_cast<const uint4*>(wst);
      float* wdx = reinterpret_cast<float*>(wst + 128);
      float acc0 = 0.f, acc1 = 0.f;
      const int j_first = u_lo < u_hi ? u_lo / ngI : -1;
      int j_cur = -1;
      bool ok = true;
      for (int ub = u_lo; ub < u_hi && ok; ub += kBatch) {
        const int nb = min(kBatch, u_hi - ub);
        // 1. one round of polls for the batch
        bool ready = lane >= nb;
        const long long t0 = clock64();
        while (true) {
          if (!ready) {
            unsigned v;
            asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(A.sync + kSyncGroups + ub + lane)
                         : "memory");
            ready = v >= (unsigned)(l + 1) * s_prod[ub + lane];
          }
          if (__all_sync(0xffffffffu, ready)) break;
          if (clock64() - t0 > kWaitCycles) {
            if (lane == 0) {
              s_abort = 1;
              raise_status(FMOE_STATUS_WAIT_TIMEOUT);
            }
            ok = false;
            break;
          }
        }
        if (!ok) break;
        // 2. one round of loads: lane holds inputs 2 lane, 2 lane + 1 of each group
        float2 av[kBatch];
#pragma unroll
        for (int t = 0; t < kBatch; ++t)
          if (t < nb) {
            const int u = ub + t;
            av[t] = __ldcg(reinterpret_cast<const float2*>(A.a + (size_t)(u / ngI) * I + (u % ngI) * 64) + lane);
          }
        // 3. quantise and accumulate each group
#pragma unroll 1
        for (int t = 0; t < nb; ++t) {
          const int u = ub + t, j = u / ngI, g = u % ngI;
          if (j != j_cur) {
            if (j_cur >= 0) {  // flush the previous expert's sums
              float* wy = cons_wy + (warp * 2 + (j_cur == j_first ? 0 : 1)) * kMaxSliceRows;
              wy[lane] = acc0;
              wy[lane + 32] = acc1;
              acc0 = acc1 = 0.f;
            }
            ok = wait_slot(j == k ? kMbSDown : kMbRDown + j, par);
            if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
            j_cur = j;
          }
          // group max of |a| in one redux (the bits of a non-negative float order as integers)
          const float m = __uint_as_float(
              __reduce_max_sync(0xffffffffu, __float_as_uint(fmaxf(fabsf(av[t].x), fabsf(av[t].y)))));
          const float inv = m > 0.f ? 32767.f / m : 0.f;
          const float delta = m * (1.f / 32767.f);
          int qa = __float2int_rn(av[t].x * inv), qb = __float2int_rn(av[t].y * inv);
          qa = qa > 32767 ? 32767 : (qa < -32767 ? -32767 : qa);
          qb = qb > 32767 ? 32767 : (qb < -32767 ? -32767 : qb);
          const int isum = __reduce_add_sync(0xffffffffu, qa + qb);
          __syncwarp();  // the previous group's staged values have been read
          reinterpret_cast<uint32_t*>(wst)[lane] = (uint32_t)(qa & 0xFFFF) | ((uint32_t)qb << 16);
          if (lane == 0) {
            wdx[0] = delta;
            wdx[1] = delta * (float)isum;
          }
          __syncwarp();
          uint4 xv[8];
#pragma unroll
          for (int q = 0; q < 8; ++q) xv[q] = wxs[q];
          const float dl = wdx[0], xsm = wdx[1];
          const bool shd = j == k;
          const uint8_t* base = shd ? sd_codes : rd_base + (size_t)j * rd_stride;
          const uint32_t drow = shd ? prow_s : prow_r;
          const uint32_t* sbb = shd ? sd_sb : reinterpret_cast<const uint32_t*>(base + rd_sb_off);
#pragma unroll 1
          for (int half = 0; half < 2; ++half) {
            const int rr = lane + 32 * half;
            if (rr >= nd) break;
            const uint8_t* cp = base + (size_t)rr * drow;
            const int A32 = shd ? group_dot<SBITS>(lds_group<SBITS>(cp, ngI, g), xv)
                                : group_dot<BITS>(lds_group<BITS>(cp, ngI, g), xv);
            const float y = group_epilogue(half ? acc1 : acc0, sbb[rr * psbrow + g], A32, dl, xsm);
            if (half) acc1 = y;
            else acc0 = y;
          }
        }
      }
      if (ok && j_cur >= 0) {
        float* wy = cons_wy + (warp * 2 + (j_cur == j_first ? 0 : 1)) * kMaxSliceRows;
        wy[lane] = acc0;
        wy[lane + 32] = acc1;
      }
    }
    __syncthreads();
    if (s_abort) break;
    // the routed down rows are consumed and the a-groups loaded: the next
    // layer's router rows and shared pairs can stream now
    if (l + 1 < A.n_layers) issue_p1(l + 1);
    // y of each expert for this slice: the warps' sums in warp order
    for (int idx = tid; idx < (k + 1) * nd; idx += kFusedThreads) {
      const int j = idx / nd, rr = idx - j * nd;
      float v = 0.f;
      for (int w = 0; w < kFusedWarps; ++w) {
        const int lo = w * per_warp;
        if (lo >= U) break;
        const int jf = lo / ngI, jl = (min(U, lo + per_warp) - 1) / ngI;
        if (jf == j) v += cons_wy[(w * 2) * kMaxSliceRows + rr];
        else if (jl == j) v += cons_wy[(w * 2 + 1) * kMaxSliceRows + rr];
      }
      ypart[j * nd + rr] = v;
    }
    __syncthreads();
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
    grid_arrive();  // B3: h' and the partial sums written
    // the shared down rows are consumed: the next layer's can stream now
    if (l + 1 < A.n_layers) issue_sdown(l + 1);
    if (!grid_wait()) break;
  }

  if (!s_abort) {
    // epilogue: xn' of the last layer for this CTA's rows
    const float r = norm_scale();
    const float* w = A.layers[A.n_layers - 1].norm_w;
    for (int i = i0 + tid; i < i1; i += kFusedThreads) A.xn[i] = ldcg_f(A.h + i) * r * w[i];
    __syncthreads();
    if (tid == 0) {
      __threadfence();
      const unsigned prev = atomicAdd(&A.sync[1], 1u);
      if (prev == (unsigned)nC - 1) {  // every CTA is past its last barrier and wait
        for (int i = 0; i < kSyncGroups + (k + 1) * ngI; ++i) A.sync[i] = 0;
        __threadfence();
      }
    }
  } else if (lane == 0) {
    // drain: wait (bounded) for this issuer's own copies still in flight
    for (int p = 0; p < 2; ++p)
      for (int s2 = 0; s2 < kMbCount; ++s2)
        if (armed[p][s2 >> 5] & (1u << (s2 & 31))) (void)mbar_wait(&mbar[s2], (uint32_t)p);
  }
}

// Host-side plan: shared-memory layout for n_ctas CTAs; false if it does not fit.
inline bool fused_plan(int H, int I, int E, int k, int bits, int sbits, int n_ctas, size_t max_smem,
                       FusedPlan* out) {
  // every per-CTA block moved by cp.async.bulk and every 16-byte shared load
  // must be 16-byte aligned: a down row's scale-bias words (I/64 * 4 bytes)
  // and a pair's (2 * H/64 * 4 bytes) must come in multiples of 16 bytes
  if ((I / 64) % 4 != 0 || (H / 64) % 2 != 0) return false;
  if (E > 2 * kFusedThreads || k > kFusedMaxK) return false;
  auto cdiv = [](long long a, long long b) { return (a + b - 1) / b; };
  const long long nr = cdiv(E + 1, n_ctas), nsp = cdiv(I, n_ctas), nq = cdiv((long long)k * I, n_ctas),
                  nd = cdiv(H, n_ctas);
  if (nr > kFusedMaxRouterRows || nsp > kFusedMaxSharedPairs || nq > kFusedMaxRoutedPairs) return false;
  const RecordLayout LR = record_layout(bits, H, I), LS = record_layout(sbits, H, I);
  const int ngH = H / 64, ngI = I / 64;
  const long long psb = 2LL * ngH * 4;
  const long long pair_r = 2 * (long long)LR.gu_row_bytes + psb;
  const long long pair_s = 2 * (long long)LS.gu_row_bytes + psb;
  const long long sa = ((long long)staged_x_bytes(I) + 15) & ~15LL;
  auto al = [](long long v) { return (v + 127) & ~127LL; };
  if (nd > kMaxSliceRows || (long long)(k + 1) * ngI > kMaxGroupCounters) return false;
  const long long a_p1 = nr * H * 4 + nsp * pair_s;
  const long long a_p2 = nq * pair_r;
  const long long cons_off = (a_p1 + 127) & ~127LL;
  const long long cons_bytes = (long long)kFusedWarps * kWStage + (long long)kFusedWarps * 2 * kMaxSliceRows * 4;
  const long long regA = a_p2 > cons_off + cons_bytes ? a_p2 : cons_off + cons_bytes;
  // padded down-row boxes (tensor copies of nd rows, each kRowPadWords wider than a row)
  const long long dw_r = (long long)LR.down_row_bytes / 4, dw_s = (long long)LS.down_row_bytes / 4;
  if (dw_r + kRowPadWords > 256 || dw_s + kRowPadWords > 256 || ngI + kRowPadWords > 256 || nd > 256) return false;
  const long long c_r = al(nd * (dw_r + kRowPadWords) * 4), c_s = al(nd * (dw_s + kRowPadWords) * 4);
  const long long sbb = al(nd * (ngI + kRowPadWords) * 4);
  const long long sdown = c_s + sbb;
  const long long rstride = c_r + sbb;
  const long long rdown = k * rstride;
  const long long xq = (long long)staged_x_bytes(H);
  FusedPlan p;
  long long o = 0;
  p.region_a = (uint32_t)o;
  p.cons = (uint32_t)(o + cons_off);
  o = al(o + regA);
  p.region_b = (uint32_t)o;
  p.nd_box = (uint32_t)nd;
  p.sd_codes = (uint32_t)o;
  p.sd_sb = (uint32_t)(o + c_s);
  p.rd_slot = (uint32_t)(o + sdown);
  p.rd_stride = (uint32_t)rstride;
  p.rd_sb = (uint32_t)c_r;
  const long long xf_bytes = (long long)H * 4;
  if (rdown >= xf_bytes) {
    p.xf = (uint32_t)(o + sdown);  // aliases the routed down rows (P1 only)
    o = al(o + sdown + rdown);
  } else {
    o = al(o + sdown + rdown);
    p.xf = (uint32_t)o;
    o = al(o + xf_bytes);
  }
  p.xq = (uint32_t)o;
  o = al(o + xq);
  p.logit = (uint32_t)o;
  o = al(o + (long long)E * 4);
  p.cand = (uint32_t)o;
  o = al(o + 2LL * kFusedWarps * kFusedMaxK * 4);
  p.ypart = (uint32_t)o;
  o = al(o + (k + 1) * nd * 4);
  p.rpart = (uint32_t)o;
  o = al(o + nr * (H >= 512 ? H / 512 : 1) * 4);
  p.prod = (uint32_t)o;
  o = al(o + 4LL * (k + 1) * ngI);
  p.mbar = (uint32_t)o;
  o = al(o + kMbCount * 8);
  p.total = (uint32_t)o;
  if ((size_t)o > max_smem) return false;
  *out = p;
  return true;
}

}  // namespace fmoe
