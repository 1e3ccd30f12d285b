// fmoe_fused.cuh -- one persistent kernel for a stack of MoE layers, batch 1.
//
// One CTA per SM, launched cooperatively so that every CTA is resident and
// grid-wide barriers are safe.  The experts' intermediate dimension is cut
// into column blocks of w = 8 (4-bit) or 16 (2-bit) units: a block is w
// gate/up row pairs plus the matching w columns of the down matrix, one
// 32-bit word of codes per hidden row (the packed record stores the down
// matrix column block by column block).  A CTA that owns a block computes
// its w SwiGLU outputs and, from them, the block's contribution to all H
// outputs of the down product -- no other CTA's data is needed until the
// partial outputs are summed.  Per layer:
//   A  xn = h' r w (every CTA, whole vector) and this CTA's router rows
//      (fp32, the shared gate vector as row E) -> logits
//   -- barrier B1 (all logits written); while it completes, the CTA runs
//      its block of the shared expert
//   D  every CTA takes the top-k of all logits itself and fetches its run of
//      routed blocks (each block's bytes are contiguous in the record)
//   E  routed blocks: gate/up -> a -> weighted down contribution, held in
//      registers (each thread owns H / 512 hidden rows)
//   F  the CTA's partial output sum_j p_j y_j + gamma y_s for all H rows ->
//      global; barrier B2
//   G  each CTA sums the partials of its slice of rows in a fixed order,
//      adds the residual -> h', and its part of sum(h'^2); barrier B3
// Source pages: "What is Flash-MoE?" (a2a-mcp.org), sections
// "Understanding Mixture-of-Experts", "2. FMA-optimised dequantisation
// kernels" and "3. Hand-tuned Metal compute shaders" (deferred command-buffer
// submission there plays the role the persistent kernel plays here: no host
// round trip between the steps or between layers).
//
// Weight bytes move global -> shared with cp.async.bulk into three block
// slots and two scale-bias entries (mbarrier completion).  At the top-k the
// CTA requests its first three routed blocks and asks the L2 to prefetch
// the rest and the next layer's router rows and shared block, so HBM keeps
// streaming while the slots turn over.  Every weight byte is read from HBM
// once per layer.  Every wait (mbarrier or grid barrier) is bounded: on
// expiry the CTA sets FMOE_STATUS_WAIT_TIMEOUT, waits (bounded) for its own
// copies in flight, and returns.
#pragma once

#include <cstdint>

#include "fmoe.h"
#include "fmoe_device.cuh"
#include "fmoe_layout.h"

namespace fmoe {

constexpr int kFusedThreads = 512;
constexpr int kFusedWarps = kFusedThreads / 32;
constexpr int kFusedMaxLayers = 32;
constexpr int kFusedMaxK = 8;
constexpr int kFusedMaxCtas = 160;      // partial outputs in the workspace: [kFusedMaxCtas][H]
constexpr int kFusedMaxRouterRows = 4;  // router rows (E experts + the shared gate) per CTA
constexpr int kFusedRowsPerThread = 8;  // hidden rows per thread in the down products: H <= 4096
constexpr int kFusedMaxRouted = 16;     // routed blocks per CTA
constexpr int kSlots = 3;
constexpr int kFirstWave = 2;  // routed blocks requested at the top-k; the rest after they land
constexpr int kSbEntries = 2;
constexpr int kMbSb = kSlots;  // mbarriers: the slots, then the scale-bias entries
constexpr int kMbCount = kSlots + kSbEntries;
constexpr long long kWaitCycles = 4000000000LL;  // ~2 s at 2 GHz

struct FusedLayer {
  const uint8_t* experts;
  const uint8_t* shared;
  const float* w_router;
  const float* w_sg;
  const float* norm_w;
};

// Shared-memory plan (byte offsets), computed on the host.  A slot holds
// one column block: [gate/up codes, 8 H bytes][down codes, 4 H bytes]
// [gate/up scale-bias, w H / 8 bytes]; an entry holds the down scale-bias
// words of one 64-group of one expert (4 H bytes).
struct FusedPlan {
  uint32_t slot[kSlots];
  uint32_t sbe[kSbEntries];
  uint32_t xs;     // staged int16 x of the layer
  uint32_t logit;  // fp32 [E]
  uint32_t cand;   // top-k candidates: u64 [warps][k]
  uint32_t red;    // fp32 [kFusedThreads]: partial sums of the row reduction
  uint32_t mbar;
  uint32_t total;
};

struct FusedArgs {
  FusedLayer layers[kFusedMaxLayers];
  int n_layers;
  int H, I, E, k;
  float eps;
  float* h;
  float* xn;
  float* logits;
  int32_t* ids;
  float* weights;
  float* gamma;
  float* a;          // [(k+1)][I], shared expert last
  // exchange words between CTAs: (epoch << 32) | fp32 bits, written and read
  // as single 64-bit accesses, so a reader that sees the epoch it waits for
  // holds the value that came with it (no separate flag or barrier)
  uint64_t* x_logit;  // [E + 1]: router logits, then sigmoid(w_sg . xn)
  uint64_t* x_part;   // [gridDim.x][H]: partial outputs
  float* ss_part;     // [gridDim.x]: partial sums of h'^2 (behind the grid barrier)
  unsigned* sync;     // [0] grid-barrier arrivals, [1] exits, [2] epoch of the last launch
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

// Asks the L2 to fetch [p, p + bytes) from HBM (no shared memory involved).
__device__ __forceinline__ void prefetch_l2(const void* p, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

// One try_wait; the thread may be suspended (up to the hint, 20 us) until the
// phase completes, so waiting warps do not compete for issue slots.
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

__device__ __forceinline__ float4 as_float4(uint4 v) {
  return make_float4(__uint_as_float(v.x), __uint_as_float(v.y), __uint_as_float(v.z), __uint_as_float(v.w));
}

__device__ __forceinline__ uint64_t ld_relaxed64(const uint64_t* p) {
  uint64_t v;
  asm volatile("ld.relaxed.gpu.global.b64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void st_relaxed64(uint64_t* p, uint64_t v) {
  asm volatile("st.relaxed.gpu.global.b64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

__device__ __forceinline__ uint64_t x_word(uint32_t epoch, float v) {
  return ((uint64_t)epoch << 32) | __float_as_uint(v);
}

__device__ __forceinline__ bool x_ready(uint64_t w, uint32_t epoch) { return (uint32_t)(w >> 32) == epoch; }

// Re-reads *p until it carries `epoch` (bounded); false on expiry.
__device__ __forceinline__ bool x_spin(const uint64_t* p, uint32_t epoch, uint64_t* w) {
  if (x_ready(*w, epoch)) return true;
  const long long t0 = clock64();
  while (clock64() - t0 < kWaitCycles) {
    *w = ld_relaxed64(p);
    if (x_ready(*w, epoch)) return true;
  }
  return false;
}

// N exchange words at p(i) (those with valid(i)): re-reads, all in one round
// trip per pass, the ones that do not yet carry `epoch` (bounded).
// While words are missing, only the first missing one is polled; once it
// has arrived, the others are re-read together.
template <int N, class Addr, class Valid>
__device__ __forceinline__ bool x_spin_all(uint64_t (&w)[N], uint32_t epoch, Addr p, Valid valid) {
  const long long t0 = clock64();
  while (true) {
    int miss = -1;
#pragma unroll
    for (int i = N - 1; i >= 0; --i)
      if (valid(i) && !x_ready(w[i], epoch)) miss = i;
    if (miss < 0) return true;
    if (clock64() - t0 > kWaitCycles) return false;
    uint64_t v = ld_relaxed64(p(miss));
    while (!x_ready(v, epoch)) {
      if (clock64() - t0 > kWaitCycles) return false;
      v = ld_relaxed64(p(miss));
    }
#pragma unroll
    for (int i = 0; i < N; ++i)
      if (valid(i) && !x_ready(w[i], epoch)) w[i] = i == miss ? v : ld_relaxed64(p(i));
  }
}

// [lo, hi) share of `total` items for part `c` of `n`
__host__ __device__ __forceinline__ void share(int total, int c, int n, int* lo, int* hi) {
  *lo = (int)(((long long)total * c) / n);
  *hi = (int)(((long long)total * (c + 1)) / n);
}

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

// Geometry of a column block of an expert with BITS-bit codes.
template <int BITS>
struct BlockGeo {
  static constexpr int kW = 32 / BITS;             // intermediate units per block
  static constexpr int kPerGroup = 64 / kW;        // blocks per 64-group
  static constexpr int kTpp = kFusedThreads / kW;  // threads per gate/up row pair
  __host__ __device__ static uint32_t gu_codes(int H) { return 8u * (uint32_t)H; }
  __host__ __device__ static uint32_t dn_codes(int H) { return 4u * (uint32_t)H; }
  __host__ __device__ static uint32_t gu_sb(int H) { return (uint32_t)kW * 2u * (uint32_t)(H / 64) * 4u; }
};

// Block state shared by the threads of a CTA.
struct BlockShared {
  float gu[kFusedWarps][4][2];  // per warp, per pair of the thread set: partial gate / up sums
};

// The staged inputs of one 64-group, kept in registers for the whole layer:
// thread t serves group t % 64 of every gate/up row it touches.
struct XGroup {
  uint4 xv[8];
  float delta, xsum;
};

__device__ __forceinline__ XGroup load_xgroup(const StagedX& sx, int ngH) {
  XGroup x;
  const int g = threadIdx.x & 63;
  if (g < ngH) {
    lds_xv(sx, ngH, g, x.xv);
    x.delta = sx.delta[g];
    x.xsum = sx.xsum[g];
  } else {
#pragma unroll
    for (int u = 0; u < 8; ++u) x.xv[u] = make_uint4(0u, 0u, 0u, 0u);
    x.delta = x.xsum = 0.f;
  }
  return x;
}

// One or two column blocks (NB), block n held in slots[n]: gate/up of
// their w row pairs each, SwiGLU, each block's w outputs rounded to 16-bit
// fixed point with its own step, then the blocks' down columns for every
// hidden row this thread owns, block n scaled by weight[n], added to y.
// Thread t works on group t % 64 of pairs t / 64 + 8 i (pair p = block
// p / w, row pair p % w of it); every warp then forms all the blocks'
// outputs itself from the per-warp sums, so one block-wide barrier separates
// the two halves.  a_out[n] (global) receives block n's w SwiGLU outputs.
// The slots may be refilled after the closing barrier.
template <int B, int NB>
__device__ __forceinline__ void run_blocks(const uint8_t* const (&slots)[2], const uint32_t* const (&dsb)[2], int H,
                                           const XGroup& xg, const float (&weight)[2], float* const (&a_out)[2],
                                           BlockShared& bs, float (&y)[kFusedRowsPerThread]) {
  using G = BlockGeo<B>;
  constexpr int kW = G::kW;
  constexpr int kNP = NB * kW;   // row pairs: 8, 16 or 32
  constexpr int kPP = kNP / 8;   // pairs per thread
  static_assert(kNP <= 32 && kPP <= 4, "one warp forms all outputs");
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int ngH = H / 64;
  const int g = tid & 63, ps = tid >> 6;
  {
    const uint32_t rb = (uint32_t)H * B / 8;
    float gs[kPP], us[kPP];
#pragma unroll
    for (int pp = 0; pp < kPP; ++pp) {
      // pair ps + 8 pp: block (8 pp) / w and row pair ps + 8 (pp % (w / 8)) of it (ps < 8)
      constexpr int kSub = kW / 8;
      const int n = (8 * pp) / kW, pl = ps + 8 * (pp % kSub);
      gs[pp] = us[pp] = 0.f;
      if (g < ngH) {
        const uint8_t* rg = slots[n] + (size_t)(2 * pl) * rb;
        const uint32_t* sbg = reinterpret_cast<const uint32_t*>(slots[n] + G::gu_codes(H) + G::dn_codes(H)) +
                              2 * pl * ngH;
        const GroupCodes<B> cg = lds_group<B>(rg, ngH, g);
        const GroupCodes<B> cu = lds_group<B>(rg + rb, ngH, g);
        gs[pp] = group_epilogue(0.f, sbg[g], group_dot<B>(cg, xg.xv), xg.delta, xg.xsum);
        us[pp] = group_epilogue(0.f, sbg[ngH + g], group_dot<B>(cu, xg.xv), xg.delta, xg.xsum);
      }
    }
#pragma unroll
    for (int pp = 0; pp < kPP; ++pp) {
      const float gsum = warp_sum(gs[pp]), usum = warp_sum(us[pp]);
      if (lane == 0) {
        bs.gu[warp][pp][0] = gsum;
        bs.gu[warp][pp][1] = usum;
      }
    }
  }
  __syncthreads();
  // every warp: SwiGLU of all pairs (lane l < kNP: pair l, whose sums sit in
  // warps 2 (l % 8), 2 (l % 8) + 1, slot l / 8), one fixed-point step per
  // block, the int16 pairs of every block spread to all lanes
  uint32_t xw[NB][8];
  float p1[NB], p2[NB];
  {
    float a = 0.f;
    if (lane < kNP) {
      const int pw = 2 * (lane & 7), pp = lane >> 3;
      a = silu_mul(bs.gu[pw][pp][0] + bs.gu[pw + 1][pp][0], bs.gu[pw][pp][1] + bs.gu[pw + 1][pp][1]);
      if (warp == 0) (NB == 2 && lane >= kW ? a_out[NB - 1] : a_out[0])[lane % kW] = a;
    }
    const int mine = lane / kW;  // this lane's block (>= NB: none)
    float delta_m = 0.f;
#pragma unroll
    for (int n = 0; n < NB; ++n) {
      const float m = __uint_as_float(__reduce_max_sync(0xffffffffu, mine == n ? __float_as_uint(fabsf(a)) : 0u));
      const float delta = m * (1.f / 32767.f);
      if (mine == n) delta_m = m > 0.f ? 32767.f / m : 0.f;
      p1[n] = weight[n] * delta;
    }
    int q = __float2int_rn(a * delta_m);
    q = q > 32767 ? 32767 : (q < -32767 ? -32767 : q);
#pragma unroll
    for (int n = 0; n < NB; ++n) p2[n] = p1[n] * (float)__reduce_add_sync(0xffffffffu, mine == n ? q : 0);
    const int q_hi = __shfl_down_sync(0xffffffffu, q, 1);
    const uint32_t word = (uint32_t)(q & 0xFFFF) | ((uint32_t)q_hi << 16);
#pragma unroll
    for (int n = 0; n < NB; ++n) {
#pragma unroll
      for (int i = 0; i < 8; ++i) xw[n][i] = i < kW / 2 ? __shfl_sync(0xffffffffu, word, n * kW + 2 * i) : 0u;
    }
  }
  {
    const uint32_t* dc[NB];
#pragma unroll
    for (int n = 0; n < NB; ++n) dc[n] = reinterpret_cast<const uint32_t*>(slots[n] + G::gu_codes(H));
#pragma unroll
    for (int m = 0; m < kFusedRowsPerThread; ++m) {
      const int i = tid + m * kFusedThreads;
      if (i < H) {
        float v = y[m];
#pragma unroll
        for (int n = 0; n < NB; ++n) {
          const uint32_t w = dc[n][i], sbw = dsb[n][i];
          const int acc = B == 4 ? word_dot4(w, make_uint4(xw[n][0], xw[n][1], xw[n][2], xw[n][3]))
                                 : word_dot2(w, make_uint4(xw[n][0], xw[n][1], xw[n][2], xw[n][3]),
                                             make_uint4(xw[n][4], xw[n][5], xw[n][6], xw[n][7]));
          const float sc = __uint_as_float(sbw << 16), bi = __uint_as_float(sbw & 0xFFFF0000u);
          v = fmaf(sc, p1[n] * (float)acc, fmaf(bi, p2[n], v));
        }
        y[m] = v;
      }
    }
  }
  __syncthreads();
}

// ------------------------------------------------------------ the kernel --
template <int BITS, int SBITS>  // routed and shared code widths
__global__ void __launch_bounds__(kFusedThreads, 1) fused_stack_kernel(const __grid_constant__ FusedArgs A) {
  using GR = BlockGeo<BITS>;
  using GS = BlockGeo<SBITS>;
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ int s_ids[kFusedMaxK];
  __shared__ float s_p[kFusedMaxK];
  __shared__ float s_gamma;
  __shared__ float s_rp[kFusedWarps][kFusedMaxRouterRows];
  __shared__ float s_red[kFusedWarps];
  __shared__ BlockShared s_blk;

  const int c = blockIdx.x, nC = gridDim.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int H = A.H, I = A.I, E = A.E, k = A.k;
  const int ngH = H / 64;
  const FusedPlan& P = A.plan;
  uint64_t* mbar = reinterpret_cast<uint64_t*>(smem + P.mbar);
  const StagedX sx = staged_x_at(smem + P.xs, H);
  float* slog = reinterpret_cast<float*>(smem + P.logit);
  uint64_t* cand = reinterpret_cast<uint64_t*>(smem + P.cand);
  float* sred = reinterpret_cast<float*>(smem + P.red);

  // static work of this CTA
  const int nr = c <= E ? (E - c) / nC + 1 : 0;  // router rows c, c + nC, ... <= E (row E: shared gate)
  const int NBr = I * BITS / 32, NBs = I * SBITS / 32;
  const bool has_shared = c < NBs;  // shared block c
  int q0, q1, i0, i1;
  share(k * NBr, c, nC, &q0, &q1);  // routed blocks, expert-major
  share(H, c, nC, &i0, &i1);        // hidden rows of the final sums
  const int nq = q1 - q0, nd = i1 - i0;
  const RecordLayout LR = record_layout(BITS, H, I);
  const RecordLayout LS = record_layout(SBITS, H, I);
  const bool xthr = tid * 8 < H;  // this thread holds inputs 8 tid .. 8 tid + 7

  if (tid == 0) {
    for (int i = 0; i < kMbCount; ++i) mbar_init(&mbar[i], 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();

  uint32_t phase = 0;  // per mbarrier: parity of its next completion (same in every thread)
  uint32_t armed = 0;  // lane 0 of an issuing warp: its mbarriers with copies in flight

  // ---- copies (lane 0 of one warp per mbarrier: slot s <- warp s, entry e
  // <- warp kSlots + e, so each issuer drains its own copies on abort) ----
  auto arm = [&](int mb, uint32_t bytes) {
    mbar_expect_tx(&mbar[mb], bytes);
    armed |= 1u << mb;
  };
  // column block nb of the record `rec` into slot s
  auto issue_block = [&](int s, const uint8_t* rec, const RecordLayout& L, int nb, uint32_t gu_sb_bytes) {
    uint8_t* dst = smem + P.slot[s];
    const uint32_t gub = 8u * (uint32_t)H, dnb = 4u * (uint32_t)H;
    arm(s, gub + dnb + gu_sb_bytes);
    bulk_g2s(dst, rec + L.gu_codes + (size_t)nb * gub, gub, &mbar[s]);
    bulk_g2s(dst + gub, rec + L.down_codes + (size_t)nb * dnb, dnb, &mbar[s]);
    bulk_g2s(dst + gub + dnb, rec + L.gu_sb + (size_t)nb * gu_sb_bytes, gu_sb_bytes, &mbar[s]);
  };
  auto prefetch_block = [&](const uint8_t* rec, const RecordLayout& L, int nb, uint32_t gu_sb_bytes) {
    const uint32_t gub = 8u * (uint32_t)H, dnb = 4u * (uint32_t)H;
    prefetch_l2(rec + L.gu_codes + (size_t)nb * gub, gub);
    prefetch_l2(rec + L.down_codes + (size_t)nb * dnb, dnb);
    prefetch_l2(rec + L.gu_sb + (size_t)nb * gu_sb_bytes, gu_sb_bytes);
  };
  // down scale-bias words of 64-group g of a record into entry e
  auto issue_sb = [&](int e, const uint8_t* rec, const RecordLayout& L, int g) {
    arm(kMbSb + e, 4u * (uint32_t)H);
    bulk_g2s(smem + P.sbe[e], rec + L.down_sb + (size_t)g * H * 4, 4u * (uint32_t)H, &mbar[kMbSb + e]);
  };
  // layer l's shared block -> slot 1 (warp 1), its scale-bias -> entry 0 (warp kSlots); lane 0 only
  auto issue_shared = [&](int l) {
    if (!has_shared) return;
    const uint8_t* rec = A.layers[l].shared;
    if (warp == 1) {
      fence_proxy_async();
      issue_block(1, rec, LS, c, GS::gu_sb(H));
    } else if (warp == kSlots) {
      fence_proxy_async();
      issue_sb(0, rec, LS, c / GS::kPerGroup);
    }
  };

  // L2 prefetch of layer l's router rows and shared block (any one thread)
  auto prefetch_next = [&](int l) {
    const FusedLayer& NX = A.layers[l];
    for (int m = 0; m < nr; ++m) {
      const int row = c + m * nC;
      prefetch_l2(row < E ? NX.w_router + (size_t)row * H : NX.w_sg, 4u * (uint32_t)H);
    }
    if (has_shared) {
      prefetch_block(NX.shared, LS, c, GS::gu_sb(H));
      prefetch_l2(NX.shared + LS.down_sb + (size_t)(c / GS::kPerGroup) * H * 4, 4u * (uint32_t)H);
    }
  };

  // ---- waits (all threads; the outcome is agreed block-wide) ----
  auto wait_mb = [&](int mb) -> bool {
    const bool ok = mbar_wait(&mbar[mb], (phase >> mb) & 1u);
    phase ^= 1u << mb;
    if (lane == 0 && ok) armed &= ~(1u << mb);
    if (__syncthreads_and(ok)) return true;
    if (tid == 0) raise_status(FMOE_STATUS_WAIT_TIMEOUT);
    return false;
  };

  // block-wide agreement after a round of exchange reads
  auto x_agree = [&](bool ok) -> bool {
    if (__syncthreads_and(ok)) return true;
    if (tid == 0) raise_status(FMOE_STATUS_WAIT_TIMEOUT);
    return false;
  };
  // grid barrier after h' (every CTA needs all of it): arrive once this
  // CTA's rows are written, wait at the start of the next layer
  // (release/acquire on one counter, bounded spin)
  unsigned bar_target = 0;
  auto grid_arrive = [&]() {
    __syncthreads();
    bar_target += (unsigned)nC;
    if (tid == 0) asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(A.sync) : "memory");
  };
  auto grid_wait = [&]() -> bool {
    bool ok = true;
    if (tid == 0) {
      ok = false;
      const long long t0 = clock64();
      while (true) {
        unsigned v;
        asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(A.sync) : "memory");
        if (v >= bar_target) { ok = true; break; }
        if (clock64() - t0 > kWaitCycles) break;
      }
    }
    return x_agree(ok);
  };
  // r = (sum of the CTAs' partial sums of h'^2 / H + eps)^(-1/2), summed in
  // the same order in every CTA (after the grid barrier)
  auto norm_scale = [&]() -> float {
    float v = tid < nC ? ldcg_f(A.ss_part + tid) : 0.f;
    v = warp_sum(v);
    if (lane == 0) s_red[warp] = v;
    __syncthreads();
    float t = 0.f;
#pragma unroll
    for (int wi = 0; wi < kFusedWarps; ++wi) t += s_red[wi];
    __syncthreads();
    return 1.f / sqrtf(t / (float)H + A.eps);
  };

  const uint32_t base = __ldcg(A.sync + 2);  // epochs of this launch: base + 2 l + 1, base + 2 l + 2
  if (lane == 0 && A.n_layers > 0) issue_shared(0);

  float yr[kFusedRowsPerThread], ys[kFusedRowsPerThread];
  bool aborted = false;
  for (int l = 0; l < A.n_layers; ++l) {
    const FusedLayer& LY = A.layers[l];
#pragma unroll
    for (int m = 0; m < kFusedRowsPerThread; ++m) yr[m] = ys[m] = 0.f;
    // ------------------------------------------------------------- A --
    // router rows (requested before anything they do not depend on)
    float4 wr[kFusedMaxRouterRows][2];
#pragma unroll
    for (int m = 0; m < kFusedMaxRouterRows; ++m) {
      const int row = c + m * nC;
      if (m < nr && xthr) {
        const float* src = (row < E ? LY.w_router + (size_t)row * H : LY.w_sg) + tid * 8;
        wr[m][0] = as_float4(ld_stream(src));
        wr[m][1] = as_float4(ld_stream(src + 4));
      } else {
        wr[m][0] = wr[m][1] = make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
    float xv[8];
    if (l == 0) {
      float4 v0 = make_float4(0.f, 0.f, 0.f, 0.f), v1 = v0;
      if (xthr) {
        v0 = __ldcg(reinterpret_cast<const float4*>(A.xn + tid * 8));
        v1 = __ldcg(reinterpret_cast<const float4*>(A.xn + tid * 8 + 4));
      }
      xv[0] = v0.x; xv[1] = v0.y; xv[2] = v0.z; xv[3] = v0.w;
      xv[4] = v1.x; xv[5] = v1.y; xv[6] = v1.z; xv[7] = v1.w;
    } else {
      if (!grid_wait()) { aborted = true; break; }  // h' of the previous layer written
      float4 h0 = make_float4(0.f, 0.f, 0.f, 0.f), h1 = h0, w0 = h0, w1 = h0;
      const float* wprev = A.layers[l - 1].norm_w;
      if (xthr) {
        h0 = __ldcg(reinterpret_cast<const float4*>(A.h + tid * 8));
        h1 = __ldcg(reinterpret_cast<const float4*>(A.h + tid * 8 + 4));
        w0 = __ldg(reinterpret_cast<const float4*>(wprev + tid * 8));
        w1 = __ldg(reinterpret_cast<const float4*>(wprev + tid * 8 + 4));
      }
      const float r = norm_scale();
      xv[0] = h0.x * r * w0.x; xv[1] = h0.y * r * w0.y; xv[2] = h0.z * r * w0.z; xv[3] = h0.w * r * w0.w;
      xv[4] = h1.x * r * w1.x; xv[5] = h1.y * r * w1.y; xv[6] = h1.z * r * w1.z; xv[7] = h1.w * r * w1.w;
    }
    const uint32_t e_logit = base + 2u * (uint32_t)l + 1u, e_part = e_logit + 1u;
    // stage x: 8 consecutive threads share one 64-group
    {
      float m = 0.f;
#pragma unroll
      for (int i = 0; i < 8; ++i) m = fmaxf(m, fabsf(xv[i]));
      m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
      m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
      m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 4));
      const float inv = m > 0.f ? 32767.f / m : 0.f;
      const float delta = m * (1.f / 32767.f);
      int q[8], sum = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        int t = __float2int_rn(xv[i] * inv);
        t = t > 32767 ? 32767 : (t < -32767 ? -32767 : t);
        q[i] = t;
        sum += t;
      }
      sum += __shfl_xor_sync(0xffffffffu, sum, 1);
      sum += __shfl_xor_sync(0xffffffffu, sum, 2);
      sum += __shfl_xor_sync(0xffffffffu, sum, 4);
      if (xthr) {
        const int g = tid >> 3, u = tid & 7;
        sx.xs[u * ngH + g] = make_uint4((uint32_t)(q[0] & 0xFFFF) | ((uint32_t)q[1] << 16),
                                        (uint32_t)(q[2] & 0xFFFF) | ((uint32_t)q[3] << 16),
                                        (uint32_t)(q[4] & 0xFFFF) | ((uint32_t)q[5] << 16),
                                        (uint32_t)(q[6] & 0xFFFF) | ((uint32_t)q[7] << 16));
        if (u == 0) {
          sx.delta[g] = delta;
          sx.xsum[g] = delta * (float)sum;
        }
      }
    }
    // router partial dot products, reduced in warp order
#pragma unroll
    for (int m = 0; m < kFusedMaxRouterRows; ++m) {
      float d = wr[m][0].x * xv[0];
      d = fmaf(wr[m][0].y, xv[1], d);
      d = fmaf(wr[m][0].z, xv[2], d);
      d = fmaf(wr[m][0].w, xv[3], d);
      d = fmaf(wr[m][1].x, xv[4], d);
      d = fmaf(wr[m][1].y, xv[5], d);
      d = fmaf(wr[m][1].z, xv[6], d);
      d = fmaf(wr[m][1].w, xv[7], d);
      d = warp_sum(d);
      if (lane == 0) s_rp[warp][m] = d;
    }
    __syncthreads();
    if (tid < nr) {
      float v = 0.f;
      for (int w = 0; w < kFusedWarps; ++w) v += s_rp[w][tid];
      const int row = c + tid * nC;
      if (row < E) A.logits[row] = v;
      else A.gamma[0] = v = 1.f / (1.f + expf(-v));
      st_relaxed64(A.x_logit + row, x_word(e_logit, v));
    }
    const XGroup xg = load_xgroup(sx, ngH);
    // ------------------------------------------------------------- C --
    // while the other CTAs finish: this CTA's block of the shared expert
    if (has_shared) {
      if (!wait_mb(1) || !wait_mb(kMbSb + 0)) { aborted = true; break; }
      const uint8_t* const sl[2] = {smem + P.slot[1], nullptr};
      const uint32_t* const sb[2] = {reinterpret_cast<const uint32_t*>(smem + P.sbe[0]), nullptr};
      const float wt[2] = {1.f, 0.f};
      float* const ao[2] = {A.a + (size_t)k * I + (size_t)c * GS::kW, nullptr};
      run_blocks<SBITS, 1>(sl, sb, H, xg, wt, ao, s_blk, ys);
    }
    // ------------------------------------------------------------- D --
    {
      // routing: every thread keys up to two logits; per-warp top-k, then one
      // warp merges the warps' candidates
      uint64_t key[2];
      bool nan_seen = false;
      float lv[2];
      {
        uint64_t lw[2], gw = 0;
        bool ok = true;
        if (tid == 0) gw = ld_relaxed64(A.x_logit + E);
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          const int e = tid + i * kFusedThreads;
          lw[i] = e < E ? ld_relaxed64(A.x_logit + e) : 0;
        }
        {
          uint64_t all3[3] = {lw[0], lw[1], gw};
          ok = x_spin_all(all3, e_logit, [&](int i) { return A.x_logit + (i < 2 ? tid + i * kFusedThreads : E); },
                          [&](int i) { return i < 2 ? tid + i * kFusedThreads < E : tid == 0; });
          lw[0] = all3[0];
          lw[1] = all3[1];
          gw = all3[2];
        }
#pragma unroll
        for (int i = 0; i < 2; ++i) lv[i] = __uint_as_float((uint32_t)lw[i]);
        if (tid == 0) s_gamma = __uint_as_float((uint32_t)gw);
        if (!x_agree(ok)) { aborted = true; break; }
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
    }
    // requests: the first routed blocks into the slots, the down scale-bias
    // of their (at most two) 64-groups, L2 prefetches of the remaining
    // blocks and of the next layer's router rows and shared block.  A routed
    // block q (= j * NBr + nb) lies in 64-group q / kPerGroup of the
    // concatenated experts.
    // Jobs are spread over the warps' lane 0 so they go out in parallel:
    // block b < kSlots <- warp b, entry e <- warp kSlots + e, L2 prefetch of
    // the blocks b >= kSlots <- the following warps.
    const int key0 = q0 / GR::kPerGroup, key1 = (q1 - 1) / GR::kPerGroup;
    const int ngI = I / 64;
    if (lane == 0) {
      if (warp < kFirstWave) {
        if (warp < nq) {
          const int q = q0 + warp;
          fence_proxy_async();
          issue_block(warp, LY.experts + (size_t)s_ids[q / NBr] * LR.bytes, LR, q % NBr, GR::gu_sb(H));
        }
      } else if (warp >= kSlots && warp < kSlots + kSbEntries) {
        const int e = warp - kSlots;
        if (nq > 0 && (e == 0 || key1 != key0)) {
          const int key = e == 0 ? key0 : key1;
          fence_proxy_async();
          issue_sb(e, LY.experts + (size_t)s_ids[key / ngI] * LR.bytes, LR, key % ngI);
        }
      }
    }
    // the second wave (the other slots, L2 prefetch of the later blocks) goes
    // out once the first wave has landed, so that the first blocks are not
    // slowed by requests for the later ones
    auto second_wave = [&]() {
      if (lane != 0) return;
      if (warp >= kFirstWave && warp < kSlots) {
        if (warp < nq) {
          const int q = q0 + warp;
          fence_proxy_async();
          issue_block(warp, LY.experts + (size_t)s_ids[q / NBr] * LR.bytes, LR, q % NBr, GR::gu_sb(H));
        }
      } else if (warp >= kSlots + kSbEntries) {
        for (int b = kSlots + (warp - kSlots - kSbEntries); b < nq; b += kFusedWarps - kSlots - kSbEntries) {
          const int q = q0 + b;
          prefetch_block(LY.experts + (size_t)s_ids[q / NBr] * LR.bytes, LR, q % NBr, GR::gu_sb(H));
        }
      }
    };
    // ------------------------------------------------------------- E --
    // routed blocks two at a time (block b in slot b % kSlots); a freed slot
    // takes block b + kSlots at once
    {
      unsigned sb_ready = 0;  // bit e: entry e waited for in this layer
      for (int b = 0; b < nq; b += 2) {
        const int nb_round = nq - b >= 2 ? 2 : 1;
        const uint8_t* sl[2] = {nullptr, nullptr};
        const uint32_t* sb[2] = {nullptr, nullptr};
        float wt[2] = {0.f, 0.f};
        float* ao[2] = {nullptr, nullptr};
#pragma unroll
        for (int n = 0; n < 2; ++n) {
          if (n >= nb_round) break;
          const int q = q0 + b + n, j = q / NBr, nbk = q % NBr;
          const int s = (b + n) % kSlots, e = q / GR::kPerGroup == key0 ? 0 : 1;
          if (!wait_mb(s)) { aborted = true; break; }
          if (!(sb_ready & (1u << e))) {
            if (!wait_mb(kMbSb + e)) { aborted = true; break; }
            sb_ready |= 1u << e;
          }
          sl[n] = smem + P.slot[s];
          sb[n] = reinterpret_cast<const uint32_t*>(smem + P.sbe[e]);
          wt[n] = s_p[j];
          ao[n] = A.a + (size_t)j * I + (size_t)nbk * GR::kW;
        }
        if (aborted) break;
        if (b == 0) second_wave();
        const uint8_t* const slc[2] = {sl[0], sl[1]};
        const uint32_t* const sbc[2] = {sb[0], sb[1]};
        const float wtc[2] = {wt[0], wt[1]};
        float* const aoc[2] = {ao[0], ao[1]};
        if (nb_round == 2) run_blocks<BITS, 2>(slc, sbc, H, xg, wtc, aoc, s_blk, yr);
        else run_blocks<BITS, 1>(slc, sbc, H, xg, wtc, aoc, s_blk, yr);
        // the freed slots take their next blocks
#pragma unroll
        for (int n = 0; n < 2; ++n) {
          if (n >= nb_round) break;
          const int bb = b + n, s = bb % kSlots;
          if (warp == s && lane == 0 && bb + kSlots < nq) {
            const int q2 = q0 + bb + kSlots;
            fence_proxy_async();
            issue_block(s, LY.experts + (size_t)s_ids[q2 / NBr] * LR.bytes, LR, q2 % NBr, GR::gu_sb(H));
          }
        }
        // once the first round is done, the next layer's router rows and
        // shared block may compete for HBM
        if (b == 0 && warp == kFusedWarps - 1 && lane == 0 && l + 1 < A.n_layers) prefetch_next(l + 1);
      }
      if (aborted) break;
      if (nq == 0 && warp == kFusedWarps - 1 && lane == 0 && l + 1 < A.n_layers) prefetch_next(l + 1);
    }
    // every slot and entry is consumed: the next layer's shared block can come in
    if (lane == 0 && l + 1 < A.n_layers) issue_shared(l + 1);
    // ------------------------------------------------------------- F --
    {
      const float gm = s_gamma;
      uint64_t* part = A.x_part + (size_t)c * H;
#pragma unroll
      for (int m = 0; m < kFusedRowsPerThread; ++m) {
        const int i = tid + m * kFusedThreads;
        if (i < H) st_relaxed64(part + i, x_word(e_part, fmaf(gm, ys[m], yr[m])));
      }
    }
    // ------------------------------------------------------------- G --
    {
      // rows i0 + r, r < nd: ngr threads per row each sum every ngr-th CTA's
      // partial; then one thread per row adds those sums in order
      const int ngr = nd > 0 ? kFusedThreads / nd : 0;
      const int r = nd > 0 ? tid % nd : 0, pg = nd > 0 ? tid / nd : kFusedThreads;
      const float hres = tid < nd ? A.h[i0 + tid] : 0.f;  // this CTA's own rows
      bool ok = true;
      if (pg < ngr) {
        constexpr int kLoads = (kFusedMaxCtas * 32 + kFusedThreads - 1) / kFusedThreads;  // ngr >= 512 / 32
        uint64_t v[kLoads];
#pragma unroll
        for (int t2 = 0; t2 < kLoads; ++t2) {
          const int p = pg + t2 * ngr;
          v[t2] = p < nC ? ld_relaxed64(A.x_part + (size_t)p * H + i0 + r) : x_word(e_part, 0.f);
        }
        ok = x_spin_all(v, e_part, [&](int t2) { return A.x_part + (size_t)(pg + t2 * ngr) * H + i0 + r; },
                        [&](int t2) { return pg + t2 * ngr < nC; });
        float acc = 0.f;
#pragma unroll
        for (int t2 = 0; t2 < kLoads; ++t2) acc += __uint_as_float((uint32_t)v[t2]);
        sred[pg * nd + r] = acc;
      }
      if (!x_agree(ok)) { aborted = true; break; }
      float ss = 0.f;
      if (tid < nd) {
        float v = hres;
        for (int g = 0; g < ngr; ++g) v += sred[g * nd + tid];
        A.h[i0 + tid] = v;
        ss = v * v;
      }
      if (warp == 0) {
        ss = warp_sum(ss);
        if (lane == 0) A.ss_part[c] = ss;
      }
    }
    grid_arrive();  // h' and the partial sums written
  }

  if (!aborted && A.n_layers > 0 && grid_wait()) {
    // epilogue: xn' of the last layer for this CTA's rows (h' written by this thread)
    const float r_last = norm_scale();
    const float* w = A.layers[A.n_layers - 1].norm_w;
    if (tid < nd) A.xn[i0 + tid] = A.h[i0 + tid] * r_last * w[i0 + tid];
    __syncthreads();
    if (tid == 0) {
      __threadfence();
      const unsigned prev = atomicAdd(&A.sync[1], 1u);
      if (prev == (unsigned)nC - 1) {  // every CTA has read the epoch base and is past its last exchange
        A.sync[2] = base + 2u * (uint32_t)A.n_layers + 2u;
        A.sync[0] = 0;
        A.sync[1] = 0;
        __threadfence();
      }
    }
  } else if (lane == 0) {
    // drain: wait (bounded) for this issuer's copies still in flight
    for (int mb = 0; mb < kMbCount; ++mb)
      if (armed & (1u << mb)) (void)mbar_wait(&mbar[mb], (phase >> mb) & 1u);
  }
}

// Host-side plan: shared-memory layout for n_ctas CTAs; false if the shape
// does not fit the kernel.
inline bool fused_plan(int H, int I, int E, int k, int bits, int sbits, int n_ctas, size_t max_smem,
                       FusedPlan* out) {
  if (H < 64 || H % 64 || I < 64 || I % 64 || H > kFusedThreads * kFusedRowsPerThread) return false;
  if (E < 1 || E > 2 * kFusedThreads || k < 1 || k > kFusedMaxK || k > E) return false;
  if (n_ctas < 1 || n_ctas > kFusedMaxCtas) return false;
  if (E + 1 > kFusedMaxRouterRows * n_ctas) return false;
  auto wn = [](int b) { return 32 / b; };
  const int nbr = I / wn(bits), nbs = I / wn(sbits);
  if (nbs > n_ctas) return false;  // one shared block per CTA at most
  // routed blocks per CTA; a CTA's run spans at most two 64-groups
  const int per_cta = (k * nbr + n_ctas - 1) / n_ctas;
  if (per_cta > kFusedMaxRouted || per_cta > 64 / wn(bits) + 1) return false;
  if ((H + n_ctas - 1) / n_ctas > 32) return false;  // rows per CTA in the final sums: one warp
  auto blk = [&](int b) -> long long { return 12LL * H + (long long)wn(b) * 2 * (H / 64) * 4; };
  const long long slot = blk(bits) > blk(sbits) ? blk(bits) : blk(sbits);
  auto al = [](long long v) { return (v + 127) & ~127LL; };
  FusedPlan p;
  long long o = 0;
  for (int s = 0; s < kSlots; ++s) {
    p.slot[s] = (uint32_t)o;
    o = al(o + slot);
  }
  for (int e = 0; e < kSbEntries; ++e) {
    p.sbe[e] = (uint32_t)o;
    o = al(o + 4LL * H);
  }
  p.xs = (uint32_t)o;
  o = al(o + (long long)staged_x_bytes(H));
  p.logit = (uint32_t)o;
  o = al(o + 4LL * E);
  p.cand = (uint32_t)o;
  o = al(o + 8LL * kFusedWarps * kFusedMaxK);
  p.red = (uint32_t)o;
  o = al(o + 4LL * kFusedThreads);
  p.mbar = (uint32_t)o;
  o = al(o + 8LL * kMbCount);
  p.total = (uint32_t)o;
  if ((size_t)o > max_smem) return false;
  *out = p;
  return true;
}

}  // namespace fmoe
