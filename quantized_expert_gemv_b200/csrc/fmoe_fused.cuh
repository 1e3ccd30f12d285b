// fmoe_fused.cuh -- one persistent kernel for a stack of MoE layers, one or two tokens.
//
// One CTA per SM, launched cooperatively so that every CTA is resident.  The
// experts' intermediate dimension is cut into column blocks of w = 8 (4-bit)
// or 16 (2-bit) units: a block is w gate/up row pairs plus the matching w
// columns of the down matrix, one 32-bit word of codes per hidden row (the
// packed record stores the down matrix column block by column block).  A CTA
// that owns a block computes its w SwiGLU outputs and, from them, the
// block's contribution to all H outputs of the down product; the CTAs'
// partial outputs are summed at the end of the layer.  Per layer:
//   A  (all warps) xn = h' r w from the previous layer's h' and sums of
//      squares (exchange words), staged as 24-bit block floating point;
//      this CTA's router rows (fp32; the shared gate vector is row E) ->
//      logits, published as exchange words
//   E  two warp groups in a pipeline over the CTA's blocks (shared block
//      first, then its routed blocks), each block in one of three shared-
//      memory slots filled by bulk copies:
//        gate/up warps (0-7): the block's gate/up group dot products, SwiGLU,
//          the w outputs rounded to 24-bit block floating point -> handed to
//          the down warps through shared memory and an mbarrier
//        down warps (8-15): first read all logits, take the top-k, issue the
//          routed blocks' copies; then for every block the down columns of
//          all H rows (each thread 16 rows), weighted by the block's gate
//          weight; a finished block's slot takes the next block at once
//   F  the CTA's partial output for all H rows -> the workspace
//   G  (all warps) each CTA sums the partials of its slice of rows in a
//      fixed order (deterministic), adds the residual -> h' and its part of
//      sum(h'^2), published for the next layer's A
// The shared block does not depend on the routing: it is fetched during the
// previous layer and its gate/up products run while the logits travel, so
// the routed data, which cannot be requested before the top-k, has the
// memory system to itself.  Every CTA's routed blocks lie in one 64-group of
// one expert (the groups are spread over the CTAs), so one 16 KB entry holds
// their down scale-bias words, and their down products share one scale per
// row: they are accumulated unscaled and scaled once per layer.
// Two tokens per launch (NT = 2): both tokens' xn are staged, every router
// row is read once and dotted with both, the shared expert's blocks are
// read once and applied to both tokens (gate/up, SwiGLU and down products
// per token from the same codes in shared memory), and the exchanges carry
// both tokens at once, so the chain of dependent steps is paid once for
// the pair.  The routed 64-groups of the NT k (token, selected expert)
// pairs are spread over the CTAs: each CTA's routed blocks belong to one
// token and one expert.  A CTA's partial output for the other token is its
// shared-block contribution (or zero), written as soon as it is known.
// Source pages: "What is Flash-MoE?" (a2a-mcp.org), sections
// "Understanding Mixture-of-Experts", "2. FMA-optimised dequantisation
// kernels" and "3. Hand-tuned Metal compute shaders" (deferred command-buffer
// submission there plays the role the persistent kernel plays here: no host
// round trip between the steps or between layers).
//
// Exchanges between CTAs.  Router logits (E + 1 words, read whole by every
// CTA): exchange words, (epoch << 32) | fp32 bits, written and read as
// single 64-bit accesses, so a reader that sees the epoch it waits for holds
// the value that came with it -- no fence on either side; each writing warp
// adds to a relaxed counter after its stores, one thread per reading CTA
// polls that counter with a short sleep between polls (polling words that
// are still being written would slow the writers down), and only then are
// the words read (re-read, with a sleep, while a store has not landed: the
// counter is a hint, the epochs decide).  Partial outputs and h' (with its
// sums of squares): fp32 with coalesced stores, then one release-add per
// CTA on the exchange's counter; one thread per reading CTA polls it with
// acquire loads, and after a CTA-local barrier the threads read the values
// with 16-byte L2 loads where the layout allows.  The counters grow over the
// launch's layers; the last CTA to leave returns them to zero.  Every wait
// (mbarrier, counter, exchange word) is bounded: on expiry the CTA sets
// FMOE_STATUS_WAIT_TIMEOUT, records the abort in shared memory (later waits
// return at once, every warp still passes every named barrier), waits
// (bounded) for its own copies in flight, and returns.
#pragma once

#include <cstdint>

#include "fmoe.h"
#include "fmoe_device.cuh"
#include "fmoe_layout.h"

namespace fmoe {

constexpr int kFusedThreads = 512;
constexpr int kFusedWarps = kFusedThreads / 32;
constexpr int kGuThreads = 256;  // warps 0-7: gate/up, SwiGLU
constexpr int kGuWarps = kGuThreads / 32;
constexpr int kDnThreads = kFusedThreads - kGuThreads;  // warps 8-15: routing, copies, down products
constexpr int kDnWarps = kDnThreads / 32;
constexpr int kFusedMaxLayers = 32;
constexpr int kFusedMaxK = 8;
constexpr int kFusedMaxE = 1024;
constexpr int kFusedMaxH = 4096;
constexpr int kFusedMaxCtas = 160;      // partial outputs in the workspace: [kFusedMaxCtas][kFusedMaxH]
constexpr int kFusedMaxNT = 2;          // tokens per launch
// token strides of the exchange buffers (their sizes do not depend on the shape)
constexpr int kXLogitStride = kFusedMaxE + 1;
constexpr int kXSsStride = kFusedMaxCtas;
constexpr int kXHStride = kFusedMaxH;
constexpr size_t kXPartStride = (size_t)kFusedMaxCtas * kFusedMaxH;
constexpr int kFusedMaxRouterRows = 4;  // router rows (E experts + the shared gate) per CTA
constexpr int kDnQuads = 4;             // groups of 4 consecutive hidden rows per down thread: H <= 4096
constexpr int kDnRowsT = 4 * kDnQuads;  // hidden rows per down thread
constexpr int kDnKeys = kFusedMaxE / kDnThreads;  // logits per down thread in the top-k
constexpr int kSlots = 3;
constexpr int kDnxWords = 16;  // per slot: hi words [0, 8), lo words [8, 12), step, step * sum
// mbarriers
constexpr int kMbFull = 0;                 // [kSlots] a slot's bytes have landed
constexpr int kMbReady = kMbFull + kSlots;  // [kSlots] a slot's SwiGLU outputs are staged
constexpr int kMbSbShared = kMbReady + kSlots;
constexpr int kMbSbRouted = kMbSbShared + 1;
constexpr int kMbRouter = kMbSbRouted + 1;  // the layer's router rows have landed
constexpr int kMbCount = kMbRouter + 1;
constexpr int kBarGu = 1, kBarDn = 2;       // named barriers of the two warp groups
constexpr long long kWaitCycles = 4000000000LL;  // ~2 s at 2 GHz
// exchange counters (words of the workspace's counter area)
constexpr int kCntH = 0;      // CTAs that published h' and their sum of squares (all layers so far)
constexpr int kCntExit = 1;   // CTAs that left the kernel
constexpr int kEpoch = 2;     // epoch of the last launch (router-logit exchange words)
constexpr int kCntLogit = 3;  // router logits published
constexpr int kCntPart = 4;   // CTAs that published their partial outputs
constexpr unsigned kPollSleepNs = 32;    // between polls of a counter
constexpr unsigned kRepollSleepNs = 64;  // between re-reads of an exchange word

constexpr int kTimelinePoints = 48;

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
  uint32_t sbe[2];  // shared expert, routed experts
  uint32_t xs;      // staged x of the layer, per token (24-bit block floating point)
  uint32_t xs_stride;
  uint32_t logit;   // fp32 [E]
  uint32_t cand;    // top-k candidates: u64 [kDnWarps][k]
  uint32_t gred;    // gate/up partial sums: fp32 [2][NT][kGuWarps][8]
  uint32_t dnx;     // staged SwiGLU outputs per slot and token: u32 [kSlots][NT][kDnxWords]
  uint32_t red;     // fp32 [kFusedThreads]: partial sums of the row reduction
  uint32_t mbar;
  uint32_t total;
};

struct FusedArgs {
  FusedLayer layers[kFusedMaxLayers];
  int n_layers;
  int H, I, E, k;
  float eps;
  // per token, token-major (the launch's first token at the pointer); the
  // intermediates of layer l at their pointer + l * lstride bytes (0: every
  // layer writes the same place)
  float* h;           // [NT][H]
  float* xn;          // [NT][H]
  float* logits;      // [NT][E]
  int32_t* ids;       // [NT][k]
  float* weights;     // [NT][k]
  float* gamma;       // [NT]
  float* a;           // [NT][(k+1)][I], shared expert last
  float* tr_xn;       // [NT][H] per layer: the layer's input xn (nullptr: not recorded)
  float* tr_h;        // [NT][H] per layer: the layer's output h' (nullptr: not recorded)
  size_t lstride;
  uint64_t* x_logit;  // [NT][kXLogitStride]: router logits, then sigmoid(w_sg . xn) (exchange words)
  float* x_h;      // [NT][kXHStride]: h' of the layer
  float* x_ss;     // [NT][kXSsStride]: per-CTA sums of h'^2
  float* x_part;   // [NT][kXPartStride]: partial outputs, [gridDim.x][H] per token
  unsigned* sync;  // counters kCntH, kCntExit, kCntLogit, kCntPart; logit epoch base kEpoch
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

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
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

__device__ __forceinline__ void named_bar(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// 16-byte shared-memory load (a plain load, so the compiler may schedule it
// freely but never above an mbarrier wait, whose asm clobbers memory).
__device__ __forceinline__ uint4 lds128(const void* p) { return *reinterpret_cast<const uint4*>(p); }

__device__ __forceinline__ float4 as_float4(uint4 v) {
  return make_float4(__uint_as_float(v.x), __uint_as_float(v.y), __uint_as_float(v.z), __uint_as_float(v.w));
}

__device__ __forceinline__ void cnt_release_add(unsigned* p, unsigned v) {
  asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Bounded poll (one thread) until *p >= target, with acquire semantics when
// ACQ; false on expiry.
template <bool ACQ = false>
__device__ __forceinline__ bool cnt_wait(const unsigned* p, unsigned target) {
  const long long t0 = clock64();
  while (true) {
    unsigned v;
    if (ACQ) asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    else asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    if ((int)(v - target) >= 0) return true;
    if (clock64() - t0 > kWaitCycles) return false;
    __nanosleep(kPollSleepNs);
  }
}

__device__ __forceinline__ uint64_t ld_relaxed64(const uint64_t* p) {
  uint64_t v;
  asm volatile("ld.relaxed.gpu.global.b64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void st_relaxed64(uint64_t* p, uint64_t v) {
  asm volatile("st.relaxed.gpu.global.b64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

__device__ __forceinline__ void cnt_add(unsigned* p, unsigned v) {
  asm volatile("red.relaxed.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ uint64_t x_word(uint32_t epoch, float v) {
  return ((uint64_t)epoch << 32) | __float_as_uint(v);
}

__device__ __forceinline__ bool x_ready(uint64_t w, uint32_t epoch) { return (uint32_t)(w >> 32) == epoch; }

__device__ __forceinline__ float x_value(uint64_t w) { return __uint_as_float((uint32_t)w); }

// N exchange words at p(i) (those with valid(i)), already read once into w:
// re-reads the ones that do not carry `epoch` yet, with a sleep between
// rounds (bounded); false on expiry.
template <int N, class Addr, class Valid>
__device__ __forceinline__ bool x_settle(uint64_t (&w)[N], uint32_t epoch, Addr p, Valid valid) {
  const long long t0 = clock64();
  while (true) {
    bool miss = false;
#pragma unroll
    for (int i = 0; i < N; ++i) miss |= valid(i) && !x_ready(w[i], epoch);
    if (!miss) return true;
    if (clock64() - t0 > kWaitCycles) return false;
    __nanosleep(kRepollSleepNs);
#pragma unroll
    for (int i = 0; i < N; ++i)
      if (valid(i) && !x_ready(w[i], epoch)) w[i] = ld_relaxed64(p(i));
  }
}

// [lo, hi) share of `total` items for part `c` of `n`
__host__ __device__ __forceinline__ void share(int total, int c, int n, int* lo, int* hi) {
  *lo = (int)(((long long)total * c) / n);
  *hi = (int)(((long long)total * (c + 1)) / n);
}

// The 64-group of the routed blocks that CTA c of nC owns when the Gr groups
// of the k selected experts are spread over the CTAs (Gr <= nC): group j
// goes to CTAs [floor(j nC / Gr), floor((j + 1) nC / Gr)).
__host__ __device__ __forceinline__ int routed_group_of(int c, int nC, int Gr) {
  return (int)(((long long)(c + 1) * Gr - 1) / nC);
}

template <int BITS>
__device__ __forceinline__ GroupCodes<BITS> lds_group(const uint8_t* row, int ng, int g) {
  GroupCodes<BITS> gc;
  gc.c[0] = lds128(row + chunk_off<BITS>(ng, g, 0));
  if (BITS == 4) gc.c[BITS == 4 ? 1 : 0] = lds128(row + chunk_off<BITS>(ng, g, 1));
  return gc;
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
  // each lane sorts its keys (largest first): a round looks at the heads only
  auto cs = [&](int i, int j) {
    const uint64_t a = key[i], b = key[j];
    key[i] = a > b ? a : b;
    key[j] = a > b ? b : a;
  };
  if (PER >= 2) cs(0, 1);
  if (PER == 4) {
    cs(2, 3);
    cs(0, 2);
    cs(1, 3);
    cs(1, 2);
  }
  uint64_t mine = 0;
  for (int r = 0; r < k; ++r) {
    const uint64_t best = key[0];
    const uint32_t hi = __reduce_max_sync(0xffffffffu, (uint32_t)(best >> 32));
    const uint32_t lo = __reduce_max_sync(0xffffffffu, (uint32_t)(best >> 32) == hi ? (uint32_t)best : 0u);
    const uint64_t win = ((uint64_t)hi << 32) | lo;
    if (best == win) {  // keys are unique (the index is part of the key): the winning lane drops its head
#pragma unroll
      for (int i = 0; i + 1 < PER; ++i) key[i] = key[i + 1];
      key[PER - 1] = 0;
    }
    if (lane == r) mine = win;
  }
  return mine;
}

// Sum over the warp of V values per lane at once (V a power of two <= 32):
// lane l returns the total of value l >> (5 - log2 V).  Halving exchanges
// first (V / 2 + V / 4 + ... shuffles), then a plain butterfly.
template <int V>
__device__ __forceinline__ float warp_sum_multi(float (&v)[V]) {
  const int lane = threadIdx.x & 31;
  int o = 16;
#pragma unroll
  for (int n = V; n > 1; n >>= 1, o >>= 1) {
    const bool up = (lane & o) != 0;
#pragma unroll
    for (int i = 0; i < n / 2; ++i) {
      const float send = up ? v[i] : v[i + n / 2];
      const float keep = up ? v[i + n / 2] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
    }
  }
  float r = v[0];
  for (; o > 0; o >>= 1) r += __shfl_xor_sync(0xffffffffu, r, o);
  return r;
}

// Geometry of a column block of an expert with BITS-bit codes.
template <int BITS>
struct BlockGeo {
  static constexpr int kW = 32 / BITS;       // intermediate units per block
  static constexpr int kPerGroup = 64 / kW;  // blocks per 64-group
  static constexpr int kPairsPerThread = kW / 4;  // a gate/up thread's row pairs per block
  __host__ __device__ static uint32_t gu_codes(int H) { return 8u * (uint32_t)H; }
  __host__ __device__ static uint32_t dn_codes(int H) { return 4u * (uint32_t)H; }
  __host__ __device__ static uint32_t gu_sb(int H) { return (uint32_t)kW * 2u * (uint32_t)(H / 64) * 4u; }
};

// The staged inputs of one 64-group, kept in registers by a gate/up thread
// for the whole layer: thread t serves group t % 64 of every row it touches.
struct XGroup {
  uint4 xv[8];
  uint2 xl[8];
  float delta, xsum;
};

__device__ __forceinline__ XGroup load_xgroup(const StagedX& sx, int ngH) {
  XGroup x;
  const int g = threadIdx.x & 63;
  if (g < ngH) {
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      x.xv[u] = lds128(sx.xs + u * ngH + g);
      x.xl[u] = sx.xl[u * ngH + g];
    }
    x.delta = sx.delta[g];
    x.xsum = sx.xsum[g];
  } else {
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      x.xv[u] = make_uint4(0u, 0u, 0u, 0u);
      x.xl[u] = make_uint2(0u, 0u);
    }
    x.delta = x.xsum = 0.f;
  }
  return x;
}

// Gate/up part of one block (gate/up threads): thread t takes group t % 64
// of row pairs t / 64 + 4 i (both rows of each), and writes its warp's sums
// to gred [warp][value] (value 2 i: gate of pair i, 2 i + 1: up).
template <int B>
__device__ __forceinline__ void block_gateup(const uint8_t* slot, int H, const XGroup& xg, float* gred) {
  using G = BlockGeo<B>;
  constexpr int kV = 2 * G::kPairsPerThread;  // 4 or 8 values per thread
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int ngH = H / 64, g = tid & 63, ps = tid >> 6;
  const uint32_t rb = (uint32_t)H * B / 8;
  const uint32_t* sbw = reinterpret_cast<const uint32_t*>(slot + G::gu_codes(H) + G::dn_codes(H));
  float v[kV];
#pragma unroll
  for (int i = 0; i < G::kPairsPerThread; ++i) {
    v[2 * i] = v[2 * i + 1] = 0.f;
    if (g < ngH) {
      const int pl = ps + 4 * i;
      const uint8_t* rg = slot + (size_t)(2 * pl) * rb;
      const GroupCodes<B> cg = lds_group<B>(rg, ngH, g);
      const GroupCodes<B> cu = lds_group<B>(rg + rb, ngH, g);
      v[2 * i] = group_epilogue(0.f, sbw[2 * pl * ngH + g], group_dot<B>(cg, xg.xv, xg.xl), xg.delta, xg.xsum);
      v[2 * i + 1] =
          group_epilogue(0.f, sbw[(2 * pl + 1) * ngH + g], group_dot<B>(cu, xg.xv, xg.xl), xg.delta, xg.xsum);
    }
  }
  const float r = warp_sum_multi<kV>(v);
  constexpr int kLanesPer = 32 / kV;
  if ((lane & (kLanesPer - 1)) == 0) gred[warp * 8 + lane / kLanesPer] = r;
}

// SwiGLU of one block from the gate/up sums (gate/up warp 0): lane p < w
// forms a_p (returned); the w outputs get one power-of-two step (24-bit
// block floating point) and go to dnx (high parts, low parts, step,
// step * sum) for the down warps.
template <int B>
__device__ __forceinline__ float block_swiglu(const float* gred, uint32_t* dnx) {
  using G = BlockGeo<B>;
  constexpr int kW = G::kW;
  const int lane = threadIdx.x & 31;
  float a = 0.f;
  if (lane < kW) {
    const int ps = lane & 3, i = lane >> 2;
    const float gs = gred[(2 * ps) * 8 + 2 * i] + gred[(2 * ps + 1) * 8 + 2 * i];
    const float us = gred[(2 * ps) * 8 + 2 * i + 1] + gred[(2 * ps + 1) * 8 + 2 * i + 1];
    a = silu_mul(gs, us);
  }
  const float m = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(fabsf(a))));
  float inv, delta;
  bfp_step(m, &inv, &delta);
  const int q = bfp_int(a, inv);
  const int qsum = __reduce_add_sync(0xffffffffu, q);
  const uint32_t hi = (uint32_t)(q >> 8) & 0xFFFFu, lo = (uint32_t)q & 0xFFu;
  const uint32_t hi1 = __shfl_down_sync(0xffffffffu, hi, 1);
  const uint32_t lo1 = __shfl_down_sync(0xffffffffu, lo, 1);
  const uint32_t lo2 = __shfl_down_sync(0xffffffffu, lo, 2);
  const uint32_t lo3 = __shfl_down_sync(0xffffffffu, lo, 3);
  if (lane < kW && (lane & 1) == 0) dnx[lane >> 1] = hi | (hi1 << 16);
  if (lane < kW && (lane & 3) == 0) dnx[8 + (lane >> 2)] = lo | (lo1 << 8) | (lo2 << 16) | (lo3 << 24);
  if (lane == 0) {
    dnx[12] = __float_as_uint(delta);
    dnx[13] = __float_as_uint(delta * (float)qsum);
  }
  return a;
}

// Down part of one block (down threads): for the thread's row quads, the
// block's code words times the staged SwiGLU outputs; returns the 24-bit
// value sums in t[16] (rows 4 (t' + 256 m) + r at t[4 m + r]).
template <int B>
__device__ __forceinline__ void block_down(const uint8_t* slot, const uint32_t* dnx, int H, float (&t)[kDnRowsT]) {
  using G = BlockGeo<B>;
  const int td = threadIdx.x - kGuThreads;
  const uint4 h0 = lds128(dnx), h1 = lds128(dnx + 4), l01 = lds128(dnx + 8);
  const uint32_t* dc = reinterpret_cast<const uint32_t*>(slot + G::gu_codes(H));
#pragma unroll
  for (int m = 0; m < kDnQuads; ++m) {
    const int row = 4 * (td + kDnThreads * m);
    if (row < H) {
      const uint4 w = lds128(dc + row);
      const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const Acc2 acc = B == 4 ? word_dot4(ws[r], h0, make_uint2(l01.x, l01.y))
                                : word_dot2(ws[r], h0, h1, make_uint2(l01.x, l01.y), make_uint2(l01.z, l01.w));
        t[4 * m + r] = acc_value(acc);
      }
    } else {
#pragma unroll
      for (int r = 0; r < 4; ++r) t[4 * m + r] = 0.f;
    }
  }
}

// ------------------------------------------------------------ timeline --
// Built with FMOE_TIMELINE (quantized_expert_gemv_b200/timeline.py): each
// CTA records the global timer (ns) at the phase boundaries of one layer of
// a launch, g_fmoe_ts[CTA][point]; the points are listed in timeline.py.
// Without it FMOE_TS compiles to nothing.
#ifdef FMOE_TIMELINE
__device__ unsigned long long g_fmoe_ts[kFusedMaxCtas][kTimelinePoints];
__device__ int g_fmoe_ts_layer;
#define FMOE_TS(i)                                                                   \
  do {                                                                               \
    if (l == g_fmoe_ts_layer) {                                                      \
      unsigned long long t_;                                                         \
      asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t_)::"memory");               \
      g_fmoe_ts[blockIdx.x][(i)] = t_;                                               \
    }                                                                                \
  } while (0)
#else
#define FMOE_TS(i) \
  do {             \
  } while (0)
#endif

// ------------------------------------------------------------ the kernel --
template <int BITS, int SBITS, int NT>  // routed and shared code widths, tokens per launch
__global__ void __launch_bounds__(kFusedThreads, 1) fused_stack_kernel(const __grid_constant__ FusedArgs A) {
  static_assert(NT >= 1 && NT <= kFusedMaxNT, "tokens per launch");
  using GR = BlockGeo<BITS>;
  using GS = BlockGeo<SBITS>;
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ float s_gamma[NT];
  __shared__ float s_rp[kFusedWarps][NT][kFusedMaxRouterRows];
  __shared__ float s_red[NT][kFusedWarps];
  __shared__ volatile int s_abort;
  __shared__ int s_nan;

  const int c = blockIdx.x, nC = gridDim.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int H = A.H, I = A.I, E = A.E, k = A.k;
  const int ngH = H / 64, ngI = I / 64;
  const FusedPlan& P = A.plan;
  uint64_t* mbar = reinterpret_cast<uint64_t*>(smem + P.mbar);
  auto sx_of = [&](int t) { return staged_x_at(smem + P.xs + (size_t)t * P.xs_stride, H); };
  float* slog = reinterpret_cast<float*>(smem + P.logit);
  uint64_t* cand = reinterpret_cast<uint64_t*>(smem + P.cand);
  float* gred = reinterpret_cast<float*>(smem + P.gred);
  uint32_t* dnx = reinterpret_cast<uint32_t*>(smem + P.dnx);

  // ---- static work of this CTA ----
  const int nr = c <= E ? (E - c) / nC + 1 : 0;  // router rows c, c + nC, ... <= E (row E: shared gate)
  const int NBs = I * SBITS / 32;
  const int S = c < NBs ? 1 : 0;  // shared block c
  // routed blocks: [rb0, rb1) of 64-group jg of the NT k (token, selected
  // expert) pairs' groups (pair = jg / ngI: token tr = pair / k, its jj-th
  // expert; group gr = jg % ngI)
  const int Gr = NT * k * ngI;
  const int jg = routed_group_of(c, nC, Gr);
  int rb0, rb1, cs0;
  {
    cs0 = (int)(((long long)jg * nC) / Gr);
    const int cs1 = (int)(((long long)(jg + 1) * nC) / Gr);
    share(GR::kPerGroup, c - cs0, cs1 - cs0, &rb0, &rb1);
  }
  const int nq = rb1 - rb0, pair = jg / ngI, gr = jg % ngI;
  const int tr = NT == 1 ? 0 : pair / k, jj = NT == 1 ? pair : pair % k;
  // the CTA that writes token tr's ids and gate weights: the first of its first group
  const bool route_writer = jj == 0 && gr == 0 && c == cs0;
  const int nseq = S + nq;  // blocks per layer: the shared one first
  int i0, i1;
  share(H, c, nC, &i0, &i1);  // hidden rows of the final sums
  const RecordLayout LR = record_layout(BITS, H, I);
  const RecordLayout LS = record_layout(SBITS, H, I);
  const bool xthr = tid * 8 < H;  // this thread holds inputs 8 tid .. 8 tid + 7
  const int td = tid - kGuThreads, dw = warp - kGuWarps;  // down threads: index and warp in the group
  const bool issuer = tid == kGuThreads;  // the first down thread: counters and polls of the down warps
  // copies: lane 0 of down warp s issues slot s (s < kSlots), down warps
  // kWarpSb, kWarpSb + 1 the two scale-bias entries, kWarpRt the router
  // rows, the warps after them the L2 prefetches -- one owner per mbarrier,
  // owners in different warps
  constexpr int kWarpSb = kSlots, kWarpRt = kSlots + 2, kWarpPf = kSlots + 3;
  const bool owner = dw >= 0 && lane == 0;

  if (tid == 0) {
    for (int i = 0; i < kMbCount; ++i) mbar_init(&mbar[i], 1);
    s_abort = 0;
    s_nan = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();

  // owner lane: mbarriers it has armed, and per mbarrier the parity of the
  // next phase it will arm (each phase of a copy barrier is armed once, by it)
  uint32_t armed = 0, next_par = 0;
  auto arm = [&](int mb, uint32_t bytes) {
    mbar_expect_tx(&mbar[mb], bytes);
    armed |= 1u << mb;
    next_par ^= 1u << mb;
  };
  // column block nb of the record `rec` into slot s (slot s's owner)
  auto issue_block = [&](int s, const uint8_t* rec, const RecordLayout& L, int nb, uint32_t gu_sb_bytes) {
    uint8_t* dst = smem + P.slot[s];
    const uint32_t gub = 8u * (uint32_t)H, dnb = 4u * (uint32_t)H;
    fence_proxy_async();
    arm(kMbFull + s, gub + dnb + gu_sb_bytes);
    bulk_g2s(dst, rec + L.gu_codes + (size_t)nb * gub, gub, &mbar[kMbFull + s]);
    bulk_g2s(dst + gub, rec + L.down_codes + (size_t)nb * dnb, dnb, &mbar[kMbFull + s]);
    bulk_g2s(dst + gub + dnb, rec + L.gu_sb + (size_t)nb * gu_sb_bytes, gu_sb_bytes, &mbar[kMbFull + s]);
  };
  auto prefetch_block = [&](const uint8_t* rec, const RecordLayout& L, int nb, uint32_t gu_sb_bytes) {
    const uint32_t gub = 8u * (uint32_t)H, dnb = 4u * (uint32_t)H;
    prefetch_l2(rec + L.gu_codes + (size_t)nb * gub, gub);
    prefetch_l2(rec + L.down_codes + (size_t)nb * dnb, dnb);
    prefetch_l2(rec + L.gu_sb + (size_t)nb * gu_sb_bytes, gu_sb_bytes);
  };
  // down scale-bias words of 64-group g of a record into entry e (its owner)
  auto issue_sb = [&](int e, const uint8_t* rec, const RecordLayout& L, int g) {
    fence_proxy_async();
    arm(kMbSbShared + e, 4u * (uint32_t)H);
    bulk_g2s(smem + P.sbe[e], rec + L.down_sb + (size_t)g * H * 4, 4u * (uint32_t)H, &mbar[kMbSbShared + e]);
  };
  auto routed_nb = [&](int p) { return gr * GR::kPerGroup + rb0 + p - S; };  // block of position p >= S
  // block at position p of layer l into its slot, by the slot's owner; rid:
  // the selected expert of this CTA's routed group
  auto issue_pos = [&](int l, uint32_t sq, int p, int rid) {
    const int s = (int)((sq + (uint32_t)p) % kSlots);
    if (!owner || dw != s) return;
    if (p < S) issue_block(s, A.layers[l].shared, LS, c, GS::gu_sb(H));
    else issue_block(s, A.layers[l].experts + (size_t)rid * LR.bytes, LR, routed_nb(p), GR::gu_sb(H));
  };
  // Layer l's router rows (rows c + m nC, row E: the shared gate vector) into
  // the two slots that do not hold the layer's first block (sq_l: its first
  // position): rows 0-2 in one, row 3 in the other.  Issued once every block
  // before the layer is done; read in the layer's phase A, before the top-k
  // requests the routed blocks into those slots.
  auto router_row_at = [&](uint32_t sq_l, int m) -> float* {
    const int s = (int)((sq_l + 1u + (m >= 3 ? 1u : 0u)) % kSlots);
    return reinterpret_cast<float*>(smem + P.slot[s]) + (size_t)(m % 3) * H;
  };
  // the intermediates of layer l (per-layer records when tracing)
  auto lay = [&](auto* p, int l) {
    return reinterpret_cast<decltype(p)>(reinterpret_cast<char*>(p) + (size_t)l * A.lstride);
  };
  auto issue_router = [&](int l, uint32_t sq_l) {
    if (!owner || dw != kWarpRt || nr == 0) return;
    const FusedLayer& NX = A.layers[l];
    fence_proxy_async();
    arm(kMbRouter, 4u * (uint32_t)H * (uint32_t)nr);
    for (int m = 0; m < nr; ++m) {
      const int row = c + m * nC;
      bulk_g2s(router_row_at(sq_l, m), row < E ? NX.w_router + (size_t)row * H : NX.w_sg, 4u * (uint32_t)H,
               &mbar[kMbRouter]);
    }
  };

  // bounded mbarrier wait; false once this CTA has aborted (every later wait
  // returns at once)
  auto wait_mb = [&](int mb, uint32_t parity) -> bool {
    if (s_abort) return false;
    if (mbar_try(&mbar[mb], parity)) return true;
    const long long t0 = clock64();
    while (!s_abort) {
      if (mbar_try(&mbar[mb], parity)) return true;
      if (clock64() - t0 > kWaitCycles) {
        s_abort = 1;
        raise_status(FMOE_STATUS_WAIT_TIMEOUT);
        return false;
      }
    }
    return false;
  };
  auto set_abort = [&]() {
    if (!s_abort) {
      s_abort = 1;
      raise_status(FMOE_STATUS_WAIT_TIMEOUT);
    }
  };
  // CTA-wide wait for a counter (thread 0 polls, with acquire loads)
  auto cta_cnt_wait = [&](int which, unsigned target) -> bool {
    bool ok = true;
    if (tid == 0) ok = cnt_wait<true>(A.sync + which, target);
    if (__syncthreads_and(ok && !s_abort)) return true;
    if (tid == 0) raise_status(FMOE_STATUS_WAIT_TIMEOUT);
    return false;
  };
  // per token: r = (sum of the CTAs' partial sums of h'^2 / H + eps)^(-1/2),
  // summed in the same order in every CTA (thread t < nC holds CTA t's partials)
  auto norm_scales = [&](float (&r)[NT]) {
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      const float v = warp_sum(tid < nC ? __ldcg(A.x_ss + (size_t)t * kXSsStride + tid) : 0.f);
      if (lane == 0) s_red[t][warp] = v;
    }
    __syncthreads();
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      float s = 0.f;
#pragma unroll
      for (int wi = 0; wi < kFusedWarps; ++wi) s += s_red[t][wi];
      r[t] = 1.f / sqrtf(s / (float)H + A.eps);
    }
    __syncthreads();
  };
  // the down threads' rows of a partial output: quads 4 (td + kDnThreads m)
  auto store_rows = [&](float* part, const float (&v)[kDnRowsT]) {
#pragma unroll
    for (int m = 0; m < kDnQuads; ++m) {
      const int row = 4 * (td + kDnThreads * m);
      if (row < H)
        __stcg(reinterpret_cast<float4*>(part + row), make_float4(v[4 * m], v[4 * m + 1], v[4 * m + 2], v[4 * m + 3]));
    }
  };

  const uint32_t base = __ldcg(A.sync + kEpoch);  // logit epoch of layer l: base + l + 1
  uint32_t sq = 0;  // blocks of earlier layers (slot of position p: (sq + p) % 3)
  // the first layer's shared block, its down scale-bias entry and router rows
  if (A.n_layers > 0 && S) {
    issue_pos(0, 0u, 0, 0);
    if (owner && dw == kWarpSb) issue_sb(0, A.layers[0].shared, LS, c / GS::kPerGroup);
  }
  if (A.n_layers > 0) issue_router(0, 0u);

  bool aborted = false;
  for (int l = 0; l < A.n_layers; ++l) {
    const FusedLayer& LY = A.layers[l];
    if (tid == 0) FMOE_TS(0);
    const uint32_t e_logit = base + (uint32_t)l + 1u;
    // ------------------------------------------------------------- A --
    float xv[NT][8];
    if (l == 0) {
#pragma unroll
      for (int t = 0; t < NT; ++t) {
        float4 v0 = make_float4(0.f, 0.f, 0.f, 0.f), v1 = v0;
        if (xthr) {
          v0 = __ldcg(reinterpret_cast<const float4*>(A.xn + (size_t)t * H + tid * 8));
          v1 = __ldcg(reinterpret_cast<const float4*>(A.xn + (size_t)t * H + tid * 8 + 4));
        }
        xv[t][0] = v0.x; xv[t][1] = v0.y; xv[t][2] = v0.z; xv[t][3] = v0.w;
        xv[t][4] = v1.x; xv[t][5] = v1.y; xv[t][6] = v1.z; xv[t][7] = v1.w;
      }
    } else {
      // h' and the sums of squares of the previous layer: every CTA has published them
      if (!cta_cnt_wait(kCntH, (unsigned)l * (unsigned)nC)) { aborted = true; break; }
      if (tid == 0) FMOE_TS(1);
      float4 w0 = make_float4(0.f, 0.f, 0.f, 0.f), w1 = w0;
      const float* wprev = A.layers[l - 1].norm_w;
      if (xthr) {
        w0 = __ldg(reinterpret_cast<const float4*>(wprev + tid * 8));
        w1 = __ldg(reinterpret_cast<const float4*>(wprev + tid * 8 + 4));
      }
      float4 hv[NT][2];
#pragma unroll
      for (int t = 0; t < NT; ++t) {
        hv[t][0] = hv[t][1] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (xthr) {
          hv[t][0] = __ldcg(reinterpret_cast<const float4*>(A.x_h + (size_t)t * kXHStride + tid * 8));
          hv[t][1] = __ldcg(reinterpret_cast<const float4*>(A.x_h + (size_t)t * kXHStride + tid * 8 + 4));
        }
      }
      float r[NT];
      norm_scales(r);
#pragma unroll
      for (int t = 0; t < NT; ++t) {
        const float4 h0 = hv[t][0], h1 = hv[t][1];
        const float rt = r[t];
        xv[t][0] = h0.x * rt * w0.x; xv[t][1] = h0.y * rt * w0.y; xv[t][2] = h0.z * rt * w0.z;
        xv[t][3] = h0.w * rt * w0.w; xv[t][4] = h1.x * rt * w1.x; xv[t][5] = h1.y * rt * w1.y;
        xv[t][6] = h1.z * rt * w1.z; xv[t][7] = h1.w * rt * w1.w;
      }
    }
    if (tid == 0) FMOE_TS(2);
    if (A.tr_xn && xthr) {
#pragma unroll
      for (int t = 0; t < NT; ++t) {
        float* tx = lay(A.tr_xn, l) + (size_t)t * H + tid * 8;
        __stcg(reinterpret_cast<float4*>(tx), make_float4(xv[t][0], xv[t][1], xv[t][2], xv[t][3]));
        __stcg(reinterpret_cast<float4*>(tx + 4), make_float4(xv[t][4], xv[t][5], xv[t][6], xv[t][7]));
      }
    }
    // stage x: 8 consecutive threads share one 64-group
#pragma unroll
    for (int t = 0; t < NT; ++t) stage_unit(xv[t], xthr, tid >> 3, tid & 7, ngH, sx_of(t));
    // router partial dot products (rows in shared memory, each read once for
    // all tokens): value t R + m of a thread is token t's product with row
    // m; each warp reduces all of them at once, then warp 0 adds the warps'
    // sums in warp order
    if (tid == 0) FMOE_TS(3);
    if (nr > 0 && !wait_mb(kMbRouter, (uint32_t)l & 1u)) set_abort();
    if (tid == 0) FMOE_TS(4);
    constexpr int kRV = NT * kFusedMaxRouterRows;  // values per thread: a power of two
    float dv[kRV];
#pragma unroll
    for (int m = 0; m < kFusedMaxRouterRows; ++m) {
      float4 wr[2] = {make_float4(0.f, 0.f, 0.f, 0.f), make_float4(0.f, 0.f, 0.f, 0.f)};
      if (m < nr && xthr && !s_abort) {
        const float* rr = router_row_at(sq, m) + tid * 8;
        wr[0] = as_float4(lds128(rr));
        wr[1] = as_float4(lds128(rr + 4));
      }
#pragma unroll
      for (int t = 0; t < NT; ++t) {
        float d = wr[0].x * xv[t][0];
        d = fmaf(wr[0].y, xv[t][1], d);
        d = fmaf(wr[0].z, xv[t][2], d);
        d = fmaf(wr[0].w, xv[t][3], d);
        d = fmaf(wr[1].x, xv[t][4], d);
        d = fmaf(wr[1].y, xv[t][5], d);
        d = fmaf(wr[1].z, xv[t][6], d);
        d = fmaf(wr[1].w, xv[t][7], d);
        dv[t * kFusedMaxRouterRows + m] = d;
      }
    }
    {
      const float d = warp_sum_multi<kRV>(dv);  // lane l: the total of value l / (32 / kRV)
      constexpr int kLanesPer = 32 / kRV;
      if ((lane & (kLanesPer - 1)) == 0) {
        const int v = lane / kLanesPer;
        s_rp[warp][v / kFusedMaxRouterRows][v % kFusedMaxRouterRows] = d;
      }
    }
    __syncthreads();
    if (tid == 0) FMOE_TS(5);
    if (warp == 0) {
      const int t = lane / kFusedMaxRouterRows, m = lane % kFusedMaxRouterRows;
      if (t < NT && m < nr) {
        float v = 0.f;
        for (int w = 0; w < kFusedWarps; ++w) v += s_rp[w][t][m];
        const int row = c + m * nC;
        if (row < E) lay(A.logits, l)[(size_t)t * E + row] = v;
        else lay(A.gamma, l)[t] = v = 1.f / (1.f + expf(-v));
        st_relaxed64(A.x_logit + (size_t)t * kXLogitStride + row, x_word(e_logit, v));
      }
      __syncwarp();
      if (lane == 0 && nr > 0) cnt_add(A.sync + kCntLogit, (unsigned)nr);
    }
    if (tid == 0) FMOE_TS(6);
    // ------------------------------------------------------------- E --
    if (warp < kGuWarps) {
      // ---- gate/up warps ----
      // the staged inputs of the token of the first block: the shared block
      // runs token 0 first, the routed blocks take token tr
      XGroup xg = load_xgroup(sx_of(S ? 0 : tr), ngH);
      for (int p = 0; p < nseq; ++p) {
        const uint32_t pos = sq + (uint32_t)p;
        const int s = (int)(pos % kSlots);
        const bool ok = wait_mb(kMbFull + s, (pos / kSlots) & 1u);
        if (tid == 0 && p < 5) FMOE_TS(7 + p);
        float* gb = gred + (pos & 1u) * (NT * kGuWarps * 8);
        const uint8_t* sl = smem + P.slot[s];
        if (ok) {
          if (p < S) {
            block_gateup<SBITS>(sl, H, xg, gb);
#pragma unroll
            for (int t = 1; t < NT; ++t) {
              xg = load_xgroup(sx_of(t), ngH);
              block_gateup<SBITS>(sl, H, xg, gb + t * (kGuWarps * 8));
            }
            if (NT > 1 && tr != NT - 1) xg = load_xgroup(sx_of(tr), ngH);
          } else {
            block_gateup<BITS>(sl, H, xg, gb);
          }
        }
        named_bar(kBarGu, kGuThreads);
        if (warp == 0) {
          if (lane == 0 && p < 5) FMOE_TS(12 + p);
          uint32_t* dx = dnx + s * (NT * kDnxWords);
          if (p < S) {
            float a[NT];
#pragma unroll
            for (int t = 0; t < NT; ++t) a[t] = block_swiglu<SBITS>(gb + t * (kGuWarps * 8), dx + t * kDnxWords);
            __syncwarp();
            if (lane == 0) mbar_arrive(&mbar[kMbReady + s]);
            // the SwiGLU outputs to the workspace, after the hand-off (a global
            // store before the arrive would make it wait for the store)
#pragma unroll
            for (int t = 0; t < NT; ++t)
              if (lane < GS::kW) lay(A.a, l)[((size_t)t * (k + 1) + k) * I + (size_t)c * GS::kW + lane] = a[t];
          } else {
            const float a = block_swiglu<BITS>(gb, dx);
            __syncwarp();
            if (lane == 0) mbar_arrive(&mbar[kMbReady + s]);
            if (lane < GR::kW)
              lay(A.a, l)[((size_t)tr * (k + 1) + jj) * I + (size_t)routed_nb(p) * GR::kW + lane] = a;
          }
        }
      }
    } else {
      // ---- down warps: routing first (token tr's top-k; every token's gamma) ----
      int rid;      // the selected expert of this CTA's routed group
      float wt_r;   // its gate weight
      {
        // every CTA has published its router rows: (l + 1) (E + 1) in all
        if (issuer && !cnt_wait<false>(A.sync + kCntLogit, (unsigned)(l + 1) * (unsigned)(E + 1))) set_abort();
        named_bar(kBarDn, kDnThreads);
        if (issuer) FMOE_TS(17);
        const uint64_t* xl_tr = A.x_logit + (size_t)tr * kXLogitStride;
        uint64_t lw[kDnKeys + 1];
#pragma unroll
        for (int i = 0; i < kDnKeys; ++i) {
          const int e = td + i * kDnThreads;
          lw[i] = e < E ? ld_relaxed64(xl_tr + e) : 0;
        }
        lw[kDnKeys] = td < NT ? ld_relaxed64(A.x_logit + (size_t)td * kXLogitStride + E) : 0;
        if (!x_settle(lw, e_logit,
                      [&](int i) {
                        return i < kDnKeys ? xl_tr + td + i * kDnThreads
                                           : A.x_logit + (size_t)td * kXLogitStride + E;
                      },
                      [&](int i) { return i < kDnKeys ? td + i * kDnThreads < E : td < NT; }))
          set_abort();
        if (td < NT) s_gamma[td] = x_value(lw[kDnKeys]);
        uint64_t key[kDnKeys];
        bool nan_seen = false;
#pragma unroll
        for (int i = 0; i < kDnKeys; ++i) {
          const int e = td + i * kDnThreads;
          key[i] = 0;
          if (e < E) {
            const float v = x_value(lw[i]);
            nan_seen |= isnan(v);
            slog[e] = v;
            key[i] = route_key(v, e);
          }
        }
        const uint64_t wk = E <= 2 * kDnThreads ? warp_select_keys<2>(key, k) : warp_select_keys<kDnKeys>(key, k);
        if (lane < k) cand[dw * k + lane] = wk;
        if (__any_sync(0xffffffffu, nan_seen) && lane == 0) s_nan = 1;
        if (issuer) FMOE_TS(18);
        named_bar(kBarDn, kDnThreads);
        // every down warp merges the warps' candidates itself (same result in
        // each): the top-k ids, and the softmax of their logits
        uint64_t kk[2];
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          const int idx = lane + 32 * i;
          kk[i] = idx < kDnWarps * k ? cand[idx] : 0;
        }
        const uint64_t win = warp_select_keys<2>(kk, k);
        const int sel = lane < k ? key_index(win) : 0;
        const float val = lane < k ? slog[sel] : 0.f;
        float m = -INFINITY;
        for (int r = 0; r < k; ++r) {
          const float vr = __shfl_sync(0xffffffffu, val, r);
          if (!isnan(vr)) m = fmaxf(m, vr);
        }
        const float pe = (lane < k && !isnan(val)) ? expf(val - m) : 0.f;
        const float z = warp_sum(pe);
        const float pw = z > 0.f ? pe / z : 0.f;
        rid = __shfl_sync(0xffffffffu, sel, jj);
        wt_r = __shfl_sync(0xffffffffu, pw, jj);
        if (route_writer && dw == 0) {
          if (lane < k) {
            lay(A.ids, l)[(size_t)tr * k + lane] = sel;
            lay(A.weights, l)[(size_t)tr * k + lane] = pw;
          }
          if (lane == 0 && s_nan) raise_status(FMOE_STATUS_NAN_LOGIT);
        }
        if (issuer) FMOE_TS(19);
        // requests, each by its owner: the routed blocks that have a free
        // slot, their down scale-bias entry, L2 prefetches of the later
        // ones, and the next layer's shared block when its slot is free
        if (owner && !s_abort) {
          for (int p = S; p < nseq && p < kSlots; ++p) issue_pos(l, sq, p, rid);
          if (nq > 0 && dw == kWarpSb + 1) issue_sb(1, LY.experts + (size_t)rid * LR.bytes, LR, gr);
          if (dw >= kWarpPf)
            for (int p = kSlots + dw - kWarpPf; p < nseq; p += kDnWarps - kWarpPf)
              prefetch_block(LY.experts + (size_t)rid * LR.bytes, LR, routed_nb(p), GR::gu_sb(H));
          if (S && l + 1 < A.n_layers && nseq < kSlots) issue_pos(l + 1, sq + (uint32_t)nseq, 0, 0);
        }
      }
      if (issuer) FMOE_TS(20);
      // the other tokens' partial outputs of a CTA without a shared block: zero
      if (NT > 1 && !S) {
        float zr[kDnRowsT];
#pragma unroll
        for (int m = 0; m < kDnRowsT; ++m) zr[m] = 0.f;
#pragma unroll
        for (int t = 0; t < NT; ++t)
          if (t != tr) store_rows(A.x_part + (size_t)t * kXPartStride + (size_t)c * H, zr);
      }
      // ---- down products, block by block ----
      float yacc[kDnRowsT];  // the shared block's contribution to token tr
      float uacc[kDnRowsT];  // routed blocks: sum of step * weight * value, scaled per row at the end
#pragma unroll
      for (int m = 0; m < kDnRowsT; ++m) yacc[m] = uacc[m] = 0.f;
      float p2sum = 0.f;  // routed blocks: sum of step * weight * sum xi (times the row's bias at the end)
      for (int p = 0; p < nseq; ++p) {
        const uint32_t pos = sq + (uint32_t)p;
        const int s = (int)(pos % kSlots);
        bool ok = wait_mb(kMbReady + s, (pos / kSlots) & 1u);
        ok = ok && wait_mb(kMbFull + s, (pos / kSlots) & 1u);
        if (p == 0 && S) ok = ok && wait_mb(kMbSbShared, (uint32_t)l & 1u);
        if (issuer && p < 5) FMOE_TS(21 + p);
        if (ok) {
          const uint8_t* sl = smem + P.slot[s];
          const uint32_t* dx = dnx + s * (NT * kDnxWords);
          float t[kDnRowsT];
          if (p < S) {
            // the shared block: every token's down products from the same codes
            const uint32_t* sbe = reinterpret_cast<const uint32_t*>(smem + P.sbe[0]);
#pragma unroll
            for (int tk = 0; tk < NT; ++tk) {
              const uint32_t* dxt = dx + tk * kDnxWords;
              block_down<SBITS>(sl, dxt, H, t);
              const float p1 = s_gamma[tk] * __uint_as_float(dxt[12]), p2 = s_gamma[tk] * __uint_as_float(dxt[13]);
              float v[kDnRowsT];
#pragma unroll
              for (int mq = 0; mq < kDnQuads; ++mq) {
                const int row = 4 * (td + kDnThreads * mq);
                uint4 sb = make_uint4(0u, 0u, 0u, 0u);
                if (row < H) sb = lds128(sbe + row);
                const uint32_t sw[4] = {sb.x, sb.y, sb.z, sb.w};
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                  const float sc = __uint_as_float(sw[r] << 16), bi = __uint_as_float(sw[r] & 0xFFFF0000u);
                  v[4 * mq + r] = fmaf(sc, p1 * t[4 * mq + r], bi * p2);
                }
              }
              if (tk == tr) {
#pragma unroll
                for (int mm = 0; mm < kDnRowsT; ++mm) yacc[mm] = v[mm];
              } else {
                store_rows(A.x_part + (size_t)tk * kXPartStride + (size_t)c * H, v);
              }
            }
          } else {
            block_down<BITS>(sl, dx, H, t);
            const float p1 = wt_r * __uint_as_float(dx[12]);
            p2sum = fmaf(wt_r, __uint_as_float(dx[13]), p2sum);
#pragma unroll
            for (int mm = 0; mm < kDnRowsT; ++mm) uacc[mm] = fmaf(p1, t[mm], uacc[mm]);
          }
        }
        named_bar(kBarDn, kDnThreads);  // every down thread is done with the slot
        if (issuer && p < 5) FMOE_TS(26 + p);
        if (owner && !s_abort) {
          // the slot takes the block three positions on: this layer's, or
          // the next layer's shared block
          const int pn = p + kSlots;
          if (pn < nseq) issue_pos(l, sq, pn, rid);
          else if (pn == nseq && S && l + 1 < A.n_layers) issue_pos(l + 1, sq + (uint32_t)nseq, 0, 0);
          // the shared entry is free: the next layer's comes in
          if (p == 0 && S && l + 1 < A.n_layers && dw == kWarpSb)
            issue_sb(0, A.layers[l + 1].shared, LS, c / GS::kPerGroup);
        }
      }
      // every block of the layer is done: the next layer's router rows come in
      if (l + 1 < A.n_layers && !s_abort) issue_router(l + 1, sq + (uint32_t)nseq);
      // ---- F: routed blocks scaled per row, token tr's partial output out ----
      bool ok = true;
      if (nq > 0) ok = wait_mb(kMbSbRouted, (uint32_t)l & 1u);
      const uint32_t* sbe = reinterpret_cast<const uint32_t*>(smem + P.sbe[1]);
      float* part = A.x_part + (size_t)tr * kXPartStride + (size_t)c * H;
#pragma unroll
      for (int m = 0; m < kDnQuads; ++m) {
        const int row = 4 * (td + kDnThreads * m);
        if (row < H) {
          float v[4];
          if (nq > 0 && ok) {
            const uint4 sb = lds128(sbe + row);
            const uint32_t sw[4] = {sb.x, sb.y, sb.z, sb.w};
#pragma unroll
            for (int r = 0; r < 4; ++r) {
              const float sc = __uint_as_float(sw[r] << 16), bi = __uint_as_float(sw[r] & 0xFFFF0000u);
              v[r] = fmaf(sc, uacc[4 * m + r], fmaf(bi, p2sum, yacc[4 * m + r]));
            }
          } else {
#pragma unroll
            for (int r = 0; r < 4; ++r) v[r] = yacc[4 * m + r];
          }
          __stcg(reinterpret_cast<float4*>(part + row), make_float4(v[0], v[1], v[2], v[3]));
        }
      }
      if (issuer) FMOE_TS(31);
      named_bar(kBarDn, kDnThreads);
      if (issuer) cnt_release_add(A.sync + kCntPart, 1u);
    }
    if (issuer) FMOE_TS(32);
    sq += (uint32_t)nseq;
    if (__syncthreads_or(s_abort)) { aborted = true; break; }
    // ------------------------------------------------------------- G --
    {
      // values q = t nd + r (token t, row i0 + r), q < nv: ngr threads per
      // value each sum every ngr-th CTA's partial; then warp 0 adds those
      // sums in order (lane r: row i0 + r of every token)
      const int nd = i1 - i0, nv = NT * nd;
      const int ngr = nv > 0 ? kFusedThreads / nv : 0;
      const int q = nv > 0 ? tid % nv : 0, pg = nv > 0 ? tid / nv : kFusedThreads;
      const int tq = nd > 0 ? q / nd : 0, r = nd > 0 ? q % nd : 0;
      float hres[NT];  // this CTA's own rows
#pragma unroll
      for (int t = 0; t < NT; ++t) hres[t] = tid < nd ? A.h[(size_t)t * H + i0 + tid] : 0.f;
      if (!cta_cnt_wait(kCntPart, (unsigned)(l + 1) * (unsigned)nC)) { aborted = true; break; }
      if (tid == 0) FMOE_TS(33);
      float* sred = reinterpret_cast<float*>(smem + P.red);
      if (pg < ngr) {
        // ngr >= kFusedThreads / (32 NT)
        constexpr int kLoads = (kFusedMaxCtas * 32 * NT + kFusedThreads - 1) / kFusedThreads;
        const float* src = A.x_part + (size_t)tq * kXPartStride + i0 + r;
        float v[kLoads];
#pragma unroll
        for (int t2 = 0; t2 < kLoads; ++t2) {
          const int p = pg + t2 * ngr;
          v[t2] = p < nC ? __ldcg(src + (size_t)p * H) : 0.f;
        }
        float acc = 0.f;
#pragma unroll
        for (int t2 = 0; t2 < kLoads; ++t2) acc += v[t2];
        sred[pg * nv + q] = acc;
      }
      __syncthreads();
      if (tid == 0) FMOE_TS(34);
      if (warp == 0) {
        float ss[NT];
#pragma unroll
        for (int t = 0; t < NT; ++t) {
          ss[t] = 0.f;
          if (tid < nd) {
            float v = hres[t];
            for (int g = 0; g < ngr; ++g) v += sred[g * nv + t * nd + tid];
            A.h[(size_t)t * H + i0 + tid] = v;
            __stcg(A.x_h + (size_t)t * kXHStride + i0 + tid, v);
            if (A.tr_h) lay(A.tr_h, l)[(size_t)t * H + i0 + tid] = v;
            ss[t] = v * v;
          }
          ss[t] = warp_sum(ss[t]);
          if (lane == 0) __stcg(A.x_ss + (size_t)t * kXSsStride + c, ss[t]);
        }
        __syncwarp();
        if (lane == 0) cnt_release_add(A.sync + kCntH, 1u);  // warp 0 wrote every row of this CTA (nd <= 32)
      }
      if (tid == 0) FMOE_TS(35);
    }
  }

  // after the last layer: every CTA's adds have landed
  bool done = !aborted && A.n_layers > 0;
  if (done) done = cta_cnt_wait(kCntH, (unsigned)A.n_layers * (unsigned)nC);
  if (done) {
    // epilogue: xn' of the last layer for this CTA's rows (h' written by this CTA)
    float r_last[NT];
    norm_scales(r_last);
    const float* w = A.layers[A.n_layers - 1].norm_w;
    if (tid < i1 - i0) {
#pragma unroll
      for (int t = 0; t < NT; ++t)
        A.xn[(size_t)t * H + i0 + tid] = A.h[(size_t)t * H + i0 + tid] * r_last[t] * w[i0 + tid];
    }
    __syncthreads();
    if (tid == 0) {
      __threadfence();
      const unsigned prev = atomicAdd(&A.sync[kCntExit], 1u);
      if (prev == (unsigned)nC - 1) {  // every CTA is past its last counter wait
        A.sync[kEpoch] = base + (uint32_t)A.n_layers + 1u;
        A.sync[kCntH] = 0;
        A.sync[kCntLogit] = 0;
        A.sync[kCntPart] = 0;
        A.sync[kCntExit] = 0;
        __threadfence();
      }
    }
  }
  if (owner) {
    // drain: wait (bounded) for this lane's copies still in flight -- the
    // last phase armed on each barrier (earlier phases have completed: a
    // slot or entry is re-armed only after its previous contents were used).
    // On a clean exit these phases have completed already.
    for (int mb = 0; mb < kMbCount; ++mb)
      if (armed & (1u << mb)) (void)mbar_wait(&mbar[mb], ((next_par >> mb) & 1u) ^ 1u);
  }
}

// Host-side plan: shared-memory layout for n_ctas CTAs and nt tokens per
// launch; false if the shape does not fit the kernel.
inline bool fused_plan(int H, int I, int E, int k, int bits, int sbits, int nt, int n_ctas, size_t max_smem,
                       FusedPlan* out) {
  if (nt < 1 || nt > kFusedMaxNT) return false;
  if (H < 64 || H % 64 || I < 64 || I % 64 || H > kFusedMaxH) return false;
  if (E < 1 || E > kFusedMaxE || k < 1 || k > kFusedMaxK || k > E) return false;
  if (n_ctas < 1 || n_ctas > kFusedMaxCtas) return false;
  if (E + 1 > kFusedMaxRouterRows * n_ctas) return false;
  auto wn = [](int b) { return 32 / b; };
  const int nbs = I / wn(sbits);
  if (nbs > n_ctas) return false;        // one shared block per CTA at most
  if (nt * k * (I / 64) > n_ctas) return false;  // one routed 64-group per CTA at most
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
  for (int e = 0; e < 2; ++e) {
    p.sbe[e] = (uint32_t)o;
    o = al(o + 4LL * H);
  }
  p.xs = (uint32_t)o;
  p.xs_stride = (uint32_t)al((long long)staged_x_bytes(H));
  o = al(o + (long long)nt * p.xs_stride);
  p.logit = (uint32_t)o;
  o = al(o + 4LL * E);
  p.cand = (uint32_t)o;
  o = al(o + 8LL * (kDnWarps * kFusedMaxK + 1));
  p.gred = (uint32_t)o;
  o = al(o + 4LL * 2 * nt * kGuWarps * 8);
  p.dnx = (uint32_t)o;
  o = al(o + 4LL * kSlots * nt * kDnxWords);
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
