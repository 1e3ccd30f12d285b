// fmoe_cache.cuh -- host-memory expert tier with a device cache of expert
// records (included once, at the end of fmoe_kernels.cu).
//
// The routed experts of every layer stay in (pinned) host memory; a fixed
// number of device slots holds the records most recently used, shared by
// all layers, least recently used evicted first.  One layer step: the
// router and top-k run on the device, the step's expert ids come back to
// the host (the step waits for them: the host decides what to copy), every
// missing record is copied into a slot, the layer's table of record
// addresses is updated, and the expert products and the combine run on the
// device reading the records through that table.
// Source pages: "What is Flash-MoE?" (a2a-mcp.org), section "1. SSD expert
// streaming" (experts fetched per layer from a slower tier after routing;
// the pages rely on the OS page cache rather than a custom cache) -- here
// the slower tier is host memory over PCIe and the cache is explicit.
#pragma once

#include <cstdint>
#include <unordered_map>
#include <vector>

struct fmoe_expert_cache {
  fmoe_layer_desc desc;
  int n_layers;
  size_t rec;                                  // bytes of one routed record
  std::vector<const uint8_t*> host_layers;     // per layer: E records in host memory
  int n_slots;
  uint8_t* d_slots;                            // device: n_slots records
  uint64_t* d_table;                           // device: [n_layers][E] record addresses
  uint64_t* h_table;                           // pinned mirror of d_table
  int32_t* h_ids;                              // pinned: one step's ids
  int max_tokens;
  std::vector<int64_t> slot_key;               // layer * E + id held by each slot, -1: empty
  std::vector<uint64_t> slot_stamp;            // last use of each slot
  std::unordered_map<int64_t, int> where;      // key -> slot
  uint64_t clock, hits, misses, bytes_in;
};

namespace fmoe {

// Chooses the slot for a missing key: an empty slot, else the least recently
// used one whose record this step does not need (stamp < step_start).
static int cache_victim(const fmoe_expert_cache* c, uint64_t step_start) {
  int best = -1;
  for (int s = 0; s < c->n_slots; ++s) {
    if (c->slot_key[s] < 0) return s;
    if (c->slot_stamp[s] >= step_start) continue;
    if (best < 0 || c->slot_stamp[s] < c->slot_stamp[best]) best = s;
  }
  return best;
}

// Makes every id of the step resident: hits refresh their stamp, misses take
// a victim slot and enqueue the copy of their record on `st`.  Returns the
// number of copies, or -1 when the slots cannot hold the step's experts.
static int cache_admit(fmoe_expert_cache* c, int layer, const int32_t* ids, int n, cudaStream_t st) {
  const int E = c->desc.n_experts;
  const uint64_t step_start = ++c->clock;
  int copies = 0;
  for (int i = 0; i < n; ++i) {
    const int id = ids[i];
    if (id < 0 || id >= E) continue;  // the kernels zero a bad slot and flag it
    const int64_t key = (int64_t)layer * E + id;
    auto it = c->where.find(key);
    if (it != c->where.end()) {
      if (c->slot_stamp[it->second] < step_start) ++c->hits;  // once per expert and step
      c->slot_stamp[it->second] = step_start;
      continue;
    }
    const int s = cache_victim(c, step_start);
    if (s < 0) return -1;
    if (c->slot_key[s] >= 0) {
      c->h_table[c->slot_key[s]] = 0;
      c->where.erase(c->slot_key[s]);
    }
    uint8_t* dst = c->d_slots + (size_t)s * c->rec;
    if (cudaMemcpyAsync(dst, c->host_layers[layer] + (size_t)id * c->rec, c->rec, cudaMemcpyHostToDevice, st) !=
        cudaSuccess)
      return -2;
    c->slot_key[s] = key;
    c->slot_stamp[s] = step_start;
    c->where[key] = s;
    c->h_table[key] = reinterpret_cast<uint64_t>(dst);
    ++c->misses;
    c->bytes_in += c->rec;
    ++copies;
  }
  return copies;
}

}  // namespace fmoe

extern "C" int fmoe_cache_create(const fmoe_layer_desc* d, int n_layers, const void* const* h_layer_experts,
                                 int n_slots, void* d_slots, size_t d_slots_bytes, uint64_t* d_table,
                                 int max_tokens, fmoe_expert_cache** out) {
  if (!d || !out || !h_layer_experts || !d_slots || !d_table || n_layers < 1 || n_slots < 1 || max_tokens < 1)
    return FMOE_ERR_INVALID_ARG;
  *out = nullptr;
  if (!desc_valid(d)) return FMOE_ERR_INVALID_ARG;
  if (!desc_supported(d)) return FMOE_ERR_UNSUPPORTED;
  const size_t rec = record_layout(d->bits, d->hidden, d->inter).bytes;
  if (d_slots_bytes < rec * (size_t)n_slots) return FMOE_ERR_BUFFER_TOO_SMALL;
  if (!aligned16(d_slots) || !aligned16(d_table)) return FMOE_ERR_INVALID_ARG;
  for (int l = 0; l < n_layers; ++l)
    if (!h_layer_experts[l]) return FMOE_ERR_INVALID_ARG;
  fmoe_expert_cache* c = new fmoe_expert_cache();
  c->desc = *d;
  c->n_layers = n_layers;
  c->rec = rec;
  for (int l = 0; l < n_layers; ++l) c->host_layers.push_back(static_cast<const uint8_t*>(h_layer_experts[l]));
  c->n_slots = n_slots;
  c->d_slots = static_cast<uint8_t*>(d_slots);
  c->d_table = d_table;
  c->max_tokens = max_tokens;
  const size_t table_bytes = (size_t)n_layers * d->n_experts * sizeof(uint64_t);
  if (cudaHostAlloc(reinterpret_cast<void**>(&c->h_table), table_bytes, cudaHostAllocDefault) != cudaSuccess ||
      cudaHostAlloc(reinterpret_cast<void**>(&c->h_ids), (size_t)max_tokens * d->top_k * sizeof(int32_t),
                    cudaHostAllocDefault) != cudaSuccess) {
    if (c->h_table) cudaFreeHost(c->h_table);
    delete c;
    return FMOE_ERR_CUDA;
  }
  std::memset(c->h_table, 0, table_bytes);
  c->slot_key.assign(n_slots, -1);
  c->slot_stamp.assign(n_slots, 0);
  c->clock = c->hits = c->misses = c->bytes_in = 0;
  if (cudaMemcpy(d_table, c->h_table, table_bytes, cudaMemcpyHostToDevice) != cudaSuccess) {
    cudaFreeHost(c->h_table);
    cudaFreeHost(c->h_ids);
    delete c;
    return FMOE_ERR_CUDA;
  }
  *out = c;
  return FMOE_OK;
}

extern "C" int fmoe_cache_destroy(fmoe_expert_cache* c) {
  if (!c) return FMOE_ERR_INVALID_ARG;
  cudaFreeHost(c->h_table);
  cudaFreeHost(c->h_ids);
  delete c;
  return FMOE_OK;
}

extern "C" int fmoe_cache_stats(const fmoe_expert_cache* c, uint64_t* hits, uint64_t* misses, uint64_t* bytes_in) {
  if (!c) return FMOE_ERR_INVALID_ARG;
  if (hits) *hits = c->hits;
  if (misses) *misses = c->misses;
  if (bytes_in) *bytes_in = c->bytes_in;
  return FMOE_OK;
}

extern "C" int fmoe_cache_layer_forward(fmoe_expert_cache* c, int layer, const fmoe_layer_weights* lw,
                                        const float* d_logits, float* d_h, float* d_xn, int T, void* d_ws,
                                        size_t ws_bytes, cudaStream_t st) {
  using namespace fmoe;
  if (!c || !lw || layer < 0 || layer >= c->n_layers || T < 1 || T > c->max_tokens) return FMOE_ERR_INVALID_ARG;
  if (!same_desc(lw->desc, c->desc)) return FMOE_ERR_INVALID_ARG;
  const fmoe_layer_desc& d = lw->desc;
  // the routed records come from the cache: only the other fields are checked
  if (!lw->shared || !lw->w_router || !lw->w_shared_gate || !lw->norm_w || !aligned16(lw->shared) ||
      !aligned16(lw->w_router) || !aligned16(lw->w_shared_gate) || !aligned16(lw->norm_w))
    return FMOE_ERR_INVALID_ARG;
  if (!d_h || !d_xn || !d_ws || !aligned16(d_h) || !aligned16(d_xn) || !aligned16(d_ws) ||
      (d_logits && !aligned16(d_logits)) || !disjoint(d_h, d_xn, (size_t)T * d.hidden * 4))
    return FMOE_ERR_INVALID_ARG;
  const WsLayout w = ws_layout(d.hidden, d.inter, d.n_experts, d.top_k, T);
  if (ws_bytes < w.bytes) return FMOE_ERR_BUFFER_TOO_SMALL;
  unsigned char* base = static_cast<unsigned char*>(d_ws);
  float* part = reinterpret_cast<float*>(base + w.part);
  float* logits = reinterpret_cast<float*>(base + w.logits);
  int32_t* ids = reinterpret_cast<int32_t*>(base + w.ids);
  float* weights = reinterpret_cast<float*>(base + w.weights);
  float* gamma = reinterpret_cast<float*>(base + w.gamma);
  float* a = reinterpret_cast<float*>(base + w.a);
  float* y = reinterpret_cast<float*>(base + w.y);
  int rc;
  if (d_logits) {
    rc = cuda_rc(cudaMemcpyAsync(logits, d_logits, (size_t)T * d.n_experts * 4, cudaMemcpyDeviceToDevice, st));
    if (rc == FMOE_OK) rc = launch_topk(nullptr, logits, T, d.n_experts, d.top_k, logits, ids, weights, nullptr, st);
  } else {
    rc = launch_router(d_xn, lw->w_router, lw->w_shared_gate, T, d.hidden, d.n_experts, part, st);
    if (rc == FMOE_OK) rc = launch_topk(part, nullptr, T, d.n_experts, d.top_k, logits, ids, weights, gamma, st);
  }
  if (rc != FMOE_OK) return rc;
  // the host learns the step's experts (this is where the step waits)
  const int n = T * d.top_k;
  if (cudaMemcpyAsync(c->h_ids, ids, (size_t)n * 4, cudaMemcpyDeviceToHost, st) != cudaSuccess ||
      cudaStreamSynchronize(st) != cudaSuccess)
    return FMOE_ERR_CUDA;
  const int copies = cache_admit(c, layer, c->h_ids, n, st);
  if (copies == -1) return FMOE_ERR_BUFFER_TOO_SMALL;
  if (copies < 0) return FMOE_ERR_CUDA;
  uint64_t* row = c->d_table + (size_t)layer * d.n_experts;
  if (cudaMemcpyAsync(row, c->h_table + (size_t)layer * d.n_experts, (size_t)d.n_experts * 8, cudaMemcpyHostToDevice,
                      st) != cudaSuccess)
    return FMOE_ERR_CUDA;
  ExpertSet es = expert_set(lw);
  es.experts = nullptr;
  es.rec_table = row;
  const GroupWork gw = group_work(base, w);
  rc = launch_experts(es, d_xn, ids, T, a, y, lw->w_shared_gate, d_logits ? gamma : nullptr, &gw, base + w.tcx,
                      base + w.tca, T > 1 ? base + w.g_xs : nullptr, st);
  if (rc != FMOE_OK) return rc;
  return launch_combine(y, weights, gamma, d_h, lw->norm_w, d.eps, T, d.top_k, d.hidden, d_h, d_xn, st);
}
