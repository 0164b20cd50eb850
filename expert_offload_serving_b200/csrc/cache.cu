// Step 5: the GPU expert cache -- LRU residency of expert blobs in device
// slots, filled from pinned host pools, shared by the MoE layers of a model.
//
// Pages: a global LRU expert cache in VRAM follows the router and shares its
// decisions across MoE layers (freetoken.wiki "FreeToken 753b model",
// mechanism table, "Global LRU expert cache"; the paragraph after it compares
// its miss rate with per-layer caches of equal capacity); a missed expert is
// copied over PCIe into the GPU cache and kept (explainx.ai hardware guide,
// "Decode"); the host pool is the source of truth and experts sit there in
// their final layout, pinned, so the first request runs from a cold cache;
// the cache can be rebuilt at a safe scheduler point under a new VRAM budget
// without reloading the host pool (futuresignalnews.com, mechanism 3,
// "Elastic Memory Management"; freetoken.wiki, mechanism table, "Elastic
// memory management").
//
// The bookkeeping is host integer state over keys (layer, expert) = l*E + e:
// key_of_slot, last_used, slot_of_key.  One slot pool serves every layer;
// each layer has its own device slot table (slot_of_expert of that layer) and
// its own host pool.  A fill is one cudaMemcpyAsync of the whole blob on the
// caller's side stream after it waits on the event of the last kernel that
// read the pool or a slot table (so an evicted slot is never overwritten
// while a previous kernel still reads it), followed by small kernels that
// apply the slot-table changes in device memory; the caller's main stream
// waits on fill_done.  A resize keeps the most recently used residents,
// moves them device-to-device into the first slots of the new pool and
// rewrites the tables.
#include <algorithm>
#include <vector>

#include "common.cuh"

struct moe_cache {
  moe_shape shape;
  int n_layers;
  int n_slots;
  size_t blob_bytes;
  uint8_t* slot_pool;                        // device
  std::vector<const uint8_t*> host_pools;    // pinned host, one per layer
  std::vector<int32_t*> slot_tables;         // device [E], one per layer
  std::vector<int32_t> key_of_slot, last_used, slot_of_key;
  // set when enqueueing a fill or a resize failed part-way: a copy may have
  // reached a slot whose table entry was never updated, so no later call
  // may trust the device state
  bool broken = false;
  bool plan_only() const { return slot_pool == nullptr; }
};

namespace moe {
namespace {

constexpr int kMaxUpdates = 32;
struct TableUpdates {
  int n;
  int32_t* table[kMaxUpdates];
  int32_t expert[kMaxUpdates];
  int32_t value[kMaxUpdates];
};

__global__ void apply_table_updates(int E, TableUpdates u) {
  // updates are applied in order by one thread: an evicted expert's -1 and a
  // newly resident expert's slot never collide within one call
  if (threadIdx.x == 0 && blockIdx.x == 0)
    for (int i = 0; i < u.n; ++i)
      if (u.expert[i] >= 0 && u.expert[i] < E) u.table[i][u.expert[i]] = u.value[i];
}

// Collects (layer table, expert, value) updates and launches them in batches
// of kMaxUpdates on one stream, in order.
struct UpdateBatch {
  moe_cache* c;
  cudaStream_t stream;
  TableUpdates u{};
  moe_status add(int32_t key, int32_t value) {
    const int E = c->shape.E;
    u.table[u.n] = c->slot_tables[key / E];
    u.expert[u.n] = key % E;
    u.value[u.n++] = value;
    return u.n == kMaxUpdates ? flush() : MOE_OK;
  }
  moe_status flush() {
    if (u.n == 0) return MOE_OK;
    apply_table_updates<<<1, 32, 0, stream>>>(c->shape.E, u);
    MOE_LAUNCH_CHECK("apply_table_updates");
    u.n = 0;
    return MOE_OK;
  }
};

struct Fill {
  int32_t key, s, old;
};

// The copies of a planned fill, then the kernels that write its slot-table
// changes, on `side` after `reads_done`.  That event must follow the last
// kernel of the previous step (or layer) that reads the pool or a slot table
// (the combine reads the table), or a victim slot could be overwritten, or
// its table entry cleared, while that step still uses it.
moe_status enqueue_fills(moe_cache* c, const std::vector<Fill>& plan, cudaStream_t side,
                         cudaEvent_t reads_done) {
  if (reads_done != nullptr) MOE_CUDA_TRY(cudaStreamWaitEvent(side, reads_done, 0));
  const int E = c->shape.E;
  for (const Fill& f : plan)
    MOE_CUDA_TRY(cudaMemcpyAsync(c->slot_pool + static_cast<size_t>(f.s) * c->blob_bytes,
                                 c->host_pools[f.key / E] + static_cast<size_t>(f.key % E) * c->blob_bytes,
                                 c->blob_bytes, cudaMemcpyHostToDevice, side));
  UpdateBatch ub{c, side};
  for (const Fill& f : plan) {
    moe_status st = MOE_OK;
    if (f.old >= 0) st = ub.add(f.old, -1);
    if (st == MOE_OK) st = ub.add(f.key, f.s);
    if (st != MOE_OK) return st;
  }
  return ub.flush();
}

moe_status create(moe_shape s, int n_layers, int n_slots, void* slot_pool, const void* const* host_pools,
                   int32_t* const* slot_tables, moe_cache** out) {
  moe_status st = check_shape(s);
  if (st != MOE_OK) return st;
  MOE_REQUIRE(out != nullptr, "null output handle");
  MOE_REQUIRE(n_layers >= 1 && n_layers <= 4096, "n_layers=%d outside [1, 4096]", n_layers);
  MOE_REQUIRE(n_slots >= 1 && n_slots <= (1 << 20), "n_slots=%d", n_slots);
  const bool plan_only = slot_pool == nullptr && host_pools == nullptr && slot_tables == nullptr;
  if (!plan_only) {
    MOE_REQUIRE(slot_pool && host_pools && slot_tables,
                "slot_pool, host pools and slot tables must all be set (or all NULL)");
    MOE_REQUIRE(aligned(slot_pool, 256), "misaligned slot pool");
    for (int l = 0; l < n_layers; ++l)
      MOE_REQUIRE(host_pools[l] && slot_tables[l] && aligned(host_pools[l], 16) && aligned(slot_tables[l], 4),
                  "layer %d: null or misaligned host pool or slot table", l);
  }
  moe_cache* c = new (std::nothrow) moe_cache();
  if (!c) return fail(MOE_ERR_CAPACITY, "out of host memory");
  c->shape = s;
  c->n_layers = n_layers;
  c->n_slots = n_slots;
  c->blob_bytes = blob_layout(s.fmt, s.d, s.I).bytes;
  c->slot_pool = static_cast<uint8_t*>(slot_pool);
  if (!plan_only)
    for (int l = 0; l < n_layers; ++l) {
      c->host_pools.push_back(static_cast<const uint8_t*>(host_pools[l]));
      c->slot_tables.push_back(slot_tables[l]);
    }
  c->key_of_slot.assign(n_slots, -1);
  c->last_used.assign(n_slots, -1);
  c->slot_of_key.assign(static_cast<size_t>(n_layers) * s.E, -1);
  *out = c;
  return MOE_OK;
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" moe_status moe_cache_create(moe_shape s, int n_slots, void* slot_pool, const void* host_pool,
                                       int32_t* slot_of_expert_dev, moe_cache** out) {
  clear_error();
  const bool none = !slot_pool && !host_pool && !slot_of_expert_dev;
  if (!none)
    MOE_REQUIRE(slot_pool && host_pool && slot_of_expert_dev,
                "slot_pool, host_pool and slot_of_expert_dev must all be set (or all NULL)");
  const void* pools[1] = {host_pool};
  int32_t* tables[1] = {slot_of_expert_dev};
  return create(s, 1, n_slots, slot_pool, none ? nullptr : pools, none ? nullptr : tables, out);
}

extern "C" moe_status moe_cache_create_layers(moe_shape s, int n_layers, int n_slots, void* slot_pool,
                                              const void* const* host_pools, int32_t* const* slot_tables_dev,
                                              moe_cache** out) {
  clear_error();
  return create(s, n_layers, n_slots, slot_pool, host_pools, slot_tables_dev, out);
}

extern "C" moe_status moe_cache_destroy(moe_cache* c) {
  delete c;
  return MOE_OK;
}

extern "C" moe_status moe_cache_query(const moe_cache* c, int32_t* slot_of_expert, int32_t* expert_of_slot,
                                      int32_t* last_used) {
  clear_error();
  MOE_REQUIRE(c != nullptr, "null cache");
  if (slot_of_expert) std::copy(c->slot_of_key.begin(), c->slot_of_key.end(), slot_of_expert);
  if (expert_of_slot) std::copy(c->key_of_slot.begin(), c->key_of_slot.end(), expert_of_slot);
  if (last_used) std::copy(c->last_used.begin(), c->last_used.end(), last_used);
  return MOE_OK;
}

extern "C" moe_status moe_cache_fill_layer(moe_cache* c, int layer, const int32_t* experts, int n, int step,
                                           const int32_t* protect, int n_protect, cudaStream_t side,
                                           cudaEvent_t reads_done, cudaEvent_t fill_done, int32_t* fills,
                                           int32_t* n_fills) {
  clear_error();
  MOE_REQUIRE(c != nullptr, "null cache");
  if (c->broken)
    return fail(MOE_ERR_CUDA, "an earlier fill or resize failed part-way; the device slots are undefined: "
                              "recreate the cache");
  MOE_REQUIRE(layer >= 0 && layer < c->n_layers, "layer %d outside [0, %d)", layer, c->n_layers);
  MOE_REQUIRE(n >= 0 && n_protect >= 0, "negative count");
  MOE_REQUIRE(n == 0 || experts != nullptr, "null experts");
  MOE_REQUIRE(n_protect == 0 || protect != nullptr, "null protect list");
  const int E = c->shape.E;
  const int32_t base = layer * E;
  std::vector<int32_t> want(experts, experts + n);
  for (int32_t e : want) MOE_REQUIRE(e >= 0 && e < E, "expert id %d outside [0, %d)", e, E);
  std::sort(want.begin(), want.end());
  want.erase(std::unique(want.begin(), want.end()), want.end());
  std::vector<char> prot(c->slot_of_key.size(), 0);
  for (int32_t e : want) prot[base + e] = 1;
  for (int i = 0; i < n_protect; ++i) {
    MOE_REQUIRE(protect[i] >= 0 && protect[i] < E, "protected id %d outside [0, %d)", protect[i], E);
    prot[base + protect[i]] = 1;
  }
  // plan on copies so that a capacity failure leaves the cache unchanged
  std::vector<int32_t> kos = c->key_of_slot, lu = c->last_used, sok = c->slot_of_key;
  for (int32_t e : want)
    if (sok[base + e] >= 0) lu[sok[base + e]] = step;
  std::vector<Fill> plan;
  for (int32_t e : want) {
    const int32_t key = base + e;
    if (sok[key] >= 0) continue;
    int s = -1;
    for (int q = 0; q < c->n_slots; ++q)
      if (kos[q] < 0) { s = q; break; }
    if (s < 0) {
      for (int q = 0; q < c->n_slots; ++q) {
        if (prot[kos[q]]) continue;
        if (s < 0 || lu[q] < lu[s]) s = q;   // strict: ties keep the lower slot
      }
    }
    if (s < 0)
      return fail(MOE_ERR_CAPACITY, "step %d: %zu experts to hold but no evictable slot among %d",
                  step, want.size(), c->n_slots);
    const int32_t old = kos[s];
    if (old >= 0) sok[old] = -1;
    kos[s] = key;
    sok[key] = s;
    lu[s] = step;
    plan.push_back({key, s, old});
  }
  // enqueue the copies and the slot-table updates
  if (!c->plan_only()) {
    moe_status st = plan.empty() ? MOE_OK : enqueue_fills(c, plan, side, reads_done);
    if (st == MOE_OK && fill_done != nullptr) {
      const cudaError_t e = cudaEventRecord(fill_done, side);
      if (e != cudaSuccess) st = fail(MOE_ERR_CUDA, "cudaEventRecord(fill_done) failed: %s", cudaGetErrorString(e));
    }
    if (st != MOE_OK) {
      c->broken = !plan.empty();
      return st;
    }
  }
  c->key_of_slot.swap(kos);
  c->last_used.swap(lu);
  c->slot_of_key.swap(sok);
  if (fills)
    for (size_t i = 0; i < plan.size(); ++i) {
      fills[3 * i] = plan[i].key - base;
      fills[3 * i + 1] = plan[i].s;
      fills[3 * i + 2] = plan[i].old;       // a key: layer * E + expert (the expert itself with one layer)
    }
  if (n_fills) *n_fills = static_cast<int32_t>(plan.size());
  return MOE_OK;
}

extern "C" moe_status moe_cache_fill(moe_cache* c, const int32_t* experts, int n, int step,
                                     const int32_t* protect, int n_protect, cudaStream_t side,
                                     cudaEvent_t reads_done, cudaEvent_t fill_done, int32_t* fills,
                                     int32_t* n_fills) {
  return moe_cache_fill_layer(c, 0, experts, n, step, protect, n_protect, side, reads_done, fill_done, fills,
                              n_fills);
}

extern "C" moe_status moe_cache_resize(moe_cache* c, int new_n_slots, void* new_slot_pool, cudaStream_t stream,
                                       cudaEvent_t reads_done, int32_t* kept, int32_t* n_kept) {
  clear_error();
  MOE_REQUIRE(c != nullptr, "null cache");
  if (c->broken) return fail(MOE_ERR_CUDA, "an earlier fill or resize failed part-way: recreate the cache");
  MOE_REQUIRE(new_n_slots >= 1 && new_n_slots <= (1 << 20), "new_n_slots=%d", new_n_slots);
  if (!c->plan_only()) {
    MOE_REQUIRE(new_slot_pool != nullptr && aligned(new_slot_pool, 256), "null or misaligned new slot pool");
    MOE_REQUIRE(new_slot_pool != c->slot_pool || new_n_slots <= c->n_slots,
                "growing in place: pass a new pool of new_n_slots blobs");
  }
  // residents ranked by recency (last_used descending, lower slot first)
  std::vector<int> res;
  for (int q = 0; q < c->n_slots; ++q)
    if (c->key_of_slot[q] >= 0) res.push_back(q);
  std::stable_sort(res.begin(), res.end(), [&](int a, int b) { return c->last_used[a] > c->last_used[b]; });
  const size_t n_keep = std::min(res.size(), static_cast<size_t>(new_n_slots));
  std::vector<int> keep(res.begin(), res.begin() + n_keep), drop(res.begin() + n_keep, res.end());
  std::sort(keep.begin(), keep.end());        // the kept move down in their slot order
  std::vector<int32_t> kos(new_n_slots, -1), lu(new_n_slots, -1), sok = c->slot_of_key;
  for (int q : drop) sok[c->key_of_slot[q]] = -1;
  for (size_t j = 0; j < keep.size(); ++j) {
    const int q = keep[j];
    kos[j] = c->key_of_slot[q];
    lu[j] = c->last_used[q];
    sok[kos[j]] = static_cast<int32_t>(j);
  }
  if (!c->plan_only()) {
    uint8_t* dst = static_cast<uint8_t*>(new_slot_pool);
    const bool same = dst == c->slot_pool;
    moe_status st = MOE_OK;
    cudaError_t e = cudaSuccess;
    if (reads_done != nullptr) e = cudaStreamWaitEvent(stream, reads_done, 0);
    // slot j <= keep[j]: in place, a copy never reads a slot an earlier copy wrote
    for (size_t j = 0; j < keep.size() && e == cudaSuccess; ++j)
      if (!same || static_cast<int>(j) != keep[j])
        e = cudaMemcpyAsync(dst + j * c->blob_bytes, c->slot_pool + static_cast<size_t>(keep[j]) * c->blob_bytes,
                            c->blob_bytes, cudaMemcpyDeviceToDevice, stream);
    if (e != cudaSuccess) st = fail(MOE_ERR_CUDA, "resize copy failed: %s", cudaGetErrorString(e));
    UpdateBatch ub{c, stream};
    for (int q : drop)
      if (st == MOE_OK) st = ub.add(c->key_of_slot[q], -1);
    for (size_t j = 0; j < keep.size() && st == MOE_OK; ++j)
      if (!same || static_cast<int>(j) != keep[j]) st = ub.add(kos[j], static_cast<int32_t>(j));
    if (st == MOE_OK) st = ub.flush();
    if (st != MOE_OK) {
      c->broken = true;
      return st;
    }
    c->slot_pool = dst;
  }
  if (kept)
    for (size_t j = 0; j < keep.size(); ++j) {
      kept[2 * j] = kos[j];
      kept[2 * j + 1] = keep[j];
    }
  if (n_kept) *n_kept = static_cast<int32_t>(keep.size());
  c->n_slots = new_n_slots;
  c->key_of_slot.swap(kos);
  c->last_used.swap(lu);
  c->slot_of_key.swap(sok);
  return MOE_OK;
}

extern "C" moe_status moe_check_status(int32_t* dev_status, cudaStream_t stream) {
  clear_error();
  MOE_REQUIRE(dev_status != nullptr, "null status word");
  int32_t h = 0;
  MOE_CUDA_TRY(cudaMemcpyAsync(&h, dev_status, sizeof(h), cudaMemcpyDeviceToHost, stream));
  MOE_CUDA_TRY(cudaStreamSynchronize(stream));
  MOE_CUDA_TRY(cudaMemsetAsync(dev_status, 0, sizeof(int32_t), stream));
  MOE_CUDA_TRY(cudaStreamSynchronize(stream));
  if (h == 0) return MOE_OK;
  if (h == MOE_ERR_DEVICE) return fail(MOE_ERR_DEVICE, "a kernel met an out-of-range index");
  if (h == MOE_ERR_TIMEOUT) return fail(MOE_ERR_TIMEOUT, "a bounded device wait ran out");
  return fail(static_cast<moe_status>(h), "device status %d", h);
}
