// Step 5: the GPU expert cache -- LRU residency of expert blobs in device
// slots, filled from a pinned host pool.
//
// Pages: a global LRU expert cache in VRAM follows the router (freetoken.wiki
// "FreeToken 753b model", mechanism table; explainx.ai hardware guide,
// "Decode": a missed expert is copied over PCIe into the GPU cache and kept);
// the host pool is the source of truth and experts sit there in their final
// layout, pinned, so the first request runs from a cold cache
// (futuresignalnews.com, mechanism 3).
//
// The bookkeeping is host integer state (expert_of_slot, last_used,
// slot_of_expert).  A fill is one cudaMemcpyAsync of the whole blob on the
// caller's side stream after it waits on the event of the last kernel that
// read the pool (so an evicted slot is never overwritten while a previous FFN
// still reads it), followed by one small kernel that applies the slot-table
// changes in device memory; the caller's main stream waits on fill_done.
#include <algorithm>
#include <vector>

#include "common.cuh"

struct moe_cache {
  moe_shape shape;
  int n_slots;
  size_t blob_bytes;
  uint8_t* slot_pool;          // device
  const uint8_t* host_pool;    // pinned host
  int32_t* slot_table_dev;     // device [E]
  std::vector<int32_t> expert_of_slot, last_used, slot_of_expert;
  // set when enqueueing a fill failed part-way: a copy may have reached a
  // victim slot whose table entry was never updated, so no later fill or FFN
  // may trust the device state
  bool broken = false;
};

namespace moe {
namespace {

constexpr int kMaxUpdates = 32;
struct TableUpdates {
  int n;
  int32_t expert[kMaxUpdates];
  int32_t value[kMaxUpdates];
};

__global__ void apply_table_updates(int32_t* table, int E, TableUpdates u) {
  // updates are applied in order by one thread: an evicted expert's -1 and a
  // newly resident expert's slot never collide within one call
  if (threadIdx.x == 0 && blockIdx.x == 0)
    for (int i = 0; i < u.n; ++i)
      if (u.expert[i] >= 0 && u.expert[i] < E) table[u.expert[i]] = u.value[i];
}

struct Fill {
  int32_t e, s, old;
};

// The copies of a planned fill, then the kernels that write its slot-table
// changes, on `side` after `reads_done`.  That event must follow the last
// kernel of the previous step that reads the pool or the slot table (the
// combine reads the table), or a victim slot could be overwritten, or its
// table entry cleared, while that step still uses it.
moe_status enqueue_fills(moe_cache* c, const std::vector<Fill>& plan, cudaStream_t side,
                         cudaEvent_t reads_done) {
  if (reads_done != nullptr) MOE_CUDA_TRY(cudaStreamWaitEvent(side, reads_done, 0));
  for (const Fill& f : plan)
    MOE_CUDA_TRY(cudaMemcpyAsync(c->slot_pool + static_cast<size_t>(f.s) * c->blob_bytes,
                                 c->host_pool + static_cast<size_t>(f.e) * c->blob_bytes, c->blob_bytes,
                                 cudaMemcpyHostToDevice, side));
  TableUpdates u{};
  for (size_t i = 0; i < plan.size(); ++i) {
    if (plan[i].old >= 0) {
      u.expert[u.n] = plan[i].old;
      u.value[u.n++] = -1;
    }
    u.expert[u.n] = plan[i].e;
    u.value[u.n++] = plan[i].s;
    if (u.n > kMaxUpdates - 2 || i + 1 == plan.size()) {
      apply_table_updates<<<1, 32, 0, side>>>(c->slot_table_dev, c->shape.E, u);
      MOE_LAUNCH_CHECK("apply_table_updates");
      u.n = 0;
    }
  }
  return MOE_OK;
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" moe_status moe_cache_create(moe_shape s, int n_slots, void* slot_pool, const void* host_pool,
                                       int32_t* slot_of_expert_dev, moe_cache** out) {
  clear_error();
  moe_status st = check_shape(s);
  if (st != MOE_OK) return st;
  MOE_REQUIRE(out != nullptr, "null output handle");
  MOE_REQUIRE(n_slots >= 1 && n_slots <= (1 << 20), "n_slots=%d", n_slots);
  const bool plan_only = !slot_pool && !host_pool && !slot_of_expert_dev;
  if (!plan_only) {
    MOE_REQUIRE(slot_pool && host_pool && slot_of_expert_dev,
                "slot_pool, host_pool and slot_of_expert_dev must all be set (or all NULL)");
    MOE_REQUIRE(aligned(slot_pool, 256) && aligned(host_pool, 16) && aligned(slot_of_expert_dev, 4),
                "misaligned pool or slot table");
  }
  moe_cache* c = new (std::nothrow) moe_cache();
  if (!c) return fail(MOE_ERR_CAPACITY, "out of host memory");
  c->shape = s;
  c->n_slots = n_slots;
  c->blob_bytes = blob_layout(s.fmt, s.d, s.I).bytes;
  c->slot_pool = static_cast<uint8_t*>(slot_pool);
  c->host_pool = static_cast<const uint8_t*>(host_pool);
  c->slot_table_dev = slot_of_expert_dev;
  c->expert_of_slot.assign(n_slots, -1);
  c->last_used.assign(n_slots, -1);
  c->slot_of_expert.assign(s.E, -1);
  *out = c;
  return MOE_OK;
}

extern "C" moe_status moe_cache_destroy(moe_cache* c) {
  delete c;
  return MOE_OK;
}

extern "C" moe_status moe_cache_query(const moe_cache* c, int32_t* slot_of_expert, int32_t* expert_of_slot,
                                      int32_t* last_used) {
  clear_error();
  MOE_REQUIRE(c != nullptr, "null cache");
  if (slot_of_expert) std::copy(c->slot_of_expert.begin(), c->slot_of_expert.end(), slot_of_expert);
  if (expert_of_slot) std::copy(c->expert_of_slot.begin(), c->expert_of_slot.end(), expert_of_slot);
  if (last_used) std::copy(c->last_used.begin(), c->last_used.end(), last_used);
  return MOE_OK;
}

extern "C" moe_status moe_cache_fill(moe_cache* c, const int32_t* experts, int n, int step,
                                     const int32_t* protect, int n_protect, cudaStream_t side,
                                     cudaEvent_t reads_done, cudaEvent_t fill_done, int32_t* fills,
                                     int32_t* n_fills) {
  clear_error();
  MOE_REQUIRE(c != nullptr, "null cache");
  if (c->broken)
    return fail(MOE_ERR_CUDA, "an earlier fill failed part-way; the device slots are undefined: recreate the cache");
  MOE_REQUIRE(n >= 0 && n_protect >= 0, "negative count");
  MOE_REQUIRE(n == 0 || experts != nullptr, "null experts");
  MOE_REQUIRE(n_protect == 0 || protect != nullptr, "null protect list");
  const int E = c->shape.E;
  std::vector<int32_t> want(experts, experts + n);
  for (int32_t e : want) MOE_REQUIRE(e >= 0 && e < E, "expert id %d outside [0, %d)", e, E);
  std::sort(want.begin(), want.end());
  want.erase(std::unique(want.begin(), want.end()), want.end());
  std::vector<char> prot(E, 0);
  for (int32_t e : want) prot[e] = 1;
  for (int i = 0; i < n_protect; ++i) {
    MOE_REQUIRE(protect[i] >= 0 && protect[i] < E, "protected id %d outside [0, %d)", protect[i], E);
    prot[protect[i]] = 1;
  }
  // plan on copies so that a capacity failure leaves the cache unchanged
  std::vector<int32_t> eos = c->expert_of_slot, lu = c->last_used, soe = c->slot_of_expert;
  for (int32_t e : want)
    if (soe[e] >= 0) lu[soe[e]] = step;
  std::vector<Fill> plan;
  for (int32_t e : want) {
    if (soe[e] >= 0) continue;
    int s = -1;
    for (int q = 0; q < c->n_slots; ++q)
      if (eos[q] < 0) { s = q; break; }
    if (s < 0) {
      for (int q = 0; q < c->n_slots; ++q) {
        if (prot[eos[q]]) continue;
        if (s < 0 || lu[q] < lu[s]) s = q;   // strict: ties keep the lower slot
      }
    }
    if (s < 0)
      return fail(MOE_ERR_CAPACITY, "step %d: %zu experts to hold but no evictable slot among %d",
                  step, want.size(), c->n_slots);
    const int32_t old = eos[s];
    if (old >= 0) soe[old] = -1;
    eos[s] = e;
    soe[e] = s;
    lu[s] = step;
    plan.push_back({e, s, old});
  }
  // enqueue the copies and the slot-table updates
  if (c->slot_pool != nullptr) {
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
  c->expert_of_slot.swap(eos);
  c->last_used.swap(lu);
  c->slot_of_expert.swap(soe);
  if (fills)
    for (size_t i = 0; i < plan.size(); ++i) {
      fills[3 * i] = plan[i].e;
      fills[3 * i + 1] = plan[i].s;
      fills[3 * i + 2] = plan[i].old;
    }
  if (n_fills) *n_fills = static_cast<int32_t>(plan.size());
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
