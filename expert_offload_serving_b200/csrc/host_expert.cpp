// C entry points of the host share of a decode step: the host expert FFN over
// the pinned host pool, and the bandwidth profile the q* split is computed
// from (freetoken.wiki "FreeToken 753b model", "Measure System Bandwidth": the
// runtime profiles PCIe transfer bandwidth and host-memory bandwidth and
// splits cache misses by them; explainx.ai hardware guide, "Decode": both
// paths run at once and their partial sums merge exactly).
#include <algorithm>
#include <chrono>
#include <cstring>
#include <vector>

#include "common.cuh"
#include "host_ffn.h"

using namespace moe;

namespace {

moe_status gather_pairs(moe_shape s, const int32_t* experts, int n_experts, const int32_t* idx, const float* gate,
                        int T, int k, std::vector<host::HostPairs>* out) {
  // distinct ids in ascending order: the fp32 sums do not depend on how the
  // caller lists the experts
  std::vector<char> listed(s.E, 0);
  for (int i = 0; i < n_experts; ++i) {
    const int e = experts[i];
    MOE_REQUIRE(e >= 0 && e < s.E, "expert id %d outside [0, %d)", e, s.E);
    listed[e] = 1;
  }
  std::vector<int> slot_of(s.E, -1);
  for (int e = 0; e < s.E; ++e)
    if (listed[e]) {
      slot_of[e] = static_cast<int>(out->size());
      out->push_back(host::HostPairs{e, {}, {}});
    }
  for (int t = 0; t < T; ++t)
    for (int j = 0; j < k; ++j) {
      const int e = idx[static_cast<size_t>(t) * k + j];
      MOE_REQUIRE(e >= 0 && e < s.E, "idx[%d][%d] = %d outside [0, %d)", t, j, e, s.E);
      if (slot_of[e] >= 0) {
        (*out)[slot_of[e]].tok.push_back(t);
        (*out)[slot_of[e]].gate.push_back(gate[static_cast<size_t>(t) * k + j]);
      }
    }
  // experts without pairs in this step cost nothing
  out->erase(std::remove_if(out->begin(), out->end(), [](const host::HostPairs& p) { return p.tok.empty(); }),
             out->end());
  return MOE_OK;
}

int clamp_threads(int n_threads) {
  const int hw = host::default_threads();
  return n_threads <= 0 ? hw : std::min(n_threads, hw);
}

}  // namespace

extern "C" moe_status moe_host_expert_ffn(moe_shape s, const void* host_pool, const int32_t* experts,
                                          int n_experts, const void* x, const int32_t* idx, const float* gate,
                                          int T, int k, float* out, int n_threads) {
  clear_error();
  moe_status st = check_shape(s);
  if (st != MOE_OK) return st;
  MOE_REQUIRE(T >= 0 && k >= 1 && k <= 32 && k <= s.E, "T=%d, k=%d, E=%d", T, k, s.E);
  MOE_REQUIRE(n_experts >= 0, "n_experts=%d", n_experts);
  if (T == 0) return MOE_OK;
  MOE_REQUIRE(host_pool && x && idx && gate && out, "null pointer");
  MOE_REQUIRE(n_experts == 0 || experts != nullptr, "null expert list");
  std::vector<host::HostPairs> pairs;
  st = gather_pairs(s, experts, n_experts, idx, gate, T, k, &pairs);
  if (st != MOE_OK) return st;
  // bf16 activations -> fp32 once per token
  std::vector<float> xf(static_cast<size_t>(T) * s.d);
  const uint16_t* xb = static_cast<const uint16_t*>(x);
  for (size_t i = 0; i < xf.size(); ++i) {
    const uint32_t bits = static_cast<uint32_t>(xb[i]) << 16;
    std::memcpy(&xf[i], &bits, 4);
  }
  const size_t B = blob_layout(s.fmt, s.d, s.I).bytes;
  host::expert_ffn(s, static_cast<const uint8_t*>(host_pool), B, pairs, xf.data(), T, out, clamp_threads(n_threads));
  return MOE_OK;
}

extern "C" moe_status moe_profile_bandwidth(moe_shape s, const void* host_pool, int n_blobs, void* dev_buf,
                                            size_t dev_bytes, int n_threads, cudaStream_t stream, double* h2d_gbs,
                                            double* host_gbs) {
  clear_error();
  moe_status st = check_shape(s);
  if (st != MOE_OK) return st;
  const size_t B = blob_layout(s.fmt, s.d, s.I).bytes;
  MOE_REQUIRE(n_blobs >= 1 && n_blobs <= s.E, "n_blobs=%d outside [1, E=%d]", n_blobs, s.E);
  MOE_REQUIRE(host_pool && h2d_gbs && host_gbs, "null pointer");
  MOE_REQUIRE(dev_buf == nullptr || (aligned(dev_buf, 256) && dev_bytes >= B),
              "dev_buf must be 256-byte aligned and hold one blob (%zu bytes)", B);
  const uint8_t* pool = static_cast<const uint8_t*>(host_pool);
  *h2d_gbs = 0.0;
  if (dev_buf != nullptr) {
    // pinned host -> device, whole blobs, timed on the stream with events
    const size_t slots = dev_bytes / B;
    cudaEvent_t e0, e1;
    MOE_CUDA_TRY(cudaEventCreate(&e0));
    MOE_CUDA_TRY(cudaEventCreate(&e1));
    auto copy = [&](int i) {
      return cudaMemcpyAsync(static_cast<uint8_t*>(dev_buf) + (i % slots) * B, pool + static_cast<size_t>(i) * B, B,
                             cudaMemcpyHostToDevice, stream);
    };
    cudaError_t err = copy(0);                                  // warm-up
    if (err == cudaSuccess) err = cudaEventRecord(e0, stream);
    for (int i = 0; i < n_blobs && err == cudaSuccess; ++i) err = copy(i);
    if (err == cudaSuccess) err = cudaEventRecord(e1, stream);
    if (err == cudaSuccess) err = cudaEventSynchronize(e1);
    float ms = 0.f;
    if (err == cudaSuccess) err = cudaEventElapsedTime(&ms, e0, e1);
    cudaEventDestroy(e0);
    cudaEventDestroy(e1);
    if (err != cudaSuccess) return fail(MOE_ERR_CUDA, "bandwidth profile copy failed: %s", cudaGetErrorString(err));
    *h2d_gbs = static_cast<double>(n_blobs) * B / (ms * 1e-3) / 1e9;
  }
  // host expert kernel: one token through each of the first n_blobs experts
  std::vector<float> x(s.d, 0.01f), out(s.d);
  std::vector<host::HostPairs> pairs;
  for (int e = 0; e < n_blobs; ++e) pairs.push_back(host::HostPairs{e, {0}, {1.0f}});
  const int th = clamp_threads(n_threads);
  std::vector<host::HostPairs> warm(pairs.begin(), pairs.begin() + 1);
  host::expert_ffn(s, pool, B, warm, x.data(), 1, out.data(), th);
  const auto t0 = std::chrono::steady_clock::now();
  host::expert_ffn(s, pool, B, pairs, x.data(), 1, out.data(), th);
  const double sec = std::chrono::duration<double>(std::chrono::steady_clock::now() - t0).count();
  *host_gbs = static_cast<double>(n_blobs) * B / sec / 1e9;
  return MOE_OK;
}
