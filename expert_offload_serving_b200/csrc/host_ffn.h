// Host-side expert FFN (the CPU share of a step's cache misses): interface
// between the host-compiled kernel (host_ffn.cc) and the C entry points.
#pragma once

#include <cstddef>
#include <cstdint>
#include <vector>

#include "layout.h"

namespace moe {
namespace host {

// One host-computed expert and its pairs: token row and gate of each.
struct HostPairs {
  int expert;
  std::vector<int> tok;
  std::vector<float> gate;
};

// out[t][c] (fp32 [T][d], overwritten) = sum over the listed experts' pairs of
// gate * SwiGLU_e(x[t])[c]; x is fp32 [T][d]; expert e's blob is at
// host_pool + e * blob_bytes.  Runs on `threads` threads (the caller included).
void expert_ffn(moe_shape s, const uint8_t* host_pool, size_t blob_bytes, const std::vector<HostPairs>& experts,
                const float* x, int T, float* out, int threads);

int default_threads();

}  // namespace host
}  // namespace moe
