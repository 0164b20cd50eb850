// Step 1: top-k expert selection with softmax-renormalised gates.
//
// Each token picks k of E experts (freetoken.wiki, "FreeToken 753b model",
// section "FreeToken 753b Model Explained": 6 of 256); the router is used
// unmodified (ainewsfeed.tech, third paragraph), so the gates are the softmax
// of the selected logits.
//
// One warp per token.  The E logits of the row sit in registers, VPL per lane
// (lane l holds experts l, l+32, ...).  k rounds of a warp arg-max under the
// total order (logit descending, index ascending) pick the experts in output
// order; the owner lane marks its winner taken.  The gate of choice j is
// exp(l_j - l_0) / sum_i exp(l_i - l_0), summed over the k choices.
#include <cfloat>
#include <climits>

#include "common.cuh"

namespace moe {
namespace {

template <int VPL>
__global__ void __launch_bounds__(256) route_topk_kernel(const float* __restrict__ logits, int T, int E,
                                                         int k, int32_t* __restrict__ idx,
                                                         float* __restrict__ gate) {
  pdl_wait();     // idx and gate may still be read by the previous step's combine
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (t >= T) return;
  const float* row = logits + static_cast<size_t>(t) * E;
  float v[VPL];
#pragma unroll
  for (int j = 0; j < VPL; ++j) {
    const int e = lane + 32 * j;
    v[j] = (e < E) ? __ldg(row + e) : 0.0f;
  }
  uint32_t taken = 0;
  float my_v = 0.0f, top = 0.0f;
  int my_e = 0;
  for (int i = 0; i < k; ++i) {
    float bv = 0.0f;
    int be = INT_MAX;   // INT_MAX: no candidate on this lane
#pragma unroll
    for (int j = 0; j < VPL; ++j) {
      const int e = lane + 32 * j;
      const bool ok = (e < E) && !((taken >> j) & 1u);
      if (ok && (be == INT_MAX || v[j] > bv)) {   // strict: the lower index keeps a tie
        bv = v[j];
        be = e;
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const float ov = __shfl_xor_sync(kFull, bv, off);
      const int oe = __shfl_xor_sync(kFull, be, off);
      const bool better = (oe != INT_MAX) &&
                          (be == INT_MAX || ov > bv || (ov == bv && oe < be));
      if (better) {
        bv = ov;
        be = oe;
      }
    }
    if (be != INT_MAX && (be & 31) == lane) taken |= 1u << (be >> 5);
    if (i == 0) top = bv;
    if (lane == i) {
      my_v = bv;
      my_e = be;
    }
  }
  float z = (lane < k) ? expf(my_v - top) : 0.0f;
  float sum = z;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(kFull, sum, off);
  if (lane < k) {
    idx[static_cast<size_t>(t) * k + lane] = my_e;
    gate[static_cast<size_t>(t) * k + lane] = z / sum;
  }
}

template <int VPL>
cudaError_t launch_route(const float* logits, int T, int E, int k, int32_t* idx, float* gate,
                         cudaStream_t s) {
  const int threads = 256;
  const int blocks = (T * 32 + threads - 1) / threads;
  const cudaError_t e = launch_pdl(route_topk_kernel<VPL>, dim3(blocks), dim3(threads), 0, s, logits, T, E, k, idx,
                                   gate);
  return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace
}  // namespace moe

using namespace moe;

moe_status moe::check_route_args(const float* logits, int T, int E, int k, const int32_t* idx, const float* gate) {
  MOE_REQUIRE(T >= 0, "T=%d < 0", T);
  MOE_REQUIRE(E >= 1 && E <= 1024, "E=%d outside [1, 1024]", E);
  MOE_REQUIRE(k >= 1 && k <= E && k <= 32, "k=%d outside [1, min(E, 32)]", k);
  MOE_REQUIRE(T <= (1 << 24) / k, "T*k too large");
  if (T == 0) return MOE_OK;
  MOE_REQUIRE(logits && idx && gate, "null pointer");
  MOE_REQUIRE(aligned(logits, 4) && aligned(idx, 4) && aligned(gate, 4), "misaligned pointer");
  return MOE_OK;
}

extern "C" moe_status moe_route_topk(const float* logits, int T, int E, int k, int32_t* idx,
                                     float* gate, cudaStream_t stream) {
  clear_error();
  moe_status st = check_route_args(logits, T, E, k, idx, gate);
  if (st != MOE_OK || T == 0) return st;
  DeviceInfo dev;
  st = current_device(&dev);
  if (st != MOE_OK) return st;
  cudaError_t err;
  if (E <= 32) err = launch_route<1>(logits, T, E, k, idx, gate, stream);
  else if (E <= 64) err = launch_route<2>(logits, T, E, k, idx, gate, stream);
  else if (E <= 128) err = launch_route<4>(logits, T, E, k, idx, gate, stream);
  else if (E <= 256) err = launch_route<8>(logits, T, E, k, idx, gate, stream);
  else if (E <= 512) err = launch_route<16>(logits, T, E, k, idx, gate, stream);
  else err = launch_route<32>(logits, T, E, k, idx, gate, stream);
  if (err != cudaSuccess) return fail(MOE_ERR_CUDA, "route_topk launch: %s", cudaGetErrorString(err));
  return MOE_OK;
}
