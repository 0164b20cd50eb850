// Step 4: gate-weighted combine with the exact merge of partial sums computed
// elsewhere.  The CPU and GPU shares of a step's experts are summed into one
// result; the split is a scheduling choice, not an approximation
// (explainx.ai hardware guide, section "Decode: decide whether to move an
// expert or compute where it lives"; ainewsfeed.tech, third paragraph).
//
//   out[t][c] = sum_{j=0..k-1, expert on GPU} gate[t][j] * y_perm[inv_perm[t*k+j]][c]
//               + host_partial[t][c]
//
// A pure streaming kernel: each thread owns 4 consecutive columns of one token
// (128-bit loads/stores), adds the k GPU terms in order j = 0..k-1 in fp32,
// then the host partial.  Bytes moved per token: (k_gpu + 1 + 1) * d * 4.
#include "common.cuh"

namespace moe {
namespace {

__global__ void __launch_bounds__(256) combine_kernel(const float* __restrict__ y_perm,
                                                      const int32_t* __restrict__ idx,
                                                      const float* __restrict__ gate,
                                                      const int32_t* __restrict__ inv_perm,
                                                      const int32_t* __restrict__ slot,
                                                      const float* host_partial, int T, int k, int d,
                                                      int E_bound, int nq, float* out) {
  pdl_wait();     // y_perm comes from the FFN launched before
  pdl_trigger();
  const int t = blockIdx.y;
  const int c4 = blockIdx.x * blockDim.x + threadIdx.x;   // index of a float4 in the row
  if (t >= T || c4 * 4 >= d) return;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  // groups of 8 pairs: each level of the index chain (idx -> slot, inv_perm ->
  // y_perm row) is loaded for the whole group before the next, so a token
  // waits on ~4 dependent loads instead of 4 k; the sum keeps the order j = 0..k-1
  for (int j0 = 0; j0 < k; j0 += 8) {
    int e[8], q[8];
    float g[8];
    bool use[8];
#pragma unroll
    for (int jj = 0; jj < 8; ++jj) {
      const int p = t * k + j0 + jj;
      use[jj] = j0 + jj < k;
      e[jj] = use[jj] ? __ldg(idx + p) : 0;
      q[jj] = use[jj] ? __ldg(inv_perm + p) : -1;
      g[jj] = use[jj] ? __ldg(gate + p) : 0.f;
    }
#pragma unroll
    for (int jj = 0; jj < 8; ++jj) {
      if (slot != nullptr && use[jj]) use[jj] = e[jj] >= 0 && e[jj] < E_bound && __ldg(slot + e[jj]) >= 0;
      use[jj] = use[jj] && q[jj] >= 0 && q[jj] < nq;
    }
    float4 y[8];
#pragma unroll
    for (int jj = 0; jj < 8; ++jj)
      y[jj] = use[jj] ? __ldg(reinterpret_cast<const float4*>(y_perm + static_cast<size_t>(q[jj]) * d) + c4)
                      : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int jj = 0; jj < 8; ++jj) {
      if (!use[jj]) continue;
      acc.x = fmaf(g[jj], y[jj].x, acc.x);
      acc.y = fmaf(g[jj], y[jj].y, acc.y);
      acc.z = fmaf(g[jj], y[jj].z, acc.z);
      acc.w = fmaf(g[jj], y[jj].w, acc.w);
    }
  }
  if (host_partial != nullptr) {
    const float4 h = reinterpret_cast<const float4*>(host_partial + static_cast<size_t>(t) * d)[c4];
    acc.x += h.x;
    acc.y += h.y;
    acc.z += h.z;
    acc.w += h.w;
  }
  reinterpret_cast<float4*>(out + static_cast<size_t>(t) * d)[c4] = acc;
}

}  // namespace
}  // namespace moe

using namespace moe;

moe_status moe::check_combine_args(const float* y_perm, const int32_t* idx, const float* gate,
                                   const int32_t* inv_perm, const float* host_partial, int T, int k, int d, int E,
                                   const float* out) {
  MOE_REQUIRE(T >= 0 && k >= 1 && k <= 32 && d >= 4 && d % 4 == 0, "T=%d, k=%d, d=%d", T, k, d);
  MOE_REQUIRE(E >= 1 && E <= 1024, "E=%d outside [1, 1024]", E);
  MOE_REQUIRE(static_cast<long long>(T) * k <= (1 << 24), "T*k too large");
  if (T == 0) return MOE_OK;
  MOE_REQUIRE(y_perm && idx && gate && inv_perm && out, "null pointer");
  MOE_REQUIRE(aligned(y_perm, 16) && aligned(out, 16) && (!host_partial || aligned(host_partial, 16)),
              "y_perm, out and host_partial must be 16-byte aligned");
  MOE_REQUIRE(T <= 65535, "T=%d above the grid limit 65535", T);
  return MOE_OK;
}

extern "C" moe_status moe_combine_merge(const float* y_perm, const int32_t* idx, const float* gate,
                                        const int32_t* inv_perm, const int32_t* slot_of_expert,
                                        const float* host_partial, int T, int k, int d, int E,
                                        float* out, cudaStream_t stream) {
  clear_error();
  moe_status st = check_combine_args(y_perm, idx, gate, inv_perm, host_partial, T, k, d, E, out);
  if (st != MOE_OK || T == 0) return st;
  DeviceInfo dev;
  st = current_device(&dev);
  if (st != MOE_OK) return st;
  const int threads = 256;
  dim3 grid((d / 4 + threads - 1) / threads, T);
  MOE_CUDA_TRY(launch_pdl(combine_kernel, grid, dim3(threads), 0, stream, y_perm, idx, gate, inv_perm,
                          slot_of_expert, host_partial, T, k, d, E, T * k, out));
  MOE_LAUNCH_CHECK("combine_kernel");
  return MOE_OK;
}
