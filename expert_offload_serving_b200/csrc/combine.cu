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
  const int t = blockIdx.y;
  const int c4 = blockIdx.x * blockDim.x + threadIdx.x;   // index of a float4 in the row
  if (t >= T || c4 * 4 >= d) return;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int j = 0; j < k; ++j) {
    const int p = t * k + j;
    const int e = __ldg(idx + p);
    if (slot != nullptr) {
      if (e < 0 || e >= E_bound) continue;
      if (__ldg(slot + e) < 0) continue;
    }
    const int q = __ldg(inv_perm + p);
    if (q < 0 || q >= nq) continue;
    const float g = __ldg(gate + p);
    const float4 y = __ldg(reinterpret_cast<const float4*>(y_perm + static_cast<size_t>(q) * d) + c4);
    acc.x = fmaf(g, y.x, acc.x);
    acc.y = fmaf(g, y.y, acc.y);
    acc.z = fmaf(g, y.z, acc.z);
    acc.w = fmaf(g, y.w, acc.w);
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

extern "C" moe_status moe_combine_merge(const float* y_perm, const int32_t* idx, const float* gate,
                                        const int32_t* inv_perm, const int32_t* slot_of_expert,
                                        const float* host_partial, int T, int k, int d, int E,
                                        float* out, cudaStream_t stream) {
  clear_error();
  MOE_REQUIRE(T >= 0 && k >= 1 && k <= 32 && d >= 4 && d % 4 == 0, "T=%d, k=%d, d=%d", T, k, d);
  MOE_REQUIRE(E >= 1 && E <= 1024, "E=%d outside [1, 1024]", E);
  MOE_REQUIRE(static_cast<long long>(T) * k <= (1 << 24), "T*k too large");
  if (T == 0) return MOE_OK;
  MOE_REQUIRE(y_perm && idx && gate && inv_perm && out, "null pointer");
  MOE_REQUIRE(aligned(y_perm, 16) && aligned(out, 16) && (!host_partial || aligned(host_partial, 16)),
              "y_perm, out and host_partial must be 16-byte aligned");
  MOE_REQUIRE(T <= 65535, "T=%d above the grid limit 65535", T);
  DeviceInfo dev;
  moe_status st = current_device(&dev);
  if (st != MOE_OK) return st;
  const int threads = 256;
  dim3 grid((d / 4 + threads - 1) / threads, T);
  combine_kernel<<<grid, threads, 0, stream>>>(y_perm, idx, gate, inv_perm, slot_of_expert,
                                               host_partial, T, k, d, E, T * k, out);
  MOE_LAUNCH_CHECK("combine_kernel");
  return MOE_OK;
}
