// Step 3 (FP4 tensor-core path, MOE_FFN_ACT_NVFP4): not built yet.
#include "common.cuh"

namespace moe {

size_t prefill_workspace_bytes(moe_shape s, int T, int k) {
  (void)s;
  (void)T;
  (void)k;
  return 0;
}

moe_status launch_ffn_prefill(moe_shape, const void*, int, int, const int32_t*, const int32_t*,
                              const int32_t*, const void*, int, const float*, float*, void*, int32_t*,
                              const DeviceInfo&, cudaStream_t) {
  return fail(MOE_ERR_UNSUPPORTED, "the NVFP4 tensor-core path is not built in this version");
}

}  // namespace moe
