// moe_layer_forward: the layer's four steps from one host call (route ->
// permute -> expert FFN -> combine, or the FFN's fused combine), enqueued on
// one stream.  Every step's arguments are checked before the first one is
// enqueued, so a rejected call leaves the stream untouched; each step is then
// the public entry point itself, so checks and results are exactly those of
// the individual calls.
#include "common.cuh"

extern "C" moe_status moe_layer_forward(moe_shape s, const float* logits, const void* x, int T, int k,
                                        int32_t* idx, float* gate, int32_t* offsets, int32_t* perm,
                                        int32_t* inv_perm, void* scratch, size_t scratch_bytes,
                                        const int32_t* slot_of_expert, const void* slot_pool, int n_slots,
                                        float* y_perm, int flags, void* workspace, size_t ws_bytes,
                                        const float* host_partial, float* out, int32_t* dev_status,
                                        cudaStream_t stream) {
  ::moe::clear_error();
  const bool fused = (flags & MOE_FFN_ACT_NVFP4) != 0;
  moe_status st = ::moe::check_route_args(logits, T, s.E, k, idx, gate);
  if (st == MOE_OK) st = ::moe::check_permute_args(idx, T, k, s.E, offsets, perm, inv_perm, scratch, scratch_bytes);
  if (st == MOE_OK)
    st = ::moe::check_ffn_args(s, x, T, k, offsets, perm, slot_of_expert, slot_pool, n_slots, gate,
                        fused ? nullptr : y_perm, fused ? out : nullptr, flags, workspace, ws_bytes);
  if (st == MOE_OK && !fused)
    st = ::moe::check_combine_args(y_perm, idx, gate, inv_perm, host_partial, T, k, s.d, s.E, out);
  if (st != MOE_OK) return st;
  if (fused) MOE_REQUIRE(out != nullptr, "out is required");
  st = moe_route_topk(logits, T, s.E, k, idx, gate, stream);
  if (st != MOE_OK) return st;
  st = moe_permute(idx, T, k, s.E, offsets, perm, inv_perm, scratch, scratch_bytes, dev_status, stream);
  if (st != MOE_OK) return st;
  if (fused) {
    ::moe::clear_error();
    if (T > 0) {
      const size_t bytes = static_cast<size_t>(T) * s.d * sizeof(float);
      if (host_partial != nullptr) {
        if (host_partial != out)
          MOE_CUDA_TRY(cudaMemcpyAsync(out, host_partial, bytes, cudaMemcpyDeviceToDevice, stream));
      } else {
        MOE_CUDA_TRY(cudaMemsetAsync(out, 0, bytes, stream));
      }
    }
    return moe_expert_ffn(s, x, T, k, offsets, perm, slot_of_expert, slot_pool, n_slots, gate, nullptr, out, flags,
                          workspace, ws_bytes, dev_status, stream);
  }
  st = moe_expert_ffn(s, x, T, k, offsets, perm, slot_of_expert, slot_pool, n_slots, gate, y_perm, nullptr, flags,
                      workspace, ws_bytes, dev_status, stream);
  if (st != MOE_OK) return st;
  return moe_combine_merge(y_perm, idx, gate, inv_perm, slot_of_expert, host_partial, T, k, s.d, s.E, out, stream);
}
