// moe_expert_ffn: argument checks and dispatch between the CUDA-core path
// (bf16/fp32 activations; decode-sized groups) and the FP4 tensor-core path
// (MOE_FFN_ACT_NVFP4: NVFP4 activations x NVFP4 weights on tcgen05).
#include "common.cuh"

namespace moe {
size_t decode_workspace_bytes(moe_shape s, int T, int k);
moe_status launch_ffn_decode(moe_shape s, const void* x, int T, int k, const int32_t* offsets,
                             const int32_t* perm, const int32_t* slot, const void* pool, int n_slots,
                             const float* gate, float* y_perm, float* out, void* ws, int32_t* status,
                             const DeviceInfo& dev, cudaStream_t stream);
size_t prefill_workspace_bytes(moe_shape s, int T, int k);
moe_status launch_ffn_prefill(moe_shape s, const void* x, int T, int k, const int32_t* offsets,
                              const int32_t* perm, const int32_t* slot, const void* pool, int n_slots,
                              const float* gate, float* out, void* ws, int32_t* status,
                              const DeviceInfo& dev, cudaStream_t stream);
}  // namespace moe

using namespace moe;

extern "C" size_t moe_expert_ffn_workspace_bytes(moe_shape s, int T, int k, int flags) {
  if (check_shape(s) != MOE_OK || T < 0 || k < 1 || k > 32) return 0;
  if (flags & MOE_FFN_ACT_NVFP4) return prefill_workspace_bytes(s, T, k);
  return decode_workspace_bytes(s, T, k);
}

extern "C" int moe_expert_ffn_launches(moe_shape s, int T, int k, int flags) {
  if (check_shape(s) != MOE_OK || T <= 0 || k < 1 || k > 32) return 0;
  if (flags & MOE_FFN_ACT_NVFP4) return 4;                 // quantise x, gather, GEMM1, GEMM2
  const int gemvs = decode_one_launch(s.fmt, T) ? 1 : 2;
  if (s.fmt == MOE_W_MXFP4 && mx_tiled(s.d, s.I)) return 1 + gemvs;   // + the split of x into E4M3 terms
  if (s.fmt == MOE_W_BF16 && bf16_blocked(s.d, s.I)) return gemvs;
  return 2;                                                // CUDA-core gate/up, down
}

moe_status moe::check_ffn_args(moe_shape s, const void* x, int T, int k, const int32_t* offsets,
                               const int32_t* perm, const int32_t* slot_of_expert, const void* slot_pool,
                               int n_slots, const float* gate, const float* y_perm, const float* out, int flags,
                               const void* workspace, size_t ws_bytes) {
  moe_status st = check_shape(s);
  if (st != MOE_OK) return st;
  MOE_REQUIRE(T >= 0 && k >= 1 && k <= 32 && k <= s.E, "T=%d, k=%d, E=%d", T, k, s.E);
  MOE_REQUIRE(static_cast<long long>(T) * k <= (1 << 24), "T*k too large");
  MOE_REQUIRE((flags & ~MOE_FFN_ACT_NVFP4) == 0, "unknown flags 0x%x", flags);
  if (T == 0) return MOE_OK;
  MOE_REQUIRE(x && offsets && perm && slot_of_expert && slot_pool, "null pointer");
  MOE_REQUIRE(n_slots >= 1, "n_slots=%d", n_slots);
  MOE_REQUIRE(aligned(x, 16) && aligned(slot_pool, 256) && aligned(offsets, 4) && aligned(perm, 4) &&
                  aligned(slot_of_expert, 4),
              "misaligned pointer (x 16 B, slot_pool 256 B, int arrays 4 B)");
  if (y_perm != nullptr) {
    MOE_REQUIRE(aligned(y_perm, 16), "misaligned y_perm");
  } else {
    MOE_REQUIRE(out != nullptr && gate != nullptr, "y_perm is NULL: out and gate are required");
    MOE_REQUIRE(aligned(out, 16) && aligned(gate, 4), "misaligned out or gate");
  }
  if (flags & MOE_FFN_ACT_NVFP4) {
    MOE_REQUIRE(s.fmt == MOE_W_NVFP4, "MOE_FFN_ACT_NVFP4 needs NVFP4 weights");
    MOE_REQUIRE(y_perm == nullptr, "MOE_FFN_ACT_NVFP4 writes out (fused combine); y_perm must be NULL");
    MOE_REQUIRE(s.d % 256 == 0 && s.I % 256 == 0, "the FP4 tensor-core path needs d, I multiples of 256");
  }
  const size_t need = moe_expert_ffn_workspace_bytes(s, T, k, flags);
  if (need > 0 && (workspace == nullptr || ws_bytes < need))
    return fail(MOE_ERR_CAPACITY, "workspace needs %zu bytes, got %zu", need, ws_bytes);
  MOE_REQUIRE(workspace == nullptr || aligned(workspace, 256), "workspace must be 256-byte aligned");
  return MOE_OK;
}

extern "C" moe_status moe_expert_ffn(moe_shape s, const void* x, int T, int k, const int32_t* offsets,
                                     const int32_t* perm, const int32_t* slot_of_expert,
                                     const void* slot_pool, int n_slots, const float* gate,
                                     float* y_perm, float* out, int flags, void* workspace,
                                     size_t ws_bytes, int32_t* dev_status, cudaStream_t stream) {
  clear_error();
  moe_status st = check_ffn_args(s, x, T, k, offsets, perm, slot_of_expert, slot_pool, n_slots, gate, y_perm,
                                 out, flags, workspace, ws_bytes);
  if (st != MOE_OK || T == 0) return st;
  // every argument check is done: only now touch the device
  DeviceInfo dev;
  st = current_device(&dev);
  if (st != MOE_OK) return st;
  if (flags & MOE_FFN_ACT_NVFP4) {
    return launch_ffn_prefill(s, x, T, k, offsets, perm, slot_of_expert, slot_pool, n_slots, gate, out,
                              workspace, dev_status, dev, stream);
  }
  return launch_ffn_decode(s, x, T, k, offsets, perm, slot_of_expert, slot_pool, n_slots, gate, y_perm,
                           out, workspace, dev_status, dev, stream);
}
