// Shared definitions of libmoe: error reporting, argument checks, the expert
// blob layout, and small device helpers.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/moe.h"
#include "layout.h"

namespace moe {

// ---------------------------------------------------------------- errors
moe_status fail(moe_status st, const char* fmt, ...);
void clear_error();

#define MOE_REQUIRE(cond, ...)                                   \
  do {                                                           \
    if (!(cond)) return ::moe::fail(MOE_ERR_INVALID_ARG, __VA_ARGS__); \
  } while (0)

#define MOE_CUDA_TRY(call)                                                        \
  do {                                                                            \
    cudaError_t e_ = (call);                                                      \
    if (e_ != cudaSuccess)                                                        \
      return ::moe::fail(MOE_ERR_CUDA, "%s failed: %s", #call, cudaGetErrorString(e_)); \
  } while (0)

#define MOE_LAUNCH_CHECK(what)                                                    \
  do {                                                                            \
    cudaError_t e_ = cudaGetLastError();                                          \
    if (e_ != cudaSuccess)                                                        \
      return ::moe::fail(MOE_ERR_CUDA, "launch of %s failed: %s", what, cudaGetErrorString(e_)); \
  } while (0)

inline bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Argument checks of the four steps.  They touch no device: each entry point
// runs its own before the first CUDA call, and moe_layer_forward runs all four
// before it enqueues anything.
moe_status check_route_args(const float* logits, int T, int E, int k, const int32_t* idx, const float* gate);
moe_status check_permute_args(const int32_t* idx, int T, int k, int E, const int32_t* offsets,
                              const int32_t* perm, const int32_t* inv_perm, const void* scratch,
                              size_t scratch_bytes);
moe_status check_ffn_args(moe_shape s, const void* x, int T, int k, const int32_t* offsets, const int32_t* perm,
                          const int32_t* slot_of_expert, const void* slot_pool, int n_slots, const float* gate,
                          const float* y_perm, const float* out, int flags, const void* workspace,
                          size_t ws_bytes);
moe_status check_combine_args(const float* y_perm, const int32_t* idx, const float* gate, const int32_t* inv_perm,
                              const float* host_partial, int T, int k, int d, int E, const float* out);

// Device attributes of the current device (cached per device id).
struct DeviceInfo { int id, sm_count, cc_major, cc_minor; size_t smem_optin; };
moe_status current_device(DeviceInfo* out);

moe_status check_shape(moe_shape s);

// Limit of the tensor-core kernels' bounded waits, in ns (moe_set_wait_limit_ns),
// and the testing aid of moe_set_test_stall.
uint64_t wait_limit_ns();
int test_stall();

// Schedule of the tcgen05 decode GEMVs: gate/up and down in one cooperative
// launch (true) or in two launches.
bool decode_one_launch(int fmt, int T);

// ---------------------------------------------------------------- device helpers
constexpr unsigned kFull = 0xffffffffu;

// Programmatic dependent launch.  The decode step's kernels are launched with
// launch_pdl, so each may start (and run its prologue) while the kernel before
// it on the stream finishes.  Each executes pdl_wait() before its first access
// to memory that earlier work writes or reads -- it returns once the previous
// grid has completed and its writes are visible -- and pdl_trigger() after it,
// letting the next kernel be scheduled.  Without a programmatic launch both
// are no-ops.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       Args... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

__device__ __forceinline__ void report(int32_t* status, int code) {
  if (status != nullptr) atomicCAS(status, 0, code);
}

// Exclusive block scan (blockDim <= 1024); ws >= 33 ints of shared memory.
__device__ inline int block_scan(int v, int* ws, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(kFull, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) ws[warp] = x;
  __syncthreads();
  if (warp == 0) {
    const int nw = (blockDim.x + 31) >> 5;
    const int w = (lane < nw) ? ws[lane] : 0;
    int s = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(kFull, s, o);
      if (lane >= o) s += y;
    }
    ws[lane] = s - w;
    if (lane == 31) ws[32] = s;
  }
  __syncthreads();
  const int r = ws[warp] + x - v;
  *total = ws[32];
  __syncthreads();
  return r;
}


}  // namespace moe
