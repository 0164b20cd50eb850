// Step 2: stable permutation of token-expert pairs by expert.
//
// Grouping the pairs of a step by expert lets each expert's FFN run once over
// all tokens routed to it; in prefill, thousands of tokens of a layer reach
// nearly the whole expert set (ainewsfeed.tech, second paragraph).  The pages
// do not say how; this is a stable counting sort of p = t*k + j by idx[t][j]:
// offsets = exclusive scan of the per-expert counts, and within an expert the
// pairs keep ascending p, so perm is unique and comparable bit for bit.
//
// The pairs are cut into tiles of 1024 (one CTA of 32 warps each).  Inside a
// tile, the stable rank of a pair among same-expert pairs is
//   (same-expert pairs in earlier warps) + (same-expert lanes below it),
// from __match_any_sync plus a [warp][expert] count table in shared memory
// that is prefix-summed over warps.  One tile (T*k <= 1024, every decode
// step) is a single fused launch with no scratch.  More tiles take three
// launches: per-tile histograms -> one scan over (tile, expert) that yields
// offsets and per-tile bases -> the ranked scatter.
#include <mutex>

#include "common.cuh"

namespace moe {
namespace {

constexpr int kTile = 1024;   // pairs per tile == threads per CTA

__device__ __forceinline__ unsigned lanemask_lt() {
  unsigned m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

// Exclusive scan over the block (<= 1024 threads); returns the prefix of v and
// writes the block total to *total.  ws: 33 ints of shared memory.
__device__ int block_exclusive_scan(int v, int* ws, int* total) {
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
    int w = (lane < nw) ? ws[lane] : 0;
    int s = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(kFull, s, o);
      if (lane >= o) s += y;
    }
    ws[lane] = s - w;             // exclusive prefix of warp sums
    if (lane == 31) ws[32] = s;   // total
  }
  __syncthreads();
  const int r = ws[warp] + x - v;
  *total = ws[32];
  __syncthreads();
  return r;
}

// Loads pair i of the tile, validates its expert, and returns its stable rank
// among the same-expert pairs of the tile.  wcnt: [32][E] uint16 scratch in
// shared memory; tile_cnt (shared, E ints) receives the tile's counts.
__device__ int tile_rank(const int32_t* __restrict__ idx, int n, int E, int32_t* status,
                         uint16_t* wcnt, int* tile_cnt, int* e_out) {
  const int warp = threadIdx.x >> 5;
  for (int q = threadIdx.x; q < 32 * E; q += blockDim.x) wcnt[q] = 0;
  const int i = blockIdx.x * kTile + threadIdx.x;
  int e = (i < n) ? idx[i] : -1;
  if (i < n && (e < 0 || e >= E)) {
    report(status, MOE_ERR_DEVICE);
    e = -1;
  }
  __syncthreads();
  const unsigned same = __match_any_sync(kFull, e);
  const int rank_w = __popc(same & lanemask_lt());
  if (e >= 0 && rank_w == 0) wcnt[warp * E + e] = static_cast<uint16_t>(__popc(same));
  __syncthreads();
  for (int x = threadIdx.x; x < E; x += blockDim.x) {
    int run = 0;
    for (int w = 0; w < 32; ++w) {
      const int c = wcnt[w * E + x];
      wcnt[w * E + x] = static_cast<uint16_t>(run);
      run += c;
    }
    tile_cnt[x] = run;
  }
  __syncthreads();
  *e_out = e;
  return (e >= 0) ? wcnt[warp * E + e] + rank_w : 0;
}

// One tile holds every pair: ranks, counts, scan and scatter in one launch.
__global__ void __launch_bounds__(kTile) permute_fused_kernel(const int32_t* __restrict__ idx, int n,
                                                              int E, int32_t* __restrict__ offsets,
                                                              int32_t* __restrict__ perm,
                                                              int32_t* __restrict__ inv_perm,
                                                              int32_t* status) {
  pdl_wait();   // its inputs come from the previous kernel; its outputs may still be read
  pdl_trigger();
  extern __shared__ __align__(16) unsigned char smem[];
  int* tile_cnt = reinterpret_cast<int*>(smem);            // [E]
  int* ws = tile_cnt + E;                                  // [33]
  uint16_t* wcnt = reinterpret_cast<uint16_t*>(ws + 36);   // [32][E]
  int e;
  const int rank = tile_rank(idx, n, E, status, wcnt, tile_cnt, &e);
  // exclusive scan of the counts over experts (E <= 1024 = blockDim)
  const int c = (threadIdx.x < E) ? tile_cnt[threadIdx.x] : 0;
  int total;
  const int off = block_exclusive_scan(c, ws, &total);
  if (threadIdx.x < E) {
    offsets[threadIdx.x] = off;
    tile_cnt[threadIdx.x] = off;    // reuse as the expert base
  }
  if (threadIdx.x == 0) offsets[E] = total;
  __syncthreads();
  const int i = threadIdx.x;
  if (i < n) {
    if (e >= 0) {
      const int pos = tile_cnt[e] + rank;
      perm[pos] = i;
      inv_perm[i] = pos;
    } else {
      inv_perm[i] = -1;
    }
  }
  if (i >= total && i < n) perm[i] = -1;
}

// Multi-tile, launch 1: histogram of each tile -> counts[tile][E].
__global__ void __launch_bounds__(kTile) permute_count_kernel(const int32_t* __restrict__ idx, int n,
                                                              int E, int32_t* __restrict__ counts) {
  pdl_wait();   // its inputs come from the previous kernel; its outputs may still be read
  pdl_trigger();
  extern __shared__ __align__(16) unsigned char smem[];
  int* hist = reinterpret_cast<int*>(smem);
  for (int x = threadIdx.x; x < E; x += blockDim.x) hist[x] = 0;
  __syncthreads();
  const int i = blockIdx.x * kTile + threadIdx.x;
  if (i < n) {
    const int e = idx[i];
    if (e >= 0 && e < E) atomicAdd(&hist[e], 1);
  }
  __syncthreads();
  for (int x = threadIdx.x; x < E; x += blockDim.x)
    counts[static_cast<size_t>(blockIdx.x) * E + x] = hist[x];
}

// Multi-tile, launch 2 (one CTA): counts[tile][e] -> base[tile][e] (in
// place, = offsets[e] + pairs of expert e in earlier tiles), offsets, tail.
__global__ void __launch_bounds__(kTile) permute_scan_kernel(int32_t* __restrict__ counts, int ntiles,
                                                             int n, int E, int32_t* __restrict__ offsets,
                                                             int32_t* __restrict__ perm) {
  pdl_wait();   // its inputs come from the previous kernel; its outputs may still be read
  pdl_trigger();
  __shared__ int ws[36];
  const int e = threadIdx.x;
  int run = 0;
  if (e < E) {
    for (int t = 0; t < ntiles; ++t) {
      const int c = counts[static_cast<size_t>(t) * E + e];
      counts[static_cast<size_t>(t) * E + e] = run;
      run += c;
    }
  }
  int total;
  const int off = block_exclusive_scan(e < E ? run : 0, ws, &total);
  if (e < E) {
    offsets[e] = off;
    for (int t = 0; t < ntiles; ++t) counts[static_cast<size_t>(t) * E + e] += off;
  }
  if (e == 0) offsets[E] = total;
  for (int q = total + threadIdx.x; q < n; q += blockDim.x) perm[q] = -1;
}

// Multi-tile, launch 3: ranked scatter of every tile.
__global__ void __launch_bounds__(kTile) permute_scatter_kernel(const int32_t* __restrict__ idx, int n,
                                                                int E, const int32_t* __restrict__ base,
                                                                int32_t* __restrict__ perm,
                                                                int32_t* __restrict__ inv_perm,
                                                                int32_t* status) {
  pdl_wait();   // its inputs come from the previous kernel; its outputs may still be read
  pdl_trigger();
  extern __shared__ __align__(16) unsigned char smem[];
  int* tile_cnt = reinterpret_cast<int*>(smem);
  uint16_t* wcnt = reinterpret_cast<uint16_t*>(tile_cnt + E + 36);
  int e;
  const int rank = tile_rank(idx, n, E, status, wcnt, tile_cnt, &e);
  const int i = blockIdx.x * kTile + threadIdx.x;
  if (i < n) {
    if (e >= 0) {
      const int pos = base[static_cast<size_t>(blockIdx.x) * E + e] + rank;
      perm[pos] = i;
      inv_perm[i] = pos;
    } else {
      inv_perm[i] = -1;
    }
  }
}

size_t rank_smem_bytes(int E) { return (static_cast<size_t>(E) + 36) * 4 + 32 * static_cast<size_t>(E) * 2; }

// The opt-in shared-memory limit is raised once per device to the largest
// size any E needs, so later calls (including ones under stream capture)
// only launch.
moe_status ensure_smem_attr(const DeviceInfo& dev) {
  static bool done[64] = {};
  if (done[dev.id]) return MOE_OK;
  const int most = static_cast<int>(rank_smem_bytes(1024));
  const int lim = static_cast<int>(dev.smem_optin) < most ? static_cast<int>(dev.smem_optin) : most;
  MOE_CUDA_TRY(cudaFuncSetAttribute(permute_fused_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, lim));
  MOE_CUDA_TRY(cudaFuncSetAttribute(permute_scatter_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, lim));
  done[dev.id] = true;
  return MOE_OK;
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" size_t moe_permute_scratch_bytes(int T, int k, int E) {
  if (T <= 0 || k <= 0 || E <= 0) return 0;
  const long long n = static_cast<long long>(T) * k;
  const long long ntiles = (n + kTile - 1) / kTile;
  if (ntiles <= 1) return 0;
  return static_cast<size_t>(ntiles) * E * sizeof(int32_t);
}

moe_status moe::check_permute_args(const int32_t* idx, int T, int k, int E, const int32_t* offsets,
                                   const int32_t* perm, const int32_t* inv_perm, const void* scratch,
                                   size_t scratch_bytes) {
  MOE_REQUIRE(T >= 0 && k >= 1 && k <= 32, "T=%d, k=%d", T, k);
  MOE_REQUIRE(E >= 1 && E <= 1024, "E=%d outside [1, 1024]", E);
  MOE_REQUIRE(static_cast<long long>(T) * k <= (1 << 24), "T*k too large");
  MOE_REQUIRE(offsets != nullptr, "null offsets");
  MOE_REQUIRE(aligned(offsets, 4), "misaligned offsets");
  if (T == 0) return MOE_OK;
  MOE_REQUIRE(idx && perm && inv_perm, "null pointer");
  MOE_REQUIRE(aligned(idx, 4) && aligned(perm, 4) && aligned(inv_perm, 4), "misaligned pointer");
  const size_t need = moe_permute_scratch_bytes(T, k, E);   // 0 when the pairs fit one tile
  if (need > 0 && (scratch == nullptr || scratch_bytes < need))
    return fail(MOE_ERR_CAPACITY, "moe_permute needs %zu bytes of scratch, got %zu", need, scratch_bytes);
  MOE_REQUIRE(need == 0 || aligned(scratch, 4), "misaligned scratch");
  return MOE_OK;
}

extern "C" moe_status moe_permute(const int32_t* idx, int T, int k, int E, int32_t* offsets,
                                  int32_t* perm, int32_t* inv_perm, void* scratch,
                                  size_t scratch_bytes, int32_t* dev_status, cudaStream_t stream) {
  clear_error();
  moe_status st = check_permute_args(idx, T, k, E, offsets, perm, inv_perm, scratch, scratch_bytes);
  if (st != MOE_OK) return st;
  const int n = T * k;
  DeviceInfo dev;
  st = current_device(&dev);
  if (st != MOE_OK) return st;
  if (n == 0) {
    MOE_CUDA_TRY(cudaMemsetAsync(offsets, 0, (E + 1) * sizeof(int32_t), stream));
    return MOE_OK;
  }
  const size_t smem = rank_smem_bytes(E);
  MOE_REQUIRE(smem <= dev.smem_optin, "E=%d needs %zu bytes of shared memory", E, smem);
  st = ensure_smem_attr(dev);
  if (st != MOE_OK) return st;
  const int ntiles = (n + kTile - 1) / kTile;
  if (ntiles == 1) {
    MOE_CUDA_TRY(launch_pdl(permute_fused_kernel, dim3(1), dim3(kTile), smem, stream, idx, n, E, offsets, perm,
                            inv_perm, dev_status));
    MOE_LAUNCH_CHECK("permute_fused_kernel");
    return MOE_OK;
  }
  int32_t* counts = static_cast<int32_t*>(scratch);
  MOE_CUDA_TRY(launch_pdl(permute_count_kernel, dim3(ntiles), dim3(kTile), E * sizeof(int), stream, idx, n, E,
                          counts));
  MOE_LAUNCH_CHECK("permute_count_kernel");
  MOE_CUDA_TRY(launch_pdl(permute_scan_kernel, dim3(1), dim3(kTile), 0, stream, counts, ntiles, n, E, offsets, perm));
  MOE_LAUNCH_CHECK("permute_scan_kernel");
  MOE_CUDA_TRY(launch_pdl(permute_scatter_kernel, dim3(ntiles), dim3(kTile), smem, stream, idx, n, E, counts, perm,
                          inv_perm, dev_status));
  MOE_LAUNCH_CHECK("permute_scatter_kernel");
  return MOE_OK;
}

// ---------------------------------------------------------------------------
// moe_permute_noalloc: moe_permute with its scratch taken from a fixed array
// compiled into the library, for callers that cannot allocate device memory.
// The array lives in every device's memory for as long as the library is
// loaded.  Its device address is looked up once per device, by the first call
// made with that device current.
namespace {

constexpr size_t kNoAllocScratchBytes = MOE_PERMUTE_NOALLOC_MAX_SCRATCH;
static_assert(kNoAllocScratchBytes % 256 == 0, "scratch size must keep 256-byte alignment");

static __device__ __align__(256) unsigned char g_permute_scratch[kNoAllocScratchBytes];

std::mutex g_noalloc_mu;
void* g_noalloc_addr[64] = {};

// Device address of g_permute_scratch on the current device.  In host code the
// symbol itself is only a host-side stand-in, never a device address.
moe_status noalloc_scratch(const DeviceInfo& dev, void** out) {
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (g_noalloc_addr[dev.id] == nullptr) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_permute_scratch);
    if (e != cudaSuccess)
      return fail(MOE_ERR_CUDA, "cudaGetSymbolAddress(permute scratch) failed: %s", cudaGetErrorString(e));
    g_noalloc_addr[dev.id] = p;
  }
  *out = g_noalloc_addr[dev.id];
  return MOE_OK;
}

}  // namespace

extern "C" moe_status moe_permute_noalloc(const int32_t* idx, int T, int k, int E, int32_t* offsets,
                                          int32_t* perm, int32_t* inv_perm, int32_t* dev_status,
                                          cudaStream_t stream) {
  clear_error();
  MOE_REQUIRE(T >= 0 && k >= 1 && k <= 32, "T=%d, k=%d", T, k);
  MOE_REQUIRE(E >= 1 && E <= 1024, "E=%d outside [1, 1024]", E);
  MOE_REQUIRE(static_cast<long long>(T) * k <= (1 << 24), "T*k too large");
  const size_t need = moe_permute_scratch_bytes(T, k, E);
  if (need > kNoAllocScratchBytes)
    return fail(MOE_ERR_CAPACITY,
                "moe_permute_noalloc: T=%d, k=%d, E=%d needs %zu bytes of scratch; its fixed array holds %zu "
                "(use moe_permute with caller scratch)",
                T, k, E, need, kNoAllocScratchBytes);
  DeviceInfo dev;
  moe_status st = current_device(&dev);
  if (st != MOE_OK) return st;
  void* scratch = nullptr;
  if (need > 0) {
    st = noalloc_scratch(dev, &scratch);
    if (st != MOE_OK) return st;
  }
  return moe_permute(idx, T, k, E, offsets, perm, inv_perm, scratch, need > 0 ? kNoAllocScratchBytes : 0,
                     dev_status, stream);
}
