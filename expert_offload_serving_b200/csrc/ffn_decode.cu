// Step 3 (decode path): grouped SwiGLU expert FFN for decode-sized groups.
//
// In decode a step touches few experts and each expert sees few tokens, so
// the layer is bound by streaming the selected experts' weights from HBM
// (explainx.ai hardware guide, "Decode: decide whether to move an expert or
// compute where it lives": the GPU runs the cached experts).  For every
// expert e resident in the cache (slot >= 0) and every token row routed to it:
//     h = W_g x,  u = W_u x,  a = silu(h) * u,  y = W_d a.
//
// Two launches:
//   phase 1  rows of W_g and W_u -> a[q][i] (fp32 workspace, q = sorted pair)
//   phase 2  rows of W_d         -> y_perm[q][c]  or  out[t][c] += gate * y
// Work units are (active expert, warp tile of weight rows, pass of token
// rows); each CTA first builds the list of active experts (tokens > 0,
// slot >= 0) from the offsets and the slot table, and units are split into
// contiguous ranges over all warps of a persistent grid (one CTA per SM).
// Weights are streamed HBM -> shared memory by cp.async.bulk into a 3-stage
// ring per warp (one row per lane, mbarrier-completed, L2 evict-first), so
// the bytes in flight do not depend on registers.
//
// FP4 weights (CUDA cores): 4-row tiles (phase 1: gate rows i, i+1 and up
// rows i, i+1), <= 2 token rows per pass; lanes split each 1 KB row slice in
// 16-byte chunks (32 FP4 weights): conflict-free 128-bit shared loads, E2M1 ->
// f16x2 by cvt, times the E8M0 or E4M3 block scale, packed fp32 FMAs against
// the activations (read through L1), and a warp reduce-scatter at the end.
// bf16 weights: the same CUDA-core scheme with 8 bf16 weights per 16 bytes.
// This file serves NVFP4 weights and the shapes outside the tensor-core
// layouts: bf16 blobs in the tile layout and MXFP4 blobs in the stage-tiled
// layout (d, I multiples of 256) go to the tcgen05 GEMVs in ffn_decode_tc.cu.
#include <cuda_fp16.h>

#include <cstdlib>
#include <cstring>
#include "common.cuh"
#include "tc.cuh"

namespace moe {
namespace {

using namespace ::moe::tc;

constexpr int kWarps = 16;                 // warps per CTA (each its own pipeline)
constexpr int kRW = 4;                      // weight rows per warp tile
constexpr int kSlice = 1024;               // bytes of one row per stage
constexpr int kStages = 3;                 // ring depth per warp
constexpr int kStageBytes = kRW * kSlice;  // 4 KB
constexpr size_t kSmemBytes = static_cast<size_t>(kWarps) * kStages * kStageBytes + 1024;

struct FfnParams {
  int E, d, I, T, k, n_slots, fmt;
  const int32_t* offsets;
  const int32_t* perm;
  const int32_t* slot;
  const uint8_t* pool;
  size_t blob_bytes;
  BlobLayout L;
  const uint16_t* x;     // bf16 bits [T][d]
  float* a_ws;           // [T*k][I]
  float* y_perm;         // [T*k][d] or null
  float* out;            // [T][d] when y_perm is null
  const float* gate;     // [T*k]
  int32_t* status;
};

// ------------------------------------------------------------ small helpers
__device__ __forceinline__ void ffma2(float2& acc, float2 a, float2 b) { acc = __ffma2_rn(a, b, acc); }

__device__ __forceinline__ float2 bf16x2_to_float2(uint32_t u) {
  return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xffff0000u));
}

// two E2M1 codes (low nibble = even element) -> f16x2 (low half = even element)
__device__ __forceinline__ uint32_t e2m1x2_to_f16x2(uint32_t byte) {
  uint32_t r;
  asm("{ .reg .b8 b; cvt.u8.u32 b, %1; cvt.rn.f16x2.e2m1x2 %0, b; }" : "=r"(r) : "r"(byte));
  return r;
}

// two E4M3 scale bytes (low byte first) -> f16x2
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t two) {
  uint32_t r;
  asm("{ .reg .b16 s; cvt.u16.u32 s, %1; cvt.rn.f16x2.e4m3x2 %0, s; }" : "=r"(r) : "r"(two));
  return r;
}

__device__ __forceinline__ uint32_t hmul2_u32(uint32_t a, uint32_t b) {
  __half2 r = __hmul2(*reinterpret_cast<__half2*>(&a), *reinterpret_cast<__half2*>(&b));
  return *reinterpret_cast<uint32_t*>(&r);
}

__device__ __forceinline__ float2 f16x2_to_float2(uint32_t u) {
  return __half22float2(*reinterpret_cast<__half2*>(&u));
}

__device__ __forceinline__ float e8m0_to_float(uint32_t b) {
  if (b == 0u) return __uint_as_float(0x00400000u);   // 2^-127
  if (b == 255u) return __uint_as_float(0x7fc00000u); // NaN
  return __uint_as_float(b << 23);
}

// Reduce-scatter of V partial sums across the warp.  After it, the lane holds
// R = max(1, V/32) full sums in v[0..R-1], for value indices
// (lane >> (5 - S)) * R + i, S = min(log2 V, 5).
template <int V>
__device__ __forceinline__ void warp_reduce_scatter(float (&v)[V], int lane) {
  constexpr int LOGV = (V >= 64) ? 6 : (V >= 32) ? 5 : (V >= 16) ? 4 : (V >= 8) ? 3 : (V >= 4) ? 2 : (V >= 2) ? 1 : 0;
  static_assert((1 << LOGV) == V && V <= 64, "V must be a power of two <= 64");
#pragma unroll
  for (int st = 0; st < 5; ++st) {
    const int s = 16 >> st;
    if (st < LOGV) {
      const int half = V >> (st + 1);
      const bool upper = (lane & s) != 0;
#pragma unroll
      for (int i = 0; i < V / 2; ++i) {
        if (i < half) {
          const float keep = upper ? v[i + half] : v[i];
          const float send = upper ? v[i] : v[i + half];
          v[i] = keep + __shfl_xor_sync(kFull, send, s);
        }
      }
    } else {
      v[0] += __shfl_xor_sync(kFull, v[0], s);
    }
  }
}

// ------------------------------------------------------------ bulk copies
// (mbarrier, bulk-copy and L2-policy wrappers: tc.cuh).  Weights are read once
// per layer call: they stream through L2 with an evict-first policy so the
// activations and the SwiGLU workspace stay cached.

// Small expert sets: when every active expert's blob together fits well
// inside L2, the first launch asks L2 to fetch all of them at once (16 KB bulk
// prefetches spread over every lane of the grid), so all DRAM requests of the
// layer are in flight from the start and both launches then stream from L2.
constexpr size_t kPrefetchCap = 96ull << 20;
__device__ void prefetch_active_blobs(const FfnParams& P, const int16_t* act, int n_act) {
  if (static_cast<size_t>(n_act) * P.blob_bytes > kPrefetchCap) return;
  constexpr size_t kChunk = 16384;
  const size_t per = (P.blob_bytes + kChunk - 1) / kChunk;
  const size_t total = per * static_cast<size_t>(n_act);
  const size_t lanes = static_cast<size_t>(gridDim.x) * blockDim.x;
  for (size_t c = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; c < total; c += lanes) {
    const int a = static_cast<int>(c / per);
    const size_t off = (c % per) * kChunk;
    const uint8_t* blob = P.pool + static_cast<size_t>(__ldg(P.slot + act[a])) * P.blob_bytes;
    const uint32_t bytes = static_cast<uint32_t>(min(kChunk, P.blob_bytes - off));
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(blob + off), "r"(bytes) : "memory");
  }
}

// ------------------------------------------------------------ weight decode
// Dequantised weights of one 8-element sub-chunk m of a 16-byte chunk.
template <int FMT>
struct Weights;

template <>
struct Weights<MOE_W_BF16> {
  static constexpr int EPC = 8;   // elements per 16-byte chunk
  static constexpr int SUB = 1;   // 8-element sub-chunks per chunk
  struct Scale {};
  __device__ static Scale scale(const uint8_t*, int, int, int) { return {}; }
  __device__ static void decode(const uint4& raw, int, Scale, float2 (&w)[4]) {
    w[0] = bf16x2_to_float2(raw.x);
    w[1] = bf16x2_to_float2(raw.y);
    w[2] = bf16x2_to_float2(raw.z);
    w[3] = bf16x2_to_float2(raw.w);
  }
};

template <>
struct Weights<MOE_W_MXFP4> {
  static constexpr int EPC = 32;
  static constexpr int SUB = 4;
  struct Scale { float s; };
  // scales: [R][K/32] bytes; chunk c is block c of row r
  __device__ static Scale scale(const uint8_t* sbase, int r, int c, int K) {
    return {e8m0_to_float(__ldg(sbase + static_cast<size_t>(r) * (K >> 5) + c))};
  }
  __device__ static void decode(const uint4& raw, int m, Scale sc, float2 (&w)[4]) {
    const uint32_t word = (m == 0) ? raw.x : (m == 1) ? raw.y : (m == 2) ? raw.z : raw.w;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 f = f16x2_to_float2(e2m1x2_to_f16x2((word >> (8 * j)) & 0xffu));
      w[j] = __fmul2_rn(f, make_float2(sc.s, sc.s));
    }
  }
};

template <>
struct Weights<MOE_W_NVFP4> {
  static constexpr int EPC = 32;
  static constexpr int SUB = 4;
  struct Scale { uint32_t s01; };   // f16x2 of the scales of blocks 2c and 2c+1
  __device__ static Scale scale(const uint8_t* sbase, int r, int c, int K) {
    const uint16_t two = __ldg(reinterpret_cast<const uint16_t*>(sbase + sf_atom_offset(r, 2 * c, K)));
    return {e4m3x2_to_f16x2(two)};
  }
  __device__ static void decode(const uint4& raw, int m, Scale sc, float2 (&w)[4]) {
    const uint32_t word = (m == 0) ? raw.x : (m == 1) ? raw.y : (m == 2) ? raw.z : raw.w;
    // sub-chunks 0,1 hold block 2c; 2,3 hold block 2c+1.  code * scale is exact in f16.
    const uint32_t s = (m < 2) ? (sc.s01 & 0xffffu) * 0x10001u : (sc.s01 >> 16) * 0x10001u;
#pragma unroll
    for (int j = 0; j < 4; ++j)
      w[j] = f16x2_to_float2(hmul2_u32(e2m1x2_to_f16x2((word >> (8 * j)) & 0xffu), s));
  }
};

// ------------------------------------------------------------ activations
// Token rows: bf16 (phase 1, x) or fp32 (phase 2, the SwiGLU workspace).
struct XBf16 {
  const uint16_t* base;
  int ld;   // elements per row
  __device__ void load(int row, int k0, float2 (&xf)[4]) const {
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(base + static_cast<size_t>(row) * ld + k0));
    xf[0] = bf16x2_to_float2(v.x);
    xf[1] = bf16x2_to_float2(v.y);
    xf[2] = bf16x2_to_float2(v.z);
    xf[3] = bf16x2_to_float2(v.w);
  }
};

struct XF32 {
  const float* base;
  int ld;
  __device__ void load(int row, int k0, float2 (&xf)[4]) const {
    const float4* p = reinterpret_cast<const float4*>(base + static_cast<size_t>(row) * ld + k0);
    const float4 a = __ldg(p), b = __ldg(p + 1);
    xf[0] = make_float2(a.x, a.y);
    xf[1] = make_float2(a.z, a.w);
    xf[2] = make_float2(b.x, b.y);
    xf[3] = make_float2(b.z, b.w);
  }
};

// Dot products of kRW weight rows with NT token rows over K.
//   wrow[r]: byte address of row r's codes; srow/rg: scale region and global
//   row index of row r (FP4); xrows[t]: row index into xs.
// ------------------------------------------------------------ work decomposition
// Token rows per pass: 4 for bf16, 2 for FP4 (whose dequantisation keeps more
// registers live); larger passes would spill at 128 registers per thread.
template <int FMT>
__host__ __device__ constexpr int nt_max() { return FMT == MOE_W_BF16 ? 4 : 2; }

struct Unit {
  int e, tile, q0, tb, nt;   // expert, warp tile, first sorted row, first token row of the pass, rows
};

template <int FMT, int PHASE>
__device__ __forceinline__ Unit decode_unit(const FfnParams& P, const int16_t* act, const int32_t* ustart,
                                            int n_act, long long u) {
  constexpr int kNTMax = nt_max<FMT>();
  int lo = 0, hi = n_act;   // last a with ustart[a] <= u
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (ustart[mid] <= u) lo = mid;
    else hi = mid;
  }
  Unit U;
  U.e = act[lo];
  U.q0 = __ldg(P.offsets + U.e);
  const int ne = __ldg(P.offsets + U.e + 1) - U.q0;
  const int passes = (ne + kNTMax - 1) / kNTMax;
  const int local = static_cast<int>(u - ustart[lo]);
  U.tile = local / passes;
  const int pass = local % passes;
  U.tb = pass * kNTMax;
  U.nt = min(kNTMax, ne - U.tb);
  return U;
}

// Byte address of weight row r (0..7) of a unit's tile.
template <int FMT, int PHASE>
__device__ __forceinline__ const uint8_t* tile_row(const FfnParams& P, const uint8_t* blob, int tile, int r,
                                                   size_t row_bytes, int* grow, int* mat) {
  if (PHASE == 1) {
    constexpr int H = kRW / 2;   // gate rows first, then the up rows of the same indices
    const bool up = r >= H;
    const int i = H * tile + (up ? r - H : r);
    const int row = (FMT == MOE_W_NVFP4) ? gu_row(i, up) : i;
    *grow = row;
    *mat = up ? 1 : 0;
    return blob + (up ? P.L.wu : P.L.wg) + static_cast<size_t>(row) * row_bytes;
  }
  const int row = kRW * tile + r;
  *grow = row;
  *mat = 2;
  return blob + P.L.wd + static_cast<size_t>(row) * row_bytes;
}

// The warp's pipeline state: items are (unit, slice) in order; item j lives
// in stage j % kStages and completes phase (j / kStages) & 1 of its barrier.
// Issuing: lane r (< 8) holds the address of weight row r of the unit being
// issued, so one warp instruction issues the 8 row copies of a stage.
struct Pipe {
  uint8_t* ring;       // kStages * kStageBytes
  uint64_t* bar;       // kStages
  long long beg, n_units, next_issue, n_items;
  int slices;
  bool ok;
  long long issue_unit;        // unit whose row addresses lane_row holds (-1: none)
  const uint8_t* lane_row;     // this lane's weight row of issue_unit (lanes < kRW)
  uint64_t policy;             // L2 policy of the weight copies
};

template <int FMT, int PHASE>
__device__ __forceinline__ void issue_item(const FfnParams& P, const int16_t* act, const int32_t* ustart,
                                           int n_act, Pipe& pp, size_t row_bytes, int lane) {
  const long long j = pp.next_issue++;
  const long long u = pp.beg + j / pp.slices;
  const int sl = static_cast<int>(j % pp.slices);
  const int st = static_cast<int>(j % kStages);
  if (u != pp.issue_unit) {
    const Unit U = decode_unit<FMT, PHASE>(P, act, ustart, n_act, u);
    const uint8_t* blob = P.pool + static_cast<size_t>(__ldg(P.slot + U.e)) * P.blob_bytes;
    int g, m;
    pp.lane_row = tile_row<FMT, PHASE>(P, blob, U.tile, lane & (kRW - 1), row_bytes, &g, &m);
    pp.issue_unit = u;
  }
  const size_t off = static_cast<size_t>(sl) * kSlice;
  const uint32_t bytes = static_cast<uint32_t>(min(static_cast<size_t>(kSlice), row_bytes - off));
  // the stage was last read by this warp's generic loads; order them before the async writes
  __syncwarp();
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  if (lane == 0) mbar_expect_tx(&pp.bar[st], bytes * kRW);
  __syncwarp();
  if (lane < kRW)
    bulk_load(pp.ring + st * kStageBytes + lane * kSlice, pp.lane_row + off, bytes, &pp.bar[st], pp.policy);
}

__device__ __forceinline__ float silu(float h) { return h / (1.0f + expf(-h)); }

// All slices of one unit with NT token rows per pass.
template <int FMT, int PHASE, int NT>
__device__ void run_unit(const FfnParams& P, const int16_t* act, const int32_t* ustart, int n_act, Pipe& pp,
                         const Unit& U, size_t row_bytes, long long& j, int lane) {
  using W = Weights<FMT>;
  const int K = (PHASE == 1) ? P.d : P.I;
  const uint8_t* blob = P.pool + static_cast<size_t>(__ldg(P.slot + U.e)) * P.blob_bytes;
  const uint8_t* sreg[kRW];
  int grow[kRW];
  float tscale[kRW];
  const float* ts = reinterpret_cast<const float*>(blob + P.L.ts);
#pragma unroll
  for (int r = 0; r < kRW; ++r) {
    int g, mat;
    tile_row<FMT, PHASE>(P, blob, U.tile, r, row_bytes, &g, &mat);
    grow[r] = g;
    sreg[r] = blob + (mat == 0 ? P.L.sg : mat == 1 ? P.L.su : P.L.sd);
    tscale[r] = (FMT == MOE_W_NVFP4) ? __ldg(ts + mat) : 1.0f;
  }
  int xrows[NT];
#pragma unroll
  for (int t = 0; t < NT; ++t) {
    const int q = U.q0 + U.tb + min(t, U.nt - 1);   // padding rows repeat the last real one
    if (PHASE == 1) {
      int p = __ldg(P.perm + q);
      if (p < 0 || p >= P.T * P.k) {
        report(P.status, MOE_ERR_DEVICE);
        p = 0;
      }
      xrows[t] = p / P.k;
    } else {
      xrows[t] = q;
    }
  }
  float2 acc[kRW][NT];
#pragma unroll
  for (int r = 0; r < kRW; ++r)
#pragma unroll
    for (int t = 0; t < NT; ++t) acc[r][t] = make_float2(0.f, 0.f);

  for (int sl = 0; sl < pp.slices; ++sl, ++j) {
    if (pp.next_issue < pp.n_items) issue_item<FMT, PHASE>(P, act, ustart, n_act, pp, row_bytes, lane);
    const int st = static_cast<int>(j % kStages);
    if (!__all_sync(kFull, mbar_wait(&pp.bar[st], static_cast<uint32_t>((j / kStages) & 1), nullptr))) {
      pp.ok = false;
      return;
    }
    const uint8_t* stage = pp.ring + st * kStageBytes;
    const int valid = static_cast<int>(min(static_cast<size_t>(kSlice), row_bytes - static_cast<size_t>(sl) * kSlice));
#pragma unroll 1
    for (int h = 0; h < 2; ++h) {
      const int c = lane + 32 * h;                 // 16-byte chunk inside the 1 KB slice
      if (c * 16 >= valid) break;
      const int k0 = (sl * kSlice + c * 16) * W::EPC / 16;   // first K element of the chunk
      // FP4 reuses a row's 16 bytes for 4 sub-chunks: keep them; bf16 uses each once
      constexpr int kHeld = (W::SUB > 1) ? kRW : 1;
      uint4 raw[kHeld];
      typename W::Scale sc[kRW];
#pragma unroll
      for (int r = 0; r < kRW; ++r) {
        if constexpr (W::SUB > 1) raw[r < kHeld ? r : 0] = *reinterpret_cast<const uint4*>(stage + r * kSlice + c * 16);
        sc[r] = W::scale(sreg[r], grow[r], k0 / W::EPC, K);
      }
#pragma unroll
      for (int m = 0; m < W::SUB; ++m) {
        // activations of at most 4 tokens are live at a time; weights are
        // decoded once per 4-token group
        constexpr int GS = NT < 4 ? NT : 4;
#pragma unroll
        for (int g = 0; g < NT / GS; ++g) {
          float2 xf[GS][4];
#pragma unroll
          for (int t = 0; t < GS; ++t) {
            if (PHASE == 1) XBf16{P.x, P.d}.load(xrows[g * GS + t], k0 + 8 * m, xf[t]);
            else XF32{P.a_ws, P.I}.load(xrows[g * GS + t], k0 + 8 * m, xf[t]);
          }
#pragma unroll
          for (int r = 0; r < kRW; ++r) {
            float2 w[4];
            if constexpr (W::SUB > 1) {
              W::decode(raw[r < kHeld ? r : 0], m, sc[r], w);
            } else {
              const uint4 one = *reinterpret_cast<const uint4*>(stage + r * kSlice + c * 16);
              W::decode(one, m, sc[r], w);
            }
            // q outer, tokens inner: consecutive FMAs update different accumulators
#pragma unroll
            for (int q = 0; q < 4; ++q)
#pragma unroll
              for (int t = 0; t < GS; ++t) ffma2(acc[r][g * GS + t], w[q], xf[t][q]);
          }
        }
      }
    }
  }
  // reduce over the warp: value index v = r * NT + t
  constexpr int V = kRW * NT;
  constexpr int LOGV = (V >= 64) ? 6 : (V >= 32) ? 5 : (V >= 16) ? 4 : (V >= 8) ? 3 : 2;
  constexpr int S = LOGV < 5 ? LOGV : 5;
  constexpr int R = (V >> S);
  float v[V];
#pragma unroll
  for (int r = 0; r < kRW; ++r)
#pragma unroll
    for (int t = 0; t < NT; ++t) v[r * NT + t] = acc[r][t].x + acc[r][t].y;
  warp_reduce_scatter<V>(v, lane);
  const bool writer = (lane & ((1 << (5 - S)) - 1)) == 0;
#pragma unroll
  for (int i = 0; i < R; ++i) {
    const int vi = (lane >> (5 - S)) * R + i;
    const int r = vi / NT, t = vi % NT;
    if (PHASE == 1) {
      // lanes < 16 hold gate rows (r < kRW/2); lane ^ 16 holds the up row of the same (i, token)
      const float other = __shfl_xor_sync(kFull, v[i], 16);
      if (writer && lane < 16 && t < U.nt) {
        const float hh = v[i] * tscale[r];
        const float uu = other * tscale[r + kRW / 2];
        P.a_ws[static_cast<size_t>(U.q0 + U.tb + t) * P.I + (kRW / 2) * U.tile + r] = silu(hh) * uu;
      }
    } else if (writer && t < U.nt) {
      const int q = U.q0 + U.tb + t;
      const int row = kRW * U.tile + r;
      const float y = v[i] * tscale[r];
      if (P.y_perm != nullptr) {
        P.y_perm[static_cast<size_t>(q) * P.d + row] = y;
      } else {
        const int p = __ldg(P.perm + q);
        if (p >= 0 && p < P.T * P.k)
          atomicAdd(P.out + static_cast<size_t>(p / P.k) * P.d + row, __ldg(P.gate + p) * y);
      }
    }
  }
}

template <int FMT, int PHASE>
__global__ void __launch_bounds__(kWarps * 32, 1) ffn_decode_kernel(FfnParams P) {
  static_assert(kWarps * kStages <= 64, "barrier array");
  extern __shared__ __align__(128) uint8_t smem_raw[];
  __shared__ int16_t s_act[1024];
  __shared__ int32_t s_ustart[1025];
  __shared__ int s_ws[36];
  __shared__ __align__(8) uint64_t s_bar[kWarps * kStages];
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int tiles_per_e = (PHASE == 1) ? P.I / (kRW / 2) : P.d / kRW;
  // active experts (tokens > 0, resident) in expert order, with their unit counts
  const int per = (P.E + blockDim.x - 1) / blockDim.x;
  const int e0 = threadIdx.x * per;
  int cnt = 0, units = 0;
  uint32_t mask = 0;   // per <= 2
  const int npairs = P.T * P.k;
  for (int jx = 0; jx < per; ++jx) {
    const int e = e0 + jx;
    if (e >= P.E) break;
    const int a = __ldg(P.offsets + e), b = __ldg(P.offsets + e + 1);
    if (b <= a) continue;
    if (a < 0 || b > npairs) {
      report(P.status, MOE_ERR_DEVICE);
      continue;
    }
    const int s = __ldg(P.slot + e);
    if (s < 0) continue;
    if (s >= P.n_slots) {
      report(P.status, MOE_ERR_DEVICE);
      continue;
    }
    mask |= 1u << jx;
    ++cnt;
  }
  int n_act;
  int pos = block_scan(cnt, s_ws, &n_act);
  for (int jx = 0; jx < per; ++jx)
    if (mask & (1u << jx)) {
      const int e = e0 + jx;
      const int ne = __ldg(P.offsets + e + 1) - __ldg(P.offsets + e);
      s_act[pos++] = static_cast<int16_t>(e);
      units += tiles_per_e * ((ne + nt_max<FMT>() - 1) / nt_max<FMT>());
    }
  int total_units;
  int ustart = block_scan(units, s_ws, &total_units);
  pos -= cnt;
  for (int jx = 0; jx < per; ++jx)
    if (mask & (1u << jx)) {
      const int e = e0 + jx;
      const int ne = __ldg(P.offsets + e + 1) - __ldg(P.offsets + e);
      s_ustart[pos++] = ustart;
      ustart += tiles_per_e * ((ne + nt_max<FMT>() - 1) / nt_max<FMT>());
    }
  if (threadIdx.x < kWarps * kStages) mbar_init(&s_bar[threadIdx.x], 1);
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  __syncthreads();

  const int K = (PHASE == 1) ? P.d : P.I;
  const size_t row_bytes = (FMT == MOE_W_BF16) ? static_cast<size_t>(K) * 2 : static_cast<size_t>(K) / 2;
  const long long nw = static_cast<long long>(gridDim.x) * kWarps;
  const long long gw = static_cast<long long>(blockIdx.x) * kWarps + warp;
  Pipe pp;
  pp.ring = smem_raw + static_cast<size_t>(warp) * kStages * kStageBytes;
  pp.bar = s_bar + warp * kStages;
  pp.beg = total_units * gw / nw;
  pp.n_units = total_units * (gw + 1) / nw - pp.beg;
  pp.slices = static_cast<int>((row_bytes + kSlice - 1) / kSlice);
  pp.n_items = pp.n_units * pp.slices;
  pp.next_issue = 0;
  pp.ok = true;
  pp.issue_unit = -1;
  pp.lane_row = nullptr;
  pp.policy = policy_evict_first();
  if (PHASE == 1) prefetch_active_blobs(P, s_act, n_act);
  // prime the ring with kStages - 1 items
  for (int i = 0; i < kStages - 1 && pp.next_issue < pp.n_items; ++i)
    issue_item<FMT, PHASE>(P, s_act, s_ustart, n_act, pp, row_bytes, lane);
  long long j = 0;
  for (long long u = 0; u < pp.n_units && pp.ok; ++u) {
    const Unit U = decode_unit<FMT, PHASE>(P, s_act, s_ustart, n_act, pp.beg + u);
    if (U.nt == 1) run_unit<FMT, PHASE, 1>(P, s_act, s_ustart, n_act, pp, U, row_bytes, j, lane);
    else if (nt_max<FMT>() == 2 || U.nt == 2) run_unit<FMT, PHASE, 2>(P, s_act, s_ustart, n_act, pp, U, row_bytes, j, lane);
    else run_unit<FMT, PHASE, (nt_max<FMT>() > 2 ? 4 : 2)>(P, s_act, s_ustart, n_act, pp, U, row_bytes, j, lane);
  }
  if (!pp.ok) {
    report(P.status, MOE_ERR_TIMEOUT);
  }
  // every issued copy has landed before the CTA leaves (bounded)
  for (long long i = j; i < pp.next_issue; ++i) {
    const uint64_t t0 = now_ns();
    while (!mbar_try(&pp.bar[i % kStages], static_cast<uint32_t>((i / kStages) & 1)) && now_ns() - t0 <= kWaitNs) {
    }
  }
}

template <int FMT, int PHASE>
moe_status launch_phase(const FfnParams& P, const DeviceInfo& dev, cudaStream_t s) {
  static bool attr[64] = {};
  if (!attr[dev.id]) {
    MOE_CUDA_TRY(cudaFuncSetAttribute(ffn_decode_kernel<FMT, PHASE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      static_cast<int>(kSmemBytes)));
    attr[dev.id] = true;
  }
  const int tiles_per_e = (PHASE == 1) ? P.I / (kRW / 2) : P.d / kRW;
  const long long most = static_cast<long long>(min(P.E, P.T * P.k)) * tiles_per_e *
                         ((P.T * P.k + nt_max<FMT>() - 1) / nt_max<FMT>());
  long long blocks = (most + kWarps - 1) / kWarps;
  if (blocks > dev.sm_count) blocks = dev.sm_count;
  if (blocks < 1) blocks = 1;
  ffn_decode_kernel<FMT, PHASE><<<static_cast<int>(blocks), kWarps * 32, kSmemBytes, s>>>(P);
  MOE_LAUNCH_CHECK("ffn_decode_kernel");
  return MOE_OK;
}

template <int FMT>
moe_status launch_decode(const FfnParams& P, const DeviceInfo& dev, cudaStream_t s) {
  if (kSmemBytes > dev.smem_optin) return fail(MOE_ERR_UNSUPPORTED, "needs %zu bytes of shared memory", kSmemBytes);
  moe_status st = launch_phase<FMT, 1>(P, dev, s);
  if (st != MOE_OK) return st;
  return launch_phase<FMT, 2>(P, dev, s);
}

}  // namespace

size_t decode_mx_workspace_bytes(moe_shape s, int T, int k);

// One cooperative launch saves the second launch and its pipeline fill, but
// its down units wait on their expert's gate/up units, while the two-launch
// schedule streams the down GEMV's weights during the gate/up tail (it is a
// programmatic dependent launch).  Measured on B200 (fraction of HBM
// bandwidth, one launch vs two): bf16 T = 1 0.40 / 0.47, T = 16 0.85 / 0.91,
// T = 64 0.74 / 0.85; MXFP4 T = 1 0.37 / 0.35, T = 8 0.64 / 0.68.  So one
// launch only for MXFP4 single-token steps.
bool decode_one_launch(int fmt, int T) {
  static const int forced = [] {
    const char* e = std::getenv("MOE_DECODE_SCHEDULE");
    if (e == nullptr) return 0;
    if (std::strcmp(e, "one") == 0) return 1;
    if (std::strcmp(e, "two") == 0) return 2;
    return 0;
  }();
  if (forced != 0) return forced == 1;
  return fmt == MOE_W_MXFP4 && T <= 1;
}

size_t decode_workspace_bytes(moe_shape s, int T, int k) {
  // MXFP4 tensor-core path: the E4M3 terms of x and a with their scales;
  // otherwise a: fp32 (CUDA-core path) or the two 16-bit planes of the bf16
  // tensor-core path
  if (s.fmt == MOE_W_MXFP4 && mx_tiled(s.d, s.I)) return decode_mx_workspace_bytes(s, T, k);
  // bf16 tile layout: + one gate/up completion counter per expert (one-launch schedule)
  const size_t extra = (s.fmt == MOE_W_BF16 && bf16_blocked(s.d, s.I)) ? round_up(static_cast<size_t>(s.E) * 4, 256) : 0;
  return round_up(static_cast<size_t>(T) * k * s.I * sizeof(float), 256) + extra;
}

moe_status launch_decode_tc(moe_shape s, const void* x, int T, int k, const int32_t* offsets, const int32_t* perm,
                            const int32_t* slot, const void* pool, int n_slots, const float* gate, float* y_perm,
                            float* out, void* ws, int32_t* status, const DeviceInfo& dev, cudaStream_t stream);

moe_status launch_decode_mx(moe_shape s, const void* x, int T, int k, const int32_t* offsets, const int32_t* perm,
                            const int32_t* slot, const void* pool, int n_slots, const float* gate, float* y_perm,
                            float* out, void* ws, int32_t* status, const DeviceInfo& dev, cudaStream_t stream);

moe_status launch_ffn_decode(moe_shape s, const void* x, int T, int k, const int32_t* offsets,
                             const int32_t* perm, const int32_t* slot, const void* pool, int n_slots,
                             const float* gate, float* y_perm, float* out, void* ws,
                             int32_t* status, const DeviceInfo& dev, cudaStream_t stream) {
  if (s.fmt == MOE_W_MXFP4 && mx_tiled(s.d, s.I))
    return launch_decode_mx(s, x, T, k, offsets, perm, slot, pool, n_slots, gate, y_perm, out, ws, status, dev,
                            stream);
  if (s.fmt == MOE_W_BF16 && bf16_blocked(s.d, s.I))
    return launch_decode_tc(s, x, T, k, offsets, perm, slot, pool, n_slots, gate, y_perm, out, ws, status, dev,
                            stream);
  FfnParams P{};
  P.E = s.E;
  P.d = s.d;
  P.I = s.I;
  P.T = T;
  P.k = k;
  P.n_slots = n_slots;
  P.fmt = s.fmt;
  P.offsets = offsets;
  P.perm = perm;
  P.slot = slot;
  P.pool = static_cast<const uint8_t*>(pool);
  P.L = blob_layout(s.fmt, s.d, s.I);
  P.blob_bytes = P.L.bytes;
  P.x = static_cast<const uint16_t*>(x);
  P.a_ws = static_cast<float*>(ws);
  P.y_perm = y_perm;
  P.out = out;
  P.gate = gate;
  P.status = status;
  switch (s.fmt) {
    case MOE_W_BF16: return launch_decode<MOE_W_BF16>(P, dev, stream);
    case MOE_W_MXFP4: return launch_decode<MOE_W_MXFP4>(P, dev, stream);
    case MOE_W_NVFP4: return launch_decode<MOE_W_NVFP4>(P, dev, stream);
    default: return fail(MOE_ERR_INVALID_ARG, "unknown format %d", s.fmt);
  }
}

}  // namespace moe
