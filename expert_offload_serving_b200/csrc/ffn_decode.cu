// Step 3 (CUDA-core path): grouped SwiGLU expert FFN for decode-sized groups.
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
// A warp tile is 4 weight rows (phase 1: gate rows i, i+1 and up rows i, i+1,
// so the SwiGLU is formed in registers; phase 2: 4 rows of W_d) against up to
// 8 token rows at a time.  Lanes split K in 16-byte chunks (8 bf16 or 32 FP4
// weights): chunk c of a row is read by lane c % 32 with one 128-bit
// streaming load, dequantised in registers (E2M1 -> f16x2 by cvt, times the
// E8M0 or E4M3 block scale), and multiplied with the token's activations by
// packed fp32 FMAs (fma.rn.f32x2).  A reduce-scatter over the warp (31
// shuffles for 32 values) leaves each lane one finished dot product.
// Work: every (active expert, warp tile) pair, split into contiguous ranges
// over all warps of a persistent grid; each CTA first compacts the list of
// active experts (tokens > 0 and slot >= 0) from the offsets and slot table.
#include <cuda_fp16.h>

#include "common.cuh"

namespace moe {
namespace {

constexpr int kWarps = 4;    // warps per CTA
constexpr int kRW = 4;       // weight rows per warp tile
constexpr int kNTMax = 8;    // token rows per pass

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
__device__ __forceinline__ uint4 ld_stream(const uint8_t* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

__device__ __forceinline__ void ffma2(float2& acc, float2 a, float2 b) {
  unsigned long long A, B, C;
  asm("mov.b64 %0, {%1, %2};" : "=l"(A) : "f"(a.x), "f"(a.y));
  asm("mov.b64 %0, {%1, %2};" : "=l"(B) : "f"(b.x), "f"(b.y));
  asm("mov.b64 %0, {%1, %2};" : "=l"(C) : "f"(acc.x), "f"(acc.y));
  asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(C) : "l"(A), "l"(B));
  asm("mov.b64 {%0, %1}, %2;" : "=f"(acc.x), "=f"(acc.y) : "l"(C));
}

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

// Exclusive block scan (blockDim <= 1024); ws >= 33 ints of shared memory.
__device__ int block_scan(int v, int* ws, int* total) {
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

// Reduce-scatter of V partial sums across the warp: afterwards the lane
// returns the full sum of value index (lane >> (5 - log2 V)).
template <int V>
__device__ __forceinline__ float warp_reduce_scatter(float (&v)[V], int lane) {
  constexpr int LOGV = (V >= 32) ? 5 : (V >= 16) ? 4 : (V >= 8) ? 3 : (V >= 4) ? 2 : (V >= 2) ? 1 : 0;
  static_assert((1 << LOGV) == V && V <= 32, "V must be a power of two <= 32");
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
  return v[0];
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
      w[j] = make_float2(f.x * sc.s, f.y * sc.s);
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
template <int FMT, int NT, class XS>
__device__ __forceinline__ void tile_dot(const uint8_t* const (&wrow)[kRW], const uint8_t* const (&sreg)[kRW],
                                         const int (&rg)[kRW], int K, const XS& xs,
                                         const int (&xrows)[NT], int lane, float (&res)[kRW * NT]) {
  using W = Weights<FMT>;
  float2 acc[kRW][NT];
#pragma unroll
  for (int r = 0; r < kRW; ++r)
#pragma unroll
    for (int t = 0; t < NT; ++t) acc[r][t] = make_float2(0.f, 0.f);
  const int nc = K / W::EPC;
#pragma unroll 2
  for (int c = lane; c < nc; c += 32) {
    uint4 raw[kRW];
    typename W::Scale sc[kRW];
#pragma unroll
    for (int r = 0; r < kRW; ++r) raw[r] = ld_stream(wrow[r] + static_cast<size_t>(c) * 16);
#pragma unroll
    for (int r = 0; r < kRW; ++r) sc[r] = W::scale(sreg[r], rg[r], c, K);
#pragma unroll
    for (int m = 0; m < W::SUB; ++m) {
      float2 w[kRW][4];
#pragma unroll
      for (int r = 0; r < kRW; ++r) W::decode(raw[r], m, sc[r], w[r]);
#pragma unroll
      for (int t = 0; t < NT; ++t) {
        float2 xf[4];
        xs.load(xrows[t], c * W::EPC + 8 * m, xf);
#pragma unroll
        for (int r = 0; r < kRW; ++r)
#pragma unroll
          for (int j = 0; j < 4; ++j) ffma2(acc[r][t], w[r][j], xf[j]);
      }
    }
  }
#pragma unroll
  for (int r = 0; r < kRW; ++r)
#pragma unroll
    for (int t = 0; t < NT; ++t) res[r * NT + t] = acc[r][t].x + acc[r][t].y;
}

__device__ __forceinline__ float silu(float h) { return h / (1.0f + expf(-h)); }

// One warp tile of phase 1 (gate/up rows i0, i0+1) or phase 2 (W_d rows
// 4*tile .. 4*tile+3) for the token rows [tb, tb + nt) of expert e.
template <int FMT, int PHASE, int NT>
__device__ void run_tile(const FfnParams& P, const uint8_t* blob, int tile, int q0, int tb, int nt,
                         int lane) {
  const int K = (PHASE == 1) ? P.d : P.I;
  const size_t row_bytes = (FMT == MOE_W_BF16) ? static_cast<size_t>(K) * 2 : static_cast<size_t>(K) / 2;
  const uint8_t* wrow[kRW];
  const uint8_t* sreg[kRW];
  int rg[kRW];
  float tscale[kRW];
  const float* ts = reinterpret_cast<const float*>(blob + P.L.ts);
#pragma unroll
  for (int r = 0; r < kRW; ++r) {
    size_t moff, soff;
    int row, mat;
    if (PHASE == 1) {
      mat = (r < 2) ? 0 : 1;            // gate rows first, then up rows
      row = 2 * tile + (r & 1);
      moff = mat == 0 ? P.L.wg : P.L.wu;
      soff = mat == 0 ? P.L.sg : P.L.su;
    } else {
      mat = 2;
      row = 4 * tile + r;
      moff = P.L.wd;
      soff = P.L.sd;
    }
    wrow[r] = blob + moff + static_cast<size_t>(row) * row_bytes;
    sreg[r] = blob + soff;
    rg[r] = row;
    tscale[r] = (FMT == MOE_W_NVFP4) ? __ldg(ts + mat) : 1.0f;
  }
  int xrows[NT];
#pragma unroll
  for (int t = 0; t < NT; ++t) {
    const int q = q0 + tb + min(t, nt - 1);   // padding rows repeat the last real one
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
  float res[kRW * NT];
  if (PHASE == 1) {
    XBf16 xs{P.x, P.d};
    tile_dot<FMT, NT>(wrow, sreg, rg, K, xs, xrows, lane, res);
  } else {
    XF32 xs{P.a_ws, P.I};
    tile_dot<FMT, NT>(wrow, sreg, rg, K, xs, xrows, lane, res);
  }
  constexpr int V = kRW * NT;
  constexpr int LOGV = (V >= 32) ? 5 : (V >= 16) ? 4 : (V >= 8) ? 3 : 2;
  const float val = warp_reduce_scatter<V>(res, lane);
  const int vi = lane >> (5 - LOGV);
  const int r = vi / NT, t = vi % NT;
  const bool writer = (lane & ((1 << (5 - LOGV)) - 1)) == 0;
  if (PHASE == 1) {
    // lanes < 16 hold gate rows, lane ^ 16 the up row of the same (i, token)
    const float other = __shfl_xor_sync(kFull, val, 16);
    if (writer && lane < 16 && t < nt) {
      const float h = val * tscale[0];
      const float u = other * tscale[2];
      const int q = q0 + tb + t;
      P.a_ws[static_cast<size_t>(q) * P.I + 2 * tile + r] = silu(h) * u;
    }
  } else if (writer && t < nt) {
    const int q = q0 + tb + t;
    const int row = 4 * tile + r;
    const float y = val * tscale[0];
    if (P.y_perm != nullptr) {
      P.y_perm[static_cast<size_t>(q) * P.d + row] = y;
    } else {
      const int p = __ldg(P.perm + q);
      if (p >= 0 && p < P.T * P.k)
        atomicAdd(P.out + static_cast<size_t>(p / P.k) * P.d + row, __ldg(P.gate + p) * y);
    }
  }
}

template <int FMT, int PHASE>
__global__ void __launch_bounds__(kWarps * 32) ffn_decode_kernel(FfnParams P) {
  __shared__ int16_t s_act[1024];
  __shared__ int s_ws[36];
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  // compact the active experts (tokens > 0, resident) in expert order
  const int per = (P.E + blockDim.x - 1) / blockDim.x;
  const int e0 = threadIdx.x * per;
  int cnt = 0;
  uint32_t mask = 0;   // per <= 8
  const int npairs = P.T * P.k;
  for (int j = 0; j < per; ++j) {
    const int e = e0 + j;
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
    mask |= 1u << j;
    ++cnt;
  }
  int n_act;
  int pos = block_scan(cnt, s_ws, &n_act);
  for (int j = 0; j < per; ++j)
    if (mask & (1u << j)) s_act[pos++] = static_cast<int16_t>(e0 + j);
  __syncthreads();

  const int tiles_per_e = (PHASE == 1) ? P.I / 2 : P.d / kRW;
  const long long total = static_cast<long long>(n_act) * tiles_per_e;
  const long long nw = static_cast<long long>(gridDim.x) * kWarps;
  const long long gw = static_cast<long long>(blockIdx.x) * kWarps + warp;
  const long long beg = total * gw / nw, end = total * (gw + 1) / nw;
  for (long long w = beg; w < end; ++w) {
    const int e = s_act[w / tiles_per_e];
    const int tile = static_cast<int>(w % tiles_per_e);
    const int q0 = __ldg(P.offsets + e);
    const int ne = __ldg(P.offsets + e + 1) - q0;
    const uint8_t* blob = P.pool + static_cast<size_t>(__ldg(P.slot + e)) * P.blob_bytes;
    for (int tb = 0; tb < ne; tb += kNTMax) {
      const int nt = min(kNTMax, ne - tb);
      if (nt == 1) run_tile<FMT, PHASE, 1>(P, blob, tile, q0, tb, nt, lane);
      else if (nt == 2) run_tile<FMT, PHASE, 2>(P, blob, tile, q0, tb, nt, lane);
      else if (nt <= 4) run_tile<FMT, PHASE, 4>(P, blob, tile, q0, tb, nt, lane);
      else run_tile<FMT, PHASE, 8>(P, blob, tile, q0, tb, nt, lane);
    }
  }
}

template <int FMT, int PHASE>
moe_status launch_phase(const FfnParams& P, const DeviceInfo& dev, cudaStream_t s) {
  static int occ[64] = {};
  if (occ[dev.id] == 0) {
    int o = 0;
    MOE_CUDA_TRY(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&o, ffn_decode_kernel<FMT, PHASE>,
                                                               kWarps * 32, 0));
    occ[dev.id] = o > 0 ? o : 1;
  }
  const int tiles_per_e = (PHASE == 1) ? P.I / 2 : P.d / kRW;
  const long long most = static_cast<long long>(min(P.E, P.T * P.k)) * tiles_per_e;
  long long blocks = (most + kWarps - 1) / kWarps;
  const long long cap = static_cast<long long>(dev.sm_count) * occ[dev.id];
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  ffn_decode_kernel<FMT, PHASE><<<static_cast<int>(blocks), kWarps * 32, 0, s>>>(P);
  MOE_LAUNCH_CHECK("ffn_decode_kernel");
  return MOE_OK;
}

template <int FMT>
moe_status launch_decode(const FfnParams& P, const DeviceInfo& dev, cudaStream_t s) {
  moe_status st = launch_phase<FMT, 1>(P, dev, s);
  if (st != MOE_OK) return st;
  return launch_phase<FMT, 2>(P, dev, s);
}

}  // namespace

size_t decode_workspace_bytes(moe_shape s, int T, int k) {
  return round_up(static_cast<size_t>(T) * k * s.I * sizeof(float), 256);
}

moe_status launch_ffn_decode(moe_shape s, const void* x, int T, int k, const int32_t* offsets,
                             const int32_t* perm, const int32_t* slot, const void* pool, int n_slots,
                             const float* gate, float* y_perm, float* out, void* ws,
                             int32_t* status, const DeviceInfo& dev, cudaStream_t stream) {
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
