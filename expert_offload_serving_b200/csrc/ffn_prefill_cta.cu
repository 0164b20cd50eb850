// Step 3 (FP4 tensor-core path, MOE_FFN_ACT_NVFP4), single-CTA tiles: the
// grouped SwiGLU expert FFN as two block-scaled FP4 GEMMs on the
// 5th-generation tensor cores, for steps whose experts hold at most ~128
// token rows each (T * k <= 128 * E; ffn_prefill.cu runs the others on CTA
// pairs with 224-row chunks, which would pad such groups to 224).
//
// In prefill many tokens of a layer reach nearly every expert, so each
// expert's FFN is a dense contraction over a group of ~100 token rows
// (ainewsfeed.tech, second paragraph; explainx.ai hardware guide, "Prefill:
// load almost every expert without idling the GPU").  The pages give no
// kernel; on B200 the contraction belongs on tcgen05 with NVFP4 operands.
//
// Launches (one stream):
//   quant_tokens_cta x rows -> NVFP4 (E2M1 codes, one E4M3 scale per 16,
//                unit tensor scale), once per token;
//   gather_x128  copies them in expert order into an expert-padded layout:
//                expert e's rows start at a multiple of 128, so every
//                128-row B tile and its scale atoms align.
//   gemm<1>      D[128 x N] = W_gu tile (64 gate + 64 up rows) x X^T over K = d;
//                epilogue: a = silu(g_g * D_gate) * (g_u * D_up), requantised
//                to NVFP4 into the padded A matrix.
//   gemm<2>      D = W_d tile (128 rows of d) x A^T over K = I; epilogue:
//                out[t][row] += gate * g_d * D  (red.global.add.v4 on 4
//                consecutive rows after a shared-memory transpose: the combine).
// gemm is a persistent kernel, one CTA per SM, warp-specialised:
//   warp 0      TMA producer: 128x128-byte A and B tiles (SWIZZLE_128B, no
//               multicast) plus the 2 KB scale-atom slices by bulk copy, into
//               a 5-stage ring guarded by mbarriers;
//   warp 1      TMEM owner and MMA issuer: per stage, tcgen05.cp of the scale
//               atoms into TMEM, then 4 tcgen05.mma kind::mxf4nvf4 block16
//               (K = 64 each) into one of two TMEM accumulators;
//   warps 2-9   epilogue, two groups of four warps (each warp reads its 32
//               TMEM lanes; the groups take alternate 16-column slabs),
//               overlapped with the next tile's main loop.
// Every wait is bounded; on expiry the CTA records MOE_ERR_TIMEOUT in the
// status word, stops issuing, drains what it issued and frees its TMEM.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_fp16.h>

#include "common.cuh"
#include "tc.cuh"

namespace moe {
namespace {

using namespace ::moe::tc;

constexpr int BM = 128;                 // weight rows per tile
constexpr int BN = 128;                 // token rows per tile (max MMA N used)
constexpr int BKB = 128;                // bytes of K per stage (256 FP4 elements)
constexpr int STAGES = 5;
constexpr int A_BYTES = BM * BKB;       // 16 KB
constexpr int B_BYTES = BN * BKB;       // 16 KB
constexpr int SF_BYTES = 2048;          // 4 atoms of 128 rows x 4 scales
constexpr int STAGE_BYTES = A_BYTES + B_BYTES + 2 * SF_BYTES;
constexpr int EPI_GROUPS = 2;           // epilogue warp groups (each covers the 4 TMEM lane quadrants)
constexpr int EPI_THREADS = 128 * EPI_GROUPS;
constexpr int EPI_BYTES = EPI_GROUPS * 16 * 128 * 4 + 2 * 128 * 4;   // a transposed 16-column slab per group + column info
constexpr int TMEM_COLS = 512;
constexpr int ACC_COLS = 128;           // per accumulator buffer
constexpr int SFA_COL = 256, SFB_COL = 272;
constexpr int THREADS = 64 + EPI_THREADS;   // producer, MMA, epilogue groups

struct GemmParams {
  uint64_t wait_ns;          // limit of every bounded wait (default 2 s)
  int stall;                 // testing aid: CTA 0's epilogue waits on a barrier nothing arrives on
  int E, d, I, T, k, n_slots, max_chunks;
  const int32_t* offsets;
  const int32_t* perm;
  const int32_t* slot;
  const float* gate;
  const uint8_t* pool;       // slot pool
  size_t blob_bytes;
  BlobLayout L;
  const uint8_t* act_sf;     // scale atoms of the B operand
  uint8_t* aq;               // gemm<1> output codes  [rows][I/2]
  uint8_t* aq_sf;            // gemm<1> output scale atoms
  float* out;                // gemm<2> output [T][d]
  int32_t* status;
};

// ------------------------------------------------------------------ FP4 MMA wrappers
// Instruction descriptor: kind::mxf4nvf4, A and B E2M1 (packed), K-major,
// UE4M3 scales, M = 128, N = n.
__device__ __forceinline__ uint32_t idesc_fp4(int n) {
  return (1u << 7) | (1u << 10) | (static_cast<uint32_t>(n >> 3) << 17) | (static_cast<uint32_t>(BM >> 4) << 24);
}

__device__ __forceinline__ void tc_cp_sf(uint32_t tmem, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(tmem), "l"(sdesc) : "memory");
}

__device__ __forceinline__ void tc_mma_fp4(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc,
                                           uint32_t sfa, uint32_t sfb, uint32_t acc) {
  asm volatile(
      "{ .reg .pred p; setp.ne.b32 p, %6, 0; "
      "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%4], [%5], p; }" ::"r"(
          d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(sfa), "r"(sfb), "r"(acc)
      : "memory");
}


// ------------------------------------------------------------------ NVFP4 quantisation
// 16 values -> E4M3 scale byte s = e4m3_rn_satfinite(amax / 6) and 8 code
// bytes q_i = e2m1_rn_satfinite(v_i / s) (IEEE fp32 division; all zero when s
// is 0).  Element 2i goes to the low nibble.
__device__ __forceinline__ uint32_t e4m3_byte(float x) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(x));
  return r & 0xffu;
}

__device__ __forceinline__ float e4m3_value(uint32_t byte) {
  uint32_t h;
  asm("{ .reg .b16 s; cvt.u16.u32 s, %1; cvt.rn.f16x2.e4m3x2 %0, s; }" : "=r"(h) : "r"(byte));
  return __half2float(__ushort_as_half(static_cast<unsigned short>(h & 0xffffu)));
}

__device__ __forceinline__ uint32_t e2m1x2_byte(float lo, float hi) {
  uint32_t r;
  asm("{ .reg .b8 b; cvt.rn.satfinite.e2m1x2.f32 b, %1, %2; cvt.u32.u8 %0, b; }" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// codes of 8 values (already divided by the scale) -> 4 bytes
__device__ __forceinline__ uint32_t pack8(const float (&q)[8]) {
  return e2m1x2_byte(q[0], q[1]) | (e2m1x2_byte(q[2], q[3]) << 8) | (e2m1x2_byte(q[4], q[5]) << 16) |
         (e2m1x2_byte(q[6], q[7]) << 24);
}

// ------------------------------------------------------------------ shared prologue
// Chunks: 128-row pieces of each evaluated expert's group (tokens > 0,
// slot >= 0).  chunk_start[e] = exclusive prefix of the chunk counts; chunk c
// occupies padded rows [128 c, 128 c + 128).
__device__ int build_chunks(const int32_t* __restrict__ offsets, const int32_t* __restrict__ slot, int E,
                            int n_pairs, int n_slots, int32_t* chunk_start, int* ws, int32_t* status) {
  const int per = (E + blockDim.x - 1) / blockDim.x;
  const int e0 = threadIdx.x * per;
  int cnt = 0;
  for (int j = 0; j < per; ++j) {
    const int e = e0 + j;
    if (e >= E) break;
    const int a = offsets[e], b = offsets[e + 1];
    int c = 0;
    if (b > a) {
      if (a < 0 || b > n_pairs) {
        report(status, MOE_ERR_DEVICE);
      } else {
        const int s = slot[e];
        if (s >= n_slots) report(status, MOE_ERR_DEVICE);
        else if (s >= 0) c = (b - a + BN - 1) / BN;
      }
    }
    cnt += c;
  }
  // block exclusive scan of cnt
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = cnt;
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
  int run = ws[warp] + x - cnt;
  for (int j = 0; j < per; ++j) {
    const int e = e0 + j;
    if (e >= E) break;
    chunk_start[e] = run;
    const int a = offsets[e], b = offsets[e + 1];
    if (b > a && a >= 0 && b <= n_pairs) {
      const int s = slot[e];
      if (s >= 0 && s < n_slots) run += (b - a + BN - 1) / BN;
    }
  }
  const int total = ws[32];
  if (threadIdx.x == 0) chunk_start[E] = total;
  __syncthreads();
  return total;
}

// Unit u -> (chunk, M tile), chunk-major for both GEMMs: the CTAs working at
// the same time share one activation tile, and the M tiles of an expert with
// several chunks are re-read while still in L2.  (Measured against M-tile-major
// order for GEMM2, which keeps one 128-column slab of out hot for the fused
// combine: equal at T = 4096, 8-9 % slower at T >= 16384.)
__device__ __forceinline__ void unit_coords(int u, int MT, int* c, int* m) {
  *c = u / MT;
  *m = u % MT;
}

// expert of chunk c: the last e with chunk_start[e] <= c
__device__ __forceinline__ int chunk_expert(const int32_t* chunk_start, int E, int c) {
  int lo = 0, hi = E;   // invariant: chunk_start[lo] <= c < chunk_start[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (chunk_start[mid] <= c) lo = mid;
    else hi = mid;
  }
  return lo;
}

// ------------------------------------------------------------------ quant_x
// NVFP4 quantisation of each token row once (T rows, not T*k): codes into
// xt[t][d/2] and scale bytes into xts[t][d/16], one warp per row.
__global__ void __launch_bounds__(256) quant_tokens_cta_kernel(const uint16_t* __restrict__ x, int d, int T,
                                                          uint8_t* __restrict__ xt, uint8_t* __restrict__ xts) {
  const int lane = threadIdx.x & 31;
  const int warps = blockDim.x >> 5;
  const int nb = d / 16;
  for (int t = blockIdx.x * warps + (threadIdx.x >> 5); t < T; t += gridDim.x * warps) {
    const uint16_t* xr = x + static_cast<size_t>(t) * d;
    for (int b = lane; b < nb; b += 32) {
      const uint4 u0 = __ldg(reinterpret_cast<const uint4*>(xr + 16 * b));
      const uint4 u1 = __ldg(reinterpret_cast<const uint4*>(xr + 16 * b + 8));
      const uint32_t w32[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
      float v[16];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        v[2 * j] = __uint_as_float(w32[j] << 16);
        v[2 * j + 1] = __uint_as_float(w32[j] & 0xffff0000u);
      }
      float amax = 0.f;
#pragma unroll
      for (int j = 0; j < 16; ++j) amax = fmaxf(amax, fabsf(v[j]));
      const uint32_t sb = e4m3_byte(__fdiv_rn(amax, 6.0f));
      const float s = e4m3_value(sb);
      float q0[8], q1[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        q0[j] = (s > 0.f) ? __fdiv_rn(v[j], s) : 0.f;
        q1[j] = (s > 0.f) ? __fdiv_rn(v[8 + j], s) : 0.f;
      }
      *reinterpret_cast<uint2*>(xt + static_cast<size_t>(t) * (d / 2) + 8 * b) = make_uint2(pack8(q0), pack8(q1));
      xts[static_cast<size_t>(t) * nb + b] = static_cast<uint8_t>(sb);
    }
  }
}

// Gather: every real row of every chunk copies its token's codes into
// xq[128 c + r][d/2] and its scale bytes, 4 blocks (one atom row) at a
// time, into the atom layout of the padded matrix.  One warp per row.
__global__ void __launch_bounds__(256) gather_x128_kernel(const uint8_t* __restrict__ xt,
                                                      const uint8_t* __restrict__ xts, int d, int T, int k, int E,
                                                      int n_slots, const int32_t* __restrict__ offsets,
                                                      const int32_t* __restrict__ perm,
                                                      const int32_t* __restrict__ slot, uint8_t* __restrict__ xq,
                                                      uint8_t* __restrict__ xsf, int32_t* status) {
  __shared__ int32_t chunk_start[1025];
  __shared__ int ws[36];
  const int n_pairs = T * k;
  const int n_chunks = build_chunks(offsets, slot, E, n_pairs, n_slots, chunk_start, ws, status);
  const int lane = threadIdx.x & 31;
  const int warps = blockDim.x >> 5;
  const long long rows = static_cast<long long>(n_chunks) * BN;
  const int row_bytes = d / 2, nb = d / 16;
  for (long long w = static_cast<long long>(blockIdx.x) * warps + (threadIdx.x >> 5); w < rows;
       w += static_cast<long long>(gridDim.x) * warps) {
    const int c = static_cast<int>(w / BN), r = static_cast<int>(w % BN);
    const int e = chunk_expert(chunk_start, E, c);
    const int q = offsets[e] + (c - chunk_start[e]) * BN + r;
    if (q >= offsets[e + 1]) continue;                      // padding row: never read back
    int p = perm[q];
    if (p < 0 || p >= n_pairs) {
      report(status, MOE_ERR_DEVICE);
      p = 0;
    }
    const int t = p / k;
    const int prow = c * BN + r;
    const uint4* src = reinterpret_cast<const uint4*>(xt + static_cast<size_t>(t) * row_bytes);
    uint4* dst = reinterpret_cast<uint4*>(xq + static_cast<size_t>(prow) * row_bytes);
    for (int i = lane; i < row_bytes / 16; i += 32) dst[i] = __ldg(src + i);
    const uint32_t* ssrc = reinterpret_cast<const uint32_t*>(xts + static_cast<size_t>(t) * nb);
    for (int g = lane; g < nb / 4; g += 32)
      *reinterpret_cast<uint32_t*>(xsf + sf_atom_offset(prow, 4 * g, d)) = __ldg(ssrc + g);
  }
}

// ------------------------------------------------------------------ the GEMMs
template <int PHASE>
__global__ void __launch_bounds__(THREADS, 1) gemm_fp4_cta_kernel(const __grid_constant__ CUtensorMap tm_w,
                                                              const __grid_constant__ CUtensorMap tm_act,
                                                              GemmParams P) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stage_base = smem;
  float* epi_all = reinterpret_cast<float*>(smem + STAGES * STAGE_BYTES);
  int32_t* col_t = reinterpret_cast<int32_t*>(epi_all + EPI_GROUPS * 16 * 128);
  float* col_g = reinterpret_cast<float*>(col_t + 128);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES + EPI_BYTES);
  uint64_t* full = bars;                   // [STAGES]
  uint64_t* empty = bars + STAGES;         // [STAGES]
  uint64_t* tfull = bars + 2 * STAGES;     // [2]
  uint64_t* tempty = bars + 2 * STAGES + 2;// [2]
  uint64_t* drain = bars + 2 * STAGES + 4; // [1]
  uint64_t* stall = bars + 2 * STAGES + 5; // [1] never arrived on (testing aid)
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 6);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  volatile int* epi_fail = reinterpret_cast<volatile int*>(tmem_holder + 2);
  int32_t* chunk_start = reinterpret_cast<int32_t*>(tmem_holder + 4);   // [E+1]
  __shared__ int ws[36];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int K = (PHASE == 1) ? P.d : P.I;
  const int KS = K / (2 * BKB);                 // stages of 256 elements
  const int MT = (PHASE == 1) ? (2 * P.I) / BM : P.d / BM;
  const int n_pairs = P.T * P.k;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], EPI_THREADS);
    }
    mbar_init(drain, 1);
    mbar_init(stall, 1);
    *abort_flag = 0;
    *epi_fail = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_holder)),
                 "r"(TMEM_COLS));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  const int n_chunks = build_chunks(P.offsets, P.slot, P.E, n_pairs, P.n_slots, chunk_start, ws, P.status);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const int n_chunks_used = min(n_chunks, P.max_chunks);
  const int n_units = n_chunks_used * MT;

  if (warp == 0) {
    // ---------------------------------------------------------- TMA producer
    const uint64_t pol_stream = policy_evict_first(), pol_keep = policy_evict_last();
    int stage = 0;
    uint32_t phase = 0;
    int issued = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
      int c, m;
      unit_coords(u, MT, &c, &m);
      const int e = chunk_expert(chunk_start, P.E, c);
      const int sl = P.slot[e];
      const uint8_t* sfa_src = P.pool + static_cast<size_t>(sl) * P.blob_bytes +
                               (PHASE == 1 ? P.L.sg : P.L.sd) + static_cast<size_t>(m) * (K / 64) * 512;
      const uint8_t* sfb_src = P.act_sf + static_cast<size_t>(c) * (K / 64) * 512;
      // a weight tile read by one chunk streams through L2; one that the
      // expert's further chunks read again is kept
      const uint64_t pol_a = (chunk_start[e + 1] - chunk_start[e] > 1) ? pol_keep : pol_stream;
      for (int ks = 0; ks < KS; ++ks) {
        if (!__all_sync(kFull, mbar_wait(&empty[stage], phase ^ 1u, abort_flag, P.wait_ns))) {
          ok = false;
          break;
        }
        if (elect_one()) {
          uint8_t* sA = stage_base + stage * STAGE_BYTES;
          uint8_t* sB = sA + A_BYTES;
          uint8_t* sSFA = sB + B_BYTES;
          uint8_t* sSFB = sSFA + SF_BYTES;
          mbar_expect_tx(&full[stage], STAGE_BYTES);
          tma_load_3d(sA, &tm_w, &full[stage], ks * BKB, m * BM, sl, pol_a);
          tma_load_2d(sB, &tm_act, &full[stage], ks * BKB, c * BN, pol_keep);
          bulk_load(sSFA, sfa_src + ks * SF_BYTES, SF_BYTES, &full[stage], pol_a);
          bulk_load(sSFB, sfb_src + ks * SF_BYTES, SF_BYTES, &full[stage], pol_keep);
        }
        __syncwarp();
        ++issued;
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
    if (!ok) {
      report(P.status, MOE_ERR_TIMEOUT);
      *abort_flag = 1;
    }
    // drain: wait (bounded) until the copies last issued into the ring have
    // landed, so none is in flight when the CTA exits
    const int outstanding = issued < STAGES ? issued : STAGES;
    int s = stage;
    uint32_t ph = phase;
    for (int i = 0; i < outstanding; ++i) {
      if (--s < 0) {
        s = STAGES - 1;
        ph ^= 1u;
      }
      mbar_drain(&full[s], ph);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    int stage = 0;
    uint32_t phase = 0;
    int it = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x, ++it) {
      int c, m_unused;
      unit_coords(u, MT, &c, &m_unused);
      const int e = chunk_expert(chunk_start, P.E, c);
      const int row0 = P.offsets[e] + (c - chunk_start[e]) * BN;
      const int nvalid = min(BN, P.offsets[e + 1] - row0);
      const int nmma = (nvalid + 15) & ~15;
      const uint32_t idesc = idesc_fp4(nmma);
      const int acc = it & 1;
      if (!__all_sync(kFull, mbar_wait(&tempty[acc], ((it >> 1) & 1) ^ 1u, abort_flag, P.wait_ns))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t d_tmem = tmem + acc * ACC_COLS;
      for (int ks = 0; ks < KS; ++ks) {
        if (!__all_sync(kFull, mbar_wait(&full[stage], phase, abort_flag, P.wait_ns))) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (elect_one()) {
          uint8_t* sA = stage_base + stage * STAGE_BYTES;
          uint8_t* sB = sA + A_BYTES;
          uint8_t* sSFA = sB + B_BYTES;
          uint8_t* sSFB = sSFA + SF_BYTES;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            tc_cp_sf(tmem + SFA_COL + 4 * j, desc_sf(smem_u32(sSFA + 512 * j)));
            tc_cp_sf(tmem + SFB_COL + 4 * j, desc_sf(smem_u32(sSFB + 512 * j)));
          }
          const uint64_t da = desc_sw128(smem_u32(sA));
          const uint64_t db = desc_sw128(smem_u32(sB));
#pragma unroll
          for (int j = 0; j < 4; ++j)
            tc_mma_fp4(d_tmem, da + 2 * j, db + 2 * j, idesc, tmem + SFA_COL + 4 * j, tmem + SFB_COL + 4 * j,
                       (ks > 0 || j > 0) ? 1u : 0u);
          tc_commit(&empty[stage]);
        }
        __syncwarp();
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (!ok) break;
      if (elect_one()) tc_commit(&tfull[acc]);
      __syncwarp();
    }
    if (!ok) {
      report(P.status, MOE_ERR_TIMEOUT);
      *abort_flag = 1;
    }
    // every MMA this thread issued has completed before TMEM is released
    if (elect_one()) tc_commit(drain);
    __syncwarp();
    mbar_drain(drain, 0);
  } else {
    // ---------------------------------------------------------- epilogue (warps 2..9)
    const int quad = warp & 3;                  // TMEM lanes 32*quad .. 32*quad+31
    const int grp = (warp - 2) >> 2;            // column group: slabs grp, grp+2, ...
    const int et = ((warp - 2) & 3) * 32 + lane;   // 0..127 within the group
    const int eall = (warp - 2) * 32 + lane;       // 0..255 over both groups
    float* epi = epi_all + grp * 16 * 128;
    const int bar_grp = 1 + grp, bar_all = 3;
    const float* ts = nullptr;
    int it = 0;
    // testing aid (moe_set_test_stall): CTA 0's epilogue first waits on a
    // barrier that nothing arrives on, so the bounded wait runs out and the
    // abort path (record, stop issuing, drain, free TMEM) runs for real
    bool ok = !(P.stall && blockIdx.x == 0 && !mbar_wait(stall, 0, abort_flag, P.wait_ns));
    for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x, ++it) {
      int c, m;
      unit_coords(u, MT, &c, &m);
      const int e = chunk_expert(chunk_start, P.E, c);
      const int row0 = P.offsets[e] + (c - chunk_start[e]) * BN;
      const int nvalid = min(BN, P.offsets[e + 1] - row0);
      const uint8_t* blob = P.pool + static_cast<size_t>(P.slot[e]) * P.blob_bytes;
      ts = reinterpret_cast<const float*>(blob + P.L.ts);
      const int acc = it & 1;
      if (PHASE == 2) {
        // column c <-> pair at sorted position row0 + c: its token and gate
        named_sync(bar_all, EPI_THREADS);       // the previous tile's readers are done
        if (eall < nvalid) {
          const int p = P.perm[row0 + eall];
          const bool good = p >= 0 && p < n_pairs;
          if (!good) report(P.status, MOE_ERR_DEVICE);
          col_t[eall] = good ? p / P.k : -1;
          col_g[eall] = good ? P.gate[p] : 0.f;
        }
      }
      // the eight epilogue warps agree before any leaves: a warp alone at a
      // named barrier would wait for good (this barrier also publishes the
      // column info written above)
      if (!mbar_wait(&tfull[acc], (it >> 1) & 1, abort_flag, P.wait_ns)) *epi_fail = 1;
      named_sync(bar_all, EPI_THREADS);
      if (*epi_fail) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t tbase = tmem + (static_cast<uint32_t>(32 * quad) << 16) + acc * ACC_COLS;
      const float g_mat = (PHASE == 1) ? 0.f : __ldg(ts + 2);
      const float g_gate = (PHASE == 1) ? __ldg(ts + 0) : 0.f, g_up = (PHASE == 1) ? __ldg(ts + 1) : 0.f;
      for (int cc = 16 * grp; cc < nvalid; cc += 16 * EPI_GROUPS) {
        float v[16];
        tmem_ld16(tbase + cc, v);
        if (PHASE == 2) {
          // transpose the slab through shared memory (epi[col][row]), then each
          // thread adds 4 consecutive output rows of one column with one
          // vector reduction: out[t][row .. row+3] += gate * g_d * y
#pragma unroll
          for (int j = 0; j < 16; ++j) epi[j * 128 + 32 * quad + lane] = v[j];
          named_sync(bar_grp, 128);
#pragma unroll
          for (int it2 = 0; it2 < 4; ++it2) {
            const int item = et + 128 * it2;          // 16 columns x 32 row quads
            const int cl = item >> 5, rq = item & 31;
            const int col = cc + cl;
            if (col < nvalid) {
              const int t = col_t[col];
              if (t >= 0) {
                const float gm = col_g[col] * g_mat;
                const float4 y = *reinterpret_cast<const float4*>(epi + cl * 128 + 4 * rq);
                float* dst = P.out + static_cast<size_t>(t) * P.d + m * BM + 4 * rq;
                asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(dst), "f"(gm * y.x),
                             "f"(gm * y.y), "f"(gm * y.z), "f"(gm * y.w)
                             : "memory");
              }
            }
          }
          named_sync(bar_grp, 128);
        } else {
          // transpose the 16-column slab through shared memory: epi[col][row]
#pragma unroll
          for (int j = 0; j < 16; ++j) epi[j * 128 + 32 * quad + lane] = v[j];
          named_sync(bar_grp, 128);
          // item: column cl, 16-block b of the 64 intermediate indices, half h
          const int cl = et >> 3, b = (et >> 1) & 3, h = et & 1;
          const int col = cc + cl;
          float a[8];
          float amax = 0.f;
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const int il = 16 * b + 8 * h + j;
            const float hg = epi[cl * 128 + il] * g_gate;
            const float hu = epi[cl * 128 + 64 + il] * g_up;
            a[j] = __fdividef(hg, 1.0f + __expf(-hg)) * hu;
            amax = fmaxf(amax, fabsf(a[j]));
          }
          amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, 1));
          const uint32_t sb = e4m3_byte(__fdiv_rn(amax, 6.0f));
          const float s = e4m3_value(sb);
          float q[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) q[j] = (s > 0.f) ? __fdiv_rn(a[j], s) : 0.f;
          const uint32_t codes = pack8(q);
          if (col < nvalid) {
            const int prow = c * BN + col;
            const int i0 = m * 64;                       // first intermediate index of the tile
            *reinterpret_cast<uint32_t*>(P.aq + static_cast<size_t>(prow) * (P.I / 2) + (i0 + 16 * b + 8 * h) / 2) =
                codes;
            if (h == 0) P.aq_sf[sf_atom_offset(prow, i0 / 16 + b, P.I)] = static_cast<uint8_t>(sb);
          }
          named_sync(bar_grp, 128);
        }
      }
      tc_fence_before();
      mbar_arrive(&tempty[acc]);
    }
    if (!ok) {
      report(P.status, MOE_ERR_TIMEOUT);
      *abort_flag = 1;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS));
  }
}

// ------------------------------------------------------------------ host side
// Byte-element tensor map, box 128 (bytes of K) x 128 rows, 128-byte swizzle.
moe_status make_map(CUtensorMap* map, const void* base, int rank, const uint64_t* dims, const uint64_t* strides) {
  const uint32_t box[3] = {static_cast<uint32_t>(BKB), 128u, 1u};
  const CUresult r = encode_tiled_sw128(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, rank, base, dims, strides, box);
  if (r == CUDA_ERROR_NOT_FOUND) return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
  if (r != CUDA_SUCCESS) return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
  return MOE_OK;
}

struct PrefillWs {
  size_t rows;            // padded row capacity (multiple of 128)
  size_t xt, xts, xq, xsf, aq, asf, bytes;
};

PrefillWs prefill_ws(moe_shape s, int T, int k) {
  PrefillWs w{};
  const size_t n = static_cast<size_t>(T) * k;
  const size_t act = n < static_cast<size_t>(s.E) ? n : static_cast<size_t>(s.E);
  w.rows = round_up(n + act * (BN - 1), BN);
  size_t o = 0;
  w.xt = o; o = round_up(o + static_cast<size_t>(T) * (s.d / 2), 1024);
  w.xts = o; o = round_up(o + static_cast<size_t>(T) * (s.d / 16), 1024);
  w.xq = o; o = round_up(o + w.rows * (s.d / 2), 1024);
  w.xsf = o; o = round_up(o + w.rows * (s.d / 16), 1024);
  w.aq = o; o = round_up(o + w.rows * (s.I / 2), 1024);
  w.asf = o; o = round_up(o + w.rows * (s.I / 16), 1024);
  w.bytes = o;
  return w;
}

constexpr size_t kGemmSmem = STAGES * STAGE_BYTES + EPI_BYTES + 256 + 1025 * 4 + 1024;
static_assert((2 * STAGES + 6) * 8 + 16 <= 256, "barrier area");

}  // namespace

size_t prefill_cta_workspace_bytes(moe_shape s, int T, int k) { return prefill_ws(s, T, k).bytes; }

moe_status launch_ffn_prefill_cta(moe_shape s, const void* x, int T, int k, const int32_t* offsets,
                                  const int32_t* perm, const int32_t* slot, const void* pool, int n_slots,
                                  const float* gate, float* out, void* ws_ptr, int32_t* status,
                                  const DeviceInfo& dev, cudaStream_t stream) {
  MOE_REQUIRE(s.d % 256 == 0 && s.I % 256 == 0, "the FP4 tensor-core path needs d, I multiples of 256");
  if (kGemmSmem > dev.smem_optin)
    return fail(MOE_ERR_UNSUPPORTED, "needs %zu bytes of shared memory per CTA", kGemmSmem);
  const PrefillWs w = prefill_ws(s, T, k);
  uint8_t* base = static_cast<uint8_t*>(ws_ptr);
  uint8_t* xq = base + w.xq;
  uint8_t* xsf = base + w.xsf;
  uint8_t* aq = base + w.aq;
  uint8_t* asf = base + w.asf;
  const BlobLayout L = blob_layout(s.fmt, s.d, s.I);
  const int max_chunks = static_cast<int>(w.rows / BN);

  static bool attr_done[64] = {};
  if (!attr_done[dev.id]) {
    MOE_CUDA_TRY(cudaFuncSetAttribute(gemm_fp4_cta_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      static_cast<int>(kGemmSmem)));
    MOE_CUDA_TRY(cudaFuncSetAttribute(gemm_fp4_cta_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      static_cast<int>(kGemmSmem)));
    attr_done[dev.id] = true;
  }

  // tensor maps: weights [slot][rows][K bytes], activations [rows][K bytes]
  CUtensorMap tm_gu, tm_d, tm_x, tm_a;
  const uint8_t* pool8 = static_cast<const uint8_t*>(pool);
  {
    const uint64_t dims[3] = {static_cast<uint64_t>(s.d / 2), static_cast<uint64_t>(2 * s.I),
                              static_cast<uint64_t>(n_slots)};
    const uint64_t str[2] = {static_cast<uint64_t>(s.d / 2), L.bytes};
    moe_status st = make_map(&tm_gu, pool8 + L.wg, 3, dims, str);
    if (st != MOE_OK) return st;
  }
  {
    const uint64_t dims[3] = {static_cast<uint64_t>(s.I / 2), static_cast<uint64_t>(s.d),
                              static_cast<uint64_t>(n_slots)};
    const uint64_t str[2] = {static_cast<uint64_t>(s.I / 2), L.bytes};
    moe_status st = make_map(&tm_d, pool8 + L.wd, 3, dims, str);
    if (st != MOE_OK) return st;
  }
  {
    const uint64_t dims[2] = {static_cast<uint64_t>(s.d / 2), w.rows};
    const uint64_t str[1] = {static_cast<uint64_t>(s.d / 2)};
    moe_status st = make_map(&tm_x, xq, 2, dims, str);
    if (st != MOE_OK) return st;
  }
  {
    const uint64_t dims[2] = {static_cast<uint64_t>(s.I / 2), w.rows};
    const uint64_t str[1] = {static_cast<uint64_t>(s.I / 2)};
    moe_status st = make_map(&tm_a, aq, 2, dims, str);
    if (st != MOE_OK) return st;
  }

  {
    const long long rows = static_cast<long long>(w.rows);
    long long blocks = (rows + 7) / 8;
    const long long cap = static_cast<long long>(dev.sm_count) * 8;
    if (blocks > cap) blocks = cap;
    long long tb = (static_cast<long long>(T) + 7) / 8;
    if (tb > cap) tb = cap;
    quant_tokens_cta_kernel<<<static_cast<int>(tb), 256, 0, stream>>>(static_cast<const uint16_t*>(x), s.d, T,
                                                                 base + w.xt, base + w.xts);
    MOE_LAUNCH_CHECK("quant_tokens_cta_kernel");
    gather_x128_kernel<<<static_cast<int>(blocks), 256, 0, stream>>>(base + w.xt, base + w.xts, s.d, T, k, s.E,
                                                                  n_slots, offsets, perm, slot, xq, xsf, status);
    MOE_LAUNCH_CHECK("gather_x128_kernel");
  }
  GemmParams P{};
  P.wait_ns = wait_limit_ns();
  P.stall = test_stall();
  P.E = s.E;
  P.d = s.d;
  P.I = s.I;
  P.T = T;
  P.k = k;
  P.n_slots = n_slots;
  P.max_chunks = max_chunks;
  P.offsets = offsets;
  P.perm = perm;
  P.slot = slot;
  P.gate = gate;
  P.pool = pool8;
  P.blob_bytes = L.bytes;
  P.L = L;
  P.status = status;
  P.out = out;
  const int grid = dev.sm_count;
  P.act_sf = xsf;
  P.aq = aq;
  P.aq_sf = asf;
  gemm_fp4_cta_kernel<1><<<grid, THREADS, kGemmSmem, stream>>>(tm_gu, tm_x, P);
  MOE_LAUNCH_CHECK("gemm_fp4_cta_kernel<1>");
  P.act_sf = asf;
  gemm_fp4_cta_kernel<2><<<grid, THREADS, kGemmSmem, stream>>>(tm_d, tm_a, P);
  MOE_LAUNCH_CHECK("gemm_fp4_cta_kernel<2>");
  return MOE_OK;
}

}  // namespace moe
