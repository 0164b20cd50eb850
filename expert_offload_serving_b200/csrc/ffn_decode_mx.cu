// Step 3 at decode sizes for MXFP4 weights on the 5th-generation tensor cores
// (moe_expert_ffn without MOE_FFN_ACT_NVFP4, MXFP4 blobs in the stage-tiled
// layout, i.e. d and I multiples of 256): the grouped SwiGLU expert FFN as two
// skinny block-scaled GEMMs that read the E2M1 weights as stored.
//
// A decode layer call is bound by reading the routed experts' weights from HBM
// (explainx.ai hardware guide, "Decode: decide whether to move an expert or
// compute where it lives").  The weights are never converted on the SM: TMA
// loads each stage's packed E2M1 codes with the 16U4_ALIGN16B expansion (16
// codes into every 16-byte slot, the operand layout of
// tcgen05.mma kind::mxf8f6f4), the E8M0 block scales go to TMEM by tcgen05.cp,
// and the tensor core applies them (block_scale, one scale per 32 K elements).
//
// That kind multiplies FP8/FP6/FP4 by FP8/FP6/FP4, so the activations enter as
// sums of E4M3 terms, each term with its own E8M0 scale per 32 elements
// (chosen from the block's largest remaining magnitude, so no term saturates):
//   x (bf16, 8 significant bits)  -> 2 terms, exact unless an element is more
//                                     than ~2^18 below its block's maximum;
//   a (fp32, the SwiGLU output)   -> 4 terms (16 significant bits), residual
//                                     below 2^-16 of each block's maximum.
// The terms are stacked along N: term j's TN token rows are B rows
// j*TN .. j*TN+TN-1, so one MMA per 32-element K step reads the weight tile
// from shared memory once for all terms (a skinny MMA costs about the same
// whatever its N: the A operand read dominates), and the epilogue adds the
// terms' fp32 accumulator columns.
//
//   split_x:  x [T][d] -> 2 E4M3 planes + 2 scale planes, once per token.
//   gemv<1>:  D[128 x 2 TN] = W_gu tile (64 gate + 64 up rows of the same
//             intermediate indices) x [X_0; X_1]^T over K = d, the x terms
//             of <= TN token rows gathered by one-row TMA loads.  Epilogue: a = silu(D_gate) *
//             D_up split into 4 E4M3 planes + scales (warp-wide maxima over
//             the 32 lanes = one 32-element block of I).
//   gemv<2>:  D[128 x 4 TN] = W_d tile x [A_0; A_1; A_2; A_3]^T over K = I.
//             Epilogue: y_perm rows, or out[t] += gate * y (fused combine).
//
// Work unit = (expert, 128-row tile, chunk of <= TN pairs), expert-major,
// dealt round-robin to one persistent CTA per SM.  Warp 0 produces the weight
// stages (two TMA boxes + one bulk copy of the scale atoms per 17 KB tile,
// with an L2 prefetch cursor PF_ITEMS tiles ahead), warp 1 owns TMEM and
// issues tcgen05.cp + tcgen05.mma, warps 2-5 run the epilogue on
// double-buffered accumulators, warp 6 loads the token-row terms and their
// scale atoms.  Every wait is bounded: on expiry the CTA records
// MOE_ERR_TIMEOUT, stops issuing, drains what it issued and frees its TMEM.
#include <algorithm>
#include <cstdlib>

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "common.cuh"
#include "tc.cuh"

namespace moe {

namespace {

using namespace ::moe::tc;

constexpr int TM = 128;                    // weight rows per tile
constexpr int KSTAGE = 256;                // K elements per stage (one blob tile)
constexpr int A_BOX = 128 * 128;           // one TMA box: 128 rows x 128 padded codes
constexpr int A_SMEM = 2 * A_BOX + 1024;   // codes (expanded) + 2 scale atoms
// bytes a weight stage's barrier expects: the 16U4_ALIGN16B loads count the
// packed codes they read (8 KB per box), not the expanded 16 KB they write
constexpr uint32_t A_TX = 2 * (A_BOX / 2) + 1024;
constexpr int ACC_COLS = 128;              // 4 terms x 32 token rows
constexpr int SFA_COL = 2 * ACC_COLS;      // TMEM: 2 accumulators, then scale factors
constexpr int SFB_COL = SFA_COL + 8;
constexpr int TMEM_COLS = 512;
constexpr int NX = 2;                      // E4M3 terms of x
constexpr int NA = 4;                      // E4M3 terms of a
constexpr int PF_ITEMS = 2;                // L2 prefetch distance (tiles; measured best of 0, 2, 4, 8, 12)
constexpr int kSmemBudget = 226 * 1024;
constexpr int kMaxE = 1024;
constexpr int kBarBytes = 512;
constexpr int THREADS = 7 * 32;
constexpr int BPROD_WARP = 6;

struct MxParams {
  uint64_t wait_ns;          // limit of every bounded wait (default 2 s)
  int pf_items;              // L2 prefetch distance in stages
  int stall;                 // testing aid: CTA 0's epilogue waits on a barrier nothing arrives on
  int E, d, I, T, k, n_slots;
  int a_rows;              // rows of each a-term plane: max(T*k, 32), so a TN-row box always fits
  int x_rows;              // rows of each x-term plane: max(T, 32)
  const int32_t* offsets;
  const int32_t* perm;
  const int32_t* slot;
  const float* gate;
  const uint8_t* pool;
  size_t blob_bytes;
  BlobLayout L;
  const uint8_t* xs;       // [32/TN][d/128][x_rows][16] E8M0 scales of the x terms (sf_plane / sf_byte)
  uint8_t* aq;             // [NA][a_rows][I] E4M3 terms of a (rows = sorted pairs)
  uint8_t* as;             // [32/TN][I/128][a_rows][16] their E8M0 scales (sf_plane / sf_byte)
  int32_t* done1;          // one-launch schedule: per expert, gate/up units finished (zeroed before)
  float* y_perm;
  float* out;
  int32_t* status;
};

// Tensor maps of one launch: the weight tiles of both GEMVs; the x terms as
// one-row boxes (TN = 32: the rows of a unit's pairs, gathered) and as boxes
// of TN rows of both terms with their scale rows (TN <= 16: every token of
// the step); the a terms and their scale rows (boxes of TN rows of every
// term, resp. every scale plane).  A TN-row box is the stacked B operand of
// one 128-element half in one copy.
struct MxMaps {
  CUtensorMap w1, w2, x, xall, xs, a, as;
};

// Scale rows of stacked terms.  B row r = j*TN + t (term j, token row t)
// takes its 4 scales of a 128-element half from byte 4*(r/32) of the 16-byte
// row r%32 of the half's scale-factor atom.  With G = 32/TN term row blocks
// per 32 atom rows, term j sits in plane j%G (atom rows (j%G)*TN + t) at byte
// group j/G, so the scale rows are stored [plane][atom][row] with 16 bytes
// per row: a copy of TN consecutive rows of one atom of each plane (one
// contiguous run per plane) lands in place.
template <int TN>
__device__ __forceinline__ int sf_plane(int j) { return j % (32 / TN); }
template <int TN>
__device__ __forceinline__ int sf_byte(int j) { return 4 * (j / (32 / TN)); }

template <int PHASE, int TN>
struct Cfg {
  static constexpr int NT = PHASE == 1 ? NX : NA;                // terms of the B operand (PHASE 3: both GEMVs)
  static constexpr int G = 32 / TN;                              // term planes per 32 scale-atom rows
  static constexpr int B_ATOM = TN * 128;                        // TN rows x 128 E4M3 values
  static constexpr int B_CODES = NT * 2 * B_ATOM;                // per 128-element half: the terms' rows stacked
  static constexpr int B_STAGE = B_CODES + 1024;                 // + one scale atom per half
  static constexpr int UP_BYTES = PHASE != 2 ? 64 * 33 * 4 : 0;
  static constexpr int FIXED = 1024 + UP_BYTES + kBarBytes + 3 * (kMaxE + 1) * 4;   // + the unit table
  // token-row stages: the rows come from L2 (x, or the a terms gemv<1> just
  // wrote), and the ring must cover an L2 round trip at the weight stream's
  // pace (~0.4 us per stage): 4 where they fit beside 4+ weight stages
  static constexpr int SB = B_STAGE <= 12 * 1024 ? 4 : (PHASE == 1 ? 3 : 2);
  static constexpr int SA_FIT = (kSmemBudget - FIXED - SB * B_STAGE) / A_SMEM;
  static constexpr int SA = SA_FIT > 8 ? 8 : SA_FIT;
  static constexpr int A_RING = SA * A_SMEM;
  static constexpr int B_RING = SB * B_STAGE;
  static constexpr int N_BARS = 2 * SA + 2 * SB + 6;
  static_assert(TN == 8 || TN == 16 || TN == 32, "chunk width");
  static_assert(A_SMEM % 1024 == 0 && B_STAGE % 1024 == 0 && B_ATOM % 1024 == 0, "1024-byte alignment");
  static_assert(SA >= 3, "weight ring");
  static_assert(FIXED + A_RING + B_RING <= kSmemBudget, "shared memory budget");
  static_assert(SFB_COL + 8 <= TMEM_COLS && NT * TN <= ACC_COLS, "TMEM budget");
  static_assert(N_BARS * 8 + 16 <= kBarBytes, "barrier area");
};

template <int PHASE, int TN>
constexpr size_t smem_bytes(int E) {
  using C = Cfg<PHASE, TN>;
  return 1024 + static_cast<size_t>(C::A_RING) + C::B_RING + C::UP_BYTES + kBarBytes +
         3 * static_cast<size_t>(E + 1) * 4;
}

struct Unit {
  int e, m, q0, nvalid, ph;   // ph: 1 = gate/up GEMV, 2 = down GEMV
};

// unit u -> (phase, expert, tile, chunk of TN pairs).  ustart[e] = first unit
// of expert e in the table built with tiles1 tiles per chunk.  The one-launch
// schedule (PHASE 3) runs the n1 = ustart[E] gate/up units, then the down
// units, whose table is ustart scaled by tiles2 / tiles1.
template <int PHASE, int TN>
__device__ __forceinline__ Unit unit_of(const MxParams& P, const int32_t* ustart, int tiles1, int tiles2, int u) {
  int ph = PHASE == 3 ? 1 : PHASE, num = 1, den = 1;
  if (PHASE == 3 && u >= ustart[P.E]) {
    ph = 2;
    u -= ustart[P.E];
    num = tiles2;
    den = tiles1;
  }
  int lo = 0, hi = P.E;   // start(lo) <= u < start(hi)
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (ustart[mid] / den * num <= u) lo = mid;
    else hi = mid;
  }
  Unit U;
  U.e = lo;
  U.ph = ph;
  const int32_t* eoff = ustart + P.E + 1;   // the unit table's copy of offsets
  const int q_begin = eoff[lo], ne = eoff[lo + 1] - q_begin;
  const int chunks = (ne + TN - 1) / TN;
  const int local = u - ustart[lo] / den * num;
  U.m = local / chunks;
  const int c = local % chunks;
  U.q0 = q_begin + c * TN;
  U.nvalid = min(TN, ne - c * TN);
  return U;
}

// First byte of the blob tile (expert U.e, row tile U.m, k tile 0) of the unit's phase.
__device__ __forceinline__ const uint8_t* tile_base(const MxParams& P, const Unit& U, const int32_t* eslot) {
  const int K = (U.ph == 1) ? P.d : P.I;
  const uint8_t* blob = P.pool + static_cast<size_t>(eslot[U.e]) * P.blob_bytes;
  return blob + (U.ph == 1 ? P.L.wg : P.L.wd) + static_cast<size_t>(U.m) * (K / KSTAGE) * kMxTileBytes;
}

__device__ __forceinline__ void prefetch_l2(const void* p, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

// ------------------------------------------------------------------ E4M3 / E8M0 terms
// E8M0 byte of the smallest power of two 2^e with amax <= 448 * 2^e (448 =
// 1.75 * 2^8 is the largest E4M3 value), so that amax / 2^e rounds to a
// finite E4M3; byte 0 (2^-127) for zero, subnormal or small amax.
__device__ __forceinline__ uint32_t e8m0_for(float amax) {
  const uint32_t b = __float_as_uint(amax);
  const int be = static_cast<int>((b >> 23) & 255u);
  if (be == 0) return 0u;
  const int byte = be - 8 + ((b & 0x7fffffu) > 0x600000u ? 1 : 0);
  return static_cast<uint32_t>(byte < 0 ? 0 : byte);
}

// 2^-(byte - 127) (exact, normal fp32 for byte <= 253)
__device__ __forceinline__ float inv_pow2(uint32_t byte) { return __uint_as_float((254u - byte) << 23); }

// v * 2^(byte - 127), exact for the E4M3 values v multiplies here
__device__ __forceinline__ float times_pow2(float v, uint32_t byte) {
  if (byte >= 1u) return v * __uint_as_float(byte << 23);
  return (v * 5.421010862427522e-20f) * 1.0842021724855044e-19f;   // 2^-64 * 2^-63
}

// fp32 -> E4M3 byte, round to nearest even, saturating to +-448
__device__ __forceinline__ uint32_t e4m3_rn(float v) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(v));
  return r & 0xffu;
}

__device__ __forceinline__ float e4m3_to_f32(uint32_t byte) {
  uint32_t h;
  asm("{ .reg .b16 s; cvt.u16.u32 s, %1; cvt.rn.f16x2.e4m3x2 %0, s; }" : "=r"(h) : "r"(byte));
  return __half2float(__ushort_as_half(static_cast<unsigned short>(h & 0xffffu)));
}

// ------------------------------------------------------------------ split_x
// One thread per 32-element block of a token row: NX E4M3 terms of the
// bf16 values, each term with the E8M0 scale of the block's remaining maximum.
// TN: the GEMV's token rows per term (the scale rows' plane and byte group).
template <int TN>
__global__ void __launch_bounds__(256) mx_split_x_kernel(const uint16_t* __restrict__ x, int T, int x_rows, int d,
                                                         uint8_t* __restrict__ xq, uint8_t* __restrict__ xs,
                                                         int32_t* __restrict__ zero, int n_zero) {
  pdl_wait();     // the terms and counters may still be read by the previous step's GEMVs
  pdl_trigger();
  const int nb = d / 32;
  // the one-launch GEMV's per-expert counters start at zero (this kernel runs right before it)
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n_zero; i += gridDim.x * blockDim.x) zero[i] = 0;
  const long long n = static_cast<long long>(T) * nb;
  for (long long g = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; g < n;
       g += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int t = static_cast<int>(g / nb), b = static_cast<int>(g % nb);
    const uint4* src = reinterpret_cast<const uint4*>(x + static_cast<size_t>(t) * d + 32 * b);
    float r[32];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint4 u = __ldg(src + i);
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        r[8 * i + 2 * j] = __uint_as_float(w[j] << 16);
        r[8 * i + 2 * j + 1] = __uint_as_float(w[j] & 0xffff0000u);
      }
    }
#pragma unroll
    for (int term = 0; term < NX; ++term) {
      float amax = 0.f;
#pragma unroll
      for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(r[i]));
      const uint32_t sb = e8m0_for(amax);
      const float inv = inv_pow2(sb);
      uint32_t packed[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) packed[i] = 0;
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const uint32_t q = e4m3_rn(r[i] * inv);
        packed[i >> 2] |= q << (8 * (i & 3));
        r[i] -= times_pow2(e4m3_to_f32(q), sb);
      }
      uint4* dst = reinterpret_cast<uint4*>(xq + (static_cast<size_t>(term) * x_rows + t) * d + 32 * b);
      dst[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
      dst[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
      // scale of block b in byte b % 4 of the term's byte group of the 16-byte
      // row of atom b / 4 (the tcgen05 scale-factor atom's row pitch, so one
      // copy of a row lands in place)
      xs[((static_cast<size_t>(sf_plane<TN>(term)) * (nb / 4) + b / 4) * x_rows + t) * 16 + sf_byte<TN>(term) + (b & 3)] =
          static_cast<uint8_t>(sb);
    }
  }
}

// ------------------------------------------------------------------ the GEMVs
__device__ __forceinline__ int token_of(const MxParams& P, const Unit& U, int lane, int n_pairs) {
  int tok = 0;
  if (U.ph == 1 && lane < U.nvalid) {
    const int p = __ldg(P.perm + U.q0 + lane);
    if (p < 0 || p >= n_pairs) report(P.status, MOE_ERR_DEVICE);
    else tok = p / P.k;
  }
  return tok;
}

// Token-row terms of K stage ks of unit U into the B stage at sB, and their
// E8M0 scale atoms after them, all asynchronous copies completing on bar
// (whose expected bytes lane 0 posts first).  Per 128-element half h the
// terms' rows are stacked (term j at rows j*TN..) in one 128-byte-swizzled
// tile, and one scale atom covers them all.  gemv<1>: one-row TMA loads of
// the x planes and 16-byte bulk copies of their scale rows (lane q: pair
// q0 + q; a tensor copy needs a 128-byte-aligned destination, an atom row is
// 16 bytes); gemv<2>: one TMA box of a-plane rows per term and one box of
// scale rows per scale plane (landing on a 256-byte boundary).  Rows past the
// unit's pairs hold stale bytes; their MMA columns are never read.  Called by
// all lanes of one warp.
template <class C, int TN>
__device__ __forceinline__ void load_b(const MxParams& P, const MxMaps& M, const Unit& U, int ks, int tok,
                                       uint8_t* sB, uint64_t* bar, uint64_t pol, int lane) {
  uint8_t* sf = sB + C::B_CODES;
  const int nt = U.ph == 1 ? NX : NA;       // terms of this unit's B operand
  // gemv<1> with TN <= 16 (T <= TN) loads every token's rows, else the unit's pairs' rows
  const uint32_t rows = (U.ph == 1 && TN == 32) ? static_cast<uint32_t>(U.nvalid) : static_cast<uint32_t>(TN);
  const int planes = nt < C::G ? nt : C::G;   // scale planes of this unit's terms
  if (lane == 0) mbar_expect_tx(bar, rows * 2 * static_cast<uint32_t>(nt * 128 + planes * 16));
  __syncwarp();
  if (U.ph == 2) {
    if (lane == 0) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        tma_load_3d(sB + h * NA * C::B_ATOM, &M.a, bar, ks * KSTAGE + 128 * h, U.q0, 0, pol);
        tma_load_3d(sf + h * 512, &M.as, bar, 4 * U.q0, 2 * ks + h, 0, pol);
      }
    }
  } else if (TN <= 16) {
    if (lane == 0) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        tma_load_3d(sB + h * NX * C::B_ATOM, &M.xall, bar, ks * KSTAGE + 128 * h, 0, 0, pol);
        tma_load_3d(sf + h * 512, &M.xs, bar, 0, 2 * ks + h, 0, pol);
      }
    }
  } else if (lane < U.nvalid) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
#pragma unroll
      for (int j = 0; j < NX; ++j)
        tma_load_3d(sB + (h * NX + j) * C::B_ATOM + lane * 128, &M.x, bar, ks * KSTAGE + 128 * h, tok, j, pol);
#pragma unroll
      for (int g = 0; g < (NX < C::G ? NX : C::G); ++g)
        bulk_load(sf + h * 512 + (g * TN + lane) * 16,
                  P.xs + ((static_cast<size_t>(g) * (P.d / 128) + 2 * ks + h) * P.x_rows + tok) * 16, 16, bar, pol);
    }
  }
}

// One-launch schedule: lane 0 waits (bounded, like every wait) until all
// `target` gate/up units of expert e have published their a rows, then orders
// the TMA loads that follow after what it observed.  `seen` is the counter
// value lane 0 loaded ahead of time (relaxed, while the previous unit
// streamed): when it already reaches the target, a fence gives the acquire
// without another trip to memory.  One verdict for the warp.
__device__ __forceinline__ bool wait_expert_ready(const MxParams& P, int e, int target, int seen,
                                                  volatile int* abort_flag, int lane) {
  bool ok = true;
  if (lane == 0) {
    if (seen >= target) {
      asm volatile("fence.acq_rel.gpu;" ::: "memory");
    } else {
      const uint64_t t0 = now_ns();
      for (;;) {
        int v;
        asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(P.done1 + e) : "memory");
        if (v >= target) break;
        if (*abort_flag || now_ns() - t0 > P.wait_ns) {
          ok = false;
          break;
        }
        __nanosleep(256);
      }
    }
    asm volatile("fence.proxy.async.global;" ::: "memory");
  }
  return __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
}

// The counter of expert e, loaded without ordering (a prefetch for the wait above).
__device__ __forceinline__ int peek_expert_counter(const MxParams& P, int e) {
  int v;
  asm volatile("ld.relaxed.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(P.done1 + e) : "memory");
  return v;
}

__device__ __forceinline__ void drain_ring(uint64_t* full, int n, int issued, int stage, uint32_t phase) {
  const int outstanding = issued < n ? issued : n;
  for (int i = 0; i < outstanding; ++i) {
    if (--stage < 0) {
      stage = n - 1;
      phase ^= 1u;
    }
    mbar_drain(&full[stage], phase);
  }
}

__device__ __forceinline__ void tma_load_5d(void* dst, const CUtensorMap* map, uint64_t* bar, int c0, int c1,
                                            int c2, int c3, int c4, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.5d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint [%0], "
      "[%1, {%3, %4, %5, %6, %7}], [%2], %8;" ::"r"(smem_u32(dst)),
      "l"(map), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(c4), "l"(policy)
      : "memory");
}

__device__ __forceinline__ void tc_cp_sf(uint32_t tmem, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(tmem), "l"(sdesc) : "memory");
}

// Instruction descriptor, kind::mxf8f6f4: A = E2M1 (weights), B = E4M3
// (activation terms), both K-major, E8M0 scales, M = 128, N = n; sf = the
// byte of each 32-bit scale cell (the 32-element block within the atom's 4).
__device__ __forceinline__ uint32_t idesc_mx(int n, uint32_t sf) {
  return (sf << 4) | (5u << 7) | (0u << 10) | (static_cast<uint32_t>(n >> 3) << 17) | (1u << 23) |
         (static_cast<uint32_t>(TM >> 4) << 24) | (sf << 29);
}

__device__ __forceinline__ void tc_mma_mx(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t sfa,
                                          uint32_t sfb, uint32_t acc) {
  asm volatile(
      "{ .reg .pred p; setp.ne.b32 p, %6, 0; "
      "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale.scale_vec::1X [%0], %1, %2, %3, [%4], [%5], p; }" ::"r"(
          d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(sfa), "r"(sfb), "r"(acc)
      : "memory");
}

__device__ __forceinline__ float silu(float h) { return h / (1.0f + expf(-h)); }

// v[t] for a t < TN known only at run time, without indexing registers
// dynamically (which would move v to local memory).
template <int TN>
__device__ __forceinline__ float pick(const float (&v)[32], int t) {
  float g = v[0];
#pragma unroll
  for (int j = 1; j < TN; ++j) g = (t == j) ? v[j] : g;
  return g;
}

// Token row c's result for this warp's 32 TMEM lanes: the sum over the nt
// stacked terms of accumulator columns j*TN + c (fp32, terms in order).
template <int TN>
__device__ __forceinline__ void load_terms(uint32_t taddr, int nt, float (&v)[32]) {
  if (TN == 8) {
    float t[8];
#pragma unroll
    for (int c = 0; c < 32; ++c) v[c] = 0.f;
#pragma unroll
    for (int j = 0; j < NA; ++j) {
      if (j >= nt) break;
      tmem_ld8(taddr + 8 * j, t);
#pragma unroll
      for (int c = 0; c < 8; ++c) v[c] += t[c];
    }
  } else if (TN == 16) {
    float t[16];
#pragma unroll
    for (int c = 0; c < 32; ++c) v[c] = 0.f;
#pragma unroll
    for (int j = 0; j < NA; ++j) {
      if (j >= nt) break;
      tmem_ld16(taddr + 16 * j, t);
#pragma unroll
      for (int c = 0; c < 16; ++c) v[c] += t[c];
    }
  } else {
    float t[32];
    tmem_ld32(taddr, v);
#pragma unroll
    for (int j = 1; j < NA; ++j) {
      if (j >= nt) break;
      tmem_ld32(taddr + 32 * j, t);
#pragma unroll
      for (int c = 0; c < 32; ++c) v[c] += t[c];
    }
  }
}

template <int PHASE, int TN>
__global__ void __launch_bounds__(THREADS, 1)
    gemv_mx_kernel(const __grid_constant__ MxMaps M, const MxParams P) {
  using C = Cfg<PHASE, TN>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* ring_b = smem + C::A_RING;
  float* up_buf = reinterpret_cast<float*>(ring_b + C::B_RING);
  uint64_t* bars = reinterpret_cast<uint64_t*>(ring_b + C::B_RING + C::UP_BYTES);
  uint64_t* full = bars;                        // [SA] weight tile landed
  uint64_t* empty = bars + C::SA;               // [SA] weight tile free
  uint64_t* tfull = bars + 2 * C::SA;           // [2]
  uint64_t* tempty = tfull + 2;                 // [2]
  uint64_t* drain = tfull + 4;                  // [1]
  uint64_t* bfull = tfull + 5;                  // [SB] token-row terms landed
  uint64_t* bempty = bfull + C::SB;             // [SB] token-row terms free
  uint64_t* stall = bempty + C::SB;             // [1] never arrived on (testing aid)
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + C::N_BARS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  volatile int* epi_fail = reinterpret_cast<volatile int*>(tmem_holder + 2);
  int32_t* ustart = reinterpret_cast<int32_t*>(ring_b + C::B_RING + C::UP_BYTES + kBarBytes);
  int32_t* eoff = ustart + (P.E + 1);          // offsets[0..E] and slot[0..E-1], read once
  int32_t* eslot = eoff + (P.E + 1);
  __shared__ int ws[36];
  __shared__ int s_ctok[2][32];        // down units: each column's token and gate (two units in flight)
  __shared__ float s_cgate[2][32];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int MT1 = P.I / 64, MT2 = P.d / TM;     // tiles per chunk: gate/up, down
  const int MT = PHASE == 2 ? MT2 : MT1;          // ... of the unit table built below
  auto ks_of = [&](const Unit& U) { return (U.ph == 1 ? P.d : P.I) / KSTAGE; };
  const int n_pairs = P.T * P.k;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::SA; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 128);
    }
    mbar_init(drain, 1);
    mbar_init(stall, 1);
    for (int s = 0; s < C::SB; ++s) {
      mbar_init(&bfull[s], 1);
      mbar_init(&bempty[s], 1);
    }
    *abort_flag = 0;
    *epi_fail = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_holder)),
                 "r"(TMEM_COLS));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }

  // the routing tables come from the kernels launched before (programmatic
  // dependents start early: barriers and TMEM above, before the wait); the
  // down GEMV instead waits in its token-row producer, so that its weights
  // stream during the gate/up tail
  if (PHASE != 2) pdl_wait();
  // ---- units per expert (evaluated experts only) and their exclusive prefix
  const int per = (P.E + THREADS - 1) / THREADS;
  const int e0 = threadIdx.x * per;
  int cnt = 0;
  for (int j = 0; j < per; ++j) {
    const int e = e0 + j;
    if (e >= P.E) break;
    const int a = __ldg(P.offsets + e), b = __ldg(P.offsets + e + 1);
    if (b <= a) continue;
    if (a < 0 || b > n_pairs) {
      report(P.status, MOE_ERR_DEVICE);
      continue;
    }
    const int s = __ldg(P.slot + e);
    if (s >= P.n_slots) {
      report(P.status, MOE_ERR_DEVICE);
      continue;
    }
    if (s < 0) continue;
    cnt += MT * ((b - a + TN - 1) / TN);
  }
  int total = 0;
  int run = block_scan(cnt, ws, &total);
  for (int j = 0; j < per; ++j) {
    const int e = e0 + j;
    if (e >= P.E) break;
    ustart[e] = run;
    const int a = __ldg(P.offsets + e), b = __ldg(P.offsets + e + 1);
    const int s = __ldg(P.slot + e);
    eoff[e] = a;                 // copies for the unit lookups (no global load on a producer's path)
    eslot[e] = s;
    if (b > a && a >= 0 && b <= n_pairs && s >= 0 && s < P.n_slots) run += MT * ((b - a + TN - 1) / TN);
  }
  if (threadIdx.x == 0) {
    ustart[P.E] = total;
    eoff[P.E] = __ldg(P.offsets + P.E);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const int n_units = PHASE == 3 ? total + total / MT1 * MT2 : total;
  // two-launch schedule: the down GEMV (launched as a programmatic dependent)
  // may take each SM as soon as this CTA leaves it; it streams its weights
  // at once and waits for this grid only before reading the a terms
  if (PHASE == 1) pdl_trigger();

  if (warp == 0) {
    // ------------------------------------------------------------ weight producer
    const uint64_t pol_stream = policy_evict_first();
    int stage = 0;
    uint32_t phase = 0;
    int issued = 0;
    bool ok = true;
    int pf_u = blockIdx.x, pf_ks = 0, pf_ahead = 0, pf_KS = 0;
    const uint8_t* pf_base = nullptr;
    if (pf_u < n_units) {
      const Unit V = unit_of<PHASE, TN>(P, ustart, MT, MT2, pf_u);
      pf_base = tile_base(P, V, eslot);
      pf_KS = ks_of(V);
    }
    for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
      const Unit U = unit_of<PHASE, TN>(P, ustart, MT, MT2, u);
      const int sl = eslot[U.e];
      const uint8_t* abase = tile_base(P, U, eslot);
      const CUtensorMap* tm_w = U.ph == 1 ? &M.w1 : &M.w2;
      const int KS = ks_of(U);
      for (int ks = 0; ks < KS; ++ks) {
        if (!__all_sync(0xffffffffu, mbar_wait<true>(&empty[stage], phase ^ 1u, abort_flag, P.wait_ns))) {
          ok = false;
          break;
        }
        uint8_t* sA = smem + stage * A_SMEM;
        if (lane == 0) {
          mbar_expect_tx(&full[stage], A_TX);
          // codes: two boxes of 128 rows x 128 codes, expanded by the TMA into
          // 16-byte slots; coordinates (k in tile, row, k tile, row tile, slot)
          tma_load_5d(sA, tm_w, &full[stage], 0, 0, ks, U.m, sl, pol_stream);
          tma_load_5d(sA + A_BOX, tm_w, &full[stage], 128, 0, ks, U.m, sl, pol_stream);
          bulk_load(sA + 2 * A_BOX, abase + static_cast<size_t>(ks) * kMxTileBytes + 16384, 1024, &full[stage],
                    pol_stream);
          while (pf_u < n_units && pf_ahead < P.pf_items) {
            prefetch_l2(pf_base + static_cast<size_t>(pf_ks) * kMxTileBytes, kMxTileBytes);
            ++pf_ahead;
            if (++pf_ks == pf_KS) {
              pf_ks = 0;
              pf_u += gridDim.x;
              if (pf_u < n_units) {
                const Unit V = unit_of<PHASE, TN>(P, ustart, MT, MT2, pf_u);
                pf_base = tile_base(P, V, eslot);
                pf_KS = ks_of(V);
              }
            }
          }
          --pf_ahead;
        }
        __syncwarp();
        ++issued;
        if (++stage == C::SA) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
    __syncwarp();
    if (!ok) {
      report(P.status, MOE_ERR_TIMEOUT);
      *abort_flag = 1;
    }
    drain_ring(full, C::SA, issued, stage, phase);
  } else if (warp == BPROD_WARP) {
    // ------------------------------------------------------------ token-row producer
    const uint64_t pol_keep = policy_evict_last();
    int stage = 0;
    uint32_t phase = 0;
    int issued = 0;
    bool ok = true;
    int seen = -1;                       // lane 0: this unit's expert counter, loaded ahead
    // the down GEMV of the two-launch schedule: the gate/up grid is complete
    // and its a terms are visible before the first of them is read
    if (PHASE == 2) {
      pdl_wait();
      pdl_trigger();             // the combine after this GEMV may be scheduled
    }
    for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
      const Unit U = unit_of<PHASE, TN>(P, ustart, MT, MT2, u);
      const int tok = TN == 32 ? token_of(P, U, lane, n_pairs) : 0;
      const int KS = ks_of(U);
      if (PHASE == 3 && U.ph == 2) {
        // the a terms of this expert's pairs come from every gate/up unit of the expert
        if (!wait_expert_ready(P, U.e, ustart[U.e + 1] - ustart[U.e], seen, abort_flag, lane)) {
          ok = false;
          break;
        }
      }
      if (PHASE == 3 && lane == 0 && u + static_cast<int>(gridDim.x) < n_units) {
        const Unit V = unit_of<PHASE, TN>(P, ustart, MT, MT2, u + gridDim.x);
        seen = V.ph == 2 ? peek_expert_counter(P, V.e) : -1;   // consumed at the next unit
      }
      for (int ks = 0; ks < KS; ++ks) {
        if (!__all_sync(0xffffffffu, mbar_wait<true>(&bempty[stage], phase ^ 1u, abort_flag, P.wait_ns))) {
          ok = false;
          break;
        }
        load_b<C, TN>(P, M, U, ks, tok, ring_b + stage * C::B_STAGE, &bfull[stage], pol_keep, lane);
        __syncwarp();
        ++issued;
        if (++stage == C::SB) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
    if (!ok) {
      report(P.status, MOE_ERR_TIMEOUT);
      *abort_flag = 1;
    }
    drain_ring(bfull, C::SB, issued, stage, phase);
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    int sb = 0, sa = 0;
    uint32_t pb = 0, pa = 0;
    int it = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x, ++it) {
      const Unit U = unit_of<PHASE, TN>(P, ustart, MT, MT2, u);
      const int KS = ks_of(U);
      const int nt = U.ph == 1 ? NX : NA;       // terms of the unit's B operand, stacked along N
      const uint32_t n_mma = static_cast<uint32_t>(nt * TN);
      const int acc = it & 1;
      if (!__all_sync(0xffffffffu, mbar_wait<true>(&tempty[acc], ((it >> 1) & 1) ^ 1u, abort_flag, P.wait_ns))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t d_tmem = tmem + acc * ACC_COLS;
      for (int ks = 0; ks < KS; ++ks) {
        // one verdict for the warp: its lanes then take the same path to elect.sync
        if (!__all_sync(0xffffffffu, mbar_wait<true>(&bfull[sb], pb, abort_flag, P.wait_ns) &&
                                         mbar_wait<true>(&full[sa], pa, abort_flag, P.wait_ns))) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (elect_one()) {
          const uint8_t* sA = smem + sa * A_SMEM;
          const uint8_t* sB = ring_b + sb * C::B_STAGE;
          // scale atoms -> TMEM: weights and token-row terms, one atom per
          // 128-element half (4 blocks of 32)
          tc_cp_sf(tmem + SFA_COL, desc_sf(smem_u32(sA + 2 * A_BOX)));
          tc_cp_sf(tmem + SFA_COL + 4, desc_sf(smem_u32(sA + 2 * A_BOX + 512)));
          tc_cp_sf(tmem + SFB_COL, desc_sf(smem_u32(sB + C::B_CODES)));
          tc_cp_sf(tmem + SFB_COL + 4, desc_sf(smem_u32(sB + C::B_CODES + 512)));
#pragma unroll
          for (int kk = 0; kk < KSTAGE / 32; ++kk) {   // K = 32 per MMA: +32 bytes of the expanded rows
            const int h = kk >> 2, sub = kk & 3;
            const uint64_t da = desc_sw128(smem_u32(sA + h * A_BOX)) + 2 * sub;
            const uint64_t db = desc_sw128(smem_u32(sB + h * nt * C::B_ATOM)) + 2 * sub;
            const uint32_t idesc = idesc_mx(static_cast<int>(n_mma), static_cast<uint32_t>(sub));
            tc_mma_mx(d_tmem, da, db, idesc, tmem + SFA_COL + 4 * h, tmem + SFB_COL + 4 * h,
                      (ks > 0 || kk > 0) ? 1u : 0u);
          }
          tc_commit(&empty[sa]);
          tc_commit(&bempty[sb]);
        }
        __syncwarp();
        if (++sb == C::SB) {
          sb = 0;
          pb ^= 1u;
        }
        if (++sa == C::SA) {
          sa = 0;
          pa ^= 1u;
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
    if (elect_one()) tc_commit(drain);
    __syncwarp();
    mbar_drain(drain, 0);
  } else {
    // ------------------------------------------------------------ epilogue (warps 2..5)
    const int quad = warp & 3;                       // TMEM lanes 32*quad .. 32*quad+31
    int it = 0;
    // testing aid (moe_set_test_stall): CTA 0's epilogue first waits on a
    // barrier that nothing arrives on, so the bounded wait runs out and the
    // abort path (record, stop issuing, drain, free TMEM) runs for real
    const bool stalled = P.stall && blockIdx.x == 0 && !mbar_wait<true>(stall, 0, abort_flag, P.wait_ns);
    if (stalled) {
      report(P.status, MOE_ERR_TIMEOUT);
      *abort_flag = 1;
    }
    for (int u = blockIdx.x; u < n_units && !stalled; u += gridDim.x, ++it) {
      const Unit U = unit_of<PHASE, TN>(P, ustart, MT, MT2, u);
      const int acc = it & 1;
      if (((U.ph == 2 && P.y_perm == nullptr) || (U.ph == 1 && TN <= 16)) && quad == 0 && lane < U.nvalid) {
        // the unit's column info (its pairs' tokens; for the down GEMV's
        // combine also their gates), fetched while its accumulator is
        // computed (the barrier after the wait publishes it; the other buffer
        // may still be read by warps finishing the previous unit)
        const int p = __ldg(P.perm + U.q0 + lane);
        const bool good = p >= 0 && p < n_pairs;
        if (!good) report(P.status, MOE_ERR_DEVICE);
        s_ctok[acc][lane] = good ? p / P.k : (U.ph == 1 ? 0 : -1);
        s_cgate[acc][lane] = good && U.ph == 2 ? __ldg(P.gate + p) : 0.f;
      }
      // the four warps leave together: a warp alone at a named barrier would wait for good
      if (!mbar_wait<true>(&tfull[acc], (it >> 1) & 1, abort_flag, P.wait_ns)) *epi_fail = 1;
      named_sync(1, 128);
      if (*epi_fail) {
        report(P.status, MOE_ERR_TIMEOUT);
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      float v[32];
      load_terms<TN>(tmem + (static_cast<uint32_t>(32 * quad) << 16) + acc * ACC_COLS, U.ph == 1 ? NX : NA, v);
      tc_fence_before();
      mbar_arrive(&tempty[acc]);
      if (U.ph == 1) {
        // rows 0..63 of the tile are gate rows, 64..127 the matching up rows
        if (quad >= 2) {
          const int i = 32 * (quad - 2) + lane;
#pragma unroll
          for (int c = 0; c < 32; ++c) up_buf[i * 33 + c] = v[c];
        }
        named_sync(1, 128);
        if (quad < 2) {
          // this warp's 32 lanes hold one 32-element block of I for every pair
          const int i = 32 * quad + lane;
          const size_t col = static_cast<size_t>(64) * U.m + i;
          const size_t blk = static_cast<size_t>(2) * U.m + quad;
          const int nbi = P.I / 32;
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            if (c < U.nvalid) {
              // B column of pair c: its token (TN <= 16: every token's rows), else c
              const int bc = TN <= 16 ? s_ctok[acc][c] : c;
              float r = silu(TN <= 16 ? pick<TN>(v, bc) : v[c]) * up_buf[i * 33 + bc];
              const size_t q = static_cast<size_t>(U.q0 + c);
#pragma unroll
              for (int j = 0; j < NA; ++j) {
                const uint32_t amax = __reduce_max_sync(0xffffffffu, __float_as_uint(fabsf(r)));
                const uint32_t sb = e8m0_for(__uint_as_float(amax));
                const uint32_t t = e4m3_rn(r * inv_pow2(sb));
                r -= times_pow2(e4m3_to_f32(t), sb);
                const size_t plane = static_cast<size_t>(j) * P.a_rows;
                P.aq[(plane + q) * P.I + col] = static_cast<uint8_t>(t);
                if (lane == 0)
                  P.as[((static_cast<size_t>(sf_plane<TN>(j)) * (nbi / 4) + blk / 4) * P.a_rows + q) * 16 +
                       sf_byte<TN>(j) + (blk & 3)] = static_cast<uint8_t>(sb);
              }
            }
          }
          // one-launch schedule: the a terms are published to other CTAs (read
          // there by TMA): each writer orders its stores before the async
          // proxy, the barrier below orders them before one thread's gpu-scope
          // fence, and that fence before the counter increment (one fence per
          // unit instead of one per thread)
          if (PHASE == 3) asm volatile("fence.proxy.async.global;" ::: "memory");
        }
        named_sync(1, 128);
        if (PHASE == 3 && warp == 2 && lane == 0) {
          __threadfence();
          atomicAdd(P.done1 + U.e, 1);
        }
      } else {
        const int row = TM * U.m + 32 * quad + lane;
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          if (c < U.nvalid) {
            const int q = U.q0 + c;
            if (P.y_perm != nullptr) {
              P.y_perm[static_cast<size_t>(q) * P.d + row] = v[c];
            } else {
              const int t = s_ctok[acc][c];
              if (t >= 0) atomicAdd(P.out + static_cast<size_t>(t) * P.d + row, s_cgate[acc][c] * v[c]);
            }
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS));
  }
}

template <int PHASE, int TN>
moe_status launch_phase(const MxParams& P, const MxMaps& M, const DeviceInfo& dev, cudaStream_t s) {
  const size_t smem = smem_bytes<PHASE, TN>(P.E);
  if (smem > dev.smem_optin) return fail(MOE_ERR_UNSUPPORTED, "MXFP4 decode GEMV needs %zu bytes of shared memory", smem);
  static size_t attr[64] = {};
  if (attr[dev.id] < smem) {
    MOE_CUDA_TRY(cudaFuncSetAttribute(gemv_mx_kernel<PHASE, TN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      static_cast<int>(smem)));
    attr[dev.id] = smem;
  }
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(dev.sm_count);
  cfg.blockDim = dim3(THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  // the one-launch schedule's CTAs wait on each other's gate/up units: all of
  // them must be resident at once, which a cooperative launch guarantees
  // the two-launch schedule's GEMVs are programmatic dependents of the kernel
  // before each (gate/up: the routing tables; down: the a terms), waiting for
  // it in-kernel; the cooperative one-launch schedule is a plain launch
  cudaLaunchAttribute at[2];
  at[0].id = cudaLaunchAttributeCooperative;
  at[0].val.cooperative = PHASE == 3 ? 1 : 0;
  at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[1].val.programmaticStreamSerializationAllowed = PHASE != 3 ? 1 : 0;
  cfg.attrs = at;
  cfg.numAttrs = 2;
  MOE_CUDA_TRY(cudaLaunchKernelEx(&cfg, gemv_mx_kernel<PHASE, TN>, M, P));
  MOE_LAUNCH_CHECK("gemv_mx_kernel");
  return MOE_OK;
}

// 5-D map over the stage tiles of one matrix of every slot: (k within the
// tile: 256 codes, row within the tile: 128, k tile, row tile, slot); the box
// is 128 codes x 128 rows, each 16 codes expanded into a 16-byte slot.
CUresult encode_weight_map(CUtensorMap* map, const uint8_t* region0, int K, int R, int n_slots,
                           size_t blob_bytes) {
  auto fn = encode_tiled_fn();
  if (!fn) return CUDA_ERROR_NOT_FOUND;
  const int KT = K / KSTAGE, RT = R / TM;
  cuuint64_t gdim[5] = {static_cast<cuuint64_t>(KSTAGE), static_cast<cuuint64_t>(TM), static_cast<cuuint64_t>(KT),
                        static_cast<cuuint64_t>(RT), static_cast<cuuint64_t>(n_slots)};
  cuuint64_t gstr[4] = {128, static_cast<cuuint64_t>(kMxTileBytes),
                        static_cast<cuuint64_t>(KT) * kMxTileBytes, static_cast<cuuint64_t>(blob_bytes)};
  cuuint32_t box[5] = {128, static_cast<cuuint32_t>(TM), 1, 1, 1};
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, 5, const_cast<uint8_t*>(region0), gdim, gstr, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
}

struct MxWorkspace {
  size_t xq, xs, aq, as, done1, bytes;
};

MxWorkspace mx_workspace(moe_shape s, int T, int k) {
  MxWorkspace W{};
  const size_t n = static_cast<size_t>(T) * k;
  size_t o = 0;
  const size_t tx = T > 32 ? T : 32;       // rows of an x-term plane (MxParams::x_rows)
  W.xq = o; o = round_up(o + static_cast<size_t>(NX) * tx * s.d, 256);
  W.xs = o; o = round_up(o + static_cast<size_t>(NX) * tx * (s.d / 128) * 16, 256);
  const size_t na = n > 32 ? n : 32;       // rows of an a-term plane (MxParams::a_rows)
  W.aq = o; o = round_up(o + static_cast<size_t>(NA) * na * s.I, 256);
  W.as = o; o = round_up(o + static_cast<size_t>(NA) * na * (s.I / 128) * 16, 256);
  W.done1 = o; o = round_up(o + static_cast<size_t>(s.E) * sizeof(int32_t), 256);
  W.bytes = o;
  return W;
}

template <int TN>
moe_status launch_both(const MxParams& P, const MxMaps& M, const DeviceInfo& dev, cudaStream_t stream) {
  if (decode_one_launch(MOE_W_MXFP4, P.T)) return launch_phase<3, TN>(P, M, dev, stream);   // counters zeroed by mx_split_x_kernel
  moe_status st = launch_phase<1, TN>(P, M, dev, stream);
  if (st != MOE_OK) return st;
  return launch_phase<2, TN>(P, M, dev, stream);
}

}  // namespace

size_t decode_mx_workspace_bytes(moe_shape s, int T, int k) { return mx_workspace(s, T, k).bytes; }

// Split x, then both GEMV launches, for MXFP4 blobs in the stage-tiled layout.
moe_status launch_decode_mx(moe_shape s, const void* x, int T, int k, const int32_t* offsets, const int32_t* perm,
                            const int32_t* slot, const void* pool, int n_slots, const float* gate, float* y_perm,
                            float* out, void* ws, int32_t* status, const DeviceInfo& dev, cudaStream_t stream) {
  const MxWorkspace W = mx_workspace(s, T, k);
  uint8_t* w8 = static_cast<uint8_t*>(ws);
  MxParams P{};
  P.wait_ns = wait_limit_ns();
  P.pf_items = PF_ITEMS;
  P.stall = test_stall();
  P.E = s.E;
  P.d = s.d;
  P.I = s.I;
  P.T = T;
  P.k = k;
  P.n_slots = n_slots;
  P.offsets = offsets;
  P.perm = perm;
  P.slot = slot;
  P.gate = gate;
  P.pool = static_cast<const uint8_t*>(pool);
  P.L = blob_layout(s.fmt, s.d, s.I);
  P.blob_bytes = P.L.bytes;
  P.xs = w8 + W.xs;
  P.aq = w8 + W.aq;
  P.as = w8 + W.as;
  P.done1 = reinterpret_cast<int32_t*>(w8 + W.done1);
  P.y_perm = y_perm;
  P.out = out;
  P.status = status;
  const uint64_t n = static_cast<uint64_t>(T) * k;
  const uint64_t na = n > 32 ? n : 32;
  P.a_rows = static_cast<int>(na);
  const uint64_t tx = T > 32 ? T : 32;
  P.x_rows = static_cast<int>(tx);
  const int tn = T <= 8 ? 8 : (T <= 16 ? 16 : 32);   // token rows per term (the GEMV's TN)
  MxMaps M;
  CUresult r = encode_weight_map(&M.w1, P.pool + P.L.wg, s.d, 2 * s.I, n_slots, P.blob_bytes);
  if (r == CUDA_SUCCESS) r = encode_weight_map(&M.w2, P.pool + P.L.wd, s.I, s.d, n_slots, P.blob_bytes);
  if (r != CUDA_SUCCESS) return fail(MOE_ERR_CUDA, "tensor map of the MXFP4 weights failed (%d)", static_cast<int>(r));
  {
    // the x terms: (code, token, term); one-row boxes, and boxes of TN rows of
    // both terms with their scale rows (byte in the atom row, atom, token, plane)
    const uint64_t dims[3] = {static_cast<uint64_t>(s.d), tx, static_cast<uint64_t>(NX)};
    const uint64_t str[2] = {static_cast<uint64_t>(s.d), tx * s.d};
    const uint32_t box[3] = {128u, 1u, 1u};
    r = encode_tiled_sw128(&M.x, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, w8 + W.xq, dims, str, box);
    const uint32_t boxall[3] = {128u, static_cast<uint32_t>(tn), static_cast<uint32_t>(NX)};
    if (r == CUDA_SUCCESS) r = encode_tiled_sw128(&M.xall, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, w8 + W.xq, dims, str, boxall);
    const uint32_t planes = static_cast<uint32_t>(std::min(32 / tn, NX));
    // scale rows [plane][atom][token][16 bytes] as 32-bit words: a box of TN
    // consecutive rows of one atom per plane is one contiguous run
    const uint64_t sdims[3] = {tx * 4, static_cast<uint64_t>(s.d / 128), planes};
    const uint64_t sstr[2] = {tx * 16, static_cast<uint64_t>(s.d / 128) * tx * 16};
    const uint32_t sbox[3] = {static_cast<uint32_t>(4 * tn), 1u, planes};
    if (r == CUDA_SUCCESS) r = encode_tiled_plain(&M.xs, CU_TENSOR_MAP_DATA_TYPE_UINT32, 3, w8 + W.xs, sdims, sstr, sbox);
    if (r != CUDA_SUCCESS) return fail(MOE_ERR_CUDA, "tensor map of the x terms failed (%d)", static_cast<int>(r));
  }
  {
    // the a terms: (code, pair, term), a box of TN pairs of all NA terms; rows
    // past the planes' end read as zeros
    const uint64_t dims[3] = {static_cast<uint64_t>(s.I), na, static_cast<uint64_t>(NA)};
    const uint64_t str[2] = {static_cast<uint64_t>(s.I), na * s.I};
    const uint32_t box[3] = {128u, static_cast<uint32_t>(tn), static_cast<uint32_t>(NA)};
    r = encode_tiled_sw128(&M.a, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, w8 + W.aq, dims, str, box);
    // their scale rows [plane][atom][pair][16 bytes] as 32-bit words, a box of
    // TN consecutive pairs of one atom per plane
    const uint32_t planes = static_cast<uint32_t>(std::min(32 / tn, NA));
    const uint64_t sdims[3] = {na * 4, static_cast<uint64_t>(s.I / 128), planes};
    const uint64_t sstr[2] = {na * 16, static_cast<uint64_t>(s.I / 128) * na * 16};
    const uint32_t sbox[3] = {static_cast<uint32_t>(4 * tn), 1u, planes};
    if (r == CUDA_SUCCESS) r = encode_tiled_plain(&M.as, CU_TENSOR_MAP_DATA_TYPE_UINT32, 3, w8 + W.as, sdims, sstr, sbox);
    if (r != CUDA_SUCCESS) return fail(MOE_ERR_CUDA, "tensor map of the a terms failed (%d)", static_cast<int>(r));
  }
  {
    const long long blocks = static_cast<long long>(T) * (s.d / 32);
    const int grid = static_cast<int>((blocks + 255) / 256 < dev.sm_count * 4 ? (blocks + 255) / 256 : dev.sm_count * 4);
    auto split = T <= 8 ? mx_split_x_kernel<8> : (T <= 16 ? mx_split_x_kernel<16> : mx_split_x_kernel<32>);
    MOE_CUDA_TRY(launch_pdl(split, dim3(grid), dim3(256), 0, stream, static_cast<const uint16_t*>(x), T, P.x_rows,
                            s.d, w8 + W.xq, w8 + W.xs, P.done1, decode_one_launch(MOE_W_MXFP4, T) ? s.E : 0));
    MOE_LAUNCH_CHECK("mx_split_x_kernel");
  }
  if (T <= 8) return launch_both<8>(P, M, dev, stream);
  return T <= 16 ? launch_both<16>(P, M, dev, stream) : launch_both<32>(P, M, dev, stream);
}

}  // namespace moe
