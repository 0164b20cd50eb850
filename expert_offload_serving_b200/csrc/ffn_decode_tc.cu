// Step 3 at decode sizes on the 5th-generation tensor cores for bf16 blobs in
// the tile layout (moe_expert_ffn without MOE_FFN_ACT_NVFP4): the grouped
// SwiGLU expert FFN as two skinny GEMMs.  (MXFP4 blobs run on the block-scaled
// kind in ffn_decode_mx.cu.)
//
// At decode sizes a layer call is bound by reading the routed experts' weights
// from HBM (explainx.ai hardware guide, "Decode: decide whether to move an
// expert or compute where it lives": one token touches few experts).  Bulk
// copies move whole weight stages (128 rows x 128 elements, 32 KB) into shared
// memory, where the stage is the A operand of tcgen05.mma as it lands -- no SM
// instruction is spent per weight element; one thread issues the MMAs, the few
// token rows of a group being the N side and the accumulators living in TMEM.
//
//   gemv<1>: D[128 x N] = W_gu tile (64 gate + 64 up rows of the same
//            intermediate indices) x X^T over K = d, N <= 32 token rows
//            gathered by one-row TMA loads of x.  Epilogue: a = silu(D_gate) *
//            D_up, stored as two bf16 planes hi + lo (a - hi - lo ~ 2^-17 |a|)
//            in the workspace, rows = sorted pairs.
//   gemv<2>: D[128 x N] = W_d tile x (A_hi + A_lo)^T over K = I (two MMAs per
//            k-step).  Epilogue: y_perm rows, or out[t] += gate * y (the fused
//            combine).
//
// Work unit = (expert, 128-row tile, chunk of <= TN pairs; TN = 16 when T <=
// 16, else 32), expert-major, chunks fastest, dealt round-robin to one
// persistent CTA per SM.  Warp 0 produces the weight stages (bulk copy, L2
// prefetch two stages ahead), warp 1 owns TMEM and issues the MMAs, four
// warps run the epilogue on double-buffered TMEM accumulators, and the last
// warp loads the token rows into a ring of their own.  The weight ring takes
// the shared memory the rest leaves (5 stages of 32 KB), so that the GEMVs
// keep enough bytes in flight to run near the HBM rate.  Every wait is
// bounded: on expiry the CTA records MOE_ERR_TIMEOUT, stops issuing, drains
// what it issued and frees its TMEM.
#include <cstdlib>

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "common.cuh"
#include "tc.cuh"

namespace moe {

struct TcDecodeParams {
  uint64_t wait_ns;          // limit of every bounded wait (default 2 s)
  int pf_items;              // L2 prefetch distance in stages
  int stall;                 // testing aid: CTA 0's epilogue waits on a barrier nothing arrives on
  int E, d, I, T, k, n_slots;
  int a_box_rows[3];         // rows of the a-plane TMA boxes: min(8 | 16 | 32, T*k)
  const int32_t* offsets;
  const int32_t* perm;
  const int32_t* slot;
  const float* gate;
  const uint8_t* pool;
  size_t blob_bytes;
  BlobLayout L;
  uint16_t* a_planes;        // [2][T*k][I] bf16: hi, lo
  int32_t* done1;            // fused launch: per expert, gemv<1> units finished (zeroed before the launch)
  float* y_perm;             // [T*k][d] or null (then out)
  float* out;                // [T][d] (fused combine)
  int32_t* status;
};

namespace {

using namespace ::moe::tc;

constexpr int TM = 128;                  // weight rows per tile
constexpr int ACC_COLS = 32;             // TMEM columns per accumulator
constexpr int PF_ITEMS = 2;              // L2 prefetch distance (stages; measured best of 0, 2, 4, 8, 12)
constexpr int kSmemBudget = 226 * 1024;  // opt-in shared memory of one CTA (227 KB) less the static 1 KB
constexpr int kMaxE = 1024;              // experts the unit table is sized for
constexpr int kBarBytes = 512;           // mbarriers, the TMEM address and two flags

// Per (phase, chunk width) geometry.  TN = pairs per chunk (the MMA's N is 16
// or 32): 16 whenever T <= 16, since an expert holds at most one pair per
// token, which halves the token-row buffers and frees room for weight stages.
//
// Weight stages (SA) and token-row stages (SB) are separate rings, each with
// its own producer warp, and the weight ring takes every byte the token rows
// leave: the token rows come from L2 (x, or the a planes just written), so a
// few stages cover them.  The MMA frees both.
template <int FMT, int PHASE, int TN>
struct Cfg {
  static_assert(FMT == MOE_W_BF16, "bf16 blobs only");
  static constexpr int KSTAGE = 128;                             // K elements per stage
  static constexpr int ATOMS = KSTAGE / 64;                      // B atoms per plane
  static constexpr int B_ATOM = TN * 128;                        // one 64-element atom of TN token rows
  static constexpr int A_STAGE = 2 * TM * 128;                   // weight bytes per stage
  static constexpr int B_STAGE = (PHASE == 1 ? 1 : 2) * ATOMS * B_ATOM;   // PHASE 3: both GEMVs
  static constexpr int UP_BYTES = PHASE != 2 ? 64 * 33 * 4 : 0;  // up-row exchange
  static constexpr int FIXED = 1024 + UP_BYTES + kBarBytes + 3 * (kMaxE + 1) * 4;   // + the unit table
  static constexpr int SB = B_STAGE <= 8192 ? (PHASE == 1 && TN == 32 ? 4 : 5) : 3;   // token-row stages
  static constexpr int SA_FIT = (kSmemBudget - FIXED - SB * B_STAGE) / A_STAGE;
  static constexpr int SA = (TN == 16 && PHASE == 1) ? 5 : (SA_FIT > 12 ? 12 : SA_FIT);   // weight stages
  static constexpr int A_RING = SA * A_STAGE;
  static constexpr int B_RING = SB * B_STAGE;
  static constexpr int EPI_WARP0 = 2;
  static constexpr int BPROD_WARP = EPI_WARP0 + 4;               // the token-row producer
  static constexpr int THREADS = (EPI_WARP0 + 5) * 32;
  static constexpr int TMEM_COLS = 64;
  static constexpr int N_BARS = 2 * SA + 2 * SB + 6;
  static_assert(TN == 16 || TN == 32, "chunk width");
  static_assert(A_STAGE % 1024 == 0 && B_STAGE % 1024 == 0, "stages must keep 1024-byte alignment");
  static_assert(SA >= 3, "weight ring");
  static_assert(FIXED + A_RING + B_RING <= kSmemBudget, "shared memory budget");
  static_assert(N_BARS * 8 + 16 <= kBarBytes, "barrier area");
};

template <int FMT, int PHASE, int TN>
constexpr size_t smem_bytes(int E) {
  using C = Cfg<FMT, PHASE, TN>;
  return 1024 + static_cast<size_t>(C::A_RING) + C::B_RING + C::UP_BYTES + kBarBytes +
         3 * static_cast<size_t>(E + 1) * 4;
}

struct Unit {
  int e, m, q0, nvalid, ph;   // ph: 1 = gate/up GEMV, 2 = down GEMV
};

// unit u -> (phase, expert, tile, chunk of TN pairs).  ustart[e] = first unit
// of expert e in the table built with tiles1 tiles per chunk.  A fused launch
// (PHASE 3) runs the n1 = ustart[E] gate/up units first and then the down
// units, whose table is ustart scaled by tiles2 / tiles1 (both phases count
// tiles x chunks(e) per expert).
template <int PHASE, int TN>
__device__ __forceinline__ Unit unit_of(const TcDecodeParams& P, const int32_t* ustart, int tiles1, int tiles2,
                                        int u) {
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

// First byte of unit U's weight tile (its K stages follow at A_STAGE).
template <int FMT>
__device__ __forceinline__ const uint8_t* tile_base(const TcDecodeParams& P, const Unit& U, const int32_t* eslot) {
  using C = Cfg<FMT, 1, 32>;   // the weight stages depend on neither phase nor TN
  const int K = (U.ph == 1) ? P.d : P.I;
  const uint8_t* blob = P.pool + static_cast<size_t>(eslot[U.e]) * P.blob_bytes;
  return blob + (U.ph == 1 ? P.L.wg : P.L.wd) + static_cast<size_t>(U.m) * (K / C::KSTAGE) * C::A_STAGE;
}

__device__ __forceinline__ void prefetch_l2(const void* p, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

__device__ __forceinline__ float silu(float h) { return h / (1.0f + expf(-h)); }

__device__ __forceinline__ void split_bf16(float a, uint16_t* hi, uint16_t* lo) {
  const __nv_bfloat16 h = __float2bfloat16_rn(a);
  const __nv_bfloat16 l = __float2bfloat16_rn(a - __bfloat162float(h));
  *hi = __bfloat16_as_ushort(h);
  *lo = __bfloat16_as_ushort(l);
}

// gemv<1>: the token of each of the unit's pairs (lane q: pair q0 + q).
__device__ __forceinline__ int token_of(const TcDecodeParams& P, const Unit& U, int lane, int n_pairs) {
  int tok = 0;
  if (U.ph == 1 && lane < U.nvalid) {
    const int p = __ldg(P.perm + U.q0 + lane);
    if (p < 0 || p >= n_pairs) report(P.status, MOE_ERR_DEVICE);
    else tok = p / P.k;
  }
  return tok;
}

// gemv<2>: the smallest a-plane box (8, 16 or 32 rows) that holds the unit's
// pairs.  With TN = 16 a unit has at most min(16, T*k) pairs, box 1.
template <int TN>
__device__ __forceinline__ int a_box(const TcDecodeParams& P, int nvalid) {
  if (nvalid <= P.a_box_rows[0]) return 0;
  return (TN == 16 || nvalid <= P.a_box_rows[1]) ? 1 : 2;
}

// Bytes that land in a token-row stage of unit U.
template <class C, int TN>
__device__ __forceinline__ uint32_t b_bytes(const TcDecodeParams& P, const Unit& U) {
  const uint32_t rows =
      U.ph == 1 ? static_cast<uint32_t>(U.nvalid) : 2u * static_cast<uint32_t>(P.a_box_rows[a_box<TN>(P, U.nvalid)]);
  return rows * C::ATOMS * 128u;
}

// Token rows of K stage ks of unit U into sB, completing on bar (whose
// expected bytes lane 0 has posted): gemv<1> one row TMA of x per pair and
// atom, lane q loading pair q0 + q; gemv<2> both planes of the a box, rows
// past the unit's pairs never read back.  Called by all lanes of one warp.
template <class C, int TN>
__device__ __forceinline__ void load_b(const TcDecodeParams& P, const Unit& U, int ks, int tok, uint8_t* sB,
                                       uint64_t* bar, const CUtensorMap* tm_x, const CUtensorMap* tm_a,
                                       const CUtensorMap* tm_a16, const CUtensorMap* tm_a8, uint64_t pol, int lane) {
  if (U.ph == 2) {
    if (lane == 0) {
      const int bi = a_box<TN>(P, U.nvalid);
      const CUtensorMap* tm = bi == 0 ? tm_a8 : (bi == 1 ? tm_a16 : tm_a);
#pragma unroll
      for (int pl = 0; pl < 2; ++pl)
#pragma unroll
        for (int a = 0; a < C::ATOMS; ++a)
          tma_load_3d(sB + (pl * C::ATOMS + a) * C::B_ATOM, tm, bar, ks * C::KSTAGE + 64 * a, U.q0, pl, pol);
    }
  } else if (lane < U.nvalid) {
#pragma unroll
    for (int a = 0; a < C::ATOMS; ++a)
      tma_load_2d(sB + a * C::B_ATOM + lane * 128, tm_x, bar, ks * C::KSTAGE + 64 * a, tok, pol);
  }
}

// One-launch schedule: lane 0 waits (bounded, like every wait) until all
// `target` gate/up units of expert e have published their a rows, then orders
// the TMA loads that follow after what it observed.  `seen` is the counter
// value lane 0 loaded ahead of time (relaxed, while the previous unit
// streamed): when it already reaches the target, a fence gives the acquire
// without another trip to memory.  One verdict for the warp.
__device__ __forceinline__ bool wait_expert_ready(const TcDecodeParams& P, int e, int target, int seen,
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
__device__ __forceinline__ int peek_expert_counter(const TcDecodeParams& P, int e) {
  int v;
  asm volatile("ld.relaxed.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(P.done1 + e) : "memory");
  return v;
}

// Waits for the copies of the last min(issued, n) stages of a ring to land.
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

template <int FMT, int PHASE, int TN>
__global__ void __launch_bounds__(Cfg<FMT, PHASE, TN>::THREADS, 1)
    gemv_tc_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_a,
                   const __grid_constant__ CUtensorMap tm_a16, const __grid_constant__ CUtensorMap tm_a8,
                   TcDecodeParams P) {
  using C = Cfg<FMT, PHASE, TN>;
  constexpr int THREADS = C::THREADS;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* ring_b = smem + C::A_RING;           // token-row stages
  float* up_buf = reinterpret_cast<float*>(ring_b + C::B_RING);
  uint64_t* bars = reinterpret_cast<uint64_t*>(ring_b + C::B_RING + C::UP_BYTES);
  uint64_t* full = bars;                        // [SA] weight stage landed
  uint64_t* empty = bars + C::SA;               // [SA] weight stage free
  uint64_t* tfull = bars + 2 * C::SA;           // [2]
  uint64_t* tempty = tfull + 2;                 // [2]
  uint64_t* drain = tfull + 4;                  // [1]
  uint64_t* bfull = tfull + 5;                  // [SB] token rows landed
  uint64_t* bempty = bfull + C::SB;             // [SB] token rows free
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
  auto ks_of = [&](const Unit& U) { return (U.ph == 1 ? P.d : P.I) / C::KSTAGE; };
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
                 "r"(C::TMEM_COLS));
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
    // L2 prefetch cursor over this CTA's (unit, stage) items
    int pf_u = blockIdx.x, pf_ks = 0, pf_ahead = 0, pf_KS = 0;
    const uint8_t* pf_base = nullptr;
    if (pf_u < n_units) {
      const Unit V = unit_of<PHASE, TN>(P, ustart, MT, MT2, pf_u);
      pf_base = tile_base<FMT>(P, V, eslot);
      pf_KS = ks_of(V);
    }
    for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
      const Unit U = unit_of<PHASE, TN>(P, ustart, MT, MT2, u);
      const uint8_t* abase = tile_base<FMT>(P, U, eslot);
      const int KS = ks_of(U);
      for (int ks = 0; ks < KS; ++ks) {
        // one verdict for the warp: its lanes take the same path
        if (!__all_sync(0xffffffffu, mbar_wait<true>(&empty[stage], phase ^ 1u, abort_flag, P.wait_ns))) {
          ok = false;
          break;
        }
        uint8_t* sA = smem + stage * C::A_STAGE;
        if (lane == 0) {
          mbar_expect_tx(&full[stage], C::A_STAGE);
          bulk_load(sA, abase + static_cast<size_t>(ks) * C::A_STAGE, C::A_STAGE, &full[stage], pol_stream);
          // keep the L2 prefetch cursor PF_ITEMS stages ahead of this one (the
          // bulk copies of a CTA complete in order, so prefetching whole blobs
          // up front would queue ahead of the stages the pipeline waits for)
          while (pf_u < n_units && pf_ahead < P.pf_items) {
            prefetch_l2(pf_base + static_cast<size_t>(pf_ks) * C::A_STAGE, C::A_STAGE);
            ++pf_ahead;
            if (++pf_ks == pf_KS) {
              pf_ks = 0;
              pf_u += gridDim.x;
              if (pf_u < n_units) {
                const Unit V = unit_of<PHASE, TN>(P, ustart, MT, MT2, pf_u);
                pf_base = tile_base<FMT>(P, V, eslot);
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
    // drain: the copies last issued into the ring have landed before exit
    drain_ring(full, C::SA, issued, stage, phase);
  } else if (warp == C::BPROD_WARP) {
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
      const int tok = token_of(P, U, lane, n_pairs);
      const int KS = ks_of(U);
      if (PHASE == 3 && U.ph == 2) {
        // the a rows of this expert's pairs come from every gate/up unit of the expert
        const int target = ustart[U.e + 1] - ustart[U.e];
        if (!wait_expert_ready(P, U.e, target, seen, abort_flag, lane)) {
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
        uint8_t* sB = ring_b + stage * C::B_STAGE;
        if (lane == 0) mbar_expect_tx(&bfull[stage], b_bytes<C, TN>(P, U));
        __syncwarp();
        load_b<C, TN>(P, U, ks, tok, sB, &bfull[stage], &tm_x, &tm_a, &tm_a16, &tm_a8, pol_keep, lane);
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
    int stage = 0, sa = 0;         // token-row ring; weight ring
    uint32_t phase = 0, pa = 0;
    int it = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x, ++it) {
      const Unit U = unit_of<PHASE, TN>(P, ustart, MT, MT2, u);
      const int KS = ks_of(U);
      const int n_mma = U.nvalid <= 16 ? 16 : 32;
      const uint32_t idesc = idesc_bf16(TM, n_mma);
      const int acc = it & 1;
      if (!__all_sync(0xffffffffu, mbar_wait<true>(&tempty[acc], ((it >> 1) & 1) ^ 1u, abort_flag, P.wait_ns))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t d_tmem = tmem + acc * ACC_COLS;
      for (int ks = 0; ks < KS; ++ks) {
        // the token rows and the weight stage have landed
        // one verdict for the warp: its lanes then take the same path to elect.sync
        const bool got = __all_sync(0xffffffffu, mbar_wait<true>(&bfull[stage], phase, abort_flag, P.wait_ns) &&
                                                     mbar_wait<true>(&full[sa], pa, abort_flag, P.wait_ns));
        if (!got) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (elect_one()) {
          const uint8_t* sA = smem + sa * C::A_STAGE;
          const uint8_t* sB = ring_b + stage * C::B_STAGE;
#pragma unroll
          for (int kk = 0; kk < C::KSTAGE / 16; ++kk) {   // K = 16 per MMA: +32 bytes
            const int a = kk >> 2;
            const uint64_t dh = desc_sw128(smem_u32(sB + a * C::B_ATOM)) + 2 * (kk & 3);
            const uint64_t dl = desc_sw128(smem_u32(sB + (C::ATOMS + a) * C::B_ATOM)) + 2 * (kk & 3);
            const uint32_t first = (ks > 0 || kk > 0) ? 1u : 0u;
            const uint64_t da = desc_sw128(smem_u32(sA + a * TM * 128)) + 2 * (kk & 3);
            tc_mma_bf16(d_tmem, da, dh, idesc, first);
            if (U.ph == 2) tc_mma_bf16(d_tmem, da, dl, idesc, 1u);
          }
          tc_commit(&empty[sa]);
          tc_commit(&bempty[stage]);
        }
        __syncwarp();
        if (++stage == C::SB) {
          stage = 0;
          phase ^= 1u;
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
    // ------------------------------------------------------------ epilogue (last four warps)
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
      if (U.ph == 2 && P.y_perm == nullptr && quad == 0 && lane < U.nvalid) {
        // the unit's column info, fetched while its accumulator is computed
        // (the barrier after the wait publishes it; the other buffer may still
        // be read by warps finishing the previous unit)
        const int p = __ldg(P.perm + U.q0 + lane);
        const bool good = p >= 0 && p < n_pairs;
        s_ctok[acc][lane] = good ? p / P.k : -1;
        s_cgate[acc][lane] = good ? __ldg(P.gate + p) : 0.f;
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
      tmem_ld32(tmem + (static_cast<uint32_t>(32 * quad) << 16) + acc * ACC_COLS, v);
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
          const int i = 32 * quad + lane;
          const size_t col = static_cast<size_t>(64) * U.m + i;
          const size_t plane = static_cast<size_t>(n_pairs) * P.I;
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            if (c < U.nvalid) {
              const float a = silu(v[c]) * up_buf[i * 33 + c];
              uint16_t hi, lo;
              split_bf16(a, &hi, &lo);
              const size_t o = static_cast<size_t>(U.q0 + c) * P.I + col;
              P.a_planes[o] = hi;
              P.a_planes[plane + o] = lo;
            }
          }
          // fused launch: the a rows are published to other CTAs (read there by TMA)
          if (PHASE == 3) {
            asm volatile("fence.proxy.async.global;" ::: "memory");
            __threadfence();
          }
        }
        named_sync(1, 128);
        if (PHASE == 3 && warp == C::EPI_WARP0 && lane == 0) atomicAdd(P.done1 + U.e, 1);
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
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(C::TMEM_COLS));
  }
}

template <int FMT, int PHASE, int TN>
moe_status launch_phase(const TcDecodeParams& P, const CUtensorMap& tx, const CUtensorMap& ta, const CUtensorMap& ta16,
                        const CUtensorMap& ta8, const DeviceInfo& dev, cudaStream_t s) {
  const size_t smem = smem_bytes<FMT, PHASE, TN>(P.E);
  if (smem > dev.smem_optin) return fail(MOE_ERR_UNSUPPORTED, "decode GEMV needs %zu bytes of shared memory", smem);
  static size_t attr[64] = {};
  if (attr[dev.id] < smem) {
    MOE_CUDA_TRY(cudaFuncSetAttribute(gemv_tc_kernel<FMT, PHASE, TN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      static_cast<int>(smem)));
    attr[dev.id] = smem;
  }
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(dev.sm_count);
  cfg.blockDim = dim3(Cfg<FMT, PHASE, TN>::THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  // the fused launch's CTAs wait on each other's gate/up units: all of them
  // must be resident at once, which a cooperative launch guarantees
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
  MOE_CUDA_TRY(cudaLaunchKernelEx(&cfg, gemv_tc_kernel<FMT, PHASE, TN>, tx, ta, ta16, ta8, P));
  MOE_LAUNCH_CHECK("gemv_tc_kernel");
  return MOE_OK;
}

template <int FMT, int TN>
moe_status launch_both(const TcDecodeParams& P, const CUtensorMap& tm_x, const CUtensorMap (&tm_a)[3],
                       const DeviceInfo& dev, cudaStream_t stream) {
  if (decode_one_launch(FMT, P.T)) {
    MOE_CUDA_TRY(cudaMemsetAsync(P.done1, 0, static_cast<size_t>(P.E) * sizeof(int32_t), stream));
    return launch_phase<FMT, 3, TN>(P, tm_x, tm_a[2], tm_a[1], tm_a[0], dev, stream);
  }
  moe_status st = launch_phase<FMT, 1, TN>(P, tm_x, tm_a[2], tm_a[1], tm_a[0], dev, stream);
  if (st != MOE_OK) return st;
  return launch_phase<FMT, 2, TN>(P, tm_x, tm_a[2], tm_a[1], tm_a[0], dev, stream);
}

}  // namespace

// Both GEMV launches for bf16 blobs in the tile layout.  ws holds the a
// planes (T*k*I*4 bytes).
moe_status launch_decode_tc(moe_shape s, const void* x, int T, int k, const int32_t* offsets, const int32_t* perm,
                            const int32_t* slot, const void* pool, int n_slots, const float* gate, float* y_perm,
                            float* out, void* ws, int32_t* status, const DeviceInfo& dev, cudaStream_t stream) {
  TcDecodeParams P{};
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
  P.a_planes = static_cast<uint16_t*>(ws);
  P.done1 = reinterpret_cast<int32_t*>(static_cast<uint8_t*>(ws) +
                                       round_up(static_cast<size_t>(T) * k * s.I * sizeof(float), 256));
  P.y_perm = y_perm;
  P.out = out;
  P.status = status;
  const uint64_t n = static_cast<uint64_t>(T) * k;
  for (int i = 0; i < 3; ++i) {
    const uint64_t r = static_cast<uint64_t>(8) << i;   // 8, 16, 32 (the widest chunk)
    P.a_box_rows[i] = static_cast<int>(n < r ? n : r);
  }
  CUtensorMap tm_x, tm_a[3];
  {
    const uint64_t dims[2] = {static_cast<uint64_t>(s.d), static_cast<uint64_t>(T)};
    const uint64_t str[1] = {static_cast<uint64_t>(s.d) * 2};
    const uint32_t box[2] = {64u, 1u};
    const CUresult r = encode_tiled_sw128(&tm_x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, x, dims, str, box);
    if (r != CUDA_SUCCESS) return fail(MOE_ERR_CUDA, "tensor map of x failed (%d)", static_cast<int>(r));
  }
  for (int i = 0; i < 3; ++i) {
    const uint64_t dims[3] = {static_cast<uint64_t>(s.I), n, 2};
    const uint64_t str[2] = {static_cast<uint64_t>(s.I) * 2, n * s.I * 2};
    const uint32_t box[3] = {64u, static_cast<uint32_t>(P.a_box_rows[i]), 1u};
    const CUresult r = encode_tiled_sw128(&tm_a[i], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, ws, dims, str, box);
    if (r != CUDA_SUCCESS) return fail(MOE_ERR_CUDA, "tensor map of the a planes failed (%d)", static_cast<int>(r));
  }
  // an expert holds at most one pair per token: with T <= 16 every chunk fits 16 rows
  return T <= 16 ? launch_both<MOE_W_BF16, 16>(P, tm_x, tm_a, dev, stream)
                 : launch_both<MOE_W_BF16, 32>(P, tm_x, tm_a, dev, stream);
}

}  // namespace moe
