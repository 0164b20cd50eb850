// Step 3 on bf16 weights (moe_expert_ffn without MOE_FFN_ACT_NVFP4, bf16 blobs
// in the tensor-core tile layout): the grouped SwiGLU expert FFN as two skinny
// GEMMs on the 5th-generation tensor cores.
//
// At decode sizes a layer call is bound by reading the routed experts' weights
// from HBM (explainx.ai hardware guide, "Decode: decide whether to move an
// expert or compute where it lives": one token touches few experts).  Here no
// SM instruction is spent per weight element: bulk copies move 32 KB weight
// stages into shared memory and one thread issues tcgen05.mma over them, with
// the few token rows of the group as the N side and the accumulators in TMEM.
//
//   gemv<1>: D[128 x N] = W_gu tile (64 gate + 64 up rows of the same
//            intermediate indices) x X^T over K = d, N <= 32 token rows
//            gathered by one-row TMA loads of x.  Epilogue: a = silu(D_gate) *
//            D_up, stored as two bf16 planes hi + lo (a - hi - lo ~ 2^-17 |a|)
//            in the workspace, rows = sorted pair positions.
//   gemv<2>: D[128 x N] = W_d tile x (A_hi + A_lo)^T over K = I (two MMAs per
//            k-step).  Epilogue: y_perm rows, or out[t] += gate * y (the fused
//            combine).
//
// Work unit = (expert, 128-row tile, chunk of <= 32 of the expert's pairs),
// expert-major, chunks fastest, dealt round-robin to one persistent CTA per
// SM.  Warp 0 produces (bulk copy of the weight stage, TMA loads of the token
// rows, L2 prefetch of the weight stages a few items ahead), warp 1 owns TMEM
// and issues the MMAs, warps 2-5 run the epilogue on double-buffered TMEM
// accumulators.  Every wait is bounded: on expiry the CTA records
// MOE_ERR_TIMEOUT, stops issuing, drains what it issued and frees its TMEM.
#include <cuda_bf16.h>

#include "common.cuh"
#include "tc.cuh"

namespace moe {

struct TcDecodeParams {
  int E, d, I, T, k, n_slots;
  int a_box_rows;            // rows of one TMA box of the a planes (min(32, T*k))
  const int32_t* offsets;
  const int32_t* perm;
  const int32_t* slot;
  const float* gate;
  const uint8_t* pool;
  size_t blob_bytes;
  BlobLayout L;
  __nv_bfloat16* a_planes;   // [2][T*k][I]: hi, lo
  float* y_perm;             // [T*k][d] or null (then out)
  float* out;                // [T][d] (fused combine)
  int32_t* status;
};

namespace {

using namespace ::moe::tc;

constexpr int TM = 128;                  // weight rows per tile
constexpr int TN = 32;                   // pairs per chunk (max MMA N)
constexpr int A_ATOM = TM * 128;         // one 64-element atom of a tile: 16 KB
constexpr int B_ATOM = TN * 128;         // one atom of the token rows: 4 KB
constexpr int ATOMS = 2;                 // atoms per stage: K = 128
constexpr int A_STAGE = ATOMS * A_ATOM;  // 32 KB, one bulk copy
constexpr int THREADS = 192;             // producer, MMA, 4 epilogue warps
constexpr int ACC_COLS = 32;             // TMEM columns per accumulator
constexpr int TMEM_COLS = 64;            // two accumulators
constexpr int PF_ITEMS = 4;              // L2 prefetch distance (stages)
constexpr size_t kBlobPrefetchCap = 96ull << 20;

template <int PHASE> struct Cfg;
template <> struct Cfg<1> {
  static constexpr int B_BYTES = ATOMS * B_ATOM;              // x rows
  static constexpr int STAGE = A_STAGE + B_BYTES;             // 40 KB
  static constexpr int STAGES = 5;
  static constexpr int UP_BYTES = 64 * 33 * 4;                // up-row exchange
};
template <> struct Cfg<2> {
  static constexpr int B_BYTES = 2 * ATOMS * B_ATOM;          // a hi + lo rows
  static constexpr int STAGE = A_STAGE + B_BYTES;             // 48 KB
  static constexpr int STAGES = 4;
  static constexpr int UP_BYTES = 0;
};

template <int PHASE>
constexpr size_t smem_bytes(int E) {
  return 1024 + static_cast<size_t>(Cfg<PHASE>::STAGES) * Cfg<PHASE>::STAGE + Cfg<PHASE>::UP_BYTES + 256 +
         static_cast<size_t>(E + 1) * 4;
}

struct Unit {
  int e, m, q0, nvalid;
};

// unit u -> (expert, tile, chunk); ustart[e] = first unit of expert e
__device__ __forceinline__ Unit unit_of(const TcDecodeParams& P, const int32_t* ustart, int MT, int u) {
  int lo = 0, hi = P.E;   // ustart[lo] <= u < ustart[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (ustart[mid] <= u) lo = mid;
    else hi = mid;
  }
  Unit U;
  U.e = lo;
  const int q_begin = __ldg(P.offsets + lo), ne = __ldg(P.offsets + lo + 1) - q_begin;
  const int chunks = (ne + TN - 1) / TN;
  const int local = u - ustart[lo];
  U.m = local / chunks;
  const int c = local % chunks;
  U.q0 = q_begin + c * TN;
  U.nvalid = min(TN, ne - c * TN);
  return U;
}

// First byte of unit U's weight tile (its K stages follow at A_STAGE).
template <int PHASE>
__device__ __forceinline__ const uint8_t* tile_base(const TcDecodeParams& P, const Unit& U) {
  const int K = (PHASE == 1) ? P.d : P.I;
  const uint8_t* blob = P.pool + static_cast<size_t>(__ldg(P.slot + U.e)) * P.blob_bytes;
  return blob + (PHASE == 1 ? P.L.wg : P.L.wd) + static_cast<size_t>(U.m) * (K / 64) * A_ATOM;
}

__device__ __forceinline__ void prefetch_l2(const void* p, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

__device__ __forceinline__ float silu(float h) { return h / (1.0f + expf(-h)); }

template <int PHASE>
__global__ void __launch_bounds__(THREADS, 1) gemv_bf16_kernel(const __grid_constant__ CUtensorMap tm_b,
                                                               TcDecodeParams P) {
  using C = Cfg<PHASE>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float* up_buf = reinterpret_cast<float*>(smem + C::STAGES * C::STAGE);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::STAGES * C::STAGE + C::UP_BYTES);
  uint64_t* full = bars;                        // [STAGES]
  uint64_t* empty = bars + C::STAGES;           // [STAGES]
  uint64_t* tfull = bars + 2 * C::STAGES;       // [2]
  uint64_t* tempty = bars + 2 * C::STAGES + 2;  // [2]
  uint64_t* drain = bars + 2 * C::STAGES + 4;   // [1]
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 2 * C::STAGES + 5);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  volatile int* epi_fail = reinterpret_cast<volatile int*>(tmem_holder + 2);
  int32_t* ustart = reinterpret_cast<int32_t*>(smem + C::STAGES * C::STAGE + C::UP_BYTES + 256);
  __shared__ int ws[36];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int K = (PHASE == 1) ? P.d : P.I;
  const int KS = K / (64 * ATOMS);
  const int MT = (PHASE == 1) ? P.I / 64 : P.d / TM;
  const int n_pairs = P.T * P.k;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 128);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    *epi_fail = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_holder)),
                 "r"(TMEM_COLS));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }

  // ---- units per expert (evaluated experts only) and their exclusive prefix
  const int per = (P.E + THREADS - 1) / THREADS;
  const int e0 = threadIdx.x * per;
  int cnt = 0, act = 0;
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
    ++act;
  }
  int total = 0;
  int run = block_scan(cnt, ws, &total);
  int n_act = 0;
  block_scan(act, ws, &n_act);
  for (int j = 0; j < per; ++j) {
    const int e = e0 + j;
    if (e >= P.E) break;
    ustart[e] = run;
    const int a = __ldg(P.offsets + e), b = __ldg(P.offsets + e + 1);
    const int s = __ldg(P.slot + e);
    if (b > a && a >= 0 && b <= n_pairs && s >= 0 && s < P.n_slots) run += MT * ((b - a + TN - 1) / TN);
  }
  if (threadIdx.x == 0) ustart[P.E] = total;
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const int n_units = total;

  // small expert sets: request every active blob into L2 up front (all of the
  // layer's DRAM reads in flight at once); the weights come through L2 anyway
  if (PHASE == 1 && static_cast<size_t>(n_act) * P.blob_bytes <= kBlobPrefetchCap) {
    const size_t chunk = 16384;
    const size_t per_blob = (P.blob_bytes + chunk - 1) / chunk;
    const size_t stride = static_cast<size_t>(gridDim.x) * THREADS;
    size_t idx = static_cast<size_t>(blockIdx.x) * THREADS + threadIdx.x;
    for (int e = 0; e < P.E; ++e) {
      if (ustart[e + 1] == ustart[e]) continue;
      const uint8_t* blob = P.pool + static_cast<size_t>(__ldg(P.slot + e)) * P.blob_bytes;
      for (; idx < per_blob; idx += stride) {
        const size_t off = idx * chunk;
        prefetch_l2(blob + off, static_cast<uint32_t>(min(chunk, P.blob_bytes - off)));
      }
      idx -= per_blob;
    }
  }

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    const uint64_t pol_stream = policy_evict_first(), pol_keep = policy_evict_last();
    const bool pf_on = static_cast<size_t>(n_act) * P.blob_bytes > kBlobPrefetchCap;
    int stage = 0;
    uint32_t phase = 0;
    int issued = 0;
    bool ok = true;
    // L2 prefetch cursor over this CTA's (unit, stage) items
    int pf_u = blockIdx.x, pf_ks = 0, pf_ahead = 0;
    const uint8_t* pf_base = nullptr;
    if (pf_on && pf_u < n_units) pf_base = tile_base<PHASE>(P, unit_of(P, ustart, MT, pf_u));
    for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
      const Unit U = unit_of(P, ustart, MT, u);
      const uint8_t* abase = tile_base<PHASE>(P, U);
      int tok = 0;
      if (PHASE == 1 && lane < U.nvalid) {
        const int p = __ldg(P.perm + U.q0 + lane);
        if (p < 0 || p >= n_pairs) report(P.status, MOE_ERR_DEVICE);
        else tok = p / P.k;
      }
      for (int ks = 0; ks < KS; ++ks) {
        if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        uint8_t* sA = smem + stage * C::STAGE;
        uint8_t* sB = sA + A_STAGE;
        if (lane == 0) {
          const uint32_t bytes =
              A_STAGE + (PHASE == 1 ? 2u * U.nvalid : 2u * ATOMS * static_cast<uint32_t>(P.a_box_rows)) * 128u;
          mbar_expect_tx(&full[stage], bytes);
          bulk_load(sA, abase + static_cast<size_t>(ks) * A_STAGE, A_STAGE, &full[stage], pol_stream);
          if (PHASE == 2) {
#pragma unroll
            for (int pl = 0; pl < 2; ++pl)
#pragma unroll
              for (int a = 0; a < ATOMS; ++a)
                tma_load_3d(sB + (pl * ATOMS + a) * B_ATOM, &tm_b, &full[stage], ks * 128 + 64 * a, U.q0, pl,
                            pol_keep);
          }
          // keep the L2 prefetch cursor PF_ITEMS stages ahead of this one
          if (pf_on) {
            while (pf_u < n_units && pf_ahead < PF_ITEMS) {
              prefetch_l2(pf_base + static_cast<size_t>(pf_ks) * A_STAGE, A_STAGE);
              ++pf_ahead;
              if (++pf_ks == KS) {
                pf_ks = 0;
                pf_u += gridDim.x;
                if (pf_u < n_units) pf_base = tile_base<PHASE>(P, unit_of(P, ustart, MT, pf_u));
              }
            }
            --pf_ahead;
          }
        }
        __syncwarp();
        if (PHASE == 1 && lane < U.nvalid) {
#pragma unroll
          for (int a = 0; a < ATOMS; ++a)
            tma_load_2d(sB + a * B_ATOM + lane * 128, &tm_b, &full[stage], ks * 128 + 64 * a, tok, pol_keep);
        }
        __syncwarp();
        ++issued;
        if (++stage == C::STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
    if (!ok) {
      report(P.status, MOE_ERR_TIMEOUT);
      *abort_flag = 1;
    }
    // drain: the copies last issued into the ring have landed before exit
    const int outstanding = issued < C::STAGES ? issued : C::STAGES;
    int s = stage;
    uint32_t ph = phase;
    for (int i = 0; i < outstanding; ++i) {
      if (--s < 0) {
        s = C::STAGES - 1;
        ph ^= 1u;
      }
      mbar_drain(&full[s], ph);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    int stage = 0;
    uint32_t phase = 0;
    int it = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x, ++it) {
      const Unit U = unit_of(P, ustart, MT, u);
      const uint32_t idesc = idesc_bf16(TM, U.nvalid <= 16 ? 16 : 32);
      const int acc = it & 1;
      if (!mbar_wait(&tempty[acc], ((it >> 1) & 1) ^ 1u, abort_flag)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t d_tmem = tmem + acc * ACC_COLS;
      for (int ks = 0; ks < KS; ++ks) {
        if (!mbar_wait(&full[stage], phase, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (elect_one()) {
          uint8_t* sA = smem + stage * C::STAGE;
          uint8_t* sB = sA + A_STAGE;
#pragma unroll
          for (int a = 0; a < ATOMS; ++a) {
            const uint64_t da = desc_sw128(smem_u32(sA + a * A_ATOM));
            const uint64_t dh = desc_sw128(smem_u32(sB + a * B_ATOM));
            const uint64_t dl = desc_sw128(smem_u32(sB + (ATOMS + a) * B_ATOM));
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {   // K = 16 per MMA: +32 bytes
              tc_mma_bf16(d_tmem, da + 2 * kk, dh + 2 * kk, idesc, (ks > 0 || a > 0 || kk > 0) ? 1u : 0u);
              if (PHASE == 2) tc_mma_bf16(d_tmem, da + 2 * kk, dl + 2 * kk, idesc, 1u);
            }
          }
          tc_commit(&empty[stage]);
        }
        __syncwarp();
        if (++stage == C::STAGES) {
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
    if (elect_one()) tc_commit(drain);
    __syncwarp();
    mbar_drain(drain, 0);
  } else {
    // ------------------------------------------------------------ epilogue (warps 2..5)
    const int quad = warp & 3;                       // TMEM lanes 32*quad .. 32*quad+31
    int it = 0;
    for (int u = blockIdx.x; u < n_units; u += gridDim.x, ++it) {
      const Unit U = unit_of(P, ustart, MT, u);
      const int acc = it & 1;
      // the four warps leave together: a warp alone at a named barrier would wait for good
      if (!mbar_wait(&tfull[acc], (it >> 1) & 1, abort_flag)) *epi_fail = 1;
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
      if (PHASE == 1) {
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
              const __nv_bfloat16 hi = __float2bfloat16_rn(a);
              const __nv_bfloat16 lo = __float2bfloat16_rn(a - __bfloat162float(hi));
              const size_t o = static_cast<size_t>(U.q0 + c) * P.I + col;
              P.a_planes[o] = hi;
              P.a_planes[plane + o] = lo;
            }
          }
        }
        named_sync(1, 128);
      } else {
        const int row = TM * U.m + 32 * quad + lane;
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          if (c < U.nvalid) {
            const int q = U.q0 + c;
            if (P.y_perm != nullptr) {
              P.y_perm[static_cast<size_t>(q) * P.d + row] = v[c];
            } else {
              const int p = __ldg(P.perm + q);
              if (p >= 0 && p < n_pairs)
                atomicAdd(P.out + static_cast<size_t>(p / P.k) * P.d + row, __ldg(P.gate + p) * v[c]);
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

template <int PHASE>
moe_status launch_phase(const TcDecodeParams& P, const CUtensorMap& tm, const DeviceInfo& dev, cudaStream_t s) {
  const size_t smem = smem_bytes<PHASE>(P.E);
  if (smem > dev.smem_optin) return fail(MOE_ERR_UNSUPPORTED, "decode GEMV needs %zu bytes of shared memory", smem);
  static size_t attr[64] = {};
  if (attr[dev.id] < smem) {
    MOE_CUDA_TRY(cudaFuncSetAttribute(gemv_bf16_kernel<PHASE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      static_cast<int>(smem)));
    attr[dev.id] = smem;
  }
  gemv_bf16_kernel<PHASE><<<dev.sm_count, THREADS, smem, s>>>(tm, P);
  MOE_LAUNCH_CHECK("gemv_bf16_kernel");
  return MOE_OK;
}

}  // namespace

// bf16 blobs in the tile layout: both GEMV launches.  ws holds the a planes
// (T*k*I*4 bytes).
moe_status launch_decode_tc(moe_shape s, const void* x, int T, int k, const int32_t* offsets, const int32_t* perm,
                            const int32_t* slot, const void* pool, int n_slots, const float* gate, float* y_perm,
                            float* out, void* ws, int32_t* status, const DeviceInfo& dev, cudaStream_t stream) {
  TcDecodeParams P{};
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
  P.a_planes = static_cast<__nv_bfloat16*>(ws);
  P.y_perm = y_perm;
  P.out = out;
  P.status = status;
  const uint64_t n = static_cast<uint64_t>(T) * k;
  P.a_box_rows = static_cast<int>(n < static_cast<uint64_t>(TN) ? n : static_cast<uint64_t>(TN));
  CUtensorMap tm_x, tm_a;
  {
    const uint64_t dims[2] = {static_cast<uint64_t>(s.d), static_cast<uint64_t>(T)};
    const uint64_t str[1] = {static_cast<uint64_t>(s.d) * 2};
    const uint32_t box[2] = {64u, 1u};
    const CUresult r = encode_tiled_sw128(&tm_x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, x, dims, str, box);
    if (r != CUDA_SUCCESS) return fail(MOE_ERR_CUDA, "tensor map of x failed (%d)", static_cast<int>(r));
  }
  {
    const uint64_t dims[3] = {static_cast<uint64_t>(s.I), n, 2};
    const uint64_t str[2] = {static_cast<uint64_t>(s.I) * 2, n * s.I * 2};
    const uint32_t box[3] = {64u, static_cast<uint32_t>(P.a_box_rows), 1u};
    const CUresult r = encode_tiled_sw128(&tm_a, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, ws, dims, str, box);
    if (r != CUDA_SUCCESS) return fail(MOE_ERR_CUDA, "tensor map of the a planes failed (%d)", static_cast<int>(r));
  }
  moe_status st = launch_phase<1>(P, tm_x, dev, stream);
  if (st != MOE_OK) return st;
  return launch_phase<2>(P, tm_a, dev, stream);
}

}  // namespace moe
