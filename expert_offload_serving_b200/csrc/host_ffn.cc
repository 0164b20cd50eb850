// The host side of the split of a decode step's cache misses: the SwiGLU
// expert FFN computed on the CPU cores, straight from the expert blobs in the
// pinned host pool, for the experts the split leaves on the host
// (explainx.ai hardware guide, "Decode: decide whether to move an expert or
// compute where it lives": a missed expert can run on the CPU against
// host-resident weights, concurrently with the fills; freetoken.wiki
// "FreeToken 753b model", "How MoE Paging and Caching Work": bandwidth-adaptive
// execution splits misses between PCIe fills and CPU computation).
//
// moe_host_expert_ffn writes the gate-weighted partial sum of the pairs whose
// expert is in the host set; moe_combine_merge adds it to the GPU share.  The
// work is bound by reading the experts' weight bytes from host memory, so each
// weight row is decoded once (MXFP4 / NVFP4: E2M1 codes through a 16-entry
// table, times the block scale; bf16: a shift) and multiplied into every pair
// of its expert.  Two passes: gate/up rows (tasks = 64-row chunks of I per
// expert), then down rows (tasks = 64-row chunks of d, each summing every host
// expert into its own output columns, so no two tasks write the same word).
// Tasks run on a persistent pool of worker threads plus the caller.
//
// This file is compiled by the host compiler (not nvcc): the AVX2 + FMA path
// is selected at run time when the CPU has it, else a scalar path computes the
// same sums.
#include "host_ffn.h"

#include <algorithm>
#include <atomic>
#include <chrono>
#include <cmath>
#include <condition_variable>
#include <cstring>
#include <functional>
#include <mutex>
#include <thread>
#include <vector>

#include <immintrin.h>

namespace moe {
namespace host {

namespace {

// ------------------------------------------------------------------ thread pool
// Persistent workers.  Each run() publishes a job that lives on the caller's
// stack; a worker joins it under the lock (at most `threads - 1` join), takes
// task indices from the job's counter, and leaves under the lock.  run()
// returns only when every task is done and every worker that joined has left,
// and it unpublishes the job first, so no worker ever touches a finished job.
class Pool {
 public:
  static Pool& get() {
    static Pool p;
    return p;
  }

  void run(int n, int threads, const std::function<void(int)>& fn) {
    if (n <= 0) return;
    threads = std::max(1, std::min(threads, n));
    if (threads == 1) {
      for (int i = 0; i < n; ++i) fn(i);
      return;
    }
    std::lock_guard<std::mutex> one_job(call_mu_);
    Job job;
    job.fn = &fn;
    job.n = n;
    job.max_joiners = threads - 1;
    {
      std::lock_guard<std::mutex> g(mu_);
      ensure(threads - 1);
      job_ = &job;
      ++gen_;
    }
    cv_.notify_all();
    work(job);
    std::unique_lock<std::mutex> g(mu_);
    done_cv_.wait(g, [&] { return job.done.load() == n && job.inside == 0; });
    job_ = nullptr;
  }

  ~Pool() {
    {
      std::lock_guard<std::mutex> g(mu_);
      stop_ = true;
    }
    cv_.notify_all();
    for (auto& t : workers_) t.join();
  }

 private:
  struct Job {
    const std::function<void(int)>* fn = nullptr;
    int n = 0, max_joiners = 0, joined = 0, inside = 0;
    std::atomic<int> next{0}, done{0};
  };

  void ensure(int want) {
    while (static_cast<int>(workers_.size()) < want) workers_.emplace_back([this] { loop(); });
  }

  static void work(Job& j) {
    for (;;) {
      const int i = j.next.fetch_add(1);
      if (i >= j.n) break;
      (*j.fn)(i);
      j.done.fetch_add(1);
    }
  }

  void loop() {
    uint64_t seen = 0;
    for (;;) {
      Job* j = nullptr;
      {
        std::unique_lock<std::mutex> g(mu_);
        cv_.wait(g, [&] { return stop_ || (job_ != nullptr && gen_ != seen); });
        if (stop_) return;
        seen = gen_;
        j = job_;
        if (j->joined >= j->max_joiners) continue;
        ++j->joined;
        ++j->inside;
      }
      work(*j);
      {
        std::lock_guard<std::mutex> g(mu_);
        --j->inside;
      }
      done_cv_.notify_all();
    }
  }

  std::mutex call_mu_, mu_;
  std::condition_variable cv_, done_cv_;
  std::vector<std::thread> workers_;
  Job* job_ = nullptr;
  uint64_t gen_ = 0;
  bool stop_ = false;
};

// ------------------------------------------------------------------ weight rows
// E2M1 magnitudes times two (0, 0.5, 1, 1.5, 2, 3, 4, 6 -> small integers),
// with the sign bit; the block scale carries the factor 1/2.
constexpr int8_t kE2m1x2[16] = {0, 1, 2, 3, 4, 6, 8, 12, 0, -1, -2, -3, -4, -6, -8, -12};

inline float e8m0(uint8_t b) {
  if (b == 255) return NAN;
  if (b == 0) return std::ldexp(1.0f, -127);
  uint32_t bits = static_cast<uint32_t>(b) << 23;
  float f;
  std::memcpy(&f, &bits, 4);
  return f;
}

inline float e4m3(uint8_t b) {
  const int s = b >> 7, e = (b >> 3) & 15, m = b & 7;
  if (e == 15 && m == 7) return NAN;
  const float mag = e == 0 ? std::ldexp(static_cast<float>(m), -9) : std::ldexp(1.0f + m / 8.0f, e - 7);
  return s ? -mag : mag;
}

inline float bf16f(uint16_t h) {
  const uint32_t bits = static_cast<uint32_t>(h) << 16;
  float f;
  std::memcpy(&f, &bits, 4);
  return f;
}

// Which matrix of an expert blob a row belongs to.
enum Mat { GATE = 0, UP = 1, DOWN = 2 };

// Decodes row r (gate/up: intermediate index; down: output index) of one
// matrix of a blob into dst[K] floats.
struct Rows {
  moe_shape s;
  BlobLayout L;
  float ts[3];                 // NVFP4 tensor scales (gate, up, down) of the current blob

  void decode(const uint8_t* blob, Mat m, int r, float* dst) const {
    const int K = m == DOWN ? s.I : s.d;
    if (s.fmt == MOE_W_BF16) {
      if (bf16_blocked(s.d, s.I)) {
        const int row = m == DOWN ? r : gu_row(r, m == UP);
        const uint8_t* base = blob + (m == DOWN ? L.wd : L.wg);
        for (int k = 0; k < K; k += 8) {
          const uint16_t* src = reinterpret_cast<const uint16_t*>(base + sw128_offset(row, k, K));
          for (int j = 0; j < 8; ++j) dst[k + j] = bf16f(src[j]);
        }
      } else {
        const uint16_t* src =
            reinterpret_cast<const uint16_t*>(blob + (m == GATE ? L.wg : m == UP ? L.wu : L.wd)) +
            static_cast<size_t>(r) * K;
        for (int k = 0; k < K; ++k) dst[k] = bf16f(src[k]);
      }
      return;
    }
    if (s.fmt == MOE_W_MXFP4) {
      const uint8_t *codes, *sc;
      const bool tiled = mx_tiled(s.d, s.I);
      const int row = (tiled && m != DOWN) ? gu_row(r, m == UP) : r;
      for (int j = 0; j < K / 32; ++j) {
        if (tiled) {
          const uint8_t* base = blob + (m == DOWN ? L.wd : L.wg);
          codes = base + mx_tile_code_offset(row, 16 * j, K);
          sc = base + mx_tile_scale_offset(row, j, K);
        } else {
          codes = blob + (m == GATE ? L.wg : m == UP ? L.wu : L.wd) + static_cast<size_t>(r) * (K / 2) + 16 * j;
          sc = blob + (m == GATE ? L.sg : m == UP ? L.su : L.sd) + static_cast<size_t>(r) * (K / 32) + j;
        }
        const float scale = 0.5f * e8m0(*sc);
        for (int i = 0; i < 16; ++i) {
          dst[32 * j + 2 * i] = kE2m1x2[codes[i] & 15] * scale;
          dst[32 * j + 2 * i + 1] = kE2m1x2[codes[i] >> 4] * scale;
        }
      }
      return;
    }
    // NVFP4: W_gu rows interleaved (gu_row), scales in scale-factor atoms
    const int row = m == DOWN ? r : gu_row(r, m == UP);
    const uint8_t* codes = blob + (m == DOWN ? L.wd : L.wg) + static_cast<size_t>(row) * (K / 2);
    const uint8_t* sbase = blob + (m == DOWN ? L.sd : L.sg);
    const float g = ts[m];
    for (int j = 0; j < K / 16; ++j) {
      const float scale = 0.5f * e4m3(sbase[sf_atom_offset(row, j, K)]) * g;
      for (int i = 0; i < 8; ++i) {
        dst[16 * j + 2 * i] = kE2m1x2[codes[8 * j + i] & 15] * scale;
        dst[16 * j + 2 * i + 1] = kE2m1x2[codes[8 * j + i] >> 4] * scale;
      }
    }
  }
};

// dot products of one decoded row with n vectors (each K floats)
float dot_scalar(const float* w, const float* v, int K) {
  float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
  int k = 0;
  for (; k + 4 <= K; k += 4) {
    a0 += w[k] * v[k];
    a1 += w[k + 1] * v[k + 1];
    a2 += w[k + 2] * v[k + 2];
    a3 += w[k + 3] * v[k + 3];
  }
  for (; k < K; ++k) a0 += w[k] * v[k];
  return (a0 + a1) + (a2 + a3);
}

__attribute__((target("avx2,fma"))) float dot_avx2(const float* w, const float* v, int K) {
  __m256 a0 = _mm256_setzero_ps(), a1 = _mm256_setzero_ps(), a2 = _mm256_setzero_ps(), a3 = _mm256_setzero_ps();
  int k = 0;
  for (; k + 32 <= K; k += 32) {
    a0 = _mm256_fmadd_ps(_mm256_loadu_ps(w + k), _mm256_loadu_ps(v + k), a0);
    a1 = _mm256_fmadd_ps(_mm256_loadu_ps(w + k + 8), _mm256_loadu_ps(v + k + 8), a1);
    a2 = _mm256_fmadd_ps(_mm256_loadu_ps(w + k + 16), _mm256_loadu_ps(v + k + 16), a2);
    a3 = _mm256_fmadd_ps(_mm256_loadu_ps(w + k + 24), _mm256_loadu_ps(v + k + 24), a3);
  }
  __m256 a = _mm256_add_ps(_mm256_add_ps(a0, a1), _mm256_add_ps(a2, a3));
  __m128 h = _mm_add_ps(_mm256_castps256_ps128(a), _mm256_extractf128_ps(a, 1));
  h = _mm_add_ps(h, _mm_movehl_ps(h, h));
  h = _mm_add_ss(h, _mm_shuffle_ps(h, h, 1));
  float r = _mm_cvtss_f32(h);
  for (; k < K; ++k) r += w[k] * v[k];
  return r;
}

// MXFP4 row of the tiled layout decoded with AVX2: 16 code bytes -> 32 values
// per block (nibbles through the E2M1 table by a byte shuffle, then int8 ->
// fp32 times half the E8M0 scale).
__attribute__((target("avx2,fma"))) void decode_mx_tiled_avx2(const uint8_t* base, int row, int K, float* dst) {
  const __m128i lut = _mm_loadu_si128(reinterpret_cast<const __m128i*>(kE2m1x2));
  const __m128i m0f = _mm_set1_epi8(0x0f);
  for (int j = 0; j < K / 32; ++j) {
    const uint8_t* codes = base + mx_tile_code_offset(row, 16 * j, K);
    const __m256 sc = _mm256_set1_ps(0.5f * e8m0(base[mx_tile_scale_offset(row, j, K)]));
    const __m128i b = _mm_loadu_si128(reinterpret_cast<const __m128i*>(codes));
    const __m128i lo = _mm_and_si128(b, m0f);
    const __m128i hi = _mm_and_si128(_mm_srli_epi16(b, 4), m0f);
    const __m128i e0 = _mm_shuffle_epi8(lut, _mm_unpacklo_epi8(lo, hi));   // elements 0..15
    const __m128i e1 = _mm_shuffle_epi8(lut, _mm_unpackhi_epi8(lo, hi));   // elements 16..31
    float* d = dst + 32 * j;
    _mm256_storeu_ps(d, _mm256_mul_ps(_mm256_cvtepi32_ps(_mm256_cvtepi8_epi32(e0)), sc));
    _mm256_storeu_ps(d + 8, _mm256_mul_ps(_mm256_cvtepi32_ps(_mm256_cvtepi8_epi32(_mm_srli_si128(e0, 8))), sc));
    _mm256_storeu_ps(d + 16, _mm256_mul_ps(_mm256_cvtepi32_ps(_mm256_cvtepi8_epi32(e1)), sc));
    _mm256_storeu_ps(d + 24, _mm256_mul_ps(_mm256_cvtepi32_ps(_mm256_cvtepi8_epi32(_mm_srli_si128(e1, 8))), sc));
  }
}

bool have_avx2() {
  static const bool ok = __builtin_cpu_supports("avx2") && __builtin_cpu_supports("fma");
  return ok;
}

inline float silu(float h) { return h / (1.0f + std::exp(-h)); }

}  // namespace

int default_threads() {
  const unsigned n = std::thread::hardware_concurrency();
  return n == 0 ? 1 : static_cast<int>(n);
}

void expert_ffn(moe_shape s, const uint8_t* host_pool, size_t blob_bytes, const std::vector<HostPairs>& experts,
                const float* x, int T, float* out, int threads) {
  const BlobLayout L = blob_layout(s.fmt, s.d, s.I);
  const bool avx = have_avx2();
  const bool mx_fast = avx && s.fmt == MOE_W_MXFP4 && mx_tiled(s.d, s.I);
  const int n_e = static_cast<int>(experts.size());
  constexpr int CH = 64;                                   // rows per task
  // a[e][pair][I]
  std::vector<size_t> a_off(n_e + 1, 0);
  for (int e = 0; e < n_e; ++e) a_off[e + 1] = a_off[e] + experts[e].tok.size() * static_cast<size_t>(s.I);
  std::vector<float> a(a_off[n_e]);

  auto rows_of = [&](const uint8_t* blob) {
    Rows R{s, L, {1.f, 1.f, 1.f}};
    if (s.fmt == MOE_W_NVFP4) std::memcpy(R.ts, blob + L.ts, sizeof(R.ts));
    return R;
  };
  auto decode = [&](const Rows& R, const uint8_t* blob, Mat m, int r, float* dst) {
    if (mx_fast) {
      const int K = m == DOWN ? s.I : s.d;
      decode_mx_tiled_avx2(blob + (m == DOWN ? L.wd : L.wg), m == DOWN ? r : gu_row(r, m == UP), K, dst);
    } else {
      R.decode(blob, m, r, dst);
    }
  };
  auto dot = [&](const float* w, const float* v, int K) { return avx ? dot_avx2(w, v, K) : dot_scalar(w, v, K); };

  // pass 1: a = silu(W_g x) * (W_u x) for every pair of every host expert
  const int chunks1 = (s.I + CH - 1) / CH;
  Pool::get().run(n_e * chunks1, threads, [&](int task) {
    const int e = task / chunks1, c0 = (task % chunks1) * CH;
    const HostPairs& P = experts[e];
    const uint8_t* blob = host_pool + static_cast<size_t>(P.expert) * blob_bytes;
    const Rows R = rows_of(blob);
    std::vector<float> wg(s.d), wu(s.d);
    for (int i = c0; i < std::min(s.I, c0 + CH); ++i) {
      decode(R, blob, GATE, i, wg.data());
      decode(R, blob, UP, i, wu.data());
      for (size_t p = 0; p < P.tok.size(); ++p) {
        const float* xv = x + static_cast<size_t>(P.tok[p]) * s.d;
        const float h = dot(wg.data(), xv, s.d), u = dot(wu.data(), xv, s.d);
        a[a_off[e] + p * s.I + i] = silu(h) * u;
      }
    }
  });
  // pass 2: out[t][c] = sum over host pairs of gate * (W_d a)[c]
  const int chunks2 = (s.d + CH - 1) / CH;
  Pool::get().run(chunks2, threads, [&](int task) {
    const int c0 = task * CH, c1 = std::min(s.d, c0 + CH);
    for (int t = 0; t < T; ++t)
      for (int c = c0; c < c1; ++c) out[static_cast<size_t>(t) * s.d + c] = 0.f;
    std::vector<float> wd(s.I);
    for (int e = 0; e < n_e; ++e) {
      const HostPairs& P = experts[e];
      const uint8_t* blob = host_pool + static_cast<size_t>(P.expert) * blob_bytes;
      const Rows R = rows_of(blob);
      for (int c = c0; c < c1; ++c) {
        decode(R, blob, DOWN, c, wd.data());
        for (size_t p = 0; p < P.tok.size(); ++p)
          out[static_cast<size_t>(P.tok[p]) * s.d + c] += P.gate[p] * dot(wd.data(), a.data() + a_off[e] + p * s.I, s.I);
      }
    }
  });
}

}  // namespace host
}  // namespace moe
