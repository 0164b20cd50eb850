// The q split of a decode step's cache misses.  A missed expert either is
// copied over PCIe into the GPU cache and runs there, or runs on the host
// against its host-resident weights; the two partial sums merge exactly
// (explainx.ai hardware guide, "Decode: decide whether to move an expert or
// compute where it lives"; futuresignalnews.com article, "Bandwidth-Adaptive
// Execution (The q* Policy)").  The pages name the policy -- q*, from the
// profiled PCIe and host-memory bandwidths, so that both paths run at once --
// but print no formula.  Reading: every miss moves one blob of B bytes, either
// over PCIe (a fill) or through host memory (host compute), so the two paths
// finish together when n_fill * B / bw_pcie = (m - n_fill) * B / bw_host,
// i.e. n_fill = m * bw_pcie / (bw_pcie + bw_host), rounded half up.  The
// misses with the most routed tokens are the ones filled (ties: lower id), so
// the host runs the experts with the least work.
#include <algorithm>
#include <cmath>
#include <vector>

#include "common.cuh"

using namespace moe;

extern "C" moe_status moe_split_misses(const int32_t* misses, int m, const int32_t* tokens_per_expert, int E,
                                       double q, double bw_pcie, double bw_host, int32_t* filled,
                                       int32_t* n_filled, int32_t* host, int32_t* n_host) {
  clear_error();
  MOE_REQUIRE(E >= 1 && E <= 1024, "E=%d outside [1, 1024]", E);
  MOE_REQUIRE(m >= 0 && m <= E, "m=%d outside [0, E=%d]", m, E);
  MOE_REQUIRE(n_filled != nullptr && n_host != nullptr, "null count");
  MOE_REQUIRE(m == 0 || (misses && tokens_per_expert && filled && host), "null pointer");
  double share;
  if (q < 0) {
    MOE_REQUIRE(std::isfinite(bw_pcie) && std::isfinite(bw_host) && bw_pcie > 0 && bw_host > 0,
                "q < 0 selects q*: bw_pcie and bw_host must be positive (got %g, %g)", bw_pcie, bw_host);
    share = m * bw_pcie / (bw_pcie + bw_host);
  } else {
    MOE_REQUIRE(q <= 1, "q=%g outside [0, 1]", q);
    share = q * m;
  }
  std::vector<char> seen(E, 0);
  std::vector<int32_t> ranked(misses, misses + m);
  for (int32_t e : ranked) {
    MOE_REQUIRE(e >= 0 && e < E, "expert id %d outside [0, %d)", e, E);
    MOE_REQUIRE(!seen[e], "expert %d listed twice", e);
    seen[e] = 1;
  }
  const int n_fill = std::max(0, std::min(m, static_cast<int>(std::floor(share + 0.5))));
  std::sort(ranked.begin(), ranked.end(), [&](int32_t a, int32_t b) {
    return tokens_per_expert[a] != tokens_per_expert[b] ? tokens_per_expert[a] > tokens_per_expert[b] : a < b;
  });
  std::sort(ranked.begin(), ranked.begin() + n_fill);
  std::sort(ranked.begin() + n_fill, ranked.end());
  std::copy(ranked.begin(), ranked.begin() + n_fill, filled);
  std::copy(ranked.begin() + n_fill, ranked.end(), host);
  *n_filled = n_fill;
  *n_host = m - n_fill;
  return MOE_OK;
}
