// Gradient of the loss with respect to the selector scores, through the log-softmax gate.
//
// [SAS] review, "Why the four design choices matter": the gate of a selected history block is
// log g_m = s_m - LSE(s), the LSE running over the normaliser set N (all history blocks of the
// row, or only its selected ones).  With dg_m = dL/dg_m from the gate gradient,
//     ds_c = [c in S] g_c dg_c - pi_c * A,   A = sum_{m in S} g_m dg_m,   pi = softmax_N(s),
// and pi_c = 0 outside N.  One warp per row: the LSE over N, the K gates and A by warp
// reductions, then one pass that writes ds over the row's history blocks (0 beyond them).
#include "bsa_common.cuh"

namespace bsa {
namespace {

constexpr int kRowsPerBlock = 8;  // one warp per row

__global__ void __launch_bounds__(32 * kRowsPerBlock)
    selector_grad_kernel(const float* __restrict__ scores, int scores_ld,
                         const int* __restrict__ n_cand, const int* __restrict__ idx,
                         const int* __restrict__ count, int K, const float* __restrict__ dg,
                         int all_history, int rows, float* __restrict__ ds, int ds_ld) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long r = (long long)blockIdx.x * kRowsPerBlock + warp;
  if (r >= rows) return;
  const float* s = scores + r * scores_ld;
  const int nc = min(max(n_cand[r], 0), min(scores_ld, ds_ld));
  const int cnt = count ? min(count[r], K) : K;
  // lane k < K holds slot k: its block (or -1) and dg
  int m = -1;
  float dgk = 0.f;
  for (int k = lane; k < K; k += 32) {  // K <= 32 is checked on the host: one slot per lane
    const int x = k < cnt ? idx[r * K + k] : -1;
    if (x >= 0 && x < nc) {
      m = x;
      dgk = dg[r * K + k];
    }
  }
  const float sm = m >= 0 ? s[m] : -INFINITY;
  // LSE over the normaliser set
  float mx = -INFINITY;
  if (all_history) {
    for (int c = lane; c < nc; c += 32) mx = fmaxf(mx, s[c]);
  } else {
    mx = sm;
  }
  mx = warp_max(mx);
  float acc = 0.f;
  if (mx != -INFINITY) {
    if (all_history) {
      for (int c = lane; c < nc; c += 32) acc += expf(s[c] - mx);
    } else if (m >= 0) {
      acc = expf(sm - mx);
    }
  }
  acc = warp_sum(acc);
  const float L = mx == -INFINITY ? 0.f : mx + logf(acc);
  const float gk = m >= 0 ? expf(sm - L) : 0.f;
  const float A = warp_sum(gk * dgk);
  float* out = ds + r * ds_ld;
  for (int c = lane; c < ds_ld; c += 32) {
    float v = 0.f;
    if (c < nc && all_history) v = -expf(s[c] - L) * A;
    out[c] = v;
  }
  __syncwarp();
  if (m >= 0) out[m] += gk * dgk - (all_history ? 0.f : gk * A);
}

}  // namespace
}  // namespace bsa

extern "C" bsa_status bsa_selector_grad(const float* scores, int scores_ld, const int* n_cand,
                                        const int* idx, const int* count, int K, const float* dg,
                                        bsa_gate_norm norm, int rows, float* ds, int ds_ld,
                                        void* stream) {
  using namespace bsa;
  BSA_REQUIRE(scores && n_cand && idx && dg && ds, BSA_ERR_ARG);
  BSA_REQUIRE(rows > 0 && K > 0 && scores_ld > 0 && ds_ld > 0, BSA_ERR_ARG);
  BSA_REQUIRE(norm == BSA_NORM_SELECTED || norm == BSA_NORM_ALL_HISTORY, BSA_ERR_ARG);
  BSA_REQUIRE(K <= 32, BSA_ERR_UNSUPPORTED);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const unsigned grid = (unsigned)((rows + kRowsPerBlock - 1) / kRowsPerBlock);
  selector_grad_kernel<<<grid, 32 * kRowsPerBlock, 0, st>>>(
      scores, scores_ld, n_cand, idx, count, K, dg, norm == BSA_NORM_ALL_HISTORY ? 1 : 0, rows,
      ds, ds_ld);
  BSA_LAUNCH_CHECK();
  return BSA_OK;
}
