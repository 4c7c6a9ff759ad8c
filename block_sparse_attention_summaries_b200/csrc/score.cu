// Decode block scoring: s_c = q . kbar_c / sqrt(d) (+ the FreeSolo erf distance bias).
//
// [SAS] review, "Background" Eq. 3 and "Decoding efficiency" (Fig. 7c): every decode step scores
// the summary of every history block, the part of the step that grows with the context.
// [FreeSolo] summary page, "How it works": the cell score
//     r_ic = q_i . kbar_c / sqrt(d) + lambda_h * a_c * erf((i - p_c) / (2 sigma_h)).
//
// Warp-level GEMV bound by HBM: the G query heads of one kv group share every summary row, so a
// row is read once for all of them.  A warp takes R = 32/G rows at a time, each lane holding d/32
// elements of the row and of the G queries; the R*G = 32 partial dot products are finished with
// one 31-shuffle transpose-reduce, after which lane l owns (row l/G, head l%G).
#include "bsa_common.cuh"

namespace bsa {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;

template <typename T, int D, int G>
__global__ void __launch_bounds__(kThreads)
    score_decode_kernel(const T* __restrict__ q, int Hq, int Hk, int n, int b, int C,
                        const int* __restrict__ seq_lens, const float* __restrict__ mean_k,
                        const float* __restrict__ max_norm, const float* __restrict__ centre,
                        const float* __restrict__ lam, const float* __restrict__ sig,
                        int prefix_block, int rows_per_cta, float* __restrict__ scores,
                        int* __restrict__ n_cand) {
  constexpr int EPL = D / 32;  // elements of a row per lane
  constexpr int R = 32 / G;    // rows per warp step
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int kh = blockIdx.y;
  const int bi = blockIdx.z;
  const int L = seq_lens ? min(seq_lens[bi], n) : n;
  const int pos = L - 1;
  int nc = prefix_block > 0 ? ((pos / prefix_block) * prefix_block) / b : pos / b;
  nc = min(nc, C);

  const float scale = rsqrtf((float)D);
  float qv[G][EPL];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const T* qp = q + ((size_t)bi * Hq + kh * G + g) * D + lane * EPL;
    float tmp[EPL];
    load_vec<T, EPL>(qp, tmp);
#pragma unroll
    for (int e = 0; e < EPL; ++e) qv[g][e] = tmp[e];
  }

  const int c_begin = blockIdx.x * rows_per_cta;
  const int c_end = min(C, c_begin + rows_per_cta);
  const float* mk = mean_k + (size_t)(bi * Hk + kh) * C * D;

  // my (row, head) after the transpose-reduce
  const int my_r = lane / G;
  const int my_g = lane % G;
  const int h = kh * G + my_g;
  const float lam_h = lam ? lam[h] : 0.f;
  const float inv2sig = lam ? 0.5f / sig[h] : 0.f;
  float* srow = scores + ((size_t)bi * Hq + h) * C;

  for (int c0 = c_begin + warp * R; c0 < c_end; c0 += kWarps * R) {
    float a[32];
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const int c = c0 + r;
      float x[EPL];
      if (c < nc) {
        load_vec<float, EPL>(mk + (size_t)c * D + lane * EPL, x);
      } else {
#pragma unroll
        for (int e = 0; e < EPL; ++e) x[e] = 0.f;
      }
#pragma unroll
      for (int g = 0; g < G; ++g) {
        float s = 0.f;
#pragma unroll
        for (int e = 0; e < EPL; ++e) s = fmaf(qv[g][e], x[e], s);
        a[r * G + g] = s;
      }
    }
    warp_transpose_reduce32(a, lane);
    const int c = c0 + my_r;
    if (c < c_end) {
      float s;
      if (c < nc) {
        s = a[0] * scale;
        if (lam) {
          const size_t row = (size_t)(bi * Hk + kh) * C + c;
          s += lam_h * max_norm[row] * erff(((float)pos - centre[row]) * inv2sig);
        }
      } else {
        s = -INFINITY;
      }
      srow[c] = s;
    }
  }
  if (n_cand && blockIdx.x == 0 && threadIdx.x < G) n_cand[(size_t)bi * Hq + kh * G + threadIdx.x] = nc;
}

template <typename T, int D>
bsa_status dispatch_g(int G, dim3 grid, const void* q, int Hq, int Hk, int n, int b, int C,
                      const int* seq_lens, const float* mean_k, const float* max_norm,
                      const float* centre, const float* lam, const float* sig, int prefix_block,
                      int rows_per_cta, float* scores, int* n_cand, cudaStream_t st) {
  const T* qq = static_cast<const T*>(q);
#define BSA_SCORE_LAUNCH(GG)                                                                   \
  score_decode_kernel<T, D, GG><<<grid, kThreads, 0, st>>>(qq, Hq, Hk, n, b, C, seq_lens,      \
                                                           mean_k, max_norm, centre, lam, sig, \
                                                           prefix_block, rows_per_cta, scores, \
                                                           n_cand)
  switch (G) {
    case 1: BSA_SCORE_LAUNCH(1); break;
    case 2: BSA_SCORE_LAUNCH(2); break;
    case 4: BSA_SCORE_LAUNCH(4); break;
    case 8: BSA_SCORE_LAUNCH(8); break;
    default: return BSA_ERR_UNSUPPORTED;
  }
#undef BSA_SCORE_LAUNCH
  return BSA_OK;
}

}  // namespace
}  // namespace bsa

extern "C" bsa_status bsa_score_blocks(const void* q, bsa_dtype dt, int B, int Hq, int Hk, int n,
                                       int d, int b, const int* seq_lens, const float* mean_k,
                                       const float* max_norm, const float* centre,
                                       const float* lambda_h, const float* sigma_h,
                                       int prefix_block, float* scores, int* n_cand,
                                       void* stream) {
  using namespace bsa;
  BSA_REQUIRE(dtype_ok(dt), BSA_ERR_DTYPE);
  BSA_REQUIRE(q && mean_k && scores, BSA_ERR_ARG);
  BSA_REQUIRE(B > 0 && Hq > 0 && Hk > 0 && n > 0 && d > 0 && b > 0 && prefix_block >= 0,
              BSA_ERR_ARG);
  BSA_REQUIRE((lambda_h == nullptr) == (sigma_h == nullptr), BSA_ERR_ARG);
  BSA_REQUIRE(!lambda_h || (max_norm && centre), BSA_ERR_ARG);
  BSA_REQUIRE(Hq % Hk == 0, BSA_ERR_SHAPE);
  BSA_REQUIRE(group_ok(Hq, Hk), BSA_ERR_UNSUPPORTED);
  BSA_REQUIRE(head_dim_ok(d), BSA_ERR_UNSUPPORTED);
  BSA_REQUIRE(Hk <= 65535 && B <= 65535, BSA_ERR_UNSUPPORTED);
  BSA_REQUIRE(all_aligned16(q, mean_k), BSA_ERR_ARG);
  const int C = ceil_div(n, b);
  const int G = Hq / Hk;
  const int R = 32 / G;
  // about four CTAs per SM in total, each a whole number of warp steps
  const long long total_rows = (long long)C * B * Hk;
  int rows = (int)((total_rows + 4LL * kSMs - 1) / (4LL * kSMs));
  const int step = kWarps * R;
  rows = std::max(step, ceil_div(rows, step) * step);
  dim3 grid(ceil_div(C, rows), Hk, B);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  bsa_status rc;
  if (dt == BSA_BF16)
    rc = d == 64 ? dispatch_g<__nv_bfloat16, 64>(G, grid, q, Hq, Hk, n, b, C, seq_lens, mean_k,
                                                 max_norm, centre, lambda_h, sigma_h,
                                                 prefix_block, rows, scores, n_cand, st)
                 : dispatch_g<__nv_bfloat16, 128>(G, grid, q, Hq, Hk, n, b, C, seq_lens, mean_k,
                                                  max_norm, centre, lambda_h, sigma_h,
                                                  prefix_block, rows, scores, n_cand, st);
  else
    rc = d == 64 ? dispatch_g<float, 64>(G, grid, q, Hq, Hk, n, b, C, seq_lens, mean_k, max_norm,
                                         centre, lambda_h, sigma_h, prefix_block, rows, scores,
                                         n_cand, st)
                 : dispatch_g<float, 128>(G, grid, q, Hq, Hk, n, b, C, seq_lens, mean_k,
                                          max_norm, centre, lambda_h, sigma_h, prefix_block,
                                          rows, scores, n_cand, st);
  if (rc != BSA_OK) return rc;
  BSA_LAUNCH_CHECK();
  return BSA_OK;
}
