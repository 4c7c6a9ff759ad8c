// FS-L: pre-query pruning of the FreeSolo cells and selection over the kept cells (decode).
//
// [FreeSolo] "How it differs", FS-L variant: before any query arrives each head keeps its W most
// recent cells and the P cells of largest maximum key norm; a query then scores only the kept
// cells with the full method's cell score
//     r_c = q . kbar_c / sqrt(d) + lambda_h a_c erf((i - p_c) / (2 sigma_h))
// and reads its K best, so the per-query cost is O(W + P) instead of O(C).
//   * Pruning: the radix select of the Top-K call over the maximum key norms of the older cells,
//     with the W newest kept outright and written after them (one CTA per (batch, head)).
//   * Selection: one warp per (batch, head) decode query; lane l scores kept cells l, l + 32, ...
//     by itself (q staged in shared memory and read as broadcasts, the cell's mean key as 16-byte
//     loads, all of them in flight at once), then an exact rank count for the top K (ties to the
//     lower cell index, NaN last).
#include "bsa_common.cuh"

namespace bsa {

void launch_topk_rows(const float* scores, int rows, int C, int ld, const int* n_cand, int units,
                      int q_block, int b, int K, int* idx, int* count, int out_ld,
                      int keep_newest, cudaStream_t st);

namespace {

constexpr int kMaxKept = 128;  // W + P
constexpr int kRowsPerCta = 4;

__device__ __forceinline__ uint32_t fsl_key(float f) {
  if (f != f) return 0u;
  if (f == 0.f) f = 0.f;
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

template <typename T, int D>
__global__ void __launch_bounds__(32 * kRowsPerCta)
    fsl_select_kernel(const T* __restrict__ q, int B, int H, const int* __restrict__ pos,
                      const float* __restrict__ mean_k, const float* __restrict__ max_norm,
                      const float* __restrict__ centre, int C, const float* __restrict__ lam,
                      const float* __restrict__ sig, const int* __restrict__ cand,
                      const int* __restrict__ cand_count, int cand_ld, int K,
                      int* __restrict__ idx, int* __restrict__ count) {
  __shared__ uint32_t s_key[kRowsPerCta][kMaxKept];
  __shared__ __align__(16) float s_q[kRowsPerCta][D];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * kRowsPerCta + warp;  // (batch, head)
  if (row >= B * H) return;
  const int bi = row / H, h = row % H;
  const int i = pos[bi];
  const int nk = min(max(cand_count[row], 0), min(cand_ld, kMaxKept));
  for (int e = lane; e < D; e += 32) s_q[warp][e] = Elem<T>::to_f(q[(size_t)row * D + e]);
  __syncwarp();
  const float scale = rsqrtf((float)D);
  const float lm = lam ? lam[h] : 0.f;
  const float inv2s = lam ? 0.5f / sig[h] : 0.f;
  const int* crow = cand + (size_t)row * cand_ld;
  const size_t srow = (size_t)row * C;
  uint32_t* keys = s_key[warp];
  const float4* qs = reinterpret_cast<const float4*>(s_q[warp]);
#pragma unroll
  for (int t = 0; t < kMaxKept / 32; ++t) {
    const int j = lane + 32 * t;
    if (j < nk) {
      const int c = crow[j];
      const float4* kp = reinterpret_cast<const float4*>(mean_k + (srow + c) * D);
      float a0 = 0.f, a1 = 0.f;
#pragma unroll
      for (int e4 = 0; e4 < D / 4; ++e4) {
        const float4 kv = kp[e4], qv = qs[e4];
        a0 = fmaf(qv.x, kv.x, fmaf(qv.y, kv.y, a0));
        a1 = fmaf(qv.z, kv.z, fmaf(qv.w, kv.w, a1));
      }
      float r = (a0 + a1) * scale;
      if (lam) r += lm * max_norm[srow + c] * erff(((float)i - centre[srow + c]) * inv2s);
      keys[j] = fsl_key(r);
    }
  }
  __syncwarp();
  // exact top K by rank counting over <= 128 keys (4 per lane); ties to the lower kept slot,
  // which is the lower cell index because the kept list is ascending
  const int kk = min(K, nk);
  uint32_t mk[4];
  int rk[4];
#pragma unroll
  for (int t = 0; t < 4; ++t) {
    mk[t] = lane + 32 * t < nk ? keys[lane + 32 * t] : 0u;
    rk[t] = 0;
  }
  for (int j = 0; j < nk; ++j) {
    const uint32_t kj = keys[j];
#pragma unroll
    for (int t = 0; t < 4; ++t) rk[t] += (kj > mk[t] || (kj == mk[t] && j < lane + 32 * t)) ? 1 : 0;
  }
  int* out = idx + (size_t)row * K;
  const unsigned lt = (1u << lane) - 1u;
  int taken = 0;
#pragma unroll
  for (int t = 0; t < 4; ++t) {
    const bool take = lane + 32 * t < nk && rk[t] < kk;
    const unsigned tb = __ballot_sync(0xffffffffu, take);
    if (take) out[taken + __popc(tb & lt)] = crow[lane + 32 * t];
    taken += __popc(tb);
  }
  for (int j = kk + lane; j < K; j += 32) out[j] = -1;
  if (count && lane == 0) count[row] = kk;
}

}  // namespace
}  // namespace bsa

extern "C" bsa_status bsa_fsl_prune(const float* max_norm, int rows, int C, const int* n_cells,
                                    int W, int P, int* cand, int* cand_count, void* stream) {
  using namespace bsa;
  BSA_REQUIRE(max_norm && n_cells && cand, BSA_ERR_ARG);
  BSA_REQUIRE(rows >= 0 && C >= 0 && W >= 0 && P > 0, BSA_ERR_ARG);
  BSA_REQUIRE(C <= 16384 && P <= 256 && W + P <= kMaxKept, BSA_ERR_UNSUPPORTED);
  if (rows == 0) return BSA_OK;
  launch_topk_rows(max_norm, rows, C, C, n_cells, 0, 0, 0, P, cand, cand_count, W + P, W,
                   static_cast<cudaStream_t>(stream));
  BSA_LAUNCH_CHECK();
  return BSA_OK;
}

extern "C" bsa_status bsa_fsl_select(const void* q, bsa_dtype dt, int B, int H, int d,
                                     const int* pos, const float* mean_k, const float* max_norm,
                                     const float* centre, int C, const float* lambda_h,
                                     const float* sigma_h, const int* cand,
                                     const int* cand_count, int cand_ld, int K, int* idx,
                                     int* count, void* stream) {
  using namespace bsa;
  BSA_REQUIRE(dtype_ok(dt), BSA_ERR_DTYPE);
  BSA_REQUIRE(q && pos && mean_k && cand && cand_count && idx, BSA_ERR_ARG);
  BSA_REQUIRE((lambda_h == nullptr) == (sigma_h == nullptr), BSA_ERR_ARG);
  BSA_REQUIRE(!lambda_h || (max_norm && centre), BSA_ERR_ARG);
  BSA_REQUIRE(B > 0 && H > 0 && C >= 0 && cand_ld > 0 && K > 0, BSA_ERR_ARG);
  BSA_REQUIRE(head_dim_ok(d), BSA_ERR_UNSUPPORTED);
  BSA_REQUIRE(cand_ld <= kMaxKept, BSA_ERR_UNSUPPORTED);
  BSA_REQUIRE(all_aligned16(q, mean_k), BSA_ERR_ARG);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int rows = B * H;
  const unsigned grid = (unsigned)((rows + kRowsPerCta - 1) / kRowsPerCta);
  if (dt == BSA_BF16) {
    if (d == 64)
      fsl_select_kernel<__nv_bfloat16, 64><<<grid, 32 * kRowsPerCta, 0, st>>>(
          static_cast<const __nv_bfloat16*>(q), B, H, pos, mean_k, max_norm, centre, C,
          lambda_h, sigma_h, cand, cand_count, cand_ld, K, idx, count);
    else
      fsl_select_kernel<__nv_bfloat16, 128><<<grid, 32 * kRowsPerCta, 0, st>>>(
          static_cast<const __nv_bfloat16*>(q), B, H, pos, mean_k, max_norm, centre, C,
          lambda_h, sigma_h, cand, cand_count, cand_ld, K, idx, count);
  } else {
    if (d == 64)
      fsl_select_kernel<float, 64><<<grid, 32 * kRowsPerCta, 0, st>>>(
          static_cast<const float*>(q), B, H, pos, mean_k, max_norm, centre, C, lambda_h,
          sigma_h, cand, cand_count, cand_ld, K, idx, count);
    else
      fsl_select_kernel<float, 128><<<grid, 32 * kRowsPerCta, 0, st>>>(
          static_cast<const float*>(q), B, H, pos, mean_k, max_norm, centre, C, lambda_h,
          sigma_h, cand, cand_count, cand_ld, K, idx, count);
  }
  BSA_LAUNCH_CHECK();
  return BSA_OK;
}
