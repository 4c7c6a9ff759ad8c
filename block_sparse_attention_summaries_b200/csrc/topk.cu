// Top-K block selection with lower-index tie-break.
//
// [SAS] review, "Background" Eq. 3 (I = Top-K(s, K)) and the worked example, step 3; "Decoding
// efficiency" (Fig. 7c) names sorting every candidate block the real decode bottleneck at long
// context.  Nothing here sorts: one CTA per row runs an exact radix select on order-preserving
// 32-bit keys (four 8-bit digit passes over a shared histogram) to find the K-th largest key T and
// how many keys equal to T are still needed, then one block-wide prefix scan in index order emits
// the selected indices already ascending: every key above T, then the lowest-indexed keys equal
// to T.  That is exactly "larger score first, lower index first among equal scores".
#include "bsa_common.cuh"

namespace bsa {
namespace {

// Order-preserving key: larger float -> larger key; -0.0 == +0.0; NaN -> 0 (below -inf).
__device__ __forceinline__ uint32_t float_key(float f) {
  if (f != f) return 0u;
  if (f == 0.f) f = 0.f;
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

template <int THREADS>
__device__ __forceinline__ int block_exclusive_scan(int x, int* warp_tot, int& total) {
  constexpr int NW = THREADS / 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = x;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  int before = 0, tot = 0;
#pragma unroll
  for (int w = 0; w < NW; ++w) {
    const int t = warp_tot[w];
    before += (w < warp) ? t : 0;
    tot += t;
  }
  __syncthreads();
  total = tot;
  return before + incl - x;
}

template <int THREADS, int ITEMS>
__global__ void __launch_bounds__(THREADS)
    topk_kernel(const float* __restrict__ scores, int C, int ld, const int* __restrict__ n_cand,
                int units, int q_block, int b, int K, int* __restrict__ idx,
                int* __restrict__ count, int out_ld, int keep_newest) {
  __shared__ uint32_t hist[256];
  __shared__ int warp_tot[THREADS / 32];
  __shared__ uint32_t s_digit;
  __shared__ int s_above;

  const int row = blockIdx.x;
  const int tid = threadIdx.x;
  int nc;
  if (n_cand)
    nc = n_cand[row];
  else if (units > 0)
    nc = ((row % units) * q_block) / b;
  else
    nc = C;
  nc = max(0, min(nc, C));
  // the keep_newest newest candidates are kept outright (FS-L) and follow the K selected among
  // the older ones; their indices are all larger, so the row stays ascending
  const int newest = min(keep_newest, nc);
  nc -= newest;
  // K < 0: the upper half of the candidates, ceil(nc / 2) (FS-B's high-norm cells)
  const int kk = K < 0 ? (nc + 1) / 2 : min(K, nc);
  int* out = idx + (size_t)row * out_ld;
  if (count && tid == 0) count[row] = kk + newest;
  for (int j = kk + tid; j < out_ld; j += THREADS) out[j] = j - kk < newest ? nc + (j - kk) : -1;

  if (kk == nc) {  // every candidate is selected (includes nc == 0)
    for (int j = tid; j < kk; j += THREADS) out[j] = j;
    return;
  }

  const float* srow = scores + (size_t)row * ld;
  const int i0 = tid * ITEMS;
  uint32_t key[ITEMS];
#pragma unroll
  for (int e = 0; e < ITEMS; ++e) {
    const int i = i0 + e;
    key[e] = i < nc ? float_key(srow[i]) : 0u;
  }

  uint32_t prefix = 0, mask = 0;
  int rem = kk;
#pragma unroll 1
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int j = tid; j < 256; j += THREADS) hist[j] = 0;
    __syncthreads();
#pragma unroll
    for (int e = 0; e < ITEMS; ++e)
      if (i0 + e < nc && (key[e] & mask) == prefix) atomicAdd(&hist[(key[e] >> shift) & 255u], 1u);
    __syncthreads();
    if (tid < 32) {
      uint32_t hb[8];
      uint32_t local = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        hb[j] = hist[tid * 8 + j];
        local += hb[j];
      }
      // exclusive suffix sum over lanes: keys in bins above this lane's bins
      uint32_t incl = local;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        uint32_t y = __shfl_down_sync(0xffffffffu, incl, o);
        if (tid + o < 32) incl += y;
      }
      uint32_t running = incl - local;
#pragma unroll
      for (int j = 7; j >= 0; --j) {
        if (running < (uint32_t)rem && running + hb[j] >= (uint32_t)rem) {
          s_digit = (uint32_t)(tid * 8 + j);
          s_above = (int)running;
        }
        running += hb[j];
      }
    }
    __syncthreads();
    prefix |= s_digit << shift;
    mask |= 255u << shift;
    rem -= s_above;
    __syncthreads();
  }
  const uint32_t T = prefix;  // the K-th largest key; `rem` keys equal to T are still needed

  int eq = 0;
#pragma unroll
  for (int e = 0; e < ITEMS; ++e) eq += (i0 + e < nc && key[e] == T);
  int tot;
  int eq_before = block_exclusive_scan<THREADS>(eq, warp_tot, tot);
  int sel = 0;
  {
    int r = eq_before;
#pragma unroll
    for (int e = 0; e < ITEMS; ++e) {
      if (i0 + e >= nc) continue;
      if (key[e] > T) {
        ++sel;
      } else if (key[e] == T) {
        sel += (r < rem);
        ++r;
      }
    }
  }
  int pos = block_exclusive_scan<THREADS>(sel, warp_tot, tot);
  {
    int r = eq_before;
#pragma unroll
    for (int e = 0; e < ITEMS; ++e) {
      if (i0 + e >= nc) continue;
      bool take = false;
      if (key[e] > T) {
        take = true;
      } else if (key[e] == T) {
        take = r < rem;
        ++r;
      }
      if (take) out[pos++] = i0 + e;
    }
  }
}

}  // namespace
}  // namespace bsa

namespace bsa {
void launch_topk_rows(const float* scores, int rows, int C, int ld, const int* n_cand, int units,
                      int q_block, int b, int K, int* idx, int* count, int out_ld,
                      int keep_newest, cudaStream_t st) {
  if (C <= 256)
    topk_kernel<256, 1><<<rows, 256, 0, st>>>(scores, C, ld, n_cand, units, q_block, b, K, idx,
                                              count, out_ld, keep_newest);
  else if (C <= 1024)
    topk_kernel<256, 4><<<rows, 256, 0, st>>>(scores, C, ld, n_cand, units, q_block, b, K, idx,
                                              count, out_ld, keep_newest);
  else if (C <= 4096)
    topk_kernel<512, 8><<<rows, 512, 0, st>>>(scores, C, ld, n_cand, units, q_block, b, K, idx,
                                              count, out_ld, keep_newest);
  else
    topk_kernel<1024, 16><<<rows, 1024, 0, st>>>(scores, C, ld, n_cand, units, q_block, b, K, idx,
                                                 count, out_ld, keep_newest);
}
}  // namespace bsa

extern "C" bsa_status bsa_topk_blocks(const float* scores, int rows, int C, int ld,
                                      const int* n_cand, int units, int q_block, int b, int K,
                                      int* idx, int* count, void* stream) {
  using namespace bsa;
  BSA_REQUIRE(scores && idx, BSA_ERR_ARG);
  BSA_REQUIRE(rows >= 0 && C >= 0 && K > 0 && ld >= C && units >= 0, BSA_ERR_ARG);
  BSA_REQUIRE(units == 0 || n_cand || (q_block > 0 && b > 0), BSA_ERR_ARG);
  BSA_REQUIRE(C <= 16384 && K <= 256, BSA_ERR_UNSUPPORTED);
  if (rows == 0) return BSA_OK;
  launch_topk_rows(scores, rows, C, ld, n_cand, units, q_block, b, K, idx, count, K, 0,
                   static_cast<cudaStream_t>(stream));
  BSA_LAUNCH_CHECK();
  return BSA_OK;
}
