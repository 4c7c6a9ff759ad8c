// Per-block key summaries: mean key, max key norm, centre position.
//
// [FreeSolo] summary page, "How it works": every cell of consecutive tokens keeps its mean key
// (the content used for routing), its centre position (for the relative-distance term) and the
// largest key norm inside it (a query-independent priority).  The same mean key is the pooled
// block summary a selector scores in [SAS] ("Limitations" of the review).
//
// HBM-bound reduction: one CTA per (batch, kv head, block) reads the block's b x d keys once with
// 16-byte vector loads (all loads of a thread issued before they are consumed) and writes d + 2
// floats.  Traffic per block = b*d*sizeof(T) read + (d+2)*4 written.
#include "bsa_common.cuh"

namespace bsa {
namespace {

constexpr int kThreads = 256;

template <typename T, int D>
__global__ void __launch_bounds__(kThreads)
    summaries_kernel(const T* __restrict__ k, int Hk, int n, int b, int C, int first_block,
                     const int* __restrict__ seq_lens, float* __restrict__ mean_k,
                     float* __restrict__ max_norm, float* __restrict__ centre) {
  constexpr int VEC = 16 / sizeof(T);  // elements per 16-byte load
  constexpr int VPR = D / VEC;         // threads covering one key row
  constexpr int RPP = kThreads / VPR;  // rows per pass
  constexpr int UNROLL = 4;
  static_assert(VPR <= 32 && 32 % VPR == 0, "row must map onto a power-of-two lane group");

  __shared__ float red[RPP][D];
  __shared__ float wmax[kThreads / 32];

  const int kh = blockIdx.y;
  const int bi = blockIdx.z;
  const int L = seq_lens ? min(seq_lens[bi], n) : n;
  // first_block < 0: the block holding this row's newest token (decode append)
  const int c = first_block >= 0 ? first_block + blockIdx.x : (L - 1) / b;
  const int lo = c * b;
  const int hi = min(lo + b, L);
  const int cnt = max(0, hi - lo);

  const int tid = threadIdx.x;
  const int vc = tid % VPR;
  const int r0 = tid / VPR;
  const T* base = k + ((size_t)(bi * Hk + kh) * n + lo) * D + vc * VEC;

  float sum[VEC];
#pragma unroll
  for (int e = 0; e < VEC; ++e) sum[e] = 0.f;
  float nmax = 0.f;

  // The trip count is uniform over the CTA so that every lane reaches the group shuffles.
  for (int base_row = 0; base_row < cnt; base_row += RPP * UNROLL) {
    float x[UNROLL][VEC];
#pragma unroll
    for (int u = 0; u < UNROLL; ++u) {
      const int rr = base_row + r0 + u * RPP;
      if (rr < cnt) {
        load_vec<T, VEC>(base + (size_t)rr * D, x[u]);
      } else {
#pragma unroll
        for (int e = 0; e < VEC; ++e) x[u][e] = 0.f;
      }
    }
#pragma unroll
    for (int u = 0; u < UNROLL; ++u) {
      float sq = 0.f;
#pragma unroll
      for (int e = 0; e < VEC; ++e) {
        sum[e] += x[u][e];
        sq = fmaf(x[u][e], x[u][e], sq);
      }
#pragma unroll
      for (int o = VPR / 2; o > 0; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
      nmax = fmaxf(nmax, sqrtf(sq));  // rows past cnt contribute 0, below every real norm
    }
  }

#pragma unroll
  for (int e = 0; e < VEC; ++e) red[r0][vc * VEC + e] = sum[e];
  nmax = warp_max(nmax);
  if ((tid & 31) == 0) wmax[tid >> 5] = nmax;
  __syncthreads();

  const size_t row = (size_t)(bi * Hk + kh) * C + c;
  for (int t = tid; t < D; t += kThreads) {
    float s = 0.f;
#pragma unroll 8
    for (int r = 0; r < RPP; ++r) s += red[r][t];
    mean_k[row * D + t] = cnt ? s / (float)cnt : 0.f;
  }
  if (tid == 0) {
    float m = 0.f;
#pragma unroll
    for (int w = 0; w < kThreads / 32; ++w) m = fmaxf(m, wmax[w]);
    if (max_norm) max_norm[row] = m;
    if (centre) {
      // mean of the positions lo .. hi-1 (of a full block when no token is valid)
      const int last = cnt ? hi - 1 : lo + b - 1;
      centre[row] = 0.5f * (float)lo + 0.5f * (float)last;
    }
  }
}

template <typename T, int D>
void launch(const void* k, int B, int Hk, int n, int b, int C, int first, int nblk,
            const int* seq_lens, float* mean_k, float* max_norm, float* centre,
            cudaStream_t st) {
  dim3 grid(nblk, Hk, B);
  summaries_kernel<T, D><<<grid, kThreads, 0, st>>>(static_cast<const T*>(k), Hk, n, b, C, first,
                                                    seq_lens, mean_k, max_norm, centre);
}

}  // namespace
}  // namespace bsa

extern "C" bsa_status bsa_build_block_summaries(const void* k, bsa_dtype dt, int B, int Hk,
                                                int n, int d, int b, const int* seq_lens,
                                                int first_block, int num_blocks, float* mean_k,
                                                float* max_norm, float* centre, void* stream) {
  using namespace bsa;
  BSA_REQUIRE(dtype_ok(dt), BSA_ERR_DTYPE);
  BSA_REQUIRE(k && mean_k, BSA_ERR_ARG);
  BSA_REQUIRE(B > 0 && Hk > 0 && n > 0 && d > 0 && b > 0, BSA_ERR_ARG);
  BSA_REQUIRE(Hk <= 65535 && B <= 65535, BSA_ERR_UNSUPPORTED);
  BSA_REQUIRE(head_dim_ok(d), BSA_ERR_UNSUPPORTED);
  BSA_REQUIRE(b <= 1024, BSA_ERR_UNSUPPORTED);
  BSA_REQUIRE(all_aligned16(k, mean_k), BSA_ERR_ARG);
  const int C = ceil_div(n, b);
  if (first_block < 0) {  // per-row current block
    first_block = -1;
    num_blocks = 1;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (dt == BSA_BF16) {
      if (d == 64) launch<__nv_bfloat16, 64>(k, B, Hk, n, b, C, -1, 1, seq_lens, mean_k, max_norm, centre, st);
      else launch<__nv_bfloat16, 128>(k, B, Hk, n, b, C, -1, 1, seq_lens, mean_k, max_norm, centre, st);
    } else {
      if (d == 64) launch<float, 64>(k, B, Hk, n, b, C, -1, 1, seq_lens, mean_k, max_norm, centre, st);
      else launch<float, 128>(k, B, Hk, n, b, C, -1, 1, seq_lens, mean_k, max_norm, centre, st);
    }
    BSA_LAUNCH_CHECK();
    return BSA_OK;
  }
  BSA_REQUIRE(first_block <= C, BSA_ERR_SHAPE);
  if (num_blocks < 0) num_blocks = C - first_block;
  BSA_REQUIRE(first_block + num_blocks <= C, BSA_ERR_SHAPE);
  if (num_blocks == 0) return BSA_OK;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (dt == BSA_BF16) {
    if (d == 64)
      launch<__nv_bfloat16, 64>(k, B, Hk, n, b, C, first_block, num_blocks, seq_lens, mean_k,
                                max_norm, centre, st);
    else
      launch<__nv_bfloat16, 128>(k, B, Hk, n, b, C, first_block, num_blocks, seq_lens, mean_k,
                                 max_norm, centre, st);
  } else {
    if (d == 64)
      launch<float, 64>(k, B, Hk, n, b, C, first_block, num_blocks, seq_lens, mean_k, max_norm,
                        centre, st);
    else
      launch<float, 128>(k, B, Hk, n, b, C, first_block, num_blocks, seq_lens, mean_k, max_norm,
                         centre, st);
  }
  BSA_LAUNCH_CHECK();
  return BSA_OK;
}

namespace bsa {
namespace {

// fp32 -> bf16 with round-to-nearest-even, four values per thread
__global__ void __launch_bounds__(256)
    round_bf16_kernel(const float* __restrict__ x, __nv_bfloat16* __restrict__ y, long long count) {
  const long long i = ((long long)blockIdx.x * blockDim.x + threadIdx.x) * 4;
  if (i + 4 <= count) {
    const float4 v = *reinterpret_cast<const float4*>(x + i);
    __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y), b = __floats2bfloat162_rn(v.z, v.w);
    *reinterpret_cast<uint2*>(y + i) =
        make_uint2(*reinterpret_cast<uint32_t*>(&a), *reinterpret_cast<uint32_t*>(&b));
  } else {
    for (long long j = i; j < count; ++j) y[j] = __float2bfloat16_rn(x[j]);
  }
}

}  // namespace
}  // namespace bsa

extern "C" bsa_status bsa_round_summaries_bf16(const float* mean_k, void* out, long long count,
                                               void* stream) {
  using namespace bsa;
  BSA_REQUIRE(mean_k && out && count >= 0, BSA_ERR_ARG);
  BSA_REQUIRE(all_aligned16(mean_k, out), BSA_ERR_ARG);
  if (count == 0) return BSA_OK;
  const long long threads = (count + 3) / 4;
  round_bf16_kernel<<<(unsigned)((threads + 255) / 256), 256, 0, static_cast<cudaStream_t>(stream)>>>(
      mean_k, static_cast<__nv_bfloat16*>(out), count);
  BSA_LAUNCH_CHECK();
  return BSA_OK;
}
