// FreeSolo long branch, cell-major on the tensor cores.
//
// [FreeSolo] summary page, "How it works": each query attends, with one softmax over raw
// (unrotated) q and k, to the tokens of the K cells it selected, and the result is mixed with the
// sliding-window branch, o = (1 - alpha_h) o_short + alpha_h o_long.
//
// Every query picks only K cells of `cell` tokens, but queries that pick the same cell share its
// keys.  So the work is regrouped by cell instead of by query:
//   1. fs_long_count_kernel: each valid (query, slot) pair takes a position in its cell's list
//      (warp-aggregated atomics: neighbouring queries tend to pick the same cells);
//   2. fs_long_offsets_kernel: each cell reserves a contiguous range of the pair list and one
//      tile per 128 of its pairs (a warp scan, then one atomic per warp on the two totals: the
//      order of the cells in the lists does not matter);
//   3. fs_long_scatter_kernel: pairs written in cell order;
//   4. fs_long_tile_kernel: per tile, the 128 queries' rows are gathered into shared memory
//      (cp.async, 128-byte swizzle), the cell's K and V arrive by TMA, S = Q K^T is one M = 128,
//      N = cell tcgen05 chain, a thread per row takes the softmax over the cell (max, exp2, sum),
//      and P V is a second chain; the normalised output row (bf16) and (max, sum) (fp32) go to
//      the pair's partial record;
//   5. fs_long_combine_kernel: a warp per query merges its partials (log-sum-exp) and mixes the
//      result into the short-branch output already in o.
// Only the selected (query, key) pairs are multiplied: no masked work, and no tile holds a query
// that did not select its cell (padding rows of a cell's last tile aside).  The partial outputs
// are stored in bf16 like P inside the MMA: one more rounding of at most 2^-9 relative before the
// fp32 merge, the same size as the final bf16 rounding of o.
#include <cudaTypedefs.h>

#include <map>
#include <mutex>

#include "tc_common.cuh"

namespace bsa {
namespace {

constexpr int kRowsL = 128;    // pairs per tile (tcgen05 M)
constexpr int kThreadsL = 128;
constexpr int kMaxKL = 8;      // slots per query

struct FsLongWs {
  int* ccount;     // [cells] pairs per cell
  int* cell_off;   // [cells] first pair of the cell in `pairs`
  int* ntiles;     // [2]: tiles, pairs reserved so far
  int4* tiles;     // [tile_cap] (global cell, first pair, pairs, 0)
  int* slotpos;    // [rows * K] position of the pair in its cell's list, -1 if not attended
  int* pairs;      // [rows * K] pair ids (row * K + slot) in cell order
  float2* part_ml; // [rows * K] (max of the scaled logits in log2 units, sum of exp2)
  __nv_bfloat16* part_o;  // [rows * K][d] output normalised by its sum
  long long tile_cap;
};

long long cells_of(int B, int H, int n, int cell) {
  return (long long)B * H * ((n + cell - 1) / cell);
}

size_t carve(const void* base, int B, int H, int n, int d, int cell, int K, FsLongWs* w) {
  const long long rows = (long long)B * H * n;
  const long long pairs = rows * K;
  const long long cells = cells_of(B, H, n, cell);
  const long long tile_cap = (pairs + kRowsL - 1) / kRowsL + cells + 1;
  uintptr_t p = align_up(reinterpret_cast<uintptr_t>(base), (uintptr_t)256);
  const uintptr_t p0 = p;
  auto take = [&](size_t bytes) {
    const uintptr_t r = p;
    p = align_up(p + bytes, (uintptr_t)256);
    return r;
  };
  FsLongWs t;
  t.ccount = reinterpret_cast<int*>(take((size_t)cells * 4));
  t.cell_off = reinterpret_cast<int*>(take((size_t)cells * 4));
  t.ntiles = reinterpret_cast<int*>(take(16));
  t.tiles = reinterpret_cast<int4*>(take((size_t)tile_cap * 16));
  t.slotpos = reinterpret_cast<int*>(take((size_t)pairs * 4));
  t.pairs = reinterpret_cast<int*>(take((size_t)pairs * 4));
  t.part_ml = reinterpret_cast<float2*>(take((size_t)pairs * 8));
  t.part_o = reinterpret_cast<__nv_bfloat16*>(take((size_t)pairs * d * 2));
  t.tile_cap = tile_cap;
  if (w) *w = t;
  return (size_t)(p - p0) + 256;
}

// ---- 1. positions of the attended (query, slot) pairs in their cells' lists -------------------
// A slot is attended when it holds a cell wholly at or before the query, not repeated by an
// earlier slot of the same query.
__global__ void __launch_bounds__(256)
    fs_long_count_kernel(const int* __restrict__ idx, const int* __restrict__ count, int H, int n,
                         int K, int cell, int C, long long rows, int* __restrict__ ccount,
                         int* __restrict__ slotpos) {
  const long long row = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const int lane = threadIdx.x & 31;
  const bool live = row < rows;
  const int i = live ? (int)(row % n) : 0;
  const long long bh = live ? row / n : 0;
  const int cnt = live ? (count ? min(max(count[row], 0), K) : K) : 0;
  int prev[kMaxKL];
#pragma unroll
  for (int k = 0; k < kMaxKL; ++k) {
    if (k >= K) break;  // uniform
    int c = k < cnt ? idx[row * K + k] : -1;
    bool ok = c >= 0 && c < C && (long long)(c + 1) * cell <= (long long)i + 1;
#pragma unroll
    for (int e = 0; e < k; ++e) ok = ok && prev[e] != c;
    prev[k] = ok ? c : -1;
    const int key = ok ? (int)(bh * C + c) : -1;  // cells < 2^31
    const unsigned same = __match_any_sync(0xffffffffu, key);
    const int leader = __ffs(same) - 1;
    int base = 0;
    if (ok && lane == leader) base = atomicAdd(&ccount[key], __popc(same));
    base = __shfl_sync(0xffffffffu, base, leader);
    if (live) slotpos[row * K + k] = ok ? base + __popc(same & ((1u << lane) - 1u)) : -1;
  }
}

// ---- 2. cell offsets and the tile list ----------------------------------------------------
__global__ void __launch_bounds__(256)
    fs_long_offsets_kernel(const int* __restrict__ ccount, long long cells,
                           int* __restrict__ cell_off, int4* __restrict__ tiles,
                           long long tile_cap, int* __restrict__ totals) {
  const long long c = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const int lane = threadIdx.x & 31;
  const int cp = c < cells ? ccount[c] : 0;
  const int ct = (cp + kRowsL - 1) / kRowsL;
  int ip = cp, it = ct;  // inclusive warp scans
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int yp = __shfl_up_sync(0xffffffffu, ip, o), yt = __shfl_up_sync(0xffffffffu, it, o);
    if (lane >= o) {
      ip += yp;
      it += yt;
    }
  }
  int bt = 0, bp = 0;
  if (lane == 31 && it > 0) {
    bt = atomicAdd(&totals[0], it);
    bp = atomicAdd(&totals[1], ip);
  }
  bt = __shfl_sync(0xffffffffu, bt, 31) + it - ct;
  bp = __shfl_sync(0xffffffffu, bp, 31) + ip - cp;
  if (c >= cells || cp == 0) return;
  cell_off[c] = bp;
  for (int q = 0; q < ct; ++q)
    if (bt + q < tile_cap)
      tiles[bt + q] = make_int4((int)c, bp + q * kRowsL, min(kRowsL, cp - q * kRowsL), 0);
}

// ---- 3. pairs in cell order -------------------------------------------------------------------
__global__ void __launch_bounds__(256)
    fs_long_scatter_kernel(const int* __restrict__ idx, const int* __restrict__ slotpos, int n,
                           int K, int C, long long rows, const int* __restrict__ cell_off,
                           int* __restrict__ pairs) {
  const long long pid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (pid >= rows * K) return;
  const int sp = slotpos[pid];
  if (sp < 0) return;
  const long long row = pid / K;
  const long long gc = (row / n) * C + idx[pid];
  pairs[cell_off[gc] + sp] = (int)pid;
}

// ---- 4. tiles: 128 gathered queries x one cell ------------------------------------------------
struct LongTileParams {
  const __nv_bfloat16* q;
  const int4* tiles;
  const int* ntiles;
  const int* pairs;
  float2* part_ml;
  __nv_bfloat16* part_o;
  int* status;
  int n, C, K;
  long long tile_cap;
  float c2;  // log2(e) / sqrt(d)
};

template <int D>
struct LongSmem {
  static constexpr int kHalves = D / 64;
  static constexpr int kQ = 0;                        // [half][128 rows x 128 B]
  static constexpr int kK = kQ + kHalves * 16384;     // [half][64 rows x 128 B]
  static constexpr int kV = kK + kHalves * 8192;      // [half][64 rows x 128 B]
  static constexpr int kP = kV + kHalves * 8192;      // [128 rows x 128 B]
  static constexpr int kTotal = kP + 16384;
  // TMEM: S in columns [0, 64), O in [64, 64 + D)
  static constexpr uint32_t kCols = D == 64 ? 128 : 256;
};

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}

template <int D>
constexpr int kCtasPerSm = D == 64 ? 4 : 2;  // TMEM: 4 x 128 or 2 x 256 of 512 columns
static_assert(kCtasPerSm<64> * LongSmem<64>::kCols <= 512 &&
                  kCtasPerSm<128> * LongSmem<128>::kCols <= 512,
              "resident CTAs must not oversubscribe TMEM");
static_assert(kCtasPerSm<64> * (LongSmem<64>::kTotal + 3 * 1024) <= 233472 &&
                  kCtasPerSm<128> * (LongSmem<128>::kTotal + 3 * 1024) <= 233472,
              "resident CTAs must fit the SM's shared memory");

template <int D, int CELL>
__global__ void __launch_bounds__(kThreadsL, kCtasPerSm<D>)
    fs_long_tile_kernel(const __grid_constant__ CUtensorMap tmk,
                        const __grid_constant__ CUtensorMap tmv, const LongTileParams p) {
  using L = LongSmem<D>;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ __align__(8) uint64_t bars[3];
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;
  uint64_t* kv_full = bars + 0;
  uint64_t* s_done = bars + 1;
  uint64_t* o_done = bars + 2;
  const int tid = threadIdx.x, warp = tid >> 5;
  if (tid == 0) {
    mbar_init(kv_full, 1);
    mbar_init(s_done, 1);
    mbar_init(o_done, 1);
    fence_mbar_init();
    s_abort = 0;
    tc::prefetch_tmap(&tmk);
    tc::prefetch_tmap(&tmv);
  }
  if (warp == 0) {
    tc::tmem_alloc(&s_tmem, L::kCols);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = s_tmem;
  const uint32_t lane_base = (uint32_t)(32 * warp) << 16;
  const uint32_t sQ = smem_u32(smem + L::kQ);
  const int ntiles = (int)min((long long)*p.ntiles, p.tile_cap);  // tiles reserved
  constexpr uint32_t idS = tc::idesc_bf16(kRowsL, CELL, false, false);
  constexpr uint32_t idO = tc::idesc_bf16(kRowsL, D, false, true);

  for (int t = blockIdx.x, it = 0; t < ntiles; t += gridDim.x, ++it) {
    const int4 tile = p.tiles[t];
    const int bh = tile.x / p.C, c = tile.x - bh * p.C;
    const int m = tile.z;
    const uint32_t ph = (uint32_t)it & 1u;
    if (tid == 0) {
      mbar_arrive_expect_tx(kv_full, 2 * L::kHalves * CELL * 128);
      const int y = bh * p.n + c * CELL;
#pragma unroll
      for (int hf = 0; hf < L::kHalves; ++hf) {
        tc::tma_load_2d(smem + L::kK + hf * 8192, &tmk, hf * 64, y, kv_full);
        tc::tma_load_2d(smem + L::kV + hf * 8192, &tmv, hf * 64, y, kv_full);
      }
    }
    // this thread's query row (zeros past the tile's last pair)
    int pid = -1;
    if (tid < m) {
      pid = p.pairs[tile.y + tid];
      const __nv_bfloat16* src = p.q + (size_t)(pid / p.K) * D;
#pragma unroll
      for (int hf = 0; hf < L::kHalves; ++hf)
#pragma unroll
        for (int ch = 0; ch < 8; ++ch)
          cp_async16(sQ + hf * 16384 + tc::sw128_offset(tid, ch), src + hf * 64 + ch * 8);
    } else {
#pragma unroll
      for (int hf = 0; hf < L::kHalves; ++hf)
#pragma unroll
        for (int ch = 0; ch < 8; ++ch)
          *reinterpret_cast<uint4*>(smem + L::kQ + hf * 16384 + tc::sw128_offset(tid, ch)) =
              make_uint4(0, 0, 0, 0);
    }
    asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
    fence_proxy_async();
    tc::fence_before_sync();
    __syncthreads();
    if (tid == 0) {
      tc::fence_after_sync();
      if (mbar_wait_bounded(kv_full, ph)) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const int hf = kk >> 2, off = (kk & 3) * 32;
          const uint64_t a = tc::smem_desc_sw128(smem + L::kQ + hf * 16384 + off, 16, 1024);
          const uint64_t b = tc::smem_desc_sw128(smem + L::kK + hf * 8192 + off, 16, 1024);
          tc::mma_f16_ss(tmem, a, b, idS, kk > 0 ? 1u : 0u);
        }
      } else {
        s_abort = 1;
      }
      tc::mma_commit(s_done);  // also when nothing was issued: the others must not wait forever
    }
    bool ok = mbar_wait_bounded(s_done, ph);
    tc::fence_after_sync();
    // softmax over the cell, one row per thread (log2 units)
    constexpr int kLd = CELL < 32 ? 32 : CELL;
    float s[kLd];
#pragma unroll
    for (int cb = 0; cb < kLd; cb += 32) tc::tmem_ld32(tmem + lane_base + cb, s + cb);
    tc::tmem_wait_ld();
    tc::reg_fence(s);
    float mx = -INFINITY;
#pragma unroll
    for (int j = 0; j < CELL; ++j) mx = fmaxf(mx, s[j]);
    const float m2 = mx * p.c2;
    float l = 0.f;
#pragma unroll
    for (int j = 0; j < CELL; ++j) {
      s[j] = tc::ex2_approx(fmaf(s[j], p.c2, -m2));
      l += s[j];
    }
#pragma unroll
    for (int ch = 0; ch < CELL / 8; ++ch) {
      __nv_bfloat162 h0 = __floats2bfloat162_rn(s[8 * ch + 0], s[8 * ch + 1]);
      __nv_bfloat162 h1 = __floats2bfloat162_rn(s[8 * ch + 2], s[8 * ch + 3]);
      __nv_bfloat162 h2 = __floats2bfloat162_rn(s[8 * ch + 4], s[8 * ch + 5]);
      __nv_bfloat162 h3 = __floats2bfloat162_rn(s[8 * ch + 6], s[8 * ch + 7]);
      *reinterpret_cast<uint4*>(smem + L::kP + tc::sw128_offset(tid, ch)) =
          make_uint4(*reinterpret_cast<uint32_t*>(&h0), *reinterpret_cast<uint32_t*>(&h1),
                     *reinterpret_cast<uint32_t*>(&h2), *reinterpret_cast<uint32_t*>(&h3));
    }
    fence_proxy_async();
    tc::fence_before_sync();
    __syncthreads();
    if (tid == 0) {
      tc::fence_after_sync();
      if (ok && !s_abort) {
#pragma unroll
        for (int kk = 0; kk < CELL / 16; ++kk) {
          const uint64_t a = tc::smem_desc_sw128(smem + L::kP + kk * 32, 16, 1024);
          const uint64_t b = tc::smem_desc_sw128(smem + L::kV + kk * 2048, 8192, 1024);
          tc::mma_f16_ss(tmem + 64u, a, b, idO, kk > 0 ? 1u : 0u);
        }
      }
      tc::mma_commit(o_done);
    }
    ok = mbar_wait_bounded(o_done, ph) && ok;
    tc::fence_after_sync();
    const bool stop = __syncthreads_or(!ok || s_abort);
    if (stop) {
      if (tid == 0) s_abort = 1;
      break;
    }
    // normalised output row (bf16) and (max, sum) to the pair's record
    const float inv_l = 1.f / l;
#pragma unroll
    for (int cb = 0; cb < D; cb += 32) {
      float o[32];
      tc::tmem_ld32(tmem + lane_base + 64u + cb, o);
      tc::tmem_wait_ld();
      tc::reg_fence(o);
      if (pid >= 0) {
        uint4* dst = reinterpret_cast<uint4*>(p.part_o + (size_t)pid * D + cb);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          __nv_bfloat162 h0 = __floats2bfloat162_rn(o[8 * e + 0] * inv_l, o[8 * e + 1] * inv_l);
          __nv_bfloat162 h1 = __floats2bfloat162_rn(o[8 * e + 2] * inv_l, o[8 * e + 3] * inv_l);
          __nv_bfloat162 h2 = __floats2bfloat162_rn(o[8 * e + 4] * inv_l, o[8 * e + 5] * inv_l);
          __nv_bfloat162 h3 = __floats2bfloat162_rn(o[8 * e + 6] * inv_l, o[8 * e + 7] * inv_l);
          dst[e] = make_uint4(*reinterpret_cast<uint32_t*>(&h0), *reinterpret_cast<uint32_t*>(&h1),
                              *reinterpret_cast<uint32_t*>(&h2), *reinterpret_cast<uint32_t*>(&h3));
        }
      }
    }
    if (pid >= 0) p.part_ml[pid] = make_float2(m2, l);
    tc::fence_before_sync();
    __syncthreads();  // TMEM and shared memory are reused by the next tile
  }
  tc::fence_before_sync();
  __syncthreads();
  if (s_abort && tid == 0) report_timeout(p.status, 7);
  if (warp == 0) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, L::kCols);
  }
}

// ---- 5. merge a query's partials and mix into the short-branch output -----------------------
template <int D>
__global__ void __launch_bounds__(256)
    fs_long_combine_kernel(const int* __restrict__ slotpos, const float2* __restrict__ part_ml,
                           const __nv_bfloat16* __restrict__ part_o,
                           const float* __restrict__ alpha, int H, int n, int K, long long rows,
                           __nv_bfloat16* __restrict__ o) {
  constexpr int E = D / 32;  // elements per lane
  const long long row = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  float M = -INFINITY;
  for (int k = 0; k < K; ++k)
    if (slotpos[row * K + k] >= 0) M = fmaxf(M, part_ml[row * K + k].x);
  if (M == -INFINITY) return;  // no cell attended: o keeps the short branch
  float acc[E];
#pragma unroll
  for (int e = 0; e < E; ++e) acc[e] = 0.f;
  float Lsum = 0.f;
  for (int k = 0; k < K; ++k) {
    if (slotpos[row * K + k] < 0) continue;
    const float2 ml = part_ml[row * K + k];
    const float w = ml.y * exp2f(ml.x - M);  // this pair's share of the softmax mass
    Lsum += w;
    const __nv_bfloat16* src = part_o + (size_t)(row * K + k) * D + lane * E;
#pragma unroll
    for (int e = 0; e < E; e += 2) {
      const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(src + e));
      acc[e] = fmaf(w, f.x, acc[e]);
      acc[e + 1] = fmaf(w, f.y, acc[e + 1]);
    }
  }
  const float a = alpha[(row / n) % H];
  const float inv = 1.f / Lsum;
  __nv_bfloat16* dst = o + (size_t)row * D + lane * E;
#pragma unroll
  for (int e = 0; e < E; e += 2) {
    const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(dst + e));
    *reinterpret_cast<__nv_bfloat162*>(dst + e) = __floats2bfloat162_rn(
        (1.f - a) * f.x + a * (acc[e] * inv), (1.f - a) * f.y + a * (acc[e + 1] * inv));
  }
}

// ---- host side ------------------------------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 encode_long() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult qr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &qr) ==
            cudaSuccess &&
        qr == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    else
      (void)cudaGetLastError();
  });
  return fn;
}

bool map_cells(CUtensorMap* m, const void* base, long long rows, int D, int box_rows) {
  auto enc = encode_long();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)D * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Persistent grid: the SM count times the CTAs per SM the kernel is built for (its launch bounds;
// shared memory and the 512 TMEM columns allow exactly that many).  The runtime occupancy query
// is not used: for this kernel it reported one CTA per SM where four are resident.
int persistent_grid(const void* kern, int smem, int per_sm) {
  static std::mutex mu;
  static std::map<std::pair<int, const void*>, int> cache;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  std::lock_guard<std::mutex> lock(mu);
  const auto key = std::make_pair(dev, kern);
  auto f = cache.find(key);
  if (f != cache.end()) return f->second;
  int sms = 0;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
          cudaSuccess ||
      cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                           (int)cudaSharedmemCarveoutMaxShared) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    (void)cudaGetLastError();
    return -1;
  }
  cache[key] = sms * per_sm;
  return sms * per_sm;
}

}  // namespace

bool long_cells_supported(int d, int cell, int K, long long rows) {
  return (d == 64 || d == 128) && (cell == 16 || cell == 32 || cell == 64) && K >= 1 &&
         K <= kMaxKL && rows * K < (1ll << 31);
}

size_t long_cells_workspace(int B, int H, int n, int d, int cell, int K) {
  return carve(nullptr, B, H, n, d, cell, K, nullptr);
}

// q, k, v: raw (unrotated) bf16 [B, H, n, d]; o holds the short branch (bf16) and receives the mix.
bsa_status long_cells(const void* q, const void* k, const void* v, int B, int H, int n, int d,
                      int cell, const int* idx, const int* count, int K, const float* alpha,
                      void* o, void* ws, size_t ws_bytes, int* status, cudaStream_t st) {
  if (!ws || ws_bytes < long_cells_workspace(B, H, n, d, cell, K)) return BSA_ERR_WORKSPACE;
  const long long rows = (long long)B * H * n;
  const int C = (n + cell - 1) / cell;
  const long long cells = cells_of(B, H, n, cell);
  if (rows >= (1ll << 31) || cells >= (1ll << 31)) return BSA_ERR_UNSUPPORTED;
  FsLongWs w;
  carve(ws, B, H, n, d, cell, K, &w);
  if (cudaMemsetAsync(w.ccount, 0, (size_t)cells * 4, st) != cudaSuccess ||
      cudaMemsetAsync(w.ntiles, 0, 16, st) != cudaSuccess)
    return BSA_ERR_CUDA;
  fs_long_count_kernel<<<(unsigned)((rows + 255) / 256), 256, 0, st>>>(idx, count, H, n, K, cell,
                                                                        C, rows, w.ccount,
                                                                        w.slotpos);
  BSA_LAUNCH_CHECK();
  fs_long_offsets_kernel<<<(unsigned)((cells + 255) / 256), 256, 0, st>>>(
      w.ccount, cells, w.cell_off, w.tiles, w.tile_cap, w.ntiles);
  BSA_LAUNCH_CHECK();
  fs_long_scatter_kernel<<<(unsigned)((rows * K + 255) / 256), 256, 0, st>>>(
      idx, w.slotpos, n, K, C, rows, w.cell_off, w.pairs);
  BSA_LAUNCH_CHECK();
  CUtensorMap tmk, tmv;
  if (!map_cells(&tmk, k, rows, d, cell) || !map_cells(&tmv, v, rows, d, cell)) return BSA_ERR_CUDA;
  LongTileParams p{};
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.tiles = w.tiles; p.ntiles = w.ntiles; p.pairs = w.pairs;
  p.part_ml = w.part_ml; p.part_o = w.part_o; p.status = status;
  p.n = n; p.C = C; p.K = K; p.tile_cap = w.tile_cap;
  p.c2 = 1.4426950408889634f / sqrtf((float)d);
  auto run = [&](auto kern, int smem) -> bsa_status {
    const int grid = persistent_grid(reinterpret_cast<const void*>(kern), smem,
                                     d == 64 ? kCtasPerSm<64> : kCtasPerSm<128>);
    if (grid < 1) return BSA_ERR_CUDA;
    kern<<<grid, kThreadsL, smem, st>>>(tmk, tmv, p);
    BSA_LAUNCH_CHECK();
    return BSA_OK;
  };
  bsa_status rc;
  if (d == 64) {
    constexpr int sm = LongSmem<64>::kTotal + 1024;
    rc = cell == 16 ? run(fs_long_tile_kernel<64, 16>, sm)
         : cell == 32 ? run(fs_long_tile_kernel<64, 32>, sm)
                      : run(fs_long_tile_kernel<64, 64>, sm);
  } else {
    constexpr int sm = LongSmem<128>::kTotal + 1024;
    rc = cell == 16 ? run(fs_long_tile_kernel<128, 16>, sm)
         : cell == 32 ? run(fs_long_tile_kernel<128, 32>, sm)
                      : run(fs_long_tile_kernel<128, 64>, sm);
  }
  if (rc != BSA_OK) return rc;
  const unsigned cblocks = (unsigned)((rows * 32 + 255) / 256);
  if (d == 64)
    fs_long_combine_kernel<64><<<cblocks, 256, 0, st>>>(w.slotpos, w.part_ml, w.part_o, alpha, H,
                                                         n, K, rows,
                                                         static_cast<__nv_bfloat16*>(o));
  else
    fs_long_combine_kernel<128><<<cblocks, 256, 0, st>>>(w.slotpos, w.part_ml, w.part_o, alpha,
                                                          H, n, K, rows,
                                                          static_cast<__nv_bfloat16*>(o));
  BSA_LAUNCH_CHECK();
  return BSA_OK;
}

}  // namespace bsa
