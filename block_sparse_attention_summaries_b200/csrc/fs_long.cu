// FreeSolo long branch, cell-major on the tensor cores.
//
// [FreeSolo] summary page, "How it works": each query attends, with one softmax over raw
// (unrotated) q and k, to the tokens of the K cells it selected, and the result is mixed with the
// sliding-window branch, o = (1 - alpha_h) o_short + alpha_h o_long.
//
// Every query picks only K cells of `cell` tokens, but queries that pick the same cell share its
// keys.  So the work is regrouped by cell instead of by query:
//   1. fs_long_count_block_kernel (n a multiple of 256) or fs_long_count_kernel: each valid
//      (query, slot) pair takes a position in its cell's list (shared-memory counters per
//      block of 256 queries and one global atomic per cell and block, or warp-aggregated
//      atomics: neighbouring queries tend to pick the same cells);
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
#include <type_traits>

#include "tc_common.cuh"

namespace bsa {
namespace {

constexpr int kRowsL = 128;    // pairs per tile (tcgen05 M)
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

// The same positions with the atomics aggregated over a block of 256 queries of one (batch,
// head) (n a multiple of 256): each pair first takes a place among the block's pairs of its cell
// (shared-memory counters, one per cell of the head), then every cell the block touched reserves
// that many places in the cell's list with one global atomic.
__global__ void __launch_bounds__(256)
    fs_long_count_block_kernel(const int* __restrict__ idx, const int* __restrict__ count, int n,
                               int K, int cell, int C, int* __restrict__ ccount,
                               int* __restrict__ slotpos) {
  extern __shared__ int s_cnt[];  // [C] pairs of each cell in this block, then their base
  const long long row = (long long)blockIdx.x * 256 + threadIdx.x;  // rows = B H n, n % 256 == 0
  const int i = (int)(row % n);
  const long long bh = ((long long)blockIdx.x * 256) / n;  // one (batch, head) per block
  for (int c = threadIdx.x; c < C; c += 256) s_cnt[c] = 0;
  __syncthreads();
  const int cnt = count ? min(max(count[row], 0), K) : K;
  int cells[kMaxKL], local[kMaxKL];
#pragma unroll
  for (int k = 0; k < kMaxKL; ++k) {
    cells[k] = -1;
    local[k] = 0;
    if (k >= K) continue;
    const int c = k < cnt ? idx[row * K + k] : -1;
    bool ok = c >= 0 && c < C && (long long)(c + 1) * cell <= (long long)i + 1;
#pragma unroll
    for (int e = 0; e < k; ++e) ok = ok && cells[e] != c;
    if (ok) {
      cells[k] = c;
      local[k] = atomicAdd(&s_cnt[c], 1);
    }
  }
  __syncthreads();
  for (int c = threadIdx.x; c < C; c += 256) {
    const int m = s_cnt[c];
    s_cnt[c] = m > 0 ? atomicAdd(&ccount[bh * C + c], m) : 0;
  }
  __syncthreads();
#pragma unroll
  for (int k = 0; k < kMaxKL; ++k)
    if (k < K) slotpos[row * K + k] = cells[k] >= 0 ? s_cnt[cells[k]] + local[k] : -1;
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
// Warp roles: 0-3 softmax and epilogue (thread = tile row = TMEM lane); 4 the producer (the tile's
// query rows by TMA row gathers, four rows per instruction into the 128-byte-swizzled tile, the
// cell's K and V by tiled TMA, all completing on the stage's barrier; it prefetches the next
// tile's pair ids meanwhile); 5 the MMA issuer, which issues S of a tile as soon as its stage has
// landed and P V as soon as its P is written.  S and O (TMEM) and P (shared memory) are
// double-buffered, so the softmax of one tile overlaps the gathers and MMAs of its neighbours;
// NS (2 or 3) stages of gathers are in flight per CTA.
struct LongTileParams {
  const __nv_bfloat16* q;
  const int4* tiles;
  const int* ntiles;
  const int* pairs;
  float2* part_ml;
  __nv_bfloat16* part_o;
  int* status;
  int n, C, K, rows;
  long long tile_cap;
  float c2;  // log2(e) / sqrt(d)
};

template <int D, int CELL>
struct LongSmem {
  static constexpr int kHalves = D / 64;
  static constexpr int kCtasPerSm = D == 64 ? 2 : 1;  // TMEM: 2 x 256 or 1 x 512 columns
  static constexpr int kQBytes = kHalves * 16384;      // [half][128 rows x 128 B]
  static constexpr int kKVBytes = kHalves * CELL * 128;  // [half][CELL rows x 128 B]
  static constexpr int kStageBytes = kQBytes + 2 * kKVBytes;  // Q, K, V
  static constexpr int kBytes(int ns) { return ns * kStageBytes + 2 * 16384 + ns * 128 * 4; }
  // three stages where the SM's shared memory still holds kCtasPerSm CTAs, else two
  static constexpr int kStages = kCtasPerSm * (kBytes(3) + 3 * 1024) <= 233472 ? 3 : 2;
  static constexpr int kThreads = 6 * 32;
  static constexpr int kP = kStages * kStageBytes;  // [2][128 rows x 128 B]
  static constexpr int kPid = kP + 2 * 16384;       // [kStages][128] pair ids
  static constexpr int kTotal = kPid + kStages * 128 * 4;
  // TMEM: S[b] at column 64 b, O[b] at 128 + D b
  static constexpr uint32_t kCols = D == 64 ? 256 : 512;
  static_assert(kCtasPerSm * kCols <= 512, "resident CTAs must not oversubscribe TMEM");
  static_assert(kCtasPerSm * (kTotal + 3 * 1024) <= 233472,
                "resident CTAs must fit the SM's shared memory");
};

// Four rows (y0..y3) of a 2-D tensor map whose box is one row high, columns from x, into four
// consecutive rows of shared memory (with the map's swizzle), completing on `bar`.
__device__ __forceinline__ void tma_gather4(uint32_t dst, const CUtensorMap* map, int x, int y0,
                                            int y1, int y2, int y3, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile::gather4.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4, %5, %6}], [%7];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y0), "r"(y1), "r"(y2), "r"(y3),
      "r"(smem_u32(bar))
      : "memory");
}

template <int D, int CELL>
__global__ void __launch_bounds__(LongSmem<D, CELL>::kThreads, LongSmem<D, CELL>::kCtasPerSm)
    fs_long_tile_kernel(const __grid_constant__ CUtensorMap tmq,
                        const __grid_constant__ CUtensorMap tmk,
                        const __grid_constant__ CUtensorMap tmv, const LongTileParams p) {
  using L = LongSmem<D, CELL>;
  constexpr int NS = L::kStages;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = smem_align1024(smem_raw);
  __shared__ __align__(8) uint64_t bars[2 * 3 + 9];
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;
  uint64_t* full = bars;                // [NS] the producer's arrival + the stage's bytes
  uint64_t* empty = bars + NS;          // [NS] P V of the stage's tile done
  uint64_t* s_full = bars + 2 * NS;     // [2]
  uint64_t* p_full = bars + 2 * NS + 2; // [2] 128 softmax threads
  uint64_t* o_full = bars + 2 * NS + 4; // [2]
  uint64_t* o_free = bars + 2 * NS + 6; // [2] 128 softmax threads
  uint64_t* fin = bars + 2 * NS + 8;
  int* pid_s = reinterpret_cast<int*>(smem + L::kPid);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int i = 0; i < NS; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], 128);
      mbar_init(&o_full[i], 1);
      mbar_init(&o_free[i], 128);
    }
    mbar_init(fin, 1);
    fence_mbar_init();
    s_abort = 0;
    tc::prefetch_tmap(&tmq);
    tc::prefetch_tmap(&tmk);
    tc::prefetch_tmap(&tmv);
  }
  if (warp == 5) {
    tc::tmem_alloc(&s_tmem, L::kCols);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = s_tmem;
  const int ntiles = (int)min((long long)*p.ntiles, p.tile_cap);
  const int first = blockIdx.x, stride = gridDim.x;
  const int my = first < ntiles ? (ntiles - first + stride - 1) / stride : 0;  // this CTA's tiles
  volatile int* abort_flag = &s_abort;

  if (warp == 4) {
    // ---------------------------------------------------------------- producer
    const int rows_total = p.rows;  // a row coordinate past the end reads zeros
    // Descriptors run two tiles ahead and pair ids one tile ahead, so that no load issued here
    // is waited for in the iteration that issued it.
    auto desc = [&](int j) {
      return j < my ? p.tiles[first + j * stride] : make_int4(0, 0, 0, 0);
    };
    auto ids = [&](const int4& t, int (&out)[4]) {  // rows 4 lane .. 4 lane + 3 of the tile
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
        const int r = 4 * lane + q4;
        out[q4] = r < t.z ? p.pairs[t.y + r] : -1;
      }
    };
    int4 tile = desc(0), tile_next = desc(1);
    int pid[4], pid_next[4];
    ids(tile, pid);
    for (int j = 0; j < my; ++j) {
      const int s = j % NS;
      bool ok = true;
      if (j >= NS) ok = mbar_wait_bounded(&empty[s], ((j / NS) - 1) & 1);
      if (!__all_sync(0xffffffffu, ok) || *abort_flag) {
        *abort_flag = 1;
        break;
      }
      unsigned char* qs = smem + s * L::kStageBytes;
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) pid_s[s * 128 + 4 * lane + q4] = pid[q4];
      __syncwarp();  // the ids are written before the stage's arrival releases them
      const int bh = tile.x / p.C, c = tile.x - bh * p.C;
      if (lane == 0)
        mbar_arrive_expect_tx(&full[s], L::kHalves * 128 * 128 + 2 * L::kHalves * CELL * 128);
      __syncwarp();
      int y[4];
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) y[q4] = pid[q4] >= 0 ? pid[q4] / p.K : rows_total;
#pragma unroll
      for (int hf = 0; hf < L::kHalves; ++hf)
        tma_gather4(smem_u32(qs + hf * 16384 + 4 * lane * 128), &tmq, hf * 64, y[0], y[1], y[2],
                    y[3], &full[s]);
      if (lane == 0) {
        const int yk = bh * p.n + c * CELL;
#pragma unroll
        for (int hf = 0; hf < L::kHalves; ++hf) {
          tc::tma_load_2d(qs + L::kQBytes + hf * CELL * 128, &tmk, hf * 64, yk, &full[s]);
          tc::tma_load_2d(qs + L::kQBytes + L::kKVBytes + hf * CELL * 128, &tmv, hf * 64, yk,
                          &full[s]);
        }
      }
      ids(tile_next, pid_next);
      const int4 tile_after = desc(j + 2);
      tile = tile_next;
      tile_next = tile_after;
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) pid[q4] = pid_next[q4];
    }
  } else if (warp == 5) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0 && my > 0) {
      constexpr uint32_t idS = tc::idesc_bf16(kRowsL, CELL, false, false);
      constexpr uint32_t idO = tc::idesc_bf16(kRowsL, D, false, true);
      auto issue_s = [&](int j) {
        const unsigned char* st = smem + (j % NS) * L::kStageBytes;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const int hf = kk >> 2, off = (kk & 3) * 32;
          const uint64_t a = tc::smem_desc_sw128(st + hf * 16384 + off, 16, 1024);
          const uint64_t b =
              tc::smem_desc_sw128(st + L::kQBytes + hf * CELL * 128 + off, 16, 1024);
          tc::mma_f16_ss(tmem + 64u * (uint32_t)(j & 1), a, b, idS, kk > 0 ? 1u : 0u);
        }
        tc::mma_commit(&s_full[j & 1]);
      };
      // Issue whichever is ready first: S of tile js (its stage loaded, its S / O buffer free) or
      // P V of tile jp (its P written).  Each barrier polled is at most one phase ahead of the
      // phase awaited, so a parity test cannot pass early.
      bool ok = true;
      int js = 0, jp = 0;
      uint32_t idle = 0;
      while (jp < my) {
        bool progressed = false;
        if (js < my && mbar_try_wait(&full[js % NS], (js / NS) & 1) &&
            (js < 2 || mbar_try_wait(&o_free[js & 1], ((js >> 1) - 1) & 1))) {
          tc::fence_after_sync();
          issue_s(js);
          ++js;
          progressed = true;
        }
        if (jp < js && mbar_try_wait(&p_full[jp & 1], (jp >> 1) & 1)) {
          tc::fence_after_sync();
          const unsigned char* st = smem + (jp % NS) * L::kStageBytes;
          const unsigned char* pt = smem + L::kP + (jp & 1) * 16384;
#pragma unroll
          for (int kk = 0; kk < CELL / 16; ++kk) {
            const uint64_t a = tc::smem_desc_sw128(pt + kk * 32, 16, 1024);
            const uint64_t b = tc::smem_desc_sw128(st + L::kQBytes + L::kKVBytes + kk * 2048,
                                                   CELL * 128, 1024);
            tc::mma_f16_ss(tmem + 128u + (uint32_t)(D * (jp & 1)), a, b, idO, kk > 0 ? 1u : 0u);
          }
          tc::mma_commit(&o_full[jp & 1]);
          tc::mma_commit(&empty[jp % NS]);
          ++jp;
          progressed = true;
        }
        if (progressed) {
          idle = 0;
        } else if (++idle > (1u << 22) || *abort_flag) {
          ok = false;
          break;
        }
      }
      if (!ok) *abort_flag = 1;
      tc::mma_commit(fin);  // every MMA issued has completed before TMEM is released
      if (!mbar_wait_bounded(fin, 0)) *abort_flag = 1;
    }
  } else {
    // ---------------------------------------------------------------- softmax and epilogue
    const uint32_t lane_base = (uint32_t)(32 * warp) << 16;
    for (int j = 0; j < my; ++j) {
      const int b = j & 1, s = j % NS;
      bool ok = mbar_wait_bounded(&full[s], (j / NS) & 1);  // the stage's pair ids
      const int pid = ok ? pid_s[s * 128 + tid] : -1;
      ok = ok && mbar_wait_bounded(&s_full[b], (j >> 1) & 1);
      if (!__all_sync(0xffffffffu, ok) || *abort_flag) {
        *abort_flag = 1;
        break;
      }
      tc::fence_after_sync();
      constexpr int kLd = CELL < 32 ? 32 : CELL;
      float sv[kLd];
#pragma unroll
      for (int cb = 0; cb < kLd; cb += 32) tc::tmem_ld32(tmem + lane_base + 64u * b + cb, sv + cb);
      tc::tmem_wait_ld();
      tc::reg_fence(sv);
      float mx = -INFINITY;
#pragma unroll
      for (int e = 0; e < CELL; ++e) mx = fmaxf(mx, sv[e]);
      const float m2 = mx * p.c2;
      float l = 0.f;
#pragma unroll
      for (int e = 0; e < CELL; ++e) {
        sv[e] = tc::ex2_approx(fmaf(sv[e], p.c2, -m2));
        l += sv[e];
      }
      unsigned char* pt = smem + L::kP + b * 16384;
#pragma unroll
      for (int ch = 0; ch < CELL / 8; ++ch) {
        __nv_bfloat162 h0 = __floats2bfloat162_rn(sv[8 * ch + 0], sv[8 * ch + 1]);
        __nv_bfloat162 h1 = __floats2bfloat162_rn(sv[8 * ch + 2], sv[8 * ch + 3]);
        __nv_bfloat162 h2 = __floats2bfloat162_rn(sv[8 * ch + 4], sv[8 * ch + 5]);
        __nv_bfloat162 h3 = __floats2bfloat162_rn(sv[8 * ch + 6], sv[8 * ch + 7]);
        *reinterpret_cast<uint4*>(pt + tc::sw128_offset(tid, ch)) =
            make_uint4(*reinterpret_cast<uint32_t*>(&h0), *reinterpret_cast<uint32_t*>(&h1),
                       *reinterpret_cast<uint32_t*>(&h2), *reinterpret_cast<uint32_t*>(&h3));
      }
      fence_proxy_async();
      tc::fence_before_sync();
      mbar_arrive(&p_full[b]);
      ok = mbar_wait_bounded(&o_full[b], (j >> 1) & 1);
      if (!__all_sync(0xffffffffu, ok)) {
        *abort_flag = 1;
        break;
      }
      tc::fence_after_sync();
      // normalised output row (bf16) and (max, sum) to the pair's record
      const float inv_l = 1.f / l;
#pragma unroll
      for (int c0 = 0; c0 < D; c0 += 64) {  // 64 columns per TMEM round trip
        float o[64];
        tc::tmem_ld32(tmem + lane_base + 128u + (uint32_t)(D * b) + c0, o);
        tc::tmem_ld32(tmem + lane_base + 128u + (uint32_t)(D * b) + c0 + 32, o + 32);
        tc::tmem_wait_ld();
        tc::reg_fence(o);
        if (pid >= 0) {
          uint4* dst = reinterpret_cast<uint4*>(p.part_o + (size_t)pid * D + c0);
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            __nv_bfloat162 h0 = __floats2bfloat162_rn(o[8 * e + 0] * inv_l, o[8 * e + 1] * inv_l);
            __nv_bfloat162 h1 = __floats2bfloat162_rn(o[8 * e + 2] * inv_l, o[8 * e + 3] * inv_l);
            __nv_bfloat162 h2 = __floats2bfloat162_rn(o[8 * e + 4] * inv_l, o[8 * e + 5] * inv_l);
            __nv_bfloat162 h3 = __floats2bfloat162_rn(o[8 * e + 6] * inv_l, o[8 * e + 7] * inv_l);
            dst[e] =
                make_uint4(*reinterpret_cast<uint32_t*>(&h0), *reinterpret_cast<uint32_t*>(&h1),
                           *reinterpret_cast<uint32_t*>(&h2), *reinterpret_cast<uint32_t*>(&h3));
          }
        }
      }
      if (pid >= 0) p.part_ml[pid] = make_float2(m2, l);
      tc::fence_before_sync();
      mbar_arrive(&o_free[b]);
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (s_abort && tid == 0) report_timeout(p.status, 7);
  if (warp == 5) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, L::kCols);
  }
}

// ---- 5. merge a query's partials and mix into the short-branch output -----------------------
// A thread per (query, 8 output elements): it loads the query's slot positions and (max, sum)
// itself (the 16 / 8 threads of a query read the same words, served once per warp), all K partial
// chunks and the short-branch chunk up front, and merges without any exchange between threads.
// Slots that were not attended have no record: their loads are in bounds but unused (selected
// away, never multiplied, so whatever the buffer holds cannot leak into the result).
template <int D>
__global__ void __launch_bounds__(256)
    fs_long_combine_kernel(const int* __restrict__ slotpos, const float2* __restrict__ part_ml,
                           const __nv_bfloat16* __restrict__ part_o,
                           const float* __restrict__ alpha, int H, int n, int K, long long rows,
                           __nv_bfloat16* __restrict__ o) {
  constexpr int TPR = D / 8;  // threads per query
  const long long gid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long row = gid / TPR;
  const int c8 = (int)(gid % TPR) * 8;
  if (row >= rows) return;
  const long long r0 = row * K;
  int sp[kMaxKL];
  float2 ml[kMaxKL];
  uint4 part[kMaxKL];
#pragma unroll
  for (int k = 0; k < kMaxKL; ++k) {
    if (k < K) {
      sp[k] = slotpos[r0 + k];
      ml[k] = part_ml[r0 + k];
      part[k] = *reinterpret_cast<const uint4*>(part_o + (size_t)(r0 + k) * D + c8);
    }
  }
  __nv_bfloat16* dst = o + (size_t)row * D + c8;
  const uint4 sh = *reinterpret_cast<const uint4*>(dst);
  float M = -INFINITY;
#pragma unroll
  for (int k = 0; k < kMaxKL; ++k)
    if (k < K && sp[k] >= 0) M = fmaxf(M, ml[k].x);
  if (M == -INFINITY) return;  // no cell attended: o keeps the short branch
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  float Lsum = 0.f;
#pragma unroll
  for (int k = 0; k < kMaxKL; ++k) {
    if (k < K && sp[k] >= 0) {
      const float w = ml[k].y * exp2f(ml[k].x - M);  // the slot's share of the softmax mass
      Lsum += w;
      const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&part[k]);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __bfloat1622float2(h[e]);
        acc[2 * e] = fmaf(w, f.x, acc[2 * e]);
        acc[2 * e + 1] = fmaf(w, f.y, acc[2 * e + 1]);
      }
    }
  }
  const float a = alpha[(row / n) % H];
  const float inv = 1.f / Lsum;
  const __nv_bfloat162* hs = reinterpret_cast<const __nv_bfloat162*>(&sh);
  uint4 out;
  __nv_bfloat162* ho = reinterpret_cast<__nv_bfloat162*>(&out);
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float2 f = __bfloat1622float2(hs[e]);
    ho[e] = __floats2bfloat162_rn((1.f - a) * f.x + a * (acc[2 * e] * inv),
                                  (1.f - a) * f.y + a * (acc[2 * e + 1] * inv));
  }
  *reinterpret_cast<uint4*>(dst) = out;
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

template <typename T>
struct Tag {
  using type = T;
};

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
  if (n % 256 == 0 && C <= 12288) {  // a block is 256 queries of one head; C counters fit 48 KB
    fs_long_count_block_kernel<<<(unsigned)(rows / 256), 256, (size_t)C * 4, st>>>(
        idx, count, n, K, cell, C, w.ccount, w.slotpos);
  } else {
    fs_long_count_kernel<<<(unsigned)((rows + 255) / 256), 256, 0, st>>>(idx, count, H, n, K, cell,
                                                                          C, rows, w.ccount,
                                                                          w.slotpos);
  }
  BSA_LAUNCH_CHECK();
  fs_long_offsets_kernel<<<(unsigned)((cells + 255) / 256), 256, 0, st>>>(
      w.ccount, cells, w.cell_off, w.tiles, w.tile_cap, w.ntiles);
  BSA_LAUNCH_CHECK();
  fs_long_scatter_kernel<<<(unsigned)((rows * K + 255) / 256), 256, 0, st>>>(
      idx, w.slotpos, n, K, C, rows, w.cell_off, w.pairs);
  BSA_LAUNCH_CHECK();
  CUtensorMap tmq, tmk, tmv;
  if (!map_cells(&tmq, q, rows, d, 1) || !map_cells(&tmk, k, rows, d, cell) ||
      !map_cells(&tmv, v, rows, d, cell))
    return BSA_ERR_CUDA;
  LongTileParams p{};
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.tiles = w.tiles; p.ntiles = w.ntiles; p.pairs = w.pairs;
  p.part_ml = w.part_ml; p.part_o = w.part_o; p.status = status;
  p.n = n; p.C = C; p.K = K; p.rows = (int)rows; p.tile_cap = w.tile_cap;
  p.c2 = 1.4426950408889634f / sqrtf((float)d);
  auto run = [&](auto kern, int smem, int threads, int per_sm) -> bsa_status {
    const int grid = persistent_grid(reinterpret_cast<const void*>(kern), smem, per_sm);
    if (grid < 1) return BSA_ERR_CUDA;
    kern<<<grid, threads, smem, st>>>(tmq, tmk, tmv, p);
    BSA_LAUNCH_CHECK();
    return BSA_OK;
  };
  auto run_dc = [&](auto kern, auto tag) -> bsa_status {
    using L = typename decltype(tag)::type;
    return run(kern, L::kTotal + 1024, L::kThreads, L::kCtasPerSm);
  };
  bsa_status rc;
  if (d == 64)
    rc = cell == 16   ? run_dc(fs_long_tile_kernel<64, 16>, Tag<LongSmem<64, 16>>{})
         : cell == 32 ? run_dc(fs_long_tile_kernel<64, 32>, Tag<LongSmem<64, 32>>{})
                      : run_dc(fs_long_tile_kernel<64, 64>, Tag<LongSmem<64, 64>>{});
  else
    rc = cell == 16   ? run_dc(fs_long_tile_kernel<128, 16>, Tag<LongSmem<128, 16>>{})
         : cell == 32 ? run_dc(fs_long_tile_kernel<128, 32>, Tag<LongSmem<128, 32>>{})
                      : run_dc(fs_long_tile_kernel<128, 64>, Tag<LongSmem<128, 64>>{});
  if (rc != BSA_OK) return rc;
  const unsigned cblocks = (unsigned)((rows * (d / 8) + 255) / 256);
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
