// FreeSolo cell selection on the tensor cores: score tile Q_blk x Kbar^T (tcgen05, TMEM) with the
// erf distance bias and the per-query Top-K in the epilogue.
//
// [FreeSolo] summary page, "How it works": the candidate prefix is fixed per query block of 128
// queries, so all 128 queries of a block score the same cells:
//     r_ic = q_i . kbar_c / sqrt(d) + lambda_h * a_c * erf((i - p_c) / (2 sigma_h)),
// and each query keeps its K best cells.
//
// * One CTA per (batch, head, query block of 128): an M = 128 tile, full tcgen05 rate.
// * The fp32 mean keys are split once into bf16 hi + lo (kbar = hi + lo to ~2^-16 relative); the
//   product q . kbar is accumulated as Q hi^T + Q lo^T in fp32 TMEM, so the scores keep the
//   precision the 1e-4 index bar needs while the contraction runs on bf16 tensor cores.
// * Cells stream through a 2-stage TMA ring (128 cells per chunk at d = 64, 64 at d = 128) into
//   double-buffered TMEM.
// * The bias of cell c for row r is a degree-4 Taylor expansion of erf around the tile's middle
//   row, x0 = (i0 + 63.5 - p_c) / (2 sigma): the derivatives of erf are Hermite polynomials times
//   2/sqrt(pi) exp(-x^2), so each cell needs one erf and one exp for its five coefficients.  The
//   step t = (r - 63.5) / (2 sigma) is at most 64 / (2 sigma); the truncation error is below
//   |t|^5 / 5! * max|erf^(5)|.  The sum over k of t_r^k coef_k(c) is a rank-5 product, so it runs
//   on the tensor cores too: one extra K = 16 slice per part with A = [t^k high | t^k low] (per
//   query row, written once) and B = [sqrt(d) coef high | sqrt(d) coef high] for the first part,
//   [sqrt(d) coef low | 0] for the second (per cell, written by the epilogue one chunk ahead), all
//   bf16 splits with ~2^-18 relative error.  TMEM then holds q . kbar + bias / scale.
// * Sixteen epilogue warps at d = 64, eight at d = 128 (chunks of 128 and 64 cells):
//   warp w reads TMEM lanes 32 (w % 4) .. and the w / 4-th group of 32 columns of a chunk; each
//   keeps a register Top-K list ordered by (score desc, index asc); the lists of a row are merged
//   at the end.  A list is seeded with its first K cells; after that a group of 32 cells is
//   compared raw (TMEM value against the list's threshold times sqrt(d), lowered by 2^-20 so that
//   no cell above the threshold is missed) and only the flagged cells are scaled and offered.
//   Where the Taylor step is too large (small sigma) the bias MMA is skipped and the epilogue
//   evaluates erf per pair.
#include <cudaTypedefs.h>

#include <mutex>

#include "tc_common.cuh"

namespace bsa {
namespace {

constexpr int kRows = 128;  // queries per tile (= query block)
constexpr int kMaxTop = 8;  // K <= 8: rows keep a list of 4 (K <= 4) or 8 slots

struct FsTcParams {
  int B, H, n, C, cell, K;
  const float* max_norm;
  const float* centre;
  const float* lam;
  const float* sig;
  int* idx;
  int* count;
  int* status;
};

template <int D>
struct FsTcSmem {
  static constexpr int kNC = D == 64 ? 128 : 64;  // cells per chunk (TMEM: 2 x kNC columns)
  static constexpr int kEpiWarps = 4 * (kNC / 32);  // four lane quarters x 32-column groups
  static constexpr int kThreads = (kEpiWarps + 2) * 32;
  static constexpr int kQBytes = kRows * D * 2;
  static constexpr int kChunkBytes = kNC * D * 2;  // one of hi / lo
  static constexpr int kQ = 0;
  static constexpr int kAx = kQBytes;              // bias A: [128 rows x 128 B] (first 64 B used)
  static constexpr int kStage = kAx + kRows * 128;
  static constexpr int kStageBytes = 2 * kChunkBytes;
  static constexpr int kBx = kStage + 2 * kStageBytes;  // bias B: [2][kNC rows x 128 B]
  static constexpr int kLp = kBx + 2 * kNC * 128;       // [2][kNC] (lambda a_c, p_c), erf path
  // [32][kEpiWarps * 32] floats: the values of a thread's current 32-cell group, column tid
  // (also the merge buffer at the end: [kMaxTop][kEpiWarps * 32] keys, then as many indices)
  static constexpr int kStash = kLp + 2 * kNC * 8;
  static constexpr int kBars = kStash + 32 * kEpiWarps * 32 * 4;
  static constexpr int kTotal = kBars + 256;
};

// Order key of a score plus one: 0 marks an empty slot, NaN ranks just above it (below every
// number), -0 counts as +0; larger keys are larger scores.
__device__ __forceinline__ uint32_t okey1(float f) {
  if (f != f) return 1u;
  if (f == 0.f) f = 0.f;
  const uint32_t u = __float_as_uint(f);
  return ((u & 0x80000000u) ? ~u : (u | 0x80000000u)) + 1u;
}
__device__ __forceinline__ float okey1_to_float(uint32_t k1) {
  const uint32_t k = k1 - 1u;
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

// A row's KT best cells, descending by (score, then lower cell index).
template <int KT>
struct TopList {
  uint32_t key[KT];
  int idx[KT];
  float thr;  // NaN while a slot is empty, else the score of the last slot
  __device__ __forceinline__ void init() {
#pragma unroll
    for (int q = 0; q < KT; ++q) {
      key[q] = 0u;
      idx[q] = -1;
    }
    thr = __int_as_float(0x7fc00000);
  }
  // cells offered in increasing index order: an equal key never displaces an entry
  __device__ __forceinline__ void offer_in_order(float r, int c) {
    uint32_t k = okey1(r);
    if (k <= key[KT - 1]) return;
    int ci = c;
#pragma unroll
    for (int q = 0; q < KT; ++q) {
      const bool gt = k > key[q];
      const uint32_t tk = key[q];
      const int ti = idx[q];
      key[q] = gt ? k : tk;
      idx[q] = gt ? ci : ti;
      k = gt ? tk : k;
      ci = gt ? ti : ci;
    }
    thr = key[KT - 1] == 0u ? __int_as_float(0x7fc00000) : okey1_to_float(key[KT - 1]);
  }
  // any order: ties go to the lower index
  __device__ __forceinline__ void offer(uint32_t k, int c) {
    int ci = c;
#pragma unroll
    for (int q = 0; q < KT; ++q) {
      const bool gt = k > key[q] || (k == key[q] && k != 0u && (unsigned)ci < (unsigned)idx[q]);
      const uint32_t tk = key[q];
      const int ti = idx[q];
      key[q] = gt ? k : tk;
      idx[q] = gt ? ci : ti;
      k = gt ? tk : k;
      ci = gt ? ti : ci;
    }
  }
};

// NaN-propagating max / min: a comparator that sees a NaN puts NaN on both its outputs, so a
// network below never duplicates a finite value and a NaN input can only make its result NaN
__device__ __forceinline__ float fmax_nan(float a, float b) {
  float r;
  asm("max.NaN.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ float fmin_nan(float a, float b) {
  float r;
  asm("min.NaN.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(b));
  return r;
}
// v[o .. o + N) into descending order when it is bitonic (N a power of two, fixed indices)
template <int N>
__device__ __forceinline__ void bitonic_merge_desc(float (&v)[32], int o) {
#pragma unroll
  for (int j = N / 2; j > 0; j >>= 1)
#pragma unroll
    for (int e = 0; e < N; ++e)
      if ((e ^ j) > e) {
        const float x = v[o + e], y = v[o + (e ^ j)];
        v[o + e] = fmax_nan(x, y);
        v[o + (e ^ j)] = fmin_nan(x, y);
      }
}
// K-th largest of 32 values (destroys v): sort runs of K with bitonic networks, then halve the
// runs, keeping the K largest of each pair (elementwise max against the reversed partner is a
// bitonic sequence holding them)
template <int K>
__device__ __forceinline__ float kth_largest32(float (&v)[32]) {
#pragma unroll
  for (int g = 0; g < 32 / K; ++g)
#pragma unroll
    for (int k = 2; k <= K; k <<= 1)
#pragma unroll
      for (int j = k / 2; j > 0; j >>= 1)
#pragma unroll
        for (int e = 0; e < K; ++e)
          if ((e ^ j) > e) {
            const float x = v[g * K + e], y = v[g * K + (e ^ j)];
            const bool desc = (e & k) == 0;
            v[g * K + e] = desc ? fmax_nan(x, y) : fmin_nan(x, y);
            v[g * K + (e ^ j)] = desc ? fmin_nan(x, y) : fmax_nan(x, y);
          }
#pragma unroll
  for (int w = 32 / K; w > 1; w >>= 1)
#pragma unroll
    for (int g = 0; g < w / 2; ++g) {
#pragma unroll
      for (int e = 0; e < K; ++e)
        v[g * K + e] = fmax_nan(v[g * K + e], v[(g + w / 2) * K + K - 1 - e]);
      bitonic_merge_desc<K>(v, g * K);
    }
  return v[K - 1];
}
// a little below x, so that a value compared against it is never dropped by rounding
__device__ __forceinline__ float lowered(float x) {
  return x - fmaf(fabsf(x), 0x1p-20f, 0x1p-100f);
}

template <int D, int KT>
__global__ void __launch_bounds__(FsTcSmem<D>::kThreads, 1)
    freesolo_select_tc_kernel(const __grid_constant__ CUtensorMap tmq,
                              const __grid_constant__ CUtensorMap tmhi,
                              const __grid_constant__ CUtensorMap tmlo, const FsTcParams p) {
  using L = FsTcSmem<D>;
  constexpr int kNC = L::kNC;
  constexpr int kEpiWarps = L::kEpiWarps;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = smem_align1024(smem_raw);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBars);
  uint64_t* q_full = bars + 0;
  uint64_t* kv_full = bars + 1;   // [2]
  uint64_t* kv_empty = bars + 3;  // [2]
  uint64_t* s_full = bars + 5;    // [2]
  uint64_t* s_free = bars + 7;    // [2]
  uint64_t* fin = bars + 9;
  uint64_t* ax_full = bars + 10;  // bias A written
  uint64_t* bx_full = bars + 11;  // [2] bias B of a chunk written
  float2* lp = reinterpret_cast<float2*>(smem + L::kLp);
  float* stash = reinterpret_cast<float*>(smem + L::kStash);
  uint32_t* merge_key = reinterpret_cast<uint32_t*>(smem + L::kStash);
  int* merge_idx = reinterpret_cast<int*>(smem + L::kStash) + kMaxTop * kEpiWarps * 32;
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;
  // each list's current threshold (its K-th score, NaN while not full), [column group][row]:
  // any value a list ever held bounds its row's K-th best from below, so reads need no ordering
  __shared__ float s_thr[kEpiWarps * 32];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int qb = blockIdx.x, h = blockIdx.y, bi = blockIdx.z;
  const int i0 = qb * kRows;
  const int nc = min(p.C, i0 / p.cell);  // cells wholly before the query block
  const int nchunks = (nc + kNC - 1) / kNC;
  const size_t crow0 = ((size_t)bi * p.H + h) * p.C;

  if (tid == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&kv_full[i], 1);
      mbar_init(&kv_empty[i], 1);
      mbar_init(&s_full[i], 1);
      mbar_init(&s_free[i], kEpiWarps * 32);
      mbar_init(&bx_full[i], kNC);
    }
    mbar_init(ax_full, kRows);
    mbar_init(fin, 1);
    fence_mbar_init();
    s_abort = 0;
  }
  if (tid < kEpiWarps * 32) s_thr[tid] = __int_as_float(0x7fc00000);
  if (warp == kEpiWarps + 1) {
    tc::tmem_alloc(&s_tmem, 2 * kNC);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = s_tmem;

  if (warp == kEpiWarps) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0 && nchunks > 0) {
      mbar_arrive_expect_tx(q_full, L::kQBytes);
      const int yq = (bi * p.H + h) * p.n + i0;
      for (int hf = 0; hf < D / 64; ++hf)
        tc::tma_load_2d(smem + L::kQ + hf * (kRows * 128), &tmq, hf * 64, yq, q_full);
      int issued = 0;
      for (int j = 0; j < nchunks; ++j) {
        const int st = j & 1;
        if (j >= 2 && !mbar_wait_bounded(&kv_empty[st], ((j >> 1) - 1) & 1)) {
          s_abort = 1;
          break;
        }
        issued = j + 1;
        mbar_arrive_expect_tx(&kv_full[st], L::kStageBytes);
        const int yc = (int)crow0 + j * kNC;
        unsigned char* base = smem + L::kStage + st * L::kStageBytes;
        for (int hf = 0; hf < D / 64; ++hf) {
          tc::tma_load_2d(base + hf * (kNC * 128), &tmhi, hf * 64, yc, &kv_full[st]);
          tc::tma_load_2d(base + L::kChunkBytes + hf * (kNC * 128), &tmlo, hf * 64, yc,
                          &kv_full[st]);
        }
      }
      // on abort, let the loads already issued land before the CTA exits
      if (s_abort) {
        (void)mbar_wait_bounded(q_full, 0, 1u << 16);
        for (int j = max(0, issued - 2); j < issued; ++j)
          (void)mbar_wait_bounded(&kv_full[j & 1], (j >> 1) & 1, 1u << 16);
      }
    }
  } else if (warp == kEpiWarps + 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0 && nchunks > 0) {
      constexpr uint32_t idS = tc::idesc_bf16(kRows, kNC, false, false);
      const bool taylor = 64.f * fabsf(0.5f / p.sig[h]) <= 0.125f;  // as in the epilogue
      bool ok = mbar_wait_bounded(q_full, 0) && (!taylor || mbar_wait_bounded(ax_full, 0));
      for (int j = 0; ok && j < nchunks; ++j) {
        const int st = j & 1;
        ok = mbar_wait_bounded(&kv_full[st], (j >> 1) & 1);
        if (ok && j >= 2) ok = mbar_wait_bounded(&s_free[st], ((j >> 1) - 1) & 1);
        if (ok && taylor) ok = mbar_wait_bounded(&bx_full[st], (j >> 1) & 1);
        if (!ok) break;
        tc::fence_after_sync();
        const uint32_t d_s = tmem + (uint32_t)(st * kNC);
        const unsigned char* base = smem + L::kStage + st * L::kStageBytes;
        const unsigned char* bx = smem + L::kBx + st * (kNC * 128);
#pragma unroll
        for (int part = 0; part < 2; ++part) {  // kbar hi, then kbar lo, into one accumulator
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const int hf = kk >> 2, off = (kk & 3) * 32;
            const uint64_t a =
                tc::smem_desc_sw128(smem + L::kQ + hf * (kRows * 128) + off, 16, 1024);
            const uint64_t b = tc::smem_desc_sw128(
                base + part * L::kChunkBytes + hf * (kNC * 128) + off, 16, 1024);
            tc::mma_f16_ss(d_s, a, b, idS, (part > 0 || kk > 0) ? 1u : 0u);
          }
          if (taylor) {  // + [t^k hi | t^k lo] x [coef' hi | coef' hi] (part 0), x [coef' lo | 0]
            const uint64_t a = tc::smem_desc_sw128(smem + L::kAx + part * 32, 16, 1024);
            const uint64_t b = tc::smem_desc_sw128(bx + part * 32, 16, 1024);
            tc::mma_f16_ss(d_s, a, b, idS, 1u);
          }
        }
        tc::mma_commit(&s_full[st]);
        tc::mma_commit(&kv_empty[st]);
      }
      if (!ok) s_abort = 1;
      tc::mma_commit(fin);
      if (!mbar_wait_bounded(fin, 0)) s_abort = 1;
    }
  } else {
    // ------------------------------------------------------------------ epilogue warps
    const int sub = warp & 3, grp = warp >> 2;  // lane quarter, 32-column group of a chunk
    const int row = 32 * sub + lane;
    const int i = i0 + row;
    const uint32_t lane_base = (uint32_t)(32 * sub) << 16;
    const float scale = rsqrtf((float)D);
    const float sqrt_d = sqrtf((float)D);
    const float lam = p.lam[h];
    const float inv2s = 0.5f / p.sig[h];
    // Taylor expansion about the tile's middle row while the step stays small (|t| <= 1/8, where
    // the truncation is below 14 |t|^5 / 120 * lambda a_c = 4e-6 lambda a_c), else erf per pair.
    const bool taylor = 64.f * fabsf(inv2s) <= 0.125f;
    const float t = ((float)row - 63.5f) * inv2s;
    // The row's list (one per column group); a scan flags the cells of its 32-cell group that
    // can still be among the row's K best (score not below the largest threshold any of the
    // row's lists holds), parks the group's values in this thread's stash column, and the lane
    // offers its own flagged cells in index order.
    TopList<KT> top;
    top.init();
    auto insert_hits = [&](uint32_t hit, const float (&v)[32], float mul, int cbase) {
      const int left = nc - cbase;
      if (left < 32) hit &= (1u << left) - 1u;
      if (!hit) return;
#pragma unroll
      for (int e = 0; e < 32; ++e) stash[e * (kEpiWarps * 32) + tid] = v[e];
      while (hit) {
        const int e = __ffs(hit) - 1;
        hit &= hit - 1u;
        // the same product the unflagged path would have formed
        top.offer_in_order(stash[e * (kEpiWarps * 32) + tid] * mul, cbase + e);
      }
    };
    // the largest threshold of the row's lists (NaN while none is full)
    auto row_threshold = [&]() {
      float t = top.thr;
#pragma unroll
      for (int g = 0; g < kEpiWarps / 4; ++g)
        t = fmaxf(t, reinterpret_cast<volatile float*>(s_thr)[g * kRows + row]);
      return t;
    };
    // The list of a warp's first full group is still empty (the same for every lane: the test is
    // warp-uniform); the group's own K-th largest value is then the bound.  The two bias forms
    // are separate straight-line loops so the one that runs stays small.
    auto scan_mma_bias = [&](float (&sv)[32], int cbase, uint32_t taddr) {  // bias in TMEM
      // sv * scale >= t implies sv >= lowered(t * sqrt d)
      float tv = lowered(row_threshold() * sqrt_d);
      if (top.key[KT - 1] == 0u && nc - cbase >= 32) {
        tv = fmaxf(tv, lowered(kth_largest32<KT>(sv)));
        tc::tmem_ld32(taddr, sv);
        tc::tmem_wait_ld();
        tc::reg_fence(sv);
      }
      uint32_t hit = 0u;  // NaN bound: every cell
#pragma unroll
      for (int e = 0; e < 32; ++e) hit |= !(sv[e] < tv) ? (1u << e) : 0u;
      insert_hits(hit, sv, scale, cbase);
      s_thr[tid] = top.thr;
    };
    auto scan_direct = [&](const float (&sv)[32], const float2* lpb, int cbase) {
      float rr[32];
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        const float2 l2 = lpb[e];
        rr[e] = fmaf(sv[e], scale, l2.x * erff(((float)i - l2.y) * inv2s));
      }
      float tv = row_threshold();
      if (top.key[KT - 1] == 0u && nc - cbase >= 32) {
        // the K-th largest of K block maxima (blocks of 32 / K cells): K distinct cells reach it
        float bm = __int_as_float(0x7f800000);
#pragma unroll
        for (int g = 0; g < KT; ++g) {
          float m = rr[g * (32 / KT)];
#pragma unroll
          for (int e = 1; e < 32 / KT; ++e) m = fmax_nan(m, rr[g * (32 / KT) + e]);
          bm = fmin_nan(bm, m);
        }
        tv = fmaxf(tv, bm);
      }
      uint32_t hit = 0u;
#pragma unroll
      for (int e = 0; e < 32; ++e) hit |= !(rr[e] < tv) ? (1u << e) : 0u;
      insert_hits(hit, rr, 1.f, cbase);
      s_thr[tid] = top.thr;
    };
    // bias operands: the A rows (t^k of this row, once) and the B rows of chunk jj (one cell per
    // thread), 128-byte swizzled like the TMA tiles; slot k < 5 of B is sqrt(d) lambda a_c
    // erf^(k)(x0) / k! (so that TMEM holds q . kbar + bias / scale)
    auto pack8 = [](const float (&x)[8], uint4& w) {
      __nv_bfloat162 h0 = __floats2bfloat162_rn(x[0], x[1]), h1 = __floats2bfloat162_rn(x[2], x[3]);
      __nv_bfloat162 h2 = __floats2bfloat162_rn(x[4], x[5]), h3 = __floats2bfloat162_rn(x[6], x[7]);
      w = make_uint4(*reinterpret_cast<uint32_t*>(&h0), *reinterpret_cast<uint32_t*>(&h1),
                     *reinterpret_cast<uint32_t*>(&h2), *reinterpret_cast<uint32_t*>(&h3));
    };
    auto split8 = [](const float (&x)[8], float (&hi)[8], float (&lo)[8]) {
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        hi[k] = __bfloat162float(__float2bfloat16_rn(x[k]));
        lo[k] = x[k] - hi[k];
      }
    };
    // chunk jj's rows are written by the threads of column group jj % (kEpiWarps / 4), one cell
    // each, so that the work rotates over the warps
    auto write_bx = [&](int jj) {
      const int wt = tid - kRows * (jj % (kEpiWarps / 4));
      if (wt >= 0 && wt < kNC) {
        const int c = jj * kNC + wt;
        float cf[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        float2 l2 = make_float2(0.f, 0.f);
        if (c < nc) {
          const float la = lam * p.max_norm[crow0 + c];
          const float pc = p.centre[crow0 + c];
          l2 = make_float2(la, pc);
          if (taylor) {
            const float x = ((float)i0 + 63.5f - pc) * inv2s;
            const float x2 = x * x;
            const float e = 1.1283791670955126f * expf(-x2);  // first derivative of erf
            const float ls = la * sqrtf((float)D);
            cf[0] = ls * erff(x);
            cf[1] = ls * e;
            cf[2] = ls * (-x * e);
            cf[3] = ls * ((4.f * x2 - 2.f) * e) * (1.f / 6.f);
            cf[4] = ls * ((12.f * x - 8.f * x2 * x) * e) * (1.f / 24.f);
          }
        }
        lp[(jj & 1) * kNC + wt] = l2;
        if (taylor) {
          float hi[8], lo[8];
          split8(cf, hi, lo);
          uint4 whi, wlo;
          pack8(hi, whi);
          pack8(lo, wlo);
          unsigned char* rowp = smem + L::kBx + (jj & 1) * (kNC * 128);
          *reinterpret_cast<uint4*>(rowp + tc::sw128_offset(wt, 0)) = whi;
          *reinterpret_cast<uint4*>(rowp + tc::sw128_offset(wt, 1)) = whi;
          *reinterpret_cast<uint4*>(rowp + tc::sw128_offset(wt, 2)) = wlo;
          *reinterpret_cast<uint4*>(rowp + tc::sw128_offset(wt, 3)) = make_uint4(0, 0, 0, 0);
          fence_proxy_async();
          mbar_arrive(&bx_full[jj & 1]);
        }
      }
    };
    if (taylor && nchunks > 0) {
      if (tid < kRows) {  // A rows: powers of this row's Taylor step
        float pw[8] = {1.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        const float tr = ((float)tid - 63.5f) * inv2s;
#pragma unroll
        for (int k = 1; k < 5; ++k) pw[k] = pw[k - 1] * tr;
        float hi[8], lo[8];
        split8(pw, hi, lo);
        uint4 whi, wlo;
        pack8(hi, whi);
        pack8(lo, wlo);
        unsigned char* ax = smem + L::kAx;
        *reinterpret_cast<uint4*>(ax + tc::sw128_offset(tid, 0)) = whi;
        *reinterpret_cast<uint4*>(ax + tc::sw128_offset(tid, 1)) = wlo;
        *reinterpret_cast<uint4*>(ax + tc::sw128_offset(tid, 2)) = whi;
        *reinterpret_cast<uint4*>(ax + tc::sw128_offset(tid, 3)) = wlo;
        fence_proxy_async();
        mbar_arrive(ax_full);
      }
    }
    for (int jj = 0; jj < 2 && jj < nchunks; ++jj) write_bx(jj);
    bool ok = true;
    for (int j = 0; j < nchunks; ++j) {
      const int st = j & 1;
      ok = __all_sync(0xffffffffu, ok && !*reinterpret_cast<volatile int*>(&s_abort));
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait_bounded(&s_full[st], (j >> 1) & 1));
      tc::fence_after_sync();
      const int colh = grp * 32;
      const int cb = j * kNC + colh;
      if (ok && cb < nc) {  // warp-uniform
        const uint32_t col = (uint32_t)(st * kNC + colh);
        float sv[32];
        tc::tmem_ld32(tmem + lane_base + col, sv);
        tc::tmem_wait_ld();
        tc::reg_fence(sv);
        if (taylor)
          scan_mma_bias(sv, cb, tmem + lane_base + col);
        else
          scan_direct(sv, lp + st * kNC + colh, cb);
      }
      // every epilogue warp passes this barrier once per chunk, also after a failed wait: the
      // chunk's (lambda a_c, p_c) and bias B rows are free once every warp has scanned it
      asm volatile("bar.sync 1, %0;" ::"r"(kEpiWarps * 32));
      if (ok && j + 2 < nchunks) write_bx(j + 2);
      tc::fence_before_sync();
      mbar_arrive(&s_free[st]);
    }
    if (!ok) s_abort = 1;
    // merge the column groups' lists of each row, order the winners by index, write
    asm volatile("bar.sync 1, %0;" ::"r"(kEpiWarps * 32));  // stash free: merge reuses it
#pragma unroll
    for (int e = 0; e < KT; ++e) {
      merge_key[e * (kEpiWarps * 32) + tid] = top.key[e];
      merge_idx[e * (kEpiWarps * 32) + tid] = top.idx[e];
    }
    asm volatile("bar.sync 1, %0;" ::"r"(kEpiWarps * 32));
    if (grp == 0 && i < p.n) {
#pragma unroll
      for (int g = 1; g < kEpiWarps / 4; ++g)
#pragma unroll
        for (int e = 0; e < KT; ++e)
          top.offer(merge_key[e * (kEpiWarps * 32) + tid + kRows * g],
                    merge_idx[e * (kEpiWarps * 32) + tid + kRows * g]);
      const int kk = min(p.K, nc);
      int sel[KT];
#pragma unroll
      for (int e = 0; e < KT; ++e) sel[e] = e < kk ? top.idx[e] : INT_MAX;
#pragma unroll
      for (int a = 0; a < KT; ++a)
#pragma unroll
        for (int b2 = 0; b2 + 1 < KT - a; ++b2) {
          const int lo = min(sel[b2], sel[b2 + 1]), hi = max(sel[b2], sel[b2 + 1]);
          sel[b2] = lo;
          sel[b2 + 1] = hi;
        }
      int* out = p.idx + (((size_t)bi * p.H + h) * p.n + i) * p.K;
#pragma unroll
      for (int e = 0; e < KT; ++e)
        if (e < p.K) out[e] = e < kk ? sel[e] : -1;
      if (p.count) p.count[((size_t)bi * p.H + h) * p.n + i] = kk;
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (s_abort && tid == 0) report_timeout(p.status, 5);
  if (warp == kEpiWarps + 1) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, 2 * kNC);
  }
}

// kbar (fp32) -> bf16 hi, lo with kbar ~ hi + lo
__global__ void split_hi_lo_kernel(const float* __restrict__ x, __nv_bfloat16* __restrict__ hi,
                                   __nv_bfloat16* __restrict__ lo, long long count) {
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= count) return;
  const float v = x[i];
  const __nv_bfloat16 h = __float2bfloat16_rn(v);
  hi[i] = h;
  lo[i] = __float2bfloat16_rn(v - __bfloat162float(h));
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fs() {
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

bool map2d(CUtensorMap* m, const void* base, long long rows, int D, int box_rows) {
  auto enc = encode_fs();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)D * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

size_t freesolo_select_tc_workspace(int B, int H, int n, int d, int cell) {
  const long long C = (n + cell - 1) / cell;
  return (size_t)256 + (size_t)2 * B * H * C * d * 2 + 256;
}

bool freesolo_select_tc_supported(bsa_dtype dt, int d, int q_block, int K) {
  return dt == BSA_BF16 && (d == 64 || d == 128) && q_block == kRows && K <= kMaxTop;
}

// Workspace: [0, 256) status word (zeroed by the caller before first use), then kbar hi, kbar lo.
bsa_status freesolo_select_tc(const void* q, int B, int H, int n, int d, int cell,
                              const float* mean_k, const float* max_norm, const float* centre,
                              const float* lam, const float* sig, int K, int* idx, int* count,
                              void* ws, size_t ws_bytes, cudaStream_t st) {
  const int C = (n + cell - 1) / cell;
  if (!ws || ws_bytes < freesolo_select_tc_workspace(B, H, n, d, cell)) return BSA_ERR_WORKSPACE;
  if ((long long)B * H * n >= (1ll << 31) || (long long)B * H * C >= (1ll << 31))
    return BSA_ERR_UNSUPPORTED;  // TMA row coordinates are 32-bit
  const long long cnt = (long long)B * H * C * d;
  __nv_bfloat16* hi = reinterpret_cast<__nv_bfloat16*>(
      align_up(reinterpret_cast<uintptr_t>(ws) + 256, (uintptr_t)256));
  __nv_bfloat16* lo = hi + cnt;
  split_hi_lo_kernel<<<(unsigned)((cnt + 255) / 256), 256, 0, st>>>(mean_k, hi, lo, cnt);
  BSA_LAUNCH_CHECK();
  const int nc_box = d == 64 ? FsTcSmem<64>::kNC : FsTcSmem<128>::kNC;
  CUtensorMap tmq, tmhi, tmlo;
  if (!map2d(&tmq, q, (long long)B * H * n, d, kRows) ||
      !map2d(&tmhi, hi, (long long)B * H * C, d, nc_box) ||
      !map2d(&tmlo, lo, (long long)B * H * C, d, nc_box))
    return BSA_ERR_CUDA;
  FsTcParams p{};
  p.B = B; p.H = H; p.n = n; p.C = C; p.cell = cell; p.K = K;
  p.max_norm = max_norm; p.centre = centre; p.lam = lam; p.sig = sig;
  p.idx = idx; p.count = count; p.status = static_cast<int*>(ws);
  const dim3 grid((n + kRows - 1) / kRows, H, B);
  auto run = [&](auto kern, int smem, int threads) -> bsa_status {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
        cudaSuccess) {
      (void)cudaGetLastError();
      return BSA_ERR_CUDA;
    }
    kern<<<grid, threads, smem, st>>>(tmq, tmhi, tmlo, p);
    BSA_LAUNCH_CHECK();
    return BSA_OK;
  };
  using S64 = FsTcSmem<64>;
  using S128 = FsTcSmem<128>;
  if (d == 64)
    return K <= 4 ? run(freesolo_select_tc_kernel<64, 4>, S64::kTotal + 1024, S64::kThreads)
                  : run(freesolo_select_tc_kernel<64, 8>, S64::kTotal + 1024, S64::kThreads);
  return K <= 4 ? run(freesolo_select_tc_kernel<128, 4>, S128::kTotal + 1024, S128::kThreads)
                : run(freesolo_select_tc_kernel<128, 8>, S128::kTotal + 1024, S128::kThreads);
}

}  // namespace bsa
