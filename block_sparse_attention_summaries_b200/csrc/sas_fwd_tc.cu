// SAS training-mode sparse prefill forward on the tensor cores, steps split between two softmax
// warpgroups.
//
// [SAS] review: "Background" Eq. 2 (exact softmax over the selected set only), "The new approach"
// Eq. 4 / Eq. 9 (current block always kept with gate 1; in training mode log g_m added to the
// logits of selected history block m), "How it works" (the gate fused into a tiled qK^T loop with
// an online softmax; unselected blocks never enter).  "Why the four design choices matter": the
// outer gate variant scales a block's value contributions by g_m outside the softmax.
//
// A unit is 64 queries of one head sharing one selection; a CTA takes the pair of units of heads
// 2hp, 2hp+1 at one unit position (one kv head).  The two units are M = 64 tiles in complementary
// halves of the TMEM lanes (unit it's row r at lane 32 (r / 16) + 16 it + r % 16): S = [Q_0; Q_1]
// [K_0; K_1]^T is one M = 128, N = 128 chain (queries TMA-loaded in 16-row boxes into that lane
// order), and P V is an M = 64, N = d chain per unit.  A TMEM load takes one column address for the
// whole warp, so each softmax warp loads both units' 64 score columns and every lane keeps its own.
//
// The steps of the pair (selected history blocks, fully masked fillers, the diagonal block last)
// alternate between two softmax warpgroups: warpgroup w takes steps w, w + 2, ... with its own
// score tile, P buffer, output accumulator and running (max, sum).  While one warpgroup computes
// exponentials the other's scores and P V run on the tensor cores, and a warpgroup's next scores
// are issued as soon as it has read its current ones.  The two partial softmaxes merge in the
// epilogue (log-sum-exp of the two (max, sum) pairs; each warpgroup writes half the columns).
//   warps 0-3: softmax, even steps    warps 4-7: softmax, odd steps
//   warp 8:    Q and K producer (TMA)  warp 9: MMA issuer    warp 10: V producer
// TMEM: S_w at 128 w, O_w at 256 + d w (512 columns).  K ring 3 slots (6 at d = 64) freed when
// S completes, V ring 2 slots (4) freed when P V completes.  Every mbarrier wait is bounded; on
// timeout the CTA records it, skips the rest of its work and still releases TMEM.
#include <cudaTypedefs.h>

#include <mutex>

#include "tc_common.cuh"

namespace bsa {
namespace {

constexpr int kU = 64;          // queries per unit = keys per block
constexpr int kMaxSel = 64;     // selected history blocks per unit
constexpr int kSasThreads = 352;
constexpr float kSLog2e = 1.4426950408889634f;
constexpr float kSLn2 = 0.6931471805599453f;
constexpr float kSRescale = 8.f;

// max(a, b, c) in one instruction (the three-input form of sm_100)
__device__ __forceinline__ float max3f(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

struct SasParams {
  int B, Hq, Hk, n, U, K;
  const int* idx;
  const int* count;
  int gate, norm;
  const float* scores;
  int scores_ld;
  void* o;
  float* lse;
  int* status;
};

template <int D>
struct SasSmem {
  static constexpr int kTile = kU * D * 2;  // one [64 x D] bf16 tile
  static constexpr int kKSlots = D == 64 ? 6 : 3;
  static constexpr int kVSlots = D == 64 ? 4 : 2;
  static constexpr int kQ = 0;                              // [half][128 rows x 128 B]
  static constexpr int kK = 2 * kTile;                      // [slot][half][2 units x 64 rows]
  static constexpr int kV = kK + kKSlots * 2 * kTile;       // [slot][unit] tiles
  static constexpr int kPBytes = kU * 64 * 2;               // [64 x 64] bf16
  static constexpr int kP = kV + kVSlots * 2 * kTile;       // [warpgroup][unit]
  static constexpr int kTotal = kP + 4 * kPBytes;
};

template <int D>
__global__ void __launch_bounds__(kSasThreads, 1)
    sas_fwd_tc_kernel(const __grid_constant__ CUtensorMap tmq,
                      const __grid_constant__ CUtensorMap tmk,
                      const __grid_constant__ CUtensorMap tmv, const SasParams p) {
  using L = SasSmem<D>;
  constexpr int KS = L::kKSlots, VS = L::kVSlots;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = smem_align1024(smem_raw);
  __shared__ __align__(8) uint64_t bars[30];
  uint64_t* q_full = bars + 0;
  uint64_t* k_full = bars + 1;    // [KS <= 6]
  uint64_t* k_empty = bars + 7;   // [KS]
  uint64_t* v_full = bars + 13;   // [VS <= 4]
  uint64_t* v_empty = bars + 17;  // [VS]
  uint64_t* s_full = bars + 21;   // [2] per warpgroup
  uint64_t* s_free = bars + 23;
  uint64_t* p_full = bars + 25;
  uint64_t* o_done = bars + 27;
  uint64_t* fin = bars + 29;
  __shared__ uint32_t s_tmem;
  __shared__ int s_blk[2][kMaxSel];
  __shared__ float s_bias[2][kMaxSel];  // log2 g_m of each selected block
  __shared__ int s_cnt[2];
  __shared__ int s_abort;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int u = blockIdx.x, hp = blockIdx.y, bi = blockIdx.z;
  const int G = p.Hq / p.Hk;
  const int kh = (2 * hp) / G;

  // ---- prologue: block lists and gate biases of both units (warps 0 and 1) -----------------
  if (warp < 2) {
    const int it = warp;
    const int nc = u;  // history blocks before unit u
    const size_t row = ((size_t)bi * p.Hq + 2 * hp + it) * p.U + u;
    const int cnt_in = p.count ? min(p.count[row], p.K) : p.K;
    int base = 0;
    for (int j0 = 0; j0 < cnt_in; j0 += 32) {
      const int j = j0 + lane;
      const int m = j < cnt_in ? p.idx[row * p.K + j] : -1;
      const bool good = j < cnt_in && m >= 0 && m < nc;
      const unsigned bal = __ballot_sync(0xffffffffu, good);
      const int at = base + __popc(bal & ((1u << lane) - 1u));
      if (good && at < kMaxSel) s_blk[it][at] = m;
      base += __popc(bal);
    }
    base = min(base, kMaxSel);
    __syncwarp();
    if (p.gate != BSA_GATE_NONE) {
      const float* srow = p.scores + row * p.scores_ld;
      float mx = -INFINITY, acc = 0.f;
      if (p.norm == BSA_NORM_ALL_HISTORY) {
        for (int c = lane; c < nc; c += 32) mx = fmaxf(mx, srow[c]);
        mx = warp_max(mx);
        for (int c = lane; c < nc; c += 32) acc += exp2f((srow[c] - mx) * kSLog2e);
      } else {
        for (int j = lane; j < base; j += 32) mx = fmaxf(mx, srow[s_blk[it][j]]);
        mx = warp_max(mx);
        for (int j = lane; j < base; j += 32) acc += exp2f((srow[s_blk[it][j]] - mx) * kSLog2e);
      }
      acc = warp_sum(acc);
      const float lnorm = mx == -INFINITY ? 0.f : mx + logf(acc);
      for (int j = lane; j < base; j += 32) s_bias[it][j] = (srow[s_blk[it][j]] - lnorm) * kSLog2e;
    } else {
      for (int j = lane; j < base; j += 32) s_bias[it][j] = 0.f;
    }
    if (lane == 0) s_cnt[it] = base;
  }
  if (tid == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < KS; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&k_empty[i], 1);
    }
    for (int i = 0; i < VS; ++i) {
      mbar_init(&v_full[i], 1);
      mbar_init(&v_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_free[i], 128);
      mbar_init(&p_full[i], 128);
      mbar_init(&o_done[i], 1);
    }
    mbar_init(fin, 1);
    fence_mbar_init();
    s_abort = 0;
  }
  if (warp == 9) {
    tc::tmem_alloc(&s_tmem, 512);
    tc::tmem_relinquish();
  }
  if (warp == 8 && lane == 0) {
    tc::prefetch_tmap(&tmq);
    tc::prefetch_tmap(&tmk);
    tc::prefetch_tmap(&tmv);
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const int steps = max(s_cnt[0], s_cnt[1]) + 1;  // the diagonal block is the last step
  const uint32_t tmem = s_tmem;
  // step j of unit it: history block, filler (fully masked) or the diagonal block
  auto step_block = [&](int it, int j) { return j < s_cnt[it] ? s_blk[it][j] : u; };
  auto kslot = [&](int sl) { return smem + L::kK + sl * 2 * L::kTile; };
  auto vtile = [&](int sl, int it) { return smem + L::kV + (2 * sl + it) * L::kTile; };
  auto ptile = [&](int w, int it) { return smem + L::kP + (2 * w + it) * L::kPBytes; };

  if (warp == 8 || warp == 10) {
    // ------------------------------------------- producers: warp 8 Q and K, warp 10 V
    if (lane == 0) {
      const bool is_k = warp == 8;
      if (is_k) {  // 16-row boxes into the accumulator lane order
        mbar_arrive_expect_tx(q_full, 2 * L::kTile);
        for (int it = 0; it < 2; ++it) {
          const int y = ((bi * p.Hq + 2 * hp + it) * p.n) + u * kU;
          for (int hf = 0; hf < D / 64; ++hf)
            for (int b4 = 0; b4 < 4; ++b4)
              tc::tma_load_2d(smem + L::kQ + hf * 16384 + (32 * b4 + 16 * it) * 128, &tmq,
                              hf * 64, y + 16 * b4, q_full);
        }
      }
      const int nslots = is_k ? KS : VS;
      uint64_t* full = is_k ? k_full : v_full;
      uint64_t* empty = is_k ? k_empty : v_empty;
      const CUtensorMap* tm = is_k ? &tmk : &tmv;
      int issued = 0;
      bool ok = true;
      for (int j = 0; j < steps; ++j) {
        const int sl = j % nslots;
        if (j >= nslots && !mbar_wait_bounded(&empty[sl], ((j / nslots) - 1) & 1)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&full[sl], 2 * L::kTile);
        for (int it = 0; it < 2; ++it) {
          const int y = ((bi * p.Hk + kh) * p.n) + step_block(it, j) * kU;
          unsigned char* dst = is_k ? kslot(sl) + it * 8192 : vtile(sl, it);
          for (int hf = 0; hf < D / 64; ++hf)
            tc::tma_load_2d(dst + hf * (is_k ? 16384 : 8192), tm, hf * 64, y, &full[sl]);
        }
        issued = j + 1;
      }
      if (!ok) {  // loads still in flight land before the CTA leaves
        s_abort = 1;
        for (int j = max(0, issued - nslots); j < issued; ++j)
          (void)mbar_wait_bounded(&full[j % nslots], (j / nslots) & 1, 1u << 16);
      }
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = tc::idesc_bf16(128, 128, false, false);
      constexpr uint32_t idO = tc::idesc_bf16(64, D, false, true);
      auto issue_s = [&](int j) {
        const int sl = j % KS;
        const uint32_t d_s = tmem + (uint32_t)((j & 1) * 128);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const int hf = kk >> 2, off = (kk & 3) * 32;
          const uint64_t a = tc::smem_desc_sw128(smem + L::kQ + hf * 16384 + off, 16, 1024);
          const uint64_t b = tc::smem_desc_sw128(kslot(sl) + hf * 16384 + off, 16, 1024);
          tc::mma_f16_ss(d_s, a, b, idS, kk > 0);
        }
        tc::mma_commit(&s_full[j & 1]);
        tc::mma_commit(&k_empty[sl]);
      };
      bool ok = mbar_wait_bounded(q_full, 0);
      for (int j = 0; ok && j < min(2, steps); ++j) {
        ok = mbar_wait_bounded(&k_full[j], 0);
        if (!ok) break;
        tc::fence_after_sync();
        issue_s(j);
      }
      for (int j = 0; ok && j < steps; ++j) {
        const int w = j & 1;
        // the scores two steps ahead, once this step's warpgroup has read its score tile
        if (j + 2 < steps) {
          const int j2 = j + 2;
          ok = mbar_wait_bounded(&s_free[w], (j >> 1) & 1) &&
               mbar_wait_bounded(&k_full[j2 % KS], (j2 / KS) & 1);
          if (!ok) break;
          tc::fence_after_sync();
          issue_s(j2);
        }
        // P V of this step into its warpgroup's accumulator
        ok = mbar_wait_bounded(&p_full[w], (j >> 1) & 1) &&
             mbar_wait_bounded(&v_full[j % VS], (j / VS) & 1);
        if (!ok) break;
        tc::fence_after_sync();
        for (int it = 0; it < 2; ++it) {
          const uint32_t d_o =
              tmem + (uint32_t)(256 + D * w) + ((uint32_t)(16 * it) << 16);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {  // 64 keys in steps of 16
            const uint64_t a = tc::smem_desc_sw128(ptile(w, it) + kk * 32, 16, 1024);
            const uint64_t b = tc::smem_desc_sw128(vtile(j % VS, it) + kk * 2048, 8192, 1024);
            tc::mma_f16_ss(d_o, a, b, idO, (j >= 2 || kk > 0) ? 1u : 0u);
          }
        }
        tc::mma_commit(&o_done[w]);
        tc::mma_commit(&v_empty[j % VS]);
      }
      if (!ok) s_abort = 1;
      // drain: every MMA this thread issued has completed before TMEM is released
      tc::mma_commit(fin);
      if (!mbar_wait_bounded(fin, 0)) s_abort = 1;
    }
  } else {
    // ---------------------------------------- softmax: warps 0-3 even steps, 4-7 odd steps
    const int w = warp >> 2, wq = warp & 3;   // warpgroup, TMEM sub-partition
    const int it = lane >> 4;                 // unit of this thread's row
    const int r = 16 * wq + (lane & 15);      // row within the unit
    const int i = u * kU + r;                 // query position
    const int tl = 32 * wq + lane;            // TMEM lane of the row
    const uint32_t lane_base = (uint32_t)(32 * wq) << 16;
    const uint32_t s_col = (uint32_t)(128 * w);
    const uint32_t o_col = (uint32_t)(256 + D * w);
    const float qk_scale = rsqrtf((float)D) * kSLog2e;
    const bool outer = p.gate == BSA_GATE_OUTER;
    const int nw = (steps - w + 1) / 2;       // steps of this warpgroup
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int k = 0; k < nw && ok; ++k) {
      const int j = w + 2 * k;
      ok = __all_sync(0xffffffffu, mbar_wait_bounded(&s_full[w], k & 1));
      if (!ok) break;
      tc::fence_after_sync();
      // this row's 64 scores: columns 64 it .. 64 it + 63 of the score tile
      float x[64];
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        float t[32];
        tc::tmem_ld32(tmem + lane_base + s_col + (uint32_t)(32 * hh), x + 32 * hh);
        tc::tmem_ld32(tmem + lane_base + s_col + (uint32_t)(64 + 32 * hh), t);
        tc::tmem_wait_ld();
        tc::reg_fence(t);
#pragma unroll
        for (int c = 0; c < 32; ++c) x[32 * hh + c] = it ? t[c] : x[32 * hh + c];
      }
      tc::fence_before_sync();
      mbar_arrive(&s_free[w]);
      const bool is_cur = j == steps - 1;
      const bool filler = !is_cur && j >= s_cnt[it];
      const float lg = (!is_cur && !filler) ? s_bias[it][j] : 0.f;  // log2 g_m
      // inner gate: a logit bias; outer gate: P scaled by g_m for P V (the row sum stays ungated)
      const float bias = outer ? 0.f : lg;
      const float vs = outer ? tc::ex2_approx(lg) : 1.f;
      // keys the row sees: all of a history block, none of a filler, c <= r on the diagonal (the
      // masked form runs for the whole warp when any of its rows needs it)
      uint64_t keep = filler ? 0ull : ~0ull;
      if (is_cur) keep &= r >= 63 ? ~0ull : ((2ull << r) - 1ull);
      if (__any_sync(0xffffffffu, keep != ~0ull)) {
#pragma unroll
        for (int c = 0; c < 64; ++c) x[c] = ((keep >> c) & 1ull) ? x[c] : -INFINITY;
      }
      // row maximum of the raw scores (three-input maxima); the scale is positive and the bias
      // the same for the whole block, so the logit maximum is max * scale + bias and each key
      // needs one FMA before its exp2
      float mx4[4];
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) mx4[q4] = max3f(x[q4], x[4 + q4], x[8 + q4]);  // 0-11
#pragma unroll
      for (int c = 12; c + 8 <= 64; c += 8) {  // 12-59
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) mx4[q4] = max3f(mx4[q4], x[c + q4], x[c + 4 + q4]);
      }
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) mx4[q4] = fmaxf(mx4[q4], x[60 + q4]);  // 60-63
      const float mraw = max3f(mx4[0], mx4[1], fmaxf(mx4[2], mx4[3]));
      const float mx = mraw == -INFINITY ? -INFINITY : fmaf(mraw, qk_scale, bias);
      const float m_new = fmaxf(m_run, mx);
      // the first finite max needs no O scaling (the row's O and l are still 0); later ones
      // rescale O only when the max grows by more than 2^8
      const bool rescale = m_run != -INFINITY && m_new > m_run + kSRescale;
      float corr = 1.f;
      if (rescale) corr = tc::ex2_approx(m_run - m_new);
      if (rescale || m_run == -INFINITY) m_run = m_new;
      // masked keys give 2^-inf = 0; a row with nothing seen yet subtracts 0
      const float off = bias - (m_run == -INFINITY ? 0.f : m_run);
      // two keys per packed FMA (exponent argument), packed multiply (gate) and packed add (four
      // pairs of partial row sums)
      const uint64_t sc2 = tc::pack_f2(qk_scale, qk_scale), off2 = tc::pack_f2(off, off);
      const uint64_t vs2 = tc::pack_f2(vs, vs);
      uint64_t sum2[4] = {0ull, 0ull, 0ull, 0ull};
      uint32_t pk[32];
#pragma unroll
      for (int c = 0; c < 64; c += 2) {
        float a0, a1;
        tc::unpack_f2(tc::fma_f2(tc::pack_f2(x[c], x[c + 1]), sc2, off2), a0, a1);
        const uint64_t p2 = tc::pack_f2(tc::ex2_approx(a0), tc::ex2_approx(a1));
        sum2[(c >> 1) & 3] = tc::add_f2(sum2[(c >> 1) & 3], p2);
        float g0, g1;
        tc::unpack_f2(tc::mul_f2(p2, vs2), g0, g1);
        const __nv_bfloat162 h2 = __floats2bfloat162_rn(g0, g1);
        pk[c / 2] = *reinterpret_cast<const uint32_t*>(&h2);
      }
      float sl[8];
#pragma unroll
      for (int e = 0; e < 4; ++e) tc::unpack_f2(sum2[e], sl[2 * e], sl[2 * e + 1]);
      l_run = l_run * corr + (((sl[0] + sl[1]) + (sl[2] + sl[3])) + ((sl[4] + sl[5]) + (sl[6] + sl[7])));
      // this warpgroup's previous P V (step j - 2) has completed before its accumulator is
      // rescaled and its P buffer rewritten
      if (k > 0) {
        ok = __all_sync(0xffffffffu, mbar_wait_bounded(&o_done[w], (k - 1) & 1));
        if (!ok) break;
        tc::fence_after_sync();
        if (__any_sync(0xffffffffu, rescale)) {  // warp-wide TMEM round trip, others x 1
          if (!rescale) corr = 1.f;
          for (int c0 = 0; c0 < D; c0 += 32) {
            float ov[32];
            tc::tmem_ld32(tmem + lane_base + o_col + (uint32_t)c0, ov);
            tc::tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 32; ++c) ov[c] *= corr;
            tc::tmem_st32(tmem + lane_base + o_col + (uint32_t)c0, ov);
          }
          tc::tmem_wait_st();
        }
      }
      // P row -> shared memory, 128-byte swizzled K-major [64 x 64]
      unsigned char* prow = ptile(w, it);
#pragma unroll
      for (int ch = 0; ch < 8; ++ch) {
        const uint4 w4 = make_uint4(pk[4 * ch], pk[4 * ch + 1], pk[4 * ch + 2], pk[4 * ch + 3]);
        *reinterpret_cast<uint4*>(prow + tc::sw128_offset(r, ch)) = w4;
      }
      fence_proxy_async();
      tc::fence_before_sync();
      mbar_arrive(&p_full[w]);
    }
    // epilogue: both warpgroups' last P V complete, their (max, sum) exchanged; warpgroup w
    // writes columns [w d / 2, (w + 1) d / 2) of every row
    if (ok && nw > 0) ok = __all_sync(0xffffffffu, mbar_wait_bounded(&o_done[w], (nw - 1) & 1));
    if (!ok) s_abort = 1;
    // past this barrier both accumulators are final and no MMA reads the queries any more (every
    // S is issued before the last P V of either warpgroup): the query tile holds the exchange
    tc::fence_before_sync();
    asm volatile("bar.sync 1, 256;" ::: "memory");
    tc::fence_after_sync();
    float* s_ml = reinterpret_cast<float*>(smem + L::kQ);  // [warpgroup][max, sum][TMEM lane]
    const bool fine = !s_abort;
    if (fine) {
      s_ml[(2 * w) * 128 + tl] = m_run;
      s_ml[(2 * w + 1) * 128 + tl] = l_run;
    }
    asm volatile("bar.sync 1, 256;" ::: "memory");
    if (fine) {
      const bool has1 = steps > 1;  // warpgroup 1 wrote its accumulator
      const float m0 = s_ml[tl], l0 = s_ml[128 + tl];
      const float m1 = has1 ? s_ml[256 + tl] : -INFINITY, l1 = has1 ? s_ml[384 + tl] : 0.f;
      const float M = fmaxf(m0, m1);
      const float c0 = m0 == -INFINITY ? 0.f : tc::ex2_approx(m0 - M);
      const float c1 = m1 == -INFINITY ? 0.f : tc::ex2_approx(m1 - M);
      const float lsum = l0 * c0 + l1 * c1;
      const float inv = 1.f / lsum;
      const float a0 = c0 * inv, a1 = c1 * inv;
      const bool live = i < p.n;
      const size_t orow = ((size_t)bi * p.Hq + 2 * hp + it) * p.n + i;
      __nv_bfloat16* op = static_cast<__nv_bfloat16*>(p.o) + orow * D;
#pragma unroll
      for (int cb = 0; cb < D / 2; cb += 32) {
        const int col = w * (D / 2) + cb;
        float oa[32], ob[32];
        tc::tmem_ld32(tmem + lane_base + 256u + (uint32_t)col, oa);
        if (has1) tc::tmem_ld32(tmem + lane_base + (uint32_t)(256 + D + col), ob);
        tc::tmem_wait_ld();
        if (!has1) {
#pragma unroll
          for (int c = 0; c < 32; ++c) ob[c] = 0.f;
        }
        if (live) {
#pragma unroll
          for (int c = 0; c < 32; c += 8) {
            uint32_t pw[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const __nv_bfloat162 h = __floats2bfloat162_rn(
                  fmaf(oa[c + 2 * e], a0, ob[c + 2 * e] * a1),
                  fmaf(oa[c + 2 * e + 1], a0, ob[c + 2 * e + 1] * a1));
              pw[e] = *reinterpret_cast<const uint32_t*>(&h);
            }
            *reinterpret_cast<uint4*>(op + col + c) = make_uint4(pw[0], pw[1], pw[2], pw[3]);
          }
        }
      }
      if (live && w == 0 && p.lse) p.lse[orow] = (M + log2f(lsum)) * kSLn2;
    }
  }

  tc::fence_before_sync();
  __syncthreads();
  if (s_abort && tid == 0) report_timeout(p.status, 3);
  if (warp == 9) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, 512);
  }
}

PFN_cuTensorMapEncodeTiled_v12000 sas_encode() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    else
      (void)cudaGetLastError();
  });
  return fn;
}

bool sas_map(CUtensorMap* m, const void* base, long long rows, int D, int box_rows) {
  auto enc = sas_encode();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)D * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D>
bsa_status launch_sas(const void* q, const void* k, const void* v, const SasParams& p,
                      cudaStream_t st) {
  CUtensorMap tmq, tmk, tmv;
  if (!sas_map(&tmq, q, (long long)p.B * p.Hq * p.n, D, 16) ||
      !sas_map(&tmk, k, (long long)p.B * p.Hk * p.n, D, kU) ||
      !sas_map(&tmv, v, (long long)p.B * p.Hk * p.n, D, kU))
    return BSA_ERR_CUDA;
  const int smem = SasSmem<D>::kTotal + 1024;  // + alignment slack
  auto kern = sas_fwd_tc_kernel<D>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
      cudaSuccess) {
    (void)cudaGetLastError();
    return BSA_ERR_CUDA;
  }
  const dim3 grid(p.U, p.Hq / 2, p.B);
  kern<<<grid, kSasThreads, smem, st>>>(tmq, tmk, tmv, p);
  return BSA_OK;
}

}  // namespace

// Forward of the sparse prefill with per-unit selection (q_block = b = 64), paired heads.
bsa_status sas_fwd_tc(const void* q, const void* k, const void* v, int B, int Hq, int Hk, int n,
                      int d, const int* idx, const int* count, int K, int gate, int norm,
                      const float* scores, int scores_ld, void* o, float* lse, int* status,
                      cudaStream_t st) {
  if ((d != 64 && d != 128) || K > kMaxSel || (Hq / Hk) % 2 != 0) return BSA_ERR_UNSUPPORTED;
  SasParams p{};
  p.B = B; p.Hq = Hq; p.Hk = Hk; p.n = n; p.U = ceil_div(n, kU); p.K = K;
  p.idx = idx; p.count = count; p.gate = gate; p.norm = norm;
  p.scores = scores; p.scores_ld = scores_ld; p.o = o; p.lse = lse; p.status = status;
  const bsa_status rc = d == 64 ? launch_sas<64>(q, k, v, p, st) : launch_sas<128>(q, k, v, p, st);
  if (rc != BSA_OK) return rc;
  BSA_LAUNCH_CHECK();
  return BSA_OK;
}

}  // namespace bsa
