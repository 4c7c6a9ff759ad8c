// SAS training-mode sparse prefill forward on the tensor cores, two unit pairs per CTA in
// ping-pong.
//
// [SAS] review: "Background" Eq. 2 (exact softmax over the selected set only), "The new approach"
// Eq. 4 / Eq. 9 (current block always kept with gate 1; in training mode log g_m added to the
// logits of selected history block m), "How it works" (the gate fused into a tiled qK^T loop with
// an online softmax; unselected blocks never enter).  "Why the four design choices matter": the
// outer gate variant scales a block's value contributions by g_m outside the softmax.
//
// A unit is 64 queries of one head sharing one selection; a pair is heads 2hp, 2hp+1 at one unit
// (one kv head).  The two units of a pair are M = 64 tiles in complementary halves of the TMEM
// lanes (unit it's row r at lane 32 (r / 16) + 16 it + r % 16), so S = [Q_0; Q_1] [K_0; K_1]^T is
// one M = 128, N = 128 chain and each softmax thread owns one row.  A CTA takes two pairs -- the
// same heads at units 2x and 2x + 1 -- and runs them in ping-pong: every pair has its own softmax
// warpgroup, its own score tile and output accumulator in TMEM (4 x 128 columns), and the MMA
// thread alternates between the pairs (P V of one pair, then the next S of that pair, while the
// other pair's softmax runs), so the exponentials of one pair hide behind the other's MMAs.
//   warps 0-3: softmax of pair 0      warps 4-7: softmax of pair 1
//   warp 8:    Q and K producer (TMA)  warp 9: MMA issuer    warp 10: V producer
// Steps: both pairs walk max(selected count) + 1 blocks (history blocks, fully masked fillers for
// shorter units, the diagonal block last); the global step sequence is pair 0 step 0, pair 1
// step 0, pair 0 step 1, ..., and the K and V rings hold one pair-step per slot.  The softmax reads
// its 64 scores in two 32-column halves twice (maximum first, then exponentials), which keeps the
// register footprint inside the 352-thread budget.  Every mbarrier wait is bounded.
#include <cudaTypedefs.h>

#include <mutex>

#include "tc_common.cuh"

namespace bsa {
namespace {

constexpr int kU = 64;          // queries per unit = keys per block
constexpr int kMaxSel = 32;     // selected history blocks per unit (static shared memory)
constexpr int kSasThreads = 352;
constexpr float kSLog2e = 1.4426950408889634f;
constexpr float kSLn2 = 0.6931471805599453f;
constexpr float kSRescale = 8.f;

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
  static constexpr int kTile = kU * D * 2;   // one [64 x D] bf16 tile
  static constexpr int kPair = 2 * kTile;    // [half][2 units x 64 rows x 128 B]
  static constexpr int kQ = 0;               // [pair] Q pairs
  static constexpr int kK = 2 * kPair;       // [2 slots] K pairs
  static constexpr int kV = kK + 2 * kPair;  // [2 slots][2 units] V tiles
  static constexpr int kPBytes = kU * 64 * 2;
  static constexpr int kP = kV + 2 * kPair;  // [pair][unit] P tiles
  static constexpr int kTotal = kP + 4 * kPBytes;
};

template <int D>
__global__ void __launch_bounds__(kSasThreads, 1)
    sas_fwd_tc_kernel(const __grid_constant__ CUtensorMap tmq,
                      const __grid_constant__ CUtensorMap tmk,
                      const __grid_constant__ CUtensorMap tmv, const SasParams p) {
  using L = SasSmem<D>;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ __align__(8) uint64_t bars[20];
  uint64_t* q_full = bars + 0;    // [2] per pair
  uint64_t* k_full = bars + 2;    // [2] per slot
  uint64_t* k_empty = bars + 4;
  uint64_t* v_full = bars + 6;
  uint64_t* v_empty = bars + 8;
  uint64_t* s_full = bars + 10;   // [2] per pair
  uint64_t* s_free = bars + 12;
  uint64_t* p_full = bars + 14;
  uint64_t* o_done = bars + 16;
  uint64_t* fin = bars + 18;
  __shared__ uint32_t s_tmem;
  __shared__ int s_blk[4][kMaxSel];     // item = 2 pair + unit-in-pair
  __shared__ float s_bias[4][kMaxSel];  // log2 g_m of each selected block
  __shared__ int s_cnt[4];
  __shared__ int s_abort;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int hp = blockIdx.y, bi = blockIdx.z;
  const int G = p.Hq / p.Hk;
  const int kh = (2 * hp) / G;
  auto item_head = [&](int item) { return 2 * hp + (item & 1); };
  auto item_unit = [&](int item) { return 2 * (int)blockIdx.x + (item >> 1); };

  // ---- prologue: block lists and gate biases of the four items (warps 0-3) ----------------
  if (warp < 4) {
    const int item = warp, u = item_unit(item);
    const bool ok = u < p.U;
    const int nc = u;  // history blocks before unit u
    int base = 0;
    if (ok) {
      const size_t row = ((size_t)bi * p.Hq + item_head(item)) * p.U + u;
      const int cnt_in = p.count ? min(p.count[row], p.K) : p.K;
      for (int j0 = 0; j0 < cnt_in; j0 += 32) {
        const int j = j0 + lane;
        const int m = j < cnt_in ? p.idx[row * p.K + j] : -1;
        const bool good = j < cnt_in && m >= 0 && m < nc;
        const unsigned bal = __ballot_sync(0xffffffffu, good);
        const int at = base + __popc(bal & ((1u << lane) - 1u));
        if (good && at < kMaxSel) s_blk[item][at] = m;
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
          for (int j = lane; j < base; j += 32) mx = fmaxf(mx, srow[s_blk[item][j]]);
          mx = warp_max(mx);
          for (int j = lane; j < base; j += 32) acc += exp2f((srow[s_blk[item][j]] - mx) * kSLog2e);
        }
        acc = warp_sum(acc);
        const float lnorm = mx == -INFINITY ? 0.f : mx + logf(acc);
        for (int j = lane; j < base; j += 32) s_bias[item][j] = (srow[s_blk[item][j]] - lnorm) * kSLog2e;
      } else {
        for (int j = lane; j < base; j += 32) s_bias[item][j] = 0.f;
      }
    }
    if (lane == 0) s_cnt[item] = base;
  }
  if (tid == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&k_full[i], 1);
      mbar_init(&k_empty[i], 1);
      mbar_init(&v_full[i], 1);
      mbar_init(&v_empty[i], 1);
      mbar_init(&s_full[i], 1);
      mbar_init(&s_free[i], 128);
      mbar_init(&p_full[i], 128);
      mbar_init(&o_done[i], 1);
    }
    mbar_init(fin, 1);
    fence_mbar_init();
    s_abort = 0;
  }
  if (warp == 9) {  // pair pr: S at 256 pr, O at 256 pr + 128
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
  const int nst = max(max(s_cnt[0], s_cnt[1]), max(s_cnt[2], s_cnt[3])) + 1;  // steps per pair
  const int ng = 2 * nst;                                                   // pair-steps
  const uint32_t tmem = s_tmem;
  // step j of item: history block, filler (masked) or the diagonal block (last step)
  auto step_block = [&](int item, int j) {
    const int u = item_unit(item);
    return j < s_cnt[item] ? s_blk[item][j] : (u < p.U ? u : 0);
  };
  auto qpair = [&](int pr) { return smem + L::kQ + pr * L::kPair; };
  auto kslot = [&](int sl) { return smem + L::kK + sl * L::kPair; };
  auto vtile = [&](int sl, int it) { return smem + L::kV + (2 * sl + it) * L::kTile; };
  auto ptile = [&](int pr, int it) { return smem + L::kP + (2 * pr + it) * L::kPBytes; };

  if (warp == 8 || warp == 10) {
    // ------------------------------------------- producers: warp 8 Q and K, warp 10 V
    if (lane == 0) {
      const bool is_k = warp == 8;
      if (is_k) {  // both pairs' queries, 16-row boxes into the accumulator lane order
        for (int pr = 0; pr < 2; ++pr) {
          mbar_arrive_expect_tx(&q_full[pr], L::kPair);
          for (int it = 0; it < 2; ++it) {
            const int item = 2 * pr + it;
            const int u = min(item_unit(item), p.U - 1);
            const int y = ((bi * p.Hq + item_head(item)) * p.n) + u * kU;
            for (int hf = 0; hf < D / 64; ++hf)
              for (int b4 = 0; b4 < 4; ++b4)
                tc::tma_load_2d(qpair(pr) + hf * 16384 + (32 * b4 + 16 * it) * 128, &tmq,
                                hf * 64, y + 16 * b4, &q_full[pr]);
          }
        }
      }
      uint64_t* full = is_k ? k_full : v_full;
      uint64_t* empty = is_k ? k_empty : v_empty;
      const CUtensorMap* tm = is_k ? &tmk : &tmv;
      int issued = 0;
      bool ok = true;
      for (int g = 0; g < ng; ++g) {
        const int sl = g & 1, pr = g & 1, j = g >> 1;
        if (g >= 2 && !mbar_wait_bounded(&empty[sl], ((g >> 1) - 1) & 1)) { ok = false; break; }
        mbar_arrive_expect_tx(&full[sl], L::kPair);
        for (int it = 0; it < 2; ++it) {
          const int y = ((bi * p.Hk + kh) * p.n) + step_block(2 * pr + it, j) * kU;
          unsigned char* dst = is_k ? kslot(sl) + it * 8192 : vtile(sl, it);
          for (int hf = 0; hf < D / 64; ++hf)
            tc::tma_load_2d(dst + hf * (is_k ? 16384 : 8192), tm, hf * 64, y, &full[sl]);
        }
        issued = g + 1;
      }
      if (!ok) {
        s_abort = 1;
        for (int g = max(0, issued - 2); g < issued; ++g)
          (void)mbar_wait_bounded(&full[g & 1], (g >> 1) & 1, 1u << 16);
      }
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = tc::idesc_bf16(128, 128, false, false);
      constexpr uint32_t idO = tc::idesc_bf16(64, D, false, true);
      auto issue_s = [&](int g) {
        const int pr = g & 1, sl = g & 1;
        const uint32_t d_s = tmem + (uint32_t)(pr * 256);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const int hf = kk >> 2, off = (kk & 3) * 32;
          const uint64_t a = tc::smem_desc_sw128(qpair(pr) + hf * 16384 + off, 16, 1024);
          const uint64_t b = tc::smem_desc_sw128(kslot(sl) + hf * 16384 + off, 16, 1024);
          tc::mma_f16_ss(d_s, a, b, idS, kk > 0);
        }
        tc::mma_commit(&s_full[pr]);
        tc::mma_commit(&k_empty[sl]);
      };
      bool ok = mbar_wait_bounded(&q_full[0], 0) && mbar_wait_bounded(&q_full[1], 0);
      // S of both pairs' first steps
      for (int g = 0; ok && g < min(2, ng); ++g) {
        ok = mbar_wait_bounded(&k_full[g & 1], 0);
        if (!ok) break;
        tc::fence_after_sync();
        issue_s(g);
      }
      for (int g = 0; ok && g < ng; ++g) {
        const int pr = g & 1, j = g >> 1, sl = g & 1;
        // P V of pair-step g once its softmax has written P
        ok = mbar_wait_bounded(&p_full[pr], j & 1) && mbar_wait_bounded(&v_full[sl], j & 1);
        if (!ok) break;
        tc::fence_after_sync();
        for (int it = 0; it < 2; ++it) {
          const uint32_t d_o = tmem + (uint32_t)(pr * 256 + 128) + ((uint32_t)(16 * it) << 16);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {  // 64 keys in steps of 16
            const uint64_t a = tc::smem_desc_sw128(ptile(pr, it) + kk * 32, 16, 1024);
            const uint64_t b = tc::smem_desc_sw128(vtile(sl, it) + kk * 2048, 8192, 1024);
            tc::mma_f16_ss(d_o, a, b, idO, (j > 0 || kk > 0) ? 1u : 0u);
          }
        }
        tc::mma_commit(&o_done[pr]);
        tc::mma_commit(&v_empty[sl]);
        // the next S of this pair: its softmax has read S (s_free) and its K block has landed
        if (g + 2 < ng) {
          const int g2 = g + 2;
          ok = mbar_wait_bounded(&s_free[pr], j & 1) &&
               mbar_wait_bounded(&k_full[g2 & 1], (g2 >> 1) & 1);
          if (!ok) break;
          tc::fence_after_sync();
          issue_s(g2);
        }
      }
      if (!ok) s_abort = 1;
      tc::mma_commit(fin);
      if (!mbar_wait_bounded(fin, 0)) s_abort = 1;
    }
  } else {
    // ---------------------------------------------------- softmax: warps 0-3 pair 0, 4-7 pair 1
    const int pr = warp >> 2, w4 = warp & 3;
    const int it = lane >> 4;                 // unit of this thread's row within the pair
    const int item = 2 * pr + it;
    const int r = 16 * w4 + (lane & 15);      // row within the unit
    const int u = item_unit(item);
    const bool live_item = u < p.U;
    const int i = u * kU + r;                 // query position
    const uint32_t lane_base = (uint32_t)(32 * w4) << 16;
    const uint32_t s_col = (uint32_t)(pr * 256 + 64 * it);  // this unit's 64 score columns
    const uint32_t o_col = (uint32_t)(pr * 256 + 128);
    const float qk_scale = rsqrtf((float)D) * kSLog2e;
    const bool outer = p.gate == BSA_GATE_OUTER;
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int j = 0; j < nst && ok; ++j) {
      ok = __all_sync(0xffffffffu, mbar_wait_bounded(&s_full[pr], j & 1));
      if (!ok) break;
      tc::fence_after_sync();
      const bool is_cur = j == nst - 1;
      const bool filler = !is_cur && j >= s_cnt[item];
      const float lg = (!is_cur && !filler) ? s_bias[item][j] : 0.f;  // log2 g_m
      const float bias = outer ? 0.f : lg;
      const float vs = outer ? tc::ex2_approx(lg) : 1.f;
      // keys visible to the row: all of a history block, none of a filler, c <= r on the diagonal
      uint64_t keep = filler ? 0ull : ~0ull;
      if (is_cur) keep &= r >= 63 ? ~0ull : ((2ull << r) - 1ull);
      // pass 1: the row maximum over both 32-column halves
      float mx = -INFINITY;
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        float x[32];
        tc::tmem_ld32(tmem + lane_base + s_col + (uint32_t)(32 * hh), x);
        tc::tmem_wait_ld();
        tc::reg_fence(x);
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          const float z = ((keep >> (32 * hh + c)) & 1ull) ? fmaf(x[c], qk_scale, bias) : -INFINITY;
          mx = fmaxf(mx, z);
        }
      }
      const float m_new = fmaxf(m_run, mx);
      const bool rescale = m_run != -INFINITY && m_new > m_run + kSRescale;
      float corr = 1.f;
      if (rescale) corr = tc::ex2_approx(m_run - m_new);
      if (rescale || m_run == -INFINITY) m_run = m_new;
      const float m_use = m_run == -INFINITY ? 0.f : m_run;
      // O may be rescaled only after P_{j-1} V_{j-1} completed; the pair's P tile may be
      // rewritten only then as well (one P buffer per pair)
      const bool any_rescale = j > 0 && __any_sync(0xffffffffu, rescale);
      if (j > 0) {
        ok = __all_sync(0xffffffffu, mbar_wait_bounded(&o_done[pr], (j - 1) & 1));
        if (!ok) break;
        tc::fence_after_sync();
      }
      if (any_rescale) {
        if (!rescale) corr = 1.f;
#pragma unroll
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
      // pass 2: exponentials, row sum, P (128-byte swizzled K-major [64 x 64]) half by half
      float sum = 0.f;
      unsigned char* prow = ptile(pr, it);
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        float x[32];
        tc::tmem_ld32(tmem + lane_base + s_col + (uint32_t)(32 * hh), x);
        tc::tmem_wait_ld();
        tc::reg_fence(x);
        if (hh == 1) {  // both halves read: the score tile is free for the next S
          tc::fence_before_sync();
          mbar_arrive(&s_free[pr]);
        }
        uint32_t pk[16];
#pragma unroll
        for (int c = 0; c < 32; c += 2) {
          const bool k0 = (keep >> (32 * hh + c)) & 1ull, k1 = (keep >> (32 * hh + c + 1)) & 1ull;
          const float p0 = k0 ? tc::ex2_approx(fmaf(x[c], qk_scale, bias) - m_use) : 0.f;
          const float p1 = k1 ? tc::ex2_approx(fmaf(x[c + 1], qk_scale, bias) - m_use) : 0.f;
          sum += p0 + p1;
          const __nv_bfloat162 h2 = __floats2bfloat162_rn(p0 * vs, p1 * vs);
          pk[c / 2] = *reinterpret_cast<const uint32_t*>(&h2);
        }
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
          const uint4 w4v = make_uint4(pk[4 * ch], pk[4 * ch + 1], pk[4 * ch + 2], pk[4 * ch + 3]);
          *reinterpret_cast<uint4*>(prow + tc::sw128_offset(r, 4 * hh + ch)) = w4v;
        }
      }
      l_run = l_run * corr + sum;
      fence_proxy_async();
      tc::fence_before_sync();
      mbar_arrive(&p_full[pr]);
    }
    // epilogue: O / l (and lse) once the pair's last P V completed
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait_bounded(&o_done[pr], (nst - 1) & 1));
    if (ok) {
      tc::fence_after_sync();
      const bool live = live_item && i < p.n;
      const size_t orow = ((size_t)bi * p.Hq + item_head(item)) * p.n + i;
      const float inv = 1.f / l_run;
      __nv_bfloat16* op = static_cast<__nv_bfloat16*>(p.o) + orow * D;
      // this thread's accumulator row sits in lanes 16 it + (lane & 15) of its sub-partition
      for (int c0 = 0; c0 < D; c0 += 32) {
        float ov[32];
        tc::tmem_ld32(tmem + lane_base + o_col + (uint32_t)c0, ov);
        tc::tmem_wait_ld();
        if (live) {
#pragma unroll
          for (int c = 0; c < 32; c += 8) {
            uint4 w4v;
            __nv_bfloat162 h;
            h = __floats2bfloat162_rn(ov[c] * inv, ov[c + 1] * inv);
            w4v.x = *reinterpret_cast<uint32_t*>(&h);
            h = __floats2bfloat162_rn(ov[c + 2] * inv, ov[c + 3] * inv);
            w4v.y = *reinterpret_cast<uint32_t*>(&h);
            h = __floats2bfloat162_rn(ov[c + 4] * inv, ov[c + 5] * inv);
            w4v.z = *reinterpret_cast<uint32_t*>(&h);
            h = __floats2bfloat162_rn(ov[c + 6] * inv, ov[c + 7] * inv);
            w4v.w = *reinterpret_cast<uint32_t*>(&h);
            *reinterpret_cast<uint4*>(op + c0 + c) = w4v;
          }
        }
      }
      if (live && p.lse) p.lse[orow] = (m_run + log2f(l_run)) * kSLn2;
    }
    if (!ok) s_abort = 1;
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
  const dim3 grid((p.U + 1) / 2, p.Hq / 2, p.B);
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
