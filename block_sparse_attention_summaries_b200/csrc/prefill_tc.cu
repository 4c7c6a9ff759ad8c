// FreeSolo long branch over unit block unions, and the SAS gate gradient, on the 5th-generation
// tensor cores (tcgen05 + TMEM + TMA).
//
// [FreeSolo] "How it works": the NoPE long branch attends each query to the tokens of its top-K
// cells, and the two branches mix through alpha_h.  For cells other than 16, 32 or 64 tokens this
// runs per 64-query unit over the sorted union of the 64-key blocks that hold the unit's rows'
// cells, with a per-row mask keeping only the row's own cells (the cell-major kernel of fs_long.cu
// takes cells of 16, 32 and 64).
//
// One CTA takes two units (units 2up and 2up+1 of head h) and runs them in lockstep over their
// union lists.  Each unit is an M = 64 tile; the two tiles' accumulators occupy complementary
// halves of the TMEM lanes (rows of unit 0 in lanes 0-15 of every 32-lane sub-partition, unit 1 in
// lanes 16-31), so the four softmax warps own one row per thread.
//
//   warp 4  (1 thread): TMA producer: Q tiles once, then per step the K blocks of both units
//                       (128-byte swizzled 64x64 boxes) into their ring.
//   warp 5  (1 thread): MMA issuer: S_j = Q K_j^T into a double-buffered TMEM score tile, issued one
//                       step ahead; O += P_j V_j once the softmax has written P_j.
//   warp 6  (1 thread): V producer.
//   warps 0-3 (128):    softmax: tcgen05.ld of the score row, the row's cell mask, online max with
//                       lazy rescaling (O in TMEM is rescaled only when the row max grows by more
//                       than 2^8), P written to shared memory in the MMA's swizzled layout;
//                       epilogue: o = (1 - alpha) o_short + alpha o_long.
// Every mbarrier wait is bounded; on timeout the CTA records it, skips the rest of its work and
// still reaches its final barrier and TMEM release.  The SAS forward has its own kernel
// (sas_fwd_tc.cu).
#include <cudaTypedefs.h>

#include <mutex>

#include "tc_common.cuh"

namespace bsa {
namespace {

constexpr int kTiles = 64;         // queries per unit = keys per block
constexpr int kMaxKtc = 64;        // selected history blocks per unit
constexpr int kThreadsTc = 192;    // gate gradient: 4 reduction warps + producer + MMA
constexpr int kThreadsFwd = 224;   // forward: 4 softmax warps + K producer + MMA + V producer
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescale = 8.f;    // lazy rescale threshold (log2 units)

struct TcParams {
  int B, Hq, Hk, n, U;
  void* o;
  int* status;
  // each unit walks the sorted union of the 64-key blocks that hold its rows' selected cells; a
  // row sees only the keys of its own cells
  const int* ulist;    // [B * Hq * U][ucap] union blocks of each unit
  const int* ucnt;     // [B * Hq * U]
  int ucap;
  const int* sel;      // [B, Hq, n, ksel] selected cells, -1 padded
  const int* sel_cnt;  // [B, Hq, n] or null
  int ksel, cell;
  const float* alpha;  // [Hq] mixing weight of the long branch
};

template <int D>
struct TcSmem {
  static constexpr int kHalves = D / 64;
  static constexpr int kTileBytes = kTiles * D * 2;  // one [64 x D] bf16 tile
  // K ring slots are freed when S_j completes, V ring slots when P_j V_j completes; gathers take
  // a few microseconds to land, so the rings run as deep as shared memory allows
  static constexpr int kKSlots = D == 64 ? 6 : 3;
  static constexpr int kVSlots = D == 64 ? 4 : 2;
  // queries: [half][128 rows x 128 B], unit it's row r at row 32 (r / 16) + 16 it + r % 16, the
  // lane order of the M = 64 accumulators; K slot: [half][128 rows], unit 0 rows 0-63, unit 1
  // rows 64-127 -- so one M = 128, N = 128 MMA chain gives both units' scores
  static constexpr int kQ = 0;
  static constexpr int kK = 2 * kTileBytes;          // [kKSlots][half][2 units x 64 rows]
  static constexpr int kV = kK + kKSlots * 2 * kTileBytes;  // [kVSlots][2 units]
  static constexpr int kP = kV + kVSlots * 2 * kTileBytes;  // [2 buffers][2 units] [64 x 64] bf16
  static constexpr int kPBytes = kTiles * 64 * 2;
  static constexpr int kTotal = kP + 4 * kPBytes;  // mbarriers live in static shared memory
};

template <int D>
__global__ void __launch_bounds__(kThreadsFwd, 1)
    long_union_tc_kernel(const __grid_constant__ CUtensorMap tmq,
                      const __grid_constant__ CUtensorMap tmk,
                      const __grid_constant__ CUtensorMap tmv, const TcParams p) {
  using L = TcSmem<D>;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  // 1024-byte alignment of the swizzled tiles
  unsigned char* smem = smem_align1024(smem_raw);
  __shared__ __align__(8) uint64_t bars[30];
  uint64_t* q_full = bars + 0;
  uint64_t* k_full = bars + 1;    // [kKSlots <= 6]
  uint64_t* k_empty = bars + 7;   // [kKSlots]
  uint64_t* v_full = bars + 13;   // [kVSlots <= 4]
  uint64_t* v_empty = bars + 17;  // [kVSlots]
  uint64_t* s_full = bars + 21;   // [2]
  uint64_t* s_free = bars + 23;   // [2]
  uint64_t* p_full = bars + 25;   // [2] per P buffer
  uint64_t* o_done = bars + 27;   // [2] P_j V_j done, per P buffer
  uint64_t* fin = bars + 29;

  __shared__ uint32_t s_tmem;
  __shared__ int s_cnt[2];
  __shared__ int s_abort;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int bi = blockIdx.z;
  // the two work items: units 2up, 2up+1 of head h
  const int hq[2] = {(int)blockIdx.y, (int)blockIdx.y};
  const int uu[2] = {2 * (int)blockIdx.x, 2 * (int)blockIdx.x + 1};
  const bool item_ok[2] = {uu[0] < p.U, uu[1] < p.U};
  const int G = p.Hq / p.Hk;
  const int kh = hq[0] / G;

  // ---- prologue: the sizes of both items' union lists (warps 0 and 1) ---------------------
  if (warp < 2 && lane == 0) {
    const int it = warp;
    const size_t urow = ((size_t)bi * p.Hq + hq[it]) * p.U + uu[it];
    s_cnt[it] = item_ok[it] ? min(p.ucnt[urow], p.ucap) : 0;
  }
  if (tid == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < L::kKSlots; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&k_empty[i], 1);
    }
    for (int i = 0; i < L::kVSlots; ++i) {
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
  if (warp == 5) {  // S: 2 x 128 columns, O: D columns at 256
    tc::tmem_alloc(&s_tmem, 512);
    tc::tmem_relinquish();
  }
  if (warp == 4 && lane == 0) {
    tc::prefetch_tmap(&tmq);
    tc::prefetch_tmap(&tmk);
    tc::prefetch_tmap(&tmv);
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const int steps = max(s_cnt[0], s_cnt[1]);
  const uint32_t tmem = s_tmem;
  // step j of unit it: a block of its union, or a filler (fully masked) past the list's end
  auto step_block = [&](int it, int j) {
    const size_t urow = ((size_t)bi * p.Hq + hq[it]) * p.U + uu[it];
    return j < s_cnt[it] ? p.ulist[urow * p.ucap + j] : 0;
  };

  auto kslot = [&](int slot) { return smem + L::kK + slot * 2 * L::kTileBytes; };
  auto vtile = [&](int slot, int it) { return smem + L::kV + (2 * slot + it) * L::kTileBytes; };
  auto ptile = [&](int buf, int it) { return smem + L::kP + (2 * buf + it) * L::kPBytes; };

  if (warp == 4 || warp == 6) {
    // ------------------------------------------------ TMA producers: warp 4 Q and K, warp 6 V
    // Each runs ahead as far as its ring allows: K_j once S_{j-3} completed, V_j once
    // P_{j-2} V_{j-2} completed.
    if (lane == 0 && steps > 0) {
      const bool is_k = warp == 4;
      if (is_k) {  // 16-row boxes into the accumulator lane order
        mbar_arrive_expect_tx(q_full, 2 * L::kTileBytes);
        for (int it = 0; it < 2; ++it) {
          const int y = ((bi * p.Hq + hq[it]) * p.n) + uu[it] * kTiles;
          for (int hf = 0; hf < L::kHalves; ++hf)
            for (int b4 = 0; b4 < 4; ++b4)
              tc::tma_load_2d(smem + L::kQ + hf * 16384 + (32 * b4 + 16 * it) * 128, &tmq,
                              hf * 64, y + 16 * b4, q_full);
        }
      }
      const int nslots = is_k ? L::kKSlots : L::kVSlots;
      uint64_t* full = is_k ? k_full : v_full;
      uint64_t* empty = is_k ? k_empty : v_empty;
      const CUtensorMap* tm = is_k ? &tmk : &tmv;
      int issued = 0;
      for (int j = 0; j < steps; ++j) {
        const int sl = j % nslots;
        if (j >= nslots && !mbar_wait_bounded(&empty[sl], ((j / nslots) - 1) & 1)) {
          s_abort = 1;
          break;
        }
        mbar_arrive_expect_tx(&full[sl], 2 * L::kTileBytes);
        for (int it = 0; it < 2; ++it) {
          const int y = ((bi * p.Hk + kh) * p.n) + step_block(it, j) * kTiles;
          unsigned char* dst = is_k ? kslot(sl) + it * 8192 : vtile(sl, it);
          for (int hf = 0; hf < L::kHalves; ++hf)
            tc::tma_load_2d(dst + hf * (is_k ? 16384 : 8192), tm, hf * 64, y, &full[sl]);
        }
        issued = j + 1;
      }
      if (s_abort)  // loads still in flight land before the CTA leaves
        for (int j = max(0, issued - nslots); j < issued; ++j)
          (void)mbar_wait_bounded(&full[j % nslots], (j / nslots) & 1, 1u << 16);
    }
  } else if (warp == 5) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0 && steps > 0) {
      constexpr uint32_t idS = tc::idesc_bf16(128, 128, false, false);
      constexpr uint32_t idO = tc::idesc_bf16(64, D, false, true);
      // S_j = [Q_0; Q_1] [K_0; K_1]^T as one M = 128, N = 128 chain (full tensor-core rate);
      // the cross products Q_0 K_1^T, Q_1 K_0^T land in columns the softmax ignores
      auto issue_s = [&](int j) {
        const int st = j & 1, sl = j % L::kKSlots;
        const uint32_t d_s = tmem + (uint32_t)(st * 128);
        const unsigned char* kb = kslot(sl);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const int hf = kk >> 2, off = (kk & 3) * 32;
          const uint64_t a = tc::smem_desc_sw128(smem + L::kQ + hf * 16384 + off, 16, 1024);
          const uint64_t b = tc::smem_desc_sw128(kb + hf * 16384 + off, 16, 1024);
          tc::mma_f16_ss(d_s, a, b, idS, kk > 0);
        }
        tc::mma_commit(&s_full[st]);
        tc::mma_commit(&k_empty[sl]);
      };
      bool ok = mbar_wait_bounded(q_full, 0) && mbar_wait_bounded(&k_full[0], 0);
      if (ok) {
        tc::fence_after_sync();
        issue_s(0);
      }
      for (int j = 0; ok && j < steps; ++j) {
        if (j + 1 < steps) {  // S_{j+1} one step ahead of the softmax
          const int j1 = j + 1;
          ok = mbar_wait_bounded(&k_full[j1 % L::kKSlots], (j1 / L::kKSlots) & 1);
          if (ok && j1 >= 2) ok = mbar_wait_bounded(&s_free[j1 & 1], ((j1 >> 1) - 1) & 1);
          if (!ok) break;
          tc::fence_after_sync();
          issue_s(j1);
        }
        const int pb = j & 1;
        ok = mbar_wait_bounded(&p_full[pb], (j >> 1) & 1) &&
             mbar_wait_bounded(&v_full[j % L::kVSlots], (j / L::kVSlots) & 1);
        if (!ok) break;
        tc::fence_after_sync();
        for (int it = 0; it < 2; ++it) {
          const uint32_t d_o = tmem + 256u + ((uint32_t)(16 * it) << 16);
          const unsigned char* vt = vtile(j % L::kVSlots, it);
          const unsigned char* pt = ptile(pb, it);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {  // 64 keys in steps of 16
            const uint64_t a = tc::smem_desc_sw128(pt + kk * 32, 16, 1024);
            const uint64_t b = tc::smem_desc_sw128(vt + kk * 2048, 8192, 1024);
            tc::mma_f16_ss(d_o, a, b, idO, (j > 0 || kk > 0) ? 1u : 0u);
          }
        }
        tc::mma_commit(&o_done[pb]);
        tc::mma_commit(&v_empty[j % L::kVSlots]);
      }
      if (!ok) s_abort = 1;
      // drain: every MMA this thread issued has completed before TMEM is released
      tc::mma_commit(fin);
      if (!mbar_wait_bounded(fin, 0)) s_abort = 1;
    }
  } else {
    // ---------------------------------------------------------------- softmax warps 0-3
    const int it = lane >> 4;                  // item of this thread's row
    const int r = 16 * warp + (lane & 15);     // row within the unit
    const int i = uu[it] * kTiles + r;         // query position
    const uint32_t lane_base = (uint32_t)(32 * warp) << 16;
    const float qk_scale = rsqrtf((float)D) * kLog2e;
    // this row's cells that lie wholly at or before it (never a future key)
    constexpr int kSelMax = 8;
    int my_cells[kSelMax];
    int nmine = 0;
#pragma unroll
    for (int k = 0; k < kSelMax; ++k) my_cells[k] = -1;
    if (item_ok[it] && i < p.n) {
      const size_t qrow = ((size_t)bi * p.Hq + hq[it]) * p.n + i;
      const int cnt = p.sel_cnt ? min(p.sel_cnt[qrow], p.ksel) : p.ksel;
#pragma unroll
      for (int k = 0; k < kSelMax; ++k) {
        const int c = k < cnt ? p.sel[qrow * p.ksel + k] : -1;
        if (c >= 0 && (long long)(c + 1) * p.cell <= i + 1) {
          my_cells[k] = c;
          ++nmine;
        }
      }
    }
    const uint64_t cell_bits = p.cell >= 64 ? ~0ull : ((1ull << p.cell) - 1ull);
    // per cell of this row, once: its 64-key block and its keys' bits in that block (a cell
    // never straddles two blocks: its size divides 64); block -1 for an empty slot
    int cell_blk[kSelMax];
    uint64_t cell_keys[kSelMax];
#pragma unroll
    for (int k = 0; k < kSelMax; ++k) {
      const long long first = (long long)my_cells[k] * p.cell;
      cell_blk[k] = my_cells[k] >= 0 ? (int)(first / kTiles) : -1;
      cell_keys[k] = my_cells[k] >= 0 ? cell_bits << (int)(first % kTiles) : 0ull;
    }
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    // the step's block index is read one step ahead (in the long branch it comes from global
    // memory and its latency would otherwise sit on every step)
    int blk_next = steps > 0 ? step_block(it, 0) : 0;
    for (int j = 0; j < steps && ok; ++j) {
      const int st = j & 1;
      const int blk = blk_next;
      if (j + 1 < steps) blk_next = step_block(it, j + 1);
      ok = __all_sync(0xffffffffu, mbar_wait_bounded(&s_full[st], (j >> 1) & 1));
      if (!ok) break;
      tc::fence_after_sync();
      // keys of this block the row may see: the keys of the row's own cells (none for a filler)
      const bool filler = j >= s_cnt[it];
      const float bias = 0.f;
      uint64_t keep = filler ? 0ull : ~0ull;
      if (!filler) {
        uint64_t mine = 0ull;
#pragma unroll
        for (int k = 0; k < kSelMax; ++k) mine |= cell_blk[k] == blk ? cell_keys[k] : 0ull;
        keep &= mine;
      }
      // a warp none of whose rows sees a key of this block skips the scores entirely (most steps
      // of the long branch, where a row's few cells sit in a handful of the unit's blocks)
      const bool warp_live = __any_sync(0xffffffffu, keep != 0ull);
      // this row's 64 scores: columns 64 it .. 64 it + 63 of the score tile (the load is
      // warp-wide, so both units' column ranges are read and each lane keeps its own)
      float x[64];
      if (warp_live) {
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          float t[32];
          tc::tmem_ld32(tmem + lane_base + (uint32_t)(st * 128 + 32 * hh), x + 32 * hh);
          tc::tmem_ld32(tmem + lane_base + (uint32_t)(st * 128 + 64 + 32 * hh), t);
          tc::tmem_wait_ld();
          tc::reg_fence(t);
#pragma unroll
          for (int c = 0; c < 32; ++c) x[32 * hh + c] = it ? t[c] : x[32 * hh + c];
        }
      }
      tc::fence_before_sync();
      mbar_arrive(&s_free[st]);
      float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
      if (warp_live) {
        if (p.cell >= 8) {
          // cell masks are whole 8-key chunks: per chunk a (scale, bias) of (0, -inf) masks it
          // with the same one FMA per key as the unmasked path (scores are finite); every lane
          // takes this path, so a warp whose rows see different cells does not diverge
#pragma unroll
          for (int ch = 0; ch < 8; ++ch) {
            const bool kc = ((keep >> (8 * ch)) & 0xFFull) != 0ull;
            const float sc_c = kc ? qk_scale : 0.f, b_c = kc ? bias : -INFINITY;
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const int c = 8 * ch + e;
              x[c] = fmaf(x[c], sc_c, b_c);
              mx4[c & 3] = fmaxf(mx4[c & 3], x[c]);
            }
          }
        } else if (keep == ~0ull) {
#pragma unroll
          for (int c = 0; c < 64; ++c) {
            x[c] = fmaf(x[c], qk_scale, bias);
            mx4[c & 3] = fmaxf(mx4[c & 3], x[c]);
          }
        } else {
#pragma unroll
          for (int c = 0; c < 64; ++c) {
            x[c] = ((keep >> c) & 1ull) ? fmaf(x[c], qk_scale, bias) : -INFINITY;
            mx4[c & 3] = fmaxf(mx4[c & 3], x[c]);
          }
        }
      }
      const float mx = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3]));
      const float m_new = fmaxf(m_run, mx);
      // the first finite max needs no O scaling (the row's O and l are still 0); later ones
      // rescale O only when the max grows by more than 2^8
      const bool rescale = m_run != -INFINITY && m_new > m_run + kRescale;
      float corr = 1.f;
      if (rescale) corr = tc::ex2_approx(m_run - m_new);
      if (rescale || m_run == -INFINITY) m_run = m_new;
      // masked keys hold -inf and give 2^-inf = 0; a row with nothing seen yet subtracts 0
      const float m_use = m_run == -INFINITY ? 0.f : m_run;
      float sum4[4] = {0.f, 0.f, 0.f, 0.f};
      uint32_t pk[32];
      if (warp_live) {
#pragma unroll
        for (int c = 0; c < 64; c += 2) {
          const float p0 = tc::ex2_approx(x[c] - m_use);
          const float p1 = tc::ex2_approx(x[c + 1] - m_use);
          sum4[(c >> 1) & 3] += p0 + p1;
          const __nv_bfloat162 h2 = __floats2bfloat162_rn(p0, p1);
          pk[c / 2] = *reinterpret_cast<const uint32_t*>(&h2);
        }
      } else {
#pragma unroll
        for (int c = 0; c < 32; ++c) pk[c] = 0u;
      }
      const float sum = (sum4[0] + sum4[1]) + (sum4[2] + sum4[3]);
      l_run = l_run * corr + sum;
      // O may be rescaled only after P_{j-1} V_{j-1} completed; P buffer j & 1 may be rewritten
      // once P_{j-2} V_{j-2} completed (implied by the former)
      const bool any_rescale = j > 0 && __any_sync(0xffffffffu, rescale);
      if (any_rescale) {
        ok = __all_sync(0xffffffffu, mbar_wait_bounded(&o_done[(j - 1) & 1], ((j - 1) >> 1) & 1));
      } else if (j >= 2) {
        ok = __all_sync(0xffffffffu, mbar_wait_bounded(&o_done[j & 1], ((j - 2) >> 1) & 1));
      }
      if (!ok) break;
      tc::fence_after_sync();
      {
        // O row *= corr; the TMEM round trip is warp-wide (.sync.aligned), lanes that keep their
        // max multiply by 1
        if (any_rescale) {
          if (!rescale) corr = 1.f;
          for (int c0 = 0; c0 < D; c0 += 32) {
            float ov[32];
            tc::tmem_ld32(tmem + lane_base + 256u + (uint32_t)c0, ov);
            tc::tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 32; ++c) ov[c] *= corr;
            tc::tmem_st32(tmem + lane_base + 256u + (uint32_t)c0, ov);
          }
          tc::tmem_wait_st();
        }
      }
      // P row -> shared memory, 128-byte swizzled K-major [64 x 64]
      unsigned char* prow = ptile(j & 1, it);
#pragma unroll
      for (int ch = 0; ch < 8; ++ch) {
        const uint4 w4 = make_uint4(pk[4 * ch], pk[4 * ch + 1], pk[4 * ch + 2], pk[4 * ch + 3]);
        *reinterpret_cast<uint4*>(prow + tc::sw128_offset(r, ch)) = w4;
      }
      fence_proxy_async();
      tc::fence_before_sync();
      mbar_arrive(&p_full[j & 1]);
    }
    // epilogue (nothing to do without a step: the long branch of units that selected nothing)
    if (ok && steps > 0)
      ok = __all_sync(0xffffffffu,
                      mbar_wait_bounded(&o_done[(steps - 1) & 1], ((steps - 1) >> 1) & 1));
    if (ok && steps > 0) {
      tc::fence_after_sync();
      // the long branch mixes into the short branch already in o, for rows that saw a cell
      const bool live = i < p.n && item_ok[it] && nmine > 0;
      const size_t orow = ((size_t)bi * p.Hq + hq[it]) * p.n + i;
      const float a_mix = p.alpha[hq[it]];
      const float inv = a_mix / l_run;
      __nv_bfloat16* op = static_cast<__nv_bfloat16*>(p.o) + orow * D;
      for (int c0 = 0; c0 < D; c0 += 32) {
        float ov[32];
        tc::tmem_ld32(tmem + lane_base + 256u + (uint32_t)c0, ov);
        tc::tmem_wait_ld();
        if (live) {
#pragma unroll
          for (int c = 0; c < 32; c += 8) {  // o = (1 - alpha) o_short + alpha o_long
            float sh[8];
            load_vec<__nv_bfloat16, 8>(op + c0 + c, sh);
#pragma unroll
            for (int e = 0; e < 8; ++e) ov[c + e] = fmaf(ov[c + e], inv, (1.f - a_mix) * sh[e]);
            uint4 w4;
            __nv_bfloat162 h;
            h = __floats2bfloat162_rn(ov[c], ov[c + 1]);
            w4.x = *reinterpret_cast<uint32_t*>(&h);
            h = __floats2bfloat162_rn(ov[c + 2], ov[c + 3]);
            w4.y = *reinterpret_cast<uint32_t*>(&h);
            h = __floats2bfloat162_rn(ov[c + 4], ov[c + 5]);
            w4.z = *reinterpret_cast<uint32_t*>(&h);
            h = __floats2bfloat162_rn(ov[c + 6], ov[c + 7]);
            w4.w = *reinterpret_cast<uint32_t*>(&h);
            *reinterpret_cast<uint4*>(op + c0 + c) = w4;
          }
        }
      }
    } else if (steps > 0) {
      ok = false;
    }
    if (!ok) s_abort = 1;
  }

  tc::fence_before_sync();
  __syncthreads();
  if (s_abort && tid == 0) report_timeout(p.status, 3);
  if (warp == 5) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, 512);
  }
}

// ---- gate gradient on the tensor cores -----------------------------------------------------
//
// [SAS] review, "Why the four design choices matter", Eq. 5 (inner gate):
//     dg_m = sum_{i in B_m} (ptilde_i / g_m) do^T (v_i - o),
// summed over the unit's queries, in the stable form
//     dg_m = sum_q sum_{j in B_m} exp(z_qj - lse_q) (do_q . v_j - do_q . o_q),   z = q . k / sqrt(d).
// One CTA per pair of units (heads h and h+1 at unit u), rows in the lane order of the M = 64
// accumulators.  Per selected history block j the MMA thread computes Z_j = [Q_0; Q_1] [K_0; K_1]^T
// and DV_j = [dO_0; dO_1] [V_0; V_1]^T as M = 128, N = 128 chains (the cross products are never
// read) into a double-buffered TMEM pair; each reduction-warp thread reduces its row, and the 64
// rows of a unit are summed with shuffles and shared-memory atomics into dg of that block.
template <int D>
struct GgSmem {
  static constexpr int kHalves = D / 64;
  static constexpr int kTileBytes = kTiles * D * 2;
  static constexpr int kPair = 2 * kTileBytes;        // [half][2 units x 64 rows x 128 B]
  static constexpr int kQ = 0;                        // Q pair, then dO pair
  static constexpr int kStage = 2 * kPair;            // stages: K pair, V pair
  static constexpr int kStageBytes = 2 * kPair;
  static constexpr int kBars = kStage + 2 * kStageBytes;
  static constexpr int kTotal = kBars + 1024;
};

struct GgParams {
  int B, Hq, Hk, n, U, K;
  const int* idx;
  const int* count;
  int norm;
  const float* scores;
  int scores_ld;
  const void* o;
  const float* lse;
  const void* dout;
  float* dg;
  int* status;
  int outer;  // outer gate: dg_m = sum p do . v_j (no do . o term)
};

template <int D>
__global__ void __launch_bounds__(kThreadsTc, 1)
    gate_grad_tc_kernel(const __grid_constant__ CUtensorMap tmq,
                        const __grid_constant__ CUtensorMap tmdo,
                        const __grid_constant__ CUtensorMap tmk,
                        const __grid_constant__ CUtensorMap tmv, const GgParams p) {
  using L = GgSmem<D>;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = smem_align1024(smem_raw);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBars);
  uint64_t* q_full = bars + 0;
  uint64_t* kv_full = bars + 1;   // [2]
  uint64_t* kv_empty = bars + 3;  // [2]
  uint64_t* s_full = bars + 5;    // [2]
  uint64_t* s_free = bars + 7;    // [2]
  uint64_t* fin = bars + 9;

  __shared__ uint32_t s_tmem;
  __shared__ int s_blk[2][kMaxKtc];
  __shared__ int s_slot[2][kMaxKtc];
  __shared__ float s_dg[2][kMaxKtc];
  __shared__ int s_cnt[2];
  __shared__ int s_abort;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int u = blockIdx.x, hp = blockIdx.y, bi = blockIdx.z;
  const int hq[2] = {2 * hp, 2 * hp + 1};
  const int G = p.Hq / p.Hk;
  const int kh = hq[0] / G;
  const int nc = u;

  if (warp < 2) {  // block lists (with their idx slots) of both units
    const int it = warp;
    const size_t row = ((size_t)bi * p.Hq + hq[it]) * p.U + u;
    const int cnt_in = p.count ? min(p.count[row], p.K) : p.K;
    int base = 0;
    for (int j0 = 0; j0 < cnt_in; j0 += 32) {
      const int j = j0 + lane;
      const int m = j < cnt_in ? p.idx[row * p.K + j] : -1;
      const bool ok = j < cnt_in && m >= 0 && m < nc;
      const unsigned bal = __ballot_sync(0xffffffffu, ok);
      const int at = base + __popc(bal & ((1u << lane) - 1u));
      if (ok && at < kMaxKtc) {
        s_blk[it][at] = m;
        s_slot[it][at] = j;
      }
      base += __popc(bal);
    }
    base = min(base, kMaxKtc);
    for (int j = lane; j < kMaxKtc; j += 32) s_dg[it][j] = 0.f;
    if (lane == 0) s_cnt[it] = base;
  }
  if (tid == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&kv_full[i], 1);
      mbar_init(&kv_empty[i], 1);
      mbar_init(&s_full[i], 1);
      mbar_init(&s_free[i], 128);
    }
    mbar_init(fin, 1);
    fence_mbar_init();
    s_abort = 0;
  }
  if (warp == 5) {  // two stages of (Z: 128 columns, DV: 128 columns)
    tc::tmem_alloc(&s_tmem, 512);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const int steps = max(s_cnt[0], s_cnt[1]);
  const uint32_t tmem = s_tmem;
  auto step_block = [&](int it, int j) { return j < s_cnt[it] ? s_blk[it][j] : u; };
  // pairs: which 0 = Q, 1 = dO; in a stage which 0 = K, 1 = V; half hf at + hf * 16384
  auto qpair = [&](int which) { return smem + L::kQ + which * L::kPair; };
  auto stage_pair = [&](int st, int which) {
    return smem + L::kStage + st * L::kStageBytes + which * L::kPair;
  };

  if (steps > 0) {
    if (warp == 4) {
      if (lane == 0) {
        // 16-row boxes: unit it's row r at row 32 (r / 16) + 16 it + r % 16 of the pair
        mbar_arrive_expect_tx(q_full, 4 * L::kTileBytes);
        for (int it = 0; it < 2; ++it) {
          const int y = ((bi * p.Hq + hq[it]) * p.n) + u * kTiles;
          for (int hf = 0; hf < L::kHalves; ++hf)
            for (int b4 = 0; b4 < 4; ++b4) {
              const int off = hf * 16384 + (32 * b4 + 16 * it) * 128;
              tc::tma_load_2d(qpair(0) + off, &tmq, hf * 64, y + 16 * b4, q_full);
              tc::tma_load_2d(qpair(1) + off, &tmdo, hf * 64, y + 16 * b4, q_full);
            }
        }
        int issued = 0;
        for (int j = 0; j < steps; ++j) {
          const int st = j & 1;
          if (j >= 2 && !mbar_wait_bounded(&kv_empty[st], ((j >> 1) - 1) & 1)) {
            s_abort = 1;
            break;
          }
          issued = j + 1;
          mbar_arrive_expect_tx(&kv_full[st], 4 * L::kTileBytes);
          for (int it = 0; it < 2; ++it) {
            const int y = ((bi * p.Hk + kh) * p.n) + step_block(it, j) * kTiles;
            for (int hf = 0; hf < L::kHalves; ++hf) {
              const int off = hf * 16384 + it * 8192;
              tc::tma_load_2d(stage_pair(st, 0) + off, &tmk, hf * 64, y, &kv_full[st]);
              tc::tma_load_2d(stage_pair(st, 1) + off, &tmv, hf * 64, y, &kv_full[st]);
            }
          }
        }
        if (s_abort)
          for (int j = max(0, issued - 2); j < issued; ++j)
            (void)mbar_wait_bounded(&kv_full[j & 1], (j >> 1) & 1, 1u << 16);
      }
    } else if (warp == 5) {
      if (lane == 0) {
        constexpr uint32_t idS = tc::idesc_bf16(128, 128, false, false);
        bool ok = mbar_wait_bounded(q_full, 0);
        for (int j = 0; ok && j < steps; ++j) {
          const int st = j & 1;
          ok = mbar_wait_bounded(&kv_full[st], (j >> 1) & 1);
          if (ok && j >= 2) ok = mbar_wait_bounded(&s_free[st], ((j >> 1) - 1) & 1);
          if (!ok) break;
          tc::fence_after_sync();
          const uint32_t d_z = tmem + (uint32_t)(st * 256);
          const uint32_t d_dv = d_z + 128u;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const int off = (kk >> 2) * 16384 + (kk & 3) * 32;
            tc::mma_f16_ss(d_z, tc::smem_desc_sw128(qpair(0) + off, 16, 1024),
                           tc::smem_desc_sw128(stage_pair(st, 0) + off, 16, 1024), idS, kk > 0);
            tc::mma_f16_ss(d_dv, tc::smem_desc_sw128(qpair(1) + off, 16, 1024),
                           tc::smem_desc_sw128(stage_pair(st, 1) + off, 16, 1024), idS, kk > 0);
          }
          tc::mma_commit(&s_full[st]);
          tc::mma_commit(&kv_empty[st]);
        }
        if (!ok) s_abort = 1;
        tc::mma_commit(fin);
        if (!mbar_wait_bounded(fin, 0)) s_abort = 1;
      }
    } else {
      // reduction warps: thread = one query row of one unit
      const int it = lane >> 4;
      const int r = 16 * warp + (lane & 15);
      const int i = u * kTiles + r;
      const bool live = i < p.n;
      const size_t qrow = ((size_t)bi * p.Hq + hq[it]) * p.n + (live ? i : 0);
      float Di = 0.f, lse2 = 0.f;
      if (live) {
        const __nv_bfloat16* orow = static_cast<const __nv_bfloat16*>(p.o) + qrow * D;
        const __nv_bfloat16* drow = static_cast<const __nv_bfloat16*>(p.dout) + qrow * D;
        for (int c = 0; !p.outer && c < D; c += 8) {
          float a[8], bb[8];
          load_vec<__nv_bfloat16, 8>(orow + c, a);
          load_vec<__nv_bfloat16, 8>(drow + c, bb);
#pragma unroll
          for (int e = 0; e < 8; ++e) Di = fmaf(a[e], bb[e], Di);
        }
        lse2 = p.lse[qrow] * kLog2e;
      }
      const uint32_t lane_base = (uint32_t)(32 * warp) << 16;
      const float zs = rsqrtf((float)D) * kLog2e;
      bool ok = true;
      for (int j = 0; j < steps; ++j) {
        const int st = j & 1;
        ok = __all_sync(0xffffffffu, mbar_wait_bounded(&s_full[st], (j >> 1) & 1));
        if (!ok) break;
        tc::fence_after_sync();
        // this row's 64 columns of Z and DV: unit it's block (the loads are warp-wide, so each
        // lane keeps its own unit's half); 32 columns at a time
        const bool use = live && j < s_cnt[it];
        // two columns per packed FMA (exponent argument), packed add (dv - D_i) and packed FMA
        // (two pairs of partial sums)
        const uint64_t zs2 = tc::pack_f2(zs, zs), nl2 = tc::pack_f2(-lse2, -lse2);
        const uint64_t nd2 = tc::pack_f2(-Di, -Di);
        uint64_t t2[2] = {0ull, 0ull};
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          float za[32], zb[32], da[32], db[32];
          const uint32_t base = tmem + lane_base + (uint32_t)(st * 256 + 32 * hh);
          tc::tmem_ld32(base, za);
          tc::tmem_ld32(base + 64u, zb);
          tc::tmem_ld32(base + 128u, da);
          tc::tmem_ld32(base + 192u, db);
          tc::tmem_wait_ld();
          tc::reg_fence(za);
          tc::reg_fence(zb);
          tc::reg_fence(da);
          tc::reg_fence(db);
          if (use) {
#pragma unroll
            for (int c = 0; c < 32; c += 2) {
              const uint64_t z2 = tc::pack_f2(it ? zb[c] : za[c], it ? zb[c + 1] : za[c + 1]);
              const uint64_t d2 = tc::pack_f2(it ? db[c] : da[c], it ? db[c + 1] : da[c + 1]);
              float a0, a1;
              tc::unpack_f2(tc::fma_f2(z2, zs2, nl2), a0, a1);
              const uint64_t e2 = tc::pack_f2(tc::ex2_approx(a0), tc::ex2_approx(a1));
              t2[(c >> 1) & 1] = tc::fma_f2(e2, tc::add_f2(d2, nd2), t2[(c >> 1) & 1]);
            }
          }
        }
        tc::fence_before_sync();
        mbar_arrive(&s_free[st]);
        float t4[4];
        tc::unpack_f2(t2[0], t4[0], t4[1]);
        tc::unpack_f2(t2[1], t4[2], t4[3]);
        float t = (t4[0] + t4[1]) + (t4[2] + t4[3]);
        // sum over the 16 rows of this unit held by this warp, then across warps
#pragma unroll
        for (int o2 = 8; o2 > 0; o2 >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o2);
        if ((lane & 15) == 0 && j < s_cnt[it]) atomicAdd(&s_dg[it][j], t);
      }
      if (!ok) s_abort = 1;
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp < 2) {  // results of both units, every idx slot (0 where nothing was selected)
    const int it = warp;
    const size_t row = ((size_t)bi * p.Hq + hq[it]) * p.U + u;
    for (int j = lane; j < p.K; j += 32) p.dg[row * p.K + j] = 0.f;
    __syncwarp();
    for (int j = lane; j < s_cnt[it]; j += 32) p.dg[row * p.K + s_slot[it][j]] = s_dg[it][j];
  }
  if (s_abort && tid == 0) report_timeout(p.status, 4);
  if (warp == 5) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, 512);
  }
}

// ---- FreeSolo long branch: union of each unit's selected blocks -----------------------------
//
// One CTA of 64 threads per (unit of 64 queries, head, batch): every query marks the 64-key blocks
// holding its selected cells (only cells wholly at or before the query) in a bitmap; warp 0 then
// writes the marked blocks in increasing order.
__global__ void __launch_bounds__(64)
    freesolo_union_kernel(const int* __restrict__ sel, const int* __restrict__ sel_cnt, int H,
                          int n, int U, int ksel, int cell, int ucap, int* __restrict__ ucnt,
                          int* __restrict__ ulist) {
  extern __shared__ uint32_t ubits[];
  const int u = blockIdx.x, h = blockIdx.y, bi = blockIdx.z, tid = threadIdx.x;
  const int nblk = (n + kTiles - 1) / kTiles, nwords = (nblk + 31) / 32;
  for (int w = tid; w < nwords; w += 64) ubits[w] = 0u;
  __syncthreads();
  const int i = u * kTiles + tid;
  if (i < n) {
    const size_t row = ((size_t)bi * H + h) * n + i;
    const int cnt = sel_cnt ? min(sel_cnt[row], ksel) : ksel;
    for (int k = 0; k < cnt; ++k) {
      const int c = sel[row * ksel + k];
      if (c >= 0 && (long long)(c + 1) * cell <= i + 1) {
        const int blk = (int)((long long)c * cell / kTiles);
        atomicOr(&ubits[blk >> 5], 1u << (blk & 31));
      }
    }
  }
  __syncthreads();
  if (tid < 32) {
    const size_t urow = ((size_t)bi * H + h) * U + u;
    int base = 0;
    for (int w0 = 0; w0 < nwords; w0 += 32) {
      const int w = w0 + tid;
      uint32_t b = w < nwords ? ubits[w] : 0u;
      const int cw = __popc(b);
      int incl = cw;
#pragma unroll
      for (int o2 = 1; o2 < 32; o2 <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o2);
        if (tid >= o2) incl += y;
      }
      int pos = base + incl - cw;
      while (b) {
        const int t = __ffs(b) - 1;
        b &= b - 1u;
        if (pos < ucap) ulist[urow * ucap + pos] = w * 32 + t;
        ++pos;
      }
      base += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (tid == 0) ucnt[urow] = min(base, ucap);
  }
}

// ---- host side -----------------------------------------------------------------------------

PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
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

// 2-D map over a [rows, D] bf16 row-major tensor, boxes of 64 columns x box_rows rows,
// 128-byte swizzle.
bool make_map(CUtensorMap* m, const void* base, long long rows, int D, int box_rows = 64) {
  auto enc = get_encode();
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
bsa_status launch_tc(const void* q, const void* k, const void* v, const TcParams& p,
                     cudaStream_t st) {
  CUtensorMap tmq, tmk, tmv;
  if (!make_map(&tmq, q, (long long)p.B * p.Hq * p.n, D, 16) ||
      !make_map(&tmk, k, (long long)p.B * p.Hk * p.n, D) ||
      !make_map(&tmv, v, (long long)p.B * p.Hk * p.n, D))
    return BSA_ERR_CUDA;
  const int smem = TcSmem<D>::kTotal + 1024;  // + alignment slack
  auto kern = long_union_tc_kernel<D>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
      cudaSuccess) {
    (void)cudaGetLastError();
    return BSA_ERR_CUDA;
  }
  const dim3 grid((p.U + 1) / 2, p.Hq, p.B);
  kern<<<grid, kThreadsFwd, smem, st>>>(tmq, tmk, tmv, p);
  return BSA_OK;
}

template <int D>
bsa_status launch_gg(const void* q, const void* k, const void* v, const void* dout,
                     const GgParams& p, cudaStream_t st) {
  CUtensorMap tmq, tmdo, tmk, tmv;
  if (!make_map(&tmq, q, (long long)p.B * p.Hq * p.n, D, 16) ||
      !make_map(&tmdo, dout, (long long)p.B * p.Hq * p.n, D, 16) ||
      !make_map(&tmk, k, (long long)p.B * p.Hk * p.n, D) ||
      !make_map(&tmv, v, (long long)p.B * p.Hk * p.n, D))
    return BSA_ERR_CUDA;
  const int smem = GgSmem<D>::kTotal + 1024;
  auto kern = gate_grad_tc_kernel<D>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
      cudaSuccess) {
    (void)cudaGetLastError();
    return BSA_ERR_CUDA;
  }
  dim3 grid(p.U, p.Hq / 2, p.B);
  kern<<<grid, kThreadsTc, smem, st>>>(tmq, tmdo, tmk, tmv, p);
  return BSA_OK;
}

}  // namespace

bsa_status gate_grad_tc(const void* q, const void* k, const void* v, const void* o,
                        const float* lse, const void* dout, int B, int Hq, int Hk, int n, int d,
                        const int* idx, const int* count, int K, int norm, const float* scores,
                        int scores_ld, float* dg, int* status, int outer, cudaStream_t st) {
  GgParams p{};
  p.outer = outer;
  p.B = B; p.Hq = Hq; p.Hk = Hk; p.n = n; p.U = ceil_div(n, kTiles); p.K = K;
  p.idx = idx; p.count = count; p.norm = norm; p.scores = scores; p.scores_ld = scores_ld;
  p.o = o; p.lse = lse; p.dout = dout; p.dg = dg; p.status = status;
  bsa_status rc = d == 64 ? launch_gg<64>(q, k, v, dout, p, st)
                          : launch_gg<128>(q, k, v, dout, p, st);
  if (rc != BSA_OK) return rc;
  BSA_LAUNCH_CHECK();
  return BSA_OK;
}

// Long branch of the FreeSolo prefill on the tensor cores over each unit's block union, mixing
// into o.
// Workspace: union counts [B * H * U] then lists [B * H * U][ucap], ucap = min(64 * 8, blocks).
static int long_ucap(int n) { return min(64 * 8, ceil_div(n, kTiles)); }

size_t long_attn_tc_workspace(int B, int H, int n) {
  const size_t units = (size_t)B * H * ceil_div(n, kTiles);
  return units * sizeof(int) * (1 + (size_t)long_ucap(n)) + 256;
}

bool long_attn_tc_supported(int d, int cell, int ksel) {
  // cells must tile the 64-key blocks: a power of two up to 64
  return (d == 64 || d == 128) && cell >= 1 && cell <= kTiles && (kTiles % cell) == 0 &&
         ((cell & (cell - 1)) == 0) && ksel >= 1 && ksel <= 8;
}

bsa_status long_attn_tc(const void* q, const void* k, const void* v, int B, int H, int n, int d,
                        int cell, const int* sel, const int* sel_cnt, int ksel,
                        const float* alpha, void* o, void* ws, size_t ws_bytes, int* status,
                        cudaStream_t st) {
  if (!ws || ws_bytes < long_attn_tc_workspace(B, H, n)) return BSA_ERR_WORKSPACE;
  const int U = ceil_div(n, kTiles);
  const int ucap = long_ucap(n);
  int* ucnt = reinterpret_cast<int*>(align_up(reinterpret_cast<uintptr_t>(ws), (uintptr_t)256));
  int* ulist = ucnt + (size_t)B * H * U;
  const int nwords = ceil_div(ceil_div(n, kTiles), 32);
  freesolo_union_kernel<<<dim3(U, H, B), 64, nwords * sizeof(uint32_t), st>>>(
      sel, sel_cnt, H, n, U, ksel, cell, ucap, ucnt, ulist);
  BSA_LAUNCH_CHECK();
  TcParams p{};
  p.B = B; p.Hq = H; p.Hk = H; p.n = n; p.U = U;
  p.o = o; p.status = status;
  p.ulist = ulist; p.ucnt = ucnt; p.ucap = ucap;
  p.sel = sel; p.sel_cnt = sel_cnt; p.ksel = ksel; p.cell = cell; p.alpha = alpha;
  bsa_status rc = d == 64 ? launch_tc<64>(q, k, v, p, st) : launch_tc<128>(q, k, v, p, st);
  if (rc != BSA_OK) return rc;
  BSA_LAUNCH_CHECK();
  return BSA_OK;
}

bool prefill_tc_supported(bsa_dtype dt, int d, int b, int q_block, int K, int Hq, int Hk) {
  if (dt != BSA_BF16 || b != kTiles || q_block != kTiles || K > kMaxKtc) return false;
  if (d != 64 && d != 128) return false;
  const int G = Hq / Hk;
  return G % 2 == 0;  // units are paired by head within one kv group
}

bsa_status sas_fwd_tc(const void* q, const void* k, const void* v, int B, int Hq, int Hk, int n,
                      int d, const int* idx, const int* count, int K, int gate, int norm,
                      const float* scores, int scores_ld, void* o, float* lse, int* status,
                      cudaStream_t st);

bsa_status prefill_tc(const void* q, const void* k, const void* v, int B, int Hq, int Hk, int n,
                      int d, int b, const int* idx, const int* count, int K, int gate, int norm,
                      const float* scores, int scores_ld, void* o, float* lse, int* status,
                      cudaStream_t st) {
  (void)b;
  // the forward runs on the step-split kernel of sas_fwd_tc.cu, which takes every shape that
  // prefill_tc_supported admits
  return sas_fwd_tc(q, k, v, B, Hq, Hk, n, d, idx, count, K, gate, norm, scores, scores_ld, o, lse,
                    status, st);
}

}  // namespace bsa
