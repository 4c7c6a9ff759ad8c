// FreeSolo short branch on the tensor cores: RoPE sliding-window attention in 128-query tiles.
//
// [FreeSolo] summary page, "How it works": the short branch of every head is sliding-window
// attention with RoPE over a fixed window (w = 512) of the latest keys, the query's own included.
// q and k arrive already rotated (the rotation kernel runs first), so a tile is plain attention
// over a band of keys.
//
// B200 design.  A tile is 128 consecutive queries of one head (one M = 128 MMA: the accumulator
// row of query r is TMEM lane r, so each softmax thread owns one query).  Its keys are the 64-key
// blocks from floor((128 p - w + 1) / 64) to the tile's last block (10 blocks at w = 512); every
// block is loaded once for all 128 queries, S_b = Q K_b^T is one M = 128, N = 64 chain and
// O += P_b V_b one M = 128, N = d chain, and each row masks the keys outside [i - w + 1, i].
// The grid is persistent (two CTAs per SM at d = 64: 256 TMEM columns and ~105 KB of shared
// memory each), every CTA walking tiles blockIdx.x, blockIdx.x + gridDim.x, ...; its producers
// run ahead across tile boundaries (two Q buffers, rings of K and V blocks), the MMA thread issues
// S two steps ahead of the softmax (three S buffers in TMEM), and the next tile's first P V waits
// only until the epilogue has read the previous tile's O.
//   warps 0-3: softmax (row = 32 warp + lane), epilogue O / l -> o (bf16)
//   warp 4:    Q and K producer (TMA, 128-byte swizzle)      warp 6: V producer
//   warp 5:    MMA issuer (one thread)
// Every mbarrier wait is bounded; a role whose wait runs out stops, records the timeout and the
// CTA still reaches its final barrier and releases TMEM.
#include <cudaTypedefs.h>

#include <mutex>

#include "tc_common.cuh"

namespace bsa {
namespace {

constexpr int kWT = 128;        // queries per tile
constexpr int kWB = 64;         // keys per block
constexpr int kWThreads = 224;  // 4 softmax warps + Q/K producer + MMA + V producer
constexpr float kWLog2e = 1.4426950408889634f;
constexpr float kWRescale = 8.f;  // lazy O rescale threshold (log2 units)

// max(a, b, c) in one instruction (the three-input form of sm_100)
__device__ __forceinline__ float max3f(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

template <int D>
struct WinSmem {
  static constexpr int kQBytes = kWT * D * 2;    // [half][128 rows x 128 B]
  static constexpr int kBlkBytes = kWB * D * 2;  // [half][64 rows x 128 B]
  static constexpr int kKSlots = 3;
  static constexpr int kVSlots = 2;
  static constexpr int kPBytes = kWT * kWB * 2;  // [128 rows x 128 B], 128-byte swizzle
  static constexpr int kQ = 0;                   // two Q buffers
  static constexpr int kK = kQ + 2 * kQBytes;
  static constexpr int kV = kK + kKSlots * kBlkBytes;
  static constexpr int kP = kV + kVSlots * kBlkBytes;  // two P buffers
  static constexpr int kTotal = kP + 2 * kPBytes;
  static constexpr int kPerSM = D == 64 ? 2 : 1;
  static constexpr int kSBufs = 3;                          // S buffers in TMEM, 64 columns each
  static constexpr uint32_t kOCol = kSBufs * kWB;           // O: D columns after them
  static constexpr uint32_t kTmemCols = kOCol + D <= 256 ? 256 : 512;
  static_assert(kPerSM * kTmemCols <= 512, "the CTAs of an SM share its 512 TMEM columns");
};

struct WinParams {
  int BH, n, window, ntile, ntiles;
  void* o;
  int* status;
};

// (tile, step) walker shared by every role: tile t = (bh, p) in blockIdx.x + k gridDim.x order,
// steps over the tile's key blocks [first, last]
struct WinCursor {
  int t, bh, p, first, nst, s;
  __device__ void tile_setup(const WinParams& w) {
    bh = t / w.ntile;
    p = t % w.ntile;
    const int lo = kWT * p - w.window + 1;
    first = lo <= 0 ? 0 : lo / kWB;
    const int last = min((kWT * p + kWT - 1) / kWB, (w.n - 1) / kWB);
    nst = last - first + 1;
    s = 0;
  }
  __device__ bool valid(const WinParams& w) const { return t < w.ntiles; }
  __device__ void start(const WinParams& w) {
    t = blockIdx.x;
    if (valid(w)) tile_setup(w);
  }
  __device__ void next(const WinParams& w) {  // to the next step (or the first of the next tile)
    if (++s == nst) {
      t += gridDim.x;
      if (valid(w)) tile_setup(w);
    }
  }
};

template <int D>
__global__ void __launch_bounds__(kWThreads, WinSmem<D>::kPerSM)
    window_tc_kernel(const __grid_constant__ CUtensorMap tmq,
                     const __grid_constant__ CUtensorMap tmk,
                     const __grid_constant__ CUtensorMap tmv, const WinParams w) {
  using L = WinSmem<D>;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = smem_align1024(smem_raw);
  __shared__ __align__(8) uint64_t bars[26];
  uint64_t* q_full = bars + 0;    // [2]
  uint64_t* q_empty = bars + 2;   // [2]
  uint64_t* k_full = bars + 4;    // [3]
  uint64_t* k_empty = bars + 7;   // [3]
  uint64_t* v_full = bars + 10;   // [2]
  uint64_t* v_empty = bars + 12;  // [2]
  uint64_t* s_full = bars + 14;   // [3]
  uint64_t* s_free = bars + 17;   // [3]
  uint64_t* p_full = bars + 20;   // [2]
  uint64_t* o_done = bars + 22;   // [2] P_g V_g done (per P buffer)
  uint64_t* o_free = bars + 24;   // the epilogue has read O
  uint64_t* fin = bars + 25;
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&q_empty[i], 1);
      mbar_init(&v_full[i], 1);
      mbar_init(&v_empty[i], 1);
      mbar_init(&p_full[i], 128);
      mbar_init(&o_done[i], 1);
    }
    for (int i = 0; i < L::kKSlots; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&k_empty[i], 1);
    }
    for (int i = 0; i < L::kSBufs; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_free[i], 128);
    }
    mbar_init(o_free, 128);
    mbar_init(fin, 1);
    fence_mbar_init();
    s_abort = 0;
  }
  if (warp == 5) {
    tc::tmem_alloc(&s_tmem, L::kTmemCols);
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
  const uint32_t tmem = s_tmem;
  auto qbuf = [&](int b) { return smem + L::kQ + b * L::kQBytes; };
  auto kblk = [&](int slot) { return smem + L::kK + slot * L::kBlkBytes; };
  auto vblk = [&](int slot) { return smem + L::kV + slot * L::kBlkBytes; };
  auto pbuf = [&](int b) { return smem + L::kP + b * L::kPBytes; };

  if (warp == 4 || warp == 6) {
    // -------------------------------------------------- producers: warp 4 Q and K, warp 6 V
    if (lane == 0) {
      const bool is_k = warp == 4;
      const int nslots = is_k ? L::kKSlots : L::kVSlots;
      uint64_t* full = is_k ? k_full : v_full;
      uint64_t* empty = is_k ? k_empty : v_empty;
      const CUtensorMap* tm = is_k ? &tmk : &tmv;
      WinCursor c;
      c.start(w);
      int g = 0, ti = 0;  // global step, tile counter
      bool ok = true;
      while (ok && c.valid(w)) {
        if (is_k && c.s == 0) {  // the tile's queries into Q buffer ti & 1
          const int qb = ti & 1;
          if (ti >= 2 && !mbar_wait_bounded(&q_empty[qb], ((ti >> 1) - 1) & 1)) { ok = false; break; }
          mbar_arrive_expect_tx(&q_full[qb], L::kQBytes);
          for (int hf = 0; hf < D / 64; ++hf)
            tc::tma_load_2d(qbuf(qb) + hf * (kWT * 128), &tmq, hf * 64, c.bh * w.n + kWT * c.p,
                            &q_full[qb]);
        }
        const int sl = g % nslots;
        if (g >= nslots && !mbar_wait_bounded(&empty[sl], ((g / nslots) - 1) & 1)) { ok = false; break; }
        mbar_arrive_expect_tx(&full[sl], L::kBlkBytes);
        const int y = c.bh * w.n + (c.first + c.s) * kWB;
        unsigned char* dst = is_k ? kblk(sl) : vblk(sl);
        for (int hf = 0; hf < D / 64; ++hf)
          tc::tma_load_2d(dst + hf * (kWB * 128), tm, hf * 64, y, &full[sl]);
        ++g;
        const bool tile_end = c.s + 1 == c.nst;
        c.next(w);
        if (tile_end) ++ti;
      }
      if (!ok) {
        s_abort = 1;
        // copies still in flight land before the CTA leaves
        for (int j = max(0, g - nslots); j < g; ++j)
          (void)mbar_wait_bounded(&full[j % nslots], (j / nslots) & 1, 1u << 16);
      }
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = tc::idesc_bf16(kWT, kWB, false, false);
      constexpr uint32_t idO = tc::idesc_bf16(kWT, D, false, true);
      // S_g = Q K_g^T into S buffer g % 3
      auto issue_s = [&](int g, int qb) {
        const uint32_t d_s = tmem + (uint32_t)((g % L::kSBufs) * kWB);
        const unsigned char* kb = kblk(g % L::kKSlots);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const int hf = kk >> 2, off = (kk & 3) * 32;
          const uint64_t a = tc::smem_desc_sw128(qbuf(qb) + hf * (kWT * 128) + off, 16, 1024);
          const uint64_t b = tc::smem_desc_sw128(kb + hf * (kWB * 128) + off, 16, 1024);
          tc::mma_f16_ss(d_s, a, b, idS, kk > 0);
        }
        tc::mma_commit(&s_full[g % L::kSBufs]);
        tc::mma_commit(&k_empty[g % L::kKSlots]);
      };
      bool ok = true;
      // the S cursor runs two steps ahead of the P V cursor
      WinCursor cs, cp;
      cs.start(w);
      cp.start(w);
      int gs = 0, ts = 0;  // S cursor: global step, tile counter
      auto s_step = [&]() -> bool {  // issue S at the S cursor, advance it
        const int qb = ts & 1;
        if (cs.s == 0 && !mbar_wait_bounded(&q_full[qb], (ts >> 1) & 1)) return false;
        if (!mbar_wait_bounded(&k_full[gs % L::kKSlots], (gs / L::kKSlots) & 1)) return false;
        if (gs >= L::kSBufs &&
            !mbar_wait_bounded(&s_free[gs % L::kSBufs], ((gs / L::kSBufs) - 1) & 1))
          return false;
        tc::fence_after_sync();
        issue_s(gs, qb);
        const bool tile_end = cs.s + 1 == cs.nst;
        if (tile_end) tc::mma_commit(&q_empty[qb]);  // the tile's last S has read its queries
        ++gs;
        cs.next(w);
        if (tile_end) ++ts;
        return true;
      };
      for (int a = 0; a < L::kSBufs - 1 && ok && cs.valid(w); ++a) ok = s_step();
      int g = 0, tp = 0;  // P V cursor
      while (ok && cp.valid(w)) {
        if (cs.valid(w)) {
          ok = s_step();
          if (!ok) break;
        }
        const int pb = g & 1;
        ok = mbar_wait_bounded(&p_full[pb], (g >> 1) & 1) &&
             mbar_wait_bounded(&v_full[g % L::kVSlots], (g / L::kVSlots) & 1);
        if (ok && cp.s == 0 && tp > 0) ok = mbar_wait_bounded(o_free, (tp - 1) & 1);
        if (!ok) break;
        tc::fence_after_sync();
        const uint32_t d_o = tmem + L::kOCol;
        const unsigned char* vt = vblk(g % L::kVSlots);
#pragma unroll
        for (int kk = 0; kk < kWB / 16; ++kk) {  // 64 keys in steps of 16
          const uint64_t a = tc::smem_desc_sw128(pbuf(pb) + kk * 32, 16, 1024);
          const uint64_t b = tc::smem_desc_sw128(vt + kk * 2048, kWB * 128, 1024);
          tc::mma_f16_ss(d_o, a, b, idO, (cp.s > 0 || kk > 0) ? 1u : 0u);
        }
        tc::mma_commit(&o_done[pb]);
        tc::mma_commit(&v_empty[g % L::kVSlots]);
        ++g;
        const bool tile_end = cp.s + 1 == cp.nst;
        cp.next(w);
        if (tile_end) ++tp;
      }
      if (!ok) s_abort = 1;
      tc::mma_commit(fin);  // every MMA issued has completed before TMEM is released
      if (!mbar_wait_bounded(fin, 0)) s_abort = 1;
    }
  } else {
    // ------------------------------------------------------------------ softmax warps 0-3
    const int r = 32 * warp + lane;  // query row of the tile = TMEM lane
    const uint32_t lane_base = (uint32_t)(32 * warp) << 16;
    const float qk_scale = rsqrtf((float)D) * kWLog2e;
    bool ok = true;
    WinCursor c;
    c.start(w);
    int g = 0, ti = 0;
    float m_run = -INFINITY, l_run = 0.f;
    while (ok && c.valid(w)) {
      const int i = kWT * c.p + r;  // query position
      const int b = c.first + c.s;  // key block
      const int st = g & 1;              // P buffer
      const int sb = g % L::kSBufs;      // S buffer
      ok = __all_sync(0xffffffffu, mbar_wait_bounded(&s_full[sb], (g / L::kSBufs) & 1));
      if (!ok) break;
      tc::fence_after_sync();
      float x[64];
      tc::tmem_ld32(tmem + lane_base + (uint32_t)(sb * kWB), x);
      tc::tmem_ld32(tmem + lane_base + (uint32_t)(sb * kWB + 32), x + 32);
      tc::tmem_wait_ld();
      tc::reg_fence(x);
      tc::fence_before_sync();
      mbar_arrive(&s_free[sb]);
      // keys of block b the row sees: j in [i - window + 1, i]; the masked form runs for the
      // whole warp when any of its rows needs it (most blocks of a tile need none)
      const int lo = i - w.window + 1 - kWB * b, hi = i - kWB * b;  // column bounds
      if (!__all_sync(0xffffffffu, lo <= 0 && hi >= kWB - 1)) {
        // the kept columns [max(lo, 0), min(hi, 63)] as two 32-bit masks: one bit test per column
        const int ca = max(lo, 0), cz = min(hi, kWB - 1);
        uint64_t keep = 0ull;
        if (ca <= cz) keep = (cz >= 63 ? ~0ull : ((2ull << cz) - 1ull)) & ~((1ull << ca) - 1ull);
        const uint32_t k0 = (uint32_t)keep, k1 = (uint32_t)(keep >> 32);
#pragma unroll
        for (int col = 0; col < kWB; ++col)
          x[col] = ((col < 32 ? k0 : k1) & (1u << (col & 31))) ? x[col] : -INFINITY;
      }
      // row maximum of the raw scores (three-input maxima), then in log2 units: the scale is
      // positive, so the maximum commutes with it and each key needs one FMA before its exp2
      static_assert(kWB == 64, "the maximum below covers 64 columns");
      float mx4[4];
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) mx4[q4] = max3f(x[q4], x[4 + q4], x[8 + q4]);  // 0-11
#pragma unroll
      for (int col = 12; col + 8 <= kWB; col += 8) {  // 12-59
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) mx4[q4] = max3f(mx4[q4], x[col + q4], x[col + 4 + q4]);
      }
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) mx4[q4] = fmaxf(mx4[q4], x[60 + q4]);  // 60-63
      const float mx = max3f(mx4[0], mx4[1], fmaxf(mx4[2], mx4[3])) * qk_scale;
      const float m_new = fmaxf(m_run, mx);
      const bool rescale = m_run != -INFINITY && m_new > m_run + kWRescale;
      float corr = 1.f;
      if (rescale) corr = tc::ex2_approx(m_run - m_new);
      if (rescale || m_run == -INFINITY) m_run = m_new;
      const float neg_m = m_run == -INFINITY ? 0.f : -m_run;  // masked keys give 2^-inf = 0
      // two keys per packed FMA (exponent argument) and per packed add (four pairs of partial
      // row sums)
      const uint64_t sc2 = tc::pack_f2(qk_scale, qk_scale), nm2 = tc::pack_f2(neg_m, neg_m);
      uint64_t sum2[4] = {0ull, 0ull, 0ull, 0ull};
      uint32_t pk[32];
#pragma unroll
      for (int col = 0; col < kWB; col += 2) {
        float a0, a1;
        tc::unpack_f2(tc::fma_f2(tc::pack_f2(x[col], x[col + 1]), sc2, nm2), a0, a1);
        const float p0 = tc::ex2_approx(a0);
        const float p1 = tc::ex2_approx(a1);
        sum2[(col >> 1) & 3] = tc::add_f2(sum2[(col >> 1) & 3], tc::pack_f2(p0, p1));
        const __nv_bfloat162 h2 = __floats2bfloat162_rn(p0, p1);
        pk[col / 2] = *reinterpret_cast<const uint32_t*>(&h2);
      }
      float sl[8];
#pragma unroll
      for (int e = 0; e < 4; ++e) tc::unpack_f2(sum2[e], sl[2 * e], sl[2 * e + 1]);
      l_run = l_run * corr + (((sl[0] + sl[1]) + (sl[2] + sl[3])) + ((sl[4] + sl[5]) + (sl[6] + sl[7])));
      // O may be rescaled only after P_{g-1} V_{g-1} (same tile) completed; P buffer st may be
      // rewritten once P_{g-2} V_{g-2} completed (implied by the former)
      const bool any_rescale = c.s > 0 && __any_sync(0xffffffffu, rescale);
      if (any_rescale) {
        ok = __all_sync(0xffffffffu, mbar_wait_bounded(&o_done[(g - 1) & 1], ((g - 1) >> 1) & 1));
      } else if (g >= 2) {
        ok = __all_sync(0xffffffffu, mbar_wait_bounded(&o_done[st], ((g - 2) >> 1) & 1));
      }
      if (!ok) break;
      tc::fence_after_sync();
      if (any_rescale) {
        if (!rescale) corr = 1.f;
#pragma unroll
        for (int c0 = 0; c0 < D; c0 += 32) {
          float ov[32];
          tc::tmem_ld32(tmem + lane_base + L::kOCol + (uint32_t)c0, ov);
          tc::tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) ov[e] *= corr;
          tc::tmem_st32(tmem + lane_base + L::kOCol + (uint32_t)c0, ov);
        }
        tc::tmem_wait_st();
      }
      // P row -> shared memory, 128-byte swizzled K-major [128 x 64]
      unsigned char* prow = pbuf(st);
#pragma unroll
      for (int ch = 0; ch < 8; ++ch) {
        const uint4 w4 = make_uint4(pk[4 * ch], pk[4 * ch + 1], pk[4 * ch + 2], pk[4 * ch + 3]);
        *reinterpret_cast<uint4*>(prow + tc::sw128_offset(r, ch)) = w4;
      }
      fence_proxy_async();
      tc::fence_before_sync();
      mbar_arrive(&p_full[st]);
      const bool tile_end = c.s + 1 == c.nst;
      if (tile_end) {
        // epilogue: O / l -> o once the tile's last P V completed; then O is free for the next
        ok = __all_sync(0xffffffffu, mbar_wait_bounded(&o_done[st], (g >> 1) & 1));
        if (!ok) break;
        tc::fence_after_sync();
        const bool live = i < w.n;
        const float inv = 1.f / l_run;
        __nv_bfloat16* op = static_cast<__nv_bfloat16*>(w.o) + ((size_t)c.bh * w.n + i) * D;
#pragma unroll
        for (int c0 = 0; c0 < D; c0 += 32) {
          float ov[32];
          tc::tmem_ld32(tmem + lane_base + L::kOCol + (uint32_t)c0, ov);
          tc::tmem_wait_ld();
          if (live) {
#pragma unroll
            for (int e = 0; e < 32; e += 8) {
              uint4 w4;
              __nv_bfloat162 h;
              h = __floats2bfloat162_rn(ov[e] * inv, ov[e + 1] * inv);
              w4.x = *reinterpret_cast<uint32_t*>(&h);
              h = __floats2bfloat162_rn(ov[e + 2] * inv, ov[e + 3] * inv);
              w4.y = *reinterpret_cast<uint32_t*>(&h);
              h = __floats2bfloat162_rn(ov[e + 4] * inv, ov[e + 5] * inv);
              w4.z = *reinterpret_cast<uint32_t*>(&h);
              h = __floats2bfloat162_rn(ov[e + 6] * inv, ov[e + 7] * inv);
              w4.w = *reinterpret_cast<uint32_t*>(&h);
              *reinterpret_cast<uint4*>(op + c0 + e) = w4;
            }
          }
        }
        tc::fence_before_sync();
        mbar_arrive(o_free);
        m_run = -INFINITY;
        l_run = 0.f;
        ++ti;
      }
      ++g;
      c.next(w);
    }
    if (!ok) s_abort = 1;
  }

  tc::fence_before_sync();
  __syncthreads();
  if (s_abort && tid == 0) report_timeout(w.status, 4);
  if (warp == 5) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, L::kTmemCols);
  }
}

PFN_cuTensorMapEncodeTiled_v12000 win_encode() {
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

// [rows, D] bf16, boxes of 64 columns x box_rows rows, 128-byte swizzle
bool win_map(CUtensorMap* m, const void* base, long long rows, int D, int box_rows) {
  auto enc = win_encode();
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
bsa_status launch_window(const void* q, const void* k, const void* v, const WinParams& w,
                         cudaStream_t st) {
  using L = WinSmem<D>;
  CUtensorMap tmq, tmk, tmv;
  const long long rows = (long long)w.BH * w.n;
  if (!win_map(&tmq, q, rows, D, kWT) || !win_map(&tmk, k, rows, D, kWB) ||
      !win_map(&tmv, v, rows, D, kWB))
    return BSA_ERR_CUDA;
  const int smem = L::kTotal + 1024;  // + alignment slack
  auto kern = window_tc_kernel<D>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
      cudaSuccess) {
    (void)cudaGetLastError();
    return BSA_ERR_CUDA;
  }
  const int grid = std::min(w.ntiles, L::kPerSM * kSMs);
  kern<<<grid, kWThreads, smem, st>>>(tmq, tmk, tmv, w);
  return BSA_OK;
}

}  // namespace

// Short branch of the FreeSolo prefill: q, k rotated (bf16), v raw; o = the window attention.
bsa_status window_attn_tc(const void* q, const void* k, const void* v, int B, int H, int Hk,
                          int n, int d, int window, void* o, int* status, cudaStream_t st) {
  if (Hk != H || (d != 64 && d != 128) || window < 1) return BSA_ERR_UNSUPPORTED;
  WinParams w;
  w.BH = B * H;
  w.n = n;
  w.window = window;
  w.ntile = ceil_div(n, kWT);
  w.ntiles = w.BH * w.ntile;
  w.o = o;
  w.status = status;
  const bsa_status rc =
      d == 64 ? launch_window<64>(q, k, v, w, st) : launch_window<128>(q, k, v, w, st);
  if (rc != BSA_OK) return rc;
  BSA_LAUNCH_CHECK();
  return BSA_OK;
}

}  // namespace bsa
