// Fused decode step: block scoring -> Top-K -> GQA union -> sparse attention -> merge, in one
// launch, one thread-block cluster per (batch, kv head).
//
// [SAS] review, "How it works" step 6 and "Decoding efficiency" (Fig. 7): at inference every
// decode step scores the summaries of all history blocks, keeps the Top-K plus the current block
// and attends their tokens; scoring and Top-K grow with the context and dominate long-context
// steps.  [FreeSolo] summary page, "How it works": optional erf distance bias of the cell score.
//
// B200 design.  The step is HBM-bound (summaries + selected K/V) and short (~10 us), so launch
// boundaries, global round trips and serial latency chains cost as much as the bytes.  The CL
// CTAs of a cluster (CL <= 16) cooperate through distributed shared memory (DSMEM):
//   1. CTA r scores its slice of the history blocks: the mean-key rows stream through a
//      two-stage shared-memory ring filled by bulk copies (TMA engine); the G query heads of the
//      group share every row (one 31-shuffle transpose-reduce per 32/G rows).  Per head, a warp
//      selects the slice's local Top-K (bisection on order-preserving keys with warp reductions)
//      and PUSHES the candidates into every peer's merge buffer with DSMEM stores.
//   2. cluster barrier; each CTA selects the global Top-K per head from its own merge buffer
//      (same exact order everywhere: larger score, then lower index) and builds the sorted union
//      of the G heads' selections (a bitmap over the history blocks, compacted by one warp), plus
//      the current block, with a head mask per entry.
//   3. CTA r attends union entries r, r+CL, ...  bf16: each K/V block arrives as 128-byte swizzled
//      64x64 TMA tiles; two groups of four warps take alternate entries; a warp owns 16 tokens of
//      a block and computes S = Q K^T and O += P V with warp-level MMAs (the G heads padded to 16
//      rows), keeping its own online-softmax state, so the per-block work is ~30 MMAs per warp
//      instead of ~1,200 scalar FMAs/shuffles.  fp32: the same split with scalar FMAs.  The CTA
//      holding the current block also rewrites that block's summary from shared memory.
//   4. Each CTA merges its warps, then pushes to CTA r' the partial (m, l, o) of the output columns
//      CTA r' owns; cluster barrier; each CTA finishes its columns and writes o (and lse).
// Variants (flags of bsa_decode_step_ex): shared selection -- the group's score of a block is the
// mean of its G heads' scores, ranked once and attended by every head (one selection per kv
// head instead of G); bf16 summaries -- the mean keys are read (and appended) in bf16, halving the
// summary bytes, with fp32 accumulation of the dot products.
// Every CTA reaches every cluster barrier (no early exit); every mbarrier wait is bounded.
#include <cudaTypedefs.h>

#include <map>
#include <mutex>
#include <tuple>
#include <type_traits>

#include "tc_common.cuh"

namespace bsa {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kMaxCL = 16;
constexpr int kMaxKf = 32;        // Top-K bound of the fused path
constexpr int kMaxUnion = 8 * kMaxKf + 1;
constexpr int kMaxWords = 512;    // history bitmap words: C <= 16384
constexpr int kSub = 64;          // summary rows per ring stage
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescale = 8.f;   // lazy rescale threshold (log2 units)

struct FusedParams {
  const void* q;
  const void* k;
  const void* v;
  int B, Hq, Hk, n, b, C, K;
  const int* seq_lens;
  void* mean_k;  // [B, Hk, C, d] in the summary type (fp32, or bf16 on the 64-token bf16 path)
  float* max_norm;
  float* centre;
  int append;
  const float* lam;
  const float* sig;
  int prefix_block;
  void* o;
  float* lse;
  int* idx;
  int* count;
  int* status;
  int chunk;  // history blocks scored per CTA (multiple of kSub)
  int shared;  // one selection per kv head from the mean of its heads' scores
};

// ---- cluster helpers ---------------------------------------------------------------------

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_size() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;"
               ::: "memory");
}
__device__ __forceinline__ uint32_t dsmem_addr(const void* p, uint32_t rank) {
  uint32_t out;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(out) : "r"(smem_u32(p)), "r"(rank));
  return out;
}
__device__ __forceinline__ void st_dsmem_u32(uint32_t addr, uint32_t v) {
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}
__device__ __forceinline__ void st_dsmem_f32(uint32_t addr, float v) {
  asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(addr), "f"(v) : "memory");
}

__device__ __forceinline__ uint32_t order_key(float f) {
  if (f != f) return 0u;
  if (f == 0.f) f = 0.f;
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Top-K of N order keys (shared memory, index order) by one warp: an exact radix select with
// 4-bit digits.  The keys sit in registers (lane l holds positions l + 32 j).  Each pass counts
// the next digit of the keys that share the prefix found so far: every lane keeps sixteen 4-bit
// counters in one 64-bit word (at most 8 keys between two flushes into 16-bit fields), the eight
// 32-bit words of 16-bit bins are summed over the warp, and the pass keeps the digit at which the
// count of keys at or above the threshold reaches K.  It stops as soon as that count is exactly K
// ({key >= T} is then the answer); otherwise after the last digit T is the K-th largest key and
// the lowest-indexed keys equal to T fill the remaining places.
// Writes the selected positions ascending to `out`; returns min(K, N).  Up to 64 keys an exact
// rank count (below) is cheaper than the radix passes.
constexpr int kSelItems = 16;  // N <= 32 * kSelItems

// count of digit d in the reduced words: parity p = d & 1 picks words 4p.., the byte k = d >> 1
// of the nibble-split word sits in b[k & 1] as 16-bit field k >> 1 (see flush_nibbles)
__device__ __forceinline__ int bin_count(const uint32_t (&r)[8], int d) {
  const int p = d & 1, k = d >> 1, which = k & 1, f = k >> 1;
  return (int)((r[p * 4 + which * 2 + (f >> 1)] >> ((f & 1) * 16)) & 0xFFFFu);
}
// add sixteen 4-bit counters (nibble d = count of digit d) to eight words of 16-bit bins
__device__ __forceinline__ void flush_nibbles(uint64_t a, uint32_t (&r)[8]) {
  const uint64_t m4 = 0x0F0F0F0F0F0F0F0Full, m8 = 0x00FF00FF00FF00FFull;
  const uint64_t n0 = a & m4, n1 = (a >> 4) & m4;  // even digits / odd digits, one per byte
  const uint64_t b[4] = {n0 & m8, (n0 >> 8) & m8, n1 & m8, (n1 >> 8) & m8};
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    r[2 * q] += (uint32_t)b[q];
    r[2 * q + 1] += (uint32_t)(b[q] >> 32);
  }
}

// Small N (<= 32 R): rank every key by counting the keys above it (ties: the lower position
// ranks higher) and keep ranks below K -- N broadcast loads per lane, no passes.
template <int R>
__device__ __forceinline__ int warp_select_rank(const uint32_t* keys, int N, int kk, int lane,
                                                int* out) {
  uint32_t mk[R];
  int rk[R];
#pragma unroll
  for (int q = 0; q < R; ++q) {
    mk[q] = lane + 32 * q < N ? keys[lane + 32 * q] : 0u;
    rk[q] = 0;
  }
  for (int j = 0; j < N; ++j) {
    const uint32_t kj = keys[j];
#pragma unroll
    for (int q = 0; q < R; ++q) rk[q] += (kj > mk[q] || (kj == mk[q] && j < lane + 32 * q)) ? 1 : 0;
  }
  const unsigned lt = (1u << lane) - 1u;
  int taken = 0;
#pragma unroll
  for (int q = 0; q < R; ++q) {
    const bool take = lane + 32 * q < N && rk[q] < kk;
    const unsigned tb = __ballot_sync(0xffffffffu, take);
    if (take) out[taken + __popc(tb & lt)] = lane + 32 * q;
    taken += __popc(tb);
  }
  __syncwarp();
  return taken;
}

__device__ __noinline__ int warp_select(const uint32_t* keys, int N, int K, int lane, int* out) {
  const int kk = min(K, N);
  if (kk <= 0) return 0;
  if (kk == N) {
    for (int i = lane; i < N; i += 32) out[i] = i;
    __syncwarp();
    return N;
  }
  if (N <= 64) return warp_select_rank<2>(keys, N, kk, lane, out);
  const int nv = (N - lane + 31) >> 5;  // keys of this lane: positions lane + 32 j, j < nv
  uint32_t kr[kSelItems];
#pragma unroll
  for (int j = 0; j < kSelItems; ++j) kr[j] = j < nv ? keys[lane + 32 * j] : 0u;
  uint32_t T = 0;  // digits fixed so far (higher bits)
  int above = 0;   // keys strictly above the prefix (they are selected)
  bool exact = false;
  for (int shift = 28; shift >= 0 && !exact; shift -= 4) {
    const uint32_t hi_mask = shift == 28 ? 0u : (0xFFFFFFFFu << (shift + 4));
    uint32_t r[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
#pragma unroll
    for (int j0 = 0; j0 < kSelItems; j0 += 8) {
      if (j0 > 0 && j0 >= nv) break;
      uint64_t acc = 0;
#pragma unroll
      for (int j = j0; j < j0 + 8; ++j) {
        const uint32_t x = kr[j];
        const bool in = j < nv && (x & hi_mask) == T;
        acc += in ? (1ull << (((x >> shift) & 15u) * 4u)) : 0ull;
      }
      flush_nibbles(acc, r);
    }
#pragma unroll
    for (int q = 0; q < 8; ++q) r[q] = __reduce_add_sync(0xffffffffu, r[q]);
    // largest digit v with above + count(digit >= v) >= kk; keys with a larger digit are taken
    int run = above, v = 0, run_at_v = 0;
#pragma unroll
    for (int d = 15; d >= 0; --d) {
      const int c = bin_count(r, d);
      if (run < kk && run + c >= kk) {
        v = d;
        run_at_v = run + c;
      }
      run += c;
    }
    int up = above;
#pragma unroll
    for (int d = 15; d >= 0; --d)
      if (d > v) up += bin_count(r, d);
    T |= (uint32_t)v << shift;
    above = up;
    exact = (run_at_v == kk);
  }
  const int rem = kk - above;  // keys equal to the full threshold still to take (if not exact)
  int taken = 0, eq_seen = 0;
  const unsigned lt = (1u << lane) - 1u;
#pragma unroll
  for (int j = 0; j < kSelItems; ++j) {
    if (32 * j >= N) break;  // warp-uniform
    const bool valid = j < nv;
    const uint32_t x = kr[j];
    bool take;
    unsigned eqb = 0u;
    if (exact) {
      // T holds the digits down to the stopping pass, zeros below: x >= T compares prefixes
      take = valid && x >= T;
    } else {
      const bool eq = valid && x == T;
      eqb = __ballot_sync(0xffffffffu, eq);
      take = (valid && x > T) || (eq && eq_seen + __popc(eqb & lt) < rem);
    }
    const unsigned tb = __ballot_sync(0xffffffffu, take);
    if (take) out[taken + __popc(tb & lt)] = 32 * j + lane;
    taken += __popc(tb);
    eq_seen += __popc(eqb);
  }
  __syncwarp();
  return taken;
}

// ---- warp MMA (legacy mma.sync, bf16 in, fp32 accumulate) ---------------------------------
__device__ __forceinline__ void mma_16816(float* c, uint32_t a0, uint32_t a1, uint32_t a2,
                                          uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t& r0, uint32_t& r1,
                                              uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// Shared-memory layout (dynamic part).  MMA: the bf16 warp-MMA path over 64-token blocks.
template <typename T, int D, int G, bool MMA>
struct FusedSmem {
  // region A: summary ring (2 x kSub x D fp32) / K,V stages (2 x {K,V} tile) / warp partials
  __host__ __device__ static size_t tile(int b) {
    return align_up((size_t)(MMA ? 64 : b) * D * sizeof(T), 1024);
  }
  __host__ __device__ static size_t region_a(int b) {
    size_t x = (size_t)2 * kSub * D * sizeof(float);
    x = max_sz(x, 4 * tile(b));
    x = max_sz(x, (size_t)kWarps * G * (D + 2) * 4 + 4096);  // warp partials
    return align_up(x, 1024);
  }
  __host__ __device__ static size_t scores(int chunk) { return align_up((size_t)G * chunk * 4, 16); }
  __host__ __device__ static size_t merge(int CL, int K) { return align_up((size_t)G * CL * K * 8, 16); }
  __host__ __device__ static size_t recv(int CL) {
    return align_up((size_t)CL * G * (D / CL + 2) * 4, 16);
  }
  __host__ __device__ static size_t zp(int b) { return 2 * align_up((size_t)b * G * 4, 16); }
  __host__ __device__ static size_t bytes(int b, int chunk, int CL, int K) {
    return region_a(b) + scores(chunk) + merge(CL, K) + recv(CL) + zp(b) + 256 + 1024;
  }
};

template <typename T, typename TS, int D, int G, bool MMA>
__global__ void __launch_bounds__(kThreads, 2) decode_fused_kernel(
    const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv,
    const FusedParams p) {
  constexpr bool kMma = MMA;
  static_assert(!MMA || std::is_same<T, __nv_bfloat16>::value, "warp MMAs take bf16");
  constexpr int EPL = D / 32;
  constexpr int R = 32 / G;

  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ int s_pick[G][kMaxKf];
  __shared__ int s_sel[G][kMaxKf];
  __shared__ int s_nsel[G];
  __shared__ uint32_t s_bits[kMaxWords];
  __shared__ int s_ublk[kMaxUnion];
  __shared__ unsigned s_umask[kMaxUnion];
  __shared__ int s_U;
  __shared__ int s_abort;
  __shared__ float s_red[kWarps];
  __shared__ float s_m[G], s_l[G], s_corr[G];

  const int b = p.b, K = p.K, Hq = p.Hq;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int rank = (int)cluster_rank();
  const int CL = (int)cluster_size();
  const int kh = blockIdx.y, bi = blockIdx.z;
  const int h0 = kh * G;
  const int L = p.seq_lens ? min(p.seq_lens[bi], p.n) : p.n;
  const int pos = L - 1;
  const int cur = pos / b;
  int nc = p.prefix_block > 0 ? ((pos / p.prefix_block) * p.prefix_block) / b : cur;
  nc = max(0, min(nc, cur));

  using SM = FusedSmem<T, D, G, MMA>;
  TS* ring = reinterpret_cast<TS*>(smem);  // fits: region A holds 2 x kSub fp32 rows
  TS* mean_k = static_cast<TS*>(p.mean_k);
  const int Gs = p.shared ? 1 : G;  // selections made per group
  unsigned char* after_a = smem + SM::region_a(b);
  uint32_t* s_keys = reinterpret_cast<uint32_t*>(after_a);                  // [G][chunk]
  unsigned char* merge = after_a + SM::scores(p.chunk);                        // [G][CL*K] x 2
  uint32_t* m_key = reinterpret_cast<uint32_t*>(merge);
  int* m_idx = reinterpret_cast<int*>(merge) + G * CL * K;
  float* recv = reinterpret_cast<float*>(merge + SM::merge(CL, K));          // [CL][G][cols+2]
  float* zs = reinterpret_cast<float*>(merge + SM::merge(CL, K) + SM::recv(CL));
  float* ps = zs + align_up((size_t)b * G, 4);
  uint64_t* bar = reinterpret_cast<uint64_t*>(merge + SM::merge(CL, K) + SM::recv(CL) + SM::zp(b));
  // bar[0], bar[1]: summary ring; bar[2], bar[3]: K/V stages

  if (tid == 0) {
    for (int i = 0; i < 4; ++i) mbar_init(&bar[i], 1);
    fence_mbar_init();
    s_abort = 0;
    s_U = 0;
  }
  if (tid < G) {
    s_m[tid] = -INFINITY;
    s_l[tid] = 0.f;
  }
  __syncthreads();

  // ---- 1. score my slice of the history blocks --------------------------------------------
  float qv[G][EPL];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    float tmp[EPL];
    load_vec<T, EPL>(static_cast<const T*>(p.q) + ((size_t)bi * Hq + h0 + g) * D + lane * EPL,
                     tmp);
#pragma unroll
    for (int e = 0; e < EPL; ++e) qv[g][e] = tmp[e];
  }
  const int c_lo = min(nc, rank * p.chunk);
  const int c_hi = min(nc, c_lo + p.chunk);
  const int rows = c_hi - c_lo;
  const int nsub = (rows + kSub - 1) / kSub;
  const TS* mk = mean_k + ((size_t)(bi * p.Hk + kh) * p.C) * D;
  auto issue_sub = [&](int j) {
    const int r0 = c_lo + j * kSub;
    const int nr = min(kSub, c_hi - r0);
    const uint32_t bytes = (uint32_t)(nr * D * sizeof(TS));
    mbar_arrive_expect_tx(&bar[j & 1], bytes);
    bulk_g2s(ring + (size_t)(j & 1) * kSub * D, mk + (size_t)r0 * D, bytes, &bar[j & 1]);
  };
  if (tid == 0)
    for (int j = 0; j < min(nsub, 2); ++j) issue_sub(j);
  const float scale = rsqrtf((float)D);
  const int my_r = lane / G, my_g = lane % G;
  const float lam_h = p.lam ? p.lam[h0 + my_g] : 0.f;
  const float inv2sig = p.lam ? 0.5f / p.sig[h0 + my_g] : 0.f;
  for (int j = 0; j < nsub; ++j) {
    if (!s_abort && !mbar_wait_bounded(&bar[j & 1], (j >> 1) & 1)) s_abort = 1;
    __syncthreads();
    if (!s_abort) {
      const int r0 = j * kSub;
      const int nr = min(kSub, rows - r0);
      const TS* base = ring + (size_t)(j & 1) * kSub * D;
      for (int t0 = warp * R; t0 < nr; t0 += kWarps * R) {
        float a[32];
#pragma unroll
        for (int r = 0; r < R; ++r) {
          float x[EPL];
          if (t0 + r < nr) {
            load_vec<TS, EPL>(base + (size_t)(t0 + r) * D + lane * EPL, x);
          } else {
#pragma unroll
            for (int e = 0; e < EPL; ++e) x[e] = 0.f;
          }
#pragma unroll
          for (int g = 0; g < G; ++g) {
            float s = 0.f;
#pragma unroll
            for (int e = 0; e < EPL; ++e) s = fmaf(qv[g][e], x[e], s);
            a[r * G + g] = s;
          }
        }
        warp_transpose_reduce32(a, lane);
        const int t = t0 + my_r;
        float s = a[0] * scale;
        if (p.lam && t < nr) {
          const size_t row = (size_t)(bi * p.Hk + kh) * p.C + c_lo + r0 + t;
          s += lam_h * p.max_norm[row] * erff(((float)pos - p.centre[row]) * inv2sig);
        }
        if (p.shared) {  // mean over the G lanes of this row (lane = my_r * G + my_g)
#pragma unroll
          for (int o = 1; o < G; o <<= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
          s *= 1.f / (float)G;
        }
        if (t < nr && my_g < Gs) s_keys[my_g * p.chunk + r0 + t] = order_key(s);
      }
    }
    __syncthreads();
    if (tid == 0 && j + 2 < nsub && !s_abort) issue_sub(j + 2);
  }
  // local Top-K per head (per group when shared), pushed into every CTA's merge buffer at slot
  // rank*K
  for (int g = warp; g < Gs; g += kWarps) {
    const uint32_t* keys = s_keys + g * p.chunk;
    const int cnt = warp_select(keys, rows, K, lane, s_pick[g]);
    for (int e = lane; e < CL * K; e += 32) {
      const int r = e / K, j = e % K;
      const uint32_t key = j < cnt ? keys[s_pick[g][j]] : 0u;
      const int gi = j < cnt ? c_lo + s_pick[g][j] : -1;  // -1: empty slot
      const int slot = g * CL * K + rank * K + j;
      st_dsmem_u32(dsmem_addr(&m_key[slot], r), key);
      st_dsmem_u32(dsmem_addr(&m_idx[slot], r), (uint32_t)gi);
    }
  }
  cluster_sync();

  // ---- 2. global Top-K per head, then the union -------------------------------------------
  const int nwords = (nc + 31) / 32;
  for (int w = tid; w < nwords; w += kThreads) s_bits[w] = 0u;
  for (int g = warp; g < Gs; g += kWarps) {
    // empty slots carry key 0 and index -1: compact the valid ones first (index order kept)
    uint32_t* mk_g = m_key + g * CL * K;
    int* mi_g = m_idx + g * CL * K;
    int nvalid = 0;
    for (int e0 = 0; e0 < CL * K; e0 += 32) {
      const int e = e0 + lane;
      const bool ok = e < CL * K && mi_g[e] >= 0;
      const uint32_t kk2 = ok ? mk_g[e] : 0u;
      const int ii = ok ? mi_g[e] : 0;
      const unsigned bal = __ballot_sync(0xffffffffu, ok);
      __syncwarp();
      if (ok) {
        const int at = nvalid + __popc(bal & ((1u << lane) - 1u));
        mk_g[at] = kk2;
        mi_g[at] = ii;
      }
      nvalid += __popc(bal);
      __syncwarp();
    }
    const int cnt = warp_select(mk_g, nvalid, K, lane, s_pick[g]);
    for (int j = lane; j < cnt; j += 32) s_sel[g][j] = mi_g[s_pick[g][j]];
    if (lane == 0) s_nsel[g] = cnt;
  }
  __syncthreads();
  if (rank == 0) {  // optional outputs: the selection of every head
    for (int e = tid; e < G * K; e += kThreads) {
      const int g = e / K, j = e % K, gs = p.shared ? 0 : g;
      const size_t row = (size_t)bi * Hq + h0 + g;
      if (p.idx) p.idx[row * K + j] = j < s_nsel[gs] ? s_sel[gs][j] : -1;
      if (p.count && j == 0) p.count[row] = s_nsel[gs];
    }
  }
  for (int e = tid; e < Gs * K; e += kThreads) {
    const int g = e / K, j = e % K;
    if (j < s_nsel[g]) {
      const int x = s_sel[g][j];
      atomicOr(&s_bits[x >> 5], 1u << (x & 31));
    }
  }
  for (int e = tid; e < kMaxUnion; e += kThreads) s_umask[e] = 0u;
  __syncthreads();
  if (warp == 0) {  // compact the bitmap into the sorted union (one word per lane up to 32)
    const int per = (nwords + 31) / 32;
    int mine = 0;
    for (int w = lane * per; w < min(nwords, (lane + 1) * per); ++w) mine += __popc(s_bits[w]);
    int incl = mine;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    int at = incl - mine;
    for (int w = lane * per; w < min(nwords, (lane + 1) * per); ++w) {
      uint32_t bits = s_bits[w];
      while (bits) {
        const int bit = __ffs(bits) - 1;
        bits &= bits - 1;
        s_ublk[at++] = w * 32 + bit;
      }
    }
    if (lane == 31) {
      s_ublk[incl] = cur;  // the current block, always kept, follows every history block
      s_umask[incl] = (1u << G) - 1u;
      s_U = incl + 1;
    }
  }
  __syncthreads();
  const int U = s_U;
  for (int e = tid; e < Gs * K; e += kThreads) {  // head masks by binary search in the union
    const int g = e / K, j = e % K;
    if (j < s_nsel[g]) {
      const int x = s_sel[g][j];
      int lo = 0, hi = U - 2;
      while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (s_ublk[mid] < x) lo = mid + 1; else hi = mid;
      }
      atomicOr(&s_umask[lo], p.shared ? (1u << G) - 1u : 1u << g);
    }
  }
  __syncthreads();

  // ---- 3. attend my union entries -----------------------------------------------------------
  const int ne = rank < U ? (U - rank + CL - 1) / CL : 0;
  auto entry_tokens = [&](int m) { return m == cur ? pos - cur * b + 1 : b; };
  float* wpart = reinterpret_cast<float*>(smem);  // reused after phase 3: [warp][G][D+2]

  if constexpr (kMma) {
    // two groups of four warps take alternate entries; stage st = entry & 1 holds K then V
    const int grp = warp >> 2, wg = warp & 3;
    const size_t tl = SM::tile(b);
    auto ktile = [&](int st) { return smem + (size_t)st * 2 * tl; };
    auto vtile = [&](int st) { return smem + (size_t)st * 2 * tl + tl; };
    uint64_t* kvbar = bar + 2;
    const int row0 = (bi * p.Hk + kh) * p.n;
    auto issue_kv = [&](int i) {
      const int m = s_ublk[rank + i * CL];
      const int st = i & 1;
      mbar_arrive_expect_tx(&kvbar[st], 2 * 64 * D * 2);
#pragma unroll
      for (int hf = 0; hf < D / 64; ++hf) {
        tc::tma_load_2d(ktile(st) + hf * 8192, &tmk, hf * 64, row0 + m * b, &kvbar[st]);
        tc::tma_load_2d(vtile(st) + hf * 8192, &tmv, hf * 64, row0 + m * b, &kvbar[st]);
      }
    };
    if (tid == 0 && !s_abort) {
      fence_proxy_async();  // generic accesses of phase 1 precede the async writes into region A
      if (ne > 0) issue_kv(0);
      if (ne > 1) issue_kv(1);
    }
    // A fragments of Q (rows = heads, zero beyond G), pre-scaled into log2 units
    const int grow = lane >> 2, tig = lane & 3;
    uint32_t qa0[D / 16], qa1[D / 16];
    {
      const float qs = scale * kLog2e;
      const T* qrow = static_cast<const T*>(p.q) + ((size_t)bi * Hq + h0 + min(grow, G - 1)) * D;
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks) {
        float x0 = 0.f, x1 = 0.f, x2 = 0.f, x3 = 0.f;
        if (grow < G) {
          x0 = Elem<T>::to_f(qrow[16 * ks + 2 * tig]) * qs;
          x1 = Elem<T>::to_f(qrow[16 * ks + 2 * tig + 1]) * qs;
          x2 = Elem<T>::to_f(qrow[16 * ks + 2 * tig + 8]) * qs;
          x3 = Elem<T>::to_f(qrow[16 * ks + 2 * tig + 9]) * qs;
        }
        qa0[ks] = pack_bf16(x0, x1);
        qa1[ks] = pack_bf16(x2, x3);
      }
    }
    // O^T accumulators: m-tile mt covers d rows 16 mt .. 16 mt + 15, columns are heads
    float oacc[D / 16][4];
#pragma unroll
    for (int c = 0; c < D / 16; ++c) oacc[c][0] = oacc[c][1] = oacc[c][2] = oacc[c][3] = 0.f;
    float m_run = -INFINITY, l_part = 0.f;
    for (int i = grp; i < ne; i += 2) {
      const int st = i & 1;
      const int m = s_ublk[rank + i * CL];
      const unsigned hm = s_umask[rank + i * CL];
      const int tok = entry_tokens(m);
      // group-uniform decision: the OR over the group's four warps of "my wait ran out"
      const int bad = mbar_wait_bounded(&kvbar[st], (i >> 1) & 1) ? 0 : 1;
      int any_bad;
      asm volatile(
          "{\n\t.reg .pred pin, pout;\n\t"
          "setp.ne.s32 pin, %1, 0;\n\t"
          "barrier.red.or.pred pout, %2, 128, pin;\n\t"
          "selp.s32 %0, 1, 0, pout;\n\t}"
          : "=r"(any_bad)
          : "r"(bad), "r"(1 + grp)
          : "memory");
      if (any_bad) {
        s_abort = 1;
        break;
      }
      const unsigned char* kt = ktile(st);
      const unsigned char* vt = vtile(st);
      const int t0 = wg * 16;  // this warp's 16 tokens
      // S = Q K^T over two 8-token tiles
      float sfr[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        const int tokr = t0 + 8 * nt + grow;  // B fragment row (token)
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const int hf = ks >> 2, ch = (ks & 3) * 2;
          const unsigned char* rowp = kt + hf * 8192 + tokr * 128;
          const uint32_t b0 =
              *reinterpret_cast<const uint32_t*>(rowp + ((ch ^ (tokr & 7)) << 4) + 4 * tig);
          const uint32_t b1 =
              *reinterpret_cast<const uint32_t*>(rowp + (((ch + 1) ^ (tokr & 7)) << 4) + 4 * tig);
          mma_16816(sfr[nt], qa0[ks], 0u, qa1[ks], 0u, b0, b1);
        }
      }
      // masks, per-row online softmax (row = head grow; the quad shares the row)
      const bool head_on = grow < G && ((hm >> grow) & 1u);
      float mx = -INFINITY;
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int t = t0 + 8 * nt + 2 * tig + e;
          if (!head_on || t >= tok) sfr[nt][e] = -INFINITY;
          mx = fmaxf(mx, sfr[nt][e]);
        }
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      float corr = 1.f;  // rescale of head `grow` (lazy: only when its max grows by > 2^8)
      if (mx > m_run + kRescale || (m_run == -INFINITY && mx != -INFINITY)) {
        corr = m_run == -INFINITY ? 0.f : exp2f(m_run - mx);
        m_run = mx;
        l_part *= corr;
      }
      // O^T columns are heads: this lane holds heads 2 tig and 2 tig + 1
      const float corr_a = __shfl_sync(0xffffffffu, corr, 8 * tig);
      const float corr_b = __shfl_sync(0xffffffffu, corr, 8 * tig + 4);
      if (__any_sync(0xffffffffu, corr_a != 1.f || corr_b != 1.f)) {
#pragma unroll
        for (int c = 0; c < D / 16; ++c) {
          oacc[c][0] *= corr_a;
          oacc[c][1] *= corr_b;
          oacc[c][2] *= corr_a;
          oacc[c][3] *= corr_b;
        }
      }
      float pv[2][2];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const float z = sfr[nt][e];
          pv[nt][e] = z == -INFINITY ? 0.f : exp2f(z - m_run);
          l_part += pv[nt][e];
        }
      // P^T as the B operand (k = tokens, n = heads): exactly the S accumulator pairs
      const uint32_t pb0 = pack_bf16(pv[0][0], pv[0][1]);
      const uint32_t pb1 = pack_bf16(pv[1][0], pv[1][1]);
      // O^T += V^T P^T: A fragments of V^T by transposed 8x8 loads of the swizzled V tile
#pragma unroll
      for (int mt = 0; mt < D / 16; ++mt) {
        const int mi = lane >> 3, rr = lane & 7;
        const int tokr = t0 + (mi >> 1) * 8 + rr;
        const int chunk = 2 * mt + (mi & 1);  // 16-byte chunk along d (0..D/8-1)
        const int hf = chunk >> 3, cin = chunk & 7;
        const uint32_t addr =
            smem_u32(vt + hf * 8192 + tokr * 128 + ((cin ^ (tokr & 7)) << 4));
        uint32_t v0, v1, v2, v3;
        ldsm_x4_trans(addr, v0, v1, v2, v3);
        mma_16816(oacc[mt], v0, v1, v2, v3, pb0, pb1);
      }
      // the block being filled: rewrite its summary from the swizzled K tile
      if (p.append && m == cur) {  // taken by the whole group that holds the current block
        const int gt = tid & 127;
        const int col = gt;  // one column per thread (D <= 128)
        if (col < D) {
          float sum = 0.f;
          const int hf = col >> 6, cin = (col & 63) >> 3, e8 = col & 7;
          for (int t = 0; t < tok; ++t)
            sum += Elem<T>::to_f(*reinterpret_cast<const T*>(
                kt + hf * 8192 + t * 128 + ((cin ^ (t & 7)) << 4) + e8 * 2));
          mean_k[((size_t)(bi * p.Hk + kh) * p.C + cur) * D + col] = Elem<TS>::from_f(sum / (float)tok);
        }
        // max key norm: thread t < tok takes token t
        float nrm = 0.f;
        if (gt < tok) {
          float sq = 0.f;
          for (int c8 = 0; c8 < D / 8; ++c8) {
            const int hf = c8 >> 3, cin = c8 & 7;
            float xx[8];
            load_vec<T, 8>(reinterpret_cast<const T*>(kt + hf * 8192 + gt * 128 +
                                                      ((cin ^ (gt & 7)) << 4)),
                           xx);
#pragma unroll
            for (int e = 0; e < 8; ++e) sq = fmaf(xx[e], xx[e], sq);
          }
          nrm = sqrtf(sq);
        }
        nrm = warp_max(nrm);
        if (lane == 0) s_red[4 * grp + wg] = nrm;
        asm volatile("bar.sync %0, 128;" ::"r"(1 + grp));
        if (gt == 0) {
          const float* rr = s_red + 4 * grp;
          float nm = fmaxf(fmaxf(rr[0], rr[1]), fmaxf(rr[2], rr[3]));
          const size_t row = (size_t)(bi * p.Hk + kh) * p.C + cur;
          if (p.max_norm) p.max_norm[row] = nm;
          if (p.centre) p.centre[row] = 0.5f * (float)(cur * b) + 0.5f * (float)(cur * b + tok - 1);
        }
      }
      asm volatile("bar.sync %0, 128;" ::"r"(1 + grp));  // stage free
      if (wg == 0 && lane == 0 && i + 2 < ne) issue_kv(i + 2);
    }
    if (s_abort && tid == 0) {
      for (int i = 0; i < 2; ++i) (void)mbar_wait_bounded(&kvbar[i], 0, 1u << 12);
      report_timeout(p.status, 2);
    }
    __syncthreads();
    // warp partials (rows < G): m, l and o
    l_part += __shfl_xor_sync(0xffffffffu, l_part, 1);
    l_part += __shfl_xor_sync(0xffffffffu, l_part, 2);
    if (grow < G && tig == 0) {
      float* wp = wpart + ((size_t)warp * G + grow) * (D + 2);
      wp[D] = m_run;
      wp[D + 1] = l_part;
    }
#pragma unroll
    for (int e = 0; e < 2; ++e) {  // O^T element (d, head 2 tig + e)
      const int hh = 2 * tig + e;
      if (hh < G) {
        float* wp = wpart + ((size_t)warp * G + hh) * (D + 2);
#pragma unroll
        for (int mt = 0; mt < D / 16; ++mt) {
          wp[16 * mt + grow] = oacc[mt][e];
          wp[16 * mt + grow + 8] = oacc[mt][2 + e];
        }
      }
    }
    __syncthreads();
  } else {
    // fp32: scalar FMAs; warps split each block's tokens, one CTA-wide softmax per block
    const size_t tl = SM::tile(b);
    T* kbuf[2] = {reinterpret_cast<T*>(smem), reinterpret_cast<T*>(smem + 2 * tl)};
    T* vbuf[2] = {reinterpret_cast<T*>(smem + tl), reinterpret_cast<T*>(smem + 3 * tl)};
    uint64_t* kvbar = bar + 2;
    const T* kbase = static_cast<const T*>(p.k) + (size_t)(bi * p.Hk + kh) * p.n * D;
    const T* vbase = static_cast<const T*>(p.v) + (size_t)(bi * p.Hk + kh) * p.n * D;
    auto issue_kv = [&](int i) {
      const int m = s_ublk[rank + i * CL];
      const uint32_t bytes = (uint32_t)(entry_tokens(m) * D * sizeof(T));
      const int st = i & 1;
      mbar_arrive_expect_tx(&kvbar[st], 2 * bytes);
      bulk_g2s(kbuf[st], kbase + (size_t)m * b * D, bytes, &kvbar[st]);
      bulk_g2s(vbuf[st], vbase + (size_t)m * b * D, bytes, &kvbar[st]);
    };
    if (tid == 0 && !s_abort) {
      fence_proxy_async();
      if (ne > 0) issue_kv(0);
      if (ne > 1) issue_kv(1);
    }
    constexpr int CG = D / 2;
    constexpr int TP = kThreads / CG;
    float qa[G][EPL];
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
      for (int e = 0; e < EPL; ++e) qa[g][e] = qv[g][e] * scale * kLog2e;
    const int cg = tid % CG, tp = tid / CG;
    float acc[G][2];
#pragma unroll
    for (int g = 0; g < G; ++g) acc[g][0] = acc[g][1] = 0.f;
    for (int i = 0; i < ne; ++i) {
      const int st = i & 1;
      const int m = s_ublk[rank + i * CL];
      const unsigned hm = s_umask[rank + i * CL];
      const int tok = entry_tokens(m);
      if (!s_abort && !mbar_wait_bounded(&kvbar[st], (i >> 1) & 1)) s_abort = 1;
      __syncthreads();
      if (s_abort) break;
      const T* kt = kbuf[st];
      const T* vt = vbuf[st];
      for (int t0 = warp * R; t0 < tok; t0 += kWarps * R) {
        float a[32];
#pragma unroll
        for (int r = 0; r < R; ++r) {
          float x[EPL];
          if (t0 + r < tok) {
            load_vec<T, EPL>(kt + (size_t)(t0 + r) * D + lane * EPL, x);
          } else {
#pragma unroll
            for (int e = 0; e < EPL; ++e) x[e] = 0.f;
          }
#pragma unroll
          for (int g = 0; g < G; ++g) {
            float sacc = 0.f;
#pragma unroll
            for (int e = 0; e < EPL; ++e) sacc = fmaf(qa[g][e], x[e], sacc);
            a[r * G + g] = sacc;
          }
        }
        warp_transpose_reduce32(a, lane);
        const int t = t0 + lane / G, g = lane % G;
        if (t < tok) zs[t * G + g] = ((hm >> g) & 1u) ? a[0] : -INFINITY;
      }
      if (p.append && m == cur) {
        for (int col = tid; col < D; col += kThreads) {
          float sum = 0.f;
          for (int t = 0; t < tok; ++t) sum += Elem<T>::to_f(kt[(size_t)t * D + col]);
          mean_k[((size_t)(bi * p.Hk + kh) * p.C + cur) * D + col] = Elem<TS>::from_f(sum / (float)tok);
        }
        float nmax = 0.f;
        for (int t = warp; t < tok; t += kWarps) {
          float x[EPL];
          load_vec<T, EPL>(kt + (size_t)t * D + lane * EPL, x);
          float sq = 0.f;
#pragma unroll
          for (int e = 0; e < EPL; ++e) sq = fmaf(x[e], x[e], sq);
          nmax = fmaxf(nmax, sqrtf(warp_sum(sq)));
        }
        if (lane == 0) s_red[warp] = nmax;
      }
      __syncthreads();
      if (p.append && m == cur && tid == 0) {
        float nm = 0.f;
        for (int w = 0; w < kWarps; ++w) nm = fmaxf(nm, s_red[w]);
        const size_t row = (size_t)(bi * p.Hk + kh) * p.C + cur;
        if (p.max_norm) p.max_norm[row] = nm;
        if (p.centre) p.centre[row] = 0.5f * (float)(cur * b) + 0.5f * (float)(cur * b + tok - 1);
      }
      for (int g = warp; g < G; g += kWarps) {
        float mx = -INFINITY;
        for (int t = lane; t < tok; t += 32) mx = fmaxf(mx, zs[t * G + g]);
        mx = warp_max(mx);
        const float m_old = s_m[g];
        const float m_new = fmaxf(m_old, mx);
        float sum = 0.f;
        for (int t = lane; t < tok; t += 32) {
          const float pvv = (m_new == -INFINITY) ? 0.f : exp2f(zs[t * G + g] - m_new);
          ps[t * G + g] = pvv;
          sum += pvv;
        }
        sum = warp_sum(sum);
        if (lane == 0) {
          const float corr = (m_old == -INFINITY) ? 0.f : exp2f(m_old - m_new);
          s_corr[g] = corr;
          s_l[g] = s_l[g] * corr + sum;
          s_m[g] = m_new;
        }
      }
      __syncthreads();
#pragma unroll
      for (int g = 0; g < G; ++g) {
        acc[g][0] *= s_corr[g];
        acc[g][1] *= s_corr[g];
      }
      for (int t = tp; t < tok; t += TP) {
        float vv[2];
        load_vec<T, 2>(vt + (size_t)t * D + 2 * cg, vv);
#pragma unroll
        for (int g = 0; g < G; ++g) {
          const float pw = ps[t * G + g];
          acc[g][0] = fmaf(pw, vv[0], acc[g][0]);
          acc[g][1] = fmaf(pw, vv[1], acc[g][1]);
        }
      }
      __syncthreads();
      if (tid == 0 && i + 2 < ne) issue_kv(i + 2);
    }
    if (s_abort && tid == 0) {
      for (int i = 0; i < 2; ++i) (void)mbar_wait_bounded(&kvbar[i], 0, 1u << 12);
      report_timeout(p.status, 2);
    }
    __syncthreads();
    // token partitions tp -> "warp partial" slots 0..TP-1 with the shared (m, l)
    for (int e = tid; e < kWarps * G * (D + 2); e += kThreads) wpart[e] = 0.f;
    __syncthreads();
#pragma unroll
    for (int g = 0; g < G; ++g) {
      float* wp = wpart + ((size_t)tp * G + g) * (D + 2);
      wp[2 * cg] = acc[g][0];
      wp[2 * cg + 1] = acc[g][1];
      if (cg == 0) {
        wp[D] = s_m[g];
        wp[D + 1] = tp == 0 ? s_l[g] : 0.f;
      }
    }
    for (int w = TP + tid; w < kWarps; w += kThreads)  // unused slots: empty
      for (int g = 0; g < G; ++g) wpart[((size_t)w * G + g) * (D + 2) + D] = -INFINITY;
    __syncthreads();
  }

  // ---- 4. merge the warps, push column slices to their owners, finish -----------------------
  const int cols = D / CL;
  // per head: combined max over warps, then weights
  for (int g = warp; g < G; g += kWarps) {
    float M = -INFINITY;
    if (lane < kWarps) M = wpart[((size_t)lane * G + g) * (D + 2) + D];
    M = warp_max(M);
    float lsum = 0.f;
    if (lane < kWarps) {
      const float mw = wpart[((size_t)lane * G + g) * (D + 2) + D];
      const float w = mw == -INFINITY ? 0.f : exp2f(mw - M);
      lsum = w * wpart[((size_t)lane * G + g) * (D + 2) + D + 1];
    }
    lsum = warp_sum(lsum);
    if (lane == 0) {
      s_m[g] = M;
      s_l[g] = lsum;
    }
  }
  __syncthreads();
  for (int e = tid; e < G * D; e += kThreads) {
    const int g = e / D, col = e % D;
    const float M = s_m[g];
    float osum = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      const float mw = wpart[((size_t)w * G + g) * (D + 2) + D];
      if (mw != -INFINITY) osum = fmaf(exp2f(mw - M), wpart[((size_t)w * G + g) * (D + 2) + col], osum);
    }
    // push to the owner of this column: recv[rank][g][col % cols], plus (m, l)
    const int owner = col / cols;
    float* slot = recv + ((size_t)rank * G + g) * (cols + 2);
    st_dsmem_f32(dsmem_addr(&slot[col % cols], owner), osum);
    if (col % cols == 0) {
      st_dsmem_f32(dsmem_addr(&slot[cols], owner), M);
      st_dsmem_f32(dsmem_addr(&slot[cols + 1], owner), s_l[g]);
    }
  }
  cluster_sync();
  for (int e = tid; e < G * cols; e += kThreads) {
    const int g = e / cols, cc = e % cols, col = rank * cols + cc;
    float M = -INFINITY;
    for (int r = 0; r < CL; ++r) M = fmaxf(M, recv[((size_t)r * G + g) * (cols + 2) + cols]);
    float lsum = 0.f, osum = 0.f;
    for (int r = 0; r < CL; ++r) {
      const float* slot = recv + ((size_t)r * G + g) * (cols + 2);
      const float mr = slot[cols];
      if (mr == -INFINITY) continue;
      const float w = exp2f(mr - M);
      lsum = fmaf(w, slot[cols + 1], lsum);
      osum = fmaf(w, slot[cc], osum);
    }
    const size_t row = (size_t)bi * Hq + h0 + g;
    static_cast<T*>(p.o)[row * D + col] = Elem<T>::from_f(osum / lsum);
    if (col == 0 && p.lse) p.lse[row] = (M + log2f(lsum)) * kLn2;
  }
}

int pick_cluster(int groups) {
  // the largest power of two (2..16) keeping every cluster resident at two CTAs per SM
  int cl = 2;
  while (cl * 2 <= kMaxCL && groups * cl * 2 <= 2 * kSMs) cl <<= 1;
  return cl;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
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

bool kv_map(CUtensorMap* m, const void* base, long long rows, int D) {
  auto enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)D * 2};
  cuuint32_t box[2] = {64, 64};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Host-side per-call costs kept off the decode path: the occupancy of a (device, kernel, shared
// memory, cluster size) and the shared-memory attribute of a kernel are looked up once.
struct LaunchCache {
  std::mutex mu;
  std::map<std::tuple<int, const void*, size_t, int>, int> clusters;  // -> max active clusters
  std::map<std::pair<int, const void*>, size_t> smem_set;              // -> attribute set to
};
LaunchCache& launch_cache() {
  static LaunchCache c;
  return c;
}

template <typename T, typename TS, int D, int G, bool MMA>
bsa_status launch_fused(FusedParams& p, cudaStream_t st) {
  using SM = FusedSmem<T, D, G, MMA>;
  CUtensorMap tmk{}, tmv{};
  if (MMA) {
    const long long rows = (long long)p.B * p.Hk * p.n;
    if (!kv_map(&tmk, p.k, rows, D) || !kv_map(&tmv, p.v, rows, D)) return BSA_ERR_CUDA;
  }
  const int groups = p.B * p.Hk;
  int CL = pick_cluster(groups);
  auto kern = decode_fused_kernel<T, TS, D, G, MMA>;
  for (;;) {
    const int chunk = std::max(kSub, ceil_div(ceil_div(std::max(p.C, 1), CL), kSub) * kSub);
    if (chunk > 32 * kSelItems) {  // the local select holds at most 512 keys per head
      if (CL < kMaxCL) { CL <<= 1; continue; }
      return BSA_ERR_UNSUPPORTED;
    }
    p.chunk = chunk;
    const size_t smem = SM::bytes(p.b, chunk, CL, p.K) + 1024;  // + alignment slack
    if (smem > 220 * 1024) return BSA_ERR_UNSUPPORTED;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
      (void)cudaGetLastError();
      return BSA_ERR_CUDA;
    }
    LaunchCache& lc = launch_cache();
    {
      std::lock_guard<std::mutex> lock(lc.mu);
      size_t& set_to = lc.smem_set[{dev, reinterpret_cast<const void*>(kern)}];
      if (set_to < smem) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
            cudaSuccess) {
          (void)cudaGetLastError();
          return BSA_ERR_CUDA;
        }
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) !=
            cudaSuccess)
          (void)cudaGetLastError();  // portable cluster sizes still work
        set_to = smem;
      }
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(CL, p.Hk, p.B);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = CL;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int nclusters = 0;
    {
      std::lock_guard<std::mutex> lock(lc.mu);
      const auto key = std::make_tuple(dev, reinterpret_cast<const void*>(kern), smem, CL);
      auto it = lc.clusters.find(key);
      if (it != lc.clusters.end()) {
        nclusters = it->second;
      } else {
        if (cudaOccupancyMaxActiveClusters(&nclusters, kern, &cfg) != cudaSuccess) {
          (void)cudaGetLastError();
          nclusters = 0;
        }
        lc.clusters[key] = nclusters;
      }
    }
    if (nclusters <= 0) {
      if (CL <= 2) return BSA_ERR_UNSUPPORTED;
      CL >>= 1;
      continue;
    }
    if (cudaLaunchKernelEx(&cfg, kern, tmk, tmv, p) != cudaSuccess) {
      (void)cudaGetLastError();
      return BSA_ERR_CUDA;
    }
    return BSA_OK;
  }
}

template <typename T, typename TS, int D, bool MMA>
bsa_status dispatch_fused(int G, FusedParams& p, cudaStream_t st) {
  switch (G) {
    case 1: return launch_fused<T, TS, D, 1, MMA>(p, st);
    case 2: return launch_fused<T, TS, D, 2, MMA>(p, st);
    case 4: return launch_fused<T, TS, D, 4, MMA>(p, st);
    case 8: return launch_fused<T, TS, D, 8, MMA>(p, st);
    default: return BSA_ERR_UNSUPPORTED;
  }
}

}  // namespace
}  // namespace bsa

extern "C" bsa_status bsa_decode_step_ex(const void* q, const void* k, const void* v,
                                         bsa_dtype dt, int B, int Hq, int Hk, int n, int d, int b,
                                         const int* seq_lens, void* mean_k, float* max_norm,
                                         float* centre, int append, const float* lambda_h,
                                         const float* sigma_h, int prefix_block, int K, void* o,
                                         float* lse, int* idx, int* count, int* status,
                                         int flags, void* stream) {
  using namespace bsa;
  BSA_REQUIRE(dtype_ok(dt), BSA_ERR_DTYPE);
  BSA_REQUIRE(q && k && v && mean_k && o, BSA_ERR_ARG);
  BSA_REQUIRE(B > 0 && Hq > 0 && Hk > 0 && n > 0 && d > 0 && b > 0 && K > 0 && prefix_block >= 0,
              BSA_ERR_ARG);
  BSA_REQUIRE((flags & ~(BSA_DECODE_SHARED_SELECTION | BSA_DECODE_BF16_SUMMARIES)) == 0,
              BSA_ERR_ARG);
  BSA_REQUIRE((lambda_h == nullptr) == (sigma_h == nullptr), BSA_ERR_ARG);
  BSA_REQUIRE(!lambda_h || (max_norm && centre), BSA_ERR_ARG);
  BSA_REQUIRE(Hq % Hk == 0, BSA_ERR_SHAPE);
  BSA_REQUIRE(group_ok(Hq, Hk), BSA_ERR_UNSUPPORTED);
  BSA_REQUIRE(head_dim_ok(d), BSA_ERR_UNSUPPORTED);
  BSA_REQUIRE(K <= kMaxKf && b <= 128, BSA_ERR_UNSUPPORTED);
  BSA_REQUIRE((size_t)b * d * (dt == BSA_BF16 ? 2 : 4) <= 32768, BSA_ERR_UNSUPPORTED);
  BSA_REQUIRE(B <= 65535 && Hk <= 65535, BSA_ERR_UNSUPPORTED);
  BSA_REQUIRE(all_aligned16(q, k, v, o, mean_k), BSA_ERR_ARG);
  const bool bf16_sum = (flags & BSA_DECODE_BF16_SUMMARIES) != 0;
  // bf16 summaries ride on the 64-token bf16 path (warp MMAs over TMA tiles)
  BSA_REQUIRE(!bf16_sum || (dt == BSA_BF16 && b == 64), BSA_ERR_UNSUPPORTED);
  const int C = ceil_div(n, b);
  BSA_REQUIRE(C <= kMaxWords * 32, BSA_ERR_UNSUPPORTED);
  FusedParams p{};
  p.q = q; p.k = k; p.v = v;
  p.B = B; p.Hq = Hq; p.Hk = Hk; p.n = n; p.b = b; p.C = C; p.K = K;
  p.seq_lens = seq_lens; p.mean_k = mean_k; p.max_norm = max_norm; p.centre = centre;
  p.append = append; p.lam = lambda_h; p.sig = sigma_h; p.prefix_block = prefix_block;
  p.o = o; p.lse = lse; p.idx = idx; p.count = count; p.status = status;
  p.shared = (flags & BSA_DECODE_SHARED_SELECTION) != 0;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  using bf = __nv_bfloat16;
  bsa_status rc;
  if (dt == BSA_BF16 && b == 64 && bf16_sum)
    rc = d == 64 ? dispatch_fused<bf, bf, 64, true>(Hq / Hk, p, st)
                 : dispatch_fused<bf, bf, 128, true>(Hq / Hk, p, st);
  else if (dt == BSA_BF16 && b == 64)  // 64-token blocks: warp MMAs over swizzled TMA tiles
    rc = d == 64 ? dispatch_fused<bf, float, 64, true>(Hq / Hk, p, st)
                 : dispatch_fused<bf, float, 128, true>(Hq / Hk, p, st);
  else if (dt == BSA_BF16)
    rc = d == 64 ? dispatch_fused<bf, float, 64, false>(Hq / Hk, p, st)
                 : dispatch_fused<bf, float, 128, false>(Hq / Hk, p, st);
  else
    rc = d == 64 ? dispatch_fused<float, float, 64, false>(Hq / Hk, p, st)
                 : dispatch_fused<float, float, 128, false>(Hq / Hk, p, st);
  if (rc != BSA_OK) return rc;
  BSA_LAUNCH_CHECK();
  return BSA_OK;
}

extern "C" bsa_status bsa_decode_step(const void* q, const void* k, const void* v, bsa_dtype dt,
                                      int B, int Hq, int Hk, int n, int d, int b,
                                      const int* seq_lens, float* mean_k, float* max_norm,
                                      float* centre, int append, const float* lambda_h,
                                      const float* sigma_h, int prefix_block, int K, void* o,
                                      float* lse, int* idx, int* count, int* status,
                                      void* stream) {
  return bsa_decode_step_ex(q, k, v, dt, B, Hq, Hk, n, d, b, seq_lens, mean_k, max_norm, centre,
                            append, lambda_h, sigma_h, prefix_block, K, o, lse, idx, count,
                            status, 0, stream);
}
