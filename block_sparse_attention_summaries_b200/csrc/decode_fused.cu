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
//   1. CTA r scores its slice of the history blocks.  Its mean-key rows stream through a ring of
//      shared-memory stages filled by bulk copies (TMA engine), every stage issued at the start
//      (refilled as they drain when the slice is larger than the ring); the G query heads of the
//      group share every row (one 31-shuffle transpose-reduce per 32/G rows).
//   2. Selection.  When the history fits one warp select (<= 512 blocks) every CTA pushes its
//      slice's order keys into every peer's copy of the whole row (DSMEM vector stores), and after
//      one cluster barrier each CTA selects every head's Top-K from the whole row itself.  Longer
//      histories select a local Top-K per slice and merge the CL x K candidates the same way.
//      The warp select takes the K-th largest of 64 group maxima as a threshold (at least K keys
//      lie at or above it), compacts the keys at or above it in index order and ranks them
//      exactly; a radix select with 4-bit digits is the fallback when too many keys pass.
//   3. Each CTA builds the sorted union of the G heads' selections (a bitmap over the history
//      blocks, compacted by one warp) plus the current block, with a head mask per entry.
//   4. bf16, 64-token blocks: the union's tokens are cut into 16-token slices and every CTA of
//      the cluster takes an equal contiguous range of them; slices arrive as 128-byte swizzled
//      16-row TMA boxes, four slices per stage, through a ring of stages; one group of four warps
//      takes a stage, each warp one slice, and computes S = Q K^T and O += P V with warp-level
//      MMAs (the G heads padded to 16 rows) with its own online-softmax state, so the per-slice
//      work is ~30 MMAs per warp instead of ~1,200 scalar FMAs/shuffles.  Other block sizes and
//      fp32: CTA r attends union entries r, r+CL, ... with scalar FMAs, the CTA holding the
//      current block rewriting that block's summary from shared memory.
//   5. Each CTA merges its warps, then pushes to CTA r' the partial (m, l, o) of the output columns
//      CTA r' owns; cluster barrier; each CTA finishes its columns and writes o (and lse).
// On the 64-token bf16 path the summary of the block being filled is rewritten by the last CTA of
// the cluster from global memory, while its first K/V stages are in flight.
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
constexpr int kSelItems = 16;     // keys per lane of one warp select: N <= 512
constexpr int kSelMax = 32 * kSelItems;
constexpr int kCandMax = 64;      // candidates the threshold pass may leave for exact ranking
constexpr int kScratchPerWarp = 2 * kCandMax + 4;  // candidate keys (+ 4 padding), positions
constexpr int kMaxStages = 8;     // ring stages (summaries or K/V)
constexpr int kSlice = 16;        // tokens per warp slice (64-token bf16 path)
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
  int chunk;   // history blocks scored per CTA (multiple of kSub)
  int shared;  // one selection per kv head from the mean of its heads' scores
  int gather;  // whole-row selection (history <= kSelMax blocks) instead of local + merge
  int row_ld;  // stride of the whole-row key copies (gather) in keys
  int ns;      // summary ring stages
  int nkv;     // K/V ring stages
  int host_io;  // q and o through their device mappings of page-locked host memory (modes 0, 2)
  // Long histories in two launches: mode 1 scores one chunk of the history per CTA (no cluster)
  // and writes every selecting head's chunk Top-K to `cand`; mode 2 merges those lists and runs
  // phases 3-5.  Mode 0 is the whole step in one launch.
  int mode;
  // Mode 3 is the attention of a given selection (the decode form of bsa_sparse_attn_fwd):
  // phases 3-5 over sel_idx [B, Hq, K] (entries outside the history ignored), sel_count [B, Hq].
  const int* sel_idx;
  const int* sel_count;
  int nchunk;      // chunks per group (modes 1 and 2)
  int cand_ld;     // words per (chunk, head) record: K keys, K positions (rank order), count
  uint32_t* cand;  // [B * Hk][nchunk][Gs][cand_ld]
  // dynamic shared-memory layout (byte offsets from the 1024-aligned base)
  int off_keys, off_sel, off_hbits, off_recv, off_zp, off_bar;
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
__device__ __forceinline__ void cluster_arrive_relaxed() {
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
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
__device__ __forceinline__ void st_dsmem_v4(uint32_t addr, uint4 v) {
  asm volatile("st.shared::cluster.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x),
               "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}
// Arrive, with release at cluster scope, on the mbarrier at a shared::cluster address.
__device__ __forceinline__ void mbar_arrive_remote(uint32_t addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(addr)
               : "memory");
}
// Bounded wait with acquire at cluster scope (for a phase completed by another CTA's arrive).
__device__ __forceinline__ bool mbar_wait_cluster_bounded(uint64_t* bar, uint32_t parity,
                                                          uint32_t limit = (1u << 20)) {
  for (uint32_t it = 0; it < limit; ++it) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    if (ok) return true;
  }
  return false;
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

// ---- warp Top-K selection -------------------------------------------------------------------
// All selections rank order keys (larger first) and break ties toward the lower position; the
// positions of the winners are written ascending.

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

// Exact rank select over N <= 32 R keys: rank every key by counting the keys above it (ties: the
// lower position ranks higher) and keep ranks below kk -- N broadcast loads per lane.
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
#pragma unroll 4
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

// Exact radix select with 4-bit digits (lane l holds positions l + 32 j in registers).
// Each pass counts the next digit of the keys that share the prefix found so far: every lane keeps
// sixteen 4-bit counters in one 64-bit word (at most 8 keys between two flushes into 16-bit
// fields), the eight 32-bit words of 16-bit bins are summed over the warp, and the pass keeps the
// digit at which the count of keys at or above the threshold reaches K.  It stops as soon as that
// count is exactly K ({key >= T} is then the answer); otherwise after the last digit T is the K-th
// largest key and the lowest-indexed keys equal to T fill the remaining places.
__device__ __noinline__ int warp_select_radix(const uint32_t* keys, int N, int kk, int lane,
                                              int* out) {
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

// Top-min(K, N) of N <= kSelMax order keys (shared memory, index order) by one warp; writes the
// winners' positions ascending to `out`, returns their number.  `ck` / `cp` are the warp's
// scratch for kCandMax candidate keys / positions (ck 16-byte aligned, kCandMax + 4 entries).
//
// Threshold pass: lane l holds positions l + 32 j; the even-j and odd-j keys of every lane form 64
// groups.  T0 = the kk-th largest group maximum (a bitonic sort of the 64 maxima across the warp,
// fifteen shuffle stages): the kk groups whose maxima reach T0 hold kk distinct keys >= T0, so
// every key of the Top-kk is >= T0.  The keys >= T0 are compacted in position order (usually a few
// more than kk) and ranked exactly; if more than kCandMax pass, the radix select runs on all N
// keys instead.  Every step is a short dependency chain: the sixteen compaction ballots are
// independent of one another and the ranking reads the candidates four at a time.
__device__ __noinline__ int warp_select(const uint32_t* keys, int N, int K, int lane, int* out,
                                           uint32_t* ck, int* cp) {
  const int kk = min(K, N);
  if (kk <= 0) return 0;
  if (kk == N) {
    for (int i = lane; i < N; i += 32) out[i] = i;
    __syncwarp();
    return N;
  }
  if (N <= kCandMax) return warp_select_rank<kCandMax / 32>(keys, N, kk, lane, out);
  const int nv = (N - lane + 31) >> 5;  // keys of this lane: positions lane + 32 j, j < nv
  uint32_t kr[kSelItems];
#pragma unroll
  for (int j = 0; j < kSelItems; ++j) kr[j] = j < nv ? keys[lane + 32 * j] : 0u;
  // group maxima: element e = 2 lane + h of the 64 (h = 0: even j, h = 1: odd j)
  uint32_t v0 = 0u, v1 = 0u;
#pragma unroll
  for (int j = 0; j < kSelItems; j += 2) {
    v0 = max(v0, kr[j]);
    v1 = max(v1, kr[j + 1]);
  }
  // bitonic sort of the 64 maxima, descending: in a block of size k the lower element of a
  // compared pair keeps the larger value when the block runs downward ((e & k) == 0)
#pragma unroll
  for (int k = 2; k <= 64; k <<= 1) {
    const bool down = ((2 * lane) & k) == 0;
#pragma unroll
    for (int jj = k >> 1; jj > 0; jj >>= 1) {
      if (jj == 1) {  // the pair sits in one lane
        const uint32_t hi = max(v0, v1), lo = min(v0, v1);
        v0 = down ? hi : lo;
        v1 = down ? lo : hi;
      } else {
        const int lm = jj >> 1;  // partner lane distance
        const uint32_t w0 = __shfl_xor_sync(0xffffffffu, v0, lm);
        const uint32_t w1 = __shfl_xor_sync(0xffffffffu, v1, lm);
        const bool keep_max = ((lane & lm) == 0) == down;
        v0 = keep_max ? max(v0, w0) : min(v0, w0);
        v1 = keep_max ? max(v1, w1) : min(v1, w1);
      }
    }
  }
  const uint32_t T0 = __shfl_sync(0xffffffffu, ((kk - 1) & 1) ? v1 : v0, (kk - 1) >> 1);
  uint32_t cm = 0u;  // my candidates: bit j for position 32 j + lane
#pragma unroll
  for (int j = 0; j < kSelItems; ++j) cm |= (j < nv && kr[j] >= T0) ? (1u << j) : 0u;
  const int cnt = __reduce_add_sync(0xffffffffu, __popc(cm));
  if (cnt > kCandMax) return warp_select_radix(keys, N, kk, lane, out);
  // compact in position order: the candidates at j take places P_j + (rank among lanes), P_j the
  // candidates at smaller j
  const unsigned lt = (1u << lane) - 1u;
  unsigned bal[kSelItems];
#pragma unroll
  for (int j = 0; j < kSelItems; ++j) bal[j] = __ballot_sync(0xffffffffu, (cm >> j) & 1u);
  int base = 0;
#pragma unroll
  for (int j = 0; j < kSelItems; ++j) {
    if ((cm >> j) & 1u) {
      const int at = base + __popc(bal[j] & lt);
      ck[at] = kr[j];
      cp[at] = 32 * j + lane;
    }
    base += __popc(bal[j]);
  }
  if (lane < 4) ck[cnt + lane] = 0u;  // padding of the last group of four (never taken)
  __syncwarp();
  // rank the candidates (ties: the lower position ranks higher); the winners keep the
  // candidates' ascending position order
  uint32_t mk[2];
  int rk[2];
#pragma unroll
  for (int q = 0; q < 2; ++q) {
    mk[q] = lane + 32 * q < cnt ? ck[lane + 32 * q] : 0u;
    rk[q] = 0;
  }
  const uint4* ck4 = reinterpret_cast<const uint4*>(ck);
  const int n4 = (cnt + 3) >> 2;
#pragma unroll 4
  for (int c = 0; c < n4; ++c) {
    const uint4 g4 = ck4[c];
    const uint32_t kv[4] = {g4.x, g4.y, g4.z, g4.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int j = 4 * c + e;
#pragma unroll
      for (int q = 0; q < 2; ++q)
        rk[q] += (kv[e] > mk[q] || (kv[e] == mk[q] && j < lane + 32 * q)) ? 1 : 0;
    }
  }
  int taken = 0;
  const int mypos[2] = {lane < cnt ? cp[lane] : 0, lane + 32 < cnt ? cp[lane + 32] : 0};
  __syncwarp();
#pragma unroll
  for (int q = 0; q < 2; ++q) {
    const bool take = lane + 32 * q < cnt && rk[q] < kk;
    const unsigned tb = __ballot_sync(0xffffffffu, take);
    if (take) out[taken + __popc(tb & lt)] = mypos[q];
    taken += __popc(tb);
  }
  __syncwarp();
  return taken;
}

// Bitonic sort of one value per lane across the warp: descending (largest at lane 0) or ascending.
template <typename V, bool kDescending>
__device__ __forceinline__ V warp_sort(V v, int lane) {
#pragma unroll
  for (int k = 2; k <= 32; k <<= 1) {
#pragma unroll
    for (int j = k >> 1; j > 0; j >>= 1) {
      const V o = __shfl_xor_sync(0xffffffffu, v, j);
      // the block of size k runs in the final direction when (lane & k) == 0; the lower lane of
      // a pair keeps the value that comes first in its block's direction
      const bool first = (((lane & k) == 0) == ((lane & j) == 0));
      v = (first == kDescending) ? (v > o ? v : o) : (v < o ? v : o);
    }
  }
  return v;
}

// The largest 64-bit value over the warp (two 32-bit reductions: the high words, then the low
// words of the lanes holding the largest high word).
__device__ __forceinline__ unsigned long long warp_max_u64(unsigned long long v) {
  const uint32_t hi = __reduce_max_sync(0xffffffffu, (uint32_t)(v >> 32));
  const uint32_t lo = __reduce_max_sync(0xffffffffu, (uint32_t)(v >> 32) == hi ? (uint32_t)v : 0u);
  return ((unsigned long long)hi << 32) | lo;
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
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
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

// Byte sizes of the pieces of the dynamic shared memory (host and device agree through them).
template <typename T, typename TS, int D, int G, bool MMA>
struct FusedSmem {
  // one K/V stage: four 16-token slices (MMA) or one whole block (scalar path), K then V
  __host__ __device__ static size_t kv_tile(int b) {
    return align_up((size_t)(MMA ? 64 : b) * D * sizeof(T), 1024);
  }
  __host__ __device__ static size_t kv_stage(int b) { return 2 * kv_tile(b); }
  __host__ __device__ static size_t sum_stage() { return (size_t)kSub * D * sizeof(TS); }
  __host__ __device__ static size_t partials() {
    return align_up((size_t)kWarps * G * (D + 2) * 4, 1024);
  }
  __host__ __device__ static size_t keys(int chunk) { return align_up((size_t)G * chunk * 4, 16); }
  __host__ __device__ static size_t sel(int gather, int row_ld, int CL, int K) {
    return gather ? align_up((size_t)G * row_ld * 4, 16) : align_up((size_t)G * CL * K * 8, 16);
  }
  // per-head selection bitmaps, the union bitmap and the union's prefix counts per word
  __host__ __device__ static size_t hbits(int C) { return align_up((size_t)(G + 2) * ((C + 31) / 32) * 4, 16); }
  __host__ __device__ static size_t recv(int CL) {
    return align_up((size_t)CL * G * (D / CL + 2) * 4, 16);
  }
  __host__ __device__ static size_t zp(int b) { return MMA ? 0 : 2 * align_up((size_t)b * G * 4, 16); }
};

// kMode: 0 the whole step; 1 and 2 the two launches of a long history; 3 the attention of a given
// selection (FusedParams::mode), each its own instantiation so that the one-launch step's code is
// unchanged by them.
// kHostIO: q and o through their device mappings of page-locked host memory (its own
// instantiation too: the staging of q and the packed stores of o leave the device-buffer code
// unchanged).
template <typename T, typename TS, int D, int G, bool MMA, int kMode = 0, bool kHostIO = false>
__global__ void __launch_bounds__(kThreads, 2) decode_fused_kernel(
    const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv,
    const __grid_constant__ CUtensorMap tmk64, const __grid_constant__ CUtensorMap tmv64,
    const FusedParams p) {
  constexpr bool kMma = MMA;
  static_assert(!MMA || std::is_same<T, __nv_bfloat16>::value, "warp MMAs take bf16");
  static_assert(kMode == 0 || MMA, "modes 1-3 are the 64-token bf16 path");
  static_assert(!kHostIO || (MMA && (kMode == 0 || kMode == 2)), "host I/O: cluster steps");
  constexpr int EPL = D / 32;
  constexpr int R = 32 / G;

  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = smem_align1024(smem_raw);
  __shared__ int s_pick[kWarps][kMaxKf];
  __shared__ int s_sel[G][kMaxKf];
  __shared__ int s_nsel[G];
  __shared__ int s_ublk[kMaxUnion];
  __shared__ unsigned s_umask[kMaxUnion];
  // select candidates (per warp: kCandMax + 4 keys, kCandMax positions) / append partials
  __shared__ __align__(16) uint32_t s_scratch[kWarps * kScratchPerWarp];
  __shared__ int s_kv_par[kMaxStages];   // phase parity of the last copy into each slot (-1: none)
  __shared__ int s_gst[kMaxStages];      // global K/V stage held by each slot (-1: none left)
  __shared__ unsigned s_next;            // (rank 0) dynamic K/V stages handed out so far
  __shared__ int s_U;
  __shared__ int s_abort;
  __shared__ float s_red[kWarps];
  __shared__ float s_m[G], s_l[G], s_corr[G];
  __shared__ float s_wt[G][kWarps];  // merge weights of the warp partials
  __shared__ float s_fw[G][kMaxCL];  // merge weights of the CTAs' partials (owner side)
  __shared__ float s_fm[G], s_fl[G];
  // With q in page-locked host memory, the group's G query rows are read once by rank 0 of the
  // cluster and pushed to every CTA (one read of q per group).  bf16 path, cluster modes.
  constexpr bool kStageQ = kHostIO;
  __shared__ __align__(16) T s_q[kStageQ ? G * D : 8];
  __shared__ __align__(8) uint64_t s_qbar;
  static_assert(kWarps * kScratchPerWarp >= kWarps * 128, "append partials fit the scratch");

  // The K/V tensor maps are kernel parameters: their descriptors are fetched while the launch
  // waits, not at the first copy after the selection.
  if (kMma && threadIdx.x == 0) {
    tc::prefetch_tmap(&tmk);
    tc::prefetch_tmap(&tmv);
    tc::prefetch_tmap(&tmk64);
    tc::prefetch_tmap(&tmv64);
  }
  // Programmatic dependent launch: every input may come from the work queued before this kernel
  // on the stream, so nothing is read before that work has completed and its writes are visible;
  // a launch queued after this one may be scheduled at once and wait the same way.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int b = p.b, K = p.K, Hq = p.Hq;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // mode 1 runs without clusters: the CTA's chunk is its x index
  const int rank = kMode == 1 ? (int)blockIdx.x : (int)cluster_rank();
  const int CL = kMode == 1 ? (int)gridDim.x : (int)cluster_size();
  const int kh = blockIdx.y, bi = blockIdx.z;
  const int h0 = kh * G;
  const int L = p.seq_lens ? min(p.seq_lens[bi], p.n) : p.n;
  const int pos = L - 1;
  const int cur = pos / b;
  int nc = p.prefix_block > 0 ? ((pos / p.prefix_block) * p.prefix_block) / b : cur;
  nc = max(0, min(nc, cur));
  const int NS = p.ns, NKV = p.nkv;

  using SM = FusedSmem<T, TS, D, G, MMA>;
  TS* ring = reinterpret_cast<TS*>(smem);  // region A: summary ring, then K/V ring, then partials
  TS* mean_k = static_cast<TS*>(p.mean_k);
  uint32_t* s_keys = reinterpret_cast<uint32_t*>(smem + p.off_keys);  // [G][chunk]
  uint32_t* sel_buf = reinterpret_cast<uint32_t*>(smem + p.off_sel);  // whole rows / merge
  uint32_t* hbits = reinterpret_cast<uint32_t*>(smem + p.off_hbits);  // [Gs][nwords] selections
  float* recv = reinterpret_cast<float*>(smem + p.off_recv);  // [CL][G][cols], then [CL][G][2]
  float* zs = reinterpret_cast<float*>(smem + p.off_zp);
  float* ps = zs + align_up((size_t)b * G, 4);
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + p.off_bar);
  // bar[0 .. NS): summary stages; bar[NS .. NS + NKV): K/V stages

  if (tid == 0) {
    for (int i = 0; i < NS + NKV; ++i) mbar_init(&bar[i], 1);
    if constexpr (kStageQ) mbar_init(&s_qbar, 1);
    fence_mbar_init();
    if (kMode == 2) {  // the group's chunk lists (one contiguous block) into region A, first
      const size_t words = (size_t)p.nchunk * (p.shared ? 1 : G) * p.cand_ld;
      mbar_arrive_expect_tx(&bar[0], (uint32_t)(words * 4));
      bulk_g2s(ring, p.cand + (size_t)(bi * p.Hk + kh) * words, (uint32_t)(words * 4), &bar[0]);
    }
    for (int i = 0; i < kMaxStages; ++i) s_kv_par[i] = -1;
    s_next = 0;
    s_abort = 0;
    s_U = 0;
  }
  if (tid < G) {
    s_m[tid] = -INFINITY;
    s_l[tid] = 0.f;
  }
  const int Gs = p.shared ? 1 : G;  // selections made per group
  const int nwords = (nc + 31) / 32;
  uint32_t* s_ubits = hbits + Gs * nwords;  // union of the selections over the history blocks
  int* s_upre = reinterpret_cast<int*>(s_ubits + nwords);  // union entries before each word
  if (kMode != 1)
    for (int e = tid; e < (Gs + 1) * nwords; e += kThreads) hbits[e] = 0u;
  __syncthreads();
  // every CTA of the cluster has started before any peer writes into its shared memory
  if (kMode != 1) cluster_arrive_relaxed();

  // ---- 1. score my slice of the history blocks --------------------------------------------
  const int c_lo = min(nc, rank * p.chunk);
  const int c_hi = min(nc, c_lo + p.chunk);
  const int rows = c_hi - c_lo;
  const int nsub = kMode >= 2 ? 0 : (rows + kSub - 1) / kSub;  // modes 2 and 3 score nothing
  const TS* mk = mean_k + ((size_t)(bi * p.Hk + kh) * p.C) * D;
  // summaries and K/V are read once per step: their L2 lines go first, so that the kernel's code
  // (fetched again by every launch) stays in L2 (the policy is made where it is used: one
  // instruction, no register held across the kernel)
  auto issue_sub = [&](int j) {
    const int r0 = c_lo + j * kSub;
    const int nr = min(kSub, c_hi - r0);
    const uint32_t bytes = (uint32_t)(nr * D * sizeof(TS));
    mbar_arrive_expect_tx(&bar[j % NS], bytes);
    bulk_g2s_stream(ring + (size_t)(j % NS) * kSub * D, mk + (size_t)r0 * D, bytes, &bar[j % NS],
                    l2_evict_first());
  };
  int sub_issued = 0;  // (thread 0) summary stages issued so far
  if (tid == 0)
    for (; sub_issued < min(nsub, NS); ++sub_issued) issue_sub(sub_issued);
  const int cand_group = Gs * p.cand_ld;  // mode 2: words per chunk of the lists
  const T* qsrc = static_cast<const T*>(p.q) + ((size_t)bi * Hq + h0) * D;  // the G rows
  constexpr bool stage_q = kStageQ;
  if constexpr (stage_q) {
    // rank 0 reads the G rows once and pushes them to every CTA, then arrives on each CTA's q
    // barrier (its threads wait for the cluster here; the other CTAs' threads in phase 2)
    constexpr int kQ16 = G * D * (int)sizeof(T) / 16;
    static_assert(kQ16 <= kThreads, "one 16-byte piece of q per thread");
    if (rank == 0) {
      uint4 x = make_uint4(0u, 0u, 0u, 0u);
      if (tid < kQ16) x = reinterpret_cast<const uint4*>(qsrc)[tid];
      cluster_wait();  // every peer has started: DSMEM stores may begin
      if (tid < kQ16)
        for (int r = 0; r < CL; ++r) st_dsmem_v4(dsmem_addr(reinterpret_cast<uint4*>(s_q) + tid, r), x);
      __syncthreads();
      if (tid < CL) mbar_arrive_remote(dsmem_addr(&s_qbar, tid));
    }
    if (!mbar_wait_cluster_bounded(&s_qbar, 0)) s_abort = 1;  // reported with phase 1's timeouts
    qsrc = s_q;
  }
  float qv[G][EPL];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    float tmp[EPL];
    load_vec<T, EPL>(qsrc + (size_t)g * D + lane * EPL, tmp);
#pragma unroll
    for (int e = 0; e < EPL; ++e) qv[g][e] = tmp[e];
  }
  const float scale = rsqrtf((float)D);
  const int my_r = lane / G, my_g = lane % G;
  const float lam_h = p.lam ? p.lam[h0 + my_g] : 0.f;
  const float inv2sig = p.lam ? 0.5f / p.sig[h0 + my_g] : 0.f;
  for (int j = 0; j < nsub; ++j) {
    if (!s_abort && !mbar_wait_bounded(&bar[j % NS], (j / NS) & 1)) s_abort = 1;
    __syncthreads();
    if (!s_abort) {
      const int r0 = j * kSub;
      const int nr = min(kSub, rows - r0);
      const TS* base = ring + (size_t)(j % NS) * kSub * D;
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
    if (j + NS < nsub) {  // the stage is drained: refill it
      __syncthreads();
      if (tid == 0 && !s_abort) issue_sub(sub_issued++);
    }
  }
  __syncthreads();
  if (s_abort && tid == 0) {
    // summary copies still in flight: the last stage issued into each slot, on its own parity
    for (int j = max(0, sub_issued - NS); j < sub_issued; ++j)
      (void)mbar_wait_bounded(&bar[j % NS], (j / NS) & 1, 1u << 12);
    report_timeout(p.status, 1);
  }

  // ---- 2. Top-K per head (per group when shared) -----------------------------------------
  uint32_t* ck = s_scratch + warp * kScratchPerWarp;
  int* cp = reinterpret_cast<int*>(ck + kCandMax + 4);
  // every peer has started: DSMEM stores may begin (rank 0 of a q-staging launch waited already)
  if (kMode != 1 && !(stage_q && rank == 0)) cluster_wait();
  if constexpr (kMode == 1) {
    // this chunk's Top-K of every selecting head in rank order (key descending, ties to the lower
    // block: the pair sorts as key, then the complement of the block index), with its count
    for (int g = warp; g < Gs; g += kWarps) {
      const uint32_t* keys = s_keys + g * p.chunk;
      const int cnt = s_abort ? 0 : warp_select(keys, rows, K, lane, s_pick[warp], ck, cp);
      unsigned long long e = 0ull;  // empty places sort last
      if (lane < cnt)
        e = ((unsigned long long)keys[s_pick[warp][lane]] << 32) |
            (unsigned long long)(~(uint32_t)(c_lo + s_pick[warp][lane]));
      e = warp_sort<unsigned long long, true>(e, lane);
      uint32_t* rec = p.cand + (((size_t)(bi * p.Hk + kh) * p.nchunk + rank) * Gs + g) * p.cand_ld;
      if (lane < cnt) {
        rec[lane] = (uint32_t)(e >> 32);
        rec[K + lane] = ~(uint32_t)e;
      }
      if (lane == 0) rec[2 * K] = (uint32_t)cnt;
    }
    return;
  }
  if constexpr (kMode == 3) {
    // the given selection of every head: entries outside the history are ignored, repeats
    // collapse in the bitmaps
    const unsigned lt = (1u << lane) - 1u;
    for (int g = warp; g < G; g += kWarps) {
      const size_t row = (size_t)bi * Hq + h0 + g;
      const int cnt = p.sel_count ? min(p.sel_count[row], K) : K;
      int taken = 0;
      for (int j0 = 0; j0 < cnt; j0 += 32) {
        const int j = j0 + lane;
        const int m = j < cnt ? p.sel_idx[row * K + j] : -1;
        const bool good = j < cnt && m >= 0 && m < nc;
        const unsigned bal = __ballot_sync(0xffffffffu, good);
        if (good) {
          s_sel[g][taken + __popc(bal & lt)] = m;
          atomicOr(&hbits[g * nwords + (m >> 5)], 1u << (m & 31));
          atomicOr(&s_ubits[m >> 5], 1u << (m & 31));
        }
        taken += __popc(bal);
      }
      if (lane == 0) s_nsel[g] = taken;
    }
  } else if constexpr (kMode == 2) {
    // Merge of the chunk lists.  Each list is in rank order; an entry is its key, then the
    // complement of its block index (never 0; 0 marks "none").  Lane c follows chunk c's list
    // with its head and the entry after it.  Every entry below a head is at most the largest of
    // those next entries X, so all heads above X are larger than everything left outside the
    // heads: a round takes them all at once (while they fit in K; otherwise one round takes the
    // largest head alone) and advances their lists.  The K taken are the K largest of the whole
    // history, since each of them is in its chunk's list.
    if (!s_abort && !mbar_wait_bounded(&bar[0], 0)) s_abort = 1;
    __syncthreads();
    const uint32_t* blk = reinterpret_cast<const uint32_t*>(ring);
    const unsigned lt = (1u << lane) - 1u;
    for (int g = warp; g < Gs && !s_abort; g += kWarps) {
      const uint32_t* rec = blk + (size_t)min(lane, p.nchunk - 1) * cand_group + g * p.cand_ld;
      const int n_c = lane < p.nchunk ? (int)rec[2 * K] : 0;
      auto entry = [&](int j) -> unsigned long long {
        return j < n_c ? ((unsigned long long)rec[j] << 32) | (unsigned long long)(~rec[K + j])
                       : 0ull;
      };
      int ptr = 0;
      unsigned long long hc = entry(0), nx = entry(1);
      int* out = s_pick[warp];
      int taken = 0;
      while (taken < K) {
        if (__ballot_sync(0xffffffffu, hc != 0ull) == 0u) break;
        const unsigned long long X = warp_max_u64(nx);
        bool take = hc != 0ull && hc > X;
        unsigned tb = __ballot_sync(0xffffffffu, take);
        if (taken + __popc(tb) > K) {  // too many at once: the largest head alone
          const unsigned long long m = warp_max_u64(hc);
          take = hc != 0ull && hc == m;
          tb = __ballot_sync(0xffffffffu, take);
        }
        if (take) {
          out[taken + __popc(tb & lt)] = (int)~(uint32_t)hc;
          ++ptr;
          hc = nx;
          nx = entry(ptr + 1);
        }
        taken += __popc(tb);
      }
      __syncwarp();
      int mine = lane < taken ? out[lane] : 0x7fffffff;
      mine = warp_sort<int, false>(mine, lane);  // ascending block order
      if (lane < taken) {
        s_sel[g][lane] = mine;
        atomicOr(&hbits[g * nwords + (mine >> 5)], 1u << (mine & 31));
        atomicOr(&s_ubits[mine >> 5], 1u << (mine & 31));
      }
      if (lane == 0) s_nsel[g] = taken;
    }
    if (s_abort && tid == 0) {
      (void)mbar_wait_bounded(&bar[0], 0, 1u << 12);  // the copy may still be in flight
      report_timeout(p.status, 1);
    }
    if (s_abort && tid < Gs) s_nsel[tid] = 0;
  } else if (p.gather) {
    // push my slice of every selecting head's keys into every CTA's whole-row copy
    const int nvec = rows >> 2, tail = rows & 3;
    const int per_g = CL * (nvec + tail);
    for (int e = tid; e < Gs * per_g; e += kThreads) {
      const int g = e / per_g, rem = e % per_g;
      const int r = rem / (nvec + tail), v = rem % (nvec + tail);
      const uint32_t* src = s_keys + g * p.chunk;
      uint32_t* dst = sel_buf + (size_t)g * p.row_ld + c_lo;
      if (v < nvec) {
        const uint4 x = *reinterpret_cast<const uint4*>(src + 4 * v);
        st_dsmem_v4(dsmem_addr(dst + 4 * v, r), x);
      } else {
        const int t = 4 * nvec + (v - nvec);
        st_dsmem_u32(dsmem_addr(dst + t, r), src[t]);
      }
    }
    cluster_sync();
    for (int g = warp; g < Gs; g += kWarps) {
      const int cnt = warp_select(sel_buf + (size_t)g * p.row_ld, nc, K, lane, s_pick[warp], ck, cp);
      for (int j = lane; j < cnt; j += 32) {
        const int x = s_pick[warp][j];
        s_sel[g][j] = x;
        atomicOr(&hbits[g * nwords + (x >> 5)], 1u << (x & 31));
        atomicOr(&s_ubits[x >> 5], 1u << (x & 31));
      }
      if (lane == 0) s_nsel[g] = cnt;
    }
  } else {
    // local Top-K per head, pushed into every CTA's merge buffer at slot rank * K
    uint32_t* m_key = sel_buf;
    int* m_idx = reinterpret_cast<int*>(sel_buf) + G * CL * K;
    for (int g = warp; g < Gs; g += kWarps) {
      const uint32_t* keys = s_keys + g * p.chunk;
      const int cnt = warp_select(keys, rows, K, lane, s_pick[warp], ck, cp);
      for (int e = lane; e < CL * K; e += 32) {
        const int r = e / K, j = e % K;
        const uint32_t key = j < cnt ? keys[s_pick[warp][j]] : 0u;
        const int gi = j < cnt ? c_lo + s_pick[warp][j] : -1;  // -1: empty slot
        const int slot = g * CL * K + rank * K + j;
        st_dsmem_u32(dsmem_addr(&m_key[slot], r), key);
        st_dsmem_u32(dsmem_addr(&m_idx[slot], r), (uint32_t)gi);
      }
    }
    cluster_sync();
    for (int g = warp; g < Gs; g += kWarps) {
      // empty slots carry key 0 and index -1: compact the valid ones first (index order kept:
      // slot order is rank order and each rank's slots are ascending)
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
      const int cnt = warp_select(mk_g, nvalid, K, lane, s_pick[warp], ck, cp);
      for (int j = lane; j < cnt; j += 32) {
        const int x = mi_g[s_pick[warp][j]];
        s_sel[g][j] = x;
        atomicOr(&hbits[g * nwords + (x >> 5)], 1u << (x & 31));
        atomicOr(&s_ubits[x >> 5], 1u << (x & 31));
      }
      if (lane == 0) s_nsel[g] = cnt;
    }
  }
  __syncthreads();

  // ---- 3. the union of the selections, plus the current block ------------------------------
  // Every selection has set its bits in its head's bitmap and in the union bitmap.  The union in
  // block order comes from exclusive prefix counts of the union words: each selected entry finds
  // its place on its own, and the lowest head holding a block writes that block's entry with the
  // mask of every head holding it.  The current block, always kept, follows every history block.
  if (rank == 0) {  // optional outputs: the selection of every head
    for (int e = tid; e < G * K; e += kThreads) {
      const int g = e / K, j = e % K, gs = p.shared ? 0 : g;
      const size_t row = (size_t)bi * Hq + h0 + g;
      if (p.idx) p.idx[row * K + j] = j < s_nsel[gs] ? s_sel[gs][j] : -1;
      if (p.count && j == 0) p.count[row] = s_nsel[gs];
    }
  }
  if (warp == kWarps - 1) {  // a contiguous run of words per lane
    const int per = (nwords + 31) / 32;
    const int w0 = min(nwords, lane * per), w1 = min(nwords, w0 + per);
    int mine = 0;
    for (int w = w0; w < w1; ++w) mine += __popc(s_ubits[w]);
    int incl = mine;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    int run = incl - mine;
    for (int w = w0; w < w1; ++w) {
      s_upre[w] = run;
      run += __popc(s_ubits[w]);
    }
    if (lane == 31) s_U = incl;  // history entries
  }
  __syncthreads();
  for (int e = tid; e < Gs * K; e += kThreads) {
    const int g = e / K, j = e % K;
    if (j < s_nsel[g]) {
      const int x = s_sel[g][j], w = x >> 5;
      const uint32_t bit = 1u << (x & 31);
      unsigned m = 0u;
      for (int h = Gs - 1; h >= 0; --h) m = (m << 1) | ((hbits[h * nwords + w] & bit) ? 1u : 0u);
      if ((m & ((1u << g) - 1u)) == 0u) {  // no lower head holds the block
        const int at = s_upre[w] + __popc(s_ubits[w] & (bit - 1u));
        s_ublk[at] = x;
        s_umask[at] = p.shared ? (1u << G) - 1u : m;
      }
    }
  }
  if (tid == 0) {
    const int uh = s_U;
    s_ublk[uh] = cur;
    s_umask[uh] = (1u << G) - 1u;
    s_U = uh + 1;
  }
  __syncthreads();
  const int U = s_U;

  // ---- 4. attend my share of the union ------------------------------------------------------
  float* wpart = reinterpret_cast<float*>(smem);  // reused after phase 4: [warp][G][D+2]

  if constexpr (kMma) {
    // 16-token slices: history entries have 4, the current block ceil(tok / 16); a global stage
    // holds four consecutive slices (K then V tiles, 64 rows x 128 bytes per 64-column half,
    // 128-byte swizzle).  CTA r first takes global stages r, r + CL, ... into its NKV slots; every
    // later stage is handed out by a counter in rank 0's shared memory when a slot frees, so CTAs
    // whose copies land early take more of the union (HBM serves the CTAs of a cluster unevenly:
    // with static shares the slowest CTA took twice the median).  Local stage i (the i-th stage a
    // CTA takes) is processed by warp group i & 1.
    const int tok_cur = pos - cur * b + 1;
    const int s_hist = 4 * (U - 1);
    const int S_tot = s_hist + (tok_cur + kSlice - 1) / kSlice;
    const int G_st = (S_tot + 3) / 4;
    const int grp = warp >> 2, wg = warp & 3;
    const uint32_t next_addr = dsmem_addr(&s_next, 0);
    const size_t tl = SM::kv_tile(b);
    auto ktile = [&](int st) { return smem + (size_t)st * 2 * tl; };
    auto vtile = [&](int st) { return smem + (size_t)st * 2 * tl + tl; };
    uint64_t* kvbar = bar + NS;
    const int row0 = (bi * p.Hk + kh) * p.n;
    // Group 0 owns slots [0, n0), group 1 slots [n0, NKV) (n0 = ceil(NKV / 2)); a group's k-th
    // local stage uses its slot k % n in phase k / n, and the group refills that slot itself once
    // it has finished the stage.  A group therefore never waits on a phase of a slot that has not
    // been issued yet, however far it runs ahead of the other.
    const int n0 = (NKV + 1) >> 1;
    const int nmine = grp == 0 ? n0 : NKV - n0, sbase = grp == 0 ? 0 : n0;
    // slice -> (block, first token of the slice within the block)
    auto slice_blk = [&](int s) { return s < s_hist ? s_ublk[s >> 2] : cur; };
    auto slice_tok0 = [&](int s) { return s < s_hist ? (s & 3) * kSlice : (s - s_hist) * kSlice; };
    // slot st's next phase (parity par) holds global stage g (g < 0: none left; the phase then
    // completes with no data, and the group that reaches it stops)
    auto issue_kv = [&](int st, uint32_t par, int g) {
      s_gst[st] = g;
      if (g < 0) {
        mbar_arrive(&kvbar[st]);
        return;
      }
      s_kv_par[st] = (int)par;
      const int first = 4 * g;
      const int nsl = min(4, S_tot - first);
      mbar_arrive_expect_tx(&kvbar[st], (uint32_t)(nsl * 2 * kSlice * D * 2));
      const uint64_t pol = l2_evict_first();
      if (first < s_hist) {  // a whole history block (four aligned slices): 64-row boxes
        const int y = row0 + s_ublk[g] * b;
#pragma unroll
        for (int hf = 0; hf < D / 64; ++hf) {
          tc::tma_load_2d_hint(ktile(st) + hf * 8192, &tmk64, hf * 64, y, &kvbar[st], pol);
          tc::tma_load_2d_hint(vtile(st) + hf * 8192, &tmv64, hf * 64, y, &kvbar[st], pol);
        }
        return;
      }
      for (int w = 0; w < nsl; ++w) {
        const int s = first + w;
        const int y = row0 + slice_blk(s) * b + slice_tok0(s);
#pragma unroll
        for (int hf = 0; hf < D / 64; ++hf) {
          tc::tma_load_2d_hint(ktile(st) + hf * 8192 + w * kSlice * 128, &tmk, hf * 64, y,
                               &kvbar[st], pol);
          tc::tma_load_2d_hint(vtile(st) + hf * 8192 + w * kSlice * 128, &tmv, hf * 64, y,
                               &kvbar[st], pol);
        }
      }
    };
    if (lane == 0 && warp < NKV && !s_abort) {  // slot st filled by warp st
      fence_proxy_async();  // generic accesses of phase 1 precede the async writes into region A
      issue_kv(warp, 0u, rank + CL * warp < G_st ? rank + CL * warp : -1);
    }
    if (p.append && rank == CL - 1) {
      // the block being filled: its summary rewritten from its keys in global memory by the last
      // CTA while its first K/V stages are in flight; every row is requested at once (a warp
      // takes rows warp, warp + 8, ...: at most 8 of a 64-token block)
      const T* kb =
          static_cast<const T*>(p.k) + ((size_t)(bi * p.Hk + kh) * p.n + (size_t)cur * b) * D;
      float x[8][EPL];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int t = warp + kWarps * u;
        if (t < tok_cur) {
          load_vec<T, EPL>(kb + (size_t)t * D + lane * EPL, x[u]);
        } else {
#pragma unroll
          for (int e = 0; e < EPL; ++e) x[u][e] = 0.f;
        }
      }
      float cs[EPL];
#pragma unroll
      for (int e = 0; e < EPL; ++e) cs[e] = 0.f;
      float nmax = 0.f;
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        float sq = 0.f;
#pragma unroll
        for (int e = 0; e < EPL; ++e) {
          cs[e] += x[u][e];
          sq = fmaf(x[u][e], x[u][e], sq);
        }
        nmax = fmaxf(nmax, sqrtf(warp_sum(sq)));  // rows past the block add 0
      }
      float* part = reinterpret_cast<float*>(s_scratch);  // [kWarps][D]
#pragma unroll
      for (int e = 0; e < EPL; ++e) part[warp * D + lane * EPL + e] = cs[e];
      if (lane == 0) s_red[warp] = nmax;
      __syncthreads();
      const size_t row = (size_t)(bi * p.Hk + kh) * p.C + cur;
      for (int col = tid; col < D; col += kThreads) {
        float sum = 0.f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) sum += part[w * D + col];
        mean_k[row * D + col] = Elem<TS>::from_f(sum / (float)tok_cur);
      }
      if (tid == 0) {
        float nm = 0.f;
        for (int w = 0; w < kWarps; ++w) nm = fmaxf(nm, s_red[w]);
        if (p.max_norm) p.max_norm[row] = nm;
        if (p.centre)
          p.centre[row] = 0.5f * (float)(cur * b) + 0.5f * (float)(cur * b + tok_cur - 1);
      }
    }
    // B fragments of Q^T (k = d, n = heads, zero beyond G), pre-scaled into log2 units
    const int grow = lane >> 2, tig = lane & 3;
    uint32_t qa0[D / 16], qa1[D / 16];
    {
      const float qs = scale * kLog2e;
      const T* qrow = qsrc + (size_t)min(grow, G - 1) * D;
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
    // online softmax of heads 2 tig and 2 tig + 1 (the accumulator columns this lane holds)
    float m_run[2] = {-INFINITY, -INFINITY}, l_part[2] = {0.f, 0.f};
    // the group leader asks for the global stage of its next refill one stage ahead, so that the
    // remote atomic's round trip overlaps a stage's work
    const bool leader = wg == 0 && lane == 0;
    int g_ahead = -1;
    auto grab = [&]() {
      uint32_t v;
      asm volatile("atom.shared::cluster.add.u32 %0, [%1], 1;" : "=r"(v) : "r"(next_addr) : "memory");
      const int g = CL * NKV + (int)v;
      return g < G_st ? g : -1;
    };
    if (leader && !s_abort) g_ahead = grab();
    for (int k = 0; !s_abort; ++k) {
      const int st = sbase + k % nmine;
      const uint32_t par = (uint32_t)((k / nmine) & 1);
      // group-uniform decision: the OR over the group's four warps of "my wait ran out"
      const int bad = mbar_wait_bounded(&kvbar[st], par) ? 0 : 1;
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
      const int gst = s_gst[st];
      if (gst < 0) break;  // no stage left for this group (uniform over the group)
      const int s = 4 * gst + wg;  // this warp's slice
      if (s < S_tot) {
        const int m = slice_blk(s);
        const unsigned hm = s < s_hist ? s_umask[s >> 2] : (1u << G) - 1u;
        const int tv = m == cur ? min(kSlice, tok_cur - slice_tok0(s)) : kSlice;  // valid tokens
        const unsigned char* kt = ktile(st);
        const unsigned char* vt = vtile(st);
        const int t0 = wg * kSlice;  // this warp's 16 rows of the stage tile
        // S^T = K Q^T (m = the slice's 16 tokens, n = heads): one m16n8k16 per 16-wide d step,
        // its A fragments (K rows) from one ldmatrix.x4 (matrices: tokens 0-7 / 8-15 x d chunks
        // 2 (ks & 3) and 2 (ks & 3) + 1)
        float sfr[4] = {0.f, 0.f, 0.f, 0.f};
        {
          const int mi = lane >> 3, rr = lane & 7;
          const int tokr = t0 + ((mi & 1) << 3) + rr;  // the token row this lane addresses
#pragma unroll
          for (int ks = 0; ks < D / 16; ++ks) {
            const int chunk = (ks & 3) * 2 + (mi >> 1);
            const uint32_t addr =
                smem_u32(kt + (ks >> 2) * 8192 + tokr * 128 + ((chunk ^ (tokr & 7)) << 4));
            uint32_t a0, a1, a2, a3;
            ldsm_x4(addr, a0, a1, a2, a3);
            mma_16816(sfr, a0, a1, a2, a3, qa0[ks], qa1[ks]);
          }
        }
        // masks and the online softmax per head; this lane holds tokens grow and grow + 8 of
        // heads 2 tig + e (sfr[e], sfr[2 + e]); the slice's other tokens of the same heads are in
        // the lanes of the same tig
        float pv[2][2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int h = 2 * tig + e;
          const bool head_on = h < G && ((hm >> h) & 1u);
          if (!head_on || grow >= tv) sfr[e] = -INFINITY;
          if (!head_on || grow + 8 >= tv) sfr[2 + e] = -INFINITY;
          float mx = fmaxf(sfr[e], sfr[2 + e]);
          mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
          mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
          mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
          // lazy rescale: only when the head's max grows by more than 2^8
          float corr = 1.f;
          if (mx > m_run[e] + kRescale || (m_run[e] == -INFINITY && mx != -INFINITY)) {
            corr = m_run[e] == -INFINITY ? 0.f : exp2f(m_run[e] - mx);
            m_run[e] = mx;
            l_part[e] *= corr;
          }
          if (__any_sync(0xffffffffu, corr != 1.f)) {
#pragma unroll
            for (int c = 0; c < D / 16; ++c) {
              oacc[c][e] *= corr;
              oacc[c][2 + e] *= corr;
            }
          }
          pv[0][e] = sfr[e] == -INFINITY ? 0.f : exp2f(sfr[e] - m_run[e]);
          pv[1][e] = sfr[2 + e] == -INFINITY ? 0.f : exp2f(sfr[2 + e] - m_run[e]);
          l_part[e] += pv[0][e] + pv[1][e];
        }
        // P^T as the B operand (k = tokens, n = heads): the 8 x 8 blocks (tokens 0-7 and 8-15 x
        // heads) this lane holds by token rows, transposed in registers
        uint32_t pb0, pb1;
        {
          const uint32_t x0 = pack_bf16(pv[0][0], pv[0][1]), x1 = pack_bf16(pv[1][0], pv[1][1]);
          asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(pb0) : "r"(x0));
          asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(pb1) : "r"(x1));
        }
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
      }
      asm volatile("bar.sync %0, 128;" ::"r"(1 + grp));  // stage free
      if (leader) {
        issue_kv(st, par ^ 1u, g_ahead);
        if (g_ahead >= 0) g_ahead = grab();
      }
    }
    __syncthreads();
    // a group stops at the first slot whose phase holds no stage, after every slot ahead of it in
    // its ring: no copy is left in flight unless a wait ran out (s_abort is uniform here)
    if (s_abort) {
      if (tid == 0) {
        // copies still in flight: the last stage issued into each slot; waiting on its own phase
        // parity returns at once if it already landed
        for (int st = 0; st < NKV; ++st)
          if (s_kv_par[st] >= 0)
            (void)mbar_wait_bounded(&kvbar[st], (uint32_t)s_kv_par[st], 1u << 12);
        report_timeout(p.status, 2);
      }
      __syncthreads();
    }
    // warp partials (heads < G): m, l and o
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      l_part[e] += __shfl_xor_sync(0xffffffffu, l_part[e], 4);
      l_part[e] += __shfl_xor_sync(0xffffffffu, l_part[e], 8);
      l_part[e] += __shfl_xor_sync(0xffffffffu, l_part[e], 16);
      const int h = 2 * tig + e;
      if (grow == 0 && h < G) {
        float* wp = wpart + ((size_t)warp * G + h) * (D + 2);
        wp[D] = m_run[e];
        wp[D + 1] = l_part[e];
      }
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
    // fp32 / other block sizes: scalar FMAs; CTA r takes union entries r, r + CL, ...; warps split
    // each block's tokens, one CTA-wide softmax per block
    const int ne = rank < U ? (U - rank + CL - 1) / CL : 0;
    auto entry_tokens = [&](int m) { return m == cur ? pos - cur * b + 1 : b; };
    const size_t tl = SM::kv_tile(b);
    T* kbuf[2] = {reinterpret_cast<T*>(smem), reinterpret_cast<T*>(smem + 2 * tl)};
    T* vbuf[2] = {reinterpret_cast<T*>(smem + tl), reinterpret_cast<T*>(smem + 3 * tl)};
    uint64_t* kvbar = bar + NS;
    const T* kbase = static_cast<const T*>(p.k) + (size_t)(bi * p.Hk + kh) * p.n * D;
    const T* vbase = static_cast<const T*>(p.v) + (size_t)(bi * p.Hk + kh) * p.n * D;
    auto issue_kv = [&](int i) {
      const int m = s_ublk[rank + i * CL];
      const uint32_t bytes = (uint32_t)(entry_tokens(m) * D * sizeof(T));
      const int st = i & 1;
      mbar_arrive_expect_tx(&kvbar[st], 2 * bytes);
      const uint64_t pol = l2_evict_first();
      bulk_g2s_stream(kbuf[st], kbase + (size_t)m * b * D, bytes, &kvbar[st], pol);
      bulk_g2s_stream(vbuf[st], vbase + (size_t)m * b * D, bytes, &kvbar[st], pol);
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
    int i_stop = ne;
    const int n_run = s_abort ? 0 : ne;  // nothing was issued after an earlier timeout
    for (int i = 0; i < n_run; ++i) {
      const int st = i & 1;
      const int m = s_ublk[rank + i * CL];
      const unsigned hm = s_umask[rank + i * CL];
      const int tok = entry_tokens(m);
      if (!s_abort && !mbar_wait_bounded(&kvbar[st], (i >> 1) & 1)) s_abort = 1;
      __syncthreads();
      if (s_abort) {
        i_stop = i;
        break;
      }
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
    if (s_abort && tid == 0 && n_run > 0) {
      // copies in flight: stages i_stop and i_stop + 1 (if issued), each on its own parity
      for (int j = i_stop; j < min(ne, i_stop + 2); ++j)
        (void)mbar_wait_bounded(&kvbar[j & 1], (j >> 1) & 1, 1u << 12);
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

  // ---- 5. merge the warps, push column slices to their owners, finish -----------------------
  const int cols = D / CL;
  // per head: combined max over warps, each warp's weight, the weighted sum of the l's
  for (int g = warp; g < G; g += kWarps) {
    const float mw = lane < kWarps ? wpart[((size_t)lane * G + g) * (D + 2) + D] : -INFINITY;
    const float M = warp_max(mw);
    const float w = mw == -INFINITY ? 0.f : exp2f(mw - M);
    if (lane < kWarps) s_wt[g][lane] = w;
    float lsum = lane < kWarps ? w * wpart[((size_t)lane * G + g) * (D + 2) + D + 1] : 0.f;
    lsum = warp_sum(lsum);
    if (lane == 0) {
      s_m[g] = M;
      s_l[g] = lsum;
    }
  }
  __syncthreads();
  // four consecutive columns per thread, pushed to their owner with one 16-byte store:
  // recv[rank][g][col % cols]; (m, l) of the head to recv_ml[rank][g]
  static_assert((D / kMaxCL) % 4 == 0, "every owner's column slice holds whole 16-byte pieces");
  float* recv_ml = recv + (size_t)CL * G * cols;
  for (int e = tid; e < G * D / 4; e += kThreads) {
    const int g = e / (D / 4), col = (e % (D / 4)) * 4;
    float o4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      const float sw = s_wt[g][w];
      const float* wp = wpart + ((size_t)w * G + g) * (D + 2) + col;
#pragma unroll
      for (int i = 0; i < 4; ++i) o4[i] = fmaf(sw, wp[i], o4[i]);
    }
    const int owner = col / cols, cc = col % cols;
    st_dsmem_v4(dsmem_addr(recv + ((size_t)rank * G + g) * cols + cc, owner),
                make_uint4(__float_as_uint(o4[0]), __float_as_uint(o4[1]),
                           __float_as_uint(o4[2]), __float_as_uint(o4[3])));
    if (cc == 0) {
      st_dsmem_f32(dsmem_addr(&recv_ml[((size_t)rank * G + g) * 2], owner), s_m[g]);
      st_dsmem_f32(dsmem_addr(&recv_ml[((size_t)rank * G + g) * 2 + 1], owner), s_l[g]);
    }
  }
  cluster_sync();
  // per head: the largest max over the CL partials, each partial's weight and the weighted sum of
  // the l's, once (lanes of CL-wide groups; CL divides 32), so that a column costs CL FMAs
  for (int t0 = 0; t0 < G * CL; t0 += kThreads) {
    const int t = t0 + tid;
    if (t0 + (tid & ~31) < G * CL) {  // warps holding any (head, partial) pair
      const bool in = t < G * CL;
      const int g = in ? t / CL : 0, r = in ? t % CL : 0;
      const float* ml = recv_ml + ((size_t)r * G + g) * 2;
      const float mr = in ? ml[0] : -INFINITY;
      float M = mr;
      for (int o = 1; o < CL; o <<= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
      const float w = mr == -INFINITY ? 0.f : exp2f(mr - M);
      float l = in ? w * ml[1] : 0.f;
      for (int o = 1; o < CL; o <<= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
      if (in) {
        s_fw[g][r] = w;
        if (r == 0) {
          s_fm[g] = M;
          s_fl[g] = l;
        }
      }
    }
  }
  __syncthreads();
  // each thread finishes V consecutive columns of one head and writes them with one 8- or 16-byte
  // store when o lives in page-locked host memory (cols = D / CL is a power of two >= 4), one
  // column per thread otherwise
  const int V = kHostIO ? (cols >= 8 ? 8 : 4) : 1, per_g = cols / V;
  for (int e = tid; e < G * per_g; e += kThreads) {
    const int g = e / per_g, cc = (e % per_g) * V, col = rank * cols + cc;
    const float M = s_fm[g], lsum = s_fl[g];
    float osum[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int r = 0; r < CL; ++r) {
      const float* slot = recv + ((size_t)r * G + g) * cols;
      const float w = s_fw[g][r];
#pragma unroll
      for (int v = 0; v < 8; ++v)
        if (v < V) osum[v] = fmaf(w, slot[cc + v], osum[v]);
    }
    const size_t row = (size_t)bi * Hq + h0 + g;
    const float inv = 1.f / lsum;
    T* dst = static_cast<T*>(p.o) + row * D + col;
    if (V == 1) {
      *dst = Elem<T>::from_f(osum[0] / lsum);
    } else if constexpr (sizeof(T) == 2) {
      const uint32_t w0 = pack_bf16(osum[0] * inv, osum[1] * inv);
      const uint32_t w1 = pack_bf16(osum[2] * inv, osum[3] * inv);
      if (V == 8)
        *reinterpret_cast<uint4*>(dst) = make_uint4(w0, w1, pack_bf16(osum[4] * inv, osum[5] * inv),
                                                    pack_bf16(osum[6] * inv, osum[7] * inv));
      else
        *reinterpret_cast<uint2*>(dst) = make_uint2(w0, w1);
    } else {
      *reinterpret_cast<float4*>(dst) =
          make_float4(osum[0] * inv, osum[1] * inv, osum[2] * inv, osum[3] * inv);
      if (V == 8)
        *reinterpret_cast<float4*>(dst + 4) =
            make_float4(osum[4] * inv, osum[5] * inv, osum[6] * inv, osum[7] * inv);
    }
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

// K or V as [rows, D] bf16 with 64-column x box_rows boxes (16: one slice; 64: a whole block),
// 128-byte swizzle
bool kv_map(CUtensorMap* m, const void* base, long long rows, int D, int box_rows = kSlice) {
  auto enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)D * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
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
  std::map<const void*, size_t> static_smem;                           // -> static shared bytes
};
LaunchCache& launch_cache() {
  static LaunchCache c;
  return c;
}

// Shared memory one SM gives its resident CTAs (228 KB less 1 KB reserved per CTA) and the static
// shared memory of the fused kernel (G <= 8), both with margin.
constexpr size_t kSmemPerSM = 227 * 1024;
constexpr size_t kStaticSmemBound = 12 * 1024;

template <typename T, typename TS, int D, int G, bool MMA>
bsa_status launch_fused(FusedParams& p, cudaStream_t st) {
  using SM = FusedSmem<T, TS, D, G, MMA>;
  CUtensorMap tmk{}, tmv{}, tmk64{}, tmv64{};
  if (MMA) {
    const long long rows = (long long)p.B * p.Hk * p.n;
    if (!kv_map(&tmk, p.k, rows, D) || !kv_map(&tmv, p.v, rows, D) ||
        !kv_map(&tmk64, p.k, rows, D, 64) || !kv_map(&tmv64, p.v, rows, D, 64))
      return BSA_ERR_CUDA;
  }
  const int groups = p.B * p.Hk;
  int CL = pick_cluster(groups);
  auto kern = decode_fused_kernel<T, TS, D, G, MMA, 0>;
  if constexpr (MMA) {
    if (p.mode == 2) kern = decode_fused_kernel<T, TS, D, G, MMA, 2>;
    if (p.mode == 3) kern = decode_fused_kernel<T, TS, D, G, MMA, 3>;
    if (p.host_io && p.mode == 0) kern = decode_fused_kernel<T, TS, D, G, MMA, 0, true>;
    if (p.host_io && p.mode == 2) kern = decode_fused_kernel<T, TS, D, G, MMA, 2, true>;
  }
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    (void)cudaGetLastError();
    return BSA_ERR_CUDA;
  }
  int min_per_sm = 1;
  const int Gs = p.shared ? 1 : G;
  for (;;) {
    const int chunk = std::max(kSub, ceil_div(ceil_div(std::max(p.C, 1), CL), kSub) * kSub);
    if (chunk > kSelMax && p.mode == 0) {  // the local select holds at most kSelMax keys per head
      if (CL < kMaxCL) { CL <<= 1; continue; }
      return BSA_ERR_UNSUPPORTED;
    }
    p.chunk = chunk;
    // whole-row selection when every history fits one warp select
    p.gather = p.C <= kSelMax && p.mode == 0 ? 1 : 0;
    p.row_ld = (int)align_up((size_t)std::max(p.C, 1), 4);
    // Region A as large as the CTAs resident per SM allow, then the fixed pieces.  Region A holds
    // the summary ring with the keys and the whole-row / merge buffer above it (phases 1-2), then
    // the K/V ring over all of it (phase 4, once the keys are dead), then the warp partials.
    size_t off = 0;
    const size_t fixed = SM::hbits(p.C) + SM::recv(CL) + SM::zp(p.b) + 256;
    size_t tail =
        align_up(SM::keys(chunk) + SM::sel(p.gather, p.row_ld, CL, p.K), (size_t)1024);
    const size_t kvs = SM::kv_stage(p.b), sus = SM::sum_stage();
    // mode 2: region A starts with the group's chunk lists; no summary ring
    const size_t cand_bytes = align_up((size_t)p.nchunk * Gs * p.cand_ld * 4, (size_t)1024);
    const size_t head2 = cand_bytes;
    if (p.mode >= 2) tail = 0;
    const size_t need_min = p.mode >= 2 ? max_sz(max_sz(2 * kvs, head2), SM::partials())
                                        : max_sz(max_sz(2 * kvs, 2 * sus + tail), SM::partials());
    // two CTAs per SM when the grid needs them to be resident at once, unless region A's minimum
    // (two K/V stages) does not fit that way
    int per_sm = std::max(min_per_sm, groups * CL > kSMs ? 2 : 1);
    size_t ra = 0;
    for (;; per_sm = 1) {
      const size_t budget = kSmemPerSM / per_sm - kStaticSmemBound - 1024 /* alignment slack */;
      ra = budget > fixed ? (budget - fixed) / 1024 * 1024 : 0;
      if (ra >= need_min || per_sm == 1) break;
    }
    if (ra < need_min) return BSA_ERR_UNSUPPORTED;
    ra = std::min(ra, max_sz(max_sz((size_t)kMaxStages * kvs, (size_t)kMaxStages * sus + tail),
                             max_sz(SM::partials(), p.mode == 2 ? head2 : 0)));
    p.ns = p.mode >= 2 ? 1 : (int)std::min<size_t>(kMaxStages, (ra - tail) / sus);
    p.nkv = MMA ? (int)std::min<size_t>(kMaxStages, ra / kvs) : 2;
    p.off_keys = p.mode >= 2 ? 0 : (int)(ra - tail);
    p.off_sel = p.mode >= 2 ? (int)cand_bytes : p.off_keys + (int)SM::keys(chunk);
    off = align_up(ra, 1024);
    p.off_hbits = (int)off;
    off += SM::hbits(p.C);
    p.off_recv = (int)off;
    off += SM::recv(CL);
    p.off_zp = (int)off;
    off += SM::zp(p.b);
    off = align_up(off, 16);
    p.off_bar = (int)off;
    off += 256;
    const size_t smem = off + 1024;  // + alignment slack of the dynamic base
    if (smem > 227 * 1024) return BSA_ERR_UNSUPPORTED;
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
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = CL;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    // the kernel may be scheduled while the previous launch on the stream drains (it waits for
    // that launch's completion before reading anything)
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
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
    if (nclusters < groups && per_sm == 1 && min_per_sm == 1) {
      // not every cluster is resident at one CTA per SM (large clusters are placed one per GPC):
      // two CTAs per SM with smaller rings keep the whole grid in one wave
      min_per_sm = 2;
      continue;
    }
    if (cudaLaunchKernelEx(&cfg, kern, tmk, tmv, tmk64, tmv64, p) != cudaSuccess) {
      (void)cudaGetLastError();
      return BSA_ERR_CUDA;
    }
    return BSA_OK;
  }
}

// The two-launch plan of a long history (more than kSelMax blocks) on the 64-token bf16 path:
// about two CTAs per SM over the groups (each chunk at most kSelMax blocks), and the group's chunk
// lists small enough for the merge launch's shared memory.  nchunk = 0: the plan does not apply.
struct SplitPlan {
  int nchunk = 0, chunk = 0, cand_ld = 0;
  size_t bytes = 0;  // workspace
};
SplitPlan split_plan(int B, int Hk, int G, int C, int K, bool shared, bool mma) {
  SplitPlan s;
  if (!mma || C <= kSelMax) return s;
  const int groups = B * Hk, Gs = shared ? 1 : G;
  int nchunk = std::max(ceil_div(C, kSelMax), std::min(32, ceil_div(2 * kSMs, groups)));
  const int chunk = std::max(kSub, ceil_div(ceil_div(C, nchunk), kSub) * kSub);
  nchunk = ceil_div(C, chunk);
  const int cand_ld = (int)align_up((size_t)(2 * K + 2), (size_t)4);
  if (nchunk > 32 || (size_t)nchunk * Gs * cand_ld * 4 > 64 * 1024) return s;
  s.nchunk = nchunk;
  s.chunk = chunk;
  s.cand_ld = cand_ld;
  s.bytes = (size_t)groups * nchunk * Gs * cand_ld * 4;
  return s;
}

size_t static_smem_bytes(const void* kern) {
  LaunchCache& lc = launch_cache();
  std::lock_guard<std::mutex> lock(lc.mu);
  auto it = lc.static_smem.find(kern);
  if (it != lc.static_smem.end()) return it->second;
  cudaFuncAttributes fa{};
  size_t v = kStaticSmemBound;
  if (cudaFuncGetAttributes(&fa, kern) == cudaSuccess)
    v = fa.sharedSizeBytes;
  else
    (void)cudaGetLastError();
  lc.static_smem[kern] = v;
  return v;
}

// Launch 1 of the long-history plan (mode 1): CTA (c, kh, b) scores chunk c of group (b, kh) and
// writes every selecting head's chunk Top-K to the workspace; no cluster, two CTAs per SM with a
// summary ring as deep as that leaves room for.  Launch 2 is launch_fused in mode 2.
template <typename T, typename TS, int D, int G, bool MMA>
bsa_status launch_chunk_topk(const FusedParams& p, cudaStream_t st) {
  using SM = FusedSmem<T, TS, D, G, MMA>;
  auto kern = decode_fused_kernel<T, TS, D, G, MMA, 1>;
  FusedParams p1 = p;
  p1.mode = 1;
  p1.gather = 0;
  p1.row_ld = 4;
  const size_t sus = SM::sum_stage();
  const size_t keys = align_up(SM::keys(p.chunk), (size_t)1024);
  // two CTAs per SM: 228 KB less 1 KB reserved per CTA, the static part, alignment slack
  const size_t budget = 228 * 1024 / 2 - 1024 - static_smem_bytes(reinterpret_cast<const void*>(kern)) - 1024;
  const size_t small = SM::recv(1) + SM::zp(p.b) + 256 + 64;
  if (budget < keys + small + sus) return BSA_ERR_UNSUPPORTED;
  const int need_st = ceil_div(p.chunk, kSub);
  p1.ns = (int)std::min<size_t>(std::min(kMaxStages, need_st), (budget - keys - small) / sus);
  p1.nkv = 1;
  size_t off = (size_t)p1.ns * sus;
  p1.off_keys = (int)off;
  p1.off_sel = (int)off;
  off += keys;
  p1.off_hbits = (int)off;  // no bitmaps in mode 1
  p1.off_recv = (int)off;
  off += SM::recv(1);
  p1.off_zp = (int)off;
  off += SM::zp(p.b);
  off = align_up(off, 16);
  p1.off_bar = (int)off;
  off += 256;
  const size_t smem = off + 1024;
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
      set_to = smem;
    }
  }
  CUtensorMap tm{};  // mode 1 copies no K/V: the maps are never used
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.nchunk, p.Hk, p.B);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kern, tm, tm, tm, tm, p1) != cudaSuccess) {
    (void)cudaGetLastError();
    return BSA_ERR_CUDA;
  }
  return BSA_OK;
}

template <typename T, typename TS, int D, int G, bool MMA>
bsa_status launch_step(FusedParams& p, const SplitPlan& plan, uint32_t* ws, cudaStream_t st) {
  if constexpr (MMA) {
    if (plan.nchunk > 0 && ws) {
      p.nchunk = plan.nchunk;
      p.chunk = plan.chunk;
      p.cand_ld = plan.cand_ld;
      p.cand = ws;
      const bsa_status rc = launch_chunk_topk<T, TS, D, G, MMA>(p, st);
      if (rc != BSA_OK) return rc;
      p.mode = 2;
    }
  }
  return launch_fused<T, TS, D, G, MMA>(p, st);
}

template <typename T, typename TS, int D, bool MMA>
bsa_status dispatch_fused(int G, FusedParams& p, cudaStream_t st, uint32_t* ws = nullptr,
                          size_t ws_bytes = 0) {
  SplitPlan plan = split_plan(p.B, p.Hk, G, p.C, p.K, p.shared != 0, MMA);
  if (plan.nchunk > 0 && ws && ws_bytes < plan.bytes) return BSA_ERR_WORKSPACE;
  if (!ws) plan = SplitPlan{};
  switch (G) {
    case 1: return launch_step<T, TS, D, 1, MMA>(p, plan, ws, st);
    case 2: return launch_step<T, TS, D, 2, MMA>(p, plan, ws, st);
    case 4: return launch_step<T, TS, D, 4, MMA>(p, plan, ws, st);
    case 8: return launch_step<T, TS, D, 8, MMA>(p, plan, ws, st);
    default: return BSA_ERR_UNSUPPORTED;
  }
}

}  // namespace
}  // namespace bsa

namespace bsa {
namespace {

// q of a host-I/O step into the workspace: the host reads are issued at once (the launch may be
// scheduled while the previous step still runs), the stores into the staging buffer only after
// the work queued before it -- the previous step, which reads that buffer -- has completed.
__global__ void __launch_bounds__(128) stage_q_kernel(const uint4* __restrict__ src,
                                                      uint4* __restrict__ dst, int n16) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  uint4 x = make_uint4(0u, 0u, 0u, 0u);
  if (i < n16) x = src[i];
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  if (i < n16) dst[i] = x;
}

constexpr int kHostIo = 4;  // BSA_DECODE_HOST_IO

size_t q_stage_offset(size_t plan_bytes) { return align_up(plan_bytes, (size_t)256); }

bsa_status decode_step_impl(const void* q, const void* k, const void* v, bsa_dtype dt, int B,
                            int Hq, int Hk, int n, int d, int b, const int* seq_lens,
                            void* mean_k, float* max_norm, float* centre, int append,
                            const float* lambda_h, const float* sigma_h, int prefix_block, int K,
                            void* o, float* lse, int* idx, int* count, int* status, int flags,
                            void* workspace, size_t workspace_bytes, bool allow_host_io,
                            void* stream) {
  BSA_REQUIRE(dtype_ok(dt), BSA_ERR_DTYPE);
  BSA_REQUIRE(q && k && v && mean_k && o, BSA_ERR_ARG);
  BSA_REQUIRE(B > 0 && Hq > 0 && Hk > 0 && n > 0 && d > 0 && b > 0 && K > 0 && prefix_block >= 0,
              BSA_ERR_ARG);
  const int known = BSA_DECODE_SHARED_SELECTION | BSA_DECODE_BF16_SUMMARIES |
                    (allow_host_io ? kHostIo : 0);
  BSA_REQUIRE((flags & ~known) == 0, BSA_ERR_ARG);
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
  BSA_REQUIRE(!workspace || aligned16(workspace), BSA_ERR_ARG);
  uint32_t* ws = workspace_bytes > 0 ? static_cast<uint32_t*>(workspace) : nullptr;
  if (flags & kHostIo) {
    // q and o in page-locked host memory: o written by the step straight to its device mapping;
    // q read through its device mapping by rank 0 of each cluster, once per group, on the
    // one-launch bf16 path, and otherwise staged into the workspace (after the chunk lists) by a
    // copy kernel first
    const bool mma = dt == BSA_BF16 && b == 64;
    const SplitPlan sp = split_plan(B, Hk, Hq / Hk, C, K, p.shared != 0, mma);
    const size_t qoff = q_stage_offset(sp.bytes);
    const size_t qbytes = (size_t)B * Hq * d * (dt == BSA_BF16 ? 2 : 4);
    BSA_REQUIRE(ws && workspace_bytes >= qoff + qbytes, BSA_ERR_WORKSPACE);
    void* qd = nullptr;
    void* od = nullptr;
    if (cudaHostGetDevicePointer(&qd, const_cast<void*>(q), 0) != cudaSuccess ||
        cudaHostGetDevicePointer(&od, o, 0) != cudaSuccess || !aligned16(qd) || !aligned16(od)) {
      (void)cudaGetLastError();
      return BSA_ERR_ARG;
    }
    p.o = od;
    p.q = qd;
    p.host_io = 1;
    if (!(mma && sp.nchunk == 0)) {
      unsigned char* stage = reinterpret_cast<unsigned char*>(ws) + qoff;
      const int n16 = (int)(qbytes / 16);
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3((unsigned)ceil_div(n16, 128), 1, 1);
      cfg.blockDim = dim3(128, 1, 1);
      cfg.stream = st;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
      attr[0].val.programmaticStreamSerializationAllowed = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      if (cudaLaunchKernelEx(&cfg, stage_q_kernel, static_cast<const uint4*>(qd),
                             reinterpret_cast<uint4*>(stage), n16) != cudaSuccess) {
        (void)cudaGetLastError();
        return BSA_ERR_CUDA;
      }
      p.q = stage;
    }
  }
  bsa_status rc;
  if (dt == BSA_BF16 && b == 64 && bf16_sum)
    rc = d == 64 ? dispatch_fused<bf, bf, 64, true>(Hq / Hk, p, st, ws, workspace_bytes)
                 : dispatch_fused<bf, bf, 128, true>(Hq / Hk, p, st, ws, workspace_bytes);
  else if (dt == BSA_BF16 && b == 64)  // 64-token blocks: warp MMAs over swizzled TMA tiles
    rc = d == 64 ? dispatch_fused<bf, float, 64, true>(Hq / Hk, p, st, ws, workspace_bytes)
                 : dispatch_fused<bf, float, 128, true>(Hq / Hk, p, st, ws, workspace_bytes);
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

}  // namespace

// Decode attention of a given selection on the cluster step (mode 3): bf16 K/V in 64-token blocks,
// no gate.  BSA_ERR_UNSUPPORTED for every other request (the caller then takes the split-K kernel).
bsa_status decode_attn_given(const void* q, const void* k, const void* v, bsa_dtype dt, int B,
                             int Hq, int Hk, int n, int d, int b, const int* seq_lens,
                             const int* idx, const int* count, int K, int gate, void* o,
                             float* lse, int* status, cudaStream_t st) {
  if (dt != BSA_BF16 || b != 64 || gate != BSA_GATE_NONE || (d != 64 && d != 128) ||
      K > kMaxKf || Hq % Hk != 0 || !group_ok(Hq, Hk) || B > 65535 || Hk > 65535)
    return BSA_ERR_UNSUPPORTED;
  const int C = ceil_div(n, b);
  if (C > kMaxWords * 32) return BSA_ERR_UNSUPPORTED;
  FusedParams p{};
  p.q = q; p.k = k; p.v = v;
  p.B = B; p.Hq = Hq; p.Hk = Hk; p.n = n; p.b = b; p.C = C; p.K = K;
  p.seq_lens = seq_lens;
  p.o = o; p.lse = lse; p.status = status;
  p.sel_idx = idx; p.sel_count = count;
  p.mode = 3;
  using bf = __nv_bfloat16;
  const int G = Hq / Hk;
  bsa_status rc;
  switch (G) {
    case 1: rc = d == 64 ? launch_fused<bf, float, 64, 1, true>(p, st) : launch_fused<bf, float, 128, 1, true>(p, st); break;
    case 2: rc = d == 64 ? launch_fused<bf, float, 64, 2, true>(p, st) : launch_fused<bf, float, 128, 2, true>(p, st); break;
    case 4: rc = d == 64 ? launch_fused<bf, float, 64, 4, true>(p, st) : launch_fused<bf, float, 128, 4, true>(p, st); break;
    case 8: rc = d == 64 ? launch_fused<bf, float, 64, 8, true>(p, st) : launch_fused<bf, float, 128, 8, true>(p, st); break;
    default: rc = BSA_ERR_UNSUPPORTED;
  }
  return rc;
}

}  // namespace bsa

extern "C" bsa_status bsa_decode_step_ex(const void* q, const void* k, const void* v,
                                         bsa_dtype dt, int B, int Hq, int Hk, int n, int d, int b,
                                         const int* seq_lens, void* mean_k, float* max_norm,
                                         float* centre, int append, const float* lambda_h,
                                         const float* sigma_h, int prefix_block, int K, void* o,
                                         float* lse, int* idx, int* count, int* status,
                                         int flags, void* stream) {
  return bsa::decode_step_impl(q, k, v, dt, B, Hq, Hk, n, d, b, seq_lens, mean_k, max_norm,
                               centre, append, lambda_h, sigma_h, prefix_block, K, o, lse, idx,
                               count, status, flags, nullptr, 0, false, stream);
}

extern "C" size_t bsa_decode_step_workspace_bytes(int B, int Hq, int Hk, int n, int d, int b,
                                                  int K, int flags, int dt) {
  using namespace bsa;
  if (B <= 0 || Hq <= 0 || Hk <= 0 || n <= 0 || d <= 0 || b <= 0 || K <= 0 || Hq % Hk != 0)
    return 0;
  const bool mma = dt == BSA_BF16 && b == 64 && (d == 64 || d == 128);
  const size_t plan = split_plan(B, Hk, Hq / Hk, ceil_div(n, b), K,
                                 (flags & BSA_DECODE_SHARED_SELECTION) != 0, mma).bytes;
  if (!(flags & kHostIo)) return plan;
  return q_stage_offset(plan) + (size_t)B * Hq * d * (dt == BSA_BF16 ? 2 : 4);
}

extern "C" bsa_status bsa_decode_step_ws(const void* q, const void* k, const void* v,
                                         bsa_dtype dt, int B, int Hq, int Hk, int n, int d, int b,
                                         const int* seq_lens, void* mean_k, float* max_norm,
                                         float* centre, int append, const float* lambda_h,
                                         const float* sigma_h, int prefix_block, int K, void* o,
                                         float* lse, int* idx, int* count, int* status,
                                         int flags, void* workspace, size_t workspace_bytes,
                                         void* stream) {
  return bsa::decode_step_impl(q, k, v, dt, B, Hq, Hk, n, d, b, seq_lens, mean_k, max_norm,
                               centre, append, lambda_h, sigma_h, prefix_block, K, o, lse, idx,
                               count, status, flags, workspace, workspace_bytes, true, stream);
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
