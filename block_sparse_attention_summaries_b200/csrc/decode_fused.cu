// Fused decode step: block scoring -> Top-K -> GQA union -> sparse attention -> merge, in one
// launch, one thread-block cluster per (batch, kv head).
//
// [SAS] review, "How it works" step 6 and "Decoding efficiency" (Fig. 7): at inference every
// decode step scores the summaries of all history blocks, keeps the Top-K plus the current block
// and attends their tokens; scoring and Top-K grow with the context and dominate long-context
// steps.  [FreeSolo] summary page, "How it works": optional erf distance bias of the cell score.
//
// B200 design.  The step is HBM-bound (summaries + selected K/V) and short (~10 us), so launch
// boundaries and global round trips cost as much as the data.  The CL CTAs of a cluster (CL <= 16)
// cooperate through distributed shared memory (DSMEM) instead of global scratch:
//   1. CTA r scores its slice of the history blocks: the mean-key rows stream through a
//      shared-memory ring filled by bulk copies (TMA engine); the G query heads of the group
//      share every row (one 31-shuffle transpose-reduce per 32/G rows); a per-head warp radix
//      select keeps the slice's local Top-K.
//   2. cluster barrier; every CTA reads all CL local lists over DSMEM and selects the global Top-K
//      per head (the same exact order everywhere: larger score, then lower index), then the
//      sorted union of the G heads' selections plus the current block.
//   3. CTA r attends union entries r, r+CL, ...: each K/V block is one contiguous bulk copy,
//      double-buffered; logits for all G heads, per-head masks for blocks a head did not select;
//      the CTA holding the current block also rewrites that block's summary from shared memory.
//   4. cluster barrier; CTA r merges the CL partial (m, l, o) for its slice of the output columns
//      over DSMEM and writes o (and lse).
// Every CTA reaches every cluster barrier (no early exit); every mbarrier wait is bounded.
#include "bsa_common.cuh"

namespace bsa {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kMaxCL = 16;
constexpr int kMaxKf = 32;        // Top-K bound of the fused path
constexpr int kMaxUnion = 8 * kMaxKf + 1;
constexpr int kSub = 64;          // summary rows per ring stage
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

struct FusedParams {
  const void* q;
  const void* k;
  const void* v;
  int B, Hq, Hk, n, b, C, K;
  const int* seq_lens;
  float* mean_k;
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
  int ns;     // ring stages
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
// Address of `p` (this CTA's shared memory) in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t dsmem_addr(const void* p, uint32_t rank) {
  uint32_t out;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(out) : "r"(smem_u32(p)), "r"(rank));
  return out;
}
__device__ __forceinline__ uint32_t ld_dsmem_u32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
  return v;
}
__device__ __forceinline__ float ld_dsmem_f32(uint32_t addr) {
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
  return v;
}

__device__ __forceinline__ uint32_t order_key(float f) {
  if (f != f) return 0u;
  if (f == 0.f) f = 0.f;
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Top-K of N keys held in shared memory, by one warp: exact radix select of the K-th largest key
// (8-bit digits, the warp's own 256-bin histogram), then one ordered pass that takes every key
// above it and the lowest-indexed keys equal to it.  Writes the positions of the selected keys in
// ascending order to `out` and returns their number min(K, N).
__device__ int warp_topk(const uint32_t* keys, int N, int K, uint32_t* hist, int lane, int* out) {
  const int kk = min(K, N);
  if (kk <= 0) return 0;
  if (kk == N) {
    for (int i = lane; i < N; i += 32) out[i] = i;
    __syncwarp();
    return N;
  }
  uint32_t prefix = 0, mask = 0;
  int rem = kk;
  for (int shift = 24; shift >= 0; shift -= 8) {
#pragma unroll
    for (int j = 0; j < 8; ++j) hist[lane * 8 + j] = 0;
    __syncwarp();
    for (int i = lane; i < N; i += 32) {
      const uint32_t x = keys[i];
      if ((x & mask) == prefix) atomicAdd(&hist[(x >> shift) & 255u], 1u);
    }
    __syncwarp();
    uint32_t hb[8], local = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      hb[j] = hist[lane * 8 + j];
      local += hb[j];
    }
    uint32_t incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_down_sync(0xffffffffu, incl, o);
      if (lane + o < 32) incl += y;
    }
    uint32_t running = incl - local;
    int digit = -1, above = 0;
#pragma unroll
    for (int j = 7; j >= 0; --j) {
      if (running < (uint32_t)rem && running + hb[j] >= (uint32_t)rem) {
        digit = lane * 8 + j;
        above = (int)running;
      }
      running += hb[j];
    }
    const unsigned who = __ballot_sync(0xffffffffu, digit >= 0);
    const int src = __ffs(who) - 1;
    digit = __shfl_sync(0xffffffffu, digit, src);
    above = __shfl_sync(0xffffffffu, above, src);
    prefix |= (uint32_t)digit << shift;
    mask |= 255u << shift;
    rem -= above;
    __syncwarp();
  }
  const uint32_t T = prefix;
  int taken = 0, eq_seen = 0;
  const unsigned lt = (1u << lane) - 1u;
  for (int base = 0; base < N; base += 32) {
    const int i = base + lane;
    const uint32_t x = i < N ? keys[i] : 0u;
    const bool valid = i < N;
    const bool gt = valid && x > T;
    const bool eq = valid && x == T;
    const unsigned eqb = __ballot_sync(0xffffffffu, eq);
    const bool take = gt || (eq && eq_seen + __popc(eqb & lt) < rem);
    const unsigned tb = __ballot_sync(0xffffffffu, take);
    if (take) out[taken + __popc(tb & lt)] = i;
    taken += __popc(tb);
    eq_seen += __popc(eqb);
  }
  __syncwarp();
  return taken;
}

template <typename T, int D, int G>
struct FusedSmem {
  // region A: summary ring (ns x kSub x D floats) / K,V stages (2 x 2 x b x D x T) / partials
  __host__ __device__ static size_t tile(int b) { return align_up((size_t)b * D * sizeof(T), 128); }
  __host__ __device__ static size_t region_a(int b, int ns) {
    size_t x = (size_t)ns * kSub * D * sizeof(float);
    x = max_sz(x, 4 * tile(b));
    x = max_sz(x, (size_t)G * kMaxCL * kMaxKf * 8);                  // merge buffers
    x = max_sz(x, (size_t)(kThreads / (D / 2) + 1) * G * D * 4);     // split reduction, partials
    return align_up(x, 1024);
  }
  __host__ __device__ static size_t scores(int chunk) { return align_up((size_t)G * chunk * 4, 16); }
  __host__ __device__ static size_t bytes(int b, int ns, int chunk) {
    return region_a(b, ns) + scores(chunk) + 2 * align_up((size_t)b * G * 4, 16) + 1024;
  }
};

template <typename T, int D, int G>
__global__ void __launch_bounds__(kThreads) decode_fused_kernel(const FusedParams p) {
  constexpr int EPL = D / 32;
  constexpr int R = 32 / G;
  constexpr int CG = D / 2;
  constexpr int TP = kThreads / CG;

  extern __shared__ __align__(1024) unsigned char smem[];
  // static shared state
  __shared__ uint32_t s_hist[kWarps][256];
  __shared__ uint32_t s_ckey[G][kMaxKf];   // local Top-K keys (read by the cluster)
  __shared__ int s_cidx[G][kMaxKf];        // and their global block indices
  __shared__ int s_ccnt[G];
  __shared__ int s_pick[G][kMaxKf];
  __shared__ int s_sel[G][kMaxKf];
  __shared__ int s_nsel[G];
  __shared__ int s_list[kMaxUnion];
  __shared__ unsigned char s_first[kMaxUnion];
  __shared__ int s_ublk[kMaxUnion];
  __shared__ unsigned s_umask[kMaxUnion];
  __shared__ int s_U;
  __shared__ float s_m[G], s_l[G], s_corr[G];
  __shared__ int s_abort;
  __shared__ float s_red[kWarps];

  const int b = p.b, K = p.K, Hq = p.Hq, D2 = D;
  (void)D2;
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

  const size_t ra = FusedSmem<T, D, G>::region_a(b, p.ns);
  float* ring = reinterpret_cast<float*>(smem);
  float* s_sc = reinterpret_cast<float*>(smem + ra);  // [G][chunk]
  float* zs = reinterpret_cast<float*>(smem + ra + FusedSmem<T, D, G>::scores(p.chunk));
  float* ps = zs + align_up((size_t)b * G, 4);
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + FusedSmem<T, D, G>::bytes(b, p.ns, p.chunk) -
                                              1024);
  // bar[0 .. ns): summary ring; bar[ns], bar[ns+1]: K/V stages

  if (tid == 0) {
    for (int i = 0; i < p.ns + 2; ++i) mbar_init(&bar[i], 1);
    fence_mbar_init();
    s_abort = 0;
    s_U = 0;
  }
  if (tid < G) {
    s_m[tid] = -INFINITY;
    s_l[tid] = 0.f;
  }
  __syncthreads();

  // query slices (pre-scaled by 1/sqrt(d) for scoring)
  float qv[G][EPL];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    float tmp[EPL];
    load_vec<T, EPL>(static_cast<const T*>(p.q) + ((size_t)bi * Hq + h0 + g) * D + lane * EPL,
                     tmp);
#pragma unroll
    for (int e = 0; e < EPL; ++e) qv[g][e] = tmp[e];
  }

  // ---- 1. score my slice of the history blocks --------------------------------------------
  const int c_lo = min(nc, rank * p.chunk);
  const int c_hi = min(nc, c_lo + p.chunk);
  const int rows = c_hi - c_lo;
  const int nsub = (rows + kSub - 1) / kSub;
  const float* mk = p.mean_k + ((size_t)(bi * p.Hk + kh) * p.C) * D;
  auto issue_sub = [&](int j) {
    const int r0 = c_lo + j * kSub;
    const int nr = min(kSub, c_hi - r0);
    const int st = j % p.ns;
    const uint32_t bytes = (uint32_t)(nr * D * sizeof(float));
    mbar_arrive_expect_tx(&bar[st], bytes);
    bulk_g2s(ring + (size_t)st * kSub * D, mk + (size_t)r0 * D, bytes, &bar[st]);
  };
  if (tid == 0)
    for (int j = 0; j < min(nsub, p.ns); ++j) issue_sub(j);
  const float scale = rsqrtf((float)D);
  const int my_r = lane / G, my_g = lane % G;
  const float lam_h = p.lam ? p.lam[h0 + my_g] : 0.f;
  const float inv2sig = p.lam ? 0.5f / p.sig[h0 + my_g] : 0.f;
  for (int j = 0; j < nsub; ++j) {
    const int st = j % p.ns;
    if (!s_abort && !mbar_wait_bounded(&bar[st], (j / p.ns) & 1)) s_abort = 1;
    __syncthreads();
    if (!s_abort) {
      const int r0 = j * kSub;
      const int nr = min(kSub, rows - r0);
      const float* base = ring + (size_t)st * kSub * D;
      for (int t0 = warp * R; t0 < nr; t0 += kWarps * R) {
        float a[32];
#pragma unroll
        for (int r = 0; r < R; ++r) {
          float x[EPL];
          if (t0 + r < nr) {
            load_vec<float, EPL>(base + (size_t)(t0 + r) * D + lane * EPL, x);
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
        if (t < nr) {
          float s = a[0] * scale;
          if (p.lam) {
            const size_t row = (size_t)(bi * p.Hk + kh) * p.C + c_lo + r0 + t;
            s += lam_h * p.max_norm[row] * erff(((float)pos - p.centre[row]) * inv2sig);
          }
          reinterpret_cast<uint32_t*>(s_sc)[my_g * p.chunk + r0 + t] = order_key(s);
        }
      }
    }
    __syncthreads();
    if (tid == 0 && j + p.ns < nsub && !s_abort) issue_sub(j + p.ns);
  }
  // local Top-K per head (warp g)
  for (int g = warp; g < G; g += kWarps) {
    const uint32_t* keys = reinterpret_cast<const uint32_t*>(s_sc) + g * p.chunk;
    const int cnt = warp_topk(keys, rows, K, s_hist[warp], lane, s_pick[g]);
    for (int j = lane; j < cnt; j += 32) {
      const int i = s_pick[g][j];
      s_ckey[g][j] = keys[i];
      s_cidx[g][j] = c_lo + i;
    }
    if (lane == 0) s_ccnt[g] = cnt;
  }
  cluster_sync();

  // ---- 2. global Top-K per head over all CTAs' lists, then the union ----------------------
  // merge buffers [G][CL*K] keys and block indices, in region A (the ring is idle now)
  uint32_t* mkey_all = reinterpret_cast<uint32_t*>(smem);
  int* midx_all = reinterpret_cast<int*>(smem) + G * kMaxCL * kMaxKf;
  for (int g = warp; g < G; g += kWarps) {
    uint32_t* s_mkey_g = mkey_all + g * kMaxCL * kMaxKf;
    int* s_midx_g = midx_all + g * kMaxCL * kMaxKf;
    int tot = 0;
    for (int r = 0; r < CL; ++r) {
      const int cnt = (int)ld_dsmem_u32(dsmem_addr(&s_ccnt[g], r));
      for (int j = lane; j < cnt; j += 32) {
        s_mkey_g[tot + j] = ld_dsmem_u32(dsmem_addr(&s_ckey[g][j], r));
        s_midx_g[tot + j] = (int)ld_dsmem_u32(dsmem_addr(&s_cidx[g][j], r));
      }
      tot += cnt;
    }
    __syncwarp();
    const int cnt = warp_topk(s_mkey_g, tot, K, s_hist[warp], lane, s_pick[g]);
    for (int j = lane; j < cnt; j += 32) s_sel[g][j] = s_midx_g[s_pick[g][j]];
    if (lane == 0) s_nsel[g] = cnt;
  }
  __syncthreads();
  if (rank == 0) {  // optional outputs: the selection of every head
    for (int e = tid; e < G * K; e += kThreads) {
      const int g = e / K, j = e % K;
      const size_t row = (size_t)bi * Hq + h0 + g;
      if (p.idx) p.idx[row * K + j] = j < s_nsel[g] ? s_sel[g][j] : -1;
      if (p.count && j == 0) p.count[row] = s_nsel[g];
    }
  }
  const int nlist = G * K + 1;
  for (int t = tid; t < nlist; t += kThreads) {
    int x = INT_MAX;
    if (t == nlist - 1) {
      x = cur;
    } else {
      const int g = t / K, j = t % K;
      if (j < s_nsel[g]) x = s_sel[g][j];
    }
    s_list[t] = x;
    s_umask[t] = 0u;
  }
  __syncthreads();
  {
    int nf = 0;
    for (int t = tid; t < nlist; t += kThreads) {
      const int x = s_list[t];
      bool first = x != INT_MAX;
      for (int u = 0; u < t && first; ++u) first = s_list[u] != x;
      s_first[t] = first;
      nf += first;
    }
    nf = __reduce_add_sync(0xffffffffu, nf);
    if (lane == 0 && nf) atomicAdd(&s_U, nf);
  }
  __syncthreads();
  for (int t = tid; t < nlist; t += kThreads) {
    const int x = s_list[t];
    if (x == INT_MAX) continue;
    int rk = 0;
    for (int u = 0; u < nlist; ++u) rk += (s_first[u] && s_list[u] < x);
    if (s_first[t]) s_ublk[rk] = x;
    atomicOr(&s_umask[rk], (t == nlist - 1) ? ((1u << G) - 1u) : (1u << (t / K)));
  }
  __syncthreads();
  const int U = s_U;

  // ---- 3. attend my union entries -----------------------------------------------------------
  const size_t tl = FusedSmem<T, D, G>::tile(b);
  T* kbuf[2] = {reinterpret_cast<T*>(smem), reinterpret_cast<T*>(smem + tl)};
  T* vbuf[2] = {reinterpret_cast<T*>(smem + 2 * tl), reinterpret_cast<T*>(smem + 3 * tl)};
  uint64_t* kvbar = bar + p.ns;
  const T* kbase = static_cast<const T*>(p.k) + (size_t)(bi * p.Hk + kh) * p.n * D;
  const T* vbase = static_cast<const T*>(p.v) + (size_t)(bi * p.Hk + kh) * p.n * D;
  const int ne = rank < U ? (U - rank + CL - 1) / CL : 0;
  auto block_tokens = [&](int m) { return m == cur ? pos - cur * b + 1 : b; };
  auto issue_kv = [&](int i) {
    const int m = s_ublk[rank + i * CL];
    const uint32_t bytes = (uint32_t)(block_tokens(m) * D * sizeof(T));
    const int st = i & 1;
    mbar_arrive_expect_tx(&kvbar[st], 2 * bytes);
    bulk_g2s(kbuf[st], kbase + (size_t)m * b * D, bytes, &kvbar[st]);
    bulk_g2s(vbuf[st], vbase + (size_t)m * b * D, bytes, &kvbar[st]);
  };
  if (tid == 0 && !s_abort) {
    fence_proxy_async();  // ring reads of phase 1 precede the async writes into region A
    if (ne > 0) issue_kv(0);
    if (ne > 1) issue_kv(1);
  }
  const float qs2 = kLog2e;  // qv already carries nothing but raw q; logits in log2 units
  float qa[G][EPL];
#pragma unroll
  for (int g = 0; g < G; ++g)
#pragma unroll
    for (int e = 0; e < EPL; ++e) qa[g][e] = qv[g][e] * scale * qs2;
  const int cg = tid % CG, tp = tid / CG;
  float acc[G][2];
#pragma unroll
  for (int g = 0; g < G; ++g) acc[g][0] = acc[g][1] = 0.f;

  for (int i = 0; i < ne; ++i) {
    const int st = i & 1;
    const int m = s_ublk[rank + i * CL];
    const unsigned hm = s_umask[rank + i * CL];
    const int tok = block_tokens(m);
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
    // the block being filled: rewrite its summary from the tile already in shared memory
    if (p.append && m == cur) {
      for (int col = tid; col < D; col += kThreads) {
        float sum = 0.f;
        for (int t = 0; t < tok; ++t) sum += Elem<T>::to_f(kt[(size_t)t * D + col]);
        p.mean_k[((size_t)(bi * p.Hk + kh) * p.C + cur) * D + col] = sum / (float)tok;
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
        const float pv = (m_new == -INFINITY) ? 0.f : exp2f(zs[t * G + g] - m_new);
        ps[t * G + g] = pv;
        sum += pv;
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

  // ---- 4. partials in shared memory, merged across the cluster -----------------------------
  float* red = reinterpret_cast<float*>(smem);  // [TP][G][D], then the partial o [G][D]
#pragma unroll
  for (int g = 0; g < G; ++g) {
    red[((size_t)tp * G + g) * D + 2 * cg] = acc[g][0];
    red[((size_t)tp * G + g) * D + 2 * cg + 1] = acc[g][1];
  }
  __syncthreads();
  float* part = red + (size_t)TP * G * D;  // [G][D]
  for (int e = tid; e < G * D; e += kThreads) {
    float sum = 0.f;
    for (int u = 0; u < TP; ++u) sum += red[(size_t)u * G * D + e];
    part[e] = sum;
  }
  cluster_sync();
  const int cols = D / CL;  // output columns merged by this CTA
  for (int e = tid; e < G * cols; e += kThreads) {
    const int g = e / cols, col = rank * cols + e % cols;
    float M = -INFINITY;
    for (int r = 0; r < CL; ++r) M = fmaxf(M, ld_dsmem_f32(dsmem_addr(&s_m[g], r)));
    float lsum = 0.f, osum = 0.f;
    for (int r = 0; r < CL; ++r) {
      const float mr = ld_dsmem_f32(dsmem_addr(&s_m[g], r));
      const float w = (mr == -INFINITY) ? 0.f : exp2f(mr - M);
      if (w != 0.f) {
        lsum = fmaf(w, ld_dsmem_f32(dsmem_addr(&s_l[g], r)), lsum);
        osum = fmaf(w, ld_dsmem_f32(dsmem_addr(&part[g * D + col], r)), osum);
      }
    }
    const size_t row = (size_t)bi * Hq + h0 + g;
    static_cast<T*>(p.o)[row * D + col] = Elem<T>::from_f(osum / lsum);
    if (col == 0 && p.lse) p.lse[row] = (M + log2f(lsum)) * kLn2;
  }
  cluster_sync();  // keep this CTA's shared memory alive until every peer has read it
}

int pick_cluster(int groups) {
  // the largest power of two (2..16) keeping all clusters resident at about two CTAs per SM
  int cl = 2;
  while (cl * 2 <= kMaxCL && groups * cl * 2 <= 2 * kSMs) cl <<= 1;
  return cl;
}

template <typename T, int D, int G>
bsa_status launch_fused(FusedParams& p, cudaStream_t st) {
  const int groups = p.B * p.Hk;
  int CL = pick_cluster(groups);
  if (D / CL < 1) CL = D;
  const int chunk = std::max(kSub, ceil_div(ceil_div(std::max(p.C, 1), CL), kSub) * kSub);
  p.chunk = chunk;
  p.ns = 3;
  auto kern = decode_fused_kernel<T, D, G>;
  size_t smem = FusedSmem<T, D, G>::bytes(p.b, p.ns, chunk);
  if (smem > 200 * 1024) {
    p.ns = 2;
    smem = FusedSmem<T, D, G>::bytes(p.b, p.ns, chunk);
  }
  if (smem > 200 * 1024) return BSA_ERR_UNSUPPORTED;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
      cudaSuccess) {
    (void)cudaGetLastError();
    return BSA_ERR_CUDA;
  }
  if (CL > 8 &&
      cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess) {
    (void)cudaGetLastError();
    CL = 8;
  }
  for (;;) {
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
    if (cudaOccupancyMaxActiveClusters(&nclusters, kern, &cfg) != cudaSuccess || nclusters <= 0) {
      (void)cudaGetLastError();
      if (CL <= 2) return BSA_ERR_UNSUPPORTED;
      CL >>= 1;
      const int ch = std::max(kSub, ceil_div(ceil_div(std::max(p.C, 1), CL), kSub) * kSub);
      p.chunk = ch;
      smem = FusedSmem<T, D, G>::bytes(p.b, p.ns, ch);
      if (smem > 200 * 1024) return BSA_ERR_UNSUPPORTED;
      if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
          cudaSuccess) {
        (void)cudaGetLastError();
        return BSA_ERR_CUDA;
      }
      continue;
    }
    if (cudaLaunchKernelEx(&cfg, kern, p) != cudaSuccess) {
      (void)cudaGetLastError();
      return BSA_ERR_CUDA;
    }
    return BSA_OK;
  }
}

template <typename T, int D>
bsa_status dispatch_fused(int G, FusedParams& p, cudaStream_t st) {
  switch (G) {
    case 1: return launch_fused<T, D, 1>(p, st);
    case 2: return launch_fused<T, D, 2>(p, st);
    case 4: return launch_fused<T, D, 4>(p, st);
    case 8: return launch_fused<T, D, 8>(p, st);
    default: return BSA_ERR_UNSUPPORTED;
  }
}

}  // namespace
}  // namespace bsa

extern "C" bsa_status bsa_decode_step(const void* q, const void* k, const void* v, bsa_dtype dt,
                                      int B, int Hq, int Hk, int n, int d, int b,
                                      const int* seq_lens, float* mean_k, float* max_norm,
                                      float* centre, int append, const float* lambda_h,
                                      const float* sigma_h, int prefix_block, int K, void* o,
                                      float* lse, int* idx, int* count, int* status,
                                      void* stream) {
  using namespace bsa;
  BSA_REQUIRE(dtype_ok(dt), BSA_ERR_DTYPE);
  BSA_REQUIRE(q && k && v && mean_k && o, BSA_ERR_ARG);
  BSA_REQUIRE(B > 0 && Hq > 0 && Hk > 0 && n > 0 && d > 0 && b > 0 && K > 0 && prefix_block >= 0,
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
  const int C = ceil_div(n, b);
  BSA_REQUIRE(ceil_div(C, kMaxCL) <= 1024 * 1024, BSA_ERR_UNSUPPORTED);
  FusedParams p{};
  p.q = q; p.k = k; p.v = v;
  p.B = B; p.Hq = Hq; p.Hk = Hk; p.n = n; p.b = b; p.C = C; p.K = K;
  p.seq_lens = seq_lens; p.mean_k = mean_k; p.max_norm = max_norm; p.centre = centre;
  p.append = append; p.lam = lambda_h; p.sig = sigma_h; p.prefix_block = prefix_block;
  p.o = o; p.lse = lse; p.idx = idx; p.count = count; p.status = status;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  bsa_status rc;
  if (dt == BSA_BF16)
    rc = d == 64 ? dispatch_fused<__nv_bfloat16, 64>(Hq / Hk, p, st)
                 : dispatch_fused<__nv_bfloat16, 128>(Hq / Hk, p, st);
  else
    rc = d == 64 ? dispatch_fused<float, 64>(Hq / Hk, p, st)
                 : dispatch_fused<float, 128>(Hq / Hk, p, st);
  if (rc != BSA_OK) return rc;
  BSA_LAUNCH_CHECK();
  return BSA_OK;
}
