// FS-L: pre-query pruning of the FreeSolo cells and selection over the kept cells (decode).
//
// [FreeSolo] "How it differs", FS-L variant: before any query arrives each head keeps its W most
// recent cells and the P cells of largest maximum key norm; a query then scores only the kept
// cells with the full method's cell score
//     r_c = q . kbar_c / sqrt(d) + lambda_h a_c erf((i - p_c) / (2 sigma_h))
// and reads its K best, so the per-query cost is O(W + P) instead of O(C).
//   * Pruning: the radix select of the Top-K call over the maximum key norms of the older cells,
//     with the W newest kept outright and written after them (one CTA per (batch, head)).
//   * Selection: one warp per (batch, head) decode query; lane l scores kept cells l, l + 32, ...
//     by itself (q staged in shared memory and read as broadcasts, the cell's mean key as 16-byte
//     loads, all of them in flight at once), then an exact rank count for the top K (ties to the
//     lower cell index, NaN last).
//   * Fixed-size state ("How it differs": O(N) cost, a state of fixed size): per (batch, head) the
//     P kept older cells, ascending.  When the candidate prefix grows by one cell, the cell leaving
//     the W newest joins the older ones and replaces the lowest-ranked kept cell if it outranks it
//     (it has the highest index, so only a strictly larger norm key does); one warp per row, the
//     row's P cells and their norm keys in shared memory, O(P / 32) per new cell.
//   * Decode output: one thread-block cluster of kFslCL CTAs per (batch, head).  Every CTA scores
//     the kept cells and takes the same top K; CTA r attends a quarter of the RoPE window and
//     every kFslCL-th selected cell (NoPE), each warp keeping an online softmax of one branch;
//     the partial (max, sum, output) of both branches meet in CTA 0 through distributed shared
//     memory, which mixes o = (1 - alpha_h) o_short + alpha_h o_long.  RoPE enters through the
//     relative angle: <R_i q, R_j k> = sum over pairs t of (q_a k_a + q_b k_b) cos((j - i) w_t)
//     + (q_b k_a - q_a k_b) sin((j - i) w_t), w_t = theta^(-2t/d), so the raw q and raw keys are
//     read and only angles below the window length (in radians times w_t) are evaluated, stepped
//     from token to token by the angle-addition rule.
#include "bsa_common.cuh"

namespace bsa {

void launch_topk_rows(const float* scores, int rows, int C, int ld, const int* n_cand, int units,
                      int q_block, int b, int K, int* idx, int* count, int out_ld,
                      int keep_newest, cudaStream_t st);

namespace {

constexpr int kMaxKept = 128;  // W + P
constexpr int kRowsPerCta = 4;

__device__ __forceinline__ uint32_t fsl_key(float f) {
  if (f != f) return 0u;
  if (f == 0.f) f = 0.f;
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

template <typename T, int D>
__global__ void __launch_bounds__(32 * kRowsPerCta)
    fsl_select_kernel(const T* __restrict__ q, int B, int H, const int* __restrict__ pos,
                      const float* __restrict__ mean_k, const float* __restrict__ max_norm,
                      const float* __restrict__ centre, int C, const float* __restrict__ lam,
                      const float* __restrict__ sig, const int* __restrict__ cand,
                      const int* __restrict__ cand_count, int cand_ld, int K,
                      int* __restrict__ idx, int* __restrict__ count) {
  __shared__ uint32_t s_key[kRowsPerCta][kMaxKept];
  __shared__ __align__(16) float s_q[kRowsPerCta][D];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * kRowsPerCta + warp;  // (batch, head)
  if (row >= B * H) return;
  const int bi = row / H, h = row % H;
  const int i = pos[bi];
  const int nk = min(max(cand_count[row], 0), min(cand_ld, kMaxKept));
  for (int e = lane; e < D; e += 32) s_q[warp][e] = Elem<T>::to_f(q[(size_t)row * D + e]);
  __syncwarp();
  const float scale = rsqrtf((float)D);
  const float lm = lam ? lam[h] : 0.f;
  const float inv2s = lam ? 0.5f / sig[h] : 0.f;
  const int* crow = cand + (size_t)row * cand_ld;
  const size_t srow = (size_t)row * C;
  uint32_t* keys = s_key[warp];
  const float4* qs = reinterpret_cast<const float4*>(s_q[warp]);
#pragma unroll
  for (int t = 0; t < kMaxKept / 32; ++t) {
    const int j = lane + 32 * t;
    if (j < nk) {
      const int c = crow[j];
      const float4* kp = reinterpret_cast<const float4*>(mean_k + (srow + c) * D);
      float a0 = 0.f, a1 = 0.f;
#pragma unroll
      for (int e4 = 0; e4 < D / 4; ++e4) {
        const float4 kv = kp[e4], qv = qs[e4];
        a0 = fmaf(qv.x, kv.x, fmaf(qv.y, kv.y, a0));
        a1 = fmaf(qv.z, kv.z, fmaf(qv.w, kv.w, a1));
      }
      float r = (a0 + a1) * scale;
      if (lam) r += lm * max_norm[srow + c] * erff(((float)i - centre[srow + c]) * inv2s);
      keys[j] = fsl_key(r);
    }
  }
  __syncwarp();
  // exact top K by rank counting over <= 128 keys (4 per lane); ties to the lower kept slot,
  // which is the lower cell index because the kept list is ascending
  const int kk = min(K, nk);
  uint32_t mk[4];
  int rk[4];
#pragma unroll
  for (int t = 0; t < 4; ++t) {
    mk[t] = lane + 32 * t < nk ? keys[lane + 32 * t] : 0u;
    rk[t] = 0;
  }
  for (int j = 0; j < nk; ++j) {
    const uint32_t kj = keys[j];
#pragma unroll
    for (int t = 0; t < 4; ++t) rk[t] += (kj > mk[t] || (kj == mk[t] && j < lane + 32 * t)) ? 1 : 0;
  }
  int* out = idx + (size_t)row * K;
  const unsigned lt = (1u << lane) - 1u;
  int taken = 0;
#pragma unroll
  for (int t = 0; t < 4; ++t) {
    const bool take = lane + 32 * t < nk && rk[t] < kk;
    const unsigned tb = __ballot_sync(0xffffffffu, take);
    if (take) out[taken + __popc(tb & lt)] = crow[lane + 32 * t];
    taken += __popc(tb);
  }
  for (int j = kk + lane; j < K; j += 32) out[j] = -1;
  if (count && lane == 0) count[row] = kk;
}

// ---- fixed-size state update -------------------------------------------------------------

constexpr int kStateMaxP = 128;
constexpr int kStateRowsPerCta = 4;

// a worse than b: smaller key, or equal keys and the higher cell index (lower rank)
__device__ __forceinline__ bool fsl_worse(uint32_t ka, int ia, uint32_t kb, int ib) {
  return ka < kb || (ka == kb && ia > ib);
}

__global__ void __launch_bounds__(32 * kStateRowsPerCta)
    fsl_state_update_kernel(const float* __restrict__ max_norm, int rows, int C,
                            const int* __restrict__ n_cells, int W, int P, int* __restrict__ older,
                            int* __restrict__ older_count, int* __restrict__ state_cells,
                            int* __restrict__ cand, int* __restrict__ cand_count, int cand_ld) {
  __shared__ int s_idx[kStateRowsPerCta][kStateMaxP];
  __shared__ uint32_t s_key[kStateRowsPerCta][kStateMaxP];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * kStateRowsPerCta + warp;
  if (row >= rows) return;
  int* mi = s_idx[warp];
  uint32_t* mkey = s_key[warp];
  const float* nrm = max_norm + (size_t)row * C;
  int cnt = min(max(older_count[row], 0), P);
  const int from = max(state_cells[row], 0);
  const int to = min(max(n_cells[row], from), C);
  for (int j = lane; j < cnt; j += 32) {
    const int c = older[(size_t)row * P + j];
    mi[j] = c;
    mkey[j] = fsl_key(nrm[c]);
  }
  __syncwarp();
  // cells joining the older ones: c = m - 1 - W for m = from + 1 .. to, in order
  const int c_first = max(0, from - W), c_last = to - W;  // [c_first, c_last)
  const unsigned lt = (1u << lane) - 1u;
  for (int c0 = c_first; c0 < c_last; c0 += 32) {
    const int nb = min(32, c_last - c0);
    const uint32_t my_key = lane < nb ? fsl_key(nrm[c0 + lane]) : 0u;  // prefetch 32 joiners
    for (int t = 0; t < nb; ++t) {
      const int c = c0 + t;
      const uint32_t kc = __shfl_sync(0xffffffffu, my_key, t);
      if (cnt < P) {  // room left: the cell joins (it is the newest, so it goes last)
        if (lane == 0) {
          mi[cnt] = c;
          mkey[cnt] = kc;
        }
        ++cnt;
        __syncwarp();
        continue;
      }
      // the lowest-ranked kept cell and its position
      uint32_t wk = 0xFFFFFFFFu;
      int wi = -1, wp = -1;
      for (int j = lane; j < cnt; j += 32)
        if (wp < 0 || fsl_worse(mkey[j], mi[j], wk, wi)) {
          wk = mkey[j];
          wi = mi[j];
          wp = j;
        }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const uint32_t ok = __shfl_xor_sync(0xffffffffu, wk, o);
        const int oi = __shfl_xor_sync(0xffffffffu, wi, o);
        const int op = __shfl_xor_sync(0xffffffffu, wp, o);
        if (op >= 0 && (wp < 0 || fsl_worse(ok, oi, wk, wi))) {
          wk = ok;
          wi = oi;
          wp = op;
        }
      }
      if (kc > wk) {  // strictly outranks it (equal keys: the lower index, the kept one, wins)
        // drop position wp, shift the rest down by one, append c (the list stays ascending)
        int mv[kStateMaxP / 32];
        uint32_t mkv[kStateMaxP / 32];
#pragma unroll
        for (int u = 0; u < kStateMaxP / 32; ++u) {
          const int j = lane + 32 * u;
          if (j >= wp && j + 1 < cnt) {
            mv[u] = mi[j + 1];
            mkv[u] = mkey[j + 1];
          }
        }
        __syncwarp();
#pragma unroll
        for (int u = 0; u < kStateMaxP / 32; ++u) {
          const int j = lane + 32 * u;
          if (j >= wp && j + 1 < cnt) {
            mi[j] = mv[u];
            mkey[j] = mkv[u];
          }
        }
        if (lane == 0) {
          mi[cnt - 1] = c;
          mkey[cnt - 1] = kc;
        }
      }
      __syncwarp();
    }
  }
  (void)lt;
  for (int j = lane; j < cnt; j += 32) older[(size_t)row * P + j] = mi[j];
  for (int j = cnt + lane; j < P; j += 32) older[(size_t)row * P + j] = -1;
  // the kept cells: the older ones (ascending) then the W newest
  const int r0 = max(0, to - W);
  const int total = cnt + (to - r0);
  int* crow = cand + (size_t)row * cand_ld;
  for (int j = lane; j < cand_ld; j += 32)
    crow[j] = j < cnt ? mi[j] : (j < total ? r0 + (j - cnt) : -1);
  if (lane == 0) {
    older_count[row] = cnt;
    state_cells[row] = to;
    if (cand_count) cand_count[row] = total;
  }
}

// ---- decode output: RoPE window + NoPE long branch over the selected kept cells ------------

constexpr int kFslCL = 4;          // CTAs per (batch, head)
constexpr int kFslThreads = 256;
constexpr int kFslWarps = kFslThreads / 32;
constexpr int kFslMaxK = 8;
constexpr float kFslLog2e = 1.4426950408889634f;

struct FslDecodeParams {
  const void* q;
  const void* k;
  const void* v;
  int B, H, n, cell, C;
  const int* pos;
  const float* mean_k;
  const float* max_norm;
  const float* centre;
  const float* lam;
  const float* sig;
  const float* alpha;
  const int* cand;
  const int* cand_count;
  int cand_ld, K, window;
  double log_theta;
  void* o;
  int* idx;
  int* count;
  int* status;
  int wpc;        // window tokens per CTA
  int cpc;        // selected cells per CTA (ceil(K / kFslCL))
  int off_long;   // byte offsets in the dynamic shared memory
  int off_bar;
};

__device__ __forceinline__ uint32_t fsl_cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void fsl_cluster_arrive() {
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void fsl_cluster_wait() {
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ void fsl_cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;"
               ::: "memory");
}
__device__ __forceinline__ void fsl_st_remote(float* p, uint32_t rank, float v) {
  uint32_t a;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(a) : "r"(smem_u32(p)), "r"(rank));
  asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(a), "f"(v) : "memory");
}

template <typename T, int D>
__global__ void __launch_bounds__(kFslThreads) fsl_decode_kernel(const FslDecodeParams p) {
  constexpr int E = D / 32;   // elements per lane: l, l + 32, ...; pairs (t, t + D/2) share a lane
  constexpr int NP = E / 2;   // RoPE pairs per lane: t = lane + 32 u
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ uint32_t s_key[kMaxKept];
  __shared__ int s_sel[kFslMaxK];
  __shared__ int s_nsel;
  __shared__ __align__(16) float s_q[D];
  __shared__ float s_part[kFslWarps][D + 2];       // per warp: o, m, l (log2 domain)
  __shared__ float s_recv[kFslCL][2][D + 2];       // CTA 0: per CTA and branch
  __shared__ int s_abort;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int rank = (int)fsl_cluster_rank();
  const int h = blockIdx.y, bi = blockIdx.z;
  const int row = bi * p.H + h;
  const int i = min(max(p.pos[bi], 0), p.n - 1);
  const size_t hrow = (size_t)row * p.n;  // first key row of this (batch, head)
  const T* kb = static_cast<const T*>(p.k) + hrow * D;
  const T* vb = static_cast<const T*>(p.v) + hrow * D;
  T* kw = reinterpret_cast<T*>(smem);                     // [wpc][D] window keys
  T* vw = kw + (size_t)p.wpc * D;                         // [wpc][D] window values
  T* kl = reinterpret_cast<T*>(smem + p.off_long);        // [cpc * cell][D] long-branch keys
  T* vl = kl + (size_t)p.cpc * p.cell * D;
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + p.off_bar);  // [0] window, [1] long

  // this CTA's window tokens: [w_lo, w_hi) inside [i - window + 1, i]
  const int lo = max(0, i - p.window + 1);
  const int w_lo = min(i + 1, lo + rank * p.wpc);
  const int w_hi = min(i + 1, w_lo + p.wpc);
  if (tid == 0) {
    mbar_init(&bar[0], 1);
    mbar_init(&bar[1], 1);
    fence_mbar_init();
    s_abort = 0;
    if (w_hi > w_lo) {
      const uint32_t bytes = (uint32_t)((w_hi - w_lo) * D * sizeof(T));
      mbar_arrive_expect_tx(&bar[0], 2 * bytes);
      bulk_g2s(kw, kb + (size_t)w_lo * D, bytes, &bar[0]);
      bulk_g2s(vw, vb + (size_t)w_lo * D, bytes, &bar[0]);
    }
  }
  for (int e = tid; e < D; e += kFslThreads)
    s_q[e] = Elem<T>::to_f(static_cast<const T*>(p.q)[(size_t)row * D + e]);
  __syncthreads();
  fsl_cluster_arrive();  // every CTA has started before peers write into its shared memory

  // ---- selection among the kept cells (every CTA, same arithmetic as bsa_fsl_select) --------
  const int nk = min(max(p.cand_count[row], 0), min(p.cand_ld, kMaxKept));
  const int* crow = p.cand + (size_t)row * p.cand_ld;
  {
    const float scale = rsqrtf((float)D);
    const float lm = p.lam ? p.lam[h] : 0.f;
    const float inv2s = p.lam ? 0.5f / p.sig[h] : 0.f;
    const size_t srow = (size_t)row * p.C;
    const float4* qs = reinterpret_cast<const float4*>(s_q);
    for (int j = tid; j < nk; j += kFslThreads) {
      const int c = crow[j];
      const float4* kp = reinterpret_cast<const float4*>(p.mean_k + (srow + c) * D);
      float a0 = 0.f, a1 = 0.f;
#pragma unroll
      for (int e4 = 0; e4 < D / 4; ++e4) {
        const float4 kv = kp[e4], qv = qs[e4];
        a0 = fmaf(qv.x, kv.x, fmaf(qv.y, kv.y, a0));
        a1 = fmaf(qv.z, kv.z, fmaf(qv.w, kv.w, a1));
      }
      float r = (a0 + a1) * scale;
      if (p.lam) r += lm * p.max_norm[srow + c] * erff(((float)i - p.centre[srow + c]) * inv2s);
      s_key[j] = fsl_key(r);
    }
  }
  __syncthreads();
  if (warp == 0) {
    const int kk = min(p.K, nk);
    uint32_t mk[4];
    int rk[4];
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      mk[t] = lane + 32 * t < nk ? s_key[lane + 32 * t] : 0u;
      rk[t] = 0;
    }
    for (int j = 0; j < nk; ++j) {
      const uint32_t kj = s_key[j];
#pragma unroll
      for (int t = 0; t < 4; ++t) rk[t] += (kj > mk[t] || (kj == mk[t] && j < lane + 32 * t)) ? 1 : 0;
    }
    const unsigned lt = (1u << lane) - 1u;
    int taken = 0;
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const bool take = lane + 32 * t < nk && rk[t] < kk;
      const unsigned tb = __ballot_sync(0xffffffffu, take);
      if (take) s_sel[taken + __popc(tb & lt)] = crow[lane + 32 * t];
      taken += __popc(tb);
    }
    if (lane == 0) s_nsel = taken;
  }
  __syncthreads();
  const int nsel = s_nsel;
  // my cells: slots rank, rank + CL, ... of the (ascending) selection
  const int my_cells = nsel > rank ? (nsel - rank + kFslCL - 1) / kFslCL : 0;
  if (tid == 0 && my_cells > 0) {
    const uint32_t bytes = (uint32_t)(p.cell * D * sizeof(T));
    mbar_arrive_expect_tx(&bar[1], 2 * bytes * my_cells);
    for (int u = 0; u < my_cells; ++u) {
      const int c = s_sel[rank + u * kFslCL];
      bulk_g2s(kl + (size_t)u * p.cell * D, kb + (size_t)c * p.cell * D, bytes, &bar[1]);
      bulk_g2s(vl + (size_t)u * p.cell * D, vb + (size_t)c * p.cell * D, bytes, &bar[1]);
    }
  }
  if (rank == 0 && p.idx) {  // optional outputs: the selected cells, ascending
    for (int j = tid; j < p.K; j += kFslThreads) p.idx[(size_t)row * p.K + j] = j < nsel ? s_sel[j] : -1;
    if (tid == 0 && p.count) p.count[row] = nsel;
  }

  // ---- the two branches: warps 0 .. 3 the window, warps 4 .. 7 the long branch ---------------
  float qr[E];
#pragma unroll
  for (int e = 0; e < E; ++e) qr[e] = s_q[lane + 32 * e] * (rsqrtf((float)D) * kFslLog2e);
  const bool is_win = warp < kFslWarps / 2;
  const int sub = warp % (kFslWarps / 2);
  const int ntok = is_win ? w_hi - w_lo : my_cells * p.cell;
  const T* kt = is_win ? kw : kl;
  const T* vt = is_win ? vw : vl;
  float m_run = -INFINITY, l_run = 0.f, acc[E];
#pragma unroll
  for (int e = 0; e < E; ++e) acc[e] = 0.f;
  bool ready = true;
  if (ntok > 0) ready = mbar_wait_bounded(&bar[is_win ? 0 : 1], 0);
  if (!ready) s_abort = 1;
  // token chunks of 32: chunk c0 = 32 (sub + 4 u)
  for (int c0 = 32 * sub; ready && c0 < ntok; c0 += 32 * (kFslWarps / 2)) {
    const int nt = min(32, ntok - c0);
    float a[32];
    if (is_win) {
      // rotation of each pair by the relative angle (j - i) w_t, stepped by w_t per token
      float cw[NP], sw[NP], cs[NP], sn[NP];
#pragma unroll
      for (int u = 0; u < NP; ++u) {
        const int t = lane + 32 * u;
        const double w = exp(-2.0 * t / D * p.log_theta);
        double ang = (double)(w_lo + c0 - i) * w;
        ang -= 6.283185307179586 * rint(ang / 6.283185307179586);
        sincosf((float)ang, &sn[u], &cs[u]);
        float sw1, cw1;
        sincosf((float)w, &sw1, &cw1);
        cw[u] = cw1;
        sw[u] = sw1;
      }
#pragma unroll
      for (int r = 0; r < 32; ++r) {
        float s = 0.f;
        if (r < nt) {
          const T* kr = kt + (size_t)(c0 + r) * D;
#pragma unroll
          for (int u = 0; u < NP; ++u) {
            const float ka = Elem<T>::to_f(kr[lane + 32 * u]);
            const float kb2 = Elem<T>::to_f(kr[lane + 32 * u + D / 2]);
            const float qa = qr[u], qb = qr[u + NP];
            s = fmaf(fmaf(qa, ka, qb * kb2), cs[u], s);
            s = fmaf(fmaf(qb, ka, -qa * kb2), sn[u], s);
          }
        }
        a[r] = s;
#pragma unroll
        for (int u = 0; u < NP; ++u) {  // step to the next token
          const float c2 = cs[u] * cw[u] - sn[u] * sw[u];
          sn[u] = fmaf(sn[u], cw[u], cs[u] * sw[u]);
          cs[u] = c2;
        }
      }
    } else {
#pragma unroll
      for (int r = 0; r < 32; ++r) {
        float s = 0.f;
        if (r < nt) {
          const T* kr = kt + (size_t)(c0 + r) * D;
#pragma unroll
          for (int e = 0; e < E; ++e) s = fmaf(qr[e], Elem<T>::to_f(kr[lane + 32 * e]), s);
        }
        a[r] = s;
      }
    }
    warp_transpose_reduce32(a, lane);
    const float z = lane < nt ? a[0] : -INFINITY;  // logit of token c0 + lane (log2 units)
    const float mx = fmaxf(m_run, warp_max(z));
    const float corr = m_run == -INFINITY ? 0.f : exp2f(m_run - mx);
    const float pz = z == -INFINITY ? 0.f : exp2f(z - mx);
    l_run = l_run * corr + warp_sum(pz);
#pragma unroll
    for (int e = 0; e < E; ++e) acc[e] *= corr;
    for (int r = 0; r < nt; ++r) {
      const float pr = __shfl_sync(0xffffffffu, pz, r);
      const T* vr = vt + (size_t)(c0 + r) * D;
#pragma unroll
      for (int e = 0; e < E; ++e) acc[e] = fmaf(pr, Elem<T>::to_f(vr[lane + 32 * e]), acc[e]);
    }
    m_run = mx;
  }
#pragma unroll
  for (int e = 0; e < E; ++e) s_part[warp][lane + 32 * e] = acc[e];
  if (lane == 0) {
    s_part[warp][D] = m_run;
    s_part[warp][D + 1] = l_run;
  }
  __syncthreads();
  if (s_abort && tid == 0) {
    // copies that may still be in flight: give them a bounded chance to land, record the timeout
    (void)mbar_wait_bounded(&bar[0], 0, 1u << 12);
    if (my_cells > 0) (void)mbar_wait_bounded(&bar[1], 0, 1u << 12);
    if (p.status) atomicCAS(p.status, 0, 3);
  }
  // combine the four warps of each branch, push the CTA's two partials to CTA 0
  fsl_cluster_wait();
  for (int e = tid; e < 2 * (D + 2); e += kFslThreads) {
    const int br = e / (D + 2), col = e % (D + 2);
    const int w0 = br * (kFslWarps / 2);
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kFslWarps / 2; ++w) M = fmaxf(M, s_part[w0 + w][D]);
    float val;
    if (col == D) {
      val = M;
    } else {
      val = 0.f;
#pragma unroll
      for (int w = 0; w < kFslWarps / 2; ++w) {
        const float mw = s_part[w0 + w][D];
        if (mw != -INFINITY) val = fmaf(exp2f(mw - M), s_part[w0 + w][col == D + 1 ? D + 1 : col], val);
      }
    }
    fsl_st_remote(&s_recv[rank][br][col], 0, val);
  }
  fsl_cluster_sync();
  if (rank == 0) {
    const float al = nsel > 0 ? p.alpha[h] : 0.f;
    for (int col = tid; col < D; col += kFslThreads) {
      float out = 0.f;
#pragma unroll
      for (int br = 0; br < 2; ++br) {
        float M = -INFINITY;
        for (int r = 0; r < kFslCL; ++r) M = fmaxf(M, s_recv[r][br][D]);
        float L = 0.f, O = 0.f;
        for (int r = 0; r < kFslCL; ++r) {
          const float mr = s_recv[r][br][D];
          if (mr == -INFINITY) continue;
          const float w = exp2f(mr - M);
          L = fmaf(w, s_recv[r][br][D + 1], L);
          O = fmaf(w, s_recv[r][br][col], O);
        }
        const float ob = L > 0.f ? O / L : 0.f;
        out += br == 0 ? (1.f - al) * ob : al * ob;
      }
      static_cast<T*>(p.o)[(size_t)row * D + col] = Elem<T>::from_f(out);
    }
  }
}

template <typename T, int D>
bsa_status launch_fsl_decode(FslDecodeParams& p, cudaStream_t st) {
  p.wpc = ceil_div(p.window, kFslCL);
  p.cpc = ceil_div(p.K, kFslCL);
  const size_t win = align_up((size_t)2 * p.wpc * D * sizeof(T), 128);
  const size_t lng = align_up((size_t)2 * p.cpc * p.cell * D * sizeof(T), 128);
  p.off_long = (int)win;
  p.off_bar = (int)(win + lng);
  const size_t smem = win + lng + 64;
  if (smem > 200 * 1024) return BSA_ERR_UNSUPPORTED;
  auto kern = fsl_decode_kernel<T, D>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
      cudaSuccess) {
    (void)cudaGetLastError();
    return BSA_ERR_CUDA;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(kFslCL, p.H, p.B);
  cfg.blockDim = dim3(kFslThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = kFslCL;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kern, p) != cudaSuccess) {
    (void)cudaGetLastError();
    return BSA_ERR_CUDA;
  }
  return BSA_OK;
}

}  // namespace
}  // namespace bsa

extern "C" bsa_status bsa_fsl_state_update(const float* max_norm, int rows, int C,
                                           const int* n_cells, int W, int P, int* older,
                                           int* older_count, int* state_cells, int* cand,
                                           int* cand_count, void* stream) {
  using namespace bsa;
  BSA_REQUIRE(max_norm && n_cells && older && older_count && state_cells && cand, BSA_ERR_ARG);
  BSA_REQUIRE(rows >= 0 && C >= 0 && W >= 0 && P > 0, BSA_ERR_ARG);
  BSA_REQUIRE(P <= kStateMaxP && W + P <= kMaxKept, BSA_ERR_UNSUPPORTED);
  if (rows == 0) return BSA_OK;
  const unsigned grid = (unsigned)((rows + kStateRowsPerCta - 1) / kStateRowsPerCta);
  fsl_state_update_kernel<<<grid, 32 * kStateRowsPerCta, 0, static_cast<cudaStream_t>(stream)>>>(
      max_norm, rows, C, n_cells, W, P, older, older_count, state_cells, cand, cand_count, W + P);
  BSA_LAUNCH_CHECK();
  return BSA_OK;
}

extern "C" bsa_status bsa_fsl_decode(const void* q, const void* k, const void* v, bsa_dtype dt,
                                     int B, int H, int n, int d, const int* pos, int cell,
                                     const float* mean_k, const float* max_norm,
                                     const float* centre, const float* lambda_h,
                                     const float* sigma_h, const float* alpha_h, const int* cand,
                                     const int* cand_count, int cand_ld, int K, int window,
                                     float rope_theta, void* o, int* idx, int* count, int* status,
                                     void* stream) {
  using namespace bsa;
  BSA_REQUIRE(dtype_ok(dt), BSA_ERR_DTYPE);
  BSA_REQUIRE(q && k && v && pos && mean_k && alpha_h && cand && cand_count && o, BSA_ERR_ARG);
  BSA_REQUIRE((lambda_h == nullptr) == (sigma_h == nullptr), BSA_ERR_ARG);
  BSA_REQUIRE(!lambda_h || (max_norm && centre), BSA_ERR_ARG);
  BSA_REQUIRE(B > 0 && H > 0 && n > 0 && cell > 0 && cand_ld > 0 && K > 0 && window > 0 &&
                  rope_theta > 0.f,
              BSA_ERR_ARG);
  BSA_REQUIRE(head_dim_ok(d), BSA_ERR_UNSUPPORTED);
  BSA_REQUIRE(cand_ld <= kMaxKept && K <= kFslMaxK && cell <= 128 && window <= 1024,
              BSA_ERR_UNSUPPORTED);
  BSA_REQUIRE(B <= 65535 && H <= 65535, BSA_ERR_UNSUPPORTED);
  BSA_REQUIRE(all_aligned16(q, k, v, o, mean_k), BSA_ERR_ARG);
  FslDecodeParams p{};
  p.q = q; p.k = k; p.v = v;
  p.B = B; p.H = H; p.n = n; p.cell = cell; p.C = ceil_div(n, cell);
  p.pos = pos; p.mean_k = mean_k; p.max_norm = max_norm; p.centre = centre;
  p.lam = lambda_h; p.sig = sigma_h; p.alpha = alpha_h;
  p.cand = cand; p.cand_count = cand_count; p.cand_ld = cand_ld; p.K = K; p.window = window;
  p.log_theta = std::log((double)rope_theta);
  p.o = o; p.idx = idx; p.count = count; p.status = status;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  bsa_status rc;
  if (dt == BSA_BF16)
    rc = d == 64 ? launch_fsl_decode<__nv_bfloat16, 64>(p, st)
                 : launch_fsl_decode<__nv_bfloat16, 128>(p, st);
  else
    rc = d == 64 ? launch_fsl_decode<float, 64>(p, st) : launch_fsl_decode<float, 128>(p, st);
  if (rc != BSA_OK) return rc;
  BSA_LAUNCH_CHECK();
  return BSA_OK;
}

extern "C" bsa_status bsa_fsl_prune(const float* max_norm, int rows, int C, const int* n_cells,
                                    int W, int P, int* cand, int* cand_count, void* stream) {
  using namespace bsa;
  BSA_REQUIRE(max_norm && n_cells && cand, BSA_ERR_ARG);
  BSA_REQUIRE(rows >= 0 && C >= 0 && W >= 0 && P > 0, BSA_ERR_ARG);
  BSA_REQUIRE(C <= 16384 && P <= 256 && W + P <= kMaxKept, BSA_ERR_UNSUPPORTED);
  if (rows == 0) return BSA_OK;
  launch_topk_rows(max_norm, rows, C, C, n_cells, 0, 0, 0, P, cand, cand_count, W + P, W,
                   static_cast<cudaStream_t>(stream));
  BSA_LAUNCH_CHECK();
  return BSA_OK;
}

extern "C" bsa_status bsa_fsl_select(const void* q, bsa_dtype dt, int B, int H, int d,
                                     const int* pos, const float* mean_k, const float* max_norm,
                                     const float* centre, int C, const float* lambda_h,
                                     const float* sigma_h, const int* cand,
                                     const int* cand_count, int cand_ld, int K, int* idx,
                                     int* count, void* stream) {
  using namespace bsa;
  BSA_REQUIRE(dtype_ok(dt), BSA_ERR_DTYPE);
  BSA_REQUIRE(q && pos && mean_k && cand && cand_count && idx, BSA_ERR_ARG);
  BSA_REQUIRE((lambda_h == nullptr) == (sigma_h == nullptr), BSA_ERR_ARG);
  BSA_REQUIRE(!lambda_h || (max_norm && centre), BSA_ERR_ARG);
  BSA_REQUIRE(B > 0 && H > 0 && C >= 0 && cand_ld > 0 && K > 0, BSA_ERR_ARG);
  BSA_REQUIRE(head_dim_ok(d), BSA_ERR_UNSUPPORTED);
  BSA_REQUIRE(cand_ld <= kMaxKept, BSA_ERR_UNSUPPORTED);
  BSA_REQUIRE(all_aligned16(q, mean_k), BSA_ERR_ARG);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int rows = B * H;
  const unsigned grid = (unsigned)((rows + kRowsPerCta - 1) / kRowsPerCta);
  if (dt == BSA_BF16) {
    if (d == 64)
      fsl_select_kernel<__nv_bfloat16, 64><<<grid, 32 * kRowsPerCta, 0, st>>>(
          static_cast<const __nv_bfloat16*>(q), B, H, pos, mean_k, max_norm, centre, C,
          lambda_h, sigma_h, cand, cand_count, cand_ld, K, idx, count);
    else
      fsl_select_kernel<__nv_bfloat16, 128><<<grid, 32 * kRowsPerCta, 0, st>>>(
          static_cast<const __nv_bfloat16*>(q), B, H, pos, mean_k, max_norm, centre, C,
          lambda_h, sigma_h, cand, cand_count, cand_ld, K, idx, count);
  } else {
    if (d == 64)
      fsl_select_kernel<float, 64><<<grid, 32 * kRowsPerCta, 0, st>>>(
          static_cast<const float*>(q), B, H, pos, mean_k, max_norm, centre, C, lambda_h,
          sigma_h, cand, cand_count, cand_ld, K, idx, count);
    else
      fsl_select_kernel<float, 128><<<grid, 32 * kRowsPerCta, 0, st>>>(
          static_cast<const float*>(q), B, H, pos, mean_k, max_norm, centre, C, lambda_h,
          sigma_h, cand, cand_count, cand_ld, K, idx, count);
  }
  BSA_LAUNCH_CHECK();
  return BSA_OK;
}
