// Decode sparse attention: exact softmax of one query per (batch, query head) over the tokens of
// its selected history blocks and its current block.
//
// [SAS] review, "Background" Eq. 2 (attention restricted to the selected set S, cost O(|S|)),
// "The new approach" Eq. 4 / Eq. 9 (current block always kept with gate 1; optional log-gate on
// the selected history blocks), "How it works" step 6 (inference: plain Top-K then sparse
// attention); [Monodratic] (guaranteed local block, exact causal softmax over selected tokens).
//
// B200 design (HBM-bound, no tensor cores: 2 FLOP per byte moved):
//  * The G query heads of a kv group usually pick overlapping blocks, so a CTA works on the UNION
//    of the group's selections (plus the current block): every selected K/V block crosses HBM
//    once and is scored against all G heads, each head masking blocks it did not select.
//  * A selected block of b tokens is one contiguous b*d run of K (and of V) in the [B,Hk,n,d]
//    cache, so the gather is a single untiled bulk copy (cp.async.bulk, the TMA engine) per
//    tensor per block, double-buffered in shared memory and completed on an mbarrier.
//  * Split-K: S CTAs per (batch, kv head) take union entries s, s+S, ... and write partial
//    (m, l, o) per head; the last CTA to arrive (atomic counter, no spinning) merges the S
//    partials with the online-softmax combine and resets the counter for the next call.
//  * Logits of R = 32/G tokens x G heads are reduced with one 31-shuffle transpose-reduce.
#include "bsa_common.cuh"

#include <mutex>

namespace bsa {
namespace {

constexpr int kThreads = 128;
constexpr int kWarps = kThreads / 32;
constexpr int kMaxList = 512;  // G*K + 1 entries of the union candidates
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

struct DecodeParams {
  const void* q;
  const void* k;
  const void* v;
  int B, Hq, Hk, n, b, K;
  const int* seq_lens;
  const int* idx;
  const int* count;
  int gate;  // bsa_gate_mode
  int norm;  // bsa_gate_norm
  const float* scores;
  int scores_ld;
  void* o;
  float* lse;
  float* part;    // [B, Hq, S, D + 2]
  int* counters;  // [B * Hk]
  int* status;
  int S;
};

// Shared-memory layout (dynamic): a stage area holding two K/V stages (reused afterwards for the
// split reduction and the merge weights), then the per-block logits and weights.
template <typename T, int D, int G>
struct DecodeSmem {
  __host__ __device__ static size_t tile_bytes(int b) { return align_up((size_t)b * D * sizeof(T), 128); }
  __host__ __device__ static size_t stage_bytes(int b, int S) {
    const size_t tp = kThreads / (D / 2);
    size_t x = 4 * tile_bytes(b);
    x = max_sz(x, align_up(tp * G * D * sizeof(float), 128));  // split reduction
    x = max_sz(x, align_up((size_t)G * S * sizeof(float), 128));  // merge weights
    return x;
  }
  __host__ __device__ static size_t bytes(int b, int S) {
    return stage_bytes(b, S) + align_up((size_t)b * G * 4, 16) * 2  // z, p  [b][G]
           + 256;                                                    // barriers
  }
};

template <typename T, int D, int G>
__global__ void __launch_bounds__(kThreads)
    decode_attn_kernel(const DecodeParams p) {
  constexpr int EPL = D / 32;  // head-dim elements per lane (logits)
  constexpr int R = 32 / G;    // tokens per transpose-reduce step
  constexpr int CG = D / 2;    // column pairs (PV)
  constexpr int TP = kThreads / CG > 0 ? kThreads / CG : 1;  // token partitions (PV)
  static_assert(kThreads % CG == 0, "PV mapping");

  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ int s_list[kMaxList];
  __shared__ unsigned char s_first[kMaxList];
  __shared__ int s_ublk[kMaxList];
  __shared__ unsigned int s_umask[kMaxList];
  __shared__ int s_U;
  __shared__ float s_lse_norm[G];
  __shared__ float s_m[G], s_l[G], s_corr[G];
  __shared__ int s_last;
  __shared__ int s_abort;

  const int b = p.b;
  const size_t tile = DecodeSmem<T, D, G>::tile_bytes(b);
  const size_t stage = DecodeSmem<T, D, G>::stage_bytes(b, p.S);
  T* kbuf[2] = {reinterpret_cast<T*>(smem), reinterpret_cast<T*>(smem + tile)};
  T* vbuf[2] = {reinterpret_cast<T*>(smem + 2 * tile), reinterpret_cast<T*>(smem + 3 * tile)};
  float* zs = reinterpret_cast<float*>(smem + stage);  // [b][G]
  float* ps = zs + align_up((size_t)b * G, 4);          // [b][G]
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + DecodeSmem<T, D, G>::bytes(b, p.S) - 256);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int s = blockIdx.x, kh = blockIdx.y, bi = blockIdx.z;
  const int S = p.S, K = p.K, Hq = p.Hq;
  const int L = p.seq_lens ? min(p.seq_lens[bi], p.n) : p.n;
  const int pos = L - 1;
  const int cur = pos / b;
  const int h0 = kh * G;

  // ---- 1. union of the group's selections plus the current block -----------------------
  const int nlist = G * K + 1;
  if (tid == 0) s_U = 0;
  for (int t = tid; t < nlist; t += kThreads) {
    int x = INT_MAX;
    if (t == nlist - 1) {
      x = cur;
    } else {
      const int g = t / K, j = t % K;
      const size_t row = (size_t)bi * Hq + h0 + g;
      const int cnt = p.count ? p.count[row] : K;
      if (j < cnt) {
        const int m = p.idx[row * K + j];
        if (m >= 0 && m < cur) x = m;  // entries outside the history are ignored
      }
    }
    s_list[t] = x;
    s_umask[t] = 0u;
  }
  __syncthreads();
  {
    int nfirst = 0;
    for (int t = tid; t < nlist; t += kThreads) {
      const int x = s_list[t];
      bool first = x != INT_MAX;
      for (int u = 0; u < t && first; ++u) first = s_list[u] != x;
      s_first[t] = first;
      nfirst += first;
    }
    nfirst = __reduce_add_sync(0xffffffffu, nfirst);
    if (lane == 0 && nfirst) atomicAdd(&s_U, nfirst);
  }
  __syncthreads();
  for (int t = tid; t < nlist; t += kThreads) {
    const int x = s_list[t];
    if (x == INT_MAX) continue;
    int rank = 0;
    for (int u = 0; u < nlist; ++u) rank += (s_first[u] && s_list[u] < x);
    if (s_first[t]) s_ublk[rank] = x;
    const unsigned bit = (t == nlist - 1) ? ((1u << G) - 1u) : (1u << (t / K));
    atomicOr(&s_umask[rank], bit);
  }
  __syncthreads();
  const int U = s_U;

  // ---- 2. gate normalisers ---------------------------------------------------------------
  const bool gated = p.gate == BSA_GATE_LOG_SOFTMAX;
  if (gated) {
    for (int g = warp; g < G; g += kWarps) {
      const size_t row = (size_t)bi * Hq + h0 + g;
      const float* srow = p.scores + row * p.scores_ld;
      float mx = -INFINITY, acc = 0.f;
      if (p.norm == BSA_NORM_ALL_HISTORY) {
        for (int c = lane; c < cur; c += 32) mx = fmaxf(mx, srow[c]);
        mx = warp_max(mx);
        for (int c = lane; c < cur; c += 32) acc += exp2f((srow[c] - mx) * kLog2e);
      } else {
        const int cnt = p.count ? p.count[row] : K;
        for (int j = lane; j < min(cnt, K); j += 32) {
          const int m = p.idx[row * K + j];
          if (m >= 0 && m < cur) mx = fmaxf(mx, srow[m]);
        }
        mx = warp_max(mx);
        for (int j = lane; j < min(cnt, K); j += 32) {
          const int m = p.idx[row * K + j];
          if (m >= 0 && m < cur) acc += exp2f((srow[m] - mx) * kLog2e);
        }
      }
      acc = warp_sum(acc);
      if (lane == 0) s_lse_norm[g] = (mx == -INFINITY) ? 0.f : mx + logf(acc);
    }
  }

  // ---- 3. stream my union entries through two shared-memory stages ------------------------
  const int ne = s < U ? (U - s + S - 1) / S : 0;
  if (tid == 0) {
    mbar_init(&bar[0], 1);
    mbar_init(&bar[1], 1);
    fence_mbar_init();
    s_abort = 0;
  }
  if (tid < G) {
    s_m[tid] = -INFINITY;
    s_l[tid] = 0.f;
  }
  __syncthreads();

  const T* kbase = static_cast<const T*>(p.k) + (size_t)(bi * p.Hk + kh) * p.n * D;
  const T* vbase = static_cast<const T*>(p.v) + (size_t)(bi * p.Hk + kh) * p.n * D;
  auto block_tokens = [&](int m) { return m == cur ? pos - cur * b + 1 : b; };
  auto issue = [&](int i) {
    const int m = s_ublk[s + i * S];
    const uint32_t bytes = (uint32_t)(block_tokens(m) * D * sizeof(T));
    const int st = i & 1;
    mbar_arrive_expect_tx(&bar[st], 2 * bytes);
    bulk_g2s(kbuf[st], kbase + (size_t)m * b * D, bytes, &bar[st]);
    bulk_g2s(vbuf[st], vbase + (size_t)m * b * D, bytes, &bar[st]);
  };
  if (tid == 0) {
    if (ne > 0) issue(0);
    if (ne > 1) issue(1);
  }

  // query slices, pre-scaled so logits come out in log2 units
  float qv[G][EPL];
  {
    const float qs = rsqrtf((float)D) * kLog2e;
#pragma unroll
    for (int g = 0; g < G; ++g) {
      float tmp[EPL];
      load_vec<T, EPL>(static_cast<const T*>(p.q) + ((size_t)bi * Hq + h0 + g) * D + lane * EPL,
                       tmp);
#pragma unroll
      for (int e = 0; e < EPL; ++e) qv[g][e] = tmp[e] * qs;
    }
  }
  const int cg = tid % CG, tp = tid / CG;
  float acc[G][2];
#pragma unroll
  for (int g = 0; g < G; ++g) acc[g][0] = acc[g][1] = 0.f;

  int i_stop = ne;  // the iteration at which a timed-out wait ended the loop (ne: none did)
  for (int i = 0; i < ne; ++i) {
    const int st = i & 1;
    const int ue = s + i * S;
    const int m = s_ublk[ue];
    const unsigned hm = s_umask[ue];
    const int tok = block_tokens(m);
    float bias[G];
#pragma unroll
    for (int g = 0; g < G; ++g) {
      bias[g] = 0.f;
      if (gated && m != cur)
        bias[g] = (p.scores[((size_t)bi * Hq + h0 + g) * p.scores_ld + m] - s_lse_norm[g]) * kLog2e;
    }
    if (!mbar_wait_bounded(&bar[st], (i >> 1) & 1)) s_abort = 1;
    __syncthreads();
    if (s_abort) {
      i_stop = i;
      break;
    }
    const T* kt = kbuf[st];
    const T* vt = vbuf[st];

    // logits: groups of R tokens, round-robin over warps
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
          for (int e = 0; e < EPL; ++e) sacc = fmaf(qv[g][e], x[e], sacc);
          a[r * G + g] = sacc;
        }
      }
      warp_transpose_reduce32(a, lane);
      const int t = t0 + lane / G, g = lane % G;
      if (t < tok) {
        float z = a[0];
        float bg = 0.f;
#pragma unroll
        for (int gg = 0; gg < G; ++gg)
          if (gg == g) bg = bias[gg];
        z = ((hm >> g) & 1u) ? z + bg : -INFINITY;
        zs[t * G + g] = z;
      }
    }
    __syncthreads();

    // per-head online softmax over this block
    for (int g = warp; g < G; g += kWarps) {
      float mx = -INFINITY;
      for (int t = lane; t < tok; t += 32) mx = fmaxf(mx, zs[t * G + g]);
      mx = warp_max(mx);
      const float m_old = s_m[g];
      const float m_new = fmaxf(m_old, mx);
      float sum = 0.f;
      for (int t = lane; t < tok; t += 32) {
        const float z = zs[t * G + g];
        const float pv = (m_new == -INFINITY) ? 0.f : exp2f(z - m_new);
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

    // P V for this block
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const float c = s_corr[g];
      acc[g][0] *= c;
      acc[g][1] *= c;
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
    __syncthreads();  // stage st and zs/ps free again
    if (tid == 0 && i + 2 < ne) issue(i + 2);
  }

  const bool aborted = s_abort != 0;
  if (aborted) {
    // The copies still in flight are those of iterations i_stop and i_stop + 1 (if issued), with
    // the parities of their own phases; give them a bounded chance to land before the CTA leaves
    // its shared memory, then record the timeout.  The CTA still arrives on the counter below, so
    // the counter ends the call at zero for the next one.
    if (tid == 0) {
      for (int j = i_stop; j < min(ne, i_stop + 2); ++j)
        (void)mbar_wait_bounded(&bar[j & 1], (j >> 1) & 1, 1u << 16);
      report_timeout(p.status, 1);
    }
  } else {
    // ---- 4. partial (m, l, o) of this split -----------------------------------------------
    float* red = reinterpret_cast<float*>(smem);  // reuse the K stage: [TP][G][D]
#pragma unroll
    for (int g = 0; g < G; ++g) {
      red[((size_t)tp * G + g) * D + 2 * cg] = acc[g][0];
      red[((size_t)tp * G + g) * D + 2 * cg + 1] = acc[g][1];
    }
    __syncthreads();
    for (int e = tid; e < G * D; e += kThreads) {
      const int g = e / D, dcol = e % D;
      float sum = 0.f;
      for (int u = 0; u < TP; ++u) sum += red[((size_t)u * G + g) * D + dcol];
      float* pp = p.part + (((size_t)bi * Hq + h0 + g) * S + s) * (D + 2);
      pp[dcol] = sum;
      if (dcol == 0) {
        pp[D] = s_m[g];
        pp[D + 1] = s_l[g];
      }
    }
  }

  // ---- 5. the last CTA of this (batch, kv head) merges the S partials --------------------
  __threadfence();
  __syncthreads();
  if (tid == 0) {
    const int prev = atomicAdd(&p.counters[bi * p.Hk + kh], 1);
    s_last = (prev == S - 1);
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  // A split that timed out wrote the status word before it arrived: its partial is missing, so
  // the merge is skipped (the output is not written; the caller reads BSA_ERR_TIMEOUT) and the
  // counter is reset for the next call.
  if (p.status && *reinterpret_cast<volatile int*>(p.status) != 0) {
    if (tid == 0) p.counters[bi * p.Hk + kh] = 0;
    return;
  }
  float* wgt = reinterpret_cast<float*>(smem);  // [G][S] merge weights, in the stage area
  for (int g = warp; g < G; g += kWarps) {
    const float* pb = p.part + ((size_t)bi * Hq + h0 + g) * S * (D + 2);
    float M = -INFINITY;
    for (int u = lane; u < S; u += 32) M = fmaxf(M, __ldcg(pb + (size_t)u * (D + 2) + D));
    M = warp_max(M);
    float lsum = 0.f;
    for (int u = lane; u < S; u += 32) {
      const float mu = __ldcg(pb + (size_t)u * (D + 2) + D);
      const float lu = __ldcg(pb + (size_t)u * (D + 2) + D + 1);
      const float w = (mu == -INFINITY) ? 0.f : exp2f(mu - M);
      wgt[g * S + u] = w;
      lsum += w * lu;
    }
    lsum = warp_sum(lsum);
    if (lane == 0) {
      s_l[g] = lsum;
      s_m[g] = M;
    }
  }
  __syncthreads();
  for (int e = tid; e < G * D; e += kThreads) {
    const int g = e / D, dcol = e % D;
    const float* pb = p.part + ((size_t)bi * Hq + h0 + g) * S * (D + 2);
    float sum = 0.f;
    for (int u = 0; u < S; ++u) {
      const float w = wgt[g * S + u];
      if (w != 0.f) sum = fmaf(w, __ldcg(pb + (size_t)u * (D + 2) + dcol), sum);
    }
    const float out = sum / s_l[g];
    static_cast<T*>(p.o)[((size_t)bi * Hq + h0 + g) * D + dcol] = Elem<T>::from_f(out);
    if (dcol == 0 && p.lse) p.lse[(size_t)bi * Hq + h0 + g] = (s_m[g] + log2f(s_l[g])) * kLn2;
  }
  if (tid == 0) p.counters[bi * p.Hk + kh] = 0;
}

template <typename T, int D, int G>
bsa_status launch_decode(const DecodeParams& p, cudaStream_t st) {
  const size_t smem = DecodeSmem<T, D, G>::bytes(p.b, p.S);
  auto kern = decode_attn_kernel<T, D, G>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
      cudaSuccess) {
    (void)cudaGetLastError();
    return BSA_ERR_CUDA;
  }
  dim3 grid(p.S, p.Hk, p.B);
  kern<<<grid, kThreads, smem, st>>>(p);
  return BSA_OK;
}

template <typename T, int D>
bsa_status dispatch_decode(int G, const DecodeParams& p, cudaStream_t st) {
  switch (G) {
    case 1: return launch_decode<T, D, 1>(p, st);
    case 2: return launch_decode<T, D, 2>(p, st);
    case 4: return launch_decode<T, D, 4>(p, st);
    case 8: return launch_decode<T, D, 8>(p, st);
    default: return BSA_ERR_UNSUPPORTED;
  }
}

}  // namespace

// Split count and workspace layout shared by the size query and the launch.
int decode_splits(int B, int Hk, int G, int K) {
  const int want = ceil_div(4 * kSMs, B * Hk);
  return std::max(1, std::min(want, std::min(G * K + 1, kMaxList)));
}

size_t decode_workspace_bytes(int B, int Hq, int Hk, int d, int K, int S) {
  (void)K;
  size_t off = 256;                                        // status word(s)
  off += align_up((size_t)B * Hk * sizeof(int), 256);      // arrival counters
  off += (size_t)B * Hq * S * (d + 2) * sizeof(float);     // partials
  return off;
}

bsa_status decode_attn(const void* q, const void* k, const void* v, bsa_dtype dt, int B, int Hq,
                       int Hk, int n, int d, int b, const int* seq_lens, const int* idx,
                       const int* count, int K, int gate, int norm, const float* scores,
                       int scores_ld, void* o, float* lse, void* ws, size_t ws_bytes,
                       cudaStream_t st) {
  const int G = Hq / Hk;
  const int S = decode_splits(B, Hk, G, K);
  if (!ws || ws_bytes < decode_workspace_bytes(B, Hq, Hk, d, K, S)) return BSA_ERR_WORKSPACE;
  if ((size_t)b * d * (dt == BSA_BF16 ? 2 : 4) > 32768) return BSA_ERR_UNSUPPORTED;
  if (G * K + 1 > kMaxList) return BSA_ERR_UNSUPPORTED;
  DecodeParams p;
  p.q = q; p.k = k; p.v = v;
  p.B = B; p.Hq = Hq; p.Hk = Hk; p.n = n; p.b = b; p.K = K;
  p.seq_lens = seq_lens; p.idx = idx; p.count = count;
  p.gate = gate; p.norm = norm; p.scores = scores; p.scores_ld = scores_ld;
  p.o = o; p.lse = lse;
  unsigned char* w = static_cast<unsigned char*>(ws);
  p.status = reinterpret_cast<int*>(w);
  p.counters = reinterpret_cast<int*>(w + 256);
  p.part = reinterpret_cast<float*>(w + 256 + align_up((size_t)B * Hk * sizeof(int), 256));
  p.S = S;
  bsa_status rc;
  if (dt == BSA_BF16)
    rc = d == 64 ? dispatch_decode<__nv_bfloat16, 64>(G, p, st)
                 : dispatch_decode<__nv_bfloat16, 128>(G, p, st);
  else
    rc = d == 64 ? dispatch_decode<float, 64>(G, p, st) : dispatch_decode<float, 128>(G, p, st);
  if (rc != BSA_OK) return rc;
  BSA_LAUNCH_CHECK();
  return BSA_OK;
}

}  // namespace bsa

// ------------------------------------------------------------------------------------------
// Decode attention without any caller-provided or library-allocated workspace.
//
// Some callers cannot hand the library device memory: an inference engine that plans every
// device byte up front and forbids any allocation outside that plan, a plugin invoked by a host
// framework that owns the allocator and exposes none to it, or a driver loop whose latency budget
// rules out an allocator call.  For them the split-K scratch (status word, arrival counters,
// per-split partials) lives in one file-scope device array of fixed size that every GPU loading
// this library holds until the process exits.  Callers still pass inputs and outputs.
// ------------------------------------------------------------------------------------------

namespace bsa {
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(4) << 20;  // 4 MiB per device
__device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mutex;
void* g_noalloc_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device, looked up once per device.  In
// host code `g_noalloc_scratch` names a host-side stand-in, not device memory, so the address
// must come from cudaGetSymbolAddress with the device current.
bsa_status noalloc_scratch(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    (void)cudaGetLastError();
    return BSA_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) {
      (void)cudaGetLastError();
      return BSA_ERR_CUDA;
    }
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return BSA_OK;
}

}  // namespace
}  // namespace bsa

extern "C" bsa_status bsa_sparse_attn_decode_noalloc(
    const void* q, const void* k, const void* v, bsa_dtype dt, int B, int Hq, int Hk, int n,
    int d, int b, const int* seq_lens, const int* idx, const int* count, int K,
    bsa_gate_mode gate, bsa_gate_norm norm, const float* scores, int scores_ld, void* o,
    float* lse, void* stream) {
  using namespace bsa;
  BSA_REQUIRE(dtype_ok(dt), BSA_ERR_DTYPE);
  BSA_REQUIRE(q && k && v && idx && o, BSA_ERR_ARG);
  BSA_REQUIRE(B > 0 && Hq > 0 && Hk > 0 && n > 0 && d > 0 && b > 0 && K > 0, BSA_ERR_ARG);
  BSA_REQUIRE(Hq % Hk == 0, BSA_ERR_SHAPE);
  BSA_REQUIRE(group_ok(Hq, Hk), BSA_ERR_UNSUPPORTED);
  BSA_REQUIRE(head_dim_ok(d), BSA_ERR_UNSUPPORTED);
  BSA_REQUIRE(B <= 65535 && Hk <= 65535 && b <= 128, BSA_ERR_UNSUPPORTED);
  BSA_REQUIRE(all_aligned16(q, k, v, o), BSA_ERR_ARG);
  BSA_REQUIRE(gate == BSA_GATE_NONE || gate == BSA_GATE_LOG_SOFTMAX || gate == BSA_GATE_OUTER,
              BSA_ERR_ARG);
  BSA_REQUIRE(gate != BSA_GATE_OUTER, BSA_ERR_UNSUPPORTED);  // a training-mode (prefill) gate
  BSA_REQUIRE(norm == BSA_NORM_SELECTED || norm == BSA_NORM_ALL_HISTORY, BSA_ERR_ARG);
  if (gate == BSA_GATE_LOG_SOFTMAX) {
    BSA_REQUIRE(scores != nullptr, BSA_ERR_ARG);
    BSA_REQUIRE(scores_ld >= ceil_div(n, b), BSA_ERR_SHAPE);
  }
  const int S = decode_splits(B, Hk, Hq / Hk, K);
  const size_t need = decode_workspace_bytes(B, Hq, Hk, d, K, S);
  if (need > kNoAllocScratchBytes) return BSA_ERR_WORKSPACE;  // beyond the fixed scratch
  void* ws = nullptr;
  bsa_status rc = noalloc_scratch(&ws);
  if (rc != BSA_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // the array keeps the previous call's contents: zero the status word and arrival counters
  const size_t zero_bytes = 256 + align_up((size_t)B * Hk * sizeof(int), 256);
  if (cudaMemsetAsync(ws, 0, zero_bytes, st) != cudaSuccess) {
    (void)cudaGetLastError();
    return BSA_ERR_CUDA;
  }
  return decode_attn(q, k, v, dt, B, Hq, Hk, n, d, b, seq_lens, idx, count, K, gate, norm,
                     scores, scores_ld, o, lse, ws, kNoAllocScratchBytes, st);
}

extern "C" bsa_status bsa_noalloc_status(void* stream) {
  using namespace bsa;
  void* ws = nullptr;
  const bsa_status rc = noalloc_scratch(&ws);
  if (rc != BSA_OK) return rc;
  return bsa_workspace_status(ws, stream);  // the status word sits at the array's start
}
