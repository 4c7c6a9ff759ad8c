// Row-wise sparse prefill attention and gate gradient on CUDA cores (one warp per query).
//
// [SAS] review: "Background" Eq. 2 (exact softmax restricted to the selected set), "The new
// approach" Eq. 4 / Eq. 9 (current block kept with gate 1, log-gate added to the logits of the
// selected history blocks), "Why the four design choices matter" Eq. 5 (inner-gate gradient
//     dg_m = sum_{i in B_m} (ptilde_i / g_m) do^T (v_i - o)).
//
// This is the general path: any query-unit size (per-query selection included), fp32 inputs
// (whose 1e-4 bar rules out tf32 tensor cores), and any shape the tensor-core kernel does not
// take.  Each lane holds d/32 elements of q, the running (max, sum) are warp-uniform, four tokens
// are in flight per step.  Gate gradient is computed in the stable form
//     dg_m = sum_i sum_{j in B_m} exp(z_ij - lse_i) (do_i . v_j - do_i . o_i),
// (ptilde_j / g_m = exp(z_j + log g_m - lse) / g_m = exp(z_j - lse), z without the gate).
// Outer gate (the gate outside the softmax, the ablation of "Why the four design choices
// matter"): o_i = sum_j g_m(j) p_j v_j with p the ungated softmax, so the forward scales each
// block's value contributions by g_m (the normaliser stays ungated) and
//     dg_m = sum_i sum_{j in B_m} exp(z_ij - lse_i) do_i . v_j.
#include "bsa_common.cuh"

namespace bsa {

int decode_splits(int B, int Hk, int G, int K);
size_t decode_workspace_bytes(int B, int Hq, int Hk, int d, int K, int S);
bsa_status decode_attn(const void* q, const void* k, const void* v, bsa_dtype dt, int B, int Hq,
                       int Hk, int n, int d, int b, const int* seq_lens, const int* idx,
                       const int* count, int K, int gate, int norm, const float* scores,
                       int scores_ld, void* o, float* lse, void* ws, size_t ws_bytes,
                       cudaStream_t st);
bsa_status decode_attn_given(const void* q, const void* k, const void* v, bsa_dtype dt, int B,
                             int Hq, int Hk, int n, int d, int b, const int* seq_lens,
                             const int* idx, const int* count, int K, int gate, void* o,
                             float* lse, int* status, cudaStream_t st);
bool prefill_tc_supported(bsa_dtype dt, int d, int b, int q_block, int K, int Hq, int Hk);
bsa_status gate_grad_tc(const void* q, const void* k, const void* v, const void* o,
                        const float* lse, const void* dout, int B, int Hq, int Hk, int n, int d,
                        const int* idx, const int* count, int K, int norm, const float* scores,
                        int scores_ld, float* dg, int* status, int outer, cudaStream_t st);
bsa_status prefill_tc(const void* q, const void* k, const void* v, int B, int Hq, int Hk, int n,
                      int d, int b, const int* idx, const int* count, int K, int gate, int norm,
                      const float* scores, int scores_ld, void* o, float* lse, int* status,
                      cudaStream_t st);

namespace {

constexpr int kThreads = 128;
constexpr int kWarps = kThreads / 32;
constexpr int kMaxSel = 256;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

struct RowParams {
  const void* q;
  const void* k;
  const void* v;
  const void* o_in;  // gate grad: forward output
  const float* lse_in;
  const void* dout;
  int B, Hq, Hk, n, b, q_block, U, K;
  const int* idx;
  const int* count;
  int gate, norm;
  const float* scores;
  int scores_ld;
  void* o;
  float* lse;
  float* dg;
};

// The unit's selected blocks (validated, ascending as given) and the gate normaliser.
struct UnitSel {
  int m[kMaxSel];
  int slot[kMaxSel];
  int cnt;
};

__device__ __forceinline__ int unit_candidates(int u, int q_block, int b) {
  return (int)(((long long)u * q_block) / b);
}

// Load the unit's selection into shared memory (one warp); returns the gate LSE (log2 units).
__device__ float load_unit(const RowParams& p, int bi, int h, int u, UnitSel& sel, int lane) {
  const size_t row = ((size_t)bi * p.Hq + h) * p.U + u;
  const int nc = unit_candidates(u, p.q_block, p.b);
  const int cnt = p.count ? min(p.count[row], p.K) : p.K;
  // compact valid entries preserving order
  int base = 0;
  for (int j0 = 0; j0 < cnt; j0 += 32) {
    const int j = j0 + lane;
    int m = -1;
    if (j < cnt) m = p.idx[row * p.K + j];
    const bool ok = j < cnt && m >= 0 && m < nc;
    const unsigned bal = __ballot_sync(0xffffffffu, ok);
    if (ok) {
      const int at = base + __popc(bal & ((1u << lane) - 1u));
      sel.m[at] = m;
      sel.slot[at] = j;
    }
    base += __popc(bal);
  }
  if (lane == 0) sel.cnt = base;
  __syncwarp();
  if (p.gate == BSA_GATE_NONE) return 0.f;
  const float* srow = p.scores + row * p.scores_ld;
  float mx = -INFINITY, acc = 0.f;
  if (p.norm == BSA_NORM_ALL_HISTORY) {
    for (int c = lane; c < nc; c += 32) mx = fmaxf(mx, srow[c]);
    mx = warp_max(mx);
    for (int c = lane; c < nc; c += 32) acc += exp2f((srow[c] - mx) * kLog2e);
  } else {
    for (int j = lane; j < base; j += 32) mx = fmaxf(mx, srow[sel.m[j]]);
    mx = warp_max(mx);
    for (int j = lane; j < base; j += 32) acc += exp2f((srow[sel.m[j]] - mx) * kLog2e);
  }
  acc = warp_sum(acc);
  return mx == -INFINITY ? 0.f : mx * kLog2e + log2f(acc);
}

template <typename T, int D>
__global__ void __launch_bounds__(kThreads) prefill_rowwise_kernel(const RowParams p) {
  constexpr int EPL = D / 32;
  __shared__ UnitSel sel[kWarps];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int i = blockIdx.x * kWarps + warp;  // query position
  const int h = blockIdx.y, bi = blockIdx.z;
  if (i >= p.n) return;
  const int G = p.Hq / p.Hk, kh = h / G;
  const int u = i / p.q_block;
  const int cur = i / p.b;
  UnitSel& S = sel[warp];
  const float lse_norm = load_unit(p, bi, h, u, S, lane);
  const size_t urow = ((size_t)bi * p.Hq + h) * p.U + u;
  const float* srow = p.gate != BSA_GATE_NONE ? p.scores + urow * p.scores_ld : nullptr;
  const bool outer = p.gate == BSA_GATE_OUTER;

  const T* qp = static_cast<const T*>(p.q) + (((size_t)bi * p.Hq + h) * p.n + i) * D + lane * EPL;
  const T* kb = static_cast<const T*>(p.k) + ((size_t)bi * p.Hk + kh) * p.n * D + lane * EPL;
  const T* vb = static_cast<const T*>(p.v) + ((size_t)bi * p.Hk + kh) * p.n * D + lane * EPL;
  float qv[EPL];
  load_vec<T, EPL>(qp, qv);
  const float qs = rsqrtf((float)D) * kLog2e;
#pragma unroll
  for (int e = 0; e < EPL; ++e) qv[e] *= qs;

  float m_run = -INFINITY, l_run = 0.f, acc[EPL];
#pragma unroll
  for (int e = 0; e < EPL; ++e) acc[e] = 0.f;

  // token stream: selected history blocks (with their gate: a logit bias inside the softmax, or
  // a value scale outside it), then the current block
  auto run = [&](int lo, int hi, float bias, float vscale) {
    for (int j0 = lo; j0 < hi; j0 += 4) {
      float z[4], vv[4][EPL];
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const int j = j0 + r;
        float kx[EPL];
        if (j < hi) {
          load_vec<T, EPL>(kb + (size_t)j * D, kx);
          load_vec<T, EPL>(vb + (size_t)j * D, vv[r]);
        } else {
#pragma unroll
          for (int e = 0; e < EPL; ++e) kx[e] = vv[r][e] = 0.f;
        }
        float s = 0.f;
#pragma unroll
        for (int e = 0; e < EPL; ++e) s = fmaf(qv[e], kx[e], s);
        z[r] = s;
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1)
#pragma unroll
        for (int r = 0; r < 4; ++r) z[r] += __shfl_xor_sync(0xffffffffu, z[r], o);
      float mx = m_run;
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        z[r] = (j0 + r < hi) ? z[r] + bias : -INFINITY;
        mx = fmaxf(mx, z[r]);
      }
      const float corr = m_run == -INFINITY ? 0.f : exp2f(m_run - mx);
      l_run *= corr;
#pragma unroll
      for (int e = 0; e < EPL; ++e) acc[e] *= corr;
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const float pw = z[r] == -INFINITY ? 0.f : exp2f(z[r] - mx);
        l_run += pw;
        const float pv = pw * vscale;
#pragma unroll
        for (int e = 0; e < EPL; ++e) acc[e] = fmaf(pv, vv[r][e], acc[e]);
      }
      m_run = mx;
    }
  };
  for (int j = 0; j < S.cnt; ++j) {
    const int m = S.m[j];
    const float lg = srow ? srow[m] * kLog2e - lse_norm : 0.f;  // log2 g_m
    run(m * p.b, min((m + 1) * p.b, p.n), outer ? 0.f : lg, outer ? exp2f(lg) : 1.f);
  }
  run(cur * p.b, i + 1, 0.f, 1.f);

  T* op = static_cast<T*>(p.o) + (((size_t)bi * p.Hq + h) * p.n + i) * D + lane * EPL;
  const float inv = 1.f / l_run;
#pragma unroll
  for (int e = 0; e < EPL; ++e) op[e] = Elem<T>::from_f(acc[e] * inv);
  if (p.lse && lane == 0) p.lse[((size_t)bi * p.Hq + h) * p.n + i] = (m_run + log2f(l_run)) * kLn2;
}

template <typename T, int D>
__global__ void __launch_bounds__(kThreads) gate_grad_rowwise_kernel(const RowParams p) {
  constexpr int EPL = D / 32;
  __shared__ UnitSel sel[kWarps];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int i = blockIdx.x * kWarps + warp;
  const int h = blockIdx.y, bi = blockIdx.z;
  if (i >= p.n) return;
  const int G = p.Hq / p.Hk, kh = h / G;
  const int u = i / p.q_block;
  UnitSel& S = sel[warp];
  (void)load_unit(p, bi, h, u, S, lane);
  const size_t urow = ((size_t)bi * p.Hq + h) * p.U + u;
  const size_t qrow = ((size_t)bi * p.Hq + h) * p.n + i;
  const bool outer = p.gate == BSA_GATE_OUTER;

  float qv[EPL], dov[EPL], ov[EPL];
  load_vec<T, EPL>(static_cast<const T*>(p.q) + qrow * D + lane * EPL, qv);
  load_vec<T, EPL>(static_cast<const T*>(p.dout) + qrow * D + lane * EPL, dov);
  load_vec<T, EPL>(static_cast<const T*>(p.o_in) + qrow * D + lane * EPL, ov);
  const float qs = rsqrtf((float)D) * kLog2e;
  float Di = 0.f;
#pragma unroll
  for (int e = 0; e < EPL; ++e) {
    qv[e] *= qs;
    Di = fmaf(dov[e], ov[e], Di);
  }
  Di = warp_sum(Di);
  const float lse2 = p.lse_in[qrow] * kLog2e;
  const T* kb = static_cast<const T*>(p.k) + ((size_t)bi * p.Hk + kh) * p.n * D + lane * EPL;
  const T* vb = static_cast<const T*>(p.v) + ((size_t)bi * p.Hk + kh) * p.n * D + lane * EPL;

  for (int j = 0; j < S.cnt; ++j) {
    const int m = S.m[j];
    const int lo = m * p.b, hi = min((m + 1) * p.b, p.n);
    float tot = 0.f;
    for (int t0 = lo; t0 < hi; t0 += 4) {
      float z[4], dv[4];
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        float kx[EPL], vx[EPL];
        const int t = t0 + r;
        if (t < hi) {
          load_vec<T, EPL>(kb + (size_t)t * D, kx);
          load_vec<T, EPL>(vb + (size_t)t * D, vx);
        } else {
#pragma unroll
          for (int e = 0; e < EPL; ++e) kx[e] = vx[e] = 0.f;
        }
        z[r] = 0.f;
        dv[r] = 0.f;
#pragma unroll
        for (int e = 0; e < EPL; ++e) {
          z[r] = fmaf(qv[e], kx[e], z[r]);
          dv[r] = fmaf(dov[e], vx[e], dv[r]);
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1)
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          z[r] += __shfl_xor_sync(0xffffffffu, z[r], o);
          dv[r] += __shfl_xor_sync(0xffffffffu, dv[r], o);
        }
#pragma unroll
      for (int r = 0; r < 4; ++r)
        if (t0 + r < hi) tot += exp2f(z[r] - lse2) * (outer ? dv[r] : dv[r] - Di);
    }
    if (lane == 0) atomicAdd(&p.dg[urow * p.K + S.slot[j]], tot);
  }
}

template <typename T>
bool launch_rowwise(bool grad, int d, const RowParams& p, cudaStream_t st) {
  dim3 grid(ceil_div(p.n, kWarps), p.Hq, p.B);
  if (grad) {
    if (d == 64) gate_grad_rowwise_kernel<T, 64><<<grid, kThreads, 0, st>>>(p);
    else gate_grad_rowwise_kernel<T, 128><<<grid, kThreads, 0, st>>>(p);
  } else {
    if (d == 64) prefill_rowwise_kernel<T, 64><<<grid, kThreads, 0, st>>>(p);
    else prefill_rowwise_kernel<T, 128><<<grid, kThreads, 0, st>>>(p);
  }
  return true;
}

bsa_status check_common(const void* q, const void* k, const void* v, bsa_dtype dt, int B, int Hq,
                        int Hk, int n, int d, int b, const int* idx, int K) {
  BSA_REQUIRE(dtype_ok(dt), BSA_ERR_DTYPE);
  BSA_REQUIRE(q && k && v && idx, BSA_ERR_ARG);
  BSA_REQUIRE(B > 0 && Hq > 0 && Hk > 0 && n > 0 && d > 0 && b > 0 && K > 0, BSA_ERR_ARG);
  BSA_REQUIRE(Hq % Hk == 0, BSA_ERR_SHAPE);
  BSA_REQUIRE(group_ok(Hq, Hk), BSA_ERR_UNSUPPORTED);
  BSA_REQUIRE(head_dim_ok(d), BSA_ERR_UNSUPPORTED);
  BSA_REQUIRE(B <= 65535 && Hq <= 65535, BSA_ERR_UNSUPPORTED);
  BSA_REQUIRE(K <= kMaxSel, BSA_ERR_UNSUPPORTED);
  BSA_REQUIRE(all_aligned16(q, k, v), BSA_ERR_ARG);
  return BSA_OK;
}

}  // namespace
}  // namespace bsa

extern "C" size_t bsa_sparse_attn_workspace_bytes(int B, int Hq, int Hk, int nq, int n, int d,
                                                  int b, int K) {
  using namespace bsa;
  (void)n;
  (void)b;
  if (B <= 0 || Hq <= 0 || Hk <= 0 || Hq % Hk || d <= 0 || K <= 0) return 0;
  if (nq != 1) return 256;  // status word only
  return decode_workspace_bytes(B, Hq, Hk, d, K, decode_splits(B, Hk, Hq / Hk, K));
}

extern "C" bsa_status bsa_sparse_attn_fwd(const void* q, const void* k, const void* v,
                                          bsa_dtype dt, int B, int Hq, int Hk, int nq, int n,
                                          int d, int b, const int* seq_lens, int q_block,
                                          const int* idx, const int* count, int K,
                                          bsa_gate_mode gate, bsa_gate_norm norm,
                                          const float* scores, int scores_ld, void* o,
                                          float* lse, void* workspace, size_t workspace_bytes,
                                          void* stream) {
  using namespace bsa;
  bsa_status rc = check_common(q, k, v, dt, B, Hq, Hk, n, d, b, idx, K);
  if (rc != BSA_OK) return rc;
  BSA_REQUIRE(o, BSA_ERR_ARG);
  BSA_REQUIRE(all_aligned16(o), BSA_ERR_ARG);
  BSA_REQUIRE(gate == BSA_GATE_NONE || gate == BSA_GATE_LOG_SOFTMAX || gate == BSA_GATE_OUTER,
              BSA_ERR_ARG);
  BSA_REQUIRE(norm == BSA_NORM_SELECTED || norm == BSA_NORM_ALL_HISTORY, BSA_ERR_ARG);
  if (gate != BSA_GATE_NONE) {
    BSA_REQUIRE(scores != nullptr, BSA_ERR_ARG);
    BSA_REQUIRE(scores_ld >= ceil_div(n, b), BSA_ERR_SHAPE);
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (nq == 1) {
    BSA_REQUIRE(gate != BSA_GATE_OUTER, BSA_ERR_UNSUPPORTED);  // a training-mode (prefill) gate
    BSA_REQUIRE(b <= 128, BSA_ERR_UNSUPPORTED);
    // bf16 in 64-token blocks without a gate: the cluster step of bsa_decode_step on the given
    // selection (warp MMAs over TMA tiles); its status word is the workspace's
    const int G = Hq / Hk;
    const int S = decode_splits(B, Hk, G, K);
    BSA_REQUIRE(workspace && workspace_bytes >= decode_workspace_bytes(B, Hq, Hk, d, K, S),
                BSA_ERR_WORKSPACE);
    rc = decode_attn_given(q, k, v, dt, B, Hq, Hk, n, d, b, seq_lens, idx, count, K, gate, o, lse,
                           static_cast<int*>(workspace), st);
    if (rc == BSA_OK) {
      BSA_LAUNCH_CHECK();
      return BSA_OK;
    }
    if (rc != BSA_ERR_UNSUPPORTED) return rc;
    return decode_attn(q, k, v, dt, B, Hq, Hk, n, d, b, seq_lens, idx, count, K, gate, norm,
                       scores, scores_ld, o, lse, workspace, workspace_bytes, st);
  }
  BSA_REQUIRE(nq == n, BSA_ERR_SHAPE);
  BSA_REQUIRE(seq_lens == nullptr, BSA_ERR_ARG);
  BSA_REQUIRE(q_block > 0 && q_block <= n, BSA_ERR_ARG);
  if (prefill_tc_supported(dt, d, b, q_block, K, Hq, Hk)) {
    int* status = (workspace && workspace_bytes >= 256) ? static_cast<int*>(workspace) : nullptr;
    return prefill_tc(q, k, v, B, Hq, Hk, n, d, b, idx, count, K, gate, norm, scores, scores_ld,
                      o, lse, status, st);
  }
  RowParams p{};
  p.q = q; p.k = k; p.v = v;
  p.B = B; p.Hq = Hq; p.Hk = Hk; p.n = n; p.b = b; p.q_block = q_block;
  p.U = ceil_div(n, q_block); p.K = K;
  p.idx = idx; p.count = count; p.gate = gate; p.norm = norm;
  p.scores = scores; p.scores_ld = scores_ld; p.o = o; p.lse = lse;
  if (dt == BSA_BF16) launch_rowwise<__nv_bfloat16>(false, d, p, st);
  else launch_rowwise<float>(false, d, p, st);
  BSA_LAUNCH_CHECK();
  return BSA_OK;
}

namespace bsa {
namespace {

bsa_status gate_grad_impl(const void* q, const void* k, const void* v, const void* o,
                          const float* lse, const void* dout, bsa_dtype dt, int B, int Hq, int Hk,
                          int n, int d, int b, int q_block, const int* idx, const int* count,
                          int K, bsa_gate_norm norm, const float* scores, int scores_ld,
                          float* dg, bool outer, void* stream) {
  bsa_status rc = check_common(q, k, v, dt, B, Hq, Hk, n, d, b, idx, K);
  if (rc != BSA_OK) return rc;
  BSA_REQUIRE(o && lse && dout && dg && scores, BSA_ERR_ARG);
  BSA_REQUIRE(all_aligned16(o, dout), BSA_ERR_ARG);
  BSA_REQUIRE(norm == BSA_NORM_SELECTED || norm == BSA_NORM_ALL_HISTORY, BSA_ERR_ARG);
  BSA_REQUIRE(q_block > 0 && q_block <= n, BSA_ERR_ARG);
  BSA_REQUIRE(scores_ld >= ceil_div(n, b), BSA_ERR_SHAPE);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (prefill_tc_supported(dt, d, b, q_block, K, Hq, Hk)) {
    // the gradient of the gated forward: the gate enters only through lse and o here
    return gate_grad_tc(q, k, v, o, lse, dout, B, Hq, Hk, n, d, idx, count, K, norm, scores,
                        scores_ld, dg, nullptr, outer ? 1 : 0, st);
  }
  RowParams p{};
  p.q = q; p.k = k; p.v = v; p.o_in = o; p.lse_in = lse; p.dout = dout;
  p.B = B; p.Hq = Hq; p.Hk = Hk; p.n = n; p.b = b; p.q_block = q_block;
  p.U = ceil_div(n, q_block); p.K = K;
  p.idx = idx; p.count = count; p.gate = outer ? BSA_GATE_OUTER : BSA_GATE_LOG_SOFTMAX;
  p.norm = norm; p.scores = scores; p.scores_ld = scores_ld; p.dg = dg;
  if (cudaMemsetAsync(dg, 0, (size_t)B * Hq * p.U * K * sizeof(float), st) != cudaSuccess) {
    (void)cudaGetLastError();
    return BSA_ERR_CUDA;
  }
  if (dt == BSA_BF16) launch_rowwise<__nv_bfloat16>(true, d, p, st);
  else launch_rowwise<float>(true, d, p, st);
  BSA_LAUNCH_CHECK();
  return BSA_OK;
}

}  // namespace
}  // namespace bsa

extern "C" bsa_status bsa_gate_grad(const void* q, const void* k, const void* v, const void* o,
                                    const float* lse, const void* dout, bsa_dtype dt, int B,
                                    int Hq, int Hk, int n, int d, int b, int q_block,
                                    const int* idx, const int* count, int K, bsa_gate_norm norm,
                                    const float* scores, int scores_ld, float* dg,
                                    void* stream) {
  return bsa::gate_grad_impl(q, k, v, o, lse, dout, dt, B, Hq, Hk, n, d, b, q_block, idx, count,
                             K, norm, scores, scores_ld, dg, false, stream);
}

extern "C" bsa_status bsa_gate_grad_outer(const void* q, const void* k, const void* v,
                                          const void* o, const float* lse, const void* dout,
                                          bsa_dtype dt, int B, int Hq, int Hk, int n, int d,
                                          int b, int q_block, const int* idx, const int* count,
                                          int K, bsa_gate_norm norm, const float* scores,
                                          int scores_ld, float* dg, void* stream) {
  return bsa::gate_grad_impl(q, k, v, o, lse, dout, dt, B, Hq, Hk, n, d, b, q_block, idx, count,
                             K, norm, scores, scores_ld, dg, true, stream);
}

extern "C" bsa_status bsa_workspace_status(void* workspace, void* stream) {
  if (!workspace) return BSA_ERR_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int word = 0;
  if (cudaMemcpyAsync(&word, workspace, sizeof(int), cudaMemcpyDeviceToHost, st) != cudaSuccess ||
      cudaStreamSynchronize(st) != cudaSuccess) {
    (void)cudaGetLastError();
    return BSA_ERR_CUDA;
  }
  if (word == 0) return BSA_OK;
  const int zero = 0;
  if (cudaMemcpyAsync(workspace, &zero, sizeof(int), cudaMemcpyHostToDevice, st) != cudaSuccess ||
      cudaStreamSynchronize(st) != cudaSuccess) {
    (void)cudaGetLastError();
    return BSA_ERR_CUDA;
  }
  return BSA_ERR_TIMEOUT;
}

extern "C" const char* bsa_status_string(bsa_status s) {
  switch (s) {
    case BSA_OK: return "ok";
    case BSA_ERR_ARG: return "invalid argument";
    case BSA_ERR_SHAPE: return "inconsistent shapes";
    case BSA_ERR_DTYPE: return "unknown dtype";
    case BSA_ERR_UNSUPPORTED: return "unsupported configuration";
    case BSA_ERR_CUDA: return "CUDA error";
    case BSA_ERR_TIMEOUT: return "device wait timed out";
    case BSA_ERR_WORKSPACE: return "workspace missing or too small";
  }
  return "unknown status";
}

extern "C" int bsa_version(void) { return 100; }
