// FreeSolo two-branch prefill: per-query cell selection, RoPE sliding-window branch, NoPE long
// branch over the selected cells, per-head mix.
//
// [FreeSolo] summary page, "How it works":
//  * cells of `cell` consecutive tokens keep a mean key, a centre position and a max key norm;
//  * the candidate prefix is fixed per query block of q_block queries: cells lying wholly before
//    floor(i / q_block) * q_block;
//  * cell score r_ic = q_i . kbar_c / sqrt(d) + lambda_h * a_c * erf((i - p_c) / (2 sigma_h));
//    each query keeps its top-K cells and reads their raw tokens with one softmax (NoPE);
//  * the short branch is RoPE attention over a fixed window of the `window` latest keys;
//  * the two branch outputs are combined through a per-head scalar alpha_h:
//    o = (1 - alpha_h) o_short + alpha_h o_long (o = o_short when no cell is a candidate).
//
// Kernels:
//  * select: one thread per query; the CTA's 128 queries share the candidate cells, whose
//    summaries are staged through shared memory and read as broadcasts; a register top-K list
//    ordered by (score desc, index asc) is kept per query.
//  * rope_keys: K rotated once into the workspace.  Angles pos * theta^(-2t/d) are formed and
//    reduced modulo 2 pi in fp64 (positions reach 2^16 and more, where an fp32 angle would be off
//    by ~1e-2 rad), then sin/cos are taken in fp32.
//  * rope_qk (bf16, tensor-core branch): Q and K rotated in one pass, sharing each position's
//    angles; the frequencies theta^(-2t/d) come from a table formed once on the host in fp64, the
//    angle is reduced in fp64 as above and its sine and cosine are the fast fp32 ones on
//    [-pi, pi] (absolute error ~1e-6, far below the bf16 rounding of the result).
//  * attn: one warp per query, lane l holding elements {l, l+32, ...} so that every rotate-half
//    pair (t, t + d/2) sits in one lane; online softmax over the window, then over the selected
//    cells, then the mix.
#include <cmath>

#include "bsa_common.cuh"

namespace bsa {

bsa_status window_attn_tc(const void* q, const void* k, const void* v, int B, int H, int Hk,
                          int n, int d, int window, void* o, int* status, cudaStream_t st);
size_t long_attn_tc_workspace(int B, int H, int n);
bool long_attn_tc_supported(int d, int cell, int ksel);
bsa_status long_attn_tc(const void* q, const void* k, const void* v, int B, int H, int n, int d,
                        int cell, const int* sel, const int* sel_cnt, int ksel,
                        const float* alpha, void* o, void* ws, size_t ws_bytes, int* status,
                        cudaStream_t st);
bool long_cells_supported(int d, int cell, int K, long long rows);
size_t long_cells_workspace(int B, int H, int n, int d, int cell, int K);
bsa_status long_cells(const void* q, const void* k, const void* v, int B, int H, int n, int d,
                      int cell, const int* idx, const int* count, int K, const float* alpha,
                      void* o, void* ws, size_t ws_bytes, int* status, cudaStream_t st);
size_t freesolo_select_tc_workspace(int B, int H, int n, int d, int cell);
bool freesolo_select_tc_supported(bsa_dtype dt, int d, int q_block, int K);
bsa_status freesolo_select_tc(const void* q, int B, int H, int n, int d, int cell,
                              const float* mean_k, const float* max_norm, const float* centre,
                              const float* lam, const float* sig, int K, int* idx, int* count,
                              void* ws, size_t ws_bytes, cudaStream_t st);

namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr int kSelThreads = 128;
constexpr int kSelChunk = 64;  // summary rows staged per pass
constexpr int kMaxK = 8;

__device__ __forceinline__ uint32_t order_key(float f) {
  if (f != f) return 0u;
  if (f == 0.f) f = 0.f;
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

template <typename T, int D>
__global__ void __launch_bounds__(kSelThreads)
    freesolo_select_kernel(const T* __restrict__ q, int H, int n, int cell, int q_block, int C,
                           const float* __restrict__ mean_k, const float* __restrict__ max_norm,
                           const float* __restrict__ centre, const float* __restrict__ lam,
                           const float* __restrict__ sig, int K, int* __restrict__ idx,
                           int* __restrict__ count) {
  __shared__ __align__(16) float s_k[kSelChunk][D];
  __shared__ float s_a[kSelChunk], s_p[kSelChunk];
  const int h = blockIdx.y, bi = blockIdx.z;
  const int i0 = blockIdx.x * kSelThreads;
  const int i = i0 + threadIdx.x;
  const bool live = i < n;
  const int ii = live ? i : n - 1;
  const int nc = ((ii / q_block) * q_block) / cell;
  const int last = min(n, i0 + kSelThreads) - 1;
  const int nc_max = ((last / q_block) * q_block) / cell;

  float qv[D];
  {
    const float sc = rsqrtf((float)D);
    const T* qp = q + (((size_t)bi * H + h) * n + ii) * D;
#pragma unroll
    for (int e = 0; e < D; e += 8) {
      float t[8];
      load_vec<T, 8>(qp + e, t);
#pragma unroll
      for (int j = 0; j < 8; ++j) qv[e + j] = t[j] * sc;
    }
  }
  const float lam_h = lam[h];
  const float inv2sig = 0.5f / sig[h];
  const float fi = (float)ii;
  uint64_t best[kMaxK];
#pragma unroll
  for (int j = 0; j < kMaxK; ++j) best[j] = 0ull;  // empty slot ranks below everything

  const size_t srow0 = ((size_t)bi * H + h) * C;
  for (int c0 = 0; c0 < nc_max; c0 += kSelChunk) {
    const int rows = min(kSelChunk, nc_max - c0);
    __syncthreads();
    for (int e = threadIdx.x; e < rows * (D / 4); e += kSelThreads) {
      const int r = e / (D / 4), c4 = e % (D / 4);
      reinterpret_cast<float4*>(s_k[r])[c4] =
          reinterpret_cast<const float4*>(mean_k + (srow0 + c0 + r) * D)[c4];
    }
    for (int r = threadIdx.x; r < rows; r += kSelThreads) {
      s_a[r] = max_norm[srow0 + c0 + r];
      s_p[r] = centre[srow0 + c0 + r];
    }
    __syncthreads();
    const int my_rows = min(rows, nc - c0);
    for (int r = 0; r < my_rows; ++r) {
      float dot = 0.f;
#pragma unroll
      for (int e = 0; e < D; e += 4) {
        const float4 kk = reinterpret_cast<const float4*>(s_k[r])[e / 4];
        dot = fmaf(qv[e], kk.x, dot);
        dot = fmaf(qv[e + 1], kk.y, dot);
        dot = fmaf(qv[e + 2], kk.z, dot);
        dot = fmaf(qv[e + 3], kk.w, dot);
      }
      const float rsc = dot + lam_h * s_a[r] * erff((fi - s_p[r]) * inv2sig);
      const uint32_t c = (uint32_t)(c0 + r);
      const uint64_t comp = ((uint64_t)order_key(rsc) << 32) | (uint64_t)(0xFFFFFFFFu - c);
      if (comp > best[kMaxK - 1]) {
        uint64_t x = comp;
#pragma unroll
        for (int j = 0; j < kMaxK; ++j) {  // insertion into the descending list
          if (j < K && x > best[j]) {
            const uint64_t t = best[j];
            best[j] = x;
            x = t;
          }
        }
      }
    }
  }
  if (!live) return;
  const int kk = min(K, nc);
  int sel[kMaxK];
#pragma unroll
  for (int j = 0; j < kMaxK; ++j)
    sel[j] = j < kk ? (int)(0xFFFFFFFFu - (uint32_t)(best[j] & 0xFFFFFFFFu)) : INT_MAX;
  // ascending block order
#pragma unroll
  for (int a = 0; a < kMaxK; ++a)
#pragma unroll
    for (int b2 = 0; b2 + 1 < kMaxK - a; ++b2)
      if (sel[b2] > sel[b2 + 1]) {
        const int t = sel[b2];
        sel[b2] = sel[b2 + 1];
        sel[b2 + 1] = t;
      }
  int* out = idx + (((size_t)bi * H + h) * n + i) * K;
  for (int j = 0; j < K; ++j) {
    int vj = -1;
#pragma unroll
    for (int jj = 0; jj < kMaxK; ++jj)
      if (jj == j && jj < kk) vj = sel[jj];
    out[j] = vj;
  }
  if (count) count[((size_t)bi * H + h) * n + i] = kk;
}

// Rotate every key at its absolute position (rotate-half pairing, base theta).
template <typename T, int D>
__global__ void rope_keys_kernel(const T* __restrict__ k, T* __restrict__ kr, long long rows,
                                 int n, double log_theta) {
  const long long pair = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (pair >= rows * (D / 2)) return;
  const long long row = pair / (D / 2);
  const int t = (int)(pair % (D / 2));
  const int pos = (int)(row % n);
  const double inv_freq = exp(-2.0 * t / D * log_theta);
  double ang = (double)pos * inv_freq;
  ang -= 6.283185307179586 * rint(ang / 6.283185307179586);
  float s, c;
  sincosf((float)ang, &s, &c);
  const T* src = k + row * D;
  const float a = Elem<T>::to_f(src[t]);
  const float b = Elem<T>::to_f(src[t + D / 2]);
  T* dst = kr + row * D;
  dst[t] = Elem<T>::from_f(a * c - b * s);
  dst[t + D / 2] = Elem<T>::from_f(b * c + a * s);
}

// Rotation of q and k for the tensor-core branch: a thread per (row, group of four pairs t),
// 8-byte loads and stores of both halves.
template <int D>
struct InvFreq {
  double f[D / 2];
};

template <int D>
__global__ void __launch_bounds__(256)
    rope_qk_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
                   __nv_bfloat16* __restrict__ qr, __nv_bfloat16* __restrict__ kr, long long rows,
                   int n, const InvFreq<D> inv) {
  constexpr int G = D / 8;  // groups of four pairs per row
  const long long gid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (gid >= rows * G) return;
  const long long row = gid / G;
  const int t0 = (int)(gid % G) * 4;
  const double pos = (double)(row % n);
  float c[4], s[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    double ang = pos * inv.f[t0 + e];
    ang = fma(-6.283185307179586, rint(ang * 0.15915494309189535), ang);
    __sincosf((float)ang, &s[e], &c[e]);
  }
  auto rotate = [&](const __nv_bfloat16* src, __nv_bfloat16* dst) {
    const uint2 lo = *reinterpret_cast<const uint2*>(src + row * D + t0);
    const uint2 hi = *reinterpret_cast<const uint2*>(src + row * D + t0 + D / 2);
    const __nv_bfloat162* a = reinterpret_cast<const __nv_bfloat162*>(&lo);
    const __nv_bfloat162* b = reinterpret_cast<const __nv_bfloat162*>(&hi);
    uint2 olo, ohi;
    __nv_bfloat162* x = reinterpret_cast<__nv_bfloat162*>(&olo);
    __nv_bfloat162* y = reinterpret_cast<__nv_bfloat162*>(&ohi);
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const float2 fa = __bfloat1622float2(a[e]), fb = __bfloat1622float2(b[e]);
      const int u = 2 * e, w = 2 * e + 1;
      x[e] = __floats2bfloat162_rn(fa.x * c[u] - fb.x * s[u], fa.y * c[w] - fb.y * s[w]);
      y[e] = __floats2bfloat162_rn(fb.x * c[u] + fa.x * s[u], fb.y * c[w] + fa.y * s[w]);
    }
    *reinterpret_cast<uint2*>(dst + row * D + t0) = olo;
    *reinterpret_cast<uint2*>(dst + row * D + t0 + D / 2) = ohi;
  };
  rotate(q, qr);
  rotate(k, kr);
}

template <int D>
void launch_rope_qk(const void* q, const void* k, void* qr, void* kr, long long rows, int n,
                    double log_theta, cudaStream_t st) {
  InvFreq<D> inv;
  for (int t = 0; t < D / 2; ++t) inv.f[t] = std::exp(-2.0 * t / D * log_theta);
  const long long threads = rows * (D / 8);
  rope_qk_kernel<D><<<(unsigned)((threads + 255) / 256), 256, 0, st>>>(
      static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k),
      static_cast<__nv_bfloat16*>(qr), static_cast<__nv_bfloat16*>(kr), rows, n, inv);
}

struct FsParams {
  const void* q;
  const void* k;
  const void* v;
  const void* k_rot;
  int short_in_o;  // 1: o already holds the short branch (tensor-core window kernel)
  int H, n, cell, window, K;
  double log_theta;
  const float* alpha;
  const int* idx;
  const int* count;
  void* o;
};

template <typename T, int D>
__global__ void __launch_bounds__(128) freesolo_attn_kernel(const FsParams p) {
  constexpr int E = D / 32;  // elements per lane: l, l+32, ...
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int i = blockIdx.x * 4 + warp;
  const int h = blockIdx.y, bi = blockIdx.z;
  if (i >= p.n) return;
  const size_t hrow = ((size_t)bi * p.H + h) * p.n;
  const T* qp = static_cast<const T*>(p.q) + (hrow + i) * D;
  const T* kb = static_cast<const T*>(p.k) + hrow * D;
  const T* krb = static_cast<const T*>(p.k_rot) + hrow * D;
  const T* vb = static_cast<const T*>(p.v) + hrow * D;
  const float sc = rsqrtf((float)D) * kLog2e;

  float qraw[E], qrot[E];
#pragma unroll
  for (int e = 0; e < E; ++e) qraw[e] = Elem<T>::to_f(qp[lane + 32 * e]);
  // rotate q at position i: pairs (t, t + D/2) live in this lane as (e, e + E/2)
  // (not needed when the short branch already ran on the tensor cores)
#pragma unroll
  for (int e = 0; e < (p.short_in_o ? 0 : E / 2); ++e) {
    const int t = lane + 32 * e;
    const double inv_freq = exp(-2.0 * t / D * p.log_theta);
    double ang = (double)i * inv_freq;
    ang -= 6.283185307179586 * rint(ang / 6.283185307179586);
    float s, c;
    sincosf((float)ang, &s, &c);
    const float a = qraw[e], b = qraw[e + E / 2];
    qrot[e] = a * c - b * s;
    qrot[e + E / 2] = b * c + a * s;
  }
#pragma unroll
  for (int e = 0; e < E; ++e) {
    qrot[e] *= sc;
    qraw[e] *= sc;
  }

  // online softmax over tokens [lo, hi) of key base kk with query qq
  auto attend = [&](const T* kk, const float* qq, int lo, int hi, const int* cells, int ncells,
                    float& m_run, float& l_run, float* acc) {
    m_run = -INFINITY;
    l_run = 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) acc[e] = 0.f;
    const int total = cells ? ncells * p.cell : hi - lo;
    for (int t0 = 0; t0 < total; t0 += 4) {
      float z[4], vv[4][E];
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const int t = t0 + r;
        float s = 0.f;
        if (t < total) {
          const int j = cells ? cells[t / p.cell] * p.cell + t % p.cell : lo + t;
#pragma unroll
          for (int e = 0; e < E; ++e) {
            s = fmaf(qq[e], Elem<T>::to_f(kk[(size_t)j * D + lane + 32 * e]), s);
            vv[r][e] = Elem<T>::to_f(vb[(size_t)j * D + lane + 32 * e]);
          }
        } else {
#pragma unroll
          for (int e = 0; e < E; ++e) vv[r][e] = 0.f;
        }
        z[r] = s;
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1)
#pragma unroll
        for (int r = 0; r < 4; ++r) z[r] += __shfl_xor_sync(0xffffffffu, z[r], o);
      float mx = m_run;
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        if (t0 + r >= total) z[r] = -INFINITY;
        mx = fmaxf(mx, z[r]);
      }
      const float corr = m_run == -INFINITY ? 0.f : exp2f(m_run - mx);
      l_run *= corr;
#pragma unroll
      for (int e = 0; e < E; ++e) acc[e] *= corr;
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const float pw = z[r] == -INFINITY ? 0.f : exp2f(z[r] - mx);
        l_run += pw;
#pragma unroll
        for (int e = 0; e < E; ++e) acc[e] = fmaf(pw, vv[r][e], acc[e]);
      }
      m_run = mx;
    }
  };

  float out[E];
  if (p.short_in_o) {
    const T* orow = static_cast<const T*>(p.o) + (hrow + i) * D;
#pragma unroll
    for (int e = 0; e < E; ++e) out[e] = Elem<T>::to_f(orow[lane + 32 * e]);
  } else {
    float ms, ls, os[E];
    attend(krb, qrot, max(0, i - p.window + 1), i + 1, nullptr, 0, ms, ls, os);
#pragma unroll
    for (int e = 0; e < E; ++e) out[e] = os[e] / ls;
  }

  const size_t qrow = hrow + i;
  const int cnt = min(p.count ? p.count[qrow] : p.K, p.K);
  int cells[kMaxK];
  int nsel = 0;
  for (int j = 0; j < cnt; ++j) {
    const int c = p.idx[qrow * p.K + j];
    // only cells wholly at or before the query are read (no future token, no out-of-range row)
    if (c >= 0 && (c + 1) * p.cell <= i + 1 && nsel < kMaxK) cells[nsel++] = c;
  }
  if (nsel == 0 && p.short_in_o) return;  // o already final
  if (nsel > 0) {
    float ml, ll, ol[E];
    attend(kb, qraw, 0, 0, cells, nsel, ml, ll, ol);
    const float a = p.alpha[h];
#pragma unroll
    for (int e = 0; e < E; ++e) out[e] = (1.f - a) * out[e] + a * (ol[e] / ll);
  }
  T* op = static_cast<T*>(p.o) + qrow * D;
#pragma unroll
  for (int e = 0; e < E; ++e) op[lane + 32 * e] = Elem<T>::from_f(out[e]);
}

template <typename T, int D>
void launch_select(dim3 grid, cudaStream_t st, const void* q, int H, int n, int cell, int qb,
                   int C, const float* mk, const float* mx, const float* ce, const float* lam,
                   const float* sig, int K, int* idx, int* count) {
  freesolo_select_kernel<T, D><<<grid, kSelThreads, 0, st>>>(
      static_cast<const T*>(q), H, n, cell, qb, C, mk, mx, ce, lam, sig, K, idx, count);
}

template <typename T, int D>
void launch_attn(const FsParams& p, int B, cudaStream_t st, void* k_rot) {
  const long long rows = (long long)B * p.H * p.n;
  const long long pairs = rows * (D / 2);
  rope_keys_kernel<T, D><<<(unsigned)((pairs + 255) / 256), 256, 0, st>>>(
      static_cast<const T*>(p.k), static_cast<T*>(k_rot), rows, p.n, p.log_theta);
  dim3 grid(ceil_div(p.n, 4), p.H, B);
  freesolo_attn_kernel<T, D><<<grid, 128, 0, st>>>(p);
}

}  // namespace
}  // namespace bsa

extern "C" bsa_status bsa_freesolo_select(const void* q, bsa_dtype dt, int B, int H, int n, int d,
                                          int cell, int q_block, const float* mean_k,
                                          const float* max_norm, const float* centre,
                                          const float* lambda_h, const float* sigma_h, int K,
                                          int* idx, int* count, void* workspace,
                                          size_t workspace_bytes, void* stream) {
  using namespace bsa;
  BSA_REQUIRE(dtype_ok(dt), BSA_ERR_DTYPE);
  BSA_REQUIRE(q && mean_k && max_norm && centre && lambda_h && sigma_h && idx, BSA_ERR_ARG);
  BSA_REQUIRE(B > 0 && H > 0 && n > 0 && d > 0 && cell > 0 && q_block > 0 && K > 0, BSA_ERR_ARG);
  BSA_REQUIRE(head_dim_ok(d), BSA_ERR_UNSUPPORTED);
  BSA_REQUIRE(K <= kMaxK, BSA_ERR_UNSUPPORTED);
  BSA_REQUIRE(B <= 65535 && H <= 65535, BSA_ERR_UNSUPPORTED);
  BSA_REQUIRE(all_aligned16(q, mean_k), BSA_ERR_ARG);
  const int C = ceil_div(n, cell);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (freesolo_select_tc_supported(dt, d, q_block, K))
    return freesolo_select_tc(q, B, H, n, d, cell, mean_k, max_norm, centre, lambda_h, sigma_h, K,
                              idx, count, workspace, workspace_bytes, st);
  dim3 grid(ceil_div(n, kSelThreads), H, B);
  if (dt == BSA_BF16) {
    if (d == 64) launch_select<__nv_bfloat16, 64>(grid, st, q, H, n, cell, q_block, C, mean_k, max_norm, centre, lambda_h, sigma_h, K, idx, count);
    else launch_select<__nv_bfloat16, 128>(grid, st, q, H, n, cell, q_block, C, mean_k, max_norm, centre, lambda_h, sigma_h, K, idx, count);
  } else {
    if (d == 64) launch_select<float, 64>(grid, st, q, H, n, cell, q_block, C, mean_k, max_norm, centre, lambda_h, sigma_h, K, idx, count);
    else launch_select<float, 128>(grid, st, q, H, n, cell, q_block, C, mean_k, max_norm, centre, lambda_h, sigma_h, K, idx, count);
  }
  BSA_LAUNCH_CHECK();
  return BSA_OK;
}

extern "C" size_t bsa_freesolo_select_workspace_bytes(bsa_dtype dt, int B, int H, int n, int d,
                                                       int cell, int q_block, int K) {
  using namespace bsa;
  if (B <= 0 || H <= 0 || n <= 0 || d <= 0 || cell <= 0) return 0;
  return freesolo_select_tc_supported(dt, d, q_block, K)
             ? freesolo_select_tc_workspace(B, H, n, d, cell)
             : 0;
}

extern "C" size_t bsa_freesolo_workspace_bytes(bsa_dtype dt, int B, int H, int n, int d,
                                                int cell, int K) {
  using namespace bsa;
  if (B <= 0 || H <= 0 || n <= 0 || d <= 0 || cell <= 0 || K <= 0) return 0;
  // status word, rotated keys; bf16 adds the rotated queries of the tensor-core window branch and
  // the long branch's scratch: cell-major pair lists and partial outputs, or per-unit block unions
  const size_t rows = (size_t)B * H * n;
  if (dt != BSA_BF16) return 256 + rows * d * 4;
  const size_t lw = long_cells_supported(d, cell, K, (long long)rows)
                        ? long_cells_workspace(B, H, n, d, cell, K)
                        : long_attn_tc_workspace(B, H, n);
  return 256 + 2 * rows * d * 2 + lw;
}

extern "C" bsa_status bsa_freesolo_attn(const void* q, const void* k, const void* v, bsa_dtype dt,
                                        int B, int H, int n, int d, int cell, int window,
                                        float rope_theta, const float* alpha_h, const int* idx,
                                        const int* count, int K, void* o, void* workspace,
                                        size_t workspace_bytes, void* stream) {
  using namespace bsa;
  BSA_REQUIRE(dtype_ok(dt), BSA_ERR_DTYPE);
  BSA_REQUIRE(q && k && v && alpha_h && idx && o, BSA_ERR_ARG);
  BSA_REQUIRE(B > 0 && H > 0 && n > 0 && d > 0 && cell > 0 && window > 0 && K > 0 &&
                  rope_theta > 1.f,
              BSA_ERR_ARG);
  BSA_REQUIRE(head_dim_ok(d), BSA_ERR_UNSUPPORTED);
  BSA_REQUIRE(K <= kMaxK, BSA_ERR_UNSUPPORTED);
  BSA_REQUIRE(B <= 65535 && H <= 65535, BSA_ERR_UNSUPPORTED);
  BSA_REQUIRE(all_aligned16(q, k, v, o, workspace), BSA_ERR_ARG);
  if (!workspace || workspace_bytes < bsa_freesolo_workspace_bytes(dt, B, H, n, d, cell, K))
    return BSA_ERR_WORKSPACE;
  FsParams p;
  p.q = q; p.k = k; p.v = v;
  p.k_rot = static_cast<unsigned char*>(workspace) + 256;
  p.short_in_o = 0;
  p.H = H; p.n = n; p.cell = cell; p.window = window; p.K = K;
  p.log_theta = log((double)rope_theta);
  p.alpha = alpha_h; p.idx = idx; p.count = count; p.o = o;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  void* kr = const_cast<void*>(p.k_rot);
  if (dt == BSA_BF16) {
    // short branch on the tensor cores: rotate q and k once, sliding-window tiles over them
    const long long rows = (long long)B * H * n;
    void* qr = static_cast<unsigned char*>(workspace) + 256 + (size_t)rows * d * 2;
    if (d == 64) launch_rope_qk<64>(q, k, qr, kr, rows, n, p.log_theta, st);
    else launch_rope_qk<128>(q, k, qr, kr, rows, n, p.log_theta, st);
    BSA_LAUNCH_CHECK();
    int* status = static_cast<int*>(workspace);
    bsa_status rc = window_attn_tc(qr, kr, v, B, H, H, n, d, window, o, status, st);
    unsigned char* lws = static_cast<unsigned char*>(qr) + (size_t)rows * d * 2;
    const size_t used = (size_t)(lws - static_cast<unsigned char*>(workspace));
    if (rc == BSA_OK && long_cells_supported(d, cell, K, rows)) {
      // long branch on the tensor cores, regrouped by cell: only the selected pairs are computed
      return long_cells(q, k, v, B, H, n, d, cell, idx, count, K, alpha_h, o, lws,
                        workspace_bytes - used, status, st);
    }
    if (rc == BSA_OK && long_attn_tc_supported(d, cell, K)) {
      // long branch on the tensor cores over each unit's union of selected blocks
      return long_attn_tc(q, k, v, B, H, n, d, cell, idx, count, K, alpha_h, o, lws,
                          workspace_bytes - used, status, st);
    }
    if (rc == BSA_OK) {
      p.short_in_o = 1;
      dim3 grid(ceil_div(n, 4), H, B);
      if (d == 64) freesolo_attn_kernel<__nv_bfloat16, 64><<<grid, 128, 0, st>>>(p);
      else freesolo_attn_kernel<__nv_bfloat16, 128><<<grid, 128, 0, st>>>(p);
      BSA_LAUNCH_CHECK();
      return BSA_OK;
    }
    if (rc != BSA_ERR_UNSUPPORTED) return rc;
  }
  if (dt == BSA_BF16) {
    if (d == 64) launch_attn<__nv_bfloat16, 64>(p, B, st, kr);
    else launch_attn<__nv_bfloat16, 128>(p, B, st, kr);
  } else {
    if (d == 64) launch_attn<float, 64>(p, B, st, kr);
    else launch_attn<float, 128>(p, B, st, kr);
  }
  BSA_LAUNCH_CHECK();
  return BSA_OK;
}
