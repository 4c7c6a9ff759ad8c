// FS-B: two forests of cell summaries per head, searched by a beam, re-ranked by log-sum-exp.
//
// [FreeSolo] "How it differs", FS-B: no cell is discarded; per head one forest holds the whole
// prefix and one the cells of norm at or above the median; every node stores a mean key, a
// radius, a maximum norm and a minimum position; a beam of W_b nodes per level descends each
// forest by the node score U_v, an upper bound of the cell scores below v; the cells reached are
// re-ranked by log-sum-exp over their token keys and the top K are read.
//
// Reading of the tree shape (the page gives the node contents, not the construction): a forest
// over m cells in position order is the row of perfect binary trees given by the set bits of m,
// largest first.  Every node of such a forest is a dyadic range [j 2^h, (j + 1) 2^h) of the
// forest's cell list lying inside [0, m), so the nodes of level h are j < floor(m / 2^h) and the
// root of height h (if bit h of m is set) is j = 2 floor(m / 2^(h+1)).  Node summaries: mean key =
// mean of the leaves' mean keys (the mean of its two children's), radius = the largest distance
// of a leaf mean key from it, maximum norm and minimum position over the leaves.  Node score:
//     U_v = (q . mu_v + ||q|| rho_v) / sqrt(d) + lambda a_max erf((i - p_min) / (2 sigma)),
// which bounds q . kbar_c / sqrt(d) + lambda a_c erf((i - p_c) / (2 sigma)) for every leaf c
// (Cauchy-Schwarz; erf increasing; lambda >= 0) and equals it at a leaf.
//
// B200 layout.  The forests of a (batch, head) row are level-major pyramids in one caller buffer
// (fixed offsets from C, so one buffer serves any prefix length): per forest and node the mean key
// (d floats) and (rho, a_max, p_min); plus the second forest's cell list.  Build: the top-K kernel
// picks the upper half of the norms (the second forest's cells, ascending); one CTA per (row,
// forest) fills level 0 and halves level by level; one thread per (row, forest, leaf) measures its
// distance to every ancestor and raises the ancestor's radius (warp-reduced, then an atomic max
// on the float's bits, valid for non-negative floats).  Search: one CTA per row; warp f walks
// forest f level by level (the beam's children and the level's root, at most 2 W_b + 1 nodes, one
// per lane pair, ranked exactly by (U as float32, lower first cell)), then all warps re-rank the
// union of the two final beams by log-sum-exp over each cell's token keys and keep the top K.
#include "bsa_common.cuh"

namespace bsa {

void launch_topk_rows(const float* scores, int rows, int C, int ld, const int* n_cand, int units,
                      int q_block, int b, int K, int* idx, int* count, int out_ld,
                      int keep_newest, cudaStream_t st);

namespace {

constexpr int kFsbMaxBeam = 16;
constexpr int kFsbMaxK = 8;
constexpr int kFsbThreads = 256;
constexpr int kFsbMaxC = 16384;

__host__ __device__ inline int fsb_levels(int C) {  // levels of a pyramid over up to C cells
  int L = 1;
  while ((1 << L) <= C) ++L;
  return L;
}
__host__ __device__ inline long long fsb_level_offset(int C, int h) {  // first node of level h
  long long off = 0;
  for (int g = 0; g < h; ++g) off += C >> g;
  return off;
}
__host__ __device__ inline long long fsb_nodes(int C) { return fsb_level_offset(C, fsb_levels(C)); }

// Byte layout of the forest buffer of `rows` rows (per row: forest 0 then forest 1).
struct FsbLayout {
  long long nodes;  // nodes per forest
  size_t mu, meta, list, count, total;
  __host__ __device__ FsbLayout(int rows, int C, int d) {
    nodes = fsb_nodes(C);
    mu = 0;                                                            // [rows][2][nodes][d]
    meta = align_up(mu + (size_t)rows * 2 * nodes * d * 4, 256);       // [rows][2][nodes][4]
    list = align_up(meta + (size_t)rows * 2 * nodes * 4 * 4, 256);     // [rows][C] (forest 1)
    count = align_up(list + (size_t)rows * C * 4, 256);                // [rows][2]
    total = align_up(count + (size_t)rows * 2 * 4, 256);
  }
};

struct FsbBuild {
  const float* mean_k;
  const float* max_norm;
  const float* centre;
  const int* n_cells;
  int rows, C;
  float* mu;
  float* meta;  // rho, a_max, p_min, (unused)
  int* list;
  int* count;
};

__device__ __forceinline__ int fsb_cell(const FsbBuild& p, int row, int f, int j) {
  return f == 0 ? j : p.list[(size_t)row * p.C + j];
}

// Level 0 and the mean keys / maxima of every level: one CTA per (row, forest).
template <int D>
__global__ void __launch_bounds__(kFsbThreads) fsb_build_levels_kernel(const FsbBuild p) {
  const int row = blockIdx.x, f = blockIdx.y;
  const int nc = min(max(p.n_cells[row], 0), p.C);
  const int m = f == 0 ? nc : (nc + 1) / 2;
  const long long nodes = fsb_nodes(p.C);
  float* mu = p.mu + ((size_t)row * 2 + f) * nodes * D;
  float* meta = p.meta + ((size_t)row * 2 + f) * nodes * 4;
  if (threadIdx.x == 0) p.count[row * 2 + f] = m;
  const float* mk = p.mean_k + (size_t)row * p.C * D;
  for (int e = threadIdx.x; e < m * (D / 4); e += kFsbThreads) {
    const int j = e / (D / 4), c4 = e % (D / 4);
    const int c = fsb_cell(p, row, f, j);
    reinterpret_cast<float4*>(mu + (size_t)j * D)[c4] =
        reinterpret_cast<const float4*>(mk + (size_t)c * D)[c4];
    if (c4 == 0) {
      meta[(size_t)j * 4 + 0] = 0.f;
      meta[(size_t)j * 4 + 1] = p.max_norm[(size_t)row * p.C + c];
      meta[(size_t)j * 4 + 2] = p.centre[(size_t)row * p.C + c];
      meta[(size_t)j * 4 + 3] = 0.f;
    }
  }
  __syncthreads();
  const int L = fsb_levels(p.C);
  for (int h = 1; h < L && (m >> h) > 0; ++h) {
    const long long o0 = fsb_level_offset(p.C, h - 1), o1 = fsb_level_offset(p.C, h);
    const int nh = m >> h;
    for (int e = threadIdx.x; e < nh * (D / 4); e += kFsbThreads) {
      const int j = e / (D / 4), c4 = e % (D / 4);
      const float4 a = reinterpret_cast<const float4*>(mu + (o0 + 2 * j) * D)[c4];
      const float4 b = reinterpret_cast<const float4*>(mu + (o0 + 2 * j + 1) * D)[c4];
      reinterpret_cast<float4*>(mu + (o1 + j) * D)[c4] =
          make_float4(0.5f * (a.x + b.x), 0.5f * (a.y + b.y), 0.5f * (a.z + b.z), 0.5f * (a.w + b.w));
      if (c4 == 0) {
        meta[(o1 + j) * 4 + 0] = 0.f;  // radius: raised by the leaves afterwards
        meta[(o1 + j) * 4 + 1] = fmaxf(meta[(o0 + 2 * j) * 4 + 1], meta[(o0 + 2 * j + 1) * 4 + 1]);
        meta[(o1 + j) * 4 + 2] = fminf(meta[(o0 + 2 * j) * 4 + 2], meta[(o0 + 2 * j + 1) * 4 + 2]);
        meta[(o1 + j) * 4 + 3] = 0.f;
      }
    }
    __syncthreads();
  }
}

// Radii: thread per (row, forest, leaf j); the leaves of a warp are 32 consecutive positions, so
// at height h >= 5 they share one ancestor and below it groups of 2^h lanes do.
template <int D>
__global__ void __launch_bounds__(kFsbThreads) fsb_build_radius_kernel(const FsbBuild p) {
  const int row = blockIdx.y, f = blockIdx.z;
  const int j = blockIdx.x * kFsbThreads + threadIdx.x;
  const int lane = threadIdx.x & 31;
  const int nc = min(max(p.n_cells[row], 0), p.C);
  const int m = f == 0 ? nc : (nc + 1) / 2;
  if (blockIdx.x * kFsbThreads >= m) return;  // whole CTA past the leaves (uniform)
  const long long nodes = fsb_nodes(p.C);
  const float* mu = p.mu + ((size_t)row * 2 + f) * nodes * D;
  float* meta = p.meta + ((size_t)row * 2 + f) * nodes * 4;
  const bool leaf = j < m;
  const float* kc = mu + (size_t)(leaf ? j : 0) * D;  // level 0 holds the leaves' mean keys
  const int L = fsb_levels(p.C);
  for (int h = 1; h < L; ++h) {
    const int node = j >> h;
    const bool has = leaf && node < (m >> h);
    if (!__any_sync(0xffffffffu, has)) break;  // no lane has an ancestor this high
    float dist = 0.f;
    if (has) {
      const float* a = mu + (fsb_level_offset(p.C, h) + node) * D;
      float acc = 0.f;
#pragma unroll 8
      for (int c4 = 0; c4 < D / 4; ++c4) {
        const float4 x = reinterpret_cast<const float4*>(kc)[c4];
        const float4 y = reinterpret_cast<const float4*>(a)[c4];
        const float dx = x.x - y.x, dy = x.y - y.y, dz = x.z - y.z, dw = x.w - y.w;
        acc = fmaf(dx, dx, fmaf(dy, dy, fmaf(dz, dz, fmaf(dw, dw, acc))));
      }
      dist = sqrtf(acc);
    }
    // max over the lanes sharing the ancestor: groups of min(2^h, 32) consecutive lanes
    const int span = h >= 5 ? 32 : (1 << h);
    for (int o = 1; o < span; o <<= 1) dist = fmaxf(dist, __shfl_xor_sync(0xffffffffu, dist, o));
    if (has && (lane & (span - 1)) == 0)
      atomicMax(reinterpret_cast<int*>(meta + (fsb_level_offset(p.C, h) + node) * 4), __float_as_int(dist));
  }
}

// ---- search -------------------------------------------------------------------------------

struct FsbSearch {
  const void* q;
  const void* k;
  int B, H, n, cell, C;
  const int* pos;
  const float* mu;
  const float* meta;
  const int* list;
  const int* count;
  const float* lam;
  const float* sig;
  int width, K;
  int* idx;
  int* nsel;
  float* lse;  // optional [B, H, K] re-rank scores of the selected cells
};

__device__ __forceinline__ uint32_t fsb_key(float f) {
  if (f != f) return 0u;
  if (f == 0.f) f = 0.f;
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

template <typename T, int D>
__global__ void __launch_bounds__(kFsbThreads) fsb_search_kernel(const FsbSearch p) {
  constexpr int NW = kFsbThreads / 32;
  __shared__ __align__(16) float s_q[D];
  __shared__ float s_qn;
  __shared__ int s_beam[2][kFsbMaxBeam];   // node index within its level (final: cell index)
  __shared__ int s_nbeam[2];
  __shared__ int s_cand[2 * kFsbMaxBeam];
  __shared__ float s_rr[2 * kFsbMaxBeam];
  __shared__ int s_ncand;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int h_idx = blockIdx.x, bi = blockIdx.y;
  const int row = bi * p.H + h_idx;
  const int i = min(max(p.pos[bi], 0), p.n - 1);
  const T* qp = static_cast<const T*>(p.q) + (size_t)row * D;
  for (int e = tid; e < D; e += kFsbThreads) s_q[e] = Elem<T>::to_f(qp[e]);
  __syncthreads();
  if (warp == 0) {
    float ss = 0.f;
    for (int e = lane; e < D; e += 32) ss = fmaf(s_q[e], s_q[e], ss);
    ss = warp_sum(ss);
    if (lane == 0) s_qn = sqrtf(ss);
  }
  __syncthreads();
  const float scale = rsqrtf((float)D);
  const float lm = p.lam ? p.lam[h_idx] : 0.f;
  const float inv2s = p.lam ? 0.5f / p.sig[h_idx] : 0.f;
  const long long nodes = fsb_nodes(p.C);
  const int L = fsb_levels(p.C);

  if (warp < 2) {  // warp f walks forest f
    const int f = warp;
    const int m = p.count[row * 2 + f];
    const float* mu = p.mu + ((size_t)row * 2 + f) * nodes * D;
    const float* meta = p.meta + ((size_t)row * 2 + f) * nodes * 4;
    int nb = 0;  // beam size; beam nodes in s_beam[f]
    int top = -1;
    for (int h = L - 1; h >= 0; --h)
      if ((m >> h) & 1) { top = h; break; }
    for (int h = top; h >= 0; --h) {
      // pool: children of the beam (2 nb), then this level's root if bit h of m is set
      const int npool = 2 * nb + (((m >> h) & 1) ? 1 : 0);
      uint64_t key[2];
      int node[2];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int e = lane + 32 * u;
        key[u] = 0ull;
        node[u] = -1;
        if (e < npool) {
          const int j = e < 2 * nb ? 2 * s_beam[f][e >> 1] + (e & 1) : ((m >> (h + 1)) << 1);
          const float* a = mu + (fsb_level_offset(p.C, h) + j) * D;
          const float* mt = meta + (fsb_level_offset(p.C, h) + j) * 4;
          float acc0 = 0.f, acc1 = 0.f;
#pragma unroll 8
          for (int c4 = 0; c4 < D / 4; ++c4) {
            const float4 x = reinterpret_cast<const float4*>(a)[c4];
            const float4 y = reinterpret_cast<const float4*>(s_q)[c4];
            acc0 = fmaf(x.x, y.x, fmaf(x.y, y.y, acc0));
            acc1 = fmaf(x.z, y.z, fmaf(x.w, y.w, acc1));
          }
          float U = fmaf(s_qn, mt[0], acc0 + acc1) * scale;
          if (p.lam) U += lm * mt[1] * erff(((float)i - mt[2]) * inv2s);
          // rank key: U (order-preserving) high, then the lower first cell first
          const int first = f == 0 ? (j << h) : p.list[(size_t)row * p.C + (j << h)];
          key[u] = ((uint64_t)fsb_key(U) << 32) | (uint64_t)(0xFFFFFFFFu - (uint32_t)first);
          node[u] = j;
        }
      }
      // exact rank among the pool (distinct keys: the first cells differ)
      int rk[2] = {0, 0};
      const unsigned long long k0 = key[0], k1 = key[1];
      for (int src = 0; src < min(npool, 32); ++src) {
        const unsigned long long ks = __shfl_sync(0xffffffffu, k0, src);
        rk[0] += ks > k0 ? 1 : 0;
        rk[1] += ks > k1 ? 1 : 0;
      }
      for (int src = 32; src < npool; ++src) {  // warp-uniform bound: the pool's 33rd entry
        const unsigned long long ks = __shfl_sync(0xffffffffu, k1, src - 32);
        rk[0] += ks > k0 ? 1 : 0;
        rk[1] += ks > k1 ? 1 : 0;
      }
      const int keep = min(p.width, npool);
      __syncwarp();
#pragma unroll
      for (int u = 0; u < 2; ++u)
        if (node[u] >= 0 && rk[u] < keep) s_beam[f][rk[u]] = node[u];
      nb = keep;
      __syncwarp();
    }
    // the leaf beam: cells
    if (lane < nb) s_beam[f][lane] = f == 0 ? s_beam[f][lane] : p.list[(size_t)row * p.C + s_beam[f][lane]];
    if (lane == 0) s_nbeam[f] = nb;
  }
  __syncthreads();
  // union of the two leaf beams (ascending, duplicates once)
  if (tid == 0) {
    int a = 0, b = 0, u = 0;
    const int na = s_nbeam[0], nbb = s_nbeam[1];
    int A[kFsbMaxBeam], Bv[kFsbMaxBeam];
    for (int x = 0; x < na; ++x) A[x] = s_beam[0][x];
    for (int x = 0; x < nbb; ++x) Bv[x] = s_beam[1][x];
    // sort both (at most 16 each; insertion)
    for (int x = 1; x < na; ++x) { int v = A[x], y = x - 1; while (y >= 0 && A[y] > v) { A[y + 1] = A[y]; --y; } A[y + 1] = v; }
    for (int x = 1; x < nbb; ++x) { int v = Bv[x], y = x - 1; while (y >= 0 && Bv[y] > v) { Bv[y + 1] = Bv[y]; --y; } Bv[y + 1] = v; }
    while (a < na || b < nbb) {
      int v;
      if (b >= nbb || (a < na && A[a] < Bv[b])) v = A[a++];
      else if (a >= na || Bv[b] < A[a]) v = Bv[b++];
      else { v = A[a++]; ++b; }
      s_cand[u++] = v;
    }
    s_ncand = u;
  }
  __syncthreads();
  // re-rank: log-sum-exp of q . k_j / sqrt(d) over each candidate cell's tokens (warp per cell)
  const int ncand = s_ncand;
  const T* kb = static_cast<const T*>(p.k) + (size_t)row * p.n * D;
  for (int x = warp; x < ncand; x += NW) {
    const int c = s_cand[x];
    const int lo = c * p.cell, hi = min(p.n, lo + p.cell);
    float mx = -INFINITY, sum = 0.f;
    for (int t0 = lo; t0 < hi; t0 += 32) {
      const int t = t0 + lane;
      float z = -INFINITY;
      if (t < hi) {
        float acc = 0.f;
        const T* kr = kb + (size_t)t * D;
#pragma unroll
        for (int e0 = 0; e0 < D; e0 += Elem<T>::kPer16B) {
          float xv[Elem<T>::kPer16B];
          Elem<T>::load16(kr + e0, xv);
#pragma unroll
          for (int u = 0; u < Elem<T>::kPer16B; ++u) acc = fmaf(xv[u], s_q[e0 + u], acc);
        }
        z = acc * scale;
      }
      const float m2 = fmaxf(mx, warp_max(z));
      const float add = warp_sum(z == -INFINITY ? 0.f : expf(z - m2));
      sum = (mx == -INFINITY ? 0.f : sum * expf(mx - m2)) + add;
      mx = m2;
    }
    if (lane == 0) s_rr[x] = mx + logf(sum);
  }
  __syncthreads();
  if (warp == 0) {  // top K of the re-rank scores (ties: lower cell, NaN last)
    const int kk = min(p.K, ncand);
    const uint32_t mk = lane < ncand ? fsb_key(s_rr[lane]) : 0u;
    int rk = 0;
    for (int x = 0; x < ncand; ++x) {
      const uint32_t kx = fsb_key(s_rr[x]);
      rk += (kx > mk || (kx == mk && x < lane)) ? 1 : 0;
    }
    const bool take = lane < ncand && rk < kk;
    const unsigned tb = __ballot_sync(0xffffffffu, take);
    const int at = __popc(tb & ((1u << lane) - 1u));
    if (take) {
      p.idx[(size_t)row * p.K + at] = s_cand[lane];
      if (p.lse) p.lse[(size_t)row * p.K + at] = s_rr[lane];
    }
    for (int x = kk + lane; x < p.K; x += 32) {
      p.idx[(size_t)row * p.K + x] = -1;
      if (p.lse) p.lse[(size_t)row * p.K + x] = -INFINITY;
    }
    if (lane == 0 && p.nsel) p.nsel[row] = kk;
  }
}

}  // namespace
}  // namespace bsa

extern "C" size_t bsa_fsb_forest_bytes(int B, int H, int C, int d) {
  using namespace bsa;
  if (B <= 0 || H <= 0 || C <= 0 || C > kFsbMaxC || !head_dim_ok(d)) return 0;
  return FsbLayout(B * H, C, d).total;
}

extern "C" bsa_status bsa_fsb_build(const float* mean_k, const float* max_norm,
                                    const float* centre, int B, int H, int C, int d,
                                    const int* n_cells, void* forest, size_t forest_bytes,
                                    void* stream) {
  using namespace bsa;
  BSA_REQUIRE(mean_k && max_norm && centre && n_cells && forest, BSA_ERR_ARG);
  BSA_REQUIRE(B > 0 && H > 0 && C > 0 && d > 0, BSA_ERR_ARG);
  BSA_REQUIRE(head_dim_ok(d) && C <= kFsbMaxC, BSA_ERR_UNSUPPORTED);
  BSA_REQUIRE(B <= 65535 && H <= 65535, BSA_ERR_UNSUPPORTED);
  BSA_REQUIRE(all_aligned16(mean_k, forest), BSA_ERR_ARG);
  const int rows = B * H;
  const FsbLayout lay(rows, C, d);
  BSA_REQUIRE(forest_bytes >= lay.total, BSA_ERR_WORKSPACE);
  unsigned char* w = static_cast<unsigned char*>(forest);
  FsbBuild p;
  p.mean_k = mean_k; p.max_norm = max_norm; p.centre = centre; p.n_cells = n_cells;
  p.rows = rows; p.C = C;
  p.mu = reinterpret_cast<float*>(w + lay.mu);
  p.meta = reinterpret_cast<float*>(w + lay.meta);
  p.list = reinterpret_cast<int*>(w + lay.list);
  p.count = reinterpret_cast<int*>(w + lay.count);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // the second forest's cells: the upper half of the norms, ascending
  launch_topk_rows(max_norm, rows, C, C, n_cells, 0, 0, 0, -1, p.list, nullptr, C, 0, st);
  dim3 g1(rows, 2);
  dim3 g2((C + kFsbThreads - 1) / kFsbThreads, rows, 2);
  if (d == 64) {
    fsb_build_levels_kernel<64><<<g1, kFsbThreads, 0, st>>>(p);
    fsb_build_radius_kernel<64><<<g2, kFsbThreads, 0, st>>>(p);
  } else {
    fsb_build_levels_kernel<128><<<g1, kFsbThreads, 0, st>>>(p);
    fsb_build_radius_kernel<128><<<g2, kFsbThreads, 0, st>>>(p);
  }
  BSA_LAUNCH_CHECK();
  return BSA_OK;
}

extern "C" bsa_status bsa_fsb_select(const void* q, const void* k, bsa_dtype dt, int B, int H,
                                     int n, int d, const int* pos, int cell, const void* forest,
                                     size_t forest_bytes, const float* lambda_h,
                                     const float* sigma_h, int width, int K, int* idx,
                                     int* count, float* lse, void* stream) {
  using namespace bsa;
  BSA_REQUIRE(dtype_ok(dt), BSA_ERR_DTYPE);
  BSA_REQUIRE(q && k && pos && forest && idx, BSA_ERR_ARG);
  BSA_REQUIRE((lambda_h == nullptr) == (sigma_h == nullptr), BSA_ERR_ARG);
  BSA_REQUIRE(B > 0 && H > 0 && n > 0 && d > 0 && cell > 0 && width > 0 && K > 0, BSA_ERR_ARG);
  BSA_REQUIRE(head_dim_ok(d) && width <= kFsbMaxBeam && K <= kFsbMaxK, BSA_ERR_UNSUPPORTED);
  BSA_REQUIRE(B <= 65535 && H <= 65535, BSA_ERR_UNSUPPORTED);
  BSA_REQUIRE(all_aligned16(q, k, forest), BSA_ERR_ARG);
  const int C = ceil_div(n, cell);
  BSA_REQUIRE(C <= kFsbMaxC, BSA_ERR_UNSUPPORTED);
  const FsbLayout lay(B * H, C, d);
  BSA_REQUIRE(forest_bytes >= lay.total, BSA_ERR_WORKSPACE);
  const unsigned char* w = static_cast<const unsigned char*>(forest);
  FsbSearch p;
  p.q = q; p.k = k; p.B = B; p.H = H; p.n = n; p.cell = cell; p.C = C; p.pos = pos;
  p.mu = reinterpret_cast<const float*>(w + lay.mu);
  p.meta = reinterpret_cast<const float*>(w + lay.meta);
  p.list = reinterpret_cast<const int*>(w + lay.list);
  p.count = reinterpret_cast<const int*>(w + lay.count);
  p.lam = lambda_h; p.sig = sigma_h; p.width = width; p.K = K;
  p.idx = idx; p.nsel = count; p.lse = lse;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  dim3 grid(H, B);
  if (dt == BSA_BF16) {
    if (d == 64) fsb_search_kernel<__nv_bfloat16, 64><<<grid, kFsbThreads, 0, st>>>(p);
    else fsb_search_kernel<__nv_bfloat16, 128><<<grid, kFsbThreads, 0, st>>>(p);
  } else {
    if (d == 64) fsb_search_kernel<float, 64><<<grid, kFsbThreads, 0, st>>>(p);
    else fsb_search_kernel<float, 128><<<grid, kFsbThreads, 0, st>>>(p);
  }
  BSA_LAUNCH_CHECK();
  return BSA_OK;
}
