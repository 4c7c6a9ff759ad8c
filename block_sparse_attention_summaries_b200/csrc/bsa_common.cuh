// Shared device/host helpers of libbsa (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>
#include <climits>
#include <cmath>

#include "../../include/bsa.h"

namespace bsa {

constexpr int kMaxGroup = 8;  // largest GQA group (Hq / Hk) with a kernel

// ------------------------------------------------------------------------------------------
// Host-side argument checks
// ------------------------------------------------------------------------------------------

#define BSA_REQUIRE(cond, code) \
  do {                          \
    if (!(cond)) return (code); \
  } while (0)

#define BSA_LAUNCH_CHECK()                                  \
  do {                                                      \
    if (cudaPeekAtLastError() != cudaSuccess) {             \
      (void)cudaGetLastError();                             \
      return BSA_ERR_CUDA;                                  \
    }                                                       \
  } while (0)

// Vector loads and bulk copies need 16-byte aligned tensors (a null pointer counts as aligned:
// optional arguments are checked for presence separately).
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
template <typename... Ps>
inline bool all_aligned16(const Ps*... ps) { return (aligned16(ps) && ...); }

inline bool dtype_ok(bsa_dtype dt) { return dt == BSA_F32 || dt == BSA_BF16; }
inline bool head_dim_ok(int d) { return d == 64 || d == 128; }
inline bool group_ok(int Hq, int Hk) {
  if (Hk <= 0 || Hq <= 0 || Hq % Hk) return false;
  int g = Hq / Hk;
  return g == 1 || g == 2 || g == 4 || g == 8;
}
__host__ __device__ inline int ceil_div(int a, int b) { return (a + b - 1) / b; }
__host__ __device__ inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
__host__ __device__ inline size_t max_sz(size_t a, size_t b) { return a > b ? a : b; }

// Grid sizing targets a B200 (148 SMs); sizes derive from shapes only, never from a device query,
// so workspace sizes are reproducible and host-side checks need no GPU.
constexpr int kSMs = 148;

// ------------------------------------------------------------------------------------------
// Element access
// ------------------------------------------------------------------------------------------

template <typename T>
struct Elem;

template <>
struct Elem<float> {
  static constexpr int kPer16B = 4;
  __device__ static __forceinline__ void load16(const float* p, float* out) {
    float4 x = *reinterpret_cast<const float4*>(p);
    out[0] = x.x; out[1] = x.y; out[2] = x.z; out[3] = x.w;
  }
  __device__ static __forceinline__ float to_f(float x) { return x; }
  __device__ static __forceinline__ float from_f(float x) { return x; }
};

template <>
struct Elem<__nv_bfloat16> {
  static constexpr int kPer16B = 8;
  __device__ static __forceinline__ void load16(const __nv_bfloat16* p, float* out) {
    uint4 x = *reinterpret_cast<const uint4*>(p);
    const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      out[2 * i] = __uint_as_float(w[i] << 16);
      out[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
  }
  __device__ static __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
  __device__ static __forceinline__ __nv_bfloat16 from_f(float x) { return __float2bfloat16_rn(x); }
};

// Load `N` consecutive elements (N * sizeof(T) a multiple of 8 bytes) as floats.
template <typename T, int N>
__device__ __forceinline__ void load_vec(const T* p, float* out) {
  if constexpr (sizeof(T) == 2) {
    static_assert(N % 4 == 0 || N == 2, "bf16 vector width");
    if constexpr (N == 2) {
      uint32_t w = *reinterpret_cast<const uint32_t*>(p);
      out[0] = __uint_as_float(w << 16);
      out[1] = __uint_as_float(w & 0xFFFF0000u);
    } else if constexpr (N % 8 == 0) {
#pragma unroll
      for (int i = 0; i < N / 8; ++i) {
        uint4 x = reinterpret_cast<const uint4*>(p)[i];
        const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          out[8 * i + 2 * j] = __uint_as_float(w[j] << 16);
          out[8 * i + 2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
        }
      }
    } else {
#pragma unroll
      for (int i = 0; i < N / 4; ++i) {
        uint2 x = reinterpret_cast<const uint2*>(p)[i];
        out[4 * i + 0] = __uint_as_float(x.x << 16);
        out[4 * i + 1] = __uint_as_float(x.x & 0xFFFF0000u);
        out[4 * i + 2] = __uint_as_float(x.y << 16);
        out[4 * i + 3] = __uint_as_float(x.y & 0xFFFF0000u);
      }
    }
  } else {
    static_assert(N % 2 == 0, "f32 vector width");
    if constexpr (N % 4 == 0) {
#pragma unroll
      for (int i = 0; i < N / 4; ++i) {
        float4 x = reinterpret_cast<const float4*>(p)[i];
        out[4 * i + 0] = x.x; out[4 * i + 1] = x.y; out[4 * i + 2] = x.z; out[4 * i + 3] = x.w;
      }
    } else {
#pragma unroll
      for (int i = 0; i < N / 2; ++i) {
        float2 x = reinterpret_cast<const float2*>(p)[i];
        out[2 * i + 0] = x.x; out[2 * i + 1] = x.y;
      }
    }
  }
}

// ------------------------------------------------------------------------------------------
// Warp helpers
// ------------------------------------------------------------------------------------------

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}

// Transpose-reduce: every lane holds 32 partial sums a[0..31]; afterwards a[0] of lane l is the
// warp-wide sum of entry l.  31 shuffles instead of 32 * 5.
__device__ __forceinline__ void warp_transpose_reduce32(float (&a)[32], int lane) {
#pragma unroll
  for (int w = 16; w >= 1; w >>= 1) {
    const bool upper = (lane & w) != 0;
#pragma unroll
    for (int j = 0; j < w; ++j) {
      float send = upper ? a[j] : a[j + w];
      float keep = upper ? a[j + w] : a[j];
      a[j] = keep + __shfl_xor_sync(0xffffffffu, send, w);
    }
  }
}

// ------------------------------------------------------------------------------------------
// mbarrier + bulk copy (TMA, untiled) wrappers
// ------------------------------------------------------------------------------------------

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// The dynamic shared memory advanced to its first 1024-byte boundary.  The advance is taken as an
// offset on the array itself, so every pointer derived from the result stays visibly in the
// shared state space and its accesses compile to shared-memory instructions; rounding the address
// through an integer would hide that and turn them into generic accesses, which queue in the same
// pipeline as global-memory requests.
__device__ __forceinline__ unsigned char* smem_align1024(unsigned char* raw) {
  return raw + ((1024u - (smem_u32(raw) & 1023u)) & 1023u);
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait: returns false (and the caller must bail out) after `limit` polls.  Each
// try_wait may itself suspend for a hardware time slice, so the bound is well above any
// legitimate copy latency yet ends in far under a second.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity,
                                                  uint32_t limit = (1u << 20)) {
  for (uint32_t it = 0; it < limit; ++it)
    if (mbar_try_wait(bar, parity)) return true;
  return false;
}

// Global -> shared bulk copy completing on `bar` (both addresses 16-byte aligned, bytes % 16 == 0).
__device__ __forceinline__ void bulk_g2s(void* smem_dst, const void* gmem_src, uint32_t bytes,
                                         uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(smem_dst)),
      "l"(gmem_src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// An L2 policy under which the lines a copy brings in are the first to be evicted: for data
// streamed once per launch (the K/V cache, block summaries), so that it does not push out what
// every launch reuses (the kernel's code, its small inputs).
__device__ __forceinline__ uint64_t l2_evict_first() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}
__device__ __forceinline__ void bulk_g2s_stream(void* smem_dst, const void* gmem_src,
                                                uint32_t bytes, uint64_t* bar, uint64_t pol) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1], %2, [%3], %4;" ::"r"(smem_u32(smem_dst)),
      "l"(gmem_src), "r"(bytes), "r"(smem_u32(bar)), "l"(pol)
      : "memory");
}

// Status word at the start of a workspace: set once by the first failing CTA.
__device__ __forceinline__ void report_timeout(int* status, int where) {
  if (status) atomicCAS(status, 0, where);
}

}  // namespace bsa
