// lod_common.cuh -- shared device helpers of the LoD attention kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "lod.h"

namespace lod {

constexpr int kChunk = 256;  // tokens per indexed chunk ("How It Works", paragraph 1)
constexpr int kPage = 16;    // keys per page (same paragraph)
constexpr int kMaxClusters = 16;
constexpr int kMaxTopGroups = 16;
constexpr int kMaxTopPages = 4;

// Workspace header: the device status word and padding to 256 bytes.
constexpr size_t kWsHeader = 256;

// ---------------------------------------------------------------- element I/O

template <typename T>
struct Elem;

template <>
struct Elem<float> {
  __device__ __forceinline__ static float to_f(float x) { return x; }
  __device__ __forceinline__ static float from_f(float x) { return x; }
};

template <>
struct Elem<__nv_bfloat16> {
  __device__ __forceinline__ static float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
  __device__ __forceinline__ static __nv_bfloat16 from_f(float x) { return __float2bfloat16_rn(x); }
};

// Load N consecutive elements (N * sizeof(T) in {4, 8, 16} bytes, naturally
// aligned) as floats, through the read-only path.
template <typename T, int N>
__device__ __forceinline__ void load_f(const T* __restrict__ p, float (&v)[N]) {
  if constexpr (sizeof(T) == 4) {
    if constexpr (N == 4) {
      float4 a = __ldg(reinterpret_cast<const float4*>(p));
      v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    } else if constexpr (N == 2) {
      float2 a = __ldg(reinterpret_cast<const float2*>(p));
      v[0] = a.x; v[1] = a.y;
    } else {
#pragma unroll
      for (int i = 0; i < N; ++i) v[i] = __ldg(reinterpret_cast<const float*>(p) + i);
    }
  } else {
    static_assert(N % 2 == 0, "bf16 loads come in pairs");
    if constexpr (N == 8) {
      uint4 a = __ldg(reinterpret_cast<const uint4*>(p));
      uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        v[2 * i] = __uint_as_float(w[i] << 16);
        v[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
      }
    } else if constexpr (N == 4) {
      uint2 a = __ldg(reinterpret_cast<const uint2*>(p));
      v[0] = __uint_as_float(a.x << 16);
      v[1] = __uint_as_float(a.x & 0xffff0000u);
      v[2] = __uint_as_float(a.y << 16);
      v[3] = __uint_as_float(a.y & 0xffff0000u);
    } else {
      static_assert(N == 2, "unsupported bf16 vector width");
      uint32_t a = __ldg(reinterpret_cast<const unsigned int*>(p));
      v[0] = __uint_as_float(a << 16);
      v[1] = __uint_as_float(a & 0xffff0000u);
    }
  }
}

// ---------------------------------------------------------------- warp helpers

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Candidate order used by every top-k of the method: larger score first,
// then lower id (the tie rule of the rankings).
__device__ __forceinline__ bool cand_better(float s, int id, float s2, int id2) {
  return s > s2 || (s == s2 && id < id2);
}

// Warp-wide argmax of (score, -id): every lane receives the winner.
__device__ __forceinline__ void warp_best(float& s, int& id) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    float s2 = __shfl_xor_sync(0xffffffffu, s, o);
    int i2 = __shfl_xor_sync(0xffffffffu, id, o);
    if (cand_better(s2, i2, s, id)) {
      s = s2;
      id = i2;
    }
  }
}

__device__ __forceinline__ void set_status(uint32_t* status, uint32_t bits) {
  if (status) atomicOr(status, bits);
}

// ---------------------------------------------------------------- sm_100 PTX helpers

// Packed fp32 FMA on a pair (one instruction, two independent FMAs).
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
  unsigned long long d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;"
      : "=l"(d)
      : "l"(*reinterpret_cast<unsigned long long*>(&a)), "l"(*reinterpret_cast<unsigned long long*>(&b)),
        "l"(*reinterpret_cast<unsigned long long*>(&c)));
  return *reinterpret_cast<float2*>(&d);
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

// Arrive once and announce `bytes` of asynchronous copies for the current phase.
__device__ __forceinline__ void mbar_arrive_expect(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

// Plain arrive (release, CTA scope) on `bar`.
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// Four-byte asynchronous copy global -> shared; `valid` false writes a zero
// (nothing is read from `src`).
__device__ __forceinline__ void cp_async4_zfill(void* dst, const void* src, bool valid) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(smem_u32(dst)), "l"(src),
               "r"(valid ? 4u : 0u)
               : "memory");
}
// Sixteen-byte asynchronous copy global -> shared (both 16-byte aligned),
// bypassing L1; `valid` false writes zeros (nothing is read from `src`).
__device__ __forceinline__ void cp_async16_zfill(void* dst, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src),
               "r"(valid ? 16u : 0u)
               : "memory");
}
// One arrival on `bar` once every cp.async this thread issued before has
// landed (the arrival counts toward the barrier's expected count).
__device__ __forceinline__ void cp_async_mbar_arrive_noinc(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// Named barrier over `nthreads` threads (whole warps) that also returns
// whether `pred` held on any of them.
__device__ __forceinline__ bool bar_red_or(int id, int nthreads, bool pred) {
  uint32_t r;
  asm volatile(
      "{ .reg .pred q, p; setp.ne.u32 q, %1, 0; bar.red.or.pred p, %2, %3, q; selp.u32 %0, 1, 0, p; }"
      : "=r"(r)
      : "r"((uint32_t)pred), "r"(id), "r"(nthreads)
      : "memory");
  return r != 0;
}
__device__ __forceinline__ void bar_named_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}
__device__ __forceinline__ uint32_t lanemask_lt() {
  uint32_t m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

// 2^x on the special-function unit (approximate, flushes denormals; 2^-inf = 0).
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Two floats rounded (RNE) to bf16 and packed, `lo` in the low half.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// Bring the 128-byte line holding `p` into L2 (no register result, no wait).
__device__ __forceinline__ void prefetch_l2(const void* p) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

// One-dimensional TMA bulk copy global -> shared (both 16-byte aligned, bytes % 16 == 0),
// completing on `bar`.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cta.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// bulk_g2s with an L2 cache policy (see createpolicy).
__device__ __forceinline__ void bulk_g2s_hint(void* dst, const void* src, uint32_t bytes, uint64_t* bar,
                                              uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cta.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::
          "r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

// L2 policy for data read once: its lines are evicted first.
__device__ __forceinline__ uint64_t l2_policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// 16-byte read-only load with an L2 cache policy.
__device__ __forceinline__ uint4 ldg_hint(const void* p, uint64_t policy) {
  uint4 v;
  asm volatile("ld.global.nc.L2::cache_hint.v4.u32 {%0, %1, %2, %3}, [%4], %5;"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p), "l"(policy));
  return v;
}

// Bounded wait for phase `parity` of `bar`.  Returns false (and records
// LOD_ST_TIMEOUT) if the phase has not completed after about two billion
// cycles (about a second); it never suspends the thread for longer than the
// hardware's default try_wait interval.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, uint32_t* status) {
  const uint32_t b = smem_u32(bar);
  uint32_t done;
  asm volatile(
      "{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2; selp.u32 %0, 1, 0, p; }"
      : "=r"(done)
      : "r"(b), "r"(parity)
      : "memory");
  if (done) return true;
  const long long t0 = clock64();
  while (true) {
    asm volatile(
        "{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2; selp.u32 %0, 1, 0, p; }"
        : "=r"(done)
        : "r"(b), "r"(parity)
        : "memory");
    if (done) return true;
    if (clock64() - t0 > (2ll << 30)) break;
  }
  set_status(status, LOD_ST_TIMEOUT);
  return false;
}

// Programmatic dependent launch: let the next kernel in the stream start its
// prologue, and (in that kernel) wait for this grid's memory to be visible.
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// SplitMix64 generator output for state x (Steele, Lea, Flood, OOPSLA 2014).
__device__ __forceinline__ uint64_t splitmix64(uint64_t x) {
  uint64_t z = x + 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

// Orderable 64-bit key of group `id` with score s: a larger key is a better
// group (higher score, then smaller id; the same order as comparing the
// floats); 0 = no group (score -inf).
__device__ __forceinline__ uint64_t group_key(float s, int64_t id) {
  if (s == -INFINITY) return 0;
  uint32_t b = s == 0.f ? 0u : __float_as_uint(s);  // -0 orders as +0
  b ^= (b & 0x80000000u) ? 0xffffffffu : 0x80000000u;
  return ((uint64_t)b << 32) | (uint32_t)(0xffffffffu - (uint32_t)id);
}
// Orderable 32-bit key of a score (larger = better; -0 as +0); 0 = -inf.
__device__ __forceinline__ uint32_t okey32(float s) {
  if (s == -INFINITY) return 0u;
  const uint32_t b = s == 0.f ? 0u : __float_as_uint(s);
  return b ^ ((b & 0x80000000u) ? 0xffffffffu : 0x80000000u);
}
__device__ __forceinline__ float key_score(uint64_t k) {
  uint32_t b = (uint32_t)(k >> 32);
  b = (b & 0x80000000u) ? (b ^ 0x80000000u) : ~b;
  return __uint_as_float(b);
}
__device__ __forceinline__ int key_id(uint64_t k) { return (int)(0xffffffffu - (uint32_t)k); }

}  // namespace lod
