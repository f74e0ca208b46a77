// Device helpers shared by the verify kernels (sm_100a).
#pragma once

#include <cooperative_groups.h>
#include <cstdint>
#include <cuda_runtime.h>

#include "dspark_verify.h"

namespace dspark {

namespace cg = cooperative_groups;

constexpr int kMaxK = 32;  // drafts per sequence (one warp lane per draft in the decisions)

// Logit storage types. bf16 logits are carried as raw 16-bit patterns.
struct bf16_t {
  uint16_t bits;
};

template <typename T>
struct Elem;
template <>
struct Elem<bf16_t> {
  static constexpr int kBytes = 2;
  static constexpr int kPerVec16 = 8;
  __device__ __forceinline__ static float load1(const bf16_t* p) {
    uint16_t h = __ldg(reinterpret_cast<const unsigned short*>(p));
    return __uint_as_float(static_cast<uint32_t>(h) << 16);
  }
  // 8 bf16 in a 16-byte word -> 8 floats, in element order.
  __device__ __forceinline__ static void unpack(const uint4& v, float* f) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      f[2 * k] = __uint_as_float(w[k] << 16);
      f[2 * k + 1] = __uint_as_float(w[k] & 0xffff0000u);
    }
  }
};
template <>
struct Elem<float> {
  static constexpr int kBytes = 4;
  static constexpr int kPerVec16 = 4;
  __device__ __forceinline__ static float load1(const float* p) { return __ldg(p); }
  __device__ __forceinline__ static void unpack(const uint4& v, float* f) {
    f[0] = __uint_as_float(v.x);
    f[1] = __uint_as_float(v.y);
    f[2] = __uint_as_float(v.z);
    f[3] = __uint_as_float(v.w);
  }
};

// 2^x on the SFU (PTX ex2.approx.ftz.f32). ex2(-inf) = 0, ex2(NaN) = NaN.
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Streaming 16-byte global load that does not allocate in L1.
__device__ __forceinline__ uint4 ld_stream16(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// A softmax partial over a set of logits: m = reference (scaled max), s = sum of
// 2^(z*scale - m). The empty set is (m = -inf, s = 0).
struct SoftPart {
  float m;
  float s;
};

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = __fadd_rn(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

__device__ __forceinline__ bool is_finite(float x) { return fabsf(x) <= 3.402823466e38f; }

// ---------------------------------------------------------------- packed / warp arithmetic

// Two floats in one 64-bit register pair, for the sm_100 f32x2 FMA-pipe instructions. Each
// lane of a packed op rounds exactly like the scalar op (round to nearest, no flush).
__device__ __forceinline__ uint64_t pk2(float a, float b) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ void upk2(uint64_t v, float& a, float& b) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t sub2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t mul2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

// max of three with NaN propagation (a NaN anywhere gives NaN).
__device__ __forceinline__ float max3_nan(float a, float b, float c) {
  float d;
  asm("max.NaN.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
__device__ __forceinline__ float max_nan(float a, float b) {
  float d;
  asm("max.NaN.f32 %0, %1, %2;" : "=f"(d) : "f"(a), "f"(b));
  return d;
}
// Elementwise max of two bf16 pairs, NaN-propagating.
__device__ __forceinline__ uint32_t max_nan_bf16x2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.NaN.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
// Warp-wide max (every lane gets it), NaN-propagating.
__device__ __forceinline__ float warp_max_nan(float v) {
  float d;
  asm volatile("redux.sync.max.NaN.f32 %0, %1, 0xffffffff;" : "=f"(d) : "f"(v));
  return d;
}

// Merge 32 lane-held softmax parts (m = reference, s = sum against it; empty = (-inf, 0))
// into one, identical on every lane: M = max m, S = sum s * 2^(m - M). Products and sums are
// rounded explicitly (no FMA contraction) and the butterfly is symmetric, so every lane ends
// with the same bits.
__device__ __forceinline__ SoftPart warp_soft_merge_lanes(float m, float s) {
  const float M = warp_max_nan(m);
  float w = s == 0.f ? 0.f : __fmul_rn(s, ex2(__fsub_rn(m, M)));
  w = warp_sum(w);
  return {M, w};
}

// ---------------------------------------------------------------- programmatic launch

__device__ __forceinline__ void grid_dependency_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void grid_dependents_launch() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

}  // namespace dspark
