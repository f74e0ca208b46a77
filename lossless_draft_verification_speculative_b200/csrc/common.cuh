// Device helpers shared by the verify kernels (sm_100a).
#pragma once

#include <cooperative_groups.h>
#include <cstdint>
#include <cuda_runtime.h>

#include "dspark_verify.h"

namespace dspark {

namespace cg = cooperative_groups;

constexpr int kMaxK = 32;
constexpr int kMaxWarps = 16;        // warps per CTA in the sampling pass
constexpr int kMaxCluster = 16;      // CTAs per cluster (non-portable size, opt-in)
constexpr int kMaxChunks = kMaxWarps * kMaxCluster;
constexpr int kLaneElems = 32;       // register-resident logits per lane per row
constexpr int kChunkElems = 32 * kLaneElems;  // contiguous tokens per warp chunk
constexpr int kFinishThreads = 256;  // finish kernel block (>= kMaxChunks)
constexpr unsigned long long kWaitLimitNs = 2000000000ull;  // bounded waits give up after 2 s

static_assert(kFinishThreads >= kMaxChunks, "finish kernel scans one chunk per thread");

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

// 2^x on the FMA pipe, for loops whose SFU is the bottleneck. x = n + f with n = rint(x)
// (the 1.5 * 2^23 shift) and |f| <= 1/2; 2^f = p(f), the degree-5 polynomial with p(0) = 1
// fitted to the relative error on [-1/2, 1/2] by gen_exp2_poly.py (max relative error of the
// whole float32 evaluation 1.7e-7, as the SFU's); 2^n is added to the exponent bits. Results
// below 2^-125 (and x = -inf) are 0, as on the flush-to-zero SFU path. Not for NaN or +inf.
__device__ __forceinline__ float exp2_poly(float x) {
  const float xc = fmaxf(x, -125.f);
  const float t = __fadd_rn(xc, 12582912.f);
  const float f = __fsub_rn(xc, __fsub_rn(t, 12582912.f));
  float p = __int_as_float(0x3aade4f2);
  p = __fmaf_rn(p, f, __int_as_float(0x3c1e7545));
  p = __fmaf_rn(p, f, __int_as_float(0x3d635b93));
  p = __fmaf_rn(p, f, __int_as_float(0x3e75fcde));
  p = __fmaf_rn(p, f, __int_as_float(0x3f317215));
  p = __fmaf_rn(p, f, 1.f);
  const float r = __int_as_float(__float_as_int(p) + (__float_as_int(t) << 23));
  return x < -125.f ? 0.f : r;
}

__device__ __forceinline__ unsigned long long globaltimer_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
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
// 2^(z*scale - m). The empty set is (m = -inf, s = 0). Merging rescales both sums to the
// larger reference. Products and sums are rounded explicitly (no FMA contraction), so the
// merge is commutative bit for bit and every lane of a butterfly ends with the same value.
struct SoftPart {
  float m;
  float s;
};

__device__ __forceinline__ SoftPart soft_empty() { return {-__int_as_float(0x7f800000), 0.f}; }

__device__ __forceinline__ SoftPart soft_merge(SoftPart a, SoftPart b) {
  if (a.s == 0.f) return b;
  if (b.s == 0.f) return a;
  const float M = fmaxf(a.m, b.m);
  const float sa = __fmul_rn(a.s, ex2(__fsub_rn(a.m, M)));
  const float sb = __fmul_rn(b.s, ex2(__fsub_rn(b.m, M)));
  return {M, __fadd_rn(sa, sb)};
}

__device__ __forceinline__ SoftPart warp_soft_merge(SoftPart a) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    SoftPart b{__shfl_xor_sync(0xffffffffu, a.m, o), __shfl_xor_sync(0xffffffffu, a.s, o)};
    a = soft_merge(a, b);
  }
  return a;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

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
// into one, identical on every lane: M = max m, S = sum s * 2^(m - M).
__device__ __forceinline__ SoftPart warp_soft_merge_lanes(float m, float s) {
  const float M = warp_max_nan(m);
  float w = s == 0.f ? 0.f : __fmul_rn(s, ex2(__fsub_rn(m, M)));
  w = warp_sum(w);
  return {M, w};
}

// ---------------------------------------------------------------- mbarrier / bulk copy

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// Shared-memory fetch-add with acquire-release ordering at CTA scope; returns the old value.
__device__ __forceinline__ unsigned smem_atomic_add_acq_rel(unsigned* p, unsigned v) {
  unsigned old;
  asm volatile("atom.acq_rel.cta.shared::cta.add.u32 %0, [%1], %2;"
               : "=r"(old)
               : "r"(smem_u32(p)), "r"(v)
               : "memory");
  return old;
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t tx) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(tx)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return done != 0;
}

// Bounded wait on an mbarrier phase: returns false if it did not complete within the limit.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = globaltimer_ns();
  for (uint32_t it = 0;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 255u) == 255u && globaltimer_ns() - t0 > kWaitLimitNs) return false;
  }
}

__device__ __forceinline__ bool mbar_try_wait_cluster(uint64_t* bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return done != 0;
}

// Bounded wait for a phase completed by other CTAs of the cluster (st.async data).
__device__ __forceinline__ bool mbar_wait_cluster_bounded(uint64_t* bar, uint32_t parity) {
  if (mbar_try_wait_cluster(bar, parity)) return true;
  const unsigned long long t0 = globaltimer_ns();
  for (uint32_t it = 0;; ++it) {
    if (mbar_try_wait_cluster(bar, parity)) return true;
    if ((it & 255u) == 255u && globaltimer_ns() - t0 > kWaitLimitNs) return false;
  }
}

// Store 16 bytes into CTA `rank`'s shared memory at the address that `local` has in this CTA,
// completing 16 transaction bytes on that CTA's mbarrier at the address `local_bar` has here.
__device__ __forceinline__ void st_async_peer(const void* local, const uint64_t* local_bar,
                                              uint32_t rank, float4 v) {
  uint32_t dst, bar;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(dst) : "r"(smem_u32(local)), "r"(rank));
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(bar) : "r"(smem_u32(local_bar)), "r"(rank));
  asm volatile(
      "st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.f32 [%0], {%1, %2, %3, %4}, [%5];" ::"r"(dst),
      "f"(v.x), "f"(v.y), "f"(v.z), "f"(v.w), "r"(bar)
      : "memory");
}

// 1-D bulk copy global -> this CTA's shared memory, completing on `bar` (no multicast).
// dst, src 16-byte aligned; bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes,
                                         uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// ---------------------------------------------------------------- programmatic launch

__device__ __forceinline__ void grid_dependency_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void grid_dependents_launch() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---------------------------------------------------------------- problem description

// Row addressing of the logit block (the pages' StepOut.logits + BlockOut.per_pos_logits).
template <typename T>
struct Rows {
  const T* p1;
  const T* pv;
  const T* q;
  int64_t ld_p1;
  int64_t ld_pv;
  int B, K, V;
  __device__ __forceinline__ const T* prow(int b, int i) const {
    return i == 0 ? p1 + static_cast<int64_t>(b) * ld_p1
                  : pv + static_cast<int64_t>(b) * ld_pv + static_cast<int64_t>(i - 1) * V;
  }
  __device__ __forceinline__ const T* qrow(int b, int i) const {
    return q + (static_cast<int64_t>(b) * K + i) * static_cast<int64_t>(V);
  }
};

// Per-chunk record of the sampling pass: the softmax reference the chunk's exponentials
// were taken against, the factor that turns them into probabilities, and the chunk's mass.
//   P rows: {ref_p, c_p, sum_v p[v], 0}
//   draft pairs: {ref_q, c_q, sum_v max(p[v] - q[v], 0), 0}
struct ChunkRec {
  float ref;
  float c;
  float mass;
  float pad;
};

}  // namespace dspark
