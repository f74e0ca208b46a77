// Pass 1 of the verify step: every logit row of the block is read from HBM exactly once.
//
// The work is split into units (row, chunk): chunk c of a row is its tokens
// [2048c, min(V, 2048(c+1))). Units are numbered sequence-major (sequence b: P rows 0..K,
// then for the sampling policy Q rows 0..K-1; within a row, chunks in order), and each warp
// of one full wave takes an equal contiguous run of them. A warp streams a unit with 16-byte
// loads, several in flight per lane, keeps per-lane running statistics, merges its lanes and
// writes one record for the unit. A record is a function of the unit's logits alone (not of
// the launch geometry), so identical rows give identical statistics. No warp waits for
// another: all warps of the wave finish together and the kernel is a plain stream.
//
// Records. Sampling: (ref, sum) with ref = max_v z[v] * scale and sum = sum_v 2^(z[v]*scale
// - ref), the online-softmax pair (Milakov & Gimelshein 2018) in base 2; (-inf, 0) for a
// chunk with no value above -inf; a NaN or +inf anywhere makes the pair non-finite. Greedy:
// (max, lowest token index of the max) on the raw logits (order is unchanged by 1/T > 0).
#pragma once

#include <climits>

#include "common.cuh"

namespace dspark {

constexpr int kThreads = 256;            // both kernels
constexpr int kWarps = kThreads / 32;
constexpr int kStreamCtasPerSm = 4;      // 4 x 256 threads x 64 registers fill the SM
constexpr int kBatchVecs = 8;            // loads each lane keeps in flight
constexpr int kCE = 2048;                // tokens per chunk (pass-1 unit, pass-2 chunk)
constexpr int kMaxChunkCount = 128;      // chunks per row (V <= 262144)

// The logit rows of one call. Row i of sequence b: P rows i = 0..K (p_1 .. p_{K+1}), then Q
// rows i = K+1 .. 2K (q_1 .. q_K) when the call samples.
struct RowSet {
  const void* p1;
  const void* pv;
  const void* q;
  int64_t ld_p1;
  int64_t ld_pv;
  int K;
  int V;
  int rows;  // K + 1 (greedy) or 2K + 1 (sampling)
};

template <typename T>
__device__ __forceinline__ const T* row_ptr(const RowSet& rs, int b, int i) {
  if (i == 0) return static_cast<const T*>(rs.p1) + static_cast<int64_t>(b) * rs.ld_p1;
  if (i <= rs.K)
    return static_cast<const T*>(rs.pv) + static_cast<int64_t>(b) * rs.ld_pv +
           static_cast<int64_t>(i - 1) * rs.V;
  return static_cast<const T*>(rs.q) +
         (static_cast<int64_t>(b) * rs.K + (i - rs.K - 1)) * rs.V;
}

struct StreamParams {
  RowSet rs;
  long long n_units;  // B * rows * nch
  long long upw;      // units per warp
  int nch;            // chunks per row
  float scale;        // log2(e) / T (sampling)
  float2* rec;        // [n_units]: record of unit u at u
};

// ------------------------------------------------------------------------ batch loads

// Lane `lane`'s share of one batch: vectors base + lane + 32k, k < kBatchVecs, of a row whose
// vectors end at nv1. Vectors at or past nv1 read as -inf.
template <typename T>
__device__ __forceinline__ void load_batch(const T* row, long long base, long long nv1, int lane,
                                           uint4* v) {
  constexpr int VEC = Elem<T>::kPerVec16;
  const uint32_t ninf = Elem<T>::kBytes == 2 ? 0xff80ff80u : 0xff800000u;
#pragma unroll
  for (int k = 0; k < kBatchVecs; ++k) {
    const long long vi = base + lane + 32 * k;
    v[k] = vi < nv1 ? ld_stream16(row + vi * VEC) : make_uint4(ninf, ninf, ninf, ninf);
  }
}

template <typename T>
__device__ __forceinline__ void load_batch_scalar(const T* row, long long base, long long n1,
                                                  int lane, float* z) {
#pragma unroll
  for (int k = 0; k < kBatchVecs; ++k) {
    const long long e = base + lane + 32 * k;
    z[k] = e < n1 ? Elem<T>::load1(row + e) : -__int_as_float(0x7f800000);
  }
}

// ------------------------------------------------------------------- sampling records

// Running per-lane state of the online softmax: m = raw max (NaN-propagating), s = sum of
// 2^(z*scale - ref(m)), ref(m) = m*scale (0 while m = -inf, when every term is 0).
struct LaneSoft {
  float m;
  float s;
};

__device__ __forceinline__ float soft_ref(float m, float scale) {
  return m == -__int_as_float(0x7f800000) ? 0.f : __fmul_rn(m, scale);
}

// Move the lane state to a batch whose max is bm; returns the reference of the batch's terms.
__device__ __forceinline__ float soft_rebase(LaneSoft& st, float bm, float scale) {
  if (!(bm <= st.m)) {  // a larger max, or a NaN
    const float mn = max_nan(st.m, bm);
    if (st.s != 0.f)
      st.s = __fmul_rn(st.s, ex2(__fsub_rn(soft_ref(st.m, scale), soft_ref(mn, scale))));
    st.m = mn;
  }
  return soft_ref(st.m, scale);
}

// acc += 2^(z*scale - ref) over N values, in packed pairs.
template <int N>
__device__ __forceinline__ void soft_terms(uint64_t& acc, const float* z, uint64_t s2,
                                           uint64_t nr2) {
#pragma unroll
  for (int e = 0; e < N; e += 2) {
    float a0, a1;
    upk2(fma2(pk2(z[e], z[e + 1]), s2, nr2), a0, a1);
    acc = add2(acc, pk2(ex2(a0), ex2(a1)));
  }
}

__device__ __forceinline__ void soft_add(LaneSoft& st, uint64_t acc) {
  float lo, hi;
  upk2(acc, lo, hi);
  st.s = __fadd_rn(st.s, __fadd_rn(lo, hi));
}

// NaN-propagating max of one raw 16-byte vector of logits.
__device__ __forceinline__ float vec_max(const uint4& w, bf16_t) {
  const uint32_t m = max_nan_bf16x2(max_nan_bf16x2(w.x, w.y), max_nan_bf16x2(w.z, w.w));
  return max_nan(__uint_as_float(m << 16), __uint_as_float(m & 0xffff0000u));
}
__device__ __forceinline__ float vec_max(const uint4& w, float) {
  return max_nan(max_nan(__uint_as_float(w.x), __uint_as_float(w.y)),
                 max_nan(__uint_as_float(w.z), __uint_as_float(w.w)));
}

// NaN-propagating max of a batch of raw vectors.
__device__ __forceinline__ float batch_max(const uint4* v, bf16_t) {
  uint32_t m = max_nan_bf16x2(max_nan_bf16x2(v[0].x, v[0].y), max_nan_bf16x2(v[0].z, v[0].w));
#pragma unroll
  for (int k = 1; k < kBatchVecs; ++k)
    m = max_nan_bf16x2(max_nan_bf16x2(m, max_nan_bf16x2(v[k].x, v[k].y)),
                       max_nan_bf16x2(v[k].z, v[k].w));
  return max_nan(__uint_as_float(m << 16), __uint_as_float(m & 0xffff0000u));
}
__device__ __forceinline__ float batch_max(const uint4* v, float) {
  float m = max_nan(__uint_as_float(v[0].x), __uint_as_float(v[0].y));
  m = max3_nan(m, __uint_as_float(v[0].z), __uint_as_float(v[0].w));
#pragma unroll
  for (int k = 1; k < kBatchVecs; ++k) {
    m = max3_nan(m, __uint_as_float(v[k].x), __uint_as_float(v[k].y));
    m = max3_nan(m, __uint_as_float(v[k].z), __uint_as_float(v[k].w));
  }
  return m;
}

__device__ __forceinline__ float2 soft_record(const LaneSoft& st, float scale) {
  const float ninf = -__int_as_float(0x7f800000);
  const float refm = st.m == ninf ? ninf : __fmul_rn(st.m, scale);
  const SoftPart w = warp_soft_merge_lanes(refm, st.s);
  return make_float2(w.m, w.m == ninf ? 0.f : w.s);
}

template <typename T, int VEC>
__device__ __forceinline__ float2 piece_softmax(const T* row, long long o0, long long o1,
                                                int lane, float scale) {
  LaneSoft st{-__int_as_float(0x7f800000), 0.f};
  const uint64_t s2 = pk2(scale, scale);
  if constexpr (VEC == 1) {
    for (long long base = o0; base < o1; base += 32 * kBatchVecs) {
      float z[kBatchVecs];
      load_batch_scalar<T>(row, base, o1, lane, z);
      float bm = z[0];
#pragma unroll
      for (int k = 1; k < kBatchVecs; ++k) bm = max_nan(bm, z[k]);
      const float ref = soft_rebase(st, bm, scale);
      uint64_t acc = pk2(0.f, 0.f);
      soft_terms<kBatchVecs>(acc, z, s2, pk2(-ref, -ref));
      soft_add(st, acc);
    }
  } else {
    const long long nv1 = o1 / VEC;
    for (long long base = o0 / VEC; base < nv1; base += 32 * kBatchVecs) {
      uint4 v[kBatchVecs];
      load_batch<T>(row, base, nv1, lane, v);
      const float ref = soft_rebase(st, batch_max(v, T{}), scale);
      const uint64_t nr2 = pk2(-ref, -ref);
      uint64_t acc = pk2(0.f, 0.f);
#pragma unroll
      for (int k = 0; k < kBatchVecs; ++k) {
        float z[VEC];
        Elem<T>::unpack(v[k], z);
        soft_terms<VEC>(acc, z, s2, nr2);
      }
      soft_add(st, acc);
    }
  }
  return soft_record(st, scale);
}

// --------------------------------------------------------------------- greedy records

// Per lane: the max over this lane's tokens and the first of its vectors that holds it (the
// vector's raw bits are kept, so the index search needs no second read).
template <typename T, int VEC>
__device__ __forceinline__ float2 piece_argmax(const T* row, long long o0, long long o1,
                                               int lane) {
  const float ninf = -__int_as_float(0x7f800000);
  float m = ninf;
  long long best = -1;  // vector index (token index on the scalar path)
  uint4 braw = make_uint4(0, 0, 0, 0);
  if constexpr (VEC == 1) {
    for (long long base = o0; base < o1; base += 32 * kBatchVecs) {
      float z[kBatchVecs];
      load_batch_scalar<T>(row, base, o1, lane, z);
#pragma unroll
      for (int k = 0; k < kBatchVecs; ++k) {
        if ((z[k] > m || z[k] != z[k]) && m == m) {  // keep the first NaN
          m = z[k];
          best = base + lane + 32 * k;
        }
      }
    }
  } else {
    const long long nv1 = o1 / VEC;
    for (long long base = o0 / VEC; base < nv1; base += 32 * kBatchVecs) {
      uint4 v[kBatchVecs];
      load_batch<T>(row, base, nv1, lane, v);
#pragma unroll
      for (int k = 0; k < kBatchVecs; ++k) {
        const float vm = vec_max(v[k], T{});
        if ((vm > m || vm != vm) && m == m) {
          m = vm;
          best = base + lane + 32 * k;
          braw = v[k];
        }
      }
    }
  }
  const float M = warp_max_nan(m);
  unsigned first = 0xffffffffu;
  if (m == M && M > ninf) {
    if constexpr (VEC == 1) {
      first = static_cast<unsigned>(best);
    } else {
      float z[VEC];
      Elem<T>::unpack(braw, z);
#pragma unroll
      for (int e = VEC - 1; e >= 0; --e)
        if (z[e] == M) first = static_cast<unsigned>(best * VEC + e);
    }
  }
  unsigned f;
  asm volatile("redux.sync.min.u32 %0, %1, 0xffffffff;" : "=r"(f) : "r"(first));
  return make_float2(M, __int_as_float(static_cast<int>(f == 0xffffffffu ? INT_MAX : f)));
}

// --------------------------------------------------------------------------- kernel

template <typename T, int VEC, bool kSample>
__global__ void __launch_bounds__(kThreads, kStreamCtasPerSm) stream_stats_kernel(
    const StreamParams p) {
  // the finish kernel may be scheduled as soon as these CTAs retire
  grid_dependents_launch();
  const int lane = threadIdx.x & 31;
  const long long w = static_cast<long long>(blockIdx.x) * kWarps + (threadIdx.x >> 5);
  const long long u0 = w * p.upw;
  const long long u1 = min(u0 + p.upw, p.n_units);
  const long long V = p.rs.V;
  for (long long u = u0; u < u1; ++u) {
    const long long r = u / p.nch;
    const int c = static_cast<int>(u - r * p.nch);
    const int b = static_cast<int>(r / p.rs.rows);
    const int i = static_cast<int>(r - static_cast<long long>(b) * p.rs.rows);
    const T* row = row_ptr<T>(p.rs, b, i);
    const long long o0 = static_cast<long long>(c) * kCE;
    const long long o1 = min(V, o0 + kCE);
    float2 rec;
    if constexpr (kSample)
      rec = piece_softmax<T, VEC>(row, o0, o1, lane, p.scale);
    else
      rec = piece_argmax<T, VEC>(row, o0, o1, lane);
    if (lane == 0) p.rec[u] = rec;
  }
}

}  // namespace dspark
