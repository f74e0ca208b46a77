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
  long long upw;      // units per warp (contiguous runs)
  long long warps;    // warps of the grid (strided order)
  int strided;        // 1: warp w takes units w, w + warps, ...; 0: a contiguous run
  int nch;            // chunks per row
  int stages;         // ring kernel: shared-memory stages per warp
  float scale;        // log2(e) / T (sampling)
  float2* rec;        // [n_units]: record of unit u at u
  const int32_t* drafts;  // [B, K] (sampling)
  float* gather;      // [B, K, 2] (sampling): P_i[x_i], Q_i[x_i] as float
};



// Record of a unit whose data never arrived (a bounded wait gave up): its second word has
// these bits, which no statistics record has (arithmetic NaNs are 0x7fffffff, indices >= 0).
constexpr uint32_t kTimeoutRecBits = 0xffffffffu;

// (sequence b, row i, chunk c) of a unit, stepped through a warp's run in order.
struct UnitPos {
  int b, i, c;
  __device__ __forceinline__ void init(long long u, int nch, int rows) {
    const long long r = u / nch;
    c = static_cast<int>(u - r * nch);
    b = static_cast<int>(r / rows);
    i = static_cast<int>(r - static_cast<long long>(b) * rows);
  }
  __device__ __forceinline__ void next(int nch, int rows) {
    if (++c == nch) {
      c = 0;
      if (++i == rows) {
        i = 0;
        ++b;
      }
    }
  }
};

// Steps a unit position by a fixed stride n = q * nch + rc (rc < nch) without dividing:
// c += rc with a carry into the row, the row advances by q or q + 1, and the row index
// (b * rows + i) is split the same way with precomputed quotients of both row steps.
struct UnitStride {
  int rc;                   // stride mod nch
  int qi0, qb0, qi1, qb1;   // row steps q and q + 1 as (mod rows, div rows)
  __device__ __forceinline__ void init(long long n, int nch, int rows) {
    const long long q = n / nch;
    rc = static_cast<int>(n - q * nch);
    qb0 = static_cast<int>(q / rows);
    qi0 = static_cast<int>(q - static_cast<long long>(qb0) * rows);
    qb1 = static_cast<int>((q + 1) / rows);
    qi1 = static_cast<int>(q + 1 - static_cast<long long>(qb1) * rows);
  }
  __device__ __forceinline__ void step(UnitPos& at, int nch, int rows) const {
    at.c += rc;
    int di = qi0, db = qb0;
    if (at.c >= nch) {
      at.c -= nch;
      di = qi1;
      db = qb1;
    }
    at.i += di;
    at.b += db;
    if (at.i >= rows) {
      at.i -= rows;
      ++at.b;
    }
  }
};

// Sampling: the unit that holds a draft token x_i of a draft row (P row i < K, or Q row i)
// also writes that token's logit for pass 2, so pass 2 need not fetch it from HBM.
// `xd` is drafts[b, draft index of row i] (or -1), loaded before the unit's math.
template <typename T>
__device__ __forceinline__ int unit_draft(const StreamParams& p, const UnitPos& at, int lane) {
  const int K = p.rs.K;
  if (lane != 0 || at.i == K) return -1;
  const int di = at.i < K ? at.i : at.i - K - 1;
  return __ldg(p.drafts + static_cast<size_t>(at.b) * K + di);
}
template <typename T>
__device__ __forceinline__ void unit_gather(const StreamParams& p, const UnitPos& at, const T* row,
                                            int xd, int o0, int o1) {
  if (xd < o0 || xd >= o1) return;  // not in this unit (or not lane 0, or an invalid id)
  const int K = p.rs.K;
  const int di = at.i < K ? at.i : at.i - K - 1;
  p.gather[(static_cast<size_t>(at.b) * K + di) * 2 + (at.i > K)] = Elem<T>::load1(row + xd);
}

// ------------------------------------------------------------------------ batch loads

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

// Where a unit's 16-byte vectors come from: global memory (vector vi of the row) or this
// warp's shared-memory stage (vector vi - nv0 of the stage).
template <typename T>
struct GlobalVecs {
  const T* row;
  __device__ __forceinline__ uint4 operator()(long long vi) const {
    return ld_stream16(row + vi * Elem<T>::kPerVec16);
  }
};
struct StageVecs {
  const uint4* stage;
  long long nv0;
  __device__ __forceinline__ uint4 operator()(long long vi) const { return stage[vi - nv0]; }
};

template <typename T, class Src>
__device__ __forceinline__ void load_batch_from(const Src& src, long long base, long long nv1,
                                                int lane, uint4* v) {
  const uint32_t ninf = Elem<T>::kBytes == 2 ? 0xff80ff80u : 0xff800000u;
#pragma unroll
  for (int k = 0; k < kBatchVecs; ++k) {
    const long long vi = base + lane + 32 * k;
    v[k] = vi < nv1 ? src(vi) : make_uint4(ninf, ninf, ninf, ninf);
  }
}

// Softmax record of the row's vectors [nv0, nv1) (16-byte path).
template <typename T, class Src>
__device__ __forceinline__ float2 unit_softmax_vec(const Src& src, long long nv0, long long nv1,
                                                   int lane, float scale) {
  constexpr int VEC = Elem<T>::kPerVec16;
  LaneSoft st{-__int_as_float(0x7f800000), 0.f};
  const uint64_t s2 = pk2(scale, scale);
  for (long long base = nv0; base < nv1; base += 32 * kBatchVecs) {
    uint4 v[kBatchVecs];
    load_batch_from<T>(src, base, nv1, lane, v);
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
  return soft_record(st, scale);
}

template <typename T, int VEC>
__device__ __forceinline__ float2 piece_softmax(const T* row, long long o0, long long o1,
                                                int lane, float scale) {
  if constexpr (VEC == 1) {
    LaneSoft st{-__int_as_float(0x7f800000), 0.f};
    const uint64_t s2 = pk2(scale, scale);
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
    return soft_record(st, scale);
  } else {
    return unit_softmax_vec<T>(GlobalVecs<T>{row}, o0 / VEC, o1 / VEC, lane, scale);
  }
}

// --------------------------------------------------------------------- greedy records

// Per lane: the max over this lane's tokens and the first of its vectors that holds it (the
// vector's raw bits are kept, so the index search needs no second read).
// Lowest index of the warp's maximum, given each lane's max m and the raw bits of the first of
// its vectors that holds it (vector index best; scalar path: token index).
template <typename T, int VEC>
__device__ __forceinline__ float2 argmax_record(float m, long long best, const uint4& braw) {
  const float M = warp_max_nan(m);
  unsigned first = 0xffffffffu;
  if (m == M && M > -__int_as_float(0x7f800000)) {
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

// Argmax record of the row's vectors [nv0, nv1) (16-byte path). Per lane: the max over its
// tokens and the first of its vectors that holds it (raw bits kept, no second read).
template <typename T, class Src>
__device__ __forceinline__ float2 unit_argmax_vec(const Src& src, long long nv0, long long nv1,
                                                  int lane) {
  float m = -__int_as_float(0x7f800000);
  long long best = -1;
  uint4 braw = make_uint4(0, 0, 0, 0);
  for (long long base = nv0; base < nv1; base += 32 * kBatchVecs) {
    uint4 v[kBatchVecs];
    load_batch_from<T>(src, base, nv1, lane, v);
#pragma unroll
    for (int k = 0; k < kBatchVecs; ++k) {
      const float vm = vec_max(v[k], T{});
      if ((vm > m || vm != vm) && m == m) {  // keep the first NaN
        m = vm;
        best = base + lane + 32 * k;
        braw = v[k];
      }
    }
  }
  return argmax_record<T, Elem<T>::kPerVec16>(m, best, braw);
}

template <typename T, int VEC>
__device__ __forceinline__ float2 piece_argmax(const T* row, long long o0, long long o1,
                                               int lane) {
  if constexpr (VEC == 1) {
    float m = -__int_as_float(0x7f800000);
    long long best = -1;
    for (long long base = o0; base < o1; base += 32 * kBatchVecs) {
      float z[kBatchVecs];
      load_batch_scalar<T>(row, base, o1, lane, z);
#pragma unroll
      for (int k = 0; k < kBatchVecs; ++k) {
        if ((z[k] > m || z[k] != z[k]) && m == m) {
          m = z[k];
          best = base + lane + 32 * k;
        }
      }
    }
    return argmax_record<T, 1>(m, best, make_uint4(0, 0, 0, 0));
  } else {
    return unit_argmax_vec<T>(GlobalVecs<T>{row}, o0 / VEC, o1 / VEC, lane);
  }
}

// --------------------------------------------------------------------------- kernel

template <typename T, int VEC, bool kSample>
__global__ void __launch_bounds__(kThreads, kStreamCtasPerSm) stream_stats_kernel(
    const StreamParams p) {
  // the finish kernel may be scheduled as soon as these CTAs retire
  grid_dependents_launch();
  const int lane = threadIdx.x & 31;
  const long long w = static_cast<long long>(blockIdx.x) * kWarps + (threadIdx.x >> 5);
  // units of this warp: u0, u0 + du, ... below u1 (a contiguous run, or a grid stride)
  const long long u0 = p.strided ? w : w * p.upw;
  const long long u1 = p.strided ? p.n_units : min(u0 + p.upw, p.n_units);
  const long long du = p.strided ? p.warps : 1;
  if (u0 >= u1) return;
  UnitPos at;
  at.init(u0, p.nch, p.rs.rows);
  UnitStride stride;
  stride.init(du, p.nch, p.rs.rows);
  const int V = p.rs.V;
  for (long long u = u0; u < u1; u += du) {
    const T* row = row_ptr<T>(p.rs, at.b, at.i);
    const int o0 = at.c * kCE;
    const int o1 = min(V, o0 + kCE);
    float2 rec;
    if constexpr (kSample) {
      const int xd = unit_draft<T>(p, at, lane);
      rec = piece_softmax<T, VEC>(row, o0, o1, lane, p.scale);
      unit_gather<T>(p, at, row, xd, o0, o1);
    } else {
      rec = piece_argmax<T, VEC>(row, o0, o1, lane);
    }
    if (lane == 0) p.rec[u] = rec;
    stride.step(at, p.nch, p.rs.rows);
  }
}

// ---------------------------------------------------------------- ring kernel (16-byte path)

// The same pass with each warp's next units staged in shared memory by 1-D bulk copies
// (cp.async.bulk, one per unit, issued by lane 0 `stages` units ahead), so a warp's loads stay
// in flight while it computes. Stage and mbarrier per (warp, slot); no data is shared between
// warps. A unit's bytes: min(V - 2048c, 2048) tokens, a multiple of 16 bytes on this path.
constexpr int kRingCtasPerSm = 2;
constexpr int kMaxStages = 4;

template <typename T>
__device__ __forceinline__ void issue_unit(const StreamParams& p, const UnitPos& at,
                                           unsigned char* stage, uint64_t* bar) {
  const int o0 = at.c * kCE;
  const int n = min(p.rs.V - o0, kCE);
  const uint32_t bytes = static_cast<uint32_t>(n) * Elem<T>::kBytes;
  mbar_arrive_expect_tx(bar, bytes);
  bulk_g2s(stage, row_ptr<T>(p.rs, at.b, at.i) + o0, bytes, bar);
}

template <typename T, bool kSample>
__global__ void __launch_bounds__(kThreads, kRingCtasPerSm) stream_stats_ring_kernel(
    const StreamParams p) {
  extern __shared__ __align__(128) unsigned char smem[];
  grid_dependents_launch();
  constexpr int VEC = Elem<T>::kPerVec16;
  constexpr int UB = kCE * Elem<T>::kBytes;  // bytes per stage
  const int lane = threadIdx.x & 31, wi = threadIdx.x >> 5;
  const int S = p.stages;
  unsigned char* ring = smem + static_cast<size_t>(wi) * S * UB;
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + static_cast<size_t>(kWarps) * S * UB) +
                  wi * kMaxStages;
  const long long w = static_cast<long long>(blockIdx.x) * kWarps + wi;
  const long long u0 = w * p.upw;
  const long long u1 = min(u0 + p.upw, p.n_units);
  if (u0 >= u1) return;
  const int n = static_cast<int>(u1 - u0);
  UnitPos at, ahead;
  at.init(u0, p.nch, p.rs.rows);
  ahead = at;
  if (lane == 0) {
    for (int s = 0; s < S; ++s) mbar_init(&bar[s], 1);
    fence_mbar_init();
    for (int k = 0; k < S && k < n; ++k) {
      issue_unit<T>(p, ahead, ring + k * UB, &bar[k]);
      ahead.next(p.nch, p.rs.rows);
    }
  }
  __syncwarp();
  const int V = p.rs.V;
  int issued = S < n ? S : n;  // units whose copies were issued (lane 0's count, kept warp-wide)
  int first_failed = -1;       // first unit whose wait gave up
  bool failed = false;
  for (int k = 0; k < n; ++k) {
    const int st = k % S;
    float2 rec;
    if (!failed) {
      failed = !__all_sync(0xffffffffu, mbar_wait_bounded(&bar[st], (k / S) & 1));
      if (failed) first_failed = k;
    }
    if (!failed) {
      const int o0 = at.c * kCE;
      const int o1 = min(V, o0 + kCE);
      const StageVecs src{reinterpret_cast<const uint4*>(ring + st * UB), o0 / VEC};
      if constexpr (kSample) {
        const int xd = unit_draft<T>(p, at, lane);
        rec = unit_softmax_vec<T>(src, o0 / VEC, o1 / VEC, lane, p.scale);
        unit_gather<T>(p, at, row_ptr<T>(p.rs, at.b, at.i), xd, o0, o1);
      } else {
        rec = unit_argmax_vec<T>(src, o0 / VEC, o1 / VEC, lane);
      }
    } else {
      rec = make_float2(0.f, __uint_as_float(kTimeoutRecBits));
    }
    __syncwarp();  // every lane is done with the stage
    if (lane == 0) {
      p.rec[u0 + k] = rec;
      if (!failed && k + S < n) {
        fence_proxy_async_smem();  // the stage's reads come before the copy that refills it
        issue_unit<T>(p, ahead, ring + st * UB, &bar[st]);
        ahead.next(p.nch, p.rs.rows);
      }
    }
    if (!failed && k + S < n) ++issued;
    at.next(p.nch, p.rs.rows);
  }
  if (failed) {
    // copies still in flight land in this warp's stages: wait for them (bounded) before exit
    for (int k = first_failed; k < issued; ++k) mbar_wait_bounded(&bar[k % S], (k / S) & 1);
  }
}

}  // namespace dspark
