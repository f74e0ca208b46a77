// Pass 1 of the verify step: every logit row of the block is read from HBM exactly once.
//
// The work is split into units (row, chunk): chunk c of a row is its tokens
// [2048c, min(V, 2048(c+1))). Units are numbered row-major across the batch: a row slot
// (below), then the sequence, then the chunk; each SM's CTA owns every grid-th unit and hands
// them to its warps in order. A warp streams a unit with
// 16-byte
// loads, several in flight per lane, keeps per-lane running statistics, merges its lanes and
// writes one record for the unit. A record is a function of the unit's logits alone (not of
// the launch geometry), so identical rows give identical statistics. No warp waits for
// another.
//
// Records. Sampling: (ref, sum) with ref = max_v z[v] * scale and sum = sum_v 2^(z[v]*scale
// - ref), the online-softmax pair (Milakov & Gimelshein 2018) in base 2; (-inf, 0) for a
// chunk with no value above -inf; a NaN or +inf anywhere makes the pair non-finite. Greedy:
// (max, lowest token index of the max) on the raw logits (order is unchanged by 1/T > 0).
// A mixed batch gives each sequence its own draft count K_b and temperature T_b: its units
// of rows it does not use (P rows past K_b, Q rows past its drafts, every Q row when T_b is
// 0) are skipped without a read, and its records are argmax records when T_b is 0, softmax
// records at scale log2(e) / T_b otherwise.
#pragma once

#include <climits>
#include <type_traits>

#include "common.cuh"

namespace dspark {

constexpr int kThreads = 256;            // pass-2 CTAs
constexpr int kWarps = kThreads / 32;
constexpr int kStreamThreads = 1024;     // pass 1: one CTA of 32 warps per SM (64 registers)
constexpr int kStreamWarps = kStreamThreads / 32;
constexpr int kBatchVecs = 8;            // loads each lane keeps in flight
constexpr int kCE = 2048;                // tokens per chunk (pass-1 unit, pass-2 chunk)
constexpr int kMaxChunkCount = 128;      // chunks per row (V <= 262144)

// What a call computes.
constexpr int kModeGreedy = 0;  // greedy_accept: argmax records of P rows
constexpr int kModeSample = 1;  // speculative_sample_accept: softmax records of P and Q rows
constexpr int kModeMixed = 2;   // a mixed batch: per-sequence draft count and temperature

// The logit rows of one call. Row i of sequence b: P rows i = 0..K (p_1 .. p_{K+1}), then Q
// rows i = K+1 .. 2K (q_1 .. q_K) when the call samples.
struct RowSet {
  const void* p1;
  const void* pv;
  const void* q;
  int32_t ld_p1;  // element strides (the host takes these below 2^31)
  int32_t ld_pv;
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

// Unsigned division by a divisor fixed per call, by multiplication: q = floor(n * m / 2^(32+s))
// with m = ceil(2^(32+s) / d), s = ceil(log2 d), exact for every n < 2^32 (m < 2^33 is kept as
// m_hi * 2^32 + m_lo; hs = m_hi << 8 | s). Integer multiplies only: no SFU or conversion
// instructions. Eight bytes (see StreamParamsMixed on the size of kernel parameters).
struct FastDiv {
  uint32_t m_lo, hs;
  __device__ __forceinline__ uint32_t div(uint32_t n) const {
    const uint64_t t = static_cast<uint64_t>(__umulhi(n, m_lo)) + ((hs >> 8) ? n : 0u);
    return static_cast<uint32_t>(t >> (hs & 0xffu));
  }
};

struct StreamParams {
  RowSet rs;
  uint32_t n_units;   // B * rows * nch (< 2^31)
  int nch;            // chunks per row
  int B;              // sequences
  FastDiv by_nch;     // division by nch
  FastDiv by_seqs;    // division by B

  float scale;        // log2(e) / T (sampling)
  float2* rec;        // [B, rows, nch]: the records, by (sequence, row, chunk)
  const int32_t* drafts;  // [B, K] (sampling)
  float* gather;      // [B, K, 2] (sampling): P_i[x_i], Q_i[x_i] as float
};

// A mixed batch's parameters add its per-sequence arrays. They are kept out of StreamParams:
// the back-to-back sampling call's time moved by up to a microsecond with the size and layout
// of the two kernels' parameter structs alone, the arithmetic unchanged (the cause is not
// known; these structs are the fastest layout measured), so the other modes carry none of
// the mixed batch's fields.
struct StreamParamsMixed : StreamParams {
  const int32_t* n_drafts;  // [B] K_b, or null for K
  const float* temps;       // [B] T_b
};
template <int kMode>
using StreamParamsOf = std::conditional_t<kMode == kModeMixed, StreamParamsMixed, StreamParams>;

// A sequence of a mixed batch: its draft count K_b, whether its parameters are valid
// (0 <= K_b <= K, T_b finite and >= 0, log2(e) / T_b finite), whether it is greedy (T_b == 0)
// and its scale log2(e) / T_b, rounded exactly as the host rounds a call's single scale.
struct SeqMode {
  int kb;
  bool ok;
  bool greedy;
  float scale;
};
__device__ __forceinline__ SeqMode seq_mode(const int32_t* n_drafts, const float* temps, int b,
                                            int K) {
  SeqMode m;
  m.kb = n_drafts ? __ldg(n_drafts + b) : K;
  const float T = __ldg(temps + b);
  m.greedy = T == 0.f;
  m.scale = T > 0.f ? static_cast<float>(1.4426950408889634 / static_cast<double>(T)) : 0.f;
  m.ok = m.kb >= 0 && m.kb <= K && T >= 0.f && T <= 3.402823466e38f &&
         (m.greedy || m.scale <= 3.402823466e38f);
  return m;
}

// Which rows of a sequence a call reads: P rows 0..kb (row kb is the bonus row) and, when it
// samples, the Q rows of its kb drafts. Row r of the block: P rows 0..K, then Q rows.
struct RowFilter {
  int K, kb;
  bool q;
  __device__ __forceinline__ bool operator()(int r) const {
    return r <= K ? r <= kb : (q && r - K - 1 < kb);
  }
};

// (sequence b, row i, chunk c) of a unit.
struct UnitPos {
  int b, i, c;
};

// Unit u: chunk c = u mod nch, sequence b = (u / nch) mod B, row slot r = u / (nch B). The
// slots take every sequence's rows in the order P_K (the bonus row), then for i = K-1 down to
// 0: P_i, then Q_i when sampling. The rows read last, still in L2 when pass 2 re-reads the row
// pair of a rejection at j, are then the low ones, where rejections concentrate (each draft
// is accepted with probability below one, so j = 0 is the most likely single outcome).
__device__ __forceinline__ UnitPos unit_pos(const StreamParams& p, uint32_t u) {
  UnitPos at;
  const uint32_t q = p.by_nch.div(u);
  at.c = static_cast<int>(u - q * static_cast<uint32_t>(p.nch));
  const uint32_t r = p.by_seqs.div(q);
  at.b = static_cast<int>(q - r * static_cast<uint32_t>(p.B));
  const int K = p.rs.K;
  if (r == 0) {
    at.i = K;
  } else if (p.rs.rows == K + 1) {  // greedy: P rows only
    at.i = K - static_cast<int>(r);
  } else {
    const int t = static_cast<int>(r) - 1;
    const int pair = K - 1 - (t >> 1);
    at.i = (t & 1) ? K + 1 + pair : pair;
  }
  return at;
}

// Index of a unit's record: rows of a sequence together, chunks in order within a row.
__device__ __forceinline__ size_t record_index(const StreamParams& p, const UnitPos& at) {
  return (static_cast<size_t>(at.b) * p.rs.rows + at.i) * p.nch + at.c;
}

// Sampling: the unit that holds a draft token x_i of a draft row (P row i < nd, or Q row i;
// nd = K, or a mixed batch's K_b) also writes that token's logit for pass 2, so pass 2 need
// not fetch it from HBM. `xd` is drafts[b, draft index of row i] (or -1), loaded before the
// unit's math.
template <typename T, bool kMixed>
__device__ __forceinline__ int unit_draft(const StreamParams& p, const UnitPos& at, int lane,
                                          int nd) {
  const int K = p.rs.K;
  if (lane != 0 || (kMixed ? (at.i <= K && at.i >= nd) : at.i == K)) return -1;
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

// Where a unit's 16-byte vectors come from: vector vi of the row in global memory.
template <typename T>
struct GlobalVecs {
  const T* row;
  __device__ __forceinline__ uint4 operator()(long long vi) const {
    return ld_stream16(row + vi * Elem<T>::kPerVec16);
  }
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

// One CTA per SM. CTA k owns units k, k + grid, k + 2 grid, ... and hands them to its warps in
// order from a shared-memory counter, one at a time: lane 0 asks for the next unit while the
// warp works on the current one, so the atomic's latency is hidden, and the warps that the SM's
// scheduler favours simply take more units. Every SM holds the same share of the work and its
// warps finish together; no global atomic, fence or barrier is involved. The whole grid sweeps
// the units front to back, so the rows read last (row pair 0 of every sequence) are the ones
// still in L2 when pass 2 runs.
template <typename T, int VEC, int kMode>
__global__ void __launch_bounds__(kStreamThreads, 1) stream_stats_kernel(
    const StreamParamsOf<kMode> p) {
  __shared__ unsigned s_next;
  // Launched as a programmatic dependent of whatever precedes it in the stream, so that its
  // CTAs are resident as the previous kernel drains: nothing is read before that kernel has
  // completed and its writes are visible. Only then may the finish kernel be scheduled (it
  // reads the drafts and uniforms before waiting for this pass).
  grid_dependency_wait();
  grid_dependents_launch();
  const int lane = threadIdx.x & 31;
  const int wi = threadIdx.x >> 5;
  const int V = p.rs.V;
  const unsigned k = blockIdx.x, G = gridDim.x;
  const unsigned n_mine = k < p.n_units ? (p.n_units - 1 - k) / G + 1 : 0;  // this CTA's units
  if (threadIdx.x == 0) s_next = kStreamWarps;  // the first kStreamWarps go to warps 0..31
  __syncthreads();
  unsigned nxt = 0;
  unsigned m = wi;
  while (m < n_mine) {
    if (lane == 0) nxt = atomicAdd(&s_next, 1u);
    const unsigned u = k + m * G;
    const UnitPos at = unit_pos(p, u);
    const T* row = row_ptr<T>(p.rs, at.b, at.i);
    const int o0 = at.c * kCE;
    const int o1 = min(V, o0 + kCE);
    float2 rec;
    bool used = true;
    if constexpr (kMode == kModeSample) {
      const int xd = unit_draft<T, false>(p, at, lane, p.rs.K);
      rec = piece_softmax<T, VEC>(row, o0, o1, lane, p.scale);
      unit_gather<T>(p, at, row, xd, o0, o1);
    } else if constexpr (kMode == kModeGreedy) {
      rec = piece_argmax<T, VEC>(row, o0, o1, lane);
    } else {
      const SeqMode sm = seq_mode(p.n_drafts, p.temps, at.b, p.rs.K);
      used = sm.ok && RowFilter{p.rs.K, sm.kb, !sm.greedy}(at.i);
      if (used) {
        if (sm.greedy) {
          rec = piece_argmax<T, VEC>(row, o0, o1, lane);
        } else {
          const int xd = unit_draft<T, true>(p, at, lane, sm.kb);
          rec = piece_softmax<T, VEC>(row, o0, o1, lane, sm.scale);
          unit_gather<T>(p, at, row, xd, o0, o1);
        }
      }
    }
    if (lane == 0 && used) p.rec[record_index(p, at)] = rec;
    m = __shfl_sync(0xffffffffu, nxt, 0);
  }
}

}  // namespace dspark
