// Both verify policies as one persistent kernel of warp-specialised tasks (sm_100a).
//
// Every CTA has kStreamWarps streaming warps and one dependent-task warp.
//   * Streaming warps run the STREAM tasks in one global order, round-robin, and never wait
//     on another warp: STREAM(b, r, c) reads chunk c (2048 tokens) of row r of sequence b
//     once from HBM through the warp's ring of shared-memory stages (1-D bulk copies, no
//     multicast) and writes the chunk's record - sampling: max and sum of 2^(z*s - ref);
//     greedy: max and lowest index - then counts it in the sequence's counter. The count is
//     a non-returning release add, issued one task late so the record's store has already
//     completed and the release costs no wait.
//   * Dependent-task warps run, in order and round-robin, per sequence b:
//       DECIDE(b)   waits for all rows x chunks records of b, merges them into the row
//                   statistics, runs the accept tests (p_i(x_i), q_i(x_i), or the argmax
//                   comparison) and finds j. Greedy ends here.
//       RESID(b, c) sampling, j < K: chunk c of max(p_j - q_j, 0) from P_j and Q_j again
//                   (streamed moments before, so normally still in L2), its mass.
//       SAMPLE(b)   sampling: float64 scan of the chunk masses of the draw's law (residual j,
//                   or p_K from the STREAM records), then only the selected chunk is re-read
//                   and scanned to pick the token.
//     A dependent task waits (bounded) only on STREAM tasks, which always progress, or on
//     dependent tasks earlier in the same order, so the schedule cannot deadlock while all
//     CTAs are resident. The last task of a sequence (SAMPLE, or greedy's DECIDE) resets the
//     sequence's counters, so the workspace's counter region is zero again after a call.
#pragma once

#include <climits>

#include "common.cuh"

namespace dspark {

constexpr int kTaskThreads = 256;
constexpr int kTaskWarps = kTaskThreads / 32;
constexpr int kStreamWarps = kTaskWarps - 1;  // warp kStreamWarps runs dependent tasks
constexpr int kMaxRows = 2 * kMaxK + 1;
constexpr int kPubLane = 31;  // the streaming lane that publishes records (lane 0 produces)
constexpr int kPubBatch = 4;  // STREAM records counted per release fence
constexpr int kResidGroup = 2;  // chunks per RESID task
constexpr int kCE = 2048;               // tokens per chunk
constexpr int kCL = kCE / 32;           // tokens per lane per chunk
constexpr int kMaxChunkCount = 128;     // chunks per row (V <= 262144)
constexpr int kMaxTaskStages = 4;

enum TaskType { T_NOOP = 0, T_STREAM = 1, T_DECIDE = 2, T_RESID = 3, T_SAMPLE = 4 };

// What DECIDE leaves for RESID and SAMPLE. "p" is the P row of the draw (j, or K for the
// bonus), "q" the Q row j; ip, iq are 1/S of those rows.
struct SeqDecision {
  int j;
  int status;
  float mp, ip, mq, iq;
  int pad0, pad1;
};

// The dependent-task queue (zero between calls; the last dependent warp to leave resets it).
struct DepQueue {
  unsigned next;    // next dependent task to hand out
  unsigned exited;  // dependent warps that found the queue empty
  unsigned pad[2];
};

// Per-sequence counters (zero between calls; SAMPLE, or greedy's DECIDE, resets them).
struct SeqCounters {
  unsigned streamed;    // STREAM tasks of the sequence whose record is written
  unsigned decided;     // DECIDE finished
  unsigned resid_done;  // RESID tasks finished
  unsigned pad;
};

struct TaskParams {
  const void* p1;
  const void* pv;
  const void* q;
  int64_t ld_p1;
  int64_t ld_pv;
  int B, K, V;
  float scale;  // log2(e) / T (sampling)
  const int32_t* drafts;
  const float* uniforms;
  // schedule
  int nch;               // chunks per row
  int rows;              // rows per sequence: 2K+1 (sampling) or K+1 (greedy)
  long long n_stream;    // STREAM tasks: B * rows * nch
  int n_resid;           // RESID tasks per sequence: ceil(nch / kResidGroup) (sampling)
  int n_dep_per_seq;     // dependent tasks per sequence: n_resid + 2 (sampling) or 1 (greedy)
  int stream_warps;      // streaming warps in the grid
  int dep_warps;         // dependent-task warps in the grid
  int stages;
  // workspace
  float2* chunk_stat;    // [B, rows, nch]: (ref, sum) | (max, argmax bits)
  float2* row_stat;      // [B, rows]: (M, S) | (max, argmax bits)
  SeqCounters* seq_cnt;  // [B]
  DepQueue* dq;          // [1]
  SeqDecision* dec;      // [B]
  float* resid_mass;     // [B, nch]
  dspark_accept_out_t out;
};

// ------------------------------------------------------------------ global sync helpers

__device__ __forceinline__ unsigned atomic_add_acq_rel_gpu(unsigned* p, unsigned v) {
  unsigned old;
  asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v)
               : "memory");
  return old;
}
__device__ __forceinline__ void red_release_gpu(unsigned* p, unsigned v) {
  asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ void red_relaxed_gpu(unsigned* p, unsigned v) {
  asm volatile("red.relaxed.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ void fence_acq_rel_gpu() {
  asm volatile("fence.acq_rel.gpu;" ::: "memory");
}
__device__ __forceinline__ void st_release_gpu(unsigned* p, unsigned v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ unsigned ld_acquire_gpu(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
// Loads of data other warps wrote in this launch: through L2, never a stale L1 line.
__device__ __forceinline__ float2 ld_cg_f2(const float2* p) { return __ldcg(p); }
__device__ __forceinline__ float ld_cg_f(const float* p) { return __ldcg(p); }

// Wait (lane 0 polls, bounded) until *p >= target; returns false on timeout.
__device__ __forceinline__ bool wait_counter(const unsigned* p, unsigned target) {
  bool ok = true;
  if ((threadIdx.x & 31) == 0) {
    if (ld_acquire_gpu(p) < target) {
      const unsigned long long t0 = globaltimer_ns();
      while (ld_acquire_gpu(p) < target) {
        __nanosleep(200);
        if (globaltimer_ns() - t0 > kWaitLimitNs) {
          ok = false;
          break;
        }
      }
    }
  }
  ok = __shfl_sync(0xffffffffu, ok, 0);
  __syncwarp();
  return ok;
}

// The decision record as written by another warp in this launch (read through L2).
__device__ __forceinline__ SeqDecision load_decision(const SeqDecision* d) {
  const int4 a = __ldcg(reinterpret_cast<const int4*>(d));
  const int4 c = __ldcg(reinterpret_cast<const int4*>(d) + 1);
  SeqDecision r;
  r.j = a.x;
  r.status = a.y;
  r.mp = __int_as_float(a.z);
  r.ip = __int_as_float(a.w);
  r.mq = __int_as_float(c.x);
  r.iq = __int_as_float(c.y);
  r.pad0 = r.pad1 = 0;
  return r;
}

// ---------------------------------------------------------------- stream task positions

// STREAM task s = (b * rows + r) * nch + c, sequence-major so that sequences complete in
// order. A streaming warp runs s = w, w + N, ... (N = streaming warps); its position is
// stepped without a division by (qb, qr, qc) = N in base (rows*nch, nch).
struct StreamPos {
  long long s;
  int b, r, c;
};
struct StreamStep {
  int qb, qr, qc, rows, nch;
  __device__ __forceinline__ void advance(StreamPos& sp, long long n) const {
    sp.s += n;
    sp.c += qc;
    if (sp.c >= nch) {
      sp.c -= nch;
      ++sp.r;
    }
    sp.r += qr;
    if (sp.r >= rows) {
      sp.r -= rows;
      ++sp.b;
    }
    sp.b += qb;
  }
};

// Row r of sequence b: P rows 0..K, then Q rows 0..K-1.
template <typename T>
__device__ __forceinline__ const T* row_ptr(const TaskParams& p, int b, int r) {
  const int K = p.K;
  if (r == 0) return static_cast<const T*>(p.p1) + static_cast<int64_t>(b) * p.ld_p1;
  if (r <= K)
    return static_cast<const T*>(p.pv) + static_cast<int64_t>(b) * p.ld_pv +
           static_cast<int64_t>(r - 1) * p.V;
  return static_cast<const T*>(p.q) + (static_cast<int64_t>(b) * K + (r - K - 1)) * p.V;
}

// This lane's VEC tokens of vector k of a chunk: tokens (k*32 + lane)*VEC + e (k*32 + lane on
// the scalar path); -inf at or past `valid`.
template <typename T, int VEC>
__device__ __forceinline__ void lane_vec(const T* gl_chunk, int valid, int k, int lane, float* z) {
  const float ninf = -__int_as_float(0x7f800000);
  if constexpr (VEC == 1) {
    const int e = k * 32 + lane;
    z[0] = e < valid ? Elem<T>::load1(gl_chunk + e) : ninf;
  } else {
    const int vi = k * 32 + lane;
    if (vi * VEC < valid) {
      Elem<T>::unpack(ld_stream16(gl_chunk + vi * VEC), z);
    } else {
#pragma unroll
      for (int e = 0; e < VEC; ++e) z[e] = ninf;
    }
  }
}

// This lane's vector k of a chunk as raw 16 bytes; vectors at or past `valid` read as -inf.
template <typename T>
__device__ __forceinline__ uint4 lane_raw(const T* gl_chunk, int valid, int k, int lane) {
  constexpr int VEC = Elem<T>::kPerVec16;
  const int vi = k * 32 + lane;
  if (vi * VEC < valid) return ld_stream16(gl_chunk + vi * VEC);
  const uint32_t ninf = Elem<T>::kBytes == 2 ? 0xff80ff80u : 0xff800000u;
  return make_uint4(ninf, ninf, ninf, ninf);
}

// All kCL tokens of this lane, z[k*VEC + e] = lane_vec(k)[e] (direct-load STREAM path).
template <typename T, int VEC>
__device__ __forceinline__ void chunk_lane_values(const T* gl_chunk, int valid, int lane, float* z) {
#pragma unroll
  for (int k = 0; k < kCL / VEC; ++k) lane_vec<T, VEC>(gl_chunk, valid, k, lane, z + k * VEC);
}

__device__ __forceinline__ int lane_token(int cbase, int k, int lane, int vec) {
  return cbase + ((k / vec) * 32 + lane) * vec + (k % vec);
}

// ------------------------------------------------------------------------ STREAM parts

// Sampling, from registers: chunk max (NaN-propagating), reference, warp sum of
// 2^(z*s - ref). Record: (ref, or -inf for a chunk with nothing above -inf; sum).
__device__ __forceinline__ float2 stream_softmax_part(const float* z, float scale) {
  const float ninf = -__int_as_float(0x7f800000);
  float m = ninf;
#pragma unroll
  for (int k = 0; k < kCL; k += 2) m = max3_nan(m, z[k], z[k + 1]);
  m = warp_max_nan(m);
  const float ref = m == ninf ? 0.f : __fmul_rn(m, scale);
  const uint64_t s2 = pk2(scale, scale);
  const uint64_t nr2 = pk2(-ref, -ref);
  uint64_t acc = pk2(0.f, 0.f);
#pragma unroll
  for (int k = 0; k < kCL; k += 2) {
    float a0, a1;
    upk2(fma2(pk2(z[k], z[k + 1]), s2, nr2), a0, a1);
    acc = add2(acc, pk2(ex2(a0), ex2(a1)));
  }
  float lo, hi;
  upk2(acc, lo, hi);
  return make_float2(m == ninf ? ninf : ref, warp_sum(__fadd_rn(lo, hi)));
}

// Greedy, from registers: chunk max (NaN-propagating) and its lowest token.
// Record: (max, token bits).
template <int VEC>
__device__ __forceinline__ float2 stream_argmax_part(const float* z, int cbase, int lane) {
  const float ninf = -__int_as_float(0x7f800000);
  float m = ninf;
#pragma unroll
  for (int k = 0; k < kCL; k += 2) m = max3_nan(m, z[k], z[k + 1]);
  const float M = warp_max_nan(m);
  int first = INT_MAX;
  if (m == M && M > ninf) {  // only lanes that hold the maximum look for it
#pragma unroll
    for (int k = kCL - 1; k >= 0; --k)
      if (z[k] == M) first = lane_token(cbase, k, lane, VEC);
  }
  unsigned f;
  asm volatile("redux.sync.min.u32 %0, %1, 0xffffffff;" : "=r"(f) : "r"(static_cast<unsigned>(first)));
  return make_float2(M, __int_as_float(static_cast<int>(f)));
}

// The same two parts read straight from this warp's shared-memory stage in two passes (max,
// then exponentials), so no chunk is held in registers. 16-byte vector path only.
template <typename T>
__device__ __forceinline__ float lane_max_smem(const uint4* st, int valid, int lane);

template <>
__device__ __forceinline__ float lane_max_smem<bf16_t>(const uint4* st, int valid, int lane) {
  uint32_t m = 0xff80ff80u;  // (-inf, -inf)
#pragma unroll
  for (int k = 0; k < kCL / 8; ++k) {
    const int vi = k * 32 + lane;
    if (vi * 8 < valid) {
      const uint4 w = st[vi];
      m = max_nan_bf16x2(max_nan_bf16x2(m, w.x), max_nan_bf16x2(w.y, max_nan_bf16x2(w.z, w.w)));
    }
  }
  return max_nan(__uint_as_float(m << 16), __uint_as_float(m & 0xffff0000u));
}

template <>
__device__ __forceinline__ float lane_max_smem<float>(const uint4* st, int valid, int lane) {
  float m = -__int_as_float(0x7f800000);
#pragma unroll
  for (int k = 0; k < kCL / 4; ++k) {
    const int vi = k * 32 + lane;
    if (vi * 4 < valid) {
      const uint4 w = st[vi];
      m = max3_nan(m, max3_nan(__uint_as_float(w.x), __uint_as_float(w.y), __uint_as_float(w.z)),
                   __uint_as_float(w.w));
    }
  }
  return m;
}

template <typename T>
__device__ __forceinline__ float2 stream_softmax_part_smem(const unsigned char* stage, int valid,
                                                           int lane, float scale) {
  constexpr int VEC = Elem<T>::kPerVec16;
  const float ninf = -__int_as_float(0x7f800000);
  const uint4* st = reinterpret_cast<const uint4*>(stage);
  const float m = warp_max_nan(lane_max_smem<T>(st, valid, lane));
  const float ref = m == ninf ? 0.f : __fmul_rn(m, scale);
  const uint64_t s2 = pk2(scale, scale);
  const uint64_t nr2 = pk2(-ref, -ref);
  uint64_t acc = pk2(0.f, 0.f);
#pragma unroll
  for (int k = 0; k < kCL / VEC; ++k) {
    const int vi = k * 32 + lane;
    if (vi * VEC < valid) {
      float z[VEC];
      Elem<T>::unpack(st[vi], z);
#pragma unroll
      for (int e = 0; e < VEC; e += 2) {
        float a0, a1;
        upk2(fma2(pk2(z[e], z[e + 1]), s2, nr2), a0, a1);
        acc = add2(acc, pk2(ex2(a0), ex2(a1)));
      }
    }
  }
  float lo, hi;
  upk2(acc, lo, hi);
  return make_float2(m == ninf ? ninf : ref, warp_sum(__fadd_rn(lo, hi)));
}

// Max of one 16-byte vector of logits (NaN-propagating).
__device__ __forceinline__ float vec_max(const uint4& w, bf16_t) {
  const uint32_t m = max_nan_bf16x2(max_nan_bf16x2(w.x, w.y), max_nan_bf16x2(w.z, w.w));
  return max_nan(__uint_as_float(m << 16), __uint_as_float(m & 0xffff0000u));
}
__device__ __forceinline__ float vec_max(const uint4& w, float) {
  return max_nan(max_nan(__uint_as_float(w.x), __uint_as_float(w.y)),
                 max_nan(__uint_as_float(w.z), __uint_as_float(w.w)));
}

template <typename T>
__device__ __forceinline__ float2 stream_argmax_part_smem(const unsigned char* stage, int valid,
                                                          int cbase, int lane) {
  constexpr int VEC = Elem<T>::kPerVec16;
  const float ninf = -__int_as_float(0x7f800000);
  const uint4* st = reinterpret_cast<const uint4*>(stage);
  // lane max and the first of this lane's vectors that holds it
  float m = ninf;
  int kbest = -1;
#pragma unroll
  for (int k = 0; k < kCL / VEC; ++k) {
    const int vi = k * 32 + lane;
    if (vi * VEC < valid) {
      const float v = vec_max(st[vi], T{});
      if (v > m || v != v) {
        if (m == m) kbest = k;  // keep the first NaN, otherwise the first larger vector
        m = max_nan(m, v);
      }
    }
  }
  const float M = warp_max_nan(m);
  int first = INT_MAX;
  if (m == M && M > ninf) {  // only lanes that hold the maximum look at one vector
    const int vi = kbest * 32 + lane;
    float z[VEC];
    Elem<T>::unpack(st[vi], z);
#pragma unroll
    for (int e = VEC - 1; e >= 0; --e)
      if (z[e] == M) first = cbase + vi * VEC + e;
  }
  unsigned f;
  asm volatile("redux.sync.min.u32 %0, %1, 0xffffffff;" : "=r"(f) : "r"(static_cast<unsigned>(first)));
  return make_float2(M, __int_as_float(static_cast<int>(f)));
}

// Merge the chunk records of one row, v[k] = record lane + 32k (missing ones empty).
template <bool kSample>
__device__ __forceinline__ float2 merge_row_vals(const float2* v) {
  constexpr int NPL = kMaxChunkCount / 32;
  const float ninf = -__int_as_float(0x7f800000);
  float m = ninf;
#pragma unroll
  for (int k = 0; k < NPL; ++k) m = max_nan(m, v[k].x);
  const float M = warp_max_nan(m);
  if constexpr (kSample) {
    float s = 0.f;
#pragma unroll
    for (int k = 0; k < NPL; ++k)
      s = __fadd_rn(s, v[k].y == 0.f ? 0.f : __fmul_rn(v[k].y, ex2(__fsub_rn(v[k].x, M))));
    return make_float2(M, warp_sum(s));
  } else {
    unsigned first = 0xffffffffu;
#pragma unroll
    for (int k = 0; k < NPL; ++k)
      if (v[k].x == M) first = min(first, static_cast<unsigned>(__float_as_int(v[k].y)));
    unsigned f;
    asm volatile("redux.sync.min.u32 %0, %1, 0xffffffff;" : "=r"(f) : "r"(first));
    return make_float2(M, __int_as_float(static_cast<int>(f)));
  }
}

// ---------------------------------------------------------------------- output helpers

__device__ __forceinline__ bool stat_ok(float2 st) {
  return is_finite(st.x) && is_finite(st.y) && st.y > 0.f;
}

constexpr int kErrBits = DSPARK_SEQ_BAD_DRAFT | DSPARK_SEQ_NONFINITE | DSPARK_SEQ_TIMEOUT;

__device__ __forceinline__ void write_error(const TaskParams& p, int b, int status, int lane) {
  const int K = p.K;
  for (int t = lane; t <= K; t += 32) p.out.tokens[static_cast<size_t>(b) * (K + 1) + t] = -1;
  if (lane == 0) {
    p.out.n_accepted[b] = 0;
    p.out.next_token[b] = -1;
    if (p.out.status) p.out.status[b] = status;
    if (p.out.resid_mass) p.out.resid_mass[b] = __int_as_float(0x7fffffff);
  }
}

// Accepted drafts x_0..x_{j-1} and -1 after position j (the token at j is written later).
__device__ __forceinline__ void write_prefix(const TaskParams& p, int b, int j, int lane) {
  const int K = p.K;
  for (int t = lane; t <= K; t += 32)
    if (t != j)
      p.out.tokens[static_cast<size_t>(b) * (K + 1) + t] =
          t < j ? p.drafts[static_cast<size_t>(b) * K + t] : -1;
  if (lane == 0) p.out.n_accepted[b] = j;
}

__device__ __forceinline__ void reset_sequence(const TaskParams& p, int b, int lane) {
  if (lane == 0) {
    p.seq_cnt[b].streamed = 0;
    p.seq_cnt[b].decided = 0;
    p.seq_cnt[b].resid_done = 0;
  }
}

// DECIDE's first step: every row's statistics from the sequence's chunk records, into
// row_stat (global, for SAMPLE) and rs (this warp's shared-memory copy). The records of
// kRowBatch rows are loaded together, so the merge costs a couple of L2 round trips.
template <bool kSample>
__device__ __forceinline__ void merge_rows(const TaskParams& p, int b, int lane, float2* rs) {
  constexpr int NPL = kMaxChunkCount / 32;
  constexpr int kRowBatch = 4;
  const float ninf = -__int_as_float(0x7f800000);
  const float2 empty = make_float2(ninf, kSample ? 0.f : __int_as_float(INT_MAX));
  const float2* rec = p.chunk_stat + static_cast<size_t>(b) * p.rows * p.nch;
  for (int r0 = 0; r0 < p.rows; r0 += kRowBatch) {
    float2 v[kRowBatch][NPL];
#pragma unroll
    for (int rr = 0; rr < kRowBatch; ++rr) {
#pragma unroll
      for (int k = 0; k < NPL; ++k) {
        const int r = r0 + rr, c = lane + 32 * k;
        v[rr][k] = (r < p.rows && c < p.nch) ? ld_cg_f2(rec + static_cast<size_t>(r) * p.nch + c)
                                              : empty;
      }
    }
#pragma unroll
    for (int rr = 0; rr < kRowBatch; ++rr) {
      const float2 st = merge_row_vals<kSample>(v[rr]);
      if (lane == 0 && r0 + rr < p.rows) {
        rs[r0 + rr] = st;
        p.row_stat[static_cast<size_t>(b) * p.rows + r0 + rr] = st;
      }
    }
  }
  __syncwarp();
}

// ---------------------------------------------------------------------- DECIDE tasks

__device__ __forceinline__ void decide_greedy(const TaskParams& p, int b, int lane, bool ok_wait,
                                              int x, const float2* rs) {
  const int K = p.K, K1 = K + 1;
  const float ninf = -__int_as_float(0x7f800000);
  int status = ok_wait ? 0 : DSPARK_SEQ_TIMEOUT;
  float2 a = make_float2(0.f, 0.f);
  if (lane < K1) a = rs[lane];
  const int arg = __float_as_int(a.y);
  // NaN anywhere, a +inf maximum, or nothing above -inf: not a usable row
  const bool bad = lane < K1 && (!(a.x > ninf) || !(a.x < -ninf) || arg == INT_MAX);
  if (__any_sync(0xffffffffu, bad)) status |= DSPARK_SEQ_NONFINITE;
  if (__any_sync(0xffffffffu, lane < K && (x < 0 || x >= p.V))) status |= DSPARK_SEQ_BAD_DRAFT;
  const unsigned mis = __ballot_sync(0xffffffffu, lane < K && x != arg);
  const int j = mis ? __ffs(mis) - 1 : K;
  const int token = __shfl_sync(0xffffffffu, arg, j);
  if (status & kErrBits) {
    write_error(p, b, status, lane);
  } else {
    write_prefix(p, b, j, lane);
    if (lane == 0) {
      p.out.tokens[static_cast<size_t>(b) * K1 + j] = token;
      p.out.next_token[b] = token;
      if (p.out.status) p.out.status[b] = 0;
    }
  }
  __syncwarp();
  reset_sequence(p, b, lane);
}

__device__ __forceinline__ void decide_sample(const TaskParams& p, int b, int lane, bool ok_wait,
                                              int x, float zpx, float zqx, float ui,
                                              const float2* rs) {
  const int K = p.K, K1 = K + 1;
  const float fnan = __int_as_float(0x7fffffff);
  int status = ok_wait ? 0 : DSPARK_SEQ_TIMEOUT;
  bool accept = false;
  float px = fnan, qx = fnan;
  // row statistics: P rows on lanes 0..K, Q rows on lanes 0..K-1
  float2 sp = make_float2(0.f, 1.f), sq = make_float2(0.f, 1.f);
  if (lane < K1) sp = rs[lane];
  if (lane < K) sq = rs[K1 + lane];
  const bool bad = (lane < K1 && !stat_ok(sp)) || (lane < K && !stat_ok(sq));
  if (__any_sync(0xffffffffu, bad)) status |= DSPARK_SEQ_NONFINITE;
  const bool bad_draft = lane < K && (x < 0 || x >= p.V);
  if (__any_sync(0xffffffffu, bad_draft)) status |= DSPARK_SEQ_BAD_DRAFT;
  if (lane < K && !bad_draft) {
    px = __fdiv_rn(ex2(__fmaf_rn(zpx, p.scale, -sp.x)), sp.y);
    qx = __fdiv_rn(ex2(__fmaf_rn(zqx, p.scale, -sq.x)), sq.y);
    accept = __fmul_rn(ui, qx) < px;
  }
  if (lane < K) {
    if (p.out.p_draft) p.out.p_draft[static_cast<size_t>(b) * K + lane] = px;
    if (p.out.q_draft) p.out.q_draft[static_cast<size_t>(b) * K + lane] = qx;
  }
  const unsigned rej = __ballot_sync(0xffffffffu, lane < K && !accept);
  const int j = rej ? __ffs(rej) - 1 : K;
  const float mpj = __shfl_sync(0xffffffffu, sp.x, j), spj = __shfl_sync(0xffffffffu, sp.y, j);
  const float mqj = __shfl_sync(0xffffffffu, sq.x, j), sqj = __shfl_sync(0xffffffffu, sq.y, j);
  if (status & kErrBits) {
    write_error(p, b, status, lane);
  } else {
    write_prefix(p, b, j, lane);
  }
  if (lane == 0) {
    SeqDecision d;
    d.j = j;
    d.status = status;
    d.mp = mpj;
    d.ip = __fdiv_rn(1.f, spj);
    d.mq = mqj;
    d.iq = j < K ? __fdiv_rn(1.f, sqj) : 0.f;
    d.pad0 = d.pad1 = 0;
    p.dec[b] = d;
  }
  __syncwarp();
  if (lane == 0) st_release_gpu(&p.seq_cnt[b].decided, 1u);
}

// ---------------------------------------------------------------------- RESID / SAMPLE

// Per-token mass of the draw's law with the row normalisers of DECIDE. RESID and SAMPLE use
// exactly this arithmetic, so the chunk SAMPLE re-reads reproduces RESID's values bit for bit.
__device__ __forceinline__ float resid_value(float zp, float zq, float s, const SeqDecision& d) {
  const float ep = ex2(__fmaf_rn(zp, s, -d.mp));
  const float eq = ex2(__fmaf_rn(zq, s, -d.mq));
  return fmaxf(__fmaf_rn(ep, d.ip, -__fmul_rn(eq, d.iq)), 0.f);
}
__device__ __forceinline__ float p_value(float zp, float s, const SeqDecision& d) {
  return __fmul_rn(ex2(__fmaf_rn(zp, s, -d.mp)), d.ip);
}

template <typename T, int VEC>
__device__ __forceinline__ void resid_task(const TaskParams& p, int b, int g, int lane, bool ok_wait) {
  const SeqDecision d = load_decision(p.dec + b);
  const bool active = ok_wait && d.j < p.K && !(d.status & kErrBits);
  const int c_end = min(p.nch, (g + 1) * kResidGroup);
  for (int c = g * kResidGroup; c < c_end; ++c) {
    float mass = 0.f;
    if (active) {
      const int cbase = c * kCE;
      const int valid = min(kCE, p.V - cbase);
      const T* pr = row_ptr<T>(p, b, d.j) + cbase;
      const T* qr = row_ptr<T>(p, b, p.K + 1 + d.j) + cbase;
      float acc = 0.f;
      constexpr int NV = kCL / VEC;
      if constexpr (VEC == 1) {
#pragma unroll 4
        for (int k = 0; k < NV; ++k) {
          float zp, zq;
          lane_vec<T, 1>(pr, valid, k, lane, &zp);
          lane_vec<T, 1>(qr, valid, k, lane, &zq);
          acc = __fadd_rn(acc, resid_value(zp, zq, p.scale, d));
        }
      } else {
        // all raw vectors of both rows in flight at once, unpacked one vector at a time
        uint4 rp[NV], rq[NV];
#pragma unroll
        for (int k = 0; k < NV; ++k) {
          rp[k] = lane_raw<T>(pr, valid, k, lane);
          rq[k] = lane_raw<T>(qr, valid, k, lane);
        }
#pragma unroll
        for (int k = 0; k < NV; ++k) {
          float zp[VEC], zq[VEC];
          Elem<T>::unpack(rp[k], zp);
          Elem<T>::unpack(rq[k], zq);
#pragma unroll
          for (int e = 0; e < VEC; ++e) acc = __fadd_rn(acc, resid_value(zp[e], zq[e], p.scale, d));
        }
      }
      mass = warp_sum(acc);
    } else if (!ok_wait) {
      mass = __int_as_float(0x7fffffff);
    }
    if (lane == 0) p.resid_mass[static_cast<size_t>(b) * p.nch + c] = mass;
  }
  __syncwarp();
  if (lane == 0) red_release_gpu(&p.seq_cnt[b].resid_done, 1u);
}

template <typename T, int VEC>
__device__ __forceinline__ void sample_task(const TaskParams& p, int b, int lane, bool ok_wait) {
  const int K = p.K, K1 = K + 1, nch = p.nch;
  const SeqDecision d = load_decision(p.dec + b);
  int status = d.status | (ok_wait ? 0 : DSPARK_SEQ_TIMEOUT);
  if (status & kErrBits) {
    write_error(p, b, status, lane);
    __syncwarp();
    reset_sequence(p, b, lane);
    return;
  }
  const int j = d.j;
  const float uK = p.uniforms[static_cast<size_t>(b) * K1 + K];
  bool resid = j < K;
  const int jrow = resid ? j : K;
  // chunk masses of the draw's law in float64; lane l holds chunks l*NPL .. l*NPL+NPL-1, so a
  // prefix over lanes is a prefix in token order
  constexpr int NPL = kMaxChunkCount / 32;
  double Zres = 0.0;
  int token = -1;
  for (int attempt = 0; attempt < 2; ++attempt) {
    double m[NPL];
#pragma unroll
    for (int k = 0; k < NPL; ++k) {
      const int c = lane * NPL + k;
      double v = 0.0;
      if (c < nch) {
        if (resid) {
          v = static_cast<double>(ld_cg_f(p.resid_mass + static_cast<size_t>(b) * nch + c));
        } else {
          const float2 r =
              ld_cg_f2(p.chunk_stat + (static_cast<size_t>(b) * p.rows + jrow) * nch + c);
          v = r.y == 0.f
                  ? 0.0
                  : static_cast<double>(__fmul_rn(__fmul_rn(r.y, ex2(__fsub_rn(r.x, d.mp))), d.ip));
        }
      }
      m[k] = v;
    }
    double ls = 0.0;
#pragma unroll
    for (int k = 0; k < NPL; ++k) ls += m[k];
    double incl = ls;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const double y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    const double Z = __shfl_sync(0xffffffffu, incl, 31);
    if (attempt == 0) Zres = Z;
    if (resid && !(Z > 0.0)) {
      resid = false;  // residual mass rounded to zero: draw from p_j instead
      status |= DSPARK_SEQ_ZERO_RESIDUAL;
      continue;
    }
    // the chunk holding the target
    const double target = static_cast<double>(uK) * Z;
    double run = incl - ls;
    int cfound = -1, clast = -1;
    double before = 0.0;
#pragma unroll
    for (int k = 0; k < NPL; ++k) {
      const double nxt = run + m[k];
      if (m[k] > 0.0) {
        clast = lane * NPL + k;
        if (cfound < 0 && run <= target && target < nxt) {
          cfound = lane * NPL + k;
          before = run;
        }
      }
      run = nxt;
    }
    const unsigned hit = __ballot_sync(0xffffffffu, cfound >= 0);
    int c;
    float tin;
    if (hit) {
      const int hl = __ffs(hit) - 1;
      c = __shfl_sync(0xffffffffu, cfound, hl);
      tin = static_cast<float>(target - __shfl_sync(0xffffffffu, before, hl));
    } else {  // rounding left the target past the last mass: take the last token
      int cl = clast;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) cl = max(cl, __shfl_xor_sync(0xffffffffu, cl, o));
      c = cl;
      tin = __int_as_float(0x7f800000);
    }
    // the chunk: recompute per-token masses exactly as RESID did, scan in token order
    // (vector kv of every lane, lanes in order, then vector kv+1)
    if (c >= 0) {
      constexpr int NV = kCL / VEC;
      const int cbase = c * kCE;
      const int valid = min(kCE, p.V - cbase);
      const T* pr = row_ptr<T>(p, b, jrow) + cbase;
      const T* qr = resid ? row_ptr<T>(p, b, K1 + j) + cbase : pr;
      // the lane's vectors of both rows, half a chunk in flight at a time
      constexpr int kHalf = NV > 1 ? NV / 2 : 1;
      float carry = 0.f;
      int lastpos = -1;
#pragma unroll
      for (int h0 = 0; h0 < NV; h0 += kHalf) {
        float zp[kHalf * VEC], zq[kHalf * VEC];
#pragma unroll
        for (int kk = 0; kk < kHalf; ++kk) {
          lane_vec<T, VEC>(pr, valid, h0 + kk, lane, zp + kk * VEC);
          if (resid) lane_vec<T, VEC>(qr, valid, h0 + kk, lane, zq + kk * VEC);
        }
#pragma unroll
        for (int kk = 0; kk < kHalf; ++kk) {
          const int kv = h0 + kk;
          float val[VEC];
          float lsum = 0.f;
#pragma unroll
          for (int e = 0; e < VEC; ++e) {
            val[e] = resid ? resid_value(zp[kk * VEC + e], zq[kk * VEC + e], p.scale, d)
                           : p_value(zp[kk * VEC + e], p.scale, d);
            if (val[e] > 0.f) lastpos = max(lastpos, cbase + (kv * 32 + lane) * VEC + e);
            lsum = __fadd_rn(lsum, val[e]);
          }
          float inc = lsum;
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const float y = __shfl_up_sync(0xffffffffu, inc, o);
            if (lane >= o) inc = __fadd_rn(inc, y);
          }
          float ex = __shfl_up_sync(0xffffffffu, inc, 1);
          if (lane == 0) ex = 0.f;
          const float bef = __fadd_rn(carry, ex);
          const float aft = __fadd_rn(carry, inc);
          const unsigned h = __ballot_sync(0xffffffffu, token < 0 && bef <= tin && tin < aft);
          if (h) {
            const int hl = __ffs(h) - 1;
            int cand = -1;
            if (lane == hl) {
              float r = bef;
              int lastv = -1;
#pragma unroll
              for (int e = 0; e < VEC; ++e) {
                const float nx = __fadd_rn(r, val[e]);
                const int id = cbase + (kv * 32 + lane) * VEC + e;
                if (val[e] > 0.f) lastv = id;
                if (cand < 0 && r <= tin && tin < nx) cand = id;
                r = nx;
              }
              if (cand < 0) cand = lastv;
            }
            token = __shfl_sync(0xffffffffu, cand, hl);
          }
          carry = __shfl_sync(0xffffffffu, aft, 31);
        }
      }
      if (token < 0) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
          lastpos = max(lastpos, __shfl_xor_sync(0xffffffffu, lastpos, o));
        token = lastpos;
      }
    }
    break;
  }
  if (lane == 0) {
    p.out.tokens[static_cast<size_t>(b) * K1 + j] = token;
    p.out.next_token[b] = token;
    if (p.out.status) p.out.status[b] = status;
    if (p.out.resid_mass) p.out.resid_mass[b] = j < K ? static_cast<float>(Zres) : 1.0f;
  }
  __syncwarp();
  reset_sequence(p, b, lane);
}

// ------------------------------------------------------------------------- the kernel

template <typename T, int VEC, bool kSample, bool kTma>
__device__ __forceinline__ void stream_warp(const TaskParams& p, unsigned char* ring, uint64_t* full,
                                            int sw, int lane) {
  constexpr int EB = Elem<T>::kBytes;
  constexpr uint32_t kChunkBytes = kCE * EB;
  const int S = p.stages;
  const long long N = p.stream_warps;
  StreamStep step;
  step.rows = p.rows;
  step.nch = p.nch;
  const long long per_b = static_cast<long long>(p.rows) * p.nch;
  step.qb = static_cast<int>(N / per_b);
  step.qr = static_cast<int>((N - step.qb * per_b) / p.nch);
  step.qc = static_cast<int>(N - step.qb * per_b - static_cast<long long>(step.qr) * p.nch);
  StreamPos start;
  start.s = sw;
  start.b = static_cast<int>(sw / per_b);
  start.r = static_cast<int>((sw - start.b * per_b) / p.nch);
  start.c = static_cast<int>(sw - start.b * per_b - static_cast<long long>(start.r) * p.nch);

  if constexpr (kTma) {
    if (lane == 0) {
      for (int s = 0; s < S; ++s) mbar_init(&full[s], 1);
      fence_mbar_init();
    }
    __syncwarp();
  }
  // Producer (lane 0): copies this warp's next STREAM chunks ahead into the ring.
  StreamPos prod = start;
  int pstage = 0, in_flight = 0;
  bool dead = false;
  auto produce = [&]() {
    while (in_flight < S && prod.s < p.n_stream) {
      const int cbase = prod.c * kCE;
      const uint32_t bytes = static_cast<uint32_t>(min(kCE, p.V - cbase)) * EB;
      uint64_t* bar = &full[pstage];
      mbar_arrive_expect_tx(bar, bytes);
      bulk_g2s(ring + static_cast<size_t>(pstage) * kChunkBytes, row_ptr<T>(p, prod.b, prod.r) + cbase,
               bytes, bar);
      step.advance(prod, N);
      if (++pstage == S) pstage = 0;
      ++in_flight;
    }
  };
  if constexpr (kTma) {
    if (lane == 0) produce();
  }

  // Records stored but not yet counted: up to kPubBatch of them are counted together after a
  // single release fence (fence.acq_rel.gpu, then relaxed adds), which is what a release
  // costs. Kept in lane kPubLane, which stores the records, and never lane 0, whose bulk
  // copies are in flight.
  int pend[kPubBatch];
  int npend = 0;
  auto publish = [&]() {
    if (lane == kPubLane && npend > 0) {
      fence_acq_rel_gpu();
      for (int i = 0; i < npend; ++i) red_relaxed_gpu(&p.seq_cnt[pend[i]].streamed, 1u);
    }
    npend = 0;
  };
  int cstage = 0;
  uint32_t cphase = 0;
  for (StreamPos sp = start; sp.s < p.n_stream; step.advance(sp, N)) {
    const int cbase = sp.c * kCE;
    const int valid = min(kCE, p.V - cbase);
    float2 rec;
    if constexpr (kTma) {
      if (!dead) dead = !mbar_wait_bounded(&full[cstage], cphase);
      dead = __any_sync(0xffffffffu, dead);
      const unsigned char* stage = ring + static_cast<size_t>(cstage) * kChunkBytes;
      if constexpr (kSample) {
        rec = stream_softmax_part_smem<T>(stage, valid, lane, p.scale);
      } else {
        rec = stream_argmax_part_smem<T>(stage, valid, cbase, lane);
      }
      if (++cstage == S) {
        cstage = 0;
        cphase ^= 1u;
      }
      // Every value read from the stage has been consumed above (it fed the warp-wide
      // reductions), so the stage can be refilled.
      __syncwarp();
      if (lane == 0 && !dead) {
        --in_flight;
        produce();
      }
      if (dead) rec = make_float2(__int_as_float(0x7fffffff), __int_as_float(0x7fffffff));
    } else {
      float z[kCL];
      chunk_lane_values<T, VEC>(row_ptr<T>(p, sp.b, sp.r) + cbase, valid, lane, z);
      if constexpr (kSample) {
        rec = stream_softmax_part(z, p.scale);
      } else {
        rec = stream_argmax_part<VEC>(z, cbase, lane);
      }
    }
    if (lane == kPubLane) p.chunk_stat[(static_cast<size_t>(sp.b) * p.rows + sp.r) * p.nch + sp.c] = rec;
    pend[npend++] = sp.b;
    if (npend == kPubBatch) publish();
  }
  publish();

  if constexpr (kTma) {
    // Never leave with bulk copies in flight into this warp's stages.
    if (lane == 0 && in_flight > 0) {
      for (int n = 0; n < in_flight; ++n) {
        (void)mbar_wait_bounded(&full[cstage], cphase);
        if (++cstage == S) {
          cstage = 0;
          cphase ^= 1u;
        }
      }
    }
    __syncwarp();
  }
}

// Dependent tasks are handed out in order from one queue: task d = b * n_dep_per_seq + k,
// k == 0 DECIDE(b), 1 <= k <= n_resid RESID(b, k - 1), k == n_resid + 1 SAMPLE(b).
template <typename T, int VEC, bool kSample>
__device__ __forceinline__ void dependent_warp(const TaskParams& p, float2* rs, int lane) {
  const int K = p.K;
  const unsigned total = static_cast<unsigned>(p.B) * static_cast<unsigned>(p.n_dep_per_seq);
  const unsigned stream_target = static_cast<unsigned>(p.rows * p.nch);
  for (;;) {
    unsigned d = 0;
    if (lane == 0) d = atomicAdd(&p.dq->next, 1u);
    d = __shfl_sync(0xffffffffu, d, 0);
    if (d >= total) break;
    const int b = static_cast<int>(d / static_cast<unsigned>(p.n_dep_per_seq));
    const int k = static_cast<int>(d - static_cast<unsigned>(b) * p.n_dep_per_seq);
    if (k == 0) {
      // the inputs first: they do not depend on other tasks
      int x = 0;
      if (lane < K) x = p.drafts[static_cast<size_t>(b) * K + lane];
      if constexpr (kSample) {
        float zpx = 0.f, zqx = 0.f, ui = 0.f;
        if (lane < K) {
          if (x >= 0 && x < p.V) {
            zpx = Elem<T>::load1(row_ptr<T>(p, b, lane) + x);
            zqx = Elem<T>::load1(row_ptr<T>(p, b, K + 1 + lane) + x);
          }
          ui = p.uniforms[static_cast<size_t>(b) * (K + 1) + lane];
        }
        const bool ok = wait_counter(&p.seq_cnt[b].streamed, stream_target);
        merge_rows<true>(p, b, lane, rs);
        decide_sample(p, b, lane, ok, x, zpx, zqx, ui, rs);
      } else {
        const bool ok = wait_counter(&p.seq_cnt[b].streamed, stream_target);
        merge_rows<false>(p, b, lane, rs);
        decide_greedy(p, b, lane, ok, x, rs);
      }
    } else if constexpr (kSample) {
      if (k <= p.n_resid) {
        const bool ok = wait_counter(&p.seq_cnt[b].decided, 1u);
        resid_task<T, VEC>(p, b, k - 1, lane, ok);
      } else {
        const bool ok = wait_counter(&p.seq_cnt[b].resid_done, static_cast<unsigned>(p.n_resid));
        sample_task<T, VEC>(p, b, lane, ok);
      }
    }
  }
  // the last dependent warp to leave resets the queue for the next call
  if (lane == 0) {
    const unsigned e = atomicAdd(&p.dq->exited, 1u);
    if (e == static_cast<unsigned>(p.dep_warps - 1)) {
      p.dq->next = 0;
      p.dq->exited = 0;
    }
  }
}

template <typename T, int VEC, bool kSample, bool kTma>
__global__ void __launch_bounds__(kTaskThreads, 2) verify_tasks_kernel(const TaskParams p) {
  extern __shared__ __align__(128) unsigned char smem[];
  constexpr int EB = Elem<T>::kBytes;
  constexpr uint32_t kChunkBytes = kCE * EB;
  __shared__ float2 s_rows[kMaxRows];  // the dependent warp's row statistics
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (warp < kStreamWarps) {
    const int S = p.stages;
    unsigned char* ring = smem + static_cast<size_t>(warp) * S * kChunkBytes;
    uint64_t* full =
        reinterpret_cast<uint64_t*>(smem + static_cast<size_t>(kStreamWarps) * S * kChunkBytes) +
        warp * kMaxTaskStages;
    stream_warp<T, VEC, kSample, kTma>(p, ring, full, blockIdx.x * kStreamWarps + warp, lane);
  } else {
    dependent_warp<T, VEC, kSample>(p, s_rows, lane);
  }
}

}  // namespace dspark
