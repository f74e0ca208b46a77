// Pass 2 of the verify step: per-sequence decisions and the correction / bonus draw.
//
// Greedy: one CTA per sequence merges the pass-1 argmax records of its K+1 rows (a warp per
// row), compares the drafts with the row argmaxes and writes the AcceptResult.
//
// Sampling: one thread-block cluster of G = ceil(n_chunks / 32) CTAs of 32 warps per sequence
// (2 for V = 129280, at most 4), one CTA per SM; batches whose clusters of 16-warp CTAs
// (ceil(n_chunks / 16) per sequence) fit on the SMs take those, which spread a sequence's
// chunks over twice the SMs and load each chunk in one round. Small clusters of whole-SM CTAs
// are placed at once: with 8-CTA clusters of 8-warp CTAs the GPU left a cluster unplaced until others had
// finished (the clusters must fit in a GPC). Every CTA merges the 2K+1 rows' softmax records
// and takes the accept decisions (the same inputs and arithmetic in each, so the same j);
// after the early-exit waves it loads the decision they stored instead. Each warp then
// computes one 2048-token chunk of the draw's law, r = max(p_j - q_j, 0) after a rejection
// (j < K), p_K for the bonus (j = K), keeping the sums of every 8-token group in shared
// memory and sending the chunk's mass to every CTA of the cluster (distributed shared memory).
// After one cluster barrier every CTA locates the chunk that holds the draw (float64 prefix
// over the chunk masses); its owner finds the group from its group sums, re-reads that
// group's 8 tokens and scans them.
//
// Both kernels start with the loads that do not depend on pass 1 (drafts, uniforms) and then
// wait for pass 1 to complete (programmatic dependent launch).
#pragma once

#include "stream.cuh"

namespace dspark {

constexpr int kErrBits =
    DSPARK_SEQ_BAD_DRAFT | DSPARK_SEQ_NONFINITE | DSPARK_SEQ_TIMEOUT | DSPARK_SEQ_BAD_PARAM;
constexpr int kMaxRows = 2 * kMaxK + 1;
constexpr int kFinWarps = 32;       // warps per sampling-finish CTA: one chunk each
constexpr int kFinWarpsSmall = 16;  // the same for small batches, 128 registers per thread
constexpr int kFinMaxCpc = 32;      // chunks per finish CTA at most
constexpr int kPlanSMs = 148;       // SMs of a B200: the small-batch layout while B * G fits

// Kernel parameters (see StreamParamsMixed on their size). The sampling kernel's cluster size
// G and chunks per CTA, ceil(n_chunks / G), come from its launch.
struct FinishParams {
  RowSet rs;
  const int32_t* drafts;    // [B, K]
  const float* uniforms;    // [B, K+1] (sampling)
  int nch;                  // chunks per row
  float scale;              // log2(e) / T
  const float2* rec;        // pass-1 records [B * rows, nch]
  const float* gather;      // [B, K, 2]: P_i[x_i], Q_i[x_i] written by pass 1 (sampling)
  dspark_accept_out_t out;
};

// A mixed batch's per-sequence arrays, kept out of FinishParams for the reason given at
// StreamParamsMixed.
struct FinishParamsMixed : FinishParams {
  const int32_t* n_drafts;  // [B] K_b, or null for K
  const float* temps;       // [B] T_b
};

// The pass-1 records of one row, held by one warp: chunk lane + 32k. Missing ones are empty.
constexpr int kRecPerLane = kMaxChunkCount / 32;
struct RowRecs {
  float2 v[kRecPerLane];
};

template <bool kSample>
__device__ __forceinline__ void load_row(const FinishParams& p, long long r, int lane,
                                         RowRecs& rr) {
  const float2* rec = p.rec + r * p.nch;
  const float2 empty =
      make_float2(-__int_as_float(0x7f800000), kSample ? 0.f : __int_as_float(INT_MAX));
#pragma unroll
  for (int k = 0; k < kRecPerLane; ++k) {
    const int c = lane + 32 * k;
    rr.v[k] = c < p.nch ? __ldcg(rec + c) : empty;
  }
}

// Merge a row's records (every lane gets the result). Sampling: (M, S) with M the largest
// reference and S the sum rescaled to it. Greedy: (max, lowest index of the max).
template <bool kSample>
__device__ __forceinline__ float2 reduce_row(const RowRecs& rr) {
  float m = -__int_as_float(0x7f800000);
#pragma unroll
  for (int k = 0; k < kRecPerLane; ++k) m = max_nan(m, rr.v[k].x);
  const float M = warp_max_nan(m);
  if constexpr (kSample) {
    float s = 0.f;
#pragma unroll
    for (int k = 0; k < kRecPerLane; ++k)
      s = __fadd_rn(s, rr.v[k].y == 0.f ? 0.f : __fmul_rn(rr.v[k].y, ex2(__fsub_rn(rr.v[k].x, M))));
    return make_float2(M, warp_sum(s));
  } else {
    unsigned first = 0xffffffffu;
#pragma unroll
    for (int k = 0; k < kRecPerLane; ++k)
      if (rr.v[k].x == M) first = min(first, static_cast<unsigned>(__float_as_int(rr.v[k].y)));
    unsigned f;
    asm volatile("redux.sync.min.u32 %0, %1, 0xffffffff;" : "=r"(f) : "r"(first));
    return make_float2(M, __int_as_float(static_cast<int>(f)));
  }
}

// The rows of sequence b into s_stat (row r at s_stat[r]): all of them, or with kFiltered
// those that `used` selects. Warp w of kW merges rows w, w + kW, ..., two at a time so that
// their loads overlap.
template <bool kSample, bool kFiltered, int kW = kWarps, class Filter = RowFilter>
__device__ __forceinline__ void merge_rows(const FinishParams& p, int b, const Filter& used,
                                           int wi, int lane, float2* s_stat) {
  const int rows = p.rs.rows;
  const long long r0 = static_cast<long long>(b) * rows;
  for (int r = wi; r < rows; r += 2 * kW) {
    RowRecs a, c;
    const bool one = !kFiltered || used(r);
    const bool two = r + kW < rows && (!kFiltered || used(r + kW));
    if (one) load_row<kSample>(p, r0 + r, lane, a);
    if (two) load_row<kSample>(p, r0 + r + kW, lane, c);
    if (one) {
      const float2 sa = reduce_row<kSample>(a);
      if (lane == 0) s_stat[r] = sa;
    }
    if (two) {
      const float2 sc = reduce_row<kSample>(c);
      if (lane == 0) s_stat[r + kW] = sc;
    }
  }
}

__device__ __forceinline__ bool stat_ok(float2 st) {
  return is_finite(st.x) && is_finite(st.y) && st.y > 0.f;
}

// Error result: n = 0, tokens all -1, next -1, the cause in status.
__device__ __forceinline__ void write_error(const FinishParams& p, int b, int status, int t,
                                            int nt) {
  const int K1 = p.rs.K + 1;
  for (int k = t; k < K1; k += nt) p.out.tokens[static_cast<size_t>(b) * K1 + k] = -1;
  if (t == 0) {
    p.out.n_accepted[b] = 0;
    p.out.next_token[b] = -1;
    if (p.out.status) p.out.status[b] = status;
    if (p.out.resid_mass) p.out.resid_mass[b] = __int_as_float(0x7fffffff);
  }
}

// x_0..x_{j-1} (from the shared-memory copy xs of the drafts), then `token` at j, then -1.
__device__ __forceinline__ void write_tokens(const FinishParams& p, int b, int j, int token,
                                             const int* xs, int t, int nt) {
  const int K1 = p.rs.K + 1;
  for (int k = t; k < K1; k += nt)
    p.out.tokens[static_cast<size_t>(b) * K1 + k] = k < j ? xs[k] : (k == j ? token : -1);
  if (t == 0) {
    p.out.n_accepted[b] = j;
    p.out.next_token[b] = token;
  }
}

// ------------------------------------------------------------------------------ greedy

// Greedy finish of sequence b with nd drafts (every thread of the CTA; its P rows 0..nd are
// merged): x = drafts[b, lane] in warp 0's lanes below nd, already copied to s_x. kFiltered:
// the records are laid out for sampling rows (a mixed batch) and rows past nd are skipped.
template <bool kFiltered, int kW = kWarps>
__device__ __forceinline__ void greedy_finish(const FinishParams& p, int b, int nd, int x, int wi,
                                              int lane, float2* s_arg, const int* s_x) {
  merge_rows<false, kFiltered, kW>(p, b, RowFilter{p.rs.K, nd, false}, wi, lane, s_arg);
  __syncthreads();
  if (wi != 0) return;
  const float ninf = -__int_as_float(0x7f800000);
  bool bad = false;
  for (int r = lane; r <= nd; r += 32) {
    const float2 a = s_arg[r];
    // NaN anywhere, a +inf maximum, or nothing above -inf: not a usable row
    bad |= !(a.x > ninf) || !(a.x < -ninf) || __float_as_int(a.y) == INT_MAX;
  }
  int status = __any_sync(0xffffffffu, bad) ? DSPARK_SEQ_NONFINITE : 0;
  if (__any_sync(0xffffffffu, lane < nd && (x < 0 || x >= p.rs.V))) status |= DSPARK_SEQ_BAD_DRAFT;
  const int arg = lane < nd ? __float_as_int(s_arg[lane].y) : -1;
  const unsigned mis = __ballot_sync(0xffffffffu, lane < nd && x != arg);
  const int j = mis ? __ffs(mis) - 1 : nd;
  if (status & kErrBits) {
    write_error(p, b, status, lane, 32);
    return;
  }
  write_tokens(p, b, j, __float_as_int(s_arg[j].y), s_x, lane, 32);
  if (lane == 0 && p.out.status) p.out.status[b] = 0;
}

template <typename T>
__global__ void __launch_bounds__(kThreads) finish_greedy_kernel(const FinishParams p) {
  __shared__ float2 s_arg[kMaxK + 1];
  __shared__ int s_x[kMaxK];
  // the next kernel in the stream may be scheduled as these CTAs retire (it waits for them)
  grid_dependents_launch();
  const int lane = threadIdx.x & 31, wi = threadIdx.x >> 5;
  const int b = blockIdx.x;
  const int K = p.rs.K;
  int x = 0;
  if (wi == 0 && lane < K) {
    x = p.drafts[static_cast<size_t>(b) * K + lane];
    s_x[lane] = x;
  }
  grid_dependency_wait();
  greedy_finish<false>(p, b, K, x, wi, lane, s_arg, s_x);
}

// ---------------------------------------------------------------------------- sampling

// The row normalisers of the draw's law, and the decision.
struct Decision {
  int j;
  int nd;  // the sequence's draft count: j < nd is a rejection, j == nd the bonus
  int status;
  float mp, ip;  // p_j (or p_K): reference and 1 / sum
  float mq, iq;  // q_j: reference and 1 / sum (iq = 0 for the bonus)
};

// The values of the draw's law at a group's 8 tokens, in token order. The group sums, the chunk
// masses and the draw's scan all come from exactly these values, so the scan reproduces the
// sums it located:
//   p value:        p_j(v) = 2^(z_p[v]*s - m_p) * (1 / S_p)
//   residual value: max(p_j(v) - q_j(v), 0), rounded as fma(e_p, 1/S_p, -(e_q * (1/S_q)))
// (the residual equals p on the bonus row, which has no q). Pairs of tokens share one packed
// f32x2 instruction where the arithmetic allows; each half rounds like the scalar operation.
template <bool kResid>
__device__ __forceinline__ void law_values(const float* zp, const float* zq, float s,
                                           const Decision& d, float* out) {
  const uint64_t s2 = pk2(s, s);
  const uint64_t nmp = pk2(-d.mp, -d.mp), ip = pk2(d.ip, d.ip);
#pragma unroll
  for (int e = 0; e < 8; e += 2) {
    float a0, a1;
    upk2(fma2(pk2(zp[e], zp[e + 1]), s2, nmp), a0, a1);
    const uint64_t ep = pk2(ex2(a0), ex2(a1));
    if constexpr (kResid) {
      float c0, c1;
      upk2(fma2(pk2(zq[e], zq[e + 1]), s2, pk2(-d.mq, -d.mq)), c0, c1);
      const uint64_t neq = mul2(pk2(ex2(c0), ex2(c1)), pk2(-d.iq, -d.iq));
      float r0, r1;
      upk2(fma2(ep, ip, neq), r0, r1);
      out[e] = fmaxf(r0, 0.f);
      out[e + 1] = fmaxf(r1, 0.f);
    } else {
      upk2(mul2(ep, ip), out[e], out[e + 1]);
    }
  }
}

// A group: 8 consecutive tokens 8q .. 8q+7 of a chunk (q = 0..255). Lane l of a warp handles
// groups q = l + 32k, k = 0..7, so a round of loads is coalesced across the warp.
constexpr int kGroups = kCE / 8;

// The 8 logits of a group of one row (t0 = first token, a multiple of 8); -inf past V.
template <typename T, int VEC>
struct GroupRaw {
  static constexpr int NW = VEC == 1 ? 1 : 8 / VEC;
  uint4 w[NW];   // vector path: raw words
  float z[VEC == 1 ? 8 : 1];  // scalar path: values
  __device__ __forceinline__ void load(const T* row, int t0, int V) {
    const float ninf = -__int_as_float(0x7f800000);
    if constexpr (VEC == 1) {
#pragma unroll
      for (int e = 0; e < 8; ++e) z[e] = t0 + e < V ? Elem<T>::load1(row + t0 + e) : ninf;
    } else {
      const uint32_t nb = Elem<T>::kBytes == 2 ? 0xff80ff80u : 0xff800000u;
#pragma unroll
      for (int h = 0; h < NW; ++h)
        w[h] = t0 + h * VEC < V ? ld_stream16(row + t0 + h * VEC) : make_uint4(nb, nb, nb, nb);
    }
  }
  __device__ __forceinline__ void values(float* out) const {
    if constexpr (VEC == 1) {
#pragma unroll
      for (int e = 0; e < 8; ++e) out[e] = z[e];
    } else {
#pragma unroll
      for (int h = 0; h < NW; ++h) Elem<T>::unpack(w[h], out + h * VEC);
    }
  }
};

// The law's values at a group's 8 tokens (residual when kResid, else p), in token order.
template <typename T, int VEC, bool kResid>
__device__ __forceinline__ void group_values(const GroupRaw<T, VEC>& gp, const GroupRaw<T, VEC>& gq,
                                             float s, const Decision& d, float* v) {
  float zp[8], zq[8];
  gp.values(zp);
  if constexpr (kResid) gq.values(zq);
  law_values<kResid>(zp, zq, s, d, v);
}

// Sum of a group's 8 law values in token order.
template <typename T, int VEC, bool kResid>
__device__ __forceinline__ float group_sum(const GroupRaw<T, VEC>& gp, const GroupRaw<T, VEC>& gq,
                                           float s, const Decision& d) {
  float v[8];
  group_values<T, VEC, kResid>(gp, gq, s, d, v);
  float acc = 0.f;
#pragma unroll
  for (int e = 0; e < 8; ++e) acc = __fadd_rn(acc, v[e]);
  return acc;
}

// Chunk c of the draw's law (kResid: the residual of row pair j, else p of row j), one warp:
// the 256 group sums into part (token order) and the chunk's mass on every lane. Out of line:
// its registers are allocated apart from the kernel's (the finish has several call sites).
template <typename T, int VEC, bool kResid, bool kWide = false>
__device__ __forceinline__ float chunk_work(const RowSet& rs, float scale, int b, int c,
                                            const Decision& d, int lane, float* part) {
  const int K = rs.K, V = rs.V;
  const T* pr = row_ptr<T>(rs, b, d.j);
  const T* qr = kResid ? row_ptr<T>(rs, b, K + 1 + d.j) : pr;
  constexpr int kPerLane = kGroups / 32;  // groups per lane
  // groups in flight per row: all 8 (one round) with 128 registers per thread on bf16 rows
  constexpr int kRound = VEC == 8 ? (kWide ? 8 : 4) : (VEC == 4 ? 2 : 1);
  float acc = 0.f;
#pragma unroll
  for (int k0 = 0; k0 < kPerLane; k0 += kRound) {
    GroupRaw<T, VEC> gp[kRound], gq[kRound];
#pragma unroll
    for (int k = 0; k < kRound; ++k) {
      const int t0 = c * kCE + ((k0 + k) * 32 + lane) * 8;
      gp[k].load(pr, t0, V);
      if constexpr (kResid) gq[k].load(qr, t0, V);
    }
#pragma unroll
    for (int k = 0; k < kRound; ++k) {
      const float gsum = group_sum<T, VEC, kResid>(gp[k], gq[k], scale, d);
      part[(k0 + k) * 32 + lane] = gsum;
      acc = __fadd_rn(acc, gsum);
    }
  }
  return warp_sum(acc);
}

// Where the draw falls among the chunks of its row: float64 prefix over the chunk masses
// (lane l holds chunks l*kMassPerLane .. l*kMassPerLane + kMassPerLane - 1, zero past the
// row), target u*Z, first chunk whose inclusive prefix passes it. Every lane gets the result.
constexpr int kMassPerLane = kMaxChunkCount / 32;
struct ChunkPick {
  int c;       // chunk that holds the draw; -1 when no chunk has mass
  double tin;  // the target measured from the chunk's start (+inf: past the last mass)
  double z;    // the law's total mass
};

__device__ __forceinline__ ChunkPick pick_chunk(const float (&ms)[kMassPerLane], float u,
                                                int lane) {
  constexpr int NPL = kMassPerLane;
  double m[NPL];
  double ls = 0.0;
#pragma unroll
  for (int k = 0; k < NPL; ++k) {
    m[k] = ms[k];
    ls += m[k];
  }
  double incl = ls;  // inclusive prefix over lanes
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const double a = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += a;
  }
  ChunkPick pk;
  pk.z = __shfl_sync(0xffffffffu, incl, 31);
  const double target = static_cast<double>(u) * pk.z;
  double run = incl - ls;
  int cfound = -1, clast = -1;
  double before = 0.0;
#pragma unroll
  for (int k = 0; k < NPL; ++k) {
    const double nxt = run + m[k];
    if (m[k] > 0.0) {
      clast = lane * NPL + k;
      if (cfound < 0 && run <= target && target < nxt) {
        cfound = clast;
        before = run;
      }
    }
    run = nxt;
  }
  const unsigned hit = __ballot_sync(0xffffffffu, cfound >= 0);
  if (hit) {
    const int hl = __ffs(hit) - 1;
    pk.c = __shfl_sync(0xffffffffu, cfound, hl);
    pk.tin = target - __shfl_sync(0xffffffffu, before, hl);
  } else {  // rounding left the target past the last mass: the last token with mass
    int cl = clast;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) cl = max(cl, __shfl_xor_sync(0xffffffffu, cl, o));
    pk.c = cl;
    pk.tin = __int_as_float(0x7f800000);
  }
  return pk;
}

// The token of chunk c at the target tin (measured from the chunk's start), given the chunk's
// 256 group sums `part` (token order) of the law (kResid: residual, else p): the group from a
// scan of the sums, then that group's 8 tokens re-read and recomputed exactly as their sum
// was, scanned by lane 0. Rounding that leaves the target past the chunk's sums picks its last
// token with mass. Every lane gets the token.
template <typename T, int VEC, bool kResid>
__device__ __forceinline__ int pick_token(const RowSet& rs, float scale, int b, const Decision& d,
                                          int c, float tin, const float* part, int lane) {
  const int j = d.j;
  // lane l scans the chunk's groups 8l .. 8l+7 (token order)
  float gv[8];
  float lsum = 0.f;
  int lastg = -1;
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    gv[e] = part[lane * 8 + e];
    lsum = __fadd_rn(lsum, gv[e]);
    if (gv[e] > 0.f) lastg = lane * 8 + e;
  }
  float inc = lsum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const float y = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc = __fadd_rn(inc, y);
  }
  float ex = __shfl_up_sync(0xffffffffu, inc, 1);
  if (lane == 0) ex = 0.f;
  int qsel = -1;
  float gin = 0.f;
  if (ex <= tin && tin < inc) {
    float r = ex;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float nx = __fadd_rn(r, gv[e]);
      if (qsel < 0 && gv[e] > 0.f && r <= tin && tin < nx) {
        qsel = lane * 8 + e;
        gin = __fsub_rn(tin, r);
      }
      r = nx;
    }
  }
  const unsigned h = __ballot_sync(0xffffffffu, qsel >= 0);
  bool last_mode = false;
  if (h) {
    const int hl = __ffs(h) - 1;
    qsel = __shfl_sync(0xffffffffu, qsel, hl);
    gin = __shfl_sync(0xffffffffu, gin, hl);
  } else {  // rounding: the chunk's last group with mass, its last token with mass
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) lastg = max(lastg, __shfl_xor_sync(0xffffffffu, lastg, o));
    qsel = lastg;
    last_mode = true;
  }
  int token = -1;
  if (qsel >= 0 && lane == 0) {
    const int K = rs.K, V = rs.V;
    const T* pr = row_ptr<T>(rs, b, j);
    const T* qr = kResid ? row_ptr<T>(rs, b, K + 1 + j) : pr;
    const int t0 = c * kCE + qsel * 8;
    GroupRaw<T, VEC> gp, gq;
    gp.load(pr, t0, V);
    if constexpr (kResid) gq.load(qr, t0, V);
    float v[8];
    group_values<T, VEC, kResid>(gp, gq, scale, d, v);
    float r = 0.f;
    int cand = -1, lastv = -1;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float nx = __fadd_rn(r, v[e]);
      if (v[e] > 0.f) lastv = t0 + e;
      if (!last_mode && cand < 0 && v[e] > 0.f && r <= gin && gin < nx) cand = t0 + e;
      r = nx;
    }
    token = cand >= 0 ? cand : lastv;
  }
  return __shfl_sync(0xffffffffu, token, 0);
}

// L2 prefetch of `bytes` bytes (a multiple of 16, 16-byte aligned) from global memory.
__device__ __forceinline__ void prefetch_l2(const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

// What the sampling finish starts from: the pass-1 records of a uniform call or of a mixed
// batch (it merges them and takes the decisions), or the decisions that the early-exit waves
// stored (early_exit.cuh).
constexpr int kFinUniform = 0;
constexpr int kFinMixed = 1;
constexpr int kFinEarlyExit = 2;

struct FinishParamsEarlyExit : FinishParams {
  const Decision* dec;  // [B], written by the wave that ended each sequence
};
template <int kFin>
using FinishParamsOf = std::conditional_t<
    kFin == kFinMixed, FinishParamsMixed,
    std::conditional_t<kFin == kFinEarlyExit, FinishParamsEarlyExit, FinishParams>>;

// Sampling finish. Launched as clusters of G CTAs of kW warps, one cluster per sequence; CTA g
// of the cluster owns chunks g*cpc .. g*cpc + cpc - 1 of the draw's law (warp w: local chunks
// w, w + kW, ...).
template <typename T, int VEC, int kFin, int kW>
__global__ void __launch_bounds__(kW * 32, 1) finish_sample_kernel(const FinishParamsOf<kFin> p) {
  constexpr bool kMixed = kFin == kFinMixed;
  constexpr int kT = kW * 32;
  constexpr bool kWide = kW <= kFinWarpsSmall;  // 128 registers per thread
  extern __shared__ float s_part[];  // [cpc][kGroups]: group sums of the draw's law
  __shared__ float2 s_stat[kMaxRows];
  __shared__ float s_mass[kMaxChunkCount];  // every chunk's mass of the draw's law
  __shared__ float s_u[kMaxK + 1];
  __shared__ int s_x[kMaxK];
  __shared__ float2 s_zg[kMaxK];
  // the next kernel in the stream may be scheduled as these CTAs retire (it waits for them)
  grid_dependents_launch();
  cg::cluster_group cluster = cg::this_cluster();
  const int tid = threadIdx.x, lane = tid & 31, wi = tid >> 5;
  const int G = static_cast<int>(cluster.num_blocks());
  const int cpc = (p.nch + G - 1) / G;  // chunks per CTA
  const int b = blockIdx.x / G;
  const int g = static_cast<int>(cluster.block_rank());
  const int K = p.rs.K, K1 = K + 1, V = p.rs.V, rows = p.rs.rows;
  // the sequence's draft count nd and scale: K and the call's scale, or, in a mixed batch,
  // its own (a greedy sequence takes the greedy finish in CTA 0; no cluster barrier follows)
  int nd = K;
  float scale = p.scale;
  if constexpr (kMixed) {
    const SeqMode sm = seq_mode(p.n_drafts, p.temps, b, K);
    if (!sm.ok) {
      if (g == 0) write_error(p, b, DSPARK_SEQ_BAD_PARAM, tid, kT);
      return;
    }
    nd = sm.kb;
    scale = sm.scale;
    if (sm.greedy) {
      if (g != 0) return;
      int xg = 0;
      if (tid < nd) {
        xg = p.drafts[static_cast<size_t>(b) * K + tid];
        s_x[tid] = xg;
      }
      grid_dependency_wait();
      greedy_finish<true, kW>(p, b, nd, xg, wi, lane, s_stat, s_x);
      return;
    }
  }

  // inputs that pass 1 does not write: drafts, uniforms
  int x = -1;
  if (tid < nd) x = p.drafts[static_cast<size_t>(b) * K + tid];
  if (tid <= nd) s_u[tid] = p.uniforms[static_cast<size_t>(b) * K1 + tid];
  grid_dependency_wait();
  Decision d;
  if constexpr (kFin == kFinEarlyExit) {
    if (tid < nd) s_x[tid] = x;
    d = p.dec[b];  // every warp reads the stored decision itself
    __syncthreads();
  } else {
    // the draft tokens' logits, gathered by pass 1, in flight with the records' below
    float2 zg = make_float2(0.f, 0.f);
    if (tid < nd) {
      s_x[tid] = x;
      if (x >= 0 && x < V)
        zg = __ldcg(reinterpret_cast<const float2*>(p.gather) + static_cast<size_t>(b) * K + tid);
    }

    // the (reference, sum) of every row the sequence uses
    const RowFilter used{K, nd, true};
    merge_rows<true, kMixed, kW>(p, b, used, wi, lane, s_stat);
    if (tid < nd) s_zg[tid] = zg;
    __syncthreads();

    // decisions, by every warp (the same inputs and arithmetic, so the same j everywhere):
    // draft i on lane i
    int status = 0;
    bool bad = false;
    for (int r = lane; r < rows; r += 32) bad |= (!kMixed || used(r)) && !stat_ok(s_stat[r]);
    if (__any_sync(0xffffffffu, bad)) status |= DSPARK_SEQ_NONFINITE;
    const int xl = lane < nd ? s_x[lane] : 0;
    const bool bad_draft = lane < nd && (xl < 0 || xl >= V);
    if (__any_sync(0xffffffffu, bad_draft)) status |= DSPARK_SEQ_BAD_DRAFT;
    const float fnan = __int_as_float(0x7fffffff);
    float px = fnan, qx = fnan;
    bool accept = false;
    if (lane < nd && !bad_draft) {
      const float2 sp = s_stat[lane], sq = s_stat[K1 + lane], zg = s_zg[lane];
      // p_i(x_i) = 2^(z*s - M) / S (division within 2 ulp: no IEEE slow path)
      px = __fdividef(ex2(__fmaf_rn(zg.x, scale, -sp.x)), sp.y);
      qx = __fdividef(ex2(__fmaf_rn(zg.y, scale, -sq.x)), sq.y);
      accept = __fmul_rn(s_u[lane], qx) < px;
    }
    const unsigned rej = __ballot_sync(0xffffffffu, lane < nd && !accept);
    const int j = rej ? __ffs(rej) - 1 : nd;
    if (g == 0 && wi == 0 && lane < K) {
      if (p.out.p_draft) p.out.p_draft[static_cast<size_t>(b) * K + lane] = px;
      if (p.out.q_draft) p.out.q_draft[static_cast<size_t>(b) * K + lane] = qx;
    }
    const float2 sp = s_stat[j];
    d.j = j;
    d.nd = nd;
    d.status = status;
    d.mp = sp.x;
    d.ip = __fdividef(1.f, sp.y);
    if (j < nd) {
      const float2 sq = s_stat[K1 + j];
      d.mq = sq.x;
      d.iq = __fdividef(1.f, sq.y);
    } else {
      d.mq = 0.f;
      d.iq = 0.f;
    }
  }
  // this CTA's chunk range of the draw's rows into L2, ahead of the warps' second loads
  if (VEC > 1 && lane == 0 && wi >= kW - 2 && !(d.status & kErrBits)) {
    const int t0 = g * cpc * kCE;
    const int t1 = min(V, t0 + cpc * kCE);
    const bool q_row = wi == kW - 1;
    if (t0 < t1 && (!q_row || d.j < d.nd)) {
      const uint32_t bytes = static_cast<uint32_t>(t1 - t0) * Elem<T>::kBytes;
      prefetch_l2(row_ptr<T>(p.rs, b, q_row ? K1 + d.j : d.j) + t0, bytes);
    }
  }

  // this CTA's chunks of the draw's law (the residual after a rejection, p_K for the bonus):
  // group sums into shared memory, chunk masses to every CTA of the cluster
  const bool resid = d.j < d.nd;
  if (!(d.status & kErrBits)) {
    for (int lc = wi; lc < cpc; lc += kW) {
      const int c = g * cpc + lc;
      if (c >= p.nch) break;
      float* pr = s_part + static_cast<size_t>(lc) * kGroups;
      const float m = resid ? chunk_work<T, VEC, true, kWide>(p.rs, scale, b, c, d, lane, pr)
                            : chunk_work<T, VEC, false, kWide>(p.rs, scale, b, c, d, lane, pr);
      if (lane < G) cluster.map_shared_rank(s_mass, lane)[c] = m;
    }
  }
  cluster.sync();  // every chunk mass has landed in every CTA; group sums are visible CTA-wide

  if (d.status & kErrBits) {
    if (g == 0) write_error(p, b, d.status, tid, kT);
    return;
  }

  // ---- which chunk holds the draw (warp 0 of every CTA, the same float64 arithmetic on the
  // same masses)
  const int j = d.j;
  int status = d.status;
  bool use_p = !resid;
  if (resid) {
    // a residual whose every value rounded to zero (impossible in exact arithmetic after a
    // rejection): draw from p_j instead. Every warp of the cluster sees the same masses and
    // takes this branch together; the masses are rewritten only after every CTA read them.
    bool any = false;
    for (int c = lane; c < p.nch; c += 32) any |= s_mass[c] > 0.f;
    if (!__any_sync(0xffffffffu, any)) {
      use_p = true;
      status |= DSPARK_SEQ_ZERO_RESIDUAL;
      cluster.sync();
      for (int lc = wi; lc < cpc; lc += kW) {
        const int c = g * cpc + lc;
        if (c >= p.nch) break;
        const float m = chunk_work<T, VEC, false>(p.rs, scale, b, c, d, lane,
                                                  s_part + static_cast<size_t>(lc) * kGroups);
        if (lane < G) cluster.map_shared_rank(s_mass, lane)[c] = m;
      }
      cluster.sync();
    }
  }
  if (wi != 0) return;
  float ms[kMassPerLane];
#pragma unroll
  for (int k = 0; k < kMassPerLane; ++k) {
    const int c = lane * kMassPerLane + k;
    ms[k] = c < p.nch ? s_mass[c] : 0.f;
  }
  const ChunkPick pk = pick_chunk(ms, s_u[nd], lane);
  const int c = pk.c;
  const int owner = c >= 0 ? c / cpc : 0;
  if (owner != g) return;  // another CTA draws
  if (lane == 0) {
    if (p.out.resid_mass)
      p.out.resid_mass[b] = resid ? (use_p ? 0.f : static_cast<float>(pk.z)) : 1.f;
    if (p.out.status) p.out.status[b] = status;
  }
  int token = -1;
  if (c >= 0) {
    const float* part = s_part + static_cast<size_t>(c - g * cpc) * kGroups;
    const float tin = static_cast<float>(pk.tin);
    token = use_p ? pick_token<T, VEC, false>(p.rs, scale, b, d, c, tin, part, lane)
                  : pick_token<T, VEC, true>(p.rs, scale, b, d, c, tin, part, lane);
  }
  write_tokens(p, b, j, token, s_x, lane, 32);
}

}  // namespace dspark
