// Pass 2 of the verify step: per-sequence decisions and the correction / bonus draw.
//
// Greedy: one CTA per sequence merges the pass-1 argmax records of its K+1 rows (a warp per
// row), compares the drafts with the row argmaxes and writes the AcceptResult.
//
// Sampling: G CTAs per sequence, G = ceil(n_chunks / 8). Every CTA of a sequence merges the
// 2K+1 rows' softmax records and takes the accept decisions (the same inputs and arithmetic
// in each, so the same j). It then computes, one 2048-token chunk per warp, the mass of the
// draw's law: r = max(p_j - q_j, 0) after a rejection (j < K), p_K for the bonus (j = K).
// The last CTA of the sequence to finish (a counter in the workspace) draws the token by
// inverse CDF: float64 prefix over the chunk masses, then a re-read and scan of the one
// chunk that holds the target. No CTA waits for another.
//
// Both kernels start with the loads that do not depend on pass 1 (drafts, uniforms, the
// draft-token logits) and then wait for pass 1 to complete (programmatic dependent launch).
#pragma once

#include "stream.cuh"

namespace dspark {

constexpr int kErrBits = DSPARK_SEQ_BAD_DRAFT | DSPARK_SEQ_NONFINITE | DSPARK_SEQ_TIMEOUT;
constexpr int kMaxRows = 2 * kMaxK + 1;

struct FinishParams {
  RowSet rs;
  const int32_t* drafts;    // [B, K]
  const float* uniforms;    // [B, K+1] (sampling)
  int B;
  int G;                    // CTAs per sequence (sampling)
  int nch;                  // chunks per row
  float scale;              // log2(e) / T
  const float2* rec;        // pass-1 records [B * rows, nch]
  float2* mass;             // [B, nch]: (mass of the draw's law, mass of p_j) per chunk
  unsigned* arrive;         // [B], zero between calls
  dspark_accept_out_t out;
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

// Rows 0..rows-1 of sequence b into s_stat: warp w merges rows w, w + 8, ..., two at a time
// so that their loads overlap.
template <bool kSample>
__device__ __forceinline__ void merge_rows(const FinishParams& p, int b, int rows, int wi,
                                           int lane, float2* s_stat) {
  const long long r0 = static_cast<long long>(b) * rows;
  for (int r = wi; r < rows; r += 2 * kWarps) {
    RowRecs a, c;
    load_row<kSample>(p, r0 + r, lane, a);
    const bool two = r + kWarps < rows;
    if (two) load_row<kSample>(p, r0 + r + kWarps, lane, c);
    const float2 sa = reduce_row<kSample>(a);
    if (lane == 0) s_stat[r] = sa;
    if (two) {
      const float2 sc = reduce_row<kSample>(c);
      if (lane == 0) s_stat[r + kWarps] = sc;
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

// x_0..x_{j-1}, then `token` at j, then -1.
__device__ __forceinline__ void write_tokens(const FinishParams& p, int b, int j, int token, int t,
                                             int nt) {
  const int K = p.rs.K, K1 = K + 1;
  for (int k = t; k < K1; k += nt)
    p.out.tokens[static_cast<size_t>(b) * K1 + k] =
        k < j ? p.drafts[static_cast<size_t>(b) * K + k] : (k == j ? token : -1);
  if (t == 0) {
    p.out.n_accepted[b] = j;
    p.out.next_token[b] = token;
  }
}

// ------------------------------------------------------------------------------ greedy

template <typename T>
__global__ void __launch_bounds__(kThreads) finish_greedy_kernel(const FinishParams p) {
  __shared__ float2 s_arg[kMaxK + 1];
  const int lane = threadIdx.x & 31, wi = threadIdx.x >> 5;
  const int b = blockIdx.x;
  const int K = p.rs.K, K1 = K + 1;
  int x = 0;
  if (wi == 0 && lane < K) x = p.drafts[static_cast<size_t>(b) * K + lane];
  grid_dependency_wait();
  merge_rows<false>(p, b, K1, wi, lane, s_arg);
  __syncthreads();
  if (wi != 0) return;
  const float ninf = -__int_as_float(0x7f800000);
  bool bad = false;
  for (int r = lane; r < K1; r += 32) {
    const float2 a = s_arg[r];
    // NaN anywhere, a +inf maximum, or nothing above -inf: not a usable row
    bad |= !(a.x > ninf) || !(a.x < -ninf) || __float_as_int(a.y) == INT_MAX;
  }
  int status = __any_sync(0xffffffffu, bad) ? DSPARK_SEQ_NONFINITE : 0;
  if (__any_sync(0xffffffffu, lane < K && (x < 0 || x >= p.rs.V))) status |= DSPARK_SEQ_BAD_DRAFT;
  const int arg = lane < K ? __float_as_int(s_arg[lane].y) : -1;
  const unsigned mis = __ballot_sync(0xffffffffu, lane < K && x != arg);
  const int j = mis ? __ffs(mis) - 1 : K;
  if (status & kErrBits) {
    write_error(p, b, status, lane, 32);
    return;
  }
  write_tokens(p, b, j, __float_as_int(s_arg[j].y), lane, 32);
  if (lane == 0 && p.out.status) p.out.status[b] = 0;
}

// ---------------------------------------------------------------------------- sampling

// The row normalisers of the draw's law, and the decision.
struct Decision {
  int j;
  int status;
  float mp, ip;  // p_j (or p_K): reference and 1 / sum
  float mq, iq;  // q_j: reference and 1 / sum (iq = 0 for the bonus)
};

// Per-token mass of the draw's law. The chunk masses and the draw's scan use exactly this
// arithmetic, so the scan reproduces the masses it located.
__device__ __forceinline__ float p_value(float zp, float s, const Decision& d) {
  return __fmul_rn(ex2(__fmaf_rn(zp, s, -d.mp)), d.ip);
}
__device__ __forceinline__ float resid_value(float zp, float zq, float s, const Decision& d) {
  const float ep = ex2(__fmaf_rn(zp, s, -d.mp));
  const float eq = ex2(__fmaf_rn(zq, s, -d.mq));
  return fmaxf(__fmaf_rn(ep, d.ip, -__fmul_rn(eq, d.iq)), 0.f);
}

// The 8 consecutive tokens t0 .. t0+7 of a row (t0 a multiple of 8); -inf past V.
template <typename T, int VEC>
__device__ __forceinline__ void load8(const T* row, int t0, int V, float* z) {
  const float ninf = -__int_as_float(0x7f800000);
  if constexpr (VEC == 1) {
#pragma unroll
    for (int e = 0; e < 8; ++e) z[e] = t0 + e < V ? Elem<T>::load1(row + t0 + e) : ninf;
  } else {
#pragma unroll
    for (int h = 0; h < 8; h += VEC) {
      if (t0 + h < V) {
        Elem<T>::unpack(ld_stream16(row + t0 + h), z + h);
      } else {
#pragma unroll
        for (int e = 0; e < VEC; ++e) z[h + e] = ninf;
      }
    }
  }
}

// Sum of the draw's law and of p_j over 8 raw tokens groups (accumulated in place).
template <typename T>
__device__ __forceinline__ void mass_terms(const uint4& wp, const uint4& wq, bool has_q,
                                           const FinishParams& p, const Decision& d, float& acc_r,
                                           float& acc_p) {
  constexpr int VEC = Elem<T>::kPerVec16;
  float zp[VEC];
  Elem<T>::unpack(wp, zp);
  if (has_q) {
    float zq[VEC];
    Elem<T>::unpack(wq, zq);
#pragma unroll
    for (int e = 0; e < VEC; ++e) {
      acc_r = __fadd_rn(acc_r, resid_value(zp[e], zq[e], p.scale, d));
      acc_p = __fadd_rn(acc_p, p_value(zp[e], p.scale, d));
    }
  } else {
#pragma unroll
    for (int e = 0; e < VEC; ++e) acc_p = __fadd_rn(acc_p, p_value(zp[e], p.scale, d));
  }
}

// (mass of the draw's law, mass of p_j) over chunk c, one warp. The order of the sum is free:
// the draw's scan recomputes the per-token values and only locates the chunk with these.
template <typename T, int VEC>
__device__ __forceinline__ float2 chunk_mass(const FinishParams& p, int b, int c, const Decision& d,
                                             int lane) {
  const int K = p.rs.K, V = p.rs.V;
  const T* pr = row_ptr<T>(p.rs, b, d.j) + static_cast<size_t>(c) * kCE;
  const T* qr = d.j < K ? row_ptr<T>(p.rs, b, K + 1 + d.j) + static_cast<size_t>(c) * kCE : nullptr;
  const int valid = min(kCE, V - c * kCE);
  float acc_r = 0.f, acc_p = 0.f;
  if constexpr (VEC == 1) {
    for (int t = lane; t < valid; t += 32) {
      const float zp = Elem<T>::load1(pr + t);
      if (qr) acc_r = __fadd_rn(acc_r, resid_value(zp, Elem<T>::load1(qr + t), p.scale, d));
      acc_p = __fadd_rn(acc_p, p_value(zp, p.scale, d));
    }
  } else {
    // 8 vectors of each row in flight per lane (bf16: the whole chunk)
    constexpr int NV = kCE / VEC / 32;
    constexpr int NB = NV < 8 ? NV : 8;
    const int nvv = valid / VEC;
#pragma unroll
    for (int k0 = 0; k0 < NV; k0 += NB) {
      uint4 wp[NB], wq[NB] = {};
#pragma unroll
      for (int k = 0; k < NB; ++k) {
        const int vi = (k0 + k) * 32 + lane;
        const bool ok = vi < nvv;
        const uint32_t ninf = Elem<T>::kBytes == 2 ? 0xff80ff80u : 0xff800000u;
        wp[k] = ok ? ld_stream16(pr + vi * VEC) : make_uint4(ninf, ninf, ninf, ninf);
        if (qr) wq[k] = ok ? ld_stream16(qr + vi * VEC) : make_uint4(ninf, ninf, ninf, ninf);
      }
#pragma unroll
      for (int k = 0; k < NB; ++k) mass_terms<T>(wp[k], wq[k], qr != nullptr, p, d, acc_r, acc_p);
    }
  }
  acc_p = warp_sum(acc_p);
  acc_r = qr ? warp_sum(acc_r) : acc_p;
  return make_float2(acc_r, acc_p);
}

template <typename T, int VEC>
__global__ void __launch_bounds__(kThreads) finish_sample_kernel(const FinishParams p) {
  __shared__ float2 s_stat[kMaxRows];
  __shared__ float s_zp[kMaxK], s_zq[kMaxK], s_u[kMaxK + 1];
  __shared__ int s_x[kMaxK];
  __shared__ Decision s_dec;
  __shared__ int s_last;
  __shared__ float s_wtot[kWarps];
  __shared__ double s_tin;
  __shared__ int s_chunk, s_use_p, s_token, s_lastpos;
  const int tid = threadIdx.x, lane = tid & 31, wi = tid >> 5;
  const int b = blockIdx.x / p.G, g = blockIdx.x - b * p.G;
  const int K = p.rs.K, K1 = K + 1, V = p.rs.V, rows = p.rs.rows;

  // inputs that pass 1 does not write: drafts, uniforms, the draft tokens' logits
  if (tid < K) {
    const int x = p.drafts[static_cast<size_t>(b) * K + tid];
    s_x[tid] = x;
    float zp = 0.f, zq = 0.f;
    if (x >= 0 && x < V) {
      zp = Elem<T>::load1(row_ptr<T>(p.rs, b, tid) + x);
      zq = Elem<T>::load1(row_ptr<T>(p.rs, b, K1 + tid) + x);
    }
    s_zp[tid] = zp;
    s_zq[tid] = zq;
  }
  if (tid <= K) s_u[tid] = p.uniforms[static_cast<size_t>(b) * K1 + tid];
  grid_dependency_wait();

  // every row's (reference, sum)
  merge_rows<true>(p, b, rows, wi, lane, s_stat);
  __syncthreads();

  // decisions (warp 0; draft i on lane i)
  if (wi == 0) {
    int status = 0;
    bool bad = false;
    for (int r = lane; r < rows; r += 32) bad |= !stat_ok(s_stat[r]);
    if (__any_sync(0xffffffffu, bad)) status |= DSPARK_SEQ_NONFINITE;
    const int x = lane < K ? s_x[lane] : 0;
    const bool bad_draft = lane < K && (x < 0 || x >= V);
    if (__any_sync(0xffffffffu, bad_draft)) status |= DSPARK_SEQ_BAD_DRAFT;
    const float fnan = __int_as_float(0x7fffffff);
    float px = fnan, qx = fnan;
    bool accept = false;
    if (lane < K && !bad_draft) {
      const float2 sp = s_stat[lane], sq = s_stat[K1 + lane];
      px = __fdiv_rn(ex2(__fmaf_rn(s_zp[lane], p.scale, -sp.x)), sp.y);
      qx = __fdiv_rn(ex2(__fmaf_rn(s_zq[lane], p.scale, -sq.x)), sq.y);
      accept = __fmul_rn(s_u[lane], qx) < px;
    }
    const unsigned rej = __ballot_sync(0xffffffffu, lane < K && !accept);
    const int j = rej ? __ffs(rej) - 1 : K;
    if (g == 0 && lane < K) {
      if (p.out.p_draft) p.out.p_draft[static_cast<size_t>(b) * K + lane] = px;
      if (p.out.q_draft) p.out.q_draft[static_cast<size_t>(b) * K + lane] = qx;
    }
    if (lane == 0) {
      const float2 sp = s_stat[j];
      Decision d;
      d.j = j;
      d.status = status;
      d.mp = sp.x;
      d.ip = __fdiv_rn(1.f, sp.y);
      if (j < K) {
        const float2 sq = s_stat[K1 + j];
        d.mq = sq.x;
        d.iq = __fdiv_rn(1.f, sq.y);
      } else {
        d.mq = 0.f;
        d.iq = 0.f;
      }
      s_dec = d;
    }
  }
  __syncthreads();
  const Decision d = s_dec;

  // this CTA's chunks of the draw's law
  if (!(d.status & kErrBits)) {
    const int c = g * kWarps + wi;
    if (c < p.nch) {
      const float2 m = chunk_mass<T, VEC>(p, b, c, d, lane);
      if (lane == 0) {
        p.mass[static_cast<size_t>(b) * p.nch + c] = m;
        __threadfence();  // the mass is visible before this CTA's arrival is counted
      }
    }
  }
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    const unsigned old = atomicAdd(p.arrive + b, 1u);
    s_last = old == static_cast<unsigned>(p.G - 1);
    if (s_last) p.arrive[b] = 0;  // every CTA of b has arrived: reset for the next call
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();

  if (d.status & kErrBits) {
    write_error(p, b, d.status, tid, kThreads);
    return;
  }

  // ---- the draw (the last CTA of the sequence)
  const int j = d.j;
  int status = d.status;
  const float uK = s_u[K];
  // chunk masses in float64: warp 0, lane l holds chunks 4l .. 4l+3 (token order)
  constexpr int NPL = kMaxChunkCount / 32;
  bool use_p = j == K;
  if (wi == 0) {
    double mr[NPL], mp[NPL];
    double zr = 0.0, zpm = 0.0;
#pragma unroll
    for (int k = 0; k < NPL; ++k) {
      const int c = lane * NPL + k;
      float2 m = make_float2(0.f, 0.f);
      if (c < p.nch) m = __ldcg(p.mass + static_cast<size_t>(b) * p.nch + c);
      mr[k] = m.x;
      mp[k] = m.y;
      zr += mr[k];
      zpm += mp[k];
    }
    // totals over lanes (every lane the same sums in the same order)
    double Zr = zr, Zp = zpm;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const double a = __shfl_up_sync(0xffffffffu, Zr, o), c2 = __shfl_up_sync(0xffffffffu, Zp, o);
      if (lane >= o) {
        Zr += a;
        Zp += c2;
      }
    }
    // Zr / Zp now hold inclusive prefixes over lanes; the totals sit on lane 31
    const double Zres = __shfl_sync(0xffffffffu, Zr, 31);
    if (!use_p && !(Zres > 0.0)) {  // residual mass rounded to zero: draw from p_j instead
      use_p = true;
      status |= DSPARK_SEQ_ZERO_RESIDUAL;
    }
    double m[NPL];
#pragma unroll
    for (int k = 0; k < NPL; ++k) m[k] = use_p ? mp[k] : mr[k];
    const double incl = use_p ? Zp : Zr;
    const double ls = use_p ? zpm : zr;
    const double Z = __shfl_sync(0xffffffffu, incl, 31);
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
          cfound = clast;
          before = run;
        }
      }
      run = nxt;
    }
    const unsigned hit = __ballot_sync(0xffffffffu, cfound >= 0);
    int c;
    double tin;
    if (hit) {
      const int hl = __ffs(hit) - 1;
      c = __shfl_sync(0xffffffffu, cfound, hl);
      tin = target - __shfl_sync(0xffffffffu, before, hl);
    } else {  // rounding left the target past the last mass: the chunk's last token
      int cl = clast;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) cl = max(cl, __shfl_xor_sync(0xffffffffu, cl, o));
      c = cl;
      tin = __int_as_float(0x7f800000);
    }
    if (lane == 0) {
      s_tin = tin;
      s_chunk = c;
      s_use_p = use_p;
      s_token = INT_MAX;
      s_lastpos = -1;
      if (p.out.resid_mass) p.out.resid_mass[b] = j < K ? (use_p ? 0.f : static_cast<float>(Zres)) : 1.f;
      if (p.out.status) p.out.status[b] = status;
    }
  }
  __syncthreads();
  const int c = s_chunk;
  const float tin = static_cast<float>(s_tin);
  use_p = s_use_p != 0;
  if (c >= 0) {
    // per-token masses of chunk c exactly as chunk_mass computed them; warp w scans tokens
    // c*2048 + 256w .. +255, lane l holds 8 consecutive ones
    const T* pr = row_ptr<T>(p.rs, b, j);
    const T* qr = !use_p ? row_ptr<T>(p.rs, b, K1 + j) : nullptr;
    const int t0 = c * kCE + wi * 256 + lane * 8;
    float zp[8], val[8];
    load8<T, VEC>(pr, t0, V, zp);
    if (qr) {
      float zq[8];
      load8<T, VEC>(qr, t0, V, zq);
#pragma unroll
      for (int e = 0; e < 8; ++e) val[e] = resid_value(zp[e], zq[e], p.scale, d);
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) val[e] = p_value(zp[e], p.scale, d);
    }
    float lsum = 0.f;
    int lastv = -1;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      lsum = __fadd_rn(lsum, val[e]);
      if (val[e] > 0.f) lastv = t0 + e;
    }
    float inc = lsum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const float y = __shfl_up_sync(0xffffffffu, inc, o);
      if (lane >= o) inc = __fadd_rn(inc, y);
    }
    if (lane == 31) s_wtot[wi] = inc;
    if (lastv >= 0) atomicMax(&s_lastpos, lastv);
    __syncthreads();
    float wbase = 0.f;
    for (int w = 0; w < wi; ++w) wbase = __fadd_rn(wbase, s_wtot[w]);
    float ex = __shfl_up_sync(0xffffffffu, inc, 1);
    if (lane == 0) ex = 0.f;
    float r = __fadd_rn(wbase, ex);
    if (r <= tin && tin < __fadd_rn(wbase, inc)) {
      int cand = -1;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float nx = __fadd_rn(r, val[e]);
        if (cand < 0 && val[e] > 0.f && r <= tin && tin < nx) cand = t0 + e;
        r = nx;
      }
      if (cand < 0) cand = lastv;
      if (cand >= 0) atomicMin(&s_token, cand);
    }
    __syncthreads();
  }
  if (tid == 0) {
    int token = s_token;
    if (token == INT_MAX) token = s_lastpos;  // rounding: the last token with mass
    s_token = token;
  }
  __syncthreads();
  write_tokens(p, b, j, s_token, tid, kThreads);
}

}  // namespace dspark
