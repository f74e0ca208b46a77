// speculative_sample_accept on sm_100a: pass 1 (row statistics and chunk masses) and the
// finish kernel (decide, then the pass-2 inverse-CDF draw on the one selected row).
//
// Pass 1 is a persistent kernel over thread-block clusters. A work unit is one position i of
// one sequence b: the pair (P row i, Q row i) for i < K, or the bonus row P_K alone. The V
// axis of a unit is split over the CTAs of a cluster, and within a CTA over its warps: warp w
// of CTA r owns the contiguous "chunk" c = r * warps + w of 1024 tokens (32 lanes x 32
// register-resident logits). Each row element is read from HBM exactly once, by 1-D bulk
// copies (cp.async.bulk, no multicast) into a shared-memory stage ring, and lands in
// registers where it stays until the unit is finished:
//   1. chunk max -> exponentials 2^(z*s - ref) against the chunk's own reference (one SFU op
//      per element), chunk sums;
//   2. CTA merge in shared memory, cluster merge over DSMEM -> the row's (max, sum) for P_i
//      and Q_i, identical bit for bit in every CTA;
//   3. per chunk the factors c = 2^(ref - M) / S that turn the register exponentials into
//      probabilities, and from registers the residual mass sum_v max(p[v] - q[v], 0) of the
//      chunk (no second read of the row).
// The finish kernel (one CTA per sequence) then gathers p_i(x_i), q_i(x_i), finds the first
// rejection j, scans the chunk masses of the selected row (residual j, or P_K for the bonus)
// in float64 to find the chunk holding the draw, re-reads only that chunk (2-4 KB) and redoes
// the per-element arithmetic bit for bit to pick the token.
#pragma once

#include "common.cuh"

namespace dspark {

constexpr int kMaxStages = 4;

struct SampleParams {
  const void* p1;
  const void* pv;
  const void* q;
  int64_t ld_p1;
  int64_t ld_pv;
  int B, K, V;
  float scale;        // log2(e) / T
  int n_chunks;       // chunks per row
  int warps;          // warps per CTA
  int cluster;        // CTAs per cluster
  int n_units;        // B * (K+1)
  int n_clusters;     // clusters in the persistent grid
  int stages;         // shared-memory ring depth (bulk-copy variant)
  int slice_elems;    // V elements per CTA slice = warps * 1024
  float2* rowstat;    // [B*(K+1) P rows, then B*K Q rows]: (M, S)
  ChunkRec* chunk_p;  // [B*(K+1), n_chunks]
  ChunkRec* chunk_r;  // [B*K, n_chunks]
  uint8_t* unit_flags;  // [B*(K+1), cluster]
};

// Shared memory of the pass-1 kernel after the stage ring.
struct Pass1Smem {
  uint64_t full[kMaxStages];
  float4 red[kMaxWarps];
  float4 dsm[2];
};

__host__ __device__ inline size_t pass1_ring_bytes(int stages, int slice_elems, int elem_bytes) {
  return static_cast<size_t>(stages) * 2 * static_cast<size_t>(slice_elems) * elem_bytes;
}

// Fill z[0..31] with this lane's logits of one row slice: z[k*VEC + e] is element
// (k*32 + lane)*VEC + e of the warp's chunk. Elements at or past V read as -inf.
template <typename T, int VEC, bool kTma>
__device__ __forceinline__ void load_lane_logits(const unsigned char* stage_row,
                                                 const T* gl_row_slice, int slice_valid,
                                                 int warp, int lane, float* z) {
  constexpr int NV = kLaneElems / VEC;
  const float ninf = -__int_as_float(0x7f800000);
  if constexpr (VEC == 1) {
#pragma unroll
    for (int k = 0; k < NV; ++k) {
      const int eo = warp * kLaneElems * 32 + k * 32 + lane;
      z[k] = eo < slice_valid ? Elem<T>::load1(gl_row_slice + eo) : ninf;
    }
  } else {
    uint4 raw[NV];
#pragma unroll
    for (int k = 0; k < NV; ++k) {
      const int vi = warp * 32 * NV + k * 32 + lane;
      if (vi * VEC < slice_valid) {
        if constexpr (kTma) {
          raw[k] = reinterpret_cast<const uint4*>(stage_row)[vi];
        } else {
          raw[k] = ld_stream16(gl_row_slice + vi * VEC);
        }
      }
    }
#pragma unroll
    for (int k = 0; k < NV; ++k) {
      const int vi = warp * 32 * NV + k * 32 + lane;
      if (vi * VEC < slice_valid) {
        Elem<T>::unpack(raw[k], z + k * VEC);
      } else {
#pragma unroll
        for (int e = 0; e < VEC; ++e) z[k * VEC + e] = ninf;
      }
    }
  }
}

// Exponentiate the lane's logits against the chunk reference and return the lane's sum.
// ref = fl(max * scale), or 0 for a chunk with no value above -inf (then every finite
// element is absent and only NaN survives, as NaN).
__device__ __forceinline__ float exp_and_sum(float* z, float scale, float ref) {
  float s0 = 0.f, s1 = 0.f;
#pragma unroll
  for (int k = 0; k < kLaneElems; k += 2) {
    z[k] = ex2(__fmaf_rn(z[k], scale, -ref));
    z[k + 1] = ex2(__fmaf_rn(z[k + 1], scale, -ref));
    s0 = __fadd_rn(s0, z[k]);
    s1 = __fadd_rn(s1, z[k + 1]);
  }
  return __fadd_rn(s0, s1);
}

template <typename T, int VEC, bool kTma>
__global__ void __launch_bounds__(kMaxWarps * 32, 1) sample_rowstats_kernel(const SampleParams prm) {
  extern __shared__ __align__(128) unsigned char smem[];
  constexpr int EB = Elem<T>::kBytes;
  const float ninf = -__int_as_float(0x7f800000);

  cg::cluster_group cluster = cg::this_cluster();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int csize = prm.cluster;
  const int crank = static_cast<int>(cluster.block_rank());
  const int cid = blockIdx.x / csize;
  const int K = prm.K, V = prm.V, K1 = K + 1;
  const Rows<T> rows{static_cast<const T*>(prm.p1), static_cast<const T*>(prm.pv),
                     static_cast<const T*>(prm.q), prm.ld_p1, prm.ld_pv, prm.B, K, V};

  const int slice_start = crank * prm.slice_elems;
  const int slice_valid = max(0, min(prm.slice_elems, V - slice_start));
  const size_t slice_bytes = static_cast<size_t>(prm.slice_elems) * EB;
  const int my_units =
      cid < prm.n_units ? (prm.n_units - cid + prm.n_clusters - 1) / prm.n_clusters : 0;

  unsigned char* ring = smem;
  Pass1Smem* sm = reinterpret_cast<Pass1Smem*>(
      smem + (kTma ? pass1_ring_bytes(prm.stages, prm.slice_elems, EB) : 0));

  // Producer: one thread issues the bulk copies of unit t into stage t % stages.
  auto issue = [&](int t) {
    const int u = cid + t * prm.n_clusters;
    const int b = u / K1, i = u - b * K1;
    const bool pair = i < K;
    const int s = t % prm.stages;
    const uint32_t bytes = static_cast<uint32_t>(slice_valid) * EB;
    mbar_arrive_expect_tx(&sm->full[s], pair ? 2u * bytes : bytes);
    if (bytes) {
      unsigned char* dst = ring + static_cast<size_t>(s) * 2 * slice_bytes;
      bulk_g2s(dst, rows.prow(b, i) + slice_start, bytes, &sm->full[s]);
      if (pair) bulk_g2s(dst + slice_bytes, rows.qrow(b, i) + slice_start, bytes, &sm->full[s]);
    }
  };

  bool timed_out = false;
  int issued = 0;     // units whose copies were issued
  int waited = 0;     // units whose copies completed
  if constexpr (kTma) {
    if (tid == 0) {
      for (int s = 0; s < prm.stages; ++s) mbar_init(&sm->full[s], 1);
      fence_mbar_init();
    }
    __syncthreads();
    if (tid == 0) {
      for (; issued < min(prm.stages, my_units); ++issued) issue(issued);
    }
  }

  for (int t = 0; t < my_units; ++t) {
    const int u = cid + t * prm.n_clusters;
    const int b = u / K1, i = u - b * K1;
    const bool pair = i < K;  // uniform over the cluster
    float zp[kLaneElems], zq[kLaneElems];

    if constexpr (kTma) {
      const int s = t % prm.stages;
      bool my_timeout = false;
      if (!timed_out) my_timeout = !mbar_wait_bounded(&sm->full[s], (t / prm.stages) & 1);
      const unsigned char* src = ring + static_cast<size_t>(s) * 2 * slice_bytes;
      load_lane_logits<T, VEC, true>(src, nullptr, slice_valid, warp, lane, zp);
      if (pair) load_lane_logits<T, VEC, true>(src + slice_bytes, nullptr, slice_valid, warp, lane, zq);
      // Every thread has its copy of the stage in registers: the stage is free again.
      timed_out = __syncthreads_or(timed_out || my_timeout) != 0;
      if (!timed_out) waited = t + 1;
      if (tid == 0 && !timed_out && issued < my_units) {
        fence_proxy_async_smem();
        issue(issued++);
      }
    } else {
      load_lane_logits<T, VEC, false>(nullptr, rows.prow(b, i) + slice_start, slice_valid, warp,
                                      lane, zp);
      if (pair)
        load_lane_logits<T, VEC, false>(nullptr, rows.qrow(b, i) + slice_start, slice_valid,
                                        warp, lane, zq);
    }
    if (timed_out) {
#pragma unroll
      for (int k = 0; k < kLaneElems; ++k) zp[k] = zq[k] = __int_as_float(0x7fffffff);
    }

    // 1. chunk maxima and exponentials against the chunk reference
    float mp = ninf, mq = ninf;
#pragma unroll
    for (int k = 0; k < kLaneElems; ++k) mp = fmaxf(mp, zp[k]);
    mp = warp_max(mp);
    const float refp = mp == ninf ? 0.f : __fmul_rn(mp, prm.scale);
    const float sp = warp_sum(exp_and_sum(zp, prm.scale, refp));
    const SoftPart wp{mp == ninf ? ninf : refp, sp};
    SoftPart wq = soft_empty();
    float refq = 0.f;
    if (pair) {
#pragma unroll
      for (int k = 0; k < kLaneElems; ++k) mq = fmaxf(mq, zq[k]);
      mq = warp_max(mq);
      refq = mq == ninf ? 0.f : __fmul_rn(mq, prm.scale);
      const float sq = warp_sum(exp_and_sum(zq, prm.scale, refq));
      wq = SoftPart{mq == ninf ? ninf : refq, sq};
    }

    // 2. CTA merge, then cluster merge over DSMEM (double-buffered slot: one barrier per unit)
    if (lane == 0) sm->red[warp] = make_float4(wp.m, wp.s, wq.m, wq.s);
    __syncthreads();
    if (warp == 0) {
      const float4 v = lane < prm.warps ? sm->red[lane] : make_float4(ninf, 0.f, ninf, 0.f);
      const SoftPart a = warp_soft_merge(SoftPart{v.x, v.y});
      const SoftPart c = warp_soft_merge(SoftPart{v.z, v.w});
      if (lane == 0) sm->dsm[t & 1] = make_float4(a.m, a.s, c.m, c.s);
    }
    cluster.sync();
    float4 rv = make_float4(ninf, 0.f, ninf, 0.f);
    if (lane < csize) rv = *cluster.map_shared_rank(&sm->dsm[t & 1], lane);
    const SoftPart P = warp_soft_merge(SoftPart{rv.x, rv.y});
    const SoftPart Q = pair ? warp_soft_merge(SoftPart{rv.z, rv.w}) : soft_empty();

    // 3. probability factors and chunk masses
    const float cp = mp == ninf ? 0.f : __fdiv_rn(ex2(__fsub_rn(refp, P.m)), P.s);
    const float psum = __fmul_rn(sp, cp);
    float cq = 0.f, rsum = 0.f;
    if (pair) {
      cq = mq == ninf ? 0.f : __fdiv_rn(ex2(__fsub_rn(refq, Q.m)), Q.s);
      float r0 = 0.f, r1 = 0.f;
#pragma unroll
      for (int k = 0; k < kLaneElems; k += 2) {
        r0 = __fadd_rn(r0, fmaxf(__fmaf_rn(zp[k], cp, -__fmul_rn(zq[k], cq)), 0.f));
        r1 = __fadd_rn(r1, fmaxf(__fmaf_rn(zp[k + 1], cp, -__fmul_rn(zq[k + 1], cq)), 0.f));
      }
      rsum = warp_sum(__fadd_rn(r0, r1));
    }

    const int c = crank * prm.warps + warp;
    const int prow = b * K1 + i;
    if (lane == 0 && c < prm.n_chunks) {
      *reinterpret_cast<float4*>(prm.chunk_p + static_cast<size_t>(prow) * prm.n_chunks + c) =
          make_float4(refp, cp, psum, 0.f);
      if (pair)
        *reinterpret_cast<float4*>(prm.chunk_r +
                                   static_cast<size_t>(b * K + i) * prm.n_chunks + c) =
            make_float4(refq, cq, rsum, 0.f);
    }
    if (crank == 0 && tid == 0) {
      prm.rowstat[prow] = make_float2(P.m, P.s);
      if (pair) prm.rowstat[prm.B * K1 + b * K + i] = make_float2(Q.m, Q.s);
    }
    if (tid == 0)
      prm.unit_flags[static_cast<size_t>(u) * csize + crank] =
          timed_out ? static_cast<uint8_t>(DSPARK_SEQ_TIMEOUT) : 0;
  }

  if constexpr (kTma) {
    // Never leave with bulk copies in flight into this CTA's shared memory.
    if (timed_out && tid == 0) {
      for (int t = waited; t < issued; ++t)
        (void)mbar_wait_bounded(&sm->full[t % prm.stages], (t / prm.stages) & 1);
    }
  }
  grid_dependents_launch();
  // No CTA may exit while a peer can still read its DSMEM slot.
  cluster.sync();
}

// ------------------------------------------------------------------------ finish kernel

struct FinishParams {
  const void* p1;
  const void* pv;
  const void* q;
  int64_t ld_p1;
  int64_t ld_pv;
  int B, K, V;
  float scale;
  const int32_t* drafts;
  const float* uniforms;
  int n_chunks;
  int cluster;
  const float2* rowstat;
  const ChunkRec* chunk_p;
  const ChunkRec* chunk_r;
  const uint8_t* unit_flags;
  dspark_accept_out_t out;
};

__device__ __forceinline__ bool stat_ok(float2 st) {
  return is_finite(st.x) && is_finite(st.y) && st.y > 0.f;
}

// Writes the AcceptResult of sequence b. Called by every thread of the block.
__device__ __forceinline__ void write_result(const dspark_accept_out_t& out, const int32_t* drafts,
                                             int b, int K, int j, int token, int status) {
  const int tid = threadIdx.x;
  const bool err = (status & (DSPARK_SEQ_BAD_DRAFT | DSPARK_SEQ_NONFINITE | DSPARK_SEQ_TIMEOUT)) != 0;
  for (int t = tid; t <= K; t += blockDim.x) {
    int v = -1;
    if (!err) v = t < j ? drafts[static_cast<size_t>(b) * K + t] : (t == j ? token : -1);
    out.tokens[static_cast<size_t>(b) * (K + 1) + t] = v;
  }
  if (tid == 0) {
    out.n_accepted[b] = err ? 0 : j;
    out.next_token[b] = err ? -1 : token;
    if (out.status) out.status[b] = status;
  }
}

template <typename T, int VEC>
__global__ void __launch_bounds__(kFinishThreads) sample_finish_kernel(const FinishParams prm) {
  grid_dependency_wait();
  constexpr int NV = kLaneElems / VEC;
  constexpr int CE = 32 * kLaneElems;
  const float ninf = -__int_as_float(0x7f800000);
  const float fnan = __int_as_float(0x7fffffff);
  const int b = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int K = prm.K, V = prm.V, K1 = K + 1, nch = prm.n_chunks;
  const Rows<T> rows{static_cast<const T*>(prm.p1), static_cast<const T*>(prm.pv),
                     static_cast<const T*>(prm.q), prm.ld_p1, prm.ld_pv, prm.B, K, V};

  __shared__ int s_j, s_err, s_chunk, s_lastpos, s_token;
  __shared__ float s_px[kMaxK], s_qx[kMaxK];
  __shared__ double s_incl[kFinishThreads];
  __shared__ double s_wtot[kFinishThreads / 32];

  // A. accept tests: p_i(x_i), q_i(x_i) from the row statistics, first rejection j.
  if (warp == 0) {
    int err = 0;
    bool accept = false;
    float px = fnan, qx = fnan;
    if (lane < K) {
      const int x = prm.drafts[static_cast<size_t>(b) * K + lane];
      const float2 sp = prm.rowstat[b * K1 + lane];
      const float2 sq = prm.rowstat[prm.B * K1 + b * K + lane];
      if (!stat_ok(sp) || !stat_ok(sq)) err |= DSPARK_SEQ_NONFINITE;
      if (x < 0 || x >= V) {
        err |= DSPARK_SEQ_BAD_DRAFT;
      } else {
        const float zp = Elem<T>::load1(rows.prow(b, lane) + x);
        const float zq = Elem<T>::load1(rows.qrow(b, lane) + x);
        px = __fdiv_rn(ex2(__fmaf_rn(zp, prm.scale, -sp.x)), sp.y);
        qx = __fdiv_rn(ex2(__fmaf_rn(zq, prm.scale, -sq.x)), sq.y);
      }
      const float uu = prm.uniforms[static_cast<size_t>(b) * K1 + lane];
      accept = __fmul_rn(uu, qx) < px;
      s_px[lane] = px;
      s_qx[lane] = qx;
    }
    if (lane == 0 && !stat_ok(prm.rowstat[b * K1 + K])) err |= DSPARK_SEQ_NONFINITE;
    for (int f = lane; f < K1 * prm.cluster; f += 32)
      err |= prm.unit_flags[static_cast<size_t>(b) * K1 * prm.cluster + f];
    err = __reduce_or_sync(0xffffffffu, err);
    const unsigned rej = __ballot_sync(0xffffffffu, lane < K && !accept);
    if (lane == 0) {
      s_j = rej ? __ffs(rej) - 1 : K;
      s_err = err;
    }
  }
  __syncthreads();
  const int j = s_j;
  int status = s_err;
  if (status & (DSPARK_SEQ_BAD_DRAFT | DSPARK_SEQ_NONFINITE | DSPARK_SEQ_TIMEOUT)) {
    write_result(prm.out, prm.drafts, b, K, j, -1, status);
    if (prm.out.p_draft && tid < K) prm.out.p_draft[static_cast<size_t>(b) * K + tid] = s_px[tid];
    if (prm.out.q_draft && tid < K) prm.out.q_draft[static_cast<size_t>(b) * K + tid] = s_qx[tid];
    if (prm.out.resid_mass && tid == 0) prm.out.resid_mass[b] = fnan;
    return;
  }

  // B. chunk of the draw: float64 scan of the selected row's chunk masses.
  const float uK = prm.uniforms[static_cast<size_t>(b) * K1 + K];
  bool resid = j < K;
  int jrow = resid ? j : K;  // P row of the draw (residual j, fallback p_j, or bonus p_K)
  double Z = 0.0, excl_c = 0.0, Zres = 0.0;
  int c = -1;
  float tin = 0.f;
  for (int attempt = 0; attempt < 2; ++attempt) {
    const ChunkRec* rec = resid ? prm.chunk_r + static_cast<size_t>(b * K + j) * nch
                                : prm.chunk_p + static_cast<size_t>(b * K1 + jrow) * nch;
    const double m = tid < nch ? static_cast<double>(rec[tid].mass) : 0.0;
    double incl = m;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const double y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane == 31) s_wtot[warp] = incl;
    if (tid == 0) {
      s_chunk = -1;
      s_lastpos = -1;
    }
    __syncthreads();
    double woff = 0.0;
    for (int w = 0; w < warp; ++w) woff += s_wtot[w];
    incl += woff;
    s_incl[tid] = incl;
    Z = 0.0;
    for (int w = 0; w < kFinishThreads / 32; ++w) Z += s_wtot[w];
    __syncthreads();
    if (attempt == 0) Zres = Z;
    if (resid && !(Z > 0.0)) {
      resid = false;  // residual mass rounded to zero: draw from p_j instead
      status |= DSPARK_SEQ_ZERO_RESIDUAL;
      continue;
    }
    const double target = static_cast<double>(uK) * Z;
    const double excl = tid ? s_incl[tid - 1] : 0.0;
    if (tid < nch && m > 0.0) {
      if (excl <= target && target < incl) s_chunk = tid;
      atomicMax(&s_lastpos, tid);
    }
    __syncthreads();
    c = s_chunk;
    if (c >= 0) {
      excl_c = c ? s_incl[c - 1] : 0.0;
      tin = static_cast<float>(target - excl_c);
    } else {
      c = s_lastpos;  // rounding left the target past the last mass: take the last token
      tin = __int_as_float(0x7f800000);
    }
    break;
  }

  // C. pass 2 on the one chunk: recompute the per-element masses exactly as pass 1 did and
  //    take the first token whose running mass passes the target.
  if (warp == 0) {
    int token = -1;
    if (c >= 0) {
      const ChunkRec rp = prm.chunk_p[static_cast<size_t>(b * K1 + jrow) * nch + c];
      ChunkRec rq{0.f, 0.f, 0.f, 0.f};
      if (resid) rq = prm.chunk_r[static_cast<size_t>(b * K + j) * nch + c];
      const int cbase = c * CE;
      const T* prow_c = rows.prow(b, jrow) + cbase;
      const T* qrow_c = resid ? rows.qrow(b, j) + cbase : nullptr;
      const int cvalid = min(CE, V - cbase);
      float zp[kLaneElems], zq[kLaneElems];
      load_lane_logits<T, VEC, false>(nullptr, prow_c, cvalid, 0, lane, zp);
      if (resid) load_lane_logits<T, VEC, false>(nullptr, qrow_c, cvalid, 0, lane, zq);
      float val[kLaneElems];
      int lastpos = -1;
#pragma unroll
      for (int k = 0; k < kLaneElems; ++k) {
        const float ep = ex2(__fmaf_rn(zp[k], prm.scale, -rp.ref));
        if (resid) {
          const float eq = ex2(__fmaf_rn(zq[k], prm.scale, -rq.ref));
          val[k] = fmaxf(__fmaf_rn(ep, rp.c, -__fmul_rn(eq, rq.c)), 0.f);
        } else {
          val[k] = __fmul_rn(ep, rp.c);
        }
        const int e = cbase + ((k / VEC) * 32 + lane) * VEC + (k % VEC);
        if (val[k] > 0.f) lastpos = max(lastpos, e);
      }
      float carry = 0.f;
#pragma unroll
      for (int kv = 0; kv < NV; ++kv) {
        float ls = 0.f;
#pragma unroll
        for (int e = 0; e < VEC; ++e) ls = __fadd_rn(ls, val[kv * VEC + e]);
        float incl = ls;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const float y = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl = __fadd_rn(incl, y);
        }
        float ex = __shfl_up_sync(0xffffffffu, incl, 1);
        if (lane == 0) ex = 0.f;
        const float before = __fadd_rn(carry, ex);
        const float after = __fadd_rn(carry, incl);
        const unsigned hit = __ballot_sync(0xffffffffu, before <= tin && tin < after);
        if (hit) {
          const int hl = __ffs(hit) - 1;
          int cand = -1;
          if (lane == hl) {
            float run = before;
            int lastv = -1;
#pragma unroll
            for (int e = 0; e < VEC; ++e) {
              const float nxt = __fadd_rn(run, val[kv * VEC + e]);
              const int id = cbase + (kv * 32 + lane) * VEC + e;
              if (val[kv * VEC + e] > 0.f) lastv = id;
              if (cand < 0 && run <= tin && tin < nxt) cand = id;
              run = nxt;
            }
            if (cand < 0) cand = lastv;
          }
          token = __shfl_sync(0xffffffffu, cand, hl);
          break;
        }
        carry = __shfl_sync(0xffffffffu, after, 31);
      }
      if (token < 0) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) lastpos = max(lastpos, __shfl_xor_sync(0xffffffffu, lastpos, o));
        token = lastpos;
      }
    }
    if (lane == 0) s_token = token;
  }
  __syncthreads();
  const int token = s_token;
  write_result(prm.out, prm.drafts, b, K, j, token, status);
  if (prm.out.p_draft && tid < K) prm.out.p_draft[static_cast<size_t>(b) * K + tid] = s_px[tid];
  if (prm.out.q_draft && tid < K) prm.out.q_draft[static_cast<size_t>(b) * K + tid] = s_qx[tid];
  if (prm.out.resid_mass && tid == 0)
    prm.out.resid_mass[b] = j < K ? static_cast<float>(Zres) : 1.0f;
  (void)ninf;
}

}  // namespace dspark
