// speculative_sample_accept on sm_100a: pass 1 (row statistics and chunk masses) and the
// finish kernel (decide, then the pass-2 inverse-CDF draw on the one selected chunk).
//
// Pass 1 is a persistent kernel over thread-block clusters. A work unit is one position i of
// one sequence b: the pair (P row i, Q row i) for i < K, or the bonus row P_K alone. The V
// axis of a unit is split over the CTAs of a cluster and, within a CTA, over its warps: warp
// w of CTA r owns the contiguous chunk c = r * warps + w of 1024 tokens (32 lanes x 32
// register-resident logits). Each row element is read from HBM exactly once:
//   * every warp runs its own ring of shared-memory stages filled by 1-D bulk copies
//     (cp.async.bulk, no multicast) completing on per-warp mbarriers, so a warp refills the
//     stage it has just read without waiting for the rest of the CTA;
//   * the chunk's logits land in registers and stay there until the unit is done: chunk max,
//     one 2^x per element against the chunk's own reference, chunk sums (packed f32x2 math);
//   * the last warp of the CTA to finish merges the warp parts and st.async-es the CTA part
//     into every CTA of the cluster, completing on their exchange mbarrier; each warp then
//     merges the cluster's parts into the row's (max, sum) for P_i and Q_i - no cluster-wide
//     barrier per unit;
//   * per chunk, the factors c = 2^(ref - M) / S that turn the register exponentials into
//     probabilities, and from registers the residual mass sum_v max(p[v] - q[v], 0) of the
//     chunk (no second read of the row).
// The finish kernel (one CTA per sequence) gathers p_i(x_i), q_i(x_i), finds the first
// rejection j, scans the chunk masses of the selected row (residual j, or P_K for the bonus)
// in float64 to find the chunk holding the draw, re-reads only that chunk and redoes the
// per-element arithmetic bit for bit to pick the token.
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
  int stages;         // per-warp ring depth (bulk-copy variant)
  float2* rowstat;    // [B*(K+1) P rows, then B*K Q rows]: (M, S)
  ChunkRec* chunk_p;  // [B*(K+1), n_chunks]
  ChunkRec* chunk_r;  // [B*K, n_chunks]
  uint8_t* unit_flags;  // [B*(K+1), cluster, warps]
};

// Shared memory of the pass-1 kernel after the stage rings.
struct Pass1Smem {
  uint64_t full[kMaxWarps * kMaxStages];  // per-warp ring stages
  uint64_t xbar[2];                       // cluster exchange, by unit parity
  float4 red[2][kMaxWarps];               // warp parts, by unit parity
  float4 slot[2][kMaxCluster];            // CTA parts received from the cluster
  unsigned cnt[2];                        // warps done with units of each parity
};

__host__ __device__ inline size_t pass1_ring_bytes(int warps, int stages, int elem_bytes) {
  return static_cast<size_t>(warps) * stages * 2 * kChunkElems * elem_bytes;
}

// This lane's 32 logits of one chunk: z[k*VEC + e] is token (k*32 + lane)*VEC + e of the
// chunk (k*32 + lane for the scalar path). Tokens at or past `valid` read as -inf.
template <typename T, int VEC, bool kFromSmem>
__device__ __forceinline__ void load_chunk(const unsigned char* smem_chunk, const T* gl_chunk,
                                           int valid, int lane, float* z) {
  constexpr int NV = kLaneElems / VEC;
  const float ninf = -__int_as_float(0x7f800000);
  if constexpr (VEC == 1) {
#pragma unroll
    for (int k = 0; k < NV; ++k) {
      const int e = k * 32 + lane;
      z[k] = e < valid ? Elem<T>::load1(gl_chunk + e) : ninf;
    }
  } else {
    uint4 raw[NV];
    const bool full_chunk = valid >= kChunkElems;
#pragma unroll
    for (int k = 0; k < NV; ++k) {
      const int vi = k * 32 + lane;
      if (full_chunk || vi * VEC < valid) {
        if constexpr (kFromSmem) {
          raw[k] = reinterpret_cast<const uint4*>(smem_chunk)[vi];
        } else {
          raw[k] = ld_stream16(gl_chunk + vi * VEC);
        }
      }
    }
#pragma unroll
    for (int k = 0; k < NV; ++k) {
      const int vi = k * 32 + lane;
      if (full_chunk || vi * VEC < valid) {
        Elem<T>::unpack(raw[k], z + k * VEC);
      } else {
#pragma unroll
        for (int e = 0; e < VEC; ++e) z[k * VEC + e] = ninf;
      }
    }
  }
}

// Chunk reference: fl(max * scale), 0 when the chunk has no value above -inf; NaN when the
// chunk holds a NaN (or +inf, through inf - inf), which then poisons the row's sum.
struct ChunkExp {
  float max;  // raw max (NaN-propagating)
  float ref;  // reference the exponentials are taken against
  float sum;  // warp-reduced sum of 2^(z*scale - ref)
};

__device__ __forceinline__ ChunkExp chunk_exp(float* z, float scale) {
  const float ninf = -__int_as_float(0x7f800000);
  float m = ninf;
#pragma unroll
  for (int k = 0; k < kLaneElems; k += 2) m = max3_nan(m, z[k], z[k + 1]);
  m = warp_max_nan(m);
  const float ref = m == ninf ? 0.f : __fmul_rn(m, scale);
  const uint64_t s2 = pk2(scale, scale);
  const uint64_t nr2 = pk2(-ref, -ref);
  uint64_t acc = pk2(0.f, 0.f);
#pragma unroll
  for (int k = 0; k < kLaneElems; k += 2) {
    float a0, a1;
    upk2(fma2(pk2(z[k], z[k + 1]), s2, nr2), a0, a1);
    z[k] = ex2(a0);
    z[k + 1] = ex2(a1);
    acc = add2(acc, pk2(z[k], z[k + 1]));
  }
  float lo, hi;
  upk2(acc, lo, hi);
  return {m, ref, warp_sum(__fadd_rn(lo, hi))};
}

template <typename T, int VEC, bool kTma>
__global__ void __launch_bounds__(kMaxWarps * 32, 1) sample_rowstats_kernel(const SampleParams prm) {
  extern __shared__ __align__(128) unsigned char smem[];
  constexpr int EB = Elem<T>::kBytes;
  constexpr uint32_t kChunkBytes = kChunkElems * EB;
  const float ninf = -__int_as_float(0x7f800000);
  const float fnan = __int_as_float(0x7fffffff);

  cg::cluster_group cluster = cg::this_cluster();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int W = prm.warps, C = prm.cluster, S = prm.stages;
  const int crank = static_cast<int>(cluster.block_rank());
  const int cid = blockIdx.x / C;
  const int K = prm.K, V = prm.V, K1 = K + 1;
  const Rows<T> rows{static_cast<const T*>(prm.p1), static_cast<const T*>(prm.pv),
                     static_cast<const T*>(prm.q), prm.ld_p1, prm.ld_pv, prm.B, K, V};

  const int chunk = crank * W + warp;  // this warp's chunk of every row
  const int c0 = chunk * kChunkElems;
  const int cvalid = max(0, min(kChunkElems, V - c0));
  const uint32_t cbytes = static_cast<uint32_t>(cvalid) * EB;
  const int my_units =
      cid < prm.n_units ? (prm.n_units - cid + prm.n_clusters - 1) / prm.n_clusters : 0;

  unsigned char* my_ring =
      smem + (kTma ? static_cast<size_t>(warp) * S * 2 * kChunkBytes : 0);
  Pass1Smem* sm = reinterpret_cast<Pass1Smem*>(smem + (kTma ? pass1_ring_bytes(W, S, EB) : 0));

  // Lane 0 of each warp issues the copies of its own chunk of unit t into stage t % S.
  auto issue = [&](int t) {
    const int u = cid + t * prm.n_clusters;
    const int b = u / K1, i = u - b * K1;
    const bool pair = i < K;
    const int s = t % S;
    uint64_t* bar = &sm->full[warp * kMaxStages + s];
    mbar_arrive_expect_tx(bar, pair ? 2u * cbytes : cbytes);
    if (cbytes) {
      unsigned char* dst = my_ring + static_cast<size_t>(s) * 2 * kChunkBytes;
      bulk_g2s(dst, rows.prow(b, i) + c0, cbytes, bar);
      if (pair) bulk_g2s(dst + kChunkBytes, rows.qrow(b, i) + c0, cbytes, bar);
    }
  };

  if (threadIdx.x == 0) {
    if constexpr (kTma) {
      for (int w = 0; w < W; ++w)
        for (int s = 0; s < S; ++s) mbar_init(&sm->full[w * kMaxStages + s], 1);
    }
    mbar_init(&sm->xbar[0], 1);
    mbar_init(&sm->xbar[1], 1);
    sm->cnt[0] = sm->cnt[1] = 0;
    fence_mbar_init();
  }
  // Every CTA's barriers must exist before any peer st.async-es into them.
  cluster.sync();

  bool dead = false;  // a bounded wait gave up: stop waiting, poison results, keep exchanging
  int issued = 0, waited = 0;
  if constexpr (kTma) {
    if (lane == 0)
      for (; issued < min(S, my_units); ++issued) issue(issued);
    issued = __shfl_sync(0xffffffffu, issued, 0);
  }

  for (int t = 0; t < my_units; ++t) {
    const int u = cid + t * prm.n_clusters;
    const int b = u / K1, i = u - b * K1;
    const bool pair = i < K;  // uniform over the cluster
    const int par = t & 1;
    float zp[kLaneElems], zq[kLaneElems];

    if constexpr (kTma) {
      const int s = t % S;
      if (!dead) dead = !mbar_wait_bounded(&sm->full[warp * kMaxStages + s], (t / S) & 1);
      const unsigned char* src = my_ring + static_cast<size_t>(s) * 2 * kChunkBytes;
      load_chunk<T, VEC, true>(src, nullptr, cvalid, lane, zp);
      if (pair) load_chunk<T, VEC, true>(src + kChunkBytes, nullptr, cvalid, lane, zq);
      dead = __any_sync(0xffffffffu, dead);
      __syncwarp();
      if (!dead) waited = t + 1;
      if (lane == 0 && !dead && issued < my_units) {
        fence_proxy_async_smem();  // our reads of the stage precede the refill
        issue(issued);
      }
      if (!dead && issued < my_units) ++issued;
    } else {
      load_chunk<T, VEC, false>(nullptr, rows.prow(b, i) + c0, cvalid, lane, zp);
      if (pair) load_chunk<T, VEC, false>(nullptr, rows.qrow(b, i) + c0, cvalid, lane, zq);
    }
    if (dead) {
#pragma unroll
      for (int k = 0; k < kLaneElems; ++k) zp[k] = zq[k] = fnan;
    }

    // 1. chunk maxima, exponentials, chunk sums
    const ChunkExp ep = chunk_exp(zp, prm.scale);
    ChunkExp eq{ninf, 0.f, 0.f};
    if (pair) eq = chunk_exp(zq, prm.scale);

    // 2. CTA merge by the last warp, then exchange over the cluster
    if (lane == 0)
      sm->red[par][warp] = make_float4(ep.max == ninf ? ninf : ep.ref, ep.sum,
                                       eq.max == ninf ? ninf : eq.ref, eq.sum);
    __syncwarp();
    // Per-parity counters only grow: each unit adds W, so the unit's last warp is the one that
    // sees old % W == W - 1 (a warp reaches unit t+2 only after every warp finished unit t).
    unsigned old = 0;
    if (lane == 0) old = smem_atomic_add_acq_rel(&sm->cnt[par], 1u);
    old = __shfl_sync(0xffffffffu, old, 0);
    if (old % static_cast<unsigned>(W) == static_cast<unsigned>(W - 1)) {
      const float4 v = lane < W ? sm->red[par][lane] : make_float4(ninf, 0.f, ninf, 0.f);
      const SoftPart a = warp_soft_merge_lanes(v.x, v.y);
      const SoftPart c = warp_soft_merge_lanes(v.z, v.w);
      if (lane == 0) mbar_arrive_expect_tx(&sm->xbar[par], static_cast<uint32_t>(C) * 16u);
      __syncwarp();
      if (lane < C) st_async_peer(&sm->slot[par][crank], &sm->xbar[par], lane,
                                  make_float4(a.m, a.s, c.m, c.s));
    }
    if (!dead) dead = !mbar_wait_cluster_bounded(&sm->xbar[par], (t >> 1) & 1);
    dead = __any_sync(0xffffffffu, dead);
    const float4 rv = lane < C ? sm->slot[par][lane] : make_float4(ninf, 0.f, ninf, 0.f);
    SoftPart P = warp_soft_merge_lanes(rv.x, rv.y);
    SoftPart Q = pair ? warp_soft_merge_lanes(rv.z, rv.w) : soft_empty();
    if (dead) P.s = Q.s = fnan;

    // 3. probability factors, residual and chunk masses
    const float cp = ep.max == ninf ? 0.f : __fdiv_rn(ex2(__fsub_rn(ep.ref, P.m)), P.s);
    const float psum = __fmul_rn(ep.sum, cp);
    float cq = 0.f, rsum = 0.f;
    if (pair) {
      cq = eq.max == ninf ? 0.f : __fdiv_rn(ex2(__fsub_rn(eq.ref, Q.m)), Q.s);
      const uint64_t cp2 = pk2(cp, cp), ncq2 = pk2(-cq, -cq);
      uint64_t racc = pk2(0.f, 0.f);
#pragma unroll
      for (int k = 0; k < kLaneElems; k += 2) {
        const uint64_t tq = mul2(pk2(zq[k], zq[k + 1]), ncq2);
        float r0, r1;
        upk2(fma2(pk2(zp[k], zp[k + 1]), cp2, tq), r0, r1);
        racc = add2(racc, pk2(fmaxf(r0, 0.f), fmaxf(r1, 0.f)));
      }
      float lo, hi;
      upk2(racc, lo, hi);
      rsum = warp_sum(__fadd_rn(lo, hi));
    }

    const int prow = b * K1 + i;
    if (lane == 0) {
      if (chunk < prm.n_chunks) {
        *reinterpret_cast<float4*>(prm.chunk_p + static_cast<size_t>(prow) * prm.n_chunks +
                                   chunk) = make_float4(ep.ref, cp, psum, 0.f);
        if (pair)
          *reinterpret_cast<float4*>(prm.chunk_r +
                                     static_cast<size_t>(b * K + i) * prm.n_chunks + chunk) =
              make_float4(eq.ref, cq, rsum, 0.f);
      }
      if (crank == 0 && warp == 0) {
        prm.rowstat[prow] = make_float2(P.m, P.s);
        if (pair) prm.rowstat[prm.B * K1 + b * K + i] = make_float2(Q.m, Q.s);
      }
      prm.unit_flags[(static_cast<size_t>(u) * C + crank) * W + warp] =
          dead ? static_cast<uint8_t>(DSPARK_SEQ_TIMEOUT) : 0;
    }
  }

  if constexpr (kTma) {
    // Never leave with bulk copies in flight into this CTA's shared memory.
    if (dead && lane == 0) {
      for (int t = waited; t < issued; ++t)
        (void)mbar_wait_bounded(&sm->full[warp * kMaxStages + t % S], (t / S) & 1);
    }
  }
  grid_dependents_launch();
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
  int warps;
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
  const bool err =
      (status & (DSPARK_SEQ_BAD_DRAFT | DSPARK_SEQ_NONFINITE | DSPARK_SEQ_TIMEOUT)) != 0;
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

// Block-wide inclusive float64 scan of one value per thread (kFinishThreads threads).
// Leaves every thread's inclusive prefix in incl[] and returns the total.
__device__ __forceinline__ double block_scan_incl(double m, double* incl, double* wtot) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  double x = m;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const double y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) wtot[warp] = x;
  __syncthreads();
  double off = 0.0, tot = 0.0;
  for (int w = 0; w < kFinishThreads / 32; ++w) {
    if (w < warp) off += wtot[w];
    tot += wtot[w];
  }
  incl[tid] = x + off;
  __syncthreads();
  return tot;
}

template <typename T, int VEC>
__global__ void __launch_bounds__(kFinishThreads) sample_finish_kernel(const FinishParams prm) {
  constexpr int NV = kLaneElems / VEC;
  const float fnan = __int_as_float(0x7fffffff);
  const int b = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int K = prm.K, V = prm.V, K1 = K + 1, nch = prm.n_chunks;
  const Rows<T> rows{static_cast<const T*>(prm.p1), static_cast<const T*>(prm.pv),
                     static_cast<const T*>(prm.q), prm.ld_p1, prm.ld_pv, prm.B, K, V};

  __shared__ int s_j, s_err, s_chunk, s_lastpos, s_token;
  __shared__ float s_px[kMaxK], s_qx[kMaxK];
  __shared__ float s_mass[(kMaxK + 1) * kMaxChunks];
  __shared__ double s_incl[kFinishThreads];
  __shared__ double s_wtot[kFinishThreads / 32];

  // A0. Inputs only (no dependence on pass 1): drafts, the draft logits, the uniforms.
  int x = 0;
  float zpx = 0.f, zqx = 0.f, ui = 0.f;
  bool bad_draft = false;
  if (warp == 0 && lane < K) {
    x = prm.drafts[static_cast<size_t>(b) * K + lane];
    bad_draft = x < 0 || x >= V;
    if (!bad_draft) {
      zpx = Elem<T>::load1(rows.prow(b, lane) + x);
      zqx = Elem<T>::load1(rows.qrow(b, lane) + x);
    }
    ui = prm.uniforms[static_cast<size_t>(b) * K1 + lane];
  }
  const float uK = prm.uniforms[static_cast<size_t>(b) * K1 + K];

  grid_dependency_wait();

  // A1. Everything pass 1 wrote that the decision may need, in one round trip.
  for (int e = tid; e < K1 * nch; e += kFinishThreads) {
    const int r = e / nch, c = e - r * nch;
    s_mass[e] = r < K ? prm.chunk_r[static_cast<size_t>(b * K + r) * nch + c].mass
                      : prm.chunk_p[static_cast<size_t>(b * K1 + K) * nch + c].mass;
  }
  int flags = 0;
  const int nflags = K1 * prm.cluster * prm.warps;
  const uint8_t* fl = prm.unit_flags + static_cast<size_t>(b) * nflags;
  for (int f = tid; f < nflags; f += kFinishThreads) flags |= fl[f];
  flags = __syncthreads_or(flags) ? DSPARK_SEQ_TIMEOUT : 0;

  if (warp == 0) {
    int err = flags;
    bool accept = false;
    if (lane < K) {
      const float2 sp = prm.rowstat[b * K1 + lane];
      const float2 sq = prm.rowstat[prm.B * K1 + b * K + lane];
      if (!stat_ok(sp) || !stat_ok(sq)) err |= DSPARK_SEQ_NONFINITE;
      if (bad_draft) err |= DSPARK_SEQ_BAD_DRAFT;
      float px = fnan, qx = fnan;
      if (!bad_draft) {
        px = __fdiv_rn(ex2(__fmaf_rn(zpx, prm.scale, -sp.x)), sp.y);
        qx = __fdiv_rn(ex2(__fmaf_rn(zqx, prm.scale, -sq.x)), sq.y);
      }
      accept = __fmul_rn(ui, qx) < px;
      s_px[lane] = px;
      s_qx[lane] = qx;
    }
    if (lane == 0 && !stat_ok(prm.rowstat[b * K1 + K])) err |= DSPARK_SEQ_NONFINITE;
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

  // B. Chunk of the draw: float64 scan of the selected row's chunk masses.
  bool resid = j < K;
  const int jrow = resid ? j : K;  // P row of the draw (residual j, fallback p_j, bonus p_K)
  double Zres = 0.0;
  int c = -1;
  float tin = 0.f;
  for (int attempt = 0; attempt < 2; ++attempt) {
    double m = 0.0;
    if (tid < nch) {
      if (attempt == 0) m = static_cast<double>(s_mass[jrow * nch + tid]);
      else m = static_cast<double>(prm.chunk_p[static_cast<size_t>(b * K1 + jrow) * nch + tid].mass);
    }
    if (tid == 0) {
      s_chunk = -1;
      s_lastpos = -1;
    }
    const double Z = block_scan_incl(m, s_incl, s_wtot);
    if (attempt == 0) Zres = Z;
    if (resid && !(Z > 0.0)) {
      resid = false;  // residual mass rounded to zero: draw from p_j instead
      status |= DSPARK_SEQ_ZERO_RESIDUAL;
      continue;
    }
    const double target = static_cast<double>(uK) * Z;
    const double incl = s_incl[tid];
    const double excl = tid ? s_incl[tid - 1] : 0.0;
    if (tid < nch && m > 0.0) {
      if (excl <= target && target < incl) s_chunk = tid;
      atomicMax(&s_lastpos, tid);
    }
    __syncthreads();
    c = s_chunk;
    if (c >= 0) {
      tin = static_cast<float>(target - (c ? s_incl[c - 1] : 0.0));
    } else {
      c = s_lastpos;  // rounding left the target past the last mass: take the last token
      tin = __int_as_float(0x7f800000);
    }
    break;
  }

  // C. Pass 2 on the one chunk: recompute the per-element masses exactly as pass 1 did and
  //    take the first token whose running mass passes the target.
  if (warp == 0) {
    int token = -1;
    if (c >= 0) {
      const ChunkRec rp = prm.chunk_p[static_cast<size_t>(b * K1 + jrow) * nch + c];
      ChunkRec rq{0.f, 0.f, 0.f, 0.f};
      if (resid) rq = prm.chunk_r[static_cast<size_t>(b * K + j) * nch + c];
      const int cbase = c * kChunkElems;
      const int cvalid = min(kChunkElems, V - cbase);
      float zp[kLaneElems], zq[kLaneElems];
      load_chunk<T, VEC, false>(nullptr, rows.prow(b, jrow) + cbase, cvalid, lane, zp);
      if (resid) load_chunk<T, VEC, false>(nullptr, rows.qrow(b, j) + cbase, cvalid, lane, zq);
      float val[kLaneElems];
      int lastpos = -1;
#pragma unroll
      for (int k = 0; k < kLaneElems; ++k) {
        const float ep = ex2(__fmaf_rn(zp[k], prm.scale, -rp.ref));
        if (resid) {
          const float eq = ex2(__fmaf_rn(zq[k], prm.scale, -rq.ref));
          val[k] = fmaxf(__fmaf_rn(ep, rp.c, __fmul_rn(eq, -rq.c)), 0.f);
        } else {
          val[k] = __fmul_rn(ep, rp.c);
        }
        const int e = cbase + ((k / VEC) * 32 + lane) * VEC + (k % VEC);
        if (val[k] > 0.f) lastpos = max(lastpos, e);
      }
      float carry = 0.f;
      int hit_kv = -1, hit_lane = -1;
      float hit_before = 0.f;
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
        if (hit && hit_kv < 0) {
          hit_kv = kv;
          hit_lane = __ffs(hit) - 1;
          hit_before = __shfl_sync(0xffffffffu, before, hit_lane);
        }
        carry = __shfl_sync(0xffffffffu, after, 31);
      }
      if (hit_kv >= 0) {
        int cand = -1;
        if (lane == hit_lane) {
          float run = hit_before;
          int lastv = -1;
#pragma unroll
          for (int kv = 0; kv < NV; ++kv) {
            if (kv != hit_kv) continue;
#pragma unroll
            for (int e = 0; e < VEC; ++e) {
              const float v = val[kv * VEC + e];
              const float nxt = __fadd_rn(run, v);
              const int id = cbase + (kv * 32 + lane) * VEC + e;
              if (v > 0.f) lastv = id;
              if (cand < 0 && run <= tin && tin < nxt) cand = id;
              run = nxt;
            }
          }
          if (cand < 0) cand = lastv;
        }
        token = __shfl_sync(0xffffffffu, cand, hit_lane);
      }
      if (token < 0) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
          lastpos = max(lastpos, __shfl_xor_sync(0xffffffffu, lastpos, o));
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
}

}  // namespace dspark
