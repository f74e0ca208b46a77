// Early exit: the verify step read row pair by row pair, each sequence stopping at its first
// rejection (or greedy mismatch).
//
// A draft is accepted with probability below one (the DeepSeek-V4-Flash DSpark drafter card
// reports acceptance between 52% and 91%), so most blocks end well before row K, and the rows
// after a sequence's first rejection j cannot change its result. The pairs (P_i, Q_i) are
// taken in waves (wave_schedule below: 1, 2, 4, ... pairs for large batches, 2, 8, 32, ...
// for the others, cut at K), the last wave adding the bonus row P_K. A wave is two launches:
//  - ee_stream_kernel: pass 1 (stream.cuh) over the units of the wave's rows of the
//    sequences still alive, in the same record layout as a full call (so a record, a
//    function of its unit's logits alone, is bit-identical to the full call's);
//  - ee_decide_kernel: per alive sequence, the records of the wave's rows merged and its
//    drafts tested, with exactly the arithmetic of the full finish. A sequence that stops in
//    the wave stores its decision (sampling) or writes its result (greedy); the others are
//    appended to the next wave's list.
// The sampling finish (finish.cuh, kFinEarlyExit) then draws every sequence's token from its
// stored decision. Launch count: two per wave plus the finish when sampling.
//
// Reading of the error rules: the drafts are inputs and are all checked in wave 0 (a bad id
// ends the sequence before any row is read); a row is checked when it is read and lies at or
// before the stop, so a bad row after a sequence's first rejection is never reported.
#pragma once

#include "finish.cuh"

namespace dspark {

constexpr int kMaxWaves = 8;  // K <= 32 takes at most 6 waves, of 1, 2, 4, 8, 16 and 1 pairs

// The wave schedule: waves of `first`, first * growth, ... pairs, cut at K. A wave has a fixed
// cost (the stream's ramp and tail, the decisions' launch and merge: about 5 us), so when a
// row pair of the whole batch is smaller than kEeBigPairBytes (the stream of one pair would
// not hide it) the waves are 2, 8, 32, ... pairs; larger batches take 1, 2, 4, ... pairs.
// (B=64, K=7, V=129280: 2 waves, [0, 2) and [2, 7); B=256, K=15, V=262144: 4 waves.)
struct WaveSchedule {
  int first, growth;
};
constexpr long long kEeBigPairBytes = 64ll << 20;
inline WaveSchedule wave_schedule(long long B, long long V, int elem_bytes, bool sample) {
  const long long pair = B * V * elem_bytes * (sample ? 2 : 1);
  return pair >= kEeBigPairBytes ? WaveSchedule{1, 2} : WaveSchedule{2, 4};
}

// Pairs [lo, hi) of wave w.
inline void wave_range(const WaveSchedule& ws, int w, int K, int& lo, int& hi) {
  long long a = 0, n = ws.first;
  for (int i = 0; i < w && a < K; ++i) {
    a += n;
    n *= ws.growth;
  }
  lo = static_cast<int>(a < K ? a : K);
  hi = static_cast<int>(a + n < K ? a + n : K);
}

// The wave's rows: P_i (and Q_i when sampling) for pairs i in [lo, hi), and P_K in the last.
struct WaveRows {
  int K, lo, hi;
  bool last, q;
  __device__ __forceinline__ bool operator()(int r) const {
    if (r <= K) return (r >= lo && r < hi) || (last && r == K);
    const int i = r - K - 1;
    return q && i >= lo && i < hi;
  }
};

// The wave's place in the call, shared by its two kernels.
struct WaveArgs {
  int lo, hi;
  int last;        // 1: this wave holds the bonus row (and ends every sequence still alive)
  int wave;        // w; wave 0 takes every sequence in order
  const int* alive;  // this wave's sequences (wave > 0), n = cnt[wave]
  int* alive_next;   // the next wave's list
  int* cnt;          // [kMaxWaves]: cnt[w] = sequences alive at wave w (w >= 1)
};

struct EeStreamParams : StreamParams {
  WaveArgs wv;
};

struct EeDecideParams : FinishParams {
  WaveArgs wv;
  Decision* dec;  // [B] (sampling): the decision of the wave that ends the sequence
};

// Pass 1 of a wave. Units are (row slot, alive index, chunk), slot-major as in a full call:
// P_K first in the last wave, then the pairs from hi - 1 down to lo (P_i, then Q_i), so the
// low pairs, where rejections concentrate, are read last and are still in L2 for the finish.
// Lane 0 fetches the sequence of the warp's next unit from the alive list while the warp
// streams the current one, so that lookup is off the critical path.
template <typename T, int VEC, bool kSample>
__global__ void __launch_bounds__(kStreamThreads, 1) ee_stream_kernel(const EeStreamParams p) {
  __shared__ unsigned s_next;
  grid_dependency_wait();
  grid_dependents_launch();
  const WaveArgs& wv = p.wv;
  if (wv.wave == 0 && blockIdx.x == 0 && threadIdx.x < kMaxWaves) wv.cnt[threadIdx.x] = 0;
  const int lane = threadIdx.x & 31;
  const int wi = threadIdx.x >> 5;
  const int V = p.rs.V, K = p.rs.K;
  const uint32_t n_alive = wv.wave == 0 ? static_cast<uint32_t>(p.B)
                                        : static_cast<uint32_t>(__ldcg(wv.cnt + wv.wave));
  constexpr int kPer = kSample ? 2 : 1;
  const uint32_t slots = static_cast<uint32_t>((wv.hi - wv.lo) * kPer + wv.last);
  const uint32_t per_slot = n_alive * static_cast<uint32_t>(p.nch);
  const uint32_t n_units = per_slot * slots;
  const unsigned k = blockIdx.x, G = gridDim.x;
  const unsigned n_mine = k < n_units ? (n_units - 1 - k) / G + 1 : 0;
  if (threadIdx.x == 0) s_next = kStreamWarps;
  __syncthreads();
  // the sequence of this CTA's m-th unit
  const auto seq_of = [&](unsigned m) -> int {
    const uint32_t a = (k + m * G) % per_slot / static_cast<uint32_t>(p.nch);
    return wv.wave == 0 ? static_cast<int>(a) : __ldcg(wv.alive + a);
  };
  unsigned nxt = 0;
  unsigned m = wi;
  int bcur = m < n_mine ? seq_of(m) : 0;
  while (m < n_mine) {
    int bnext = 0;
    if (lane == 0) {
      nxt = atomicAdd(&s_next, 1u);
      if (nxt < n_mine) bnext = seq_of(nxt);
    }
    const unsigned u = k + m * G;
    UnitPos at;
    at.b = bcur;
    at.c = static_cast<int>(u % static_cast<uint32_t>(p.nch));
    const int s = static_cast<int>(u / per_slot) - wv.last;
    if (s < 0) {
      at.i = K;
    } else {
      const int pair = wv.hi - 1 - s / kPer;
      at.i = (s % kPer) ? K + 1 + pair : pair;
    }
    const T* row = row_ptr<T>(p.rs, at.b, at.i);
    const int o0 = at.c * kCE;
    const int o1 = min(V, o0 + kCE);
    float2 rec;
    if constexpr (kSample) {
      const int xd = unit_draft<T, false>(p, at, lane, K);
      rec = piece_softmax<T, VEC>(row, o0, o1, lane, p.scale);
      unit_gather<T>(p, at, row, xd, o0, o1);
    } else {
      rec = piece_argmax<T, VEC>(row, o0, o1, lane);
    }
    if (lane == 0) p.rec[record_index(p, at)] = rec;
    m = __shfl_sync(0xffffffffu, nxt, 0);
    bcur = __shfl_sync(0xffffffffu, bnext, 0);
  }
}

__device__ __forceinline__ bool argmax_bad(float2 a) {
  // NaN anywhere, a +inf maximum, or nothing above -inf
  return !(a.x > -__int_as_float(0x7f800000)) || !(a.x < __int_as_float(0x7f800000)) ||
         __float_as_int(a.y) == INT_MAX;
}

// The decisions of a wave: one CTA per sequence alive at it (the grid covers B; CTAs past the
// alive count return at once). Merges the wave's rows, then warp 0 tests draft i on lane i for
// i in [lo, hi), with the full finish's arithmetic; the first lane whose rows are bad or whose
// test fails is the stop j (a bad row there is an error). No stop and no bonus row in this
// wave: the sequence goes on to the next wave.
template <bool kSample>
__global__ void __launch_bounds__(kThreads) ee_decide_kernel(const EeDecideParams p) {
  __shared__ float2 s_stat[kMaxRows];
  __shared__ int s_x[kMaxK];
  grid_dependents_launch();
  const WaveArgs& wv = p.wv;
  const int tid = threadIdx.x, lane = tid & 31, wi = tid >> 5;
  const int K = p.rs.K, K1 = K + 1, V = p.rs.V;
  grid_dependency_wait();
  const int n_alive = wv.wave == 0 ? static_cast<int>(gridDim.x) : __ldcg(wv.cnt + wv.wave);
  if (static_cast<int>(blockIdx.x) >= n_alive) return;
  const int b = wv.wave == 0 ? static_cast<int>(blockIdx.x) : __ldcg(wv.alive + blockIdx.x);
  const WaveRows rows{K, wv.lo, wv.hi, wv.last != 0, kSample};
  merge_rows<kSample, true, kWarps, WaveRows>(p, b, rows, wi, lane, s_stat);
  __syncthreads();
  if (wi != 0) return;

  const float fnan = __int_as_float(0x7fffffff);
  const int x = lane < K ? p.drafts[static_cast<size_t>(b) * K + lane] : 0;
  if (lane < K) s_x[lane] = x;
  __syncwarp();
  if (wv.wave == 0 && __any_sync(0xffffffffu, lane < K && (x < 0 || x >= V))) {
    write_error(p, b, DSPARK_SEQ_BAD_DRAFT, lane, 32);
    if constexpr (kSample) {
      if (lane < K && p.out.p_draft) p.out.p_draft[static_cast<size_t>(b) * K + lane] = fnan;
      if (lane < K && p.out.q_draft) p.out.q_draft[static_cast<size_t>(b) * K + lane] = fnan;
      if (lane == 0) {
        Decision d{};
        d.status = DSPARK_SEQ_BAD_DRAFT;
        p.dec[b] = d;
      }
    }
    return;
  }

  const bool in = lane >= wv.lo && lane < wv.hi;
  bool bad = false, pass = true;
  float px = fnan, qx = fnan;
  if (in) {
    if constexpr (kSample) {
      const float2 sp = s_stat[lane], sq = s_stat[K1 + lane];
      bad = !stat_ok(sp) || !stat_ok(sq);
      const float2 zg =
          __ldcg(reinterpret_cast<const float2*>(p.gather) + static_cast<size_t>(b) * K + lane);
      px = __fdividef(ex2(__fmaf_rn(zg.x, p.scale, -sp.x)), sp.y);
      qx = __fdividef(ex2(__fmaf_rn(zg.y, p.scale, -sq.x)), sq.y);
      pass = __fmul_rn(p.uniforms[static_cast<size_t>(b) * K1 + lane], qx) < px;
    } else {
      const float2 a = s_stat[lane];
      bad = argmax_bad(a);
      pass = x == __float_as_int(a.y);
    }
  }
  const unsigned stops = __ballot_sync(0xffffffffu, in && (bad || !pass));
  int j = -1, status = 0;
  if (stops) {
    j = __ffs(stops) - 1;
    if (__shfl_sync(0xffffffffu, bad, j)) status = DSPARK_SEQ_NONFINITE;
  } else if (wv.last) {
    j = K;
    const float2 a = s_stat[K];
    if (kSample ? !stat_ok(a) : argmax_bad(a)) status = DSPARK_SEQ_NONFINITE;
  }
  if constexpr (kSample) {
    // the tested drafts' probabilities up to the stop; NaN past it, through row K-1
    const bool ends = j >= 0;
    if (lane < K && lane >= wv.lo && (in || ends)) {
      const bool val = in && (!ends || lane <= j);
      if (p.out.p_draft) p.out.p_draft[static_cast<size_t>(b) * K + lane] = val ? px : fnan;
      if (p.out.q_draft) p.out.q_draft[static_cast<size_t>(b) * K + lane] = val ? qx : fnan;
    }
  }
  if (j < 0) {  // every draft of the wave accepted: on to the next wave
    if (lane == 0) wv.alive_next[atomicAdd(wv.cnt + wv.wave + 1, 1)] = b;
    return;
  }
  if (status) {
    write_error(p, b, status, lane, 32);
    if constexpr (kSample) {
      if (lane == 0) {
        Decision d{};
        d.status = status;
        p.dec[b] = d;
      }
    }
    return;
  }
  if constexpr (kSample) {
    if (lane == 0) {
      const float2 sp = s_stat[j];
      Decision d;
      d.j = j;
      d.nd = K;
      d.status = 0;
      d.mp = sp.x;
      d.ip = __fdividef(1.f, sp.y);
      if (j < K) {
        const float2 sq = s_stat[K1 + j];
        d.mq = sq.x;
        d.iq = __fdividef(1.f, sq.y);
      } else {
        d.mq = 0.f;
        d.iq = 0.f;
      }
      p.dec[b] = d;
    }
  } else {
    write_tokens(p, b, j, __float_as_int(s_stat[j].y), s_x, lane, 32);
    if (lane == 0 && p.out.status) p.out.status[b] = 0;
  }
}

}  // namespace dspark
