// greedy_accept on sm_100a.
//
// Pass 1 streams the K+1 base rows of every sequence once (P only; Q is never read) and
// computes, per 8192-token slice of a row, the lowest-index maximum and whether a NaN was
// seen. Each thread walks its 32 elements in ascending token order with a strict ">" so it
// keeps the first of equal maxima; the warp/CTA merges break ties toward the lower index.
// Float comparison makes -0.0 and +0.0 equal, as the definition asks.
// The finish kernel (one CTA per sequence) merges the slices of each row into a_r, accepts
// drafts while x_i == a_i, and emits a_j (the greedy semantics of plain sequential decoding).
#pragma once

#include <climits>

#include "common.cuh"

namespace dspark {

constexpr int kGreedyThreads = 256;
constexpr int kGreedyThreadElems = 32;
constexpr int kGreedySliceElems = kGreedyThreads * kGreedyThreadElems;  // 8192

struct GreedyParams {
  const void* p1;
  const void* pv;
  int64_t ld_p1;
  int64_t ld_pv;
  int B, K, V;
  const int32_t* drafts;
  int slices;    // CTAs per row
  int4* part;    // [B*(K+1), slices]: {max value bits, index (INT_MAX: none), nan seen, 0}
  dspark_accept_out_t out;
};

struct ArgBest {
  float v;
  int i;
};

// Lower index wins among equal values; no value is NaN here.
__device__ __forceinline__ ArgBest arg_better(ArgBest a, ArgBest b) {
  return (b.v > a.v || (b.v == a.v && b.i < a.i)) ? b : a;
}

__device__ __forceinline__ ArgBest warp_arg_best(ArgBest a) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    ArgBest b{__shfl_xor_sync(0xffffffffu, a.v, o), __shfl_xor_sync(0xffffffffu, a.i, o)};
    a = arg_better(a, b);
  }
  return a;
}

template <typename T, int VEC>
__global__ void __launch_bounds__(kGreedyThreads) greedy_argmax_kernel(const GreedyParams prm) {
  constexpr int G = kGreedyThreadElems / VEC;  // loads per thread
  const float ninf = -__int_as_float(0x7f800000);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int K1 = prm.K + 1;
  const int row = blockIdx.x / prm.slices;
  const int sl = blockIdx.x - row * prm.slices;
  const int b = row / K1, i = row - b * K1;
  const Rows<T> rows{static_cast<const T*>(prm.p1), static_cast<const T*>(prm.pv), nullptr,
                     prm.ld_p1, prm.ld_pv, prm.B, prm.K, prm.V};
  const T* base = rows.prow(b, i);
  const int V = prm.V;
  const int sbase = sl * kGreedySliceElems;

  float z[kGreedyThreadElems];
  if constexpr (VEC == 1) {
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const int e = sbase + g * kGreedyThreads + tid;
      z[g] = e < V ? Elem<T>::load1(base + e) : ninf;
    }
  } else {
    uint4 raw[G];
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const int e = sbase + (g * kGreedyThreads + tid) * VEC;
      if (e < V) raw[g] = ld_stream16(base + e);
    }
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const int e = sbase + (g * kGreedyThreads + tid) * VEC;
      if (e < V) {
        Elem<T>::unpack(raw[g], z + g * VEC);
      } else {
#pragma unroll
        for (int k = 0; k < VEC; ++k) z[g * VEC + k] = ninf;
      }
    }
  }

  ArgBest best{ninf, INT_MAX};
  bool nan = false;
#pragma unroll
  for (int g = 0; g < G; ++g) {
#pragma unroll
    for (int k = 0; k < VEC; ++k) {
      const float v = z[g * VEC + k];
      const int e = VEC == 1 ? sbase + g * kGreedyThreads + tid
                             : sbase + (g * kGreedyThreads + tid) * VEC + k;
      if (v > best.v) best = ArgBest{v, e};
      nan |= v != v;
    }
  }
  best = warp_arg_best(best);
  const bool any_nan = __any_sync(0xffffffffu, nan);

  __shared__ ArgBest s_best[kGreedyThreads / 32];
  __shared__ int s_nan[kGreedyThreads / 32];
  if (lane == 0) {
    s_best[warp] = best;
    s_nan[warp] = any_nan;
  }
  __syncthreads();
  if (warp == 0) {
    ArgBest a = lane < kGreedyThreads / 32 ? s_best[lane] : ArgBest{ninf, INT_MAX};
    int n = lane < kGreedyThreads / 32 ? s_nan[lane] : 0;
    a = warp_arg_best(a);
    n = __reduce_or_sync(0xffffffffu, n);
    if (lane == 0)
      prm.part[static_cast<size_t>(row) * prm.slices + sl] = make_int4(__float_as_int(a.v), a.i, n, 0);
  }
  grid_dependents_launch();
}

template <int WARPS>
__global__ void __launch_bounds__(WARPS * 32) greedy_finish_kernel(const GreedyParams prm) {
  grid_dependency_wait();
  const float ninf = -__int_as_float(0x7f800000);
  const int b = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int K = prm.K, K1 = K + 1;
  __shared__ int s_arg[kMaxK + 1];
  __shared__ int s_bad[kMaxK + 1];
  __shared__ int s_j, s_err;

  for (int r = warp; r < K1; r += WARPS) {
    const int4* pr = prm.part + static_cast<size_t>(b * K1 + r) * prm.slices;
    ArgBest a{ninf, INT_MAX};
    int n = 0;
    for (int s = lane; s < prm.slices; s += 32) {
      const int4 v = pr[s];
      a = arg_better(a, ArgBest{__int_as_float(v.x), v.y});
      n |= v.z;
    }
    a = warp_arg_best(a);
    n = __reduce_or_sync(0xffffffffu, n);
    if (lane == 0) {
      s_arg[r] = a.i;
      // NaN anywhere, a +inf maximum, or no value above -inf: not a usable row.
      s_bad[r] = n || a.i == INT_MAX || !(a.v < __int_as_float(0x7f800000));
    }
  }
  __syncthreads();
  if (warp == 0) {
    int err = 0;
    bool match = false;
    if (lane < K) {
      const int x = prm.drafts[static_cast<size_t>(b) * K + lane];
      if (x < 0 || x >= prm.V) err |= DSPARK_SEQ_BAD_DRAFT;
      match = x == s_arg[lane];
    }
    for (int r = lane; r < K1; r += 32)
      if (s_bad[r]) err |= DSPARK_SEQ_NONFINITE;
    err = __reduce_or_sync(0xffffffffu, err);
    const unsigned mis = __ballot_sync(0xffffffffu, lane < K && !match);
    if (lane == 0) {
      s_j = mis ? __ffs(mis) - 1 : K;
      s_err = err;
    }
  }
  __syncthreads();
  const int j = s_j;
  const int err = s_err;
  const int token = err ? -1 : s_arg[j];
  for (int t = tid; t <= K; t += blockDim.x) {
    int v = -1;
    if (!err) v = t < j ? prm.drafts[static_cast<size_t>(b) * K + t] : (t == j ? token : -1);
    prm.out.tokens[static_cast<size_t>(b) * K1 + t] = v;
  }
  if (tid == 0) {
    prm.out.n_accepted[b] = err ? 0 : j;
    prm.out.next_token[b] = token;
    if (prm.out.status) prm.out.status[b] = err;
  }
}

}  // namespace dspark
