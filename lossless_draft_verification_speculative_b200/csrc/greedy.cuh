// greedy_accept on sm_100a.
//
// Pass 1 streams the K+1 base rows of every sequence once (P only; Q is never read). Per
// 8192-token slice of a row it takes the maximum with a NaN-propagating max (two bf16 tokens
// per packed instruction, so a NaN anywhere shows up as a NaN maximum at no extra cost), then
// the lowest index holding it: only the threads whose own maximum equals the slice maximum
// (usually one) walk their tokens. Float equality makes -0.0 and +0.0 equal, as the
// definition asks.
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

// Max of this thread's logits. bf16 vectors use the packed NaN-propagating max (two tokens
// per instruction); a NaN anywhere makes the result NaN, so NaN rows are caught for free.
template <typename T, int VEC>
__device__ __forceinline__ float thread_max(const uint4* raw, const float* z);

template <>
__device__ __forceinline__ float thread_max<bf16_t, 8>(const uint4* raw, const float*) {
  uint32_t m = 0xff80ff80u;  // (-inf, -inf)
#pragma unroll
  for (int g = 0; g < kGreedyThreadElems / 8; ++g) {
    m = max_nan_bf16x2(m, raw[g].x);
    m = max_nan_bf16x2(m, raw[g].y);
    m = max_nan_bf16x2(m, raw[g].z);
    m = max_nan_bf16x2(m, raw[g].w);
  }
  return max_nan(__uint_as_float(m << 16), __uint_as_float(m & 0xffff0000u));
}

template <typename T, int VEC>
__device__ __forceinline__ float thread_max(const uint4*, const float* z) {
  float m = -__int_as_float(0x7f800000);
#pragma unroll
  for (int k = 0; k < kGreedyThreadElems; k += 2) m = max3_nan(m, z[k], z[k + 1]);
  return m;
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
  // token of this thread's k-th value (ascending in k)
  auto token = [&](int k) {
    return VEC == 1 ? sbase + k * kGreedyThreads + tid
                    : sbase + ((k / VEC) * kGreedyThreads + tid) * VEC + (k % VEC);
  };

  uint4 raw[VEC == 1 ? 1 : G];
  float z[kGreedyThreadElems];
  if constexpr (VEC == 1) {
#pragma unroll
    for (int k = 0; k < G; ++k) {
      const int e = token(k);
      z[k] = e < V ? Elem<T>::load1(base + e) : ninf;
    }
  } else {
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const int e = sbase + (g * kGreedyThreads + tid) * VEC;
      raw[g] = e < V ? ld_stream16(base + e)
                     : (Elem<T>::kBytes == 2 ? make_uint4(0xff80ff80u, 0xff80ff80u, 0xff80ff80u,
                                                          0xff80ff80u)
                                             : make_uint4(0xff800000u, 0xff800000u, 0xff800000u,
                                                          0xff800000u));
    }
    if constexpr (Elem<T>::kBytes == 4) {
#pragma unroll
      for (int g = 0; g < G; ++g) Elem<T>::unpack(raw[g], z + g * VEC);
    }
  }

  const float tm = thread_max<T, VEC>(raw, z);
  const float wm = warp_max_nan(tm);
  __shared__ float s_wmax[kGreedyThreads / 32];
  __shared__ float s_max;
  __shared__ int s_idx;
  if (lane == 0) s_wmax[warp] = wm;
  if (tid == 0) s_idx = INT_MAX;
  __syncthreads();
  if (warp == 0) {
    const float v = lane < kGreedyThreads / 32 ? s_wmax[lane] : ninf;
    const float m = warp_max_nan(v);
    if (lane == 0) s_max = m;
  }
  __syncthreads();
  const float M = s_max;
  // Only threads holding the slice maximum look for its first position (usually one thread).
  if (tm == M && M > ninf) {
    float zz[kGreedyThreadElems];
    if constexpr (VEC == 1 || Elem<T>::kBytes == 4) {
#pragma unroll
      for (int k = 0; k < kGreedyThreadElems; ++k) zz[k] = z[k];
    } else {
#pragma unroll
      for (int g = 0; g < G; ++g) Elem<T>::unpack(raw[g], zz + g * VEC);
    }
    int first = INT_MAX;
#pragma unroll
    for (int k = kGreedyThreadElems - 1; k >= 0; --k)
      if (zz[k] == M) first = token(k);
    atomicMin(&s_idx, first);
  }
  __syncthreads();
  if (tid == 0) {
    const bool nan = M != M;
    prm.part[static_cast<size_t>(row) * prm.slices + sl] =
        make_int4(__float_as_int(nan ? ninf : M), nan || !(M > ninf) ? INT_MAX : s_idx, nan, 0);
  }
  grid_dependents_launch();
}

template <int WARPS>
__global__ void __launch_bounds__(WARPS * 32) greedy_finish_kernel(const GreedyParams prm) {
  const float ninf = -__int_as_float(0x7f800000);
  const int b = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int K = prm.K, K1 = K + 1;
  // The drafts are an input, not a result of pass 1: read them before waiting for it.
  const int x = (warp == 0 && lane < K) ? prm.drafts[static_cast<size_t>(b) * K + lane] : 0;
  grid_dependency_wait();
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
      s_bad[r] = n || a.i == INT_MAX || !(a.v < __int_as_float(0x7f800000)) || !(a.v > ninf);
    }
  }
  __syncthreads();
  if (warp == 0) {
    int err = 0;
    bool match = false;
    if (lane < K) {
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
