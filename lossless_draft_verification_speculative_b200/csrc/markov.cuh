// The drafter's Markov-head table mat-vec: y[b, v] = sum_k W[v, k] h[b, k] over the table
// markov_w2 (V rows of R = 256 values; the DeepSeek-V4-Flash DSpark drafter card ships it in
// F16 or in GGUF Q8_0 and says the ds4 engine reads it in full four times per draft block).
//
// These are the one-state kernels (several states take the tensor-core kernels). The table is
// read once per call; the work per byte is a few multiply-adds, so the kernel is an HBM
// stream. One CTA of 8 warps per resident slot walks groups of rows grid-stride; a warp keeps
// a group's loads in flight together:
//  - F16: a row is 512 bytes, one 16-byte piece (8 halves) per lane; 8 rows per group. Lane l
//    holds h[8l .. 8l+7] in registers and multiplies its pieces; each row's 32 partial sums are
//    added by its own butterfly (8 independent chains).
//  - Q8_0: a row is 8 blocks of 34 bytes
//    (272 bytes, so rows start 16-byte aligned). A group of 8 consecutive rows (2176 bytes) is
//    copied by 16-byte asynchronous copies into one of the warp's two shared buffers, so the
//    next group is in flight while the warp decodes this one; lane l decodes blocks (row l/8,
//    block l%8) and (row 4 + l/8, block l%8): d * sum_i q[i] h[b, 32 block + i] as exact
//    integer dot products (__dp4a) of the signed bytes with three signed-byte digit planes of
//    the state (below), and the 8 blocks of a row are added by a butterfly over the lanes of
//    the row.
// Sums run in a fixed order (independent of the launch geometry). The kernels are
// programmatic dependent launches: each waits for the kernel before it (which may produce h)
// before reading anything, then lets the next one be scheduled, so back-to-back calls (the
// engine reads the table four times per draft block) overlap their launch latency.
#pragma once

#include <cuda_fp16.h>

#include "common.cuh"

namespace dspark {

constexpr int kMarkovRank = 256;     // R: the only rank the drafters ship
constexpr int kMarkovThreads = 256;  // 8 warps per CTA
constexpr int kQ8RowBytes = kMarkovRank / 32 * 34;  // 272
constexpr int kQ8Rows = 8;                          // rows per warp group (Q8_0)

// 8 halves (a 16-byte word) -> 8 floats, in element order.
__device__ __forceinline__ void unpack_f16x8(const uint4& w, float* f) {
  const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const float2 p = __half22float2(*reinterpret_cast<const __half2*>(&u[k]));
    f[2 * k] = p.x;
    f[2 * k + 1] = p.y;
  }
}

__global__ void __launch_bounds__(kMarkovThreads) markov_f16_kernel(const uint16_t* __restrict__ W,
                                                                    int V, const float* h,
                                                                    float* y) {
  constexpr int ROWS = 8;
  grid_dependency_wait();  // h comes from the kernel before (programmatic launch)
  grid_dependents_launch();
  const int lane = threadIdx.x & 31;
  const int gw = blockIdx.x * (kMarkovThreads / 32) + (threadIdx.x >> 5);
  const int nw = gridDim.x * (kMarkovThreads / 32);
  float hr[8];
  {
    const float4 a = __ldg(reinterpret_cast<const float4*>(h + 8 * lane));
    const float4 c = __ldg(reinterpret_cast<const float4*>(h + 8 * lane + 4));
    hr[0] = a.x; hr[1] = a.y; hr[2] = a.z; hr[3] = a.w;
    hr[4] = c.x; hr[5] = c.y; hr[6] = c.z; hr[7] = c.w;
  }
  for (long long v0 = static_cast<long long>(gw) * ROWS; v0 < V;
       v0 += static_cast<long long>(nw) * ROWS) {
    uint4 w[ROWS];
#pragma unroll
    for (int r = 0; r < ROWS; ++r)
      w[r] = v0 + r < V ? ld_stream16(W + (v0 + r) * kMarkovRank + 8 * lane)
                        : make_uint4(0, 0, 0, 0);
    // a butterfly per row, the rows' chains independent of one another
#pragma unroll
    for (int r = 0; r < ROWS; ++r) {
      float f[8];
      unpack_f16x8(w[r], f);
      float acc = __fmul_rn(f[0], hr[0]);
#pragma unroll
      for (int e = 1; e < 8; ++e) acc = __fmaf_rn(f[e], hr[e], acc);
      acc = warp_sum(acc);
      if (lane == 0 && v0 + r < V) y[v0 + r] = acc;
    }
  }
}

// 16 bytes global -> shared without registers (bypassing L1); n = 0 zero-fills.
__device__ __forceinline__ void cp_async16(void* dst, const void* src, int n) {
  const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(dst));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(d), "l"(src), "r"(n)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// The state as signed-byte digits, for the Q8_0 products on the integer dot-product unit
// (__dp4a): per table block j (32 values), a power-of-two scale s = 2^x (the
// smallest with max_i |h_i| / s <= 127 over the block; 2^0 for an all-zero block) and three
// digit planes with
//   h_i = s (a_i + (b_i + (c_i + e_i) / 254) / 254),   |a_i|, |b_i|, |c_i| <= 127, |e_i| <= 1/2,
// each digit the nearest integer to the scaled remainder. Then sum_i q_i h_i =
// s (A + (B + C / 254) / 254) + err with A = sum_i q_i a_i etc. exact 32-bit dot products of
// signed bytes (|A| <= 32 * 128 * 127 < 2^22) and |err| <= s / (2 * 254^2) sum_i |q_i|
// < 2^-22 max_i |h_i| sum_i |q_i| (s < 2 max_i |h_i| / 127); the rest is float32 rounding of
// the combination. Layout: [plane][block][12 words], 8 words of digits and 4 of
// padding, so that the 8 lanes of a row, one per block, read their 16-byte words from 8
// disjoint groups of 4 banks.
constexpr int kQ8Planes = 3;
constexpr int kQ8Blocks = kMarkovRank / 32;  // 8
constexpr int kQ8DigWords = 12;              // per (plane, block), 8 used
constexpr int kQ8StateWords = kQ8Planes * kQ8Blocks * kQ8DigWords;

// x * 2^k exactly (when the result is a normal float), for -252 <= k <= 254.
__device__ __forceinline__ float mul_pow2(float x, int k) {
  const int k1 = k > 127 ? 127 : (k < -126 ? -126 : k);
  return __fmul_rn(__fmul_rn(x, __int_as_float((k1 + 127) << 23)),
                   __int_as_float((k - k1 + 127) << 23));
}

// One warp: the digits of the state's block j (lane i holds element i) into dig (the state's
// words) and the block's exponent x into ex[j].
__device__ __forceinline__ void q8_state_digits(float hv, int j, int lane, int8_t* dig, int* ex) {
  const float ah = fabsf(hv);
  const uint32_t mb = __reduce_max_sync(0xffffffffu, __float_as_uint(ah));  // |h| bits are ordered
  const float m = __uint_as_float(mb);
  int x = 0;
  if (m > 0.f && m <= 3.402823466e38f) {
    // floor(log2 m) from the bits (subnormals included); s = 2^(that - 6), or twice that when
    // m / s would exceed 127
    const int be = static_cast<int>(mb >> 23);
    const int lg = be != 0 ? be - 127 : -149 + (31 - __clz(static_cast<int>(mb & 0x7fffffu)));
    x = lg - 6;
    if (mul_pow2(m, -x) > 127.f) x += 1;
  }
  const float v = mul_pow2(hv, -x);  // exact: |v| <= 127
  const float a = rintf(v);
  const float r1 = __fmul_rn(__fsub_rn(v, a), 254.f);  // exact: |v - a| <= 1/2
  const float b = rintf(r1);
  const float c = rintf(__fmul_rn(__fsub_rn(r1, b), 254.f));
  // (a non-finite state value leaves its digits undefined; its exponent marks the block)
  dig[((0 * kQ8Blocks + j) * kQ8DigWords) * 4 + lane] = static_cast<int8_t>(a);
  dig[((1 * kQ8Blocks + j) * kQ8DigWords) * 4 + lane] = static_cast<int8_t>(b);
  dig[((2 * kQ8Blocks + j) * kQ8DigWords) * 4 + lane] = static_cast<int8_t>(c);
  if (lane == 0) ex[j] = m <= 3.402823466e38f ? x : 1024;  // 1024: non-finite
}

// |x| < 2^22 as a float, exactly, without the int-to-float converter.
__device__ __forceinline__ float small_int_to_float(int x) {
  return __fsub_rn(__int_as_float(x + 0x4B400000), 12582912.f);
}

// A warp's groups are double-buffered: the copy of its next group is in flight while it
// decodes the current one. Lane l takes blocks (row l/8, block l%8) and (row 4 + l/8, block
// l%8): three integer dot-product chains over the block's 32 signed bytes
// (read as aligned 32-bit words, funnel-shifted when the block starts 2 bytes into a word)
// against the state's digit planes, then s (A + (B + C / 254) / 254) times the block scale d;
// the 8 blocks of a row are added by a butterfly over the lanes of the row.
__global__ void __launch_bounds__(kMarkovThreads, 4) markov_q8_0_kernel(
    const uint8_t* __restrict__ W, int V, const float* h, float* y) {
  constexpr int kGroupBytes = kQ8Rows * kQ8RowBytes;  // 2176
  constexpr int kPieces = kGroupBytes / 16;           // 136 16-byte pieces per group
  __shared__ __align__(16) uint8_t s_rows[kMarkovThreads / 32][2][kGroupBytes];
  __shared__ __align__(16) int8_t s_dig[kQ8StateWords * 4];
  __shared__ int s_ex[kQ8Blocks];
  const int lane = threadIdx.x & 31, wi = threadIdx.x >> 5;
  const int blk = lane & 7;
  const int gw = blockIdx.x * (kMarkovThreads / 32) + wi;
  const int nw = gridDim.x * (kMarkovThreads / 32);
  const long long stride = static_cast<long long>(nw) * kQ8Rows;
  // copy of the group at row v0 into buffer st (rows past V zero-filled), as one commit group
  auto fetch = [&](long long v0, int st) {
    const long long nbytes = (V - v0 < kQ8Rows ? V - v0 : kQ8Rows) * kQ8RowBytes;
    const uint8_t* src = W + v0 * kQ8RowBytes;
#pragma unroll
    for (int k = 0; k < (kPieces + 31) / 32; ++k) {
      const int c = lane + 32 * k;
      if (c < kPieces) {
        const bool in = 16LL * c < nbytes;
        cp_async16(&s_rows[wi][st][16 * c], in ? src + 16 * c : W, in ? 16 : 0);
      }
    }
    cp_async_commit();
  };
  grid_dependency_wait();  // h comes from the kernel before (programmatic launch)
  grid_dependents_launch();
  long long v0 = static_cast<long long>(gw) * kQ8Rows;
  if (v0 < V) fetch(v0, 0);
  static_assert(kMarkovThreads / 32 == kQ8Blocks, "one warp per table block");
  // the state's digits: warp w takes block w
  q8_state_digits(__ldg(h + wi * 32 + lane), wi, lane, s_dig, s_ex);
  __syncthreads();
  const int xb = s_ex[blk];  // this lane's block exponent
  for (int st = 0; v0 < V; v0 += stride, st ^= 1) {
    if (v0 + stride < V) {
      fetch(v0 + stride, st ^ 1);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncwarp();  // every lane's copies of this group have landed
    const uint8_t* buf = s_rows[wi][st];
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const int row = half * 4 + (lane >> 3);
      const int qoff = row * kQ8RowBytes + blk * 34 + 2;  // first signed byte of the block
      const float d = __half2float(*reinterpret_cast<const __half*>(buf + qoff - 2));
      const uint32_t* wp = reinterpret_cast<const uint32_t*>(buf + (qoff & ~3));
      const uint32_t sh = (qoff & 3) * 8;  // 0 or 16
      int q[8];
      uint32_t lo = wp[0];
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        // a block 2 bytes into a word ends 2 bytes into a 9th
        const uint32_t hi = (k < 7 || sh) ? wp[k + 1] : 0u;
        q[k] = static_cast<int>(__funnelshift_r(lo, hi, sh));
        lo = hi;
      }
      int acc[kQ8Planes];
#pragma unroll
      for (int pl = 0; pl < kQ8Planes; ++pl) {
        const int4* dg = reinterpret_cast<const int4*>(s_dig) +
                         (pl * kQ8Blocks + blk) * (kQ8DigWords / 4);
        const int4 g0 = dg[0], g1 = dg[1];
        int a = __dp4a(q[0], g0.x, 0);
        a = __dp4a(q[1], g0.y, a);
        a = __dp4a(q[2], g0.z, a);
        a = __dp4a(q[3], g0.w, a);
        a = __dp4a(q[4], g1.x, a);
        a = __dp4a(q[5], g1.y, a);
        a = __dp4a(q[6], g1.z, a);
        acc[pl] = __dp4a(q[7], g1.w, a);
      }
      float f = __fmaf_rn(small_int_to_float(acc[2]), 1.f / 254.f, small_int_to_float(acc[1]));
      f = __fmaf_rn(f, 1.f / 254.f, small_int_to_float(acc[0]));
      // d s f; a non-finite state block gives NaN
      float s = xb == 1024 ? __int_as_float(0x7fc00000) : mul_pow2(__fmul_rn(d, f), xb);
#pragma unroll
      for (int o = 1; o < 8; o <<= 1) s = __fadd_rn(s, __shfl_xor_sync(0xffffffffu, s, o));
      if (blk == 0 && v0 + row < V) y[v0 + row] = s;
    }
    __syncwarp();  // the buffer is refilled two groups on
  }
}

}  // namespace dspark
