// The drafter's Markov-head table mat-vec: y[b, v] = sum_k W[v, k] h[b, k] over the table
// markov_w2 (V rows of R = 256 values; the DeepSeek-V4-Flash DSpark drafter card ships it in
// F16 or in GGUF Q8_0 and says the ds4 engine reads it in full four times per draft block).
//
// The table is read once per call; the work per byte is a few multiply-adds, so the kernel is
// an HBM stream. One CTA of 8 warps per resident slot walks groups of rows grid-stride; a warp
// keeps a group's loads in flight together:
//  - F16: a row is 512 bytes, one 16-byte piece (8 halves) per lane; 8 rows per group (4 with
//    3 or 4 states). Lane l holds h[b, 8l .. 8l+7] in registers, multiplies its pieces, and
//    each row's 32 partial sums are added by a butterfly.
//  - Q8_0: a row is 8 blocks of 34 bytes (272 bytes, so rows start 16-byte aligned). A group
//    of 8 consecutive rows (2176 bytes) is copied with 16-byte loads into the warp's shared
//    buffer; lane l then decodes blocks (row l/8, block l%8) and (row 4 + l/8, block l%8):
//    d * sum_i q[i] h[b, 32 block + i], and the 8 blocks of a row are added by a butterfly
//    over the lanes of the row.
// Sums run in float32 in a fixed order (independent of the launch geometry).
#pragma once

#include <cuda_fp16.h>

#include "common.cuh"

namespace dspark {

constexpr int kMarkovRank = 256;     // R: the only rank the drafters ship
constexpr int kMarkovThreads = 256;  // 8 warps per CTA
constexpr int kMarkovMaxStates = 4;  // states per launch (the host splits larger batches)
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

template <int NB>
__global__ void __launch_bounds__(kMarkovThreads) markov_f16_kernel(const uint16_t* __restrict__ W,
                                                                    int V, const float* h,
                                                                    float* y, int ldy) {
  constexpr int ROWS = NB <= 2 ? 8 : 4;
  const int lane = threadIdx.x & 31;
  const int gw = blockIdx.x * (kMarkovThreads / 32) + (threadIdx.x >> 5);
  const int nw = gridDim.x * (kMarkovThreads / 32);
  float hr[NB][8];
#pragma unroll
  for (int b = 0; b < NB; ++b) {
    const float4 a = __ldg(reinterpret_cast<const float4*>(h + b * kMarkovRank + 8 * lane));
    const float4 c = __ldg(reinterpret_cast<const float4*>(h + b * kMarkovRank + 8 * lane + 4));
    hr[b][0] = a.x; hr[b][1] = a.y; hr[b][2] = a.z; hr[b][3] = a.w;
    hr[b][4] = c.x; hr[b][5] = c.y; hr[b][6] = c.z; hr[b][7] = c.w;
  }
  for (long long v0 = static_cast<long long>(gw) * ROWS; v0 < V;
       v0 += static_cast<long long>(nw) * ROWS) {
    uint4 w[ROWS];
#pragma unroll
    for (int r = 0; r < ROWS; ++r)
      w[r] = v0 + r < V ? ld_stream16(W + (v0 + r) * kMarkovRank + 8 * lane)
                        : make_uint4(0, 0, 0, 0);
#pragma unroll
    for (int r = 0; r < ROWS; ++r) {
      float f[8];
      unpack_f16x8(w[r], f);
#pragma unroll
      for (int b = 0; b < NB; ++b) {
        float acc = __fmul_rn(f[0], hr[b][0]);
#pragma unroll
        for (int e = 1; e < 8; ++e) acc = __fmaf_rn(f[e], hr[b][e], acc);
        acc = warp_sum(acc);
        if (lane == 0 && v0 + r < V) y[static_cast<long long>(b) * ldy + v0 + r] = acc;
      }
    }
  }
}

template <int NB>
__global__ void __launch_bounds__(kMarkovThreads) markov_q8_0_kernel(const uint8_t* __restrict__ W,
                                                                     int V, const float* h,
                                                                     float* y, int ldy) {
  __shared__ __align__(16) uint8_t s_rows[kMarkovThreads / 32][kQ8Rows * kQ8RowBytes];
  // the states, block by block with a stride of 33 floats, so that the 8 lanes of a row (one
  // per block) read 8 different banks
  __shared__ float s_h[NB][8 * 33];
  for (int i = threadIdx.x; i < NB * kMarkovRank; i += kMarkovThreads) {
    const int b = i / kMarkovRank, k = i % kMarkovRank;
    s_h[b][(k >> 5) * 33 + (k & 31)] = h[i];
  }
  __syncthreads();
  const int lane = threadIdx.x & 31, wi = threadIdx.x >> 5;
  const int gw = blockIdx.x * (kMarkovThreads / 32) + wi;
  const int nw = gridDim.x * (kMarkovThreads / 32);
  uint8_t* buf = s_rows[wi];
  constexpr int kPieces = kQ8Rows * kQ8RowBytes / 16;   // 136 16-byte pieces per group
  const int blk = lane & 7;
  for (long long v0 = static_cast<long long>(gw) * kQ8Rows; v0 < V;
       v0 += static_cast<long long>(nw) * kQ8Rows) {
    const long long nbytes = (V - v0 < kQ8Rows ? V - v0 : kQ8Rows) * kQ8RowBytes;
    const uint8_t* src = W + v0 * kQ8RowBytes;
    uint4 piece[(kPieces + 31) / 32];
#pragma unroll
    for (int k = 0; k < (kPieces + 31) / 32; ++k) {
      const int c = lane + 32 * k;
      piece[k] = c < kPieces && 16LL * c < nbytes ? ld_stream16(src + 16 * c)
                                                 : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int k = 0; k < (kPieces + 31) / 32; ++k) {
      const int c = lane + 32 * k;
      if (c < kPieces) *reinterpret_cast<uint4*>(buf + 16 * c) = piece[k];
    }
    __syncwarp();
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const int row = half * 4 + (lane >> 3);
      const uint8_t* blockp = buf + row * kQ8RowBytes + blk * 34;
      const float d = __half2float(*reinterpret_cast<const __half*>(blockp));
      float acc[NB];
#pragma unroll
      for (int b = 0; b < NB; ++b) acc[b] = 0.f;
#pragma unroll
      for (int i = 0; i < 32; i += 2) {
        const uint16_t two = *reinterpret_cast<const uint16_t*>(blockp + 2 + i);
        const float q0 = static_cast<float>(static_cast<int8_t>(two & 0xff));
        const float q1 = static_cast<float>(static_cast<int8_t>(two >> 8));
#pragma unroll
        for (int b = 0; b < NB; ++b) {
          acc[b] = __fmaf_rn(q0, s_h[b][33 * blk + i], acc[b]);
          acc[b] = __fmaf_rn(q1, s_h[b][33 * blk + i + 1], acc[b]);
        }
      }
#pragma unroll
      for (int b = 0; b < NB; ++b) {
        float s = __fmul_rn(d, acc[b]);
#pragma unroll
        for (int o = 1; o < 8; o <<= 1) s = __fadd_rn(s, __shfl_xor_sync(0xffffffffu, s, o));
        if (blk == 0 && v0 + row < V) y[static_cast<long long>(b) * ldy + v0 + row] = s;
      }
    }
    __syncwarp();  // the buffer is refilled by the next group
  }
}

}  // namespace dspark
