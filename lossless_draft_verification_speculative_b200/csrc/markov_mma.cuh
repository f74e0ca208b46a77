// The Markov-head mat-vec y[b, v] = sum_k W[v, k] h[b, k] on the fifth-generation tensor cores
// (tcgen05), with one read of the table per launch (the DeepSeek-V4-Flash DSpark drafter card,
// "Files": markov_w2 in F16 or Q8_0, 8 blocks of 34 bytes per row of R = 256 in Q8_0; the engine
// reads it four times per draft block). Three kernels:
//  - markov_q8_0_mma_kernel (below): Q8_0, up to 64 states, the bytes converted to float16;
//  - markov_f16_mma_kernel: F16, up to 64 states, the table loaded by TMA as stored;
//  - markov_q8_0_i8_kernel: Q8_0, up to 10 states, integer MMAs on the bytes as stored.
// The host (dspark_markov_matvec) picks one by format and number of states.
//
// markov_q8_0_mma_kernel. Exact operands. A Q8_0 value is d q with q a signed byte, exact in float16; the block scale
// d is per (row, block of 32), so each block gets its own float32 accumulators and d is
// applied afterwards. Each state h_b is scaled by a power of two 2^e_b (m_b 2^e_b in
// [2^14, 2^15), m_b = max_k |h[b, k]|) and split into float16 parts hi + lo, which represent it
// to within 2^-23 m_b (|h 2^e - hi| <= 8, so lo rounds at 2^-9 or finer); every product
// q * part is exact in float32. The parts are the two halves of the MMA's N: B row b is hi_b,
// row N + b is lo_b. Per tile of 128 rows and block j:
//   D_j[r, b] + D_j[r, N + b] = sum_{k in block j} q[r, k] (hi[b, k] + lo[b, k])  (tensor cores)
//   y[b, r] = 2^-e_b sum_j d[r, j] (D_j[r, b] + D_j[r, N + b])             (CUDA cores, f32)
//
// One CTA per SM (persistent over tiles t = blockIdx.x + i gridDim.x), 14 warps. A work item
// is a quarter tile (2 blocks, K = 64: one 128-byte swizzle atom); item i of the CTA is quarter
// i % 4 of its tile i / 4.
//  - warp 0, one lane: copies each tile's 128 rows x 272 bytes (contiguous in the table) into
//    a shared staging ring with one bulk asynchronous copy (cp.async.bulk, mbarrier
//    completion); warp 0 also allocates and frees the tensor memory.
//  - warp 1, one lane: per item, per block, 2 MMAs (K = 16 each) of M = 128, N = 2 x 16..64
//    into the block's accumulators, then two commits: the item's A slab is free, its
//    accumulators are ready.
//  - warps 2-5 and 6-9, two teams of 128 threads (thread = tile row), team T converting
//    quarters T and T + 2 of every tile into A slabs T and T + 2 (each team double-buffered):
//    the q bytes to float16 in the 128-byte-swizzled K-major layout, the scales d to float32
//    in a ring of 8 items.
//  - warps 10-13, 128 threads (thread = tile row = TMEM lane; lane quarter = warp % 4): per
//    item, read the accumulators from tensor memory (tcgen05.ld), add hi + lo, multiply by d
//    and accumulate; after the fourth quarter write y.
// Rings: 2-3 staging buffers (a tile each), 4 A slabs (16 KB), 8 scale sets, 2-8 accumulator
// slots in tensor memory (4 N columns each). Every mbarrier wait is bounded (about a second);
// a wait that runs out sets an abort flag that ends every role's loop, counts the event in a
// device counter (dspark_pipeline_timeouts), lets the copies and MMAs in flight finish (again
// bounded) and frees the tensor memory before the CTA exits. `withhold` (tests of that path
// only) makes each CTA's producer skip its first copy, so the waits for it run out.
#pragma once

#include <cuda.h>  // CUtensorMap (the type only; no driver calls here)
#include <cuda_fp16.h>

#include "common.cuh"
#include "markov.cuh"

namespace dspark {

constexpr int kMmaRows = 128;          // tile rows (MMA M)
constexpr int kMmaMaxStates = 64;      // states per launch (MMA N = 2 x 64 at most)
constexpr int kMmaThreads = 448;       // 14 warps
constexpr int kMmaTeam = 128;          // threads of a converter team or of the epilogue
constexpr int kQ8RowBytesT = 272;      // 8 blocks x 34 bytes
constexpr int kMmaRawBytes = kMmaRows * kQ8RowBytesT;  // 34816, a staging buffer
constexpr int kMmaSlabBytes = kMmaRows * 128;          // 16384: 128 rows x 64 halves
constexpr int kMmaTmemCols = 512;

__device__ unsigned long long g_pipeline_timeouts = 0;

// ---------------------------------------------------------------- mbarrier / async helpers

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint32_t bar, int count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_arrive_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wait for the phase of the given parity to complete, for at most about a second (2^31 SM
// clocks); false (and the CTA's abort flag set) when it runs out or another role aborted.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort) {
  if (mbar_try(bar, parity)) return true;
  const long long t0 = clock64();
  while (true) {
    if (mbar_try(bar, parity)) return true;
    if (*abort) return false;
    if (clock64() - t0 > (1ll << 31)) {
      *abort = 1;
      atomicAdd(&g_pipeline_timeouts, 1ull);
      return false;
    }
  }
}

__device__ __forceinline__ void bulk_copy_g2s(uint32_t dst, const void* src, uint32_t bytes,
                                              uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---------------------------------------------------------------- tcgen05 helpers

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// The CTA's tensor memory: all 512 columns (one CTA per SM), allocated by one warp, which
// writes the base address to *slot; freed by one warp once every MMA and load is done.
__device__ __forceinline__ void tmem_alloc_all(uint32_t* slot) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(slot)),
               "r"(kMmaTmemCols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  tc_fence_before();
}
__device__ __forceinline__ void tmem_free_all(uint32_t base) {
  tc_fence_after();
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(base),
               "r"(kMmaTmemCols)
               : "memory");
}

// After an abort: wait (about a second at most) for the phase of the given parity of `bar` to
// complete, i.e. for the asynchronous copy or the MMAs it tracks to land.
__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t parity) {
  const long long t0 = clock64();
  while (!mbar_try(bar, parity) && clock64() - t0 < (1ll << 31)) {
  }
}

// Shared-memory matrix descriptor of a K-major operand in the 128-byte swizzle layout: rows of
// 128 bytes, 8-row groups 1024 bytes apart (the group stride), the 16-byte chunk c of row r
// stored at chunk c ^ (r % 8); the group base is 1024-byte aligned. A K step of 16 halves
// (32 bytes) inside the 128-byte row advances the start address by 32.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
  return static_cast<uint64_t>((saddr >> 4) & 0x3FFFu) | (1ull << 16) |  // leading offset (unused)
         (64ull << 32) |                                                // group stride 1024 B
         (1ull << 46) |                                                 // descriptor version
         (2ull << 61);                                                  // 128-byte swizzle
}

// Instruction descriptor: kind::f16, A and B float16, K-major, D float32, M = 128, N.
__host__ __device__ constexpr uint32_t mma_idesc_f16(int n) {
  return (1u << 4) | (static_cast<uint32_t>(n >> 3) << 17) | (static_cast<uint32_t>(128 >> 4) << 24);
}

__device__ __forceinline__ void mma_f16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                        uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void mma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::
                   "r"(bar)
               : "memory");
}

// 16 consecutive float32 columns of this warp's 32 TMEM lanes (one row per lane).
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float* v) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}
// 8 consecutive float32 columns of this warp's 32 TMEM lanes.
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, float* v) {
  uint32_t r[8];
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                 "=r"(r[6]), "=r"(r[7])
               : "r"(taddr)
               : "memory");
#pragma unroll
  for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_ld_wait() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// ---------------------------------------------------------------- the kernel

struct MmaQ8Smem {
  // offsets (bytes) from the 1024-aligned dynamic shared-memory base
  int b_off, slab_off, d_off, raw_off, bar_off, total;
};

constexpr int kMmaSlabs = 4;   // one per quarter
constexpr int kMmaDRing = 8;   // scale sets (items) in flight

__host__ __device__ constexpr int mma_raw_stages(int n) { return n <= 48 ? 3 : 2; }
// accumulator slots in the 512 TMEM columns: 4 N columns each (2 blocks x hi, lo), at most 8
__host__ __device__ constexpr int mma_tmem_slots(int n) { return 512 / (4 * n) < 8 ? 512 / (4 * n) : 8; }

__host__ __device__ inline MmaQ8Smem mma_q8_smem(int n) {
  MmaQ8Smem s{};
  s.b_off = 0;                                     // 4 atoms x 2n rows x 128 B
  s.slab_off = s.b_off + 4 * 2 * n * 128;          // 4 x 16 KB
  s.d_off = s.slab_off + kMmaSlabs * kMmaSlabBytes;  // 8 x 2 blocks x 128 rows float
  s.raw_off = s.d_off + kMmaDRing * 2 * kMmaRows * 4;
  s.bar_off = s.raw_off + mma_raw_stages(n) * kMmaRawBytes;
  s.total = s.bar_off + 1024 + 1024;  // barriers, flags, scales; slack to align the base
  return s;
}

// Converts this thread's row of quarter QQ (blocks 2 QQ and 2 QQ + 1: raw bytes [68 QQ,
// 68 QQ + 68)) from the staging buffer into the A slab (one swizzle atom). The 80 bytes from
// the 16-byte boundary below 68 QQ are read as 5 aligned 16-byte words; pairs of q bytes (even
// offsets, never split across a word) become float16x2 through a byte permute into 0x64 bytes
// (1024 + (q + 128)) and an exact subtraction of 1152. The scales go to d[bl * 128 + r].
template <int QQ>
__device__ __forceinline__ void q8_convert_quarter(const uint8_t* raw_row, uint8_t* slab,
                                                   float* d, int r) {
  constexpr int kStart = (68 * QQ) & ~15;
  uint32_t w[20];
#pragma unroll
  for (int c = 0; c < 5; ++c) {
    const uint4 v = *reinterpret_cast<const uint4*>(raw_row + kStart + 16 * c);
    w[4 * c] = v.x; w[4 * c + 1] = v.y; w[4 * c + 2] = v.z; w[4 * c + 3] = v.w;
  }
  const __half2 bias = __halves2half2(__ushort_as_half(0x6480), __ushort_as_half(0x6480));
#pragma unroll
  for (int bl = 0; bl < 2; ++bl) {
    const int s = 68 * QQ - kStart + 34 * bl;  // the block's first byte (the scale), even
    d[bl * kMmaRows + r] = __half2float(__ushort_as_half(
        static_cast<unsigned short>((w[s >> 2] >> (8 * (s & 3))) & 0xffffu)));
    uint32_t h2[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const int o = s + 2 + 2 * j;  // even: the pair sits in one word
      const uint32_t x = w[o >> 2] ^ 0x80808080u;
      const uint32_t sel = (o & 3) == 0 ? 0x4140u : 0x4342u;
      const uint32_t p = __byte_perm(x, 0x64646464u, sel);
      const __half2 v = __hsub2(*reinterpret_cast<const __half2*>(&p), bias);
      h2[j] = *reinterpret_cast<const uint32_t*>(&v);
    }
    // block bl = K [32 bl, 32 bl + 32) of the atom: 16-byte chunks 4 bl .. 4 bl + 3
    uint8_t* row = slab + r * 128;
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      const int c = 4 * bl + m;
      *reinterpret_cast<uint4*>(row + ((c ^ (r & 7)) << 4)) =
          make_uint4(h2[4 * m], h2[4 * m + 1], h2[4 * m + 2], h2[4 * m + 3]);
    }
  }
}

// 2^e as a float for -126 <= e <= 127 (exact).
__device__ __forceinline__ float pow2f(int e) { return __int_as_float((e + 127) << 23); }

// floor(log2 m) for a finite m > 0 (subnormals included).
__device__ __forceinline__ int ilog2f(float m) {
  const uint32_t u = __float_as_uint(m);
  const int be = static_cast<int>(u >> 23);
  return be != 0 ? be - 127 : -149 + (31 - __clz(static_cast<int>(u & 0x7fffffu)));
}

// The B operand of the Markov MMAs, built by warps w0 .. w0 + NW - 1 of the CTA: state b
// (rows nb..N-1 zero) scaled by 2^e_b (m_b 2^e_b in [2^14, 2^15)) and split into float16 hi
// (B row b) and lo (B row N + b), 128-byte-swizzled K-major: atom k / 64, row n, 16-byte chunk
// (k % 64) / 8 stored at chunk ((k % 64) / 8) ^ (n % 8), element k % 8. s_scale[b] and
// s_scale[64 + b] receive 2^-e_b as two exact factors. Ends with the proxy fence that makes the
// writes visible to the tensor cores (the caller synchronises the builders afterwards).
template <int N, int NW>
__device__ __forceinline__ void build_b_operand(const float* h, int nb, uint8_t* s_b,
                                                float* s_scale, int w, int lane) {
  constexpr int kPer = (N + NW - 1) / NW;
  float hv[kPer][8];
#pragma unroll
  for (int u = 0; u < kPer; ++u) {
    const int b = w + NW * u;
#pragma unroll
    for (int j = 0; j < 8; ++j) hv[u][j] = b < nb ? __ldg(h + b * kMarkovRank + lane + 32 * j) : 0.f;
  }
#pragma unroll
  for (int u = 0; u < kPer; ++u) {
    const int b = w + NW * u;
    if (b >= N) break;
    float m = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j) m = max_nan(m, fabsf(hv[u][j]));  // NaN anywhere: m NaN
    m = warp_max_nan(m);
    int e = 0;
    if (m > 0.f && m <= 3.402823466e38f) e = 14 - ilog2f(m);  // m 2^e in [2^14, 2^15)
    // 2^e in two exact factors (e in [-114, 163]); 2^-e likewise
    const int e1 = e > 127 ? 127 : e, e2 = e - e1;
    const float f1 = pow2f(e1), f2 = pow2f(e2);
    if (lane == 0) {
      const int g1 = -e < -126 ? -126 : -e;
      s_scale[b] = pow2f(g1);
      s_scale[64 + b] = pow2f(-e - g1);
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int k = lane + 32 * j;
      const float x = __fmul_rn(__fmul_rn(hv[u][j], f1), f2);
      const __half hi = __float2half_rn(x);
      // (a non-finite x keeps lo = 0: its products are those of x itself)
      const __half lo =
          is_finite(x) ? __float2half_rn(__fsub_rn(x, __half2float(hi))) : __float2half_rn(0.f);
      const int off_hi = (k >> 6) * (2 * N * 128) + b * 128 +
                         ((((k & 63) >> 3) ^ (b & 7)) << 4) + (k & 7) * 2;
      const int off_lo = (k >> 6) * (2 * N * 128) + (N + b) * 128 +
                         ((((k & 63) >> 3) ^ ((N + b) & 7)) << 4) + (k & 7) * 2;
      *reinterpret_cast<__half*>(s_b + off_hi) = hi;
      *reinterpret_cast<__half*>(s_b + off_lo) = lo;
    }
  }
  fence_proxy_async_smem();
}

template <int N>
__global__ void __launch_bounds__(kMmaThreads, 1)
    markov_q8_0_mma_kernel(const uint8_t* __restrict__ W, int V, const float* h, int nb,
                           float* y, int ldy, int withhold) {
  constexpr int kRaw = mma_raw_stages(N);
  constexpr int kSlots = mma_tmem_slots(N);
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
  const MmaQ8Smem L = mma_q8_smem(N);
  uint8_t* s_b = sm + L.b_off;
  uint8_t* s_slab = sm + L.slab_off;
  float* s_d = reinterpret_cast<float*>(sm + L.d_off);
  uint8_t* s_raw = sm + L.raw_off;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L.bar_off);
  uint64_t* raw_full = bars;        // [3] producer (expect_tx) + the copy's bytes
  uint64_t* raw_empty = bars + 3;   // [3] both converter teams (256)
  uint64_t* slab_full = bars + 6;   // [4] a converter team (128)
  uint64_t* slab_free = bars + 10;  // [4] MMA commit
  uint64_t* d_full = bars + 14;     // [8] a converter team (128)
  uint64_t* d_free = bars + 22;     // [8] the epilogue (128)
  uint64_t* acc_full = bars + 30;   // [8] MMA commit
  uint64_t* acc_empty = bars + 38;  // [8] the epilogue (128)
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(bars + 46);
  volatile int* s_abort = reinterpret_cast<volatile int*>(bars + 47);
  float* s_scale = reinterpret_cast<float*>(bars + 48);  // [2][64]: 2^-e_b as two factors

  const int tid = threadIdx.x, wi = tid >> 5, lane = tid & 31;
  const int n_tiles = (V + kMmaRows - 1) / kMmaRows;
  const int my_tiles = blockIdx.x < n_tiles ? (n_tiles - 1 - blockIdx.x) / gridDim.x + 1 : 0;
  const int n_items = 4 * my_tiles;

  if (tid == 0) {
    for (int i = 0; i < 3; ++i) {
      mbar_init(smem_u32(&raw_full[i]), 1);
      mbar_init(smem_u32(&raw_empty[i]), 2 * kMmaTeam);
    }
    for (int i = 0; i < kMmaSlabs; ++i) {
      mbar_init(smem_u32(&slab_full[i]), kMmaTeam);
      mbar_init(smem_u32(&slab_free[i]), 1);
    }
    for (int i = 0; i < 8; ++i) {
      mbar_init(smem_u32(&d_full[i]), kMmaTeam);
      mbar_init(smem_u32(&d_free[i]), kMmaTeam);
      mbar_init(smem_u32(&acc_full[i]), 1);
      mbar_init(smem_u32(&acc_empty[i]), kMmaTeam);
    }
    *s_abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (wi == 0) tmem_alloc_all(s_tmem);
  __syncthreads();  // barriers initialised, tensor memory allocated

  grid_dependency_wait();  // h comes from the kernel before (programmatic launch)
  grid_dependents_launch();

  if (wi == 0) {
    // ---- producer: one bulk copy per tile (the first ones overlap the split below)
    if (lane == 0) {
      int armed = 0;
      for (int j = 0; j < my_tiles; ++j) {
        const int st = j % kRaw;
        if (!mbar_wait(smem_u32(&raw_empty[st]), ((j / kRaw) & 1) ^ 1, s_abort)) break;
        const long long t = blockIdx.x + static_cast<long long>(j) * gridDim.x;
        const int rows = V - t * kMmaRows < kMmaRows ? static_cast<int>(V - t * kMmaRows) : kMmaRows;
        const uint32_t bytes = static_cast<uint32_t>(rows * kQ8RowBytesT);
        if (withhold && j == 0) continue;  // (timeout test: this tile never arrives)
        mbar_arrive_tx(smem_u32(&raw_full[st]), bytes);
        bulk_copy_g2s(smem_u32(s_raw + st * kMmaRawBytes), W + t * kMmaRows * kQ8RowBytesT,
                      bytes, smem_u32(&raw_full[st]));
        armed = j + 1;
      }
      if (*s_abort) {
        // let the copies in flight land before the CTA's shared memory goes away
        for (int j = armed - kRaw < 0 ? 0 : armed - kRaw; j < armed; ++j) {
          if (withhold && j == 0) continue;
          drain_wait(smem_u32(&raw_full[j % kRaw]), (j / kRaw) & 1);
        }
      }
    }
  } else {
    // ---- warps 1-13: the B operand
    build_b_operand<N, 13>(h, nb, s_b, s_scale, wi - 1, lane);
    asm volatile("bar.sync 1, %0;" ::"n"(kMmaThreads - 32) : "memory");  // warps 1-13
    const uint32_t tbase = *s_tmem;
    tc_fence_after();

    if (wi == 1) {
      // ---- MMA issuer
      if (lane == 0) {
        constexpr uint32_t idesc = mma_idesc_f16(2 * N);
        const uint32_t b0 = smem_u32(s_b);
        int issued = 0;
        for (int i = 0; i < n_items; ++i) {
          const int qq = i & 3, ts = i % kSlots;
          if (!mbar_wait(smem_u32(&slab_full[qq]), (i >> 2) & 1, s_abort)) break;
          if (!mbar_wait(smem_u32(&acc_empty[ts]), ((i / kSlots) & 1) ^ 1, s_abort)) break;
          tc_fence_after();
          const uint32_t a0 = smem_u32(s_slab + qq * kMmaSlabBytes);
#pragma unroll
          for (int bl = 0; bl < 2; ++bl) {
            const uint32_t d_tmem = tbase + ts * (4 * N) + bl * (2 * N);
#pragma unroll
            for (int w = 0; w < 2; ++w) {
              const uint32_t in_atom = 64 * bl + 32 * w;  // bytes into the 128-byte row
              const uint64_t ad = sw128_desc(a0 + in_atom);
              const uint64_t bd = sw128_desc(b0 + qq * (2 * N * 128) + in_atom);
              mma_f16(d_tmem, ad, bd, idesc, w != 0);
            }
          }
          mma_commit(smem_u32(&slab_free[qq]));
          mma_commit(smem_u32(&acc_full[ts]));
          issued = i + 1;
        }
        if (*s_abort && issued > 0) {
          // the last commit completes once every MMA issued before it has
          const int i = issued - 1;
          drain_wait(smem_u32(&acc_full[i % kSlots]), (i / kSlots) & 1);
        }
      }
    } else if (wi < 10) {
      // ---- converter team T: quarters T and T + 2 of every tile
      const int T = wi >= 6;
      const int r = 32 * ((wi - 2) & 3) + lane;  // tile row
      bool live = true;
      for (int j = 0; j < my_tiles && live; ++j) {
        const int st = j % kRaw;
        const uint8_t* raw_row = s_raw + st * kMmaRawBytes + r * kQ8RowBytesT;
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
          const int qq = T + 2 * h2, i = 4 * j + qq, di = i % kMmaDRing;
          bool ok = h2 == 1 || mbar_wait(smem_u32(&raw_full[st]), (j / kRaw) & 1, s_abort);
          ok = ok && mbar_wait(smem_u32(&slab_free[qq]), (j & 1) ^ 1, s_abort);
          ok = ok && mbar_wait(smem_u32(&d_free[di]), ((i / kMmaDRing) & 1) ^ 1, s_abort);
          if (!__all_sync(0xffffffffu, ok)) {
            live = false;
            break;
          }
          uint8_t* slab = s_slab + qq * kMmaSlabBytes;
          float* d = s_d + di * 2 * kMmaRows;
          if (qq == 0)
            q8_convert_quarter<0>(raw_row, slab, d, r);
          else if (qq == 1)
            q8_convert_quarter<1>(raw_row, slab, d, r);
          else if (qq == 2)
            q8_convert_quarter<2>(raw_row, slab, d, r);
          else
            q8_convert_quarter<3>(raw_row, slab, d, r);
          fence_proxy_async_smem();
          mbar_arrive(smem_u32(&slab_full[qq]));
          mbar_arrive(smem_u32(&d_full[di]));
        }
        if (live) mbar_arrive(smem_u32(&raw_empty[st]));
      }
    } else {
      // ---- epilogue: thread = tile row = TMEM lane
      const int q = wi & 3;
      const int r = 32 * q + lane;
      bool live = true;
      for (int j = 0; j < my_tiles && live; ++j) {
        float acc[N];
#pragma unroll
        for (int c = 0; c < N; ++c) acc[c] = 0.f;
        for (int qq = 0; qq < 4; ++qq) {
          const int i = 4 * j + qq, ts = i % kSlots, di = i % kMmaDRing;
          bool ok = mbar_wait(smem_u32(&acc_full[ts]), (i / kSlots) & 1, s_abort);
          ok = ok && mbar_wait(smem_u32(&d_full[di]), (i / kMmaDRing) & 1, s_abort);
          if (!__all_sync(0xffffffffu, ok)) {
            live = false;
            break;
          }
          tc_fence_after();
          const uint32_t ta = tbase + (static_cast<uint32_t>(32 * q) << 16) + ts * (4 * N);
          const float* d = s_d + di * 2 * kMmaRows;
#pragma unroll
          for (int bl = 0; bl < 2; ++bl) {
            const float dv = d[bl * kMmaRows + r];
            // (columns in chunks of 16, or 8 at N >= 48 to stay within the registers)
            constexpr int kC = N >= 48 ? 8 : 16;
#pragma unroll
            for (int c = 0; c < N; c += kC) {
              float vh[kC], vl[kC];
              if constexpr (kC == 16) {
                tmem_ld16(ta + bl * (2 * N) + c, vh);
                tmem_ld16(ta + bl * (2 * N) + N + c, vl);
              } else {
                tmem_ld8(ta + bl * (2 * N) + c, vh);
                tmem_ld8(ta + bl * (2 * N) + N + c, vl);
              }
              tmem_ld_wait();
#pragma unroll
              for (int k = 0; k < kC; ++k)
                acc[c + k] = __fmaf_rn(dv, __fadd_rn(vh[k], vl[k]), acc[c + k]);
            }
          }
          tc_fence_before();
          mbar_arrive(smem_u32(&acc_empty[ts]));
          mbar_arrive(smem_u32(&d_free[di]));
        }
        if (!live) break;
        const long long t = blockIdx.x + static_cast<long long>(j) * gridDim.x;
        const long long row = t * kMmaRows + r;
        if (row < V) {
#pragma unroll
          for (int c = 0; c < N; ++c)
            if (c < nb)
              y[static_cast<long long>(c) * ldy + row] =
                  __fmul_rn(__fmul_rn(acc[c], s_scale[c]), s_scale[64 + c]);
        }
      }
    }
  }

  __syncthreads();
  if (wi == 0) tmem_free_all(*s_tmem);
}

// ---------------------------------------------------------------- the F16 table

// The same mat-vec over an F16 table (V x 256 halves, row-major): one float32 accumulator per
// (row, hi/lo part, state) over all 256 k, so no per-block scale and no conversion. The tensor
// memory accelerator (TMA) loads each quarter tile (128 rows x 64 halves) straight into a
// 128-byte-swizzled A stage, 8 stages (128 KB) in flight. One CTA per SM, 6 warps: warp 0 one
// lane issues the TMA loads, warp 1 one lane the MMAs (4 K-steps per quarter, 16 per tile,
// N = 2 x 16..64, into the tile's accumulator slot; a commit frees each stage, another marks
// the tile's accumulators ready), warps 2-5 read the accumulators (thread = row = TMEM lane)
// and write y = (D_hi + D_lo) 2^-e_b; warps 1-5 build the B operand first.
//   y[b, r] = 2^-e_b (sum_k W[r, k] hi[b, k] + sum_k W[r, k] lo[b, k])
// Every product is exact in float32; the tensor cores sum them in float32.
constexpr int kF16MmaThreads = 192;
constexpr int kF16Stages = 8;                    // A stages of 16 KB
constexpr int kF16StageBytes = kMmaRows * 128;   // 128 rows x 64 halves

__host__ __device__ constexpr int f16_tmem_slots(int n) { return 512 / (2 * n) < 4 ? 512 / (2 * n) : 4; }
__host__ __device__ constexpr int f16_mma_smem(int n) {
  return 4 * 2 * n * 128 + kF16Stages * kF16StageBytes + 1024 + 1024;
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y,
                                            uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
      "[%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}

template <int N>
__global__ void __launch_bounds__(kF16MmaThreads, 1)
    markov_f16_mma_kernel(const __grid_constant__ CUtensorMap tmap, int V, const float* h, int nb,
                          float* y, int ldy, int withhold) {
  constexpr int kSlots = f16_tmem_slots(N);
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
  uint8_t* s_b = sm;                                  // 4 atoms x 2N rows x 128 B
  uint8_t* s_a = sm + 4 * 2 * N * 128;                // kF16Stages x 16 KB
  uint64_t* bars = reinterpret_cast<uint64_t*>(s_a + kF16Stages * kF16StageBytes);
  uint64_t* a_full = bars;                            // [8] TMA (expect_tx) + bytes
  uint64_t* a_free = bars + 8;                        // [8] MMA commit
  uint64_t* acc_full = bars + 16;                     // [4] MMA commit
  uint64_t* acc_empty = bars + 20;                    // [4] the epilogue (128)
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(bars + 24);
  volatile int* s_abort = reinterpret_cast<volatile int*>(bars + 25);
  float* s_scale = reinterpret_cast<float*>(bars + 26);  // [2][64]

  const int tid = threadIdx.x, wi = tid >> 5, lane = tid & 31;
  const int n_tiles = (V + kMmaRows - 1) / kMmaRows;
  const int my_tiles = blockIdx.x < n_tiles ? (n_tiles - 1 - blockIdx.x) / gridDim.x + 1 : 0;

  if (tid == 0) {
    for (int i = 0; i < kF16Stages; ++i) {
      mbar_init(smem_u32(&a_full[i]), 1);
      mbar_init(smem_u32(&a_free[i]), 1);
    }
    for (int i = 0; i < 4; ++i) {
      mbar_init(smem_u32(&acc_full[i]), 1);
      mbar_init(smem_u32(&acc_empty[i]), kMmaTeam);
    }
    *s_abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap)) : "memory");
  }
  if (wi == 0) tmem_alloc_all(s_tmem);
  __syncthreads();

  grid_dependency_wait();  // h comes from the kernel before (programmatic launch)
  grid_dependents_launch();

  if (wi == 0) {
    // ---- producer: one TMA load per quarter tile
    if (lane == 0) {
      const int n_items = 4 * my_tiles;
      int armed = 0;
      for (int i = 0; i < n_items; ++i) {
        const int st = i % kF16Stages;
        if (!mbar_wait(smem_u32(&a_free[st]), ((i / kF16Stages) & 1) ^ 1, s_abort)) break;
        const int t = blockIdx.x + (i >> 2) * gridDim.x;
        if (withhold && i == 0) continue;  // (timeout test: this stage never arrives)
        mbar_arrive_tx(smem_u32(&a_full[st]), kF16StageBytes);
        tma_load_2d(smem_u32(s_a + st * kF16StageBytes), &tmap, 64 * (i & 3), t * kMmaRows,
                    smem_u32(&a_full[st]));
        armed = i + 1;
      }
      if (*s_abort) {
        for (int i = armed - kF16Stages < 0 ? 0 : armed - kF16Stages; i < armed; ++i) {
          if (withhold && i == 0) continue;
          drain_wait(smem_u32(&a_full[i % kF16Stages]), (i / kF16Stages) & 1);
        }
      }
    }
  } else {
    build_b_operand<N, 5>(h, nb, s_b, s_scale, wi - 1, lane);
    asm volatile("bar.sync 1, %0;" ::"n"(kF16MmaThreads - 32) : "memory");  // warps 1-5
    const uint32_t tbase = *s_tmem;
    tc_fence_after();
    if (wi == 1) {
      // ---- MMA issuer
      if (lane == 0) {
        constexpr uint32_t idesc = mma_idesc_f16(2 * N);
        const uint32_t b0 = smem_u32(s_b);
        int last = -1;
        bool live = true;
        for (int j = 0; j < my_tiles && live; ++j) {
          const int ts = j % kSlots;
          if (!mbar_wait(smem_u32(&acc_empty[ts]), ((j / kSlots) & 1) ^ 1, s_abort)) break;
          for (int qq = 0; qq < 4; ++qq) {
            const int i = 4 * j + qq, st = i % kF16Stages;
            if (!mbar_wait(smem_u32(&a_full[st]), (i / kF16Stages) & 1, s_abort)) {
              live = false;
              break;
            }
            tc_fence_after();
            const uint32_t a0 = smem_u32(s_a + st * kF16StageBytes);
#pragma unroll
            for (int w = 0; w < 4; ++w)
              mma_f16(tbase + ts * (2 * N), sw128_desc(a0 + 32 * w),
                      sw128_desc(b0 + qq * (2 * N * 128) + 32 * w), idesc, (qq | w) != 0);
            mma_commit(smem_u32(&a_free[st]));
          }
          if (!live) break;
          mma_commit(smem_u32(&acc_full[ts]));
          last = j;
        }
        if (*s_abort && last >= 0) {
          drain_wait(smem_u32(&acc_full[last % kSlots]), (last / kSlots) & 1);
        }
      }
    } else {
      // ---- epilogue: thread = tile row = TMEM lane
      const int q = wi & 3;
      const int r = 32 * q + lane;
      for (int j = 0; j < my_tiles; ++j) {
        const int ts = j % kSlots;
        if (!__all_sync(0xffffffffu,
                        mbar_wait(smem_u32(&acc_full[ts]), (j / kSlots) & 1, s_abort)))
          break;
        tc_fence_after();
        const uint32_t ta = tbase + (static_cast<uint32_t>(32 * q) << 16) + ts * (2 * N);
        const long long row = static_cast<long long>(blockIdx.x + j * gridDim.x) * kMmaRows + r;
#pragma unroll
        for (int c = 0; c < N; c += 16) {
          float vh[16], vl[16];
          tmem_ld16(ta + c, vh);
          tmem_ld16(ta + N + c, vl);
          tmem_ld_wait();
          if (row < V) {
#pragma unroll
            for (int k = 0; k < 16; ++k)
              if (c + k < nb)
                y[static_cast<long long>(c + k) * ldy + row] = __fmul_rn(
                    __fmul_rn(__fadd_rn(vh[k], vl[k]), s_scale[c + k]), s_scale[64 + c + k]);
          }
        }
        tc_fence_before();
        mbar_arrive(smem_u32(&acc_empty[ts]));
      }
    }
  }

  __syncthreads();
  if (wi == 0) tmem_free_all(*s_tmem);
}

// ---------------------------------------------------------------- Q8_0, few states, int8

// The Q8_0 mat-vec for 1 to 10 states on the integer tensor cores (kind::i8), with no
// conversion: the table bytes are the A operand as stored. TMA copies each tile's 272-byte rows
// in 3 windows of 128 bytes (128 rows x 128 bytes, 128-byte swizzle; the bytes past 272 read as
// zeros) into one shared stage, and 9 MMAs (one per 32-byte K step) accumulate the whole row
// into one set of int32 columns: column j G + p NB + s belongs to block j, digit plane p,
// state s (three signed-byte digit planes per state and block, as in the CUDA-core kernel;
// G = 3 NB, or 3 NB rounded up to 8 beyond 5 states).
// B column (j, p, s) holds those digits at block j's 32 byte positions (34 j + 2 ..) and zeros
// everywhere else, so each column sums block j's products alone: the scale bytes and the other
// blocks drop out, and the sums are exact. The epilogue (thread = row = TMEM lane) reads each
// block's scale d from the staged bytes and adds
//   d 2^(x_sj - X_s) (A + (B + C / 254) / 254)
// over the 8 blocks (x_sj the block's digit exponent, X_s the state's largest), then writes
// 2^X_s times the sum. One CTA per SM, 6 warps: warp 0 one lane issues the TMA copies (3-4
// tile stages), warp 1 one lane the 9 MMAs per tile and their commit, warps 2-5 the epilogue,
// which also releases the stage (its scale bytes are read there); warps 1-5 build the digits
// first.
constexpr int kI8Threads = 192;
constexpr int kI8MaxStates = 10;
constexpr int kI8Windows = 3;                      // 128-byte windows per 272-byte row
constexpr int kI8WinBytes = kMmaRows * 128;        // 16384
constexpr int kI8TileBytes = kI8Windows * kI8WinBytes;  // 49152
constexpr int kI8KSteps = 9;                       // 32-byte K steps covering 272 bytes

// Columns per block: 3 NB (up to 5 states, blocks packed), else 3 NB rounded up to 8 (so each
// block's columns load as whole 8-column groups); MMA N for NB states (8 blocks, rounded up to
// 16), its tile stages and accumulator slots in the 512 TMEM columns
__host__ __device__ constexpr int i8_g(int nb) { return nb <= 5 ? 3 * nb : (3 * nb + 7) / 8 * 8; }
__host__ __device__ constexpr int i8_n(int nb) {
  return nb <= 5 ? (24 * nb + 15) / 16 * 16 : 8 * i8_g(nb);
}
__host__ __device__ constexpr int i8_stages(int nb) { return nb <= 4 ? 4 : 3; }
__host__ __device__ constexpr int i8_slots(int nb) { return 512 / i8_n(nb) < 4 ? 512 / i8_n(nb) : 4; }
__host__ __device__ constexpr int i8_b_bytes(int nb) { return kI8KSteps * i8_n(nb) * 32; }
__host__ __device__ constexpr int i8_mma_smem(int nb) {
  return i8_stages(nb) * kI8TileBytes + i8_b_bytes(nb) + 1024 + 1024;
}

// Shared-memory descriptor of a K-major operand in the 32-byte swizzle layout: rows of 32
// bytes, 8-row groups 256 bytes apart, the 16-byte chunk c of row r stored at c ^ ((r / 4) % 2).
__device__ __forceinline__ uint64_t sw32_desc(uint32_t saddr) {
  return static_cast<uint64_t>((saddr >> 4) & 0x3FFFu) | (1ull << 16) |  // leading offset (unused)
         (16ull << 32) |                                                // group stride 256 B
         (1ull << 46) |                                                 // descriptor version
         (6ull << 61);                                                  // 32-byte swizzle
}

// Instruction descriptor: kind::i8, A and B signed 8-bit, K-major, D signed 32-bit, M = 128, N.
__host__ __device__ constexpr uint32_t mma_idesc_s8(int n) {
  return (2u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(n >> 3) << 17) |
         (static_cast<uint32_t>(128 >> 4) << 24);
}

__device__ __forceinline__ void mma_s8(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                       uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// 4 consecutive 32-bit TMEM columns of this warp's 32 lanes.
__device__ __forceinline__ void tmem_ld4(uint32_t taddr, float* v) {
  uint32_t r[4];
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(taddr)
               : "memory");
#pragma unroll
  for (int i = 0; i < 4; ++i) v[i] = __uint_as_float(r[i]);
}

// Byte offset of (row n, byte k) in a 32-byte-swizzled K-major operand.
__device__ __forceinline__ int sw32_off(int n, int k) {
  return n * 32 + ((((k >> 4) ^ (n >> 2)) & 1) << 4) + (k & 15);
}
// Byte offset of (row n, byte k < 128) in a 128-byte-swizzled atom.
__device__ __forceinline__ int sw128_off(int n, int k) {
  return n * 128 + ((((k >> 4) ^ n) & 7) << 4) + (k & 15);
}

template <int NB>
__global__ void __launch_bounds__(kI8Threads, 1)
    markov_q8_0_i8_kernel(const __grid_constant__ CUtensorMap tmap, int V, const float* h,
                          float* y, int ldy, int withhold) {
  constexpr int kN = i8_n(NB);
  constexpr int kG = i8_g(NB);
  constexpr int kStages = i8_stages(NB);
  constexpr int kSlots = i8_slots(NB);
  constexpr int kBBytes = i8_b_bytes(NB);
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
  uint8_t* s_a = sm;                                   // kStages x 3 windows x 16 KB
  uint8_t* s_b = sm + kStages * kI8TileBytes;          // [K step][kN x 32 B]
  uint64_t* bars = reinterpret_cast<uint64_t*>(s_b + kBBytes);
  uint64_t* t_full = bars;          // [4] TMA (expect_tx) + bytes
  uint64_t* t_free = bars + 4;      // [4] the epilogue (128)
  uint64_t* acc_full = bars + 8;    // [4] MMA commit
  uint64_t* acc_empty = bars + 12;  // [4] the epilogue (128)
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(bars + 16);
  volatile int* s_abort = reinterpret_cast<volatile int*>(bars + 17);
  int* s_x = reinterpret_cast<int*>(bars + 18);        // [NB][8] block exponents

  const int tid = threadIdx.x, wi = tid >> 5, lane = tid & 31;
  const int n_tiles = (V + kMmaRows - 1) / kMmaRows;
  const int my_tiles = blockIdx.x < n_tiles ? (n_tiles - 1 - blockIdx.x) / gridDim.x + 1 : 0;

  if (tid == 0) {
    for (int i = 0; i < 4; ++i) {
      mbar_init(smem_u32(&t_full[i]), 1);
      mbar_init(smem_u32(&t_free[i]), kMmaTeam);
      mbar_init(smem_u32(&acc_full[i]), 1);
      mbar_init(smem_u32(&acc_empty[i]), kMmaTeam);
    }
    *s_abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap)) : "memory");
  }
  if (wi == 0) tmem_alloc_all(s_tmem);
  // the B operands start as zeros (warps 1-5)
  for (int i = tid - 32; i >= 0 && i < kBBytes / 16; i += kI8Threads - 32)
    reinterpret_cast<uint4*>(s_b)[i] = make_uint4(0, 0, 0, 0);
  __syncthreads();

  grid_dependency_wait();  // h comes from the kernel before (programmatic launch)
  grid_dependents_launch();

  if (wi == 0) {
    // ---- producer: 3 TMA copies per tile into one stage
    if (lane == 0) {
      int armed = 0;
      for (int j = 0; j < my_tiles; ++j) {
        const int st = j % kStages;
        if (!mbar_wait(smem_u32(&t_free[st]), ((j / kStages) & 1) ^ 1, s_abort)) break;
        const int t = blockIdx.x + j * gridDim.x;
        if (withhold && j == 0) continue;  // (timeout test: this tile never arrives)
        mbar_arrive_tx(smem_u32(&t_full[st]), kI8TileBytes);
#pragma unroll
        for (int w = 0; w < kI8Windows; ++w)
          tma_load_2d(smem_u32(s_a + st * kI8TileBytes + w * kI8WinBytes), &tmap, 128 * w,
                      t * kMmaRows, smem_u32(&t_full[st]));
        armed = j + 1;
      }
      if (*s_abort) {
        for (int j = armed - kStages < 0 ? 0 : armed - kStages; j < armed; ++j) {
          if (withhold && j == 0) continue;
          drain_wait(smem_u32(&t_full[j % kStages]), (j / kStages) & 1);
        }
      }
    }
  } else {
    // ---- warps 1-5: digits of (state s, block j) pairs t = s * 8 + j, warp w taking pairs
    // w - 1, w + 4, ...; all of a warp's state values are loaded before any is used
    constexpr int kPairs = (NB * kQ8Blocks + 4) / 5;
    float hvs[kPairs];
#pragma unroll
    for (int u = 0; u < kPairs; ++u) {
      const int t = wi - 1 + 5 * u;
      hvs[u] = t < NB * kQ8Blocks ? __ldg(h + (t / kQ8Blocks) * kMarkovRank + (t % kQ8Blocks) * 32 + lane) : 0.f;
    }
#pragma unroll
    for (int u = 0; u < kPairs; ++u) {
      const int t = wi - 1 + 5 * u;
      if (t >= NB * kQ8Blocks) break;
      const int st = t / kQ8Blocks, j = t % kQ8Blocks;
      const float hv = hvs[u];
      const float ah = fabsf(hv);
      const uint32_t mb = __reduce_max_sync(0xffffffffu, __float_as_uint(ah));
      const float m = __uint_as_float(mb);
      int x = 0;
      if (m > 0.f && m <= 3.402823466e38f) {
        const int be = static_cast<int>(mb >> 23);
        const int lg = be != 0 ? be - 127 : -149 + (31 - __clz(static_cast<int>(mb & 0x7fffffu)));
        x = lg - 6;
        if (mul_pow2(m, -x) > 127.f) x += 1;
      }
      const float v = mul_pow2(hv, -x);
      const float a = rintf(v);
      const float r1 = __fmul_rn(__fsub_rn(v, a), 254.f);
      const float bb = rintf(r1);
      const float c = rintf(__fmul_rn(__fsub_rn(r1, bb), 254.f));
      // element lane of block j is table byte g = 34 j + 2 + lane: K step g / 32, byte g % 32;
      // B columns j kG + p NB + st
      const int g = 34 * j + 2 + lane;
      uint8_t* bm = s_b + (g >> 5) * (kN * 32);
      const int n0 = j * kG + st;
      bm[sw32_off(n0, g & 31)] = static_cast<uint8_t>(static_cast<int8_t>(a));
      bm[sw32_off(n0 + NB, g & 31)] = static_cast<uint8_t>(static_cast<int8_t>(bb));
      bm[sw32_off(n0 + 2 * NB, g & 31)] = static_cast<uint8_t>(static_cast<int8_t>(c));
      if (lane == 0) s_x[st * 8 + j] = m <= 3.402823466e38f ? x : 1024;  // 1024: non-finite
    }
    fence_proxy_async_smem();
    asm volatile("bar.sync 1, %0;" ::"n"(kI8Threads - 32) : "memory");  // warps 1-5
    const uint32_t tbase = *s_tmem;
    tc_fence_after();
    if (wi == 1) {
      // ---- MMA issuer: per tile, per block, its two 32-byte K steps into the block's columns
      if (lane == 0) {
        constexpr uint32_t idesc = mma_idesc_s8(kN);
        const uint32_t b0 = smem_u32(s_b);
        int last = -1;
        for (int j = 0; j < my_tiles; ++j) {
          const int st = j % kStages, ts = j % kSlots;
          if (!mbar_wait(smem_u32(&t_full[st]), (j / kStages) & 1, s_abort)) break;
          if (!mbar_wait(smem_u32(&acc_empty[ts]), ((j / kSlots) & 1) ^ 1, s_abort)) break;
          tc_fence_after();
          const uint32_t a0 = smem_u32(s_a + st * kI8TileBytes);
#pragma unroll
          for (int k = 0; k < kI8KSteps; ++k)  // K step k: window k / 4, 32 (k % 4) bytes in
            mma_s8(tbase + ts * kN, sw128_desc(a0 + (k >> 2) * kI8WinBytes + 32 * (k & 3)),
                   sw32_desc(b0 + k * (kN * 32)), idesc, k != 0);
          mma_commit(smem_u32(&acc_full[ts]));
          last = j;
        }
        if (*s_abort && last >= 0) {
          drain_wait(smem_u32(&acc_full[last % kSlots]), (last / kSlots) & 1);
        }
      }
    } else {
      // ---- epilogue: thread = tile row = TMEM lane
      const int q = wi & 3;
      const int r = 32 * q + lane;
      // per state: X_s and (up to 5 states, in registers) the block factors 2^(x_sj - X_s)
      // (0 below 2^-126)
      int X[NB];
      constexpr int kGf = NB <= 5 ? NB : 1;
      float gf[kGf][kQ8Blocks];
#pragma unroll
      for (int s2 = 0; s2 < NB; ++s2) {
        int mx = s_x[s2 * 8];
#pragma unroll
        for (int j = 1; j < kQ8Blocks; ++j) mx = max(mx, s_x[s2 * 8 + j]);
        X[s2] = mx;
        if constexpr (NB <= 5) {
#pragma unroll
          for (int j = 0; j < kQ8Blocks; ++j) {
            const int dx = s_x[s2 * 8 + j] - mx;
            gf[s2][j] = dx >= -126 ? pow2f(dx) : 0.f;
          }
        }
      }
      for (int j = 0; j < my_tiles; ++j) {
        const int st = j % kStages, ts = j % kSlots;
        if (!__all_sync(0xffffffffu,
                        mbar_wait(smem_u32(&acc_full[ts]), (j / kSlots) & 1, s_abort)))
          break;
        tc_fence_after();
        const uint32_t ta = tbase + (static_cast<uint32_t>(32 * q) << 16) + ts * kN;
        const uint8_t* tile = s_a + st * kI8TileBytes;
        float dd[kQ8Blocks];
#pragma unroll
        for (int blk = 0; blk < kQ8Blocks; ++blk) {
          // the block's scale: bytes 34 blk .. 34 blk + 1 (even; one 16-byte chunk)
          const int o = 34 * blk;
          dd[blk] = __half2float(*reinterpret_cast<const __half*>(
              tile + (o >> 7) * kI8WinBytes + sw128_off(r, o & 127)));
        }
        float acc[NB];
#pragma unroll
        for (int s2 = 0; s2 < NB; ++s2) acc[s2] = 0.f;
        // block blk's plane digits of state s2, as integers, into acc
        auto add_block = [&](const float* vb, int blk, float gfac, int s2) {
          const int A = __float_as_int(vb[s2]), Bv = __float_as_int(vb[s2 + NB]),
                    C = __float_as_int(vb[s2 + 2 * NB]);
          float f = __fmaf_rn(small_int_to_float(C), 1.f / 254.f, small_int_to_float(Bv));
          f = __fmaf_rn(f, 1.f / 254.f, small_int_to_float(A));
          acc[s2] = __fmaf_rn(__fmul_rn(dd[blk], gfac), f, acc[s2]);
        };
        if constexpr (NB <= 5) {
          // every column at once, one wait
          float v[kN];
#pragma unroll
          for (int c = 0; c < kN; c += 16) tmem_ld16(ta + c, v + c);
          tmem_ld_wait();
#pragma unroll
          for (int blk = 0; blk < kQ8Blocks; ++blk)
#pragma unroll
            for (int s2 = 0; s2 < NB; ++s2) add_block(v + blk * kG, blk, gf[s2][blk], s2);
        } else {
          // block by block: its kG columns as 8-column loads, one wait each
#pragma unroll
          for (int blk = 0; blk < kQ8Blocks; ++blk) {
            float v[kG];
#pragma unroll
            for (int c = 0; c < kG; c += 8) tmem_ld8(ta + blk * kG + c, v + c);
            tmem_ld_wait();
#pragma unroll
            for (int s2 = 0; s2 < NB; ++s2) {
              const int dx = s_x[s2 * 8 + blk] - X[s2];
              add_block(v, blk, dx >= -126 ? pow2f(dx) : 0.f, s2);
            }
          }
        }
        tc_fence_before();
        mbar_arrive(smem_u32(&acc_empty[ts]));
        mbar_arrive(smem_u32(&t_free[st]));
        const long long row = static_cast<long long>(blockIdx.x + j * gridDim.x) * kMmaRows + r;
        if (row < V) {
#pragma unroll
          for (int s2 = 0; s2 < NB; ++s2)
            y[static_cast<long long>(s2) * ldy + row] =
                X[s2] >= 1024 ? __int_as_float(0x7fc00000) : mul_pow2(acc[s2], X[s2]);
        }
      }
    }
  }

  __syncthreads();
  if (wi == 0) tmem_free_all(*s_tmem);
}

}  // namespace dspark
