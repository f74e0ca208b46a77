// C ABI of the DSpark block verify/accept step: argument checks, launch planning and the
// two kernel launches of a call (pass 1 in stream.cuh, pass 2 in finish.cuh).
#include <atomic>
#include <climits>
#include <cmath>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "common.cuh"
#include "early_exit.cuh"
#include "finish.cuh"
#include "markov.cuh"
#include "markov_mma.cuh"
#include "stream.cuh"

namespace dspark {
namespace {

constexpr int kAbiVersion = 6;  // 6: dspark_pipeline_timeouts
constexpr int kMaxDevices = 64;

// Tuning switch, read at every call: DSPARK_MAX_CTAS caps the pass-1 CTAs (0 = one per SM).
int max_ctas_override() {
  const char* s = std::getenv("DSPARK_MAX_CTAS");
  const int n = s ? std::atoi(s) : 0;
  return n > 0 ? n : 0;
}

// ------------------------------------------------------------------------------ plans

int elem_bytes(dspark_dtype_t dt) { return dt == DSPARK_F32 ? 4 : 2; }

bool shape_ok(int B, int K, int V) {
  if (B < 0 || K < 0 || K > kMaxK || V < 1) return false;
  if (static_cast<long long>(B) * (2 * K + 1) >= (1LL << 31)) return false;
  return true;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

struct Plan {
  int vec;  // elements per load: 16-byte vectors (8 bf16 / 4 fp32) or 1
  int nch;  // 2048-token chunks per row
  int fw;   // warps per sampling-finish CTA: 16 (small batches) or 32
  int G;    // pass-2 CTAs per sequence (one cluster), sampling
  int cpc;  // chunks per pass-2 CTA
};

bool make_plan(int B, int V, dspark_dtype_t dt, bool aligned16, Plan* pl) {
  const int es = elem_bytes(dt);
  const long long nch = (static_cast<long long>(V) + kCE - 1) / kCE;
  if (nch < 1 || nch > kMaxChunkCount) return false;
  pl->vec = aligned16 ? 16 / es : 1;
  pl->nch = static_cast<int>(nch);
  // sampling finish, one CTA per SM and one chunk per warp: CTAs of 16 warps (G = ceil(nch /
  // 16) <= 8 per cluster, each warp's chunk in one load round) while the batch's clusters fit
  // on the SMs of a B200, else 32 warps (G = ceil(nch / 32) <= 4)
  const int g16 = (pl->nch + kFinWarpsSmall - 1) / kFinWarpsSmall;
  if (static_cast<long long>(B) * g16 <= kPlanSMs) {
    pl->fw = kFinWarpsSmall;
    pl->G = g16;
  } else {
    pl->fw = kFinWarps;
    pl->G = (pl->nch + kFinWarps - 1) / kFinWarps;
  }
  pl->cpc = (pl->nch + pl->G - 1) / pl->G;
  return true;
}

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// Workspace: the pass-1 records, one float2 per (row, chunk) unit of 2K+1 rows per sequence,
// then the draft tokens' logits (sampling), then what the early-exit waves keep: each
// sequence's decision, two lists of alive sequences and the per-wave alive counts. Pass 1
// writes every record, and the gather of every draft id in [0, V), before pass 2 reads them;
// the first early-exit wave zeroes the counts; so the workspace needs no initialisation.
struct WsLayout {
  size_t rec, gather, dec, alive, cnt, total;
};

WsLayout ws_layout(long long B, long long K, int nch) {
  const long long rows = 2 * K + 1;
  WsLayout w{};
  w.rec = 0;
  w.gather = align256(sizeof(float2) * static_cast<size_t>(B * rows * nch));
  w.dec = w.gather + align256(sizeof(float2) * static_cast<size_t>(B * K));
  w.alive = w.dec + align256(sizeof(Decision) * static_cast<size_t>(B));
  w.cnt = w.alive + align256(sizeof(int) * 2 * static_cast<size_t>(B));
  w.total = w.cnt + align256(sizeof(int) * kMaxWaves);
  return w;
}

// Early-exit waves for K drafts: pairs [2^w - 1, 2^(w+1) - 1) cut at K, the last one ending at K.
int n_waves(const WaveSchedule& ws, int K) {
  int w = 0, lo = 0, hi = 0;
  for (;; ++w) {
    wave_range(ws, w, K, lo, hi);
    if (hi >= K) return w + 1;
  }
}

// Constants of FastDiv for divisor d >= 1 (see stream.cuh).
FastDiv fast_div(uint32_t d) {
  FastDiv f{};
  uint32_t s = 0;
  while ((1ull << s) < d) ++s;
  const unsigned __int128 num = static_cast<unsigned __int128>(1) << (32 + s);
  const unsigned __int128 m = (num + d - 1) / d;
  f.m_lo = static_cast<uint32_t>(m & 0xffffffffu);
  f.hs = static_cast<uint32_t>(m >> 32) << 8 | s;
  return f;
}

// --------------------------------------------------------------- per-device launch state

std::mutex g_mu;
struct OccEntry {
  const void* fn;
  int dev;
  size_t smem;
  int ctas;  // co-resident CTAs of the kernel on the device
};
OccEntry g_occ[64];
int g_occ_n = 0;
struct SmemLimit {
  const void* fn;
  int dev;
  size_t bytes;  // the kernel's dynamic shared-memory limit, as last raised
};
SmemLimit g_lim[64];
int g_lim_n = 0;

// CTAs of `fn` (`threads` threads, `smem` dynamic shared memory) resident on the current
// device at once. Raises the kernel's dynamic shared-memory limit first when `smem` is above
// it; the limit is never lowered, so a call that needs less shared memory cannot break a
// later call that needs more.
int resident_ctas(const void* fn, int threads, size_t smem, cudaError_t* err) {
  int dev = 0;
  *err = cudaGetDevice(&dev);
  if (*err != cudaSuccess) return 0;
  std::lock_guard<std::mutex> lk(g_mu);
  SmemLimit* lim = nullptr;
  for (int n = 0; n < g_lim_n; ++n)
    if (g_lim[n].fn == fn && g_lim[n].dev == dev) lim = &g_lim[n];
  if (smem > 0 && (!lim || smem > lim->bytes)) {
    *err = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                static_cast<int>(smem));
    if (*err != cudaSuccess) return 0;
    if (!lim && g_lim_n < 64) {
      g_lim[g_lim_n] = SmemLimit{fn, dev, 0};
      lim = &g_lim[g_lim_n++];
    }
    if (lim) lim->bytes = smem;
  }
  for (int n = 0; n < g_occ_n; ++n)
    if (g_occ[n].fn == fn && g_occ[n].dev == dev && g_occ[n].smem == smem) return g_occ[n].ctas;
  int per_sm = 0, sms = 0;
  *err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, threads, smem);
  if (*err != cudaSuccess) return 0;
  *err = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (*err != cudaSuccess) return 0;
  const int n = per_sm * sms;
  if (g_occ_n < 64) g_occ[g_occ_n++] = OccEntry{fn, dev, smem, n};
  return n;
}

struct Call {
  RowSet rs;
  int B;
  const int32_t* drafts;
  const float* uniforms;
  const int32_t* n_drafts;  // mixed batch: [B] or null
  const float* temps;       // mixed batch: [B]
  float scale;
  dspark_accept_out_t out;
  char* ws;
};

// The sampling finish: one cluster of pl.G CTAs of kW warps per sequence, each with pl.cpc
// chunks of group sums in dynamic shared memory, as a programmatic dependent of the kernel
// before it.
template <typename T, int VEC, int kFin, int kW>
dspark_status_t launch_finish_sample_w(const FinishParamsOf<kFin>& fp, const Plan& pl, int B,
                                       cudaStream_t stream) {
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = static_cast<unsigned>(pl.G);
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(static_cast<long long>(B) * pl.G), 1, 1);
  cfg.blockDim = dim3(kW * 32, 1, 1);
  cfg.dynamicSmemBytes = static_cast<size_t>(pl.cpc) * kGroups * sizeof(float);
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  {
    // once per kernel instantiation and device: room for the group sums of up to 32 chunks
    static std::atomic<bool> ready[kMaxDevices];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return DSPARK_ERR_CUDA;
    if (!ready[dev].load(std::memory_order_acquire)) {
      if (cudaFuncSetAttribute(finish_sample_kernel<T, VEC, kFin, kW>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(kFinMaxCpc * kGroups * sizeof(float))) !=
          cudaSuccess)
        return DSPARK_ERR_CUDA;
      ready[dev].store(true, std::memory_order_release);
    }
  }
  return cudaLaunchKernelEx(&cfg, finish_sample_kernel<T, VEC, kFin, kW>, fp) == cudaSuccess
             ? DSPARK_OK
             : DSPARK_ERR_CUDA;
}

template <typename T, int VEC, int kFin>
dspark_status_t launch_finish_sample(const FinishParamsOf<kFin>& fp, const Plan& pl, int B,
                                     cudaStream_t stream) {
  return pl.fw == kFinWarpsSmall
             ? launch_finish_sample_w<T, VEC, kFin, kFinWarpsSmall>(fp, pl, B, stream)
             : launch_finish_sample_w<T, VEC, kFin, kFinWarps>(fp, pl, B, stream);
}

// Pass 1 over every (row, chunk) unit (one CTA per SM, every grid-th unit), then pass 2.
// Both are programmatic dependent launches: pass 1's CTAs become resident while the previous
// kernel in the stream drains and wait for it to complete before reading anything (this hides
// the launch latency between back-to-back calls, about 2 us); pass 2's CTAs load what pass 1
// does not write and then wait for pass 1.
template <typename T, int VEC, int kMode>
dspark_status_t run_call(const Call& c, const Plan& pl, cudaStream_t stream,
                         bool pass1_only = false) {
  constexpr bool kSample = kMode != kModeGreedy;
  constexpr int kFin = kMode == kModeMixed ? kFinMixed : kFinUniform;
  const void* k1 = reinterpret_cast<const void*>(&stream_stats_kernel<T, VEC, kMode>);
  cudaError_t e = cudaSuccess;
  int ctas = resident_ctas(k1, kStreamThreads, 0, &e);
  if (e != cudaSuccess) return DSPARK_ERR_CUDA;
  if (ctas < 1) return DSPARK_ERR_UNSUPPORTED;
  if (max_ctas_override() && max_ctas_override() < ctas) ctas = max_ctas_override();
  const WsLayout w = ws_layout(c.B, c.rs.K, pl.nch);
  const long long n_units = static_cast<long long>(c.B) * c.rs.rows * pl.nch;
  if (n_units >= (1LL << 31)) return DSPARK_ERR_UNSUPPORTED;  // unit indices stay in 32 bits
  const long long want = (n_units + kStreamWarps - 1) / kStreamWarps;
  const int grid1 = static_cast<int>(want < ctas ? want : ctas);

  StreamParamsOf<kMode> sp{};
  sp.rs = c.rs;
  sp.nch = pl.nch;
  sp.n_units = static_cast<uint32_t>(n_units);
  sp.B = c.B;
  sp.by_nch = fast_div(static_cast<uint32_t>(pl.nch));
  sp.by_seqs = fast_div(static_cast<uint32_t>(c.B));
  sp.scale = c.scale;
  sp.rec = reinterpret_cast<float2*>(c.ws + w.rec);
  sp.drafts = c.drafts;
  sp.gather = reinterpret_cast<float*>(c.ws + w.gather);
  if constexpr (kMode == kModeMixed) {
    sp.n_drafts = c.n_drafts;
    sp.temps = c.temps;
  }
  {
    cudaLaunchAttribute a1[1];
    a1[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    a1[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t c1 = {};
    c1.gridDim = dim3(static_cast<unsigned>(grid1), 1, 1);
    c1.blockDim = dim3(kStreamThreads, 1, 1);
    c1.dynamicSmemBytes = 0;
    c1.stream = stream;
    c1.attrs = a1;
    c1.numAttrs = 1;
    e = cudaLaunchKernelEx(&c1, stream_stats_kernel<T, VEC, kMode>, sp);
    if (e != cudaSuccess) return DSPARK_ERR_CUDA;
  }
  if (pass1_only) return DSPARK_OK;

  FinishParamsOf<kFin> fp{};
  fp.rs = c.rs;
  fp.drafts = c.drafts;
  fp.uniforms = c.uniforms;
  fp.nch = pl.nch;
  fp.scale = c.scale;
  fp.rec = sp.rec;
  fp.gather = sp.gather;
  if constexpr (kMode == kModeMixed) {
    fp.n_drafts = c.n_drafts;
    fp.temps = c.temps;
  }
  fp.out = c.out;
  if constexpr (kSample) {
    return launch_finish_sample<T, VEC, kFin>(fp, pl, c.B, stream);
  } else {
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(c.B), 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, finish_greedy_kernel<T>, fp);
    return e == cudaSuccess ? DSPARK_OK : DSPARK_ERR_CUDA;
  }
}

// Early exit (early_exit.cuh): per wave, pass 1 over the alive sequences' rows of the wave and
// the wave's decisions; then, when sampling, the finish from the stored decisions. Every
// launch is a programmatic dependent of the one before.
template <typename T, int VEC, bool kSample>
dspark_status_t run_early_exit(const Call& c, const Plan& pl, cudaStream_t stream) {
  const void* k1 = reinterpret_cast<const void*>(&ee_stream_kernel<T, VEC, kSample>);
  cudaError_t e = cudaSuccess;
  int ctas = resident_ctas(k1, kStreamThreads, 0, &e);
  if (e != cudaSuccess) return DSPARK_ERR_CUDA;
  if (ctas < 1) return DSPARK_ERR_UNSUPPORTED;
  if (max_ctas_override() && max_ctas_override() < ctas) ctas = max_ctas_override();
  const long long total_units = static_cast<long long>(c.B) * c.rs.rows * pl.nch;
  if (total_units >= (1LL << 31)) return DSPARK_ERR_UNSUPPORTED;
  const WsLayout w = ws_layout(c.B, c.rs.K, pl.nch);
  const int K = c.rs.K;
  const WaveSchedule sched = wave_schedule(c.B, c.rs.V, static_cast<int>(sizeof(T)), kSample);
  const int W = n_waves(sched, K);
  int* alive[2] = {reinterpret_cast<int*>(c.ws + w.alive),
                   reinterpret_cast<int*>(c.ws + w.alive) + c.B};
  int* cnt = reinterpret_cast<int*>(c.ws + w.cnt);
  Decision* dec = reinterpret_cast<Decision*>(c.ws + w.dec);

  cudaLaunchAttribute pdl[1];
  pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl[0].val.programmaticStreamSerializationAllowed = 1;
  for (int wv = 0; wv < W; ++wv) {
    WaveArgs wa{};
    wave_range(sched, wv, K, wa.lo, wa.hi);
    wa.last = wv == W - 1;
    wa.wave = wv;
    wa.alive = alive[wv & 1];
    wa.alive_next = alive[(wv + 1) & 1];
    wa.cnt = cnt;

    EeStreamParams sp{};
    sp.rs = c.rs;
    sp.nch = pl.nch;
    sp.B = c.B;
    sp.scale = c.scale;
    sp.rec = reinterpret_cast<float2*>(c.ws + w.rec);
    sp.drafts = c.drafts;
    sp.gather = reinterpret_cast<float*>(c.ws + w.gather);
    sp.wv = wa;
    const long long slots = static_cast<long long>(wa.hi - wa.lo) * (kSample ? 2 : 1) + wa.last;
    const long long want = (static_cast<long long>(c.B) * slots * pl.nch + kStreamWarps - 1) /
                           kStreamWarps;  // units of a wave in which every sequence is alive
    cudaLaunchConfig_t c1 = {};
    c1.gridDim = dim3(static_cast<unsigned>(want < ctas ? want : ctas), 1, 1);
    c1.blockDim = dim3(kStreamThreads, 1, 1);
    c1.stream = stream;
    c1.attrs = pdl;
    c1.numAttrs = 1;
    e = cudaLaunchKernelEx(&c1, ee_stream_kernel<T, VEC, kSample>, sp);
    if (e != cudaSuccess) return DSPARK_ERR_CUDA;

    EeDecideParams dp{};
    dp.rs = c.rs;
    dp.drafts = c.drafts;
    dp.uniforms = c.uniforms;
    dp.nch = pl.nch;
    dp.scale = c.scale;
    dp.rec = sp.rec;
    dp.gather = sp.gather;
    dp.out = c.out;
    dp.wv = wa;
    dp.dec = dec;
    cudaLaunchConfig_t c2 = {};
    c2.gridDim = dim3(static_cast<unsigned>(c.B), 1, 1);
    c2.blockDim = dim3(kThreads, 1, 1);
    c2.stream = stream;
    c2.attrs = pdl;
    c2.numAttrs = 1;
    e = cudaLaunchKernelEx(&c2, ee_decide_kernel<kSample>, dp);
    if (e != cudaSuccess) return DSPARK_ERR_CUDA;
  }
  if constexpr (!kSample) {
    return DSPARK_OK;
  } else {
    FinishParamsEarlyExit fp{};
    fp.rs = c.rs;
    fp.drafts = c.drafts;
    fp.uniforms = c.uniforms;
    fp.nch = pl.nch;
    fp.scale = c.scale;
    fp.rec = reinterpret_cast<float2*>(c.ws + w.rec);
    fp.gather = reinterpret_cast<float*>(c.ws + w.gather);
    fp.out = c.out;
    fp.dec = dec;
    return launch_finish_sample<T, VEC, kFinEarlyExit>(fp, pl, c.B, stream);
  }
}

bool out_ok(const dspark_accept_out_t& o) { return o.n_accepted && o.tokens && o.next_token; }

dspark_status_t check_common(const void* p1, int64_t ld_p1, const void* pv, int64_t ld_pv,
                             dspark_dtype_t dtype, const int32_t* drafts, int B, int K, int V,
                             const dspark_accept_out_t& out) {
  if (dtype != DSPARK_BF16 && dtype != DSPARK_F32) return DSPARK_ERR_INVALID_ARG;
  if (!shape_ok(B, K, V)) return DSPARK_ERR_INVALID_ARG;
  if (B == 0) return DSPARK_OK;
  if (!p1 || !out_ok(out)) return DSPARK_ERR_INVALID_ARG;
  if (K > 0 && (!pv || !drafts)) return DSPARK_ERR_INVALID_ARG;
  if (ld_p1 < V || (K > 0 && ld_pv < static_cast<int64_t>(K) * V)) return DSPARK_ERR_INVALID_ARG;
  const size_t es = static_cast<size_t>(elem_bytes(dtype));
  if (!aligned(p1, es) || (K > 0 && !aligned(pv, es))) return DSPARK_ERR_UNSUPPORTED;
  if (V > kMaxChunkCount * kCE) return DSPARK_ERR_UNSUPPORTED;
  if (ld_p1 > INT32_MAX || ld_pv > INT32_MAX) return DSPARK_ERR_UNSUPPORTED;  // 32-bit strides
  return DSPARK_OK;
}

Call make_call(const void* p1, int64_t ld_p1, const void* pv, int64_t ld_pv, const void* q,
               const int32_t* drafts, const float* uniforms, int B, int K, int V, float scale,
               int rows, void* workspace, const dspark_accept_out_t& out) {
  Call c{};
  c.rs.p1 = p1;
  c.rs.pv = pv;
  c.rs.q = q;
  c.rs.ld_p1 = static_cast<int32_t>(ld_p1);
  c.rs.ld_pv = static_cast<int32_t>(ld_pv);
  c.rs.K = K;
  c.rs.V = V;
  c.rs.rows = rows;
  c.B = B;
  c.drafts = drafts;
  c.uniforms = uniforms;
  c.scale = scale;
  c.out = out;
  c.ws = static_cast<char*>(workspace);
  return c;
}

// ----------------------------------------------------- fixed scratch, no allocation
// Scratch of dspark_speculative_sample_accept_static. Some callers cannot allocate device
// memory where they verify: a serving loop that gave every free byte of HBM to its KV-cache
// pool at start-up has no allocator left to draw a workspace from, and a host runtime in
// another language may hold no device allocator at all. For them the library keeps one
// fixed array per device, part of its own module image, so a call allocates nothing.
// Every call on a device uses the same array: calls that overlap on the GPU race on it.
static __device__ __align__(256) unsigned char g_static_scratch[DSPARK_STATIC_SCRATCH_BYTES];

std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of the fixed scratch on the current device, looked up once per device
// (cudaGetSymbolAddress, with that device current) and cached.
dspark_status_t static_scratch_address(void** addr) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return DSPARK_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return DSPARK_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (!g_scratch_addr[dev]) {
    void* a = nullptr;
    if (cudaGetSymbolAddress(&a, g_static_scratch) != cudaSuccess || !a) return DSPARK_ERR_CUDA;
    g_scratch_addr[dev] = a;
  }
  *addr = g_scratch_addr[dev];
  return DSPARK_OK;
}

// The Markov-head mat-vec for one state on the CUDA cores.
dspark_status_t markov_launch(const void* table, dspark_table_t type, int V, const float* h,
                              float* y, cudaStream_t stream) {
  const bool q8 = type == DSPARK_TABLE_Q8_0;
  const void* fn = q8 ? reinterpret_cast<const void*>(&markov_q8_0_kernel)
                      : reinterpret_cast<const void*>(&markov_f16_kernel);
  cudaError_t e = cudaSuccess;
  const int ctas = resident_ctas(fn, kMarkovThreads, 0, &e);
  if (e != cudaSuccess) return DSPARK_ERR_CUDA;
  if (ctas < 1) return DSPARK_ERR_UNSUPPORTED;
  const long long rows_per_cta = (kMarkovThreads / 32) * (q8 ? kQ8Rows : 8);
  const long long want = (V + rows_per_cta - 1) / rows_per_cta;
  const int grid = static_cast<int>(want < ctas ? want : ctas);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
  cfg.blockDim = dim3(kMarkovThreads, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (q8) {
    e = cudaLaunchKernelEx(&cfg, markov_q8_0_kernel, static_cast<const uint8_t*>(table), V, h,
                           y);
  } else {
    e = cudaLaunchKernelEx(&cfg, markov_f16_kernel, static_cast<const uint16_t*>(table), V, h,
                           y);
  }
  return e == cudaSuccess ? DSPARK_OK : DSPARK_ERR_CUDA;
}

// Q8_0 routing by the number of states (measured on a 129280-row table): one state on the
// CUDA-core kernel (8.0 us; the integer tensor-core kernel takes 10.0), 2 to kI8MaxStates (10)
// on the integer tensor cores (four states: 10.5 us against 15.3 on the CUDA cores), more on
// the float16 tensor-core kernel, 64 states per launch.
constexpr int kMarkovCudaCoreStates = 1;

// The Q8_0 mat-vec on the tensor cores for nb <= N states (N = 16, 32, 48 or 64): one CTA per
// SM over the 128-row tiles.
template <int N>
dspark_status_t markov_mma_launch(const void* table, int V, const float* h, int nb, float* y,
                                  int ldy, cudaStream_t stream, int withhold) {
  const void* fn = reinterpret_cast<const void*>(&markov_q8_0_mma_kernel<N>);
  const size_t smem = static_cast<size_t>(mma_q8_smem(N).total);
  cudaError_t e = cudaSuccess;
  const int ctas = resident_ctas(fn, kMmaThreads, smem, &e);
  if (e != cudaSuccess) return DSPARK_ERR_CUDA;
  if (ctas < 1) return DSPARK_ERR_UNSUPPORTED;
  const int n_tiles = (V + kMmaRows - 1) / kMmaRows;
  const int grid = n_tiles < ctas ? n_tiles : ctas;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
  cfg.blockDim = dim3(kMmaThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, markov_q8_0_mma_kernel<N>, static_cast<const uint8_t*>(table), V,
                         h, nb, y, ldy, withhold);
  return e == cudaSuccess ? DSPARK_OK : DSPARK_ERR_CUDA;
}

// cuTensorMapEncodeTiled from the driver, looked up once through the runtime (the library
// links no driver library of its own).
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn tensor_map_encoder() {
  static EncodeTiledFn fn = nullptr;
  static bool looked = false;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!looked) {
    looked = true;
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// Batches of up to this many states take the CUDA-core F16 kernel; larger ones the
// tensor-core kernel, 64 states per launch.
constexpr int kMarkovF16CudaCoreStates = 1;

// The F16 mat-vec on the tensor cores for nb <= N states: a tensor map over the V x 256 table
// (boxes of 128 rows x 64 halves, 128-byte swizzle, rows past V read as zeros).
template <int N>
dspark_status_t markov_f16_mma_launch(const void* table, int V, const float* h, int nb, float* y,
                                      int ldy, cudaStream_t stream, int withhold) {
  const EncodeTiledFn enc = tensor_map_encoder();
  if (!enc) return DSPARK_ERR_UNSUPPORTED;
  alignas(64) CUtensorMap map;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(kMarkovRank), static_cast<cuuint64_t>(V)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(kMarkovRank) * 2};
  const cuuint32_t box[2] = {64, kMmaRows};
  const cuuint32_t es[2] = {1, 1};
  if (enc(&map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(table), dims, strides, box,
          es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return DSPARK_ERR_UNSUPPORTED;
  const void* fn = reinterpret_cast<const void*>(&markov_f16_mma_kernel<N>);
  const size_t smem = static_cast<size_t>(f16_mma_smem(N));
  cudaError_t e = cudaSuccess;
  const int ctas = resident_ctas(fn, kF16MmaThreads, smem, &e);
  if (e != cudaSuccess) return DSPARK_ERR_CUDA;
  if (ctas < 1) return DSPARK_ERR_UNSUPPORTED;
  const int n_tiles = (V + kMmaRows - 1) / kMmaRows;
  const int grid = n_tiles < ctas ? n_tiles : ctas;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
  cfg.blockDim = dim3(kF16MmaThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, markov_f16_mma_kernel<N>, map, V, h, nb, y, ldy, withhold);
  return e == cudaSuccess ? DSPARK_OK : DSPARK_ERR_CUDA;
}

// The Q8_0 mat-vec on the integer tensor cores for NB <= kI8MaxStates states: a tensor map
// over the V x 272-byte table (boxes of 128 rows x 128 bytes, 128-byte swizzle, bytes past the
// row and rows past V read as zeros).
template <int NB>
dspark_status_t markov_i8_launch(const void* table, int V, const float* h, float* y, int ldy,
                                 cudaStream_t stream, int withhold) {
  const EncodeTiledFn enc = tensor_map_encoder();
  if (!enc) return DSPARK_ERR_UNSUPPORTED;
  alignas(64) CUtensorMap map;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(kQ8RowBytes), static_cast<cuuint64_t>(V)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(kQ8RowBytes)};
  const cuuint32_t box[2] = {128, kMmaRows};
  const cuuint32_t es[2] = {1, 1};
  if (enc(&map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(table), dims, strides, box,
          es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return DSPARK_ERR_UNSUPPORTED;
  const void* fn = reinterpret_cast<const void*>(&markov_q8_0_i8_kernel<NB>);
  const size_t smem = static_cast<size_t>(i8_mma_smem(NB));
  cudaError_t e = cudaSuccess;
  const int ctas = resident_ctas(fn, kI8Threads, smem, &e);
  if (e != cudaSuccess) return DSPARK_ERR_CUDA;
  if (ctas < 1) return DSPARK_ERR_UNSUPPORTED;
  const int n_tiles = (V + kMmaRows - 1) / kMmaRows;
  const int grid = n_tiles < ctas ? n_tiles : ctas;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
  cfg.blockDim = dim3(kI8Threads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, markov_q8_0_i8_kernel<NB>, map, V, h, y, ldy, withhold);
  return e == cudaSuccess ? DSPARK_OK : DSPARK_ERR_CUDA;
}

}  // namespace
}  // namespace dspark

using namespace dspark;

namespace dspark {
namespace {
// The Markov mat-vec dispatch; withhold != 0 (tests of the timeout path) is only accepted
// where the call takes a pipelined tensor-core kernel.
dspark_status_t markov_matvec_impl(const void* table, dspark_table_t type, int V, int R,
                                   const float* h, int B, float* y, void* stream, int withhold) {
  if (type != DSPARK_TABLE_F16 && type != DSPARK_TABLE_Q8_0) return DSPARK_ERR_INVALID_ARG;
  if (V < 0 || R < 1 || B < 0) return DSPARK_ERR_INVALID_ARG;
  if (V == 0 || B == 0) return DSPARK_OK;
  if (!table || !h || !y) return DSPARK_ERR_INVALID_ARG;
  if (R != kMarkovRank) return DSPARK_ERR_UNSUPPORTED;
  if (!aligned(table, 16) || !aligned(h, 16) || !aligned(y, 4)) return DSPARK_ERR_UNSUPPORTED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (withhold && ((type == DSPARK_TABLE_Q8_0 && B <= kMarkovCudaCoreStates) ||
                   (type == DSPARK_TABLE_F16 && B <= kMarkovF16CudaCoreStates)))
    return DSPARK_ERR_UNSUPPORTED;
  if (type == DSPARK_TABLE_Q8_0 && B > kMarkovCudaCoreStates && B <= kI8MaxStates) {
    switch (B) {
      case 2: return markov_i8_launch<2>(table, V, h, y, V, s, withhold);
      case 3: return markov_i8_launch<3>(table, V, h, y, V, s, withhold);
      case 4: return markov_i8_launch<4>(table, V, h, y, V, s, withhold);
      case 5: return markov_i8_launch<5>(table, V, h, y, V, s, withhold);
      case 6: return markov_i8_launch<6>(table, V, h, y, V, s, withhold);
      case 7: return markov_i8_launch<7>(table, V, h, y, V, s, withhold);
      case 8: return markov_i8_launch<8>(table, V, h, y, V, s, withhold);
      case 9: return markov_i8_launch<9>(table, V, h, y, V, s, withhold);
      default: return markov_i8_launch<10>(table, V, h, y, V, s, withhold);
    }
  }
  if (type == DSPARK_TABLE_Q8_0 && B > kMarkovCudaCoreStates) {
    for (int b0 = 0; b0 < B; b0 += kMmaMaxStates) {
      const int nb = B - b0 < kMmaMaxStates ? B - b0 : kMmaMaxStates;
      const float* hb = h + static_cast<size_t>(b0) * R;
      float* yb = y + static_cast<size_t>(b0) * V;
      dspark_status_t st;
      if (nb <= 16)
        st = markov_mma_launch<16>(table, V, hb, nb, yb, V, s, withhold);
      else if (nb <= 32)
        st = markov_mma_launch<32>(table, V, hb, nb, yb, V, s, withhold);
      else if (nb <= 48)
        st = markov_mma_launch<48>(table, V, hb, nb, yb, V, s, withhold);
      else
        st = markov_mma_launch<64>(table, V, hb, nb, yb, V, s, withhold);
      if (st != DSPARK_OK) return st;
    }
    return DSPARK_OK;
  }
  if (type == DSPARK_TABLE_F16 && B > kMarkovF16CudaCoreStates) {
    for (int b0 = 0; b0 < B; b0 += kMmaMaxStates) {
      const int nb = B - b0 < kMmaMaxStates ? B - b0 : kMmaMaxStates;
      const float* hb = h + static_cast<size_t>(b0) * R;
      float* yb = y + static_cast<size_t>(b0) * V;
      dspark_status_t st;
      if (nb <= 16)
        st = markov_f16_mma_launch<16>(table, V, hb, nb, yb, V, s, withhold);
      else if (nb <= 32)
        st = markov_f16_mma_launch<32>(table, V, hb, nb, yb, V, s, withhold);
      else if (nb <= 48)
        st = markov_f16_mma_launch<48>(table, V, hb, nb, yb, V, s, withhold);
      else
        st = markov_f16_mma_launch<64>(table, V, hb, nb, yb, V, s, withhold);
      if (st != DSPARK_OK) return st;
    }
    return DSPARK_OK;
  }
  // one state (B == 1 here)
  return markov_launch(table, type, V, h, y, s);
}
}  // namespace
}  // namespace dspark

extern "C" {

const char* dspark_status_string(int status) {
  switch (status) {
    case DSPARK_OK: return "DSPARK_OK";
    case DSPARK_ERR_INVALID_ARG: return "DSPARK_ERR_INVALID_ARG";
    case DSPARK_ERR_UNSUPPORTED: return "DSPARK_ERR_UNSUPPORTED";
    case DSPARK_ERR_CUDA: return "DSPARK_ERR_CUDA";
    case DSPARK_ERR_WORKSPACE: return "DSPARK_ERR_WORKSPACE";
    default: return "DSPARK_ERR_UNKNOWN";
  }
}

int dspark_version(void) { return kAbiVersion; }

size_t dspark_workspace_bytes(int B, int K, int V, dspark_dtype_t dtype) {
  if (dtype != DSPARK_BF16 && dtype != DSPARK_F32) return 0;
  if (!shape_ok(B, K, V)) return 0;
  Plan pl;
  if (!make_plan(B, V, dtype, false, &pl)) return 0;
  return ws_layout(B, K, pl.nch).total;
}

size_t dspark_workspace_zero_bytes(int B, int K) {
  (void)B;
  (void)K;
  return 0;  // no part of the workspace needs initialisation
}

dspark_status_t dspark_plan(int B, int K, int V, dspark_dtype_t dtype, int aligned16,
                            dspark_plan_t* plan) {
  if (!plan || (dtype != DSPARK_BF16 && dtype != DSPARK_F32) || !shape_ok(B, K, V))
    return DSPARK_ERR_INVALID_ARG;
  Plan pl;
  if (!make_plan(B, V, dtype, aligned16 != 0, &pl)) return DSPARK_ERR_UNSUPPORTED;
  plan->elems_per_load = pl.vec;
  plan->loads_in_flight = kBatchVecs;
  plan->stream_threads_per_cta = kStreamThreads;
  plan->threads_per_cta = kThreads;
  plan->chunk_elems = kCE;
  plan->n_chunks = pl.nch;
  plan->greedy_units_per_sequence = (K + 1) * pl.nch;
  plan->sampling_units_per_sequence = (2 * K + 1) * pl.nch;
  plan->finish_ctas_per_sequence = pl.G;
  plan->finish_threads_per_cta = pl.fw * 32;
  return DSPARK_OK;
}

dspark_status_t dspark_greedy_accept(const void* p1, int64_t ld_p1, const void* pv, int64_t ld_pv,
                                     dspark_dtype_t dtype, const int32_t* drafts, int B, int K,
                                     int V, dspark_accept_out_t out, void* workspace,
                                     size_t workspace_bytes, void* stream) {
  dspark_status_t st = check_common(p1, ld_p1, pv, ld_pv, dtype, drafts, B, K, V, out);
  if (st != DSPARK_OK || B == 0) return st;
  const size_t es = static_cast<size_t>(elem_bytes(dtype));
  const bool a16 = aligned(p1, 16) && (K == 0 || aligned(pv, 16)) && (ld_p1 * es) % 16 == 0 &&
                   (K == 0 || (ld_pv * es) % 16 == 0) && (V * es) % 16 == 0;
  Plan pl;
  if (!make_plan(B, V, dtype, a16, &pl)) return DSPARK_ERR_UNSUPPORTED;
  if (!workspace || workspace_bytes < ws_layout(B, K, pl.nch).total || !aligned(workspace, 256))
    return DSPARK_ERR_WORKSPACE;
  const Call c = make_call(p1, ld_p1, pv, ld_pv, nullptr, drafts, nullptr, B, K, V, 0.f, K + 1,
                           workspace, out);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (dtype == DSPARK_BF16)
    return a16 ? run_call<bf16_t, 8, kModeGreedy>(c, pl, s)
               : run_call<bf16_t, 1, kModeGreedy>(c, pl, s);
  return a16 ? run_call<float, 4, kModeGreedy>(c, pl, s) : run_call<float, 1, kModeGreedy>(c, pl, s);
}

dspark_status_t dspark_speculative_sample_accept(const void* p1, int64_t ld_p1, const void* pv,
                                                 int64_t ld_pv, const void* q,
                                                 dspark_dtype_t dtype, const int32_t* drafts,
                                                 int B, int K, int V, float temperature,
                                                 const float* uniforms, dspark_accept_out_t out,
                                                 void* workspace, size_t workspace_bytes,
                                                 void* stream) {
  if (!(temperature >= 0.f) || !std::isfinite(temperature)) return DSPARK_ERR_INVALID_ARG;
  if (temperature == 0.f)
    return dspark_greedy_accept(p1, ld_p1, pv, ld_pv, dtype, drafts, B, K, V, out, workspace,
                                workspace_bytes, stream);
  dspark_status_t st = check_common(p1, ld_p1, pv, ld_pv, dtype, drafts, B, K, V, out);
  if (st != DSPARK_OK || B == 0) return st;
  if (!uniforms || (K > 0 && !q)) return DSPARK_ERR_INVALID_ARG;
  const size_t es = static_cast<size_t>(elem_bytes(dtype));
  if (K > 0 && !aligned(q, es)) return DSPARK_ERR_UNSUPPORTED;
  const bool a16 = aligned(p1, 16) && (K == 0 || (aligned(pv, 16) && aligned(q, 16))) &&
                   (ld_p1 * es) % 16 == 0 && (K == 0 || (ld_pv * es) % 16 == 0) &&
                   (V * es) % 16 == 0;
  Plan pl;
  if (!make_plan(B, V, dtype, a16, &pl)) return DSPARK_ERR_UNSUPPORTED;
  if (!workspace || workspace_bytes < ws_layout(B, K, pl.nch).total || !aligned(workspace, 256))
    return DSPARK_ERR_WORKSPACE;
  const float scale = static_cast<float>(1.4426950408889634 / static_cast<double>(temperature));
  if (!std::isfinite(scale)) return DSPARK_ERR_INVALID_ARG;
  const Call c = make_call(p1, ld_p1, pv, ld_pv, q, drafts, uniforms, B, K, V, scale, 2 * K + 1,
                           workspace, out);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (dtype == DSPARK_BF16)
    return a16 ? run_call<bf16_t, 8, kModeSample>(c, pl, s)
               : run_call<bf16_t, 1, kModeSample>(c, pl, s);
  return a16 ? run_call<float, 4, kModeSample>(c, pl, s) : run_call<float, 1, kModeSample>(c, pl, s);
}

dspark_status_t dspark_sample_pass1(const void* p1, int64_t ld_p1, const void* pv, int64_t ld_pv,
                                   const void* q, dspark_dtype_t dtype, const int32_t* drafts,
                                   int B, int K, int V, float temperature, void* workspace,
                                   size_t workspace_bytes, void* stream) {
  if (!(temperature > 0.f) || !std::isfinite(temperature)) return DSPARK_ERR_INVALID_ARG;
  if (dtype != DSPARK_BF16 && dtype != DSPARK_F32) return DSPARK_ERR_INVALID_ARG;
  if (!shape_ok(B, K, V)) return DSPARK_ERR_INVALID_ARG;
  if (B == 0) return DSPARK_OK;
  if (!p1 || (K > 0 && (!pv || !drafts || !q))) return DSPARK_ERR_INVALID_ARG;
  if (ld_p1 < V || (K > 0 && ld_pv < static_cast<int64_t>(K) * V)) return DSPARK_ERR_INVALID_ARG;
  const size_t es = static_cast<size_t>(elem_bytes(dtype));
  if (!aligned(p1, es) || (K > 0 && (!aligned(pv, es) || !aligned(q, es))))
    return DSPARK_ERR_UNSUPPORTED;
  if (V > kMaxChunkCount * kCE || ld_p1 > INT32_MAX || ld_pv > INT32_MAX)
    return DSPARK_ERR_UNSUPPORTED;
  const bool a16 = aligned(p1, 16) && (K == 0 || (aligned(pv, 16) && aligned(q, 16))) &&
                   (ld_p1 * es) % 16 == 0 && (K == 0 || (ld_pv * es) % 16 == 0) &&
                   (V * es) % 16 == 0;
  Plan pl;
  if (!make_plan(B, V, dtype, a16, &pl)) return DSPARK_ERR_UNSUPPORTED;
  if (!workspace || workspace_bytes < ws_layout(B, K, pl.nch).total || !aligned(workspace, 256))
    return DSPARK_ERR_WORKSPACE;
  const float scale = static_cast<float>(1.4426950408889634 / static_cast<double>(temperature));
  if (!std::isfinite(scale)) return DSPARK_ERR_INVALID_ARG;
  const Call c = make_call(p1, ld_p1, pv, ld_pv, q, drafts, nullptr, B, K, V, scale, 2 * K + 1,
                           workspace, dspark_accept_out_t{});
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (dtype == DSPARK_BF16)
    return a16 ? run_call<bf16_t, 8, kModeSample>(c, pl, s, true)
               : run_call<bf16_t, 1, kModeSample>(c, pl, s, true);
  return a16 ? run_call<float, 4, kModeSample>(c, pl, s, true)
             : run_call<float, 1, kModeSample>(c, pl, s, true);
}

dspark_status_t dspark_mixed_accept(const void* p1, int64_t ld_p1, const void* pv, int64_t ld_pv,
                                    const void* q, dspark_dtype_t dtype, const int32_t* drafts,
                                    const int32_t* n_drafts, int B, int K, int V,
                                    const float* temperatures, const float* uniforms,
                                    dspark_accept_out_t out, void* workspace,
                                    size_t workspace_bytes, void* stream) {
  dspark_status_t st = check_common(p1, ld_p1, pv, ld_pv, dtype, drafts, B, K, V, out);
  if (st != DSPARK_OK || B == 0) return st;
  if (!temperatures || !uniforms || (K > 0 && !q)) return DSPARK_ERR_INVALID_ARG;
  const size_t es = static_cast<size_t>(elem_bytes(dtype));
  if (K > 0 && !aligned(q, es)) return DSPARK_ERR_UNSUPPORTED;
  const bool a16 = aligned(p1, 16) && (K == 0 || (aligned(pv, 16) && aligned(q, 16))) &&
                   (ld_p1 * es) % 16 == 0 && (K == 0 || (ld_pv * es) % 16 == 0) &&
                   (V * es) % 16 == 0;
  Plan pl;
  if (!make_plan(B, V, dtype, a16, &pl)) return DSPARK_ERR_UNSUPPORTED;
  if (!workspace || workspace_bytes < ws_layout(B, K, pl.nch).total || !aligned(workspace, 256))
    return DSPARK_ERR_WORKSPACE;
  Call c = make_call(p1, ld_p1, pv, ld_pv, q, drafts, uniforms, B, K, V, 0.f, 2 * K + 1,
                     workspace, out);
  c.n_drafts = n_drafts;
  c.temps = temperatures;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (dtype == DSPARK_BF16)
    return a16 ? run_call<bf16_t, 8, kModeMixed>(c, pl, s)
               : run_call<bf16_t, 1, kModeMixed>(c, pl, s);
  return a16 ? run_call<float, 4, kModeMixed>(c, pl, s) : run_call<float, 1, kModeMixed>(c, pl, s);
}

dspark_status_t dspark_early_exit_accept(const void* p1, int64_t ld_p1, const void* pv,
                                        int64_t ld_pv, const void* q, dspark_dtype_t dtype,
                                        const int32_t* drafts, int B, int K, int V,
                                        float temperature, const float* uniforms,
                                        dspark_accept_out_t out, void* workspace,
                                        size_t workspace_bytes, void* stream) {
  if (!(temperature >= 0.f) || !std::isfinite(temperature)) return DSPARK_ERR_INVALID_ARG;
  dspark_status_t st = check_common(p1, ld_p1, pv, ld_pv, dtype, drafts, B, K, V, out);
  if (st != DSPARK_OK || B == 0) return st;
  const bool sample = temperature > 0.f;
  const size_t es = static_cast<size_t>(elem_bytes(dtype));
  if (sample) {
    if (!uniforms || (K > 0 && !q)) return DSPARK_ERR_INVALID_ARG;
    if (K > 0 && !aligned(q, es)) return DSPARK_ERR_UNSUPPORTED;
  }
  const bool a16 = aligned(p1, 16) && (K == 0 || (aligned(pv, 16) && (!sample || aligned(q, 16)))) &&
                   (ld_p1 * es) % 16 == 0 && (K == 0 || (ld_pv * es) % 16 == 0) &&
                   (V * es) % 16 == 0;
  Plan pl;
  if (!make_plan(B, V, dtype, a16, &pl)) return DSPARK_ERR_UNSUPPORTED;
  if (!workspace || workspace_bytes < ws_layout(B, K, pl.nch).total || !aligned(workspace, 256))
    return DSPARK_ERR_WORKSPACE;
  float scale = 0.f;
  if (sample) {
    scale = static_cast<float>(1.4426950408889634 / static_cast<double>(temperature));
    if (!std::isfinite(scale)) return DSPARK_ERR_INVALID_ARG;
  }
  // the record layout of a full call: 2K+1 rows per sequence when sampling, K+1 for greedy
  const Call c = make_call(p1, ld_p1, pv, ld_pv, sample ? q : nullptr, drafts,
                           sample ? uniforms : nullptr, B, K, V, scale,
                           sample ? 2 * K + 1 : K + 1, workspace, out);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (dtype == DSPARK_BF16) {
    if (sample)
      return a16 ? run_early_exit<bf16_t, 8, true>(c, pl, s) : run_early_exit<bf16_t, 1, true>(c, pl, s);
    return a16 ? run_early_exit<bf16_t, 8, false>(c, pl, s) : run_early_exit<bf16_t, 1, false>(c, pl, s);
  }
  if (sample)
    return a16 ? run_early_exit<float, 4, true>(c, pl, s) : run_early_exit<float, 1, true>(c, pl, s);
  return a16 ? run_early_exit<float, 4, false>(c, pl, s) : run_early_exit<float, 1, false>(c, pl, s);
}

dspark_status_t dspark_markov_matvec(const void* table, dspark_table_t type, int V, int R,
                                     const float* h, int B, float* y, void* stream) {
  return markov_matvec_impl(table, type, V, R, h, B, y, stream, 0);
}

dspark_status_t dspark_markov_matvec_withheld(const void* table, dspark_table_t type, int V,
                                              int R, const float* h, int B, float* y,
                                              void* stream) {
  return markov_matvec_impl(table, type, V, R, h, B, y, stream, 1);
}

dspark_status_t dspark_pipeline_timeouts(unsigned long long* count) {
  if (!count) return DSPARK_ERR_INVALID_ARG;
  return cudaMemcpyFromSymbol(count, g_pipeline_timeouts, sizeof(*count)) == cudaSuccess
             ? DSPARK_OK
             : DSPARK_ERR_CUDA;
}

dspark_status_t dspark_speculative_sample_accept_static(const void* p1, int64_t ld_p1,
                                                        const void* pv, int64_t ld_pv,
                                                        const void* q, dspark_dtype_t dtype,
                                                        const int32_t* drafts, int B, int K, int V,
                                                        float temperature, const float* uniforms,
                                                        dspark_accept_out_t out, void* stream) {
  // every synchronous check first, so that a rejected call enqueues nothing
  if (!(temperature >= 0.f) || !std::isfinite(temperature)) return DSPARK_ERR_INVALID_ARG;
  dspark_status_t st = check_common(p1, ld_p1, pv, ld_pv, dtype, drafts, B, K, V, out);
  if (st != DSPARK_OK || B == 0) return st;
  if (temperature > 0.f) {
    if (!uniforms || (K > 0 && !q)) return DSPARK_ERR_INVALID_ARG;
    if (K > 0 && !aligned(q, static_cast<size_t>(elem_bytes(dtype)))) return DSPARK_ERR_UNSUPPORTED;
  }
  const size_t need = dspark_workspace_bytes(B, K, V, dtype);
  if (need == 0) return DSPARK_ERR_UNSUPPORTED;
  if (need > DSPARK_STATIC_SCRATCH_BYTES) return DSPARK_ERR_WORKSPACE;
  void* scratch = nullptr;
  st = static_scratch_address(&scratch);
  if (st != DSPARK_OK) return st;
  // nothing in the scratch needs clearing: each call writes every word of it that it reads
  return dspark_speculative_sample_accept(p1, ld_p1, pv, ld_pv, q, dtype, drafts, B, K, V,
                                          temperature, uniforms, out, scratch,
                                          DSPARK_STATIC_SCRATCH_BYTES, stream);
}

}  // extern "C"
