// C ABI of the DSpark block verify/accept step: argument checks, launch planning and the
// kernel launch. The device work is the task kernel of tasks.cuh.
#include <cmath>
#include <cstdlib>
#include <mutex>

#include "common.cuh"
#include "tasks.cuh"

namespace dspark {
namespace {

constexpr int kAbiVersion = 2;
constexpr int kMaxDevices = 64;
constexpr size_t kRingBudgetPerCta = 100 * 1024;  // shared memory for one CTA's rings

// ------------------------------------------------------------------------- tuning knobs

struct Tuning {
  int stages = 0;        // 0 = automatic
  bool no_tma = false;   // direct loads instead of the bulk-copy rings
  int max_ctas = 0;      // 0 = as many as fit
};

const Tuning& tuning() {
  static const Tuning t = [] {
    Tuning v;
    if (const char* s = std::getenv("DSPARK_STAGES")) v.stages = std::atoi(s);
    if (const char* s = std::getenv("DSPARK_NO_TMA")) v.no_tma = std::atoi(s) != 0;
    if (const char* s = std::getenv("DSPARK_MAX_CTAS")) v.max_ctas = std::atoi(s);
    if (v.stages < 0 || v.stages > kMaxTaskStages) v.stages = 0;
    if (v.max_ctas < 0) v.max_ctas = 0;
    return v;
  }();
  return t;
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
  int vec;     // elements per load: 16-byte vectors (8 bf16 / 4 fp32) or 1
  int nch;     // 2048-token chunks per row
  int stages;  // ring depth per warp, 0 = direct loads
};

bool make_plan(int V, dspark_dtype_t dt, bool aligned16, Plan* pl) {
  const int es = elem_bytes(dt);
  const long long nch = (static_cast<long long>(V) + kCE - 1) / kCE;
  if (nch < 1 || nch > kMaxChunkCount) return false;
  pl->vec = aligned16 ? 16 / es : 1;
  pl->nch = static_cast<int>(nch);
  pl->stages = 0;
  if (aligned16 && !tuning().no_tma) {
    int st = static_cast<int>(kRingBudgetPerCta / (static_cast<size_t>(kStreamWarps) * kCE * es));
    st = st < 2 ? 2 : (st > kMaxTaskStages ? kMaxTaskStages : st);
    if (tuning().stages) st = tuning().stages;
    pl->stages = st;
  }
  return true;
}

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// Workspace regions. The counters come first: they must be zero before a call, and every
// call leaves them zero again. The rest needs no initialisation.
struct WsLayout {
  size_t dq, seq_cnt, chunk_stat, row_stat, dec, resid, total;
};

WsLayout ws_layout(long long B, long long K, int nch) {
  const long long rows = 2 * K + 1;
  WsLayout w{};
  size_t off = 0;
  w.dq = off;
  off = align256(off + sizeof(DepQueue));
  w.seq_cnt = off;
  off = align256(off + sizeof(SeqCounters) * static_cast<size_t>(B));
  w.chunk_stat = off;
  off = align256(off + sizeof(float2) * static_cast<size_t>(B * rows * nch));
  w.row_stat = off;
  off = align256(off + sizeof(float2) * static_cast<size_t>(B * rows));
  w.dec = off;
  off = align256(off + sizeof(SeqDecision) * static_cast<size_t>(B));
  w.resid = off;
  off = align256(off + sizeof(float) * static_cast<size_t>(B * nch));
  w.total = off;
  return w;
}

// --------------------------------------------------------------- per-device launch state

std::mutex g_mu;
struct OccEntry {
  void* fn;
  int dev;
  size_t smem;
  int ctas;  // co-resident CTAs on the device
};
OccEntry g_occ[64];
int g_occ_n = 0;
bool g_attr_done[kMaxDevices][16] = {};

// CTAs of the task kernel that fit on the device at once (the schedule needs them all
// resident); 0 if it cannot launch.
int resident_ctas(void* fn, int fn_id, size_t smem, cudaError_t* err) {
  int dev = 0;
  *err = cudaGetDevice(&dev);
  if (*err != cudaSuccess) return 0;
  std::lock_guard<std::mutex> lk(g_mu);
  for (int n = 0; n < g_occ_n; ++n)
    if (g_occ[n].fn == fn && g_occ[n].dev == dev && g_occ[n].smem == smem) return g_occ[n].ctas;
  if (dev < kMaxDevices && !g_attr_done[dev][fn_id]) {
    // allow the largest dynamic shared memory the device takes next to the static part
    int optin = 0;
    *err = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    if (*err != cudaSuccess) return 0;
    cudaFuncAttributes fa;
    *err = cudaFuncGetAttributes(&fa, fn);
    if (*err != cudaSuccess) return 0;
    if (smem + fa.sharedSizeBytes > static_cast<size_t>(optin)) return 0;
    *err = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                optin - static_cast<int>(fa.sharedSizeBytes));
    if (*err != cudaSuccess) return 0;
    g_attr_done[dev][fn_id] = true;
  }
  int per_sm = 0, sms = 0;
  *err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, kTaskThreads, smem);
  if (*err != cudaSuccess) return 0;
  *err = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (*err != cudaSuccess) return 0;
  const int n = per_sm * sms;
  if (g_occ_n < 64) g_occ[g_occ_n++] = OccEntry{fn, dev, smem, n};
  return n;
}

template <typename T, int VEC, bool kSample, bool kTma>
dspark_status_t run_tasks(TaskParams prm, const Plan& pl, int fn_id, cudaStream_t stream) {
  const size_t smem =
      kTma ? static_cast<size_t>(kStreamWarps) * pl.stages * kCE * Elem<T>::kBytes +
                 static_cast<size_t>(kStreamWarps) * kMaxTaskStages * sizeof(uint64_t)
           : 0;
  void* fn = reinterpret_cast<void*>(&verify_tasks_kernel<T, VEC, kSample, kTma>);
  cudaError_t e = cudaSuccess;
  int ctas = resident_ctas(fn, fn_id, smem, &e);
  if (e != cudaSuccess) return DSPARK_ERR_CUDA;
  if (ctas < 1) return DSPARK_ERR_UNSUPPORTED;
  if (tuning().max_ctas) ctas = ctas < tuning().max_ctas ? ctas : tuning().max_ctas;
  prm.n_stream = static_cast<long long>(prm.B) * prm.rows * prm.nch;
  prm.n_resid = (prm.nch + kResidGroup - 1) / kResidGroup;
  prm.n_dep_per_seq = kSample ? prm.n_resid + 2 : 1;
  // no more CTAs than there is streaming work for
  const long long want = (prm.n_stream + kStreamWarps - 1) / kStreamWarps;
  if (want < ctas) ctas = static_cast<int>(want < 1 ? 1 : want);
  prm.stages = pl.stages;
  prm.stream_warps = ctas * kStreamWarps;
  prm.dep_warps = ctas;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(ctas), 1, 1);
  cfg.blockDim = dim3(kTaskThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cfg.numAttrs = 0;
  e = cudaLaunchKernelEx(&cfg, verify_tasks_kernel<T, VEC, kSample, kTma>, prm);
  return e == cudaSuccess ? DSPARK_OK : DSPARK_ERR_CUDA;
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
  return DSPARK_OK;
}

TaskParams base_params(const void* p1, int64_t ld_p1, const void* pv, int64_t ld_pv, const void* q,
                       const int32_t* drafts, const float* uniforms, int B, int K, int V,
                       float scale, int rows, const Plan& pl, void* workspace,
                       const dspark_accept_out_t& out) {
  const WsLayout w = ws_layout(B, K, pl.nch);
  char* ws = static_cast<char*>(workspace);
  TaskParams prm{};
  prm.p1 = p1;
  prm.pv = pv;
  prm.q = q;
  prm.ld_p1 = ld_p1;
  prm.ld_pv = ld_pv;
  prm.B = B;
  prm.K = K;
  prm.V = V;
  prm.scale = scale;
  prm.drafts = drafts;
  prm.uniforms = uniforms;
  prm.nch = pl.nch;
  prm.rows = rows;
  prm.chunk_stat = reinterpret_cast<float2*>(ws + w.chunk_stat);
  prm.row_stat = reinterpret_cast<float2*>(ws + w.row_stat);
  prm.seq_cnt = reinterpret_cast<SeqCounters*>(ws + w.seq_cnt);
  prm.dq = reinterpret_cast<DepQueue*>(ws + w.dq);
  prm.dec = reinterpret_cast<SeqDecision*>(ws + w.dec);
  prm.resid_mass = reinterpret_cast<float*>(ws + w.resid);
  prm.out = out;
  return prm;
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

}  // namespace
}  // namespace dspark

using namespace dspark;

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
  if (!make_plan(V, dtype, false, &pl)) return 0;
  return ws_layout(B, K, pl.nch).total;
}

size_t dspark_workspace_zero_bytes(int B, int K) {
  if (!shape_ok(B, K, 1)) return 0;
  Plan pl{1, 1, 0};
  return ws_layout(B, K, pl.nch).chunk_stat;
}

dspark_status_t dspark_plan(int B, int K, int V, dspark_dtype_t dtype, int aligned16,
                            dspark_plan_t* plan) {
  if (!plan || (dtype != DSPARK_BF16 && dtype != DSPARK_F32) || !shape_ok(B, K, V))
    return DSPARK_ERR_INVALID_ARG;
  Plan pl;
  if (!make_plan(V, dtype, aligned16 != 0, &pl)) return DSPARK_ERR_UNSUPPORTED;
  plan->elems_per_load = pl.vec;
  plan->chunk_elems = kCE;
  plan->n_chunks = pl.nch;
  plan->threads_per_cta = kTaskThreads;
  plan->stages = pl.stages;
  plan->sampling_tasks_per_sequence =
      (2 * K + 1) * pl.nch + (pl.nch + kResidGroup - 1) / kResidGroup + 2;
  plan->greedy_tasks_per_sequence = (K + 1) * pl.nch + 1;
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
  if (!make_plan(V, dtype, a16, &pl)) return DSPARK_ERR_UNSUPPORTED;
  if (!workspace || workspace_bytes < ws_layout(B, K, pl.nch).total || !aligned(workspace, 256))
    return DSPARK_ERR_WORKSPACE;
  TaskParams prm = base_params(p1, ld_p1, pv, ld_pv, nullptr, drafts, nullptr, B, K, V, 0.f,
                               K + 1, pl, workspace, out);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (dtype == DSPARK_BF16) {
    if (!a16) return run_tasks<bf16_t, 1, false, false>(prm, pl, 0, s);
    if (pl.stages) return run_tasks<bf16_t, 8, false, true>(prm, pl, 1, s);
    return run_tasks<bf16_t, 8, false, false>(prm, pl, 2, s);
  }
  if (!a16) return run_tasks<float, 1, false, false>(prm, pl, 3, s);
  if (pl.stages) return run_tasks<float, 4, false, true>(prm, pl, 4, s);
  return run_tasks<float, 4, false, false>(prm, pl, 5, s);
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
  if (!make_plan(V, dtype, a16, &pl)) return DSPARK_ERR_UNSUPPORTED;
  if (!workspace || workspace_bytes < ws_layout(B, K, pl.nch).total || !aligned(workspace, 256))
    return DSPARK_ERR_WORKSPACE;
  const float scale = static_cast<float>(1.4426950408889634 / static_cast<double>(temperature));
  if (!std::isfinite(scale)) return DSPARK_ERR_INVALID_ARG;
  TaskParams prm = base_params(p1, ld_p1, pv, ld_pv, q, drafts, uniforms, B, K, V, scale,
                               2 * K + 1, pl, workspace, out);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (dtype == DSPARK_BF16) {
    if (!a16) return run_tasks<bf16_t, 1, true, false>(prm, pl, 6, s);
    if (pl.stages) return run_tasks<bf16_t, 8, true, true>(prm, pl, 7, s);
    return run_tasks<bf16_t, 8, true, false>(prm, pl, 8, s);
  }
  if (!a16) return run_tasks<float, 1, true, false>(prm, pl, 9, s);
  if (pl.stages) return run_tasks<float, 4, true, true>(prm, pl, 10, s);
  return run_tasks<float, 4, true, false>(prm, pl, 11, s);
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
  // the counters at the front of the scratch must start at zero
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(scratch, 0, dspark_workspace_zero_bytes(B, K), s) != cudaSuccess)
    return DSPARK_ERR_CUDA;
  return dspark_speculative_sample_accept(p1, ld_p1, pv, ld_pv, q, dtype, drafts, B, K, V,
                                          temperature, uniforms, out, scratch,
                                          DSPARK_STATIC_SCRATCH_BYTES, stream);
}

}  // extern "C"
