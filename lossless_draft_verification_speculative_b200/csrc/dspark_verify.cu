// C ABI of the DSpark block verify/accept step: argument checks, launch planning and the
// kernel launches. All device work is in greedy.cuh and sample_pass.cuh.
#include <cmath>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "common.cuh"
#include "greedy.cuh"
#include "sample_pass.cuh"

namespace dspark {
namespace {

constexpr int kAbiVersion = 1;
constexpr int kMaxDevices = 64;
constexpr size_t kSmemBudgetPerSm = 200 * 1024;  // shared memory we plan to use per SM

// ------------------------------------------------------------------------- tuning knobs

struct Tuning {
  int stages = 0;        // 0 = automatic
  bool no_tma = false;   // direct register loads instead of the bulk-copy ring
  int max_cluster = kMaxCluster;
};

const Tuning& tuning() {
  static const Tuning t = [] {
    Tuning v;
    if (const char* s = std::getenv("DSPARK_STAGES")) v.stages = std::atoi(s);
    if (const char* s = std::getenv("DSPARK_NO_TMA")) v.no_tma = std::atoi(s) != 0;
    if (const char* s = std::getenv("DSPARK_MAX_CLUSTER")) {
      const int c = std::atoi(s);
      if (c == 1 || c == 2 || c == 4 || c == 8 || c == 16) v.max_cluster = c;
    }
    if (v.stages < 0 || v.stages > kMaxStages) v.stages = 0;
    return v;
  }();
  return t;
}

// ------------------------------------------------------------------------------ plans

int elem_bytes(dspark_dtype_t dt) { return dt == DSPARK_F32 ? 4 : 2; }

struct Plan {
  int vec;          // elements per load: 16-byte vectors (8 bf16 / 4 fp32) or 1
  int n_chunks;     // 1024-token chunks per row
  int warps;        // warps per CTA = chunks per CTA
  int cluster;      // CTAs per cluster
  int slice_elems;  // V elements per CTA slice
  int stages;       // bulk-copy ring depth, 0 = direct loads
  int greedy_slices;
};

bool make_plan(int V, dspark_dtype_t dt, bool aligned16, Plan* pl) {
  const int es = elem_bytes(dt);
  const int chunk = 32 * kLaneElems;
  const long long nch = (static_cast<long long>(V) + chunk - 1) / chunk;
  if (nch < 1 || nch > kMaxChunks) return false;
  int cl = 1;
  while (cl < tuning().max_cluster && (nch + cl - 1) / cl > 8) cl *= 2;
  const int warps = static_cast<int>((nch + cl - 1) / cl);
  if (warps > kMaxWarps) return false;
  pl->vec = aligned16 ? 16 / es : 1;
  pl->n_chunks = static_cast<int>(nch);
  pl->warps = warps;
  pl->cluster = cl;
  pl->slice_elems = warps * chunk;
  pl->greedy_slices = (V + kGreedySliceElems - 1) / kGreedySliceElems;
  pl->stages = 0;
  if (aligned16 && !tuning().no_tma) {
    // Aim for two CTAs per SM up to 8 warps, one above; at least 2 and at most 4 stages.
    const size_t stage_bytes = pass1_ring_bytes(warps, 1, es);
    const int ctas_per_sm = warps <= 8 ? 2 : 1;
    int st = static_cast<int>(kSmemBudgetPerSm / ctas_per_sm / stage_bytes);
    st = st < 2 ? 2 : (st > kMaxStages ? kMaxStages : st);
    if (tuning().stages) st = tuning().stages;
    pl->stages = st;
  }
  return true;
}

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// Workspace regions (byte offsets); the same layout serves both policies.
struct WsLayout {
  size_t rowstat, chunk_p, chunk_r, unit_flags, greedy_part, total;
};

WsLayout ws_layout(long long B, long long K, const Plan& pl) {
  WsLayout w{};
  size_t off = 0;
  w.rowstat = off;
  off = align256(off + sizeof(float2) * static_cast<size_t>(B * (K + 1) + B * K));
  w.chunk_p = off;
  off = align256(off + sizeof(ChunkRec) * static_cast<size_t>(B * (K + 1) * pl.n_chunks));
  w.chunk_r = off;
  off = align256(off + sizeof(ChunkRec) * static_cast<size_t>(B * K * pl.n_chunks));
  w.unit_flags = off;
  off = align256(off + static_cast<size_t>(B * (K + 1) * pl.cluster * pl.warps));
  w.greedy_part = off;
  off = align256(off + sizeof(int4) * static_cast<size_t>(B * (K + 1) * pl.greedy_slices));
  w.total = off;
  return w;
}

bool shape_ok(int B, int K, int V) {
  if (B < 0 || K < 0 || K > kMaxK || V < 1) return false;
  if (static_cast<long long>(B) * (K + 1) >= (1LL << 31)) return false;
  return true;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// --------------------------------------------------------------- per-device launch state

template <typename T, int VEC, bool kTma>
struct Pass1Kernel {
  static void* fn() { return reinterpret_cast<void*>(&sample_rowstats_kernel<T, VEC, kTma>); }
};

std::mutex g_mu;

struct OccKey {
  void* fn;
  int dev, threads, cluster;
  size_t smem;
};
struct OccEntry {
  OccKey k;
  int clusters;
};
OccEntry g_occ[256];
int g_occ_n = 0;
bool g_attr_done[kMaxDevices][16] = {};

// Max co-resident clusters of a pass-1 configuration, cached; 0 if it cannot launch.
int max_clusters(void* fn, int fn_id, int threads, size_t smem, int cluster, cudaError_t* err) {
  int dev = 0;
  *err = cudaGetDevice(&dev);
  if (*err != cudaSuccess) return 0;
  std::lock_guard<std::mutex> lk(g_mu);
  for (int n = 0; n < g_occ_n; ++n) {
    const OccKey& k = g_occ[n].k;
    if (k.fn == fn && k.dev == dev && k.threads == threads && k.cluster == cluster && k.smem == smem)
      return g_occ[n].clusters;
  }
  if (dev < kMaxDevices && !g_attr_done[dev][fn_id]) {
    *err = cudaFuncSetAttribute(fn, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (*err != cudaSuccess) return 0;
    *err = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
    if (*err != cudaSuccess) return 0;
    g_attr_done[dev][fn_id] = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(cluster, 1, 1);
  cfg.blockDim = dim3(threads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = cluster;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  *err = cudaOccupancyMaxActiveClusters(&n, fn, &cfg);
  if (*err != cudaSuccess) return 0;
  if (g_occ_n < 256) g_occ[g_occ_n++] = OccEntry{OccKey{fn, dev, threads, cluster, smem}, n};
  return n;
}

template <typename KernelT, typename ParamT>
cudaError_t launch(KernelT kernel, dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                   int cluster, bool pdl, const ParamT& prm) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  int na = 0;
  if (cluster > 0) {
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = cluster;
    attr[na].val.clusterDim.y = 1;
    attr[na].val.clusterDim.z = 1;
    ++na;
  }
  if (pdl) {
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  return cudaLaunchKernelEx(&cfg, kernel, prm);
}

// ------------------------------------------------------------------------------ greedy

template <typename T, int VEC>
dspark_status_t run_greedy(const GreedyParams& prm, cudaStream_t stream) {
  const long long rows = static_cast<long long>(prm.B) * (prm.K + 1);
  const long long grid = rows * prm.slices;
  if (grid >= (1LL << 31)) return DSPARK_ERR_UNSUPPORTED;
  cudaError_t e = launch(greedy_argmax_kernel<T, VEC>, dim3(static_cast<unsigned>(grid)),
                         dim3(kGreedyThreads), 0, stream, 0, false, prm);
  if (e != cudaSuccess) return DSPARK_ERR_CUDA;
  e = launch(greedy_finish_kernel<8>, dim3(prm.B), dim3(256), 0, stream, 0, true, prm);
  return e == cudaSuccess ? DSPARK_OK : DSPARK_ERR_CUDA;
}

// ------------------------------------------------------------------------------ sampling

template <typename T, int VEC, bool kTma>
dspark_status_t run_sample(SampleParams prm, const FinishParams& fin, const Plan& pl, int fn_id,
                           cudaStream_t stream) {
  const int threads = pl.warps * 32;
  const size_t smem =
      (kTma ? pass1_ring_bytes(pl.warps, pl.stages, Elem<T>::kBytes) : 0) + sizeof(Pass1Smem);
  void* fn = Pass1Kernel<T, VEC, kTma>::fn();
  cudaError_t e = cudaSuccess;
  const int mc = max_clusters(fn, fn_id, threads, smem, pl.cluster, &e);
  if (e != cudaSuccess) return DSPARK_ERR_CUDA;
  if (mc < 1) return DSPARK_ERR_UNSUPPORTED;
  prm.n_clusters = prm.n_units < mc ? prm.n_units : mc;
  e = launch(sample_rowstats_kernel<T, VEC, kTma>,
             dim3(static_cast<unsigned>(prm.n_clusters * pl.cluster)), dim3(threads), smem, stream,
             pl.cluster, false, prm);
  if (e != cudaSuccess) return DSPARK_ERR_CUDA;
  e = launch(sample_finish_kernel<T, VEC>, dim3(prm.B), dim3(kFinishThreads), 0, stream, 0, true,
             fin);
  return e == cudaSuccess ? DSPARK_OK : DSPARK_ERR_CUDA;
}

bool out_ok(const dspark_accept_out_t& o) {
  return o.n_accepted && o.tokens && o.next_token;
}

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
  if (V > kMaxChunks * 32 * kLaneElems) return DSPARK_ERR_UNSUPPORTED;
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
  return ws_layout(B, K, pl).total;
}

dspark_status_t dspark_plan(int B, int K, int V, dspark_dtype_t dtype, int aligned16,
                            dspark_plan_t* plan) {
  if (!plan || (dtype != DSPARK_BF16 && dtype != DSPARK_F32) || !shape_ok(B, K, V))
    return DSPARK_ERR_INVALID_ARG;
  Plan pl;
  if (!make_plan(V, dtype, aligned16 != 0, &pl)) return DSPARK_ERR_UNSUPPORTED;
  plan->elems_per_load = pl.vec;
  plan->elems_per_lane = kLaneElems;
  plan->chunk_elems = 32 * kLaneElems;
  plan->n_chunks = pl.n_chunks;
  plan->warps_per_cta = pl.warps;
  plan->cluster_ctas = pl.cluster;
  plan->stages = pl.stages;
  plan->greedy_slices = pl.greedy_slices;
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
  const WsLayout w = ws_layout(B, K, pl);
  if (!workspace || workspace_bytes < w.total || !aligned(workspace, 256))
    return DSPARK_ERR_WORKSPACE;
  GreedyParams prm{};
  prm.p1 = p1;
  prm.pv = pv;
  prm.ld_p1 = ld_p1;
  prm.ld_pv = ld_pv;
  prm.B = B;
  prm.K = K;
  prm.V = V;
  prm.drafts = drafts;
  prm.slices = pl.greedy_slices;
  prm.part = reinterpret_cast<int4*>(static_cast<char*>(workspace) + w.greedy_part);
  prm.out = out;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (dtype == DSPARK_BF16)
    return a16 ? run_greedy<bf16_t, 8>(prm, s) : run_greedy<bf16_t, 1>(prm, s);
  return a16 ? run_greedy<float, 4>(prm, s) : run_greedy<float, 1>(prm, s);
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
  const WsLayout w = ws_layout(B, K, pl);
  if (!workspace || workspace_bytes < w.total || !aligned(workspace, 256))
    return DSPARK_ERR_WORKSPACE;
  const float scale = static_cast<float>(1.4426950408889634 / static_cast<double>(temperature));
  if (!std::isfinite(scale)) return DSPARK_ERR_INVALID_ARG;
  char* ws = static_cast<char*>(workspace);

  SampleParams prm{};
  prm.p1 = p1;
  prm.pv = pv;
  prm.q = q;
  prm.ld_p1 = ld_p1;
  prm.ld_pv = ld_pv;
  prm.B = B;
  prm.K = K;
  prm.V = V;
  prm.scale = scale;
  prm.n_chunks = pl.n_chunks;
  prm.warps = pl.warps;
  prm.cluster = pl.cluster;
  prm.n_units = B * (K + 1);
  prm.stages = pl.stages;
  prm.rowstat = reinterpret_cast<float2*>(ws + w.rowstat);
  prm.chunk_p = reinterpret_cast<ChunkRec*>(ws + w.chunk_p);
  prm.chunk_r = reinterpret_cast<ChunkRec*>(ws + w.chunk_r);
  prm.unit_flags = reinterpret_cast<uint8_t*>(ws + w.unit_flags);

  FinishParams fin{};
  fin.p1 = p1;
  fin.pv = pv;
  fin.q = q;
  fin.ld_p1 = ld_p1;
  fin.ld_pv = ld_pv;
  fin.B = B;
  fin.K = K;
  fin.V = V;
  fin.scale = scale;
  fin.drafts = drafts;
  fin.uniforms = uniforms;
  fin.n_chunks = pl.n_chunks;
  fin.cluster = pl.cluster;
  fin.warps = pl.warps;
  fin.rowstat = prm.rowstat;
  fin.chunk_p = prm.chunk_p;
  fin.chunk_r = prm.chunk_r;
  fin.unit_flags = prm.unit_flags;
  fin.out = out;

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (dtype == DSPARK_BF16) {
    if (!a16) return run_sample<bf16_t, 1, false>(prm, fin, pl, 0, s);
    if (pl.stages) return run_sample<bf16_t, 8, true>(prm, fin, pl, 1, s);
    return run_sample<bf16_t, 8, false>(prm, fin, pl, 2, s);
  }
  if (!a16) return run_sample<float, 1, false>(prm, fin, pl, 3, s);
  if (pl.stages) return run_sample<float, 4, true>(prm, fin, pl, 4, s);
  return run_sample<float, 4, false>(prm, fin, pl, 5, s);
}

}  // extern "C"
