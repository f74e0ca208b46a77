/*
 * dspark_verify.h - C ABI of the DSpark block-draft verify/accept step on B200 (sm_100a).
 *
 * What the calls compute
 * ----------------------
 * One decode cycle of block speculative decoding ends with a verify step. The base model
 * has produced, for every sequence b of the batch, a logit block of K+1 rows:
 *   row 0      p_1          from the step that produced the anchor token (free, never recomputed)
 *   rows 1..K  p_2..p_{K+1} from ONE verify forward over the K drafted tokens; row K is the
 *                           bonus position.
 * (Page "dspark-mlx 0.1.0__py3-none-any.whl", dspark_mlx/adapter.py, module docstring
 * "Logit conventions", and the StepOut / BlockOut dataclasses: StepOut.logits [b, V] is p_1,
 * BlockOut.per_pos_logits [b, K, V] is p_2..p_{K+1}.) The drafter supplied K draft tokens
 * x_0..x_{K-1} and, for the sampling policy, the K draft logit rows q_1..q_K they were drawn
 * from. The same wheel's dspark_mlx/__init__.py exports the two accept policies
 * greedy_accept and speculative_sample_accept and their AcceptResult; this header is their
 * device form.
 *
 *  - greedy_accept: accepted prefix = the leading drafts equal to the lowest-index argmax of
 *    their base row; the emitted token is the argmax of the first mismatching row (or of the
 *    bonus row when all K match). Output equals plain greedy decoding (mlx-dspark 0.0.1
 *    README, "How it works").
 *  - speculative_sample_accept: the lossless rejection rule (Leviathan et al. 2023, Chen et
 *    al. 2023): with p_i = softmax(P_i / T), q_i = softmax(Q_i / T), draft x_i is accepted iff
 *    u[b,i] * q_i(x_i) < p_i(x_i); at the first rejection j the correction is drawn from
 *    normalize(max(p_j - q_j, 0)); when all K are accepted the bonus is drawn from p_{K+1}.
 *    Both draws use u[b,K] by inverse CDF in ascending token order: the smallest v with
 *    sum_{t<=v} r[t] > u[b,K] * sum(r). The emitted tokens are distributed exactly as the
 *    target's (the adapter.py docstring's "lossless accept policy"; the DeepSeek-V4-Flash
 *    DSpark drafter card's "lossless by construction").
 *
 * Beside these: dspark_mixed_accept (a serving batch with per-sequence draft counts and
 * temperatures), dspark_early_exit_accept (rows read only up to each sequence's first
 * rejection), dspark_markov_matvec (the drafter's Markov-head table mat-vec), and
 * dspark_sample_pass1 (the sampling call's stream kernel alone, for timing it).
 *
 * Conventions common to every entry point
 * ---------------------------------------
 *  - Every buffer pointer is a DEVICE pointer owned by the caller. The library allocates no
 *    device memory, never synchronizes the stream, and returns as soon as its kernels are
 *    enqueued on `stream` (a cudaStream_t passed as void*; NULL = the legacy default stream).
 *  - Logits are row-major, contiguous along V, of type `dtype` (bf16 or fp32), consumed as
 *    given (soft-capping, masking etc. are the producer's job). -inf entries are allowed
 *    (masked tokens).
 *  - Returned synchronously: DSPARK_ERR_INVALID_ARG for a bad argument (nothing enqueued),
 *    DSPARK_ERR_UNSUPPORTED for a shape beyond the kernels' limits or a pointer not aligned to
 *    its element size, DSPARK_ERR_WORKSPACE for a missing or short workspace, DSPARK_ERR_CUDA
 *    if a launch failed. B == 0 is a no-op returning DSPARK_OK.
 *  - Data errors are reported per sequence on the device, never by a trap: a draft id outside
 *    [0, V), or a row holding NaN or +inf or no finite value, makes that sequence's result
 *    n_accepted = 0, tokens all -1, next_token = -1, with the cause in status[b].
 *  - Limits: 0 <= K <= 32; 1 <= V <= 262144; B * (2K+1) < 2^31; row strides ld_p1, ld_pv
 *    below 2^31 elements (larger ones: DSPARK_ERR_UNSUPPORTED).
 *  - Calls that share a workspace must not overlap on the GPU (same stream, or ordered).
 *  - Programmatic dependent launch: a call's first kernel is launched as a programmatic
 *    dependent of the kernel before it in the stream and waits for that kernel to complete
 *    before reading any input, and a call's last kernel lets the next kernel in the stream be
 *    scheduled early. A caller that launches its next kernel with programmatic stream
 *    serialization must, as always, have it wait (griddepcontrol.wait /
 *    cudaGridDependencySynchronize) before reading the results.
 */
#ifndef DSPARK_VERIFY_H
#define DSPARK_VERIFY_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  DSPARK_OK = 0,
  DSPARK_ERR_INVALID_ARG = 1,
  DSPARK_ERR_UNSUPPORTED = 2,
  DSPARK_ERR_CUDA = 3,
  DSPARK_ERR_WORKSPACE = 4
} dspark_status_t;

typedef enum { DSPARK_BF16 = 0, DSPARK_F32 = 1 } dspark_dtype_t;

/* Per-sequence bits written to out.status[b]. */
#define DSPARK_SEQ_BAD_DRAFT 1     /* a draft id outside [0, V)                           */
#define DSPARK_SEQ_NONFINITE 2     /* a row with NaN / +inf, or with no finite value       */
#define DSPARK_SEQ_ZERO_RESIDUAL 4 /* not an error: residual mass rounded to 0 after a
                                      rejection; the correction was drawn from p_j          */
#define DSPARK_SEQ_TIMEOUT 8       /* reserved: the kernels have no waits that can give up  */
#define DSPARK_SEQ_BAD_PARAM 16    /* dspark_mixed_accept: a draft count outside [0, K], or a
                                      negative or non-finite temperature (or one so small that
                                      log2(e)/T overflows)                                    */

/* AcceptResult: device buffers, caller-allocated. Required: n_accepted, tokens, next_token.
 * The optional ones (NULL = not written) are diagnostics of the sampling policy. */
typedef struct {
  int32_t* n_accepted; /* [B]      j in [0, K]: accepted drafts = n_keep for the host's KV rollback */
  int32_t* tokens;     /* [B, K+1] x_0..x_{j-1}, then the correction / bonus token, then -1      */
  int32_t* next_token; /* [B]      the correction (j < K) or the bonus token (j == K)            */
  int32_t* status;     /* [B] or NULL: DSPARK_SEQ_* bits, 0 = ok                                 */
  float* p_draft;      /* [B, K] or NULL: p_i(x_i)  (sampling only)                              */
  float* q_draft;      /* [B, K] or NULL: q_i(x_i)  (sampling only)                              */
  float* resid_mass;   /* [B] or NULL: Z_j = sum max(p_j - q_j, 0) if j < K, else 1 (sampling)  */
} dspark_accept_out_t;

/* Human-readable name of a dspark_status_t value. Never NULL. */
const char* dspark_status_string(int status);

/* Library ABI version (bumped on any incompatible change; 4: the workspace grew by the
 * early-exit waves' state, so a size taken from an older library is too small). */
int dspark_version(void);

/* Bytes of device workspace the verify calls need for this shape (valid for both policies).
 * Returns 0 when the shape is invalid or unsupported.
 * The size covers every policy, dspark_early_exit_accept included.
 * A workspace needs no initialisation: a call writes every word of it that it reads.
 * dspark_workspace_zero_bytes returns the size of the prefix that must be zero before a call,
 * which is 0 for this library (kept so that callers can clear generically). One workspace
 * serves one call at a time. */
size_t dspark_workspace_bytes(int B, int K, int V, dspark_dtype_t dtype);
size_t dspark_workspace_zero_bytes(int B, int K);

/* Launch geometry of the calls for this shape (for tests and reports).
 * Returns DSPARK_OK and fills the fields, or an error for an invalid / unsupported shape.
 * `aligned16` says whether every row start will be 16-byte aligned (vector path).
 * A call runs two kernels on `stream`. Pass 1 reads every logit row once: its units are the
 * (row, chunk) pairs, numbered row-major across the batch; the CTA on each SM takes every
 * grid-th unit and hands them to its warps in order, and each unit gets one statistics
 * record. Pass 2, a programmatic dependent launch, takes the per-sequence decisions and, when
 * sampling, computes the draw's law chunk by chunk and draws the token. */
typedef struct {
  int elems_per_load;              /* 8 (bf16) / 4 (fp32) on the 16-byte path, 1 on the scalar path */
  int loads_in_flight;             /* loads each lane of pass 1 keeps in flight                    */
  int stream_threads_per_cta;      /* pass 1: one CTA of this many threads per SM                  */
  int threads_per_cta;             /* pass 2 of the greedy policy, early-exit decisions           */
  int chunk_elems;                 /* tokens per chunk (pass-1 unit, pass-2 chunk)                */
  int n_chunks;                    /* chunks per row                                              */
  int greedy_units_per_sequence;   /* pass-1 units of one sequence, greedy: (K+1) * n_chunks      */
  int sampling_units_per_sequence; /* pass-1 units of one sequence, sampling: (2K+1) * n_chunks   */
  int finish_ctas_per_sequence;    /* pass-2 CTAs per sequence (one cluster), sampling policy:
                                      ceil(n_chunks / 32), one chunk per warp                    */
  int finish_threads_per_cta;      /* pass-2 CTA size of the sampling policy (32 warps)           */
} dspark_plan_t;
dspark_status_t dspark_plan(int B, int K, int V, dspark_dtype_t dtype, int aligned16,
                            dspark_plan_t* plan);

/* greedy_accept.
 *  p1      [B, V] base logits p_1; row b starts at p1 + b * ld_p1 (elements, ld_p1 >= V).
 *  pv      [B, K, V] base logits p_2..p_{K+1}; sequence b starts at pv + b * ld_pv
 *          (elements, ld_pv >= K * V), its K rows are V apart. May be NULL when K == 0.
 *          A contiguous [B, K+1, V] block is p1 = blk, pv = blk + V, ld_p1 = ld_pv = (K+1) * V.
 *  drafts  [B, K] int32 draft token ids (NULL allowed when K == 0).
 *  Writes n_accepted, tokens, next_token and status; ignores the sampling diagnostics. */
dspark_status_t dspark_greedy_accept(const void* p1, int64_t ld_p1, const void* pv, int64_t ld_pv,
                                     dspark_dtype_t dtype, const int32_t* drafts, int B, int K,
                                     int V, dspark_accept_out_t out, void* workspace,
                                     size_t workspace_bytes, void* stream);

/* speculative_sample_accept.
 *  p1, ld_p1, pv, ld_pv, drafts as for greedy_accept.
 *  q         [B, K, V] draft logits q_1..q_K, contiguous (row (b, i) at q + (b*K + i) * V); the
 *            distribution the drafts were drawn from, before temperature.
 *  temperature  T > 0 divides both P and Q logits; T == 0 runs greedy_accept (q and uniforms
 *            are then not read); T < 0 or non-finite is INVALID_ARG.
 *  uniforms  [B, K+1] float32 in [0, 1): u[b, i] is the accept test of draft i, u[b, K] the one
 *            draw used for the correction or the bonus token. The caller supplies the randomness,
 *            so a call is a pure function of its inputs. */
dspark_status_t dspark_speculative_sample_accept(const void* p1, int64_t ld_p1, const void* pv,
                                                 int64_t ld_pv, const void* q,
                                                 dspark_dtype_t dtype, const int32_t* drafts,
                                                 int B, int K, int V, float temperature,
                                                 const float* uniforms, dspark_accept_out_t out,
                                                 void* workspace, size_t workspace_bytes,
                                                 void* stream);

/* Pass 1 of speculative_sample_accept alone: the stream of every P and Q row and its
 * statistics records, written to the workspace, with no decision and no output. It is the
 * call's dominant kernel; this entry point lets a benchmark time that kernel on its own (a
 * full call launches it and then the finish, which events on the stream cannot separate).
 * Arguments as for speculative_sample_accept; T must be > 0 (T == 0 has no sampling pass:
 * INVALID_ARG). Returns after enqueueing one kernel on `stream`. */
dspark_status_t dspark_sample_pass1(const void* p1, int64_t ld_p1, const void* pv, int64_t ld_pv,
                                   const void* q, dspark_dtype_t dtype, const int32_t* drafts,
                                   int B, int K, int V, float temperature, void* workspace,
                                   size_t workspace_bytes, void* stream);

/* A mixed serving batch: each sequence verifies its own number of drafts at its own
 * temperature, greedy where that temperature is 0. The pages truncate a block per step
 * through the drafter's confidence head or cap it (mlx-dspark README, "Tuning":
 * --confidence-threshold, --max-draft), and serve batches (the ds4 batched-serving fork the
 * DeepSeek-V4-Flash DSpark drafter card names); this is the verify step of such a batch.
 *  p1, ld_p1, pv, ld_pv, q, drafts as for speculative_sample_accept, for the batch's largest
 *            block K (q is required when K > 0, even if every sequence is greedy).
 *  n_drafts  [B] int32 K_b in [0, K], or NULL for K everywhere.
 *  temperatures [B] float32 T_b: > 0 samples at T_b, == 0 verifies greedily.
 *  uniforms  [B, K+1] float32 in [0, 1): u[b, i] (i < K_b) tests draft i, u[b, K_b] is the draw.
 *  Sequence b is the single-policy step on its own block: P rows 0..K_b (row K_b is its
 *  bonus row), Q rows 0..K_b-1, drafts 0..K_b-1. Rows, drafts and uniforms past those are
 *  never read (the stream skips the rows: they cost no bandwidth) and may hold anything.
 *  Results are laid out for K: tokens [B, K+1] with -1 after the drawn token; n_accepted in
 *  [0, K_b]; p_draft / q_draft / resid_mass are written for sampling sequences only (entries
 *  past K_b NaN). A K_b outside [0, K] or a bad T_b makes that sequence an error
 *  (DSPARK_SEQ_BAD_PARAM: n = 0, tokens -1, next -1). */
dspark_status_t dspark_mixed_accept(const void* p1, int64_t ld_p1, const void* pv, int64_t ld_pv,
                                    const void* q, dspark_dtype_t dtype, const int32_t* drafts,
                                    const int32_t* n_drafts, int B, int K, int V,
                                    const float* temperatures, const float* uniforms,
                                    dspark_accept_out_t out, void* workspace,
                                    size_t workspace_bytes, void* stream);

/* Early exit: the verify step reading each sequence's rows in draft order and stopping at
 * its first rejection (greedy: its first mismatch). The pages report acceptance between 52%
 * and 91% (DeepSeek-V4-Flash DSpark drafter card), so most blocks end early, and the rows
 * after a sequence's first rejection j cannot change its result; the large blocks (B=256,
 * K=15, V=262144 reads 4.2 GB in full) then read a fraction of their bytes.
 *  Arguments as for speculative_sample_accept (T == 0: greedy; q and uniforms may then be
 *  NULL), with the same workspace.
 *  The pairs (P_i, Q_i) are read in waves (the last wave adds the bonus row P_K); each wave
 *  reads only the sequences that accepted every earlier draft. When one row pair of the whole
 *  batch (B * V elements of P, and of Q when sampling) takes at least 64 MiB the waves are 1,
 *  2, 4, ... pairs, else 2, 8, 32, ... pairs (a wave costs about 5 us beyond its bytes, which
 *  a smaller pair does not hide), cut at K. A call launches two kernels per wave and, when
 *  sampling, the finish.
 *  Results: on blocks whose rows are all usable, identical to speculative_sample_accept /
 *  greedy_accept (same records, decisions and draw). Rows after the stop are never read, so
 *  a NaN or inf there is not reported; a bad row at or before the stop, or a bad bonus row
 *  after a full accept, gives DSPARK_SEQ_NONFINITE; a bad draft id gives
 *  DSPARK_SEQ_BAD_DRAFT alone (nothing is read). p_draft / q_draft are written up to the stop
 *  and NaN after it. */
dspark_status_t dspark_early_exit_accept(const void* p1, int64_t ld_p1, const void* pv,
                                        int64_t ld_pv, const void* q, dspark_dtype_t dtype,
                                        const int32_t* drafts, int B, int K, int V,
                                        float temperature, const float* uniforms,
                                        dspark_accept_out_t out, void* workspace,
                                        size_t workspace_bytes, void* stream);

/* The drafter's Markov-head table mat-vec (the drafter side of the cycle, beside the verify
 * step): y[b, v] = sum_k W[v, k] h[b, k] over the table markov_w2, V rows of R values. The
 * DeepSeek-V4-Flash DSpark drafter card ("Files") ships the table in F16 or in GGUF Q8_0 and
 * says the ds4 engine reads it in full four times per draft block (0.18 ms per call in Q8_0,
 * 0.63 ms in F16, on a GB10).
 *  table  device; DSPARK_TABLE_F16: V x R half floats, row-major (row v = vocab entry v);
 *         DSPARK_TABLE_Q8_0: V rows of R/32 GGUF Q8_0 blocks of 34 bytes (a little-endian
 *         float16 scale d, then 32 signed bytes q; value d * q[i]). 16-byte aligned.
 *  R      the Markov rank: 256 (other ranks: DSPARK_ERR_UNSUPPORTED).
 *  h      device [B, R] float32 states, 16-byte aligned.
 *  y      device [B, V] float32 results (row b at y + b * V).
 *  F16, B == 1: float32 sums in a fixed order on the CUDA cores.
 *  F16, B > 1: on the tensor cores (tcgen05), the table read once per 64 states (loaded by
 *    TMA tensor copies): each state scaled by a power of two and split into float16 hi + lo
 *    (within 2^-23 of its largest |h|); the products with the exact table halves are summed
 *    in float32 by the tensor cores, one sum per part over all R values.
 *  Q8_0, B <= 10: one read of the table; exact integer dot products of each block's bytes with
 *    three signed-byte digit planes of the state (within 2^-22 of the block's largest |h|),
 *    combined and scaled by d in float32: on the CUDA cores for B == 1, on the integer tensor
 *    cores (tcgen05 kind::i8, the table loaded as stored by TMA) for B = 2..10.
 *  Q8_0, B > 10: on the tensor cores (tcgen05), the table read once per 64 states. Each state is
 *    scaled by a power of two and split into float16 parts hi + lo (within 2^-23 of its
 *    largest |h|); each block's 32 products q * part are exact and summed in float32 by the
 *    tensor cores, then scaled by d and the 8 blocks added by float32 FMAs in a fixed order.
 *  A non-finite state value gives non-finite results. B == 0 or V == 0 is a no-op. */
typedef enum { DSPARK_TABLE_F16 = 0, DSPARK_TABLE_Q8_0 = 1 } dspark_table_t;
dspark_status_t dspark_markov_matvec(const void* table, dspark_table_t type, int V, int R,
                                     const float* h, int B, float* y, void* stream);

/* The number of waits inside the library's pipelined kernels (the tensor-core mat-vecs) that
 * ran out (about a second each) on the current device since the library was loaded: 0 unless
 * a kernel gave up; a kernel that gives up frees its resources and leaves its outputs
 * incomplete. Synchronous (waits for the device). DSPARK_ERR_INVALID_ARG for a NULL count. */
dspark_status_t dspark_pipeline_timeouts(unsigned long long* count);

/* For tests of the timeout path only: dspark_markov_matvec with each CTA's first table copy
 * withheld in its pipelined tensor-core kernels, so that the waits for it run out (about a
 * second) and the kernels give up as described above: the call returns DSPARK_OK, y is left
 * incomplete and dspark_pipeline_timeouts grows. DSPARK_ERR_UNSUPPORTED where the call would
 * take a CUDA-core kernel (one state), which has no waits. Same arguments as
 * dspark_markov_matvec. */
dspark_status_t dspark_markov_matvec_withheld(const void* table, dspark_table_t type, int V,
                                              int R, const float* h, int B, float* y,
                                              void* stream);

/* speculative_sample_accept without a workspace argument. The pages have no counterpart of
 * this entry point: it exists for callers that cannot allocate device memory where they
 * verify (a serving loop whose KV-cache pool took all free HBM at start-up and left no
 * allocator to draw a workspace from; a host runtime with no device allocator of its own).
 *  Arguments, results and T == 0 behaviour are those of dspark_speculative_sample_accept.
 *  Scratch: one fixed array of DSPARK_STATIC_SCRATCH_BYTES per device, in the library's own
 *    module image; the call allocates nothing. A shape whose dspark_workspace_bytes exceeds
 *    that size is rejected with DSPARK_ERR_WORKSPACE before anything is enqueued (the limit
 *    holds e.g. B = 64, K = 7, V = 129280 bf16, about 0.5 MB; not B = 256, K = 15, V = 262144).
 *  Set-up: the first call on a device, with that device current, looks up the array's device
 *    address (cudaGetSymbolAddress) and keeps it; make that first call before any stream
 *    capture on that device. A failed look-up returns DSPARK_ERR_CUDA. The call runs on the
 *    CURRENT device: make the device that holds the buffers current first. The kept address
 *    belongs to the device's primary context as it was at the first call; after a
 *    cudaDeviceReset of that device the library must be reloaded before this entry is used
 *    again.
 *  The array needs no clearing: each call writes every word of it that it reads.
 *  All calls on one device share the array: calls that overlap on the GPU race and give
 *    wrong results. Order them (one stream, or events). */
#define DSPARK_STATIC_SCRATCH_BYTES ((size_t)4 << 20)
dspark_status_t dspark_speculative_sample_accept_static(const void* p1, int64_t ld_p1,
                                                        const void* pv, int64_t ld_pv,
                                                        const void* q, dspark_dtype_t dtype,
                                                        const int32_t* drafts, int B, int K, int V,
                                                        float temperature, const float* uniforms,
                                                        dspark_accept_out_t out, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* DSPARK_VERIFY_H */
