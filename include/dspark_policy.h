/*
 * dspark_policy.h - host-side speculation policy fed by the verify step's results.
 *
 * Source: the DeepSeek-V4-Flash DSpark drafter card, closing paragraph of "Usage": draft
 * acceptance is content-dependent (52-91% across workloads); since ds4 fork v0.1.1 a terminal
 * yield-quench controller turns speculation off per request when acceptance cannot pay the
 * verify cost (worst case about 0.96x plain decode), and a kv-depth gate hands requests with
 * more than 64k tokens of context to plain decode. The card gives no formula; the readings
 * below are this library's.
 *
 *  - Yield: the tokens a verify cycle commits, n_accepted + 1 (the accepted drafts plus the
 *    correction or bonus token; AcceptResult of dspark_verify.h).
 *  - Cost: a speculative cycle (drafting plus one verify forward over K+1 positions) costs
 *    `break_even` plain decode steps. Speculation pays while the mean yield is at least
 *    that: a request then commits its tokens in less time than plain decode would.
 *  - Quench: after `warmup` cycles, a request whose mean yield over its last `window`
 *    cycles falls below `break_even` stops speculating, for good ("terminal"): it decodes
 *    plainly from then on, so it never loses more than its first cycles' excess cost.
 *  - kv-depth gate: a request whose context (KV cache depth, tokens) exceeds `kv_limit`
 *    decodes plainly from then on (the card's gate: 64k = 65536).
 *
 * The policy is plain host code (no CUDA): it runs on host copies of n_accepted and of the
 * context depths, between verify cycles. All pointers here are HOST pointers owned by the
 * caller; the functions keep no state of their own and allocate nothing.
 */
#ifndef DSPARK_POLICY_H
#define DSPARK_POLICY_H

#include <stdint.h>

#include "dspark_verify.h"

#ifdef __cplusplus
extern "C" {
#endif

#define DSPARK_QUENCH_MAX_WINDOW 64
#define DSPARK_MAX_DRAFTS 32 /* the largest n_accepted a verify call returns (K <= 32) */

typedef struct {
  double break_even; /* cost of one speculative cycle in plain decode steps (> 0): the mean
                        committed tokens per cycle below which speculation does not pay */
  int32_t warmup;    /* cycles a request speculates before it is first judged (>= 1) */
  int32_t window;    /* cycles in the trailing mean of the yield, 1..DSPARK_QUENCH_MAX_WINDOW */
  int64_t kv_limit;  /* context depth (tokens) above which a request decodes plainly; 0: no gate */
} dspark_quench_config_t;

typedef enum {
  DSPARK_SPEC_ON = 0,        /* speculating */
  DSPARK_SPEC_OFF_YIELD = 1, /* quenched: the mean yield fell below break_even */
  DSPARK_SPEC_OFF_KV = 2     /* gated: the context grew past kv_limit */
} dspark_spec_state_t;

/* One request's controller state (caller-owned; set up by dspark_quench_reset). */
typedef struct {
  int32_t state;     /* dspark_spec_state_t */
  int32_t cycles;    /* verify cycles seen while speculating */
  int64_t committed; /* tokens those cycles committed */
  int32_t window_sum;                       /* committed tokens of the last min(cycles, window) */
  int32_t ring[DSPARK_QUENCH_MAX_WINDOW];   /* committed tokens per cycle, cycle c at c % window */
} dspark_quench_state_t;

/* Start n requests in the speculating state. DSPARK_ERR_INVALID_ARG if n < 0 or states is
 * NULL with n > 0. */
dspark_status_t dspark_quench_reset(dspark_quench_state_t* states, int n);

/* One step of the controller for n requests.
 *  n_accepted [n]: each request's n_accepted from the verify call of this step, or a negative
 *                  value when the request was not verified this step (no update).
 *  kv_depth   [n] or NULL: each request's context depth after the step (NULL: no gate).
 *  speculate  [n] out: 1 if the request should draft and verify next step, else 0.
 * Requests already off stay off (their n_accepted is ignored). A request that was verified
 * with n_accepted > DSPARK_MAX_DRAFTS (32) is an argument error. Returns
 * DSPARK_ERR_INVALID_ARG, with nothing changed, for a bad config (break_even not a finite
 * number > 0, warmup < 1, window outside 1..DSPARK_QUENCH_MAX_WINDOW, kv_limit < 0), NULL arrays
 * with n > 0, n < 0, or a bad n_accepted. */
dspark_status_t dspark_quench_update(const dspark_quench_config_t* config,
                                     dspark_quench_state_t* states, int n,
                                     const int32_t* n_accepted, const int64_t* kv_depth,
                                     int32_t* speculate);

#ifdef __cplusplus
}
#endif

#endif /* DSPARK_POLICY_H */
