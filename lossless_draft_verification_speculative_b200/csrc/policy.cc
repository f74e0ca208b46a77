// The yield-quench speculation policy (include/dspark_policy.h): host code, no CUDA.
#include <cmath>
#include <cstring>

#include "dspark_policy.h"

namespace {

bool config_ok(const dspark_quench_config_t* c) {
  return c && std::isfinite(c->break_even) && c->break_even > 0.0 && c->warmup >= 1 &&
         c->window >= 1 && c->window <= DSPARK_QUENCH_MAX_WINDOW && c->kv_limit >= 0;
}

// One verified cycle of a speculating request that committed `t` tokens.
void add_cycle(const dspark_quench_config_t& c, dspark_quench_state_t& s, int32_t t) {
  const int slot = s.cycles % c.window;
  if (s.cycles >= c.window) s.window_sum -= s.ring[slot];  // the cycle leaving the window
  s.ring[slot] = t;
  s.window_sum += t;
  s.cycles += 1;
  s.committed += t;
  if (s.cycles >= c.warmup) {
    const int in_window = s.cycles < c.window ? s.cycles : c.window;
    // mean yield over the window below the break-even yield: window_sum < break_even * n
    if (static_cast<double>(s.window_sum) < c.break_even * in_window)
      s.state = DSPARK_SPEC_OFF_YIELD;
  }
}

}  // namespace

extern "C" {

dspark_status_t dspark_quench_reset(dspark_quench_state_t* states, int n) {
  if (n < 0 || (n > 0 && !states)) return DSPARK_ERR_INVALID_ARG;
  for (int b = 0; b < n; ++b) {
    std::memset(&states[b], 0, sizeof(dspark_quench_state_t));
    states[b].state = DSPARK_SPEC_ON;
  }
  return DSPARK_OK;
}

dspark_status_t dspark_quench_update(const dspark_quench_config_t* config,
                                     dspark_quench_state_t* states, int n,
                                     const int32_t* n_accepted, const int64_t* kv_depth,
                                     int32_t* speculate) {
  if (!config_ok(config) || n < 0) return DSPARK_ERR_INVALID_ARG;
  if (n == 0) return DSPARK_OK;
  if (!states || !n_accepted || !speculate) return DSPARK_ERR_INVALID_ARG;
  // every argument is checked before any state changes
  for (int b = 0; b < n; ++b)
    if (states[b].state == DSPARK_SPEC_ON && n_accepted[b] > DSPARK_MAX_DRAFTS)
      return DSPARK_ERR_INVALID_ARG;
  const dspark_quench_config_t& c = *config;
  for (int b = 0; b < n; ++b) {
    dspark_quench_state_t& s = states[b];
    if (s.state == DSPARK_SPEC_ON && n_accepted[b] >= 0) add_cycle(c, s, n_accepted[b] + 1);
    if (s.state == DSPARK_SPEC_ON && c.kv_limit > 0 && kv_depth && kv_depth[b] > c.kv_limit)
      s.state = DSPARK_SPEC_OFF_KV;
    speculate[b] = s.state == DSPARK_SPEC_ON ? 1 : 0;
  }
  return DSPARK_OK;
}

}  // extern "C"
