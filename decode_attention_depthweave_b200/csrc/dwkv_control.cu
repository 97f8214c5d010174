// dwkv_control.cu -- the probe-driven tier threshold ("DepthWeave-KV: Token-Adaptive
// Cross-Layer Residual Factorization for Long-Context KV Cache Compression", §3 Method):
//   * Eq. (2): the router raises a token from the low rank level to the high one when its
//     salience sigma(u^T phi) exceeds the depth window's threshold tau_m;
//   * Eq. (3) paragraph: probes run every p decode steps; when the observed error exceeds a
//     tolerance tau_m is lowered (more tokens take the high level), and after several quiet
//     probe intervals it is raised again (the memory budget).
// Host code only: the probe itself is dwkv_probe and the move of stored tokens between tiers
// is dwkv_retier.  The salience scores are the caller's (the router's learned weights are not
// part of this library).
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <new>
#include <string>
#include <vector>

#include "dwkv.h"

struct dwkv_tier_ctrl {
    dwkv_tier_policy pol;
    std::vector<float> tau;      // per group
    std::vector<int32_t> quiet;  // probes in a row at or below the tolerance, per group
};

namespace dwkv {
void set_last_error(const char* msg);     // dwkv_api.cu: the message dwkv_last_error() returns
}

namespace {
dwkv_status ctrl_fail(dwkv_status st, const char* msg) {
    dwkv::set_last_error(msg);
    return st;
}
}  // namespace

extern "C" {

dwkv_status dwkv_tier_controller_create(const dwkv_tier_policy* pol, int32_t num_groups, dwkv_tier_controller* out) {
    if (!out) return ctrl_fail(DWKV_ERR_INVALID_ARG, "out is NULL");
    *out = nullptr;
    if (!pol) return ctrl_fail(DWKV_ERR_INVALID_ARG, "policy is NULL");
    if (num_groups <= 0) return ctrl_fail(DWKV_ERR_INVALID_ARG, "num_groups must be positive");
    const bool finite = std::isfinite(pol->tol) && std::isfinite(pol->tau_init) && std::isfinite(pol->tau_min) &&
                        std::isfinite(pol->tau_max) && std::isfinite(pol->tau_step_down) && std::isfinite(pol->tau_step_up);
    if (!finite || pol->tol < 0.f || pol->tau_min > pol->tau_max || pol->tau_init < pol->tau_min ||
        pol->tau_init > pol->tau_max || pol->tau_step_down < 0.f || pol->tau_step_up < 0.f)
        return ctrl_fail(DWKV_ERR_INVALID_ARG, "policy: need finite values, tol >= 0, tau_min <= tau_init <= tau_max, "
                                               "steps >= 0");
    if (pol->quiet_intervals < 1 || pol->probe_every < 1)
        return ctrl_fail(DWKV_ERR_INVALID_ARG, "policy: quiet_intervals and probe_every must be >= 1");
    auto* c = new (std::nothrow) dwkv_tier_ctrl();
    if (!c) return ctrl_fail(DWKV_ERR_CAPACITY, "out of host memory");
    c->pol = *pol;
    c->tau.assign((size_t)num_groups, pol->tau_init);
    c->quiet.assign((size_t)num_groups, 0);
    *out = c;
    return DWKV_OK;
}

dwkv_status dwkv_tier_controller_destroy(dwkv_tier_controller c) {
    if (!c) return ctrl_fail(DWKV_ERR_INVALID_ARG, "controller is NULL");
    delete c;
    return DWKV_OK;
}

int32_t dwkv_tier_controller_due(dwkv_tier_controller c, int64_t step) {
    if (!c || step < 0) return 0;
    return step % c->pol.probe_every == 0 ? 1 : 0;
}

dwkv_status dwkv_tier_controller_threshold(dwkv_tier_controller c, int32_t group, float* tau) {
    if (!c || !tau) return ctrl_fail(DWKV_ERR_INVALID_ARG, "controller or tau is NULL");
    if (group < 0 || group >= (int32_t)c->tau.size()) return ctrl_fail(DWKV_ERR_INVALID_ARG, "group out of range");
    *tau = c->tau[(size_t)group];
    return DWKV_OK;
}

dwkv_status dwkv_tier_controller_observe(dwkv_tier_controller c, int32_t group, float err, int32_t* lowered) {
    if (!c) return ctrl_fail(DWKV_ERR_INVALID_ARG, "controller is NULL");
    if (group < 0 || group >= (int32_t)c->tau.size()) return ctrl_fail(DWKV_ERR_INVALID_ARG, "group out of range");
    if (std::isnan(err)) return ctrl_fail(DWKV_ERR_INVALID_ARG, "err is NaN");
    float& tau = c->tau[(size_t)group];
    int32_t& q = c->quiet[(size_t)group];
    int32_t low = 0;
    if (err > c->pol.tol) {
        const float t = tau - c->pol.tau_step_down;
        tau = t < c->pol.tau_min ? c->pol.tau_min : t;
        q = 0;
        low = 1;
    } else if (++q >= c->pol.quiet_intervals) {
        const float t = tau + c->pol.tau_step_up;
        tau = t > c->pol.tau_max ? c->pol.tau_max : t;
        q = 0;
    }
    if (lowered) *lowered = low;
    return DWKV_OK;
}

dwkv_status dwkv_tier_controller_route(dwkv_tier_controller c, int32_t group, int32_t n, const float* salience,
                                       const uint8_t* base_tier, int32_t high_tier, uint8_t* tier_out) {
    if (!c) return ctrl_fail(DWKV_ERR_INVALID_ARG, "controller is NULL");
    if (group < 0 || group >= (int32_t)c->tau.size()) return ctrl_fail(DWKV_ERR_INVALID_ARG, "group out of range");
    if (n < 0 || high_tier < 0 || high_tier >= DWKV_MAX_TIERS)
        return ctrl_fail(DWKV_ERR_INVALID_ARG, "n or high_tier out of range");
    if (n && (!salience || !base_tier || !tier_out)) return ctrl_fail(DWKV_ERR_INVALID_ARG, "NULL array");
    const float tau = c->tau[(size_t)group];
    for (int32_t t = 0; t < n; ++t) {
        const uint8_t b = base_tier[t];
        tier_out[t] = (salience[t] > tau && (int32_t)b < high_tier) ? (uint8_t)high_tier : b;
    }
    return DWKV_OK;
}

}  // extern "C"
