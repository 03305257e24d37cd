// param_checks.h -- the domain check of tara_params, shared by the device-buffer and the
// host-buffer entry points (host code only).
#pragma once

#include <cmath>

#include "tara_attn.h"

namespace tara {

inline int check_params(const tara_params* p) {
  auto finite = [](float x) { return std::isfinite(x); };
  if (!finite(p->window) || !finite(p->falloff) || !finite(p->strength) || !finite(p->cap) ||
      !finite(p->softmax_scale))
    return TARA_ERR_PARAM;
  if (p->falloff <= 0.0f || p->window < 0.0f || p->strength < 0.0f || p->cap < 0.0f ||
      p->softmax_scale < 0.0f)
    return TARA_ERR_PARAM;
  for (int i = 0; i < 9; ++i)
    if (!finite(p->gain[i]) || p->gain[i] <= 0.0f) return TARA_ERR_PARAM;
  if (p->n_extra_bindings < 0 || p->n_extra_bindings > TARA_MAX_EXTRA_BINDINGS)
    return TARA_ERR_PARAM;
  for (int k = 0; k < p->n_extra_bindings; ++k)
    for (int i = 0; i < 9; ++i)
      if (!finite(p->extra_gain[k][i]) || p->extra_gain[k][i] <= 0.0f) return TARA_ERR_PARAM;
  if (p->qk_int8 != 0 && p->qk_int8 != 1) return TARA_ERR_PARAM;
  return TARA_OK;
}

}  // namespace tara
