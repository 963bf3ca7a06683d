// bias_controller.cpp -- host-side PID controller of the expert biases.
//
// LongCat-Flash write-up ("Meituan's large model goes viral for its speed",
// section "Zero-computation experts"): the expert-specific bias terms are
// adjusted from recent expert usage, decoupled from the training objective,
// by a PID controller from control theory, so that the share of picks that
// land on zero-computation experts -- and with it the compute per token --
// stays where it is wanted.  The page gives no gains, set-point or window;
// the plainest reading is used:
//
//   set-point   the zero experts together take a fraction rho of all T*K
//               picks and the FFN experts share the rest evenly:
//               L*_i = (1 - rho) T K / N (i < N),  rho T K / Z (i >= N)
//   error       e_i = (L*_i - L_i) / (T K / E), the load shortfall of expert
//               i in units of the mean load
//   law         b_i = base_i + clip(kp e_i + ki sum_s e_i(s) + kd (e_i - e_i,prev))
//
// with base_i the bias when the controller was (re)started.  An expert that
// gets too few picks has e_i > 0 and its bias rises.  With a clip, a step
// whose unclipped output lies beyond it on the side its error pushes towards
// leaves the integral as it was (conditional integration against integral
// windup): after a long saturated stretch the bias leaves the clip as soon as
// the error turns.  Arithmetic in double.
#include <cmath>
#include <cstdint>

#include "../../include/moe_zc.h"

extern "C" int moe_zc_bias_controller_init(const float* b, int32_t E, float* state) {
  if (!b || !state || E < 1) return MOE_ZC_ERR_INVALID_ARG;
  for (int32_t i = 0; i < E; ++i) {
    state[i] = b[i];          // base
    state[E + i] = 0.f;       // integral of the error
    state[2 * E + i] = 0.f;   // previous error
  }
  return MOE_ZC_OK;
}

extern "C" int moe_zc_bias_controller_step(const int32_t* counts, int32_t N, int32_t Z,
                                           int64_t tokens, int32_t K, const moe_zc_pid* pid,
                                           float* state, float* b) {
  if (!counts || !pid || !state || !b) return MOE_ZC_ERR_INVALID_ARG;
  if (N < 0 || Z < 0 || N + Z < 1 || tokens <= 0 || K < 1 || K > N + Z)
    return MOE_ZC_ERR_INVALID_ARG;
  const double rho = pid->target_zero_frac;
  if (!(rho >= 0.0 && rho <= 1.0)) return MOE_ZC_ERR_INVALID_ARG;
  if ((N == 0 && rho != 1.0) || (Z == 0 && rho != 0.0)) return MOE_ZC_ERR_INVALID_ARG;
  const int32_t E = N + Z;
  const double picks = static_cast<double>(tokens) * K;
  const double mean = picks / E;
  const double clip = pid->max_shift;
  for (int32_t i = 0; i < E; ++i) {
    const double target = i < N ? (1.0 - rho) * picks / N : rho * picks / Z;
    const double e = (target - counts[i]) / mean;
    double integral = static_cast<double>(state[E + i]) + e;
    const double deriv = e - static_cast<double>(state[2 * E + i]);
    double shift = pid->kp * e + pid->ki * integral + pid->kd * deriv;
    if (clip > 0.0) {
      if (std::fabs(shift) > clip && (shift > 0.0) == (e > 0.0) && e != 0.0) {
        integral = static_cast<double>(state[E + i]);   // saturated: do not wind up
        shift = pid->kp * e + pid->ki * integral + pid->kd * deriv;
      }
      shift = std::fmax(-clip, std::fmin(clip, shift));
    }
    b[i] = static_cast<float>(static_cast<double>(state[i]) + shift);
    state[E + i] = static_cast<float>(integral);
    state[2 * E + i] = static_cast<float>(e);
  }
  return MOE_ZC_OK;
}
