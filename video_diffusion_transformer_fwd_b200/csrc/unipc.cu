// UniPC multistep sampler for the flow-matching latent ("Wan2.2 I2V inference
// trace" (damodev.csdn.net), section 4 "DIT": the latent update
// "UniPC: x_noise <- step(v, t, x_noise)"). The update is the UniPC method
// (Zhao et al., 2023, "UniPC: A Unified Predictor-Corrector Framework for
// Fast Sampling of Diffusion Models") in its data-prediction form with
// B(h) = e^h - 1, orders 1 and 2: with alpha = 1 - sigma, lambda =
// log(alpha / sigma) and the data prediction m = x - sigma v, one step
//   corrector (UniC, refines the sample reached by the previous step with the
//               new evaluation m_i):
//     x_c = (s_i / s_{i-1}) last - a_i h_phi_1 m_{i-1}
//           - a_i B_h (rho_0 (m_{i-2} - m_{i-1}) / r_1 + rho_last (m_i - m_{i-1}))
//   predictor (UniP, to the next sigma):
//     x_next = (s_{i+1} / s_i) x_c - a_{i+1} h_phi_1 m_i - a_{i+1} B_h 0.5 (m_{i-1} - m_i) / r_1
// is a linear combination of x, last, m_i, m_{i-1}, m_{i-2}: the host turns
// the schedule into its eight coefficients and one kernel applies them.
#include "common.cuh"

#include <math.h>

namespace wan {
namespace {

double flow_lambda(double s) { return s == 0.0 ? INFINITY : log(1.0 - s) - log(s); }

// h_phi_1 = B_h = e^{-h} - 1 and b_1, b_2 of the order conditions
void phis(double h, double &h_phi_1, double &B_h, double &b1, double &b2) {
  const double hh = -h;
  h_phi_1 = expm1(hh);
  B_h = h_phi_1;
  double h_phi_k = h_phi_1 / hh - 1.0;       // hh phi_2(hh)
  b1 = h_phi_k / B_h;
  h_phi_k = h_phi_k / hh - 0.5;              // hh phi_3(hh)
  b2 = h_phi_k * 2.0 / B_h;
}

__global__ void unipc_step_kernel(float *__restrict__ x, float *__restrict__ last, float *__restrict__ m_out,
                                  const float *__restrict__ m1, const float *__restrict__ m2,
                                  const void *__restrict__ v_cond, const void *__restrict__ v_uncond, int v_bf16,
                                  size_t n, float g, float sigma, float cx, float c_last, float c_m1, float c_m2,
                                  float c_mi, float p_xc, float p_mi, float p_m1) {
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
    float vc, vu;
    if (v_bf16) {
      vc = __bfloat162float(static_cast<const __nv_bfloat16 *>(v_cond)[i]);
      vu = v_uncond ? __bfloat162float(static_cast<const __nv_bfloat16 *>(v_uncond)[i]) : vc;
    } else {
      vc = static_cast<const float *>(v_cond)[i];
      vu = v_uncond ? static_cast<const float *>(v_uncond)[i] : vc;
    }
    const float v = fmaf(g, vc - vu, vu);                 // classifier-free guidance
    const float xi = x[i];
    const float mi = fmaf(-sigma, v, xi);                 // data prediction
    float xc = cx * xi;
    if (c_last != 0.f) xc = fmaf(c_last, last[i], xc);
    if (m1) xc = fmaf(c_m1, m1[i], xc);
    if (m2) xc = fmaf(c_m2, m2[i], xc);
    xc = fmaf(c_mi, mi, xc);
    float xn = fmaf(p_xc, xc, p_mi * mi);
    if (m1) xn = fmaf(p_m1, m1[i], xn);
    m_out[i] = mi;
    last[i] = xc;
    x[i] = xn;
  }
}

}  // namespace
}  // namespace wan

using namespace wan;

extern "C" {

int wan_unipc_coefficients(const double *sigmas, int num_sigmas, int step, int order, int lower_order_final,
                           double coef[8]) {
  if (!sigmas || !coef) return set_error(WAN_EINVAL, "NULL argument");
  const int n = num_sigmas - 1;                        // model evaluations
  if (n < 1 || step < 0 || step >= n) return set_error(WAN_EINVAL, "step %d of %d", step, n);
  if (order < 1 || order > 2) return set_error(WAN_EUNSUPPORTED, "UniPC order %d (1 or 2)", order);
  for (int k = 0; k <= n; ++k)
    if (!(sigmas[k] >= 0.0 && sigmas[k] < 1.0) || (k > 0 && !(sigmas[k] < sigmas[k - 1])))
      return set_error(WAN_EINVAL, "sigmas must decrease within [0, 1)");
  for (int k = 0; k < n; ++k)
    if (sigmas[k] == 0.0) return set_error(WAN_EINVAL, "only the last sigma may be 0");
  // order of the predictor step taken from sigma_j: warm-up, then the full
  // order; the last step first order when asked (always when it lands on 0)
  auto order_at = [&](int j) {
    int o = order < j + 1 ? order : j + 1;
    if ((lower_order_final || sigmas[j + 1] == 0.0) && n - j < o) o = n - j;
    if (sigmas[j + 1] == 0.0) o = 1;
    return o;
  };
  const int i = step;
  double cx = 1.0, c_last = 0.0, c_m1 = 0.0, c_m2 = 0.0, c_mi = 0.0;
  if (i > 0) {                                         // corrector with the order of the previous step
    const int oc = order_at(i - 1);
    const double s0 = sigmas[i - 1], t = sigmas[i], at = 1.0 - t;
    const double h = flow_lambda(t) - flow_lambda(s0);
    double h_phi_1, B_h, b1, b2;
    phis(h, h_phi_1, B_h, b1, b2);
    cx = 0.0;
    c_last = t / s0;
    if (oc == 1) {
      const double rho = 0.5;
      c_m1 = -at * h_phi_1 + at * B_h * rho;
      c_mi = -at * B_h * rho;
    } else {
      const double r1 = (flow_lambda(sigmas[i - 2]) - flow_lambda(s0)) / h;
      // R = [[1, 1], [r1, 1]], R rho = b
      const double rho0 = (b1 - b2) / (1.0 - r1), rho1 = (b2 - r1 * b1) / (1.0 - r1);
      c_m2 = -at * B_h * rho0 / r1;
      c_mi = -at * B_h * rho1;
      c_m1 = -at * h_phi_1 + at * B_h * (rho0 / r1 + rho1);
    }
  }
  const int op = order_at(i);
  const double s0 = sigmas[i], t = sigmas[i + 1], at = 1.0 - t;
  const double h = flow_lambda(t) - flow_lambda(s0);
  double h_phi_1, B_h, b1, b2;
  phis(h, h_phi_1, B_h, b1, b2);
  double p_xc = t / s0, p_mi = -at * h_phi_1, p_m1 = 0.0;
  if (op == 2) {
    const double r1 = (flow_lambda(sigmas[i - 1]) - flow_lambda(s0)) / h;
    p_m1 = -0.5 * at * B_h / r1;
    p_mi += 0.5 * at * B_h / r1;
  }
  const double c[8] = {cx, c_last, c_m1, c_m2, c_mi, p_xc, p_mi, p_m1};
  for (int k = 0; k < 8; ++k) {
    if (!isfinite(c[k])) return set_error(WAN_EINVAL, "UniPC coefficient %d not finite at step %d", k, i);
    coef[k] = c[k];
  }
  return WAN_OK;
}

int wan_unipc_step(float *x, float *last, float *m_out, const float *m_prev1, const float *m_prev2,
                   const void *v_cond, const void *v_uncond, int v_dtype, size_t n, float guide_scale,
                   float sigma, const double coef[8], wan_stream_t stream) {
  if (n == 0) return WAN_OK;
  if (!x || !last || !m_out || !v_cond || !coef) return set_error(WAN_EINVAL, "NULL argument");
  if (v_dtype != WAN_F32 && v_dtype != WAN_BF16) return set_error(WAN_EUNSUPPORTED, "v dtype %d", v_dtype);
  if ((coef[2] != 0.0 || coef[7] != 0.0) && !m_prev1) return set_error(WAN_EINVAL, "m_prev1 needed");
  if (coef[3] != 0.0 && !m_prev2) return set_error(WAN_EINVAL, "m_prev2 needed");
  const void *ps[] = {x, last, m_out, m_prev1, m_prev2, v_cond, v_uncond};
  for (const void *p : ps)
    if (p && !aligned16(p)) return set_error(WAN_EALIGN, "pointer not 16-byte aligned");
  cudaStream_t s = (cudaStream_t)stream;
  size_t g = (n + 255) / 256;
  if (g > 148 * 16) g = 148 * 16;
  WAN_PROF(WAN_K_EULER, s, (unipc_step_kernel<<<(int)g, 256, 0, s>>>(
      x, last, m_out, coef[2] != 0.0 || coef[7] != 0.0 ? m_prev1 : nullptr, coef[3] != 0.0 ? m_prev2 : nullptr,
      v_cond, v_uncond, v_dtype == WAN_BF16, n, guide_scale, sigma, (float)coef[0], (float)coef[1],
      (float)coef[2], (float)coef[3], (float)coef[4], (float)coef[5], (float)coef[6], (float)coef[7]), 0));
  WAN_CHECK_LAUNCH("unipc_step");
  return WAN_OK;
}

}  // extern "C"
