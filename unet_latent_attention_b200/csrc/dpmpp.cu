// Classifier-free guidance fused with a DPM-Solver++(2M) latent update (sd_cfg_dpmpp_2m_step).
//
// "从零实现扩散模型推理引擎：Rust + wgpu 的 GPU 加速图像生成架构" §4 keeps a DPM-Solver++ scheduler next to
// DDIM (order 1 = DDIM-equivalent, order 2 = second order from a sample history, Karras sigmas)
// without printing its update. The update here is the published DPM-Solver++(2M) multistep
// method (Lu, Zhou, Bao, Chen, Li and Zhu, 2022) in the variance-preserving parametrisation:
//
//   g  = eps_u + w (eps_c - eps_u)                       guided noise prediction (§7)
//   D  = (x - sigma_t g) / alpha_t                        data prediction, kept as the history
//   x' = (sigma_n / sigma_t) x - alpha_n expm1(-h) Dhat,  h = lambda_n - lambda_t,
//   Dhat = D (order 1) or (1 + 1/(2r)) D - 1/(2r) D_prev, r = (lambda_t - lambda_p) / h (order 2)
//
// with alpha = sqrt(alpha_bar), sigma = sqrt(1 - alpha_bar), lambda = log(alpha / sigma). Order 3
// (sd_cfg_dpmpp_3m_step; the page's "三阶") integrates exactly the quadratic through the last three
// data predictions in lambda. Every order reduces to x' = A x + k0 D + k1 D_prev + k2 D_prev2 with
// coefficients formed on the host in double; per element the kernel reads x, eps_u, eps_c and the
// history it needs and writes x' and D: 20, 24 or 28 bytes, one pass, 16-byte vector accesses.
#include <cmath>

#include "sd_internal.h"

namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ float4 ld_stream(const float4* p) {
  float4 v;
  asm volatile("ld.global.cs.v4.f32 {%0,%1,%2,%3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "l"(p));
  return v;
}

__device__ __forceinline__ void st_stream(float4* p, float4 v) {
  asm volatile("st.global.cs.v4.f32 [%0], {%1,%2,%3,%4};" ::"l"(p), "f"(v.x), "f"(v.y), "f"(v.z), "f"(v.w)
               : "memory");
}

// Per-step constants: D = x * inv_a - s_over_a * g; x' = A x + k0 D + k1 D_prev + k2 D_prev2.
struct Coef {
  float w, inv_a, s_over_a, A, k0, k1, k2;
};

template <int ORDER>
__device__ __forceinline__ void step1(float x, float eu, float ec, float d1, float d2, const Coef& c, float& xo,
                                      float& d) {
  const float g = fmaf(c.w, ec - eu, eu);
  d = fmaf(-c.s_over_a, g, x * c.inv_a);
  float hist = 0.f;
  if constexpr (ORDER >= 2) hist = c.k1 * d1;
  if constexpr (ORDER == 3) hist = fmaf(c.k2, d2, hist);
  xo = fmaf(c.A, x, fmaf(c.k0, d, hist));
}

// x_out may alias x and d_out may alias d_prev or d_prev2 exactly: each element is read, then
// written, by the same thread.
template <int ORDER>
__global__ void __launch_bounds__(kThreads) dpmpp_vec4(const float4* x, const float4* __restrict__ eu,
                                                       const float4* __restrict__ ec, const float4* dprev,
                                                       const float4* dprev2, float4* xo, float4* dout, int64_t n4,
                                                       Coef c) {
  sd::grid_dep_wait();
  sd::grid_dep_launch();
  const int64_t stride = static_cast<int64_t>(gridDim.x) * kThreads;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x; i < n4; i += stride) {
    const float4 a = ld_stream(x + i), u = ld_stream(eu + i), e = ld_stream(ec + i);
    const float4 p = ORDER >= 2 ? ld_stream(dprev + i) : make_float4(0.f, 0.f, 0.f, 0.f);
    const float4 q = ORDER == 3 ? ld_stream(dprev2 + i) : make_float4(0.f, 0.f, 0.f, 0.f);
    float4 r, d;
    step1<ORDER>(a.x, u.x, e.x, p.x, q.x, c, r.x, d.x);
    step1<ORDER>(a.y, u.y, e.y, p.y, q.y, c, r.y, d.y);
    step1<ORDER>(a.z, u.z, e.z, p.z, q.z, c, r.z, d.z);
    step1<ORDER>(a.w, u.w, e.w, p.w, q.w, c, r.w, d.w);
    st_stream(xo + i, r);
    st_stream(dout + i, d);
  }
}

// Scalar path: the tail that is not a whole float4, and inputs without 16-byte alignment.
template <int ORDER>
__global__ void __launch_bounds__(kThreads) dpmpp_scalar(const float* x, const float* __restrict__ eu,
                                                         const float* __restrict__ ec, const float* dprev,
                                                         const float* dprev2, float* xo, float* dout, int64_t n,
                                                         Coef c) {
  sd::grid_dep_wait();
  sd::grid_dep_launch();
  const int64_t stride = static_cast<int64_t>(gridDim.x) * kThreads;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x; i < n; i += stride) {
    float r, d;
    step1<ORDER>(x[i], eu[i], ec[i], ORDER >= 2 ? dprev[i] : 0.f, ORDER == 3 ? dprev2[i] : 0.f, c, r, d);
    xo[i] = r;
    dout[i] = d;
  }
}

int grid_for(int64_t items) {
  const int64_t cap = static_cast<int64_t>(sd::sm_count()) * 8;  // 8 resident 256-thread CTAs per SM
  int64_t g = (items + kThreads - 1) / kThreads;
  if (g > cap) g = cap;
  return static_cast<int>(g < 1 ? 1 : g);
}

template <class... P, class... A>
cudaError_t launch(int grid, cudaStream_t s, void (*kern)(P...), A... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(kThreads);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  cfg.attrs = attr;
  cfg.numAttrs = sd::pdl_attr(&attr[0]);
  return cudaLaunchKernelEx(&cfg, kern, static_cast<P>(args)...);
}

double lambda_of(double alpha_bar) { return 0.5 * std::log(alpha_bar / (1.0 - alpha_bar)); }

template <int ORDER>
sd_status run(const float* x, const float* eps_u, const float* eps_c, const float* d_prev, const float* d_prev2,
              float* x_out, float* d_out, int64_t n, const Coef& c, cudaStream_t s) {
  const bool vec = sd::aligned16(x) && sd::aligned16(eps_u) && sd::aligned16(eps_c) && sd::aligned16(x_out) &&
                   sd::aligned16(d_out) && (ORDER == 1 || sd::aligned16(d_prev)) &&
                   (ORDER < 3 || sd::aligned16(d_prev2));
  int64_t done = 0;
  if (vec && n >= 4) {
    const int64_t n4 = n / 4;
    const cudaError_t e = launch(grid_for(n4), s, dpmpp_vec4<ORDER>, reinterpret_cast<const float4*>(x),
                                 reinterpret_cast<const float4*>(eps_u), reinterpret_cast<const float4*>(eps_c),
                                 reinterpret_cast<const float4*>(d_prev), reinterpret_cast<const float4*>(d_prev2),
                                 reinterpret_cast<float4*>(x_out), reinterpret_cast<float4*>(d_out), n4, c);
    if (e != cudaSuccess) return sd::cuda_check(e, "DPM-Solver++ step launch");
    done = n4 * 4;
  }
  if (done < n)
    return sd::cuda_check(launch(grid_for(n - done), s, dpmpp_scalar<ORDER>, x + done, eps_u + done, eps_c + done,
                                 ORDER >= 2 ? d_prev + done : nullptr, ORDER == 3 ? d_prev2 + done : nullptr,
                                 x_out + done, d_out + done, n - done, c),
                          "DPM-Solver++ step launch");
  return SD_OK;
}

}  // namespace

extern "C" sd_status sd_cfg_dpmpp_2m_step(const float* x, const float* eps_u, const float* eps_c, const float* d_prev,
                                          float* x_out, float* d_out, int64_t n, float w, double alpha_prev,
                                          double alpha_t, double alpha_next, int order, void* stream) {
  const char* fn = "sd_cfg_dpmpp_2m_step";
  if (n < 0) return sd::fail(SD_ERR_INVALID_ARG, "%s: n < 0", fn);
  if (order != 1 && order != 2) return sd::fail(SD_ERR_INVALID_ARG, "%s: order must be 1 or 2", fn);
  if (!std::isfinite(w)) return sd::fail(SD_ERR_INVALID_ARG, "%s: w is not finite", fn);
  if (!(alpha_t > 0.0 && alpha_t < 1.0))
    return sd::fail(SD_ERR_INVALID_ARG, "%s: alpha_t must lie in (0, 1) (sigma_t > 0)", fn);
  if (!(alpha_next > 0.0 && alpha_next <= 1.0))
    return sd::fail(SD_ERR_INVALID_ARG, "%s: alpha_next must lie in (0, 1]", fn);
  if (order == 2) {
    if (!(alpha_prev > 0.0 && alpha_prev < 1.0))
      return sd::fail(SD_ERR_INVALID_ARG, "%s: alpha_prev must lie in (0, 1)", fn);
    if (alpha_next >= 1.0)
      return sd::fail(SD_ERR_INVALID_ARG, "%s: the step to alpha_bar = 1 (sigma = 0) is first order", fn);
    if (alpha_next == alpha_t || alpha_prev == alpha_t)
      return sd::fail(SD_ERR_INVALID_ARG, "%s: order 2 needs distinct alpha_prev, alpha_t, alpha_next", fn);
  }
  if (n == 0) return SD_OK;
  if (!x || !eps_u || !eps_c || !x_out || !d_out || (order == 2 && !d_prev))
    return sd::fail(SD_ERR_INVALID_ARG, "%s: null pointer", fn);
  const int64_t bytes = n * static_cast<int64_t>(sizeof(float));
  // x_out may equal x, d_out may equal d_prev; no other overlap among inputs and outputs.
  const bool bad_x = (x_out != x && sd::overlaps(x_out, bytes, x, bytes)) || sd::overlaps(x_out, bytes, eps_u, bytes) ||
                     sd::overlaps(x_out, bytes, eps_c, bytes) || sd::overlaps(x_out, bytes, d_out, bytes) ||
                     (order == 2 && sd::overlaps(x_out, bytes, d_prev, bytes));
  const bool bad_d = sd::overlaps(d_out, bytes, x, bytes) || sd::overlaps(d_out, bytes, eps_u, bytes) ||
                     sd::overlaps(d_out, bytes, eps_c, bytes) ||
                     (order == 2 && d_out != d_prev && sd::overlaps(d_out, bytes, d_prev, bytes));
  if (bad_x || bad_d)
    return sd::fail(SD_ERR_INVALID_ARG, "%s: outputs overlap inputs (only x_out == x and d_out == d_prev allowed)", fn);

  const double a_t = std::sqrt(alpha_t), s_t = std::sqrt(1.0 - alpha_t);
  const double a_n = std::sqrt(alpha_next), s_n = std::sqrt(1.0 - alpha_next);
  Coef c{w, static_cast<float>(1.0 / a_t), static_cast<float>(s_t / a_t), 0.f, 0.f, 0.f, 0.f};
  double B;
  if (alpha_next >= 1.0) {  // sigma_n = 0: exp(-h) = 0, x' = alpha_n D = D
    c.A = 0.f;
    B = a_n;
  } else {
    const double h = lambda_of(alpha_next) - lambda_of(alpha_t);
    c.A = static_cast<float>(s_n / s_t);
    B = -a_n * std::expm1(-h);
  }
  c.k0 = static_cast<float>(B);
  if (order == 2) {  // Dhat = (1 + 1/(2r)) D - 1/(2r) D_prev
    const double h = lambda_of(alpha_next) - lambda_of(alpha_t);
    const double r = (lambda_of(alpha_t) - lambda_of(alpha_prev)) / h;
    c.k0 = static_cast<float>(B * (1.0 + 0.5 / r));
    c.k1 = static_cast<float>(-B * 0.5 / r);
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return order == 2 ? run<2>(x, eps_u, eps_c, d_prev, nullptr, x_out, d_out, n, c, s)
                    : run<1>(x, eps_u, eps_c, d_prev, nullptr, x_out, d_out, n, c, s);
}

extern "C" sd_status sd_cfg_dpmpp_3m_step(const float* x, const float* eps_u, const float* eps_c,
                                          const float* d_prev, const float* d_prev2, float* x_out, float* d_out,
                                          int64_t n, float w, double alpha_prev2, double alpha_prev, double alpha_t,
                                          double alpha_next, void* stream) {
  const char* fn = "sd_cfg_dpmpp_3m_step";
  if (n < 0) return sd::fail(SD_ERR_INVALID_ARG, "%s: n < 0", fn);
  if (!std::isfinite(w)) return sd::fail(SD_ERR_INVALID_ARG, "%s: w is not finite", fn);
  for (double a : {alpha_prev2, alpha_prev, alpha_t})
    if (!(a > 0.0 && a < 1.0)) return sd::fail(SD_ERR_INVALID_ARG, "%s: alpha_prev2, alpha_prev, alpha_t must lie in (0, 1)", fn);
  if (!(alpha_next > 0.0 && alpha_next < 1.0))
    return sd::fail(SD_ERR_INVALID_ARG, "%s: alpha_next must lie in (0, 1) (the step to sigma = 0 is first order)", fn);
  const double l2 = lambda_of(alpha_prev2), l1 = lambda_of(alpha_prev), lt = lambda_of(alpha_t),
               ln = lambda_of(alpha_next);
  if (l2 == l1 || l1 == lt || lt == ln)
    return sd::fail(SD_ERR_INVALID_ARG, "%s: the four noise levels must be distinct", fn);
  if (n == 0) return SD_OK;
  if (!x || !eps_u || !eps_c || !d_prev || !d_prev2 || !x_out || !d_out)
    return sd::fail(SD_ERR_INVALID_ARG, "%s: null pointer", fn);
  const int64_t bytes = n * static_cast<int64_t>(sizeof(float));
  // x_out may equal x; d_out may equal d_prev or d_prev2 (the history rotates); nothing else overlaps.
  const bool bad_x = (x_out != x && sd::overlaps(x_out, bytes, x, bytes)) || sd::overlaps(x_out, bytes, eps_u, bytes) ||
                     sd::overlaps(x_out, bytes, eps_c, bytes) || sd::overlaps(x_out, bytes, d_out, bytes) ||
                     sd::overlaps(x_out, bytes, d_prev, bytes) || sd::overlaps(x_out, bytes, d_prev2, bytes);
  const bool bad_d = sd::overlaps(d_out, bytes, x, bytes) || sd::overlaps(d_out, bytes, eps_u, bytes) ||
                     sd::overlaps(d_out, bytes, eps_c, bytes) ||
                     (d_out != d_prev && sd::overlaps(d_out, bytes, d_prev, bytes)) ||
                     (d_out != d_prev2 && sd::overlaps(d_out, bytes, d_prev2, bytes));
  if (bad_x || bad_d)
    return sd::fail(SD_ERR_INVALID_ARG, "%s: outputs overlap inputs (only x_out == x, d_out == d_prev or d_prev2)", fn);
  // m0 = D, m1 = D_prev, m2 = D_prev2; D1 = h D' and D2 = h^2 D''/2 of the quadratic through them;
  // x' = (s_n/s_t) x + phi1 m0 + phi2 D1 + phi3 D2, folded into coefficients of m0, m1, m2.
  const double a_t = std::sqrt(alpha_t), s_t = std::sqrt(1.0 - alpha_t);
  const double a_n = std::sqrt(alpha_next), s_n = std::sqrt(1.0 - alpha_next);
  const double h = ln - lt, r0 = (lt - l1) / h, r1 = (l1 - l2) / h, em = std::expm1(-h);
  const double phi1 = -a_n * em, phi2 = a_n * (em / h + 1.0), phi3 = -2.0 * a_n * ((em + h) / (h * h) - 0.5);
  const double beta = r0 / (r0 + r1), gam = 1.0 / (r0 + r1);
  Coef c{w, static_cast<float>(1.0 / a_t), static_cast<float>(s_t / a_t), static_cast<float>(s_n / s_t),
         static_cast<float>(phi1 + phi2 * (1.0 + beta) / r0 + phi3 * gam / r0),
         static_cast<float>(-phi2 * ((1.0 + beta) / r0 + beta / r1) - phi3 * gam * (1.0 / r0 + 1.0 / r1)),
         static_cast<float>(phi2 * beta / r1 + phi3 * gam / r1)};
  return run<3>(x, eps_u, eps_c, d_prev, d_prev2, x_out, d_out, n, c, static_cast<cudaStream_t>(stream));
}
