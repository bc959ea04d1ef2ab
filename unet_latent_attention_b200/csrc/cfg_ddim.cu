// Fused classifier-free guidance + deterministic DDIM latent update (sd_cfg_ddim_step).
//
// Guidance: g = eps_u + w (eps_c - eps_u) ("从零实现扩散模型推理引擎：Rust + wgpu 的 GPU 加速图像生成架构" §7;
// "本地部署扩散模型架构与底层运行原理深度解析", 示例说明). DDIM with eta = 0 (engine page §1, §4):
// x' = sqrt(a_prev) (x - sqrt(1 - a_t) g) / sqrt(a_t) + sqrt(1 - a_prev) g, folded on the host into
// x' = A x + Bc g. Per element: three fp32 loads, one store (16 bytes), two FMAs and a multiply.
// HBM-bound: one pass, 16-byte vector accesses, a grid of a few waves over all SMs with a
// grid-stride loop, streaming cache hints (every byte is touched once).
#include <cmath>

#include "sd_internal.h"

namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ float4 ld_stream(const float4* p) {
  float4 v;
  asm volatile("ld.global.cs.v4.f32 {%0,%1,%2,%3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "l"(p));
  return v;
}

__device__ __forceinline__ void st_stream(float4* p, float4 v) {
  asm volatile("st.global.cs.v4.f32 [%0], {%1,%2,%3,%4};" :: "l"(p), "f"(v.x), "f"(v.y), "f"(v.z), "f"(v.w)
               : "memory");
}

__device__ __forceinline__ float guided_step(float x, float eu, float ec, float w, float A, float Bc) {
  const float g = fmaf(w, ec - eu, eu);
  return fmaf(A, x, Bc * g);
}

// x_out may alias x exactly: each element is read and then written by the same thread.
__global__ void __launch_bounds__(kThreads) cfg_ddim_vec4(const float4* x, const float4* __restrict__ eu,
                                                          const float4* __restrict__ ec, float4* xo,
                                                          int64_t n4, float w, float A, float Bc) {
  sd::grid_dep_wait();
  sd::grid_dep_launch();
  const int64_t stride = static_cast<int64_t>(gridDim.x) * kThreads;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x; i < n4; i += stride) {
    const float4 a = ld_stream(x + i), u = ld_stream(eu + i), c = ld_stream(ec + i);
    float4 r;
    r.x = guided_step(a.x, u.x, c.x, w, A, Bc);
    r.y = guided_step(a.y, u.y, c.y, w, A, Bc);
    r.z = guided_step(a.z, u.z, c.z, w, A, Bc);
    r.w = guided_step(a.w, u.w, c.w, w, A, Bc);
    st_stream(xo + i, r);
  }
}

// Scalar path: the tail that is not a whole float4, and inputs without 16-byte alignment.
__global__ void __launch_bounds__(kThreads) cfg_ddim_scalar(const float* x, const float* __restrict__ eu,
                                                            const float* __restrict__ ec, float* xo,
                                                            int64_t n, float w, float A, float Bc) {
  sd::grid_dep_wait();
  sd::grid_dep_launch();
  const int64_t stride = static_cast<int64_t>(gridDim.x) * kThreads;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x; i < n; i += stride)
    xo[i] = guided_step(x[i], eu[i], ec[i], w, A, Bc);
}

int grid_for(int64_t items) {
  const int64_t cap = static_cast<int64_t>(sd::sm_count()) * 8;  // 8 resident 256-thread CTAs per SM
  int64_t g = (items + kThreads - 1) / kThreads;
  if (g > cap) g = cap;
  return static_cast<int>(g < 1 ? 1 : g);
}

// Launch with programmatic stream serialization (see sd_internal.h).
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

}  // namespace

extern "C" sd_status sd_cfg_ddim_step(const float* x, const float* eps_u, const float* eps_c, float* x_out,
                                      int64_t n, float w, double alpha_t, double alpha_prev, void* stream) {
  if (n < 0) return sd::fail(SD_ERR_INVALID_ARG, "sd_cfg_ddim_step: n < 0");
  if (!std::isfinite(w)) return sd::fail(SD_ERR_INVALID_ARG, "sd_cfg_ddim_step: w is not finite");
  if (!(alpha_t > 0.0 && alpha_t <= 1.0) || !(alpha_prev > 0.0 && alpha_prev <= 1.0))
    return sd::fail(SD_ERR_INVALID_ARG, "sd_cfg_ddim_step: alpha_t and alpha_prev must lie in (0, 1]");
  if (n == 0) return SD_OK;
  if (!x || !eps_u || !eps_c || !x_out) return sd::fail(SD_ERR_INVALID_ARG, "sd_cfg_ddim_step: null pointer");
  const int64_t bytes = n * static_cast<int64_t>(sizeof(float));
  if ((x_out != x && sd::overlaps(x_out, bytes, x, bytes)) || sd::overlaps(x_out, bytes, eps_u, bytes) ||
      sd::overlaps(x_out, bytes, eps_c, bytes))
    return sd::fail(SD_ERR_INVALID_ARG, "sd_cfg_ddim_step: x_out overlaps an input (only x_out == x is allowed)");

  // x' = A x + Bc g, A = sqrt(a_prev / a_t), Bc = sqrt(1 - a_prev) - sqrt(a_prev (1 - a_t) / a_t)
  const double A = std::sqrt(alpha_prev / alpha_t);
  const double Bc = std::sqrt(1.0 - alpha_prev) - std::sqrt(alpha_prev * (1.0 - alpha_t) / alpha_t);
  cudaStream_t s = static_cast<cudaStream_t>(stream);

  const bool vec = sd::aligned16(x) && sd::aligned16(eps_u) && sd::aligned16(eps_c) && sd::aligned16(x_out);
  int64_t done = 0;
  if (vec && n >= 4) {
    const int64_t n4 = n / 4;
    cudaError_t e = launch(grid_for(n4), s, cfg_ddim_vec4, reinterpret_cast<const float4*>(x),
                           reinterpret_cast<const float4*>(eps_u), reinterpret_cast<const float4*>(eps_c),
                           reinterpret_cast<float4*>(x_out), n4, w, static_cast<float>(A), static_cast<float>(Bc));
    if (e != cudaSuccess) return sd::cuda_check(e, "sd_cfg_ddim_step launch");
    done = n4 * 4;
  }
  if (done < n) {
    const int64_t rest = n - done;
    return sd::cuda_check(launch(grid_for(rest), s, cfg_ddim_scalar, x + done, eps_u + done, eps_c + done,
                                 x_out + done, rest, w, static_cast<float>(A), static_cast<float>(Bc)),
                          "sd_cfg_ddim_step launch");
  }
  return SD_OK;
}
