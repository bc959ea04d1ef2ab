"""CPU oracle for the latent-diffusion hot path: TEST INFRASTRUCTURE ONLY.

Plain, slow, fp64 numpy restatements of what the CUDA library computes:

* ``attention``       softmax(Q K^T * scale) V per (batch, head)             -> oracle/attention.py
* ``group_norm``      per-group mean / biased variance, then per-channel affine -> oracle/group_norm.py
* ``group_norm_silu`` SiLU (v * sigmoid(v)) of the GroupNorm output            -> oracle/group_norm.py
* ``cfg_ddim_step``   classifier-free guidance followed by a deterministic DDIM update
                      (eta = 0), plus the scaled-linear noise schedule      -> oracle/ddim.py
* ``cfg_dpmpp_2m_step`` guidance followed by a DPM-Solver++(2M) multistep update, plus
                      Karras sigmas                                        -> oracle/dpmpp.py

Sources, cited in each function by page title and section:

* "从零实现扩散模型推理引擎：Rust + wgpu 的 GPU 加速图像生成架构" (ybb.press; the Rust + wgpu engine
  page): §1 (sampling loop with a DDIM step), §3.1 (GroupNorm reduction), §3.2 (flash
  cross-attention and its online-softmax recurrence), §4 (scheduler trait, alphas_cumprod,
  order 1 = DDIM), §7 (CFG loop, batch order [uncond, cond]).
* "本地部署扩散模型架构与底层运行原理深度解析" (cloud.baidu.com; the local-deployment page): section
  "示例说明" (denoising-loop pseudo-code with the guidance formula).

Only ``tests/``, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline / reference arm may
import this package. The CUDA library never calls it and shares no code with it. Every function is
pinned by ``tests/test_oracle_*.py`` against closed forms, invariants, hand-worked cases and
independent library routines; none is "parity unpinned".
"""
from .attention import attention, attention_rows, softmax_weights
from .group_norm import group_norm, group_norm_silu, group_stats, silu
from .ddim import (cfg, ddim_step, cfg_ddim_step, scaled_linear_betas, alphas_cumprod,
                   ddim_timesteps, ddim_schedule, cfg_ddim_loop)
from .dpmpp import (lam, data_prediction, dpmpp_2m_step, cfg_dpmpp_2m_step, dpmpp_3m_step, cfg_dpmpp_3m_step,
                    karras_sigmas, alpha_bar_of_sigma,
                    sd_sigma_range, dpmpp_2m_schedule, cfg_dpmpp_2m_loop, dpmpp_3m_schedule, cfg_dpmpp_3m_loop)

__all__ = ["attention", "attention_rows", "softmax_weights", "group_norm", "group_norm_silu", "group_stats",
           "silu", "cfg", "ddim_step", "cfg_ddim_step", "scaled_linear_betas", "alphas_cumprod", "ddim_timesteps",
           "ddim_schedule", "cfg_ddim_loop", "lam", "data_prediction", "dpmpp_2m_step", "cfg_dpmpp_2m_step",
           "dpmpp_3m_step", "cfg_dpmpp_3m_step", "karras_sigmas", "alpha_bar_of_sigma", "sd_sigma_range", "dpmpp_2m_schedule", "cfg_dpmpp_2m_loop",
           "dpmpp_3m_schedule", "cfg_dpmpp_3m_loop"]
