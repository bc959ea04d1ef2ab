/*
 * sd_kernels.h -- C ABI of the latent-diffusion hot-path kernels for NVIDIA B200 (sm_100a).
 *
 * Three operations of one UNet denoising step, each an asynchronous launch on a caller stream:
 *
 *   sd_group_norm     GroupNorm of an NCHW fp32 activation (the reduction that feeds every UNet
 *                     block); sd_group_norm_silu fuses the SiLU that follows it.
 *   sd_attention      multi-head softmax(Q K^T * scale) V for the spatial-transformer blocks
 *                     (bf16; sd_attention_f16 takes fp16 tensors):
 *                     self-attention (K, V from the latent map, Lk = H*W) and cross-attention
 *                     (K, V from the projected 77-token text context).
 *   sd_cfg_ddim_step  classifier-free guidance fused with a deterministic DDIM latent update;
 *                     sd_cfg_dpmpp_2m_step fuses it with a DPM-Solver++(2M) update instead.
 *
 * Sources: "从零实现扩散模型推理引擎：Rust + wgpu 的 GPU 加速图像生成架构" (the Rust + wgpu engine page):
 * §1 sampling loop, §3.1 GroupNorm reduction, §3.2 flash cross-attention with online softmax, §4
 * scheduler step(model_output, timestep, sample, eta), §6 step_inplace, §7 CFG loop; and
 * "本地部署扩散模型架构与底层运行原理深度解析", section 示例说明 (guidance pseudo-code).
 *
 * Conventions for every entry point:
 *  - Pointers named x, y, q, k, v, o, eps_* are DEVICE pointers to contiguous row-major
 *    tensors owned by the caller; the library never frees, keeps or reallocates them.
 *  - `stream` is a cudaStream_t passed as void* (NULL = the legacy default stream). The call
 *    enqueues work and returns; results are ready when the stream reaches that point.
 *  - Argument errors are detected on the host, before anything is launched, and returned
 *    synchronously (SD_ERR_INVALID_ARG, SD_ERR_UNSUPPORTED, SD_ERR_MISALIGNED). A size of zero
 *    (empty tensor) returns SD_OK without a launch. A failed launch returns SD_ERR_CUDA; the
 *    CUDA error text is available from sd_last_error().
 *  - Device-side failures (a bounded wait inside a kernel that gave up) are recorded in a
 *    per-device status word and reported by sd_device_status(); kernels never trap.
 *  - Calls are thread-safe; each uses the device that is current on the calling thread.
 */
#ifndef SD_KERNELS_H
#define SD_KERNELS_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum sd_status {
  SD_OK = 0,
  SD_ERR_INVALID_ARG = 1,  /* null pointer, negative size, bad divisibility, partial overlap */
  SD_ERR_UNSUPPORTED = 2,  /* a size outside what the kernels implement (e.g. head dim)      */
  SD_ERR_MISALIGNED = 3,   /* a pointer that breaks a documented alignment rule             */
  SD_ERR_CUDA = 4,         /* a CUDA runtime call or launch failed; see sd_last_error()     */
  SD_ERR_TIMEOUT = 5       /* a kernel's bounded wait expired (reported by sd_device_status)*/
} sd_status;

/*
 * GroupNorm, "从零实现扩散模型推理引擎：Rust + wgpu 的 GPU 加速图像生成架构" §3.1: for each batch b and
 * group g (channels [g*C/G, (g+1)*C/G), all H*W positions: one contiguous span in NCHW),
 *   mean = sum/N, var = sum((x-mean)^2)/N (biased), rstd = 1/sqrt(var + eps),
 *   y[b,c,h,w] = (x[b,c,h,w] - mean) * rstd * gamma[c] + beta[c].
 *  x, y   : fp32 [B, C, H, W] contiguous. y may equal x exactly (in place); any other overlap
 *           is SD_ERR_INVALID_ARG.
 *  gamma, beta : fp32 [C].
 *  groups : must divide C (SD_ERR_INVALID_ARG otherwise); 32 in Stable Diffusion.
 *  eps    : > 0 and finite (1e-5 in Stable Diffusion).
 * Statistics are accumulated in fp32 with a pairwise (Chan et al.) merge. Groups of up to
 * 262144 elements and at most 128 channels, with H*W % 4 == 0 and 16-byte aligned x and y, are
 * read from HBM once (a thread-block cluster of up to 8 CTAs holds the group in registers); other
 * shapes take a streaming path of the same single launch that reads x twice. No global scratch
 * is used. The CTAs of a cluster exchange their partial statistics through distributed shared
 * memory; the wait for the peers' triples is bounded (about a second): should it expire, the
 * output is undefined and sd_device_status() reports SD_ERR_TIMEOUT.
 */
sd_status sd_group_norm(const float* x, const float* gamma, const float* beta, float* y,
                        int64_t B, int64_t C, int64_t H, int64_t W, int64_t groups, float eps,
                        void* stream);

/*
 * GroupNorm followed by SiLU in one launch: the GroupNorm + SiLU single-kernel fusion named in
 * "从零实现扩散模型推理引擎：Rust + wgpu 的 GPU 加速图像生成架构" §9 (the activation that follows GroupNorm
 * in the UNet's residual blocks). The page does not define SiLU; it is taken as
 *   y = v * sigmoid(v) = v / (1 + exp(-v)),  v = GroupNorm(x) as in sd_group_norm.
 *  x, gamma, beta, B..eps : as in sd_group_norm.
 *  y        : [B, C, H, W] contiguous, fp32 (out_bf16 = 0) or bf16 (out_bf16 = 1, round to nearest
 *             even), the input of the next convolution. With an fp32 output y may equal x (in
 *             place); a bf16 y must not overlap x. Other overlaps: SD_ERR_INVALID_ARG.
 *  out_bf16 : 0 or 1 (SD_ERR_INVALID_ARG otherwise).
 * Same statistics, paths and errors as sd_group_norm; a bf16 y takes the single-read path when it
 * is 8-byte aligned.
 */
sd_status sd_group_norm_silu(const float* x, const float* gamma, const float* beta, void* y,
                             int64_t B, int64_t C, int64_t H, int64_t W, int64_t groups, float eps,
                             int out_bf16, void* stream);

/*
 * Attention, "从零实现扩散模型推理引擎：Rust + wgpu 的 GPU 加速图像生成架构" §3.2: for each batch b, head h
 * and query row i, O[b,h,i,:] = sum_j softmax_j(scale * Q[b,h,i,:] . K[b,h,j,:]) V[b,h,j,:].
 * The kernel is a flash-style forward pass (tiles of 128 queries x 128 keys, running max and
 * running sum, normalisation at the end) on the sm_100a tensor cores with fp32 accumulation. For
 * Lk <= 80 (the 77-token text context) a second kernel keeps all of K and V resident in shared
 * memory and takes one exact softmax pass per 128-row query tile (§3.2's cross-attention).
 *  q      : bf16 [B, heads, Lq, dh] contiguous.
 *  k, v   : bf16 [B, heads, Lk, dh] contiguous (self-attention: Lk = Lq = H*W;
 *           cross-attention: Lk = 77 text tokens, already projected to heads x dh).
 *  o      : bf16 [B, heads, Lq, dh] contiguous; must not overlap q, k or v.
 *  dh     : one of 40, 64, 80, 160 (SD1.5 and SDXL head sizes); others are SD_ERR_UNSUPPORTED.
 *  scale  : finite and >= 0 (SD_ERR_INVALID_ARG if not finite, SD_ERR_UNSUPPORTED if negative);
 *           callers normally pass 1/sqrt(dh).
 *  Lq, Lk : >= 1 and <= 2^30, any value (ragged tails are masked). B*heads < 2^31.
 * All four pointers must be 16-byte aligned (SD_ERR_MISALIGNED otherwise).
 * Scratch: when a shape has more query-tile items than the GPU has SMs, some items are split
 * between two CTAs of the persistent grid, which hand partial results over through a per-device
 * workspace that the first such call allocates (cudaMalloc, about 50-100 KB per SM) and later calls
 * grow; sd_attention_noalloc avoids that allocation. The hand-off never waits for a CTA to be
 * scheduled, so the launch needs no particular number of free SMs; two launches that split items
 * must not run concurrently on one device (they share the workspace).
 */
sd_status sd_attention(const void* q, const void* k, const void* v, void* o,
                       int64_t B, int64_t heads, int64_t Lq, int64_t Lk, int64_t dh, float scale,
                       void* stream);

/*
 * sd_attention on IEEE fp16 tensors: the engine page's precision choice
 * ("从零实现扩散模型推理引擎：Rust + wgpu 的 GPU 加速图像生成架构" §5.2, Precision::Fp16, named as enough
 * for SD1.5/SDXL). q, k, v and o are fp16 [B, heads, L, dh]; everything else (arguments, layouts,
 * alignment, errors, scratch) is as in sd_attention. The tensor cores multiply fp16 by fp16 with
 * fp32 accumulation; P is rounded to fp16 for P V, and O is written as fp16 (round to nearest).
 */
sd_status sd_attention_f16(const void* q, const void* k, const void* v, void* o,
                           int64_t B, int64_t heads, int64_t Lq, int64_t Lk, int64_t dh, float scale,
                           void* stream);

/*
 * sd_attention with the element type and memory layout as arguments (an interface of this library:
 * the layout a fused QKV projection writes, read without a transpose).
 *  dtype  : 0 = bf16 (as sd_attention), 1 = fp16 (as sd_attention_f16).
 *  layout : 0 = [B, heads, L, dh] (as sd_attention);
 *           1 = [B, L, heads, dh] for q, k, v and o (heads interleaved in each row of the sequence;
 *           read through a 4-D TMA tensor map, O written in the same layout).
 * Other values of dtype or layout are SD_ERR_INVALID_ARG; everything else as in sd_attention.
 */
sd_status sd_attention_layout(const void* q, const void* k, const void* v, void* o,
                              int64_t B, int64_t heads, int64_t Lq, int64_t Lk, int64_t dh, float scale,
                              int dtype, int layout, void* stream);

/*
 * sd_attention_noalloc -- the same computation, arguments, layouts and errors as sd_attention, for
 * callers that cannot allocate device memory. (The source pages have no counterpart: this is an
 * interface of this library.)
 *
 * Why it exists: sd_attention allocates a scratch workspace with cudaMalloc the first time a shape
 * splits a query-tile item between two CTAs, and grows it when a later shape needs more. That is not
 * possible for every caller: code that is being captured into a CUDA graph may not call cudaMalloc,
 * a framework that owns all device memory through its own allocator may forbid outside
 * allocations, and a latency-critical loop cannot absorb the device synchronisation that
 * cudaMalloc and cudaFree imply. This entry point never calls cudaMalloc, cudaFree or any
 * allocating routine: its scratch is a 16 MiB file-scope device array that every GPU loading the
 * library holds until the process exits (enough for every head dim this library supports on up
 * to 148 SMs). A shape whose scratch would exceed 16 MiB is rejected with SD_ERR_UNSUPPORTED and
 * nothing is launched.
 *
 *  - Every call first looks up the array's device address on the current device
 *    (cudaGetSymbolAddress, cached per device and CUDA context, so a context created again after
 *    cudaDeviceReset is noticed); the first call on a device does the actual lookup, so make that
 *    first call before any stream capture on that device.
 *  - Every call uses the same array, which keeps the previous call's contents; each call clears
 *    the part that must start at zero with an asynchronous memset on `stream` before its kernel.
 *  - Calls whose executions overlap on the GPU (different streams, no ordering between them) race
 *    on the array and produce wrong results; order them on one stream or with events.
 */
sd_status sd_attention_noalloc(const void* q, const void* k, const void* v, void* o,
                               int64_t B, int64_t heads, int64_t Lq, int64_t Lk, int64_t dh, float scale,
                               void* stream);

/*
 * Guided DDIM step. Guidance from "从零实现扩散模型推理引擎：Rust + wgpu 的 GPU 加速图像生成架构" §7 and
 * "本地部署扩散模型架构与底层运行原理深度解析" (示例说明): g = eps_u + w * (eps_c - eps_u), where eps_u and
 * eps_c are the unconditional and conditional halves of the UNet output (batch order
 * [uncond, cond]). Sampler step (engine page §1 and §4, DDIM with eta = 0):
 *   x' = sqrt(alpha_prev) * (x - sqrt(1 - alpha_t) * g) / sqrt(alpha_t) + sqrt(1 - alpha_prev) * g
 * evaluated as x' = A*x + Bc*g with A = sqrt(alpha_prev/alpha_t) and
 * Bc = sqrt(1 - alpha_prev) - sqrt(alpha_prev (1 - alpha_t) / alpha_t), both formed in double on
 * the host; alpha_* are cumulative products (alpha-bar) in (0, 1].
 *  x, eps_u, eps_c, x_out : fp32, n elements each. x_out may equal x (the engine's in-place
 *           step); any other overlap of x_out with an input is SD_ERR_INVALID_ARG.
 * Any alignment is accepted; 16-byte aligned pointers take the vectorised path.
 */
sd_status sd_cfg_ddim_step(const float* x, const float* eps_u, const float* eps_c, float* x_out,
                           int64_t n, float w, double alpha_t, double alpha_prev, void* stream);

/*
 * Guided DPM-Solver++(2M) step. The engine page ("从零实现扩散模型推理引擎：Rust + wgpu 的 GPU 加速图像生成
 * 架构" §4) keeps a DPM-Solver++ scheduler (order 1 = DDIM-equivalent, order 2 from a sample history,
 * Karras sigmas, lower_order_final) without printing its update; this is the published
 * DPM-Solver++(2M) multistep method (Lu et al. 2022) on cumulative products alpha_bar:
 *   alpha = sqrt(alpha_bar), sigma = sqrt(1 - alpha_bar), lambda = log(alpha / sigma),
 *   g = eps_u + w (eps_c - eps_u),  D = (x - sigma_t g) / alpha_t,  h = lambda_next - lambda_t,
 *   order 1: x' = (sigma_next / sigma_t) x - alpha_next expm1(-h) D            (= the DDIM step)
 *   order 2: r = (lambda_t - lambda_prev) / h,
 *            x' = (sigma_next / sigma_t) x - alpha_next expm1(-h) ((1 + 1/(2r)) D - D_prev / (2r)).
 * The step to alpha_next = 1 (sigma = 0, the end of sampling) must be order 1 and returns D.
 *  x, eps_u, eps_c : fp32, n elements each (eps_* as in sd_cfg_ddim_step).
 *  d_prev : fp32 n elements, the previous step's D (order 2 only; may be NULL for order 1).
 *  x_out  : fp32 n, the new latent; may equal x.
 *  d_out  : fp32 n, this step's D (the history for the next step); may equal d_prev.
 *  alpha_t in (0, 1), alpha_next in (0, 1], alpha_prev in (0, 1) (order 2: distinct from alpha_t,
 *  and alpha_next != alpha_t); order is 1 or 2. Other values, a NULL d_prev for order 2 and any
 *  other overlap between outputs and inputs are SD_ERR_INVALID_ARG.
 * All coefficients are formed in double on the host. Any alignment is accepted; 16-byte aligned
 * pointers take the vectorised path.
 */
sd_status sd_cfg_dpmpp_2m_step(const float* x, const float* eps_u, const float* eps_c, const float* d_prev,
                               float* x_out, float* d_out, int64_t n, float w, double alpha_prev,
                               double alpha_t, double alpha_next, int order, void* stream);

/*
 * Guided third-order multistep DPM-Solver++ step (the engine page's order 3, §4). With
 * m0 = D = (x - sigma_t g) / alpha_t, m1 = d_prev (taken at alpha_prev), m2 = d_prev2 (at
 * alpha_prev2), h = lambda_next - lambda_t, r0 = (lambda_t - lambda_prev) / h,
 * r1 = (lambda_prev - lambda_prev2) / h:
 *   D1_0 = (m0 - m1) / r0, D1_1 = (m1 - m2) / r1,
 *   D1 = D1_0 + r0 / (r0 + r1) (D1_0 - D1_1), D2 = (D1_0 - D1_1) / (r0 + r1),
 *   x' = (sigma_next / sigma_t) x - alpha_next expm1(-h) m0 + alpha_next (expm1(-h) / h + 1) D1
 *        - 2 alpha_next ((expm1(-h) + h) / h^2 - 1/2) D2,
 * the exact exponential integral of the quadratic through (lambda, m) of the three steps.
 *  x, eps_u, eps_c, x_out : as in sd_cfg_dpmpp_2m_step.
 *  d_prev, d_prev2 : fp32 n, the data predictions of the previous two steps.
 *  d_out  : fp32 n, this step's D; may equal d_prev or d_prev2 (the caller rotates the history).
 *  alpha_prev2, alpha_prev, alpha_t, alpha_next : in (0, 1), pairwise distinct in lambda; the step
 *           to alpha_bar = 1 is first order (sd_cfg_dpmpp_2m_step with order 1).
 * Other values, NULL pointers and other overlaps are SD_ERR_INVALID_ARG.
 */
sd_status sd_cfg_dpmpp_3m_step(const float* x, const float* eps_u, const float* eps_c, const float* d_prev,
                               const float* d_prev2, float* x_out, float* d_out, int64_t n, float w,
                               double alpha_prev2, double alpha_prev, double alpha_t, double alpha_next,
                               void* stream);

/* Human-readable name of a status code (static string, never NULL). */
const char* sd_status_string(sd_status status);

/* Detail of the last error returned on the calling thread (static per-thread buffer). */
const char* sd_last_error(void);

/*
 * Synchronises `stream`, then reads the current device's status word. Returns SD_ERR_TIMEOUT if
 * any kernel of this library gave up a bounded wait since the last reset, SD_ERR_CUDA if the
 * synchronisation failed, SD_OK otherwise. reset != 0 clears the word afterwards; if a kernel had
 * given up, it also clears sd_attention's hand-off workspace on this device (an aborted launch may
 * have left split-item flags set).
 */
sd_status sd_device_status(void* stream, int reset);

/*
 * Test hook, pure host code: writes to out[0 .. grid] the unit boundaries that sd_attention's
 * persistent grid uses for `items` query-tile items of `nkv` K/V tiles on `grid` CTAs (CTA c owns
 * units [out[c], out[c+1])), with the schedule cost model of head dim `dh`. SD_ERR_INVALID_ARG if
 * items, nkv or grid is < 1, grid > 256, grid > items, or out is NULL.
 */
sd_status sd_debug_attention_ranges(int64_t items, int64_t nkv, int64_t grid, int64_t dh, int64_t* out);

/*
 * Test hook for the failure path: flags bit 0 makes every later sd_attention launch (any thread,
 * any device) skip loading its first V tile, so each CTA's bounded wait expires after about one
 * second, the CTA drains its own copies, frees its tensor memory and returns, and
 * sd_device_status() reports SD_ERR_TIMEOUT. Outputs of such launches are undefined. Bit 1 holds
 * back the tail piece of every item split between two CTAs by about 50 us before it claims the
 * hand-off slot, so that the head piece claims and publishes and the tail piece merges (the
 * results are unchanged). flags = 0 restores normal operation. Not for production use.
 */
void sd_debug_set_fault(int flags);

/* Library version, major*10000 + minor*100 + patch. */
int sd_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SD_KERNELS_H */
