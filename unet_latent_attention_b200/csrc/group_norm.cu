// GroupNorm over NCHW fp32 (sd_group_norm).
//
// "从零实现扩散模型推理引擎：Rust + wgpu 的 GPU 加速图像生成架构" §3.1 reduces a group to its sum and sum of
// squares with a 256-wide workgroup tree, then mean = sum/N, var = sumsq/N - mean^2 (biased) and
// inv_std = 1/sqrt(var + eps); the page elides the normalise/affine tail. Here:
//
//  * A group (C/G channels x H*W, one contiguous span in NCHW) is split over a thread-block
//    cluster of up to 8 CTAs. Each thread loads its part of the group into registers with 16-byte
//    streaming loads, so HBM is read exactly once (the resident path).
//  * Statistics stay in fp32 but are merged as (count, mean, M2) triples with the pairwise update
//    of Chan, Golub and LeVeque (1979) instead of sum / sum-of-squares, which cancels when
//    |mean| >> std. Resident path with clusters of up to 4 CTAs: warp shuffles, then every warp
//    sends its triple into every cluster peer's shared memory with st.async, counted on the peer's
//    mbarrier (no cluster-wide barrier on the critical path); clusters of 8 and the streaming
//    path: shared memory across warps, then one push per CTA into distributed shared memory behind
//    one cluster barrier. Every CTA of a cluster merges the triples in one fixed order, so all of
//    them obtain bit-identical statistics.
//  * The tail is fused: y = x * a_c + b_c with a_c = rstd * gamma[c], b_c = beta[c] - mean * a_c.
//    sd_group_norm_silu adds the SiLU activation, v * sigmoid(v), that follows GroupNorm in the
//    UNet's residual blocks (the page's GroupNorm + SiLU single-kernel fusion, §9), with an fp32 or
//    bf16 output.
//
// Shapes the resident path cannot hold (groups above 8 x 32768 elements, more than 128 channels per
// group, H*W not a multiple of 4, pointers not 16-byte aligned) take the streaming path: the same cluster merge, but each CTA
// sweeps its part twice (statistics, then normalise), so x is read twice (the second time mostly
// from L2). Neither path uses global scratch memory.
#include <cooperative_groups.h>
#include <cuda_bf16.h>

#include <cmath>

#include "sd_internal.h"

namespace cg = cooperative_groups;

namespace {

constexpr int kThreads = 256;  // streaming path
constexpr int kMaxGroupChannels = 128;  // resident path: channels per group staged in shared memory
constexpr int kMaxCluster = 8;
constexpr int kMaxItems = 16;  // float4 per thread on the resident path

#ifndef SD_GN_POLICY
#define SD_GN_POLICY 0
#endif

// ---------------------------------------------------------------- cluster exchange primitives
__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
// The same shared-memory offset in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t peer_addr(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}
// 16-byte store into a peer's shared memory that counts its bytes on the peer's mbarrier.
__device__ __forceinline__ void st_async_peer(uint32_t dst, float4 v, uint32_t peer_bar) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.f32 [%0], {%1, %2, %3, %4}, [%5];"
               :: "r"(dst), "f"(v.x), "f"(v.y), "f"(v.z), "f"(v.w), "r"(peer_bar) : "memory");
}
__device__ __forceinline__ void cluster_arrive_release() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait_acquire() {
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ void bar_init_expect(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" :: "r"(bar) : "memory");
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}"
               :: "r"(bar), "r"(bytes) : "memory");
}
// Waits (acquire, cluster scope) for phase 0 of `bar`; gives up after about a second and reports a
// timeout in the status word instead of hanging.
__device__ __forceinline__ void bar_wait_cluster(uint32_t bar, unsigned int* err) {
  const long long t0 = clock64();
  for (uint32_t it = 0;; ++it) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], 0;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok) : "r"(bar) : "memory");
    if (ok) return;
    if ((it & 63u) == 63u && clock64() - t0 > 2000000000LL) {
      atomicOr(err, sd::kDevErrTimeout);
      return;
    }
  }
}


struct Stats {
  float n, mean, m2;
};

// Chan et al. pairwise merge of two (count, mean, sum of squared deviations) triples.
__device__ __forceinline__ Stats merge(Stats a, Stats b) {
  const float n = a.n + b.n;
  if (n == 0.f) return a;
  const float d = b.mean - a.mean;
  const float fb = b.n / n;
  return Stats{n, fmaf(d, fb, a.mean), a.m2 + b.m2 + d * d * a.n * fb};
}

__device__ __forceinline__ Stats shfl_down(Stats s, int off) {
  return Stats{__shfl_down_sync(0xffffffffu, s.n, off), __shfl_down_sync(0xffffffffu, s.mean, off),
               __shfl_down_sync(0xffffffffu, s.m2, off)};
}

// The same merge with the approximate division (2 ulp): on the resident path's critical chain
// (the statistics are complete only when the last of a cluster's loads lands, and the stores wait
// for them), so its latency matters more than the last bit of the weight.
__device__ __forceinline__ Stats merge_fast(Stats a, Stats b) {
  const float n = a.n + b.n;
  if (n == 0.f) return a;
  const float d = b.mean - a.mean;
  const float fb = __fdividef(b.n, n);
  return Stats{n, fmaf(d, fb, a.mean), a.m2 + b.m2 + d * d * a.n * fb};
}

// Merges the triples of lanes [0, n) (n a power of two, at most 32) toward lane 0 in a fixed tree
// and returns lane 0's result in every lane: every warp that runs it on the same inputs gets the
// same bits.
__device__ __forceinline__ Stats warp_tree_merge(Stats st, int n) {
  const int lane = threadIdx.x & 31;
  for (int off = n >> 1; off > 0; off >>= 1) {
    const Stats o = shfl_down(st, off);
    if (lane + off < n) st = merge_fast(st, o);
  }
  return Stats{__shfl_sync(0xffffffffu, st.n, 0), __shfl_sync(0xffffffffu, st.mean, 0),
               __shfl_sync(0xffffffffu, st.m2, 0)};
}

// Exact statistics of four values (two sweeps over registers).
__device__ __forceinline__ Stats stats4(float4 v, float n) {
  if (n == 0.f) return Stats{0.f, 0.f, 0.f};
  const float mean = (v.x + v.y + v.z + v.w) * 0.25f;
  const float a = v.x - mean, b = v.y - mean, c = v.z - mean, d = v.w - mean;
  return Stats{4.f, mean, a * a + b * b + c * c + d * d};
}

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

// Epilogues: the affine output in fp32 (sd_group_norm), or SiLU of it in fp32 or bf16.
enum Epi : int { kAffine = 0, kSiluF32 = 1, kSiluBf16 = 2 };

// v * sigmoid(v). The division is the approximate one (reciprocal then multiply, 2 ulp): exact
// IEEE division made the fused kernel compute-bound. For v < -88, 1 + exp(-v) is +inf and the
// result is -0.
__device__ __forceinline__ float silu(float v) { return __fdividef(v, 1.0f + __expf(-v)); }

// Stores four consecutive outputs (element index 4 * i4 of y).
template <int EPI>
__device__ __forceinline__ void store4(void* y, int64_t i4, float4 v) {
  if constexpr (EPI != kAffine) v = make_float4(silu(v.x), silu(v.y), silu(v.z), silu(v.w));
  if constexpr (EPI == kSiluBf16) {
    const __nv_bfloat162 lo = __floats2bfloat162_rn(v.x, v.y), hi = __floats2bfloat162_rn(v.z, v.w);
    uint2 u;
    u.x = *reinterpret_cast<const uint32_t*>(&lo);
    u.y = *reinterpret_cast<const uint32_t*>(&hi);
    asm volatile("st.global.cs.v2.b32 [%0], {%1,%2};" :: "l"(reinterpret_cast<uint2*>(y) + i4), "r"(u.x), "r"(u.y)
                 : "memory");
  } else {
    st_stream(reinterpret_cast<float4*>(y) + i4, v);
  }
}

template <int EPI>
__device__ __forceinline__ void store1(void* y, int64_t i, float v) {
  if constexpr (EPI != kAffine) v = silu(v);
  if constexpr (EPI == kSiluBf16) reinterpret_cast<__nv_bfloat16*>(y)[i] = __float2bfloat16_rn(v);
  else reinterpret_cast<float*>(y)[i] = v;
}

// Reduces the thread's triple over the CTA, pushes the CTA's triple into slot `rank` of every
// cluster peer's shared memory, and after one cluster barrier merges the slots in rank order, so
// that every CTA obtains the same mean and rstd (left in shared memory). No CTA touches another's
// shared memory after the barrier, so CTAs may exit without a second cluster-wide sync.
__device__ __forceinline__ void cluster_group_stats(Stats st, float eps, float* s_mean, float* s_rstd,
                                                    Stats* s_warp, Stats* s_all) {
  cg::cluster_group cluster = cg::this_cluster();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    const Stats o = shfl_down(st, off);
    if (lane + off < 32) st = merge(st, o);
  }
  if (lane == 0) s_warp[warp] = st;
  __syncthreads();
  const unsigned cs = cluster.num_blocks();
  if (threadIdx.x == 0) {
    Stats a = s_warp[0];
    const int nw = blockDim.x >> 5;
    for (int w = 1; w < nw; ++w) a = merge(a, s_warp[w]);
    const unsigned rank = cluster.block_rank();
    for (unsigned r = 0; r < cs; ++r) *cluster.map_shared_rank(&s_all[rank], r) = a;
  }
  cluster.sync();  // release/acquire: every peer's slot write is visible
  if (threadIdx.x == 0) {
    Stats a = s_all[0];
    for (unsigned r = 1; r < cs; ++r) a = merge(a, s_all[r]);
    const float var = a.n > 0.f ? fmaxf(a.m2 / a.n, 0.f) : 0.f;
    *s_mean = a.mean;
    *s_rstd = rsqrtf(var + eps);
  }
  __syncthreads();
}

// Resident path's statistics, then the per-channel affine of the group: the thread's triple is
// merged over its warp (shuffles), the warps' triples by warp 0 (one shuffle tree), and warp 0's
// lanes push the CTA's triple into slot `rank` of every peer's shared memory at once; after one
// cluster barrier warp 0 merges the slots in a fixed tree (so every CTA of the cluster obtains the
// same bits) and writes a_c = rstd * gamma_c and b_c = beta_c - mean * a_c for the group's cpg
// channels (gamma and beta already staged in s_a / s_b) into shared memory.
__device__ __forceinline__ void cluster_group_affine(Stats st, float eps, int cpg, float* s_a, float* s_b,
                                                     Stats* s_warp, Stats* s_all) {
  cg::cluster_group cluster = cg::this_cluster();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    const Stats o = shfl_down(st, off);
    if (lane + off < 32) st = merge_fast(st, o);
  }
  if (lane == 0) s_warp[warp] = st;
  __syncthreads();
  const int cs = static_cast<int>(cluster.num_blocks());
  if (warp == 0) {
    const int nw = blockDim.x >> 5;  // 8, 16 or 32
    const Stats a = warp_tree_merge(lane < nw ? s_warp[lane] : Stats{0.f, 0.f, 0.f}, nw);
    if (lane < cs) *cluster.map_shared_rank(&s_all[cluster.block_rank()], lane) = a;
  }
  cluster.sync();  // release/acquire: every peer's slot write is visible
  if (warp == 0) {
    const Stats a = warp_tree_merge(lane < cs ? s_all[lane] : Stats{0.f, 0.f, 0.f}, cs);
    const float var = a.n > 0.f ? fmaxf(a.m2 / a.n, 0.f) : 0.f;
    const float rstd = rsqrtf(var + eps);
    for (int c = lane; c < cpg; c += 32) {
      const float ac = rstd * s_a[c];
      s_b[c] = fmaf(-a.mean, ac, s_b[c]);
      s_a[c] = ac;
    }
  }
  __syncthreads();
}

// Resident path's statistics without a cluster barrier: each warp merges its threads' triples
// (shuffles) and sends the warp's triple, by st.async, into slot (rank, warp) of every peer's
// shared memory, where the bytes complete the peer's mbarrier (armed for cs x nw slots before the
// cluster's arrive at kernel start). Warp 0 waits for its own barrier, merges the cs x nw slots in
// one fixed order (every CTA obtains the same bits) and writes a_c = rstd * gamma_c and
// b_c = beta_c - mean * a_c for the group's cpg channels. A CTA receives no slot after its wait,
// so CTAs may exit without a second cluster-wide sync.
template <int NW>
__device__ __forceinline__ void cluster_group_affine_async(Stats st, float eps, int cpg, float* s_a, float* s_b,
                                                           float4* s_part, uint32_t bar, unsigned int* err) {
  cg::cluster_group cluster = cg::this_cluster();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int cs = static_cast<int>(cluster.num_blocks()), rank = static_cast<int>(cluster.block_rank());
  const Stats w = warp_tree_merge(st, 32);
  cluster_wait_acquire();  // every peer's barrier is armed
  if (lane < cs)
    st_async_peer(peer_addr(smem_addr(&s_part[rank * NW + warp]), lane), make_float4(w.n, w.mean, w.m2, 0.f),
                  peer_addr(bar, lane));
  if (warp == 0) {
    bar_wait_cluster(bar, err);
    Stats a{0.f, 0.f, 0.f};
    for (int k = lane; k < cs * NW; k += 32) {
      const float4 p = s_part[k];
      a = merge_fast(a, Stats{p.x, p.y, p.z});
    }
    a = warp_tree_merge(a, 32);
    const float var = a.n > 0.f ? fmaxf(a.m2 / a.n, 0.f) : 0.f;
    const float rstd = rsqrtf(var + eps);
    for (int c = lane; c < cpg; c += 32) {
      const float ac = rstd * s_a[c];
      s_b[c] = fmaf(-a.mean, ac, s_b[c]);
      s_a[c] = ac;
    }
  }
  __syncthreads();
}

// Resident path: one cluster of `cs` CTAs per (b, g); CTA `rank` owns elements
// [rank*chunk, (rank+1)*chunk) of the group, chunk a multiple of 4, held in registers.
// 512-thread CTAs with up to 10 float4 per thread are compiled for 2 resident CTAs per SM (64
// registers). Otherwise one such CTA fills an SM, clusters of 8 then fit twice per GPC, and the
// SDXL-sized groups (10 x 16384 elements) run in about four waves: measured 37.5 -> 24.1 us on
// [2, 320, 128, 128].
#ifndef SD_GN_MINB
#define SD_GN_MINB 1
#endif

// Resident CTAs per SM the register budget is compiled for: enough CTAs in flight to cover the
// load latency (256-thread CTAs: 4 with at most 5 float4 per thread, 3 with at most 10).
constexpr int gn_min_blocks(int items, int threads) {
  return threads == 512 ? ((SD_GN_MINB && items <= 10) ? 2 : 1)
                        : threads == 256 ? (items <= 5 ? 4 : items <= 10 ? 3 : 1) : 1;
}

// XCHG selects the statistics exchange: per-warp st.async into every peer (measured faster with
// clusters of up to 4 CTAs) or one push per CTA and a cluster barrier (faster with clusters of 8:
// [8,320,96,96] 52.1 -> 47.5 us, [16,320,128,128] 125.6 -> 124.2 us).
template <int ITEMS, int THREADS, int EPI, bool XCHG>
__global__ void __launch_bounds__(THREADS, gn_min_blocks(ITEMS, THREADS)) gn_resident(const float* x, const float* __restrict__ gamma,
                                                        const float* __restrict__ beta, void* y,
                                                        int group_elems, int chunk, int hw, int cpg, int groups,
                                                        float eps, unsigned int* err) {
  __shared__ float s_a[kMaxGroupChannels], s_b[kMaxGroupChannels];
  __shared__ float4 s_part[XCHG ? kMaxCluster * (THREADS / 32) : 1];
  __shared__ Stats s_warp[XCHG ? 1 : THREADS / 32];
  __shared__ Stats s_all[XCHG ? 1 : kMaxCluster];
  __shared__ uint64_t s_bar;
  cg::cluster_group cluster = cg::this_cluster();
  if constexpr (XCHG) {
    // Shared memory only, so it may overlap the previous kernel: arm the barrier that counts the
    // cluster's cs x nw incoming triples, then tell the peers it is armed.
    if (threadIdx.x == 0)
      bar_init_expect(smem_addr(&s_bar), static_cast<uint32_t>(cluster.num_blocks() * (THREADS / 32) * sizeof(float4)));
    cluster_arrive_release();
  }
  sd::grid_dep_wait();
  sd::grid_dep_launch();
  const int rank = static_cast<int>(cluster.block_rank());
  const int64_t grp = blockIdx.x / cluster.num_blocks();  // b * groups + g
  const int g = static_cast<int>(grp % groups);
  const int64_t base = grp * group_elems + static_cast<int64_t>(rank) * chunk;
  const float4* xg = reinterpret_cast<const float4*>(x + base);
  const int n4 = chunk >> 2;

  float4 v[ITEMS];
#pragma unroll
  for (int i = 0; i < ITEMS; ++i) {
    const int idx = threadIdx.x + i * THREADS;
    v[i] = idx < n4 ? ld_stream(xg + idx) : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  // the group's gamma and beta, staged while the loads above are in flight
  for (int c = threadIdx.x; c < cpg; c += THREADS) {
    s_a[c] = __ldg(gamma + g * cpg + c);
    s_b[c] = __ldg(beta + g * cpg + c);
  }
  // Thread triple: exact mean of its values, then M2 about it.
  float sum = 0.f, cnt = 0.f;
#pragma unroll
  for (int i = 0; i < ITEMS; ++i) {
    if (threadIdx.x + i * THREADS < n4) {
      sum += (v[i].x + v[i].y) + (v[i].z + v[i].w);
      cnt += 4.f;
    }
  }
  Stats st{cnt, cnt > 0.f ? sum / cnt : 0.f, 0.f};
#pragma unroll
  for (int i = 0; i < ITEMS; ++i) {
    if (threadIdx.x + i * THREADS < n4) {
      const float a = v[i].x - st.mean, b = v[i].y - st.mean, c = v[i].z - st.mean, d = v[i].w - st.mean;
      st.m2 += a * a + b * b + c * c + d * d;
    }
  }
  if constexpr (XCHG) cluster_group_affine_async<THREADS / 32>(st, eps, cpg, s_a, s_b, s_part, smem_addr(&s_bar), err);
  else cluster_group_affine(st, eps, cpg, s_a, s_b, s_warp, s_all);

  const int64_t base4 = base >> 2;  // base is a multiple of 4 (chunk and group_elems are)
  // Channel (within the group) of this thread's item i, element rank * chunk + 4 (tid + i THREADS):
  // one division here, then a step of 4 THREADS elements per item (hw % 4 == 0: a float4 never
  // straddles channels).
  const int e_first = rank * chunk + 4 * static_cast<int>(threadIdx.x);
  int ch = e_first / hw, rem = e_first - ch * hw;
  const int step_c = 4 * THREADS / hw, step_r = 4 * THREADS - step_c * hw;
#pragma unroll
  for (int i = 0; i < ITEMS; ++i) {
    const int idx = threadIdx.x + i * THREADS;
    if (idx < n4) {
      const float a = s_a[ch], b = s_b[ch];
      store4<EPI>(y, base4 + idx, make_float4(fmaf(v[i].x, a, b), fmaf(v[i].y, a, b), fmaf(v[i].z, a, b),
                                              fmaf(v[i].w, a, b)));
    }
    ch += step_c;
    rem += step_r;
    if (rem >= hw) {
      rem -= hw;
      ++ch;
    }
  }
}

// Streaming path: any shape and alignment. CTA `rank` of the cluster owns elements [lo, hi) of the
// group; sweep 1 builds the triple (exact stats of each run of four values, merged pairwise),
// sweep 2 normalises.
template <int EPI>
__global__ void __launch_bounds__(kThreads) gn_streaming(const float* x, const float* __restrict__ gamma,
                                                         const float* __restrict__ beta, void* y,
                                                         int64_t group_elems, int64_t chunk, int64_t hw, int cpg,
                                                         int groups, float eps) {
  __shared__ Stats s_warp[kThreads / 32];
  __shared__ Stats s_all[kMaxCluster];
  __shared__ float s_mean, s_rstd;
  sd::grid_dep_wait();
  sd::grid_dep_launch();
  cg::cluster_group cluster = cg::this_cluster();
  const int64_t rank = cluster.block_rank();
  const int64_t grp = blockIdx.x / cluster.num_blocks();
  const int g = static_cast<int>(grp % groups);
  const int64_t lo = rank * chunk;
  const int64_t hi = lo + chunk < group_elems ? lo + chunk : group_elems;
  const float* xg = x + grp * group_elems;
  const int64_t y0 = grp * group_elems;

  Stats st{0.f, 0.f, 0.f};
  for (int64_t e = lo + 4 * threadIdx.x; e < hi; e += 4 * kThreads) {
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    const int64_t m = hi - e < 4 ? hi - e : 4;
    v.x = xg[e];
    if (m > 1) v.y = xg[e + 1];
    if (m > 2) v.z = xg[e + 2];
    if (m > 3) v.w = xg[e + 3];
    Stats r;
    if (m == 4) {
      r = stats4(v, 4.f);
    } else {  // ragged tail of the part: exact stats of m values
      float s = v.x + (m > 1 ? v.y : 0.f) + (m > 2 ? v.z : 0.f);
      const float mu = s / static_cast<float>(m);
      float q = (v.x - mu) * (v.x - mu);
      if (m > 1) q += (v.y - mu) * (v.y - mu);
      if (m > 2) q += (v.z - mu) * (v.z - mu);
      r = Stats{static_cast<float>(m), mu, q};
    }
    st = merge(st, r);
  }
  cluster_group_stats(st, eps, &s_mean, &s_rstd, s_warp, s_all);
  const float mean = s_mean, rstd = s_rstd;
  for (int64_t e = lo + threadIdx.x; e < hi; e += kThreads) {
    const int c = g * cpg + static_cast<int>(e / hw);
    const float a = rstd * __ldg(gamma + c);
    store1<EPI>(y, y0 + e, fmaf(xg[e], a, fmaf(-mean, a, __ldg(beta + c))));
  }
}

template <int ITEMS, int THREADS, int EPI>
cudaError_t launch_resident(dim3 grid, int cs, cudaStream_t s, const float* x, const float* gamma,
                            const float* beta, void* y, int group_elems, int chunk, int hw, int cpg, int groups,
                            float eps) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(THREADS);
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = cs;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1 + sd::pdl_attr(&attr[1]);
  unsigned int* err = sd::device_status_word();
  if (!err) return cudaErrorUnknown;
  if (cs <= 4)
    return cudaLaunchKernelEx(&cfg, gn_resident<ITEMS, THREADS, EPI, true>, x, gamma, beta, y, group_elems, chunk, hw,
                              cpg, groups, eps, err);
  return cudaLaunchKernelEx(&cfg, gn_resident<ITEMS, THREADS, EPI, false>, x, gamma, beta, y, group_elems, chunk, hw,
                            cpg, groups, eps, err);
}

// One GroupNorm launch with epilogue EPI; `name` prefixes error messages.
template <int EPI>
sd_status group_norm_impl(const char* name, const float* x, const float* gamma, const float* beta, void* y, int64_t B,
                          int64_t C, int64_t H, int64_t W, int64_t groups, float eps, void* stream) {
  if (B < 0 || C < 0 || H < 0 || W < 0) return sd::fail(SD_ERR_INVALID_ARG, "%s: negative size", name);
  if (groups <= 0 || (C > 0 && C % groups != 0))
    return sd::fail(SD_ERR_INVALID_ARG, "%s: groups must be positive and divide C", name);
  if (!(eps > 0.f) || !std::isfinite(eps)) return sd::fail(SD_ERR_INVALID_ARG, "%s: eps must be > 0", name);
  if (B == 0 || C == 0 || H == 0 || W == 0) return SD_OK;
  if (!x || !gamma || !beta || !y) return sd::fail(SD_ERR_INVALID_ARG, "%s: null pointer", name);
  const int64_t hw = H * W;
  const int64_t cpg = C / groups;
  const int64_t group_elems = cpg * hw;
  const int64_t n_groups = B * groups;
  if (group_elems > (int64_t(1) << 31) - 1 || n_groups * kMaxCluster > 0x7fffffff)
    return sd::fail(SD_ERR_UNSUPPORTED, "%s: tensor too large", name);
  constexpr int64_t kOutBytes = EPI == kSiluBf16 ? 2 : 4;
  const int64_t xbytes = B * C * hw * static_cast<int64_t>(sizeof(float)), ybytes = B * C * hw * kOutBytes;
  const int64_t pbytes = C * static_cast<int64_t>(sizeof(float));
  // In place (y == x) only with an fp32 output: each element is read before it is overwritten.
  const bool in_place = EPI != kSiluBf16 && static_cast<const void*>(y) == static_cast<const void*>(x);
  if ((!in_place && sd::overlaps(y, ybytes, x, xbytes)) || sd::overlaps(y, ybytes, gamma, pbytes) ||
      sd::overlaps(y, ybytes, beta, pbytes))
    return sd::fail(SD_ERR_INVALID_ARG, "%s: y overlaps an input (only y == x with an fp32 output is allowed)", name);
  cudaStream_t s = static_cast<cudaStream_t>(stream);

  // Resident path: a (cluster size, CTA size) pair that holds the group in registers (at most
  // kMaxItems float4 per thread, 8 for 1024-thread CTAs) with chunk a multiple of 4 elements.
  // Policy (measured on the SD shapes): the smallest cluster and CTA size that still put about
  // one CTA on every SM.
  const bool y_vec = EPI == kSiluBf16 ? (reinterpret_cast<uintptr_t>(y) & 7u) == 0 : sd::aligned16(y);
  const bool vec_ok = hw % 4 == 0 && cpg <= kMaxGroupChannels && sd::aligned16(x) && y_vec;
  int cs = 0, threads = 0;
  if (vec_ok && SD_GN_POLICY == 0 && group_elems % 16 == 0) {
    // Groups of 40960-81920 elements (the SD/SDXL top levels, 10 or 20 channels of 64 x 64): clusters
    // of 4 CTAs x 512 threads with 5-10 float4 per thread, two CTAs per SM -- measured faster than
    // 8 x 256 ([2,320,64,64] 7.7 -> 7.5 us, [2,640,64,64] 13.7 -> 11.7, [16,640,64,64] 66.8 -> 61.0).
    const int64_t sms = sd::sm_count();
    const int64_t need = (group_elems / 4 / 4 + 511) / 512;
    if (need >= 5 && need <= 10 && n_groups * 4 >= sms) {
      cs = 4;
      threads = 512;
    }
  }
  if (vec_ok && SD_GN_POLICY == 0 && !cs) {
    // First choice (measured on the inner UNet levels): 256-thread CTAs in the smallest cluster that
    // still gives one CTA per SM, if that holds at most 6 float4 per thread -- half as many CTAs and
    // cheaper cluster barriers ([2,640,32,32] 5.9 -> 5.1 us, [2,1280,16,16] 5.7 -> 4.0 us). With
    // more values per thread (e.g. [2,320,64,64]) the rule below is faster.
    const int64_t sms = sd::sm_count();
    for (int c = 1; c <= kMaxCluster && !cs; c *= 2) {
      if (group_elems % (4 * c) != 0 || group_elems / c > int64_t(256) * 4 * 6 || n_groups * c < sms) continue;
      cs = c;
      threads = 256;
    }
  }
  if (vec_ok && !cs) {
    const int64_t sms = sd::sm_count();
    const int64_t want = SD_GN_POLICY == 0 ? 2 * sms : SD_GN_POLICY == 1 ? 0 : sms;
    const int tlist0[3] = {256, 512, 1024};
    const int tlist1[3] = {1024, 512, 256};
    const int* tl = SD_GN_POLICY == 0 ? tlist0 : tlist1;
    for (int ti = 0; ti < 3 && !cs; ++ti) {
      const int th = tl[ti];
      const int max_items = th == 1024 ? 8 : kMaxItems;
      for (int c = 1; c <= kMaxCluster; c *= 2) {
        if (group_elems % (4 * c) != 0 || group_elems / c > int64_t(th) * 4 * max_items) continue;
        if (n_groups * c < want && c < kMaxCluster) continue;
        cs = c;
        threads = th;
        break;
      }
    }
  }
  cudaError_t err;
  if (cs > 0) {
    const int chunk = static_cast<int>(group_elems / cs);
    const int need = (chunk / 4 + threads - 1) / threads;
    const dim3 grid(static_cast<unsigned>(n_groups * cs));
    const int ge = static_cast<int>(group_elems), ihw = static_cast<int>(hw), icpg = static_cast<int>(cpg),
              ig = static_cast<int>(groups);
#define SD_GN_CASE(N, T) \
  if (threads == T && need <= N) err = launch_resident<N, T, EPI>(grid, cs, s, x, gamma, beta, y, ge, chunk, ihw, icpg, ig, eps); else
#define SD_GN_T(T) SD_GN_CASE(1, T) SD_GN_CASE(2, T) SD_GN_CASE(3, T) SD_GN_CASE(4, T) SD_GN_CASE(5, T) \
    SD_GN_CASE(6, T) SD_GN_CASE(8, T)
    SD_GN_T(256) SD_GN_T(512) SD_GN_T(1024) SD_GN_CASE(10, 256) SD_GN_CASE(12, 256) SD_GN_CASE(16, 256)
    SD_GN_CASE(10, 512) SD_GN_CASE(12, 512) SD_GN_CASE(16, 512) err = cudaErrorInvalidValue;
#undef SD_GN_T
#undef SD_GN_CASE
  } else {
    // Streaming path: a cluster of up to 8 CTAs per group, each with at least 1024 elements.
    int c = 1;
    while (c < kMaxCluster && group_elems / (2 * c) >= 1024) c *= 2;
    const int64_t chunk = (group_elems + c - 1) / c;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(n_groups * c));
    cfg.blockDim = dim3(kThreads);
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = c;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1 + sd::pdl_attr(&attr[1]);
    err = cudaLaunchKernelEx(&cfg, gn_streaming<EPI>, x, gamma, beta, y, group_elems, chunk, hw,
                             static_cast<int>(cpg), static_cast<int>(groups), eps);
  }
  return sd::cuda_check(err, "group norm launch");
}

}  // namespace

extern "C" sd_status sd_group_norm(const float* x, const float* gamma, const float* beta, float* y, int64_t B,
                                   int64_t C, int64_t H, int64_t W, int64_t groups, float eps, void* stream) {
  return group_norm_impl<kAffine>("sd_group_norm", x, gamma, beta, y, B, C, H, W, groups, eps, stream);
}

extern "C" sd_status sd_group_norm_silu(const float* x, const float* gamma, const float* beta, void* y, int64_t B,
                                        int64_t C, int64_t H, int64_t W, int64_t groups, float eps, int out_bf16,
                                        void* stream) {
  if (out_bf16 != 0 && out_bf16 != 1) return sd::fail(SD_ERR_INVALID_ARG, "sd_group_norm_silu: out_bf16 must be 0 or 1");
  return out_bf16 ? group_norm_impl<kSiluBf16>("sd_group_norm_silu", x, gamma, beta, y, B, C, H, W, groups, eps, stream)
                  : group_norm_impl<kSiluF32>("sd_group_norm_silu", x, gamma, beta, y, B, C, H, W, groups, eps, stream);
}
