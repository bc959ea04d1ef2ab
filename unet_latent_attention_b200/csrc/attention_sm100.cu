// Multi-head attention forward for the UNet spatial transformer on sm_100a (sd_attention).
//
// Computes O = softmax(Q K^T * scale) V per (batch, head) with the tiled online-softmax scheme of
// "从零实现扩散模型推理引擎：Rust + wgpu 的 GPU 加速图像生成架构" §3.2 (running row max m, running sum l,
// output rescaled by exp(m_prev - m)); the page's WGSL kernel (64x64 tiles, fp32 workgroup arrays,
// output normalised every step) is prior art for another machine. The B200 design:
//
//  * One CTA owns NQ query tiles of 128 rows of one (b, h) and streams the key/value sequence in
//    tiles of BN keys. Q and the K/V tiles arrive by TMA (3-D tensor maps over [B*h, L, dh],
//    128-byte swizzle, boxes 64 wide in dh) into a ring of STAGES shared-memory stages; rows past
//    the sequence end and columns past dh are zero-filled by the TMA unit, which pads dh = 40 to
//    the MMA depth 48 and masks ragged tails for free.
//  * One thread issues the tensor-core work: S = Q K^T (tcgen05.mma, bf16 in, fp32 accumulate,
//    M = 128, N = BN, K = 16 per instruction) into tensor memory, then O += P V with P read
//    straight from tensor memory (the "A in TMEM" form) and V from shared memory (N-major B).
//  * Four warps per query tile (one TMEM lane quarter each, one thread per row) run the softmax:
//    tcgen05.ld the S row, row max, exp2 with scale*log2(e) folded into one FMA, row sum, pack to
//    bf16 and tcgen05.st P over the S columns. The running max is only raised when it grows by
//    more than 2^8 (lazy rescaling), so most tiles skip the O correction. Normalisation by l is
//    deferred to the epilogue, which equals the page's per-step form in exact arithmetic.
//  * Two query tiles per CTA (NQ = 2) share every K/V tile, halving L2->SM traffic, and let one
//    tile's softmax overlap the other tile's matrix products.
//  * Every wait on an mbarrier is bounded (about one second); on expiry the CTA records
//    SD_ERR_TIMEOUT in the device status word, drains its own in-flight copies and MMAs, frees its
//    tensor memory and returns. Nothing traps.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <mutex>

#include "sd_internal.h"
#include "sm100_ptx.cuh"

namespace {

using namespace sm100;

constexpr int BM = 128;                          // query rows per tile = TMEM lanes
constexpr long long kWaitLimitCycles = 2000000000LL;  // ~1 s at B200 clocks

template <int DHP_, int BN_, int NQ_, int STAGES_>
struct Cfg {
  static constexpr int DHP = DHP_;        // head dim padded to the MMA granule (16)
  static constexpr int BN = BN_;          // keys per K/V tile
  static constexpr int NQ = NQ_;          // 128-row query tiles per CTA
  static constexpr int STAGES = STAGES_;  // K/V ring depth
  static constexpr int NCH = (DHP + 63) / 64;  // 64-element (128-byte) swizzle chunks along dh
  static constexpr int Q_TILE_BYTES = NCH * BM * 128;
  static constexpr int KV_TILE_BYTES = NCH * BN * 128;
  static constexpr int Q_OFF = 0;
  static constexpr int K_OFF = Q_OFF + NQ * Q_TILE_BYTES;
  static constexpr int V_OFF = K_OFF + STAGES * KV_TILE_BYTES;
  static constexpr int BAR_OFF = V_OFF + STAGES * KV_TILE_BYTES;
  // q_full, k_full[S], v_full[S], kv_empty[S], s_full[NQ], p_full[NQ], o_done[NQ], final
  static constexpr int NBARS = 1 + 3 * STAGES + 3 * NQ + 1;
  static constexpr int MISC_OFF = BAR_OFF + NBARS * 8;
  static constexpr int SMEM_BYTES = MISC_OFF + 16 + 1024;  // + slack to align the base to 1024
  static constexpr int TM_TILE = 256;                      // TMEM columns per query tile: S | O
  static constexpr int TM_COLS = NQ * TM_TILE;
  static constexpr int NUM_WARPS = 2 + 4 * NQ;  // producer, MMA issuer, 4 softmax warps per tile
  static constexpr int THREADS = 32 * NUM_WARPS;
  static_assert(DHP % 16 == 0 && DHP <= 256, "MMA N must be a multiple of 16");
  static_assert(BN % 32 == 0 && BN + DHP <= TM_TILE, "S and O must fit the tile's TMEM columns");
  static_assert(TM_COLS == 256 || TM_COLS == 512, "TMEM allocation is a power of two");
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
};

struct Bars {
  uint32_t base;
  int stages, nq;
  __device__ uint32_t q_full() const { return base; }
  __device__ uint32_t k_full(int s) const { return base + 8 * (1 + s); }
  __device__ uint32_t v_full(int s) const { return base + 8 * (1 + stages + s); }
  __device__ uint32_t kv_empty(int s) const { return base + 8 * (1 + 2 * stages + s); }
  __device__ uint32_t s_full(int t) const { return base + 8 * (1 + 3 * stages + t); }
  __device__ uint32_t p_full(int t) const { return base + 8 * (1 + 3 * stages + nq + t); }
  __device__ uint32_t o_done(int t) const { return base + 8 * (1 + 3 * stages + 2 * nq + t); }
  __device__ uint32_t fin() const { return base + 8 * (1 + 3 * stages + 3 * nq); }
};

// Bounded wait. Returns false if this CTA has aborted or the limit expired (then it raises the
// CTA's abort flag and the device status word). `abortable = false` is for teardown drains.
__device__ __noinline__ bool wait_bar(uint32_t bar, uint32_t parity, volatile int* abort_flag, unsigned int* err,
                                      bool abortable = true) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 127u) == 0) {
      if (abortable && *abort_flag) return false;
      if (clock64() - t0 > kWaitLimitCycles) {
        *abort_flag = 1;
        atomicOr(err, sd::kDevErrTimeout);
        return false;
      }
    }
  }
}

template <class C>
__global__ void __launch_bounds__(C::THREADS, 1)
    attn_fwd_sm100(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, __nv_bfloat16* __restrict__ out, int Lq, int Lk,
                   int dh, float scale_log2, unsigned int* err, int debug_flags) {
  constexpr int BN = C::BN, NQ = C::NQ, STAGES = C::STAGES, NCH = C::NCH, DHP = C::DHP;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const Bars bars{sbase + C::BAR_OFF, STAGES, NQ};
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::MISC_OFF + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = blockIdx.y;
  const int q0 = blockIdx.x * (BM * NQ);
  const int nkv = (Lk + BN - 1) / BN;

  if (threadIdx.x == 0) {
    mbar_init(bars.q_full(), 1);
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(bars.k_full(s), 1);
      mbar_init(bars.v_full(s), 1);
      mbar_init(bars.kv_empty(s), 1);
    }
    for (int t = 0; t < NQ; ++t) {
      mbar_init(bars.s_full(t), 1);
      mbar_init(bars.p_full(t), 128);
      mbar_init(bars.o_done(t), 1);
    }
    mbar_init(bars.fin(), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), C::TM_COLS);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int issued[STAGES];
#pragma unroll
      for (int s = 0; s < STAGES; ++s) issued[s] = 0;
      mbar_arrive_expect_tx(bars.q_full(), NQ * C::Q_TILE_BYTES);
      for (int t = 0; t < NQ; ++t)
        for (int c = 0; c < NCH; ++c)
          tma_load_3d(sbase + C::Q_OFF + t * C::Q_TILE_BYTES + c * BM * 128, &tm_q, bars.q_full(), c * 64,
                      q0 + t * BM, bh);
      for (int j = 0; j < nkv; ++j) {
        const int s = j % STAGES, round = j / STAGES;
        if (j >= STAGES && !wait_bar(bars.kv_empty(s), (round - 1) & 1, abort_flag, err)) break;
        mbar_arrive_expect_tx(bars.k_full(s), C::KV_TILE_BYTES);
        for (int c = 0; c < NCH; ++c)
          tma_load_3d(sbase + C::K_OFF + s * C::KV_TILE_BYTES + c * BN * 128, &tm_k, bars.k_full(s), c * 64,
                      j * BN, bh);
        issued[s] = round + 1;
        if ((debug_flags & 1) && j == 0) break;  // test hook: V tile 0 never arrives
        mbar_arrive_expect_tx(bars.v_full(s), C::KV_TILE_BYTES);
        for (int c = 0; c < NCH; ++c)
          tma_load_3d(sbase + C::V_OFF + s * C::KV_TILE_BYTES + c * BN * 128, &tm_v, bars.v_full(s), c * 64,
                      j * BN, bh);
      }
      // Drain: every copy this thread issued has landed before the CTA may exit.
      wait_bar(bars.q_full(), 0, abort_flag, err, false);
      for (int s = 0; s < STAGES; ++s)
        if (issued[s] > 0) {
          wait_bar(bars.k_full(s), (issued[s] - 1) & 1, abort_flag, err, false);
          if (!(debug_flags & 1)) wait_bar(bars.v_full(s), (issued[s] - 1) & 1, abort_flag, err, false);
        }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(BM, BN, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(BM, DHP, true);
      auto issue_qk = [&](int t, int s) {
        const uint32_t d = tmem + t * C::TM_TILE;  // S: columns [0, BN)
#pragma unroll
        for (int ks = 0; ks < DHP / 16; ++ks) {
          const uint32_t off = (ks >> 2) * (BM * 128) + (ks & 3) * 32;
          const uint32_t offk = (ks >> 2) * (BN * 128) + (ks & 3) * 32;
          const uint64_t a = smem_desc(sbase + C::Q_OFF + t * C::Q_TILE_BYTES + off, 16, 1024);
          const uint64_t b = smem_desc(sbase + C::K_OFF + s * C::KV_TILE_BYTES + offk, 16, 1024);
          mma_ss(d, a, b, idesc_qk, ks > 0 ? 1u : 0u);
        }
      };
      auto issue_pv = [&](int t, int s, bool first) {
        const uint32_t d = tmem + t * C::TM_TILE + BN;  // O: columns [BN, BN + DHP)
        const uint32_t a = tmem + t * C::TM_TILE;       // P: bf16 pairs over S columns [0, BN/2)
#pragma unroll
        for (int ks = 0; ks < BN / 16; ++ks) {
          const uint64_t b = smem_desc(sbase + C::V_OFF + s * C::KV_TILE_BYTES + ks * 16 * 128, BN * 128, 1024);
          mma_ts(d, a + ks * 8, b, idesc_pv, (!first || ks > 0) ? 1u : 0u);
        }
      };
      bool ok = wait_bar(bars.q_full(), 0, abort_flag, err) && wait_bar(bars.k_full(0), 0, abort_flag, err);
      if (ok) {
        tc_fence_after();
        for (int t = 0; t < NQ; ++t) {
          issue_qk(t, 0);
          mma_commit(bars.s_full(t));
        }
      }
      for (int j = 0; ok && j < nkv; ++j) {
        const int s = j % STAGES;
        const uint32_t ph = (j / STAGES) & 1;
        for (int t = 0; ok && t < NQ; ++t) {
          ok = wait_bar(bars.p_full(t), j & 1, abort_flag, err) &&
               (t > 0 || wait_bar(bars.v_full(s), ph, abort_flag, err));
          if (!ok) break;
          tc_fence_after();
          issue_pv(t, s, j == 0);
          mma_commit(bars.o_done(t));
          if (t == NQ - 1) mma_commit(bars.kv_empty(s));
          if (j + 1 < nkv) {
            const int s1 = (j + 1) % STAGES;
            const uint32_t ph1 = ((j + 1) / STAGES) & 1;
            // P aliases S: the next S may only be written once this P V has been consumed.
            ok = wait_bar(bars.o_done(t), j & 1, abort_flag, err) &&
                 (t > 0 || wait_bar(bars.k_full(s1), ph1, abort_flag, err));
            if (!ok) break;
            tc_fence_after();
            issue_qk(t, s1);
            mma_commit(bars.s_full(t));
          }
        }
      }
      // Drain: all tensor-core work issued by this thread completes before TMEM is released.
      mma_commit(bars.fin());
      wait_bar(bars.fin(), 0, abort_flag, err, false);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------------ softmax warps
    const int t = (warp - 2) >> 2;  // query tile of this warpgroup
    const int quarter = warp & 3;   // TMEM lane quarter this warp may access
    const int row = quarter * 32 + lane;
    const uint32_t tS = tmem + t * C::TM_TILE + (static_cast<uint32_t>(quarter * 32) << 16);
    const uint32_t tO = tS + BN;
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int j = 0; j < nkv; ++j) {
      // warp-uniform outcome: the tcgen05 copies below are .sync.aligned
      if (!__all_sync(0xffffffffu, wait_bar(bars.s_full(t), j & 1, abort_flag, err))) {
        ok = false;
        break;
      }
      tc_fence_after();
      float sv[BN];
#pragma unroll
      for (int c = 0; c < BN / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(tS + c * 32, r);
#pragma unroll
        for (int i = 0; i < 32; ++i) sv[c * 32 + i] = __uint_as_float(r[i]);
      }
      tmem_wait_ld();
      const int valid = Lk - j * BN;
      if (valid < BN) {
#pragma unroll
        for (int i = 0; i < BN; ++i)
          if (i >= valid) sv[i] = -INFINITY;
      }
      float mx = sv[0];
#pragma unroll
      for (int i = 1; i < BN; ++i) mx = fmaxf(mx, sv[i]);
      const float m_new = fmaxf(m_run, mx * scale_log2);
      // Lazy rescale (always on the first tile). The decision is warp-uniform: the tcgen05 copies
      // of O below are .sync.aligned, and rescaling a row whose max barely moved is still exact.
      if (__any_sync(0xffffffffu, m_new > m_run + 8.0f)) {
        const float alpha = ex2_approx(m_run - m_new);
        l_run *= alpha;
        if (j > 0) {
#pragma unroll
          for (int c = 0; c < DHP / 16; ++c) {
            uint32_t r[16];
            tmem_ld16(tO + c * 16, r);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 16; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
            tmem_st16(tO + c * 16, r);
          }
        }
        m_run = m_new;
      }
      const float neg_m = -m_run;
      float rs = 0.f;
#pragma unroll
      for (int c = 0; c < BN / 32; ++c) {
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float p0 = ex2_approx(fmaf(sv[c * 32 + 2 * i], scale_log2, neg_m));
          const float p1 = ex2_approx(fmaf(sv[c * 32 + 2 * i + 1], scale_log2, neg_m));
          rs += p0 + p1;
          pk[i] = pack_bf16x2(p0, p1);
        }
        tmem_st16(tS + c * 16, pk);
      }
      l_run += rs;
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bars.p_full(t));
    }
    if (ok && __all_sync(0xffffffffu, wait_bar(bars.o_done(t), (nkv - 1) & 1, abort_flag, err))) {
      tc_fence_after();
      const int qrow = q0 + t * BM + row;
      const float inv_l = 1.0f / l_run;
      uint32_t packed[DHP / 2];
#pragma unroll
      for (int c = 0; c < DHP / 16; ++c) {
        uint32_t r[16];
        tmem_ld16(tO + c * 16, r);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 8; ++i)
          packed[c * 8 + i] = pack_bf16x2(__uint_as_float(r[2 * i]) * inv_l, __uint_as_float(r[2 * i + 1]) * inv_l);
      }
      if (qrow < Lq) {
        uint4* dst = reinterpret_cast<uint4*>(out + (static_cast<size_t>(bh) * Lq + qrow) * dh);
        const int n16 = dh / 8;  // 16-byte groups of 8 bf16
#pragma unroll
        for (int i = 0; i < DHP / 8; ++i)
          if (i < n16) dst[i] = make_uint4(packed[4 * i], packed[4 * i + 1], packed[4 * i + 2], packed[4 * i + 3]);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TM_COLS);
  }
}

// ---------------------------------------------------------------------------- host side
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 3-D map over a contiguous bf16 [planes, rows, dh] tensor, box {64, box_rows, 1}, 128-byte swizzle.
sd_status make_map(CUtensorMap* map, const void* ptr, int64_t dh, int64_t rows, int64_t planes, int box_rows) {
  auto fn = encode_fn();
  if (!fn) return sd::fail(SD_ERR_CUDA, "sd_attention: cuTensorMapEncodeTiled is unavailable");
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(dh), static_cast<cuuint64_t>(rows),
                              static_cast<cuuint64_t>(planes)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(dh * 2), static_cast<cuuint64_t>(rows * dh * 2)};
  const cuuint32_t box[3] = {64, static_cast<cuuint32_t>(box_rows), 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return sd::fail(SD_ERR_CUDA, "sd_attention: cuTensorMapEncodeTiled failed (%d)", (int)r);
  return SD_OK;
}

int g_debug_flags = 0;

template <class C>
sd_status launch(const void* q, const void* k, const void* v, void* o, int64_t BH, int64_t Lq, int64_t Lk,
                 int64_t dh, float scale, cudaStream_t s) {
  CUtensorMap mq, mk, mv;
  sd_status st = make_map(&mq, q, dh, Lq, BH, BM);
  if (st == SD_OK) st = make_map(&mk, k, dh, Lk, BH, C::BN);
  if (st == SD_OK) st = make_map(&mv, v, dh, Lk, BH, C::BN);
  if (st != SD_OK) return st;
  unsigned int* err = sd::device_status_word();
  if (!err) return SD_ERR_CUDA;
  auto kern = attn_fwd_sm100<C>;
  st = sd::cuda_check(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES),
                      "cudaFuncSetAttribute(attention smem)");
  if (st != SD_OK) return st;
  const dim3 grid(static_cast<unsigned>((Lq + BM * C::NQ - 1) / (BM * C::NQ)), static_cast<unsigned>(BH));
  const float scale_log2 = scale * 1.4426950408889634f;
  kern<<<grid, C::THREADS, C::SMEM_BYTES, s>>>(mq, mk, mv, static_cast<__nv_bfloat16*>(o), static_cast<int>(Lq),
                                                static_cast<int>(Lk), static_cast<int>(dh), scale_log2, err,
                                                g_debug_flags);
  return sd::cuda_check(cudaGetLastError(), "sd_attention launch");
}

}  // namespace

extern "C" sd_status sd_attention(const void* q, const void* k, const void* v, void* o, int64_t B, int64_t heads,
                                  int64_t Lq, int64_t Lk, int64_t dh, float scale, void* stream) {
  if (B < 0 || heads < 0 || Lq < 0 || Lk < 0) return sd::fail(SD_ERR_INVALID_ARG, "sd_attention: negative size");
  if (dh != 40 && dh != 64 && dh != 80 && dh != 160)
    return sd::fail(SD_ERR_UNSUPPORTED, "sd_attention: head dim %lld not in {40, 64, 80, 160}", (long long)dh);
  if (!std::isfinite(scale)) return sd::fail(SD_ERR_INVALID_ARG, "sd_attention: scale is not finite");
  if (B == 0 || heads == 0 || Lq == 0) return SD_OK;
  if (Lk == 0) return sd::fail(SD_ERR_INVALID_ARG, "sd_attention: Lk must be >= 1 when Lq >= 1");
  if (!q || !k || !v || !o) return sd::fail(SD_ERR_INVALID_ARG, "sd_attention: null pointer");
  const int64_t BH = B * heads;
  if (BH > 65535 || Lq > (int64_t(1) << 30) || Lk > (int64_t(1) << 30))
    return sd::fail(SD_ERR_UNSUPPORTED, "sd_attention: B*heads must be <= 65535 and L <= 2^30");
  if (!sd::aligned16(q) || !sd::aligned16(k) || !sd::aligned16(v) || !sd::aligned16(o))
    return sd::fail(SD_ERR_MISALIGNED, "sd_attention: q, k, v and o must be 16-byte aligned");
  const int64_t qbytes = BH * Lq * dh * 2, kvbytes = BH * Lk * dh * 2;
  if (sd::overlaps(o, qbytes, q, qbytes) || sd::overlaps(o, qbytes, k, kvbytes) || sd::overlaps(o, qbytes, v, kvbytes))
    return sd::fail(SD_ERR_INVALID_ARG, "sd_attention: o overlaps q, k or v");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  switch (dh) {
    case 40: return launch<Cfg<48, 128, 2, 3>>(q, k, v, o, BH, Lq, Lk, dh, scale, s);
    case 64: return launch<Cfg<64, 128, 2, 3>>(q, k, v, o, BH, Lq, Lk, dh, scale, s);
    case 80: return launch<Cfg<80, 128, 2, 2>>(q, k, v, o, BH, Lq, Lk, dh, scale, s);
    default: return launch<Cfg<160, 64, 1, 3>>(q, k, v, o, BH, Lq, Lk, dh, scale, s);
  }
}

// Test hook (declared in sd_kernels.h): bit 0 makes the next attention launches skip their first
// V tile so that the kernel's bounded wait expires and reports SD_ERR_TIMEOUT.
extern "C" void sd_debug_set_fault(int flags) { g_debug_flags = flags; }
