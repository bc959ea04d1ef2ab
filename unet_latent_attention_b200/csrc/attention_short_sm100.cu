// Attention over a short key sequence on sm_100a: the cross-attention of the UNet's spatial
// transformer, where K and V come from the 77-token text context (sd_attention with Lk <= 80).
//
// "从零实现扩散模型推理引擎：Rust + wgpu 的 GPU 加速图像生成架构" §3.2 computes cross-attention with Q from
// the latent map and K/V from the text encoder, tile by tile with an online softmax, and notes that
// at 77 text tokens the tiled form gains little. With at most 80 keys the whole key sequence fits one
// tile, so this kernel keeps all of K and V resident in shared memory and takes one exact softmax
// pass per query tile (no running max, no rescaling):
//
//  * The work is the list of 128-row query tiles of all (batch, head) planes. A persistent grid of
//    one CTA per SM takes an equal contiguous range of tiles (mostly one head, so K/V are loaded once
//    per CTA or twice at a head boundary; two K/V buffers let the next head load early).
//  * The producer issues the TMA loads of every Q tile of the range as soon as a shared-memory slot
//    is free (up to QS in flight), so the whole range streams in at full bandwidth from the start.
//  * The MMA issuer computes S = Q K^T (M = 128, N = 80: keys 77..79 are the TMA's zero fill, masked
//    to -inf) into one of NSLOT tensor-memory slots as soon as a tile's Q has landed, and
//    O = P V once the softmax has written P over S in the same slot (the "A in TMEM" form), O going
//    over the columns of S that the softmax has already read (5 slots of 96 columns at dh 40 instead
//    of 4 of 128: 5% faster on the batched-serving shape). The row sums come out of P V through a
//    column of ones written into V (column dh).
//  * Two softmax warpgroups (three at dh 64) take tiles in turn: tcgen05.ld of the 80 scores, row max, exp2,
//    tcgen05.st of P, and the epilogue (tcgen05.ld of O, division by the row sum, 16-byte stores of
//    the row), each warp taking whichever of its next softmax and its oldest epilogue is ready.
//  * Every wait is bounded; on expiry the CTA records SD_ERR_TIMEOUT, drains and returns.
#include <cuda.h>
#include <cuda_bf16.h>

#include <algorithm>
#include <atomic>

#include "attn_common.cuh"
#include "sd_internal.h"
#include "sm100_ptx.cuh"

#ifndef SD_SHORT_POLY
#define SD_SHORT_POLY 2
#endif
#ifndef SD_SHORT_PERSIST
#define SD_SHORT_PERSIST 0  // 1: always the persistent multi-tile form (never one query tile per CTA)
#endif

namespace {

using namespace sm100;
using namespace sd::attn;

template <int DH_, bool F16_, bool BLHD_>
struct ShortCfg {
  static constexpr int DH = DH_;
  static constexpr bool F16 = F16_;
  static constexpr bool BLHD = BLHD_;
  static constexpr int BN = kShortMaxKeys;             // keys in the resident tile
  static constexpr int POLY = SD_SHORT_POLY;           // of every 8 column pairs, exp2 on the FMA pipe
  static constexpr int DHP = (DH + 15) / 16 * 16;      // Q K^T depth padded to the MMA granule
  static constexpr int NPV = (DH + 1 + 15) / 16 * 16;  // N of O = P V: O columns, then the row sum at DH
  static constexpr int NCH = (DHP + 63) / 64;          // 128-byte swizzle chunks of Q and K rows
  static constexpr int NCHV = (NPV + 63) / 64;         // chunks of V rows (the ones column included)
  static constexpr int Q_TILE = NCH * BM * 128;
  static constexpr int K_BYTES = NCH * BN * 128;
  static constexpr int V_BYTES = NCHV * BN * 128;
  // Tensor-memory columns of one slot: S in [0, BN), P written over its first BN / 2 columns, O from
  // column OFS_O over the part of S that the softmax has read before P V runs.
  static constexpr int OFS_O = BN / 2 + 8;
  static constexpr int TM_W = OFS_O + NPV;
  static constexpr int NSLOT = 512 / TM_W < 8 ? 512 / TM_W : 8;
  // K/V buffers: two when they fit beside at least two Q slots, else one
  static constexpr int KVB = 2 * (K_BYTES + V_BYTES) + 2 * Q_TILE <= 200 * 1024 ? 2 : 1;
  static constexpr int QS_FIT = (200 * 1024 - KVB * (K_BYTES + V_BYTES)) / Q_TILE;
  static constexpr int QS = QS_FIT < 8 ? QS_FIT : 8;  // Q tiles in flight
  static constexpr int Q_OFF = 0;
  static constexpr int K_OFF = Q_OFF + QS * Q_TILE;
  static constexpr int V_OFF = K_OFF + KVB * K_BYTES;
  static constexpr int BAR_OFF = V_OFF + KVB * V_BYTES;
  // q_full[QS], q_empty[QS], k_full[KVB], v_full[KVB], v_ready[KVB], kv_empty[KVB], s_full[NSLOT],
  // p_full[NSLOT], o_full[NSLOT], slot_free[NSLOT], fin[2] (one per MMA-issuing warp)
  static constexpr int NBARS = 2 * QS + 4 * KVB + 4 * NSLOT + 2;
  static constexpr int MISC_OFF = BAR_OFF + NBARS * 8;
  static constexpr int SMEM_BYTES = MISC_OFF + 16 + 1024;  // + slack to align the base to 1024
  // Warps: 0 TMA producer, 1 S = Q K^T issuer (and TMEM owner), 2 O = P V issuer, 3 V fix-up;
  // warpgroups 1 .. NWG run the softmax and epilogue of tiles in turn.
  static constexpr int SOFT_WARP0 = 4;
  // Softmax warpgroups taking alternate tiles; a tile's slot must outlive NWG tiles. Three at dh 64
  // (SDXL level 1: 10.9 -> 10.1 us), two elsewhere (three measured 1% slower at dh 40).
  static constexpr int NWG = DH == 64 && NSLOT >= 3 ? 3 : 2;
  static constexpr int THREADS = 128 + 128 * NWG;
  static_assert(QS >= 1 && NSLOT >= 2 && NSLOT >= NWG, "resources");
  static_assert(NSLOT * TM_W <= 512, "tensor memory holds 512 columns");
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
  static_assert(NPV <= 256 && NPV % 16 == 0 && BN % 16 == 0, "MMA shapes");
};

template <class C>
struct ShortBars {
  uint32_t base;
  __device__ uint32_t q_full(int i) const { return base + 8 * i; }
  __device__ uint32_t q_empty(int i) const { return base + 8 * (C::QS + i); }
  __device__ uint32_t k_full(int b) const { return base + 8 * (2 * C::QS + b); }
  __device__ uint32_t v_full(int b) const { return base + 8 * (2 * C::QS + C::KVB + b); }
  __device__ uint32_t v_ready(int b) const { return base + 8 * (2 * C::QS + 2 * C::KVB + b); }
  __device__ uint32_t kv_empty(int b) const { return base + 8 * (2 * C::QS + 3 * C::KVB + b); }
  __device__ uint32_t s_full(int s) const { return base + 8 * (2 * C::QS + 4 * C::KVB + s); }
  __device__ uint32_t p_full(int s) const { return base + 8 * (2 * C::QS + 4 * C::KVB + C::NSLOT + s); }
  __device__ uint32_t o_full(int s) const { return base + 8 * (2 * C::QS + 4 * C::KVB + 2 * C::NSLOT + s); }
  __device__ uint32_t slot_free(int s) const { return base + 8 * (2 * C::QS + 4 * C::KVB + 3 * C::NSLOT + s); }
  __device__ uint32_t fin(int w) const { return base + 8 * (2 * C::QS + 4 * C::KVB + 4 * C::NSLOT + w); }
};

template <class C>
__global__ void __launch_bounds__(C::THREADS, 1)
    attn_short_sm100(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, uint16_t* __restrict__ out, int Lq, int Lk, int dh,
                     float scale_log2, unsigned int* err, int debug_flags, int tiles_per_head, long long n_tiles,
                     int lay_heads) {
  constexpr int BN = C::BN, NSLOT = C::NSLOT, QS = C::QS, KVB = C::KVB, NCH = C::NCH, NCHV = C::NCHV;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const ShortBars<C> bars{sbase + C::BAR_OFF};
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::MISC_OFF + 4);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // this CTA's tiles [t0, t0 + n): an equal share of the tile list
  const long long t0 = n_tiles * blockIdx.x / gridDim.x;
  const int n = static_cast<int>(n_tiles * (blockIdx.x + 1) / gridDim.x - t0);
  // Plane and first query row of local tile i. One 64-bit division at entry; 32-bit arithmetic after
  // (a 64-bit division is a long software routine, and these run once per tile in every role).
  const unsigned tph = static_cast<unsigned>(tiles_per_head);
  const int bh0 = static_cast<int>(t0 / tiles_per_head);
  const unsigned qt0 = static_cast<unsigned>(t0 - static_cast<long long>(bh0) * tiles_per_head);
  auto head_of = [&](int i) { return bh0 + static_cast<int>((qt0 + static_cast<unsigned>(i)) / tph); };
  auto row0_of = [&](int i) { return static_cast<int>((qt0 + static_cast<unsigned>(i)) % tph) * BM; };

  if (threadIdx.x == 0) {
    for (int i = 0; i < QS; ++i) {
      mbar_init(bars.q_full(i), 1);
      mbar_init(bars.q_empty(i), 1);
    }
    for (int b = 0; b < KVB; ++b) {
      mbar_init(bars.k_full(b), 1);
      mbar_init(bars.v_full(b), 1);
      mbar_init(bars.v_ready(b), 1);
      mbar_init(bars.kv_empty(b), 1);
    }
    for (int s = 0; s < NSLOT; ++s) {
      mbar_init(bars.s_full(s), 1);
      mbar_init(bars.p_full(s), 128);
      mbar_init(bars.o_full(s), 1);
      mbar_init(bars.slot_free(s), 128);
    }
    mbar_init(bars.fin(0), 1);
    mbar_init(bars.fin(1), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), 512);
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
  // Everything above touched only shared memory, tensor memory and the kernel parameters: it may
  // overlap the end of the previous kernel on the stream. Global memory waits for that kernel.
  sd::grid_dep_wait();
  sd::grid_dep_launch();

  if (warp < C::SOFT_WARP0) {
    if (warp == 0 && lane == 0) {
      // ---------------------------------------------------------------- TMA producer
      int hv = -1, prev = -1, q_issued = 0, kv_issued = 0;
      bool ok = true, v_skipped = false;
      for (int i = 0; i < n && ok; ++i) {
        const int bh = head_of(i);
        if (bh != prev) {  // a new head: its K and V into the next K/V buffer
          ++hv;
          const int b = hv % KVB;
          if (hv >= KVB && !wait_bar(bars.kv_empty(b), (hv / KVB - 1) & 1, abort_flag, err)) break;
          mbar_arrive_expect_tx(bars.k_full(b), C::K_BYTES);
          for (int c = 0; c < NCH; ++c)
            load_rows<C::BLHD>(sbase + C::K_OFF + b * C::K_BYTES + c * BN * 128, &tm_k, bars.k_full(b), c * 64, 0,
                               bh, lay_heads);
          kv_issued = hv + 1;
          if ((debug_flags & 1) && hv == 0) {  // test hook: the first V tile never arrives
            v_skipped = true;
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(bars.v_full(b), C::V_BYTES);
          for (int c = 0; c < NCHV; ++c)
            load_rows<C::BLHD>(sbase + C::V_OFF + b * C::V_BYTES + c * BN * 128, &tm_v, bars.v_full(b), c * 64, 0,
                               bh, lay_heads);
          prev = bh;
        }
        const int qs = i % QS;
        if (i >= QS && !wait_bar(bars.q_empty(qs), (i / QS - 1) & 1, abort_flag, err)) break;
        mbar_arrive_expect_tx(bars.q_full(qs), C::Q_TILE);
        for (int c = 0; c < NCH; ++c)
          load_rows<C::BLHD>(sbase + C::Q_OFF + qs * C::Q_TILE + c * BM * 128, &tm_q, bars.q_full(qs), c * 64,
                             row0_of(i), bh, lay_heads);
        q_issued = i + 1;
      }
      // Drain: every copy this thread issued has landed before the CTA may exit.
      for (int i = q_issued - 1; i >= 0 && i >= q_issued - QS; --i)
        wait_bar(bars.q_full(i % QS), (i / QS) & 1, abort_flag, err, false);
      for (int h = kv_issued - 1; h >= 0 && h >= kv_issued - KVB; --h) {
        wait_bar(bars.k_full(h % KVB), (h / KVB) & 1, abort_flag, err, false);
        if (!(v_skipped && h == kv_issued - 1)) wait_bar(bars.v_full(h % KVB), (h / KVB) & 1, abort_flag, err, false);
      }
    } else if (warp == 1 && lane == 0) {
      // ---------------------------------------------------------------- S = Q K^T issuer
      // Tiles in order: S of tile i needs its Q, its head's K and a free tensor-memory slot. The
      // waits suspend the thread (no polling that would take issue slots from the softmax warps of
      // this sub-partition); P V is issued by warp 2.
      constexpr uint32_t idesc_qk = idesc_f16kind_f32(BM, BN, false, C::F16);
      int hq = 0, prev = n > 0 ? head_of(0) : -1;
      for (int iq = 0; iq < n; ++iq) {
        if (iq > 0 && head_of(iq) != prev) {
          prev = head_of(iq);
          ++hq;
        }
        const int slot = iq % NSLOT, qs = iq % QS, b = hq % KVB;
        if (!wait_bar(bars.q_full(qs), (iq / QS) & 1, abort_flag, err) ||
            !wait_bar(bars.k_full(b), (hq / KVB) & 1, abort_flag, err) ||
            (iq >= NSLOT && !wait_bar(bars.slot_free(slot), (iq / NSLOT - 1) & 1, abort_flag, err)))
          break;
        tc_fence_after();
        const uint32_t d = tmem + slot * C::TM_W;
#pragma unroll
        for (int ks = 0; ks < C::DHP / 16; ++ks) {
          const uint32_t offq = (ks >> 2) * (BM * 128) + (ks & 3) * 32;
          const uint32_t offk = (ks >> 2) * (BN * 128) + (ks & 3) * 32;
          const uint64_t ad = smem_desc(sbase + C::Q_OFF + qs * C::Q_TILE + offq, 16, 1024);
          const uint64_t bd = smem_desc(sbase + C::K_OFF + b * C::K_BYTES + offk, 16, 1024);
          mma_ss(d, ad, bd, idesc_qk, ks > 0 ? 1u : 0u);
        }
        mma_commit(bars.s_full(slot));
        mma_commit(bars.q_empty(qs));
      }
      // Drain: all tensor-core work issued by this thread completes before TMEM is released.
      mma_commit(bars.fin(0));
      wait_bar(bars.fin(0), 0, abort_flag, err, false);
    } else if (warp == 2 && lane == 0) {
      // ---------------------------------------------------------------- O = P V issuer
      // Tiles in order: P V of tile i needs its P (written over S by the softmax) and its head's V
      // with the ones column. After the last P V of a head the K/V buffer is released: every S of
      // that head has completed, since each P V waited for its tile's softmax.
      constexpr uint32_t idesc_pv = idesc_f16kind_f32(BM, C::NPV, true, C::F16);
      int hp = 0, prev = n > 0 ? head_of(0) : -1;
      for (int ip = 0; ip < n; ++ip) {
        if (ip > 0 && head_of(ip) != prev) {
          prev = head_of(ip);
          ++hp;
        }
        const int slot = ip % NSLOT, b = hp % KVB;
        if (!wait_bar(bars.p_full(slot), (ip / NSLOT) & 1, abort_flag, err) ||
            !wait_bar(bars.v_ready(b), (hp / KVB) & 1, abort_flag, err))
          break;
        tc_fence_after();
        const uint32_t d = tmem + slot * C::TM_W + C::OFS_O, a = tmem + slot * C::TM_W;
#pragma unroll
        for (int ks = 0; ks < BN / 16; ++ks) {
          const uint64_t bd = smem_desc(sbase + C::V_OFF + b * C::V_BYTES + ks * 16 * 128, BN * 128, 1024);
          mma_ts(d, a + ks * 8, bd, idesc_pv, ks > 0 ? 1u : 0u);
        }
        mma_commit(bars.o_full(slot));
        if (ip + 1 == n || head_of(ip + 1) != prev) mma_commit(bars.kv_empty(b));
      }
      mma_commit(bars.fin(1));
      wait_bar(bars.fin(1), 0, abort_flag, err, false);
    } else if (warp == 3) {
      // ---------------------------------------------------------------- V fix-up
      // Writes 1.0 into column DH of every row of each landed V buffer (128-byte swizzled rows: the
      // 16-byte granule g of row r sits at granule g ^ (r % 8)), so P V also sums the row of P.
      constexpr int ch = C::DH / 64, byte = (C::DH % 64) * 2, g = byte >> 4, gb = byte & 15;
      int hv = -1, prev = -1;
      for (int i = 0; i < n; ++i) {
        const int bh = head_of(i);
        if (bh == prev) continue;
        prev = bh;
        ++hv;
        const int b = hv % KVB;
        if (!__all_sync(0xffffffffu, wait_bar(bars.v_full(b), (hv / KVB) & 1, abort_flag, err))) break;
        uint8_t* vt = smem + C::V_OFF + b * C::V_BYTES + ch * BN * 128;
        for (int r = lane; r < BN; r += 32)
          *reinterpret_cast<uint16_t*>(vt + r * 128 + ((g ^ (r & 7)) << 4) + gb) = C::F16 ? 0x3C00u : 0x3F80u;
        fence_proxy_async_smem();  // generic-proxy stores -> visible to the tensor core
        __syncwarp();
        if (lane == 0) mbar_arrive(bars.v_ready(b));
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------------ softmax + epilogue
    const int wg = (warp - C::SOFT_WARP0) >> 2;  // tiles wg, wg + 2, ...
    const int quarter = warp & 3;               // TMEM lane quarter this warp may access
    const int row = quarter * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    bool ok = true;

    auto softmax = [&](int i) -> bool {
      const int slot = i % NSLOT;
      if (!__all_sync(0xffffffffu, wait_bar(bars.s_full(slot), (i / NSLOT) & 1, abort_flag, err))) return false;
      tc_fence_after();
      const uint32_t tS = tmem + lane_off + slot * C::TM_W;
      float sv[BN];
      {
        uint32_t r0[32], r1[32], r2[16];
        tmem_ld32(tS, r0);
        tmem_ld32(tS + 32, r1);
        tmem_ld16(tS + 64, r2);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 32; ++j) sv[j] = __uint_as_float(r0[j]);
#pragma unroll
        for (int j = 0; j < 32; ++j) sv[32 + j] = __uint_as_float(r1[j]);
#pragma unroll
        for (int j = 0; j < 16; ++j) sv[64 + j] = __uint_as_float(r2[j]);
      }
#pragma unroll
      for (int j = 0; j < BN; ++j)
        if (j >= Lk) sv[j] = -INFINITY;
      float pm[16];
#pragma unroll
      for (int k = 0; k < 16; ++k) pm[k] = max3f(sv[k], sv[16 + k], sv[32 + k]);
#pragma unroll
      for (int k = 0; k < 16; ++k) pm[k] = max3f(pm[k], sv[48 + k], sv[64 + k]);
      const float mx = fmaxf(max3f(max3f(pm[0], pm[1], pm[2]), max3f(pm[3], pm[4], pm[5]), max3f(pm[6], pm[7], pm[8])),
                             max3f(max3f(pm[9], pm[10], pm[11]), max3f(pm[12], pm[13], pm[14]), pm[15]));
      const float neg_m = -mx * scale_log2;
      uint32_t pk[BN / 2];
#pragma unroll
      for (int b = 0; b < BN / 2; ++b) {
        float x0, x1;
        fma2(x0, x1, sv[2 * b], sv[2 * b + 1], scale_log2, scale_log2, neg_m, neg_m);
        if ((b & 7) < C::POLY) {  // FMA-pipe exp2 for POLY of every 8 pairs, the rest on the SFU
          exp2_poly2(x0, x1, x0, x1);
        } else {
          x0 = ex2_approx(x0);
          x1 = ex2_approx(x1);
        }
        pk[b] = C::F16 ? pack_f16x2(x0, x1) : pack_bf16x2(x0, x1);
      }
      // P over S: the scores are in registers, so the slot's first BN/2 columns take P
      {
        uint32_t a[16], c[16], e[8];
#pragma unroll
        for (int j = 0; j < 16; ++j) a[j] = pk[j];
#pragma unroll
        for (int j = 0; j < 16; ++j) c[j] = pk[16 + j];
#pragma unroll
        for (int j = 0; j < 8; ++j) e[j] = pk[32 + j];
        tmem_st16(tS, a);
        tmem_st16(tS + 16, c);
        tmem_st8(tS + 32, e);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bars.p_full(slot));
      return true;
    };

    auto epilogue = [&](int i) -> bool {
      const int slot = i % NSLOT;
      if (!__all_sync(0xffffffffu, wait_bar(bars.o_full(slot), (i / NSLOT) & 1, abort_flag, err))) return false;
      tc_fence_after();
      const uint32_t tO = tmem + lane_off + slot * C::TM_W + C::OFS_O;
      const int bh = head_of(i), qrow = row0_of(i) + row;
      const size_t orow = C::BLHD ? (static_cast<size_t>(bh / lay_heads) * Lq + qrow) * lay_heads + bh % lay_heads
                                  : static_cast<size_t>(bh) * Lq + qrow;
      uint4* dst = reinterpret_cast<uint4*>(out + orow * dh);
      // 16 O columns -> 8 packed pairs -> two 16-byte stores (the last group of dh 40 is one store)
      auto store16 = [&](int c, const uint32_t (&r)[16], float inv_l) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          if (c * 2 + h >= C::DH / 8) break;
          uint32_t w[4];
#pragma unroll
          for (int j = 0; j < 4; ++j)
            w[j] = C::F16 ? pack_f16x2(__uint_as_float(r[8 * h + 2 * j]) * inv_l, __uint_as_float(r[8 * h + 2 * j + 1]) * inv_l)
                          : pack_bf16x2(__uint_as_float(r[8 * h + 2 * j]) * inv_l, __uint_as_float(r[8 * h + 2 * j + 1]) * inv_l);
          if (qrow < Lq) dst[c * 2 + h] = make_uint4(w[0], w[1], w[2], w[3]);
        }
      };
      constexpr int NC = C::NPV / 16;
      if constexpr (C::NPV <= 96) {  // all of O in registers, one wait
        uint32_t ov[NC][16];
#pragma unroll
        for (int c = 0; c < NC; ++c) tmem_ld16(tO + c * 16, ov[c]);
        tmem_wait_ld();
        tc_fence_before();
        mbar_arrive(bars.slot_free(slot));  // O is in registers: the slot may take the next tile
        const float inv_l = 1.0f / __uint_as_float(ov[C::DH / 16][C::DH % 16]);
#pragma unroll
        for (int c = 0; c < NC; ++c) store16(c, ov[c], inv_l);
      } else {  // wide heads: the row-sum chunk first, then O 16 columns at a time
        uint32_t lc[16];
        tmem_ld16(tO + (C::DH / 16) * 16, lc);
        tmem_wait_ld();
        const float inv_l = 1.0f / __uint_as_float(lc[C::DH % 16]);
#pragma unroll 1
        for (int c = 0; c < C::DH / 16; ++c) {
          uint32_t r[16];
          tmem_ld16(tO + c * 16, r);
          tmem_wait_ld();
          store16(c, r, inv_l);
        }
        tc_fence_before();
        mbar_arrive(bars.slot_free(slot));
      }
      return true;
    };

    // Each warp takes whichever of its warpgroup's next steps is ready: the epilogue of its oldest
    // tile whose O is complete, else the softmax of its next tile whose S is complete. Probing a
    // barrier of tile i only after this warp finished tile i - NWG is safe: the issuers work in tile
    // order and a commit covers all of the issuing thread's earlier MMAs, so the slot's previous phase
    // has completed and a parity probe cannot see a stale phase.
    int ns = wg, ne = wg;  // next tile to softmax, next tile to write out
    long long t_idle = clock64();
    uint32_t spins = 0;
    while (ok && ne < n) {
      if (ne < ns && __all_sync(0xffffffffu, mbar_test_wait(bars.o_full(ne % NSLOT), (ne / NSLOT) & 1))) {
        if (!epilogue(ne)) ok = false;
        ne += C::NWG;
        t_idle = clock64();
        continue;
      }
      if (ns < n && __all_sync(0xffffffffu, mbar_test_wait(bars.s_full(ns % NSLOT), (ns / NSLOT) & 1))) {
        if (!softmax(ns)) ok = false;
        ns += C::NWG;
        t_idle = clock64();
        continue;
      }
      if ((++spins & 31u) == 0) {
        if (*abort_flag) ok = false;
        else if (clock64() - t_idle > kWaitLimitCycles) {
          *abort_flag = 1;
          atomicOr(err, sd::kDevErrTimeout);
          ok = false;
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <class C>
sd_status launch_cfg(const void* q, const void* k, const void* v, void* o, int64_t BH, int64_t Lq, int64_t Lk,
                     int64_t dh, float scale, cudaStream_t s, int64_t lay_heads) {
  CUtensorMap mq, mk, mv;
  sd_status st = make_map(&mq, q, dh, Lq, BH, BM, C::F16, lay_heads);
  if (st == SD_OK) st = make_map(&mk, k, dh, Lk, BH, C::BN, C::F16, lay_heads);
  if (st == SD_OK) st = make_map(&mv, v, dh, Lk, BH, C::BN, C::F16, lay_heads);
  if (st != SD_OK) return st;
  unsigned int* err = sd::device_status_word();
  if (!err) return SD_ERR_CUDA;
  auto kern = attn_short_sm100<C>;
  static std::atomic<uint64_t> smem_set{0};  // one bit per device: opt-in to large shared memory done
  int dev = 0;
  st = sd::cuda_check(cudaGetDevice(&dev), "cudaGetDevice");
  if (st != SD_OK) return st;
  const uint64_t bit = uint64_t(1) << (dev & 63);
  if (!(smem_set.load(std::memory_order_acquire) & bit)) {
    st = sd::cuda_check(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES),
                        "cudaFuncSetAttribute(short attention smem)");
    if (st != SD_OK) return st;
    smem_set.fetch_or(bit, std::memory_order_acq_rel);
  }
  const int64_t tph = (Lq + BM - 1) / BM;  // query tiles per (batch, head) plane
  const int64_t n_tiles = BH * tph;
  if (tph > 0x7fffffff || n_tiles > (int64_t(1) << 40)) return sd::fail(SD_ERR_UNSUPPORTED, "sd_attention: too many tiles");
  const int64_t G = std::min<int64_t>(sd::sm_count(), n_tiles);
  if (n_tiles / G > 0x7fffffff) return sd::fail(SD_ERR_UNSUPPORTED, "sd_attention: too many tiles per CTA");
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(G));
  cfg.blockDim = dim3(C::THREADS);
  cfg.dynamicSmemBytes = C::SMEM_BYTES;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  cfg.attrs = attr;
  cfg.numAttrs = sd::pdl_attr(&attr[0]);
  return sd::cuda_check(cudaLaunchKernelEx(&cfg, kern, mq, mk, mv, static_cast<uint16_t*>(o), static_cast<int>(Lq),
                                           static_cast<int>(Lk), static_cast<int>(dh), scale * 1.4426950408889634f, err,
                                           g_debug_flags, static_cast<int>(tph), static_cast<long long>(n_tiles),
                                           static_cast<int>(lay_heads)),
                        "sd_attention (short key sequence) launch");
}

// ------------------------------------------------------------------ one query tile per CTA
// The default form: a CTA takes one 128-row query tile, so the GPU runs several tiles' chains
// (loads, S, softmax, P V, stores) at once on every SM and their latencies overlap; three to four
// of these CTAs fit one SM. Tensor memory of a CTA: S in columns [0, 80), P written over its first
// 40 columns, and O (then the row sum for L_IN_V) from column OFS_O, over the columns of S that the
// softmax has already read: 128 columns for dh 40 and 64, 256 for dh 80 and 160.
template <int DH_, bool F16_, bool BLHD_>
struct TileCfg {
  static constexpr int DH = DH_;
  static constexpr bool F16 = F16_;
  static constexpr bool BLHD = BLHD_;
  static constexpr int BN = kShortMaxKeys;
  static constexpr int POLY = SD_SHORT_POLY;
  static constexpr int DHP = (DH + 15) / 16 * 16;
  static constexpr bool L_IN_V = DH != 64;  // the row sum from a ones column, except where it would widen V
  static constexpr int NPV = L_IN_V ? (DH + 1 + 15) / 16 * 16 : DHP;
  static constexpr int NCH = (DHP + 63) / 64;
  static constexpr int NCHV = (NPV + 63) / 64;
  static constexpr int Q_BYTES = NCH * BM * 128;
  static constexpr int K_BYTES = NCH * BN * 128;
  static constexpr int V_BYTES = NCHV * BN * 128;
  static constexpr int Q_OFF = 0, K_OFF = Q_BYTES, V_OFF = K_OFF + K_BYTES;
  static constexpr int BAR_OFF = V_OFF + V_BYTES;
  // qk_full, v_full, v_ready, s_full, p_full, o_full, fin
  static constexpr int NBARS = 7;
  static constexpr int MISC_OFF = BAR_OFF + NBARS * 8;
  static constexpr int SMEM_BYTES = MISC_OFF + 16 + 1024;
  static constexpr int OFS_O = BN / 2 + 8;  // past P (BN / 2 columns), 16-aligned
  static constexpr int TM_COLS = OFS_O + NPV <= 128 ? 128 : 256;
  static constexpr int THREADS = 160;  // warp 0: loads, MMAs, V fix-up; warps 1-4: softmax, epilogue
  static_assert(OFS_O % 16 == 0 && OFS_O + NPV <= TM_COLS, "tensor-memory layout");
};

template <class C>
__global__ void __launch_bounds__(C::THREADS, C::TM_COLS == 128 ? 4 : 2)
    attn_tile_sm100(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, uint16_t* __restrict__ out, int Lq, int Lk, int dh,
                    float scale_log2, unsigned int* err, int debug_flags, int tiles_per_head, int lay_heads) {
  constexpr int BN = C::BN, NCH = C::NCH, NCHV = C::NCHV;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar = sbase + C::BAR_OFF;
  const uint32_t qk_full = bar, v_full = bar + 8, v_ready = bar + 16, s_full = bar + 24, p_full = bar + 32,
                 o_full = bar + 40, fin = bar + 48;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::MISC_OFF + 4);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = static_cast<int>(blockIdx.x / static_cast<unsigned>(tiles_per_head));
  const int row0 = static_cast<int>(blockIdx.x % static_cast<unsigned>(tiles_per_head)) * BM;

  if (threadIdx.x == 0) {
    mbar_init(qk_full, 1);
    mbar_init(v_full, 1);
    mbar_init(v_ready, 1);
    mbar_init(s_full, 1);
    mbar_init(p_full, 128);
    mbar_init(o_full, 1);
    mbar_init(fin, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), C::TM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  sd::grid_dep_wait();
  sd::grid_dep_launch();

  if (warp == 0) {
    if (lane == 0) {
      // loads, then S = Q K^T once Q and K have landed, then O = P V once P is written
      mbar_arrive_expect_tx(qk_full, C::Q_BYTES + C::K_BYTES);
      for (int c = 0; c < NCH; ++c) {
        load_rows<C::BLHD>(sbase + C::Q_OFF + c * BM * 128, &tm_q, qk_full, c * 64, row0, bh, lay_heads);
        load_rows<C::BLHD>(sbase + C::K_OFF + c * BN * 128, &tm_k, qk_full, c * 64, 0, bh, lay_heads);
      }
      const bool skip_v = debug_flags & 1;  // test hook: V never arrives, the waits below expire
      if (!skip_v) {
        mbar_arrive_expect_tx(v_full, C::V_BYTES);
        for (int c = 0; c < NCHV; ++c)
          load_rows<C::BLHD>(sbase + C::V_OFF + c * BN * 128, &tm_v, v_full, c * 64, 0, bh, lay_heads);
      }
      constexpr uint32_t idesc_qk = idesc_f16kind_f32(BM, BN, false, C::F16);
      constexpr uint32_t idesc_pv = idesc_f16kind_f32(BM, C::NPV, true, C::F16);
      bool issued_pv = false;
      if (wait_bar(qk_full, 0, abort_flag, err)) {
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < C::DHP / 16; ++ks) {
          const uint32_t off = (ks >> 2) * (BM * 128) + (ks & 3) * 32;
          const uint32_t offk = (ks >> 2) * (BN * 128) + (ks & 3) * 32;
          mma_ss(tmem, smem_desc(sbase + C::Q_OFF + off, 16, 1024), smem_desc(sbase + C::K_OFF + offk, 16, 1024),
                 idesc_qk, ks > 0 ? 1u : 0u);
        }
        mma_commit(s_full);
        if (wait_bar(p_full, 0, abort_flag, err) && wait_bar(C::L_IN_V ? v_ready : v_full, 0, abort_flag, err)) {
          tc_fence_after();
#pragma unroll
          for (int ks = 0; ks < BN / 16; ++ks)
            mma_ts(tmem + C::OFS_O, tmem + ks * 8, smem_desc(sbase + C::V_OFF + ks * 16 * 128, BN * 128, 1024), idesc_pv,
                   ks > 0 ? 1u : 0u);
          mma_commit(o_full);
          issued_pv = true;
        }
      }
      mma_commit(fin);
      wait_bar(fin, 0, abort_flag, err, false);
      // drain: the copies issued above have landed before the CTA may exit
      wait_bar(qk_full, 0, abort_flag, err, false);
      if (!skip_v) wait_bar(v_full, 0, abort_flag, err, false);
      (void)issued_pv;
    } else if constexpr (C::L_IN_V) {
      // V fix-up: 1.0 in column DH of every key row (128-byte swizzle: granule g of row r at g ^ (r % 8))
      constexpr int ch = C::DH / 64, byte = (C::DH % 64) * 2, g = byte >> 4, gb = byte & 15;
      if (__all_sync(0xfffffffeu, wait_bar(v_full, 0, abort_flag, err))) {
        uint8_t* vt = smem + C::V_OFF + ch * BN * 128;
        for (int r = lane - 1; r < BN; r += 31)
          *reinterpret_cast<uint16_t*>(vt + r * 128 + ((g ^ (r & 7)) << 4) + gb) = C::F16 ? 0x3C00u : 0x3F80u;
        fence_proxy_async_smem();
        __syncwarp(0xfffffffeu);
        if (lane == 1) mbar_arrive(v_ready);
      }
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- softmax and epilogue
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t tl = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    if (__all_sync(0xffffffffu, wait_bar(s_full, 0, abort_flag, err))) {
      tc_fence_after();
      float sv[BN];
      {
        uint32_t r0[32], r1[32], r2[16];
        tmem_ld32(tl, r0);
        tmem_ld32(tl + 32, r1);
        tmem_ld16(tl + 64, r2);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 32; ++j) sv[j] = __uint_as_float(r0[j]);
#pragma unroll
        for (int j = 0; j < 32; ++j) sv[32 + j] = __uint_as_float(r1[j]);
#pragma unroll
        for (int j = 0; j < 16; ++j) sv[64 + j] = __uint_as_float(r2[j]);
      }
#pragma unroll
      for (int j = 0; j < BN; ++j)
        if (j >= Lk) sv[j] = -INFINITY;
      float pm[16];
#pragma unroll
      for (int k = 0; k < 16; ++k) pm[k] = max3f(sv[k], sv[16 + k], sv[32 + k]);
#pragma unroll
      for (int k = 0; k < 16; ++k) pm[k] = max3f(pm[k], sv[48 + k], sv[64 + k]);
      const float mx = fmaxf(max3f(max3f(pm[0], pm[1], pm[2]), max3f(pm[3], pm[4], pm[5]), max3f(pm[6], pm[7], pm[8])),
                             max3f(max3f(pm[9], pm[10], pm[11]), max3f(pm[12], pm[13], pm[14]), pm[15]));
      const float neg_m = -mx * scale_log2;
      uint32_t pk[BN / 2];
      float ls0 = 0.f, ls1 = 0.f;
#pragma unroll
      for (int b = 0; b < BN / 2; ++b) {
        float x0, x1;
        fma2(x0, x1, sv[2 * b], sv[2 * b + 1], scale_log2, scale_log2, neg_m, neg_m);
        if ((b & 7) < C::POLY) {
          exp2_poly2(x0, x1, x0, x1);
        } else {
          x0 = ex2_approx(x0);
          x1 = ex2_approx(x1);
        }
        if constexpr (!C::L_IN_V) add2(ls0, ls1, ls0, ls1, x0, x1);
        pk[b] = C::F16 ? pack_f16x2(x0, x1) : pack_bf16x2(x0, x1);
      }
      {
        uint32_t a[16], c[16], e[8];
#pragma unroll
        for (int j = 0; j < 16; ++j) a[j] = pk[j];
#pragma unroll
        for (int j = 0; j < 16; ++j) c[j] = pk[16 + j];
#pragma unroll
        for (int j = 0; j < 8; ++j) e[j] = pk[32 + j];
        tmem_st16(tl, a);
        tmem_st16(tl + 16, c);
        tmem_st8(tl + 32, e);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(p_full);
      if (__all_sync(0xffffffffu, wait_bar(o_full, 0, abort_flag, err))) {
        tc_fence_after();
        const uint32_t tO = tl + C::OFS_O;
        const int qrow = row0 + row;
        const size_t orow = C::BLHD ? (static_cast<size_t>(bh / lay_heads) * Lq + qrow) * lay_heads + bh % lay_heads
                                    : static_cast<size_t>(bh) * Lq + qrow;
        uint4* dst = reinterpret_cast<uint4*>(out + orow * dh);
        float inv_l;
        if constexpr (C::L_IN_V) {
          uint32_t lc[16];
          tmem_ld16(tO + (C::DH / 16) * 16, lc);
          tmem_wait_ld();
          inv_l = 1.0f / __uint_as_float(lc[C::DH % 16]);
        } else {
          inv_l = 1.0f / (ls0 + ls1);
        }
#pragma unroll 2
        for (int c = 0; c < C::DH / 16 + (C::DH % 16 ? 1 : 0); ++c) {
          uint32_t r[16];
          tmem_ld16(tO + c * 16, r);
          tmem_wait_ld();
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            if (c * 2 + h >= C::DH / 8) break;
            uint32_t w[4];
#pragma unroll
            for (int j = 0; j < 4; ++j)
              w[j] = C::F16 ? pack_f16x2(__uint_as_float(r[8 * h + 2 * j]) * inv_l, __uint_as_float(r[8 * h + 2 * j + 1]) * inv_l)
                            : pack_bf16x2(__uint_as_float(r[8 * h + 2 * j]) * inv_l, __uint_as_float(r[8 * h + 2 * j + 1]) * inv_l);
            if (qrow < Lq) dst[c * 2 + h] = make_uint4(w[0], w[1], w[2], w[3]);
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TM_COLS);
  }
}

template <class C>
sd_status launch_tile(const void* q, const void* k, const void* v, void* o, int64_t BH, int64_t Lq, int64_t Lk,
                      int64_t dh, float scale, cudaStream_t s, int64_t lay_heads) {
  CUtensorMap mq, mk, mv;
  sd_status st = make_map(&mq, q, dh, Lq, BH, BM, C::F16, lay_heads);
  if (st == SD_OK) st = make_map(&mk, k, dh, Lk, BH, C::BN, C::F16, lay_heads);
  if (st == SD_OK) st = make_map(&mv, v, dh, Lk, BH, C::BN, C::F16, lay_heads);
  if (st != SD_OK) return st;
  unsigned int* err = sd::device_status_word();
  if (!err) return SD_ERR_CUDA;
  auto kern = attn_tile_sm100<C>;
  static std::atomic<uint64_t> smem_set{0};
  int dev = 0;
  st = sd::cuda_check(cudaGetDevice(&dev), "cudaGetDevice");
  if (st != SD_OK) return st;
  const uint64_t bit = uint64_t(1) << (dev & 63);
  if (!(smem_set.load(std::memory_order_acquire) & bit)) {
    st = sd::cuda_check(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES),
                        "cudaFuncSetAttribute(tile attention smem)");
    if (st != SD_OK) return st;
    smem_set.fetch_or(bit, std::memory_order_acq_rel);
  }
  const int64_t tph = (Lq + BM - 1) / BM;
  const int64_t n_tiles = BH * tph;
  if (n_tiles > 0x7fffffff) return sd::fail(SD_ERR_UNSUPPORTED, "sd_attention: too many query tiles");
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(n_tiles));
  cfg.blockDim = dim3(C::THREADS);
  cfg.dynamicSmemBytes = C::SMEM_BYTES;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  cfg.attrs = attr;
  cfg.numAttrs = sd::pdl_attr(&attr[0]);
  return sd::cuda_check(cudaLaunchKernelEx(&cfg, kern, mq, mk, mv, static_cast<uint16_t*>(o), static_cast<int>(Lq),
                                           static_cast<int>(Lk), static_cast<int>(dh), scale * 1.4426950408889634f, err,
                                           g_debug_flags, static_cast<int>(tph), static_cast<int>(lay_heads)),
                        "sd_attention (one query tile per CTA) launch");
}

template <bool F16, bool BLHD>
sd_status dispatch_dh(const void* q, const void* k, const void* v, void* o, int64_t BH, int64_t Lq, int64_t Lk,
                      int64_t dh, float scale, cudaStream_t s, int64_t lay_heads) {
  // One tile per CTA while every tile fits one wave of resident CTAs (their chains then overlap);
  // beyond that, the persistent form, whose CTAs keep up to 8 tiles' loads in flight.
  const int64_t n_tiles = BH * ((Lq + BM - 1) / BM);
  const int per_sm = (dh == 40 || dh == 64) ? 4 : 2;  // the tile kernel's resident CTAs per SM
  if (!SD_SHORT_PERSIST && n_tiles <= static_cast<int64_t>(per_sm) * sd::sm_count()) {
    switch (dh) {
      case 40: return launch_tile<TileCfg<40, F16, BLHD>>(q, k, v, o, BH, Lq, Lk, dh, scale, s, lay_heads);
      case 64: return launch_tile<TileCfg<64, F16, BLHD>>(q, k, v, o, BH, Lq, Lk, dh, scale, s, lay_heads);
      case 80: return launch_tile<TileCfg<80, F16, BLHD>>(q, k, v, o, BH, Lq, Lk, dh, scale, s, lay_heads);
      case 160: return launch_tile<TileCfg<160, F16, BLHD>>(q, k, v, o, BH, Lq, Lk, dh, scale, s, lay_heads);
      default: return sd::fail(SD_ERR_UNSUPPORTED, "sd_attention: head dim %lld", (long long)dh);
    }
  }
  switch (dh) {
    case 40: return launch_cfg<ShortCfg<40, F16, BLHD>>(q, k, v, o, BH, Lq, Lk, dh, scale, s, lay_heads);
    case 64: return launch_cfg<ShortCfg<64, F16, BLHD>>(q, k, v, o, BH, Lq, Lk, dh, scale, s, lay_heads);
    case 80: return launch_cfg<ShortCfg<80, F16, BLHD>>(q, k, v, o, BH, Lq, Lk, dh, scale, s, lay_heads);
    case 160: return launch_cfg<ShortCfg<160, F16, BLHD>>(q, k, v, o, BH, Lq, Lk, dh, scale, s, lay_heads);
    default: return sd::fail(SD_ERR_UNSUPPORTED, "sd_attention: head dim %lld", (long long)dh);
  }
}

}  // namespace

sd_status sd::attn::launch_short(const void* q, const void* k, const void* v, void* o, int64_t BH, int64_t Lq,
                                 int64_t Lk, int64_t dh, float scale, cudaStream_t s, bool f16, int64_t lay_heads) {
  if (lay_heads)
    return f16 ? dispatch_dh<true, true>(q, k, v, o, BH, Lq, Lk, dh, scale, s, lay_heads)
               : dispatch_dh<false, true>(q, k, v, o, BH, Lq, Lk, dh, scale, s, lay_heads);
  return f16 ? dispatch_dh<true, false>(q, k, v, o, BH, Lq, Lk, dh, scale, s, lay_heads)
             : dispatch_dh<false, false>(q, k, v, o, BH, Lq, Lk, dh, scale, s, lay_heads);
}
