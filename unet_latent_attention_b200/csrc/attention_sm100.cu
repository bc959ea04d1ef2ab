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
//  * One thread issues the tensor-core work from an event loop over the query tiles: S = Q K^T
//    (tcgen05.mma, bf16 in, fp32 accumulate, M = 128, N = BN, K = 16 per instruction) into tensor
//    memory, O += P V with P read straight from tensor memory (the "A in TMEM" form) and V from
//    shared memory (N-major B), and l += P * ones (a 16-column MMA against an all-ones tile) for
//    the softmax row sums, so the sums use exactly the bf16 probabilities that multiply V.
//  * Four warps per query tile (one TMEM lane quarter each, one thread per row) run the softmax:
//    tcgen05.ld the S row and release it (the next S = Q K^T starts at once), row max over
//    independent 3-input-max chains, exp2 with scale*log2(e) folded into one packed FMA, pack to
//    bf16 and tcgen05.st P into its own TMEM columns once the previous P V has consumed them. The
//    running max is only raised when it grows by more than 2^8 (lazy rescaling), so most tiles
//    skip the O correction; normalisation by l is deferred to the epilogue, which equals the
//    page's per-step form in exact arithmetic.
//  * Two query tiles per CTA (NQ = 2) share every K/V tile, halving L2->SM traffic, and keep the
//    tensor core busy with one tile while the other is in its softmax.
//  * Every wait on an mbarrier is bounded (about one second); on expiry the CTA records
//    SD_ERR_TIMEOUT in the device status word, drains its own in-flight copies and MMAs, frees its
//    tensor memory and returns. Nothing traps.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <algorithm>
#include <cmath>
#include <map>
#include <mutex>
#include <tuple>
#include <vector>

#include "sd_internal.h"
#include "sm100_ptx.cuh"
#include "attn_common.cuh"

namespace sd {
namespace attn {

int g_debug_flags = 0;

static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
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

sd_status make_map(CUtensorMap* map, const void* ptr, int64_t dh, int64_t rows, int64_t planes, int box_rows,
                   bool f16, int64_t lay_heads) {
  auto fn = encode_fn();
  if (!fn) return sd::fail(SD_ERR_CUDA, "sd_attention: cuTensorMapEncodeTiled is unavailable");
  const cuuint32_t rank = lay_heads ? 4 : 3;
  cuuint64_t dims[4], strides[3];
  cuuint32_t box[4];
  if (lay_heads) {
    dims[0] = dh, dims[1] = lay_heads, dims[2] = rows, dims[3] = planes / lay_heads;
    strides[0] = dh * 2, strides[1] = lay_heads * dh * 2, strides[2] = rows * lay_heads * dh * 2;
    box[0] = 64, box[1] = 1, box[2] = static_cast<cuuint32_t>(box_rows), box[3] = 1;
  } else {
    dims[0] = dh, dims[1] = rows, dims[2] = planes;
    strides[0] = dh * 2, strides[1] = rows * dh * 2;
    box[0] = 64, box[1] = static_cast<cuuint32_t>(box_rows), box[2] = 1;
  }
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  const CUresult r = fn(map, f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank,
                        const_cast<void*>(ptr), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return sd::fail(SD_ERR_CUDA, "sd_attention: cuTensorMapEncodeTiled failed (%d)", (int)r);
  return SD_OK;
}


}  // namespace attn
}  // namespace sd

namespace {

using namespace sm100;
using namespace sd::attn;

enum : int { kSplitPublish = 1, kSplitMerge = 2, kSplitAbort = 3 };  // split hand-off decisions

#ifndef SD_POLY_PAIRS
#define SD_POLY_PAIRS -1  // tuning override of the per-head-dim choice in the launch table
#endif

#ifndef SD_P_CHUNKED
#define SD_P_CHUNKED -1  // tuning override of Cfg::CHUNK_P (-1: the per-config choice)
#endif

#ifndef SD_PING_RELEASE
#define SD_PING_RELEASE -1  // tuning override of Cfg::PING_RELEASE (-1: the per-config choice)
#endif

#ifndef SD_REGSPLIT
#define SD_REGSPLIT 1  // setmaxnreg: 120 registers per helper thread, 192 per softmax thread (two query tiles)
#endif

#ifndef SD_PINGPONG
#define SD_PINGPONG 1  // alternate the two query tiles' exp2 phases on each SM sub-partition
#endif

#ifndef SD_CROSS_NQ
#define SD_CROSS_NQ 2  // query tiles per CTA for key sequences of at most 96 tokens
#endif

#ifndef SD_EXP_BLOCK
#define SD_EXP_BLOCK 1  // column pairs per exp2 block (1 = pair by pair)
#endif

#ifndef SD_PING_SHORT
#define SD_PING_SHORT 1  // ping-pong also for the single 96-key tile of short key sequences
#endif

#ifndef SD_SMALL_NQ1
#define SD_SMALL_NQ1 1  // one query tile per CTA while there are at most this many query tiles per SM
#endif

#ifndef SD_STAGES_SMALL
#define SD_STAGES_SMALL 4  // K/V ring depth for head dims <= 64 (one 16 KB K and V tile per stage)
#endif


// P_SEP: P has its own TMEM columns (else it overwrites S, and the next S waits for P V).
// L_IN_V: the softmax row sums come out of the P V product itself: a fix-up warp writes bf16 1.0
//         into column DH of every V tile once it lands (the TMA zero-fills columns >= DH), so O's
//         column DH accumulates sum_j P_ij with no extra MMA (else fp32 adds in registers).
// F16: the tensors (and P) are fp16 instead of bf16. BLHD: the tensors are [B, L, heads, dh]
// instead of [B, heads, L, dh] (a compile-time choice, so that the default layout's code is not
// touched by the other's addressing).
template <int DH_, int BN_, int NQ_, int STAGES_, bool P_SEP_, bool L_IN_V_, int POLY_ = 0, bool F16_ = false,
          bool BLHD_ = false>
struct Cfg {
  static constexpr bool F16 = F16_;
  static constexpr bool BLHD = BLHD_;
  static constexpr int DH = DH_;          // true head dim
  static constexpr int DHP = (DH + 15) / 16 * 16;  // Q K^T depth padded to the MMA granule (16)
  static constexpr int BN = BN_;          // keys per K/V tile
  static constexpr int NQ = NQ_;          // 128-row query tiles per CTA
  static constexpr int STAGES = STAGES_;  // K/V ring depth
  static constexpr bool P_SEP = P_SEP_;
  static constexpr bool L_IN_V = L_IN_V_;
  static constexpr int NPV = L_IN_V ? (DH + 1 + 15) / 16 * 16 : DHP;  // N of O += P V (O, then l)
  static constexpr int NCH = (DHP + 63) / 64;    // 64-element (128-byte) swizzle chunks of Q and K
  static constexpr int NCHV = (NPV + 63) / 64;   // chunks of a V tile (the ones column included)
  static constexpr int Q_TILE_BYTES = NCH * BM * 128;
  static constexpr int K_TILE_BYTES = NCH * BN * 128;
  static constexpr int V_TILE_BYTES = NCHV * BN * 128;
  static constexpr int Q_OFF = 0;
  // Two Q buffers (when shared memory allows) let the next item's Q load during this one.
  static constexpr int QBUF = 2 * NQ * NCH * BM * 128 + STAGES * (NCH + NCHV) * BN * 128 <= 200 * 1024 ? 2 : 1;
  static constexpr int K_OFF = Q_OFF + QBUF * NQ * Q_TILE_BYTES;
  static constexpr int V_OFF = K_OFF + STAGES * K_TILE_BYTES;
  static constexpr int BAR_OFF = V_OFF + STAGES * V_TILE_BYTES;
  // q_full, k_full[S], v_full[S], v_ready[S], kv_empty[S], s_full[NQ], s_free[NQ], p_full[NQ], o_done[NQ],
  // fin[NQ], the exp tokens tok[2][4] of the two tiles' warps on each SM sub-partition, q_empty[2],
  // split_dec[2], split_written[2]
  static constexpr int NBARS = 2 + 4 * STAGES + 5 * NQ + 8 + 2 + 4;
  static constexpr int MISC_OFF = BAR_OFF + NBARS * 8;
  // misc: TMEM base address, abort flag, the split hand-off decisions of the two piece kinds
  static constexpr int SMEM_BYTES = MISC_OFF + 16 + 1024;  // + slack to align the base to 1024
  // TMEM columns of one query tile: S | P (if separate) | O (NPV columns, l at column DH)
  static constexpr int TM_S = 0;
  static constexpr int TM_P = P_SEP ? BN : 0;
  static constexpr int TM_O = BN + (P_SEP ? BN / 2 : 0);
  static constexpr int TM_USED = TM_O + NPV;
  static constexpr int TM_TILE = TM_USED <= 256 ? 256 : 512;
  static constexpr int TM_COLS = NQ * TM_TILE;
  // Warpgroup 0 holds the helpers -- warp 0: TMA producer; warp 1: MMA issuer of tile 0 (and TMEM
  // owner); warp 2: MMA issuer of tile 1; warp 3: V fix-up (L_IN_V) -- and warpgroups 1 .. NQ run
  // the softmax of one query tile each (warp w reads TMEM lane quarter w % 4).
  static_assert(NQ <= 2, "two MMA issuers in warpgroup 0");
  static constexpr int FIX_WARP = 3;
  static constexpr int SOFT_WARP0 = 4;
  static constexpr int NUM_WARPS = 4 + 4 * NQ;
  static constexpr int THREADS = 32 * NUM_WARPS;
  // Register split (setmaxnreg) for NQ = 2: the helper warpgroup drops to REG_HELPER per thread and
  // the two softmax warpgroups rise to REG_SOFT, within the launch's 384 x 168 (measured on B200:
  // 120 / 192 is 3-5% faster than no split at dh 40, 64 and 80; 56 / 224 starves the helpers).
  static constexpr int REG_HELPER = 120, REG_SOFT = 192;
  static_assert(NQ != 2 || 128 * REG_HELPER + 256 * REG_SOFT <= 168 * 384, "register split exceeds the launch budget");
  // Split-item hand-off slot: raw O (NPV fp32 per row) and (m, l) per row of the NQ tiles.
  static constexpr int SLOT_FLOATS = NQ * BM * (NPV + 2);
  // Column pairs after which a softmax warp passes the ping-pong token (measured: half-way for
  // dh 64, whose exp2 loop also sums the row in fp32; at the end of the loop otherwise).
  static constexpr int PING_RELEASE = (DH == 64 && BN == 128) ? BN / 4 : BN / 2;
  // Store P in 16-column chunks inside the exp2 loop (measured: faster for the single short key
  // tile of cross-attention, slower for the long key loops).
  static constexpr bool CHUNK_P = BN < 128;
  // Costs of the persistent schedule in K/V-tile units (measured; see part_ranges).
  static constexpr double COST_SEG = DH == 64 ? 1.3 : 1.0, COST_TAIL = DH == 64 ? 0.5 : 0.6,
                          COST_HEAD = DH == 64 ? 1.4 : 0.9;
  // Of every 8 column pairs, this many take the FMA-pipe exp2 instead of the special-function unit.
  static constexpr int POLY_PAIRS = SD_POLY_PAIRS >= 0 ? SD_POLY_PAIRS : POLY_;
  static_assert(NPV % 16 == 0 && NPV <= 256, "MMA N must be a multiple of 16 and at most 256");
  static_assert(BN % 32 == 0, "S is read in 32-column chunks");
  static_assert(TM_COLS <= 512, "tensor memory holds 512 columns");
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
};

struct Bars {
  uint32_t base;
  int stages, nq;
  __device__ uint32_t q_full(int b) const { return base + 8 * b; }
  __device__ uint32_t k_full(int s) const { return base + 8 * (2 + s); }
  __device__ uint32_t v_full(int s) const { return base + 8 * (2 + stages + s); }
  __device__ uint32_t v_ready(int s) const { return base + 8 * (2 + 2 * stages + s); }
  __device__ uint32_t kv_empty(int s) const { return base + 8 * (2 + 3 * stages + s); }
  __device__ uint32_t s_full(int t) const { return base + 8 * (2 + 4 * stages + t); }
  __device__ uint32_t s_free(int t) const { return base + 8 * (2 + 4 * stages + nq + t); }
  __device__ uint32_t p_full(int t) const { return base + 8 * (2 + 4 * stages + 2 * nq + t); }
  __device__ uint32_t o_done(int t) const { return base + 8 * (2 + 4 * stages + 3 * nq + t); }
  __device__ uint32_t fin() const { return base + 8 * (2 + 4 * stages + 4 * nq); }
  __device__ uint32_t tok(int t, int q) const { return base + 8 * (2 + 4 * stages + 5 * nq + 4 * t + q); }
  __device__ uint32_t q_empty(int b) const { return base + 8 * (2 + 4 * stages + 5 * nq + 8 + b); }
  // split-item hand-off of the tail piece (kind 0) and the head piece (kind 1): the MMA issuer's
  // decision is published, and this piece's slot has been written by every softmax thread
  __device__ uint32_t split_dec(int kind) const { return base + 8 * (2 + 4 * stages + 5 * nq + 10 + kind); }
  __device__ uint32_t split_written(int kind) const { return base + 8 * (2 + 4 * stages + 5 * nq + 12 + kind); }
};

// Persistent schedule: the work is items x nkv units (an item = NQ query tiles of one (b, h); a
// unit = one K/V tile of it). CTA c owns units [c U / G, (c+1) U / G) in item-major order, so every
// CTA gets the same amount of work whatever the number of SMs; with G <= items each range spans at
// least nkv units, so an item is split across at most two CTAs: a "head" piece [0, k) at the end
// of CTA c's range and a "tail" piece [k, nkv) at the start of CTA c+1's range.
struct Seg {
  int it, kb, ke;
};

// Unit ranges of the persistent grid: CTA c owns units [u[c], u[c+1]). Passed by value (kernel
// parameter space), filled on the host: evenly, or balanced by a cost model (see part_ranges).
constexpr int kMaxCtas = 256;
constexpr size_t kCounterBytes = kMaxCtas * sizeof(unsigned int);  // split-item counters, workspace head
struct Part {
  long long u[kMaxCtas + 1];
};

// One tile of rows [row, row + box) of head plane bh, 64 head-dim columns from x. lay_heads = 0:
// tensors [B*heads, L, dh] (3-D map); lay_heads = heads: tensors [B, L, heads, dh] (4-D map over
// {dh, heads, L, B}). Both put the same rows x 128 bytes into shared memory.
__device__ __forceinline__ bool next_seg(long long& u, long long u1, int nkv, Seg& sg) {
  if (u >= u1) return false;
  sg.it = static_cast<int>(u / nkv);
  sg.kb = static_cast<int>(u % nkv);
  const long long rest = u1 - u;
  sg.ke = rest < nkv - sg.kb ? sg.kb + static_cast<int>(rest) : nkv;
  u += sg.ke - sg.kb;
  return true;
}

template <class C>
__global__ void __launch_bounds__(C::THREADS, 1)
    attn_fwd_sm100(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, uint16_t* __restrict__ out, int Lq, int Lk,
                   int dh, float scale_log2, unsigned int* err, int debug_flags, int qpairs, int items,
                   float* __restrict__ ws, unsigned int* flags, int lay_heads,
                   const __grid_constant__ Part part) {
  constexpr int BN = C::BN, NQ = C::NQ, STAGES = C::STAGES, NCH = C::NCH, NCHV = C::NCHV, DHP = C::DHP;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const Bars bars{sbase + C::BAR_OFF, STAGES, NQ};
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::MISC_OFF + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nkv = (Lk + BN - 1) / BN;
  const long long u0 = part.u[blockIdx.x], u1 = part.u[blockIdx.x + 1];

  if (threadIdx.x == 0) {
    mbar_init(bars.q_full(0), 1);
    mbar_init(bars.q_full(1), 1);
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(bars.k_full(s), 1);
      mbar_init(bars.v_full(s), 1);
      mbar_init(bars.v_ready(s), 1);
      mbar_init(bars.kv_empty(s), NQ);  // one tcgen05.commit per query tile's MMA issuer
    }
    for (int t = 0; t < NQ; ++t) {
      mbar_init(bars.s_full(t), 1);
      mbar_init(bars.s_free(t), 128);
      mbar_init(bars.p_full(t), 128);
      mbar_init(bars.o_done(t), 1);
    }
    for (int t = 0; t < NQ; ++t) mbar_init(bars.fin() + 8 * t, 1);
    for (int i = 0; i < 8; ++i) mbar_init(bars.tok(i >> 2, i & 3), 1);
    mbar_init(bars.q_empty(0), NQ);
    mbar_init(bars.q_empty(1), NQ);
    for (int kind = 0; kind < 2; ++kind) {
      mbar_init(bars.split_dec(kind), 1);
      mbar_init(bars.split_written(kind), NQ * BM);
    }
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
  // Everything above touched only shared memory, tensor memory and the kernel parameters: it may
  // overlap the end of the previous kernel on the stream. Global memory waits for that kernel.
  sd::grid_dep_wait();
  sd::grid_dep_launch();

  if (warp < C::SOFT_WARP0) {
  // ==================================================================== helper warpgroup
  if constexpr (SD_REGSPLIT && NQ == 2) regs_dec<C::REG_HELPER>();  // registers move to the softmax warpgroups
  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int issued[STAGES];
#pragma unroll
      for (int s = 0; s < STAGES; ++s) issued[s] = 0;
      long long u = u0;
      Seg sg;
      int nseg = 0, g = 0;  // segments started, K/V tiles issued (the ring position)
      bool ok = true;
      while (ok && next_seg(u, u1, nkv, sg)) {
        const int bh = sg.it / qpairs, q0 = (sg.it % qpairs) * (BM * NQ);
        // Q buffer qb is reused by the segment after next, once both tiles have issued their last
        // S = Q K^T of the segment that used it.
        const int qb = nseg % C::QBUF;
        if (nseg >= C::QBUF && !wait_bar(bars.q_empty(qb), (nseg / C::QBUF - 1) & 1, abort_flag, err)) break;
        mbar_arrive_expect_tx(bars.q_full(qb), NQ * C::Q_TILE_BYTES);
        for (int t = 0; t < NQ; ++t)
          for (int c = 0; c < NCH; ++c)
            load_rows<C::BLHD>(sbase + C::Q_OFF + (qb * NQ + t) * C::Q_TILE_BYTES + c * BM * 128, &tm_q, bars.q_full(qb),
                      c * 64, q0 + t * BM, bh, lay_heads);
        ++nseg;
        for (int j = sg.kb; j < sg.ke; ++j, ++g) {
          const int s = g % STAGES, round = g / STAGES;
          if (g >= STAGES && !wait_bar(bars.kv_empty(s), (round - 1) & 1, abort_flag, err)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(bars.k_full(s), C::K_TILE_BYTES);
          for (int c = 0; c < NCH; ++c)
            load_rows<C::BLHD>(sbase + C::K_OFF + s * C::K_TILE_BYTES + c * BN * 128, &tm_k, bars.k_full(s), c * 64,
                      j * BN, bh, lay_heads);
          issued[s] = round + 1;
          if ((debug_flags & 1) && g == 0) {  // test hook: the first V tile never arrives
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(bars.v_full(s), C::V_TILE_BYTES);
          for (int c = 0; c < NCHV; ++c)
            load_rows<C::BLHD>(sbase + C::V_OFF + s * C::V_TILE_BYTES + c * BN * 128, &tm_v, bars.v_full(s), c * 64,
                      j * BN, bh, lay_heads);
        }
      }
      // Drain: every copy this thread issued has landed before the CTA may exit.
      for (int k = nseg - 1; k >= 0 && k >= nseg - C::QBUF; --k)
        wait_bar(bars.q_full(k % C::QBUF), (k / C::QBUF) & 1, abort_flag, err, false);
      for (int s = 0; s < STAGES; ++s)
        if (issued[s] > 0) {
          wait_bar(bars.k_full(s), (issued[s] - 1) & 1, abort_flag, err, false);
          if (!((debug_flags & 1) && s == 0 && issued[s] == 1))
            wait_bar(bars.v_full(s), (issued[s] - 1) & 1, abort_flag, err, false);
        }
    }
    __syncwarp();  // lanes 1-31 wait for lane 0 here: the warp meets the CTA barrier below as a whole
  } else if (warp == 1 || (NQ == 2 && warp == 2)) {
    // ------------------------------------------------------------------ MMA issuer of one tile
    // One issuing warp per query tile: a tcgen05.mma occupies its issuing thread for tens to
    // hundreds of cycles, so two tiles' instruction streams must not queue behind each other.
    const int t = warp - 1;
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_f16kind_f32(BM, BN, false, C::F16);
      constexpr uint32_t idesc_pv = idesc_f16kind_f32(BM, C::NPV, true, C::F16);
      uint32_t tq = sbase + C::Q_OFF + t * C::Q_TILE_BYTES;  // the current segment's Q buffer
      auto issue_qk = [&](int s) {  // S = Q K_s^T over the padded head dim
        const uint32_t d = tmem + t * C::TM_TILE + C::TM_S;
#pragma unroll
        for (int ks = 0; ks < DHP / 16; ++ks) {
          const uint32_t off = (ks >> 2) * (BM * 128) + (ks & 3) * 32;
          const uint32_t offk = (ks >> 2) * (BN * 128) + (ks & 3) * 32;
          const uint64_t a = smem_desc(tq + off, 16, 1024);
          const uint64_t b = smem_desc(sbase + C::K_OFF + s * C::K_TILE_BYTES + offk, 16, 1024);
          mma_ss(d, a, b, idesc_qk, ks > 0 ? 1u : 0u);
        }
      };
      auto issue_pv = [&](int s, bool first) {  // O (+)= P V_s, P from TMEM (16 keys = 8 columns)
        const uint32_t d = tmem + t * C::TM_TILE + C::TM_O;
        const uint32_t a = tmem + t * C::TM_TILE + C::TM_P;
#pragma unroll
        for (int ks = 0; ks < BN / 16; ++ks) {
          const uint64_t b = smem_desc(sbase + C::V_OFF + s * C::V_TILE_BYTES + ks * 16 * 128, BN * 128, 1024);
          mma_ts(d, a + ks * 8, b, idesc_pv, (!first || ks > 0) ? 1u : 0u);
        }
      };
      // Two cursors over the CTA's K/V tiles, issued in whichever order they become ready:
      // S_g = Q K_g^T (needs K_g, the segment's Q, and the softmax's release of the previous S --
      // with P over S, the completion of the previous P V), and O += P_g V_g (needs P_g and V_g;
      // the first P V of a segment overwrites O, which the softmax has read out before it stores
      // that segment's first P). P V goes first when both are ready: it frees the K/V stage the
      // producer is waiting for. The S cursor runs ahead into the next segment, so its first S
      // overlaps the previous segment's last P V and epilogue. Barrier phases run on the
      // CTA-wide K/V tile counts gq, gp.
      long long uq = u0, up = u0;
      Seg sq, sp;
      bool have_q = next_seg(uq, u1, nkv, sq), have_p = next_seg(up, u1, nkv, sp);
      int nseg_q = 0, jq = 0, jp = 0, gq = 0, gp = 0;
      bool ok = true;
      long long t_idle = clock64();
      // The last tile's issuer also decides the split hand-off (below): it claims a split piece's
      // slot when it issues the piece's last S, so the atomic's round trip overlaps that tile's
      // softmax, and publishes the decision to the softmax warps when it issues the last P V.
      const bool decider = t == NQ - 1;
      unsigned int claim_head = 0u, claim_tail = 0u;
      uint32_t spins = 0;
      while (ok && have_p) {
        const bool can_pv = gp < gq && mbar_test_wait(bars.p_full(t), gp & 1) &&
                            mbar_test_wait(C::L_IN_V ? bars.v_ready(gp % STAGES) : bars.v_full(gp % STAGES),
                                           (gp / STAGES) & 1);
        if (can_pv) {
          tc_fence_after();
          issue_pv(gp % STAGES, jp == 0);
          mma_commit(bars.o_done(t));
          mma_commit(bars.kv_empty(gp % STAGES));
          ++gp;
          if (++jp == sp.ke - sp.kb) {
            if (decider && (sp.kb > 0 || sp.ke < nkv)) {
              const int kind = sp.ke < nkv ? 1 : 0;  // 1: head piece, 0: tail piece
              const unsigned int old = kind ? claim_head : claim_tail;
              int d = old == 0u ? kSplitPublish : kSplitMerge;
              if (old == 1u) {  // the other piece claimed the slot: wait until it has been completed
                volatile unsigned int* f = flags + (kind ? static_cast<int>(blockIdx.x) : static_cast<int>(blockIdx.x) - 1);
                const long long w0 = clock64();
                for (uint32_t it = 0; *f != 2u; ++it) {
                  __nanosleep(32);
                  if ((it & 63u) == 63u && (*abort_flag || clock64() - w0 > kWaitLimitCycles)) {
                    if (!*abort_flag) {
                      *abort_flag = 1;
                      atomicOr(err, sd::kDevErrTimeout);
                    }
                    d = kSplitAbort;
                    break;
                  }
                }
              }
              if (d == kSplitMerge) __threadfence();
              reinterpret_cast<volatile int*>(smem + C::MISC_OFF + 8)[kind] = d;
              mbar_arrive(bars.split_dec(kind));
            }
            have_p = next_seg(up, u1, nkv, sp);
            jp = 0;
          }
          t_idle = clock64();
          continue;
        }
        const int qb = nseg_q % C::QBUF;
        const bool can_qk = have_q && (jq > 0 || mbar_test_wait(bars.q_full(qb), (nseg_q / C::QBUF) & 1)) &&
                            mbar_test_wait(bars.k_full(gq % STAGES), (gq / STAGES) & 1) &&
                            (gq == 0 || mbar_test_wait(C::P_SEP ? bars.s_free(t) : bars.o_done(t), (gq - 1) & 1));
        if (can_qk) {
          tc_fence_after();
          tq = sbase + C::Q_OFF + (qb * NQ + t) * C::Q_TILE_BYTES;
          issue_qk(gq % STAGES);
          mma_commit(bars.s_full(t));
          ++gq;
          if (++jq == sq.ke - sq.kb) {
            if (decider && (sq.kb > 0 || sq.ke < nkv)) {  // claim: counter 0 -> 1 makes this piece the publisher
              if ((debug_flags & 2) && sq.ke == nkv) {  // test hook: hold tail pieces back ~50 us (head finishes first)
                const long long h0 = clock64();
                while (clock64() - h0 < 100000) __nanosleep(500);
              }
              const unsigned int old =
                  atomicCAS(flags + (sq.ke < nkv ? static_cast<int>(blockIdx.x) : static_cast<int>(blockIdx.x) - 1), 0u, 1u);
              if (sq.ke < nkv) claim_head = old;
              else claim_tail = old;
            }
            mma_commit(bars.q_empty(qb));  // this tile is done reading the segment's Q
            have_q = next_seg(uq, u1, nkv, sq);
            jq = 0;
            ++nseg_q;
          }
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
      // Drain: all tensor-core work issued by this thread completes before TMEM is released.
      const uint32_t fin = bars.fin() + 8 * t;
      mma_commit(fin);
      wait_bar(fin, 0, abort_flag, err, false);
    }
    __syncwarp();
  } else if (C::L_IN_V && warp == C::FIX_WARP) {

    // ------------------------------------------------------------------ V fix-up warp
    // Writes bf16 1.0 into column DH of every landed V tile (128-byte swizzled rows: the 16-byte
    // granule g of row r sits at granule g ^ (r % 8)), then hands the tile to the MMA issuer.
    constexpr int ch = C::DH / 64, byte = (C::DH % 64) * 2, g = byte >> 4, gb = byte & 15;
    const int total = static_cast<int>(u1 - u0);  // K/V tiles this CTA streams
    for (int j = 0; j < total; ++j) {
      const int s = j % STAGES;
      if (!__all_sync(0xffffffffu, wait_bar(bars.v_full(s), (j / STAGES) & 1, abort_flag, err))) break;
      uint8_t* vt = smem + C::V_OFF + s * C::V_TILE_BYTES + ch * BN * 128;
#pragma unroll
      for (int r = lane; r < BN; r += 32)
        *reinterpret_cast<uint16_t*>(vt + r * 128 + ((g ^ (r & 7)) << 4) + gb) = C::F16 ? 0x3C00u : 0x3F80u;  // 1.0
      fence_proxy_async_smem();  // generic-proxy stores -> visible to the tensor core
      __syncwarp();
      if (lane == 0) mbar_arrive(bars.v_ready(s));
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TM_COLS);
  }
  } else {
  // ==================================================================== softmax warpgroups
  if constexpr (SD_REGSPLIT && NQ == 2) regs_inc<C::REG_SOFT>();
  {
    // ------------------------------------------------------------------ softmax warps
    const int t = (warp - C::SOFT_WARP0) >> 2;  // query tile of this warpgroup
    const int quarter = warp & 3;   // TMEM lane quarter this warp may access
    const int row = quarter * 32 + lane;
    const uint32_t tbase = tmem + t * C::TM_TILE + (static_cast<uint32_t>(quarter * 32) << 16);
    const uint32_t tS = tbase + C::TM_S, tP = tbase + C::TM_P, tO = tbase + C::TM_O;
    bool ok = true;
    constexpr bool kPing = SD_PINGPONG && NQ == 2 && (SD_PING_SHORT || BN == 128);
    long long u = u0;
    Seg sg;
    int gi = 0;  // CTA-wide K/V tile count: the phase of every per-tile barrier
    int nseg_done = 0;
    while (ok && next_seg(u, u1, nkv, sg)) {
    const int bh = sg.it / qpairs, q0 = (sg.it % qpairs) * (BM * NQ);
    float m_run = -INFINITY, l_run = 0.f;
    for (int j = sg.kb; j < sg.ke; ++j, ++gi) {
      const bool first = j == sg.kb;  // O and l are (re)initialised by this segment's first P V
      // warp-uniform outcome: the tcgen05 copies below are .sync.aligned
      if (!__all_sync(0xffffffffu, wait_bar(bars.s_full(t), gi & 1, abort_flag, err))) {
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
      if constexpr (C::P_SEP) {  // S is in registers: the next S = Q K^T may overwrite it
        tc_fence_before();
        mbar_arrive(bars.s_free(t));
      }
      const int valid = Lk - j * BN;
      if (valid < BN) {
#pragma unroll
        for (int i = 0; i < BN; ++i)
          if (i >= valid) sv[i] = -INFINITY;
      }
      // Row max as 16 independent chains of 3-input max, then a short tree.
      float pm[16];
#pragma unroll
      for (int k = 0; k < 16; ++k) pm[k] = sv[k];
#pragma unroll
      for (int i = 16; i + 32 <= BN; i += 32)
#pragma unroll
        for (int k = 0; k < 16; ++k) pm[k] = max3f(pm[k], sv[i + k], sv[i + 16 + k]);
      if constexpr ((BN / 16) % 2 == 0) {
#pragma unroll
        for (int k = 0; k < 16; ++k) pm[k] = fmaxf(pm[k], sv[BN - 16 + k]);
      }
      const float mx = fmaxf(max3f(max3f(pm[0], pm[1], pm[2]), max3f(pm[3], pm[4], pm[5]), max3f(pm[6], pm[7], pm[8])),
                             max3f(max3f(pm[9], pm[10], pm[11]), max3f(pm[12], pm[13], pm[14]), pm[15]));
      const float m_new = fmaxf(m_run, mx * scale_log2);
      // Lazy rescale (always on the first tile). The decision is warp-uniform: the tcgen05 copies
      // of O and l below are .sync.aligned, and rescaling a row whose max barely moved is exact.
      const bool rescale = __any_sync(0xffffffffu, m_new > m_run + 8.0f);
      const float alpha = rescale ? ex2_approx(m_run - m_new) : 1.0f;
      if (rescale) m_run = m_new;
      // With CHUNK_P, P goes to tensor memory in 16-column chunks as the exp2 loop produces it,
      // which needs the previous P V complete (and O rescaled) first; waiting for it here does not
      // hold the ping-pong token.
      constexpr bool kChunkP = SD_P_CHUNKED >= 0 ? SD_P_CHUNKED != 0 : C::CHUNK_P;
      if (kChunkP) {
        if (C::P_SEP && gi > 0) {
          if (!__all_sync(0xffffffffu, wait_bar(bars.o_done(t), (gi - 1) & 1, abort_flag, err))) {
            ok = false;
            break;
          }
          tc_fence_after();
        }
        if (rescale && !first) {
#pragma unroll
          for (int c = 0; c < C::NPV / 16; ++c) {  // O columns, the row-sum column DH among them
            const uint32_t addr = tO + c * 16;
            uint32_t r[16];
            tmem_ld16(addr, r);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 16; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
            tmem_st16(addr, r);
          }
        }
      }
      // Ping-pong: the special-function unit of a sub-partition serves one tile's exp2 phase at a
      // time; the other tile's warp on it does its row max, P store and S load meanwhile. Tile 0
      // goes first; each warp hands the token to its partner (same sub-partition) after its exps.
      if (kPing && (t == 1 || gi > 0)) {
        if (!__all_sync(0xffffffffu, wait_bar(bars.tok(t, quarter), (t == 1 ? gi : gi - 1) & 1, abort_flag, err))) {
          ok = false;
          break;
        }
      }
      const float neg_m = -m_run;
      uint32_t pk[BN / 2];
      float ls0 = 0.f, ls1 = 0.f, ls2 = 0.f, ls3 = 0.f;
      // Exponentials in blocks of EB column pairs: all arguments, then all exp2 (special-function
      // unit, or the FMA-pipe polynomial for POLY_PAIRS of every 8 pairs), then all packing, so
      // that a warp keeps many independent exp2 in flight instead of waiting on each pair.
      constexpr int EB = SD_EXP_BLOCK;
      // The token goes to the partner warp after kRelease column pairs: its exp2 phase then
      // overlaps the rest of this one (two warps keep the special-function unit busier than one).
      constexpr int kRel = SD_PING_RELEASE >= 0 ? SD_PING_RELEASE : C::PING_RELEASE;
      constexpr int kRelease = kRel > BN / 2 ? BN / 2 : kRel / EB * EB;
#pragma unroll
      for (int b = 0; b < BN / 2; b += EB) {
        if (kPing && kRelease < BN / 2 && b == kRelease) {
          __syncwarp();
          if (lane == 0) mbar_arrive(bars.tok(1 - t, quarter));
        }
        float x[2 * EB];
#pragma unroll
        for (int i = 0; i < EB; ++i)  // s * scale * log2(e) - m, two columns per instruction
          fma2(x[2 * i], x[2 * i + 1], sv[2 * (b + i)], sv[2 * (b + i) + 1], scale_log2, scale_log2, neg_m, neg_m);
#pragma unroll
        for (int i = 0; i < EB; ++i) {
          if (((b + i) & 7) < C::POLY_PAIRS) {
            exp2_poly2(x[2 * i], x[2 * i + 1], x[2 * i], x[2 * i + 1]);
          } else {
            x[2 * i] = ex2_approx(x[2 * i]);
            x[2 * i + 1] = ex2_approx(x[2 * i + 1]);
          }
        }
#pragma unroll
        for (int i = 0; i < EB; ++i) {
          if constexpr (!C::L_IN_V) {  // fp32 row sums in two chains of pairs (half the dependent adds)
            if ((b + i) & 1) add2(ls2, ls3, ls2, ls3, x[2 * i], x[2 * i + 1]);
            else add2(ls0, ls1, ls0, ls1, x[2 * i], x[2 * i + 1]);
          }
          pk[b + i] = C::F16 ? pack_f16x2(x[2 * i], x[2 * i + 1]) : pack_bf16x2(x[2 * i], x[2 * i + 1]);
        }
        if (kChunkP && (b + EB) % 16 == 0) {  // 16 packed columns done: store them now
          const int c = (b + EB) / 16 - 1;
          uint32_t r[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) r[i] = pk[c * 16 + i];
          tmem_st16(tP + c * 16, r);
        }
      }
      if constexpr (!C::L_IN_V) l_run = fmaf(l_run, alpha, (ls0 + ls1) + (ls2 + ls3));
      if (kPing && kRelease == BN / 2) {
        __syncwarp();
        if (lane == 0) mbar_arrive(bars.tok(1 - t, quarter));
      }
      // The previous P V (and the O it accumulates) must be complete before P and O are touched.
      if (!kChunkP && C::P_SEP && gi > 0) {
        if (!__all_sync(0xffffffffu, wait_bar(bars.o_done(t), (gi - 1) & 1, abort_flag, err))) {
          ok = false;
          break;
        }
        tc_fence_after();
      }
      if (!kChunkP && rescale && !first) {
#pragma unroll
        for (int c = 0; c < C::NPV / 16; ++c) {  // O columns, the row-sum column DH among them
          const uint32_t addr = tO + c * 16;
          uint32_t r[16];
          tmem_ld16(addr, r);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 16; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
          tmem_st16(addr, r);
        }
      }
#pragma unroll
      for (int c = 0; c < BN / 32; ++c) {
        if (kChunkP) break;
        uint32_t r[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) r[i] = pk[c * 16 + i];
        tmem_st16(tP + c * 16, r);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bars.p_full(t));
    }
    if (!ok || !__all_sync(0xffffffffu, wait_bar(bars.o_done(t), (gi - 1) & 1, abort_flag, err))) {
      ok = false;
      break;
    }
    // ------------------------------------------------ epilogue of the segment (one row per thread)
    tc_fence_after();
    float ov[C::NPV];
#pragma unroll
    for (int c = 0; c < C::NPV / 16; ++c) {
      uint32_t r[16];
      tmem_ld16(tO + c * 16, r);
      tmem_wait_ld();
#pragma unroll
      for (int i = 0; i < 16; ++i) ov[c * 16 + i] = __uint_as_float(r[i]);
    }
    float lsum = C::L_IN_V ? ov[C::DH] : l_run;
    const int slot_row = t * BM + row;
    if (sg.kb > 0 || sg.ke < nkv) {
      // Split item: a head piece (keys [0, k), at the end of CTA c's range) and a tail piece (keys
      // [k, nkv), at the start of CTA c+1's range) share one slot and one counter of boundary c.
      // The piece whose last S = Q K^T is issued first claims the slot (counter 0 -> 1, by the
      // last tile's MMA issuer, which publishes the decision here), writes its raw O, m and l
      // there and marks it complete (-> 2); the other piece merges the two and stores O, then
      // resets the counter for the next launch. No CTA ever waits for another CTA to start: the
      // only cross-CTA wait is the other piece's issuer waiting for a claimed slot to be
      // completed, by a CTA that is already running and whose write depends on nothing else.
      const int kind = sg.ke < nkv ? 1 : 0;  // 1: head piece, 0: tail piece
      const int bnd = kind ? static_cast<int>(blockIdx.x) : static_cast<int>(blockIdx.x) - 1;
      float* slot = ws + static_cast<size_t>(bnd) * C::SLOT_FLOATS;
      unsigned int* cnt = flags + bnd;
      volatile int* dec = reinterpret_cast<volatile int*>(smem + C::MISC_OFF + 8) + kind;
      const bool leader_warp = warp == C::SOFT_WARP0 + 4 * NQ - 1;  // completes a publication, resets after a merge
      __syncwarp();
      if (!__all_sync(0xffffffffu, wait_bar(bars.split_dec(kind), 0, abort_flag, err)) || *dec == kSplitAbort) {
        ok = false;
        break;
      }
      // Slot layout: for each warp of 32 rows, float4 i of all 32 rows is one contiguous 512-byte
      // run (coalesced writes and reads: a row-major slot made every access of a warp touch 32
      // lines), then (m, l) of every row.
      if (*dec == kSplitPublish) {
        float4* dst = reinterpret_cast<float4*>(slot) + (slot_row >> 5) * (C::NPV / 4) * 32 + lane;
#pragma unroll
        for (int i = 0; i < C::NPV / 4; ++i)
          dst[i * 32] = make_float4(ov[4 * i], ov[4 * i + 1], ov[4 * i + 2], ov[4 * i + 3]);
        reinterpret_cast<float2*>(slot + NQ * BM * C::NPV)[slot_row] = make_float2(m_run, lsum);
        // Every softmax thread arrives (release, CTA scope); the leader waits for all of them, then
        // makes the slot visible device-wide with one fence and marks it complete.
        mbar_arrive(bars.split_written(kind));
        if (leader_warp) {
          if (!__all_sync(0xffffffffu, wait_bar(bars.split_written(kind), 0, abort_flag, err))) {
            ok = false;
            break;
          }
          if (lane == 0) {
            __threadfence();
            atomicExch(cnt, 2u);
          }
          __syncwarp();
        }
        ++nseg_done;
        continue;
      }
      if (leader_warp && lane == 0) atomicExch(cnt, 0u);  // both pieces are done with the counter
      // Merge in one fixed order, O = O_head * 2^(m_head - m) + O_tail * 2^(m_tail - m), so the result
      // is the same bit for bit whichever piece merges. The slot is read through L2 only.
      const float4* src = reinterpret_cast<const float4*>(slot) + (slot_row >> 5) * (C::NPV / 4) * 32 + lane;
      const float2 ml = __ldcg(reinterpret_cast<const float2*>(slot + NQ * BM * C::NPV) + slot_row);
      const float m_head = kind ? m_run : ml.x, m_tail = kind ? ml.x : m_run;
      const float m_all = fmaxf(m_head, m_tail);
      const float a_h = ex2_approx(m_head - m_all), a_t = ex2_approx(m_tail - m_all);
      auto comb = [&](float mine, float theirs) {
        return kind ? fmaf(mine, a_h, theirs * a_t) : fmaf(theirs, a_h, mine * a_t);
      };
#pragma unroll
      for (int i = 0; i < C::NPV / 4; ++i) {
        const float4 o4 = __ldcg(src + i * 32);
        ov[4 * i] = comb(ov[4 * i], o4.x);
        ov[4 * i + 1] = comb(ov[4 * i + 1], o4.y);
        ov[4 * i + 2] = comb(ov[4 * i + 2], o4.z);
        ov[4 * i + 3] = comb(ov[4 * i + 3], o4.w);
      }
      lsum = C::L_IN_V ? ov[C::DH] : comb(lsum, ml.y);
    }
    const int qrow = q0 + t * BM + row;
    const float inv_l = 1.0f / lsum;
    uint32_t packed[DHP / 2];
#pragma unroll
    for (int i = 0; i < DHP / 2; ++i)
      packed[i] = C::F16 ? pack_f16x2(ov[2 * i] * inv_l, ov[2 * i + 1] * inv_l)
                         : pack_bf16x2(ov[2 * i] * inv_l, ov[2 * i + 1] * inv_l);
    if (qrow < Lq) {
      const size_t orow = C::BLHD ? (static_cast<size_t>(bh / lay_heads) * Lq + qrow) * lay_heads + bh % lay_heads
                                  : static_cast<size_t>(bh) * Lq + qrow;
      uint4* dst = reinterpret_cast<uint4*>(out + orow * dh);
      const int n16 = dh / 8;  // 16-byte groups of 8 bf16
#pragma unroll
      for (int i = 0; i < DHP / 8; ++i)
        if (i < n16) dst[i] = make_uint4(packed[4 * i], packed[4 * i + 1], packed[4 * i + 2], packed[4 * i + 3]);
    }
    ++nseg_done;
    }
  }
  tc_fence_before();
  __syncthreads();
  }
}

// ---------------------------------------------------------------------------- host side

// Per-device hand-off workspace of the persistent schedule (slots of split items + their counters).
// Allocated on first need and grown, never shrunk; counters start at zero and every launch leaves
// them at zero. Launches of sd_attention that run concurrently on one device (different streams)
// must not both split items: they would share the slots.
struct Workspace {
  void* ptr = nullptr;
  size_t bytes = 0;
};
Workspace g_ws[64];
std::mutex g_ws_mu;

sd_status workspace(size_t bytes, cudaStream_t s, void** out) {
  int dev = 0;
  sd_status st = sd::cuda_check(cudaGetDevice(&dev), "cudaGetDevice");
  if (st != SD_OK) return st;
  if (dev >= 64) return sd::fail(SD_ERR_UNSUPPORTED, "sd_attention: device index >= 64");
  std::lock_guard<std::mutex> lock(g_ws_mu);
  Workspace& w = g_ws[dev];
  if (w.bytes < bytes) {
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    cudaStreamIsCapturing(s, &cap);
    if (cap != cudaStreamCaptureStatusNone)
      return sd::fail(SD_ERR_CUDA, "sd_attention: the split-item workspace (%zu bytes) must be allocated before "
                                   "stream capture; run the same shape once outside the capture", bytes);
    if (w.ptr) {
      st = sd::cuda_check(cudaDeviceSynchronize(), "cudaDeviceSynchronize(workspace growth)");
      if (st == SD_OK) st = sd::cuda_check(cudaFree(w.ptr), "cudaFree(workspace)");
      w.ptr = nullptr;
      w.bytes = 0;
      if (st != SD_OK) return st;
    }
    st = sd::cuda_check(cudaMalloc(&w.ptr, bytes), "cudaMalloc(workspace)");
    if (st != SD_OK) return st;
    st = sd::cuda_check(cudaMemset(w.ptr, 0, bytes), "cudaMemset(workspace)");
    if (st != SD_OK) return st;
    w.bytes = bytes;
  }
  *out = w.ptr;
  return SD_OK;
}

}  // namespace

sd_status sd::attention_clear_handoff(cudaStream_t s) {
  int dev = 0;
  sd_status st = sd::cuda_check(cudaGetDevice(&dev), "cudaGetDevice");
  if (st != SD_OK || dev >= 64) return st;
  std::lock_guard<std::mutex> lock(g_ws_mu);
  const Workspace& w = g_ws[dev];
  if (!w.ptr) return SD_OK;
  return sd::cuda_check(cudaMemsetAsync(w.ptr, 0, w.bytes, s), "cudaMemsetAsync(attention workspace)");
}

namespace {

// Fixed scratch of sd_attention_noalloc: a file-scope device array, so that entry point never
// allocates. Every device that loads the library holds it until the process exits. Zero at module
// load; each call clears the hand-off counters it uses before its launch.
constexpr size_t kFixedScratchBytes = size_t(16) << 20;
__device__ __align__(256) unsigned char g_fixed_scratch[kFixedScratchBytes];
struct FixedAddr {
  void* ctx = nullptr;  // the context the address belongs to
  void* addr = nullptr;
};
FixedAddr g_fixed_addr[64];
std::mutex g_fixed_mu;

// Device address of g_fixed_scratch on the current device. The name of the array in host code is a
// host-side stand-in, not a device address, so it is resolved with that device current and cached
// per device, together with the context it was resolved in: if the device's primary context was
// destroyed and created again (cudaDeviceReset), the address is looked up again.
sd_status fixed_scratch(void** out) {
  int dev = 0;
  sd_status st = sd::cuda_check(cudaGetDevice(&dev), "cudaGetDevice");
  if (st != SD_OK) return st;
  if (dev >= 64) return sd::fail(SD_ERR_UNSUPPORTED, "sd_attention_noalloc: device index >= 64");
  void* ctx = nullptr;
  st = sd::current_context(&ctx);
  if (st != SD_OK) return st;
  std::lock_guard<std::mutex> lock(g_fixed_mu);
  FixedAddr& f = g_fixed_addr[dev];
  if (!f.addr || f.ctx != ctx) {
    void* p = nullptr;
    st = sd::cuda_check(cudaGetSymbolAddress(&p, g_fixed_scratch), "cudaGetSymbolAddress(fixed scratch)");
    if (st != SD_OK) return st;
    f.addr = p;
    f.ctx = ctx;
  }
  *out = f.addr;
  return SD_OK;
}

#ifndef SD_BALANCE
#define SD_BALANCE 1  // unit ranges balanced by the cost model below (0: equal unit counts)
#endif

// Per-CTA unit ranges. Equal unit counts leave CTAs with more segment boundaries, or ending in a
// split item's merge, finishing last. Measured on B200 with global-timer spans (SD1.5 and SDXL
// shapes), in K/V-tile units: each segment boundary costs about 1.0 tile, publishing a tail piece
// 0.6, merging a head piece 0.9 (dh 40; 1.3, 0.5 and 1.4 for dh 64). The range of each CTA is
// chosen so that tiles plus these costs stay below the smallest bound T that covers all units;
// a range never lies strictly inside one item, so an item still spans at most two consecutive
// CTAs. Results are cached per shape.
struct CostModel {
  double seg, tail, head;
};

double range_cost(long long a, long long b, long long nkv, const CostModel& m) {
  const long long segs = (b - 1) / nkv - a / nkv + 1;
  return static_cast<double>(b - a) + m.seg * static_cast<double>(segs - 1) + (a % nkv ? m.tail : 0.0) +
         (b % nkv ? m.head : 0.0);
}

bool inside_one_item(long long a, long long b, long long nkv) {
  return a % nkv != 0 && b % nkv != 0 && a / nkv == (b - 1) / nkv;
}

bool fill_ranges(long long U, long long nkv, int G, const CostModel& m, double T, long long* u) {
  long long a = 0;
  u[0] = 0;
  for (int c = 0; c < G; ++c) {
    if (a >= U) {
      u[c + 1] = U;
      continue;
    }
    long long best = -1;
    const long long hi = std::min<long long>(U, a + static_cast<long long>(T) + 1);
    for (long long b = hi; b > a && b + 64 > hi; --b)
      if (!inside_one_item(a, b, nkv) && range_cost(a, b, nkv, m) <= T) {
        best = b;
        break;
      }
    if (best < 0) return false;
    u[c + 1] = best;
    a = best;
  }
  return a == U;
}

void part_ranges(long long U, long long nkv, int G, const CostModel& m, long long* u) {
  auto even = [&] {
    for (int c = 0; c <= G; ++c) u[c] = U * c / G;
  };
  if (!SD_BALANCE || nkv <= 1) return even();
  static std::mutex mu;
  static std::map<std::tuple<long long, long long, int, double, double, double>, std::vector<long long>> cache;
  const auto key = std::make_tuple(U, nkv, G, m.seg, m.tail, m.head);
  std::lock_guard<std::mutex> lock(mu);
  auto it = cache.find(key);
  if (it == cache.end()) {
    std::vector<long long> v(G + 1);
    double lo = static_cast<double>(U) / G, hi = lo + 4.0 * (m.seg + m.tail + m.head) + 2.0;
    if (!fill_ranges(U, nkv, G, m, hi, v.data())) {
      for (int c = 0; c <= G; ++c) v[c] = U * c / G;  // no balanced split found: equal counts
    } else {
      for (int i = 0; i < 40; ++i) {  // smallest T (to 1e-3 tiles) that still covers all units
        const double mid = 0.5 * (lo + hi);
        if (fill_ranges(U, nkv, G, m, mid, v.data())) hi = mid;
        else lo = mid;
      }
      fill_ranges(U, nkv, G, m, hi, v.data());
    }
    it = cache.emplace(key, std::move(v)).first;
  }
  std::copy(it->second.begin(), it->second.end(), u);
}

// `fixed` selects the caller-side contract of sd_attention_noalloc: scratch from g_fixed_scratch
// instead of the growable workspace, with its flags cleared on the stream first.
template <class C>
sd_status launch(const void* q, const void* k, const void* v, void* o, int64_t BH, int64_t Lq, int64_t Lk,
                 int64_t dh, float scale, cudaStream_t s, bool fixed, int64_t lay_heads) {
  CUtensorMap mq, mk, mv;
  sd_status st = sd::attn::make_map(&mq, q, dh, Lq, BH, BM, C::F16, lay_heads);
  if (st == SD_OK) st = sd::attn::make_map(&mk, k, dh, Lk, BH, C::BN, C::F16, lay_heads);
  if (st == SD_OK) st = sd::attn::make_map(&mv, v, dh, Lk, BH, C::BN, C::F16, lay_heads);
  if (st != SD_OK) return st;
  unsigned int* err = sd::device_status_word();
  if (!err) return SD_ERR_CUDA;
  auto kern = attn_fwd_sm100<C>;
  static std::atomic<uint64_t> smem_set{0};  // one bit per device: opt-in to large shared memory done
  int dev = 0;
  st = sd::cuda_check(cudaGetDevice(&dev), "cudaGetDevice");
  if (st != SD_OK) return st;
  const uint64_t bit = uint64_t(1) << (dev & 63);
  if (!(smem_set.load(std::memory_order_acquire) & bit)) {
    st = sd::cuda_check(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES),
                        "cudaFuncSetAttribute(attention smem)");
    if (st != SD_OK) return st;
    smem_set.fetch_or(bit, std::memory_order_acq_rel);
  }
  // Persistent grid: one CTA per SM (shared memory admits one), each owning an equal share of the
  // items x K/V-tiles units; items split between two CTAs hand over through the workspace. The
  // hand-off never waits for a CTA to start, so the grid needs no co-residency: CTAs that cannot be
  // resident at once (SMs held by other work) only run later.
  const int64_t qpairs = (Lq + BM * C::NQ - 1) / (BM * C::NQ);
  const int64_t items = BH * qpairs;
  const int64_t nkv = (Lk + C::BN - 1) / C::BN;
  const int64_t G = std::min<int64_t>(std::min<int64_t>(sd::sm_count(), items), kMaxCtas);
  if (items > 0x7fffffff || items * nkv > (int64_t(1) << 40))
    return sd::fail(SD_ERR_UNSUPPORTED, "sd_attention: too many tiles");
  float* ws = nullptr;
  unsigned int* flags = nullptr;
  if (G < items && nkv > 1) {
    // Layout: the boundary counters first, at the same place for every configuration (a launch of
    // one head dim must never find another configuration's slot data where it expects counters
    // that the previous launches left at zero), then the slots.
    const size_t need = kCounterBytes + static_cast<size_t>(G) * C::SLOT_FLOATS * sizeof(float);
    void* p = nullptr;
    if (fixed) {
      if (need > kFixedScratchBytes)
        return sd::fail(SD_ERR_UNSUPPORTED, "sd_attention_noalloc: this shape needs %zu bytes of scratch; the fixed "
                                            "buffer holds %zu", need, kFixedScratchBytes);
      st = fixed_scratch(&p);
      if (st != SD_OK) return st;
      st = sd::cuda_check(cudaMemsetAsync(p, 0, kCounterBytes, s), "cudaMemsetAsync(fixed scratch counters)");
    } else {
      st = workspace(need, s, &p);
    }
    if (st != SD_OK) return st;
    flags = static_cast<unsigned int*>(p);
    ws = reinterpret_cast<float*>(static_cast<char*>(p) + kCounterBytes);
  }
  Part part;
  part_ranges(items * nkv, nkv, static_cast<int>(G), CostModel{C::COST_SEG, C::COST_TAIL, C::COST_HEAD}, part.u);
  for (int64_t c = 0; c < G; ++c)  // the hand-off takes at most two pieces per item
    if (inside_one_item(part.u[c], part.u[c + 1], nkv))
      return sd::fail(SD_ERR_UNSUPPORTED, "sd_attention: internal error: a CTA range inside one item");
  const float scale_log2 = scale * 1.4426950408889634f;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(G));
  cfg.blockDim = dim3(C::THREADS);
  cfg.dynamicSmemBytes = C::SMEM_BYTES;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  cfg.attrs = attr;
  cfg.numAttrs = sd::pdl_attr(&attr[0]);
  return sd::cuda_check(
      cudaLaunchKernelEx(&cfg, kern, mq, mk, mv, static_cast<uint16_t*>(o), static_cast<int>(Lq),
                         static_cast<int>(Lk), static_cast<int>(dh), scale_log2, err, sd::attn::g_debug_flags,
                         static_cast<int>(qpairs), static_cast<int>(items), ws, flags, static_cast<int>(lay_heads),
                         part),
      "sd_attention launch");
}

}  // namespace

namespace {

// The launch table: a configuration per head dim and key length, for one element type.
template <bool F16, bool BLHD>
sd_status dispatch(const void* q, const void* k, const void* v, void* o, int64_t BH, int64_t Lq, int64_t Lk,
                   int64_t dh, float scale, cudaStream_t s, bool fixed, int64_t lay_heads) {
  // Short key sequences (the 77-token text context): all of K and V resident, one exact softmax pass.
  if (Lk <= sd::attn::kShortMaxKeys) return sd::attn::launch_short(q, k, v, o, BH, Lq, Lk, dh, scale, s, F16, lay_heads);
  if (Lk <= 96) {  // one 96-key tile, no online rescale
    switch (dh) {
      case 40: return launch<Cfg<40, 96, SD_CROSS_NQ, 2, true, true, 0, F16, BLHD>>(q, k, v, o, BH, Lq, Lk, dh, scale, s, fixed, lay_heads);
      case 64: return launch<Cfg<64, 96, SD_CROSS_NQ, 2, true, false, 0, F16, BLHD>>(q, k, v, o, BH, Lq, Lk, dh, scale, s, fixed, lay_heads);
      case 80: return launch<Cfg<80, 96, SD_CROSS_NQ, 2, true, true, 0, F16, BLHD>>(q, k, v, o, BH, Lq, Lk, dh, scale, s, fixed, lay_heads);
      default: break;  // dh = 160 already uses 64-key tiles
    }
  }
  // Few query tiles (every tile can have an SM of its own): one query tile per CTA, so that twice as
  // many SMs share the work. With one tile the dh 80 tile's S, P and O fit 512 tensor-memory columns
  // side by side, so the next S no longer waits for P V (measured 20.7 -> 16.8 us at [2,8,1024,1024,80]
  // with 2 of 8 exp2 pairs on the FMA pipe).
  if (SD_SMALL_NQ1 && BH * ((Lq + BM - 1) / BM) <= SD_SMALL_NQ1 * sd::sm_count()) {
    switch (dh) {
      case 40: return launch<Cfg<40, 128, 1, 4, true, true, 2, F16, BLHD>>(q, k, v, o, BH, Lq, Lk, dh, scale, s, fixed, lay_heads);
      case 64: return launch<Cfg<64, 128, 1, 4, true, false, 2, F16, BLHD>>(q, k, v, o, BH, Lq, Lk, dh, scale, s, fixed, lay_heads);
      case 80: return launch<Cfg<80, 128, 1, 2, true, true, 2, F16, BLHD>>(q, k, v, o, BH, Lq, Lk, dh, scale, s, fixed, lay_heads);
      default: break;
    }
  }
  switch (dh) {
    case 40: return launch<Cfg<40, 128, 2, SD_STAGES_SMALL, true, true, 2, F16, BLHD>>(q, k, v, o, BH, Lq, Lk, dh, scale, s, fixed, lay_heads);
    case 64: return launch<Cfg<64, 128, 2, SD_STAGES_SMALL, true, false, 2, F16, BLHD>>(q, k, v, o, BH, Lq, Lk, dh, scale, s, fixed, lay_heads);
    case 80: return launch<Cfg<80, 128, 2, 2, false, true, 0, F16, BLHD>>(q, k, v, o, BH, Lq, Lk, dh, scale, s, fixed, lay_heads);
    default: return launch<Cfg<160, 64, 1, 3, true, true, 0, F16, BLHD>>(q, k, v, o, BH, Lq, Lk, dh, scale, s, fixed, lay_heads);
  }
}

sd_status attention_impl(const void* q, const void* k, const void* v, void* o, int64_t B, int64_t heads, int64_t Lq,
                         int64_t Lk, int64_t dh, float scale, void* stream, bool fixed, bool f16 = false,
                         bool blhd = false) {
  if (B < 0 || heads < 0 || Lq < 0 || Lk < 0) return sd::fail(SD_ERR_INVALID_ARG, "sd_attention: negative size");
  if (dh != 40 && dh != 64 && dh != 80 && dh != 160)
    return sd::fail(SD_ERR_UNSUPPORTED, "sd_attention: head dim %lld not in {40, 64, 80, 160}", (long long)dh);
  if (!std::isfinite(scale)) return sd::fail(SD_ERR_INVALID_ARG, "sd_attention: scale is not finite");
  // The kernels take each row's maximum score times the scale as the softmax shift, which is the
  // maximum of the scaled scores only for scale >= 0.
  if (scale < 0.f) return sd::fail(SD_ERR_UNSUPPORTED, "sd_attention: negative scale");
  if (B == 0 || heads == 0 || Lq == 0) return SD_OK;
  if (Lk == 0) return sd::fail(SD_ERR_INVALID_ARG, "sd_attention: Lk must be >= 1 when Lq >= 1");
  if (!q || !k || !v || !o) return sd::fail(SD_ERR_INVALID_ARG, "sd_attention: null pointer");
  const int64_t BH = B * heads;
  if (BH > (int64_t(1) << 31) - 1 || Lq > (int64_t(1) << 30) || Lk > (int64_t(1) << 30))
    return sd::fail(SD_ERR_UNSUPPORTED, "sd_attention: B*heads must be < 2^31 and L <= 2^30");
  if (!sd::aligned16(q) || !sd::aligned16(k) || !sd::aligned16(v) || !sd::aligned16(o))
    return sd::fail(SD_ERR_MISALIGNED, "sd_attention: q, k, v and o must be 16-byte aligned");
  const int64_t qbytes = BH * Lq * dh * 2, kvbytes = BH * Lk * dh * 2;
  if (sd::overlaps(o, qbytes, q, qbytes) || sd::overlaps(o, qbytes, k, kvbytes) || sd::overlaps(o, qbytes, v, kvbytes))
    return sd::fail(SD_ERR_INVALID_ARG, "sd_attention: o overlaps q, k or v");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int64_t lay_heads = blhd ? heads : 0;
  if (blhd)
    return f16 ? dispatch<true, true>(q, k, v, o, BH, Lq, Lk, dh, scale, s, fixed, lay_heads)
               : dispatch<false, true>(q, k, v, o, BH, Lq, Lk, dh, scale, s, fixed, lay_heads);
  return f16 ? dispatch<true, false>(q, k, v, o, BH, Lq, Lk, dh, scale, s, fixed, lay_heads)
             : dispatch<false, false>(q, k, v, o, BH, Lq, Lk, dh, scale, s, fixed, lay_heads);
}

}  // namespace

extern "C" sd_status sd_attention(const void* q, const void* k, const void* v, void* o, int64_t B, int64_t heads,
                                  int64_t Lq, int64_t Lk, int64_t dh, float scale, void* stream) {
  return attention_impl(q, k, v, o, B, heads, Lq, Lk, dh, scale, stream, false);
}

// The same attention on fp16 tensors (see sd_kernels.h).
extern "C" sd_status sd_attention_f16(const void* q, const void* k, const void* v, void* o, int64_t B, int64_t heads,
                                      int64_t Lq, int64_t Lk, int64_t dh, float scale, void* stream) {
  return attention_impl(q, k, v, o, B, heads, Lq, Lk, dh, scale, stream, false, true);
}

// General entry: element type and memory layout as arguments (see sd_kernels.h).
extern "C" sd_status sd_attention_layout(const void* q, const void* k, const void* v, void* o, int64_t B,
                                         int64_t heads, int64_t Lq, int64_t Lk, int64_t dh, float scale, int dtype,
                                         int layout, void* stream) {
  if (dtype != 0 && dtype != 1) return sd::fail(SD_ERR_INVALID_ARG, "sd_attention_layout: dtype must be 0 or 1");
  if (layout != 0 && layout != 1) return sd::fail(SD_ERR_INVALID_ARG, "sd_attention_layout: layout must be 0 or 1");
  return attention_impl(q, k, v, o, B, heads, Lq, Lk, dh, scale, stream, false, dtype == 1, layout == 1);
}

// Same computation for callers that cannot allocate device memory (see sd_kernels.h): scratch comes
// from the fixed file-scope array, whose device address every call resolves first (cached per
// device and context).
extern "C" sd_status sd_attention_noalloc(const void* q, const void* k, const void* v, void* o, int64_t B,
                                          int64_t heads, int64_t Lq, int64_t Lk, int64_t dh, float scale,
                                          void* stream) {
  void* p = nullptr;  // resolve the array's address on every call (cached), whatever the shape
  const sd_status st = fixed_scratch(&p);
  if (st != SD_OK) return st;
  return attention_impl(q, k, v, o, B, heads, Lq, Lk, dh, scale, stream, true);
}

// Test hook (declared in sd_kernels.h): the unit ranges the persistent grid would use for `items`
// items of `nkv` K/V tiles on `grid` CTAs with the cost model of head dim `dh`; pure host code.
extern "C" sd_status sd_debug_attention_ranges(int64_t items, int64_t nkv, int64_t grid, int64_t dh, int64_t* out) {
  if (items < 1 || nkv < 1 || grid < 1 || grid > kMaxCtas || grid > items || !out)
    return sd::fail(SD_ERR_INVALID_ARG, "sd_debug_attention_ranges: bad arguments");
  const CostModel m = dh == 64 ? CostModel{1.3, 0.5, 1.4} : CostModel{1.0, 0.6, 0.9};
  long long u[kMaxCtas + 1];
  part_ranges(items * nkv, nkv, static_cast<int>(grid), m, u);
  for (int64_t c = 0; c <= grid; ++c) out[c] = u[c];
  return SD_OK;
}

// Test hook (declared in sd_kernels.h): bit 0 makes the next attention launches skip their first
// V tile so that the kernel's bounded wait expires and reports SD_ERR_TIMEOUT; bit 1 holds the tail
// pieces of split items back, so that head pieces finish first and the tail pieces merge.
extern "C" void sd_debug_set_fault(int flags) { sd::attn::g_debug_flags = flags; }
