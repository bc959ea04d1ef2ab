// Pieces shared by the two attention kernels (the general flash kernel in attention_sm100.cu and
// the short-key-sequence kernel in attention_short_sm100.cu): the tile height, the bounded mbarrier
// wait, the TMA row loads of both memory layouts, and the host-side tensor-map encoder.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "sd_internal.h"
#include "sm100_ptx.cuh"

namespace sd {
namespace attn {

constexpr int BM = 128;                               // query rows per tile = TMEM lanes
constexpr long long kWaitLimitCycles = 2000000000LL;  // ~1 s at B200 clocks

#ifdef __CUDACC__
// Bounded wait. Returns false if this CTA has aborted or the limit expired (then it raises the
// CTA's abort flag and the device status word). `abortable = false` is for teardown drains.
__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, volatile int* abort_flag, unsigned int* err,
                                         bool abortable = true) {
  if (sm100::mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  for (uint32_t it = 1;; ++it) {
    if (sm100::mbar_try_wait(bar, parity)) return true;
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

// One tile of rows [row, row + box) of head plane bh, 64 head-dim columns from x. lay_heads = 0:
// tensors [B*heads, L, dh] (3-D map); lay_heads = heads: tensors [B, L, heads, dh] (4-D map over
// {dh, heads, L, B}). Both put the same rows x 128 bytes into shared memory.
template <bool BLHD>
__device__ __forceinline__ void load_rows(uint32_t dst, const CUtensorMap* map, uint32_t bar, int x, int row, int bh,
                                          int lay_heads) {
  if constexpr (BLHD) sm100::tma_load_4d(dst, map, bar, x, bh % lay_heads, row, bh / lay_heads);
  else sm100::tma_load_3d(dst, map, bar, x, row, bh);
}
#endif

// Tensor map over a contiguous 16-bit [planes, rows, dh] tensor with box {64, box_rows, 1} and
// 128-byte swizzle (lay_heads = 0), or over [planes / heads, rows, heads, dh] as the 4-D map
// {dh, heads, rows, B} with box {64, 1, box_rows, 1} (lay_heads = heads). Columns past dh and rows
// past `rows` read as zero.
sd_status make_map(CUtensorMap* map, const void* ptr, int64_t dh, int64_t rows, int64_t planes, int box_rows,
                   bool f16, int64_t lay_heads);

// Test-hook flags of sd_debug_set_fault (bit 0: skip the first V tile; bit 1: hold tail pieces).
extern int g_debug_flags;

// The short-key-sequence kernel (Lk <= kShortMaxKeys): all of K and V resident, one exact softmax
// pass per query tile. Arguments as in the general launch; `lay_heads` = heads for [B, L, heads, dh].
constexpr int kShortMaxKeys = 80;
sd_status launch_short(const void* q, const void* k, const void* v, void* o, int64_t BH, int64_t Lq, int64_t Lk,
                       int64_t dh, float scale, cudaStream_t s, bool f16, int64_t lay_heads);

}  // namespace attn
}  // namespace sd
