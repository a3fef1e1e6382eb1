// Pieces shared by the two tensor-core attention kernels (bf16 and e4m3
// operands): the work unit, the order of the two key-block streams, bounded
// waits and the warpgroup register split.
#pragma once

#include "fkv_internal.cuh"
#include "sm100_common.cuh"

namespace fkv {
namespace sm100 {

// One 128-query tile of one (layer, head).  Its keys are the nA valid rows
// of the compressed cache (range A, nbA blocks of 128) followed by the Lq rows
// of the chunk; blocks [0, nb0) form stream 0 and [nb0, nb) stream 1.
struct Unit {
  int lh, qt, nbA, nb, nb0, nb1;
  int64_t nA;
};

template <class Args>
__device__ __forceinline__ Unit decode(const Args& a, int tile) {
  Unit t;
  t.lh = tile / a.n_qtiles;
  t.qt = tile - t.lh * a.n_qtiles;
  int64_t cnt = a.kept_cnt[t.lh];
  cnt = cnt < 0 ? 0 : (cnt > a.max_kept ? a.max_kept : cnt);
  int64_t nA = cnt * a.seg_len;
  if (nA > a.comp_rows) nA = a.comp_rows;
  t.nA = nA;
  t.nbA = int((nA + 127) / 128);
  t.nb = t.nbA + int((a.Lq + 127) / 128);
  t.nb0 = (t.nb + 1) / 2;
  t.nb1 = t.nb - t.nb0;
  return t;
}

// Position of (stream h, its j-th block) in the unit's load / MMA order:
// s0 b0, s1 b0, s0 b1, s1 b1, ..., then the rest of stream 0.
__device__ __forceinline__ int seq_pos(const Unit& t, int h, int j) {
  return j < t.nb1 ? 2 * j + h : t.nb1 + j;
}
// Key block index of (stream h, j).
__device__ __forceinline__ int block_of(const Unit& t, int h, int j) { return h ? t.nb0 + j : j; }

__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort,
                                          long long limit = kWaitCycles) {
  const bool ok = mbar_wait(bar, parity, abort, limit);
  return __all_sync(0xffffffffu, ok);
}

// Bounded wait that ignores the abort flag: used to let this CTA's own
// copies and MMAs finish before its shared memory and TMEM are released.
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity))
    if (clock64() - t0 > kWaitCycles) return;
}

template <uint32_t kRegs>
__device__ __forceinline__ void regs_increase() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegs));
}
template <uint32_t kRegs>
__device__ __forceinline__ void regs_decrease() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegs));
}

}  // namespace sm100
}  // namespace fkv
