// common.cuh -- device helpers shared by the hybrid_v2 kernels (sm_100a).
#pragma once

#include <cstdint>
#include <cuda_fp16.h>

#include "hyb_kv.h"

namespace hyb {

// hot-zone tokens per sequence: a run-time power of two in {16, 32, 64, 128}
// (hot_tokens of the descriptor); kMaxHot bounds it
constexpr int kMaxHot = 128;
constexpr int kBlock = 64;        // tokens per cold block
constexpr int kDim = 128;         // head dimension
constexpr int kTileBytes = kBlock * kDim;        // one K or V tile, INT8
constexpr int kTilePairBytes = 2 * kTileBytes;   // K tile + V tile of one (block, kv head)
constexpr int kHotTokenBytes = 2 * kDim * 2;     // K row + V row, FP16
// FP16 rows (hot ring, FP16 cold blocks) are staged 32 rows (16 KB) at a time
constexpr int kItemRows = 32;
constexpr int kItemBytes = kItemRows * kHotTokenBytes;
// quantization_bits 0: an FP16 cold block keeps the hot ring's row layout
// (K row then V row per token), 32 KB per (block, kv head)
constexpr int kFp16BlockBytes = kBlock * kHotTokenBytes;

// First error wins; later errors leave the word unchanged.
__device__ __forceinline__ void set_status(int32_t *status, int code) {
  if (status) atomicCAS(status, 0, code);
}

__device__ __forceinline__ uint32_t smem_addr(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---- mbarrier (CTA scope) ----
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count)
               : "memory");
}

__device__ __forceinline__ void mbar_fence_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t tx) {
  asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(
                   smem_addr(bar)),
               "r"(tx)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar))
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Non-blocking test of phase `parity` of `bar`.
__device__ __forceinline__ bool mbar_test_wait(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Limits below this many cycles are checked with non-blocking tests (a
// try_wait may suspend the thread in hardware for a while by itself).
constexpr long long kShortWaitCycles = 1ll << 20;

// Wait for phase `parity` of `bar` to complete, giving up after about
// `limit_cycles` SM clock cycles.  Returns false on timeout.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t *bar, uint32_t parity,
                                                  long long limit_cycles) {
  if (limit_cycles < kShortWaitCycles) {
    const long long t0 = clock64();
    while (!mbar_test_wait(bar, parity)) {
      if (clock64() - t0 > limit_cycles) return false;
    }
    return true;
  }
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > limit_cycles) return false;
  }
  return true;
}

// ---- 1-D bulk copy global -> shared (TMA engine), completes on an mbarrier.
// No cluster multicast.  dst and src 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes,
                                         uint64_t *bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint "
      "[%0], [%1], %2, [%3], %4;" ::"r"(smem_addr(dst)),
      "l"(src), "r"(bytes), "r"(smem_addr(bar)), "l"(policy)
      : "memory");
}

// Order this thread's generic-proxy writes to shared memory before later
// async-proxy (bulk copy) writes to the same bytes.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// L2 policy for data read once per decode step (KV tiles): evict first.
__device__ __forceinline__ uint64_t l2_policy_evict_first() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

// Arrival counter increment with acquire-release semantics at GPU scope.
// Used after a CTA barrier by one thread: it publishes the writes the CTA
// made before the barrier (release), and the thread that sees the final
// count observes every other CTA's published writes (acquire).
__device__ __forceinline__ int atomic_add_acq_rel_gpu(int32_t *p, int v) {
  int old;
  asm volatile("atom.add.acq_rel.gpu.s32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}

// ---- integer helpers ----
// Sign-extend the four 4-bit values held in the low nibbles of the bytes of
// u (high nibbles zero) to four int8 bytes.
__device__ __forceinline__ uint32_t sext_nibbles(uint32_t u) {
  return ((u ^ 0x08080808u) + 0x78787878u) ^ 0x80808080u;
}

__device__ __forceinline__ int clamp_code(int v, int q) { return v > q ? q : (v < -q ? -q : v); }

// ---- the cold-zone quantizer (IEEE division, round half to even, clamp) ----
// code of x under scale s; a zero scale (all-zero group) gives code 0
__device__ __forceinline__ int quantize(float x, float s, int q) {
  if (s == 0.f) return 0;
  return clamp_code(__float2int_rn(__fdiv_rn(x, s)), q);
}

// a code sealed under s_old, re-expressed under the larger scale s_new
__device__ __forceinline__ int requantize(int c, float s_old, float s_new, int q) {
  return clamp_code(__float2int_rn(__fdiv_rn(__fmul_rn(static_cast<float>(c), s_old), s_new)), q);
}

// INT4 packing: element e (0..7) of a 32-bit word is byte e%4, low nibble for
// e < 4, high nibble for e >= 4 (4-bit two's complement)
__device__ __forceinline__ int nib_get(uint32_t w, int e) {
  const int v = (w >> (8 * (e & 3) + 4 * (e >> 2))) & 0xf;
  return v >= 8 ? v - 16 : v;
}

__device__ __forceinline__ uint32_t nib_put(uint32_t w, int e, int c) {
  const int sh = 8 * (e & 3) + 4 * (e >> 2);
  return (w & ~(0xfu << sh)) | (static_cast<uint32_t>(c & 0xf) << sh);
}

// Re-quantization of the codes already in a tile.  `tbl` maps every code c
// to its re-quantized value tbl[c + 127]; only codes of slots < first change.
// Words of a tile, by layout: INT8 K token-major (32 words per slot), INT8 V
// channel-major with swizzled 16-byte chunks (16 words per channel row), INT4
// K (16 words per slot), INT4 V (8 words per channel row, swizzled 8-byte
// units).  requant_nwords() is the number of leading words that can hold
// sealed codes.
__device__ __forceinline__ int requant_nwords(int kv, bool int4, int first) {
  return !int4 ? (kv == 0 ? first * 32 : kTileBytes / 4) : (kv == 0 ? first * 16 : kTileBytes / 8);
}

__device__ __forceinline__ uint32_t requant_word(uint32_t x, int w, int kv, bool int4, int first,
                                                 const int8_t *tbl) {
  uint32_t y = x;
  if (!int4) {
    const int row = w >> 4;
    const int base = kv == 0 ? 0 : 16 * (((w >> 2) & 3) ^ ((row >> 1) & 3)) + 4 * (w & 3);
#pragma unroll
    for (int e = 0; e < 4; e++) {
      if (kv != 0 && base + e >= first) continue;
      const int c = static_cast<int8_t>((x >> (8 * e)) & 0xff);
      y = (y & ~(0xffu << (8 * e))) | (static_cast<uint32_t>(static_cast<uint8_t>(tbl[c + 127])) << (8 * e));
    }
  } else {
    const int row = w >> 3;
    const int base = kv == 0 ? 0 : 16 * (((w >> 1) & 3) ^ ((row >> 2) & 3)) + 8 * (w & 1);
#pragma unroll
    for (int e = 0; e < 8; e++) {
      if (kv != 0 && base + e >= first) continue;
      y = nib_put(y, e, tbl[nib_get(x, e) + 127]);
    }
  }
  return y;
}

}  // namespace hyb
