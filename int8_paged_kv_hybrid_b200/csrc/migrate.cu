// migrate.cu -- hyb_kv_migrate: cold blocks move between the INT8 ("L1") and
// the INT4 ("L2") tier in place, each with a new scale.
//
// Method: web page "DeepSeek V4混合式KV Cache推理优化实战解析", section 3.3
// (blocks are promoted to L1 / demoted to L2 by their access interval) and
// section 3.2 (a block that changes tier is given a new scale inside the
// kernel, with no host copy).  The tier is a count per sequence -- logical
// blocks below n_int4_blocks[b] are INT4 -- and a migration moves that count
// to target[b]: every sealed block between the two counts is re-quantized to
// the other width.  Per (block, kv head, K|V):
//   a = max |code * scale|   (= max|code| * scale: FP32 rounding is monotone)
//   scale' = a / Q'          (IEEE division; Q' = 7 or 127)
//   code' = clamp(round-half-even(code * scale / scale'), -Q', Q')
// -- the arithmetic of a tail block's re-quantization in hyb_kv_append, so the
// result is bit-exact with the oracle.
//
// One CTA per (block to move, kv head, sequence), 256 threads per 64-token
// sub-block of the block (512 for 128-token blocks, whose two sub-blocks
// share the scale): each thread holds its part of the K and V tiles in
// registers (codes of slots not yet sealed are taken as 0), the new scale
// and a 256-entry code table are computed, and the tiles are written back in
// the new packing.  A demoted tile's upper 4 KB (unused by INT4 codes) is
// left as it was: no reader of an INT4 tile looks at it.  A second launch
// then commits the new counts, after every CTA of the first has read the old
// ones.
#include "kernels.cuh"

namespace hyb {

constexpr int kMigThreads = 256;               // per 64-token sub-block
constexpr int kMigWarpsMax = 2 * kMigThreads / 32;  // 128-token blocks

// The sequence's move, or false (sequence left as it is) when the target is
// outside [0, max_blocks] or farther than max_delta from the current count.
__device__ __forceinline__ bool tier_move(const MigrateArgs &a, int b, int &lo, int &hi, int &tgt) {
  const int cur = a.n_int4[b];
  tgt = a.target[b];
  if (cur < 0 || cur > a.max_blocks || tgt < 0 || tgt > a.max_blocks || tgt - cur > a.max_delta ||
      cur - tgt > a.max_delta)
    return false;
  lo = min(cur, tgt);
  hi = max(cur, tgt);
  return true;
}

// Four table entries for the four INT8 codes of x, as bytes of one word.
// Entry u of the table holds the new code of the INT8 code whose byte is
// (u - 127) mod 256 (the -128 byte, never produced, reads as -127).
__device__ __forceinline__ uint32_t tbl4(const uint8_t *tbl, uint32_t x) {
  const uint32_t u = __vadd4(x, 0x7f7f7f7fu);  // per-byte index
  return static_cast<uint32_t>(tbl[u & 0xff]) | (static_cast<uint32_t>(tbl[(u >> 8) & 0xff]) << 8) |
         (static_cast<uint32_t>(tbl[(u >> 16) & 0xff]) << 16) | (static_cast<uint32_t>(tbl[u >> 24]) << 24);
}

// Largest |code| of the four INT8 codes of x (-128 read as 127).
__device__ __forceinline__ uint32_t absmax4(uint32_t x) {
  const uint32_t a = __vabsss4(x);  // per-byte |code|, saturating
  return max(max(a & 0xff, (a >> 8) & 0xff), max((a >> 16) & 0xff, a >> 24));
}

__global__ void __launch_bounds__(2 * kMigThreads) migrate_kernel(const MigrateArgs a) {
  const int k = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int tid_all = threadIdx.x, lane = tid_all & 31, warp = tid_all >> 5;
  const int nwarps = blockDim.x >> 5;
  const int u = tid_all / kMigThreads;    // this thread's sub-block
  const int tid = tid_all % kMigThreads;  // ... and its index there
  const int Bt = 1 << a.bshift;
  int lo, hi, tgt;
  if (!tier_move(a, b, lo, hi, tgt)) {
    if (k == 0 && h == 0 && tid_all == 0) set_status(a.status, HYB_STATUS_BAD_TIER);
    return;
  }
  const int i = lo + k;
  if (i >= hi) return;
  const int Lc = max(0, a.seq_lens[b] - a.hot_tokens);
  if (i * Bt >= Lc) return;  // nothing sealed in this block yet: only its tier changes
  const int sealed = max(0, min(min(kBlock, Bt), Lc - i * Bt - u * kBlock));  // in this sub-block
  const int phys = a.block_table[(size_t)b * a.max_blocks + i];
  if (phys < 0 || phys >= a.num_phys) {
    if (tid_all == 0) set_status(a.status, HYB_STATUS_BAD_BLOCK);
    return;
  }
  const bool demote = i < tgt;  // INT8 -> INT4
  const int qn = demote ? 7 : 127;

  __shared__ int red[2][kMigWarpsMax];
  __shared__ float s_new[2];
  __shared__ uint8_t tbl[2][256];
  uint8_t *tile = a.cold + ((((size_t)phys * a.hkv + h) << a.lsub) + u) * kTilePairBytes;

  // Every packed word maps onto a local piece of the other packing, so each
  // thread keeps its part of both tiles in registers, as INT8 bytes:
  //   INT8 K vector v (16 B): token v/8, channels 16(v%8)..+15
  //        <-> INT4 K words 2v, 2v+1 (8 channels each, same token);
  //   INT8 V vector v (16 B): channel v/4, the 16 slots of chunk position v%4
  //        <-> the INT4 V unit (2 words) of those 16 slots.
  // Thread tid takes INT8 vectors tid and tid + 256 of each tile.
  uint32_t x[2][2][4];  // [kv][vector][word]
#pragma unroll
  for (int kv = 0; kv < 2; kv++) {
#pragma unroll
    for (int r = 0; r < 2; r++) {
      const int v = tid + kMigThreads * r;
      if (demote) {
        const uint4 q = reinterpret_cast<const uint4 *>(tile + kv * kTileBytes)[v];
        x[kv][r][0] = q.x; x[kv][r][1] = q.y; x[kv][r][2] = q.z; x[kv][r][3] = q.w;
      } else {
        // INT4 source: the two words that hold the same 16 codes
        const uint32_t *src = reinterpret_cast<const uint32_t *>(tile + kv * kTileBytes);
        int wi;
        if (kv == 0) {
          wi = 2 * v;
        } else {
          const int c = v / 4;
          const int j = (v % 4) ^ ((c >> 1) & 3);  // slots 16j..16j+15
          wi = c * 8 + 2 * (j ^ ((c >> 2) & 3));
        }
        const uint2 p = *reinterpret_cast<const uint2 *>(src + wi);
        // sign-extend the nibbles to bytes: low nibbles are codes 0..3 of a
        // word, high nibbles codes 4..7
        x[kv][r][0] = sext_nibbles(p.x & 0x0f0f0f0fu);
        x[kv][r][1] = sext_nibbles((p.x >> 4) & 0x0f0f0f0fu);
        x[kv][r][2] = sext_nibbles(p.y & 0x0f0f0f0fu);
        x[kv][r][3] = sext_nibbles((p.y >> 4) & 0x0f0f0f0fu);
      }
    }
  }
  if (sealed < kBlock) {
    // a partial tail block: slots not yet sealed count as code 0
#pragma unroll
    for (int kv = 0; kv < 2; kv++)
#pragma unroll
      for (int r = 0; r < 2; r++) {
        const int v = tid + kMigThreads * r;
#pragma unroll
        for (int q = 0; q < 4; q++)
#pragma unroll
          for (int e = 0; e < 4; e++) {
            int t;
            if (kv == 0) {
              t = v / 8;
            } else {
              const int c = v / 4;
              t = 16 * ((v % 4) ^ ((c >> 1) & 3)) + 4 * q + e;
            }
            if (t >= sealed) x[kv][r][q] &= ~(0xffu << (8 * e));
          }
      }
  }
  // ---- largest |code| per tile, new scale, code table ----
#pragma unroll
  for (int kv = 0; kv < 2; kv++) {
    uint32_t m = 0;
#pragma unroll
    for (int r = 0; r < 2; r++)
#pragma unroll
      for (int q = 0; q < 4; q++) m = max(m, absmax4(x[kv][r][q]));
#pragma unroll
    for (int d = 16; d > 0; d >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, d));
    if (lane == 0) red[kv][warp] = static_cast<int>(m);
  }
  __syncthreads();
  if (tid_all < 2) {
    const int kvr = tid_all;
    int m = 0;
    for (int w = 0; w < nwarps; w++) m = max(m, red[kvr][w]);
    m = min(m, 127);
    const float s_old = a.scales[((size_t)phys * a.hkv + h) * 2 + kvr];
    s_new[kvr] = __fdiv_rn(__fmul_rn(static_cast<float>(m), s_old), static_cast<float>(qn));
  }
  __syncthreads();
  for (int e = tid_all; e < 2 * 256; e += blockDim.x) {
    const int kv = e >> 8, ue = e & 255;
    const int c = ue == 255 ? -127 : ue - 127;
    const float s_old = a.scales[((size_t)phys * a.hkv + h) * 2 + kv];
    const int cn = s_new[kv] == 0.f ? 0 : requantize(c, s_old, s_new[kv], qn);
    // INT4: the nibble; INT8: the byte
    tbl[kv][ue] = static_cast<uint8_t>(demote ? (cn & 0xf) : (cn & 0xff));
  }
  __syncthreads();  // every thread has read the old scales and its tile words

  // ---- write the tiles in the new packing, then the scales ----
#pragma unroll
  for (int kv = 0; kv < 2; kv++) {
    const uint8_t *tb = tbl[kv];
#pragma unroll
    for (int r = 0; r < 2; r++) {
      const int v = tid + kMigThreads * r;
      const uint32_t *w = x[kv][r];
      if (demote) {
        // codes 0..3 in the low nibbles, 4..7 in the high nibbles of a word
        const uint32_t o0 = tbl4(tb, w[0]) | (tbl4(tb, w[1]) << 4);
        const uint32_t o1 = tbl4(tb, w[2]) | (tbl4(tb, w[3]) << 4);
        uint2 *dst = reinterpret_cast<uint2 *>(tile + kv * kTileBytes);
        if (kv == 0) {
          dst[v] = make_uint2(o0, o1);
        } else {
          const int c = v / 4;
          const int j = (v % 4) ^ ((c >> 1) & 3);
          dst[c * 4 + (j ^ ((c >> 2) & 3))] = make_uint2(o0, o1);
        }
      } else {
        reinterpret_cast<uint4 *>(tile + kv * kTileBytes)[v] =
            make_uint4(tbl4(tb, w[0]), tbl4(tb, w[1]), tbl4(tb, w[2]), tbl4(tb, w[3]));
      }
    }
  }
  if (tid_all < 2) a.scales[((size_t)phys * a.hkv + h) * 2 + tid_all] = s_new[tid_all];
}

// The new counts, once every CTA of migrate_kernel has read the old ones.
__global__ void migrate_commit_kernel(const MigrateArgs a, int batch) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= batch) return;
  int lo, hi, tgt;
  if (tier_move(a, b, lo, hi, tgt)) a.n_int4[b] = tgt;
}

cudaError_t launch_migrate(const MigrateArgs &a, int batch, cudaStream_t stream) {
  if (a.max_delta > 0) {
    dim3 grid(a.max_delta, a.hkv, batch);
    migrate_kernel<<<grid, kMigThreads << a.lsub, 0, stream>>>(a);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  migrate_commit_kernel<<<(batch + 127) / 128, 128, 0, stream>>>(a, batch);
  return cudaGetLastError();
}

}  // namespace hyb
