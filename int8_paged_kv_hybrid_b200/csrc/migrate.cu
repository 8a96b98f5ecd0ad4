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
// One CTA per (block to move, kv head, sequence): the K and V tiles are
// unpacked into shared memory (codes of slots not yet sealed are taken as 0),
// the new scale and a 255-entry code table are computed, and the tiles are
// written back in the new packing (a demoted tile's unused upper 4 KB is
// zeroed).  A second launch then commits the new counts, after every CTA of
// the first has read the old ones.
#include "kernels.cuh"

namespace hyb {

constexpr int kMigThreads = 256;
constexpr int kMigWarps = kMigThreads / 32;

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

__global__ void __launch_bounds__(kMigThreads) migrate_kernel(const MigrateArgs a) {
  const int k = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int lo, hi, tgt;
  if (!tier_move(a, b, lo, hi, tgt)) {
    if (k == 0 && h == 0 && tid == 0) set_status(a.status, HYB_STATUS_BAD_TIER);
    return;
  }
  const int i = lo + k;
  if (i >= hi) return;
  const int Lc = max(0, a.seq_lens[b] - kHot);
  if (i * kBlock >= Lc) return;  // nothing sealed in this block yet: only its tier changes
  const int sealed = min(kBlock, Lc - i * kBlock);
  const int phys = a.block_table[(size_t)b * a.max_blocks + i];
  if (phys < 0 || phys >= a.num_phys) {
    if (tid == 0) set_status(a.status, HYB_STATUS_BAD_BLOCK);
    return;
  }
  const bool demote = i < tgt;  // INT8 -> INT4
  const int qn = demote ? 7 : 127;

  __shared__ __align__(16) int8_t cs[2][kBlock][kDim];  // codes, logical [kv][slot][channel]
  __shared__ int red[2][kMigWarps];
  __shared__ float s_new[2];
  __shared__ int8_t tbl[2][256];
  uint8_t *tile = a.cold + ((size_t)phys * a.hkv + h) * kTilePairBytes;

  // ---- unpack the old tiles; slots not yet sealed count as code 0 ----
  int amax[2] = {0, 0};
  if (demote) {
    // INT8: 512 16-byte vectors per tile
    for (int kv = 0; kv < 2; kv++) {
      const uint4 *src = reinterpret_cast<const uint4 *>(tile + kv * kTileBytes);
      for (int v = tid; v < kTileBytes / 16; v += kMigThreads) {
        const uint4 x = src[v];
        const uint32_t w[4] = {x.x, x.y, x.z, x.w};
        const int o = 16 * v;
#pragma unroll
        for (int e = 0; e < 16; e++) {
          // -128 is never produced; a corrupt byte is clamped so the table index stays in range
          int code = max(-127, static_cast<int>(static_cast<int8_t>((w[e >> 2] >> (8 * (e & 3))) & 0xff)));
          int t, c;
          if (kv == 0) {
            t = o / kDim;
            c = o % kDim + e;
          } else {
            c = o / kBlock;
            const int j = ((o % kBlock) / 16) ^ ((c >> 1) & 3);
            t = 16 * j + e;
          }
          if (t >= sealed) code = 0;
          cs[kv][t][c] = static_cast<int8_t>(code);
          amax[kv] = max(amax[kv], abs(code));
        }
      }
    }
  } else {
    // INT4: 1024 32-bit words per tile, 8 codes each
    for (int kv = 0; kv < 2; kv++) {
      const uint32_t *src = reinterpret_cast<const uint32_t *>(tile + kv * kTileBytes);
      for (int w = tid; w < kTileBytes / 8; w += kMigThreads) {
        const uint32_t x = src[w];
#pragma unroll
        for (int e = 0; e < 8; e++) {
          int code = nib_get(x, e);
          int t, c;
          if (kv == 0) {
            t = w / 16;
            c = 8 * (w % 16) + e;
          } else {
            c = w / 8;
            const int wi = w % 8;
            const int j = (wi >> 1) ^ ((c >> 2) & 3);
            t = 16 * j + 8 * (wi & 1) + e;
          }
          if (t >= sealed) code = 0;
          cs[kv][t][c] = static_cast<int8_t>(code);
          amax[kv] = max(amax[kv], abs(code));
        }
      }
    }
  }
  // ---- largest |code| per tile, new scale, code table ----
#pragma unroll
  for (int kv = 0; kv < 2; kv++) {
    int m = amax[kv];
#pragma unroll
    for (int d = 16; d > 0; d >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, d));
    if (lane == 0) red[kv][warp] = m;
  }
  __syncthreads();
  if (tid < 2) {
    int m = 0;
#pragma unroll
    for (int w = 0; w < kMigWarps; w++) m = max(m, red[tid][w]);
    const float s_old = a.scales[((size_t)phys * a.hkv + h) * 2 + tid];
    s_new[tid] = __fdiv_rn(__fmul_rn(static_cast<float>(m), s_old), static_cast<float>(qn));
  }
  __syncthreads();
  for (int e = tid; e < 2 * 255; e += kMigThreads) {
    const int kv = e / 255, c = e % 255 - 127;
    const float s_old = a.scales[((size_t)phys * a.hkv + h) * 2 + kv];
    tbl[kv][c + 127] = static_cast<int8_t>(s_new[kv] == 0.f ? 0 : requantize(c, s_old, s_new[kv], qn));
  }
  __syncthreads();  // every thread has read the old scales and tiles

  // ---- write the tiles in the new packing, then the scales ----
  if (demote) {
    for (int kv = 0; kv < 2; kv++) {
      uint32_t *dst = reinterpret_cast<uint32_t *>(tile + kv * kTileBytes);
      for (int w = tid; w < kTileBytes / 8; w += kMigThreads) {
        uint32_t x = 0;
#pragma unroll
        for (int e = 0; e < 8; e++) {
          int t, c;
          if (kv == 0) {
            t = w / 16;
            c = 8 * (w % 16) + e;
          } else {
            c = w / 8;
            const int wi = w % 8;
            const int j = (wi >> 1) ^ ((c >> 2) & 3);
            t = 16 * j + 8 * (wi & 1) + e;
          }
          x = nib_put(x, e, tbl[kv][cs[kv][t][c] + 127]);
        }
        dst[w] = x;
      }
      uint4 *hi4 = reinterpret_cast<uint4 *>(tile + kv * kTileBytes + kTileBytes / 2);
      for (int v = tid; v < kTileBytes / 2 / 16; v += kMigThreads) hi4[v] = make_uint4(0u, 0u, 0u, 0u);
    }
  } else {
    for (int kv = 0; kv < 2; kv++) {
      uint32_t *dst = reinterpret_cast<uint32_t *>(tile + kv * kTileBytes);
      for (int w = tid; w < kTileBytes / 4; w += kMigThreads) {
        const int o = 4 * w;
        uint32_t x = 0;
#pragma unroll
        for (int e = 0; e < 4; e++) {
          int t, c;
          if (kv == 0) {
            t = o / kDim;
            c = o % kDim + e;
          } else {
            c = o / kBlock;
            const int j = ((o % kBlock) / 16) ^ ((c >> 1) & 3);
            t = 16 * j + (o % 16) + e;
          }
          x |= static_cast<uint32_t>(static_cast<uint8_t>(tbl[kv][cs[kv][t][c] + 127])) << (8 * e);
        }
        dst[w] = x;
      }
    }
  }
  if (tid < 2) a.scales[((size_t)phys * a.hkv + h) * 2 + tid] = s_new[tid];
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
    migrate_kernel<<<grid, kMigThreads, 0, stream>>>(a);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  migrate_commit_kernel<<<(batch + 127) / 128, 128, 0, stream>>>(a, batch);
  return cudaGetLastError();
}

}  // namespace hyb
