// append.cu -- hyb_kv_append: seal tokens leaving the hot zone into cold
// blocks and write the newest tokens into the hot ring.
//
// Method: web page "DeepSeek V4混合式KV Cache推理优化实战解析", section 4.2
// (quantize_int8 of the cold part), sections 2.1 / 3.1 (INT8, INT4 for L2
// blocks, block size 64, hot zone = most recent 32 tokens in FP16) and 3.2
// (per-block scale held in the block header, re-assigned inside the kernel);
// section 5.2 (quantization_bits 0: the cold zone stays FP16 -- sealed rows
// are copied unchanged).
//
// One CTA per sequence; warp w handles (kv head, K|V) pairs w, w+nwarps, ...
// A warp owns everything it writes (its tiles' bytes, its scale words and its
// hot-ring rows), so no inter-warp ordering is needed until seq_lens[b] is
// advanced after the final barrier.  Lane l covers channels 4l..4l+3.
//
// Bit-exactness: absmax is exact; the scale is an IEEE FP32 division; codes
// use IEEE division and round-half-even conversion; the re-quantization is an
// FP32 multiply followed by an IEEE division.  No contraction into FMA can
// occur in these expressions (__fmul_rn / __fdiv_rn are never fused).
#include "kernels.cuh"

namespace hyb {

// Re-quantize the codes of slots [0, first) of one tile from s_old to s_new.
// Every possible code is re-quantized once (table in shared memory, same
// arithmetic as requantize()); the tile is then rewritten by lookup, with
// its words loaded 16 at a time so their latencies overlap.
__device__ void requant_tile(uint8_t *tile, int kv, bool int4, int first, float s_old,
                             float s_new, int q, int lane, int8_t *tbl) {
  for (int c = lane - 127; c <= 127; c += 32)
    tbl[c + 127] = static_cast<int8_t>(requantize(c, s_old, s_new, q));
  __syncwarp();
  uint32_t *w32 = reinterpret_cast<uint32_t *>(tile);
  const int nwords = requant_nwords(kv, int4, first);
  constexpr int kBatch = 16;
  for (int w0 = lane; w0 < nwords; w0 += 32 * kBatch) {
    uint32_t x[kBatch];
#pragma unroll
    for (int j = 0; j < kBatch; j++) {
      const int w = w0 + 32 * j;
      x[j] = w < nwords ? w32[w] : 0u;
    }
#pragma unroll
    for (int j = 0; j < kBatch; j++) {
      const int w = w0 + 32 * j;
      if (w < nwords) w32[w] = requant_word(x[j], w, kv, int4, first, tbl);
    }
  }
  __syncwarp();
}

// Four FP16 channels 4*lane..4*lane+3 of position t (K if kv == 0, else V).
__device__ __forceinline__ void load4(const AppendArgs &a, int b, int h, int kv, int L_old, int t,
                                      int lane, float x[4]) {
  const __half *src;
  if (t < L_old)
    src = a.hot + ((((size_t)b * a.hkv + h) * a.hot_tokens + (t & (a.hot_tokens - 1))) * 2 + kv) * kDim;
  else
    src = (kv ? a.v_new : a.k_new) + (((size_t)b * a.max_new + (t - L_old)) * a.hkv + h) * kDim;
  const uint2 raw = *reinterpret_cast<const uint2 *>(src + 4 * lane);
  const __half2 lo = *reinterpret_cast<const __half2 *>(&raw.x);
  const __half2 hi = *reinterpret_cast<const __half2 *>(&raw.y);
  x[0] = __low2float(lo);
  x[1] = __high2float(lo);
  x[2] = __low2float(hi);
  x[3] = __high2float(hi);
}

__global__ void __launch_bounds__(512) append_kernel(AppendArgs a) {
  const int b = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nwarps = blockDim.x >> 5;
  const int L_old = a.seq_lens[b];
  const int n = a.n_new[b];
  if (n < 0 || n > a.max_new || L_old < 0) {
    if (threadIdx.x == 0) set_status(a.status, HYB_STATUS_BAD_N_NEW);
    return;
  }
  const long long L_new_ll = static_cast<long long>(L_old) + n;
  const int B = 1 << a.bshift;  // tokens per block
  if (L_new_ll - a.hot_tokens > static_cast<long long>(a.max_blocks) * B || L_new_ll > 0x7fffffffLL) {
    if (threadIdx.x == 0) set_status(a.status, HYB_STATUS_CAPACITY);
    return;
  }
  if (n == 0) return;
  const int L_new = static_cast<int>(L_new_ll);
  const int e0 = max(0, L_old - a.hot_tokens), e1 = max(0, L_new - a.hot_tokens);
  __shared__ int8_t s_tbl[16][256];  // per-warp re-quantization tables

  for (int pair = warp; pair < 2 * a.hkv; pair += nwarps) {
    const int h = pair >> 1, kv = pair & 1;
    for (int p0 = e0; p0 < e1;) {
      const int i = p0 / B;
      const int p1 = min((i + 1) * B, e1);
      const int first = p0 - i * B;
      const int phys = a.block_table[(size_t)b * a.max_blocks + i];
      if (phys < 0 || phys >= a.num_phys) {
        if (lane == 0) set_status(a.status, HYB_STATUS_BAD_BLOCK);
        p0 = p1;
        continue;
      }
      if (a.quant_bits == 0) {
        // FP16 cold block: the rows move unchanged (K row then V row per slot)
        __half *blk = reinterpret_cast<__half *>(a.cold + ((size_t)phys * a.hkv + h) * B * kHotTokenBytes);
        for (int t = p0; t < p1; t++) {
          const __half *src;
          if (t < L_old)
            src = a.hot + ((((size_t)b * a.hkv + h) * a.hot_tokens + (t & (a.hot_tokens - 1))) * 2 + kv) * kDim;
          else
            src = (kv ? a.v_new : a.k_new) + (((size_t)b * a.max_new + (t - L_old)) * a.hkv + h) * kDim;
          __half *dst = blk + ((t - i * B) * 2 + kv) * kDim;
          *reinterpret_cast<uint2 *>(dst + 4 * lane) = *reinterpret_cast<const uint2 *>(src + 4 * lane);
        }
        p0 = p1;
        continue;
      }
      const bool int4 = a.quant_bits == 4 || (a.n_int4 != nullptr && i < a.n_int4[b]);
      const int q = int4 ? 7 : 127;
      // absmax over the group's tokens and channels
      float amax = 0.f;
      for (int t0 = p0; t0 < p1; t0 += 8) {
        float x[8][4];
#pragma unroll
        for (int u = 0; u < 8; u++)
          if (t0 + u < p1) load4(a, b, h, kv, L_old, t0 + u, lane, x[u]);
#pragma unroll
        for (int u = 0; u < 8; u++)
          if (t0 + u < p1)
            for (int j = 0; j < 4; j++) amax = fmaxf(amax, fabsf(x[u][j]));
      }
      for (int m = 16; m > 0; m >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, m));
      const float s_c = __fdiv_rn(amax, static_cast<float>(q));
      // the block's 64-slot sub-blocks: K tile + V tile each
      uint8_t *tile0 = a.cold + ((((size_t)phys * a.hkv + h) << a.lsub) * 2 + kv) * kTileBytes;
      float *sp = a.scales + ((size_t)phys * a.hkv + h) * 2 + kv;
      float s = s_c;
      if (first != 0) {
        const float s_old = *sp;
        if (s_c > s_old) {
          for (int u = 0; u <= a.lsub; u++) {
            const int first_u = min(max(first - kBlock * u, 0), kBlock);
            if (first_u > 0)
              requant_tile(tile0 + (size_t)u * kTilePairBytes, kv, int4, first_u, s_old, s_c, q, lane, s_tbl[warp]);
          }
        } else {
          s = s_old;
        }
      }
      __syncwarp();
      for (int t0 = p0; t0 < p1; t0 += 8) {
        float xb[8][4];
#pragma unroll
        for (int u = 0; u < 8; u++)
          if (t0 + u < p1) load4(a, b, h, kv, L_old, t0 + u, lane, xb[u]);
#pragma unroll
        for (int u = 0; u < 8; u++) {
        const int t = t0 + u;
        if (t >= p1) break;
        const int slot_b = t - i * B;  // slot in the block: slot_b % 64 of sub-block slot_b / 64
        const int slot = slot_b & (kBlock - 1);
        uint8_t *tile = tile0 + (size_t)(slot_b >> 6) * kTilePairBytes;
        int c[4];
        for (int j = 0; j < 4; j++) c[j] = quantize(xb[u][j], s, q);
        if (!int4 && kv == 0) {
          uint32_t w = 0;
          for (int j = 0; j < 4; j++) w |= static_cast<uint32_t>(c[j] & 0xff) << (8 * j);
          *reinterpret_cast<uint32_t *>(tile + slot * kDim + 4 * lane) = w;
        } else if (!int4) {
          for (int j = 0; j < 4; j++) {
            const int ch = 4 * lane + j;
            tile[ch * 64 + 16 * ((slot >> 4) ^ ((ch >> 1) & 3)) + (slot & 15)] =
                static_cast<uint8_t>(c[j]);
          }
        } else if (kv == 0) {
          uint32_t nib = 0;
          for (int j = 0; j < 4; j++) nib |= static_cast<uint32_t>(c[j] & 0xf) << (8 * j);
          const uint32_t other = __shfl_xor_sync(0xffffffffu, nib, 1);
          if ((lane & 1) == 0)
            *reinterpret_cast<uint32_t *>(tile + slot * 64 + 4 * (lane >> 1)) = nib | (other << 4);
        } else {
          for (int j = 0; j < 4; j++) {
            const int ch = 4 * lane + j;
            const int unit = (slot >> 4) ^ ((ch >> 2) & 3);
            const int in = slot & 15;
            uint8_t *byte = tile + ch * 32 + unit * 8 + (in >> 3) * 4 + (in & 3);
            const uint8_t old = *byte;
            *byte = (in & 4) ? static_cast<uint8_t>((old & 0x0f) | ((c[j] & 0xf) << 4))
                             : static_cast<uint8_t>((old & 0xf0) | (c[j] & 0xf));
          }
        }
        }
      }
      if (lane == 0) *sp = s;
      __syncwarp();
      p0 = p1;
    }
    // newest min(n, hot) tokens into the hot ring (after their slots' old
    // occupants were read above)
    const int nh = min(n, a.hot_tokens);
    for (int t = L_new - nh; t < L_new; t++) {
      const __half *src =
          (kv ? a.v_new : a.k_new) + (((size_t)b * a.max_new + (t - L_old)) * a.hkv + h) * kDim;
      __half *dst = a.hot + ((((size_t)b * a.hkv + h) * a.hot_tokens + (t & (a.hot_tokens - 1))) * 2 + kv) * kDim;
      *reinterpret_cast<uint2 *>(dst + 4 * lane) = *reinterpret_cast<const uint2 *>(src + 4 * lane);
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) a.seq_lens[b] = L_new;
}

cudaError_t launch_append(const AppendArgs &a, int batch, cudaStream_t stream) {
  const int nwarps = min(2 * a.hkv, 16);
  append_kernel<<<batch, 32 * nwarps, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace hyb
