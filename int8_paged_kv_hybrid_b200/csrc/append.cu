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
// Grid (2 * Hkv, batch): one CTA of 128 threads per (sequence, kv head,
// K|V).  Per cold block that receives sealed tokens: the new values are read
// once for the absmax (thread = channel), quantized into a shared-memory code
// matrix, and the block's tiles are then rewritten word by word with
// coalesced 32-bit stores -- each word assembled from the code matrix, from
// the codes already in the tile (re-quantized when the block's scale grows)
// or left alone.  A CTA owns every byte it writes (its tiles' K or V half, its
// scale word, its hot-ring rows).  A second launch advances seq_lens once
// every CTA of the first has read it.
//
// Bit-exactness: absmax is exact; the scale is an IEEE FP32 division; codes
// use IEEE division and round-half-even conversion; the re-quantization is an
// FP32 multiply followed by an IEEE division.  No contraction into FMA can
// occur in these expressions (__fmul_rn / __fdiv_rn are never fused).
#include "kernels.cuh"

namespace hyb {

constexpr int kAppendThreads = 128;  // thread = channel in the value passes

// Validity of sequence b's call (the same test in both launches): n_new in
// [0, max_new], seq_lens >= 0, and the new length within the block table.
// Returns 0, or the status code to record.
__device__ __forceinline__ int append_check(const AppendArgs &a, int L_old, int n) {
  if (n < 0 || n > a.max_new || L_old < 0) return HYB_STATUS_BAD_N_NEW;
  const long long L_new = static_cast<long long>(L_old) + n;
  if (L_new - a.hot_tokens > static_cast<long long>(a.max_blocks) << a.bshift || L_new > 0x7fffffffLL)
    return HYB_STATUS_CAPACITY;
  return 0;
}

// FP16 value of position t, channel c (K if kv == 0, else V): from the hot
// ring for positions already in the cache, else from the call's input.
__device__ __forceinline__ const __half *src_row(const AppendArgs &a, int b, int h, int kv, int L_old, int t) {
  if (t < L_old)
    return a.hot + ((((size_t)b * a.hkv + h) * a.hot_tokens + (t & (a.hot_tokens - 1))) * 2 + kv) * kDim;
  return (kv ? a.v_new : a.k_new) + (((size_t)b * a.max_new + (t - L_old)) * a.hkv + h) * kDim;
}

// Slot (within its 64-slot sub-block) and channel of element e of word w of a
// tile, for the four tile formats (see the cold-pool layout in hyb_kv.h).
__device__ __forceinline__ void word_elem(int w, int e, int kv, bool int4, int &slot, int &ch) {
  if (!int4) {
    if (kv == 0) {  // K INT8: token-major, 32 words per slot row
      slot = w >> 5;
      ch = 4 * (w & 31) + e;
    } else {        // V INT8: channel row of 16 words, 16-byte chunks swizzled
      ch = w >> 4;
      const int chunk = ((w >> 2) & 3) ^ ((ch >> 1) & 3);
      slot = 16 * chunk + 4 * (w & 3) + e;
    }
  } else {
    if (kv == 0) {  // K INT4: 16 words per slot row, 8 channels per word
      slot = w >> 4;
      ch = 8 * (w & 15) + e;
    } else {        // V INT4: channel row of 8 words, 8-byte units swizzled
      ch = w >> 3;
      const int unit = ((w >> 1) & 3) ^ ((ch >> 2) & 3);
      slot = 16 * unit + 8 * (w & 1) + e;
    }
  }
}

// Code matrix of one block's new slots, one byte per code.  K: token-major
// rows of 128 channels, so that the 4 (8) codes of an INT8 (INT4) K word are
// consecutive bytes; V: channel-major rows of the block's slots (pitch 132,
// which spreads the per-channel stores over the banks), so that the codes of
// a V word are consecutive bytes too.
constexpr int kCmPitchV = 2 * kBlock + 4;
union CodeMatrix {
  int8_t k[2 * kBlock][kDim];   // [block slot - first][channel]
  int8_t v[kDim][kCmPitchV];    // [channel][block slot - first]
};

struct AppendSmem {
  __half xs[2 * kBlock][kDim];  // the block's new values [block slot - first][channel]
  CodeMatrix cm;
  int8_t tbl[256];              // re-quantization table
  float s_max[kAppendThreads / 32];
};

__global__ void __launch_bounds__(kAppendThreads) append_kernel(AppendArgs a) {
  const int pair = blockIdx.x, b = blockIdx.y;
  const int h = pair >> 1, kv = pair & 1;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int L_old = a.seq_lens[b];
  const int n = a.n_new[b];
  const int bad = append_check(a, L_old, n);
  if (bad) {
    if (tid == 0 && pair == 0) set_status(a.status, bad);
    return;
  }
  if (n == 0) return;
  const int L_new = L_old + n;
  const int H = a.hot_tokens;
  const int B = 1 << a.bshift;  // tokens per block
  const int e0 = max(0, L_old - H), e1 = max(0, L_new - H);
  extern __shared__ __align__(16) uint8_t smem_raw[];
  AppendSmem &sm = *reinterpret_cast<AppendSmem *>(smem_raw);
  auto &xs = sm.xs;
  auto &cm = sm.cm;
  auto &tbl = sm.tbl;
  auto &s_max = sm.s_max;
  const int c = tid;  // channel

  for (int p0 = e0; p0 < e1;) {
    const int i = p0 / B;
    const int p1 = min((i + 1) * B, e1);
    const int first = p0 - i * B, last = p1 - i * B;  // new slots [first, last) of the block
    const int nn = p1 - p0;
    const int phys = a.block_table[(size_t)b * a.max_blocks + i];
    if (phys < 0 || phys >= a.num_phys) {
      if (tid == 0) set_status(a.status, HYB_STATUS_BAD_BLOCK);
      p0 = p1;
      continue;
    }
    // the new values of channel c, 16 loads in flight at a time, into xs;
    // their absmax (FP32, exact)
    float amax = 0.f;
    for (int t0 = 0; t0 < nn; t0 += 16) {
      __half x[16];
#pragma unroll
      for (int u = 0; u < 16; u++)
        x[u] = t0 + u < nn ? src_row(a, b, h, kv, L_old, p0 + t0 + u)[c] : __float2half_rn(0.f);
#pragma unroll
      for (int u = 0; u < 16; u++) {
        if (t0 + u < nn) {
          xs[t0 + u][c] = x[u];
          amax = fmaxf(amax, fabsf(__half2float(x[u])));
        }
      }
    }
    if (a.quant_bits == 0) {
      // FP16 cold block: the rows move unchanged (K row then V row per slot)
      __half *blk = reinterpret_cast<__half *>(a.cold + ((size_t)phys * a.hkv + h) * B * kHotTokenBytes);
      for (int t = 0; t < nn; t++) blk[((first + t) * 2 + kv) * kDim + c] = xs[t][c];
      __syncthreads();  // xs reused by the next block
      p0 = p1;
      continue;
    }
    const bool int4 = a.quant_bits == 4 || (a.n_int4 != nullptr && i < a.n_int4[b]);
    const int q = int4 ? 7 : 127;
#pragma unroll
    for (int m = 16; m > 0; m >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, m));
    if (lane == 0) s_max[warp] = amax;
    __syncthreads();
    amax = fmaxf(fmaxf(s_max[0], s_max[1]), fmaxf(s_max[2], s_max[3]));
    const float s_c = __fdiv_rn(amax, static_cast<float>(q));
    float *sp = a.scales + ((size_t)phys * a.hkv + h) * 2 + kv;
    float s = s_c;
    bool rq = false;
    float s_old = 0.f;
    if (first != 0) {
      s_old = *sp;
      if (s_c > s_old) rq = true;
      else s = s_old;
    }
    if (rq)
      for (int cc = tid - 127; cc <= 127; cc += kAppendThreads) tbl[cc + 127] = static_cast<int8_t>(requantize(cc, s_old, s, q));
    // the new slots' codes, in the layout of this CTA's half (K or V)
    for (int t = 0; t < nn; t++) {
      const int8_t code = static_cast<int8_t>(quantize(__half2float(xs[t][c]), s, q));
      if (kv == 0) cm.k[t][c] = code;
      else cm.v[c][t] = code;
    }
    __syncthreads();
    // rewrite the tiles of the block's 64-slot sub-blocks: only words holding
    // a new slot, or an existing one when the scale grew
    const int St = min(B, kBlock);
    const int lo = rq ? 0 : first;  // slots [lo, last) change
    const int ne = int4 ? 8 : 4;    // codes per 32-bit word
    for (int u = (lo / kBlock); u <= (last - 1) / kBlock; u++) {
      uint32_t *tile = reinterpret_cast<uint32_t *>(
          a.cold + ((((size_t)phys * a.hkv + h) << a.lsub) + u) * kTilePairBytes + kv * kTileBytes);
      const int s0 = max(lo - kBlock * u, 0), s1 = min(last - kBlock * u, St);  // slots of this sub-block
      const int fu = first - kBlock * u;  // new slots of this sub-block start at fu (may be < 0 or > s1)
      // words to visit: K rows [s0, s1); V every channel row (its words are
      // filtered by slot range)
      const int wpr = int4 ? (kv == 0 ? 16 : 8) : (kv == 0 ? 32 : 16);  // words per row
      const int w_begin = kv == 0 ? s0 * wpr : 0;
      const int w_end = kv == 0 ? s1 * wpr : kDim * wpr;
      for (int w = w_begin + tid; w < w_end; w += kAppendThreads) {
        // element e of the word: K -> (slot0, ch0 + e), V -> (slot0 + e, ch0)
        int slot0, ch0;
        word_elem(w, 0, kv, int4, slot0, ch0);
        if (kv != 0 && (slot0 + ne <= s0 || slot0 >= s1)) continue;  // no slot of the word changes
        const bool all_new = slot0 >= fu && (kv == 0 || slot0 + ne <= s1);
        uint32_t y;
        if (all_new && !int4) {
          // four new INT8 codes: consecutive bytes of the code matrix
          const int8_t *src = kv == 0 ? &cm.k[slot0 - fu][ch0] : &cm.v[ch0][slot0 - fu];
          y = kv == 0 ? *reinterpret_cast<const uint32_t *>(src)
                      : static_cast<uint32_t>(static_cast<uint8_t>(src[0])) |
                            (static_cast<uint32_t>(static_cast<uint8_t>(src[1])) << 8) |
                            (static_cast<uint32_t>(static_cast<uint8_t>(src[2])) << 16) |
                            (static_cast<uint32_t>(static_cast<uint8_t>(src[3])) << 24);
        } else {
          const uint32_t x = all_new ? 0u : tile[w];
          y = x;
#pragma unroll
          for (int e = 0; e < 8; e++) {
            if (e >= ne) break;
            const int sl = kv == 0 ? slot0 : slot0 + e;
            const int ch = kv == 0 ? ch0 + e : ch0;
            if (sl < s0 || sl >= s1) continue;  // unchanged
            int code;
            if (sl >= fu) {
              code = kv == 0 ? cm.k[sl - fu][ch] : cm.v[ch][sl - fu];  // new slot
            } else {  // existing slot under a grown scale
              const int old = int4 ? nib_get(x, e) : static_cast<int8_t>((x >> (8 * e)) & 0xff);
              code = tbl[old + 127];
            }
            if (int4) y = nib_put(y, e, code);
            else y = (y & ~(0xffu << (8 * e))) | (static_cast<uint32_t>(code & 0xff) << (8 * e));
          }
        }
        tile[w] = y;
      }
    }
    if (tid == 0) *sp = s;
    __syncthreads();  // xs, cm and tbl are reused by the next block
    p0 = p1;
  }
  // newest min(n, hot) tokens into the hot ring (their slots' old occupants
  // were read above, before the barrier)
  __syncthreads();
  const int nh = min(n, H);
  for (int t = L_new - nh; t < L_new; t++) {
    const __half *src = (kv ? a.v_new : a.k_new) + (((size_t)b * a.max_new + (t - L_old)) * a.hkv + h) * kDim;
    __half *dst = a.hot + ((((size_t)b * a.hkv + h) * H + (t & (H - 1))) * 2 + kv) * kDim;
    dst[c] = src[c];
  }
}

// seq_lens[b] += n_new[b] for every valid call, after append_kernel (stream order).
__global__ void append_lens_kernel(AppendArgs a, int batch) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= batch) return;
  const int L_old = a.seq_lens[b];
  const int n = a.n_new[b];
  if (append_check(a, L_old, n) == 0) a.seq_lens[b] = L_old + n;
}

cudaError_t launch_append(const AppendArgs &a, int batch, cudaStream_t stream) {
  static int configured_dev_mask = 0;  // one bit per device
  int dev = 0;
  cudaError_t e0 = cudaGetDevice(&dev);
  if (e0 != cudaSuccess) return e0;
  if (dev < 31 && !(configured_dev_mask & (1 << dev))) {
    e0 = cudaFuncSetAttribute(append_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              static_cast<int>(sizeof(AppendSmem)));
    if (e0 != cudaSuccess) return e0;
    configured_dev_mask |= 1 << dev;
  }
  append_kernel<<<dim3(2 * a.hkv, batch), kAppendThreads, sizeof(AppendSmem), stream>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  append_lens_kernel<<<(batch + 127) / 128, 128, 0, stream>>>(a, batch);
  return cudaGetLastError();
}

}  // namespace hyb
