// sparse.cu -- sparse L2 attention: of the tokens a sequence holds in its INT4
// ("L2") cold blocks, each query head attends only the top_k with the
// largest scores; the rest of the cache is attended densely by the decode
// kernel (run with l2_skip), and the two softmax pieces are merged here.
//
// Method: web page "DeepSeek V4混合式KV Cache推理优化实战解析", section 2.2 (L2
// cold blocks keep only the KV of the top-k attention scores) and section 5.3
// (sparse_top_k: default 32, min(128, context_length / 256) for long
// contexts).  Selection key of an L2 token for a query head: the exact
// integer dot product of the head's q in 16-bit fixed point (the decode
// kernel's quantize_q) with the token's INT4 K codes, times the block's K
// scale, in FP32; equal keys keep the older position.
//
//  l2_score_kernel   grid (chunks of L2 blocks, Hkv, batch): the keys of every
//                    L2 token for the G query heads of a kv head, from the
//                    INT4 K tiles only (4 KB per block).
//  l2_topk_kernel    grid (Hq, batch): radix select of the top_k keys (four
//                    8-bit passes over histograms in shared memory), ordered
//                    compaction of the selected positions, softmax over them
//                    in FP32 with their INT4 V codes, and the log-sum-exp
//                    merge with the dense pass's output and log-sum-exp.
#include "kernels.cuh"

namespace hyb {

constexpr int kScoreThreads = 128;
constexpr float kLn2f = 0.6931471805599453f;

// Tokens of sequence b held in its INT4 blocks (the oldest ones), or 0 when
// its length is out of range (the dense pass reports that).
__device__ __forceinline__ int l2_count(const SparseArgs &a, int b) {
  const int L = a.seq_lens[b];
  if (L < 0) return 0;
  const int Lc = max(0, L - a.hot_tokens);
  const long long n4 = a.quant_bits == 4 ? a.max_blocks : (a.n_int4 ? a.n_int4[b] : 0);
  const long long n = min(static_cast<long long>(Lc), max(0LL, n4) << a.bshift);
  return n > a.max_l2 ? -1 : static_cast<int>(n);
}

// Monotone map of a finite float to uint32 (larger float, larger word).
__device__ __forceinline__ uint32_t key_order(float f) {
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ int sext4(uint32_t nib) { return static_cast<int>(nib << 28) >> 28; }

__global__ void __launch_bounds__(kScoreThreads) l2_score_kernel(const SparseArgs a) {
  const int chunk = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = a.hq / a.hkv;
  const int n = l2_count(a, b);
  if (n <= 0) return;
  // units of St tokens: 64-token sub-blocks (a block is 1 << lsub of them),
  // or whole 32-token blocks
  const int St = min(kBlock, 1 << a.bshift);
  const int nb = (n + St - 1) / St;
  const int blk0 = chunk * a.blocks_per_cta;
  if (blk0 >= nb) return;

  // q of the G heads in 16-bit fixed point, as the decode kernel makes it
  __shared__ alignas(16) int16_t qi[8][kDim];
  for (int j = warp; j < G; j += kScoreThreads / 32) {
    const __half *qh = a.q + ((size_t)b * a.hq + h * G + j) * kDim;
    float qv[4];
    float amax = 0.f;
#pragma unroll
    for (int t = 0; t < 4; t++) {
      qv[t] = __half2float(qh[lane + 32 * t]);
      amax = fmaxf(amax, fabsf(qv[t]));
    }
#pragma unroll
    for (int m = 16; m > 0; m >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, m));
    const float inv = amax > 0.f ? 32767.f / amax : 0.f;
#pragma unroll
    for (int t = 0; t < 4; t++) {
      const int v = __float2int_rn(qv[t] * inv);
      qi[j][lane + 32 * t] = static_cast<int16_t>(max(-32767, min(32767, v)));
    }
  }
  __syncthreads();

  // the chunk's INT4 K tiles (4 KB each) staged in shared memory, every
  // thread's loads issued together
  constexpr int kMaxChunk = 4;
  __shared__ alignas(16) uint32_t tiles[kMaxChunk][1024];
  __shared__ int s_phys[kMaxChunk];
  const int nblk = min(nb - blk0, min(a.blocks_per_cta, kMaxChunk));
  uint4 stage[kMaxChunk][2];
#pragma unroll
  for (int t = 0; t < kMaxChunk; t++) {
    stage[t][0] = make_uint4(0u, 0u, 0u, 0u);
    stage[t][1] = stage[t][0];
    if (t < nblk) {
      const int unit = blk0 + t;
      const int phys = a.block_table[(size_t)b * a.max_blocks + (unit >> a.lsub)];
      const bool okp = phys >= 0 && phys < a.num_phys;
      if (tid == 0) s_phys[t] = okp ? phys : -1;
      if (!okp && tid == 0) set_status(a.status, HYB_STATUS_BAD_BLOCK);
      if (okp) {
        const size_t pair = (((size_t)phys * a.hkv + h) << a.lsub) + (unit & ((1 << a.lsub) - 1));
        const uint4 *src = reinterpret_cast<const uint4 *>(a.cold + pair * kTilePairBytes);
        stage[t][0] = src[tid];
        stage[t][1] = src[kScoreThreads + tid];
      }
    }
  }
#pragma unroll
  for (int t = 0; t < kMaxChunk; t++) {
    if (t < nblk) {
      // 16-byte chunk c of token row r stored at chunk c ^ ((r / 2) % 4), so
      // that the reads below spread over the banks
#pragma unroll
      for (int r2 = 0; r2 < 2; r2++) {
        const int v = r2 * kScoreThreads + tid, row = v >> 2;
        reinterpret_cast<uint4 *>(tiles[t])[row * 4 + ((v & 3) ^ ((row >> 1) & 3))] = stage[t][r2];
      }
    }
  }
  __syncthreads();

  // thread: token tok of a block, half of its 16 words (channels 8wi..8wi+7)
  const int tok = tid >> 1, half = tid & 1;
  for (int t = 0; t < nblk; t++) {
    const int blk = blk0 + t;
    const int phys = s_phys[t];
    const bool okp = phys >= 0;
    int dot[8];
#pragma unroll
    for (int g = 0; g < 8; g++) dot[g] = 0;
    if (okp) {
      // INT4 K: 64 bytes per token, word w holds channels 8w..8w+7 (byte i:
      // channel 8w+i in the low nibble, 8w+4+i in the high nibble)
      // per word: the codes as bytes (channels 8w..8w+3, then 8w+4..8w+7)
      // against q pairs, two 16x8-bit products per dp2a, exact in int32
      // the two threads of a token take alternate words (wi = 2w + half), so
      // their q chunks are adjacent
      const uint32_t *kp = tiles[t] + tok * 16;
      const int sw = (tok >> 1) & 3;
#pragma unroll 2
      for (int w = 0; w < 8; w++) {
        const int wi = 2 * w + half;
        const uint32_t word = kp[(((wi >> 2) ^ sw) << 2) + (wi & 3)];
        const int lo4 = static_cast<int>(sext_nibbles(word & 0x0f0f0f0fu));
        const int hi4 = static_cast<int>(sext_nibbles((word >> 4) & 0x0f0f0f0fu));
        const int cb = 8 * wi;
#pragma unroll
        for (int g = 0; g < 8; g++) {
          if (g < G) {
            const uint4 qp = *reinterpret_cast<const uint4 *>(&qi[g][cb]);  // channels cb..cb+7
            int d = dot[g];
            d = __dp2a_lo(static_cast<int>(qp.x), lo4, d);
            d = __dp2a_hi(static_cast<int>(qp.y), lo4, d);
            d = __dp2a_lo(static_cast<int>(qp.z), hi4, d);
            d = __dp2a_hi(static_cast<int>(qp.w), hi4, d);
            dot[g] = d;
          }
        }
      }
    }
#pragma unroll
    for (int g = 0; g < 8; g++) dot[g] += __shfl_xor_sync(0xffffffffu, dot[g], 1);
    const int pos = blk * St + tok;
    if (half == 0 && tok < St && pos < n) {
      const float sk = okp ? a.scales[((size_t)phys * a.hkv + h) * 2] : 0.f;
#pragma unroll
      for (int g = 0; g < 8; g++) {
        if (g < G) {
          // the key orders tokens as their logits do: negated for a negative
          // softmax scale
          float key = okp ? __fmul_rn(__int2float_rn(dot[g]), sk) : -INFINITY;
          if (okp && a.qk_scale < 0.f) key = -key;
          if (key == 0.f) key = 0.f;  // -0 and +0 are one key
          a.keys[((size_t)b * a.hq + h * G + g) * a.max_l2 + pos] = key;
        }
      }
    }
  }
}

// Exclusive prefix count of `flag` over the CTA's kT threads in thread order;
// *total gets the CTA's count.  Every thread calls it.
template <int kT>
__device__ __forceinline__ int cta_prefix(bool flag, int *s_warp, int tid, int *total) {
  const int lane = tid & 31, warp = tid >> 5;
  const unsigned bal = __ballot_sync(0xffffffffu, flag);
  if (lane == 0) s_warp[warp] = __popc(bal);
  __syncthreads();
  int before = 0, all = 0;
#pragma unroll
  for (int w = 0; w < kT / 32; w++) {
    const int c = s_warp[w];
    before += w < warp ? c : 0;
    all += c;
  }
  __syncthreads();
  *total = all;
  return before + __popc(bal & ((1u << lane) - 1u));
}

template <int kT>
__device__ __forceinline__ float cta_reduce(float v, float *s_red, int tid, bool is_max) {
  const int lane = tid & 31, warp = tid >> 5;
#pragma unroll
  for (int m = 16; m > 0; m >>= 1) {
    const float o = __shfl_xor_sync(0xffffffffu, v, m);
    v = is_max ? fmaxf(v, o) : v + o;
  }
  if (lane == 0) s_red[warp] = v;
  __syncthreads();
  float r = s_red[0];
#pragma unroll
  for (int w = 1; w < kT / 32; w++) r = is_max ? fmaxf(r, s_red[w]) : r + s_red[w];
  __syncthreads();
  return r;
}

// kT threads per CTA: 1024 for long L2 ranges, 256 for short ones.
template <int kT>
__global__ void __launch_bounds__(kT) l2_topk_kernel(const SparseArgs a) {
  constexpr int kTopkThreads = kT;
  constexpr int kWarpsT = kT / 32;
  const int hh = blockIdx.x, b = blockIdx.y;
  const int tid = threadIdx.x;
  const int G = a.hq / a.hkv;
  const int h = hh / G;
  const int n = l2_count(a, b);
  const int k = min(a.top_k, max(n, 0));
  if (k <= 0) return;  // no L2 token attended: the dense result stands
  const float *keys = a.keys + ((size_t)b * a.hq + hh) * a.max_l2;

  constexpr int kParts = kTopkThreads / kDim;
  constexpr int kHists = kWarpsT / 4;
  __shared__ int hist[kHists][256];  // one histogram per 4 warps (fewer colliding atomics)
  __shared__ int s_warp[kTopkThreads / 32];
  __shared__ float s_red[kTopkThreads / 32];
  __shared__ int s_digit, s_need, s_eq, s_cnt;
  __shared__ int s_pos[kMaxTopK];
  __shared__ float s_p[kMaxTopK];
  __shared__ float s_sv[kMaxTopK];
  __shared__ int s_vt[kMaxTopK];
  __shared__ float s_acc[kParts][kDim];
  const float4 *keys4 = reinterpret_cast<const float4 *>(keys);  // rows are 256-byte aligned
  const int n4 = (n + 3) / 4;

  // ---- the k-th largest key (exact), by four 8-bit radix passes ----
  uint32_t thr = 0;
  int need_eq = k, n_eq = 0;
  if (k < n) {
    uint32_t prefix = 0, mask = 0;
    int need = k;
    for (int pass = 0; pass < 4; pass++) {
      const int shift = 24 - 8 * pass;
      for (int i = tid; i < kHists * 256; i += kT) hist[i >> 8][i & 255] = 0;
      __syncthreads();
      const int warp = tid >> 5, lane = tid & 31;
      // the same trip count for every lane, so that whole warps match bins
      for (int i4b = 0; i4b < n4; i4b += kT) {
        const int i4 = i4b + tid;
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        if (i4 < n4) v = keys4[i4];
        const float e[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int t = 0; t < 4; t++) {
          const uint32_t u = key_order(e[t]);
          const bool in = i4 < n4 && 4 * i4 + t < n && (u & mask) == prefix;
          const int bin = in ? static_cast<int>((u >> shift) & 255u) : 256;
          // lanes with the same bin add once, by their lowest lane
          const unsigned peers = __match_any_sync(0xffffffffu, bin);
          if (in && lane == __ffs(peers) - 1) atomicAdd(&hist[warp >> 2][bin], __popc(peers));
        }
      }
      __syncthreads();
      // fold the warps' histograms into the first
      for (int d = tid; d < 256; d += kT) {
        int sum = 0;
#pragma unroll
        for (int w = 0; w < kHists; w++) sum += hist[w][d];
        hist[0][d] = sum;
      }
      __syncthreads();
      if (tid == 0) {
        int above = 0, d = 255;
        for (; d > 0; d--) {
          if (above + hist[0][d] >= need) break;
          above += hist[0][d];
        }
        s_digit = d;
        s_need = need - above;
        s_eq = hist[0][d];  // after the last pass: the keys equal to the threshold
      }
      __syncthreads();
      prefix |= static_cast<uint32_t>(s_digit) << shift;
      mask |= 255u << shift;
      need = s_need;
      n_eq = s_eq;
      __syncthreads();
    }
    thr = prefix;
    need_eq = need;
  }

  // ---- the selected positions ----
  if (k >= n) {
    for (int i = tid; i < n; i += kTopkThreads) s_pos[i] = i;
  } else if (need_eq == n_eq) {
    // every key >= the threshold is taken: gather in any order, then sort
    if (tid == 0) s_cnt = 0;
    __syncthreads();
    for (int i4 = tid; i4 < n4; i4 += kTopkThreads) {
      const float4 v = keys4[i4];
      const float e[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int t = 0; t < 4; t++) {
        const int i = 4 * i4 + t;
        if (i < n && key_order(e[t]) >= thr) {
          const int slot = atomicAdd(&s_cnt, 1);
          if (slot < kMaxTopK) s_pos[slot] = i;
        }
      }
    }
    __syncthreads();
    // bitonic sort of the k positions (ascending), padded to a power of two
    int p2 = 1;
    while (p2 < k) p2 <<= 1;
    for (int i = k + tid; i < p2; i += kTopkThreads) s_pos[i] = 0x7fffffff;
    __syncthreads();
    for (int size = 2; size <= p2; size <<= 1) {
      for (int stride = size >> 1; stride > 0; stride >>= 1) {
        for (int i = tid; i < p2; i += kTopkThreads) {
          const int j = i ^ stride;
          if (j > i) {
            const int x = s_pos[i], y = s_pos[j];
            const bool up = (i & size) == 0;
            if ((x > y) == up) {
              s_pos[i] = y;
              s_pos[j] = x;
            }
          }
        }
        __syncthreads();
      }
    }
  } else {
    // only some of the keys equal to the threshold are taken (the older
    // ones): ordered compaction in position order
    int base = 0, eq_seen = 0;
    for (int c0 = 0; c0 < n; c0 += kTopkThreads) {
      const int i = c0 + tid;
      const uint32_t u = i < n ? key_order(keys[i]) : 0u;
      const bool gt = i < n && u > thr;
      const bool eq = i < n && u == thr;
      int eq_tot;
      const int eq_rank = cta_prefix<kT>(eq, s_warp, tid, &eq_tot);
      const bool sel = gt || (eq && eq_seen + eq_rank < need_eq);
      eq_seen += eq_tot;
      int sel_tot;
      const int r = cta_prefix<kT>(sel, s_warp, tid, &sel_tot);
      if (sel && base + r < kMaxTopK) s_pos[base + r] = i;
      base += sel_tot;
    }
  }
  __syncthreads();
  const int ns = k;
  // the selection, left in the workspace for the caller
  for (int j = tid; j < ns; j += kTopkThreads) a.sel[((size_t)b * a.hq + hh) * a.sel_stride + j] = s_pos[j];

  // ---- softmax over the selected tokens (log2 domain, FP32) ----
  const __half *qh = a.q + ((size_t)b * a.hq + hh) * kDim;
  float qa = tid < kDim ? fabsf(__half2float(qh[tid])) : 0.f;
  const float amax = cta_reduce<kT>(qa, s_red, tid, true);
  const float coef = (amax / 32767.f) * fabsf(a.qk_scale);  // keys carry the sign of the scale
  float zmax = -INFINITY;
  for (int j = tid; j < ns; j += kTopkThreads) {
    const int pos = s_pos[j];
    const int phys = a.block_table[(size_t)b * a.max_blocks + (pos >> a.bshift)];
    const bool okp = phys >= 0 && phys < a.num_phys;
    const float z = keys[pos] * coef;
    s_p[j] = z;
    // the sub-block pair holding pos
    s_vt[j] = okp ? (((phys * a.hkv + h) << a.lsub) + ((pos & ((1 << a.bshift) - 1)) >> 6)) : -1;
    s_sv[j] = okp ? a.scales[((size_t)phys * a.hkv + h) * 2 + 1] : 0.f;
    zmax = fmaxf(zmax, z);
  }
  const float m = cta_reduce<kT>(zmax, s_red, tid, true);
  float lsum = 0.f;
  for (int j = tid; j < ns; j += kTopkThreads) {
    const float p = exp2f(s_p[j] - m);
    s_p[j] = p;
    lsum += p;
  }
  const float l = cta_reduce<kT>(lsum, s_red, tid, false);

  // ---- P.V over the selected tokens' INT4 V codes (channel c, kParts slices of the list) ----
  const int c = tid & (kDim - 1), part = tid >> 7;
  float acc = 0.f;
  for (int j = part; j < ns; j += kParts) {
    const int vt = s_vt[j];
    if (vt < 0) continue;
    const int slot = s_pos[j] & ((1 << a.bshift) - 1) & (kBlock - 1);
    const uint8_t *vtile = a.cold + (size_t)vt * kTilePairBytes + kTileBytes;
    const uint8_t byte =
        vtile[c * 32 + 8 * ((slot >> 4) ^ ((c >> 2) & 3)) + ((slot & 15) >> 3) * 4 + (slot & 3)];
    const int code = sext4((slot & 4) ? (byte >> 4) : (byte & 0xfu));
    acc = fmaf(s_p[j] * s_sv[j], static_cast<float>(code), acc);
  }
  s_acc[part][c] = acc;
  __syncthreads();
  if (part == 0) {
#pragma unroll
    for (int t = 1; t < kParts; t++) acc += s_acc[t][c];
    // merge with the dense pass (its output and natural-log log-sum-exp)
    const size_t row = (size_t)b * a.hq + hh;
    const float o_s = acc / l;
    const float lse_s = (m + log2f(l)) * kLn2f;
    const float lse_d = a.lse[row];
    const float o_d = __half2float(a.out[row * kDim + c]);
    const float M = fmaxf(lse_d, lse_s);
    const float wd = lse_d == -INFINITY ? 0.f : expf(lse_d - M);
    const float ws = expf(lse_s - M);
    a.out[row * kDim + c] = __float2half_rn((wd * o_d + ws * o_s) / (wd + ws));
    if (c == 0) a.lse[row] = M + logf(wd + ws);
  }
}

cudaError_t launch_sparse_l2(const SparseArgs &a, int batch, cudaStream_t stream) {
  if (a.max_l2 <= 0 || a.top_k <= 0) return cudaSuccess;
  const int St = min(kBlock, 1 << a.bshift);
  const int max_nb = (a.max_l2 + St - 1) / St;
  dim3 g1((max_nb + a.blocks_per_cta - 1) / a.blocks_per_cta, a.hkv, batch);
  l2_score_kernel<<<g1, kScoreThreads, 0, stream>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  dim3 g2(a.hq, batch);
  if (a.max_l2 >= 32768)
    l2_topk_kernel<1024><<<g2, 1024, 0, stream>>>(a);
  else
    l2_topk_kernel<256><<<g2, 256, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace hyb
