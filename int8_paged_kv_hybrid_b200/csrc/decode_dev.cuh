// decode_dev.cuh -- device building blocks of the decode kernel
// (decode.cu): the per-item arithmetic on a staged cold block or hot ring, the fused
// append of the decode step, the merge of the four warps' softmax states and
// the log-sum-exp merge of partial results.  The arithmetic is described at
// the top of decode.cu.
#pragma once

#include <cfloat>

#include "kernels.cuh"

namespace hyb {

constexpr int kWarps = 4;
constexpr int kThreads = 32 * kWarps;
constexpr int kStages = 3;
constexpr long long kWaitCycles = 1ll << 31;  // ~1 s at B200 clocks
constexpr float kLn2 = 0.69314718055994531f;

template <int G>
__host__ __device__ constexpr int pow2_heads() {
  return G <= 1 ? 1 : (G <= 2 ? 2 : (G <= 4 ? 4 : 8));
}

// 2^x on the SFU (max relative error ~2^-22); 2^-inf = +0.
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Sum P per-lane values over the 8 lanes of a lane octet.  Lane l holds its
// values in the order head = k ^ x(l) (see head_xor); at each level a lane
// keeps its lower half and adds the partner's upper half, which (because the
// partner's order differs in exactly that bit) holds the same heads.  On
// return v[0] is the octet total for head x(l).
template <int P, typename T>
__device__ __forceinline__ void transpose_reduce(T (&v)[P]) {
  int c = P;
#pragma unroll
  for (int m = 4; m >= 1; m >>= 1) {
    if (c > 1) {
#pragma unroll
      for (int k = 0; k < c / 2; k++) v[k] += __shfl_xor_sync(0xffffffffu, v[k + c / 2], m);
      c /= 2;
    } else {
      v[0] += __shfl_xor_sync(0xffffffffu, v[0], m);
    }
  }
}

// Head order of a lane: value k of the lane is head k ^ head_xor(lane).
template <int P>
__device__ __forceinline__ int head_xor(int lane) {
  if constexpr (P == 8) return lane & 7;
  if constexpr (P == 4) return (lane >> 1) & 3;
  if constexpr (P == 2) return (lane >> 2) & 1;
  return 0;
}

// Barrier over all threads of all CTAs of the cluster (release / acquire).
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile(
      "barrier.cluster.arrive.release.aligned;\n\t"
      "barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Load a float from the shared memory of CTA `rank` of this cluster, at the
// offset `local` has in this CTA's shared memory.
__device__ __forceinline__ float ld_cluster_f32(const float *local, int rank) {
  uint32_t remote;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(smem_addr(local)), "r"(rank));
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(remote) : "memory");
  return v;
}

__device__ __forceinline__ void unpack_int4(uint32_t x, uint32_t &lo, uint32_t &hi) {
  lo = sext_nibbles(x & 0x0f0f0f0fu);
  hi = sext_nibbles((x >> 4) & 0x0f0f0f0fu);
}

// Scratch of the fused append in shared memory.
struct SealScratch {
  int8_t rqt[2][256];  // re-quantization tables of the tail block (K, V)
  float seal_s[2];     // the tail block's scales after sealing
  int seal_rq[2];      // 1 if the tail block's codes were re-quantized
  alignas(16) __half erow[2 * kDim];  // the evicted token: K row, V row (FP16)
};

// Fused decode step, seal half: the token leaving the hot zone (position e =
// L_old - hot, its FP16 rows in ss.erow) is quantized into its slot of the
// tail block (slot e % block of the block: slot e % 64 of sub-block
// (e % block) / 64), inside the staged copy of that sub-block (tile_st,
// scales *scl_tail, so that this attention sees it) and in the cache
// (tile_tail = physical block * Hkv + kv head).  A grown scale re-quantizes
// the staged sub-block here and an earlier sub-block of the block in
// requant_staged.  Same arithmetic as
// hyb_kv_append: absmax scale, a grown scale re-quantizes the codes already
// in the block, RNE codes.  Called by the whole CTA.
__device__ __forceinline__ void fused_seal(SealScratch &ss, uint8_t *tile_st, float2 *scl_tail, int tile_tail,
                                           bool int4_tail, const DecodeArgs &a, int L_old, bool do_seal, int tid,
                                           int warp, int lane) {
  // A tail block the block table does not give (entry < 0 or past the pool;
  // HYB_STATUS_BAD_BLOCK is set when the entry is read): the evicted token is
  // not sealed and nothing is written through the tile, as hyb_kv_append
  // skips such a block.
  do_seal = do_seal && tile_tail >= 0;
  if (!do_seal) return;
  const int e = L_old - a.hot_tokens;  // position sealed
  const int slot_b = e & ((1 << a.bshift) - 1);  // its slot in the block
  const int slot = slot_b & (kBlock - 1);     // ... and in its sub-block
  const bool int4 = int4_tail;
  const int Q = int4 ? 7 : 127;
  if (warp < 2) {
    // warp 0: K, warp 1: V -- absmax of the evicted token, new scale
    const int kv = warp;
    const __half *row = ss.erow + kv * kDim;
    float amax = 0.f;
#pragma unroll
    for (int j = 0; j < 4; j++) amax = fmaxf(amax, fabsf(__half2float(row[4 * lane + j])));
#pragma unroll
    for (int m = 16; m > 0; m >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, m));
    const float s_c = __fdiv_rn(amax, static_cast<float>(Q));
    const float s_old = kv ? scl_tail->y : scl_tail->x;
    float s_new = s_c;
    int rq = 0;
    if (slot_b != 0) {
      if (s_c > s_old) rq = 1;
      else s_new = s_old;
    }
    if (rq)
      for (int c = lane - 127; c <= 127; c += 32)
        ss.rqt[kv][c + 127] = static_cast<int8_t>(requantize(c, s_old, s_new, Q));
    if (lane == 0) {
      ss.seal_s[kv] = s_new;
      ss.seal_rq[kv] = rq;
    }
  }
  __syncthreads();
  if (tid == 0) *scl_tail = make_float2(ss.seal_s[0], ss.seal_s[1]);  // attention uses these
  // codes already in the tail block, under a grown scale
#pragma unroll
  for (int kv = 0; kv < 2; kv++) {
    if (!ss.seal_rq[kv]) continue;
    uint32_t *w32 = reinterpret_cast<uint32_t *>(tile_st + kv * kTileBytes);
    const int nw = requant_nwords(kv, int4, slot);
    for (int w = tid; w < nw; w += kThreads) w32[w] = requant_word(w32[w], w, kv, int4, slot, ss.rqt[kv]);
  }
  __syncthreads();
  const int c = tid;  // channel
  {
    // the evicted token's codes into slot `slot`
    const int ck = quantize(__half2float(ss.erow[c]), ss.seal_s[0], Q);
    const int cv = quantize(__half2float(ss.erow[kDim + c]), ss.seal_s[1], Q);
    if (!int4) {
      tile_st[slot * kDim + c] = static_cast<uint8_t>(ck);
      tile_st[kTileBytes + c * 64 + 16 * ((slot >> 4) ^ ((c >> 1) & 3)) + (slot & 15)] = static_cast<uint8_t>(cv);
    } else {
      // K: channels c and c+4 of an 8-channel group share a byte; the thread of
      // the lower one writes both (its partner's code comes by shuffle)
      const int ck_hi = __shfl_down_sync(0xffffffffu, ck, 4);
      if ((c & 4) == 0) {
        uint8_t *byte = tile_st + slot * 64 + 4 * (c >> 3) + (c & 3);
        *byte = static_cast<uint8_t>((ck & 0xf) | ((ck_hi & 0xf) << 4));
      }
      const int unit = (slot >> 4) ^ ((c >> 2) & 3);
      const int in = slot & 15;
      uint8_t *byte = tile_st + kTileBytes + c * 32 + unit * 8 + (in >> 3) * 4 + (in & 3);
      *byte = (in & 4) ? static_cast<uint8_t>((*byte & 0x0f) | ((cv & 0xf) << 4))
                       : static_cast<uint8_t>((*byte & 0xf0) | (cv & 0xf));
    }
  }
  __syncthreads();
  {
    // write back what changed in the tail block: scales, then the whole tile
    // if its codes were re-quantized, else the sealed token's codes
    uint8_t *gtile = a.cold + ((static_cast<size_t>(tile_tail) << a.lsub) + (slot_b >> 6)) * kTilePairBytes;
    if (tid < 2) a.scales[(size_t)tile_tail * 2 + tid] = ss.seal_s[tid];
#pragma unroll
    for (int kv = 0; kv < 2; kv++) {
      uint8_t *g = gtile + kv * kTileBytes;
      const uint8_t *t = tile_st + kv * kTileBytes;
      if (ss.seal_rq[kv]) {
        // the bytes the block's codes occupy: K rows of its slots only (a
        // 32-token block stages and owns the first half of a K tile), the
        // whole V tile
        const int st_tok = min(kBlock, 1 << a.bshift);
        const int kbytes = (int4 ? 64 : kDim) * st_tok;
        const int nvec = (kv == 0 ? kbytes : (int4 ? kTileBytes / 2 : kTileBytes)) / 16;
        for (int v = tid; v < nvec; v += kThreads)
          reinterpret_cast<uint4 *>(g)[v] = reinterpret_cast<const uint4 *>(t)[v];
      } else if (kv == 0) {
        const int rowb = int4 ? 64 : kDim;
        if (tid * 16 < rowb)
          reinterpret_cast<uint4 *>(g + slot * rowb)[tid] = reinterpret_cast<const uint4 *>(t + slot * rowb)[tid];
      } else {
        const int off = !int4 ? c * 64 + 16 * ((slot >> 4) ^ ((c >> 1) & 3)) + (slot & 15)
                              : c * 32 + 8 * ((slot >> 4) ^ ((c >> 2) & 3)) + ((slot & 15) >> 3) * 4 + (slot & 3);
        g[off] = t[off];
      }
    }
  }
  __syncthreads();
}

// Fused decode step, seal half for FP16 cold blocks (quantization_bits 0):
// the evicted token's rows (ss.erow) move unchanged to slot e % 64 of the
// tail block -- in its staged half-block item (row_st, rows slot % 32) and in
// the cache.  Thread tid moves channel tid of both rows.
__device__ __forceinline__ void fused_seal_fp16(const SealScratch &ss, uint8_t *row_st, int tile_tail,
                                                const DecodeArgs &a, int L_old, bool do_seal, int tid) {
  if (!do_seal || tile_tail < 0) return;
  const int slot = (L_old - a.hot_tokens) & ((1 << a.bshift) - 1);
  const int c = tid;
  const __half k_old = ss.erow[c], v_old = ss.erow[kDim + c];
  __half *trow = reinterpret_cast<__half *>(row_st + (slot % kItemRows) * kHotTokenBytes);
  trow[c] = k_old;
  trow[kDim + c] = v_old;
  __half *grow = reinterpret_cast<__half *>(a.cold + ((size_t)tile_tail << a.bshift) * kHotTokenBytes +
                                            slot * kHotTokenBytes);
  grow[c] = k_old;
  grow[kDim + c] = v_old;
  __syncthreads();
}

// Fused decode step, 128-token blocks: the seal landed in the block's second
// sub-block and grew the block's scale -- the first sub-block's codes (all 64
// slots, staged in tile_st) are re-quantized with the seal's tables, for this
// attention and in the cache (sub-block pair index pair0 = (physical block *
// Hkv + kv head) * 2).  Called by the whole CTA after fused_seal.
__device__ __forceinline__ void requant_staged(const SealScratch &ss, uint8_t *tile_st, int pair0, bool int4,
                                               const DecodeArgs &a, int tid) {
#pragma unroll
  for (int kv = 0; kv < 2; kv++) {
    if (!ss.seal_rq[kv]) continue;
    uint32_t *w32 = reinterpret_cast<uint32_t *>(tile_st + kv * kTileBytes);
    const int nw = requant_nwords(kv, int4, kBlock);
    for (int w = tid; w < nw; w += kThreads) w32[w] = requant_word(w32[w], w, kv, int4, kBlock, ss.rqt[kv]);
  }
  __syncthreads();
  uint8_t *g = a.cold + (size_t)pair0 * kTilePairBytes;
#pragma unroll
  for (int kv = 0; kv < 2; kv++) {
    if (!ss.seal_rq[kv]) continue;
    const int nvec = (int4 ? kTileBytes / 2 : kTileBytes) / 16;
    for (int v = tid; v < nvec; v += kThreads)
      reinterpret_cast<uint4 *>(g + kv * kTileBytes)[v] = reinterpret_cast<const uint4 *>(tile_st + kv * kTileBytes)[v];
  }
  __syncthreads();
}

// Fused decode step, ring half: the new token goes to ring slot rs = L_old %
// hot -- row rs % 32 of its staged hot item (item_st, for this attention) and
// the cache.  Thread tid writes channel tid of both rows.
__device__ __forceinline__ void ring_put(uint8_t *item_st, int rs, __half2 new_kv, const DecodeArgs &a, int b,
                                         int h, int tid) {
  const int c = tid;
  __half *srow = reinterpret_cast<__half *>(item_st + (rs % kItemRows) * kHotTokenBytes);
  srow[c] = __low2half(new_kv);
  srow[kDim + c] = __high2half(new_kv);
  __half *grow = reinterpret_cast<__half *>(a.hot) + ((((size_t)b * a.hkv + h) * a.hot_tokens + rs) * 2) * kDim;
  grow[c] = __low2half(new_kv);
  grow[kDim + c] = __high2half(new_kv);
  __syncthreads();
}

// Raise a warp's running max to cover an item's logits, whose maximum over a
// lane's tokens is zmax (lane's head hx): m_run per head, the accumulators
// and the lane's denominator (l_lane + psum_lane / 32767) are rescaled.
// Warp-uniform call; rare once the first blocks are seen.
template <int G, int P>
__device__ __forceinline__ void raise_max(float zmax, float (&m_run)[G], float (&acc)[G][4], float &m_hx,
                                          float &l_lane, int &psum_lane, int hx) {
  float mb = zmax;
  mb = fmaxf(mb, __shfl_xor_sync(0xffffffffu, mb, 8));
  mb = fmaxf(mb, __shfl_xor_sync(0xffffffffu, mb, 16));
  float alpha_hx = 1.f;
#pragma unroll
  for (int hh = 0; hh < G; hh++) {
    const float mbh = __shfl_sync(0xffffffffu, mb, hh * (8 / P));  // a lane holding head hh
    if (mbh > m_run[hh]) {
      const float alpha = ex2(m_run[hh] - mbh);
#pragma unroll
      for (int kk = 0; kk < 4; kk++) acc[hh][kk] *= alpha;
      if (hh == hx) alpha_hx = alpha;
      m_run[hh] = mbh;
    }
    if (hh == hx) m_hx = m_run[hh];
  }
  if (alpha_hx != 1.f) {
    l_lane = (l_lane + static_cast<float>(psum_lane) * (1.f / 32767.f)) * alpha_hx;
    psum_lane = 0;
  }
}

// Log-sum-exp merge of n partial results of the G query heads of one kv head
// (read from global memory through L2).  Partial j is entry slot_of(j) of an
// array of partials: head hh's 128 FP32 at o + slot * o_js + hh * o_hs, its
// log2-sum-exp at lse + slot * l_js + hh * l_hs (-inf: empty, output 0).
// Warp w merges heads w, w + 4, ...; lane l channels 4l..4l+3; the loads of
// kMergeFan partials are issued together.  Writes the FP16 output rows
// [G][128] at out (and the natural-log lse at lse_out), or, when out is null,
// the merged FP32 rows at p_o (head stride p_hs floats) with their
// log2-sum-exp at p_lse (head stride p_lhs).
template <int G, typename SlotOf>
__device__ __forceinline__ void merge_splits(const float *o, size_t o_js, size_t o_hs, const float *lse, size_t l_js,
                                             size_t l_hs, int n, SlotOf slot_of, int warp, int lane, __half *out,
                                             float *lse_out, float *p_o, size_t p_hs, float *p_lse, size_t p_lhs) {
  for (int hh = warp; hh < G; hh += kWarps) {
    float m = -INFINITY, den = 0.f;
    float4 num = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int j0 = 0; j0 < n; j0 += kMergeFan) {
      const int nj = min(kMergeFan, n - j0);
      const long long my_slot = lane < nj ? static_cast<long long>(slot_of(j0 + lane)) : 0;
      float4 ov[kMergeFan];
#pragma unroll
      for (int j = 0; j < kMergeFan; j++) {
        const long long sj = __shfl_sync(0xffffffffu, my_slot, j);
        ov[j] = j < nj ? __ldcg(reinterpret_cast<const float4 *>(o + sj * o_js + hh * o_hs + 4 * lane))
                       : make_float4(0.f, 0.f, 0.f, 0.f);
      }
      const float lj = lane < nj ? __ldcg(lse + my_slot * l_js + hh * l_hs) : -INFINITY;
      float mr = lj;
#pragma unroll
      for (int d = 16; d > 0; d >>= 1) mr = fmaxf(mr, __shfl_xor_sync(0xffffffffu, mr, d));
      const float mn = fmaxf(m, mr);
      if (mn == -INFINITY) continue;  // nothing but empty partials so far
      const float sc = ex2(m - mn);
      num.x *= sc; num.y *= sc; num.z *= sc; num.w *= sc;
      den *= sc;
      m = mn;
      const float wl = ex2(lj - m);  // lane j's weight (0 for an empty partial)
      float ws = wl;
#pragma unroll
      for (int d = 16; d > 0; d >>= 1) ws += __shfl_xor_sync(0xffffffffu, ws, d);
      den += ws;
#pragma unroll
      for (int j = 0; j < kMergeFan; j++) {
        const float wj = __shfl_sync(0xffffffffu, wl, j);
        num.x = fmaf(wj, ov[j].x, num.x);
        num.y = fmaf(wj, ov[j].y, num.y);
        num.z = fmaf(wj, ov[j].z, num.z);
        num.w = fmaf(wj, ov[j].w, num.w);
      }
    }
    const float inv = den > 0.f ? 1.f / den : 0.f;
    const float lse2 = den > 0.f ? m + log2f(den) : -INFINITY;
    if (out) {
      __half2 h01 = __floats2half2_rn(num.x * inv, num.y * inv);
      __half2 h23 = __floats2half2_rn(num.z * inv, num.w * inv);
      uint2 pk;
      pk.x = *reinterpret_cast<uint32_t *>(&h01);
      pk.y = *reinterpret_cast<uint32_t *>(&h23);
      *reinterpret_cast<uint2 *>(out + hh * kDim + 4 * lane) = pk;
      if (lane == 0 && lse_out) lse_out[hh] = lse2 * kLn2;
    } else {
      *reinterpret_cast<float4 *>(p_o + hh * p_hs + 4 * lane) =
          make_float4(num.x * inv, num.y * inv, num.z * inv, num.w * inv);
      if (lane == 0) p_lse[hh * p_lhs] = lse2;
    }
  }
}

// q of one kv head's G query heads in 16-bit fixed point per head: warp w
// quantizes heads w, w + 4, ... of qf (FP32 [P][128], rows >= G zero) into qi
// and the step max|q| / 32767 into sq.  Callers synchronise around it.
template <int P>
__device__ __forceinline__ void quantize_q(const float (*qf)[kDim], int16_t (*qi)[kDim], float *sq, int warp,
                                           int lane) {
  for (int j = warp; j < P; j += kWarps) {
    float amax = 0.f;
    for (int c = lane; c < kDim; c += 32) amax = fmaxf(amax, fabsf(qf[j][c]));
#pragma unroll
    for (int m = 16; m > 0; m >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, m));
    const float inv = amax > 0.f ? 32767.f / amax : 0.f;
    for (int c = lane; c < kDim; c += 32) {
      const int v = __float2int_rn(qf[j][c] * inv);
      qi[j][c] = static_cast<int16_t>(max(-32767, min(32767, v)));
    }
    if (lane == 0) sq[j] = amax > 0.f ? amax / 32767.f : 0.f;
  }
}

// The lane's q pairs: its 16 channels (16cs..16cs+15) of every head, in the
// lane's head order (value k is head k ^ hx).
template <int P>
__device__ __forceinline__ void load_qp(const int16_t (*qi)[kDim], int hx, int cs, uint32_t (&qp)[P][8]) {
#pragma unroll
  for (int k = 0; k < P; k++) {
    const uint4 *src = reinterpret_cast<const uint4 *>(&qi[k ^ hx][16 * cs]);
    const uint4 x0 = src[0], x1 = src[1];
    qp[k][0] = x0.x; qp[k][1] = x0.y; qp[k][2] = x0.z; qp[k][3] = x0.w;
    qp[k][4] = x1.x; qp[k][5] = x1.y; qp[k][6] = x1.z; qp[k][7] = x1.w;
  }
}

// One full INT8 cold block (all 64 tokens valid), for one warp.  The warp's
// tokens are 16w..16w+15; lane (tg, cs) takes tokens 16w + 4tg + step, step
// 0..3 (channels 16cs..16cs+15), so the four weight codes an owner lane
// produces for its head are adjacent and leave in one 8-byte store.  k_lane
// and v_lane are the lane's byte offsets of its K row (step 0) and of its V
// words inside a stage; pc is this warp's weight-code rows.  Same arithmetic
// as the general path; no masks, no INT4 branches, offsets fixed per lane.
template <int G, int P>
__device__ __forceinline__ void cold_block_full(const uint8_t *stage, int k_lane, int v_lane,
                                                const uint32_t (&qp)[P][8], float coef, float cv,
                                                uint16_t (*pc_rows)[16], int hx, int tg, bool owner,
                                                float (&m_run)[G], float (&acc)[G][4], float &m_hx,
                                                float &l_lane, int &psum_lane) {
  float z[4];
#pragma unroll
  for (int step = 0; step < 4; step++) {
    const uint4 v = *reinterpret_cast<const uint4 *>(stage + k_lane + step * kDim);
    const uint32_t kw[4] = {v.x, v.y, v.z, v.w};
    int dot[P];
#pragma unroll
    for (int kk = 0; kk < P; kk++) dot[kk] = 0;
#pragma unroll
    for (int j = 0; j < 4; j++) {
#pragma unroll
      for (int kk = 0; kk < P; kk++)
        dot[kk] = __dp2a_lo(static_cast<int>(qp[kk][2 * j]), static_cast<int>(kw[j]), dot[kk]);
#pragma unroll
      for (int kk = 0; kk < P; kk++)
        dot[kk] = __dp2a_hi(static_cast<int>(qp[kk][2 * j + 1]), static_cast<int>(kw[j]), dot[kk]);
    }
    transpose_reduce<P>(dot);
    z[step] = static_cast<float>(dot[0]) * coef;
  }
  {
    const float zmax = fmaxf(fmaxf(z[0], z[1]), fmaxf(z[2], z[3]));
    if (__any_sync(0xffffffffu, zmax > m_hx)) raise_max<G, P>(zmax, m_run, acc, m_hx, l_lane, psum_lane, hx);
  }
  uint32_t pc[4];
#pragma unroll
  for (int step = 0; step < 4; step++) {
    const float pq = fmaf(ex2(z[step] - m_hx), 32767.f, 12582912.f);
    pc[step] = __float_as_uint(pq) - 0x4B400000u;
    psum_lane += static_cast<int>(pc[step]);
  }
  if (owner)
    *reinterpret_cast<uint2 *>(&pc_rows[hx][4 * tg]) = make_uint2(pc[0] | (pc[1] << 16), pc[2] | (pc[3] << 16));
  __syncwarp();
  uint32_t vw[4][4];
#pragma unroll
  for (int kk = 0; kk < 4; kk++) {
    const uint4 v = *reinterpret_cast<const uint4 *>(stage + v_lane + 32 * kBlock * kk);
    vw[kk][0] = v.x; vw[kk][1] = v.y; vw[kk][2] = v.z; vw[kk][3] = v.w;
  }
#pragma unroll
  for (int hh = 0; hh < G; hh++) {
    const uint4 pa = *reinterpret_cast<const uint4 *>(&pc_rows[hh][0]);
    const uint4 pb = *reinterpret_cast<const uint4 *>(&pc_rows[hh][8]);
    const uint32_t pp[8] = {pa.x, pa.y, pa.z, pa.w, pb.x, pb.y, pb.z, pb.w};
    int ai[4] = {0, 0, 0, 0};
#pragma unroll
    for (int j = 0; j < 4; j++) {
#pragma unroll
      for (int kk = 0; kk < 4; kk++) {
        ai[kk] = __dp2a_lo(static_cast<int>(pp[2 * j]), static_cast<int>(vw[kk][j]), ai[kk]);
        ai[kk] = __dp2a_hi(static_cast<int>(pp[2 * j + 1]), static_cast<int>(vw[kk][j]), ai[kk]);
      }
    }
#pragma unroll
    for (int kk = 0; kk < 4; kk++) acc[hh][kk] = fmaf(cv, static_cast<float>(ai[kk]), acc[hh][kk]);
  }
}

// A cold block that is INT4 or not full (nv = valid tokens from this warp's
// first one), for one warp: lane (tg, cs) takes tokens 16w + 4step + tg.
// Same arithmetic as cold_block_full.
template <int G, int P>
__device__ __forceinline__ void cold_block_general(const uint8_t *stage, int nv, bool int4, int warp, int lane,
                                                   int tg, int cs, const uint32_t (&qp)[P][8], float coef,
                                                   float cv, uint16_t (*pc_rows)[16], int hx, bool owner,
                                                   float (&m_run)[G], float (&acc)[G][4], float &m_hx,
                                                   float &l_lane, int &psum_lane) {
  float z[4];
#pragma unroll
  for (int step = 0; step < 4; step++) {
    const int t = 16 * warp + 4 * step + tg;
    uint32_t kw[4];
    if (!int4) {
      const uint4 v = *reinterpret_cast<const uint4 *>(stage + t * kDim + 16 * cs);
      kw[0] = v.x; kw[1] = v.y; kw[2] = v.z; kw[3] = v.w;
    } else {
      const uint2 v = *reinterpret_cast<const uint2 *>(stage + t * 64 + 8 * cs);
      unpack_int4(v.x, kw[0], kw[1]);
      unpack_int4(v.y, kw[2], kw[3]);
    }
    int dot[P];
#pragma unroll
    for (int kk = 0; kk < P; kk++) dot[kk] = 0;
#pragma unroll
    for (int j = 0; j < 4; j++) {
#pragma unroll
      for (int kk = 0; kk < P; kk++)
        dot[kk] = __dp2a_lo(static_cast<int>(qp[kk][2 * j]), static_cast<int>(kw[j]), dot[kk]);
#pragma unroll
      for (int kk = 0; kk < P; kk++)
        dot[kk] = __dp2a_hi(static_cast<int>(qp[kk][2 * j + 1]), static_cast<int>(kw[j]), dot[kk]);
    }
    transpose_reduce<P>(dot);
    z[step] = (4 * step + tg < nv) ? static_cast<float>(dot[0]) * coef : -INFINITY;
  }
  // the running max must cover these logits (rare after the first blocks)
  {
    const float zmax = fmaxf(fmaxf(z[0], z[1]), fmaxf(z[2], z[3]));
    if (__any_sync(0xffffffffu, zmax > m_hx)) raise_max<G, P>(zmax, m_run, acc, m_hx, l_lane, psum_lane, hx);
  }
  // 16-bit weights relative to the running max: round(32767 * 2^(z - m))
  // via the 1.5*2^23 magic add
  uint32_t pc[4];
#pragma unroll
  for (int step = 0; step < 4; step++) {
    const float pq = fmaf(ex2(z[step] - m_hx), 32767.f, 12582912.f);
    pc[step] = __float_as_uint(pq) - 0x4B400000u;
    psum_lane += static_cast<int>(pc[step]);
  }
  if (owner) {
#pragma unroll
    for (int step = 0; step < 4; step++)
      pc_rows[hx][4 * step + tg] = static_cast<uint16_t>(pc[step]);
  }
  __syncwarp();
  // P.V over this warp's 16 tokens; lane owns channels lane + 32*kk
  uint32_t vw[4][4];
#pragma unroll
  for (int kk = 0; kk < 4; kk++) {
    const int c = lane + 32 * kk;
    if (!int4) {
      const uint4 v = *reinterpret_cast<const uint4 *>(
          stage + kTileBytes + c * 64 + 16 * (warp ^ ((c >> 1) & 3)));
      vw[kk][0] = v.x; vw[kk][1] = v.y; vw[kk][2] = v.z; vw[kk][3] = v.w;
    } else {
      const uint2 v = *reinterpret_cast<const uint2 *>(
          stage + kTileBytes + c * 32 + 8 * (warp ^ ((c >> 2) & 3)));
      unpack_int4(v.x, vw[kk][0], vw[kk][1]);
      unpack_int4(v.y, vw[kk][2], vw[kk][3]);
    }
  }
#pragma unroll
  for (int hh = 0; hh < G; hh++) {
    // p codes of this warp's 16 tokens, as 16-bit pairs (tokens 2i, 2i+1)
    const uint4 pa = *reinterpret_cast<const uint4 *>(&pc_rows[hh][0]);
    const uint4 pb = *reinterpret_cast<const uint4 *>(&pc_rows[hh][8]);
    const uint32_t pp[8] = {pa.x, pa.y, pa.z, pa.w, pb.x, pb.y, pb.z, pb.w};
    int ai[4] = {0, 0, 0, 0};
#pragma unroll
    for (int j = 0; j < 4; j++) {
#pragma unroll
      for (int kk = 0; kk < 4; kk++) {
        ai[kk] = __dp2a_lo(static_cast<int>(pp[2 * j]), static_cast<int>(vw[kk][j]), ai[kk]);
        ai[kk] = __dp2a_hi(static_cast<int>(pp[2 * j + 1]), static_cast<int>(vw[kk][j]), ai[kk]);
      }
    }
#pragma unroll
    for (int kk = 0; kk < 4; kk++) acc[hh][kk] = fmaf(cv, static_cast<float>(ai[kk]), acc[hh][kk]);
  }
}

// The hot ring (nhot FP16 tokens, K and V interleaved per token), for one
// warp: tokens 8w..8w+7, FP32 arithmetic on the FP16 values with q in FP32
// (qf [P][128]); weights go through ph_rows ([G][8], this warp's).
template <int G, int P>
__device__ __forceinline__ void hot_item(const uint8_t *stage, int nhot, int warp, int lane, int tg, int cs,
                                         const float (*qf)[kDim], float qk_scale, float (*ph_rows)[8], int hx,
                                         bool owner, float (&m_run)[G], float (&acc)[G][4], float &m_hx,
                                         float &l_lane, int &psum_lane) {
  const int nv = nhot - 8 * warp;
  if (nv > 0) {
    float z[2];
#pragma unroll
    for (int step = 0; step < 2; step++) {
      const int t = 8 * warp + 4 * step + tg;
      const uint4 *kp = reinterpret_cast<const uint4 *>(stage + t * kHotTokenBytes + 32 * cs);
      const uint4 k0 = kp[0], k1 = kp[1];
      const uint32_t kr[8] = {k0.x, k0.y, k0.z, k0.w, k1.x, k1.y, k1.z, k1.w};
      float kf[16];
#pragma unroll
      for (int j = 0; j < 8; j++) {
        const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&kr[j]));
        kf[2 * j] = f.x;
        kf[2 * j + 1] = f.y;
      }
      float dot[P];
#pragma unroll
      for (int kk = 0; kk < P; kk++) {
        const float4 *qv4 = reinterpret_cast<const float4 *>(&qf[kk ^ hx][16 * cs]);
        float d = 0.f;
#pragma unroll
        for (int j = 0; j < 4; j++) {
          const float4 qq = qv4[j];
          d = fmaf(qq.x, kf[4 * j], d);
          d = fmaf(qq.y, kf[4 * j + 1], d);
          d = fmaf(qq.z, kf[4 * j + 2], d);
          d = fmaf(qq.w, kf[4 * j + 3], d);
        }
        dot[kk] = d;
      }
      transpose_reduce<P>(dot);
      z[step] = (4 * step + tg < nv) ? dot[0] * qk_scale : -INFINITY;
    }
    {
      const float zmax = fmaxf(z[0], z[1]);
      if (__any_sync(0xffffffffu, zmax > m_hx)) raise_max<G, P>(zmax, m_run, acc, m_hx, l_lane, psum_lane, hx);
    }
    float pv[2];
#pragma unroll
    for (int step = 0; step < 2; step++) {
      pv[step] = ex2(z[step] - m_hx);
      l_lane += pv[step];
    }
    if (owner) {
      ph_rows[hx][tg] = pv[0];
      ph_rows[hx][4 + tg] = pv[1];
    }
    __syncwarp();
    float ah[G][4];
#pragma unroll
    for (int hh = 0; hh < G; hh++)
#pragma unroll
      for (int kk = 0; kk < 4; kk++) ah[hh][kk] = 0.f;
    const int ntok = min(nv, 8);
    for (int tt = 0; tt < ntok; tt++) {
      const __half *vrow =
          reinterpret_cast<const __half *>(stage + (8 * warp + tt) * kHotTokenBytes) + kDim;
      float v[4];
#pragma unroll
      for (int kk = 0; kk < 4; kk++) v[kk] = __half2float(vrow[lane + 32 * kk]);
#pragma unroll
      for (int hh = 0; hh < G; hh++) {
        const float p = ph_rows[hh][tt];
#pragma unroll
        for (int kk = 0; kk < 4; kk++) ah[hh][kk] = fmaf(p, v[kk], ah[hh][kk]);
      }
    }
#pragma unroll
    for (int hh = 0; hh < G; hh++)
#pragma unroll
      for (int kk = 0; kk < 4; kk++) acc[hh][kk] += ah[hh][kk];
  }
}

// End of a split: the four warps' online-softmax states merged into the
// split's normalised output for channel tid (o_s per head) and its
// log2-sum-exp per head (-inf and 0 when empty).  mbuf: FP32 [kWarps][G][128]
// and mrun / lrun [kWarps][G] in shared memory.  Two CTA barriers; on return
// mbuf may be reused.
template <int G, int P>
__device__ __forceinline__ void merge_warps(float *mbuf, float (*mrun)[G], float (*lrun)[G], const float (&m_run)[G],
                                            const float (&acc)[G][4], float l_lane, int psum_lane, int warp,
                                            int lane, int tid, float (&o_s)[G], float (&lse2_s)[G]) {
  // denominators: this lane's partial for head hx, summed over the 4 token
  // groups, then gathered per head from a lane that holds it
  float l_run[G];
  {
    float lt = l_lane + static_cast<float>(psum_lane) * (1.f / 32767.f);
    lt += __shfl_xor_sync(0xffffffffu, lt, 8);
    lt += __shfl_xor_sync(0xffffffffu, lt, 16);
#pragma unroll
    for (int hh = 0; hh < G; hh++) l_run[hh] = __shfl_sync(0xffffffffu, lt, hh * (8 / P));
  }
#pragma unroll
  for (int hh = 0; hh < G; hh++)
#pragma unroll
    for (int kk = 0; kk < 4; kk++) mbuf[(warp * G + hh) * kDim + lane + 32 * kk] = acc[hh][kk];
  if (lane == 0) {
#pragma unroll
    for (int hh = 0; hh < G; hh++) {
      mrun[warp][hh] = m_run[hh];
      lrun[warp][hh] = l_run[hh];
    }
  }
  __syncthreads();
#pragma unroll
  for (int hh = 0; hh < G; hh++) {
    o_s[hh] = 0.f;
    lse2_s[hh] = -INFINITY;
    float mm = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; w++) mm = fmaxf(mm, mrun[w][hh]);
    float num = 0.f, den = 0.f;
    if (mm != -INFINITY) {
#pragma unroll
      for (int w = 0; w < kWarps; w++) {
        const float f = ex2(mrun[w][hh] - mm);
        num = fmaf(f, mbuf[(w * G + hh) * kDim + tid], num);
        den = fmaf(f, lrun[w][hh], den);
      }
    }
    if (den > 0.f) {
      o_s[hh] = num * __frcp_rn(den);
      lse2_s[hh] = mm + __log2f(den);
    }
  }
  __syncthreads();
}

}  // namespace hyb
