// decode_dev.cuh -- device building blocks of the decode kernel
// (decode.cu): the per-item arithmetic on a staged cold block or FP16 rows
// (tensor-core mma.sync), the fused append of the decode step, the merge of
// the four warps' softmax states and the log-sum-exp merge of partial
// results.  The arithmetic is described at the top of decode.cu.
#pragma once

#include <cfloat>

#include "kernels.cuh"
#include "mma.cuh"

namespace hyb {

constexpr int kWarps = 4;
constexpr int kThreads = 32 * kWarps;
constexpr int kStages = 3;
constexpr long long kWaitCycles = kDefaultWaitCycles;  // drain waits (never shortened)
constexpr float kLn2 = 0.69314718055994531f;
// FP16 rows (hot ring, FP16 cold blocks) are staged one 512-byte row per bulk
// copy at this pitch, so that the 8 rows an ldmatrix reads start 16 bytes
// apart modulo 128 (distinct banks).
constexpr int kRowStride = kHotTokenBytes + 16;
constexpr int kStageBytes = kItemRows * kRowStride;  // >= kTilePairBytes
static_assert(kStageBytes >= kTilePairBytes, "a stage holds a K + V tile pair");
// Merge buffer pitch (floats per head row): 136 puts the 32 lanes' stores of
// merge_warps in distinct banks.
constexpr int kMbufPitch = kDim + 8;
// q as a 24-bit fixed-point integer per head: |q_int| <= 127 * 65536, three
// signed base-256 digits (hi, mid, lo), each in [-128, 127].
constexpr float kQFix = 8323072.f;  // 127 * 65536
// softmax weights in 16-bit fixed point relative to their group's maximum
constexpr float kPFix = 65535.f;

// Query-head slots per kv head: one quad of 4 (G <= 4) or two (G <= 8).
template <int G>
__host__ __device__ constexpr int head_quads() {
  return G <= 4 ? 1 : 2;
}

// 2^x on the SFU (max relative error ~2^-22); 2^-inf = +0.
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Barrier of the threads that run the per-item arithmetic: the whole CTA
// (kNamed false), or the 128 consumer threads of a warp-specialized CTA
// (named barrier 1; the producer warp never takes part).
template <bool kNamed>
__device__ __forceinline__ void work_sync() {
  if constexpr (kNamed) asm volatile("bar.sync 1, 128;" ::: "memory");
  else __syncthreads();
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
template <bool kNamed = false>
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
  work_sync<kNamed>();
  if (tid == 0) *scl_tail = make_float2(ss.seal_s[0], ss.seal_s[1]);  // attention uses these
  // codes already in the tail block, under a grown scale
#pragma unroll
  for (int kv = 0; kv < 2; kv++) {
    if (!ss.seal_rq[kv]) continue;
    uint32_t *w32 = reinterpret_cast<uint32_t *>(tile_st + kv * kTileBytes);
    if (kv == 0) {
      // K, token-major: the words of slots < slot lead the tile
      const int nw = requant_nwords(0, int4, slot);
      for (int w = tid; w < nw; w += kThreads) w32[w] = requant_word(w32[w], w, 0, int4, slot, ss.rqt[0]);
    } else {
      // V, channel-major: per channel row only the words of tokens < slot
      // (4 INT8 or 8 INT4 tokens a word, at their swizzled places)
      const int tw = int4 ? 8 : 4;  // tokens per word
      const int per_row = (slot + tw - 1) / tw;
      for (int i = tid; i < kDim * per_row; i += kThreads) {
        const int r = i / per_row, tj = i - r * per_row;
        const int w = int4 ? r * 8 + 2 * ((tj >> 1) ^ ((r >> 2) & 3)) + (tj & 1)
                           : r * 16 + 4 * ((tj >> 2) ^ ((r >> 1) & 3)) + (tj & 3);
        w32[w] = requant_word(w32[w], w, 1, int4, slot, ss.rqt[1]);
      }
    }
  }
  work_sync<kNamed>();
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
  work_sync<kNamed>();
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
  fence_proxy_async_smem();  // the staged tile is refilled by bulk copies later
  work_sync<kNamed>();
}

// Fused decode step, seal half for FP16 cold blocks (quantization_bits 0):
// the evicted token's rows (ss.erow) move unchanged to slot e % 64 of the
// tail block -- in its staged half-block item (row_st, rows slot % 32 at the
// staging pitch kRowStride) and in the cache.  Thread tid moves channel tid of both rows.
template <bool kNamed = false>
__device__ __forceinline__ void fused_seal_fp16(const SealScratch &ss, uint8_t *row_st, int tile_tail,
                                                const DecodeArgs &a, int L_old, bool do_seal, int tid) {
  if (!do_seal || tile_tail < 0) return;
  const int slot = (L_old - a.hot_tokens) & ((1 << a.bshift) - 1);
  const int c = tid;
  const __half k_old = ss.erow[c], v_old = ss.erow[kDim + c];
  __half *trow = reinterpret_cast<__half *>(row_st + (slot % kItemRows) * kRowStride);
  trow[c] = k_old;
  trow[kDim + c] = v_old;
  __half *grow = reinterpret_cast<__half *>(a.cold + ((size_t)tile_tail << a.bshift) * kHotTokenBytes +
                                            slot * kHotTokenBytes);
  grow[c] = k_old;
  grow[kDim + c] = v_old;
  fence_proxy_async_smem();
  work_sync<kNamed>();
}

// Fused decode step, 128-token blocks: the seal landed in the block's second
// sub-block and grew the block's scale -- the first sub-block's codes (all 64
// slots, staged in tile_st) are re-quantized with the seal's tables, for this
// attention and in the cache (sub-block pair index pair0 = (physical block *
// Hkv + kv head) * 2).  Called by the whole CTA after fused_seal.
template <bool kNamed = false>
__device__ __forceinline__ void requant_staged(const SealScratch &ss, uint8_t *tile_st, int pair0, bool int4,
                                               const DecodeArgs &a, int tid) {
#pragma unroll
  for (int kv = 0; kv < 2; kv++) {
    if (!ss.seal_rq[kv]) continue;
    uint32_t *w32 = reinterpret_cast<uint32_t *>(tile_st + kv * kTileBytes);
    const int nw = requant_nwords(kv, int4, kBlock);
    for (int w = tid; w < nw; w += kThreads) w32[w] = requant_word(w32[w], w, kv, int4, kBlock, ss.rqt[kv]);
  }
  work_sync<kNamed>();
  uint8_t *g = a.cold + (size_t)pair0 * kTilePairBytes;
#pragma unroll
  for (int kv = 0; kv < 2; kv++) {
    if (!ss.seal_rq[kv]) continue;
    const int nvec = (int4 ? kTileBytes / 2 : kTileBytes) / 16;
    for (int v = tid; v < nvec; v += kThreads)
      reinterpret_cast<uint4 *>(g + kv * kTileBytes)[v] = reinterpret_cast<const uint4 *>(tile_st + kv * kTileBytes)[v];
  }
  fence_proxy_async_smem();
  work_sync<kNamed>();
}

// Fused decode step, ring half: the new token goes to ring slot rs = L_old %
// hot -- row rs % 32 of its staged hot item (item_st, row pitch kPitch), for
// this attention (the kernel writes it into the ring in HBM separately).
// Thread tid writes channel tid of both rows.
template <bool kNamed = false, int kPitch = kRowStride>
__device__ __forceinline__ void ring_put(uint8_t *item_st, int rs, __half2 new_kv, int tid) {
  const int c = tid;
  __half *srow = reinterpret_cast<__half *>(item_st + (rs % kItemRows) * kPitch);
  srow[c] = __low2half(new_kv);
  srow[kDim + c] = __high2half(new_kv);
  fence_proxy_async_smem();
  work_sync<kNamed>();
}

// Log-sum-exp merge of n partial results of the G query heads of one kv head
// (read from global memory through L2).  Partial j is entry slot_of(j) of an
// array of partials: head hh's 128 FP32 at o + slot * o_js + hh * o_hs, its
// log2-sum-exp at lse + slot * l_js + hh * l_hs (-inf: empty, output 0).
// Warp w merges heads w, w + 4, ...; lane l channels 4l..4l+3; the loads of
// kFan partials are issued together.  Writes the FP16 output rows
// [G][128] at out (and the natural-log lse at lse_out), or, when out is null,
// the merged FP32 rows at p_o (head stride p_hs floats) with their
// log2-sum-exp at p_lse (head stride p_lhs).
template <int G, typename SlotOf, int kFan = kMergeFan>
__device__ __forceinline__ void merge_splits(const float *o, size_t o_js, size_t o_hs, const float *lse, size_t l_js,
                                             size_t l_hs, int n, SlotOf slot_of, int warp, int lane, __half *out,
                                             float *lse_out, float *p_o, size_t p_hs, float *p_lse, size_t p_lhs) {
  for (int hh = warp; hh < G; hh += kWarps) {
    float m = -INFINITY, den = 0.f;
    float4 num = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int j0 = 0; j0 < n; j0 += kFan) {
      const int nj = min(kFan, n - j0);
      const long long my_slot = lane < nj ? static_cast<long long>(slot_of(j0 + lane)) : 0;
      float4 ov[kFan];
#pragma unroll
      for (int j = 0; j < kFan; j++) {
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
      for (int j = 0; j < kFan; j++) {
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


// ---------------------------------------------------------------------------
// Per-item arithmetic on the tensor cores (mma.sync).  A lane is (g, t) =
// (lane / 4, lane % 4).  Two layouts meet here:
//  * score layout -- the C fragment of the QK product: lane (g, t) holds the
//    logits of head 4 * nt + g / 2 (head quad nt) for its tokens;
//  * value layout -- the C fragment of the P.V product: lane (g, t) holds the
//    output of head 4 * nt + t for channels 16 * mt + g and 16 * mt + g + 8
//    (mt = 0..7); a warp's online-softmax state lives in this layout.
// ---------------------------------------------------------------------------

// Online-softmax state of one warp (value layout).
template <int NT>
struct WarpState {
  float acc[NT][8][2];  // unnormalised output, head 4nt + t, channels 16mt + g (+ 8)
  float m_run[NT];      // running maximum logit (log2 domain) of head 4nt + t
  float l_run[NT];      // sum of the weights relative to m_run
};

template <int NT>
__device__ __forceinline__ void state_init(WarpState<NT> &st) {
#pragma unroll
  for (int nt = 0; nt < NT; nt++) {
    st.m_run[nt] = -INFINITY;
    st.l_run[nt] = 0.f;
#pragma unroll
    for (int mt = 0; mt < 8; mt++) st.acc[nt][mt][0] = st.acc[nt][mt][1] = 0.f;
  }
}

// A group of tokens (its maximum logit mx, its weights' sum S relative to mx)
// joins the state of one head: the running maximum is raised to cover mx
// (rescaling what was accumulated), the sum grows by 2^(mx - m_run) * S, and
// the factor 2^(mx - m_run) that the group's P.V result takes is returned.
// An empty group (mx = -inf) changes nothing and gets factor 0.
__device__ __forceinline__ float group_update(float mx, float S, float &m_run, float &l_run, float (&acc)[8][2]) {
  if (mx > m_run) {
    const float alpha = ex2(m_run - mx);  // 0 for the first group
#pragma unroll
    for (int mt = 0; mt < 8; mt++) {
      acc[mt][0] *= alpha;
      acc[mt][1] *= alpha;
    }
    l_run *= alpha;
    m_run = mx;
  }
  const float e = mx == -INFINITY ? 0.f : ex2(mx - m_run);
  l_run = fmaf(e, S, l_run);
  return e;
}

// q of one kv head's query heads, prepared once per CTA: every thread holds
// channel tid of each head (qv, FP32 from FP16).  Writes the head's 24-bit
// fixed-point digits qd[h][0..2][c] (hi, mid, lo), its FP16 copy qh[h][c] and
// the fixed-point step sq[h] = max|q_h| / kQFix; heads >= G are zero.
// qmax_w [kWarps][NH] is scratch.  Two CTA barriers.
template <int G, int NH, bool kNamed = false>
__device__ __forceinline__ void prepare_q(const float (&qv)[G], int8_t (*qd)[3][kDim], __half (*qh)[kDim],
                                          float *sq, float (*qmax_w)[NH], int warp, int lane, int tid) {
#pragma unroll
  for (int j = 0; j < G; j++) {
    float m = fabsf(qv[j]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0) qmax_w[warp][j] = m;
  }
  work_sync<kNamed>();
#pragma unroll
  for (int j = 0; j < NH; j++) {
    int8_t d0 = 0, d1 = 0, d2 = 0;
    __half hv = __float2half_rn(0.f);
    if (j < G) {
      const float M = fmaxf(fmaxf(qmax_w[0][j], qmax_w[1][j]), fmaxf(qmax_w[2][j], qmax_w[3][j]));
      const float inv = M > 0.f ? kQFix / M : 0.f;
      int qi = __float2int_rn(qv[j] * inv);
      qi = max(-8323072, min(8323072, qi));
      const int lo = ((qi + 128) & 255) - 128;
      const int r = (qi - lo) >> 8;
      const int mid = ((r + 128) & 255) - 128;
      const int hi = (r - mid) >> 8;
      d0 = static_cast<int8_t>(hi);
      d1 = static_cast<int8_t>(mid);
      d2 = static_cast<int8_t>(lo);
      hv = __float2half_rn(qv[j]);
      if (tid == 0) sq[j] = M / kQFix;
    } else if (tid == 0) {
      sq[j] = 0.f;
    }
    qd[j][0][tid] = d0;
    qd[j][1][tid] = d1;
    qd[j][2][tid] = d2;
    qh[j][tid] = hv;
  }
  work_sync<kNamed>();
}

// The QK A fragments of this lane (score layout).  Rows of the 16 x 32 A
// operand per head quad nt: row 2i = hi digits of head 4nt + i, row 2i + 8 =
// its mid digits, row 2i + 1 = its lo digits, row 2i + 9 = 0.  The k index of
// k-step ks maps to channel d as k = 4t' + i -> d = 32t' + 8ks + i and
// k = 16 + 4t' + i -> d = 32t' + 8ks + 4 + i, so lane (g, t) needs channels
// 32t .. 32t + 31 only (the K loads below follow the same map).
template <int NT>
__device__ __forceinline__ void load_qfrag(const int8_t (*qd)[3][kDim], int g, int t, uint32_t (&qa)[NT][4][4]) {
  const bool even = (g & 1) == 0;
#pragma unroll
  for (int nt = 0; nt < NT; nt++) {
    const int h = 4 * nt + (g >> 1);
    const int8_t *dig = qd[h][even ? 0 : 2];
    const int8_t *mid = qd[h][1];
#pragma unroll
    for (int ks = 0; ks < 4; ks++) {
      const int c = 32 * t + 8 * ks;
      qa[nt][ks][0] = *reinterpret_cast<const uint32_t *>(dig + c);
      qa[nt][ks][2] = *reinterpret_cast<const uint32_t *>(dig + c + 4);
      qa[nt][ks][1] = even ? *reinterpret_cast<const uint32_t *>(mid + c) : 0u;
      qa[nt][ks][3] = even ? *reinterpret_cast<const uint32_t *>(mid + c + 4) : 0u;
    }
  }
}

// One 64-token INT8 or INT4 sub-block staged at `stage` (K tile, then V tile
// at +8 KB), for one warp: its 16 tokens 16w .. 16w + 15 (tokens >= nvalid
// are masked when kMasked).
//  QK: mma m16n8k32 s8 per (head quad, 8-token column tile j, k-step): the
//      digits of q against the K codes, exact in int32; the lane pair (g,
//      g ^ 1) joins hi/mid and lo into the logit.  Column n of tile j is
//      token 16w + 4(n / 2) + 2j + n % 2, so lane (g, t) ends up with the
//      logits of tokens 16w + 4t + u, u = 0..3, in C order.
//  Softmax weights: p = rint(65535 * 2^(z - mx)), mx = the 16-token group's
//      maximum for the head (16-bit fixed point relative to the group's own
//      maximum), split into a high and a low byte.
//  P.V: mma m16n8k16 s8 x u8 per (channel tile, head quad): A = V codes of 16
//      channels x the warp's 16 tokens (ldmatrix on the channel-major tile),
//      B columns 2i / 2i + 1 = the high / low bytes of head i's weights, so
//      lane (g, t) gets head t's two partial sums per channel and joins them
//      exactly (256 * hi + lo) before the FP32 fold with the V scale.
// coef[nt]: K scale * q step of head 4nt + g/2 * softmax scale * log2(e);
// sv: V scale; psel: prmt selector of the lane's weight byte (g odd: low);
// v_lane: shared address of this lane's V row for the ldmatrix of channel
// tile pair 0 (INT8).
template <int NT, bool kInt4, bool kMasked>
__device__ __forceinline__ void cold_item(const uint8_t *stage, int nvalid, int warp, int g, int t,
                                          const uint32_t (&qa)[NT][4][4], const float (&coef)[NT], float sv,
                                          uint32_t psel, uint32_t v_lane, WarpState<NT> &st) {
  const bool even = (g & 1) == 0;
  int c[NT][2][4];
#pragma unroll
  for (int nt = 0; nt < NT; nt++)
#pragma unroll
    for (int j = 0; j < 2; j++) c[nt][j][0] = c[nt][j][1] = c[nt][j][2] = c[nt][j][3] = 0;
#pragma unroll
  for (int j = 0; j < 2; j++) {
    const int tok = 16 * warp + 4 * (g >> 1) + 2 * j + (g & 1);
    uint32_t kw[8];
    if constexpr (!kInt4) {
      const uint4 x0 = *reinterpret_cast<const uint4 *>(stage + tok * kDim + 32 * t);
      const uint4 x1 = *reinterpret_cast<const uint4 *>(stage + tok * kDim + 32 * t + 16);
      kw[0] = x0.x; kw[1] = x0.y; kw[2] = x0.z; kw[3] = x0.w;
      kw[4] = x1.x; kw[5] = x1.y; kw[6] = x1.z; kw[7] = x1.w;
    } else {
      // INT4 word ks of the lane's 16 bytes holds channels 32t + 8ks + 0..7:
      // low nibbles 0..3, high nibbles 4..7 -- exactly the two B registers
      const uint4 x = *reinterpret_cast<const uint4 *>(stage + tok * 64 + 16 * t);
      const uint32_t w4[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
      for (int ks = 0; ks < 4; ks++) unpack_int4(w4[ks], kw[2 * ks], kw[2 * ks + 1]);
    }
#pragma unroll
    for (int ks = 0; ks < 4; ks++)
#pragma unroll
      for (int nt = 0; nt < NT; nt++)
        mma_s8s8_k32(c[nt][j], qa[nt][ks][0], qa[nt][ks][1], qa[nt][ks][2], qa[nt][ks][3], kw[2 * ks],
                     kw[2 * ks + 1]);
  }
  const int m1 = even ? 256 : 1;
  const float w_self = even ? 256.f : 1.f, w_other = even ? 1.f : 256.f;
  uint32_t pb[NT];
  float f[NT];
#pragma unroll
  for (int nt = 0; nt < NT; nt++) {
    float z[4];
#pragma unroll
    for (int j = 0; j < 2; j++)
#pragma unroll
      for (int e = 0; e < 2; e++) {
        const int x = c[nt][j][e] * m1 + c[nt][j][2 + e];  // even: 256 hi + mid; odd: lo
        const int y = __shfl_xor_sync(0xffffffffu, x, 4);
        const float zz = fmaf(static_cast<float>(x), w_self, static_cast<float>(y) * w_other) * coef[nt];
        z[2 * j + e] = (kMasked && 16 * warp + 4 * t + 2 * j + e >= nvalid) ? -INFINITY : zz;
      }
    float mx = fmaxf(fmaxf(z[0], z[1]), fmaxf(z[2], z[3]));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
    const float mref = mx == -INFINITY ? 0.f : mx;
    uint32_t p[4];
    int S = 0;
#pragma unroll
    for (int u = 0; u < 4; u++) {
      // rint(65535 * 2^(z - mx)) by the 1.5 * 2^23 magic add (exact for [0, 2^22))
      p[u] = __float_as_uint(fmaf(ex2(z[u] - mref), kPFix, 12582912.f)) - 0x4B400000u;
      S += static_cast<int>(p[u]);
    }
    S += __shfl_xor_sync(0xffffffffu, S, 1);
    S += __shfl_xor_sync(0xffffffffu, S, 2);
    pb[nt] = prmt(prmt(p[0], p[1], 0x5410u), prmt(p[2], p[3], 0x5410u), psel);
    // the group's statistics for head 4nt + t (from lane 8t, which has g = 2t)
    const float mx_t = __shfl_sync(0xffffffffu, mx, 8 * t);
    const int S_t = __shfl_sync(0xffffffffu, S, 8 * t);
    const float e = group_update(mx_t, static_cast<float>(S_t) * (1.f / kPFix), st.m_run[nt], st.l_run[nt],
                                 st.acc[nt]);
    f[nt] = e * sv * (1.f / kPFix);
  }
  // V codes of channel tiles 2mp, 2mp + 1 and the P.V products
  uint32_t v_off0 = 0, v_off1 = 0;
  if constexpr (kInt4) {
    // INT4 V: channel row c at 32c bytes, the 8-byte unit of tokens 16w..16w+15
    // at (w ^ ((c / 4) % 4)) * 8, tokens 8i..8i+7 in its word i (low nibbles
    // first); lane (g, t) needs channel 16mt + g (+ 8), tokens 16w + 4t + 0..3
    v_off0 = kTileBytes + g * 32 + 8 * (warp ^ (g >> 2)) + 4 * (t >> 1);
    v_off1 = kTileBytes + (g + 8) * 32 + 8 * (warp ^ (2 + (g >> 2))) + 4 * (t >> 1);
  }
#pragma unroll
  for (int mp = 0; mp < 4; mp++) {
    uint32_t va[4];
    if constexpr (!kInt4) {
      ldmatrix_x4(va, v_lane + mp * 32 * kBlock);
    } else {
      const int sh = 4 * (t & 1);
#pragma unroll
      for (int h2 = 0; h2 < 2; h2++) {
        const int mt = 2 * mp + h2;
        const uint32_t x0 = *reinterpret_cast<const uint32_t *>(stage + v_off0 + mt * 16 * 32);
        const uint32_t x1 = *reinterpret_cast<const uint32_t *>(stage + v_off1 + mt * 16 * 32);
        va[2 * h2] = sext_nibbles((x0 >> sh) & 0x0f0f0f0fu);
        va[2 * h2 + 1] = sext_nibbles((x1 >> sh) & 0x0f0f0f0fu);
      }
    }
#pragma unroll
    for (int h2 = 0; h2 < 2; h2++) {
      const int mt = 2 * mp + h2;
#pragma unroll
      for (int nt = 0; nt < NT; nt++) {
        int d[4];
        mma_s8u8_k16_z(d, va[2 * h2], va[2 * h2 + 1], pb[nt]);
        st.acc[nt][mt][0] = fmaf(f[nt], static_cast<float>(d[0] * 256 + d[1]), st.acc[nt][mt][0]);
        st.acc[nt][mt][1] = fmaf(f[nt], static_cast<float>(d[2] * 256 + d[3]), st.acc[nt][mt][1]);
      }
    }
  }
}

// nrow FP16 rows (K row, V row) staged at `stage` with pitch kPitch (kRowStride,
// 16 bytes of padding, spreads ldmatrix rows over the banks) -- the hot ring, or
// half of an FP16 cold block -- for one warp: rows 8w ..
// 8w + 7 (rows >= nrow masked; their V is read from the zero row at
// zero_addr).  QK: mma m16n8k16 f16 (FP32 accumulation) of the FP16 q (A
// rows g: head g/2, rows g + 8: head 4 + g/2) with the K rows (ldmatrix);
// weights 2^(z - mx) relative to the 8-row group's maximum, in FP16; P.V: mma
// m16n8k8 f16 of the V rows (ldmatrix.trans) with B columns 2i = head i's
// weights, 2i + 1 = 0, so lane (g, t) gets head t's sums.
template <int NT, int kPitch = kRowStride>
__device__ __forceinline__ void hot_item(const uint8_t *stage, int nrow, int warp, int lane, int g, int t,
                                         const __half (*qh)[kDim], float qk_scale, uint32_t zero_addr,
                                         WarpState<NT> &st) {
  const int nv = nrow - 8 * warp;
  if (nv <= 0) return;
  const uint32_t row0 = smem_addr(stage) + (8 * warp + (lane & 7)) * kPitch;
  float c[4] = {0.f, 0.f, 0.f, 0.f};
  const __half *q0 = qh[g >> 1];
  const __half *q1 = qh[NT > 1 ? 4 + (g >> 1) : 0];
#pragma unroll
  for (int xq = 0; xq < 4; xq++) {
    uint32_t kb[4];
    ldmatrix_x4(kb, row0 + 16 * (lane >> 3) + 64 * xq);
#pragma unroll
    for (int kk = 0; kk < 2; kk++) {
      const int d0 = 16 * (2 * xq + kk) + 2 * t;
      const uint32_t a0 = *reinterpret_cast<const uint32_t *>(q0 + d0);
      const uint32_t a2 = *reinterpret_cast<const uint32_t *>(q0 + d0 + 8);
      const uint32_t a1 = NT > 1 ? *reinterpret_cast<const uint32_t *>(q1 + d0) : 0u;
      const uint32_t a3 = NT > 1 ? *reinterpret_cast<const uint32_t *>(q1 + d0 + 8) : 0u;
      mma_f16_k16(c, a0, a1, a2, a3, kb[2 * kk], kb[2 * kk + 1]);
    }
  }
  uint32_t pb[NT];
  float f[NT];
#pragma unroll
  for (int nt = 0; nt < NT; nt++) {
    float z[2];
#pragma unroll
    for (int e = 0; e < 2; e++) z[e] = (2 * t + e < nv) ? c[2 * nt + e] * qk_scale : -INFINITY;
    float mx = fmaxf(z[0], z[1]);
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
    const float mref = mx == -INFINITY ? 0.f : mx;
    const __half2 hp = __floats2half2_rn(ex2(z[0] - mref), ex2(z[1] - mref));
    const float2 pr = __half22float2(hp);  // the weights as the tensor cores see them
    float S = pr.x + pr.y;
    S += __shfl_xor_sync(0xffffffffu, S, 1);
    S += __shfl_xor_sync(0xffffffffu, S, 2);
    pb[nt] = (g & 1) ? 0u : *reinterpret_cast<const uint32_t *>(&hp);
    const float mx_t = __shfl_sync(0xffffffffu, mx, 8 * t);
    const float S_t = __shfl_sync(0xffffffffu, S, 8 * t);
    f[nt] = group_update(mx_t, S_t, st.m_run[nt], st.l_run[nt], st.acc[nt]);
  }
  const bool row_ok = (lane & 7) < nv;
#pragma unroll
  for (int xp = 0; xp < 4; xp++) {
    uint32_t va[4];
    ldmatrix_x4_trans(va, row_ok ? row0 + kHotTokenBytes / 2 + 16 * (lane >> 3) + 64 * xp : zero_addr);
#pragma unroll
    for (int h2 = 0; h2 < 2; h2++) {
      const int mt = 2 * xp + h2;
#pragma unroll
      for (int nt = 0; nt < NT; nt++) {
        float d[4];
        mma_f16_k8_z(d, va[2 * h2], va[2 * h2 + 1], pb[nt]);
        st.acc[nt][mt][0] = fmaf(f[nt], d[0], st.acc[nt][mt][0]);
        st.acc[nt][mt][1] = fmaf(f[nt], d[2], st.acc[nt][mt][1]);
      }
    }
  }
}

// End of a split: the four warps' states merged into the split's normalised
// output for channel tid (o_s per head) and its log2-sum-exp per head (-inf
// and 0 when empty).  mbuf: FP32 [kWarps][4 * NT][kMbufPitch], mrun / lrun
// [kWarps][4 * NT] in shared memory.  Two CTA barriers; on return mbuf may be
// reused.
template <int G, int NT, bool kNamed = false>
__device__ __forceinline__ void merge_warps(float *mbuf, float (*mrun)[4 * NT], float (*lrun)[4 * NT],
                                            const WarpState<NT> &st, int warp, int lane, int tid, float (&o_s)[G],
                                            float (&lse2_s)[G]) {
  const int g = lane >> 2, t = lane & 3;
#pragma unroll
  for (int nt = 0; nt < NT; nt++) {
    float *row = mbuf + (warp * 4 * NT + 4 * nt + t) * kMbufPitch;
#pragma unroll
    for (int mt = 0; mt < 8; mt++) {
      row[16 * mt + g] = st.acc[nt][mt][0];
      row[16 * mt + g + 8] = st.acc[nt][mt][1];
    }
    if (g == 0) {
      mrun[warp][4 * nt + t] = st.m_run[nt];
      lrun[warp][4 * nt + t] = st.l_run[nt];
    }
  }
  work_sync<kNamed>();
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
        const float fw = ex2(mrun[w][hh] - mm);
        num = fmaf(fw, mbuf[(w * 4 * NT + hh) * kMbufPitch + tid], num);
        den = fmaf(fw, lrun[w][hh], den);
      }
    }
    if (den > 0.f) {
      o_s[hh] = num * __frcp_rn(den);
      lse2_s[hh] = mm + __log2f(den);
    }
  }
  work_sync<kNamed>();
}

}  // namespace hyb
