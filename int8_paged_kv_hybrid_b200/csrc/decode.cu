// decode.cu -- hyb_decode_attn: split-KV single-query attention over the
// hybrid_v2 cache (FP16 hot ring + INT8/INT4 cold blocks behind a block
// table) on sm_100a CUDA cores.
//
// Method: web page "DeepSeek V4混合式KV Cache推理优化实战解析", section 4.2
// (attention over the FP16 hot zone plus the dequantized cold zone; one
// softmax over both, merged by log-sum-exp instead of the page's torch.cat),
// section 3.2 (hot zone: K and V interleaved per token, 512-byte aligned).
//
// Work decomposition: one CTA (4 warps) per (split, kv head, sequence).  A
// split is a run of up to `split_blocks` cold blocks; the split that holds
// the sequence's last cold block also attends the hot ring.  Each cold block
// (K tile 8 KB + V tile 8 KB, or 4 + 4 KB for INT4) and the hot ring (16 KB)
// is one pipeline item, brought into a 3-stage shared-memory ring by the TMA
// engine with one 1-D bulk copy (no cluster multicast) completing on an
// mbarrier; every wait is bounded.  Three CTAs fit on an SM for up to 4 query
// heads per kv head (two above that).
//
// Arithmetic (per kv head, for its G = Hq/Hkv query heads):
//  * q is turned into 16-bit fixed point per query head (q_i = rint(q * 32767
//    / max|q|)); a cold logit is the exact int32 dot product of q_i with the
//    K codes (dp2a: two 16x8-bit products per instruction), times
//    max|q|/32767 * K-scale * softmax_scale * log2(e).  Eight lanes share a
//    token (16 channels each); each lane keeps its heads in a lane-dependent
//    order (head = k XOR x(lane)) so the cross-lane reduction that leaves one
//    head's total in each lane needs no selects.
//  * Warp w owns tokens 16w..16w+15 of every block and keeps its own online
//    softmax state (running max, sum, FP32 output accumulator) per head,
//    rescaling only when the running max grows.  Its softmax weights relative
//    to the 16-token maximum are 16-bit fixed point (p_i = rint(32767 *
//    2^(z - max))); P.V is again an exact int32 dp2a sum over the V codes,
//    folded into the FP32 state with the V scale.
//  * Hot tokens are attended in FP32 from the FP16 values (never quantized).
//  * The 4 warp states are merged in FP32 at the end of the split; the last
//    CTA of a (sequence, kv head) to finish merges the splits (log-sum-exp)
//    and writes the FP16 output.
// Tensor cores are not used: per byte of KV the work is a few integer
// multiply-adds, and the kernel is bound by HBM bandwidth.
#include <cfloat>

#include "kernels.cuh"

namespace hyb {

constexpr int kWarps = 4;
constexpr int kThreads = 32 * kWarps;
constexpr int kStages = 3;
constexpr int kMaxSplitBlocks = 128;  // == kThreads: one block-table entry per thread
constexpr long long kWaitCycles = 1ll << 31;  // ~1 s at B200 clocks
constexpr float kLn2 = 0.69314718055994531f;

template <int G>
__host__ __device__ constexpr int pow2_heads() {
  return G <= 1 ? 1 : (G <= 2 ? 2 : (G <= 4 ? 4 : 8));
}

template <int G>
struct DecodeSmem {
  static constexpr int P = pow2_heads<G>();
  alignas(128) uint8_t ring[kStages][kTilePairBytes];
  uint64_t full[kStages];   // data of the stage landed (TMA transaction count)
  uint64_t empty[kStages];  // every warp is done with the stage
  int32_t phys[kMaxSplitBlocks];
  float2 scl[kMaxSplitBlocks];  // (K scale, V scale) of each block of the split
  alignas(16) float qf[P][kDim];     // q in FP32 (rows >= G are zero)
  alignas(16) int16_t qi[P][kDim];   // q in 16-bit fixed point (rows >= G are zero)
  float sq[P];                       // fixed-point step of each head's q
  alignas(16) uint16_t pcode[kWarps][G][16];
  alignas(16) float phot[kWarps][G][8];
  float mrun[kWarps][G];
  float lrun[kWarps][G];
  int8_t rqt[2][256];  // fused step: re-quantization tables of the tail block (K, V)
  float seal_s[2];     // fused step: the tail block's scales after sealing
  int seal_rq[2];      // fused step: 1 if the tail block's codes were re-quantized
  float cl_l[G];   // this split's log2-sum-exp per head, read by the cluster's merge
  int last;
  int abort_flag;
};

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

// Fused decode step: append the sequence's new token inside the staged copies
// of the tail block (item ncold-1) and the hot ring (item ncold), with the
// arithmetic of hyb_kv_append (bit-exact), and write back what changed.  All
// threads of the CTA call it.
template <int G>
__device__ __forceinline__ void fused_append(DecodeSmem<G> &sm, const DecodeArgs &a, int b, int h, int L_old,
                                          int i0, int ncold, int n_int4_b, bool do_seal, __half2 new_kv,
                                          int tid, int warp, int lane) {
  uint8_t *hot_st = sm.ring[ncold % kStages];
  const int rs = L_old % kHot;  // ring slot of the evicted and of the new token
  const int e = L_old - kHot;   // position sealed (when do_seal)
  const int slot = do_seal ? e % kBlock : 0;
  const int ti = do_seal ? ncold - 1 : 0;  // tail item of this split
  const bool int4 = do_seal && (i0 + ti) < n_int4_b;
  const int Q = int4 ? 7 : 127;
  uint8_t *tile_st = sm.ring[ti % kStages];
  if (do_seal && warp < 2) {
    // warp 0: K, warp 1: V -- absmax of the evicted token, new scale
    const int kv = warp;
    const __half *row = reinterpret_cast<const __half *>(hot_st + rs * kHotTokenBytes) + kv * kDim;
    float amax = 0.f;
#pragma unroll
    for (int j = 0; j < 4; j++) amax = fmaxf(amax, fabsf(__half2float(row[4 * lane + j])));
#pragma unroll
    for (int m = 16; m > 0; m >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, m));
    const float s_c = __fdiv_rn(amax, static_cast<float>(Q));
    const float s_old = kv ? sm.scl[ti].y : sm.scl[ti].x;
    float s_new = s_c;
    int rq = 0;
    if (slot != 0) {
      if (s_c > s_old) rq = 1;
      else s_new = s_old;
    }
    if (rq)
      for (int c = lane - 127; c <= 127; c += 32)
        sm.rqt[kv][c + 127] = static_cast<int8_t>(requantize(c, s_old, s_new, Q));
    if (lane == 0) {
      sm.seal_s[kv] = s_new;
      sm.seal_rq[kv] = rq;
    }
  }
  __syncthreads();
  if (do_seal && tid == 0) sm.scl[ti] = make_float2(sm.seal_s[0], sm.seal_s[1]);  // attention uses these
  if (do_seal) {
    // codes already in the tail block, under a grown scale
#pragma unroll
    for (int kv = 0; kv < 2; kv++) {
      if (!sm.seal_rq[kv]) continue;
      uint32_t *w32 = reinterpret_cast<uint32_t *>(tile_st + kv * kTileBytes);
      const int nw = requant_nwords(kv, int4, slot);
      for (int w = tid; w < nw; w += kThreads) w32[w] = requant_word(w32[w], w, kv, int4, slot, sm.rqt[kv]);
    }
  }
  __syncthreads();
  const int c = tid;  // channel
  if (do_seal) {
    // the evicted token's codes into slot `slot`
    const __half *krow = reinterpret_cast<const __half *>(hot_st + rs * kHotTokenBytes);
    const int ck = quantize(__half2float(krow[c]), sm.seal_s[0], Q);
    const int cv = quantize(__half2float(krow[kDim + c]), sm.seal_s[1], Q);
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
  // the new token into the ring slot: the staged copy (for this attention) and the cache
  {
    __half *srow = reinterpret_cast<__half *>(hot_st + rs * kHotTokenBytes);
    srow[c] = __low2half(new_kv);
    srow[kDim + c] = __high2half(new_kv);
    __half *grow = reinterpret_cast<__half *>(a.hot) + ((((size_t)b * a.hkv + h) * kHot + rs) * 2) * kDim;
    grow[c] = __low2half(new_kv);
    grow[kDim + c] = __high2half(new_kv);
  }
  if (do_seal) {
    // write back what changed in the tail block: scales, then the whole tile
    // if its codes were re-quantized, else the sealed token's codes
    const int phys = sm.phys[ti];
    uint8_t *gtile = a.cold + ((size_t)phys * a.hkv + h) * kTilePairBytes;
    if (tid < 2) a.scales[((size_t)phys * a.hkv + h) * 2 + tid] = sm.seal_s[tid];
#pragma unroll
    for (int kv = 0; kv < 2; kv++) {
      uint8_t *g = gtile + kv * kTileBytes;
      const uint8_t *t = tile_st + kv * kTileBytes;
      if (sm.seal_rq[kv]) {
        const int nvec = (int4 ? kTileBytes / 2 : kTileBytes) / 16;
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
// (read from global memory through L2).  Partial j of head hh: 128 FP32 at
// o + hh * o_hs + j * 128 and its log2-sum-exp at lse + hh * l_hs + j (-inf:
// empty, output 0).  Warp w merges heads w, w + 4, ...; lane l channels
// 4l..4l+3; the loads of kMergeFan partials are issued together.  Writes the
// FP16 output rows [G][128] at out (and the natural-log lse at lse_out), or,
// when out is null, the merged FP32 rows at p_o (row stride p_s * 128) with
// their log2-sum-exp at p_lse (stride p_s).
template <int G>
__device__ __forceinline__ void merge_splits(const float *o, size_t o_hs, const float *lse, size_t l_hs, int n,
                                             int warp, int lane, __half *out, float *lse_out, float *p_o,
                                             float *p_lse, int p_s) {
  for (int hh = warp; hh < G; hh += kWarps) {
    const float *oh = o + hh * o_hs + 4 * lane;
    const float *lh = lse + hh * l_hs;
    float m = -INFINITY, den = 0.f;
    float4 num = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int j0 = 0; j0 < n; j0 += kMergeFan) {
      const int nj = min(kMergeFan, n - j0);
      float4 ov[kMergeFan];
#pragma unroll
      for (int j = 0; j < kMergeFan; j++)
        ov[j] = j < nj ? __ldcg(reinterpret_cast<const float4 *>(oh + (size_t)(j0 + j) * kDim))
                       : make_float4(0.f, 0.f, 0.f, 0.f);
      const float lj = lane < nj ? __ldcg(lh + j0 + lane) : -INFINITY;
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
      *reinterpret_cast<float4 *>(p_o + (size_t)hh * p_s * kDim + 4 * lane) =
          make_float4(num.x * inv, num.y * inv, num.z * inv, num.w * inv);
      if (lane == 0) p_lse[(size_t)hh * p_s] = lse2;
    }
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

// kCluster: the grid is launched in clusters of n_splits CTAs (the splits of
// one (sequence, kv head)); splits are merged through distributed shared
// memory instead of the workspace.
template <int G, bool kCluster>
__global__ void __launch_bounds__(kThreads, (G <= 4 ? 3 : 2)) decode_kernel(const DecodeArgs a) {
  constexpr int P = pow2_heads<G>();
  extern __shared__ __align__(128) uint8_t smem_raw[];
  DecodeSmem<G> &sm = *reinterpret_cast<DecodeSmem<G> *>(smem_raw);

  const int s = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int S = a.n_splits;
  const int hq0 = h * G;
  const int i0 = s * a.split_blocks;

  // independent loads first: the sequence length, this split's block-table
  // entries (one per thread, clamped to the row) and q
  const int L_old = a.seq_lens[b];
  int n_app = a.n_new ? a.n_new[b] : 0;  // fused step: tokens appended to this sequence
  const int i_tid = i0 + tid;
  const int phys_raw =
      (tid < a.split_blocks && i_tid < a.max_blocks) ? a.block_table[(size_t)b * a.max_blocks + i_tid] : -1;
  float qv[G];
#pragma unroll
  for (int j = 0; j < G; j++) qv[j] = __half2float(a.q[((size_t)b * a.hq + hq0) * kDim + j * kDim + tid]);

  if (n_app < 0 || n_app > 1) {
    if (tid == 0 && s == 0 && h == 0) set_status(a.status, HYB_STATUS_BAD_N_NEW);
    n_app = 0;
  }
  int L = L_old + n_app;
  if (L_old < 0 || L > a.max_seq_len) {
    // sequence skipped: treated as empty (zero output, lse -inf), not appended to
    if (tid == 0 && s == 0 && h == 0) set_status(a.status, HYB_STATUS_SEQ_LEN);
    L = 0;
    n_app = 0;
  }
  if (a.n_new && tid == 32) {
    // every CTA of the grid has read seq_lens[b] once this count is complete;
    // the last one advances it
    const int ticket = atomicAdd(&a.seq_cnt[b], 1);
    if (ticket == static_cast<int>(gridDim.x * gridDim.y) - 1) {
      a.seq_lens[b] = L_old + n_app;
      a.seq_cnt[b] = 0;
    }
  }
  const int Lc = max(0, L - kHot);
  const int nblk = (Lc + kBlock - 1) / kBlock;
  const int Sb = max(1, (nblk + a.split_blocks - 1) / a.split_blocks);
  // past this sequence's last split: no work and no partial (a cluster member
  // still takes part in the cluster's merge, with an empty state)
  if (!kCluster && s >= Sb) return;
  const int ncold = max(0, min(nblk, i0 + a.split_blocks) - i0);
  const int nhot = (s == Sb - 1) ? min(L, kHot) : 0;
  const int nitems = ncold + (nhot > 0 ? 1 : 0);
  // fused step, in the split that holds the tail block and the hot ring: the
  // new token goes to ring slot L_old % 32 (whose old occupant, position
  // L_old - 32, is sealed into the tail block first)
  const bool do_ring = n_app == 1 && nhot > 0;
  const bool do_seal = do_ring && L_old >= kHot;
  const int k_fused = do_seal ? ncold - 1 : ncold;  // item at which the append is done
  __half2 new_kv = __halves2half2(__float2half_rn(0.f), __float2half_rn(0.f));
  if (do_ring) {
    const size_t o = ((size_t)b * a.hkv + h) * kDim + tid;
    new_kv = __halves2half2(a.k_new[o], a.v_new[o]);
  }
  const int n_int4_b = a.quant_bits == 4 ? 0x7fffffff : (a.n_int4 ? a.n_int4[b] : 0);

  if (tid == 0) {
#pragma unroll
    for (int st = 0; st < kStages; st++) {
      mbar_init(&sm.full[st], 1);
      mbar_init(&sm.empty[st], kWarps);
    }
    sm.abort_flag = 0;
    mbar_fence_init();
  }
  if (tid < ncold) {
    int phys = phys_raw;
    if (phys < 0 || phys >= a.num_phys) {
      set_status(a.status, HYB_STATUS_BAD_BLOCK);
      phys = -1;
    }
    sm.phys[tid] = phys;
  }
#pragma unroll
  for (int j = 0; j < P; j++) sm.qf[j][tid] = j < G ? qv[j] : 0.f;
  __syncthreads();

  const uint64_t pol = l2_policy_evict_first();
  auto issue = [&](int k) {
    const int st = k % kStages;
    uint8_t *dst = sm.ring[st];
    if (k < ncold) {
      const int phys = sm.phys[k];
      if (phys < 0) {
        mbar_arrive(&sm.full[st]);
        return;
      }
      const uint8_t *src = a.cold + ((size_t)phys * a.hkv + h) * kTilePairBytes;
      if (i0 + k >= n_int4_b) {
        mbar_arrive_expect_tx(&sm.full[st], kTilePairBytes);
        bulk_g2s(dst, src, kTilePairBytes, &sm.full[st], pol);
      } else {
        mbar_arrive_expect_tx(&sm.full[st], kTileBytes);
        bulk_g2s(dst, src, kTileBytes / 2, &sm.full[st], pol);
        bulk_g2s(dst + kTileBytes, src + kTileBytes, kTileBytes / 2, &sm.full[st], pol);
      }
    } else {
      const uint8_t *src = a.hot + ((size_t)b * a.hkv + h) * kHotBytes;
      const uint32_t bytes = static_cast<uint32_t>(nhot) * kHotTokenBytes;
      mbar_arrive_expect_tx(&sm.full[st], bytes);
      bulk_g2s(dst, src, bytes, &sm.full[st], pol);
    }
  };
  // block scales: requested before the bulk copies so that they do not queue
  // behind them; stored once they arrive (overlapping the copies)
  float2 sc_ld = make_float2(0.f, 0.f);
  if (tid < ncold && sm.phys[tid] >= 0)
    sc_ld = __ldg(reinterpret_cast<const float2 *>(a.scales + ((size_t)sm.phys[tid] * a.hkv + h) * 2));
  int issued = 0;
  if (tid == 0) {
    issued = min(nitems, kStages);
    for (int k = 0; k < issued; k++) issue(k);
  }
  if (tid < ncold) sm.scl[tid] = sc_ld;
  // q in 16-bit fixed point per head (padding heads stay zero)
  for (int j = warp; j < P; j += kWarps) {
    float amax = 0.f;
    for (int c = lane; c < kDim; c += 32) amax = fmaxf(amax, fabsf(sm.qf[j][c]));
#pragma unroll
    for (int m = 16; m > 0; m >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, m));
    const float inv = amax > 0.f ? 32767.f / amax : 0.f;
    for (int c = lane; c < kDim; c += 32) {
      const int v = __float2int_rn(sm.qf[j][c] * inv);
      sm.qi[j][c] = static_cast<int16_t>(max(-32767, min(32767, v)));
    }
    if (lane == 0) sm.sq[j] = amax > 0.f ? amax / 32767.f : 0.f;
  }
  __syncthreads();

  const int tg = lane >> 3, cs = lane & 7;
  const int hx = head_xor<P>(lane);   // this lane's value k is head k ^ hx; its final head is hx
  const bool owner = (lane & (8 / P - 1)) == 0 && hx < G;
  const float sq_hd = sm.sq[hx];
  // full-block path: the lane's K row (tokens 16w + 4tg + step) and V words
  const int k_lane = (16 * warp + 4 * tg) * kDim + 16 * cs;
  const int v_lane = kTileBytes + lane * kBlock + 16 * (warp ^ ((lane >> 1) & 3));

  uint32_t qp[P][8];  // q pairs of this lane's 16 channels, in the lane's head order
#pragma unroll
  for (int k = 0; k < P; k++) {
    const uint4 *src = reinterpret_cast<const uint4 *>(&sm.qi[k ^ hx][16 * cs]);
    const uint4 x0 = src[0], x1 = src[1];
    qp[k][0] = x0.x; qp[k][1] = x0.y; qp[k][2] = x0.z; qp[k][3] = x0.w;
    qp[k][4] = x1.x; qp[k][5] = x1.y; qp[k][6] = x1.z; qp[k][7] = x1.w;
  }

  // Online-softmax state of this warp.  m_run: running max per head (the
  // same in every lane); acc: unnormalised output of the lane's channels;
  // weights are taken relative to m_run, so the denominator can be summed
  // per lane (head hx, its own tokens) and reduced across lanes only at the
  // end: l_lane (FP32) plus psum_lane (integer sum of 16-bit weight codes).
  float m_run[G], acc[G][4];
#pragma unroll
  for (int hh = 0; hh < G; hh++) {
    m_run[hh] = -INFINITY;
#pragma unroll
    for (int kk = 0; kk < 4; kk++) acc[hh][kk] = 0.f;
  }
  float m_hx = hx < G ? -INFINITY : INFINITY;  // m_run of this lane's head (+inf: padding head)
  float l_lane = 0.f;
  int psum_lane = 0;

  bool aborted = false;
  int next_issue = issued;  // thread 0: next item to bring in
  for (int k = 0; k < nitems; k++) {
    const int st = k % kStages;
    // thread 0 refills stages the warps have released: item k must be in
    // flight before anyone waits for it, later ones only if already free
    if (tid == 0) {
      for (; next_issue < min(nitems, k + kStages); next_issue++) {
        const int j = next_issue - kStages;  // previous item of that stage
        if (next_issue <= k + ((do_ring && k == k_fused) ? 1 : 0)) {
          if (!mbar_wait_bounded(&sm.empty[j % kStages], (j / kStages) & 1, kWaitCycles)) {
            set_status(a.status, HYB_STATUS_TIMEOUT);
            sm.abort_flag = 1;
            break;
          }
        } else if (!mbar_try_wait(&sm.empty[j % kStages], (j / kStages) & 1)) {
          break;
        }
        issue(next_issue);
      }
      issued = next_issue;
    }
    bool ok = mbar_wait_bounded(&sm.full[st], (k / kStages) & 1, kWaitCycles);
    if (!ok && lane == 0) set_status(a.status, HYB_STATUS_TIMEOUT);
    if (do_ring && k == k_fused) {
      // ---------------- fused append (whole CTA, in the staged copies) ----------------
      const int kh = ncold;  // the hot item
      if (k != kh) ok = ok && mbar_wait_bounded(&sm.full[kh % kStages], (kh / kStages) & 1, kWaitCycles);
      ok = __syncthreads_and(ok) != 0;
      if (ok) fused_append<G>(sm, a, b, h, L_old, i0, ncold, n_int4_b, do_seal, new_kv, tid, warp, lane);
    }
    ok = ok && *reinterpret_cast<volatile int *>(&sm.abort_flag) == 0;
    const uint8_t *stage = sm.ring[st];
    if (ok && k < ncold) {
      // ---------------- cold block ----------------
      const int i = i0 + k;
      const int nvalid = sm.phys[k] < 0 ? 0 : min(kBlock, Lc - i * kBlock);
      const int nv = nvalid - 16 * warp;
      const bool int4 = i < n_int4_b;
      const float2 sc = sm.scl[k];
      const float coef = sq_hd * sc.x * a.qk_scale;
      if (nvalid == kBlock && !int4) {
        cold_block_full<G, P>(stage, k_lane, v_lane, qp, coef, sc.y * (1.f / 32767.f), sm.pcode[warp], hx, tg,
                              owner, m_run, acc, m_hx, l_lane, psum_lane);
      } else if (nv > 0) {
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
            sm.pcode[warp][hx][4 * step + tg] = static_cast<uint16_t>(pc[step]);
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
        const float cv = sc.y * (1.f / 32767.f);
#pragma unroll
        for (int hh = 0; hh < G; hh++) {
          // p codes of this warp's 16 tokens, as 16-bit pairs (tokens 2i, 2i+1)
          const uint4 pa = *reinterpret_cast<const uint4 *>(&sm.pcode[warp][hh][0]);
          const uint4 pb = *reinterpret_cast<const uint4 *>(&sm.pcode[warp][hh][8]);
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
    } else if (ok) {
      // ---------------- hot ring (FP16, FP32 math) ----------------
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
            const float4 *qv4 = reinterpret_cast<const float4 *>(&sm.qf[kk ^ hx][16 * cs]);
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
          z[step] = (4 * step + tg < nv) ? dot[0] * a.qk_scale : -INFINITY;
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
          sm.phot[warp][hx][tg] = pv[0];
          sm.phot[warp][hx][4 + tg] = pv[1];
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
            const float p = sm.phot[warp][hh][tt];
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
    __syncwarp();
    if (!ok) {
      sm.abort_flag = 1;
      aborted = true;
      break;
    }
    if (lane == 0) mbar_arrive(&sm.empty[st]);
  }
  aborted = __syncthreads_or(aborted) != 0;
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

  if (aborted) {
    // let every copy still in flight land before the CTA's shared memory is
    // released: the last item issued into each stage
    if (tid == 0) {
      for (int j = max(0, issued - kStages); j < issued; j++)
        (void)mbar_wait_bounded(&sm.full[j % kStages], (j / kStages) & 1, kWaitCycles);
    }
    __syncthreads();
  } else {
    // ---------------- merge the 4 warp states ----------------
    float *mbuf = reinterpret_cast<float *>(&sm.ring[0][0]);  // [kWarps][G][kDim]
#pragma unroll
    for (int hh = 0; hh < G; hh++)
#pragma unroll
      for (int kk = 0; kk < 4; kk++) mbuf[(warp * G + hh) * kDim + lane + 32 * kk] = acc[hh][kk];
    if (lane == 0) {
#pragma unroll
      for (int hh = 0; hh < G; hh++) {
        sm.mrun[warp][hh] = m_run[hh];
        sm.lrun[warp][hh] = l_run[hh];
      }
    }
    __syncthreads();
  }
  // this split's normalised output (channel tid) and log2-sum-exp per head
  float o_s[G], lse2_s[G];
#pragma unroll
  for (int hh = 0; hh < G; hh++) {
    o_s[hh] = 0.f;
    lse2_s[hh] = -INFINITY;
    if (aborted) continue;
    const float *mbuf = reinterpret_cast<const float *>(&sm.ring[0][0]);
    float mm = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; w++) mm = fmaxf(mm, sm.mrun[w][hh]);
    float num = 0.f, den = 0.f;
    if (mm != -INFINITY) {
#pragma unroll
      for (int w = 0; w < kWarps; w++) {
        const float f = ex2(sm.mrun[w][hh] - mm);
        num = fmaf(f, mbuf[(w * G + hh) * kDim + tid], num);
        den = fmaf(f, sm.lrun[w][hh], den);
      }
    }
    if (den > 0.f) {
      o_s[hh] = num * __frcp_rn(den);
      lse2_s[hh] = mm + __log2f(den);
    }
  }
  if constexpr (kCluster) {
    // ---------------- split merge across the cluster (distributed shared memory) ----------------
    float *cl_o = reinterpret_cast<float *>(&sm.ring[0][0]);  // [G][kDim], this split's output
    __syncthreads();  // the warp-merge buffer above is no longer read
#pragma unroll
    for (int hh = 0; hh < G; hh++) cl_o[hh * kDim + tid] = o_s[hh];
    if (tid == 0) {
#pragma unroll
      for (int hh = 0; hh < G; hh++) sm.cl_l[hh] = lse2_s[hh];
    }
    cluster_sync_all();
    // CTA s of the cluster merges output elements [s*per, (s+1)*per)
    const int per = (G * kDim + S - 1) / S;
    for (int e = s * per + tid; e < min((s + 1) * per, G * kDim); e += kThreads) {
      const int hh = e / kDim, c = e - hh * kDim;
      float lj[16];
      float m = -INFINITY;
#pragma unroll
      for (int j = 0; j < 16; j++) {
        lj[j] = j < S ? ld_cluster_f32(&sm.cl_l[hh], j) : -INFINITY;
        m = fmaxf(m, lj[j]);
      }
      float num = 0.f, den = 0.f;
      if (m != -INFINITY) {
#pragma unroll
        for (int j = 0; j < 16; j++) {
          if (j < S) {
            const float wgt = ex2(lj[j] - m);
            num = fmaf(wgt, ld_cluster_f32(&cl_o[hh * kDim + c], j), num);
            den += wgt;
          }
        }
      }
      const size_t row = (size_t)b * a.hq + hq0 + hh;
      a.out[row * kDim + c] = __float2half_rn(den > 0.f ? num / den : 0.f);
      if (c == 0 && a.lse_out) a.lse_out[row] = den > 0.f ? (m + log2f(den)) * kLn2 : -INFINITY;
    }
    cluster_sync_all();  // no CTA leaves while its shared memory may still be read
    return;
  }
  if (Sb == 1) {
#pragma unroll
    for (int hh = 0; hh < G; hh++) {
      const size_t row = (size_t)b * a.hq + hq0 + hh;
      a.out[row * kDim + tid] = __float2half_rn(o_s[hh]);
      if (tid == 0 && a.lse_out) a.lse_out[row] = lse2_s[hh] * kLn2;
    }
    return;
  }
  // ---------------- split merge in global memory ----------------
  // The last CTA of (sequence, kv head) to finish merges the splits; with
  // more than kMergeFan splits, the last CTA of each group of kMergeFan
  // splits merges the group first and the last group merges the groups.
  const size_t row0 = (size_t)b * a.hq + hq0;
#pragma unroll
  for (int hh = 0; hh < G; hh++) {
    a.o_part[((row0 + hh) * S + s) * kDim + tid] = o_s[hh];
    if (tid == 0) a.lse_part[(row0 + hh) * S + s] = lse2_s[hh];
  }
  const int unit = b * a.hkv + h;
  const bool grouped = Sb > kMergeFan;
  const int grp = s / kMergeFan;
  __threadfence();
  __syncthreads();
  if (tid == 0) {
    int32_t *cnt = grouped ? &a.g_counters[(size_t)unit * a.n_groups + grp] : &a.counters[unit];
    const int need = grouped ? min(kMergeFan, Sb - grp * kMergeFan) : Sb;
    const int last = atomicAdd(cnt, 1) == need - 1;
    if (last) *cnt = 0;  // ready for the next call
    sm.last = last;
  }
  __syncthreads();
  if (!sm.last) return;
  __threadfence();
  if (!grouped) {
    merge_splits<G>(a.o_part + row0 * S * kDim, (size_t)S * kDim, a.lse_part + row0 * S, S, Sb, warp, lane,
                    a.out + row0 * kDim, a.lse_out ? a.lse_out + row0 : nullptr, nullptr, nullptr, 0);
    return;
  }
  const int NG = a.n_groups;
  const int j0 = grp * kMergeFan;
  merge_splits<G>(a.o_part + (row0 * S + j0) * kDim, (size_t)S * kDim, a.lse_part + row0 * S + j0, S,
                  min(kMergeFan, Sb - j0), warp, lane, nullptr, nullptr, a.g_part + (row0 * NG + grp) * kDim,
                  a.g_lse + row0 * NG + grp, NG);
  __threadfence();
  __syncthreads();
  if (tid == 0) {
    const int ngb = (Sb + kMergeFan - 1) / kMergeFan;
    const int last = atomicAdd(&a.counters[unit], 1) == ngb - 1;
    if (last) a.counters[unit] = 0;
    sm.last = last;
  }
  __syncthreads();
  if (!sm.last) return;
  __threadfence();
  merge_splits<G>(a.g_part + row0 * NG * kDim, (size_t)NG * kDim, a.g_lse + row0 * NG, NG,
                  (Sb + kMergeFan - 1) / kMergeFan, warp, lane, a.out + row0 * kDim,
                  a.lse_out ? a.lse_out + row0 : nullptr, nullptr, nullptr, 0);
}

// Largest cluster the decode kernel is launched with (portable size).
constexpr int kMaxCluster = 8;

template <int G>
static cudaError_t launch_decode_g(const DecodeArgs &a, int batch, cudaStream_t stream) {
  const size_t smem = sizeof(DecodeSmem<G>);
  static int configured_dev_mask = 0;  // one bit per device
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 31 && !(configured_dev_mask & (1 << dev))) {
    e = cudaFuncSetAttribute(decode_kernel<G, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem));
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(decode_kernel<G, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    configured_dev_mask |= 1 << dev;
  }
  dim3 grid(a.n_splits, a.hkv, batch);
  if (a.n_splits >= 2 && a.n_splits <= kMaxCluster) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = a.n_splits;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, decode_kernel<G, true>, a);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
  }
  decode_kernel<G, false><<<grid, kThreads, smem, stream>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_decode(const DecodeArgs &a, int group, int batch, cudaStream_t stream) {
  switch (group) {
    case 1: return launch_decode_g<1>(a, batch, stream);
    case 2: return launch_decode_g<2>(a, batch, stream);
    case 3: return launch_decode_g<3>(a, batch, stream);
    case 4: return launch_decode_g<4>(a, batch, stream);
    case 5: return launch_decode_g<5>(a, batch, stream);
    case 6: return launch_decode_g<6>(a, batch, stream);
    case 7: return launch_decode_g<7>(a, batch, stream);
    case 8: return launch_decode_g<8>(a, batch, stream);
    default: return cudaErrorInvalidValue;
  }
}

int decode_max_cluster() { return kMaxCluster; }

int decode_max_split_blocks() { return kMaxSplitBlocks; }

// CTAs of the decode kernel one SM holds at once for this head group (0 if
// the device cannot be queried).
int decode_ctas_per_sm(int group) {
  static int cached[32][9];  // [device][group], 0 = not yet known
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  if (dev >= 0 && dev < 32 && group >= 1 && group <= 8 && cached[dev][group] > 0)
    return cached[dev][group];
  int n = 0;
  cudaError_t e = cudaErrorInvalidValue;
  switch (group) {
#define HYB_OCC(g)                                                                          \
  case g:                                                                                   \
    e = cudaFuncSetAttribute(decode_kernel<g, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, \
                             static_cast<int>(sizeof(DecodeSmem<g>)));                      \
    if (e == cudaSuccess)                                                                   \
      e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, decode_kernel<g, false>, kThreads, \
                                                        sizeof(DecodeSmem<g>));             \
    break;
    HYB_OCC(1) HYB_OCC(2) HYB_OCC(3) HYB_OCC(4) HYB_OCC(5) HYB_OCC(6) HYB_OCC(7) HYB_OCC(8)
#undef HYB_OCC
    default: break;
  }
  if (e != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  if (dev >= 0 && dev < 32 && group >= 1 && group <= 8) cached[dev][group] = n;
  return n;
}

}  // namespace hyb
