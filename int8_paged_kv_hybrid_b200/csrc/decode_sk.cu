// decode_sk.cu -- hyb_decode_attn / hyb_decode_step for batches whose splits
// do not fit in one wave of CTAs: a persistent kernel with a stream-K
// schedule.  Same arithmetic as decode.cu (web page "DeepSeek
// V4混合式KV Cache推理优化实战解析", section 4.2: attention over the FP16 hot
// zone plus the dequantized cold zone, merged by log-sum-exp).
//
// Work: each (sequence, kv head) unit is a row of positions, one per cold
// block, the last one also holding the hot ring (so that the fused step's
// seal of the tail block and its write of the ring stay in one CTA); an
// empty sequence has one position with nothing to read.  Units are laid end
// to end (sequence-major, then kv head) and the grid -- as many CTAs as fit
// on the GPU at once -- cuts the row into equal contiguous ranges: CTA c
// takes positions [ceil(cT/grid), ceil((c+1)T/grid)).  Every CTA therefore
// reads the same number of cold blocks whatever the length mix.
//
// A piece is the part of a split (split_blocks positions of a unit) inside
// one CTA's range.  Piece (split sigma, CTA c) writes its partial result to
// slot sigma + c (distinct for all pieces; the pieces of a split have
// consecutive slots).  The last piece of a split to finish merges the split
// into the slot of its first piece; the last split of a unit to finish merges
// the unit (in groups of kMergeFan splits first when there are more) and
// writes the FP16 output.  A unit that is one piece writes its output
// directly.
//
// Pipeline: as in decode.cu, thread 0 brings items (a cold block's K+V tiles,
// or the hot ring) into a 3-stage shared-memory ring with 1-D bulk copies
// (no cluster multicast); it runs across piece and unit boundaries.  The
// block-table entries and scales of the CTA's positions are read ahead into
// a shared-memory table, 128 positions at a time.  Every wait is bounded.
#include "decode_dev.cuh"

namespace hyb {

constexpr int kSkMaxBatch = 256;  // sequence table in shared memory
constexpr int kTbl = 128;         // positions described per table fill (one per thread)
constexpr int kItemRing = 512;    // item descriptors held (two fills of at most 256 items)
// item kinds (low 2 bits of a descriptor's meta word; the byte count above)
constexpr int kItemNone = 0;   // cold block with an invalid block-table entry: nothing to read
constexpr int kItemCold8 = 1;  // INT8 cold block: K + V tiles, 16 KB
constexpr int kItemCold4 = 2;  // INT4 cold block: two 4 KB halves
constexpr int kItemHot = 3;    // hot ring: meta >> 2 bytes

template <int G>
struct SkSmem {
  static constexpr int P = pow2_heads<G>();
  alignas(128) uint8_t ring[kStages][kTilePairBytes];
  uint64_t full[kStages];   // data of the stage landed (TMA transaction count)
  uint64_t empty[kStages];  // every warp is done with the stage
  // descriptors of the CTA's items (item i at i % kItemRing), filled ahead of
  // the producer by all threads: cold block -> its tile phys * Hkv + h, hot
  // ring -> b * Hkv + h; kind and bytes; cold block scales
  int32_t isrc[kItemRing];
  int32_t imeta[kItemRing];
  float2 iscl[kItemRing];
  int n_loaded;  // items described so far
  int32_t seq_L[kSkMaxBatch];     // attended length (after this call's append; 0 if skipped)
  int32_t seq_Lold[kSkMaxBatch];  // length before the append
  int8_t seq_app[kSkMaxBatch];    // tokens appended by this call (0 or 1)
  int32_t pos0[kSkMaxBatch + 1];  // first position of each sequence
  int32_t spl0[kSkMaxBatch + 1];  // first split of each sequence
  alignas(16) float qf[P][kDim];
  alignas(16) int16_t qi[P][kDim];
  float sq[P];
  alignas(16) uint16_t pcode[kWarps][G][16];
  alignas(16) float phot[kWarps][G][8];
  alignas(16) float mbuf[kWarps][G][kDim];
  float mrun[kWarps][G];
  float lrun[kWarps][G];
  SealScratch seal;
  int scan[2][kWarps];
  int flag;
  int abort_flag;
};

// Positions of one unit of a sequence of attended length L.
__device__ __forceinline__ int sk_npos(int L) {
  const int nblk = (max(0, L - kHot) + kBlock - 1) / kBlock;
  return max(1, nblk);
}

template <int G>
__global__ void __launch_bounds__(kThreads, (G <= 4 ? 3 : 2)) decode_sk_kernel(const DecodeArgs a) {
  constexpr int P = pow2_heads<G>();
  extern __shared__ __align__(128) uint8_t smem_raw[];
  SkSmem<G> &sm = *reinterpret_cast<SkSmem<G> *>(smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int B = a.batch, hkv = a.hkv, tb = a.split_blocks;
  const long long cta = blockIdx.x;

  if (tid == 0) {
#pragma unroll
    for (int st = 0; st < kStages; st++) {
      mbar_init(&sm.full[st], 1);
      mbar_init(&sm.empty[st], kWarps);
    }
    sm.abort_flag = 0;
    mbar_fence_init();
  }

  // ---------------- sequence table: lengths, positions and splits (prefix sums) ----------------
  {
    int carry_p = 0, carry_s = 0;
    for (int b0 = 0; b0 < B; b0 += kThreads) {
      const int b = b0 + tid;
      int np = 0, ns = 0;
      if (b < B) {
        const int L_old = a.seq_lens[b];
        int n_app = a.n_new ? a.n_new[b] : 0;
        if (n_app < 0 || n_app > 1) {
          if (cta == 0) set_status(a.status, HYB_STATUS_BAD_N_NEW);
          n_app = 0;
        }
        int L = L_old + n_app;
        if (L_old < 0 || L > a.max_seq_len) {
          // sequence skipped: treated as empty (zero output, lse -inf), not appended to
          if (cta == 0) set_status(a.status, HYB_STATUS_SEQ_LEN);
          L = 0;
          n_app = 0;
        }
        sm.seq_L[b] = L;
        sm.seq_Lold[b] = L_old;
        sm.seq_app[b] = static_cast<int8_t>(n_app);
        const int nb = sk_npos(L);
        np = hkv * nb;
        ns = hkv * ((nb + tb - 1) / tb);
      }
      // exclusive block scan of (np, ns)
      int ip = np, is = ns;
#pragma unroll
      for (int d = 1; d < 32; d <<= 1) {
        const int tp = __shfl_up_sync(0xffffffffu, ip, d), ts = __shfl_up_sync(0xffffffffu, is, d);
        if (lane >= d) {
          ip += tp;
          is += ts;
        }
      }
      if (lane == 31) {
        sm.scan[0][warp] = ip;
        sm.scan[1][warp] = is;
      }
      __syncthreads();
      int wp = 0, wsum = 0, tot_p = 0, tot_s = 0;
#pragma unroll
      for (int w = 0; w < kWarps; w++) {
        if (w < warp) {
          wp += sm.scan[0][w];
          wsum += sm.scan[1][w];
        }
        tot_p += sm.scan[0][w];
        tot_s += sm.scan[1][w];
      }
      if (b < B) {
        sm.pos0[b] = carry_p + wp + ip - np;
        sm.spl0[b] = carry_s + wsum + is - ns;
      }
      carry_p += tot_p;
      carry_s += tot_s;
      __syncthreads();
    }
    if (tid == 0) {
      sm.pos0[B] = carry_p;
      sm.spl0[B] = carry_s;
    }
  }
  __syncthreads();
  // fused step: once every CTA has read the lengths, the last one advances them
  if (a.n_new) {
    if (tid == 0) {
      const int ticket = atomicAdd(&a.seq_cnt[0], 1);
      sm.flag = ticket == static_cast<int>(gridDim.x) - 1;
      if (sm.flag) a.seq_cnt[0] = 0;
    }
    __syncthreads();
    if (sm.flag)
      for (int b = tid; b < B; b += kThreads) a.seq_lens[b] = sm.seq_Lold[b] + sm.seq_app[b];
  }

  // CTAs beyond the number of positions get no range, so that every CTA in
  // [0, grid) owns at least one position (a split's pieces are then exactly
  // the CTAs from the owner of its first position to that of its last)
  const long long T = sm.pos0[B];
  const long long grid = min(static_cast<long long>(gridDim.x), T);
  const int lo = cta < grid ? static_cast<int>((cta * T + grid - 1) / grid) : 0;
  const int hi = cta < grid ? static_cast<int>(((cta + 1) * T + grid - 1) / grid) : 0;
  auto cta_of = [&](int g) { return static_cast<int>((static_cast<long long>(g) * grid) / T); };
  // sequence holding position g
  auto seq_of = [&](int g) {
    int l = 0, r = B - 1;
    while (l < r) {
      const int m = (l + r + 1) >> 1;
      if (sm.pos0[m] <= g) l = m;
      else r = m - 1;
    }
    return l;
  };
  // Describe the items of positions lo + 128m + tid (a cold block and/or the
  // hot ring each), numbered on from the items described so far.
  auto fill = [&](int m) {
    const int g = lo + m * kTbl + tid;
    int src0 = -1, meta0 = kItemNone, src1 = 0, meta1 = 0, cnt = 0;
    float2 sc = make_float2(0.f, 0.f);
    if (g < hi) {
      const int b = seq_of(g);
      const int L = sm.seq_L[b];
      const int nb = sk_npos(L);
      const int off = g - sm.pos0[b];
      const int h = off / nb, j = off - h * nb;
      const int nblk = (max(0, L - kHot) + kBlock - 1) / kBlock;
      if (j < nblk) {
        const int phys = j < a.max_blocks ? a.block_table[(size_t)b * a.max_blocks + j] : -1;
        const int n_int4_b = a.quant_bits == 4 ? 0x7fffffff : (a.n_int4 ? a.n_int4[b] : 0);
        if (phys < 0 || phys >= a.num_phys) {
          set_status(a.status, HYB_STATUS_BAD_BLOCK);
        } else {
          src0 = phys * hkv + h;
          meta0 = j < n_int4_b ? kItemCold4 : kItemCold8;
          sc = __ldg(reinterpret_cast<const float2 *>(a.scales + (size_t)src0 * 2));
        }
        cnt = 1;
      }
      if (j == nb - 1 && L > 0) {
        const int hot_src = b * hkv + h, hot_meta = kItemHot | ((min(L, kHot) * kHotTokenBytes) << 2);
        if (cnt == 0) {
          src0 = hot_src;
          meta0 = hot_meta;
        } else {
          src1 = hot_src;
          meta1 = hot_meta;
        }
        cnt++;
      }
    }
    // number the items: exclusive scan of cnt over the CTA
    int x = cnt;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, x, d);
      if (lane >= d) x += t;
    }
    if (lane == 31) sm.scan[0][warp] = x;
    __syncthreads();
    int base = sm.n_loaded, total = 0;
#pragma unroll
    for (int w = 0; w < kWarps; w++) {
      if (w < warp) base += sm.scan[0][w];
      total += sm.scan[0][w];
    }
    base += x - cnt;
    if (cnt > 0) {
      const int k0 = base % kItemRing;
      sm.isrc[k0] = src0;
      sm.imeta[k0] = meta0;
      sm.iscl[k0] = sc;
    }
    if (cnt > 1) {
      const int k1 = (base + 1) % kItemRing;
      sm.isrc[k1] = src1;
      sm.imeta[k1] = meta1;
    }
    __syncthreads();
    if (tid == 0) sm.n_loaded += total;
    __syncthreads();
  };
  if (tid == 0) sm.n_loaded = 0;
  __syncthreads();
  fill(0);
  if (hi - lo > kTbl) fill(1);

  const uint64_t pol = l2_policy_evict_first();
  // ---------------- producer (thread 0) ----------------
  // Issue described items while fewer than kStages are ahead of consumer item
  // `it`; items up to must_until are waited for if their stage is still busy.
  int p_it = 0;  // items issued (thread 0)
  auto produce = [&](int it, int must_until) {
    const int lim = min(it + kStages, sm.n_loaded);
    for (; p_it < lim; p_it++) {
      const int j = p_it - kStages;  // previous item of that stage
      if (j >= 0) {
        if (p_it <= must_until) {
          if (!mbar_wait_bounded(&sm.empty[j % kStages], (j / kStages) & 1, kWaitCycles)) {
            set_status(a.status, HYB_STATUS_TIMEOUT);
            sm.abort_flag = 1;
            break;
          }
        } else if (!mbar_try_wait(&sm.empty[j % kStages], (j / kStages) & 1)) {
          break;
        }
      }
      const int st = p_it % kStages;
      const int slot = p_it % kItemRing;
      const int src = sm.isrc[slot], meta = sm.imeta[slot];
      uint8_t *dst = sm.ring[st];
      const int kind = meta & 3;
      if (kind == kItemCold8) {
        mbar_arrive_expect_tx(&sm.full[st], kTilePairBytes);
        bulk_g2s(dst, a.cold + (size_t)src * kTilePairBytes, kTilePairBytes, &sm.full[st], pol);
      } else if (kind == kItemCold4) {
        const uint8_t *g = a.cold + (size_t)src * kTilePairBytes;
        mbar_arrive_expect_tx(&sm.full[st], kTileBytes);
        bulk_g2s(dst, g, kTileBytes / 2, &sm.full[st], pol);
        bulk_g2s(dst + kTileBytes, g + kTileBytes, kTileBytes / 2, &sm.full[st], pol);
      } else if (kind == kItemHot) {
        const uint32_t bytes = static_cast<uint32_t>(meta) >> 2;
        mbar_arrive_expect_tx(&sm.full[st], bytes);
        bulk_g2s(dst, a.hot + (size_t)src * kHotBytes, bytes, &sm.full[st], pol);
      } else {
        mbar_arrive(&sm.full[st]);
      }
    }
  };
  if (tid == 0) produce(0, -1);  // the first items go out before q is prepared

  // ---------------- consumers ----------------
  const int tg = lane >> 3, cs = lane & 7;
  const int hx = head_xor<P>(lane);
  const bool owner = (lane & (8 / P - 1)) == 0 && hx < G;
  const int k_lane = (16 * warp + 4 * tg) * kDim + 16 * cs;
  const int v_lane = kTileBytes + lane * kBlock + 16 * (warp ^ ((lane >> 1) & 3));
  uint32_t qp[P][8];
  float sq_hd = 0.f;
  int it = 0;  // items consumed
  bool aborted = false;

  int g = lo;
  int b = 0, h = 0, j = 0;
  if (lo < hi) {
    b = seq_of(lo);
    const int off = lo - sm.pos0[b];
    const int nb = sk_npos(sm.seq_L[b]);
    h = off / nb;
    j = off - h * nb;
  }
  int q_unit = -1;  // unit whose q is loaded
  while (g < hi && !aborted) {
    const int L = sm.seq_L[b];
    const int nb = sk_npos(L);
    const int nblk = (max(0, L - kHot) + kBlock - 1) / kBlock;
    const int Lc = max(0, L - kHot);
    const int Su = (nb + tb - 1) / tb;
    const int s = j / tb;
    const int unit_g0 = sm.pos0[b] + h * nb;
    const int split_g0 = unit_g0 + s * tb;
    const int split_g1 = unit_g0 + min(nb, (s + 1) * tb);
    const int g_end = min(hi, split_g1);
    const int unit = b * hkv + h;
    const int hq0 = h * G;
    const size_t row0 = (size_t)b * a.hq + hq0;

    if (unit != q_unit) {
      // q of this unit: FP32 (hot ring) and 16-bit fixed point (cold blocks)
      float qv[G];
#pragma unroll
      for (int jj = 0; jj < G; jj++) qv[jj] = __half2float(a.q[(row0 + jj) * kDim + tid]);
      __syncthreads();  // the previous unit's q is no longer read
#pragma unroll
      for (int jj = 0; jj < P; jj++) sm.qf[jj][tid] = jj < G ? qv[jj] : 0.f;
      __syncthreads();
      quantize_q<P>(sm.qf, sm.qi, sm.sq, warp, lane);
      __syncthreads();
      load_qp<P>(sm.qi, hx, cs, qp);
      sq_hd = sm.sq[hx];
      q_unit = unit;
    }
    // fused step: the unit's new token goes to ring slot L_old % 32, its old
    // occupant (position L_old - 32) into the tail block first
    const int L_old = sm.seq_Lold[b];
    const bool do_ring = sm.seq_app[b] == 1 && L > 0;
    const bool do_seal = do_ring && L_old >= kHot;
    __half2 new_kv = __halves2half2(__float2half_rn(0.f), __float2half_rn(0.f));
    if (do_ring && g_end == split_g1 && split_g1 == unit_g0 + nb) {
      const size_t o = ((size_t)b * hkv + h) * kDim + tid;
      new_kv = __halves2half2(a.k_new[o], a.v_new[o]);
    }
    const int n_int4_b = a.quant_bits == 4 ? 0x7fffffff : (a.n_int4 ? a.n_int4[b] : 0);

    float m_run[G], acc[G][4];
#pragma unroll
    for (int hh = 0; hh < G; hh++) {
      m_run[hh] = -INFINITY;
#pragma unroll
      for (int kk = 0; kk < 4; kk++) acc[hh][kk] = 0.f;
    }
    float m_hx = hx < G ? -INFINITY : INFINITY;
    float l_lane = 0.f;
    int psum_lane = 0;

    for (; g < g_end; g++, j++) {
      const int rel = g - lo;
      if (rel % kTbl == 0 && rel >= kTbl) {
        // entering table chunk m: chunk m + 1 into the buffer chunk m - 1 used
        __syncthreads();
        fill(rel / kTbl + 1);
        __syncthreads();
      }
      const bool has_cold = j < nblk, has_hot = j == nb - 1 && L > 0;
      for (int part = 0; part < 2; part++) {
        if (part == 0 && !has_cold) continue;
        if (part == 1 && !has_hot) break;
        const bool fuse_here = do_ring && has_hot && (do_seal ? part == 0 : part == 1);
        if (tid == 0) produce(it, it + (fuse_here && part == 0 ? 1 : 0));
        const int st = it % kStages;
        bool ok = *reinterpret_cast<volatile int *>(&sm.abort_flag) == 0;
        ok = ok && mbar_wait_bounded(&sm.full[st], (it / kStages) & 1, kWaitCycles);
        if (fuse_here) {
          const int ih = it + (part == 0 ? 1 : 0);  // the hot item
          if (ih != it) ok = ok && mbar_wait_bounded(&sm.full[ih % kStages], (ih / kStages) & 1, kWaitCycles);
          ok = __syncthreads_and(ok) != 0;
          if (ok) {
            const int slot = it % kItemRing;  // the tail block (when sealing)
            fused_append(sm.seal, sm.ring[ih % kStages], sm.ring[it % kStages], &sm.iscl[slot], sm.isrc[slot],
                         do_seal && j < n_int4_b, a, b, h, L_old, do_seal, new_kv, tid, warp, lane);
          }
        }
        if (!ok) {
          if (lane == 0) set_status(a.status, HYB_STATUS_TIMEOUT);
          sm.abort_flag = 1;
        } else {
          const uint8_t *stage = sm.ring[st];
          if (part == 0) {
            const int slot = it % kItemRing;
            const int kind = sm.imeta[slot] & 3;
            const int nvalid = kind == kItemNone ? 0 : min(kBlock, Lc - j * kBlock);
            const int nv = nvalid - 16 * warp;
            const bool int4 = kind == kItemCold4;
            const float2 sc = sm.iscl[slot];
            const float coef = sq_hd * sc.x * a.qk_scale;
            if (nvalid == kBlock && !int4) {
              cold_block_full<G, P>(stage, k_lane, v_lane, qp, coef, sc.y * (1.f / 32767.f), sm.pcode[warp], hx,
                                    tg, owner, m_run, acc, m_hx, l_lane, psum_lane);
            } else if (nv > 0) {
              cold_block_general<G, P>(stage, nv, int4, warp, lane, tg, cs, qp, coef, sc.y * (1.f / 32767.f),
                                       sm.pcode[warp], hx, owner, m_run, acc, m_hx, l_lane, psum_lane);
            }
          } else {
            hot_item<G, P>(stage, min(L, kHot), warp, lane, tg, cs, sm.qf, a.qk_scale, sm.phot[warp], hx, owner,
                           m_run, acc, m_hx, l_lane, psum_lane);
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.empty[st]);
        it++;
      }
    }
    // ---------------- end of the piece ----------------
    aborted = __syncthreads_or(*reinterpret_cast<volatile int *>(&sm.abort_flag) != 0) != 0;
    if (aborted) break;
    float o_s[G], lse2_s[G];
    merge_warps<G, P>(&sm.mbuf[0][0][0], sm.mrun, sm.lrun, m_run, acc, l_lane, psum_lane, warp, lane, tid, o_s,
                      lse2_s);
    const int c_first = cta_of(split_g0), c_last = cta_of(split_g1 - 1);
    const long long sigma = sm.spl0[b] + static_cast<long long>(h) * Su + s;  // global split index
    const int gstride = G * kDim;
    auto write_out = [&]() {
#pragma unroll
      for (int hh = 0; hh < G; hh++) {
        a.out[(row0 + hh) * kDim + tid] = __float2half_rn(o_s[hh]);
        if (tid == 0 && a.lse_out) a.lse_out[row0 + hh] = lse2_s[hh] * kLn2;
      }
    };
    auto write_slot = [&](long long slot) {
#pragma unroll
      for (int hh = 0; hh < G; hh++) {
        a.o_part[slot * gstride + hh * kDim + tid] = o_s[hh];
        if (tid == 0) a.lse_part[slot * G + hh] = lse2_s[hh];
      }
    };
    // arrival on a counter by the whole CTA (its writes published first);
    // true in every thread of the CTA that completes the count
    auto arrive = [&](int32_t *cnt, int need) {
      __threadfence();
      __syncthreads();
      if (tid == 0) {
        const int last = atomicAdd(cnt, 1) == need - 1;
        if (last) *cnt = 0;  // ready for the next call
        sm.flag = last;
      }
      __syncthreads();
      const bool last = sm.flag != 0;
      if (last) __threadfence();
      return last;
    };
    bool unit_ready = false;  // the split's result is in slot sigma + c_first
    if (c_first == c_last) {
      if (Su == 1) {
        write_out();
      } else {
        write_slot(sigma + c_first);
        unit_ready = true;
      }
    } else {
      write_slot(sigma + cta);
      if (arrive(&a.sk_split_cnt[sigma], c_last - c_first + 1)) {
        const long long s0 = sigma + c_first;
        if (Su == 1) {
          merge_splits<G>(a.o_part, gstride, kDim, a.lse_part, G, 1, c_last - c_first + 1,
                          [s0](int jj) { return s0 + jj; }, warp, lane, a.out + row0 * kDim,
                          a.lse_out ? a.lse_out + row0 : nullptr, nullptr, 0, nullptr, 0);
        } else {
          merge_splits<G>(a.o_part, gstride, kDim, a.lse_part, G, 1, c_last - c_first + 1,
                          [s0](int jj) { return s0 + jj; }, warp, lane, nullptr, nullptr,
                          a.o_part + s0 * gstride, kDim, a.lse_part + s0 * G, 1);
          unit_ready = true;
        }
      }
    }
    if (unit_ready) {
      // split results of the unit: split k's is in slot spl + k + cta_of(its first position)
      const long long spl = sm.spl0[b] + static_cast<long long>(h) * Su;
      auto split_slot = [&](int k) {
        return spl + k + static_cast<long long>(cta_of(unit_g0 + k * tb));
      };
      if (Su <= kMergeFan) {
        if (arrive(&a.counters[unit], Su))
          merge_splits<G>(a.o_part, gstride, kDim, a.lse_part, G, 1, Su, split_slot, warp, lane,
                          a.out + row0 * kDim, a.lse_out ? a.lse_out + row0 : nullptr, nullptr, 0, nullptr, 0);
      } else {
        const int NG = a.n_groups;
        const int grp = s / kMergeFan, k0 = grp * kMergeFan;
        const int ngu = (Su + kMergeFan - 1) / kMergeFan;
        if (arrive(&a.g_counters[(size_t)unit * NG + grp], min(kMergeFan, Su - k0))) {
          const long long gslot = (long long)unit * NG + grp;
          merge_splits<G>(a.o_part, gstride, kDim, a.lse_part, G, 1, min(kMergeFan, Su - k0),
                          [&](int k) { return split_slot(k0 + k); }, warp, lane, nullptr, nullptr,
                          a.g_part + gslot * gstride, kDim, a.g_lse + gslot * G, 1);
          if (arrive(&a.counters[unit], ngu)) {
            const long long gs0 = (long long)unit * NG;
            merge_splits<G>(a.g_part, gstride, kDim, a.g_lse, G, 1, ngu, [gs0](int k) { return gs0 + k; }, warp,
                            lane, a.out + row0 * kDim, a.lse_out ? a.lse_out + row0 : nullptr, nullptr, 0, nullptr,
                            0);
          }
        }
      }
    }
    // next piece
    if (j == nb) {
      j = 0;
      if (++h == hkv) {
        h = 0;
        b++;
      }
    }
  }
  if (aborted) {
    // let every copy still in flight land before the CTA's shared memory is released
    __syncthreads();
    if (tid == 0)
      for (int k = it; k < p_it; k++) (void)mbar_wait_bounded(&sm.full[k % kStages], (k / kStages) & 1, kWaitCycles);
    __syncthreads();
  }
}

template <int G>
static cudaError_t launch_sk_g(const DecodeArgs &a, int grid, cudaStream_t stream) {
  const size_t smem = sizeof(SkSmem<G>);
  static int configured_dev_mask = 0;  // one bit per device
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 31 && !(configured_dev_mask & (1 << dev))) {
    e = cudaFuncSetAttribute(decode_sk_kernel<G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    configured_dev_mask |= 1 << dev;
  }
  decode_sk_kernel<G><<<grid, kThreads, smem, stream>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_decode_sk(const DecodeArgs &a, int group, int grid, cudaStream_t stream) {
  switch (group) {
    case 1: return launch_sk_g<1>(a, grid, stream);
    case 2: return launch_sk_g<2>(a, grid, stream);
    case 3: return launch_sk_g<3>(a, grid, stream);
    case 4: return launch_sk_g<4>(a, grid, stream);
    case 5: return launch_sk_g<5>(a, grid, stream);
    case 6: return launch_sk_g<6>(a, grid, stream);
    case 7: return launch_sk_g<7>(a, grid, stream);
    case 8: return launch_sk_g<8>(a, grid, stream);
    default: return cudaErrorInvalidValue;
  }
}

int decode_sk_max_batch() { return kSkMaxBatch; }

// CTAs of the persistent kernel one SM holds at once (0 if unknown).
int decode_sk_ctas_per_sm(int group) {
  static int cached[32][9];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  if (dev >= 0 && dev < 32 && group >= 1 && group <= 8 && cached[dev][group] > 0) return cached[dev][group];
  int n = 0;
  cudaError_t e = cudaErrorInvalidValue;
  switch (group) {
#define HYB_SK_OCC(g)                                                                             \
  case g:                                                                                         \
    e = cudaFuncSetAttribute(decode_sk_kernel<g>, cudaFuncAttributeMaxDynamicSharedMemorySize,    \
                             static_cast<int>(sizeof(SkSmem<g>)));                                \
    if (e == cudaSuccess)                                                                         \
      e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, decode_sk_kernel<g>, kThreads,        \
                                                        sizeof(SkSmem<g>));                       \
    break;
    HYB_SK_OCC(1) HYB_SK_OCC(2) HYB_SK_OCC(3) HYB_SK_OCC(4) HYB_SK_OCC(5) HYB_SK_OCC(6) HYB_SK_OCC(7)
    HYB_SK_OCC(8)
#undef HYB_SK_OCC
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
