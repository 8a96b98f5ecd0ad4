// decode_kernel.cuh -- hyb_decode_attn: split-KV single-query attention over the
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
// the sequence's last cold block also attends the hot ring.  Pipeline items:
// a 64-token sub-block of a cold block (K tile 8 KB + V tile 8 KB, or 4 + 4
// KB for INT4; a 128-token block is two, a 32-token block the first half of
// one), 32 FP16 rows (16 KB) of an FP16 cold block, and 32 rows of the hot
// ring.  Each item is brought into a 3-stage shared-memory ring by the TMA
// engine with 1-D bulk copies (no cluster multicast) completing on an
// mbarrier; every wait is bounded.  Three CTAs fit on an SM for up to 4 query
// heads per kv head (two above that).  When all splits are resident at once
// (one wave) 2..8 splits of a (sequence, kv head) run as one thread-block
// cluster and merge through distributed shared memory; otherwise the last
// split to finish merges them from the workspace.
//
// Arithmetic (per kv head, for its G = Hq/Hkv query heads), on the tensor
// cores with warp-level mma.sync (decode_dev.cuh has the fragment layouts):
//  * q is turned into 24-bit fixed point per query head (q_i = rint(q *
//    127 * 65536 / max|q|)), held as three signed base-256 digits; a cold
//    logit is the exact integer dot product of q_i with the K codes (int8
//    mma, one A row per digit, joined in the lane pair that holds them),
//    times max|q| / (127 * 65536) * K-scale * softmax_scale * log2(e).
//  * Warp w owns tokens 16w..16w+15 of every 64-token sub-block.  Its
//    softmax weights are 16-bit fixed point relative to the maximum of their
//    16-token group (p_i = rint(65535 * 2^(z - group max))); P.V is an exact
//    int8 x uint8 mma of the V codes with the weights' high and low bytes,
//    folded into the warp's FP32 online-softmax state (per head: running max,
//    sum, output) with the V scale and 2^(group max - running max).
//  * FP16 rows (hot ring, FP16 cold blocks) go through f16 mma with FP32
//    accumulation on the FP16 q, K and V, weights in FP16 relative to the
//    8-row group's maximum.
//  * The 4 warp states are merged in FP32 at the end of the split; the last
//    CTA of a (sequence, kv head) to finish merges the splits (log-sum-exp)
//    and writes the FP16 output.
// Per KV byte the work is small (a GEMV per kv head); the tensor cores take
// the integer dot products so that the loop keeps up with HBM.
#pragma once

#include "decode_dev.cuh"

namespace hyb {

constexpr int kMaxSplitBlocks = 128;  // == kThreads: one block-table entry per thread

template <int G>
struct DecodeSmem {
  static constexpr int NT = head_quads<G>();  // head quads
  static constexpr int NH = 4 * NT;           // head slots (heads >= G are zero)
  alignas(128) uint8_t ring[kStages][kStageBytes];
  uint64_t full[kStages];   // data of the stage landed (TMA transaction count)
  uint64_t empty[kStages];  // every warp is done with the stage
  int32_t phys[kMaxSplitBlocks];
  float2 scl[kMaxSplitBlocks];  // (K scale, V scale) of each block of the split
  alignas(16) int8_t qd[NH][3][kDim];  // q in 24-bit fixed point: hi, mid, lo digits
  alignas(16) __half qh[NH][kDim];     // q in FP16 (FP16 rows)
  float sq[NH];                        // fixed-point step of each head's q
  float qmax_w[kWarps][NH];
  float mrun[kWarps][NH];
  float lrun[kWarps][NH];
  SealScratch seal;  // fused step
  float cl_l[G];     // this split's log2-sum-exp per head, read by the cluster's merge
  alignas(16) uint32_t zero16[4];  // a zero 16-byte row for masked FP16 rows
  int rel_cnt[kStages];  // warps done with the stage's current item
  int issued;            // items issued so far (in order)
  int last;
  int abort_flag;
};

// kCluster: the grid is launched in clusters of n_splits CTAs (the splits of
// one (sequence, kv head)); splits are merged through distributed shared
// memory instead of the workspace.  kF16: FP16 cold blocks (quantization_bits
// 0), each attended as two items of 32 rows with the hot ring's arithmetic.
// kSkip: sparse L2 mode -- the sequence's INT4 ("L2") blocks are left to the
// top-k kernels, and the splits cover the blocks from its INT4 count on.
// kBshift: log2 of the tokens per block (block_size 32: 5, 64: 6, 128: 7); a
// 128-token block is two 64-token sub-blocks, a 32-token block the first half
// of one.
template <int G, bool kCluster, bool kF16, bool kSkip, int kBshift>
__global__ void __launch_bounds__(kThreads, (G <= 4 ? 4 : 3)) decode_kernel(const DecodeArgs a) {
  constexpr int NT = head_quads<G>();
  constexpr int NH = 4 * NT;
  extern __shared__ __align__(128) uint8_t smem_raw[];
  DecodeSmem<G> &sm = *reinterpret_cast<DecodeSmem<G> *>(smem_raw);

  const int s = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int S = a.n_splits;
  const int hq0 = h * G;
  int ib = 0;  // first block of the splits
  if constexpr (kSkip) {
    const int n4 = a.quant_bits == 4 ? a.max_blocks : (a.n_int4 ? a.n_int4[b] : 0);
    ib = min(max(n4, 0), a.max_blocks);
  }
  const int i0 = ib + s * a.split_blocks;

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
  const int H = a.hot_tokens;
  const int Lc = max(0, L - H);
  constexpr int lsub = kBshift > 6 ? kBshift - 6 : 0;  // a block is 1 << lsub sub-blocks
  constexpr int Bt = 1 << kBshift;                      // tokens per block
  constexpr int St = Bt < kBlock ? Bt : kBlock;         // tokens per sub-block
  const int nblk = (Lc + Bt - 1) / Bt;
  constexpr bool fp16 = kF16;
  constexpr int ish = fp16 ? kBshift - 5 : lsub;  // log2 of the items per block
  // Splits of this sequence: runs of split_blocks cold blocks from block ib
  // on; the last split also attends the hot ring, whose items count as
  // (up to split_blocks) blocks when the sequence is cut, so that no split
  // has more than split_blocks blocks' worth of items (the hot ring may then
  // be alone in its split)
  const int nrem = max(0, nblk - ib);
  const int dh = (min(L, H) + kItemRows - 1) / kItemRows;  // hot items
  const int dhb = min((dh + (1 << ish) - 1) >> ish, a.split_blocks);
  const int Sb = max(1, (nrem + dhb + a.split_blocks - 1) / a.split_blocks);
  // Fused step: the last CTA of the sequence advances seq_lens[b].  A CTA
  // takes its ticket only after a barrier that follows every one of its
  // threads' reads of seq_lens[b], so the CTA holding the last ticket writes
  // after every CTA of the sequence (itself included) has read the old
  // length.  Until then no CTA can see the new value, so L_old (and every
  // choice made from it, such as the early return below) is the same in all
  // threads of a CTA.
  auto take_ticket = [&]() {
    const int ticket = atomicAdd(&a.seq_cnt[b], 1);
    if (ticket == static_cast<int>(gridDim.x * gridDim.y) - 1) {
      a.seq_lens[b] = L_old + n_app;
      a.seq_cnt[b] = 0;
    }
  };
  // past this sequence's last split: no work and no partial (a cluster member
  // still takes part in the cluster's merge, with an empty state)
  if (!kCluster && s >= Sb) {
    if (a.n_new) {
      __syncthreads();
      if (tid == 32) take_ticket();
    }
    return;
  }
  const int ncold = max(0, min(nblk, i0 + a.split_blocks) - i0);
  // Items: one per 64-token sub-block (16 KB K + V tiles), or per 32 rows of
  // FP16 (the hot ring, FP16 cold blocks: 2 << lsub items per block)
  const bool holds_hot = s == Sb - 1;
  const bool holds_tail = ncold > 0 && i0 + ncold == nblk;  // the sequence's last cold block
  const int nhot = holds_hot ? min(L, H) : 0;
  const int ncold_it = ncold << ish;
  const int kh = ncold_it;  // the first hot item
  const int nitems = ncold_it + (nhot + kItemRows - 1) / kItemRows;
  // Fused step: the new token goes to ring slot rs = L_old % hot, whose old
  // occupant (position L_old - hot) is sealed into the tail block.  The CTA
  // holding the tail block reads that occupant in its prologue, seals it at
  // the tail block's item, and writes the new token into the ring in HBM
  // (after its own read of the slot); the CTA holding the hot ring puts the
  // new token into its staged copy of the slot -- which, if the tail block is
  // in another CTA, may have been copied before or after that write, so the
  // staged put makes both cases the same.  With nothing to seal (L_old <
  // hot), the hot-ring CTA writes the ring in HBM itself.
  const bool do_seal_seq = n_app == 1 && L_old >= H;  // a token leaves the hot zone
  const bool do_seal = do_seal_seq && holds_tail;
  const bool do_ring = n_app == 1 && holds_hot;       // staged put
  const bool ring_hbm = n_app == 1 && (do_seal_seq ? holds_tail : holds_hot);
  const int rs = L_old & (H - 1);
  const int k_ring = kh + rs / kItemRows;
  // slot of the sealed token in the tail block; in the split that seals, the
  // tail block's sub-blocks run last-first, so that a scale the seal grows
  // reaches the earlier sub-block before that one is attended (k_rq)
  const int slot_e = do_seal ? (L_old - H) % Bt : 0;
  const int nsub1 = (1 << lsub) - 1;
  const int k_seal = !do_seal ? -1
                     : fp16   ? ((ncold - 1) << ish) + slot_e / kItemRows
                              : ((ncold - 1) << lsub) + nsub1 - (slot_e >> 6);
  const int k_rq = (!fp16 && do_seal && (slot_e >> 6) > 0) ? ((ncold - 1) << lsub) + nsub1 : -1;
  // item k: its block, and (cold INT8/INT4 items) its sub-block
  auto item_block = [&](int k) { return k >> ish; };
  auto item_sub = [&](int k) {
    const int part = k & ((1 << ish) - 1);
    return (do_seal && (k >> ish) == ncold - 1) ? nsub1 - part : part;
  };
  __half2 new_kv = __halves2half2(__float2half_rn(0.f), __float2half_rn(0.f));
  __half2 old_kv = new_kv;
  if (do_ring || ring_hbm) {
    const size_t o = ((size_t)b * a.hkv + h) * kDim + tid;
    new_kv = __halves2half2(a.k_new[o], a.v_new[o]);
  }
  if (do_seal) {
    const __half *er = reinterpret_cast<const __half *>(a.hot) + (((size_t)b * a.hkv + h) * H + rs) * 2 * kDim;
    old_kv = __halves2half2(er[tid], er[kDim + tid]);
  }
  if (ring_hbm) {
    // the new token into the ring in HBM; thread tid writes channel tid of
    // both rows, after (in program order) its own read of the old occupant
    __half *grow = reinterpret_cast<__half *>(a.hot) + (((size_t)b * a.hkv + h) * H + rs) * 2 * kDim;
    grow[tid] = __low2half(new_kv);
    grow[kDim + tid] = __high2half(new_kv);
  }
  const int n_int4_b = a.quant_bits == 4 ? 0x7fffffff : (a.n_int4 ? a.n_int4[b] : 0);

  if (tid == 0) {
#pragma unroll
    for (int st = 0; st < kStages; st++) {
      mbar_init(&sm.full[st], 1);
      mbar_init(&sm.empty[st], kWarps);
      sm.rel_cnt[st] = 0;
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
  if (tid < 4) sm.zero16[tid] = 0u;
  __syncthreads();

  const uint64_t pol = l2_policy_evict_first();
  auto issue = [&](int k) {
    const int st = k % kStages;
    uint8_t *dst = sm.ring[st];
    if (k < ncold_it) {
      const int kb = item_block(k);
      const int phys = sm.phys[kb];
      const int part = k & ((1 << ish) - 1);
      const int u = fp16 ? 0 : item_sub(k);
      const int nrow = fp16 ? min(kItemRows, Lc - (i0 + kb) * Bt - part * kItemRows)
                            : Lc - (i0 + kb) * Bt - u * kBlock;
      if (phys < 0 || nrow <= 0) {
        mbar_arrive(&sm.full[st]);
        return;
      }
      if (fp16) {
        // up to 32 of the block's sealed rows, one copy per row at the staging pitch
        const uint8_t *src = a.cold + ((size_t)phys * a.hkv + h) * Bt * kHotTokenBytes + part * kItemBytes;
        const int nr = min(nrow, kItemRows);
        mbar_arrive_expect_tx(&sm.full[st], static_cast<uint32_t>(nr) * kHotTokenBytes);
        for (int r = 0; r < nr; r++)
          bulk_g2s(dst + r * kRowStride, src + r * kHotTokenBytes, kHotTokenBytes, &sm.full[st], pol);
        return;
      }
      const uint8_t *src = a.cold + ((((size_t)phys * a.hkv + h) << lsub) + u) * kTilePairBytes;
      if (i0 + kb >= n_int4_b) {
        if constexpr (St == kBlock) {
          mbar_arrive_expect_tx(&sm.full[st], kTilePairBytes);
          bulk_g2s(dst, src, kTilePairBytes, &sm.full[st], pol);
        } else {
          // a 32-token block: the K rows it holds, and its V tile (whose
          // rows interleave its slots with the unused ones)
          mbar_arrive_expect_tx(&sm.full[st], St * kDim + kTileBytes);
          bulk_g2s(dst, src, St * kDim, &sm.full[st], pol);
          bulk_g2s(dst + kTileBytes, src + kTileBytes, kTileBytes, &sm.full[st], pol);
        }
      } else {
        mbar_arrive_expect_tx(&sm.full[st], St * kDim / 2 + kTileBytes / 2);
        bulk_g2s(dst, src, St * kDim / 2, &sm.full[st], pol);
        bulk_g2s(dst + kTileBytes, src + kTileBytes, kTileBytes / 2, &sm.full[st], pol);
      }
    } else {
      // hot item j: ring slots 32j .. min(32j + 32, nhot) - 1
      const int j = k - kh;
      const uint8_t *src = a.hot + (((size_t)b * a.hkv + h) * H + j * kItemRows) * kHotTokenBytes;
      const int nr = min(kItemRows, nhot - j * kItemRows);
      mbar_arrive_expect_tx(&sm.full[st], static_cast<uint32_t>(nr) * kHotTokenBytes);
      for (int r = 0; r < nr; r++)
        bulk_g2s(dst + r * kRowStride, src + r * kHotTokenBytes, kHotTokenBytes, &sm.full[st], pol);
    }
  };
  // block scales: requested before the bulk copies so that they do not queue
  // behind them; stored once they arrive (overlapping the copies)
  float2 sc_ld = make_float2(0.f, 0.f);
  if (!fp16 && tid < ncold && sm.phys[tid] >= 0)
    sc_ld = __ldg(reinterpret_cast<const float2 *>(a.scales + ((size_t)sm.phys[tid] * a.hkv + h) * 2));
  if (tid == 0) {
    sm.issued = min(nitems, kStages);
    for (int k = 0; k < sm.issued; k++) issue(k);
  }
  if (tid < ncold) sm.scl[tid] = sc_ld;
  // the sealed token's rows: their load depends on seq_lens[b] (the ring
  // slot), so they are stored only after the copies are on their way; the
  // barriers of the q preparation below publish them before the seal's item
  if (do_seal) {
    sm.seal.erow[tid] = __low2half(old_kv);
    sm.seal.erow[kDim + tid] = __high2half(old_kv);
  }
  // q of the head group in 24-bit fixed point and FP16 (padding heads zero)
  prepare_q<G, NH>(qv, sm.qd, sm.qh, sm.sq, sm.qmax_w, warp, lane, tid);

  const int g = lane >> 2, t = lane & 3;
  uint32_t qa[NT][4][4];  // this lane's QK A fragments
  load_qfrag<NT>(sm.qd, g, t, qa);
  float sqh[NT];  // q step of this lane's score-layout head 4nt + g/2
#pragma unroll
  for (int nt = 0; nt < NT; nt++) sqh[nt] = sm.sq[4 * nt + (g >> 1)];
  const uint32_t psel = (g & 1) ? 0x6420u : 0x7531u;  // low / high byte of a 16-bit weight
  // this lane's ldmatrix row of the INT8 V tile in stage 0: channel lane of
  // the first channel-tile pair, chunk of tokens 16w..16w+15 (swizzled)
  const uint32_t v_lane0 = smem_addr(sm.ring[0]) + kTileBytes + lane * kBlock + 16 * (warp ^ ((lane >> 1) & 3));
  const uint32_t zero_addr = smem_addr(sm.zero16);

  // The sequence-length ticket (every thread read seq_lens[b] before the
  // barrier that follows the block-table loads); taken here so that its round
  // trip overlaps the wait for the first stage
  if (a.n_new && tid == 32) take_ticket();

  // Online-softmax state of this warp (value layout, see decode_dev.cuh)
  WarpState<NT> ws;
  state_init<NT>(ws);

  // Pipeline: item k sits in stage k % kStages.  Each warp releases a stage
  // when it is done with it (mbarrier `empty`, release semantics); the last
  // warp to release it -- elected by a shared counter -- waits on that
  // barrier (already complete, acquire semantics) and issues item k +
  // kStages into the stage at once, whichever warp that is, so that a
  // released stage never waits for one particular warp.  Items are issued in
  // order (the last release of item k precedes that of item k + 1).
  // Once a wait runs out, a warp stops waiting, computing and releasing but
  // still goes through the remaining items, so that every warp passes the
  // same CTA barriers (those of the fused append); no later item is issued.
  bool aborted = false;
  for (int k = 0; k < nitems; k++) {
    const int st = k % kStages;
    aborted = aborted || *reinterpret_cast<volatile int *>(&sm.abort_flag) != 0;
    bool ok = !aborted && mbar_wait_bounded(&sm.full[st], (k / kStages) & 1, a.wait_cycles);
    if (!ok && !aborted && lane == 0) set_status(a.status, HYB_STATUS_TIMEOUT);
    if (k == k_seal || k == k_rq || (do_ring && k == k_ring)) {
      // ---------------- fused append (whole CTA, in the staged copies) ----------------
      ok = __syncthreads_and(ok) != 0;
      const int tb = ncold - 1;  // the tail block
      if (ok && k == k_seal) {
        if (fp16)
          fused_seal_fp16(sm.seal, sm.ring[st], sm.phys[tb] * a.hkv + h, a, L_old, true, tid);
        else
          fused_seal(sm.seal, sm.ring[st], &sm.scl[tb], sm.phys[tb] * a.hkv + h, (i0 + tb) < n_int4_b, a, L_old,
                     true, tid, warp, lane);
      } else if (ok && k == k_rq) {
        if (sm.phys[tb] >= 0)
          requant_staged(sm.seal, sm.ring[st], (sm.phys[tb] * a.hkv + h) << lsub, (i0 + tb) < n_int4_b, a, tid);
      } else if (ok) {
        ring_put(sm.ring[st], rs, new_kv, tid);
      }
    }
    ok = ok && *reinterpret_cast<volatile int *>(&sm.abort_flag) == 0;
    const uint8_t *stage = sm.ring[st];
    // rows of an FP16 item: the hot ring, or half of an FP16 cold block
    int nrow = min(kItemRows, nhot - (k - kh) * kItemRows);
    if (k < ncold_it)
      nrow = !fp16 || sm.phys[item_block(k)] < 0
                 ? 0
                 : min(kItemRows, Lc - (i0 + item_block(k)) * Bt - (k & ((1 << ish) - 1)) * kItemRows);
    if (ok && !fp16 && k < ncold_it) {
      // ---------------- cold sub-block (64 tokens) ----------------
      const int kb = item_block(k);
      const int i = i0 + kb;
      const int nvalid = sm.phys[kb] < 0 ? 0 : min(St, Lc - i * Bt - item_sub(k) * kBlock);
      const int nv = nvalid - 16 * warp;
      const bool int4 = i < n_int4_b;
      const float2 sc = sm.scl[kb];
      const float cf = sc.x * a.qk_scale;
      float coef[NT];
#pragma unroll
      for (int nt = 0; nt < NT; nt++) coef[nt] = sqh[nt] * cf;
      const uint32_t v_lane = v_lane0 + st * kStageBytes;
      if (nvalid == kBlock && !int4) {
        cold_item<NT, false, false>(stage, kBlock, warp, g, t, qa, coef, sc.y, psel, v_lane, ws);
      } else if (nv > 0) {
        if (int4)
          cold_item<NT, true, true>(stage, nvalid, warp, g, t, qa, coef, sc.y, psel, v_lane, ws);
        else
          cold_item<NT, false, true>(stage, nvalid, warp, g, t, qa, coef, sc.y, psel, v_lane, ws);
      }
    } else if (ok && nrow > 0) {
      // ---------------- FP16 rows: hot ring or FP16 cold half block ----------------
      hot_item<NT>(stage, nrow, warp, lane, g, t, sm.qh, a.qk_scale, zero_addr, ws);
    }
    __syncwarp();
    if (!ok) {
      sm.abort_flag = 1;
      aborted = true;
      continue;
    }
    if (lane == 0) {
      mbar_arrive(&sm.empty[st]);
      if (atomicAdd(&sm.rel_cnt[st], 1) == kWarps - 1) {
        sm.rel_cnt[st] = 0;  // no warp touches it again before item k + kStages lands
        const int nk = k + kStages;
        if (nk < nitems && *reinterpret_cast<volatile int *>(&sm.abort_flag) == 0) {
          if (!mbar_wait_bounded(&sm.empty[st], (k / kStages) & 1, a.wait_cycles)) {
            set_status(a.status, HYB_STATUS_TIMEOUT);
            sm.abort_flag = 1;
          } else {
            issue(nk);
            sm.issued = nk + 1;
          }
        }
      }
    }
  }
  aborted = __syncthreads_or(aborted) != 0;
  // this split's normalised output (channel tid) and log2-sum-exp per head
  float o_s[G], lse2_s[G];
  if (aborted) {
    // let every copy still in flight land before the CTA's shared memory is
    // released: the last item issued into each stage
    if (tid == 0) {
      const int issued = *reinterpret_cast<volatile int *>(&sm.issued);
      for (int j = max(0, issued - kStages); j < issued; j++)
        (void)mbar_wait_bounded(&sm.full[j % kStages], (j / kStages) & 1, kWaitCycles);
    }
    __syncthreads();
#pragma unroll
    for (int hh = 0; hh < G; hh++) {
      o_s[hh] = 0.f;
      lse2_s[hh] = -INFINITY;
    }
  } else {
    merge_warps<G, NT>(reinterpret_cast<float *>(&sm.ring[0][0]), sm.mrun, sm.lrun, ws, warp, lane, tid, o_s,
                       lse2_s);
  }
  if constexpr (kCluster) {
    // ---------------- split merge across the cluster (distributed shared memory) ----------------
    float *cl_o = reinterpret_cast<float *>(&sm.ring[0][0]);  // [G][kDim], this split's output
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
  // arrival: the CTA barrier orders every thread's partial stores before
  // thread 0's acquire-release increment, which publishes them; the CTA that
  // completes the count acquires every other CTA's (the merge then reads the
  // partials through L2, __ldcg)
  __syncthreads();
  if (tid == 0) {
    int32_t *cnt = grouped ? &a.g_counters[(size_t)unit * a.n_groups + grp] : &a.counters[unit];
    const int need = grouped ? min(kMergeFan, Sb - grp * kMergeFan) : Sb;
    const int last = atomic_add_acq_rel_gpu(cnt, 1) == need - 1;
    if (last) *cnt = 0;  // ready for the next call
    sm.last = last;
  }
  __syncthreads();
  if (!sm.last) return;
  if (!grouped) {
    merge_splits<G>(a.o_part + row0 * S * kDim, kDim, (size_t)S * kDim, a.lse_part + row0 * S, 1, S, Sb,
                    [](int j) { return j; }, warp, lane, a.out + row0 * kDim, a.lse_out ? a.lse_out + row0 : nullptr,
                    nullptr, 0, nullptr, 0);
    return;
  }
  const int NG = a.n_groups;
  const int j0 = grp * kMergeFan;
  merge_splits<G>(a.o_part + (row0 * S + j0) * kDim, kDim, (size_t)S * kDim, a.lse_part + row0 * S + j0, 1, S,
                  min(kMergeFan, Sb - j0), [](int j) { return j; }, warp, lane, nullptr, nullptr,
                  a.g_part + (row0 * NG + grp) * kDim, (size_t)NG * kDim, a.g_lse + row0 * NG + grp, NG);
  __syncthreads();
  if (tid == 0) {
    const int ngb = (Sb + kMergeFan - 1) / kMergeFan;
    const int last = atomic_add_acq_rel_gpu(&a.counters[unit], 1) == ngb - 1;
    if (last) a.counters[unit] = 0;
    sm.last = last;
  }
  __syncthreads();
  if (!sm.last) return;
  merge_splits<G>(a.g_part + row0 * NG * kDim, kDim, (size_t)NG * kDim, a.g_lse + row0 * NG, 1, NG,
                  (Sb + kMergeFan - 1) / kMergeFan, [](int j) { return j; }, warp, lane, a.out + row0 * kDim,
                  a.lse_out ? a.lse_out + row0 : nullptr, nullptr, 0, nullptr, 0);
}

// Largest cluster the decode kernel is launched with (sizes above 8 are
// non-portable; B200 allows 16).  The split merge reads up to 16 partners.
constexpr int kMaxCluster = 16;

template <int G, bool kF16, bool kSkip, int kBshift>
cudaError_t launch_decode_g(const DecodeArgs &a, int batch, bool cluster, cudaStream_t stream) {
  const size_t smem = sizeof(DecodeSmem<G>);
  static int configured_dev_mask = 0;  // one bit per device (per instantiation)
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 31 && !(configured_dev_mask & (1 << dev))) {
    e = cudaFuncSetAttribute(decode_kernel<G, false, kF16, kSkip, kBshift>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(decode_kernel<G, true, kF16, kSkip, kBshift>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(decode_kernel<G, true, kF16, kSkip, kBshift>,
                               cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
    configured_dev_mask |= 1 << dev;
  }
  dim3 grid(a.n_splits, a.hkv, batch);
  if (cluster && a.n_splits >= 2 && a.n_splits <= kMaxCluster) {
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
    e = cudaLaunchKernelEx(&cfg, decode_kernel<G, true, kF16, kSkip, kBshift>, a);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
  }
  decode_kernel<G, false, kF16, kSkip, kBshift><<<grid, kThreads, smem, stream>>>(a);
  return cudaGetLastError();
}

template <bool kF16, bool kSkip, int kBshift>
cudaError_t launch_decode_f(const DecodeArgs &a, int group, int batch, bool cluster, cudaStream_t stream) {
  switch (group) {
    case 1: return launch_decode_g<1, kF16, kSkip, kBshift>(a, batch, cluster, stream);
    case 2: return launch_decode_g<2, kF16, kSkip, kBshift>(a, batch, cluster, stream);
    case 3: return launch_decode_g<3, kF16, kSkip, kBshift>(a, batch, cluster, stream);
    case 4: return launch_decode_g<4, kF16, kSkip, kBshift>(a, batch, cluster, stream);
    case 5: return launch_decode_g<5, kF16, kSkip, kBshift>(a, batch, cluster, stream);
    case 6: return launch_decode_g<6, kF16, kSkip, kBshift>(a, batch, cluster, stream);
    case 7: return launch_decode_g<7, kF16, kSkip, kBshift>(a, batch, cluster, stream);
    case 8: return launch_decode_g<8, kF16, kSkip, kBshift>(a, batch, cluster, stream);
    default: return cudaErrorInvalidValue;
  }
}


// CTAs of the decode kernel (plain variant) one SM holds at once for head
// group `group` (0 on error).
template <bool kF16, bool kSkip, int kBshift>
int decode_occupancy(int group) {
  int n = 0;
  cudaError_t e = cudaErrorInvalidValue;
  switch (group) {
#define HYB_OCC(gg)                                                                                        \
  case gg:                                                                                                 \
    e = cudaFuncSetAttribute(decode_kernel<gg, false, kF16, kSkip, kBshift>,                               \
                             cudaFuncAttributeMaxDynamicSharedMemorySize,                                 \
                             static_cast<int>(sizeof(DecodeSmem<gg>)));                                    \
    if (e == cudaSuccess)                                                                                  \
      e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, decode_kernel<gg, false, kF16, kSkip, kBshift>, \
                                                        kThreads, sizeof(DecodeSmem<gg>));                 \
    break;
    HYB_OCC(1) HYB_OCC(2) HYB_OCC(3) HYB_OCC(4) HYB_OCC(5) HYB_OCC(6) HYB_OCC(7) HYB_OCC(8)
#undef HYB_OCC
    default: break;
  }
  if (e != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  return n;
}

// How many clusters of `csize` CTAs of the cluster-merge kernel (plain
// variant) can be resident on the device at once, for head group `group`
// (0 on error or when such clusters cannot run).
template <int G, bool kF16, bool kSkip, int kBshift>
int decode_active_clusters_g(int csize) {
  auto kern = decode_kernel<G, true, kF16, kSkip, kBshift>;
  const size_t smem = sizeof(DecodeSmem<G>);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e == cudaSuccess) e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  int n = 0;
  if (e == cudaSuccess) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(csize, 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = csize;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaOccupancyMaxActiveClusters(&n, kern, &cfg);
  }
  if (e != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  return n;
}

template <bool kF16, bool kSkip, int kBshift>
int decode_active_clusters(int group, int csize) {
  switch (group) {
    case 1: return decode_active_clusters_g<1, kF16, kSkip, kBshift>(csize);
    case 2: return decode_active_clusters_g<2, kF16, kSkip, kBshift>(csize);
    case 3: return decode_active_clusters_g<3, kF16, kSkip, kBshift>(csize);
    case 4: return decode_active_clusters_g<4, kF16, kSkip, kBshift>(csize);
    case 5: return decode_active_clusters_g<5, kF16, kSkip, kBshift>(csize);
    case 6: return decode_active_clusters_g<6, kF16, kSkip, kBshift>(csize);
    case 7: return decode_active_clusters_g<7, kF16, kSkip, kBshift>(csize);
    case 8: return decode_active_clusters_g<8, kF16, kSkip, kBshift>(csize);
    default: return 0;
  }
}

}  // namespace hyb
