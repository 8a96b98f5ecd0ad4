// decode_persist.cuh -- persistent, warp-specialized variant of the decode
// kernel (decode_kernel.cuh) for plans whose splits run in several waves:
// 64-token INT8/INT4 cold blocks, attention or fused decode step.
//
// Method: web page "DeepSeek V4混合式KV Cache推理优化实战解析", section 4.2
// (attention over the FP16 hot zone plus the dequantized cold zone, one
// softmax merged by log-sum-exp), section 3.2 (hot zone layout).  The
// per-item arithmetic is the decode kernel's (decode_dev.cuh).
//
// Why: a split is a short piece of work (8-32 blocks).  A CTA that runs one
// split spends a global round trip before its first copy and its epilogue
// with nothing in flight; with thousands of splits that idle share caps the
// copy rate well below HBM.  Here each CTA lives for the whole launch:
//  * warp 4 (producer) takes work units -- one (split, kv head, sequence) --
//    from a global counter, prepares each unit's metadata (block-table
//    entries, block scales, q) in one of two shared-memory slots, and streams
//    the units' items through the copy ring back to back: the next unit's
//    copies are in flight while the consumers finish the current one;
//  * warps 0-3 (consumers) take the units in the same order: q in fixed
//    point, the items (cold_item / hot_item), the fused append where the
//    unit has it, then the unit's epilogue -- the warp merge and the split
//    merge through the workspace -- while the producer keeps the ring full.
// The ring has 4 stages of 16 KB for G <= 4: with copies landing ~2.5 us
// after issue under load and ~0.6 us of arithmetic per item and CTA, 3
// stages left the consumers waiting on most items.  Above G = 4 an item
// takes twice the arithmetic and 3 stages cover the latency; 3 CTAs per SM
// either way (128 registers: 3 CTAs of 5 warps put 4 warps on some SM
// sub-partitions, whose register file holds 16 K).  A stage holds one tile
// pair, or 32 hot rows at a 512-byte pitch.
// The consumers synchronise among themselves with named barriers 1 (all
// four) and 2..4 (pairs, for the warp merge); the producer takes part in no
// CTA barrier after the start.  Every wait is bounded; after a timeout the
// producer hands out the remaining units with no items (their rows end with
// zero output and -inf log-sum-exp through the usual merge) and drains its
// copies before exiting.
#pragma once

#include "decode_dev.cuh"

namespace hyb {

constexpr int kPThreads = kThreads + 32;      // 4 consumer warps + 1 producer warp
constexpr int kPStageBytes = kTilePairBytes;  // one tile pair, or 32 hot rows
constexpr int kPRowPitch = kHotTokenBytes;    // hot rows in a stage
static_assert(kItemRows * kPRowPitch == kPStageBytes, "32 hot rows fill a stage");

template <int G>
struct PersistCfg {
  static constexpr int NT = head_quads<G>();
  static constexpr int NH = 4 * NT;
  static constexpr int kStages = G <= 4 ? 4 : 3;
  static constexpr int kCtasPerSm = 3;
};

// One work unit as the producer hands it to the consumers.
template <int G>
struct PersistMeta {
  static constexpr int NH = PersistCfg<G>::NH;
  int unit;          // -1: no more units for this CTA
  int b, h, s, Sb;   // sequence, kv head, split, splits of the sequence
  int i0, ncold, nhot, nitems, Lc;
  int L_old, n_int4_b;
  // fused step: seal the evicted token here / put the new token into the
  // staged ring / write the new token into the ring in HBM
  int do_seal, do_ring, ring_hbm, pad;
  int32_t phys[kPMaxSplitBlocks];
  float2 scl[kPMaxSplitBlocks];
  // per query head h: kQFix / max|q_h| and its fixed-point step max|q_h| /
  // kQFix (0 for rows >= G or an all-zero q)
  float qinv[NH], qstep[NH];
  alignas(16) __half q[NH][kDim];  // FP16 q of the kv head's query heads, rows >= G zero
};

// A finished unit's split merge, decided one unit later: the arrival
// counter's answer comes back while the next unit runs.
struct PendMerge {
  int b, h, Sb, grp, need, level;  // level 0: all splits; 1: a group of kMergeFan, then the groups
  int32_t *cnt;
};

template <int G>
struct PersistSmem {
  static constexpr int NH = PersistCfg<G>::NH;
  static constexpr int S = PersistCfg<G>::kStages;
  alignas(128) uint8_t ring[S][kPStageBytes];
  uint64_t full[S];             // data of the stage landed (TMA transaction count)
  uint64_t empty[S];            // the 4 consumer warps are done with the stage
  uint64_t meta_full[2];        // the producer published the slot
  uint64_t meta_empty[2];       // the 4 consumer warps are done with the slot
  PersistMeta<G> meta[2];
  int32_t seq_len[kPMaxBatch];     // seq_lens at the start of the launch
  int32_t ubase[kPMaxBatch + 1];   // first work unit of the sequence of rank r; [B]: all units
  uint8_t order[kPMaxBatch];       // sequence of rank r (longest splits first)
  int8_t n_new[kPMaxBatch];        // tokens appended (0/1); -1: length error, nothing attended
  union {
    struct {
      int8_t qd[NH][3][kDim];      // q digits of the unit (read into registers once)
      SealScratch seal;            // fused step: written at the unit's start, used during its items
    } w;
    float mg[2][NH * kMbufPitch];  // warp merge, in the unit's epilogue: two warps' outputs (value layout)
  } u;
  float mg_m[2][NH], mg_l[2][NH];
  alignas(16) uint32_t zero16[4];
  PendMerge pend;
  int pend_last;  // the pending split merge is this CTA's to do
  int last;
  int abort_flag;
};

// AND of `pred` over the 128 consumer threads (named barrier 1).
__device__ __forceinline__ bool consumers_and(bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "barrier.red.and.pred q, 1, 128, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(pred ? 1u : 0u)
      : "memory");
  return r != 0;
}

// Partial j of a split merge is split j (8 partials fetched at a time: the
// merge runs beside the next unit's registers).
struct IdentSlot {
  __device__ __forceinline__ int operator()(int j) const { return j; }
};

// Named barrier `id` among `n` threads (two consumer warps: n = 64).
__device__ __forceinline__ void pair_sync(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

__device__ __forceinline__ bool aborted_now(const int *flag) { return *reinterpret_cast<const volatile int *>(flag) != 0; }

// A warp's online-softmax state (value layout) into the merge buffer.
template <int NT>
__device__ __forceinline__ void store_state(const WarpState<NT> &st, float *acc, float *m, float *l, int g, int t) {
#pragma unroll
  for (int nt = 0; nt < NT; nt++) {
    const int hd = 4 * nt + t;
    float *row = acc + hd * kMbufPitch;
#pragma unroll
    for (int mt = 0; mt < 8; mt++) {
      row[16 * mt + g] = st.acc[nt][mt][0];
      row[16 * mt + g + 8] = st.acc[nt][mt][1];
    }
    if (g == 0) {
      m[hd] = st.m_run[nt];
      l[hd] = st.l_run[nt];
    }
  }
}

// ... and another warp's state from it joins this warp's: both rescaled to
// the larger running maximum (an empty state, maximum -inf, weighs 0).
template <int NT>
__device__ __forceinline__ void absorb_state(WarpState<NT> &st, const float *acc, const float *m, const float *l,
                                             int g, int t) {
#pragma unroll
  for (int nt = 0; nt < NT; nt++) {
    const int hd = 4 * nt + t;
    const float mo = m[hd], lo = l[hd];
    const float mn = fmaxf(st.m_run[nt], mo);
    const float fs = mn == -INFINITY ? 0.f : ex2(st.m_run[nt] - mn);
    const float fo = mn == -INFINITY ? 0.f : ex2(mo - mn);
    const float *row = acc + hd * kMbufPitch;
#pragma unroll
    for (int mt = 0; mt < 8; mt++) {
      st.acc[nt][mt][0] = fmaf(fo, row[16 * mt + g], st.acc[nt][mt][0] * fs);
      st.acc[nt][mt][1] = fmaf(fo, row[16 * mt + g + 8], st.acc[nt][mt][1] * fs);
    }
    st.l_run[nt] = fmaf(fo, lo, st.l_run[nt] * fs);
    st.m_run[nt] = mn;
  }
}

template <int G>
__global__ void __launch_bounds__(kPThreads, PersistCfg<G>::kCtasPerSm) decode_persist_kernel(const DecodeArgs a) {
  constexpr int NT = PersistCfg<G>::NT;
  constexpr int NH = PersistCfg<G>::NH;
  constexpr int S = PersistCfg<G>::kStages;
  extern __shared__ __align__(128) uint8_t smem_raw[];
  PersistSmem<G> &sm = *reinterpret_cast<PersistSmem<G> *>(smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int B = a.batch;
  const int NS = a.n_splits;  // workspace stride of the splits
  const int tb = a.split_blocks;
  const int H = a.hot_tokens;
  const bool fused = a.n_new != nullptr;

  if (tid == 0) {
#pragma unroll
    for (int st = 0; st < S; st++) {
      mbar_init(&sm.full[st], 1);
      mbar_init(&sm.empty[st], kWarps);
    }
    for (int i = 0; i < 2; i++) {
      mbar_init(&sm.meta_full[i], 1);
      mbar_init(&sm.meta_empty[i], kWarps);
    }
    sm.abort_flag = 0;
    sm.pend_last = 0;
    mbar_fence_init();
  }
  if (tid < 4) sm.zero16[tid] = 0u;
  // a merge launch that follows (defer_merge) may be placed on the SMs as
  // this launch's CTAs leave them; it waits for this grid's results itself
  if (tid == 0) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  // lengths at launch and the work units of each sequence: its splits with
  // work (at least one, which writes the output of an empty sequence) times
  // the kv heads.  Units are numbered sequence by sequence, so the counter
  // hands out no empty units, and the sequences with the longest splits come
  // first (longest processing time first: the units handed out last are the
  // short ones, so the CTAs finish close together).
  int32_t *key = reinterpret_cast<int32_t *>(&sm.u);  // items of a split, until the first unit
  for (int i = tid; i < B; i += kPThreads) {
    const int L_old = a.seq_lens[i];
    int n_app = fused ? a.n_new[i] : 0;
    if (n_app < 0 || n_app > 1) {
      set_status(a.status, HYB_STATUS_BAD_N_NEW);
      n_app = 0;
    }
    int L = L_old + n_app;
    bool bad = false;
    if (L_old < 0 || L > a.max_seq_len) {
      set_status(a.status, HYB_STATUS_SEQ_LEN);
      bad = true;
      L = 0;
    }
    const int nblk = (max(0, L - H) + kBlock - 1) / kBlock;
    int Sb, items;
    if (a.min_splits > 0) {
      items = nblk + (L > 0 ? 1 : 0);
      Sb = per_seq_splits(items, a.min_splits);
    } else {
      items = nblk + min((min(L, H) + kItemRows - 1) / kItemRows, tb);
      Sb = max(1, (items + tb - 1) / tb);
    }
    if (Sb > NS) {  // cannot happen with a plan for this max_seq_len: guards the workspace
      set_status(a.status, HYB_STATUS_SEQ_LEN);
      bad = true;
      Sb = 1;
    }
    sm.seq_len[i] = L_old;
    sm.n_new[i] = static_cast<int8_t>(bad ? -1 : n_app);
    sm.ubase[i] = Sb * a.hkv;
    key[i] = (items + Sb - 1) / Sb;
  }
  __syncthreads();
  for (int i = tid; i < B; i += kPThreads) {
    const int ki = key[i];
    int r = 0;
    for (int j = 0; j < B; j++) {
      const int kj = key[j];
      r += (kj > ki || (kj == ki && j < i)) ? 1 : 0;
    }
    sm.order[r] = static_cast<uint8_t>(i);
  }
  __syncthreads();
  if (warp == 0) {
    // exclusive prefix of the unit counts in rank order (8 ranks per lane);
    // every count is read before any is overwritten
    int v[kPMaxBatch / 32];
    int sum = 0;
#pragma unroll
    for (int j = 0; j < kPMaxBatch / 32; j++) {
      const int r = (kPMaxBatch / 32) * lane + j;
      v[j] = r < B ? sm.ubase[sm.order[r]] : 0;
      sum += v[j];
    }
    __syncwarp();
    int incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int n = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += n;
    }
    int run = incl - sum;
#pragma unroll
    for (int j = 0; j < kPMaxBatch / 32; j++) {
      const int i = (kPMaxBatch / 32) * lane + j;
      if (i < B) sm.ubase[i] = run;
      run += v[j];
    }
    if (lane == 31) sm.ubase[B] = incl;
  }
  __syncthreads();  // the last CTA-wide barrier: from here on the producer runs on its own

  if (warp == kWarps) {
    // =============================== producer ===============================
    const uint64_t pol = l2_policy_evict_first();
    int slot = 0;
    int uses[2] = {0, 0};  // times each meta slot was published
    int qi = 0;            // items issued by this CTA (stage qi % S)
    const int U = sm.ubase[B];  // work units of the launch
    int rcur = 0;               // rank of the last unit's sequence (units come in increasing order)
    struct Unit {
      int u, b, h, s, Sb, i0, ncold, nhot, nitems, Lc, L_old, n_int4_b;
      bool do_seal, do_ring, ring_hbm;
    };
    auto describe = [&](int u) {
      Unit x;
      while (sm.ubase[rcur + 1] <= u) rcur++;
      x.u = u;
      x.b = sm.order[rcur];
      const int r = u - sm.ubase[rcur];
      x.Sb = (sm.ubase[rcur + 1] - sm.ubase[rcur]) / a.hkv;
      x.h = r / x.Sb;
      x.s = r - x.h * x.Sb;
      x.L_old = sm.seq_len[x.b];
      const int n8 = sm.n_new[x.b];
      const int n_app = max(n8, 0);
      const int L = n8 < 0 ? 0 : x.L_old + n_app;
      x.Lc = max(0, L - H);
      const int nblk = (x.Lc + kBlock - 1) / kBlock;
      // the sequence's c items (cold blocks, then the hot ring) in Sb
      // near-equal runs, so that all its units are the same size (the key of
      // the longest-first order) and none exceeds split_blocks items
      const long long c = a.min_splits > 0 ? nblk + (L > 0 ? 1 : 0)
                                           : nblk + min((min(L, H) + kItemRows - 1) / kItemRows, tb);
      x.i0 = static_cast<int>(x.s * c / x.Sb);
      x.ncold = max(0, min(nblk, static_cast<int>((x.s + 1) * c / x.Sb)) - x.i0);
      const bool holds_hot = x.s == x.Sb - 1;
      const bool holds_tail = x.ncold > 0 && x.i0 + x.ncold == nblk;
      x.nhot = holds_hot ? min(L, H) : 0;
      x.nitems = x.ncold + (x.nhot + kItemRows - 1) / kItemRows;
      const bool seal_seq = n_app == 1 && x.L_old >= H;
      x.do_seal = seal_seq && holds_tail;
      x.do_ring = n_app == 1 && holds_hot;
      x.ring_hbm = n_app == 1 && (seal_seq ? holds_tail : holds_hot);
      x.n_int4_b = a.quant_bits == 4 ? 0x7fffffff : (a.n_int4 ? a.n_int4[x.b] : 0);
      return x;
    };
    // the next unit of this CTA: claimed from the counter (claim), then
    // described once the counter's answer is back (take).  A unit is
    // claimed only a few items before the current one's copies are all out,
    // not a whole unit ahead: a CTA that took a long unit late must not hold
    // another one while the others run out of work.
    // The first unit of CTA c is unit c; the counter hands out the units
    // from gridDim.x on.
    int pend = blockIdx.x;
    auto claim = [&]() {
      if (lane == 0) pend = static_cast<int>(gridDim.x) + atomicAdd(&a.unit_ctr[0], 1);
    };
    auto take = [&]() -> Unit {
      const int u = __shfl_sync(0xffffffffu, pend, 0);
      Unit x;
      if (u >= U) {
        x.u = -1;
        return x;
      }
      return describe(u);
    };
    // a unit's loads (independent of each other): the block-table entry of
    // this lane's block, 4 channels of q per head
    struct Loads {
      int phys;
      float2 sc;
      uint2 q[G];
    };
    auto load = [&](const Unit &x) {
      Loads l;
      l.phys = (lane < x.ncold) ? a.block_table[(size_t)x.b * a.max_blocks + x.i0 + lane] : -1;
      l.sc = make_float2(0.f, 0.f);
      const __half *qb = a.q + ((size_t)x.b * a.hq + x.h * G) * kDim;
#pragma unroll
      for (int j = 0; j < G; j++) l.q[j] = *reinterpret_cast<const uint2 *>(qb + j * kDim + 4 * lane);
      return l;
    };
    // the block-table entries once they are in: an invalid block's becomes
    // -1 (no copy, no scale)
    auto check_phys = [&](const Unit &x, Loads &l) {
      if (lane < x.ncold && (l.phys < 0 || l.phys >= a.num_phys)) {
        set_status(a.status, HYB_STATUS_BAD_BLOCK);
        l.phys = -1;
      }
    };
    // the block scales of a unit: a second round trip, issued once its
    // block-table entries are in
    auto load_scales = [&](const Unit &x, Loads &l) {
      check_phys(x, l);
      if (lane < x.ncold && l.phys >= 0)
        l.sc = __ldg(reinterpret_cast<const float2 *>(a.scales + ((size_t)l.phys * a.hkv + x.h) * 2));
    };
    // publish a unit in the current slot, once the consumers are done with
    // the unit that used it two units ago (a handshake, not a data wait: it
    // keeps the full limit)
    auto publish = [&](const Unit &x, const Loads &l) {
      PersistMeta<G> &m = sm.meta[slot];
      if (uses[slot] > 0 && !mbar_wait_bounded(&sm.meta_empty[slot], (uses[slot] - 1) & 1, kWaitCycles)) {
        if (lane == 0) set_status(a.status, HYB_STATUS_TIMEOUT);
        sm.abort_flag = 1;
      }
      const bool ab = aborted_now(&sm.abort_flag);
      m.phys[lane] = l.phys;
      m.scl[lane] = l.sc;
      // each head's largest |q| over the lanes' 4 channels, and from it the
      // reciprocal and the step of the consumers' 24-bit fixed point
      float qinv = 0.f, qstep = 0.f;  // head `lane`'s
#pragma unroll
      for (int j = 0; j < G; j++) {
        *reinterpret_cast<uint2 *>(&m.q[j][4 * lane]) = l.q[j];
        const __half2 p0 = *reinterpret_cast<const __half2 *>(&l.q[j].x);
        const __half2 p1 = *reinterpret_cast<const __half2 *>(&l.q[j].y);
        float mx = fmaxf(fmaxf(fabsf(__low2float(p0)), fabsf(__high2float(p0))),
                         fmaxf(fabsf(__low2float(p1)), fabsf(__high2float(p1))));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        if (lane == j) {
          qinv = mx > 0.f ? kQFix / mx : 0.f;
          qstep = mx / kQFix;
        }
      }
#pragma unroll
      for (int j = G; j < NH; j++) *reinterpret_cast<uint2 *>(&m.q[j][4 * lane]) = make_uint2(0u, 0u);
      if (lane < NH) {
        m.qinv[lane] = qinv;
        m.qstep[lane] = qstep;
      }
      if (lane == 0) {
        m.unit = x.u;
        m.b = x.b;
        m.h = x.h;
        m.s = x.s;
        m.Sb = x.Sb;
        m.i0 = x.i0;
        m.ncold = x.ncold;
        m.nhot = x.nhot;
        m.nitems = ab ? 0 : x.nitems;
        m.Lc = x.Lc;
        m.L_old = x.L_old;
        m.n_int4_b = x.n_int4_b;
        m.do_seal = ab ? 0 : x.do_seal;
        m.do_ring = ab ? 0 : x.do_ring;
        m.ring_hbm = ab ? 0 : x.ring_hbm;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.meta_full[slot]);
      uses[slot]++;
    };
    // issue item k of unit x into the next stage (the block-table entry of
    // cold item k is lane k's l.phys)
    bool ab = false;
    auto issue = [&](const Unit &x, int k, const Loads &l) {
      const int st = qi % S;
      if (qi >= S && !ab && !mbar_wait_bounded(&sm.empty[st], ((qi / S) - 1) & 1, a.wait_cycles)) {
        if (lane == 0) set_status(a.status, HYB_STATUS_TIMEOUT);
        sm.abort_flag = 1;
        ab = true;
      }
      uint8_t *dst = sm.ring[st];
      if (k < x.ncold) {
        const int phys = __shfl_sync(0xffffffffu, l.phys, k);
        if (lane == 0) {
          if (phys < 0 || ab) {
            mbar_arrive(&sm.full[st]);
          } else {
            const uint8_t *src = a.cold + ((size_t)phys * a.hkv + x.h) * kTilePairBytes;
            if (x.i0 + k >= x.n_int4_b) {
              mbar_arrive_expect_tx(&sm.full[st], kTilePairBytes);
              bulk_g2s(dst, src, kTilePairBytes, &sm.full[st], pol);
            } else {
              mbar_arrive_expect_tx(&sm.full[st], kTileBytes);
              bulk_g2s(dst, src, kTileBytes / 2, &sm.full[st], pol);
              bulk_g2s(dst + kTileBytes, src + kTileBytes, kTileBytes / 2, &sm.full[st], pol);
            }
          }
        }
      } else {
        // hot item j: ring slots 32j .. min(32j + 32, nhot) - 1, one row per lane
        const int j = k - x.ncold;
        const int nr = min(kItemRows, x.nhot - j * kItemRows);
        if (lane == 0) {
          if (ab) mbar_arrive(&sm.full[st]);
          else mbar_arrive_expect_tx(&sm.full[st], static_cast<uint32_t>(nr) * kHotTokenBytes);
        }
        __syncwarp();
        if (!ab && lane < nr) {
          const uint8_t *src = a.hot + (((size_t)x.b * a.hkv + x.h) * H + j * kItemRows + lane) * kHotTokenBytes;
          bulk_g2s(dst + lane * kPRowPitch, src, kHotTokenBytes, &sm.full[st], pol);
        }
      }
      qi++;
    };

    Unit cur = take();
    Loads lcur;
    // The first unit's copies go out only after its scales are in: issued
    // earlier, the copies of all CTAs would fill the memory queues ahead of
    // the scale loads, and the descriptor would come later than the data.
    if (cur.u >= 0) {
      lcur = load(cur);
      load_scales(cur, lcur);
    }
    while (cur.u >= 0) {
      publish(cur, lcur);
      slot ^= 1;
      ab = ab || aborted_now(&sm.abort_flag);
      // the next unit: claimed 6 items before the end of this one's copies,
      // described and its block-table entries and q requested 2 items
      // later, its scales 2 items after that (each round trip overlaps
      // copies of this unit waiting for free stages)
      const int n = cur.nitems;
      const int k_claim = max(0, n - 6);
      const int k_take = min(n - 1, k_claim + 2);
      const int k_scl = min(n - 1, k_take + 2);
      Unit nxt;
      nxt.u = -1;
      Loads lnxt;
      bool claimed = false, taken = false;
      for (int k = 0; k < n && !ab; k++) {
        if (k == k_claim) {
          claim();
          claimed = true;
        }
        issue(cur, k, lcur);
        if (k == k_take) {
          nxt = take();
          taken = true;
          if (nxt.u >= 0) lnxt = load(nxt);
        }
        if (k == k_scl && nxt.u >= 0) load_scales(nxt, lnxt);
      }
      if (!taken) {  // no items, or a timeout stopped the copies: claim (once) and describe now
        if (!claimed) claim();
        nxt = take();
        if (nxt.u >= 0) {
          lnxt = load(nxt);
          load_scales(nxt, lnxt);
        }
      }
      cur = nxt;
      lcur = lnxt;
    }
    // no more units: the sentinel
    if (uses[slot] > 0 && !mbar_wait_bounded(&sm.meta_empty[slot], (uses[slot] - 1) & 1, kWaitCycles)) {
      if (lane == 0) set_status(a.status, HYB_STATUS_TIMEOUT);
      sm.abort_flag = 1;
    }
    if (lane == 0) {
      sm.meta[slot].unit = -1;
      mbar_arrive(&sm.meta_full[slot]);
    }
    // let every copy still in flight land before the CTA's shared memory is
    // released: the last item issued into each stage
    if (lane == 0) {
      for (int j = max(0, qi - S); j < qi; j++)
        (void)mbar_wait_bounded(&sm.full[j % S], (j / S) & 1, kWaitCycles);
    }
    // the last CTA to exit resets the counters and (fused step) advances
    // seq_lens: every CTA read the lengths at its start, before it arrived
    if (lane == 0 && atomic_add_acq_rel_gpu(&a.unit_ctr[1], 1) == static_cast<int>(gridDim.x) - 1) {
      a.unit_ctr[0] = 0;
      a.unit_ctr[1] = 0;
      if (fused)
        for (int i = 0; i < B; i++) a.seq_lens[i] = sm.seq_len[i] + max(static_cast<int>(sm.n_new[i]), 0);
    }
    return;
  }

  // =============================== consumers ===============================
  const int g = lane >> 2, t = lane & 3;
  const uint32_t psel = (g & 1) ? 0x6420u : 0x7531u;
  const uint32_t zero_addr = smem_addr(sm.zero16);
  const uint32_t v_lane0 = smem_addr(sm.ring[0]) + kTileBytes + lane * kBlock + 16 * (warp ^ ((lane >> 1) & 3));
  int slot = 0;
  int uses[2] = {0, 0};
  int qc = 0;  // items consumed (stage qc % S)
  // the previous unit's split merge: thread 0 holds its arrival ticket
  bool have_pend = false;
  int ticket = 0;

  // thread 0, before a consumer barrier: is the pending merge this CTA's?
  auto pend_decide = [&]() {
    if (tid == 0) {
      int last = 0;
      if (have_pend) {
        last = ticket == sm.pend.need - 1;
        if (last) *sm.pend.cnt = 0;
      }
      sm.pend_last = last;
    }
    have_pend = false;
  };
  // all consumers, after that barrier (from their copy of the descriptor):
  // run it -- thread 0's acquiring arrival and the barrier order the other
  // units' partials before these reads
  auto pend_run = [&](const PendMerge &p) {
    const size_t row0 = (size_t)p.b * a.hq + p.h * G;
    const int unit = p.b * a.hkv + p.h;
    float *lse_row = a.lse_out ? a.lse_out + row0 : nullptr;
    if (p.level == 0) {
      merge_splits<G, IdentSlot, 8>(a.o_part + row0 * NS * kDim, kDim, (size_t)NS * kDim, a.lse_part + row0 * NS, 1,
                                 NS, p.Sb, IdentSlot{}, warp, lane, a.out + row0 * kDim, lse_row, nullptr, 0, nullptr,
                                 0);
      return;
    }
    // a group of kMergeFan splits, then (the group that finishes last) the groups
    const int NG = a.n_groups;
    const int j0 = p.grp * kMergeFan;
    merge_splits<G, IdentSlot, 8>(a.o_part + (row0 * NS + j0) * kDim, kDim, (size_t)NS * kDim,
                               a.lse_part + row0 * NS + j0, 1, NS, min(kMergeFan, p.Sb - j0), IdentSlot{}, warp, lane,
                               nullptr, nullptr, a.g_part + (row0 * NG + p.grp) * kDim, (size_t)NG * kDim,
                               a.g_lse + row0 * NG + p.grp, NG);
    work_sync<true>();
    if (tid == 0) {
      const int ngb = (p.Sb + kMergeFan - 1) / kMergeFan;
      const int last2 = atomic_add_acq_rel_gpu(&a.counters[unit], 1) == ngb - 1;
      if (last2) a.counters[unit] = 0;
      sm.last = last2;
    }
    work_sync<true>();
    if (sm.last)
      merge_splits<G, IdentSlot, 8>(a.g_part + row0 * NG * kDim, kDim, (size_t)NG * kDim, a.g_lse + row0 * NG, 1, NG,
                                 (p.Sb + kMergeFan - 1) / kMergeFan, IdentSlot{}, warp, lane, a.out + row0 * kDim,
                                 lse_row, nullptr, 0, nullptr, 0);
  };

  for (;;) {
    if (!mbar_wait_bounded(&sm.meta_full[slot], uses[slot] & 1, kWaitCycles)) {
      if (tid == 0) set_status(a.status, HYB_STATUS_TIMEOUT);
      sm.abort_flag = 1;
      break;
    }
    const PersistMeta<G> &m = sm.meta[slot];
    if (m.unit < 0) break;
    const int b = m.b, h = m.h, s = m.s, Sb = m.Sb, i0 = m.i0, ncold = m.ncold, nhot = m.nhot,
              nitems = m.nitems, Lc = m.Lc, L_old = m.L_old, n_int4_b = m.n_int4_b;
    const bool do_seal = m.do_seal != 0, do_ring = m.do_ring != 0, ring_hbm = m.ring_hbm != 0;
    const int hq0 = h * G;
    const int rs = L_old & (H - 1);
    // fused step: channel tid of the evicted token (ring slot rs) and of the
    // new token, loaded now and first used at the seal's item, the ring's
    // item and after the items, so that no consumer waits for them here.
    // The evicted token is read before the new one is written to the same
    // bytes by the same thread.
    __half *const grow = reinterpret_cast<__half *>(a.hot) + (((size_t)b * a.hkv + h) * H + rs) * 2 * kDim;
    __half2 old_kv = __halves2half2(__float2half_rn(0.f), __float2half_rn(0.f)), new_kv = old_kv;
    if (do_seal) old_kv = __halves2half2(grow[tid], grow[kDim + tid]);
    if (do_ring || ring_hbm) {
      const size_t kvo = ((size_t)b * a.hkv + h) * kDim + tid;
      new_kv = __halves2half2(a.k_new[kvo], a.v_new[kvo]);
    }
    // q of the unit's heads in 24-bit fixed point (the producer found each
    // head's largest |q|): thread tid writes channel tid's digits
    {
#pragma unroll
      for (int j = 0; j < NH; j++) {
        int8_t d0 = 0, d1 = 0, d2 = 0;
        if (j < G) {
          int qi = __float2int_rn(__half2float(m.q[j][tid]) * m.qinv[j]);
          qi = max(-8323072, min(8323072, qi));
          const int lo = ((qi + 128) & 255) - 128;
          const int r = (qi - lo) >> 8;
          const int mid = ((r + 128) & 255) - 128;
          const int hi = (r - mid) >> 8;
          d0 = static_cast<int8_t>(hi);
          d1 = static_cast<int8_t>(mid);
          d2 = static_cast<int8_t>(lo);
        }
        sm.u.w.qd[j][0][tid] = d0;
        sm.u.w.qd[j][1][tid] = d1;
        sm.u.w.qd[j][2][tid] = d2;
      }
    }
    work_sync<true>();
    uint32_t qa[NT][4][4];
    load_qfrag<NT>(sm.u.w.qd, g, t, qa);
    float sqh[NT];
#pragma unroll
    for (int nt = 0; nt < NT; nt++) sqh[nt] = m.qstep[4 * nt + (g >> 1)];
    const int k_seal = do_seal ? ncold - 1 : -1;
    const int k_ring = do_ring ? ncold + rs / kItemRows : -1;

    WarpState<NT> ws;
    state_init<NT>(ws);
    for (int k = 0; k < nitems; k++) {
      const int st = qc % S;
      bool ok = !aborted_now(&sm.abort_flag) && mbar_wait_bounded(&sm.full[st], (qc / S) & 1, a.wait_cycles);
      if (!ok && lane == 0 && !aborted_now(&sm.abort_flag)) set_status(a.status, HYB_STATUS_TIMEOUT);
      if (k == k_seal || k == k_ring) {
        if (k == k_seal) {
          // published to the other consumers by the barrier below
          sm.u.w.seal.erow[tid] = __low2half(old_kv);
          sm.u.w.seal.erow[kDim + tid] = __high2half(old_kv);
        }
        ok = consumers_and(ok);
        if (ok && k == k_seal)
          fused_seal<true>(sm.u.w.seal, sm.ring[st], &sm.meta[slot].scl[ncold - 1],
                           m.phys[ncold - 1] * a.hkv + h, (i0 + ncold - 1) < n_int4_b, a, L_old, true, tid, warp,
                           lane);
        else if (ok)
          ring_put<true, kPRowPitch>(sm.ring[st], rs, new_kv, tid);
      }
      if (!ok) sm.abort_flag = 1;
      const uint8_t *stage = sm.ring[st];
      if (ok && k < ncold) {
        const int i = i0 + k;
        const int nvalid = m.phys[k] < 0 ? 0 : min(kBlock, Lc - i * kBlock);
        const int nv = nvalid - 16 * warp;
        const bool int4 = i < n_int4_b;
        const float2 sc = m.scl[k];
        const float cf = sc.x * a.qk_scale;
        float coef[NT];
#pragma unroll
        for (int nt = 0; nt < NT; nt++) coef[nt] = sqh[nt] * cf;
        const uint32_t v_lane = v_lane0 + st * kPStageBytes;
        if (nvalid == kBlock && !int4) {
          cold_item<NT, false, false>(stage, kBlock, warp, g, t, qa, coef, sc.y, psel, v_lane, ws);
        } else if (nv > 0) {
          if (int4)
            cold_item<NT, true, true>(stage, nvalid, warp, g, t, qa, coef, sc.y, psel, v_lane, ws);
          else
            cold_item<NT, false, true>(stage, nvalid, warp, g, t, qa, coef, sc.y, psel, v_lane, ws);
        }
      } else if (ok) {
        const int nrow = min(kItemRows, nhot - (k - ncold) * kItemRows);
        hot_item<NT, kPRowPitch>(stage, nrow, warp, lane, g, t, m.q, a.qk_scale, zero_addr, ws);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.empty[st]);
      qc++;
    }
    if (ring_hbm) {
      // the new token into the ring in HBM (after this thread's read of the
      // evicted token from the same bytes)
      grow[tid] = __low2half(new_kv);
      grow[kDim + tid] = __high2half(new_kv);
    }
    // the slot is not read after this point (the epilogue works from
    // registers and the merge buffer)
    __syncwarp();
    if (lane == 0) mbar_arrive(&sm.meta_empty[slot]);
    uses[slot]++;
    slot ^= 1;

    // ---------------- the unit's epilogue ----------------
    // is the previous unit's split merge this CTA's (its arrival has come
    // back by now)?  After this barrier every warp is past its q digits, so
    // the merge buffer, which overlaps them, is free.
    pend_decide();
    work_sync<true>();
    const bool run_pend = sm.pend_last != 0;
    PendMerge pm;
    if (run_pend) pm = sm.pend;
    // warp merge in two rounds of pairs: 2 -> 0 and 3 -> 1, then 1 -> 0
    if (warp >= 2) store_state<NT>(ws, sm.u.mg[warp - 2], sm.mg_m[warp - 2], sm.mg_l[warp - 2], g, t);
    pair_sync(2 + (warp & 1), 64);
    if (warp < 2) absorb_state<NT>(ws, sm.u.mg[warp], sm.mg_m[warp], sm.mg_l[warp], g, t);
    if (warp == 1) store_state<NT>(ws, sm.u.mg[1], sm.mg_m[1], sm.mg_l[1], g, t);
    if (warp < 2) pair_sync(4, 64);
    if (warp == 0) absorb_state<NT>(ws, sm.u.mg[1], sm.mg_m[1], sm.mg_l[1], g, t);
    // the merge buffer is free again (the next unit writes its q digits
    // there), and every warp holds its copy of the pending merge
    work_sync<true>();
    if (warp == 0) {
      // lane (g, t): head 4nt + t, channels 16mt + g (+ 8)
      const size_t row0 = (size_t)b * a.hq + hq0;
#pragma unroll
      for (int nt = 0; nt < NT; nt++) {
        const int hh = 4 * nt + t;
        if (hh < G) {
          const float l = ws.l_run[nt];
          const float inv = l > 0.f ? __frcp_rn(l) : 0.f;
          const float lse2 = l > 0.f ? ws.m_run[nt] + __log2f(l) : -INFINITY;
          if (Sb == 1 && !a.defer_merge) {
            __half *o = a.out + (row0 + hh) * kDim;
#pragma unroll
            for (int mt = 0; mt < 8; mt++) {
              o[16 * mt + g] = __float2half_rn(ws.acc[nt][mt][0] * inv);
              o[16 * mt + g + 8] = __float2half_rn(ws.acc[nt][mt][1] * inv);
            }
            if (g == 0 && a.lse_out) a.lse_out[row0 + hh] = lse2 * kLn2;
          } else {
            float *o = a.o_part + ((row0 + hh) * NS + s) * kDim;
#pragma unroll
            for (int mt = 0; mt < 8; mt++) {
              o[16 * mt + g] = ws.acc[nt][mt][0] * inv;
              o[16 * mt + g + 8] = ws.acc[nt][mt][1] * inv;
            }
            if (g == 0) a.lse_part[(row0 + hh) * NS + s] = lse2;
          }
        }
      }
    }
    // the previous unit's split merge runs now, with this unit's state out of
    // the registers
    if (run_pend) pend_run(pm);
    if (warp == 0) {
      if (a.defer_merge) {
        // the merge comes after the launch: it needs the split count
        if (s == 0 && lane == 0) a.split_count[b * a.hkv + h] = Sb;
      } else if (Sb > 1) {
        // arrival: the last unit of (sequence, kv head) -- or of its group of
        // kMergeFan splits -- merges; the answer is read at the next epilogue
        __syncwarp();
        if (lane == 0) {
          const int unit = b * a.hkv + h;
          const bool grouped = Sb > kMergeFan;
          const int grp = s / kMergeFan;
          int32_t *cnt = grouped ? &a.g_counters[(size_t)unit * a.n_groups + grp] : &a.counters[unit];
          ticket = atomic_add_acq_rel_gpu(cnt, 1);
          sm.pend.b = b;
          sm.pend.h = h;
          sm.pend.Sb = Sb;
          sm.pend.grp = grp;
          sm.pend.need = grouped ? min(kMergeFan, Sb - grp * kMergeFan) : Sb;
          sm.pend.level = grouped ? 1 : 0;
          sm.pend.cnt = cnt;
        }
        have_pend = true;
      }
    }
  }
  // the last unit's split merge
  pend_decide();
  work_sync<true>();
  if (sm.pend_last) {
    const PendMerge pm = sm.pend;
    pend_run(pm);
  }
}

// After a persistent launch with defer_merge: the splits of query head hq of
// sequence b -- split_count[b][hq / G] of them, written by the launch --
// merged by log-sum-exp.  Method: the same merge as hyb_combine (web page
// "DeepSeek V4混合式KV Cache推理优化实战解析", section 4.2, step 5).  One
// CTA of 16 warps per (query head, sequence): warp w takes every 16th split
// from w, with all of its partials' loads in flight at once (lane l:
// channels 4l .. 4l + 3); the 16 subsets then join through shared memory.
constexpr int kCombWarps = 16;
constexpr int kCombBatch = 8;  // partials a warp loads at a time

template <int G>
__global__ void __launch_bounds__(32 * kCombWarps) persist_combine_kernel(const DecodeArgs a) {
  __shared__ float4 s_num[kCombWarps][32];
  __shared__ float s_m[kCombWarps], s_den[kCombWarps];
  const int hq = blockIdx.x, b = blockIdx.y;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int NS = a.n_splits;
  // launched as a programmatic dependent of the persistent kernel: nothing
  // of its results is read before that grid has completed
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int Sb = min(max(a.split_count[b * a.hkv + hq / G], 1), NS);
  const size_t row = (size_t)b * a.hq + hq;
  const float *o = a.o_part + row * NS * kDim + 4 * lane;
  const float *lse = a.lse_part + row * NS;
  float m = -INFINITY, den = 0.f;
  float4 num = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int j0 = warp; j0 < Sb; j0 += kCombWarps * kCombBatch) {
    float4 ov[kCombBatch];
    float lv[kCombBatch];
#pragma unroll
    for (int jj = 0; jj < kCombBatch; jj++) {
      const int j = j0 + jj * kCombWarps;
      ov[jj] = j < Sb ? __ldcg(reinterpret_cast<const float4 *>(o + (size_t)j * kDim)) : make_float4(0.f, 0.f, 0.f, 0.f);
      lv[jj] = j < Sb ? __ldcg(lse + j) : -INFINITY;
    }
    float mr = m;
#pragma unroll
    for (int jj = 0; jj < kCombBatch; jj++) mr = fmaxf(mr, lv[jj]);
    if (mr == -INFINITY) continue;  // nothing but empty partials so far
    const float sc = ex2(m - mr);
    num.x *= sc; num.y *= sc; num.z *= sc; num.w *= sc;
    den *= sc;
    m = mr;
#pragma unroll
    for (int jj = 0; jj < kCombBatch; jj++) {
      const float wj = ex2(lv[jj] - m);  // 0 for an empty partial
      den += wj;
      num.x = fmaf(wj, ov[jj].x, num.x);
      num.y = fmaf(wj, ov[jj].y, num.y);
      num.z = fmaf(wj, ov[jj].z, num.z);
      num.w = fmaf(wj, ov[jj].w, num.w);
    }
  }
  s_num[warp][lane] = num;
  if (lane == 0) {
    s_m[warp] = m;
    s_den[warp] = den;
  }
  __syncthreads();
  if (warp == 0) {
    float mm = -INFINITY;
#pragma unroll
    for (int p = 0; p < kCombWarps; p++) mm = fmaxf(mm, s_m[p]);
    float dd = 0.f;
    float4 nn = make_float4(0.f, 0.f, 0.f, 0.f);
    if (mm != -INFINITY) {
#pragma unroll
      for (int p = 0; p < kCombWarps; p++) {
        const float wp = ex2(s_m[p] - mm);
        const float4 v = s_num[p][lane];
        dd = fmaf(wp, s_den[p], dd);
        nn.x = fmaf(wp, v.x, nn.x);
        nn.y = fmaf(wp, v.y, nn.y);
        nn.z = fmaf(wp, v.z, nn.z);
        nn.w = fmaf(wp, v.w, nn.w);
      }
    }
    const float inv = dd > 0.f ? 1.f / dd : 0.f;
    const __half2 h01 = __floats2half2_rn(nn.x * inv, nn.y * inv);
    const __half2 h23 = __floats2half2_rn(nn.z * inv, nn.w * inv);
    uint2 pk;
    pk.x = *reinterpret_cast<const uint32_t *>(&h01);
    pk.y = *reinterpret_cast<const uint32_t *>(&h23);
    *reinterpret_cast<uint2 *>(a.out + row * kDim + 4 * lane) = pk;
    if (lane == 0 && a.lse_out) a.lse_out[row] = dd > 0.f ? (mm + log2f(dd)) * kLn2 : -INFINITY;
  }
}

template <int G>
cudaError_t launch_persist_combine_g(const DecodeArgs &a, int batch, cudaStream_t stream) {
  // a programmatic dependent launch of the persistent kernel before it
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.hq, batch);
  cfg.blockDim = dim3(32 * kCombWarps, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, persist_combine_kernel<G>, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <int G>
cudaError_t launch_decode_persist_g(const DecodeArgs &a, int batch, int ctas, cudaStream_t stream) {
  const size_t smem = sizeof(PersistSmem<G>);
  static int configured_dev_mask = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 31 && !(configured_dev_mask & (1 << dev))) {
    e = cudaFuncSetAttribute(decode_persist_kernel<G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    configured_dev_mask |= 1 << dev;
  }
  (void)batch;
  decode_persist_kernel<G><<<dim3(ctas), kPThreads, smem, stream>>>(a);
  return cudaGetLastError();
}

template <int G>
int decode_persist_occupancy_g() {
  const size_t smem = sizeof(PersistSmem<G>);
  int n = 0;
  cudaError_t e = cudaFuncSetAttribute(decode_persist_kernel<G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e == cudaSuccess) e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, decode_persist_kernel<G>, kPThreads, smem);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  return n;
}

}  // namespace hyb
