// hyb_host.cu -- the C ABI declared in include/hyb_kv.h and include/hyb_measure.h: argument checks,
// split planning, workspace sizing and kernel launches.  No memory is
// allocated here; every buffer belongs to the caller.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <algorithm>
#include <atomic>
#include <cstring>

#include "hyb_measure.h"
#include "kernels.cuh"

namespace {

thread_local int g_last_cuda_error = 0;

// limit of the decode pipeline's bounded waits (hyb_set_wait_limit); 0 = default
std::atomic<long long> g_wait_cycles{0};

int cuda_fail(cudaError_t e) {
  g_last_cuda_error = static_cast<int>(e);
  return HYB_ERR_CUDA;
}

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int sm_count() {
  // cached per device: the planner runs on every call
  static int cached[32];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    dev = 0;
  }
  if (dev >= 0 && dev < 32 && cached[dev] > 0) return cached[dev];
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
    cudaGetLastError();  // clear the sticky-free error this query may leave
    return 148;          // B200 (not cached: a later call on a device may answer)
  }
  if (dev >= 0 && dev < 32) cached[dev] = n;
  return n;
}

constexpr size_t kWsAlign = 256;

size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

}  // namespace

extern "C" {

int hyb_version(void) { return 10000; }

int hyb_stream_read(const void *src, size_t bytes, uint32_t *sink, hyb_stream_t stream) {
  if (bytes == 0) return HYB_OK;  // nothing to read: no launch, no pointer is touched
  if (!src || !sink || !aligned(src, 16) || !aligned(sink, 4) || bytes % 16 != 0) return HYB_ERR_INVALID_VALUE;
  const size_t n16 = bytes / 16;
  const size_t per_cta = static_cast<size_t>(hyb::kStreamReadThreads);
  const size_t want = (n16 + per_cta - 1) / per_cta;  // no CTA without a load
  const int grid = static_cast<int>(std::min<size_t>(want, static_cast<size_t>(sm_count()) * hyb::kStreamReadCtasPerSm));
  const cudaError_t e = hyb::launch_stream_read(src, bytes, sink, grid, stream);
  return e == cudaSuccess ? HYB_OK : cuda_fail(e);
}

int hyb_set_wait_limit(int64_t cycles) {
  g_wait_cycles.store(cycles > 0 ? static_cast<long long>(cycles) : 0, std::memory_order_relaxed);
  return HYB_OK;
}

int hyb_last_cuda_error(void) { return g_last_cuda_error; }

const char *hyb_strerror(int code) {
  switch (code) {
    case HYB_OK: return "ok";
    case HYB_ERR_INVALID_VALUE: return "invalid value (configuration, shape, null or misaligned pointer)";
    case HYB_ERR_UNSUPPORTED: return "unsupported configuration (only hot 32 / block 64 / head_dim 128, Hq/Hkv <= 8)";
    case HYB_ERR_WORKSPACE: return "workspace missing or too small";
    case HYB_ERR_CUDA: return "CUDA error (see hyb_last_cuda_error)";
    case HYB_ERR_SCRATCH_LIMIT: return "problem needs more scratch than the static buffer of hyb_decode_attn_noalloc";
    case 100 + HYB_STATUS_OK: return "device status: ok";
    case 100 + HYB_STATUS_BAD_BLOCK: return "device status: block-table entry out of range";
    case 100 + HYB_STATUS_BAD_N_NEW: return "device status: n_new out of range";
    case 100 + HYB_STATUS_CAPACITY: return "device status: sequence outgrew its block table";
    case 100 + HYB_STATUS_SEQ_LEN: return "device status: seq_lens out of range for decode";
    case 100 + HYB_STATUS_TIMEOUT: return "device status: a bounded wait in a kernel ran out";
    case 100 + HYB_STATUS_BAD_TIER:
      return "device status: a migration target outside the block table or beyond max_delta";
    default: return "unknown code";
  }
}

// log2 of the 64-token sub-blocks per block (block_size 32, 64: 0; 128: 1)
static int lsub_of(const hyb_cache_desc *d) { return d->block_size == 2 * hyb::kBlock ? 1 : 0; }
// log2 of the tokens per block (32: 5, 64: 6, 128: 7)
static int bshift_of(const hyb_cache_desc *d) { return d->block_size == 32 ? 5 : d->block_size == 64 ? 6 : 7; }

int hyb_check_desc(const hyb_cache_desc *d) {
  if (!d) return HYB_ERR_INVALID_VALUE;
  // hybrid_v2 contract (page sections 3.1 / 5.1)
  const int h = d->hot_tokens;
  if (!(h == 16 || h == 32 || h == 64 || h == 128)) return HYB_ERR_INVALID_VALUE;
  if (d->block_size <= 0 || d->block_size % 8 != 0) return HYB_ERR_INVALID_VALUE;
  // 8 or 4 (section 3.1); 0 keeps the cold zone in FP16 (section 5.2)
  if (d->quant_bits != 8 && d->quant_bits != 4 && d->quant_bits != 0) return HYB_ERR_INVALID_VALUE;
  if (d->head_dim <= 0 || d->num_kv_heads <= 0 || d->num_q_heads <= 0 || d->batch <= 0 ||
      d->num_phys_blocks < 0 || d->max_blocks_per_seq <= 0)
    return HYB_ERR_INVALID_VALUE;
  if (d->num_q_heads % d->num_kv_heads != 0) return HYB_ERR_INVALID_VALUE;
  if (d->reserved != 0) return HYB_ERR_INVALID_VALUE;
  if (!d->hot || !d->cold || !d->scales || !d->block_table || !d->seq_lens || !d->status)
    return HYB_ERR_INVALID_VALUE;
  if (!aligned(d->hot, 512) || !aligned(d->cold, 16) || !aligned(d->scales, 8) ||
      !aligned(d->block_table, 4) || !aligned(d->seq_lens, 4) || !aligned(d->status, 4) ||
      (d->n_int4_blocks && !aligned(d->n_int4_blocks, 4)))
    return HYB_ERR_INVALID_VALUE;
  // what this library builds
  if ((d->block_size != 32 && d->block_size != hyb::kBlock && d->block_size != 2 * hyb::kBlock) ||
      d->head_dim != hyb::kDim)
    return HYB_ERR_UNSUPPORTED;
  if (d->num_q_heads / d->num_kv_heads > 8) return HYB_ERR_UNSUPPORTED;
  return HYB_OK;
}

int hyb_kv_append(const hyb_cache_desc *d, const int32_t *n_new, int32_t max_new, const void *k_new,
                  const void *v_new, hyb_stream_t stream) {
  const int rc = hyb_check_desc(d);
  if (rc != HYB_OK) return rc;
  if (!n_new || !k_new || !v_new || max_new <= 0 || !aligned(n_new, 4) || !aligned(k_new, 16) ||
      !aligned(v_new, 16))
    return HYB_ERR_INVALID_VALUE;
  hyb::AppendArgs a;
  a.hot = static_cast<__half *>(d->hot);
  a.cold = static_cast<uint8_t *>(d->cold);
  a.scales = d->scales;
  a.block_table = d->block_table;
  a.seq_lens = d->seq_lens;
  a.n_int4 = d->quant_bits == 8 ? d->n_int4_blocks : nullptr;
  a.status = d->status;
  a.n_new = n_new;
  a.k_new = static_cast<const __half *>(k_new);
  a.v_new = static_cast<const __half *>(v_new);
  a.hkv = d->num_kv_heads;
  a.num_phys = d->num_phys_blocks;
  a.max_blocks = d->max_blocks_per_seq;
  a.quant_bits = d->quant_bits;
  a.max_new = max_new;
  a.hot_tokens = d->hot_tokens;
  a.lsub = lsub_of(d);
  a.bshift = bshift_of(d);
  const cudaError_t e = hyb::launch_append(a, d->batch, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? HYB_OK : cuda_fail(e);
}

}  // extern "C"

namespace {

// Cold blocks per split when the splits take several waves.
constexpr int kMultiWaveSplit = 16;
// Longest automatic split of the persistent kernel for head groups above 4
// (two 4-head MMA row tiles): their blocks cost about twice the arithmetic
// of a group of up to 4, so a split of kPMaxSplitBlocks blocks runs twice as
// long and the last units handed out leave that much of a tail.  Measured on
// the Qwen2-7B mixed batch (group 7): 24-block splits 121.4 us per step, 32:
// 125.7, 16: 125.2, 12: 136.3.
constexpr int kPWideSplit = 24;
// Fewest blocks per split of a one-wave plan: a CTA's fixed cost (the
// metadata round trip before its first copy, the epilogue and the split
// merge, ~3 us) wants a few items of work.  On the Llama-3-8B batch of 8 at
// L = 2048 (33 items per sequence and kv head), 6-block splits measured
// 22.7 us per step, 4-block splits (the most the GPU holds at once) 28.5 us.
constexpr int kMinWaveSplit = 6;

// How a decode call runs: grid (ns, Hkv, batch) of the decode kernel.  When
// every split fits on the GPU at once (one wave), automatic plans cut the
// longest sequence into as many splits as fill the GPU (of at least
// kMinWaveSplit blocks), and 2..16 splits are merged inside a thread-block
// cluster when all clusters fit.  Otherwise the splits run in several waves,
// merged through the workspace (the persistent kernel where it applies).
struct Plan {
  bool cluster;  // clusters of ns CTAs (split merge in distributed shared memory)
  bool persist;  // the persistent kernel: `ctas` CTAs take the splits as work units
  int ctas;
  int tb;        // cold blocks per split (per-sequence splits: the longest sequence's)
  int per_seq;   // > 0: per-sequence splits, at least this many per sequence
  bool defer;    // persistent with more than kMergeFan splits: partials only, then persist_combine_kernel
  int ns;        // splits per (sequence, kv head), at most
};

int make_plan(const hyb_cache_desc *d, int32_t max_seq_len, int32_t split_tokens, Plan *p) {
  const int rc = hyb_check_desc(d);
  if (rc != HYB_OK) return rc;
  if (max_seq_len < 0) return HYB_ERR_INVALID_VALUE;
  const long long nblk = (static_cast<long long>(max_seq_len) - d->hot_tokens > 0)
                             ? (max_seq_len - d->hot_tokens + d->block_size - 1) / d->block_size
                             : 0;
  if (nblk > d->max_blocks_per_seq) return HYB_ERR_INVALID_VALUE;
  const int group = d->num_q_heads / d->num_kv_heads;
  const int sms = sm_count();
  int occ = hyb::decode_ctas_per_sm(group);
  if (occ <= 0) occ = group <= 4 ? 3 : 2;
  const long long slots = static_cast<long long>(sms) * occ;
  const long long units = static_cast<long long>(d->batch) * d->num_kv_heads;
  const int max_tb = hyb::decode_max_split_blocks();
  // the hot ring's items, counted in blocks when a sequence is cut into
  // splits (the kernel uses the same rule, capped at one split's blocks)
  const long long hot_n = max_seq_len < d->hot_tokens ? max_seq_len : d->hot_tokens;
  const long long dh = (hot_n + 31) / 32;
  const long long ipb = d->quant_bits == 0 ? d->block_size / 32 : (d->block_size > hyb::kBlock ? 2 : 1);
  const long long dhb = (dh + ipb - 1) / ipb;
  auto n_splits = [&](long long t) {
    const long long v = (nblk + (dhb < t ? dhb : t) + t - 1) / t;
    return v < 1 ? 1 : v;
  };
  // caches the persistent kernel takes (64-token INT8/INT4 blocks, batch
  // <= 256 sequences)
  const bool persist_ok = d->block_size == hyb::kBlock && d->quant_bits != 0 && d->batch <= hyb::kPMaxBatch;
  p->per_seq = 0;
  p->defer = false;
  if (split_tokens < 0) {
    // per-sequence splits (per_seq_splits): the persistent kernel only; where
    // it cannot run, every sequence takes the longest one's split length
    const long long n = -static_cast<long long>(split_tokens);
    if (n > 65535) return HYB_ERR_INVALID_VALUE;
    const long long c = nblk + (max_seq_len > 0 ? 1 : 0);
    const long long ns = hyb::per_seq_splits(c, n);
    const long long tb = c > 0 ? (c + ns - 1) / ns : 1;
    if (persist_ok) {
      int pocc = hyb::decode_persist_ctas_per_sm(group);
      if (pocc <= 0) pocc = 3;  // no GPU to ask: the compiled kernel's occupancy
      long long ctas = static_cast<long long>(sms) * pocc;
      if (ctas > units * ns) ctas = units * ns;
      p->cluster = false;
      p->persist = true;
      p->ctas = static_cast<int>(ctas);
      p->per_seq = static_cast<int>(n);
      p->tb = static_cast<int>(tb);
      p->ns = static_cast<int>(ns);
      p->defer = ns > hyb::kMergeFan;
      return HYB_OK;
    }
    split_tokens = static_cast<int32_t>(tb * d->block_size);
  }
  long long tb = 0;
  bool multi_wave = false;  // the automatic choice found no one-wave plan
  if (split_tokens == 0) {
    // one wave: enough splits of the longest sequence to fill the GPU, no more
    const long long s_wave = slots / units;
    if (s_wave >= 1) {
      tb = (nblk + dhb + s_wave - 1) / s_wave;
      if (tb < kMinWaveSplit) tb = kMinWaveSplit;
      if (tb > max_tb) tb = max_tb;
    }
    if (tb == 0 || tb > kMultiWaveSplit || units * n_splits(tb) > slots) {
      // several waves (also when one wave would need splits longer than
      // kMultiWaveSplit: a batch of (sequence, kv head) rows nearly as large
      // as the GPU's CTA slots would otherwise give each row one long split).
      // The persistent kernel takes these plans where it can: it hands out
      // the longest splits first and claims units late, so long splits
      // (fewer per-unit prologues and merges) cost little tail -- shorter
      // ones for wide head groups, whose blocks take longer; the split-per-CTA
      // kernel gets short splits, so that the CTA scheduler evens out rows of
      // different lengths.
      tb = !persist_ok ? kMultiWaveSplit : group > 4 ? kPWideSplit : hyb::kPMaxSplitBlocks;
      multi_wave = true;
      if (tb > nblk) tb = nblk > 0 ? nblk : 1;
    }
  } else {
    if (split_tokens % d->block_size != 0) return HYB_ERR_INVALID_VALUE;
    tb = split_tokens / d->block_size;
    if (tb < 1) return HYB_ERR_INVALID_VALUE;
  }
  const long long ns = n_splits(tb);
  if (tb > max_tb || ns > 65535) return HYB_ERR_INVALID_VALUE;
  // clusters only when every split is resident at once (a cluster holds its
  // CTAs until its slowest split is done): every (sequence, kv head)'s
  // cluster must fit on the GPU together
  p->cluster = units * ns <= slots && ns >= 2 && ns <= hyb::decode_max_cluster() &&
               units <= hyb::decode_resident_clusters(group, static_cast<int>(ns));
  // several waves of splits: the persistent kernel, whose CTAs stay resident
  // and stream the splits back to back (64-token INT8/INT4 blocks, splits of
  // up to kPMaxSplitBlocks blocks, batches of up to kPMaxBatch sequences)
  p->persist = false;
  p->ctas = 0;
  if (!p->cluster && (units * ns > slots || multi_wave) && persist_ok && tb <= hyb::kPMaxSplitBlocks) {
    int pocc = hyb::decode_persist_ctas_per_sm(group);
    if (pocc <= 0) pocc = 3;  // no GPU to ask: the compiled kernel's occupancy
    long long c = static_cast<long long>(sms) * pocc;
    if (c > units * ns) c = units * ns;
    p->persist = true;
    p->ctas = static_cast<int>(c);
    p->defer = ns > hyb::kMergeFan;
  }
  p->tb = static_cast<int>(tb);
  p->ns = static_cast<int>(ns);
  return HYB_OK;
}

// Workspace layout.  Fused step: read counters int32 [batch] first.  Splits
// merged through the workspace (not in a cluster): arrival counters int32
// [batch][Hkv] and, with more than kMergeFan splits, group arrival counters
// int32 [batch][Hkv][ng] (ng = ceil(ns / kMergeFan)); then the split outputs
// FP32 [batch][Hq][ns][128] and their log2-sum-exp FP32 [batch][Hq][ns]; then
// the group outputs FP32 [batch][Hq][ng][128] and their log2-sum-exp
// [batch][Hq][ng].  Each part starts on a 256-byte boundary; the counters
// come first.
struct WsLayout {
  size_t seq_cnt, unit_ctr, counters, g_counters, o_part, lse_part, g_part, g_lse, split_count, total;
  int n_groups;
};

WsLayout ws_layout(const hyb_cache_desc *d, const Plan &pl, bool step) {
  WsLayout w{0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0};
  size_t off = 0;
  if (step) {
    w.seq_cnt = 0;
    off = round_up(static_cast<size_t>(d->batch) * sizeof(int32_t), kWsAlign);
  }
  if (pl.persist) {
    w.unit_ctr = off;
    off += kWsAlign;
  }
  const size_t rows = static_cast<size_t>(d->batch) * d->num_q_heads;
  const size_t units = static_cast<size_t>(d->batch) * d->num_kv_heads;
  const size_t ns = static_cast<size_t>(pl.ns);
  const size_t ng = ns > static_cast<size_t>(hyb::kMergeFan) ? (ns + hyb::kMergeFan - 1) / hyb::kMergeFan : 0;
  if (!pl.cluster && ns > 1) {
    w.n_groups = static_cast<int>(ng);
    w.counters = off;
    off += round_up(units * sizeof(int32_t), kWsAlign);
    w.g_counters = off;
    off += round_up(units * ng * sizeof(int32_t), kWsAlign);
    const size_t parts = rows * ns;
    w.o_part = off;
    w.lse_part = w.o_part + round_up(parts * hyb::kDim * sizeof(float), kWsAlign);
    off = w.lse_part + round_up(parts * sizeof(float), kWsAlign);
    w.g_part = off;
    w.g_lse = w.g_part + round_up(rows * ng * hyb::kDim * sizeof(float), kWsAlign);
    off = w.g_lse + round_up(rows * ng * sizeof(float), kWsAlign);
  }
  if (pl.defer) {
    // splits of each (sequence, kv head), written by every call before it is read
    w.split_count = off;
    off += round_up(units * sizeof(int32_t), kWsAlign);
  }
  w.total = off;
  return w;
}

}  // namespace

namespace hyb {
// Leading bytes of the hyb_decode_attn workspace that must be zero before a
// call (the arrival counters); 0 when the workspace is not used.
size_t decode_ws_zero_prefix(const hyb_cache_desc *d, int32_t max_seq_len, int32_t split_tokens) {
  Plan pl;
  if (make_plan(d, max_seq_len, split_tokens, &pl) != HYB_OK) return 0;
  const WsLayout w = ws_layout(d, pl, false);
  return w.o_part > 0 ? w.o_part : w.total;  // the counters come first
}
}  // namespace hyb

extern "C" {

int hyb_decode_plan(const hyb_cache_desc *d, int32_t max_seq_len, int32_t split_tokens,
                    int32_t *split_tokens_out, int32_t *n_splits_out) {
  Plan pl;
  const int rc = make_plan(d, max_seq_len, split_tokens, &pl);
  if (rc != HYB_OK) return rc;
  if (split_tokens_out) *split_tokens_out = pl.tb * d->block_size;
  if (n_splits_out) *n_splits_out = pl.ns;
  return HYB_OK;
}

int hyb_decode_launch_info(const hyb_cache_desc *d, int32_t max_seq_len, int32_t split_tokens, int32_t *kernel,
                           int32_t *ctas, int32_t *ctas_per_sm) {
  Plan pl;
  const int rc = make_plan(d, max_seq_len, split_tokens, &pl);
  if (rc != HYB_OK) return rc;
  const int group = d->num_q_heads / d->num_kv_heads;
  const int units = d->batch * d->num_kv_heads;
  if (kernel)
    *kernel = pl.persist ? (pl.defer ? HYB_KERNEL_PERSISTENT_COMBINE : HYB_KERNEL_PERSISTENT)
                         : (pl.cluster ? HYB_KERNEL_CLUSTER : HYB_KERNEL_SPLIT_CTA);
  if (ctas) *ctas = pl.persist ? pl.ctas : units * pl.ns;
  if (ctas_per_sm)
    *ctas_per_sm = pl.persist ? hyb::decode_persist_ctas_per_sm(group) : hyb::decode_ctas_per_sm(group);
  return HYB_OK;
}

size_t hyb_decode_workspace_bytes(const hyb_cache_desc *d, int32_t max_seq_len, int32_t split_tokens) {
  Plan pl;
  if (make_plan(d, max_seq_len, split_tokens, &pl) != HYB_OK) return 0;
  return ws_layout(d, pl, false).total;
}

static int decode_launch(const hyb_cache_desc *d, const void *q, float softmax_scale, int32_t max_seq_len,
                         int32_t split_tokens, void *workspace, size_t workspace_bytes, void *out,
                         float *lse_out, hyb_stream_t stream, const int32_t *n_new, const void *k_new,
                         const void *v_new, bool l2_skip = false) {
  Plan pl;
  const int rc = make_plan(d, max_seq_len, split_tokens, &pl);
  if (rc != HYB_OK) return rc;
  if (!q || !out || !aligned(q, 16) || !aligned(out, 16) || (lse_out && !aligned(lse_out, 4)) ||
      !std::isfinite(softmax_scale))
    return HYB_ERR_INVALID_VALUE;
  const bool step = n_new != nullptr;
  if (step && (!aligned(n_new, 4) || !k_new || !v_new || !aligned(k_new, 16) || !aligned(v_new, 16)))
    return HYB_ERR_INVALID_VALUE;
  const WsLayout wl = ws_layout(d, pl, step);
  if (wl.total > 0 && (!workspace || workspace_bytes < wl.total || !aligned(workspace, 16)))
    return HYB_ERR_WORKSPACE;
  hyb::DecodeArgs a;
  a.hot = static_cast<uint8_t *>(d->hot);
  a.cold = static_cast<uint8_t *>(d->cold);
  a.scales = d->scales;
  a.block_table = d->block_table;
  a.seq_lens = d->seq_lens;
  a.n_int4 = d->quant_bits == 8 ? d->n_int4_blocks : nullptr;
  a.status = d->status;
  a.q = static_cast<const __half *>(q);
  a.out = static_cast<__half *>(out);
  a.lse_out = lse_out;
  uint8_t *ws = static_cast<uint8_t *>(workspace);
  const bool merge_ws = !pl.cluster && pl.ns > 1;
  a.counters = merge_ws ? reinterpret_cast<int32_t *>(ws + wl.counters) : nullptr;
  a.o_part = merge_ws ? reinterpret_cast<float *>(ws + wl.o_part) : nullptr;
  a.lse_part = merge_ws ? reinterpret_cast<float *>(ws + wl.lse_part) : nullptr;
  a.n_groups = merge_ws ? wl.n_groups : 0;
  a.g_counters = a.n_groups > 0 ? reinterpret_cast<int32_t *>(ws + wl.g_counters) : nullptr;
  a.g_part = a.n_groups > 0 ? reinterpret_cast<float *>(ws + wl.g_part) : nullptr;
  a.g_lse = a.n_groups > 0 ? reinterpret_cast<float *>(ws + wl.g_lse) : nullptr;
  a.hkv = d->num_kv_heads;
  a.hq = d->num_q_heads;
  a.num_phys = d->num_phys_blocks;
  a.max_blocks = d->max_blocks_per_seq;
  a.quant_bits = d->quant_bits;
  a.hot_tokens = d->hot_tokens;
  a.lsub = lsub_of(d);
  a.bshift = bshift_of(d);
  a.n_splits = pl.ns;
  a.split_blocks = pl.tb;
  a.max_seq_len = max_seq_len;
  a.qk_scale = softmax_scale * 1.4426950408889634f;
  a.n_new = n_new;
  a.k_new = static_cast<const __half *>(k_new);
  a.v_new = static_cast<const __half *>(v_new);
  a.seq_cnt = step ? reinterpret_cast<int32_t *>(ws + wl.seq_cnt) : nullptr;
  a.l2_skip = l2_skip ? 1 : 0;
  const long long wait = g_wait_cycles.load(std::memory_order_relaxed);
  a.wait_cycles = wait > 0 ? wait : hyb::kDefaultWaitCycles;
  a.batch = d->batch;
  const bool persist = pl.persist && !l2_skip;
  a.unit_ctr = pl.persist ? reinterpret_cast<int32_t *>(ws + wl.unit_ctr) : nullptr;
  a.min_splits = pl.per_seq;
  a.defer_merge = persist && pl.defer ? 1 : 0;
  a.split_count = a.defer_merge ? reinterpret_cast<int32_t *>(ws + wl.split_count) : nullptr;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int group = d->num_q_heads / d->num_kv_heads;
  cudaError_t e = persist ? hyb::launch_decode_persist(a, group, d->batch, pl.ctas, s)
                          : hyb::launch_decode(a, group, d->batch, pl.cluster, s);
  // many splits per sequence: their merge is a launch of its own, so that no
  // CTA of the persistent kernel spends the end of the launch merging
  if (e == cudaSuccess && a.defer_merge) e = hyb::launch_persist_combine(a, group, d->batch, s);
  if (e != cudaSuccess) return cuda_fail(e);
  return HYB_OK;
}

int hyb_decode_attn(const hyb_cache_desc *d, const void *q, float softmax_scale, int32_t max_seq_len,
                    int32_t split_tokens, void *workspace, size_t workspace_bytes, void *out,
                    float *lse_out, hyb_stream_t stream) {
  return decode_launch(d, q, softmax_scale, max_seq_len, split_tokens, workspace, workspace_bytes, out,
                       lse_out, stream, nullptr, nullptr, nullptr);
}

// Workspace of hyb_decode_attn_sparse: the dense pass's workspace, then a
// log-sum-exp row per (sequence, query head), then the selection keys
// [batch][Hq][max_l2], max_l2 = the cold tokens of a max_seq_len sequence,
// then the selected positions int32 [batch][Hq][sel_stride].
struct SparseWs {
  size_t dense, lse, keys, sel, total;
  int max_l2, sel_stride;
};

static int sparse_ws(const hyb_cache_desc *d, int32_t max_seq_len, int32_t split_tokens, SparseWs *w) {
  if (split_tokens < 0) return HYB_ERR_INVALID_VALUE;  // per-sequence splits: dense calls only
  Plan pl;
  const int rc = make_plan(d, max_seq_len, split_tokens, &pl);
  if (rc != HYB_OK) return rc;
  const size_t rows = static_cast<size_t>(d->batch) * d->num_q_heads;
  const long long cold = static_cast<long long>(max_seq_len) - d->hot_tokens;
  w->max_l2 = cold > 0 ? static_cast<int>((cold + hyb::kBlock - 1) / hyb::kBlock * hyb::kBlock) : 0;
  w->dense = ws_layout(d, pl, false).total;
  w->lse = round_up(w->dense, kWsAlign);
  w->keys = w->lse + round_up(rows * sizeof(float), kWsAlign);
  w->sel = w->keys + round_up(rows * static_cast<size_t>(w->max_l2) * sizeof(float), kWsAlign);
  w->sel_stride = w->max_l2 < hyb::kMaxTopK ? (w->max_l2 > 0 ? w->max_l2 : 1) : hyb::kMaxTopK;
  w->total = w->sel + round_up(rows * static_cast<size_t>(w->sel_stride) * sizeof(int32_t), kWsAlign);
  return HYB_OK;
}

size_t hyb_decode_sparse_workspace_bytes(const hyb_cache_desc *d, int32_t max_seq_len, int32_t split_tokens) {
  SparseWs w;
  if (sparse_ws(d, max_seq_len, split_tokens, &w) != HYB_OK) return 0;
  return w.total;
}

size_t hyb_decode_sparse_selection(const hyb_cache_desc *d, int32_t max_seq_len, int32_t split_tokens,
                                   int32_t *row_stride) {
  SparseWs w;
  if (sparse_ws(d, max_seq_len, split_tokens, &w) != HYB_OK) return 0;
  if (row_stride) *row_stride = w.sel_stride;
  return w.sel;
}

int hyb_decode_attn_sparse(const hyb_cache_desc *d, const void *q, float softmax_scale, int32_t max_seq_len,
                           int32_t split_tokens, int32_t top_k, void *workspace, size_t workspace_bytes,
                           void *out, float *lse_out, hyb_stream_t stream) {
  SparseWs w;
  const int rc = sparse_ws(d, max_seq_len, split_tokens, &w);
  if (rc != HYB_OK) return rc;
  if (d->quant_bits == 0) return HYB_ERR_UNSUPPORTED;  // FP16 blocks: no L2 tier
  if (top_k < 0 || top_k > hyb::kMaxTopK) return HYB_ERR_INVALID_VALUE;
  if (!workspace || workspace_bytes < w.total || !aligned(workspace, 16)) return HYB_ERR_WORKSPACE;
  uint8_t *ws = static_cast<uint8_t *>(workspace);
  float *lse = lse_out ? lse_out : reinterpret_cast<float *>(ws + w.lse);
  const int r = decode_launch(d, q, softmax_scale, max_seq_len, split_tokens, workspace, w.dense, out, lse, stream,
                              nullptr, nullptr, nullptr, true);
  if (r != HYB_OK) return r;
  hyb::SparseArgs a;
  a.cold = static_cast<const uint8_t *>(d->cold);
  a.scales = d->scales;
  a.block_table = d->block_table;
  a.seq_lens = d->seq_lens;
  a.n_int4 = d->quant_bits == 8 ? d->n_int4_blocks : nullptr;
  a.status = d->status;
  a.q = static_cast<const __half *>(q);
  a.keys = reinterpret_cast<float *>(ws + w.keys);
  a.sel = reinterpret_cast<int32_t *>(ws + w.sel);
  a.sel_stride = w.sel_stride;
  a.out = static_cast<__half *>(out);
  a.lse = lse;
  a.hkv = d->num_kv_heads;
  a.hq = d->num_q_heads;
  a.num_phys = d->num_phys_blocks;
  a.max_blocks = d->max_blocks_per_seq;
  a.quant_bits = d->quant_bits;
  a.hot_tokens = d->hot_tokens;
  a.lsub = lsub_of(d);
  a.bshift = bshift_of(d);
  a.max_l2 = w.max_l2;
  a.top_k = top_k;
  a.blocks_per_cta = 4;
  a.qk_scale = softmax_scale * 1.4426950408889634f;
  const cudaError_t e = hyb::launch_sparse_l2(a, d->batch, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? HYB_OK : cuda_fail(e);
}

int hyb_sparse_top_k(int64_t context_length) {
  if (context_length < 0) return 0;
  const int64_t k = context_length / 256;
  return k < 128 ? static_cast<int>(k) : 128;
}

size_t hyb_decode_step_workspace_bytes(const hyb_cache_desc *d, int32_t max_seq_len, int32_t split_tokens) {
  Plan pl;
  if (make_plan(d, max_seq_len, split_tokens, &pl) != HYB_OK) return 0;
  return ws_layout(d, pl, true).total;
}

int hyb_decode_step(const hyb_cache_desc *d, const int32_t *n_new, const void *k_new, const void *v_new,
                    const void *q, float softmax_scale, int32_t max_seq_len, int32_t split_tokens,
                    void *workspace, size_t workspace_bytes, void *out, float *lse_out, hyb_stream_t stream) {
  if (!n_new) return HYB_ERR_INVALID_VALUE;
  return decode_launch(d, q, softmax_scale, max_seq_len, split_tokens, workspace, workspace_bytes, out,
                       lse_out, stream, n_new, k_new, v_new);
}

int hyb_combine(int32_t batch, int32_t num_q_heads, int32_t head_dim, int32_t n_splits,
                const float *o_partial, const float *lse_partial, void *out, float *lse_out,
                hyb_stream_t stream) {
  if (batch <= 0 || num_q_heads <= 0 || n_splits < 1 || !o_partial || !lse_partial || !out ||
      !aligned(o_partial, 16) || !aligned(lse_partial, 4) || !aligned(out, 16) ||
      (lse_out && !aligned(lse_out, 4)))
    return HYB_ERR_INVALID_VALUE;
  if (head_dim != hyb::kDim) return HYB_ERR_UNSUPPORTED;
  const long long rows = static_cast<long long>(batch) * num_q_heads;
  if (rows > 0x7fffffffLL) return HYB_ERR_INVALID_VALUE;
  hyb::CombineArgs c{o_partial, lse_partial, static_cast<__half *>(out), lse_out, n_splits};
  const cudaError_t e = hyb::launch_combine(c, static_cast<int>(rows), reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? HYB_OK : cuda_fail(e);
}

int hyb_kv_migrate(const hyb_cache_desc *d, const int32_t *target_n_int4, int32_t max_delta,
                   hyb_stream_t stream) {
  const int rc = hyb_check_desc(d);
  if (rc != HYB_OK) return rc;
  if (d->quant_bits != 8) return HYB_ERR_UNSUPPORTED;
  if (!d->n_int4_blocks || !aligned(d->n_int4_blocks, 4) || !target_n_int4 || !aligned(target_n_int4, 4) ||
      max_delta < 0 || max_delta > d->max_blocks_per_seq)
    return HYB_ERR_INVALID_VALUE;
  hyb::MigrateArgs a;
  a.cold = static_cast<uint8_t *>(d->cold);
  a.scales = d->scales;
  a.block_table = d->block_table;
  a.seq_lens = d->seq_lens;
  a.n_int4 = const_cast<int32_t *>(d->n_int4_blocks);
  a.target = target_n_int4;
  a.status = d->status;
  a.hkv = d->num_kv_heads;
  a.num_phys = d->num_phys_blocks;
  a.max_blocks = d->max_blocks_per_seq;
  a.max_delta = max_delta;
  a.hot_tokens = d->hot_tokens;
  a.lsub = lsub_of(d);
  a.bshift = bshift_of(d);
  const cudaError_t e = hyb::launch_migrate(a, d->batch, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? HYB_OK : cuda_fail(e);
}

double hyb_migration_threshold_ms(const int32_t *seq_lens, int32_t n) {
  double log_sum = 0.0;
  int used = 0;
  for (int32_t i = 0; seq_lens && i < n; i++)
    if (seq_lens[i] > 0) {
      log_sum += std::log(static_cast<double>(seq_lens[i]));
      used++;
    }
  const double load_factor = used > 0 ? std::exp(log_sum / used) / 512.0 : 0.0;
  return 3000.0 * (1.0 + 0.2 * load_factor);
}

int hyb_migration_decision(double avg_interval_ms, double threshold_ms, int32_t block_is_int4) {
  if (block_is_int4) return avg_interval_ms < threshold_ms ? 1 : 0;
  return avg_interval_ms > 1.5 * threshold_ms ? -1 : 0;
}

int hyb_read_status(const hyb_cache_desc *d, int32_t *host_status, int32_t clear, hyb_stream_t stream) {
  if (!d || !d->status || !host_status) return HYB_ERR_INVALID_VALUE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemcpyAsync(host_status, d->status, sizeof(int32_t), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e == cudaSuccess && clear) {
    e = cudaMemsetAsync(d->status, 0, sizeof(int32_t), s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  }
  return e == cudaSuccess ? HYB_OK : cuda_fail(e);
}

}  // extern "C"
