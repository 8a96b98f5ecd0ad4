// kernels.cuh -- argument blocks and launchers of the hybrid_v2 kernels
// (shared by the kernels and the C-ABI layer).
#pragma once

#include <cuda_runtime.h>

#include "common.cuh"

namespace hyb {

struct AppendArgs {
  __half *hot;                // FP16 [batch][Hkv][hot][2][128]
  uint8_t *cold;              // [num_phys][Hkv][sub][2][8192] (quant_bits 0: FP16 [num_phys][Hkv][block][2][128])
  float *scales;              // [num_phys][Hkv][2]
  const int32_t *block_table; // [batch][max_blocks]
  int32_t *seq_lens;          // [batch]
  const int32_t *n_int4;      // [batch] or null
  int32_t *status;
  const int32_t *n_new;       // [batch]
  const __half *k_new;        // FP16 [batch][max_new][Hkv][128]
  const __half *v_new;
  int hkv, num_phys, max_blocks, quant_bits, max_new;
  int hot_tokens;             // hot-zone tokens (power of two, 16..128)
  int lsub;                   // log2 of the 64-token sub-blocks per block (block_size 32, 64: 0; 128: 1)
  int bshift;                 // log2 of the tokens per block (block_size 32: 5, 64: 6, 128: 7)
};

struct DecodeArgs {
  uint8_t *hot;               // written only by the fused step (new token)
  uint8_t *cold;              // written only by the fused step (sealed token)
  float *scales;
  const int32_t *block_table;
  int32_t *seq_lens;          // advanced only by the fused step
  const int32_t *n_int4;
  int32_t *status;
  const __half *q;            // FP16 [batch][Hq][128]
  __half *out;                // FP16 [batch][Hq][128]
  float *lse_out;             // [batch][Hq] or null
  float *o_part;              // [batch][Hq][n_splits][128] (n_splits > 1)
  float *lse_part;            // [batch][Hq][n_splits], log2 domain
  int32_t *counters;          // [batch][Hkv] arrivals per (sequence, kv head), zero between calls
  // more than kMergeFan splits: the splits are merged in groups of kMergeFan
  // first; group results [batch][Hq][n_groups][128] and their log2-sum-exp,
  // arrival counters per group [batch][Hkv][n_groups] (zero between calls)
  float *g_part;
  float *g_lse;
  int32_t *g_counters;
  int n_groups;
  int hkv, hq, num_phys, max_blocks, quant_bits, n_splits, split_blocks, max_seq_len;
  int hot_tokens;             // hot-zone tokens (power of two, 16..128)
  int lsub;                   // log2 of the 64-token sub-blocks per block
  int bshift;                 // log2 of the tokens per block
  float qk_scale;             // softmax_scale * log2(e)
  // fused decode step (null for attention only): append n_new[b] in {0, 1}
  // tokens first; k_new / v_new FP16 [batch][Hkv][128]; seq_cnt [batch]
  // counts the CTAs that have read seq_lens[b] (zero between calls)
  const int32_t *n_new;
  const __half *k_new;
  const __half *v_new;
  int32_t *seq_cnt;
  // sparse L2 mode: the INT4 ("L2") blocks are left out of this pass (they
  // are attended by the top-k kernels of sparse.cu)
  int l2_skip;
  // limit (SM cycles) of the copy pipeline's bounded waits
  long long wait_cycles;
  // persistent kernel: [0] work-unit counter, [1] exit counter of the CTAs
  // (zero between calls; the last CTA to exit resets both) and the batch
  int32_t *unit_ctr;
  int batch;
  // persistent kernel: > 0 = per-sequence splits (per_seq_splits), at least
  // this many per sequence; 0 = runs of split_blocks blocks
  int min_splits;
  // persistent kernel: every unit writes its partial, the unit of split 0
  // writes the sequence's split count into split_count[sequence][kv head],
  // and persist_combine_kernel merges them after the launch (no arrivals)
  int defer_merge;
  int32_t *split_count;
};

// Persistent decode kernel limits: blocks per split (one block-table entry
// per producer lane) and sequences per call (their lengths are staged in
// shared memory).
constexpr int kPMaxSplitBlocks = 32;

// Per-sequence splits: a sequence of nblk cold blocks and a non-empty hot
// ring counts c = nblk + 1 items (the ring as one), and is cut into
// per_seq_splits(c, n) splits of near-equal length -- split s covers items
// [s * c / S, (s + 1) * c / S) (floor), the ring being the last item -- at
// least n of them (one per item when c < n), at most kPMaxSplitBlocks items
// each.  Non-decreasing in c.
__host__ __device__ inline int per_seq_splits(long long c, long long n) {
  if (c <= 0) return 1;
  long long s = (c + kPMaxSplitBlocks - 1) / kPMaxSplitBlocks;
  if (s < n) s = n;
  if (s > c) s = c;
  return static_cast<int>(s);
}
constexpr int kPMaxBatch = 256;

struct MigrateArgs {
  uint8_t *cold;              // [num_phys][Hkv][2][8192]
  float *scales;              // [num_phys][Hkv][2]
  const int32_t *block_table; // [batch][max_blocks]
  const int32_t *seq_lens;    // [batch]
  int32_t *n_int4;            // [batch]: INT4 blocks per sequence, moved to target
  const int32_t *target;      // [batch]
  int32_t *status;
  int hkv, num_phys, max_blocks, max_delta;
  int hot_tokens;             // hot-zone tokens
  int lsub;                   // log2 of the 64-token sub-blocks per block
  int bshift;                 // log2 of the tokens per block
};

// Sparse L2 attention (top-k of the INT4-block tokens per query head).
struct SparseArgs {
  const uint8_t *cold;        // [num_phys][Hkv][2][8192]
  const float *scales;        // [num_phys][Hkv][2]
  const int32_t *block_table; // [batch][max_blocks]
  const int32_t *seq_lens;    // [batch]
  const int32_t *n_int4;      // [batch] or null
  int32_t *status;
  const __half *q;            // FP16 [batch][Hq][128]
  float *keys;                // [batch][Hq][max_l2] selection keys (workspace)
  __half *out;                // FP16 [batch][Hq][128]: the dense pass's result in, the merged result out
  float *lse;                 // [batch][Hq]: the dense pass's log-sum-exp in, merged out (natural log)
  int32_t *sel;               // [batch][Hq][sel_stride]: the selected L2 positions, ascending (workspace)
  int sel_stride;
  int hkv, hq, num_phys, max_blocks, quant_bits, hot_tokens, max_l2, top_k, blocks_per_cta;
  int lsub;                   // log2 of the 64-token sub-blocks per block
  int bshift;                 // log2 of the tokens per block
  float qk_scale;             // softmax_scale * log2(e)
};

// Largest top_k of the sparse L2 mode (the selected positions live in shared memory).
constexpr int kMaxTopK = 1024;

struct CombineArgs {
  const float *o_part;        // [rows][n_splits][128]
  const float *lse_part;      // [rows][n_splits]
  __half *out;                // [rows][128]
  float *lse_out;             // [rows] or null
  int n_splits;
};

// Partial results merged per round (and per group when there are more).
constexpr int kMergeFan = 16;

// Default limit of a bounded wait: 2^31 SM cycles, about 1 s at B200 clocks.
constexpr long long kDefaultWaitCycles = 1ll << 31;

cudaError_t launch_append(const AppendArgs &a, int batch, cudaStream_t stream);
cudaError_t launch_decode(const DecodeArgs &a, int group, int batch, bool cluster, cudaStream_t stream);
cudaError_t launch_decode_persist(const DecodeArgs &a, int group, int batch, int ctas, cudaStream_t stream);
int decode_persist_ctas_per_sm(int group);
// The log-sum-exp merge after a persistent launch with defer_merge: one CTA
// per (query head, sequence) merges its split_count[] splits.
cudaError_t launch_persist_combine(const DecodeArgs &a, int group, int batch, cudaStream_t stream);
cudaError_t launch_migrate(const MigrateArgs &a, int batch, cudaStream_t stream);
cudaError_t launch_combine(const CombineArgs &a, int rows, cudaStream_t stream);
cudaError_t launch_sparse_l2(const SparseArgs &a, int batch, cudaStream_t stream);
// hyb_stream_read: one streaming read of `bytes` (a multiple of 16) at src,
// grid CTAs of kStreamReadThreads threads
constexpr int kStreamReadThreads = 256;
constexpr int kStreamReadCtasPerSm = 8;
cudaError_t launch_stream_read(const void *src, size_t bytes, uint32_t *sink, int grid, cudaStream_t stream);
int decode_max_split_blocks();
int decode_ctas_per_sm(int group);
int decode_max_cluster();
int decode_resident_clusters(int group, int csize);
size_t decode_ws_zero_prefix(const hyb_cache_desc *d, int32_t max_seq_len, int32_t split_tokens);

}  // namespace hyb
