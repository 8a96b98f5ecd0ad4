/*
 * hyb_kv.h -- C ABI of the B200 (sm_100a) hybrid_v2 KV-cache decode library.
 *
 * The method: web page "DeepSeek V4混合式KV Cache推理优化实战解析" (cited as
 * [hybrid_v2 page] below).  A sequence's KV cache has two tiers:
 *   - a hot zone holding the most recent hot_tokens (32 in the page's example
 *     set; 16, 64 or 128 also built) tokens in FP16, never quantized,
 *     K and V interleaved per token, 512-byte aligned (sections 2.1, 3.1, 3.2);
 *   - a cold zone holding all earlier tokens in 64-token (or 32- or 128-token) blocks of symmetric
 *     INT8 with a block-wise scale, INT4 for the "L2" cold blocks (sections
 *     2.1, 2.2, 3.1), reached through a block table (section 3.2, block header).
 * The three fields of the hybrid_v2 contract are hot_tokens (power of two),
 * quantization_bits (4 or 8) and block_size (a multiple of 8); this library
 * implements block_size 32, 64 or 128 with hot_tokens 16, 32, 64 or 128 and
 * quantization_bits 8 or 4
 * (section 3.1; section 5.1 for the invalid-value error), and
 * quantization_bits 0, which the page's section 5.2 gives as the switch that
 * keeps the cold zone in FP16.
 *
 * Calls:
 *   hyb_kv_append      seal tokens leaving the hot zone into cold blocks
 *                      (absmax / RNE / clamp quantization) and write the new
 *                      tokens into the hot ring ([hybrid_v2 page] 4.2, step 2)
 *   hyb_decode_attn    single-query attention of q[B][Hq][d] over hot + cold,
 *                      GQA, split-KV, FP32 accumulation, FP16 output
 *                      ([hybrid_v2 page] 4.2, steps 3-5)
 *   hyb_decode_step    the two above fused: append of one token per sequence
 *                      and attention in a single launch
 *   hyb_kv_migrate     move cold blocks between the INT8 and the INT4 tier in
 *                      place with new scales ([hybrid_v2 page] 3.2, 3.3), and
 *                      hyb_migration_threshold_ms / hyb_migration_decision,
 *                      the page's adaptive migration policy (host functions)
 *   hyb_combine        log-sum-exp merge of split partial results (the merge
 *                      that replaces the page's torch.cat of step 5)
 *
 * Conventions for every call:
 *   - Pointers named "device" are CUDA device pointers the caller allocated;
 *     the library allocates no memory and keeps no pointer after a call
 *     returns.  Buffers must stay alive until the stream work completes.
 *   - Work is enqueued asynchronously on `stream` (0 = legacy default stream).
 *   - Return value: HYB_OK (0) or a negative HYB_ERR_* code; on an error
 *     return nothing was enqueued (HYB_ERR_CUDA: a launch failed; the CUDA
 *     error is kept for hyb_last_cuda_error()).
 *   - Errors found on the device (a block-table entry out of range, an n_new
 *     above max_new, a sequence outgrowing its block table, a bounded wait
 *     that ran out) never trap: the kernel skips the affected unit and records
 *     the first such HYB_STATUS_* code in the sticky device word desc->status
 *     (atomic compare-and-swap from 0).  Read it with hyb_read_status().
 *   - Not thread-safe with respect to the same cache: calls on one cache must
 *     be ordered on one stream (or by events).
 */
#ifndef HYB_KV_H
#define HYB_KV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *hyb_stream_t; /* same type as cudaStream_t */

/* return codes */
#define HYB_OK 0
#define HYB_ERR_INVALID_VALUE (-1) /* bad config value, shape, null or misaligned pointer;
                                      named after the page's CUDA_ERROR_INVALID_VALUE (3.1) */
#define HYB_ERR_UNSUPPORTED (-2)   /* valid per the page but not built: block_size not 32, 64 or 128,
                                      head_dim != 128, Hq/Hkv > 8 */
#define HYB_ERR_WORKSPACE (-3)     /* workspace missing or smaller than required */
#define HYB_ERR_CUDA (-4)          /* a CUDA runtime call or launch failed */
#define HYB_ERR_SCRATCH_LIMIT (-5) /* hyb_decode_attn_noalloc: the call needs more scratch
                                      than the library's static buffer holds */

/* device status codes (sticky, first error wins) */
#define HYB_STATUS_OK 0
#define HYB_STATUS_BAD_BLOCK 1     /* block-table entry < 0 or >= num_phys_blocks; block skipped */
#define HYB_STATUS_BAD_N_NEW 2     /* n_new[b] < 0 or > max_new; sequence b left unchanged */
#define HYB_STATUS_CAPACITY 3      /* append would need more than max_blocks_per_seq blocks;
                                      sequence b left unchanged */
#define HYB_STATUS_SEQ_LEN 4       /* seq_lens[b] < 0 or > max_seq_len at decode; b skipped */
#define HYB_STATUS_TIMEOUT 5       /* a bounded wait inside a kernel gave up; unit skipped */
#define HYB_STATUS_BAD_TIER 6      /* hyb_kv_migrate: target[b] outside [0, max_blocks_per_seq] or
                                      more than max_delta blocks from n_int4_blocks[b]; sequence
                                      left unchanged */

/*
 * The cache descriptor (host struct; the pointers inside are device memory).
 *
 * Geometry: hot_tokens HOT in {16, 32, 64, 128} (32 is the page's value),
 * block_size BLK = 32, 64 or 128 (64 is the page's value), head_dim D = 128,
 * num_kv_heads Hkv >= 1, num_q_heads Hq a multiple of Hkv with Hq/Hkv <= 8
 * (query head h reads kv head h / (Hq/Hkv)), quant_bits 8 (INT8 cold blocks;
 * logical blocks below n_int4_blocks[b] are INT4), 4 (every cold block INT4)
 * or 0 (FP16 cold blocks, nothing quantized; n_int4_blocks and scales are not
 * read).
 *
 * Token positions 0..L-1 of sequence b (L = seq_lens[b]): positions >= L-HOT
 * are hot, the others cold; cold position p lives in logical block p/BLK,
 * slot p%BLK, of physical block block_table[b][p/BLK].
 *
 * Memory layouts (all little-endian, all device memory):
 *   hot    FP16 [batch][Hkv][HOT][2][D]: per (sequence, kv head) a ring of HOT
 *          token slots, slot = position % HOT, each slot the K row (D halves)
 *          followed by the V row (D halves) -- 512 B per token, HOT * 512 B
 *          per (sequence, kv head).  Base 512-byte aligned ([hybrid_v2 page]
 *          3.2).
 *   cold   bytes [num_phys_blocks][Hkv][BLK/64][2][8192]: per physical block
 *          and kv head, per 64-token sub-block (slot t of a block is slot
 *          t % 64 of sub-block t / 64), a K tile then a V tile of 64 tokens
 *          x 128 channels; the tiles below use the sub-block's slot t.  A
 *          block's sub-blocks share its scales.  A 32-token block takes
 *          slots 0..31 of one such tile pair (BLK/64 read as 1).  Base
 *          16-byte aligned.
 *            K, INT8: token-major, code of (slot t, channel c) at t*128 + c.
 *            V, INT8: channel-major rows of 64 bytes; the 16-byte chunk
 *              holding slots 16j..16j+15 of channel c is stored at chunk
 *              position j ^ ((c/2) % 4): byte c*64 + 16*(j ^ ((c/2)%4)) + t%16.
 *            INT4 tiles use the first 4096 bytes: 4-bit two's complement
 *              codes, eight consecutive codes e = 0..7 along the packed axis
 *              per 32-bit word, code e in byte e%4, low nibble for e < 4 and
 *              high nibble for e >= 4.
 *            K, INT4: 64 bytes per token; channel c in word t*16 + c/8.
 *            V, INT4: channel-major rows of 32 bytes in four 8-byte units of
 *              16 slots, unit j stored at unit position j ^ ((c/4) % 4);
 *              slots 16j..16j+7 in the unit's first word, the rest in its
 *              second.
 *          Codes are in [-127, 127] (INT8) or [-7, 7] (INT4); -128 / -8 are
 *          never produced.  Bytes of slots not yet sealed are never written.
 *   scales FP32 [num_phys_blocks][Hkv][2]: K scale, V scale of each tile;
 *          the value of a cold element is code * scale.
 *   cold, quant_bits 0: FP16 [num_phys_blocks][Hkv][BLK][2][D]: per physical
 *          block and kv head BLK token slots in the hot ring's row layout (K
 *          row then V row, 512 B per token), BLK * 512 B per (block, kv
 *          head); slot t at byte t*512.  Base 16-byte aligned.
 *   block_table int32 [batch][max_blocks_per_seq]; entries for blocks a
 *          sequence does not reach are ignored.  A block that appends write
 *          into must belong to one sequence only.
 *   seq_lens int32 [batch]: tokens in each sequence; hyb_kv_append advances it.
 *   n_int4_blocks int32 [batch] or NULL: logical blocks below it are INT4
 *          ("L2" blocks, [hybrid_v2 page] 2.2 / 3.1).  A block's format is
 *          fixed when its first token is sealed; do not change n_int4_blocks
 *          for blocks that already hold tokens.
 *   status int32 device word, 0 = ok (see HYB_STATUS_*).
 * A fresh cache is: seq_lens all 0, status 0 (contents of hot / cold / scales
 * do not matter).
 */
typedef struct hyb_cache_desc {
  int32_t hot_tokens;         /* 16, 32, 64 or 128 */
  int32_t block_size;         /* 32, 64 or 128 */
  int32_t head_dim;           /* must be 128 */
  int32_t quant_bits;         /* 8, 4 or 0 (FP16 cold blocks) */
  int32_t num_kv_heads;       /* Hkv >= 1 */
  int32_t num_q_heads;        /* Hq, multiple of Hkv, Hq/Hkv <= 8 */
  int32_t num_phys_blocks;    /* physical blocks in `cold` / `scales` */
  int32_t max_blocks_per_seq; /* columns of block_table */
  int32_t batch;              /* sequences */
  int32_t reserved;           /* set to 0 */
  void *hot;                  /* device, see above */
  void *cold;                 /* device */
  float *scales;              /* device */
  const int32_t *block_table; /* device */
  int32_t *seq_lens;          /* device */
  const int32_t *n_int4_blocks; /* device or NULL */
  int32_t *status;            /* device */
} hyb_cache_desc;

/*
 * Host-only check of a descriptor (no GPU needed, nothing enqueued).
 * Returns HYB_OK, HYB_ERR_INVALID_VALUE (hot_tokens not a power of two in
 * {16, 32, 64, 128}, block_size not a multiple of 8, quant_bits not 8, 4 or 0,
 * non-positive sizes, Hq not a multiple of Hkv, null or misaligned pointers)
 * or HYB_ERR_UNSUPPORTED (a valid configuration with block_size not 32, 64 or 128, or
 * head_dim != 128, or Hq/Hkv > 8).  The contract is the page's section 3.1
 * and 5.1 (quant_bits 0: section 5.2).
 */
int hyb_check_desc(const hyb_cache_desc *desc);

/*
 * Append n_new[b] tokens to every sequence b ([hybrid_v2 page] 4.2 step 2,
 * quantize_int8, and 2.1 / 3.2 for the tiers).
 *   n_new  device int32 [batch], each in [0, max_new].
 *   k_new, v_new  device FP16 [batch][max_new][Hkv][D]; row j of sequence b
 *          is position seq_lens[b] + j.  Rows j >= n_new[b] are not read.
 *          16-byte aligned.
 * For L_old = seq_lens[b] and L_new = L_old + n_new[b], the positions
 * max(0, L_old-HOT) .. max(0, L_new-HOT)-1 leave the hot zone in ascending
 * order (their FP16 values come from the hot ring, or straight from k_new /
 * v_new for new tokens that never become hot).  They are grouped by logical
 * block; per group, kv head and K|V:
 *   a   = max |x| over the group's tokens and channels (FP32, exact),
 *   s_c = a / Q in IEEE FP32 (Q = 127, or 7 for INT4 blocks),
 *   if the block held no token: s = s_c;
 *   else if s_c > s_old: every code c already in the block becomes
 *        clamp(rint((c * s_old) / s_c), -Q, Q) and s = s_c;
 *   else s = s_old;
 *   new codes = (s == 0) ? 0 : clamp(rint(x / s), -Q, Q)   (rint: half to even).
 * (quant_bits 0: the rows are copied unchanged, no scale.)  Then the newest
 * min(n_new[b], HOT) tokens are written to hot slots position % HOT and
 * seq_lens[b] = L_new.  The result is bit-exact and does
 * not depend on the launch configuration.
 * Device errors: HYB_STATUS_BAD_N_NEW or HYB_STATUS_CAPACITY (sequence
 * untouched), HYB_STATUS_BAD_BLOCK (that block skipped, seq_lens still
 * advanced -- the cache is then damaged and must be rebuilt).
 */
int hyb_kv_append(const hyb_cache_desc *desc, const int32_t *n_new, int32_t max_new,
                  const void *k_new, const void *v_new, hyb_stream_t stream);

/*
 * Split planning for hyb_decode_attn (host only).  max_seq_len is a host
 * upper bound of seq_lens[b]; split_tokens is a multiple of BLK (tokens per
 * split of the cold range) or 0 for automatic.  A sequence's cold blocks are
 * cut into runs of tb = split_tokens / BLK blocks; the last split also
 * attends the hot ring, whose ceil(min(L, HOT) / 32) items of 32 FP16 rows
 * count as h = min(tb, ceil(items / I)) blocks (I = items per block: 1 for
 * INT8/INT4 blocks of 32 or 64 tokens, 2 for 128-token blocks, BLK / 32 for
 * FP16 blocks), so that no split holds more than tb blocks' worth of items.
 * A sequence's splits follow that rule in the kernels that take one CTA per
 * split; the persistent kernel (several waves, 64-token INT8/INT4 blocks)
 * cuts sequence b's c_b = nblk_b + h_b items into S_b = max(1, ceil(c_b /
 * tb)) runs of near-equal length instead -- split s takes items
 * [floor(s c_b / S_b), floor((s + 1) c_b / S_b)), the ring being the last --
 * the same count of splits, none longer than tb blocks.
 * Writes the split size used and the number of splits per sequence,
 * n_splits = max(1, ceil((nblk + h) / tb)), nblk = ceil(max(0, max_seq_len -
 * HOT) / BLK).  Returns HYB_OK or HYB_ERR_INVALID_VALUE.  The automatic
 * choice depends on the GPU's SM count (device 0 of the current context
 * when none is current).
 * split_tokens = -n (1 <= n <= 65535) asks for per-sequence splits: a
 * sequence with nblk_b cold blocks counts c_b = nblk_b + 1 items (the hot
 * ring as one; c_b = 0 when it is empty) and is cut into
 * S_b = min(c_b, max(n, ceil(c_b / 32))) splits of near-equal length --
 * split s takes items [floor(s c_b / S_b), floor((s + 1) c_b / S_b)), the
 * ring being the last -- so every sequence with at least n blocks gets at
 * least n splits of at most 32 blocks, as long as the longest allows.  Then
 * n_splits = S for c = nblk + 1 of max_seq_len, and split_tokens_out is the
 * longest sequence's split length (ceil(c / n_splits) blocks).  This needs
 * 64-token INT8/INT4 blocks and batch <= 256 (the persistent kernel); other
 * caches take the longest sequence's split length for every sequence
 * (n_splits and split_tokens_out as for split_tokens = that length).
 * hyb_decode_attn_sparse does not take it (HYB_ERR_INVALID_VALUE).
 */
int hyb_decode_plan(const hyb_cache_desc *desc, int32_t max_seq_len, int32_t split_tokens,
                    int32_t *split_tokens_out, int32_t *n_splits_out);

/*
 * Which decode kernel hyb_decode_attn / hyb_decode_step launch for these
 * arguments (host only; the same plan as hyb_decode_plan):
 *   HYB_KERNEL_SPLIT_CTA   one CTA per (split, kv head, sequence), splits
 *                          merged through the workspace by the last to finish;
 *   HYB_KERNEL_CLUSTER     the same CTAs, the splits of a (sequence, kv head)
 *                          one thread-block cluster merged in distributed
 *                          shared memory;
 *   HYB_KERNEL_PERSISTENT  `ctas` resident CTAs that take the splits as work
 *                          units from a counter (64-token INT8/INT4 blocks,
 *                          batch <= 256, splits of at most 32 blocks), the
 *                          splits merged inside the launch;
 *   HYB_KERNEL_PERSISTENT_COMBINE  the same kernel when a sequence may have
 *                          more than 16 splits: it writes every split's
 *                          partial and a second launch (one CTA per query
 *                          head and sequence) merges them by log-sum-exp.
 * Writes the kernel, the CTAs of the launch and the CTAs one SM holds (the
 * device's occupancy for that kernel; 0 when no device can be queried).  Any
 * output pointer may be NULL.  Returns HYB_OK or HYB_ERR_INVALID_VALUE (the
 * cases hyb_decode_plan rejects).  A benchmark or a scheduler reads it; the
 * attention calls do not need it.
 */
#define HYB_KERNEL_SPLIT_CTA 0
#define HYB_KERNEL_CLUSTER 1
#define HYB_KERNEL_PERSISTENT 2
#define HYB_KERNEL_PERSISTENT_COMBINE 3
int hyb_decode_launch_info(const hyb_cache_desc *desc, int32_t max_seq_len, int32_t split_tokens,
                           int32_t *kernel, int32_t *ctas, int32_t *ctas_per_sm);

/* Bytes of workspace hyb_decode_attn needs for these arguments, or 0 with an
 * invalid descriptor.  It is 0 when each sequence takes one split, or when
 * the splits of every (sequence, kv head) run as one thread-block cluster
 * (2..16 splits, all clusters resident on the GPU at once) and are merged
 * through distributed shared memory. */
size_t hyb_decode_workspace_bytes(const hyb_cache_desc *desc, int32_t max_seq_len,
                                  int32_t split_tokens);

/*
 * Single-query decode attention over hot + cold ([hybrid_v2 page] 4.2 steps
 * 3-5; one softmax over all L keys of each sequence, no mask):
 *   out[b][h] = sum_j softmax_j(z) V_j,  z_j = softmax_scale * (q[b][h] . K_j),
 *   K_j, V_j = FP16 hot values, or code * scale for cold positions, of kv
 *   head h / (Hq/Hkv).
 *   q        device FP16 [batch][Hq][D], 16-byte aligned.
 *   softmax_scale  finite, usually 1/sqrt(D).
 *   max_seq_len    host upper bound of seq_lens (a larger device value sets
 *            HYB_STATUS_SEQ_LEN and that sequence is skipped).
 *   split_tokens   multiple of BLK, 0 = automatic, or -n = at least n splits
 *            per sequence (hyb_decode_plan).
 *   workspace, workspace_bytes  device scratch of at least
 *            hyb_decode_workspace_bytes() bytes (may be NULL when that is 0),
 *            16-byte aligned.  It must be zero-filled before its first use;
 *            every completed call leaves it ready for the next one (its
 *            arrival counters back at zero).  Calls that share a workspace
 *            must not overlap on the GPU.
 *   out      device FP16 [batch][Hq][D] (round to nearest even), 16-byte aligned.
 *   lse_out  device FP32 [batch][Hq] natural-log log-sum-exp of the logits, or NULL.
 * An empty sequence (L = 0) gives out = 0 and lse = -inf.
 * Launches (hyb_decode_launch_info tells which): one wave of splits -- one
 * CTA per (split, kv head, sequence); when a (sequence, kv head) has 2..16
 * splits whose clusters can all be resident, its splits form a thread-block
 * cluster and are merged by log-sum-exp (the same merge as hyb_combine)
 * through distributed shared memory, otherwise the last CTA of a (sequence,
 * kv head) to finish merges them through the workspace.  Several waves, or
 * per-sequence splits -- the persistent kernel: resident CTAs take the splits
 * as work units; up to 16 splits per sequence are merged inside the launch
 * (by the unit that finishes last), more by a second launch (one CTA per
 * query head and sequence) after it.
 * Arithmetic (tensor cores, warp-level mma): cold dot products run exactly
 * in integers -- q in 24-bit fixed point per head (relative to its largest
 * channel) against the codes, and softmax weights in 16-bit fixed point
 * relative to the maximum of their 16-token group against the V codes; FP16
 * rows (hot ring, FP16 cold blocks) with FP16 weights relative to their
 * 8-row group's maximum and FP32 accumulation; the online softmax, the
 * per-block scale products and all merges in FP32.  Accuracy versus exact
 * FP64 attention on the same cache: max-abs error <= 2e-3 and per-row
 * relative L2 <= 1e-3 on the measured workloads, an attention sink 12 nats
 * above a 32K-token tail and a q with one channel 100x the others.
 */
int hyb_decode_attn(const hyb_cache_desc *desc, const void *q, float softmax_scale,
                    int32_t max_seq_len, int32_t split_tokens, void *workspace,
                    size_t workspace_bytes, void *out, float *lse_out, hyb_stream_t stream);

/*
 * Sparse L2 decode attention ([hybrid_v2 page] 2.2: the L2 cold blocks keep
 * only the KV of the top-k attention scores; 5.3: sparse_top_k).  As
 * hyb_decode_attn, except that of the tokens a sequence holds in its INT4
 * ("L2") blocks -- logical blocks below n_int4_blocks[b] (quant_bits 8), every
 * cold block (quant_bits 4) -- each query head attends only the top_k with
 * the largest attention scores (logits), plus every other token.  The
 * selection ranks by a key that approximates the logit:
 *   key_j = (float)(sum_c qi_c * Kcode_j,c) * Kscale_j   (FP32, one rounding
 *           per operation; -0 counts as +0; negated for a negative
 *           softmax_scale),
 *   qi_c  = clamp(rint(q_c * (32767 / max_c |q_c|)), -32767, 32767),
 * the head's q in 16-bit fixed point; equal keys keep the older position.
 * So a kept token's logit is never below an unselected token's by more than
 * their two key errors, |softmax_scale| * max|q| / 32767 * 0.502 * Kscale_j
 * * sum_c |Kcode_j,c| + 2^-22 * |logit_j| each (where two logits are closer
 * than that, either choice is a correct top-k).  All L2 tokens are attended
 * when there are at most top_k of them; top_k 0 attends none.  The selection
 * is left in the workspace (hyb_decode_sparse_selection).  Accuracy as
 * hyb_decode_attn over the selected set.
 *   top_k      0 .. 1024 (the page's default is 32; see hyb_sparse_top_k).
 *   workspace  at least hyb_decode_sparse_workspace_bytes() bytes, 16-byte
 *              aligned, zero-filled before its first use (its leading part is
 *              the dense pass's workspace); holds the keys of every L2 token.
 * Launches: the decode kernel over everything but the L2 blocks, a scoring
 * kernel over the L2 blocks' INT4 K tiles, and a top-k kernel per (sequence,
 * query head) that selects, attends the selected tokens' V and merges with
 * the dense result by log-sum-exp.
 * Returns as hyb_decode_attn, plus HYB_ERR_UNSUPPORTED for quant_bits 0 (FP16
 * cold blocks have no L2 tier) and HYB_ERR_INVALID_VALUE for top_k outside
 * 0..1024.
 */
int hyb_decode_attn_sparse(const hyb_cache_desc *desc, const void *q, float softmax_scale,
                           int32_t max_seq_len, int32_t split_tokens, int32_t top_k, void *workspace,
                           size_t workspace_bytes, void *out, float *lse_out, hyb_stream_t stream);

/* Bytes of workspace hyb_decode_attn_sparse needs (0 with an invalid descriptor). */
size_t hyb_decode_sparse_workspace_bytes(const hyb_cache_desc *desc, int32_t max_seq_len,
                                         int32_t split_tokens);

/*
 * Where hyb_decode_attn_sparse leaves its selection ([hybrid_v2 page] 2.2:
 * which L2 tokens each query head kept).  Returns the byte offset, inside a
 * workspace sized by hyb_decode_sparse_workspace_bytes() for the same
 * (desc, max_seq_len, split_tokens), of an int32 array [batch][Hq][stride]
 * (*row_stride = stride, at most 1024): after a call with top_k > 0, row
 * (b, h) holds in its first min(top_k, L2 tokens of b) entries the positions
 * attended, ascending (a position p < L2 tokens of b is token p of the
 * sequence); other entries, and every entry of a row whose sequence has no
 * L2 token or of a call with top_k 0, are left as they were.  The offset is
 * never 0 for a valid descriptor; 0 means invalid arguments.  Host only;
 * reading the array is the caller's (device memory, after the stream
 * completes).
 */
size_t hyb_decode_sparse_selection(const hyb_cache_desc *desc, int32_t max_seq_len, int32_t split_tokens,
                                   int32_t *row_stride);

/* The page's sparse_top_k rule ([hybrid_v2 page] 5.3): min(128,
 * context_length / 256) (0 for a negative length).  Host only. */
int hyb_sparse_top_k(int64_t context_length);

/*
 * hyb_decode_attn without a caller-provided workspace (the pages have no
 * counterpart: this is an integration convenience).  For callers that cannot
 * allocate device memory when they run attention -- code handed a fixed
 * device-memory budget at start-up, plugins whose host application owns the
 * allocator, decode loops where an allocation could block or fail -- the
 * scratch comes from one static device array compiled into the library
 * (hyb_noalloc_scratch_limit() bytes, 4 MiB, held by every GPU that loads the
 * library until the process exits).  Same arguments and results as
 * hyb_decode_attn minus the workspace.
 *   - Allocates nothing (no cudaMalloc / cudaFree).
 *   - The first call on a device looks up the array's device address for that
 *     device; make that first call before any stream capture on the device.
 *   - All calls on a device share the array and it keeps the last call's
 *     contents; each call clears the part that must start at zero.  Calls
 *     that overlap on the GPU race on the array: order them (one stream, or
 *     events).
 *   - Returns HYB_ERR_SCRATCH_LIMIT, enqueuing nothing, when the problem
 *     needs more scratch than the limit (hyb_decode_workspace_bytes() >
 *     hyb_noalloc_scratch_limit()).
 */
int hyb_decode_attn_noalloc(const hyb_cache_desc *desc, const void *q, float softmax_scale,
                            int32_t max_seq_len, int32_t split_tokens, void *out, float *lse_out,
                            hyb_stream_t stream);

/* Bytes of the static scratch array behind hyb_decode_attn_noalloc. */
size_t hyb_noalloc_scratch_limit(void);

/*
 * One decode step in one launch (two when the attention's splits are merged
 * by a launch of their own, as hyb_decode_attn says): hyb_kv_append of
 * n_new[b] in {0, 1} tokens
 * followed by hyb_decode_attn over the grown cache ([hybrid_v2 page] 4.2,
 * steps 2-5 fused).  The CTA that attends a sequence's tail block and hot ring
 * seals the token leaving the hot zone inside its staged copies (same
 * arithmetic as hyb_kv_append, bit-exact), writes the changed codes, scale
 * and ring slot back, and attends the updated copies; seq_lens[b] is
 * advanced by the last CTA of the sequence (persistent kernel: by the last
 * CTA of the launch).
 *   n_new    device int32 [batch], each 0 or 1 (other values: that sequence
 *            gets HYB_STATUS_BAD_N_NEW and is attended without appending).
 *   k_new, v_new  device FP16 [batch][1][Hkv][D] (the hyb_kv_append layout
 *            with max_new = 1), 16-byte aligned.
 *   max_seq_len   host upper bound of the lengths AFTER the append.
 *   workspace     at least hyb_decode_step_workspace_bytes() bytes (never 0:
 *            it holds a counter per sequence), zero-filled before first use,
 *            left ready for the next call; calls sharing it must not overlap.
 * Other arguments and the result as for hyb_decode_attn.
 */
int hyb_decode_step(const hyb_cache_desc *desc, const int32_t *n_new, const void *k_new,
                    const void *v_new, const void *q, float softmax_scale, int32_t max_seq_len,
                    int32_t split_tokens, void *workspace, size_t workspace_bytes, void *out,
                    float *lse_out, hyb_stream_t stream);

/* Bytes of workspace hyb_decode_step needs for these arguments (0 with an
 * invalid descriptor). */
size_t hyb_decode_step_workspace_bytes(const hyb_cache_desc *desc, int32_t max_seq_len,
                                       int32_t split_tokens);

/*
 * Log-sum-exp merge of split partial results ([hybrid_v2 page] 4.2 step 5,
 * done as a softmax merge):
 *   rows = batch * num_q_heads;  o_partial device FP32 [rows][n_splits][D],
 *   each split's normalised output; lse_partial device FP32 [rows][n_splits]
 *   (natural log, -inf for an empty split).
 *   out[r] = sum_s w_s o_s / sum_s w_s with w_s = exp(lse_s - max_s lse_s),
 *   written as FP16 [rows][D]; lse_out[r] = max + log(sum_s w_s) (FP32, or
 *   NULL).  All-empty rows give 0 and -inf.
 * head_dim must be 128; n_splits >= 1.
 */
int hyb_combine(int32_t batch, int32_t num_q_heads, int32_t head_dim, int32_t n_splits,
                const float *o_partial, const float *lse_partial, void *out, float *lse_out,
                hyb_stream_t stream);

/*
 * hyb_kv_migrate -- move cold blocks between the INT8 ("L1") and the INT4
 * ("L2") tier in place ([hybrid_v2 page] 3.3: blocks are promoted or demoted
 * by their access interval; 3.2: a block that changes tier is given a new
 * scale inside the kernel, with no host copy).
 *
 * The tier is a count per sequence: logical blocks below n_int4_blocks[b]
 * are INT4.  For every sequence that count moves to target_n_int4[b]; each
 * block holding a sealed token between the old and the new count is
 * re-quantized to the other width, per (kv head, K|V):
 *   scale' = max|code * scale| / Q'   (Q' = 7 or 127, IEEE FP32 division)
 *   code'  = clamp(round-half-even(code * scale / scale'), -Q', Q')
 * -- the arithmetic of a tail block's re-quantization in hyb_kv_append; an
 * all-zero tile gets scale 0.  A demoted tile is rewritten in INT4 in its
 * first 4096 bytes and its other 4096 bytes are zeroed; a promoted tile is
 * rewritten whole; slots not yet sealed get code 0.  Blocks with nothing
 * sealed only change tier (later appends seal into them at the new width).
 * Then n_int4_blocks[b] = target_n_int4[b].  Moving a tier back does not
 * restore precision an INT4 round lost.
 *
 *   desc           quant_bits 8 and n_int4_blocks non-NULL; this is the one
 *                  call that writes through desc->n_int4_blocks.
 *   target_n_int4  device int32 [batch], 4-byte aligned, each in
 *                  [0, max_blocks_per_seq].
 *   max_delta      host upper bound of |target_n_int4[b] - n_int4_blocks[b]|
 *                  over the batch (it sizes the grid), 0..max_blocks_per_seq.
 * Returns HYB_OK, HYB_ERR_INVALID_VALUE (bad descriptor, NULL n_int4_blocks,
 * NULL or misaligned target, max_delta out of range), HYB_ERR_UNSUPPORTED
 * (quant_bits 4: every block is INT4 already; quant_bits 0: FP16 blocks have
 * no tiers) or HYB_ERR_CUDA.  Device
 * errors: HYB_STATUS_BAD_TIER (that sequence left unchanged) and
 * HYB_STATUS_BAD_BLOCK (that block skipped).  Asynchronous on `stream`; it
 * must not overlap on the GPU with any other call on the same cache.
 */
int hyb_kv_migrate(const hyb_cache_desc *desc, const int32_t *target_n_int4, int32_t max_delta,
                   hyb_stream_t stream);

/*
 * The adaptive migration threshold of [hybrid_v2 page] 3.3, in ms (host
 * function, no GPU): 3000 * (1 + 0.2 * load_factor), load_factor = geometric
 * mean of the batch's sequence lengths / 512.  seq_lens is a HOST array of n
 * entries; lengths <= 0 are left out of the mean (none left: load_factor 0).
 * Returns 3000 for n <= 0 or a NULL array.
 */
double hyb_migration_threshold_ms(const int32_t *seq_lens, int32_t n);

/*
 * The page's decision for one block (host function): +1 promote an INT4
 * block whose mean access interval is below the threshold, -1 demote an INT8
 * block whose mean interval is above 1.5 x the threshold, 0 otherwise.
 */
int hyb_migration_decision(double avg_interval_ms, double threshold_ms, int32_t block_is_int4);

/* Copy the device status word to *host_status (waits for `stream`), and
 * reset it to 0 when `clear` is nonzero. */
int hyb_read_status(const hyb_cache_desc *desc, int32_t *host_status, int32_t clear,
                    hyb_stream_t stream);

/*
 * Limit, in SM clock cycles, of each bounded wait of the decode kernel's
 * copy pipeline (a stage's data landing, a stage being released), for every
 * later hyb_decode_attn / hyb_decode_step / hyb_decode_attn_sparse /
 * hyb_decode_attn_noalloc launch of this process.  cycles <= 0 restores the
 * default, 2^31 cycles (about 1 s at B200 clocks).  No counterpart in the
 * pages: it exists so that the timeout path can be exercised -- with a limit
 * of a few cycles the first wait gives up, the kernel records
 * HYB_STATUS_TIMEOUT, lets every bulk copy it issued land (that drain wait
 * always keeps the default limit), and returns with its rows' output zero
 * and log-sum-exp -inf.  A timed-out hyb_decode_step may have appended its
 * token to some kv heads and not others; the status word says the step
 * failed.  Host only; takes effect at the next launch.  Returns HYB_OK.
 */
int hyb_set_wait_limit(int64_t cycles);

/* Text of a HYB_ERR_* return code or HYB_STATUS_* code (status codes are
 * passed as 100 + code). Never NULL. */
const char *hyb_strerror(int code);

/* CUDA error number behind the last HYB_ERR_CUDA of this thread (0 if none). */
int hyb_last_cuda_error(void);

/* Library version, 10000*major + 100*minor + patch. */
int hyb_version(void);

#ifdef __cplusplus
}
#endif

#endif /* HYB_KV_H */
