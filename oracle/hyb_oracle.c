/*
 * hyb_oracle.c -- CPU oracle for the hybrid_v2 two-tier KV cache.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
 * cpu_baseline / reference legs of bench.py may load this library.  The GPU
 * library never links, calls or includes anything from here, and this file
 * includes nothing from the GPU side.
 *
 * What it computes (source: the web page "DeepSeek V4混合式KV Cache推理优化实战解析",
 * cited below as [hybrid_v2 page] with its section numbers):
 *   - The hybrid_v2 cache contract (section 3.1): hot zone of 32 tokens kept in
 *     FP16 and never quantized; cold zone in 64-token blocks of INT8 (INT4 for
 *     "L2" cold blocks) with a block-wise scale (sections 2.1, 2.2, 3.2).
 *   - The hot zone is the MOST RECENT 32 tokens (section 2.1).  (The vLLM
 *     snippet of section 4.2 slices the first 32 instead; the prose wins.)
 *   - Quantization of the cold part (section 4.2, "quantize_int8"): symmetric
 *     absmax scaling, one FP32 scale per (block, kv-head, K|V),
 *     scale = absmax / Q with Q = 127 (INT8) or 7 (INT4), codes =
 *     clamp(round-half-even(x / scale), -Q, Q).
 *   - A block that is filled over several calls keeps one scale: when newly
 *     sealed tokens need a larger scale, the codes already in the block are
 *     re-quantized to the new scale in place (section 3.2 says a re-tiered
 *     block gets a new INT8 scale assigned in the kernel; the page is silent on
 *     partial blocks -- this is the plainest reading that keeps the block
 *     layout fixed).
 *   - quantization_bits 0 (section 5.2: quantization switched off, the cold
 *     zone kept in FP16): sealed tokens keep their FP16 values in the block.
 *   - Sparse "L2" blocks (section 2.2: the L2 cold blocks keep only the KV of
 *     the top-k attention scores; section 5.3: sparse_top_k, default 32, and
 *     the rule min(128, context_length / 256)): in ora_decode_topk each query
 *     head attends, of the tokens in its sequence's INT4 blocks, only the
 *     top_k with the largest attention scores, plus every other token.  The
 *     score of a token is its attention logit, softmax_scale * sum_c q_c *
 *     (code_c * scale), in FP64 -- the same number the softmax below uses.
 *     Equal scores keep the older position first.  ora_decode_sel attends a
 *     given selection instead (any valid top-k set, for a caller whose
 *     selection may resolve near-ties differently), and ora_l2_scores returns
 *     the scores themselves.
 *   - Attention (section 4.2, steps 3-5): one softmax over hot and cold keys
 *     together, on the dequantized cold values (code * scale) and the FP16 hot
 *     values, evaluated here in FP64.  The page's torch.cat of two separately
 *     normalised outputs is not a softmax over the union; the exact softmax
 *     over the union is the definition used.
 *
 * Everything here is deliberately plain: per-element loops, no blocking, no
 * vectorisation, FP32 arithmetic exactly where the quantizer defines it (IEEE
 * division, rintf under the default round-to-nearest-even mode; build with
 * -ffp-contract=off so no multiply-add is fused) and FP64 for attention.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORA_OK 0
#define ORA_ERR_INVALID -1
#define ORA_ERR_NOMEM -2

/* ------------------------------------------------------------------ */
/* IEEE 754 binary16 -> double, written from the format definition:   */
/* 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits.            */
/* ------------------------------------------------------------------ */
double ora_half_to_double(uint16_t h) {
  int sign = (h >> 15) & 1;
  int expo = (h >> 10) & 0x1f;
  int frac = h & 0x3ff;
  double v;
  if (expo == 0) {
    v = ldexp((double)frac, -24); /* subnormal: frac * 2^-24 */
  } else if (expo == 31) {
    v = frac ? NAN : INFINITY;
  } else {
    v = ldexp((double)(1024 + frac), expo - 25); /* (1 + frac/1024) * 2^(expo-15) */
  }
  return sign ? -v : v;
}

/* All 65536 binary16 values as float, filled from the definition above. */
static float half_table[65536];
static int half_table_ready = 0;

static void build_half_table(void) {
  if (half_table_ready) return;
  for (int i = 0; i < 65536; i++) half_table[i] = (float)ora_half_to_double((uint16_t)i);
  half_table_ready = 1;
}

static float half_to_float(uint16_t h) { return half_table[h]; }

/* ------------------------------------------------------------------ */
/* Cache state, kept in LOGICAL form: per sequence, per logical block. */
/* ------------------------------------------------------------------ */
typedef struct {
  int batch, hkv, hq, d, hot, block, max_blocks, quant_bits;
  int32_t *len;     /* [batch] tokens in the cache                      */
  int32_t *n_int4;  /* [batch] logical blocks < n_int4 are INT4 ("L2")  */
  uint16_t *ring;   /* [batch][hkv][hot][2][d] FP16 bits, slot = pos % hot */
  /* per (batch, logical block): NULL until the first token is sealed */
  int8_t **codes;   /* each [hkv][2][block][d], unpacked codes          */
  uint16_t **half;  /* quant_bits 0: each [hkv][2][block][d] FP16 bits  */
  float **scale;    /* each [hkv][2]                                    */
  int *qmax;        /* [batch*max_blocks] 127 or 7 once sealed (-1: FP16), else 0 */
} ora_cache;

void ora_free(ora_cache *c);

ora_cache *ora_new(int batch, int hkv, int hq, int d, int hot, int block,
                   int max_blocks, int quant_bits) {
  if (batch <= 0 || hkv <= 0 || hq <= 0 || hq % hkv || d <= 0 || hot <= 0 ||
      block <= 0 || max_blocks < 0 || (quant_bits != 8 && quant_bits != 4 && quant_bits != 0))
    return NULL;
  build_half_table();
  ora_cache *c = (ora_cache *)calloc(1, sizeof(ora_cache));
  if (!c) return NULL;
  c->batch = batch; c->hkv = hkv; c->hq = hq; c->d = d; c->hot = hot;
  c->block = block; c->max_blocks = max_blocks; c->quant_bits = quant_bits;
  size_t nb = (size_t)batch * (max_blocks > 0 ? max_blocks : 1);
  c->len = (int32_t *)calloc(batch, sizeof(int32_t));
  c->n_int4 = (int32_t *)calloc(batch, sizeof(int32_t));
  c->ring = (uint16_t *)calloc((size_t)batch * hkv * hot * 2 * d, sizeof(uint16_t));
  c->codes = (int8_t **)calloc(nb, sizeof(int8_t *));
  c->scale = (float **)calloc(nb, sizeof(float *));
  c->qmax = (int *)calloc(nb, sizeof(int));
  c->half = (uint16_t **)calloc(nb, sizeof(uint16_t *));
  if (!c->len || !c->n_int4 || !c->ring || !c->codes || !c->scale || !c->qmax || !c->half) {
    ora_free(c);
    return NULL;
  }
  return c;
}

void ora_free(ora_cache *c) {
  if (!c) return;
  size_t nb = (size_t)c->batch * (c->max_blocks > 0 ? c->max_blocks : 1);
  if (c->codes)
    for (size_t i = 0; i < nb; i++) free(c->codes[i]);
  if (c->scale)
    for (size_t i = 0; i < nb; i++) free(c->scale[i]);
  if (c->half)
    for (size_t i = 0; i < nb; i++) free(c->half[i]);
  free(c->codes); free(c->scale); free(c->qmax); free(c->half);
  free(c->len); free(c->n_int4); free(c->ring);
  free(c);
}

int ora_set_n_int4(ora_cache *c, const int32_t *n_int4) {
  for (int b = 0; b < c->batch; b++) c->n_int4[b] = n_int4 ? n_int4[b] : 0;
  return ORA_OK;
}

int32_t ora_len(const ora_cache *c, int b) { return c->len[b]; }

static uint16_t *ring_row(ora_cache *c, int b, int h, int slot, int kv) {
  return c->ring + ((((size_t)b * c->hkv + h) * c->hot + slot) * 2 + kv) * c->d;
}

/* Round half to even on FP32, as the IEEE default rounding mode does. */
static float rne(float x) { return rintf(x); }

static int clampi(int v, int q) { return v > q ? q : (v < -q ? -q : v); }

/*
 * One append call for the whole batch, [hybrid_v2 page] sections 2.1, 3.2, 4.2:
 * n_new[b] new tokens for sequence b, FP16 K and V laid out
 * [batch][max_new][hkv][d].  Tokens that leave the hot zone are sealed into
 * their cold block; the newest (up to hot) tokens go to the hot ring.
 * Returns ORA_ERR_INVALID (and changes nothing) when any n_new is negative or
 * above max_new or when a sequence would outgrow max_blocks cold blocks.
 */
int ora_append(ora_cache *c, const int32_t *n_new, int max_new,
               const uint16_t *k_new, const uint16_t *v_new) {
  const int d = c->d, hot = c->hot, blk = c->block, hkv = c->hkv;
  for (int b = 0; b < c->batch; b++) {
    int n = n_new[b];
    if (n < 0 || n > max_new) return ORA_ERR_INVALID;
    long L_new = (long)c->len[b] + n;
    long cold_new = L_new > hot ? L_new - hot : 0;
    if (cold_new > (long)c->max_blocks * blk) return ORA_ERR_INVALID;
  }
  for (int b = 0; b < c->batch; b++) {
    const int n = n_new[b];
    const int L_old = c->len[b];
    const int L_new = L_old + n;
    const int e0 = L_old > hot ? L_old - hot : 0; /* first position leaving */
    const int e1 = L_new > hot ? L_new - hot : 0; /* one past the last      */
    /* FP16 bits of position p, channel ch, for head h and K (kv=0) or V (1). */
#define SRC(p, h, kv, ch)                                                      \
  ((p) < L_old ? ring_row(c, b, h, (p) % hot, kv)[ch]                          \
               : ((kv) == 0 ? k_new : v_new)[(((size_t)b * max_new + ((p) - L_old)) * hkv + (h)) * d + (ch)])
    /* group the evicted positions by logical block, ascending */
    for (int p0 = e0; p0 < e1;) {
      const int i = p0 / blk;
      const int p1 = (i + 1) * blk < e1 ? (i + 1) * blk : e1;
      const size_t bi = (size_t)b * c->max_blocks + i;
      const int first_slot = p0 - i * blk;
      if (c->quant_bits == 0) {
        /* FP16 cold block: the tokens keep their FP16 values */
        if (!c->half[bi]) {
          c->half[bi] = (uint16_t *)calloc((size_t)hkv * 2 * blk * d, sizeof(uint16_t));
          if (!c->half[bi]) return ORA_ERR_NOMEM;
          c->qmax[bi] = -1;
        }
        for (int h = 0; h < hkv; h++)
          for (int kv = 0; kv < 2; kv++)
            for (int p = p0; p < p1; p++)
              for (int ch = 0; ch < d; ch++)
                c->half[bi][(((size_t)h * 2 + kv) * blk + (p - i * blk)) * d + ch] = SRC(p, h, kv, ch);
        p0 = p1;
        continue;
      }
      const int q = (c->quant_bits == 4 || i < c->n_int4[b]) ? 7 : 127;
      if (!c->codes[bi]) {
        c->codes[bi] = (int8_t *)calloc((size_t)hkv * 2 * blk * d, 1);
        c->scale[bi] = (float *)calloc((size_t)hkv * 2, sizeof(float));
        if (!c->codes[bi] || !c->scale[bi]) return ORA_ERR_NOMEM;
        c->qmax[bi] = q;
      }
      for (int h = 0; h < hkv; h++) {
        for (int kv = 0; kv < 2; kv++) {
          int8_t *cd = c->codes[bi] + ((size_t)h * 2 + kv) * blk * d;
          float *sp = c->scale[bi] + h * 2 + kv;
          /* absmax over the group's tokens x channels (exact in FP32) */
          float a = 0.0f;
          for (int p = p0; p < p1; p++)
            for (int ch = 0; ch < d; ch++) {
              float x = fabsf(half_to_float(SRC(p, h, kv, ch)));
              if (x > a) a = x;
            }
          float s_c = a / (float)q;
          float s;
          if (first_slot == 0) {
            s = s_c; /* empty block: its scale comes from these tokens */
          } else {
            s = *sp;
            if (s_c > s) {
              /* grow the scale; re-quantize the codes already sealed */
              for (int t = 0; t < first_slot; t++)
                for (int ch = 0; ch < d; ch++) {
                  float old = (float)cd[t * d + ch] * s;
                  cd[t * d + ch] = (int8_t)clampi((int)rne(old / s_c), q);
                }
              s = s_c;
            }
          }
          *sp = s;
          for (int p = p0; p < p1; p++)
            for (int ch = 0; ch < d; ch++) {
              float x = half_to_float(SRC(p, h, kv, ch));
              int code = (s == 0.0f) ? 0 : clampi((int)rne(x / s), q);
              cd[(p - i * blk) * d + ch] = (int8_t)code;
            }
        }
      }
      p0 = p1;
    }
    /* newest min(n, hot) tokens into the hot ring, slot = position % hot */
    const int first_hot = L_new - (n < hot ? n : hot);
    for (int p = first_hot; p < L_new; p++)
      for (int h = 0; h < hkv; h++)
        for (int kv = 0; kv < 2; kv++) {
          const uint16_t *src = ((kv == 0) ? k_new : v_new) +
                                (((size_t)b * max_new + (p - L_old)) * hkv + h) * d;
          memcpy(ring_row(c, b, h, p % hot, kv), src, (size_t)d * sizeof(uint16_t));
        }
#undef SRC
    c->len[b] = L_new;
  }
  return ORA_OK;
}

/*
 * Tier migration, [hybrid_v2 page] section 3.3: a cold block moves between
 * the INT8 ("L1") and the INT4 ("L2") tier and is given a new scale in place
 * (section 3.2).  The tier is kept as a count per sequence -- logical blocks
 * below n_int4[b] are INT4 -- so a migration moves that count to target[b]:
 * every sealed block between the old and the new count is re-quantized to
 * the other width, per (kv head, K|V):
 *   a = max over the block of |code * scale|          (FP32)
 *   scale' = a / Q'                                    (Q' = 7 or 127)
 *   code' = clamp(round-half-even(code * scale / scale'), -Q', Q')
 * (the arithmetic ora_append uses to re-quantize a tail block; a block of
 * zeros gets scale 0 and codes 0).  Blocks with no sealed token only change
 * tier.  Returns ORA_ERR_INVALID and changes nothing for a target outside
 * [0, max_blocks], or for a cache whose cold zone is all INT4.
 */
int ora_migrate(ora_cache *c, const int32_t *target) {
  const int d = c->d, blk = c->block, hkv = c->hkv;
  if (c->quant_bits != 8) return ORA_ERR_INVALID;
  for (int b = 0; b < c->batch; b++)
    if (target[b] < 0 || target[b] > c->max_blocks) return ORA_ERR_INVALID;
  for (int b = 0; b < c->batch; b++) {
    const int cur = c->n_int4[b], tgt = target[b];
    const int lo = cur < tgt ? cur : tgt, hi = cur < tgt ? tgt : cur;
    for (int i = lo; i < hi; i++) {
      const size_t bi = (size_t)b * c->max_blocks + i;
      if (!c->codes[bi]) continue; /* nothing sealed yet */
      const int q = i < tgt ? 7 : 127;
      for (int h = 0; h < hkv; h++) {
        for (int kv = 0; kv < 2; kv++) {
          int8_t *cd = c->codes[bi] + ((size_t)h * 2 + kv) * blk * d;
          float *sp = c->scale[bi] + h * 2 + kv;
          const float s_old = *sp;
          float a = 0.0f;
          for (int t = 0; t < blk; t++)
            for (int ch = 0; ch < d; ch++) {
              float x = fabsf((float)cd[t * d + ch] * s_old);
              if (x > a) a = x;
            }
          const float s_new = a / (float)q;
          for (int t = 0; t < blk; t++)
            for (int ch = 0; ch < d; ch++) {
              float v = (float)cd[t * d + ch] * s_old;
              cd[t * d + ch] = (int8_t)(s_new == 0.0f ? 0 : clampi((int)rne(v / s_new), q));
            }
          *sp = s_new;
        }
      }
      c->qmax[bi] = q;
    }
    c->n_int4[b] = tgt;
  }
  return ORA_OK;
}

int32_t ora_n_int4(const ora_cache *c, int b) { return c->n_int4[b]; }

/*
 * Adaptive migration threshold, [hybrid_v2 page] section 3.3, in ms:
 * 3000 * (1 + 0.2 * load_factor), load_factor = geometric mean of the
 * batch's sequence lengths / 512.  Sequences of length 0 are left out of the
 * mean (no sequence at all: load_factor 0).
 */
double ora_migration_threshold_ms(const int32_t *lens, int n) {
  double log_sum = 0.0;
  int m = 0;
  for (int i = 0; i < n; i++)
    if (lens[i] > 0) {
      log_sum += log((double)lens[i]);
      m++;
    }
  const double load_factor = m > 0 ? exp(log_sum / m) / 512.0 : 0.0;
  return 3000.0 * (1.0 + 0.2 * load_factor);
}

/*
 * Per-block decision of section 3.3: an INT4 ("L2") block whose mean access
 * interval is below the threshold moves up (+1); an INT8 ("L1") block whose
 * mean interval is above 1.5 x the threshold moves down (-1); otherwise 0.
 */
int ora_migration_decision(double avg_interval_ms, double threshold_ms, int is_int4) {
  if (is_int4 && avg_interval_ms < threshold_ms) return 1;
  if (!is_int4 && avg_interval_ms > 1.5 * threshold_ms) return -1;
  return 0;
}

/* Value of position p (channel ch) of head h, K (kv=0) or V (kv=1), in FP64:
 * hot FP16 value, or code * scale for a cold position. */
static double kv_value(const ora_cache *c, int b, int h, int kv, int p, int ch) {
  const int L = c->len[b];
  const int cold = L > c->hot ? L - c->hot : 0;
  if (p >= cold)
    return (double)half_to_float(
        c->ring[((((size_t)b * c->hkv + h) * c->hot + p % c->hot) * 2 + kv) * c->d + ch]);
  const int i = p / c->block;
  const size_t bi = (size_t)b * c->max_blocks + i;
  if (c->quant_bits == 0)
    return (double)half_to_float(c->half[bi][(((size_t)h * 2 + kv) * c->block + (p - i * c->block)) * c->d + ch]);
  const int8_t code = c->codes[bi][(((size_t)h * 2 + kv) * c->block + (p - i * c->block)) * c->d + ch];
  return (double)code * (double)c->scale[bi][h * 2 + kv];
}

/* Tokens of sequence b held in its INT4 ("L2") blocks: the oldest ones, in
 * logical blocks below n_int4[b] (every cold block when quant_bits is 4; none
 * with FP16 blocks). */
static int l2_tokens(const ora_cache *c, int b) {
  const int L = c->len[b];
  const int cold = L > c->hot ? L - c->hot : 0;
  long n4 = c->quant_bits == 4 ? c->max_blocks : c->quant_bits == 8 ? c->n_int4[b] : 0;
  const long cap = n4 * c->block;
  return cold < cap ? cold : (int)cap;
}

/* Attention logit of position p for query head qh (kv head hk), FP64:
 * softmax_scale * sum_c q_c * K_{p,c}, K from kv_value. */
static double logit(const ora_cache *c, int b, int hk, const uint16_t *qh, double softmax_scale, int p) {
  double acc = 0.0;
  for (int ch = 0; ch < c->d; ch++) acc += (double)half_to_float(qh[ch]) * kv_value(c, b, hk, 0, p, ch);
  return softmax_scale * acc;
}

typedef struct { double key; int pos; } l2_cand;

/* Order: larger score first, then the older position. */
static int cand_cmp(const void *x, const void *y) {
  const l2_cand *a = (const l2_cand *)x, *b = (const l2_cand *)y;
  if (a->key != b->key) return a->key > b->key ? -1 : 1;
  return a->pos - b->pos;
}

static int cmp_int(const void *x, const void *y) {
  const int a = *(const int *)x, b = *(const int *)y;
  return a < b ? -1 : (a > b);
}

/* Softmax attention of query head hh (kv head hk) over the n positions pos[]
 * of sequence b, FP64: o[d], *lse (natural log); no position: o = 0, -inf. */
static void attend(const ora_cache *c, int b, int hk, const uint16_t *qh, double softmax_scale,
                   const int *pos, int n, double *z, double *o, double *lse) {
  double m = -INFINITY;
  for (int j = 0; j < n; j++) {
    z[j] = logit(c, b, hk, qh, softmax_scale, pos[j]);
    if (z[j] > m) m = z[j];
  }
  double l = 0.0;
  for (int j = 0; j < n; j++) {
    z[j] = exp(z[j] - m);
    l += z[j];
  }
  for (int ch = 0; ch < c->d; ch++) {
    double acc = 0.0;
    for (int j = 0; j < n; j++) acc += z[j] * kv_value(c, b, hk, 1, pos[j], ch);
    o[ch] = n > 0 ? acc / l : 0.0;
  }
  *lse = n > 0 ? m + log(l) : -INFINITY;
}

/*
 * Single-query decode attention, FP64, for the (b, query head) pairs listed in
 * `pairs` (2*npairs ints) or for all pairs when pairs == NULL.
 * q: FP16 [batch][hq][d].  Query head h reads kv head h / (hq/hkv).
 * out: [batch][hq][d], lse: [batch][hq] (natural log); entries of pairs not
 * listed are left untouched.  An empty sequence gives out = 0, lse = -inf.
 * The L2 tokens a row attends:
 *   sel == NULL, top_k < 0:  all of them (dense);
 *   sel == NULL, top_k >= 0: the top_k with the largest logits (ties: the
 *                            older position), all of them when there are no
 *                            more;
 *   sel != NULL:             the sel_count[r] positions sel[r * sel_stride
 *                            ...] of row r = b * hq + h (each must be an L2
 *                            position of b, no repeats), for any top_k.
 * Every token that is not in an L2 block is attended.
 */
static int decode_rows(const ora_cache *c, const uint16_t *q, double softmax_scale, int top_k,
                       const int32_t *sel, int sel_stride, const int32_t *sel_count, const int32_t *pairs,
                       int npairs, double *out, double *lse, int nthreads) {
  const int d = c->d, g = c->hq / c->hkv;
  const int total = pairs ? npairs : c->batch * c->hq;
  if (nthreads < 1) nthreads = 1;
  int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads) reduction(| : bad)
  for (int w = 0; w < total; w++) {
    const int b = pairs ? pairs[2 * w] : w / c->hq;
    const int hh = pairs ? pairs[2 * w + 1] : w % c->hq;
    const size_t row = (size_t)b * c->hq + hh;
    const int hk = hh / g;
    const int L = c->len[b];
    const uint16_t *qh = q + row * d;
    int *pos = (int *)malloc(sizeof(int) * (L > 0 ? L : 1));
    double *z = (double *)malloc(sizeof(double) * (L > 0 ? L : 1));
    if (!pos || !z) {
      bad = 1;
      free(pos); free(z);
      continue;
    }
    int n = 0;
    const int n2 = (top_k < 0 && !sel) ? 0 : l2_tokens(c, b);
    if (sel) {
      const int cnt = sel_count[row];
      if (cnt < 0 || cnt > n2) bad = 1;
      for (int t = 0; t < cnt && t < n2; t++) {
        const int p = sel[row * (size_t)sel_stride + t];
        if (p < 0 || p >= n2) {
          bad = 1;
          continue;
        }
        pos[n++] = p;
      }
      qsort(pos, n, sizeof(int), cmp_int);
      for (int t = 1; t < n; t++)
        if (pos[t] == pos[t - 1]) bad = 1;
    } else if (n2 > 0) {
      l2_cand *cand = (l2_cand *)malloc(sizeof(l2_cand) * n2);
      if (!cand) {
        bad = 1;
        free(pos); free(z);
        continue;
      }
      for (int p = 0; p < n2; p++) {
        cand[p].key = logit(c, b, hk, qh, softmax_scale, p);
        cand[p].pos = p;
      }
      qsort(cand, n2, sizeof(l2_cand), cand_cmp);
      const int keep = top_k < n2 ? top_k : n2;
      for (int t = 0; t < keep; t++) pos[n++] = cand[t].pos;
      qsort(pos, n, sizeof(int), cmp_int);
      free(cand);
    }
    for (int p = n2; p < L; p++) pos[n++] = p;
    attend(c, b, hk, qh, softmax_scale, pos, n, z, out + row * d, &lse[row]);
    free(z);
    free(pos);
  }
  return bad ? ORA_ERR_INVALID : ORA_OK;
}

int ora_decode_topk(const ora_cache *c, const uint16_t *q, double softmax_scale, int top_k,
                    const int32_t *pairs, int npairs, double *out, double *lse, int nthreads) {
  return decode_rows(c, q, softmax_scale, top_k, NULL, 0, NULL, pairs, npairs, out, lse, nthreads);
}

int ora_decode_sel(const ora_cache *c, const uint16_t *q, double softmax_scale, const int32_t *sel,
                   int sel_stride, const int32_t *sel_count, const int32_t *pairs, int npairs, double *out,
                   double *lse, int nthreads) {
  if (!sel || !sel_count || sel_stride < 0) return ORA_ERR_INVALID;
  return decode_rows(c, q, softmax_scale, 0, sel, sel_stride, sel_count, pairs, npairs, out, lse, nthreads);
}

/* The attention logits of the L2 tokens of sequence b for query head hh (the
 * scores the top-k selection ranks): scores[p] for p < the returned count. */
int ora_l2_scores(const ora_cache *c, const uint16_t *q, double softmax_scale, int b, int hh, double *scores) {
  if (b < 0 || b >= c->batch || hh < 0 || hh >= c->hq) return ORA_ERR_INVALID;
  const int n2 = l2_tokens(c, b);
  const uint16_t *qh = q + ((size_t)b * c->hq + hh) * c->d;
  for (int p = 0; p < n2; p++) scores[p] = logit(c, b, hh / (c->hq / c->hkv), qh, softmax_scale, p);
  return n2;
}

int ora_decode(const ora_cache *c, const uint16_t *q, double softmax_scale,
               const int32_t *pairs, int npairs, double *out, double *lse,
               int nthreads) {
  return ora_decode_topk(c, q, softmax_scale, -1, pairs, npairs, out, lse, nthreads);
}

/* The page's rule for sparse_top_k (section 5.3): min(128, context_length / 256). */
int ora_sparse_top_k(long context_length) {
  const long k = context_length / 256;
  return k < 128 ? (int)k : 128;
}

/*
 * Log-sum-exp merge of per-split partial results, FP64 (the split-KV
 * "flash-decoding" combine; the merge of softmax pieces that the page's
 * torch.cat of section 4.2 stands in for).  o_part: [rows][n_splits][d],
 * each the softmax-normalised output of one split; lse_part: [rows][n_splits]
 * (natural log, -inf for an empty split).  out: [rows][d]; lse: [rows].
 */
int ora_combine(int rows, int n_splits, int d, const double *o_part,
                const double *lse_part, double *out, double *lse) {
  for (int r = 0; r < rows; r++) {
    double m = -INFINITY;
    for (int s = 0; s < n_splits; s++)
      if (lse_part[(size_t)r * n_splits + s] > m) m = lse_part[(size_t)r * n_splits + s];
    double *o = out + (size_t)r * d;
    if (m == -INFINITY) {
      for (int ch = 0; ch < d; ch++) o[ch] = 0.0;
      lse[r] = -INFINITY;
      continue;
    }
    double wsum = 0.0;
    for (int ch = 0; ch < d; ch++) o[ch] = 0.0;
    for (int s = 0; s < n_splits; s++) {
      double w = exp(lse_part[(size_t)r * n_splits + s] - m);
      wsum += w;
      for (int ch = 0; ch < d; ch++) o[ch] += w * o_part[((size_t)r * n_splits + s) * d + ch];
    }
    for (int ch = 0; ch < d; ch++) o[ch] /= wsum;
    lse[r] = m + log(wsum);
  }
  return ORA_OK;
}

/* ------------------------------------------------------------------ */
/* Inspection of the logical state (for the oracle's own tests).       */
/* ------------------------------------------------------------------ */

/* Logical block i of sequence b: codes [hkv][2][block][d] (slots not yet
 * sealed are 0) and scales [hkv][2].  Returns Q (127 or 7), or 0 if the
 * block holds no sealed token. */
int ora_get_block(const ora_cache *c, int b, int i, int8_t *codes, float *scales) {
  const size_t bi = (size_t)b * c->max_blocks + i;
  if (b < 0 || b >= c->batch || i < 0 || i >= c->max_blocks || !c->codes[bi]) return 0;
  if (c->quant_bits == 0) return 0;
  memcpy(codes, c->codes[bi], (size_t)c->hkv * 2 * c->block * c->d);
  memcpy(scales, c->scale[bi], (size_t)c->hkv * 2 * sizeof(float));
  return c->qmax[bi];
}

/* FP16 cold block i of sequence b (quant_bits 0): FP16 bits [hkv][2][block][d]
 * (slots not yet sealed are 0).  Returns 1, or 0 if the block holds no sealed
 * token. */
int ora_get_block_fp16(const ora_cache *c, int b, int i, uint16_t *vals) {
  const size_t bi = (size_t)b * c->max_blocks + i;
  if (c->quant_bits != 0 || b < 0 || b >= c->batch || i < 0 || i >= c->max_blocks || !c->half[bi]) return 0;
  memcpy(vals, c->half[bi], (size_t)c->hkv * 2 * c->block * c->d * sizeof(uint16_t));
  return 1;
}

/* Width of logical block i of sequence b: 127 (INT8), 7 (INT4), -1 (FP16)
 * once a token is sealed in it, else 0. */
int ora_block_q(const ora_cache *c, int b, int i) {
  if (b < 0 || b >= c->batch || i < 0 || i >= c->max_blocks) return 0;
  return c->qmax[(size_t)b * c->max_blocks + i];
}

/* Hot ring of sequence b: FP16 bits [hkv][hot][2][d]. */
int ora_get_ring(const ora_cache *c, int b, uint16_t *ring) {
  memcpy(ring, c->ring + (size_t)b * c->hkv * c->hot * 2 * c->d,
         (size_t)c->hkv * c->hot * 2 * c->d * sizeof(uint16_t));
  return ORA_OK;
}

/* ------------------------------------------------------------------ */
/* The device memory format, written out from its definition:          */
/*   cold pool bytes [num_phys][hkv][2][tile] with tile = 64*d bytes   */
/*   (K tile, then V tile, per physical block of 64 tokens and kv      */
/*   head).                                                            */
/*   K tile, INT8: token-major, byte (t, ch) at t*d + ch.              */
/*   V tile, INT8: channel-major, 64 token bytes per channel row, the  */
/*     four 16-byte chunks of row ch stored at chunk index             */
/*     (t/16) XOR ((ch/2) % 4): byte (t, ch) at                        */
/*     ch*64 + (((t/16) ^ ((ch/2) % 4)) * 16) + t%16.                  */
/*   INT4 tiles use the first half of the tile.  Eight consecutive     */
/*   codes e=0..7 along the packed axis share one 32-bit word: code e  */
/*   sits in byte e%4, low nibble for e<4, high nibble for e>=4, as a  */
/*   4-bit two's complement number.                                    */
/*   K tile, INT4: token-major, 64 bytes per token; channel ch of      */
/*     token t in word t*16 + ch/8 (bytes), element ch%8.              */
/*   V tile, INT4: channel-major, 32 bytes per channel row in four     */
/*     8-byte units of 16 tokens, unit u stored at u XOR ((ch/4) % 4); */
/*     within a unit, tokens 0..7 in its first word, 8..15 in the      */
/*     second.                                                         */
/*   Blocks of 128 tokens are stored as two such 64-slot sub-blocks:   */
/*   [num_phys][hkv][2 sub-blocks][2][8192], slot t of the block in    */
/*   slot t%64 of sub-block t/64; the block keeps one scale per K|V.   */
/*   Blocks of 32 tokens use slots 0..31 of one 64-slot tile pair.     */
/*   FP16 cold blocks (quant_bits 0): cold pool bytes                  */
/*   [num_phys][hkv][block][2][d] FP16, per token the K row then the V  */
/*   row (the hot ring's layout), 512 B per token and kv head.          */
/*   scales: float [num_phys][hkv][2] (not used by FP16 blocks).        */
/*   hot ring: FP16 [batch][hkv][hot][2][d] (K row, then V row).       */
/* Only sealed slots are written; other bytes are left as they are.    */
/* The upper half of an INT4 block's tiles holds no code: its content  */
/* on the device is unspecified (a block demoted from INT8 keeps its   */
/* old bytes there), and comparisons leave it out.                     */
/* ------------------------------------------------------------------ */
static void put_nibble(uint8_t *word4, int e, int code) {
  uint8_t *byte = word4 + (e & 3);
  uint8_t nib = (uint8_t)(code & 0xf);
  if (e < 4) *byte = (uint8_t)((*byte & 0xf0) | nib);
  else *byte = (uint8_t)((*byte & 0x0f) | (nib << 4));
}

int ora_export(const ora_cache *c, const int32_t *block_table, int num_phys,
               uint8_t *cold, float *scales, uint16_t *hot, int32_t *seq_lens) {
  const int d = c->d, blk = c->block, hkv = c->hkv;
  const size_t tile = (size_t)64 * d;   /* one K or V tile of a 64-slot sub-block */
  const int nsub = blk > 64 ? blk / 64 : 1; /* sub-blocks per block */
  /* format defined for d = 128 and blocks of 32, 64 or 128 tokens */
  if (d != 128 || (blk != 32 && blk != 64 && blk != 128)) return ORA_ERR_INVALID;
  if (c->quant_bits == 0) {
    uint16_t *cold16 = (uint16_t *)cold;
    for (int b = 0; b < c->batch; b++) {
      const int L = c->len[b];
      const int cold_len = L > c->hot ? L - c->hot : 0;
      const int nblk = (cold_len + blk - 1) / blk;
      for (int i = 0; i < nblk; i++) {
        const size_t bi = (size_t)b * c->max_blocks + i;
        const int phys = block_table[(size_t)b * c->max_blocks + i];
        if (phys < 0 || phys >= num_phys) return ORA_ERR_INVALID;
        const int sealed = cold_len - i * blk < blk ? cold_len - i * blk : blk;
        for (int h = 0; h < hkv; h++)
          for (int t = 0; t < sealed; t++)
            for (int kv = 0; kv < 2; kv++)
              for (int ch = 0; ch < d; ch++)
                cold16[((((size_t)phys * hkv + h) * blk + t) * 2 + kv) * d + ch] =
                    c->half[bi][(((size_t)h * 2 + kv) * blk + t) * d + ch];
      }
      seq_lens[b] = L;
    }
    memcpy(hot, c->ring, (size_t)c->batch * hkv * c->hot * 2 * d * sizeof(uint16_t));
    return ORA_OK;
  }
  for (int b = 0; b < c->batch; b++) {
    const int L = c->len[b];
    const int cold_len = L > c->hot ? L - c->hot : 0;
    const int nblk = (cold_len + blk - 1) / blk;
    for (int i = 0; i < nblk; i++) {
      const size_t bi = (size_t)b * c->max_blocks + i;
      const int phys = block_table[(size_t)b * c->max_blocks + i];
      if (phys < 0 || phys >= num_phys) return ORA_ERR_INVALID;
      const int sealed = cold_len - i * blk < blk ? cold_len - i * blk : blk;
      for (int h = 0; h < hkv; h++) {
        for (int kv = 0; kv < 2; kv++) {
          const int8_t *cd = c->codes[bi] + ((size_t)h * 2 + kv) * blk * d;
          scales[((size_t)phys * hkv + h) * 2 + kv] = c->scale[bi][h * 2 + kv];
          for (int tb = 0; tb < sealed; tb++)
            for (int ch = 0; ch < d; ch++) {
              /* slot tb of the block: slot t = tb % 64 of sub-block tb / 64 */
              const int t = tb % 64;
              uint8_t *t8 = cold + (((((size_t)phys * hkv + h) * nsub + tb / 64) * 2) + kv) * tile;
              const int code = cd[tb * d + ch];
              if (c->qmax[bi] == 127) {
                if (kv == 0) t8[t * d + ch] = (uint8_t)code;
                else t8[ch * 64 + (((t / 16) ^ ((ch / 2) % 4)) * 16) + t % 16] = (uint8_t)code;
              } else {
                if (kv == 0) put_nibble(t8 + t * 64 + (ch / 8) * 4, ch % 8, code);
                else {
                  const int unit = (t / 16) ^ ((ch / 4) % 4);
                  const int in_unit = t % 16;
                  put_nibble(t8 + ch * 32 + unit * 8 + (in_unit / 8) * 4, in_unit % 8, code);
                }
              }
            }
        }
      }
    }
    seq_lens[b] = L;
  }
  memcpy(hot, c->ring, (size_t)c->batch * hkv * c->hot * 2 * d * sizeof(uint16_t));
  return ORA_OK;
}
