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
// is one pipeline item, brought into a 4-stage shared-memory ring by the TMA
// engine with one 1-D bulk copy (no cluster multicast) completing on an
// mbarrier; every wait is bounded.
//
// Arithmetic (per kv head, for its G = Hq/Hkv query heads):
//  * q is turned into 16-bit fixed point per query head (q_i = rint(q * 32767
//    / max|q|)); a cold logit is the exact int32 dot product of q_i with the
//    K codes (dp2a: two 16x8-bit products per instruction), times
//    max|q|/32767 * K-scale * softmax_scale * log2(e).
//  * Warp w owns tokens 16w..16w+15 of every block and keeps its own online
//    softmax state (running max, sum, FP32 output accumulator) per head.  Its
//    softmax weights relative to the 16-token maximum are 16-bit fixed point
//    (p_i = rint(32767 * 2^(z - max))); P.V is again an exact int32 dp2a sum
//    over the V codes, folded into the FP32 state with the V scale.
//  * Hot tokens are attended in FP32 from the FP16 values (never quantized).
//  * The 4 warp states are merged in FP32 at the end of the split; the
//    split's normalised output and log-sum-exp go to the workspace for
//    hyb_combine, or straight to the FP16 output when there is one split.
// Tensor cores are not used: per byte of KV the work is a few integer
// multiply-adds, and the kernel is bound by HBM bandwidth.
#include <cfloat>

#include "kernels.cuh"

namespace hyb {

constexpr int kWarps = 4;
constexpr int kThreads = 32 * kWarps;
constexpr int kStages = 4;
constexpr int kMaxSplitBlocks = 128;
constexpr long long kWaitCycles = 1ll << 31;  // ~1 s at B200 clocks
constexpr float kLn2 = 0.69314718055994531f;

template <int G>
struct DecodeSmem {
  alignas(128) uint8_t ring[kStages][kTilePairBytes];
  uint64_t full[kStages];
  int32_t phys[kMaxSplitBlocks];
  float sk[kMaxSplitBlocks];
  float sv[kMaxSplitBlocks];
  alignas(16) float qf[G][kDim];
  alignas(16) int16_t qi[G][kDim];
  float sq[G];
  alignas(16) uint16_t pcode[kWarps][G][16];
  alignas(16) float phot[kWarps][G][8];
  float wmax[kWarps][G];
  float wsum[kWarps][G];
  float mrun[kWarps][G];
  float lrun[kWarps][G];
};

template <int G>
constexpr int pow2_heads() {
  return G <= 1 ? 1 : (G <= 2 ? 2 : (G <= 4 ? 4 : 8));
}

// One level of the head-transposing reduction across lanes (xor m): lanes
// with bit m set keep the upper half of the C live values, the others the
// lower half, and each adds its partner's copy of the half it keeps.
template <int C, int P, typename T>
__device__ __forceinline__ void tr_level(T (&v)[P], int lane, int m) {
  const bool up = (lane & m) != 0;
#pragma unroll
  for (int k = 0; k < C / 2; k++) {
    const T send = up ? v[k] : v[k + C / 2];
    const T keep = up ? v[k + C / 2] : v[k];
    v[k] = keep + __shfl_xor_sync(0xffffffffu, send, m);
  }
}

// Sum each of P per-lane values over the 8 lanes of a lane octet; on return
// v[0] holds the octet total of head head_of_lane<P>(lane).
template <int P, typename T>
__device__ __forceinline__ void transpose_reduce(T (&v)[P], int lane) {
  if constexpr (P == 8) {
    tr_level<8>(v, lane, 4);
    tr_level<4>(v, lane, 2);
    tr_level<2>(v, lane, 1);
  } else if constexpr (P == 4) {
    tr_level<4>(v, lane, 4);
    tr_level<2>(v, lane, 2);
    v[0] += __shfl_xor_sync(0xffffffffu, v[0], 1);
  } else if constexpr (P == 2) {
    tr_level<2>(v, lane, 4);
    v[0] += __shfl_xor_sync(0xffffffffu, v[0], 2);
    v[0] += __shfl_xor_sync(0xffffffffu, v[0], 1);
  } else {
    v[0] += __shfl_xor_sync(0xffffffffu, v[0], 4);
    v[0] += __shfl_xor_sync(0xffffffffu, v[0], 2);
    v[0] += __shfl_xor_sync(0xffffffffu, v[0], 1);
  }
}

template <int P>
__device__ __forceinline__ int head_of_lane(int lane) {
  int hd = 0, c = P;
#pragma unroll
  for (int m = 4; m >= 1; m >>= 1) {
    if (c > 1) {
      if (lane & m) hd += c / 2;
      c /= 2;
    }
  }
  return hd;
}

__device__ __forceinline__ void unpack_int4(uint32_t x, uint32_t &lo, uint32_t &hi) {
  lo = sext_nibbles(x & 0x0f0f0f0fu);
  hi = sext_nibbles((x >> 4) & 0x0f0f0f0fu);
}

template <int G>
__global__ void __launch_bounds__(kThreads, (G <= 4 ? 3 : 2)) decode_kernel(const DecodeArgs a) {
  constexpr int P = pow2_heads<G>();
  extern __shared__ __align__(128) uint8_t smem_raw[];
  DecodeSmem<G> &sm = *reinterpret_cast<DecodeSmem<G> *>(smem_raw);

  const int s = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int S = a.n_splits;
  const int hq0 = h * G;

  int L = a.seq_lens[b];
  if (L < 0 || L > a.max_seq_len) {
    if (tid == 0 && s == 0 && h == 0) set_status(a.status, HYB_STATUS_SEQ_LEN);
    L = -1;
  }
  const int Lc = max(0, L - kHot);
  const int nblk = (Lc + kBlock - 1) / kBlock;
  const int Sb = max(1, (nblk + a.split_blocks - 1) / a.split_blocks);
  if (L < 0 || s >= Sb) {
    // nothing to attend in this split: neutral partial result
    for (int e = tid; e < G * kDim; e += kThreads) {
      const int hh = e / kDim, c = e % kDim;
      const size_t row = (size_t)b * a.hq + hq0 + hh;
      if (S > 1)
        a.o_part[(row * S + s) * kDim + c] = 0.f;
      else
        a.out[row * kDim + c] = __float2half_rn(0.f);
      if (c == 0) {
        if (S > 1)
          a.lse_part[row * S + s] = -INFINITY;
        else if (a.lse_out)
          a.lse_out[row] = -INFINITY;
      }
    }
    return;
  }
  const int i0 = s * a.split_blocks;
  const int ncold = min(nblk, i0 + a.split_blocks) - i0;
  const int nhot = (s == Sb - 1) ? min(L, kHot) : 0;
  const int nitems = ncold + (nhot > 0 ? 1 : 0);
  const int n_int4_b = a.quant_bits == 4 ? 0x7fffffff : (a.n_int4 ? a.n_int4[b] : 0);

  if (tid == 0) {
#pragma unroll
    for (int st = 0; st < kStages; st++) mbar_init(&sm.full[st], 1);
    mbar_fence_init();
  }
  for (int k = tid; k < ncold; k += kThreads) {
    int phys = a.block_table[(size_t)b * a.max_blocks + i0 + k];
    if (phys < 0 || phys >= a.num_phys) {
      set_status(a.status, HYB_STATUS_BAD_BLOCK);
      phys = -1;
    }
    sm.phys[k] = phys;
  }
  for (int e = tid; e < G * kDim; e += kThreads)
    sm.qf[e / kDim][e % kDim] = __half2float(a.q[((size_t)b * a.hq + hq0) * kDim + e]);
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
  int issued = 0;
  if (tid == 0) {
    issued = min(nitems, kStages);
    for (int k = 0; k < issued; k++) issue(k);
  }

  // block scales (their loads overlap the first copies)
  for (int k = tid; k < ncold; k += kThreads) {
    const int phys = sm.phys[k];
    float2 sc = make_float2(0.f, 0.f);
    if (phys >= 0) sc = *reinterpret_cast<const float2 *>(a.scales + ((size_t)phys * a.hkv + h) * 2);
    sm.sk[k] = sc.x;
    sm.sv[k] = sc.y;
  }
  // q in 16-bit fixed point per head
  for (int hh = warp; hh < G; hh += kWarps) {
    float amax = 0.f;
    for (int c = lane; c < kDim; c += 32) amax = fmaxf(amax, fabsf(sm.qf[hh][c]));
    for (int m = 16; m > 0; m >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, m));
    const float inv = amax > 0.f ? 32767.f / amax : 0.f;
    for (int c = lane; c < kDim; c += 32) {
      const int v = __float2int_rn(sm.qf[hh][c] * inv);
      sm.qi[hh][c] = static_cast<int16_t>(max(-32767, min(32767, v)));
    }
    if (lane == 0) sm.sq[hh] = amax > 0.f ? amax / 32767.f : 0.f;
  }
  __syncthreads();

  const int tg = lane >> 3, cs = lane & 7;
  const int hd = head_of_lane<P>(lane);
  const bool owner = (lane & (8 / P - 1)) == 0 && hd < G;
  const float sq_hd = hd < G ? sm.sq[hd] : 0.f;

  uint32_t qp[G][8];
#pragma unroll
  for (int hh = 0; hh < G; hh++) {
    const uint4 *src = reinterpret_cast<const uint4 *>(&sm.qi[hh][16 * cs]);
    const uint4 x0 = src[0], x1 = src[1];
    qp[hh][0] = x0.x; qp[hh][1] = x0.y; qp[hh][2] = x0.z; qp[hh][3] = x0.w;
    qp[hh][4] = x1.x; qp[hh][5] = x1.y; qp[hh][6] = x1.z; qp[hh][7] = x1.w;
  }

  float m_run[G], l_run[G], acc[G][4];
#pragma unroll
  for (int hh = 0; hh < G; hh++) {
    m_run[hh] = -INFINITY;
    l_run[hh] = 0.f;
#pragma unroll
    for (int kk = 0; kk < 4; kk++) acc[hh][kk] = 0.f;
  }

  bool aborted = false;
  int k_stop = nitems;
  for (int k = 0; k < nitems; k++) {
    const int st = k % kStages;
    const bool ok = mbar_wait_bounded(&sm.full[st], (k / kStages) & 1, kWaitCycles);
    if (!ok && lane == 0) set_status(a.status, HYB_STATUS_TIMEOUT);
    const uint8_t *stage = sm.ring[st];
    if (ok && k < ncold) {
      // ---------------- cold block ----------------
      const int i = i0 + k;
      const int nvalid = sm.phys[k] < 0 ? 0 : min(kBlock, Lc - i * kBlock);
      const int nv = nvalid - 16 * warp;
      if (nv > 0) {
        const bool int4 = i < n_int4_b;
        const float coef = sq_hd * sm.sk[k] * a.qk_scale;
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
          for (int hh = 0; hh < P; hh++) {
            int d = 0;
            if (hh < G) {
#pragma unroll
              for (int j = 0; j < 4; j++) {
                d = __dp2a_lo(static_cast<int>(qp[hh][2 * j]), static_cast<int>(kw[j]), d);
                d = __dp2a_hi(static_cast<int>(qp[hh][2 * j + 1]), static_cast<int>(kw[j]), d);
              }
            }
            dot[hh] = d;
          }
          transpose_reduce<P>(dot, lane);
          z[step] = (4 * step + tg < nv && hd < G) ? static_cast<float>(dot[0]) * coef : -INFINITY;
        }
        float mb = fmaxf(fmaxf(z[0], z[1]), fmaxf(z[2], z[3]));
        mb = fmaxf(mb, __shfl_xor_sync(0xffffffffu, mb, 8));
        mb = fmaxf(mb, __shfl_xor_sync(0xffffffffu, mb, 16));
        int psum = 0;
        int pc[4];
#pragma unroll
        for (int step = 0; step < 4; step++) {
          const float pv = z[step] == -INFINITY ? 0.f : exp2f(z[step] - mb);
          pc[step] = __float2int_rn(pv * 32767.f);
          psum += pc[step];
        }
        psum += __shfl_xor_sync(0xffffffffu, psum, 8);
        psum += __shfl_xor_sync(0xffffffffu, psum, 16);
        if (owner) {
#pragma unroll
          for (int step = 0; step < 4; step++)
            sm.pcode[warp][hd][4 * step + tg] = static_cast<uint16_t>(pc[step]);
          if (tg == 0) {
            sm.wmax[warp][hd] = mb;
            sm.wsum[warp][hd] = static_cast<float>(psum);
          }
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
        const float sv = sm.sv[k];
#pragma unroll
        for (int hh = 0; hh < G; hh++) {
          const uint4 pa = *reinterpret_cast<const uint4 *>(&sm.pcode[warp][hh][0]);
          const uint4 pb = *reinterpret_cast<const uint4 *>(&sm.pcode[warp][hh][8]);
          const uint32_t pp[8] = {pa.x, pa.y, pa.z, pa.w, pb.x, pb.y, pb.z, pb.w};
          int ai[4];
#pragma unroll
          for (int kk = 0; kk < 4; kk++) {
            int d = 0;
#pragma unroll
            for (int j = 0; j < 4; j++) {
              d = __dp2a_lo(static_cast<int>(pp[2 * j]), static_cast<int>(vw[kk][j]), d);
              d = __dp2a_hi(static_cast<int>(pp[2 * j + 1]), static_cast<int>(vw[kk][j]), d);
            }
            ai[kk] = d;
          }
          const float mbh = sm.wmax[warp][hh];
          const float m_new = fmaxf(m_run[hh], mbh);
          const float alpha = exp2f(m_run[hh] - m_new);
          const float beta = exp2f(mbh - m_new) * (1.f / 32767.f);
          l_run[hh] = l_run[hh] * alpha + beta * sm.wsum[warp][hh];
          const float cv = beta * sv;
#pragma unroll
          for (int kk = 0; kk < 4; kk++) acc[hh][kk] = acc[hh][kk] * alpha + cv * static_cast<float>(ai[kk]);
          m_run[hh] = m_new;
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
          for (int hh = 0; hh < P; hh++) {
            float d = 0.f;
            if (hh < G) {
              const float4 *qv = reinterpret_cast<const float4 *>(&sm.qf[hh][16 * cs]);
#pragma unroll
              for (int j = 0; j < 4; j++) {
                const float4 qq = qv[j];
                d = fmaf(qq.x, kf[4 * j], d);
                d = fmaf(qq.y, kf[4 * j + 1], d);
                d = fmaf(qq.z, kf[4 * j + 2], d);
                d = fmaf(qq.w, kf[4 * j + 3], d);
              }
            }
            dot[hh] = d;
          }
          transpose_reduce<P>(dot, lane);
          z[step] = (4 * step + tg < nv && hd < G) ? dot[0] * a.qk_scale : -INFINITY;
        }
        float mb = fmaxf(z[0], z[1]);
        mb = fmaxf(mb, __shfl_xor_sync(0xffffffffu, mb, 8));
        mb = fmaxf(mb, __shfl_xor_sync(0xffffffffu, mb, 16));
        float pv[2], psum = 0.f;
#pragma unroll
        for (int step = 0; step < 2; step++) {
          pv[step] = z[step] == -INFINITY ? 0.f : exp2f(z[step] - mb);
          psum += pv[step];
        }
        psum += __shfl_xor_sync(0xffffffffu, psum, 8);
        psum += __shfl_xor_sync(0xffffffffu, psum, 16);
        if (owner) {
          sm.phot[warp][hd][tg] = pv[0];
          sm.phot[warp][hd][4 + tg] = pv[1];
          if (tg == 0) {
            sm.wmax[warp][hd] = mb;
            sm.wsum[warp][hd] = psum;
          }
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
        for (int hh = 0; hh < G; hh++) {
          const float mbh = sm.wmax[warp][hh];
          const float m_new = fmaxf(m_run[hh], mbh);
          const float alpha = exp2f(m_run[hh] - m_new);
          const float beta = exp2f(mbh - m_new);
          l_run[hh] = l_run[hh] * alpha + beta * sm.wsum[warp][hh];
#pragma unroll
          for (int kk = 0; kk < 4; kk++) acc[hh][kk] = acc[hh][kk] * alpha + beta * ah[hh][kk];
          m_run[hh] = m_new;
        }
      }
    }
    if (__syncthreads_or(!ok)) {
      aborted = true;
      k_stop = k;
      break;
    }
    if (tid == 0 && k + kStages < nitems) {
      issue(k + kStages);
      issued = k + kStages + 1;
    }
  }

  if (aborted) {
    // let every copy still in flight land before the CTA's shared memory is released
    if (tid == 0) {
      for (int k = k_stop; k < issued; k++)
        (void)mbar_wait_bounded(&sm.full[k % kStages], (k / kStages) & 1, kWaitCycles);
    }
    __syncthreads();
    return;
  }

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
  for (int hh = 0; hh < G; hh++) {
    float mm = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; w++) mm = fmaxf(mm, sm.mrun[w][hh]);
    float num = 0.f, den = 0.f;
    if (mm != -INFINITY) {
#pragma unroll
      for (int w = 0; w < kWarps; w++) {
        const float f = exp2f(sm.mrun[w][hh] - mm);
        num = fmaf(f, mbuf[(w * G + hh) * kDim + tid], num);
        den = fmaf(f, sm.lrun[w][hh], den);
      }
    }
    const float o = den > 0.f ? num / den : 0.f;
    const float lse = den > 0.f ? (mm + log2f(den)) * kLn2 : -INFINITY;
    const size_t row = (size_t)b * a.hq + hq0 + hh;
    if (S == 1) {
      a.out[row * kDim + tid] = __float2half_rn(o);
      if (tid == 0 && a.lse_out) a.lse_out[row] = lse;
    } else {
      a.o_part[(row * S + s) * kDim + tid] = o;
      if (tid == 0) a.lse_part[row * S + s] = lse;
    }
  }
}

template <int G>
static cudaError_t launch_decode_g(const DecodeArgs &a, int batch, cudaStream_t stream) {
  const size_t smem = sizeof(DecodeSmem<G>);
  static int configured_dev_mask = 0;  // one bit per device
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 31 && !(configured_dev_mask & (1 << dev))) {
    e = cudaFuncSetAttribute(decode_kernel<G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    configured_dev_mask |= 1 << dev;
  }
  dim3 grid(a.n_splits, a.hkv, batch);
  decode_kernel<G><<<grid, kThreads, smem, stream>>>(a);
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

int decode_max_split_blocks() { return kMaxSplitBlocks; }

}  // namespace hyb
