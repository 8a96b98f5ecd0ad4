// combine.cu -- hyb_combine: log-sum-exp merge of split-KV partial results.
//
// The web page "DeepSeek V4混合式KV Cache推理优化实战解析" (section 4.2, step
// 5) joins the hot-zone and cold-zone attention outputs with torch.cat; a
// softmax over the union of keys instead needs each part's output weighted by
// exp(lse_part - lse_total).  That merge is this kernel:
//   out = sum_s exp(lse_s - m) o_s / sum_s exp(lse_s - m),  m = max_s lse_s,
//   lse = m + log(sum_s exp(lse_s - m)),
// in FP32, output rounded to FP16 (nearest even).  One CTA of 128 threads per
// (sequence, query head) row, thread = channel.
#include "kernels.cuh"

namespace hyb {

__global__ void __launch_bounds__(kDim) combine_kernel(const CombineArgs a) {
  const size_t row = blockIdx.x;
  const int c = threadIdx.x;
  const int S = a.n_splits;
  const float *lse = a.lse_part + row * S;
  float m = -INFINITY;
  for (int s = 0; s < S; s++) m = fmaxf(m, lse[s]);
  float num = 0.f, den = 0.f;
  if (m != -INFINITY) {
    const float *o = a.o_part + row * S * kDim + c;
    for (int s = 0; s < S; s++) {
      const float l = lse[s];
      if (l == -INFINITY) continue;
      const float w = __expf(l - m);
      num = fmaf(w, o[(size_t)s * kDim], num);
      den += w;
    }
  }
  a.out[row * kDim + c] = __float2half_rn(den > 0.f ? num / den : 0.f);
  if (c == 0 && a.lse_out) a.lse_out[row] = den > 0.f ? m + logf(den) : -INFINITY;
}

cudaError_t launch_combine(const CombineArgs &a, int rows, cudaStream_t stream) {
  if (rows <= 0) return cudaSuccess;
  combine_kernel<<<rows, kDim, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace hyb
