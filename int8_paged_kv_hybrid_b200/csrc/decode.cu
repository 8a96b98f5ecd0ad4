// decode.cu -- dispatch of hyb_decode_attn / hyb_decode_step launches to the
// decode kernel's instantiations (decode_kernel.cuh; one translation unit per
// block size and variant, decode_b*_*.cu), and the kernel's launch limits.
#include "kernels.cuh"

namespace hyb {

constexpr int kMaxSplitBlocksD = 128;  // == the kernel's threads: one block-table entry per thread
constexpr int kMaxClusterD = 16;       // largest cluster the kernel is launched with (non-portable above 8)

template <bool kF16, bool kSkip, int kBshift>
cudaError_t launch_decode_f(const DecodeArgs &a, int group, int batch, bool cluster, cudaStream_t stream);
template <bool kF16, bool kSkip, int kBshift>
int decode_occupancy(int group);
template <bool kF16, bool kSkip, int kBshift>
int decode_active_clusters(int group, int csize);

template <int kBshift>
static cudaError_t launch_decode_l(const DecodeArgs &a, int group, int batch, bool cluster, cudaStream_t stream) {
  if (a.quant_bits == 0) return launch_decode_f<true, false, kBshift>(a, group, batch, cluster, stream);
  if (a.l2_skip) return launch_decode_f<false, true, kBshift>(a, group, batch, cluster, stream);
  return launch_decode_f<false, false, kBshift>(a, group, batch, cluster, stream);
}

cudaError_t launch_decode(const DecodeArgs &a, int group, int batch, bool cluster, cudaStream_t stream) {
  switch (a.bshift) {
    case 5: return launch_decode_l<5>(a, group, batch, cluster, stream);
    case 6: return launch_decode_l<6>(a, group, batch, cluster, stream);
    case 7: return launch_decode_l<7>(a, group, batch, cluster, stream);
    default: return cudaErrorInvalidValue;
  }
}

int decode_max_cluster() { return kMaxClusterD; }

// Clusters of csize CTAs (2..16) that can be resident at once for this head
// group (0 if none, or the device cannot be queried); cached per device.
int decode_resident_clusters(int group, int csize) {
  static int cached[32][9][kMaxClusterD + 1];  // [device][group][size], 0 = not yet known, -1 = none
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  if (group < 1 || group > 8 || csize < 2 || csize > kMaxClusterD) return 0;
  if (dev >= 0 && dev < 32 && cached[dev][group][csize] != 0) return cached[dev][group][csize] > 0 ? cached[dev][group][csize] : 0;
  const int n = decode_active_clusters<false, false, 6>(group, csize);
  if (dev >= 0 && dev < 32) cached[dev][group][csize] = n > 0 ? n : -1;
  return n;
}

int decode_max_split_blocks() { return kMaxSplitBlocksD; }

// CTAs of the decode kernel one SM holds at once for this head group (0 if
// the device cannot be queried); cached per device.
int decode_ctas_per_sm(int group) {
  static int cached[32][9];  // [device][group], 0 = not yet known
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  if (dev >= 0 && dev < 32 && group >= 1 && group <= 8 && cached[dev][group] > 0) return cached[dev][group];
  const int n = decode_occupancy<false, false, 6>(group);
  if (n > 0 && dev >= 0 && dev < 32 && group >= 1 && group <= 8) cached[dev][group] = n;
  return n;
}

}  // namespace hyb
