// decode_persist.cu -- instantiations and dispatch of the persistent,
// warp-specialized decode kernel (decode_persist.cuh).
#include "decode_persist.cuh"

namespace hyb {

cudaError_t launch_decode_persist(const DecodeArgs &a, int group, int batch, int ctas, cudaStream_t stream) {
  switch (group) {
    case 1: return launch_decode_persist_g<1>(a, batch, ctas, stream);
    case 2: return launch_decode_persist_g<2>(a, batch, ctas, stream);
    case 3: return launch_decode_persist_g<3>(a, batch, ctas, stream);
    case 4: return launch_decode_persist_g<4>(a, batch, ctas, stream);
    case 5: return launch_decode_persist_g<5>(a, batch, ctas, stream);
    case 6: return launch_decode_persist_g<6>(a, batch, ctas, stream);
    case 7: return launch_decode_persist_g<7>(a, batch, ctas, stream);
    case 8: return launch_decode_persist_g<8>(a, batch, ctas, stream);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_persist_combine(const DecodeArgs &a, int group, int batch, cudaStream_t stream) {
  switch (group) {
    case 1: return launch_persist_combine_g<1>(a, batch, stream);
    case 2: return launch_persist_combine_g<2>(a, batch, stream);
    case 3: return launch_persist_combine_g<3>(a, batch, stream);
    case 4: return launch_persist_combine_g<4>(a, batch, stream);
    case 5: return launch_persist_combine_g<5>(a, batch, stream);
    case 6: return launch_persist_combine_g<6>(a, batch, stream);
    case 7: return launch_persist_combine_g<7>(a, batch, stream);
    case 8: return launch_persist_combine_g<8>(a, batch, stream);
    default: return cudaErrorInvalidValue;
  }
}

// CTAs of the persistent kernel one SM holds at once for this head group (0
// if the device cannot be queried); cached per device.
int decode_persist_ctas_per_sm(int group) {
  static int cached[32][9];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  if (group < 1 || group > 8) return 0;
  if (dev >= 0 && dev < 32 && cached[dev][group] > 0) return cached[dev][group];
  int n = 0;
  switch (group) {
    case 1: n = decode_persist_occupancy_g<1>(); break;
    case 2: n = decode_persist_occupancy_g<2>(); break;
    case 3: n = decode_persist_occupancy_g<3>(); break;
    case 4: n = decode_persist_occupancy_g<4>(); break;
    case 5: n = decode_persist_occupancy_g<5>(); break;
    case 6: n = decode_persist_occupancy_g<6>(); break;
    case 7: n = decode_persist_occupancy_g<7>(); break;
    case 8: n = decode_persist_occupancy_g<8>(); break;
    default: break;
  }
  if (n > 0 && dev >= 0 && dev < 32) cached[dev][group] = n;
  return n;
}

}  // namespace hyb
