// decode_b6_plain.cu -- instantiation of the decode kernel for 64-token
// blocks, dense variant (one translation unit per block size and variant so that
// the build compiles them in parallel).
#include "decode_kernel.cuh"

namespace hyb {
template cudaError_t launch_decode_f<false, false, 6>(const DecodeArgs &, int, int, bool, cudaStream_t);
template int decode_occupancy<false, false, 6>(int);
template int decode_active_clusters<false, false, 6>(int, int);
}  // namespace hyb
