// decode_b6_skip.cu -- instantiation of the decode kernel for 64-token
// blocks, sparse-L2 (INT4 blocks left out) variant (one translation unit per block size and variant so that
// the build compiles them in parallel).
#include "decode_kernel.cuh"

namespace hyb {
template cudaError_t launch_decode_f<false, true, 6>(const DecodeArgs &, int, int, bool, cudaStream_t);
}  // namespace hyb
