// decode_b7_f16.cu -- instantiation of the decode kernel for 128-token
// blocks, FP16 cold block variant (one translation unit per block size and variant so that
// the build compiles them in parallel).
#include "decode_kernel.cuh"

namespace hyb {
template cudaError_t launch_decode_f<true, false, 7>(const DecodeArgs &, int, int, bool, cudaStream_t);
}  // namespace hyb
