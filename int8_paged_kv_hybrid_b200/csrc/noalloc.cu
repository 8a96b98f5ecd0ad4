// noalloc.cu -- hyb_decode_attn_noalloc: decode attention whose scratch
// memory is a fixed buffer compiled into the library, for callers that cannot
// allocate device memory when they run attention.
//
// Who needs it: code that is handed all of its device memory up front by a
// host application (a fixed budget, a custom allocator the library cannot
// reach, plugins that are forbidden to allocate), or decode loops where an
// allocation could block or fail at the wrong moment.  hyb_decode_attn asks
// such callers for a workspace; this entry point does not.
//
// The buffer is one static device array per GPU that loads the library, held
// until the process exits.  Every call on a device shares it: calls that
// overlap on the GPU (different streams, no ordering between them) race on
// it and must not be issued.  Its contents persist between calls; the part
// that has to start at zero (the split-merge arrival counters) is cleared by
// each call before its kernel runs.
#include <cuda_runtime.h>

#include <mutex>

#include "kernels.cuh"

namespace {

// Largest scratch a call may use.  A call whose splits are merged through the
// scratch needs about rows x (splits + groups) x 516 bytes plus its arrival
// counters (rows = batch x query heads, groups = ceil(splits / 16) above 16
// splits, 512 bytes of partial output and 4 of log-sum-exp per row and
// split or group): e.g. 512 rows (batch 16 x 32 heads) x 15 splits, or 128
// rows x 59 splits.  Plans whose splits merge inside a thread-block cluster
// use none.  Problems that need more are rejected with HYB_ERR_SCRATCH_LIMIT.
constexpr size_t kScratchBytes = 4u << 20;

static __device__ __align__(256) unsigned char g_hyb_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void *g_scratch_ptr[kMaxDevices];  // device address of g_hyb_scratch, per device

// Device address of the scratch array on the current device, looked up once
// per device (the array's name is only a host-side stand-in in host code).
cudaError_t scratch_address(void **out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_hyb_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" {

size_t hyb_noalloc_scratch_limit(void) { return kScratchBytes; }

int hyb_decode_attn_noalloc(const hyb_cache_desc *desc, const void *q, float softmax_scale,
                            int32_t max_seq_len, int32_t split_tokens, void *out, float *lse_out,
                            hyb_stream_t stream) {
  int32_t st = 0, ns = 0;
  const int rc = hyb_decode_plan(desc, max_seq_len, split_tokens, &st, &ns);
  if (rc != HYB_OK) return rc;
  const size_t need = hyb_decode_workspace_bytes(desc, max_seq_len, split_tokens);
  if (need > kScratchBytes) return HYB_ERR_SCRATCH_LIMIT;
  void *ws = nullptr;
  if (need > 0) {
    const cudaError_t e = scratch_address(&ws);
    if (e != cudaSuccess) {
      cudaGetLastError();
      return HYB_ERR_CUDA;
    }
    const size_t zero = hyb::decode_ws_zero_prefix(desc, max_seq_len, split_tokens);
    if (zero > 0) {
      const cudaError_t m = cudaMemsetAsync(ws, 0, zero, reinterpret_cast<cudaStream_t>(stream));
      if (m != cudaSuccess) {
        cudaGetLastError();
        return HYB_ERR_CUDA;
      }
    }
  }
  return hyb_decode_attn(desc, q, softmax_scale, max_seq_len, split_tokens, ws, need, out, lse_out, stream);
}

}  // extern "C"
