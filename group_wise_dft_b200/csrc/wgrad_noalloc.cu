// Weight gradient of the cyclic layer for callers that cannot allocate device
// memory.
//
// eqlin_cyclic_weight_grad needs a caller-provided workspace for its per-split
// partial sums.  Some callers have no way to provide one: code that runs where
// calling cudaMalloc is not allowed or not safe (inside a custom allocator or
// a memory-pool callback, in a process whose device memory is fully reserved
// up front by a framework, or in a plugin that must not touch the device heap
// at all).  This entry point is for them: it keeps the partial sums in a
// fixed-size array that is part of the library's own device image, so the
// call itself allocates nothing.
//
// The array is a file-scope __device__ variable, so every GPU that loads the
// library holds its kNoAllocScratchBytes until the process exits.  Host code
// cannot pass the array's name to a kernel (in host code it is only a
// stand-in, not a device address), so the device address is looked up with
// cudaGetSymbolAddress, once per device, the first time this entry point runs
// on that device, and cached.  The cache does not survive cudaDeviceReset: a
// caller that resets a device must not call this entry point on it again in
// the same process.
#include <mutex>

#include "eqlin_internal.cuh"

namespace eqlin {
namespace {

// 8 MiB (the header's EQLIN_NOALLOC_SCRATCH_BYTES): one token split of a
// 160 x 160-field, N = 8 layer is 0.8 MiB, so layers of that size still get
// ten splits.
constexpr size_t kNoAllocScratchBytes = EQLIN_NOALLOC_SCRATCH_BYTES;
static_assert(kNoAllocScratchBytes == (size_t(8) << 20) && kNoAllocScratchBytes % 256 == 0,
              "the scratch size is the documented 8 MiB");

static __device__ __align__(256) float g_noalloc_scratch[kNoAllocScratchBytes / sizeof(float)];

std::mutex g_noalloc_mu;
void *g_noalloc_ptr[64] = {};   // per device: the array's device address, once looked up

// The array's device address for the current device (set-up on first use).
int noalloc_scratch(float **out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return set_error(EQLIN_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= 64) return set_error(EQLIN_ERR_UNSUPPORTED, "device index %d >= 64", dev);
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || !p)
      return set_error(EQLIN_ERR_CUDA, "cudaGetSymbolAddress of the weight-gradient scratch: %s",
                       cudaGetErrorString(e));
    g_noalloc_ptr[dev] = p;
  }
  *out = static_cast<float *>(g_noalloc_ptr[dev]);
  return EQLIN_OK;
}

}  // namespace
}  // namespace eqlin

using namespace eqlin;

extern "C" EQLIN_API int eqlin_cyclic_weight_grad_noalloc(const void *x, const void *dy, void *dW,
                                                          int64_t T, int N, int Cin, int Cout,
                                                          int dtype, eqlin_stream_t stream) {
  clear_error();
  const int shape_rc = check_cyclic_shape(N, Cin, Cout, dtype);
  if (shape_rc != EQLIN_OK) return shape_rc;
  if (T < 0) return set_error(EQLIN_ERR_INVALID_ARG, "T=%lld < 0", (long long)T);
  if (!dW || (T > 0 && (!x || !dy))) return set_error(EQLIN_ERR_INVALID_ARG, "null pointer");
  if (((uintptr_t)dW & 15u) || (T > 0 && (((uintptr_t)x & 15u) || ((uintptr_t)dy & 15u))))
    return set_error(EQLIN_ERR_ALIGN, "x, dy and dW must be 16-byte aligned");
  // as many token splits as the workspace version uses, but no more than fit
  const size_t split_bytes = cyclic_wgrad_part_bytes(1, N, Cin, Cout);
  const int64_t fit = (int64_t)(kNoAllocScratchBytes / split_bytes);
  if (T > 0 && fit < 1)
    return set_error(EQLIN_ERR_SIZE,
                     "Cin*Cout*N*4 = %zu bytes exceeds the fixed %zu-byte scratch of "
                     "eqlin_cyclic_weight_grad_noalloc; use eqlin_cyclic_weight_grad with a workspace",
                     split_bytes, kNoAllocScratchBytes);
  int S = cyclic_wgrad_splits(T, Cin, Cout);
  if (S > fit) S = (int)fit;
  float *scratch = nullptr;
  if (S > 0) {
    const int rc = noalloc_scratch(&scratch);
    if (rc != EQLIN_OK) return rc;
  }
  return launch_cyclic_wgrad(x, dy, dW, T, N, Cin, Cout, dtype, scratch, S, (cudaStream_t)stream);
}
