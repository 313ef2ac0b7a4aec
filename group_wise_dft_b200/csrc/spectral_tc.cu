// tcgen05 tensor-core path (placeholder until the fused kernel lands).
#include "eqlin_internal.cuh"

namespace eqlin {

__device__ unsigned int g_fault_word = 0;

int read_device_fault(int reset) {
  unsigned int v = 0;
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return -(int)e;
  e = cudaMemcpyFromSymbol(&v, g_fault_word, sizeof v);
  if (e != cudaSuccess) return -(int)e;
  if (reset && v) {
    const unsigned int z = 0;
    e = cudaMemcpyToSymbol(g_fault_word, &z, sizeof z);
    if (e != cudaSuccess) return -(int)e;
  }
  return (int)v;
}

bool cyclic_tc_supported(int, int, int, int) { return false; }
bool d8_tc_supported(int, int) { return false; }
size_t cyclic_tc_bytes(int, int, int) { return 0; }
size_t d8_tc_bytes(int) { return 0; }
int launch_cyclic_tc_pack(const void *, int, int, int, void *, cudaStream_t) {
  return set_error(EQLIN_ERR_UNSUPPORTED, "tensor-core path not built");
}
int launch_d8_tc_pack(const void *const[5], int, void *, cudaStream_t) {
  return set_error(EQLIN_ERR_UNSUPPORTED, "tensor-core path not built");
}
int launch_cyclic_tc(const void *, const void *, void *, int64_t, int, int, cudaStream_t) {
  return set_error(EQLIN_ERR_UNSUPPORTED, "tensor-core path not built");
}
int launch_d8_tc(const void *, const void *, void *, int64_t, int, int, cudaStream_t) {
  return set_error(EQLIN_ERR_UNSUPPORTED, "tensor-core path not built");
}

}  // namespace eqlin
