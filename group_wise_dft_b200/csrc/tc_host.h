// Host-side helpers of the tensor-core translation units.
#pragma once

#include <cuda.h>
#include <stdint.h>

namespace eqlin {

// 2-D bf16 tensor map over a row-major [outer][inner] array (row_bytes apart),
// box box_inner x box_outer elements, 128-byte swizzle or none; zero fill out
// of bounds.  Returns an EQLIN_* status.
int tma_map_2d_bf16(CUtensorMap *m, const void *ptr, uint64_t inner, uint64_t outer,
                    uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, bool swizzle128);

// Device address of the tensor-core kernels' fault word on the current device
// (looked up once per device).  Kernels of other translation units receive it
// as an argument; eqlin_device_fault reads the same word.
int fault_word_address(unsigned int **out);   // the two fault words (tc::FaultCtx)

}  // namespace eqlin
