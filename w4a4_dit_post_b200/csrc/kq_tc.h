// Internal entry points of the tensor-core quantizer (kq_tc.cu).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace kq {

struct TcGeometry {
  int nb;           // blocks per row
  int C;            // block columns per group (<= 4)
  int NC;           // column groups
  int M;            // rows
  int n_row_tiles;  // ceil(M / 128)
};

// bf16 activations only; arguments already validated by the caller.
int tc_quantize(const void* x, int64_t M, int64_t d, const float* params, uint8_t* codes,
                uint8_t* scales, cudaStream_t stream);

}  // namespace kq
