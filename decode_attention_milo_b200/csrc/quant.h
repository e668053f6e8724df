// 8-bit token factors: host interface of the quantise kernel (quant.cu).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace milo {

struct QuantShape {
  int P;   // pools (2H)
  int nb;  // blocks per pool
  int n;   // block size
  int d;   // head dim
};
struct QuantBuffers {
  const void* tok;             // bf16 token factors of the source object
  const void* dim;             // bf16 dimension factors of the source object
  const int32_t* ranks;        // [P][nb], each in [1, d]
  const int64_t* row_offsets;  // [P][nb + 1]
  void* qtok;                  // int8 codes, rank r + 1 per block (r at full rank d)
  void* qdim;                  // bf16 folded dimension factors, same ranks
  const int32_t* qranks;       // [P][nb] ranks of the 8-bit object (written by the host)
  const int64_t* qrow_offsets; // [P][nb + 1] its row offsets (written by the host)
  uint32_t* status;
};
cudaError_t launch_quantize(const QuantShape& s, const QuantBuffers& b, cudaStream_t st);

}  // namespace milo
