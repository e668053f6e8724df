// Pre-RoPE key factors: host interface of the reconstruct-then-rotate kernel (rope.cu).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace milo {

struct RopeShape {
  int H;         // KV heads
  int nb;        // blocks per pool
  int n;         // block size (multiple of 128)
  int d;         // head dim (64 or 128)
  double theta;  // rotary base (> 1)
};
struct RopeBuffers {
  const void* tok;             // bf16 token factors of the factor object
  const void* dim;             // bf16 dimension factors
  const int32_t* ranks;        // [2H][nb] (the key pools are the even ones)
  const int64_t* row_offsets;  // [2H][nb + 1]
  void* keys;                  // bf16 [H][T][d]: the rotated reconstructed keys
  uint32_t* status;
};
// Rebuilds every key block and rotates each token at its absolute position.
cudaError_t launch_rope_keys(const RopeShape& s, const RopeBuffers& b, cudaStream_t st);

}  // namespace milo
