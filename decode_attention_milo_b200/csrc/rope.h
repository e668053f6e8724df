// Pre-RoPE key factors: host interface of the reconstruct-then-rotate kernel (rope.cu).
#pragma once

#include <cuda.h>
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
  // Device-memory tensor maps of the factor object, 8 each (box heights 16, 32, ..., 128 rows, 128-byte
  // swizzle): the token factor as [rows · n/128][128] bf16 128-token slab rows (3D boxes of 64 columns × h
  // rows × 2 column blocks), the dim factor as [rows][d] bf16 (3D boxes like the token factor's for d = 128,
  // 2D boxes of 64 columns × h rows for d = 64).
  const CUtensorMap* tok_maps;
  const CUtensorMap* dim_maps;
  const int32_t* ranks;        // [2H][nb] (the key pools are the even ones)
  const int64_t* row_offsets;  // [2H][nb + 1]
  // Host copy of the map of the output, the rotated reconstructed keys [H · T][d] bf16, boxes of 128 rows
  // (3D {64, rows, 2} for d = 128, 2D {64, rows} for d = 64), 128-byte swizzle: the kernel stores with it.
  const CUtensorMap* keys_map;
  uint32_t* status;
};
// Rebuilds every key block on the tensor cores and rotates each token at its absolute position.
cudaError_t launch_rope_keys(const RopeShape& s, const RopeBuffers& b, cudaStream_t st);

}  // namespace milo
