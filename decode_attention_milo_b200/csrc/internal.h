// Host-side interfaces between the C-ABI layer and the kernel files.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace milo {

struct CompressShape {
  int H;       // KV heads
  int64_t T;   // context
  int d;       // head dim
  int n;       // block size
  int nb;      // blocks per pool
  int R;       // total rank of one allocation group: a pool, or with layer_scope all 2H pools (before capping)
  int pool_rows;  // rows per pool, min(R, nb*d) (pool scope only)
  int r_min;
  int max_sweeps;
  bool bf16;
  int rule = 0;             // 0 entropy, 1 greedy, 2 uniform, 3 caller weights
  bool layer_scope = false; // one budget over all pools of the layer
};

struct CompressBuffers {
  const void* K;
  const void* V;
  float* gram;        // [2H][nb][d][d]
  float* eigvals;     // [2H][nb][d]
  int32_t* sweeps;    // [2H][nb] Jacobi sweeps run per block (the last one converged)
  float* eigvecs;     // [2H][nb][d][d]
  double* entropy;    // [2H][nb]
  double* quotas;     // [2H][nb]
  const double* weights;  // [2H][nb] device, rule 3 only
  int32_t* ranks;     // [2H][nb]
  int64_t* row_offsets;  // [2H][nb+1]
  void* tok;          // [2H*pool_rows][n]
  void* dim;          // [2H*pool_rows][d]
  uint32_t* status;
};

// ev (optional, 5 events): recorded before the Gram, Jacobi, allocation and projection kernels and after the last.
cudaError_t launch_compress(const CompressShape& s, const CompressBuffers& b, cudaStream_t st,
                            const cudaEvent_t* ev = nullptr);
// Tensor-core Gram of bf16 blocks (d in {64, 128}, n % 128 == 0); cudaErrorNotSupported otherwise.
bool gram_tc_supported(const CompressShape& s);
cudaError_t launch_gram_tc(const CompressShape& s, const void* K, const void* V, float* gram, uint32_t* status,
                           cudaStream_t st);

// Tensor-core projection of bf16 blocks (d in {64, 128}, n % 128 == 0); cudaErrorNotSupported otherwise.
bool project_tc_supported(const CompressShape& s);
cudaError_t launch_project_tc(const CompressShape& s, const void* K, const void* V, const float* eigvecs,
                              const int32_t* ranks, const int64_t* row_offsets, void* tok, void* dim,
                              uint32_t* status, cudaStream_t st);

// Rank-space decode on CUDA cores (any dtype; the fp32 path and a cross-check for bf16).
struct DecodeShape {
  int H, nb, n, d, Bq, Hq, S;
  bool bf16;
  float scale;
};
struct DecodeBuffers {
  const void* q;
  const void* K_suf;
  const void* V_suf;
  const int32_t* ranks;
  const int64_t* row_offsets;
  const void* tok;
  const void* dim;
  float* partials;  // [(H*nb*rows) + Bq*H*G][d+2]
  void* out;
  uint32_t* status;
};
size_t simt_decode_partials_floats(const DecodeShape& s);
// ev0 / ev1 (optional) are recorded on `st` right before and right after the per-block kernel.
cudaError_t launch_decode_simt(const DecodeShape& s, const DecodeBuffers& b, cudaStream_t st,
                               cudaEvent_t ev0 = nullptr, cudaEvent_t ev1 = nullptr);

}  // namespace milo
