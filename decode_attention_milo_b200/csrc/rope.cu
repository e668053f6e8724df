// Reconstruct-then-rotate of pre-RoPE key factors, for the decode over them.
//
// Page "MILO: Efficient Many-shot In-Context Learning with Block-wise Low-rank
// Compression": pre-RoPE keys suit low-rank compression better (§3, Figure 1),
// and inference reconstructs the selected blocks before attention (§4.4, §4.5).
// With K_b ≈ U_b·B_bᵀ stored for the keys before the rotary embedding, the
// scores need the rotated keys, which no rank-space identity gives (the
// rotation depends on the token), so every block is rebuilt here:
//   K[t] = Σ_j U_b[t, j]·B_b[:, j],  then the half-split rotation of each pair
//   (i, i + d/2) by φ_i = pos·θ^(−2i/d), pos = t (the token's absolute position),
// and written as bf16 [H][T][d], the dense key layout the decode kernel reads.
// One CTA per (KV head, block, 128-token chunk): the chunk's token factor and
// the block's dimension factor in shared memory as fp32, each thread one token
// and half of its pairs, the angle reduced in fp64 before the fp32 sine and
// cosine, and the rows staged through shared memory for coalesced stores.
#include <cuda_bf16.h>

#include "common.cuh"
#include "rope.h"

namespace milo {
namespace {

constexpr int kRThreads = 256;

template <int D>
__global__ void __launch_bounds__(kRThreads) rope_keys_kernel(const __nv_bfloat16* __restrict__ tok,
                                                             const __nv_bfloat16* __restrict__ dim,
                                                             const int32_t* __restrict__ ranks,
                                                             const int64_t* __restrict__ row_offsets, int nb, int n,
                                                             int64_t T, double log2_theta,
                                                             __nv_bfloat16* __restrict__ keys, uint32_t* status) {
  constexpr int P = D / 2;               // pairs per token
  constexpr int PT = P / 2;              // pairs per thread (two threads per token)
  extern __shared__ float rs[];
  float* Us = rs;                         // [128 ranks max][128 tokens]
  float* Bs = rs + 128 * 128;             // [128 ranks max][D]
  constexpr int KS = D + 8;               // staging row stride: 16 bytes of padding spread the banks
  __nv_bfloat16* Ks = reinterpret_cast<__nv_bfloat16*>(Bs + 128 * D);  // [128 tokens][KS]
  const int cpb = n / 128;
  const int c = blockIdx.x % cpb, b = (blockIdx.x / cpb) % nb, h = blockIdx.x / (cpb * nb);
  const int r = ranks[(size_t)(2 * h) * nb + b];
  const int64_t row0 = row_offsets[(size_t)(2 * h) * (nb + 1) + b];
  if (r < 1 || r > D) {
    if (threadIdx.x == 0) atomicOr(status, kStatusDecodeBounds);
    return;
  }
  // slab c of the block: rows row0·cpb + c·r + j, 128 tokens each
  const __nv_bfloat16* u = tok + ((row0 * cpb + (int64_t)c * r) << 7);
  for (int e = threadIdx.x; e < r * 128; e += kRThreads) Us[e] = __bfloat162float(u[e]);
  for (int e = threadIdx.x; e < r * D; e += kRThreads) Bs[e] = __bfloat162float(dim[row0 * D + e]);
  __shared__ double s_freq[P];  // θ^(−2i/d)
  for (int i = threadIdx.x; i < P; i += kRThreads) s_freq[i] = exp2(-2.0 * i / D * log2_theta);
  __syncthreads();
  const int t = threadIdx.x % 128, i0 = (threadIdx.x / 128) * PT;
  float a1[PT], a2[PT];
#pragma unroll
  for (int k = 0; k < PT; ++k) a1[k] = a2[k] = 0.f;
  for (int j = 0; j < r; ++j) {
    const float uj = Us[j * 128 + t];
    const float4* b1 = reinterpret_cast<const float4*>(Bs + j * D + i0);      // the same address in a warp:
    const float4* b2 = reinterpret_cast<const float4*>(Bs + j * D + i0 + P);  // broadcast 16-byte loads
#pragma unroll
    for (int k = 0; k < PT / 4; ++k) {
      const float4 x = b1[k], y = b2[k];
      a1[4 * k] = fmaf(uj, x.x, a1[4 * k]);
      a1[4 * k + 1] = fmaf(uj, x.y, a1[4 * k + 1]);
      a1[4 * k + 2] = fmaf(uj, x.z, a1[4 * k + 2]);
      a1[4 * k + 3] = fmaf(uj, x.w, a1[4 * k + 3]);
      a2[4 * k] = fmaf(uj, y.x, a2[4 * k]);
      a2[4 * k + 1] = fmaf(uj, y.y, a2[4 * k + 1]);
      a2[4 * k + 2] = fmaf(uj, y.z, a2[4 * k + 2]);
      a2[4 * k + 3] = fmaf(uj, y.w, a2[4 * k + 3]);
    }
  }
  const int64_t pos = (int64_t)b * n + (int64_t)c * 128 + t;
  constexpr double kTwoPi = 6.283185307179586;
#pragma unroll
  for (int k = 0; k < PT; ++k) {
    const int i = i0 + k;
    // φ = pos·θ^(−2i/d) in fp64, reduced to [−π, π] before the fp32 sine and cosine
    const double phi = (double)pos * s_freq[i];
    const float red = (float)(phi - kTwoPi * rint(phi / kTwoPi));
    float sn, cs;
    sincosf(red, &sn, &cs);
    Ks[t * KS + i] = __float2bfloat16_rn(a1[k] * cs - a2[k] * sn);
    Ks[t * KS + i + P] = __float2bfloat16_rn(a2[k] * cs + a1[k] * sn);
  }
  __syncthreads();
  // rows pos0 .. pos0 + 127 of head h, 16 bytes per store
  const int64_t pos0 = (int64_t)b * n + (int64_t)c * 128;
  uint4* dst = reinterpret_cast<uint4*>(keys + ((int64_t)h * T + pos0) * D);
  for (int e = threadIdx.x; e < 128 * D / 8; e += kRThreads) {
    const int row = e / (D / 8), col = e % (D / 8);
    dst[e] = *reinterpret_cast<const uint4*>(Ks + row * KS + col * 8);
  }
}

template <int D>
size_t rope_smem() { return (size_t)(128 * 128 + 128 * D) * sizeof(float) + (size_t)128 * (D + 8) * sizeof(__nv_bfloat16); }

}  // namespace

cudaError_t launch_rope_keys(const RopeShape& s, const RopeBuffers& b, cudaStream_t st) {
  if ((s.d != 64 && s.d != 128) || s.n % 128 != 0 || s.H <= 0 || s.nb <= 0 || !(s.theta > 1.0))
    return cudaErrorInvalidValue;
  const int64_t grid = (int64_t)s.H * s.nb * (s.n / 128);
  if (grid > 0x7fffffff) return cudaErrorInvalidValue;
  const double l2t = log2(s.theta);
  const int64_t T = (int64_t)s.nb * s.n;
  cudaError_t e;
  if (s.d == 64) {
    if ((e = cudaFuncSetAttribute(rope_keys_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)rope_smem<64>())) != cudaSuccess)
      return e;
    rope_keys_kernel<64><<<(unsigned)grid, kRThreads, rope_smem<64>(), st>>>(
        static_cast<const __nv_bfloat16*>(b.tok), static_cast<const __nv_bfloat16*>(b.dim), b.ranks, b.row_offsets,
        s.nb, s.n, T, l2t, static_cast<__nv_bfloat16*>(b.keys), b.status);
  } else {
    if ((e = cudaFuncSetAttribute(rope_keys_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)rope_smem<128>())) != cudaSuccess)
      return e;
    rope_keys_kernel<128><<<(unsigned)grid, kRThreads, rope_smem<128>(), st>>>(
        static_cast<const __nv_bfloat16*>(b.tok), static_cast<const __nv_bfloat16*>(b.dim), b.ranks, b.row_offsets,
        s.nb, s.n, T, l2t, static_cast<__nv_bfloat16*>(b.keys), b.status);
  }
  return cudaGetLastError();
}

}  // namespace milo
