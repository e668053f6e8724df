// 8-bit storage of the token-side factors: asymmetric INT8 codes per rank channel of each block.
//
// Page "MILO: Efficient Many-shot In-Context Learning with Block-wise Low-rank
// Compression", §5.3: the compressed caches compose with asymmetric INT8 (and
// KIVI) quantisation for further memory savings.  The page names no scheme;
// this file takes the plainest one that keeps the decode unchanged:
//   * each rank component j of a block's token factor (U_b for keys, P_b for
//     values) over the block's n tokens is one channel: lo = min, hi = max,
//     a = (hi − lo)/255, code c_t = round((x_t − lo)/a) − 128 (half to even),
//     all in fp32 (a constant channel, a = 0, gets c_t = −128);
//   * the scales and minima go into the dimension-side factor, with one more
//     component whose codes are all 1:
//       B̂_j = a_j·B_j (j < r),   B̂_r = Σ_j (lo_j + 128·a_j)·B_j
//     so codes·B̂ᵀ reproduces the dequantized block exactly and the rank-space
//     decode runs on (codes, B̂) at rank r + 1;
//   * a block stored at full rank r = d, where one more component would exceed
//     the head dimension, takes the symmetric form: a = max|x_t|/127,
//     c_t = round(x_t/a) in [−127, 127] (a = 0 gives 0), B̂_j = a_j·B_j, rank d.
// One CTA per block: a warp per channel finds its range, then the codes, the
// all-ones row and the dimension rows are written in the factor layout of the
// new object, whose ranks and row offsets the host has computed.
#include <cuda_bf16.h>

#include "common.cuh"
#include "quant.h"

namespace milo {
namespace {

constexpr int kQThreads = 256;

__global__ void __launch_bounds__(kQThreads) quantize_kernel(const __nv_bfloat16* __restrict__ tok,
                                                            const __nv_bfloat16* __restrict__ dim,
                                                            const int32_t* __restrict__ ranks,
                                                            const int64_t* __restrict__ row_offsets, int nb, int n,
                                                            int d, int8_t* __restrict__ qtok,
                                                            __nv_bfloat16* __restrict__ qdim,
                                                            const int32_t* __restrict__ qranks,
                                                            const int64_t* __restrict__ qrow_offsets, uint32_t* status) {
  __shared__ float s_scale[128], s_lo[128];
  const int p = blockIdx.y, b = blockIdx.x;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int r = ranks[(size_t)p * nb + b];
  const int64_t row0 = row_offsets[(size_t)p * (nb + 1) + b];
  const int rq = qranks[(size_t)p * nb + b];
  const int64_t qrow0 = qrow_offsets[(size_t)p * (nb + 1) + b];
  const int cpb = n / 128;
  const bool sym = r == d;  // full rank: symmetric, no extra component
  if (r < 1 || r > d || rq != (sym ? r : r + 1)) {
    if (threadIdx.x == 0) atomicOr(status, kStatusCompressBounds);
    return;
  }
  // token t of channel j: slab t / 128, row (row0·cpb + slab·r + j), column t % 128
  auto src = [&](int j, int t) { return tok + ((row0 * cpb + (int64_t)(t >> 7) * r + j) << 7) + (t & 127); };
  auto dst = [&](int j, int t) { return qtok + ((qrow0 * cpb + (int64_t)(t >> 7) * rq + j) << 7) + (t & 127); };
  for (int j = warp; j < r; j += kQThreads / 32) {
    float lo = INFINITY, hi = -INFINITY;
    for (int t = lane; t < n; t += 32) {
      const float x = __bfloat162float(*src(j, t));
      lo = fminf(lo, x);
      hi = fmaxf(hi, x);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
      hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
    }
    // asymmetric: a = (hi − lo)/255, c = round((x − lo)/a) − 128; symmetric: a = max|x|/127, c = round(x/a)
    const float a = sym ? __fdiv_rn(fmaxf(-lo, hi), 127.0f) : __fdiv_rn(__fsub_rn(hi, lo), 255.0f);
    for (int t = lane; t < n; t += 32) {
      int c = sym ? 0 : -128;
      if (a > 0.f) {
        const float x = __bfloat162float(*src(j, t));
        if (sym) c = (int)fminf(fmaxf(rintf(__fdiv_rn(x, a)), -127.f), 127.f);
        else c = (int)fminf(fmaxf(rintf(__fdiv_rn(__fsub_rn(x, lo), a)), 0.f), 255.f) - 128;
      }
      *dst(j, t) = (int8_t)c;
    }
    if (lane == 0) {
      s_scale[j] = a;
      s_lo[j] = lo;
    }
  }
  if (!sym)
    for (int t = threadIdx.x; t < n; t += kQThreads) *dst(r, t) = 1;  // the extra component: code 1 everywhere
  __syncthreads();
  // dimension rows: B̂_j = a_j·B_j, and (asymmetric) the offset row Σ_j (lo_j + 128·a_j)·B_j
  for (int e = threadIdx.x; e < d; e += kQThreads) {
    float off = 0.f;
    for (int j = 0; j < r; ++j) {
      const float bj = __bfloat162float(dim[(row0 + j) * d + e]);
      qdim[(qrow0 + j) * d + e] = __float2bfloat16_rn(s_scale[j] * bj);
      off = fmaf(fmaf(128.f, s_scale[j], s_lo[j]), bj, off);
    }
    if (!sym) qdim[(qrow0 + r) * d + e] = __float2bfloat16_rn(off);
  }
}

}  // namespace

cudaError_t launch_quantize(const QuantShape& s, const QuantBuffers& b, cudaStream_t st) {
  if (s.n % 128 != 0 || s.d > 128 || s.P <= 0 || s.nb <= 0 || s.nb > 65535) return cudaErrorInvalidValue;
  quantize_kernel<<<dim3(s.nb, s.P), kQThreads, 0, st>>>(
      static_cast<const __nv_bfloat16*>(b.tok), static_cast<const __nv_bfloat16*>(b.dim), b.ranks, b.row_offsets, s.nb,
      s.n, s.d, static_cast<int8_t*>(b.qtok), static_cast<__nv_bfloat16*>(b.qdim), b.qranks, b.qrow_offsets, b.status);
  return cudaGetLastError();
}

}  // namespace milo
