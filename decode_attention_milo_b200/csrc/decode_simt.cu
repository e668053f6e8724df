// Rank-space decode attention on CUDA cores (fp32 path; also any dtype for cross-checks).
//
// Page "MILO: Efficient Many-shot In-Context Learning with Block-wise Low-rank
// Compression", §4.4: decoding attends over the stored low-rank caches.  With
// K_b ≈ U_b·B_bᵀ and V_b ≈ P_b·Q_bᵀ the scores of block b are (q·B_b)·U_bᵀ and
// its value sum is (p·P_b)·Q_bᵀ, so blocks are never expanded.
//
// One CTA per (block, KV head, query row) computes a softmax partial
// (m, l, acc[d]) for that block; one CTA per (suffix, query row) does the same
// for the uncompressed suffix; a combine kernel merges the partials of each
// output row.  Simple and exact in fp32; the bf16 hot path is the tensor-core
// kernel.
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace milo {
namespace {

constexpr int kThreads = 128;

__device__ float block_max(float v, float* red) {
  v = warp_max(v);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float t = red[0];
  for (int w = 1; w < kThreads / 32; ++w) t = fmaxf(t, red[w]);
  return t;
}
__device__ float block_sum(float v, float* red) {
  v = warp_sum(v);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float t = 0.f;
  for (int w = 0; w < kThreads / 32; ++w) t += red[w];
  return t;
}

template <typename T, int D>
__global__ void __launch_bounds__(kThreads) prefix_kernel(const T* __restrict__ q, const T* __restrict__ tok,
                                                         const T* __restrict__ dim,
                                                         const int32_t* __restrict__ ranks,
                                                         const int64_t* __restrict__ row_offsets, int H, int nb,
                                                         int n, int Hq, int G, float scale,
                                                         float* __restrict__ partials, uint32_t* status) {
  extern __shared__ float s[];  // n scores / probabilities
  __shared__ float qs[D], qt[D], red[kThreads / 32];
  const int rho = blockIdx.x, b = blockIdx.y, h = blockIdx.z;
  const int rows = gridDim.x;
  const int i = rho / G, g = rho % G;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const T* qrow = q + ((int64_t)i * Hq + h * G + g) * D;
  for (int c = threadIdx.x; c < D; c += kThreads) qs[c] = to_f32(qrow[c]);
  const int pk = 2 * h, pv = 2 * h + 1;
  const int rk = ranks[(int64_t)pk * nb + b], rv = ranks[(int64_t)pv * nb + b];
  if (rk < 0 || rk > D || rv < 0 || rv > D) {
    if (threadIdx.x == 0) atomicOr(status, kStatusDecodeBounds);
    return;
  }
  const int64_t ok = row_offsets[(int64_t)pk * (nb + 1) + b];
  const int64_t ov = row_offsets[(int64_t)pv * (nb + 1) + b];
  __syncthreads();
  // q̃ = q · B_b
  for (int j = warp; j < rk; j += kThreads / 32) {
    const T* brow = dim + (ok + j) * D;
    float a = 0.f;
    for (int c = lane; c < D; c += 32) a = fmaf(qs[c], to_f32(brow[c]), a);
    a = warp_sum(a);
    if (lane == 0) qt[j] = a;
  }
  __syncthreads();
  // scores = scale · q̃ · U_bᵀ
  float mloc = -INFINITY;
  for (int t = threadIdx.x; t < n; t += kThreads) {
    float a = 0.f;
    const T* col = tok + ok * n + (int64_t)(t >> 7) * (rk * 128) + (t & 127);  // chunk-major slab
    for (int j = 0; j < rk; ++j) a = fmaf(qt[j], to_f32(col[j * 128]), a);
    a *= scale;
    s[t] = a;
    mloc = fmaxf(mloc, a);
  }
  const float m = block_max(mloc, red);
  float lloc = 0.f;
  for (int t = threadIdx.x; t < n; t += kThreads) {
    const float e = expf(s[t] - m);
    s[t] = e;
    lloc += e;
  }
  const float l = block_sum(lloc, red);  // contains __syncthreads: s[] complete below
  // ã = p · P_b
  for (int j = warp; j < rv; j += kThreads / 32) {
    const T* slab = tok + ov * n + j * 128;
    float a = 0.f;
    for (int t = lane; t < n; t += 32) a = fmaf(s[t], to_f32(slab[(int64_t)(t >> 7) * (rv * 128) + (t & 127)]), a);
    a = warp_sum(a);
    if (lane == 0) qt[j] = a;
  }
  __syncthreads();
  // acc = ã · Q_bᵀ
  float* out = partials + (((int64_t)h * nb + b) * rows + rho) * (D + 2);
  for (int c = threadIdx.x; c < D; c += kThreads) {
    float a = 0.f;
    for (int j = 0; j < rv; ++j) a = fmaf(qt[j], to_f32(dim[(ov + j) * D + c]), a);
    out[c] = a;
  }
  if (threadIdx.x == 0) {
    out[D] = m;
    out[D + 1] = l;
  }
}

template <typename T, int D>
__global__ void __launch_bounds__(kThreads) suffix_kernel(const T* __restrict__ q, const T* __restrict__ Ks,
                                                         const T* __restrict__ Vs, int H, int S, int Hq, int G,
                                                         float scale, float* __restrict__ partials) {
  extern __shared__ float s[];  // S
  __shared__ float qs[D], red[kThreads / 32];
  const int g = blockIdx.x, i = blockIdx.y, h = blockIdx.z;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const T* qrow = q + ((int64_t)i * Hq + h * G + g) * D;
  for (int c = threadIdx.x; c < D; c += kThreads) qs[c] = to_f32(qrow[c]);
  __syncthreads();
  const T* K = Ks + ((int64_t)i * H + h) * S * D;
  const T* V = Vs + ((int64_t)i * H + h) * S * D;
  float mloc = -INFINITY;
  for (int t = warp; t < S; t += kThreads / 32) {
    float a = 0.f;
    for (int c = lane; c < D; c += 32) a = fmaf(qs[c], to_f32(K[(int64_t)t * D + c]), a);
    a = warp_sum(a) * scale;
    if (lane == 0) s[t] = a;
    mloc = fmaxf(mloc, a);
  }
  const float m = block_max(mloc, red);
  float lloc = 0.f;
  for (int t = threadIdx.x; t < S; t += kThreads) {
    const float e = expf(s[t] - m);
    s[t] = e;
    lloc += e;
  }
  const float l = block_sum(lloc, red);
  float* out = partials + (((int64_t)i * H + h) * G + g) * (D + 2);
  for (int c = threadIdx.x; c < D; c += kThreads) {
    float a = 0.f;
    for (int t = 0; t < S; ++t) a = fmaf(s[t], to_f32(V[(int64_t)t * D + c]), a);
    out[c] = a;
  }
  if (threadIdx.x == 0) {
    out[D] = m;
    out[D + 1] = l;
  }
}

// Merges the partials of one output row (i, hq): m = max m_k, l = Σ l_k e^{m_k−m}, out = Σ acc_k e^{m_k−m} / l.
template <typename T, int D>
__global__ void __launch_bounds__(D) combine_kernel(const float* __restrict__ partials, int H, int nb, int Hq,
                                                   int G, int rows, int S, T* __restrict__ out) {
  const int hq = blockIdx.x, i = blockIdx.y, c = threadIdx.x;
  const int h = hq / G, g = hq % G, rho = i * G + g;
  const float* pre = partials + ((int64_t)h * nb * rows + rho) * (D + 2);
  const int64_t stride = (int64_t)rows * (D + 2);
  const float* suf = partials + (int64_t)H * nb * rows * (D + 2) + (((int64_t)i * H + h) * G + g) * (D + 2);
  float m = -INFINITY;
  for (int b = 0; b < nb; ++b) m = fmaxf(m, pre[b * stride + D]);
  if (S > 0) m = fmaxf(m, suf[D]);
  float l = 0.f, acc = 0.f;
  for (int b = 0; b < nb; ++b) {
    const float* pb = pre + b * stride;
    const float w = expf(pb[D] - m);
    l = fmaf(pb[D + 1], w, l);
    acc = fmaf(pb[c], w, acc);
  }
  if (S > 0) {
    const float w = expf(suf[D] - m);
    l = fmaf(suf[D + 1], w, l);
    acc = fmaf(suf[c], w, acc);
  }
  out[((int64_t)i * Hq + hq) * D + c] = from_f32<T>(acc / l);
}

template <typename T, int D>
cudaError_t run(const DecodeShape& s, const DecodeBuffers& b, cudaStream_t st, cudaEvent_t ev0, cudaEvent_t ev1) {
  const int G = s.Hq / s.H, rows = s.Bq * G;
  const T* q = static_cast<const T*>(b.q);
  const size_t psm = (size_t)s.n * sizeof(float);
  if (psm > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(prefix_kernel<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)psm);
    if (e != cudaSuccess) return e;
  }
  if (ev0) cudaEventRecord(ev0, st);
  prefix_kernel<T, D><<<dim3(rows, s.nb, s.H), kThreads, psm, st>>>(
      q, static_cast<const T*>(b.tok), static_cast<const T*>(b.dim), b.ranks, b.row_offsets, s.H, s.nb, s.n,
      s.Hq, G, s.scale, b.partials, b.status);
  if (ev1) cudaEventRecord(ev1, st);
  if (s.S > 0) {
    const size_t ssm = (size_t)s.S * sizeof(float);
    if (ssm > 48 * 1024) {
      cudaError_t e = cudaFuncSetAttribute(suffix_kernel<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)ssm);
      if (e != cudaSuccess) return e;
    }
    suffix_kernel<T, D><<<dim3(G, s.Bq, s.H), kThreads, ssm, st>>>(
        q, static_cast<const T*>(b.K_suf), static_cast<const T*>(b.V_suf), s.H, s.S, s.Hq, G, s.scale,
        b.partials + (size_t)s.H * s.nb * rows * (D + 2));
  }
  combine_kernel<T, D><<<dim3(s.Hq, s.Bq), D, 0, st>>>(b.partials, s.H, s.nb, s.Hq, G, rows, s.S,
                                                        static_cast<T*>(b.out));
  return cudaGetLastError();
}

}  // namespace

size_t simt_decode_partials_floats(const DecodeShape& s) {
  const int G = s.Hq / s.H;
  return ((size_t)s.H * s.nb * s.Bq * G + (size_t)s.Bq * s.H * G) * (s.d + 2);
}

cudaError_t launch_decode_simt(const DecodeShape& s, const DecodeBuffers& b, cudaStream_t st, cudaEvent_t ev0,
                               cudaEvent_t ev1) {
  if (s.bf16) {
    if (s.d == 64) return run<__nv_bfloat16, 64>(s, b, st, ev0, ev1);
    return run<__nv_bfloat16, 128>(s, b, st, ev0, ev1);
  }
  if (s.d == 64) return run<float, 64>(s, b, st, ev0, ev1);
  return run<float, 128>(s, b, st, ev0, ev1);
}

}  // namespace milo
