// Block-wise low-rank compression (encode side of MILO).
//
// Page "MILO: Efficient Many-shot In-Context Learning with Block-wise Low-rank
// Compression": §4.2 splits each KV pool into blocks and approximates each
// block's keys and values separately at low rank; §4.3 sets each block's rank
// from its entropy under a fixed total budget.  Four kernels per layer, all on
// the caller's stream:
//   gram     G_b = X_bᵀ X_b in fp32  (bf16 blocks: tensor cores, gram_tc.cu; fp32: here, one CTA per block)
//   jacobi   one-sided Jacobi on G_b: eigenvalues λ_i = σ_i², eigenvectors B_b,
//            sorted descending                            (one CTA per block)
//   alloc    H_b = −Σ p ln p (p = λ/Σλ, fp64), w_b = e^{H_b}, quotas
//            clamp(lam·w_b, r_min, d) with Σ = R, largest-remainder ranks,
//            row offsets                                  (one CTA per pool)
//   project  U_b = X_b · B_b[:, :r_b], stored transposed in 128-token slabs, and B_bᵀ rows
//                                                         (one CTA per block)
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace milo {
namespace {

constexpr int kThreads = 256;
// Jacobi runs one CTA per block with 128 KB of shared memory (one CTA per SM), so it uses more warps to hide
// the latency of each round: 16 warps, 4 column pairs per warp per round (d = 128).
constexpr int kJThreads = 512;
constexpr float kJacobiTol = 1e-5f;  // relative orthogonality |a_p·a_q| / (|a_p||a_q|)

template <typename T>
__device__ __forceinline__ const T* pool_block(const T* K, const T* V, int p, int b, int64_t T_, int n,
                                               int D) {
  const T* X = (p & 1) ? V : K;
  return X + ((int64_t)(p >> 1) * T_ + (int64_t)b * n) * D;
}

// ---------------------------------------------------------------- gram
template <typename T, int D>
__global__ void __launch_bounds__(kThreads) gram_kernel(const T* __restrict__ K, const T* __restrict__ V,
                                                       int64_t T_, int n, int nb, float* __restrict__ gram) {
  constexpr int CH = 32;
  constexpr int MT = D / 16;
  __shared__ float xs[CH][D];
  const int b = blockIdx.x, p = blockIdx.y;
  const T* X = pool_block(K, V, p, b, T_, n, D);
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  float acc[MT][MT];
#pragma unroll
  for (int i = 0; i < MT; ++i)
#pragma unroll
    for (int j = 0; j < MT; ++j) acc[i][j] = 0.f;
  for (int t0 = 0; t0 < n; t0 += CH) {
    __syncthreads();
    for (int e = threadIdx.x; e < CH * D; e += kThreads)
      xs[e / D][e % D] = to_f32(X[(int64_t)(t0 + e / D) * D + (e % D)]);
    __syncthreads();
#pragma unroll 4
    for (int k = 0; k < CH; ++k) {
      float a[MT], c[MT];
#pragma unroll
      for (int i = 0; i < MT; ++i) a[i] = xs[k][ty + 16 * i];
#pragma unroll
      for (int j = 0; j < MT; ++j) c[j] = xs[k][tx + 16 * j];
#pragma unroll
      for (int i = 0; i < MT; ++i)
#pragma unroll
        for (int j = 0; j < MT; ++j) acc[i][j] = fmaf(a[i], c[j], acc[i][j]);
    }
  }
  float* G = gram + ((int64_t)p * nb + b) * D * D;
#pragma unroll
  for (int i = 0; i < MT; ++i)
#pragma unroll
    for (int j = 0; j < MT; ++j) G[(ty + 16 * i) * D + tx + 16 * j] = acc[i][j];
}

// ---------------------------------------------------------------- jacobi
// Round-robin (circle method) pairing: round s in [0, D-1), pair k in [0, D/2).
__device__ __forceinline__ void rr_pair(int D, int s, int k, int& p, int& q) {
  const int m = D - 1;
  if (k == 0) {
    p = s;
    q = m;
  } else {
    p = (s + k) % m;
    q = (s - k + m) % m;
  }
}

template <int D>
__global__ void __launch_bounds__(kJThreads) jacobi_kernel(const float* __restrict__ gram, int nb, int max_sweeps,
                                                         float* __restrict__ eigvals, float* __restrict__ eigvecs,
                                                         uint32_t* status) {
  constexpr int E = D / 32;  // elements per lane of one column
  extern __shared__ float smem[];
  float* A = smem;          // column-major: column j at A[j*D]
  float* W = smem + D * D;  // accumulated rotations, column-major
  float* lam = W + D * D;   // D
  const int blk = blockIdx.x + blockIdx.y * nb;
  const float* G = gram + (int64_t)blk * D * D;
  for (int e = threadIdx.x; e < D * D; e += kJThreads) {
    A[e] = G[e];  // G symmetric: row-major == column-major
    W[e] = (e / D == e % D) ? 1.f : 0.f;
  }
  __syncthreads();
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  constexpr int NW = kJThreads / 32;
  constexpr int PP = (D / 2) / NW;  // column pairs per warp per round
  bool converged = false;
  for (int sweep = 0; sweep < max_sweeps; ++sweep) {
    int rotated = 0;
    for (int s = 0; s < D - 1; ++s) {
      // the warp's PP pairs are handled together so that their loads and reductions overlap
      float ap[PP][E], aq[PP][E], al[PP], be[PP], ga[PP];
      int pj[PP], qj[PP];
#pragma unroll
      for (int t = 0; t < PP; ++t) {
        rr_pair(D, s, warp + t * NW, pj[t], qj[t]);
        al[t] = be[t] = ga[t] = 0.f;
#pragma unroll
        for (int e = 0; e < E; ++e) {
          ap[t][e] = A[pj[t] * D + lane + 32 * e];
          aq[t][e] = A[qj[t] * D + lane + 32 * e];
          al[t] = fmaf(ap[t][e], ap[t][e], al[t]);
          be[t] = fmaf(aq[t][e], aq[t][e], be[t]);
          ga[t] = fmaf(ap[t][e], aq[t][e], ga[t]);
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1)
#pragma unroll
        for (int t = 0; t < PP; ++t) {
          al[t] += __shfl_xor_sync(0xffffffffu, al[t], o);
          be[t] += __shfl_xor_sync(0xffffffffu, be[t], o);
          ga[t] += __shfl_xor_sync(0xffffffffu, ga[t], o);
        }
#pragma unroll
      for (int t = 0; t < PP; ++t) {
        if (ga[t] != 0.f && fabsf(ga[t]) > kJacobiTol * sqrtf(al[t]) * sqrtf(be[t])) {
          const float zeta = (be[t] - al[t]) / (2.f * ga[t]);
          const float tn = (zeta >= 0.f ? 1.f : -1.f) / (fabsf(zeta) + sqrtf(1.f + zeta * zeta));
          const float c = 1.f / sqrtf(1.f + tn * tn);
          const float sn = c * tn;
          const int p = pj[t], q = qj[t];
#pragma unroll
          for (int e = 0; e < E; ++e) {
            A[p * D + lane + 32 * e] = c * ap[t][e] - sn * aq[t][e];
            A[q * D + lane + 32 * e] = sn * ap[t][e] + c * aq[t][e];
            const float wp = W[p * D + lane + 32 * e], wq = W[q * D + lane + 32 * e];
            W[p * D + lane + 32 * e] = c * wp - sn * wq;
            W[q * D + lane + 32 * e] = sn * wp + c * wq;
          }
          rotated = 1;
        }
      }
      __syncthreads();
    }
    if (!__syncthreads_or(rotated)) {
      converged = true;
      break;
    }
  }
  if (!converged && threadIdx.x == 0) atomicOr(status, kStatusNoConvergence);
  // eigenvalue of column j = |G w_j| = norm of A's column j
  for (int j = warp; j < D; j += kJThreads / 32) {
    float ss = 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const float v = A[j * D + lane + 32 * e];
      ss = fmaf(v, v, ss);
    }
    ss = warp_sum(ss);
    if (lane == 0) lam[j] = sqrtf(ss);
  }
  __syncthreads();
  // sort descending by counting (ties: lower column first)
  for (int j = warp; j < D; j += kJThreads / 32) {
    const float lj = lam[j];
    int rank = 0;
    for (int i = lane; i < D; i += 32) rank += (lam[i] > lj) || (lam[i] == lj && i < j);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) rank += __shfl_xor_sync(0xffffffffu, rank, o);
    if (lane == 0) eigvals[(int64_t)blk * D + rank] = lj;
    float* dst = eigvecs + ((int64_t)blk * D + rank) * D;
#pragma unroll
    for (int e = 0; e < E; ++e) dst[lane + 32 * e] = W[j * D + lane + 32 * e];
  }
}

// ---------------------------------------------------------------- alloc
__device__ __forceinline__ double clampd(double x, double lo, double hi) { return fmin(fmax(x, lo), hi); }

__global__ void __launch_bounds__(kThreads) alloc_kernel(const float* __restrict__ eigvals, int nb, int D, int R,
                                                        int r_min, int pool_rows, double* __restrict__ entropy,
                                                        double* __restrict__ quotas, int32_t* __restrict__ ranks,
                                                        int64_t* __restrict__ row_offsets) {
  extern __shared__ double sh[];
  double* w = sh;             // nb
  double* q = w + nb;         // nb
  double* frac = q + nb;      // nb
  int* fl = (int*)(frac + nb);  // nb
  __shared__ double s_lam;
  __shared__ int s_rem;
  const int p = blockIdx.x;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  // entropy and weights
  for (int b = warp; b < nb; b += kThreads / 32) {
    const float* lam = eigvals + ((int64_t)p * nb + b) * D;
    double tot = 0.0;
    for (int i = lane; i < D; i += 32) tot += fmax((double)lam[i], 0.0);
    tot = warp_sum(tot);
    double h = 0.0;
    if (tot > 0.0) {
      for (int i = lane; i < D; i += 32) {
        const double pi = fmax((double)lam[i], 0.0) / tot;
        if (pi > 0.0) h -= pi * log(pi);
      }
      h = warp_sum(h);
    }
    if (lane == 0) {
      entropy[(int64_t)p * nb + b] = h;
      w[b] = exp(h);
    }
  }
  __syncthreads();
  const bool full = (int64_t)R >= (int64_t)nb * D;
  if (full) {
    for (int b = threadIdx.x; b < nb; b += kThreads) {
      q[b] = D;
      fl[b] = D;
      frac[b] = 0.0;
    }
    if (threadIdx.x == 0) s_rem = 0;
    __syncthreads();
  } else {
    // water level: smallest kink with sum >= R and largest kink with sum < R
    double lo = -1.0, hi = INFINITY;
    for (int k = threadIdx.x; k < 2 * nb; k += kThreads) {
      const double kink = (k & 1 ? (double)D : (double)r_min) / w[k >> 1];
      double f = 0.0;
      for (int b = 0; b < nb; ++b) f += clampd(kink * w[b], r_min, D);
      if (f >= (double)R) hi = fmin(hi, kink);
      else lo = fmax(lo, kink);
    }
    // block min / max
    for (int o = 16; o > 0; o >>= 1) {
      hi = fmin(hi, __shfl_xor_sync(0xffffffffu, hi, o));
      lo = fmax(lo, __shfl_xor_sync(0xffffffffu, lo, o));
    }
    __shared__ double red_lo[kThreads / 32], red_hi[kThreads / 32];
    if (lane == 0) {
      red_lo[warp] = lo;
      red_hi[warp] = hi;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      double L = -1.0, Hh = INFINITY;
      for (int i = 0; i < kThreads / 32; ++i) {
        L = fmax(L, red_lo[i]);
        Hh = fmin(Hh, red_hi[i]);
      }
      double fh = 0.0;
      for (int b = 0; b < nb; ++b) fh += clampd(Hh * w[b], r_min, D);
      double lam;
      if (fh == (double)R) {
        lam = Hh;
      } else {
        const double mid = 0.5 * (L + Hh);
        double fixed = 0.0, W = 0.0;
        for (int b = 0; b < nb; ++b) {
          const double x = mid * w[b];
          if (x <= r_min) fixed += r_min;
          else if (x >= D) fixed += D;
          else W += w[b];
        }
        lam = ((double)R - fixed) / W;
      }
      s_lam = lam;
    }
    __syncthreads();
    const double lam = s_lam;
    int partial = 0;
    for (int b = threadIdx.x; b < nb; b += kThreads) {
      const double qb = clampd(lam * w[b], r_min, D);
      const double f = floor(qb);
      q[b] = qb;
      fl[b] = (int)f;
      frac[b] = qb - f;
      partial += (int)f;
    }
    for (int o = 16; o > 0; o >>= 1) partial += __shfl_xor_sync(0xffffffffu, partial, o);
    __shared__ int red_i[kThreads / 32];
    if (lane == 0) red_i[warp] = partial;
    __syncthreads();
    if (threadIdx.x == 0) {
      int tot = 0;
      for (int i = 0; i < kThreads / 32; ++i) tot += red_i[i];
      s_rem = R - tot;
    }
    __syncthreads();
  }
  const int rem = s_rem;
  for (int b = threadIdx.x; b < nb; b += kThreads) {
    int rank = 0;
    const double fb = frac[b];
    for (int c = 0; c < nb; ++c) rank += (frac[c] > fb) || (frac[c] == fb && c < b);
    const int r = fl[b] + (rank < rem ? 1 : 0);
    ranks[(int64_t)p * nb + b] = r;
    quotas[(int64_t)p * nb + b] = q[b];
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int64_t off = (int64_t)p * pool_rows;
    int64_t* ro = row_offsets + (int64_t)p * (nb + 1);
    for (int b = 0; b < nb; ++b) {
      ro[b] = off;
      off += ranks[(int64_t)p * nb + b];
    }
    ro[nb] = off;
  }
}

// ---------------------------------------------------------------- project
template <typename T, int D>
__global__ void __launch_bounds__(kThreads) project_kernel(const T* __restrict__ K, const T* __restrict__ V,
                                                          int64_t T_, int n, int nb,
                                                          const float* __restrict__ eigvecs,
                                                          const int32_t* __restrict__ ranks,
                                                          const int64_t* __restrict__ row_offsets,
                                                          T* __restrict__ tok, T* __restrict__ dim,
                                                          uint32_t* status) {
  constexpr int CH = 64;
  extern __shared__ float sm[];
  float* Bs = sm;            // [D][D] rows = eigenvectors
  float* xt = sm + D * D;    // [D][CH] transposed token chunk
  const int b = blockIdx.x, p = blockIdx.y;
  const int r = ranks[(int64_t)p * nb + b];
  const int64_t row0 = row_offsets[(int64_t)p * (nb + 1) + b];
  if (r < 0 || r > D) {
    if (threadIdx.x == 0) atomicOr(status, kStatusCompressBounds);
    return;
  }
  const float* ev = eigvecs + ((int64_t)p * nb + b) * D * D;
  for (int e = threadIdx.x; e < r * D; e += kThreads) {
    const float v = ev[e];
    Bs[e] = v;
    dim[(row0 + e / D) * D + (e % D)] = from_f32<T>(v);
  }
  const T* X = pool_block(K, V, p, b, T_, n, D);
  const int tt = threadIdx.x % CH, j0 = threadIdx.x / CH;
  constexpr int JS = kThreads / CH;
  for (int t0 = 0; t0 < n; t0 += CH) {
    __syncthreads();
    for (int e = threadIdx.x; e < CH * D; e += kThreads) {
      const int t = e / D, c = e % D;
      xt[c * CH + t] = to_f32(X[(int64_t)(t0 + t) * D + c]);
    }
    __syncthreads();
    for (int j = j0; j < r; j += JS) {
      float acc = 0.f;
#pragma unroll 8
      for (int c = 0; c < D; ++c) acc = fmaf(xt[c * CH + tt], Bs[j * D + c], acc);
      const int t = t0 + tt;  // chunk-major: [t / 128][j][t % 128] inside the block's slab
      tok[row0 * n + (int64_t)(t >> 7) * (r * 128) + j * 128 + (t & 127)] = from_f32<T>(acc);
    }
  }
}

template <typename T, int D>
cudaError_t run(const CompressShape& s, const CompressBuffers& bf, cudaStream_t st) {
  const T* K = static_cast<const T*>(bf.K);
  const T* V = static_cast<const T*>(bf.V);
  dim3 grid(s.nb, 2 * s.H);
  // bf16 blocks: Gram on the tensor cores (gram_tc.cu); fp32 blocks: on the CUDA cores
  const cudaError_t ge = launch_gram_tc(s, K, V, bf.gram, bf.status, st);
  if (ge == cudaErrorNotSupported) {
    cudaGetLastError();
    gram_kernel<T, D><<<grid, kThreads, 0, st>>>(K, V, s.T, s.n, s.nb, bf.gram);
  } else if (ge != cudaSuccess) {
    return ge;
  }
  const size_t jsm = (2 * D * D + D) * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(jacobi_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)jsm);
  if (e != cudaSuccess) return e;
  jacobi_kernel<D><<<grid, kJThreads, jsm, st>>>(bf.gram, s.nb, s.max_sweeps, bf.eigvals, bf.eigvecs, bf.status);
  const size_t asm_ = (size_t)s.nb * (3 * sizeof(double) + sizeof(int));
  e = cudaFuncSetAttribute(alloc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)asm_);
  if (e != cudaSuccess) return e;
  alloc_kernel<<<2 * s.H, kThreads, asm_, st>>>(bf.eigvals, s.nb, D, s.R, s.r_min, s.pool_rows, bf.entropy,
                                                 bf.quotas, bf.ranks, bf.row_offsets);
  const size_t psm = (D * D + D * 64) * sizeof(float);
  e = cudaFuncSetAttribute(project_kernel<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)psm);
  if (e != cudaSuccess) return e;
  project_kernel<T, D><<<grid, kThreads, psm, st>>>(K, V, s.T, s.n, s.nb, bf.eigvecs, bf.ranks, bf.row_offsets,
                                                    static_cast<T*>(bf.tok), static_cast<T*>(bf.dim), bf.status);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_compress(const CompressShape& s, const CompressBuffers& b, cudaStream_t st) {
  if (s.bf16) {
    if (s.d == 64) return run<__nv_bfloat16, 64>(s, b, st);
    return run<__nv_bfloat16, 128>(s, b, st);
  }
  if (s.d == 64) return run<float, 64>(s, b, st);
  return run<float, 128>(s, b, st);
}

}  // namespace milo
