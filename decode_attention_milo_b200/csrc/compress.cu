// Block-wise low-rank compression (encode side of MILO).
//
// Page "MILO: Efficient Many-shot In-Context Learning with Block-wise Low-rank
// Compression": §4.2 splits each KV pool into blocks and approximates each
// block's keys and values separately at low rank; §4.3 sets each block's rank
// from its entropy under a fixed total budget.  Four kernels per layer, all on
// the caller's stream:
//   gram     G_b = X_bᵀ X_b in fp32  (bf16 blocks: tensor cores, gram_tc.cu; fp32: here, one CTA per block)
//   eig      pivoted Cholesky of G_b, then one-sided Jacobi on the columns of its factor: eigenvalues
//            λ_i = σ_i², eigenvectors B_b, sorted descending      (one CTA per block)
//   alloc    H_b = −Σ p ln p (p = λ/Σλ, fp64), w_b = e^{H_b}, quotas
//            clamp(lam·w_b, r_min, d) with Σ = R, largest-remainder ranks,
//            row offsets                                  (one CTA per pool)
//   project  U_b = X_b · B_b[:, :r_b], stored transposed in 128-token slabs, and B_bᵀ rows
//            (bf16 blocks: tensor cores, project_tc.cu; fp32: here, one CTA per block)
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace milo {
namespace {

constexpr int kThreads = 256;
constexpr float kJacobiTol = 1e-5f;  // relative orthogonality |a_p·a_q| / (|a_p||a_q|)
// A sweep whose largest relative off-diagonal stays below this ends the iteration: cyclic Jacobi converges
// quadratically, so what remains after it is of order 1e-7, below kJacobiTol, and the next sweep would
// rotate nothing.
constexpr float kJacobiExit = 3e-4f;

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

// ---------------------------------------------------------------- eigen-decomposition
// Eigen-decomposition of G_b by one-sided Jacobi preconditioned with a pivoted Cholesky factor
// (the preconditioning of Demmel–Veselić and Drmač for Jacobi SVD): G = L̃ L̃ᵀ with L̃ the Cholesky
// factor under diagonal pivoting, its rows kept in the original index order; then one-sided Jacobi
// orthogonalises the columns of L̃, L̃·U = B·Σ, so that G = (L̃U)(L̃U)ᵀ = B Σ² Bᵀ: the eigenvalues are the
// squared column norms and the eigenvectors the normalised columns, already in the original order.
// The rows of the pivoted factor are graded and nearly orthogonal, so the sweeps are few, and no
// accumulated rotation matrix is needed (the columns themselves become the eigenvectors).  Pivots below a
// floor far under fp32 resolution (1e-9 of the mean diagonal) are raised to it, so that a rank-deficient
// block still yields an orthonormal basis.
constexpr int kEThreads = 256;

template <int D>
__global__ void __launch_bounds__(kEThreads, 3) eig_kernel(const float* __restrict__ gram, int nb, int max_sweeps,
                                                       float* __restrict__ eigvals, float* __restrict__ eigvecs,
                                                       int32_t* __restrict__ sweeps_out, uint32_t* status) {
  constexpr int E = D / 32;           // elements per lane of one column
  constexpr int NW = kEThreads / 32;  // warps
  constexpr int PP = (D / 2) / NW;    // column pairs per warp per round
  extern __shared__ float smem[];
  float* A = smem;              // column-major [D][D]: the Schur complement, then the columns of L̃
  float* nrm = A + D * D;       // [D] squared column norms during the sweeps
  int* done = reinterpret_cast<int*>(nrm + D);  // [D] index already pivoted
  __shared__ float s_floor;
  __shared__ int s_piv;
  const int bidx = blockIdx.x + blockIdx.y * nb;
  const float* Gg = gram + (int64_t)bidx * D * D;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  for (int e = threadIdx.x; e < D * D; e += kEThreads) A[e] = Gg[e];
  for (int i = threadIdx.x; i < D; i += kEThreads) done[i] = 0;
  __syncthreads();
  if (warp == 0) {
    float tr = 0.f;
    for (int i = lane; i < D; i += 32) tr += fmaxf(A[i * D + i], 0.f);
    tr = warp_sum(tr);
    if (lane == 0) s_floor = fmaxf(1e-9f * tr / D, 1e-30f);
  }
  // ---- pivoted Cholesky, in place
  for (int k = 0; k < D; ++k) {
    if (warp == 0) {
      float best = -INFINITY;
      int bi = 0;
      for (int i = lane; i < D; i += 32) {
        const float v = done[i] ? -INFINITY : A[i * D + i];
        if (v > best) {
          best = v;
          bi = i;
        }
      }
      for (int o = 16; o > 0; o >>= 1) {
        const float ob = __shfl_xor_sync(0xffffffffu, best, o);
        const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
        if (ob > best || (ob == best && oi < bi)) {
          best = ob;
          bi = oi;
        }
      }
      if (lane == 0) s_piv = bi;
    }
    __syncthreads();
    const int p = s_piv;
    const float piv = fmaxf(A[p * D + p], s_floor);
    const float l = sqrtf(piv), il = 1.f / l;
    __syncthreads();  // every thread has read the pivot before column p changes
    // column p becomes column k of L̃: remaining rows scaled, the pivot row l, eliminated rows 0
    for (int i = threadIdx.x; i < D; i += kEThreads) {
      float* a = &A[p * D + i];
      *a = i == p ? l : (done[i] ? 0.f : *a * il);
    }
    __syncthreads();
    if (threadIdx.x == 0) done[p] = 1;
    // Schur complement of the remaining indices: A[i][j] -= L̃[i][k] L̃[j][k].  A thread keeps one row i
    // (A[j·D + i] is row i of column j) and walks the columns j ≡ tid / D (mod kEThreads / D); eliminated rows
    // and columns hold 0 in column p and are skipped (a column skip is uniform across the warp)
    {
      const int i = threadIdx.x % D;
      const float li = A[p * D + i];
      if (i != p && li != 0.f) {
        for (int j = threadIdx.x / D; j < D; j += kEThreads / D) {
          const float lj = A[p * D + j];
          if (j != p && lj != 0.f) A[j * D + i] = fmaf(-li, lj, A[j * D + i]);
        }
      }
    }
    __syncthreads();
  }
  // every column has now been pivoted: the columns of A are the columns of L̃ (in pivot order)
  // ---- one-sided Jacobi on the columns of L̃ (round-robin pairs), norms carried along.
  // Eight lanes take one pair, so a warp works on four pairs at once: lane l of group g = lane / 8 holds
  // the float4 at elements 32e + 4l .. + 3 (e < d/32) of both columns of the group's pair.  The dot product
  // then reduces over three shuffle levels, and each scalar step of the rotation serves four pairs.
  for (int j = warp; j < D; j += NW) {
    float ss = 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) ss = fmaf(A[j * D + lane + 32 * e], A[j * D + lane + 32 * e], ss);
    ss = warp_sum(ss);
    if (lane == 0) nrm[j] = ss;
  }
  __syncthreads();  // a pair reads norms that other warps wrote
  constexpr int IT = PP / 4;  // groups of four pairs per warp per round
  constexpr float kTol2 = kJacobiTol * kJacobiTol, kExit2 = kJacobiExit * kJacobiExit;
  const int g = lane / 8, lq = lane % 8;
  const unsigned gmask = 0xffu << (8 * g);
  float4* A4 = reinterpret_cast<float4*>(A);
  bool converged = false;
  int sweeps_run = 0;
  for (int sweep = 0; sweep < max_sweeps; ++sweep) {
    ++sweeps_run;
    int rotated = 0, big = 0;  // big: some relative off-diagonal of this sweep reached kJacobiExit
    for (int s = 0; s < D - 1; ++s) {
#pragma unroll 1
      for (int it = 0; it < IT; ++it) {
        // round-robin pair k of round s without a division: (s, D-1) for k = 0, else (s+k, s-k) mod D-1
        const int k = warp + (4 * it + g) * NW, m = D - 1;
        int pp = s + k, qq = s - k;
        if (pp >= m) pp -= m;
        if (qq < 0) qq += m;
        const int p = k == 0 ? s : pp, q = k == 0 ? m : qq;
        float4 ap[E], aq[E];
        float gx[E];  // one partial dot product per float4, so that the FMA chains are short
#pragma unroll
        for (int e = 0; e < E; ++e) {
          ap[e] = A4[p * (D / 4) + 8 * e + lq];
          aq[e] = A4[q * (D / 4) + 8 * e + lq];
          gx[e] = fmaf(ap[e].w, aq[e].w, fmaf(ap[e].z, aq[e].z, fmaf(ap[e].y, aq[e].y, ap[e].x * aq[e].x)));
        }
#pragma unroll
        for (int w = 1; w < E; w *= 2)
#pragma unroll
          for (int e = 0; e + w < E; e += 2 * w) gx[e] += gx[e + w];
        float ga = gx[0];
        // the butterfly leaves the same sum in all eight lanes, so the group takes one branch below
#pragma unroll
        for (int o = 4; o > 0; o >>= 1) ga += __shfl_xor_sync(0xffffffffu, ga, o);
        const float al = nrm[p], be = nrm[q], ag2 = ga * ga;
        big |= ga != 0.f && ag2 >= kExit2 * al * be;
        if (ga != 0.f && ag2 > kTol2 * al * be) {
          // tan θ = sign(ζ) / (|ζ| + sqrt(1 + ζ²)), ζ = (β − α) / 2γ; cos θ from the hardware reciprocal square
          // root with one Newton–Raphson step (y ← y·(1.5 − 0.5·x·y²)), so that cos² + sin² = 1 to fp32
          // rounding; the angle itself needs no more than approximate divisions
          const float zeta = __fdividef(be - al, 2.f * ga);
          const float z2 = fmaf(zeta, zeta, 1.f);
          const float tn = copysignf(__fdividef(1.f, fabsf(zeta) + z2 * rsqrtf(z2)), zeta);
          const float x = fmaf(tn, tn, 1.f);
          float c = rsqrtf(x);
          c = c * fmaf(-0.5f * x * c, c, 1.5f);
          const float sn = c * tn, tau = __fdividef(sn, 1.f + c);
          // the rotation written as a correction of each column (a_p − s(a_q + τa_p), a_q + s(a_p − τa_q),
          // τ = s / (1 + c)): its rounding scales with the correction, not with the column, so that the many
          // small late rotations do not drift the column norms (the eigenvalues)
#pragma unroll
          for (int e = 0; e < E; ++e) {
            const float4 u = ap[e], v = aq[e];
            A4[p * (D / 4) + 8 * e + lq] = make_float4(u.x - sn * fmaf(tau, u.x, v.x), u.y - sn * fmaf(tau, u.y, v.y),
                                                      u.z - sn * fmaf(tau, u.z, v.z), u.w - sn * fmaf(tau, u.w, v.w));
            A4[q * (D / 4) + 8 * e + lq] = make_float4(v.x + sn * fmaf(-tau, v.x, u.x), v.y + sn * fmaf(-tau, v.y, u.y),
                                                      v.z + sn * fmaf(-tau, v.z, u.z), v.w + sn * fmaf(-tau, v.w, u.w));
          }
          __syncwarp(gmask);  // every lane of the group has read nrm[p], nrm[q]
          if (lq == 0) {
            nrm[p] = al - tn * ga;
            nrm[q] = be + tn * ga;
          }
          rotated = 1;
        }
      }
      __syncthreads();
    }
    // exact norms again (the carried ones drift by rounding)
    for (int j = warp; j < D; j += NW) {
      float ss = 0.f;
#pragma unroll
      for (int e = 0; e < E; ++e) ss = fmaf(A[j * D + lane + 32 * e], A[j * D + lane + 32 * e], ss);
      ss = warp_sum(ss);
      if (lane == 0) nrm[j] = ss;
    }
    const int any_rotated = __syncthreads_or(rotated), any_big = __syncthreads_or(big);
    if (!any_rotated || !any_big) {
      converged = true;
      break;
    }
  }
  if (!converged && threadIdx.x == 0) atomicOr(status, kStatusNoConvergence);
  if (threadIdx.x == 0) sweeps_out[bidx] = sweeps_run;
  // eigenvalue λ_j = |column j|², eigenvector = column j / |column j|; sorted descending (ties: lower column)
  for (int j = warp; j < D; j += NW) {
    const float lj = nrm[j];
    int rank = 0;
    for (int i = lane; i < D; i += 32) rank += (nrm[i] > lj) || (nrm[i] == lj && i < j);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) rank += __shfl_xor_sync(0xffffffffu, rank, o);
    if (lane == 0) eigvals[(int64_t)bidx * D + rank] = lj;
    const float inv = lj > 0.f ? rsqrtf(lj) : 0.f;
    float* dst = eigvecs + ((int64_t)bidx * D + rank) * D;
#pragma unroll
    for (int e = 0; e < E; ++e) dst[lane + 32 * e] = A[j * D + lane + 32 * e] * inv;
  }
}

// ---------------------------------------------------------------- alloc
__device__ __forceinline__ double clampd(double x, double lo, double hi) { return fmin(fmax(x, lo), hi); }

constexpr int kAThreads = 512;

// Sum over the CTA of one value per thread (all threads call it; red holds kAThreads / 32 entries).
template <typename V>
__device__ V cta_sum(V v, V* red) {
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  __syncthreads();
  if ((threadIdx.x & 31) == 0) red[threadIdx.x / 32] = v;
  __syncthreads();
  V t = 0;
  for (int i = 0; i < kAThreads / 32; ++i) t += red[i];
  return t;
}

// Energy share of component i of a block, from its fp32 eigenvalues (negatives count as 0), in fp64.
__device__ __forceinline__ double share_of(const float* lam, int i, double tot) {
  return tot > 0.0 ? fmax((double)lam[i], 0.0) / tot : 0.0;
}

// Candidates of a block for the greedy rule with share >= t (as fp64 bit patterns: non-negative doubles order
// like their bits): components r_min .. D-1, whose shares do not increase, so a binary search counts them.
__device__ __forceinline__ int count_at_least(const float* lam, int D, int r_min, double tot, unsigned long long t) {
  int lo = r_min, hi = D;  // the answer is the first i in [r_min, D] with share(i) < t, minus r_min
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if ((unsigned long long)__double_as_longlong(share_of(lam, mid, tot)) >= t) lo = mid + 1;
    else hi = mid;
  }
  return lo - r_min;
}

// Rank allocation over one group of N consecutive blocks [g0, g0 + N) of the [2H][nb] block order: a pool
// (one CTA per pool) or the whole layer (one CTA).  Rules (§4.3 and the §5.3 baselines):
//   0 entropy  H_b = −Σ p ln p (p = λ/Σλ, fp64), w_b = e^{H_b}, quotas clamp(lam·w_b, r_min, d) with Σ = R,
//              largest-remainder rounding (ties to the lower index)
//   1 greedy   every block starts at r_min; the R − N·r_min free units go to the largest next-component
//              energy shares λ_i/Σλ (ties to the lower block index): the K largest candidates, found by
//              bisection on their fp64 bit patterns
//   2 uniform  floor(R / N) each, the remainder to the lowest indices
//   3 weights  caller weights (the random baseline's draws) with the entropy rule's water-filling
// Row offsets: pool groups start at p · pool_rows; a layer group's pools follow each other.
__global__ void __launch_bounds__(kAThreads) alloc_kernel(const float* __restrict__ eigvals, int P, int nb, int D,
                                                         int R, int r_min, int rule, bool layer, int pool_rows,
                                                         const double* __restrict__ user_w,
                                                         double* __restrict__ entropy, double* __restrict__ quotas,
                                                         int32_t* __restrict__ ranks,
                                                         int64_t* __restrict__ row_offsets) {
  extern __shared__ double sh[];
  const int N = layer ? P * nb : nb;
  const int g0 = layer ? 0 : blockIdx.x * nb;
  double* w = sh;             // N: weights (water-filling rules) or Σλ (greedy)
  double* q = w + N;          // N: quotas
  int* fl = (int*)(q + N);    // N: integer part of the rank
  __shared__ double s_lam;
  __shared__ int s_rem;
  __shared__ double red_d[kAThreads / 32];
  __shared__ long long red_l[kAThreads / 32];
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  // entropy (always, it is an intermediate) and the rule's per-block weight
  for (int i = warp; i < N; i += kAThreads / 32) {
    const float* lam = eigvals + (int64_t)(g0 + i) * D;
    double tot = 0.0;
    for (int k = lane; k < D; k += 32) tot += fmax((double)lam[k], 0.0);
    tot = warp_sum(tot);
    double h = 0.0;
    if (tot > 0.0) {
      for (int k = lane; k < D; k += 32) {
        const double pi = fmax((double)lam[k], 0.0) / tot;
        if (pi > 0.0) h -= pi * log(pi);
      }
      h = warp_sum(h);
    }
    if (lane == 0) {
      entropy[g0 + i] = h;
      w[i] = rule == 0 ? exp(h) : rule == 3 ? user_w[g0 + i] : tot;
    }
  }
  __syncthreads();
  const bool full = (int64_t)R >= (int64_t)N * D;
  const double nan = __longlong_as_double(0x7ff8000000000000LL);
  if (full || rule == 2) {
    for (int i = threadIdx.x; i < N; i += kAThreads) {
      const int r = full ? D : R / N + (i < R % N ? 1 : 0);
      q[i] = full ? (double)D : nan;
      fl[i] = r;
    }
  } else if (rule == 1) {
    // K-th largest candidate share: the largest bit pattern t with count(share >= t) >= K
    const long long K = (long long)R - (long long)N * r_min;
    unsigned long long lo = 0, hi = (unsigned long long)__double_as_longlong(1.0) + 1;  // count(lo) >= K > count(hi)
    if (K > 0) {
      while (hi - lo > 1) {
        const unsigned long long mid = lo + (hi - lo) / 2;
        long long c = 0;
        for (int i = threadIdx.x; i < N; i += kAThreads)
          c += count_at_least(eigvals + (int64_t)(g0 + i) * D, D, r_min, w[i], mid);
        c = cta_sum<long long>(c, red_l);
        if (c >= K) lo = mid;
        else hi = mid;
      }
    }
    // blocks take every candidate above the cut; the units left at exactly the cut value go to the lowest blocks
    for (int i = threadIdx.x; i < N; i += kAThreads) {
      const float* lam = eigvals + (int64_t)(g0 + i) * D;
      const int ge = K > 0 ? count_at_least(lam, D, r_min, w[i], lo) : 0;
      const int gt = K > 0 ? count_at_least(lam, D, r_min, w[i], lo + 1) : 0;
      fl[i] = r_min + gt;
      q[i] = (double)(ge - gt);  // candidates at the cut value (reused below), quota NaN afterwards
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      long long m = K;
      for (int i = 0; i < N; ++i) m -= fl[i] - r_min;
      for (int i = 0; i < N; ++i) {
        const int take = (int)min((long long)q[i], max(m, 0LL));
        fl[i] += take;
        m -= take;
        q[i] = nan;
      }
    }
  } else {
    // water level: smallest kink with sum >= R and largest kink with sum < R
    double lo = -1.0, hi = INFINITY;
    for (int k = threadIdx.x; k < 2 * N; k += kAThreads) {
      const double kink = (k & 1 ? (double)D : (double)r_min) / w[k >> 1];
      double f = 0.0;
      for (int b = 0; b < N; ++b) f += clampd(kink * w[b], r_min, D);
      if (f >= (double)R) hi = fmin(hi, kink);
      else lo = fmax(lo, kink);
    }
    for (int o = 16; o > 0; o >>= 1) {
      hi = fmin(hi, __shfl_xor_sync(0xffffffffu, hi, o));
      lo = fmax(lo, __shfl_xor_sync(0xffffffffu, lo, o));
    }
    __shared__ double red_lo[kAThreads / 32], red_hi[kAThreads / 32];
    if (lane == 0) {
      red_lo[warp] = lo;
      red_hi[warp] = hi;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      double L = -1.0, Hh = INFINITY;
      for (int i = 0; i < kAThreads / 32; ++i) {
        L = fmax(L, red_lo[i]);
        Hh = fmin(Hh, red_hi[i]);
      }
      double fh = 0.0;
      for (int b = 0; b < N; ++b) fh += clampd(Hh * w[b], r_min, D);
      double lam;
      if (fh == (double)R) {
        lam = Hh;
      } else {
        const double mid = 0.5 * (L + Hh);
        double fixed = 0.0, W = 0.0;
        for (int b = 0; b < N; ++b) {
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
    for (int b = threadIdx.x; b < N; b += kAThreads) {
      const double qb = clampd(lam * w[b], r_min, D);
      const double f = floor(qb);
      q[b] = qb;
      fl[b] = (int)f;
      partial += (int)f;
    }
    const int tot = cta_sum<int>(partial, (int*)red_l);
    if (threadIdx.x == 0) s_rem = R - tot;
    __syncthreads();
    // largest remainder: the s_rem blocks with the largest fractional parts get one more (ties: lower index)
    const int rem = s_rem;
    for (int b = threadIdx.x; b < N; b += kAThreads) {
      int rank = 0;
      const double fb = q[b] - fl[b];
      for (int c = 0; c < N; ++c) {
        const double fc = q[c] - fl[c];
        rank += (fc > fb) || (fc == fb && c < b);
      }
      ranks[g0 + b] = fl[b] + (rank < rem ? 1 : 0);
    }
    __syncthreads();
    for (int b = threadIdx.x; b < N; b += kAThreads) fl[b] = ranks[g0 + b];
  }
  __syncthreads();
  for (int b = threadIdx.x; b < N; b += kAThreads) {
    ranks[g0 + b] = fl[b];
    quotas[g0 + b] = q[b];
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    // row offsets [P][nb + 1]: block b of pool p owns rows [ro[b], ro[b] + r); ro[nb] is the pool's end
    const int p0 = layer ? 0 : blockIdx.x, p1 = layer ? P : blockIdx.x + 1;
    int64_t off = layer ? 0 : (int64_t)blockIdx.x * pool_rows;
    for (int pp = p0; pp < p1; ++pp) {
      int64_t* ro = row_offsets + (int64_t)pp * (nb + 1);
      for (int b = 0; b < nb; ++b) {
        ro[b] = off;
        off += fl[(pp - p0) * nb + b];
      }
      ro[nb] = off;
    }
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
cudaError_t run(const CompressShape& s, const CompressBuffers& bf, cudaStream_t st, const cudaEvent_t* ev) {
  const T* K = static_cast<const T*>(bf.K);
  const T* V = static_cast<const T*>(bf.V);
  dim3 grid(s.nb, 2 * s.H);
  // ev[k] (optional) is recorded on `st` before kernel k (gram, jacobi, alloc, project) and ev[4] after the last
  auto mark = [&](int k) -> cudaError_t { return ev && ev[k] ? cudaEventRecord(ev[k], st) : cudaSuccess; };
  cudaError_t me;
  if ((me = mark(0)) != cudaSuccess) return me;
  // bf16 blocks: Gram on the tensor cores (gram_tc.cu); fp32 blocks: on the CUDA cores
  const cudaError_t ge = launch_gram_tc(s, K, V, bf.gram, bf.status, st);
  if (ge == cudaErrorNotSupported) {
    cudaGetLastError();
    gram_kernel<T, D><<<grid, kThreads, 0, st>>>(K, V, s.T, s.n, s.nb, bf.gram);
  } else if (ge != cudaSuccess) {
    return ge;
  }
  const size_t jsm = (size_t)D * D * sizeof(float) + D * (sizeof(float) + sizeof(int));
  cudaError_t e = cudaFuncSetAttribute(eig_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)jsm);
  if (e != cudaSuccess) return e;
  if ((e = mark(1)) != cudaSuccess) return e;
  eig_kernel<D><<<grid, kEThreads, jsm, st>>>(bf.gram, s.nb, s.max_sweeps, bf.eigvals, bf.eigvecs, bf.sweeps,
                                              bf.status);
  const int ngroup = s.layer_scope ? 2 * s.H * s.nb : s.nb;
  const size_t asm_ = (size_t)ngroup * (2 * sizeof(double) + sizeof(int));
  e = cudaFuncSetAttribute(alloc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)asm_);
  if (e != cudaSuccess) return e;
  if ((e = mark(2)) != cudaSuccess) return e;
  alloc_kernel<<<s.layer_scope ? 1 : 2 * s.H, kAThreads, asm_, st>>>(
      bf.eigvals, 2 * s.H, s.nb, D, s.R, s.r_min, s.rule, s.layer_scope, s.pool_rows, bf.weights, bf.entropy,
      bf.quotas, bf.ranks, bf.row_offsets);
  const size_t psm = (D * D + D * 64) * sizeof(float);
  e = cudaFuncSetAttribute(project_kernel<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)psm);
  if (e != cudaSuccess) return e;
  if ((e = mark(3)) != cudaSuccess) return e;
  // bf16 blocks: projection on the tensor cores (project_tc.cu); fp32 blocks: on the CUDA cores
  e = launch_project_tc(s, K, V, bf.eigvecs, bf.ranks, bf.row_offsets, bf.tok, bf.dim, bf.status, st);
  if (e == cudaErrorNotSupported) {
    cudaGetLastError();
    project_kernel<T, D><<<grid, kThreads, psm, st>>>(K, V, s.T, s.n, s.nb, bf.eigvecs, bf.ranks, bf.row_offsets,
                                                      static_cast<T*>(bf.tok), static_cast<T*>(bf.dim), bf.status);
  } else if (e != cudaSuccess) {
    return e;
  }
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  return mark(4);
}

}  // namespace

cudaError_t launch_compress(const CompressShape& s, const CompressBuffers& b, cudaStream_t st, const cudaEvent_t* ev) {
  if (s.bf16) {
    if (s.d == 64) return run<__nv_bfloat16, 64>(s, b, st, ev);
    return run<__nv_bfloat16, 128>(s, b, st, ev);
  }
  if (s.d == 64) return run<float, 64>(s, b, st, ev);
  return run<float, 128>(s, b, st, ev);
}

}  // namespace milo
