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
//
// One CTA of 256 threads per (KV head, block, 128-token chunk), three resident per SM:
//   - one thread loads the chunk's token-factor slab [r][128 tokens] and the block's dimension factor
//     [r][d] with one TMA box each (height r rounded up to 16; the rows past r are cleared in shared memory);
//   - the same thread issues K_chunk = U·Bᵀ as one tcgen05 MMA chain (M = 128 tokens, N = d, K = r, both
//     operands MN-major) into d TMEM columns;
//   - two threads then share TMEM lane t = one token, each half of its pairs (i, i + d/2): they rotate them
//     with the angle reduced in fp64 before the fp32 sine and cosine, and write the bf16 values into a
//     128-byte-swizzled tile in shared memory (the token-factor buffer, free once the MMA has completed);
//   - one TMA store writes the 128 × d tile to the output.
// Every wait is bounded (1 s): on expiry the kernel records kStatusDecodeTimeout, skips the rest, and gives the
// copies or MMAs it issued one more bounded wait before it frees TMEM and exits.
#include <cuda.h>
#include <cuda_bf16.h>

#include "common.cuh"
#include "rope.h"
#include "tc_ptx.cuh"

namespace milo {
namespace {

constexpr int kRThreads = 256;  // two threads per token in the epilogue, each half of the pairs
constexpr uint64_t kRWaitNs = 1000000000ull;
constexpr int kUBytes = 2 * 128 * 128;  // token-factor box [2 column blocks][≤ 128 rows][128 B], later the output tile
template <int D>
__host__ __device__ constexpr int dim_bytes() { return (D / 64) * 128 * 128; }  // dim-factor box [d/64 column blocks][≤ 128 rows][128 B]
template <int D>
constexpr size_t rope_smem() { return 1024 + kUBytes + dim_bytes<D>() + 64; }

// Warp-collective bounded wait on an mbarrier phase; false after kRWaitNs (the status flag is set).
__device__ __noinline__ bool rwait(uint32_t bar, uint32_t parity, uint32_t* status) {
  uint64_t t0 = 0;
  if ((threadIdx.x & 31) == 0) t0 = ptx::globaltimer();
  for (uint32_t i = 1;; ++i) {
    if (__all_sync(0xffffffffu, ptx::mbar_try_wait(bar, parity))) return true;
    if ((i & 63) == 0) {
      int late = 0;
      if ((threadIdx.x & 31) == 0) late = ptx::globaltimer() - t0 > kRWaitNs;
      if (__shfl_sync(0xffffffffu, late, 0)) {
        if ((threadIdx.x & 31) == 0) atomicOr(status, kStatusDecodeTimeout);
        return false;
      }
    }
  }
}

// MN-major SW128 descriptor of k-step k (16 rows) of a box [column block][rows][128 B], blocks `cbs` bytes apart.
__device__ __forceinline__ uint64_t mn_desc(uint32_t box, int k, uint32_t cbs) {
  return ptx::sw128_desc(box + (uint32_t)k * 2048u, cbs, 1024u);
}

// Writes 8 bf16 (4 packed words) at (row, col) of a 128-row tile [col / 64][128 rows][128 B], 128-byte swizzle
// (the layout a TMA box of 64 columns × 128 rows × column blocks has in shared memory).
__device__ __forceinline__ void st_out8(uint32_t tile, int row, int col, const uint32_t* w) {
  const uint32_t addr = tile + (uint32_t)(col >> 6) * 16384u + (uint32_t)row * 128u +
                        ((uint32_t)(((col & 63) >> 3) ^ (row & 7)) << 4);
  ptx::st_shared_v4(addr, w[0], w[1], w[2], w[3]);
}

template <int D>
__global__ void __launch_bounds__(kRThreads) rope_keys_kernel(const __grid_constant__ CUtensorMap kout,
                                                             const CUtensorMap* __restrict__ tok_maps,
                                                             const CUtensorMap* __restrict__ dim_maps,
                                                             const int32_t* __restrict__ ranks,
                                                             const int64_t* __restrict__ row_offsets, int nb, int n,
                                                             int64_t T, double log2_theta, uint32_t* status) {
  constexpr int P = D / 2;     // pairs per token
  constexpr int NCB = D / 64;  // 64-column blocks of a key row
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const uint32_t sU = ptx::smem_u32(smem), sB = sU + kUBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kUBytes + dim_bytes<D>());
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2);
  const uint32_t b_full = ptx::smem_u32(&bars[0]), b_done = ptx::smem_u32(&bars[1]);
  __shared__ double s_freq[P];  // θ^(−2i/d)
  const int warp = threadIdx.x / 32, t = threadIdx.x;
  const int tok = t & 127, half = t >> 7;  // epilogue: TMEM lane (token) and half of the pairs
  const int cpb = n / 128;
  const int c = blockIdx.x % cpb, b = (blockIdx.x / cpb) % nb, h = blockIdx.x / (cpb * nb);
  const int r = __ldg(ranks + (size_t)(2 * h) * nb + b);
  const int64_t row0 = __ldg(row_offsets + (size_t)(2 * h) * (nb + 1) + b);
  if (r < 1 || r > D) {
    if (t == 0) atomicOr(status, kStatusDecodeBounds);
    return;
  }
  const int rp = (r + 15) & ~15;  // box height
  if (t == 0) {
    ptx::mbar_init(b_full, 1);
    ptx::mbar_init(b_done, 1);
    ptx::fence_mbar_init();
  }
  if (warp == 0) {
    ptx::tmem_alloc(ptx::smem_u32(tmem_slot), D);
    ptx::tmem_relinquish();
  }
  for (int i = t; i < P; i += kRThreads) s_freq[i] = exp2(-2.0 * i / D * log2_theta);
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // ---- the chunk's slab rows row0·cpb + c·r + j and the block's dim rows row0 + j, j < rp
  if (t == 0) {
    const CUtensorMap* um = tok_maps + (rp / 16 - 1);
    const CUtensorMap* bm = dim_maps + (rp / 16 - 1);
    ptx::mbar_arrive_expect_tx(b_full, (uint32_t)rp * 256u + (uint32_t)(NCB * rp) * 128u);
    ptx::tma_load_3d(sU, um, b_full, 0, (int)(row0 * cpb + (int64_t)c * r), 0);
    if (D == 128) ptx::tma_load_3d(sB, bm, b_full, 0, (int)row0, 0);
    else ptx::tma_load_2d(sB, bm, b_full, 0, (int)row0);
  }
  bool ok = __syncthreads_and(rwait(b_full, 0, status));
  if (!ok) rwait(b_full, 0, status);  // after a timeout, one more bounded wait for the copies still in flight
  if (ok) {
    // rows r .. rp-1 of both boxes belong to the next chunk or block (or are past the array): clear them so
    // they add nothing (a whole 128-byte row stays in place under the swizzle)
    const int extra = rp - r, nu = 2 * extra * 8, nall = nu + NCB * extra * 8;
    for (int e = t; e < nall; e += kRThreads) {
      const bool in_u = e < nu;
      const int f = in_u ? e : e - nu, q = f >> 3;
      const uint32_t box = in_u ? sU : sB;
      ptx::st_shared_v4(box + (uint32_t)(q / extra) * (uint32_t)rp * 128u + (uint32_t)(r + q % extra) * 128u +
                            (uint32_t)(f & 7) * 16u,
                        0, 0, 0, 0);
    }
    ptx::fence_async_smem();
  }
  __syncthreads();
  // ---- K_chunk[t][i] = Σ_j U[j][t]·B[j][i]: M = 128 tokens, N = d, K = rp, A and B MN-major
  if (ok && t == 0) {
    ptx::tc_fence_after();
    constexpr uint32_t id = ptx::idesc_bf16(128, D, true, true);
    const uint32_t cbs = (uint32_t)rp * 128u;
    for (int k = 0; k < rp / 16; ++k) ptx::umma_bf16(tmem, mn_desc(sU, k, cbs), mn_desc(sB, k, cbs), id, k > 0);
    ptx::umma_commit(b_done);
  }
  const bool issued = ok;
  if (ok) ok = rwait(b_done, 0, status);
  ok = __syncthreads_and(ok);
  if (issued && !ok) rwait(b_done, 0, status);  // the same for MMAs still in flight, before TMEM is freed
  ptx::tc_fence_after();

  // ---- rotate token tok's pairs [half·d/4, half·d/4 + d/4) and stage them as bf16 (the U box is free: the MMA
  // has read it); warp w reads TMEM lanes 32·(w mod 4) .. + 31
  if (ok) {
    const uint32_t tl = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    const double pos = (double)((int64_t)b * n + (int64_t)c * 128 + tok);
    constexpr double kTwoPi = 6.283185307179586, kInvTwoPi = 0.15915494309189535;
#pragma unroll 1
    for (int i0 = half * (P / 2); i0 < (half + 1) * (P / 2); i0 += 16) {
      float x1[16], x2[16];
      ptx::tmem_ld16(tl + (uint32_t)i0, x1);
      ptx::tmem_ld16(tl + (uint32_t)(P + i0), x2);
      ptx::tmem_wait_ld();
      uint32_t w1[8], w2[8];
#pragma unroll
      for (int k = 0; k < 16; k += 2) {
        float y1[2], y2[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          // φ = pos·θ^(−2i/d) in fp64, reduced to about [−π, π] before the fp32 sine and cosine
          const double phi = pos * s_freq[i0 + k + u];
          const float red = (float)fma(-kTwoPi, rint(phi * kInvTwoPi), phi);
          float sn, cs;
          sincosf(red, &sn, &cs);
          y1[u] = x1[k + u] * cs - x2[k + u] * sn;
          y2[u] = x2[k + u] * cs + x1[k + u] * sn;
        }
        w1[k / 2] = ptx::pack_bf16(y1[0], y1[1]);
        w2[k / 2] = ptx::pack_bf16(y2[0], y2[1]);
      }
      st_out8(sU, tok, i0, w1);
      st_out8(sU, tok, i0 + 8, w1 + 4);
      st_out8(sU, tok, P + i0, w2);
      st_out8(sU, tok, P + i0 + 8, w2 + 4);
    }
    ptx::fence_async_smem();
  }
  __syncthreads();
  if (ok && t == 0) {
    // rows h·T + b·n + 128c .. + 127 of the output
    const int y = (int)((int64_t)h * T + (int64_t)b * n + (int64_t)c * 128);
    if (D == 128) ptx::tma_store_3d(&kout, sU, 0, y, 0);
    else ptx::tma_store_2d(&kout, sU, 0, y);
    ptx::bulk_commit();
    ptx::bulk_wait_all();
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 0) ptx::tmem_dealloc(tmem, D);
}

}  // namespace

cudaError_t launch_rope_keys(const RopeShape& s, const RopeBuffers& b, cudaStream_t st) {
  if ((s.d != 64 && s.d != 128) || s.n % 128 != 0 || s.H <= 0 || s.nb <= 0 || !(s.theta > 1.0) || !b.tok_maps ||
      !b.dim_maps || !b.keys_map)
    return cudaErrorInvalidValue;
  const int64_t grid = (int64_t)s.H * s.nb * (s.n / 128);
  const int64_t T = (int64_t)s.nb * s.n;
  if (grid > 0x7fffffff || s.H * T > 0x7fffffff) return cudaErrorInvalidValue;
  const double l2t = log2(s.theta);
  cudaError_t e;
  if (s.d == 64) {
    if ((e = cudaFuncSetAttribute(rope_keys_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)rope_smem<64>())) != cudaSuccess)
      return e;
    rope_keys_kernel<64><<<(unsigned)grid, kRThreads, rope_smem<64>(), st>>>(
        *b.keys_map, b.tok_maps, b.dim_maps, b.ranks, b.row_offsets, s.nb, s.n, T, l2t, b.status);
  } else {
    if ((e = cudaFuncSetAttribute(rope_keys_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)rope_smem<128>())) != cudaSuccess)
      return e;
    rope_keys_kernel<128><<<(unsigned)grid, kRThreads, rope_smem<128>(), st>>>(
        *b.keys_map, b.tok_maps, b.dim_maps, b.ranks, b.row_offsets, s.nb, s.n, T, l2t, b.status);
  }
  return cudaGetLastError();
}

}  // namespace milo
