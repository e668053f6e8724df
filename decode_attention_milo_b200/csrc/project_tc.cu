// Factor projection U_b = X_b · B_b[:, :r_b] on the sm_100a tensor cores (bf16 blocks).
//
// Page "MILO: Efficient Many-shot In-Context Learning with Block-wise Low-rank
// Compression", §4.2 and §4.4: each block's keys and values are stored as a
// low-rank pair; the token-side factor is the block projected on its leading
// right singular vectors, U_b = X_b · B_b (singular values folded in), and the
// dimension-side factor is B_b itself.
//
// The kernel computes the transpose, Uᵀ = B_rᵀ · X_bᵀ, one 128-token tile at a
// time, so that a TMEM lane holds one rank component and its columns are the
// tile's tokens: row j of the 128-token slab the decode reads is then one lane's
// 128 contiguous values.  One persistent CTA per SM walks blocks:
//  - warps 6..13 convert the fp32 eigenvectors (rows 0..r−1, rows r..127 zero)
//    to a bf16 pair hi + lo (B ≈ hi + lo to about 2^-17 relative), write them as
//    the K-major A operand (M = 128 rank rows, K = d) in shared memory with the
//    128-byte swizzle, into one of two buffers up to two blocks ahead of the
//    MMAs, and store hi as the block's dimension-side factor rows;
//  - warp 0 streams X_b through a 3-stage ring of 128-token tiles by TMA
//    (K-major B operand, N = 128 tokens);
//  - warp 1 issues tcgen05.mma kind::f16, hi and lo per k-step (bf16 products
//    are exact in fp32), into one of two 128-column TMEM accumulators;
//  - warps 2..5 read each finished accumulator (lane j = rank j) and store
//    lanes j < r as bf16 to the slab.
//
// Waits are bounded (1 s): on expiry the kernel records kStatusCompressTimeout
// and returns after its own copies and MMAs have landed.
#include <cudaTypedefs.h>

#include <algorithm>

#include "common.cuh"
#include "internal.h"
#include "tc_ptx.cuh"

namespace milo {
namespace {

constexpr int kPConvWarps = 8;  // warps 6..13: the eigenvector conversion
constexpr int kPThreads = 32 * (6 + kPConvWarps);  // warp 0 TMA, warp 1 MMA, warps 2..5 epilogue, then conversion
constexpr int kPStages = 3;
constexpr uint64_t kPWaitNs = 1000000000ull;

enum PBar { P_FULL = 0, P_EMPTY = P_FULL + kPStages, P_AREADY = P_EMPTY + kPStages, P_AFREE = P_AREADY + 2,
            P_TFULL = P_AFREE + 2, P_TEMPTY = P_TFULL + 2, P_DONE = P_TEMPTY + 2, P_COUNT };

// Warp-collective bounded wait; false after kPWaitNs (the status flag is set).
__device__ __noinline__ bool pwait(uint32_t bar, uint32_t parity, uint32_t* status) {
  uint64_t t0 = 0;
  if ((threadIdx.x & 31) == 0) t0 = ptx::globaltimer();
  for (uint32_t i = 1;; ++i) {
    if (__all_sync(0xffffffffu, ptx::mbar_try_wait(bar, parity))) return true;
    if ((i & 63) == 0) {
      int late = 0;
      if ((threadIdx.x & 31) == 0) late = ptx::globaltimer() - t0 > kPWaitNs;
      if (__shfl_sync(0xffffffffu, late, 0)) {
        if ((threadIdx.x & 31) == 0) atomicOr(status, kStatusCompressTimeout);
        return false;
      }
    }
  }
}

struct ProjMaps {
  CUtensorMap k, v;  // [rows][d] bf16: d = 128: 3D {64, rows, 2} box {64, 128, 2}; d = 64: 2D {64, rows} box {64, 128}
};

// K-major SW128 descriptor of k-step k (16 elements of d) of a 128-row tile whose 64-column blocks are 16 KB apart.
__device__ __forceinline__ uint64_t pdesc(uint32_t tile, int k) {
  return ptx::sw128_desc(tile + (uint32_t)(k >> 2) * 16384u + (uint32_t)(k & 3) * 32u, 16, 1024);
}

template <int D>
__global__ void __launch_bounds__(kPThreads) project_tc_kernel(const __grid_constant__ ProjMaps maps, int64_t T_,
                                                              int n, int nb, int nblocks,
                                                              const float* __restrict__ eigvecs,
                                                              const int32_t* __restrict__ ranks,
                                                              const int64_t* __restrict__ row_offsets,
                                                              __nv_bfloat16* __restrict__ tok,
                                                              __nv_bfloat16* __restrict__ dim,
                                                              uint32_t* __restrict__ status) {
  constexpr int NCB = D / 64;                     // 64-column blocks of d
  constexpr uint32_t kATile = 16384u * NCB;       // one 128-row bf16 operand tile
  constexpr uint32_t kStage = 16384u * NCB;       // 128 tokens × d bf16
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const uint32_t base = ptx::smem_u32(smem);
  // two A buffers (hi, lo each), then the X ring
  auto a_hi = [&](int ab) { return base + (uint32_t)(2 * ab) * kATile; };
  auto a_lo = [&](int ab) { return base + (uint32_t)(2 * ab + 1) * kATile; };
  const uint32_t ring = base + 4 * kATile;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + 4 * kATile + kPStages * kStage);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + P_COUNT);
  auto bar = [&](int i) { return ptx::smem_u32(&bars[i]); };
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  if (threadIdx.x == 0) {
    // an A operand gets one arrival from each conversion warp, an accumulator release one from each of the
    // four epilogue warps
    for (int i = 0; i < P_COUNT; ++i) {
      const bool conv = i == P_AREADY || i == P_AREADY + 1, epi = i == P_TEMPTY || i == P_TEMPTY + 1;
      ptx::mbar_init(bar(i), conv ? kPConvWarps : epi ? 4 : 1);
    }
    ptx::fence_mbar_init();
  }
  if (warp == 1) {
    ptx::tmem_alloc(ptx::smem_u32(tmem_slot), 256);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int tiles = n / 128;
  // the CTA's blocks: flat index u = blockIdx.x + k·gridDim.x over (pool p = u / nb, block b = u % nb)
  const int nmine = nblocks > (int)blockIdx.x ? (nblocks - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
  struct Blk {
    int p, b, r;
    int64_t row0;
  };
  auto blk = [&](int k) {
    Blk x;
    const int u = (int)blockIdx.x + k * (int)gridDim.x;
    x.p = u / nb;
    x.b = u % nb;
    x.r = ranks[(int64_t)x.p * nb + x.b];
    x.row0 = row_offsets[(int64_t)x.p * (nb + 1) + x.b];
    if (x.r < 1 || x.r > D) {  // every role clamps alike, so that the pipeline keeps its shape
      if (threadIdx.x == 0) atomicOr(status, kStatusCompressBounds);
      x.r = x.r < 1 ? 1 : D;
    }
    return x;
  };

  if (warp == 0) {
    // ---- producer: tile s of block k = tokens [128 s, 128 s + 128) of X_b, global tile g = k·tiles + s
    bool ok = true;
    int g = 0;
    for (int k = 0; k < nmine && ok; ++k) {
      const Blk x = blk(k);
      const int64_t xrow0 = (int64_t)(x.p >> 1) * T_ + (int64_t)x.b * n;  // first row of X_b in [H·T][d]
      const CUtensorMap* xmap = (x.p & 1) ? &maps.v : &maps.k;
      for (int s = 0; s < tiles && ok; ++s, ++g) {
        const int slot = g % kPStages;
        if (g >= kPStages && !(ok = pwait(bar(P_EMPTY + slot), ((g / kPStages) - 1) & 1, status))) break;
        if (lane == 0) {
          const uint32_t dst = ring + slot * kStage;
          ptx::mbar_arrive_expect_tx(bar(P_FULL + slot), kStage);
          if (D == 128) ptx::tma_load_3d(dst, xmap, bar(P_FULL + slot), 0, (int)(xrow0 + 128 * s), 0);
          else ptx::tma_load_2d(dst, xmap, bar(P_FULL + slot), 0, (int)(xrow0 + 128 * s));
        }
        __syncwarp();
      }
    }
    // drain: the CTA's copies have landed before it can exit
    for (int h = std::max(0, g - kPStages); h < g; ++h) pwait(bar(P_FULL + h % kPStages), (h / kPStages) & 1, status);
  } else if (warp == 1) {
    // ---- MMA issuer: Uᵀ tile = A_hi · Xᵀ + A_lo · Xᵀ, M = 128 rank rows, N = 128 tokens, K = d
    constexpr uint32_t idesc = ptx::idesc_bf16(128, 128, false, false);
    bool ok = true;
    int g = 0;
    for (int k = 0; k < nmine && ok; ++k) {
      const int ab = k & 1;
      ok = pwait(bar(P_AREADY + ab), (k >> 1) & 1, status);
      ptx::tc_fence_after();
      for (int s = 0; s < tiles && ok; ++s, ++g) {
        const int slot = g % kPStages, buf = g & 1;
        if (g >= 2) ok = pwait(bar(P_TEMPTY + buf), ((g >> 1) - 1) & 1, status);
        if (ok) ok = pwait(bar(P_FULL + slot), (g / kPStages) & 1, status);
        ptx::tc_fence_after();
        if (ok && lane == 0) {
          const uint32_t xs = ring + slot * kStage, d_t = tmem + 128u * buf;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            ptx::umma_bf16(d_t, pdesc(a_hi(ab), kk), pdesc(xs, kk), idesc, kk > 0 ? 1u : 0u);
            ptx::umma_bf16(d_t, pdesc(a_lo(ab), kk), pdesc(xs, kk), idesc, 1u);
          }
          ptx::umma_commit(bar(P_EMPTY + slot));  // the stage may be reloaded once these MMAs have read it
          ptx::umma_commit(bar(P_TFULL + buf));   // the accumulator is complete
        }
        __syncwarp();
      }
      if (ok && lane == 0) ptx::umma_commit(bar(P_AFREE + ab));  // block k's A buffer may be rewritten
      __syncwarp();
    }
    // drain: every MMA issued has completed before TMEM is freed (the epilogue normally waited already)
    if (lane == 0) ptx::umma_commit(bar(P_DONE));
    __syncwarp();
    pwait(bar(P_DONE), 0, status);
  } else if (warp >= 6) {
    // ---- warps 6..13: each block's A operand and dimension-side factor, up to two blocks ahead of the MMAs
    // (the epilogue warps never wait for a conversion)
    const int cw = warp - 6;
    bool ok = true;
    auto convert = [&](int k) {
      const Blk x = blk(k);
      const int ab = k & 1;
      // the MMAs of block k − 2 have read this buffer
      if (k >= 2) ok = ok && pwait(bar(P_AFREE + ab), ((k >> 1) - 1) & 1, status);
      if (ok) {
        const float* ev = eigvecs + ((int64_t)x.p * nb + x.b) * D * D;
        // rows j = cw, cw + kPConvWarps, ...: lane handles columns [4 lane, 4 lane + 4) of each 128-column
        // block; the loads of kRows rows are issued together so that their latencies overlap
        constexpr int kRows = 8;
        for (int j0 = cw; j0 < 128; j0 += kPConvWarps * kRows) {
          float4 vv[kRows][(D + 127) / 128];
#pragma unroll
          for (int q = 0; q < kRows; ++q) {
            const int j = j0 + kPConvWarps * q;
#pragma unroll
            for (int c0 = 0; c0 < D; c0 += 128) {
              const int c = c0 + 4 * lane;
              vv[q][c0 / 128] = make_float4(0.f, 0.f, 0.f, 0.f);
              if (c < D && j < x.r) vv[q][c0 / 128] = __ldg(reinterpret_cast<const float4*>(ev + (int64_t)j * D + c));
            }
          }
#pragma unroll
          for (int q = 0; q < kRows; ++q) {
          const int j = j0 + kPConvWarps * q;
#pragma unroll
          for (int c0 = 0; c0 < D; c0 += 128) {
            const int c = c0 + 4 * lane;
            if (c >= D) continue;
            const float4 v = vv[q][c0 / 128];
            const uint32_t h01 = ptx::pack_bf16(v.x, v.y), h23 = ptx::pack_bf16(v.z, v.w);
            const uint32_t l01 =
                ptx::pack_bf16(v.x - __uint_as_float(h01 << 16), v.y - __uint_as_float(h01 & 0xFFFF0000u));
            const uint32_t l23 =
                ptx::pack_bf16(v.z - __uint_as_float(h23 << 16), v.w - __uint_as_float(h23 & 0xFFFF0000u));
            // K-major SW128 position of (row j, column c): column block c / 64, 16-byte chunk ((c % 64) / 8) ^ (j % 8)
            const uint32_t off = (uint32_t)(c >> 6) * 16384u + (uint32_t)j * 128u +
                                 ((uint32_t)(((c & 63) >> 3) ^ (j & 7)) << 4) + (uint32_t)(c & 7) * 2u;
            asm volatile("st.shared.v2.b32 [%0], {%1, %2};" ::"r"(a_hi(ab) + off), "r"(h01), "r"(h23) : "memory");
            asm volatile("st.shared.v2.b32 [%0], {%1, %2};" ::"r"(a_lo(ab) + off), "r"(l01), "r"(l23) : "memory");
            if (j < x.r) {
              uint2 w;
              w.x = h01;
              w.y = h23;
              *reinterpret_cast<uint2*>(dim + (x.row0 + j) * D + c) = w;
            }
          }
          }
        }
      }
      ptx::fence_async_smem();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(bar(P_AREADY + ab));
    };
    for (int k = 0; k < nmine && ok; ++k) convert(k);
  } else {
    // ---- warps 2..5, the epilogue: lane j of this warp's quarter holds rank component j = 32 quarter + lane;
    // 128 tokens per tile
    const int quarter = warp & 3;  // a warp reads TMEM lanes [32 (warp % 4), 32 (warp % 4) + 32)
    bool ok = true;
    const int j = 32 * quarter + lane;
    const uint32_t tl = tmem + ((uint32_t)(32 * quarter) << 16);
    int g = 0;
    for (int k = 0; k < nmine && ok; ++k) {
      const Blk x = blk(k);
      for (int s = 0; s < tiles; ++s, ++g) {
        const int buf = g & 1;
        if (!ok || !(ok = pwait(bar(P_TFULL + buf), (g >> 1) & 1, status))) break;
        ptx::tc_fence_after();
        __nv_bfloat16* dst = tok + x.row0 * n + (int64_t)s * (x.r * 128) + (int64_t)j * 128;
#pragma unroll 1
        for (int c32 = 0; c32 < 128; c32 += 32) {
          float v[32];
          ptx::tmem_ld32(tl + 128u * buf + c32, v);
          ptx::tmem_wait_ld();
          if (j < x.r) {
            uint32_t w[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) w[e] = ptx::pack_bf16(v[2 * e], v[2 * e + 1]);
            uint4* d4 = reinterpret_cast<uint4*>(dst + c32);
#pragma unroll
            for (int q = 0; q < 4; ++q) d4[q] = make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
          }
        }
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(bar(P_TEMPTY + buf));
      }
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  if (warp == 1) ptx::tmem_dealloc(tmem, 256);
}

PFN_cuTensorMapEncodeTiled_v12000 proj_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

bool pmap(CUtensorMap* m, const void* ptr, int rank, const cuuint64_t* dims, const cuuint64_t* strides,
          const cuuint32_t* box) {
  auto fn = proj_encode_fn();
  if (!fn) return false;
  cuuint32_t es[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(ptr), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D>
constexpr int proj_smem() {
  return (4 + kPStages) * 16384 * (D / 64) + 8 * P_COUNT + 16 + 1024;
}

}  // namespace

bool project_tc_supported(const CompressShape& s) {
  return s.bf16 && (s.d == 64 || s.d == 128) && s.n % 128 == 0 && proj_encode_fn() != nullptr;
}

cudaError_t launch_project_tc(const CompressShape& s, const void* K, const void* V, const float* eigvecs,
                              const int32_t* ranks, const int64_t* row_offsets, void* tok, void* dim,
                              uint32_t* status, cudaStream_t st) {
  if (!project_tc_supported(s)) return cudaErrorNotSupported;
  const uint64_t rows = (uint64_t)s.H * s.T;
  ProjMaps maps;
  if (s.d == 128) {
    const cuuint64_t d3[3] = {64, rows, 2}, s3[2] = {256, 128};
    const cuuint32_t b3[3] = {64, 128, 2};
    if (!pmap(&maps.k, K, 3, d3, s3, b3) || !pmap(&maps.v, V, 3, d3, s3, b3)) return cudaErrorInvalidValue;
  } else {
    const cuuint64_t d2[2] = {64, rows}, s2[1] = {128};
    const cuuint32_t b2[2] = {64, 128};
    if (!pmap(&maps.k, K, 2, d2, s2, b2) || !pmap(&maps.v, V, 2, d2, s2, b2)) return cudaErrorInvalidValue;
  }
  const int64_t nblocks = 2LL * s.H * s.nb;
  if (nblocks > 0x7fffffff) return cudaErrorInvalidValue;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const unsigned grid = (unsigned)std::min<int64_t>(nblocks, sms);  // one persistent CTA per SM
  cudaError_t e;
  if (s.d == 128) {
    if ((e = cudaFuncSetAttribute(project_tc_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  proj_smem<128>())) != cudaSuccess)
      return e;
    project_tc_kernel<128><<<grid, kPThreads, proj_smem<128>(), st>>>(
        maps, s.T, s.n, s.nb, (int)nblocks, eigvecs, ranks, row_offsets, static_cast<__nv_bfloat16*>(tok),
        static_cast<__nv_bfloat16*>(dim), status);
  } else {
    if ((e = cudaFuncSetAttribute(project_tc_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  proj_smem<64>())) != cudaSuccess)
      return e;
    project_tc_kernel<64><<<grid, kPThreads, proj_smem<64>(), st>>>(
        maps, s.T, s.n, s.nb, (int)nblocks, eigvecs, ranks, row_offsets, static_cast<__nv_bfloat16*>(tok),
        static_cast<__nv_bfloat16*>(dim), status);
  }
  return cudaGetLastError();
}

}  // namespace milo
