// Per-block Gram matrices G_b = X_bᵀ X_b on the sm_100a tensor cores (bf16 blocks).
//
// Page "MILO: Efficient Many-shot In-Context Learning with Block-wise Low-rank
// Compression", §4.2: each block's keys and values are approximated at low rank
// separately; the truncated SVD starts from the block's Gram matrix (its
// eigenvalues are σ_i², its eigenvectors the right singular vectors).
//
// A unit is one block (d = 128) or a pair of consecutive blocks (d = 64, placed
// side by side as one 128-column tile; only the two diagonal 64×64 Grams are
// kept).  Two CTAs per SM each walk several units.  Warp 0 streams them through
// a 3-stage ring of 128-token tiles by TMA (128-byte swizzle, [64-column
// block][128 tokens][128 B]); warp 1 issues tcgen05.mma kind::f16 with the same
// tile as both operands, MN-major (A = X_bᵀ: M = features; B = X_b: N =
// features; K = tokens), into one of two 128×128 fp32 accumulators in TMEM
// (bf16 products are exact in fp32); warps 2..5 read a finished accumulator
// (32 TMEM lanes = rows each) and store row m of G as column m, the same matrix
// by symmetry, which makes each warp's stores contiguous, while the next unit
// is already loading.
//
// Waits are bounded (1 s): on expiry the kernel records kStatusCompressTimeout and
// returns after its own copies and MMAs have landed.
#include <cudaTypedefs.h>

#include <algorithm>

#include "common.cuh"
#include "internal.h"
#include "tc_ptx.cuh"

namespace milo {
namespace {

constexpr int kGThreads = 192;  // warp 0 TMA, warp 1 MMA, warps 2..5 epilogue
constexpr int kStages = 3;
constexpr uint32_t kStageBytes = 32768;  // 128 tokens × 128 columns × 2 B
constexpr int kGSmem = kStages * kStageBytes + 1024 + 256;
constexpr uint64_t kGWaitNs = 1000000000ull;

enum GBar { G_FULL = 0, G_EMPTY = G_FULL + kStages, G_TFULL = G_EMPTY + kStages, G_TEMPTY = G_TFULL + 2,
            G_DONE = G_TEMPTY + 2, G_COUNT };

// Warp-collective bounded wait; false after kGWaitNs (the status flag is set).
__device__ __noinline__ bool gwait(uint32_t bar, uint32_t parity, uint32_t* status) {
  uint64_t t0 = 0;
  if ((threadIdx.x & 31) == 0) t0 = ptx::globaltimer();
  for (uint32_t i = 1;; ++i) {
    if (__all_sync(0xffffffffu, ptx::mbar_try_wait(bar, parity))) return true;
    if ((i & 63) == 0) {
      int late = 0;
      if ((threadIdx.x & 31) == 0) late = ptx::globaltimer() - t0 > kGWaitNs;
      if (__shfl_sync(0xffffffffu, late, 0)) {
        if ((threadIdx.x & 31) == 0) atomicOr(status, kStatusCompressTimeout);
        return false;
      }
    }
  }
}

struct GramMaps {
  CUtensorMap k2, v2;  // 2D [rows][d], box 64 × 128 rows
  CUtensorMap k3, v3;  // 3D {64, rows, 2} (d = 128), box 64 × 128 rows × 2 column blocks
};

// MN-major SW128 descriptor of k-step k (16 tokens) of a stage [cb][128 tokens][128 B].
__device__ __forceinline__ uint64_t gdesc(uint32_t stage, int k) {
  return ptx::sw128_desc(stage + (uint32_t)k * 2048u, 16384u, 1024u);
}

template <int D>
__global__ void __launch_bounds__(kGThreads) gram_tc_kernel(const __grid_constant__ GramMaps maps, int64_t T_,
                                                           int n, int nb, int units, float* __restrict__ gram,
                                                           uint32_t* __restrict__ status) {
  constexpr int PER = D == 128 ? 1 : 2;  // blocks per unit
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const uint32_t base = ptx::smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kStages * kStageBytes);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + G_COUNT);
  auto bar = [&](int i) { return ptx::smem_u32(&bars[i]); };
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

  if (threadIdx.x == 0) {
    for (int i = 0; i < G_COUNT; ++i) ptx::mbar_init(bar(i), (i == G_TEMPTY || i == G_TEMPTY + 1) ? 4 : 1);
    ptx::fence_mbar_init();
  }
  if (warp == 0) {
    ptx::tmem_alloc(ptx::smem_u32(tmem_slot), 256);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // The CTA's units are u = blockIdx.x, + gridDim.x, ...; a unit holds PER blocks, flat index i = PER·u + j over
  // (pool p = i / nb, block b = i % nb).
  auto unit_rows = [&](int u, int64_t* row0, bool* is_v) {
#pragma unroll
    for (int j = 0; j < PER; ++j) {
      const int64_t i = (int64_t)PER * u + j;
      const int p = (int)(i / nb), b = (int)(i % nb);
      is_v[j] = p & 1;
      row0[j] = (int64_t)(p >> 1) * T_ + (int64_t)b * n;
    }
  };
  const int stages = n / 128;
  const int nmine = units > (int)blockIdx.x ? (units - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;

  if (warp == 0) {
    // ---- producer: global stage g = k·stages + s (unit k of this CTA, tokens [128 s, 128 s + 128))
    bool ok = true;
    int g = 0;
    for (int k = 0; k < nmine && ok; ++k) {
      int64_t row0[PER];
      bool is_v[PER];
      unit_rows((int)blockIdx.x + k * (int)gridDim.x, row0, is_v);
      for (int s = 0; s < stages && ok; ++s, ++g) {
        const int slot = g % kStages;
        if (g >= kStages && !(ok = gwait(bar(G_EMPTY + slot), ((g / kStages) - 1) & 1, status))) break;
        if (lane == 0) {
          const uint32_t dst = base + slot * kStageBytes;
          ptx::mbar_arrive_expect_tx(bar(G_FULL + slot), kStageBytes);
          if (D == 128) {
            ptx::tma_load_3d(dst, is_v[0] ? &maps.v3 : &maps.k3, bar(G_FULL + slot), 0, (int)(row0[0] + 128 * s), 0);
          } else {
#pragma unroll
            for (int j = 0; j < PER; ++j)
              ptx::tma_load_2d(dst + 16384u * j, is_v[j] ? &maps.v2 : &maps.k2, bar(G_FULL + slot), 0,
                               (int)(row0[j] + 128 * s));
          }
        }
        __syncwarp();
      }
    }
    // drain: the CTA's copies have landed before it can exit (the issuer normally waited on them already)
    for (int h = std::max(0, g - kStages); h < g; ++h) gwait(bar(G_FULL + h % kStages), (h / kStages) & 1, status);
  } else if (warp == 1) {
    // ---- MMA issuer: G += X_sᵀ X_s per stage, 8 k-steps of 16 tokens, into accumulator k & 1 of unit k
    constexpr uint32_t idesc = ptx::idesc_bf16(128, 128, true, true);
    bool ok = true;
    int g = 0;
    for (int k = 0; k < nmine && ok; ++k) {
      const int a = k & 1;
      // the epilogue has read this accumulator's previous unit
      if (k >= 2) ok = gwait(bar(G_TEMPTY + a), ((k >> 1) - 1) & 1, status);
      ptx::tc_fence_after();
      for (int s = 0; s < stages && ok; ++s, ++g) {
        const int slot = g % kStages;
        ok = gwait(bar(G_FULL + slot), (g / kStages) & 1, status);
        ptx::tc_fence_after();
        if (ok && lane == 0) {
          const uint32_t st = base + slot * kStageBytes;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            ptx::umma_bf16(tmem + 128u * a, gdesc(st, kk), gdesc(st, kk), idesc, (s > 0 || kk > 0) ? 1u : 0u);
          ptx::umma_commit(bar(G_EMPTY + slot));  // the stage may be reloaded once these MMAs have read it
        }
        __syncwarp();
      }
      if (ok && lane == 0) ptx::umma_commit(bar(G_TFULL + a));  // unit k's accumulator is complete
      __syncwarp();
    }
    if (lane == 0) ptx::umma_commit(bar(G_DONE));  // every MMA issued above has completed
    __syncwarp();
    gwait(bar(G_DONE), 0, status);
  } else {
    // ---- epilogue (warps 2..5, TMEM lane quarter warp & 3): row m of G → column m of the output, while the
    // producer and the issuer already work on the next unit
    const int quarter = warp & 3;
    const uint32_t tl = tmem + ((uint32_t)(32 * quarter) << 16);
    const int m = 32 * quarter + lane;  // TMEM lane = row of the 128 × 128 tile
    // d = 128: one Gram, all columns; d = 64: rows < 64 → first block's columns [0, 64), rows >= 64 → second
    // block's columns [64, 128)
    const int j = D == 128 ? 0 : (m >> 6);
    const int c0 = D == 128 ? 0 : 64 * j, mr = D == 128 ? m : (m & 63);
    for (int k = 0; k < nmine; ++k) {
      const int a = k & 1;
      if (!gwait(bar(G_TFULL + a), (k >> 1) & 1, status)) break;
      ptx::tc_fence_after();
      const int u = (int)blockIdx.x + k * (int)gridDim.x;
      float* G = gram + ((int64_t)PER * u + j) * D * D;
#pragma unroll 1
      for (int c32 = 0; c32 < D; c32 += 32) {
        float v[32];
        ptx::tmem_ld32(tl + 128u * a + c0 + c32, v);
        ptx::tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; ++e) G[(int64_t)(c32 + e) * D + mr] = v[e];
      }
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(bar(G_TEMPTY + a));
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  if (warp == 0) ptx::tmem_dealloc(tmem, 256);
}

PFN_cuTensorMapEncodeTiled_v12000 gram_encode_fn() {
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

bool gmap(CUtensorMap* m, const void* ptr, int rank, const cuuint64_t* dims, const cuuint64_t* strides,
          const cuuint32_t* box) {
  auto fn = gram_encode_fn();
  if (!fn) return false;
  cuuint32_t es[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(ptr), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool gram_tc_supported(const CompressShape& s) {
  return s.bf16 && (s.d == 64 || s.d == 128) && s.n % 128 == 0 && (s.d == 128 || (2LL * s.H * s.nb) % 2 == 0) &&
         gram_encode_fn() != nullptr;
}

cudaError_t launch_gram_tc(const CompressShape& s, const void* K, const void* V, float* gram, uint32_t* status,
                           cudaStream_t st) {
  if (!gram_tc_supported(s)) return cudaErrorNotSupported;
  const uint64_t rows = (uint64_t)s.H * s.T;
  GramMaps maps;
  {
    const cuuint64_t d2[2] = {(cuuint64_t)s.d, rows}, s2[1] = {(cuuint64_t)s.d * 2};
    const cuuint32_t b2[2] = {64, 128};
    if (!gmap(&maps.k2, K, 2, d2, s2, b2) || !gmap(&maps.v2, V, 2, d2, s2, b2)) return cudaErrorInvalidValue;
  }
  if (s.d == 128) {
    const cuuint64_t d3[3] = {64, rows, 2}, s3[2] = {256, 128};
    const cuuint32_t b3[3] = {64, 128, 2};
    if (!gmap(&maps.k3, K, 3, d3, s3, b3) || !gmap(&maps.v3, V, 3, d3, s3, b3)) return cudaErrorInvalidValue;
  } else {
    maps.k3 = maps.k2;
    maps.v3 = maps.v2;
  }
  const int64_t nblocks = 2LL * s.H * s.nb;
  const int64_t units = s.d == 128 ? nblocks : nblocks / 2;
  if (units > 0x7fffffff) return cudaErrorInvalidValue;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  // two CTAs per SM (shared memory), each walking several units so that one unit's epilogue overlaps the
  // next one's loads
  const unsigned grid = (unsigned)std::min<int64_t>(units, 2LL * sms);
  cudaError_t e;
  if (s.d == 128) {
    if ((e = cudaFuncSetAttribute(gram_tc_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, kGSmem)) !=
        cudaSuccess)
      return e;
    gram_tc_kernel<128><<<grid, kGThreads, kGSmem, st>>>(maps, s.T, s.n, s.nb, (int)units, gram, status);
  } else {
    if ((e = cudaFuncSetAttribute(gram_tc_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, kGSmem)) !=
        cudaSuccess)
      return e;
    gram_tc_kernel<64><<<grid, kGThreads, kGSmem, st>>>(maps, s.T, s.n, s.nb, (int)units, gram, status);
  }
  return cudaGetLastError();
}

}  // namespace milo
