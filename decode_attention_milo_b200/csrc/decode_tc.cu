// Rank-space decode attention over per-block low-rank factors on the sm_100a tensor cores.
//
// Page "MILO: Efficient Many-shot In-Context Learning with Block-wise Low-rank
// Compression", §4.4: at inference the stored low-rank caches are attended.
// With K_b ≈ U_b·B_bᵀ and V_b ≈ P_b·Q_bᵀ (tok rows = U_bᵀ / P_bᵀ, dim rows =
// B_bᵀ / Q_bᵀ), for the query rows of one KV head (batch × GQA group, M = 128):
//   G1  q̃  = Q · B_b                  TMEM fp32, then split into bf16 hi + lo in smem
//   G2  S   = q̃ · U_bᵀ                per 128-token chunk, two MMAs (hi, lo)
//       p   = exp2(S·scale·log2e − m)  online softmax on the CUDA cores
//   G3  ã  += p · P_b                 TMEM fp32
//   G4  acc += ã · Q_bᵀ               once per block, TMEM fp32
// and for each query's uncompressed suffix S = q·K_sufᵀ, acc += p·V_suf.
// A block's factors are read from HBM once and shared by every row.
//
// One persistent CTA per SM walks a host-built list of segments (a KV head's
// row tile over a contiguous range of 128-token chunks, or one query's suffix
// chunks), balanced by bytes.  Warp 0 issues TMA loads into a 4-stage ring in
// exactly the order warp 1 consumes them; warp 1 issues tcgen05.mma; warps
// 2..5 (one per TMEM lane quarter, one thread per row) run the softmax and the
// TMEM↔smem conversions.  Each segment leaves a partial (m, l, acc) that the
// combine kernel merges per output row.
//
// Every wait is bounded (1 s): on expiry the kernel records
// kStatusDecodeTimeout, drains its own copies and MMAs, frees TMEM and returns.
#include <cudaTypedefs.h>
#include <math.h>

#include <algorithm>
#include <cstring>
#include <mutex>
#include <vector>

#include "common.cuh"
#include "decode_tc.h"
#include "tc_ptx.cuh"

namespace milo {
namespace {

constexpr int kThreads = 192;        // 6 warps
constexpr int kStages = 4;           // TMA ring stages
constexpr int kStageBytes = 16384;   // one piece: 64 rows × 128 columns of bf16
constexpr int kChunk = 128;          // tokens per score chunk
constexpr uint64_t kWaitNs = 1000000000ull;

// shared-memory map (bytes from a 1024-aligned base)
constexpr int kOffQ = 0;          // [cb][128 rows][128 B]  query rows, K-major over d
constexpr int kOffQtHi = 32768;   // [cb][128][128 B]  q̃ high part, K-major over rank; later ã
constexpr int kOffQtLo = 65536;   // [cb][128][128 B]  q̃ low part
constexpr int kOffP = 98304;      // 2 × [cb][128][128 B]  probabilities, K-major over tokens
constexpr int kOffRing = 163840;  // kStages × [cb][64 rows][128 B]
constexpr int kOffBar = kOffRing + kStages * kStageBytes;  // 229376
constexpr int kSmemBytes = kOffBar + 1024 + 1024;          // barriers + alignment slack
constexpr uint32_t kTileCb = 16384;  // column-block stride of a 128-row tile
constexpr uint32_t kPieceCb = 8192;  // column-block stride of a 64-row piece

// TMEM columns: acc [0,128), S slots [128,256) and [256,384), q̃ / ã [384,512)
constexpr uint32_t kTmAcc = 0, kTmS0 = 128, kTmR = 384;

enum Bar {
  B_FULL = 0,
  B_EMPTY = B_FULL + kStages,
  B_QFULL = B_EMPTY + kStages,
  B_QEMPTY,
  B_QTFULL,
  B_QTREADY,
  B_SFULL,
  B_SEMPTY = B_SFULL + 2,
  B_PFULL = B_SEMPTY + 2,
  B_PEMPTY = B_PFULL + 2,
  B_ATFULL = B_PEMPTY + 2,
  B_ATREADY,
  B_ACCFULL,
  B_FINAL,
  B_COUNT
};

struct Seg {
  int type;  // 0 prefix row tile, 1 suffix of one query
  int h;     // KV head
  int tile;  // prefix: row tile; suffix: batch item
  int c0, c1;  // chunk range (prefix: chunks of the head's context; suffix: chunks of S)
  int pid;   // partial slot
  int rows;  // valid rows
  int pad;
};

struct Params {
  const Seg* segs;
  const int* seg_first;  // [grid + 1]
  const int32_t* ranks;
  const int64_t* row_offsets;
  float* part_acc;  // [pid][128][D]
  float2* part_ml;  // [pid][128]
  uint32_t* status;
  int nb, cpb, H, G, ipt, S;
  float c;  // scale · log2(e)
};

struct Shared {
  uint32_t tmem_base;
  int abort_flag;
};

// Warp-collective bounded wait on an mbarrier phase (all 32 lanes call it together; the result is uniform).
// Gives up after kWaitNs, records kStatusDecodeTimeout and raises the CTA's abort flag, or returns false at
// once when another role already aborted.  `drain` waits ignore the abort flag (used to let the CTA's own
// copies and MMAs land before it exits) but keep the time limit.
__device__ __noinline__ bool wait_bar(uint32_t bar, uint32_t parity, Shared* sh, uint32_t* status,
                                      bool drain = false) {
  if (__all_sync(0xffffffffu, ptx::mbar_try_wait(bar, parity))) return true;
  uint64_t t0 = 0;
  if ((threadIdx.x & 31) == 0) t0 = ptx::globaltimer();
  for (uint32_t i = 1;; ++i) {
    if (__all_sync(0xffffffffu, ptx::mbar_try_wait(bar, parity))) return true;
    if ((i & 63) == 0) {
      int verdict = 0;  // 0 keep waiting, 1 aborted elsewhere, 2 timed out
      if ((threadIdx.x & 31) == 0) {
        if (!drain && *(volatile int*)&sh->abort_flag) verdict = 1;
        else if (ptx::globaltimer() - t0 > kWaitNs) verdict = 2;
      }
      verdict = __shfl_sync(0xffffffffu, verdict, 0);
      if (verdict == 2 && (threadIdx.x & 31) == 0) {
        atomicOr(status, kStatusDecodeTimeout);
        *(volatile int*)&sh->abort_flag = 1;
      }
      if (verdict) return false;
    }
  }
}

__device__ __forceinline__ int pad16(int r) { return (r + 15) & ~15; }

struct BlockInfo {
  int rk, rv;
  int64_t rowk, rowv;
};
__device__ __forceinline__ bool block_info(const Params& p, int h, int b, int D, BlockInfo& bi) {
  bi.rk = p.ranks[(int64_t)(2 * h) * p.nb + b];
  bi.rv = p.ranks[(int64_t)(2 * h + 1) * p.nb + b];
  bi.rowk = p.row_offsets[(int64_t)(2 * h) * (p.nb + 1) + b];
  bi.rowv = p.row_offsets[(int64_t)(2 * h + 1) * (p.nb + 1) + b];
  return bi.rk >= 1 && bi.rk <= D && bi.rv >= 1 && bi.rv <= D;
}

// Ring position shared by producer and consumer: both walk the same item sequence.
struct Ring {
  uint32_t stage = 0, phase = 0;
  __device__ void advance() {
    if (++stage == kStages) {
      stage = 0;
      phase ^= 1;
    }
  }
};

// -------------------------------------------------------------------------------------------- producer
template <int D>
struct Producer {
  static constexpr int NCB = D / 64;
  uint32_t base;
  Ring ring;
  uint32_t q_uses = 0;
  bool issued[kStages];
  uint32_t issued_parity[kStages];
  Shared* sh;
  uint32_t* status;

  __device__ uint32_t bar(int i) const { return base + kOffBar + 8 * i; }

  // `rows` (multiple of 16, <= 64) rows × `ncb` 64-column blocks of a 2D map at (x0, y0) → one ring stage.
  __device__ bool piece(const CUtensorMap* m, int x0, int64_t y0, int rows, int ncb) {
    if (!wait_bar(bar(B_EMPTY + ring.stage), ring.phase ^ 1, sh, status)) return false;
    const uint32_t dst = base + kOffRing + ring.stage * kStageBytes;
    const uint32_t fb = bar(B_FULL + ring.stage);
    if ((threadIdx.x & 31) == 0) {
      ptx::mbar_arrive_expect_tx(fb, rows * 128 * ncb);
      for (int cb = 0; cb < ncb; ++cb)
        for (int k = 0; k < rows; k += 16)
          ptx::tma_load_2d(dst + cb * kPieceCb + k * 128, m, fb, x0 + 64 * cb, (int)(y0 + k));
    }
    issued[ring.stage] = true;
    issued_parity[ring.stage] = ring.phase;
    ring.advance();
    return true;
  }
  __device__ bool item(const CUtensorMap* m, int x0, int64_t y0, int rows, int ncb) {
    for (int r = 0; r < rows; r += 64)
      if (!piece(m, x0, y0 + r, min(64, rows - r), ncb)) return false;
    return true;
  }
  __device__ bool q_tile(const CUtensorMap* m, int y, int z, int box_rows) {
    if (!wait_bar(bar(B_QEMPTY), (q_uses & 1) ^ 1, sh, status)) return false;
    if ((threadIdx.x & 31) == 0) {
      ptx::mbar_arrive_expect_tx(bar(B_QFULL), box_rows * 128 * NCB);
      for (int cb = 0; cb < NCB; ++cb) ptx::tma_load_3d(base + kOffQ + cb * kTileCb, m, bar(B_QFULL), 64 * cb, y, z);
    }
    ++q_uses;
    return true;
  }
};

// K-major SW128 descriptor of k-step k (16 bf16) of a tile whose 64-column blocks are `cbs` bytes apart.
__device__ __forceinline__ uint64_t kdesc(uint32_t tile, int k, uint32_t cbs) {
  return ptx::sw128_desc(tile + (uint32_t)(k >> 2) * cbs + (uint32_t)(k & 3) * 32, 16, 1024);
}
// MN-major SW128 descriptor of k-step k (16 rows) of a 64-row piece (MN column blocks kPieceCb apart).
__device__ __forceinline__ uint64_t mndesc(uint32_t piece, int k) {
  return ptx::sw128_desc(piece + (uint32_t)k * 2048, kPieceCb, 1024);
}

// Writes 8 consecutive bf16 (4 packed words) at (row, col) of a K-major SW128 tile (128-row, 16 KB col blocks).
__device__ __forceinline__ void st_tile8(uint32_t tile, int row, int col, uint32_t a, uint32_t b, uint32_t c,
                                         uint32_t d) {
  const uint32_t addr = tile + (uint32_t)(col >> 6) * kTileCb + (uint32_t)row * 128 +
                        ((uint32_t)(((col & 63) >> 3) ^ (row & 7)) << 4);
  ptx::st_shared_v4(addr, a, b, c, d);
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    decode_tc_kernel(const __grid_constant__ CUtensorMap map_tok, const __grid_constant__ CUtensorMap map_dim,
                     const __grid_constant__ CUtensorMap map_qpre, const __grid_constant__ CUtensorMap map_qsuf,
                     const __grid_constant__ CUtensorMap map_ksuf, const __grid_constant__ CUtensorMap map_vsuf,
                     const Params p) {
  constexpr int NCB = D / 64;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const uint32_t base = ptx::smem_u32(smem);
  Shared* sh = reinterpret_cast<Shared*>(smem + kOffBar + 8 * B_COUNT + 64);
  auto bar = [&](int i) { return base + kOffBar + 8 * i; };
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

  // ---- setup: zero the query tile (rows no TMA box writes stay finite), barriers, TMEM
  for (int i = threadIdx.x; i < 32768 / 16; i += kThreads) ptx::st_shared_v4(base + kOffQ + 16 * i, 0, 0, 0, 0);
  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      ptx::mbar_init(bar(B_FULL + i), 1);
      ptx::mbar_init(bar(B_EMPTY + i), 1);
    }
    ptx::mbar_init(bar(B_QFULL), 1);
    ptx::mbar_init(bar(B_QEMPTY), 1);
    ptx::mbar_init(bar(B_QTFULL), 1);
    ptx::mbar_init(bar(B_QTREADY), 4);
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(bar(B_SFULL + i), 1);
      ptx::mbar_init(bar(B_SEMPTY + i), 4);
      ptx::mbar_init(bar(B_PFULL + i), 4);
      ptx::mbar_init(bar(B_PEMPTY + i), 1);
    }
    ptx::mbar_init(bar(B_ATFULL), 1);
    ptx::mbar_init(bar(B_ATREADY), 4);
    ptx::mbar_init(bar(B_ACCFULL), 1);
    ptx::mbar_init(bar(B_FINAL), 1);
    sh->abort_flag = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    ptx::tma_prefetch_desc(&map_tok);
    ptx::tma_prefetch_desc(&map_dim);
    ptx::tma_prefetch_desc(&map_qpre);
    ptx::tma_prefetch_desc(&map_qsuf);
    ptx::tma_prefetch_desc(&map_ksuf);
    ptx::tma_prefetch_desc(&map_vsuf);
  }
  if (warp == 1) {
    ptx::tmem_alloc(ptx::smem_u32(&sh->tmem_base), 512);
    ptx::tmem_relinquish();
  }
  ptx::fence_async_smem();
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = sh->tmem_base;
  const int s_begin = p.seg_first[blockIdx.x], s_end = p.seg_first[blockIdx.x + 1];

  if (warp == 0) {
    // ==================================================================== TMA producer
    Producer<D> pr;
    pr.base = base;
    pr.sh = sh;
    pr.status = p.status;
    for (int i = 0; i < kStages; ++i) pr.issued[i] = false;
    bool ok = true;
    for (int si = s_begin; si < s_end && ok; ++si) {
      const Seg sg = p.segs[si];
      if (sg.type == 0) {
        ok = pr.q_tile(&map_qpre, sg.h * p.G, sg.tile * p.ipt, p.G * p.ipt);
        for (int c = sg.c0; c < sg.c1 && ok;) {
          const int b = c / p.cpb;
          const int cend = min(sg.c1, (b + 1) * p.cpb);
          BlockInfo bi;
          if (!block_info(p, sg.h, b, D, bi)) {
            atomicOr(p.status, kStatusDecodeBounds);
            sh->abort_flag = 1;
            ok = false;
            break;
          }
          const int rkp = pad16(bi.rk), rvp = pad16(bi.rv);
          // consumption order: B_K, U(0), [U(1), P(0)], ..., [U(n-1), P(n-2)], P(n-1), Q_V
          ok = pr.item(&map_dim, 0, bi.rowk, rkp, NCB);
          // token factor slabs: chunk cc of the block is rows [row0·cpb + cc·r, +r) of the 128-wide view
          for (int cc = c; cc <= cend && ok; ++cc) {
            if (cc < cend) ok = pr.item(&map_tok, 0, bi.rowk * p.cpb + (int64_t)(cc - b * p.cpb) * bi.rk, rkp, 2);
            if (ok && cc > c)
              ok = pr.item(&map_tok, 0, bi.rowv * p.cpb + (int64_t)(cc - 1 - b * p.cpb) * bi.rv, rvp, 2);
          }
          if (ok) ok = pr.item(&map_dim, 0, bi.rowv, rvp, NCB);
          c = cend;
        }
      } else {
        ok = pr.q_tile(&map_qsuf, sg.h * p.G, sg.tile, p.G);
        const int64_t row0 = ((int64_t)sg.tile * p.H + sg.h) * p.S;
        // consumption order: K(0), [K(1), V(0)], ..., V(n-1)
        for (int c = sg.c0; c <= sg.c1 && ok; ++c) {
          if (c < sg.c1) ok = pr.item(&map_ksuf, 0, row0 + (int64_t)c * kChunk, kChunk, NCB);
          if (ok && c > sg.c0) ok = pr.item(&map_vsuf, 0, row0 + (int64_t)(c - 1) * kChunk, kChunk, NCB);
        }
      }
    }
    // drain: every copy this warp issued must have landed before the CTA exits
    for (int i = 0; i < kStages; ++i)
      if (pr.issued[i]) wait_bar(bar(B_FULL + i), pr.issued_parity[i], sh, p.status, true);
    if (pr.q_uses) wait_bar(bar(B_QFULL), (pr.q_uses - 1) & 1, sh, p.status, true);
  } else if (warp == 1) {
    // ==================================================================== MMA issuer
    Ring ring;
    uint32_t q_uses = 0, qt_uses = 0, at_uses = 0;
    uint32_t chunk_ix = 0;  // chunks processed by this CTA: S and P slot = chunk_ix & 1
    const bool leader = lane == 0;
    bool ok = true;
    auto take = [&](uint32_t& addr) -> bool {
      if (!wait_bar(bar(B_FULL + ring.stage), ring.phase, sh, p.status)) return false;
      ptx::tc_fence_after();
      addr = base + kOffRing + ring.stage * kStageBytes;
      return true;
    };
    auto release = [&]() {
      if (leader) ptx::umma_commit(bar(B_EMPTY + ring.stage));
      ring.advance();
    };
    auto wait_s_empty = [&](uint32_t k) {
      const bool r = wait_bar(bar(B_SEMPTY + (k & 1)), ((k >> 1) & 1) ^ 1, sh, p.status);
      ptx::tc_fence_after();
      return r;
    };
    auto wait_p_full = [&](uint32_t k) {
      const bool r = wait_bar(bar(B_PFULL + (k & 1)), (k >> 1) & 1, sh, p.status);
      ptx::tc_fence_after();
      return r;
    };
    const uint32_t idS = ptx::idesc_bf16(128, 128, false, true);
    for (int si = s_begin; si < s_end && ok; ++si) {
      const Seg sg = p.segs[si];
      if (!(ok = wait_bar(bar(B_QFULL), q_uses & 1, sh, p.status))) break;
      ++q_uses;
      ptx::tc_fence_after();
      if (sg.type == 0) {
        bool first_block = true;
        for (int c = sg.c0; c < sg.c1 && ok;) {
          const int b = c / p.cpb;
          const int cend = min(sg.c1, (b + 1) * p.cpb);
          const int nch = cend - c;
          BlockInfo bi;
          if (!block_info(p, sg.h, b, D, bi)) {
            atomicOr(p.status, kStatusDecodeBounds);
            sh->abort_flag = 1;
            ok = false;
            break;
          }
          const int rkp = pad16(bi.rk), rvp = pad16(bi.rv);
          // G1: q̃ = Q · B_b → TMEM R (free: ã of the previous block was converted before its G4)
          for (int r0 = 0; r0 < rkp && ok; r0 += 64) {
            uint32_t pc;
            if (!(ok = take(pc))) break;
            const int np = min(64, rkp - r0);
            if (leader)
              for (int k = 0; k < D / 16; ++k)
                ptx::umma_bf16(tmem + kTmR + r0, kdesc(base + kOffQ, k, kTileCb), kdesc(pc, k, kPieceCb),
                               ptx::idesc_bf16(128, np, false, false), k > 0);
            release();
          }
          if (!ok) break;
          if (leader) {
            ptx::umma_commit(bar(B_QTFULL));
            if (cend == sg.c1) ptx::umma_commit(bar(B_QEMPTY));  // last read of Q in this segment
          }
          if (!(ok = wait_bar(bar(B_QTREADY), qt_uses & 1, sh, p.status))) break;
          ++qt_uses;
          ptx::tc_fence_after();
          for (int j = 0; j <= nch && ok; ++j) {
            if (j < nch) {
              // G2(j): S = q̃_hi·U + q̃_lo·U
              const uint32_t k = chunk_ix + j;
              if (!(ok = wait_s_empty(k))) break;
              const uint32_t dS = tmem + kTmS0 + 128 * (k & 1);
              for (int r0 = 0; r0 < rkp && ok; r0 += 64) {
                uint32_t pc;
                if (!(ok = take(pc))) break;
                const int kk = min(64, rkp - r0) / 16;
                if (leader)
                  for (int t = 0; t < kk; ++t) {
                    const uint64_t bd = mndesc(pc, t);
                    const int ka = r0 / 16 + t;
                    ptx::umma_bf16(dS, kdesc(base + kOffQtHi, ka, kTileCb), bd, idS, ka > 0);
                    ptx::umma_bf16(dS, kdesc(base + kOffQtLo, ka, kTileCb), bd, idS, 1);
                  }
                release();
              }
              if (!ok) break;
              if (leader) ptx::umma_commit(bar(B_SFULL + (k & 1)));
            }
            if (j > 0) {
              // G3(j-1): ã += p · P_b
              const uint32_t k = chunk_ix + j - 1;
              if (!(ok = wait_p_full(k))) break;
              const uint32_t pt = base + kOffP + 32768 * (k & 1);
              for (int r0 = 0; r0 < rvp && ok; r0 += 64) {
                uint32_t pc;
                if (!(ok = take(pc))) break;
                const int np = min(64, rvp - r0);
                if (leader)
                  for (int t = 0; t < kChunk / 16; ++t)
                    ptx::umma_bf16(tmem + kTmR + r0, kdesc(pt, t, kTileCb), kdesc(pc, t, kPieceCb),
                                   ptx::idesc_bf16(128, np, false, false), (t > 0 || j > 1) ? 1u : 0u);
                release();
              }
              if (!ok) break;
              if (leader) ptx::umma_commit(bar(B_PEMPTY + (k & 1)));
            }
          }
          if (!ok) break;
          chunk_ix += nch;
          if (leader) ptx::umma_commit(bar(B_ATFULL));
          // G4: acc += ã · Q_bᵀ once the softmax warps have moved ã to smem
          if (!(ok = wait_bar(bar(B_ATREADY), at_uses & 1, sh, p.status))) break;
          ++at_uses;
          ptx::tc_fence_after();
          for (int r0 = 0; r0 < rvp && ok; r0 += 64) {
            uint32_t pc;
            if (!(ok = take(pc))) break;
            const int kk = min(64, rvp - r0) / 16;
            if (leader)
              for (int t = 0; t < kk; ++t) {
                const int ka = r0 / 16 + t;
                ptx::umma_bf16(tmem + kTmAcc, kdesc(base + kOffQtHi, ka, kTileCb), mndesc(pc, t),
                               ptx::idesc_bf16(128, D, false, true), (ka > 0 || !first_block) ? 1u : 0u);
              }
            release();
          }
          if (!ok) break;
          c = cend;
          first_block = false;
        }
        if (ok && leader) ptx::umma_commit(bar(B_ACCFULL));
      } else {
        const int nch = sg.c1 - sg.c0;
        for (int j = 0; j <= nch && ok; ++j) {
          if (j < nch) {
            // G2'(j): S = q · K_sufᵀ, two 64-token pieces
            const uint32_t k = chunk_ix + j;
            if (!(ok = wait_s_empty(k))) break;
            const uint32_t dS = tmem + kTmS0 + 128 * (k & 1);
            for (int pi = 0; pi < 2 && ok; ++pi) {
              uint32_t pc;
              if (!(ok = take(pc))) break;
              if (leader)
                for (int t = 0; t < D / 16; ++t)
                  ptx::umma_bf16(dS + 64 * pi, kdesc(base + kOffQ, t, kTileCb), kdesc(pc, t, kPieceCb),
                                 ptx::idesc_bf16(128, 64, false, false), t > 0);
              release();
            }
            if (!ok) break;
            if (leader) {
              ptx::umma_commit(bar(B_SFULL + (k & 1)));
              if (j == nch - 1) ptx::umma_commit(bar(B_QEMPTY));
            }
          }
          if (j > 0) {
            // G3'(j-1): acc += p · V_suf
            const uint32_t k = chunk_ix + j - 1;
            if (!(ok = wait_p_full(k))) break;
            const uint32_t pt = base + kOffP + 32768 * (k & 1);
            for (int pi = 0; pi < 2 && ok; ++pi) {
              uint32_t pc;
              if (!(ok = take(pc))) break;
              if (leader)
                for (int t = 0; t < 4; ++t)
                  ptx::umma_bf16(tmem + kTmAcc, kdesc(pt, 4 * pi + t, kTileCb), mndesc(pc, t),
                                 ptx::idesc_bf16(128, D, false, true), (j > 1 || pi > 0 || t > 0) ? 1u : 0u);
              release();
            }
            if (!ok) break;
            if (leader) ptx::umma_commit(bar(B_PEMPTY + (k & 1)));
          }
        }
        if (!ok) break;
        chunk_ix += nch;
        if (leader) ptx::umma_commit(bar(B_ACCFULL));
      }
    }
    // drain: every MMA issued must complete before TMEM is freed
    if (leader) ptx::umma_commit(bar(B_FINAL));
    __syncwarp();
    wait_bar(bar(B_FINAL), 0, sh, p.status, true);
  } else {
    // ==================================================================== softmax warpgroup
    const int quarter = warp & 3;
    const int row = 32 * quarter + lane;
    const uint32_t tl = tmem + ((uint32_t)(32 * quarter) << 16);
    uint32_t chunk_ix = 0, qt_uses = 0, at_uses = 0, acc_uses = 0;
    bool ok = true;
    // one arrival per warp on the barriers the warpgroup signals (init count 4)
    auto arrive = [&](int b) {
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(bar(b));
    };
    for (int si = s_begin; si < s_end && ok; ++si) {
      const Seg sg = p.segs[si];
      // a warp whose 32 rows are all padding only keeps the barrier protocol
      const bool active = 32 * quarter < sg.rows;
      float m_used = -INFINITY, l = 0.f;
      bool first_chunk = true;
      const bool prefix = sg.type == 0;
      int c = sg.c0;
      bool first_block = true;
      while (c < sg.c1 && ok) {
        int cend, rv = 0, rvp = 0;
        if (prefix) {
          const int b = c / p.cpb;
          cend = min(sg.c1, (b + 1) * p.cpb);
          BlockInfo bi;
          if (!block_info(p, sg.h, b, D, bi)) {
            ok = false;
            break;
          }
          rv = bi.rv;
          rvp = pad16(bi.rv);
          const int rk = bi.rk, rkp = pad16(bi.rk);
          // q̃ (fp32, TMEM) → bf16 hi + lo in smem, columns >= r zeroed
          if (!(ok = wait_bar(bar(B_QTFULL), qt_uses & 1, sh, p.status))) break;
          ++qt_uses;
          ptx::tc_fence_after();
          if (active) {
            for (int half = 0; half < rkp; half += 64) {
              float v[64];
#pragma unroll
              for (int q = 0; q < 4; ++q) ptx::tmem_ld16(tl + kTmR + half + 16 * q, v + 16 * q);
              ptx::tmem_wait_ld();
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                const int col = half + 16 * q;
                if (col < rkp) {
                  uint32_t hi[8], lo[8];
#pragma unroll
                  for (int e = 0; e < 16; e += 2) {
                    const float a = (col + e < rk) ? v[16 * q + e] : 0.f;
                    const float b2 = (col + e + 1 < rk) ? v[16 * q + e + 1] : 0.f;
                    const uint32_t h2 = ptx::pack_bf16(a, b2);
                    hi[e / 2] = h2;
                    lo[e / 2] =
                        ptx::pack_bf16(a - __uint_as_float(h2 << 16), b2 - __uint_as_float(h2 & 0xFFFF0000u));
                  }
                  st_tile8(base + kOffQtHi, row, col, hi[0], hi[1], hi[2], hi[3]);
                  st_tile8(base + kOffQtHi, row, col + 8, hi[4], hi[5], hi[6], hi[7]);
                  st_tile8(base + kOffQtLo, row, col, lo[0], lo[1], lo[2], lo[3]);
                  st_tile8(base + kOffQtLo, row, col + 8, lo[4], lo[5], lo[6], lo[7]);
                }
              }
            }
            ptx::fence_async_smem();
          }
          ptx::tc_fence_before();
          arrive(B_QTREADY);
        } else {
          cend = sg.c1;
        }
        for (int cc = c; cc < cend && ok; ++cc) {
          const uint32_t k = chunk_ix;
          const uint32_t slot = k & 1;
          if (!(ok = wait_bar(bar(B_SFULL + slot), (k >> 1) & 1, sh, p.status))) break;
          ptx::tc_fence_after();
          float s[kChunk];
          if (active) {
#pragma unroll
            for (int q = 0; q < kChunk / 16; ++q) ptx::tmem_ld16(tl + kTmS0 + 128 * slot + 16 * q, s + 16 * q);
            ptx::tmem_wait_ld();
          }
          ptx::tc_fence_before();
          arrive(B_SEMPTY + slot);
          float alpha = 1.f;
          bool grow = false;
          if (active) {
            if (!prefix) {
              const int valid = p.S - cc * kChunk;
#pragma unroll
              for (int j = 0; j < kChunk; ++j)
                if (j >= valid) s[j] = -INFINITY;
            }
            // tree max (8 independent lanes of reduction, then fold)
            float m8[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) m8[e] = s[e];
#pragma unroll
            for (int j = 8; j < kChunk; j += 8)
#pragma unroll
              for (int e = 0; e < 8; ++e) m8[e] = fmaxf(m8[e], s[j + e]);
            float mx = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])),
                             fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
            mx *= p.c;
            // keep the running max in use unless the chunk exceeds it by more than 2^8 (then rescale)
            grow = !first_chunk && mx > m_used + 8.f;
            if (grow) {
              alpha = ptx::ex2(m_used - mx);
              m_used = mx;
              l *= alpha;
            }
            if (first_chunk) m_used = mx;
          }
          if (__any_sync(0xffffffffu, grow)) {
            // rare: rescale what this warp's rows accumulated so far (alpha = 1 for rows that did not grow)
            const bool have_at = prefix && cc > c;  // ã holds earlier chunks of this block
            const bool have_acc = prefix ? !first_block : true;
            if (have_at || !prefix) {
              // the previous G3 must have landed before ã (or the suffix acc) is touched
              if (!(ok = wait_bar(bar(B_PEMPTY + ((k - 1) & 1)), ((k - 1) >> 1) & 1, sh, p.status))) break;
              ptx::tc_fence_after();
            }
            if (have_at) {
              for (int c16 = 0; c16 < rvp; c16 += 16) {
                float v[16];
                ptx::tmem_ld16(tl + kTmR + c16, v);
                ptx::tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 16; ++e) v[e] *= alpha;
                ptx::tmem_st16(tl + kTmR + c16, v);
              }
            }
            if (have_acc) {
              for (int c16 = 0; c16 < D; c16 += 16) {
                float v[16];
                ptx::tmem_ld16(tl + kTmAcc + c16, v);
                ptx::tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 16; ++e) v[e] *= alpha;
                ptx::tmem_st16(tl + kTmAcc + c16, v);
              }
            }
            ptx::tmem_wait_st();
          }
          first_chunk = false;
          // p = exp2(S·c − m), row sum, bf16 tile
          if (!(ok = wait_bar(bar(B_PEMPTY + slot), ((k >> 1) & 1) ^ 1, sh, p.status))) break;
          if (active) {
            const uint32_t pt = base + kOffP + 32768 * slot;
            float ls[4] = {0.f, 0.f, 0.f, 0.f};  // independent partial row sums
#pragma unroll
            for (int g8 = 0; g8 < kChunk / 8; ++g8) {
              uint32_t w[4];
#pragma unroll
              for (int e = 0; e < 8; e += 2) {
                const float a = ptx::ex2(fmaf(s[8 * g8 + e], p.c, -m_used));
                const float b2 = ptx::ex2(fmaf(s[8 * g8 + e + 1], p.c, -m_used));
                ls[e / 2] += a + b2;
                w[e / 2] = ptx::pack_bf16(a, b2);
              }
              st_tile8(pt, row, 8 * g8, w[0], w[1], w[2], w[3]);
            }
            l += (ls[0] + ls[1]) + (ls[2] + ls[3]);
            ptx::fence_async_smem();
          }
          ptx::tc_fence_before();
          arrive(B_PFULL + slot);
          ++chunk_ix;
        }
        if (!ok) break;
        if (prefix) {
          // ã (fp32, TMEM) → bf16 in smem (over q̃_hi, whose readers are done), columns >= r zeroed
          if (!(ok = wait_bar(bar(B_ATFULL), at_uses & 1, sh, p.status))) break;
          ++at_uses;
          ptx::tc_fence_after();
          if (active) {
            for (int half = 0; half < rvp; half += 64) {
              float v[64];
#pragma unroll
              for (int q = 0; q < 4; ++q) ptx::tmem_ld16(tl + kTmR + half + 16 * q, v + 16 * q);
              ptx::tmem_wait_ld();
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                const int col = half + 16 * q;
                if (col < rvp) {
                  uint32_t w[8];
#pragma unroll
                  for (int e = 0; e < 16; e += 2)
                    w[e / 2] = ptx::pack_bf16(col + e < rv ? v[16 * q + e] : 0.f,
                                              col + e + 1 < rv ? v[16 * q + e + 1] : 0.f);
                  st_tile8(base + kOffQtHi, row, col, w[0], w[1], w[2], w[3]);
                  st_tile8(base + kOffQtHi, row, col + 8, w[4], w[5], w[6], w[7]);
                }
              }
            }
            ptx::fence_async_smem();
          }
          ptx::tc_fence_before();
          arrive(B_ATREADY);
        }
        c = cend;
        first_block = false;
      }
      if (!ok) break;
      // segment result: (m, l, acc) of this row
      if (!(ok = wait_bar(bar(B_ACCFULL), acc_uses & 1, sh, p.status))) break;
      ++acc_uses;
      ptx::tc_fence_after();
      if (active) {
        float* dst = p.part_acc + ((int64_t)sg.pid * 128 + row) * D;
        for (int half = 0; half < D; half += 64) {
          float v[64];
#pragma unroll
          for (int q = 0; q < 4; ++q) ptx::tmem_ld16(tl + kTmAcc + half + 16 * q, v + 16 * q);
          ptx::tmem_wait_ld();
          if (row < sg.rows) {
#pragma unroll
            for (int e = 0; e < 64; e += 4)
              *reinterpret_cast<float4*>(dst + half + e) = make_float4(v[e], v[e + 1], v[e + 2], v[e + 3]);
          }
        }
        if (row < sg.rows) p.part_ml[(int64_t)sg.pid * 128 + row] = make_float2(m_used, l);
      }
      ptx::tc_fence_before();
    }
  }

  // ---- teardown: every role has drained its own async work; free TMEM
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  if (warp == 1) ptx::tmem_dealloc(tmem, 512);
}

// Merges the partials of one output row (i, hq): m = max m_k, l = Σ l_k 2^{m_k−m},
// out = Σ acc_k 2^{m_k−m} / l.  The (m, l) pairs are read in parallel first, so the
// acc loads of the second phase are independent of each other.
constexpr int kMaxParts = 1024;
template <int D>
__global__ void __launch_bounds__(D) combine_tc_kernel(const float* __restrict__ part_acc,
                                                      const float2* __restrict__ part_ml,
                                                      const int* __restrict__ pre_range,
                                                      const int* __restrict__ suf_range, int H, int Hq, int ipt,
                                                      int nrt, __nv_bfloat16* __restrict__ out) {
  __shared__ float wgt[kMaxParts];
  __shared__ int src[kMaxParts];
  __shared__ float red[D / 32];
  __shared__ float s_m, s_l;
  const int hq = blockIdx.x, i = blockIdx.y, c = threadIdx.x;
  const int G = Hq / H, h = hq / G, g = hq % G;
  const int rt = i / ipt, prow = (i % ipt) * G + g;
  const int p0 = pre_range[2 * (h * nrt + rt)], p1 = pre_range[2 * (h * nrt + rt) + 1];
  const int s0 = suf_range[2 * (i * H + h)], s1 = suf_range[2 * (i * H + h) + 1];
  const int npre = p1 - p0, nall = npre + (s1 - s0);
  float mloc = -INFINITY;
  for (int t = c; t < nall; t += D) {
    const int idx = t < npre ? (p0 + t) * 128 + prow : (s0 + t - npre) * 128 + g;
    src[t] = idx;
    const float2 ml = part_ml[idx];
    wgt[t] = ml.x;
    mloc = fmaxf(mloc, ml.x);
  }
  mloc = warp_max(mloc);
  if ((c & 31) == 0) red[c / 32] = mloc;
  __syncthreads();
  if (c == 0) {
    float m = red[0];
    for (int w = 1; w < D / 32; ++w) m = fmaxf(m, red[w]);
    s_m = m;
  }
  __syncthreads();
  const float m = s_m;
  float lloc = 0.f;
  for (int t = c; t < nall; t += D) {
    const float w = exp2f(wgt[t] - m);
    wgt[t] = w;
    lloc = fmaf(part_ml[src[t]].y, w, lloc);
  }
  lloc = warp_sum(lloc);
  __syncthreads();
  if ((c & 31) == 0) red[c / 32] = lloc;
  __syncthreads();
  if (c == 0) {
    float l = 0.f;
    for (int w = 0; w < D / 32; ++w) l += red[w];
    s_l = l;
  }
  __syncthreads();
  float acc0 = 0.f, acc1 = 0.f, acc2 = 0.f, acc3 = 0.f;
  int t = 0;
  for (; t + 4 <= nall; t += 4) {
    acc0 = fmaf(part_acc[(int64_t)src[t] * D + c], wgt[t], acc0);
    acc1 = fmaf(part_acc[(int64_t)src[t + 1] * D + c], wgt[t + 1], acc1);
    acc2 = fmaf(part_acc[(int64_t)src[t + 2] * D + c], wgt[t + 2], acc2);
    acc3 = fmaf(part_acc[(int64_t)src[t + 3] * D + c], wgt[t + 3], acc3);
  }
  for (; t < nall; ++t) acc0 = fmaf(part_acc[(int64_t)src[t] * D + c], wgt[t], acc0);
  out[((int64_t)i * Hq + hq) * D + c] = __float2bfloat16_rn(((acc0 + acc1) + (acc2 + acc3)) / s_l);
}

// ------------------------------------------------------------------------------------------------ host
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
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

bool make_map(CUtensorMap* m, const void* ptr, int rank, const uint64_t* dims, const uint64_t* strides_bytes,
              const uint32_t* box) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t gd[3], gs[2];
  cuuint32_t bx[3], es[3] = {1, 1, 1};
  for (int i = 0; i < rank; ++i) {
    gd[i] = dims[i];
    bx[i] = box[i];
  }
  for (int i = 0; i + 1 < rank; ++i) gs[i] = strides_bytes[i];
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(ptr), gd, gs, bx, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

struct TcPlan {
  int Bq = 0, Hq = 0, S = 0;
  int grid = 0, nsegs = 0, ipt = 0, nrt = 0;
  int* d_work = nullptr;  // seg_first | segs | pre_range | suf_range
  int off_segs = 0, off_pre = 0, off_suf = 0;
  float* part_acc = nullptr;
  float2* part_ml = nullptr;
  const void* tok = nullptr;
  const void* dim = nullptr;
  CUtensorMap map_tok, map_dim;
};

bool tc_supported(const DecodeShape& s) {
  const int G = s.Hq / s.H;
  return s.bf16 && (s.d == 64 || s.d == 128) && s.n % kChunk == 0 && G >= 1 && G <= 128 && s.Hq % s.H == 0 &&
         encode_fn() != nullptr;
}

int tc_launches(const DecodeShape&) { return 2; }

void tc_plan_destroy(TcPlan* plan) {
  if (!plan) return;
  cudaFree(plan->d_work);
  cudaFree(plan->part_acc);
  cudaFree(plan->part_ml);
  delete plan;
}

// fixed per-chunk, per-block and per-suffix-unit times used to balance the work list (measured orders)
constexpr double kChunkNs = 700.0, kBlockNs = 1500.0, kUnitNs = 1500.0;

static cudaError_t build_plan(TcPlan* pl, const DecodeShape& s, const TcInputs& in) {
  const int H = s.H, nb = s.nb, D = s.d, G = s.Hq / s.H, Bq = s.Bq, S = s.S;
  const int cpb = s.n / kChunk;
  const int ipt = std::min(Bq, 128 / G);
  const int nrt = (Bq + ipt - 1) / ipt;
  const int nsc = (S + kChunk - 1) / kChunk;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  // atoms in processing order with their byte cost
  struct Atom {
    int type, h, tile, c;
    double cost;
  };
  std::vector<Atom> atoms;
  for (int h = 0; h < H; ++h)
    for (int rt = 0; rt < nrt; ++rt)
      for (int b = 0; b < nb; ++b) {
        const int rk = in.host_ranks[(size_t)(2 * h) * nb + b], rv = in.host_ranks[(size_t)(2 * h + 1) * nb + b];
        // cost in nanoseconds: bytes at ~44 GB/s per SM, plus the fixed time of a chunk (softmax of
        // 128 × 128 scores) and of a block (q̃ and ã round trips through TMEM and smem)
        for (int cc = 0; cc < cpb; ++cc)
          atoms.push_back({0, h, rt, b * cpb + cc,
                           (2.0 * (rk + rv) * kChunk + (cc == 0 ? 2.0 * (rk + rv) * D : 0.0)) / 44.0 + kChunkNs +
                               (cc == 0 ? kBlockNs : 0.0)});
      }
  for (int i = 0; i < Bq; ++i)
    for (int h = 0; h < H; ++h)
      for (int c = 0; c < nsc; ++c)
        atoms.push_back({1, h, i, c, 2.0 * 2.0 * kChunk * D / 44.0 + kChunkNs + (c == 0 ? kUnitNs : 0.0)});
  double total = 0;
  for (auto& a : atoms) total += a.cost;
  const int grid = std::max(1, std::min(sms, (int)atoms.size()));
  std::vector<Seg> segs;
  std::vector<int> seg_first(grid + 1, 0);
  std::vector<int> pre_range(2 * H * nrt, 0), suf_range(2 * Bq * H, 0);
  double cum = 0;
  int cta = 0;
  for (size_t a = 0; a < atoms.size(); ++a) {
    const Atom& at = atoms[a];
    const double mid = cum + 0.5 * at.cost;
    cum += at.cost;
    while (cta + 1 < grid && mid >= total * (cta + 1) / grid) {
      ++cta;
      seg_first[cta] = (int)segs.size();
    }
    const bool cont = !segs.empty() && seg_first[cta] < (int)segs.size() && segs.back().type == at.type &&
                      segs.back().h == at.h && segs.back().tile == at.tile && segs.back().c1 == at.c;
    if (cont) {
      segs.back().c1 = at.c + 1;
    } else {
      Seg sg{};
      sg.type = at.type;
      sg.h = at.h;
      sg.tile = at.tile;
      sg.c0 = at.c;
      sg.c1 = at.c + 1;
      sg.pid = (int)segs.size();
      sg.rows = at.type == 0 ? std::min(ipt, Bq - at.tile * ipt) * G : G;
      segs.push_back(sg);
    }
  }
  for (int k = cta + 1; k <= grid; ++k) seg_first[k] = (int)segs.size();
  // partial ranges per output row group (segments of one (h, tile) / (i, h) are consecutive)
  for (int h = 0; h < H; ++h)
    for (int rt = 0; rt < nrt; ++rt) pre_range[2 * (h * nrt + rt)] = pre_range[2 * (h * nrt + rt) + 1] = -1;
  for (int i = 0; i < Bq; ++i)
    for (int h = 0; h < H; ++h) suf_range[2 * (i * H + h)] = suf_range[2 * (i * H + h) + 1] = 0;
  for (auto& sg : segs) {
    int* r = sg.type == 0 ? &pre_range[2 * (sg.h * nrt + sg.tile)] : &suf_range[2 * (sg.tile * H + sg.h)];
    if (sg.type == 0 && r[0] < 0) r[0] = sg.pid;
    if (sg.type == 1 && r[1] == 0 && r[0] == 0) r[0] = sg.pid;
    r[1] = sg.pid + 1;
  }
  for (int i = 0; i < 2 * H * nrt; ++i)
    if (pre_range[i] < 0) pre_range[i] = 0;
  for (int h = 0; h < H; ++h)
    for (int i = 0; i < Bq; ++i) {
      const int rt = i / ipt;
      const int parts = pre_range[2 * (h * nrt + rt) + 1] - pre_range[2 * (h * nrt + rt)] +
                        suf_range[2 * (i * H + h) + 1] - suf_range[2 * (i * H + h)];
      if (parts > kMaxParts) return cudaErrorInvalidValue;
    }
  pl->off_segs = grid + 1;
  pl->off_pre = pl->off_segs + (int)segs.size() * (int)(sizeof(Seg) / sizeof(int));
  pl->off_suf = pl->off_pre + 2 * H * nrt;
  const int nwords = pl->off_suf + 2 * Bq * H;
  std::vector<int> host(nwords);
  std::copy(seg_first.begin(), seg_first.end(), host.begin());
  std::memcpy(host.data() + pl->off_segs, segs.data(), segs.size() * sizeof(Seg));
  std::copy(pre_range.begin(), pre_range.end(), host.begin() + pl->off_pre);
  std::copy(suf_range.begin(), suf_range.end(), host.begin() + pl->off_suf);
  cudaError_t e;
  if ((e = cudaMalloc((void**)&pl->d_work, nwords * sizeof(int))) != cudaSuccess) return e;
  if ((e = cudaMemcpy(pl->d_work, host.data(), nwords * sizeof(int), cudaMemcpyHostToDevice)) != cudaSuccess)
    return e;
  const size_t np = std::max<size_t>(1, segs.size());
  if ((e = cudaMalloc((void**)&pl->part_acc, np * 128 * D * sizeof(float))) != cudaSuccess) return e;
  if ((e = cudaMalloc((void**)&pl->part_ml, np * 128 * sizeof(float2))) != cudaSuccess) return e;
  pl->Bq = Bq;
  pl->Hq = s.Hq;
  pl->S = S;
  pl->grid = grid;
  pl->nsegs = (int)segs.size();
  pl->ipt = ipt;
  pl->nrt = nrt;
  // factor maps
  const uint64_t rows = (uint64_t)2 * H * in.pool_rows;
  {
    // the token factor as a [rows · n/128][128] array of 128-token slab rows
    const uint64_t dims[2] = {(uint64_t)kChunk, rows * cpb}, st[1] = {(uint64_t)kChunk * 2};
    const uint32_t box[2] = {64, 16};
    if (!make_map(&pl->map_tok, in.tok, 2, dims, st, box)) return cudaErrorInvalidValue;
  }
  {
    const uint64_t dims[2] = {(uint64_t)D, rows}, st[1] = {(uint64_t)D * 2};
    const uint32_t box[2] = {64, 16};
    if (!make_map(&pl->map_dim, in.dim, 2, dims, st, box)) return cudaErrorInvalidValue;
  }
  pl->tok = in.tok;
  pl->dim = in.dim;
  auto kfn = D == 64 ? (const void*)decode_tc_kernel<64> : (const void*)decode_tc_kernel<128>;
  return cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
}

cudaError_t tc_decode(TcPlan** plan, const DecodeShape& s, const TcInputs& in, void* out, cudaStream_t st,
                      cudaEvent_t ev0, cudaEvent_t ev1) {
  TcPlan* pl = *plan;
  if (!pl || pl->Bq != s.Bq || pl->Hq != s.Hq || pl->S != s.S || pl->tok != in.tok) {
    tc_plan_destroy(pl);
    *plan = nullptr;
    pl = new TcPlan();
    cudaError_t e = build_plan(pl, s, in);
    if (e != cudaSuccess) {
      tc_plan_destroy(pl);
      return e;
    }
    *plan = pl;
  }
  const int D = s.d, G = s.Hq / s.H;
  CUtensorMap mq_pre, mq_suf, mk, mv;
  {
    const uint64_t dims[3] = {(uint64_t)D, (uint64_t)s.Hq, (uint64_t)s.Bq};
    const uint64_t strd[2] = {(uint64_t)D * 2, (uint64_t)s.Hq * D * 2};
    const uint32_t box_pre[3] = {64, (uint32_t)G, (uint32_t)pl->ipt};
    const uint32_t box_suf[3] = {64, (uint32_t)G, 1};
    if (!make_map(&mq_pre, in.q, 3, dims, strd, box_pre)) return cudaErrorInvalidValue;
    if (!make_map(&mq_suf, in.q, 3, dims, strd, box_suf)) return cudaErrorInvalidValue;
  }
  if (s.S > 0) {
    const uint64_t dims[2] = {(uint64_t)D, (uint64_t)s.Bq * s.H * s.S}, strd[1] = {(uint64_t)D * 2};
    const uint32_t box[2] = {64, 16};
    if (!make_map(&mk, in.K_suf, 2, dims, strd, box)) return cudaErrorInvalidValue;
    if (!make_map(&mv, in.V_suf, 2, dims, strd, box)) return cudaErrorInvalidValue;
  } else {
    mk = pl->map_dim;
    mv = pl->map_dim;
  }
  Params p;
  p.seg_first = pl->d_work;
  p.segs = reinterpret_cast<const Seg*>(pl->d_work + pl->off_segs);
  p.ranks = in.ranks;
  p.row_offsets = in.row_offsets;
  p.part_acc = pl->part_acc;
  p.part_ml = pl->part_ml;
  p.status = in.status;
  p.nb = s.nb;
  p.cpb = s.n / kChunk;
  p.H = s.H;
  p.G = G;
  p.ipt = pl->ipt;
  p.S = s.S;
  p.c = s.scale * 1.4426950408889634f;
  cudaError_t e;
  if (ev0 && (e = cudaEventRecord(ev0, st)) != cudaSuccess) return e;
  if (D == 64)
    decode_tc_kernel<64><<<pl->grid, kThreads, kSmemBytes, st>>>(pl->map_tok, pl->map_dim, mq_pre, mq_suf, mk, mv, p);
  else
    decode_tc_kernel<128><<<pl->grid, kThreads, kSmemBytes, st>>>(pl->map_tok, pl->map_dim, mq_pre, mq_suf, mk, mv,
                                                                   p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (ev1 && (e = cudaEventRecord(ev1, st)) != cudaSuccess) return e;
  const int* pre = pl->d_work + pl->off_pre;
  const int* suf = pl->d_work + pl->off_suf;
  if (D == 64)
    combine_tc_kernel<64><<<dim3(s.Hq, s.Bq), 64, 0, st>>>(pl->part_acc, pl->part_ml, pre, suf, s.H, s.Hq, pl->ipt,
                                                          pl->nrt, static_cast<__nv_bfloat16*>(out));
  else
    combine_tc_kernel<128><<<dim3(s.Hq, s.Bq), 128, 0, st>>>(pl->part_acc, pl->part_ml, pre, suf, s.H, s.Hq,
                                                            pl->ipt, pl->nrt, static_cast<__nv_bfloat16*>(out));
  return cudaGetLastError();
}


// ================================================================================================
// Decode without allocation: the same kernels, with their scratch (work list and partials) in a
// fixed device array.  See milo_decode_attn_noalloc in milo.h.
// ================================================================================================
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;  // 32 MiB, held by every device that loads us
constexpr int kNoAllocMaxWords = 1 << 18;                  // host-side work-list staging (1 MiB)
constexpr int kNoAllocMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_noalloc_mu;
void* g_noalloc_dev_ptr[kNoAllocMaxDevices];  // device address of g_noalloc_scratch, per device
int g_noalloc_host_words[kNoAllocMaxWords];   // work list staging, guarded by g_noalloc_mu

// Byte-balanced work list as in build_plan, written into `w` without heap allocation.
// Returns the number of words used, or -1 if `cap` words are not enough.
int build_worklist_fixed(const DecodeShape& s, const int32_t* host_ranks, int grid, int* w, int cap, int& nsegs,
                         int& off_segs, int& off_pre, int& off_suf, int& ipt_out, int& nrt_out) {
  const int H = s.H, nb = s.nb, D = s.d, G = s.Hq / s.H, Bq = s.Bq, S = s.S;
  const int cpb = s.n / kChunk;
  const int ipt = std::min(Bq, 128 / G);
  const int nrt = (Bq + ipt - 1) / ipt;
  const int nsc = (S + kChunk - 1) / kChunk;
  const int seg_words = (int)(sizeof(Seg) / sizeof(int));
  auto for_each_atom = [&](auto&& fn) {
    for (int h = 0; h < H; ++h)
      for (int rt = 0; rt < nrt; ++rt)
        for (int b = 0; b < nb; ++b) {
          const int rk = host_ranks[(size_t)(2 * h) * nb + b], rv = host_ranks[(size_t)(2 * h + 1) * nb + b];
          for (int cc = 0; cc < cpb; ++cc)
            fn(0, h, rt, b * cpb + cc,
               (2.0 * (rk + rv) * kChunk + (cc == 0 ? 2.0 * (rk + rv) * D : 0.0)) / 44.0 + kChunkNs +
                   (cc == 0 ? kBlockNs : 0.0));
        }
    for (int i = 0; i < Bq; ++i)
      for (int h = 0; h < H; ++h)
        for (int c = 0; c < nsc; ++c)
          fn(1, h, i, c, 2.0 * 2.0 * kChunk * D / 44.0 + kChunkNs + (c == 0 ? kUnitNs : 0.0));
  };
  double total = 0;
  for_each_atom([&](int, int, int, int, double cost) { total += cost; });
  off_segs = grid + 1;
  if (off_segs > cap) return -1;
  int* seg_first = w;
  Seg* segs = reinterpret_cast<Seg*>(w + off_segs);
  const int max_segs = (cap - off_segs) / seg_words;
  for (int k = 0; k <= grid; ++k) seg_first[k] = 0;
  int n = 0, cta = 0;
  bool overflow = false;
  double cum = 0;
  for_each_atom([&](int type, int h, int tile, int c, double cost) {
    if (overflow) return;
    const double mid = cum + 0.5 * cost;
    cum += cost;
    while (cta + 1 < grid && mid >= total * (cta + 1) / grid) {
      ++cta;
      seg_first[cta] = n;
    }
    if (n > 0 && seg_first[cta] < n && segs[n - 1].type == type && segs[n - 1].h == h && segs[n - 1].tile == tile &&
        segs[n - 1].c1 == c) {
      segs[n - 1].c1 = c + 1;
      return;
    }
    if (n >= max_segs) {
      overflow = true;
      return;
    }
    Seg sg{};
    sg.type = type;
    sg.h = h;
    sg.tile = tile;
    sg.c0 = c;
    sg.c1 = c + 1;
    sg.pid = n;
    sg.rows = type == 0 ? std::min(ipt, Bq - tile * ipt) * G : G;
    segs[n++] = sg;
  });
  if (overflow) return -1;
  for (int k = cta + 1; k <= grid; ++k) seg_first[k] = n;
  off_pre = off_segs + n * seg_words;
  off_suf = off_pre + 2 * H * nrt;
  const int nwords = off_suf + 2 * Bq * H;
  if (nwords > cap) return -1;
  int* pre = w + off_pre;
  int* suf = w + off_suf;
  for (int i = 0; i < 2 * H * nrt; ++i) pre[i] = -1;
  for (int i = 0; i < 2 * Bq * H; ++i) suf[i] = 0;
  for (int q = 0; q < n; ++q) {
    const Seg& sg = segs[q];
    int* r = sg.type == 0 ? &pre[2 * (sg.h * nrt + sg.tile)] : &suf[2 * (sg.tile * H + sg.h)];
    if (sg.type == 0 && r[0] < 0) r[0] = sg.pid;
    if (sg.type == 1 && r[1] == 0 && r[0] == 0) r[0] = sg.pid;
    r[1] = sg.pid + 1;
  }
  for (int i = 0; i < 2 * H * nrt; ++i)
    if (pre[i] < 0) pre[i] = 0;
  for (int h = 0; h < H; ++h)
    for (int i = 0; i < Bq; ++i) {
      const int rt = i / ipt;
      const int parts = pre[2 * (h * nrt + rt) + 1] - pre[2 * (h * nrt + rt)] + suf[2 * (i * H + h) + 1] -
                        suf[2 * (i * H + h)];
      if (parts > kMaxParts) return -1;
    }
  nsegs = n;
  ipt_out = ipt;
  nrt_out = nrt;
  return nwords;
}

}  // namespace

size_t tc_noalloc_scratch_bytes() { return kNoAllocScratchBytes; }

cudaError_t tc_decode_noalloc(const DecodeShape& s, const TcInputs& in, void* out, cudaStream_t st,
                              bool* too_large) {
  *too_large = false;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kNoAllocMaxDevices) return cudaErrorInvalidDevice;
  if (!g_noalloc_dev_ptr[dev]) {
    // once per device, with that device current: host code cannot use the array's name as a device address
    void* ptr = nullptr;
    if ((e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch)) != cudaSuccess) return e;
    g_noalloc_dev_ptr[dev] = ptr;
    auto kfn = s.d == 64 ? (const void*)decode_tc_kernel<64> : (const void*)decode_tc_kernel<128>;
    if ((e = cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes)) != cudaSuccess)
      return e;
  }
  unsigned char* scratch = static_cast<unsigned char*>(g_noalloc_dev_ptr[dev]);
  int sms = 148;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  const int cpb = s.n / kChunk, nsc = (s.S + kChunk - 1) / kChunk;
  const int64_t natoms = (int64_t)s.H * ((s.Bq + std::min(s.Bq, 128 / (s.Hq / s.H)) - 1) /
                                         std::min(s.Bq, 128 / (s.Hq / s.H))) * s.nb * cpb +
                         (int64_t)s.Bq * s.H * nsc;
  const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(sms, natoms));
  int nsegs = 0, off_segs = 0, off_pre = 0, off_suf = 0, ipt = 0, nrt = 0;
  const int nwords = build_worklist_fixed(s, in.host_ranks, grid, g_noalloc_host_words, kNoAllocMaxWords, nsegs,
                                          off_segs, off_pre, off_suf, ipt, nrt);
  const size_t words_bytes = ((size_t)std::max(nwords, 0) * sizeof(int) + 255) & ~(size_t)255;
  const size_t ml_bytes = ((size_t)nsegs * 128 * sizeof(float2) + 255) & ~(size_t)255;
  const size_t acc_bytes = (size_t)nsegs * 128 * s.d * sizeof(float);
  if (nwords < 0 || words_bytes + ml_bytes + acc_bytes > kNoAllocScratchBytes) {
    *too_large = true;
    return cudaErrorInvalidValue;
  }
  int* d_work = reinterpret_cast<int*>(scratch);
  float2* part_ml = reinterpret_cast<float2*>(scratch + words_bytes);
  float* part_acc = reinterpret_cast<float*>(scratch + words_bytes + ml_bytes);
  // pageable source: the call returns once the words are staged, so the host buffer can be reused
  if ((e = cudaMemcpyAsync(d_work, g_noalloc_host_words, (size_t)nwords * sizeof(int), cudaMemcpyHostToDevice, st)) !=
      cudaSuccess)
    return e;
  const int D = s.d, G = s.Hq / s.H;
  CUtensorMap map_tok, map_dim, mq_pre, mq_suf, mk, mv;
  const uint64_t rows = (uint64_t)2 * s.H * in.pool_rows;
  {
    const uint64_t dims[2] = {(uint64_t)kChunk, rows * cpb}, strd[1] = {(uint64_t)kChunk * 2};
    const uint32_t box[2] = {64, 16};
    if (!make_map(&map_tok, in.tok, 2, dims, strd, box)) return cudaErrorInvalidValue;
  }
  {
    const uint64_t dims[2] = {(uint64_t)D, rows}, strd[1] = {(uint64_t)D * 2};
    const uint32_t box[2] = {64, 16};
    if (!make_map(&map_dim, in.dim, 2, dims, strd, box)) return cudaErrorInvalidValue;
  }
  {
    const uint64_t dims[3] = {(uint64_t)D, (uint64_t)s.Hq, (uint64_t)s.Bq};
    const uint64_t strd[2] = {(uint64_t)D * 2, (uint64_t)s.Hq * D * 2};
    const uint32_t box_pre[3] = {64, (uint32_t)G, (uint32_t)ipt};
    const uint32_t box_suf[3] = {64, (uint32_t)G, 1};
    if (!make_map(&mq_pre, in.q, 3, dims, strd, box_pre)) return cudaErrorInvalidValue;
    if (!make_map(&mq_suf, in.q, 3, dims, strd, box_suf)) return cudaErrorInvalidValue;
  }
  if (s.S > 0) {
    const uint64_t dims[2] = {(uint64_t)D, (uint64_t)s.Bq * s.H * s.S}, strd[1] = {(uint64_t)D * 2};
    const uint32_t box[2] = {64, 16};
    if (!make_map(&mk, in.K_suf, 2, dims, strd, box)) return cudaErrorInvalidValue;
    if (!make_map(&mv, in.V_suf, 2, dims, strd, box)) return cudaErrorInvalidValue;
  } else {
    mk = map_dim;
    mv = map_dim;
  }
  Params p;
  p.seg_first = d_work;
  p.segs = reinterpret_cast<const Seg*>(d_work + off_segs);
  p.ranks = in.ranks;
  p.row_offsets = in.row_offsets;
  p.part_acc = part_acc;
  p.part_ml = part_ml;
  p.status = in.status;
  p.nb = s.nb;
  p.cpb = cpb;
  p.H = s.H;
  p.G = G;
  p.ipt = ipt;
  p.S = s.S;
  p.c = s.scale * 1.4426950408889634f;
  if (D == 64)
    decode_tc_kernel<64><<<grid, kThreads, kSmemBytes, st>>>(map_tok, map_dim, mq_pre, mq_suf, mk, mv, p);
  else
    decode_tc_kernel<128><<<grid, kThreads, kSmemBytes, st>>>(map_tok, map_dim, mq_pre, mq_suf, mk, mv, p);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if (D == 64)
    combine_tc_kernel<64><<<dim3(s.Hq, s.Bq), 64, 0, st>>>(part_acc, part_ml, d_work + off_pre, d_work + off_suf,
                                                          s.H, s.Hq, ipt, nrt, static_cast<__nv_bfloat16*>(out));
  else
    combine_tc_kernel<128><<<dim3(s.Hq, s.Bq), 128, 0, st>>>(part_acc, part_ml, d_work + off_pre, d_work + off_suf,
                                                            s.H, s.Hq, ipt, nrt, static_cast<__nv_bfloat16*>(out));
  return cudaGetLastError();
}

}  // namespace milo
