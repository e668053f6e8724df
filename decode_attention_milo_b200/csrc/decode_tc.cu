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

constexpr int kThreads = 192;        // warp 0: TMA producer; warp 1: MMA issuer; warps 2..5: softmax
constexpr int kSigQt = 1, kSigP = 2, kSigAt = 3;  // named barriers: softmax warps → MMA warp
constexpr int kRingBytes = 94208;   // TMA ring: variable-size items, each one contiguous tile
constexpr int kItemSlots = 16;       // items in flight at most (one FULL/EMPTY barrier pair each)
constexpr int kChunk = 128;          // tokens per score chunk
constexpr uint64_t kWaitNs = 1000000000ull;

// shared-memory map (bytes from a 1024-aligned base)
constexpr int kOffQ = 0;          // [cb][128 rows][128 B]  query rows, K-major over d
constexpr int kOffQtHi = 32768;   // [cb][128][128 B]  q̃ high part, K-major over rank
constexpr int kOffQtLo = 65536;   // [cb][128][128 B]  q̃ low part
constexpr int kOffP = 98304;      // [cb][128][128 B]  probabilities (K-major over tokens); then ã for G4
constexpr int kOffRing = 131072;  // kRingBytes of items laid out [64-column block][rows][128 B]
constexpr int kOffBar = kOffRing + kRingBytes;             // 225280: barriers, then the Shared block
constexpr int kBarRegion = 4096;
constexpr int kSmemBytes = kOffBar + kBarRegion + 1024;     // + alignment slack (230400)
constexpr uint32_t kTileCb = 16384;  // column-block stride of a 128-row tile
constexpr int kMaxSegsSmem = 16, kMaxBlocksSmem = 64;  // per-CTA work tables staged in smem

// TMEM columns: acc [0,128), two S slots [128,256) and [256,384) (q̃ of a block also passes through
// an S slot), ã [384,512)
constexpr uint32_t kTmAcc = 0, kTmS0 = 128, kTmA = 384;

enum Bar {
  B_FULL = 0,
  B_EMPTY = B_FULL + kItemSlots,
  B_QFULL = B_EMPTY + kItemSlots,
  B_QEMPTY,
  B_SFULL,
  B_PEMPTY = B_SFULL + 2,
  B_ATFULL,
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

struct BlockInfo {
  int rk, rv;
  int64_t rowk, rowv;
};

// Per-CTA state in shared memory: the CTA's segments and the rank / row offset of every block they
// touch, staged once at start so that no role reads them from global memory inside the pipeline.
struct Shared {
  uint32_t tmem_base;
  int abort_flag;
  int nseg;        // segments of this CTA staged (0 when they did not fit: roles read global memory)
  int nblk;        // blocks staged
  int blk0[kMaxSegsSmem + 1];  // first table entry of each segment
  Seg segs[kMaxSegsSmem];
  BlockInfo blocks[kMaxBlocksSmem];
  uint32_t pos_log[kItemSlots], len_log[kItemSlots];  // producer's record of the items in flight
};
static_assert(8 * B_COUNT + 64 + sizeof(Shared) <= kBarRegion, "barrier region too small");

// Warp-collective bounded wait on an mbarrier phase (all 32 lanes call it together; the result is uniform).
// Gives up after kWaitNs, records kStatusDecodeTimeout and raises the CTA's abort flag, or returns false at
// once when another role already aborted.  `drain` waits ignore the abort flag (used to let the CTA's own
// copies and MMAs land before it exits) but keep the time limit.
__device__ __noinline__ bool wait_bar_slow(uint32_t bar, uint32_t parity, Shared* sh, uint32_t* status,
                                           bool drain) {
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

__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, Shared* sh, uint32_t* status,
                                         bool drain = false) {
  if (__all_sync(0xffffffffu, ptx::mbar_try_wait(bar, parity))) return true;
  return wait_bar_slow(bar, parity, sh, status, drain);
}

__device__ __forceinline__ int pad16(int r) { return (r + 15) & ~15; }

__device__ __forceinline__ bool block_info(const Params& p, int h, int b, int D, BlockInfo& bi) {
  bi.rk = p.ranks[(int64_t)(2 * h) * p.nb + b];
  bi.rv = p.ranks[(int64_t)(2 * h + 1) * p.nb + b];
  bi.rowk = p.row_offsets[(int64_t)(2 * h) * (p.nb + 1) + b];
  bi.rowv = p.row_offsets[(int64_t)(2 * h + 1) * (p.nb + 1) + b];
  return bi.rk >= 1 && bi.rk <= D && bi.rv >= 1 && bi.rv <= D;
}

// Block `k` (0-based, in walk order) of segment `si` of this CTA: from the smem table when staged.
__device__ __forceinline__ bool seg_block(const Params& p, const Shared* sh, int si_local, int k, int h, int b, int D,
                                          BlockInfo& bi) {
  if (sh->nseg > 0) {
    bi = sh->blocks[sh->blk0[si_local] + k];
    return bi.rk >= 1 && bi.rk <= D && bi.rv >= 1 && bi.rv <= D;
  }
  return block_info(p, h, b, D, bi);
}
__device__ __forceinline__ Seg get_seg(const Params& p, const Shared* sh, int s_begin, int si) {
  return sh->nseg > 0 ? sh->segs[si - s_begin] : p.segs[si];
}

// Placement of items in the TMA ring.  Producer and consumer call place() with the same sizes in the same
// order, so they agree on every item's offset without exchanging it; an item that does not fit before the
// end of the ring starts at offset 0.
struct RingPlace {
  uint32_t head = 0;  // next free byte offset
  uint32_t n = 0;     // items placed so far
  __device__ uint32_t place(uint32_t bytes) {
    const uint32_t pos = head + bytes <= (uint32_t)kRingBytes ? head : 0u;
    head = pos + bytes;
    ++n;
    return pos;
  }
};

// Block range of a prefix segment: chunks [c0, c1) cover blocks c0/cpb .. (c1-1)/cpb.
struct BlockWalk {
  int c, c1, cpb;
  __device__ int block() const { return c / cpb; }
  __device__ int chunks() const { return min(c1, (c / cpb + 1) * cpb) - c; }  // chunks of this block here
  __device__ int first_cc() const { return c - (c / cpb) * cpb; }            // chunk index inside the block
  __device__ bool has_next() const { return c + chunks() < c1; }
  __device__ void next() { c += chunks(); }
};

// -------------------------------------------------------------------------------------------- producer
template <int D>
struct Producer {
  static constexpr int NCB = D / 64;
  uint32_t base;
  RingPlace ring;
  uint32_t oldest = 0;  // first item not yet known to be released
  uint32_t q_uses = 0;
  Shared* sh;
  uint32_t* status;
  uint32_t* pos_log;  // [kItemSlots] offsets of the items in flight (smem, producer only)
  uint32_t* len_log;  // [kItemSlots] their sizes

  __device__ uint32_t bar(int i) const { return base + kOffBar + 8 * i; }

  // Waits until the oldest item in flight has been consumed and forgets it.
  __device__ bool retire_oldest() {
    const uint32_t j = oldest;
    if (!wait_bar(bar(B_EMPTY + j % kItemSlots), (j / kItemSlots) & 1, sh, status)) return false;
    ++oldest;
    return true;
  }

  // `rows` (multiple of 16, <= 128) rows × `ncb` 64-column blocks of a 2D map at (x0, y0) → one item,
  // laid out [cb][rows][128 B].
  __device__ bool item(const CUtensorMap* m, int x0, int64_t y0, int rows, int ncb) {
    const uint32_t bytes = (uint32_t)rows * 128u * ncb;
    const uint32_t i = ring.n;
    const uint32_t pos = ring.place(bytes);
    // free the space: retire the oldest items while any item in flight overlaps it (after a wrap a newer
    // item can overlap while the oldest does not), and keep at most kItemSlots in flight
    while (oldest < i) {
      bool busy = i - oldest >= (uint32_t)kItemSlots;
      for (uint32_t j = oldest; j < i && !busy; ++j) {
        const uint32_t k = j % kItemSlots;
        busy = pos < pos_log[k] + len_log[k] && pos_log[k] < pos + bytes;
      }
      if (!busy) break;
      if (!retire_oldest()) return false;
    }
    pos_log[i % kItemSlots] = pos;
    len_log[i % kItemSlots] = bytes;
    const uint32_t dst = base + kOffRing + pos;
    const uint32_t fb = bar(B_FULL + i % kItemSlots);
    if ((threadIdx.x & 31) == 0) {
      ptx::mbar_arrive_expect_tx(fb, bytes);
      for (int cb = 0; cb < ncb; ++cb)
        for (int k = 0; k < rows; k += 16)
          ptx::tma_load_2d(dst + cb * rows * 128 + k * 128, m, fb, x0 + 64 * cb, (int)(y0 + k));
    }
    __syncwarp();
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
// Offset, in descriptor units (16 B), of k-step k of a K-major operand whose column blocks are `cbs` apart.
__device__ __forceinline__ uint64_t kstep(int k, uint32_t cbs) {
  return (uint64_t)(((uint32_t)(k >> 2) * cbs + (uint32_t)(k & 3) * 32) >> 4);
}
// MN-major SW128 descriptor of an item [cb][rows][128 B]: k-step k (16 rows) starts 2048 B further.
__device__ __forceinline__ uint64_t mndesc(uint32_t item, int k, uint32_t cbs) {
  return ptx::sw128_desc(item + (uint32_t)k * 2048, cbs, 1024);
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
    for (int i = 0; i < kItemSlots; ++i) {
      ptx::mbar_init(bar(B_FULL + i), 1);
      ptx::mbar_init(bar(B_EMPTY + i), 1);
    }
    ptx::mbar_init(bar(B_QFULL), 1);
    ptx::mbar_init(bar(B_QEMPTY), 1);
    ptx::mbar_init(bar(B_SFULL), 1);
    ptx::mbar_init(bar(B_SFULL + 1), 1);
    ptx::mbar_init(bar(B_PEMPTY), 1);
    ptx::mbar_init(bar(B_ATFULL), 1);
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
  const int s_begin = p.seg_first[blockIdx.x], s_end = p.seg_first[blockIdx.x + 1];
  // stage this CTA's segments and the rank / row offsets of their blocks in shared memory
  const int nseg_here = s_end - s_begin;
  const bool stage_tables = nseg_here <= kMaxSegsSmem;
  if (stage_tables && (int)threadIdx.x < nseg_here) sh->segs[threadIdx.x] = p.segs[s_begin + threadIdx.x];
  __syncthreads();
  if (threadIdx.x == 0) {
    int nblk = 0;
    for (int i = 0; i < (stage_tables ? nseg_here : 0); ++i) {
      sh->blk0[i] = nblk;
      const Seg& sg = sh->segs[i];
      if (sg.type == 0) nblk += (sg.c1 - 1) / p.cpb - sg.c0 / p.cpb + 1;
    }
    sh->blk0[stage_tables ? nseg_here : 0] = nblk;
    const bool fits = stage_tables && nblk <= kMaxBlocksSmem;
    sh->nblk = fits ? nblk : 0;
    sh->nseg = fits ? nseg_here : 0;
  }
  __syncthreads();
  for (int t = threadIdx.x; t < sh->nblk; t += kThreads) {
    int i = 0;
    while (sh->blk0[i + 1] <= t) ++i;
    const Seg& sg = sh->segs[i];
    BlockInfo bi;
    block_info(p, sg.h, sg.c0 / p.cpb + (t - sh->blk0[i]), D, bi);
    sh->blocks[t] = bi;
  }
  ptx::fence_async_smem();
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = sh->tmem_base;

  if (warp == 0) {
    // ==================================================================== TMA producer
    // Loads items in exactly the order the issuing warp consumes them (see the softmax section).
    Producer<D> pr;
    pr.base = base;
    pr.sh = sh;
    pr.status = p.status;
    pr.pos_log = sh->pos_log;
    pr.len_log = sh->len_log;
    bool ok = true;
    auto bad_block = [&]() {
      atomicOr(p.status, kStatusDecodeBounds);
      sh->abort_flag = 1;
      return false;
    };
    // token-factor slab of chunk cc (index inside the block) of a block: rows [row0·cpb + cc·r, +r)
    auto tok_item = [&](int64_t row0, int r, int cc) {
      return pr.item(&map_tok, 0, row0 * p.cpb + (int64_t)cc * r, pad16(r), 2);
    };
    auto dim_item = [&](int64_t row0, int r) { return pr.item(&map_dim, 0, row0, pad16(r), NCB); };
    for (int si = s_begin; si < s_end && ok; ++si) {
      const Seg sg = get_seg(p, sh, s_begin, si);
      if (sg.type == 0) {
        ok = pr.q_tile(&map_qpre, sg.h * p.G, sg.tile * p.ipt, p.G * p.ipt);
        BlockWalk w{sg.c0, sg.c1, p.cpb};
        BlockInfo bi, bn, prev;
        bool have_prev = false;
        int kb = 0;
        if (ok && !seg_block(p, sh, si - s_begin, kb, sg.h, w.block(), D, bi)) ok = bad_block();
        if (ok) ok = dim_item(bi.rowk, bi.rk);  // B_K of the first block
        while (ok) {
          const int n = w.chunks(), cc0 = w.first_cc();
          const bool next = w.has_next();
          if (next && !seg_block(p, sh, si - s_begin, kb + 1, sg.h, w.block() + 1, D, bn)) ok = bad_block();
          if (ok) ok = tok_item(bi.rowk, bi.rk, cc0);                       // U(0)
          if (ok && n >= 2) ok = tok_item(bi.rowk, bi.rk, cc0 + 1);         // U(1)
          else if (ok && next) ok = dim_item(bn.rowk, bn.rk);               // B_K(next)
          if (ok && have_prev) ok = dim_item(prev.rowv, prev.rv);           // Q_V(previous block)
          for (int j = 0; j < n && ok; ++j) {
            ok = tok_item(bi.rowv, bi.rv, cc0 + j);                         // P(j)
            if (ok && j + 2 < n) ok = tok_item(bi.rowk, bi.rk, cc0 + j + 2);  // U(j+2)
            else if (ok && j + 2 == n && next) ok = dim_item(bn.rowk, bn.rk);  // B_K(next)
          }
          if (!ok || !next) break;
          prev = bi;
          have_prev = true;
          w.next();
          bi = bn;
          ++kb;
        }
        if (ok) ok = dim_item(bi.rowv, bi.rv);  // Q_V of the last block
      } else {
        ok = pr.q_tile(&map_qsuf, sg.h * p.G, sg.tile, p.G);
        const int64_t row0 = ((int64_t)sg.tile * p.H + sg.h) * p.S;
        const int n = sg.c1 - sg.c0;
        auto kv = [&](const CUtensorMap* m, int j) {
          return pr.item(m, 0, row0 + (int64_t)(sg.c0 + j) * kChunk, kChunk, NCB);
        };
        if (ok) ok = kv(&map_ksuf, 0);
        if (ok && n >= 2) ok = kv(&map_ksuf, 1);
        for (int j = 0; j < n && ok; ++j) {
          ok = kv(&map_vsuf, j);
          if (ok && j + 2 < n) ok = kv(&map_ksuf, j + 2);
        }
      }
    }
    // drain: every copy this warp issued must have landed before the CTA exits
    for (uint32_t j = pr.oldest; j < pr.ring.n; ++j)
      wait_bar(bar(B_FULL + j % kItemSlots), (j / kItemSlots) & 1, sh, p.status, true);
    if (pr.q_uses) wait_bar(bar(B_QFULL), (pr.q_uses - 1) & 1, sh, p.status, true);
  } else if (warp == 1) {
    // ==================================================================== MMA issuer (warp 1)
    // Issues the tensor-core MMAs when the softmax warps signal (named barriers: q̃ ready, P ready, ã ready)
    // that the smem operands they produce are complete, so issuing overlaps the next softmax step.
    const bool leader = lane == 0;
    bool ok = true;
    auto sync_wg = [&](int id) {  // wait for the softmax warps' signal `id`
      asm volatile("bar.sync %0, 160;" ::"r"(id) : "memory");
      ptx::tc_fence_after();
    };
    // ---------------- MMA issue (warp 1 only)
    RingPlace ring;          // consumer view of the TMA ring
    uint32_t cur = 0;        // item being consumed
    uint32_t sidx_i = 0;     // S-slot uses issued
    uint32_t q_uses = 0;
    auto take = [&](int rows, int ncb, uint32_t& addr) -> bool {
      cur = ring.n;
      const uint32_t pos = ring.place((uint32_t)rows * 128u * ncb);
      if (!wait_bar(bar(B_FULL + cur % kItemSlots), (cur / kItemSlots) & 1, sh, p.status)) return false;
      ptx::tc_fence_after();
      addr = base + kOffRing + pos;
      return true;
    };
    auto release = [&]() {  // the item's space is free once the MMAs issued so far have read it
      if (leader) ptx::umma_commit(bar(B_EMPTY + cur % kItemSlots));
    };
    constexpr uint32_t idS = ptx::idesc_bf16(128, 128, false, true);
    constexpr uint32_t idD = ptx::idesc_bf16(128, D, false, true);
    auto s_commit = [&]() {
      if (leader) ptx::umma_commit(bar(B_SFULL + (sidx_i & 1)));
      ++sidx_i;
    };
    // G1: q̃ = Q · B_b into the next S slot, N = padded rank
    auto g1 = [&](int rk) -> bool {
      const int rp = pad16(rk);
      uint32_t it;
      if (!take(rp, NCB, it)) return false;
      if (leader) {
        const uint64_t db = kdesc(it, 0, 0);
        const uint32_t cbs = (uint32_t)rp * 128u, id = ptx::idesc_bf16(128, rp, false, false);
        const uint32_t d = tmem + kTmS0 + 128 * (sidx_i & 1);
#pragma unroll 1
        for (int k = 0; k < D / 16; ++k) ptx::umma_bf16(d, kdesc(base + kOffQ, 0, kTileCb) + kstep(k, kTileCb), db + kstep(k, cbs), id, k > 0);
      }
      release();
      s_commit();
      return true;
    };
    // G2: S = q̃_hi·U + q̃_lo·U into the next S slot (B MN-major, N = 128 tokens)
    auto g2 = [&](int rk) -> bool {
      const int rp = pad16(rk);
      uint32_t it;
      if (!take(rp, 2, it)) return false;
      if (leader) {
        const uint32_t d = tmem + kTmS0 + 128 * (sidx_i & 1);
        const uint64_t db = mndesc(it, 0, (uint32_t)rp * 128u);
        for (int t = 0; t < rp / 16; ++t) {
          const uint64_t bd = db + (uint64_t)(t * 128);
          ptx::umma_bf16(d, kdesc(base + kOffQtHi, 0, kTileCb) + kstep(t, kTileCb), bd, idS, t > 0);
          ptx::umma_bf16(d, kdesc(base + kOffQtLo, 0, kTileCb) + kstep(t, kTileCb), bd, idS, 1);
        }
      }
      release();
      s_commit();
      return true;
    };
    // G3: ã (+)= p · P_b, N = padded rank; `fresh` overwrites ã
    auto g3 = [&](int rv, bool fresh) -> bool {
      const int rp = pad16(rv);
      uint32_t it;
      if (!take(rp, 2, it)) return false;
      if (leader) {
        const uint64_t db = kdesc(it, 0, 0);
        const uint32_t cbs = (uint32_t)rp * 128u, id = ptx::idesc_bf16(128, rp, false, false);
#pragma unroll 1
        for (int t = 0; t < kChunk / 16; ++t)
          ptx::umma_bf16(tmem + kTmA, kdesc(base + kOffP, 0, kTileCb) + kstep(t, kTileCb), db + kstep(t, cbs), id, (t > 0 || !fresh) ? 1u : 0u);
      }
      release();
      return true;
    };
    // G4: acc (+)= ã · Q_bᵀ, ã in the P buffer, B MN-major, N = d
    auto g4 = [&](int rv, bool fresh) -> bool {
      const int rp = pad16(rv);
      uint32_t it;
      if (!take(rp, NCB, it)) return false;
      if (leader) {
        const uint64_t db = mndesc(it, 0, (uint32_t)rp * 128u);
        for (int t = 0; t < rp / 16; ++t)
          ptx::umma_bf16(tmem + kTmAcc, kdesc(base + kOffP, 0, kTileCb) + kstep(t, kTileCb), db + (uint64_t)(t * 128), idD,
                         (t > 0 || !fresh) ? 1u : 0u);
      }
      release();
      return true;
    };
    // G2' (suffix): S = q · K_sufᵀ, B K-major over d, N = 128 tokens
    auto g2s = [&]() -> bool {
      uint32_t it;
      if (!take(kChunk, NCB, it)) return false;
      if (leader) {
        const uint64_t db = kdesc(it, 0, 0);
        const uint32_t d = tmem + kTmS0 + 128 * (sidx_i & 1), id = ptx::idesc_bf16(128, kChunk, false, false);
#pragma unroll
        for (int t = 0; t < D / 16; ++t) ptx::umma_bf16(d, kdesc(base + kOffQ, 0, kTileCb) + kstep(t, kTileCb), db + kstep(t, kChunk * 128u), id, t > 0);
      }
      release();
      s_commit();
      return true;
    };
    // G3' (suffix): acc (+)= p · V_suf, B MN-major, K = 128 tokens, N = d
    auto g3s = [&](bool fresh) -> bool {
      uint32_t it;
      if (!take(kChunk, NCB, it)) return false;
      if (leader) {
        const uint64_t db = mndesc(it, 0, kChunk * 128u);
#pragma unroll
        for (int t = 0; t < kChunk / 16; ++t)
          ptx::umma_bf16(tmem + kTmAcc, kdesc(base + kOffP, 0, kTileCb) + kstep(t, kTileCb), db + (uint64_t)(t * 128), idD,
                         (t > 0 || !fresh) ? 1u : 0u);
      }
      release();
      return true;
    };
    auto commit = [&](int b) {
      if (leader) ptx::umma_commit(bar(b));
    };
    auto wait_q = [&]() -> bool {
      const bool r = wait_bar(bar(B_QFULL), q_uses & 1, sh, p.status);
      ++q_uses;
      ptx::tc_fence_after();
      return r;
    };
    bool bounds_ok = true;
    for (int si = s_begin; si < s_end && bounds_ok; ++si) {
      const Seg sg = get_seg(p, sh, s_begin, si);
      if (sg.type == 0) {
        BlockWalk w{sg.c0, sg.c1, p.cpb};
        BlockInfo bi, bn, prev;
        int kb = 0;
        bool have_prev = false;
        if (!seg_block(p, sh, si - s_begin, kb, sg.h, w.block(), D, bi)) {
          bounds_ok = false;
          break;
        }
        if (ok) {
          ok = wait_q() && g1(bi.rk);
          if (ok && !w.has_next()) commit(B_QEMPTY);  // last read of Q in this segment
        }
        while (true) {
          const int n = w.chunks();
          const bool next = w.has_next();
          bool next_is_last = false;
          if (next) {
            if (!seg_block(p, sh, si - s_begin, kb + 1, sg.h, w.block() + 1, D, bn)) {
              bounds_ok = false;
              break;
            }
            BlockWalk w2 = w;
            w2.next();
            next_is_last = !w2.has_next();
          }
          auto g1_next = [&]() -> bool {
            if (!g1(bn.rk)) return false;
            if (next_is_last) commit(B_QEMPTY);
            return true;
          };
          sync_wg(kSigQt);
          if (ok) {
            ok = g2(bi.rk);
            if (ok && n >= 2) ok = g2(bi.rk);
            else if (ok && next) ok = g1_next();
          }
          if (have_prev) {
            sync_wg(kSigAt);
            if (ok) {
              ok = g4(prev.rv, kb == 1);
              commit(B_PEMPTY);
            }
          }
          for (int j = 0; j < n; ++j) {
            sync_wg(kSigP);
            if (ok) {
              ok = g3(bi.rv, j == 0);
              commit(j + 1 < n ? B_PEMPTY : B_ATFULL);
              if (ok && j + 2 < n) ok = g2(bi.rk);
              else if (ok && j + 2 == n && next) ok = g1_next();
            }
          }
          if (!next) break;
          prev = bi;
          have_prev = true;
          w.next();
          bi = bn;
          ++kb;
        }
        if (!bounds_ok) break;
        sync_wg(kSigAt);
        if (ok) {
          ok = g4(bi.rv, kb == 0);
          commit(B_PEMPTY);
          commit(B_ACCFULL);
        }
      } else {
        const int n = sg.c1 - sg.c0;
        if (ok) {
          ok = wait_q() && g2s();
          if (ok && n >= 2) ok = g2s();
          if (ok && n <= 2) commit(B_QEMPTY);
        }
        for (int j = 0; j < n; ++j) {
          sync_wg(kSigP);
          if (ok) {
            ok = g3s(j == 0);
            commit(B_PEMPTY);
            if (ok && j + 2 < n) {
              ok = g2s();
              if (ok && j + 2 == n - 1) commit(B_QEMPTY);
            }
          }
        }
        if (ok) commit(B_ACCFULL);
      }
    }
    // drain: every MMA issued must complete before TMEM is freed
    commit(B_FINAL);
    __syncwarp();
    wait_bar(bar(B_FINAL), 0, sh, p.status, true);
  } else {
    // ==================================================================== softmax warpgroup (warps 2..5)
    // One thread per row and TMEM lane; signals the MMA warp through named barriers when its smem output
    // (q̃, P or ã) is complete.
    const int quarter = warp & 3;
    const int row = 32 * quarter + lane;
    const uint32_t tl = tmem + ((uint32_t)(32 * quarter) << 16);
    uint32_t sidx = 0, pk = 0, at_uses = 0, acc_uses = 0;  // consumption counters
    bool ok = true;
    auto signal = [&](int id) {  // arrive on the MMA warp's named barrier `id` (does not wait)
      ptx::tc_fence_before();
      asm volatile("bar.arrive %0, 160;" ::"r"(id) : "memory");
    };
    // ---------------- softmax helpers (all four warps)
    // q̃ of a block (fp32, in the next S slot) → bf16 hi + lo in smem, columns >= r zeroed
    // Every helper below ends with the warpgroup barrier, also after a failed wait, so that the four warps
    // always execute the same sequence of named barriers (which have no time limit).
    auto convert_qt = [&](bool active, int rk) -> bool {
      if (!wait_bar(bar(B_SFULL + (sidx & 1)), (sidx >> 1) & 1, sh, p.status)) {
        ++sidx;
        signal(kSigQt);
        return false;
      }
      ptx::tc_fence_after();
      const uint32_t src = tl + kTmS0 + 128 * (sidx & 1);
      if (active) {
        for (int c16 = 0; c16 < pad16(rk); c16 += 16) {
          float v[16];
          ptx::tmem_ld16(src + c16, v);
          ptx::tmem_wait_ld();
          uint32_t hi[8], lo[8];
#pragma unroll
          for (int e = 0; e < 16; e += 2) {
            const float a = (c16 + e < rk) ? v[e] : 0.f;
            const float b2 = (c16 + e + 1 < rk) ? v[e + 1] : 0.f;
            const uint32_t h2 = ptx::pack_bf16(a, b2);
            hi[e / 2] = h2;
            lo[e / 2] = ptx::pack_bf16(a - __uint_as_float(h2 << 16), b2 - __uint_as_float(h2 & 0xFFFF0000u));
          }
          st_tile8(base + kOffQtHi, row, c16, hi[0], hi[1], hi[2], hi[3]);
          st_tile8(base + kOffQtHi, row, c16 + 8, hi[4], hi[5], hi[6], hi[7]);
          st_tile8(base + kOffQtLo, row, c16, lo[0], lo[1], lo[2], lo[3]);
          st_tile8(base + kOffQtLo, row, c16 + 8, lo[4], lo[5], lo[6], lo[7]);
        }
        ptx::fence_async_smem();
      }
      ++sidx;
      signal(kSigQt);
      return true;
    };
    // ã (fp32, TMEM) → bf16 in the P buffer (its last reader, G3, has completed), columns >= r zeroed
    auto convert_at = [&](bool active, int rv) -> bool {
      if (!wait_bar(bar(B_ATFULL), at_uses & 1, sh, p.status)) {
        ++at_uses;
        signal(kSigAt);
        return false;
      }
      ++at_uses;
      ptx::tc_fence_after();
      if (active) {
        for (int c16 = 0; c16 < pad16(rv); c16 += 16) {
          float v[16];
          ptx::tmem_ld16(tl + kTmA + c16, v);
          ptx::tmem_wait_ld();
          uint32_t wv[8];
#pragma unroll
          for (int e = 0; e < 16; e += 2)
            wv[e / 2] = ptx::pack_bf16(c16 + e < rv ? v[e] : 0.f, c16 + e + 1 < rv ? v[e + 1] : 0.f);
          st_tile8(base + kOffP, row, c16, wv[0], wv[1], wv[2], wv[3]);
          st_tile8(base + kOffP, row, c16 + 8, wv[4], wv[5], wv[6], wv[7]);
        }
        ptx::fence_async_smem();
      }
      signal(kSigAt);
      return true;
    };
    // one chunk of scores: online softmax, probabilities into the P buffer.  `rescale_at` / `rescale_acc`
    // say whether ã / acc hold earlier chunks that a grown running max must rescale.
    auto chunk = [&](bool active, int valid, bool& first_chunk, float& m_used, float& l, bool rescale_at,
                     int rvp, bool rescale_acc) -> bool {
      const uint32_t slot = sidx & 1;
      if (!wait_bar(bar(B_SFULL + slot), (sidx >> 1) & 1, sh, p.status)) {
        ++sidx;
        ++pk;
        signal(kSigP);
        return false;
      }
      ptx::tc_fence_after();
      ++sidx;
      const uint32_t src = tl + kTmS0 + 128 * slot;
      float alpha = 1.f;
      bool grow = false;
      if (active) {
        // pass 1 over the scores (32 columns at a time, compact loop): the chunk's row max
        float m8[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) m8[e] = -INFINITY;
#pragma unroll 1
        for (int c32 = 0; c32 < kChunk; c32 += 32) {
          float s[32];
          ptx::tmem_ld32(src + c32, s);
          ptx::tmem_wait_ld();
#pragma unroll
          for (int t = 0; t < 32; t += 8)
#pragma unroll
            for (int e = 0; e < 8; ++e) m8[e] = fmaxf(m8[e], c32 + t + e < valid ? s[t + e] : -INFINITY);
        }
        float mx = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])), fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
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
      if (pk > 0) {
        // the previous chunk's G3 (or the previous block's G4, which read ã from the P buffer) has landed
        if (!wait_bar(bar(B_PEMPTY), (pk - 1) & 1, sh, p.status)) {
          ++pk;
          signal(kSigP);
          return false;
        }
        ptx::tc_fence_after();
      }
      if (__any_sync(0xffffffffu, grow)) {
        // rare: rescale what this warp's rows accumulated so far (alpha = 1 for rows that did not grow)
        if (rescale_at) {
          for (int c16 = 0; c16 < rvp; c16 += 16) {
            float v[16];
            ptx::tmem_ld16(tl + kTmA + c16, v);
            ptx::tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 16; ++e) v[e] *= alpha;
            ptx::tmem_st16(tl + kTmA + c16, v);
          }
        }
        if (rescale_acc) {
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
      if (active) {
        // pass 2: p = exp2(S·c − m) as bf16 into the P buffer, row sum in fp32 (32 columns at a time)
        float ls[4] = {0.f, 0.f, 0.f, 0.f};  // independent partial row sums
#pragma unroll 1
        for (int c32 = 0; c32 < kChunk; c32 += 32) {
          float s[32];
          ptx::tmem_ld32(src + c32, s);
          ptx::tmem_wait_ld();
#pragma unroll
          for (int g8 = 0; g8 < 4; ++g8) {
            uint32_t wv[4];
#pragma unroll
            for (int e = 0; e < 8; e += 2) {
              const int t = c32 + 8 * g8 + e;
              const float a = t < valid ? ptx::ex2(fmaf(s[8 * g8 + e], p.c, -m_used)) : 0.f;
              const float b2 = t + 1 < valid ? ptx::ex2(fmaf(s[8 * g8 + e + 1], p.c, -m_used)) : 0.f;
              ls[e / 2] += a + b2;
              wv[e / 2] = ptx::pack_bf16(a, b2);
            }
            st_tile8(base + kOffP, row, c32 + 8 * g8, wv[0], wv[1], wv[2], wv[3]);
          }
        }
        l += (ls[0] + ls[1]) + (ls[2] + ls[3]);
        ptx::fence_async_smem();
      }
      ++pk;
      signal(kSigP);
      return true;
    };
    auto write_partial = [&](const Seg& sg, bool active, float m_used, float l) -> bool {
      if (!wait_bar(bar(B_ACCFULL), acc_uses & 1, sh, p.status)) {
        ++acc_uses;
        return false;
      }
      ++acc_uses;
      ptx::tc_fence_after();
      if (active) {
        float* dst = p.part_acc + ((int64_t)sg.pid * 128 + row) * D;
        for (int c16 = 0; c16 < D; c16 += 16) {
          float v[16];
          ptx::tmem_ld16(tl + kTmAcc + c16, v);
          ptx::tmem_wait_ld();
          if (row < sg.rows) {
#pragma unroll
            for (int e = 0; e < 16; e += 4)
              *reinterpret_cast<float4*>(dst + c16 + e) = make_float4(v[e], v[e + 1], v[e + 2], v[e + 3]);
          }
        }
        if (row < sg.rows) p.part_ml[(int64_t)sg.pid * 128 + row] = make_float2(m_used, l);
      }
      // acc is read before any MMA of the next segment writes it: those follow a later signal
      return true;
    };
    auto fail_bounds = [&]() {
      if (warp == 2 && lane == 0) atomicOr(p.status, kStatusDecodeBounds);
      sh->abort_flag = 1;
      return false;
    };

    // The loops below depend only on the work list, never on `ok`: after a failure (an expired wait, which
    // also raises the CTA's abort flag so that later waits return at once) the warps still walk the same
    // steps and barriers, skipping the work, and then leave together.
    bool bounds_ok = true;
    for (int si = s_begin; si < s_end && bounds_ok; ++si) {
      const Seg sg = get_seg(p, sh, s_begin, si);
      const bool active = 32 * quarter < sg.rows;  // a warp whose rows are all padding keeps the protocol only
      float m_used = -INFINITY, l = 0.f;
      bool first_chunk = true;
      if (sg.type == 0) {
        BlockWalk w{sg.c0, sg.c1, p.cpb};
        BlockInfo bi, bn, prev;
        int kb = 0;
        bool have_prev = false;
        if (!seg_block(p, sh, si - s_begin, kb, sg.h, w.block(), D, bi)) {
          bounds_ok = fail_bounds();
          break;
        }
        while (true) {
          const int n = w.chunks();
          const bool next = w.has_next();
          bool next_is_last = false;
          if (next) {
            if (!seg_block(p, sh, si - s_begin, kb + 1, sg.h, w.block() + 1, D, bn)) {
              bounds_ok = fail_bounds();
              break;
            }
            BlockWalk w2 = w;
            w2.next();
            next_is_last = !w2.has_next();
          }
          // q̃ of this block to smem, then the first two S-slot uses
          ok = convert_qt(active, bi.rk) && ok;
          // the previous block's ã to smem and its expansion G4
          if (have_prev) {
            ok = convert_at(active, prev.rv) && ok;
          }
          for (int j = 0; j < n; ++j) {
            ok = chunk(active, kChunk, first_chunk, m_used, l, j > 0, pad16(bi.rv), have_prev) && ok;
          }
          if (!next) break;
          prev = bi;
          have_prev = true;
          w.next();
          bi = bn;
          ++kb;
        }
        if (!bounds_ok) break;
        // the last block's ã and G4, then the segment's result
        ok = convert_at(active, bi.rv) && ok;
        ok = write_partial(sg, active, m_used, l) && ok;
      } else {
        const int n = sg.c1 - sg.c0;
        for (int j = 0; j < n; ++j) {
          const int valid = min(kChunk, p.S - (sg.c0 + j) * kChunk);
          ok = chunk(active, valid, first_chunk, m_used, l, false, 0, j > 0) && ok;
        }
        ok = write_partial(sg, active, m_used, l) && ok;
      }
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
