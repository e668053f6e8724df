// Rank-space decode attention over per-block low-rank factors on the sm_100a tensor cores.
//
// Page "MILO: Efficient Many-shot In-Context Learning with Block-wise Low-rank
// Compression", §4.4: at inference the stored low-rank caches are attended.
// With K_b ≈ U_b·B_bᵀ and V_b ≈ P_b·Q_bᵀ (tok rows = U_bᵀ / P_bᵀ, dim rows =
// B_bᵀ / Q_bᵀ), for the query rows of one KV head (batch × GQA group, M = 128):
//   G1  q̃  = Q · B_b                  TMEM fp32, then split into bf16 hi + lo in smem
//   G2  S   = q̃ · U_bᵀ                per 128-token chunk, two MMAs (hi, lo) per k-step
//       p   = exp2(S·scale·log2e − m)  online softmax on the CUDA cores, packed bf16 back into TMEM
//   G3  ã  += p · P_b                 A operand p read from TMEM, fp32 in TMEM
//   G4  acc += ã · Q_bᵀ               once per block, ã packed bf16 in TMEM as the A operand
// and for each query's uncompressed suffix S = q·K_sufᵀ, acc += p·V_suf.
// A block's factors are read from HBM once and shared by every row.
//
// One persistent CTA per SM walks a host-built list of segments (a KV head's
// row tile over a contiguous range of 128-token chunks, or one query's suffix
// chunks), balanced by estimated time.  Warp 0 issues TMA loads into a byte
// ring in exactly the order warp 1 consumes them; warp 1 issues tcgen05.mma;
// warps 4..11 (two warpgroups splitting each tile by columns, one thread per
// row and TMEM lane) run the softmax and the TMEM conversions.  Scores use two
// TMEM slots, so the softmax of one chunk overlaps G3 of the previous chunk
// and G2 of the next.  Each segment leaves a partial (m, l, acc) that the
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
#include "rope.h"
#include "tc_ptx.cuh"

namespace milo {
namespace {

// warp 0: TMA producer; warp 1: MMA issuer; warps kSoftWarp0 .. kSoftWarp0 + 7: softmax (with kSoftWarp0 = 4,
// warps 2 and 3 are idle and warpgroup 0 holds only the producer and the issuer).
constexpr int kSoftWarp0 = 2;
constexpr int kThreads = 32 * (kSoftWarp0 + 8);
// 8-bit mode: two more warps (kConvWarp0, kConvWarp0 + 1) convert the int8 token-factor tiles to bf16
constexpr int kConvWarp0 = kSoftWarp0 + 8;
template <bool Q8>
constexpr int threads_of() { return Q8 ? kThreads + 64 : kThreads; }
// Register split (setmaxnreg, needs kSoftWarp0 = 4): warpgroup 0 gives registers to the two softmax
// warpgroups.  The split must fit in what the launch allocates (kThreads × kLaunchRegs), or the increase
// would wait forever: the host refuses a build whose kernel was allocated fewer registers.
constexpr bool kRegSplit = false;
constexpr int kRegsLow = 120, kRegsHigh = 192, kLaunchRegs = 168;
static_assert(!kRegSplit || (kSoftWarp0 == 4 && 128 * kRegsLow + 256 * kRegsHigh <= kThreads * kLaunchRegs),
              "register split exceeds the launch");
constexpr int kSigThreads = 288;  // softmax warps + MMA warp on a signal barrier
// named barriers (0 is __syncthreads): softmax warps → MMA warp (P alternates by S slot), one per TMEM
// lane quarter for its two softmax warps, and one for all softmax warps
constexpr int kSigQt = 1, kSigAt = 2, kSigP0 = 3, kPairBar0 = 5, kSoftBar = 9, kConvBar = 10;
constexpr int kItemSlots = 16;       // items in flight at most (one FULL/EMPTY barrier pair each)
constexpr int kChunk = 128;          // tokens per score chunk
constexpr uint64_t kWaitNs = 1000000000ull;
constexpr uint32_t kSleepNs = 2000;  // suspend-time hint of one try_wait in a wait loop

// shared-memory map (bytes from a 1024-aligned base)
constexpr int kOffQ = 0;          // [cb][128 rows][128 B]  query rows, K-major over d
constexpr int kOffQtHi = 32768;   // [cb][128][128 B]  q̃ high part, K-major over rank
constexpr int kOffQtLo = 65536;   // [cb][128][128 B]  q̃ low part
constexpr int kOffStage = 98304;  // 8-bit mode: [2][kStageBytes] bf16 token-factor tiles converted from the ring
constexpr int kStageBytes = 32768;
constexpr int kBarRegion = 8192;
// The TMA ring (variable-size items, each one contiguous tile laid out [64-column block][rows][128 B]), then the
// barriers and the Shared block.  The 8-bit mode gives part of the ring to the two staging tiles.
template <bool Q8>
struct Smem {
  static constexpr int kOffRing = Q8 ? kOffStage + 2 * kStageBytes : 98304;
  static constexpr int kRingBytes = Q8 ? 59392 : 122880;
  static constexpr int kOffBar = kOffRing + kRingBytes;
  static constexpr int kBytes = kOffBar + kBarRegion + 1024;  // + alignment slack
};
static_assert(Smem<false>::kBytes <= 232448 && Smem<true>::kBytes <= 232448, "227 KB of shared memory per CTA");
constexpr uint32_t kTileCb = 16384;  // column-block stride of a 128-row tile
constexpr int kMaxSegsSmem = 16, kMaxBlocksSmem = 64;  // per-CTA work tables staged in smem

// TMEM columns: acc [0,128), two S slots [128,256) and [256,384) (q̃ of a block also passes through
// an S slot; p is packed over the scores it came from), ã [384,512) (packed in place for G4 as bf16 high
// and low parts)
constexpr uint32_t kTmAcc = 0, kTmS0 = 128, kTmA = 384;

// TMEM column, relative to its region, of k-step t (16 bf16) of an A operand that the two softmax
// warpgroups packed in place: warpgroup w holds K indices [64w, 64w + 64) in columns [64w, 64w + 32).
__device__ __forceinline__ uint32_t ta_col(int t) { return (uint32_t)(64 * (t >> 2) + 8 * (t & 3)); }


enum Bar {
  B_FULL = 0,
  B_EMPTY = B_FULL + kItemSlots,
  B_QFULL = B_EMPTY + kItemSlots,
  B_QEMPTY,
  B_SFULL,                // [2] S slot written (G1 / G2 / G2')
  B_SFREE = B_SFULL + 2,  // [2] p in the S slot read (G3 / G3')
  B_ATFULL = B_SFREE + 2, // ã of a block complete
  B_ACCDONE,              // acc written (G4, or a suffix segment's last G3')
  B_FINAL,
  B_STAGED,               // [2] 8-bit mode: bf16 staging tile k written by the converter warps
  B_STFREE = B_STAGED + 2,  // [2] 8-bit mode: staging tile k read by the MMAs
  B_COUNT = B_STFREE + 2
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

// One TMA load of the producer's walk, built on the host in the order the issuing warp consumes the data.
// Ring items (kinds 0 and 1) land at byte `a` of the ring; a query tile (kind 2) lands in the query buffer
// at coordinates (y, z = a).  Before a ring item is issued the producer retires the `retire` oldest ring
// items in flight (waits until the MMAs that read them have completed), which frees its bytes and slot.
struct Item {
  uint32_t a;      // ring byte offset (kinds 0, 1) or z coordinate (kind 2)
  int32_t y;       // row coordinate
  uint32_t bytes;  // bytes the load delivers
  uint32_t meta;   // map index (bits 0-7) | kind (bits 8-9: 0 2D box, 1 3D box, 2 query tile) | retire (16-23)
};
static_assert(sizeof(Item) == 16, "items are loaded as 16-byte words");
constexpr uint32_t kItem2D = 0, kItem3D = 1, kItemQ = 2;

struct CtaRec;
struct PlanMaps;
struct Params {
  const Seg* segs;
  const CtaRec* recs;    // [grid]
  const Item* items;     // every CTA's items, CTA k's at [recs[k].item0, + recs[k].nitems)
  const PlanMaps* gmaps;
  const int32_t* ranks;
  const int64_t* row_offsets;
  float* part_acc;  // [pid][128][D]
  float2* part_ml;  // [pid][128]
  const int* sel;   // [H][nb]: the k-th selected block of each head (block selection), or null for every block
  uint32_t* status;
  int nb, cpb, H, G, ipt, S;
  float c;  // scale · log2(e)
};

struct BlockInfo {
  int rk, rv;
  int64_t rowk, rowv;
};

// Tensor maps of one row-major bf16 operand array (rows of 64 or 128 columns), one per item height
// h = 16, 32, ..., 128 rows, so that every item is a single TMA instruction: for 128-column arrays 3D maps
// (x: 64 columns, y: rows, z: the two 64-column blocks) whose box of h rows × both column blocks lands in
// shared memory as [column block][h][128 B]; for 64-column arrays 2D boxes of h rows × 64 columns.
struct RowMaps {
  CUtensorMap m[8];
};
// The maps of one call's arrays, passed as the kernel parameter (kept small: a launch copies its parameters).
struct Maps {
  CUtensorMap ksuf, vsuf;  // suffix keys and values, boxes of 128 rows
  CUtensorMap qpre, qsuf;  // query rows of a prefix row tile / of one query
  CUtensorMap krope;       // dense-key mode: the rotated prefix keys [H·T][d], boxes of 128 rows
};
// The maps of a plan's factors and partials, in device memory (128-byte aligned), written once per plan.
struct PlanMaps {
  RowMaps tok, dim;
  CUtensorMap pacc;  // partial accumulators [segments · 128][d] fp32, boxes of 128 rows × 32 columns
};
// An item's map index: [0, 16) counts CUtensorMaps from the start of PlanMaps, [16, 20) from the start of Maps.
constexpr int kMapTok = 0, kMapDim = 8, kMapKsuf = 16, kMapVsuf = 17, kMapQpre = 18, kMapQsuf = 19, kMapKrope = 20;
static_assert(sizeof(RowMaps) == 8 * sizeof(CUtensorMap), "row maps hold 8 boxes");
static_assert(sizeof(Maps) == 5 * sizeof(CUtensorMap), "call maps in the order of the item map index");

// One CTA's work, built on the host: its segments and the rank / row offset of every block they touch, in
// the order the roles walk them.  The CTA copies it to shared memory with one coalesced load at start, so
// that no role reads a table from global memory inside the pipeline.
struct CtaRec {
  int nseg;        // segments staged (0 when they did not fit: the roles read the global tables)
  int nblk;        // blocks staged
  int s_begin, s_end;          // the CTA's range in the global segment list
  int blk0[kMaxSegsSmem + 1];  // first block entry of each segment
  int item0, nitems;           // the CTA's producer items in Params::items
  int pad;
  Seg segs[kMaxSegsSmem];
  BlockInfo blocks[kMaxBlocksSmem];
};
static_assert(sizeof(CtaRec) % 16 == 0, "records are copied in 16-byte words");

// Per-CTA state in shared memory.
struct Shared {
  uint32_t tmem_base;
  int abort_flag;
  int pad[2];
  CtaRec rec;
  float mx_x[2][2][128];  // row maxima exchanged by the two softmax warpgroups (double-buffered)
  float l_x[128];         // warpgroup 1's row sums at a segment's end
};
constexpr int kSharedOff = (8 * B_COUNT + 64 + 15) & ~15;  // 16-byte aligned for the record copy
static_assert(kSharedOff + sizeof(Shared) <= kBarRegion, "barrier region too small");

// Warp-collective bounded wait on an mbarrier phase (all 32 lanes call it together; the result is uniform).
// Gives up after kWaitNs, records kStatusDecodeTimeout and raises the CTA's abort flag, or returns false at
// once when another role already aborted.  `drain` waits ignore the abort flag (used to let the CTA's own
// copies and MMAs land before it exits) but keep the time limit.
__device__ __noinline__ bool wait_bar_slow(uint32_t bar, uint32_t parity, Shared* sh, uint32_t* status,
                                           bool drain) {
  uint64_t t0 = 0;
  if ((threadIdx.x & 31) == 0) t0 = ptx::globaltimer();
  for (uint32_t i = 1;; ++i) {
    // sleep in the wait (woken when the phase completes) rather than spin: the waiting roles share the
    // SM sub-partitions with the TMA and MMA-issuing warps, whose issue slots the spinning would take
    if (__all_sync(0xffffffffu, ptx::mbar_try_wait_sleep(bar, parity, kSleepNs))) return true;
    if ((i & 63) == 0) {
      int outcome = 0;  // 0 keep waiting, 1 aborted elsewhere, 2 timed out
      if ((threadIdx.x & 31) == 0) {
        if (!drain && *(volatile int*)&sh->abort_flag) outcome = 1;
        else if (ptx::globaltimer() - t0 > kWaitNs) outcome = 2;
      }
      outcome = __shfl_sync(0xffffffffu, outcome, 0);
      if (outcome == 2 && (threadIdx.x & 31) == 0) {
        atomicOr(status, kStatusDecodeTimeout);
        *(volatile int*)&sh->abort_flag = 1;
      }
      if (outcome) return false;
    }
  }
}

__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, Shared* sh, uint32_t* status,
                                         bool drain = false) {
  if (__all_sync(0xffffffffu, ptx::mbar_try_wait(bar, parity))) return true;
  return wait_bar_slow(bar, parity, sh, status, drain);
}

// Multiplies `ncols` (a multiple of 16) fp32 TMEM columns of this warp's lanes by `alpha` (warp-collective).
__device__ __forceinline__ void rescale_tmem(uint32_t taddr, int ncols, float alpha) {
  for (int c16 = 0; c16 < ncols; c16 += 16) {
    float t16[16];
    ptx::tmem_ld16(taddr + c16, t16);
    ptx::tmem_wait_ld();
#pragma unroll
    for (int e = 0; e < 16; ++e) t16[e] *= alpha;
    ptx::tmem_st16(taddr + c16, t16);
  }
  ptx::tmem_wait_st();
}

__device__ __forceinline__ int pad16(int r) { return (r + 15) & ~15; }

// Block k of head h's walk (the k-th selected block when a selection is given) → its ranks and row offsets.
__device__ __forceinline__ bool block_info(const Params& p, int h, int k, int D, BlockInfo& bi) {
  const int b = p.sel ? p.sel[(int64_t)h * p.nb + k] : k;
  if ((unsigned)b >= (unsigned)p.nb) return false;
  bi.rk = p.ranks[(int64_t)(2 * h) * p.nb + b];
  bi.rv = p.ranks[(int64_t)(2 * h + 1) * p.nb + b];
  bi.rowk = p.row_offsets[(int64_t)(2 * h) * (p.nb + 1) + b];
  bi.rowv = p.row_offsets[(int64_t)(2 * h + 1) * (p.nb + 1) + b];
  return bi.rk >= 1 && bi.rk <= D && bi.rv >= 1 && bi.rv <= D;
}

// Block `k` (0-based, in walk order) of segment `si` of this CTA: from the smem table when staged.
__device__ __forceinline__ bool seg_block(const Params& p, const Shared* sh, int si_local, int k, int h, int b, int D,
                                          BlockInfo& bi) {
  if (sh->rec.nseg > 0) {
    bi = sh->rec.blocks[sh->rec.blk0[si_local] + k];
    return bi.rk >= 1 && bi.rk <= D && bi.rv >= 1 && bi.rv <= D;
  }
  return block_info(p, h, b, D, bi);
}
__device__ __forceinline__ Seg get_seg(const Params& p, const Shared* sh, int s_begin, int si) {
  return sh->rec.nseg > 0 ? sh->rec.segs[si - s_begin] : p.segs[si];
}

// Placement of items in the TMA ring.  Producer and consumer call place() with the same sizes in the same
// order, so they agree on every item's offset without exchanging it; an item that does not fit before the
// end of the ring starts at offset 0.
template <int kRing>
struct RingPlace {
  uint32_t head = 0;  // next free byte offset
  uint32_t n = 0;     // items placed so far
  __device__ uint32_t place(uint32_t bytes) {
    const uint32_t pos = head + bytes <= (uint32_t)kRing ? head : 0u;
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

// MODE: kModeRank (bf16 factors, rank-space scores), kMode8bit (int8 token factors), kModeDenseKeys (the scores
// of the prefix against dense rotated keys, values in rank space).
constexpr int kModeRank = 0, kMode8bit = 1, kModeDenseKeys = 2;
template <int D, int MODE>
__global__ void __launch_bounds__(threads_of<MODE == kMode8bit>(), 1)
    decode_tc_kernel(const __grid_constant__ Maps maps,
                     const Params p) {
  constexpr int NCB = D / 64;
  constexpr bool Q8 = MODE == kMode8bit, DK = MODE == kModeDenseKeys;
  using L = Smem<Q8>;
  constexpr int kNThreads = threads_of<Q8>();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const uint32_t base = ptx::smem_u32(smem);
  Shared* sh = reinterpret_cast<Shared*>(smem + L::kOffBar + kSharedOff);
  auto bar = [&](int i) { return base + L::kOffBar + 8 * i; };
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

  // ---- setup: zero the query tile (rows no TMA box writes stay finite), barriers, TMEM
  for (int i = threadIdx.x; i < 32768 / 16; i += kNThreads) ptx::st_shared_v4(base + kOffQ + 16 * i, 0, 0, 0, 0);
  if (threadIdx.x == 0) {
    for (int i = 0; i < kItemSlots; ++i) {
      ptx::mbar_init(bar(B_FULL + i), 1);
      ptx::mbar_init(bar(B_EMPTY + i), 1);
    }
    ptx::mbar_init(bar(B_QFULL), 1);
    ptx::mbar_init(bar(B_QEMPTY), 1);
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(bar(B_SFULL + i), 1);
      ptx::mbar_init(bar(B_SFREE + i), 1);
    }
    ptx::mbar_init(bar(B_ATFULL), 1);
    ptx::mbar_init(bar(B_ACCDONE), 1);
    ptx::mbar_init(bar(B_FINAL), 1);
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(bar(B_STAGED + i), 1);
      ptx::mbar_init(bar(B_STFREE + i), 1);
    }
    sh->abort_flag = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    ptx::tma_prefetch_desc(&maps.qpre);
    ptx::tma_prefetch_desc(&maps.qsuf);
  }
  if (warp == 1) {
    ptx::tmem_alloc(ptx::smem_u32(&sh->tmem_base), 512);
    ptx::tmem_relinquish();
  }
  // this CTA's work record (segments and block tables) into shared memory: one coalesced load
  {
    const int4* src = reinterpret_cast<const int4*>(p.recs + blockIdx.x);
    int4* dst = reinterpret_cast<int4*>(&sh->rec);
    for (int i = threadIdx.x; i < (int)(sizeof(CtaRec) / 16); i += kNThreads) dst[i] = src[i];
  }
  __syncthreads();
  const int s_begin = sh->rec.s_begin, s_end = sh->rec.s_end;
  ptx::fence_async_smem();
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = sh->tmem_base;
  // the combine kernel that follows may launch now (it waits for this grid before reading the partials)
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  if (warp < kSoftWarp0) {
  // the register decrease dominates the producer's and the MMA issuer's code
  if (kRegSplit) asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsLow));
  if (warp == 0) {
    // ==================================================================== TMA producer
    // Walks the CTA's item list: the host has fixed every load's map, coordinates, ring offset and how many
    // older items must be released before it, so that each item costs a few instructions here.  Lane l holds
    // item i0 + l of the current batch of 32; the batch after it is loaded while this one is issued.
    const Item* items = p.items + sh->rec.item0;
    const int nitems = sh->rec.nitems;
    const CUtensorMap* gmap0 = reinterpret_cast<const CUtensorMap*>(p.gmaps);
    // Everything before this point reads the library's own tables; the loads below read the caller's q,
    // suffix and factors, which the kernel before this one on the stream may still be writing (the launch is
    // a programmatic dependent): wait for that grid first.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const CUtensorMap* pmap0 = reinterpret_cast<const CUtensorMap*>(&maps);
    auto load_item = [&](int i) -> uint4 {
      return i < nitems ? __ldg(reinterpret_cast<const uint4*>(items + i)) : make_uint4(0, 0, 0, 0);
    };
    uint32_t oldest = 0, ring_n = 0, q_uses = 0;
    bool ok = true;
    uint4 cur = load_item(lane);
    for (int i0 = 0; i0 < nitems && ok; i0 += 32) {
      const uint4 nxt = load_item(i0 + 32 + lane);
      const int nb = min(32, nitems - i0);
      for (int k = 0; k < nb && ok; ++k) {
        const uint32_t a = __shfl_sync(0xffffffffu, cur.x, k);
        const int y = (int)__shfl_sync(0xffffffffu, cur.y, k);
        const uint32_t bytes = __shfl_sync(0xffffffffu, cur.z, k);
        const uint32_t meta = __shfl_sync(0xffffffffu, cur.w, k);
        const uint32_t mi = meta & 255u;
        const CUtensorMap* tm = mi < (uint32_t)kMapKsuf ? gmap0 + mi : pmap0 + (mi - kMapKsuf);
        const uint32_t kind = (meta >> 8) & 3u;
        if (kind == kItemQ) {
          ok = wait_bar(bar(B_QEMPTY), (q_uses & 1) ^ 1, sh, p.status);
          if (ok && lane == 0) {
            ptx::mbar_arrive_expect_tx(bar(B_QFULL), bytes);
            for (int cb = 0; cb < NCB; ++cb)
              ptx::tma_load_3d(base + kOffQ + cb * kTileCb, tm, bar(B_QFULL), 64 * cb, y, (int)a);
          }
          ++q_uses;
          continue;
        }
        for (uint32_t r = (meta >> 16) & 255u; r > 0 && ok; --r, ++oldest)
          ok = wait_bar(bar(B_EMPTY + oldest % kItemSlots), (oldest / kItemSlots) & 1, sh, p.status);
        if (!ok) break;
        const uint32_t fb = bar(B_FULL + ring_n % kItemSlots);
        if (lane == 0) {
          ptx::mbar_arrive_expect_tx(fb, bytes);
          if (kind == kItem3D) ptx::tma_load_3d(base + L::kOffRing + a, tm, fb, 0, y, 0);
          else ptx::tma_load_2d(base + L::kOffRing + a, tm, fb, 0, y);
        }
        __syncwarp();
        ++ring_n;
      }
      cur = nxt;
    }
    // drain: every copy this warp issued must have landed before the CTA exits
    for (uint32_t j = oldest; j < ring_n; ++j)
      wait_bar(bar(B_FULL + j % kItemSlots), (j / kItemSlots) & 1, sh, p.status, true);
    if (q_uses) wait_bar(bar(B_QFULL), (q_uses - 1) & 1, sh, p.status, true);
  } else if (warp == 1) {
    // ==================================================================== MMA issuer (warp 1)
    // Issues the tensor-core MMAs when the softmax warps signal (named barriers) that what they produce is
    // complete: q̃ in smem, P in an S slot of TMEM, or ã packed in TMEM.  The probabilities and ã are the A
    // operands of G3 / G4 straight from TMEM.
    const bool leader = lane == 0;
    bool ok = true;
    auto sync_wg = [&](int id) {  // wait for the softmax warps' signal `id`
      asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(kSigThreads) : "memory");
      ptx::tc_fence_after();
    };
    RingPlace<L::kRingBytes> ring;       // consumer view of the TMA ring
    uint32_t cur = 0;                    // item being consumed
    uint32_t use_i = 0, use_c = 0;       // S-slot uses issued / consumed (signalled)
    uint32_t q_uses = 0;
    uint32_t sfree_odd = 0;              // bit s: B_SFREE[s] committed an odd number of times
    auto take = [&](int rows, int ncb, uint32_t& addr) -> bool {
      cur = ring.n;
      const uint32_t pos = ring.place((uint32_t)rows * 128u * ncb);
      if (!wait_bar(bar(B_FULL + cur % kItemSlots), (cur / kItemSlots) & 1, sh, p.status)) return false;
      ptx::tc_fence_after();
      addr = base + L::kOffRing + pos;
      return true;
    };
    auto release = [&]() {  // the item's space is free once the MMAs issued so far have read it
      if (leader) ptx::umma_commit(bar(B_EMPTY + cur % kItemSlots));
    };
    // Token-factor tiles (U, P).  In the 8-bit mode the converter warps turn the ring's int8 tile into a bf16
    // staging tile and release the ring item themselves; the MMAs read the staging tile, which is free again
    // once they complete.
    uint32_t staged = 0, stage_k = 0;  // staging tiles consumed; the tile of the current item
    auto take_tok = [&](int rows, uint32_t& addr) -> bool {
      if (!Q8) return take(rows, 2, addr);
      cur = ring.n;
      ring.place((uint32_t)rows * 128u);  // one byte per token: the ring holds the codes
      stage_k = staged & 1;
      const bool got = wait_bar(bar(B_STAGED + stage_k), (staged >> 1) & 1, sh, p.status);
      ++staged;
      if (!got) return false;
      ptx::tc_fence_after();
      addr = base + kOffStage + stage_k * kStageBytes;
      return true;
    };
    auto release_tok = [&]() {
      if (!Q8) release();
      else if (leader) ptx::umma_commit(bar(B_STFREE + stage_k));
    };
    auto commit = [&](int b) {
      if (leader) ptx::umma_commit(bar(b));
    };
    // An MMA that overwrites a TMEM region which an earlier MMA of this thread reads as its A operand (p in
    // an S slot, ã) needs no wait: the tensor pipe executes one thread's MMAs in issue order, and each reads
    // its operands before any later one writes its accumulator.
    auto slot_free = [&](uint32_t) -> bool { return true; };
    auto s_commit = [&]() {
      commit(B_SFULL + (use_i & 1));
      ++use_i;
    };
    auto p_commit = [&](uint32_t s) {  // P in slot s has been read once the MMAs issued so far complete
      commit(B_SFREE + s);
      sfree_odd ^= 1u << s;
    };
    constexpr uint32_t idS = ptx::idesc_bf16(128, 128, false, true);
    constexpr uint32_t idD = ptx::idesc_bf16(128, D, false, true);
    // G1: q̃ = Q · B_b into the next S slot, N = padded rank
    auto g1 = [&](int rk) -> bool {
      const int rp = pad16(rk);
      uint32_t it;
      if (!slot_free(use_i & 1) || !take(rp, NCB, it)) return false;
      if (leader) {
        const uint64_t da = kdesc(base + kOffQ, 0, kTileCb), db = kdesc(it, 0, 0);
        const uint32_t cbs = (uint32_t)rp * 128u, id = ptx::idesc_bf16(128, rp, false, false);
        const uint32_t d = tmem + kTmS0 + 128 * (use_i & 1);
#pragma unroll 1
        for (int k = 0; k < D / 16; ++k) ptx::umma_bf16(d, da + kstep(k, kTileCb), db + kstep(k, cbs), id, k > 0);
      }
      release();
      s_commit();
      return true;
    };
    // G2: S = q̃_hi·U + q̃_lo·U into the next S slot (B MN-major, N = 128 tokens)
    auto g2 = [&](int rk) -> bool {
      const int rp = pad16(rk);
      uint32_t it;
      if (!slot_free(use_i & 1) || !take_tok(rp, it)) return false;
      if (leader) {
        const uint32_t d = tmem + kTmS0 + 128 * (use_i & 1);
        const uint64_t db = mndesc(it, 0, (uint32_t)rp * 128u);
        const uint64_t dh = kdesc(base + kOffQtHi, 0, kTileCb), dl = kdesc(base + kOffQtLo, 0, kTileCb);
        for (int t = 0; t < rp / 16; ++t) {
          const uint64_t bd = db + (uint64_t)(t * 128);
          ptx::umma_bf16(d, dh + kstep(t, kTileCb), bd, idS, t > 0);
          ptx::umma_bf16(d, dl + kstep(t, kTileCb), bd, idS, 1);
        }
      }
      release_tok();
      s_commit();
      return true;
    };
    // G3: ã (+)= p · P_b, p packed in S slot s, N = padded rank; `fresh` overwrites ã
    auto g3 = [&](int rv, bool fresh, uint32_t s) -> bool {
      const int rp = pad16(rv);
      uint32_t it;
      if (!take_tok(rp, it)) return false;
      if (leader) {
        const uint64_t db = kdesc(it, 0, 0);
        const uint32_t cbs = (uint32_t)rp * 128u, id = ptx::idesc_bf16(128, rp, false, false);
        const uint32_t a = tmem + kTmS0 + 128 * s;
#pragma unroll
        for (int t = 0; t < kChunk / 16; ++t)
          ptx::umma_bf16_ta(tmem + kTmA, a + ta_col(t), db + kstep(t, cbs), id, (t > 0 || !fresh) ? 1u : 0u);
      }
      release_tok();
      p_commit(s);
      return true;
    };
    // G4: acc (+)= ã · Q_bᵀ, ã packed in TMEM, B MN-major, N = d
    auto g4 = [&](int rv, bool fresh) -> bool {
      const int rp = pad16(rv);
      uint32_t it;
      if (!take(rp, NCB, it)) return false;
      if (leader) {
        const uint64_t db = mndesc(it, 0, (uint32_t)rp * 128u);
        for (int t = 0; t < rp / 16; ++t) {  // ã's high part, then its low part (32 columns further)
          const uint64_t bd = db + (uint64_t)(t * 128);
          ptx::umma_bf16_ta(tmem + kTmAcc, tmem + kTmA + ta_col(t), bd, idD, (t > 0 || !fresh) ? 1u : 0u);
          ptx::umma_bf16_ta(tmem + kTmAcc, tmem + kTmA + ta_col(t) + 32, bd, idD, 1u);
        }
      }
      release();
      commit(B_ACCDONE);
      return true;
    };
    // G2' (suffix): S = q · K_sufᵀ, B K-major over d, N = 128 tokens
    auto g2s = [&]() -> bool {
      uint32_t it;
      if (!slot_free(use_i & 1) || !take(kChunk, NCB, it)) return false;
      if (leader) {
        const uint64_t da = kdesc(base + kOffQ, 0, kTileCb), db = kdesc(it, 0, 0);
        const uint32_t d = tmem + kTmS0 + 128 * (use_i & 1), id = ptx::idesc_bf16(128, kChunk, false, false);
#pragma unroll
        for (int t = 0; t < D / 16; ++t)
          ptx::umma_bf16(d, da + kstep(t, kTileCb), db + kstep(t, kChunk * 128u), id, t > 0);
      }
      release();
      s_commit();
      return true;
    };
    // G3' (suffix): acc (+)= p · V_suf, p packed in S slot s, B MN-major, K = 128 tokens, N = d
    auto g3s = [&](bool fresh, uint32_t s) -> bool {
      uint32_t it;
      if (!take(kChunk, NCB, it)) return false;
      if (leader) {
        const uint64_t db = mndesc(it, 0, kChunk * 128u);
        const uint32_t a = tmem + kTmS0 + 128 * s;
#pragma unroll
        for (int t = 0; t < kChunk / 16; ++t)
          ptx::umma_bf16_ta(tmem + kTmAcc, a + ta_col(t), db + (uint64_t)(t * 128), idD, (t > 0 || !fresh) ? 1u : 0u);
      }
      release();
      p_commit(s);
      return true;
    };
    auto wait_q = [&]() -> bool {
      const bool r = wait_bar(bar(B_QFULL), q_uses & 1, sh, p.status);
      ++q_uses;
      ptx::tc_fence_after();
      return r;
    };
    auto sync_p = [&]() -> uint32_t {  // the softmax warps' P of the next consumed use; returns its slot
      const uint32_t s = use_c & 1;
      sync_wg(kSigP0 + (int)s);
      ++use_c;
      return s;
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
        // dense-key mode: no q̃ (the prefix scores are Q·Kᵀ like the suffix's), Q is read by every G2
        auto g2k = [&]() -> bool { return DK ? g2s() : g2(bi.rk); };
        if (ok) {
          ok = wait_q() && (DK || g1(bi.rk));
          if (!DK && ok && !w.has_next()) commit(B_QEMPTY);  // last read of Q in this segment
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
          if (!DK) {
            sync_wg(kSigQt);
            ++use_c;
          }
          if (ok) {
            ok = g2k();
            if (ok && n >= 2) ok = g2k();
            else if (!DK && ok && next) ok = g1_next();
          }
          if (have_prev) {
            sync_wg(kSigAt);
            if (ok) ok = g4(prev.rv, kb == 1);
          }
          for (int j = 0; j < n; ++j) {
            const uint32_t s = sync_p();
            if (ok) {
              ok = g3(bi.rv, j == 0, s);
              if (ok && j + 1 == n) commit(B_ATFULL);
              if (ok && j + 2 < n) ok = g2k();
              else if (!DK && ok && j + 2 == n && next) ok = g1_next();
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
        if (ok) ok = g4(bi.rv, kb == 0);
        if (DK && ok) commit(B_QEMPTY);  // every G2 of the segment has read Q
      } else {
        const int n = sg.c1 - sg.c0;
        if (ok) {
          ok = wait_q() && g2s();
          if (ok && n >= 2) ok = g2s();
          if (ok && n <= 2) commit(B_QEMPTY);
        }
        for (int j = 0; j < n; ++j) {
          const uint32_t s = sync_p();
          if (ok) {
            ok = g3s(j == 0, s);
            if (ok && j + 2 < n) {
              ok = g2s();
              if (ok && j + 2 == n - 1) commit(B_QEMPTY);
            }
          }
        }
        if (ok) commit(B_ACCDONE);
      }
    }
    // drain: every MMA issued must complete before TMEM is freed
    commit(B_FINAL);
    __syncwarp();
    wait_bar(bar(B_FINAL), 0, sh, p.status, true);
  }
  } else if (Q8 && warp >= kConvWarp0) {
    // ==================================================================== 8-bit converter (two warps)
    // Follows the producer's item list and turns every int8 token-factor tile of the ring into the bf16 tile
    // that the MMAs read, in one of two staging tiles: the codes c in [-128, 127] are exact in bf16.  The ring
    // item is released as soon as it has been read; the staging tile when the MMAs that read it complete.
    const int ct = threadIdx.x - 32 * kConvWarp0;  // 0..63
    const Item* items = p.items + sh->rec.item0;
    const int nitems = sh->rec.nitems;
    uint32_t ring_n = 0, staged = 0;
    // The loop depends only on the item list: after a failed wait both warps still take the same barriers.
    for (int i = 0; i < nitems; ++i) {
      const uint4 it = __ldg(reinterpret_cast<const uint4*>(items + i));
      const uint32_t kind = (it.w >> 8) & 3u, mi = it.w & 255u;
      if (kind == kItemQ) continue;
      const uint32_t ri = ring_n++;
      if (mi >= (uint32_t)kMapTok + 8) continue;  // not a token-factor tile
      const uint32_t k = staged & 1;
      bool got = wait_bar(bar(B_FULL + ri % kItemSlots), (ri / kItemSlots) & 1, sh, p.status);
      if (got) got = wait_bar(bar(B_STFREE + k), ((staged >> 1) & 1) ^ 1, sh, p.status);
      ++staged;
      got = ptx::bar_and(kConvBar, 64, got);
      if (got) {
        ptx::tc_fence_after();
        const int rows = (int)(it.z >> 7);  // one byte per token, 128 tokens per row
        const uint32_t src = base + L::kOffRing + it.x;
        const uint32_t dst = base + kOffStage + k * kStageBytes;
        // unit (row j, 16-byte chunk c): the 16 codes of tokens 16c .. 16c + 15, read from the TMA's 128-byte
        // swizzled row and written as two 16-byte bf16 chunks of the [64-token block][rows][128 B] tile
        for (int u = ct; u < rows * 8; u += 64) {
          const int j = u >> 3, c = u & 7;
          const uint4 w = ptx::ld_shared_v4(src + (uint32_t)j * 128u + ((uint32_t)(c ^ (j & 7)) << 4));
          const uint32_t wd[4] = {w.x ^ 0x80808080u, w.y ^ 0x80808080u, w.z ^ 0x80808080u, w.w ^ 0x80808080u};
          uint32_t o[8];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            // byte b = c + 128 as the low mantissa bits of 2^23: (2^23 + b) − (2^23 + 128) = c exactly
            float f[4];
#pragma unroll
            for (int e = 0; e < 4; ++e)
              f[e] = __uint_as_float(__byte_perm(wd[q], 0x4B000000u, 0x7540u | e)) - 8388736.0f;
            o[2 * q] = __byte_perm(__float_as_uint(f[0]), __float_as_uint(f[1]), 0x7632u);
            o[2 * q + 1] = __byte_perm(__float_as_uint(f[2]), __float_as_uint(f[3]), 0x7632u);
          }
          const uint32_t row = dst + (uint32_t)(c >> 2) * (uint32_t)rows * 128u + (uint32_t)j * 128u;
          const int ch = 2 * (c & 3);
          ptx::st_shared_v4(row + ((uint32_t)(ch ^ (j & 7)) << 4), o[0], o[1], o[2], o[3]);
          ptx::st_shared_v4(row + ((uint32_t)((ch + 1) ^ (j & 7)) << 4), o[4], o[5], o[6], o[7]);
        }
        ptx::fence_async_smem();
      }
      asm volatile("bar.sync %0, 64;" ::"r"(kConvBar) : "memory");
      if (got && ct == 0) {
        ptx::mbar_arrive(bar(B_EMPTY + ri % kItemSlots));  // the codes have been read
        ptx::mbar_arrive(bar(B_STAGED + k));
      }
    }
  } else {
  if (kRegSplit) asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsHigh));
  {
    // ==================================================================== softmax (warps 4..11)
    // Two warpgroups split every 128-column tile by columns: warpgroup wg takes columns [64wg, 64wg + 64).
    // Warp w serves TMEM lane quarter w & 3 (one thread per row); the two warps of a quarter exchange their
    // row maxima through shared memory.  Signals reach the MMA warp through named barriers.
    const int wg = (warp - kSoftWarp0) >> 2;
    const int quarter = warp & 3;
    const int row = 32 * quarter + lane;
    const uint32_t tl = tmem + ((uint32_t)(32 * quarter) << 16);
    const int pair_id = kPairBar0 + quarter;
    uint32_t use = 0;                 // S-slot uses consumed
    uint32_t sfree_odd = 0;           // bit s: B_SFREE[s] commits (as the MMA warp counts them) are odd
    uint32_t at_uses = 0, accdone_n = 0, xpar = 0;
    bool ok = true;
    auto signal = [&](int id) {  // arrive on the MMA warp's named barrier `id` (does not wait)
      ptx::tc_fence_before();
      asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(kSigThreads) : "memory");
    };
    auto pair_sync = [&]() { asm volatile("bar.sync %0, 64;" ::"r"(pair_id) : "memory"); };
    // Every helper below ends with its signal, also after a failed wait, so that all warps always execute
    // the same sequence of named barriers (which have no time limit).
    // q̃ of a block (fp32, in the next S slot) → bf16 hi + lo in smem, columns >= r zeroed
    auto convert_qt = [&](bool active, int rk) -> bool {
      const uint32_t s = use & 1;
      const bool got = wait_bar(bar(B_SFULL + s), (use >> 1) & 1, sh, p.status);
      ++use;
      if (got) {
        ptx::tc_fence_after();
        const uint32_t src = tl + kTmS0 + 128 * s;
        if (active) {
#pragma unroll 1
          for (int c16 = 16 * wg; c16 < pad16(rk); c16 += 32) {
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
      }
      signal(kSigQt);
      return got;
    };
    // ã (fp32, TMEM) → bf16 high and low parts packed in place (warpgroup wg: ranks [64wg, 64wg + 64), high
    // part in columns [64wg, 64wg + 32), low part in [64wg + 32, 64wg + 64)), ranks >= r zeroed.  G4 takes both,
    // so that ã keeps about 16 bits: with 8-bit factors its entries are sums of codes whose large terms cancel
    // against the zero-point component, and one bf16 rounding of them would be visible in the output.
    auto convert_at = [&](bool active, int rv) -> bool {
      const bool got = wait_bar(bar(B_ATFULL), at_uses & 1, sh, p.status);
      ++at_uses;
      ++accdone_n;  // the G4 this signal releases commits B_ACCDONE
      if (got) {
        ptx::tc_fence_after();
        if (active && 64 * wg < pad16(rv)) {
          // half h's high part lands on columns [16h, 16h + 16) (half 0's, read first) and its low part on
          // [32 + 16h, 32 + 16h + 16) (half 1's): half 0's low part waits until half 1 has been read
          const uint32_t at = tl + kTmA + 64 * wg;
          auto split = [&](const float* v, int h, uint32_t* hi, uint32_t* lo) {
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const int r0 = 64 * wg + 32 * h + 2 * e;
              const float a = r0 < rv ? v[2 * e] : 0.f;
              const float b2 = r0 + 1 < rv ? v[2 * e + 1] : 0.f;
              hi[e] = ptx::pack_bf16(a, b2);
              lo[e] = ptx::pack_bf16(a - __uint_as_float(hi[e] << 16), b2 - __uint_as_float(hi[e] & 0xFFFF0000u));
            }
          };
          float v[32];
          uint32_t hi[16], lo0[16], lo1[16];
          ptx::tmem_ld32(at, v);
          ptx::tmem_wait_ld();
          split(v, 0, hi, lo0);
          ptx::tmem_st16u(at, hi);
          ptx::tmem_ld32(at + 32, v);
          ptx::tmem_wait_ld();
          ptx::tmem_st16u(at + 32, lo0);
          split(v, 1, hi, lo1);
          ptx::tmem_st16u(at + 16, hi);
          ptx::tmem_st16u(at + 48, lo1);
          ptx::tmem_wait_st();
        }
      }
      signal(kSigAt);
      return got;
    };
    // One chunk of scores: online softmax, probabilities packed into the S slot's TMEM for G3.
    // prev_chunk: the previous S-slot use was a chunk of this segment (its G3 wrote ã, or acc in a suffix);
    // at_cols: padded rank of ã (0: no ã); acc_live: acc holds earlier results; acc_by_g4: by a G4.
    auto chunk = [&](bool active, int valid, bool& first_chunk, float& m_used, float& l, bool prev_chunk,
                     int at_cols, bool acc_live, bool acc_by_g4) -> bool {
      const uint32_t s = use & 1, ps = s ^ 1;
      // the pair barrier below runs whether or not the wait succeeded: it depends only on `active`,
      // which both warps of a lane quarter share
      const bool got = wait_bar(bar(B_SFULL + s), (use >> 1) & 1, sh, p.status);
      if (got) ptx::tc_fence_after();
      ++use;
      const uint32_t src = tl + kTmS0 + 128 * s + 64 * wg;
      float alpha = 1.f;
      bool grow = false;
      // The scores are read from TMEM twice, 32 columns at a time (max pass, then exp pass), so that few
      // registers stay live across the exchange with the partner warp.
      float v[32];
      if (active) {
        float mx = -INFINITY;
        if (got) {
          float m8[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) m8[e] = -INFINITY;
#pragma unroll 1
          for (int h = 0; h < 2; ++h) {
            ptx::tmem_ld32(src + 32 * h, v);
            ptx::tmem_wait_ld();
            if (valid >= kChunk) {
#pragma unroll
              for (int i = 0; i < 32; ++i) m8[i & 7] = fmaxf(m8[i & 7], v[i]);
            } else {
#pragma unroll
              for (int i = 0; i < 32; ++i)
                m8[i & 7] = fmaxf(m8[i & 7], 64 * wg + 32 * h + i < valid ? v[i] : -INFINITY);
            }
          }
          mx = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])), fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
          ptx::tmem_ld32(src, v);  // first half of the exp pass, in flight during the exchange
        }
        sh->mx_x[xpar][wg][row] = mx;
        pair_sync();
        mx = fmaxf(mx, sh->mx_x[xpar][wg ^ 1][row]) * p.c;
        // keep the running max in use unless the chunk exceeds it by more than 2^8 (then rescale)
        grow = got && !first_chunk && mx > m_used + 8.f;
        if (grow) {
          alpha = ptx::ex2(m_used - mx);
          m_used = mx;
          l *= alpha;
        }
        if (got && first_chunk) m_used = mx;
      }
      xpar ^= 1;
      first_chunk = false;
      if (__any_sync(0xffffffffu, grow)) {
        // rare: rescale what this warp's rows accumulated so far (alpha = 1 for rows that did not grow),
        // once the MMAs that wrote it have landed
        bool w_ok = true;
        if (prev_chunk) w_ok = wait_bar(bar(B_SFREE + ps), ((sfree_odd >> ps) & 1) ^ 1, sh, p.status);
        if (w_ok && acc_by_g4) w_ok = wait_bar(bar(B_ACCDONE), (accdone_n - 1) & 1, sh, p.status);
        ptx::tc_fence_after();
        if (w_ok) {
          if (prev_chunk && at_cols > 64 * wg) rescale_tmem(tl + kTmA + 64 * wg, min(at_cols - 64 * wg, 64), alpha);
          if (acc_live) rescale_tmem(tl + kTmAcc + wg * (D / 2), D / 2, alpha);
          ptx::tmem_wait_st();
        }
      }
      if (active && got) {
        // p = exp2(S·c − m) packed as bf16 over this warpgroup's columns of the slot, row sum in fp32.
        // Packed half h lands on score columns [16h, 16h + 16) of this warpgroup, which were read before.
        float ls0 = 0.f, ls1 = 0.f;
        const float nm = -m_used;
#pragma unroll 1
        for (int h = 0; h < 2; ++h) {
          if (h == 1) ptx::tmem_ld32(src + 32, v);
          ptx::tmem_wait_ld();
          if (valid < kChunk) {  // a ragged suffix chunk: zero the probabilities of the missing tokens
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = 64 * wg + 32 * h + i < valid ? v[i] : -INFINITY;
          }
          uint32_t pw[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const float a = ptx::ex2(fmaf(v[2 * e], p.c, nm));
            const float b2 = ptx::ex2(fmaf(v[2 * e + 1], p.c, nm));
            if (e & 1) ls1 += a + b2;
            else ls0 += a + b2;
            pw[e] = ptx::pack_bf16(a, b2);
          }
          ptx::tmem_st16u(tl + kTmS0 + 128 * s + 64 * wg + 16 * h, pw);
        }
        ptx::tmem_wait_st();
        l += ls0 + ls1;
      }
      sfree_odd ^= 1u << s;
      signal(kSigP0 + (int)s);
      return got;
    };
    // The segment's acc goes to global memory through shared memory (the q̃ region, idle at a segment's
    // end) and TMA tile stores: each 32-column block is staged as 128 rows × 128 B with the 128-byte
    // swizzle, which the store undoes and which keeps the staging stores free of bank conflicts.
    const bool storer = warp == kSoftWarp0 && lane == 0;
    bool store_pending = false;
    auto soft_sync = [&]() { asm volatile("bar.sync %0, %1;" ::"r"(kSoftBar), "r"(256) : "memory"); };
    bool dep_done = false;  // the previous combine on this stream (if any) has finished reading the partials
    auto write_partial = [&](const Seg& sg, bool active, float m_used, float l) -> bool {
      if (!dep_done) {
        asm volatile("griddepcontrol.wait;" ::: "memory");
        dep_done = true;
      }
      const bool got = wait_bar(bar(B_ACCDONE), (accdone_n - 1) & 1, sh, p.status);
      if (got) ptx::tc_fence_after();
      if (active) {
        if (got) {
#pragma unroll 1
          for (int c32 = 0; c32 < D / 2; c32 += 32) {
            float v[32];
            ptx::tmem_ld32(tl + kTmAcc + wg * (D / 2) + c32, v);
            ptx::tmem_wait_ld();
            const uint32_t blk = base + kOffQtHi + (uint32_t)((wg * (D / 2) + c32) / 32) * 16384u + (uint32_t)row * 128u;
#pragma unroll
            for (int j = 0; j < 8; ++j)
              ptx::st_shared_v4(blk + (uint32_t)((j ^ (row & 7)) << 4), __float_as_uint(v[4 * j]),
                                __float_as_uint(v[4 * j + 1]), __float_as_uint(v[4 * j + 2]),
                                __float_as_uint(v[4 * j + 3]));
          }
        }
        if (wg == 1) sh->l_x[row] = l;
        pair_sync();  // unconditional for active warps (see chunk)
        if (got && wg == 0 && row < sg.rows)
          p.part_ml[(int64_t)sg.pid * 128 + row] = make_float2(m_used, l + sh->l_x[row]);
      }
      ptx::fence_async_smem();
      soft_sync();
      if (storer) {
        for (int cb = 0; cb < D / 32; ++cb) ptx::tma_store_2d(&p.gmaps->pacc, base + kOffQtHi + 16384u * cb, 32 * cb, sg.pid * 128);
        ptx::bulk_commit();
        store_pending = true;
      }
      // acc is read before any MMA of the next segment writes it: those follow a later signal
      return got;
    };
    auto fail_bounds = [&]() {
      if (warp == kSoftWarp0 && lane == 0) atomicOr(p.status, kStatusDecodeBounds);
      sh->abort_flag = 1;
      return false;
    };

    // The loops below depend only on the work list, never on `ok`: after a failure (an expired wait, which
    // also raises the CTA's abort flag so that later waits return at once) the warps still walk the same
    // steps and barriers, skipping the work, and then leave together.
    // One walk serves both segment kinds, so that each helper is expanded once: a prefix segment runs, per
    // block, q̃ → (the previous block's ã) → its chunks, and finally the last block's ã; a suffix segment
    // runs its chunks.
    bool bounds_ok = true;
    for (int si = s_begin; si < s_end && bounds_ok; ++si) {
      const Seg sg = get_seg(p, sh, s_begin, si);
      const bool pre = sg.type == 0;
      const bool active = 32 * quarter < sg.rows;  // a warp whose rows are all padding keeps the protocol only
      if (si > s_begin) {  // the previous segment's bulk store has read the staging area (the q̃ region)
        if (storer && store_pending) ptx::bulk_wait_read();
        store_pending = false;
        soft_sync();
      }
      float m_used = -INFINITY, l = 0.f;
      bool first_chunk = true;
      BlockWalk w{sg.c0, sg.c1, p.cpb};
      BlockInfo bi{}, bn{}, prev{};
      int kb = 0;
      bool have_prev = false, done = false;
      if (pre && !seg_block(p, sh, si - s_begin, kb, sg.h, w.block(), D, bi)) {
        bounds_ok = fail_bounds();
        break;
      }
      while (true) {
        int n = sg.c1 - sg.c0;
        bool next = false;
        if (pre && !done) {
          n = w.chunks();
          next = w.has_next();
          if (next && !seg_block(p, sh, si - s_begin, kb + 1, sg.h, w.block() + 1, D, bn)) {
            bounds_ok = fail_bounds();
            break;
          }
          if (!DK) ok = convert_qt(active, bi.rk) && ok;  // q̃ of this block to smem
        }
        if (have_prev) ok = convert_at(active, prev.rv) && ok;  // the previous block's ã for its G4
        if (done) break;
        for (int j = 0; j < n; ++j) {
          const int valid = pre ? kChunk : min(kChunk, p.S - (sg.c0 + j) * kChunk);
          ok = chunk(active, valid, first_chunk, m_used, l, j > 0, pre ? pad16(bi.rv) : 0, pre ? have_prev : j > 0,
                     pre && have_prev) && ok;
        }
        if (!pre) break;
        prev = bi;
        have_prev = true;
        if (next) {
          w.next();
          bi = bn;
          ++kb;
        } else {
          done = true;  // one more pass for the last block's ã
        }
      }
      if (!bounds_ok) break;
      if (!pre) ++accdone_n;  // the MMA warp commits B_ACCDONE after a suffix segment's last G3'
      ok = write_partial(sg, active, m_used, l) && ok;
    }
    if (storer && store_pending) ptx::bulk_wait_all();  // the last store has completed before the CTA exits
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
  // launched as a programmatic dependent of the decode kernel: its launch overlaps the decode's last CTAs, and
  // this waits until the decode grid has completed and its partials are visible
  asm volatile("griddepcontrol.wait;" ::: "memory");
  // the next decode call on this stream may start its set-up and loads now; it waits for this grid before it
  // writes the partials read here
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
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
// The combine kernel for one decode call, launched with programmatic stream serialization so that its launch
// overlaps the tail of the decode kernel before it (it waits for that grid with griddepcontrol.wait).
cudaError_t launch_combine(const DecodeShape& s, const float* part_acc, const float2* part_ml, const int* pre,
                           const int* suf, int ipt, int nrt, void* out, cudaStream_t st) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(s.Hq, s.Bq);
  cfg.blockDim = dim3(s.d);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  __nv_bfloat16* o = static_cast<__nv_bfloat16*>(out);
  if (s.d == 64)
    return cudaLaunchKernelEx(&cfg, combine_tc_kernel<64>, part_acc, part_ml, pre, suf, s.H, s.Hq, ipt, nrt, o);
  return cudaLaunchKernelEx(&cfg, combine_tc_kernel<128>, part_acc, part_ml, pre, suf, s.H, s.Hq, ipt, nrt, o);
}

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
              const uint32_t* box, CUtensorMapDataType dt = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t gd[3], gs[2];
  cuuint32_t bx[3], es[3] = {1, 1, 1};
  for (int i = 0; i < rank; ++i) {
    gd[i] = dims[i];
    bx[i] = box[i];
  }
  for (int i = 0; i + 1 < rank; ++i) gs[i] = strides_bytes[i];
  return fn(m, dt, rank, const_cast<void*>(ptr), gd, gs, bx, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Prepares the decode kernel for head dimension d: its shared-memory size, and a check that the launch
// allocates the registers that the kernel's register split (setmaxnreg) redistributes.
template <int MODE>
const void* kernel_of(int d) {
  return d == 64 ? (const void*)decode_tc_kernel<64, MODE> : (const void*)decode_tc_kernel<128, MODE>;
}
cudaError_t prepare_kernel(int d, int mode) {
  const void* kfn = mode == kMode8bit ? kernel_of<kMode8bit>(d)
                    : mode == kModeDenseKeys ? kernel_of<kModeDenseKeys>(d) : kernel_of<kModeRank>(d);
  cudaFuncAttributes fa;
  cudaError_t e = cudaFuncGetAttributes(&fa, kfn);
  if (e != cudaSuccess) return e;
  if (kRegSplit && fa.numRegs < kLaunchRegs) return cudaErrorInvalidConfiguration;
  return cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              mode == kMode8bit ? Smem<true>::kBytes : Smem<false>::kBytes);
}
// Launched with programmatic stream serialization: when the operation before it on the stream is a kernel (the
// previous decode call's combine, say), this grid's launch and set-up (barriers, TMEM, its work record) overlap
// that kernel, and the producer waits for it (griddepcontrol.wait) before loading any caller data; the softmax
// warps wait again before the first partial write.  Not in the dense-key mode, whose keys the kernel right
// before it writes.
template <int MODE>
cudaError_t launch_mode(int d, int grid, const Maps& maps, const Params& p, cudaStream_t st) {
  constexpr bool q8 = MODE == kMode8bit;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(threads_of<q8>());
  cfg.dynamicSmemBytes = Smem<q8>::kBytes;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = MODE == kModeDenseKeys ? 0 : 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (d == 64) return cudaLaunchKernelEx(&cfg, decode_tc_kernel<64, MODE>, maps, p);
  return cudaLaunchKernelEx(&cfg, decode_tc_kernel<128, MODE>, maps, p);
}
// Launches the decode kernel of head dimension d in `mode`.
cudaError_t launch_decode_kernel(int d, int mode, int grid, const Maps& maps, const Params& p, cudaStream_t st) {
  if (mode == kMode8bit) return launch_mode<kMode8bit>(d, grid, maps, p, st);
  if (mode == kModeDenseKeys) return launch_mode<kModeDenseKeys>(d, grid, maps, p, st);
  return launch_mode<kModeRank>(d, grid, maps, p, st);
}
int mode_of(const TcInputs& in) { return in.q8 ? kMode8bit : in.rope_keys ? kModeDenseKeys : kModeRank; }

// The map of a [rows][width] bf16 array with boxes of h rows: 3D for 128 columns (x: 64 columns, y: rows,
// z: the two 64-column blocks), 2D for 64 columns.
bool make_rows_map(CUtensorMap* m, const void* ptr, uint64_t width, uint64_t rows, uint32_t h) {
  if (width == 128) {
    const uint64_t d3[3] = {64, rows, 2}, s3[2] = {width * 2, 128};
    const uint32_t b3[3] = {64, h, 2};
    return make_map(m, ptr, 3, d3, s3, b3);
  }
  const uint64_t d2[2] = {width, rows}, s2[1] = {width * 2};
  const uint32_t b2[2] = {64, h};
  return make_map(m, ptr, 2, d2, s2, b2);
}
// The maps of a [rows][width] bf16 array, one per box height 16, 32, ..., 128 rows.
bool make_row_maps(RowMaps* rm, const void* ptr, uint64_t width, uint64_t rows) {
  std::memset(rm, 0, sizeof(RowMaps));
  for (int k = 0; k < 8; ++k)
    if (!make_rows_map(&rm->m[k], ptr, width, rows, 16u * (k + 1))) return false;
  return true;
}
// The same for the int8 codes of an 8-bit token factor: [rows][128] bytes, boxes of 128 bytes × h rows.
bool make_code_maps(RowMaps* rm, const void* ptr, uint64_t rows) {
  std::memset(rm, 0, sizeof(RowMaps));
  const uint64_t d2[2] = {128, rows}, s2[1] = {128};
  for (int k = 0; k < 8; ++k) {
    const uint32_t b2[2] = {128, 16u * (k + 1)};
    if (!make_map(&rm->m[k], ptr, 2, d2, s2, b2, CU_TENSOR_MAP_DATA_TYPE_UINT8)) return false;
  }
  return true;
}

// Map of the partial accumulators: [rows][d] fp32, 128-row × 32-column boxes, 128-byte swizzle.
bool make_pacc_map(CUtensorMap* m, float* part_acc, int64_t nseg, int d) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t gd[2] = {(cuuint64_t)d, (cuuint64_t)std::max<int64_t>(1, nseg) * 128}, gs[1] = {(cuuint64_t)d * 4};
  cuuint32_t bx[2] = {32, 128}, es[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, part_acc, gd, gs, bx, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

// Maps of one call's query and suffix arrays.
bool make_call_maps(Maps* M, const DecodeShape& s, const TcInputs& in, int ipt) {
  const int D = s.d, G = s.Hq / s.H;
  const uint64_t dims[3] = {(uint64_t)D, (uint64_t)s.Hq, (uint64_t)s.Bq};
  const uint64_t strd[2] = {(uint64_t)D * 2, (uint64_t)s.Hq * D * 2};
  const uint32_t box_pre[3] = {64, (uint32_t)G, (uint32_t)ipt};
  const uint32_t box_suf[3] = {64, (uint32_t)G, 1};
  if (!make_map(&M->qpre, in.q, 3, dims, strd, box_pre)) return false;
  if (!make_map(&M->qsuf, in.q, 3, dims, strd, box_suf)) return false;
  if (s.S > 0) {
    const uint64_t rows = (uint64_t)s.Bq * s.H * s.S;
    if (!make_rows_map(&M->ksuf, in.K_suf, D, rows, kChunk) || !make_rows_map(&M->vsuf, in.V_suf, D, rows, kChunk))
      return false;
  } else {
    M->ksuf = M->qpre;  // never read
    M->vsuf = M->qpre;
  }
  M->krope = M->qpre;  // replaced in the dense-key mode
  return true;
}

}  // namespace

struct TcPlan {
  int Bq = 0, Hq = 0, S = 0;
  std::vector<uint8_t> mask;  // the block selection this plan was built for (empty: every block)
  int off_sel = -1;
  int off_rec = 0;            // per-CTA records (CtaRec) in d_work
  int off_items = 0;          // producer items (Item) in d_work
  int grid = 0, nsegs = 0, ipt = 0, nrt = 0;
  int* d_work = nullptr;  // seg_first | segs | pre_range | suf_range
  int off_segs = 0, off_pre = 0, off_suf = 0;
  float* part_acc = nullptr;
  float2* part_ml = nullptr;
  const void* tok = nullptr;
  const void* dim = nullptr;
  PlanMaps* d_maps = nullptr;  // the factor and partial maps in device memory
  bool q8 = false;             // 8-bit token factors
  bool rope = false;           // pre-RoPE key factors: the decode scores the rotated keys below
  void* krope = nullptr;       // [H][T][d] bf16 rotated reconstructed keys (dense-key mode)
};

bool tc_shape_ok(const DecodeShape& s) {
  const int G = s.Hq / s.H;
  return s.bf16 && (s.d == 64 || s.d == 128) && s.n % kChunk == 0 && G >= 1 && G <= 128 && s.Hq % s.H == 0;
}

bool tc_supported(const DecodeShape& s) { return tc_shape_ok(s) && encode_fn() != nullptr; }

int tc_launches(const DecodeShape&, bool rope_keys) { return rope_keys ? 3 : 2; }

void tc_plan_destroy(TcPlan* plan) {
  if (!plan) return;
  cudaFree(plan->d_work);
  cudaFree(plan->part_acc);
  cudaFree(plan->part_ml);
  cudaFree(plan->d_maps);
  cudaFree(plan->krope);
  delete plan;
}

// Estimated time of one work atom, used to balance the work list across CTAs.  The weights come from a
// least-squares fit of per-CTA run times on B200 against their work (about 0.9 µs per prefix chunk, 0.8 µs
// per suffix chunk, 2.6 µs per block visited and per segment): a 128-token chunk costs about the same
// whatever its ranks (softmax and MMA issue dominate its bytes), the first chunk of a block adds the q̃ and
// ã round trips (G1, conversions, G4), the first chunk of a suffix unit adds a segment's partial.
constexpr double kChunkNs = 750.0, kSufChunkNs = 370.0, kBlockNs = 2600.0, kUnitNs = 2600.0, kBytesPerNs = 150.0;
inline double prefix_atom_ns(int rk, int rv, int cc, int d) {
  const double bytes = 2.0 * (rk + rv) * kChunk + (cc == 0 ? 2.0 * (rk + rv) * d : 0.0);
  return bytes / kBytesPerNs + kChunkNs + (cc == 0 ? kBlockNs : 0.0);
}
inline double suffix_atom_ns(int c, int d) {
  return 2.0 * 2.0 * kChunk * d / kBytesPerNs + kSufChunkNs + (c == 0 ? kUnitNs : 0.0);
}

// The decode work list, written into `w` without heap allocation: atoms (one 128-token chunk of one KV head's
// row tile, or one chunk of one query's suffix) in processing order, cut into `grid` runs of about equal
// estimated time; consecutive atoms of one (head, tile) or (query, head) in a run form a segment.  Layout of
// `w`: seg_first [grid + 1] | segments | pre_range [2·H·nrt] | suf_range [2·Bq·H] (each range: the partial
// slots [first, end) of one output row group).  Returns the number of words used, or -1 if `cap` is too small
// or a row would have more than kMaxParts partials.
int build_worklist_fixed(const DecodeShape& s, const int32_t* host_ranks, int grid, int* w, int cap, int& nsegs,
                         int& off_segs, int& off_pre, int& off_suf, int& ipt_out, int& nrt_out,
                         const uint8_t* mask, int* off_sel) {
  const int H = s.H, nb = s.nb, D = s.d, G = s.Hq / s.H, Bq = s.Bq, S = s.S;
  const int cpb = s.n / kChunk;
  const int ipt = std::min(Bq, 128 / G);
  const int nrt = (Bq + ipt - 1) / ipt;
  const int nsc = (S + kChunk - 1) / kChunk;
  const int seg_words = (int)(sizeof(Seg) / sizeof(int));
  // prefix chunks are numbered along each head's walk: the k-th walked block (the k-th selected one under a
  // selection) holds chunks [k·cpb, k·cpb + cpb)
  auto for_each_atom = [&](auto&& fn) {
    for (int h = 0; h < H; ++h)
      for (int rt = 0; rt < nrt; ++rt) {
        int k = 0;
        for (int b = 0; b < nb; ++b) {
          if (mask && !mask[(size_t)h * nb + b]) continue;
          const int rk = host_ranks[(size_t)(2 * h) * nb + b], rv = host_ranks[(size_t)(2 * h + 1) * nb + b];
          for (int cc = 0; cc < cpb; ++cc) fn(0, h, rt, k * cpb + cc, prefix_atom_ns(rk, rv, cc, D));
          ++k;
        }
      }
    for (int i = 0; i < Bq; ++i)
      for (int h = 0; h < H; ++h)
        for (int c = 0; c < nsc; ++c)
          fn(1, h, i, c, suffix_atom_ns(c, D));
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
  const int nwords = off_suf + 2 * Bq * H + (mask ? H * nb : 0);
  if (nwords > cap) return -1;
  if (off_sel) *off_sel = mask ? off_suf + 2 * Bq * H : -1;
  if (mask) {  // the selected blocks of each head in order (entries past a head's count are unused)
    int* sel = w + off_suf + 2 * Bq * H;
    for (int h = 0; h < H; ++h) {
      int k = 0;
      for (int b = 0; b < nb; ++b)
        if (mask[(size_t)h * nb + b]) sel[(size_t)h * nb + k++] = b;
      for (; k < nb; ++k) sel[(size_t)h * nb + k] = 0;
    }
  }
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

// Work atoms of a decode shape (128-token chunks of every (KV head, row tile) walk and of every suffix).
int64_t count_atoms(const DecodeShape& s, const uint8_t* mask) {
  const int cpb = s.n / kChunk, nsc = (s.S + kChunk - 1) / kChunk;
  const int ipt = std::min(s.Bq, 128 / (s.Hq / s.H)), nrt = (s.Bq + ipt - 1) / ipt;
  int64_t blocks = (int64_t)s.H * s.nb;
  if (mask) {
    blocks = 0;
    for (int64_t i = 0; i < (int64_t)s.H * s.nb; ++i) blocks += mask[i] ? 1 : 0;
  }
  return blocks * nrt * cpb + (int64_t)s.Bq * s.H * nsc;
}
// The per-CTA work records for a work list `w` (build_worklist_fixed's layout): each CTA's segments with the
// rank and row offset of every block they walk (the k-th selected block of a head under a selection), the row
// offsets taken as the running sum of the ranks over pools and blocks in order (the factor layout).  A CTA
// whose work does not fit its record gets nseg = 0 and reads the global tables instead.
void build_records(const DecodeShape& s, const int32_t* host_ranks, const int* w, int grid, int off_segs,
                   int off_sel, CtaRec* recs) {
  const int nb = s.nb, cpb = s.n / kChunk;
  std::vector<int64_t> row0((size_t)2 * s.H * nb);
  int64_t acc = 0;
  for (size_t i = 0; i < row0.size(); ++i) {
    row0[i] = acc;
    acc += host_ranks[i];
  }
  const Seg* segs = reinterpret_cast<const Seg*>(w + off_segs);
  const int* sel = off_sel >= 0 ? w + off_sel : nullptr;
  for (int k = 0; k < grid; ++k) {
    CtaRec& r = recs[k];
    std::memset(&r, 0, sizeof(CtaRec));
    r.s_begin = w[k];
    r.s_end = w[k + 1];
    const int nseg = r.s_end - r.s_begin;
    int nblk = 0;
    bool fits = nseg <= kMaxSegsSmem;
    for (int i = 0; i < nseg && fits; ++i) {
      const Seg& sg = segs[r.s_begin + i];
      r.segs[i] = sg;
      r.blk0[i] = nblk;
      if (sg.type != 0) continue;
      for (int vb = sg.c0 / cpb; vb <= (sg.c1 - 1) / cpb; ++vb) {
        if (nblk >= kMaxBlocksSmem) {
          fits = false;
          break;
        }
        const int b = sel ? sel[(size_t)sg.h * nb + vb] : vb;
        BlockInfo& bi = r.blocks[nblk++];
        bi.rk = host_ranks[(size_t)(2 * sg.h) * nb + b];
        bi.rv = host_ranks[(size_t)(2 * sg.h + 1) * nb + b];
        bi.rowk = row0[(size_t)(2 * sg.h) * nb + b];
        bi.rowv = row0[(size_t)(2 * sg.h + 1) * nb + b];
      }
    }
    if (fits) {
      r.blk0[nseg] = nblk;
      r.nseg = nseg;
      r.nblk = nblk;
    } else {
      std::memset(r.blk0, 0, sizeof(r.blk0));
      r.nseg = 0;
      r.nblk = 0;
    }
  }
}
constexpr int kRecWords = (int)(sizeof(CtaRec) / sizeof(int));

// The producer's item list of every CTA, in the order the MMA warp consumes the data: per prefix segment the
// query tile, B_K of the first block, then per block U(0), U(1) (or B_K of the next block when the block has
// one chunk here), Q_V of the previous block, and per chunk j P(j) followed by U(j + 2) (or B_K of the next
// block in place of the first missing U), and finally Q_V of the last block; per suffix segment the query
// tile, K(0), K(1), then per chunk V(j) followed by K(j + 2).  Ring offsets follow the MMA warp's placement
// (an item that does not fit before the end of the ring starts at offset 0), and each ring item retires the
// oldest items in flight until its bytes are free and fewer than kItemSlots items are outstanding.  Writes
// at most `cap` items to `out` and sets every record's item range; returns the item count, or -1 when `cap` is
// too small, a coordinate does not fit the TMA's 32 bits or a rank lies outside [1, d].
int64_t build_items(const DecodeShape& s, const int32_t* host_ranks, const int* w, int grid, int off_segs,
                    int off_sel, CtaRec* recs, Item* out, int64_t cap, int mode) {
  const bool q8 = mode == kMode8bit, dk = mode == kModeDenseKeys;
  const uint32_t ring_bytes = q8 ? Smem<true>::kRingBytes : Smem<false>::kRingBytes;
  const int nb = s.nb, cpb = s.n / kChunk, G = s.Hq / s.H, ncb = s.d / 64;
  const int ipt = std::min(s.Bq, 128 / G);
  std::vector<int64_t> row0((size_t)2 * s.H * nb);
  int64_t acc = 0;
  for (size_t i = 0; i < row0.size(); ++i) {
    row0[i] = acc;
    acc += host_ranks[i];
  }
  const Seg* segs = reinterpret_cast<const Seg*>(w + off_segs);
  const int* sel = off_sel >= 0 ? w + off_sel : nullptr;
  auto pad = [](int r) { return (r + 15) & ~15; };
  bool fits = true;
  int64_t cnt = 0;
  auto push = [&](const Item& it) {
    if (cnt < cap) out[cnt] = it;
    else fits = false;
    ++cnt;
  };
  for (int k = 0; k < grid && fits; ++k) {
    recs[k].item0 = (int)cnt;
    uint32_t head = 0, n = 0, oldest = 0;  // the ring as the MMA warp places it
    uint32_t pos_of[kItemSlots];          // offsets of the items in flight (at most kItemSlots)
    auto ring = [&](int map, int64_t y, int rows, int nc) {  // `map`: the item's final map index
      if (y > INT32_MAX || rows < 16 || rows > 128) fits = false;
      const uint32_t bytes = (uint32_t)rows * 128u * nc;
      const uint32_t pos = head + bytes <= ring_bytes ? head : 0u;
      uint32_t retire = 0;
      while (oldest < n) {
        const uint32_t tail = pos_of[oldest % kItemSlots];
        const bool room = tail < head ? (pos + bytes <= tail || pos >= head) : (pos + bytes <= tail && pos >= head);
        if (room && n - oldest < (uint32_t)kItemSlots) break;
        ++oldest;
        ++retire;
      }
      head = pos + bytes;
      pos_of[n % kItemSlots] = pos;
      ++n;
      const uint32_t kind = nc == 2 ? kItem3D : kItem2D;
      push(Item{pos, (int32_t)y, bytes, (uint32_t)map | kind << 8 | retire << 16});
    };
    auto qtile = [&](int map, int y, int z, int box_rows) {
      push(Item{(uint32_t)z, y, (uint32_t)box_rows * 128u * ncb, (uint32_t)map | kItemQ << 8});
    };
    struct BI {
      int rk, rv;
      int64_t rowk, rowv;
      int b;  // the block's index in its pool
    };
    for (int si = w[k]; si < w[k + 1]; ++si) {
      const Seg& sg = segs[si];
      if (sg.type != 0) {
        qtile(kMapQsuf, sg.h * G, sg.tile, G);
        const int64_t r0 = ((int64_t)sg.tile * s.H + sg.h) * s.S;
        const int nc = sg.c1 - sg.c0;
        auto kv = [&](int map, int j) { ring(map, r0 + (int64_t)(sg.c0 + j) * kChunk, kChunk, ncb); };
        kv(kMapKsuf, 0);
        if (nc >= 2) kv(kMapKsuf, 1);
        for (int j = 0; j < nc; ++j) {
          kv(kMapVsuf, j);
          if (j + 2 < nc) kv(kMapKsuf, j + 2);
        }
        continue;
      }
      qtile(kMapQpre, sg.h * G, sg.tile * ipt, G * ipt);
      auto info = [&](int vb) {
        const int b = sel ? sel[(size_t)sg.h * nb + vb] : vb;
        const size_t ik = (size_t)(2 * sg.h) * nb + b, iv = (size_t)(2 * sg.h + 1) * nb + b;
        const BI r{host_ranks[ik], host_ranks[iv], row0[ik], row0[iv], b};
        if (r.rk < 1 || r.rk > s.d || r.rv < 1 || r.rv > s.d) fits = false;
        return r;
      };
      auto dim_item = [&](int64_t r0, int r) { ring(kMapDim + pad(r) / 16 - 1, r0, pad(r), ncb); };
      auto tok_item = [&](int64_t r0, int r, int cc) {
        // bf16: two 64-token column blocks; 8-bit: one 128-byte row of codes per component
        ring(kMapTok + pad(r) / 16 - 1, r0 * cpb + (int64_t)cc * r, pad(r), q8 ? 1 : 2);
      };
      // the keys of chunk cc of a block: its K factor slab, or (dense-key mode) 128 rows of the rotated keys
      auto key_item = [&](const BI& x, int cc) {
        if (dk) ring(kMapKrope, ((int64_t)sg.h * s.nb + x.b) * s.n + (int64_t)cc * kChunk, kChunk, ncb);
        else tok_item(x.rowk, x.rk, cc);
      };
      int c = sg.c0;
      BI bi = info(c / cpb), prev{};
      bool have_prev = false;
      if (!dk) dim_item(bi.rowk, bi.rk);
      while (true) {
        const int blk = c / cpb, cc0 = c - blk * cpb;
        const int nch = std::min(sg.c1, (blk + 1) * cpb) - c;
        const bool next = c + nch < sg.c1;
        const BI bn = next ? info(blk + 1) : BI{};
        key_item(bi, cc0);
        if (nch >= 2) key_item(bi, cc0 + 1);
        else if (next && !dk) dim_item(bn.rowk, bn.rk);
        if (have_prev) dim_item(prev.rowv, prev.rv);
        for (int j = 0; j < nch; ++j) {
          tok_item(bi.rowv, bi.rv, cc0 + j);
          if (j + 2 < nch) key_item(bi, cc0 + j + 2);
          else if (j + 2 == nch && next && !dk) dim_item(bn.rowk, bn.rk);
        }
        if (!next) break;
        prev = bi;
        have_prev = true;
        c += nch;
        bi = bn;
      }
      dim_item(bi.rowv, bi.rv);
    }
    recs[k].nitems = (int)(cnt - recs[k].item0);
  }
  return fits && cnt <= INT32_MAX ? cnt : -1;
}
constexpr int kItemWords = (int)(sizeof(Item) / sizeof(int));
// Items of a work list at most: per atom (a 128-token chunk) its two ring items, and per segment (at most one
// per atom) a query tile and per block visit (at most one per atom) two dim-factor items.
int64_t items_cap(const DecodeShape& s, const uint8_t* mask = nullptr) { return 5 * count_atoms(s, mask); }

// CTAs of the decode kernel: one per SM, fewer when there are fewer atoms.
int plan_grid(const DecodeShape& s, int sms, const uint8_t* mask = nullptr) {
  return (int)std::max<int64_t>(1, std::min<int64_t>(sms, count_atoms(s, mask)));
}
// Words a work list can need at most (every atom its own segment).
int64_t worklist_cap(const DecodeShape& s, int grid, const uint8_t* mask = nullptr) {
  const int ipt = std::min(s.Bq, 128 / (s.Hq / s.H)), nrt = (s.Bq + ipt - 1) / ipt;
  return grid + 1 + count_atoms(s, mask) * (int64_t)(sizeof(Seg) / sizeof(int)) + 2LL * s.H * nrt +
         2LL * s.Bq * s.H + (mask ? (int64_t)s.H * s.nb : 0);
}

static cudaError_t build_plan(TcPlan* pl, const DecodeShape& s, const TcInputs& in, const uint8_t* mask) {
  const int D = s.d;
  const int cpb = s.n / kChunk;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int grid = plan_grid(s, sms, mask);
  const int64_t cap = worklist_cap(s, grid, mask);
  if (cap > (int64_t)1 << 30) return cudaErrorInvalidValue;
  std::vector<int> host((size_t)cap + 4 + (size_t)grid * kRecWords);
  int nsegs = 0, off_segs = 0, off_pre = 0, off_suf = 0, ipt = 0, nrt = 0;
  const int nwords = build_worklist_fixed(s, in.host_ranks, grid, host.data(), (int)cap, nsegs, off_segs, off_pre,
                                          off_suf, ipt, nrt, mask, &pl->off_sel);
  if (mask) pl->mask.assign(mask, mask + (size_t)s.H * s.nb);
  if (nwords < 0) return cudaErrorInvalidValue;
  // per-CTA records after the work list, then the producer items, each 16-byte aligned
  pl->off_rec = (nwords + 3) & ~3;
  CtaRec* recs = reinterpret_cast<CtaRec*>(host.data() + pl->off_rec);
  build_records(s, in.host_ranks, host.data(), grid, off_segs, pl->off_sel, recs);
  const int off_items = pl->off_rec + grid * kRecWords;
  const int64_t icap = items_cap(s, mask);
  host.resize((size_t)off_items + (size_t)icap * kItemWords);
  recs = reinterpret_cast<CtaRec*>(host.data() + pl->off_rec);
  const int64_t nitems = build_items(s, in.host_ranks, host.data(), grid, off_segs, pl->off_sel, recs,
                                     reinterpret_cast<Item*>(host.data() + off_items), icap, mode_of(in));
  if (nitems < 0 || off_items + nitems * kItemWords > INT32_MAX) return cudaErrorInvalidValue;
  pl->off_items = off_items;
  const int nwords_all = (int)(off_items + nitems * kItemWords);
  pl->off_segs = off_segs;
  pl->off_pre = off_pre;
  pl->off_suf = off_suf;
  cudaError_t e;
  if ((e = cudaMalloc((void**)&pl->d_work, (size_t)nwords_all * sizeof(int))) != cudaSuccess) return e;
  if ((e = cudaMemcpy(pl->d_work, host.data(), (size_t)nwords_all * sizeof(int), cudaMemcpyHostToDevice)) !=
      cudaSuccess)
    return e;
  const size_t np = std::max<size_t>(1, (size_t)nsegs);
  if ((e = cudaMalloc((void**)&pl->part_acc, np * 128 * D * sizeof(float))) != cudaSuccess) return e;
  if ((e = cudaMalloc((void**)&pl->part_ml, np * 128 * sizeof(float2))) != cudaSuccess) return e;
  pl->Bq = s.Bq;
  pl->Hq = s.Hq;
  pl->S = s.S;
  pl->grid = grid;
  pl->nsegs = nsegs;
  pl->ipt = ipt;
  pl->nrt = nrt;
  // factor maps: the token factor as a [rows · n/128][128] array of 128-token slab rows, the dim factor
  // as [rows][d]
  const uint64_t rows = (uint64_t)in.total_rows;
  PlanMaps pm;
  if (!(in.q8 ? make_code_maps(&pm.tok, in.tok, rows * cpb) : make_row_maps(&pm.tok, in.tok, kChunk, rows * cpb)))
    return cudaErrorInvalidValue;
  if (!make_row_maps(&pm.dim, in.dim, D, rows)) return cudaErrorInvalidValue;
  if (!make_pacc_map(&pm.pacc, pl->part_acc, pl->nsegs, D)) return cudaErrorInvalidValue;
  if ((e = cudaMalloc((void**)&pl->d_maps, sizeof(PlanMaps))) != cudaSuccess) return e;
  if ((e = cudaMemcpy(pl->d_maps, &pm, sizeof(PlanMaps), cudaMemcpyHostToDevice)) != cudaSuccess) return e;
  pl->tok = in.tok;
  pl->dim = in.dim;
  pl->q8 = in.q8;
  pl->rope = in.rope_keys;
  if (in.rope_keys &&
      (e = cudaMalloc(&pl->krope, (size_t)s.H * s.nb * s.n * s.d * 2)) != cudaSuccess)
    return e;
  return prepare_kernel(D, mode_of(in));
}

cudaError_t tc_decode(TcPlan** plan, const DecodeShape& s, const TcInputs& in, void* out, cudaStream_t st,
                      cudaEvent_t ev0, cudaEvent_t ev1, const uint8_t* mask) {
  TcPlan* pl = *plan;
  const bool same_mask = pl && (mask ? pl->mask.size() == (size_t)s.H * s.nb &&
                                           std::memcmp(pl->mask.data(), mask, pl->mask.size()) == 0
                                     : pl->mask.empty());
  if (!pl || pl->Bq != s.Bq || pl->Hq != s.Hq || pl->S != s.S || pl->tok != in.tok || pl->q8 != in.q8 ||
      pl->rope != in.rope_keys || !same_mask) {
    tc_plan_destroy(pl);
    *plan = nullptr;
    pl = new TcPlan();
    cudaError_t e = build_plan(pl, s, in, mask);
    if (e != cudaSuccess) {
      tc_plan_destroy(pl);
      return e;
    }
    *plan = pl;
  }
  const int D = s.d, G = s.Hq / s.H;
  Maps maps;
  if (!make_call_maps(&maps, s, in, pl->ipt)) return cudaErrorInvalidValue;
  if (in.rope_keys) {
    // the prefix keys, rebuilt from their pre-RoPE factors and rotated, as [H·T][d] rows
    if (!make_rows_map(&maps.krope, pl->krope, D, (uint64_t)s.H * s.nb * s.n, kChunk)) return cudaErrorInvalidValue;
    const RopeShape rs{s.H, s.nb, s.n, s.d, in.rope_theta};
    const CUtensorMap* pmaps = reinterpret_cast<const CUtensorMap*>(pl->d_maps);
    const RopeBuffers rb{pmaps + kMapTok, pmaps + kMapDim, in.ranks, in.row_offsets, &maps.krope, in.status};
    cudaError_t re = launch_rope_keys(rs, rb, st);
    if (re != cudaSuccess) return re;
  }
  Params p;
  p.recs = reinterpret_cast<const CtaRec*>(pl->d_work + pl->off_rec);
  p.items = reinterpret_cast<const Item*>(pl->d_work + pl->off_items);
  p.gmaps = pl->d_maps;
  p.segs = reinterpret_cast<const Seg*>(pl->d_work + pl->off_segs);
  p.ranks = in.ranks;
  p.row_offsets = in.row_offsets;
  p.part_acc = pl->part_acc;
  p.part_ml = pl->part_ml;
  p.sel = pl->off_sel >= 0 ? pl->d_work + pl->off_sel : nullptr;
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
  e = launch_decode_kernel(D, mode_of(in), pl->grid, maps, p, st);
  if (e != cudaSuccess) return e;
  if (ev1 && (e = cudaEventRecord(ev1, st)) != cudaSuccess) return e;
  const int* pre = pl->d_work + pl->off_pre;
  const int* suf = pl->d_work + pl->off_suf;
  return launch_combine(s, pl->part_acc, pl->part_ml, pre, suf, pl->ipt, pl->nrt, out, st);
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
bool g_noalloc_ready[kNoAllocMaxDevices][4];  // decode kernel prepared on the device, per (head dim, 8-bit mode)
alignas(16) int g_noalloc_host_words[kNoAllocMaxWords];  // work list and records staging, guarded by g_noalloc_mu

}  // namespace

int tc_worklist(const DecodeShape& s, const int32_t* host_ranks, int sms, int* w, int64_t cap, int64_t* info) {
  if (cap > INT32_MAX) cap = INT32_MAX;
  const int grid = plan_grid(s, sms);
  int nsegs = 0, off_segs = 0, off_pre = 0, off_suf = 0, ipt = 0, nrt = 0;
  const int nwords = build_worklist_fixed(s, host_ranks, grid, w, (int)cap, nsegs, off_segs, off_pre, off_suf, ipt,
                                          nrt, nullptr, nullptr);
  if (nwords < 0) return -1;
  const int64_t v[8] = {nwords, nsegs, grid, off_segs, off_pre, off_suf, ipt, nrt};
  for (int i = 0; i < 8; ++i) info[i] = v[i];
  return nwords;
}

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
  }
  const int kind = (s.d == 64 ? 0 : 1) + (in.q8 ? 2 : 0);
  if (!g_noalloc_ready[dev][kind]) {
    if ((e = prepare_kernel(s.d, mode_of(in))) != cudaSuccess) return e;
    g_noalloc_ready[dev][kind] = true;
  }
  unsigned char* scratch = static_cast<unsigned char*>(g_noalloc_dev_ptr[dev]);
  int sms = 148;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  const int cpb = s.n / kChunk;
  const int grid = plan_grid(s, sms);
  int nsegs = 0, off_segs = 0, off_pre = 0, off_suf = 0, ipt = 0, nrt = 0;
  // the work list, then the per-CTA records (16-byte aligned) in the same staging buffer
  const int rec_words = grid * kRecWords;
  int nwords = build_worklist_fixed(s, in.host_ranks, grid, g_noalloc_host_words, kNoAllocMaxWords - rec_words - 4,
                                    nsegs, off_segs, off_pre, off_suf, ipt, nrt, nullptr, nullptr);
  int off_rec = 0, off_items = 0;
  if (nwords >= 0) {
    off_rec = (nwords + 3) & ~3;
    CtaRec* recs = reinterpret_cast<CtaRec*>(g_noalloc_host_words + off_rec);
    build_records(s, in.host_ranks, g_noalloc_host_words, grid, off_segs, -1, recs);
    off_items = off_rec + rec_words;
    const int64_t room = ((int64_t)kNoAllocMaxWords - off_items) / kItemWords;
    const int64_t nitems = room > 0 ? build_items(s, in.host_ranks, g_noalloc_host_words, grid, off_segs, -1, recs,
                                                  reinterpret_cast<Item*>(g_noalloc_host_words + off_items), room,
                                                  mode_of(in))
                                    : -1;
    nwords = nitems < 0 ? -1 : (int)(off_items + nitems * kItemWords);
  }
  // the plan's maps after the items, 128-byte aligned
  constexpr int kMapWords = (int)(sizeof(PlanMaps) / sizeof(int));
  const int off_maps = (std::max(nwords, 0) + 31) & ~31;
  if (nwords >= 0) nwords = off_maps + kMapWords <= kNoAllocMaxWords ? off_maps + kMapWords : -1;
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
  const int D = s.d, G = s.Hq / s.H;
  PlanMaps pm;
  const uint64_t rows = (uint64_t)in.total_rows;
  if (!(in.q8 ? make_code_maps(&pm.tok, in.tok, rows * cpb) : make_row_maps(&pm.tok, in.tok, kChunk, rows * cpb)))
    return cudaErrorInvalidValue;
  if (!make_row_maps(&pm.dim, in.dim, D, rows)) return cudaErrorInvalidValue;
  if (!make_pacc_map(&pm.pacc, part_acc, nsegs, D)) return cudaErrorInvalidValue;
  std::memcpy(g_noalloc_host_words + off_maps, &pm, sizeof(PlanMaps));
  // pageable source: the call returns once the words are staged, so the host buffer can be reused
  if ((e = cudaMemcpyAsync(d_work, g_noalloc_host_words, (size_t)nwords * sizeof(int), cudaMemcpyHostToDevice, st)) !=
      cudaSuccess)
    return e;
  Maps maps;
  if (!make_call_maps(&maps, s, in, ipt)) return cudaErrorInvalidValue;
  Params p;
  p.recs = reinterpret_cast<const CtaRec*>(d_work + off_rec);
  p.items = reinterpret_cast<const Item*>(d_work + off_items);
  p.gmaps = reinterpret_cast<const PlanMaps*>(d_work + off_maps);
  p.segs = reinterpret_cast<const Seg*>(d_work + off_segs);
  p.ranks = in.ranks;
  p.row_offsets = in.row_offsets;
  p.part_acc = part_acc;
  p.part_ml = part_ml;
  p.sel = nullptr;
  p.status = in.status;
  p.nb = s.nb;
  p.cpb = cpb;
  p.H = s.H;
  p.G = G;
  p.ipt = ipt;
  p.S = s.S;
  p.c = s.scale * 1.4426950408889634f;
  if ((e = launch_decode_kernel(D, mode_of(in), grid, maps, p, st)) != cudaSuccess) return e;
  return launch_combine(s, part_acc, part_ml, d_work + off_pre, d_work + off_suf, ipt, nrt, out, st);
}

}  // namespace milo
