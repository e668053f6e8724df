/*
 * milo.h — C ABI of the B200 (sm_100a) compressed-KV decode attention library.
 *
 * The method is MILO (page "MILO: Efficient Many-shot In-Context Learning with
 * Block-wise Low-rank Compression"):
 *   §4.2  the many-shot KV cache is split into blocks of several examples and
 *         each block's keys and values get their own low-rank approximation;
 *   §4.3  the ranks of the blocks come from their entropy under a fixed total
 *         rank budget;
 *   §4.4  encoding partitions the context, analyses entropy and stores the
 *         low-rank caches; decoding attends over them.
 *
 * Two calls carry the method: milo_compress (encode) and milo_decode_attn
 * (decode).  Everything else manages the factor object they share.
 *
 * Conventions for every call:
 *  - All tensors are dense, row-major, and live in device memory unless a
 *    parameter says "host".  The library never takes ownership of a caller's
 *    buffer and never keeps a pointer to it after the call returns.
 *  - `stream` is a cudaStream_t passed as void* (NULL = the legacy default
 *    stream).  Calls are asynchronous on it unless marked "synchronises".
 *  - Errors are reported only through the return value.  Invalid arguments
 *    are rejected before anything is launched or allocated.  Errors found by
 *    a kernel (non-convergence, a failed bounds check, an expired wait) are
 *    recorded in the factor object's device status word and read back by
 *    milo_factors_status.  No call aborts the process or traps the GPU.
 *  - There is no CPU fallback: without an sm_100 device every compute call
 *    returns MILO_ERR_CUDA.
 *
 * Layout of a factor object (one layer):
 *   pool p = 2*h + t for KV head h and tensor t (0 = keys, 1 = values);
 *   block b of pool p has rank r = ranks[p*nb + b] and owns rows
 *   [row0, row0 + r), row0 = row_offsets[p*(nb+1) + b], of two arrays:
 *     dim  [rows][d]  dimension-side factor: row row0+j is column j of B_b
 *     tok  r·n elements from element row0·n: the token-side factor
 *          U_b = X_b·B_b (X_b the n×d block) transposed and cut into
 *          128-token slabs, element (j, t) at
 *          row0·n + (t / 128)·(r·128) + j·128 + (t % 128)
 *   so that X_b ≈ U_b · B_bᵀ.  The blocks of a pool are consecutive and the
 *   pools follow each other (pool p starts at row p * pool_rows when every pool
 *   has the same rank sum).  Factor elements have the dtype of the compressed
 *   cache, except in 8-bit objects (MILO_I8, made by milo_factors_quantize):
 *   there tok holds int8 codes and dim holds bf16, and every block carries one
 *   more component than it was compressed with (see milo_factors_quantize).
 */
#ifndef MILO_H_
#define MILO_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MILO_ABI_VERSION 4

typedef enum {
  MILO_OK = 0,
  MILO_ERR_INVALID_ARGUMENT = 1, /* a shape, pointer or option is out of range  */
  MILO_ERR_UNSUPPORTED = 2,      /* valid in principle, not built (e.g. d = 96) */
  MILO_ERR_BUDGET = 3,           /* budget below num_blocks * r_min             */
  MILO_ERR_NO_CONVERGENCE = 4,   /* eigensolver hit max_sweeps                  */
  MILO_ERR_DEVICE_CHECK = 5,     /* a kernel's bounds check or bounded wait failed */
  MILO_ERR_CUDA = 6,             /* a CUDA runtime/driver call failed           */
  MILO_ERR_OUT_OF_MEMORY = 7
} milo_status;

/* MILO_I8 describes factor objects only: int8 token factors, bf16 dimension factors. */
typedef enum { MILO_F32 = 0, MILO_BF16 = 1, MILO_I8 = 2 } milo_dtype;

/* milo_compress flags */
#define MILO_KEEP_INTERMEDIATES 1u /* keep fp32 eigenpairs, fp64 entropies and quotas */

typedef struct milo_factors milo_factors; /* opaque, device-resident, library-owned */

/* Allocation rules (milo_compress_rule): the entropy rule of §4.3, the greedy marginal-gain
 * form §4.3 describes in words, and the uniform and random baselines of §5.3 (random: the
 * caller draws the weights and passes them in). */
typedef enum {
  MILO_ALLOC_ENTROPY = 0, /* ranks ∝ exp(H_b), water-filling, largest remainder (milo_compress) */
  MILO_ALLOC_GREEDY = 1,  /* from r_min, each unit to the largest next-component energy share */
  MILO_ALLOC_UNIFORM = 2, /* floor(R / blocks) each, the remainder to the lowest block indices */
  MILO_ALLOC_WEIGHTS = 3  /* ranks ∝ caller weights, with the entropy rule's water-filling */
} milo_alloc_rule;
/* Budget scope: R = floor(budget*T*d/(n+d)) rank units per pool (one KV head's keys or values),
 * or P·R units shared by all P = 2H pools of the layer (blocks ordered pool p = 2h + t, then block). */
typedef enum { MILO_POOL_HEAD = 0, MILO_POOL_LAYER = 1 } milo_pool_scope;

typedef struct {
  int32_t num_kv_heads;  /* H */
  int32_t num_blocks;    /* nb = context / block_size */
  int32_t block_size;    /* n */
  int32_t head_dim;      /* d */
  int64_t context;       /* T */
  int32_t r_min;
  int32_t pool_rows;     /* rows per pool = min(R, nb*d), R = floor(budget*T*d/(n+d)); 0 if pools differ */
  int32_t dtype;         /* milo_dtype */
  int32_t alloc_rule;    /* milo_alloc_rule */
  int32_t pool_scope;    /* milo_pool_scope */
  int32_t reserved;
  int64_t total_rows;    /* rows of tok (in units of n) and dim: Σ of every block's rank */
  const int32_t* ranks;       /* device [2H][nb]                         */
  const int64_t* row_offsets; /* device [2H][nb+1]                       */
  const void* tok;            /* device, 2H*pool_rows*n elements (slabs)  */
  const void* dim;            /* device [2H*pool_rows][d]                */
  /* present only with MILO_KEEP_INTERMEDIATES, else NULL: */
  const float* eigvals;       /* device [2H][nb][d], descending (λ_i = σ_i²)           */
  const float* eigvecs;       /* device [2H][nb][d][d], row i = eigenvector of λ_i      */
  const double* entropy;      /* device [2H][nb], H_b                                  */
  const double* quotas;       /* device [2H][nb], real quotas before rounding          */
  /* present for objects made by milo_compress (NULL for imported ones): */
  const int32_t* sweeps;      /* device [2H][nb], Jacobi sweeps run per block (the last  */
                              /* one rotated no pair or left every relative off-diagonal  */
                              /* below 3e-4; max_sweeps means no convergence)             */
} milo_factors_desc;

/*
 * milo_compress — encode one layer's KV cache into per-block low-rank factors.
 * Source: §4.2 (block partition, separate low-rank approximation of each
 * block's keys and values) and §4.3 (ranks from block entropy under a total
 * budget).  Steps, all on `stream`: per block the Gram matrix X_bᵀX_b (fp32),
 * its eigen-decomposition by one-sided Jacobi (λ_i = σ_i², eigenvectors = the
 * right singular vectors), the spectral entropy H_b = −Σ p_i ln p_i with
 * p_i = λ_i/Σλ, ranks ∝ exp(H_b) summing to R = floor(budget·T·d/(n+d)) per
 * pool (clamped to [r_min, d], largest-remainder rounding), and the
 * projection U_b = X_b·B_b[:, :r_b].
 *   K, V        device [H][T][d] in `dtype`; read only.
 *   block_size  n: T % n == 0, n % 128 == 0, n >= d; at most 8192 blocks
 *               (T / n) per pool, else MILO_ERR_UNSUPPORTED.
 *   head_dim    d ∈ {64, 128}.
 *   budget      storage budget > 0 (fraction of the raw cache; > 1 allowed).
 *   r_min       1 <= r_min <= d; MILO_ERR_BUDGET if R < nb*r_min.
 *   max_sweeps  Jacobi sweep limit, 0 = default (30).  Hitting it sets
 *               MILO_ERR_NO_CONVERGENCE in the status word (not the return).
 *   flags       MILO_KEEP_INTERMEDIATES or 0.
 *   out         receives a new factor object; destroy with milo_factors_destroy.
 * Allocates device memory (cudaMalloc) for the factor object and its scratch;
 * does not synchronise.
 */
milo_status milo_compress(const void* K, const void* V, int32_t dtype, int32_t num_kv_heads,
                          int64_t context, int32_t head_dim, int32_t block_size, double budget,
                          int32_t r_min, int32_t max_sweeps, uint32_t flags, void* stream,
                          milo_factors** out);

/*
 * milo_compress_rule — milo_compress with a chosen allocation rule and budget
 * scope (§4.3's greedy form, §5.3's uniform and random baselines, and a
 * layer-wide budget; see milo_alloc_rule and milo_pool_scope).  The Gram,
 * eigen-decomposition and projection steps are those of milo_compress.
 *   rule          milo_alloc_rule.
 *   scope         milo_pool_scope; MILO_POOL_LAYER allocates one budget of
 *                 2H·R units over all 2H·nb blocks (at most 8192 blocks).
 *   host_weights  host [2H][nb], finite and > 0, for MILO_ALLOC_WEIGHTS only
 *                 (NULL otherwise); copied before the call returns.
 * The greedy rule takes its decisions on the fp32 eigenvalues in fp64 (shares
 * λ_i/Σλ); the quotas intermediate is NaN for the greedy and uniform rules.
 * Other arguments, results and errors as milo_compress.
 */
milo_status milo_compress_rule(const void* K, const void* V, int32_t dtype, int32_t num_kv_heads,
                               int64_t context, int32_t head_dim, int32_t block_size, double budget,
                               int32_t r_min, int32_t max_sweeps, uint32_t flags, int32_t rule,
                               int32_t scope, const double* host_weights, void* stream,
                               milo_factors** out);

/*
 * milo_compress_profiled — milo_compress that also records caller-created CUDA
 * events (cudaEvent_t passed as void*) on `stream` between its kernels:
 * events[0] before the Gram kernel, events[1] before the Jacobi eigensolver,
 * events[2] before the entropy and rank allocation kernel, events[3] before the
 * projection kernel and events[4] after it, so cudaEventElapsedTime between
 * neighbours gives each step's duration.  `events` is host memory, 5 entries,
 * any of them NULL (not recorded); events itself may be NULL.  Same arguments,
 * results and errors as milo_compress otherwise.
 */
milo_status milo_compress_profiled(const void* K, const void* V, int32_t dtype, int32_t num_kv_heads,
                                   int64_t context, int32_t head_dim, int32_t block_size, double budget,
                                   int32_t r_min, int32_t max_sweeps, uint32_t flags, void* stream,
                                   milo_factors** out, void* const* events);

/*
 * milo_decode_attn — one decode step of softmax attention over the compressed
 * prefix and each query's uncompressed suffix.
 * Source: §4.4 (inference attends over the stored low-rank caches).  Every
 * block is attended (no selection).  Computed in rank space: per block
 * q̃ = q·B_b, scores = scale·q̃·U_bᵀ, one online softmax over all blocks and
 * the suffix, value sum (p·P_b)·Q_bᵀ.  Query head hq reads KV head
 * hq / (num_q_heads / H).
 *   q         device [batch][num_q_heads][d], dtype of the factors.
 *   f         factor object from milo_compress or milo_factors_import.
 *   K_suffix, V_suffix  device [batch][H][suffix_len][d]; may be NULL when
 *             suffix_len == 0.
 *   scale     softmax scale; <= 0 selects 1/sqrt(d).
 *   out       device [batch][num_q_heads][d], dtype of the factors.
 * The first call for a given (batch, num_q_heads, suffix_len) synchronises
 * `stream` once to read the ranks and build the work list, and may allocate
 * scratch; later calls with the same shape do neither, so they can be captured
 * in a CUDA graph (make one call with the shape before capturing, and let the
 * factors be complete before the capture starts).  Calls that share a factor
 * object share its scratch and must be ordered on one stream.
 */
milo_status milo_decode_attn(const void* q, int32_t batch, int32_t num_q_heads,
                             const milo_factors* f, const void* K_suffix, const void* V_suffix,
                             int32_t suffix_len, float scale, void* out, void* stream);

/*
 * milo_decode_attn_select — milo_decode_attn over a selection of the
 * compressed blocks.  Source: §4.4 (decoding retrieves the selected blocks and
 * attends over them sparsely).  The blocks of KV head h that the mask leaves
 * out take no part in the softmax of any query of that head; the suffix is
 * always attended.
 *   host_block_mask  host [H][nb], nonzero = attend; read during the call only.
 * The selection is applied through the work list: a call whose mask differs
 * from the previous call's on this factor object rebuilds it (one host-to-
 * device copy, and scratch allocation when it grows), so a fixed selection
 * costs nothing extra.  bf16 factors only (MILO_ERR_UNSUPPORTED for fp32).
 * MILO_ERR_INVALID_ARGUMENT when suffix_len == 0 and some head selects no
 * block.  Other arguments, results and errors as milo_decode_attn.
 */
milo_status milo_decode_attn_select(const void* q, int32_t batch, int32_t num_q_heads,
                                    const milo_factors* f, const void* K_suffix, const void* V_suffix,
                                    int32_t suffix_len, float scale, const uint8_t* host_block_mask,
                                    void* out, void* stream);

/*
 * milo_decode_attn_rope — milo_decode_attn for factors of keys compressed before
 * the rotary embedding.  Source: §3 and Figure 1 (pre-RoPE keys are more
 * low-rank, which suits block-wise compression) and §4.4–§4.5 (inference
 * reconstructs the selected blocks before attention).  The rank-space identity
 * does not hold for rotated keys (the rotation depends on the token), so this
 * call first rebuilds every key block K_b = U_b·B_bᵀ and rotates each token t of
 * the prefix at its absolute position t: dimension i < d/2 pairs with i + d/2
 * and the pair turns by t·rope_theta^(−2i/d),
 *   y_i = x_i·cos φ − x_{i+d/2}·sin φ,  y_{i+d/2} = x_{i+d/2}·cos φ + x_i·sin φ,
 * into a [H][T][d] bf16 scratch held by the factor object; the decode then
 * scores q against those keys densely, with the values in rank space as in
 * milo_decode_attn.  q and the suffix keys are taken as already rotated at
 * their own positions.
 *   rope_theta       rotary base, > 1 (the Qwen2.5 models use 1e6).
 *   host_block_mask  NULL (every block) or host [H][nb] as in milo_decode_attn_select.
 * bf16 factor objects only (MILO_ERR_UNSUPPORTED for fp32 and 8-bit objects).
 * Three launches per call.  The first call for a shape allocates the scratch
 * (H·T·d·2 bytes) besides the usual work list.  Other arguments, results and
 * errors as milo_decode_attn.
 */
milo_status milo_decode_attn_rope(const void* q, int32_t batch, int32_t num_q_heads,
                                  const milo_factors* f, const void* K_suffix, const void* V_suffix,
                                  int32_t suffix_len, float scale, double rope_theta,
                                  const uint8_t* host_block_mask, void* out, void* stream);

/*
 * milo_decode_attn_profiled — milo_decode_attn that also records two caller-created
 * CUDA events (cudaEvent_t passed as void*, NULL = skip) on `stream`: event_before
 * right before the main per-block decode kernel and event_after right after it,
 * before the combine kernel, so cudaEventElapsedTime gives that kernel's duration.
 * Same arguments, results and errors as milo_decode_attn otherwise.
 */
milo_status milo_decode_attn_profiled(const void* q, int32_t batch, int32_t num_q_heads,
                                      const milo_factors* f, const void* K_suffix,
                                      const void* V_suffix, int32_t suffix_len, float scale,
                                      void* out, void* stream, void* event_before,
                                      void* event_after);

/*
 * milo_decode_attn_noalloc — milo_decode_attn for callers that cannot allocate
 * device memory.  The pages have no counterpart: it is a deployment variant.
 * Who needs it: code that runs where cudaMalloc is not allowed or not wanted —
 * inside a serving engine whose allocator owns all device memory and forbids
 * side allocations (a cudaMalloc there can fail, or take memory the engine has
 * promised elsewhere), or on a latency-critical path that cannot afford the
 * device-wide synchronisation that cudaMalloc and cudaFree imply.  milo_decode_attn allocates its work list
 * and partials on the first call for a shape; this entry point allocates nothing
 * (no cudaMalloc, cudaFree, or allocating library routine) and keeps both in one
 * fixed array in device memory of MILO_NOALLOC_SCRATCH_BYTES (32 MiB) that every
 * GPU loading the library holds until the process exits.
 *   Arguments, layout and results: as milo_decode_attn, for bf16 factors only
 *   (MILO_ERR_UNSUPPORTED for fp32).
 *   Size limit: a shape whose work list plus partials (about 66 KB per work
 *   segment at d = 128; the Qwen2.5-7B layer at batch 16 needs about 15 MB)
 *   exceed the array returns MILO_ERR_UNSUPPORTED before anything is launched.
 *   Set-up: the first call on a device looks up the array's device address
 *   (cudaGetSymbolAddress, with that device current); make that first call
 *   before any stream capture.  The first decode call of a factor object
 *   (through this entry point or milo_decode_attn) synchronises once on the
 *   factors to read their ranks into a host copy that was sized when the
 *   object was made; later calls neither synchronise nor allocate for it.
 *   Sharing: every call on a device uses the same array and leaves its contents
 *   behind; each call writes every scratch word it reads, so nothing has to
 *   start at zero, but calls that overlap on the GPU (different streams, or
 *   different factor objects at once) race on it and must be serialised.
 */
#define MILO_NOALLOC_SCRATCH_BYTES (32u << 20)
milo_status milo_decode_attn_noalloc(const void* q, int32_t batch, int32_t num_q_heads,
                                     const milo_factors* f, const void* K_suffix,
                                     const void* V_suffix, int32_t suffix_len, float scale,
                                     void* out, void* stream);

/*
 * Number of kernels one milo_decode_attn call with these arguments launches
 * (>= 1), or a negative milo_status for invalid arguments.  Host-only, no GPU work.
 */
int32_t milo_decode_launches(const milo_factors* f, int32_t batch, int32_t num_q_heads, int32_t suffix_len);

/*
 * Host only (no GPU, no CUDA call): the work list that the bf16 tensor-core decode builds for these ranks
 * and this decode shape on a GPU with num_ctas SMs (one CTA per SM, fewer when there are fewer chunks
 * than SMs), for inspection and testing.  The
 * decode splits the compressed prefix of each (KV head, row tile) into 128-token chunks and each query's
 * suffix into 128-token chunks (the rank-space decode of page "MILO", §4.4), and cuts the sequence of
 * chunks into one run per CTA of about equal estimated time.
 *   host_ranks  [2H][nb] int32 (per head: K ranks, then V ranks), each in [1, head_dim]; caller-owned.
 *   out         capacity int32 words, written: seg_first [CTAs + 1] | segments, 8 words each
 *               {kind (0 prefix, 1 suffix), KV head, row tile (prefix) or query (suffix), first chunk,
 *               end chunk, partial slot, valid rows, 0} | pre_range [2·H·tiles] | suf_range [2·batch·H]
 *               (each range: the [first, end) partial slots of one output row group).
 *   info        8 int64, written: {words used, segments, CTAs, offset of the segments, offset of
 *               pre_range, offset of suf_range, query items per row tile, row tiles per head}.
 * Errors: MILO_ERR_INVALID_ARGUMENT for a bad shape or rank, MILO_ERR_UNSUPPORTED for a shape the
 * tensor-core decode does not take or a capacity that is too small.
 */
milo_status milo_decode_worklist(const int32_t* host_ranks, int32_t num_kv_heads, int32_t num_blocks,
                                 int32_t block_size, int32_t head_dim, int32_t batch, int32_t num_q_heads,
                                 int32_t suffix_len, int32_t num_ctas, int32_t* out, int64_t capacity,
                                 int64_t* info);

/* Copies the ranks [2H][nb] to host memory. Synchronises the compress stream. */
milo_status milo_factors_ranks(const milo_factors* f, int32_t* host_ranks);

/* Fills *desc with the shape and the device pointers of f (valid until destroy). */
milo_status milo_factors_describe(const milo_factors* f, milo_factors_desc* desc);

/*
 * Synchronises the device and returns the first error recorded by a kernel
 * for f (MILO_OK if none).  *host_bits (optional) receives the raw bit mask:
 * 1 = Jacobi did not converge, 2 = compress bounds check, 4 = decode bounds
 * check, 8 = decode wait expired, 16 = compress (Gram) wait expired.
 */
milo_status milo_factors_status(const milo_factors* f, uint32_t* host_bits);

/*
 * Builds a factor object from host arrays in the layout above (a copy), e.g.
 * factors computed elsewhere or saved earlier.  host_ranks [2H][nb], each in
 * [1, d]; host_tok [rows][n] and host_dim [rows][d] in `dtype`, rows = Σ of all
 * ranks, pools in order (their sums may differ, as with a layer-wide budget);
 * host_tok holds each block's 128-token slabs as described above.  With
 * dtype MILO_I8, host_tok is int8 codes and host_dim bf16 (the form
 * milo_factors_quantize writes, each rank counting the extra component).
 * Synchronises `stream`.
 */
milo_status milo_factors_import(int32_t dtype, int32_t num_kv_heads, int64_t context,
                                int32_t head_dim, int32_t block_size, int32_t r_min,
                                const int32_t* host_ranks, const void* host_tok,
                                const void* host_dim, void* stream, milo_factors** out);

/*
 * milo_factors_quantize — 8-bit storage of a bf16 factor object's token factors.
 * Source: §5.3 (the compressed caches compose with asymmetric INT8 and KIVI
 * quantisation for further memory savings).  The page names no scheme; this is
 * asymmetric INT8 per rank channel of each block (KIVI's per-channel rule for
 * keys, applied to the token factors U_b and P_b alike):
 *   channel j of block b, values x_t over the block's n tokens:
 *     lo = min x_t, a = (max x_t − lo)/255, code c_t = round((x_t − lo)/a) − 128
 *     in [−128, 127], rounded half to even, all in fp32; a = 0 gives c_t = −128;
 *   the scales and minima are folded into the bf16 dimension factor with one
 *   extra component per block whose codes are all 1:
 *     dim row j = a_j·B_b[:, j] (j < r),  dim row r = Σ_j (lo_j + 128·a_j)·B_b[:, j],
 *   so that codes·dimᵀ is the dequantized block exactly.
 *   A block stored at full rank d, where one more component would exceed the
 *   head dimension, takes the symmetric form: a = max |x_t| / 127,
 *   c_t = round(x_t / a) in [−127, 127] (a = 0 gives 0), dim row j = a_j·B_b[:, j].
 * The new object has dtype MILO_I8, ranks r_b + 1 (r_b at full rank), row_offsets
 * the running sums of those ranks, tok of int8 codes in the slab layout above
 * (an extra row all 1 where there is one) and dim in bf16; milo_decode_attn,
 * _select and _noalloc take it as they take a bf16 object (q, suffix and out stay
 * bf16).  Token-factor bytes halve.
 *   f    bf16 factor object (MILO_ERR_UNSUPPORTED for other dtypes); not modified.
 *   out  receives the new object; destroy it with milo_factors_destroy.
 * Synchronises once on f's factors to read their ranks; allocates the new object.
 */
milo_status milo_factors_quantize(const milo_factors* f, void* stream, milo_factors** out);

/* Frees f and everything it owns (synchronises the device first). NULL is a no-op. */
void milo_factors_destroy(milo_factors* f);

const char* milo_status_string(int32_t status);
int32_t milo_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MILO_H_ */
