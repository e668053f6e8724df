// C ABI of the library (declared in include/milo.h): argument checks, the
// factor object, scratch management and launch sequencing.
#include <math.h>
#include <stdio.h>
#include <string.h>

#include <mutex>
#include <new>
#include <vector>

#include "../../include/milo.h"
#include "common.cuh"
#include "decode_tc.h"
#include "internal.h"
#include "quant.h"

struct milo_factors {
  int device = 0;
  int H = 0;
  int64_t T = 0;
  int d = 0, n = 0, nb = 0, r_min = 0, R = 0, pool_rows = 0;
  int64_t total_rows = 0;       // rows of the factor arrays: Σ of every block's rank
  int rule = 0, scope = 0;      // allocation rule and budget scope (milo_alloc_rule, milo_pool_scope)
  int dtype = 0;
  uint32_t flags = 0;
  int32_t* ranks = nullptr;
  int64_t* row_offsets = nullptr;
  void* tok = nullptr;
  void* dim = nullptr;
  uint32_t* status = nullptr;
  float* eigvals = nullptr;
  int32_t* sweeps = nullptr;
  float* eigvecs = nullptr;
  double* entropy = nullptr;
  double* quotas = nullptr;
  cudaEvent_t ready = nullptr;  // recorded after the factors are written
  // decode scratch, owned here and reused by later calls
  std::mutex mu;
  // host copy of the ranks for the work-list builder: sized when the object is made, filled (one
  // synchronisation) by the first decode call, so that no later call allocates or waits for it
  std::vector<int32_t> host_ranks;
  bool host_ranks_valid = false;
  float* partials = nullptr;
  size_t partials_floats = 0;
  milo::TcPlan* tc_plan = nullptr;
};

namespace {

size_t esize(int dtype) { return dtype == MILO_BF16 ? 2 : 4; }
// element sizes of the two factor arrays (an 8-bit object has int8 tok and bf16 dim)
size_t tok_esize(int dtype) { return dtype == MILO_I8 ? 1 : esize(dtype); }
size_t dim_esize(int dtype) { return dtype == MILO_I8 ? 2 : esize(dtype); }
// the decode reads q, the suffix and out in bf16 for bf16 and 8-bit objects
bool bf16_io(int dtype) { return dtype == MILO_BF16 || dtype == MILO_I8; }

milo_status cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return MILO_OK;
  if (e == cudaErrorMemoryAllocation) return MILO_ERR_OUT_OF_MEMORY;
  return MILO_ERR_CUDA;
}

#define MILO_CUDA(call)                                  \
  do {                                                   \
    cudaError_t e_ = (call);                             \
    if (e_ != cudaSuccess) return cuda_status(e_);       \
  } while (0)

void free_all(milo_factors* f) {
  if (!f) return;
  cudaFree(f->ranks);
  cudaFree(f->row_offsets);
  cudaFree(f->tok);
  cudaFree(f->dim);
  cudaFree(f->status);
  cudaFree(f->eigvals);
  cudaFree(f->sweeps);
  if (f->eigvecs) cudaFreeAsync(f->eigvecs, 0);
  cudaFree(f->entropy);
  cudaFree(f->quotas);
  cudaFree(f->partials);
  if (f->ready) cudaEventDestroy(f->ready);
  milo::tc_plan_destroy(f->tc_plan);
}

// Blocks per pool that milo_compress takes: its allocation step holds 28 bytes per block of a pool in
// shared memory (224 KB at this limit, within the 227 KB a CTA may use).
constexpr int kMaxAllocBlocks = 8192;

bool valid_dtype(int32_t dt) { return dt == MILO_F32 || dt == MILO_BF16 || dt == MILO_I8; }

milo_status check_layer_shape(int32_t dtype, int32_t H, int64_t T, int32_t d, int32_t n, int32_t r_min) {
  if (!valid_dtype(dtype) || H <= 0 || T <= 0 || n <= 0 || r_min < 1) return MILO_ERR_INVALID_ARGUMENT;
  if (d != 64 && d != 128) return d > 0 ? MILO_ERR_UNSUPPORTED : MILO_ERR_INVALID_ARGUMENT;
  if (T % n != 0 || n < d || n % 128 != 0 || r_min > d) return MILO_ERR_INVALID_ARGUMENT;
  if (T / n > (1 << 20) || H > 1024) return MILO_ERR_INVALID_ARGUMENT;
  return MILO_OK;
}

}  // namespace

extern "C" {

int32_t milo_abi_version(void) { return MILO_ABI_VERSION; }

const char* milo_status_string(int32_t s) {
  switch (s) {
    case MILO_OK: return "ok";
    case MILO_ERR_INVALID_ARGUMENT: return "invalid argument";
    case MILO_ERR_UNSUPPORTED: return "unsupported configuration";
    case MILO_ERR_BUDGET: return "budget below num_blocks * r_min";
    case MILO_ERR_NO_CONVERGENCE: return "eigensolver did not converge";
    case MILO_ERR_DEVICE_CHECK: return "device-side check failed";
    case MILO_ERR_CUDA: return "CUDA error";
    case MILO_ERR_OUT_OF_MEMORY: return "out of device memory";
    default: return "unknown status";
  }
}

static milo_status compress_impl(const void* K, const void* V, int32_t dtype, int32_t num_kv_heads,
                                 int64_t context, int32_t head_dim, int32_t block_size, double budget,
                                 int32_t r_min, int32_t max_sweeps, uint32_t flags, int32_t rule, int32_t scope,
                                 const double* host_weights, void* stream, milo_factors** out,
                                 const cudaEvent_t* ev) {
  if (!out) return MILO_ERR_INVALID_ARGUMENT;
  *out = nullptr;
  if (!K || !V) return MILO_ERR_INVALID_ARGUMENT;
  if (dtype == MILO_I8) return MILO_ERR_INVALID_ARGUMENT;  // the cache itself is f32 or bf16
  milo_status st = check_layer_shape(dtype, num_kv_heads, context, head_dim, block_size, r_min);
  if (st != MILO_OK) return st;
  if (!(budget > 0.0) || !isfinite(budget) || max_sweeps < 0 || (flags & ~MILO_KEEP_INTERMEDIATES))
    return MILO_ERR_INVALID_ARGUMENT;
  if (rule < MILO_ALLOC_ENTROPY || rule > MILO_ALLOC_WEIGHTS || (scope != MILO_POOL_HEAD && scope != MILO_POOL_LAYER))
    return MILO_ERR_INVALID_ARGUMENT;
  if ((rule == MILO_ALLOC_WEIGHTS) != (host_weights != nullptr)) return MILO_ERR_INVALID_ARGUMENT;
  const int nb = (int)(context / block_size);
  const int P = 2 * num_kv_heads;
  // the allocation kernel keeps 20 bytes per block of its group (a pool, or the layer) in shared memory
  if ((scope == MILO_POOL_LAYER ? (int64_t)P * nb : nb) > kMaxAllocBlocks) return MILO_ERR_UNSUPPORTED;
  if (host_weights)
    for (int64_t i = 0; i < (int64_t)P * nb; ++i)
      if (!(host_weights[i] > 0.0) || !isfinite(host_weights[i])) return MILO_ERR_INVALID_ARGUMENT;
  const double Rd = floor(budget * (double)(context * head_dim) / (double)(block_size + head_dim));
  if (Rd < (double)nb * r_min) return MILO_ERR_BUDGET;
  const int64_t full = (int64_t)nb * head_dim;
  const int R = Rd >= (double)full ? (int)full : (int)Rd;

  milo_factors* f = new (std::nothrow) milo_factors();
  if (!f) return MILO_ERR_OUT_OF_MEMORY;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  f->H = num_kv_heads;
  f->T = context;
  f->d = head_dim;
  f->n = block_size;
  f->nb = nb;
  f->r_min = r_min;
  f->R = R;
  f->pool_rows = scope == MILO_POOL_HEAD ? R : 0;
  // with one budget over the layer the pools' rank sums differ, but they still total P·R (R is capped at nb·d)
  f->total_rows = (int64_t)P * R;
  f->rule = rule;
  f->scope = scope;
  f->dtype = dtype;
  f->flags = flags;
  f->host_ranks.assign((size_t)P * nb, 0);
  const size_t rows = (size_t)f->total_rows;
  const size_t nblk = (size_t)P * nb;
  const size_t dd = (size_t)head_dim * head_dim;
  float* gram = nullptr;
  cudaError_t e = cudaGetDevice(&f->device);
  auto fail = [&](cudaError_t err) {
    if (gram) cudaFreeAsync(gram, s);
    cudaStreamSynchronize(s);
    free_all(f);
    delete f;
    return cuda_status(err);
  };
  if (e != cudaSuccess) return fail(e);
  // stream-ordered allocations: no device-wide synchronisation per array (the object's users order after
  // its ready event; milo_factors_destroy synchronises before freeing)
#define ALLOC(ptr, bytes)                                   \
  do {                                                      \
    e = cudaMallocAsync((void**)&(ptr), (bytes), s);        \
    if (e != cudaSuccess) return fail(e);                   \
  } while (0)
  ALLOC(f->ranks, nblk * sizeof(int32_t));
  ALLOC(f->row_offsets, (size_t)P * (nb + 1) * sizeof(int64_t));
  ALLOC(f->tok, rows * block_size * esize(dtype) + 256);
  ALLOC(f->dim, rows * head_dim * esize(dtype) + 256);
  ALLOC(f->status, sizeof(uint32_t));
  ALLOC(f->eigvals, nblk * head_dim * sizeof(float));
  ALLOC(f->sweeps, nblk * sizeof(int32_t));
  if ((e = cudaMallocAsync((void**)&f->eigvecs, nblk * dd * sizeof(float), s)) != cudaSuccess) return fail(e);
  ALLOC(f->entropy, nblk * sizeof(double));
  ALLOC(f->quotas, nblk * sizeof(double));
  if ((e = cudaMallocAsync((void**)&gram, nblk * dd * sizeof(float), s)) != cudaSuccess) return fail(e);
  double* d_weights = nullptr;
  if (host_weights) {
    if ((e = cudaMallocAsync((void**)&d_weights, nblk * sizeof(double), s)) != cudaSuccess) return fail(e);
    // pageable source: the copy is staged before the call returns, so the caller may reuse host_weights
    if ((e = cudaMemcpyAsync(d_weights, host_weights, nblk * sizeof(double), cudaMemcpyHostToDevice, s)) !=
        cudaSuccess) {
      cudaFreeAsync(d_weights, s);
      return fail(e);
    }
  }
#undef ALLOC
  if ((e = cudaMemsetAsync(f->status, 0, sizeof(uint32_t), s)) != cudaSuccess) return fail(e);
  if ((e = cudaMemsetAsync(f->tok, 0, rows * block_size * esize(dtype) + 256, s)) != cudaSuccess) return fail(e);
  if ((e = cudaMemsetAsync(f->dim, 0, rows * head_dim * esize(dtype) + 256, s)) != cudaSuccess) return fail(e);

  milo::CompressShape cs{num_kv_heads, context, head_dim, block_size, nb,
                         scope == MILO_POOL_LAYER ? P * R : R, R, r_min, max_sweeps ? max_sweeps : 30,
                         dtype == MILO_BF16, rule, scope == MILO_POOL_LAYER};
  milo::CompressBuffers cb{K, V, gram, f->eigvals, f->sweeps, f->eigvecs, f->entropy, f->quotas, d_weights,
                           f->ranks, f->row_offsets, f->tok, f->dim, f->status};
  if ((e = milo::launch_compress(cs, cb, s, ev)) != cudaSuccess) {
    if (d_weights) cudaFreeAsync(d_weights, s);
    return fail(e);
  }
  if (d_weights) cudaFreeAsync(d_weights, s);
  if ((e = cudaEventCreateWithFlags(&f->ready, cudaEventDisableTiming)) != cudaSuccess) return fail(e);
  if ((e = cudaEventRecord(f->ready, s)) != cudaSuccess) return fail(e);
  // The Gram scratch (and, unless kept, the eigenpairs) are released once the stream has used them.
  cudaFreeAsync(gram, s);
  gram = nullptr;
  if (!(flags & MILO_KEEP_INTERMEDIATES)) {
    cudaFreeAsync(f->eigvecs, s);
    f->eigvecs = nullptr;
  }
  *out = f;
  return MILO_OK;
}

milo_status milo_compress(const void* K, const void* V, int32_t dtype, int32_t num_kv_heads, int64_t context,
                          int32_t head_dim, int32_t block_size, double budget, int32_t r_min,
                          int32_t max_sweeps, uint32_t flags, void* stream, milo_factors** out) {
  return compress_impl(K, V, dtype, num_kv_heads, context, head_dim, block_size, budget, r_min, max_sweeps, flags,
                       MILO_ALLOC_ENTROPY, MILO_POOL_HEAD, nullptr, stream, out, nullptr);
}

milo_status milo_compress_rule(const void* K, const void* V, int32_t dtype, int32_t num_kv_heads, int64_t context,
                               int32_t head_dim, int32_t block_size, double budget, int32_t r_min,
                               int32_t max_sweeps, uint32_t flags, int32_t rule, int32_t scope,
                               const double* host_weights, void* stream, milo_factors** out) {
  return compress_impl(K, V, dtype, num_kv_heads, context, head_dim, block_size, budget, r_min, max_sweeps, flags,
                       rule, scope, host_weights, stream, out, nullptr);
}

milo_status milo_compress_profiled(const void* K, const void* V, int32_t dtype, int32_t num_kv_heads,
                                   int64_t context, int32_t head_dim, int32_t block_size, double budget,
                                   int32_t r_min, int32_t max_sweeps, uint32_t flags, void* stream,
                                   milo_factors** out, void* const* events) {
  cudaEvent_t ev[5] = {};
  if (events)
    for (int k = 0; k < 5; ++k) ev[k] = static_cast<cudaEvent_t>(events[k]);
  return compress_impl(K, V, dtype, num_kv_heads, context, head_dim, block_size, budget, r_min, max_sweeps, flags,
                       MILO_ALLOC_ENTROPY, MILO_POOL_HEAD, nullptr, stream, out, ev);
}

milo_status milo_factors_import(int32_t dtype, int32_t num_kv_heads, int64_t context, int32_t head_dim,
                                int32_t block_size, int32_t r_min, const int32_t* host_ranks,
                                const void* host_tok, const void* host_dim, void* stream, milo_factors** out) {
  if (!out) return MILO_ERR_INVALID_ARGUMENT;
  *out = nullptr;
  if (!host_ranks || !host_tok || !host_dim) return MILO_ERR_INVALID_ARGUMENT;
  milo_status st = check_layer_shape(dtype, num_kv_heads, context, head_dim, block_size, r_min);
  if (st != MILO_OK) return st;
  const int nb = (int)(context / block_size);
  const int P = 2 * num_kv_heads;
  int64_t total = 0;
  int pool_rows = -1;  // the common rank sum of the pools, or 0 when they differ
  for (int p = 0; p < P; ++p) {
    int64_t sum = 0;
    for (int b = 0; b < nb; ++b) {
      const int r = host_ranks[(size_t)p * nb + b];
      if (r < 1 || r > head_dim) return MILO_ERR_INVALID_ARGUMENT;
      sum += r;
    }
    total += sum;
    if (pool_rows < 0) pool_rows = (int)sum;
    else if (sum != pool_rows) pool_rows = 0;
  }
  milo_factors* f = new (std::nothrow) milo_factors();
  if (!f) return MILO_ERR_OUT_OF_MEMORY;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  f->H = num_kv_heads;
  f->T = context;
  f->d = head_dim;
  f->n = block_size;
  f->nb = nb;
  f->r_min = r_min;
  f->R = pool_rows;
  f->pool_rows = pool_rows;
  f->total_rows = total;
  f->scope = pool_rows ? MILO_POOL_HEAD : MILO_POOL_LAYER;
  f->dtype = dtype;
  const size_t rows = (size_t)total;
  std::vector<int64_t> offs((size_t)P * (nb + 1));
  int64_t o = 0;
  for (int p = 0; p < P; ++p) {
    for (int b = 0; b < nb; ++b) {
      offs[(size_t)p * (nb + 1) + b] = o;
      o += host_ranks[(size_t)p * nb + b];
    }
    offs[(size_t)p * (nb + 1) + nb] = o;
  }
  cudaError_t e = cudaGetDevice(&f->device);
  auto fail = [&](cudaError_t err) {
    free_all(f);
    delete f;
    return cuda_status(err);
  };
  if (e != cudaSuccess) return fail(e);
  const size_t tb = rows * block_size * tok_esize(dtype), db = rows * head_dim * dim_esize(dtype);
  if ((e = cudaMalloc((void**)&f->ranks, (size_t)P * nb * sizeof(int32_t))) != cudaSuccess) return fail(e);
  if ((e = cudaMalloc((void**)&f->row_offsets, offs.size() * sizeof(int64_t))) != cudaSuccess) return fail(e);
  if ((e = cudaMalloc(&f->tok, tb + 256)) != cudaSuccess) return fail(e);
  if ((e = cudaMalloc(&f->dim, db + 256)) != cudaSuccess) return fail(e);
  if ((e = cudaMalloc((void**)&f->status, sizeof(uint32_t))) != cudaSuccess) return fail(e);
  if ((e = cudaMemsetAsync(f->status, 0, sizeof(uint32_t), s)) != cudaSuccess) return fail(e);
  if ((e = cudaMemsetAsync(f->tok, 0, tb + 256, s)) != cudaSuccess) return fail(e);
  if ((e = cudaMemsetAsync(f->dim, 0, db + 256, s)) != cudaSuccess) return fail(e);
  if ((e = cudaMemcpyAsync(f->ranks, host_ranks, (size_t)P * nb * sizeof(int32_t), cudaMemcpyHostToDevice, s)) !=
      cudaSuccess)
    return fail(e);
  if ((e = cudaMemcpyAsync(f->row_offsets, offs.data(), offs.size() * sizeof(int64_t), cudaMemcpyHostToDevice,
                           s)) != cudaSuccess)
    return fail(e);
  if ((e = cudaMemcpyAsync(f->tok, host_tok, tb, cudaMemcpyHostToDevice, s)) != cudaSuccess) return fail(e);
  if ((e = cudaMemcpyAsync(f->dim, host_dim, db, cudaMemcpyHostToDevice, s)) != cudaSuccess) return fail(e);
  if ((e = cudaEventCreateWithFlags(&f->ready, cudaEventDisableTiming)) != cudaSuccess) return fail(e);
  if ((e = cudaEventRecord(f->ready, s)) != cudaSuccess) return fail(e);
  if ((e = cudaStreamSynchronize(s)) != cudaSuccess) return fail(e);
  f->host_ranks.assign(host_ranks, host_ranks + (size_t)P * nb);
  f->host_ranks_valid = true;
  *out = f;
  return MILO_OK;
}

milo_status milo_factors_quantize(const milo_factors* fc, void* stream, milo_factors** out) {
  if (!out) return MILO_ERR_INVALID_ARGUMENT;
  *out = nullptr;
  if (!fc) return MILO_ERR_INVALID_ARGUMENT;
  if (fc->dtype != MILO_BF16) return MILO_ERR_UNSUPPORTED;
  milo_factors* src = const_cast<milo_factors*>(fc);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int P = 2 * src->H, nb = src->nb;
  {
    std::lock_guard<std::mutex> lock(src->mu);
    if (!src->host_ranks_valid) {
      MILO_CUDA(cudaEventSynchronize(src->ready));
      MILO_CUDA(cudaMemcpy(src->host_ranks.data(), src->ranks, src->host_ranks.size() * sizeof(int32_t),
                           cudaMemcpyDeviceToHost));
      src->host_ranks_valid = true;
    }
  }
  // ranks of the 8-bit object: one more component per block below full rank (the asymmetric form)
  std::vector<int32_t> qr(src->host_ranks.size());
  std::vector<int64_t> qoff((size_t)P * (nb + 1));
  int64_t total = 0;
  for (int p = 0; p < P; ++p) {
    for (int b = 0; b < nb; ++b) {
      const int32_t r = src->host_ranks[(size_t)p * nb + b];
      qr[(size_t)p * nb + b] = r < src->d ? r + 1 : r;
      qoff[(size_t)p * (nb + 1) + b] = total;
      total += qr[(size_t)p * nb + b];
    }
    qoff[(size_t)p * (nb + 1) + nb] = total;
  }
  milo_factors* f = new (std::nothrow) milo_factors();
  if (!f) return MILO_ERR_OUT_OF_MEMORY;
  f->H = src->H;
  f->T = src->T;
  f->d = src->d;
  f->n = src->n;
  f->nb = nb;
  f->r_min = src->r_min;
  f->total_rows = total;
  // pools keep a common row count only if they stay equal after the extra components
  int64_t pool0 = qoff[nb];
  bool same = true;
  for (int p = 1; p < P; ++p) same = same && qoff[(size_t)p * (nb + 1) + nb] - qoff[(size_t)p * (nb + 1)] == pool0;
  f->pool_rows = same ? (int)pool0 : 0;
  f->R = f->pool_rows;
  f->rule = src->rule;
  f->scope = src->scope;
  f->dtype = MILO_I8;
  f->host_ranks = qr;
  f->host_ranks_valid = true;
  auto fail = [&](cudaError_t err) {
    free_all(f);
    delete f;
    return cuda_status(err);
  };
  cudaError_t e = cudaGetDevice(&f->device);
  if (e != cudaSuccess) return fail(e);
  const size_t rows = (size_t)f->total_rows;
  const size_t tb = rows * f->n, db = rows * f->d * 2;
  if ((e = cudaMalloc((void**)&f->ranks, (size_t)P * nb * sizeof(int32_t))) != cudaSuccess) return fail(e);
  if ((e = cudaMalloc((void**)&f->row_offsets, (size_t)P * (nb + 1) * sizeof(int64_t))) != cudaSuccess) return fail(e);
  if ((e = cudaMalloc(&f->tok, tb + 256)) != cudaSuccess) return fail(e);
  if ((e = cudaMalloc(&f->dim, db + 256)) != cudaSuccess) return fail(e);
  if ((e = cudaMalloc((void**)&f->status, sizeof(uint32_t))) != cudaSuccess) return fail(e);
  if ((e = cudaMemsetAsync(f->status, 0, sizeof(uint32_t), s)) != cudaSuccess) return fail(e);
  if ((e = cudaMemsetAsync(f->tok, 0, tb + 256, s)) != cudaSuccess) return fail(e);
  if ((e = cudaMemsetAsync(f->dim, 0, db + 256, s)) != cudaSuccess) return fail(e);
  if ((e = cudaMemcpy(f->ranks, qr.data(), qr.size() * sizeof(int32_t), cudaMemcpyHostToDevice)) != cudaSuccess)
    return fail(e);
  if ((e = cudaMemcpy(f->row_offsets, qoff.data(), qoff.size() * sizeof(int64_t), cudaMemcpyHostToDevice)) !=
      cudaSuccess)
    return fail(e);
  if ((e = cudaStreamWaitEvent(s, src->ready, 0)) != cudaSuccess) return fail(e);
  milo::QuantShape qs{P, nb, f->n, f->d};
  milo::QuantBuffers qb{src->tok, src->dim, src->ranks, src->row_offsets, f->tok, f->dim, f->ranks, f->row_offsets,
                        f->status};
  if ((e = milo::launch_quantize(qs, qb, s)) != cudaSuccess) return fail(e);
  if ((e = cudaEventCreateWithFlags(&f->ready, cudaEventDisableTiming)) != cudaSuccess) return fail(e);
  if ((e = cudaEventRecord(f->ready, s)) != cudaSuccess) return fail(e);
  *out = f;
  return MILO_OK;
}

milo_status milo_factors_ranks(const milo_factors* f, int32_t* host_ranks) {
  if (!f || !host_ranks) return MILO_ERR_INVALID_ARGUMENT;
  MILO_CUDA(cudaEventSynchronize(f->ready));
  MILO_CUDA(cudaMemcpy(host_ranks, f->ranks, (size_t)2 * f->H * f->nb * sizeof(int32_t), cudaMemcpyDeviceToHost));
  return MILO_OK;
}

milo_status milo_factors_describe(const milo_factors* f, milo_factors_desc* d) {
  if (!f || !d) return MILO_ERR_INVALID_ARGUMENT;
  memset(d, 0, sizeof(*d));
  d->num_kv_heads = f->H;
  d->num_blocks = f->nb;
  d->block_size = f->n;
  d->head_dim = f->d;
  d->context = f->T;
  d->r_min = f->r_min;
  d->pool_rows = f->pool_rows;
  d->dtype = f->dtype;
  d->alloc_rule = f->rule;
  d->pool_scope = f->scope;
  d->total_rows = f->total_rows;
  d->ranks = f->ranks;
  d->row_offsets = f->row_offsets;
  d->tok = f->tok;
  d->dim = f->dim;
  const bool keep = f->flags & MILO_KEEP_INTERMEDIATES;
  d->eigvals = keep ? f->eigvals : nullptr;
  d->sweeps = f->sweeps;
  d->eigvecs = keep ? f->eigvecs : nullptr;
  d->entropy = keep ? f->entropy : nullptr;
  d->quotas = keep ? f->quotas : nullptr;
  return MILO_OK;
}

milo_status milo_factors_status(const milo_factors* f, uint32_t* host_bits) {
  if (!f) return MILO_ERR_INVALID_ARGUMENT;
  MILO_CUDA(cudaDeviceSynchronize());
  uint32_t bits = 0;
  MILO_CUDA(cudaMemcpy(&bits, f->status, sizeof(bits), cudaMemcpyDeviceToHost));
  if (host_bits) *host_bits = bits;
  if (bits & milo::kStatusNoConvergence) return MILO_ERR_NO_CONVERGENCE;
  if (bits) return MILO_ERR_DEVICE_CHECK;
  return MILO_OK;
}

void milo_factors_destroy(milo_factors* f) {
  if (!f) return;
  cudaDeviceSynchronize();
  free_all(f);
  delete f;
}

milo_status milo_decode_worklist(const int32_t* host_ranks, int32_t num_kv_heads, int32_t num_blocks,
                                 int32_t block_size, int32_t head_dim, int32_t batch, int32_t num_q_heads,
                                 int32_t suffix_len, int32_t num_ctas, int32_t* out, int64_t capacity,
                                 int64_t* info) {
  if (!host_ranks || !out || !info || num_kv_heads <= 0 || num_blocks <= 0 || block_size <= 0 || head_dim <= 0 ||
      batch <= 0 || num_q_heads <= 0 || suffix_len < 0 || num_ctas <= 0 || capacity <= 0 ||
      num_q_heads % num_kv_heads != 0)
    return MILO_ERR_INVALID_ARGUMENT;
  for (int64_t i = 0; i < 2LL * num_kv_heads * num_blocks; ++i)
    if (host_ranks[i] < 1 || host_ranks[i] > head_dim) return MILO_ERR_INVALID_ARGUMENT;
  milo::DecodeShape ds{num_kv_heads, num_blocks, block_size, head_dim, batch, num_q_heads, suffix_len, true, 1.f};
  if (!milo::tc_shape_ok(ds)) return MILO_ERR_UNSUPPORTED;
  if (milo::tc_worklist(ds, host_ranks, num_ctas, out, capacity, info) < 0) return MILO_ERR_UNSUPPORTED;
  return MILO_OK;
}

int32_t milo_decode_launches(const milo_factors* f, int32_t batch, int32_t num_q_heads, int32_t suffix_len) {
  if (!f || batch <= 0 || num_q_heads <= 0 || suffix_len < 0 || num_q_heads % f->H != 0)
    return -(int32_t)MILO_ERR_INVALID_ARGUMENT;
  milo::DecodeShape ds{f->H, f->nb, f->n, f->d, batch, num_q_heads, suffix_len, bf16_io(f->dtype), 1.f};
  if (bf16_io(f->dtype) && milo::tc_supported(ds)) return milo::tc_launches(ds);
  if (f->dtype == MILO_I8) return -(int32_t)MILO_ERR_UNSUPPORTED;
  return suffix_len > 0 ? 3 : 2;
}

static milo_status decode_impl(const void* q, int32_t batch, int32_t num_q_heads, const milo_factors* fc,
                               const void* K_suffix, const void* V_suffix, int32_t suffix_len, float scale,
                               void* out, void* stream, cudaEvent_t ev0, cudaEvent_t ev1,
                               const uint8_t* mask = nullptr, double rope_theta = 0.0) {
  if (!fc || !q || !out || batch <= 0 || num_q_heads <= 0 || suffix_len < 0) return MILO_ERR_INVALID_ARGUMENT;
  milo_factors* f = const_cast<milo_factors*>(fc);
  if (num_q_heads % f->H != 0) return MILO_ERR_INVALID_ARGUMENT;
  if (suffix_len > 0 && (!K_suffix || !V_suffix)) return MILO_ERR_INVALID_ARGUMENT;
  if (!(scale == scale) || isinf(scale)) return MILO_ERR_INVALID_ARGUMENT;
  if (batch > 65535 || num_q_heads > 4096 || suffix_len > (1 << 20)) return MILO_ERR_INVALID_ARGUMENT;
  if (rope_theta != 0.0 && !(rope_theta > 1.0 && isfinite(rope_theta))) return MILO_ERR_INVALID_ARGUMENT;
  if (rope_theta != 0.0 && f->dtype != MILO_BF16) return MILO_ERR_UNSUPPORTED;  // bf16 key factors only
  if (mask && suffix_len == 0) {  // a head with no selected block and no suffix has nothing to attend
    for (int h = 0; h < f->H; ++h) {
      bool any = false;
      for (int b = 0; b < f->nb && !any; ++b) any = mask[(size_t)h * f->nb + b] != 0;
      if (!any) return MILO_ERR_INVALID_ARGUMENT;
    }
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const float sc = scale > 0.f ? scale : 1.0f / sqrtf((float)f->d);
  std::lock_guard<std::mutex> lock(f->mu);
  // Order after the factors were written.  Inside a stream capture the factors must already be complete
  // (an event recorded outside the capture cannot be waited on there), so the wait is skipped.
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  MILO_CUDA(cudaStreamIsCapturing(s, &cap));
  if (cap == cudaStreamCaptureStatusNone) MILO_CUDA(cudaStreamWaitEvent(s, f->ready, 0));
  milo::DecodeShape ds{f->H, f->nb, f->n, f->d, batch, num_q_heads, suffix_len, bf16_io(f->dtype), sc};
  milo::DecodeBuffers db{q, K_suffix, V_suffix, f->ranks, f->row_offsets, f->tok, f->dim, nullptr, out, f->status};
  if (bf16_io(f->dtype) && milo::tc_supported(ds)) {
    if (!f->host_ranks_valid) {
      MILO_CUDA(cudaStreamSynchronize(s));
      MILO_CUDA(cudaMemcpy(f->host_ranks.data(), f->ranks, f->host_ranks.size() * sizeof(int32_t),
                           cudaMemcpyDeviceToHost));
      f->host_ranks_valid = true;
    }
    milo::TcInputs in{q,        K_suffix,       V_suffix,  f->tok,        f->dim,
                      f->ranks, f->row_offsets, f->status, f->total_rows, f->host_ranks.data(),
                      f->dtype == MILO_I8, rope_theta > 0.0, rope_theta};
    return cuda_status(milo::tc_decode(&f->tc_plan, ds, in, out, s, ev0, ev1, mask));
  }
  // block selection, 8-bit factors and pre-RoPE keys run on the tensor-core decode only
  if (mask || f->dtype == MILO_I8 || rope_theta > 0.0) return MILO_ERR_UNSUPPORTED;
  const size_t need = milo::simt_decode_partials_floats(ds);
  if (need > f->partials_floats) {
    MILO_CUDA(cudaStreamSynchronize(s));
    cudaFree(f->partials);
    f->partials = nullptr;
    f->partials_floats = 0;
    MILO_CUDA(cudaMalloc((void**)&f->partials, need * sizeof(float)));
    f->partials_floats = need;
  }
  db.partials = f->partials;
  return cuda_status(milo::launch_decode_simt(ds, db, s, ev0, ev1));
}

milo_status milo_decode_attn(const void* q, int32_t batch, int32_t num_q_heads, const milo_factors* f,
                             const void* K_suffix, const void* V_suffix, int32_t suffix_len, float scale,
                             void* out, void* stream) {
  return decode_impl(q, batch, num_q_heads, f, K_suffix, V_suffix, suffix_len, scale, out, stream, nullptr,
                     nullptr);
}

milo_status milo_decode_attn_noalloc(const void* q, int32_t batch, int32_t num_q_heads, const milo_factors* fc,
                                     const void* K_suffix, const void* V_suffix, int32_t suffix_len, float scale,
                                     void* out, void* stream) {
  if (!fc || !q || !out || batch <= 0 || num_q_heads <= 0 || suffix_len < 0) return MILO_ERR_INVALID_ARGUMENT;
  milo_factors* f = const_cast<milo_factors*>(fc);
  if (num_q_heads % f->H != 0) return MILO_ERR_INVALID_ARGUMENT;
  if (suffix_len > 0 && (!K_suffix || !V_suffix)) return MILO_ERR_INVALID_ARGUMENT;
  if (!(scale == scale) || isinf(scale)) return MILO_ERR_INVALID_ARGUMENT;
  if (batch > 65535 || num_q_heads > 4096 || suffix_len > (1 << 20)) return MILO_ERR_INVALID_ARGUMENT;
  const float sc = scale > 0.f ? scale : 1.0f / sqrtf((float)f->d);
  milo::DecodeShape ds{f->H, f->nb, f->n, f->d, batch, num_q_heads, suffix_len, bf16_io(f->dtype), sc};
  if (!bf16_io(f->dtype) || !milo::tc_supported(ds)) return MILO_ERR_UNSUPPORTED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  std::lock_guard<std::mutex> lock(f->mu);
  if (!f->host_ranks_valid) {
    // the host copy was sized when the factor object was made: filling it allocates nothing
    MILO_CUDA(cudaEventSynchronize(f->ready));
    MILO_CUDA(cudaMemcpy(f->host_ranks.data(), f->ranks, f->host_ranks.size() * sizeof(int32_t),
                         cudaMemcpyDeviceToHost));
    f->host_ranks_valid = true;
  }
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  MILO_CUDA(cudaStreamIsCapturing(s, &cap));
  if (cap == cudaStreamCaptureStatusNone) MILO_CUDA(cudaStreamWaitEvent(s, f->ready, 0));
  milo::TcInputs in{q,        K_suffix,       V_suffix,  f->tok,        f->dim,
                    f->ranks, f->row_offsets, f->status, f->total_rows, f->host_ranks.data(),
                    f->dtype == MILO_I8};
  bool too_large = false;
  const cudaError_t e = milo::tc_decode_noalloc(ds, in, out, s, &too_large);
  if (too_large) return MILO_ERR_UNSUPPORTED;
  return cuda_status(e);
}

milo_status milo_decode_attn_select(const void* q, int32_t batch, int32_t num_q_heads, const milo_factors* f,
                                    const void* K_suffix, const void* V_suffix, int32_t suffix_len, float scale,
                                    const uint8_t* host_block_mask, void* out, void* stream) {
  if (!host_block_mask) return MILO_ERR_INVALID_ARGUMENT;
  return decode_impl(q, batch, num_q_heads, f, K_suffix, V_suffix, suffix_len, scale, out, stream, nullptr,
                     nullptr, host_block_mask);
}

milo_status milo_decode_attn_rope(const void* q, int32_t batch, int32_t num_q_heads, const milo_factors* f,
                                  const void* K_suffix, const void* V_suffix, int32_t suffix_len, float scale,
                                  double rope_theta, const uint8_t* host_block_mask, void* out, void* stream) {
  if (!(rope_theta > 1.0)) return MILO_ERR_INVALID_ARGUMENT;
  return decode_impl(q, batch, num_q_heads, f, K_suffix, V_suffix, suffix_len, scale, out, stream, nullptr,
                     nullptr, host_block_mask, rope_theta);
}

milo_status milo_decode_attn_profiled(const void* q, int32_t batch, int32_t num_q_heads, const milo_factors* f,
                                      const void* K_suffix, const void* V_suffix, int32_t suffix_len, float scale,
                                      void* out, void* stream, void* event_before, void* event_after) {
  return decode_impl(q, batch, num_q_heads, f, K_suffix, V_suffix, suffix_len, scale, out, stream,
                     static_cast<cudaEvent_t>(event_before), static_cast<cudaEvent_t>(event_after));
}

}  // extern "C"
