// Tensor-core (tcgen05) rank-space decode attention: host interface.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "internal.h"

namespace milo {

struct TcPlan;  // cached work list, tensor maps and scratch for one decode shape

struct TcInputs {
  const void* q;
  const void* K_suf;
  const void* V_suf;
  const void* tok;
  const void* dim;
  const int32_t* ranks;        // device [2H][nb]
  const int64_t* row_offsets;  // device [2H][nb+1]
  uint32_t* status;
  int64_t total_rows;  // rows of the factor arrays (Σ of every block's rank)
  const int32_t* host_ranks;  // [2H][nb]
  bool q8 = false;            // tok holds int8 codes (8-bit factor object), dim bf16
  // Pre-RoPE key factors: the prefix keys are rebuilt and rotated (base rope_theta) into rope_keys
  // ([H][T][d] bf16 scratch) before the decode, which then scores them densely.
  bool rope_keys = false;
  double rope_theta = 0.0;
};

// The shape check alone (no CUDA call): bf16 (or 8-bit) factors, d in {64, 128}, n % 128 == 0, GQA group <= 128.
bool tc_shape_ok(const DecodeShape& s);
bool tc_supported(const DecodeShape& s);
int tc_launches(const DecodeShape& s, bool rope_keys = false);
// ev0 / ev1 (optional) are recorded on `st` right before and right after the main decode kernel.
// mask (optional, host [H][nb], nonzero = attended): block selection; the plan is rebuilt when it changes.
cudaError_t tc_decode(TcPlan** plan, const DecodeShape& s, const TcInputs& in, void* out, cudaStream_t st,
                      cudaEvent_t ev0 = nullptr, cudaEvent_t ev1 = nullptr, const uint8_t* mask = nullptr);
void tc_plan_destroy(TcPlan* plan);

// The same decode with its scratch in a fixed device array (no allocation).  *too_large is set when
// the work list or the partials of this shape do not fit the array.
cudaError_t tc_decode_noalloc(const DecodeShape& s, const TcInputs& in, void* out, cudaStream_t st,
                              bool* too_large);
size_t tc_noalloc_scratch_bytes();
// The work list for ranks / shape on a GPU with `sms` SMs into w[cap] (host only); info as in
// milo_decode_worklist.  Returns the words used, or -1 if cap is too small.
int tc_worklist(const DecodeShape& s, const int32_t* host_ranks, int sms, int* w, int64_t cap, int64_t* info);

}  // namespace milo
