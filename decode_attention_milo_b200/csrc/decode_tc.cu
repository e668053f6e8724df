// Tensor-core (tcgen05) rank-space decode attention.
#include "decode_tc.h"

namespace milo {

struct TcPlan {};

bool tc_supported(const DecodeShape&) { return false; }

int tc_launches(const DecodeShape&) { return 2; }

cudaError_t tc_decode(TcPlan**, const DecodeShape&, const TcInputs&, void*, cudaStream_t) {
  return cudaErrorNotSupported;
}

void tc_plan_destroy(TcPlan* plan) { delete plan; }

}  // namespace milo
