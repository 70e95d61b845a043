// cf_lowrank.cu -- low-rank mode of libcf (not yet implemented: creation of
// a CF_LOWRANK state is rejected with CF_ERR_UNSUPPORTED).
#include "cf_lowrank.h"

namespace cfi {

void lowrank_plan(int64_t rows, int64_t cols, const cf_params &p, LowrankPlan *plan) {
  plan->rows = rows;
  plan->cols = cols;
  plan->rank = p.rank;
  plan->iters = p.iters;
  plan->int4 = p.lr_int4;
  plan->batch = p.batch;
  plan->supported = false;
}

cudaError_t lowrank_encode(const LowrankPlan &, const EncArgs &, const PtrTable *, float *, void *, uint64_t,
                           cudaStream_t) {
  return cudaErrorNotSupported;
}

cudaError_t lowrank_decode(const LowrankPlan &, const DecArgs &, const PtrTable *, void *, cudaStream_t) {
  return cudaErrorNotSupported;
}

}  // namespace cfi
