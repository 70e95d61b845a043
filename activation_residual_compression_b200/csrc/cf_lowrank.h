// cf_lowrank.h -- low-rank mode (warm-started subspace iteration, INT4
// factors) of libcf.  Internal.
#pragma once

#include <cuda_runtime.h>

#include "cf.h"
#include "cf_internal.h"

namespace cfi {

struct LowrankPlan {
  int64_t rows = 0, cols = 0;
  int rank = 0, rpad = 0, iters = 1, int4 = 1, batch = 1;
  size_t enc_scratch_bytes = 0;
  size_t dec_scratch_bytes = 0;
  bool supported = false;
};

void lowrank_plan(int64_t rows, int64_t cols, const cf_params &p, LowrankPlan *plan);
cudaError_t lowrank_encode(const LowrankPlan &plan, const EncArgs &args, const PtrTable *tab, float *vprev,
                           void *scratch, uint64_t seed, cudaStream_t st);
cudaError_t lowrank_decode(const LowrankPlan &plan, const DecArgs &args, const PtrTable *tab, void *scratch,
                           cudaStream_t st);

}  // namespace cfi
