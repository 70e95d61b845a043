// cf_lowrank.h -- low-rank mode (warm-started subspace iteration, INT4
// factors) of libcf.  Internal.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "cf.h"
#include "cf_internal.h"

namespace cfi {

struct LowrankBufs {
  // sender only
  __nv_bfloat16 *dhi = nullptr, *dlo = nullptr;    // residual D split in two bf16 terms, [rows][cols]
  __nv_bfloat16 *vthi = nullptr, *vtlo = nullptr;  // V^T split, [rp][cols]
  __nv_bfloat16 *qthi = nullptr, *qtlo = nullptr;  // Q^T split, [rp][rows]
  float *ypart = nullptr;                          // split-K partial products [sy][rows][rp]
  float *vpart = nullptr;                          // [sv][cols][rp]
  float *xbuf = nullptr;                           // matrix being orthonormalised [rows][rp]
  float *q = nullptr;                              // orthonormal factor [rows][rp]
  float *v = nullptr;                              // right factor [cols][rp]
  double *gpart = nullptr;                         // partial Gram matrices [nblk][rp][rp]
  double *L = nullptr;                             // Cholesky factor [rp][rp]
  int *dead = nullptr;                             // rank-deficient column flags [rp]
  int *skip2 = nullptr;                            // the sweep's first CholeskyQR pass suffices (set on the device)
  unsigned *gbar = nullptr;                        // grid-barrier counters of the two sweeps' orthonormalisation
  double *gpk = nullptr;                           // G in the Cholesky factor's packed 8 x 8 tile layout
  unsigned *amax = nullptr;                        // column absmax bit patterns of Q [rp] and V [rp]
  // both roles: reconstruction operands dequantised from the payload
  __nv_bfloat16 *uahi = nullptr, *ualo = nullptr;  // [rows][kp]
  __nv_bfloat16 *vbhi = nullptr, *vblo = nullptr;  // [cols][kp]
};

struct LowrankPlan {
  int64_t rows = 0, cols = 0;
  int rank = 0, rp = 0, kp = 0, iters = 1, int4 = 1, batch = 1;
  int role = 0, ef_explicit = 1, ef_off = 0, dtype = CF_BF16;
  double qr2_tol = 0.0;          // near-identity bound of the second CholeskyQR pass (0: full)
  uint32_t test_wait_polls = 0;  // test hook: > 0 makes the reconstruction's operand wait run out
  int sy = 1, sv = 1;            // split-K factors of the two thin GEMMs
  int nblk_gram = 1;             // row blocks of the partial Gram matrices
  int ortho_grid = 1;            // blocks of the orthonormalisation kernel (all resident at once)
  size_t enc_scratch_bytes = 0;
  size_t dec_scratch_bytes = 0;
  bool supported = false;
  LowrankBufs b;
  CUtensorMap tm_dhi, tm_dlo, tm_vthi, tm_vtlo;    // Y = D V
  CUtensorMap tm_dmhi, tm_dmlo, tm_qthi, tm_qtlo;  // V = D^T Q (D read MN-major: 64 x 64 boxes)
  CUtensorMap tm_uahi, tm_ualo, tm_vbhi, tm_vblo;  // C = U V^T
};

void lowrank_plan(int64_t rows, int64_t cols, const cf_params &p, LowrankPlan *plan);
// Carve the scratch buffers out of `scratch` and encode the TMA tensor maps.
int lowrank_bind(LowrankPlan *plan, void *scratch);
cudaError_t lowrank_encode(const LowrankPlan &plan, const EncArgs &args, const PtrTable *tab, float *vprev,
                           uint64_t step, uint64_t seed, cudaStream_t st);
cudaError_t lowrank_decode(const LowrankPlan &plan, const DecArgs &args, const PtrTable *tab, cudaStream_t st);

}  // namespace cfi
