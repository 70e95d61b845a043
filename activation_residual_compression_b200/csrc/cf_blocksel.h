// cf_blocksel.h -- Otil-style selective block transmission (CF_BLOCKSEL).
//
// Source: the Otil page, sections "Square sub-block partition",
// "Informative sub-block selection" and "Dynamic round-robin".  The token
// grid H x W (rows = H*W in raster order) is cut into b x b blocks spanning
// all channels; each selective step sends the k blocks of largest cosine
// dissimilarity against the previous activation among the blocks not yet
// sent in the current round, raw, in ascending block order.
#pragma once

#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>

#include "cf_internal.h"

namespace cfi {

constexpr int kBsMaxBlocks = 4096;        // K limit of the single-CTA selection sort
constexpr uint32_t kBsNone = 0xffffffffu;  // index of an unused payload slot

struct BlockselPlan {
  int64_t rows = 0, cols = 0;
  int H = 0, W = 0, b = 0, k = 0, K = 0, warm = 1, dtype = 0;
  // sender scratch (zeroed at creation)
  uint8_t *sent = nullptr;   // [K] 1 = sent in the current round (part of the state)
  double *part = nullptr;    // [K][b][4] per block row: <p, a>, ||p||^2, ||a||^2, changed
  uint32_t *sel = nullptr;   // [k] this step's blocks, ascending; kBsNone = unused slot
  unsigned *counter = nullptr;  // CTAs of the current encode that have written their partials
};

// Checks the configuration and fills the plan; CF_OK or an error code.
int blocksel_plan(int64_t rows, int64_t cols, int dtype, int batch, int grid_h, int block, int k, int warm,
                  BlockselPlan *P);
size_t blocksel_body_bytes(const BlockselPlan &P);
size_t blocksel_scratch_bytes(const BlockselPlan &P);  // sender
int blocksel_bind(BlockselPlan *P, void *scratch);     // sender; CF_OK or CF_ERR_CUDA

// One step (sender).  warm: the payload is a itself.  Otherwise the
// dissimilarities, the selection and the payload.  Either way prev ([rows]
// [cols] in the activation dtype, the state) becomes a.
cudaError_t blocksel_encode(const BlockselPlan &P, const void *a, void *prev, uint8_t *payload, const Header &hdr,
                            bool warm, cudaStream_t st);
// Receiver: warm, ahat = recon = the payload; otherwise the sent blocks
// replace ahat's and recon = ahat everywhere (ahat in the activation dtype).
cudaError_t blocksel_decode(const BlockselPlan &P, const uint8_t *payload, void *ahat, void *recon,
                            const Header &expect, bool warm, int *status, cudaStream_t st);

}  // namespace cfi
