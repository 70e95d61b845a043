// cf_internal.h -- internal types shared by the host layer and the kernels
// of libcf.  Not part of the ABI (include/cf.h is).
#pragma once

#include <cstddef>
#include <cstdint>

#include <cuda_runtime.h>

#include "cf.h"

namespace cfi {

constexpr int kHdrBytes = 64;
constexpr uint32_t kMagic = 0x31504643u;  // "CFP1"
constexpr int kMaxBatch = 1024;           // pointer-table capacity of the batched entry points
constexpr int kBlock = 256;               // threads per block of the streaming kernels
constexpr int kMaxCols = 8192;            // streaming modes keep a row in registers
constexpr int kMaxRank = 128;

// The 64-byte payload header, as 16 little-endian words.
struct Header {
  uint32_t w[16];
};

// Per-tensor payload body layout.
struct Layout {
  size_t body;  // bytes per tensor body (multiple of 16)
  size_t sec1;  // offset of the second section (codes / indices / U)
  size_t sec2;  // offset of the third section (low-rank V)
};

// Device pointers of a batch of tensors, passed by value in kernel
// parameter space (8 KiB; no device-side table, no scratch memory).
struct PtrTable {
  const void *p[kMaxBatch];
};
struct NoTable {};

// Arguments of the streaming encode kernels.
struct EncArgs {
  const void *a;          // contiguous activations (when no pointer table)
  float *ahat;            // [batch][rows][cols]
  float *err;             // [batch][rows][cols]
  uint8_t *payload;       // header + bodies
  int64_t rows, cols;
  int64_t body_bytes;     // per tensor
  int64_t sec1;           // offset of codes / indices in a body
  int batch;
  int ef_explicit;
  int ef_off;             // CF_EF_OFF: ahat <- fp32(a), e untouched
  int team_log2;          // threads per row = 1 << team_log2 (>= 32)
  int64_t padA_off, padA_len;  // alignment padding inside each body, zeroed by the encoder
  int64_t padB_off, padB_len;
  int *status;            // sticky device status word of the sender
  Header hdr;
};

// Arguments of the streaming decode kernels.
struct DecArgs {
  const uint8_t *payload;
  void *recon;            // contiguous recon (when no pointer table)
  float *ahat;            // receiver reconstruction [batch][rows][cols]
  int *status;            // sticky device status word
  int64_t rows, cols;
  int64_t body_bytes;
  int64_t sec1;
  int batch;
  int team_log2;
  Header expect;          // header this receiver expects
};

// Launch configuration of a streaming kernel family for one state.
struct StreamCfg {
  int team_log2;
  int vpt;        // 8-element vectors per thread
  int enc_grid;
  int dec_grid;
  int warm_grid;
  bool state_bf16;  // ahat and e stored as bf16 (the bf16-state option)
};

// ---- streaming kernels (cf_stream.cu) ----
int stream_config(int mode, int dtype, int nm_m, int nm_n, int64_t rows, int64_t cols, int batch,
                  int sm_count, int state_bf16, StreamCfg *cfg);
cudaError_t launch_encode(int mode, int dtype, int nm_m, int nm_n, const StreamCfg &cfg,
                          const EncArgs &args, const PtrTable *tab, cudaStream_t st);
cudaError_t launch_decode(int mode, int dtype, int nm_m, int nm_n, const StreamCfg &cfg,
                          const DecArgs &args, const PtrTable *tab, cudaStream_t st);
cudaError_t launch_warm_encode(int dtype, const StreamCfg &cfg, const EncArgs &args,
                               const PtrTable *tab, cudaStream_t st);
cudaError_t launch_warm_decode(int dtype, const StreamCfg &cfg, const DecArgs &args,
                               const PtrTable *tab, cudaStream_t st);

}  // namespace cfi
