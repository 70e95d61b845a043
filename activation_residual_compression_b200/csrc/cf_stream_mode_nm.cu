// cf_stream_mode_nm.cu -- instantiations of the streaming kernels for the
// N:M block sparsifier mode (one translation unit per mode so they compile in parallel).
#include "cf_stream_kernels.cuh"

namespace cfi {

const void *stream_kernel_nm(bool enc, int dtype, int nm_m, int nm_n, int vpt, bool table, bool state_bf16) {
  if (nm_m == 16 && nm_n == 1) return pick_any<M_NM, 16, 1>(enc, dtype, vpt, table, state_bf16);
  if (nm_m == 16 && nm_n == 2) return pick_any<M_NM, 16, 2>(enc, dtype, vpt, table, state_bf16);
  if (nm_m == 4 && nm_n == 1) return pick_any<M_NM, 4, 1>(enc, dtype, vpt, table, state_bf16);
  if (nm_m == 4 && nm_n == 2) return pick_any<M_NM, 4, 2>(enc, dtype, vpt, table, state_bf16);
  return nullptr;
}

}  // namespace cfi
