// cf_stream_mode_s1.cu -- instantiations of the streaming kernels for the
// 1-bit sign mode (one translation unit per mode so they compile in parallel).
#include "cf_stream_kernels.cuh"

namespace cfi {

const void *stream_kernel_s1(bool enc, int dtype, int nm_m, int nm_n, int vpt, bool table, bool state_bf16) {
  (void)nm_m;
  (void)nm_n;
  return pick_any<M_S1, 0, 0>(enc, dtype, vpt, table, state_bf16);
}

}  // namespace cfi
