// Quantiser kernels for an already transformed fp32 input (fp4_quantize_f32):
// row-wise, no rotation, every format and rounding mode except MS-EDEN (which
// needs its rotation) and square blocks (bf16 input only).
#include "quant_dispatch.cuh"
namespace fp4 {
template <>
cudaError_t launch_quant<LD_ROW_F32>(int fmt, int rnd, int had, const QParams& p, cudaStream_t s) {
  if (had != 0) return cudaErrorInvalidValue;
  if (rnd == R_AMAX) return launch_one<LD_ROW_F32, FMT_NV, R_AMAX, 0>(p, s);
  if (fmt == FMT_NV) {
    switch (rnd) {
      case R_RTN: return launch_one<LD_ROW_F32, FMT_NV, R_RTN, 0>(p, s);
      case R_QUEST: return launch_one<LD_ROW_F32, FMT_NV, R_QUEST, 0>(p, s);
      case R_FOS: return launch_one<LD_ROW_F32, FMT_NV, R_FOS, 0>(p, s);
      case R_SR: return launch_one<LD_ROW_F32, FMT_NV, R_SR, 0>(p, s);
      default: return cudaErrorInvalidValue;
    }
  }
  switch (rnd) {
    case R_RTN: return launch_one<LD_ROW_F32, FMT_MX, R_RTN, 0>(p, s);
    case R_QUEST: return launch_one<LD_ROW_F32, FMT_MX, R_QUEST, 0>(p, s);
    case R_SR: return launch_one<LD_ROW_F32, FMT_MX, R_SR, 0>(p, s);
    default: return cudaErrorInvalidValue;
  }
}
}  // namespace fp4
