// Quantiser kernels for loader 0 (see quant_kernels.cuh).
#include "quant_dispatch.cuh"
namespace fp4 {
FP4_DEFINE_LAUNCH_QUANT(0)
}  // namespace fp4
