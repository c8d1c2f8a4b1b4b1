// Quantiser kernels for loader 1 (see quant_kernels.cuh).
#include "quant_dispatch.cuh"
namespace fp4 {
FP4_DEFINE_LAUNCH_QUANT(1)
}  // namespace fp4
