// Quantiser kernels for loader 3 (see quant_kernels.cuh).
#include "quant_dispatch.cuh"
namespace fp4 {
FP4_DEFINE_LAUNCH_QUANT(3)
}  // namespace fp4
