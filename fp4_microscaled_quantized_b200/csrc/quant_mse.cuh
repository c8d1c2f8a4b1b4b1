// NVFP4 with MSE-optimal scales by alternating optimisation ("Bridging the
// Gap Between Promise and Performance for Microscaling FP4 Quantization",
// "MSE-Optimized Grid and Scale Selection"): a group step that searches every
// E4M3 scale code of each 16-element group with the tensor scale held, and a
// tensor-scale step that solves the least-squares problem with the codes held.
#pragma once
#include <cstdint>
#include <cuda_runtime.h>

namespace fp4 {

// 32-element tasks of one group-step block: its 8192 elements are one aligned
// node of the pairwise tree the tensor-scale step sums over.
constexpr int MSE_TASKS = 256;

struct MseParams {
  const uint16_t* x;          // bf16, rows x cols row-major (cols % 32 == 0)
  int64_t rows, cols;
  uint8_t* codes;             // rows x cols / 2
  uint8_t* scales;            // rows x cols / 16 (may be null)
  uint8_t* swz;               // tensor-core scale layout (may be null)
  int64_t nkb;                // 4-group column blocks of the swizzled layout
  float* ts;                  // tensor scale s_T: written by the first step, read by the others
  const uint32_t* amax_bits;  // max |x| (fp32 bits), first step only
  double2* partial;           // per block: (<x, u>, <u, u>) of its 8192 elements
  int first;                  // 1: s_T = amax / (6 * 256) (1 for an all-zero tensor)
  int* status;
};

// Blocks of a group step over rows x cols.
inline int64_t mse_blocks(int64_t rows, int64_t cols) {
  const int64_t tasks = rows * (cols / 32);
  return (tasks + MSE_TASKS - 1) / MSE_TASKS;
}

cudaError_t launch_mse_group(const MseParams& p, cudaStream_t s);
cudaError_t launch_mse_tensor(const double2* partial, int64_t n, float* ts, cudaStream_t s);

}  // namespace fp4
