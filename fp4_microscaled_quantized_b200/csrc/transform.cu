// Dense orthonormal block transforms along the inner dimension: DCT-II and
// DST-II in blocks of k = 16 .. 256 ("Bridging the Gap Between Promise and
// Performance for Microscaling FP4 Quantization", the appendix on linear
// transforms, Tables 13-14: Hadamard, DCT, DST and GSR at block sizes 16 to
// 256 for the forward-pass rotation).  bf16 in, fp32 out; the quantisers
// then read the fp32 tensor (fp4_quantize_f32).
//
// Matrix entries (fp32, in the caller's workspace, rebuilt by every call):
// the orthonormal DCT-II C[i, j] = f_i cos(pi (2j + 1) i / (2k)) (f_0 =
// sqrt(1/k), f_i = sqrt(2/k)) and DST-II S[i, j] = g_i sin(pi (2j + 1)(i + 1)
// / (2k)) (g_{k-1} = sqrt(1/k), g_i = sqrt(2/k)).  Every entry is +-f times
// cos(pi m / (2k)) for a reduced index m in [0, k] (period 4k, cos(pi - t) =
// -cos t, sin t = cos(pi/2 - t)); the angle is fp64(pi) * m / (2k), the entry
// one fp64 product rounded once to fp32.
//
// Evaluation: y_i = pairwise tree over j of fp32(M[i, j] x_j) -- level 0 adds
// j = (2m, 2m + 1), then adjacent pair sums -- every product and sum rounded
// to fp32 on its own (the tree is built by a binary counter over j whose
// merge pattern the unrolled loop fixes at compile time).
#include <cuda_runtime.h>
#include <math_constants.h>

#include "../../include/fp4.h"
#include "device_common.cuh"

namespace fp4 {

namespace {

// cos(pi m / (2k)) for an integer m >= 0 reduced to [0, k] with its sign.
__device__ __forceinline__ double reduced_cos(int64_t m, int k) {
  m %= 4 * k;
  if (m > 2 * k) m = 4 * k - m;
  const bool neg = m > k;
  if (neg) m = 2 * k - m;
  const double c = cos(__ddiv_rn(__dmul_rn(CUDART_PI, double(m)), 2.0 * double(k)));
  return neg ? -c : c;
}

__global__ void k_dense_matrix(float* m, int k, int kind) {
  for (int t = blockIdx.x * blockDim.x + threadIdx.x; t < k * k; t += gridDim.x * blockDim.x) {
    const int i = t / k, j = t % k;
    double f, c;
    if (kind == FP4_XFORM_DCT2) {
      f = __dsqrt_rn((i == 0 ? 1.0 : 2.0) / double(k));
      c = reduced_cos(int64_t(2 * j + 1) * i, k);
    } else {
      f = __dsqrt_rn((i == k - 1 ? 1.0 : 2.0) / double(k));
      c = reduced_cos(int64_t(k) - int64_t(2 * j + 1) * (i + 1) + 8 * int64_t(k) * k, k);
    }
    m[t] = __double2float_rn(__dmul_rn(f, c));
  }
}

// One CTA: R rows x I outputs of one k-block (I = min(k, 32), R = 2 x 256 / I);
// each thread computes output i of two rows together (the products as one f32x2
// multiply, each half rounded as the scalar product).  The I matrix rows are
// staged in shared memory with a one-float skew so the 32 lanes' matrix reads
// hit distinct banks; the input is staged transposed, the two rows of a thread
// side by side (a 2-float skew per column), so a lane reads both rows' x_j in
// one 8-byte load.  Tree levels above the first add sums only and run two rows
// per instruction; the first level, whose operands are products, is scalar (a
// packed add of packed products may be contracted into a multiply-add).
template <int K>
constexpr int dense_threads() { return K == 256 ? 128 : 256; }   // 256-blocks: the staging fits 48 KB

template <int K>
__global__ void __launch_bounds__(dense_threads<K>()) k_dense_transform(const uint16_t* __restrict__ x,
                                                                      float* __restrict__ y,
                                                                      const float* __restrict__ m, int64_t rows,
                                                                      int64_t cols) {
  constexpr int NT = dense_threads<K>();
  constexpr int I = K < 32 ? K : 32, RP = NT / I, R = 2 * RP, P = K + 1, XP = R + 2, DEPTH = 9;
  constexpr int ROOT = K == 16 ? 4 : K == 32 ? 5 : K == 64 ? 6 : K == 128 ? 7 : 8;   // log2 K
  __shared__ float sm[I][P];
  __shared__ __align__(8) float sx[K][XP];          // sx[j][r] = x[r0 + r][c0 + j]
  const int64_t r0 = int64_t(blockIdx.x) * R, c0 = int64_t(blockIdx.y) * K;
  const int i0 = blockIdx.z * I;
  for (int t = threadIdx.x; t < I * K; t += NT) sm[t / K][t % K] = m[(i0 + t / K) * K + t % K];
  for (int t = threadIdx.x; t < R * K; t += NT) {
    const int64_t r = r0 + t / K;
    sx[t % K][t / K] = r < rows ? __uint_as_float(uint32_t(x[r * cols + c0 + t % K]) << 16) : 0.0f;
  }
  __syncthreads();
  const int i = threadIdx.x % I, rp = threadIdx.x / I;
  float2 stack[DEPTH];
#pragma unroll
  for (int j = 0; j < K; ++j) {
    float2 v = __fmul2_rn(make_float2(sm[i][j], sm[i][j]), *reinterpret_cast<const float2*>(&sx[j][2 * rp]));
    int level = 0;
    if (j & 1) {                          // leaf j closes the subtrees of its trailing one bits
      v = make_float2(__fadd_rn(stack[0].x, v.x), __fadd_rn(stack[0].y, v.y));
      level = 1;
#pragma unroll
      for (int b = 1; b < DEPTH; ++b) {
        if (((j >> b) & 1) == 0) break;
        v = __fadd2_rn(stack[b], v);
        level = b + 1;
      }
    }
    stack[level] = v;
  }
  const int64_t ra = r0 + 2 * rp;
  if (ra < rows) y[ra * cols + c0 + i0 + i] = stack[ROOT].x;
  if (ra + 1 < rows) y[(ra + 1) * cols + c0 + i0 + i] = stack[ROOT].y;
}

template <int K>
cudaError_t launch_dense(const uint16_t* x, float* y, const float* m, int64_t rows, int64_t cols, cudaStream_t s) {
  constexpr int I = K < 32 ? K : 32, R = 2 * dense_threads<K>() / I;
  const dim3 grid(unsigned((rows + R - 1) / R), unsigned(cols / K), unsigned(K / I));
  k_dense_transform<K><<<grid, dense_threads<K>(), 0, s>>>(x, y, m, rows, cols);
  count_launch();
  return cudaGetLastError();
}

}  // namespace
}  // namespace fp4

using namespace fp4;

extern "C" size_t fp4_block_transform_workspace_size(int32_t block) {
  return (block == 16 || block == 32 || block == 64 || block == 128 || block == 256) ? size_t(block) * block * 4 : 0;
}

extern "C" int fp4_block_transform(const void* x, float* y, int64_t rows, int64_t cols, int32_t kind, int32_t block,
                                   void* ws, size_t ws_bytes, fp4_stream_t stream) {
  if (kind != FP4_XFORM_DCT2 && kind != FP4_XFORM_DST2) return FP4_ERR_UNSUPPORTED;
  const size_t need = fp4_block_transform_workspace_size(block);
  if (!need) return FP4_ERR_UNSUPPORTED;
  if (rows < 0 || cols < 0 || cols % block) return FP4_ERR_INVALID_ARG;
  if (rows == 0 || cols == 0) return FP4_OK;
  if (!x || !y) return FP4_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(x) % 16) || (reinterpret_cast<uintptr_t>(y) % 16)) return FP4_ERR_ALIGNMENT;
  if (!ws || ws_bytes < need) return FP4_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(ws) % 16) return FP4_ERR_ALIGNMENT;
  if (cols / block > 65535) return FP4_ERR_INVALID_ARG;   // one grid column per k-block
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  float* m = static_cast<float*>(ws);
  k_dense_matrix<<<unsigned((block * block + 255) / 256), 256, 0, s>>>(m, block, kind);
  count_launch();
  if (cudaGetLastError() != cudaSuccess) return FP4_ERR_CUDA;
  const uint16_t* xb = static_cast<const uint16_t*>(x);
  cudaError_t e;
  switch (block) {
    case 16: e = launch_dense<16>(xb, y, m, rows, cols, s); break;
    case 32: e = launch_dense<32>(xb, y, m, rows, cols, s); break;
    case 64: e = launch_dense<64>(xb, y, m, rows, cols, s); break;
    case 128: e = launch_dense<128>(xb, y, m, rows, cols, s); break;
    default: e = launch_dense<256>(xb, y, m, rows, cols, s); break;
  }
  return e == cudaSuccess ? FP4_OK : FP4_ERR_CUDA;
}
