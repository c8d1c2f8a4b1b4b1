// MXFP4 with fitted fractional-exponent scales, MXFP4-dagger ("Bridging the
// Gap Between Promise and Performance for Microscaling FP4 Quantization",
// "MXFP Scale Fitting", Appendix H, Table 11): instead of E8M0 powers of two,
// the 8-bit scale code q of a 32-element group stands for 2^(alpha q +
// L_min), where L_min, L_max are log2 of the tensor's smallest and largest
// AbsMax group scale s = gmax / 6 and alpha = (L_max - L_min) / 255.
//
// Three kernels:
//   k_fit_range  (grid-stride, 32 elements per lane, optional deterministic
//                block Hadamard): min and max of fp32(gmax / 6) over groups
//                with s > 0, as fp32 bit patterns (atomicMin / atomicMax);
//   k_fit_levels (one block): L = log2 of both in fp64, alpha, the fp32 table
//                of the 256 scales fp32(2^(L_min + alpha q)) and the 255
//                boundaries fp32(2^(L_min + alpha (k + 0.5))), all exponents in
//                fp64 (add and multiply rounded on their own), exp2 / log2 of
//                CUDA's math library;
//   k_fit_quant  the level of each group = the number of boundaries <= s
//                (binary search), d = table[q], codes RTN_E2M1(x * fp32(1/d)).
// A group with s = 0 (or a non-finite reciprocal scale) gets level 0 and zero
// codes; a tensor without s > 0 gets the table of s = 1.  These scales are
// not powers of two, so the E8M0 block scaling of the tensor cores cannot
// apply them: the format is quantised and de-quantised here, not multiplied.
#include "../../include/fp4.h"
#include "quant_dispatch.cuh"

namespace fp4 {
int* status_ptr();
namespace {

struct FitParams {
  const uint16_t* x;     // bf16 rows x cols
  int64_t rows, cols;
  uint8_t* codes;        // rows x cols / 2
  uint8_t* levels;       // rows x cols / 32
  float* table;          // 256
  uint32_t* range;       // workspace: [0] min, [1] max of s > 0 (fp32 bits)
  float* thr;            // workspace: 255 boundaries
  int* status;
};

// Input tasks: 32 consecutive elements of one row per lane, the (row, column)
// of lane task t = base + lane advanced by the grid stride.
template <int HAD>
__device__ __forceinline__ void load32(const FitParams& p, int64_t orow, int64_t ocol, bool active, int lane,
                                       float* x) {
  const uint4* src = reinterpret_cast<const uint4*>(p.x + orow * p.cols + ocol);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint4 v = active ? __ldg(src + i) : make_uint4(0, 0, 0, 0);
    bf16x8_to_f32(v, x + 8 * i);
  }
  if (HAD > 0) fwht32_lanes<HAD>(x, lane);
}

__device__ __forceinline__ float group_scale(const float* x) {
  const float gmax = bitsf(max(absmax16(x), absmax16(x + 16)));
  return __fdiv_rn(gmax, 6.0f);
}

template <int HAD>
__global__ void __launch_bounds__(256) k_fit_range(FitParams p) {
  __shared__ uint32_t red[2][8];
  const int lane = threadIdx.x & 31;
  const int64_t tpr = p.cols >> 5, tasks = p.rows * tpr, stride = int64_t(gridDim.x) * blockDim.x;
  uint32_t lo = 0xFFFFFFFFu, hi = 0u;
  bool bad = false;
  for (int64_t base = int64_t(blockIdx.x) * blockDim.x + (threadIdx.x & ~31); base < tasks; base += stride) {
    const int64_t t = base + lane;
    const bool active = t < tasks;
    float x[32];
    load32<HAD>(p, active ? t / tpr : 0, active ? (t % tpr) * 32 : 0, active, lane, x);
    const float s = group_scale(x);
    bad |= active && !(fabsf(s) < __int_as_float(0x7F800000));
    if (active && s > 0.0f) {
      lo = min(lo, fbits(s));
      hi = max(hi, fbits(s));
    }
  }
  if (__any_sync(0xFFFFFFFFu, bad) && lane == 0) flag_status(p.status, ST_NONFINITE);
  lo = __reduce_min_sync(0xFFFFFFFFu, lo);
  hi = __reduce_max_sync(0xFFFFFFFFu, hi);
  if (lane == 0) { red[0][threadIdx.x >> 5] = lo; red[1][threadIdx.x >> 5] = hi; }
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int w = 1; w < 8; ++w) { lo = min(lo, red[0][w]); hi = max(hi, red[1][w]); }
    if (hi > 0u) {
      atomicMin(p.range, lo);
      atomicMax(p.range + 1, hi);
    }
  }
}

__global__ void k_fit_levels(FitParams p) {
  const uint32_t lo = p.range[0], hi = p.range[1];
  const bool any = hi > 0u;
  const double s_min = any ? double(bitsf(lo)) : 1.0, s_max = any ? double(bitsf(hi)) : 1.0;
  const double l_min = log2(s_min), l_max = log2(s_max);
  const double alpha = __ddiv_rn(__dsub_rn(l_max, l_min), 255.0);
  const int q = threadIdx.x;
  p.table[q] = __double2float_rn(exp2(__dadd_rn(l_min, __dmul_rn(alpha, double(q)))));
  if (q < 255) p.thr[q] = __double2float_rn(exp2(__dadd_rn(l_min, __dmul_rn(alpha, __dadd_rn(double(q), 0.5)))));
}

template <int HAD>
__global__ void __launch_bounds__(256) k_fit_quant(FitParams p) {
  __shared__ float thr[256], table[256];
  thr[threadIdx.x] = threadIdx.x < 255 ? p.thr[threadIdx.x] : __int_as_float(0x7F800000);
  table[threadIdx.x] = p.table[threadIdx.x];
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int64_t tpr = p.cols >> 5, tasks = p.rows * tpr, stride = int64_t(gridDim.x) * blockDim.x;
  for (int64_t base = int64_t(blockIdx.x) * blockDim.x + (threadIdx.x & ~31); base < tasks; base += stride) {
    const int64_t t = base + lane;
    const bool active = t < tasks;
    const int64_t orow = active ? t / tpr : 0, ocol = active ? (t % tpr) * 32 : 0;
    float x[32];
    load32<HAD>(p, orow, ocol, active, lane, x);
    const float s = group_scale(x);
    // level = number of boundaries <= s (thr ascending; thr[255] = +inf)
    int q = 0;
#pragma unroll
    for (int step = 128; step >= 1; step >>= 1)
      if (thr[q + step - 1] <= s) q += step;
    const bool pos = s > 0.0f;
    q = pos ? q : 0;
    const float d = table[q], inv = __frcp_rn(d);
    const bool ok = pos && finite_pos(d, inv);
    uint32_t w[4];
    float v[32];
#pragma unroll
    for (int j = 0; j < 32; j += 2) st2(v, j, __fmul2_rn(ld2(x, j), splat2(inv)));
#pragma unroll
    for (int k = 0; k < 4; ++k) w[k] = ok ? enc8_hw(v + 8 * k) : 0u;
    if (active) {
      *reinterpret_cast<uint4*>(p.codes + orow * (p.cols >> 1) + (ocol >> 1)) = make_uint4(w[0], w[1], w[2], w[3]);
      p.levels[orow * (p.cols >> 5) + (ocol >> 5)] = uint8_t(q);
    }
  }
}

// De-quantisation: one 32-bit code word (8 elements of one group) per task,
// fp32(code * table[level]).
__global__ void __launch_bounds__(256) k_fit_dequant(const uint8_t* codes, const uint8_t* levels, const float* table,
                                                     int64_t rows, int64_t cols, float* out) {
  const int64_t wpr = cols >> 3, n = rows * wpr;
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n; i += int64_t(gridDim.x) * blockDim.x) {
    const int64_t r = i / wpr, c = (i - r * wpr) << 3;
    const float d = table[levels[r * (cols >> 5) + (c >> 5)]];
    float q[8];
    dec8(reinterpret_cast<const uint32_t*>(codes)[i], q);
    float4* o = reinterpret_cast<float4*>(out + (i << 3));
    o[0] = make_float4(__fmul_rn(q[0], d), __fmul_rn(q[1], d), __fmul_rn(q[2], d), __fmul_rn(q[3], d));
    o[1] = make_float4(__fmul_rn(q[4], d), __fmul_rn(q[5], d), __fmul_rn(q[6], d), __fmul_rn(q[7], d));
  }
}

template <int HAD>
cudaError_t launch_fit(const FitParams& p, cudaStream_t s) {
  const int64_t tasks = p.rows * (p.cols >> 5);
  int64_t blocks = (tasks + 255) / 256, cap = int64_t(num_sms()) * 4;
  blocks = blocks > cap ? cap : blocks;
  k_fit_range<HAD><<<unsigned(blocks), 256, 0, s>>>(p);
  k_fit_levels<<<1, 256, 0, s>>>(p);
  k_fit_quant<HAD><<<unsigned(blocks), 256, 0, s>>>(p);
  count_launch(3);
  return cudaGetLastError();
}

}  // namespace
}  // namespace fp4

using namespace fp4;

extern "C" size_t fp4_quantize_mx_fit_workspace_size(void) { return 1280; }   // 2 words, then 255 floats at 256

extern "C" int fp4_quantize_mx_fit(const void* x, int64_t rows, int64_t cols, int32_t had_block, uint8_t* codes,
                                   uint8_t* levels, float* table, void* ws, size_t ws_bytes, fp4_stream_t stream) {
  if (had_block != 0 && had_block != 16 && had_block != 32 && had_block != 64 && had_block != 128 && had_block != 256)
    return FP4_ERR_UNSUPPORTED;
  if (rows < 0 || cols < 0 || cols % 32 || (had_block && cols % had_block)) return FP4_ERR_INVALID_ARG;
  if (!table) return FP4_ERR_INVALID_ARG;
  auto al = [](const void* q, size_t a) { return (reinterpret_cast<uintptr_t>(q) % a) == 0; };
  if (!al(table, 4)) return FP4_ERR_ALIGNMENT;
  if (!ws || ws_bytes < fp4_quantize_mx_fit_workspace_size()) return FP4_ERR_WORKSPACE;
  if (!al(ws, 16)) return FP4_ERR_ALIGNMENT;
  if (rows > 0 && cols > 0) {
    if (!x || !codes || !levels) return FP4_ERR_INVALID_ARG;
    if (!al(x, 16) || !al(codes, 16)) return FP4_ERR_ALIGNMENT;
  }
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  FitParams p{};
  p.x = static_cast<const uint16_t*>(x); p.rows = rows; p.cols = cols;
  p.codes = codes; p.levels = levels; p.table = table;
  p.range = static_cast<uint32_t*>(ws);
  p.thr = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + 256);
  p.status = status_ptr();
  // range[0] starts above every finite pattern (all ones), range[1] at 0
  if (cudaMemsetAsync(p.range, 0xFF, 4, s) != cudaSuccess || cudaMemsetAsync(p.range + 1, 0, 4, s) != cudaSuccess)
    return FP4_ERR_CUDA;
  if (rows == 0 || cols == 0) {   // the table of s = 1 only
    k_fit_levels<<<1, 256, 0, s>>>(p);
    count_launch();
    return cudaGetLastError() == cudaSuccess ? FP4_OK : FP4_ERR_CUDA;
  }
  cudaError_t e;
  switch (had_block) {
    case 0: e = launch_fit<0>(p, s); break;
    case 16: e = launch_fit<16>(p, s); break;
    case 32: e = launch_fit<32>(p, s); break;
    case 64: e = launch_fit<64>(p, s); break;
    case 128: e = launch_fit<128>(p, s); break;
    default: e = launch_fit<256>(p, s); break;
  }
  return e == cudaSuccess ? FP4_OK : FP4_ERR_CUDA;
}

extern "C" int fp4_dequantize_mx_fit(const uint8_t* codes, const uint8_t* levels, const float* table, int64_t rows,
                                     int64_t cols, float* out, fp4_stream_t stream) {
  if (rows < 0 || cols < 0 || cols % 32) return FP4_ERR_INVALID_ARG;
  if (rows == 0 || cols == 0) return FP4_OK;
  if (!codes || !levels || !table || !out) return FP4_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(codes) % 4) || (reinterpret_cast<uintptr_t>(out) % 16)) return FP4_ERR_ALIGNMENT;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int64_t n = rows * (cols >> 3);
  int64_t blocks = (n + 255) / 256, cap = int64_t(num_sms()) * 8;
  blocks = blocks > cap ? cap : blocks;
  k_fit_dequant<<<unsigned(blocks), 256, 0, s>>>(codes, levels, table, rows, cols, out);
  count_launch();
  return cudaGetLastError() == cudaSuccess ? FP4_OK : FP4_ERR_CUDA;
}
