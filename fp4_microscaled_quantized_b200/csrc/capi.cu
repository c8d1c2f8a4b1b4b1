// C ABI entry points of the quantisation path (include/fp4.h): argument
// validation, workspace layout, kernel sequencing and the device status word.
#include <atomic>
#include <mutex>

#include "../../include/fp4.h"
#include "quant_dispatch.cuh"
#include "quant_mse.cuh"

namespace fp4 {

__device__ int g_status = 0;

static std::atomic<unsigned long long> g_launches{0};
void count_launch(int n) { g_launches.fetch_add(static_cast<unsigned long long>(n)); }

int num_sms() {
  static std::atomic<int> cached[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return 148;
  int v = cached[dev].load(std::memory_order_relaxed);
  if (!v) {
    int n = 0;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    v = n > 0 ? n : 148;
    cached[dev].store(v, std::memory_order_relaxed);   // every thread computes the same value
  }
  return v;
}

// Address of the status word on the current device (looked up once per device).
int* status_ptr() {
  static std::mutex mu;
  static int* addr[64] = {nullptr};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> g(mu);
  if (!addr[dev]) {
    void* a = nullptr;
    if (cudaGetSymbolAddress(&a, g_status) != cudaSuccess) return nullptr;
    addr[dev] = static_cast<int*>(a);
  }
  return addr[dev];
}

static inline bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }
static inline size_t align256(size_t n) { return (n + 255) & ~size_t(255); }

struct WsLayout {
  size_t amax = 0, pseudo = 0, eden = 0, bmax = 0, total = 0;
};

static WsLayout ws_layout(int64_t rows, int64_t cols, int fmt, int rnd, int had) {
  WsLayout w;
  if (fmt == FP4_NVFP4 && rnd == FP4_RTN_SQUARE16) {
    w.bmax = 256;
    w.total = w.bmax + align256(size_t(rows / 16) * size_t(cols / 16) * 4);
  } else if (fmt == FP4_NVFP4 && rnd == FP4_MS_EDEN && had > 0) {
    w.amax = 0;
    w.pseudo = 256;
    w.eden = w.pseudo + align256(size_t(rows) * size_t(cols / 16) * 2);
    w.total = w.eden + align256(size_t(rows) * size_t(cols / had) * 4);
  } else if (fmt == FP4_NVFP4) {
    w.total = 256;
  }
  return w;
}

static bool combo_supported(int fmt, int rnd, int had) {
  if (had != 0 && had != 16 && had != 32 && had != 64 && had != 128 && had != 256) return false;
  if (fmt == FP4_MXFP4 && (rnd == FP4_FOUR_OVER_SIX || rnd == FP4_MS_EDEN)) return false;
  int g = fmt == FP4_NVFP4 ? 16 : 32;
  if (rnd == FP4_MS_EDEN && (had == 0 || had < g)) return false;
  if (rnd == FP4_RTN_SQUARE16 && (fmt != FP4_NVFP4 || had != 0)) return false;
  return true;
}

static int check_out(const fp4_qtensor* out) {
  if (!out || !out->codes || !out->tensor_scale || (!out->scales && !out->scales_swz))
    return FP4_ERR_INVALID_ARG;
  if (!aligned(out->codes, 16) || (out->scales_swz && !aligned(out->scales_swz, 16)) ||
      (out->scales && !aligned(out->scales, 16)) || (out->mask && !aligned(out->mask, 16)) ||
      !aligned(out->tensor_scale, 4))
    return FP4_ERR_ALIGNMENT;
  return FP4_OK;
}

__global__ void k_swizzle(const uint8_t* sc, int64_t rows, int64_t ng, int64_t nkb, uint8_t* swz) {
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < rows * ng;
       i += int64_t(gridDim.x) * blockDim.x)
    swz[swz_offset(i / ng, i % ng, nkb)] = sc[i];
}

// De-quantisation: 8 elements (one 32-bit code word, inside one scale group)
// per task, fp32(fp32(q * s_group) * s_tensor), written as fp32 or bf16.
template <int OUT>
__global__ void __launch_bounds__(256) k_dequant(const uint8_t* codes, const uint8_t* scales, const float* ts,
                                                 int fmt, int64_t rows, int64_t cols, void* D) {
  const int64_t words_per_row = cols >> 3, n = rows * words_per_row;
  const int gsh = fmt == FP4_NVFP4 ? 4 : 5;
  const float t = *ts;
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n; i += int64_t(gridDim.x) * blockDim.x) {
    const int64_t r = i / words_per_row, c = (i - r * words_per_row) << 3;
    const uint32_t w = reinterpret_cast<const uint32_t*>(codes)[i];
    const uint32_t sc = scales[r * (cols >> gsh) + (c >> gsh)];
    const float sg = fmt == FP4_NVFP4 ? e4m3_value(sc) : pow2f(int(sc) - 127);
    float q[8];
    dec8(w, q);
#pragma unroll
    for (int j = 0; j < 8; ++j) q[j] = __fmul_rn(__fmul_rn(q[j], sg), t);
    if (OUT == 0) {
      float4* d = reinterpret_cast<float4*>(static_cast<float*>(D) + (i << 3));
      d[0] = make_float4(q[0], q[1], q[2], q[3]);
      d[1] = make_float4(q[4], q[5], q[6], q[7]);
    } else {
      uint32_t h[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const __nv_bfloat162 b = __floats2bfloat162_rn(q[2 * j], q[2 * j + 1]);
        h[j] = *reinterpret_cast<const uint32_t*>(&b);
      }
      *reinterpret_cast<uint4*>(static_cast<uint16_t*>(D) + (i << 3)) = make_uint4(h[0], h[1], h[2], h[3]);
    }
  }
}

// Transpose of FP4 codes (rows x cols, 2 per byte) in 64 x 64 tiles: the
// tile's 64 input rows x 32 bytes are read as 8-byte chunks (coalesced),
// spread to one code per byte in shared memory, and written back as 64
// output rows x 32 bytes.
__global__ void __launch_bounds__(256) k_transpose_codes(const uint8_t* in, int64_t rows, int64_t cols, uint8_t* out) {
  __shared__ uint8_t tile[64][65];
  const int64_t r0 = int64_t(blockIdx.y) * 64, c0 = int64_t(blockIdx.x) * 64;
  const int t = threadIdx.x, tr = t >> 2, tc = (t & 3) * 16;      // one row, 16 codes
  const uint2 w = *reinterpret_cast<const uint2*>(in + (r0 + tr) * (cols >> 1) + ((c0 + tc) >> 1));
  const uint32_t ww[2] = {w.x, w.y};
#pragma unroll
  for (int j = 0; j < 16; ++j) tile[tr][tc + j] = uint8_t((ww[j >> 3] >> (4 * (j & 7))) & 15u);
  __syncthreads();
  // output row c0 + tr, codes of input rows r0 + tc .. r0 + tc + 15
  uint32_t o[2] = {0u, 0u};
#pragma unroll
  for (int j = 0; j < 16; ++j) o[j >> 3] |= uint32_t(tile[tc + j][tr]) << (4 * (j & 7));
  *reinterpret_cast<uint2*>(out + (c0 + tr) * (rows >> 1) + ((r0 + tc) >> 1)) = make_uint2(o[0], o[1]);
}

// Scales of the transposed square-block tensor: output (r, k) (r an input
// column, k a 16-group of input rows) takes the block scale of input block
// (k, r / 16), i.e. input scale (16 k, r / 16); linear and/or tensor-core
// layout.  Thread 0 also copies the tensor scale.
__global__ void __launch_bounds__(256) k_transpose_sq16_scales(const uint8_t* in_sc, const float* in_ts, int64_t rows,
                                                               int64_t cols, uint8_t* out_sc, uint8_t* out_swz,
                                                               float* out_ts, int64_t nkb) {
  const int64_t ng = rows >> 4, n = cols * ng;      // output: cols rows x rows/16 groups
  if (blockIdx.x == 0 && threadIdx.x == 0) *out_ts = *in_ts;
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n; i += int64_t(gridDim.x) * blockDim.x) {
    const int64_t r = i / ng, k = i - r * ng;
    const uint8_t v = in_sc[(k << 4) * (cols >> 4) + (r >> 4)];
    if (out_sc) out_sc[i] = v;
    if (out_swz) out_swz[swz_offset(r, k, nkb)] = v;
  }
}

static int launch_pad(uint8_t* swz, int64_t rows, int64_t ng, cudaStream_t s) {
  int64_t nkb = (ng + 3) / 4;
  if (!swz || ((rows % 128) == 0 && (ng % 4) == 0)) return FP4_OK;
  int64_t n = (((rows + 127) / 128) * 128 - rows) * nkb * 4 + rows * (nkb * 4 - ng);
  int64_t blocks = (n + 255) / 256;
  if (blocks > 4096) blocks = 4096;
  k_swz_pad<<<unsigned(blocks), 256, 0, s>>>(swz, rows, ng, nkb);
  count_launch();
  return cudaGetLastError() == cudaSuccess ? FP4_OK : FP4_ERR_CUDA;
}

// Shared sequencing of fp4_quantize / fp4_requantize.
// Maxima |x| of the 16 x 16 blocks of a bf16 tensor (rows x cols, both
// multiples of 16), one block per thread (consecutive threads: consecutive
// blocks of a block row, so each of the 16 row loads of a warp is one
// contiguous run), as fp32 bits; the block-wide maximum goes to the global
// amax word.  With the sign bit cleared, |x| orders as an unsigned 16-bit
// integer (NaN patterns above infinity).
__global__ void __launch_bounds__(256) k_block16_max(const uint16_t* x, int64_t rows, int64_t cols, uint32_t* bmax,
                                                     uint32_t* amax, int* status) {
  __shared__ Shared sh;
  const int64_t nbc = cols >> 4, nb = (rows >> 4) * nbc;
  uint32_t acc = 0;
  for (int64_t b = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; b < nb; b += int64_t(gridDim.x) * blockDim.x) {
    const int64_t br = b / nbc, bc = b - br * nbc;
    const uint16_t* src = x + (br << 4) * cols + (bc << 4);
    uint32_t m2 = 0;
#pragma unroll 4
    for (int r = 0; r < 16; ++r) {
      const uint4* row = reinterpret_cast<const uint4*>(src + r * cols);
      const uint4 u = __ldg(row), v = __ldg(row + 1);
      m2 = __vmaxu2(m2, __vmaxu2(__vmaxu2(u.x & 0x7FFF7FFFu, u.y & 0x7FFF7FFFu),
                                 __vmaxu2(u.z & 0x7FFF7FFFu, u.w & 0x7FFF7FFFu)));
      m2 = __vmaxu2(m2, __vmaxu2(__vmaxu2(v.x & 0x7FFF7FFFu, v.y & 0x7FFF7FFFu),
                                 __vmaxu2(v.z & 0x7FFF7FFFu, v.w & 0x7FFF7FFFu)));
    }
    const uint32_t m = max(m2 & 0xFFFFu, m2 >> 16) << 16;
    bmax[b] = m;
    acc = max(acc, m);
  }
  block_max_atomic(acc, sh, amax, status);
}

static int run_quant(int load, int fmt, int rnd, int had, QParams& p, void* ws, size_t ws_bytes,
                     cudaStream_t s) {
  WsLayout L = ws_layout(p.rows, p.cols, fmt, rnd, had);
  if (L.total > 0) {
    if (!ws || ws_bytes < L.total) return FP4_ERR_WORKSPACE;
    if (!aligned(ws, 16)) return FP4_ERR_ALIGNMENT;
  }
  uint8_t* w = static_cast<uint8_t*>(ws);
  p.amax_bits = L.total ? reinterpret_cast<uint32_t*>(w + L.amax) : nullptr;
  p.pseudo = (L.pseudo ? reinterpret_cast<uint16_t*>(w + L.pseudo) : nullptr);
  p.eden_S = (L.eden ? reinterpret_cast<float*>(w + L.eden) : nullptr);
  uint32_t* bmax = L.bmax ? reinterpret_cast<uint32_t*>(w + L.bmax) : nullptr;
  p.status = status_ptr();
  p.nkb = ((p.cols / (fmt == FP4_NVFP4 ? 16 : 32)) + 3) / 4;
  auto launch = [&](int r) -> cudaError_t {
    switch (load) {
      case LD_ROW: return launch_quant<LD_ROW>(fmt, r, had, p, s);
      case LD_TRANS: return launch_quant<LD_TRANS>(fmt, r, had, p, s);
      case LD_ROW_FP4: return launch_quant<LD_ROW_FP4>(fmt, r, had, p, s);
      case LD_ROW_F32: return launch_quant<LD_ROW_F32>(fmt, r, had, p, s);
      default: return launch_quant<LD_TRANS_FP4>(fmt, r, had, p, s);
    }
  };
  if (fmt == FP4_NVFP4) {
    if (cudaMemsetAsync(p.amax_bits, 0, sizeof(uint32_t), s) != cudaSuccess) return FP4_ERR_CUDA;
    if (rnd == FP4_RTN_SQUARE16) {
      // block maxima of the input (and the global amax with them)
      const int64_t nb = (p.in_rows / 16) * (p.in_cols / 16);
      int64_t blocks = (nb + 255) / 256, cap = int64_t(num_sms()) * 8;
      if (blocks > cap) blocks = cap;
      if (blocks < 1) blocks = 1;
      k_block16_max<<<unsigned(blocks), 256, 0, s>>>(static_cast<const uint16_t*>(p.x), p.in_rows, p.in_cols,
                                                     bmax, p.amax_bits, p.status);
      count_launch();
      if (cudaGetLastError() != cudaSuccess) return FP4_ERR_CUDA;
      p.bmax = bmax;
      p.bmax_ld = p.in_cols / 16;
      p.bmax_trans = load == LD_TRANS ? 1 : 0;
    } else if (rnd != FP4_MS_EDEN && launch(R_AMAX) != cudaSuccess) {
      return FP4_ERR_CUDA;
    }
  }
  if (launch(rnd == FP4_RTN_SQUARE16 ? R_SQ16 : rnd) != cudaSuccess) return FP4_ERR_CUDA;
  if (rnd == FP4_MS_EDEN) {
    int64_t groups = p.rows * (p.cols / 16);
    int64_t blocks = (groups + 255) / 256, cap = int64_t(num_sms()) * 8;
    if (blocks > cap) blocks = cap;
    switch (had) {
      case 16: k_eden_pass2<16><<<unsigned(blocks), 256, 0, s>>>(p); break;
      case 32: k_eden_pass2<32><<<unsigned(blocks), 256, 0, s>>>(p); break;
      case 64: k_eden_pass2<64><<<unsigned(blocks), 256, 0, s>>>(p); break;
      case 128: k_eden_pass2<128><<<unsigned(blocks), 256, 0, s>>>(p); break;
      default: k_eden_pass2<256><<<unsigned(blocks), 256, 0, s>>>(p); break;
    }
    count_launch();
    if (cudaGetLastError() != cudaSuccess) return FP4_ERR_CUDA;
  }
  return launch_pad(p.swz, p.rows, p.cols / (fmt == FP4_NVFP4 ? 16 : 32), s);
}

}  // namespace fp4

using namespace fp4;

extern "C" {

size_t fp4_quantize_workspace_size(int64_t rows, int64_t cols, int32_t fmt, int32_t rounding,
                                   int32_t had_block) {
  if (rows < 0 || cols < 0) return 0;
  return ws_layout(rows, cols, fmt, rounding, had_block).total;
}

size_t fp4_swizzled_scale_bytes(int64_t rows, int64_t n_groups) {
  if (rows <= 0 || n_groups <= 0) return 0;
  return size_t((rows + 127) / 128) * size_t((n_groups + 3) / 4) * 512;
}

}  // extern "C"

namespace fp4 {
// Every argument check of fp4_quantize before its workspace check, in the
// same order (fp4_quantize_noalloc runs them before its scratch-size check so
// both entry points return the same status for the same arguments).  Sets
// out's shape fields; *empty is set for a tensor with no elements (valid,
// nothing to launch).
static int quantize_args(const void* x, int64_t in_rows, int64_t in_cols, int32_t transpose, int32_t fmt,
                         int32_t rounding, int32_t group, fp4_had had, fp4_qtensor* out, bool* empty) {
  *empty = false;
  if (fmt != FP4_MXFP4 && fmt != FP4_NVFP4) return FP4_ERR_INVALID_ARG;
  if (rounding < FP4_RTN || rounding > FP4_RTN_SQUARE16) return FP4_ERR_INVALID_ARG;
  const int g = fmt == FP4_NVFP4 ? 16 : 32;
  if (group != g) return FP4_ERR_UNSUPPORTED;
  if (!combo_supported(fmt, rounding, had.block)) return FP4_ERR_UNSUPPORTED;
  // square blocks: whole 16 x 16 blocks and 32-element rows of the output
  if (rounding == FP4_RTN_SQUARE16 && (in_rows % 16 || in_cols % 16 || (transpose ? in_rows : in_cols) % 32))
    return FP4_ERR_INVALID_ARG;
  if (in_rows < 0 || in_cols < 0 || (transpose != 0 && transpose != 1) || !out)
    return FP4_ERR_INVALID_ARG;
  const int64_t rows = transpose ? in_cols : in_rows, cols = transpose ? in_rows : in_cols;
  const int64_t chunk = had.block > g ? had.block : g;
  if (cols % chunk) return FP4_ERR_INVALID_ARG;
  if (transpose && (in_cols % 8)) return FP4_ERR_ALIGNMENT;
  out->rows = rows; out->cols = cols; out->fmt = fmt;
  if (rows == 0 || cols == 0) {   // empty tensor: nothing to launch
    *empty = true;
    return FP4_OK;
  }
  int st = check_out(out);
  if (st) return st;
  if (!x) return FP4_ERR_INVALID_ARG;
  if (!aligned(x, 16)) return FP4_ERR_ALIGNMENT;
  return FP4_OK;
}
}  // namespace fp4

extern "C" {

int fp4_quantize(const void* x, int64_t in_rows, int64_t in_cols, int32_t transpose, int32_t fmt,
                 int32_t rounding, int32_t group, fp4_had had, uint64_t seed, uint32_t tensor_tag,
                 fp4_qtensor* out, void* ws, size_t ws_bytes, fp4_stream_t stream) {
  bool empty = false;
  const int st = quantize_args(x, in_rows, in_cols, transpose, fmt, rounding, group, had, out, &empty);
  if (st || empty) return st;
  const int64_t rows = out->rows, cols = out->cols;
  QParams p{};
  p.x = x; p.in_rows = in_rows; p.in_cols = in_cols; p.rows = rows; p.cols = cols;
  p.codes = out->codes; p.scales = out->scales; p.swz = out->scales_swz; p.mask = out->mask;
  p.ts = out->tensor_scale; p.seed = seed; p.tensor_tag = tensor_tag; p.sign_tag = had.sign_tag;
  p.randomized = had.randomized ? 1 : 0;
  return run_quant(transpose ? LD_TRANS : LD_ROW, fmt, rounding, had.block, p, ws, ws_bytes,
                   reinterpret_cast<cudaStream_t>(stream));
}

int fp4_quantize_f32(const float* y, int64_t rows, int64_t cols, int32_t fmt, int32_t rounding, int32_t group,
                     uint64_t seed, uint32_t tensor_tag, fp4_qtensor* out, void* ws, size_t ws_bytes,
                     fp4_stream_t stream) {
  if (fmt != FP4_MXFP4 && fmt != FP4_NVFP4) return FP4_ERR_INVALID_ARG;
  if (rounding < FP4_RTN || rounding > FP4_RTN_SQUARE16) return FP4_ERR_INVALID_ARG;
  if (group != (fmt == FP4_NVFP4 ? 16 : 32)) return FP4_ERR_UNSUPPORTED;
  // MS-EDEN needs its own rotation; square blocks read bf16 block maxima
  if (rounding == FP4_MS_EDEN || rounding == FP4_RTN_SQUARE16 || !combo_supported(fmt, rounding, 0))
    return FP4_ERR_UNSUPPORTED;
  if (rows < 0 || cols < 0 || cols % 32 || !out) return FP4_ERR_INVALID_ARG;
  out->rows = rows; out->cols = cols; out->fmt = fmt;
  if (rows == 0 || cols == 0) return FP4_OK;
  int st = check_out(out);
  if (st) return st;
  if (!y) return FP4_ERR_INVALID_ARG;
  if (!aligned(y, 16)) return FP4_ERR_ALIGNMENT;
  QParams p{};
  p.x = y; p.in_rows = rows; p.in_cols = cols; p.rows = rows; p.cols = cols;
  p.codes = out->codes; p.scales = out->scales; p.swz = out->scales_swz; p.mask = out->mask;
  p.ts = out->tensor_scale; p.seed = seed; p.tensor_tag = tensor_tag;
  return run_quant(LD_ROW_F32, fmt, rounding, 0, p, ws, ws_bytes, reinterpret_cast<cudaStream_t>(stream));
}

int fp4_requantize(const fp4_qtensor* in, int32_t transpose, int32_t rounding, fp4_had had,
                   uint64_t seed, uint32_t tensor_tag, fp4_qtensor* out, void* ws, size_t ws_bytes,
                   fp4_stream_t stream) {
  if (!in) return FP4_ERR_INVALID_ARG;
  if ((in->rows > 0 && in->cols > 0) && (!in->codes || !in->scales || !in->tensor_scale))
    return FP4_ERR_INVALID_ARG;
  if (in->fmt != FP4_MXFP4 && in->fmt != FP4_NVFP4) return FP4_ERR_INVALID_ARG;
  if (rounding < FP4_RTN || rounding > FP4_RTN_SQUARE16 || (transpose != 0 && transpose != 1))
    return FP4_ERR_INVALID_ARG;
  if (rounding == FP4_RTN_SQUARE16) return FP4_ERR_UNSUPPORTED;   // bf16 input only
  const int fmt = in->fmt, g = fmt == FP4_NVFP4 ? 16 : 32;
  if (!combo_supported(fmt, rounding, had.block)) return FP4_ERR_UNSUPPORTED;
  if (in->rows < 0 || in->cols < 0 || in->cols % g || !out) return FP4_ERR_INVALID_ARG;
  const int64_t rows = transpose ? in->cols : in->rows, cols = transpose ? in->rows : in->cols;
  const int64_t chunk = had.block > g ? had.block : g;
  if (cols % chunk) return FP4_ERR_INVALID_ARG;
  if (transpose && (in->cols % 16)) return FP4_ERR_ALIGNMENT;
  out->rows = rows; out->cols = cols; out->fmt = fmt;
  if (rows == 0 || cols == 0) return FP4_OK;
  int st = check_out(out);
  if (st) return st;
  if (!aligned(in->codes, 16)) return FP4_ERR_ALIGNMENT;
  QParams p{};
  p.x = in->codes; p.in_scales = in->scales; p.in_ts = in->tensor_scale; p.in_fmt = fmt;
  p.in_rows = in->rows; p.in_cols = in->cols; p.rows = rows; p.cols = cols;
  p.codes = out->codes; p.scales = out->scales; p.swz = out->scales_swz; p.mask = out->mask;
  p.ts = out->tensor_scale; p.seed = seed; p.tensor_tag = tensor_tag; p.sign_tag = had.sign_tag;
  p.randomized = had.randomized ? 1 : 0;
  return run_quant(transpose ? LD_TRANS_FP4 : LD_ROW_FP4, fmt, rounding, had.block, p, ws,
                   ws_bytes, reinterpret_cast<cudaStream_t>(stream));
}

size_t fp4_quantize_mse_workspace_size(int64_t rows, int64_t cols) {
  if (rows < 0 || cols < 0 || cols % 32) return 0;
  return 256 + align256(size_t(mse_blocks(rows, cols)) * sizeof(double2));
}

int fp4_quantize_mse(const void* x, int64_t rows, int64_t cols, int32_t iters, fp4_qtensor* out, void* ws,
                     size_t ws_bytes, fp4_stream_t stream) {
  if (rows < 0 || cols < 0 || cols % 32 || iters < 0 || iters > 64 || !out) return FP4_ERR_INVALID_ARG;
  out->rows = rows; out->cols = cols; out->fmt = FP4_NVFP4;
  if (rows == 0 || cols == 0) return FP4_OK;
  int st = check_out(out);
  if (st) return st;
  if (!x) return FP4_ERR_INVALID_ARG;
  if (!aligned(x, 16)) return FP4_ERR_ALIGNMENT;
  const size_t need = fp4_quantize_mse_workspace_size(rows, cols);
  if (!ws || ws_bytes < need) return FP4_ERR_WORKSPACE;
  if (!aligned(ws, 16)) return FP4_ERR_ALIGNMENT;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* w = static_cast<uint8_t*>(ws);
  QParams p{};
  p.x = x; p.in_rows = rows; p.in_cols = cols; p.rows = rows; p.cols = cols;
  p.amax_bits = reinterpret_cast<uint32_t*>(w);
  p.status = status_ptr();
  p.nkb = ((cols / 16) + 3) / 4;
  if (cudaMemsetAsync(p.amax_bits, 0, sizeof(uint32_t), s) != cudaSuccess) return FP4_ERR_CUDA;
  if (launch_quant<LD_ROW>(FP4_NVFP4, R_AMAX, 0, p, s) != cudaSuccess) return FP4_ERR_CUDA;
  MseParams m{};
  m.x = static_cast<const uint16_t*>(x); m.rows = rows; m.cols = cols;
  m.codes = out->codes; m.scales = out->scales; m.swz = out->scales_swz; m.nkb = p.nkb;
  m.ts = out->tensor_scale; m.amax_bits = p.amax_bits;
  m.partial = reinterpret_cast<double2*>(w + 256);
  m.status = p.status;
  m.first = 1;
  if (launch_mse_group(m, s) != cudaSuccess) return FP4_ERR_CUDA;
  m.first = 0;
  for (int i = 0; i < iters; ++i) {
    if (launch_mse_tensor(m.partial, mse_blocks(rows, cols), m.ts, s) != cudaSuccess) return FP4_ERR_CUDA;
    if (launch_mse_group(m, s) != cudaSuccess) return FP4_ERR_CUDA;
  }
  return launch_pad(out->scales_swz, rows, cols / 16, s);
}

int fp4_dequantize(const fp4_qtensor* in, void* D, int32_t out_dtype, fp4_stream_t stream) {
  if (!in || (in->fmt != FP4_MXFP4 && in->fmt != FP4_NVFP4) || (out_dtype != 0 && out_dtype != 1))
    return FP4_ERR_INVALID_ARG;
  const int g = in->fmt == FP4_NVFP4 ? 16 : 32;
  if (in->rows < 0 || in->cols < 0 || in->cols % g) return FP4_ERR_INVALID_ARG;
  if (in->rows == 0 || in->cols == 0) return FP4_OK;
  if (!in->codes || !in->scales || !in->tensor_scale || !D) return FP4_ERR_INVALID_ARG;
  if (!aligned(in->codes, 16) || !aligned(D, 16) || !aligned(in->tensor_scale, 4)) return FP4_ERR_ALIGNMENT;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int64_t n = in->rows * (in->cols >> 3);
  int64_t blocks = (n + 255) / 256, cap = int64_t(num_sms()) * 8;
  if (blocks > cap) blocks = cap;
  if (out_dtype == 0)
    k_dequant<0><<<unsigned(blocks), 256, 0, s>>>(in->codes, in->scales, in->tensor_scale, in->fmt, in->rows, in->cols, D);
  else
    k_dequant<1><<<unsigned(blocks), 256, 0, s>>>(in->codes, in->scales, in->tensor_scale, in->fmt, in->rows, in->cols, D);
  count_launch();
  return cudaGetLastError() == cudaSuccess ? FP4_OK : FP4_ERR_CUDA;
}

int fp4_transpose_square16(const fp4_qtensor* in, fp4_qtensor* out, fp4_stream_t stream) {
  if (!in || !out || in->fmt != FP4_NVFP4) return FP4_ERR_INVALID_ARG;
  if (in->rows < 0 || in->cols < 0 || in->rows % 64 || in->cols % 64) return FP4_ERR_INVALID_ARG;
  out->rows = in->cols; out->cols = in->rows; out->fmt = FP4_NVFP4;
  if (in->rows == 0 || in->cols == 0) return FP4_OK;
  if (!in->codes || !in->scales || !in->tensor_scale) return FP4_ERR_INVALID_ARG;
  int st = check_out(out);
  if (st) return st;
  if (!aligned(in->codes, 16)) return FP4_ERR_ALIGNMENT;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const dim3 grid(unsigned(in->cols / 64), unsigned(in->rows / 64));
  k_transpose_codes<<<grid, 256, 0, s>>>(in->codes, in->rows, in->cols, out->codes);
  count_launch();
  const int64_t ng = in->rows / 16, n = in->cols * ng, nkb = (ng + 3) / 4;
  int64_t blocks = (n + 255) / 256, cap = int64_t(num_sms()) * 8;
  if (blocks > cap) blocks = cap;
  k_transpose_sq16_scales<<<unsigned(blocks), 256, 0, s>>>(in->scales, in->tensor_scale, in->rows, in->cols,
                                                           out->scales, out->scales_swz, out->tensor_scale, nkb);
  count_launch();
  if (cudaGetLastError() != cudaSuccess) return FP4_ERR_CUDA;
  return launch_pad(out->scales_swz, out->rows, ng, s);
}

int fp4_hadamard(const void* x, float* y, int64_t rows, int64_t cols, fp4_had had, uint64_t seed,
                 fp4_stream_t stream) {
  if (had.block != 16 && had.block != 32 && had.block != 64 && had.block != 128 && had.block != 256)
    return FP4_ERR_UNSUPPORTED;
  if (rows < 0 || cols < 0 || cols % had.block) return FP4_ERR_INVALID_ARG;
  if (rows == 0 || cols == 0) return FP4_OK;
  if (!x || !y) return FP4_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(y, 16)) return FP4_ERR_ALIGNMENT;
  QParams p{};
  p.x = x; p.rows = rows; p.cols = cols; p.seed = seed; p.sign_tag = had.sign_tag;
  p.randomized = had.randomized ? 1 : 0;
  int64_t tasks = rows * (cols / 8), blocks = (tasks + 255) / 256, cap = int64_t(num_sms()) * 8;
  if (blocks > cap) blocks = cap;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  switch (had.block) {
    case 16: k_hadamard<16><<<unsigned(blocks), 256, 0, s>>>(p, y); break;
    case 32: k_hadamard<32><<<unsigned(blocks), 256, 0, s>>>(p, y); break;
    case 64: k_hadamard<64><<<unsigned(blocks), 256, 0, s>>>(p, y); break;
    case 128: k_hadamard<128><<<unsigned(blocks), 256, 0, s>>>(p, y); break;
    default: k_hadamard<256><<<unsigned(blocks), 256, 0, s>>>(p, y); break;
  }
  count_launch();
  return cudaGetLastError() == cudaSuccess ? FP4_OK : FP4_ERR_CUDA;
}

int fp4_swizzle_scales(const uint8_t* scales, int64_t rows, int64_t n_groups, uint8_t* swz,
                       fp4_stream_t stream) {
  if (rows < 0 || n_groups < 0) return FP4_ERR_INVALID_ARG;
  if (rows == 0 || n_groups == 0) return FP4_OK;
  if (!scales || !swz) return FP4_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  int64_t nkb = (n_groups + 3) / 4, n = rows * n_groups, blocks = (n + 255) / 256;
  if (blocks > 4096) blocks = 4096;
  k_swizzle<<<unsigned(blocks), 256, 0, s>>>(scales, rows, n_groups, nkb, swz);
  count_launch();
  if (cudaGetLastError() != cudaSuccess) return FP4_ERR_CUDA;
  return launch_pad(swz, rows, n_groups, s);
}

int fp4_get_last_error(fp4_stream_t stream) {
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return FP4_ERR_CUDA;
  int* a = status_ptr();
  if (!a) return FP4_ERR_CUDA;
  int v = 0;
  if (cudaMemcpy(&v, a, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return FP4_ERR_CUDA;
  if (v) {
    int z = 0;
    cudaMemcpy(a, &z, sizeof(int), cudaMemcpyHostToDevice);
  }
  return v;
}

unsigned long long fp4_launch_count(void) { return g_launches.load(); }

int fp4_selftest_e2m1(unsigned long long* mismatches, fp4_stream_t stream) {
  if (!mismatches) return FP4_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  k_selftest_e2m1<<<unsigned(num_sms() * 8), 256, 0, s>>>(mismatches);
  count_launch();
  return cudaGetLastError() == cudaSuccess ? FP4_OK : FP4_ERR_CUDA;
}

int fp4_selftest_arith(unsigned long long* mismatches, fp4_stream_t stream) {
  if (!mismatches) return FP4_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  k_selftest_arith<<<unsigned(num_sms() * 8), 256, 0, s>>>(mismatches);
  count_launch();
  return cudaGetLastError() == cudaSuccess ? FP4_OK : FP4_ERR_CUDA;
}

const char* fp4_status_string(int st) {
  switch (st) {
    case FP4_OK: return "ok";
    case FP4_ERR_INVALID_ARG: return "invalid argument";
    case FP4_ERR_UNSUPPORTED: return "unsupported combination";
    case FP4_ERR_ALIGNMENT: return "misaligned pointer or dimension";
    case FP4_ERR_WORKSPACE: return "workspace missing or too small";
    case FP4_ERR_CUDA: return "CUDA error";
    case FP4_ERR_NONFINITE_INPUT: return "non-finite input";
    case FP4_ERR_TIMEOUT: return "device wait timed out";
    default: return "unknown status";
  }
}

}  // extern "C"

// ------------------------------------------------- allocation-free quantise --
// Scratch for fp4_quantize_noalloc: a fixed array in the library's own device
// memory (every GPU that loads the library holds it until the process exits).
// All calls share it, so two such calls that overlap on the GPU race on it.
static __device__ __align__(256) uint8_t g_noalloc_scratch[FP4_NOALLOC_SCRATCH_BYTES];

namespace fp4 {
// Device address of g_noalloc_scratch on the current device, looked up once per
// device (with that device current) on its first use; nullptr on failure.
static void* noalloc_scratch_ptr() {
  static std::mutex mu;
  static void* addr[64] = {nullptr};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> g(mu);
  if (!addr[dev]) {
    void* a = nullptr;
    if (cudaGetSymbolAddress(&a, g_noalloc_scratch) != cudaSuccess) return nullptr;
    addr[dev] = a;
  }
  return addr[dev];
}
}  // namespace fp4

extern "C" int fp4_quantize_noalloc(const void* x, int64_t in_rows, int64_t in_cols, int32_t transpose,
                                    int32_t fmt, int32_t rounding, int32_t group, fp4_had had, uint64_t seed,
                                    uint32_t tensor_tag, fp4_qtensor* out, fp4_stream_t stream) {
  // fp4_quantize's own argument checks first, so both calls give the same
  // status for the same arguments; then the size of the scratch.
  bool empty = false;
  const int st = quantize_args(x, in_rows, in_cols, transpose, fmt, rounding, group, had, out, &empty);
  if (st || empty) return st;
  const int64_t rows = out->rows, cols = out->cols;
  const size_t need = fp4_quantize_workspace_size(rows, cols, fmt, rounding, had.block);
  if (need > FP4_NOALLOC_SCRATCH_BYTES) return FP4_ERR_WORKSPACE;   // tensor too large for the array
  void* ws = nullptr;
  if (need > 0) {
    ws = noalloc_scratch_ptr();
    if (!ws) return FP4_ERR_CUDA;
  }
  // The same quantiser as fp4_quantize; the amax word it needs zeroed is
  // cleared on the stream inside (cudaMemsetAsync, no allocation).
  return fp4_quantize(x, in_rows, in_cols, transpose, fmt, rounding, group, had, seed, tensor_tag, out, ws,
                      need, stream);
}
