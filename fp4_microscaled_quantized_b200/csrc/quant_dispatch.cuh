// Host-side launch of the quantiser kernels for one loader (instantiated once
// per loader in quant_ld*.cu so the four compile in parallel).
#pragma once
#include <atomic>

#include "quant_core32.cuh"

namespace fp4 {

template <int LOAD>
cudaError_t launch_quant(int fmt, int rnd, int had, const QParams& p, cudaStream_t s);

int num_sms();

// Resident 256-thread blocks per SM of one row kernel (its registers and
// shared memory decide), cached per instantiation and device: grid-stride
// kernels launch exactly one full wave, so no block waits for a second wave
// and then runs alone at the end.
template <bool WIDE, int LOAD, int FMT, int RND, int HAD>
int resident_blocks() {
  static std::atomic<int> cached[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) dev = 0;
  int v = cached[dev].load(std::memory_order_relaxed);
  if (!v) {
    int n = 0;
    cudaError_t e;
    if constexpr (WIDE) e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, k_quant_row32<LOAD, FMT, RND, HAD>, 256, 0);
    else e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, k_quant_row<LOAD, FMT, RND, HAD>, 256, 0);
    v = (e == cudaSuccess && n >= 1) ? n : 1;
    cached[dev].store(v, std::memory_order_relaxed);   // every thread computes the same value
  }
  return v;
}

template <int LOAD, int FMT, int RND, int HAD>
cudaError_t launch_one(const QParams& p, cudaStream_t s) {
  constexpr bool TRANS = LOAD == LD_TRANS || LOAD == LD_TRANS_FP4;
  if constexpr (LOAD == LD_ROW_F32) {
    // an already transformed fp32 matrix: row-wise, 32-element tasks only
    if (HAD != 0 || (p.cols % 32) != 0) return cudaErrorInvalidValue;
    int64_t blocks = (p.rows * (p.cols >> 5) + 255) / 256;
    const int64_t cap = int64_t(num_sms()) * resident_blocks<true, LOAD, FMT, RND, HAD>();
    blocks = blocks > cap ? cap : (blocks < 1 ? 1 : blocks);
    k_quant_row32<LOAD, FMT, RND, HAD><<<dim3(unsigned(blocks)), 256, 0, s>>>(p);
    count_launch();
    return cudaGetLastError();
  } else if constexpr (RND == R_SQ16 && (HAD != 0 || LOAD == LD_ROW_FP4 || LOAD == LD_TRANS_FP4)) {
    // square blocks: bf16 input, no rotation
    return cudaErrorInvalidValue;
  } else {
    const bool wide = (p.cols % 32) == 0;   // 32 elements per lane (always so for blocks >= 32)
    if (!TRANS && wide) {
      int64_t tasks = p.rows * (p.cols >> 5);
      int64_t blocks = (tasks + 255) / 256;
      int64_t cap = int64_t(num_sms()) * resident_blocks<true, LOAD, FMT, RND, HAD>();
      if (blocks > cap) blocks = cap;
      if (blocks < 1) blocks = 1;
      k_quant_row32<LOAD, FMT, RND, HAD><<<dim3(unsigned(blocks)), 256, 0, s>>>(p);
      count_launch();
    } else if (wide) {
      using TT = T32Tile<HAD>;
      dim3 grid(unsigned((p.in_rows + TT::ROWS - 1) / TT::ROWS), unsigned((p.in_cols + TT::COLS - 1) / TT::COLS));
      k_quant_trans32<LOAD, FMT, RND, HAD><<<grid, TT::THREADS, 0, s>>>(p);
      count_launch();
    } else if constexpr (HAD <= 16 && RND != R_SQ16) {
      // inner dimension 16 mod 32: 8 elements per lane
      if (!TRANS) {
        int64_t tasks = p.rows * (p.cols >> 3);
        int64_t blocks = (tasks + 255) / 256;
        int64_t cap = int64_t(num_sms()) * resident_blocks<false, LOAD, FMT, RND, HAD>();
        if (blocks > cap) blocks = cap;
        if (blocks < 1) blocks = 1;
        k_quant_row<LOAD, FMT, RND, HAD><<<dim3(unsigned(blocks)), 256, 0, s>>>(p);
        count_launch();
      } else {
        dim3 grid(unsigned((p.in_rows + TR_IN_ROWS - 1) / TR_IN_ROWS),
                  unsigned((p.in_cols + TR_IN_COLS - 1) / TR_IN_COLS));
        k_quant_trans<LOAD, FMT, RND, HAD><<<grid, 256, 0, s>>>(p);
        count_launch();
      }
    } else {
      return cudaErrorInvalidValue;          // cols is a multiple of the block: unreachable
    }
    return cudaGetLastError();
  }
}

#define FP4_HAD_SWITCH(LOAD, FMT, RND)                                      \
  switch (had) {                                                            \
    case 0: return launch_one<LOAD, FMT, RND, 0>(p, s);                     \
    case 16: return launch_one<LOAD, FMT, RND, 16>(p, s);                   \
    case 32: return launch_one<LOAD, FMT, RND, 32>(p, s);                   \
    case 64: return launch_one<LOAD, FMT, RND, 64>(p, s);                   \
    case 128: return launch_one<LOAD, FMT, RND, 128>(p, s);                 \
    case 256: return launch_one<LOAD, FMT, RND, 256>(p, s);                 \
    default: return cudaErrorInvalidValue;                                  \
  }

#define FP4_HAD_SWITCH_ROT(LOAD, FMT, RND)                                  \
  switch (had) {                                                            \
    case 16: return launch_one<LOAD, FMT, RND, 16>(p, s);                   \
    case 32: return launch_one<LOAD, FMT, RND, 32>(p, s);                   \
    case 64: return launch_one<LOAD, FMT, RND, 64>(p, s);                   \
    case 128: return launch_one<LOAD, FMT, RND, 128>(p, s);                 \
    case 256: return launch_one<LOAD, FMT, RND, 256>(p, s);                 \
    default: return cudaErrorInvalidValue;                                  \
  }

#define FP4_DEFINE_LAUNCH_QUANT(LOAD)                                               \
  template <>                                                                       \
  cudaError_t launch_quant<LOAD>(int fmt, int rnd, int had, const QParams& p,       \
                                 cudaStream_t s) {                                  \
    if (rnd == R_AMAX) { FP4_HAD_SWITCH(LOAD, FMT_NV, R_AMAX) }                     \
    if (fmt == FMT_NV) {                                                            \
      switch (rnd) {                                                                \
        case R_RTN: { FP4_HAD_SWITCH(LOAD, FMT_NV, R_RTN) }                         \
        case R_QUEST: { FP4_HAD_SWITCH(LOAD, FMT_NV, R_QUEST) }                     \
        case R_FOS: { FP4_HAD_SWITCH(LOAD, FMT_NV, R_FOS) }                         \
        case R_SR: { FP4_HAD_SWITCH(LOAD, FMT_NV, R_SR) }                           \
        case R_EDEN: { FP4_HAD_SWITCH_ROT(LOAD, FMT_NV, R_EDEN) }                   \
        case R_SQ16: return launch_one<LOAD, FMT_NV, R_SQ16, 0>(p, s);              \
        default: return cudaErrorInvalidValue;                                      \
      }                                                                             \
    }                                                                               \
    switch (rnd) {                                                                  \
      case R_RTN: { FP4_HAD_SWITCH(LOAD, FMT_MX, R_RTN) }                           \
      case R_QUEST: { FP4_HAD_SWITCH(LOAD, FMT_MX, R_QUEST) }                       \
      case R_SR: { FP4_HAD_SWITCH(LOAD, FMT_MX, R_SR) }                             \
      default: return cudaErrorInvalidValue;                                        \
    }                                                                               \
  }

}  // namespace fp4
