// Hadamard + quantise + pack kernels (sm_100a).
//
// One per-lane core, `process8`, quantises 8 consecutive elements of one row
// of the output tensor; the G/8 lanes of a scale group (and the HAD/8 lanes of
// a rotation block) are aligned neighbours in the warp, so group maxima,
// squared-error sums and the FWHT butterflies cross lanes with shuffles.
// Four loaders feed it: row-wise bf16, transposed bf16 (a 128 x 64 tile staged
// through shared memory), and the same two for a saved FP4 tensor that is
// de-quantised on the fly (the backward re-quantisation of the Quartet II
// computation graph).
#pragma once
#include <cfloat>
#include "device_common.cuh"

namespace fp4 {

enum : int { FMT_MX = 0, FMT_NV = 1 };
// R_AMAX: the global amax pass; R_SQ16: RTN against 16 x 16 block maxima.
enum : int { R_RTN = 0, R_QUEST = 1, R_FOS = 2, R_SR = 3, R_EDEN = 4, R_AMAX = 5, R_SQ16 = 6 };
// LD_ROW_F32: an fp32 matrix that is already transformed (row-wise, 32-element
// tasks only; fp4_quantize_f32).
enum : int { LD_ROW = 0, LD_TRANS = 1, LD_ROW_FP4 = 2, LD_TRANS_FP4 = 3, LD_ROW_F32 = 4 };

struct QParams {
  // input: bf16 matrix, or a saved FP4 tensor (codes + linear scales + scale)
  const void* x;
  const uint8_t* in_scales;
  const float* in_ts;
  int32_t in_fmt;
  int64_t in_rows, in_cols;
  // quantised (output) tensor, rows x cols, groups along cols
  int64_t rows, cols;
  uint8_t* codes;
  uint8_t* scales;
  uint8_t* swz;
  uint8_t* mask;
  float* ts;
  int64_t nkb;
  // randomness
  uint64_t seed;
  uint32_t tensor_tag;
  uint32_t sign_tag;
  int32_t randomized;
  // 16 x 16 block maxima (fp32 bits) of the input, row-major with ld
  // columns; trans: the quantised tensor is the input's transpose
  const uint32_t* bmax;
  int64_t bmax_ld;
  int32_t bmax_trans;
  // workspace
  uint32_t* amax_bits;
  uint16_t* pseudo;
  float* eden_S;
  int* status;
};

// Divisors and constants (fp32, each rounded once from the exact value).
#define FP4_NV_RTN_DIV 1536.0f                                  // 6 * 256
#define FP4_NV_SR_DIV ((float)(6.0 * 16.0 / 17.0 * 448.0))       // 6 * 16/17 * 448
#define FP4_NV_SR_GDIV ((float)(6.0 * 16.0 / 17.0))              // 6 * 16/17
#define FP4_EDEN_S 6.0f                                          // MS-EDEN clip factor s
#define FP4_QUARTET_PRESCALE 0.75f
#define FP4_QUARTET_TS ((float)(4.0 / 3.0))

__device__ __forceinline__ int64_t swz_offset(int64_t r, int64_t k, int64_t nkb) {
  return ((r >> 7) * nkb + (k >> 2)) * 512 + (r & 31) * 16 + ((r >> 5) & 3) * 4 + (k & 3);
}

__device__ __forceinline__ float nv_tensor_scale(uint32_t amax_bits, float div) {
  float s = __fdiv_rn(bitsf(amax_bits), div);
  return s == 0.0f ? 1.0f : s;
}

// MS-EDEN power-of-two tensor scale: 2^ceil(log2(amax / 1536)), >= 2^-126.
__device__ __forceinline__ float eden_tensor_scale(uint32_t amax_bits) {
  float q = __fdiv_rn(bitsf(amax_bits), FP4_NV_RTN_DIV);
  if (q == 0.0f) return 1.0f;
  uint32_t b = fbits(q), man = b & 0x7FFFFFu;
  bool pow2 = (b >> 23) != 0u ? man == 0u : __popc(man) == 1;
  int k = floor_log2(q) + (pow2 ? 0 : 1);
  return pow2f(k < -126 ? -126 : k);
}

__device__ __forceinline__ bool finite_pos(float d, float inv) {
  return d > 0.0f && absbits(inv) < 0x7F800000u;
}

template <int GL>
__device__ __forceinline__ uint32_t group_mask(int lane) {
  return GL >= 32 ? 0xFFFFFFFFu : (((1u << GL) - 1u) << (lane & ~(GL - 1)));
}

template <int GL>
__device__ __forceinline__ float tree_lanes_m(float v, uint32_t m) {
#pragma unroll
  for (int o = 1; o < GL; o <<= 1) v = __fadd_rn(v, __shfl_xor_sync(m, v, o));
  return v;
}

// Squared error sum over a group of fp32((x - fp32(q * d))^2), fixed tree.
template <int GL>
__device__ __forceinline__ float group_sse(const float* x, const uint32_t* c, float d, uint32_t m) {
  float s[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    float e = __fsub_rn(x[j], __fmul_rn(e2m1_value(c[j]), d));
    s[j] = __fmul_rn(e, e);
  }
  return tree_lanes_m<GL>(tree8(s), m);
}

__device__ __forceinline__ void encode_rtn8(const float* x, float inv, bool ok, uint32_t* c) {
#pragma unroll
  for (int j = 0; j < 8; ++j) c[j] = ok ? e2m1_rtn(__fmul_rn(x[j], inv)) : 0u;
}

struct Shared {
  uint32_t signs[8];   // RHT sign bits of one rotation block (<= 256)
  uint32_t red[32];    // block reductions
};

// ------------------------------------------------------------------ core --
// x: the 8 input values (before rotation) of output row orow, columns
// ocol..ocol+7.  All 32 lanes of the warp call it together (inactive lanes
// with zeros).  Returns this lane's max |y| bits (for amax accumulation).
template <int FMT, int RND, int HAD>
__device__ __forceinline__ uint32_t process8(float* x, bool active, int64_t orow, int64_t ocol,
                                             int lane, const QParams& p, const Shared& sh,
                                             uint32_t amax_in) {
  constexpr int G = FMT == FMT_NV ? 16 : 32;
  constexpr int GL = G / 8;
  if (HAD > 0) {
    uint32_t sign = 0;
    if (p.randomized) {
      int pos = int(ocol & (HAD - 1));
      sign = (sh.signs[pos >> 5] >> (pos & 31)) & 0xFFu;
    }
    fwht8_lanes<HAD>(x, sign, lane);
  }
  uint32_t lmax = 0;
#pragma unroll
  for (int j = 0; j < 8; ++j) lmax = max(lmax, absbits(x[j]));
  if (!active) lmax = 0;
  if (RND == R_AMAX) return lmax;

  const uint32_t gm = group_mask<GL>(lane);
  const uint32_t gmaxb = max_lanes<GL>(lmax);
  const float gmax = bitsf(gmaxb);
  if (active && gmaxb >= 0x7F800000u && FMT == FMT_MX) flag_status(p.status, ST_NONFINITE);
  if (active && RND == R_EDEN && gmaxb >= 0x7F800000u) flag_status(p.status, ST_NONFINITE);

  uint32_t c[8];
  uint32_t sbyte = 0, mbits = 0;

  if (FMT == FMT_NV && RND == R_RTN) {
    float s32 = nv_tensor_scale(amax_in, FP4_NV_RTN_DIV);
    uint32_t s8 = e4m3_rtn(__fdiv_rn(gmax, __fmul_rn(s32, 6.0f)));
    float d = __fmul_rn(e4m3_value(s8), s32), inv = __frcp_rn(d);
    encode_rtn8(x, inv, finite_pos(d, inv), c);
    sbyte = s8;
  } else if (FMT == FMT_NV && RND == R_FOS) {
    float s32 = nv_tensor_scale(amax_in, FP4_NV_RTN_DIV);
    uint32_t s6 = e4m3_rtn(__fdiv_rn(gmax, __fmul_rn(s32, 6.0f)));
    uint32_t s4 = e4m3_rtn(__fdiv_rn(gmax, __fmul_rn(s32, 4.0f)));
    float d6 = __fmul_rn(e4m3_value(s6), s32), i6 = __frcp_rn(d6);
    float d4 = __fmul_rn(e4m3_value(s4), s32), i4 = __frcp_rn(d4);
    uint32_t c4[8];
    encode_rtn8(x, i6, finite_pos(d6, i6), c);
    encode_rtn8(x, i4, finite_pos(d4, i4), c4);
    float e6 = group_sse<GL>(x, c, d6, gm);
    float e4 = group_sse<GL>(x, c4, d4, gm);
    bool pick4 = e4 < e6;
#pragma unroll
    for (int j = 0; j < 8; ++j) c[j] = pick4 ? c4[j] : c[j];
    sbyte = pick4 ? s4 : s6;
  } else if (FMT == FMT_NV && RND == R_SR) {
    float s32 = nv_tensor_scale(amax_in, FP4_NV_SR_DIV);
    uint32_t s8 = e4m3_rtn(__fdiv_rn(gmax, __fmul_rn(s32, FP4_NV_SR_GDIV)));
    float d = __fmul_rn(e4m3_value(s8), s32), inv = __frcp_rn(d);
    bool ok = finite_pos(d, inv);
    int64_t idx = orow * p.cols + ocol;
    u32x4 r0 = philox_block(p.seed, uint64_t(idx) >> 2, TAG_SR_ELEM, p.tensor_tag);
    u32x4 r1 = philox_block(p.seed, (uint64_t(idx) >> 2) + 1, TAG_SR_ELEM, p.tensor_tag);
    uint32_t w[8] = {r0.x, r0.y, r0.z, r0.w, r1.x, r1.y, r1.z, r1.w};
#pragma unroll
    for (int j = 0; j < 8; ++j) c[j] = ok ? e2m1_sr(__fmul_rn(x[j], inv), u24(w[j])) : 0u;
    sbyte = s8;
  } else if (FMT == FMT_NV && RND == R_QUEST) {
    float s32 = nv_tensor_scale(amax_in, FP4_NV_RTN_DIV);
    float sq[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) sq[j] = __fmul_rn(x[j], x[j]);
    float sig2 = __fdiv_rn(tree_lanes_m<GL>(tree8(sq), gm), 16.0f);
    float hi = __fmul_rn(25.0f, sig2);
    // T2(c) = (6 * fp32(val_c * s32))^2 is non-decreasing in c, so the window
    // sig2 <= T2 <= hi is a run of codes [clo, chi]
    auto t2 = [&](int cc) {
      float t = __fmul_rn(6.0f, __fmul_rn(e4m3_value(uint32_t(cc)), s32));
      return __fmul_rn(t, t);
    };
    int lo = 1, hi_i = 127;             // first code with t2 >= sig2 (127: none)
    while (lo < hi_i) { int mid = (lo + hi_i) >> 1; if (t2(mid) >= sig2) hi_i = mid; else lo = mid + 1; }
    int clo = lo;
    lo = 0; hi_i = 126;                  // last code with t2 <= hi (0: none)
    while (lo < hi_i) { int mid = (lo + hi_i + 1) >> 1; if (t2(mid) <= hi) lo = mid; else hi_i = mid - 1; }
    int chi = lo;
    uint32_t s8;
    if (clo <= chi && chi >= 1) {
      float best = __int_as_float(0x7F800000);
      int bc = clo;
      for (int cc = clo; cc <= chi; ++cc) {   // identical bounds in the group's lanes
        float d = __fmul_rn(e4m3_value(uint32_t(cc)), s32), inv = __frcp_rn(d);
        uint32_t ct[8];
        encode_rtn8(x, inv, finite_pos(d, inv), ct);
        float e = group_sse<GL>(x, ct, d, gm);
        if (e <= best) { best = e; bc = cc; }
      }
      s8 = uint32_t(bc);
    } else {
      s8 = e4m3_rtn(__fdiv_rn(gmax, __fmul_rn(s32, 6.0f)));
    }
    float d = __fmul_rn(e4m3_value(s8), s32), inv = __frcp_rn(d);
    bool ok = finite_pos(d, inv);
    encode_rtn8(x, inv, ok, c);
#pragma unroll
    for (int j = 0; j < 8; ++j) mbits |= uint32_t(ok && fabsf(__fmul_rn(x[j], inv)) > 6.0f) << j;
    sbyte = s8;
  } else if (FMT == FMT_NV && RND == R_EDEN) {
    float pq = e8m3_round(__fdiv_rn(gmax, FP4_EDEN_S));
    float inv = __frcp_rn(pq);
    encode_rtn8(x, inv, finite_pos(pq, inv), c);
    float yy[8], yq[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      yy[j] = __fmul_rn(x[j], x[j]);
      yq[j] = __fmul_rn(x[j], __fmul_rn(e2m1_value(c[j]), pq));
    }
    float num = tree_lanes<HAD / 8>(tree8(yy));
    float den = tree_lanes<HAD / 8>(tree8(yq));
    float S = den > 0.0f ? __fdiv_rn(num, den) : 1.0f;
    if (active) {
      if ((lane & (GL - 1)) == 0)
        p.pseudo[orow * (p.cols >> 4) + (ocol >> 4)] = uint16_t(fbits(pq) >> 16);
      if ((lane & (HAD / 8 - 1)) == 0) p.eden_S[orow * (p.cols / HAD) + ocol / HAD] = S;
    }
  } else if (FMT == FMT_MX && (RND == R_RTN || RND == R_SR)) {
    int e = int(gmaxb >> 23) - 129;
    e = e < -127 ? -127 : e;
    float sc = pow2f(-e);
    if (RND == R_RTN) {
#pragma unroll
      for (int j = 0; j < 8; ++j) c[j] = e2m1_rtn(__fmul_rn(x[j], sc));
    } else {
      int64_t idx = orow * p.cols + ocol;
      u32x4 r0 = philox_block(p.seed, uint64_t(idx) >> 2, TAG_SR_ELEM, p.tensor_tag);
      u32x4 r1 = philox_block(p.seed, (uint64_t(idx) >> 2) + 1, TAG_SR_ELEM, p.tensor_tag);
      uint32_t w[8] = {r0.x, r0.y, r0.z, r0.w, r1.x, r1.y, r1.z, r1.w};
#pragma unroll
      for (int j = 0; j < 8; ++j)
        c[j] = e2m1_sr(__fmul_rn(__fmul_rn(x[j], FP4_QUARTET_PRESCALE), sc), u24(w[j]));
    }
    sbyte = uint32_t(e + 127);
  } else if (FMT == FMT_MX && RND == R_QUEST) {
    float sq[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) sq[j] = __fmul_rn(x[j], x[j]);
    float sig2 = __fdiv_rn(tree_lanes<GL>(tree8(sq)), 32.0f);
    float hi = __fmul_rn(25.0f, sig2);
    int fl = sig2 > 0.0f ? floor_log2(sig2) : -300;
    int elo = (fl >> 1) - 4;
    int be = 0;
    float bs = __int_as_float(0x7F800000);
    bool found = false;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      int e = elo + k;
      e = e < -127 ? -127 : (e > 125 ? 125 : e);
      float t = __fmul_rn(6.0f, pow2f(e));
      float tt = __fmul_rn(t, t);
      bool inwin = (sig2 <= tt) && (tt <= hi) && (sig2 > 0.0f);
      float sc = pow2f(-e), d = pow2f(e);
      uint32_t ct[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) ct[j] = e2m1_rtn(__fmul_rn(x[j], sc));
      float s = group_sse<GL>(x, ct, d, 0xFFFFFFFFu);
      if (inwin && s <= bs) { bs = s; be = e; }
      found |= inwin;
    }
    int e;
    if (found) {
      e = be;
    } else {
      e = int(gmaxb >> 23) - 129;
      e = e < -127 ? -127 : e;
    }
    float sc = pow2f(-e);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      float v = __fmul_rn(x[j], sc);
      c[j] = e2m1_rtn(v);
      mbits |= uint32_t(fabsf(v) > 6.0f) << j;
    }
    sbyte = uint32_t(e + 127);
  }

  if (active) {
    uint32_t word = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) word |= (c[j] & 15u) << (4 * j);
    *reinterpret_cast<uint32_t*>(p.codes + orow * (p.cols >> 1) + (ocol >> 1)) = word;
    if (RND != R_EDEN && (lane & (GL - 1)) == 0) {
      int64_t k = ocol / G;
      if (p.scales) p.scales[orow * (p.cols / G) + k] = uint8_t(sbyte);
      if (p.swz) p.swz[swz_offset(orow, k, p.nkb)] = uint8_t(sbyte);
    }
    if (RND == R_QUEST && p.mask) p.mask[orow * (p.cols >> 3) + (ocol >> 3)] = uint8_t(mbits);
  }
  return lmax;
}

// Fill the random sign bits of one rotation block into shared memory.
template <int HAD>
__device__ __forceinline__ void load_signs(Shared& sh, const QParams& p) {
  if (threadIdx.x < 8) sh.signs[threadIdx.x] = 0;
  __syncthreads();
  if (HAD > 0 && p.randomized && threadIdx.x < HAD / 4) {
    u32x4 b = philox_block(p.seed, threadIdx.x, TAG_RHT_SIGN, p.sign_tag);
    uint32_t bits = (b.x >> 31) | ((b.y >> 31) << 1) | ((b.z >> 31) << 2) | ((b.w >> 31) << 3);
    int pos = 4 * threadIdx.x;
    atomicOr(&sh.signs[pos >> 5], bits << (pos & 31));
  }
  __syncthreads();
}

// Block-wide max of lane values, one atomicMax per block into `dst`.
__device__ __forceinline__ void block_max_atomic(uint32_t v, Shared& sh, uint32_t* dst, int* st) {
  v = __reduce_max_sync(0xFFFFFFFFu, v);
  int w = threadIdx.x >> 5, nw = blockDim.x >> 5;
  if ((threadIdx.x & 31) == 0) sh.red[w] = v;
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t m = 0;
    for (int i = 0; i < nw; ++i) m = max(m, sh.red[i]);
    if (m >= 0x7F800000u) flag_status(st, ST_NONFINITE);
    atomicMax(dst, m);
  }
}

// Tensor scale of the quantised tensor (MS-EDEN writes its own in pass 2).
template <int FMT, int RND>
__device__ __forceinline__ void write_tensor_scale(const QParams& p, uint32_t amax_in) {
  if (RND == R_AMAX || RND == R_EDEN) return;
  if (FMT == FMT_MX) *p.ts = RND == R_SR ? FP4_QUARTET_TS : 1.0f;
  else *p.ts = nv_tensor_scale(amax_in, RND == R_SR ? FP4_NV_SR_DIV : FP4_NV_RTN_DIV);
}

__device__ __forceinline__ float fp4_in_scale(uint32_t s, int fmt) {
  return fmt == FMT_NV ? e4m3_value(s) : pow2f(int(s) - 127);
}

// ------------------------------------------------------------- kernels --
// Row-wise: the output tensor is the input (bf16 or saved FP4), grid-stride
// over 8-element tasks, 32 consecutive tasks per warp.
template <int LOAD, int FMT, int RND, int HAD>
__global__ void __launch_bounds__(256) k_quant_row(QParams p) {
  __shared__ Shared sh;
  load_signs<HAD>(sh, p);
  const int lane = threadIdx.x & 31;
  const int64_t tasks = p.rows * (p.cols >> 3);
  const int64_t tpr = p.cols >> 3;
  const uint32_t amax_in = (FMT == FMT_NV && RND != R_EDEN && RND != R_AMAX) ? *p.amax_bits : 0u;
  const float in_ts = LOAD == LD_ROW_FP4 ? *p.in_ts : 1.0f;
  if (blockIdx.x == 0 && threadIdx.x == 0) write_tensor_scale<FMT, RND>(p, amax_in);
  uint32_t acc = 0;
  const int64_t wstride = int64_t(gridDim.x) * (blockDim.x >> 5) * 32;
  for (int64_t base = (int64_t(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5)) * 32;
       base < tasks; base += wstride) {
    int64_t t = base + lane;
    bool active = t < tasks;
    int64_t orow = active ? t / tpr : 0, ocol = active ? (t % tpr) * 8 : 0;
    float x[8];
    if (LOAD == LD_ROW) {
      uint4 v = make_uint4(0, 0, 0, 0);
      if (active)
        v = __ldg(reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(p.x) + orow * p.cols + ocol));
      bf16x8_to_f32(v, x);
    } else {
      uint32_t cw = 0, sc = 0;
      if (active) {
        cw = __ldg(reinterpret_cast<const uint32_t*>(static_cast<const uint8_t*>(p.x) + orow * (p.cols >> 1) + (ocol >> 1)));
        const int gsh = p.in_fmt == FMT_NV ? 4 : 5;   // log2 of the input group size
        sc = p.in_scales[orow * (p.cols >> gsh) + (ocol >> gsh)];
      }
      float s = fp4_in_scale(sc, p.in_fmt);
#pragma unroll
      for (int j = 0; j < 8; ++j) x[j] = __fmul_rn(__fmul_rn(e2m1_value((cw >> (4 * j)) & 15u), s), in_ts);
    }
    acc = max(acc, process8<FMT, RND, HAD>(x, active, orow, ocol, lane, p, sh, amax_in));
  }
  if (RND == R_AMAX || RND == R_EDEN) block_max_atomic(acc, sh, p.amax_bits, p.status);
}

// Transposed: the output tensor is the input's transpose.  One CTA stages a
// 128 (input rows = output cols) x 64 (input cols = output rows) tile as fp32
// in shared memory, then quantises 64 output rows x 128 output columns.
constexpr int TR_IN_ROWS = 128, TR_IN_COLS = 64, TR_PITCH = 132;

template <int LOAD, int FMT, int RND, int HAD>
__global__ void __launch_bounds__(256) k_quant_trans(QParams p) {
  __shared__ Shared sh;
  __shared__ __align__(16) float tile[TR_IN_COLS][TR_PITCH];
  load_signs<HAD>(sh, p);
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int64_t r0 = int64_t(blockIdx.x) * TR_IN_ROWS, c0 = int64_t(blockIdx.y) * TR_IN_COLS;
  const int64_t R = p.in_rows, C = p.in_cols;
  {
    const int rh = w >> 2, cb = w & 3;
    const int rl = 64 * rh + 2 * lane;
    const int64_t cc = c0 + 16 * cb;
    float va[16], vb[16];
    if (LOAD == LD_TRANS) {
      const uint16_t* xb = static_cast<const uint16_t*>(p.x);
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint4 a = make_uint4(0, 0, 0, 0), b = make_uint4(0, 0, 0, 0);
        int64_t col = cc + 8 * h;
        if (col < C) {
          if (r0 + rl < R) a = __ldg(reinterpret_cast<const uint4*>(xb + (r0 + rl) * C + col));
          if (r0 + rl + 1 < R) b = __ldg(reinterpret_cast<const uint4*>(xb + (r0 + rl + 1) * C + col));
        }
        bf16x8_to_f32(a, va + 8 * h);
        bf16x8_to_f32(b, vb + 8 * h);
      }
    } else {
      const uint8_t* xc = static_cast<const uint8_t*>(p.x);
      const float in_ts = *p.in_ts;
      const int gsh = p.in_fmt == FMT_NV ? 4 : 5;   // log2 of the input group size
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        int64_t r = r0 + rl + q;
        uint2 cw = make_uint2(0, 0);
        uint32_t sa = 0, sb = 0;
        if (r < R && cc < C) {
          cw = __ldg(reinterpret_cast<const uint2*>(xc + r * (C >> 1) + (cc >> 1)));
          sa = p.in_scales[r * (C >> gsh) + (cc >> gsh)];
          sb = p.in_scales[r * (C >> gsh) + ((cc + 8) >> gsh)];
        }
        float s_a = fp4_in_scale(sa, p.in_fmt), s_b = fp4_in_scale(sb, p.in_fmt);
        float* dst = q ? vb : va;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          uint32_t code = ((j < 8 ? cw.x : cw.y) >> (4 * (j & 7))) & 15u;
          dst[j] = __fmul_rn(__fmul_rn(e2m1_value(code), j < 8 ? s_a : s_b), in_ts);
        }
      }
    }
#pragma unroll
    for (int j = 0; j < 16; ++j)
      *reinterpret_cast<float2*>(&tile[16 * cb + j][rl]) = make_float2(va[j], vb[j]);
  }
  __syncthreads();
  const uint32_t amax_in = (FMT == FMT_NV && RND != R_EDEN && RND != R_AMAX) ? *p.amax_bits : 0u;
  if (blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0) write_tensor_scale<FMT, RND>(p, amax_in);
  uint32_t acc = 0;
#pragma unroll 1
  for (int s = 0; s < 4; ++s) {
    const int orl = s * 16 + w * 2 + (lane >> 4), ocl = (lane & 15) * 8;
    const int64_t orow = c0 + orl, ocol = r0 + ocl;
    const bool active = orow < C && ocol < R;
    float x[8];
    float4 a = *reinterpret_cast<const float4*>(&tile[orl][ocl]);
    float4 b = *reinterpret_cast<const float4*>(&tile[orl][ocl + 4]);
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
    x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
    acc = max(acc, process8<FMT, RND, HAD>(x, active, active ? orow : 0, active ? ocol : 0, lane, p, sh, amax_in));
  }
  if (RND == R_AMAX || RND == R_EDEN) block_max_atomic(acc, sh, p.amax_bits, p.status);
}

// MS-EDEN second kernel: shift the pseudo-scales by the power-of-two tensor
// scale, multiply by the EDEN factor of their rotation block, stochastic
// rounding onto E4M3 (codes are untouched).
template <int HAD>
__global__ void __launch_bounds__(256) k_eden_pass2(QParams p) {
  const int64_t ng = p.cols >> 4, total = p.rows * ng;
  const float s32 = eden_tensor_scale(*p.amax_bits);
  const float inv32 = __frcp_rn(s32);
  const int64_t ns = p.cols / HAD;                 // EDEN factors per row
  if (blockIdx.x == 0 && threadIdx.x == 0) *p.ts = s32;
  if ((ng & 3) == 0) {
    // four groups k0..k0+3 of one row per thread: one Philox block, 4-byte
    // stores; the (row, group) of each task advances by the grid stride
    const int64_t nq = ng >> 2, stride = int64_t(gridDim.x) * blockDim.x;
    const int64_t q0 = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
    int64_t r = q0 / nq, kq = q0 % nq;
    const int64_t dr = stride / nq, dk = stride % nq;
    for (int64_t q = q0; q < (total >> 2); q += stride) {
      const int64_t k0 = kq << 2, gi0 = q << 2;
      const uint2 ps = *reinterpret_cast<const uint2*>(p.pseudo + gi0);
      const uint32_t pw[4] = {ps.x << 16, ps.x & 0xFFFF0000u, ps.y << 16, ps.y & 0xFFFF0000u};
      const u32x4 rb = philox_block(p.seed, uint64_t(q), TAG_SR_SCALE, p.tensor_tag);
      const uint32_t rw[4] = {rb.x, rb.y, rb.z, rb.w};
      const float* Srow = p.eden_S + r * ns + (k0 * 16) / HAD;
      uint32_t word = 0;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float S = Srow[(j * 16) / HAD];        // one factor per HAD / 16 groups
        const float t = __fmul_rn(__fmul_rn(S, bitsf(pw[j])), inv32);
        word |= e4m3_sr_bits(t, rw[j] >> 8) << (8 * j);
      }
      if (p.scales) *reinterpret_cast<uint32_t*>(p.scales + gi0) = word;
      if (p.swz) *reinterpret_cast<uint32_t*>(p.swz + swz_offset(r, k0, p.nkb)) = word;
      kq += dk;
      r += dr;
      if (kq >= nq) { kq -= nq; ++r; }
    }
    return;
  }
  for (int64_t gi = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; gi < total;
       gi += int64_t(gridDim.x) * blockDim.x) {
    int64_t r = gi / ng, k = gi % ng;
    float pq = bitsf(uint32_t(p.pseudo[gi]) << 16);
    float S = p.eden_S[r * ns + (k * 16) / HAD];
    float t = __fmul_rn(__fmul_rn(S, pq), inv32);
    uint32_t s8 = e4m3_sr_bits(t, philox_word(p.seed, uint64_t(gi), TAG_SR_SCALE, p.tensor_tag) >> 8);
    if (p.scales) p.scales[gi] = uint8_t(s8);
    if (p.swz) p.swz[swz_offset(r, k, p.nkb)] = uint8_t(s8);
  }
}

// Zero the padding of the swizzled scale layout: rows [rows, 128 * nrb) and
// groups [ng, 4 * nkb).
static __global__ void k_swz_pad(uint8_t* swz, int64_t rows, int64_t ng, int64_t nkb) {
  const int64_t nrb = (rows + 127) >> 7;
  const int64_t rows_pad = nrb * 128, ng_pad = nkb * 4;
  const int64_t n_rowpad = (rows_pad - rows) * ng_pad;       // whole padded rows
  const int64_t n_colpad = rows * (ng_pad - ng);             // padded groups of real rows
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n_rowpad + n_colpad;
       i += int64_t(gridDim.x) * blockDim.x) {
    int64_t r, k;
    if (i < n_rowpad) { r = rows + i / ng_pad; k = i % ng_pad; }
    else { int64_t j = i - n_rowpad; r = j / (ng_pad - ng); k = ng + j % (ng_pad - ng); }
    swz[swz_offset(r, k, nkb)] = 0;
  }
}

// Plain block (randomized) Hadamard to fp32.
template <int HAD>
__global__ void __launch_bounds__(256) k_hadamard(QParams p, float* y) {
  __shared__ Shared sh;
  load_signs<HAD>(sh, p);
  const int lane = threadIdx.x & 31;
  const int64_t tasks = p.rows * (p.cols >> 3), tpr = p.cols >> 3;
  const int64_t wstride = int64_t(gridDim.x) * (blockDim.x >> 5) * 32;
  for (int64_t base = (int64_t(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5)) * 32;
       base < tasks; base += wstride) {
    int64_t t = base + lane;
    bool active = t < tasks;
    int64_t orow = active ? t / tpr : 0, ocol = active ? (t % tpr) * 8 : 0;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (active) v = __ldg(reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(p.x) + orow * p.cols + ocol));
    float x[8];
    bf16x8_to_f32(v, x);
    uint32_t sign = 0;
    if (p.randomized) {
      int pos = int(ocol & (HAD - 1));
      sign = (sh.signs[pos >> 5] >> (pos & 31)) & 0xFFu;
    }
    fwht8_lanes<HAD>(x, sign, lane);
    if (active) {
      float4* dst = reinterpret_cast<float4*>(y + orow * p.cols + ocol);
      dst[0] = make_float4(x[0], x[1], x[2], x[3]);
      dst[1] = make_float4(x[4], x[5], x[6], x[7]);
    }
  }
}

}  // namespace fp4
