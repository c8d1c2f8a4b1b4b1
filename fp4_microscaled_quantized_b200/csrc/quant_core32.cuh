// Fast path of the quantiser: 32 consecutive elements of one output row per
// lane (used when the inner dimension is a multiple of 32).  Scale groups (16
// or 32) and rotation blocks up to 32 live entirely in one lane's registers;
// a 128-block spans 4 aligned lanes, so the FWHT needs two shuffle stages and
// the MS-EDEN sums two.  Arithmetic is element-for-element the same as the
// 8-per-lane path in quant_kernels.cuh (same butterfly order, same pairwise
// trees), so both produce identical bits.
#pragma once
#include <cuda_fp16.h>
#include "quant_kernels.cuh"

namespace fp4 {

// Hardware E2M1 conversion (round to nearest even, saturating at +-6) of two
// values into bits 0-7 of the result (`lo` in bits 0-3, bits 8-31 zero).
// The conversion writes a one-byte register.  Bytes cross the asm boundary
// only inside a full 32-bit register whose other bytes are zero: one-byte
// operands taken from wider registers (a four-way split of a word, or the
// upper half of one) were read from the wrong byte in some kernels.
__device__ __forceinline__ uint32_t e2m1x2_rn(float lo, float hi) {
  uint32_t r;
  asm("{\n\t.reg .b8 t;\n\t.reg .b16 h;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 t, %2, %1;\n\t"
      "mov.b16 h, {t, 0};\n\t"
      "cvt.u32.u16 %0, h;\n\t}"
      : "=r"(r) : "f"(lo), "f"(hi));
  return r;
}

// f16x2 grid values of the two codes in bits 0-7 of `b` (bits 8-31 zero;
// bits 0-3 -> low half).
__device__ __forceinline__ uint32_t e2m1x2_to_f16x2(uint32_t b) {
  uint32_t h;
  asm("{\n\t.reg .b8 t, z;\n\t.reg .b16 lo, hi;\n\t"
      "mov.b32 {lo, hi}, %1;\n\t"
      "mov.b16 {t, z}, lo;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, t;\n\t}"
      : "=r"(h) : "r"(b));
  return h;
}

// E2M1 RTN of two values as in e2m1x2_rn, returning also their grid values
// as f16x2 (exact), decoded from the same one-byte code inside the asm block.
__device__ __forceinline__ uint32_t e2m1x2_rn_dec(float lo, float hi, uint32_t& h) {
  uint32_t r;
  asm("{\n\t.reg .b8 t;\n\t.reg .b16 s;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 t, %3, %2;\n\t"
      "cvt.rn.f16x2.e2m1x2 %1, t;\n\t"
      "mov.b16 s, {t, 0};\n\t"
      "cvt.u32.u16 %0, s;\n\t}"
      : "=r"(r), "=r"(h) : "f"(lo), "f"(hi));
  return r;
}

// Clear negative-zero codes (a value rounding to 0 is stored as +0).
__device__ __forceinline__ uint32_t clear_neg_zero(uint32_t w) {
  const uint32_t nz = ((w & 0x77777777u) + 0x77777777u) & 0x88888888u;  // bit 3 set iff mag != 0
  return w & (nz | 0x77777777u);
}

// E2M1 RTN of 8 values into one word (element j in bits 4j..4j+3) with the
// hardware conversion, negative zeros kept (they decode to -0, which changes
// no error or inner product); the four bytes are joined by byte permutes.
__device__ __forceinline__ uint32_t enc8_raw(const float* v) {
  const uint32_t lo = __byte_perm(e2m1x2_rn(v[0], v[1]), e2m1x2_rn(v[2], v[3]), 0x0040u);
  const uint32_t hi = __byte_perm(e2m1x2_rn(v[4], v[5]), e2m1x2_rn(v[6], v[7]), 0x0040u);
  return __byte_perm(lo, hi, 0x5410u);
}

// The stored form: negative zeros cleared so a value rounding to 0 encodes
// as +0.
__device__ __forceinline__ uint32_t enc8_hw(const float* v) { return clear_neg_zero(enc8_raw(v)); }

// Software reference of the same word (the per-element encoder).
__device__ __forceinline__ uint32_t enc8_sw(const float* v) {
  uint32_t w = 0;
#pragma unroll
  for (int j = 0; j < 8; ++j) w |= e2m1_rtn(v[j]) << (4 * j);
  return w;
}

__device__ __forceinline__ float tree16(const float* s) { return __fadd_rn(tree8(s), tree8(s + 8)); }
__device__ __forceinline__ float tree32(const float* s) { return __fadd_rn(tree16(s), tree16(s + 16)); }

// Packed fp32 pair arithmetic (two independent IEEE round-to-nearest results
// per instruction).  a - b is fma(b, -1, a): the product is exact, so it
// rounds exactly like the subtraction, signed zeros included.
__device__ __forceinline__ float2 ld2(const float* x, int i) { return make_float2(x[i], x[i + 1]); }
__device__ __forceinline__ void st2(float* x, int i, float2 v) { x[i] = v.x; x[i + 1] = v.y; }
__device__ __forceinline__ float2 sub2(float2 a, float2 b) { return __ffma2_rn(b, make_float2(-1.0f, -1.0f), a); }
__device__ __forceinline__ float2 splat2(float v) { return make_float2(v, v); }

// The same value as tree16 (level 0 adds (2i, 2i+1), then pairs of pairs),
// with the upper levels packed: level-0 sums are paired as (n_i, n_{i+4}), so
// levels 1 and 2 each add two tree nodes per instruction.
__device__ __forceinline__ float tree16p(const float* s) {
  const float2 a0 = make_float2(__fadd_rn(s[0], s[1]), __fadd_rn(s[8], s[9]));
  const float2 a1 = make_float2(__fadd_rn(s[2], s[3]), __fadd_rn(s[10], s[11]));
  const float2 a2 = make_float2(__fadd_rn(s[4], s[5]), __fadd_rn(s[12], s[13]));
  const float2 a3 = make_float2(__fadd_rn(s[6], s[7]), __fadd_rn(s[14], s[15]));
  const float2 c = __fadd2_rn(__fadd2_rn(a0, a1), __fadd2_rn(a2, a3));
  return __fadd_rn(c.x, c.y);
}

// Three-input maximum that propagates NaN (so a non-finite input is seen by
// the status check); on finite inputs it is the exact maximum.
__device__ __forceinline__ float max3n(float a, float b, float c) {
  float d;
  asm("max.NaN.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// Bits of max |x| over 16 consecutive values.  Absolute values are
// non-negative, so the float maximum and the maximum of the bit patterns
// agree.
__device__ __forceinline__ uint32_t absmax16(const float* x) {
  const float a0 = max3n(fabsf(x[0]), fabsf(x[1]), fabsf(x[2]));
  const float a1 = max3n(fabsf(x[3]), fabsf(x[4]), fabsf(x[5]));
  const float a2 = max3n(fabsf(x[6]), fabsf(x[7]), fabsf(x[8]));
  const float a3 = max3n(fabsf(x[9]), fabsf(x[10]), fabsf(x[11]));
  const float a4 = max3n(fabsf(x[12]), fabsf(x[13]), fabsf(x[14]));
  const float b0 = max3n(a0, a1, a2), b1 = max3n(a3, a4, fabsf(x[15]));
  float r;
  asm("max.NaN.f32 %0, %1, %2;" : "=f"(r) : "f"(b0), "f"(b1));
  return fbits(r);
}

// 16 codes of x * inv (or zeros when !ok) into two words, negative zeros
// kept (enc16_raw) or cleared (enc16).
__device__ __forceinline__ void enc16_raw(const float* x, float inv, bool ok, uint32_t* w) {
  float v[16];
#pragma unroll
  for (int j = 0; j < 16; j += 2) st2(v, j, __fmul2_rn(ld2(x, j), splat2(inv)));
  w[0] = ok ? enc8_raw(v) : 0u;
  w[1] = ok ? enc8_raw(v + 8) : 0u;
}
__device__ __forceinline__ void enc16(const float* x, float inv, bool ok, uint32_t* w) {
  enc16_raw(x, inv, ok, w);
  w[0] = clear_neg_zero(w[0]);
  w[1] = clear_neg_zero(w[1]);
}

// enc8_raw of v together with the signed grid values q of the 8 codes
// (code 8 gives -0), without unpacking the word again.
__device__ __forceinline__ uint32_t enc8_dec(const float* v, float* q) {
  uint32_t b[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    uint32_t h;
    b[k] = e2m1x2_rn_dec(v[2 * k], v[2 * k + 1], h);
    const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&h));
    q[2 * k] = f.x;
    q[2 * k + 1] = f.y;
  }
  const uint32_t lo = __byte_perm(b[0], b[1], 0x0040u);
  const uint32_t hi = __byte_perm(b[2], b[3], 0x0040u);
  return __byte_perm(lo, hi, 0x5410u);
}

// enc16_raw with the grid values of the 16 codes (all zero when !ok).
__device__ __forceinline__ void enc16_dec(const float* x, float inv, bool ok, uint32_t* w, float* q) {
  float v[16];
#pragma unroll
  for (int j = 0; j < 16; j += 2) st2(v, j, __fmul2_rn(ld2(x, j), splat2(inv)));
  w[0] = enc8_dec(v, q);
  w[1] = enc8_dec(v + 8, q + 8);
  if (!ok) {
    w[0] = w[1] = 0u;
#pragma unroll
    for (int j = 0; j < 16; ++j) q[j] = 0.0f;
  }
}

// fp32 squared error of 16 elements against grid values q times d, pairwise
// tree: e = x - fp32(q d), s = fp32(e e).  The subtraction is a scalar IEEE
// operation: a packed subtraction of a packed product can be fused into one
// multiply-add by the code generator, which changes the rounding.
__device__ __forceinline__ float sse16q(const float* x, const float* q, float d) {
  float s[16];
#pragma unroll
  for (int j = 0; j < 16; j += 2) {
    const float2 qd = __fmul2_rn(ld2(q, j), splat2(d));
    const float2 e = make_float2(__fsub_rn(x[j], qd.x), __fsub_rn(x[j + 1], qd.y));
    st2(s, j, __fmul2_rn(e, e));
  }
  return tree16p(s);
}

// Signed grid values of the 8 codes of a word (element j from bits 4j..4j+3):
// the packed E2M1 -> f16x2 conversion of each byte, then f16 -> f32, both
// exact.  Code 8 gives -0.
__device__ __forceinline__ void dec8(uint32_t w, float* q) {
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const uint32_t h = e2m1x2_to_f16x2((w >> (8 * k)) & 0xFFu);
    const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&h));
    q[2 * k] = f.x;
    q[2 * k + 1] = f.y;
  }
}

// Per-lane XOR masks that apply the randomized-Hadamard signs to loaded data
// before it is unpacked: for bf16 pairs (sign bits 15 and 31 of each 32-bit
// word of two elements) and for FP4 codes (bit 3 of each nibble).  `sw` holds
// the sign bits of the lane's 32 consecutive positions.
__device__ __forceinline__ void sign_masks_bf16(uint32_t sw, uint32_t* m16) {
#pragma unroll
  for (int i = 0; i < 16; ++i) m16[i] = (((sw >> (2 * i)) & 1u) << 15) | (((sw >> (2 * i + 1)) & 1u) << 31);
}
__device__ __forceinline__ void sign_masks_fp4(uint32_t sw, uint32_t* m4) {
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    uint32_t m = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) m |= ((sw >> (8 * k + j)) & 1u) << (4 * j + 3);
    m4[k] = m;
  }
}

// Sign bits of the 32 consecutive positions starting at `pos` of a rotation
// block (pos is a multiple of 32, or 0 for 16-blocks whose pattern repeats).
template <int HAD>
__device__ __forceinline__ uint32_t lane_signs(const Shared& sh, const QParams& p, int pos) {
  if (HAD == 0 || !p.randomized) return 0u;
  if (HAD == 16) return (sh.signs[0] & 0xFFFFu) | (sh.signs[0] << 16);
  return sh.signs[(pos & (HAD - 1)) >> 5];
}

// Block FWHT over HAD consecutive elements, 32 per lane (HAD / 32 aligned
// lanes for HAD = 64, 128, 256), same butterfly order as fwht8_lanes.  The random
// signs are applied by the loaders (to the bf16 bits or the FP4 codes).  The
// h = 1 stage works inside the natural pairs (2i, 2i+1); every later stage,
// the cross-lane ones (x + o on the lower lane, o - x on the upper: one
// fma(+-1, x, o)) and the final scaling run two elements per instruction.
template <int HAD>
__device__ __forceinline__ void fwht32_lanes(float* x, int lane) {
  constexpr int HIN = HAD < 32 ? HAD : 32;
#pragma unroll
  for (int i = 0; i < 32; i += 2) {
    const float a = x[i], b = x[i + 1];
    x[i] = __fadd_rn(a, b);
    x[i + 1] = __fsub_rn(a, b);
  }
#pragma unroll
  for (int h = 2; h < HIN; h <<= 1) {
#pragma unroll
    for (int i = 0; i < 32; i += 2) {
      if (i & h) continue;
      const float2 a = ld2(x, i), b = ld2(x, i + h);
      st2(x, i, __fadd2_rn(a, b));
      st2(x, i + h, sub2(a, b));
    }
  }
#pragma unroll
  for (int hl = 1; hl < HAD / 32; hl <<= 1) {
    const float2 sgn = splat2((lane & hl) ? -1.0f : 1.0f);
#pragma unroll
    for (int i = 0; i < 32; i += 2) {
      const float2 o = make_float2(__shfl_xor_sync(0xFFFFFFFFu, x[i], hl), __shfl_xor_sync(0xFFFFFFFFu, x[i + 1], hl));
      st2(x, i, __ffma2_rn(sgn, ld2(x, i), o));
    }
  }
  const float c = hadamard_scale<HAD>();
#pragma unroll
  for (int j = 0; j < 32; j += 2) st2(x, j, __fmul2_rn(ld2(x, j), splat2(c)));
}

// e8m3_round(fp32(g / 6)) for g >= 0 or NaN.  The product with fp32(1/6)
// (relative error 2^-25) lies within 1.5 ulp of g / 6, so its bit pattern is
// within one of the correctly rounded quotient's and the E8M3 rounding of
// the two differs only when the product's low 20 bits lie within two of the
// rounding midpoint 0x80000; only then is the quotient divided exactly.
__device__ __forceinline__ float e8m3_div6(float g) {
  const float q = __fmul_rn(g, 0.166666672f);
  if (((fbits(q) + 2u - 0x80000u) & 0xFFFFFu) <= 4u) return e8m3_round(__fdiv_rn(g, 6.0f));
  return e8m3_round(q);
}

// Per-tensor constants of the NVFP4 scale rules, computed once per thread:
// the tensor scale and the divisions of the group maximum by the largest
// normalised value times it.
struct QuantConsts {
  float s32;
  ExactDiv d6;   // by fp32(6 s32) (RTN, 4/6, QuEST), fp32(6 16/17 s32) (SR), 6 (MS-EDEN)
  ExactDiv d4;   // by fp32(4 s32) (4/6)
};

template <int FMT, int RND>
__device__ __forceinline__ QuantConsts quant_consts(uint32_t amax_in) {
  QuantConsts c{};
  if (FMT != FMT_NV || RND == R_AMAX) return c;
  if (RND == R_EDEN) {
    c.s32 = 1.0f;
    c.d6 = exact_div_setup(FP4_EDEN_S);
  } else {
    c.s32 = nv_tensor_scale(amax_in, RND == R_SR ? FP4_NV_SR_DIV : FP4_NV_RTN_DIV);
    c.d6 = exact_div_setup(__fmul_rn(c.s32, RND == R_SR ? FP4_NV_SR_GDIV : 6.0f));
    c.d4 = exact_div_setup(__fmul_rn(c.s32, 4.0f));
  }
  return c;
}

template <int FMT, int RND, int HAD>
__device__ __forceinline__ uint32_t process32(float* x, bool active, int64_t orow, int64_t ocol, int lane,
                                              const QParams& p, const Shared& sh, const QuantConsts& qc) {
  constexpr int G = FMT == FMT_NV ? 16 : 32;
  constexpr int NG = 32 / G;
  if (HAD > 0) fwht32_lanes<HAD>(x, lane);      // signs already applied by the loader
  uint32_t gmb[NG];
  if (NG == 2) {
    gmb[0] = absmax16(x);
    gmb[NG - 1] = absmax16(x + 16);
  } else {
    gmb[0] = max(absmax16(x), absmax16(x + 16));
  }
  uint32_t lmax = NG == 2 ? max(gmb[0], gmb[NG - 1]) : gmb[0];
  if (!active) lmax = 0;
  if (RND == R_AMAX) return lmax;
  if (active && lmax >= 0x7F800000u && (FMT == FMT_MX || RND == R_EDEN)) flag_status(p.status, ST_NONFINITE);

  uint32_t w[4] = {0u, 0u, 0u, 0u};
  uint32_t sb[NG];
  uint32_t mbits = 0;

  if (FMT == FMT_NV && (RND == R_RTN || RND == R_SQ16 || RND == R_FOS || RND == R_SR || RND == R_QUEST)) {
    const float s32 = qc.s32;
#pragma unroll
    for (int g = 0; g < NG; ++g) {
      const float* xg = x + 16 * g;
      const float gmax = bitsf(gmb[g]);
      uint32_t* wg = w + 2 * g;
      if (RND == R_SQ16) {
        // RTN against the maximum of the group's 16 x 16 block of the input
        const int64_t oc = (ocol >> 4) + g, orb = orow >> 4;
        const float bm = bitsf(p.bmax[p.bmax_trans ? oc * p.bmax_ld + orb : orb * p.bmax_ld + oc]);
        const uint32_t s8 = e4m3_rtn(exact_div(bm, qc.d6));
        const float d = __fmul_rn(e4m3x2_value(s8).x, s32), inv = __frcp_rn(d);
        enc16(xg, inv, finite_pos(d, inv), wg);
        sb[g] = s8;
      } else if (RND == R_RTN) {
        const uint32_t s8 = e4m3_rtn(exact_div(gmax, qc.d6));
        const float d = __fmul_rn(e4m3x2_value(s8).x, s32), inv = __frcp_rn(d);
        enc16(xg, inv, finite_pos(d, inv), wg);
        sb[g] = s8;
      } else if (RND == R_FOS) {
        // both candidate scales in one conversion: s6 in bits 0-7, s4 in 8-15
        const uint32_t c2 = e4m3x2_rtn(exact_div(gmax, qc.d6), exact_div(gmax, qc.d4));
        const float2 v2 = e4m3x2_value(c2);
        const float d6 = __fmul_rn(v2.x, s32), i6 = __frcp_rn(d6);
        const float d4 = __fmul_rn(v2.y, s32), i4 = __frcp_rn(d4);
        uint32_t w6[2], w4[2];
        float q[16];
        enc16_dec(xg, i6, finite_pos(d6, i6), w6, q);
        const float e6 = sse16q(xg, q, d6);
        enc16_dec(xg, i4, finite_pos(d4, i4), w4, q);
        const bool pick4 = sse16q(xg, q, d4) < e6;   // a tie keeps the 6-scale
        wg[0] = clear_neg_zero(pick4 ? w4[0] : w6[0]);
        wg[1] = clear_neg_zero(pick4 ? w4[1] : w6[1]);
        sb[g] = pick4 ? (c2 >> 8) : (c2 & 0xFFu);
      } else if (RND == R_SR) {
        const uint32_t s8 = e4m3_rtn(exact_div(gmax, qc.d6));
        float d = __fmul_rn(e4m3x2_value(s8).x, s32), inv = __frcp_rn(d);
        const bool ok = finite_pos(d, inv);
        const uint64_t q0 = uint64_t(orow * p.cols + ocol + 16 * g) >> 2;
#pragma unroll
        for (int b = 0; b < 4; ++b) {
          u32x4 r = philox_block(p.seed, q0 + b, TAG_SR_ELEM, p.tensor_tag);
          const uint32_t rw[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int e = 4 * b + j;
            uint32_t c = ok ? e2m1_sr(__fmul_rn(xg[e], inv), u24(rw[j])) : 0u;
            wg[e >> 3] |= c << (4 * (e & 7));
          }
        }
        sb[g] = s8;
      } else {  // QuEST on the E4M3 scale grid
        float sq[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) sq[j] = __fmul_rn(xg[j], xg[j]);
        const float sig2 = __fdiv_rn(tree16(sq), 16.0f);
        const float hi = __fmul_rn(25.0f, sig2);
        auto t2 = [&](int cc) {
          float t = __fmul_rn(6.0f, __fmul_rn(e4m3_value(uint32_t(cc)), s32));
          return __fmul_rn(t, t);
        };
        int lo = 1, hi_i = 127;
        while (lo < hi_i) { int mid = (lo + hi_i) >> 1; if (t2(mid) >= sig2) hi_i = mid; else lo = mid + 1; }
        const int clo = lo;
        lo = 0; hi_i = 126;
        while (lo < hi_i) { int mid = (lo + hi_i + 1) >> 1; if (t2(mid) <= hi) lo = mid; else hi_i = mid - 1; }
        const int chi = lo;
        uint32_t s8;
        if (clo <= chi && chi >= 1) {
          float best = __int_as_float(0x7F800000);
          int bc = clo;
          for (int cc = clo; cc <= chi; ++cc) {
            float d = __fmul_rn(e4m3_value(uint32_t(cc)), s32), inv = __frcp_rn(d);
            uint32_t wt[2];
            float qv[16];
            enc16_dec(xg, inv, finite_pos(d, inv), wt, qv);   // raw codes: +-0 give the same error
            float e = sse16q(xg, qv, d);
            if (e <= best) { best = e; bc = cc; }
          }
          s8 = uint32_t(bc);
        } else {
          s8 = e4m3_rtn(exact_div(gmax, qc.d6));
        }
        float d = __fmul_rn(e4m3_value(s8), s32), inv = __frcp_rn(d);
        const bool ok = finite_pos(d, inv);
        enc16(xg, inv, ok, wg);
#pragma unroll
        for (int j = 0; j < 16; ++j)
          mbits |= uint32_t(ok && fabsf(__fmul_rn(xg[j], inv)) > 6.0f) << (16 * g + j);
        sb[g] = s8;
      }
    }
  } else if (FMT == FMT_NV && RND == R_EDEN) {
    float num_g[NG], den_g[NG];
#pragma unroll
    for (int g = 0; g < NG; ++g) {
      const float* xg = x + 16 * g;
      const float pq = e8m3_div6(bitsf(gmb[g]));
      const float inv = rcp_e8m3(pq);
      // grid values of the raw codes: a -0 instead of +0 changes only the
      // sign of zero terms, hence of an all-zero sum, which gives S = 1 either way
      float q[16], yy[16], yq[16];
      enc16_dec(xg, inv, finite_pos(pq, inv), w + 2 * g, q);
      w[2 * g] = clear_neg_zero(w[2 * g]);
      w[2 * g + 1] = clear_neg_zero(w[2 * g + 1]);
#pragma unroll
      for (int j = 0; j < 16; j += 2) {
        const float2 y2 = ld2(xg, j);
        st2(yy, j, __fmul2_rn(y2, y2));
        st2(yq, j, __fmul2_rn(y2, __fmul2_rn(ld2(q, j), splat2(pq))));
      }
      num_g[g] = tree16p(yy);      // the two halves of the 32-element tree
      den_g[g] = tree16p(yq);
      sb[g] = fbits(pq) >> 16;     // bf16 pseudo-scale (exact)
    }
    if (active) {
      *reinterpret_cast<uint32_t*>(p.pseudo + orow * (p.cols >> 4) + (ocol >> 4)) = sb[0] | (sb[NG - 1] << 16);
    }
    if (HAD == 16) {
      float S2[2];
#pragma unroll
      for (int g = 0; g < 2; ++g) S2[g] = den_g[g] > 0.0f ? __fdiv_rn(num_g[g], den_g[g]) : 1.0f;
      if (active) *reinterpret_cast<float2*>(p.eden_S + orow * (p.cols >> 4) + (ocol >> 4)) = make_float2(S2[0], S2[1]);
    } else {
      float num = __fadd_rn(num_g[0], num_g[NG - 1]), den = __fadd_rn(den_g[0], den_g[NG - 1]);
      if (HAD > 32) {                      // the block spans HAD / 32 aligned lanes
        num = tree_lanes<(HAD > 32 ? HAD / 32 : 1)>(num);
        den = tree_lanes<(HAD > 32 ? HAD / 32 : 1)>(den);
      }
      const float S = den > 0.0f ? __fdiv_rn(num, den) : 1.0f;
      if (active && (lane & (HAD > 32 ? HAD / 32 - 1 : 0)) == 0) p.eden_S[orow * (p.cols / HAD) + ocol / HAD] = S;
    }
  } else if (FMT == FMT_MX && (RND == R_RTN || RND == R_SR)) {
    int e = int(gmb[0] >> 23) - 129;
    e = e < -127 ? -127 : e;
    const float sc = pow2f(-e);
    if (RND == R_RTN) {
      float v[32];
#pragma unroll
      for (int j = 0; j < 32; j += 2) st2(v, j, __fmul2_rn(ld2(x, j), splat2(sc)));
#pragma unroll
      for (int k = 0; k < 4; ++k) w[k] = enc8_hw(v + 8 * k);
    } else {
      const uint64_t q0 = uint64_t(orow * p.cols + ocol) >> 2;
#pragma unroll
      for (int b = 0; b < 8; ++b) {
        u32x4 r = philox_block(p.seed, q0 + b, TAG_SR_ELEM, p.tensor_tag);
        const uint32_t rw[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int el = 4 * b + j;
          uint32_t c = e2m1_sr(__fmul_rn(__fmul_rn(x[el], FP4_QUARTET_PRESCALE), sc), u24(rw[j]));
          w[el >> 3] |= c << (4 * (el & 7));
        }
      }
    }
    sb[0] = uint32_t(e + 127);
  } else if (FMT == FMT_MX && RND == R_QUEST) {
    float sq[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) sq[j] = __fmul_rn(x[j], x[j]);
    const float sig2 = __fdiv_rn(tree32(sq), 32.0f);
    const float hi = __fmul_rn(25.0f, sig2);
    const int fl = sig2 > 0.0f ? floor_log2(sig2) : -300;
    const int elo = (fl >> 1) - 4;
    int be = 0;
    float bs = __int_as_float(0x7F800000);
    bool found = false;
#pragma unroll 1
    for (int k = 0; k < 8; ++k) {
      int e = elo + k;
      e = e < -127 ? -127 : (e > 125 ? 125 : e);
      const float t = __fmul_rn(6.0f, pow2f(e));
      const float tt = __fmul_rn(t, t);
      const bool inwin = (sig2 <= tt) && (tt <= hi) && (sig2 > 0.0f);
      if (!inwin) continue;              // (an out-of-window candidate never wins)
      const float sc = pow2f(-e), d = pow2f(e);
      float v[32], qv[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) v[j] = __fmul_rn(x[j], sc);
#pragma unroll
      for (int q = 0; q < 4; ++q) (void)enc8_dec(v + 8 * q, qv + 8 * q);   // grid values of the raw codes: +-0 give the same error
      const float s = __fadd_rn(sse16q(x, qv, d), sse16q(x + 16, qv + 16, d));
      if (s <= bs) { bs = s; be = e; }
      found = true;
    }
    int e;
    if (found) {
      e = be;
    } else {
      e = int(gmb[0] >> 23) - 129;
      e = e < -127 ? -127 : e;
    }
    const float sc = pow2f(-e);
    float v[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      v[j] = __fmul_rn(x[j], sc);
      mbits |= uint32_t(fabsf(v[j]) > 6.0f) << j;
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) w[q] = enc8_hw(v + 8 * q);
    sb[0] = uint32_t(e + 127);
  }

  if (active) {
    *reinterpret_cast<uint4*>(p.codes + orow * (p.cols >> 1) + (ocol >> 1)) = make_uint4(w[0], w[1], w[2], w[3]);
    if (RND != R_EDEN) {
      const int64_t k = ocol / G;
      if (NG == 2) {
        const uint16_t two = uint16_t(sb[0] | (sb[NG - 1] << 8));
        if (p.scales) *reinterpret_cast<uint16_t*>(p.scales + orow * (p.cols / G) + k) = two;
        if (p.swz) *reinterpret_cast<uint16_t*>(p.swz + swz_offset(orow, k, p.nkb)) = two;
      } else {
        if (p.scales) p.scales[orow * (p.cols / G) + k] = uint8_t(sb[0]);
        if (p.swz) p.swz[swz_offset(orow, k, p.nkb)] = uint8_t(sb[0]);
      }
    }
    if (RND == R_QUEST && p.mask) *reinterpret_cast<uint32_t*>(p.mask + orow * (p.cols >> 3) + (ocol >> 3)) = mbits;
  }
  return lmax;
}

// Resident 256-thread blocks per SM the register allocation is held to.  The
// row kernels hold the next task's 64 input bytes in registers while they
// process the current one: RTN / amax at 3 blocks (85 registers) and
// Four-Over-Six / MS-EDEN at 2 (128) run faster that way than at 4 / 3
// blocks, with or without the early load (which spills at those budgets);
// SR and QuEST keep their registers.  RTN behind a 64- to 256-point rotation
// (shuffle stages) runs faster at 4 blocks without the early load.
template <int RND, int HAD>
__host__ __device__ constexpr bool row_prefetch() {
  return !((RND == R_RTN || RND == R_SQ16) && HAD >= 64);
}
template <int RND, int HAD>
__host__ __device__ constexpr int quant_min_blocks() {
  return (RND == R_RTN || RND == R_SQ16 || RND == R_AMAX) ? (row_prefetch<RND, HAD>() ? 3 : 4)
                                                          : ((RND == R_FOS || RND == R_EDEN) ? 2 : 1);
}
// Resident 128-thread blocks per SM of the transposed kernel: its 18.6 KB
// tile and 64 registers allow 8, which overlap one block's loads with the
// others' arithmetic (smaller blocks than 256 threads wait less at the
// barrier between the two phases).
template <int RND>
__host__ __device__ constexpr int quant_trans_min_blocks() {
  return (RND == R_SR || RND == R_QUEST) ? 2 : 8;
}

// Row-wise, 32 elements per lane, grid-stride over 32-element tasks.
template <int LOAD, int FMT, int RND, int HAD>
__global__ void __launch_bounds__(256, quant_min_blocks<RND, HAD>()) k_quant_row32(QParams p) {
  __shared__ Shared sh;
  load_signs<HAD>(sh, p);
  const int lane = threadIdx.x & 31;
  const int64_t tpr = p.cols >> 5, tasks = p.rows * tpr;
  const uint32_t amax_in = (FMT == FMT_NV && RND != R_EDEN && RND != R_AMAX) ? *p.amax_bits : 0u;
  const float in_ts = LOAD == LD_ROW_FP4 ? *p.in_ts : 1.0f;
  if (blockIdx.x == 0 && threadIdx.x == 0) write_tensor_scale<FMT, RND>(p, amax_in);
  const QuantConsts qc = quant_consts<FMT, RND>(amax_in);
  uint32_t acc = 0;
  const int64_t stride = int64_t(gridDim.x) * blockDim.x;
  // The lane's 32 columns sit at the same offset of their rotation block on
  // every task (cols is a multiple of the block, the stride of 32 tasks), so
  // its sign masks are fixed for the whole loop.
  const uint32_t sw = lane_signs<HAD>(sh, p, 32 * (lane & 7));
  uint32_t sm[LOAD == LD_ROW ? 16 : 4];
  if (LOAD == LD_ROW) sign_masks_bf16(sw, sm);
  else if (LOAD == LD_ROW_FP4) sign_masks_fp4(sw, sm);
  // Row and column task of t = base + lane, advanced by the grid stride
  // without a division per task.
  const int64_t base0 = int64_t(blockIdx.x) * blockDim.x + (threadIdx.x & ~31);
  int64_t trow = (base0 + lane) / tpr, tct = (base0 + lane) % tpr;
  const int64_t drow = stride / tpr, dct = stride % tpr;
  // bf16 input: the next task's 64 bytes are loaded before this task is
  // processed, so their latency overlaps the arithmetic
  constexpr bool PF = LOAD == LD_ROW && row_prefetch<RND, HAD>();
  uint4 pv[4];
  if (PF) {
    const bool a0 = base0 + lane < tasks;
    const uint4* src = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(p.x) + (a0 ? trow * p.cols + tct * 32 : 0));
#pragma unroll
    for (int i = 0; i < 4; ++i) pv[i] = a0 ? __ldg(src + i) : make_uint4(0, 0, 0, 0);
  }
  for (int64_t base = base0; base < tasks; base += stride) {
    const int64_t t = base + lane;
    const bool active = t < tasks;
    const int64_t orow = active ? trow : 0, ocol = active ? tct * 32 : 0;
    tct += dct;
    trow += drow;
    if (tct >= tpr) { tct -= tpr; ++trow; }
    float x[32];
    if (LOAD == LD_ROW) {
      uint4 v[4];
      if (PF) {
#pragma unroll
        for (int i = 0; i < 4; ++i) v[i] = pv[i];
        const bool an = t + stride < tasks;
        const uint4* src =
            reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(p.x) + (an ? trow * p.cols + tct * 32 : 0));
#pragma unroll
        for (int i = 0; i < 4; ++i) pv[i] = an ? __ldg(src + i) : make_uint4(0, 0, 0, 0);
      } else {
        const uint4* src = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(p.x) + orow * p.cols + ocol);
#pragma unroll
        for (int i = 0; i < 4; ++i) v[i] = active ? __ldg(src + i) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        v[i].x ^= sm[4 * i]; v[i].y ^= sm[4 * i + 1]; v[i].z ^= sm[4 * i + 2]; v[i].w ^= sm[4 * i + 3];
        bf16x8_to_f32(v[i], x + 8 * i);
      }
    } else if (LOAD == LD_ROW_F32) {
      const float4* src = reinterpret_cast<const float4*>(static_cast<const float*>(p.x) + orow * p.cols + ocol);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float4 v = active ? __ldg(src + i) : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
        x[4 * i] = v.x; x[4 * i + 1] = v.y; x[4 * i + 2] = v.z; x[4 * i + 3] = v.w;
      }
    } else {
      uint4 cw = make_uint4(0, 0, 0, 0);
      uint32_t s0 = 0, s1 = 0;
      const int gsh = p.in_fmt == FMT_NV ? 4 : 5;   // log2 of the input group size
      if (active) {
        cw = __ldg(reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(p.x) + orow * (p.cols >> 1) + (ocol >> 1)));
        s0 = p.in_scales[orow * (p.cols >> gsh) + (ocol >> gsh)];
        s1 = p.in_scales[orow * (p.cols >> gsh) + ((ocol + 16) >> gsh)];
      }
      const float sa = fp4_in_scale(s0, p.in_fmt), sbv = fp4_in_scale(s1, p.in_fmt);
      const uint32_t cws[4] = {cw.x ^ sm[0], cw.y ^ sm[1], cw.z ^ sm[2], cw.w ^ sm[3]};
#pragma unroll
      for (int k = 0; k < 4; ++k) dec8(cws[k], x + 8 * k);
#pragma unroll
      for (int j = 0; j < 32; j += 2)
        st2(x, j, __fmul2_rn(__fmul2_rn(ld2(x, j), splat2(j < 16 ? sa : sbv)), splat2(in_ts)));
    }
    acc = max(acc, process32<FMT, RND, HAD>(x, active, orow, ocol, lane, p, sh, qc));
  }
  if (RND == R_AMAX || RND == R_EDEN) block_max_atomic(acc, sh, p.amax_bits, p.status);
}

// Transposed, 32 elements per lane: an input tile of T32Tile::ROWS rows (the
// output rows' length covered by one block: 128, or 256 for 256-element
// rotation blocks) x T32Tile::COLS columns (4096 elements) is staged as fp32
// with a 4-float skew every 32 columns, so the 16-byte reads of the lanes on
// one output row hit distinct banks.
template <int HAD>
struct T32Tile {
  static constexpr int THREADS = 128;
  static constexpr int ROWS = HAD > 128 ? 256 : 128;   // input rows = output columns per block
  static constexpr int COLS = THREADS * 32 / ROWS;       // input columns = output rows per block
  static constexpr int PITCH = ROWS + ROWS / 8;          // + 4 floats per 32
  static constexpr int LPR = ROWS / 32;                  // lanes per output row
};
__device__ __forceinline__ int t32_col(int c) { return c + 4 * (c >> 5); }

template <int LOAD, int FMT, int RND, int HAD>
__global__ void __launch_bounds__(T32Tile<HAD>::THREADS, quant_trans_min_blocks<RND>()) k_quant_trans32(QParams p) {
  using TT = T32Tile<HAD>;
  __shared__ Shared sh;
  __shared__ __align__(16) float tile[TT::COLS][TT::PITCH];
  load_signs<HAD>(sh, p);
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int64_t r0 = int64_t(blockIdx.x) * TT::ROWS, c0 = int64_t(blockIdx.y) * TT::COLS;
  const int64_t R = p.in_rows, C = p.in_cols;
  {
    // warp w loads input rows 64 rh + 2 lane (+1) and 16 columns 16 cb ..
    constexpr int NCB = TT::COLS / 16;
    const int rh = w / NCB, cb = w % NCB;
    const int rl = 64 * rh + 2 * lane;
    const int64_t cc = c0 + 16 * cb;
    float va[16], vb[16];
    // Input rows rl and rl + 1 are positions rl, rl + 1 of their rotation
    // block along the output rows (r0 is a multiple of 128): one sign each.
    const uint32_t sgn_a = (lane_signs<HAD>(sh, p, rl) >> (rl & 31)) & 1u;
    const uint32_t sgn_b = (lane_signs<HAD>(sh, p, rl + 1) >> ((rl + 1) & 31)) & 1u;
    if (LOAD == LD_TRANS) {
      const uint32_t ma = sgn_a * 0x80008000u, mb = sgn_b * 0x80008000u;
      const uint16_t* xb = static_cast<const uint16_t*>(p.x);
      uint4 a[2], b[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int64_t col = cc + 8 * h;
        a[h] = (col < C && r0 + rl < R) ? __ldg(reinterpret_cast<const uint4*>(xb + (r0 + rl) * C + col))
                                        : make_uint4(0, 0, 0, 0);
        b[h] = (col < C && r0 + rl + 1 < R) ? __ldg(reinterpret_cast<const uint4*>(xb + (r0 + rl + 1) * C + col))
                                            : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        a[h].x ^= ma; a[h].y ^= ma; a[h].z ^= ma; a[h].w ^= ma;
        b[h].x ^= mb; b[h].y ^= mb; b[h].z ^= mb; b[h].w ^= mb;
        bf16x8_to_f32(a[h], va + 8 * h);
        bf16x8_to_f32(b[h], vb + 8 * h);
      }
    } else {
      const uint8_t* xc = static_cast<const uint8_t*>(p.x);
      const float in_ts = *p.in_ts;
      const int gsh = p.in_fmt == FMT_NV ? 4 : 5;   // log2 of the input group size
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        const int64_t r = r0 + rl + q;
        uint2 cw = make_uint2(0, 0);
        uint32_t sa = 0;
        if (r < R && cc < C) {
          cw = __ldg(reinterpret_cast<const uint2*>(xc + r * (C >> 1) + (cc >> 1)));
          sa = p.in_scales[r * (C >> gsh) + (cc >> gsh)];
        }
        const uint32_t m = (q ? sgn_b : sgn_a) * 0x88888888u;
        const float s_a = fp4_in_scale(sa, p.in_fmt);
        float* dst = q ? vb : va;
        dec8(cw.x ^ m, dst);
        dec8(cw.y ^ m, dst + 8);
#pragma unroll
        for (int j = 0; j < 16; j += 2) st2(dst, j, __fmul2_rn(__fmul2_rn(ld2(dst, j), splat2(s_a)), splat2(in_ts)));
      }
    }
    const int pc = t32_col(rl);
#pragma unroll
    for (int j = 0; j < 16; ++j) *reinterpret_cast<float2*>(&tile[16 * cb + j][pc]) = make_float2(va[j], vb[j]);
  }
  __syncthreads();
  const uint32_t amax_in = (FMT == FMT_NV && RND != R_EDEN && RND != R_AMAX) ? *p.amax_bits : 0u;
  if (blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0) write_tensor_scale<FMT, RND>(p, amax_in);
  const QuantConsts qc = quant_consts<FMT, RND>(amax_in);
  const int orl = threadIdx.x / TT::LPR, seg = threadIdx.x % TT::LPR;
  const int64_t orow = c0 + orl, ocol = r0 + 32 * seg;
  const bool active = orow < C && ocol < R;
  float x[32];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float4 v = *reinterpret_cast<const float4*>(&tile[orl][t32_col(32 * seg) + 4 * i]);
    x[4 * i] = v.x; x[4 * i + 1] = v.y; x[4 * i + 2] = v.z; x[4 * i + 3] = v.w;
  }
  const uint32_t acc = process32<FMT, RND, HAD>(x, active, active ? orow : 0, active ? ocol : 0, lane, p, sh, qc);
  if (RND == R_AMAX || RND == R_EDEN) block_max_atomic(acc, sh, p.amax_bits, p.status);
}

// Exhaustive check of the hardware E2M1 encoder against the per-element
// software rounding over every non-NaN fp32 bit pattern, and of the hardware
// decoder over every byte of two codes; counts mismatches.
static __global__ void k_selftest_e2m1(unsigned long long* mismatches) {
  unsigned long long bad = 0;
  const uint64_t n = 1ull << 32;
  for (uint64_t i = (uint64_t(blockIdx.x) * blockDim.x + threadIdx.x) * 8; i < n;
       i += uint64_t(gridDim.x) * blockDim.x * 8) {
    float v[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const uint32_t b = uint32_t(i + j);
      v[j] = ((b & 0x7FFFFFFFu) > 0x7F800000u) ? 0.0f : bitsf(b);   // NaN -> skip (compare 0)
    }
    bad += (enc8_hw(v) != enc8_sw(v)) ? 1ull : 0ull;
  }
  // The hardware decoder against the code table, over every pair of codes.
  if (blockIdx.x == 0) {
    for (uint32_t c = threadIdx.x; c < 256u; c += blockDim.x) {
      float q[8];
      // four different bytes per word, so a byte decoded from the wrong
      // position is seen
      const uint32_t by[4] = {c, (c * 7u + 0x35u) & 0xFFu, c ^ 0xA6u, (c * 13u + 0x5Bu) & 0xFFu};
      dec8(by[0] | (by[1] << 8) | (by[2] << 16) | (by[3] << 24), q);
      for (int j = 0; j < 8; ++j)
        bad += (fbits(q[j]) != fbits(e2m1_value((by[j >> 1] >> (4 * (j & 1))) & 15u))) ? 1ull : 0ull;
    }
  }
  if (bad) atomicAdd(mismatches, bad);
}

// Exhaustive and hashed checks of the exact scale shortcuts against CUDA's
// IEEE operations; one mismatch counter each: [0] exact_div by 6 over every
// non-negative finite fp32 dividend, [1] rcp_e8m3 over every non-negative
// E8M3 value, [2] exact_div on 2^32 hashed (dividend, divisor) pairs over the
// whole divisor range with quotients 2^-25 .. 2^9, [3] the E4M3 decoder over
// every non-NaN code in both byte positions, [4] the E4M3 encoder over every
// non-negative finite fp32 value in both byte positions, [5] the MS-EDEN
// pseudo-scale e8m3_div6 over every non-negative fp32 value up to +inf.
static __global__ void k_selftest_arith(unsigned long long* mismatches) {
  unsigned long long bad[6] = {0, 0, 0, 0, 0, 0};
  const uint64_t stride = uint64_t(gridDim.x) * blockDim.x;
  const uint64_t tid = uint64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  const ExactDiv six = exact_div_setup(6.0f);
  for (uint64_t i = tid; i < 0x7F800000ull; i += stride) {
    const float a = bitsf(uint32_t(i));
    bad[0] += fbits(exact_div(a, six)) != fbits(__fdiv_rn(a, 6.0f));
    const float t1 = bitsf(uint32_t(0x7F7FFFFFull - i));
    const uint32_t c2 = e4m3x2_rtn(a, t1);
    bad[4] += (c2 & 0xFFu) != e4m3_rtn(a) || (c2 >> 8) != e4m3_rtn(t1);
  }
  for (uint64_t i = tid; i <= 0x7F800000ull; i += stride) {
    const float g = bitsf(uint32_t(i));
    bad[5] += fbits(e8m3_div6(g)) != fbits(e8m3_round(__fdiv_rn(g, 6.0f)));
  }
  for (uint64_t i = tid; i < 255ull * 8; i += stride) {   // exponent field 0..254, 3 mantissa bits
    const float pv = bitsf(uint32_t(((i >> 3) << 23) | ((i & 7) << 20)));
    bad[1] += fbits(rcp_e8m3(pv)) != fbits(__frcp_rn(pv));
  }
  for (uint64_t i = tid; i < (1ull << 32); i += stride) {
    const uint32_t h1 = uint32_t(i) * 0x9E3779B1u ^ uint32_t(i >> 13) * 0x85EBCA77u;
    const uint32_t h2 = (h1 ^ (h1 >> 15)) * 0xC2B2AE3Du;
    const uint32_t h3 = (h2 ^ (h2 >> 13)) * 0x27D4EB2Fu;
    const int eb = 27 + int(h1 % 201u);
    const float b = bitsf((uint32_t(eb) << 23) | (h2 & 0x7FFFFFu));
    int ea = eb + int(h3 % 35u) - 25;
    ea = ea < 1 ? 1 : (ea > 254 ? 254 : ea);
    const float a = bitsf((uint32_t(ea) << 23) | (h3 >> 9));
    const ExactDiv d = exact_div_setup(b);
    bad[2] += fbits(exact_div(a, d)) != fbits(__fdiv_rn(a, b));
  }
  if (blockIdx.x == 0) {
    for (uint32_t c = threadIdx.x; c < 127u; c += blockDim.x) {   // 0x7F is NaN, never a scale
      const uint32_t c1 = (c * 37u + 11u) % 127u;
      const float2 v = e4m3x2_value(c | (c1 << 8));
      bad[3] += fbits(v.x) != fbits(e4m3_value(c)) || fbits(v.y) != fbits(e4m3_value(c1));
    }
  }
#pragma unroll
  for (int k = 0; k < 6; ++k)
    if (bad[k]) atomicAdd(mismatches + k, bad[k]);
}

}  // namespace fp4
