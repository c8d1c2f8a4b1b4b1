// NVFP4 MSE-optimal scale search: the group step and the tensor-scale step
// (declarations and the definition of the two steps in quant_mse.cuh).
//
// Group step, one 32-element task (two scale groups) per thread: every
// candidate E4M3 code c = 1..126 gives d = fp32(E4M3(c) s_T) and its correctly
// rounded reciprocal (a per-block table, s_T being uniform), the RTN codes of
// x * (1/d) and their fp32 squared error (sse16q, the pairwise tree of
// fp32((x - fp32(q d))^2)); the smallest error wins, ties to the larger code.
// Candidates that the top element's own error term already rules out are not
// evaluated in full (top_term), and the scan below the seed stops where that
// term can only grow; the result is that of the exhaustive scan.
// A group whose maximum is zero (or NaN) takes code 0 and zero codes.  With
// the winning codes, u = E4M3(c) q is exact in fp32 and x u, u u are exact in
// float64; the block sums both over its 8192 consecutive elements as a
// pairwise tree (lane: 32 elements, warp: butterfly, block: 8 warps) and
// writes one (<x, u>, <u, u>) pair.
//
// Tensor-scale step, one block: the pairs of all blocks summed as a pairwise
// tree over the block index (zero-padded to a power of two, which does not
// change the value), then s_T = fp32(<x, u> / <u, u>) when both sums are
// positive and the quotient is a finite positive fp32 value; otherwise s_T is
// kept.  Both steps run in IEEE round-to-nearest arithmetic only.
#include "quant_dispatch.cuh"
#include "quant_mse.cuh"

namespace fp4 {

// Pairwise float64 tree over 16 consecutive values (level 0 adds (2i, 2i+1)).
__device__ __forceinline__ double tree16d(const double* v) {
  double a[8], b[4];
#pragma unroll
  for (int i = 0; i < 8; ++i) a[i] = __dadd_rn(v[2 * i], v[2 * i + 1]);
#pragma unroll
  for (int i = 0; i < 4; ++i) b[i] = __dadd_rn(a[2 * i], a[2 * i + 1]);
  return __dadd_rn(__dadd_rn(b[0], b[1]), __dadd_rn(b[2], b[3]));
}

// A value of the group whose magnitude is the group maximum (0 when none is,
// e.g. a NaN maximum).
__device__ __forceinline__ float top_value(const float* x, float gm) {
  float t = 0.0f;
#pragma unroll
  for (int j = 15; j >= 0; --j) t = fabsf(x[j]) == gm ? x[j] : t;
  return t;
}

// The candidate's squared-error term of one element, computed exactly as the
// candidate's group error computes it (code of fp32(x * inv) by the same
// conversion, zero when the scale is unusable; fp32((x - fp32(q d))^2)).  The
// group error is a round-to-nearest pairwise sum of non-negative terms, which
// is never smaller than any one of them, so a candidate whose top-element term
// exceeds the best error found so far cannot be the minimiser.
__device__ __forceinline__ float top_term(float xt, float d, float inv, bool ok) {
  const uint32_t code = ok ? (e2m1x2_rn(__fmul_rn(xt, inv), 0.0f) & 0xFu) : 0u;
  const float q = __half2float(__ushort_as_half(uint16_t(e2m1x2_to_f16x2(code) & 0xFFFFu)));
  const float e = __fsub_rn(xt, __fmul_rn(q, d));
  return __fmul_rn(e, e);
}

// E4M3 code nearest gm / (6 s_T), clamped to 1..126 (only a visiting order).
__device__ __forceinline__ int seed_code(float gm, float inv6) {
  const int c = int(e4m3_rtn(__fmul_rn(gm, inv6)));
  return c < 1 ? 1 : (c > 126 ? 126 : c);
}

// Full error of candidate c for one group; the smaller error wins, a tie goes
// to the larger code -- the result of an ascending scan with <=, whatever the
// order candidates are visited in.  NaN errors never win.
__device__ __forceinline__ void consider(const float* xg, int c, float d, float inv, float& best, int& bc) {
  uint32_t wt[2];
  float q[16];
  enc16_dec(xg, inv, finite_pos(d, inv), wt, q);
  const float e = sse16q(xg, q, d);
  if (e < best || (e == best && c > bc)) { best = e; bc = c; }
}

// Candidate c above the seed: evaluated in full unless its top-element term
// rules it out.
__device__ __forceinline__ void probe_up(const float* xg, float xt, int c, const float* sd, const float* si,
                                         float& best, int& bc) {
  const float d = sd[c], inv = si[c];
  if (!(top_term(xt, d, inv, finite_pos(d, inv)) > best)) consider(xg, c, d, inv, best, bc);
}

// Candidate c below the seed; returns whether smaller codes still need a
// look.  Where the scale is unusable (zero codes) or fp32(6 d) <= |top|, the
// top element's term is its clipping error (|top| - fp32(6 d))^2 (or top^2),
// which only grows as d shrinks while the best error only falls: once such a
// candidate is ruled out, so is every smaller one.
__device__ __forceinline__ bool probe_down(const float* xg, float xt, int c, const float* sd, const float* si,
                                           float& best, int& bc) {
  const float d = sd[c], inv = si[c];
  const bool ok = finite_pos(d, inv);
  if (top_term(xt, d, inv, ok) > best) return ok && __fmul_rn(6.0f, d) > fabsf(xt);
  consider(xg, c, d, inv, best, bc);
  return true;
}

__global__ void __launch_bounds__(256) k_mse_group(MseParams p) {
  __shared__ float s_d[128], s_inv[128];
  __shared__ double s_num[8], s_den[8];
  float s_T;
  if (p.first) {
    const uint32_t ab = *p.amax_bits;
    s_T = nv_tensor_scale(ab, FP4_NV_RTN_DIV);
    if (blockIdx.x == 0 && threadIdx.x == 0) {
      *p.ts = s_T;
      if ((ab & 0x7FFFFFFFu) >= 0x7F800000u) flag_status(p.status, ST_NONFINITE);
    }
  } else {
    s_T = *p.ts;
  }
  if (threadIdx.x < 128) {
    const float d = __fmul_rn(e4m3_value(threadIdx.x), s_T);
    s_d[threadIdx.x] = d;
    s_inv[threadIdx.x] = __frcp_rn(d);
  }
  __syncthreads();

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t tpr = p.cols >> 5, tasks = p.rows * tpr;
  const int64_t t = int64_t(blockIdx.x) * MSE_TASKS + threadIdx.x;
  const bool active = t < tasks;
  const int64_t orow = active ? t / tpr : 0, ocol = active ? (t - orow * tpr) * 32 : 0;
  float x[32];
  {
    const uint4* src = reinterpret_cast<const uint4*>(p.x + orow * p.cols + ocol);
#pragma unroll
    for (int i = 0; i < 4; ++i) bf16x8_to_f32(active ? __ldg(src + i) : make_uint4(0, 0, 0, 0), x + 8 * i);
  }
  const float gm0 = bitsf(absmax16(x)), gm1 = bitsf(absmax16(x + 16));
  float best0 = __int_as_float(0x7F800000), best1 = best0;
  int c0 = 0, c1 = 0;
  if (gm0 > 0.0f || gm1 > 0.0f) {
    const float xt0 = top_value(x, gm0), xt1 = top_value(x + 16, gm1);
    // Candidates are visited outward from a seed near the AbsMax scale (seed + k
    // and seed - k at step k), so the lanes of a warp evaluate in the same steps.
    const float i6 = __frcp_rn(__fmul_rn(6.0f, s_T));
    const int sd0 = seed_code(gm0, i6), sd1 = seed_code(gm1, i6);
    const bool on0 = gm0 > 0.0f, on1 = gm1 > 0.0f;
    if (on0) consider(x, sd0, s_d[sd0], s_inv[sd0], best0, c0);
    if (on1) consider(x + 16, sd1, s_d[sd1], s_inv[sd1], best1, c1);
    bool dn0 = on0, dn1 = on1;
#pragma unroll 1
    for (int k = 1; k <= 125; ++k) {
      const int u0 = sd0 + k, l0 = sd0 - k, u1 = sd1 + k, l1 = sd1 - k;
      const bool up0 = on0 && u0 <= 126, up1 = on1 && u1 <= 126;
      dn0 = dn0 && l0 >= 1;
      dn1 = dn1 && l1 >= 1;
      if (!(up0 || up1 || dn0 || dn1)) break;
      if (up0) probe_up(x, xt0, u0, s_d, s_inv, best0, c0);
      if (up1) probe_up(x + 16, xt1, u1, s_d, s_inv, best1, c1);
      if (dn0) dn0 = probe_down(x, xt0, l0, s_d, s_inv, best0, c0);
      if (dn1) dn1 = probe_down(x + 16, xt1, l1, s_d, s_inv, best1, c1);
    }
  }

  uint32_t w[4];
  enc16(x, s_inv[c0], c0 != 0 && finite_pos(s_d[c0], s_inv[c0]), w);
  enc16(x + 16, s_inv[c1], c1 != 0 && finite_pos(s_d[c1], s_inv[c1]), w + 2);
  if (active) {
    *reinterpret_cast<uint4*>(p.codes + orow * (p.cols >> 1) + (ocol >> 1)) = make_uint4(w[0], w[1], w[2], w[3]);
    const int64_t k = ocol >> 4;
    const uint16_t two = uint16_t(uint32_t(c0) | (uint32_t(c1) << 8));
    if (p.scales) *reinterpret_cast<uint16_t*>(p.scales + orow * (p.cols >> 4) + k) = two;
    if (p.swz) *reinterpret_cast<uint16_t*>(p.swz + swz_offset(orow, k, p.nkb)) = two;
  }

  // <x, u> and <u, u> of the lane's 32 elements, then over the block.
  double num, den;
  {
    float q[32];
#pragma unroll
    for (int k = 0; k < 4; ++k) dec8(w[k], q + 8 * k);
    const float sg0 = e4m3_value(uint32_t(c0)), sg1 = e4m3_value(uint32_t(c1));
    double xu[16], uu[16], h_num[2], h_den[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const double u = double(__fmul_rn(q[16 * h + j], h ? sg1 : sg0));
        xu[j] = __dmul_rn(double(x[16 * h + j]), u);
        uu[j] = __dmul_rn(u, u);
      }
      h_num[h] = tree16d(xu);
      h_den[h] = tree16d(uu);
    }
    num = __dadd_rn(h_num[0], h_num[1]);
    den = __dadd_rn(h_den[0], h_den[1]);
  }
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    num = __dadd_rn(num, __shfl_xor_sync(0xFFFFFFFFu, num, o));
    den = __dadd_rn(den, __shfl_xor_sync(0xFFFFFFFFu, den, o));
  }
  if (lane == 0) { s_num[warp] = num; s_den[warp] = den; }
  __syncthreads();
  if (threadIdx.x == 0) {
    double n4[4], d4[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      n4[i] = __dadd_rn(s_num[2 * i], s_num[2 * i + 1]);
      d4[i] = __dadd_rn(s_den[2 * i], s_den[2 * i + 1]);
    }
    p.partial[blockIdx.x] = make_double2(__dadd_rn(__dadd_rn(n4[0], n4[1]), __dadd_rn(n4[2], n4[3])),
                                         __dadd_rn(__dadd_rn(d4[0], d4[1]), __dadd_rn(d4[2], d4[3])));
  }
}

constexpr int MSE_T_THREADS = 1024;

// One block.  Thread i sums the aligned run of R = P / 1024 leaves (P the
// power of two >= n, leaves >= n zero) as a pairwise tree with a stack of
// completed subtrees (two equal-sized neighbours merge, left + right), then
// the 1024 subtree sums merge level by level in shared memory.  With fewer
// than 1024 leaves, R = 1 and the zero leaves above P leave the value as it is.
__global__ void __launch_bounds__(MSE_T_THREADS) k_mse_tensor(const double2* part, int64_t n, float* ts) {
  __shared__ double sn[MSE_T_THREADS], sd[MSE_T_THREADS];
  int64_t P = 1;
  while (P < n) P <<= 1;
  const int64_t R = P > MSE_T_THREADS ? P / MSE_T_THREADS : 1;
  const int64_t lo = int64_t(threadIdx.x) * R;
  double stn[40], std_[40];
  int64_t ssz[40];
  int top = 0;
  for (int64_t i = 0; i < R; ++i) {
    const int64_t j = lo + i;
    const double2 v = j < n ? part[j] : make_double2(0.0, 0.0);
    stn[top] = v.x; std_[top] = v.y; ssz[top] = 1; ++top;
    while (top >= 2 && ssz[top - 1] == ssz[top - 2]) {
      stn[top - 2] = __dadd_rn(stn[top - 2], stn[top - 1]);
      std_[top - 2] = __dadd_rn(std_[top - 2], std_[top - 1]);
      ssz[top - 2] <<= 1;
      --top;
    }
  }
  sn[threadIdx.x] = stn[0];
  sd[threadIdx.x] = std_[0];
  for (int h = 1; h < MSE_T_THREADS; h <<= 1) {
    __syncthreads();
    if ((threadIdx.x & (2 * h - 1)) == 0) {
      sn[threadIdx.x] = __dadd_rn(sn[threadIdx.x], sn[threadIdx.x + h]);
      sd[threadIdx.x] = __dadd_rn(sd[threadIdx.x], sd[threadIdx.x + h]);
    }
  }
  if (threadIdx.x == 0) {
    const double num = sn[0], den = sd[0];
    if (num > 0.0 && den > 0.0) {
      const float s = __double2float_rn(__ddiv_rn(num, den));
      if (s > 0.0f && absbits(s) < 0x7F800000u) *ts = s;
    }
  }
}

cudaError_t launch_mse_group(const MseParams& p, cudaStream_t s) {
  const int64_t blocks = mse_blocks(p.rows, p.cols);
  if (blocks <= 0) return cudaSuccess;
  if (blocks > 0x7FFFFFFF) return cudaErrorInvalidValue;
  k_mse_group<<<unsigned(blocks), MSE_TASKS, 0, s>>>(p);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_mse_tensor(const double2* partial, int64_t n, float* ts, cudaStream_t s) {
  if (n <= 0) return cudaSuccess;
  k_mse_tensor<<<1, MSE_T_THREADS, 0, s>>>(partial, n, ts);
  count_launch();
  return cudaGetLastError();
}

}  // namespace fp4
