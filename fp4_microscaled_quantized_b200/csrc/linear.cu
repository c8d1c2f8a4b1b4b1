// Linear-layer orchestration over the C ABI (host code): forward quantise +
// GEMM, backward transposed quantise / re-quantise + two GEMMs, all issued on
// the caller's stream with caller-owned memory.
#include "../../include/fp4.h"

namespace {

constexpr uint32_t TAG_E_ROW = 1, TAG_W_T = 2, TAG_E_T = 3, TAG_X_T = 4, TAG_X = 5, TAG_W = 6;
constexpr uint32_t GEMM_DX = 0, GEMM_DW = 1;

inline size_t a256(size_t n) { return (n + 255) & ~size_t(255); }
inline int group_of(int fmt) { return fmt == FP4_NVFP4 ? 16 : 32; }

// Device bytes of one quantised operand without linear scales or mask.
struct Operand {
  size_t codes, swz, ts, total;
};

Operand operand_bytes(int64_t rows, int64_t cols, int fmt) {
  Operand o;
  o.codes = a256(size_t(rows) * size_t(cols / 2));
  o.swz = a256(fp4_swizzled_scale_bytes(rows, cols / group_of(fmt)));
  o.ts = 256;
  o.total = o.codes + o.swz + o.ts;
  return o;
}

fp4_qtensor carve(uint8_t*& p, int64_t rows, int64_t cols, int fmt) {
  Operand o = operand_bytes(rows, cols, fmt);
  fp4_qtensor q{};
  q.codes = p;
  q.scales_swz = p + o.codes;
  q.tensor_scale = reinterpret_cast<float*>(p + o.codes + o.swz);
  q.rows = rows; q.cols = cols; q.fmt = fmt;
  p += o.total;
  return q;
}

size_t quant_ws_bwd(const fp4_recipe* r, int64_t M, int64_t N, int64_t K) {
  size_t w = 0;
  const int64_t shapes[4][2] = {{M, N}, {K, N}, {N, M}, {K, M}};
  for (auto& s : shapes) {
    size_t b = fp4_quantize_workspace_size(s[0], s[1], r->fmt, r->bwd_rounding, r->bwd_had);
    w = b > w ? b : w;
  }
  return a256(w);
}

size_t quant_ws_fwd(const fp4_recipe* r, int64_t M, int64_t N, int64_t K) {
  size_t a = fp4_quantize_workspace_size(M, K, r->fmt, r->fwd_rounding, r->fwd_had);
  const int w_rnd = r->w_rounding >= 0 ? r->w_rounding : r->fwd_rounding;
  size_t b = fp4_quantize_workspace_size(N, K, r->fmt, w_rnd, r->fwd_had);
  return a256(a > b ? a : b);
}

bool recipe_ok(const fp4_recipe* r) {
  if (!r) return false;
  if (r->fmt != FP4_MXFP4 && r->fmt != FP4_NVFP4) return false;
  if (r->out_y < 0 || r->out_y > 1 || r->out_dx < 0 || r->out_dx > 1 || r->out_dw < 0 || r->out_dw > 1)
    return false;
  if (r->mask_epilogue && (r->fwd_rounding != FP4_QUEST || r->fwd_had != 32)) return false;
  if (r->w_rounding < -1 || r->w_rounding > FP4_RTN_SQUARE16) return false;
  if (r->w_reuse && (r->w_rounding != FP4_RTN_SQUARE16 || r->fmt != FP4_NVFP4 || r->mask_epilogue)) return false;
  return true;
}

}  // namespace

extern "C" {

int fp4_recipe_preset(int32_t id, fp4_recipe* r) {
  if (!r) return FP4_ERR_INVALID_ARG;
  switch (id) {
    case FP4_RECIPE_QUARTET:
      *r = fp4_recipe{FP4_MXFP4, FP4_QUEST, 32, FP4_SR, 32, 1, 1, 0, 0, 0, -1, 0};
      return FP4_OK;
    case FP4_RECIPE_QUARTET2:
      *r = fp4_recipe{FP4_NVFP4, FP4_FOUR_OVER_SIX, 0, FP4_MS_EDEN, 128, 1, 0, 0, 0, 0, -1, 0};
      return FP4_OK;
    case FP4_RECIPE_RTN:
      *r = fp4_recipe{FP4_NVFP4, FP4_RTN, 0, FP4_RTN, 0, 0, 0, 0, 0, 0, -1, 0};
      return FP4_OK;
    case FP4_RECIPE_TETRAJET2:
      *r = fp4_recipe{FP4_NVFP4, FP4_RTN, 0, FP4_SR, 128, 1, 0, 0, 0, 0, -1, 0};
      return FP4_OK;
    case FP4_RECIPE_NVIDIA:
      *r = fp4_recipe{FP4_NVFP4, FP4_RTN, 0, FP4_SR, 16, 1, 0, 0, 0, 0, FP4_RTN_SQUARE16, 1};
      return FP4_OK;
    default:
      return FP4_ERR_INVALID_ARG;
  }
}

size_t fp4_linear_workspace_size(const fp4_recipe* r, int64_t M, int64_t N, int64_t K, int32_t is_bwd) {
  if (!recipe_ok(r) || M < 0 || N < 0 || K < 0) return 0;
  if (!is_bwd) return quant_ws_fwd(r, M, N, K);
  return quant_ws_bwd(r, M, N, K) + operand_bytes(M, N, r->fmt).total + operand_bytes(K, N, r->fmt).total +
         operand_bytes(N, M, r->fmt).total + operand_bytes(K, M, r->fmt).total;
}

int fp4_linear_fwd(const void* X, const void* W, int64_t M, int64_t N, int64_t K, const fp4_recipe* r,
                   uint64_t seed, void* Y, fp4_ctx* ctx, void* ws, size_t ws_bytes, fp4_stream_t s) {
  if (!recipe_ok(r) || !ctx) return FP4_ERR_INVALID_ARG;
  if (M < 0 || N < 0 || K < 0) return FP4_ERR_INVALID_ARG;
  const size_t need = quant_ws_fwd(r, M, N, K);
  if (need && (!ws || ws_bytes < need)) return FP4_ERR_WORKSPACE;
  const int g = group_of(r->fmt);
  const fp4_had h{r->fwd_had, 0, 0};
  int st = fp4_quantize(X, M, K, 0, r->fmt, r->fwd_rounding, g, h, seed, TAG_X, &ctx->xq, ws, ws_bytes, s);
  if (st) return st;
  const int w_rnd = r->w_rounding >= 0 ? r->w_rounding : r->fwd_rounding;
  st = fp4_quantize(W, N, K, 0, r->fmt, w_rnd, g, h, seed, TAG_W, &ctx->wq, ws, ws_bytes, s);
  if (st) return st;
  return fp4_gemm(&ctx->xq, &ctx->wq, Y, r->out_y, nullptr, 0, s);
}

int fp4_linear_bwd(const void* dY, const fp4_ctx* ctx, int64_t M, int64_t N, int64_t K, const fp4_recipe* r,
                   uint64_t step_seed, void* dX, void* dW, void* ws, size_t ws_bytes, fp4_stream_t s) {
  if (!recipe_ok(r) || !ctx || !dY) return FP4_ERR_INVALID_ARG;
  if (ctx->xq.rows != M || ctx->xq.cols != K || ctx->wq.rows != N || ctx->wq.cols != K)
    return FP4_ERR_INVALID_ARG;
  const size_t qws = quant_ws_bwd(r, M, N, K);
  const size_t need = fp4_linear_workspace_size(r, M, N, K, 1);
  if (!ws || ws_bytes < need) return FP4_ERR_WORKSPACE;
  uint8_t* p = static_cast<uint8_t*>(ws);
  void* qw = p;
  p += qws;
  fp4_qtensor e_row = carve(p, M, N, r->fmt), w_t = carve(p, K, N, r->fmt);
  fp4_qtensor e_t = carve(p, N, M, r->fmt), x_t = carve(p, K, M, r->fmt);
  const int g = group_of(r->fmt);
  const int rz = r->bwd_randomized ? 1 : 0;
  const int inv_h = r->mask_epilogue ? r->fwd_had : 0;
  int st;
  if (dX) {
    if (r->w_reuse) {
      // the forward Q(W) itself, transposed; dY without a rotation to match it
      const fp4_had h0{0, 0, GEMM_DX};
      st = fp4_quantize(dY, M, N, 0, r->fmt, r->bwd_rounding, g, h0, step_seed, TAG_E_ROW, &e_row, qw, qws, s);
      if (st) return st;
      st = fp4_transpose_square16(&ctx->wq, &w_t, s);
      if (st) return st;
    } else {
      const fp4_had h{r->bwd_had, rz, GEMM_DX};
      st = fp4_quantize(dY, M, N, 0, r->fmt, r->bwd_rounding, g, h, step_seed, TAG_E_ROW, &e_row, qw, qws, s);
      if (st) return st;
      st = fp4_requantize(&ctx->wq, 1, r->bwd_rounding, h, step_seed, TAG_W_T, &w_t, qw, qws, s);
      if (st) return st;
    }
    st = fp4_gemm(&e_row, &w_t, dX, r->out_dx, r->mask_epilogue ? ctx->xq.mask : nullptr, inv_h, s);
    if (st) return st;
  }
  if (dW) {
    const fp4_had h{r->bwd_had, rz, GEMM_DW};
    st = fp4_quantize(dY, M, N, 1, r->fmt, r->bwd_rounding, g, h, step_seed, TAG_E_T, &e_t, qw, qws, s);
    if (st) return st;
    st = fp4_requantize(&ctx->xq, 1, r->bwd_rounding, h, step_seed, TAG_X_T, &x_t, qw, qws, s);
    if (st) return st;
    st = fp4_gemm(&e_t, &x_t, dW, r->out_dw, r->mask_epilogue ? ctx->wq.mask : nullptr, inv_h, s);
    if (st) return st;
  }
  return FP4_OK;
}

}  // extern "C"
