// Validation, chunking and workspace carving of a TTT layer configuration.
#include <cmath>

#include "ttt_plan.cuh"

namespace ttt {

static size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

int plan_build(const ttt_config& c, Plan* p) {
  if (c.B < 1 || c.H < 1 || c.N < 1 || c.Nq < 1 || c.d < 1) return TTT_ERR_INVALID_ARG;
  if (c.inner < TTT_INNER_LINEAR || c.inner > TTT_INNER_GLU) return TTT_ERR_INVALID_ARG;
  if (c.loss < TTT_LOSS_MSE || c.loss > TTT_LOSS_RMSE) return TTT_ERR_INVALID_ARG;
  if (c.opt < TTT_OPT_GD || c.opt > TTT_OPT_MOMENTUM_MUON) return TTT_ERR_INVALID_ARG;
  if (c.dtype != TTT_F32 && c.dtype != TTT_BF16) return TTT_ERR_INVALID_ARG;
  if (c.causal != 0 && c.causal != 1) return TTT_ERR_INVALID_ARG;
  if (c.causal && c.Nq != c.N) return TTT_ERR_INVALID_ARG;
  const bool dw = c.inner == TTT_INNER_DWCONV;
  if ((c.inner == TTT_INNER_MLP2_GELU || c.inner == TTT_INNER_SWIGLU) && c.h < 1) return TTT_ERR_INVALID_ARG;
  // the GLU runs on the tensor-core path only (the fp32 path runs it as a SwiGLU with h = d,
  // W2 = I and TTT_FLAG_FIRST_LAYER_ONLY)
  if (c.inner == TTT_INNER_GLU && c.dtype != TTT_BF16) return TTT_ERR_UNSUPPORTED;
  if (dw) {
    if (c.ksize < 1 || c.ksize > 7 || c.ksize % 2 == 0 || c.grid_h < 1 || c.grid_w < 1 ||
        static_cast<int64_t>(c.grid_h) * c.grid_w != c.N || c.Nq != c.N)
      return TTT_ERR_INVALID_ARG;
    // the grid is one non-causal chunk; the combinations built for it
    if (c.causal || (c.chunk > 0 && c.chunk < c.N) || (c.flags & TTT_FLAG_KEY_INSTNORM) ||
        (c.loss != TTT_LOSS_MSE && c.loss != TTT_LOSS_NEG_DOT) || (c.opt != TTT_OPT_GD && c.opt != TTT_OPT_MOMENTUM))
      return TTT_ERR_UNSUPPORTED;
  }
  if ((c.flags & ~(TTT_FLAG_KEY_INSTNORM | TTT_FLAG_WEIGHT_L2NORM | TTT_FLAG_DIRECT_LAUNCH |
                   TTT_FLAG_SINGLE_CTA | TTT_FLAG_W0_PER_BATCH | TTT_FLAG_NO_UPDATE |
                   TTT_FLAG_FIRST_LAYER_ONLY)) != 0)
    return TTT_ERR_INVALID_ARG;
  if (c.ns_iters < 0 || c.ns_iters > 100) return TTT_ERR_INVALID_ARG;
  if (c.epochs < 0 || c.epochs > 64) return TTT_ERR_INVALID_ARG;
  if (!std::isfinite(c.eta_scalar) || !std::isfinite(c.lr) || !std::isfinite(c.momentum) ||
      !std::isfinite(c.in_eps) || c.in_eps < 0.0f)
    return TTT_ERR_INVALID_ARG;
  for (float v : c.ns_coeff)
    if (!std::isfinite(v)) return TTT_ERR_INVALID_ARG;
  if (static_cast<int64_t>(c.B) * c.H > 65535) return TTT_ERR_UNSUPPORTED;
  // token counts: 2^30 keys of even 64 bf16 channels already outgrow HBM; the bound keeps
  // every padded token count inside int32
  if (c.N > (1 << 30) || c.Nq > (1 << 30)) return TTT_ERR_UNSUPPORTED;
  if (c.d > 4096 || ((c.inner == TTT_INNER_MLP2_GELU || c.inner == TTT_INNER_SWIGLU) && c.h > 16384))
    return TTT_ERR_UNSUPPORTED;

  p->cfg = c;
  p->epochs = c.epochs == 0 ? 1 : c.epochs;
  const int64_t d = c.d, h = (c.inner == TTT_INNER_LINEAR || c.inner == TTT_INNER_GLU || dw) ? c.d : c.h;
  p->cfg.h = static_cast<int32_t>(h);
  p->P = dw ? d * c.ksize * c.ksize
            : c.inner == TTT_INNER_LINEAR ? d * d
            : c.inner == TTT_INNER_GLU    ? 2 * d * d
            : c.inner == TTT_INNER_MLP2_GELU ? 2 * d * h
                                             : 3 * d * h;
  p->BH = c.B * c.H;
  p->chunk = (c.chunk <= 0 || c.chunk >= c.N) ? c.N : c.chunk;
  p->nchunks = static_cast<int>((static_cast<int64_t>(c.N) + p->chunk - 1) / p->chunk);
  p->path = dw ? kPathDwconv : c.dtype == TTT_F32 ? kPathF32 : kPathBf16;

  // host staging: inputs then outputs, each 256-byte aligned
  const size_t es = c.dtype == TTT_F32 ? 4 : 2;
  size_t o = 0;
  p->stg_q = o; o = align_up(o + size_t(p->BH) * c.Nq * d * es, 256);
  p->stg_k = o; o = align_up(o + size_t(p->BH) * c.N * d * es, 256);
  p->stg_v = o; o = align_up(o + size_t(p->BH) * c.N * d * es, 256);
  p->stg_eta = o; o = align_up(o + size_t(p->BH) * c.N * 4, 256);
  p->stg_w0 = o; o = align_up(o + size_t((c.flags & TTT_FLAG_W0_PER_BATCH) ? p->BH : c.H) * p->P * 4, 256);
  p->stg_o = o; o = align_up(o + size_t(p->BH) * c.Nq * d * es, 256);
  p->stg_w = o; o = align_up(o + size_t(p->BH) * p->P * 4, 256);
  p->staging_bytes = o;

  return p->path == kPathDwconv ? plan_layout_dwconv(p)
         : p->path == kPathF32  ? plan_layout_f32(p)
                                : plan_layout_bf16(p);
}

int plan_run(const Plan& p, const Io& io, void* ws, cudaStream_t st) {
  if (cudaMemsetAsync(ws, 0, 256, st) != cudaSuccess) return TTT_ERR_CUDA;  // status word
  return p.path == kPathDwconv ? run_dwconv(p, io, ws, st)
         : p.path == kPathF32  ? run_f32(p, io, ws, st)
                               : run_bf16(p, io, ws, st);
}

}  // namespace ttt
