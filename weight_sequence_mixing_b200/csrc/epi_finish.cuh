// Weight-gradient epilogue that also finishes the weights (the plain-step and
// momentum optimizers, unsplit token reductions, rows that fit one output tile).
//
// The causal language layer takes a step after every 2048-token chunk; with the
// gradient, the optimizer and the row norm in separate launches the step is a
// chain of short kernels.  When a tile holds whole rows of the weights (N = d = h
// <= 256) its epilogue can do all of it: for each row
//   U = G (+ beta M, stored back as M),  W <- W - lr U,  W <- W / max(||W||, 1e-12)
// and then write the fp32 master row and the bf16 copies the next chunk's GEMMs read
// (the first layer [W1 blk | W3 blk] rows, W2 rows and W2^T columns).  The order of
// the update is the optimizer's (LaCT analysis, "Nonlinear memory complements local
// attention": gradient, momentum, step, L2 normalisation).
//
// Rows: problem 0 = G2 = V^T H' (rows of W2, length h); problem 1 = G13 = dZ13^T X
// (SwiGLU: 128-row blocks [W1 | W3], MLP2: rows of W1; length d).  One epilogue warp
// per TMEM lane quarter, so each thread owns one whole row.
#pragma once
#include "epilogues.cuh"

namespace ttt {

struct EpiGradFinish {
  float* Wf;        // fp32 master weights [Z][P] (canonical packed layout)
  float* M;         // momentum [Z][GR][d] in this epilogue's row order, or null
  bf16* First;      // [Z][R1][d]
  bf16* W2;         // [Z][d][h]
  bf16* W2T;        // [Z][h][d]
  unsigned* status;
  int64_t P;
  int d, h, R1, GR;
  int swiglu;
  float beta, lr;
  int rownorm, hold_w2;
  int row0[2], rows[2];

  template <int BN0, int BN1>
  __device__ void run(const EpiCtx& c) const {
    static_assert(BN1 == 0, "one product per tile");
    const bool ok = c.m < rows[c.problem];
    const bool w2 = c.problem == 0;
    const int r = c.m;
    // canonical row of the fp32 master weights, its length, and the bf16 first-layer row
    int64_t off;
    int len;
    if (w2) {
      off = (swiglu ? 2 : 1) * int64_t(h) * d + int64_t(r) * h;
      len = h;
    } else if (swiglu) {
      const int blk = r / 256, within = r % 256;
      const int k = within < 128 ? 0 : 1;  // W1 or W3
      off = int64_t(k) * h * d + int64_t(blk * 128 + within % 128) * d;
      len = d;
    } else {
      off = int64_t(r) * d;
      len = d;
    }
    float* w = Wf + c.z * P + off;
    float* mom = M ? M + (c.z * int64_t(GR) + row0[c.problem] + r) * d : nullptr;
    const bool hold = w2 && hold_w2;
    float sq = 0.0f;
    // pass 1: U, momentum, the step (every lane takes part in the TMEM loads)
#pragma unroll 1
    for (int cc = 0; cc < BN0; cc += 32) {
      float v[32];
      tmem_ld32(c.taddr + cc, v);
      if (!ok || cc >= len) continue;
      if (mom) {  // (a held W2 keeps its momentum too, as the separate optimizer kernels do)
        float mv[32];
        load_f32x32(mom + cc, mv);
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = beta * mv[j] + v[j];
        store_f32x32(mom + cc, v);
      }
      if (hold) continue;
      float wv[32];
      load_f32x32(w + cc, wv);
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        wv[j] -= lr * v[j];
        sq += wv[j] * wv[j];
      }
      store_f32x32(w + cc, wv);
    }
    if (!ok) return;
    // pass 2: row norm, bf16 copies, non-finite check
    const float inv = (rownorm && !hold) ? 1.0f / fmaxf(sqrtf(sq), 1e-12f) : 1.0f;
    bf16* brow = w2 ? W2 + (c.z * int64_t(d) + r) * h : First + (c.z * int64_t(R1) + r) * d;
    bool bad = false;
#pragma unroll 1
    for (int cc = 0; cc < len; cc += 32) {
      float wv[32];
      load_f32x32(w + cc, wv);
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        wv[j] *= inv;
        bad |= !isfinite(wv[j]);
      }
      if (inv != 1.0f) store_f32x32(w + cc, wv);
      store_bf16x32(brow + cc, wv);
      if (w2) {
        // W2^T[j][r]: the warp's lanes are consecutive rows r, so each store is coalesced
        bf16* col = W2T + (c.z * int64_t(h) + cc) * d + r;
#pragma unroll
        for (int j = 0; j < 32; ++j) col[int64_t(j) * d] = __float2bfloat16_rn(wv[j]);
      }
    }
    if (bad) set_status(status, kStatusNonFinite);
  }
};

}  // namespace ttt
