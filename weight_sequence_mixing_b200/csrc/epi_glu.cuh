// GEMM epilogues of the simplified GLU inner model F(x) = (x Wa^T) * SiLU(x Wb^T) (ViT3
// digest, section 03, inner-model table: FC(x) * SiLU(FC(x)), ViT3's F1 module; two d x d
// matrices, no biases, no output projection).
//
// Both run on tiles of Z = X [Wb_blk; Wa_blk]^T: the first-layer copy of the weights
// stores, per block of 64 output channels, the 64 gate rows (Wb) and then the 64
// linear rows (Wa), so a 128-column tile holds zb (columns 0..63) and za (64..127) of
// the same 64 channels j = 64 blk + c.
#pragma once
#include "epilogues.cuh"

namespace ttt {

// Token phase of the update: per key token t and channel j, with F_j = za_j SiLU(zb_j),
//   dF_j = -eta_t v_tj                          (negative dot loss)
//   dF_j = coef eta_t (F_j - v_tj)              (MSE, coef = 2 / (n d))
//   dZa_j = dF_j SiLU(zb_j),  dZb_j = dF_j za_j SiLU'(zb_j)
// written in bf16 to dZ [z][C][2d] in the first-layer row order (gate block, then linear
// block), zeros past the chunk, for the weight-gradient reduction G = dZ^T X.
struct EpiGluGrad {
  bf16* dZ;
  int d;           // channels
  int rows_valid;  // chunk tokens
  int64_t zs;      // dZ elements per head
  const bf16* V;   // [z][N][d]
  int64_t v_zs;
  int t0;
  const float* eta;
  int64_t eta_zs;
  float eta_scalar;
  int mse;
  float coef;
  template <int BN0, int BN1>
  __device__ void run(const EpiCtx& c) const {
    static_assert(BN0 == 128 && BN1 == 0, "a tile holds one 64-channel block: gate and linear halves");
    const bool valid = c.m < rows_valid;
    const float e = valid ? (eta ? eta[c.z * eta_zs + t0 + c.m] : eta_scalar) : 0.0f;
    const int ch0 = (c.n0 / 128) * 64;  // first channel of the block
    bf16* zrow = dZ + c.z * zs + int64_t(c.m) * (2 * d) + c.n0;
    const bf16* vrow = V + c.z * v_zs + int64_t(t0 + (valid ? c.m : 0)) * d + ch0;
#pragma unroll 1
    for (int cc = 32 * c.part; cc < 64; cc += 32 * c.nparts) {
      float zb[32], za[32], v[32];
      tmem_ld32(c.taddr + cc, zb);
      tmem_ld32(c.taddr + 64 + cc, za);
      if (valid) load_bf16x32(vrow + cc, v);
      else zero32(v);
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const float s = sigmoid_dev(zb[i]);
        const float silu = zb[i] * s;
        const float df = mse ? coef * e * (za[i] * silu - v[i]) : -e * v[i];
        const float ga = df * silu;                                     // dZa
        const float gb = df * za[i] * s * fmaf(zb[i], 1.0f - s, 1.0f);  // dZb
        zb[i] = valid ? gb : 0.0f;
        za[i] = valid ? ga : 0.0f;
      }
      store_bf16x32(zrow + cc, zb);
      store_bf16x32(zrow + 64 + cc, za);
    }
  }
};

// Apply: O[t][j] = za_j SiLU(zb_j) for query rows row0 + m (m < rows_valid), with the
// non-finite check of the layer's output.
struct EpiGluOut {
  bf16* O;
  int d;
  int rows_valid, row0;
  int64_t zs;
  unsigned* status;
  template <int BN0, int BN1>
  __device__ void run(const EpiCtx& c) const {
    static_assert(BN0 == 128 && BN1 == 0, "a tile holds one 64-channel block: gate and linear halves");
    const bool valid = c.m < rows_valid;
    bf16* row = O + c.z * zs + int64_t(row0 + c.m) * d + (c.n0 / 128) * 64;
    bool bad = false;
#pragma unroll 1
    for (int cc = 32 * c.part; cc < 64; cc += 32 * c.nparts) {
      float zb[32], za[32];
      tmem_ld32(c.taddr + cc, zb);
      tmem_ld32(c.taddr + 64 + cc, za);
      if (!valid) continue;
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        za[i] = za[i] * zb[i] * sigmoid_dev(zb[i]);
        bad |= !isfinite(za[i]);
      }
      store_bf16x32(row + cc, za);
    }
    if (bad) set_status(status, kStatusNonFinite);
  }
};

}  // namespace ttt
