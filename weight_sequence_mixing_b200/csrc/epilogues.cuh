// Fused epilogues of the tcgen05 GEMMs of the bf16 TTT path.
//
// Each functor runs on the epilogue warps of a CTA with one output row per
// thread (TMEM lane = tile row); a warp handles the 32-column chunks
// c % nparts == part and reads them with tcgen05.ld (a warp-collective: every
// thread of the warp executes every load, rows outside the problem only skip
// their stores).
#pragma once
#include <cuda_bf16.h>

#include "tc_gemm.cuh"

namespace ttt {

using bf16 = __nv_bfloat16;

// ------------------------------------------------------------------ helpers
__device__ __forceinline__ float rcp_approx(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
// Standard normal CDF Phi(x) = (1 + erf(x / sqrt 2)) / 2 and density phi(x), with erf from
// Abramowitz & Stegun, Handbook of Mathematical Functions, formula 7.1.26:
//   erf(u) = 1 - t (a1 + t (a2 + t (a3 + t (a4 + t a5)))) exp(-u^2),  t = 1 / (1 + p u),  u >= 0,
// absolute error <= 1.5e-7, far below the bf16 rounding of every GELU output.  With
// u = |x| / sqrt 2, exp(-u^2) = exp(-x^2 / 2) is also the density's exponential, so one
// evaluation serves both.  The coefficients are the published ones; here a1..a5 carry Phi's
// factor 1/2 and p the 1/sqrt 2 of u.
namespace normal_as {
constexpr float kP = 0.3275911f * 0.70710678118654752f;
constexpr float kA1 = 0.5f * 0.254829592f, kA2 = 0.5f * -0.284496736f, kA3 = 0.5f * 1.421413741f,
                kA4 = 0.5f * -1.453152027f, kA5 = 0.5f * 1.061405429f;
constexpr float kNegHalfLog2e = -0.72134752044448170f;  // -log2(e) / 2: exp(-x^2/2) = 2^(x^2 kNegHalfLog2e)
constexpr float kInvSqrt2Pi = 0.39894228040143268f;
}  // namespace normal_as
__device__ __forceinline__ void normal_cdf_pdf(float x, float& cdf, float& pdf) {
  using namespace normal_as;
  const float t = rcp_approx(fmaf(kP, fabsf(x), 1.0f));
  float y = fmaf(kA5, t, kA4);
  y = fmaf(y, t, kA3);
  y = fmaf(y, t, kA2);
  y = fmaf(y, t, kA1);
  y *= t;
  const float e = ex2_approx(x * x * kNegHalfLog2e);
  const float q = y * e;  // Phi(-|x|)
  cdf = x >= 0.0f ? 1.0f - q : q;
  pdf = e * kInvSqrt2Pi;
}
// GELU(x) = x Phi(x)
__device__ __forceinline__ float gelu_dev(float x) {
  float c, p;
  normal_cdf_pdf(x, c, p);
  return x * c;
}
// GELU(x) and its derivative Phi(x) + x phi(x)
__device__ __forceinline__ void gelu_and_grad(float x, float& g, float& gp) {
  float c, p;
  normal_cdf_pdf(x, c, p);
  g = x * c;
  gp = fmaf(x, p, c);
}
// sigma(x) = (1 + tanh(x/2)) / 2 with the hardware tanh approximation (max rel.
// error ~2^-11, below the bf16 rounding the results get)
__device__ __forceinline__ float tanh_approx(float x) {
  float y;
  asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float sigmoid_dev(float x) { return fmaf(0.5f, tanh_approx(0.5f * x), 0.5f); }

// Paired fp32 arithmetic (sm_100: one instruction for two lanes of a float2).
__device__ __forceinline__ unsigned long long f2_bits(float2 v) {
  unsigned long long r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(v.x), "f"(v.y));
  return r;
}
__device__ __forceinline__ float2 bits_f2(unsigned long long r) {
  float2 v;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(v.x), "=f"(v.y) : "l"(r));
  return v;
}
__device__ __forceinline__ float2 mul2(float2 a, float2 b) {
  unsigned long long r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(f2_bits(a)), "l"(f2_bits(b)));
  return bits_f2(r);
}
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
  unsigned long long r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(f2_bits(a)), "l"(f2_bits(b)), "l"(f2_bits(c)));
  return bits_f2(r);
}

// Two GELUs (and derivatives) at once: the same arithmetic as normal_cdf_pdf lane by lane
// (fma.rn / mul.rn per lane give bit-identical results), with the multiplies and adds
// issued as paired fp32 instructions; the reciprocal and exp2 stay per lane.
__device__ __forceinline__ void normal_cdf_pdf2(float2 x, float2& cdf, float2& pdf) {
  using namespace normal_as;
  const float2 den = fma2(make_float2(kP, kP), make_float2(fabsf(x.x), fabsf(x.y)), make_float2(1.0f, 1.0f));
  const float2 t = make_float2(rcp_approx(den.x), rcp_approx(den.y));
  float2 y = fma2(make_float2(kA5, kA5), t, make_float2(kA4, kA4));
  y = fma2(y, t, make_float2(kA3, kA3));
  y = fma2(y, t, make_float2(kA2, kA2));
  y = fma2(y, t, make_float2(kA1, kA1));
  y = mul2(y, t);
  const float2 a = mul2(mul2(x, x), make_float2(kNegHalfLog2e, kNegHalfLog2e));
  const float2 e = make_float2(ex2_approx(a.x), ex2_approx(a.y));
  const float2 q = mul2(y, e);
  cdf = make_float2(x.x >= 0.0f ? 1.0f - q.x : q.x, x.y >= 0.0f ? 1.0f - q.y : q.y);
  pdf = mul2(e, make_float2(kInvSqrt2Pi, kInvSqrt2Pi));
}
__device__ __forceinline__ float2 gelu2(float2 x) {
  float2 c, p;
  normal_cdf_pdf2(x, c, p);
  return mul2(x, c);
}
__device__ __forceinline__ void gelu_and_grad2(float2 x, float2& g, float2& gp) {
  float2 c, p;
  normal_cdf_pdf2(x, c, p);
  g = mul2(x, c);
  gp = fma2(x, p, c);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&v);
}

// 32 floats -> 32 bf16 at a 16-byte aligned address
__device__ __forceinline__ void store_bf16x32(bf16* dst, const float (&v)[32]) {
  uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint4 u;
    u.x = pack_bf16x2(v[8 * q + 0], v[8 * q + 1]);
    u.y = pack_bf16x2(v[8 * q + 2], v[8 * q + 3]);
    u.z = pack_bf16x2(v[8 * q + 4], v[8 * q + 5]);
    u.w = pack_bf16x2(v[8 * q + 6], v[8 * q + 7]);
    d4[q] = u;
  }
}

__device__ __forceinline__ void load_bf16x32(const bf16* src, float (&v)[32]) {
  const uint4* s4 = reinterpret_cast<const uint4*>(src);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint4 u = s4[q];
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      __nv_bfloat162 p = *reinterpret_cast<const __nv_bfloat162*>(&w[j]);
      float2 f = __bfloat1622float2(p);
      v[8 * q + 2 * j] = f.x;
      v[8 * q + 2 * j + 1] = f.y;
    }
  }
}

__device__ __forceinline__ void store_f32x32(float* dst, const float (&v)[32]) {
  float4* d4 = reinterpret_cast<float4*>(dst);
#pragma unroll
  for (int q = 0; q < 8; ++q) d4[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
}

__device__ __forceinline__ void load_f32x32(const float* src, float (&v)[32]) {
  const float4* s4 = reinterpret_cast<const float4*>(src);
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    float4 f = s4[q];
    v[4 * q] = f.x;
    v[4 * q + 1] = f.y;
    v[4 * q + 2] = f.z;
    v[4 * q + 3] = f.w;
  }
}

__device__ __forceinline__ void zero32(float (&v)[32]) {
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = 0.0f;
}

// ------------------------------------------------------------------ split-K partials
// out[split][z][row0_p + m][n] (fp32), rows_p valid rows of problem p; N columns.
struct EpiPartial {
  float* out;
  int64_t split_stride, z_stride;  // elements
  int ld;                          // row length (= N)
  int row0[2], rows[2];
  template <int BN0, int BN1>
  __device__ void run(const EpiCtx& c) const {
    const bool ok = c.m < rows[c.problem];
    float* rowp = out + c.split * split_stride + c.z * z_stride + int64_t(row0[c.problem] + c.m) * ld + c.n0;
#pragma unroll 1
    for (int cc = 32 * c.part; cc < BN0; cc += 32 * c.nparts) {
      float v[32];
      tmem_ld32(c.taddr + cc, v);
      if (ok && c.n0 + cc < ld) store_f32x32(rowp + cc, v);
    }
  }
};

// Unsplit weight gradients straight into the optimizer state (no partials): for
// gradient-layout row r and column n, U = beta M + G and M = U (momentum) or U = G,
// and the squared row norms Muon needs (rowsq, zeroed beforehand; at most two
// warps add to a row, so the sum does not depend on their order).
struct EpiGradDirect {
  float* U;
  float* M;      // momentum buffer or null
  float* rowsq;  // or null
  float beta;
  int64_t z_stride;  // elements per batch entry (GR * ld)
  int ld;            // d
  int row0[2], rows[2];
  // > 0: problem 0 is G2^T (rows [0, w2t_h) of the gradient layout) and its update goes into
  // the same h * d elements of U transposed, as [d][h] (W2's orientation), so that the row
  // finish reads W2's update rows contiguously; the momentum keeps the gradient layout.  The
  // lanes of a warp hold consecutive rows, so each transposed store is one 128-byte run.
  int w2t_h;
  template <int BN0, int BN1>
  __device__ void run(const EpiCtx& c) const {
    const bool ok = c.m < rows[c.problem];
    const int64_t off = c.z * z_stride + int64_t(row0[c.problem] + c.m) * ld + c.n0;
    const bool w2t = w2t_h > 0 && c.problem == 0;
    float sq = 0.0f;
#pragma unroll 1
    for (int cc = 32 * c.part; cc < BN0; cc += 32 * c.nparts) {
      float v[32];
      tmem_ld32(c.taddr + cc, v);
      if (!ok || c.n0 + cc >= ld) continue;
      if (M) {
        float mv[32];
        load_f32x32(M + off + cc, mv);
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = beta * mv[j] + v[j];
        store_f32x32(M + off + cc, v);
      }
      if (w2t) {
        float* ut = U + c.z * z_stride + int64_t(c.n0 + cc) * w2t_h + row0[0] + c.m;
#pragma unroll
        for (int j = 0; j < 32; ++j) ut[int64_t(j) * w2t_h] = v[j];
      } else {
        store_f32x32(U + off + cc, v);
      }
#pragma unroll
      for (int j = 0; j < 32; ++j) sq += v[j] * v[j];
    }
    if (rowsq && ok) atomicAdd(rowsq + c.z * (z_stride / ld) + row0[c.problem] + c.m, sq);
  }
};

// ------------------------------------------------------------------ token phase, MSE (MLP2)
// Z = X W1^T tile: H = GELU(Z) and G' = GELU'(Z) (bf16), zeros past the chunk.
struct EpiGeluSave {
  bf16* H;
  bf16* Gp;
  int ld;  // h
  int rows_valid;
  int64_t zs;
  template <int BN0, int BN1>
  __device__ void run(const EpiCtx& c) const {
    const bool valid = c.m < rows_valid;
    bf16* hrow = H + c.z * zs + int64_t(c.m) * ld + c.n0;
    bf16* grow = Gp + c.z * zs + int64_t(c.m) * ld + c.n0;
#pragma unroll 1
    for (int cc = 32 * c.part; cc < BN0; cc += 32 * c.nparts) {
      float v[32], a[32], g[32];
      tmem_ld32(c.taddr + cc, v);
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        float gz, gpz;
        gelu_and_grad(v[j], gz, gpz);
        a[j] = valid ? gz : 0.0f;
        g[j] = valid ? gpz : 0.0f;
      }
      store_bf16x32(hrow + cc, a);
      store_bf16x32(grow + cc, g);
    }
  }
};

// V_hat tile -> dL/dV_hat = coef * eta_t * (V_hat - V) (MSE, mean over the chunk's
// n*d elements: coef = 2/(n d)); zeros past the chunk.
struct EpiMseGrad {
  bf16* dY;
  int d;
  int rows_valid;
  int64_t zs;
  const bf16* V;  // [z][N][d]
  int64_t v_zs;
  int t0;
  const float* eta;
  int64_t eta_zs;
  float eta_scalar, coef;
  template <int BN0, int BN1>
  __device__ void run(const EpiCtx& c) const {
    const bool valid = c.m < rows_valid;
    const float e = valid ? (eta ? eta[c.z * eta_zs + t0 + c.m] : eta_scalar) * coef : 0.0f;
    bf16* yrow = dY + c.z * zs + int64_t(c.m) * d + c.n0;
    const bf16* vrow = V + c.z * v_zs + int64_t(t0 + (valid ? c.m : 0)) * d + c.n0;
#pragma unroll 1
    for (int cc = 32 * c.part; cc < BN0; cc += 32 * c.nparts) {
      float v[32], t[32];
      tmem_ld32(c.taddr + cc, v);
      if (c.n0 + cc >= d) continue;
      if (valid) load_bf16x32(vrow + cc, t);
      else zero32(t);
#pragma unroll
      for (int j = 0; j < 32; ++j) v[j] = e * (v[j] - t[j]);
      store_bf16x32(yrow + cc, v);
    }
  }
};

// dH tile -> dZ = dH * G' (G' saved by EpiGeluSave)
struct EpiMulSaved {
  bf16* dZ;
  const bf16* Gp;
  int ld;
  int64_t zs;
  template <int BN0, int BN1>
  __device__ void run(const EpiCtx& c) const {
    bf16* zrow = dZ + c.z * zs + int64_t(c.m) * ld + c.n0;
    const bf16* grow = Gp + c.z * zs + int64_t(c.m) * ld + c.n0;
#pragma unroll 1
    for (int cc = 32 * c.part; cc < BN0; cc += 32 * c.nparts) {
      float v[32], g[32];
      tmem_ld32(c.taddr + cc, v);
      load_bf16x32(grow + cc, g);
#pragma unroll
      for (int j = 0; j < 32; ++j) v[j] *= g[j];
      store_bf16x32(zrow + cc, v);
    }
  }
};

// ------------------------------------------------------------------ apply on queries
// First layer of F_W(Q): SwiGLU tiles hold [z1 (128) | z3 (128)] of hidden block
// n0/256 -> H = SiLU(z1) z3; MLP2 tiles hold z -> H = GELU(z).  Rows >= rows_valid skipped.
template <bool SWIGLU>
struct EpiApplyAct {
  bf16* Hq;
  int h;
  int rows_valid;
  int64_t zs;
  template <int BN0, int BN1>
  __device__ void run(const EpiCtx& c) const {
    const bool valid = c.m < rows_valid;
    if constexpr (SWIGLU) {
      bf16* row = Hq + c.z * zs + int64_t(c.m) * h + (c.n0 / BN0) * 128;
#pragma unroll 1
      for (int cc = 32 * c.part; cc < 128; cc += 32 * c.nparts) {
        float z1[32], z3[32];
        tmem_ld32(c.taddr + cc, z1);
        tmem_ld32(c.taddr + 128 + cc, z3);
#pragma unroll
        for (int j = 0; j < 32; ++j) z1[j] = z1[j] * sigmoid_dev(z1[j]) * z3[j];
        if (valid) store_bf16x32(row + cc, z1);
      }
    } else {
      bf16* row = Hq + c.z * zs + int64_t(c.m) * h + c.n0;
#pragma unroll 1
      for (int cc = 32 * c.part; cc < BN0; cc += 32 * c.nparts) {
        float z[32];
        tmem_ld32(c.taddr + cc, z);
#pragma unroll
        for (int j = 0; j < 32; ++j) z[j] = gelu_dev(z[j]);
        if (valid && c.n0 + cc < h) store_bf16x32(row + cc, z);
      }
    }
  }
};

// Output rows of O (row0 + m for m < rows_valid), bf16 or fp32, with the
// non-finite check of the layer's output.
template <typename OutT>
struct EpiStoreOut {
  OutT* O;
  int d;
  int rows_valid, row0;
  int64_t zs;
  unsigned* status;
  template <int BN0, int BN1>
  __device__ void run(const EpiCtx& c) const {
    const bool valid = c.m < rows_valid;
    OutT* row = O + c.z * zs + int64_t(row0 + c.m) * d + c.n0;
    bool bad = false;
#pragma unroll 1
    for (int cc = 32 * c.part; cc < BN0; cc += 32 * c.nparts) {
      float v[32];
      tmem_ld32(c.taddr + cc, v);
      if (!valid || c.n0 + cc >= d) continue;
#pragma unroll
      for (int j = 0; j < 32; ++j) bad |= !isfinite(v[j]);
      if constexpr (sizeof(OutT) == 2) store_bf16x32(reinterpret_cast<bf16*>(row + cc), v);
      else store_f32x32(reinterpret_cast<float*>(row + cc), v);
    }
    if (bad) set_status(status, kStatusNonFinite);
  }
};

}  // namespace ttt
