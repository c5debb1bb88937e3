// fp32 path of the TTT layer: every step in fp32 on the CUDA cores (FFMA).
//
// tcgen05 has no exact-fp32 input kind (tf32 keeps 10 mantissa bits), so the
// fp32 layer runs its contractions as tiled SIMT GEMMs.  It implements every
// inner model, loss and optimizer of the C ABI and serves small layers whose
// cost is launch latency rather than arithmetic.
//
// Steps per chunk (all heads batched in each launch, z = b*H + h):
//   [key instance-norm] -> inner forward on K -> loss gradient -> backprop ->
//   per matrix: [momentum] -> [Newton-Schulz] -> W <- W - lr U -> [row L2-norm]
// and the apply O = F_W(Q), before the update (causal) or after all chunks.
// Source: ViT3 digest section 02 (update equation); LaCT analysis, "Nonlinear
// memory complements local attention" and "Order of operations".
#include <algorithm>

#include "ttt_plan.cuh"

namespace ttt {
namespace {

// ------------------------------------------------------------------ SIMT GEMM
struct MatRef {  // element (z, r, c) at p[z*sz + r*sr + c*sc]
  const float* p;
  int64_t sz, sr, sc;
};

constexpr int SG_T = 64, SG_K = 16;

// C(z, m, n) = alpha * sum_k A(z, m, k) B(z, k, n) + beta * Cin(z, m, n)
__global__ void __launch_bounds__(256) sgemm_kernel(int M, int N, int K, float alpha, MatRef A, MatRef B, float beta,
                                                    MatRef Cin, float* C, int64_t cz, int64_t cr) {
  __shared__ float As[SG_K][SG_T + 1];
  __shared__ float Bs[SG_K][SG_T + 1];
  const int z = blockIdx.z;
  const int m0 = blockIdx.y * SG_T, n0 = blockIdx.x * SG_T;
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < K; k0 += SG_K) {
    for (int i = threadIdx.x; i < SG_T * SG_K; i += 256) {
      const int r = i / SG_K, k = i % SG_K;
      const int gm = m0 + r, gk = k0 + k;
      As[k][r] = (gm < M && gk < K) ? A.p[z * A.sz + gm * A.sr + gk * A.sc] : 0.0f;
      const int c = i % SG_T, kk = i / SG_T;
      const int gn = n0 + c, gk2 = k0 + kk;
      Bs[kk][c] = (gn < N && gk2 < K) ? B.p[z * B.sz + gk2 * B.sr + gn * B.sc] : 0.0f;
    }
    __syncthreads();
#pragma unroll
    for (int k = 0; k < SG_K; ++k) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[k][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = Bs[k][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int m = m0 + ty * 4 + i;
    if (m >= M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tx * 4 + j;
      if (n >= N) continue;
      float v = alpha * acc[i][j];
      if (beta != 0.0f) v += beta * Cin.p[z * Cin.sz + m * Cin.sr + n * Cin.sc];
      C[z * cz + m * cr + n] = v;
    }
  }
}

int sgemm(cudaStream_t st, int Z, int M, int N, int K, float alpha, MatRef A, MatRef B, float beta, MatRef Cin,
          float* C, int64_t cz, int64_t cr) {
  if (M <= 0 || N <= 0) return TTT_OK;
  dim3 grid((N + SG_T - 1) / SG_T, (M + SG_T - 1) / SG_T, Z);
  {
    StageScope _sc(kStageOther, st);
    sgemm_kernel<<<grid, 256, 0, st>>>(M, N, K, alpha, A, B, beta, Cin, C, cz, cr);
  }
  return cudaGetLastError() == cudaSuccess ? TTT_OK : TTT_ERR_CUDA;
}

// row-major [Z][rows][cols] views
MatRef rm(const float* p, int64_t sz, int64_t ld) { return MatRef{p, sz, ld, 1}; }
MatRef rmT(const float* p, int64_t sz, int64_t ld) { return MatRef{p, sz, 1, ld}; }  // transposed view

// ------------------------------------------------------------------ elementwise
__device__ __forceinline__ float gelu_f(float x) { return 0.5f * x * (1.0f + erff(x * 0.70710678118654752f)); }
__device__ __forceinline__ float gelu_grad_f(float x) {
  return 0.5f * (1.0f + erff(x * 0.70710678118654752f)) + x * 0.39894228040143268f * expf(-0.5f * x * x);
}
__device__ __forceinline__ float sigmoid_f(float x) { return 1.0f / (1.0f + expf(-x)); }

// out = act(in) (op 0: GELU, 1: SiLU)
__global__ void act_kernel(int op, int64_t n, const float* in, float* out) {
  for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < n; i += int64_t(gridDim.x) * blockDim.x) {
    const float x = in[i];
    out[i] = op == 0 ? gelu_f(x) : x * sigmoid_f(x);
  }
}

// MLP2: dZ = dH * GELU'(Z) (in place on dH)
__global__ void gelu_back_kernel(int64_t n, const float* Z, float* dH) {
  for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < n; i += int64_t(gridDim.x) * blockDim.x)
    dH[i] *= gelu_grad_f(Z[i]);
}

// SwiGLU forward: A = SiLU(Z1); H = A * Z3
__global__ void swiglu_fwd_kernel(int64_t n, const float* Z1, const float* Z3, float* A, float* H) {
  for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < n; i += int64_t(gridDim.x) * blockDim.x) {
    const float a = Z1[i] * sigmoid_f(Z1[i]);
    if (A) A[i] = a;
    H[i] = a * Z3[i];
  }
}

// SwiGLU backward: dZ3 = dH * A; dZ1 = dH * Z3 * SiLU'(Z1)   (dZ1 overwrites Z1, dZ3 overwrites dH)
__global__ void swiglu_back_kernel(int64_t n, float* Z1, const float* Z3, float* dH) {
  for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < n; i += int64_t(gridDim.x) * blockDim.x) {
    const float z1 = Z1[i], s = sigmoid_f(z1), dh = dH[i];
    Z1[i] = dh * Z3[i] * s * (1.0f + z1 * (1.0f - s));
    dH[i] = dh * z1 * s;
  }
}

// RMSE of the chunk per z: sqrt(sum_i eta_i ||Vhat_i - V_i||^2 / (n d)); one CTA of
// 256 threads per z, fixed-order tree reduction.
__global__ void rmse_kernel(int n, int d, const float* Y, int64_t y_sz, const float* V, int64_t v_sz, int t0,
                            const float* eta, int64_t eta_sz, float eta_scalar, float* rms) {
  __shared__ float red[256];
  const int z = blockIdx.x;
  float s = 0.f;
  for (int64_t i = threadIdx.x; i < int64_t(n) * d; i += blockDim.x) {
    const int r = int(i / d), c = int(i % d);
    const float e = eta ? eta[z * eta_sz + t0 + r] : eta_scalar;
    const float diff = Y[z * y_sz + i] - V[z * v_sz + int64_t(t0 + r) * d + c];
    s += e * diff * diff;
  }
  red[threadIdx.x] = s;
  __syncthreads();
  for (int w = blockDim.x / 2; w > 0; w >>= 1) {
    if (threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0) rms[z] = sqrtf(red[0] / (float(n) * float(d)));
}

// dY = dL/dV_hat for the chunk; Vhat [Z][n][d] (overwritten), V rows t0.. of [Z][N][d].
// RMSE: the MSE gradient over 2 RMSE (rms [Z] from rmse_kernel), zero where RMSE = 0.
__global__ void loss_grad_kernel(int loss, int Z, int n, int d, float* Y, int64_t y_sz, const float* V, int64_t v_sz,
                                 int t0, const float* eta, int64_t eta_sz, float eta_scalar, const float* rms) {
  const int64_t total = int64_t(Z) * n * d;
  const float mse_coef = 2.0f / (float(n) * float(d));
  for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < total; i += int64_t(gridDim.x) * blockDim.x) {
    const int z = int(i / (int64_t(n) * d));
    const int r = int((i / d) % n), c = int(i % d);
    const float v = V[z * v_sz + int64_t(t0 + r) * d + c];
    const float e = eta ? eta[z * eta_sz + t0 + r] : eta_scalar;
    float* y = Y + z * y_sz + int64_t(r) * d + c;
    if (loss == TTT_LOSS_NEG_DOT) {
      *y = -e * v;
    } else if (loss == TTT_LOSS_MSE) {
      *y = mse_coef * e * (*y - v);
    } else {
      const float q = rms[z];
      *y = q > 0.f ? e * (*y - v) / (float(n) * float(d) * q) : 0.f;
    }
  }
}

// key instance-norm over the chunk's tokens: one CTA per z
__global__ void instnorm_kernel(int n, int d, const float* K, int64_t k_sz, int t0, float eps, float* out,
                                int64_t out_sz) {
  extern __shared__ float red[];  // [blockDim]
  const int z = blockIdx.x;
  const float* src = K + z * k_sz + int64_t(t0) * d;
  float* dst = out + z * out_sz;
  for (int c0 = 0; c0 < d; c0 += 32) {
    const int c = c0 + (threadIdx.x & 31);
    const int g = threadIdx.x >> 5, G = blockDim.x >> 5;
    float s = 0.f;
    if (c < d)
      for (int r = g; r < n; r += G) s += src[int64_t(r) * d + c];
    red[threadIdx.x] = s;
    __syncthreads();
    float mean = 0.f;
    if (c < d) {
      for (int j = 0; j < G; ++j) mean += red[j * 32 + (threadIdx.x & 31)];
      mean /= float(n);
    }
    __syncthreads();
    float q = 0.f;
    if (c < d)
      for (int r = g; r < n; r += G) {
        const float t = src[int64_t(r) * d + c] - mean;
        q += t * t;
      }
    red[threadIdx.x] = q;
    __syncthreads();
    float var = 0.f;
    if (c < d) {
      for (int j = 0; j < G; ++j) var += red[j * 32 + (threadIdx.x & 31)];
      var /= float(n);
      const float rs = rsqrtf(var + eps);
      for (int r = g; r < n; r += G) dst[int64_t(r) * d + c] = (src[int64_t(r) * d + c] - mean) * rs;
    }
    __syncthreads();
  }
}

// momentum: M = beta M + G; G = M (so G holds the update direction)
__global__ void momentum_kernel(int64_t n, float beta, float* M, float* G) {
  for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < n; i += int64_t(gridDim.x) * blockDim.x) {
    const float m = beta * M[i] + G[i];
    M[i] = m;
    G[i] = m;
  }
}

// per-matrix Frobenius scale: X = src / (||src|| + 1e-7), one CTA per z; src (z, r, c) strided
__global__ void ns_normalize_kernel(int rows, int cols, MatRef src, float* X) {
  __shared__ float red[256];
  const int z = blockIdx.x;
  float s = 0.f;
  for (int i = threadIdx.x; i < rows * cols; i += blockDim.x) {
    const float v = src.p[z * src.sz + (i / cols) * src.sr + (i % cols) * src.sc];
    s += v * v;
  }
  red[threadIdx.x] = s;
  __syncthreads();
  for (int w = blockDim.x / 2; w > 0; w >>= 1) {
    if (threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
    __syncthreads();
  }
  const float inv = 1.0f / (sqrtf(red[0]) + 1e-7f);
  for (int i = threadIdx.x; i < rows * cols; i += blockDim.x)
    X[int64_t(z) * rows * cols + i] = src.p[z * src.sz + (i / cols) * src.sr + (i % cols) * src.sc] * inv;
}

// W(z, r, c) -= lr * U(z, r, c) with U strided (covers the transposed NS output)
__global__ void apply_update_kernel(int rows, int cols, float lr, MatRef U, float* W, int64_t w_sz) {
  const int z = blockIdx.y;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < rows * cols; i += gridDim.x * blockDim.x) {
    const int r = i / cols, c = i % cols;
    W[z * w_sz + i] -= lr * U.p[z * U.sz + r * U.sr + c * U.sc];
  }
}

// each row of W (z, r, :) scaled to unit L2 norm; one warp per row
__global__ void rownorm_kernel(int rows, int cols, float* W, int64_t w_sz) {
  const int z = blockIdx.y;
  const int r = blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
  if (r >= rows) return;
  float* row = W + z * w_sz + int64_t(r) * cols;
  float s = 0.f;
  for (int c = threadIdx.x & 31; c < cols; c += 32) s += row[c] * row[c];
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  const float inv = 1.0f / fmaxf(sqrtf(s), 1e-12f);
  for (int c = threadIdx.x & 31; c < cols; c += 32) row[c] *= inv;
}

// W[z] = W0[z % H] (H = rows of W0: the heads, or every batch entry and head)
__global__ void init_weights_kernel(int Z, int H, int64_t P, const float* W0, float* W) {
  const int64_t total = int64_t(Z) * P;
  for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < total; i += int64_t(gridDim.x) * blockDim.x) {
    const int z = int(i / P);
    W[i] = W0[int64_t(z % H) * P + i % P];
  }
}

__global__ void nonfinite_kernel(int64_t n, const float* x, unsigned* status) {
  bool bad = false;
  for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < n; i += int64_t(gridDim.x) * blockDim.x)
    bad |= !isfinite(x[i]);
  if (__any_sync(0xffffffffu, bad) && (threadIdx.x & 31) == 0) atomicOr(status, kStatusNonFinite);
}

int grid_for(int64_t n) { return int(std::min<int64_t>((n + 255) / 256, int64_t(sm_count()) * 16)); }

// ------------------------------------------------------------------ workspace
enum Buf { bW, bM, bG, bXn, bZ1, bZ3, bA, bH, bdH, bY, bNX, bNX2, bNS, bNT, bRms, kNumBuf };

struct F32View {
  float* b[kNumBuf];
  unsigned* status;
};

F32View view(const Plan& p, void* ws) {
  F32View v;
  uint8_t* base = static_cast<uint8_t*>(ws);
  v.status = reinterpret_cast<unsigned*>(base);
  for (int i = 0; i < kNumBuf; ++i) v.b[i] = reinterpret_cast<float*>(base + p.off[i]);
  return v;
}

struct Mat {
  const char* name;
  int rows, cols;
  int64_t off;
};

int matrices(const Plan& p, Mat* m) {
  const int d = p.cfg.d, h = p.cfg.h;
  switch (p.cfg.inner) {
    case TTT_INNER_LINEAR: m[0] = {"W", d, d, 0}; return 1;
    case TTT_INNER_MLP2_GELU:
      m[0] = {"W1", h, d, 0};
      m[1] = {"W2", d, h, int64_t(h) * d};
      return 2;
    default:
      m[0] = {"W1", h, d, 0};
      m[1] = {"W3", h, d, int64_t(h) * d};
      m[2] = {"W2", d, h, 2 * int64_t(h) * d};
      return 3;
  }
}

// F_W(X) for rows [0, n): X is a strided view; result written to Y (row-major [Z][n][d]).
// Keeps Z1/Z3/A/H in the workspace for the backward pass.
int inner_forward(const Plan& p, const F32View& v, cudaStream_t st, MatRef X, int n, float* Y, int64_t y_sz,
                  int64_t y_ld) {
  const int Z = p.BH, d = p.cfg.d, h = p.cfg.h;
  const int64_t P = p.P, R = p.off[kNumBuf], Rh = R * h;  // R = rows reserved per head
  const float* W = v.b[bW];
  const MatRef none{nullptr, 0, 0, 0};
  int r = TTT_OK;
  switch (p.cfg.inner) {
    case TTT_INNER_LINEAR:
      return sgemm(st, Z, n, d, d, 1.f, X, rmT(W, P, d), 0.f, none, Y, y_sz, y_ld);
    case TTT_INNER_MLP2_GELU:
      r = sgemm(st, Z, n, h, d, 1.f, X, rmT(W, P, d), 0.f, none, v.b[bZ1], Rh, h);
      if (r) return r;
      {
        StageScope _sc(kStageOther, st);
        act_kernel<<<grid_for(int64_t(Z) * Rh), 256, 0, st>>>(0, int64_t(Z) * Rh, v.b[bZ1], v.b[bH]);
      }
      return sgemm(st, Z, n, d, h, 1.f, rm(v.b[bH], Rh, h), rmT(W + int64_t(h) * d, P, h), 0.f, none, Y, y_sz, y_ld);
    default:
      r = sgemm(st, Z, n, h, d, 1.f, X, rmT(W, P, d), 0.f, none, v.b[bZ1], Rh, h);
      if (!r) r = sgemm(st, Z, n, h, d, 1.f, X, rmT(W + int64_t(h) * d, P, d), 0.f, none, v.b[bZ3], Rh, h);
      if (r) return r;
      {
        StageScope _sc(kStageOther, st);
        swiglu_fwd_kernel<<<grid_for(int64_t(Z) * Rh), 256, 0, st>>>(int64_t(Z) * Rh, v.b[bZ1], v.b[bZ3], v.b[bA],
                                                                     v.b[bH]);
      }
      return sgemm(st, Z, n, d, h, 1.f, rm(v.b[bH], Rh, h), rmT(W + 2 * int64_t(h) * d, P, h), 0.f, none, Y, y_sz,
                   y_ld);
  }
}

// Newton-Schulz on U (z, rows, cols) strided; result: v.b[bNX] as [Z][m][n] with m <= n.
// Returns through *out the view of the result in (rows, cols) orientation.
int newton_schulz(const Plan& p, const F32View& v, cudaStream_t st, MatRef U, int rows, int cols, MatRef* out) {
  const int Z = p.BH;
  const bool tr = rows > cols;
  const int m = tr ? cols : rows, n = tr ? rows : cols;
  MatRef src = tr ? MatRef{U.p, U.sz, U.sc, U.sr} : U;
  const int64_t mn = int64_t(m) * n, mm = int64_t(m) * m;
  float* X = v.b[bNX];
  float* X2 = v.b[bNX2];
  {
    StageScope _sc(kStageOther, st);
    ns_normalize_kernel<<<Z, 256, 0, st>>>(m, n, src, X);
  }
  if (cudaGetLastError() != cudaSuccess) return TTT_ERR_CUDA;
  const float a = p.cfg.ns_coeff[0], b = p.cfg.ns_coeff[1], c = p.cfg.ns_coeff[2];
  const MatRef none{nullptr, 0, 0, 0};
  for (int it = 0; it < p.cfg.ns_iters; ++it) {
    int r = sgemm(st, Z, m, m, n, 1.f, rm(X, mn, n), rmT(X, mn, n), 0.f, none, v.b[bNS], mm, m);  // A = X X^T
    if (!r) r = sgemm(st, Z, m, m, m, c, rm(v.b[bNS], mm, m), rm(v.b[bNS], mm, m), b, rm(v.b[bNS], mm, m),
                      v.b[bNT], mm, m);  // T = b A + c A A
    if (!r) r = sgemm(st, Z, m, n, m, 1.f, rm(v.b[bNT], mm, m), rm(X, mn, n), a, rm(X, mn, n), X2, mn, n);  // aX + T X
    if (r) return r;
    std::swap(X, X2);
  }
  *out = tr ? MatRef{X, mn, 1, n} : MatRef{X, mn, n, 1};
  return TTT_OK;
}

int update_chunk(const Plan& p, const F32View& v, const Io& io, cudaStream_t st, int t0, int n) {
  const ttt_config& c = p.cfg;
  const int Z = p.BH, d = c.d, h = c.h, N = c.N;
  const int64_t P = p.P, R = p.off[kNumBuf], Rh = R * h, Rd = R * d;
  const float* K = static_cast<const float*>(io.K);
  const float* V = static_cast<const float*>(io.V);
  const MatRef none{nullptr, 0, 0, 0};
  int r = TTT_OK;
  // keys (instance-normalised over the chunk's tokens when asked)
  MatRef X{K + int64_t(t0) * d, int64_t(N) * d, d, 1};
  if (c.flags & TTT_FLAG_KEY_INSTNORM) {
    {
      StageScope _sc(kStageOther, st);
      instnorm_kernel<<<Z, 256, 256 * sizeof(float), st>>>(n, d, K, int64_t(N) * d, t0, c.in_eps, v.b[bXn], Rd);
    }
    if (cudaGetLastError() != cudaSuccess) return TTT_ERR_CUDA;
    X = rm(v.b[bXn], Rd, d);
  }
  // forward on the keys, then dY = dL/dV_hat (written over V_hat)
  r = inner_forward(p, v, st, X, n, v.b[bY], Rd, d);
  if (r) return r;
  const int64_t tot = int64_t(Z) * n * d;
  if (c.loss == TTT_LOSS_RMSE) {
    StageScope _sc(kStageOther, st);
    rmse_kernel<<<Z, 256, 0, st>>>(n, d, v.b[bY], Rd, V, int64_t(N) * d, t0, io.eta, int64_t(N), c.eta_scalar,
                                   v.b[bRms]);
  }
  {
    StageScope _sc(kStageOther, st);
    loss_grad_kernel<<<grid_for(tot), 256, 0, st>>>(c.loss, Z, n, d, v.b[bY], Rd, V, int64_t(N) * d, t0, io.eta,
                                                     int64_t(N), c.eta_scalar, v.b[bRms]);
  }
  // backprop into the gradient buffer G [Z][P]
  float* G = v.b[bG];
  const float* W = v.b[bW];
  const MatRef dY = rm(v.b[bY], Rd, d);
  const MatRef dYT = rmT(v.b[bY], Rd, d);
  switch (c.inner) {
    case TTT_INNER_LINEAR:
      r = sgemm(st, Z, d, d, n, 1.f, dYT, X, 0.f, none, G, P, d);  // G = dY^T X
      break;
    case TTT_INNER_MLP2_GELU:
      r = sgemm(st, Z, d, h, n, 1.f, dYT, rm(v.b[bH], Rh, h), 0.f, none, G + int64_t(h) * d, P, h);  // G2 = dY^T H
      if (!r) r = sgemm(st, Z, n, h, d, 1.f, dY, rm(W + int64_t(h) * d, P, h), 0.f, none, v.b[bdH], Rh, h);  // dH
      if (!r) {
        {
          StageScope _sc(kStageOther, st);
          gelu_back_kernel<<<grid_for(int64_t(Z) * Rh), 256, 0, st>>>(int64_t(Z) * Rh, v.b[bZ1], v.b[bdH]);
        }
        r = sgemm(st, Z, h, d, n, 1.f, rmT(v.b[bdH], Rh, h), X, 0.f, none, G, P, d);  // G1 = dZ^T X
      }
      break;
    default:
      r = sgemm(st, Z, d, h, n, 1.f, dYT, rm(v.b[bH], Rh, h), 0.f, none, G + 2 * int64_t(h) * d, P, h);  // G2
      if (!r) r = sgemm(st, Z, n, h, d, 1.f, dY, rm(W + 2 * int64_t(h) * d, P, h), 0.f, none, v.b[bdH], Rh, h);
      if (!r) {
        {
          StageScope _sc(kStageOther, st);
          swiglu_back_kernel<<<grid_for(int64_t(Z) * Rh), 256, 0, st>>>(int64_t(Z) * Rh, v.b[bZ1], v.b[bZ3], v.b[bdH]);
        }
        r = sgemm(st, Z, h, d, n, 1.f, rmT(v.b[bZ1], Rh, h), X, 0.f, none, G, P, d);  // G1 = dZ1^T X
      }
      if (!r) r = sgemm(st, Z, h, d, n, 1.f, rmT(v.b[bdH], Rh, h), X, 0.f, none, G + int64_t(h) * d, P, d);  // G3
      break;
  }
  if (r) return r;
  // optimizer, per matrix
  const bool mom = c.opt == TTT_OPT_MOMENTUM || c.opt == TTT_OPT_MOMENTUM_MUON;
  const bool muon = c.opt == TTT_OPT_MUON || c.opt == TTT_OPT_MOMENTUM_MUON;
  if (mom) momentum_kernel<<<grid_for(int64_t(Z) * P), 256, 0, st>>>(int64_t(Z) * P, c.momentum, v.b[bM], G);
  Mat mats[3];
  const int nm = matrices(p, mats);
  const bool hold_w2 = (c.flags & TTT_FLAG_FIRST_LAYER_ONLY) != 0;
  for (int i = 0; i < nm; ++i) {
    const Mat& m = mats[i];
    // first-layer-only updates: W2 (the last matrix of MLP2 / SwiGLU) keeps its value
    if (hold_w2 && c.inner != TTT_INNER_LINEAR && i == nm - 1) continue;
    MatRef U{G + m.off, P, m.cols, 1};
    if (muon) {
      r = newton_schulz(p, v, st, U, m.rows, m.cols, &U);
      if (r) return r;
    }
    dim3 g1((m.rows * m.cols + 255) / 256, Z);
    {
      StageScope _sc(kStageOther, st);
      apply_update_kernel<<<g1, 256, 0, st>>>(m.rows, m.cols, c.lr, U, v.b[bW] + m.off, P);
    }
    if (c.flags & TTT_FLAG_WEIGHT_L2NORM) {
      dim3 g2((m.rows + 7) / 8, Z);
      {
        StageScope _sc(kStageOther, st);
        rownorm_kernel<<<g2, 256, 0, st>>>(m.rows, m.cols, v.b[bW] + m.off, P);
      }
    }
  }
  return cudaGetLastError() == cudaSuccess ? TTT_OK : TTT_ERR_CUDA;
}

}  // namespace

int plan_layout_f32(Plan* p) {
  const ttt_config& c = p->cfg;
  const int64_t Z = p->BH, d = c.d, h = c.h, P = p->P;
  const int64_t R = std::max<int64_t>(p->chunk, c.Nq);  // rows per head in the activation buffers
  const int64_t m = std::min(d, h), n = std::max(d, h);
  const int64_t sizes[kNumBuf] = {Z * P,     Z * P,     Z * P,     Z * R * d, Z * R * h, Z * R * h,
                                  Z * R * h, Z * R * h, Z * R * h, Z * R * d, Z * m * n, Z * m * n,
                                  Z * m * m, Z * m * m, Z};
  size_t o = 256;
  for (int i = 0; i < kNumBuf; ++i) {
    p->off[i] = o;
    o += (size_t(sizes[i]) * 4 + 255) / 256 * 256;
  }
  p->off[kNumBuf] = size_t(R);  // rows reserved per head
  p->ws_bytes = o;
  // the momentum buffer [Z][P] is the state a call hands on
  p->state_bytes = (c.opt == TTT_OPT_MOMENTUM || c.opt == TTT_OPT_MOMENTUM_MUON) ? size_t(Z * P) * 4 : 0;
  return TTT_OK;
}

int run_f32(const Plan& p, const Io& io, void* ws, cudaStream_t st) {
  const ttt_config& c = p.cfg;
  const F32View v = view(p, ws);
  const int Z = p.BH, d = c.d;
  const int64_t P = p.P;
  {
    StageScope _sc(kStageOther, st);
    const int w0_rows = (c.flags & TTT_FLAG_W0_PER_BATCH) ? Z : c.H;  // W0 [H][P] or [B*H][P]
    init_weights_kernel<<<grid_for(int64_t(Z) * P), 256, 0, st>>>(Z, w0_rows, P, io.W0, v.b[bW]);
  }
  if (io.M_in && p.state_bytes) {
    if (cudaMemcpyAsync(v.b[bM], io.M_in, p.state_bytes, cudaMemcpyDeviceToDevice, st) != cudaSuccess)
      return TTT_ERR_CUDA;
  } else if (cudaMemsetAsync(v.b[bM], 0, size_t(Z) * P * 4, st) != cudaSuccess) {
    return TTT_ERR_CUDA;
  }
  const float* Q = static_cast<const float*>(io.Q);
  float* O = static_cast<float*>(io.O);
  const int64_t q_sz = int64_t(c.Nq) * d;
  int r = TTT_OK;
  for (int ci = 0; ci < p.nchunks && !r; ++ci) {
    const int t0 = ci * p.chunk, n = std::min(p.chunk, c.N - t0);
    if (c.causal) {  // apply-then-update: chunk c reads the weights of chunks < c
      r = inner_forward(p, v, st, MatRef{Q + int64_t(t0) * d, q_sz, d, 1}, n, O + int64_t(t0) * d, q_sz, d);
      if (r) return r;
    }
    if (c.flags & TTT_FLAG_NO_UPDATE) continue;
    for (int ep = 0; ep < p.epochs && !r; ++ep) r = update_chunk(p, v, io, st, t0, n);
  }
  if (r) return r;
  if (!c.causal) {
    // the apply may cover more rows than one chunk: run it in pieces of at most R rows
    const int R = int(p.off[kNumBuf]);
    for (int s = 0; s < c.Nq && !r; s += R) {
      const int n = std::min(R, c.Nq - s);
      r = inner_forward(p, v, st, MatRef{Q + int64_t(s) * d, q_sz, d, 1}, n, O + int64_t(s) * d, q_sz, d);
    }
    if (r) return r;
  }
  if (io.W_out &&
      cudaMemcpyAsync(io.W_out, v.b[bW], size_t(Z) * P * 4, cudaMemcpyDeviceToDevice, st) != cudaSuccess)
    return TTT_ERR_CUDA;
  if (io.M_out && p.state_bytes &&
      cudaMemcpyAsync(io.M_out, v.b[bM], p.state_bytes, cudaMemcpyDeviceToDevice, st) != cudaSuccess)
    return TTT_ERR_CUDA;
  {
    StageScope _sc(kStageOther, st);
    nonfinite_kernel<<<grid_for(int64_t(Z) * c.Nq * d), 256, 0, st>>>(int64_t(Z) * c.Nq * d, O, v.status);
  }
  {
    StageScope _sc(kStageOther, st);
    nonfinite_kernel<<<grid_for(int64_t(Z) * P), 256, 0, st>>>(int64_t(Z) * P, v.b[bW], v.status);
  }
  return cudaGetLastError() == cudaSuccess ? TTT_OK : TTT_ERR_CUDA;
}

}  // namespace ttt
