// DWConv inner model of the TTT layer (the F2 module of the ViT3 design; ViT3
// digest, section 03, guideline 6 and the inner-model table).  The fast weights of
// a head are one k x k kernel per channel, applied as a 'same' depthwise
// cross-correlation with zero padding over the grid_h x grid_w token grid (tokens
// in raster order):
//   F(X)[(y,x), c] = sum_{a,b<k} Wc[c][a k + b] X[(y + a - k/2, x + b - k/2), c].
// The whole grid is one non-causal chunk: the keys and values of the grid update
// the kernels, then the queries (on the same grid) read them.
//
// The work is elementwise over (token, channel) with k*k neighbour reads and no
// contraction for the tensor cores, so it is bound by HBM bandwidth.  Tokens are
// [Z][N][d] with channels contiguous: a warp's lanes (consecutive channels) read
// consecutive addresses for every neighbour.  Weights are fp32 [Z][d][k*k].
//   tap gradient : per (token block, z, group of 128 channels), each thread owns one
//                  channel and accumulates over its block's tokens the k*k products
//                  dY_p * X_{p+tap} in registers.  dY = -eta v (dot loss), or
//                  2 eta (F(X)_p - v) / (N d) (MSE) with F(X)_p formed from the same
//                  neighbour values; fp32 partials per token block
//   weights      : per (z, channel), the partials summed in block order, momentum,
//                  W -= lr U, L2 norm of the channel's kernel, non-finite check
//   apply        : per (z, token, channel), O = sum_tap Wc * Q_{p+tap}
#include <cuda_bf16.h>

#include <algorithm>

#include "ttt_plan.cuh"

namespace ttt {
namespace {

struct DwGeom {
  int Z, N, d, gh, gw;
  int tok_per_block, blocks;  // token blocks of the tap-gradient pass
  int loss;
  float eta_scalar, mse_coef;
};

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
template <class T>
__device__ __forceinline__ T from_f(float x);
template <>
__device__ __forceinline__ float from_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

// neighbours of token p = (y, x) in channel c, zero outside the grid
template <int K, class T>
__device__ __forceinline__ void gather_taps(const T* Xz, const DwGeom& g, int p, int c, float (&nb)[K * K]) {
  constexpr int R = K / 2;
  const int y = p / g.gw, x = p - (p / g.gw) * g.gw;
#pragma unroll
  for (int a = 0; a < K; ++a) {
#pragma unroll
    for (int b = 0; b < K; ++b) {
      const int yy = y + a - R, xx = x + b - R;
      const bool in = yy >= 0 && yy < g.gh && xx >= 0 && xx < g.gw;
      nb[a * K + b] = in ? to_f(Xz[(int64_t(yy) * g.gw + xx) * g.d + c]) : 0.f;
    }
  }
}

template <int K, class T>
__global__ void __launch_bounds__(128) dw_tapgrad_kernel(DwGeom g, const T* X, const T* V, const float* eta,
                                                          const float* W, float* part) {
  constexpr int KK = K * K;
  const int z = blockIdx.y;
  const int c = blockIdx.z * blockDim.x + threadIdx.x;
  if (c >= g.d) return;  // no block-wide synchronisation below
  const int tb = blockIdx.x;
  const int p0 = tb * g.tok_per_block, p1 = min(g.N, p0 + g.tok_per_block);
  const T* Xz = X + int64_t(z) * g.N * g.d;
  const T* Vz = V + int64_t(z) * g.N * g.d;
  const bool mse = g.loss == TTT_LOSS_MSE;
  float w[KK];
#pragma unroll
  for (int t = 0; t < KK; ++t) w[t] = mse ? W[(int64_t(z) * g.d + c) * KK + t] : 0.f;
  float acc[KK];
#pragma unroll
  for (int t = 0; t < KK; ++t) acc[t] = 0.f;
  for (int p = p0; p < p1; ++p) {
    float nb[KK];
    gather_taps<K>(Xz, g, p, c, nb);
    const float e = eta ? eta[int64_t(z) * g.N + p] : g.eta_scalar;
    const float v = to_f(Vz[int64_t(p) * g.d + c]);
    float dy;
    if (mse) {
      float f = 0.f;
#pragma unroll
      for (int t = 0; t < KK; ++t) f += w[t] * nb[t];
      dy = g.mse_coef * e * (f - v);
    } else {
      dy = -e * v;
    }
#pragma unroll
    for (int t = 0; t < KK; ++t) acc[t] += dy * nb[t];
  }
  float* out = part + ((int64_t(z) * g.blocks + tb) * g.d + c) * KK;
#pragma unroll
  for (int t = 0; t < KK; ++t) out[t] = acc[t];
}

template <int K>
__global__ void dw_update_kernel(DwGeom g, const float* part, float* W, float* M, bool momentum, float beta, float lr,
                                 bool rownorm, unsigned* status) {
  constexpr int KK = K * K;
  const int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x;
  if (i >= int64_t(g.Z) * g.d) return;
  const int z = int(i / g.d), c = int(i % g.d);
  float u[KK];
#pragma unroll
  for (int t = 0; t < KK; ++t) u[t] = 0.f;
  for (int b = 0; b < g.blocks; ++b) {
    const float* pb = part + ((int64_t(z) * g.blocks + b) * g.d + c) * KK;
#pragma unroll
    for (int t = 0; t < KK; ++t) u[t] += pb[t];
  }
  float* w = W + i * KK;
  float* m = M + i * KK;
  float s = 0.f;
#pragma unroll
  for (int t = 0; t < KK; ++t) {
    float ut = u[t];
    if (momentum) {
      ut = beta * m[t] + ut;
      m[t] = ut;
    }
    const float wt = w[t] - lr * ut;
    w[t] = wt;
    s += wt * wt;
  }
  bool bad = false;
  const float inv = rownorm ? 1.0f / fmaxf(sqrtf(s), 1e-12f) : 1.0f;
#pragma unroll
  for (int t = 0; t < KK; ++t) {
    const float wt = w[t] * inv;
    w[t] = wt;
    bad |= !isfinite(wt);
  }
  if (bad) set_status(status, kStatusNonFinite);
}

template <int K, class T>
__global__ void dw_apply_kernel(DwGeom g, const T* Q, const float* W, T* O, unsigned* status) {
  constexpr int KK = K * K;
  const int64_t total = int64_t(g.Z) * g.N * g.d;
  bool bad = false;
  for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < total; i += int64_t(gridDim.x) * blockDim.x) {
    const int c = int(i % g.d);
    const int64_t zp = i / g.d;
    const int p = int(zp % g.N), z = int(zp / g.N);
    float nb[KK];
    gather_taps<K>(Q + int64_t(z) * g.N * g.d, g, p, c, nb);
    const float* w = W + (int64_t(z) * g.d + c) * KK;
    float s = 0.f;
#pragma unroll
    for (int t = 0; t < KK; ++t) s += w[t] * nb[t];
    O[i] = from_f<T>(s);
    bad |= !isfinite(s);
  }
  if (bad) set_status(status, kStatusNonFinite);
}

__global__ void dw_init_kernel(int Z, int w0_rows, int64_t P, const float* W0, float* W) {
  const int64_t total = int64_t(Z) * P;
  for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < total; i += int64_t(gridDim.x) * blockDim.x)
    W[i] = W0[int64_t(int(i / P) % w0_rows) * P + i % P];
}

enum DwBuf { dW, dM, dPart, kNumDwBuf };

DwGeom geom_of(const Plan& p) {
  const ttt_config& c = p.cfg;
  DwGeom g;
  g.Z = p.BH;
  g.N = c.N;
  g.d = c.d;
  g.gh = c.grid_h;
  g.gw = c.grid_w;
  g.tok_per_block = int(p.off[kNumDwBuf]);
  g.blocks = int(p.off[kNumDwBuf + 1]);
  g.loss = c.loss;
  g.eta_scalar = c.eta_scalar;
  g.mse_coef = 2.0f / (float(c.N) * float(c.d));
  return g;
}

int grid_1d(int64_t n) { return int(std::min<int64_t>((n + 255) / 256, int64_t(sm_count()) * 16)); }

template <int K, class T>
int run_k(const Plan& p, const Io& io, uint8_t* ws, cudaStream_t st) {
  const ttt_config& c = p.cfg;
  const DwGeom g = geom_of(p);
  unsigned* status = reinterpret_cast<unsigned*>(ws);
  float* W = reinterpret_cast<float*>(ws + p.off[dW]);
  float* M = reinterpret_cast<float*>(ws + p.off[dM]);
  float* part = reinterpret_cast<float*>(ws + p.off[dPart]);
  const int64_t ZP = int64_t(g.Z) * p.P;
  {
    StageScope _sc(kStageOther, st);
    const int w0_rows = (c.flags & TTT_FLAG_W0_PER_BATCH) ? g.Z : c.H;
    dw_init_kernel<<<grid_1d(ZP), 256, 0, st>>>(g.Z, w0_rows, p.P, io.W0, W);
  }
  if (io.M_in && p.state_bytes) {
    if (cudaMemcpyAsync(M, io.M_in, p.state_bytes, cudaMemcpyDeviceToDevice, st) != cudaSuccess) return TTT_ERR_CUDA;
  } else if (cudaMemsetAsync(M, 0, size_t(ZP) * 4, st) != cudaSuccess) {
    return TTT_ERR_CUDA;
  }
  const bool momentum = c.opt == TTT_OPT_MOMENTUM;
  const bool rownorm = (c.flags & TTT_FLAG_WEIGHT_L2NORM) != 0;
  const int epochs = (c.flags & TTT_FLAG_NO_UPDATE) ? 0 : p.epochs;
  const dim3 tg(g.blocks, g.Z, (g.d + 127) / 128);
  for (int ep = 0; ep < epochs; ++ep) {
    {
      StageScope _sc(kStageWeightGrad, st);
      dw_tapgrad_kernel<K, T><<<tg, 128, 0, st>>>(g, static_cast<const T*>(io.K), static_cast<const T*>(io.V), io.eta,
                                                   W, part);
    }
    {
      StageScope _sc(kStageFinish, st);
      dw_update_kernel<K><<<int((int64_t(g.Z) * g.d + 255) / 256), 256, 0, st>>>(g, part, W, M, momentum, c.momentum,
                                                                                  c.lr, rownorm, status);
    }
  }
  {
    StageScope _sc(kStageApply, st);
    dw_apply_kernel<K, T><<<grid_1d(int64_t(g.Z) * g.N * g.d), 256, 0, st>>>(g, static_cast<const T*>(io.Q), W,
                                                                              static_cast<T*>(io.O), status);
  }
  if (io.W_out && cudaMemcpyAsync(io.W_out, W, size_t(ZP) * 4, cudaMemcpyDeviceToDevice, st) != cudaSuccess)
    return TTT_ERR_CUDA;
  if (io.M_out && p.state_bytes &&
      cudaMemcpyAsync(io.M_out, M, p.state_bytes, cudaMemcpyDeviceToDevice, st) != cudaSuccess)
    return TTT_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? TTT_OK : TTT_ERR_CUDA;
}

template <class T>
int run_t(const Plan& p, const Io& io, uint8_t* ws, cudaStream_t st) {
  switch (p.cfg.ksize) {
    case 1: return run_k<1, T>(p, io, ws, st);
    case 3: return run_k<3, T>(p, io, ws, st);
    case 5: return run_k<5, T>(p, io, ws, st);
    case 7: return run_k<7, T>(p, io, ws, st);
    default: return TTT_ERR_UNSUPPORTED;
  }
}

}  // namespace

int plan_layout_dwconv(Plan* p) {
  const ttt_config& c = p->cfg;
  const int64_t Z = p->BH, d = c.d, KK = int64_t(c.ksize) * c.ksize;
  // token blocks: about four CTAs per SM over all (z, channel group) pairs, at least
  // 64 tokens per block; every block non-empty
  const int64_t groups = Z * ((d + 127) / 128);
  const int64_t want = std::max<int64_t>(1, (4 * kPlanSMs + groups - 1) / groups);
  const int64_t blocks0 = std::max<int64_t>(1, std::min<int64_t>(want, (c.N + 63) / 64));
  const int64_t per = (c.N + blocks0 - 1) / blocks0;
  const int64_t blocks = (c.N + per - 1) / per;
  if (blocks > 65535) return TTT_ERR_UNSUPPORTED;
  const int64_t bytes[kNumDwBuf] = {Z * p->P * 4, Z * p->P * 4, Z * blocks * d * KK * 4};
  size_t o = 256;
  for (int i = 0; i < kNumDwBuf; ++i) {
    p->off[i] = o;
    o += (size_t(bytes[i]) + 255) / 256 * 256;
  }
  p->off[kNumDwBuf] = size_t(per);
  p->off[kNumDwBuf + 1] = size_t(blocks);
  p->ws_bytes = o;
  p->state_bytes = c.opt == TTT_OPT_MOMENTUM ? size_t(bytes[dM]) : 0;
  return TTT_OK;
}

int run_dwconv(const Plan& p, const Io& io, void* ws, cudaStream_t st) {
  uint8_t* base = static_cast<uint8_t*>(ws);
  return p.cfg.dtype == TTT_F32 ? run_t<float>(p, io, base, st) : run_t<__nv_bfloat16>(p, io, base, st);
}

}  // namespace ttt
