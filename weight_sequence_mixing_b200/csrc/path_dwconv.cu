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

// Tap gradients of one token block: CTA (block, z, channel chunk) with threads
// (channel, slot); slot s takes the block's tokens p0 + s, p0 + s + S, ...  The S
// slots' register sums are added in slot order through shared memory, so the
// partial of a block does not depend on timing.
template <int K, class T>
__global__ void __launch_bounds__(256) dw_tapgrad_kernel(DwGeom g, const T* X, const T* V, const float* eta,
                                                          const float* W, float* part) {
  constexpr int KK = K * K;
  extern __shared__ float red[];  // [S][blockDim.x][KK]
  const int z = blockIdx.y;
  const int cx = threadIdx.x, slot = threadIdx.y, S = blockDim.y;
  const int c = blockIdx.z * blockDim.x + cx;
  const bool live = c < g.d;
  const int tb = blockIdx.x;
  const int p0 = tb * g.tok_per_block, p1 = min(g.N, p0 + g.tok_per_block);
  const T* Xz = X + int64_t(z) * g.N * g.d;
  const T* Vz = V + int64_t(z) * g.N * g.d;
  const bool mse = g.loss == TTT_LOSS_MSE;
  float w[KK];
#pragma unroll
  for (int t = 0; t < KK; ++t) w[t] = (mse && live) ? W[(int64_t(z) * g.d + c) * KK + t] : 0.f;
  float acc[KK];
#pragma unroll
  for (int t = 0; t < KK; ++t) acc[t] = 0.f;
  if (live) {
    for (int p = p0 + slot; p < p1; p += S) {
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
  }
  float* mine = red + (int64_t(slot) * blockDim.x + cx) * KK;
#pragma unroll
  for (int t = 0; t < KK; ++t) mine[t] = acc[t];
  __syncthreads();
  // slot-order sum: thread (cx, s) sums tap t = s, s + S, ... of channel cx
  if (live) {
    float* out = part + ((int64_t(z) * g.blocks + tb) * g.d + c) * KK;
    for (int t = slot; t < KK; t += S) {
      float u = 0.f;
      for (int j = 0; j < S; ++j) u += red[(int64_t(j) * blockDim.x + cx) * KK + t];
      out[t] = u;
    }
  }
}

// One warp per (z, channel): the lanes sum the token blocks' partials (lane l takes
// blocks l, l + 32, ...), a fixed butterfly adds the lanes, then momentum, the step
// and the kernel's L2 norm.
template <int K>
__global__ void dw_update_kernel(DwGeom g, const float* part, float* W, float* M, bool momentum, float beta, float lr,
                                 bool rownorm, unsigned* status) {
  constexpr int KK = K * K;
  const int lane = threadIdx.x & 31;
  const int64_t i = blockIdx.x * int64_t(blockDim.x / 32) + threadIdx.x / 32;
  if (i >= int64_t(g.Z) * g.d) return;  // whole warps leave together
  const int z = int(i / g.d), c = int(i % g.d);
  float u[KK];
#pragma unroll
  for (int t = 0; t < KK; ++t) u[t] = 0.f;
  for (int b = lane; b < g.blocks; b += 32) {
    const float* pb = part + ((int64_t(z) * g.blocks + b) * g.d + c) * KK;
#pragma unroll
    for (int t = 0; t < KK; ++t) u[t] += pb[t];
  }
#pragma unroll
  for (int t = 0; t < KK; ++t)
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) u[t] += __shfl_xor_sync(0xffffffffu, u[t], o);
  float* w = W + i * KK;
  float* m = M + i * KK;
  float wt[KK];
  float s = 0.f;
#pragma unroll
  for (int t = 0; t < KK; ++t) {
    float ut = u[t];
    if (momentum) ut = beta * m[t] + ut;
    wt[t] = w[t] - lr * ut;
    s += wt[t] * wt[t];
    u[t] = ut;
  }
  __syncwarp();
  const float inv = rownorm ? 1.0f / fmaxf(sqrtf(s), 1e-12f) : 1.0f;
  bool bad = false;
  for (int t = lane; t < KK; t += 32) {
    float wv = 0.f, uv = 0.f;
#pragma unroll
    for (int q = 0; q < KK; ++q)
      if (q == t) {
        wv = wt[q];
        uv = u[q];
      }
    if (momentum) m[t] = uv;
    w[t] = wv * inv;
    bad |= !isfinite(wv * inv);
  }
  if (__any_sync(0xffffffffu, bad) && lane == 0) set_status(status, kStatusNonFinite);
}

// O = sum_tap Wc * Q_{p+tap}: CTA (token chunk, z, channel chunk) with threads
// (channel, slot); the channel's k*k weights stay in registers while the slots walk
// the chunk's tokens.
template <int K, class T>
__global__ void __launch_bounds__(256) dw_apply_kernel(DwGeom g, int tok_per_cta, const T* Q, const float* W, T* O,
                                                        unsigned* status) {
  constexpr int KK = K * K;
  const int z = blockIdx.y;
  const int c = blockIdx.z * blockDim.x + threadIdx.x;
  if (c >= g.d) return;  // no block-wide synchronisation below
  const int p0 = blockIdx.x * tok_per_cta, p1 = min(g.N, p0 + tok_per_cta);
  float w[KK];
#pragma unroll
  for (int t = 0; t < KK; ++t) w[t] = W[(int64_t(z) * g.d + c) * KK + t];
  const T* Qz = Q + int64_t(z) * g.N * g.d;
  T* Oz = O + int64_t(z) * g.N * g.d;
  bool bad = false;
  for (int p = p0 + threadIdx.y; p < p1; p += blockDim.y) {
    float nb[KK];
    gather_taps<K>(Qz, g, p, c, nb);
    float s = 0.f;
#pragma unroll
    for (int t = 0; t < KK; ++t) s += w[t] * nb[t];
    Oz[int64_t(p) * g.d + c] = from_f<T>(s);
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
  // threads (channel, slot): up to 128 channels of a chunk, 256 threads per CTA
  // (the slot sums of the tap pass stay within the default 48 KB of shared memory)
  const int cx = std::min(g.d, 128);
  const int slots = std::max(1, std::min(256 / cx, 49152 / (cx * K * K * int(sizeof(float)))));
  const dim3 blk(cx, slots);
  const int cchunks = (g.d + cx - 1) / cx;
  const dim3 tg(g.blocks, g.Z, cchunks);
  const size_t red_bytes = size_t(slots) * cx * (K * K) * sizeof(float);
  for (int ep = 0; ep < epochs; ++ep) {
    {
      StageScope _sc(kStageWeightGrad, st);
      dw_tapgrad_kernel<K, T><<<tg, blk, red_bytes, st>>>(g, static_cast<const T*>(io.K), static_cast<const T*>(io.V),
                                                          io.eta, W, part);
    }
    {
      StageScope _sc(kStageFinish, st);
      dw_update_kernel<K><<<int((int64_t(g.Z) * g.d + 7) / 8), 256, 0, st>>>(g, part, W, M, momentum, c.momentum, c.lr,
                                                                             rownorm, status);
    }
  }
  {
    StageScope _sc(kStageApply, st);
    // about eight CTAs per SM over (token chunk, z, channel chunk)
    const int64_t want = std::max<int64_t>(1, (int64_t(sm_count()) * 8 + int64_t(g.Z) * cchunks - 1) /
                                                  (int64_t(g.Z) * cchunks));
    const int tok = int(std::max<int64_t>(slots, (g.N + want - 1) / want));
    const dim3 ag((g.N + tok - 1) / tok, g.Z, cchunks);
    dw_apply_kernel<K, T><<<ag, blk, 0, st>>>(g, tok, static_cast<const T*>(io.Q), W, static_cast<T*>(io.O), status);
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
