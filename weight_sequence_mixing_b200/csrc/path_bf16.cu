// bf16 path of the TTT layer: tcgen05 tensor-core GEMMs (bf16 operands, fp32
// accumulation in TMEM) with the elementwise steps fused into their epilogues.
//
// Per chunk c (tokens [t0, t0+n), all heads batched, z = b*H + h):
//   token phase  : one launch over 256-token x 128-hidden tiles on CTA pairs (dot
//                  loss; 128-token tiles on single CTAs as the fallback) computes
//                  the inner forward on the keys and the loss backprop to the hidden
//                  layer (epilogue: SiLU / GELU gating, eta_i folding), writing the
//                  bf16 activations the weight gradient needs; the MSE loss runs it
//                  as three GEMMs with fused epilogues
//   weight grads : one grouped launch of token-reduction GEMMs (MN-major operands,
//                  512-row tiles on CTA pairs or 256/128-row tiles on single CTAs,
//                  split-K over tokens, fp32 partials, deterministic reduction)
//   optimizer    : split reduction + momentum, [Newton-Schulz on tf32 tensor cores],
//                  W <- W - lr U, row L2-norm, bf16 copies of the new weights
//   apply        : O = F_W(Q) as two GEMMs (first layer + gating, second layer)
// Non-causal layers update over every chunk and apply once; causal layers apply
// with the current weights before each chunk's update.
// Source: ViT3 digest section 02 (update equation; forward on keys, loss
// backward, forward on queries); LaCT analysis "Nonlinear memory complements local
// attention" (SwiGLU fast weights, negative dot loss, per-token learning rates,
// momentum / Muon, L2 normalisation) and "Order of operations".
#include <algorithm>

#include "apply_mlp.cuh"
#include "epi_glu.cuh"
#include "epilogues.cuh"
#include "glu_update.cuh"
#include "mse_token.cuh"
#include "ns_fused.cuh"
#include "token_pair.cuh"
#include "token_phase.cuh"
#include "ttt_diag.h"
#include "ttt_plan.cuh"
#include "wgrad.cuh"
#include "wgrad_pair.cuh"

namespace ttt {
namespace {

// ------------------------------------------------------------------ workspace
enum BBuf {
  xWf,     // fp32 master weights [Z][P] (canonical packed layout)
  xMom,    // fp32 momentum, gradient layout [Z][GR][d]
  xU,      // fp32 update direction, gradient layout [Z][GR][d]
  xRowSq,  // fp32 [Z][GR] squared row norms of U
  xPart,   // fp32 split-K partials [S][Z][GR][d]
  xFirst,  // bf16 first-layer weights [Z][R1][d] (SwiGLU: blocks [W1 128 | W3 128])
  xW2T,    // bf16 W2^T [Z][h][d]
  xW2,     // bf16 W2 [Z][d][h]
  xKn,     // bf16 instance-normalised keys [Z][Cp][d]
  xAct0,   // bf16 activations [Z][Cp][h]   (H' or H)
  xAct1,   // bf16 activations [Z][Cp][2h]  (dZ13, dZ)
  xAct2,   // bf16 [Z][Cp][h]  (GELU' for MSE)
  xDY,     // bf16 [Z][Cp][d]  (dL/dV_hat for MSE / linear)
  xHq,     // bf16 apply hidden [Z][Rq][h]
  xKstat,  // fp32 key-norm partial sums [Z][Cp/128][d][2], then [Z][d][2] mean and 1/std, then
           // [Z] u32 counters of the blocks done (zero between launches)
  xNX, xNXT, xNX2, xNXT2, xNS, xNT,  // fp32 Newton-Schulz buffers [Z*nmat][...]
  kNumBBuf
};

struct Dims {
  int Z, H, N, Nq, d, h, Cp, Rq, GR, R1, nmat, m, n, splits, tile_rows, grad_bn;
  bool direct;  // unsplit gradients go straight into U (and M): no partials, no reduction
  bool src_t;  // Newton-Schulz input is the transpose of the gradient-layout source
  bool token_pairs;  // token phase (and, with tile_rows 512, weight gradients) on CTA pairs
};

int bn_for(int n) { return n % 256 == 0 ? 256 : n % 128 == 0 ? 128 : 64; }

// The GELU MLP with the MSE loss at d = 64 and h = 128 or 256 runs its token phase and
// weight gradients in one kernel (mse_token.cuh), one CTA per head and token-tile range,
// which writes split partials of the gradients.
bool mse_token_path(const ttt_config& c) {
  return c.inner == TTT_INNER_MLP2_GELU && c.loss == TTT_LOSS_MSE && c.d == 64 && (c.h == 128 || c.h == 256);
}

// The GLU at d = 64 (ViT3's heads) likewise: token GEMM, gating gradient and the gradient
// reduction in one kernel (glu_update.cuh).
bool glu_update_path(const ttt_config& c) { return c.inner == TTT_INNER_GLU && c.d == 64; }

// Either fused update: one CTA per (head, token-tile range), split partials reduced by the finish.
bool fused_update_path(const ttt_config& c) { return mse_token_path(c) || glu_update_path(c); }

Dims dims_of(const Plan& p) {
  const ttt_config& c = p.cfg;
  Dims D{};
  D.Z = p.BH;
  D.H = c.H;
  D.N = c.N;
  D.Nq = c.Nq;
  D.d = c.d;
  D.h = c.h;
  D.Cp = (p.chunk + 127) / 128 * 128;
  D.Rq = c.causal ? D.Cp : (c.Nq + 127) / 128 * 128;
  switch (c.inner) {
    case TTT_INNER_LINEAR: D.GR = c.d; D.R1 = c.d; D.nmat = 1; break;
    case TTT_INNER_MLP2_GELU: D.GR = 2 * c.h; D.R1 = c.h; D.nmat = 2; break;
    case TTT_INNER_GLU: D.GR = 2 * c.d; D.R1 = 2 * c.d; D.nmat = 2; break;
    default: D.GR = 3 * c.h; D.R1 = 2 * c.h; D.nmat = 3; break;
  }
  const int rows_src = c.inner == TTT_INNER_LINEAR ? c.d : c.h;
  D.src_t = rows_src > c.d;
  D.m = std::min(rows_src, c.d);
  D.n = std::max(rows_src, c.d);
  D.splits = int(p.off[kNumBBuf]);
  D.tile_rows = int(p.off[kNumBBuf + 1]);
  D.grad_bn = int(p.off[kNumBBuf + 2]);
  const bool muon = c.opt == TTT_OPT_MUON || c.opt == TTT_OPT_MOMENTUM_MUON;
  // with Muon the squared row norms are summed over the tiles of a row: allow at
  // most two contributions per row (order-independent)
  D.direct = D.splits == 1 && !(muon && D.grad_bn != c.d) && !fused_update_path(c);
  D.token_pairs = (c.flags & TTT_FLAG_SINGLE_CTA) == 0;
  return D;
}


// ------------------------------------------------------------------ small kernels
// Per canonical weight row: which matrix, its length, and where its gradient /
// Newton-Schulz rows live.
struct RowMap {
  int inner, d, h, GR;
  int64_t P;
  __host__ __device__ int nrows() const {
    return inner == TTT_INNER_LINEAR ? d : inner == TTT_INNER_MLP2_GELU ? h + d : inner == TTT_INNER_GLU ? 2 * d
                                                                                                          : 2 * h + d;
  }
  // matrix index k, row inside it, row length, offset of the matrix in the packed layout
  __device__ void locate(int R, int& k, int& r, int& len, int64_t& off) const {
    if (inner == TTT_INNER_LINEAR) { k = 0; r = R; len = d; off = 0; return; }
    if (inner == TTT_INNER_GLU) {  // [Wa | Wb], both d x d
      k = R < d ? 0 : 1; r = R < d ? R : R - d; len = d; off = int64_t(k) * d * d;
      return;
    }
    if (inner == TTT_INNER_MLP2_GELU) {
      if (R < h) { k = 0; r = R; len = d; off = 0; }
      else { k = 1; r = R - h; len = h; off = int64_t(h) * d; }
      return;
    }
    if (R < h) { k = 0; r = R; len = d; off = 0; }
    else if (R < 2 * h) { k = 1; r = R - h; len = d; off = int64_t(h) * d; }
    else { k = 2; r = R - 2 * h; len = h; off = 2 * int64_t(h) * d; }
  }
  __device__ bool is_w2(int k) const {
    return (inner == TTT_INNER_MLP2_GELU || inner == TTT_INNER_SWIGLU) && k == (inner == TTT_INNER_SWIGLU ? 2 : 1);
  }
  // gradient-layout row of row r of a first-layer matrix k (W1, W3 or linear W)
  __device__ int grad_row(int k, int r) const {
    if (inner == TTT_INNER_LINEAR) return r;
    if (inner == TTT_INNER_GLU) return 128 * (r / 64) + (k == 0 ? 64 : 0) + (r % 64);  // [Wb 64 | Wa 64] blocks
    if (inner == TTT_INNER_MLP2_GELU) return h + r;
    return h + 256 * (r / 128) + (k == 1 ? 128 : 0) + (r % 128);
  }
  // bf16 first-layer row of row r of matrix k
  __device__ int first_row(int k, int r) const {
    if (inner == TTT_INNER_SWIGLU) return 256 * (r / 128) + (k == 1 ? 128 : 0) + (r % 128);
    if (inner == TTT_INNER_GLU) return 128 * (r / 64) + (k == 0 ? 64 : 0) + (r % 64);
    return r;
  }
};

// One warp per canonical weight row: [W -= lr U] -> [row L2-norm] -> bf16 copies
// (+ the non-finite check of the layer's weights).  W2^T is made from the bf16 W2
// afterwards by transpose_w2_kernel.
//   mode 0: no update (initial weights: W = W0 first when W0 is given; W0 [w0_rows][P],
//           row z % w0_rows for batch-head z)
//   mode 1: U from the gradient layout (w2t_u: W2's rows of it stored as [d][h] instead)
//   mode 2: U from the Newton-Schulz result (X [m][n], XT [n][m] per matrix)
//   mode 3: U summed here from the split-K partials part[splits][z][GR][d] (in split order,
//           as the split reduction would), with momentum M = beta M + U when Mom is given:
//           every element of the gradient layout belongs to exactly one row of one matrix
// hold_w2: the rows of W2 keep their values (first-layer-only updates): no step,
// no row norm; their bf16 copies are rewritten unchanged.
__global__ void finish_rows_kernel(RowMap rm, int mode, float lr, bool rownorm, bool hold_w2, float* Wf,
                                   const float* U, const float* X, const float* XT, int m, int n, bool src_t,
                                   bf16* First, bf16* W2T, bf16* W2, unsigned* status, const float* W0 = nullptr,
                                   int w0_rows = 1, const float* part = nullptr, int splits = 0, float* Mom = nullptr,
                                   float beta = 0.f, bool w2t_u = false) {
  const int z = blockIdx.y;
  const int R = blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
  if (R >= rm.nrows()) return;
  const int lane = threadIdx.x & 31;
  int k, r, len;
  int64_t off;
  rm.locate(R, k, r, len, off);
  float* w = Wf + z * rm.P + off + int64_t(r) * len;
  const bool w2 = rm.is_w2(k);
  const int nmat = rm.inner == TTT_INNER_LINEAR ? 1 : rm.inner == TTT_INNER_MLP2_GELU ? 2 : 3;
  if (w2 && hold_w2) {
    mode = 0;
    rownorm = false;
  }
  if (mode == 0 && W0) {
    const float* src = W0 + int64_t(z % w0_rows) * rm.P + off + int64_t(r) * len;
    for (int i = lane; i < len; i += 32) w[i] = src[i];
  }
  if (mode == 1) {
    const float* Uz = U + int64_t(z) * rm.GR * rm.d;
    if (!w2) {
      const float* u = Uz + int64_t(rm.grad_row(k, r)) * rm.d;
      for (int i = lane; i < len; i += 32) w[i] -= lr * u[i];
    } else if (w2t_u) {  // W2's update stored as [d][h]: row r is contiguous
      const float* u = Uz + int64_t(r) * rm.h;
      for (int i = lane; i < len; i += 32) w[i] -= lr * u[i];
    } else {  // W2 row r = column r of the G2^T rows [0, h)
      for (int i = lane; i < len; i += 32) w[i] -= lr * Uz[int64_t(i) * rm.d + r];
    }
  } else if (mode == 3) {
    const int64_t zoff = int64_t(z) * rm.GR * rm.d, sstride = int64_t(gridDim.y) * rm.GR * rm.d;
    auto grad = [&](int64_t idx) {
      float u = part[zoff + idx];
      for (int sp = 1; sp < splits; ++sp) u += part[sp * sstride + zoff + idx];
      if (Mom) {
        const float mm = beta * Mom[zoff + idx] + u;
        Mom[zoff + idx] = mm;
        u = mm;
      }
      return u;
    };
    if (!w2) {
      const int64_t g0 = int64_t(rm.grad_row(k, r)) * rm.d;
      for (int i = lane; i < len; i += 32) w[i] -= lr * grad(g0 + i);
    } else {  // W2 row r = column r of the G2^T rows [0, h)
      for (int i = lane; i < len; i += 32) w[i] -= lr * grad(int64_t(i) * rm.d + r);
    }
  } else if (mode == 2) {
    const int64_t mn = int64_t(m) * n;
    const float* Xk = X + (int64_t(z) * nmat + k) * mn;
    const float* XTk = XT + (int64_t(z) * nmat + k) * mn;
    // result in the source orientation is (src_t ? XT : X); W2 rows are its columns
    const float* src = w2 ? (src_t ? Xk : XTk) : (src_t ? XTk : Xk);
    const float* u = src + int64_t(r) * len;
    for (int i = lane; i < len; i += 32) w[i] -= lr * u[i];
  }
  float inv = 1.0f;
  if (rownorm) {
    float s = 0.f;
    for (int i = lane; i < len; i += 32) s += w[i] * w[i];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    inv = 1.0f / fmaxf(sqrtf(s), 1e-12f);
  }
  bool bad = false;
  if (!w2) {
    const int r1 = rm.inner == TTT_INNER_SWIGLU ? 2 * rm.h
                   : rm.inner == TTT_INNER_GLU   ? 2 * rm.d
                   : rm.inner == TTT_INNER_LINEAR ? rm.d
                                                  : rm.h;
    bf16* f = First + (int64_t(z) * r1 + rm.first_row(k, r)) * rm.d;
    for (int i = lane; i < len; i += 32) {
      const float v = w[i] * inv;
      w[i] = v;
      bad |= !isfinite(v);
      f[i] = __float2bfloat16_rn(v);
    }
  } else {
    bf16* w2row = W2 + (int64_t(z) * rm.d + r) * rm.h;
    for (int i = lane; i < len; i += 32) {
      const float v = w[i] * inv;
      w[i] = v;
      bad |= !isfinite(v);
      w2row[i] = __float2bfloat16_rn(v);
    }
  }
  if (__any_sync(0xffffffffu, bad) && lane == 0) set_status(status, kStatusNonFinite);
}

// W2^T [z][h][d] from W2 [z][d][h] (bf16) through 32 x 32 shared-memory tiles.
__global__ void transpose_w2_kernel(int d, int h, const bf16* W2, bf16* W2T) {
  __shared__ bf16 tile[32][34];
  const int z = blockIdx.z, c0 = blockIdx.x * 32, r0 = blockIdx.y * 32;  // rows of W2 = d, cols = h
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  const bf16* src = W2 + int64_t(z) * d * h;
  bf16* dst = W2T + int64_t(z) * d * h;
  for (int j = ty; j < 32; j += 8)
    if (r0 + j < d && c0 + tx < h) tile[j][tx] = src[int64_t(r0 + j) * h + c0 + tx];
  __syncthreads();
  for (int j = ty; j < 32; j += 8)
    if (c0 + j < h && r0 + tx < d) dst[int64_t(c0 + j) * d + r0 + tx] = tile[tx][j];
}

// Key instance-norm (per head, per channel, over the chunk's tokens).  Both passes
// move the keys in 16-byte pieces of 8 channels: thread t owns piece t % cpr of a row
// (cpr = channels / 8 of the current window of at most 2048 channels) and rows
// t / cpr, t / cpr + 256 / cpr, ...
//
// Pass 1: per (z, block of rb tokens), channel sums and sums of squares -> part[z][blk][ch][2].
// The block that finishes last for its head (a counter per head, reset by that block)
// combines the block sums in block order, in double (the biased variance is
// E[k^2] - E[k]^2), into the mean and 1/sqrt(var + eps) -> stats[z][ch][2].
__global__ void keystats_kernel(int n, int d, int rb, const bf16* K, int64_t k_zs, int t0, float eps, float* part,
                                float* stats, unsigned* done) {
  __shared__ float red[2][2048];  // [sum | sum of squares][row group x channel of the window]
  __shared__ bool last;
  const int z = blockIdx.y, blk = blockIdx.x, nb = gridDim.x;
  const int tid = threadIdx.x;
  const int rows = min(n - blk * rb, rb);
  for (int c0 = 0; c0 < d; c0 += 2048) {
    const int w = min(d - c0, 2048), cpr = w / 8, groups = 256 / cpr;
    const int piece = tid % cpr, grp = tid / cpr;
    float s[8] = {}, q[8] = {};
    if (grp < groups) {
      const bf16* base = K + z * k_zs + int64_t(t0 + int64_t(blk) * rb) * d + c0 + 8 * piece;
#pragma unroll 8
      for (int r = grp; r < rows; r += groups) {
        const uint4 u = *reinterpret_cast<const uint4*>(base + int64_t(r) * d);
        const uint32_t wd[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&wd[i]));
          s[2 * i] += f.x;
          s[2 * i + 1] += f.y;
          q[2 * i] = fmaf(f.x, f.x, q[2 * i]);
          q[2 * i + 1] = fmaf(f.y, f.y, q[2 * i + 1]);
        }
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        red[0][grp * w + 8 * piece + i] = s[i];
        red[1][grp * w + 8 * piece + i] = q[i];
      }
    }
    __syncthreads();
    for (int e = tid; e < 2 * w; e += blockDim.x) {
      const int which = e / w, ch = e % w;
      float t = 0.f;
      for (int gi = 0; gi < groups; ++gi) t += red[which][gi * w + ch];
      part[((int64_t(z) * nb + blk) * d + c0 + ch) * 2 + which] = t;
    }
    __syncthreads();
  }
  // the last block of head z to finish finalises its statistics
  __threadfence();
  __syncthreads();
  if (tid == 0) last = atomicAdd(&done[z], 1u) == static_cast<unsigned>(nb - 1);
  __syncthreads();
  if (!last) return;
  __threadfence();
  for (int ch = tid; ch < d; ch += blockDim.x) {
    double sum = 0.0, sq = 0.0;
    const float2* pz = reinterpret_cast<const float2*>(part) + int64_t(z) * nb * d + ch;
    int b = 0;
    // eight blocks' sums in flight at a time, added in block order
    for (; b + 8 <= nb; b += 8) {
      float2 v[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] = __ldcg(pz + int64_t(b + i) * d);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        sum += v[i].x;
        sq += v[i].y;
      }
    }
    for (; b < nb; ++b) {
      const float2 v = __ldcg(pz + int64_t(b) * d);
      sum += v.x;
      sq += v.y;
    }
    const double mean = sum / n;
    const double var = fmax(sq / n - mean * mean, 0.0);
    stats[(int64_t(z) * d + ch) * 2] = static_cast<float>(mean);
    stats[(int64_t(z) * d + ch) * 2 + 1] = static_cast<float>(1.0 / sqrt(var + eps));
  }
  if (tid == 0) done[z] = 0u;
}

// Pass 2: normalise the chunk's keys, Kn = (k - mean) * rstd, zeros for rows past the chunk.
__global__ void keynorm_kernel(int n, int d, const bf16* K, int64_t k_zs, int t0, const float* stats, bf16* Kn,
                               int64_t kn_zs) {
  extern __shared__ float st[];  // [d] mean, [d] rstd
  const int z = blockIdx.y, blk = blockIdx.x;
  for (int ch = threadIdx.x; ch < d; ch += blockDim.x) {
    st[ch] = stats[(int64_t(z) * d + ch) * 2];
    st[d + ch] = stats[(int64_t(z) * d + ch) * 2 + 1];
  }
  __syncthreads();
  const int cpr = d / 8;  // 16-byte pieces per row
  const int total = 128 * cpr;
#pragma unroll 4
  for (int e = threadIdx.x; e < total; e += blockDim.x) {
    const int r = e / cpr, ch = 8 * (e % cpr);
    const int row = blk * 128 + r;
    uint4 out = make_uint4(0u, 0u, 0u, 0u);
    if (row < n) {
      const uint4 u = *reinterpret_cast<const uint4*>(K + z * k_zs + int64_t(t0 + row) * d + ch);
      const uint32_t wd[4] = {u.x, u.y, u.z, u.w};
      uint32_t o[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&wd[i]));
        const int c = ch + 2 * i;
        const __nv_bfloat162 b = __floats2bfloat162_rn((f.x - st[c]) * st[d + c], (f.y - st[c + 1]) * st[d + c + 1]);
        o[i] = *reinterpret_cast<const uint32_t*>(&b);
      }
      out = make_uint4(o[0], o[1], o[2], o[3]);
    }
    *reinterpret_cast<uint4*>(Kn + z * kn_zs + int64_t(row) * d + ch) = out;
  }
}

// One warp per gradient row: sum the split-K partials in split order, momentum,
// write the update direction U and its squared norm.
__global__ void reduce_grad_kernel(int Z, int GR, int d, int splits, const float* part, bool momentum, float beta,
                                   float* Mom, float* U, float* rowsq) {
  const int z = blockIdx.y;
  const int g = blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
  if (g >= GR) return;
  const int lane = threadIdx.x & 31;
  const int64_t row = (int64_t(z) * GR + g) * d;
  const int64_t sstride = int64_t(Z) * GR * d;
  float sq = 0.f;
  for (int i = lane * 4; i < d; i += 128) {
    float4 acc = *reinterpret_cast<const float4*>(part + row + i);
    for (int s = 1; s < splits; ++s) {
      const float4 t = *reinterpret_cast<const float4*>(part + s * sstride + row + i);
      acc.x += t.x; acc.y += t.y; acc.z += t.z; acc.w += t.w;
    }
    if (momentum) {
      float4 m = *reinterpret_cast<const float4*>(Mom + row + i);
      m.x = beta * m.x + acc.x; m.y = beta * m.y + acc.y; m.z = beta * m.z + acc.z; m.w = beta * m.w + acc.w;
      *reinterpret_cast<float4*>(Mom + row + i) = m;
      acc = m;
    }
    *reinterpret_cast<float4*>(U + row + i) = acc;
    sq += acc.x * acc.x + acc.y * acc.y + acc.z * acc.z + acc.w * acc.w;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
  if (lane == 0 && rowsq) rowsq[int64_t(z) * GR + g] = sq;
}

// Newton-Schulz input of matrix k: its gradient-layout source M_src [rows_src][d]
// scaled by 1/(||M_src||_F + 1e-7), written in source orientation to A and transposed
// to B.  (X0, X0^T) = src_t ? (B, A) : (A, B).  Every CTA of the matrix sums the squared
// row norms (rowsq) itself, in the same fixed order, so all of them scale by the same value.
__global__ void ns_prep_kernel(RowMap rm, int nmat, const float* U, const float* rowsq, float* A, float* Bt) {
  __shared__ float tile[32][33];
  __shared__ float red[256];
  const int zk = blockIdx.z, z = zk / nmat, k = zk % nmat;
  const int rows_src = rm.inner == TTT_INNER_LINEAR ? rm.d : rm.h;
  const int d = rm.d;
  const bool w2 = rm.is_w2(k);
  const int r0 = blockIdx.y * 32, c0 = blockIdx.x * 32;
  {
    float q = 0.f;
    for (int r = threadIdx.x; r < rows_src; r += blockDim.x)
      q += rowsq[int64_t(z) * rm.GR + (w2 ? r : rm.grad_row(k, r))];
    red[threadIdx.x] = q;
    __syncthreads();
    for (int w = blockDim.x / 2; w > 0; w >>= 1) {
      if (threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
      __syncthreads();
    }
  }
  const float s = 1.0f / (sqrtf(red[0]) + 1e-7f);
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;  // 32 x 8 threads
  const int64_t mn = int64_t(rows_src) * d;
  for (int j = ty; j < 32; j += 8) {
    const int r = r0 + j, c = c0 + tx;
    float v = 0.f;
    if (r < rows_src && c < d) {
      const int g = w2 ? r : rm.grad_row(k, r);
      v = U[(int64_t(z) * rm.GR + g) * d + c] * s;
      A[zk * mn + int64_t(r) * d + c] = v;
    }
    tile[j][tx] = v;
  }
  __syncthreads();
  for (int j = ty; j < 32; j += 8) {
    const int c = c0 + j, r = r0 + tx;
    if (r < rows_src && c < d) Bt[zk * mn + int64_t(c) * rows_src + r] = tile[tx][j];
  }
}

// linear + negative dot loss: dY = -eta_t v_t for the chunk's rows (zeros past it)
__global__ void neg_eta_rows_kernel(int n, int Cp, int d, const bf16* V, int64_t v_zs, int t0, const float* eta,
                                    int64_t eta_zs, float eta_scalar, bf16* dY, int64_t y_zs) {
  const int z = blockIdx.y;
  for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < int64_t(Cp) * d; i += int64_t(gridDim.x) * blockDim.x) {
    const int r = int(i / d), c = int(i % d);
    float v = 0.f;
    if (r < n) {
      const float e = eta ? eta[z * eta_zs + t0 + r] : eta_scalar;
      v = -e * __bfloat162float(V[z * v_zs + int64_t(t0 + r) * d + c]);
    }
    dY[z * y_zs + i] = __float2bfloat16_rn(v);
  }
}

// RMSE loss: the MSE gradient dY = 2 eta (V_hat - V) / (n d) is already in DY (bf16,
// rows [0, n) of each z).  Per z, L = sqrt(sum eta (V_hat - V)^2 / (n d)), recovered from
// dY as sqrt(sum_{eta != 0} dY^2 / eta * n d / 4); then dY <- dY / (2 L), the RMSE
// gradient (zero where L = 0).  One CTA of 256 threads per z, fixed-order reduction.
__global__ void rmse_scale_kernel(int n, int d, bf16* DY, int64_t y_zs, int t0, const float* eta, int64_t eta_zs,
                                  float eta_scalar) {
  __shared__ float red[256];
  const int z = blockIdx.x;
  bf16* y = DY + z * y_zs;
  const int64_t total = int64_t(n) * d;
  float s = 0.f;
  for (int64_t i = threadIdx.x; i < total; i += blockDim.x) {
    const float e = eta ? eta[z * eta_zs + t0 + int(i / d)] : eta_scalar;
    const float v = __bfloat162float(y[i]);
    if (e != 0.f) s += v * v / e;
  }
  red[threadIdx.x] = s;
  __syncthreads();
  for (int w = blockDim.x / 2; w > 0; w >>= 1) {
    if (threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
    __syncthreads();
  }
  const float L = sqrtf(fmaxf(red[0] * (float(n) * float(d) * 0.25f), 0.f));
  const float scale = L > 0.f ? 0.5f / L : 0.f;
  for (int64_t i = threadIdx.x; i < total; i += blockDim.x) y[i] = __float2bfloat16_rn(__bfloat162float(y[i]) * scale);
}

// ------------------------------------------------------------------ host helpers
struct BView {
  uint8_t* base;
  unsigned* status;
  template <typename T>
  T* at(const Plan& p, int i) const { return reinterpret_cast<T*>(base + p.off[i]); }
};

#define TRY(x)                       \
  do {                               \
    int _r = (x);                    \
    if (_r != TTT_OK) return _r;     \
  } while (0)
#define TRY_CUDA(x)                               \
  do {                                            \
    if ((x) != cudaSuccess) return TTT_ERR_CUDA;  \
  } while (0)

// A TMA map plus the box it was encoded with (checked against every launch).
struct TM {
  CUtensorMap m;
  int box = 0;
  int eb = 0;
};

// row-major [Z][rows][cols] view as a TMA map; box rows `box`
int tmap(TM* t, const void* p, int eb, int64_t cols, int64_t rows, int64_t Z, int box) {
  t->box = box;
  t->eb = eb;
  return make_tmap(&t->m, p, eb, cols, rows, Z, cols, cols * rows, box) ? TTT_OK : TTT_ERR_INVALID_ARG;
}

// Launch through the engine after checking that every map's box matches the
// tile the kernel loads (K-major: the tile's rows; MN-major: 128/EB rows), so the
// bytes a stage expects are exactly the bytes TMA delivers.
template <int BN0, int BN1, bool AMN, bool BMN, int EB, int STAGES, int EW = 4, class Epi>
int gemm(const TM& a0, const TM& b0, const TM& a1, const TM& b1, const TcGeom& g, const Epi& e, unsigned* status,
         cudaStream_t st, bool persistent = false) {
  const int run = 128 / EB;
  const int ra = AMN ? run : 128;
  const int rb0 = BMN ? run : BN0;
  const int rb1 = BMN ? run : (BN1 > 0 ? BN1 : BN0);
  const bool second = BN1 > 0 || g.m_tiles1 > 0;
  if (a0.box != ra || b0.box != rb0 || a0.eb != EB || b0.eb != EB) return TTT_ERR_INVALID_ARG;
  if (second && (a1.box != ra || b1.box != rb1 || a1.eb != EB || b1.eb != EB)) return TTT_ERR_INVALID_ARG;
  if (g.kblocks <= 0 || g.kb_per_split <= 0) return TTT_ERR_INVALID_ARG;
  StageScope sc(g_stage, st);
  return launch_tc_gemm<BN0, BN1, AMN, BMN, EB, STAGES, EW>(a0.m, b0.m, a1.m, b1.m, g, e, status, st, persistent) ==
                 cudaSuccess
             ? TTT_OK
             : TTT_ERR_CUDA;
}

TcGeom geom(int mt0, int mt1, int nt, int kblocks, int Z, int splits) {
  TcGeom g;
  g.m_tiles0 = mt0;
  g.m_tiles1 = mt1;
  g.n_tiles = nt;
  g.kblocks = kblocks;
  g.batches = Z;
  g.kb_per_split = (kblocks + splits - 1) / splits;
  g.splits = (kblocks + g.kb_per_split - 1) / g.kb_per_split;
  return g;
}

struct Ctx {
  const Plan& p;
  Dims D;
  BView v;
  const Io& io;
  cudaStream_t st;
  RowMap rm;
  TM tK, tV, tKmn, tVmn, tQ, tFirst, tW2T, tW2;
  int bn_first = 0;
  bool apply_pending = false;  // an apply on io.aux still reads the bf16 weight copies
};

// An unsplit plain or momentum step of a model with W2 stores W2's update (G2^T) in U
// transposed, as [d][h] (EpiGradDirect::w2t_h): nothing else reads those rows of U then.
bool w2_update_transposed(const Ctx& c) {
  const ttt_config& cfg = c.p.cfg;
  const bool muon = cfg.opt == TTT_OPT_MUON || cfg.opt == TTT_OPT_MOMENTUM_MUON;
  return c.D.direct && !muon && (cfg.inner == TTT_INNER_MLP2_GELU || cfg.inner == TTT_INNER_SWIGLU);
}

// bf16 W2^T from the freshly written bf16 W2: the B operand of the single-CTA token
// kernel and of the generic MSE path's dH = dY W2.  The pair token kernel, the fused MSE
// token kernel and the apply read W2 itself.
int transpose_w2(Ctx& c) {
  const ttt_config& cfg = c.p.cfg;
  if (cfg.inner == TTT_INNER_LINEAR || cfg.inner == TTT_INNER_GLU || mse_token_path(cfg)) return TTT_OK;
  if (cfg.loss == TTT_LOSS_NEG_DOT && c.D.token_pairs &&
      (cfg.inner == TTT_INNER_SWIGLU ? token_pair_capacity<true>() : token_pair_capacity<false>()) > 0)
    return TTT_OK;
  const Dims& D = c.D;
  cudaStream_t st = c.st;
  {
    StageScope _sc(kStageFinish, st);
    transpose_w2_kernel<<<dim3((D.h + 31) / 32, (D.d + 31) / 32, D.Z), 256, 0, st>>>(
        D.d, D.h, c.v.at<bf16>(c.p, xW2), c.v.at<bf16>(c.p, xW2T));
  }
  return cudaGetLastError() == cudaSuccess ? TTT_OK : TTT_ERR_CUDA;
}

// update-direction -> weights (+ Newton-Schulz when the optimizer is Muon)
int optimizer_step(Ctx& c) {
  cudaStream_t st = c.st;
  // the chunk's apply on the side stream reads the bf16 weights this step rewrites
  if (c.apply_pending) {
    TRY_CUDA(cudaStreamWaitEvent(st, c.io.ev_join, 0));
    c.apply_pending = false;
  }
  const Plan& p = c.p;
  const Dims& D = c.D;
  const ttt_config& cfg = p.cfg;
  const bool mom = cfg.opt == TTT_OPT_MOMENTUM || cfg.opt == TTT_OPT_MOMENTUM_MUON;
  const bool muon = cfg.opt == TTT_OPT_MUON || cfg.opt == TTT_OPT_MOMENTUM_MUON;
  const bool hold_w2 = (cfg.flags & TTT_FLAG_FIRST_LAYER_ONLY) != 0;
  // plain and momentum steps of models without W2 (linear, GLU) sum the split partials
  // inside the row finish (no separate reduction pass).  Not with W2: its rows' updates are
  // strided columns of G2^T, and summing the partials there costs more than the reduction
  // saves; nor with Muon, which needs the reduced rows and their norms first.
  const bool fold = !D.direct && !muon && !hold_w2 && (cfg.inner == TTT_INNER_LINEAR || cfg.inner == TTT_INNER_GLU);
  if (!D.direct && !fold) {
    dim3 g((D.GR + 7) / 8, D.Z);
    {
      StageScope _sc(kStageReduce, st);
      reduce_grad_kernel<<<g, 256, 0, c.st>>>(D.Z, D.GR, D.d, D.splits, c.v.at<float>(p, xPart), mom, cfg.momentum,
                                              c.v.at<float>(p, xMom), c.v.at<float>(p, xU),
                                              muon ? c.v.at<float>(p, xRowSq) : nullptr);
    }
    TRY_CUDA(cudaGetLastError());
  }
  float* X = c.v.at<float>(p, xNX);
  float* XT = c.v.at<float>(p, xNXT);
  if (muon) {
    const int ZK = D.Z * D.nmat;
    const int rows_src = cfg.inner == TTT_INNER_LINEAR ? D.d : D.h;
    dim3 g((D.d + 31) / 32, (rows_src + 31) / 32, ZK);
    float* A = D.src_t ? XT : X;
    float* B = D.src_t ? X : XT;
    {
      StageScope _sc(kStageNewtonSchulz, st);
      ns_prep_kernel<<<g, 256, 0, c.st>>>(c.rm, D.nmat, c.v.at<float>(p, xU), c.v.at<float>(p, xRowSq), A, B);
    }
    TRY_CUDA(cudaGetLastError());
    // all Newton-Schulz iterations of every matrix in one clustered launch
    NsGeom ng;
    ng.m = D.m;
    ng.n = D.n;
    ng.iters = cfg.ns_iters;
    ng.a = cfg.ns_coeff[0];
    ng.b = cfg.ns_coeff[1];
    ng.c = cfg.ns_coeff[2];
    ng.X = X;
    ng.XT = XT;
    ng.X2 = c.v.at<float>(p, xNX2);
    ng.XT2 = c.v.at<float>(p, xNXT2);
    ng.S = c.v.at<float>(p, xNS);
    ng.T = c.v.at<float>(p, xNT);
    {
      StageScope sc(kStageNewtonSchulz, st);
      TRY_CUDA(launch_ns_fused(ZK, ng, c.v.status, st));
    }
    if (cfg.ns_iters & 1) {
      X = ng.X2;
      XT = ng.XT2;
    }
  }
  dim3 g((c.rm.nrows() + 7) / 8, D.Z);
  {
    StageScope _sc(kStageFinish, st);
    finish_rows_kernel<<<g, 256, 0, c.st>>>(c.rm, muon ? 2 : fold ? 3 : 1, cfg.lr,
                                            (cfg.flags & TTT_FLAG_WEIGHT_L2NORM) != 0, hold_w2, c.v.at<float>(p, xWf),
                                            c.v.at<float>(p, xU), X, XT, D.m, D.n, D.src_t, c.v.at<bf16>(p, xFirst),
                                            c.v.at<bf16>(p, xW2T), c.v.at<bf16>(p, xW2), c.v.status, nullptr, 1,
                                            c.v.at<float>(p, xPart), D.splits, mom ? c.v.at<float>(p, xMom) : nullptr,
                                            cfg.momentum, w2_update_transposed(c));
  }
  TRY_CUDA(cudaGetLastError());
  return transpose_w2(c);
}

// Weight-gradient token reductions of one chunk: problem 0 (rows0 output rows of
// the gradient layout, from row 0) and, when rows1 > 0, problem 1 (rows1 rows, from
// row r1), both N = d, K = the chunk's padded tokens.  Split-K writes fp32 partials
// for reduce_grad_kernel; an unsplit reduction writes U (and M) directly.
template <class Epi>
int grad_launch(Ctx& c, const TM& a0, const TM& b0, const TM& a1, const TM& b1, int rows0, int rows1, int b0k,
                int b1k, const Epi& ep) {
  const Dims& D = c.D;
  const int d = D.d, bnd = D.grad_bn, kbt = D.Cp / 64;
  unsigned* status = c.v.status;
  if (a0.box != 64 || b0.box != 64 || (rows1 > 0 && (a1.box != 64 || b1.box != 64))) return TTT_ERR_INVALID_ARG;
  if (D.tile_rows == 512 && rows0 % 512 == 0 && rows1 % 512 == 0 && (bnd == 256 || bnd == 128) &&
      (bnd == 256 ? wgrad_pair_capacity<256, 4, Epi>() : wgrad_pair_capacity<128, 5, Epi>()) > 0) {
    TcGeom gg = geom(rows0 / 512, rows1 / 512, d / bnd, kbt, D.Z, D.splits);
    gg.b0.k = b0k;
    gg.b1.k = b1k;
    StageScope sc(kStageWeightGrad, c.st);
    cudaError_t e = bnd == 256 ? launch_wgrad_pair<256, 4>(a0.m, b0.m, a1.m, b1.m, gg, ep, status, c.st)
                               : launch_wgrad_pair<128, 5>(a0.m, b0.m, a1.m, b1.m, gg, ep, status, c.st);
    return e == cudaSuccess ? TTT_OK : TTT_ERR_CUDA;
  }
  if (D.tile_rows >= 256 && rows0 % 256 == 0 && rows1 % 256 == 0) {
    TcGeom gg = geom(rows0 / 256, rows1 / 256, d / bnd, kbt, D.Z, D.splits);
    gg.b0.k = b0k;
    gg.b1.k = b1k;
    StageScope sc(kStageWeightGrad, c.st);
    cudaError_t e = bnd == 256 ? launch_wgrad<256, 3>(a0.m, b0.m, a1.m, b1.m, gg, ep, status, c.st)
                    : bnd == 128 ? launch_wgrad<128, 4>(a0.m, b0.m, a1.m, b1.m, gg, ep, status, c.st)
                                 : launch_wgrad<64, 4>(a0.m, b0.m, a1.m, b1.m, gg, ep, status, c.st);
    return e == cudaSuccess ? TTT_OK : TTT_ERR_CUDA;
  }
  TcGeom gg = geom(rows0 / 128, rows1 / 128, d / bnd, kbt, D.Z, D.splits);
  gg.b0.k = b0k;
  gg.b1.k = b1k;
  if (bnd == 256) return gemm<256, 0, true, true, 2, 4, 8>(a0, b0, a1, b1, gg, ep, status, c.st, true);
  if (bnd == 128) return gemm<128, 0, true, true, 2, 6, 8>(a0, b0, a1, b1, gg, ep, status, c.st, true);
  return gemm<64, 0, true, true, 2, 4, 8>(a0, b0, a1, b1, gg, ep, status, c.st, true);
}

int grad_gemm(Ctx& c, const TM& a0, const TM& b0, const TM& a1, const TM& b1, int rows0, int rows1, int r1, int b0k,
              int b1k) {
  const Plan& p = c.p;
  const Dims& D = c.D;
  const ttt_config& cfg = p.cfg;
  const int d = D.d;
  const int64_t pz = int64_t(D.GR) * d;
  StageCtx stage(kStageWeightGrad);
  if (!D.direct) {
    EpiPartial ep{c.v.at<float>(p, xPart), int64_t(D.Z) * pz, pz, d, {0, r1}, {rows0, rows1}};
    return grad_launch(c, a0, b0, a1, b1, rows0, rows1, b0k, b1k, ep);
  }
  const bool mom = cfg.opt == TTT_OPT_MOMENTUM || cfg.opt == TTT_OPT_MOMENTUM_MUON;
  const bool muon = cfg.opt == TTT_OPT_MUON || cfg.opt == TTT_OPT_MOMENTUM_MUON;
  float* rowsq = muon ? c.v.at<float>(p, xRowSq) : nullptr;
  if (rowsq && cudaMemsetAsync(rowsq, 0, size_t(D.Z) * D.GR * 4, c.st) != cudaSuccess) return TTT_ERR_CUDA;
  EpiGradDirect ep{c.v.at<float>(p, xU), mom ? c.v.at<float>(p, xMom) : nullptr, rowsq, cfg.momentum, pz, d,
                   {0, r1}, {rows0, rows1}, w2_update_transposed(c) ? D.h : 0};
  return grad_launch(c, a0, b0, a1, b1, rows0, rows1, b0k, b1k, ep);
}

// RMSE: rescale the chunk's MSE gradient in DY by 1/(2 RMSE) per head.
int rmse_scale(Ctx& c, bf16* DY, int t0, int n) {
  {
    StageScope _sc(kStageKeyNorm, c.st);
    rmse_scale_kernel<<<c.D.Z, 256, 0, c.st>>>(n, c.D.d, DY, int64_t(c.D.Cp) * c.D.d, t0, c.io.eta, c.D.N,
                                               c.p.cfg.eta_scalar);
  }
  return cudaGetLastError() == cudaSuccess ? TTT_OK : TTT_ERR_CUDA;
}

// Token phase of the negative-dot update: activations H' and dZ(13) of chunk
// tokens [t0, t0+n) for the weight-gradient GEMMs (token_phase.cuh).
int token_phase(Ctx& c, const TM& tX, int xoff, int t0, int n, bf16* Hp, bf16* dZ, bool swiglu) {
  const Dims& D = c.D;
  const int Z = D.Z, d = D.d, h = D.h, Cp = D.Cp;
  const int dzc = swiglu ? 2 * h : h;
  // CTA pairs (256-token tiles) when a pair can be resident; each CTA then loads
  // half of every weight block: [W1_blk; W3_blk] rows by halves, W2^T rows by halves
  const bool pairs = D.token_pairs && (swiglu ? token_pair_capacity<true>() : token_pair_capacity<false>()) > 0;
  // output boxes: [32 rows][16 columns] (pair kernel) or [32 rows][32 columns]
  const int bc = pairs ? 16 : 32;
  CUtensorMap sH, sD;
  if (!make_tmap_ex(&sH, Hp, 2, h, Cp, Z, h, int64_t(Cp) * h, bc, 32, 2 * bc) ||
      !make_tmap_ex(&sD, dZ, 2, dzc, Cp, Z, dzc, int64_t(Cp) * dzc, bc, 32, 2 * bc))
    return TTT_ERR_INVALID_ARG;
  const int bz = swiglu ? 256 : 128;
  if (tX.box != 128 || c.tV.box != 128 || c.tW2T.box != 128 || c.tFirst.box != bz) return TTT_ERR_INVALID_ARG;
  TokGeom g;
  g.m_tiles = Cp / 128;
  g.n_tiles = h / 128;
  g.batches = Z;
  g.kblocks = d / 64;
  g.x_off = xoff;
  g.v_off = t0;
  g.rows_valid = n;
  g.rows_alloc = Cp;
  g.t0 = t0;
  g.eta = c.io.eta;
  g.eta_zs = D.N;
  g.eta_scalar = c.p.cfg.eta_scalar;
  StageScope sc(kStageTokenPhase, c.st);
  cudaError_t e;
  if (pairs) {
    TM fh, wh;
    TRY(tmap(&fh, c.v.at<bf16>(c.p, xFirst), 2, d, D.R1, Z, swiglu ? 128 : 64));
    TRY(tmap(&wh, c.v.at<bf16>(c.p, xW2), 2, h, d, Z, 64));  // W2 [d][h], MN-major 64 x 64 boxes
    g.m_tiles = (Cp + 255) / 256;
    e = swiglu ? launch_token_pair<true>(tX.m, fh.m, c.tV.m, wh.m, sH, sD, g, c.v.status, c.st)
               : launch_token_pair<false>(tX.m, fh.m, c.tV.m, wh.m, sH, sD, g, c.v.status, c.st);
  } else {
    e = swiglu ? launch_token_dot<true>(tX.m, c.tFirst.m, c.tV.m, c.tW2T.m, sH, sD, g, c.v.status, c.st)
               : launch_token_dot<false>(tX.m, c.tFirst.m, c.tV.m, c.tW2T.m, sH, sD, g, c.v.status, c.st);
  }
  return e == cudaSuccess ? TTT_OK : TTT_ERR_CUDA;
}

// one chunk's weight update: tokens [t0, t0+n)
int update_chunk(Ctx& c, int t0, int n) {
  cudaStream_t st = c.st;
  const Plan& p = c.p;
  const Dims& D = c.D;
  const ttt_config& cfg = p.cfg;
  const int Z = D.Z, d = D.d, h = D.h, Cp = D.Cp;
  const bf16* K = static_cast<const bf16*>(c.io.K);
  const bf16* V = static_cast<const bf16*>(c.io.V);
  // keys: the input (token offset t0) or their instance-normalised copy (offset 0)
  const TM* tX = &c.tK;
  const TM* tXmn = &c.tKmn;
  int xoff = t0;
  TM tKn, tKnmn;
  const float* kstats = nullptr;  // per-channel key statistics the fused MSE kernel applies itself
  if (cfg.flags & TTT_FLAG_KEY_INSTNORM) {
    float* kst = c.v.at<float>(p, xKstat);
    // blocks of rb tokens: about two blocks per SM over all heads, each with many loads in flight
    const int rb = static_cast<int>(std::max<int64_t>(128, std::min<int64_t>(1024, (int64_t(n) * Z / (2 * kPlanSMs) + 127) / 128 * 128)));
    const int nb = (n + rb - 1) / rb;
    float* kfin = kst + size_t(Z) * (Cp / 128) * d * 2;                   // [Z][d][2] mean, rstd
    unsigned* kdone = reinterpret_cast<unsigned*>(kfin + size_t(Z) * d * 2);  // [Z] blocks finished
    {
      StageScope _sc(kStageKeyNorm, st);
      keystats_kernel<<<dim3(nb, Z), 256, 0, c.st>>>(n, d, rb, K, int64_t(D.N) * d, t0, cfg.in_eps, kst, kfin,
                                                     kdone);
    }
    TRY_CUDA(cudaGetLastError());
    kstats = kfin;
  }
  if ((cfg.flags & TTT_FLAG_KEY_INSTNORM) && !mse_token_path(cfg)) {
    bf16* Kn = c.v.at<bf16>(p, xKn);
    const dim3 gk(Cp / 128, Z);
    {
      StageScope _sc(kStageKeyNorm, st);
      keynorm_kernel<<<gk, 256, 2 * d * sizeof(float), c.st>>>(n, d, K, int64_t(D.N) * d, t0, kstats, Kn,
                                                               int64_t(Cp) * d);
    }
    TRY_CUDA(cudaGetLastError());
    TRY(tmap(&tKn, Kn, 2, d, Cp, Z, 128));
    TRY(tmap(&tKnmn, Kn, 2, d, Cp, Z, 64));
    tX = &tKn;
    tXmn = &tKnmn;
    xoff = 0;
  }
  bf16* A0 = c.v.at<bf16>(p, xAct0);
  bf16* A1 = c.v.at<bf16>(p, xAct1);
  bf16* A2 = c.v.at<bf16>(p, xAct2);
  bf16* DY = c.v.at<bf16>(p, xDY);
  const int bnd = bn_for(d);
  unsigned* status = c.v.status;
  const int mt = Cp / 128;

  StageCtx stage(kStageTokenPhase);
  if (cfg.inner == TTT_INNER_SWIGLU) {
    // token phase: p = V W2[:, blk], [z1 | z3] = X [W1;W3]_blk^T  -> H', dZ13
    TRY(token_phase(c, *tX, xoff, t0, n, A0, A1, true));
    // weight gradients: G2^T = H'^T V  (rows [0,h)),  G13 = dZ13^T X  (rows [h, 3h))
    TM tH, tD;
    TRY(tmap(&tH, A0, 2, h, Cp, Z, 64));
    TRY(tmap(&tD, A1, 2, 2 * h, Cp, Z, 64));
    TRY(grad_gemm(c, tH, c.tVmn, tD, *tXmn, h, 2 * h, h, t0, xoff));
  } else if (cfg.inner == TTT_INNER_MLP2_GELU && cfg.loss == TTT_LOSS_NEG_DOT) {
    TRY(token_phase(c, *tX, xoff, t0, n, A0, A1, false));
    TM tH, tD;
    TRY(tmap(&tH, A0, 2, h, Cp, Z, 64));
    TRY(tmap(&tD, A1, 2, h, Cp, Z, 64));
    TRY(grad_gemm(c, tH, c.tVmn, tD, *tXmn, h, h, h, t0, xoff));
  } else if (mse_token_path(cfg)) {
    // one kernel: Z, GELU, V_hat, the MSE gradient, dH, dZ and the gradient reductions
    // G2^T = H^T dY, G1 = dZ^T X per (head, token-tile range) -> split partials (mse_token.cuh)
    TM tw1, tw2;
    TRY(tmap(&tw1, c.v.at<bf16>(p, xFirst), 2, d, h, Z, h));
    TRY(tmap(&tw2, c.v.at<bf16>(p, xW2), 2, h, d, Z, 64));
    if (tX->box != 128 || c.tV.box != 128 || D.direct) return TTT_ERR_INVALID_ARG;
    MseGeom mg;
    mg.m_tiles = (n + 127) / 128;
    mg.batches = Z;
    mg.splits = D.splits;
    mg.rows_valid = n;
    mg.x_off = xoff;
    mg.v_off = t0;
    mg.t0 = t0;
    mg.eta = c.io.eta;
    mg.eta_zs = D.N;
    mg.eta_scalar = cfg.eta_scalar;
    mg.coef = 2.0f / (float(n) * float(d));
    mg.part = c.v.at<float>(p, xPart);
    mg.kstats = kstats;  // key instance-norm applied to the raw key tiles in the kernel
    {
      StageScope sc(kStageTokenPhase, c.st);
      const cudaError_t e = h == 256 ? launch_mse_token<256>(tX->m, c.tV.m, tw1.m, tw2.m, mg, status, c.st)
                                     : launch_mse_token<128>(tX->m, c.tV.m, tw1.m, tw2.m, mg, status, c.st);
      TRY_CUDA(e);
    }
  } else if (cfg.inner == TTT_INNER_MLP2_GELU) {  // MSE, RMSE
    // Z = X W1^T -> H = GELU(Z), G' = GELU'(Z)
    EpiGeluSave e1{A0, A2, h, n, int64_t(Cp) * h};
    TcGeom g1 = geom(mt, 0, h / bn_for(h), d / 64, Z, 1);
    g1.a0.mn = xoff;
    if (bn_for(h) == 256) TRY((gemm<256, 0, false, false, 2, 4, 8>(*tX, c.tFirst, *tX, c.tFirst, g1, e1, status, c.st, true)));
    else TRY((gemm<128, 0, false, false, 2, 4, 8>(*tX, c.tFirst, *tX, c.tFirst, g1, e1, status, c.st, true)));
    // V_hat = H W2^T -> dY = 2 eta (V_hat - V)/(n d)
    TM tHk, tY, tYmn, tH, tD;
    TRY(tmap(&tHk, A0, 2, h, Cp, Z, 128));
    EpiMseGrad e2{DY, d, n, int64_t(Cp) * d, V, int64_t(D.N) * d, t0, c.io.eta, D.N, cfg.eta_scalar,
                  2.0f / (float(n) * float(d))};
    TcGeom g2 = geom(mt, 0, d / bnd, h / 64, Z, 1);
    if (bnd == 256) TRY((gemm<256, 0, false, false, 2, 4, 8>(tHk, c.tW2, tHk, c.tW2, g2, e2, status, c.st, true)));
    else if (bnd == 128) TRY((gemm<128, 0, false, false, 2, 4, 8>(tHk, c.tW2, tHk, c.tW2, g2, e2, status, c.st, true)));
    else TRY((gemm<64, 0, false, false, 2, 4, 8>(tHk, c.tW2, tHk, c.tW2, g2, e2, status, c.st, true)));
    if (cfg.loss == TTT_LOSS_RMSE) TRY(rmse_scale(c, DY, t0, n));
    // dH = dY W2 -> dZ = dH G'
    TRY(tmap(&tY, DY, 2, d, Cp, Z, 128));
    EpiMulSaved e3{A1, A2, h, int64_t(Cp) * h};
    TcGeom g3 = geom(mt, 0, h / bn_for(h), d / 64, Z, 1);
    if (bn_for(h) == 256) TRY((gemm<256, 0, false, false, 2, 4, 8>(tY, c.tW2T, tY, c.tW2T, g3, e3, status, c.st, true)));
    else TRY((gemm<128, 0, false, false, 2, 4, 8>(tY, c.tW2T, tY, c.tW2T, g3, e3, status, c.st, true)));
    // G2^T = H^T dY (rows [0,h)), G1 = dZ^T X (rows [h,2h))
    TRY(tmap(&tH, A0, 2, h, Cp, Z, 64));
    TRY(tmap(&tYmn, DY, 2, d, Cp, Z, 64));
    TRY(tmap(&tD, A1, 2, h, Cp, Z, 64));
    TRY(grad_gemm(c, tH, tYmn, tD, *tXmn, h, h, h, 0, xoff));
  } else if (glu_update_path(cfg)) {
    // one kernel: Z = X [Wb; Wa]^T, the gating gradient and G = dZ^T X per (head, token-tile
    // range) -> split partials (glu_update.cuh)
    TM tw;
    TRY(tmap(&tw, c.v.at<bf16>(p, xFirst), 2, d, 2 * d, Z, 128));
    if (tX->box != 128 || c.tV.box != 128 || D.direct) return TTT_ERR_INVALID_ARG;
    GluGeom gg;
    gg.m_tiles = (n + 127) / 128;
    gg.batches = Z;
    gg.splits = D.splits;
    gg.rows_valid = n;
    gg.x_off = xoff;
    gg.v_off = t0;
    gg.t0 = t0;
    gg.eta = c.io.eta;
    gg.eta_zs = D.N;
    gg.eta_scalar = cfg.eta_scalar;
    gg.mse = cfg.loss == TTT_LOSS_MSE ? 1 : 0;
    gg.coef = 2.0f / (float(n) * float(d));
    gg.part = c.v.at<float>(p, xPart);
    {
      StageScope sc(kStageTokenPhase, c.st);
      TRY_CUDA(launch_glu_update(tX->m, c.tV.m, tw.m, gg, status, c.st));
    }
  } else if (cfg.inner == TTT_INNER_GLU) {
    // Z = X [Wb_blk; Wa_blk]^T per 64-channel block -> dZ (gate, linear), then G = dZ^T X
    EpiGluGrad eg{A1, d, n, int64_t(Cp) * 2 * d, V, int64_t(D.N) * d, t0, c.io.eta, D.N, cfg.eta_scalar,
                  cfg.loss == TTT_LOSS_MSE ? 1 : 0, 2.0f / (float(n) * float(d))};
    TcGeom gz = geom(mt, 0, (2 * d) / 128, d / 64, Z, 1);
    gz.a0.mn = xoff;
    TRY((gemm<128, 0, false, false, 2, 4, 8>(*tX, c.tFirst, *tX, c.tFirst, gz, eg, status, c.st, true)));
    TM tD;
    TRY(tmap(&tD, A1, 2, 2 * d, Cp, Z, 64));
    TRY(grad_gemm(c, tD, *tXmn, tD, *tXmn, 2 * d, 0, 0, xoff, 0));
  } else {  // linear
    if (cfg.loss != TTT_LOSS_NEG_DOT) {  // MSE, RMSE
      EpiMseGrad e2{DY, d, n, int64_t(Cp) * d, V, int64_t(D.N) * d, t0, c.io.eta, D.N, cfg.eta_scalar,
                    2.0f / (float(n) * float(d))};
      TcGeom g2 = geom(mt, 0, d / bnd, d / 64, Z, 1);
      g2.a0.mn = xoff;
      if (bnd == 256) TRY((gemm<256, 0, false, false, 2, 4, 8>(*tX, c.tFirst, *tX, c.tFirst, g2, e2, status, c.st, true)));
      else if (bnd == 128) TRY((gemm<128, 0, false, false, 2, 4, 8>(*tX, c.tFirst, *tX, c.tFirst, g2, e2, status, c.st, true)));
      else TRY((gemm<64, 0, false, false, 2, 4, 8>(*tX, c.tFirst, *tX, c.tFirst, g2, e2, status, c.st, true)));
      if (cfg.loss == TTT_LOSS_RMSE) TRY(rmse_scale(c, DY, t0, n));
    } else {
      {
        StageScope _sc(kStageKeyNorm, st);
        neg_eta_rows_kernel<<<dim3(64, Z), 256, 0, c.st>>>(n, Cp, d, V, int64_t(D.N) * d, t0, c.io.eta, D.N,
                                                           cfg.eta_scalar, DY, int64_t(Cp) * d);
      }
      TRY_CUDA(cudaGetLastError());
    }
    TM tYmn;
    TRY(tmap(&tYmn, DY, 2, d, Cp, Z, 64));
    TRY(grad_gemm(c, tYmn, *tXmn, tYmn, *tXmn, d, 0, 0, xoff, 0));
  }
  return optimizer_step(c);
}

// O rows [row0, row0 + rows) = F_W(Q rows [row0, row0 + rows))
int apply_rows(Ctx& c, int row0, int rows) {
  StageCtx stage(kStageApply);
  const Plan& p = c.p;
  const Dims& D = c.D;
  const ttt_config& cfg = p.cfg;
  const int Z = D.Z, d = D.d, h = D.h;
  const int mt = (rows + 127) / 128;
  const int bnd = bn_for(d);
  unsigned* status = c.v.status;
  bf16* O = static_cast<bf16*>(c.io.O);
  EpiStoreOut<bf16> eo{O, d, rows, row0, int64_t(D.Nq) * d, status};
  if (cfg.inner == TTT_INNER_LINEAR) {
    TcGeom g = geom(mt, 0, d / bnd, d / 64, Z, 1);
    g.a0.mn = row0;
    if (bnd == 256) TRY((gemm<256, 0, false, false, 2, 4, 8>(c.tQ, c.tFirst, c.tQ, c.tFirst, g, eo, status, c.st, true)));
    else if (bnd == 128) TRY((gemm<128, 0, false, false, 2, 4, 8>(c.tQ, c.tFirst, c.tQ, c.tFirst, g, eo, status, c.st, true)));
    else TRY((gemm<64, 0, false, false, 2, 4, 8>(c.tQ, c.tFirst, c.tQ, c.tFirst, g, eo, status, c.st, true)));
    return TTT_OK;
  }
  if (cfg.inner == TTT_INNER_GLU) {  // O = za * SiLU(zb) straight from the first-layer tiles
    EpiGluOut eo2{O, d, rows, row0, int64_t(D.Nq) * d, status};
    TcGeom g = geom(mt, 0, (2 * d) / 128, d / 64, Z, 1);
    g.a0.mn = row0;
    TRY((gemm<128, 0, false, false, 2, 4, 8>(c.tQ, c.tFirst, c.tQ, c.tFirst, g, eo2, status, c.st, true)));
    return TTT_OK;
  }
  if (d == 64 || d == 128 || d == 256) {
    // one kernel, hidden layer on chip (apply_mlp.cuh)
    const bool swiglu = cfg.inner == TTT_INNER_SWIGLU;
    TM tf, tw;
    TRY(tmap(&tf, c.v.at<bf16>(p, xFirst), 2, d, D.R1, Z, swiglu ? 256 : 128));
    TRY(tmap(&tw, c.v.at<bf16>(p, xW2), 2, h, d, Z, d));
    if (c.tQ.box != 128) return TTT_ERR_INVALID_ARG;
    ApplyGeom ag;
    ag.m_tiles = mt;
    ag.batches = Z;
    ag.hblocks = h / 128;
    ag.rows_valid = rows;
    ag.row0 = row0;
    ag.o_zs = int64_t(D.Nq) * d;
    StageScope sc(kStageApply, c.st);
    cudaError_t e = cudaErrorInvalidValue;
    if (swiglu) {
      e = d == 256 ? launch_apply_mlp<true, 256>(c.tQ.m, tf.m, tw.m, ag, O, status, c.st)
          : d == 128 ? launch_apply_mlp<true, 128>(c.tQ.m, tf.m, tw.m, ag, O, status, c.st)
                     : launch_apply_mlp<true, 64>(c.tQ.m, tf.m, tw.m, ag, O, status, c.st);
    } else {
      e = d == 256 ? launch_apply_mlp<false, 256>(c.tQ.m, tf.m, tw.m, ag, O, status, c.st)
          : d == 128 ? launch_apply_mlp<false, 128>(c.tQ.m, tf.m, tw.m, ag, O, status, c.st)
                     : launch_apply_mlp<false, 64>(c.tQ.m, tf.m, tw.m, ag, O, status, c.st);
    }
    return e == cudaSuccess ? TTT_OK : TTT_ERR_CUDA;
  }
  bf16* Hq = c.v.at<bf16>(p, xHq);
  if (cfg.inner == TTT_INNER_SWIGLU) {
    EpiApplyAct<true> e{Hq, h, rows, int64_t(D.Rq) * h};
    TcGeom g = geom(mt, 0, h / 128, d / 64, Z, 1);
    g.a0.mn = row0;
    TRY((gemm<256, 0, false, false, 2, 4, 8>(c.tQ, c.tFirst, c.tQ, c.tFirst, g, e, status, c.st, true)));
  } else {
    EpiApplyAct<false> e{Hq, h, rows, int64_t(D.Rq) * h};
    const int bnh = c.bn_first;
    TcGeom g = geom(mt, 0, h / bnh, d / 64, Z, 1);
    g.a0.mn = row0;
    if (bnh == 256) TRY((gemm<256, 0, false, false, 2, 4, 8>(c.tQ, c.tFirst, c.tQ, c.tFirst, g, e, status, c.st, true)));
    else TRY((gemm<128, 0, false, false, 2, 4, 8>(c.tQ, c.tFirst, c.tQ, c.tFirst, g, e, status, c.st, true)));
  }
  TM tHq;
  TRY(tmap(&tHq, Hq, 2, h, D.Rq, Z, 128));
  TcGeom g2 = geom(mt, 0, d / bnd, h / 64, Z, 1);
  if (bnd == 256) TRY((gemm<256, 0, false, false, 2, 4, 8>(tHq, c.tW2, tHq, c.tW2, g2, eo, status, c.st, true)));
  else if (bnd == 128) TRY((gemm<128, 0, false, false, 2, 4, 8>(tHq, c.tW2, tHq, c.tW2, g2, eo, status, c.st, true)));
  else TRY((gemm<64, 0, false, false, 2, 4, 8>(tHq, c.tW2, tHq, c.tW2, g2, eo, status, c.st, true)));
  return TTT_OK;
}

// Weight-gradient launch shape: split-K count and output tile height (256 rows
// = two accumulators sharing B, when the rows allow it and the tiles alone keep
// the SMs busy).
void choose_grad_shape(const Plan& p, int Cp, int* splits, int* tile_rows, int* grad_bn) {
  const ttt_config& c = p.cfg;
  const int d = c.d, h = c.h;
  const int bnd = bn_for(d);
  const int rows = c.inner == TTT_INNER_LINEAR ? d
                   : c.inner == TTT_INNER_GLU ? 2 * d
                   : c.inner == TTT_INNER_MLP2_GELU ? 2 * h
                                                    : 3 * h;
  const int r0 = c.inner == TTT_INNER_LINEAR ? d : c.inner == TTT_INNER_GLU ? 2 * d : h;
  const int kblocks = Cp / 64;
  if (fused_update_path(c)) {
    // the fused update kernels: one CTA per (head, token-tile range), one wave of them
    *splits = std::max(1, std::min(Cp / 128, kPlanSMs / std::max(1, p.BH)));
    *tile_rows = 128;
    *grad_bn = 64;
    return;
  }
  // each split reduces at least 1024 tokens: below that the fp32 partials it writes
  // and the reduction reads cost more than the parallelism gains; chunks of at most
  // 4096 tokens are not split at all (the gradient then goes straight to the optimizer)
  const int smax = kblocks <= 64 ? 1 : std::min(64, std::max(1, kblocks / 16));
  const int tiles256 = (r0 % 256 == 0 && rows % 256 == 0) ? rows / 256 * (d / bnd) * p.BH : 0;
  *tile_rows = (tiles256 > 0 && tiles256 * smax >= kPlanSMs) ? 256 : 128;
  // 512-row tiles on CTA pairs (74 pairs): each CTA brings in a third fewer bytes
  const bool pairs_ok = (c.flags & TTT_FLAG_SINGLE_CTA) == 0 && bnd >= 128;
  const int tiles512 = (pairs_ok && r0 % 512 == 0 && rows % 512 == 0) ? rows / 512 * (d / bnd) * p.BH : 0;
  if (tiles512 > 0 && tiles512 * smax >= kPlanSMs / 2) *tile_rows = 512;
  const int units = *tile_rows == 512 ? kPlanSMs / 2 : kPlanSMs;  // tiles that run at once
  const int tiles = rows / *tile_rows * (d / bnd) * p.BH;
  // single CTAs: about two waves of tiles (long K ranges per split, few partials to
  // reduce); CTA pairs: as many splits as fit one wave of the pairs (two waves measured
  // 1.2% slower on the million-token scene layer: twice the partials to write and reduce)
  int s = tiles <= 0 ? 1
          : *tile_rows == 512 ? std::max(1, units / tiles)
                              : std::max(1, (2 * units + tiles / 2) / tiles);
  s = std::min(s, smax);
  const int per = (kblocks + s - 1) / s;  // every split owns at least one k-block
  *splits = (kblocks + per - 1) / per;
  // an unsplit reduction that leaves SMs idle uses narrower tiles (twice the CTAs);
  // not with Muon, whose row norms must then sum over at most two parts of a row
  const bool muon = c.opt == TTT_OPT_MUON || c.opt == TTT_OPT_MOMENTUM_MUON;
  *grad_bn = bnd;
  if (*splits == 1 && !muon && *tile_rows == 128 && tiles < units && bnd >= 128) *grad_bn = bnd / 2;
}

}  // namespace

int plan_layout_bf16(Plan* p) {
  const ttt_config& c = p->cfg;
  const int d = c.d, h = c.h;
  // supported shapes of the tensor-core path
  if (d % 64 != 0) return TTT_ERR_UNSUPPORTED;
  const bool glu = c.inner == TTT_INNER_GLU;
  if (c.inner != TTT_INNER_LINEAR && !glu && h % 128 != 0) return TTT_ERR_UNSUPPORTED;
  // GLU: the plain and momentum steps with the dot or MSE loss (RMSE needs the chunk's whole
  // loss before any gradient; Muon is not built for it)
  if (glu && (c.loss == TTT_LOSS_RMSE || c.opt == TTT_OPT_MUON || c.opt == TTT_OPT_MOMENTUM_MUON))
    return TTT_ERR_UNSUPPORTED;
  // the weight-gradient GEMMs tile their output rows (h per matrix, d for the linear
  // model) by 128
  if (c.inner == TTT_INNER_LINEAR && d % 128 != 0) return TTT_ERR_UNSUPPORTED;
  if (c.inner == TTT_INNER_SWIGLU && c.loss != TTT_LOSS_NEG_DOT) return TTT_ERR_UNSUPPORTED;
  const bool muon = c.opt == TTT_OPT_MUON || c.opt == TTT_OPT_MOMENTUM_MUON;
  if (muon && (d % 128 != 0 || (c.inner != TTT_INNER_LINEAR && h % 128 != 0))) return TTT_ERR_UNSUPPORTED;
  const int Cp = (p->chunk + 127) / 128 * 128;
  int splits = 1, tile_rows = 128, grad_bn = 64;
  choose_grad_shape(*p, Cp, &splits, &tile_rows, &grad_bn);
  p->off[kNumBBuf] = size_t(splits);
  p->off[kNumBBuf + 1] = size_t(tile_rows);
  p->off[kNumBBuf + 2] = size_t(grad_bn);
  const Dims D = dims_of(*p);
  const int64_t Z = D.Z, P = p->P, GR = D.GR, nm = int64_t(D.m) * D.n, mm = int64_t(D.m) * D.m;
  const int64_t ZK = Z * D.nmat;
  const bool mlp_mse = c.inner == TTT_INNER_MLP2_GELU && c.loss != TTT_LOSS_NEG_DOT;  // MSE, RMSE
  const bool act = c.inner != TTT_INNER_LINEAR && !glu;  // a hidden layer and W2
  const bool spill = !mse_token_path(c);                   // activations go through HBM
  const int64_t bytes[kNumBBuf] = {
      Z * P * 4,
      Z * GR * d * 4,
      Z * GR * d * 4,
      Z * GR * 4,
      D.direct ? 0 : int64_t(D.splits) * Z * GR * d * 4,
      Z * D.R1 * d * 2,
      act ? Z * h * d * 2 : 0,
      act ? Z * d * h * 2 : 0,
      ((c.flags & TTT_FLAG_KEY_INSTNORM) && !mse_token_path(c)) ? Z * Cp * d * 2 : 0,
      (act && spill) ? Z * Cp * h * 2 : 0,
      ((act && spill) || (glu && !glu_update_path(c))) ? Z * Cp * 2 * h * 2 : 0,  // dZ13 / dZ (GLU: h = d)
      (mlp_mse && spill) ? Z * Cp * h * 2 : 0,
      ((mlp_mse && spill) || !act) ? Z * Cp * d * 2 : 0,
      (act && d != 64 && d != 128 && d != 256) ? Z * D.Rq * h * 2 : 0,  // two-GEMM apply only (d = 512)
      (c.flags & TTT_FLAG_KEY_INSTNORM) ? Z * (Cp / 128 + 1) * d * 2 * 4 + Z * 4 : 0,  // block sums, mean / rstd, counters
      muon ? ZK * nm * 4 : 0,
      muon ? ZK * nm * 4 : 0,
      muon ? ZK * nm * 4 : 0,
      muon ? ZK * nm * 4 : 0,
      muon ? ZK * mm * 4 : 0,
      muon ? ZK * mm * 4 : 0,
  };
  size_t o = 256;
  for (int i = 0; i < kNumBBuf; ++i) {
    p->off[i] = o;
    o += (size_t(bytes[i]) + 1023) / 1024 * 1024;
  }
  p->ws_bytes = o;
  // the momentum buffer, in its gradient layout, is the state a call hands on
  p->state_bytes = (c.opt == TTT_OPT_MOMENTUM || c.opt == TTT_OPT_MOMENTUM_MUON) ? size_t(bytes[xMom]) : 0;
  return TTT_OK;
}

int run_bf16(const Plan& p, const Io& io, void* ws, cudaStream_t st) {
  const ttt_config& cfg = p.cfg;
  Ctx c{p, dims_of(p), BView{static_cast<uint8_t*>(ws), static_cast<unsigned*>(ws)}, io, st,
        RowMap{cfg.inner, cfg.d, cfg.h, 0, p.P}};
  const Dims& D = c.D;
  c.rm.GR = D.GR;
  const int Z = D.Z, d = D.d, h = D.h;
  // tensor maps of the inputs and of the bf16 weight copies
  TRY(tmap(&c.tK, io.K, 2, d, D.N, Z, 128));
  TRY(tmap(&c.tV, io.V, 2, d, D.N, Z, 128));
  TRY(tmap(&c.tKmn, io.K, 2, d, D.N, Z, 64));
  TRY(tmap(&c.tVmn, io.V, 2, d, D.N, Z, 64));
  TRY(tmap(&c.tQ, io.Q, 2, d, D.Nq, Z, 128));
  bf16* First = c.v.at<bf16>(p, xFirst);
  const int bn_first = cfg.inner == TTT_INNER_SWIGLU ? 256
                       : cfg.inner == TTT_INNER_GLU  ? 128
                       : cfg.inner == TTT_INNER_MLP2_GELU
                           ? (cfg.loss == TTT_LOSS_NEG_DOT ? 128 : bn_for(h))
                           : bn_for(d);
  c.bn_first = bn_first;
  TRY(tmap(&c.tFirst, First, 2, d, D.R1, Z, bn_first));
  if (cfg.inner == TTT_INNER_MLP2_GELU || cfg.inner == TTT_INNER_SWIGLU) {
    TRY(tmap(&c.tW2T, c.v.at<bf16>(p, xW2T), 2, d, h, Z, cfg.loss == TTT_LOSS_NEG_DOT ? 128 : bn_for(h)));
    TRY(tmap(&c.tW2, c.v.at<bf16>(p, xW2), 2, h, d, Z, bn_for(d)));
  }
  // W = W0 per batch entry (W0 [H][P] shared by the batch entries, or [B*H][P] with one
  // state per entry) and its bf16 copies in one pass; zero momentum
  const int w0_rows = (cfg.flags & TTT_FLAG_W0_PER_BATCH) ? Z : cfg.H;
  if (io.M_in && p.state_bytes)
    TRY_CUDA(cudaMemcpyAsync(c.v.at<float>(p, xMom), io.M_in, p.state_bytes, cudaMemcpyDeviceToDevice, st));
  else
    TRY_CUDA(cudaMemsetAsync(c.v.at<float>(p, xMom), 0, size_t(Z) * D.GR * d * 4, st));
  if (cfg.flags & TTT_FLAG_KEY_INSTNORM) {  // the key-statistics counters start at zero
    float* kfin = c.v.at<float>(p, xKstat) + size_t(Z) * (D.Cp / 128) * d * 2;
    TRY_CUDA(cudaMemsetAsync(kfin + size_t(Z) * d * 2, 0, size_t(Z) * 4, st));
  }
  {
    dim3 g((c.rm.nrows() + 7) / 8, Z);
    {
      StageScope _sc(kStageFinish, st);
      finish_rows_kernel<<<g, 256, 0, st>>>(c.rm, 0, 0.f, false, false, c.v.at<float>(p, xWf), nullptr, nullptr,
                                            nullptr, 0, 0, false, First, c.v.at<bf16>(p, xW2T), c.v.at<bf16>(p, xW2),
                                            c.v.status, io.W0, w0_rows);
    }
    TRY_CUDA(cudaGetLastError());
    TRY(transpose_w2(c));
  }
  // causal with a side stream: chunk c's apply (reads W_c) runs beside chunk c's token
  // phase and gradient GEMMs (read W_c too); the optimizer step that replaces W_c waits for it
  const bool overlap = cfg.causal && io.aux && io.ev_fork && io.ev_join;
  for (int ci = 0; ci < p.nchunks; ++ci) {
    const int t0 = ci * p.chunk, n = std::min(p.chunk, cfg.N - t0);
    if (cfg.causal && overlap) {
      TRY_CUDA(cudaEventRecord(io.ev_fork, st));
      TRY_CUDA(cudaStreamWaitEvent(io.aux, io.ev_fork, 0));
      c.st = io.aux;
      const int r = apply_rows(c, t0, n);
      c.st = st;
      TRY(r);
      TRY_CUDA(cudaEventRecord(io.ev_join, io.aux));
      c.apply_pending = true;
    } else if (cfg.causal) {
      TRY(apply_rows(c, t0, n));
    }
    if (cfg.flags & TTT_FLAG_NO_UPDATE) continue;
    for (int ep = 0; ep < p.epochs; ++ep) TRY(update_chunk(c, t0, n));
  }
  if (overlap) TRY_CUDA(cudaStreamWaitEvent(st, io.ev_join, 0));  // join the side stream
  if (!cfg.causal) TRY(apply_rows(c, 0, cfg.Nq));
  if (io.W_out)
    TRY_CUDA(cudaMemcpyAsync(io.W_out, c.v.at<float>(p, xWf), size_t(Z) * p.P * 4, cudaMemcpyDeviceToDevice, st));
  if (io.M_out && p.state_bytes)
    TRY_CUDA(cudaMemcpyAsync(io.M_out, c.v.at<float>(p, xMom), p.state_bytes, cudaMemcpyDeviceToDevice, st));
  return TTT_OK;
}

}  // namespace ttt

extern "C" int ttt_token_pair_capacity(int swiglu) {
  return swiglu ? ttt::token_pair_capacity<true>() : ttt::token_pair_capacity<false>();
}

namespace {
template <bool RESB>
int64_t list_pair_tiles(const ttt::TokGeom& g, int pairs, int* counts, int* tiles, int64_t max_tiles) {
  int64_t listed = 0;
  for (int p = 0; p < pairs; ++p) {
    const ttt::PairTiles<RESB> t(g, p, pairs);
    counts[p] = t.count;
    for (int k = 0; k < t.count; ++k, ++listed) {
      if (listed >= max_tiles) return -1;
      t.at(g, pairs, k, tiles[3 * listed], tiles[3 * listed + 1], tiles[3 * listed + 2]);
    }
  }
  return listed;
}
}  // namespace

extern "C" int ttt_pair_schedule(int m_tiles, int n_tiles, int batches, int kblocks, int cap_resident,
                                 int cap_streaming, int* resident, int* pairs, int* counts, int* tiles,
                                 int64_t max_tiles) {
  if (m_tiles < 1 || n_tiles < 1 || batches < 1 || kblocks < 1 || cap_resident < 0 || cap_streaming < 0 ||
      !resident || !pairs || !counts || max_tiles < 0 || (!tiles && max_tiles > 0))
    return TTT_ERR_INVALID_ARG;
  if (static_cast<long long>(m_tiles) * n_tiles * batches > 0x7fffffffLL) return TTT_ERR_INVALID_ARG;
  ttt::TokGeom g{};
  g.m_tiles = m_tiles;
  g.n_tiles = n_tiles;
  g.batches = batches;
  g.kblocks = kblocks;
  bool resb = false;
  int np = 0;
  if (!ttt::pair_grid(g, cap_resident, cap_streaming, resb, np)) return TTT_ERR_UNSUPPORTED;
  *resident = resb ? 1 : 0;
  *pairs = np;
  const int64_t n = resb ? list_pair_tiles<true>(g, np, counts, tiles, max_tiles)
                         : list_pair_tiles<false>(g, np, counts, tiles, max_tiles);
  return n < 0 ? TTT_ERR_INVALID_ARG : static_cast<int>(n);
}

extern "C" int ttt_plan_info(const ttt_handle* h, int* info, int n) {
  if (!h || !info || n < 0) return TTT_ERR_INVALID_ARG;
  const ttt::Plan& p = h->plan;
  int v[7] = {static_cast<int>(p.path), static_cast<int>(p.chunk), static_cast<int>(p.nchunks), 0, 0, 0, 0};
  if (p.path == ttt::kPathBf16) {
    const ttt::Dims D = ttt::dims_of(p);
    v[3] = D.splits;
    v[4] = D.tile_rows;
    v[5] = D.grad_bn;
    v[6] = D.direct ? 1 : 0;
  }
  const int m = n < 7 ? n : 7;
  for (int i = 0; i < m; ++i) info[i] = v[i];
  return m;
}
