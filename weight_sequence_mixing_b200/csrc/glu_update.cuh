// Update of the simplified GLU inner model F(x) = (x Wa^T) * SiLU(x Wb^T) for d = 64 (ViT3's
// F1 heads; ViT3 digest section 03, inner-model table; the update of section 02) in one
// kernel: for every 128-token tile of a chunk
//   Z    = X [Wb; Wa]^T                 (TMEM, 128 columns: zb | za; two buffers)
//   dF   = -eta v (dot loss) or coef eta (F - v) (MSE), F = za SiLU(zb)
//   dZa  = dF SiLU(zb),  dZb = dF za SiLU'(zb)      (-> shared memory, [gate | linear])
//   G   += dZ^T X                       (TMEM, 128 rows [Wb; Wa] x 64 columns)
// with V staged by TMA beside the keys, so dZ never reaches HBM and no separate gradient
// GEMM runs.  A CTA owns one head and one contiguous range of its token tiles (as in
// mse_token.cuh) and writes its G once, as an fp32 split partial in the gradient layout
// [split][z][2d][d] (rows [0, 64) Wb, [64, 128) Wa), for the row finish to sum.
//
// Pipelining: Z of the next tile is issued before G of the current one, into the other Z
// buffer; dZ has two shared-memory buffers, so the gating of tile j + 1 overlaps G of tile j.
// A key/value slot stays busy until G of its tile has read the keys, so four slots keep the
// loads of the next tiles in flight across that chain.
//
// Warps: 0 TMA producer (keys and values of four tiles in flight, the head's weights once),
// 1 MMA issuer, 2..17 epilogue (four per TMEM lane quarter; warp part p owns channels
// [16 p, 16 p + 16)).  Every wait is bounded.
#pragma once
#include "epi_glu.cuh"
#include "mse_token.cuh"

namespace ttt {

struct GluGeom {
  int m_tiles;          // 128-token tiles of the chunk holding keys (ceil(n / 128))
  int batches, splits;  // heads (z), token-tile ranges per head: one CTA each
  int rows_valid;       // tokens in the chunk
  int x_off, v_off;     // token offsets of the key and value maps
  int t0;               // chunk's first token (eta index)
  const float* eta;
  int64_t eta_zs;
  float eta_scalar;
  int mse;              // 1: MSE loss, 0: dot loss
  float coef;           // 2 / (n d) (MSE)
  float* part;          // [splits][z][128][64] fp32 gradient partials
};

struct GluShape {
  static constexpr int TILE = 128 * 128;  // 128 rows x 64 bf16
  static constexpr int W_BYTES = TILE;    // [Wb 64 rows | Wa 64 rows] x 64
  static constexpr int DZ_BYTES = 2 * TILE;  // [128 tokens][gate 64 | linear 64] as two k-blocks
  static constexpr int NSLOT = 4;  // key/value slots
  static constexpr int EW = 16;
  static constexpr int CH = 64 / (EW / 4);  // channels per epilogue thread
  static constexpr int SMEM = 1024 + NSLOT * 2 * TILE + W_BYTES + 2 * DZ_BYTES + 256;
  static constexpr uint32_t GCOL = 256;  // TMEM columns of G
  static_assert(SMEM <= 227 * 1024, "shared memory");
};

__global__ void __launch_bounds__(64 + 32 * GluShape::EW, 1)
    glu_update_kernel(const __grid_constant__ CUtensorMap tX, const __grid_constant__ CUtensorMap tV,
                      const __grid_constant__ CUtensorMap tW, const GluGeom g, unsigned* status) {
  using S = GluShape;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* xv = smem;  // [slot][X tile | V tile]
  uint8_t* ws = xv + S::NSLOT * 2 * S::TILE;
  uint8_t* dzs = ws + S::W_BYTES;  // [buffer][2 k-blocks]
  uint64_t* xfull = reinterpret_cast<uint64_t*>(dzs + 2 * S::DZ_BYTES);  // [NSLOT]
  uint64_t* xempty = xfull + S::NSLOT;  // [NSLOT]: G (commit) and the epilogue's V reads are done with the slot
  uint64_t* zfull = xempty + S::NSLOT;  // [2] Z buffer written
  uint64_t* zempty = zfull + 2;   // [2] Z buffer read
  uint64_t* dzfull = zempty + 2;  // [2] dZ buffer written
  uint64_t* dzempty = dzfull + 2;  // [2] G done reading the dZ buffer
  uint64_t* wfull = dzempty + 2;
  uint64_t* gdone = wfull + 1;
  uint64_t* drain = gdone + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = static_cast<int>(lane_id());
  const int z = blockIdx.x / g.splits, sp = blockIdx.x % g.splits;
  const int mt0 = static_cast<int>(int64_t(sp) * g.m_tiles / g.splits);
  const int ntiles = static_cast<int>(int64_t(sp + 1) * g.m_tiles / g.splits) - mt0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S::NSLOT; ++s) {
      mbar_init(&xfull[s], 1);
      mbar_init(&xempty[s], 1 + S::EW);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&zfull[s], 1);
      mbar_init(&zempty[s], S::EW);
      mbar_init(&dzfull[s], S::EW);
      mbar_init(&dzempty[s], 1);
    }
    mbar_init(wfull, 1);
    mbar_init(gdone, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    if (elect_one() && ntiles > 0) {
      tma_prefetch_desc(&tX);
      tma_prefetch_desc(&tV);
      tma_prefetch_desc(&tW);
      mbar_arrive_expect_tx(wfull, S::W_BYTES);
      tma_load_3d(ws, &tW, wfull, 0, 0, z);
      for (int j = 0; j < ntiles; ++j) {
        const int s = j % S::NSLOT, mt = mt0 + j;
        if (j >= S::NSLOT && !mbar_wait(&xempty[s], ((j - S::NSLOT) / S::NSLOT) & 1, abort_flag)) break;
        uint8_t* slot = xv + s * 2 * S::TILE;
        mbar_arrive_expect_tx(&xfull[s], 2 * S::TILE);
        tma_load_3d(slot, &tX, &xfull[s], 0, g.x_off + mt * 128, z);
        tma_load_3d(slot + S::TILE, &tV, &xfull[s], 0, g.v_off + mt * 128, z);
      }
      if (*abort_flag) {
        const unsigned long long t0 = global_ns();
        while (global_ns() - t0 < 1000000ull) {
        }
      }
    }
  } else if (warp == 1) {
    if (elect_one() && ntiles > 0) {
      constexpr uint32_t idZ = make_idesc(128, 128, 1, false, false);  // Z = X [Wb; Wa]^T
      constexpr uint32_t idG = make_idesc(128, 64, 1, true, true);     // G = dZ^T X, both MN-major
      const uint32_t wa = smem_u32(ws);
      // G += dZ^T X of tile jj: A = dZ buffer jj & 1 read MN-major (64-column runs of the 128
      // rows 16 KB apart, 16-token steps of 2 KB), B = the keys of slot jj % NSLOT
      auto issue_g = [&](int jj) -> bool {
        const int b = jj & 1;
        if (!mbar_wait(&dzfull[b], (jj >> 1) & 1, abort_flag)) return false;
        tc_fence_after();
        const int xs = jj % S::NSLOT;
        const uint32_t da = smem_u32(dzs + b * S::DZ_BYTES), xa = smem_u32(xv + xs * 2 * S::TILE);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_f16(tmem_base + S::GCOL, make_sdesc_sw128(da + kk * 2048, S::TILE, 1024),
                  make_sdesc_sw128(xa + kk * 2048, S::TILE, 1024), idG, (jj > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&dzempty[b]);
        mma_commit(&xempty[xs]);
        return true;
      };
      bool ok = mbar_wait(wfull, 0, abort_flag);
      for (int j = 0; j < ntiles && ok; ++j) {
        const int b = j & 1, xs = j % S::NSLOT;
        if (!(ok = mbar_wait(&xfull[xs], (j / S::NSLOT) & 1, abort_flag))) break;
        // Z buffer b was last read by the epilogue of tile j - 2
        if (j >= 2 && !(ok = mbar_wait(&zempty[b], ((j - 2) >> 1) & 1, abort_flag))) break;
        tc_fence_after();
        const uint32_t xa = smem_u32(xv + xs * 2 * S::TILE);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_f16(tmem_base + b * 128, make_sdesc_sw128(xa + kk * 32, 16, 1024),
                  make_sdesc_sw128(wa + kk * 32, 16, 1024), idZ, kk > 0 ? 1u : 0u);
        mma_commit(&zfull[b]);
        if (j > 0 && !(ok = issue_g(j - 1))) break;
      }
      if (ok && issue_g(ntiles - 1)) mma_commit(gdone);
      if (*abort_flag) {
        volatile int never = 0;
        mma_commit(drain);
        mbar_wait(drain, 0, &never);
      }
    }
  } else {
    const int q = warp & 3;
    const int part = (warp - 2) >> 2;  // channels [CH part, CH part + CH)
    const int row = q * 32 + lane;
    const uint32_t tq = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
    bool ok = true;
    for (int j = 0; j < ntiles && ok; ++j) {
      const int b = j & 1, xs = j % S::NSLOT;
      const int m = (mt0 + j) * 128 + row;
      const bool valid = m < g.rows_valid;
      ok = __all_sync(0xffffffffu, mbar_wait(&zfull[b], (j >> 1) & 1, abort_flag));
      if (!ok) break;
      tc_fence_after();
      uint32_t rb[S::CH], ra[S::CH];
      tmem_ld16_async(tq + b * 128 + S::CH * part, rb);
      tmem_ld16_async(tq + b * 128 + 64 + S::CH * part, ra);
      tmem_wait_regs(rb);
      tmem_wait_regs(ra);
      float zb[S::CH], za[S::CH];
#pragma unroll
      for (int i = 0; i < S::CH; ++i) {
        zb[i] = __uint_as_float(rb[i]);
        za[i] = __uint_as_float(ra[i]);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&zempty[b]);
      // this row's 32 values of V from the slot's V tile (128-byte swizzled rows)
      const uint8_t* vt = xv + xs * 2 * S::TILE + S::TILE;
      float v[S::CH];
#pragma unroll
      for (int k = 0; k < S::CH / 8; ++k) {
        const uint4 u = *sw128_chunk(const_cast<uint8_t*>(vt), row, (S::CH / 8) * part + k);
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[i]));
          v[8 * k + 2 * i] = f.x;
          v[8 * k + 2 * i + 1] = f.y;
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&xempty[xs]);
      const float e = valid ? (g.eta ? g.eta[z * g.eta_zs + g.t0 + m] : g.eta_scalar) : 0.0f;
#pragma unroll
      for (int i = 0; i < S::CH; ++i) {
        const float s = sigmoid_dev(zb[i]);
        const float silu = zb[i] * s;
        const float df = g.mse ? g.coef * e * (za[i] * silu - v[i]) : -e * v[i];
        const float ga = df * silu;                                     // dZa
        const float gb = df * za[i] * s * fmaf(zb[i], 1.0f - s, 1.0f);  // dZb
        zb[i] = valid ? gb : 0.0f;
        za[i] = valid ? ga : 0.0f;
      }
      // the dZ buffer was last read by G of tile j - 2
      if (j >= 2) {
        ok = __all_sync(0xffffffffu, mbar_wait(&dzempty[b], ((j - 2) >> 1) & 1, abort_flag));
        if (!ok) break;
      }
      uint8_t* dz = dzs + b * S::DZ_BYTES;
#pragma unroll
      for (int k = 0; k < S::CH / 8; ++k) {
        *sw128_chunk(dz, row, (S::CH / 8) * part + k) =
            make_uint4(pack_bf16x2(zb[8 * k], zb[8 * k + 1]), pack_bf16x2(zb[8 * k + 2], zb[8 * k + 3]),
                       pack_bf16x2(zb[8 * k + 4], zb[8 * k + 5]), pack_bf16x2(zb[8 * k + 6], zb[8 * k + 7]));
        *sw128_chunk(dz + S::TILE, row, (S::CH / 8) * part + k) =
            make_uint4(pack_bf16x2(za[8 * k], za[8 * k + 1]), pack_bf16x2(za[8 * k + 2], za[8 * k + 3]),
                       pack_bf16x2(za[8 * k + 4], za[8 * k + 5]), pack_bf16x2(za[8 * k + 6], za[8 * k + 7]));
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&dzfull[b]);
    }
    // the CTA's partial of G: this warp's CH columns of rows 32 q .. 32 q + 31
    if (ok && ntiles > 0) ok = __all_sync(0xffffffffu, mbar_wait(gdone, 0, abort_flag));
    if (ok) {
      tc_fence_after();
      uint32_t gr[S::CH];
      if (ntiles > 0) {
        tmem_ld16_async(tq + S::GCOL + S::CH * part, gr);
        tmem_wait_regs(gr);
      } else {
#pragma unroll
        for (int i = 0; i < S::CH; ++i) gr[i] = 0u;
      }
      float* dst = g.part + ((int64_t(sp) * g.batches + z) * 128 + row) * 64 + S::CH * part;
#pragma unroll
      for (int i = 0; i < S::CH; i += 4)
        *reinterpret_cast<float4*>(dst + i) = make_float4(__uint_as_float(gr[i]), __uint_as_float(gr[i + 1]),
                                                          __uint_as_float(gr[i + 2]), __uint_as_float(gr[i + 3]));
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (threadIdx.x == 0 && *abort_flag) set_status(status, kStatusTimeout);
  if (warp == 1) tmem_dealloc(tmem_base, 512);
}

inline cudaError_t launch_glu_update(const CUtensorMap& tX, const CUtensorMap& tV, const CUtensorMap& tW,
                                     const GluGeom& g, unsigned* status, cudaStream_t st) {
  using S = GluShape;
  static OncePerDevice configured;
  const int set = configured.run(current_device(), [&] {
    return cudaFuncSetAttribute(glu_update_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, S::SMEM);
  });
  if (set != 0) return static_cast<cudaError_t>(set);
  if (g.splits < 1 || g.batches < 1 || g.m_tiles < 1) return cudaErrorInvalidValue;
  const long long grid = static_cast<long long>(g.batches) * g.splits;
  if (grid > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  glu_update_kernel<<<static_cast<int>(grid), 64 + 32 * S::EW, S::SMEM, st>>>(tX, tV, tW, g, status);
  return cudaGetLastError();
}

}  // namespace ttt
