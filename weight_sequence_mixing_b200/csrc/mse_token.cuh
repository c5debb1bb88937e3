// Token phase of the GELU-MLP update with the MSE loss in one kernel (d = 64; h = 128 or
// 256: the ViT3-like heads).  For every 128-token tile of a chunk (ViT3 digest section 02:
// forward on the keys, loss backward):
//   Z    = X W1^T                      (TMEM columns [0, h))
//   H    = GELU(Z), G' = GELU'(Z)      (H -> shared memory as the next MMA's operand and
//                                       to HBM for the weight gradients; G' stays in the
//                                       epilogue threads' registers)
//   V^   = H W2^T                      (TMEM columns [256, 320))
//   dY   = 2 eta_t (V^ - V) / (n d)    (-> shared memory and HBM)
//   dH   = dY W2                       (TMEM columns [256, 256 + h): W2 [d][h] read as an
//                                       MN-major operand from the same tile as for V^)
//   dZ   = dH * G'                     (-> HBM)
// H, dY and dZ are what the weight-gradient reductions read (G2^T = H^T dY, G1 = dZ^T X);
// rows past the chunk are written as zeros.  The three GEMMs of a tile are chained
// through TMEM and shared memory: neither Z nor G' nor V^ reaches HBM, and the next
// tile's Z overlaps this tile's later phases (Z and V^ / dH use separate TMEM columns).
//
// Warps: 0 TMA producer (keys and values of two tiles in flight; W1, W2 of the current
// head resident), 1 MMA issuer, 2..17 epilogue (four per TMEM lane quarter; warp slot s
// owns hidden columns [s h/4, (s+1) h/4) and 16 of the 64 output channels).  Every wait
// is bounded.
#pragma once
#include "epilogues.cuh"

namespace ttt {

struct MseGeom {
  int m_tiles, batches;  // 128-token tiles per head, heads (z)
  int rows_valid;        // tokens in the chunk
  int x_off, v_off;      // token offsets of the key and value maps
  int t0;                // chunk's first token (eta index)
  const float* eta;
  int64_t eta_zs;
  float eta_scalar, coef;  // coef = 2 / (n d)
  bf16* H;                 // [z][Cp][h]
  bf16* dY;                // [z][Cp][d]
  bf16* dZ;                // [z][Cp][h]
  int64_t h_zs, y_zs;      // elements per head of H (and dZ) and of dY
};

template <int HID>
struct MseShape {
  static constexpr int D = 64;
  static constexpr int TILE = 128 * 128;              // 128 rows x 64 bf16
  static constexpr int W1_BYTES = HID * 128;          // [HID][64]
  static constexpr int W2_BYTES = (HID / 64) * 64 * 128;  // [64][HID] as HID/64 blocks of 64 columns
  static constexpr int H_BYTES = (HID / 64) * TILE;   // [128][HID] as HID/64 k-blocks
  static constexpr int EW = 16;
  static constexpr int SMEM = 1024 + 2 * 2 * TILE + W1_BYTES + W2_BYTES + H_BYTES + TILE + 256;
  static constexpr int COLS = HID / 4;                // hidden columns per epilogue thread
  static_assert(HID == 128 || HID == 256, "h");
  static_assert(SMEM <= 227 * 1024, "shared memory");
};

// 16-byte chunk k of row r of a 128-byte-row, 128-byte-swizzled tile sits at k ^ (r & 7)
__device__ __forceinline__ uint4* sw128_chunk(uint8_t* tile, int r, int k) {
  return reinterpret_cast<uint4*>(tile + r * 128 + 16 * (k ^ (r & 7)));
}

template <int HID>
__global__ void __launch_bounds__(64 + 32 * MseShape<HID>::EW, 1)
    mse_token_kernel(const __grid_constant__ CUtensorMap tX, const __grid_constant__ CUtensorMap tV,
                     const __grid_constant__ CUtensorMap tW1, const __grid_constant__ CUtensorMap tW2,
                     const MseGeom g, unsigned* status) {
  using S = MseShape<HID>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* xv = smem;                       // [slot][X tile | V tile]
  uint8_t* w1s = xv + 2 * 2 * S::TILE;
  uint8_t* w2s = w1s + S::W1_BYTES;
  uint8_t* hs = w2s + S::W2_BYTES;
  uint8_t* dys = hs + S::H_BYTES;
  uint64_t* xfull = reinterpret_cast<uint64_t*>(dys + S::TILE);  // [2]
  uint64_t* xempty = xfull + 2;   // [2]: the Z MMAs (commit) and the dY epilogue are done with the slot
  uint64_t* wfull = xempty + 2;   // the head's weights landed
  uint64_t* wrelease = wfull + 1;  // the last MMA reading a head's weights completed
  uint64_t* zfull = wrelease + 1;
  uint64_t* zempty = zfull + 1;
  uint64_t* hfull = zempty + 1;
  uint64_t* vfull = hfull + 1;
  uint64_t* dyfull = vfull + 1;
  uint64_t* dhfull = dyfull + 1;
  uint64_t* dhempty = dhfull + 1;
  uint64_t* drain = dhempty + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = static_cast<int>(lane_id());
  const int total = g.m_tiles * g.batches;

  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(&xfull[s], 1);
      mbar_init(&xempty[s], 1 + S::EW);
    }
    mbar_init(wfull, 1);
    mbar_init(wrelease, 1);
    mbar_init(zfull, 1);
    mbar_init(zempty, S::EW);
    mbar_init(hfull, S::EW);
    mbar_init(vfull, 1);
    mbar_init(dyfull, S::EW);
    mbar_init(dhfull, 1);
    mbar_init(dhempty, S::EW);
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
    if (elect_one()) {
      tma_prefetch_desc(&tX);
      tma_prefetch_desc(&tV);
      tma_prefetch_desc(&tW1);
      tma_prefetch_desc(&tW2);
      int j = 0, zw = -1, nw = 0;  // tiles, head of the resident weights, weight loads
      for (int t = blockIdx.x; t < total; t += gridDim.x, ++j) {
        const int mt = t % g.m_tiles, z = t / g.m_tiles;
        if (z != zw) {
          // the MMAs of the previous head must be done reading its weights (one release per
          // head change, in order: the phases alternate)
          if (nw > 0 && !mbar_wait(wrelease, (nw - 1) & 1, abort_flag)) break;
          mbar_arrive_expect_tx(wfull, S::W1_BYTES + S::W2_BYTES);
          tma_load_3d(w1s, &tW1, wfull, 0, 0, z);
          for (int b = 0; b < HID / 64; ++b) tma_load_3d(w2s + b * 64 * 128, &tW2, wfull, 64 * b, 0, z);
          zw = z;
          ++nw;
        }
        const int s = j & 1;
        if (j >= 2 && !mbar_wait(&xempty[s], ((j - 2) >> 1) & 1, abort_flag)) break;
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
    if (elect_one()) {
      constexpr uint32_t idZ = make_idesc(128, HID, 1, false, false);
      constexpr uint32_t idV = make_idesc(128, 64, 1, false, false);
      constexpr uint32_t idH = make_idesc(128, HID, 1, false, true);  // B = W2 [d][h], MN-major
      const uint32_t w1a = smem_u32(w1s), w2a = smem_u32(w2s), ha = smem_u32(hs), dya = smem_u32(dys);
      int j = 0, zw = -1, nw = 0;
      for (int t = blockIdx.x; t < total; t += gridDim.x, ++j) {
        const int z = t / g.m_tiles;
        const int s = j & 1;
        if (z != zw) {
          if (!mbar_wait(wfull, nw & 1, abort_flag)) break;
          zw = z;
          ++nw;
        }
        // Z of the previous tile read out of TMEM; this tile's keys landed
        if (j > 0 && !mbar_wait(zempty, (j - 1) & 1, abort_flag)) break;
        if (!mbar_wait(&xfull[s], (j >> 1) & 1, abort_flag)) break;
        tc_fence_after();
        const uint32_t xa = smem_u32(xv + s * 2 * S::TILE);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_f16(tmem_base, make_sdesc_sw128(xa + kk * 32, 16, 1024), make_sdesc_sw128(w1a + kk * 32, 16, 1024), idZ,
                  kk > 0 ? 1u : 0u);
        mma_commit(zfull);
        mma_commit(&xempty[s]);
        // V^ = H W2^T once H is in shared memory and the previous tile's dH has been read
        if (!mbar_wait(hfull, j & 1, abort_flag)) break;
        if (j > 0 && !mbar_wait(dhempty, (j - 1) & 1, abort_flag)) break;
        tc_fence_after();
        for (int kb = 0; kb < HID / 64; ++kb)
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_f16(tmem_base + 256, make_sdesc_sw128(ha + kb * S::TILE + kk * 32, 16, 1024),
                    make_sdesc_sw128(w2a + kb * 64 * 128 + kk * 32, 16, 1024), idV, (kb > 0 || kk > 0) ? 1u : 0u);
        mma_commit(vfull);
        // dH = dY W2 once dY is in shared memory (V^ has been read by then)
        if (!mbar_wait(dyfull, j & 1, abort_flag)) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_f16(tmem_base + 256, make_sdesc_sw128(dya + kk * 32, 16, 1024),
                  make_sdesc_sw128(w2a + kk * 16 * 128, 64 * 128, 1024), idH, kk > 0 ? 1u : 0u);
        mma_commit(dhfull);
        // the next tile of this CTA reads another head's weights: release these
        const int tn = t + static_cast<int>(gridDim.x);
        if (tn < total && tn / g.m_tiles != z) mma_commit(wrelease);
      }
      if (*abort_flag) {
        volatile int never = 0;
        mma_commit(drain);
        mbar_wait(drain, 0, &never);
      }
    }
  } else {
    const int q = warp & 3;
    const int slot = (warp - 2) >> 2;
    const int row = q * 32 + lane;
    const uint32_t tq = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
    const int c0 = slot * S::COLS;  // hidden columns [c0, c0 + COLS)
    int j = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < total && ok; t += gridDim.x, ++j) {
      const int mt = t % g.m_tiles, z = t / g.m_tiles;
      const int s = j & 1;
      const int m = mt * 128 + row;
      const bool valid = m < g.rows_valid;
      bf16* hrow = g.H + z * g.h_zs + int64_t(m) * HID + c0;
      bf16* zrow = g.dZ + z * g.h_zs + int64_t(m) * HID + c0;
      bf16* yrow = g.dY + z * g.y_zs + int64_t(m) * S::D + slot * 16;
      // ---- E1: H = GELU(Z), G' kept packed in registers
      ok = __all_sync(0xffffffffu, mbar_wait(zfull, j & 1, abort_flag));
      if (!ok) break;
      tc_fence_after();
      uint32_t gp[S::COLS / 2];
#pragma unroll
      for (int cc = 0; cc < S::COLS; cc += 32) {
        float zv[32], hv[32];
        tmem_ld32(tq + c0 + cc, zv);
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          float g0, g1, p0, p1;
          gelu_and_grad(zv[i], g0, p0);
          gelu_and_grad(zv[i + 1], g1, p1);
          hv[i] = valid ? g0 : 0.f;
          hv[i + 1] = valid ? g1 : 0.f;
          gp[(cc + i) / 2] = pack_bf16x2(p0, p1);
        }
        // H: the k-block of column c0 + cc in shared memory (next MMA's operand) and HBM
        uint8_t* kb = hs + ((c0 + cc) / 64) * S::TILE;
        const int k0 = ((c0 + cc) % 64) / 8;
#pragma unroll
        for (int k = 0; k < 4; ++k)
          *sw128_chunk(kb, row, k0 + k) =
              make_uint4(pack_bf16x2(hv[8 * k], hv[8 * k + 1]), pack_bf16x2(hv[8 * k + 2], hv[8 * k + 3]),
                         pack_bf16x2(hv[8 * k + 4], hv[8 * k + 5]), pack_bf16x2(hv[8 * k + 6], hv[8 * k + 7]));
        if (m < g.m_tiles * 128) store_bf16x32(hrow + cc, hv);
      }
      tc_fence_before();
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(zempty);
        mbar_arrive(hfull);
      }
      // ---- E2: dY = coef eta (V^ - V) on this warp's 16 output channels
      ok = __all_sync(0xffffffffu, mbar_wait(vfull, j & 1, abort_flag));
      if (!ok) break;
      tc_fence_after();
      {
        uint32_t vr[16];
        tmem_ld16_async(tq + 256 + slot * 16, vr);
        tmem_wait_regs(vr);
        const float e = valid ? (g.eta ? g.eta[z * g.eta_zs + g.t0 + m] : g.eta_scalar) * g.coef : 0.f;
        const uint8_t* vt = xv + s * 2 * S::TILE + S::TILE;  // the V tile (128-byte swizzled rows)
        float y[16];
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          const uint4 u = *sw128_chunk(const_cast<uint8_t*>(vt), row, slot * 2 + k);
          const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[i]));
            y[8 * k + 2 * i] = valid ? e * (__uint_as_float(vr[8 * k + 2 * i]) - f.x) : 0.f;
            y[8 * k + 2 * i + 1] = valid ? e * (__uint_as_float(vr[8 * k + 2 * i + 1]) - f.y) : 0.f;
          }
        }
        uint32_t yp[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) yp[i] = pack_bf16x2(y[2 * i], y[2 * i + 1]);
        *sw128_chunk(dys, row, slot * 2) = make_uint4(yp[0], yp[1], yp[2], yp[3]);
        *sw128_chunk(dys, row, slot * 2 + 1) = make_uint4(yp[4], yp[5], yp[6], yp[7]);
        if (m < g.m_tiles * 128) {
          uint4* yd = reinterpret_cast<uint4*>(yrow);
          yd[0] = make_uint4(yp[0], yp[1], yp[2], yp[3]);
          yd[1] = make_uint4(yp[4], yp[5], yp[6], yp[7]);
        }
      }
      tc_fence_before();
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(dyfull);
        mbar_arrive(&xempty[s]);
      }
      // ---- E3: dZ = dH * G'
      ok = __all_sync(0xffffffffu, mbar_wait(dhfull, j & 1, abort_flag));
      if (!ok) break;
      tc_fence_after();
#pragma unroll
      for (int cc = 0; cc < S::COLS; cc += 32) {
        float dh[32];
        tmem_ld32(tq + 256 + c0 + cc, dh);
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          const float2 gpf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&gp[(cc + i) / 2]));
          dh[i] = valid ? dh[i] * gpf.x : 0.f;
          dh[i + 1] = valid ? dh[i + 1] * gpf.y : 0.f;
        }
        if (m < g.m_tiles * 128) store_bf16x32(zrow + cc, dh);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(dhempty);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (threadIdx.x == 0 && *abort_flag) set_status(status, kStatusTimeout);
  if (warp == 1) tmem_dealloc(tmem_base, 512);
}

template <int HID>
cudaError_t launch_mse_token(const CUtensorMap& tX, const CUtensorMap& tV, const CUtensorMap& tW1,
                             const CUtensorMap& tW2, const MseGeom& g, unsigned* status, cudaStream_t st) {
  using S = MseShape<HID>;
  auto kern = mse_token_kernel<HID>;
  static OncePerDevice configured;
  const int set = configured.run(current_device(), [&] {
    return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, S::SMEM);
  });
  if (set != 0) return static_cast<cudaError_t>(set);
  const long long total = static_cast<long long>(g.m_tiles) * g.batches;
  if (total <= 0) return cudaSuccess;
  if (total > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  const int grid = static_cast<int>(std::min<long long>(total, sm_count()));
  kern<<<grid, 64 + 32 * S::EW, S::SMEM, st>>>(tX, tV, tW1, tW2, g, status);
  return cudaGetLastError();
}

}  // namespace ttt
