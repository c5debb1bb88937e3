// Token phase and weight gradients of the GELU-MLP update with the MSE loss in one kernel
// (d = 64; h = 128 or 256: the ViT3-like heads).  For every 128-token tile of a chunk
// (ViT3 digest section 02: forward on the keys, loss backward, gradients of W1 and W2):
//   Z    = X W1^T                      (TMEM columns [0, h))
//   H    = GELU(Z), G' = GELU'(Z)      (H -> shared memory; G' stays in the epilogue
//                                       threads' registers)
//   V^   = H W2^T                      (TMEM columns [0, 64): Z has been read by then)
//   dY   = 2 eta_t (V^ - V) / (n d)    (-> shared memory)
//   G2^T += H^T dY                     (TMEM accumulators, see below)
//   dH   = dY W2                       (TMEM columns [0, h): W2 [d][h] read as an MN-major
//                                       operand from the same tile as for V^)
//   dZ   = dH * G'                     (-> shared memory, over H)
//   G1   += dZ^T X                     (TMEM accumulators)
// Nothing of a tile reaches HBM: the gradients of W2 (as G2^T [h][d]) and W1 [h][d] stay
// in TMEM columns [256, 256 + 128 h / 64) as 128-row x 64-column accumulators, summed
// over the CTA's tiles, and are written once, as fp32 split partials in the gradient
// layout [split][z][2h][d] (rows [0, h) G2^T, rows [h, 2h) G1), for the split reduction.
//
// A CTA owns one head z and one contiguous range of its token tiles (split sp of the
// chunk's tiles), so the head's weights are loaded once.  Tiles run one after another
// (a tile's TMEM-chained steps leave no room in TMEM for a second tile), but each step is
// staggered by 64-column k-blocks of the hidden layer: Z is issued as h/64 MMAs of 64
// columns, the gating starts on the first while the others run, V^ accumulates k-block by
// k-block as the gating finishes them; dH likewise feeds dZ, and G1 of a 128-row block of h
// and the next tile's Z k-blocks go as soon as their dZ k-blocks are written.  Rows past
// the chunk are zero in H, dY and dZ, so they add nothing.
//
// Key instance-norm (kstats given): the keys arrive raw and warp 0 normalises each tile in
// shared memory, x_hat = (x - mean) rstd per channel, before the Z MMAs read it (and G1
// then reduces against the normalised keys), so no normalised copy of K goes through HBM.
//
// Warps: 0 TMA producer (keys and values of two tiles in flight; all its lanes normalise
// the keys), 1 MMA issuer, 2..17 epilogue (four per TMEM lane quarter; warp slot s owns
// hidden columns [64 k + 16 s, 64 k + 16 s + 16) of every k-block k and 16 of the 64 output
// channels).  Every wait is bounded.
#pragma once
#include "epilogues.cuh"

namespace ttt {

struct MseGeom {
  int m_tiles;          // 128-token tiles of the chunk holding keys (ceil(n / 128))
  int batches, splits;  // heads (z), token-tile ranges per head: one CTA each
  int rows_valid;       // tokens in the chunk
  int x_off, v_off;     // token offsets of the key and value maps
  int t0;               // chunk's first token (eta index)
  const float* eta;
  int64_t eta_zs;
  float eta_scalar, coef;  // coef = 2 / (n d)
  float* part;             // [splits][z][2h][64] fp32 gradient partials
  const float* kstats;     // [z][64][2] mean, 1/std of the chunk's keys per channel, or null
};

template <int HID>
struct MseShape {
  static constexpr int D = 64;
  static constexpr int TILE = 128 * 128;                  // 128 rows x 64 bf16
  static constexpr int W1_BYTES = HID * 128;              // [HID][64]
  static constexpr int W2_BYTES = (HID / 64) * 64 * 128;  // [64][HID] as HID/64 blocks of 64 columns
  static constexpr int H_BYTES = (HID / 64) * TILE;       // [128][HID] as HID/64 k-blocks (H, then dZ)
  static constexpr int EW = 16;
  static constexpr int SMEM = 1024 + 2 * 2 * TILE + W1_BYTES + W2_BYTES + H_BYTES + TILE + 2 * 64 * 4 + 256;
  static constexpr int COLS = HID / 4;          // hidden columns per epilogue thread
  static constexpr int KB = HID / 64;           // 64-column k-blocks of the hidden layer
  static constexpr int NACC = 2 * (HID / 128);  // 128 x 64 gradient accumulators
  static constexpr uint32_t GCOL = 256;         // first TMEM column of the accumulators
  static_assert(HID == 128 || HID == 256, "h");
  static_assert(SMEM <= 227 * 1024, "shared memory");
};

// 16-byte chunk k of row r of a 128-byte-row, 128-byte-swizzled tile sits at k ^ (r & 7)
__device__ __forceinline__ uint4* sw128_chunk(uint8_t* tile, int r, int k) {
  return reinterpret_cast<uint4*>(tile + r * 128 + 16 * (k ^ (r & 7)));
}

// 16 values of this thread's row as bf16 into columns [k0 8, k0 8 + 16) of a swizzled k-block
__device__ __forceinline__ void put_row16(uint8_t* kb, int row, int k0, const float (&v)[16]) {
#pragma unroll
  for (int k = 0; k < 2; ++k)
    *sw128_chunk(kb, row, k0 + k) =
        make_uint4(pack_bf16x2(v[8 * k], v[8 * k + 1]), pack_bf16x2(v[8 * k + 2], v[8 * k + 3]),
                   pack_bf16x2(v[8 * k + 4], v[8 * k + 5]), pack_bf16x2(v[8 * k + 6], v[8 * k + 7]));
}

template <int HID>
__global__ void __launch_bounds__(64 + 32 * MseShape<HID>::EW, 1)
    mse_token_kernel(const __grid_constant__ CUtensorMap tX, const __grid_constant__ CUtensorMap tV,
                     const __grid_constant__ CUtensorMap tW1, const __grid_constant__ CUtensorMap tW2,
                     const MseGeom g, unsigned* status) {
  using S = MseShape<HID>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* xv = smem;  // [slot][X tile | V tile]
  uint8_t* w1s = xv + 2 * 2 * S::TILE;
  uint8_t* w2s = w1s + S::W1_BYTES;
  uint8_t* hs = w2s + S::W2_BYTES;
  uint8_t* dys = hs + S::H_BYTES;
  float* nsc = reinterpret_cast<float*>(dys + S::TILE);  // [64] rstd, [64] -mean rstd
  uint64_t* xfull = reinterpret_cast<uint64_t*>(nsc + 2 * 64);  // [2]
  uint64_t* xempty = xfull + 2;  // [2]: G1 (commit) and the dY epilogue are done with the slot
  uint64_t* wfull = xempty + 2;  // the head's weights landed
  uint64_t* zk = wfull + 1;      // [KB] Z k-block in TMEM (the previous tile's G1 of its rows done)
  uint64_t* hk = zk + S::KB;     // [KB] H k-block in shared memory, its Z read
  uint64_t* vfull = hk + S::KB;  // V^ in TMEM
  uint64_t* dyfull = vfull + 1;  // dY in shared memory, V^ read
  uint64_t* dhk = dyfull + 1;    // [KB] dH k-block in TMEM, the tile's G2^T done (H no longer read)
  uint64_t* dzk = dhk + S::KB;   // [KB] dZ k-block in shared memory, its dH read
  uint64_t* gdone = dzk + S::KB;  // the last tile's G1 done: the accumulators are final
  uint64_t* xnorm = gdone + 1;    // [2]: the slot's keys normalised (key instance-norm only)
  uint64_t* drain = xnorm + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = static_cast<int>(lane_id());
  const int z = blockIdx.x / g.splits, sp = blockIdx.x % g.splits;
  const int mt0 = static_cast<int>(int64_t(sp) * g.m_tiles / g.splits);
  const int ntiles = static_cast<int>(int64_t(sp + 1) * g.m_tiles / g.splits) - mt0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(&xfull[s], 1);
      mbar_init(&xempty[s], 1 + S::EW);
      mbar_init(&xnorm[s], 1);
    }
    mbar_init(wfull, 1);
    for (int k = 0; k < S::KB; ++k) {
      mbar_init(&zk[k], 1);
      mbar_init(&hk[k], S::EW);
      mbar_init(&dhk[k], 1);
      mbar_init(&dzk[k], S::EW);
    }
    mbar_init(vfull, 1);
    mbar_init(dyfull, S::EW);
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
    const bool norm = g.kstats != nullptr;
    if (norm) {
      for (int c = lane; c < 64; c += 32) {
        const float mean = g.kstats[(int64_t(z) * 64 + c) * 2], rstd = g.kstats[(int64_t(z) * 64 + c) * 2 + 1];
        nsc[c] = rstd;
        nsc[64 + c] = -mean * rstd;
      }
      __syncwarp();
    }
    if (ntiles > 0) {
      if (lane == 0) {
        tma_prefetch_desc(&tX);
        tma_prefetch_desc(&tV);
        tma_prefetch_desc(&tW1);
        tma_prefetch_desc(&tW2);
        mbar_arrive_expect_tx(wfull, S::W1_BYTES + S::W2_BYTES);
        tma_load_3d(w1s, &tW1, wfull, 0, 0, z);
        for (int b = 0; b < HID / 64; ++b) tma_load_3d(w2s + b * 64 * 128, &tW2, wfull, 64 * b, 0, z);
      }
      for (int j = 0; j < ntiles; ++j) {
        const int s = j & 1, mt = mt0 + j;
        if (j >= 2 && !__all_sync(0xffffffffu, mbar_wait(&xempty[s], ((j - 2) >> 1) & 1, abort_flag))) break;
        uint8_t* slot = xv + s * 2 * S::TILE;
        if (lane == 0) {
          mbar_arrive_expect_tx(&xfull[s], 2 * S::TILE);
          tma_load_3d(slot, &tX, &xfull[s], 0, g.x_off + mt * 128, z);
          tma_load_3d(slot + S::TILE, &tV, &xfull[s], 0, g.v_off + mt * 128, z);
        }
        if (!norm) continue;
        // normalise the 128 x 64 key tile in place: 16-byte chunk p of row r holds channels
        // 8 (p ^ (r & 7)) .. + 7 (128-byte swizzle); lane l takes chunk l % 8 of rows l / 8 + 4 i
        if (!__all_sync(0xffffffffu, mbar_wait(&xfull[s], (j >> 1) & 1, abort_flag))) break;
#pragma unroll 4
        for (int i = 0; i < 32; ++i) {
          const int r = lane / 8 + 4 * i, p = lane % 8, c0 = 8 * (p ^ (r & 7));
          uint4* ch = reinterpret_cast<uint4*>(slot + r * 128 + 16 * p);
          const uint4 u = *ch;
          const uint32_t w[4] = {u.x, u.y, u.z, u.w};
          uint32_t o[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[e]));
            const int c = c0 + 2 * e;
            o[e] = pack_bf16x2(fmaf(f.x, nsc[c], nsc[64 + c]), fmaf(f.y, nsc[c + 1], nsc[64 + c + 1]));
          }
          *ch = make_uint4(o[0], o[1], o[2], o[3]);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&xnorm[s]);
      }
      if (*abort_flag) {
        const unsigned long long t0 = global_ns();
        while (global_ns() - t0 < 1000000ull) {
        }
      }
    }
  } else if (warp == 1) {
    if (elect_one() && ntiles > 0) {
      constexpr uint32_t idZ = make_idesc(128, 64, 1, false, false);  // one 64-column k-block of Z
      constexpr uint32_t idV = make_idesc(128, 64, 1, false, false);
      constexpr uint32_t idH = make_idesc(128, 64, 1, false, true);   // B = a W2 [d][h] block, MN-major
      constexpr uint32_t idG = make_idesc(128, 64, 1, true, true);    // A = H^T / dZ^T, B = dY / X
      const uint32_t w1a = smem_u32(w1s), w2a = smem_u32(w2s), ha = smem_u32(hs), dya = smem_u32(dys);
      // Z k-block kb of tile jj: X W1[64 kb .. 64 kb + 64)^T into TMEM columns [64 kb, 64 kb + 64)
      auto issue_z = [&](int jj, int kb) {
        const uint32_t xa = smem_u32(xv + (jj & 1) * 2 * S::TILE);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_f16(tmem_base + 64 * kb, make_sdesc_sw128(xa + kk * 32, 16, 1024),
                  make_sdesc_sw128(w1a + kb * 64 * 128 + kk * 32, 16, 1024), idZ, kk > 0 ? 1u : 0u);
        mma_commit(&zk[kb]);
      };
      // G1 rows [128 blk, 128 blk + 128) += dZ^T X of tile jj (keys in slot jj & 1); the
      // operands are read MN-major: 64-column runs of h 16 KB apart, 16-token steps of 2 KB
      auto issue_g1 = [&](int jj, int blk) {
        const uint32_t xa = smem_u32(xv + (jj & 1) * 2 * S::TILE);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_f16(tmem_base + S::GCOL + 64 * (HID / 128 + blk),
                  make_sdesc_sw128(ha + blk * 2 * S::TILE + kk * 2048, S::TILE, 1024),
                  make_sdesc_sw128(xa + kk * 2048, S::TILE, 1024), idG, (jj > 0 || kk > 0) ? 1u : 0u);
      };
      auto keys_ready = [&](int jj) {
        return mbar_wait(g.kstats ? &xnorm[jj & 1] : &xfull[jj & 1], (jj >> 1) & 1, abort_flag);
      };
      bool ok = mbar_wait(wfull, 0, abort_flag) && keys_ready(0);
      if (ok) {
        tc_fence_after();
        for (int kb = 0; kb < S::KB; ++kb) issue_z(0, kb);
      }
      for (int j = 0; j < ntiles && ok; ++j) {
        const int s = j & 1;
        // V^ = H W2^T, one k-block of H at a time as the gating writes them (V^ takes TMEM
        // columns [0, 64), Z's first k-block, which has been read by then)
        for (int kb = 0; kb < S::KB && ok; ++kb) {
          if (!(ok = mbar_wait(&hk[kb], j & 1, abort_flag))) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_f16(tmem_base, make_sdesc_sw128(ha + kb * S::TILE + kk * 32, 16, 1024),
                    make_sdesc_sw128(w2a + kb * 64 * 128 + kk * 32, 16, 1024), idV, (kb > 0 || kk > 0) ? 1u : 0u);
        }
        if (!ok) break;
        mma_commit(vfull);
        // dY in shared memory (V^ has been read): G2^T += H^T dY, then dH = dY W2 by k-blocks
        if (!(ok = mbar_wait(dyfull, j & 1, abort_flag))) break;
        tc_fence_after();
        for (int blk = 0; blk < HID / 128; ++blk)
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_f16(tmem_base + S::GCOL + 64 * blk, make_sdesc_sw128(ha + blk * 2 * S::TILE + kk * 2048, S::TILE, 1024),
                    make_sdesc_sw128(dya + kk * 2048, S::TILE, 1024), idG, (j > 0 || kk > 0) ? 1u : 0u);
        for (int kb = 0; kb < S::KB; ++kb) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_f16(tmem_base + 64 * kb, make_sdesc_sw128(dya + kk * 32, 16, 1024),
                    make_sdesc_sw128(w2a + kb * 64 * 128 + kk * 16 * 128, 64 * 128, 1024), idH, kk > 0 ? 1u : 0u);
          mma_commit(&dhk[kb]);
        }
        // per 128-row block of h, once its two dZ k-blocks are written (and their dH read):
        // G1 of this tile, then the next tile's Z k-blocks in the freed TMEM columns (their
        // completion tells the gating that G1 has finished reading those k-blocks of dZ)
        const bool next = j + 1 < ntiles;
        for (int blk = 0; blk < HID / 128 && ok; ++blk) {
          if (!(ok = mbar_wait(&dzk[2 * blk], j & 1, abort_flag) && mbar_wait(&dzk[2 * blk + 1], j & 1, abort_flag)))
            break;
          tc_fence_after();
          issue_g1(j, blk);
          if (next) {
            if (blk == 0 && !(ok = keys_ready(j + 1))) break;
            tc_fence_after();
            issue_z(j + 1, 2 * blk);
            issue_z(j + 1, 2 * blk + 1);
          }
        }
        if (!ok) break;
        mma_commit(&xempty[s]);
      }
      if (ok) mma_commit(gdone);
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
    bool ok = true;
    for (int j = 0; j < ntiles && ok; ++j) {
      const int s = j & 1;
      const int m = (mt0 + j) * 128 + row;
      const bool valid = m < g.rows_valid;
      // ---- E1, k-block by k-block: H = GELU(Z) into shared memory (the previous tile's G1,
      // which read dZ there, completed before this k-block of Z did), G' kept packed in registers
      uint32_t gp[S::COLS / 2];
#pragma unroll
      for (int kb = 0; kb < S::KB; ++kb) {
        ok = __all_sync(0xffffffffu, mbar_wait(&zk[kb], j & 1, abort_flag));
        if (!ok) break;
        tc_fence_after();
        uint32_t zr[16];
        float hv[16];
        tmem_ld16_async(tq + 64 * kb + 16 * slot, zr);
        tmem_wait_regs(zr);
#pragma unroll
        for (int i = 0; i < 16; i += 2) {
          float2 gv, pv;
          gelu_and_grad2(make_float2(__uint_as_float(zr[i]), __uint_as_float(zr[i + 1])), gv, pv);
          hv[i] = valid ? gv.x : 0.f;
          hv[i + 1] = valid ? gv.y : 0.f;
          gp[kb * 8 + i / 2] = pack_bf16x2(pv.x, pv.y);
        }
        put_row16(hs + kb * S::TILE, row, 2 * slot, hv);
        tc_fence_before();
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&hk[kb]);
      }
      if (!ok) break;
      // ---- E2: dY = coef eta (V^ - V) on this warp's 16 output channels
      ok = __all_sync(0xffffffffu, mbar_wait(vfull, j & 1, abort_flag));
      if (!ok) break;
      tc_fence_after();
      {
        uint32_t vr[16];
        tmem_ld16_async(tq + slot * 16, vr);
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
      }
      tc_fence_before();
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(dyfull);
        mbar_arrive(&xempty[s]);
      }
      // ---- E3, k-block by k-block: dZ = dH * G' into shared memory over H (G2^T, its last
      // reader, is done)
#pragma unroll
      for (int kb = 0; kb < S::KB; ++kb) {
        ok = __all_sync(0xffffffffu, mbar_wait(&dhk[kb], j & 1, abort_flag));
        if (!ok) break;
        tc_fence_after();
        uint32_t dr[16];
        tmem_ld16_async(tq + 64 * kb + 16 * slot, dr);
        tmem_wait_regs(dr);
        float dh[16];
#pragma unroll
        for (int i = 0; i < 16; i += 2) {
          const float2 gpf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&gp[kb * 8 + i / 2]));
          dh[i] = valid ? __uint_as_float(dr[i]) * gpf.x : 0.f;
          dh[i + 1] = valid ? __uint_as_float(dr[i + 1]) * gpf.y : 0.f;
        }
        put_row16(hs + kb * S::TILE, row, 2 * slot, dh);
        tc_fence_before();
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&dzk[kb]);
      }
    }
    // ---- the CTA's gradient partials: accumulator columns [slot PER, (slot + 1) PER)
    if (ok && ntiles > 0) ok = __all_sync(0xffffffffu, mbar_wait(gdone, 0, abort_flag));
    if (ok) {
      tc_fence_after();
      constexpr int PER = 16 * S::NACC;  // columns per warp slot (64 or 32)
      const int a0 = slot * PER;
      const int acc = a0 / 64, col0 = a0 % 64;
      const int grow = (acc < S::NACC / 2 ? 128 * acc : HID + 128 * (acc - S::NACC / 2)) + row;
      float* dst = g.part + ((int64_t(sp) * g.batches + z) * (2 * HID) + grow) * 64 + col0;
#pragma unroll
      for (int cc = 0; cc < PER; cc += 32) {
        float v[32];
        if (ntiles > 0) {
          tmem_ld32(tq + S::GCOL + a0 + cc, v);
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = 0.f;
        }
#pragma unroll
        for (int i = 0; i < 32; i += 4)
          *reinterpret_cast<float4*>(dst + cc + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
      }
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
  if (g.splits < 1 || g.batches < 1 || g.m_tiles < 1) return cudaErrorInvalidValue;
  const long long grid = static_cast<long long>(g.batches) * g.splits;
  if (grid > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  kern<<<static_cast<int>(grid), 64 + 32 * S::EW, S::SMEM, st>>>(tX, tV, tW1, tW2, g, status);
  return cudaGetLastError();
}

}  // namespace ttt
