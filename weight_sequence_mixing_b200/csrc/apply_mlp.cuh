// Apply on the queries, O = F_W(Q), as one kernel with the hidden layer kept on chip
// (ViT3 digest section 02: the queries read the updated fast weights; LaCT analysis,
// "Nonlinear memory complements local attention": SwiGLU F(x) = (SiLU(x W1^T) * x W3^T) W2^T).
//
// A CTA owns 128 query rows of one head at a time (persistent over tiles).  The row
// tile of Q stays in shared memory; for every block of 128 hidden units
//   Z   = Q [W1_blk; W3_blk]^T (SwiGLU: z1 | z3, 256 TMEM columns; GELU MLP: z, 128)
//   H   = SiLU(z1) z3  (or GELU(z)), bf16, written by the epilogue warps straight into
//         shared memory in the 128-byte-swizzled K-major layout an MMA operand needs
//   O  += H W2[:, blk]^T  (d TMEM columns, accumulated over the hidden blocks)
// and after the last block the epilogue writes O.  The next block's Z MMAs overlap
// the gating of the current one (Z is read out of TMEM before the gating math).
// d <= 256 (O and Z together fit the 512 TMEM columns).
//
// Warps: 0 TMA producer, 1 MMA issuer, then EW epilogue warps (EW / 4 per TMEM lane
// quarter; warp part j of a quarter owns 128 / (EW / 4) adjacent hidden columns of a block,
// inside one 64-column k-block of the H operand, and the matching share of O's columns).
// Every wait is bounded.
#pragma once
#include "epilogues.cuh"
#include "gelu_fwd.cuh"

namespace ttt {

struct ApplyGeom {
  int m_tiles, batches;  // 128-row query tiles per head, heads (z)
  int hblocks;           // h / 128
  int rows_valid;        // query rows of each head
  int row0;              // first query row of this call (causal chunks) in Q and O
  int64_t o_zs;          // elements between heads in O
};

template <bool SWIGLU, int D, int EPIW = 8>
struct ApplyShape {
  static constexpr int KB = D / 64;                  // k-blocks of Q (64 channels each)
  static constexpr int ZN = SWIGLU ? 256 : 128;      // first-layer rows per hidden block
  static constexpr int Q_BYTES = KB * 128 * 128;     // 128 rows x D bf16
  static constexpr int H_BYTES = 2 * 128 * 128;      // 128 rows x 128 hidden bf16
  static constexpr int STAGE = (ZN > D ? ZN : D) * 128;  // one B k-block (64 K elements)
  static constexpr int STAGES = 3;
  static constexpr int EW = EPIW;                    // epilogue warps: EW / 4 per TMEM lane quarter
  static constexpr int NQ = EW / 4;
  static constexpr int HC = 128 / NQ;                // hidden columns of a block per epilogue thread
  static_assert(EW == 8 || EW == 16, "epilogue warps");
  static constexpr int SMEM = 1024 + Q_BYTES + H_BYTES + STAGES * STAGE + 256;
  static constexpr uint32_t Z_COL = 256;             // Z accumulator columns [256, 256 + ZN)
  static_assert(D == 64 || D == 128 || D == 256, "d");
  static_assert(SMEM <= 227 * 1024, "shared memory");
};

template <bool SWIGLU, int D, int EPIW>
__global__ void __launch_bounds__(64 + 32 * ApplyShape<SWIGLU, D, EPIW>::EW, 1)
    apply_mlp_kernel(const __grid_constant__ CUtensorMap tQ, const __grid_constant__ CUtensorMap tFirst,
                     const __grid_constant__ CUtensorMap tW2, const ApplyGeom g, bf16* O, unsigned* status) {
  using S = ApplyShape<SWIGLU, D, EPIW>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* qs = smem;
  uint8_t* hs = qs + S::Q_BYTES;
  uint8_t* ring = hs + S::H_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(ring + S::STAGES * S::STAGE);
  uint64_t* empty = full + S::STAGES;
  uint64_t* qfull = empty + S::STAGES;  // the tile's Q rows landed
  uint64_t* qempty = qfull + 1;         // the tile's MMAs are done with them
  uint64_t* zfull = qempty + 1;         // Z of a hidden block is in TMEM
  uint64_t* zempty = zfull + 1;         // the epilogue has read it
  uint64_t* hfull = zempty + 1;         // H of the block is in shared memory
  uint64_t* hempty = hfull + 1;         // the O MMAs reading H are done
  uint64_t* ofull = hempty + 1;         // O of the tile is complete
  uint64_t* oempty = ofull + 1;         // the epilogue has read O
  uint64_t* drain = oempty + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = static_cast<int>(lane_id());
  const int total = g.m_tiles * g.batches;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(qfull, 1);
    mbar_init(qempty, 1);
    mbar_init(zfull, 1);
    mbar_init(zempty, S::EW);
    mbar_init(hfull, S::EW);
    mbar_init(hempty, 1);
    mbar_init(ofull, 1);
    mbar_init(oempty, S::EW);
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

  // The CTA's hidden blocks in order, across its tiles: block nb is block nb % hblocks of
  // the CTA's tile nb / hblocks.  The MMA issuer runs one block ahead: Z of block nb + 1 is
  // issued as soon as the epilogue has read Z of block nb out of TMEM, before the O
  // MMAs of block nb (which wait for its gating), so the next block's Z is ready when
  // the epilogue gets to it; the next tile's Q is loaded as soon as the current tile's
  // last Z MMA has read Q.  The producer fills the operand ring in the same order:
  // [Q(0)] Z(0), then per block nb: [Q(next tile)] Z(nb + 1), O(nb).
  const int ntiles_cta = total > static_cast<int>(blockIdx.x) ? (total - 1 - blockIdx.x) / gridDim.x + 1 : 0;
  const int nblocks = ntiles_cta * g.hblocks;
  auto tile_of = [&](int jt) { return static_cast<int>(blockIdx.x) + jt * static_cast<int>(gridDim.x); };

  if (warp == 0) {
    if (elect_one() && nblocks > 0) {
      tma_prefetch_desc(&tQ);
      tma_prefetch_desc(&tFirst);
      tma_prefetch_desc(&tW2);
      int it = 0;
      bool stop = false;
      // one ring slot per k-block: the first-layer rows of a block (K = d) or W2's columns (K = hidden)
      auto ring_load = [&](bool first_layer, int i, int hb, int z) {
        const int s = it % S::STAGES;
        const uint32_t ph = (it / S::STAGES) & 1;
        if (it >= S::STAGES && !mbar_wait(&empty[s], ph ^ 1, abort_flag)) {
          stop = true;
          return;
        }
        uint8_t* st = ring + s * S::STAGE;
        if (first_layer) {
          mbar_arrive_expect_tx(&full[s], S::ZN * 128);
          tma_load_3d(st, &tFirst, &full[s], i * 64, hb * S::ZN, z);
        } else {
          mbar_arrive_expect_tx(&full[s], D * 128);
          tma_load_3d(st, &tW2, &full[s], hb * 128 + i * 64, 0, z);
        }
        ++it;
      };
      // Q of the CTA's tile jt (after the previous tile's Z MMAs have read Q)
      auto q_load = [&](int jt) {
        if (jt > 0 && !mbar_wait(qempty, (jt - 1) & 1, abort_flag)) {
          stop = true;
          return;
        }
        const int t = tile_of(jt), mt = t % g.m_tiles, z = t / g.m_tiles;
        mbar_arrive_expect_tx(qfull, S::Q_BYTES);
        for (int kb = 0; kb < S::KB; ++kb) tma_load_3d(qs + kb * 128 * 128, &tQ, qfull, kb * 64, g.row0 + mt * 128, z);
      };
      auto z_loads = [&](int nb) {
        const int jt = nb / g.hblocks, hb = nb % g.hblocks, z = tile_of(jt) / g.m_tiles;
        if (hb == 0) q_load(jt);
        for (int i = 0; i < S::KB && !stop; ++i) ring_load(true, i, hb, z);
      };
      z_loads(0);
      for (int nb = 0; nb < nblocks && !stop; ++nb) {
        if (nb + 1 < nblocks) z_loads(nb + 1);
        const int hb = nb % g.hblocks, z = tile_of(nb / g.hblocks) / g.m_tiles;
        for (int i = 0; i < 2 && !stop; ++i) ring_load(false, i, hb, z);
      }
      if (*abort_flag) {
        // copies already in flight land within microseconds; give them a millisecond
        const unsigned long long t0 = global_ns();
        while (global_ns() - t0 < 1000000ull) {
        }
      }
    }
  } else if (warp == 1) {
    if (elect_one() && nblocks > 0) {
      constexpr uint32_t idZ = make_idesc(128, S::ZN, 1, false, false);
      constexpr uint32_t idO = make_idesc(128, D, 1, false, false);
      const uint32_t qbase = smem_u32(qs), hbase = smem_u32(hs), rbase = smem_u32(ring);
      int it = 0;
      bool ok = true;
      // Z = Q [W1_blk; W3_blk]^T of block nb (Z has been read out of TMEM by then)
      auto issue_z = [&](int nb) {
        const int jt = nb / g.hblocks, hb = nb % g.hblocks;
        if (hb == 0 && !(ok = mbar_wait(qfull, jt & 1, abort_flag))) return;
        tc_fence_after();
        for (int kb = 0; kb < S::KB; ++kb, ++it) {
          const int s = it % S::STAGES;
          if (!(ok = mbar_wait(&full[s], (it / S::STAGES) & 1, abort_flag))) return;
          tc_fence_after();
          const uint32_t a = qbase + kb * 128 * 128, b = rbase + s * S::STAGE;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_f16(tmem_base + S::Z_COL, make_sdesc_sw128(a + kk * 32, 16, 1024),
                    make_sdesc_sw128(b + kk * 32, 16, 1024), idZ, (kb > 0 || kk > 0) ? 1u : 0u);
          mma_commit(&empty[s]);
        }
        mma_commit(zfull);
        if (hb == g.hblocks - 1) mma_commit(qempty);  // the tile's last read of Q
      };
      issue_z(0);
      for (int nb = 0; nb < nblocks && ok; ++nb) {
        const int jt = nb / g.hblocks, hb = nb % g.hblocks;
        if (nb + 1 < nblocks) {
          if (!(ok = mbar_wait(zempty, nb & 1, abort_flag))) break;
          issue_z(nb + 1);
          if (!ok) break;
        }
        // H of block nb written by the epilogue (and, for a tile's first block, O of the
        // previous tile read out of TMEM): O += H W2[:, blk]^T
        if (!(ok = mbar_wait(hfull, nb & 1, abort_flag))) break;
        if (hb == 0 && jt > 0 && !(ok = mbar_wait(oempty, (jt - 1) & 1, abort_flag))) break;
        tc_fence_after();
        for (int kh = 0; kh < 2 && ok; ++kh, ++it) {
          const int s = it % S::STAGES;
          if (!(ok = mbar_wait(&full[s], (it / S::STAGES) & 1, abort_flag))) break;
          tc_fence_after();
          const uint32_t a = hbase + kh * 128 * 128, b = rbase + s * S::STAGE;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_f16(tmem_base, make_sdesc_sw128(a + kk * 32, 16, 1024), make_sdesc_sw128(b + kk * 32, 16, 1024),
                    idO, (hb > 0 || kh > 0 || kk > 0) ? 1u : 0u);
          mma_commit(&empty[s]);
        }
        if (!ok) break;
        mma_commit(hempty);
        if (hb == g.hblocks - 1) mma_commit(ofull);
      }
      if (*abort_flag) {
        volatile int never = 0;
        mma_commit(drain);
        mbar_wait(drain, 0, &never);
      }
    }
  } else {
    const int q = warp & 3;
    const int part = (warp - 2) >> 2;  // hidden columns [HC part, HC part + HC) of a block
    const int hc0 = part * S::HC;
    const int row = q * 32 + lane;
    const uint32_t tq = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
    // this thread's row of H's k-block hc0 / 64, from 16-byte chunk (hc0 % 64) / 8 on
    uint8_t* hk = hs + (hc0 / 64) * 128 * 128 + row * 128;
    const int k0 = (hc0 % 64) / 8;
    int j = 0, nz = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < total && ok; t += gridDim.x, ++j) {
      const int mt = t % g.m_tiles, z = t / g.m_tiles;
      for (int hb = 0; hb < g.hblocks; ++hb, ++nz) {
        ok = __all_sync(0xffffffffu, mbar_wait(zfull, nz & 1, abort_flag));
        if (!ok) break;
        tc_fence_after();
        // read this thread's HC hidden columns of Z (and z3), then release the TMEM
        uint32_t packed[S::HC / 2];
#pragma unroll
        for (int c = 0; c < S::HC / 32; ++c) {
          float z1[32], z3[32];
          tmem_ld32(tq + S::Z_COL + hc0 + c * 32, z1);
          if constexpr (SWIGLU) tmem_ld32(tq + S::Z_COL + 128 + hc0 + c * 32, z3);
#pragma unroll
          for (int i = 0; i < 32; i += 2) {
            float a, b;
            if constexpr (SWIGLU) {
              a = z1[i] * sigmoid_dev(z1[i]) * z3[i];
              b = z1[i + 1] * sigmoid_dev(z1[i + 1]) * z3[i + 1];
            } else {
              const float2 gv = gelu_fwd2(make_float2(z1[i], z1[i + 1]));
              a = gv.x;
              b = gv.y;
            }
            packed[c * 16 + i / 2] = pack_bf16x2(a, b);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(zempty);
        // the previous block's O MMAs are done reading H
        if (nz > 0) {
          ok = __all_sync(0xffffffffu, mbar_wait(hempty, (nz - 1) & 1, abort_flag));
          if (!ok) break;
        }
        // HC bf16 = HC / 8 chunks of 16 bytes; chunk k of row r sits at k ^ (r & 7)
#pragma unroll
        for (int k = 0; k < S::HC / 8; ++k)
          *reinterpret_cast<uint4*>(hk + 16 * ((k0 + k) ^ (row & 7))) =
              make_uint4(packed[4 * k], packed[4 * k + 1], packed[4 * k + 2], packed[4 * k + 3]);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(hfull);
      }
      if (!ok) break;
      ok = __all_sync(0xffffffffu, mbar_wait(ofull, j & 1, abort_flag));
      if (!ok) break;
      tc_fence_after();
      const int m = mt * 128 + row;
      const bool valid = m < g.rows_valid;
      bf16* orow = O + z * g.o_zs + int64_t(g.row0 + m) * D;
      bool bad = false;
      // O columns [part D / NQ, (part + 1) D / NQ) of this thread's row
      constexpr int OC = D / S::NQ;
      if constexpr (OC >= 32) {
#pragma unroll 1
        for (int cc = part * OC; cc < (part + 1) * OC; cc += 32) {
          float v[32];
          tmem_ld32(tmem_base + (static_cast<uint32_t>(q * 32) << 16) + cc, v);
          if (!valid) continue;
#pragma unroll
          for (int i = 0; i < 32; ++i) bad |= !isfinite(v[i]);
          store_bf16x32(orow + cc, v);
        }
      } else {  // 16 columns
        uint32_t r[16];
        tmem_ld16_async(tmem_base + (static_cast<uint32_t>(q * 32) << 16) + part * OC, r);
        tmem_wait_regs(r);
        if (valid) {
          uint32_t w[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float a = __uint_as_float(r[2 * i]), b = __uint_as_float(r[2 * i + 1]);
            bad |= !isfinite(a) || !isfinite(b);
            w[i] = pack_bf16x2(a, b);
          }
          uint4* o4 = reinterpret_cast<uint4*>(orow + part * OC);
          o4[0] = make_uint4(w[0], w[1], w[2], w[3]);
          o4[1] = make_uint4(w[4], w[5], w[6], w[7]);
        }
      }
      if (bad) set_status(status, kStatusNonFinite);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(oempty);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (threadIdx.x == 0 && *abort_flag) set_status(status, kStatusTimeout);
  if (warp == 1) tmem_dealloc(tmem_base, 512);
}

// The GELU MLP's epilogue (an erf per hidden unit) is the slower one: it gets 16 warps.
template <bool SWIGLU, int D>
cudaError_t launch_apply_mlp(const CUtensorMap& tQ, const CUtensorMap& tFirst, const CUtensorMap& tW2,
                             const ApplyGeom& g, bf16* O, unsigned* status, cudaStream_t st) {
  constexpr int EPIW = SWIGLU ? 8 : 16;
  using S = ApplyShape<SWIGLU, D, EPIW>;
  auto kern = apply_mlp_kernel<SWIGLU, D, EPIW>;
  static OncePerDevice configured;
  const int set = configured.run(current_device(), [&] {
    return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, S::SMEM);
  });
  if (set != 0) return static_cast<cudaError_t>(set);
  const long long total = static_cast<long long>(g.m_tiles) * g.batches;
  if (total <= 0) return cudaSuccess;
  if (total > 0x7fffffffLL || g.hblocks <= 0) return cudaErrorInvalidConfiguration;
  const int grid = static_cast<int>(std::min<long long>(total, sm_count()));
  kern<<<grid, 64 + 32 * S::EW, S::SMEM, st>>>(tQ, tFirst, tW2, g, O, status);
  return cudaGetLastError();
}

}  // namespace ttt
