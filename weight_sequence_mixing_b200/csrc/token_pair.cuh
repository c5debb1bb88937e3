// Token phase of the negative-dot-loss update on CTA pairs (tcgen05 cta_group::2).
//
// Same arithmetic as token_dot_kernel (token_phase.cuh): for every tile of chunk
// tokens x 128 hidden units it forms P = V W2[:, blk] and Z13 = X [W1_blk; W3_blk]^T
// (W2's columns are read straight from W2 [d][h] as an MN-major operand, so no W2^T
// copy is needed)
// and writes H' and dZ13 (MLP2: H' and dZ) for the weight-gradient GEMMs (LaCT
// analysis, "Nonlinear memory complements local attention").
//
// Here a tile is 256 tokens, computed by the two CTAs of a cluster as one M = 256
// tensor-core operation: each CTA stages its own 128 token rows (A) and one half
// of the weight block's rows (B), and the even CTA issues MMAs that read both
// CTAs' shared memory and accumulate its 128 rows in its own TMEM and the other
// 128 rows in the peer's.  Each CTA therefore brings in half of the weight bytes a
// single-CTA tile needs for the same multiply-adds: per 64-token-column k-block a
// CTA loads 16 KB of tokens + 8 KB (P) / 16 KB (Z, SwiGLU) of weights instead of
// 16 KB + 16 KB / 32 KB, which is what limits the single-CTA kernel (the rate at
// which an SM can pull operand tiles out of L2).
//
// Two ways to feed the weights.  Streaming (any d): every operand stage carries a k-block
// of tokens and the matching k-block of the weight block, and consecutive tiles of a pair
// step through the hidden blocks.  Resident (d <= 256): a pair keeps its half of one
// hidden block's weights (W2 columns and [W1; W3] rows, 96 KB per CTA for SwiGLU at
// d = 256) in shared memory and walks a range of token tiles; the stages carry tokens
// only, so a CTA pulls 128 instead of 224 KB per tile out of L2.  The pairs come in
// groups of h / 128, one per hidden block, that walk the same token tiles, so every key
// and value tile still crosses HBM once and is read from L2 by the rest of its group.
// The weights are reloaded when the range crosses into the next head, after every MMA
// that read them has completed (the last stage's release).
//
// TMEM per CTA: Z13 in columns [0, 256), P in one of two 128-column slots (256 or
// 384, alternating by tile), so a tile's P phase overlaps the previous tile's
// epilogue.  An epilogue warp reads its first 32-column chunk, computes and packs
// it, reads the second chunk and then releases the tile's TMEM, before any of its
// stores; the leader's next Z phase waits only for that release.
//
// Protocol (CTA 0 of the pair = leader, CTA 1 = peer):
//   full[s]    (leader only)  the leader's producer arms it with both CTAs' bytes;
//                             both producers' TMA loads count their bytes on it.
//   empty[s]   (both)         the leader's MMA commit arrives on both CTAs' copies.
//   wfull      (leader only)  resident weights: both CTAs' weight bytes of a head.
//   tmem_full  (both)         the leader's commit after a tile's last MMA.
//   tmem_empty (leader only)  one arrival per epilogue warp of both CTAs: the tile's
//                             Z13 and P columns have been read.
// All waits are bounded; the kernel ends with a cluster barrier so that neither CTA
// leaves (or frees its TMEM) while the other may still touch its shared memory.
#pragma once
#include "token_phase.cuh"

namespace ttt {

constexpr int kPairResMaxKb = 4;  // resident weights: up to 4 k-blocks (d <= 256)
// Resident weights only when every pair of a full wave of groups gets at least this many
// token tiles to spread its weight load over (the causal language layer's 2048-token chunks
// give a pair one or two: streaming measured faster there).
constexpr int kResMinTiles = 4;

template <bool SWIGLU, bool RESB>
struct PairShape {
  static constexpr int A_BYTES = 128 * 128;         // this CTA's 128 tokens x 64 bf16
  static constexpr int BZ_ROWS = SWIGLU ? 128 : 64;  // this CTA's half of the first-layer rows
  static constexpr int BZ_BYTES = BZ_ROWS * 128;
  static constexpr int BP_ROWS = 64;  // this CTA's half of the block's 128 W2 columns
  static constexpr int BP_BYTES = BP_ROWS * 128;
  static constexpr int Z_STAGE = A_BYTES + BZ_BYTES;
  static constexpr int P_STAGE = A_BYTES + BP_BYTES;
  // streaming: a stage holds a k-block of tokens and one of weights; resident: tokens only
  static constexpr int SLOT = RESB ? A_BYTES : (Z_STAGE > P_STAGE ? Z_STAGE : P_STAGE);
  static constexpr int KB_RES = kPairResMaxKb;
  static constexpr int WP_BYTES = RESB ? KB_RES * BP_BYTES : 0;  // resident W2 columns [kb]
  static constexpr int WZ_BYTES = RESB ? KB_RES * BZ_BYTES : 0;  // resident first-layer rows [kb]
  // operand ring: the P and Z phases are bound by what is in flight.  Resident SwiGLU
  // weights leave room for 7 stages only with one output box per warp: the stages pay
  // more than the box (7 stages and 1 box ran 3% faster than 6 and 2, 5 and 3, 4 and 4)
  static constexpr int STAGES = RESB ? (SWIGLU ? 7 : 8) : 6;
  static constexpr int EW = 16;           // epilogue warps: 4 per TMEM lane quarter
  static constexpr int STG_BYTES = 1024;  // one [32 rows][16 bf16] output box
  static constexpr int STG_BOXES = RESB && SWIGLU ? 1 : 2;  // ring of output boxes per epilogue warp
  static constexpr int STG_WARP = STG_BOXES * STG_BYTES;
  static constexpr int SMEM = 1024 + WP_BYTES + WZ_BYTES + STAGES * SLOT + EW * STG_WARP + 256;
  static constexpr int ZN = SWIGLU ? 256 : 128;  // MMA N of the Z phase (both halves)
  static_assert(SMEM <= 227 * 1024, "shared memory");
  static_assert(2 * STAGES + 4 <= 30, "barrier area");
};

// The tiles of one pair, in processing order.  Streaming: tile k is t = pair + k npairs
// of the (z, token tile, hidden block) sequence, hidden block fastest.  Resident: the
// pair owns hidden block pair % n_tiles and the range of (z, token tile) pairs of its group.
template <bool RESB>
struct PairTiles {
  int count, u0, nt;
  __host__ __device__ PairTiles(const TokGeom& g, int pair, int npairs) {
    if constexpr (RESB) {
      const int groups = npairs / g.n_tiles, gi = pair / g.n_tiles;
      const int64_t U = int64_t(g.batches) * g.m_tiles;
      nt = pair % g.n_tiles;
      u0 = gi < groups ? static_cast<int>(gi * U / groups) : 0;
      count = gi < groups ? static_cast<int>((gi + 1) * U / groups) - u0 : 0;
    } else {
      const int total = g.m_tiles * g.n_tiles * g.batches;
      nt = 0;
      u0 = pair;
      count = pair < total ? (total - pair + npairs - 1) / npairs : 0;
    }
  }
  __host__ __device__ void at(const TokGeom& g, int npairs, int k, int& z, int& mt, int& n) const {
    if constexpr (RESB) {
      const int u = u0 + k;
      z = u / g.m_tiles;
      mt = u % g.m_tiles;
      n = nt;
    } else {
      const int t = u0 + k * npairs;
      n = t % g.n_tiles;
      mt = (t / g.n_tiles) % g.m_tiles;
      z = t / (g.n_tiles * g.m_tiles);
    }
  }
};

template <bool SWIGLU, bool RESB>
__global__ void __launch_bounds__(64 + 32 * PairShape<SWIGLU, RESB>::EW, 1)
    token_pair_kernel(const __grid_constant__ CUtensorMap tX, const __grid_constant__ CUtensorMap tFirst,
                      const __grid_constant__ CUtensorMap tV, const __grid_constant__ CUtensorMap tW2,
                      const __grid_constant__ CUtensorMap tHp, const __grid_constant__ CUtensorMap tDZ,
                      const TokGeom g, unsigned* status) {
  using S = PairShape<SWIGLU, RESB>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* wp = base;                  // resident W2 columns (RESB)
  uint8_t* wz = wp + S::WP_BYTES;      // resident first-layer rows (RESB)
  uint8_t* smem = wz + S::WZ_BYTES;    // operand ring
  uint8_t* stg = smem + S::STAGES * S::SLOT;
  uint64_t* full = reinterpret_cast<uint64_t*>(stg + S::EW * S::STG_WARP);
  uint64_t* empty = full + S::STAGES;
  uint64_t* tmem_full = empty + S::STAGES;
  uint64_t* tmem_empty = tmem_full + 1;
  uint64_t* drain = tmem_empty + 1;
  uint64_t* wfull = drain + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(wfull + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const uint32_t rank = cluster_rank() & 1u;
  const bool leader = rank == 0;
  const int warp = threadIdx.x >> 5;
  const int lane = static_cast<int>(lane_id());
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const PairTiles<RESB> tiles(g, pair, npairs);  // m_tiles counts 256-token tiles
  const int KB = g.kblocks;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(tmem_full, 1);
    mbar_init(tmem_empty, 2 * S::EW);
    mbar_init(drain, 1);
    mbar_init(wfull, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, 512);
    tmem_relinquish_pair();
  }
  // both CTAs' barriers initialised and the pair's TMEM allocated before any use
  tc_fence_before();
  cluster_barrier();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    if (elect_one()) {
      tma_prefetch_desc(&tX);
      tma_prefetch_desc(&tFirst);
      tma_prefetch_desc(&tV);
      tma_prefetch_desc(&tW2);
      const uint32_t full0 = mapa_shared(smem_u32(full), 0);  // the leader's full[0]
      const uint32_t wfull0 = mapa_shared(smem_u32(wfull), 0);
      int it = 0, wz_head = -1;
      bool stop = false;
      for (int k = 0; k < tiles.count && !stop; ++k) {
        int z, mt, nt;
        tiles.at(g, npairs, k, z, mt, nt);
        const int m0 = mt * 256 + static_cast<int>(rank) * 128;
        if (RESB && z != wz_head) {
          // every MMA that read the previous head's weights has completed: the last
          // stage it issued has been released
          if (it > 0 && !mbar_wait(&empty[(it - 1) % S::STAGES], ((it - 1) / S::STAGES) & 1, abort_flag)) {
            stop = true;
            break;
          }
          if (leader) mbar_arrive_expect_tx(wfull, 2 * KB * (S::BP_BYTES + S::BZ_BYTES));
          for (int kb = 0; kb < KB; ++kb) {
            tma_load_3d_pair(wp + kb * S::BP_BYTES, &tW2, wfull0, nt * 128 + static_cast<int>(rank) * S::BP_ROWS,
                             kb * 64, z);
            tma_load_3d_pair(wz + kb * S::BZ_BYTES, &tFirst, wfull0, kb * 64,
                             nt * (2 * S::BZ_ROWS) + static_cast<int>(rank) * S::BZ_ROWS, z);
          }
          wz_head = z;
        }
        for (int phase = 0; phase < 2 && !stop; ++phase) {
          for (int kb = 0; kb < KB; ++kb, ++it) {
            const int s = it % S::STAGES;
            const uint32_t ph = (it / S::STAGES) & 1;
            if (it >= S::STAGES && !mbar_wait(&empty[s], ph ^ 1, abort_flag)) {
              stop = true;
              break;
            }
            uint8_t* st = smem + s * S::SLOT;
            const uint32_t fb = full0 + static_cast<uint32_t>(s) * 8u;
            if (phase == 0) {
              if (leader) mbar_arrive_expect_tx(&full[s], 2 * (RESB ? S::A_BYTES : S::P_STAGE));
              tma_load_3d_pair(st, &tV, fb, kb * 64, m0 + g.v_off, z);
              // W2 [d][h]: 64 of the block's columns (N) x the k-block's 64 rows (K), MN-major
              if (!RESB)
                tma_load_3d_pair(st + S::A_BYTES, &tW2, fb, nt * 128 + static_cast<int>(rank) * S::BP_ROWS, kb * 64,
                                 z);
            } else {
              if (leader) mbar_arrive_expect_tx(&full[s], 2 * (RESB ? S::A_BYTES : S::Z_STAGE));
              tma_load_3d_pair(st, &tX, fb, kb * 64, m0 + g.x_off, z);
              if (!RESB)
                tma_load_3d_pair(st + S::A_BYTES, &tFirst, fb, kb * 64,
                                 nt * (2 * S::BZ_ROWS) + static_cast<int>(rank) * S::BZ_ROWS, z);
            }
          }
        }
      }
      if (!*abort_flag) {
        // every stage released: the leader's last commits have landed here
        for (int j = max(0, it - S::STAGES); j < it; ++j)
          if (!mbar_wait(&empty[j % S::STAGES], (j / S::STAGES) & 1, abort_flag)) break;
      }
      if (*abort_flag) {
        // loads still in flight complete within microseconds; give them a millisecond
        const unsigned long long t0 = global_ns();
        while (global_ns() - t0 < 1000000ull) {
        }
      }
    }
  } else if (warp == 1) {
    if (leader && elect_one()) {
      constexpr uint32_t idP = make_idesc(256, 128, 1, false, true);
      constexpr uint32_t idZ = make_idesc(256, S::ZN, 1, false, false);
      const uint32_t sbase = smem_u32(smem), wpbase = smem_u32(wp), wzbase = smem_u32(wz);
      int it = 0, j = 0, wz_head = -1, wloads = 0;
      bool stop = false;
      for (; j < tiles.count && !stop; ++j) {
        const uint32_t pcol = (j & 1) ? 384u : 256u;
        if (RESB) {
          int z, mt, nt;
          tiles.at(g, npairs, j, z, mt, nt);
          if (z != wz_head) {  // this head's weights have landed in both CTAs
            if (!mbar_wait_cluster(wfull, wloads & 1, abort_flag)) {
              stop = true;
              break;
            }
            tc_fence_after();
            ++wloads;
            wz_head = z;
          }
        }
        for (int phase = 0; phase < 2 && !stop; ++phase) {
          if (phase == 1) {
            // both CTAs' epilogues have read the previous tile (Z13 and its P slot)
            if (j > 0 && !mbar_wait_cluster(tmem_empty, (j - 1) & 1, abort_flag)) {
              stop = true;
              break;
            }
            tc_fence_after();
          }
          const uint32_t dcol = phase == 0 ? pcol : 0u;
          const uint32_t id = phase == 0 ? idP : idZ;
          for (int kb = 0; kb < KB; ++kb, ++it) {
            const int s = it % S::STAGES;
            const uint32_t ph = (it / S::STAGES) & 1;
            if (!mbar_wait_cluster(&full[s], ph, abort_flag)) {
              stop = true;
              break;
            }
            tc_fence_after();
            const uint32_t a = sbase + s * S::SLOT;
            const uint32_t b = RESB ? (phase == 0 ? wpbase + kb * S::BP_BYTES : wzbase + kb * S::BZ_BYTES)
                                    : a + S::A_BYTES;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              // P phase: B is MN-major (16 K-rows of 128 bytes per step); Z phase: K-major
              const uint64_t db = phase == 0 ? make_sdesc_sw128(b + kk * 16 * 128, 8192, 1024)
                                             : make_sdesc_sw128(b + kk * 32, 16, 1024);
              mma_f16_pair(tmem_base + dcol, make_sdesc_sw128(a + kk * 32, 16, 1024), db, id,
                           (kb > 0 || kk > 0) ? 1u : 0u);
            }
            mma_commit_pair(&empty[s], 0x3);
          }
        }
        if (!stop) mma_commit_pair(tmem_full, 0x3);
      }
      // the last tile's epilogue arrivals (some remote) have all landed
      if (!stop && j > 0) mbar_wait_cluster(tmem_empty, (j - 1) & 1, abort_flag);
      if (*abort_flag) {
        volatile int never = 0;
        mma_commit_pair(drain, 0x1);
        mbar_wait(drain, 0, &never);
      }
    }
  } else {
    // 16 epilogue warps, four per TMEM lane quarter: warp slot s of quarter q owns the
    // 16-column chunks 16 s and 64 + 16 s of rows 32 q .. 32 q + 31 of every tile
    const int ew = warp - 2;
    const int q = warp & 3;
    const int slot = ew >> 2;
    uint8_t* my = stg + ew * S::STG_WARP;
    const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
    const uint32_t tmem_empty0 = mapa_shared(smem_u32(tmem_empty), 0);
    int nt = 0, z = 0, row = 0;
    int box = 0;  // output boxes this warp has staged: a ring of STG_BOXES in shared memory
    // stage one [32 rows][16 columns] bf16 box and store it with TMA; the ring slot's
    // previous store (STG_BOXES boxes ago) must have finished reading it
    auto emit = [&](const uint32_t (&w)[8], const CUtensorMap* m, int c0) {
      uint8_t* bx = my + (box % S::STG_BOXES) * S::STG_BYTES;
      if (lane == 0) bulk_wait_read<S::STG_BOXES - 1>();
      __syncwarp();
      stage_packed_sw32(bx, lane, w);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        tma_store_3d(m, bx, c0, row, z);
        bulk_commit();
      }
      ++box;
    };
    auto emit_chunk = [&](const uint32_t (&w)[3][8], int cc) {
      emit(w[0], &tHp, nt * 128 + cc);
      if constexpr (SWIGLU) {
        emit(w[1], &tDZ, nt * 256 + cc);
        emit(w[2], &tDZ, nt * 256 + 128 + cc);
      } else {
        emit(w[1], &tDZ, nt * 128 + cc);
      }
    };
    for (int j = 0; j < tiles.count; ++j) {
      int mt;
      tiles.at(g, npairs, j, z, mt, nt);
      const int m0 = mt * 256 + static_cast<int>(rank) * 128;
      const bool ready = __all_sync(0xffffffffu, mbar_wait_cluster(tmem_full, j & 1, abort_flag));
      if (!ready) break;
      tc_fence_after();
      const int m = m0 + q * 32 + lane;
      const bool valid = m < g.rows_valid;
      const float e = valid ? (g.eta ? g.eta[z * g.eta_zs + g.t0 + m] : g.eta_scalar) : 0.0f;
      const uint32_t pcol = (j & 1) ? 384u : 256u;
      row = m0 + q * 32;
      const bool store = row < g.rows_alloc;
      // chunk a (columns cca) is read, computed and packed to bf16 before chunk b
      // (cca + 64) is read; then TMEM is released, before any store.
      const int cca = 16 * slot;
      uint32_t wa[3][8];
      {
        uint32_t r1[16], r3[16], rp[16];
        tmem_ld16_async(taddr + cca, r1);
        if constexpr (SWIGLU) tmem_ld16_async(taddr + 128 + cca, r3);
        tmem_ld16_async(taddr + pcol + cca, rp);
        tmem_wait_regs(r1);
        if constexpr (SWIGLU) tmem_wait_regs(r3);
        tmem_wait_regs(rp);
        float hv[16], d1[16], d3[16];
        token_dot_math<SWIGLU, 16>(e, r1, r3, rp, hv, d1, d3);
        pack_row_bf16(hv, wa[0]);
        pack_row_bf16(d1, wa[1]);
        if constexpr (SWIGLU) pack_row_bf16(d3, wa[2]);
      }
      uint32_t r1[16], r3[16], rp[16];
      tmem_ld16_async(taddr + cca + 64, r1);
      if constexpr (SWIGLU) tmem_ld16_async(taddr + 128 + cca + 64, r3);
      tmem_ld16_async(taddr + pcol + cca + 64, rp);
      tmem_wait_regs(r1);
      if constexpr (SWIGLU) tmem_wait_regs(r3);
      tmem_wait_regs(rp);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(tmem_empty0);
      if (store) emit_chunk(wa, cca);
      {
        float hv[16], d1[16], d3[16];
        token_dot_math<SWIGLU, 16>(e, r1, r3, rp, hv, d1, d3);
        uint32_t wb[3][8];
        pack_row_bf16(hv, wb[0]);
        pack_row_bf16(d1, wb[1]);
        if constexpr (SWIGLU) pack_row_bf16(d3, wb[2]);
        if (store) emit_chunk(wb, cca + 64);
      }
    }
    if (lane == 0) bulk_wait0();
  }

  __syncwarp();
  tc_fence_before();
  cluster_barrier();
  tc_fence_after();
  if (threadIdx.x == 0 && *abort_flag) set_status(status, kStatusTimeout);
  if (warp == 1) tmem_dealloc_pair(tmem_base, 512);
}

template <bool SWIGLU, bool RESB>
cudaLaunchConfig_t pair_launch_config(int pairs, cudaStream_t st, cudaLaunchAttribute* attr) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * pairs, 1, 1);
  cfg.blockDim = dim3(64 + 32 * PairShape<SWIGLU, RESB>::EW, 1, 1);
  cfg.dynamicSmemBytes = PairShape<SWIGLU, RESB>::SMEM;
  cfg.stream = st;
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cfg;
}

// CTA pairs of one form of this kernel that can be resident at once (0: none).
template <bool SWIGLU, bool RESB>
int token_pair_capacity_of() {
  static IntPerDevice caps;
  return caps.get(current_device(), [] {
    auto kern = token_pair_kernel<SWIGLU, RESB>;
    int cap = 0;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, PairShape<SWIGLU, RESB>::SMEM) ==
        cudaSuccess) {
      cudaLaunchAttribute attr[1];
      cudaLaunchConfig_t cfg = pair_launch_config<SWIGLU, RESB>(1, nullptr, attr);
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) == cudaSuccess && n > 0) cap = n;
    }
    cudaGetLastError();  // a refused query leaves no sticky error behind
    return cap;
  });
}

// CTA pairs of the streaming form (the one every d accepts) that can be resident at
// once (0: none, use the single-CTA kernel).
template <bool SWIGLU>
int token_pair_capacity() {
  return token_pair_capacity_of<SWIGLU, false>();
}

// Form and grid of the pair kernel for geometry g (host logic): resident weights when
// d <= 256 and a full wave of groups (cap_res / n_tiles groups of n_tiles pairs) gives every
// pair at least kResMinTiles token tiles; streaming on min(tiles, cap_str) pairs otherwise.
// cap_res, cap_str: pairs of each form that fit the device.  false: no pair fits.
inline bool pair_grid(const TokGeom& g, int cap_res, int cap_str, bool& resb, int& pairs) {
  const long long total = static_cast<long long>(g.m_tiles) * g.n_tiles * g.batches;
  if (g.kblocks <= kPairResMaxKb && g.n_tiles > 0) {
    const long long groups = cap_res / g.n_tiles, U = static_cast<long long>(g.m_tiles) * g.batches;
    if (groups > 0 && U >= kResMinTiles * groups) {
      resb = true;
      pairs = static_cast<int>(groups * g.n_tiles);
      return true;
    }
  }
  if (cap_str <= 0) return false;
  resb = false;
  pairs = static_cast<int>(std::min<long long>(total, cap_str));
  return true;
}

// g.m_tiles counts 256-token tiles; g.rows_alloc bounds the rows the stores may write.
template <bool SWIGLU>
cudaError_t launch_token_pair(const CUtensorMap& tX, const CUtensorMap& tFirstHalf, const CUtensorMap& tV,
                              const CUtensorMap& tW2Mn, const CUtensorMap& tHp, const CUtensorMap& tDZ,
                              const TokGeom& g, unsigned* status, cudaStream_t st) {
  const long long total = static_cast<long long>(g.m_tiles) * g.n_tiles * g.batches;
  if (total <= 0) return cudaSuccess;
  if (total > 0x7fffffffLL || g.kblocks <= 0) return cudaErrorInvalidConfiguration;
  const int cap_res = g.kblocks <= kPairResMaxKb ? token_pair_capacity_of<SWIGLU, true>() : 0;
  bool resb = false;
  int pairs = 0;
  if (!pair_grid(g, cap_res, token_pair_capacity<SWIGLU>(), resb, pairs)) return cudaErrorInvalidConfiguration;
  cudaLaunchAttribute attr[1];
  if (resb) {
    cudaLaunchConfig_t cfg = pair_launch_config<SWIGLU, true>(pairs, st, attr);
    return cudaLaunchKernelEx(&cfg, token_pair_kernel<SWIGLU, true>, tX, tFirstHalf, tV, tW2Mn, tHp, tDZ, g, status);
  }
  cudaLaunchConfig_t cfg = pair_launch_config<SWIGLU, false>(pairs, st, attr);
  return cudaLaunchKernelEx(&cfg, token_pair_kernel<SWIGLU, false>, tX, tFirstHalf, tV, tW2Mn, tHp, tDZ, g, status);
}

}  // namespace ttt
