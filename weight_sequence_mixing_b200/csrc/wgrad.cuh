// Weight-gradient GEMMs of the TTT update: reductions over a chunk's tokens,
//   D[rows, cols] = sum_t A[t, rows] * B[t, cols]
// with both operands row-major [tokens][features] buffers read MN-major by TMA
// (G2^T = H'^T V, [G1; G3] = dZ13^T K, ...), split-K over tokens with fp32
// partials.  ("chunk gradients summed with each token's learning rate", LaCT
// analysis, "Nonlinear memory complements local attention"; eta is already in
// the activations.)
//
// A CTA computes a 256 x BN tile as two 128-row TMEM accumulators that share
// every B tile it loads: 2 x 128 x BN x 64 multiply-adds per (32 KB + BN x 128 B)
// brought into shared memory, which keeps the tensor pipe fed from L2 (a 128-row
// tile brings in ~1.5x the bytes per multiply-add).  Warp roles as in tc_gemm.cuh;
// the 8 epilogue warps split the two accumulators (warps 2-5: rows 0-127,
// warps 6-9: rows 128-255).
#pragma once
#include "tc_gemm.cuh"

namespace ttt {

template <int BN, int STAGES>
struct WgShape {
  static constexpr int A_BYTES = 256 * 128;  // 256 rows x 64 tokens, bf16
  static constexpr int B_BYTES = BN * 128;
  static constexpr int STAGE = A_BYTES + B_BYTES;
  static constexpr int TMEM_COLS = tmem_cols_for(2 * BN);
  static constexpr int SMEM = 1024 + STAGES * STAGE + 256;
  static_assert(BN == 64 || BN == 128 || BN == 256, "BN");
  static_assert(SMEM <= 227 * 1024, "shared memory");
};

// Same tile order as decode_tile (N-tile fastest), with 256-row M tiles.
__device__ __forceinline__ TileCoord decode_tile256(const TcGeom& g, int t, int bn) {
  TileCoord c;
  const int mtiles = g.m_tiles0 + g.m_tiles1;
  const int nt = t % g.n_tiles;
  int r = t / g.n_tiles;
  const int mt = r % mtiles;
  r /= mtiles;
  c.z = r % g.batches;
  c.split = r / g.batches;
  c.problem = mt >= g.m_tiles0 ? 1 : 0;
  c.m0 = (c.problem ? mt - g.m_tiles0 : mt) * 256;
  c.n0 = nt * bn;
  c.kb_begin = c.split * g.kb_per_split;
  c.nkb = max(0, min(g.kblocks, c.kb_begin + g.kb_per_split) - c.kb_begin);
  return c;
}

template <int BN, int STAGES, class Epi>
__global__ void __launch_bounds__(320, 1)
    wgrad_kernel(const __grid_constant__ CUtensorMap tA0, const __grid_constant__ CUtensorMap tB0,
                 const __grid_constant__ CUtensorMap tA1, const __grid_constant__ CUtensorMap tB1, const TcGeom g,
                 const Epi epi, unsigned* status) {
  using S = WgShape<BN, STAGES>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * S::STAGE);
  uint64_t* empty = full + STAGES;
  uint64_t* tmem_full = empty + STAGES;
  uint64_t* tmem_empty = tmem_full + 1;
  uint64_t* drain = tmem_empty + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int total = (g.m_tiles0 + g.m_tiles1) * g.n_tiles * g.batches * g.splits;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(tmem_full, 1);
    mbar_init(tmem_empty, 8);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, S::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    if (elect_one()) {
      tma_prefetch_desc(&tA0);
      tma_prefetch_desc(&tB0);
      if (g.m_tiles1 > 0) {
        tma_prefetch_desc(&tA1);
        tma_prefetch_desc(&tB1);
      }
      int it = 0;
      bool stop = false;
      for (int t = blockIdx.x; t < total && !stop; t += gridDim.x) {
        const TileCoord tc = decode_tile256(g, t, BN);
        const CUtensorMap* mA = tc.problem ? &tA1 : &tA0;
        const CUtensorMap* mB = tc.problem ? &tB1 : &tB0;
        const OpOff oA = tc.problem ? g.a1 : g.a0;
        const OpOff oB = tc.problem ? g.b1 : g.b0;
        for (int i = 0; i < tc.nkb; ++i, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1;
          if (it >= STAGES && !mbar_wait(&empty[s], ph ^ 1, abort_flag)) {
            stop = true;
            break;
          }
          uint8_t* st = smem + s * S::STAGE;
          mbar_arrive_expect_tx(&full[s], S::STAGE);
          const int k0 = (tc.kb_begin + i) * 64;
          load_operand<true, 2>(st, mA, &full[s], 256, tc.m0 + oA.mn, k0 + oA.k, tc.z);
          load_operand<true, 2>(st + S::A_BYTES, mB, &full[s], BN, tc.n0 + oB.mn, k0 + oB.k, tc.z);
        }
      }
      if (*abort_flag) {
        for (int j = max(0, it - STAGES); j < it; ++j) {
          volatile int never = 0;
          mbar_wait(&full[j % STAGES], (j / STAGES) & 1, &never);
        }
      }
    }
  } else if (warp == 1) {
    if (elect_one()) {
      constexpr uint32_t id = make_idesc(128, BN, 1, true, true);
      const uint32_t sbase = smem_u32(smem);
      int it = 0, j = 0;
      bool stop = false;
      for (int t = blockIdx.x; t < total && !stop; t += gridDim.x, ++j) {
        const TileCoord tc = decode_tile256(g, t, BN);
        if (j > 0 && !mbar_wait(tmem_empty, (j - 1) & 1, abort_flag)) break;
        tc_fence_after();
        for (int i = 0; i < tc.nkb; ++i, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1;
          if (!mbar_wait(&full[s], ph, abort_flag)) {
            stop = true;
            break;
          }
          tc_fence_after();
          const uint32_t a = sbase + s * S::STAGE;
          const uint32_t b = a + S::A_BYTES;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint32_t acc = (i > 0 || kk > 0) ? 1u : 0u;
            const uint64_t db = operand_desc<true, 2>(b, kk);
            // rows 0-127 are the first two 64-row boxes of A, rows 128-255 the next two
            mma_f16(tmem_base, operand_desc<true, 2>(a, kk), db, id, acc);
            mma_f16(tmem_base + BN, operand_desc<true, 2>(a + S::A_BYTES / 2, kk), db, id, acc);
          }
          mma_commit(&empty[s]);
        }
        mma_commit(tmem_full);
      }
      if (*abort_flag) {
        volatile int never = 0;
        mma_commit(drain);
        mbar_wait(drain, 0, &never);
      }
    }
  } else {
    const int q = warp & 3;
    const int sub = (warp - 2) >> 2;  // accumulator (row half) of this warp
    const int row = q * 32 + static_cast<int>(lane_id());
    int j = 0;
    for (int t = blockIdx.x; t < total; t += gridDim.x, ++j) {
      const TileCoord tc = decode_tile256(g, t, BN);
      const bool ready = __all_sync(0xffffffffu, mbar_wait(tmem_full, j & 1, abort_flag));
      if (!ready) break;
      tc_fence_after();
      EpiCtx c;
      c.taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(sub * BN);
      c.row = row;
      c.m = tc.m0 + sub * 128 + row;
      c.n0 = tc.n0;
      c.z = tc.z;
      c.split = tc.split;
      c.problem = tc.problem;
      c.part = 0;
      c.nparts = 1;
      if (tc.nkb > 0) epi.template run<BN, 0>(c);
      tc_fence_before();
      __syncwarp();
      if (lane_id() == 0) mbar_arrive(tmem_empty);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (threadIdx.x == 0 && *abort_flag) set_status(status, kStatusTimeout);
  if (warp == 1) tmem_dealloc(tmem_base, S::TMEM_COLS);
}

template <int BN, int STAGES, class Epi>
cudaError_t launch_wgrad(const CUtensorMap& a0, const CUtensorMap& b0, const CUtensorMap& a1, const CUtensorMap& b1,
                         const TcGeom& g, const Epi& epi, unsigned* status, cudaStream_t st) {
  using S = WgShape<BN, STAGES>;
  auto kern = wgrad_kernel<BN, STAGES, Epi>;
  // one CTA per SM: the accumulators may take all 512 TMEM columns
  constexpr int kSmem = S::SMEM > 116 * 1024 ? S::SMEM : 116 * 1024;
  static OncePerDevice configured;
  const int set = configured.run(current_device(), [&] {
    return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
  });
  if (set != 0) return static_cast<cudaError_t>(set);
  const long long total = static_cast<long long>(g.m_tiles0 + g.m_tiles1) * g.n_tiles * g.batches * g.splits;
  if (total <= 0) return cudaSuccess;
  if (total > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  const int grid = static_cast<int>(std::min<long long>(total, sm_count()));
  kern<<<grid, 320, kSmem, st>>>(a0, b0, a1, b1, g, epi, status);
  return cudaGetLastError();
}

}  // namespace ttt
