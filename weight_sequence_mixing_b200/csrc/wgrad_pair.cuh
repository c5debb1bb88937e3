// Weight-gradient token reductions on CTA pairs (tcgen05 cta_group::2):
//   D[rows, cols] = sum_t A[t, rows] * B[t, cols]
// the same GEMMs as wgrad_kernel (wgrad.cuh; G2^T = H'^T V, [G1; G3] = dZ13^T K ...,
// LaCT analysis, "Nonlinear memory complements local attention"), with 512 x BN
// output tiles computed by the two CTAs of a cluster.
//
// CTA r of the pair stages rows [256 r, 256 r + 256) of the tile's A rows (two
// 128-row halves) and columns [r BN/2, (r+1) BN/2) of B.  The even CTA issues, per
// 16-token step, two M = 256 pair MMAs that share B: the first takes each CTA's
// first 128 rows, the second each CTA's second 128 rows, so CTA r accumulates rows
// 256 r + [0, 128) at TMEM columns [0, BN) and 256 r + [128, 256) at [BN, 2 BN),
// every column of the tile in both.  Per 64-token k-block a CTA brings in 32 KB of A
// and BN x 64 B of B for 2 x 128 x BN x 64 multiply-adds: a third fewer bytes than
// the single-CTA 256-row tile.
//
// Barriers and teardown follow token_pair.cuh: full[s] in the leader counts both
// CTAs' TMA bytes, the leader's commits arrive on both CTAs' empty[s] and tmem_full,
// and every epilogue warp of both CTAs arrives on the leader's tmem_empty.
#pragma once
#include "tc_gemm.cuh"

namespace ttt {

template <int BN, int STAGES>
struct WgPairShape {
  static constexpr int A_BYTES = 256 * 128;     // this CTA's 256 rows x 64 tokens, bf16
  static constexpr int B_BYTES = BN / 2 * 128;  // this CTA's BN/2 columns x 64 tokens
  static constexpr int STAGE = A_BYTES + B_BYTES;
  static constexpr int SMEM = 1024 + STAGES * STAGE + 256;
  static_assert(BN == 128 || BN == 256, "each CTA's B half must be whole 64-column boxes");
  static_assert(SMEM <= 227 * 1024, "shared memory");
};

// Pair tile coordinates (N-tile fastest), 512-row M tiles.
__device__ __forceinline__ TileCoord decode_tile512(const TcGeom& g, int t, int bn) {
  TileCoord c;
  const int mtiles = g.m_tiles0 + g.m_tiles1;
  const int nt = t % g.n_tiles;
  int r = t / g.n_tiles;
  const int mt = r % mtiles;
  r /= mtiles;
  c.z = r % g.batches;
  c.split = r / g.batches;
  c.problem = mt >= g.m_tiles0 ? 1 : 0;
  c.m0 = (c.problem ? mt - g.m_tiles0 : mt) * 512;
  c.n0 = nt * bn;
  c.kb_begin = c.split * g.kb_per_split;
  c.nkb = max(0, min(g.kblocks, c.kb_begin + g.kb_per_split) - c.kb_begin);
  return c;
}

// MN-major operand rows [mn0, mn0 + rows) x 64 tokens as 64-element boxes, bytes
// counted on the leader's barrier `bar` (shared::cluster address)
__device__ __forceinline__ void load_mn_pair(uint8_t* dst, const CUtensorMap* m, uint32_t bar, int rows, int mn0,
                                             int k0, int z) {
  for (int j = 0; j < rows / 64; ++j) tma_load_3d_pair(dst + j * 64 * 128, m, bar, mn0 + j * 64, k0, z);
}

template <int BN, int STAGES, class Epi>
__global__ void __launch_bounds__(320, 1)
    wgrad_pair_kernel(const __grid_constant__ CUtensorMap tA0, const __grid_constant__ CUtensorMap tB0,
                      const __grid_constant__ CUtensorMap tA1, const __grid_constant__ CUtensorMap tB1,
                      const TcGeom g, const Epi epi, unsigned* status) {
  using S = WgPairShape<BN, STAGES>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * S::STAGE);
  uint64_t* empty = full + STAGES;
  uint64_t* tmem_full = empty + STAGES;
  uint64_t* tmem_empty = tmem_full + 1;
  uint64_t* drain = tmem_empty + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const uint32_t rank = cluster_rank() & 1u;
  const bool leader = rank == 0;
  const int warp = threadIdx.x >> 5;
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const int total = (g.m_tiles0 + g.m_tiles1) * g.n_tiles * g.batches * g.splits;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(tmem_full, 1);
    mbar_init(tmem_empty, 2 * 8);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, 512);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_barrier();
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
      const uint32_t full0 = mapa_shared(smem_u32(full), 0);
      int it = 0;
      bool stop = false;
      for (int t = pair; t < total && !stop; t += npairs) {
        const TileCoord tc = decode_tile512(g, t, BN);
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
          const uint32_t fb = full0 + static_cast<uint32_t>(s) * 8u;
          if (leader) mbar_arrive_expect_tx(&full[s], 2 * S::STAGE);
          const int k0 = (tc.kb_begin + i) * 64;
          load_mn_pair(st, mA, fb, 256, tc.m0 + static_cast<int>(rank) * 256 + oA.mn, k0 + oA.k, tc.z);
          load_mn_pair(st + S::A_BYTES, mB, fb, BN / 2, tc.n0 + static_cast<int>(rank) * (BN / 2) + oB.mn,
                       k0 + oB.k, tc.z);
        }
      }
      if (!*abort_flag) {
        for (int j = max(0, it - STAGES); j < it; ++j)
          if (!mbar_wait(&empty[j % STAGES], (j / STAGES) & 1, abort_flag)) break;
      }
      if (*abort_flag) {
        const unsigned long long t0 = global_ns();
        while (global_ns() - t0 < 1000000ull) {
        }
      }
    }
  } else if (warp == 1) {
    if (leader && elect_one()) {
      constexpr uint32_t id = make_idesc(256, BN, 1, true, true);
      const uint32_t sbase = smem_u32(smem);
      int it = 0, j = 0;
      bool stop = false;
      for (int t = pair; t < total && !stop; t += npairs, ++j) {
        const TileCoord tc = decode_tile512(g, t, BN);
        if (j > 0 && !mbar_wait_cluster(tmem_empty, (j - 1) & 1, abort_flag)) break;
        tc_fence_after();
        for (int i = 0; i < tc.nkb; ++i, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1;
          if (!mbar_wait_cluster(&full[s], ph, abort_flag)) {
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
            mma_f16_pair(tmem_base, operand_desc<true, 2>(a, kk), db, id, acc);
            mma_f16_pair(tmem_base + BN, operand_desc<true, 2>(a + S::A_BYTES / 2, kk), db, id, acc);
          }
          mma_commit_pair(&empty[s], 0x3);
        }
        if (!stop) mma_commit_pair(tmem_full, 0x3);
      }
      if (!stop && j > 0) mbar_wait_cluster(tmem_empty, (j - 1) & 1, abort_flag);
      if (*abort_flag) {
        volatile int never = 0;
        mma_commit_pair(drain, 0x1);
        mbar_wait(drain, 0, &never);
      }
    }
  } else {
    const int q = warp & 3;
    const int sub = (warp - 2) >> 2;  // accumulator (row half) of this warp
    const int row = q * 32 + static_cast<int>(lane_id());
    const uint32_t tmem_empty0 = mapa_shared(smem_u32(tmem_empty), 0);
    int j = 0;
    for (int t = pair; t < total; t += npairs, ++j) {
      const TileCoord tc = decode_tile512(g, t, BN);
      const bool ready = __all_sync(0xffffffffu, mbar_wait_cluster(tmem_full, j & 1, abort_flag));
      if (!ready) break;
      tc_fence_after();
      EpiCtx c;
      c.taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(sub * BN);
      c.row = row;
      c.m = tc.m0 + static_cast<int>(rank) * 256 + sub * 128 + row;
      c.n0 = tc.n0;
      c.z = tc.z;
      c.split = tc.split;
      c.problem = tc.problem;
      c.part = 0;
      c.nparts = 1;
      if (tc.nkb > 0) epi.template run<BN, 0>(c);
      tc_fence_before();
      __syncwarp();
      if (lane_id() == 0) mbar_arrive_cluster(tmem_empty0);
    }
  }

  __syncwarp();
  tc_fence_before();
  cluster_barrier();
  tc_fence_after();
  if (threadIdx.x == 0 && *abort_flag) set_status(status, kStatusTimeout);
  if (warp == 1) tmem_dealloc_pair(tmem_base, 512);
}

template <int BN, int STAGES, class Epi>
cudaLaunchConfig_t wgrad_pair_config(int pairs, cudaStream_t st, cudaLaunchAttribute* attr) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * pairs, 1, 1);
  cfg.blockDim = dim3(320, 1, 1);
  cfg.dynamicSmemBytes = WgPairShape<BN, STAGES>::SMEM;
  cfg.stream = st;
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cfg;
}

// CTA pairs of this instantiation that can be resident at once (0: use wgrad_kernel).
template <int BN, int STAGES, class Epi>
int wgrad_pair_capacity() {
  static IntPerDevice caps;
  return caps.get(current_device(), [] {
    auto kern = wgrad_pair_kernel<BN, STAGES, Epi>;
    int cap = 0;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, WgPairShape<BN, STAGES>::SMEM) ==
        cudaSuccess) {
      cudaLaunchAttribute attr[1];
      cudaLaunchConfig_t cfg = wgrad_pair_config<BN, STAGES, Epi>(1, nullptr, attr);
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) == cudaSuccess && n > 0) cap = n;
    }
    cudaGetLastError();
    return cap;
  });
}

// g.m_tiles0 / m_tiles1 count 512-row tiles.
template <int BN, int STAGES, class Epi>
cudaError_t launch_wgrad_pair(const CUtensorMap& a0, const CUtensorMap& b0, const CUtensorMap& a1,
                              const CUtensorMap& b1, const TcGeom& g, const Epi& epi, unsigned* status,
                              cudaStream_t st) {
  const int cap = wgrad_pair_capacity<BN, STAGES, Epi>();
  if (cap <= 0) return cudaErrorInvalidConfiguration;
  const long long total = static_cast<long long>(g.m_tiles0 + g.m_tiles1) * g.n_tiles * g.batches * g.splits;
  if (total <= 0) return cudaSuccess;
  if (total > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  const int pairs = static_cast<int>(std::min<long long>(total, cap));
  cudaLaunchAttribute attr[1];
  cudaLaunchConfig_t cfg = wgrad_pair_config<BN, STAGES, Epi>(pairs, st, attr);
  return cudaLaunchKernelEx(&cfg, wgrad_pair_kernel<BN, STAGES, Epi>, a0, b0, a1, b1, g, epi, status);
}

}  // namespace ttt
