// Newton-Schulz orthogonalisation (the Muon step of the LaCT analysis, "Nonlinear
// memory complements local attention") of a batch of m x n matrices (m <= n), all
// iterations in one launch:
//   for it in iters:  S = X X^T;  T = b S + c S S;  X <- a X + T X
// The fp32 terms b S and a X are added in the epilogues at full precision; the
// producer prefetches the S or X tile they need into shared memory with TMA while
// the tile's MMAs run, so the epilogue does not wait on global memory.
// One thread-block cluster of CS CTAs owns one matrix.  Each step is cut into
// 128 x 128 output tiles dealt round-robin to the cluster's CTAs and computed on
// the tf32 tensor cores (fp32 storage, fp32 accumulation in TMEM, two accumulator
// buffers so one tile's epilogue overlaps the next tile's MMAs); a cluster barrier
// separates the steps (every step reads what the previous one wrote).
// X is kept twice, as X [m][n] and X^T [n][m], so every operand is K-major.
//
// Stores: S and T (symmetric) are written transposed into their mirrored tiles and
// X^T column-wise, so a warp's lanes (consecutive rows) store consecutive addresses;
// X' rows go back into the prefetch buffer and leave by TMA.
// Memory ordering across a step boundary: epilogue threads write with generic
// stores and wait for their TMA stores to complete, issue fence.proxy.async.global
// and arrive on the cluster barrier with release semantics; after the acquiring
// wait the producer fences again before its TMA loads read those values.
#pragma once
#include "epilogues.cuh"

namespace ttt {

struct NsGeom {
  int m, n, iters;
  float a, b, c;
  // fp32 buffers, per matrix strides m*n (X, XT, X2, XT2) and m*m (S, T)
  float *X, *XT, *X2, *XT2, *S, *T;
};

constexpr int kNsStages = 4;
constexpr int kNsStage = 2 * 128 * 128;  // A + B tile of 32 fp32 (128 B) per row
constexpr int kNsEbuf = 4 * 128 * 128;   // one 128 x 128 fp32 epilogue operand tile (4 boxes of 32 cols)
constexpr int kNsSmem = 1024 + kNsStages * kNsStage + kNsEbuf + 256;

__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;\n" ::: "memory");
}
__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// The three steps of one iteration as tile problems.
struct NsStep {
  const CUtensorMap* A;
  const CUtensorMap* B;
  int tiles_n;  // output tiles per tile row
  int tiles;    // output tiles in all
  int kblocks;  // K / 32
};

__device__ __forceinline__ NsStep ns_step(int step, int it, const NsGeom& g, const CUtensorMap* mX,
                                          const CUtensorMap* mXT, const CUtensorMap* mX2, const CUtensorMap* mXT2,
                                          const CUtensorMap* mS, const CUtensorMap* mT) {
  const bool odd = it & 1;
  const CUtensorMap* cx = odd ? mX2 : mX;
  const CUtensorMap* cxt = odd ? mXT2 : mXT;
  const int tm = g.m / 128, tn = g.n / 128;
  NsStep s;
  if (step == 0) {  // S = X X^T   (A = X rows, B = X rows, K = n)
    s.A = cx;
    s.B = cx;
    s.tiles_n = tm;
    s.tiles = tm * tm;
    s.kblocks = g.n / 32;
  } else if (step == 1) {  // S S  (S symmetric: its rows are the K-major B operand), K = m
    s.A = mS;
    s.B = mS;
    s.tiles_n = tm;
    s.tiles = tm * tm;
    s.kblocks = g.m / 32;
  } else {  // T X  (A = T rows, B = X^T rows [n][m]), K = m
    s.A = mT;
    s.B = cxt;
    s.tiles_n = tn;
    s.tiles = tm * tn;
    s.kblocks = g.m / 32;
  }
  return s;
}

template <int CS>
__global__ void __launch_bounds__(192, 1)
    ns_fused_kernel(const __grid_constant__ CUtensorMap mX, const __grid_constant__ CUtensorMap mXT,
                    const __grid_constant__ CUtensorMap mX2, const __grid_constant__ CUtensorMap mXT2,
                    const __grid_constant__ CUtensorMap mS, const __grid_constant__ CUtensorMap mT,
                    const __grid_constant__ CUtensorMap sX, const __grid_constant__ CUtensorMap sX2, const NsGeom g,
                    unsigned* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* ebuf = smem + kNsStages * kNsStage;
  uint64_t* full = reinterpret_cast<uint64_t*>(ebuf + kNsEbuf);
  uint64_t* empty = full + kNsStages;
  uint64_t* tmem_full = empty + kNsStages;  // [2]: accumulator buffer b holds tile j when j % 2 == b
  uint64_t* tmem_empty = tmem_full + 2;     // [2]
  uint64_t* drain = tmem_empty + 2;
  uint64_t* efull = drain + 1;   // epilogue operand tile landed
  uint64_t* eempty = efull + 1;  // epilogue done with it
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(eempty + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = static_cast<int>(lane_id());
  const int rank = static_cast<int>(cluster_ctarank());
  const int zk = blockIdx.x / CS;  // matrix of this cluster
  const int64_t mn = int64_t(g.m) * g.n, mm = int64_t(g.m) * g.m;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kNsStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(&tmem_full[0], 1);
    mbar_init(&tmem_full[1], 1);
    mbar_init(&tmem_empty[0], 4);
    mbar_init(&tmem_empty[1], 4);
    mbar_init(drain, 1);
    mbar_init(efull, 1);
    mbar_init(eempty, 4);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  int it_ring = 0;  // producer / MMA position in the smem ring (lane 0 of warps 0 and 1)
  int j_tile = 0;   // tiles this CTA has computed (TMEM phases)
  int e_use = 0;    // epilogue operand tiles loaded (producer) / consumed (epilogue)
  for (int it = 0; it < g.iters; ++it) {
    for (int step = 0; step < 3; ++step) {
      const NsStep sp = ns_step(step, it, g, &mX, &mXT, &mX2, &mXT2, &mS, &mT);
      if (warp == 0) {
        if (lane == 0 && !*abort_flag) {
          fence_proxy_async_global();  // the previous step's generic stores -> these TMA loads
          const CUtensorMap* eop = step == 1 ? &mS : ((it & 1) ? &mX2 : &mX);  // S for T, X for X'
          for (int t = rank; t < sp.tiles && !*abort_flag; t += CS) {
            const int r0 = (t / sp.tiles_n) * 128, c0 = (t % sp.tiles_n) * 128;
            for (int kb = 0; kb < sp.kblocks; ++kb, ++it_ring) {
              const int s = it_ring % kNsStages;
              const uint32_t ph = (it_ring / kNsStages) & 1;
              if (it_ring >= kNsStages && !mbar_wait(&empty[s], ph ^ 1, abort_flag)) break;
              uint8_t* st = smem + s * kNsStage;
              mbar_arrive_expect_tx(&full[s], kNsStage);
              tma_load_3d(st, sp.A, &full[s], kb * 32, r0, zk);
              tma_load_3d(st + 128 * 128, sp.B, &full[s], kb * 32, c0, zk);
            }
            // after the tile's operands (so waiting for the previous epilogue never holds
            // them back): the fp32 tile its epilogue adds, S for T = b S + c S S, X for a X + T X
            if (step > 0 && !*abort_flag) {
              if (e_use > 0 && !mbar_wait(eempty, (e_use - 1) & 1, abort_flag)) break;
              mbar_arrive_expect_tx(efull, kNsEbuf);
              for (int bx = 0; bx < 4; ++bx) tma_load_3d(ebuf + bx * 128 * 128, eop, efull, c0 + 32 * bx, r0, zk);
              ++e_use;
            }
          }
        }
        __syncwarp();
      } else if (warp == 1) {
        if (lane == 0 && !*abort_flag) {
          constexpr uint32_t id = make_idesc(128, 128, 2, false, false);
          const uint32_t sbase = smem_u32(smem);
          for (int t = rank; t < sp.tiles && !*abort_flag; t += CS) {
            const int buf = j_tile & 1;
            // buffer `buf` last held tile j_tile - 2: its epilogue must have drained it
            if (j_tile >= 2 && !mbar_wait(&tmem_empty[buf], ((j_tile - 2) >> 1) & 1, abort_flag)) break;
            tc_fence_after();
            const uint32_t dacc = tmem_base + static_cast<uint32_t>(buf * 128);
            for (int kb = 0; kb < sp.kblocks; ++kb, ++it_ring) {
              const int s = it_ring % kNsStages;
              const uint32_t ph = (it_ring / kNsStages) & 1;
              if (!mbar_wait(&full[s], ph, abort_flag)) break;
              tc_fence_after();
              const uint32_t a = sbase + s * kNsStage;
              const uint32_t b = a + 128 * 128;
#pragma unroll
              for (int kk = 0; kk < 4; ++kk)
                mma_tf32(dacc, make_sdesc_sw128(a + kk * 32, 16, 1024), make_sdesc_sw128(b + kk * 32, 16, 1024), id,
                         (kb > 0 || kk > 0) ? 1u : 0u);
              mma_commit(&empty[s]);
            }
            mma_commit(&tmem_full[buf]);
            ++j_tile;
          }
        }
        __syncwarp();
      } else {
        const int q = warp & 3;
        const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
        for (int t = rank; t < sp.tiles; t += CS) {
          const int buf = j_tile & 1;
          const bool ready = __all_sync(0xffffffffu, mbar_wait(&tmem_full[buf], (j_tile >> 1) & 1, abort_flag));
          if (!ready) break;
          tc_fence_after();
          const int r0 = (t / sp.tiles_n) * 128, c0 = (t % sp.tiles_n) * 128;
          const int row = r0 + q * 32 + lane;
          const bool odd = it & 1;
          float* nxt = odd ? g.XT : g.XT2;  // X^T of the next iteration
          const uint32_t tacc = taddr + static_cast<uint32_t>(buf * 128);
          const int lrow = q * 32 + lane;  // row inside the tile (and the prefetched box)
          if (step > 0) {
            const bool landed = __all_sync(0xffffffffu, mbar_wait(efull, e_use & 1, abort_flag));
            if (!landed) break;
          }
#pragma unroll 1
          for (int cc = 0; cc < 128; cc += 32) {
            float v[32];
            tmem_ld32(tacc + cc, v);
            if (step == 0) {
              // S is symmetric: write the tile transposed, into the mirrored position, so that
              // the warp's 32 lanes (consecutive rows) store consecutive addresses
              float* colS = g.S + zk * mm + int64_t(c0 + cc) * g.m + row;
#pragma unroll
              for (int i = 0; i < 32; ++i) colS[int64_t(i) * g.m] = v[i];
            } else {
              // the prefetched fp32 tile: box cc/32, row lrow, 16-byte chunk k at k ^ (lrow & 7)
              const float4* box = reinterpret_cast<const float4*>(ebuf + (cc / 32) * 128 * 128 + lrow * 128);
              float e[32];
#pragma unroll
              for (int k = 0; k < 8; ++k) {
                const float4 f = box[k ^ (lrow & 7)];
                e[4 * k] = f.x;
                e[4 * k + 1] = f.y;
                e[4 * k + 2] = f.z;
                e[4 * k + 3] = f.w;
              }
              if (step == 1) {
                // T = b S + c S S is symmetric too: transposed, mirrored store as for S
                float* colT = g.T + zk * mm + int64_t(c0 + cc) * g.m + row;
#pragma unroll
                for (int i = 0; i < 32; ++i) colT[int64_t(i) * g.m] = g.b * e[i] + g.c * v[i];
              } else {
#pragma unroll
                for (int i = 0; i < 32; ++i) v[i] = g.a * e[i] + v[i];
                // X' rows go back into the prefetched tile's place in shared memory (same
                // swizzled layout) and leave as TMA stores after the last chunk
                float4* wbox = reinterpret_cast<float4*>(ebuf + (cc / 32) * 128 * 128 + lrow * 128);
#pragma unroll
                for (int k = 0; k < 8; ++k)
                  wbox[k ^ (lrow & 7)] = make_float4(v[4 * k], v[4 * k + 1], v[4 * k + 2], v[4 * k + 3]);
                float* colT = nxt + zk * mn + int64_t(c0 + cc) * g.m + row;
#pragma unroll
                for (int i = 0; i < 32; ++i) colT[int64_t(i) * g.m] = v[i];  // coalesced across the warp
              }
            }
          }
          if (step == 2) {
            // this warp's 32 rows of X' (4 boxes of 32 columns) from shared memory to X;
            // the prefetch buffer is released once the stores have read it
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              const CUtensorMap* dst = (it & 1) ? &sX : &sX2;
              for (int bx = 0; bx < 4; ++bx)
                tma_store_3d(dst, ebuf + bx * 128 * 128 + q * 32 * 128, c0 + 32 * bx, r0 + q * 32, zk);
              bulk_commit();
              bulk_wait_read0();
            }
          }
          if (step > 0) {
            __syncwarp();
            if (lane == 0) mbar_arrive(eempty);
            ++e_use;
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&tmem_empty[buf]);
          ++j_tile;
        }
        if (lane == 0) bulk_wait0();  // the X' stores are complete
        fence_proxy_async_global();  // these stores -> the next step's TMA loads
      }
      cluster_sync_all();
    }
  }

  if (warp == 1 && lane == 0 && *abort_flag) {
    volatile int never = 0;
    mma_commit(drain);
    mbar_wait(drain, 0, &never);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (threadIdx.x == 0 && *abort_flag) set_status(status, kStatusTimeout);
  if (warp == 1) tmem_dealloc(tmem_base, 256);
}

// X: Newton-Schulz input (normalised) in g.X / g.XT; result in (g.iters odd ? X2 : X).
template <int CS>
cudaError_t launch_ns_fused_cs(int nmat, const NsGeom& g, unsigned* status, cudaStream_t st) {
  CUtensorMap mX, mXT, mX2, mXT2, mS, mT, sX, sX2;
  const int m = g.m, n = g.n;
  if (!make_tmap(&mX, g.X, 4, n, m, nmat, n, int64_t(m) * n, 128) ||
      !make_tmap(&mXT, g.XT, 4, m, n, nmat, m, int64_t(m) * n, 128) ||
      !make_tmap(&mX2, g.X2, 4, n, m, nmat, n, int64_t(m) * n, 128) ||
      !make_tmap(&mXT2, g.XT2, 4, m, n, nmat, m, int64_t(m) * n, 128) ||
      !make_tmap(&mS, g.S, 4, m, m, nmat, m, int64_t(m) * m, 128) ||
      !make_tmap(&mT, g.T, 4, m, m, nmat, m, int64_t(m) * m, 128) ||
      // stores of one epilogue warp's 32 rows of X'
      !make_tmap(&sX, g.X, 4, n, m, nmat, n, int64_t(m) * n, 32) ||
      !make_tmap(&sX2, g.X2, 4, n, m, nmat, n, int64_t(m) * n, 32))
    return cudaErrorInvalidValue;
  auto kern = ns_fused_kernel<CS>;
  static OncePerDevice configured;
  const int set = configured.run(current_device(), [&] {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kNsSmem);
    if (e == cudaSuccess && CS > 8) e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    return e;
  });
  if (set != 0) return static_cast<cudaError_t>(set);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(nmat * CS, 1, 1);
  cfg.blockDim = dim3(192, 1, 1);
  cfg.dynamicSmemBytes = kNsSmem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = CS;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, mX, mXT, mX2, mXT2, mS, mT, sX, sX2, g, status);
}

// Whether a cluster of CS CTAs of this kernel can be resident at all on this device.
template <int CS>
bool ns_cluster_fits() {
  static IntPerDevice fit;
  return fit.get(current_device(), [] {
    auto kern = ns_fused_kernel<CS>;
    int fits = 0;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kNsSmem) == cudaSuccess &&
        (CS <= 8 || cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) == cudaSuccess)) {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(CS, 1, 1);
      cfg.blockDim = dim3(192, 1, 1);
      cfg.dynamicSmemBytes = kNsSmem;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = CS;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) == cudaSuccess && n > 0) fits = 1;
    }
    cudaGetLastError();  // a refused query leaves no sticky error behind
    return fits;
  }) == 1;
}

// Cluster size: one CTA per 128 x 128 tile of the largest step (T' X), at most 16
// (16 needs the non-portable cluster size; it fits a GPC of a B200).
inline cudaError_t launch_ns_fused(int nmat, const NsGeom& g, unsigned* status, cudaStream_t st) {
  if (g.m % 128 || g.n % 128 || g.m > g.n || nmat <= 0) return cudaErrorInvalidValue;
  const int tiles = (g.m / 128) * (g.n / 128);
  if (tiles >= 16 && ns_cluster_fits<16>()) return launch_ns_fused_cs<16>(nmat, g, status, st);
  if (tiles >= 8) return launch_ns_fused_cs<8>(nmat, g, status, st);
  if (tiles >= 4) return launch_ns_fused_cs<4>(nmat, g, status, st);
  if (tiles >= 2) return launch_ns_fused_cs<2>(nmat, g, status, st);
  return launch_ns_fused_cs<1>(nmat, g, status, st);
}

}  // namespace ttt
