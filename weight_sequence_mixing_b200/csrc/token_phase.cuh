// Token-phase kernel of the negative-dot-loss update (SwiGLU or GELU-MLP fast
// weights): for every 128-token x 128-hidden tile of a chunk it computes
//   P   = V W2[:, blk]                      128 TMEM columns (slot 256 or 384)
//   Z13 = X [W1_blk ; W3_blk]^T  (SwiGLU)    256 columns at 0   (MLP2: Z = X W1_blk^T, 128)
// and, in the epilogue, dL/dV_hat_t = -eta_t v_t pushed back through W2 and the
// gating (LaCT analysis, "Nonlinear memory complements local attention"):
//   dH = -eta_t P;  SwiGLU: H' = -eta_t SiLU(z1) z3, dZ3 = dH SiLU(z1), dZ1 = dH z3 SiLU'(z1)
//                   MLP2  : H' = -eta_t GELU(z),      dZ  = dH GELU'(z)
// H' [t][h] and dZ13 [t][2h] (blocks [dZ1 128 | dZ3 128]) / dZ [t][h] are written in bf16
// for the weight-gradient GEMMs; rows past the chunk get zeros (eta_t = 0 there).
//
// Schedule (persistent CTAs, one per SM; tiles visited hidden-block fastest):
//   warp 0 : TMA producer.  Per tile it streams the P phase (V and W2^T k-blocks),
//            then the Z phase (X and first-layer k-blocks) through a STAGES-deep ring.
//   warp 1 : MMA issuer.  A tile's P phase goes to the P slot its parity selects and
//            does not wait for TMEM: it overlaps the previous tile's epilogue.  Only
//            the Z phase waits until that epilogue has drained the accumulators.
//   warps 2-9 : epilogue.  Each warp owns 32 rows (its TMEM lane quarter) and two
//            32-column chunks; results go through a swizzled smem box and leave as
//            coalesced TMA bulk stores.
#pragma once
#include "epilogues.cuh"

namespace ttt {

struct TokGeom {
  int m_tiles, n_tiles, batches;  // Cp/128, h/128, Z
  int kblocks;                    // d / 64
  int x_off, v_off;               // token offsets of the keys and values maps
  int rows_valid;                 // tokens in the chunk
  int rows_alloc;                 // rows of the activation buffers (stores stop there)
  int t0;                         // chunk's first token (eta index)
  const float* eta;
  int64_t eta_zs;
  float eta_scalar;
};

template <bool SWIGLU>
struct TokShape {
  static constexpr int A_BYTES = 128 * 128;  // 128 rows x 64 bf16
  static constexpr int BZ_ROWS = SWIGLU ? 256 : 128;
  static constexpr int BZ_BYTES = BZ_ROWS * 128;
  static constexpr int BP_BYTES = 128 * 128;
  static constexpr int Z_STAGE = A_BYTES + BZ_BYTES;
  static constexpr int P_STAGE = A_BYTES + BP_BYTES;
  static constexpr int SLOT = Z_STAGE > P_STAGE ? Z_STAGE : P_STAGE;
  static constexpr int STAGES = SWIGLU ? 3 : 4;
  static constexpr int NOUT = SWIGLU ? 3 : 2;
  static constexpr int EW = 8;
  static constexpr int STG_BYTES = 2048;  // one [32 rows][32 bf16] output box
  static constexpr int STG_WARP = NOUT * STG_BYTES;
  static constexpr int SMEM = 1024 + STAGES * SLOT + EW * STG_WARP + 256;
  static constexpr int ZN = SWIGLU ? 256 : 128;
  static_assert(SMEM <= 227 * 1024, "shared memory");
};

// 32 floats of one row into a [32 rows][64 B] box with the 64-byte TMA swizzle
// (16-byte chunk k of row r sits at chunk k ^ ((r >> 1) & 3)).
__device__ __forceinline__ void stage_row_sw64(uint8_t* box, int r, const float (&v)[32]) {
  uint4* rowp = reinterpret_cast<uint4*>(box + r * 64);
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    uint4 u;
    u.x = pack_bf16x2(v[8 * k + 0], v[8 * k + 1]);
    u.y = pack_bf16x2(v[8 * k + 2], v[8 * k + 3]);
    u.z = pack_bf16x2(v[8 * k + 4], v[8 * k + 5]);
    u.w = pack_bf16x2(v[8 * k + 6], v[8 * k + 7]);
    rowp[k ^ ((r >> 1) & 3)] = u;
  }
}

// N floats of one row as N/2 bf16 pairs (the order stage_row_sw64 stores them in)
template <int N>
__device__ __forceinline__ void pack_row_bf16(const float (&v)[N], uint32_t (&w)[N / 2]) {
#pragma unroll
  for (int i = 0; i < N / 2; ++i) w[i] = pack_bf16x2(v[2 * i], v[2 * i + 1]);
}

// 8 packed bf16 pairs (16 columns, 32 bytes) of one row into a [32 rows][32 B] box with
// the 32-byte TMA swizzle (16-byte chunk k of row r sits at chunk k ^ ((r >> 2) & 1))
__device__ __forceinline__ void stage_packed_sw32(uint8_t* box, int r, const uint32_t (&w)[8]) {
  uint4* rowp = reinterpret_cast<uint4*>(box + r * 32);
#pragma unroll
  for (int k = 0; k < 2; ++k) rowp[k ^ ((r >> 2) & 1)] = make_uint4(w[4 * k], w[4 * k + 1], w[4 * k + 2], w[4 * k + 3]);
}

// 16 packed bf16 pairs of one row into a [32 rows][64 B] box, 64-byte TMA swizzle
__device__ __forceinline__ void stage_packed_sw64(uint8_t* box, int r, const uint32_t (&w)[16]) {
  uint4* rowp = reinterpret_cast<uint4*>(box + r * 64);
#pragma unroll
  for (int k = 0; k < 4; ++k) rowp[k ^ ((r >> 1) & 3)] = make_uint4(w[4 * k], w[4 * k + 1], w[4 * k + 2], w[4 * k + 3]);
}

// Epilogue math of N columns of one row: z1 (and z3) and p from TMEM, e = eta_t.
template <bool SWIGLU, int N = 32>
__device__ __forceinline__ void token_dot_math(float e, const uint32_t (&r1)[N], const uint32_t (&r3)[N],
                                               const uint32_t (&rp)[N], float (&hv)[N], float (&d1)[N],
                                               float (&d3)[N]) {
  if constexpr (SWIGLU) {
    // pairs of columns with the paired fp32 instructions:
    //   s = SiLU gate sigma(z1) = (1 + tanh(z1/2))/2, a = z1 s, dh = -eta p
    //   H' = -eta a z3, dZ3 = dh a, dZ1 = dh z3 s (1 + z1 (1 - s))
    const float2 ne = make_float2(-e, -e), half = make_float2(0.5f, 0.5f), one = make_float2(1.0f, 1.0f),
                 mone = make_float2(-1.0f, -1.0f);
#pragma unroll
    for (int i = 0; i < N; i += 2) {
      const float2 z1 = make_float2(__uint_as_float(r1[i]), __uint_as_float(r1[i + 1]));
      const float2 z3 = make_float2(__uint_as_float(r3[i]), __uint_as_float(r3[i + 1]));
      const float2 p = make_float2(__uint_as_float(rp[i]), __uint_as_float(rp[i + 1]));
      const float2 hz = mul2(half, z1);
      const float2 sg = fma2(half, make_float2(tanh_approx(hz.x), tanh_approx(hz.y)), half);
      const float2 a = mul2(z1, sg);
      const float2 dh = mul2(ne, p);
      const float2 h = mul2(mul2(ne, a), z3);
      const float2 g3 = mul2(dh, a);
      const float2 u = fma2(z1, fma2(sg, mone, one), one);
      const float2 g1 = mul2(mul2(dh, z3), mul2(sg, u));
      hv[i] = h.x;
      hv[i + 1] = h.y;
      d3[i] = g3.x;
      d3[i + 1] = g3.y;
      d1[i] = g1.x;
      d1[i + 1] = g1.y;
    }
  } else {
#pragma unroll
    for (int i = 0; i < N; ++i) {
      const float z1 = __uint_as_float(r1[i]);
      const float dh = -e * __uint_as_float(rp[i]);
      float gz, gpz;
      gelu_and_grad(z1, gz, gpz);
      hv[i] = -e * gz;
      d1[i] = dh * gpz;
      d3[i] = 0.0f;
    }
  }
}

template <bool SWIGLU>
__global__ void __launch_bounds__(64 + 32 * TokShape<SWIGLU>::EW, 1)
    token_dot_kernel(const __grid_constant__ CUtensorMap tX, const __grid_constant__ CUtensorMap tFirst,
                     const __grid_constant__ CUtensorMap tV, const __grid_constant__ CUtensorMap tW2T,
                     const __grid_constant__ CUtensorMap tHp, const __grid_constant__ CUtensorMap tDZ,
                     const TokGeom g, unsigned* status) {
  using S = TokShape<SWIGLU>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stg = smem + S::STAGES * S::SLOT;
  uint64_t* full = reinterpret_cast<uint64_t*>(stg + S::EW * S::STG_WARP);
  uint64_t* empty = full + S::STAGES;
  uint64_t* tmem_full = empty + S::STAGES;
  uint64_t* tmem_empty = tmem_full + 1;
  uint64_t* drain = tmem_empty + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = static_cast<int>(lane_id());
  const int total = g.m_tiles * g.n_tiles * g.batches;
  const int KB = g.kblocks;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(tmem_full, 1);
    mbar_init(tmem_empty, S::EW);
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
      tma_prefetch_desc(&tFirst);
      tma_prefetch_desc(&tV);
      tma_prefetch_desc(&tW2T);
      int it = 0;
      bool stop = false;
      for (int t = blockIdx.x; t < total && !stop; t += gridDim.x) {
        const int nt = t % g.n_tiles;
        const int mt = (t / g.n_tiles) % g.m_tiles;
        const int z = t / (g.n_tiles * g.m_tiles);
        const int m0 = mt * 128;
        for (int phase = 0; phase < 2 && !stop; ++phase) {
          for (int kb = 0; kb < KB; ++kb, ++it) {
            const int s = it % S::STAGES;
            const uint32_t ph = (it / S::STAGES) & 1;
            if (it >= S::STAGES && !mbar_wait(&empty[s], ph ^ 1, abort_flag)) {
              stop = true;
              break;
            }
            uint8_t* st = smem + s * S::SLOT;
            if (phase == 0) {
              mbar_arrive_expect_tx(&full[s], S::P_STAGE);
              tma_load_3d(st, &tV, &full[s], kb * 64, m0 + g.v_off, z);
              tma_load_3d(st + S::A_BYTES, &tW2T, &full[s], kb * 64, nt * 128, z);
            } else {
              mbar_arrive_expect_tx(&full[s], S::Z_STAGE);
              tma_load_3d(st, &tX, &full[s], kb * 64, m0 + g.x_off, z);
              tma_load_3d(st + S::A_BYTES, &tFirst, &full[s], kb * 64, nt * S::BZ_ROWS, z);
            }
          }
        }
      }
      if (*abort_flag) {
        for (int j = max(0, it - S::STAGES); j < it; ++j) {
          volatile int never = 0;
          mbar_wait(&full[j % S::STAGES], (j / S::STAGES) & 1, &never);
        }
      }
    }
  } else if (warp == 1) {
    if (elect_one()) {
      constexpr uint32_t idP = make_idesc(128, 128, 1, false, false);
      constexpr uint32_t idZ = make_idesc(128, S::ZN, 1, false, false);
      const uint32_t sbase = smem_u32(smem);
      int it = 0, j = 0;
      bool stop = false;
      for (int t = blockIdx.x; t < total && !stop; t += gridDim.x, ++j) {
        const uint32_t pcol = (j & 1) ? 384u : 256u;
        for (int phase = 0; phase < 2 && !stop; ++phase) {
          if (phase == 1) {
            // the previous tile's epilogue must have drained Z (and its P slot)
            if (j > 0 && !mbar_wait(tmem_empty, (j - 1) & 1, abort_flag)) {
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
            if (!mbar_wait(&full[s], ph, abort_flag)) {
              stop = true;
              break;
            }
            tc_fence_after();
            const uint32_t a = sbase + s * S::SLOT;
            const uint32_t b = a + S::A_BYTES;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_f16(tmem_base + dcol, make_sdesc_sw128(a + kk * 32, 16, 1024), make_sdesc_sw128(b + kk * 32, 16, 1024),
                      id, (kb > 0 || kk > 0) ? 1u : 0u);
            mma_commit(&empty[s]);
          }
        }
        if (!stop) mma_commit(tmem_full);
      }
      if (*abort_flag) {
        volatile int never = 0;
        mma_commit(drain);
        mbar_wait(drain, 0, &never);
      }
    }
  } else {
    const int ew = warp - 2;
    const int q = warp & 3;
    const int part = ew >> 2;
    uint8_t* my = stg + ew * S::STG_WARP;
    const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
    int j = 0;
    for (int t = blockIdx.x; t < total; t += gridDim.x, ++j) {
      const int nt = t % g.n_tiles;
      const int mt = (t / g.n_tiles) % g.m_tiles;
      const int z = t / (g.n_tiles * g.m_tiles);
      const int m0 = mt * 128;
      const bool ready = __all_sync(0xffffffffu, mbar_wait(tmem_full, j & 1, abort_flag));
      if (!ready) break;
      tc_fence_after();
      const int m = m0 + q * 32 + lane;
      const bool valid = m < g.rows_valid;
      const float e = valid ? (g.eta ? g.eta[z * g.eta_zs + g.t0 + m] : g.eta_scalar) : 0.0f;
      const uint32_t pcol = (j & 1) ? 384u : 256u;
#pragma unroll 1
      for (int ci = 0; ci < 2; ++ci) {
        const int cc = 32 * part + 64 * ci;
        uint32_t r1[32], r3[32], rp[32];
        tmem_ld32_async(taddr + cc, r1);
        if constexpr (SWIGLU) tmem_ld32_async(taddr + 128 + cc, r3);
        tmem_ld32_async(taddr + pcol + cc, rp);
        tmem_wait_regs(r1);
        if constexpr (SWIGLU) tmem_wait_regs(r3);
        tmem_wait_regs(rp);
        if (ci == 1) {  // last TMEM read of this tile by this warp
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(tmem_empty);
        }
        float hv[32], d1[32], d3[32];
        token_dot_math<SWIGLU>(e, r1, r3, rp, hv, d1, d3);
        // the previous bulk stores must have read the staging boxes
        if (lane == 0) bulk_wait_read0();
        __syncwarp();
        stage_row_sw64(my, lane, hv);
        stage_row_sw64(my + S::STG_BYTES, lane, d1);
        if constexpr (SWIGLU) stage_row_sw64(my + 2 * S::STG_BYTES, lane, d3);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          const int row = m0 + q * 32;
          tma_store_3d(&tHp, my, nt * 128 + cc, row, z);
          if constexpr (SWIGLU) {
            tma_store_3d(&tDZ, my + S::STG_BYTES, nt * 256 + cc, row, z);
            tma_store_3d(&tDZ, my + 2 * S::STG_BYTES, nt * 256 + 128 + cc, row, z);
          } else {
            tma_store_3d(&tDZ, my + S::STG_BYTES, nt * 128 + cc, row, z);
          }
          bulk_commit();
        }
      }
    }
    if (lane == 0) bulk_wait0();
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (threadIdx.x == 0 && *abort_flag) set_status(status, kStatusTimeout);
  if (warp == 1) tmem_dealloc(tmem_base, 512);
}

template <bool SWIGLU>
cudaError_t launch_token_dot(const CUtensorMap& tX, const CUtensorMap& tFirst, const CUtensorMap& tV,
                             const CUtensorMap& tW2T, const CUtensorMap& tHp, const CUtensorMap& tDZ,
                             const TokGeom& g, unsigned* status, cudaStream_t st) {
  using S = TokShape<SWIGLU>;
  auto kern = token_dot_kernel<SWIGLU>;
  static OncePerDevice configured;
  const int set = configured.run(current_device(), [&] {
    return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, S::SMEM);
  });
  if (set != 0) return static_cast<cudaError_t>(set);
  const long long total = static_cast<long long>(g.m_tiles) * g.n_tiles * g.batches;
  if (total <= 0) return cudaSuccess;
  if (total > 0x7fffffffLL || g.kblocks <= 0) return cudaErrorInvalidConfiguration;
  const int grid = static_cast<int>(std::min<long long>(total, sm_count()));
  kern<<<grid, 64 + 32 * S::EW, S::SMEM, st>>>(tX, tFirst, tV, tW2T, tHp, tDZ, g, status);
  return cudaGetLastError();
}

}  // namespace ttt
