// Warp-specialised tcgen05 GEMM engine for sm_100a.
//
// A CTA loops over output tiles (persistent when the grid is smaller than the
// tile count).  Each tile is 128 x BN0 (plus, optionally, a second 128 x BN1
// product of the same rows) with the accumulators in TMEM:
//   warp 0       : TMA producer (one elected thread); the STAGES-deep smem ring runs
//                  on across tiles, so the next tile's operands load during an epilogue
//   warp 1       : TMEM allocator + MMA issuer (one elected thread)
//   warps 2..    : EW epilogue warps; warp w reads TMEM lanes 32*(w%4) .. +31 (one
//                  output row per thread) and the (w-2)/4-th share of the columns
// Tiles are visited N-tile fastest, then M-tile, then batch and split: the CTAs in
// flight share their A rows (token tiles read from HBM once) and their K range.
//
// Operands are read by TMA from 3-D tensor maps [batch][rows][cols] with 128-byte
// swizzle; each operand is K-major (K contiguous) or MN-major (M/N contiguous), so
// a reduction over tokens reads row-major [tokens][features] buffers directly.
// EB is the element size: 2 = bf16 (kind::f16), 4 = fp32 read as tf32 (kind::tf32).
//
// Launch modes:
//   BN1 == 0 : one product per tile; M-tiles >= m_tiles0 belong to a second,
//              independent problem (maps A1/B1, M1 rows) that shares N and K.
//   BN1 > 0  : two products per tile, D0 = A0 B0^T (cols [0,BN0)) and
//              D1 = A1 B1^T (cols [BN0, BN0+BN1)), both over the same K range.
// Split-K: split s reduces k-blocks [s*kb_per_split, (s+1)*kb_per_split).
#pragma once
#include <algorithm>

#include "per_device.h"
#include "ptx.cuh"

namespace ttt {

struct OpOff {  // offsets added to an operand's TMA coordinates
  int mn = 0;   // along its M (A) or N (B) dimension
  int k = 0;    // along the reduction dimension
};

struct TcGeom {
  int m_tiles0 = 0, m_tiles1 = 0, n_tiles = 0;
  int M0 = 0, M1 = 0, N = 0;
  int kblocks = 0;  // k-blocks of the whole reduction
  int batches = 1, splits = 1, kb_per_split = 0;
  OpOff a0, b0, a1, b1;
};

struct EpiCtx {
  uint32_t taddr;  // TMEM address: this warp's lane quarter, accumulator column 0
  int row;         // row inside the tile (0..127)
  int m;           // row inside the problem
  int n0;          // first output column of the tile
  int z;           // batch entry
  int split;       // split-K index
  int problem;     // 0 or 1 (grouped launches)
  int part, nparts;  // this warp handles the 32-column chunks c with c % nparts == part
};

// Tile coordinates of a linear tile index (N-tile fastest).
struct TileCoord {
  int problem, m0, n0, z, split, kb_begin, nkb;
};

__device__ __forceinline__ TileCoord decode_tile(const TcGeom& g, int t, int bn0) {
  TileCoord c;
  const int mtiles = g.m_tiles0 + g.m_tiles1;
  const int nt = t % g.n_tiles;
  int r = t / g.n_tiles;
  const int mt = r % mtiles;
  r /= mtiles;
  c.z = r % g.batches;
  c.split = r / g.batches;
  c.problem = mt >= g.m_tiles0 ? 1 : 0;
  c.m0 = (c.problem ? mt - g.m_tiles0 : mt) * 128;
  c.n0 = nt * bn0;
  c.kb_begin = c.split * g.kb_per_split;
  c.nkb = max(0, min(g.kblocks, c.kb_begin + g.kb_per_split) - c.kb_begin);
  return c;
}

__host__ __device__ constexpr int tmem_cols_for(int n) {
  return n <= 32 ? 32 : n <= 64 ? 64 : n <= 128 ? 128 : n <= 256 ? 256 : 512;
}

template <int BN0, int BN1, int EB, int STAGES>
struct TcShape {
  static constexpr int BM = 128;
  static constexpr int KB_BYTES = 128;           // bytes of K per row per stage (one swizzle span)
  static constexpr int BK = KB_BYTES / EB;       // K elements per stage
  static constexpr int UK = 32 / EB;             // K elements per MMA instruction
  static constexpr int A_BYTES = BM * KB_BYTES;  // 16 KB
  static constexpr int B0_BYTES = BN0 * KB_BYTES;
  static constexpr int B1_BYTES = BN1 * KB_BYTES;
  static constexpr int STAGE_BYTES = A_BYTES + B0_BYTES + (BN1 > 0 ? A_BYTES + B1_BYTES : 0);
  static constexpr int TMEM_COLS = tmem_cols_for(BN0 + BN1);
  static constexpr int BAR_BYTES = 256;
  static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + BAR_BYTES;
  static_assert(BN0 % 16 == 0 && BN0 >= 32 && BN0 <= 256, "BN0");
  static_assert(BN1 % 16 == 0 && BN1 <= 256, "BN1");
  static_assert(BN0 + BN1 <= 512, "TMEM");
};

// fp32-as-tf32 operands must be K-major (an MN-major tf32 operand gave wrong
// products in testing); bf16 operands may be either.
template <bool A_MN, bool B_MN, int EB>
struct MajorCheck {
  static_assert(EB == 2 || (!A_MN && !B_MN), "tf32 operands must be K-major");
  static constexpr bool ok = true;
};

// Issue the TMA loads of one operand tile (rows x K-span) into `dst`.
template <bool MN, int EB>
__device__ __forceinline__ void load_operand(uint8_t* dst, const CUtensorMap* m, uint64_t* bar, int rows,
                                             int mn0, int k0, int z) {
  if constexpr (!MN) {
    // one box {BK, rows}: rows of 128 bytes along K
    tma_load_3d(dst, m, bar, k0, mn0, z);
  } else {
    // boxes {128/EB, BK}: each box is BK K-rows of a 128-byte run along M/N
    constexpr int RUN = 128 / EB;
    constexpr int BK = 128 / EB;
    const int nbox = rows / RUN;
    for (int j = 0; j < nbox; ++j) tma_load_3d(dst + j * BK * 128, m, bar, mn0 + j * RUN, k0, z);
  }
}

template <bool MN, int EB>
__device__ __forceinline__ uint64_t operand_desc(uint32_t base, int kk) {
  if constexpr (!MN) {
    return make_sdesc_sw128(base + kk * 32, 16, 1024);
  } else {
    constexpr int BK = 128 / EB;
    constexpr int UK = 32 / EB;
    return make_sdesc_sw128(base + kk * UK * 128, BK * 128, 1024);
  }
}

template <int BN0, int BN1, bool A_MN, bool B_MN, int EB, int STAGES, int EW, class Epi>
__global__ void __launch_bounds__(64 + 32 * EW, 1)
    tc_gemm_kernel(const __grid_constant__ CUtensorMap tA0, const __grid_constant__ CUtensorMap tB0,
                   const __grid_constant__ CUtensorMap tA1, const __grid_constant__ CUtensorMap tB1,
                   const TcGeom g, const Epi epi, unsigned* status) {
  using S = TcShape<BN0, BN1, EB, STAGES>;
  static_assert(EW % 4 == 0 && EW >= 4 && EW <= 16, "epilogue warps cover the 4 TMEM lane quarters");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * S::STAGE_BYTES);
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
    mbar_init(tmem_empty, EW);
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
      if (BN1 > 0 || g.m_tiles1 > 0) {
        tma_prefetch_desc(&tA1);
        tma_prefetch_desc(&tB1);
      }
      int it = 0;
      bool stop = false;
      for (int t = blockIdx.x; t < total && !stop; t += gridDim.x) {
        const TileCoord tc = decode_tile(g, t, BN0);
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
          uint8_t* st = smem + s * S::STAGE_BYTES;
          mbar_arrive_expect_tx(&full[s], S::STAGE_BYTES);
          const int k0 = (tc.kb_begin + i) * S::BK;
          load_operand<A_MN, EB>(st, mA, &full[s], S::BM, tc.m0 + oA.mn, k0 + oA.k, tc.z);
          load_operand<B_MN, EB>(st + S::A_BYTES, mB, &full[s], BN0, tc.n0 + oB.mn, k0 + oB.k, tc.z);
          if constexpr (BN1 > 0) {
            uint8_t* st1 = st + S::A_BYTES + S::B0_BYTES;
            load_operand<A_MN, EB>(st1, &tA1, &full[s], S::BM, tc.m0 + g.a1.mn, k0 + g.a1.k, tc.z);
            load_operand<B_MN, EB>(st1 + S::A_BYTES, &tB1, &full[s], BN1, tc.n0 / BN0 * BN1 + g.b1.mn,
                                   k0 + g.b1.k, tc.z);
          }
        }
      }
      if (*abort_flag) {
        // let the copies already in flight land before the CTA's smem is released
        for (int j = max(0, it - STAGES); j < it; ++j) {
          volatile int never = 0;
          mbar_wait(&full[j % STAGES], (j / STAGES) & 1, &never);
        }
      }
    }
  } else if (warp == 1) {
    if (elect_one()) {
      constexpr int fmt = EB == 2 ? 1 : 2;
      constexpr uint32_t id0 = make_idesc(128, BN0, fmt, A_MN, B_MN);
      constexpr uint32_t id1 = make_idesc(128, BN1 > 0 ? BN1 : 16, fmt, A_MN, B_MN);
      const uint32_t sbase = smem_u32(smem);
      int it = 0, j = 0;
      bool stop = false;
      for (int t = blockIdx.x; t < total && !stop; t += gridDim.x, ++j) {
        const TileCoord tc = decode_tile(g, t, BN0);
        // the previous tile's epilogue must have drained the accumulators
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
          const uint32_t a = sbase + s * S::STAGE_BYTES;
          const uint32_t b = a + S::A_BYTES;
#pragma unroll
          for (int kk = 0; kk < S::BK / S::UK; ++kk) {
            const uint32_t acc = (i > 0 || kk > 0) ? 1u : 0u;
            const uint64_t da = operand_desc<A_MN, EB>(a, kk);
            const uint64_t db = operand_desc<B_MN, EB>(b, kk);
            if constexpr (EB == 2) mma_f16(tmem_base, da, db, id0, acc);
            else mma_tf32(tmem_base, da, db, id0, acc);
            if constexpr (BN1 > 0) {
              const uint32_t a1 = b + S::B0_BYTES;
              const uint32_t b1 = a1 + S::A_BYTES;
              const uint64_t da1 = operand_desc<A_MN, EB>(a1, kk);
              const uint64_t db1 = operand_desc<B_MN, EB>(b1, kk);
              if constexpr (EB == 2) mma_f16(tmem_base + BN0, da1, db1, id1, acc);
              else mma_tf32(tmem_base + BN0, da1, db1, id1, acc);
            }
          }
          mma_commit(&empty[s]);
        }
        mma_commit(tmem_full);
      }
      if (*abort_flag) {
        // MMAs in flight finish before TMEM is released
        volatile int never = 0;
        mma_commit(drain);
        mbar_wait(drain, 0, &never);
      }
    }
  } else {
    const int q = warp & 3;
    const int row = q * 32 + static_cast<int>(lane_id());
    int j = 0;
    for (int t = blockIdx.x; t < total; t += gridDim.x, ++j) {
      const TileCoord tc = decode_tile(g, t, BN0);
      // warp-uniform decision: tcgen05.ld below is a warp-collective instruction
      const bool ready = __all_sync(0xffffffffu, mbar_wait(tmem_full, j & 1, abort_flag));
      if (!ready) break;
      tc_fence_after();
      EpiCtx c;
      c.taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
      c.row = row;
      c.m = tc.m0 + row;
      c.n0 = tc.n0;
      c.z = tc.z;
      c.split = tc.split;
      c.problem = tc.problem;
      c.part = (warp - 2) >> 2;
      c.nparts = EW / 4;
      if (tc.nkb > 0) epi.template run<BN0, BN1>(c);
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

// ---------------------------------------------------------------- host side
typedef CUresult (*PFN_tmapEncodeTiled)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                         const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                         CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                         CUtensorMapFloatOOBfill);

PFN_tmapEncodeTiled tmap_encoder();

// A 3-D view [batches][rows][cols] of a row-major buffer, as a TMA tensor map
// with 128-byte swizzle.  `k_major` picks the box: {128/EB, 128|BN rows} for a
// K-major operand (rows = M or N) and {128/EB, 128/EB rows} for an MN-major one.
// Returns false when the view violates a TMA rule (alignment, pitch, extent).
bool make_tmap(CUtensorMap* out, const void* base, int eb, int64_t cols, int64_t rows, int64_t batches,
               int64_t row_pitch_elems, int64_t batch_pitch_elems, int box_rows);
// General form: box {box_cols, box_rows}, swizzle span 32 / 64 / 128 bytes (box_cols * eb <= span).
bool make_tmap_ex(CUtensorMap* out, const void* base, int eb, int64_t cols, int64_t rows, int64_t batches,
                  int64_t row_pitch_elems, int64_t batch_pitch_elems, int box_cols, int box_rows, int swizzle);

// SMs of the current device (queried once per device)
int sm_count();
// the current device's ordinal, or -1 when it cannot be read
int current_device();

// persistent = true: at most (SMs x resident CTAs per SM) CTAs loop over the tiles;
// otherwise one CTA per tile.
template <int BN0, int BN1, bool A_MN, bool B_MN, int EB, int STAGES, int EW = 4, class Epi>
cudaError_t launch_tc_gemm(const CUtensorMap& a0, const CUtensorMap& b0, const CUtensorMap& a1,
                           const CUtensorMap& b1, const TcGeom& g, const Epi& epi, unsigned* status,
                           cudaStream_t st, bool persistent = false) {
  using S = TcShape<BN0, BN1, EB, STAGES>;
  static_assert(MajorCheck<A_MN, B_MN, EB>::ok, "");
  auto kern = tc_gemm_kernel<BN0, BN1, A_MN, B_MN, EB, STAGES, EW, Epi>;
  // TMEM holds 512 columns per SM: request enough shared memory that the CTAs
  // resident on one SM never ask for more columns than exist (an allocation
  // beyond that would stall until a neighbour frees its columns).
  constexpr int kSmemPerSM = 228 * 1024, kReservedPerCta = 1024;
  constexpr int kMaxCtas = 512 / S::TMEM_COLS;
  constexpr int kMinSmem = kSmemPerSM / (kMaxCtas + 1) - kReservedPerCta + 16;
  constexpr int kSmem = S::SMEM_BYTES > kMinSmem ? S::SMEM_BYTES : kMinSmem;
  static_assert(kSmem <= 227 * 1024, "shared memory per CTA");
  constexpr int kCtasPerSm = kSmemPerSM / (kSmem + kReservedPerCta) < kMaxCtas
                                 ? kSmemPerSM / (kSmem + kReservedPerCta)
                                 : kMaxCtas;
  static OncePerDevice configured;
  const int set = configured.run(current_device(), [&] {
    return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
  });
  if (set != 0) return static_cast<cudaError_t>(set);
  const long long total = static_cast<long long>(g.m_tiles0 + g.m_tiles1) * g.n_tiles * g.batches * g.splits;
  if (total <= 0) return cudaSuccess;
  if (total > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  long long grid = total;
  if (persistent) grid = std::min<long long>(total, static_cast<long long>(sm_count()) * (kCtasPerSm > 0 ? kCtasPerSm : 1));
  kern<<<static_cast<unsigned>(grid), 64 + 32 * EW, kSmem, st>>>(a0, b0, a1, b1, g, epi, status);
  return cudaGetLastError();
}

}  // namespace ttt
