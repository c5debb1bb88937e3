// Diagnostic entry point: one plain tcgen05 GEMM through the same engine the
// TTT path uses, so the operand layouts (K-major / MN-major, bf16 / tf32),
// ragged edges, batching and split-K can be checked against a library matmul.
#include "../../include/ttt_diag.h"
#include "epilogues.cuh"
#include "gelu_fwd.cuh"
#include "tc_gemm.cuh"

namespace ttt {
namespace {

struct EpiStorePartial {
  float* out;  // [splits][batches][M][N]
  int M, N, batches;
  template <int BN0, int BN1>
  __device__ void run(const EpiCtx& c) const {
    float* rowp = out + ((static_cast<int64_t>(c.split) * batches + c.z) * M + c.m) * N;
#pragma unroll 1
    for (int cc = 32 * c.part; cc < BN0; cc += 32 * c.nparts) {
      float v[32];
      tmem_ld32(c.taddr + cc, v);
      if (c.m < M) {
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (c.n0 + cc + j < N) rowp[c.n0 + cc + j] = v[j];
      }
    }
  }
};

template <int BN, bool AMN, bool BMN, int EB>
int run_one(const void* A, const void* B, float* C, int M, int N, int K, int batches, int splits,
            cudaStream_t st) {
  CUtensorMap ta, tb;
  const int run = 128 / EB;
  // A: K-major [batch][M][K]; MN-major [batch][K][M].  Same for B with N.
  bool ok = AMN ? make_tmap(&ta, A, EB, M, K, batches, M, static_cast<int64_t>(M) * K, run)
                : make_tmap(&ta, A, EB, K, M, batches, K, static_cast<int64_t>(M) * K, 128);
  ok = ok && (BMN ? make_tmap(&tb, B, EB, N, K, batches, N, static_cast<int64_t>(N) * K, run)
                  : make_tmap(&tb, B, EB, K, N, batches, K, static_cast<int64_t>(N) * K, BN));
  if (!ok) return TTT_ERR_INVALID_ARG;
  TcGeom g;
  g.m_tiles0 = (M + 127) / 128;
  g.n_tiles = (N + BN - 1) / BN;
  g.M0 = M;
  g.N = N;
  g.kblocks = (K + run - 1) / run;
  g.batches = batches;
  g.kb_per_split = (g.kblocks + splits - 1) / splits;
  g.splits = (g.kblocks + g.kb_per_split - 1) / g.kb_per_split;
  if (g.splits != splits) return TTT_ERR_INVALID_ARG;  // every split must own at least one k-block
  EpiStorePartial epi{C, M, N, batches};
  // odd batch counts run one CTA per tile, even ones persistent with 8 epilogue warps,
  // so both launch shapes of the engine are exercised
  cudaError_t e = (batches % 2)
                      ? launch_tc_gemm<BN, 0, AMN, BMN, EB, 4, 4>(ta, tb, ta, tb, g, epi, nullptr, st, false)
                      : launch_tc_gemm<BN, 0, AMN, BMN, EB, 4, 8>(ta, tb, ta, tb, g, epi, nullptr, st, true);
  return e == cudaSuccess ? TTT_OK : TTT_ERR_CUDA;
}

template <int BN, int EB>
int dispatch_major(int a_mn, int b_mn, const void* A, const void* B, float* C, int M, int N, int K, int batches,
                   int splits, cudaStream_t st) {
  if constexpr (EB == 4) {
    if (a_mn || b_mn) return TTT_ERR_UNSUPPORTED;
    return run_one<BN, false, false, EB>(A, B, C, M, N, K, batches, splits, st);
  } else {
  if (!a_mn && !b_mn) return run_one<BN, false, false, EB>(A, B, C, M, N, K, batches, splits, st);
  if (!a_mn && b_mn) return run_one<BN, false, true, EB>(A, B, C, M, N, K, batches, splits, st);
  if (a_mn && !b_mn) return run_one<BN, true, false, EB>(A, B, C, M, N, K, batches, splits, st);
  return run_one<BN, true, true, EB>(A, B, C, M, N, K, batches, splits, st);
  }
}

}  // namespace
}  // namespace ttt

extern "C" int ttt_selftest_gemm(int elem_bytes, int a_mn, int b_mn, int bn, int M, int N, int K, int batches,
                                 int splits, const void* A, const void* B, float* C, void* stream) {
  using namespace ttt;
  if (!A || !B || !C || M <= 0 || N <= 0 || K <= 0 || batches <= 0 || splits <= 0) return TTT_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (elem_bytes == 2) {
    if (bn == 64) return dispatch_major<64, 2>(a_mn, b_mn, A, B, C, M, N, K, batches, splits, st);
    if (bn == 128) return dispatch_major<128, 2>(a_mn, b_mn, A, B, C, M, N, K, batches, splits, st);
    if (bn == 256) return dispatch_major<256, 2>(a_mn, b_mn, A, B, C, M, N, K, batches, splits, st);
  } else if (elem_bytes == 4) {
    if (bn == 128) return dispatch_major<128, 4>(a_mn, b_mn, A, B, C, M, N, K, batches, splits, st);
    if (bn == 256) return dispatch_major<256, 4>(a_mn, b_mn, A, B, C, M, N, K, batches, splits, st);
  }
  return TTT_ERR_UNSUPPORTED;
}

namespace ttt {
namespace {

// An mbarrier that expects one arrival which never comes: the bounded wait runs out.
__global__ void stuck_wait_kernel(unsigned* status) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0 && !mbar_wait(&bar, 0, &abort_flag)) set_status(status, kStatusTimeout);
}

// The activation functions of the epilogues, elementwise: kind 0 GELU and its derivative,
// kind 1 SiLU and its derivative, kind 2 the apply's GELU alone (dy = 0).
__global__ void activation_kernel(int kind, int64_t n, const float* x, float* y, float* dy) {
  for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < n; i += int64_t(gridDim.x) * blockDim.x) {
    const float v = x[i];
    float f, g;
    if (kind == 0) {
      gelu_and_grad(v, f, g);
    } else if (kind == 2) {
      f = gelu_fwd2(make_float2(v, v)).x;
      g = 0.0f;
    } else {
      const float s = sigmoid_dev(v);
      f = v * s;
      g = s * fmaf(v, 1.0f - s, 1.0f);
    }
    y[i] = f;
    dy[i] = g;
  }
}

}  // namespace
}  // namespace ttt

extern "C" int ttt_selftest_activation(int kind, int64_t n, const float* x, float* y, float* dy, void* stream_ptr) {
  if (kind < 0 || kind > 2 || n < 0 || (n > 0 && (!x || !y || !dy))) return TTT_ERR_INVALID_ARG;
  if (n == 0) return TTT_OK;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_ptr);
  const int grid = static_cast<int>(std::min<int64_t>((n + 255) / 256, 4096));
  ttt::activation_kernel<<<grid, 256, 0, stream>>>(kind, n, x, y, dy);
  return cudaGetLastError() == cudaSuccess ? TTT_OK : TTT_ERR_CUDA;
}

extern "C" int ttt_selftest_timeout(void* status_word, void* stream_ptr) {
  if (!status_word) return TTT_ERR_INVALID_ARG;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_ptr);
  unsigned* w = static_cast<unsigned*>(status_word);
  if (cudaMemsetAsync(w, 0, sizeof(unsigned), stream) != cudaSuccess) return TTT_ERR_CUDA;
  ttt::stuck_wait_kernel<<<1, 32, 0, stream>>>(w);
  if (cudaGetLastError() != cudaSuccess) return TTT_ERR_CUDA;
  unsigned word = 0;
  if (cudaMemcpyAsync(&word, w, sizeof(word), cudaMemcpyDeviceToHost, stream) != cudaSuccess) return TTT_ERR_CUDA;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return TTT_ERR_CUDA;
  return (word & ttt::kStatusTimeout) ? TTT_ERR_TIMEOUT : TTT_OK;
}
