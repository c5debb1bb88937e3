/*
 * ttt_diag.h -- diagnostic entry points of the TTT-layer library.
 *
 * These exercise single building blocks of the forward pass so that they can be
 * checked in isolation against a library routine.  They are not part of the
 * layer's statement of the problem (no page defines them).
 */
#ifndef TTT_DIAG_H_
#define TTT_DIAG_H_

#include "ttt.h"

#ifdef __cplusplus
extern "C" {
#endif

/* One batched GEMM through the library's tcgen05 tensor-core engine:
 *   C[s][z] = sum over the k-blocks of split s of  A[z] * B[z]^T
 * elem_bytes 2: A, B bf16 (kind::f16); 4: A, B fp32 read as tf32 (kind::tf32), K-major only
 * (TTT_ERR_UNSUPPORTED otherwise).
 * A is [batches][M][K] when a_mn == 0 (K-major) and [batches][K][M] when a_mn == 1
 * (MN-major); B likewise with N.  C is fp32 [splits][batches][M][N], written for
 * every element.  bn is the output tile width (64/128/256 for bf16, 128/256 for
 * fp32).  Rows of A/B must be 16-byte multiples.  Enqueued on `stream`. */
int ttt_selftest_gemm(int elem_bytes, int a_mn, int b_mn, int bn, int M, int N, int K, int batches, int splits,
                      const void* A, const void* B, float* C, void* stream);

/* The activation functions the epilogues use, elementwise on n fp32 device values:
 *   kind 0: y = GELU(x) = x Phi(x), dy = GELU'(x) = Phi(x) + x phi(x) (Phi, phi: the standard
 *           normal CDF and density; erf from Abramowitz & Stegun 7.1.26, |error| <= 1.5e-7)
 *   kind 1: y = SiLU(x) = x sigma(x), dy = sigma(x) (1 + x (1 - sigma(x))) (sigma from the
 *           hardware tanh approximation, relative error about 2^-11)
 *   kind 2: y = GELU(x) as the fused apply evaluates it (erf from Abramowitz & Stegun 7.1.28,
 *           |error| <= 3e-7, one reciprocal and no exponential), dy = 0
 * (the GELU of the ViT3 MLP inner model and the SiLU of the SwiGLU / GLU inner models).
 * x, y, dy: device buffers of n floats, caller-owned.  Enqueued on `stream`;
 * TTT_ERR_INVALID_ARG for an unknown kind or missing buffers, TTT_ERR_CUDA if the launch fails. */
int ttt_selftest_activation(int kind, int64_t n, const float* x, float* y, float* dy, void* stream);

/* The execution plan ttt_create chose (host logic only, no GPU needed).  Writes up to
 * `n` ints into `info`, in this order:
 *   [0] path: 0 fp32 SIMT, 1 bf16 tensor cores, 2 DWConv (SIMT, either dtype)
 *   [1] chunk length in tokens, [2] number of chunks
 *   [3] split-K splits of the weight-gradient reductions (bf16 path; 0 on the others)
 *   [4] rows per weight-gradient tile: 128 or 256 on single CTAs, 512 on CTA pairs
 *   [5] output columns per weight-gradient tile
 *   [6] 1 when unsplit reductions write U (and momentum) directly, without partials
 * Returns the number of entries written, or TTT_ERR_INVALID_ARG. */
int ttt_plan_info(const ttt_handle* handle, int* info, int n);

/* Failure detection without a fault: launches one CTA that waits on an mbarrier no one
 * arrives at.  The wait gives up after the library's limit (2 s), as every wait of the
 * path does, records a timeout in the 4-byte device status word `status_word` (any
 * device buffer of at least 4 bytes, zeroed by the call first) and returns; the CUDA
 * context stays usable.  Synchronises `stream` and returns what the word maps to:
 * TTT_ERR_TIMEOUT when the wait ran out (the expected result), TTT_OK otherwise,
 * TTT_ERR_CUDA / TTT_ERR_INVALID_ARG on a launch or argument error. */
int ttt_selftest_timeout(void* status_word, void* stream);

/* Per-stage timing of a handle's forward calls.  ttt_profile_enable(h, 1)
 * clears earlier records and starts recording a CUDA event pair around every
 * kernel launch of later ttt_forward calls, on the stream the kernel runs on;
 * ttt_profile_enable(h, 0) stops.  ttt_profile_collect synchronises those events
 * and writes, per stage id s < max_stages, the summed device milliseconds and the
 * number of launches.  Stage ids and their names: ttt_stage_name(s). */
int ttt_profile_enable(ttt_handle* handle, int on);
int ttt_profile_collect(ttt_handle* handle, int max_stages, float* total_ms, int* launches);
const char* ttt_stage_name(int stage);

/* Kernel launches this handle's forward calls have enqueued since it was created. */
int64_t ttt_launch_count(const ttt_handle* handle);

/* CTA pairs of the token-phase kernel (swiglu != 0: SwiGLU fast weights, else the
 * GELU MLP) that can be resident at once on the current device; 0 means the pair
 * kernel cannot run there and the token phase falls back to single CTAs. */
int ttt_token_pair_capacity(int swiglu);

/* The token phase's CTA-pair tile schedule (host logic only, no GPU needed; LaCT analysis,
 * "Nonlinear memory complements local attention": the chunk's forward and backprop through
 * the fast weights, tile by tile).  Geometry: m_tiles 256-token tiles per head, n_tiles
 * hidden blocks of 128 units, batches heads, kblocks = d / 64.  cap_resident and
 * cap_streaming: CTA pairs of the resident-weight and the streaming form that fit the
 * device.  Chooses the form and the number of pairs as the launch does and writes them to
 * *resident (1 resident, 0 streaming) and *pairs; then, pair by pair, counts[p] = the tiles
 * of pair p and its tiles in processing order as (head, token tile, hidden block) int
 * triples in `tiles`, at most max_tiles triples (`counts` holds at least
 * max(cap_resident, cap_streaming) ints; all buffers caller-owned host memory).  Returns the
 * number of triples written; TTT_ERR_INVALID_ARG on bad arguments or a too small `tiles`,
 * TTT_ERR_UNSUPPORTED when no pair fits. */
int ttt_pair_schedule(int m_tiles, int n_tiles, int batches, int kblocks, int cap_resident, int cap_streaming,
                      int* resident, int* pairs, int* counts, int* tiles, int64_t max_tiles);

#ifdef __cplusplus
}
#endif
#endif /* TTT_DIAG_H_ */
