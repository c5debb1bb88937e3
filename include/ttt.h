/*
 * ttt.h -- C ABI of the B200 (sm_100a) TTT-layer forward pass.
 *
 * The TTT (test-time training) layer replaces Softmax attention: the keys and
 * values of a chunk form a small training set, a fast-weight inner model F_W
 * takes one full-batch gradient step on a reconstruction loss over it, and the
 * queries then read the updated weights, O = F_{W*}(Q).
 *   Source: ViT3 digest ("ViT^3 test-time training for vision"), section 02,
 *   update equation  V_hat = F_W(K_B); W <- W - eta dL(V_hat, V_B)/dW; O = F_{W*}(Q);
 *   LaCT analysis ("Test-Time Training Done Right"), sections "Fast weights",
 *   "Nonlinear memory complements local attention" and "Order of operations".
 *
 * Conventions
 *   - Every matrix is row-major.  Fast weights are stored PyTorch-Linear style,
 *     [out, in], and applied to row vectors as x W^T.  Per head they are packed
 *     one after the other (P floats per head):
 *        TTT_INNER_LINEAR     [W  (d x d)]
 *        TTT_INNER_MLP2_GELU  [W1 (h x d) | W2 (d x h)]         F(x) = GELU(x W1^T) W2^T
 *        TTT_INNER_SWIGLU     [W1 (h x d) | W3 (h x d) | W2 (d x h)]
 *                                                    F(x) = (SiLU(x W1^T) * x W3^T) W2^T
 *        TTT_INNER_DWCONV     [Wc (d x k*k)]  one k x k kernel per channel (PyTorch [d,1,k,k]):
 *                             F(X)[(y,x),c] = sum_{a,b<k} Wc[c][a k + b] X[(y+a-k/2, x+b-k/2), c]
 *                             over the grid_h x grid_w token grid (raster order), zero outside
 *                             (ViT3 digest, section 03, guideline 6 and inner-model table)
 *        TTT_INNER_GLU        [Wa (d x d) | Wb (d x d)]        F(x) = (x Wa^T) * SiLU(x Wb^T)
 *                             the simplified GLU (ViT3 digest, section 03, inner-model table;
 *                             no biases, no output projection; Wa the linear branch, Wb the gate)
 *   - Q [B,H,Nq,d], K [B,H,N,d], V [B,H,N,d] and O [B,H,Nq,d] in `dtype`
 *     (fp32 or bf16); eta [B,H,N] fp32; W0 [H,P] fp32 (shared by every batch
 *     entry; [B,H,P] with TTT_FLAG_W0_PER_BATCH); W_out [B,H,P] fp32.
 *   - Losses, summed over the chunk's tokens with the per-token learning rate eta_i:
 *        TTT_LOSS_MSE      L = sum_i eta_i ||F(k_i) - v_i||^2 / (n_chunk * d)
 *        TTT_LOSS_NEG_DOT  L = -sum_i eta_i <F(k_i), v_i>
 *        TTT_LOSS_RMSE     L = sqrt(MSE)
 *   - One step per chunk (cfg.epochs steps when set; none with TTT_FLAG_NO_UPDATE):
 *     G -> [momentum M <- beta M + G] -> [Muon: Newton-Schulz]
 *     -> W <- W - lr U -> [each row of each matrix scaled to unit L2 norm; for
 *     DWCONV each channel's kernel].  TTT_FLAG_FIRST_LAYER_ONLY holds W2.
 *   - causal = 1 (needs Nq == N): per chunk, first O_c = F_W(Q_c), then update.
 *     causal = 0: update over every chunk in order, then O = F_{W*}(Q).
 *   - Nothing persists between calls: momentum starts at zero in every call.  A
 *     caller streams the weight state by passing a call's W_out as the next call's
 *     W0 with TTT_FLAG_W0_PER_BATCH, and the momentum through ttt_forward_state.
 *
 * Ownership and threading
 *   The caller owns every buffer (inputs, outputs and the workspace); the handle
 *   owns only host-side state.  Device pointers must be 16-byte aligned and
 *   contiguous.  ttt_forward only enqueues work on `stream` and returns; it
 *   allocates no device memory.  A causal call with more than one chunk runs each
 *   chunk's apply on a second stream beside the chunk's update (forked from and
 *   joined back into `stream`, inside a captured graph too): the handle creates
 *   that stream and two events the first time it needs them on a device, outside
 *   any stream capture, and ttt_destroy releases them.  One handle must not be
 *   used on two streams, or by two threads, at once.
 *   Calls run on the device current in the calling thread.  The library sets
 *   its kernels' shared-memory and cluster attributes, and asks how many CTA
 *   pairs fit, once per device, the first time a kernel runs there; one process
 *   may drive layers on several GPUs (handles hold no device memory).
 *
 * Errors
 *   Calls return TTT_OK (0) or a negative status.  Argument errors are found on
 *   the host before anything is enqueued.  Conditions found on the device
 *   (non-finite outputs, a bounded wait that ran out) are recorded in a status
 *   word at the start of the workspace and returned by ttt_query_status.
 *   Nothing traps or asserts on the device.
 */
#ifndef TTT_H_
#define TTT_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define TTT_OK 0
#define TTT_ERR_INVALID_ARG (-1) /* null pointer, bad shape, causal with Nq != N, ... */
#define TTT_ERR_UNSUPPORTED (-2) /* a valid combination the library does not implement */
#define TTT_ERR_CUDA (-3)        /* a CUDA runtime call failed */
#define TTT_ERR_NONFINITE (-4)   /* O or W* holds Inf or NaN (device status word) */
#define TTT_ERR_TIMEOUT (-5)     /* a bounded device-side wait ran out (device status word) */
#define TTT_ERR_WORKSPACE (-6)   /* workspace too small or misaligned */

typedef enum {
  TTT_INNER_LINEAR = 0,
  TTT_INNER_MLP2_GELU = 1,
  TTT_INNER_SWIGLU = 2,
  TTT_INNER_DWCONV = 3, /* the whole grid is one non-causal chunk (Nq == N, queries on the same grid);
                           loss MSE or NEG_DOT, optimizer GD or MOMENTUM, no key instance-norm;
                           other combinations return TTT_ERR_UNSUPPORTED */
  TTT_INNER_GLU = 4      /* bf16 only; loss MSE or NEG_DOT, optimizer GD or MOMENTUM; h is ignored
                           (other combinations return TTT_ERR_UNSUPPORTED) */
} ttt_inner_kind;
typedef enum {
  TTT_LOSS_MSE = 0,      /* sum_i eta_i ||F(k_i) - v_i||^2 / (n d) over the chunk's n tokens */
  TTT_LOSS_NEG_DOT = 1,  /* -sum_i eta_i <F(k_i), v_i> */
  TTT_LOSS_RMSE = 2      /* sqrt of the MSE (ViT3 digest, section 03, inner-loss table); no step where
                            the MSE is 0.  Like MSE, not built for SWIGLU with TTT_BF16 */
} ttt_loss_kind;
typedef enum {
  TTT_OPT_GD = 0,            /* U = G */
  TTT_OPT_MOMENTUM = 1,      /* M <- beta M + G; U = M */
  TTT_OPT_MUON = 2,          /* U = NS(G) */
  TTT_OPT_MOMENTUM_MUON = 3  /* M <- beta M + G; U = NS(M) */
} ttt_opt_kind;
typedef enum { TTT_F32 = 0, TTT_BF16 = 1 } ttt_dtype;

#define TTT_FLAG_KEY_INSTNORM 1u  /* normalise each key channel over the chunk's tokens */
#define TTT_FLAG_WEIGHT_L2NORM 2u /* unit L2 norm for every weight row after each update */
#define TTT_FLAG_DIRECT_LAUNCH 4u /* launch every kernel on each call instead of replaying a cached CUDA graph */
#define TTT_FLAG_W0_PER_BATCH 16u /* W0 is [B, H, P], one fast-weight state per batch entry (the W_out
                                     of the previous call on the same sequences: streaming) */
#define TTT_FLAG_NO_UPDATE 32u /* read-only: O = F_{W0}(Q) and W_out = W0, no update (LaCT
                                  "Video and distributed": chunks that only read the state) */
#define TTT_FLAG_SINGLE_CTA 8u /* token phase and weight-gradient GEMMs on single CTAs instead of CTA
                                  pairs; same results up to fp32 summation order, for comparison and tests */
#define TTT_FLAG_FIRST_LAYER_ONLY 64u /* only the matrices that read the input take the step (W1, and
                                         W3 for SWIGLU); W2 keeps its W0 value and is not row-normalised
                                         ("Test-Time Training vs Sleep", Side one: the SD3.5-T5 layer
                                         adjusts the first layer).  No effect on LINEAR.  The simplified GLU
                                         FC(x) * SiLU(FC(x)) of the ViT3 digest (section 03, inner-model
                                         table) is a SWIGLU with h = d, W1 = the SiLU gate's matrix, W3 =
                                         the linear branch's, W2 = I and this flag */

typedef struct ttt_config {
  int32_t B, H;       /* batch entries and heads (each >= 1) */
  int32_t N, Nq;      /* key/value tokens and query tokens (each >= 1; above 2^30: unsupported) */
  int32_t d, h;       /* head dim and inner hidden width (ignored for LINEAR) */
  int32_t chunk;      /* tokens per update; <= 0 or >= N means one chunk of N */
  int32_t causal;     /* 1: apply-then-update per chunk (needs Nq == N) */
  int32_t inner;      /* ttt_inner_kind */
  int32_t loss;       /* ttt_loss_kind */
  int32_t opt;        /* ttt_opt_kind */
  int32_t dtype;      /* ttt_dtype of Q, K, V and O */
  uint32_t flags;     /* TTT_FLAG_* */
  float eta_scalar;   /* learning rate of every token when eta == NULL */
  float lr;           /* multiplies the update U (default 1) */
  float momentum;     /* beta of the momentum optimizers */
  int32_t ns_iters;   /* Newton-Schulz iterations (default 5) */
  float ns_coeff[3];  /* quintic (a, b, c), default (3.4445, -4.7750, 2.0315) */
  float in_eps;       /* instance-norm epsilon (default 1e-5) */
  int32_t epochs;     /* full-batch inner steps per chunk, 1..64 (default 1; 0 reads as 1): the
                         inner model trains for `epochs` passes over each chunk before moving on
                         (ViT3 digest, inner-training ablation); momentum carries through */
  int32_t grid_h, grid_w; /* TTT_INNER_DWCONV: the token grid, grid_h * grid_w == N (else ignored) */
  int32_t ksize;          /* TTT_INNER_DWCONV: odd kernel size 1..7 (default 3; else ignored) */
} ttt_config;

typedef struct ttt_handle ttt_handle;

/* Fill `cfg` with defaults (lr 1, momentum 0.9, 5 NS iterations with the Muon
 * quintic, in_eps 1e-5, eta_scalar 1, epochs 1); shapes are zero and must be set. */
void ttt_config_init(ttt_config* cfg);

/* Validate `cfg` and build a handle.  Host only; no device work.  Returns
 * TTT_ERR_INVALID_ARG / TTT_ERR_UNSUPPORTED and leaves *out NULL on failure. */
int ttt_create(const ttt_config* cfg, ttt_handle** out);

/* Fast-weight floats per head (P). */
int64_t ttt_param_count(const ttt_handle* handle);

/* Device workspace bytes ttt_forward needs (256-byte aligned buffer). */
size_t ttt_workspace_size(const ttt_handle* handle);

/* Enqueue one TTT-layer forward pass on `stream` (a cudaStream_t; NULL = legacy
 * default stream).  All pointers are device pointers.  eta may be NULL (then
 * cfg.eta_scalar is every token's rate); W_out may be NULL.  O and W_out are
 * fully overwritten.  Returns without waiting for the GPU.
 * On a non-NULL stream that is not being captured, the first call with a given
 * set of pointers captures the pass into a CUDA graph that later calls with the
 * same pointers replay (at most 8 pointer sets are kept per handle; the handle
 * owns the graphs).  TTT_FLAG_DIRECT_LAUNCH turns this off; a stream the caller
 * is capturing gets the kernels themselves. */
int ttt_forward(ttt_handle* handle, const void* Q, const void* K, const void* V, const float* eta,
                const float* W0, void* O, float* W_out, void* workspace, size_t workspace_bytes,
                void* stream);

/* Streaming with momentum (LaCT analysis, "Video and distributed": the fast-weight
 * state is carried from one call to the next).  With a momentum optimizer the state
 * of a sequence is (W, M); W travels as W_out -> W0 (TTT_FLAG_W0_PER_BATCH) and M as
 * an opaque device blob of ttt_state_size() bytes: the heavy-ball buffer of every
 * (batch entry, head) after the call's last step, in the library's own layout.
 *   - state_in: the state_out of an earlier call, or NULL (momentum starts at zero,
 *     as in ttt_forward).  state_out: written at the end of the pass, or NULL.
 *     They may be the same buffer.  Both 16-byte aligned device memory.
 *   - A blob is valid between handles with the same B, H, d, h, inner, opt and
 *     dtype; N, Nq, chunk, causal and the flags may differ.  A read-only call
 *     (TTT_FLAG_NO_UPDATE) hands the state on unchanged.
 *   - Without momentum ttt_state_size() is 0 and the state pointers are ignored.
 * Two calls over consecutive token ranges with (W, M) handed on give the result
 * of one call with those ranges as chunks.  Otherwise as ttt_forward. */
size_t ttt_state_size(const ttt_handle* handle);
int ttt_forward_state(ttt_handle* handle, const void* Q, const void* K, const void* V, const float* eta,
                      const float* W0, void* O, float* W_out, const void* state_in, void* state_out,
                      void* workspace, size_t workspace_bytes, void* stream);

/* The same pass on HOST buffers (pinned memory gives asynchronous copies):
 * copies the inputs into the front of `device_staging`, runs ttt_forward and
 * copies O (and W_out when non-NULL) back, all enqueued on `stream`.  The host
 * outputs are valid after the stream is synchronised. */
size_t ttt_host_staging_size(const ttt_handle* handle);
int ttt_forward_host(ttt_handle* handle, const void* Q, const void* K, const void* V, const float* eta,
                     const float* W0, void* O, float* W_out, void* device_staging, size_t staging_bytes,
                     void* workspace, size_t workspace_bytes, void* stream);

/* The same pass for callers that cannot allocate device memory (a host framework
 * that owns every allocation, a latency-critical path where cudaMalloc could stall
 * the device, code running while a CUDA graph that must stay allocation-free is
 * being captured).  The pages have no counterpart of this call: it is a property
 * of this library, not of the layer.
 *   - The workspace is the library's own static device array of
 *     TTT_NOALLOC_SCRATCH_BYTES (32 MiB).  Every GPU that loads the library holds
 *     that array until the process exits.  A layer whose ttt_workspace_size is
 *     larger is rejected with TTT_ERR_WORKSPACE before anything is enqueued.
 *   - The call allocates nothing (no cudaMalloc, cudaFree or allocating library
 *     routine).  The caller passes inputs and outputs exactly as for ttt_forward.
 *   - The first call on a device looks up the address of that device's array with
 *     that device current; make that first call before any stream capture begins.
 *     The address is kept for the life of the process: after cudaDeviceReset (or
 *     any other end of the device's primary context) the array is gone and this
 *     entry must not be called again on that device.
 *   - Every call on a device shares the one array.  Each call clears what must
 *     start at zero, but calls whose GPU work overlaps (other streams, other host
 *     threads) race on the array: serialise them.
 *   - status_out (optional, device memory, 4 bytes) receives the device status
 *     bits of this call after it completes on `stream`: 0 = ok, bit 0 = non-finite
 *     values in O or W*, bit 1 = a bounded device wait ran out.
 *   - Calls through this entry are not counted or timed by the ttt_profile_* hooks.
 * Returns TTT_OK or a negative status; enqueue only, like ttt_forward. */
#define TTT_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)
int ttt_forward_noalloc(ttt_handle* handle, const void* Q, const void* K, const void* V, const float* eta,
                        const float* W0, void* O, float* W_out, unsigned* status_out, void* stream);

/* Synchronise `stream`, read the device status word of `workspace` and clear
 * it.  Returns TTT_OK, TTT_ERR_NONFINITE, TTT_ERR_TIMEOUT or TTT_ERR_CUDA. */
int ttt_query_status(ttt_handle* handle, void* workspace, void* stream);

void ttt_destroy(ttt_handle* handle);

/* Static text for a status code. */
const char* ttt_status_string(int status);

#ifdef __cplusplus
}
#endif
#endif /* TTT_H_ */
