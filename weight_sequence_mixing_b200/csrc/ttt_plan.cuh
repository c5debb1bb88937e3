// Host-side plan of one configured TTT layer: validated sizes, chunking,
// which device path runs it, and the carving of the caller's workspace.
#pragma once
#include <cstddef>
#include <cstdint>

#include "../../include/ttt.h"
#include "profiler.cuh"
#include "ptx.cuh"

namespace ttt {

struct Io {
  const void* Q;
  const void* K;
  const void* V;
  const float* eta;
  const float* W0;
  void* O;
  float* W_out;
  const void* M_in = nullptr;  // momentum state carried in (ttt_forward_state), or null: zero
  void* M_out = nullptr;       // momentum state carried out, or null
  // a second stream of the calling device for work that may overlap the main stream's
  // (the causal layer's apply on a chunk runs beside that chunk's update), with the
  // events that fork it from and join it back into the main stream; null: no overlap
  cudaStream_t aux = nullptr;
  cudaEvent_t ev_fork = nullptr, ev_join = nullptr;
};

enum PathKind : int { kPathF32 = 0, kPathBf16 = 1, kPathDwconv = 2 };

struct Plan {
  ttt_config cfg{};
  int64_t P = 0;       // fast-weight floats per head
  int BH = 0;          // B * H
  int chunk = 0;       // tokens per chunk (== N for one chunk)
  int nchunks = 0;
  int epochs = 1;      // full-batch steps per chunk
  int path = kPathF32;
  size_t ws_bytes = 0;
  size_t state_bytes = 0;  // momentum state (0 without momentum)
  // host-staging layout (ttt_forward_host)
  size_t staging_bytes = 0, stg_q = 0, stg_k = 0, stg_v = 0, stg_eta = 0, stg_w0 = 0, stg_o = 0, stg_w = 0;
  // workspace layout: byte offsets into the caller's workspace
  size_t off[32] = {};
};

int plan_build(const ttt_config& cfg, Plan* plan);
// SMs of the current device (launch-time grid sizing; tmap.cu)
int sm_count();
// B200's SM count: the planner sizes its work splits with it, since ttt_create runs
// on the host without a device
constexpr int kPlanSMs = 148;
int plan_run(const Plan& plan, const Io& io, void* workspace, cudaStream_t st);

// per-path workspace layout and launch sequence
int plan_layout_f32(Plan* plan);
int plan_layout_bf16(Plan* plan);
int plan_layout_dwconv(Plan* plan);
int run_f32(const Plan& plan, const Io& io, void* workspace, cudaStream_t st);
int run_bf16(const Plan& plan, const Io& io, void* workspace, cudaStream_t st);
int run_dwconv(const Plan& plan, const Io& io, void* workspace, cudaStream_t st);

}  // namespace ttt

struct ttt_handle {
  ttt::Plan plan;
  ttt::Profiler prof;
  // the side stream and fork / join events of Io::aux, made for the device they were first
  // needed on (remade if a later call runs on another device)
  int aux_dev = -1;
  cudaStream_t aux = nullptr;
  cudaEvent_t ev_fork = nullptr, ev_join = nullptr;
};
