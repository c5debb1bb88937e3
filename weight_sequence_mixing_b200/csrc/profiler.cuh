// Per-stage CUDA-event timing and launch counting for one handle.
//
// While a forward call runs, ttt_forward points `g_prof` at the handle's
// profiler.  Every kernel launch of the path sits in a StageScope, which counts
// the launch and, when profiling is on, records an event pair around it on the
// launching stream, so a stage's device time is measured where it runs.
#pragma once
#include <cuda_runtime.h>

#include <vector>

namespace ttt {

enum Stage : int {
  kStageTokenPhase = 0,  // fused inner forward on keys + loss backprop to the hidden layer
  kStageWeightGrad,      // token-reduction GEMMs of the weight gradients (split-K partials)
  kStageReduce,          // split reduction + momentum
  kStageNewtonSchulz,    // Newton-Schulz GEMMs and their prologue kernels
  kStageFinish,          // W <- W - lr U, row norm, bf16 weight copies
  kStageApply,           // O = F_W(Q) GEMMs
  kStageKeyNorm,         // key instance-norm (and other per-token prologues)
  kStageOther,           // initialisation, SIMT path kernels
  kNumStages
};

struct Profiler {
  bool on = false;
  std::vector<cudaEvent_t> pool;
  std::vector<int> stage_of;  // per recorded pair
  size_t used = 0;            // event pairs used since enable
  long long launches = 0;     // kernel launches since the handle was created
};

extern thread_local Profiler* g_prof;
extern thread_local int g_stage;  // stage of the launches made inside a StageCtx

struct StageCtx {
  int prev;
  explicit StageCtx(int s) : prev(g_stage) { g_stage = s; }
  ~StageCtx() { g_stage = prev; }
};

class StageScope {
 public:
  StageScope(int stage, cudaStream_t st) : st_(st), idx_(-1) {
    Profiler* p = g_prof;
    if (!p) return;
    ++p->launches;
    if (!p->on) return;
    if (p->used * 2 + 2 > p->pool.size()) {
      for (int i = 0; i < 64; ++i) {
        cudaEvent_t e;
        if (cudaEventCreate(&e) != cudaSuccess) return;
        p->pool.push_back(e);
      }
    }
    idx_ = static_cast<long>(p->used++);
    p->stage_of.push_back(stage);
    cudaEventRecord(p->pool[2 * idx_], st_);
  }
  ~StageScope() {
    if (idx_ >= 0 && g_prof) cudaEventRecord(g_prof->pool[2 * idx_ + 1], st_);
  }

 private:
  cudaStream_t st_;
  long idx_;
};

}  // namespace ttt
