// Per-stage CUDA-event timing, launch counting and the CUDA-graph cache of a handle.
//
// While a forward call runs, ttt_forward points `g_prof` at the handle's
// profiler.  Every kernel launch of the path sits in a StageScope, which counts
// the launch and, when profiling is on, records an event pair around it on the
// launching stream, so a stage's device time is measured where it runs.
//
// A forward call normally replays a CUDA graph of its launch sequence (captured
// once per set of pointers).  Event pairs recorded while capturing become event
// nodes of that graph: they are re-recorded by every replay.  So that a replay
// never overwrites times nobody has read yet, a profiled pointer set keeps two
// graph instances with their own events and alternates between them; the times
// of an instance are read just before it is replayed again (by then the GPU has
// finished it and runs the other instance) and by ttt_profile_collect.
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

struct EvPair {
  int stage;
  cudaEvent_t a, b;
};

struct GraphInstance {
  cudaGraphExec_t exec = nullptr;
  std::vector<EvPair> pairs;  // owned by this instance
  bool unread = false;        // replayed since its times were last read
};

struct GraphEntry {
  const void* key[11] = {};
  bool profiled = false;
  long long launches = 0;  // kernel launches one replay performs
  GraphInstance inst[2];
  int ninst = 1, next = 0;
  unsigned long long last_use = 0;
};

struct Profiler {
  bool on = false;
  // direct launches: pairs from the pool, read (and returned) by harvest()
  std::vector<cudaEvent_t> pool;
  std::vector<EvPair> pending;
  // while a graph is being captured, pairs go to this instance instead
  std::vector<EvPair>* capture_into = nullptr;
  long long* capture_launches = nullptr;
  double ms[kNumStages] = {};
  long long cnt[kNumStages] = {};
  long long launches = 0;  // kernel launches enqueued since the handle was created
  std::vector<GraphEntry> graphs;
  unsigned long long tick = 0;

  cudaEvent_t take() {
    if (!pool.empty()) {
      cudaEvent_t e = pool.back();
      pool.pop_back();
      return e;
    }
    cudaEvent_t e = nullptr;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    return e;
  }
  void add(const EvPair& p) {
    float t = 0.f;
    if (cudaEventSynchronize(p.b) == cudaSuccess && cudaEventElapsedTime(&t, p.a, p.b) == cudaSuccess &&
        p.stage >= 0 && p.stage < kNumStages) {
      ms[p.stage] += t;
      cnt[p.stage] += 1;
    }
  }
  void read_instance(GraphInstance& g) {
    if (!g.unread) return;
    for (const EvPair& p : g.pairs) add(p);
    g.unread = false;
  }
  // read every recorded pair (synchronising on them) into the accumulators
  void harvest() {
    for (const EvPair& p : pending) {
      add(p);
      pool.push_back(p.a);
      pool.push_back(p.b);
    }
    pending.clear();
    for (GraphEntry& e : graphs)
      for (int i = 0; i < e.ninst; ++i) read_instance(e.inst[i]);
  }
  void reset_counters() {
    for (int i = 0; i < kNumStages; ++i) {
      ms[i] = 0.0;
      cnt[i] = 0;
    }
  }
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
  StageScope(int stage, cudaStream_t st) : st_(st) {
    Profiler* p = g_prof;
    if (!p) return;
    if (p->capture_launches) ++*p->capture_launches;
    else ++p->launches;
    if (!p->on) return;
    pair_.stage = stage;
    pair_.a = p->take();
    pair_.b = p->take();
    if (!pair_.a || !pair_.b) return;
    // while capturing, only an "external" record becomes an event-record node of the
    // graph (a plain record would just add a dependency edge)
    cudaEventRecordWithFlags(pair_.a, st_, p->capture_into ? cudaEventRecordExternal : cudaEventRecordDefault);
    active_ = true;
  }
  ~StageScope() {
    if (!active_ || !g_prof) return;
    cudaEventRecordWithFlags(pair_.b, st_, g_prof->capture_into ? cudaEventRecordExternal : cudaEventRecordDefault);
    if (g_prof->capture_into) g_prof->capture_into->push_back(pair_);
    else g_prof->pending.push_back(pair_);
  }

 private:
  cudaStream_t st_;
  EvPair pair_{};
  bool active_ = false;
};

}  // namespace ttt
