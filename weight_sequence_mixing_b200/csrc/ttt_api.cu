// C ABI of the TTT-layer forward pass: argument validation, workspace sizing,
// the device status word and the host-buffer wrapper.  The forward pass itself
// is planned (ttt_plan.cu) and enqueued by the fp32 or bf16 path.
#include <cstdio>
#include <cstring>
#include <new>

#include "../../include/ttt.h"
#include "ttt_plan.cuh"

using namespace ttt;

namespace ttt {
thread_local Profiler* g_prof = nullptr;
thread_local int g_stage = kStageOther;
}

extern "C" void ttt_config_init(ttt_config* c) {
  if (!c) return;
  std::memset(c, 0, sizeof(*c));
  c->chunk = 0;
  c->inner = TTT_INNER_MLP2_GELU;
  c->loss = TTT_LOSS_MSE;
  c->opt = TTT_OPT_GD;
  c->dtype = TTT_BF16;
  c->eta_scalar = 1.0f;
  c->lr = 1.0f;
  c->momentum = 0.9f;
  c->ns_iters = 5;
  c->epochs = 1;
  c->ksize = 3;
  c->ns_coeff[0] = 3.4445f;
  c->ns_coeff[1] = -4.7750f;
  c->ns_coeff[2] = 2.0315f;
  c->in_eps = 1e-5f;
}

extern "C" int ttt_create(const ttt_config* cfg, ttt_handle** out) {
  if (!out) return TTT_ERR_INVALID_ARG;
  *out = nullptr;
  if (!cfg) return TTT_ERR_INVALID_ARG;
  Plan plan;
  int st = plan_build(*cfg, &plan);
  if (st != TTT_OK) return st;
  ttt_handle* h = new (std::nothrow) ttt_handle;
  if (!h) return TTT_ERR_INVALID_ARG;
  h->plan = plan;
  *out = h;
  return TTT_OK;
}

extern "C" int64_t ttt_param_count(const ttt_handle* h) { return h ? h->plan.P : 0; }

extern "C" size_t ttt_workspace_size(const ttt_handle* h) { return h ? h->plan.ws_bytes : 0; }

namespace {

void destroy_entry(ttt::GraphEntry& e) {
  for (int i = 0; i < e.ninst; ++i) {
    if (e.inst[i].exec) cudaGraphExecDestroy(e.inst[i].exec);
    for (const ttt::EvPair& p : e.inst[i].pairs) {
      cudaEventDestroy(p.a);
      cudaEventDestroy(p.b);
    }
    e.inst[i] = ttt::GraphInstance{};
  }
}

// The side stream and events of a handle (see forward_impl).
void release_aux(ttt_handle* h) {
  if (h->ev_fork) cudaEventDestroy(h->ev_fork);
  if (h->ev_join) cudaEventDestroy(h->ev_join);
  if (h->aux) cudaStreamDestroy(h->aux);
  h->aux = nullptr;
  h->ev_fork = h->ev_join = nullptr;
  h->aux_dev = -1;
}

// Capture one replayable instance of the layer's launch sequence on `st`.
int capture_instance(ttt_handle* h, const Io& io, void* ws, cudaStream_t st, ttt::GraphInstance* gi,
                     long long* launches) {
  Profiler& pr = h->prof;
  *launches = 0;
  pr.capture_into = &gi->pairs;
  pr.capture_launches = launches;
  if (cudaStreamBeginCapture(st, cudaStreamCaptureModeThreadLocal) != cudaSuccess) {
    pr.capture_into = nullptr;
    pr.capture_launches = nullptr;
    return TTT_ERR_CUDA;
  }
  const int r = plan_run(h->plan, io, ws, st);
  cudaGraph_t graph = nullptr;
  const cudaError_t e = cudaStreamEndCapture(st, &graph);
  pr.capture_into = nullptr;
  pr.capture_launches = nullptr;
  if (r != TTT_OK || e != cudaSuccess || !graph) {
    if (graph) cudaGraphDestroy(graph);
    return r != TTT_OK ? r : TTT_ERR_CUDA;
  }
  const cudaError_t ie = cudaGraphInstantiate(&gi->exec, graph, 0);
  cudaGraphDestroy(graph);
  return ie == cudaSuccess ? TTT_OK : TTT_ERR_CUDA;
}

// Replay the cached graph of this pointer set (capturing it on first use).
int forward_graph(ttt_handle* h, const Io& io, void* ws, cudaStream_t st) {
  Profiler& pr = h->prof;
  const void* key[11] = {io.Q, io.K, io.V, io.eta, io.W0, io.O, io.W_out, io.M_in, io.M_out, ws, st};
  GraphEntry* hit = nullptr;
  for (GraphEntry& e : pr.graphs) {
    bool same = e.profiled == pr.on;
    for (int i = 0; i < 11 && same; ++i) same = e.key[i] == key[i];
    if (same) {
      hit = &e;
      break;
    }
  }
  if (!hit) {
    constexpr size_t kMaxGraphs = 8;
    if (pr.graphs.size() >= kMaxGraphs) {  // evict the least recently used pointer set
      size_t old = 0;
      for (size_t i = 1; i < pr.graphs.size(); ++i)
        if (pr.graphs[i].last_use < pr.graphs[old].last_use) old = i;
      pr.harvest();
      destroy_entry(pr.graphs[old]);
      pr.graphs.erase(pr.graphs.begin() + static_cast<long>(old));
    }
    GraphEntry e;
    for (int i = 0; i < 11; ++i) e.key[i] = key[i];
    e.profiled = pr.on;
    e.ninst = pr.on ? 2 : 1;
    for (int i = 0; i < e.ninst; ++i) {
      const int r = capture_instance(h, io, ws, st, &e.inst[i], &e.launches);
      if (r != TTT_OK) {
        destroy_entry(e);
        return r;
      }
    }
    pr.graphs.push_back(e);
    hit = &pr.graphs.back();
  }
  GraphInstance& gi = hit->inst[hit->next];
  hit->next = (hit->next + 1) % hit->ninst;
  hit->last_use = ++pr.tick;
  if (pr.on) pr.read_instance(gi);  // its previous replay finished: the other instance ran after it
  if (cudaGraphLaunch(gi.exec, st) != cudaSuccess) return TTT_ERR_CUDA;
  pr.launches += hit->launches;
  gi.unread = pr.on;
  return TTT_OK;
}

// Validate and enqueue one forward pass (ttt_forward, ttt_forward_state).
int forward_impl(ttt_handle* h, const Io& io, void* workspace, size_t workspace_bytes, void* stream) {
  if (!h || !io.Q || !io.K || !io.V || !io.W0 || !io.O) return TTT_ERR_INVALID_ARG;
  const void* ptrs[] = {io.Q, io.K, io.V, io.eta, io.W0, io.O, io.W_out, io.M_in, io.M_out};
  for (const void* p : ptrs)
    if (p && (reinterpret_cast<uintptr_t>(p) & 15) != 0) return TTT_ERR_INVALID_ARG;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255) != 0 || workspace_bytes < h->plan.ws_bytes)
    return TTT_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // Replay a cached graph unless the caller asked for direct launches, the stream
  // is the legacy default stream (not capturable), or the caller is capturing
  // the stream itself (then the launches go into the caller's graph).
  bool graph = !(h->plan.cfg.flags & TTT_FLAG_DIRECT_LAUNCH) && st != nullptr;
  if (graph) {
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(st, &cs) != cudaSuccess) return TTT_ERR_CUDA;
    graph = cs == cudaStreamCaptureStatusNone;
  }
  // The causal bf16 layer applies each chunk on a side stream while the main stream
  // computes the chunk's update; the stream and its events are made outside any capture.
  Io run = io;
  const Plan& pl = h->plan;
  if (pl.path == kPathBf16 && pl.cfg.causal && pl.nchunks > 1) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return TTT_ERR_CUDA;
    if (h->aux_dev != dev) {
      cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
      const bool capturing = st && cudaStreamIsCapturing(st, &cs) == cudaSuccess && cs != cudaStreamCaptureStatusNone;
      if (!capturing) {
        release_aux(h);
        if (cudaStreamCreateWithFlags(&h->aux, cudaStreamNonBlocking) != cudaSuccess ||
            cudaEventCreateWithFlags(&h->ev_fork, cudaEventDisableTiming) != cudaSuccess ||
            cudaEventCreateWithFlags(&h->ev_join, cudaEventDisableTiming) != cudaSuccess) {
          release_aux(h);
          return TTT_ERR_CUDA;
        }
        h->aux_dev = dev;
      }
    }
    if (h->aux_dev == dev) {
      run.aux = h->aux;
      run.ev_fork = h->ev_fork;
      run.ev_join = h->ev_join;
    }
  }
  g_prof = &h->prof;
  const int r = graph ? forward_graph(h, run, workspace, st) : plan_run(h->plan, run, workspace, st);
  g_prof = nullptr;
  return r;
}

}  // namespace

extern "C" int ttt_forward(ttt_handle* h, const void* Q, const void* K, const void* V, const float* eta,
                           const float* W0, void* O, float* W_out, void* workspace, size_t workspace_bytes,
                           void* stream) {
  const Io io{Q, K, V, eta, W0, O, W_out};
  return forward_impl(h, io, workspace, workspace_bytes, stream);
}

extern "C" size_t ttt_state_size(const ttt_handle* h) { return h ? h->plan.state_bytes : 0; }

extern "C" int ttt_forward_state(ttt_handle* h, const void* Q, const void* K, const void* V, const float* eta,
                                 const float* W0, void* O, float* W_out, const void* state_in, void* state_out,
                                 void* workspace, size_t workspace_bytes, void* stream) {
  // without momentum there is no state: the state pointers are ignored
  const bool has = h && h->plan.state_bytes > 0;
  const Io io{Q, K, V, eta, W0, O, W_out, has ? state_in : nullptr, has ? state_out : nullptr};
  return forward_impl(h, io, workspace, workspace_bytes, stream);
}

extern "C" size_t ttt_host_staging_size(const ttt_handle* h) { return h ? h->plan.staging_bytes : 0; }

extern "C" int ttt_forward_host(ttt_handle* h, const void* Q, const void* K, const void* V, const float* eta,
                                const float* W0, void* O, float* W_out, void* staging, size_t staging_bytes,
                                void* workspace, size_t workspace_bytes, void* stream) {
  if (!h || !Q || !K || !V || !W0 || !O) return TTT_ERR_INVALID_ARG;
  const Plan& p = h->plan;
  if (!staging || (reinterpret_cast<uintptr_t>(staging) & 255) != 0 || staging_bytes < p.staging_bytes)
    return TTT_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* base = static_cast<uint8_t*>(staging);
  void* dQ = base + p.stg_q;
  void* dK = base + p.stg_k;
  void* dV = base + p.stg_v;
  float* dEta = eta ? reinterpret_cast<float*>(base + p.stg_eta) : nullptr;
  float* dW0 = reinterpret_cast<float*>(base + p.stg_w0);
  void* dO = base + p.stg_o;
  float* dW = W_out ? reinterpret_cast<float*>(base + p.stg_w) : nullptr;
  const size_t es = p.cfg.dtype == TTT_F32 ? 4 : 2;
  const size_t nq = static_cast<size_t>(p.cfg.B) * p.cfg.H * p.cfg.Nq * p.cfg.d * es;
  const size_t nk = static_cast<size_t>(p.cfg.B) * p.cfg.H * p.cfg.N * p.cfg.d * es;
  const size_t ne = static_cast<size_t>(p.cfg.B) * p.cfg.H * p.cfg.N * 4;
  const size_t nw0 = static_cast<size_t>((p.cfg.flags & TTT_FLAG_W0_PER_BATCH) ? p.BH : p.cfg.H) * p.P * 4;
  const size_t nw = static_cast<size_t>(p.cfg.B) * p.cfg.H * p.P * 4;
  if (cudaMemcpyAsync(dQ, Q, nq, cudaMemcpyHostToDevice, st) != cudaSuccess ||
      cudaMemcpyAsync(dK, K, nk, cudaMemcpyHostToDevice, st) != cudaSuccess ||
      cudaMemcpyAsync(dV, V, nk, cudaMemcpyHostToDevice, st) != cudaSuccess ||
      (eta && cudaMemcpyAsync(dEta, eta, ne, cudaMemcpyHostToDevice, st) != cudaSuccess) ||
      cudaMemcpyAsync(dW0, W0, nw0, cudaMemcpyHostToDevice, st) != cudaSuccess)
    return TTT_ERR_CUDA;
  int r = ttt_forward(h, dQ, dK, dV, dEta, dW0, dO, dW, workspace, workspace_bytes, stream);
  if (r != TTT_OK) return r;
  if (cudaMemcpyAsync(O, dO, nq, cudaMemcpyDeviceToHost, st) != cudaSuccess) return TTT_ERR_CUDA;
  if (W_out && cudaMemcpyAsync(W_out, dW, nw, cudaMemcpyDeviceToHost, st) != cudaSuccess) return TTT_ERR_CUDA;
  return TTT_OK;
}

extern "C" int ttt_query_status(ttt_handle* h, void* workspace, void* stream) {
  if (!h || !workspace) return TTT_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  unsigned word = 0;
  if (cudaMemcpyAsync(&word, workspace, sizeof(word), cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return TTT_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return TTT_ERR_CUDA;
  if (cudaMemsetAsync(workspace, 0, sizeof(unsigned), st) != cudaSuccess) return TTT_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return TTT_ERR_CUDA;
  if (word & kStatusTimeout) return TTT_ERR_TIMEOUT;
  if (word & kStatusBadLaunch) return TTT_ERR_CUDA;
  if (word & kStatusNonFinite) return TTT_ERR_NONFINITE;
  return TTT_OK;
}

extern "C" void ttt_destroy(ttt_handle* h) {
  if (!h) return;
  Profiler& p = h->prof;
  for (GraphEntry& e : p.graphs) destroy_entry(e);
  for (const EvPair& q : p.pending) {
    cudaEventDestroy(q.a);
    cudaEventDestroy(q.b);
  }
  for (cudaEvent_t e : p.pool) cudaEventDestroy(e);
  release_aux(h);
  delete h;
}

extern "C" int ttt_profile_enable(ttt_handle* h, int on) {
  if (!h) return TTT_ERR_INVALID_ARG;
  h->prof.harvest();
  h->prof.reset_counters();
  h->prof.on = on != 0;
  return TTT_OK;
}

extern "C" int ttt_profile_collect(ttt_handle* h, int max_stages, float* total_ms, int* launches) {
  if (!h || max_stages <= 0 || !total_ms || !launches) return TTT_ERR_INVALID_ARG;
  h->prof.harvest();
  for (int i = 0; i < max_stages; ++i) {
    total_ms[i] = i < kNumStages ? static_cast<float>(h->prof.ms[i]) : 0.f;
    launches[i] = i < kNumStages ? static_cast<int>(h->prof.cnt[i]) : 0;
  }
  return TTT_OK;
}

extern "C" int64_t ttt_launch_count(const ttt_handle* h) { return h ? h->prof.launches : 0; }

extern "C" const char* ttt_stage_name(int s) {
  static const char* names[kNumStages] = {"token_phase", "weight_grad", "reduce_momentum", "newton_schulz",
                                          "finish_rows", "apply",       "key_norm",        "other"};
  return (s >= 0 && s < kNumStages) ? names[s] : "unknown";
}

extern "C" const char* ttt_status_string(int s) {
  switch (s) {
    case TTT_OK: return "ok";
    case TTT_ERR_INVALID_ARG: return "invalid argument";
    case TTT_ERR_UNSUPPORTED: return "unsupported configuration";
    case TTT_ERR_CUDA: return "CUDA error";
    case TTT_ERR_NONFINITE: return "non-finite values in the outputs";
    case TTT_ERR_TIMEOUT: return "a bounded device wait ran out";
    case TTT_ERR_WORKSPACE: return "workspace too small or misaligned";
    default: return "unknown status";
  }
}
