#include "ttt_plan.cuh"
namespace ttt {
int plan_layout_bf16(Plan* p) { p->ws_bytes = 256; return TTT_OK; }
int run_bf16(const Plan&, const Io&, void*, cudaStream_t) { return TTT_ERR_UNSUPPORTED; }
}
