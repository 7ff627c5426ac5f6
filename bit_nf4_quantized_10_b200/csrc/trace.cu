// Per-kernel device timing (see trace.cuh).  Events are created on the device
// that is current when a traced launch happens; one process is expected to
// trace one device.
#include <atomic>
#include <mutex>
#include <vector>

#include "common.cuh"
#include "trace.cuh"

namespace ql {
namespace {
struct Rec {
  int kind;
  cudaEvent_t a, b;
};
std::atomic<unsigned> g_on{0};
std::mutex g_mu;
std::vector<Rec> g_recs;
std::vector<cudaEvent_t> g_free;
const char* const kNames[TK_COUNT] = {"nf4_quantize",   "dq_tree_sum",    "dq_encode",       "nf4_dequant",
                                      "qlora_gemm_fwd", "qlora_gemm_bwd", "lora_side_proj", "lora_grad",
                                      "lora_grad_reduce", "silu_gate",    "smallm_splitk",   "lora_transpose",
                                      "adapter_merge", "fp4_codec",     "adamw_step",      "nvfp4_gemm"};
}  // namespace

const char* trace_name(int kind) { return (kind >= 0 && kind < TK_COUNT) ? kNames[kind] : "unknown"; }
bool trace_on(int kind) { return (g_on.load(std::memory_order_relaxed) >> kind) & 1u; }

cudaEvent_t trace_event() {
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_free.empty()) {
    cudaEvent_t e = g_free.back();
    g_free.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
  return e;
}

void trace_push(int kind, cudaEvent_t a, cudaEvent_t b) {
  std::lock_guard<std::mutex> lk(g_mu);
  g_recs.push_back(Rec{kind, a, b});
}

}  // namespace ql

extern "C" {

void qlora_trace_enable(int on) { qlora_trace_enable_kinds(on ? 0xFFFFFFFFu : 0u); }

void qlora_trace_enable_kinds(unsigned mask) {
  std::lock_guard<std::mutex> lk(ql::g_mu);
  for (auto& r : ql::g_recs) {
    cudaEventSynchronize(r.b);
    ql::g_free.push_back(r.a);
    ql::g_free.push_back(r.b);
  }
  ql::g_recs.clear();
  ql::g_on.store(mask);
}

int qlora_trace_read(double* total_ms, int* launches, int max_kinds) {
  std::lock_guard<std::mutex> lk(ql::g_mu);
  const int n = max_kinds < ql::TK_COUNT ? max_kinds : ql::TK_COUNT;
  for (int k = 0; k < n; ++k) {
    if (total_ms) total_ms[k] = 0.0;
    if (launches) launches[k] = 0;
  }
  for (auto& r : ql::g_recs) {
    float ms = 0.0f;
    if (cudaEventSynchronize(r.b) == cudaSuccess && cudaEventElapsedTime(&ms, r.a, r.b) == cudaSuccess &&
        r.kind < n) {
      if (total_ms) total_ms[r.kind] += ms;
      if (launches) launches[r.kind] += 1;
    }
    ql::g_free.push_back(r.a);
    ql::g_free.push_back(r.b);
  }
  ql::g_recs.clear();
  return n;
}

const char* qlora_trace_kind_name(int kind) { return ql::trace_name(kind); }

}  // extern "C"
