// Optional per-kernel device timing.  When enabled for a kernel kind
// (qlora_trace_enable, qlora_trace_enable_kinds), its launch sites record a
// CUDA event pair around the kernel on the caller's stream (which also keeps
// that launch from overlapping the previous kernel's tail); qlora_trace_read waits for the events and reports, per kernel kind,
// the launch count and total device time.  Disabled, a launch site costs one
// relaxed atomic load.
#pragma once

#include <cuda_runtime.h>

namespace ql {

enum TraceKind : int {
  TK_QUANTIZE = 0,
  TK_DQ_MEAN,
  TK_DQ_ENCODE,
  TK_DEQUANT,
  TK_GEMM_FWD,
  TK_GEMM_BWD,
  TK_PROJ,
  TK_COLACC,
  TK_COLACC_REDUCE,
  TK_SILU,
  TK_SMALLM,
  TK_TRANSPOSE,
  TK_MERGE,
  TK_FP4,
  TK_ADAMW,
  TK_FP4GEMM,
  TK_COUNT
};

const char* trace_name(int kind);
bool trace_on(int kind);
void trace_push(int kind, cudaEvent_t start, cudaEvent_t stop);
cudaEvent_t trace_event();

// RAII: records start at construction and stop at destruction when tracing.
struct TraceScope {
  int kind;
  cudaStream_t st;
  cudaEvent_t a = nullptr, b = nullptr;
  TraceScope(int k, cudaStream_t s) : kind(k), st(s) {
    if (trace_on(k)) {
      a = trace_event();
      b = trace_event();
      if (a && b) cudaEventRecord(a, st);
    }
  }
  ~TraceScope() {
    if (a && b) {
      cudaEventRecord(b, st);
      trace_push(kind, a, b);
    }
  }
};

}  // namespace ql
