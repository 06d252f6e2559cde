#pragma once
// Optional per-launch timing: while enabled, every kernel launch of the
// library is bracketed by a CUDA event pair recorded on the launch's stream.
#include <cuda_runtime.h>

namespace r4 {

void prof_mark_begin(const char* name, cudaStream_t stream);
void prof_mark_end(cudaStream_t stream);

struct ProfScope {
  cudaStream_t s;
  ProfScope(const char* name, cudaStream_t stream) : s(stream) { prof_mark_begin(name, stream); }
  ~ProfScope() { prof_mark_end(s); }
};

}  // namespace r4

// One scope object per use, named after the line (two-level paste so that
// __LINE__ expands before it is pasted).
#define R4_PROF_CAT2(a, b) a##b
#define R4_PROF_CAT(a, b) R4_PROF_CAT2(a, b)
#define R4_PROF(name, stream) ::r4::ProfScope R4_PROF_CAT(r4_prof_scope_, __LINE__)(name, stream)
