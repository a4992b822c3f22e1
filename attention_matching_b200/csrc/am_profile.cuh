// RAII bracket around one kernel launch: counts it and, while stage timing is
// enabled, records CUDA events before and after it on the launch stream.
#pragma once

#include <cuda_runtime.h>

namespace am {

class ProfScope {
 public:
  ProfScope(int stage, cudaStream_t s);
  ~ProfScope();
  ProfScope(const ProfScope&) = delete;
  ProfScope& operator=(const ProfScope&) = delete;

 private:
  int stage_;
  cudaStream_t s_;
  cudaEvent_t a_;
};

}  // namespace am

// Launch one kernel inside a profiling bracket.
#define AM_LAUNCH(stage, stream, ...)          \
  do {                                         \
    ::am::ProfScope am_prof_scope_(stage, stream); \
    __VA_ARGS__;                               \
  } while (0)
