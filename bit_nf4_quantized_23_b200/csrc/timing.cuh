// RAII event timer around library launches (timing.cu).
#pragma once

#include <cuda_runtime.h>

namespace qlora {

class TimerScope {
  public:
    TimerScope(int kind, cudaStream_t s);
    ~TimerScope();
    TimerScope(const TimerScope&) = delete;
    TimerScope& operator=(const TimerScope&) = delete;

  private:
    int kind_;
    cudaStream_t stream_;
    cudaEvent_t a_, b_;
};

}  // namespace qlora
