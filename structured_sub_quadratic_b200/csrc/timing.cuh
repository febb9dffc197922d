// Optional per-kernel timing: CUDA events recorded around every launch on the
// launching stream, enabled through monarch_attn_timing_enable().
#pragma once

#include <cuda_runtime.h>

#include <type_traits>

namespace monarch {

bool timing_enabled();

// Records a start event on construction and a stop event in stop() when
// timing is enabled; does nothing otherwise.
class KernelTimer {
 public:
  KernelTimer(const char* name, cudaStream_t stream);
  void stop();

 private:
  int slot_ = -1;
  cudaEvent_t start_ = nullptr;
  cudaStream_t stream_;
};

// Launch `f` (a lambda that performs one <<<>>> launch), timing it when
// enabled, checking the launch error and counting it in *launches.
// `f` may return the launch's cudaError_t (cudaLaunchKernelEx) or nothing
// (a <<<>>> launch, checked with cudaGetLastError).
template <typename F>
cudaError_t timed_launch(const char* name, cudaStream_t stream, int* launches, F&& f) {
  KernelTimer t(name, stream);
  cudaError_t e;
  if constexpr (std::is_same<decltype(f()), cudaError_t>::value) {
    e = f();
    if (e == cudaSuccess) e = cudaGetLastError();
  } else {
    f();
    e = cudaGetLastError();
  }
  t.stop();
  if (e == cudaSuccess) ++*launches;
  return e;
}

}  // namespace monarch
