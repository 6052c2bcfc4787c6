// Host-side count of the kernels this library enqueues, for callers that
// want to know how many launches a region issued.
#pragma once

#include <cuda_runtime.h>

namespace lcsc {

// Adds one to the process-wide count of enqueued kernels.
void note_launch();

// Passes a launch's status through, counting the launch when it was enqueued.
inline cudaError_t counted(cudaError_t e) {
  if (e == cudaSuccess) note_launch();
  return e;
}

}  // namespace lcsc
