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

// Whether launches allow programmatic stream serialisation (on unless the
// environment sets LCSC_PDL=0; read once per process).
bool pdl_enabled();

// Fills the programmatic-serialisation attribute: a kernel so launched is
// set up ahead and starts as the stream's previous kernel's last CTA exits,
// instead of after that kernel's completion has gone round the launch queue.
// Every kernel of this library starts with grid_dep_wait() (common.cuh),
// which waits for the previous kernel to complete and its writes to be
// visible before any global memory access, so the stream order of results
// is unchanged.
inline void set_pdl(cudaLaunchAttribute& attr) {
  attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr.val.programmaticStreamSerializationAllowed = pdl_enabled() ? 1 : 0;
}

#ifdef __CUDACC__
// Enqueues k<<<grid, block, smem, stream>>>(args...) with the attribute above
// and counts it.
template <typename... P, typename... A>
cudaError_t launch_pdl(void (*k)(P...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream, A&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  set_pdl(attr[0]);
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return counted(cudaLaunchKernelEx(&cfg, k, static_cast<A&&>(args)...));
}
#endif

}  // namespace lcsc
