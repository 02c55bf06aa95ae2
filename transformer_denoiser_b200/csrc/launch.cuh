// Kernel launch with programmatic dependent launch (PDL).
//
// Every kernel of the denoising loop is launched with programmatic stream
// serialization, so a kernel's CTAs may start (and run their prologue: barrier
// set-up, TMEM allocation, descriptor prefetch) while the previous kernel drains.
// Each kernel executes griddepcontrol.wait before it reads anything an earlier
// kernel wrote, which blocks until every prerequisite grid has completed and its
// memory is visible; correctness therefore does not depend on where the earlier
// kernel calls griddepcontrol.launch_dependents.  KIMODO_PDL=0 disables it.
#pragma once

#include <cuda_runtime.h>
#include <stdlib.h>

namespace kd {

inline bool pdl_enabled() {
  static int v = -1;
  if (v < 0) {
    const char* e = getenv("KIMODO_PDL");
    v = (e != nullptr && e[0] == '0') ? 0 : 1;
  }
  return v != 0;
}

template <typename... KArgs, typename... Args>
inline cudaError_t launch_kernel(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                                 Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

}  // namespace kd
