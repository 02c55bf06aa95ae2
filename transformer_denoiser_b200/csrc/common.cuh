// Common definitions for the Kimodo two-stage denoiser kernels (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

namespace kd {

// Model sizes: "Kimodo WebGPU", "Model details" table (1024 hidden, 8 heads x 128,
// 2048 FFN, 16 layers per sub-network) and "What it does" (4096-float text embedding).
constexpr int D = 1024;
constexpr int H = 8;
constexpr int DH = 128;
constexpr int F = 2048;
constexpr int L = 16;
constexpr int DTXT = 4096;
constexpr int ROOT_F = 5;
constexpr int BODY_F = 274;
constexpr int MOTION_F = ROOT_F + BODY_F;   // 279
constexpr int MAX_FRAMES = 300;
constexpr int N_TRAIN = 1000;

// Padded K extents of the input-projection operands (rows of 16-byte multiples).
constexpr int ROOT_IN_LD = 64;    // 5 features, zero padded to one 64-wide K block
constexpr int BODY_IN_LD = 320;   // 279 features, zero padded to five 64-wide K blocks

typedef __nv_bfloat16 bf16;

// Device-side error record (timeouts of bounded waits).  Lives in device memory
// owned by the context; the host reads it after synchronising.
struct DevError {
  int code;       // 0 = ok, otherwise a KIMODO_E* status
  int where;      // kernel-specific location tag
  int block;
  int info;
};

// A range of weights that a kernel pulls into L2 for the projections that follow it
// (16-byte aligned, a multiple of 16 bytes; null: none).  Weights are written only when
// they are loaded, so the prefetch may run before the kernel's dependency wait.
struct L2Prefetch {
  const void* p = nullptr;
  unsigned long long bytes = 0;
};

enum DevErrWhere : int {
  WHERE_GEMM_PRODUCER = 1,
  WHERE_GEMM_MMA = 2,
  WHERE_GEMM_EPILOGUE = 3,
  WHERE_GEMM_DRAIN = 4,
  WHERE_ATTENTION = 5,
  WHERE_WAIT_SELFTEST = 6,
};

}  // namespace kd
