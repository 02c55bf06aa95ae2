// LayerNorm over the 1024 features of a token ("Kimodo WebGPU", "WGSL compute
// shaders" table: layer normalization; "Model details": post-norm layers).
// One warp per row: the row (fp32 residual sum) is held in registers, the mean
// and the biased variance are two warp-shuffle reductions (two passes over the
// registers), eps = 1e-5; statistics in fp32, output bf16 or fp32, and optional
// row statistics, from which a later residual epilogue rebuilds the normalised row
// instead of reading it.
#include <cuda_runtime.h>

#include "common.cuh"
#include "kernels.h"
#include "launch.cuh"
#include "ptx.cuh"

namespace kd {
namespace {

// Four rows per CTA and at most 56 registers a thread: 36 warps fit on an SM, so the 4832 rows
// of a 32 x 151-token batch run in a single wave (eight-warp CTAs left a short second one).
constexpr int LN_WARPS = 4;

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

template <typename OutT>
__global__ void __launch_bounds__(LN_WARPS * 32, 9) layernorm_kernel(const float* y, OutT* __restrict__ out,
                                                       const float* __restrict__ gamma,
                                                       const float* __restrict__ beta, int M,
                                                       float* __restrict__ stats, L2Prefetch pf) {
  // gamma and beta are weights, which no kernel of the loop writes: they are staged in
  // shared memory before the dependency wait, while the previous kernel drains, so that
  // only the row itself is read after it
  __shared__ float4 sg[D / 4], sb[D / 4];
  for (int i = threadIdx.x; i < D / 4; i += LN_WARPS * 32) {
    sg[i] = reinterpret_cast<const float4*>(gamma)[i];
    sb[i] = reinterpret_cast<const float4*>(beta)[i];
  }
  if (threadIdx.x == 0) ptx::prefetch_l2_share(pf, blockIdx.x, gridDim.x);
  ptx::pdl_wait();
  ptx::pdl_trigger();
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * LN_WARPS + warp;
  if (row >= M) return;
  const float* yr = y + (long)row * D;
  float v[32];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float4 t = *reinterpret_cast<const float4*>(yr + i * 128 + lane * 4);
    v[4 * i] = t.x; v[4 * i + 1] = t.y; v[4 * i + 2] = t.z; v[4 * i + 3] = t.w;
  }
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < 32; ++i) s += v[i];
  const float mean = warp_sum(s) * (1.0f / D);
  float q = 0.f;
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const float d = v[i] - mean;
    q += d * d;
  }
  const float rstd = 1.0f / sqrtf(warp_sum(q) * (1.0f / D) + 1e-5f);
  if (stats != nullptr && lane == 0) *reinterpret_cast<float2*>(stats + 2 * (long)row) = make_float2(mean, rstd);
  OutT* orow = out + (long)row * D;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int c = i * 128 + lane * 4;
    const float4 g = sg[c / 4];
    const float4 b = sb[c / 4];
    const float r0 = (v[4 * i] - mean) * rstd * g.x + b.x;
    const float r1 = (v[4 * i + 1] - mean) * rstd * g.y + b.y;
    const float r2 = (v[4 * i + 2] - mean) * rstd * g.z + b.z;
    const float r3 = (v[4 * i + 3] - mean) * rstd * g.w + b.w;
    if constexpr (sizeof(OutT) == 2) {
      __nv_bfloat162 p0 = __floats2bfloat162_rn(r0, r1), p1 = __floats2bfloat162_rn(r2, r3);
      uint2 u;
      u.x = *reinterpret_cast<uint32_t*>(&p0);
      u.y = *reinterpret_cast<uint32_t*>(&p1);
      *reinterpret_cast<uint2*>(orow + c) = u;
    } else {
      *reinterpret_cast<float4*>(orow + c) = make_float4(r0, r1, r2, r3);
    }
  }
}

}  // namespace

cudaError_t layernorm(const float* y, void* out, bool out_bf16, const float* gamma, const float* beta, int M,
                      cudaStream_t st, float* stats, L2Prefetch pf) {
  if (M <= 0) return cudaSuccess;
  const int grid = (M + LN_WARPS - 1) / LN_WARPS;
  if (out_bf16)
    return launch_kernel(layernorm_kernel<bf16>, dim3(grid), dim3(LN_WARPS * 32), 0, st, y, static_cast<bf16*>(out), gamma, beta,
                         M, stats, pf);
  return launch_kernel(layernorm_kernel<float>, dim3(grid), dim3(LN_WARPS * 32), 0, st, y, static_cast<float*>(out), gamma, beta,
                       M, stats, pf);
}

}  // namespace kd
