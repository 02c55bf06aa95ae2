// fp32 SIMT GEMM for the fp32 precision path: D = A . B^T + epilogue, fp32
// operands and accumulation (tcgen05 has no fp32 kind, and tf32 rounding would
// exceed the fp32 path's 1e-4 tolerance).  64x64 tile, 256 threads, 4x4 outputs
// per thread, K in steps of 16 staged through shared memory.
#include <cuda_runtime.h>

#include "common.cuh"
#include "epilogue.cuh"
#include "kernels.h"
#include "launch.cuh"
#include "ptx.cuh"

namespace kd {
namespace {

constexpr int TM = 64, TN = 64, TK = 16;

template <int KIND>
__global__ void __launch_bounds__(256) gemm_f32_kernel(const float* __restrict__ A, const float* __restrict__ B,
                                                       int M, int N, int K, int lda, int ldb, EpiParams ep) {
  __shared__ __align__(16) float As[TK][TM + 4];
  __shared__ __align__(16) float Bs[TK][TN + 4];
  ptx::pdl_wait();
  ptx::pdl_trigger();
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const int m0 = blockIdx.y * TM, n0 = blockIdx.x * TN;
  float acc[4][4] = {};
  const int lr = tid >> 2, lk = (tid & 3) * 4;   // loader: row, k offset
  for (int k0 = 0; k0 < K; k0 += TK) {
    {
      const int m = m0 + lr;
      float4 a = m < M ? *reinterpret_cast<const float4*>(A + (long)m * lda + k0 + lk) : make_float4(0, 0, 0, 0);
      As[lk + 0][lr] = a.x; As[lk + 1][lr] = a.y; As[lk + 2][lr] = a.z; As[lk + 3][lr] = a.w;
      const int n = n0 + lr;
      float4 b = n < N ? *reinterpret_cast<const float4*>(B + (long)n * ldb + k0 + lk) : make_float4(0, 0, 0, 0);
      Bs[lk + 0][lr] = b.x; Bs[lk + 1][lr] = b.y; Bs[lk + 2][lr] = b.z; Bs[lk + 3][lr] = b.w;
    }
    __syncthreads();
#pragma unroll
    for (int k = 0; k < TK; ++k) {
      const float4 a = *reinterpret_cast<const float4*>(&As[k][ty * 4]);
      const float4 b = *reinterpret_cast<const float4*>(&Bs[k][tx * 4]);
      const float av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
    __syncthreads();
  }
  const int col0 = n0 + tx * 4;
  if (col0 >= ep.N) return;
#pragma unroll
  for (int i = 0; i < 4; ++i) epilogue_row<KIND, float, float, 4>(ep, m0 + ty * 4 + i, col0, acc[i]);
}

}  // namespace

cudaError_t gemm_f32(const GemmArgs& g, int kind, const EpiParams& ep, cudaStream_t st) {
  if (g.M <= 0 || g.N <= 0) return cudaSuccess;
  if (g.K % TK || g.lda % 4 || g.ldb % 4) return cudaErrorInvalidValue;
  dim3 grid((g.N + TN - 1) / TN, (g.M + TM - 1) / TM);
  const float* A = static_cast<const float*>(g.A);
  const float* B = static_cast<const float*>(g.B);
  switch (kind) {
    case EPI_BIAS: return launch_kernel(gemm_f32_kernel<EPI_BIAS>, grid, dim3(256), 0, st, A, B, g.M, g.N, g.K, g.lda, g.ldb, ep);
    case EPI_BIAS_GELU: return launch_kernel(gemm_f32_kernel<EPI_BIAS_GELU>, grid, dim3(256), 0, st, A, B, g.M, g.N, g.K, g.lda, g.ldb, ep);
    case EPI_BIAS_SILU: return launch_kernel(gemm_f32_kernel<EPI_BIAS_SILU>, grid, dim3(256), 0, st, A, B, g.M, g.N, g.K, g.lda, g.ldb, ep);
    case EPI_BIAS_RESID: return launch_kernel(gemm_f32_kernel<EPI_BIAS_RESID>, grid, dim3(256), 0, st, A, B, g.M, g.N, g.K, g.lda, g.ldb, ep);
    case EPI_INPROJ: return launch_kernel(gemm_f32_kernel<EPI_INPROJ>, grid, dim3(256), 0, st, A, B, g.M, g.N, g.K, g.lda, g.ldb, ep);
    case EPI_OUTPROJ: return launch_kernel(gemm_f32_kernel<EPI_OUTPROJ>, grid, dim3(256), 0, st, A, B, g.M, g.N, g.K, g.lda, g.ldb, ep);
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace kd
