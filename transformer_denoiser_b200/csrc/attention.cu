// Masked multi-head self-attention of the fp32 path ("Kimodo WebGPU", "WGSL compute
// shaders" table: multi-head self-attention with optional key masking).
//
// Per (sequence, head) the keys 0..n_valid-1 take part, n_valid = 1 + length
// (the condition token is always valid).  Keys at or beyond n_valid are never
// read, so padded content (even NaN) cannot reach an output.
//
// One warp per query row: scores by warp-shuffle dot products (4 dimensions per
// lane), online softmax in fp32.  The bf16 path runs the tcgen05 kernel of
// attention_tc.cu instead.
#include <cuda_runtime.h>
#include <math.h>

#include "common.cuh"
#include "kernels.h"
#include "launch.cuh"
#include "ptx.cuh"

namespace kd {
namespace {

__global__ void __launch_bounds__(128) attn_f32_kernel(const float* __restrict__ qkv, float* __restrict__ out,
                                                       const int* __restrict__ lengths, int len_mod, int S_pad,
                                                       const int* __restrict__ tok0) {
  ptx::pdl_wait();
  ptx::pdl_trigger();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int q = blockIdx.x * 4 + warp, h = blockIdx.y, seq = blockIdx.z;
  const long row0 = tok0 ? tok0[seq] : (long)seq * S_pad;
  const int S = tok0 ? tok0[seq + 1] - tok0[seq] : S_pad;
  if (q >= S) return;
  int n_valid = 1 + lengths[seq % len_mod];
  n_valid = n_valid < 1 ? 1 : (n_valid > S ? S : n_valid);
  const long rs = 3L * D;
  const float* base = qkv + row0 * rs + h * DH + lane * 4;
  const float4 qv = *reinterpret_cast<const float4*>(base + (long)q * rs);
  const float scale = 0.08838834764831845f;
  float m = -INFINITY, l = 0.f;
  float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int j = 0; j < n_valid; ++j) {
    const float4 kv = *reinterpret_cast<const float4*>(base + (long)j * rs + D);
    float d = qv.x * kv.x + qv.y * kv.y + qv.z * kv.z + qv.w * kv.w;
#pragma unroll
    for (int off = 16; off; off >>= 1) d += __shfl_xor_sync(0xffffffffu, d, off);
    const float sc = d * scale;
    const float mn = fmaxf(m, sc);
    const float a = expf(m - mn), p = expf(sc - mn);
    const float4 vv = *reinterpret_cast<const float4*>(base + (long)j * rs + 2 * D);
    l = l * a + p;
    o.x = o.x * a + p * vv.x;
    o.y = o.y * a + p * vv.y;
    o.z = o.z * a + p * vv.z;
    o.w = o.w * a + p * vv.w;
    m = mn;
  }
  const float inv = 1.f / l;
  *reinterpret_cast<float4*>(out + (row0 + q) * D + h * DH + lane * 4) =
      make_float4(o.x * inv, o.y * inv, o.z * inv, o.w * inv);
}

}  // namespace

cudaError_t attention_f32(const float* qkv, float* out, const int* lengths, int len_mod, int nseq, int S,
                          cudaStream_t st, const int* tok0) {
  if (nseq <= 0 || S <= 0) return cudaSuccess;
  dim3 grid((S + 3) / 4, H, nseq);
  return launch_kernel(attn_f32_kernel, grid, dim3(128), 0, st, qkv, out, lengths, len_mod, S, tok0);
}

}  // namespace kd
