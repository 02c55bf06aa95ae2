// Masked multi-head self-attention ("Kimodo WebGPU", "WGSL compute shaders"
// table: multi-head self-attention with optional key masking).
//
// Per (sequence, head) the keys 0..n_valid-1 take part, n_valid = 1 + length
// (the condition token is always valid).  Keys at or beyond n_valid are never
// loaded: their shared-memory rows are zero-filled and their scores are set to
// -inf by selection, so padded content (even NaN) cannot reach an output.
//
// bf16 kernel: one CTA per (head, sequence) with one warp per 16-query block (at
// most 12 warps, which then loop).  K and V of the valid keys are staged once in
// shared memory (row stride 136 bf16 to keep ldmatrix conflict-free); Q K^T and
// P V run on mma.sync m16n8k16 (bf16 in, fp32 accumulate) with an online softmax
// over 32-key blocks whose row max / sum are reduced across the 4-thread quads by
// warp shuffles.
//
// fp32 kernel (fp32 path): one warp per query row, scores by warp-shuffle dot
// products, online softmax in fp32.
#include <cuda_runtime.h>
#include <math.h>

#include "common.cuh"
#include "kernels.h"
#include "launch.cuh"
#include "ptx.cuh"

namespace kd {
namespace {

constexpr int KBLK = 32;
constexpr int ATT_MAX_WARPS = 12;
constexpr int LDS = DH + 8;   // smem row stride in bf16 elements

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// One CTA per (head, sequence); warp w handles query blocks w, w + nwarps, ... of
// 16 rows.  Q fragments are read straight from global memory into registers; K and
// V of the valid keys (rounded up to 32) sit in shared memory for all warps.
__global__ void __launch_bounds__(ATT_MAX_WARPS * 32, 1)
attn_bf16_kernel(const bf16* __restrict__ qkv, bf16* __restrict__ out, const int* __restrict__ lengths,
                 int len_mod, int S_pad, const int* __restrict__ tok0) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  ptx::pdl_wait();
  ptx::pdl_trigger();
  const int h = blockIdx.x, seq = blockIdx.y;
  // rows of this sequence: padded layout seq * S_pad + [0, S_pad), packed layout [tok0[seq], tok0[seq + 1])
  const long row0 = tok0 ? tok0[seq] : (long)seq * S_pad;
  const int S = tok0 ? tok0[seq + 1] - tok0[seq] : S_pad;
  int n_valid = 1 + lengths[seq % len_mod];
  n_valid = n_valid < 1 ? 1 : (n_valid > S ? S : n_valid);
  const int nkb = (n_valid + KBLK - 1) / KBLK;
  bf16* sK = reinterpret_cast<bf16*>(smem_raw);
  bf16* sV = sK + nkb * KBLK * LDS;

  const long rs = 3L * D;
  const bf16* base = qkv + row0 * rs + h * DH;
  const int tid = threadIdx.x, nthr = blockDim.x;
  for (int c = tid; c < nkb * KBLK * 16; c += nthr) {
    const int r = c >> 4, ch = c & 15;
    const bool v = r < n_valid;
    const bf16* src = base + (long)(v ? r : 0) * rs + ch * 8;
    ptx::cp_async_16_zfill(ptx::smem_u32(sK + r * LDS + ch * 8), src + D, v);
    ptx::cp_async_16_zfill(ptx::smem_u32(sV + r * LDS + ch * 8), src + 2 * D, v);
  }
  ptx::cp_async_commit();

  const int warp = tid >> 5, lane = tid & 31, nwarps = nthr >> 5;
  const int g = lane >> 2, c4 = lane & 3;
  const int nqb = (S + 15) / 16;
  const float scale = 0.08838834764831845f * 1.4426950408889634f;  // 1/sqrt(128) * log2(e)
  ptx::cp_async_wait_all();
  __syncthreads();

  for (int qb = warp; qb < nqb; qb += nwarps) {
    const int qw = qb * 16;
    // Q fragments of this warp's 16 rows for the 8 k-steps of the 128-wide head
    uint32_t qf[8][4];
    {
      const int r0 = qw + g, r1 = qw + g + 8;
      const uint32_t* q0 = reinterpret_cast<const uint32_t*>(base + (long)min(r0, S - 1) * rs);
      const uint32_t* q1 = reinterpret_cast<const uint32_t*>(base + (long)min(r1, S - 1) * rs);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const int w0 = kk * 8 + c4;   // 32-bit word index: dims kk*16 + 2*c4 (+1)
        qf[kk][0] = r0 < S ? q0[w0] : 0u;
        qf[kk][1] = r1 < S ? q1[w0] : 0u;
        qf[kk][2] = r0 < S ? q0[w0 + 4] : 0u;
        qf[kk][3] = r1 < S ? q1[w0 + 4] : 0u;
      }
    }
    float o[16][4];
#pragma unroll
    for (int n = 0; n < 16; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;

    for (int kb = 0; kb < nkb; ++kb) {
      float sc[4][4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        sc[j][0] = sc[j][1] = sc[j][2] = sc[j][3] = 0.f;
        const int key = kb * KBLK + j * 8 + (lane & 7);
#pragma unroll
        for (int kk2 = 0; kk2 < 4; ++kk2) {
          uint32_t b0, b1, b2, b3;
          ldsm_x4(ptx::smem_u32(sK + key * LDS + kk2 * 32 + (lane >> 3) * 8), b0, b1, b2, b3);
          mma_bf16(sc[j], qf[2 * kk2], b0, b1);
          mma_bf16(sc[j], qf[2 * kk2 + 1], b2, b3);
        }
      }
      float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int key = kb * KBLK + j * 8 + 2 * c4;
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const bool ok = key + e < n_valid;
          sc[j][e] = ok ? sc[j][e] * scale : -INFINITY;
          sc[j][e + 2] = ok ? sc[j][e + 2] * scale : -INFINITY;
          mx0 = fmaxf(mx0, sc[j][e]);
          mx1 = fmaxf(mx1, sc[j][e + 2]);
        }
      }
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
      const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
      const float a0 = exp2f(m0 - mn0), a1 = exp2f(m1 - mn1);
      m0 = mn0;
      m1 = mn1;
      float rs0 = 0.f, rs1 = 0.f;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        sc[j][0] = exp2f(sc[j][0] - mn0);
        sc[j][1] = exp2f(sc[j][1] - mn0);
        sc[j][2] = exp2f(sc[j][2] - mn1);
        sc[j][3] = exp2f(sc[j][3] - mn1);
        rs0 += sc[j][0] + sc[j][1];
        rs1 += sc[j][2] + sc[j][3];
      }
      l0 = l0 * a0 + rs0;
      l1 = l1 * a1 + rs1;
#pragma unroll
      for (int n = 0; n < 16; ++n) {
        o[n][0] *= a0; o[n][1] *= a0;
        o[n][2] *= a1; o[n][3] *= a1;
      }
      // O += P V over the two sixteen-key slices of this block
#pragma unroll
      for (int kk = 0; kk < 2; ++kk) {
        uint32_t pf[4];
        pf[0] = pack_bf16(sc[2 * kk][0], sc[2 * kk][1]);
        pf[1] = pack_bf16(sc[2 * kk][2], sc[2 * kk][3]);
        pf[2] = pack_bf16(sc[2 * kk + 1][0], sc[2 * kk + 1][1]);
        pf[3] = pack_bf16(sc[2 * kk + 1][2], sc[2 * kk + 1][3]);
        const int key = kb * KBLK + kk * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
        for (int dp = 0; dp < 8; ++dp) {
          uint32_t b0, b1, b2, b3;
          ldsm_x4_t(ptx::smem_u32(sV + key * LDS + dp * 16 + (lane >> 4) * 8), b0, b1, b2, b3);
          mma_bf16(o[2 * dp], pf, b0, b1);
          mma_bf16(o[2 * dp + 1], pf, b2, b3);
        }
      }
    }
    l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
    l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
    const float i0 = 1.f / l0, i1 = 1.f / l1;
    const int r0 = qw + g, r1 = qw + g + 8;
    bf16* ob = out + row0 * D + h * DH + 2 * c4;
#pragma unroll
    for (int n = 0; n < 16; ++n) {
      if (r0 < S)
        *reinterpret_cast<__nv_bfloat162*>(ob + (long)r0 * D + n * 8) = __floats2bfloat162_rn(o[n][0] * i0, o[n][1] * i0);
      if (r1 < S)
        *reinterpret_cast<__nv_bfloat162*>(ob + (long)r1 * D + n * 8) = __floats2bfloat162_rn(o[n][2] * i1, o[n][3] * i1);
    }
  }
}

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

size_t attention_bf16_smem(int S) {
  const int nk = ((S + KBLK - 1) / KBLK) * KBLK;
  return (size_t)(2 * nk) * LDS * sizeof(bf16);
}

cudaError_t attention_bf16(const bf16* qkv, bf16* out, const int* lengths, int len_mod, int nseq, int S,
                           cudaStream_t st, const int* tok0) {
  if (nseq <= 0 || S <= 0) return cudaSuccess;
  const size_t smem = attention_bf16_smem(S);
  int warps = (S + 15) / 16;
  warps = warps > ATT_MAX_WARPS ? ATT_MAX_WARPS : warps;
  dim3 grid(H, nseq);
  return launch_kernel(attn_bf16_kernel, grid, dim3(32 * warps), smem, st, qkv, out, lengths, len_mod, S, tok0);
}

cudaError_t attention_prepare() {
  return cudaFuncSetAttribute(attn_bf16_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              (int)attention_bf16_smem(MAX_FRAMES + 1));
}

cudaError_t attention_f32(const float* qkv, float* out, const int* lengths, int len_mod, int nseq, int S,
                          cudaStream_t st, const int* tok0) {
  if (nseq <= 0 || S <= 0) return cudaSuccess;
  dim3 grid((S + 3) / 4, H, nseq);
  return launch_kernel(attn_f32_kernel, grid, dim3(128), 0, st, qkv, out, lengths, len_mod, S, tok0);
}

}  // namespace kd
