// GEMM epilogues for the denoiser's projections.  One accumulator row segment of
// a D = A B^T + bias product becomes the stored output.  Shared by the
// tensor-core (bf16) and SIMT (fp32) GEMMs so both precisions fuse identically.
//
// Row r of every activation matrix is token (seq, pos) = (r / S, r % S); token 0
// of a sequence is the condition token, token j >= 1 is frame j - 1.
#pragma once

#include "common.cuh"

namespace kd {

enum EpiKind : int {
  EPI_BIAS = 0,       // out = acc + b
  EPI_BIAS_GELU = 1,  // out = gelu(acc + b)           (FFN1; exact erf GELU)
  EPI_BIAS_SILU = 2,  // out = silu(acc + b)           (first timestep-MLP layer)
  EPI_BIAS_RESID = 3, // out = acc + b + resid          (attention out-proj, FFN2)
  EPI_INPROJ = 4,     // token 0: cond[seq] + tvec + pe[0];  token j: acc + b + pe[j]
  EPI_OUTPROJ = 5,    // frame tokens only, written as [seq, T, ldo]; padded frames 0
};

struct EpiParams {
  const float* bias = nullptr;   // [N]
  void* out = nullptr;           // output base
  long ldo = 0;                  // output row stride (elements)
  const void* resid = nullptr;   // residual [M, ldr]; may alias `out` (read before write, per element)
  long ldr = 0;
  float* out32 = nullptr;        // EPI_INPROJ: optional fp32 copy of the tokens (row stride ldo)
  const float* pe = nullptr;     // sinusoid table [position, N]
  const float* cond = nullptr;   // text projection [nseq, N]
  const float* tvec = nullptr;   // timestep-MLP output [N] for this call's timestep
  const int* lengths = nullptr;  // valid frames per sequence, indexed seq % len_mod
  int len_mod = 1;
  int S = 1;                     // tokens per sequence
  int T = 1;                     // frames per sequence (EPI_OUTPROJ)
  int N = 0;                     // valid output columns
  int M = 0;                     // valid rows
};

__device__ __forceinline__ float gelu_erf(float x) {
  return 0.5f * x * (1.0f + erff(x * 0.70710678118654752f));
}
__device__ __forceinline__ float silu_f(float x) { return x / (1.0f + expf(-x)); }

template <typename T> __device__ __forceinline__ float to_f(T v);
template <> __device__ __forceinline__ float to_f<float>(float v) { return v; }
template <> __device__ __forceinline__ float to_f<bf16>(bf16 v) { return __bfloat162float(v); }

template <typename T> __device__ __forceinline__ T from_f(float v);
template <> __device__ __forceinline__ float from_f<float>(float v) { return v; }
template <> __device__ __forceinline__ bf16 from_f<bf16>(float v) { return __float2bfloat16_rn(v); }

// Apply the epilogue to `n` consecutive columns [col0, col0 + n) of row `row`.
// acc[i] holds column col0 + i.  OutT is the stored type, ResT the residual type.
template <int KIND, typename OutT, typename ResT, int NV>
__device__ __forceinline__ void epilogue_row(const EpiParams& e, int row, int col0, const float (&acc)[NV]) {
  if (row >= e.M) return;
  if constexpr (KIND == EPI_OUTPROJ) {
    const int seq = row / e.S, pos = row - seq * e.S;
    if (pos == 0) return;
    const int frame = pos - 1;
    const bool valid = frame < e.lengths[seq % e.len_mod];
    OutT* o = reinterpret_cast<OutT*>(e.out) + ((long)seq * e.T + frame) * e.ldo;
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      const int c = col0 + i;
      if (c < e.N) o[c] = from_f<OutT>(valid ? acc[i] + e.bias[c] : 0.0f);
    }
    return;
  } else {
    float v[NV];
    if constexpr (KIND == EPI_INPROJ) {
      const int seq = row / e.S, pos = row - seq * e.S;
      if (pos == 0) {
#pragma unroll
        for (int i = 0; i < NV; ++i) {
          const int c = min(col0 + i, e.N - 1);
          v[i] = e.cond[(long)seq * e.N + c] + e.tvec[c] + e.pe[c];
        }
      } else {
#pragma unroll
        for (int i = 0; i < NV; ++i) {
          const int c = min(col0 + i, e.N - 1);
          v[i] = acc[i] + e.bias[c] + e.pe[(long)pos * e.N + c];
        }
      }
    } else {
#pragma unroll
      for (int i = 0; i < NV; ++i) {
        const int c = min(col0 + i, e.N - 1);
        float x = acc[i] + e.bias[c];
        if constexpr (KIND == EPI_BIAS_GELU) x = gelu_erf(x);
        if constexpr (KIND == EPI_BIAS_SILU) x = silu_f(x);
        if constexpr (KIND == EPI_BIAS_RESID)
          x += to_f<ResT>(reinterpret_cast<const ResT*>(e.resid)[(long)row * e.ldr + c]);
        v[i] = x;
      }
    }
    if constexpr (KIND == EPI_INPROJ) {
      if (e.out32 != nullptr) {
        float* o32 = e.out32 + (long)row * e.ldo + col0;
#pragma unroll
        for (int i = 0; i < NV; ++i)
          if (col0 + i < e.N) o32[i] = v[i];
      }
    }
    OutT* o = reinterpret_cast<OutT*>(e.out) + (long)row * e.ldo + col0;
    constexpr int VEC = 16 / sizeof(OutT);
    if (NV % VEC == 0 && col0 + NV <= e.N && (((uintptr_t)o) & 15) == 0) {
#pragma unroll
      for (int i = 0; i < NV; i += VEC) {
        OutT tmp[VEC];
#pragma unroll
        for (int j = 0; j < VEC; ++j) tmp[j] = from_f<OutT>(v[i + j]);
        *reinterpret_cast<uint4*>(o + i) = *reinterpret_cast<const uint4*>(tmp);
      }
    } else {
#pragma unroll
      for (int i = 0; i < NV; ++i)
        if (col0 + i < e.N) o[i] = from_f<OutT>(v[i]);
    }
  }
}

}  // namespace kd
