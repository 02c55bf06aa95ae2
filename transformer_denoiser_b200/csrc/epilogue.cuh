// GEMM epilogues for the denoiser's projections.  One accumulator row segment of
// a D = A B^T + bias product becomes the stored output.  Shared by the
// tensor-core (bf16) and SIMT (fp32) GEMMs so both precisions fuse identically.
//
// Row r of every activation matrix is token (seq, pos) = (r / S, r % S); token 0
// of a sequence is the condition token, token j >= 1 is frame j - 1.
#pragma once

#include <type_traits>

#include "common.cuh"

namespace kd {

enum EpiKind : int {
  EPI_BIAS = 0,       // out = acc + b
  EPI_BIAS_GELU = 1,  // out = gelu(acc + b)           (FFN1; exact erf GELU)
  EPI_BIAS_SILU = 2,  // out = silu(acc + b)           (first timestep-MLP layer)
  EPI_BIAS_RESID = 3, // out = acc + b + resid          (attention out-proj, FFN2)
  EPI_INPROJ = 4,     // token 0: cond[seq] + tvec + pe[0];  token j: acc + b + pe[j]
  EPI_OUTPROJ = 5,    // frame tokens only, written as [seq, T, ldo]; padded frames 0
  EPI_BIAS_RESID_LN = 6, // out = acc + b + LN(resid): the residual is the un-normalised sum
                         // z of the previous sub-layer, normalised here from its row
                         // statistics (mean, 1/std) and the LayerNorm's gamma / beta
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
  int S = 1;                     // tokens per sequence (padded layout)
  // packed layout (valid tokens only): sequence s owns rows [tok0[s], tok0[s + 1]) and
  // row_seq[r] is the sequence of row r; both null for the padded layout (row = s * S + pos)
  const int* tok0 = nullptr;
  const int* row_seq = nullptr;
  // EPI_BIAS_RESID_LN: row statistics [M][2] = (mean, 1/std) and the LayerNorm affine [N]
  const float* ln_stats = nullptr;
  const float* ln_g = nullptr;
  const float* ln_b = nullptr;
  int T = 1;                     // frames per sequence (EPI_OUTPROJ)
  int N = 0;                     // valid output columns
  int M = 0;                     // valid rows
};

// erf by Abramowitz & Stegun, Handbook of Mathematical Functions, formula 7.1.26:
// erf(z) = 1 - (a1 t + a2 t^2 + a3 t^3 + a4 t^4 + a5 t^5) exp(-z^2), t = 1 / (1 + p z),
// z >= 0, absolute error <= 1.5e-7; erf is odd.  Cheaper than a full-precision erf
// and far below the bf16 rounding of the GELU output (and the fp32 path's 1e-4).
__device__ __forceinline__ float erf_as7126(float z) {
  const float a = fabsf(z);
  const float t = __fdividef(1.0f, fmaf(0.3275911f, a, 1.0f));
  float p = fmaf(1.061405429f, t, -1.453152027f);
  p = fmaf(p, t, 1.421413741f);
  p = fmaf(p, t, -0.284496736f);
  p = fmaf(p, t, 0.254829592f);
  const float e = exp2f(-a * a * 1.4426950408889634f);
  const float r = fmaf(-p * t, e, 1.0f);
  return copysignf(r, z);
}

// GELU(x) = x Phi(x) = 0.5 x (1 + erf(x / sqrt 2)) (the exact, erf-based GELU).
__device__ __forceinline__ float gelu_erf(float x) {
  return 0.5f * x * (1.0f + erf_as7126(x * 0.70710678118654752f));
}
__device__ __forceinline__ float silu_f(float x) { return x / (1.0f + expf(-x)); }

// ---- packed fp32 pairs (sm_100 f32x2 arithmetic: two lanes of work per instruction)
__device__ __forceinline__ uint64_t pk2(float a, float b) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ void upk2(uint64_t r, float& a, float& b) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(r));
}
__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t mul2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ float rcp_approx(float x) {
  float r;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}

// GELU of two values for the bf16-output tensor-core epilogues, with erf by
// Abramowitz & Stegun formula 7.1.28: for z >= 0,
//   erf(z) = 1 - (1 + a1 z + a2 z^2 + ... + a6 z^6)^-16,  |error| <= 3e-7,
// so GELU(x) = x - h for x >= 0 and h for x < 0, h = 0.5 x (1 + a1|z| + ...)^-16,
// z = x / sqrt 2.  One approximate reciprocal (relative error ~2^-22, x16 by the
// power) and f32x2 arithmetic; the total, a few 1e-6 of |x|, is far below the
// bf16 rounding of the stored result.
__device__ __forceinline__ void gelu2_as7128(float& x0, float& x1) {
  const uint64_t x = pk2(x0, x1);
  const uint64_t a = mul2(x, pk2(0.70710678118654752f, 0.70710678118654752f)) & 0x7FFFFFFF7FFFFFFFull;
  uint64_t p = fma2(a, pk2(0.0000430638f, 0.0000430638f), pk2(0.0002765672f, 0.0002765672f));
  p = fma2(p, a, pk2(0.0001520143f, 0.0001520143f));
  p = fma2(p, a, pk2(0.0092705272f, 0.0092705272f));
  p = fma2(p, a, pk2(0.0422820123f, 0.0422820123f));
  p = fma2(p, a, pk2(0.0705230784f, 0.0705230784f));
  p = fma2(p, a, pk2(1.0f, 1.0f));
  float p0, p1;
  upk2(p, p0, p1);
  uint64_t r = pk2(rcp_approx(p0), rcp_approx(p1));
  r = mul2(r, r);
  r = mul2(r, r);
  r = mul2(r, r);
  r = mul2(r, r);
  const uint64_t h = mul2(mul2(x, pk2(0.5f, 0.5f)), r);
  float h0, h1;
  upk2(h, h0, h1);
  x0 = x0 >= 0.f ? x0 - h0 : h0;
  x1 = x1 >= 0.f ? x1 - h1 : h1;
}

template <typename T> __device__ __forceinline__ float to_f(T v);
template <> __device__ __forceinline__ float to_f<float>(float v) { return v; }
template <> __device__ __forceinline__ float to_f<bf16>(bf16 v) { return __bfloat162float(v); }

template <typename T> __device__ __forceinline__ T from_f(float v);
template <> __device__ __forceinline__ float from_f<float>(float v) { return v; }
template <> __device__ __forceinline__ bf16 from_f<bf16>(float v) { return __float2bfloat16_rn(v); }

// (sequence, position) of token row `row` in either layout.
__device__ __forceinline__ void token_of_row(const EpiParams& e, int row, int& seq, int& pos) {
  if (e.row_seq != nullptr) {
    seq = e.row_seq[row];
    pos = row - e.tok0[seq];
  } else {
    seq = row / e.S;
    pos = row - seq * e.S;
  }
}

// Apply the epilogue to `n` consecutive columns [col0, col0 + n) of row `row`.
// acc[i] holds column col0 + i.  OutT is the stored type, ResT the residual type.
template <int KIND, typename OutT, typename ResT, int NV>
__device__ __forceinline__ void epilogue_row(const EpiParams& e, int row, int col0, const float (&acc)[NV]) {
  if (row >= e.M) return;
  if constexpr (KIND == EPI_OUTPROJ) {
    int seq, pos;
    token_of_row(e, row, seq, pos);
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
      int seq, pos;
      token_of_row(e, row, seq, pos);
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

namespace kd {

// ---------------------------------------------------------------------------
// Coalesced epilogue of the tensor-core GEMM.  A warp owns 32 accumulator rows;
// after tcgen05.ld each thread holds one row's CW consecutive columns.  The warp
// writes them to its shared-memory tile st[32][CW + 4] and then walks the rows
// with lanes along the columns (4 columns per lane), so every global load and
// store of bias, residual, sinusoid table and output is a contiguous row segment.

template <typename OutT>
__device__ __forceinline__ void store4(OutT* p, float a, float b, float c, float d);
template <>
__device__ __forceinline__ void store4<float>(float* p, float a, float b, float c, float d) {
  *reinterpret_cast<float4*>(p) = make_float4(a, b, c, d);
}
template <>
__device__ __forceinline__ void store4<bf16>(bf16* p, float a, float b, float c, float d) {
  __nv_bfloat162 lo = __floats2bfloat162_rn(a, b), hi = __floats2bfloat162_rn(c, d);
  uint2 u;
  u.x = *reinterpret_cast<uint32_t*>(&lo);
  u.y = *reinterpret_cast<uint32_t*>(&hi);
  *reinterpret_cast<uint2*>(p) = u;
}

__device__ __forceinline__ float4 ld4(const float* p) { return *reinterpret_cast<const float4*>(p); }

// Eight values as one 16-byte unit: fp32 stores two units of four, bf16 one unit of eight.
__device__ __forceinline__ uint32_t bf16x2_bits(float a, float b) {
  __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&v);
}

template <int CW>
struct EpiLanes {
  static constexpr int LDE = CW + 4;
  static constexpr int LPR = CW / 4;        // lanes per row
  static constexpr int RPP = 32 / LPR;      // rows per pass
  static constexpr int PASSES = 32 / RPP;
};

// Global operands of one chunk that do not depend on the accumulator (residual
// rows, sinusoid rows), loaded before the accumulator is read so their latency
// overlaps the TMEM load.  Rows past M are clamped for the load only.
template <int KIND, int CW>
__device__ __forceinline__ void epilogue_prefetch(const EpiParams& e, int row0, int col0, int lane,
                                                  float4 (&pre)[EpiLanes<CW>::PASSES], float4& bias4) {
  using Ln = EpiLanes<CW>;
  const int rsub = lane / Ln::LPR;
  const int col = col0 + (lane % Ln::LPR) * 4;
  if (col + 4 <= e.N) {
    bias4 = ld4(e.bias + col);
  } else {
    bias4.x = col < e.N ? e.bias[col] : 0.f;
    bias4.y = col + 1 < e.N ? e.bias[col + 1] : 0.f;
    bias4.z = col + 2 < e.N ? e.bias[col + 2] : 0.f;
    bias4.w = col + 3 < e.N ? e.bias[col + 3] : 0.f;
  }
  if constexpr (KIND == EPI_BIAS_RESID_LN) {
    // bias + beta, summed as the pair GEMM's epilogue sums them
    if (col + 4 <= e.N) {
      const float4 be = ld4(e.ln_b + col);
      bias4.x += be.x; bias4.y += be.y; bias4.z += be.z; bias4.w += be.w;
    }
  }
  if constexpr (KIND == EPI_BIAS_RESID || KIND == EPI_BIAS_RESID_LN || KIND == EPI_INPROJ) {
    if (col + 4 > e.N) return;
#pragma unroll
    for (int p = 0; p < Ln::PASSES; ++p) {
      const int row = min(row0 + p * Ln::RPP + rsub, e.M - 1);
      if constexpr (KIND == EPI_BIAS_RESID || KIND == EPI_BIAS_RESID_LN) {
        pre[p] = ld4(reinterpret_cast<const float*>(e.resid) + (long)row * e.ldr + col);
      } else {
        int seq, pos;
        token_of_row(e, row, seq, pos);
        pre[p] = ld4(e.pe + (long)pos * e.N + col);
      }
    }
  }
}

template <int KIND, typename OutT, int CW>
__device__ __forceinline__ void epilogue_warp_tile(const EpiParams& e, const float* st, int row0, int col0,
                                                   int lane, const float4 (&pre)[EpiLanes<CW>::PASSES],
                                                   const float4 bias4) {
  using Ln = EpiLanes<CW>;
  const int rsub = lane / Ln::LPR;
  const int cq = (lane % Ln::LPR) * 4;
  const int col = col0 + cq;
  if (col >= e.N) return;
  const bool full = col + 4 <= e.N;  // all 4 columns valid (N % 4 != 0 only at the output projection)
  const float b4[4] = {bias4.x, bias4.y, bias4.z, bias4.w};
#pragma unroll
  for (int p = 0; p < Ln::PASSES; ++p) {
    const int r = p * Ln::RPP + rsub;
    const int row = row0 + r;
    const bool in_rows = row < e.M;
    const float4 a = *reinterpret_cast<const float4*>(st + r * Ln::LDE + cq);
    float v[4] = {a.x, a.y, a.z, a.w};
    if constexpr (KIND == EPI_OUTPROJ) {
      int seq = 0, pos = 0;
      if (in_rows) token_of_row(e, row, seq, pos);
      if (in_rows && pos != 0) {
        const int frame = pos - 1;
        const bool valid = frame < e.lengths[seq % e.len_mod];
        OutT* o = reinterpret_cast<OutT*>(e.out) + ((long)seq * e.T + frame) * e.ldo + col;
#pragma unroll
        for (int j = 0; j < 4; ++j)
          if (col + j < e.N) o[j] = from_f<OutT>(valid ? v[j] + b4[j] : 0.f);
      }
    } else {
      if constexpr (KIND == EPI_INPROJ) {
        int seq = 0, pos = 1;
        if (in_rows) token_of_row(e, row, seq, pos);
        if (pos == 0) {
          const float4 cv = ld4(e.cond + (long)seq * e.N + col);
          const float4 tv = ld4(e.tvec + col);
          const float4 pv = ld4(e.pe + col);
          v[0] = cv.x + tv.x + pv.x; v[1] = cv.y + tv.y + pv.y;
          v[2] = cv.z + tv.z + pv.z; v[3] = cv.w + tv.w + pv.w;
        } else {
          const float4 pv = pre[p];
          v[0] += b4[0] + pv.x; v[1] += b4[1] + pv.y; v[2] += b4[2] + pv.z; v[3] += b4[3] + pv.w;
        }
        if (in_rows && e.out32 != nullptr) store4<float>(e.out32 + (long)row * e.ldo + col, v[0], v[1], v[2], v[3]);
      } else {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          float x = v[j] + b4[j];
          if constexpr (KIND == EPI_BIAS_SILU) x = silu_f(x);
          v[j] = x;
        }
        if constexpr (KIND == EPI_BIAS_GELU) {
          // bf16 outputs take the packed GELU of the pair GEMM, fp32 outputs the A&S 7.1.26 one
          if constexpr (std::is_same<OutT, bf16>::value) {
            gelu2_as7128(v[0], v[1]);
            gelu2_as7128(v[2], v[3]);
          } else {
#pragma unroll
            for (int j = 0; j < 4; ++j) v[j] = gelu_erf(v[j]);
          }
        }
        if constexpr (KIND == EPI_BIAS_RESID) {
          v[0] += pre[p].x; v[1] += pre[p].y; v[2] += pre[p].z; v[3] += pre[p].w;
        }
        if constexpr (KIND == EPI_BIAS_RESID_LN) {
          // the residual is the un-normalised sum z: add gamma (z - mean) / std (+ beta, in b4)
          const float2 st2 = *reinterpret_cast<const float2*>(e.ln_stats + 2 * (long)min(row, e.M - 1));
          const float ra = st2.y, rb = -st2.x * st2.y;
          const float4 g4 = ld4(e.ln_g + col);
          v[0] += fmaf(pre[p].x, ra, rb) * g4.x; v[1] += fmaf(pre[p].y, ra, rb) * g4.y;
          v[2] += fmaf(pre[p].z, ra, rb) * g4.z; v[3] += fmaf(pre[p].w, ra, rb) * g4.w;
        }
      }
      if (in_rows) {
        OutT* o = reinterpret_cast<OutT*>(e.out) + (long)row * e.ldo + col;
        if (full) {
          store4<OutT>(o, v[0], v[1], v[2], v[3]);
        } else {
          for (int j = 0; j < 4; ++j)
            if (col + j < e.N) o[j] = from_f<OutT>(v[j]);
        }
      }
    }
  }
}

}  // namespace kd
