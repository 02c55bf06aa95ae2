/*
 * kimodo_kernels.h -- kernel-level entry points of libkimodo.so.
 *
 * Each call runs exactly one of the kernels that kimodo.h's entry points chain
 * together, so that each can be checked on its own against a reference of the
 * same operation.  All tensor pointers are DEVICE pointers of the current CUDA
 * device, row-major; calls are asynchronous on `stream` (a cudaStream_t, NULL =
 * legacy default stream).  Return value and error message as in kimodo.h
 * (KIMODO_OK or KIMODO_E*, kimodo_last_error()).  The caller owns all memory.
 */
#ifndef KIMODO_KERNELS_H
#define KIMODO_KERNELS_H

#include "kimodo.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Epilogues of the projections ("Kimodo WebGPU", "WGSL compute shaders" table:
 * linear + bias, GELU, SiLU, residual add). */
enum {
  KIMODO_EPI_BIAS = 0,      /* out = A W^T + b                      */
  KIMODO_EPI_BIAS_GELU = 1, /* out = gelu_erf(A W^T + b)            */
  KIMODO_EPI_BIAS_SILU = 2, /* out = silu(A W^T + b)                */
  KIMODO_EPI_BIAS_RESID = 3 /* out = A W^T + b + resid (fp32 out)   */
};

/*
 * Tensor-core (tcgen05) GEMM, bf16 operands, fp32 accumulation:
 *   out[M, N] = epilogue(A[M, K] W[N, K]^T + bias[N]).
 * A: bf16, row stride lda elements; W: bf16, row stride ldw; both 16-byte
 * aligned with lda, ldw multiples of 8 and >= K.  bias: fp32 [N].
 * resid: fp32 [M, ldr] (KIMODO_EPI_BIAS_RESID only, else NULL); may equal out.
 * out: bf16 (out_f32 = 0) or fp32 (out_f32 = 1), row stride ldo.
 * out, resid, bias 16-byte aligned; ldo, ldr multiples of 4.
 * KIMODO_EPI_BIAS_RESID requires out_f32 = 1.  tile_n: 32, 64, 128 or 256
 * (output columns per tile; 32 and 64 are built for the bias and GELU epilogues
 * with bf16 output and the residual epilogue), or 0 to let the library choose.
 */
KIMODO_API int kimodo_gemm_bf16(const void* A, int lda, const void* W, int ldw, const float* bias,
                                const void* resid, int ldr, void* out, int ldo, int M, int N, int K,
                                int epilogue, int out_f32, int tile_n, void* stream);

/*
 * The same product on pairs of SMs (one 256-row output tile per CTA pair,
 * tcgen05 cta_group::2), the kernel the denoiser uses for its large projections.
 * Arguments as kimodo_gemm_bf16; epilogues KIMODO_EPI_BIAS and KIMODO_EPI_BIAS_GELU
 * with bf16 output and KIMODO_EPI_BIAS_RESID with fp32 output; N % 16 == 0 and output
 * rows a multiple of 16 bytes.  tile_n: output
 * columns per pair tile, 144, 160, 208 or 256 (144 or 160 with the residual
 * epilogue), or 0 for the library's choice.
 */
KIMODO_API int kimodo_gemm_bf16_pair(const void* A, int lda, const void* W, int ldw, const float* bias,
                                     const void* resid, int ldr, void* out, int ldo, int M, int N, int K,
                                     int epilogue, int out_f32, int tile_n, void* stream);

/* fp32 SIMT GEMM with the same epilogues; all operands fp32; K % 16 == 0,
 * lda, ldw multiples of 4. */
KIMODO_API int kimodo_gemm_f32(const float* A, int lda, const float* W, int ldw, const float* bias,
                               const float* resid, int ldr, float* out, int ldo, int M, int N, int K,
                               int epilogue, void* stream);

/*
 * Masked multi-head self-attention ("Kimodo WebGPU", "WGSL compute shaders":
 * multi-head self-attention with optional key masking), 8 heads x 128.
 * qkv: [nseq * S, 3072] with columns Q | K | V (head h at h * 128 inside each).
 * Sequence s attends to keys 0 .. lengths[s] (the condition token plus
 * lengths[s] frames; clamped to [1, S] keys).  out: [nseq * S, 1024].
 * 1 <= S <= 301.
 * bf16 variant: bf16 qkv/out (qkv 16-byte aligned), on the tcgen05 tensor cores:
 *   one CTA per (head, sequence, 128-query tile), S = Q K^T and O = P V in TMEM,
 *   exact fp32 softmax over all keys of a sequence.
 * f32 variant: fp32 throughout (SIMT, one warp per query).
 */
KIMODO_API int kimodo_attention_bf16(const void* qkv, void* out, const int* lengths, int nseq, int S,
                                     void* stream);
KIMODO_API int kimodo_attention_f32(const float* qkv, float* out, const int* lengths, int nseq, int S,
                                    void* stream);

/* LayerNorm over 1024 features, eps 1e-5, biased variance: y fp32 [M, 1024] ->
 * out bf16 (out_bf16 = 1) or fp32 [M, 1024]; gamma, beta fp32 [1024]. */
KIMODO_API int kimodo_layernorm(const float* y, void* out, int out_bf16, const float* gamma,
                                const float* beta, int M, void* stream);

/*
 * globalRootToLocalRoot and the body network's input ("Kimodo WebGPU",
 * "Architecture" figure: root model -> globalRootToLocalRoot -> body model), the
 * fp32 form of the kernel the two-stage step runs between its two networks.
 * root: [batch, frames, 5] global root (x, z, sin heading, cos heading, height), the
 *   root network's output for one guidance branch.  x: [batch, frames, 279] state x_t.
 * body_in (output): [batch, frames, 279] = [x[..., 5:279] | local root 5], local root =
 *   (v'x, v'z, sin d, cos d, height): the displacement from the previous frame turned
 *   into the current heading's frame, the heading change, the height; headings are
 *   normalised, and the frame before the first sits at the origin with heading 0.
 *   Frames at index >= lengths[b] get local root 0 (their body columns are copied).
 * lengths: int32 [batch], 1..frames.  1 <= batch, 1 <= frames <= 300.
 */
KIMODO_API int kimodo_global_to_local_root(const float* root, const float* x, const int* lengths, int batch,
                                           int frames, float* body_in, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* KIMODO_KERNELS_H */
