// Internal launchers of the denoiser kernels (not part of the public C ABI).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include "common.cuh"
#include "epilogue.cuh"

namespace kd {

// D[M, N] = A[M, K] . B[N, K]^T; A, B row-major with leading dimensions lda, ldb.
struct GemmArgs {
  const void* A = nullptr;
  const void* B = nullptr;
  int M = 0, N = 0, K = 0;
  int lda = 0, ldb = 0;
};

// tcgen05 bf16 GEMM.  bn in {16, 32, 64, 128, 256}; returns cudaErrorInvalidValue for an
// unsupported (bn, kind, output type) combination.
cudaError_t gemm_tc(const GemmArgs& g, int bn, int kind, bool out_f32, const EpiParams& ep, DevError* err,
                    cudaStream_t st, int num_sms);
bool gemm_tc_available();

// TMA descriptor of a row-major bf16 matrix [rows, ld] whose first `cols` columns are
// the K extent; boxes of 64 columns x box_rows rows, 128-byte swizzle, zero fill.
int make_tmap_bf16(CUtensorMap* m, const void* base, int rows, int cols, int ld, int box_rows);
// Row-major fp32 (elem 4) or bf16 (elem 2) matrix, boxes box_cols x box_rows,
// shared-memory swizzle 0, 32, 64 or 128 bytes (= the box row's bytes when nonzero).
int make_tmap_plain(CUtensorMap* m, const void* base, int elem, int rows, int cols, long ld, int box_cols,
                    int box_rows, int swizzle);

// tcgen05 GEMM on CTA pairs (256-row tiles).  bn in {144, 160, 208, 256} for EPI_BIAS /
// EPI_BIAS_GELU with bf16 output, {144, 160} for EPI_BIAS_RESID / EPI_BIAS_RESID_LN with
// fp32 output.
cudaError_t gemm_tc2(const GemmArgs& g, int bn, int kind, bool out_f32, const EpiParams& ep, DevError* err,
                     cudaStream_t st);
cudaError_t gemm_tc2_prepare();
bool gemm_tc2_supports(int kind, bool out_f32);
int gemm_tc2_pick_bn(int M, int N, int kind);
// Set the dynamic shared-memory limits of every kernel instantiation (call once
// per device before any launch or graph capture).
cudaError_t gemm_tc_prepare();

// fp32 SIMT GEMM with the same epilogues (fp32 everywhere).  K % 16 == 0.
cudaError_t gemm_f32(const GemmArgs& g, int kind, const EpiParams& ep, cudaStream_t st);

// Masked multi-head self-attention over the fused QKV matrix (columns Q | K | V,
// head h at h*DH), fp32 path.  Padded layout (tok0 null): sequence s owns rows
// s*S .. s*S + S - 1 and keys at token index >= 1 + lengths[s % len_mod] are excluded.
// Packed layout: sequence s owns rows tok0[s] .. tok0[s + 1] - 1 (its valid tokens
// only; S is then the largest sequence).  out has the rows of qkv, D columns.
cudaError_t attention_f32(const float* qkv, float* out, const int* lengths, int len_mod, int nseq, int S,
                          cudaStream_t st, const int* tok0 = nullptr);

// The same attention on the tcgen05 tensor cores (bf16 path): one CTA per (head, sequence,
// 128-query tile), exact softmax over all keys of the sequence at once.  qkv has M
// rows (16-byte aligned, row stride 3*D); S <= MAX_FRAMES + 1.  pf: weights its CTAs pull
// into L2 for the projections that follow.
cudaError_t attention_tc(const bf16* qkv, bf16* out, int M, const int* lengths, int len_mod, int nseq, int S,
                         DevError* err, cudaStream_t st, const int* tok0 = nullptr, L2Prefetch pf = {});
cudaError_t attention_tc_prepare();
size_t attention_tc_smem(int S);

// Token layout of a batch: tok0[s] = sum over s' < s of (1 + lengths[s' % len_mod]) for
// s <= nseq, and row_seq[r] = s for the rows r of sequence s (one CTA).
cudaError_t build_token_map(const int* lengths, int len_mod, int nseq, int* tok0, int* row_seq, cudaStream_t st);

// Row LayerNorm over D features: y fp32 [M, D] -> out (bf16 or fp32) [M, D], and
// optionally the row statistics (mean, 1/std) into stats [M][2]; pf: weights its CTAs pull
// into L2 for the projections that follow.
cudaError_t layernorm(const float* y, void* out, bool out_bf16, const float* gamma, const float* beta, int M,
                      cudaStream_t st, float* stats = nullptr, L2Prefetch pf = {});

// ---- motion / sampler kernels (element type of the activation matrices: bf16 or fp32)

// A[(row(seq, i)) * lda + col0 + f] = src[((seq % nsrc) * T + i) * ld_src + f0 + f], f < nf, with
// row(seq, i) = seq*S + 1 + i for every i < T (padded layout, tok0 null) or tok0[seq] + 1 + i
// for the valid frames i < lengths[seq % len_mod] only (packed layout).
cudaError_t pack_frames(const float* src, int nsrc, int ld_src, int f0, int nf, void* A, bool a_bf16, int lda,
                        int col0, int nseq, int T, int S, cudaStream_t st, const int* tok0 = nullptr,
                        const int* lengths = nullptr, int len_mod = 1);

// Body-network input of the two-stage step: for seq in [0, nseq), frame i < T (padded
// layout) or i < lengths[seq % B] (packed layout, rows as pack_frames):
//   A[.., 0:274] = x[seq % B, i, 5:279];  A[.., 274:279] = G2L(root_hat[seq])[i]  (0 for padded frames)
cudaError_t g2l_body_input(const float* root_hat, const float* x, const int* lengths, int B, int nseq, int T,
                           int S, void* A, bool a_bf16, int lda, cudaStream_t st, const int* tok0 = nullptr);

// CFG + DDIM update in place on x [B, T, 279]: x0 = u + w (c - u) from the root /
// body predictions of sequences b (cond) and B + b (uncond); x = c0 x0 + c1 x
// (+ c2 z when z [B, T, 279] is given); padded frames 0.  If A_next != nullptr the
// new root features are also packed into the root network's input matrix for
// sequences b and B + b.
cudaError_t cfg_ddim(const float* root_hat, const float* body_hat, float* x, const int* lengths, int B, int T,
                     float w, float c0, float c1, const float* z, float c2, void* A_next, bool a_bf16, int lda, int S,
                     cudaStream_t st, const int* tok0 = nullptr);

// Condition inputs: rows [0, B) = text_emb row r / takes (several takes of one prompt
// share its row), rows [B, B + null_rows) = null_emb row (r - B) % null_batch.
// out (bf16 or fp32) [rows, DTXT].
cudaError_t pack_embeddings(const float* text_emb, int B, const float* null_emb, int null_batch, int null_rows,
                            void* out, bool out_bf16, cudaStream_t st, int takes = 1);

// out[k, :] = pe[t_k, :] for k < n (sinusoid rows of the timesteps): t_k = t_single
// when steps == 0, else the k-th trailing timestep of a `steps`-step sampler,
// floor(N_TRAIN (steps - k) / steps + 1/2) - 1.
cudaError_t gather_timestep_rows(const float* pe, int t_single, int steps, int n, void* out, bool out_bf16,
                                 cudaStream_t st);

}  // namespace kd
