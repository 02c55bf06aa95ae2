// Sampler-side kernels of the two-stage DDIM step ("Kimodo WebGPU",
// "Architecture" figure: root model -> globalRootToLocalRoot -> body model ->
// CFG guidance -> DDIM update): packing frames into the networks' input
// matrices, the global-to-local root transform, and one fused kernel for the
// classifier-free-guidance combine plus the DDIM update (eta >= 0, with the
// caller's standard-normal draw for the step when eta > 0).
#include <cuda_runtime.h>
#include <math.h>

#include "common.cuh"
#include "epilogue.cuh"
#include "kernels.h"
#include "launch.cuh"
#include "ptx.cuh"

namespace kd {
namespace {

// Row of frame i of sequence seq in the activation matrices, or -1 when the packed
// layout has no row for it (a padded frame).
__device__ __forceinline__ long frame_row(const int* tok0, const int* lengths, int len_mod, int seq, int i, int S) {
  if (tok0 == nullptr) return (long)seq * S + 1 + i;
  return i < lengths[seq % len_mod] ? (long)tok0[seq] + 1 + i : -1;
}

template <typename T>
__global__ void pack_frames_kernel(const float* __restrict__ src, int nsrc, int ld_src, int f0, int nf,
                                   T* __restrict__ A, int lda, int col0, int nseq, int T_, int S,
                                   const int* __restrict__ tok0, const int* __restrict__ lengths, int len_mod) {
  ptx::pdl_wait();
  ptx::pdl_trigger();
  const long total = (long)nseq * T_ * nf;
  for (long idx = blockIdx.x * (long)blockDim.x + threadIdx.x; idx < total; idx += (long)gridDim.x * blockDim.x) {
    const int f = idx % nf;
    const long r = idx / nf;
    const int i = r % T_;
    const int seq = r / T_;
    const long row = frame_row(tok0, lengths, len_mod, seq, i, S);
    if (row < 0) continue;
    const float v = src[((long)(seq % nsrc) * T_ + i) * ld_src + f0 + f];
    A[row * lda + col0 + f] = from_f<T>(v);
  }
}

// tok0[s] = sum_{s' < s} (1 + len[s']) for s <= nseq; row_seq[r] = s on the rows of s.
__global__ void build_token_map_kernel(const int* __restrict__ lengths, int len_mod, int nseq, int* __restrict__ tok0,
                                       int* __restrict__ row_seq) {
  ptx::pdl_wait();
  ptx::pdl_trigger();
  __shared__ int s_tok0[1025];
  const bool in_smem = nseq <= 1024;
  if (threadIdx.x == 0) {
    int acc = 0;
    for (int s = 0; s < nseq; ++s) {
      if (in_smem) s_tok0[s] = acc;
      tok0[s] = acc;
      acc += 1 + lengths[s % len_mod];
    }
    if (in_smem) s_tok0[nseq] = acc;
    tok0[nseq] = acc;
  }
  __syncthreads();
  __threadfence_block();
  for (int s = 0; s < nseq; ++s) {
    const int a = in_smem ? s_tok0[s] : tok0[s];
    const int b = in_smem ? s_tok0[s + 1] : tok0[s + 1];
    for (int r = a + threadIdx.x; r < b; r += blockDim.x) row_seq[r] = s;
  }
}

// Global root (x, z, sin th, cos th, y) of frames i-1 and i -> local root
// (vx', vz', sin d, cos d, y): heading-frame displacement, relative heading and
// height.  The frame before the first sits at the origin with heading 0.
__device__ __forceinline__ void local_root(const float* prev, const float* cur, bool first, float (&o)[5]) {
  float px = 0.f, pz = 0.f, cp = 1.f, sp = 0.f;
  if (!first) {
    const float n = fmaxf(hypotf(prev[3], prev[2]), 1e-8f);
    px = prev[0];
    pz = prev[1];
    cp = prev[3] / n;
    sp = prev[2] / n;
  }
  const float n = fmaxf(hypotf(cur[3], cur[2]), 1e-8f);
  const float c = cur[3] / n, s = cur[2] / n;
  const float vx = cur[0] - px, vz = cur[1] - pz;
  o[0] = c * vx - s * vz;
  o[1] = s * vx + c * vz;
  o[2] = s * cp - c * sp;
  o[3] = c * cp + s * sp;
  o[4] = cur[4];
}

template <typename T>
__global__ void g2l_body_input_kernel(const float* __restrict__ root_hat, const float* __restrict__ x,
                                      const int* __restrict__ lengths, int B, int nseq, int T_, int S,
                                      T* __restrict__ A, int lda, const int* __restrict__ tok0) {
  ptx::pdl_wait();
  ptx::pdl_trigger();
  const int warp_global = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp_global >= nseq * T_) return;
  const int seq = warp_global / T_, i = warp_global % T_;
  const long row = frame_row(tok0, lengths, B, seq, i, S);
  if (row < 0) return;
  const float* xr = x + ((long)(seq % B) * T_ + i) * MOTION_F + ROOT_F;
  T* ar = A + row * lda;
  for (int f = lane; f < BODY_F; f += 32) ar[f] = from_f<T>(xr[f]);
  if (lane == 0) {
    float o[5] = {0.f, 0.f, 0.f, 0.f, 0.f};
    if (i < lengths[seq % B]) {
      const float* cur = root_hat + ((long)seq * T_ + i) * ROOT_F;
      local_root(cur - ROOT_F, cur, i == 0, o);
    }
#pragma unroll
    for (int k = 0; k < 5; ++k) ar[BODY_F + k] = from_f<T>(o[k]);
  }
}

template <typename T>
__global__ void cfg_ddim_kernel(const float* __restrict__ root_hat, const float* __restrict__ body_hat,
                                float* __restrict__ x, const int* __restrict__ lengths, int B, int T_, float w,
                                float c0, float c1, const float* __restrict__ z, float c2, T* __restrict__ A_next,
                                int lda, int S, const int* __restrict__ tok0) {
  ptx::pdl_wait();
  ptx::pdl_trigger();
  const long total = (long)B * T_ * MOTION_F;
  for (long idx = blockIdx.x * (long)blockDim.x + threadIdx.x; idx < total; idx += (long)gridDim.x * blockDim.x) {
    const int f = idx % MOTION_F;
    const long r = idx / MOTION_F;
    const int i = r % T_;
    const int b = r / T_;
    float xn = 0.f;
    if (i < lengths[b]) {
      float c, u;
      if (f < ROOT_F) {
        c = root_hat[((long)b * T_ + i) * ROOT_F + f];
        u = root_hat[((long)(B + b) * T_ + i) * ROOT_F + f];
      } else {
        c = body_hat[((long)b * T_ + i) * BODY_F + f - ROOT_F];
        u = body_hat[((long)(B + b) * T_ + i) * BODY_F + f - ROOT_F];
      }
      const float x0 = u + w * (c - u);
      xn = c0 * x0 + c1 * x[idx];
      if (z != nullptr) xn += c2 * z[idx];
    }
    x[idx] = xn;
    if (A_next != nullptr && f < ROOT_F) {
      const long rc = frame_row(tok0, lengths, B, b, i, S), ru = frame_row(tok0, lengths, B, B + b, i, S);
      if (rc >= 0) A_next[rc * lda + f] = from_f<T>(xn);
      if (ru >= 0) A_next[ru * lda + f] = from_f<T>(xn);
    }
  }
}

template <typename T>
__global__ void pack_embeddings_kernel(const float* __restrict__ text, int B, int takes,
                                       const float* __restrict__ null_emb, int null_batch, int null_rows,
                                       T* __restrict__ out) {
  ptx::pdl_wait();
  ptx::pdl_trigger();
  const long total = (long)(B + null_rows) * DTXT;
  for (long idx = blockIdx.x * (long)blockDim.x + threadIdx.x; idx < total; idx += (long)gridDim.x * blockDim.x) {
    const int r = idx / DTXT, c = idx % DTXT;
    const float v = r < B ? text[(long)(r / takes) * DTXT + c] : null_emb[(long)((r - B) % null_batch) * DTXT + c];
    out[idx] = from_f<T>(v);
  }
}

// Row k of the output is the sinusoid of timestep t_k: t_single when steps == 0, else
// the k-th trailing DDIM timestep floor(N_TRAIN (steps - k) / steps + 1/2) - 1.
template <typename T>
__global__ void gather_rows_kernel(const float* __restrict__ pe, int t_single, int steps, int n,
                                   T* __restrict__ out) {
  ptx::pdl_wait();
  ptx::pdl_trigger();
  const long total = (long)n * D;
  for (long idx = blockIdx.x * (long)blockDim.x + threadIdx.x; idx < total; idx += (long)gridDim.x * blockDim.x) {
    const int k = idx / D, c = idx % D;
    const int t = steps > 0 ? (2 * N_TRAIN * (steps - k) + steps) / (2 * steps) - 1 : t_single;
    out[idx] = from_f<T>(pe[(long)t * D + c]);
  }
}

#define LAUNCHK(K, G, B, ST, ...) return launch_kernel(K, dim3(G), dim3(B), 0, ST, __VA_ARGS__)

inline int blocks_for(long n, int threads = 256) {
  long b = (n + threads - 1) / threads;
  return (int)(b < 1 ? 1 : (b > 148 * 16 ? 148 * 16 : b));
}

}  // namespace

cudaError_t pack_frames(const float* src, int nsrc, int ld_src, int f0, int nf, void* A, bool a_bf16, int lda,
                        int col0, int nseq, int T, int S, cudaStream_t st, const int* tok0, const int* lengths,
                        int len_mod) {
  const long n = (long)nseq * T * nf;
  if (n <= 0) return cudaSuccess;
  if (a_bf16)
    LAUNCHK(pack_frames_kernel<bf16>, blocks_for(n), 256, st, src, nsrc, ld_src, f0, nf, static_cast<bf16*>(A), lda,
                                                            col0, nseq, T, S, tok0, lengths, len_mod);
  else
    LAUNCHK(pack_frames_kernel<float>, blocks_for(n), 256, st, src, nsrc, ld_src, f0, nf, static_cast<float*>(A), lda,
                                                             col0, nseq, T, S, tok0, lengths, len_mod);
  return cudaGetLastError();
}

cudaError_t build_token_map(const int* lengths, int len_mod, int nseq, int* tok0, int* row_seq, cudaStream_t st) {
  if (nseq <= 0) return cudaSuccess;
  LAUNCHK(build_token_map_kernel, 1, 1024, st, lengths, len_mod, nseq, tok0, row_seq);
}

cudaError_t g2l_body_input(const float* root_hat, const float* x, const int* lengths, int B, int nseq, int T,
                           int S, void* A, bool a_bf16, int lda, cudaStream_t st, const int* tok0) {
  const long warps = (long)nseq * T;
  if (warps <= 0) return cudaSuccess;
  const int grid = (int)((warps * 32 + 255) / 256);
  if (a_bf16)
    LAUNCHK(g2l_body_input_kernel<bf16>, grid, 256, st, root_hat, x, lengths, B, nseq, T, S, static_cast<bf16*>(A), lda,
                                                      tok0);
  else
    LAUNCHK(g2l_body_input_kernel<float>, grid, 256, st, root_hat, x, lengths, B, nseq, T, S, static_cast<float*>(A),
                                                       lda, tok0);
  return cudaGetLastError();
}

cudaError_t cfg_ddim(const float* root_hat, const float* body_hat, float* x, const int* lengths, int B, int T,
                     float w, float c0, float c1, const float* z, float c2, void* A_next, bool a_bf16, int lda, int S,
                     cudaStream_t st, const int* tok0) {
  const long n = (long)B * T * MOTION_F;
  if (n <= 0) return cudaSuccess;
  if (a_bf16)
    LAUNCHK(cfg_ddim_kernel<bf16>, blocks_for(n), 256, st, root_hat, body_hat, x, lengths, B, T, w, c0, c1, z, c2,
                                                         static_cast<bf16*>(A_next), lda, S, tok0);
  else
    LAUNCHK(cfg_ddim_kernel<float>, blocks_for(n), 256, st, root_hat, body_hat, x, lengths, B, T, w, c0, c1, z, c2,
                                                          static_cast<float*>(A_next), lda, S, tok0);
  return cudaGetLastError();
}

cudaError_t pack_embeddings(const float* text_emb, int B, const float* null_emb, int null_batch, int null_rows,
                            void* out, bool out_bf16, cudaStream_t st, int takes) {
  const long n = (long)(B + null_rows) * DTXT;
  if (n <= 0) return cudaSuccess;
  if (out_bf16)
    LAUNCHK(pack_embeddings_kernel<bf16>, blocks_for(n), 256, st, text_emb, B, takes, null_emb, null_batch, null_rows,
                                                                static_cast<bf16*>(out));
  else
    LAUNCHK(pack_embeddings_kernel<float>, blocks_for(n), 256, st, text_emb, B, takes, null_emb, null_batch,
                                                                 null_rows, static_cast<float*>(out));
  return cudaGetLastError();
}

cudaError_t gather_timestep_rows(const float* pe, int t_single, int steps, int n, void* out, bool out_bf16,
                                 cudaStream_t st) {
  const long total = (long)n * D;
  if (total <= 0) return cudaSuccess;
  if (out_bf16)
    LAUNCHK(gather_rows_kernel<bf16>, blocks_for(total), 256, st, pe, t_single, steps, n, static_cast<bf16*>(out));
  else
    LAUNCHK(gather_rows_kernel<float>, blocks_for(total), 256, st, pe, t_single, steps, n, static_cast<float*>(out));
  return cudaGetLastError();
}

}  // namespace kd
