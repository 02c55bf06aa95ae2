// Tensor-core GEMM for a few hundred tokens (one or a few prompts): K split over a
// thread-block cluster, partial sums reduced through distributed shared memory.
//
// With few rows, a projection has few 128-row output tiles, and a tile that streams its
// whole K extent takes K / 16 tcgen05.mma instructions in sequence; each instruction
// costs about the same time whatever its N (up to 256), so the time of a launch is set
// by the length of that chain, not by the bytes or the FLOPs.  Here the S CTAs of a
// cluster share one 128 x BN output tile (BN = 256), CTA r taking k-blocks
// [r K / S, (r + 1) K / S): every chain is S times shorter.
//
//  * Roles (192 threads): warp 0 = TMA producer (A 128 x 64 and B BN x 64 boxes, 128-byte
//    swizzle, no multicast), warp 1 = TMEM allocation and the MMA issuer (one elected
//    thread, M 128 x N BN x K 16 per instruction, fp32 accumulator in TMEM), warps 2-5 =
//    epilogue (one per TMEM lane quarter).
//  * CTA r finishes the column slice [r BN / S, (r + 1) BN / S).  After its last MMA
//    (and a cluster barrier: every CTA's pipeline has drained, so the stage buffers are
//    free everywhere) each CTA reads its fp32 partial tile from TMEM and pushes every
//    16-column chunk to the owner of the chunk's slice (remote shared-memory stores,
//    issued back to back) into a receive area [source rank][128 rows][slice] over the
//    owner's drained stages.  After a second cluster barrier (the stores are visible),
//    each CTA sums the S partials of its slice in rank order from its own shared memory
//    and runs the usual epilogue (bias, GELU, residual, LayerNorm statistics).
//  * The split S is fixed per layer shape (K / 256), so every output element sums the
//    same k ranges in the same order at every row count served by this kernel.
//  * Every mbarrier wait is bounded (2 s); on give-up the kernel records KIMODO_ETIMEOUT,
//    still passes both cluster barriers, drains its own TMA loads and MMAs, frees its
//    TMEM and returns.
#include <cuda.h>
#include <cuda_runtime.h>
#include <type_traits>

#include "common.cuh"
#include "epilogue.cuh"
#include "kernels.h"
#include "launch.cuh"
#include "ptx.cuh"

namespace kd {
namespace {

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK = 64;
constexpr int STAGES = 4;
constexpr int EPI_WARPS = 4;
constexpr int NUM_THREADS = 64 + 32 * EPI_WARPS;
constexpr int CW = 16;                                    // epilogue chunk: columns per pass
constexpr uint64_t WAIT_LIMIT_NS = 2000000000ull;
constexpr int KIMODO_ETIMEOUT_CODE = -5;

constexpr uint32_t A_BYTES = BM * BK * 2;
constexpr uint32_t B_BYTES = BN * BK * 2;
constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int RPAD = 4;                                   // receive-area row padding (floats)
// receive area: S slices of BM rows x (BN / S + RPAD) floats, BM x (BN + S RPAD) in all;
// largest for S = 8
constexpr uint32_t PART_BYTES = BM * (BN + 8 * RPAD) * 4;
constexpr uint32_t MAIN_BYTES = STAGES * STAGE_BYTES > PART_BYTES ? STAGES * STAGE_BYTES : PART_BYTES;
constexpr uint32_t EPI_BYTES = EPI_WARPS * 32 * (CW + 4) * 4;   // one staging tile per epilogue warp
constexpr uint32_t NUM_BARS = 2 * STAGES + 2;
constexpr size_t SMEM = 1024 + (size_t)MAIN_BYTES + EPI_BYTES + NUM_BARS * 8 + 16;
constexpr uint32_t IDESC = ptx::idesc_bf16_f32(BM, BN);
static_assert(SMEM <= 232448, "shared memory");

__device__ __forceinline__ void record_timeout(DevError* err, int where, volatile int* abort) {
  *abort = 1;
  if (err && atomicCAS(&err->code, 0, KIMODO_ETIMEOUT_CODE) == 0) {
    err->where = where;
    err->block = blockIdx.x;
  }
}

// 16 consecutive floats into another CTA's shared memory (shared::cluster address)
__device__ __forceinline__ void st_dsmem16(uint32_t addr, const float (&v)[16]) {
#pragma unroll
  for (int j = 0; j < 4; ++j)
    asm volatile("st.shared::cluster.v4.f32 [%0], {%1, %2, %3, %4};"
                 ::"r"(addr + 16u * j), "f"(v[4 * j]), "f"(v[4 * j + 1]), "f"(v[4 * j + 2]), "f"(v[4 * j + 3])
                 : "memory");
}

// Grid: clusters of S CTAs (S = gridDim-wise cluster size); cluster q = blockIdx.x / S
// computes output tile q (m block q % num_m_tiles, n block q / num_m_tiles).
template <int KIND, typename OutT>
__global__ void __launch_bounds__(NUM_THREADS, 1)
gemm_splitk_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, int num_m_tiles,
                   int kb_per_cta, int S, EpiParams ep, DevError* err) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sA = ptx::smem_u32(smem);
  const uint32_t sB = sA + STAGES * A_BYTES;
  float* recv = reinterpret_cast<float*>(smem);             // [S][BM][slice + RPAD], after the mainloop
  float* epi_smem = reinterpret_cast<float*>(smem + MAIN_BYTES);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + MAIN_BYTES + EPI_BYTES);
  const uint32_t bar0 = ptx::smem_u32(bars);
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (STAGES + s); };
  const uint32_t acc_bar = bar0 + 8u * (2 * STAGES);
  const uint32_t drain_bar = bar0 + 8u * (2 * STAGES + 1);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + NUM_BARS);
  volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int rank = (int)ptx::cluster_ctarank();
  const int tile = blockIdx.x / S;
  const int m_blk = tile % num_m_tiles, n_blk = tile / num_m_tiles;
  const int kb0 = rank * kb_per_cta;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      ptx::mbar_init(full_bar(s), 1);
      ptx::mbar_init(empty_bar(s), 1);
    }
    ptx::mbar_init(acc_bar, 1);
    ptx::mbar_init(drain_bar, 1);
    ptx::fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    ptx::tma_prefetch_desc(&tmA);
    ptx::tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    ptx::tmem_alloc(ptx::smem_u32(tmem_slot), BN);
    ptx::tmem_relinquish();
  }
  ptx::pdl_trigger();
  ptx::pdl_wait();
  // a launch after a recorded timeout does no work; every CTA of the cluster reads the
  // same word, so they agree
  if (threadIdx.x == 0) *abort = (err != nullptr && *reinterpret_cast<volatile int*>(&err->code) != 0) ? 1 : 0;
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const bool idle = *abort != 0;

  if (warp == 0) {
    if (lane == 0 && !idle) {
      // ---------------- TMA producer
      int stage = 0;
      uint32_t phase = 0;
      long issued = 0;
      bool ok = true;
      for (int i = 0; i < kb_per_cta; ++i) {
        if (!ptx::mbar_wait_bounded(empty_bar(stage), phase ^ 1u, abort, WAIT_LIMIT_NS)) {
          ok = false;
          break;
        }
        ptx::mbar_arrive_expect_tx(full_bar(stage), STAGE_BYTES);
        ptx::tma_load_2d(sA + stage * A_BYTES, &tmA, full_bar(stage), (kb0 + i) * BK, m_blk * BM);
        ptx::tma_load_2d(sB + stage * B_BYTES, &tmB, full_bar(stage), (kb0 + i) * BK, n_blk * BN);
        ++issued;
        if (++stage == STAGES) { stage = 0; phase ^= 1u; }
      }
      if (!ok) {
        if (!*abort) record_timeout(err, WHERE_GEMM_PRODUCER, abort);
        const long n = issued < STAGES ? issued : STAGES;
        int s = stage;
        uint32_t ph = phase;
        volatile int never = 0;
        for (long i = 0; i < n; ++i) {
          if (--s < 0) { s = STAGES - 1; ph ^= 1u; }
          ptx::mbar_wait_bounded(full_bar(s), ph, &never, WAIT_LIMIT_NS);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && !idle) {
      // ---------------- MMA issuer
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int i = 0; i < kb_per_cta; ++i) {
        if (!ptx::mbar_wait_bounded(full_bar(stage), phase, abort, WAIT_LIMIT_NS)) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        const uint32_t a0 = sA + stage * A_BYTES;
        const uint32_t b0 = sB + stage * B_BYTES;
#pragma unroll
        for (int k = 0; k < BK / 16; ++k)
          ptx::tc_mma_bf16(tmem_base, ptx::smem_desc_sw128(a0 + k * 32), ptx::smem_desc_sw128(b0 + k * 32), IDESC,
                           (i | k) != 0);
        ptx::tc_commit(empty_bar(stage));
        if (++stage == STAGES) { stage = 0; phase ^= 1u; }
      }
      if (ok) ptx::tc_commit(acc_bar);
      else if (!*abort) record_timeout(err, WHERE_GEMM_MMA, abort);
      // every MMA of this thread completes before teardown
      ptx::tc_commit(drain_bar);
      volatile int never = 0;
      if (!ptx::mbar_wait_bounded(drain_bar, 0, &never, WAIT_LIMIT_NS)) record_timeout(err, WHERE_GEMM_DRAIN, abort);
    }
  }
  bool have_acc = false;
  if (warp >= 2 && !idle) {
    // the accumulator of this CTA's k range is complete
    if (!ptx::mbar_wait_bounded(acc_bar, 0, abort, WAIT_LIMIT_NS)) {
      if (!*abort) record_timeout(err, WHERE_GEMM_EPILOGUE, abort);
    } else {
      have_acc = true;
    }
  }
  // every CTA of the cluster has drained its pipeline: the stage buffers may be overwritten
  __syncwarp();
  ptx::tc_fence_before();
  ptx::cluster_sync();

  const int slice = BN / S;
  const int rstride = slice + RPAD;   // receive-area row stride (floats)
  if (warp >= 2 && have_acc) {
    // ---------------- push the partial: chunk c of row r goes to CTA c / slice, slot rank
    ptx::tc_fence_after();
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t taddr = tmem_base + ((uint32_t)(quarter * 32) << 16);
    const uint32_t recv0 = ptx::smem_u32(recv);
    auto push = [&](const float (&v)[16], int c) {
      const int owner = c / slice;
      const uint32_t local = recv0 + (uint32_t)(((rank * BM + r) * rstride + (c - owner * slice)) * 4);
      st_dsmem16(ptx::mapa_shared(local, (uint32_t)owner), v);
    };
    // two register buffers: the TMEM load of chunk c + 16 is in flight while chunk c is pushed
    float va[16], vb[16];
    ptx::tmem_ld(taddr, va);
#pragma unroll 1
    for (int c = 0; c < BN; c += 32) {
      ptx::tmem_ld_wait();
      ptx::tmem_ld(taddr + c + 16, vb);
      push(va, c);
      ptx::tmem_ld_wait();
      if (c + 32 < BN) ptx::tmem_ld(taddr + c + 32, va);
      push(vb, c + 16);
    }
  }
  // every partial is in its owner's receive area
  __syncwarp();
  ptx::cluster_sync();

  if (warp >= 2 && !idle && !*abort) {
    // ---------------- sum the S partials of this CTA's slice in rank order, then the epilogue
    const int quarter = warp & 3;
    const int row0 = m_blk * BM + quarter * 32;
    const int r = quarter * 32 + lane;
    const int c_beg = rank * slice;
    float* st = epi_smem + (warp - 2) * 32 * (CW + 4);
    constexpr int PASSES = EpiLanes<CW>::PASSES;
    // the global operands (bias, residual rows) of chunk k + 1 load while chunk k is summed
    const int ncol = min(slice, ep.N - (n_blk * BN + c_beg));
    const int nch = ncol > 0 ? (ncol + CW - 1) / CW : 0;
    const int gcol0 = n_blk * BN + c_beg;
    auto finish = [&](int k, const float4 (&pre)[PASSES], const float4 bias4) {
      float4 sum[4] = {};
      for (int s = 0; s < S; ++s) {
        const float4* src = reinterpret_cast<const float4*>(recv + (size_t)(s * BM + r) * rstride + k * CW);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float4 p = src[j];
          sum[j].x += p.x; sum[j].y += p.y; sum[j].z += p.z; sum[j].w += p.w;
        }
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) *reinterpret_cast<float4*>(st + lane * (CW + 4) + 4 * j) = sum[j];
      __syncwarp();
      epilogue_warp_tile<KIND, OutT, CW>(ep, st, row0, gcol0 + k * CW, lane, pre, bias4);
      __syncwarp();
    };
    float4 pa[PASSES], pb[PASSES];
    float4 ba, bb;
    if (nch > 0) epilogue_prefetch<KIND, CW>(ep, row0, gcol0, lane, pa, ba);
#pragma unroll 1
    for (int k = 0; k < nch; k += 2) {
      if (k + 1 < nch) epilogue_prefetch<KIND, CW>(ep, row0, gcol0 + (k + 1) * CW, lane, pb, bb);
      finish(k, pa, ba);
      if (k + 1 >= nch) break;
      if (k + 2 < nch) epilogue_prefetch<KIND, CW>(ep, row0, gcol0 + (k + 2) * CW, lane, pa, ba);
      finish(k + 1, pb, bb);
    }
  }

  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem_base, BN);
  }
}

template <int KIND, typename OutT>
cudaError_t splitk_impl(const GemmArgs& g, const EpiParams& ep, DevError* err, cudaStream_t st, bool prepare_only) {
  auto kern = gemm_splitk_kernel<KIND, OutT>;
  if (prepare_only) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 0);
    return e;
  }
  const int kb = (g.K + BK - 1) / BK;
  const int S = gemm_splitk_factor(g.N, g.K);
  if (S < 2 || kb % S) return cudaErrorInvalidValue;
  CUtensorMap ta, tb;
  if (make_tmap_bf16(&ta, g.A, g.M, g.K, g.lda, BM) || make_tmap_bf16(&tb, g.B, g.N, g.K, g.ldb, BN))
    return cudaErrorInvalidValue;
  const int mt = (g.M + BM - 1) / BM, nt = (g.N + BN - 1) / BN;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = S;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.gridDim = dim3(mt * nt * S);
  cfg.blockDim = dim3(NUM_THREADS);
  cfg.dynamicSmemBytes = SMEM;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, kern, ta, tb, mt, kb / S, S, ep, err);
}

#define KD_SK_LIST(X) \
  X(EPI_BIAS, bf16) X(EPI_BIAS_GELU, bf16) X(EPI_BIAS_RESID, float) X(EPI_BIAS_RESID_LN, float)

cudaError_t dispatch(const GemmArgs& g, int kind, bool out_f32, const EpiParams& ep, DevError* err, cudaStream_t st,
                     bool prep) {
#define KD_SK(KIND_, OUT_)                                                                     \
  if (prep) {                                                                                \
    cudaError_t e_ = splitk_impl<KIND_, OUT_>(g, ep, err, st, true);                          \
    if (e_ != cudaSuccess) return e_;                                                        \
  } else if (kind == KIND_ && out_f32 == std::is_same<OUT_, float>::value)                   \
    return splitk_impl<KIND_, OUT_>(g, ep, err, st, false);
  KD_SK_LIST(KD_SK)
#undef KD_SK
  return prep ? cudaSuccess : cudaErrorInvalidValue;
}

}  // namespace

int gemm_splitk_factor(int N, int K) {
  if (N % BN || K % (4 * BK)) return 0;
  const int S = K / (4 * BK);               // four 64-deep k-blocks per CTA
  return (S >= 2 && S <= 8) ? S : 0;
}

bool gemm_splitk_supports(int kind, bool out_f32) {
  return ((kind == EPI_BIAS || kind == EPI_BIAS_GELU) && !out_f32) ||
         ((kind == EPI_BIAS_RESID || kind == EPI_BIAS_RESID_LN) && out_f32);
}

cudaError_t gemm_splitk(const GemmArgs& g, int kind, bool out_f32, const EpiParams& ep, DevError* err,
                        cudaStream_t st) {
  if (g.M <= 0 || g.N <= 0) return cudaSuccess;
  return dispatch(g, kind, out_f32, ep, err, st, false);
}

cudaError_t gemm_splitk_prepare() {
  GemmArgs g;
  EpiParams ep;
  return dispatch(g, 0, false, ep, nullptr, nullptr, true);
}

}  // namespace kd
