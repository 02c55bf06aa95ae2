// Tensor-core GEMM for sm_100a: D[M,N] = A[M,K] . B[N,K]^T with a fused epilogue.
//
// Serves every projection of the denoiser ("Kimodo WebGPU", "WGSL compute
// shaders" table: linear + bias, fused QKV projection, GELU, SiLU timestep MLP,
// residual add): A is the bf16 activation matrix (tokens x features), B the bf16
// weight [out x in] exactly as stored, both K-major.
//
// Design
//  * Persistent: one CTA per SM walks output tiles tile = blockIdx.x + i*gridDim.x.
//  * Warp roles (192 threads): warp 0 issues TMA tile loads (128B swizzle) into a
//    STAGES-deep shared-memory ring; warp 1 allocates TMEM and one elected lane
//    issues tcgen05.mma (128 x BN x 16 per instruction, fp32 accumulator in
//    TMEM); warps 2-5 read the accumulator with tcgen05.ld and run the epilogue.
//  * Two TMEM accumulators, so the epilogue of tile i overlaps the MMAs of i+1.
//  * Plain (non-multicast) TMA loads; out-of-range rows/columns read as zero.
//  * Every wait is bounded (2 s of wall time).  On give-up the kernel records
//    KIMODO_ETIMEOUT in the context's error word, stops all roles, waits
//    (bounded) for its own TMA loads and MMAs, frees its TMEM and returns.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdio.h>
#include <type_traits>

#include "common.cuh"
#include "epilogue.cuh"
#include "kernels.h"
#include "launch.cuh"
#include "ptx.cuh"

namespace kd {

namespace {

constexpr int BM = 128;
constexpr int BK = 64;                       // 64 bf16 = one 128-byte swizzle row
constexpr int EPI_WARPS = 8;                 // two per TMEM lane quarter, splitting the columns
constexpr int EPI_PARTS = EPI_WARPS / 4;
constexpr int NUM_THREADS = 64 + 32 * EPI_WARPS;
constexpr uint64_t WAIT_LIMIT_NS = 2000000000ull;
constexpr int KIMODO_ETIMEOUT_CODE = -5;

constexpr uint32_t tmem_cols_for(uint32_t n) {
  return n <= 32 ? 32 : n <= 64 ? 64 : n <= 128 ? 128 : n <= 256 ? 256 : 512;
}

template <int BN, int STAGES>
struct TcCfg {
  // K columns per pipeline stage: KA swizzle atoms of 64 (one TMA box each).  Below N = 256
  // two atoms per stage halve the stage hand-offs (wait, fence, commit: about 200 ns on
  // the issuing thread, more than the MMA time of a 64-column step at N <= 128).
  static constexpr int KA = BN <= 128 ? 2 : 1;
  static constexpr uint32_t ATOM_A = BM * 128;          // one 64-column atom (128-byte rows)
  static constexpr uint32_t ATOM_B = BN * 128;
  static constexpr uint32_t A_BYTES = KA * ATOM_A;
  static constexpr uint32_t B_BYTES = KA * ATOM_B;
  static constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr uint32_t TMEM_COLS = tmem_cols_for(2 * BN);
  static constexpr uint32_t NUM_BARS = 2 * STAGES + 5;
  static constexpr int CW = 16;                                        // epilogue chunk: columns per tcgen05.ld
  static constexpr int WCOLS = BN / EPI_PARTS >= 16 ? BN / EPI_PARTS : 16;  // columns per epilogue warp
  static constexpr uint32_t EPI_BYTES = EPI_WARPS * 32 * (CW + 4) * 4;  // one staging tile per epilogue warp
  static constexpr size_t SMEM = 1024 + (size_t)STAGES * STAGE_BYTES + EPI_BYTES + NUM_BARS * 8 + 16;
  static constexpr uint32_t IDESC = ptx::idesc_bf16_f32(BM, BN);
  static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "UMMA N for M=128");
  static_assert(SMEM <= 232448, "shared memory");
};

__device__ __forceinline__ void record_timeout(DevError* err, int where, volatile int* abort) {
  *abort = 1;
  if (err && atomicCAS(&err->code, 0, KIMODO_ETIMEOUT_CODE) == 0) {
    err->where = where;
    err->block = blockIdx.x;
  }
}

template <int BN, int STAGES, int KIND, typename OutT, typename ResT>
__global__ void __launch_bounds__(NUM_THREADS, 1)
gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
               int num_m_tiles, int num_n_tiles, int num_kb, EpiParams ep, DevError* err) {
  using C = TcCfg<BN, STAGES>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sA = ptx::smem_u32(smem);
  const uint32_t sB = sA + STAGES * C::A_BYTES;
  float* epi_smem = reinterpret_cast<float*>(smem + STAGES * C::STAGE_BYTES);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + STAGES * C::STAGE_BYTES + C::EPI_BYTES);
  const uint32_t bar0 = ptx::smem_u32(bars);
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (STAGES + s); };
  auto tfull_bar = [&](int a) { return bar0 + 8u * (2 * STAGES + a); };
  auto tempty_bar = [&](int a) { return bar0 + 8u * (2 * STAGES + 2 + a); };
  const uint32_t drain_bar = bar0 + 8u * (2 * STAGES + 4);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::NUM_BARS);
  volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      ptx::mbar_init(full_bar(s), 1);
      ptx::mbar_init(empty_bar(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      ptx::mbar_init(tfull_bar(a), 1);
      ptx::mbar_init(tempty_bar(a), EPI_WARPS);
    }
    ptx::mbar_init(drain_bar, 1);
    ptx::fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    ptx::tma_prefetch_desc(&tmA);
    ptx::tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    ptx::tmem_alloc(ptx::smem_u32(tmem_slot), C::TMEM_COLS);
    ptx::tmem_relinquish();
  }
  // prologue done: let the next kernel launch, then wait for the previous one
  ptx::pdl_trigger();
  ptx::pdl_wait();
  // A launch after a recorded timeout does no work (its inputs are already invalid).
  if (threadIdx.x == 0) *abort = (err != nullptr && *reinterpret_cast<volatile int*>(&err->code) != 0) ? 1 : 0;
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int num_tiles = *abort ? 0 : num_m_tiles * num_n_tiles;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer
      int stage = 0;
      uint32_t phase = 0;
      long issued = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        const int m_blk = tile % num_m_tiles, n_blk = tile / num_m_tiles;
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!ptx::mbar_wait_bounded(empty_bar(stage), phase ^ 1u, abort, WAIT_LIMIT_NS)) {
            ok = false;
            break;
          }
          ptx::mbar_arrive_expect_tx(full_bar(stage), C::STAGE_BYTES);
#pragma unroll
          for (int at = 0; at < C::KA; ++at) {
            ptx::tma_load_2d(sA + stage * C::A_BYTES + at * C::ATOM_A, &tmA, full_bar(stage), (kb * C::KA + at) * BK,
                             m_blk * BM);
            ptx::tma_load_2d(sB + stage * C::B_BYTES + at * C::ATOM_B, &tmB, full_bar(stage), (kb * C::KA + at) * BK,
                             n_blk * BN);
          }
          ++issued;
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      if (!ok) {
        if (!*abort) record_timeout(err, WHERE_GEMM_PRODUCER, abort);
        // wait for the loads this thread may still have in flight
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
    if (lane == 0) {
      // ---------------- MMA issuer
      int stage = 0;
      uint32_t phase = 0;
      int local = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++local) {
        const int acc = local & 1;
        const uint32_t acc_phase = (local >> 1) & 1;
        if (!ptx::mbar_wait_bounded(tempty_bar(acc), acc_phase ^ 1u, abort, WAIT_LIMIT_NS)) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!ptx::mbar_wait_bounded(full_bar(stage), phase, abort, WAIT_LIMIT_NS)) {
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          const uint32_t a0 = sA + stage * C::A_BYTES;
          const uint32_t b0 = sB + stage * C::B_BYTES;
#pragma unroll
          for (int k = 0; k < C::KA * BK / 16; ++k) {
            ptx::tc_mma_bf16(d_tmem, ptx::smem_desc_sw128(a0 + (k >> 2) * C::ATOM_A + (k & 3) * 32),
                             ptx::smem_desc_sw128(b0 + (k >> 2) * C::ATOM_B + (k & 3) * 32), C::IDESC, (kb | k) != 0);
          }
          ptx::tc_commit(empty_bar(stage));
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        ptx::tc_commit(tfull_bar(acc));
      }
      if (!ok && !*abort) record_timeout(err, WHERE_GEMM_MMA, abort);
      // all MMAs issued by this thread complete before teardown
      ptx::tc_commit(drain_bar);
      volatile int never = 0;
      if (!ptx::mbar_wait_bounded(drain_bar, 0, &never, WAIT_LIMIT_NS)) record_timeout(err, WHERE_GEMM_DRAIN, abort);
    }
  } else {
    // ---------------- epilogue warps 2..(1 + EPI_WARPS): TMEM lane quarter = warp % 4; part (warp - 2) / 4
    // takes columns [part * WCOLS, (part + 1) * WCOLS) of the tile (parts past BN idle)
    const int quarter = warp & 3;
    const int part = (warp - 2) >> 2;
    constexpr int CW = C::CW;
    constexpr int PASSES = EpiLanes<CW>::PASSES;
    float* st = epi_smem + (warp - 2) * 32 * (CW + 4);
    int local = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++local) {
      const int acc = local & 1;
      const uint32_t acc_phase = (local >> 1) & 1;
      if (!ptx::mbar_wait_bounded(tfull_bar(acc), acc_phase, abort, WAIT_LIMIT_NS)) {
        if (!*abort) record_timeout(err, WHERE_GEMM_EPILOGUE, abort);
        break;
      }
      ptx::tc_fence_after();
      const int m_blk = tile % num_m_tiles, n_blk = tile / num_m_tiles;
      const int row0 = m_blk * BM + quarter * 32;
      const int cbeg = min(part * C::WCOLS, BN);
      const int cend = min(cbeg + C::WCOLS, BN);
      const int valid_end = min(cend, ep.N - n_blk * BN);
      const int nch = valid_end > cbeg ? (valid_end - cbeg + CW - 1) / CW : 0;
      const uint32_t taddr = tmem_base + ((uint32_t)(quarter * 32) << 16) + acc * BN + cbeg;
      const int gcol = n_blk * BN + cbeg;
      if (nch == 0) {
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(tempty_bar(acc));
        continue;
      }
      // two register buffers: the TMEM load and global prefetch of chunk c + 1 are in
      // flight while chunk c is transposed and stored
      float va[CW], vb[CW];
      float4 pa[PASSES], pb[PASSES];
      float4 ba, bb;
      auto process = [&](float (&v)[CW], const float4 (&pre)[PASSES], const float4 bias4, int c) {
#pragma unroll
        for (int j = 0; j < CW; j += 4)
          *reinterpret_cast<float4*>(st + lane * (CW + 4) + j) = make_float4(v[j], v[j + 1], v[j + 2], v[j + 3]);
        __syncwarp();
        epilogue_warp_tile<KIND, OutT, CW>(ep, st, row0, gcol + c * CW, lane, pre, bias4);
        __syncwarp();
      };
      auto release_if_last = [&](int c) {
        if (c == nch - 1) {
          ptx::tc_fence_before();
          __syncwarp();
          if (lane == 0) ptx::mbar_arrive(tempty_bar(acc));
        }
      };
      epilogue_prefetch<KIND, CW>(ep, row0, gcol, lane, pa, ba);
      ptx::tmem_ld(taddr, va);
#pragma unroll 1
      for (int c = 0; c < nch; c += 2) {
        ptx::tmem_ld_wait();
        release_if_last(c);
        if (c + 1 < nch) {
          epilogue_prefetch<KIND, CW>(ep, row0, gcol + (c + 1) * CW, lane, pb, bb);
          ptx::tmem_ld(taddr + (c + 1) * CW, vb);
        }
        process(va, pa, ba, c);
        if (c + 1 >= nch) break;
        ptx::tmem_ld_wait();
        release_if_last(c + 1);
        if (c + 2 < nch) {
          epilogue_prefetch<KIND, CW>(ep, row0, gcol + (c + 2) * CW, lane, pa, ba);
          ptx::tmem_ld(taddr + (c + 2) * CW, va);
        }
        process(vb, pb, bb, c + 1);
      }
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

// ------------------------------------------------------------------ host side

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

template <int BN, int STAGES, int KIND, typename OutT, typename ResT>
cudaError_t launch_impl(const GemmArgs& g, const EpiParams& ep, DevError* err, cudaStream_t st, int num_sms,
                        bool prepare_only) {
  using Cf = TcCfg<BN, STAGES>;
  auto kern = gemm_tc_kernel<BN, STAGES, KIND, OutT, ResT>;
  if (prepare_only)
    return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Cf::SMEM);
  CUtensorMap ta, tb;
  if (make_tmap_bf16(&ta, g.A, g.M, g.K, g.lda, BM) || make_tmap_bf16(&tb, g.B, g.N, g.K, g.ldb, BN))
    return cudaErrorInvalidValue;
  const int mt = (g.M + BM - 1) / BM, nt = (g.N + BN - 1) / BN;
  const int tiles = mt * nt;
  const int grid = tiles < num_sms ? tiles : num_sms;
  const int kb = (g.K + Cf::KA * BK - 1) / (Cf::KA * BK);
  return launch_kernel(kern, dim3(grid), dim3(NUM_THREADS), Cf::SMEM, st, ta, tb, mt, nt, kb, ep, err);
}

}  // namespace

// Row-major bf16 matrix [rows, ld] whose first `cols` columns are the K extent.
int make_tmap_bf16(CUtensorMap* m, const void* base, int rows, int cols, int ld, int box_rows) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return -1;
  if ((reinterpret_cast<uintptr_t>(base) & 15) || (ld * 2) % 16) return -2;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)ld * 2};
  cuuint32_t box[2] = {(cuuint32_t)BK, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? 0 : -3;
}


// Row-major matrix [rows, ld] of fp32 (elem 4) or bf16 (elem 2), K extent `cols`,
// boxes of box_cols x box_rows (epilogue staging tiles), shared-memory swizzle of
// 0 (none), 32, 64 or 128 bytes; a swizzled box row must span exactly that many bytes.
int make_tmap_plain(CUtensorMap* m, const void* base, int elem, int rows, int cols, long ld, int box_cols,
                    int box_rows, int swizzle) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return -1;
  if ((reinterpret_cast<uintptr_t>(base) & 15) || (ld * elem) % 16 || (box_cols * elem) % 16) return -2;
  CUtensorMapSwizzle sw = CU_TENSOR_MAP_SWIZZLE_NONE;
  if (swizzle == 32) sw = CU_TENSOR_MAP_SWIZZLE_32B;
  else if (swizzle == 64) sw = CU_TENSOR_MAP_SWIZZLE_64B;
  else if (swizzle == 128) sw = CU_TENSOR_MAP_SWIZZLE_128B;
  else if (swizzle != 0) return -2;
  if (swizzle != 0 && box_cols * elem != swizzle) return -2;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)ld * elem};
  cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, elem == 4 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                   const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   sw, CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? 0 : -3;
}

// Dispatch on (tile N, epilogue kind, output type).  The residual is fp32 (the
// residual stream of the post-norm layers is kept in fp32; operands are bf16).
static cudaError_t dispatch(const GemmArgs& g, int bn, int kind, bool out_f32, const EpiParams& ep, DevError* err,
                            cudaStream_t st, int num_sms, bool prep) {
#define KD_TC(BN_, ST_, KIND_, OUT_)                                                            \
  if (prep) {                                                                                  \
    cudaError_t e_ = launch_impl<BN_, ST_, KIND_, OUT_, float>(g, ep, err, st, num_sms, true); \
    if (e_ != cudaSuccess) return e_;                                                          \
  } else if (bn == BN_ && kind == KIND_ && out_f32 == std::is_same<OUT_, float>::value)         \
    return launch_impl<BN_, ST_, KIND_, OUT_, float>(g, ep, err, st, num_sms, false);
  KD_TC(256, 4, EPI_BIAS, bf16)
  KD_TC(256, 4, EPI_BIAS_GELU, bf16)
  KD_TC(256, 4, EPI_BIAS_RESID, float)
  KD_TC(256, 4, EPI_BIAS_RESID_LN, float)
  KD_TC(256, 4, EPI_INPROJ, bf16)
  KD_TC(128, 3, EPI_BIAS, bf16)
  KD_TC(128, 3, EPI_BIAS, float)
  KD_TC(128, 3, EPI_BIAS_GELU, bf16)
  KD_TC(128, 3, EPI_BIAS_SILU, bf16)
  KD_TC(128, 3, EPI_BIAS_RESID, float)
  KD_TC(128, 3, EPI_BIAS_RESID_LN, float)
  KD_TC(128, 3, EPI_INPROJ, bf16)
  KD_TC(128, 3, EPI_OUTPROJ, float)
  KD_TC(64, 4, EPI_BIAS, bf16)
  KD_TC(64, 4, EPI_BIAS_GELU, bf16)
  KD_TC(64, 4, EPI_BIAS_RESID, float)
  KD_TC(64, 4, EPI_BIAS_RESID_LN, float)
  KD_TC(32, 5, EPI_BIAS, bf16)
  KD_TC(32, 5, EPI_BIAS_GELU, bf16)
  KD_TC(32, 5, EPI_BIAS_RESID, float)
  KD_TC(32, 5, EPI_BIAS_RESID_LN, float)
  KD_TC(16, 5, EPI_OUTPROJ, float)
#undef KD_TC
  return prep ? cudaSuccess : cudaErrorInvalidValue;
}

cudaError_t gemm_tc(const GemmArgs& g, int bn, int kind, bool out_f32, const EpiParams& ep, DevError* err,
                    cudaStream_t st, int num_sms) {
  if (g.M <= 0 || g.N <= 0) return cudaSuccess;
  if (g.K <= 0) return cudaErrorInvalidValue;
  return dispatch(g, bn, kind, out_f32, ep, err, st, num_sms, false);
}

cudaError_t gemm_tc_prepare() {
  GemmArgs g;
  EpiParams ep;
  return dispatch(g, 0, 0, false, ep, nullptr, nullptr, 0, true);
}

bool gemm_tc_available() { return get_encode_fn() != nullptr; }

}  // namespace kd
