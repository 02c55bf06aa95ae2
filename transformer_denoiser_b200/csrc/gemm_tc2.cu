// Tensor-core GEMM on SM pairs (tcgen05 cta_group::2) for the large per-layer
// projections: D[M,N] = A[M,K] . B[N,K]^T + fused epilogue, bf16 in, fp32 accumulate.
//
// A cluster of two CTAs computes a 256 x BN output tile.  Each CTA stages its own
// 128 rows of A and BN/2 rows of B (TMA, 128-byte swizzle, no multicast) into the
// same shared-memory offsets; the pair's leader (cluster rank 0) issues one
// 256 x BN x 16 MMA per K step that reads both CTAs' shared memory and writes
// each CTA's 128 accumulator rows into its own TMEM.  Per SM this halves the B
// traffic of a 128 x BN single-CTA tile.
//
// Roles (320 threads per CTA): warp 0 = TMA producer (both CTAs; completions are
// counted on the leader's "full" barriers), warp 1 = TMEM allocation and, in the
// leader, the MMA issuer, warps 2-9 = epilogue (two per TMEM lane quarter).  The
// leader's MMA commits arrive on both CTAs' "empty" and "accumulator full" barriers
// (tcgen05.commit multicast); both CTAs' epilogues release the accumulator on the
// leader's "accumulator empty" barrier.  Two TMEM accumulators per CTA.  Every
// wait is bounded; a timeout is recorded in the device error word.
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

constexpr int BMC = 128;                     // rows per CTA (256 per pair)
constexpr int BK = 64;
constexpr int EPI_WARPS = 8;
constexpr int NUM_THREADS = 64 + 32 * EPI_WARPS;
constexpr uint64_t WAIT_LIMIT_NS = 2000000000ull;
constexpr int KIMODO_ETIMEOUT_CODE = -5;

constexpr uint32_t tmem_cols_for(uint32_t n) {
  return n <= 32 ? 32 : n <= 64 ? 64 : n <= 128 ? 128 : n <= 256 ? 256 : 512;
}

template <int BN, int STAGES, int KIND>
struct Tc2Cfg {
  static constexpr bool RES = KIND == EPI_BIAS_RESID || KIND == EPI_BIAS_RESID_LN;
  // K columns per pipeline stage: KA swizzle atoms of 64 (one TMA box each).  Two atoms
  // halve the stage hand-offs per MMA (wait, fence, commit: measured about 200 ns on the
  // issuing thread, more than the MMA time of a 64-column step below N = 256); three such
  // stages fit beside the epilogue staging tiles.
  static constexpr int KA = 2;
  static constexpr uint32_t ATOM_A = BMC * 128;          // one 64-column atom of A (128-byte rows)
  static constexpr uint32_t ATOM_B = (BN / 2) * 128;
  static constexpr uint32_t A_BYTES = KA * ATOM_A;
  static constexpr uint32_t B_BYTES = KA * ATOM_B;
  static constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr uint32_t TMEM_COLS = tmem_cols_for(2 * BN);
  static constexpr int CW = 16;                         // columns per epilogue chunk
  static constexpr int NCH = BN / CW;
  static constexpr int PART_CH = (NCH + 1) / 2;
  static constexpr uint32_t STG_BYTES = 32 * CW * 4;     // one 32-row staging tile (fp32 size)
  // bytes of one staging row of the stored type (fp32 64, bf16 32): also the TMA swizzle span
  static constexpr int ROW_BYTES = CW * (RES ? 4 : 2);
  // staging tiles per epilogue warp: two alternating ones, or, with a residual, one per
  // chunk of the warp's tile share so the whole residual share is loaded ahead of the MMA
  // with a residual, up to four staging tiles per warp hold the residual chunks loaded ahead;
  // a fifth chunk reuses the first tile once its store has read it
  static constexpr int NBUF = RES ? (PART_CH < 4 ? PART_CH : 4) : 2;
  static constexpr uint32_t EPI_BYTES = EPI_WARPS * NBUF * STG_BYTES;
  static constexpr uint32_t NUM_BARS = 2 * STAGES + 5 + NBUF * EPI_WARPS;
  static constexpr size_t SMEM = 1024 + (size_t)STAGES * STAGE_BYTES + EPI_BYTES + NUM_BARS * 8 + 16;
  static constexpr uint32_t IDESC = ptx::idesc_bf16_f32(2 * BMC, BN);
  static_assert(BN % 16 == 0 && BN >= 32 && BN <= 256, "UMMA N for M=256");
  static_assert((BN / 2) % 8 == 0, "B half-tile rows must fill 8-row swizzle atoms");
  static_assert(SMEM <= 232448, "shared memory");
};

__device__ __forceinline__ void record_timeout(DevError* err, int where, volatile int* abort) {
  *abort = 1;
  if (err && atomicCAS(&err->code, 0, KIMODO_ETIMEOUT_CODE) == 0) {
    err->where = where;
    err->block = blockIdx.x;
  }
}

template <int BN, int STAGES, int KIND, typename OutT>
__global__ void __launch_bounds__(NUM_THREADS, 1)
gemm_tc2_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const __grid_constant__ CUtensorMap tmO, const __grid_constant__ CUtensorMap tmR,
                int num_m_tiles, int num_n_tiles, int num_kb, EpiParams ep, DevError* err) {
  using C = Tc2Cfg<BN, STAGES, KIND>;
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
  auto res_bar = [&](int ew, int b) { return bar0 + 8u * (2 * STAGES + 5 + C::NBUF * ew + b); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::NUM_BARS);
  volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = ptx::cluster_ctarank();
  const int pair = blockIdx.x >> 1;
  const int npairs = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      ptx::mbar_init(full_bar(s), 1);
      ptx::mbar_init(empty_bar(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      ptx::mbar_init(tfull_bar(a), 1);
      ptx::mbar_init(tempty_bar(a), 2 * EPI_WARPS);
    }
    ptx::mbar_init(drain_bar, 1);
    for (int i = 0; i < C::NBUF * EPI_WARPS; ++i) ptx::mbar_init(res_bar(i / C::NBUF, i % C::NBUF), 1);
    ptx::fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    ptx::tma_prefetch_desc(&tmA);
    ptx::tma_prefetch_desc(&tmB);
    ptx::tma_prefetch_desc(&tmO);
    if (C::RES) ptx::tma_prefetch_desc(&tmR);
    // The weights do not depend on the previous kernel: while it still runs, the CTAs
    // together pull this launch's whole weight matrix into L2 (one box of 64 columns x
    // BN / 2 rows per CTA and step), so the first tiles of every round find it there.
    const int nbr = (ep.N + BN / 2 - 1) / (BN / 2);   // row boxes covering N
    const int nkc = num_kb * C::KA;                      // column boxes covering K
    for (int i = blockIdx.x; i < nbr * nkc; i += gridDim.x)
      ptx::tma_prefetch_l2_2d(&tmB, (i % nkc) * BK, (i / nkc) * (BN / 2));
  }
  if (warp == 1) {
    ptx::tmem_alloc_pair(ptx::smem_u32(tmem_slot), C::TMEM_COLS);
    ptx::tmem_relinquish_pair();
  }
  // prologue done: let the next kernel launch, then wait for the previous one
  ptx::pdl_trigger();
  ptx::pdl_wait();
  // A launch after a recorded timeout does no work; both CTAs of a pair read the
  // same word (written by an earlier kernel, visible after the wait), so they agree.
  if (threadIdx.x == 0) *abort = (err != nullptr && *reinterpret_cast<volatile int*>(&err->code) != 0) ? 1 : 0;
  ptx::tc_fence_before();
  __syncwarp();
  ptx::cluster_sync();
  ptx::tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int num_tiles = *abort ? 0 : num_m_tiles * num_n_tiles;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer (both CTAs)
      int stage = 0;
      uint32_t phase = 0;
      long issued = 0;
      bool ok = true;
      for (int tile = pair; tile < num_tiles && ok; tile += npairs) {
        const int m_blk = tile % num_m_tiles, n_blk = tile / num_m_tiles;
        const int arow = m_blk * 2 * BMC + (int)rank * BMC;
        const int brow = n_blk * BN + (int)rank * (BN / 2);
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!ptx::mbar_wait_bounded(empty_bar(stage), phase ^ 1u, abort, WAIT_LIMIT_NS)) {
            ok = false;
            break;
          }
          if (rank == 0) ptx::mbar_arrive_expect_tx(full_bar(stage), 2 * C::STAGE_BYTES);
          const uint32_t lbar = ptx::mapa_shared(full_bar(stage), 0);
#pragma unroll
          for (int at = 0; at < C::KA; ++at) {
            ptx::tma_load_2d_pair(sA + stage * C::A_BYTES + at * C::ATOM_A, &tmA, lbar, (kb * C::KA + at) * BK, arow);
            ptx::tma_load_2d_pair(sB + stage * C::B_BYTES + at * C::ATOM_B, &tmB, lbar, (kb * C::KA + at) * BK, brow);
          }
          ++issued;
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      if (!ok) {
        if (!*abort) record_timeout(err, WHERE_GEMM_PRODUCER, abort);
        if (rank == 0) {   // the leader's full barriers count both CTAs' loads
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
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      // ---------------- MMA issuer (leader CTA)
      int stage = 0;
      uint32_t phase = 0;
      int local = 0;
      bool ok = true;
      for (int tile = pair; tile < num_tiles && ok; tile += npairs, ++local) {
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
          for (int k = 0; k < C::KA * BK / 16; ++k)
            ptx::tc_mma_bf16_pair(d_tmem, ptx::smem_desc_sw128(a0 + (k >> 2) * C::ATOM_A + (k & 3) * 32),
                                  ptx::smem_desc_sw128(b0 + (k >> 2) * C::ATOM_B + (k & 3) * 32), C::IDESC,
                                  (kb | k) != 0);
          ptx::tc_commit_pair(empty_bar(stage), 0x3);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        ptx::tc_commit_pair(tfull_bar(acc), 0x3);
      }
      if (!ok && !*abort) record_timeout(err, WHERE_GEMM_MMA, abort);
      ptx::tc_commit_pair(drain_bar, 0x1);
      volatile int never = 0;
      if (!ptx::mbar_wait_bounded(drain_bar, 0, &never, WAIT_LIMIT_NS)) record_timeout(err, WHERE_GEMM_DRAIN, abort);
    }
  } else {
    // ---------------- epilogue warps 2..9: TMEM lane quarter = warp % 4; part (warp - 2) / 4
    // takes chunks [part * PART_CH, ...) of the tile's BN / 16 column chunks.  Per chunk each
    // thread finishes its accumulator row (bias, activation, residual) in registers and
    // writes it into a swizzled 32 x 16 staging tile; one lane stores the tile with TMA.  Two
    // staging tiles per warp alternate; the residual chunk arrives in the staging tile by TMA.
    const int quarter = warp & 3;
    const int ew = warp - 2;
    const int part = ew >> 2;
    constexpr int CW = C::CW;
    uint8_t* stg_base = smem + STAGES * C::STAGE_BYTES + ew * C::NBUF * C::STG_BYTES;
    const uint32_t leader_tempty0 = ptx::mapa_shared(tempty_bar(0), 0);
    const uint32_t leader_tempty1 = ptx::mapa_shared(tempty_bar(1), 0);
    int cc = 0;   // chunks processed by this warp so far: staging tile cc & 1
    int local = 0;
    bool failed = false;
    for (int tile = pair; tile < num_tiles && !failed; tile += npairs, ++local) {
      const int acc = local & 1;
      const uint32_t acc_phase = (local >> 1) & 1;
      const int m_blk = tile % num_m_tiles, n_blk = tile / num_m_tiles;
      const int row0 = m_blk * 2 * BMC + (int)rank * BMC + quarter * 32;
      const int cbeg = min(part * C::PART_CH * CW, BN);
      const int cend = min(cbeg + C::PART_CH * CW, BN);
      const int valid_end = min(cend, ep.N - n_blk * BN);
      // a warp whose 32 rows all lie past M issues no loads or stores for this tile
      const int nch = (valid_end > cbeg && row0 < ep.M) ? (valid_end - cbeg + CW - 1) / CW : 0;
      const int gcol = n_blk * BN + cbeg;
      // chunk k of this tile is the warp's chunk number cc0 + k and uses staging tile (cc0 + k) % NBUF
      const int cc0 = cc;
      auto stage_tile = [&](int a) { return stg_base + (a % C::NBUF) * C::STG_BYTES; };
      // per-column operands of chunk k: bias, and for EPI_BIAS_RESID_LN the LayerNorm gamma and
      // (bias + beta), so that x = acc + (bias + beta) + (z * rstd - mean * rstd) * gamma
      auto load_bias = [&](int k, float4 (&b4)[CW / 4], float4 (&g4)[CW / 4]) {
#pragma unroll
        for (int j = 0; j < CW / 4; ++j) {
          b4[j] = ld4(ep.bias + gcol + k * CW + 4 * j);
          if constexpr (KIND == EPI_BIAS_RESID_LN) {
            const float4 be = ld4(ep.ln_b + gcol + k * CW + 4 * j);
            b4[j].x += be.x; b4[j].y += be.y; b4[j].z += be.z; b4[j].w += be.w;
            g4[j] = ld4(ep.ln_g + gcol + k * CW + 4 * j);
          }
        }
      };
      // this lane's row statistics for EPI_BIAS_RESID_LN: z * rs_a + rs_b = (z - mean) / std
      float rs_a = 1.f, rs_b = 0.f;
      if constexpr (KIND == EPI_BIAS_RESID_LN) {
        const int row = row0 + lane;
        if (nch > 0 && row < ep.M) {
          const float2 st2 = *reinterpret_cast<const float2*>(ep.ln_stats + 2 * (long)row);
          rs_a = st2.y;
          rs_b = -st2.x * st2.y;
        }
      }
      float4 ba[CW / 4], bb[CW / 4], ga[CW / 4], gb[CW / 4];
      if (nch > 0) {
        if (C::RES && lane == 0) {
          // the residual chunks of this tile, one staging tile each (up to NBUF), loaded while
          // the MMAs run; the previous tile's stores have read their staging tiles first
          ptx::bulk_wait_read<0>();
          for (int k = 0; k < nch && k < C::NBUF; ++k) {
            const int b = (cc0 + k) % C::NBUF;
            ptx::mbar_arrive_expect_tx(res_bar(ew, b), 32 * CW * 4);
            ptx::tma_load_2d(ptx::smem_u32(stage_tile(cc0 + k)), &tmR, res_bar(ew, b), gcol + k * CW, row0);
          }
        }
        load_bias(0, ba, ga);
      }
      if (!ptx::mbar_wait_bounded(tfull_bar(acc), acc_phase, abort, WAIT_LIMIT_NS)) {
        if (!*abort) record_timeout(err, WHERE_GEMM_EPILOGUE, abort);
        failed = true;
        break;
      }
      ptx::tc_fence_after();
      const uint32_t taddr = tmem_base + ((uint32_t)(quarter * 32) << 16) + acc * BN + cbeg;
      auto release = [&]() {
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive_remote(acc ? leader_tempty1 : leader_tempty0);
      };
      if (nch == 0) {
        release();
        continue;
      }
      // finish chunk k (the warp's chunk number cc == cc0 + k) from accumulator values v, bias b4
      auto process = [&](float (&v)[CW], const float4 (&b4)[CW / 4], const float4 (&g4)[CW / 4], int k) -> bool {
        uint8_t* st = stage_tile(cc);
        // this lane's row of the staging tile; its 16-byte unit u sits at unit u ^ swz
        // (the tile's TMA swizzle, so that the warp's row-per-lane accesses hit distinct banks)
        uint8_t* srow = st + lane * C::ROW_BYTES;
        const int swz = C::ROW_BYTES == 64 ? (lane >> 1) & 3 : (lane >> 2) & 1;
        float x[CW];
#pragma unroll
        for (int j = 0; j < CW / 4; ++j) {
          x[4 * j] = v[4 * j] + b4[j].x;
          x[4 * j + 1] = v[4 * j + 1] + b4[j].y;
          x[4 * j + 2] = v[4 * j + 2] + b4[j].z;
          x[4 * j + 3] = v[4 * j + 3] + b4[j].w;
        }
        if constexpr (KIND == EPI_BIAS_GELU) {
#pragma unroll
          for (int j = 0; j < CW; j += 2) gelu2_as7128(x[j], x[j + 1]);
        }
        if constexpr (KIND == EPI_BIAS_SILU) {
#pragma unroll
          for (int j = 0; j < CW; ++j) x[j] = silu_f(x[j]);
        }
        if constexpr (C::RES) {
          if (!ptx::mbar_wait_bounded(res_bar(ew, cc % C::NBUF), (cc / C::NBUF) & 1, abort, WAIT_LIMIT_NS))
            return false;
#pragma unroll
          for (int u = 0; u < CW / 4; ++u) {
            float4 r = *reinterpret_cast<const float4*>(srow + ((u ^ swz) << 4));
            if constexpr (KIND == EPI_BIAS_RESID_LN) {
              r.x = fmaf(r.x, rs_a, rs_b) * g4[u].x; r.y = fmaf(r.y, rs_a, rs_b) * g4[u].y;
              r.z = fmaf(r.z, rs_a, rs_b) * g4[u].z; r.w = fmaf(r.w, rs_a, rs_b) * g4[u].w;
            }
            x[4 * u] += r.x; x[4 * u + 1] += r.y; x[4 * u + 2] += r.z; x[4 * u + 3] += r.w;
          }
        } else {
          if (lane == 0) ptx::bulk_wait_read<1>();   // store of chunk cc - 2 has read this tile
          __syncwarp();
        }
        if constexpr (std::is_same<OutT, float>::value) {
#pragma unroll
          for (int u = 0; u < CW / 4; ++u)
            *reinterpret_cast<float4*>(srow + ((u ^ swz) << 4)) =
                make_float4(x[4 * u], x[4 * u + 1], x[4 * u + 2], x[4 * u + 3]);
        } else {
#pragma unroll
          for (int u = 0; u < CW / 8; ++u)
            *reinterpret_cast<uint4*>(srow + ((u ^ swz) << 4)) =
                make_uint4(bf16x2_bits(x[8 * u], x[8 * u + 1]), bf16x2_bits(x[8 * u + 2], x[8 * u + 3]),
                           bf16x2_bits(x[8 * u + 4], x[8 * u + 5]), bf16x2_bits(x[8 * u + 6], x[8 * u + 7]));
        }
        ptx::fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          ptx::tma_store_2d(&tmO, ptx::smem_u32(st), gcol + k * CW, row0);
          ptx::bulk_commit();
          if (C::RES && k + C::NBUF < nch) {
            // residual chunk k + NBUF into this staging tile once the store has read it
            ptx::bulk_wait_read<0>();
            const int b = cc % C::NBUF;
            ptx::mbar_arrive_expect_tx(res_bar(ew, b), 32 * CW * 4);
            ptx::tma_load_2d(ptx::smem_u32(st), &tmR, res_bar(ew, b), gcol + (k + C::NBUF) * CW, row0);
          }
        }
        ++cc;
        return true;
      };
      float va[CW], vb[CW];
      ptx::tmem_ld(taddr, va);
#pragma unroll 1
      // The accumulator is released after the last chunk's stores are issued, not before: the
      // remote arrive takes most of a microsecond, which at the last tile of a launch would
      // delay its last stores, while the MMAs that wait for it start a tile later anyway.
      for (int c = 0; c < nch; c += 2) {
        ptx::tmem_ld_wait();
        if (c + 1 < nch) {
          ptx::tmem_ld(taddr + (c + 1) * CW, vb);
          load_bias(c + 1, bb, gb);
        }
        if (!process(va, ba, ga, c)) { failed = true; break; }
        if (c == nch - 1) release();
        if (c + 1 >= nch) break;
        ptx::tmem_ld_wait();
        if (c + 2 < nch) {
          ptx::tmem_ld(taddr + (c + 2) * CW, va);
          load_bias(c + 2, ba, ga);
        }
        if (!process(vb, bb, gb, c + 1)) { failed = true; break; }
        if (c + 1 == nch - 1) release();
      }
      if (failed && !*abort) record_timeout(err, WHERE_GEMM_EPILOGUE, abort);
    }
    if (lane == 0) ptx::bulk_wait_all();
    __syncwarp();
  }

  // both CTAs finish every access to the pair's shared memory and TMEM before either leaves
  ptx::tc_fence_before();
  __syncwarp();
  ptx::cluster_sync();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc_pair(tmem_base, C::TMEM_COLS);
  }
}

// ------------------------------------------------------------------ host side

template <int BN, int STAGES, int KIND, typename OutT>
struct Tc2Launcher {
  static int max_clusters;
  static cudaError_t prepare() {
    using Cf = Tc2Cfg<BN, STAGES, KIND>;
    auto kern = gemm_tc2_kernel<BN, STAGES, KIND, OutT>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Cf::SMEM);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 0);
    cudaGetLastError();
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(2 * 74);
    cfg.blockDim = dim3(NUM_THREADS);
    cfg.dynamicSmemBytes = Cf::SMEM;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    e = cudaOccupancyMaxActiveClusters(&n, kern, &cfg);
    if (e != cudaSuccess || n < 1) {
      cudaGetLastError();
      n = 0;
    }
    max_clusters = n;
    return cudaSuccess;
  }
  static cudaError_t launch(const GemmArgs& g, const EpiParams& ep, DevError* err, cudaStream_t st) {
    using Cf = Tc2Cfg<BN, STAGES, KIND>;
    if (max_clusters < 1) return cudaErrorInvalidConfiguration;
    CUtensorMap ta, tb, to, tr;
    if (make_tmap_bf16(&ta, g.A, g.M, g.K, g.lda, BMC) || make_tmap_bf16(&tb, g.B, g.N, g.K, g.ldb, BN / 2))
      return cudaErrorInvalidValue;
    static_assert(Cf::ROW_BYTES == Cf::CW * (int)sizeof(OutT), "staging row bytes");
    if (make_tmap_plain(&to, ep.out, (int)sizeof(OutT), g.M, g.N, ep.ldo, Cf::CW, 32, Cf::ROW_BYTES))
      return cudaErrorInvalidValue;
    if (Cf::RES) {
      if (make_tmap_plain(&tr, ep.resid, 4, g.M, g.N, ep.ldr, Cf::CW, 32, Cf::ROW_BYTES)) return cudaErrorInvalidValue;
    } else {
      tr = to;
    }
    const int mt = (g.M + 2 * BMC - 1) / (2 * BMC), nt = (g.N + BN - 1) / BN;
    const int tiles = mt * nt;
    const int pairs = tiles < max_clusters ? tiles : max_clusters;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.gridDim = dim3(2 * pairs);
    cfg.blockDim = dim3(NUM_THREADS);
    cfg.dynamicSmemBytes = Cf::SMEM;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = pdl_enabled() ? 2 : 1;
    return cudaLaunchKernelEx(&cfg, gemm_tc2_kernel<BN, STAGES, KIND, OutT>, ta, tb, to, tr, mt, nt,
                              (g.K + Cf::KA * BK - 1) / (Cf::KA * BK), ep, err);
  }
};
template <int BN, int STAGES, int KIND, typename OutT>
int Tc2Launcher<BN, STAGES, KIND, OutT>::max_clusters = 0;

// Pipeline stages of a (tile N, epilogue) instantiation: as many as fit in the shared
// memory left by the epilogue staging tiles, at most 8.
template <int BN, int KIND>
constexpr int tc2_stages() {
  using C1 = Tc2Cfg<BN, 1, KIND>;
  const long fixed = 1024 + (long)C1::EPI_BYTES + (5 + C1::NBUF * EPI_WARPS) * 8 + 16;
  const long st = (232448 - fixed) / ((long)C1::STAGE_BYTES + 16);
  return st > 8 ? 8 : (int)st;
}
#define KD_TC2_ST(BN_, KIND_) tc2_stages<BN_, KIND_>()

// (tile N, epilogue, output type) per instantiation
#define KD_TC2_LIST(X)                                                                     \
  X(256, KD_TC2_ST(256, EPI_BIAS), EPI_BIAS, bf16)                                         \
  X(208, KD_TC2_ST(208, EPI_BIAS), EPI_BIAS, bf16)                                         \
  X(160, KD_TC2_ST(160, EPI_BIAS), EPI_BIAS, bf16)                                         \
  X(144, KD_TC2_ST(144, EPI_BIAS), EPI_BIAS, bf16)                                         \
  X(256, KD_TC2_ST(256, EPI_BIAS_GELU), EPI_BIAS_GELU, bf16)                               \
  X(208, KD_TC2_ST(208, EPI_BIAS_GELU), EPI_BIAS_GELU, bf16)                               \
  X(160, KD_TC2_ST(160, EPI_BIAS_GELU), EPI_BIAS_GELU, bf16)                               \
  X(144, KD_TC2_ST(144, EPI_BIAS_GELU), EPI_BIAS_GELU, bf16)                               \
  X(160, KD_TC2_ST(160, EPI_BIAS_RESID), EPI_BIAS_RESID, float)                            \
  X(144, KD_TC2_ST(144, EPI_BIAS_RESID), EPI_BIAS_RESID, float)                            \
  X(160, KD_TC2_ST(160, EPI_BIAS_RESID_LN), EPI_BIAS_RESID_LN, float)                      \
  X(144, KD_TC2_ST(144, EPI_BIAS_RESID_LN), EPI_BIAS_RESID_LN, float)

}  // namespace

cudaError_t gemm_tc2_prepare() {
#define KD_PREP(BN_, ST_, KIND_, OUT_)                                        \
  {                                                                          \
    cudaError_t e_ = Tc2Launcher<BN_, ST_, KIND_, OUT_>::prepare();          \
    if (e_ != cudaSuccess) return e_;                                        \
  }
  KD_TC2_LIST(KD_PREP)
#undef KD_PREP
  return cudaSuccess;
}

bool gemm_tc2_supports(int kind, bool out_f32) {
  return (kind == EPI_BIAS && !out_f32) || (kind == EPI_BIAS_GELU && !out_f32) ||
         ((kind == EPI_BIAS_RESID || kind == EPI_BIAS_RESID_LN) && out_f32);
}

// Tile N minimizing (rounds of pair tiles) x (N + per-tile overhead) over the available
// CTA pairs; the overhead (prologue, pipeline fill, last epilogue) was measured to be worth
// about 160 columns of MMA time per tile at K = 1024.
int gemm_tc2_pick_bn(int M, int N, int kind) {
  const int all[4] = {256, 208, 160, 144};
  const int resid[2] = {160, 144};
  const bool res = kind == EPI_BIAS_RESID || kind == EPI_BIAS_RESID_LN;
  const int* cands = res ? resid : all;
  const int ncand = res ? 2 : 4;
  using L256 = Tc2Launcher<256, KD_TC2_ST(256, EPI_BIAS), EPI_BIAS, bf16>;
  const int pairs = L256::max_clusters > 0 ? L256::max_clusters : 74;
  const long mt = (M + 2 * BMC - 1) / (2 * BMC);
  int best = cands[0];
  long best_cost = -1;
  for (int i = 0; i < ncand; ++i) {
    const int bn = cands[i];
    const long tiles = mt * ((N + bn - 1) / bn);
    const long rounds = (tiles + pairs - 1) / pairs;
    const long cost = rounds * (bn + 160);
    if (best_cost < 0 || cost < best_cost) {
      best_cost = cost;
      best = bn;
    }
  }
  return best;
}

cudaError_t gemm_tc2(const GemmArgs& g, int bn, int kind, bool out_f32, const EpiParams& ep, DevError* err,
                     cudaStream_t st) {
  if (g.M <= 0 || g.N <= 0) return cudaSuccess;
  if (g.K <= 0 || g.N % 16) return cudaErrorInvalidValue;
#define KD_RUN(BN_, ST_, KIND_, OUT_)                                            \
  if (bn == BN_ && kind == KIND_ && out_f32 == std::is_same<OUT_, float>::value) \
    return Tc2Launcher<BN_, ST_, KIND_, OUT_>::launch(g, ep, err, st);
  KD_TC2_LIST(KD_RUN)
#undef KD_RUN
  return cudaErrorInvalidValue;
}

}  // namespace kd
