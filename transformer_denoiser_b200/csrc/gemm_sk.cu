// Stream-K tensor-core GEMM on CTA pairs (tcgen05 cta_group::2) for the large
// per-layer projections: D[M,N] = A[M,K] . B[N,K]^T + fused epilogue, bf16 in,
// fp32 accumulate, 256 x 256 output tiles.
//
// The work is the list of (tile, k-block) units, tile-major.  Each of the P
// persistent CTA pairs takes one contiguous, equal share of it (units
// [p U / P, (p + 1) U / P)), so every pair does the same number of MMAs whatever
// the tile count: no partial last wave.  A share covers whole tiles plus at most
// a tail of the tile where it starts and a head of the tile where it ends.  The
// pair whose share holds a tile's last k-block finishes that tile: the other
// pairs that worked on it (its contributors) leave fp32 partial accumulators in a
// workspace slot of their own and raise a per-CTA counter; the finisher adds them
// before its epilogue.  A pair runs its contribution first, its whole tiles next
// and its finishing part last, so partial sums are ready long before they are
// read and no pair waits on one that is itself waiting.
//
// Per pair as in the 256-row pair GEMM: each CTA stages 128 rows of A and 128 rows
// of B per k-block by TMA (128-byte swizzle, no multicast); the leader issues one
// 256 x 256 x 16 MMA per K step over both CTAs' shared memory and commits to both
// CTAs' barriers; two 256-column TMEM accumulators per CTA; 8 epilogue warps
// finish rows from TMEM in registers (bias, GELU, residual read straight from
// global memory) and store 32 x 16 swizzled staging tiles by TMA.  Every wait is
// bounded; a timeout is recorded in the device error word.
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

constexpr int BMC = 128;                        // rows per CTA (256 per pair)
constexpr int BK = 64;
constexpr int BN = 256;
constexpr int STAGES = 5;
constexpr int EPI_WARPS = 8;
constexpr int NUM_THREADS = 64 + 32 * EPI_WARPS;
constexpr uint64_t WAIT_LIMIT_NS = 2000000000ull;
constexpr int KIMODO_ETIMEOUT_CODE = -5;

constexpr uint32_t A_BYTES = BMC * BK * 2;
constexpr uint32_t B_BYTES = (BN / 2) * BK * 2;
constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES;
constexpr uint32_t TMEM_COLS = 2 * BN;
constexpr int CW = 16;                          // columns per epilogue chunk
constexpr int PART_CH = BN / CW / 2;            // chunks per epilogue warp (two warps per lane quarter)
constexpr uint32_t STG_BYTES = 32 * CW * 4;     // one 32-row staging tile (fp32 size)
constexpr int NBUF = 2;
constexpr uint32_t EPI_BYTES = EPI_WARPS * NBUF * STG_BYTES;
constexpr uint32_t NUM_BARS = 2 * STAGES + 5;
constexpr size_t SMEM = 1024 + (size_t)STAGES * STAGE_BYTES + EPI_BYTES + NUM_BARS * 8 + 16;
constexpr uint32_t IDESC = ptx::idesc_bf16_f32(2 * BMC, BN);
constexpr int CTA_PARTIAL = BMC * BN;           // floats of one CTA's partial accumulator
constexpr int WARP_PARTIAL = 32 * CW * PART_CH; // floats of one epilogue warp's share of it
static_assert(SMEM <= 232448, "shared memory");

enum Role : int { FULL = 0, CONTRIB = 1, FINISH = 2 };

// Equal contiguous shares of U units over P pairs.
struct Shares {
  long U;
  int P;
  __device__ long begin(int p) const { return (long)p * U / P; }
  __device__ int owner(long u) const {   // the pair whose share holds unit u
    int p = (int)((u * P) / U);
    while (p + 1 < P && begin(p + 1) <= u) ++p;
    while (p > 0 && begin(p) > u) --p;
    return p;
  }
};

struct Unit {
  int tile, kb0, kb1, role;
};

// The units of one pair in processing order: contribution, whole tiles, finishing part.
struct PairWork {
  int n = 0;
  int KB, t_first, k_first, t_last, k_end, full_lo, n_full;
  bool single, has_contrib, has_finish;
  __device__ void init(const Shares& s, int p, int kb) {
    KB = kb;
    const long a = s.begin(p), b = s.begin(p + 1);
    if (b <= a) return;
    t_first = (int)(a / KB);
    k_first = (int)(a % KB);
    t_last = (int)((b - 1) / KB);
    k_end = (int)((b - 1) % KB) + 1;
    single = t_first == t_last;
    if (single) {
      n = 1;
      return;
    }
    has_contrib = k_end < KB;
    has_finish = k_first > 0;
    full_lo = has_finish ? t_first + 1 : t_first;
    const int full_hi = has_contrib ? t_last - 1 : t_last;
    n_full = full_hi >= full_lo ? full_hi - full_lo + 1 : 0;
    n = (int)has_contrib + n_full + (int)has_finish;
  }
  __device__ Unit get(int i) const {
    if (single) return {t_first, k_first, k_end, k_end == KB ? (k_first == 0 ? FULL : FINISH) : CONTRIB};
    if (has_contrib) {
      if (i == 0) return {t_last, 0, k_end, CONTRIB};
      --i;
    }
    if (i < n_full) return {full_lo + i, 0, KB, FULL};
    return {t_first, k_first, KB, FINISH};
  }
};

__device__ __forceinline__ void record_timeout(DevError* err, int where, volatile int* abort) {
  *abort = 1;
  if (err && atomicCAS(&err->code, 0, KIMODO_ETIMEOUT_CODE) == 0) {
    err->where = where;
    err->block = blockIdx.x;
  }
}

__device__ __forceinline__ int ld_acquire(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ float4 ld_cg4(const float* p) {
  float4 v;
  asm volatile("ld.global.cg.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "l"(p) : "memory");
  return v;
}

// Bounded wait until *flag >= target (a counter raised by other CTAs of this grid).
__device__ __forceinline__ bool wait_flag(const int* flag, int target, volatile int* abort) {
  if (ld_acquire(flag) >= target) return true;
  const uint64_t t0 = ptx::global_timer_ns();
  for (uint32_t it = 1;; ++it) {
    __nanosleep(64);
    if (ld_acquire(flag) >= target) return true;
    if ((it & 15u) == 0) {
      if (*abort) return false;
      if (ptx::global_timer_ns() - t0 > WAIT_LIMIT_NS) return false;
    }
  }
}

template <int KIND, typename OutT>
__global__ void __launch_bounds__(NUM_THREADS, 1)
gemm_sk_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
               const __grid_constant__ CUtensorMap tmO, int num_m_tiles, int num_n_tiles, int num_kb,
               EpiParams ep, float* __restrict__ partial, int* __restrict__ flags, DevError* err) {
  constexpr int ROW_BYTES = CW * (int)sizeof(OutT);   // staging row = TMA swizzle span
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sA = ptx::smem_u32(smem);
  const uint32_t sB = sA + STAGES * A_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES + EPI_BYTES);
  const uint32_t bar0 = ptx::smem_u32(bars);
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (STAGES + s); };
  auto tfull_bar = [&](int a) { return bar0 + 8u * (2 * STAGES + a); };
  auto tempty_bar = [&](int a) { return bar0 + 8u * (2 * STAGES + 2 + a); };
  const uint32_t drain_bar = bar0 + 8u * (2 * STAGES + 4);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + NUM_BARS);
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
    ptx::fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    ptx::tma_prefetch_desc(&tmA);
    ptx::tma_prefetch_desc(&tmB);
    ptx::tma_prefetch_desc(&tmO);
  }
  if (warp == 1) {
    ptx::tmem_alloc_pair(ptx::smem_u32(tmem_slot), TMEM_COLS);
    ptx::tmem_relinquish_pair();
  }
  ptx::pdl_trigger();
  ptx::pdl_wait();
  // a launch after a recorded timeout does no work (both CTAs of a pair read the same word)
  if (threadIdx.x == 0) *abort = (err != nullptr && *reinterpret_cast<volatile int*>(&err->code) != 0) ? 1 : 0;
  ptx::tc_fence_before();
  __syncwarp();
  ptx::cluster_sync();
  ptx::tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const Shares shares{(long)num_m_tiles * num_n_tiles * num_kb, npairs};
  PairWork work;
  if (!*abort) work.init(shares, pair, num_kb);

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer (both CTAs)
      int stage = 0;
      uint32_t phase = 0;
      long issued = 0;
      bool ok = true;
      for (int i = 0; i < work.n && ok; ++i) {
        const Unit u = work.get(i);
        const int m_blk = u.tile % num_m_tiles, n_blk = u.tile / num_m_tiles;
        const int arow = m_blk * 2 * BMC + (int)rank * BMC;
        const int brow = n_blk * BN + (int)rank * (BN / 2);
        for (int kb = u.kb0; kb < u.kb1; ++kb) {
          if (!ptx::mbar_wait_bounded(empty_bar(stage), phase ^ 1u, abort, WAIT_LIMIT_NS)) {
            ok = false;
            break;
          }
          if (rank == 0) ptx::mbar_arrive_expect_tx(full_bar(stage), 2 * STAGE_BYTES);
          const uint32_t lbar = ptx::mapa_shared(full_bar(stage), 0);
          ptx::tma_load_2d_pair(sA + stage * A_BYTES, &tmA, lbar, kb * BK, arow);
          ptx::tma_load_2d_pair(sB + stage * B_BYTES, &tmB, lbar, kb * BK, brow);
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
      bool ok = true;
      for (int i = 0; i < work.n && ok; ++i) {
        const Unit u = work.get(i);
        const int acc = i & 1;
        const uint32_t acc_phase = (i >> 1) & 1;
        if (!ptx::mbar_wait_bounded(tempty_bar(acc), acc_phase ^ 1u, abort, WAIT_LIMIT_NS)) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        for (int kb = u.kb0; kb < u.kb1; ++kb) {
          if (!ptx::mbar_wait_bounded(full_bar(stage), phase, abort, WAIT_LIMIT_NS)) {
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          const uint32_t a0 = sA + stage * A_BYTES;
          const uint32_t b0 = sB + stage * B_BYTES;
#pragma unroll
          for (int k = 0; k < BK / 16; ++k)
            ptx::tc_mma_bf16_pair(d_tmem, ptx::smem_desc_sw128(a0 + k * 32), ptx::smem_desc_sw128(b0 + k * 32), IDESC,
                                  (kb != u.kb0 || k != 0) ? 1u : 0u);
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
    // ---------------- epilogue warps 2..9: TMEM lane quarter = warp % 4, column half = (warp - 2) / 4
    const int quarter = warp & 3;
    const int ew = warp - 2;
    const int part = ew >> 2;
    uint8_t* stg_base = smem + STAGES * STAGE_BYTES + ew * NBUF * STG_BYTES;
    const uint32_t leader_tempty0 = ptx::mapa_shared(tempty_bar(0), 0);
    const uint32_t leader_tempty1 = ptx::mapa_shared(tempty_bar(1), 0);
    const int swz = ROW_BYTES == 64 ? (lane >> 1) & 3 : (lane >> 2) & 1;
    int cc = 0;   // chunks stored by this warp so far: staging tile cc % NBUF
    bool failed = false;
    for (int i = 0; i < work.n && !failed; ++i) {
      const Unit u = work.get(i);
      const int acc = i & 1;
      const uint32_t acc_phase = (i >> 1) & 1;
      const int m_blk = u.tile % num_m_tiles, n_blk = u.tile / num_m_tiles;
      const int row0 = m_blk * 2 * BMC + (int)rank * BMC + quarter * 32;
      const int cbeg = part * PART_CH * CW;
      const int gcol = n_blk * BN + cbeg;
      const int row = row0 + lane;
      const bool row_ok = row < ep.M;
      const int valid_end = min(cbeg + PART_CH * CW, ep.N - n_blk * BN);
      // chunks this warp stores (none when all its rows or columns lie outside the output)
      const int nch = (u.role != CONTRIB && valid_end > cbeg && row0 < ep.M) ? (valid_end - cbeg + CW - 1) / CW : 0;
      const uint32_t taddr = tmem_base + ((uint32_t)(quarter * 32) << 16) + acc * BN + cbeg;
      auto release = [&]() {
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive_remote(acc ? leader_tempty1 : leader_tempty0);
      };
      // per-thread operand loads of chunk k: bias and (for the residual kind) the row's residual
      auto load_operands = [&](int k, float4 (&b4)[CW / 4], float4 (&r4)[CW / 4]) {
#pragma unroll
        for (int j = 0; j < CW / 4; ++j) {
          b4[j] = ld4(ep.bias + gcol + k * CW + 4 * j);
          if constexpr (KIND == EPI_BIAS_RESID)
            r4[j] = row_ok ? ld4(reinterpret_cast<const float*>(ep.resid) + (long)row * ep.ldr + gcol + k * CW + 4 * j)
                           : make_float4(0.f, 0.f, 0.f, 0.f);
        }
      };
      float4 ba[CW / 4], bb[CW / 4], ra[CW / 4], rb[CW / 4];
      if (nch > 0) load_operands(0, ba, ra);
      if (!ptx::mbar_wait_bounded(tfull_bar(acc), acc_phase, abort, WAIT_LIMIT_NS)) {
        if (!*abort) record_timeout(err, WHERE_GEMM_EPILOGUE, abort);
        failed = true;
        break;
      }
      ptx::tc_fence_after();

      if (u.role == CONTRIB) {
        // leave this CTA's partial accumulator in the pair's slot, then raise the CTA's counter
        float* dst = partial + ((size_t)pair * 2 + rank) * CTA_PARTIAL + (size_t)ew * WARP_PARTIAL;
        float va[CW];
        for (int k = 0; k < PART_CH; ++k) {
          ptx::tmem_ld(taddr + k * CW, va);
          ptx::tmem_ld_wait();
          if (k == PART_CH - 1) release();
#pragma unroll
          for (int j = 0; j < CW / 4; ++j)
            *reinterpret_cast<float4*>(dst + (k * (CW / 4) + j) * 128 + lane * 4) =
                make_float4(va[4 * j], va[4 * j + 1], va[4 * j + 2], va[4 * j + 3]);
        }
        __syncwarp();
        if (lane == 0) {
          __threadfence();   // the warp's partial-sum stores before its count
          atomicAdd(flags + pair * 2 + rank, 1);
        }
        continue;
      }

      // contributors of a finished tile: the pairs before this one whose shares reach into it
      int c_lo = pair, c_hi = pair;
      if (u.role == FINISH) {
        c_lo = shares.owner((long)u.tile * num_kb);
        if (lane == 0) {
          for (int c = c_lo; c < c_hi; ++c)
            if (!wait_flag(flags + c * 2 + rank, EPI_WARPS, abort)) {
              failed = true;
              break;
            }
        }
        failed = __shfl_sync(0xffffffffu, failed ? 1 : 0, 0) != 0;
        if (failed) {
          if (!*abort) record_timeout(err, WHERE_GEMM_EPILOGUE, abort);
          release();
          break;
        }
        for (int c = c_lo; c < c_hi; ++c) (void)ld_acquire(flags + c * 2 + rank);
      }
      if (nch == 0) {
        release();
      } else {
        // finish chunk k from accumulator values v: partial sums, bias, activation, residual
        auto process = [&](float (&v)[CW], const float4 (&b4)[CW / 4], const float4 (&r4)[CW / 4], int k) {
          for (int c = c_lo; c < c_hi; ++c) {
            const float* src = partial + ((size_t)c * 2 + rank) * CTA_PARTIAL + (size_t)ew * WARP_PARTIAL;
#pragma unroll
            for (int j = 0; j < CW / 4; ++j) {
              const float4 p = ld_cg4(src + (k * (CW / 4) + j) * 128 + lane * 4);
              v[4 * j] += p.x; v[4 * j + 1] += p.y; v[4 * j + 2] += p.z; v[4 * j + 3] += p.w;
            }
          }
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
          if constexpr (KIND == EPI_BIAS_RESID) {
#pragma unroll
            for (int j = 0; j < CW / 4; ++j) {
              x[4 * j] += r4[j].x; x[4 * j + 1] += r4[j].y; x[4 * j + 2] += r4[j].z; x[4 * j + 3] += r4[j].w;
            }
          }
          uint8_t* st = stg_base + (cc % NBUF) * STG_BYTES;
          if (lane == 0) ptx::bulk_wait_read<NBUF - 1>();   // the store issued NBUF chunks ago has read it
          __syncwarp();
          uint8_t* srow = st + lane * ROW_BYTES;
          if constexpr (std::is_same<OutT, float>::value) {
#pragma unroll
            for (int q = 0; q < CW / 4; ++q)
              *reinterpret_cast<float4*>(srow + ((q ^ swz) << 4)) =
                  make_float4(x[4 * q], x[4 * q + 1], x[4 * q + 2], x[4 * q + 3]);
          } else {
#pragma unroll
            for (int q = 0; q < CW / 8; ++q)
              *reinterpret_cast<uint4*>(srow + ((q ^ swz) << 4)) =
                  make_uint4(bf16x2_bits(x[8 * q], x[8 * q + 1]), bf16x2_bits(x[8 * q + 2], x[8 * q + 3]),
                             bf16x2_bits(x[8 * q + 4], x[8 * q + 5]), bf16x2_bits(x[8 * q + 6], x[8 * q + 7]));
          }
          ptx::fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            ptx::tma_store_2d(&tmO, ptx::smem_u32(st), gcol + k * CW, row0);
            ptx::bulk_commit();
          }
          ++cc;
        };
        float va[CW], vb[CW];
        ptx::tmem_ld(taddr, va);
#pragma unroll 1
        for (int k = 0; k < nch; k += 2) {
          ptx::tmem_ld_wait();
          if (k == nch - 1) release();
          if (k + 1 < nch) {
            ptx::tmem_ld(taddr + (k + 1) * CW, vb);
            load_operands(k + 1, bb, rb);
          }
          process(va, ba, ra, k);
          if (k + 1 >= nch) break;
          ptx::tmem_ld_wait();
          if (k + 1 == nch - 1) release();
          if (k + 2 < nch) {
            ptx::tmem_ld(taddr + (k + 2) * CW, va);
            load_operands(k + 2, ba, ra);
          }
          process(vb, bb, rb, k + 1);
        }
      }
      if (u.role == FINISH) {
        // this warp has read its share of every contributor's slot: count it, and the
        // last of the finishing CTA's warps resets the counter for the next launch
        __syncwarp();
        if (lane == 0)
          for (int c = c_lo; c < c_hi; ++c)
            if (atomicAdd(flags + c * 2 + rank, 1) == 2 * EPI_WARPS - 1) atomicExch(flags + c * 2 + rank, 0);
      }
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
    ptx::tmem_dealloc_pair(tmem_base, TMEM_COLS);
  }
}

// ------------------------------------------------------------------ host side

template <int KIND, typename OutT>
struct SkLauncher {
  static int max_clusters;
  static cudaError_t prepare() {
    auto kern = gemm_sk_kernel<KIND, OutT>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(2 * 74);
    cfg.blockDim = dim3(NUM_THREADS);
    cfg.dynamicSmemBytes = SMEM;
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
  static cudaError_t launch(const GemmArgs& g, const EpiParams& ep, float* partial, int* flags, int max_pairs,
                            DevError* err, cudaStream_t st) {
    constexpr int ROW_BYTES = CW * (int)sizeof(OutT);
    if (max_clusters < 1) return cudaErrorInvalidConfiguration;
    CUtensorMap ta, tb, to;
    if (make_tmap_bf16(&ta, g.A, g.M, g.K, g.lda, BMC) || make_tmap_bf16(&tb, g.B, g.N, g.K, g.ldb, BN / 2))
      return cudaErrorInvalidValue;
    if (make_tmap_plain(&to, ep.out, (int)sizeof(OutT), g.M, g.N, ep.ldo, CW, 32, ROW_BYTES))
      return cudaErrorInvalidValue;
    const int mt = (g.M + 2 * BMC - 1) / (2 * BMC), nt = (g.N + BN - 1) / BN;
    const int kb = (g.K + BK - 1) / BK;
    const long units = (long)mt * nt * kb;
    int pairs = max_clusters < max_pairs ? max_clusters : max_pairs;
    if (units < pairs) pairs = (int)units;
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
    cfg.dynamicSmemBytes = SMEM;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = pdl_enabled() ? 2 : 1;
    return cudaLaunchKernelEx(&cfg, gemm_sk_kernel<KIND, OutT>, ta, tb, to, mt, nt, kb, ep, partial, flags, err);
  }
};
template <int KIND, typename OutT>
int SkLauncher<KIND, OutT>::max_clusters = 0;

}  // namespace

cudaError_t gemm_sk_prepare() {
  cudaError_t e = SkLauncher<EPI_BIAS, bf16>::prepare();
  if (e == cudaSuccess) e = SkLauncher<EPI_BIAS_GELU, bf16>::prepare();
  if (e == cudaSuccess) e = SkLauncher<EPI_BIAS_RESID, float>::prepare();
  return e;
}

size_t gemm_sk_workspace_floats() { return (size_t)GEMM_SK_MAX_PAIRS * 2 * CTA_PARTIAL; }

cudaError_t gemm_sk(const GemmArgs& g, int kind, bool out_f32, const EpiParams& ep, float* partial, int* flags,
                    DevError* err, cudaStream_t st) {
  if (g.M <= 0 || g.N <= 0) return cudaSuccess;
  if (g.K <= 0 || g.N % 16 || partial == nullptr || flags == nullptr) return cudaErrorInvalidValue;
  if (kind == EPI_BIAS && !out_f32)
    return SkLauncher<EPI_BIAS, bf16>::launch(g, ep, partial, flags, GEMM_SK_MAX_PAIRS, err, st);
  if (kind == EPI_BIAS_GELU && !out_f32)
    return SkLauncher<EPI_BIAS_GELU, bf16>::launch(g, ep, partial, flags, GEMM_SK_MAX_PAIRS, err, st);
  if (kind == EPI_BIAS_RESID && out_f32)
    return SkLauncher<EPI_BIAS_RESID, float>::launch(g, ep, partial, flags, GEMM_SK_MAX_PAIRS, err, st);
  return cudaErrorInvalidValue;
}

}  // namespace kd
