// Masked multi-head self-attention on the tcgen05 tensor cores ("Kimodo WebGPU",
// "WGSL compute shaders" table: multi-head self-attention with optional key masking).
//
// One CTA per (head, sequence, query tile), two CTAs per SM up to 256 keys; the S query
// rows of a sequence are split into ceil(S / 128) tiles of equal size (151: 76 + 75).
// Every key of a sequence fits in one pass (at most 301 tokens), so the softmax is
// exact, not online:
//   1. TMA stages the query tile (128 x 128), the keys and the upper half of the
//      value dimensions of the sequence's rows rounded up to 32 (128-byte swizzle, no
//      multicast; a padded sequence's keys in one box per 64-dimension half, issued one
//      box per lane); the lower value half goes into the query buffer once S is formed.
//   2. One thread issues S = Q K^T (M = 128, N = valid keys rounded up to 16,
//      K = 128) into TMEM.
//   3. Eight softmax warps (two per TMEM lane quarter, one query row per thread,
//      half of the keys each) take the row maximum over the valid keys, form
//      p = 2^((s - max) * log2(e) / sqrt(128)) (0 for keys at or beyond 1 + length,
//      which are never read, so padded content, even NaN, cannot leak), sum it,
//      and write P in bf16 into the key buffer (dead once S is formed) in the
//      K-major 128-byte-swizzle layout.  They zero the value rows past the valid
//      keys inside the MMA's K range, so 0 * garbage cannot occur either.
//   4. The same thread issues O = P V as one N = 128 MMA per 16-key step (K = keys),
//      the two 64-dimension value halves read in place as one MN-major operand whose
//      halves lie one leading-byte offset apart, into the TMEM columns S occupied (up
//      to 256 keys: a 256-column allocation); the softmax warps scale O by 1 / sum
//      and store the valid query rows in bf16.
// Rows of the key and value tiles past the sequence belong to other tokens or lie
// outside the matrix (zero fill) and are masked as above.  Every wait is bounded.
#include <cuda.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "epilogue.cuh"
#include "kernels.h"
#include "launch.cuh"
#include "ptx.cuh"

namespace kd {
namespace {

constexpr int QT = 128;                    // query rows per CTA
constexpr int KB_ROWS = 32;                // key rows are staged in multiples of 32
constexpr int SM_WARPS = 8;                // softmax / epilogue warps
constexpr int NUM_THREADS = 64 + 32 * SM_WARPS;
constexpr uint64_t WAIT_LIMIT_NS = 2000000000ull;
constexpr int KIMODO_ETIMEOUT_CODE = -5;
constexpr int MAX_KA = ((MAX_FRAMES + 1 + KB_ROWS - 1) / KB_ROWS) * KB_ROWS;   // 320 key rows
constexpr uint32_t Q_BYTES = QT * DH * 2;  // two 64-column halves of 16 KB

// Shared memory, with ka = key rows rounded up to 32 and kp = ka rounded up to 64:
// Q [2 halves][128 rows][128 B] (later the lower value half V0 [ka rows][128 B] when
// it fits), K [2 halves][ka rows][128 B] then P [kp / 64 blocks][128 rows][128 B] in a
// region of kp * 256 B, the upper value half V1 [ka rows][128 B], V0 on its own when
// it does not fit in the Q buffer, then barriers and the row-statistics exchange.
__host__ __device__ constexpr bool v0_in_q(int ka) { return (uint32_t)ka * 128 <= Q_BYTES; }
__host__ __device__ constexpr uint32_t kp_of(int ka) { return (uint32_t)((ka + 63) / 64) * 64; }
__host__ __device__ constexpr size_t smem_bytes(int ka) {
  return 1024 + Q_BYTES + (size_t)kp_of(ka) * 256 + (size_t)ka * 128 + (v0_in_q(ka) ? 0 : (size_t)ka * 128) +
         8 * 8 + 2 * 2 * QT * 4 + 16;
}

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ void record_timeout(DevError* err, volatile int* abort) {
  *abort = 1;
  if (err && atomicCAS(&err->code, 0, KIMODO_ETIMEOUT_CODE) == 0) {
    err->where = WHERE_ATTENTION;
    err->block = blockIdx.x + gridDim.x * (blockIdx.y + gridDim.y * blockIdx.z);
  }
}

// Shared-memory descriptor of an MN-major operand in the 128-byte swizzle layout:
// 64-element atoms along MN `lbo` bytes apart, 8-row groups along K 1024 bytes apart.
__device__ __forceinline__ uint64_t smem_desc_sw128_mn(uint32_t saddr, uint32_t lbo) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)(1024u >> 4) << 32;
  d |= (uint64_t)1u << 46;
  d |= (uint64_t)2u << 61;
  return d;
}

__global__ void __launch_bounds__(NUM_THREADS, 2)
attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmKV,
               const __grid_constant__ CUtensorMap tmO, bf16* __restrict__ out, const int* __restrict__ lengths, int len_mod, int S_pad, int ka,
               uint32_t tmem_cols, uint32_t o_col, const int* __restrict__ tok0, int kbox, DevError* err,
               L2Prefetch pf) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t kp = kp_of(ka);
  const bool v0q = v0_in_q(ka);
  const uint32_t sQ = ptx::smem_u32(smem);
  const uint32_t sK = sQ + Q_BYTES;                       // also P
  // value halves: V0 in the Q buffer when it fits, else right after K; V1 after them, so
  // that V1 - V0 is the (positive) stride between the two 64-dimension atoms of V
  const uint32_t sV0 = v0q ? sQ : sK + kp * 256;
  const uint32_t sV1 = sK + kp * 256 + (v0q ? 0u : (uint32_t)ka * 128);
  uint8_t* gV0 = smem + (sV0 - sQ);                       // generic addresses of the value halves
  uint8_t* gV1 = smem + (sV1 - sQ);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Q_BYTES + (size_t)kp * 256 + (size_t)ka * 128 +
                                               (v0q ? 0 : (size_t)ka * 128));
  const uint32_t bar0 = ptx::smem_u32(bars);
  const uint32_t bar_qk = bar0, bar_v1 = bar0 + 8, bar_s = bar0 + 16, bar_p = bar0 + 24, bar_o = bar0 + 32,
                 bar_v0 = bar0 + 40;
  float* xmax = reinterpret_cast<float*>(bars + 8);      // [2][QT] partial row maxima, then sums
  float* xsum = xmax + 2 * QT;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(xsum + 2 * QT);
  volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.x, seq = blockIdx.y, qt = blockIdx.z;
  // set-up that reads nothing an earlier kernel writes (barriers, TMEM, descriptors) runs
  // before the dependency wait, overlapping the previous kernel's tail
  if (threadIdx.x == 0) {
    ptx::mbar_init(bar_qk, 1);
    ptx::mbar_init(bar_v1, 1);
    ptx::mbar_init(bar_v0, 1);
    ptx::mbar_init(bar_s, 1);
    ptx::mbar_init(bar_p, SM_WARPS);
    ptx::mbar_init(bar_o, 1);
    ptx::fence_mbar_init();
    ptx::tma_prefetch_desc(&tmQ);
    ptx::tma_prefetch_desc(&tmKV);
    ptx::prefetch_l2_share(pf, blockIdx.x + gridDim.x * (blockIdx.y + (unsigned long long)gridDim.y * blockIdx.z),
                           (unsigned long long)gridDim.x * gridDim.y * gridDim.z);
  }
  if (warp == 1) {
    ptx::tmem_alloc(ptx::smem_u32(tmem_slot), tmem_cols);
    ptx::tmem_relinquish();
  }
  ptx::pdl_wait();
  ptx::pdl_trigger();
  const long row0 = tok0 ? tok0[seq] : (long)seq * S_pad;
  const int S = tok0 ? tok0[seq + 1] - tok0[seq] : S_pad;
  // the sequence's query rows in ceil(S / 128) tiles of equal size (151 tokens: 76 + 75
  // rows, so that neither CTA of a (head, sequence) is left with a short tail)
  const int n_qt = (S + QT - 1) / QT;
  const int qrows = (S + n_qt - 1) / n_qt;
  const int q0 = qt * qrows;                 // first query row of this tile
  const bool live = qt < n_qt;               // uniform over the CTA
  // key / value boxes of kbox rows covering the sequence's tokens (not only the valid ones,
  // so that the loads need not wait for the lengths)
  const int n_boxes = (S + kbox - 1) / kbox;

  if (warp == 0) {
    if (lane == 0) *abort = (!live || (err != nullptr && *reinterpret_cast<volatile int*>(&err->code) != 0)) ? 1 : 0;
    __syncwarp();
    if (!*abort) {
      // the query tile, the keys and the upper value half, one box per lane (issue from one
      // thread costs tens of ns per box), before the CTA barrier so that their latency
      // overlaps it.  A box may land before its barrier's expect-tx: the phase cannot complete
      // before that arrival.
      if (lane == 0) {
        ptx::mbar_arrive_expect_tx(bar_qk, Q_BYTES + (uint32_t)(n_boxes * kbox) * 2 * 128);
        ptx::mbar_arrive_expect_tx(bar_v1, (uint32_t)(n_boxes * kbox) * 128);
      }
      if (lane < 2) {
        ptx::tma_load_2d(sQ + lane * (QT * 128), &tmQ, bar_qk, h * DH + lane * 64, (int)row0 + q0);
      } else if (lane < 2 + 2 * n_boxes) {
        const int hf = (lane - 2) / n_boxes, b = (lane - 2) % n_boxes;
        ptx::tma_load_2d(sK + (uint32_t)(hf * ka + b * kbox) * 128, &tmKV, bar_qk, D + h * DH + hf * 64,
                         (int)row0 + b * kbox);
      } else if (lane < 2 + 3 * n_boxes) {
        const int b = lane - 2 - 2 * n_boxes;
        ptx::tma_load_2d(sV1 + (uint32_t)(b * kbox) * 128, &tmKV, bar_v1, 2 * D + h * DH + 64, (int)row0 + b * kbox);
      }
    }
  }
  // read here, used after the barrier: the load's latency overlaps it
  const int len = live ? lengths[seq % len_mod] : 0;
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const bool skip = *abort != 0;
  int n_valid = 1 + len;
  n_valid = n_valid < 1 ? 1 : (n_valid > S ? S : n_valid);
  const int n_cols = (n_valid + 15) & ~15;                 // MMA N for S = Q K^T, K range of O = P V

  if (warp == 0) {
    if (lane == 0 && !skip) {
      // ---------------- TMA (Q, K and V1 were issued at set-up)
      // the lower value half: into the query buffer once S = Q K^T no longer reads it
      bool ok = v0q ? ptx::mbar_wait_bounded(bar_s, 0, abort, WAIT_LIMIT_NS) : true;
      if (ok) {
        ptx::mbar_arrive_expect_tx(bar_v0, (uint32_t)(n_boxes * kbox) * 128);
        for (int b = 0; b < n_boxes; ++b)
          ptx::tma_load_2d(sV0 + (uint32_t)(b * kbox) * 128, &tmKV, bar_v0, 2 * D + h * DH, (int)row0 + b * kbox);
      } else if (!*abort) {
        record_timeout(err, abort);
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && !skip) {
      // ---------------- MMA issuer
      bool ok = ptx::mbar_wait_bounded(bar_qk, 0, abort, WAIT_LIMIT_NS);
      if (ok) {
        ptx::tc_fence_after();
        // S = Q K^T in N chunks of at most 256 key columns
        for (int n0 = 0; n0 < n_cols; n0 += 256) {
          const int nn = n_cols - n0 < 256 ? n_cols - n0 : 256;
          const uint32_t idesc = ptx::idesc_bf16_f32(QT, nn);
#pragma unroll
          for (int kk = 0; kk < DH / 16; ++kk) {
            const uint32_t a = sQ + (kk >> 2) * (QT * 128) + (kk & 3) * 32;
            const uint32_t b = sK + (uint32_t)((kk >> 2) * ka + n0) * 128 + (kk & 3) * 32;
            ptx::tc_mma_bf16(tmem_base + n0, ptx::smem_desc_sw128(a), ptx::smem_desc_sw128(b), idesc, kk != 0);
          }
        }
        ptx::tc_commit(bar_s);
        ok = ptx::mbar_wait_bounded(bar_p, 0, abort, WAIT_LIMIT_NS);
      }
      if (ok) {
        ptx::tc_fence_after();
        // O = P V: A = P (K-major, 64-key blocks of 16 KB), B = V (MN-major, its two 64-dimension
        // atoms V0 and V1 sV1 - sV0 bytes apart), D = TMEM columns o_col .. o_col + 127
        const uint32_t idesc = ptx::idesc_bf16_f32(QT, DH) | (1u << 16);
        for (int kk = 0; kk < n_cols / 16; ++kk) {
          const uint32_t a = sK + (kk >> 2) * (QT * 128) + (kk & 3) * 32;
          const uint32_t b = sV0 + (uint32_t)kk * 16 * 128;
          ptx::tc_mma_bf16(tmem_base + o_col, ptx::smem_desc_sw128(a), smem_desc_sw128_mn(b, sV1 - sV0), idesc,
                           kk != 0);
        }
        ptx::tc_commit(bar_o);
        volatile int never = 0;
        if (!ptx::mbar_wait_bounded(bar_o, 0, &never, WAIT_LIMIT_NS)) ok = false;
      }
      if (!ok && !*abort) record_timeout(err, abort);
    }
  } else if (!skip) {
    // ---------------- softmax and epilogue warps: lane quarter q, key half kh
    const int ew = warp - 2;
    const int q = warp & 3, kh = ew >> 2;
    const int r = q * 32 + lane;                 // query row within the tile
    const uint32_t lane_addr = (uint32_t)(q * 32) << 16;
    const int half_cols = ((n_cols / 16 + 1) / 2) * 16;       // key columns of half 0
    const int c_beg = kh == 0 ? 0 : half_cols;
    const int c_end = kh == 0 ? half_cols : n_cols;
    const float sc = 0.08838834764831845f * 1.4426950408889634f;   // log2(e) / sqrt(128)
    // query rows of this tile that exist: whole warps past them skip the softmax and the
    // epilogue (TMEM loads are warp-collective), single lanes skip their arithmetic
    const int rows_valid = S - q0 < qrows ? S - q0 : qrows;
    const bool warp_rows = q * 32 < rows_valid;
    const bool row_ok = r < rows_valid;
    bool ok = true;

    // zero the value rows n_valid .. n_cols - 1 (inside O = P V's K range) once they land
    auto zero_rows = [&](uint8_t* vh) {
      const int nz = n_cols - n_valid;
      for (int i = ew * 32 + lane; i < nz * 8; i += SM_WARPS * 32)
        *reinterpret_cast<uint4*>(vh + (size_t)(n_valid + i / 8) * 128 + (i & 7) * 16) = make_uint4(0u, 0u, 0u, 0u);
    };
    ok = ptx::mbar_wait_bounded(bar_v1, 0, abort, WAIT_LIMIT_NS);
    if (ok) zero_rows(gV1);
    if (ok) ok = ptx::mbar_wait_bounded(bar_s, 0, abort, WAIT_LIMIT_NS);
    float m = -INFINITY;
    if (ok && warp_rows) {
      ptx::tc_fence_after();
      // pass 1: row maximum over this half's valid keys
      for (int c0 = c_beg; c0 < c_end; c0 += 32) {
        if (c_end - c0 >= 32) {
          float v[32];
          ptx::tmem_ld(tmem_base + lane_addr + c0, v);
          ptx::tmem_ld_wait();
          if (c0 + 32 <= n_valid) {   // all keys valid: no masks, two independent chains
            float ma = v[0], mb = v[1];
#pragma unroll
            for (int j = 2; j < 32; j += 2) {
              ma = fmaxf(ma, v[j]);
              mb = fmaxf(mb, v[j + 1]);
            }
            m = fmaxf(m, fmaxf(ma, mb));
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (c0 + j < n_valid) m = fmaxf(m, v[j]);
          }
        } else {
          float v[16];
          ptx::tmem_ld(tmem_base + lane_addr + c0, v);
          ptx::tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 16; ++j)
            if (c0 + j < n_valid) m = fmaxf(m, v[j]);
        }
      }
    }
    xmax[kh * QT + r] = m;
    // the two warps of a lane quarter exchange their maxima (named barrier over the 8 softmax warps)
    asm volatile("bar.sync 1, %0;" ::"n"(SM_WARPS * 32) : "memory");
    m = fmaxf(xmax[r], xmax[QT + r]);
    const float msc = m * sc;
    float l = 0.f;
    if (ok && warp_rows) {
      // pass 2: p = 2^(s sc - m sc) on valid keys, 0 elsewhere; P row r into 64-key blocks
      // (swizzled).  The pass is bound by instruction issue: chunks of valid keys only skip
      // the masks, and the scaling and the row sum run on pairs (f32x2 FMA and add).
      float2 l2 = make_float2(0.f, 0.f);
      const float2 sc2 = make_float2(sc, sc), nmsc2 = make_float2(-msc, -msc);
      auto p_chunk = [&](const float* v, int c) {   // keys c .. c + 15
        uint32_t w[8];
        if (c + 16 <= n_valid) {
#pragma unroll
          for (int j = 0; j < 16; j += 2) {
            const float2 x = __ffma2_rn(make_float2(v[j], v[j + 1]), sc2, nmsc2);
            const float p0 = ex2_approx(x.x), p1 = ex2_approx(x.y);
            l2 = __fadd2_rn(l2, make_float2(p0, p1));
            w[j / 2] = bf16x2_bits(p0, p1);
          }
        } else {
#pragma unroll
          for (int j = 0; j < 16; j += 2) {
            const float p0 = c + j < n_valid ? ex2_approx(fmaf(v[j], sc, -msc)) : 0.f;
            const float p1 = c + j + 1 < n_valid ? ex2_approx(fmaf(v[j + 1], sc, -msc)) : 0.f;
            l2 = __fadd2_rn(l2, make_float2(p0, p1));
            w[j / 2] = bf16x2_bits(p0, p1);
          }
        }
        // 16 keys = two 16-byte chunks of row r in block c / 64
        uint8_t* blk = smem + Q_BYTES + (size_t)(c / 64) * (QT * 128) + (size_t)r * 128;
        const int ch = (c % 64) / 8;
        *reinterpret_cast<uint4*>(blk + (((ch) ^ (r & 7)) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
        *reinterpret_cast<uint4*>(blk + (((ch + 1) ^ (r & 7)) << 4)) = make_uint4(w[4], w[5], w[6], w[7]);
      };
      for (int c0 = c_beg; c0 < c_end; c0 += 32) {
        if (c_end - c0 >= 32) {
          float v[32];
          ptx::tmem_ld(tmem_base + lane_addr + c0, v);
          ptx::tmem_ld_wait();
          if (!row_ok) continue;
          p_chunk(v, c0);
          p_chunk(v + 16, c0 + 16);
        } else {
          float v[16];
          ptx::tmem_ld(tmem_base + lane_addr + c0, v);
          ptx::tmem_ld_wait();
          if (!row_ok) continue;
          p_chunk(v, c0);
        }
      }
      l = l2.x + l2.y;
    }
    xsum[kh * QT + r] = l;
    if (ok) ok = ptx::mbar_wait_bounded(bar_v0, 0, abort, WAIT_LIMIT_NS);
    if (ok) zero_rows(gV0);
    ptx::fence_proxy_async_smem();   // P and the zeroed value rows, before the MMA reads them
    ptx::tc_fence_before();
    __syncwarp();
    if (lane == 0) ptx::mbar_arrive(bar_p);
    asm volatile("bar.sync 1, %0;" ::"n"(SM_WARPS * 32) : "memory");
    l = xsum[r] + xsum[QT + r];
    if (ok) ok = ptx::mbar_wait_bounded(bar_o, 0, abort, WAIT_LIMIT_NS);
    if (ok && warp_rows) {
      ptx::tc_fence_after();
      // O row r, dims [64 kh, 64 kh + 64), scaled by 1 / l.  A warp whose 32 rows all exist
      // stages them (128-byte swizzle) in the query buffer, dead since O = P V completed, and
      // stores the 32 x 64 box by TMA; otherwise the existing rows are stored directly.
      const float inv = 1.f / l;
      const bool full = q * 32 + 32 <= rows_valid;
      uint8_t* stg = smem + (size_t)ew * 4096 + (size_t)lane * 128;
      bf16* orow = out + (row0 + q0 + r) * D + h * DH + kh * 64;
      for (int c0 = 0; c0 < 64; c0 += 16) {
        float v[16];
        ptx::tmem_ld(tmem_base + lane_addr + o_col + kh * 64 + c0, v);
        ptx::tmem_ld_wait();
        const uint4 w0 = make_uint4(bf16x2_bits(v[0] * inv, v[1] * inv), bf16x2_bits(v[2] * inv, v[3] * inv),
                                    bf16x2_bits(v[4] * inv, v[5] * inv), bf16x2_bits(v[6] * inv, v[7] * inv));
        const uint4 w1 = make_uint4(bf16x2_bits(v[8] * inv, v[9] * inv), bf16x2_bits(v[10] * inv, v[11] * inv),
                                    bf16x2_bits(v[12] * inv, v[13] * inv), bf16x2_bits(v[14] * inv, v[15] * inv));
        if (full) {
          const int ch = c0 / 8;
          *reinterpret_cast<uint4*>(stg + ((ch ^ (lane & 7)) << 4)) = w0;
          *reinterpret_cast<uint4*>(stg + (((ch + 1) ^ (lane & 7)) << 4)) = w1;
        } else if (row_ok) {
          *reinterpret_cast<uint4*>(orow + c0) = w0;
          *reinterpret_cast<uint4*>(orow + c0 + 8) = w1;
        }
      }
      if (full) {
        ptx::fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          ptx::tma_store_2d(&tmO, sQ + (uint32_t)ew * 4096, h * DH + kh * 64, (int)row0 + q0 + q * 32);
          ptx::bulk_commit();
          ptx::bulk_wait_all();
        }
        __syncwarp();
      }
    }
    if (!ok && !*abort) record_timeout(err, abort);
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem_base, tmem_cols);
  }
}

}  // namespace

size_t attention_tc_smem(int S) {
  const int ka = ((S + KB_ROWS - 1) / KB_ROWS) * KB_ROWS;
  return smem_bytes(ka);
}

cudaError_t attention_tc_prepare() {
  return cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              (int)smem_bytes(MAX_KA));
}

cudaError_t attention_tc(const bf16* qkv, bf16* out, int M, const int* lengths, int len_mod, int nseq, int S,
                         DevError* err, cudaStream_t st, const int* tok0, L2Prefetch pf) {
  if (nseq <= 0 || S <= 0 || M <= 0) return cudaSuccess;
  if (S > MAX_FRAMES + 1) return cudaErrorInvalidValue;
  CUtensorMap tq, tkv, to;
  const int ka = ((S + KB_ROWS - 1) / KB_ROWS) * KB_ROWS;
  // key / value rows per TMA box (a divisor of ka, so that the boxes a sequence needs never
  // pass the ka staged rows): every issued box costs the issuing thread time, so the padded
  // layout (every sequence S tokens) takes its keys in one box (two past 256 rows); the
  // packed layout, whose sequences may be far shorter than S, in boxes of 32 rows
  const int kbox = tok0 != nullptr ? KB_ROWS : (ka <= 256 ? ka : ka / 2);
  if (make_tmap_bf16(&tq, qkv, M, 3 * D, 3 * D, QT) || make_tmap_bf16(&tkv, qkv, M, 3 * D, 3 * D, kbox) ||
      make_tmap_plain(&to, out, 2, M, D, D, 64, 32, 128))
    return cudaErrorInvalidValue;
  // up to 256 keys S and then O share a 256-column TMEM allocation (two CTAs per SM);
  // beyond, S takes columns 0..303 and O 320..447 of 512
  const int n_cols_max = (S + 15) & ~15;
  const uint32_t tmem_cols = n_cols_max <= 256 ? 256u : 512u;
  const uint32_t o_col = n_cols_max <= 256 ? 0u : 320u;
  dim3 grid(H, nseq, (S + QT - 1) / QT);
  return launch_kernel(attn_tc_kernel, grid, dim3(NUM_THREADS), smem_bytes(ka), st, tq, tkv, to, out, lengths, len_mod,
                       S, ka, tmem_cols, o_col, tok0, kbox, err, pf);
}

}  // namespace kd
