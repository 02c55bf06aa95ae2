// Row-block dataflow between the kernels of a transformer layer.
//
// Every kernel of the path is launched with programmatic dependent launch, so its CTAs
// can become resident while the previous kernel still runs.  Inside a layer of a large
// batch (the CTA-pair GEMMs, attention and LayerNorm), a kernel does not wait for the
// whole previous grid (griddepcontrol.wait): it waits only for the 256-row blocks of its
// input that it is about to read, counted in per-block completion counters that the
// producing kernel raises as it finishes each part.  The tiles of a GEMM's last partial
// round then overlap the next kernel's work on the row blocks already done.
//
// Counters: ctr[event * stride + block], monotonic within one call (zeroed at its start).
// A kernel of layer epoch e (one layer of one network forward; e counts up through the
// call) adds its per-block share once per epoch, so the producer's count for block m
// after its epoch e is (e + 1) x unit x (rows of m if the unit counts rows).
//
// Progress: each kernel triggers its dependents at its start, so a dependent grid is
// launched only when every CTA of its producer has started; a CTA therefore only ever
// waits on CTAs that are resident or finished.  Every wait is bounded.
#pragma once

#include <stdint.h>
#include "common.cuh"
#include "ptx.cuh"

namespace kd {

enum FlowEvent : int { FLOW_QKV = 0, FLOW_ATTN, FLOW_O, FLOW_LN1, FLOW_FFN1, FLOW_FFN2, FLOW_LN2, FLOW_EVENTS };
constexpr int FLOW_BLOCK = 256;   // rows per block (one CTA-pair output tile row)

// Wait / signal description of one launch (plain data, passed by value to kernels).
struct Flow {
  int* ctr = nullptr;    // null: no dataflow, the kernel waits for its whole predecessor
  int stride = 0;        // counters per event
  int M = 0;             // token rows of the layer
  int wait_ev = -1;      // event awaited (-1: griddepcontrol.wait instead)
  int wait_epochs = 0;   // producer epochs completed: the target is wait_epochs x wait_unit (x rows)
  int wait_unit = 0;
  int wait_rows = 0;     // 1: the awaited count is per row of the block
  int sig_ev = -1;       // event raised (-1: none)
  const DevError* err = nullptr;   // a recorded failure ends every wait at once
};

__device__ __forceinline__ int flow_rows_in_block(const Flow& f, int blk) {
  const int r = f.M - blk * FLOW_BLOCK;
  return r < FLOW_BLOCK ? r : FLOW_BLOCK;
}

__device__ __forceinline__ int ld_acquire_gpu(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Bounded wait (one thread) until block `blk` of the awaited event has reached its target;
// then orders this thread's later generic and async-proxy (TMA) reads after it.  Returns
// false on give-up: limit_ns of wall time, *abort set, or a failure recorded in f.err by
// any kernel (so that after one timeout the later kernels do not wait out their limits).
__device__ __forceinline__ bool flow_wait(const Flow& f, int blk, volatile int* abort, uint64_t limit_ns) {
  if (f.ctr == nullptr || f.wait_ev < 0) return true;
  const int target = f.wait_epochs * f.wait_unit * (f.wait_rows ? flow_rows_in_block(f, blk) : 1);
  const int* c = f.ctr + f.wait_ev * f.stride + blk;
  if (ld_acquire_gpu(c) < target) {
    const uint64_t t0 = ptx::global_timer_ns();
    for (uint32_t it = 1;; ++it) {
      __nanosleep(64);
      if (ld_acquire_gpu(c) >= target) break;
      if ((it & 15u) == 0) {
        if (abort != nullptr && *abort) return false;
        if (f.err != nullptr && *reinterpret_cast<const volatile int*>(&f.err->code) != 0) return false;
        if (ptx::global_timer_ns() - t0 > limit_ns) return false;
      }
    }
  }
  asm volatile("fence.proxy.async.global;" ::: "memory");
  return true;
}

// Adds `n` to block `blk` of this launch's event, after this thread's earlier global
// writes (generic, and async-proxy ones that it has waited for) are visible GPU-wide.
__device__ __forceinline__ void flow_signal(const Flow& f, int blk, int n) {
  if (f.ctr == nullptr || f.sig_ev < 0 || n == 0) return;
  asm volatile("fence.proxy.async.global;" ::: "memory");
  __threadfence();
  atomicAdd(f.ctr + f.sig_ev * f.stride + blk, n);
}

}  // namespace kd
