"""Long oracle trajectories for the GPU parity tests, computed in worker processes.

A 50- or 100-step fp64 trajectory of one sequence takes the oracle a minute or more,
so the parity tests submit every one they need to a pool of `spawn` workers as soon as
collection is done (before the first GPU call); the trajectories are then computed on
the host cores while the GPU tests run, and each test waits only for its own.

Every job rebuilds its inputs from the seeded generators in `synth`, exactly as the
test does, and runs `oracle.kimodo_oracle.ddim_sample` on one sequence.
"""
from __future__ import annotations

import multiprocessing as mp
import os
from concurrent.futures import ProcessPoolExecutor

import numpy as np

# (name, batch, frames, steps, cfg): the workloads whose trajectories the tests compare
C3 = ("c3", 1, 180, 50, 2.0)          # one prompt, 180 frames
C4 = ("c4", 16, 150, 100, 2.0)        # 16 prompts, 150 frames (the benchmark)
C5 = ("c5", 64, 300, 50, 2.5)         # 64 prompts, lengths U{60..300}, garbage padding
VAR = ("var", 6, 40, 10, 2.0)         # 2 prompts x 3 takes (variations of a prompt)


def workload_inputs(spec):
    """(text_emb [B or text rows, 4096], null [4096], state x_T [B, T, 279], lengths [B])
    of a workload, from the seeded generators."""
    import synth
    name, B, T, _, _ = spec
    null = np.zeros(4096, np.float32)
    if name == "c5":
        L = synth.lengths_uniform(B, 60, 300)
        return synth.text_embeddings(B), null, synth.fill_padding(synth.noise(B, T), L), L
    if name == "var":
        return synth.text_embeddings(2, seed=481), null, synth.noise(B, T, seed=482), np.full(B, T, np.int32)
    return synth.text_embeddings(B), null, synth.noise(B, T), np.full(B, T, np.int32)


def c5_sequences():
    """Sequences of the ragged workload compared with the oracle: the shortest, the
    longest, and two others drawn with a fixed seed."""
    import synth
    L = synth.lengths_uniform(C5[1], 60, 300)
    lo, hi = int(np.argmin(L)), int(np.argmax(L))
    rest = [b for b in range(C5[1]) if b not in (lo, hi)]
    picks = np.random.default_rng(6).choice(rest, size=2, replace=False)
    return [lo, hi] + [int(b) for b in picks]


JOBS = [(C3, 0), (C4, 0), (C4, 15)] + [(C5, b) for b in c5_sequences()] + [(VAR, b) for b in range(VAR[1])]

_PARAMS = None


def _init(threads: int):
    from threadpoolctl import threadpool_limits
    global _LIMITS
    _LIMITS = threadpool_limits(threads)


def _trajectory(spec, b: int):
    import synth
    from oracle import kimodo_oracle as ko
    global _PARAMS
    if _PARAMS is None:
        _PARAMS = ko.unpack_weights(synth.weight_blob())
    name, B, T, steps, cfg = spec
    emb, null, x, L = workload_inputs(spec)
    takes = B // emb.shape[0]
    return ko.ddim_sample(_PARAMS, emb[b // takes], null, x[b], int(L[b]), steps, cfg)


class OraclePool:
    """Starts every job of JOBS at construction; result(spec, b) waits for one."""

    def __init__(self, workers: int | None = None):
        cores = os.cpu_count() or 4
        workers = workers or max(1, min(6, cores // 4))
        ctx = mp.get_context("spawn")
        self._ex = ProcessPoolExecutor(max_workers=workers, mp_context=ctx, initializer=_init,
                                       initargs=(max(1, cores // workers),))
        # longest jobs first, so that the pool's last round is short
        order = sorted(JOBS, key=lambda j: -j[0][2] * j[0][3])
        self._fut = {(spec[0], b): self._ex.submit(_trajectory, spec, b) for spec, b in order}

    def result(self, spec, b: int) -> np.ndarray:
        return self._fut[(spec[0], b)].result()

    def shutdown(self):
        """Cancel what has not started and stop the workers (a run that stopped early
        must not wait for trajectories nobody reads)."""
        procs = list(getattr(self._ex, "_processes", {}).values())
        self._ex.shutdown(wait=False, cancel_futures=True)
        for p in procs:
            if p.is_alive():
                p.terminate()
