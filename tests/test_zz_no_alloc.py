"""kimodo_denoiser_forward_noalloc, the forward for callers that must not allocate
device memory (engines with their own allocator or budget, latency-sensitive
callers), against kimodo_denoiser_forward.

This file is collected last on purpose.  Each call of the allocation-free entry
point reuses one static device array that still holds the previous call's data,
so the tests make two different calls in a row through the C ABI and check both.
"""
import numpy as np
import pytest
import torch

import synth
import transformer_denoiser_b200 as kb
from gpu_fixtures import blob, gpu_bf16, max_abs_rel, padded, rel_l2, require_cuda, valid  # noqa: F401

pytestmark = pytest.mark.gpu

TOL_BF16_FWD = 2e-2   # the bf16 path's per-forward tolerance
TOL_FP32 = 1e-4       # the fp32 path's tolerance

CALLS = [  # net, batch, frames, lengths, timestep, seed: two different calls in a row
    (kb.NET_BODY, 2, 40, [40, 17], 480, 700),
    (kb.NET_ROOT, 3, 20, [20, 5, 1], 999, 710),
]


def _inputs(net, B, T, L, seed):
    din = 5 if net == kb.NET_ROOT else 279
    x = synth.fill_padding(synth.noise(B, T, din, seed=seed), L, seed=seed + 1)
    return x, synth.text_embeddings(B, seed=seed + 2), np.array(L, np.int32)


def _call_noalloc(model, net, x, emb, t, lengths):
    lib = kb.load_library()
    B, T = x.shape[0], x.shape[1]
    out = np.full((B, T, 5 if net == kb.NET_ROOT else 274), np.nan, np.float32)
    rc = lib.kimodo_denoiser_forward_noalloc(model._ctx, net, x.ctypes.data, emb.ctypes.data, t,
                                             lengths.ctypes.data, B, T, out.ctypes.data, None)
    assert rc == 0, lib.kimodo_last_error()
    return out


@pytest.mark.parametrize("precision", [kb.BF16, kb.FP32])
def test_noalloc_forward_allocates_nothing_and_matches_forward(precision, blob):
    """On a fresh context (no workspace yet) two calls in a row leave the device's free
    memory unchanged; only then does the regular forward (which allocates its workspace)
    run, and both calls' outputs are compared with it."""
    require_cuda()
    # a first context runs the same calls once, so that every kernel the calls launch is
    # loaded before the measurement (module loading takes device memory of its own)
    warm = kb.Kimodo(blob, precision, 0)
    for net, B, T, L, t, seed in CALLS:
        x, emb, lengths = _inputs(net, B, T, L, seed)
        _call_noalloc(warm, net, x, emb, t, lengths)
    warm.close()
    model = kb.Kimodo(blob, precision, 0)
    try:
        torch.cuda.synchronize()
        free0 = torch.cuda.mem_get_info()[0]
        got = []
        for net, B, T, L, t, seed in CALLS:
            x, emb, lengths = _inputs(net, B, T, L, seed)
            got.append(_call_noalloc(model, net, x, emb, t, lengths))
        torch.cuda.synchronize()
        assert torch.cuda.mem_get_info()[0] == free0
        for (net, B, T, L, t, seed), g in zip(CALLS, got):
            x, emb, lengths = _inputs(net, B, T, L, seed)
            want = model.denoiser_forward(net, x, emb, t, lengths)
            if precision == kb.BF16:
                assert rel_l2(valid(g, L), valid(want, L)) <= TOL_BF16_FWD
            else:
                assert max_abs_rel(valid(g, L), valid(want, L)) <= TOL_FP32
            assert np.all(padded(g, L) == 0)
    finally:
        model.close()


def test_noalloc_forward_rejects_sizes_beyond_its_scratch(gpu_bf16):
    lib = kb.load_library()
    B, T = 2, 300                      # 2 x 301 tokens > 512
    x = np.zeros((B, T, 5), np.float32)
    emb = np.zeros((B, 4096), np.float32)
    lengths = np.full(B, T, np.int32)
    out = np.zeros((B, T, 5), np.float32)
    rc = lib.kimodo_denoiser_forward_noalloc(gpu_bf16._ctx, kb.NET_ROOT, x.ctypes.data, emb.ctypes.data, 999,
                                             lengths.ctypes.data, B, T, out.ctypes.data, None)
    assert rc == -1
    assert b"static scratch" in lib.kimodo_last_error()
