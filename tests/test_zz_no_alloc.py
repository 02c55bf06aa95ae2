"""kimodo_denoiser_forward_noalloc, the forward for callers that must not allocate
device memory (engines with their own allocator or budget, latency-sensitive
callers), against kimodo_denoiser_forward.

This file is collected last on purpose.  Each call of the allocation-free entry
point reuses one static device array that still holds the previous call's data,
so the test makes two different calls in a row through the C ABI and checks both.
"""
import ctypes

import numpy as np
import pytest

import synth
import transformer_denoiser_b200 as kb
from gpu_fixtures import blob, gpu_bf16, gpu_fp32, max_abs_rel, padded, rel_l2, valid  # noqa: F401

pytestmark = pytest.mark.gpu

TOL_BF16_FWD = 2e-2   # the bf16 path's per-forward tolerance
TOL_FP32 = 1e-4       # the fp32 path's tolerance

CALLS = [  # net, batch, frames, lengths, timestep, seed: two different calls in a row
    (kb.NET_BODY, 2, 40, [40, 17], 480, 700),
    (kb.NET_ROOT, 3, 20, [20, 5, 1], 999, 710),
]


def _call_noalloc(model, net, x, emb, t, lengths):
    lib = kb.load_library()
    B, T = x.shape[0], x.shape[1]
    out = np.full((B, T, 5 if net == kb.NET_ROOT else 274), np.nan, np.float32)
    rc = lib.kimodo_denoiser_forward_noalloc(model._ctx, net, x.ctypes.data, emb.ctypes.data, t,
                                             lengths.ctypes.data, B, T, out.ctypes.data, None)
    assert rc == 0, lib.kimodo_last_error()
    return out


@pytest.mark.parametrize("precision", ["bf16", "fp32"])
def test_noalloc_forward_matches_forward(precision, request):
    model = request.getfixturevalue("gpu_" + precision)
    for net, B, T, L, t, seed in CALLS:
        din = 5 if net == kb.NET_ROOT else 279
        x = synth.fill_padding(synth.noise(B, T, din, seed=seed), L, seed=seed + 1)
        emb = synth.text_embeddings(B, seed=seed + 2)
        lengths = np.array(L, np.int32)
        want = model.denoiser_forward(net, x, emb, t, lengths)
        got = _call_noalloc(model, net, x, emb, t, lengths)
        if precision == "bf16":
            assert rel_l2(valid(got, L), valid(want, L)) <= TOL_BF16_FWD
        else:
            assert max_abs_rel(valid(got, L), valid(want, L)) <= TOL_FP32
        assert np.all(padded(got, L) == 0)


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
