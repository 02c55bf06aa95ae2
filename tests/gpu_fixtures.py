"""Session fixtures and comparators shared by the GPU tests."""
import numpy as np
import pytest
import torch

import synth
import transformer_denoiser_b200 as kb
from oracle import kimodo_oracle as ko


def require_cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    kb.load_library()


@pytest.fixture(scope="session")
def blob():
    return synth.weight_blob()


@pytest.fixture(scope="session")
def params(blob):
    return ko.unpack_weights(blob)


@pytest.fixture(scope="session")
def gpu_bf16(blob):
    require_cuda()
    m = kb.Kimodo(blob, kb.BF16, 0)
    yield m
    m.close()


@pytest.fixture(scope="session")
def gpu_fp32(blob):
    require_cuda()
    m = kb.Kimodo(blob, kb.FP32, 0)
    yield m
    m.close()


def max_abs_rel(g, o):
    """max |g - o| / max |o| (the fp32 path's metric)."""
    g = np.asarray(g, np.float64)
    o = np.asarray(o, np.float64)
    return float(np.abs(g - o).max() / max(np.abs(o).max(), 1e-300))


def rel_l2(g, o):
    """||g - o||_2 / ||o||_2 (the bf16 path's metric)."""
    g = np.asarray(g, np.float64)
    o = np.asarray(o, np.float64)
    return float(np.linalg.norm(g - o) / max(np.linalg.norm(o), 1e-300))


def valid(x, lengths):
    """Concatenate the valid frames of x [B, T, F]."""
    return np.concatenate([np.asarray(x[b, :int(n)]) for b, n in enumerate(lengths)], 0)


def padded(x, lengths):
    parts = [np.asarray(x[b, int(n):]).ravel() for b, n in enumerate(lengths)]
    return np.concatenate(parts) if parts else np.zeros(0)
