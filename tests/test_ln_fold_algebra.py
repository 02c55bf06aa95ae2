"""The two identities the folded LayerNorm (KIMODO_LN_FOLD=1) rests on, checked on the
CPU against the oracle's own LayerNorm and linear layer:

1. LN(y) W^T + b = rstd * (y Wf^T) - rstd * mean * g + h, with Wf = W diag(gamma),
   g = Wf 1 (row sums) and h = W beta + b: the projection after a LayerNorm can run on
   the un-normalised rows and normalise in its epilogue.
2. The row statistics merged pairwise from 16-column chunks (each chunk's mean and sum
   of squared deviations; two blocks of n values combine as mean = (ma + mb) / 2,
   M2 = M2a + M2b + (mb - ma)^2 n / 2, Chan, Golub & LeVeque) equal the two-pass mean and
   biased variance of the whole row.
"""
import numpy as np

import synth
from oracle import kimodo_oracle as ko

D = 1024


def _fold(W, gamma, beta, b):
    Wf = W * gamma[None, :]
    return Wf, Wf.sum(axis=1), W @ beta + b


def _chunk_stats(row):
    c = row.reshape(-1, 16)
    m = c.mean(axis=1)
    return m, ((c - m[:, None]) ** 2).sum(axis=1)


def _merge_pairwise(means, m2s):
    n = 16
    means, m2s = list(means), list(m2s)
    while len(means) > 1:
        nm, nq = [], []
        for i in range(0, len(means), 2):
            d = means[i + 1] - means[i]
            nm.append((means[i] + means[i + 1]) * 0.5)
            nq.append(m2s[i] + m2s[i + 1] + d * d * (n / 2))
        means, m2s, n = nm, nq, 2 * n
    return means[0], m2s[0]


def test_fold_identity_matches_layernorm_then_linear():
    rng = np.random.default_rng(7)
    M, N = 37, 96
    y = rng.standard_normal((M, D)) * 1.7 + 0.3
    gamma = 1 + 0.02 * rng.standard_normal(D)
    beta = 0.02 * rng.standard_normal(D)
    W = 0.02 * rng.standard_normal((N, D))
    b = 0.02 * rng.standard_normal(N)
    ref = ko.linear(ko.layer_norm(y, gamma, beta), W, b)
    mean = y.mean(axis=1, keepdims=True)
    rstd = 1.0 / np.sqrt(y.var(axis=1, keepdims=True) + ko.LN_EPS)
    Wf, g, h = _fold(W, gamma, beta, b)
    got = rstd * (y @ Wf.T) - rstd * mean * g[None, :] + h[None, :]
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12 * np.abs(ref).max())


def test_fold_identity_is_not_vacuous():
    """Dropping either correction term (or folding beta into the wrong place) breaks it."""
    rng = np.random.default_rng(8)
    y = rng.standard_normal((5, D)) + 0.5
    gamma = 1 + 0.1 * rng.standard_normal(D)
    beta = 0.1 * rng.standard_normal(D)
    W = rng.standard_normal((8, D)) / 32
    b = rng.standard_normal(8)
    ref = ko.linear(ko.layer_norm(y, gamma, beta), W, b)
    mean = y.mean(axis=1, keepdims=True)
    rstd = 1.0 / np.sqrt(y.var(axis=1, keepdims=True) + ko.LN_EPS)
    Wf, g, h = _fold(W, gamma, beta, b)
    for wrong in (rstd * (y @ Wf.T) + h, rstd * (y @ Wf.T) - rstd * mean * g + b,
                  rstd * (y @ W.T) - rstd * mean * g + h):
        assert np.abs(wrong - ref).max() > 1e-3 * np.abs(ref).max()


def test_pairwise_chunk_merge_equals_two_pass_statistics():
    rng = np.random.default_rng(9)
    for shift in (0.0, 3.0, -40.0):
        row = rng.standard_normal(D) * 0.8 + shift
        m, q = _merge_pairwise(*_chunk_stats(row))
        assert abs(m - row.mean()) <= 1e-12 * max(1.0, abs(shift))
        assert abs(q / D - row.var()) <= 1e-12 * row.var()


def test_pairwise_chunk_merge_in_float32_stays_within_rounding():
    """In fp32 (the kernels' precision) the merged statistics stay within a few ulps of
    the float64 two-pass values, also for a row whose mean is large against its spread."""
    rows = synth.random_vectors((4, D), 11, 1.0).astype(np.float64)
    rows[2] += 25.0
    for row in rows.astype(np.float32):
        cm, cq = _chunk_stats(row.astype(np.float32))
        m, q = _merge_pairwise(cm.astype(np.float32), cq.astype(np.float32))
        r64 = row.astype(np.float64)
        assert abs(float(m) - r64.mean()) <= 1e-6 * max(1.0, abs(r64.mean()))
        assert abs(float(q) / D - r64.var()) <= 1e-5 * r64.var()
