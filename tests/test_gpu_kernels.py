"""Each CUDA kernel of the path against the oracle's elementary operation, called
through the kernel-level C ABI (include/kimodo_kernels.h).  Inputs are seeded;
the oracle computes in float64 on the bf16-rounded operands the kernel sees."""
import numpy as np
import pytest
import torch

import synth
import transformer_denoiser_b200 as kb
from gpu_fixtures import require_cuda
from oracle import kimodo_oracle as ko

pytestmark = pytest.mark.gpu


def _bf16(a):
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(torch.bfloat16)


def _f64(t):
    return t.float().cpu().double().numpy()


def _epi_ref(kind, acc, resid=None):
    if kind == kb.EPI_BIAS_GELU:
        return ko.gelu(acc)
    if kind == kb.EPI_BIAS_SILU:
        return ko.silu(acc)
    if kind == kb.EPI_BIAS_RESID:
        return acc + resid
    return acc


GEMM_CASES = [
    # M, N, K, lda, epilogue, out_f32, tile_n
    (300, 1024, 1024, 1024, kb.EPI_BIAS, False, 128),
    (300, 1024, 1024, 1024, kb.EPI_BIAS, False, 256),
    (4832, 3072, 1024, 1024, kb.EPI_BIAS, False, 256),     # QKV at 32 x 151 tokens
    (129, 2048, 1024, 1024, kb.EPI_BIAS_GELU, False, 256),
    (302, 1024, 2048, 2048, kb.EPI_BIAS_RESID, True, 128),
    (4832, 1024, 2048, 2048, kb.EPI_BIAS_RESID, True, 256),
    (1, 1024, 64, 64, kb.EPI_BIAS_SILU, False, 128),
    (257, 1024, 279, 320, kb.EPI_BIAS, True, 128),         # body input width, ragged K
    (200, 274, 1024, 1024, kb.EPI_BIAS, True, 128),        # body output width, ragged N
    (100, 1024, 4096, 4096, kb.EPI_BIAS, True, 128),       # text projection
    (362, 3072, 1024, 1024, kb.EPI_BIAS, False, 64),       # narrow tiles for a few hundred tokens
    (362, 2048, 1024, 1024, kb.EPI_BIAS_GELU, False, 64),
    (362, 1024, 2048, 2048, kb.EPI_BIAS_RESID, True, 32),
    (300, 1040, 1024, 1024, kb.EPI_BIAS_RESID, True, 64),  # ragged last tile, partial epilogue parts
    (130, 1008, 1024, 1024, kb.EPI_BIAS, False, 32),
    (5, 2048, 1024, 1024, kb.EPI_BIAS_GELU, False, 32),
]


@pytest.mark.parametrize("M,N,K,lda,epi,out_f32,tile", GEMM_CASES)
def test_gemm_tcgen05_vs_oracle(M, N, K, lda, epi, out_f32, tile):
    require_cuda()
    seed = M * 7 + N * 3 + K
    A = _bf16(synth.random_vectors((M, lda), seed))
    W = _bf16(synth.random_vectors((N, lda), seed + 1, 0.05))
    bias = torch.from_numpy(synth.random_vectors((N,), seed + 2, 0.1))
    resid = torch.from_numpy(synth.random_vectors((M, N), seed + 3)) if epi == kb.EPI_BIAS_RESID else None
    dev = "cuda"
    ldo = (N + 7) // 8 * 8     # output rows padded to a 16-byte multiple
    buf = torch.empty((M, ldo), dtype=torch.float32 if out_f32 else torch.bfloat16, device=dev)
    out = kb.gemm_bf16(A.to(dev), W.to(dev), bias.to(dev), epi, out_f32,
                       None if resid is None else resid.to(dev), out=buf[:, :N], K=K, tile_n=tile)
    torch.cuda.synchronize()
    ref = _epi_ref(epi, ko.linear(_f64(A)[:, :K], _f64(W)[:, :K], bias.double().numpy()),
                   None if resid is None else resid.double().numpy())
    got = out.float().cpu().double().numpy()
    scale = np.abs(ref).max()
    if out_f32:
        np.testing.assert_allclose(got, ref, rtol=0, atol=2e-5 * scale)
    else:   # bf16 output rounding: half an ulp of 8 mantissa bits
        np.testing.assert_allclose(got, ref, rtol=2 ** -8, atol=1e-5 * scale)


PAIR_CASES = [
    # M, N, K, epilogue, out_f32, tile_n (CTA-pair kernel: 256-row tiles)
    (4832, 3072, 1024, kb.EPI_BIAS, False, 208),
    (4832, 3072, 1024, kb.EPI_BIAS, False, 256),
    (4832, 2048, 1024, kb.EPI_BIAS_GELU, False, 144),
    (4832, 1024, 1024, kb.EPI_BIAS_RESID, True, 160),
    (4832, 1024, 2048, kb.EPI_BIAS_RESID, True, 144),
    (611, 1024, 1024, kb.EPI_BIAS_RESID, True, 160),
    (300, 1024, 1024, kb.EPI_BIAS, False, 160),           # second CTA of the last pair tile fully out of range
    (1283, 2048, 1024, kb.EPI_BIAS_GELU, False, 256),
]


@pytest.mark.parametrize("M,N,K,epi,out_f32,tile", PAIR_CASES)
def test_gemm_tcgen05_pair_vs_oracle(M, N, K, epi, out_f32, tile):
    require_cuda()
    seed = M * 5 + N * 7 + K + tile
    A = _bf16(synth.random_vectors((M, K), seed))
    W = _bf16(synth.random_vectors((N, K), seed + 1, 0.05))
    bias = torch.from_numpy(synth.random_vectors((N,), seed + 2, 0.1))
    resid = torch.from_numpy(synth.random_vectors((M, N), seed + 3)) if epi == kb.EPI_BIAS_RESID else None
    out = kb.gemm_bf16(A.cuda(), W.cuda(), bias.cuda(), epi, out_f32, None if resid is None else resid.cuda(),
                       tile_n=tile, pair=True)
    torch.cuda.synchronize()
    ref = _epi_ref(epi, ko.linear(_f64(A), _f64(W), bias.double().numpy()),
                   None if resid is None else resid.double().numpy())
    got = out.float().cpu().double().numpy()
    scale = np.abs(ref).max()
    if out_f32:
        np.testing.assert_allclose(got, ref, rtol=0, atol=2e-5 * scale)
    else:
        np.testing.assert_allclose(got, ref, rtol=2 ** -8, atol=1e-5 * scale)


def test_gemm_residual_in_place():
    """The residual epilogue may read and write the same fp32 buffer."""
    require_cuda()
    M, N, K = 300, 1024, 1024
    A = _bf16(synth.random_vectors((M, K), 91)).cuda()
    W = _bf16(synth.random_vectors((N, K), 92, 0.05)).cuda()
    bias = torch.from_numpy(synth.random_vectors((N,), 93, 0.1)).cuda()
    y = torch.from_numpy(synth.random_vectors((M, N), 94)).cuda()
    want = kb.gemm_bf16(A, W, bias, kb.EPI_BIAS_RESID, True, y.clone())
    kb.gemm_bf16(A, W, bias, kb.EPI_BIAS_RESID, True, y, out=y)
    torch.cuda.synchronize()
    assert torch.equal(want, y)


@pytest.mark.parametrize("M,N,K,epi", [(300, 1024, 1024, kb.EPI_BIAS), (129, 2048, 1024, kb.EPI_BIAS_GELU),
                                       (77, 1024, 2048, kb.EPI_BIAS_RESID), (33, 274, 1024, kb.EPI_BIAS),
                                       (5, 1024, 64, kb.EPI_BIAS_SILU)])
def test_gemm_f32_vs_oracle(M, N, K, epi):
    require_cuda()
    seed = 5 * M + N + 11 * K
    A = torch.from_numpy(synth.random_vectors((M, K), seed))
    W = torch.from_numpy(synth.random_vectors((N, K), seed + 1, 0.05))
    bias = torch.from_numpy(synth.random_vectors((N,), seed + 2, 0.1))
    resid = torch.from_numpy(synth.random_vectors((M, N), seed + 3)) if epi == kb.EPI_BIAS_RESID else None
    out = kb.gemm_f32(A.cuda(), W.cuda(), bias.cuda(), epi, None if resid is None else resid.cuda())
    ref = _epi_ref(epi, ko.linear(A.double().numpy(), W.double().numpy(), bias.double().numpy()),
                   None if resid is None else resid.double().numpy())
    np.testing.assert_allclose(out.cpu().double().numpy(), ref, rtol=0, atol=2e-6 * np.abs(ref).max())


def test_gelu_epilogue_error_bound():
    """GELU of the epilogues against the exact erf GELU on a dense grid.  The erf
    approximation (Abramowitz & Stegun 7.1.26) is within 1.5e-7 of erf; evaluating
    1 - p(t) exp(-z^2) in fp32 adds up to 2 ulp of 1.0 (2.4e-7), so
    |GELU error| <= 0.5 |x| (1.5e-7 + 2.4e-7) plus the fp32 rounding of the result."""
    require_cuda()
    x = np.linspace(-9, 9, 4096).astype(np.float32)
    A = np.zeros((x.size, 16), np.float32)
    A[:, 0] = x
    W = np.zeros((16, 16), np.float32)
    W[0, 0] = 1.0
    out = kb.gemm_f32(torch.from_numpy(A).cuda(), torch.from_numpy(W).cuda(), torch.zeros(16, device="cuda"),
                      kb.EPI_BIAS_GELU)
    got = out[:, 0].cpu().double().numpy()
    ref = ko.gelu(x.astype(np.float64))
    bound = 0.5 * np.abs(x) * (1.5e-7 + 2 * np.finfo(np.float32).eps) \
        + 4 * np.finfo(np.float32).eps * np.maximum(np.abs(ref), 1e-3)
    assert np.all(np.abs(got - ref) <= bound), float(np.max(np.abs(got - ref) - bound))


@pytest.mark.parametrize("pair,tile", [(False, 128), (True, 160)])
def test_gelu_bf16_epilogue_error_bound(pair, tile):
    """GELU of the bf16-output tensor-core epilogues against the exact erf GELU on a
    dense grid.  erf there is Abramowitz & Stegun 7.1.28 (|error| <= 3e-7) with an
    approximate reciprocal raised to the 16th power (relative error <= 16 * 2^-22),
    so with fp32 evaluation |GELU error| <= 0.5 |x| * 8e-6 before the result is rounded to bf16 (half an
    ulp of 8 significant bits)."""
    require_cuda()
    x = torch.linspace(-9, 9, 4096).to(torch.bfloat16)
    A = torch.zeros((x.numel(), 64), dtype=torch.bfloat16)
    A[:, 0] = x
    W = torch.zeros((16, 64), dtype=torch.bfloat16)
    W[:, 0] = 1.0
    out = kb.gemm_bf16(A.cuda(), W.cuda(), torch.zeros(16, device="cuda"), kb.EPI_BIAS_GELU, False,
                       tile_n=tile, pair=pair)
    torch.cuda.synchronize()
    got = out.float().cpu().double().numpy()
    xd = x.double().numpy()
    ref = ko.gelu(xd)[:, None]
    err = 0.5 * np.abs(xd)[:, None] * 8e-6
    bound = 2.0 ** -8 * np.abs(ref) + 1.01 * err + 1e-30
    assert np.all(np.abs(got - ref) <= bound), float(np.max(np.abs(got - ref) - bound))


def _attention_ref(qkv, lengths, S):
    nseq = len(lengths)
    out = np.zeros((nseq * S, 1024))
    for s in range(nseq):
        rows = qkv[s * S:(s + 1) * S]
        n_valid = 1 + int(lengths[s])
        for h in range(8):
            sl = slice(h * 128, (h + 1) * 128)
            q, k, v = rows[:, sl], rows[:, 1024:][:, sl], rows[:, 2048:][:, sl]
            out[s * S:(s + 1) * S, sl] = ko.attention(q, k, v, n_valid)
    return out


@pytest.mark.parametrize("S,lengths", [(31, [30]), (151, [150, 60, 0]), (301, [300, 123]), (64, [63, 64])])
def test_attention_bf16_vs_oracle(S, lengths):
    require_cuda()
    lengths = [min(n, S - 1) for n in lengths]
    nseq = len(lengths)
    qkv = _bf16(synth.random_vectors((nseq * S, 3072), S + 100))
    L = torch.tensor(lengths, dtype=torch.int32)
    out = kb.attention(qkv.cuda(), L.cuda(), nseq, S)
    ref = _attention_ref(_f64(qkv), lengths, S)
    got = out.float().cpu().double().numpy()
    err = np.linalg.norm(got - ref) / np.linalg.norm(ref)
    assert err < 1e-2, err
    assert np.abs(got - ref).max() < 3e-2 * np.abs(ref).max()


def test_attention_bf16_masked_keys_never_read():
    require_cuda()
    S, lengths = 151, [40, 150]
    qkv = _bf16(synth.random_vectors((2 * S, 3072), 77)).cuda()
    L = torch.tensor(lengths, dtype=torch.int32).cuda()
    base = kb.attention(qkv, L, 2, S)
    poisoned = qkv.clone()
    for s, n in enumerate(lengths):
        poisoned[s * S + 1 + n:(s + 1) * S, 1024:] = float("nan")
    again = kb.attention(poisoned, L, 2, S)
    torch.cuda.synchronize()
    assert torch.equal(base, again)


def test_attention_f32_vs_oracle():
    require_cuda()
    S, lengths = 41, [40, 7]
    qkv = torch.from_numpy(synth.random_vectors((2 * S, 3072), 5))
    L = torch.tensor(lengths, dtype=torch.int32)
    out = kb.attention(qkv.cuda(), L.cuda(), 2, S)
    ref = _attention_ref(qkv.double().numpy(), lengths, S)
    np.testing.assert_allclose(out.cpu().double().numpy(), ref, rtol=0, atol=2e-6 * np.abs(ref).max())


@pytest.mark.parametrize("M,out_bf16", [(1, True), (302, True), (4833, False)])
def test_layernorm_vs_oracle(M, out_bf16):
    require_cuda()
    rng = np.random.default_rng(M)
    y = (rng.standard_normal((M, 1024)) * 2 + 3).astype(np.float32)
    g = (1 + 0.1 * rng.standard_normal(1024)).astype(np.float32)
    b = (0.1 * rng.standard_normal(1024)).astype(np.float32)
    out = kb.layernorm(torch.from_numpy(y).cuda(), torch.from_numpy(g).cuda(), torch.from_numpy(b).cuda(), out_bf16)
    ref = ko.layer_norm(y.astype(np.float64), g.astype(np.float64), b.astype(np.float64))
    got = out.float().cpu().double().numpy()
    if out_bf16:
        np.testing.assert_allclose(got, ref, rtol=2 ** -8, atol=1e-6)
    else:
        np.testing.assert_allclose(got, ref, rtol=0, atol=1e-5)
