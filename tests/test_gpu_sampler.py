"""Sampler options of the C ABI (kimodo_ddim_step_ex / kimodo_ddim_sample_ex) against
the oracle: cosine schedule, step counts that do not divide 1000, and eta > 0 with
the caller's standard-normal draws.  Tolerances as in the parity tests: fp32
max|g - o| / max|o| <= 1e-4; bf16 relative L2 <= 2e-2 per step prediction and
<= 5e-2 on a trajectory."""
import ctypes
import math

import numpy as np
import pytest
import torch

import synth
import transformer_denoiser_b200 as kb
from gpu_fixtures import blob, gpu_bf16, gpu_fp32, max_abs_rel, padded, params, rel_l2, valid  # noqa: F401
from oracle import kimodo_oracle as ko

pytestmark = pytest.mark.gpu

AB_COS = ko.alphabar_cosine()


def report(name, err, tol):
    print(f"PARITY {name}: {err:.3e} (tolerance {tol:.0e})")
    assert err <= tol, (name, err)


def _coeffs(ab, t, tp, eta):
    at, ap = ab[t], (1.0 if tp < 0 else ab[tp])
    sigma = ko.ddim_sigma(at, ap, eta)
    return math.sqrt(1 - ap - sigma * sigma) / math.sqrt(1 - at), sigma


def test_fp32_step_cosine_eta(gpu_fp32, params):
    B, T, L = 1, 30, [30]
    x = synth.noise(B, T, seed=401)
    z = synth.noise(B, T, seed=402)
    emb = synth.text_embeddings(B, seed=403)
    null = np.zeros(4096, np.float32)
    got = gpu_fp32.ddim_step(x, emb, null, np.array(L, np.int32), 999, 932, 2.0, schedule="cosine", eta=0.8,
                             step_noise=z)
    ref, _ = ko.ddim_step(params, x[0], emb[0], null, L[0], 999, 932, 2.0, AB_COS, eta=0.8, z=z[0])
    report("fp32 ddim_step cosine eta 0.8 999->932 max-abs-rel", max_abs_rel(got[0], ref), 1e-4)


def test_bf16_step_cosine_eta_prediction(gpu_bf16, params):
    B, T, L = 2, 50, [50, 21]
    x = synth.fill_padding(synth.noise(B, T, seed=411), L, seed=412)
    z = synth.fill_padding(synth.noise(B, T, seed=413), L, seed=414)
    emb = synth.text_embeddings(B, seed=415)
    null = np.zeros(4096, np.float32)
    zd = torch.from_numpy(z).cuda()
    got = gpu_bf16.ddim_step(x, emb, null, np.array(L, np.int32), 999, 932, 2.0, schedule="cosine", eta=1.0,
                             step_noise=zd)
    torch.cuda.synchronize()
    c1, sigma = _coeffs(AB_COS, 999, 932, 1.0)
    assert sigma > 0.1
    for b in range(B):
        ref, _ = ko.ddim_step(params, x[b], emb[b], null, L[b], 999, 932, 2.0, AB_COS, eta=1.0, z=z[b])
        n = L[b]
        part = lambda v: v[:n] - c1 * x[b, :n] - sigma * z[b, :n]   # noqa: E731  (the prediction-carrying part)
        report(f"bf16 step cosine eta 1 seq {b} (x_prev - c1 x_t - sigma z) rel-L2", rel_l2(part(got[b]), part(ref)),
               2e-2)
        report(f"bf16 step cosine eta 1 seq {b} x_prev rel-L2", rel_l2(got[b, :n], ref[:n]), 1e-2)
    assert np.all(padded(got, L) == 0)


def test_bf16_sample_nondivisor_cosine_eta_trajectory(gpu_bf16, params):
    """7 steps (does not divide 1000), cosine schedule, eta 0.6, host draws."""
    B, T, L, steps = 1, 24, [24], 7
    noise = synth.noise(B, T, seed=421)
    sn = synth.random_vectors((steps, B, T, 279), 422, 1.0)
    emb = synth.text_embeddings(B, seed=423)
    null = np.zeros(4096, np.float32)
    got = gpu_bf16.ddim_sample(emb, null, noise, np.array(L, np.int32), steps, 2.0, schedule="cosine", eta=0.6,
                               step_noise=sn)
    ref = ko.ddim_sample(params, emb[0], null, noise[0], L[0], steps, 2.0, schedule="cosine", eta=0.6,
                         step_noise=sn[:, 0])
    assert np.all(np.isfinite(got))
    report("bf16 sample 7 steps cosine eta 0.6 trajectory rel-L2", rel_l2(got[0], ref), 5e-2)


def test_sample_ex_equals_repeated_step_ex(gpu_bf16):
    B, T, L, steps = 2, 20, np.array([20, 13], np.int32), 3
    x = synth.fill_padding(synth.noise(B, T, seed=431), L)
    sn = torch.from_numpy(synth.random_vectors((steps, B, T, 279), 432, 1.0)).cuda()
    emb = synth.text_embeddings(B, seed=433)
    null = np.zeros(4096, np.float32)
    out = gpu_bf16.ddim_sample(emb, null, x, L, steps, 2.0, schedule="cosine", eta=0.5, step_noise=sn)
    y = x.copy()
    for k, (t, tp) in enumerate(ko.ddim_timesteps_trailing(steps)):
        y = gpu_bf16.ddim_step(y, emb, null, L, t, tp, 2.0, schedule="cosine", eta=0.5, step_noise=sn[k].contiguous())
        torch.cuda.synchronize()
    np.testing.assert_allclose(out, y, rtol=0, atol=1e-5)
    assert np.all(padded(out, L) == 0)


def test_step_noise_buffer_is_read_on_every_replay(gpu_bf16):
    """The cached graph of a device step-noise buffer reads the buffer's current contents."""
    B, T, L, steps = 1, 16, np.array([16], np.int32), 4
    x = synth.noise(B, T, seed=441)
    emb = synth.text_embeddings(B, seed=442)
    null = np.zeros(4096, np.float32)
    z1 = torch.from_numpy(synth.random_vectors((steps, B, T, 279), 443, 1.0)).cuda()
    z2 = torch.from_numpy(synth.random_vectors((steps, B, T, 279), 444, 1.0)).cuda()
    buf = z1.clone()
    a = gpu_bf16.ddim_sample(emb, null, x, L, steps, 2.0, eta=1.0, step_noise=buf)
    buf.copy_(z2)
    b = gpu_bf16.ddim_sample(emb, null, x, L, steps, 2.0, eta=1.0, step_noise=buf)
    buf.copy_(z1)
    c = gpu_bf16.ddim_sample(emb, null, x, L, steps, 2.0, eta=1.0, step_noise=buf)
    torch.cuda.synchronize()
    assert np.abs(a - b).max() > 1e-3
    np.testing.assert_array_equal(a, c)


def test_eta_zero_linear_options_equal_the_plain_call(gpu_bf16):
    B, T, L = 1, 16, np.array([16], np.int32)
    x = synth.noise(B, T, seed=451)
    emb = synth.text_embeddings(B, seed=452)
    null = np.zeros(4096, np.float32)
    plain = gpu_bf16.ddim_sample(emb, null, x, L, 5, 2.0)
    lib = gpu_bf16._lib
    out = np.empty_like(x)
    opts = kb.SamplerOptions(0, 0.0, None)
    st = torch.cuda.current_stream().cuda_stream
    kb._check(lib.kimodo_ddim_sample_ex(gpu_bf16._ctx, emb.ctypes.data, null.ctypes.data, 1, x.ctypes.data,
                                        L.ctypes.data, B, T, 5, 2.0, ctypes.byref(opts), out.ctypes.data, st))
    np.testing.assert_array_equal(plain, out)


@pytest.mark.parametrize("schedule,eta,noise,steps", [(7, 0.0, False, 5), (0, 1.5, True, 5), (0, -0.1, True, 5),
                                                      (0, float("nan"), True, 5), (1, 0.3, False, 5),
                                                      (0, 0.0, False, 0), (0, 0.0, False, 1001)])
def test_sampler_option_errors(gpu_bf16, schedule, eta, noise, steps):
    B, T = 1, 8
    x = synth.noise(B, T, seed=461)
    emb = synth.text_embeddings(B, seed=462)
    null = np.zeros(4096, np.float32)
    L = np.array([8], np.int32)
    z = synth.random_vectors((max(steps, 1), B, T, 279), 463, 1.0)
    opts = kb.SamplerOptions(schedule, eta, z.ctypes.data if noise else None)
    out = np.empty_like(x)
    st = torch.cuda.current_stream().cuda_stream
    rc = gpu_bf16._lib.kimodo_ddim_sample_ex(gpu_bf16._ctx, emb.ctypes.data, null.ctypes.data, 1, x.ctypes.data,
                                             L.ctypes.data, B, T, steps, 2.0, ctypes.byref(opts), out.ctypes.data, st)
    assert rc == -1, rc


def test_variations_share_prompt_rows(gpu_bf16):
    """Several takes of one prompt (text_batch < batch): sequence b uses prompt row
    b // takes; the result equals the call with the rows repeated, and takes differ
    only by their noise."""
    B, T, L = 6, 20, np.full(6, 20, np.int32)
    prompts = synth.text_embeddings(2, seed=471)
    noise = synth.noise(B, T, seed=472)
    null = np.zeros(4096, np.float32)
    var = gpu_bf16.ddim_sample(prompts, null, noise, L, 4, 2.0)
    rep = gpu_bf16.ddim_sample(np.repeat(prompts, 3, axis=0), null, noise, L, 4, 2.0)
    np.testing.assert_array_equal(var, rep)
    assert np.abs(var[0] - var[1]).max() > 1e-3
    same = gpu_bf16.ddim_sample(prompts, null, np.repeat(noise[:1], B, axis=0), L, 4, 2.0)
    np.testing.assert_array_equal(same[0], same[2])          # same prompt, same noise
    assert np.abs(same[0] - same[3]).max() > 1e-3             # other prompt
    vs = gpu_bf16.ddim_step(noise, prompts, null, L, 999, 749, 2.0)
    rs = gpu_bf16.ddim_step(noise, np.repeat(prompts, 3, axis=0), null, L, 999, 749, 2.0)
    np.testing.assert_array_equal(vs, rs)


def test_text_batch_must_divide_batch(gpu_bf16):
    B, T = 6, 8
    x = synth.noise(B, T, seed=481)
    emb = synth.text_embeddings(4, seed=482)
    null = np.zeros(4096, np.float32)
    L = np.full(B, T, np.int32)
    opts = kb.SamplerOptions(0, 0.0, None, 4)
    out = np.empty_like(x)
    st = torch.cuda.current_stream().cuda_stream
    rc = gpu_bf16._lib.kimodo_ddim_sample_ex(gpu_bf16._ctx, emb.ctypes.data, null.ctypes.data, 1, x.ctypes.data,
                                             L.ctypes.data, B, T, 3, 2.0, ctypes.byref(opts), out.ctypes.data, st)
    assert rc == -1, rc


def test_device_timeout_is_reported_and_the_context_recovers(gpu_bf16):
    """A bounded wait that runs out (kimodo_wait_selftest: a barrier that nothing
    completes, 2 ms limit) records KIMODO_ETIMEOUT; kimodo_sync_status reports it with
    the stage's name and clears it; the next call computes what it computed before."""
    B, T, L = 1, 20, np.array([20], np.int32)
    x = synth.noise(B, T, seed=491)
    emb = synth.text_embeddings(B, seed=492)
    null = np.zeros(4096, np.float32)
    before = gpu_bf16.ddim_step(x, emb, null, L, 999, 899, 2.0)
    gpu_bf16.sync_status()
    gpu_bf16.wait_selftest(2000)
    with pytest.raises(kb.KimodoError) as e:
        gpu_bf16.sync_status()
    assert e.value.status == -5 and "wait self-test" in str(e.value)
    gpu_bf16.sync_status()                       # cleared
    after = gpu_bf16.ddim_step(x, emb, null, L, 999, 899, 2.0)
    gpu_bf16.sync_status()
    np.testing.assert_array_equal(before, after)
