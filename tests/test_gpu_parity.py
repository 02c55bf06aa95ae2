"""The CUDA path against the CPU oracle, through the C ABI (include/kimodo.h).

Workloads: the five configurations of the denoiser (fp32 root forward; one bf16
two-stage step; 50-step B=1 generation; 100-step B=16 generation; ragged B=64
generation with garbage padding), on seeded random-init weights and inputs.
Tolerances: fp32 path max|g - o| / max|o| <= 1e-4; bf16 path relative L2 <= 2e-2
per forward / step prediction and <= 5e-2 on a full trajectory; valid frames only,
padded frames must be exactly 0.
"""
import math

import numpy as np
import pytest
import torch

import synth
import transformer_denoiser_b200 as kb
from gpu_fixtures import blob, gpu_bf16, gpu_fp32, max_abs_rel, padded, params, rel_l2, valid  # noqa: F401
from oracle import kimodo_oracle as ko
from oracle_jobs import C3, C4, C5, VAR, c5_sequences, workload_inputs

pytestmark = pytest.mark.gpu

TOL_FP32 = 1e-4
TOL_BF16_FWD = 2e-2
TOL_BF16_TRAJ = 5e-2
AB = ko.alphabar_linear()


def _forward_case(model, params, net, B, T, lengths, t, seed):
    din = 5 if net == kb.NET_ROOT else 279
    x = synth.noise(B, T, din, seed=seed)
    x = synth.fill_padding(x, lengths, seed=seed + 1)
    emb = synth.text_embeddings(B, seed=seed + 2)
    got = model.denoiser_forward(net, x, emb, t, np.array(lengths, np.int32))
    name = "root" if net == kb.NET_ROOT else "body"
    ref = np.stack([ko.denoiser_forward(params[name], x[b], emb[b], t, lengths[b]) for b in range(B)])
    return got, ref


def report(name, err, tol):
    print(f"PARITY {name}: {err:.3e} (tolerance {tol:.0e})")
    assert err <= tol, (name, err)


def test_fp32_root_forward_c1(gpu_fp32, params):
    """Single root-transformer forward at t=999, B=1, T=30 (fp32)."""
    got, ref = _forward_case(gpu_fp32, params, kb.NET_ROOT, 1, 30, [30], 999, 300)
    report("fp32 root forward c1 max-abs-rel", max_abs_rel(got, ref), TOL_FP32)


def test_fp32_body_forward_ragged(gpu_fp32, params):
    got, ref = _forward_case(gpu_fp32, params, kb.NET_BODY, 2, 40, [40, 17], 480, 301)
    report("fp32 body forward ragged max-abs-rel", max_abs_rel(valid(got, [40, 17]), valid(ref, [40, 17])), TOL_FP32)
    assert np.all(padded(got, [40, 17]) == 0)


def test_fp32_ddim_step_c1(gpu_fp32, params):
    """Root + body forward and one DDIM update 999 -> 979 (fp32, B=1, T=30)."""
    B, T, L = 1, 30, [30]
    x = synth.noise(B, T)
    emb = synth.text_embeddings(B)
    null = np.zeros(4096, np.float32)
    for t, tp in [(999, 979), (999, -1)]:
        got = gpu_fp32.ddim_step(x, emb, null, np.array(L, np.int32), t, tp, 2.0)
        ref, _ = ko.ddim_step(params, x[0], emb[0], null, L[0], t, tp, 2.0, AB)
        report(f"fp32 ddim_step c1 {t}->{tp} max-abs-rel", max_abs_rel(got[0], ref), TOL_FP32)


@pytest.mark.parametrize("net", [kb.NET_ROOT, kb.NET_BODY])
def test_bf16_forward(gpu_bf16, params, net):
    L = [150, 97]
    got, ref = _forward_case(gpu_bf16, params, net, 2, 150, L, 731, 310 + net)
    report(f"bf16 forward net={net} rel-L2", rel_l2(valid(got, L), valid(ref, L)), TOL_BF16_FWD)
    assert np.all(padded(got, L) == 0)


def test_bf16_ddim_step_c2(gpu_bf16, params):
    """One two-stage bf16 step, B=1, T=150, CFG 2.0 (cond N(0,1) embedding, zero uncond)."""
    B, T, L = 1, 150, [150]
    x = synth.noise(B, T)
    emb = synth.text_embeddings(B)
    null = np.zeros(4096, np.float32)
    # with t_prev = -1 the update returns the guided x0 prediction itself
    got0 = gpu_bf16.ddim_step(x, emb, null, np.array(L, np.int32), 999, -1, 2.0)
    ref0, st = ko.ddim_step(params, x[0], emb[0], null, 150, 999, -1, 2.0, AB)
    report("bf16 ddim_step c2 x0 (cfg 2.0) rel-L2", rel_l2(got0[0], ref0), TOL_BF16_FWD)
    # 999 -> 979: compare the prediction-carrying part x_prev - c1 x_t
    got = gpu_bf16.ddim_step(x, emb, null, np.array(L, np.int32), 999, 979, 2.0)
    ref, _ = ko.ddim_step(params, x[0], emb[0], null, 150, 999, 979, 2.0, AB)
    c1 = math.sqrt(1 - AB[979]) / math.sqrt(1 - AB[999])
    report("bf16 ddim_step c2 999->979 (x_prev - c1 x_t) rel-L2", rel_l2(got[0] - c1 * x[0], ref - c1 * x[0]),
           TOL_BF16_FWD)
    report("bf16 ddim_step c2 999->979 x_prev rel-L2", rel_l2(got[0], ref), 1e-3)


def test_bf16_ddim_step_ragged_batch_and_null_broadcast(gpu_bf16, params):
    B, T, L = 3, 60, [60, 33, 1]
    x = synth.fill_padding(synth.noise(B, T, seed=41), L)
    emb = synth.text_embeddings(B, seed=42)
    null1 = np.zeros(4096, np.float32)
    nullB = np.zeros((B, 4096), np.float32)
    Li = np.array(L, np.int32)
    a = gpu_bf16.ddim_step(x, emb, null1, Li, 999, -1, 2.5)
    b = gpu_bf16.ddim_step(x, emb, nullB, Li, 999, -1, 2.5)
    np.testing.assert_array_equal(a, b)
    for i in range(B):
        ref, _ = ko.ddim_step(params, x[i], emb[i], null1, L[i], 999, -1, 2.5, AB)
        report(f"bf16 ddim_step ragged seq {i} len {L[i]} x0 (cfg 2.5) rel-L2", rel_l2(a[i, :L[i]], ref[:L[i]]),
               TOL_BF16_FWD)
    assert np.all(padded(a, L) == 0)


def test_bf16_sample_c3(gpu_bf16, oracle_refs):
    """50-step generation, B=1, 180 frames, CFG 2.0: trajectory within 5e-2."""
    emb, null, noise, L = workload_inputs(C3)
    got = gpu_bf16.ddim_sample(emb, null, noise, L, C3[3], C3[4])
    assert np.all(np.isfinite(got))
    report("bf16 sample c3 (50 steps, T=180) trajectory rel-L2", rel_l2(got[0], oracle_refs.result(C3, 0)),
           TOL_BF16_TRAJ)


def test_sample_equals_repeated_steps(gpu_bf16):
    """The captured loop gives what step-by-step calls give (same kernels)."""
    B, T, L = 2, 20, np.array([20, 13], np.int32)
    x = synth.fill_padding(synth.noise(B, T, seed=51), L)
    emb = synth.text_embeddings(B, seed=52)
    null = np.zeros(4096, np.float32)
    out = gpu_bf16.ddim_sample(emb, null, x, L, 5, 2.0)
    y = x.copy()
    for t, tp in ko.ddim_timesteps(5):
        y = gpu_bf16.ddim_step(y, emb, null, L, t, tp, 2.0)
    np.testing.assert_allclose(out, y, rtol=0, atol=1e-5)


def test_host_and_device_pointers_agree(gpu_bf16):
    B, T, L = 2, 30, np.array([30, 11], np.int32)
    x = synth.noise(B, T, seed=61)
    emb = synth.text_embeddings(B, seed=62)
    null = np.zeros(4096, np.float32)
    host = gpu_bf16.ddim_sample(emb, null, x, L, 4, 2.0)
    dev = gpu_bf16.ddim_sample(torch.from_numpy(emb).cuda(), torch.from_numpy(null).cuda(),
                               torch.from_numpy(x).cuda(), torch.from_numpy(L).cuda(), 4, 2.0)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(host, dev.cpu().numpy())
    gpu_bf16.sync_status()


@pytest.mark.parametrize("precision", ["bf16", "fp32"])
def test_packed_layout_equals_padded_layout(gpu_bf16, gpu_fp32, precision):
    """Ragged lengths given in host memory run on the packed token layout (valid tokens
    only); the same lengths in device memory run on the padded layout.  Below the pair
    GEMM's row threshold every output element is computed in the same order either way,
    so the two agree bit for bit, and padded frames are 0 in both."""
    model = gpu_bf16 if precision == "bf16" else gpu_fp32
    B, T, L = 3, 60, np.array([60, 33, 1], np.int32)
    x = synth.fill_padding(synth.noise(B, T, seed=71), L)
    emb = synth.text_embeddings(B, seed=72)
    null = np.zeros(4096, np.float32)
    packed = model.ddim_step(x, emb, null, L, 999, 966, 2.0)
    padded_ = model.ddim_step(x, emb, null, torch.from_numpy(L).cuda(), 999, 966, 2.0)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(packed, padded_)
    assert np.all(padded(packed, L) == 0)
    fp = model.denoiser_forward(kb.NET_BODY, x, emb, 500, L)
    fd = model.denoiser_forward(kb.NET_BODY, x, emb, 500, torch.from_numpy(L).cuda())
    torch.cuda.synchronize()
    np.testing.assert_array_equal(fp, fd)
    assert np.all(padded(fp, L) == 0)
    s1 = model.ddim_sample(emb, null, x, L, 3, 2.0)
    s2 = model.ddim_sample(emb, null, x, torch.from_numpy(L).cuda(), 3, 2.0)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(s1, s2)


def test_c4_full_size_sampled(gpu_bf16, oracle_refs):
    """100-step generation at B=16, T=150 (the throughput workload, as bench.py
    runs it): sequences 0 and 15 against the oracle over all 100 steps, sequence 15
    also against the same prompt sampled alone (every projection tile sums its full K
    extent in the same order at any batch size, though alone the projections run on the
    single-CTA kernel: checked to 1e-4); every output finite."""
    emb, null, noise, L = workload_inputs(C4)
    got = gpu_bf16.ddim_sample(emb, null, noise, L, C4[3], C4[4])
    assert np.all(np.isfinite(got))
    alone = gpu_bf16.ddim_sample(emb[15:16], null, noise[15:16], L[15:16], C4[3], C4[4])
    report("c4 seq 15 batched vs alone rel-L2", rel_l2(got[15], alone[0]), 1e-4)
    for b in (0, 15):
        report(f"bf16 sample c4 seq {b} (100 steps) trajectory rel-L2", rel_l2(got[b], oracle_refs.result(C4, b)),
               TOL_BF16_TRAJ)


def test_c5_ragged_garbage_sampled(gpu_bf16, oracle_refs):
    """50-step ragged batch, B=64, lengths U{60..300} padded to 300 frames with
    garbage, CFG 2.5: the shortest, the longest and two seeded random sequences
    against the oracle; garbage, zeros and NaN in the padding give bit-identical
    results; the padded token layout agrees with the packed one."""
    emb, null, garbage, L = workload_inputs(C5)
    got = gpu_bf16.ddim_sample(emb, null, garbage, L, C5[3], C5[4])
    assert np.all(np.isfinite(got))
    assert np.all(padded(got, L) == 0)
    noise = synth.noise(C5[1], C5[2])
    zeros = noise.copy()
    for b in range(C5[1]):
        zeros[b, L[b]:] = 0
    np.testing.assert_array_equal(gpu_bf16.ddim_sample(emb, null, zeros, L, C5[3], C5[4]), got)
    nans = synth.fill_padding(noise, L, nan=True)
    np.testing.assert_array_equal(gpu_bf16.ddim_sample(emb, null, nans, L, C5[3], C5[4]), got)
    # lengths in device memory: the padded token layout, the same result up to summation order
    dense = gpu_bf16.ddim_sample(emb, null, garbage, torch.from_numpy(L).cuda(), C5[3], C5[4])
    torch.cuda.synchronize()
    report("bf16 sample c5 padded vs packed layout rel-L2", rel_l2(valid(dense, L), valid(got, L)), 1e-2)
    for b in c5_sequences():
        n = int(L[b])
        report(f"bf16 sample c5 seq {b} len {n} (50 steps, cfg 2.5) trajectory rel-L2",
               rel_l2(got[b, :n], oracle_refs.result(C5, b)[:n]), TOL_BF16_TRAJ)


def test_variations_against_oracle(gpu_bf16, oracle_refs):
    """Variations of a prompt: 2 prompts x 3 takes with their own noise (text rows shared
    by the takes), 10 steps; every sequence against the oracle run on its prompt."""
    prompts, null, noise, L = workload_inputs(VAR)
    got = gpu_bf16.ddim_sample(prompts, null, noise, L, VAR[3], VAR[4])
    for b in range(VAR[1]):
        report(f"bf16 variations seq {b} (prompt {b // 3}) trajectory rel-L2",
               rel_l2(got[b], oracle_refs.result(VAR, b)), TOL_BF16_TRAJ)

