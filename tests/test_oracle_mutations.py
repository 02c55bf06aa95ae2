"""Plant plausible mistakes in the CPU oracle and check that a pin catches each.

Every mutation is applied with monkeypatch to the oracle module on the CPU; the
oracle file itself is never changed.
"""
import math

import numpy as np
import pytest

import test_oracle_pins as pins
from oracle import kimodo_oracle as ko


def _expect_fail(fn, *args, **kw):
    with pytest.raises(AssertionError):
        fn(*args, **kw)


def test_tanh_gelu_is_caught(monkeypatch):
    monkeypatch.setattr(ko, "gelu", lambda x: 0.5 * x * (1 + np.tanh(
        math.sqrt(2 / math.pi) * (x + 0.044715 * x ** 3))))
    _expect_fail(pins.test_encoder_layer_vs_torch, 32, 4, 64, 11, 7)


def test_pre_norm_layer_is_caught(monkeypatch):
    def pre_norm(h, lp, n_heads, n_valid):
        a = ko.multi_head_attention(ko.layer_norm(h, lp["ln1_g"], lp["ln1_b"]), lp["qkv_W"],
                                    lp["qkv_b"], lp["o_W"], lp["o_b"], n_heads, n_valid)
        h = h + a
        x = ko.layer_norm(h, lp["ln2_g"], lp["ln2_b"])
        return h + ko.linear(ko.gelu(ko.linear(x, lp["ff1_W"], lp["ff1_b"])), lp["ff2_W"], lp["ff2_b"])
    monkeypatch.setattr(ko, "encoder_layer", pre_norm)
    _expect_fail(pins.test_encoder_layer_vs_torch, 32, 4, 64, 11, 7)


def test_missing_attention_scale_is_caught(monkeypatch):
    monkeypatch.setattr(ko, "attention", lambda q, k, v, n: ko.softmax_rows(q @ k[:n].T) @ v[:n])
    _expect_fail(pins.test_attention_brute_force, 5, 5)


def test_masked_keys_multiplied_by_zero_is_caught(monkeypatch):
    def zero_mask(q, k, v, n):
        s = q @ k.T / math.sqrt(q.shape[-1])
        w = np.exp(s - s[:, :n].max(-1, keepdims=True))
        w[:, n:] = 0.0
        return (w / w.sum(-1, keepdims=True)) @ v
    monkeypatch.setattr(ko, "attention", zero_mask)
    _expect_fail(pins.test_attention_ignores_nan_in_masked_keys)


def test_swapped_qkv_split_is_caught(monkeypatch):
    real = ko.linear

    def mha(h, qkv_W, qkv_b, o_W, o_b, n_heads, n_valid):
        d = h.shape[-1]
        W = np.concatenate([qkv_W[d:2 * d], qkv_W[:d], qkv_W[2 * d:]])
        b = np.concatenate([qkv_b[d:2 * d], qkv_b[:d], qkv_b[2 * d:]])
        dh = d // n_heads
        qkv = real(h, W, b)
        q, k, v = qkv[:, :d], qkv[:, d:2 * d], qkv[:, 2 * d:]
        heads = [ko.attention(q[:, i * dh:(i + 1) * dh], k[:, i * dh:(i + 1) * dh],
                              v[:, i * dh:(i + 1) * dh], n_valid) for i in range(n_heads)]
        return real(np.concatenate(heads, -1), o_W, o_b)
    monkeypatch.setattr(ko, "multi_head_attention", mha)
    _expect_fail(pins.test_encoder_layer_vs_torch, 32, 4, 64, 11, 7)


def test_position_offset_is_caught(monkeypatch):
    real = ko.sinusoid

    def shifted(positions, d):
        p = np.asarray(positions, dtype=np.float64)
        return real(np.where(p > 0, p - 1, p), d) if p.size > 1 else real(p, d)
    monkeypatch.setattr(ko, "sinusoid", shifted)
    _expect_fail(pins.test_denoiser_forward_vs_torch_modules, "root")


def test_g2l_rotation_sign_is_caught(monkeypatch):
    def wrong(root, length):
        root = np.asarray(root, dtype=np.float64)
        out = np.zeros_like(root)
        px = pz = 0.0
        cp, sp = 1.0, 0.0
        for i in range(length):
            x, z, sr, cr, y = root[i]
            n = max(math.hypot(cr, sr), 1e-8)
            c, s = cr / n, sr / n
            vx, vz = x - px, z - pz
            out[i] = (c * vx + s * vz, -s * vx + c * vz, s * cp - c * sp, c * cp + s * sp, y)
            px, pz, cp, sp = x, z, c, s
        return out
    monkeypatch.setattr(ko, "global_root_to_local_root", wrong)
    _expect_fail(pins.test_g2l_worked_example)


def test_ddim_noise_sign_is_caught(monkeypatch):
    def wrong(x_t, x0, ab_t, ab_prev):
        eps = (x_t + math.sqrt(ab_t) * x0) / math.sqrt(1.0 - ab_t)
        return math.sqrt(ab_prev) * x0 + math.sqrt(1.0 - ab_prev) * eps
    monkeypatch.setattr(ko, "ddim_update", wrong)
    _expect_fail(pins.test_ddim_step_with_exact_x0_predictor)


def test_cfg_direction_is_caught(monkeypatch):
    monkeypatch.setattr(ko, "cfg_combine", lambda c, u, w: c + w * (u - c))
    _expect_fail(pins.test_cfg_special_cases)


def test_off_by_one_schedule_is_caught(monkeypatch):
    monkeypatch.setattr(ko, "alphabar_linear", lambda n=1000, b0=1e-4, b1=0.02: np.cumprod(
        1.0 - np.linspace(b0, b1, n + 1)[1:]))
    _expect_fail(pins.test_alphabar_exact_rational)


def test_layernorm_unbiased_variance_is_caught(monkeypatch):
    def wrong(x, g, b, eps=1e-5):
        mu = x.mean(-1, keepdims=True)
        var = x.var(-1, ddof=1, keepdims=True)
        return (x - mu) / np.sqrt(var + eps) * g + b
    monkeypatch.setattr(ko, "layer_norm", wrong)
    _expect_fail(pins.test_layer_norm_vs_torch)


def test_ddim_sigma_missing_root_is_caught(monkeypatch):
    monkeypatch.setattr(ko, "ddim_sigma", lambda at, ap, eta: eta * math.sqrt((1 - ap) / (1 - at)) * (1 - at / ap))
    _expect_fail(pins.test_ddim_eta_one_is_the_ddpm_posterior)


def test_ddim_step_noise_sign_is_caught(monkeypatch):
    real = ko.ddim_update_eta
    monkeypatch.setattr(ko, "ddim_update_eta", lambda x_t, x0, at, ap, eta, z: real(x_t, x0, at, ap, eta, -np.asarray(z)))
    _expect_fail(pins.test_ddim_eta_one_is_the_ddpm_posterior)


def test_cosine_schedule_index_shift_is_caught(monkeypatch):
    def shifted(n=1000, s=0.008, max_beta=0.999):
        def f(u):
            return math.cos((u + s) / (1.0 + s) * math.pi / 2.0) ** 2
        betas = np.array([min(1.0 - f(i / n) / f(max(i - 1, 0) / n), max_beta) for i in range(n)])
        return np.cumprod(1.0 - betas)
    monkeypatch.setattr(ko, "alphabar_cosine", shifted)
    _expect_fail(pins.test_cosine_schedule_telescopes)


def test_timestep_rounding_down_is_caught(monkeypatch):
    def floor_only(steps, n=1000):
        ts = [n * (steps - k) // steps - 1 for k in range(steps)]
        return [(ts[k], ts[k + 1] if k + 1 < steps else -1) for k in range(steps)]
    monkeypatch.setattr(ko, "ddim_timesteps_trailing", floor_only)
    _expect_fail(pins.test_trailing_timesteps_any_count)


def test_sinusoid_sin_cos_swapped_is_caught(monkeypatch):
    def swapped(positions, d):
        p = np.asarray(positions, dtype=np.float64).reshape(-1, 1)
        w = np.power(10000.0, -2.0 * np.arange(d // 2, dtype=np.float64) / d)
        out = np.empty((p.shape[0], d))
        out[:, 0::2] = np.cos(p * w)
        out[:, 1::2] = np.sin(p * w)
        return out
    monkeypatch.setattr(ko, "sinusoid", swapped)
    _expect_fail(pins.test_sinusoid_closed_forms)


def test_timestep_mlp_without_silu_is_caught(monkeypatch):
    def no_silu(net, t):
        e = ko.sinusoid([t], net["t_W1"].shape[1])[0]
        return ko.linear(ko.linear(e, net["t_W1"], net["t_b1"]), net["t_W2"], net["t_b2"])
    monkeypatch.setattr(ko, "timestep_mlp", no_silu)
    _expect_fail(pins.test_denoiser_forward_vs_torch_modules, "root")


def test_condition_without_timestep_is_caught(monkeypatch):
    monkeypatch.setattr(ko, "condition_vector",
                        lambda net, emb, t: ko.linear(np.asarray(emb, np.float64), net["txt_W"], net["txt_b"]))
    _expect_fail(pins.test_denoiser_forward_vs_torch_modules, "body")


def test_condition_key_masked_out_is_caught(monkeypatch):
    real = ko.attention

    def skip_condition_key(q, k, v, n):
        return real(q, k[1:], v[1:], n - 1) if n > 1 else real(q, k, v, n)
    monkeypatch.setattr(ko, "attention", skip_condition_key)
    _expect_fail(pins.test_attention_brute_force, 5, 5)
