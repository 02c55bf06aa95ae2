"""The CPU oracle pinned to facts outside itself (no GPU needed).

Each test checks the oracle against something it does not compute itself: the
sizes the pages print, closed forms, exact rational arithmetic, brute force on
tiny inputs, or a PyTorch library routine run in float64.
"""
import math
from fractions import Fraction

import numpy as np
import pytest
import torch

import synth
from oracle import kimodo_oracle as ko
from oracle_helpers import TINY, read_golden, tiny_params, tiny_shapes

torch.set_default_dtype(torch.float64)


# --------------------------------------------------------------------------- sizes

def test_param_count_matches_printed_model_size():
    g = read_golden("model_size.txt")
    n = ko.param_count()
    assert n == 281_963_799
    assert round(n / 1e6) == g["params_millions"]
    # fp16 flat file: 540 MB on the page (MiB reading), fp32 checkpoint 1.13 GB.
    assert abs(2 * n / 2**20 - g["fp16_flat_MB"]) / g["fp16_flat_MB"] < 0.01
    assert abs(4 * n / 1e9 - g["fp32_checkpoint_GB"]) / g["fp32_checkpoint_GB"] < 0.005
    s = ko.Shape()
    assert s.n_layers == g["layers_per_net"] and s.n_heads == g["heads"]
    assert s.d_model == g["hidden"] == g["heads"] * g["head_dim"] and s.d_ff == g["ffn"]
    assert s.d_text == g["text_embedding_floats"]


def test_param_count_sensitive_to_each_size():
    # a dropped bias, a wrong FFN width or a missing timestep layer moves the
    # count off 282M by more than the page's rounding.
    base = ko.param_count()
    for kw in (dict(d_ff=4096), dict(n_layers=15), dict(d_model=1024 + 64)):
        assert round(ko.param_count(ko.Shape(**kw)) / 1e6) != 282 or kw == {}
    assert base == synth.blob_size()


def test_blob_layouts_agree():
    for dims, shape in [(synth.Dims(), ko.Shape()), tiny_shapes()]:
        assert synth.blob_size(dims) == ko.param_count(shape)
    dims, shape = tiny_shapes()
    blob = synth.weight_blob(dims, seed=3)
    p = ko.unpack_weights(blob, shape)
    assert p["root"]["in_W"].shape == (TINY["d_model"], 5)
    assert p["body"]["in_W"].shape == (TINY["d_model"], 279)
    assert p["body"]["out_W"].shape == (274, TINY["d_model"])
    # LayerNorm gammas were drawn around 1, every other tensor around 0
    assert abs(p["root"]["layers"][0]["ln1_g"].mean() - 1.0) < 0.05
    assert abs(p["root"]["layers"][0]["ln1_b"].mean()) < 0.05
    with pytest.raises(ValueError):
        ko.unpack_weights(blob[:-1], shape)


# --------------------------------------------------------------------------- sinusoid

def test_sinusoid_closed_forms():
    d = 64
    pe = ko.sinusoid(np.arange(50), d)
    np.testing.assert_array_equal(pe[0, 0::2], 0.0)
    np.testing.assert_array_equal(pe[0, 1::2], 1.0)
    p = np.arange(50.0)
    np.testing.assert_allclose(pe[:, 0], np.sin(p), rtol=0, atol=1e-15)
    np.testing.assert_allclose(pe[:, 1], np.cos(p), rtol=0, atol=1e-15)
    np.testing.assert_allclose(pe[:, d - 2], np.sin(p * 10000.0 ** (-(d - 2) / d)), atol=1e-15)
    np.testing.assert_allclose(pe[:, 0::2] ** 2 + pe[:, 1::2] ** 2, 1.0, atol=1e-14)
    # shift invariance: <PE(p), PE(q)> = sum_i cos((p - q) w_i)
    g = pe @ pe.T
    for k in range(1, 10):
        np.testing.assert_allclose(np.diag(g, k), np.diag(g, k)[0], atol=1e-12)


def test_sinusoid_equals_complex_exponential():
    d = 16
    w = np.array([10000.0 ** (-2 * i / d) for i in range(d // 2)])
    z = np.exp(1j * np.outer(np.arange(7.0), w))
    pe = ko.sinusoid(np.arange(7), d)
    np.testing.assert_allclose(pe[:, 0::2], z.imag, atol=1e-15)
    np.testing.assert_allclose(pe[:, 1::2], z.real, atol=1e-15)


# --------------------------------------------------------------------------- elementwise

def test_layer_norm_identity_affine_closed_form():
    rng = np.random.default_rng(0)
    x = rng.normal(3.0, 2.0, size=(6, 1024))
    y = ko.layer_norm(x, np.ones(1024), np.zeros(1024))
    np.testing.assert_allclose(y.mean(axis=1), 0.0, atol=1e-12)
    var = x.var(axis=1)
    np.testing.assert_allclose(y.var(axis=1), var / (var + 1e-5), rtol=1e-12)
    np.testing.assert_allclose(y.var(axis=1), 1.0, atol=1e-5)


def test_layer_norm_vs_torch():
    rng = np.random.default_rng(1)
    x, g, b = rng.normal(size=(5, 1024)), rng.normal(size=1024), rng.normal(size=1024)
    ref = torch.nn.functional.layer_norm(torch.tensor(x), (1024,), torch.tensor(g),
                                         torch.tensor(b), eps=1e-5).numpy()
    np.testing.assert_allclose(ko.layer_norm(x, g, b), ref, rtol=1e-12, atol=1e-12)


def test_gelu_exact_erf():
    x = np.linspace(-8, 8, 1001)
    ref = torch.nn.functional.gelu(torch.tensor(x), approximate="none").numpy()
    np.testing.assert_allclose(ko.gelu(x), ref, rtol=1e-14, atol=1e-15)
    np.testing.assert_allclose(ko.gelu(x) - ko.gelu(-x), x, atol=1e-14)
    assert ko.gelu(np.array(0.0)) == 0.0
    assert abs(ko.gelu(np.array(1.0)) - 0.8413447460685429) < 1e-15   # Phi(1)
    # the tanh form differs by far more than the fp32 tolerance
    tanh_form = 0.5 * x * (1 + np.tanh(math.sqrt(2 / math.pi) * (x + 0.044715 * x ** 3)))
    assert np.abs(tanh_form - ko.gelu(x)).max() > 1e-4


def test_silu():
    x = np.linspace(-30, 30, 601)
    ref = torch.nn.functional.silu(torch.tensor(x)).numpy()
    np.testing.assert_allclose(ko.silu(x), ref, rtol=1e-14, atol=1e-300)


# --------------------------------------------------------------------------- attention

def _brute_attention(q, k, v, n_valid):
    S, dh = len(q), len(q[0])
    out = []
    for i in range(S):
        s = [sum(q[i][c] * k[j][c] for c in range(dh)) / math.sqrt(dh) for j in range(n_valid)]
        m = max(s)
        e = [math.exp(a - m) for a in s]
        z = sum(e)
        out.append([sum(e[j] / z * v[j][c] for j in range(n_valid)) for c in range(dh)])
    return np.array(out)


@pytest.mark.parametrize("S,n_valid", [(1, 1), (5, 5), (8, 3), (7, 1)])
def test_attention_brute_force(S, n_valid):
    rng = np.random.default_rng(S * 10 + n_valid)
    q, k, v = (rng.normal(size=(S, 4)) for _ in range(3))
    ref = _brute_attention(q.tolist(), k.tolist(), v.tolist(), n_valid)
    np.testing.assert_allclose(ko.attention(q, k, v, n_valid), ref, rtol=1e-13, atol=1e-14)


def test_attention_only_condition_key():
    rng = np.random.default_rng(2)
    q, k, v = (rng.normal(size=(9, 128)) for _ in range(3))
    out = ko.attention(q, k, v, 1)
    np.testing.assert_allclose(out, np.broadcast_to(v[0], out.shape), atol=1e-15)


def test_attention_identical_keys_average_values():
    rng = np.random.default_rng(3)
    q, v = rng.normal(size=(6, 128)), rng.normal(size=(6, 128))
    k = np.broadcast_to(rng.normal(size=128), (6, 128))
    out = ko.attention(q, k, v, 4)
    np.testing.assert_allclose(out, np.broadcast_to(v[:4].mean(0), out.shape), atol=1e-14)


def test_attention_vs_torch_sdpa_with_key_mask():
    rng = np.random.default_rng(4)
    S, n_valid = 40, 23
    q, k, v = (rng.normal(size=(S, 128)) for _ in range(3))
    mask = torch.zeros(S, S, dtype=torch.bool)
    mask[:, :n_valid] = True
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.tensor(q)[None], torch.tensor(k)[None], torch.tensor(v)[None], attn_mask=mask)[0]
    np.testing.assert_allclose(ko.attention(q, k, v, n_valid), ref.numpy(), rtol=1e-12, atol=1e-13)


def test_attention_ignores_nan_in_masked_keys():
    rng = np.random.default_rng(5)
    q, k, v = (rng.normal(size=(6, 8)) for _ in range(3))
    ref = ko.attention(q, k, v, 3)
    k[3:] = np.nan
    v[3:] = np.nan
    np.testing.assert_array_equal(ko.attention(q, k, v, 3), ref)


# --------------------------------------------------------------------------- encoder layer

def _torch_layer(lp, d, h, f):
    layer = torch.nn.TransformerEncoderLayer(d, h, f, dropout=0.0, activation="gelu",
                                             batch_first=True, norm_first=False, layer_norm_eps=1e-5)
    sd = {"self_attn.in_proj_weight": lp["qkv_W"], "self_attn.in_proj_bias": lp["qkv_b"],
          "self_attn.out_proj.weight": lp["o_W"], "self_attn.out_proj.bias": lp["o_b"],
          "linear1.weight": lp["ff1_W"], "linear1.bias": lp["ff1_b"],
          "linear2.weight": lp["ff2_W"], "linear2.bias": lp["ff2_b"],
          "norm1.weight": lp["ln1_g"], "norm1.bias": lp["ln1_b"],
          "norm2.weight": lp["ln2_g"], "norm2.bias": lp["ln2_b"]}
    layer.load_state_dict({k: torch.tensor(v) for k, v in sd.items()})
    layer.train()   # dropout is 0; train mode keeps the reference (non-fused) path
    return layer


@pytest.mark.parametrize("d,h,f,S,n_valid", [(32, 4, 64, 11, 7), (1024, 8, 2048, 20, 13)])
def test_encoder_layer_vs_torch(d, h, f, S, n_valid):
    rng = np.random.default_rng(d + S)
    lp = {"qkv_W": rng.normal(0, 0.05, (3 * d, d)), "qkv_b": rng.normal(0, 0.05, 3 * d),
          "o_W": rng.normal(0, 0.05, (d, d)), "o_b": rng.normal(0, 0.05, d),
          "ff1_W": rng.normal(0, 0.05, (f, d)), "ff1_b": rng.normal(0, 0.05, f),
          "ff2_W": rng.normal(0, 0.05, (d, f)), "ff2_b": rng.normal(0, 0.05, d),
          "ln1_g": 1 + rng.normal(0, 0.1, d), "ln1_b": rng.normal(0, 0.1, d),
          "ln2_g": 1 + rng.normal(0, 0.1, d), "ln2_b": rng.normal(0, 0.1, d)}
    x = rng.normal(size=(S, d))
    pad = torch.zeros(1, S, dtype=torch.bool)
    pad[0, n_valid:] = True
    with torch.no_grad():
        ref = _torch_layer(lp, d, h, f)(torch.tensor(x)[None], src_key_padding_mask=pad)[0].numpy()
    out = ko.encoder_layer(x, lp, h, n_valid)
    np.testing.assert_allclose(out, ref, rtol=1e-10, atol=1e-11)


# --------------------------------------------------------------------------- whole network

def _torch_network(net, shape):
    d = shape.d_model
    txt = torch.nn.Linear(shape.d_text, d)
    tmlp = torch.nn.Sequential(torch.nn.Linear(d, d), torch.nn.SiLU(), torch.nn.Linear(d, d))
    inp = torch.nn.Linear(net["in_W"].shape[1], d)
    enc = torch.nn.TransformerEncoder(
        torch.nn.TransformerEncoderLayer(d, shape.n_heads, shape.d_ff, dropout=0.0, activation="gelu",
                                         batch_first=True, norm_first=False),
        shape.n_layers, enable_nested_tensor=False)
    out = torch.nn.Linear(d, net["out_W"].shape[0])
    with torch.no_grad():
        for mod, (w, b) in ((txt, ("txt_W", "txt_b")), (tmlp[0], ("t_W1", "t_b1")),
                            (tmlp[2], ("t_W2", "t_b2")), (inp, ("in_W", "in_b")),
                            (out, ("out_W", "out_b"))):
            mod.weight.copy_(torch.tensor(net[w]))
            mod.bias.copy_(torch.tensor(net[b]))
        for layer, lp in zip(enc.layers, net["layers"]):
            layer.load_state_dict(_torch_layer(lp, d, shape.n_heads, shape.d_ff).state_dict())
    enc.train()
    return txt, tmlp, inp, enc, out


def _pe_complex(n, d):
    w = np.array([10000.0 ** (-2 * i / d) for i in range(d // 2)])
    z = np.exp(1j * np.outer(np.arange(float(n)), w))
    pe = np.empty((n, d))
    pe[:, 0::2], pe[:, 1::2] = z.imag, z.real
    return torch.tensor(pe)


@pytest.mark.parametrize("net_name", ["root", "body"])
def test_denoiser_forward_vs_torch_modules(net_name):
    params = tiny_params(seed=21)
    shape = params["shape"]
    net = params[net_name]
    T, length, t = 12, 9, 437
    rng = np.random.default_rng(7)
    feats = rng.normal(size=(T, net["in_W"].shape[1]))
    emb = rng.normal(size=shape.d_text)
    txt, tmlp, inp, enc, out = _torch_network(net, shape)
    pe = _pe_complex(max(T + 1, t + 1), shape.d_model)
    with torch.no_grad():
        cond = txt(torch.tensor(emb)) + tmlp(pe[t]) + pe[0]
        toks = torch.cat([cond[None], inp(torch.tensor(feats)) + pe[1:T + 1]], 0)[None]
        pad = torch.zeros(1, T + 1, dtype=torch.bool)
        pad[0, 1 + length:] = True
        ref = out(enc(toks, src_key_padding_mask=pad)[0, 1:]).numpy()
    got = ko.denoiser_forward(net, feats, emb, t, length, shape.n_heads)
    np.testing.assert_allclose(got[:length], ref[:length], rtol=1e-9, atol=1e-10)
    np.testing.assert_array_equal(got[length:], 0.0)


@pytest.mark.parametrize("nan", [False, True])
def test_padded_frames_do_not_reach_valid_outputs(nan):
    params = tiny_params(seed=22)
    T, length = 10, 6
    rng = np.random.default_rng(8)
    x = rng.normal(size=(1, T, 279)).astype(np.float32)
    emb = rng.normal(size=16)
    base, _ = ko.ddim_step(params, x[0], emb, np.zeros(16), length, 999, 979, 2.0)
    xg = synth.fill_padding(x, [length], nan=nan)
    assert not np.array_equal(xg, x)
    got, st = ko.ddim_step(params, xg[0], emb, np.zeros(16), length, 999, 979, 2.0)
    np.testing.assert_array_equal(got, base)
    assert np.all(np.isfinite(st["x0"][:length]))


# --------------------------------------------------------------------------- globalRootToLocalRoot

def test_g2l_worked_example():
    # Facing +90 deg (sin 1, cos 0), stepping one unit along global +x each frame:
    # in the heading frame that is one unit along local z; no turning after frame 0.
    root = np.array([[1.0, 0.0, 1.0, 0.0, 0.9],
                     [2.0, 0.0, 1.0, 0.0, 0.8],
                     [3.0, 0.0, 1.0, 0.0, 0.7]])
    loc = ko.global_root_to_local_root(root, 3)
    # frame 0: displacement (1, 0) from the origin; turn from heading 0 to 90 deg
    np.testing.assert_allclose(loc[0], [0.0, 1.0, 1.0, 0.0, 0.9], atol=1e-15)
    np.testing.assert_allclose(loc[1], [0.0, 1.0, 0.0, 1.0, 0.8], atol=1e-15)
    np.testing.assert_allclose(loc[2], [0.0, 1.0, 0.0, 1.0, 0.7], atol=1e-15)


def _random_root(rng, T):
    th = np.cumsum(rng.normal(0, 0.3, T))
    r = rng.uniform(0.5, 2.0, T)      # unnormalised heading magnitude
    return np.stack([np.cumsum(rng.normal(size=T)), np.cumsum(rng.normal(size=T)),
                     r * np.sin(th), r * np.cos(th), rng.normal(size=T)], 1), th


def test_g2l_round_trip():
    rng = np.random.default_rng(9)
    root, th = _random_root(rng, 40)
    back = ko.local_root_to_global_root(ko.global_root_to_local_root(root, 40), 40)
    want = root.copy()
    want[:, 2], want[:, 3] = np.sin(th), np.cos(th)
    np.testing.assert_allclose(back, want, atol=1e-11)
    loc = ko.global_root_to_local_root(root, 40)
    np.testing.assert_allclose(ko.global_root_to_local_root(ko.local_root_to_global_root(loc, 40), 40),
                               loc, atol=1e-11)


def test_g2l_yaw_invariance():
    rng = np.random.default_rng(10)
    root, th = _random_root(rng, 30)
    phi = 0.7
    c, s = math.cos(phi), math.sin(phi)
    rot = root.copy()
    # R_y(phi) on (x, z) and heading th -> th + phi
    rot[:, 0] = c * root[:, 0] + s * root[:, 1]
    rot[:, 1] = -s * root[:, 0] + c * root[:, 1]
    r = np.hypot(root[:, 2], root[:, 3])
    rot[:, 2], rot[:, 3] = r * np.sin(th + phi), r * np.cos(th + phi)
    a = ko.global_root_to_local_root(root, 30)
    b = ko.global_root_to_local_root(rot, 30)
    # frame 0 is measured against the fixed origin frame; every later frame is invariant
    np.testing.assert_allclose(b[1:], a[1:], atol=1e-12)


def test_g2l_straight_walk_constant_local_velocity():
    th, speed, T = 0.4, 0.05, 25
    u = np.array([math.sin(th), math.cos(th)])        # walk along the heading
    p = np.outer(np.arange(1, T + 1), u) * speed
    root = np.stack([p[:, 0], p[:, 1], np.full(T, math.sin(th)), np.full(T, math.cos(th)),
                     np.full(T, 0.9)], 1)
    loc = ko.global_root_to_local_root(root, T)
    np.testing.assert_allclose(loc[1:, 0:2], np.broadcast_to([0.0, speed], (T - 1, 2)), atol=1e-15)
    np.testing.assert_allclose(loc[1:, 2:4], np.broadcast_to([0.0, 1.0], (T - 1, 2)), atol=1e-15)
    assert np.hypot(*loc[1, :2]) == pytest.approx(speed, rel=1e-12)


def test_g2l_padded_frames_zero():
    rng = np.random.default_rng(12)
    root, _ = _random_root(rng, 10)
    loc = ko.global_root_to_local_root(root, 6)
    np.testing.assert_array_equal(loc[6:], 0.0)


# --------------------------------------------------------------------------- schedule / DDIM / CFG

def test_alphabar_exact_rational():
    ab = ko.alphabar_linear()
    b0, b1 = Fraction(1, 10000), Fraction(2, 100)
    prod = Fraction(1)
    exact = {}
    for i in range(1000):
        prod *= 1 - (b0 + (b1 - b0) * i / 999)
        if i in (0, 9, 19, 499, 979, 999):
            exact[i] = prod
    for i, v in exact.items():
        assert abs(ab[i] - float(v)) / float(v) < 1e-12, i
    assert np.all(np.diff(ab) < 0) and ab[0] == pytest.approx(1 - 1e-4, rel=1e-15)


def test_ddim_timesteps():
    ts = ko.ddim_timesteps(50)
    assert ts[0] == (999, 979) and ts[-1] == (19, -1) and len(ts) == 50
    ts = ko.ddim_timesteps(100)
    assert ts[0] == (999, 989) and ts[-1] == (9, -1)
    assert ko.ddim_timesteps(1) == [(999, -1)]
    for bad in (0, 3, 7, 1001):
        with pytest.raises(ValueError):
            ko.ddim_timesteps(bad)


def test_cosine_schedule_telescopes():
    """prod_{j<=i} (1 - beta_j) with beta_j = 1 - f((j+1)/n) / f(j/n) telescopes to
    f((i+1)/n) / f(0) wherever no beta is clipped; only the last one is (f(1) = 0)."""
    ab = ko.alphabar_cosine()
    s = 0.008

    def f(u):
        return math.cos((u + s) / (1 + s) * math.pi / 2) ** 2
    direct = np.array([f((i + 1) / 1000) / f(0.0) for i in range(1000)])
    np.testing.assert_allclose(ab[:999], direct[:999], rtol=1e-11)
    assert ab[999] == pytest.approx(ab[998] * (1 - 0.999), rel=1e-12)
    assert np.all(np.diff(ab) < 0)
    assert ab[499] == pytest.approx(0.49384, abs=1e-4)   # f(1/2) / f(0), worked by hand


def test_trailing_timesteps_any_count():
    # floor(1000 (15 - k) / 15 + 1/2) - 1, worked by hand
    want = [999, 932, 866, 799, 732, 666, 599, 532, 466, 399, 332, 266, 199, 132, 66]
    ts = ko.ddim_timesteps_trailing(15)
    assert [t for t, _ in ts] == want and [tp for _, tp in ts] == want[1:] + [-1]
    assert ko.ddim_timesteps_trailing(16)[3][0] == 812        # 812.5 + 1/2 rounds up to 813, minus 1
    for steps in (1, 2, 4, 5, 8, 10, 20, 25, 40, 50, 100, 125, 200, 250, 500, 1000):
        assert ko.ddim_timesteps_trailing(steps) == ko.ddim_timesteps(steps)
    for steps in (3, 7, 16, 35, 999):
        ts = ko.ddim_timesteps_trailing(steps)
        t = [a for a, _ in ts]
        assert len(ts) == steps and t[0] == 999 and t[-1] >= 0
        assert all(a > b for a, b in zip(t, t[1:]))
        assert all(tp == nxt for (_, tp), nxt in zip(ts, t[1:] + [-1]))
    for bad in (0, 1001):
        with pytest.raises(ValueError):
            ko.ddim_timesteps_trailing(bad)


def test_ddim_eta_zero_is_deterministic_ddim():
    ab = ko.alphabar_linear()
    rng = np.random.default_rng(31)
    x_t, x0, z = rng.normal(size=(3, 7, 279))
    for t, tp in [(999, 932), (400, 333), (66, -1)]:
        ap = 1.0 if tp < 0 else ab[tp]
        np.testing.assert_array_equal(ko.ddim_update_eta(x_t, x0, ab[t], ap, 0.0, z),
                                      ko.ddim_update(x_t, x0, ab[t], ap))


def test_ddim_eta_one_is_the_ddpm_posterior():
    """With eta = 1 the DDIM update is the DDPM posterior q(x_prev | x_t, x0) (Ho, Jain &
    Abbeel 2020, eqs. 6-7) sampled with z, for the effective alpha = ab_t / ab_prev."""
    rng = np.random.default_rng(32)
    x_t, x0, z = rng.normal(size=(3, 5, 279))
    for ab in (ko.alphabar_linear(), ko.alphabar_cosine()):
        for t, tp in [(999, 979), (500, 433), (66, 0), (66, -1)]:
            at, ap = ab[t], (1.0 if tp < 0 else ab[tp])
            alpha = at / ap
            beta = 1 - alpha
            mean = math.sqrt(ap) * beta / (1 - at) * x0 + math.sqrt(alpha) * (1 - ap) / (1 - at) * x_t
            var = (1 - ap) / (1 - at) * beta
            got = ko.ddim_update_eta(x_t, x0, at, ap, 1.0, z)
            np.testing.assert_allclose(got, mean + math.sqrt(var) * z, rtol=0, atol=1e-11)


def test_ddim_eta_keeps_the_forward_marginal():
    """Exact x0, x_t ~ q(x_t | x0) and z ~ N(0, 1): x_prev ~ N(sqrt(ab_prev) x0, 1 - ab_prev)."""
    ab = ko.alphabar_cosine()
    rng = np.random.default_rng(33)
    n = 200_000
    x0 = 0.7
    eps, z = rng.normal(size=(2, n))
    at, ap = ab[600], ab[450]
    x_t = math.sqrt(at) * x0 + math.sqrt(1 - at) * eps
    x_prev = ko.ddim_update_eta(x_t, np.full(n, x0), at, ap, 0.6, z)
    r = x_prev - math.sqrt(ap) * x0
    assert abs(r.mean()) < 5 / math.sqrt(n)
    assert r.var() == pytest.approx(1 - ap, rel=0.02)


def test_cfg_special_cases():
    rng = np.random.default_rng(13)
    c, u = rng.normal(size=(5, 279)), rng.normal(size=(5, 279))
    np.testing.assert_allclose(ko.cfg_combine(c, u, 1.0), c, rtol=0, atol=1e-15)
    np.testing.assert_array_equal(ko.cfg_combine(c, u, 0.0), u)
    np.testing.assert_allclose(ko.cfg_combine(c, u, 2.0), 2 * c - u, atol=1e-15)


def test_ddim_step_with_exact_x0_predictor():
    ab = ko.alphabar_linear()
    rng = np.random.default_rng(14)
    x0, eps = rng.normal(size=(8, 279)), rng.normal(size=(8, 279))
    for t, tp in [(999, 979), (499, 479), (19, -1)]:
        at, ap = ab[t], (1.0 if tp < 0 else ab[tp])
        x_t = math.sqrt(at) * x0 + math.sqrt(1 - at) * eps
        got, _ = ko.ddim_step(None, x_t, None, None, 8, t, tp, 2.0, ab,
                              predictor=lambda x, tt: (x0, x0))
        np.testing.assert_allclose(got, math.sqrt(ap) * x0 + math.sqrt(1 - ap) * eps, atol=1e-12)


def test_ddim_sample_constant_predictor_closed_form():
    ab = ko.alphabar_linear()
    rng = np.random.default_rng(15)
    x0 = rng.normal(size=(6, 279))
    noise = rng.normal(size=(6, 279))
    # eps implied by the first step stays constant when eta = 0
    eps = (noise - math.sqrt(ab[999]) * x0) / math.sqrt(1 - ab[999])
    trace = []
    out = ko.ddim_sample(None, None, None, noise, 6, 50, 2.0,
                         predictor=lambda x, t: (x0, x0), trace=trace)
    for (t, tp), x in zip(ko.ddim_timesteps(50), trace):
        ap = 1.0 if tp < 0 else ab[tp]
        np.testing.assert_allclose(x, math.sqrt(ap) * x0 + math.sqrt(1 - ap) * eps, atol=1e-10)
    np.testing.assert_allclose(out, x0, atol=1e-10)


def test_cfg_scale_one_is_the_cond_branch():
    params = tiny_params(seed=23)
    rng = np.random.default_rng(16)
    x = rng.normal(size=(9, 279))
    emb = rng.normal(size=16)
    ab = ko.alphabar_linear()
    got, st = ko.ddim_step(params, x, emb, np.zeros(16), 7, 999, 979, 1.0, ab)
    cond = ko.two_stage_predict(params, x, emb, 999, 7)["x0"]
    want = ko.ddim_update(x, cond, ab[999], ab[979])
    want[7:] = 0
    np.testing.assert_allclose(got, want, atol=1e-13)
    unc = ko.two_stage_predict(params, x, np.zeros(16), 999, 7)["x0"]
    assert np.abs(cond - unc)[:7].max() > 1e-6   # the branches really differ


def test_forward_count_per_50_step_generation(monkeypatch):
    g = read_golden("model_size.txt")
    params = tiny_params(seed=24)
    calls = []
    real = ko.denoiser_forward

    def counting(*a, **k):
        calls.append(1)
        return real(*a, **k)

    monkeypatch.setattr(ko, "denoiser_forward", counting)
    rng = np.random.default_rng(17)
    ko.ddim_sample(params, rng.normal(size=16), np.zeros(16), rng.normal(size=(3, 279)), 3, 50, 2.0)
    assert len(calls) == g["forwards_per_50_step_generation"]


def test_two_stage_body_reads_local_root_of_its_own_branch():
    params = tiny_params(seed=25)
    rng = np.random.default_rng(18)
    x = rng.normal(size=(8, 279))
    st = ko.two_stage_predict(params, x, rng.normal(size=16), 500, 8)
    np.testing.assert_array_equal(st["body_in"][:, :274], x[:, 5:])
    np.testing.assert_array_equal(st["body_in"][:, 274:], ko.global_root_to_local_root(st["root_out"], 8))
    np.testing.assert_array_equal(st["x0"][:, :5], st["root_out"])
    np.testing.assert_array_equal(st["x0"][:, 5:], st["body_out"])
