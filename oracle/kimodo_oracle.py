"""Plain CPU oracle of the Kimodo two-stage DDIM denoiser.

TEST INFRASTRUCTURE.  Only the test suite, the package's smoke check and the
benchmark's CPU-baseline leg may import this module.  The library's product path
never calls it and shares no code with it (no kernels, helpers, tables or
constants).

Arithmetic: numpy float64 throughout, one sequence at a time, cond and uncond
as separate forward chains (four transformer forwards per DDIM step, as the
"Kimodo WebGPU" page counts them in "What it does").  Matrix products use
numpy's matmul as a library primitive; nothing is blocked, fused or reordered.

Sources (page titles and sections):

* "Kimodo WebGPU", "Model details" table: two 16-layer post-norm
  TransformerEncoder sub-networks, 8 heads x 128, GELU, 1024 hidden, 2048 FFN;
  DDIM, 50-100 steps; classifier-free guidance w=2.0; 282M parameters.
* "Kimodo WebGPU", "Architecture" figure: per DDIM step the root model runs,
  then globalRootToLocalRoot, then the body model, then CFG guidance, then
  the DDIM update; the server supplies one 4096-float text embedding.
* "Kimodo WebGPU", "WGSL compute shaders" table: linear + bias, multi-head
  self-attention with optional key masking, LayerNorm, GELU, SiLU timestep
  MLP, fused QKV projection split into Q/K/V, residual add / scale-add.
* "kimodo.cpp 소개" (discuss.pytorch.kr), parity section: stage boundaries
  root-model I/O, global->local root, body-model I/O, CFG prediction,
  DDIM x(t-1), full diffusion state.

Readings where the pages are silent (each is listed with its reason in the
design notes of the repository):

* x0-prediction: both networks predict the clean sample.
* Linear beta schedule 1e-4..0.02 over 1000 steps (the "Model details" table
  says "cosine"; the workloads fix linear); the cosine schedule is the option
  of Nichol & Dhariwal (2021).  Trailing timesteps
  t_k = 999 - k*(1000/steps) when steps divides 1000, in general
  t_k = floor(1000 (steps - k) / steps + 1/2) - 1; alphabar(-1) = 1.  eta = 0
  by default; eta > 0 takes the caller's per-step standard-normal draws.
* Condition token at sequence position 0 = Linear(4096->1024)(embedding)
  + MLP(sinusoid(t)) with MLP = Linear -> SiLU -> Linear; frame j is token
  j+1.  A fixed interleaved sinusoid (sin at even, cos at odd features) is
  added to every token at its position.
* Exact erf GELU; LayerNorm eps 1e-5 with biased variance; attention scale
  1/sqrt(128); keys at frame index >= length are excluded, the condition key
  is always valid.
* globalRootToLocalRoot: heading-frame velocity, relative heading and height
  (formula at `global_root_to_local_root`).
* Unconditional branch = same networks with the null (zero) embedding.
  CFG x0 = u + w (c - u) over all 279 features.
* Padded frames of every output are written as 0.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np
from scipy.special import erf as _erf

ROOT_FEATS = 5
BODY_FEATS = 274
MOTION_FEATS = ROOT_FEATS + BODY_FEATS
LN_EPS = 1e-5
N_TRAIN_STEPS = 1000


@dataclass(frozen=True)
class Shape:
    """Model sizes.  Defaults: the Kimodo SOMA-RP denoiser pair."""
    d_model: int = 1024
    n_heads: int = 8
    d_ff: int = 2048
    n_layers: int = 16
    d_text: int = 4096
    root_in: int = ROOT_FEATS
    root_out: int = ROOT_FEATS
    body_in: int = BODY_FEATS + ROOT_FEATS
    body_out: int = BODY_FEATS


# ---------------------------------------------------------------------------
# Weights: flat blob -> named float64 arrays
# ---------------------------------------------------------------------------

def _net_param_count(shape: Shape, din: int, dout: int) -> int:
    d, f = shape.d_model, shape.d_ff
    layer = (3 * d * d + 3 * d) + (d * d + d) + 2 * d + (f * d + f) + (d * f + d) + 2 * d
    return ((d * shape.d_text + d) + 2 * (d * d + d) + (d * din + d)
            + shape.n_layers * layer + (dout * d + dout))


def param_count(shape: Shape = Shape()) -> int:
    """Parameters of the root + body pair (282M for the default shape, per the
    "Kimodo WebGPU" "Model details" table)."""
    return (_net_param_count(shape, shape.root_in, shape.root_out)
            + _net_param_count(shape, shape.body_in, shape.body_out))


def unpack_weights(blob, shape: Shape = Shape()) -> dict:
    """Split the flat blob into {'root': net, 'body': net} of float64 arrays.

    Order per network: text projection W,b; timestep MLP W1,b1,W2,b2; input
    projection W,b; per layer qkv W,b, out-proj W,b, ln1 g,b, ffn1 W,b,
    ffn2 W,b, ln2 g,b; output projection W,b.  Matrices are [out, in].
    """
    blob = np.asarray(blob)
    pos = [0]

    def take(*dims):
        n = int(np.prod(dims))
        if pos[0] + n > blob.size:
            raise ValueError("weight blob too short")
        a = blob[pos[0]:pos[0] + n].astype(np.float64).reshape(dims)
        pos[0] += n
        return a

    d, f = shape.d_model, shape.d_ff
    nets = {}
    for name, din, dout in (("root", shape.root_in, shape.root_out),
                            ("body", shape.body_in, shape.body_out)):
        net = {"txt_W": take(d, shape.d_text), "txt_b": take(d),
               "t_W1": take(d, d), "t_b1": take(d), "t_W2": take(d, d), "t_b2": take(d),
               "in_W": take(d, din), "in_b": take(d), "layers": []}
        for _ in range(shape.n_layers):
            net["layers"].append({
                "qkv_W": take(3 * d, d), "qkv_b": take(3 * d),
                "o_W": take(d, d), "o_b": take(d),
                "ln1_g": take(d), "ln1_b": take(d),
                "ff1_W": take(f, d), "ff1_b": take(f),
                "ff2_W": take(d, f), "ff2_b": take(d),
                "ln2_g": take(d), "ln2_b": take(d)})
        net["out_W"] = take(dout, d)
        net["out_b"] = take(dout)
        nets[name] = net
    if pos[0] != blob.size:
        raise ValueError(f"weight blob has {blob.size} floats, layout needs {pos[0]}")
    nets["shape"] = shape
    return nets


# ---------------------------------------------------------------------------
# Elementary operations ("WGSL compute shaders" table of the WebGPU page)
# ---------------------------------------------------------------------------

def sinusoid(positions, d: int) -> np.ndarray:
    """Fixed sinusoidal embedding [n, d]: feature 2i = sin(p w_i), 2i+1 = cos(p w_i),
    w_i = 10000^(-2i/d).  Used for the timestep and for token positions."""
    p = np.asarray(positions, dtype=np.float64).reshape(-1, 1)
    i = np.arange(d // 2, dtype=np.float64)
    w = np.power(10000.0, -2.0 * i / d)
    out = np.empty((p.shape[0], d), dtype=np.float64)
    out[:, 0::2] = np.sin(p * w)
    out[:, 1::2] = np.cos(p * w)
    return out


def linear(x, W, b):
    """Linear + bias: y = x W^T + b."""
    return x @ W.T + b


def gelu(x):
    """Exact GELU: x * Phi(x) = 0.5 x (1 + erf(x / sqrt 2))."""
    return 0.5 * x * (1.0 + _erf(x / math.sqrt(2.0)))


def silu(x):
    """SiLU: x * sigmoid(x)."""
    return x / (1.0 + np.exp(-x))


def layer_norm(x, g, b, eps: float = LN_EPS):
    """Per-row LayerNorm with biased variance (two-pass mean, then variance)."""
    mu = x.mean(axis=-1, keepdims=True)
    xc = x - mu
    var = (xc * xc).mean(axis=-1, keepdims=True)
    return xc / np.sqrt(var + eps) * g + b


def softmax_rows(s):
    m = s.max(axis=-1, keepdims=True)
    e = np.exp(s - m)
    return e / e.sum(axis=-1, keepdims=True)


def attention(q, k, v, n_valid: int):
    """Single-head attention softmax(q k^T / sqrt(dh)) v over keys 0..n_valid-1.

    Keys at index >= n_valid are excluded outright (sliced away), so their
    content, even NaN, cannot reach any output.
    """
    dh = q.shape[-1]
    s = (q @ k[:n_valid].T) / math.sqrt(dh)
    return softmax_rows(s) @ v[:n_valid]


def multi_head_attention(h, qkv_W, qkv_b, o_W, o_b, n_heads: int, n_valid: int):
    """Fused QKV projection, split into Q/K/V (rows Q, K, V of the weight), per-head
    masked attention on contiguous head slices, concat, output projection."""
    d = h.shape[-1]
    dh = d // n_heads
    qkv = linear(h, qkv_W, qkv_b)
    q, k, v = qkv[:, :d], qkv[:, d:2 * d], qkv[:, 2 * d:]
    heads = [attention(q[:, i * dh:(i + 1) * dh], k[:, i * dh:(i + 1) * dh],
                       v[:, i * dh:(i + 1) * dh], n_valid) for i in range(n_heads)]
    return linear(np.concatenate(heads, axis=-1), o_W, o_b)


def encoder_layer(h, lp, n_heads: int, n_valid: int):
    """Post-norm encoder layer: h = LN1(h + MHA(h)); h = LN2(h + FFN(h))."""
    a = multi_head_attention(h, lp["qkv_W"], lp["qkv_b"], lp["o_W"], lp["o_b"], n_heads, n_valid)
    h = layer_norm(h + a, lp["ln1_g"], lp["ln1_b"])
    f = linear(gelu(linear(h, lp["ff1_W"], lp["ff1_b"])), lp["ff2_W"], lp["ff2_b"])
    return layer_norm(h + f, lp["ln2_g"], lp["ln2_b"])


# ---------------------------------------------------------------------------
# One denoiser network (root or body)
# ---------------------------------------------------------------------------

def timestep_mlp(net, t):
    """SiLU timestep MLP: Linear(1024->1024) -> SiLU -> Linear(1024->1024) of sinusoid(t)."""
    e = sinusoid([t], net["t_W1"].shape[1])[0]
    return linear(silu(linear(e, net["t_W1"], net["t_b1"])), net["t_W2"], net["t_b2"])


def condition_vector(net, emb, t):
    """Text projection of the 4096-float embedding plus the timestep MLP."""
    return linear(np.asarray(emb, dtype=np.float64), net["txt_W"], net["txt_b"]) + timestep_mlp(net, t)


def denoiser_forward(net, feats, emb, t, length: int, n_heads: int = 8):
    """One sub-network forward on one sequence.

    feats [T, Din] (frames), emb [4096], integer timestep t, valid frames
    length (1 <= length <= T).  Returns [T, Dout]; frames >= length are 0.
    """
    feats = np.asarray(feats, dtype=np.float64)
    T = feats.shape[0]
    d = net["in_W"].shape[0]
    pe = sinusoid(np.arange(T + 1), d)
    h = np.empty((T + 1, d), dtype=np.float64)
    h[0] = condition_vector(net, emb, t) + pe[0]
    h[1:] = linear(feats, net["in_W"], net["in_b"]) + pe[1:]
    n_valid = 1 + int(length)
    for lp in net["layers"]:
        h = encoder_layer(h, lp, n_heads, n_valid)
    out = linear(h[1:], net["out_W"], net["out_b"])
    out[int(length):] = 0.0
    return out


# ---------------------------------------------------------------------------
# globalRootToLocalRoot ("Kimodo WebGPU", "Architecture" figure, by name)
# ---------------------------------------------------------------------------

def global_root_to_local_root(root, length: int):
    """Global root [T, 5] = (x, z, sin th, cos th, y) -> local root [T, 5].

    For frame i < length, with the heading normalised, (c, s) = (cos, sin) /
    max(|(cos, sin)|, 1e-8), and the frame before the first taken as position
    (0, 0) with heading (c, s) = (1, 0):
      v = p_i - p_{i-1}                    (x, z displacement)
      v' = R_y(-th_i) v:  vx' = c vx - s vz,  vz' = s vx + c vz
      relative heading:   cos d = c_i c_{i-1} + s_i s_{i-1},
                          sin d = s_i c_{i-1} - c_i s_{i-1}
      local = (vx', vz', sin d, cos d, y_i)
    Frames >= length are 0.
    """
    root = np.asarray(root, dtype=np.float64)
    out = np.zeros_like(root)
    px, pz, cp, sp = 0.0, 0.0, 1.0, 0.0
    for i in range(int(length)):
        x, z, sr, cr, y = root[i]
        n = max(math.hypot(cr, sr), 1e-8)
        c, s = cr / n, sr / n
        vx, vz = x - px, z - pz
        out[i] = (c * vx - s * vz, s * vx + c * vz,
                  s * cp - c * sp, c * cp + s * sp, y)
        px, pz, cp, sp = x, z, c, s
    return out


def local_root_to_global_root(local, length: int):
    """Inverse of `global_root_to_local_root` (cumulative heading and position)."""
    local = np.asarray(local, dtype=np.float64)
    out = np.zeros_like(local)
    px, pz, cp, sp = 0.0, 0.0, 1.0, 0.0
    for i in range(int(length)):
        vxl, vzl, sd, cd, y = local[i]
        c = cp * cd - sp * sd
        s = sp * cd + cp * sd
        vx = c * vxl + s * vzl
        vz = -s * vxl + c * vzl
        px, pz = px + vx, pz + vz
        out[i] = (px, pz, s, c, y)
        cp, sp = c, s
    return out


# ---------------------------------------------------------------------------
# Diffusion schedule, CFG and the DDIM update
# ---------------------------------------------------------------------------

def alphabar_linear(n: int = N_TRAIN_STEPS, beta_start: float = 1e-4, beta_end: float = 0.02):
    """alphabar_t = prod_{s<=t} (1 - beta_s) with beta linearly spaced (float64)."""
    betas = np.linspace(beta_start, beta_end, n, dtype=np.float64)
    return np.cumprod(1.0 - betas)


def ddim_timesteps(steps: int, n: int = N_TRAIN_STEPS):
    """Trailing DDIM timesteps [(t_k, t_prev_k)], t_k = n-1 - k*(n/steps)."""
    if steps < 1 or n % steps:
        raise ValueError("steps must divide the training step count")
    stride = n // steps
    return [(n - 1 - k * stride, n - 1 - (k + 1) * stride) for k in range(steps)]


def alphabar_cosine(n: int = N_TRAIN_STEPS, s: float = 0.008, max_beta: float = 0.999):
    """Cosine schedule (Nichol & Dhariwal, "Improved Denoising Diffusion Probabilistic
    Models", 2021, eq. 17): alphabar(u) = f(u) / f(0), f(u) = cos^2((u + s) / (1 + s) * pi/2)
    for u in [0, 1].  Discretised as in that paper: beta_i = min(1 - alphabar((i+1)/n) /
    alphabar(i/n), max_beta), and the table is prod_{j<=i} (1 - beta_j) (float64)."""
    def f(u):
        return math.cos((u + s) / (1.0 + s) * math.pi / 2.0) ** 2
    betas = np.array([min(1.0 - f((i + 1) / n) / f(i / n), max_beta) for i in range(n)], dtype=np.float64)
    return np.cumprod(1.0 - betas)


def ddim_timesteps_trailing(steps: int, n: int = N_TRAIN_STEPS):
    """Trailing DDIM timesteps for any step count 1 <= steps <= n:
    t_k = floor(n (steps - k) / steps + 1/2) - 1, t_prev_k = t_{k+1}, and -1 after the last.
    Equal to ddim_timesteps when steps divides n."""
    if steps < 1 or steps > n:
        raise ValueError("steps must lie in [1, n]")
    ts = [(2 * n * (steps - k) + steps) // (2 * steps) - 1 for k in range(steps)]
    return [(ts[k], ts[k + 1] if k + 1 < steps else -1) for k in range(steps)]


def alphabar_at(ab, t: int) -> float:
    return 1.0 if t < 0 else float(ab[t])


def cfg_combine(x_cond, x_uncond, w: float):
    """Classifier-free guidance: u + w (c - u)."""
    return x_uncond + w * (x_cond - x_uncond)


def ddim_update(x_t, x0, ab_t: float, ab_prev: float):
    """Deterministic (eta = 0) DDIM step from an x0 prediction:
    eps = (x_t - sqrt(ab_t) x0) / sqrt(1 - ab_t);
    x_prev = sqrt(ab_prev) x0 + sqrt(1 - ab_prev) eps."""
    eps = (x_t - math.sqrt(ab_t) * x0) / math.sqrt(1.0 - ab_t)
    return math.sqrt(ab_prev) * x0 + math.sqrt(1.0 - ab_prev) * eps


def ddim_sigma(ab_t: float, ab_prev: float, eta: float) -> float:
    """Per-step noise scale of DDIM (Song, Meng & Ermon, "Denoising Diffusion Implicit
    Models", 2021, eq. 16): sigma = eta sqrt((1 - ab_prev) / (1 - ab_t)) sqrt(1 - ab_t / ab_prev)."""
    return eta * math.sqrt((1.0 - ab_prev) / (1.0 - ab_t)) * math.sqrt(1.0 - ab_t / ab_prev)


def ddim_update_eta(x_t, x0, ab_t: float, ab_prev: float, eta: float, z):
    """Generalised DDIM step from an x0 prediction (same paper, eq. 12):
    eps = (x_t - sqrt(ab_t) x0) / sqrt(1 - ab_t);
    x_prev = sqrt(ab_prev) x0 + sqrt(1 - ab_prev - sigma^2) eps + sigma z,
    with sigma from ddim_sigma and z the caller's standard-normal draw for this step."""
    sigma = ddim_sigma(ab_t, ab_prev, eta)
    eps = (x_t - math.sqrt(ab_t) * x0) / math.sqrt(1.0 - ab_t)
    out = math.sqrt(ab_prev) * x0 + math.sqrt(1.0 - ab_prev - sigma * sigma) * eps
    if sigma != 0.0:
        out = out + sigma * np.asarray(z, dtype=np.float64)
    return out


# ---------------------------------------------------------------------------
# Two-stage step and the sampling loop
# ---------------------------------------------------------------------------

def two_stage_predict(params, x_t, emb, t: int, length: int):
    """One guidance branch: root net -> globalRootToLocalRoot -> body net.

    x_t [T, 279] = [root 5 | body 274].  The body net reads [body 274 of x_t |
    local root 5].  Returns the stage outputs and x0 = [root 5 | body 274].
    """
    n_heads = params["shape"].n_heads
    x_t = np.asarray(x_t, dtype=np.float64)
    root = denoiser_forward(params["root"], x_t[:, :ROOT_FEATS], emb, t, length, n_heads)
    local = global_root_to_local_root(root, length)
    body_in = np.concatenate([x_t[:, ROOT_FEATS:], local], axis=1)
    body = denoiser_forward(params["body"], body_in, emb, t, length, n_heads)
    return {"root_out": root, "local_root": local, "body_in": body_in, "body_out": body,
            "x0": np.concatenate([root, body], axis=1)}


def ddim_step(params, x_t, text_emb, null_emb, length: int, t: int, t_prev: int,
              cfg_scale: float, ab=None, predictor=None, eta: float = 0.0, z=None):
    """One two-stage DDIM step on one sequence.  Returns (x_prev, stages).

    predictor, if given, replaces the networks: predictor(x_t, t) -> (x0_cond,
    x0_uncond).  It serves the closed-form checks of the sampler.  eta > 0 adds
    sigma z with the caller's draw z [T, 279] (ddim_update_eta).
    """
    ab = alphabar_linear() if ab is None else ab
    x_t = np.asarray(x_t, dtype=np.float64)
    if predictor is None:
        cond = two_stage_predict(params, x_t, text_emb, t, length)
        unc = two_stage_predict(params, x_t, null_emb, t, length)
        xc, xu = cond["x0"], unc["x0"]
    else:
        cond = unc = None
        xc, xu = (np.asarray(a, dtype=np.float64) for a in predictor(x_t, t))
    x0 = cfg_combine(xc, xu, cfg_scale)
    if eta == 0.0:
        x_prev = ddim_update(x_t, x0, alphabar_at(ab, t), alphabar_at(ab, t_prev))
    else:
        x_prev = ddim_update_eta(x_t, x0, alphabar_at(ab, t), alphabar_at(ab, t_prev), eta, z)
    x_prev[int(length):] = 0.0
    return x_prev, {"cond": cond, "uncond": unc, "x0": x0}


def ddim_sample(params, text_emb, null_emb, noise, length: int, steps: int,
                cfg_scale: float, predictor=None, trace=None, schedule: str = "linear",
                eta: float = 0.0, step_noise=None):
    """Full DDIM loop on one sequence from noise [T, 279]; returns the final x.
    schedule "linear" or "cosine"; any step count in [1, 1000] (trailing spacing);
    eta > 0 draws step k's z from step_noise[k] [T, 279]."""
    ab = alphabar_linear() if schedule == "linear" else alphabar_cosine()
    x = np.asarray(noise, dtype=np.float64)
    for k, (t, t_prev) in enumerate(ddim_timesteps_trailing(steps)):
        z = None if eta == 0.0 else step_noise[k]
        x, _ = ddim_step(params, x, text_emb, null_emb, length, t, t_prev, cfg_scale, ab, predictor, eta, z)
        if trace is not None:
            trace.append(x.copy())
    return x


def ddim_sample_batch(params, text_emb, null_emb, noise, lengths, steps: int, cfg_scale: float,
                      indices=None, schedule: str = "linear", eta: float = 0.0, step_noise=None):
    """Batch of independent sequences (null_emb [4096] or [B, 4096]).  Returns
    {b: x_b} for the requested sequence indices (default: all).  step_noise, when
    eta > 0, is [steps, B, T, 279]."""
    text_emb = np.asarray(text_emb)
    null_emb = np.asarray(null_emb)
    idx = range(text_emb.shape[0]) if indices is None else indices
    res = {}
    for b in idx:
        ne = null_emb if null_emb.ndim == 1 else null_emb[b]
        sn = None if step_noise is None else np.asarray(step_noise)[:, b]
        res[b] = ddim_sample(params, text_emb[b], ne, noise[b], int(lengths[b]), steps, cfg_scale,
                             schedule=schedule, eta=eta, step_noise=sn)
    return res
