"""Seeded synthetic inputs for the two-stage DDIM denoiser.

This module is shared by the CPU oracle, the CUDA path's tests and the benchmark.
It only draws numbers: it holds none of the denoiser's arithmetic.  Every tensor
is drawn once on the host and handed, unchanged, to both implementations (the
parity method of the kimodo.cpp write-up, "kimodo.cpp가 원본과의 일치를 확인하는
방법": stored noise is fed to both sides rather than regenerated from a seed).

Recipe (shapes follow the "Kimodo WebGPU" page, "What it does" and "Model
details": a 4096-float text embedding, 30 fps clips, SOMA30 features):

* weights   seed 1: every Linear weight and bias ~ N(0, 0.02); LayerNorm
  gamma = 1 + N(0, 0.02), beta = N(0, 0.02).
* text_emb  seed 2: N(0, 1), float32 [B, 4096], distinct per prompt.
* null_emb: zeros (the unconditional branch).
* noise     seed 3: N(0, 1), float32 [B, T, 279].
* lengths   seed 4: integers uniform in [lo, hi].
* garbage   seed 5: padded frames of the noise filled with U(-1e3, 1e3)
  (or NaN for the stretch test of the key mask).
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

SEED_WEIGHTS = 1
SEED_TEXT = 2
SEED_NOISE = 3
SEED_LENGTHS = 4
SEED_GARBAGE = 5

ROOT_FEATS = 5      # (x, z, sin heading, cos heading, height)
BODY_FEATS = 274    # 30 joints x (3 position + 6D rotation) + 4 foot contacts
MOTION_FEATS = ROOT_FEATS + BODY_FEATS


@dataclass(frozen=True)
class Dims:
    """Sizes of one denoiser pair.  Defaults are the Kimodo SOMA-RP model."""
    d_model: int = 1024
    n_heads: int = 8
    d_ff: int = 2048
    n_layers: int = 16
    d_text: int = 4096
    root_in: int = ROOT_FEATS
    root_out: int = ROOT_FEATS
    body_in: int = BODY_FEATS + ROOT_FEATS
    body_out: int = BODY_FEATS


def blob_layout(dims: Dims = Dims()):
    """Canonical order of the flat float32 weight blob, as (name, shape, kind).

    kind is 'w' (Linear weight or bias) or 'ln_g' / 'ln_b' (LayerNorm affine).
    Matrices are row-major [out, in].  Root network first, then body.
    """
    d, f, dt = dims.d_model, dims.d_ff, dims.d_text
    out = []
    for net, din, dout in (("root", dims.root_in, dims.root_out),
                           ("body", dims.body_in, dims.body_out)):
        out += [(f"{net}.txt.W", (d, dt), "w"), (f"{net}.txt.b", (d,), "w"),
                (f"{net}.tmlp.W1", (d, d), "w"), (f"{net}.tmlp.b1", (d,), "w"),
                (f"{net}.tmlp.W2", (d, d), "w"), (f"{net}.tmlp.b2", (d,), "w"),
                (f"{net}.in.W", (d, din), "w"), (f"{net}.in.b", (d,), "w")]
        for l in range(dims.n_layers):
            p = f"{net}.l{l}."
            out += [(p + "qkv.W", (3 * d, d), "w"), (p + "qkv.b", (3 * d,), "w"),
                    (p + "o.W", (d, d), "w"), (p + "o.b", (d,), "w"),
                    (p + "ln1.g", (d,), "ln_g"), (p + "ln1.b", (d,), "ln_b"),
                    (p + "ff1.W", (f, d), "w"), (p + "ff1.b", (f,), "w"),
                    (p + "ff2.W", (d, f), "w"), (p + "ff2.b", (d,), "w"),
                    (p + "ln2.g", (d,), "ln_g"), (p + "ln2.b", (d,), "ln_b")]
        out += [(f"{net}.out.W", (dout, d), "w"), (f"{net}.out.b", (dout,), "w")]
    return out


def blob_size(dims: Dims = Dims()) -> int:
    return int(sum(int(np.prod(s)) for _, s, _ in blob_layout(dims)))


def weight_blob(dims: Dims = Dims(), seed: int = SEED_WEIGHTS, std: float = 0.02,
                ln_identity: bool = False) -> np.ndarray:
    """Random-init weight blob (float32, 1-D).  ln_identity sets gamma=1, beta=0."""
    rng = np.random.default_rng(seed)
    blob = rng.standard_normal(blob_size(dims), dtype=np.float32)
    blob *= np.float32(std)
    off = 0
    for _, shape, kind in blob_layout(dims):
        n = int(np.prod(shape))
        if kind == "ln_g":
            if ln_identity:
                blob[off:off + n] = 1.0
            else:
                blob[off:off + n] += np.float32(1.0)
        elif kind == "ln_b" and ln_identity:
            blob[off:off + n] = 0.0
        off += n
    return blob


def text_embeddings(batch: int, d_text: int = 4096, seed: int = SEED_TEXT) -> np.ndarray:
    rng = np.random.default_rng(seed)
    return rng.standard_normal((batch, d_text), dtype=np.float32)


def null_embeddings(batch: int, d_text: int = 4096) -> np.ndarray:
    return np.zeros((batch, d_text), dtype=np.float32)


def noise(batch: int, frames: int, feats: int = MOTION_FEATS, seed: int = SEED_NOISE) -> np.ndarray:
    rng = np.random.default_rng(seed)
    return rng.standard_normal((batch, frames, feats), dtype=np.float32)


def lengths_uniform(batch: int, lo: int, hi: int, seed: int = SEED_LENGTHS) -> np.ndarray:
    rng = np.random.default_rng(seed)
    return rng.integers(lo, hi + 1, size=batch).astype(np.int32)


def fill_padding(x: np.ndarray, lengths, seed: int = SEED_GARBAGE, lo: float = -1e3,
                 hi: float = 1e3, nan: bool = False) -> np.ndarray:
    """Copy of x [B, T, F] whose frames at index >= lengths[b] hold garbage."""
    x = np.array(x, dtype=np.float32, copy=True)
    rng = np.random.default_rng(seed)
    for b, n in enumerate(np.asarray(lengths).tolist()):
        tail = x[b, n:]
        if tail.size == 0:
            continue
        if nan:
            tail[...] = np.nan
        else:
            tail[...] = rng.uniform(lo, hi, size=tail.shape).astype(np.float32)
    return x


def random_vectors(shape, seed: int, scale: float = 1.0) -> np.ndarray:
    """Generic N(0, scale^2) float32 tensor, for kernel-level tests."""
    rng = np.random.default_rng(seed)
    return (rng.standard_normal(shape, dtype=np.float32) * np.float32(scale))
