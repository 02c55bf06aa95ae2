"""Programmatic dependent launch changes timing only: every kernel does its set-up before
griddepcontrol.wait (barriers, TMEM, descriptors, weight prefetch, the LayerNorm affine
parameters) and reads what an earlier kernel wrote only after it.  The same generation is
run in two processes, with PDL (the default) and without it (KIMODO_PDL=0, read once per
process), and the two results must agree bit for bit.  4 prompts x 150 frames give 1208
token rows per forward, so the CTA-pair GEMM, attention, LayerNorm and the motion kernels
all run."""
import os
import subprocess
import sys

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r"""
import sys
import numpy as np
sys.path.insert(0, {root!r})
import synth
import transformer_denoiser_b200 as kb
model = kb.Kimodo(synth.weight_blob(), kb.BF16, 0)
B, T = 4, 150
emb = synth.text_embeddings(B, seed=701)
null = np.zeros(4096, np.float32)
noise = synth.noise(B, T, seed=702)
lengths = np.full(B, T, np.int32)
x = model.ddim_sample(emb, null, noise, lengths, 4, 2.0)
np.save({out!r}, x)
"""


def _run(tmp_path, name, pdl):
    out = str(tmp_path / f"{name}.npy")
    env = dict(os.environ)
    if pdl:
        env.pop("KIMODO_PDL", None)
    else:
        env["KIMODO_PDL"] = "0"
    subprocess.run([sys.executable, "-c", CHILD.format(root=ROOT, out=out)], env=env, cwd=ROOT, check=True,
                   timeout=600)
    return np.load(out)


def test_pdl_and_serial_launches_agree(tmp_path):
    with_pdl = _run(tmp_path, "pdl", True)
    serial = _run(tmp_path, "serial", False)
    assert np.all(np.isfinite(with_pdl))
    np.testing.assert_array_equal(with_pdl, serial)
