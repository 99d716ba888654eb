"""The oracle's pins have teeth: each plausible slip, planted in a scratch
copy of the oracle (never in the product), makes tests/test_oracle.py fail.
CPU only; each case runs the pin file in a subprocess against the mutated
copy."""

import os
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
ORACLE = os.path.join(ROOT, "oracle", "sbattn_oracle.py")

# (text in the oracle, its mutation, what the slip is)
MUTATIONS = [
    ("out[..., 1::2] = a * s + b * c", "out[..., 1::2] = -a * s + b * c", "RoPE rotation sign"),
    ("inv_freq = theta ** (-2.0 * m / D)", "inv_freq = theta ** (-1.0 * m / D)", "RoPE frequency exponent"),
    ("return x / np.sqrt(ms + eps)", "return x / (np.sqrt(ms) + eps)", "RMSNorm eps outside the root"),
    ("np.lexsort((others, -scores_row[others]))", "np.lexsort((-others, -scores_row[others]))", "tie order"),
    ("return P @ Vs", "return P[:, ::-1] @ Vs", "softmax weights misaligned with V rows"),
    ("np.stack([n // (Hh * W), (n // W) % Hh, n % W]", "np.stack([n // (Hh * W), n % W, (n // W) % Hh]",
     "grid axis order"),
    ("return (x - mu) / np.sqrt(var + eps)", "return (x - mu) / (np.sqrt(var) + eps)", "LayerNorm eps outside the root"),
    ("var = ((x - mu) ** 2).mean(axis=-1, keepdims=True)",
     "var = ((x - mu) ** 2).sum(axis=-1, keepdims=True) / (x.shape[-1] - 1)", "unbiased variance"),
    ("return layer_norm(x, eps) * (1.0 + scale) + shift", "return layer_norm(x, eps) * scale + shift",
     "AdaLN scale without the 1 +"),
    ("return a / (1.0 + np.exp(-a))", "return a / (1.0 + np.exp(a))", "SiLU sign"),
    ("return silu(gate) * np.asarray(up, dtype=np.float64)", "return silu(up) * np.asarray(gate, dtype=np.float64)",
     "SwiGLU gate and up swapped"),
]


def _scratch_tree(dst, mutated_source):
    os.makedirs(os.path.join(dst, "oracle"))
    os.makedirs(os.path.join(dst, "block_sparse_attention_qk_b200"))
    shutil.copytree(os.path.join(ROOT, "tests", "golden"), os.path.join(dst, "tests", "golden"))
    for f in ("__init__.py", "conftest.py", "test_oracle.py"):
        shutil.copy(os.path.join(ROOT, "tests", f), os.path.join(dst, "tests", f))
    for f in os.listdir(os.path.join(ROOT, "oracle")):
        if f.endswith(".py"):
            shutil.copy(os.path.join(ROOT, "oracle", f), os.path.join(dst, "oracle", f))
    with open(os.path.join(dst, "oracle", "sbattn_oracle.py"), "w") as fh:
        fh.write(mutated_source)
    pkg = os.path.join(ROOT, "block_sparse_attention_qk_b200")
    for f in os.listdir(pkg):
        if f.endswith(".py"):
            shutil.copy(os.path.join(pkg, f), os.path.join(dst, "block_sparse_attention_qk_b200", f))


@pytest.mark.parametrize("old,new,what", MUTATIONS, ids=[m[2] for m in MUTATIONS])
def test_planted_slip_fails_a_pin(tmp_path, old, new, what):
    src = open(ORACLE).read()
    assert src.count(old) == 1, f"mutation site not found once: {old}"
    dst = str(tmp_path / "tree")
    _scratch_tree(dst, src.replace(old, new))
    env = dict(os.environ, PYTHONPATH=dst)
    r = subprocess.run([sys.executable, "-m", "pytest", "tests/test_oracle.py", "-x", "-q", "-p", "no:cacheprovider"],
                       cwd=dst, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 1, f"'{what}' was not caught by any pin:\n{r.stdout[-2000:]}"


def test_unmutated_copy_passes(tmp_path):
    dst = str(tmp_path / "tree")
    _scratch_tree(dst, open(ORACLE).read())
    env = dict(os.environ, PYTHONPATH=dst)
    r = subprocess.run([sys.executable, "-m", "pytest", "tests/test_oracle.py", "-q", "-p", "no:cacheprovider"],
                       cwd=dst, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout[-2000:]
