"""The oracle's pins must catch plausible mistakes planted in a copy of it.

Each case copies ``oracle/`` to a temporary tree, applies one textual
mutation (a swapped operand, a dropped term, a wrong sign, a transposed
nibble order) and runs the oracle pin tests there in a subprocess; at least
one pin must fail.  The real oracle is never modified.
"""

import os
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

MUTATIONS = [
    ("moe.py", "a = _silu(g) * u ", "a = _silu(u) * g "),                          # gate/up swapped
    ("moe.py", "(1.0 + g * (1.0 - sg))", "(1.0 - g * (1.0 - sg))"),               # wrong sign in silu'
    ("moe.py", '"dA_gu": s * q_gu.T @ X', '"dA_gu": q_gu.T @ X'),                  # dropped scaling
    ("moe.py", "gu = X @ w_gu.T + s * (p_gu @ B_gu.T)", "gu = X @ w_gu.T + (p_gu @ B_gu.T)"),
    ("moe.py", "yd = a @ w_d.T + s * (p_d @ B_d.T)", "yd = a @ w_d.T"),            # dropped down LoRA
    ("moe.py", "dX = dgu @ w_gu + s * (q_gu @ A_gu)", "dX = dgu @ w_gu"),          # dropped LoRA dgrad
    ("moe.py", '"dB_d": s * dyw.T @ fwd["p_d"]', '"dB_d": s * dyw.T @ fwd["p_gu"][:, :0].sum() * fwd["p_d"]'),
    ("nf4.py", "codes[..., 0::2] = hi\n    codes[..., 1::2] = lo",
     "codes[..., 0::2] = lo\n    codes[..., 1::2] = hi"),                         # nibble order
    ("nf4.py", "product = (table[codes] * scale)", "product = (table[codes[..., ::-1]] * scale)"),
    ("moe.py", 'order = np.argsort(-logits, axis=1, kind="stable")', 'order = np.argsort(logits, axis=1, kind="stable")[:, ::-1]'),
    ("moe.py", "w[t] * (dw[t] - float(np.dot(w[t], dw[t])))", "w[t] * dw[t]"),     # router: no softmax mean
    ("moe.py", "w[t] * (dw[t] - float(np.dot(w[t], dw[t])))", "(dw[t] - float(np.dot(w[t], dw[t])))"),
    ("nf4.py", "BLOCK = 64", "BLOCK = 128"),                                          # block size
    ("nf4.py", "absmax = np.abs(blocks).max(axis=-1).astype(np.float32)",
     "absmax = np.abs(blocks).max(axis=-1).astype(np.float64)"),                     # scale precision
]


@pytest.mark.parametrize("fname,old,new", MUTATIONS, ids=[m[2][:40] for m in MUTATIONS])
def test_pins_catch_mutation(tmp_path, fname, old, new):
    dst = tmp_path / "tree"
    shutil.copytree(os.path.join(ROOT, "oracle"), dst / "oracle")
    shutil.copytree(os.path.join(ROOT, "tests"), dst / "tests",
                    ignore=shutil.ignore_patterns("test_oracle_mutations.py", "__pycache__"))
    shutil.copytree(os.path.join(ROOT, "grouped_nf4_expert_b200"), dst / "grouped_nf4_expert_b200",
                    ignore=shutil.ignore_patterns("*.so", "__pycache__", "csrc"))
    path = dst / "oracle" / fname
    src = path.read_text()
    assert old in src, "mutation target not found: %r" % old
    path.write_text(src.replace(old, new, 1))
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
                        "tests/test_oracle_moe.py", "tests/test_oracle_nf4.py"],
                       cwd=dst, capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, "planted mistake went unnoticed:\n" + r.stdout[-2000:]
