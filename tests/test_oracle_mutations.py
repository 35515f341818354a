"""The oracle's pins catch plausible mistakes: each case below plants one
mistake in a copy of the oracle (a dropped term, a wrong sign or index, a
transposed operand, a swapped field) and runs the CPU pins against that copy
in a separate process; at least one pin must fail.  The oracle itself is
never modified."""

import os
import shutil
import subprocess
import sys
import tempfile
from concurrent.futures import ThreadPoolExecutor

import pytest

from conftest import ROOT

PINS = ["tests/test_oracle.py", "tests/test_oracle_variants.py", "tests/test_oracle_proj.py"]

# (name, exact text in oracle/lisa_ref.py, its planted replacement)
MUTATIONS = [
    ("ties toward the higher position", "    return np.lexsort((np.arange(n), -scores))",
     "    return np.lexsort((-np.arange(n), -scores))"),
    ("selection not in ascending position", "    keep = np.sort(_order(scores)[: min(M, n)])",
     "    keep = _order(scores)[: min(M, n)]"),
    ("window one position too long", "    lo = max(0, t - W + 1)", "    lo = max(0, t - W)"),
    ("softmax scale 1/d", "    logits = (K_sel @ q_h) / np.sqrt(d)", "    logits = (K_sel @ q_h) / d"),
    ("state update transposed", "    return S_h + np.outer(k_t, v_t)", "    return S_h + np.outer(v_t, k_t)"),
    ("readout transposed", "    return q_h @ S_h\n", "    return S_h @ q_h\n"),
    ("gate branches swapped", "    return g * o_sp + (1.0 - g) * o_lin", "    return g * o_lin + (1.0 - g) * o_sp"),
    ("gate sign", "        g = 1.0 / (1.0 + np.exp(-float(lam)))", "        g = 1.0 / (1.0 + np.exp(float(lam)))"),
    ("indexer without ReLU", "            out[gs] += w_t[j] * np.maximum(dots, 0.0)", "            out[gs] += w_t[j] * dots"),
    ("indexer weights dropped", "            out[gs] += w_t[j] * np.maximum(dots, 0.0)",
     "            out[gs] += np.maximum(dots, 0.0)"),
    ("indexer head against its group's plane", "            plane = gs if P == Gs else j\n",
     "            plane = gs if P == Gs else gs\n"),
    ("borderline rule without its floor", "    tol = rel * max(abs(sM), floor * float(np.max(np.abs(scores))))",
     "    tol = rel * abs(sM)"),
    ("decode: selection group fixed to 0", "            gs = 0 if shared_set else g\n",
     "            gs = g if shared_set and Gs > g else 0\n"),
    ("prefill: selection group fixed to 0", "                gs = 0 if shared_set else g\n", "                gs = 0\n"),
    ("linear-branch keys per head ignored", "            kl_h = k[b, g] if k_lin is None else k_lin[b, h]\n",
     "            kl_h = k[b, g]\n"),
    ("KL: sign of the indexer term", "                kl[b, t, h] = float(np.sum(pa * (la - lr)))",
     "                kl[b, t, h] = float(np.sum(pa * (la + lr)))"),
    ("front-end: k and v swapped", 'PROJ_FIELDS = ("q", "k", "v", "qidx", "kidx", "w", "lam")',
     'PROJ_FIELDS = ("q", "v", "k", "qidx", "kidx", "w", "lam")'),
    ("front-end: a field boundary off by one", "        c += wd\n", "        c += wd + (1 if name == 'k' else 0)\n"),
    ("front-end weights reversed", "    z = x @ W_in.T\n", "    z = x @ W_in.T[::-1]\n"),
    ("output projection reversed", "    return flat @ W_o.T\n", "    return (W_o @ flat.T).T[..., ::-1]\n"),
]


def _pins_fail(name, old, new):
    with tempfile.TemporaryDirectory() as tmp:
        for d in ("oracle", "lisa_inputs", "tests"):
            shutil.copytree(os.path.join(ROOT, d), os.path.join(tmp, d),
                            ignore=shutil.ignore_patterns("__pycache__"))
        path = os.path.join(tmp, "oracle", "lisa_ref.py")
        src = open(path).read()
        assert src.count(old) >= 1, f"{name}: the text to mutate is not in the oracle"
        open(path, "w").write(src.replace(old, new, 1))
        r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-m", "not gpu", "-p", "no:cacheprovider",
                            *PINS], cwd=tmp, capture_output=True, text=True, timeout=600)
        return r.returncode != 0


def test_every_planted_mistake_fails_a_pin():
    with ThreadPoolExecutor(max_workers=4) as ex:
        caught = list(ex.map(lambda m: (m[0], _pins_fail(*m)), MUTATIONS))
    missed = [n for n, c in caught if not c]
    assert not missed, f"mistakes no pin catches: {missed}"
