"""The backward oracle's pins catch plausible mistakes in it.

Each case loads a copy of ``oracle/backward.py`` with one mistake planted by a textual edit
(a dropped term, a wrong sign, the wrong state, a missing factor, a missed reduction ...)
and runs the finite-difference pins against it: at least one must fail.  The unmodified
source passes the same battery."""
import importlib.util
import os

import numpy as np
import pytest

from oracle import backward as bw
from test_oracle_backward import CASES, fd_grads, problem

SRC = bw.__file__

MUTANTS = {
    "erase_term_dropped_from_da": ("da = da - bt * np.sum(du * s, axis=-1)", "da = da"),
    "state_term_dropped_from_dk": ('dkh = dkh + np.einsum("hde,he->hd", H, ds)', "dkh = dkh"),
    "ds_sign": ("ds = -(a * bt)[:, None] * du", "ds = (a * bt)[:, None] * du"),
    "post_read_of_old_state": ('dqh = scale * np.einsum("hde,he->hd", Hn, do)',
                               'dqh = scale * np.einsum("hde,he->hd", H, do)'),
    "dbeta_without_decay": ("np.sum(du * (v[row, t] - a[:, None] * s), axis=-1)",
                            "np.sum(du * (v[row, t] - s), axis=-1)"),
    "norm_adjoint_without_projection": ("(dxh - xh * proj)", "(dxh)"),
    "dg_without_alpha": ('out["dg"][row, t] = a * da', 'out["dg"][row, t] = da'),
    "state_gradient_not_decayed": ("dHp = a[:, None, None] * dH", "dHp = dH"),
    "gqa_not_summed": ('out["dq"][row, t] += dq_h.reshape(Hk, group, dk).sum(axis=1)',
                       'out["dq"][row, t] += dq_h.reshape(Hk, group, dk)[:, 0]'),
    "reverse_ignored": ("order = list(range(t1 - 1, t0 - 1, -1)) if reverse else list(range(t0, t1))",
                        "order = list(range(t0, t1))"),
    "pre_read_added_after_erase": ("                if pre:\n                    dqh",
                                   "                if False:\n                    dqh"),
}


def _load(tmp_path, name, text):
    path = os.path.join(tmp_path, f"bw_{name}.py")
    with open(path, "w") as f:
        f.write(text)
    spec = importlib.util.spec_from_file_location(f"bw_{name}", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _battery(mod) -> list:
    failed = []
    x, up, cu = problem(1, 0, 1, 2, 3, 2, lengths=[3, 1, 4])
    cases = CASES + [dict(read_mode="post", reverse=False, qk_l2norm=True, gqa=True)]
    for kw in cases:
        kw = dict(kw)
        if kw.pop("gqa", False):
            x, up, cu = problem(2, 4, 1, 3, 2, 3)
        want = fd_grads(x, up, cu, scale=0.7, **kw)
        try:
            got = mod.backward(x["q"], x["k"], x["v"], x["g"], x["beta"], up["dO"], x["S0"],
                               up["dS_final"], cu, scale=0.7, **kw)
        except Exception:
            failed.append(str(kw))
            continue
        if not all(np.allclose(got[n], r, rtol=1e-6, atol=1e-7) for n, r in want.items()):
            failed.append(str(kw))
    return failed


def test_unmodified_passes(tmp_path):
    assert _battery(_load(tmp_path, "clean", open(SRC).read())) == []


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_caught(tmp_path, name):
    old, new = MUTANTS[name]
    text = open(SRC).read()
    assert text.count(old) == 1, f"mutation site of {name} not found once"
    assert _battery(_load(tmp_path, name, text.replace(old, new))), f"{name} not caught"
