"""The pins catch plausible mistakes in the oracle.

Each case copies ``oracle/gdr_oracle.c`` to a temporary directory, plants one
mistake by a textual edit (a wrong sign, a dropped term, a wrong index, a
transposed operand, swapped read modes ...), compiles it, and runs a battery
of the pins from ``test_oracle_pins`` against the mutant: at least one pin must
fail.  The unmodified source must pass the same battery.
"""
import os
import subprocess

import numpy as np
import pytest

import oracle
from oracle import wy_reference

from test_oracle_pins import _check_vs_exact, _random_rational_case, rand_problem

SRC = os.path.join(os.path.dirname(oracle.__file__), "gdr_oracle.c")

MUTANTS = {
    "erase_sign": ("u[j] = beta * (v[j] - alpha * sk[j]);", "u[j] = beta * (v[j] + alpha * sk[j]);"),
    "erase_drops_alpha": ("u[j] = beta * (v[j] - alpha * sk[j]);", "u[j] = beta * (v[j] - sk[j]);"),
    "write_drops_beta": ("u[j] = beta * (v[j] - alpha * sk[j]);", "u[j] = (v[j] - alpha * sk[j]);"),
    "no_decay_on_state": ("row[j] = alpha * row[j] + kd * u[j];", "row[j] = row[j] + kd * u[j];"),
    "decay_after_write": ("row[j] = alpha * row[j] + kd * u[j];", "row[j] = alpha * (row[j] + kd * u[j]);"),
    "transposed_state_read": ("for (int j = 0; j < dv; ++j) out[j] += row[j] * xd;",
                              "for (int j = 0; j < dv; ++j) out[j] += H[(size_t)j * dv + d] * xd;"),
    "read_modes_swapped": ("a->read_pre, a->scale, ob, sk, u);", "!a->read_pre, a->scale, ob, sk, u);"),
    "pre_read_unscaled": ("        state_t_times(H, q, dk, dv, o);\n        for (int j = 0; j < dv; ++j) o[j] *= scale;\n    }\n    state_t_times(H, k",
                          "        state_t_times(H, q, dk, dv, o);\n    }\n    state_t_times(H, k"),
    "gqa_modulo_index": ("hk = h / group;", "hk = h % Hk;"),
    "l2norm_by_square": ("for (int i = 0; i < n; ++i) x[i] /= den;", "for (int i = 0; i < n; ++i) x[i] /= ss;"),
    "reverse_ignored": ("const long t = a->reverse ? (t1 - 1 - i) : (t0 + i);", "const long t = t0 + i;"),
    "q_normalised_as_k": ("l2_normalise(qb, dk); l2_normalise(kb, dk);", "l2_normalise(kb, dk);"),
}


def _battery(lib) -> list:
    """Names of the pins that fail for the given compiled oracle."""
    failed = []
    for mode in ("post", "pre"):
        for l2 in (False, True):
            ok = all(_check_vs_exact(_random_rational_case(s, mode, l2, T=1 + s % 8), lib=lib)
                     for s in range(6))
            if not ok:
                failed.append(f"exact_{mode}_{'l2' if l2 else 'raw'}")
    # GQA + rectangular + varlen + reverse against the WY/UT form
    r = np.random.default_rng(11)
    lens = [33, 70, 5]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    q, k, v, g, beta, _ = rand_problem(T=int(cu[-1]), Hk=2, Hv=4, dk=12, dv=8, rng=r)
    S0 = r.standard_normal((len(lens), 4, 12, 8)) * 0.3
    for mode in ("post", "pre"):
        for rev in (False, True):
            o, S = oracle.forward(q, k, v, g, beta, S0, cu_seqlens=cu, read_mode=mode, scale=0.8,
                                  reverse=rev, _lib=lib)
            o2, S2 = wy_reference.chunked_forward(q, k, v, g, beta, S0, cu_seqlens=cu, chunk=16,
                                                  read_mode=mode, scale=0.8, reverse=rev)
            if not (np.abs(o - o2).max() < 1e-10 and np.abs(S - S2).max() < 1e-10):
                failed.append(f"wy_{mode}_{'rev' if rev else 'fwd'}")
    return failed


def _compile(src_text, tmp_path, name):
    c = tmp_path / f"{name}.c"
    so = tmp_path / f"lib{name}.so"
    c.write_text(src_text)
    subprocess.run(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c99", "-o", str(so),
                    str(c), "-lm"], check=True)
    return oracle.load_library(str(so))


def test_unmodified_oracle_passes_battery(tmp_path):
    with open(SRC) as f:
        lib = _compile(f.read(), tmp_path, "clean")
    assert _battery(lib) == []


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(name, tmp_path):
    with open(SRC) as f:
        text = f.read()
    old, new = MUTANTS[name]
    assert text.count(old) == 1, f"mutation site for {name} not found exactly once"
    lib = _compile(text.replace(old, new), tmp_path, name)
    assert _battery(lib), f"no pin caught the planted mistake {name}"
