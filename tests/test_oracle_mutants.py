"""The oracle's pins catch plausible mistakes.

Each case plants one mistake in a copy of the oracle's C source (on the CPU,
in a temporary directory), builds it, and checks that at least one pin fails
for the mutated build while every pin passes for the real one.  This shows
the pins in test_oracle.py are strong enough to catch a dropped term, a wrong
sign or index, or an off-by-one set boundary.
"""
import json
import math
import os
import subprocess

import numpy as np
import pytest

import oracle
from oracle import build as oracle_build

from test_oracle import GOLDEN, OPROJ_GOLDEN, _num, sink_index, textbook

MUTANTS = {
    "no_softmax_scale": ("const double scale = 1.0 / sqrt((double)d);",
                         "const double scale = 1.0;"),
    "window_off_by_one": ("return j < n_sink || j >= L - window;",
                          "return j < n_sink || j > L - window;"),
    "sink_off_by_one": ("return j < n_sink || j >= L - window;",
                        "return j <= n_sink || j >= L - window;"),
    "gqa_modulo_mapping": ("int kvh = h / g;", "int kvh = h % Hkv;"),
    "rel_l2_without_sqrt": ("return sqrt(num / den);", "return num / den;"),
    "strict_commit": ("return r <= lambda ? 1 : 0;", "return r < lambda ? 1 : 0;"),
    "norm_of_spec": ("den += o_exact[i] * o_exact[i];", "den += o_spec[i] * o_spec[i];"),
    "no_normalisation": ("double p = scores[j] / z;", "double p = scores[j];"),
    "no_max_subtraction": ("scores[j] = exp(scores[j] - m);", "scores[j] = exp(scores[j]);"),
    "oproj_transposed_weight": ("load_elem(w, w_dtype, (size_t)j * K + i)",
                                "load_elem(w, w_dtype, (size_t)i * N + j)"),
    "oproj_drops_last_term": ("for (int i = 0; i < K; ++i) {", "for (int i = 0; i < K - 1; ++i) {"),
    "oproj_gate_inverted": ("const double* x = commit[b] ? o_spec + (size_t)b * K : o_exact + (size_t)b * K;",
                            "const double* x = commit[b] ? o_exact + (size_t)b * K : o_spec + (size_t)b * K;"),
}


def _build_mutant(tmp_path, name):
    src = open(oracle_build.SRC).read()
    old, new = MUTANTS[name]
    assert src.count(old) == 1, f"mutation anchor for {name} not found once"
    path = tmp_path / f"{name}.c"
    path.write_text(src.replace(old, new))
    lib = str(tmp_path / f"lib{name}.so")
    subprocess.run(["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-o", lib, str(path), "-lm"],
                   check=True)
    return lib


def _pins_pass(lib):
    """Run a battery of pins against the build at ``lib``; True if all hold."""
    with open(GOLDEN) as f:
        cases = {c["name"]: c for c in json.load(f)["cases"]}
    try:
        c = cases["two_tokens_weights_quarter_three_quarters"]
        q, k, v = (np.array(_num(c[n])) for n in ("q", "k", "v"))
        for sc in c["sink_cases"]:
            o_s, o_e = oracle.head(q, k, v, sc["S"], sc["W"], lib=lib)
            if not (np.allclose(o_e, c["o_exact"], atol=1e-14) and
                    np.allclose(o_s, sc["o_spec"], atol=1e-14)):
                return False
            if abs(oracle.rel_l2(o_s, o_e, lib=lib) - sc["rel_l2"]) > 1e-13:
                return False
        c = cases["uniform_weights_flag_boundary"]
        q, k, v = (np.array(_num(c[n])) for n in ("q", "k", "v"))
        o_s, o_e = oracle.head(q, k, v, c["S"], c["W"], lib=lib)
        r = oracle.rel_l2(o_s, o_e, lib=lib)
        if r != 1.0 or oracle.commit(r, 1.0, lib=lib) != 1:
            return False
        c = cases["gqa_batch_per_token_norm"]
        res = oracle.decode(np.array(_num(c["q"])), np.array(_num(c["k"])),
                            np.array(_num(c["v"])), np.array(c["seq_lens"], np.int32),
                            c["S"], c["W"], c["lambda"], lib=lib)
        if not (np.allclose(res["out_exact"], c["o_exact"], atol=1e-14) and
                np.allclose(res["rel_l2"], c["rel_l2"], atol=1e-13)):
            return False
        # Textbook cross-check with a window boundary inside the cache.
        rng = np.random.default_rng(3)
        d, L, S, W = 16, 50, 3, 7
        q, k, v = rng.standard_normal(d), rng.standard_normal((L, d)), rng.standard_normal((L, d))
        o_s, o_e = oracle.head(q, k, v, S, W, lib=lib)
        if not (np.allclose(o_e, textbook(q, k, v, np.arange(L)), atol=1e-12) and
                np.allclose(o_s, textbook(q, k, v, sink_index(L, S, W)), atol=1e-12)):
            return False
        # Large common logit shift (exp would overflow without the max).
        k2 = k + 900.0 * math.sqrt(d) * q / (q @ q)
        o_s2, o_e2 = oracle.head(q, k2, v, S, W, lib=lib)
        if not (np.allclose(o_e2, o_e, atol=1e-9) and np.allclose(o_s2, o_s, atol=1e-9)):
            return False
        # Output projection: hand cases (non-square, gated, bf16 weights).
        with open(OPROJ_GOLDEN) as f:
            pc = {c["name"]: c for c in json.load(f)["cases"]}
        a = pc["non_square_two_tokens"]
        if not np.array_equal(oracle.oproj(np.array(a["x"]), np.array(a["w"], np.float32),
                                           lib=lib), np.array(a["y"])):
            return False
        g = pc["gated_one_commit_one_discard"]
        if not np.array_equal(oracle.oproj_gated(g["o_spec"], g["o_exact"], g["commit"],
                                                 np.array(g["w"], np.float64), lib=lib),
                              np.array(g["y"])):
            return False
    except (ValueError, FloatingPointError):
        return False
    return True


def test_real_oracle_passes_battery():
    assert _pins_pass(oracle_build.build())


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(tmp_path, name):
    lib = _build_mutant(tmp_path, name)
    assert not _pins_pass(lib), f"planted mistake {name} passed every pin"
