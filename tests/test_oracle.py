"""Pins for the fp64 oracle, checked against things other than the oracle.

Every check here comes from the definition of the method (Attention-Level
Speculation, atlas.scime.ai summary, "Approach": a sink approximation checked
against exact attention with a relative L2 threshold; ICML 2025 poster page,
abstract) or from mathematics:
  - hand-derived cases (tests/golden/hand_cases.json);
  - the special case L <= S + W, where the sink set is the whole cache;
  - the closed form for equal keys (uniform weights -> plain means);
  - invariants: weights sum to 1, outputs in the convex hull of the values,
    permutation of middle tokens, value scaling, a common logit shift;
  - a planted needle outside the window drives the error above lambda;
  - a numpy textbook softmax(q K^T / sqrt d) V on explicit index sets.
No test here needs a GPU.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_cases.json")
SQRT2LN3 = math.sqrt(2.0) * math.log(3.0)


def _num(x):
    if isinstance(x, list):
        return [_num(e) for e in x]
    if x == "sqrt2ln3":
        return SQRT2LN3
    if x == "nan":
        return float("nan")
    if x == "inf":
        return float("inf")
    return float(x)


@pytest.fixture(scope="module")
def golden():
    with open(GOLDEN) as f:
        return {c["name"]: c for c in json.load(f)["cases"]}


def textbook(q, K, V, idx):
    """numpy softmax(q K[idx]^T / sqrt d) V[idx] in float64."""
    q = np.asarray(q, np.float64)
    K = np.asarray(K, np.float64)[idx]
    V = np.asarray(V, np.float64)[idx]
    s = K @ q / np.sqrt(q.shape[0])
    w = np.exp(s - s.max())
    w /= w.sum()
    return w @ V


def sink_index(L, S, W):
    """Explicit sorted index set: first S tokens united with the last W."""
    return np.array(sorted(set(range(min(S, L))) | set(range(max(0, L - W), L))), dtype=np.int64)


# ---------------------------------------------------------------- hand cases

def test_hand_two_tokens(golden):
    c = golden["two_tokens_weights_quarter_three_quarters"]
    q = np.array(_num(c["q"]))
    k = np.array(_num(c["k"]))
    v = np.array(_num(c["v"]))
    for sc in c["sink_cases"]:
        o_s, o_e, w_s, w_e = oracle.head(q, k, v, sc["S"], sc["W"], weights=True)
        np.testing.assert_allclose(o_e, c["o_exact"], rtol=0, atol=1e-15)
        np.testing.assert_allclose(w_e, c["w_exact"], rtol=0, atol=1e-15)
        np.testing.assert_allclose(o_s, sc["o_spec"], rtol=0, atol=1e-15)
        np.testing.assert_allclose(w_s, sc["w_spec"], rtol=0, atol=1e-15)
        assert oracle.rel_l2(o_s, o_e) == pytest.approx(sc["rel_l2"], abs=1e-14)


def test_hand_flag_boundary(golden):
    c = golden["uniform_weights_flag_boundary"]
    q, k, v = (np.array(_num(c[n])) for n in ("q", "k", "v"))
    o_s, o_e = oracle.head(q, k, v, c["S"], c["W"])
    assert o_e.tolist() == c["o_exact"] and o_s.tolist() == c["o_spec"]
    r = oracle.rel_l2(o_s, o_e)
    assert r == c["rel_l2"]
    assert oracle.commit(r, 1.0) == c["commit_at_lambda_1"]
    assert oracle.commit(r, np.nextafter(1.0, 0.0)) == c["commit_just_below_1"]
    assert oracle.commit(float("nan"), 1e300) == 0


def test_hand_zero_exact_output(golden):
    c = golden["zero_exact_output_discards"]
    q, k, v = (np.array(_num(c[n])) for n in ("q", "k", "v"))
    o_s, o_e = oracle.head(q, k, v, c["S"], c["W"])
    r = oracle.rel_l2(o_s, o_e)
    assert math.isinf(r)
    assert oracle.commit(r, 1e300) == c["commit_at_lambda_1e300"]
    # D = N = 0 (identical zero outputs) is an exact approximation: r = 0.
    assert oracle.rel_l2(np.zeros(3), np.zeros(3)) == 0.0


def test_hand_gqa_batch(golden):
    c = golden["gqa_batch_per_token_norm"]
    q = np.array(_num(c["q"]))
    k = np.array(_num(c["k"]))
    v = np.array(_num(c["v"]))
    res = oracle.decode(q, k, v, np.array(c["seq_lens"], np.int32), c["S"], c["W"], c["lambda"])
    np.testing.assert_allclose(res["out_exact"], c["o_exact"], rtol=0, atol=1e-15)
    np.testing.assert_allclose(res["out_spec"], c["o_spec"], rtol=0, atol=1e-15)
    np.testing.assert_allclose(res["rel_l2"], c["rel_l2"], rtol=0, atol=1e-14)
    assert res["commit"].tolist() == c["commit"]


def test_hand_bf16_decoding(golden):
    c = golden["bf16_decoding"]
    q = np.array(c["q_bits"], np.uint16)
    k = np.array(c["k_bits"], np.uint16)
    v = np.array(c["v_bits"], np.uint16)
    o_s, o_e = oracle.head(q, k, v, c["S"], c["W"])
    assert o_e.tolist() == c["o_exact"] and o_s.tolist() == c["o_spec"]


def test_bf16_widening_matches_torch():
    """The oracle's bf16 reading equals torch's bf16 -> float64 conversion."""
    g = torch.Generator().manual_seed(5)
    x = (torch.randn(64, 16, generator=g) * 3).to(torch.bfloat16)
    bits = x.view(torch.int16).numpy().view(np.uint16)
    # One-token cache: the output is exactly that token's value row.
    for row in range(4):
        o_s, o_e = oracle.head(bits[row], bits[row:row + 1], bits[row:row + 1], 1, 0)
        np.testing.assert_array_equal(o_e, x[row].double().numpy())


# ------------------------------------------------ special cases, closed forms

@pytest.mark.parametrize("L,S,W", [(1, 4, 128), (5, 4, 1), (132, 4, 128), (100, 4, 128),
                                   (7, 0, 7), (7, 7, 0), (3, 2, 2)])
def test_whole_cache_in_sink_set_is_exact(L, S, W):
    """L <= S + W: the sink set is [0, L), so both outputs are identical, r = 0."""
    rng = np.random.default_rng(L * 31 + S)
    d = 16
    q, k, v = rng.standard_normal(d), rng.standard_normal((L, d)), rng.standard_normal((L, d))
    o_s, o_e = oracle.head(q, k, v, S, W)
    assert np.array_equal(o_s, o_e)
    assert oracle.rel_l2(o_s, o_e) == 0.0
    assert oracle.commit(0.0, 0.0) == 1


@pytest.mark.parametrize("L,S,W", [(64, 4, 8), (33, 1, 0), (33, 0, 5), (10, 4, 5)])
def test_equal_keys_closed_form(L, S, W):
    """All keys equal -> uniform weights -> O_exact = mean V, O_spec = mean V[sink set]."""
    rng = np.random.default_rng(L)
    d, Hq = 8, 3
    kv_key = rng.standard_normal(d)
    k = np.tile(kv_key, (L, 1))
    v = rng.standard_normal((L, d))
    idx = sink_index(L, S, W)
    o_s_all, o_e_all = [], []
    for h in range(Hq):
        q = rng.standard_normal(d)
        o_s, o_e = oracle.head(q, k, v, S, W)
        np.testing.assert_allclose(o_e, v.mean(axis=0), rtol=0, atol=1e-14)
        np.testing.assert_allclose(o_s, v[idx].mean(axis=0), rtol=0, atol=1e-14)
        o_s_all.append(o_s)
        o_e_all.append(o_e)
    diff = np.tile(v.mean(axis=0) - v[idx].mean(axis=0), Hq)
    ref = math.sqrt(float(diff @ diff) / (Hq * float(v.mean(axis=0) @ v.mean(axis=0))))
    assert oracle.rel_l2(np.array(o_s_all), np.array(o_e_all)) == pytest.approx(ref, rel=1e-12)


# ---------------------------------------------------------------- invariants

def _rand_head(seed, L=200, d=32):
    rng = np.random.default_rng(seed)
    return rng.standard_normal(d) * 2, rng.standard_normal((L, d)), rng.standard_normal((L, d))


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_weights_sum_to_one_and_outside_set_is_zero(seed):
    q, k, v = _rand_head(seed)
    S, W = 4, 16
    _, _, w_s, w_e = oracle.head(q, k, v, S, W, weights=True)
    assert abs(w_e.sum() - 1.0) < 1e-14 and abs(w_s.sum() - 1.0) < 1e-14
    assert (w_e > 0).all()
    inside = np.zeros(len(w_s), bool)
    inside[sink_index(len(w_s), S, W)] = True
    assert (w_s[~inside] == 0).all() and (w_s[inside] > 0).all()


@pytest.mark.parametrize("seed", [3, 4])
def test_outputs_in_convex_hull(seed):
    q, k, v = _rand_head(seed)
    o_s, o_e = oracle.head(q, k, v, 4, 16)
    idx = sink_index(len(k), 4, 16)
    assert (o_e >= v.min(axis=0) - 1e-15).all() and (o_e <= v.max(axis=0) + 1e-15).all()
    assert (o_s >= v[idx].min(axis=0) - 1e-15).all() and (o_s <= v[idx].max(axis=0) + 1e-15).all()


def test_middle_permutation_invariance():
    q, k, v = _rand_head(7)
    S, W, L = 4, 16, len(k)
    perm = np.arange(L)
    rng = np.random.default_rng(0)
    perm[S:L - W] = S + rng.permutation(L - W - S)
    o_s, o_e = oracle.head(q, k, v, S, W)
    o_s2, o_e2 = oracle.head(q, k[perm], v[perm], S, W)
    assert np.array_equal(o_s, o_s2)  # the sink set is untouched
    np.testing.assert_allclose(o_e2, o_e, rtol=0, atol=1e-14)


def test_value_scaling_keeps_rel_l2():
    q, k, v = _rand_head(8)
    o_s, o_e = oracle.head(q, k, v, 4, 16)
    o_s2, o_e2 = oracle.head(q, k, 4.0 * v, 4, 16)     # power of two: exact scaling
    assert np.array_equal(o_e2, 4.0 * o_e) and np.array_equal(o_s2, 4.0 * o_s)
    assert oracle.rel_l2(o_s2, o_e2) == pytest.approx(oracle.rel_l2(o_s, o_e), rel=1e-15)


def test_common_logit_shift_invariance():
    """k_j += c sqrt(d) q / |q|^2 adds c to every logit; softmax is unchanged."""
    q, k, v = _rand_head(9)
    d = q.shape[0]
    c = 3.25
    k2 = k + c * math.sqrt(d) * q / (q @ q)
    o_s, o_e = oracle.head(q, k, v, 4, 16)
    o_s2, o_e2 = oracle.head(q, k2, v, 4, 16)
    np.testing.assert_allclose(o_e2, o_e, rtol=0, atol=1e-12)
    np.testing.assert_allclose(o_s2, o_s, rtol=0, atol=1e-12)


# ------------------------------------------------------- needle, commit case

def _structured(seed, L, d, S, W, sink_bump, needle_bump=None, needle_pos=None, g=4):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((g, d))
    qhat = q / np.linalg.norm(q, axis=1, keepdims=True)
    k = rng.standard_normal((L, d))
    v = rng.standard_normal((L, d))
    k[:S] += sink_bump * qhat.sum(axis=0)
    if needle_bump is not None:
        k[needle_pos] += needle_bump * qhat[0]
        v[needle_pos] += 4 * rng.standard_normal(d)
    return q, k, v


def _token_r(q, k, v, S, W):
    outs = [oracle.head(q[h], k, v, S, W) for h in range(q.shape[0])]
    return oracle.rel_l2(np.array([o[0] for o in outs]), np.array([o[1] for o in outs]))


def test_strong_sinks_commit_and_needle_discards():
    L, d, S, W, lam = 4096, 64, 4, 128, 0.10
    q, k, v = _structured(11, L, d, S, W, sink_bump=24.0)
    r0 = _token_r(q, k, v, S, W)
    assert r0 <= lam and oracle.commit(r0, lam) == 1
    # Needle outside the window, bump >= sink bump + 4 logits, on head 0.
    q, k, v = _structured(11, L, d, S, W, sink_bump=24.0, needle_bump=32.0, needle_pos=1500)
    r1 = _token_r(q, k, v, S, W)
    assert r1 > lam and oracle.commit(r1, lam) == 0
    # Moving the same needle inside the window puts it back in the sink set.
    q, k, v = _structured(11, L, d, S, W, sink_bump=24.0, needle_bump=32.0, needle_pos=L - 5)
    assert _token_r(q, k, v, S, W) <= lam


# --------------------------------------------------------- textbook cross-check

@pytest.mark.parametrize("dtype", ["f64", "f32", "bf16"])
@pytest.mark.parametrize("L,S,W", [(97, 4, 16), (300, 0, 33), (64, 7, 0), (20, 4, 16)])
def test_numpy_textbook_cross_check(dtype, L, S, W):
    g = torch.Generator().manual_seed(L + S + W)
    d = 24
    qt, kt, vt = (torch.randn(*s, generator=g, dtype=torch.float64) for s in ((d,), (L, d), (L, d)))
    if dtype == "f64":
        q, k, v = qt.numpy(), kt.numpy(), vt.numpy()
    elif dtype == "f32":
        qt, kt, vt = qt.float(), kt.float(), vt.float()
        q, k, v = qt.numpy(), kt.numpy(), vt.numpy()
    else:
        qt, kt, vt = qt.bfloat16(), kt.bfloat16(), vt.bfloat16()
        q, k, v = (t.view(torch.int16).numpy().view(np.uint16) for t in (qt, kt, vt))
    qd, kd, vd = qt.double().numpy(), kt.double().numpy(), vt.double().numpy()
    o_s, o_e = oracle.head(q, k, v, S, W)
    np.testing.assert_allclose(o_e, textbook(qd, kd, vd, np.arange(L)), rtol=0, atol=1e-12)
    np.testing.assert_allclose(o_s, textbook(qd, kd, vd, sink_index(L, S, W)), rtol=0, atol=1e-12)


def test_batch_decode_matches_textbook_with_gqa_mapping():
    """Batch entry point: head h reads KV head h // g; ragged lengths; per-token r."""
    rng = np.random.default_rng(42)
    B, Hq, Hkv, d, Lmax, S, W, lam = 3, 8, 2, 16, 90, 3, 10, 0.3
    g = Hq // Hkv
    q = rng.standard_normal((B, Hq, d))
    k = rng.standard_normal((B, Hkv, Lmax, d))
    v = rng.standard_normal((B, Hkv, Lmax, d))
    lens = np.array([90, 13, 41], np.int32)
    for b in range(B):
        k[b, :, lens[b]:] = np.nan  # beyond the sequence: must never be read
        v[b, :, lens[b]:] = np.nan
    res = oracle.decode(q, k, v, lens, S, W, lam, n_threads=2)
    for b in range(B):
        L = lens[b]
        es, ee = [], []
        for h in range(Hq):
            kk, vv = k[b, h // g, :L], v[b, h // g, :L]
            ee.append(textbook(q[b, h], kk, vv, np.arange(L)))
            es.append(textbook(q[b, h], kk, vv, sink_index(L, S, W)))
        ee, es = np.array(ee), np.array(es)
        np.testing.assert_allclose(res["out_exact"][b], ee, rtol=0, atol=1e-12)
        np.testing.assert_allclose(res["out_spec"][b], es, rtol=0, atol=1e-12)
        r = np.linalg.norm(ee - es) / np.linalg.norm(ee)
        assert res["rel_l2"][b] == pytest.approx(r, rel=1e-12)
        assert res["commit"][b] == (1 if r <= lam else 0)
    assert res["threads"] == 2


def test_bad_arguments_raise():
    q = np.zeros((1, 2, 4))
    k = np.zeros((1, 1, 8, 4))
    with pytest.raises(ValueError):
        oracle.decode(q, k, k, np.array([9], np.int32), 1, 1, 0.1)      # L > Lmax
    with pytest.raises(ValueError):
        oracle.decode(q, k, k, np.array([0], np.int32), 1, 1, 0.1)      # L < 1
    with pytest.raises(ValueError):
        oracle.decode(q, k, k, np.array([4], np.int32), 0, 0, 0.1)      # empty sink set
    with pytest.raises(ValueError):
        oracle.head(np.zeros(4), np.zeros((3, 4)), np.zeros((3, 4)), -1, 2)


# ------------------------------------------------------- output projection

OPROJ_GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden",
                            "oproj_cases.json")


def _oproj_cases():
    with open(OPROJ_GOLDEN) as f:
        return {c["name"]: c for c in json.load(f)["cases"]}


def test_oproj_hand_cases():
    c = _oproj_cases()
    a = c["non_square_two_tokens"]
    y = oracle.oproj(np.array(a["x"]), np.array(a["w"], np.float32))
    assert np.array_equal(y, np.array(a["y"]))
    g = c["gated_one_commit_one_discard"]
    y = oracle.oproj_gated(g["o_spec"], g["o_exact"], g["commit"], np.array(g["w"], np.float64))
    assert np.array_equal(y, np.array(g["y"]))
    h = c["bf16_weights"]
    y = oracle.oproj(np.array(h["x"]), np.array(h["w_bf16_bits"], np.uint16))
    assert np.array_equal(y, np.array(h["y"]))


def test_oproj_one_hot_rows_pick_entries():
    """w row j = unit vector e_pi(j): y[b, j] = x[b, pi(j)] exactly."""
    rng = np.random.default_rng(11)
    K, N = 24, 17
    perm = rng.integers(0, K, N)
    w = np.zeros((N, K), np.float32)
    w[np.arange(N), perm] = 1.0
    x = rng.standard_normal((3, K))
    assert np.array_equal(oracle.oproj(x, w), x[:, perm])


def test_oproj_all_ones_gives_row_sums():
    """Closed form: w = 1 everywhere gives every output the sum of its row."""
    rng = np.random.default_rng(12)
    x = rng.standard_normal((2, 64))
    y = oracle.oproj(x, np.ones((5, 64), np.float32))
    for b in range(2):
        assert np.allclose(y[b], math.fsum(x[b]), rtol=0, atol=1e-12)


def test_oproj_is_linear_and_gating_selects_rows():
    rng = np.random.default_rng(13)
    K, N = 32, 9
    w = rng.standard_normal((N, K)).astype(np.float32)
    x1, x2 = rng.standard_normal((2, K)), rng.standard_normal((2, K))
    lhs = oracle.oproj(2.0 * x1 - 0.5 * x2, w)
    rhs = 2.0 * oracle.oproj(x1, w) - 0.5 * oracle.oproj(x2, w)
    assert np.allclose(lhs, rhs, rtol=0, atol=1e-12)
    commit = np.array([1, 0], np.uint8)
    y = oracle.oproj_gated(x1, x2, commit, w)
    assert np.array_equal(y[0], oracle.oproj(x1[:1], w)[0])
    assert np.array_equal(y[1], oracle.oproj(x2[1:], w)[0])
