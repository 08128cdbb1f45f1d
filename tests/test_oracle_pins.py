"""Pins of the fp64 oracle to facts fixed outside the oracle itself.

Each test checks the oracle against something it cannot agree with by
construction: a hand-derived worked example, counts printed by the pages,
the bf16 format definition, a closed-form identity of the method, or a
brute-force / naive-loop computation on tiny inputs.  Together they are
chosen so that a dropped term, a flipped sign, a swapped index or a
transposed operand anywhere in the oracle fails at least one of them.

Method source: "MoVA: routing the value vectors, and why the KV cache does
not notice", sections "Where the routing happens" and "So what does it
cost?".
"""
import itertools
import json
import math
import os

import numpy as np
import pytest

from oracle import mova_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _naive_silu(z):
    return z / (1.0 + math.exp(-z))


def _naive_matvec(W, x):
    # W: list of rows (n x d), x: length d.  Plain loops, no numpy.
    return [sum(W[r][j] * x[j] for j in range(len(x))) for r in range(len(W))]


# ---------------------------------------------------------------------------
# Worked examples derived by hand (tests/golden/worked_example.json)
# ---------------------------------------------------------------------------


@pytest.mark.parametrize("case", _load("worked_example.json")["cases"], ids=lambda c: c["name"])
def test_worked_example(case):
    ln3 = math.log(3.0)
    p = np.array(case["p"], dtype=np.float64)
    x = np.array(case["x"], dtype=np.float64)
    # Router weight chosen so that logit_e = ln(p_e / (1 - p_e)) for x = [1].
    Wr = np.log(p / (1.0 - p))[:, None]
    br = np.array(case["br"], dtype=np.float64)
    Wv = np.array(case["Wv_ln3"], dtype=np.float64) * ln3
    v, r = O.value_routed(x, Wr, br, Wv, case["k"], case["scale"])
    assert r["idx"].tolist() == case["idx"]
    np.testing.assert_allclose(r["w"], np.array(case["w"]), rtol=0, atol=1e-14)
    np.testing.assert_allclose(v, np.array(case["v_ln3"]) * ln3, rtol=0, atol=1e-14)


def test_sigmoid_silu_closed_forms():
    ln3 = math.log(3.0)
    assert O.sigmoid(np.array(0.0)) == 0.5
    np.testing.assert_allclose(O.sigmoid(np.array([ln3, -ln3])), [0.75, 0.25], atol=1e-15)
    np.testing.assert_allclose(O.silu(np.array([0.0, ln3, -ln3])), [0.0, 0.75 * ln3, -0.25 * ln3],
                               atol=1e-15)
    # SiLU(-z) = SiLU(z) - z, and SiLU(z) -> z for large z.
    z = np.linspace(-8, 8, 33)
    np.testing.assert_allclose(O.silu(-z), O.silu(z) - z, atol=1e-14)
    assert abs(O.silu(np.array(40.0)) - 40.0) < 1e-12


# ---------------------------------------------------------------------------
# Numbers printed by the pages (tests/golden/page_counts.json)
# ---------------------------------------------------------------------------


def test_page_counts():
    g = _load("page_counts.json")
    d, E, k = g["d_model"], g["n_experts"], g["top_k"]
    n = g["heads"] * g["head_dim"]
    assert n == 1024
    per_layer = O.expert_params_per_layer(E, d, n)
    assert round(per_layer / 1e6, 1) == g["expert_params_per_layer_rounded_M"]
    assert per_layer * g["mova_layers"] == g["expert_params_all_layers"]
    assert round(O.macs_per_token(d, n, k) / 1e6, 2) == g["macs_per_token_rounded_M"]
    assert round(O.expert_params_per_layer(1, d, n) / 1e6, 2) == g["dense_v_proj_params_rounded_M"]
    assert round(O.router_params(d, E) / 1e3) == g["router_params_rounded_K"]
    assert O.flops_per_token(d, n, k) == 2 * 10_485_760


def test_bf16_format():
    for hexbits, val in _load("bf16_patterns.json")["patterns"]:
        got = O.bf16_bits_to_f64(np.array([int(hexbits, 16)], dtype=np.uint16))[0]
        assert got == val and math.copysign(1.0, got) == math.copysign(1.0, val), hexbits


def test_f16_format():
    # Routing-given mode stores the weights in fp16 and uses them as they are.
    for hexbits, val in _load("f16_patterns.json")["patterns"]:
        a = np.array([int(hexbits, 16)], dtype=np.uint16).view(np.float16)
        got = O.to_f64(a, "f16")[0]
        assert got == val and math.copysign(1.0, got) == math.copysign(1.0, val), hexbits


# ---------------------------------------------------------------------------
# Identities of the method
# ---------------------------------------------------------------------------


def _rand_case(rng, T=5, d=12, E=8, n=6):
    x = rng.standard_normal((T, d))
    Wr = rng.standard_normal((E, d)) * 0.3
    br = rng.standard_normal(E) * 0.1
    Wv = rng.standard_normal((E, n, d)) / math.sqrt(d)
    return x, Wr, br, Wv


@pytest.mark.parametrize("k", [1, 2, 4])
def test_identical_experts_give_scaled_silu(k):
    """All experts equal W: the renormalised weights sum to 1, so
    v = scale * SiLU(W x) whatever the routing (checked with naive loops)."""
    rng = np.random.default_rng(1)
    x, Wr, br, _ = _rand_case(rng)
    d, E, n = x.shape[1], Wr.shape[0], 6
    W = rng.standard_normal((n, d)) / math.sqrt(d)
    Wv = np.broadcast_to(W, (E, n, d))
    v, _ = O.value_routed(x, Wr, br, Wv, k, 2.5)
    for t in range(x.shape[0]):
        h = _naive_matvec(W.tolist(), x[t].tolist())
        ref = [2.5 * _naive_silu(z) for z in h]
        np.testing.assert_allclose(v[t], ref, rtol=1e-13, atol=1e-13)


def test_single_expert_is_textbook_matvec():
    """E = 1, k = 1: v = scale * SiLU(W x) for a non-square W (catches a
    transposed expert operand)."""
    rng = np.random.default_rng(2)
    d, n = 7, 3
    x = rng.standard_normal((4, d))
    W = rng.standard_normal((1, n, d))
    v, r = O.value_routed(x, rng.standard_normal((1, d)), np.zeros(1), W, 1, 2.5)
    assert (r["idx"] == 0).all()
    np.testing.assert_allclose(r["w"], 2.5)
    for t in range(4):
        h = _naive_matvec(W[0].tolist(), x[t].tolist())
        np.testing.assert_allclose(v[t], [2.5 * _naive_silu(z) for z in h], rtol=1e-13)


def test_k_equals_E_selection_irrelevant():
    """k = E: every expert is selected, so the bias (which only steers the
    selection) cannot change the output."""
    rng = np.random.default_rng(3)
    x, Wr, br, Wv = _rand_case(rng)
    E = Wr.shape[0]
    v1, _ = O.value_routed(x, Wr, br, Wv, E, 2.5)
    v2, _ = O.value_routed(x, Wr, rng.standard_normal(E) * 5.0, Wv, E, 2.5)
    np.testing.assert_allclose(v1, v2, rtol=1e-13, atol=1e-13)


def test_weights_positive_and_sum_to_scale():
    rng = np.random.default_rng(4)
    x, Wr, br, _ = _rand_case(rng, T=50)
    r = O.route(x, Wr, br, 4, 2.5)
    assert (r["w"] > 0).all()
    np.testing.assert_allclose(r["w"].sum(axis=1), 2.5, rtol=1e-14)
    # Weights follow the unbiased sigmoid scores of the selected experts.
    for t in range(x.shape[0]):
        st = [1.0 / (1.0 + math.exp(-float(np.dot(x[t], Wr[e])))) for e in r["idx"][t]]
        np.testing.assert_allclose(r["w"][t], [2.5 * s / sum(st) for s in st], rtol=1e-12)


def test_weights_for_another_selection():
    # weights_for serves the parity tests when a near-tie admits a second
    # valid selection.  On the router's own selection it must give the
    # router's weights; on any selection, positive weights summing to the
    # scale, in the ratio of the selected unbiased scores.
    rng = np.random.default_rng(5)
    x, Wr, br, _ = _rand_case(rng, T=20)
    r = O.route(x, Wr, br, 4, 2.5)
    np.testing.assert_array_equal(O.weights_for(r["s"], r["idx"], 2.5), r["w"])
    alt = r["idx"].copy()
    alt[:, 3] = np.argsort(-r["b"], axis=1, kind="stable")[:, 4]  # the 5th expert instead of the 4th
    w = O.weights_for(r["s"], alt, 2.5)
    assert (w > 0).all()
    np.testing.assert_allclose(w.sum(axis=1), 2.5, rtol=1e-14)
    for t in range(x.shape[0]):
        s0 = 1.0 / (1.0 + math.exp(-float(np.dot(x[t], Wr[alt[t, 0]]))))
        for j in range(1, 4):
            sj = 1.0 / (1.0 + math.exp(-float(np.dot(x[t], Wr[alt[t, j]]))))
            assert math.isclose(w[t, j] / w[t, 0], sj / s0, rel_tol=1e-12)


def test_bias_shift_invariance():
    rng = np.random.default_rng(5)
    x, Wr, br, Wv = _rand_case(rng, T=20)
    v1, r1 = O.value_routed(x, Wr, br, Wv, 3, 2.5)
    v2, r2 = O.value_routed(x, Wr, br + 0.37, Wv, 3, 2.5)
    assert (r1["idx"] == r2["idx"]).all()
    np.testing.assert_allclose(v1, v2, rtol=1e-13)


# ---------------------------------------------------------------------------
# Selection against brute force
# ---------------------------------------------------------------------------


def _brute_top_k(b_row, k):
    """Best subset by sum of scores, lowest indices first among equals,
    then ordered by descending score (ties: lower index first)."""
    E = len(b_row)
    best = None
    for sub in itertools.combinations(range(E), k):
        key = (sum(b_row[e] for e in sub), [-e for e in sub])
        if best is None or key > best[0]:
            best = (key, sub)
    return sorted(best[1], key=lambda e: (-b_row[e], e))


@pytest.mark.parametrize("E,k", [(6, 1), (6, 2), (6, 3), (7, 4), (8, 4)])
def test_top_k_brute_force_random(E, k):
    rng = np.random.default_rng(10 + E * 10 + k)
    b = rng.standard_normal((40, E))
    got = O.select_top_k(b, k)
    for t in range(b.shape[0]):
        assert got[t].tolist() == _brute_top_k(b[t].tolist(), k)


@pytest.mark.parametrize("E,k", [(6, 2), (8, 4), (8, 3)])
def test_top_k_brute_force_ties(E, k):
    """Scores drawn from 3 values so that ties are everywhere: equal scores
    go to the lower expert index."""
    rng = np.random.default_rng(20 + E + k)
    b = rng.integers(0, 3, size=(60, E)).astype(np.float64) * 0.5
    got = O.select_top_k(b, k)
    for t in range(b.shape[0]):
        assert got[t].tolist() == _brute_top_k(b[t].tolist(), k)


def test_route_brute_force_end_to_end():
    """Tiny E, k: the whole route (logits by loops, sigmoid by math.exp,
    best subset by enumeration) against the oracle."""
    rng = np.random.default_rng(6)
    T, d, E, k = 12, 5, 6, 2
    x = rng.standard_normal((T, d))
    Wr = rng.standard_normal((E, d))
    br = rng.standard_normal(E) * 0.2
    r = O.route(x, Wr, br, k, 2.5)
    for t in range(T):
        s = [1.0 / (1.0 + math.exp(-sum(x[t, j] * Wr[e, j] for j in range(d)))) for e in range(E)]
        b = [s[e] + br[e] for e in range(E)]
        sel = _brute_top_k(b, k)
        assert r["idx"][t].tolist() == sel
        tot = sum(s[e] for e in sel)
        np.testing.assert_allclose(r["w"][t], [2.5 * s[e] / tot for e in sel], rtol=1e-12)


def test_combine_naive_loops():
    """The mixture against plain loops over tokens and slots, with the
    routing given (also the routing-given mode's definition)."""
    rng = np.random.default_rng(7)
    T, d, E, n, k = 6, 5, 4, 3, 2
    x = rng.standard_normal((T, d))
    Wv = rng.standard_normal((E, n, d))
    idx = np.array([rng.permutation(E)[:k] for _ in range(T)])
    w = rng.random((T, k)) + 0.1
    v = O.combine(x, idx, w, Wv)
    for t in range(T):
        acc = [0.0] * n
        for slot in range(k):
            h = _naive_matvec(Wv[idx[t, slot]].tolist(), x[t].tolist())
            for c in range(n):
                acc[c] += w[t, slot] * _naive_silu(h[c])
        np.testing.assert_allclose(v[t], acc, rtol=1e-13, atol=1e-14)


def test_gqa_shape_and_mapping():
    v = np.arange(3 * 1024, dtype=np.float64).reshape(3, 1024)
    g = O.as_gqa(v)
    assert g.shape == (3, 8, 128)
    for t, h, c in [(0, 0, 0), (1, 3, 5), (2, 7, 127)]:
        assert g[t, h, c] == v[t, h * 128 + c]


# ---------------------------------------------------------------------------
# Grouping by expert against a pure-Python brute force
# ---------------------------------------------------------------------------


@pytest.mark.parametrize("T,E,k", [(1, 4, 1), (7, 5, 2), (33, 8, 4), (50, 64, 4)])
def test_permutation_brute_force(T, E, k):
    rng = np.random.default_rng(T * 100 + E)
    idx = np.array([rng.permutation(E)[:k] for _ in range(T)])
    p = O.permutation(idx, E)
    flat = idx.reshape(-1).tolist()
    perm = []
    counts = []
    for e in range(E):
        mine = [f for f in range(len(flat)) if flat[f] == e]
        counts.append(len(mine))
        perm.extend(mine)
    assert p["counts"].tolist() == counts
    assert p["offsets"].tolist() == [sum(counts[:e]) for e in range(E + 1)]
    assert p["perm"].tolist() == perm
    for f in range(len(flat)):
        assert perm[p["pos"][f]] == f


def test_permutation_empty():
    p = O.permutation(np.zeros((0, 4), dtype=np.int64), 8)
    assert p["counts"].tolist() == [0] * 8
    assert p["offsets"].tolist() == [0] * 9
    assert p["perm"].size == 0 and p["pos"].size == 0


# ---------------------------------------------------------------------------
# Router partitions ("Implementation pitfalls": router numerics through the
# GEMM partitioning)
# ---------------------------------------------------------------------------


def _cancel_case(layout):
    """Expert 0's partial sums cancel; the rest have zero logits.  Returns
    (x (1, 8), Wr (3, 8), br (3,)) in fp64; values exactly representable."""
    x = np.zeros((1, 8))
    Wr = np.zeros((3, 8))
    for j, xv, wv in layout:
        x[0, j] = xv
        Wr[0, j] = wv
    br = np.array([0.0, 0.1, -1.0])
    return x, Wr, br


def test_partitioned_logits_round_each_half():
    """2^25 lands in the first half and -2^25 + 1 in the second: the second
    half's fp32 sum rounds -(2^25 - 1) to -2^25 (a tie, to even), so the
    partitioned logit is 0 while the exact one is 1 -- and the selection
    follows (expert 1's biased score 0.6 beats sigmoid(0) = 0.5 but not
    sigmoid(1) = 0.731)."""
    x, Wr, br = _cancel_case([(0, 2.0 ** 12, 2.0 ** 13), (4, 2.0 ** 12, -2.0 ** 13), (5, 1.0, 1.0)])
    assert O.router_logits(x, Wr)[0].tolist() == [1.0, 0.0, 0.0]
    assert O.router_logits_partitioned(x, Wr, 2)[0].tolist() == [0.0, 0.0, 0.0]
    plain = O.route(x, Wr, br, 2, 2.5)
    part = O.route(x, Wr, br, 2, 2.5, partitions=2)
    assert plain["idx"].tolist() == [[0, 1]]
    assert part["idx"].tolist() == [[1, 0]]
    np.testing.assert_allclose(part["w"], [[1.25, 1.25]], rtol=0, atol=1e-15)
    s1 = 1.0 / (1.0 + math.exp(-1.0))
    np.testing.assert_allclose(plain["w"], [[2.5 * s1 / (s1 + 0.5), 2.5 * 0.5 / (s1 + 0.5)]], rtol=1e-15)


def test_partitioned_logits_split_at_the_middle():
    """2^25 and -2^25 both in the first half, +1 in its last place: the first
    half sums exactly to 1, so the partitioned logit is 1; a split after two
    elements would round 1 - 2^25 to -2^25 and give 0."""
    x, Wr, br = _cancel_case([(0, 2.0 ** 12, 2.0 ** 13), (2, 2.0 ** 12, -2.0 ** 13), (3, 1.0, 1.0)])
    assert O.router_logits_partitioned(x, Wr, 2)[0].tolist() == [1.0, 0.0, 0.0]
    quarters = (np.float32(x[0, :2] @ Wr[0, :2]) + np.float32(x[0, 2:4] @ Wr[0, 2:4]))
    assert float(quarters) == 0.0  # the wrong split point gives another answer


def test_partitioned_logits_are_fp32_within_rounding():
    """On random inputs the partitioned logits are fp32 numbers within the
    three roundings of the exact logits (each half, then their sum)."""
    rng = np.random.default_rng(5)
    x = rng.standard_normal((16, 256)).astype(np.float32).astype(np.float64)
    Wr = (rng.standard_normal((8, 256)) * 0.02).astype(np.float32).astype(np.float64)
    exact = O.router_logits(x, Wr)
    part = O.router_logits_partitioned(x, Wr, 2)
    assert (part.astype(np.float32).astype(np.float64) == part).all()
    h0 = np.abs(x[:, :128] @ Wr[:, :128].T)
    h1 = np.abs(x[:, 128:] @ Wr[:, 128:].T)
    eps = 2.0 ** -24
    bound = eps * (h0 + h1) + eps * np.abs(part) + 1e-300
    assert (np.abs(part - exact) <= bound * 1.0000001).all()
    assert not (part == exact).all()  # the rounding is really there
    np.testing.assert_array_equal(O.route(x, Wr, np.zeros(8), 2, 2.5)["logits"], exact)
    np.testing.assert_array_equal(O.route(x, Wr, np.zeros(8), 2, 2.5, partitions=2)["logits"], part)


# ---------------------------------------------------------------------------
# Attend: the PV product over rematerialised values (Deep-dive, Section 4,
# Option B)
# ---------------------------------------------------------------------------


def test_attend_brute_force_loops():
    """attend against scalar loops written independently of combine/as_gqa:
    every position, slot, expert row and query head summed by hand."""
    rng = np.random.default_rng(7)
    L, d, E, k, n, H = 3, 5, 3, 2, 256, 4  # 2 KV heads, 2 query heads each
    x = rng.normal(size=(L, d))
    Wv = rng.normal(size=(E, n, d)) * 0.5
    idx = np.array([[0, 2], [1, 0], [2, 1]])
    w = rng.uniform(0.2, 1.5, size=(L, k))
    p = rng.uniform(size=(H, L))
    o = O.attend(x, idx, w, Wv, p)
    for h in range(H):
        g = h // 2  # H / (n / 128) = 2 query heads per KV head
        for c in range(128):
            acc = 0.0
            for l in range(L):
                vl = 0.0
                for s in range(k):
                    hv = sum(Wv[idx[l, s], g * 128 + c, j] * x[l, j] for j in range(d))
                    vl += w[l, s] * hv / (1.0 + math.exp(-hv))
                acc += p[h, l] * vl
            assert abs(o[h, c] - acc) <= 1e-12 * max(1.0, abs(acc))


def test_attend_one_hot_reads_one_value_row():
    """With all of a head's probability on position j, o[h] is row j of the
    value tensor in the head's KV group; query heads 2g and 2g + 1 share KV
    head g (a mapping h % (n/128) would swap groups and fail)."""
    rng = np.random.default_rng(8)
    L, d, E, k, n = 5, 6, 4, 2, 512  # 4 KV heads
    x = rng.normal(size=(L, d))
    Wv = rng.normal(size=(E, n, d))
    idx = rng.integers(0, E, size=(L, k))
    w = rng.uniform(0.1, 1.0, size=(L, k))
    H = 8
    p = np.zeros((H, L))
    js = [4, 1, 3, 0, 2, 2, 1, 4]
    for h, j in enumerate(js):
        p[h, j] = 1.0
    o = O.attend(x, idx, w, Wv, p)
    V = O.combine(x, idx, w, Wv).reshape(L, 4, 128)
    for h, j in enumerate(js):
        np.testing.assert_allclose(o[h], V[j, h // 2], rtol=0, atol=1e-13)
    assert not np.allclose(o[1], V[js[1], 1 % 4])  # the other mapping differs


def test_attend_linear_in_probabilities():
    """o is linear in probs (the attention weights enter once, outside the
    SiLU)."""
    rng = np.random.default_rng(9)
    L, d, E, k, n, H = 6, 4, 3, 2, 128, 2
    x = rng.normal(size=(L, d))
    Wv = rng.normal(size=(E, n, d))
    idx = rng.integers(0, E, size=(L, k))
    w = rng.uniform(0.1, 1.0, size=(L, k))
    a = rng.uniform(size=(H, L))
    b = rng.uniform(size=(H, L))
    np.testing.assert_allclose(O.attend(x, idx, w, Wv, 2.0 * a - b),
                               2.0 * O.attend(x, idx, w, Wv, a) - O.attend(x, idx, w, Wv, b),
                               rtol=1e-12, atol=1e-12)
