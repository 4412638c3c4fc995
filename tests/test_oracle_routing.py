"""Pins of the oracle's routing, weight-site and grouping steps (CPU only).

Each test checks the oracle against something other than itself: the worked example on the
frink-models page, a library routine (scipy's softmax), brute force over tiny inputs, or a
closed-form property that a dropped term, wrong index or transposed operand would break.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
from scipy.special import softmax as scipy_softmax

from oracle import moe_ref as ref
from mixture_experts_decode_gemv_b200.synthetic import LayerConfig

pytestmark = pytest.mark.cpu


def cfg_of(**kw):
    base = dict(name="t", hidden=8, num_experts=6, top_k=2, moe_inter=4)
    base.update(kw)
    return LayerConfig(**base)


# ---- routed-weight site: the worked example ---------------------------------------------------

def test_routed_slot_worked_example(golden_dir):
    with open(os.path.join(golden_dir, "routed_slot_worked_example.json")) as f:
        g = json.load(f)
    x = np.array(g["x"])
    xin, w = ref.routed_slot(x, g["w"], False)
    np.testing.assert_array_equal(xin, g["after_ffn"]["input"])
    assert w == g["after_ffn"]["weight"]
    xin, w = ref.routed_slot(x, g["w"], True)
    np.testing.assert_array_equal(xin, g["before_ffn"]["input"])
    assert w == g["before_ffn"]["weight"]
    for arch, flag in g["weight_before_ffn"].items():
        assert ref.weight_before_ffn(arch) is flag


# ---- top-k -------------------------------------------------------------------------------------

def _is_valid_topk(keys, ids, k):
    """Brute-force definition: the selected set holds the k best (key, -id) pairs and is listed in
    descending key order with ties to the lower id."""
    ranked = [(-keys[e], e) for e in range(len(keys))]
    chosen = sorted(ranked[e] for e in ids)
    rest = [ranked[e] for e in range(len(keys)) if e not in ids]
    if len(set(ids)) != k:
        return False
    if rest and max(chosen) > min(rest):
        return False
    return [ranked[e] for e in ids] == chosen


def test_topk_brute_force_with_ties():
    rng = np.random.default_rng(1)
    for trial in range(300):
        E = int(rng.integers(1, 9))
        k = int(rng.integers(1, E + 1))
        keys = rng.integers(0, 3, size=E).astype(np.float64)  # many ties
        ids = ref.select_top_k(keys, k)
        assert _is_valid_topk(list(keys), ids, k), (keys, ids)
        # exhaustive: among all k-subsets, the chosen set is the lexicographically best
        best = max(itertools.combinations(range(E), k),
                   key=lambda c: sorted(((keys[e], -e) for e in c), reverse=True))
        assert sorted(ids) == sorted(best)


def test_topk_on_sigmoid_equals_topk_on_raw_logits():
    rng = np.random.default_rng(2)
    c_raw = cfg_of(routing="sigmoid", select_on_raw_logits=True, norm_topk_prob=False, top_k=3,
                   num_experts=16)
    c_sig = c_raw.replace(select_on_raw_logits=False)
    for _ in range(200):
        l = rng.standard_normal(16) * 3
        a = ref.select_top_k(ref.selection_keys(l, c_raw, None), 3)
        b = ref.select_top_k(ref.selection_keys(l, c_sig, None), 3)
        assert a == b
    # and the weights are the sigmoid of the selected logits, un-normalised
    l = np.array([0.0, 2.0, -1.0, 1.0])
    ids, w = ref.route_row(l, cfg_of(num_experts=4, top_k=2, routing="sigmoid",
                                     select_on_raw_logits=True, norm_topk_prob=False), None)
    assert ids == [1, 3]
    np.testing.assert_allclose(w, [1 / (1 + math.exp(-2.0)), 1 / (1 + math.exp(-1.0))],
                               rtol=0, atol=1e-15)


def test_biased_selection_unbiased_weights():
    l = np.array([2.0, 1.0, 0.0, -1.0])
    bias = np.array([0.0, 0.0, 3.0, 0.0], dtype=np.float32)
    c = cfg_of(num_experts=4, top_k=2, routing="sigmoid", has_expert_bias=True,
               norm_topk_prob=True, routed_scaling_factor=2.5)
    ids, w = ref.route_row(l, c, bias)
    # the bias moves expert 2 into the set; the unbiased ranking would be [0, 1]
    assert ids == [2, 0]
    s2, s0 = 0.5, 1 / (1 + math.exp(-2.0))
    np.testing.assert_allclose(w, [2.5 * s2 / (s2 + s0), 2.5 * s0 / (s2 + s0)], atol=1e-15)
    # zero bias reduces to plain sigmoid top-k
    ids0, w0 = ref.route_row(l, c, np.zeros(4, dtype=np.float32))
    ids1, w1 = ref.route_row(l, c.replace(has_expert_bias=False), None)
    assert ids0 == ids1 == [0, 1]
    np.testing.assert_array_equal(w0, w1)


def test_normalised_weights_sum_to_one_then_scale():
    rng = np.random.default_rng(3)
    for routing in ("softmax", "sigmoid"):
        for rsf in (1.0, 2.5):
            c = cfg_of(num_experts=32, top_k=5, routing=routing, norm_topk_prob=True,
                       routed_scaling_factor=rsf)
            for _ in range(50):
                l = rng.standard_normal(32)
                _, w = ref.route_row(l, c, None)
                assert abs(w.sum() - np.float32(rsf)) <= 1e-14 * max(1.0, rsf)


def test_softmax_k_equals_E_is_plain_softmax():
    rng = np.random.default_rng(4)
    c = cfg_of(num_experts=7, top_k=7, routing="softmax", norm_topk_prob=True)
    for _ in range(20):
        l = rng.standard_normal(7) * 2
        ids, w = ref.route_row(l, c, None)
        np.testing.assert_allclose(w, scipy_softmax(l)[ids], rtol=1e-14, atol=0)
        # slot order is descending probability
        assert list(ids) == list(np.argsort(-l, kind="stable"))


def test_softmax_without_norm_is_probability_over_all_experts():
    rng = np.random.default_rng(5)
    c = cfg_of(num_experts=12, top_k=3, routing="softmax", norm_topk_prob=False)
    l = rng.standard_normal(12)
    ids, w = ref.route_row(l, c, None)
    np.testing.assert_allclose(w, scipy_softmax(l)[ids], rtol=1e-14, atol=0)
    assert w.sum() < 1.0


def test_top1_normalised_weight_is_one():
    rng = np.random.default_rng(6)
    for routing in ("softmax", "sigmoid"):
        c = cfg_of(num_experts=9, top_k=1, routing=routing, norm_topk_prob=True)
        _, w = ref.route_row(rng.standard_normal(9), c, None)
        assert w[0] == 1.0


# ---- grouping by expert ------------------------------------------------------------------------

def _counting_sort(flat, E):
    """Hand-written stable counting sort (independent of numpy's argsort)."""
    buckets = [[] for _ in range(E)]
    for p, e in enumerate(flat):
        buckets[e].append(p)
    order = [p for b in buckets for p in b]
    offsets = [0]
    for b in buckets:
        offsets.append(offsets[-1] + len(b))
    return order, offsets


def test_grouping_matches_counting_sort():
    rng = np.random.default_rng(8)
    for _ in range(200):
        E = int(rng.integers(1, 20))
        k = int(rng.integers(1, min(E, 8) + 1))
        m = int(rng.integers(1, 9))
        idx = np.stack([rng.choice(E, size=k, replace=False) for _ in range(m)])
        g = ref.group_by_expert(idx, E)
        order, offsets = _counting_sort(list(idx.ravel()), E)
        assert list(g["sorted_pairs"]) == order
        assert list(g["expert_offsets"]) == offsets
        te = m * k
        assert g["expert_offsets"][-1] == te
        tp = g["token_to_perm"]
        assert list(tp[g["sorted_pairs"]]) == list(range(te))
        assert list(g["sorted_pairs"][tp]) == list(range(te))
        active = [e for e in range(E) if offsets[e + 1] > offsets[e]]
        assert list(g["active"]) == active
        assert g["active_count"] == len(active) <= min(te, E)


# ---- sqrt-softplus router ----------------------------------------------------------------------

def test_sqrtsoftplus_closed_forms_and_library_softplus():
    import torch
    # softplus(0) = ln 2, so the score at 0 is sqrt(ln 2)
    assert ref.sqrtsoftplus(0.0) == math.sqrt(math.log(2.0))
    z = np.linspace(-40, 40, 801)
    # torch switches to the identity above `threshold` (default 20): move it out of the way
    lib = torch.nn.functional.softplus(torch.tensor(z, dtype=torch.float64), threshold=1e4).numpy()
    np.testing.assert_allclose(ref.softplus(z), lib, rtol=1e-14, atol=1e-300)
    # softplus(z) - softplus(-z) = z; large z: score -> sqrt(z); very negative z: score -> e^(z/2)
    np.testing.assert_allclose(ref.softplus(z) - ref.softplus(-z), z, rtol=0, atol=1e-12)
    np.testing.assert_allclose(ref.sqrtsoftplus(60.0), math.sqrt(60.0), rtol=1e-15)
    np.testing.assert_allclose(ref.sqrtsoftplus(-60.0), math.exp(-30.0), rtol=1e-12)


def test_sqrtsoftplus_routing_selects_like_raw_logits_and_weights_by_score():
    rng = np.random.default_rng(11)
    cfg = cfg_of(num_experts=16, top_k=4, routing="sqrtsoftplus", norm_topk_prob=False)
    for _ in range(50):
        l = rng.standard_normal(16) * 3
        ids, w = ref.route_row(l, cfg, None)
        assert ids == list(np.argsort(-l, kind="stable")[:4])     # an increasing score
        np.testing.assert_allclose(w, np.sqrt(np.log1p(np.exp(l[ids]))), rtol=1e-14)
    cfg_n = cfg_of(num_experts=16, top_k=4, routing="sqrtsoftplus", norm_topk_prob=True,
                   routed_scaling_factor=2.0)
    ids, w = ref.route_row(l, cfg_n, None)
    np.testing.assert_allclose(w.sum(), 2.0, rtol=1e-14)


def test_sqrtsoftplus_bias_changes_the_set_not_the_weights():
    cfg = cfg_of(num_experts=4, top_k=1, routing="sqrtsoftplus", has_expert_bias=True,
                 norm_topk_prob=False)
    l = np.array([0.5, 0.4, -1.0, 0.0])
    bias = np.array([0.0, 0.5, 0.0, 0.0], dtype=np.float32)
    ids, w = ref.route_row(l, cfg, bias)
    assert ids == [1]                                           # 0.4 + bias beats 0.5
    np.testing.assert_allclose(w, [math.sqrt(math.log1p(math.exp(0.4)))], rtol=1e-15)


# ---- router GEMV: logits known in closed form ---------------------------------------------------

class _RouterOnly:
    """A layer source with only the routing inputs (router matrix, bias, shared-gate vector)."""

    def __init__(self, cfg, router_w, expert_bias=None, shared_gate_w=None):
        self.cfg = cfg
        self._wr, self._b, self._sg = router_w, expert_bias, shared_gate_w

    def router_w(self):
        return self._wr

    def expert_bias(self):
        return self._b

    def shared_gate_w(self):
        return self._sg


def _bf16_bits(v):
    """bfloat16 storage of values that bf16 holds exactly (small integers, powers of two)."""
    b = np.asarray(v, dtype=np.float32).view(np.uint32)
    assert np.all(b & 0xFFFF == 0), "value not exact in bf16"
    return (b >> 16).astype(np.uint16)


def test_router_logits_of_scaled_basis_rows():
    # E = 5 router rows over h = 12 inputs, row e = c_e * (unit vector at position p_e), so
    # logit[r, e] = c_e * x[r, p_e] exactly; m = 3 rows (m, E and h all differ, so a transposed
    # operand or a swapped index cannot produce the right [m, E] array).
    E, h, m = 5, 12, 3
    pos = [3, 0, 11, 7, 5]
    c = [2.0, -1.0, 0.5, 3.0, -4.0]
    wr = np.zeros((E, h), np.float32)
    for e in range(E):
        wr[e, pos[e]] = c[e]
    x = np.arange(m * h, dtype=np.float32).reshape(m, h) - 17.0   # integers -17 .. 18
    want = np.array([[c[e] * x[r, pos[e]] for e in range(E)] for r in range(m)])
    cfg = cfg_of(hidden=h, num_experts=E, top_k=2, x_dtype="f32", fmt="f32")
    rt = ref.route(ref.OracleLayer(_RouterOnly(cfg, wr)), x)
    assert rt["logits"].shape == (m, E)
    np.testing.assert_array_equal(rt["logits"], want)
    for r in range(m):
        order = sorted(range(E), key=lambda e: (-want[r, e], e))[:2]
        assert list(rt["idx"][r]) == order
        p = [math.exp(want[r, e]) for e in order]                 # renormalised softmax
        np.testing.assert_allclose(rt["w"][r], [v / sum(p) for v in p], rtol=1e-14)


def test_router_logits_of_integer_rows_in_bf16():
    # bf16 router rows and activations holding small integers: every logit is an integer that
    # plain Python integer arithmetic gives exactly.
    rng = np.random.default_rng(7)
    E, h, m = 7, 16, 4
    wr = rng.integers(-3, 4, size=(E, h))
    x = rng.integers(-5, 6, size=(m, h))
    want = [[sum(int(wr[e, j]) * int(x[r, j]) for j in range(h)) for e in range(E)]
            for r in range(m)]
    cfg = cfg_of(hidden=h, num_experts=E, top_k=3, x_dtype="bf16", fmt="bf16")
    rt = ref.route(ref.OracleLayer(_RouterOnly(cfg, _bf16_bits(wr))), _bf16_bits(x))
    np.testing.assert_array_equal(rt["logits"], np.array(want, dtype=np.float64))
    for r in range(m):
        assert list(rt["idx"][r]) == sorted(range(E), key=lambda e: (-want[r][e], e))[:3]


def test_router_sigmoid_bias_and_shared_gate_from_known_logits():
    # Logits set by basis rows; the bias changes the winner while the weights stay the unbiased
    # sigmoid scores; the shared gate is sigmoid of x at the gate vector's one non-zero position.
    E, h = 4, 6
    wr = np.zeros((E, h), np.float32)
    for e, (p, c) in enumerate([(1, 1.0), (4, 1.0), (0, 2.0), (5, -1.0)]):
        wr[e, p] = c
    x = np.array([[0.5, 1.0, -2.0, 0.0, 0.75, 0.25]], np.float32)
    logits = [1.0, 0.75, 1.0, -0.25]                 # x[1], x[4], 2 x[0], -x[5]
    bias = np.array([0.0, 0.5, -0.4, 0.0], np.float32)
    sg = np.zeros(h, np.float32)
    sg[2] = 0.5                                     # w_sg . x = -1
    cfg = cfg_of(hidden=h, num_experts=E, top_k=2, x_dtype="f32", fmt="f32", routing="sigmoid",
                 has_expert_bias=True, norm_topk_prob=False, routed_scaling_factor=2.0,
                 shared_inter=4, shared_kind="sigmoid_gate")
    rt = ref.route(ref.OracleLayer(_RouterOnly(cfg, wr, bias, sg)), x)
    np.testing.assert_array_equal(rt["logits"][0], logits)
    sig = [1.0 / (1.0 + math.exp(-v)) for v in logits]
    keys = [sig[e] + float(bias[e]) for e in range(E)]   # 0.731, 1.179, 0.331, 0.438
    assert list(rt["idx"][0]) == [1, 0]
    assert sorted(range(E), key=lambda e: -keys[e])[:2] == [1, 0]
    np.testing.assert_allclose(rt["w"][0], [2.0 * sig[1], 2.0 * sig[0]], rtol=1e-14)
    np.testing.assert_allclose(rt["gamma"], [1.0 / (1.0 + math.e)], rtol=1e-14)
