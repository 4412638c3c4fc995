"""Pins of the oracle's expert math and whole-layer evaluation (CPU only)."""
import math

import numpy as np
import pytest

from oracle import moe_ref as ref
from mixture_experts_decode_gemv_b200.synthetic import (
    CONFIGS, GAP_MIN, LayerConfig, POOL_ROWS, SyntheticLayer)

pytestmark = pytest.mark.cpu


def sigmoid_tanh(z):
    """Independent formulation: sigmoid(z) = (1 + tanh(z/2)) / 2."""
    return 0.5 * (1.0 + np.tanh(0.5 * np.asarray(z, dtype=np.float64)))


def test_silu_closed_form_points():
    assert ref.silu(0.0) == 0.0
    assert ref.sigmoid(0.0) == 0.5
    # sigmoid(1) = e / (1 + e)
    np.testing.assert_allclose(ref.silu(1.0), math.e / (1 + math.e), rtol=1e-15)
    np.testing.assert_allclose(ref.silu(-2.0), -2.0 / (1 + math.e ** 2), rtol=1e-15)
    z = np.linspace(-30, 30, 1001)
    # the tanh form cancels for very negative z, hence the absolute floor
    np.testing.assert_allclose(ref.silu(z), z * sigmoid_tanh(z), rtol=1e-13, atol=1e-14)
    # asymptotes: silu(z) -> z for large z, -> 0 for very negative z
    assert abs(ref.silu(50.0) - 50.0) < 1e-15 * 50
    assert abs(ref.silu(-50.0)) < 1e-19


def test_swiglu_identity_matrices():
    x = np.array([0.0, 1.0, -2.0, 3.5])
    eye = np.eye(4)
    y = ref.swiglu_expert(eye, eye, eye, x)
    np.testing.assert_allclose(y, x * x * sigmoid_tanh(x), rtol=1e-14, atol=0)
    # permutation matrices: down undoes gate/up's permutation
    P = eye[[2, 0, 3, 1]]
    y = ref.swiglu_expert(P, P, P.T, x)
    np.testing.assert_allclose(y, x * x * sigmoid_tanh(x), rtol=1e-14, atol=0)


def test_weight_site_linearity_and_non_homogeneity():
    rng = np.random.default_rng(11)
    wg, wu, wd = (rng.standard_normal((6, 5)), rng.standard_normal((6, 5)),
                  rng.standard_normal((5, 6)))
    x = rng.standard_normal(5)
    w = 0.37
    xin, omega = ref.routed_slot(x, w, True)
    # the gate/up projections are linear: scaling the input == scaling g and u
    act_scaled_out = ref.silu(w * (wg @ x)) * (w * (wu @ x))
    np.testing.assert_allclose(wd @ act_scaled_out, ref.swiglu_expert(wg, wu, wd, xin),
                               rtol=1e-12, atol=1e-12)
    # but SwiGLU is not homogeneous: before-FFN differs from after-FFN unless w == 1
    before = omega * ref.swiglu_expert(wg, wu, wd, xin)
    xin2, omega2 = ref.routed_slot(x, w, False)
    after = omega2 * ref.swiglu_expert(wg, wu, wd, xin2)
    assert np.max(np.abs(before - after)) > 1e-3
    xin1, _ = ref.routed_slot(x, 1.0, True)
    np.testing.assert_array_equal(ref.swiglu_expert(wg, wu, wd, xin1),
                                  ref.swiglu_expert(wg, wu, wd, x))


SMALL = [
    LayerConfig(name="s_f32_softmax", hidden=64, num_experts=6, top_k=2, moe_inter=32,
                fmt="f32", x_dtype="f32", index=100),
    LayerConfig(name="s_bf16_sig_bias", hidden=64, num_experts=8, top_k=3, moe_inter=32,
                fmt="bf16", routing="sigmoid", has_expert_bias=True, routed_scaling_factor=1.7,
                index=101),
    LayerConfig(name="s_q4", hidden=128, num_experts=5, top_k=2, moe_inter=64,
                fmt="q4_affine_g64", routing="sigmoid", has_expert_bias=True, index=102),
    LayerConfig(name="s_nvfp4_shared_gate", hidden=64, num_experts=9, top_k=3, moe_inter=32,
                shared_inter=32, shared_kind="sigmoid_gate", fmt="nvfp4", index=103),
    LayerConfig(name="s_before_ffn", hidden=64, num_experts=4, top_k=1, moe_inter=32,
                shared_inter=64, shared_kind="plain", routing="sigmoid",
                select_on_raw_logits=True, norm_topk_prob=False, weight_before_ffn=True,
                index=104),
    LayerConfig(name="s_softmax_nonorm", hidden=32, num_experts=4, top_k=4, moe_inter=16,
                norm_topk_prob=False, index=105),
]


def _layer(cfg):
    lay = SyntheticLayer(cfg)
    lay.key_fn = ref.selection_key_fn(lay)
    return lay


def _dense_brute_force(cfg, lay, x):
    """Evaluate every expert on every row, mask to the routed set, and sum (no gathering)."""
    olay = ref.OracleLayer(lay, cache_experts=64)
    rt = ref.route(olay, x)
    x64 = rt["x64"]
    m = x64.shape[0]
    out = np.zeros((m, cfg.hidden))
    for r in range(m):
        mask = np.zeros(cfg.num_experts)
        for s in range(cfg.top_k):
            mask[rt["idx"][r, s]] = rt["w"][r, s]
        acc = np.zeros(cfg.hidden)
        for e in range(cfg.num_experts):
            wg, wu, wd = olay.expert(e)
            if cfg.weight_before_ffn:
                xin, scale_out = mask[e] * x64[r], 1.0 if mask[e] != 0 else 0.0
            else:
                xin, scale_out = x64[r], mask[e]
            g = wg @ xin
            act = g * sigmoid_tanh(g) * (wu @ xin)
            acc += scale_out * (wd @ act)
        if cfg.has_shared:
            sg, su, sd = olay.shared()
            g = sg @ x64[r]
            sh = sd @ (g * sigmoid_tanh(g) * (su @ x64[r]))
            if cfg.shared_kind == "sigmoid_gate":
                gw = ref.decode_activations(lay.shared_gate_w(), cfg.x_dtype)
                sh = sh * sigmoid_tanh(gw @ x64[r])
            acc += sh
        out[r] = acc
    return out


@pytest.mark.parametrize("cfg", SMALL, ids=lambda c: c.name)
def test_sparse_equals_dense_brute_force(cfg):
    lay = _layer(cfg)
    x = lay.x(8)
    out, aux = ref.moe_forward(ref.OracleLayer(lay, cache_experts=64), x)
    dense = _dense_brute_force(cfg, lay, x)
    scale = max(1.0, float(np.max(np.abs(dense))))
    np.testing.assert_allclose(out, dense, rtol=0, atol=1e-12 * scale)


@pytest.mark.parametrize("cfg", SMALL, ids=lambda c: c.name)
def test_rows_do_not_depend_on_m_and_permute(cfg):
    lay = _layer(cfg)
    olay = ref.OracleLayer(lay, cache_experts=64)
    full, _ = ref.moe_forward(olay, lay.x(POOL_ROWS))
    for r in (0, 5, 17, 63):
        one, _ = ref.moe_forward(olay, lay.x(1, offset=r))
        np.testing.assert_array_equal(one[0], full[r])
    perm = np.random.default_rng(3).permutation(POOL_ROWS)
    permuted, _ = ref.moe_forward(olay, lay.x(POOL_ROWS)[perm])
    np.testing.assert_array_equal(permuted, full[perm])


def test_shared_gate_closed_form():
    # with the routed experts' down projections zeroed, the output is gamma * shared(x)
    cfg = SMALL[3]
    lay = _layer(cfg)
    for e in range(cfg.num_experts):
        d = lay.routed_expert(e, "down")
        d.data[...] = 0
    x = lay.x(4)
    out, aux = ref.moe_forward(ref.OracleLayer(lay, cache_experts=64), x)
    olay = ref.OracleLayer(lay)
    x64 = ref.decode_activations(x, cfg.x_dtype)
    sg, su, sd = olay.shared()
    gw = ref.decode_activations(lay.shared_gate_w(), cfg.x_dtype)
    for r in range(4):
        g = sg @ x64[r]
        want = sigmoid_tanh(gw @ x64[r]) * (sd @ (g * sigmoid_tanh(g) * (su @ x64[r])))
        np.testing.assert_allclose(out[r], want, rtol=1e-13, atol=1e-14)
        np.testing.assert_allclose(aux["gamma"][r], sigmoid_tanh(gw @ x64[r]), rtol=1e-15)


def test_single_expert_layer_is_the_expert():
    cfg = LayerConfig(name="one", hidden=32, num_experts=1, top_k=1, moe_inter=16, fmt="f32",
                      x_dtype="f32", index=110)
    lay = SyntheticLayer(cfg)
    x = lay.x(3)
    out, aux = ref.moe_forward(ref.OracleLayer(lay), x)
    wg, wu, wd = ref.OracleLayer(lay).expert(0)
    for r in range(3):
        xr = x[r].astype(np.float64)
        g = wg @ xr
        np.testing.assert_allclose(out[r], wd @ (g * sigmoid_tanh(g) * (wu @ xr)),
                                   rtol=1e-13, atol=1e-14)
    assert np.all(aux["w"] == 1.0)


@pytest.mark.parametrize("name", list(CONFIGS))
def test_published_shapes_meet_the_gap_rule(name):
    cfg = CONFIGS[name]
    lay = SyntheticLayer(cfg)
    key_fn = ref.selection_key_fn(lay)
    lay.key_fn = key_fn
    x = lay.x_pool()
    assert x.shape == (POOL_ROWS, cfg.hidden)
    k = cfg.top_k
    for r in range(POOL_ROWS):
        keys = np.sort(key_fn(x[r]))[::-1][: min(k + 1, cfg.num_experts)]
        assert np.min(keys[:-1] - keys[1:]) >= GAP_MIN


def test_gelu_tanh_matches_the_library_and_closed_forms():
    import torch
    assert ref.gelu_tanh(0.0) == 0.0
    z = np.linspace(-12, 12, 2401)
    lib = torch.nn.functional.gelu(torch.tensor(z, dtype=torch.float64), approximate="tanh")
    np.testing.assert_allclose(ref.gelu_tanh(z), lib.numpy(), rtol=1e-13, atol=1e-15)
    # odd part: gelu(z) - gelu(-z) = z
    np.testing.assert_allclose(ref.gelu_tanh(z) - ref.gelu_tanh(-z), z, rtol=0, atol=1e-12)


def test_geglu_expert_with_identity_matrices():
    x = np.array([0.0, 1.0, -2.0, 3.5])
    eye = np.eye(4)
    y = ref.swiglu_expert(eye, eye, eye, x, "geglu")
    np.testing.assert_allclose(y, ref.gelu_tanh(x) * x, rtol=1e-15)
    assert not np.allclose(y, ref.swiglu_expert(eye, eye, eye, x))
