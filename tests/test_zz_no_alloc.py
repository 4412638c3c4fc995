"""The workspace-free entry point, for callers that cannot give the library device memory
(plugins whose host forbids cudaMalloc while serving, programs with all device memory reserved
at start-up). Its results must agree with moe_decode_forward on a caller workspace.

This file is collected last on purpose; it builds its own layer, so it also runs alone in a
fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

from mixture_experts_decode_gemv_b200 import binding as B
from mixture_experts_decode_gemv_b200.device_layer import DeviceLayer, make_cfg
from mixture_experts_decode_gemv_b200.synthetic import CONFIGS, LayerConfig, SyntheticLayer

pytestmark = pytest.mark.gpu

TOL = 2e-3


def _close(got: torch.Tensor, want: torch.Tensor) -> None:
    g = got.double().cpu().numpy()
    w = want.double().cpu().numpy()
    lim = TOL * np.maximum(1.0, np.abs(w))
    assert np.all(np.abs(g - w) <= lim), float(np.max(np.abs(g - w) / lim))


def test_no_alloc_matches_workspace_entry_point_on_two_calls_in_a_row():
    cfg = CONFIGS["qwen3_6_35b_a3b"]          # NVFP4 experts + sigmoid-gated shared expert
    lay = SyntheticLayer(cfg)
    dev = DeviceLayer(lay)
    m = 8
    xa = dev.x_to_device(lay.x(m, offset=0))
    xb = dev.x_to_device(lay.x(m, offset=m))
    stream = torch.cuda.current_stream()

    ws = dev.new_workspace(m)
    want_a, want_b = dev.new_out(m), dev.new_out(m)
    dev.forward(xa, want_a, ws)
    dev.forward(xb, want_b, ws)

    got_a = torch.full_like(want_a, float("nan"))
    got_b = torch.full_like(want_b, float("nan"))
    for x, out in ((xa, got_a), (xb, got_b)):      # two calls back to back, no sync between
        B.moe_decode_forward_no_alloc(dev.c, m, x, dev.router_w, dev.expert_bias, dev.routed,
                                      dev.shared, dev.shared_gate_w, out, stream)
    torch.cuda.synchronize()
    _close(got_a, want_a)
    _close(got_b, want_b)
    assert not torch.equal(got_a, got_b)


def test_no_alloc_refuses_a_layer_larger_than_its_scratch():
    big = LayerConfig(name="big", hidden=8192, num_experts=256, top_k=8, moe_inter=8192, index=999)
    c = make_cfg(big)
    need = B.moe_workspace_bytes(c, 64)
    assert need > B.MOE_NO_ALLOC_SCRATCH_BYTES
    fake = 0x7F0000000000
    mats = []
    for n, k in ((8192, 8192), (8192, 8192), (8192, 8192)):
        mm = B.moe_matrix()
        mm.format = B.MOE_FMT_BF16
        mm.packed = fake
        mm.expert_stride = n * k * 2
        mats.append(mm)
    table = B.moe_expert_table(*mats)
    rc = B.lib.moe_decode_forward_no_alloc(ctypes.byref(c), 64, fake, fake, None,
                                           ctypes.byref(table), None, None, fake, None)
    assert rc == B.MOE_ERR_WORKSPACE
