"""GPU parity of the whole layer (through the C ABI) against the float64 oracle.

Expert ids, weight order and every grouping array must match bit-exactly; outputs must satisfy
|out - ref| <= 2e-3 * max(1, |ref|) element by element. Inputs are the seeded synthetic layers
(activation rows redrawn until the top k+1 selection keys are >= 1e-3 apart).
"""
import numpy as np
import pytest
import torch

from mixture_experts_decode_gemv_b200 import binding as B
from mixture_experts_decode_gemv_b200.device_layer import DeviceLayer
from mixture_experts_decode_gemv_b200.synthetic import CONFIGS, LayerConfig, SyntheticLayer
from oracle import moe_ref as ref

pytestmark = pytest.mark.gpu

TOL = 2e-3

SMALL = {
    "tiny_m64": CONFIGS["tiny"],
    "ragged_bf16": LayerConfig(name="ragged_bf16", hidden=200, num_experts=5, top_k=3,
                               moe_inter=72, fmt="bf16", index=200),
    "ragged_q4_shared": LayerConfig(name="ragged_q4_shared", hidden=192, num_experts=6, top_k=2,
                                    moe_inter=192, shared_inter=64, shared_kind="plain",
                                    fmt="q4_affine_g64", routing="sigmoid", has_expert_bias=True,
                                    routed_scaling_factor=2.5, index=201),
    "ragged_nvfp4_gate": LayerConfig(name="ragged_nvfp4_gate", hidden=96, num_experts=7, top_k=3,
                                     moe_inter=160, shared_inter=96, shared_kind="sigmoid_gate",
                                     fmt="nvfp4", index=202),
    "k_equals_E": LayerConfig(name="k_equals_E", hidden=64, num_experts=4, top_k=4, moe_inter=32,
                              fmt="bf16", norm_topk_prob=False, index=203),
    "one_expert": LayerConfig(name="one_expert", hidden=128, num_experts=1, top_k=1,
                              moe_inter=64, fmt="f32", x_dtype="f32", index=204),
    "before_ffn_small": LayerConfig(name="before_ffn_small", hidden=256, num_experts=4, top_k=1,
                                    moe_inter=256, shared_inter=128, shared_kind="plain",
                                    fmt="bf16", routing="sigmoid", select_on_raw_logits=True,
                                    norm_topk_prob=False, weight_before_ffn=True, index=205),
    "sigmoid_raw_k2": LayerConfig(name="sigmoid_raw_k2", hidden=128, num_experts=12, top_k=2,
                                  moe_inter=64, fmt="nvfp4", routing="sigmoid",
                                  select_on_raw_logits=True, norm_topk_prob=True, index=206),
    "max_experts": LayerConfig(name="max_experts", hidden=64, num_experts=256, top_k=8,
                               moe_inter=32, fmt="bf16", index=207),
    "ragged_mxfp4": LayerConfig(name="ragged_mxfp4", hidden=160, num_experts=6, top_k=2,
                                moe_inter=96, shared_inter=64, shared_kind="plain", fmt="mxfp4",
                                routing="sigmoid", has_expert_bias=True,
                                routed_scaling_factor=1.5, index=208),
    "ragged_fp8_geglu": LayerConfig(name="ragged_fp8_geglu", hidden=112, num_experts=7, top_k=3,
                                    moe_inter=80, shared_inter=48, shared_kind="sigmoid_gate",
                                    fmt="fp8_e4m3", activation="geglu", index=209),
    "sqrtsoftplus_bias": LayerConfig(name="sqrtsoftplus_bias", hidden=128, num_experts=24,
                                     top_k=4, moe_inter=64, fmt="bf16", routing="sqrtsoftplus",
                                     has_expert_bias=True, routed_scaling_factor=2.5, index=210),
    "sqrtsoftplus_geglu_q4": LayerConfig(name="sqrtsoftplus_geglu_q4", hidden=192,
                                         num_experts=40, top_k=6, moe_inter=128,
                                         fmt="q4_affine_g64", routing="sqrtsoftplus",
                                         norm_topk_prob=False, activation="geglu", index=211),
    # hidden sizes that the chain's tensor-core gate/up tiles take (k-tiles of 4 chunks)
    "mma_fp8_geglu": LayerConfig(name="mma_fp8_geglu", hidden=128, num_experts=10, top_k=3,
                                 moe_inter=48, shared_inter=32, shared_kind="sigmoid_gate",
                                 fmt="fp8_e4m3", activation="geglu", index=212),
    "mma_mxfp4_bias": LayerConfig(name="mma_mxfp4_bias", hidden=256, num_experts=12, top_k=4,
                                  moe_inter=64, fmt="mxfp4", routing="sigmoid",
                                  has_expert_bias=True, index=213),
    "mma_bf16_ragged_rows": LayerConfig(name="mma_bf16_ragged_rows", hidden=64, num_experts=6,
                                        top_k=2, moe_inter=40, shared_inter=24,
                                        shared_kind="plain", fmt="bf16", weight_before_ffn=True,
                                        routing="sigmoid", select_on_raw_logits=True,
                                        norm_topk_prob=False, index=214),
}

_CACHE = {}


def layer_for(cfg: LayerConfig):
    if cfg.name not in _CACHE:
        lay = SyntheticLayer(cfg)
        lay.key_fn = ref.selection_key_fn(lay)
        lay.x_pool()
        _CACHE[cfg.name] = (lay, DeviceLayer(lay), ref.OracleLayer(lay, cache_experts=8))
    return _CACHE[cfg.name]


def run(dev: DeviceLayer, x_np: np.ndarray, out_dtype="f32"):
    m = x_np.shape[0]
    x = dev.x_to_device(x_np)
    ws = dev.new_workspace(m)
    out = dev.new_out(m)
    dev.forward(x, out, ws)
    torch.cuda.synchronize()
    rt = dev.read_routing(m, ws)
    status = dev.device_status(ws)
    return out.float().cpu().numpy(), rt, status


def check_routing(rt, aux, cfg, m):
    np.testing.assert_array_equal(rt["idx"], aux["idx"])
    np.testing.assert_allclose(rt["w"], aux["w"], rtol=2e-6, atol=1e-7)
    for key in ("sorted_pairs", "expert_offsets", "token_to_perm", "active"):
        np.testing.assert_array_equal(rt[key], aux[key], err_msg=key)
    assert rt["active_count"] == aux["active_count"]
    if cfg.shared_kind == "sigmoid_gate":
        np.testing.assert_allclose(rt["gamma"], aux["gamma"], rtol=2e-6, atol=1e-7)


def check_out(got, want):
    err = np.abs(got.astype(np.float64) - want)
    lim = TOL * np.maximum(1.0, np.abs(want))
    bad = err > lim
    assert not bad.any(), (f"{bad.sum()} of {bad.size} outside tolerance; worst err "
                           f"{err.max():.3g} at {np.unravel_index(err.argmax(), err.shape)}")


SMALL_M = (1, 3, 17, 64)


@pytest.mark.parametrize("name", list(SMALL))
@pytest.mark.parametrize("m", SMALL_M)
def test_small_layers_match_oracle(name, m):
    cfg = SMALL[name]
    lay, dev, olay = layer_for(cfg)
    x = lay.x(m)
    got, rt, status = run(dev, x)
    want, aux = ref.moe_forward(olay, x)
    assert status == B.MOE_OK
    check_routing(rt, aux, cfg, m)
    check_out(got, want)


# Published shapes at every m they are exercised at. The 64-row Llama-4 case checks a sample of
# rows (the oracle evaluates rows one by one); routing and grouping are checked for every row.
PUBLISHED = [(n, m) for n, c in CONFIGS.items() for m in c.m_list]
SAMPLE_ROWS = {("llama4_scout", 64): [0, 1, 13, 31, 42, 63], ("llama4_scout", 16): [0, 7, 15]}


@pytest.mark.parametrize("name,m", PUBLISHED)
def test_published_shapes_match_oracle(name, m):
    cfg = CONFIGS[name]
    lay, dev, olay = layer_for(cfg)
    x = lay.x(m)
    got, rt, status = run(dev, x)
    rows = SAMPLE_ROWS.get((name, m))
    want, aux = ref.moe_forward(olay, x, rows=rows)
    assert status == B.MOE_OK
    check_routing(rt, aux, cfg, m)
    check_out(got if rows is None else got[rows], want)


@pytest.mark.parametrize("name", ["ragged_nvfp4_gate", "ragged_q4_shared", "before_ffn_small",
                                  "mma_fp8_geglu", "mma_mxfp4_bias", "ragged_bf16",
                                  "ragged_mxfp4", "tiny_m64"])
def test_rows_do_not_depend_on_m(name):
    # A row's bits do not depend on the other rows of the call, nor on m (the grouped decode's
    # invariant): every launch path reduces each weight row in the same order.
    lay, dev, _ = layer_for(SMALL[name])
    full, _, _ = run(dev, lay.x(64))
    for r in (0, 9, 59):
        for n in (1, 2, 5):
            part, _, _ = run(dev, lay.x(n, offset=r))
            np.testing.assert_array_equal(part, full[r:r + n])


def test_repeated_calls_are_bit_identical_and_workspace_reusable():
    lay, dev, _ = layer_for(CONFIGS["qwen3_30b_a3b"])
    ws = dev.new_workspace(8)
    outs = []
    for m in (8, 1, 8, 4, 8):
        x = dev.x_to_device(lay.x(m))
        out = dev.new_out(m)
        dev.forward(x, out, ws)
        outs.append(out.cpu())
    torch.cuda.synchronize()
    assert torch.equal(outs[0], outs[2]) and torch.equal(outs[0], outs[4])
    assert torch.equal(outs[1][0], outs[3][0]) and torch.equal(outs[1][0], outs[0][0])
    assert torch.equal(outs[3], outs[0][:4])
    assert dev.device_status(ws) == B.MOE_OK


@pytest.mark.parametrize("name,m,path", [("qwen3_30b_a3b", 1, "auto"), ("lfm2_8b_a1b", 4, "auto"),
                                         ("qwen3_6_35b_a3b", 16, "auto"),
                                         ("qwen3_6_35b_a3b", 16, "chain"),
                                         ("ragged_fp8_geglu", 40, "auto")])
def test_no_write_outside_the_output_and_workspace(name, m, path):
    """Canaries: the call writes nothing in the 64 KB before and after its output and workspace."""
    cfg = SMALL.get(name) or CONFIGS[name]
    lay, dev, _ = layer_for(cfg)
    g = 65536  # guard bytes on each side (keeps the 256-byte alignment of both buffers)
    nb = dev.workspace_bytes(m)
    wbuf = torch.full((nb + 2 * g,), 0xA5, dtype=torch.uint8, device="cuda")
    ws = wbuf[g:g + nb]
    B.moe_workspace_init(ws, nb, torch.cuda.current_stream())
    out0 = dev.new_out(m)
    esz = out0.element_size()
    obuf = torch.full((out0.numel() * esz + 2 * g,), 0x5A, dtype=torch.uint8, device="cuda")
    out = obuf[g:g + out0.numel() * esz].view(out0.dtype).view(out0.shape)
    x = dev.x_to_device(lay.x(m))
    with _Path(path):
        dev.forward(x, out, ws)
    torch.cuda.synchronize()
    assert dev.device_status(ws) == B.MOE_OK
    assert bool((wbuf[:g] == 0xA5).all()) and bool((wbuf[g + nb:] == 0xA5).all())
    assert bool((obuf[:g] == 0x5A).all()) and bool((obuf[g + out0.numel() * esz:] == 0x5A).all())
    ref = dev.new_out(m)
    dev.forward(x, ref, dev.new_workspace(m))
    torch.cuda.synchronize()
    assert torch.equal(out, ref)


@pytest.mark.parametrize("m", [1, 3, 8, 40])
def test_bf16_output_is_rounded_fp32_output(m):
    # every launch path (the persistent kernel at small m, the multi-kernel path above it)
    cfg = CONFIGS["qwen3_6_35b_a3b"]
    lay, dev, _ = layer_for(cfg)
    dev_b = DeviceLayer.__new__(DeviceLayer)
    dev_b.__dict__.update(dev.__dict__)
    dev_b.c = type(dev.c).from_buffer_copy(dev.c)
    dev_b.c.out_dtype = B.MOE_FMT_BF16
    dev_b.out_dtype = "bf16"
    x = dev.x_to_device(lay.x(m))
    ws = dev.new_workspace(m)
    o32, o16 = dev.new_out(m), dev_b.new_out(m)
    dev.forward(x, o32, ws)
    dev_b.forward(x, o16, ws)
    torch.cuda.synchronize()
    assert o16.dtype == torch.bfloat16
    assert torch.equal(o16, o32.to(torch.bfloat16))


def test_refused_call_launches_nothing():
    lay, dev, _ = layer_for(SMALL["ragged_bf16"])
    m = 4
    x = dev.x_to_device(lay.x(m))
    ws = dev.new_workspace(m)
    out = torch.full((m, dev.cfg.hidden), 7.0, device="cuda")
    with pytest.raises(B.MoeError) as ei:
        B.moe_decode_forward(dev.c, m, x, dev.router_w, dev.expert_bias, dev.routed, dev.shared,
                             dev.shared_gate_w, out, ws, 1024, torch.cuda.current_stream())
    assert ei.value.status == B.MOE_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert torch.all(out == 7.0)


def test_cuda_graph_replay_matches_eager():
    lay, dev, _ = layer_for(CONFIGS["lfm2_8b_a1b"])
    m = 4
    x = dev.x_to_device(lay.x(m))
    ws = dev.new_workspace(m)
    eager, graphed = dev.new_out(m), dev.new_out(m)
    dev.forward(x, eager, ws)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        dev.forward(x, graphed, ws, stream=s)   # warm-up outside capture
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            dev.forward(x, graphed, ws, stream=s)
    torch.cuda.current_stream().wait_stream(s)
    graphed.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(eager, graphed)


# ---- the two launch paths: one persistent kernel (m <= 4) and the three-kernel chain --------

class _Path:
    """Force the multi-kernel path ("chain") or restore the automatic choice, for one block."""

    def __init__(self, name):
        self.name = name

    def __enter__(self):
        B.moe_debug_set_path(1 if self.name == "chain" else 0)

    def __exit__(self, *a):
        B.moe_debug_set_path(0)


PATH_CASES = ([(n, m) for n in ("qwen3_30b_a3b", "lfm2_8b_a1b", "qwen3_6_35b_a3b", "llama4_scout",
                                 "qwen3_30b_a3b_mxfp4", "qwen3_30b_a3b_fp8")
               for m in (1, 2, 3, 4)]
              + [(n, m) for n in SMALL for m in (1, 4, 9, 40)]
              + [("lfm2_8b_a1b", 16), ("qwen3_6_35b_a3b", 16), ("qwen3_30b_a3b", 8)])


@pytest.mark.parametrize("name,m", PATH_CASES)
def test_persistent_kernel_and_chain_agree_bitwise(name, m):
    cfg = SMALL.get(name) or CONFIGS[name]
    lay, dev, olay = layer_for(cfg)
    x = lay.x(m, offset=5)
    with _Path("chain"):
        chain, rt_c, st_c = run(dev, x)
    with _Path("auto"):
        auto, rt_a, st_a = run(dev, x)
    assert st_c == B.MOE_OK and st_a == B.MOE_OK
    for key in ("idx", "sorted_pairs", "expert_offsets", "token_to_perm", "active"):
        np.testing.assert_array_equal(rt_a[key], rt_c[key], err_msg=key)
    np.testing.assert_array_equal(rt_a["w"], rt_c["w"])
    np.testing.assert_array_equal(auto, chain)
    rows = SAMPLE_ROWS.get((name, m))
    want, _ = ref.moe_forward(olay, x, rows=rows)
    check_out(auto if rows is None else auto[rows], want)


def test_launch_count_follows_the_dispatch_rule():
    # tensor-core formats: one persistent launch at every m (three when the chain is forced);
    # f32 weights: the persistent CUDA-core kernel up to m = 4, the chain above
    lay, dev, _ = layer_for(CONFIGS["qwen3_30b_a3b"])
    assert [dev.launches(m) for m in (1, 2, 3, 4, 5, 8, 64)] == [1] * 7
    with _Path("chain"):
        assert dev.launches(1) == 3 and dev.launches(64) == 3
    lay, dev, _ = layer_for(SMALL["tiny_m64"])
    assert [dev.launches(m) for m in (1, 4, 5, 64)] == [1, 1, 3, 3]


class _Split:
    """Force a work split of the tensor-core path for one block (0 automatic, 1 whole jobs,
    2 jobs split by chunk)."""

    def __init__(self, mode):
        self.mode = mode

    def __enter__(self):
        B.moe_debug_set_split(self.mode)

    def __exit__(self, *a):
        B.moe_debug_set_split(0)


SPLIT_CASES = [("ragged_bf16", 17), ("ragged_q4_shared", 3), ("ragged_nvfp4_gate", 40),
               ("ragged_mxfp4", 9), ("ragged_fp8_geglu", 64), ("max_experts", 64),
               ("k_equals_E", 40), ("qwen3_30b_a3b", 1), ("lfm2_8b_a1b", 4),
               ("qwen3_6_35b_a3b", 16)]


@pytest.mark.parametrize("name,m", SPLIT_CASES)
def test_work_split_does_not_change_the_bits(name, m):
    # whole jobs per warp and jobs split into 256-element pieces give identical outputs, on
    # both launch paths
    cfg = SMALL.get(name) or CONFIGS[name]
    lay, dev, olay = layer_for(cfg)
    x = lay.x(m, offset=1 if m < 64 else 0)
    outs = []
    for path in ("auto", "chain"):
        for mode in (1, 2, 0):
            with _Path(path), _Split(mode):
                got, _, st = run(dev, x)
            assert st == B.MOE_OK
            outs.append(got)
    for o in outs[1:]:
        np.testing.assert_array_equal(o, outs[0])
    want, _ = ref.moe_forward(olay, x)
    check_out(outs[0], want)


def test_grid_barrier_timeout_is_reported_and_the_workspace_recovers():
    """A barrier wait and the down jobs' waits for their slot's gate/up jobs that run out (made to
    expect one arrival too many, with a ~1 ms budget) end the launch with MOE_ERR_DEVICE_TIMEOUT
    in the workspace status; after moe_workspace_init the same workspace gives the normal
    result again."""
    lay, dev, _ = layer_for(CONFIGS["qwen3_30b_a3b"])
    m = 1
    assert dev.launches(m) == 1
    x = dev.x_to_device(lay.x(m))
    ws = dev.new_workspace(m)
    want, out = dev.new_out(m), dev.new_out(m)
    dev.forward(x, want, ws)
    torch.cuda.synchronize()
    assert dev.device_status(ws) == B.MOE_OK
    B.moe_debug_barrier_test(1, 2_000_000)
    try:
        dev.forward(x, out, ws)
        torch.cuda.synchronize()
    finally:
        B.moe_debug_barrier_test(0, 0)
    assert dev.device_status(ws) == B.MOE_ERR_DEVICE_TIMEOUT
    B.moe_workspace_init(ws, ws.numel(), torch.cuda.current_stream())
    dev.forward(x, out, ws)
    torch.cuda.synchronize()
    assert dev.device_status(ws) == B.MOE_OK
    assert torch.equal(out, want)
