"""CPU tests of the C ABI: the library loads and exports every declared symbol, host-side
argument checks refuse bad calls before touching the GPU, and the pack / quantise helpers round
trip within their stated bounds (decoded by the oracle)."""
import ctypes
import os
import re

import numpy as np
import pytest
import torch

from mixture_experts_decode_gemv_b200 import binding as B
from mixture_experts_decode_gemv_b200.device_layer import make_cfg
from mixture_experts_decode_gemv_b200.synthetic import CONFIGS, LayerConfig
from oracle import moe_ref as ref

pytestmark = pytest.mark.cpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe_decode.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\*?\s+\**(moe_\w+)\s*\(", text, flags=re.M)))


def test_library_exports_every_declared_symbol():
    names = declared_functions()
    assert len(names) >= 13, names
    lib = ctypes.CDLL(B.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), f"{n} declared in moe_decode.h but not exported"
    assert set(names) == set(B.EXPORTS)


def test_header_enum_values_match_the_binding():
    import re
    with open(os.path.join(os.path.dirname(B.LIB_PATH), "..", "include", "moe_decode.h")) as f:
        text = f.read()
    vals = {k: int(v) for k, v in re.findall(r"\b(MOE_[A-Z0-9_]+)\s*=\s*(-?\d+)", text)}
    checked = 0
    for name, v in vals.items():
        if hasattr(B, name):
            assert getattr(B, name) == v, name
            checked += 1
    assert checked >= 20, checked
    # every format, routing and activation the Python side names exists in the header
    for table in (B.FORMAT_CODES, B.ROUTING_CODES, B.ACTIVATION_CODES, B.SHARED_CODES):
        assert set(table.values()) <= set(vals.values())
    # the struct layout the binding passes has the header's field count and order
    fields = re.search(r"typedef struct moe_cfg \{(.*?)\} moe_cfg;", text, re.S).group(1)
    names = re.findall(r"(?:int32_t|float)\s+(\w+);", fields)
    assert names == [f[0] for f in B.moe_cfg._fields_]


def test_version_and_status_strings():
    assert B.moe_version() == 200
    for st in range(-10, 1):
        assert B.moe_status_string(st) != "unknown status"
    assert B.moe_status_string(-99) == "unknown status"


@pytest.mark.parametrize("name", list(CONFIGS))
def test_workspace_bytes_grows_with_m(name):
    """One workspace sized for the largest m serves every smaller m: the size never shrinks."""
    c = make_cfg(CONFIGS[name])
    sizes = [B.moe_workspace_bytes(c, m) for m in range(1, 65)]
    assert all(s % 256 == 0 for s in sizes)
    assert sizes == sorted(sizes)


# ---- host-side refusals (fake, aligned device addresses: nothing is dereferenced) ----------

FAKE = 0x7F0000000000


def _fake_table(fmt=B.MOE_FMT_BF16, E=8, n=64, k=64):
    mats = []
    for (nn, kk) in ((n, k), (n, k), (k, n)):
        mm = B.moe_matrix()
        mm.format = fmt
        mm.packed = FAKE
        mm.expert_stride = nn * kk * 2
        mats.append(mm)
    return B.moe_expert_table(*mats)


def _small_cfg(**kw):
    base = dict(name="v", hidden=64, num_experts=8, top_k=2, moe_inter=64)
    base.update(kw)
    return make_cfg(LayerConfig(**base))


def _call(c, m=1, x=FAKE, rw=FAKE, bias=None, routed=None, shared=None, sg=None, out=FAKE,
          ws=FAKE, wsb=1 << 30):
    routed = routed if routed is not None else _fake_table()
    return B.lib.moe_decode_forward(
        ctypes.byref(c), m, x, rw, bias, ctypes.byref(routed),
        ctypes.byref(shared) if shared is not None else None, sg, out, ws, wsb, None)


def test_refusals_before_any_launch():
    c = _small_cfg()
    assert _call(c, m=0) == B.MOE_ERR_BAD_SHAPE
    assert _call(c, m=65) == B.MOE_ERR_BAD_SHAPE
    assert _call(c, x=None) == B.MOE_ERR_NULL_POINTER
    assert _call(c, out=None) == B.MOE_ERR_NULL_POINTER
    assert _call(c, x=FAKE + 8) == B.MOE_ERR_MISALIGNED
    assert _call(c, ws=FAKE + 128) == B.MOE_ERR_MISALIGNED
    assert _call(c, wsb=1024) == B.MOE_ERR_WORKSPACE
    bad = _small_cfg(top_k=9)
    assert _call(bad) == B.MOE_ERR_BAD_SHAPE
    bad = _small_cfg(hidden=60)
    assert _call(bad) == B.MOE_ERR_BAD_SHAPE
    bad = _small_cfg(num_experts=257, top_k=2)
    assert _call(bad) == B.MOE_ERR_BAD_SHAPE
    c2 = _small_cfg()
    c2.routing = 7
    assert _call(c2) == B.MOE_ERR_BAD_OPTION
    c3 = _small_cfg(routing="sigmoid", has_expert_bias=True)
    assert _call(c3) == B.MOE_ERR_NULL_POINTER        # bias required
    c4 = _small_cfg(routing="softmax")
    c4.has_expert_bias = 1
    assert _call(c4, bias=FAKE) == B.MOE_ERR_BAD_OPTION  # bias only with sigmoid
    c5 = _small_cfg(shared_inter=64, shared_kind="sigmoid_gate")
    assert _call(c5) == B.MOE_ERR_NULL_POINTER        # shared table required
    assert _call(c5, shared=_fake_table(E=1)) == B.MOE_ERR_NULL_POINTER  # gate vector required
    t = _fake_table()
    t.up.format = B.MOE_FMT_NVFP4
    assert _call(c, routed=t) == B.MOE_ERR_BAD_FORMAT  # gate/up formats differ
    t = _fake_table()
    t.gate.packed = FAKE + 4
    assert _call(c, routed=t) == B.MOE_ERR_MISALIGNED
    t = _fake_table(fmt=B.MOE_FMT_Q4_AFFINE_G64)
    assert _call(c, routed=t) == B.MOE_ERR_NULL_POINTER  # q4 needs scales and biases
    t = _fake_table()
    t.gate.expert_stride = 100
    assert _call(c, routed=t) == B.MOE_ERR_MISALIGNED


def test_valid_call_without_gpu_reports_cuda_or_device_error():
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    rc = _call(_small_cfg())
    assert rc in (B.MOE_ERR_CUDA, B.MOE_ERR_UNSUPPORTED_DEVICE)


def _launches(c, m=1, routed=None, shared=None, out=True):
    n = ctypes.c_int32(-1)
    routed = routed if routed is not None else _fake_table()
    return B.lib.moe_decode_launches(ctypes.byref(c), m, ctypes.byref(routed),
                                     ctypes.byref(shared) if shared is not None else None,
                                     ctypes.byref(n) if out else None)


def test_launch_count_query_refusals():
    c = _small_cfg()
    assert _launches(c, m=0) == B.MOE_ERR_BAD_SHAPE
    assert _launches(c, out=False) == B.MOE_ERR_NULL_POINTER
    t = _fake_table()
    t.up.format = B.MOE_FMT_NVFP4
    assert _launches(c, routed=t) == B.MOE_ERR_BAD_FORMAT
    c5 = _small_cfg(shared_inter=64, shared_kind="plain")
    assert _launches(c5) == B.MOE_ERR_NULL_POINTER       # shared table required
    if not torch.cuda.is_available():
        assert _launches(c) in (B.MOE_ERR_CUDA, B.MOE_ERR_UNSUPPORTED_DEVICE)


def test_barrier_test_hook_validates_its_arguments():
    assert B.lib.moe_debug_barrier_test(2, 0) == B.MOE_ERR_BAD_OPTION
    assert B.lib.moe_debug_barrier_test(-1, 0) == B.MOE_ERR_BAD_OPTION
    assert B.lib.moe_debug_barrier_test(0, -5) == B.MOE_ERR_BAD_OPTION
    assert B.lib.moe_debug_barrier_test(0, 0) == B.MOE_OK
    assert B.lib.moe_debug_set_path(2) == B.MOE_ERR_BAD_OPTION
    assert B.lib.moe_debug_set_path(-1) == B.MOE_ERR_BAD_OPTION
    assert B.lib.moe_debug_set_path(0) == B.MOE_OK
    assert B.lib.moe_debug_set_split(3) == B.MOE_ERR_BAD_OPTION
    assert B.lib.moe_debug_set_split(-1) == B.MOE_ERR_BAD_OPTION
    assert B.lib.moe_debug_set_split(0) == B.MOE_OK


# ---- pack / quantise helpers ---------------------------------------------------------------

def test_packed_bytes():
    assert B.moe_packed_bytes(B.MOE_FMT_BF16, 10, 64) == (1280, 0, 0)
    assert B.moe_packed_bytes(B.MOE_FMT_F32, 10, 64) == (2560, 0, 0)
    assert B.moe_packed_bytes(B.MOE_FMT_Q4_AFFINE_G64, 10, 128) == (640, 40, 40)
    assert B.moe_packed_bytes(B.MOE_FMT_NVFP4, 10, 128) == (640, 80, 0)
    with pytest.raises(B.MoeError):
        B.moe_packed_bytes(B.MOE_FMT_Q4_AFFINE_G64, 10, 96)


def test_pack_bf16_matches_torch_rounding():
    rng = np.random.default_rng(0)
    w = (rng.standard_normal(10000) * 10.0 ** rng.integers(-8, 8, 10000)).astype(np.float32)
    got = B.moe_pack_bf16(w)
    want = torch.from_numpy(w).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(got, want)


def test_q4_affine_quantiser_round_trip_bound():
    rng = np.random.default_rng(1)
    n, k = 16, 256
    w = (rng.standard_normal((n, k)) * 0.05).astype(np.float32)
    packed, scales, biases = B.moe_quantize_q4_affine(w)
    from mixture_experts_decode_gemv_b200.synthetic import MatrixSlab
    slab = MatrixSlab("q4_affine_g64", n, k, packed[None], scales=scales[None],
                      biases=biases[None])
    dec = ref.decode_matrix(slab, 0)
    s = np.repeat(ref.f16_to_f64(scales), 64, axis=1)
    b = np.repeat(ref.f16_to_f64(biases), 64, axis=1)
    wg = w.astype(np.float64).reshape(n, k // 64, 64)
    lo, hi = wg.min(axis=2), wg.max(axis=2)
    s_exact = np.repeat((hi - lo) / 15.0, 64, axis=1)
    # half a step, plus what fp16 rounding of scale and bias can add over 15 steps
    bound = s / 2 + 15 * np.abs(s - s_exact) + np.abs(b - np.repeat(lo, 64, axis=1)) + 1e-12
    assert np.all(np.abs(dec - w) <= bound)
    # the library's own decoder agrees with the oracle's
    lib_dec = B.moe_dequantize(B.MOE_FMT_Q4_AFFINE_G64, packed, scales, biases, None, n, k)
    np.testing.assert_array_equal(lib_dec, dec.astype(np.float32))


def test_nvfp4_quantiser_round_trip_bound():
    rng = np.random.default_rng(2)
    n, k = 16, 256
    w = (rng.standard_normal((n, k)) * 0.05).astype(np.float32)
    packed, scales, ts = B.moe_quantize_nvfp4(w)
    from mixture_experts_decode_gemv_b200.synthetic import MatrixSlab
    slab = MatrixSlab("nvfp4", n, k, packed[None], scales=scales[None], tensor_scale=ts)
    dec = ref.decode_matrix(slab, 0)
    blk = np.repeat(ref.e4m3_value(scales), 16, axis=1) * float(ts[0])
    v = w.astype(np.float64) / blk              # value on the E2M1 grid scale
    q = dec / blk
    grid = np.array([0, .5, 1, 1.5, 2, 3, 4, 6])
    # distance to the nearest grid point, or the saturation excess above 6
    step = np.where(np.abs(v) < 2, 0.25, np.where(np.abs(v) < 4, 0.5, 1.0))
    err = np.abs(q - v)
    assert np.all(err <= step + np.maximum(0, np.abs(v) - 6) + 1e-9)
    # every decoded value is on the grid
    assert np.all(np.isin(np.abs(q), grid))
    lib_dec = B.moe_dequantize(B.MOE_FMT_NVFP4, packed, scales, None, ts, n, k)
    np.testing.assert_allclose(lib_dec, dec.astype(np.float32), rtol=1e-7, atol=0)


def test_mxfp4_quantiser_round_trip_bound():
    rng = np.random.default_rng(4)
    n, k = 16, 256
    w = (rng.standard_normal((n, k)) * 0.05).astype(np.float32)
    w[3, :32] = 0.0                                   # an all-zero block
    packed, scales = B.moe_quantize_mxfp4(w)
    from mixture_experts_decode_gemv_b200.synthetic import MatrixSlab
    slab = MatrixSlab("mxfp4", n, k, packed[None], scales=scales[None])
    dec = ref.decode_matrix(slab, 0)
    # the block scale is 2^(floor(log2 max|w|) - 2): the block maximum lands in [4, 8) on the
    # E2M1 grid, whose largest value is 6
    blk = np.repeat(ref.e8m0_value(scales), 32, axis=1)
    amax = np.abs(w.astype(np.float64)).reshape(n, k // 32, 32).max(axis=2)
    nz = amax > 0
    np.testing.assert_array_equal(
        scales[nz].astype(int) - 127, np.floor(np.log2(amax[nz])).astype(int) - 2)
    assert scales[3, 0] == 127
    v = w.astype(np.float64) / blk
    q = dec / blk
    grid = np.array([0, .5, 1, 1.5, 2, 3, 4, 6])
    step = np.where(np.abs(v) < 2, 0.25, np.where(np.abs(v) < 4, 0.5, 1.0))
    err = np.abs(q - v)
    assert np.all(err <= step + np.maximum(0, np.abs(v) - 6) + 1e-9)
    assert np.all(np.isin(np.abs(q), grid))
    lib_dec = B.moe_dequantize(B.MOE_FMT_MXFP4, packed, scales, None, None, n, k)
    np.testing.assert_array_equal(lib_dec, dec.astype(np.float32))
    assert B.moe_packed_bytes(B.MOE_FMT_MXFP4, 10, 128) == (640, 40, 0)


def test_fp8_quantiser_round_trip_bound():
    rng = np.random.default_rng(5)
    n, k = 8, 64
    w = (rng.standard_normal((n, k)) * 0.05).astype(np.float32)
    packed, ts = B.moe_quantize_fp8_e4m3(w)
    assert ts[0] == np.float32(np.abs(w.astype(np.float64)).max() / 448.0)
    from mixture_experts_decode_gemv_b200.synthetic import MatrixSlab
    dec = ref.decode_matrix(MatrixSlab("fp8_e4m3", n, k, packed[None], tensor_scale=ts), 0)
    v = w.astype(np.float64) / float(ts[0])
    # E4M3 has 3 mantissa bits: a normal value is within 2^-4 relative of its code; below 2^-6
    # the subnormal step is 2^-9
    err = np.abs(dec / float(ts[0]) - v)
    assert np.all(err <= np.maximum(np.abs(v) * 2.0 ** -4, 2.0 ** -10) + 1e-12)
    lib_dec = B.moe_dequantize(B.MOE_FMT_FP8_E4M3, packed, None, None, ts, n, k)
    np.testing.assert_array_equal(lib_dec, dec.astype(np.float32))
    assert B.moe_packed_bytes(B.MOE_FMT_FP8_E4M3, 10, 64) == (640, 0, 0)


def test_new_options_are_refused_out_of_range():
    c = _small_cfg()
    c.activation = 2
    assert _call(c) == B.MOE_ERR_BAD_OPTION
    c = _small_cfg()
    c.routing = 3
    assert _call(c) == B.MOE_ERR_BAD_OPTION
    c = _small_cfg(routing="sqrtsoftplus", has_expert_bias=True)
    assert _call(c) == B.MOE_ERR_NULL_POINTER         # bias required, as for sigmoid
    t = _fake_table(fmt=B.MOE_FMT_FP8_E4M3)
    assert _call(_small_cfg(), routed=t) == B.MOE_ERR_NULL_POINTER  # fp8 needs its scales


def test_dequantize_bf16_and_f32_plain():
    w = np.arange(12, dtype=np.float32).reshape(3, 4) - 5.5
    np.testing.assert_array_equal(B.moe_dequantize(B.MOE_FMT_F32, w, None, None, None, 3, 4), w)
    bits = B.moe_pack_bf16(w)
    np.testing.assert_array_equal(B.moe_dequantize(B.MOE_FMT_BF16, bits, None, None, None, 3, 4),
                                  ref.bf16_to_f64(bits).astype(np.float32))
