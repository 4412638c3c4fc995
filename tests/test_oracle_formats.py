"""Pins of the oracle's weight-format decoders against the format definitions and library
routines (CPU only)."""
import os

import numpy as np
import pytest
import torch

from oracle import moe_ref as ref
from mixture_experts_decode_gemv_b200.synthetic import MatrixSlab

pytestmark = pytest.mark.cpu


def _read_table(path):
    codes, vals = [], []
    with open(path) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            c, v = line.split()
            codes.append(int(c, 16))
            vals.append(float(v))
    return np.array(codes), np.array(vals)


def test_e2m1_all_sixteen_codes(golden_dir):
    codes, vals = _read_table(os.path.join(golden_dir, "e2m1_values.txt"))
    assert len(codes) == 16
    got = ref.e2m1_value(codes)
    np.testing.assert_array_equal(got, vals)
    # signed zero for code 8
    assert np.signbit(ref.e2m1_value(np.array([8])))[0]


def test_e4m3_golden_codes(golden_dir):
    codes, vals = _read_table(os.path.join(golden_dir, "e4m3_values.txt"))
    got = ref.e4m3_value(codes)
    np.testing.assert_array_equal(np.isnan(got), np.isnan(vals))
    ok = ~np.isnan(vals)
    np.testing.assert_array_equal(got[ok], vals[ok])


def test_e4m3_every_code_matches_torch_float8():
    codes = np.arange(256, dtype=np.uint8)
    lib = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = ref.e4m3_value(codes)
    np.testing.assert_array_equal(np.isnan(got), np.isnan(lib))
    ok = ~np.isnan(lib)
    np.testing.assert_array_equal(got[ok], lib[ok])


@pytest.mark.filterwarnings("ignore::RuntimeWarning")
def test_bf16_and_f16_known_bits():
    np.testing.assert_array_equal(
        ref.bf16_to_f64(np.array([0x3F80, 0xC000, 0x0000, 0x3E80, 0x4049], dtype=np.uint16)),
        [1.0, -2.0, 0.0, 0.25, 3.140625])
    np.testing.assert_array_equal(
        ref.f16_to_f64(np.array([0x3800, 0xBC00, 0x3C00, 0x0001], dtype=np.uint16)),
        [0.5, -1.0, 1.0, 2.0 ** -24])
    # bf16 decode agrees with torch's bfloat16 for random bit patterns (finite ones)
    rng = np.random.default_rng(7)
    bits = rng.integers(0, 1 << 16, size=4096, dtype=np.uint16)
    lib = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    got = ref.bf16_to_f64(bits)
    fin = np.isfinite(lib)
    np.testing.assert_array_equal(got[fin], lib[fin])


def test_nibble_order_low_first():
    packed = np.array([[0x21, 0xF0]], dtype=np.uint8)
    np.testing.assert_array_equal(ref.unpack_nibbles(packed, 4), [[1, 2, 0, 15]])


def test_q4_affine_hand_built():
    # one row of 64 codes q = 0..15 repeated; scale 0.5, bias -1  ->  w = 0.5 q - 1
    q = np.tile(np.arange(16, dtype=np.uint8), 4)
    packed = (q[0::2] | (q[1::2] << 4)).astype(np.uint8)[None, None, :]
    scale = np.array([[[0x3800]]], dtype=np.uint16)   # 0.5
    bias = np.array([[[0xBC00]]], dtype=np.uint16)    # -1.0
    slab = MatrixSlab("q4_affine_g64", 1, 64, packed, scales=scale, biases=bias)
    w = ref.decode_matrix(slab, 0)
    np.testing.assert_array_equal(w[0], 0.5 * q - 1.0)


def test_q4_affine_group_boundaries():
    # two groups with different scale/bias: the group of element j is j // 64
    q = np.full(128, 3, dtype=np.uint8)
    packed = (q[0::2] | (q[1::2] << 4)).astype(np.uint8)[None, None, :]
    scales = np.array([[[0x3C00, 0x4000]]], dtype=np.uint16)   # 1.0, 2.0
    biases = np.array([[[0x0000, 0x3C00]]], dtype=np.uint16)   # 0.0, 1.0
    slab = MatrixSlab("q4_affine_g64", 1, 128, packed, scales=scales, biases=biases)
    w = ref.decode_matrix(slab, 0)[0]
    np.testing.assert_array_equal(w[:64], 3.0)
    np.testing.assert_array_equal(w[64:], 7.0)


def test_nvfp4_hand_built():
    # 32 codes: block 0 all code 7 (6.0), block 1 all code 0xF (-6.0)
    q = np.array([7] * 16 + [15] * 16, dtype=np.uint8)
    packed = (q[0::2] | (q[1::2] << 4)).astype(np.uint8)[None, None, :]
    scales = np.array([[[0x38, 0x40]]], dtype=np.uint8)          # 1.0, 2.0
    ts = np.array([0.25], dtype=np.float32)
    slab = MatrixSlab("nvfp4", 1, 32, packed, scales=scales, tensor_scale=ts)
    w = ref.decode_matrix(slab, 0)[0]
    np.testing.assert_array_equal(w[:16], 6.0 * 1.0 * 0.25)
    np.testing.assert_array_equal(w[16:], -6.0 * 2.0 * 0.25)


def test_nvfp4_every_code_times_scale():
    codes = np.arange(16, dtype=np.uint8)
    q = np.concatenate([codes, codes])
    packed = (q[0::2] | (q[1::2] << 4)).astype(np.uint8)[None, None, :]
    scales = np.array([[[0x01, 0x7E]]], dtype=np.uint8)          # 2^-9 and 448
    ts = np.array([1.0], dtype=np.float32)
    slab = MatrixSlab("nvfp4", 1, 32, packed, scales=scales, tensor_scale=ts)
    w = ref.decode_matrix(slab, 0)[0]
    e2m1 = np.array([0, .5, 1, 1.5, 2, 3, 4, 6, -0., -.5, -1, -1.5, -2, -3, -4, -6])
    np.testing.assert_array_equal(w[:16], e2m1 * 2.0 ** -9)
    np.testing.assert_array_equal(w[16:], e2m1 * 448.0)


def test_e8m0_golden_codes(golden_dir):
    codes, vals = _read_table(os.path.join(golden_dir, "e8m0_values.txt"))
    got = ref.e8m0_value(codes)
    np.testing.assert_array_equal(np.isnan(got), np.isnan(vals))
    np.testing.assert_array_equal(got[~np.isnan(vals)], vals[~np.isnan(vals)])


def test_e8m0_every_code_is_a_power_of_two():
    c = np.arange(255)
    v = ref.e8m0_value(c)
    m, ex = np.frexp(v)                       # v = m * 2**ex with m in [0.5, 1)
    np.testing.assert_array_equal(m, 0.5)
    np.testing.assert_array_equal(ex - 1, c - 127)


def test_mxfp4_hand_built():
    # 64 codes in two 32-element blocks: block 0 all code 5 (3.0), block 1 all code 0xA (-1.0)
    q = np.array([5] * 32 + [0xA] * 32, dtype=np.uint8)
    packed = (q[0::2] | (q[1::2] << 4)).astype(np.uint8)[None, None, :]
    scales = np.array([[[0x7F, 0x81]]], dtype=np.uint8)          # 1.0, 4.0
    slab = MatrixSlab("mxfp4", 1, 64, packed, scales=scales)
    w = ref.decode_matrix(slab, 0)[0]
    np.testing.assert_array_equal(w[:32], 3.0)
    np.testing.assert_array_equal(w[32:], -4.0)


def test_mxfp4_with_unit_scales_is_plain_e2m1_and_scales_by_powers_of_two():
    rng = np.random.default_rng(3)
    q = rng.integers(0, 16, size=(3, 96), dtype=np.uint8)
    packed = (q[:, 0::2] | (q[:, 1::2] << 4)).astype(np.uint8)[None]
    sc = rng.integers(100, 150, size=(1, 3, 3), dtype=np.uint8)
    w = ref.decode_matrix(MatrixSlab("mxfp4", 3, 96, packed, scales=sc), 0)
    plain = ref.decode_matrix(MatrixSlab("mxfp4", 3, 96, packed,
                                         scales=np.full_like(sc, 0x7F)), 0)
    np.testing.assert_array_equal(plain, ref.e2m1_value(q))
    np.testing.assert_array_equal(w, plain * np.exp2(np.repeat(sc[0].astype(float) - 127, 32, 1)))


def test_fp8_e4m3_hand_built(golden_dir):
    codes, vals = _read_table(os.path.join(golden_dir, "e4m3_values.txt"))
    ok = ~np.isnan(vals)
    row = codes[ok].astype(np.uint8)
    k = 16
    data = np.zeros((1, 2, k), np.uint8)
    data[0, 0, :row.size] = row
    data[0, 1, :] = 0x38                                       # 1.0 everywhere
    slab = MatrixSlab("fp8_e4m3", 2, k, data, tensor_scale=np.array([0.5], np.float32))
    w = ref.decode_matrix(slab, 0)
    np.testing.assert_array_equal(w[0, :row.size], vals[ok] * 0.5)
    np.testing.assert_array_equal(w[1], 0.5)
