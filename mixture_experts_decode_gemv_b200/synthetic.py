"""Seeded synthetic decode-time MoE layers.

Every input of one MoE layer (activation rows, router matrix, expert bias, shared-expert gate
vector and the routed / shared expert weight slabs) is drawn here from numpy PCG64 sub-streams.
Each array has its own stream, keyed by what it is (``SeedSequence(seed, spawn_key=...)``), so a
single expert of a single projection can be regenerated on its own.

This module is deliberately free of the layer's arithmetic: it never computes a router logit, a
routing weight, an expert product, or the value that a packed 4-bit code stands for. Quantised
weights are drawn directly as random codes plus random scale fields; their storage layout is the
library's (``[N, K/2]`` bytes, element ``2j`` in the low nibble of byte ``j``). The only operation
applied to drawn numbers is the round-to-nearest-even conversion of float32 samples to bfloat16
storage, which is how bf16 inputs are produced.

The one rule that needs layer arithmetic, redrawing an activation row whose top ``k+1`` selection
keys have a gap below ``1e-3``, is applied through a caller-supplied ``key_fn``; this module only
compares the keys that ``key_fn`` returns.
"""
from __future__ import annotations

import dataclasses
from dataclasses import dataclass, field
from typing import Callable, Dict, Optional, Sequence, Tuple

import numpy as np

SEED_BASE = 0x30E0
POOL_ROWS = 64
GAP_MIN = 1e-3
MAX_REDRAWS = 10_000

# Stream tags (first element of every spawn key).
TAG_X_ROW = 1
TAG_ROUTER = 2
TAG_EXPERT = 3
TAG_SHARED = 4
TAG_BIAS = 5
TAG_SHARED_GATE = 6

PROJ = {"gate": 0, "up": 1, "down": 2}

FORMATS = ("f32", "bf16", "q4_affine_g64", "nvfp4", "mxfp4", "fp8_e4m3")

# Statistics used to give random codes an N(0, 1/fan_in)-like spread.
#  - 4-bit affine: codes uniform on 0..15 have variance 255/12 = 21.25 and mean 7.5.
#  - NVFP4: uniform E2M1 codes have mean-square magnitude 8.5625; block scale codes are drawn
#    from E4M3 0x30..0x40 (0.5 .. 2.0), mean-square about 1.5, so 0.28 / sqrt(fan_in) as the
#    per-matrix fp32 scale gives roughly unit-variance logits downstream.
#  - MXFP4: the same codes; the E8M0 block scale is the power of two nearest to
#    1 / (sqrt(8.5625 * fan_in)), times 2^-1, 2^0 or 2^1 drawn uniformly per block.
#  - FP8 E4M3: random sign, exponent field uniform on 5..9 (2^-2 .. 2^2) and mantissa uniform on
#    0..7 (no NaN codes); mean-square value 4.2625 * 2.1484375, so the per-matrix fp32 scale
#    1 / sqrt(that * fan_in) gives variance 1 / fan_in.
_Q4_CODE_VAR = 21.25
_E2M1_MEAN_SQUARE = 8.5625
_E4M3_DRAWN_MEAN_SQUARE = ((1 / 16 + 1 / 4 + 1 + 4 + 16) / 5) * (1100 / 8 / 64)
_NVFP4_TENSOR_SCALE = 0.28
_E4M3_SCALE_CODE_LO = 0x30
_E4M3_SCALE_CODE_HI = 0x40


@dataclass(frozen=True)
class LayerConfig:
    """Shape and routing options of one MoE layer (one row per published model shape)."""

    name: str
    hidden: int
    num_experts: int
    top_k: int
    moe_inter: int
    shared_inter: int = 0
    fmt: str = "bf16"              # routed and shared expert weight format
    x_dtype: str = "bf16"          # activations, router matrix and shared gate vector
    routing: str = "softmax"       # "softmax" | "sigmoid" | "sqrtsoftplus"
    norm_topk_prob: bool = True
    select_on_raw_logits: bool = False
    has_expert_bias: bool = False
    routed_scaling_factor: float = 1.0
    weight_before_ffn: bool = False
    shared_kind: str = "none"      # "none" | "plain" | "sigmoid_gate"
    activation: str = "swiglu"     # "swiglu" (silu(g) * u) | "geglu" (gelu_tanh(g) * u)
    m_list: Tuple[int, ...] = (1,)
    index: int = 0                 # seed = SEED_BASE + index

    @property
    def seed(self) -> int:
        return SEED_BASE + self.index

    @property
    def has_shared(self) -> bool:
        return self.shared_kind != "none" and self.shared_inter > 0

    def replace(self, **kw) -> "LayerConfig":
        return dataclasses.replace(self, **kw)


# The five published shapes. Sizes, formats and routing options follow the model shapes the
# MoE decode pages target; the m lists are the row counts each shape is exercised at.
TINY = LayerConfig(
    name="tiny", hidden=256, num_experts=8, top_k=2, moe_inter=128, fmt="f32", x_dtype="f32",
    routing="softmax", norm_topk_prob=True, m_list=(1, 4), index=0)
QWEN3_30B_A3B = LayerConfig(
    name="qwen3_30b_a3b", hidden=2048, num_experts=128, top_k=8, moe_inter=768, fmt="bf16",
    routing="softmax", norm_topk_prob=True, m_list=(1, 2, 4, 8), index=1)
LFM2_8B_A1B = LayerConfig(
    name="lfm2_8b_a1b", hidden=2048, num_experts=32, top_k=4, moe_inter=1792,
    fmt="q4_affine_g64", routing="sigmoid", has_expert_bias=True, norm_topk_prob=True,
    routed_scaling_factor=1.0, m_list=(1, 4, 16), index=2)
QWEN3_6_35B_A3B = LayerConfig(
    name="qwen3_6_35b_a3b", hidden=2048, num_experts=256, top_k=8, moe_inter=512,
    shared_inter=512, shared_kind="sigmoid_gate", fmt="nvfp4", routing="softmax",
    norm_topk_prob=True, m_list=(1, 8, 16), index=3)
LLAMA4_SCOUT = LayerConfig(
    name="llama4_scout", hidden=5120, num_experts=16, top_k=1, moe_inter=8192,
    shared_inter=8192, shared_kind="plain", fmt="bf16", routing="sigmoid",
    select_on_raw_logits=True, norm_topk_prob=False, weight_before_ffn=True,
    m_list=(1, 16, 64), index=4)

# MXFP4 experts (E2M1 codes with an E8M0 scale per 32 elements) on the Qwen3-30B-A3B shape: the
# native MXFP4 expert format the pages' prefill helpers handle, at decode sizes.
QWEN3_30B_A3B_MXFP4 = QWEN3_30B_A3B.replace(name="qwen3_30b_a3b_mxfp4", fmt="mxfp4",
                                           m_list=(1, 4), index=5)

# FP8 (E4M3, one scale per expert matrix) experts on the same shape: the pages' FP8 grouped decode.
QWEN3_30B_A3B_FP8 = QWEN3_30B_A3B.replace(name="qwen3_30b_a3b_fp8", fmt="fp8_e4m3",
                                         m_list=(1, 4), index=6)

CONFIGS: Dict[str, LayerConfig] = {
    c.name: c for c in (TINY, QWEN3_30B_A3B, LFM2_8B_A1B, QWEN3_6_35B_A3B, LLAMA4_SCOUT,
                        QWEN3_30B_A3B_MXFP4, QWEN3_30B_A3B_FP8)
}


def rng_for(cfg: LayerConfig, *key: int) -> np.random.Generator:
    """The PCG64 sub-stream of ``cfg`` keyed by ``key`` (tag first)."""
    ss = np.random.SeedSequence(cfg.seed, spawn_key=tuple(int(k) for k in key))
    return np.random.Generator(np.random.PCG64(ss))


def to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 samples to bfloat16 storage (round to nearest, ties to even)."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    return ((u + np.uint32(0x7FFF) + lsb) >> np.uint32(16)).astype(np.uint16)


def _draw_dense(g: np.random.Generator, shape, fan_in: int, dtype: str) -> np.ndarray:
    a = g.standard_normal(shape, dtype=np.float32)
    a *= np.float32(1.0 / np.sqrt(fan_in))
    if dtype == "f32":
        return a
    if dtype == "bf16":
        return to_bf16_bits(a)
    raise ValueError(dtype)


def _pack_nibbles(codes: np.ndarray) -> np.ndarray:
    """Store 4-bit codes two per byte, element 2j in the low nibble of byte j."""
    return (codes[..., 0::2] | (codes[..., 1::2] << np.uint8(4))).astype(np.uint8)


@dataclass
class MatrixSlab:
    """One projection of E experts, each an ``[n, k]`` matrix, in the library's storage.

    ``data``: f32 -> float32 ``[E, n, k]``; bf16 -> uint16 ``[E, n, k]``; fp8_e4m3 -> uint8
    ``[E, n, k]``; 4-bit formats -> uint8 ``[E, n, k/2]``. ``scales``: q4 -> fp16 bits ``[E, n, k/64]``; nvfp4 -> E4M3 codes
    ``[E, n, k/16]``. ``biases``: q4 -> fp16 bits ``[E, n, k/64]``. ``tensor_scale``: nvfp4 ->
    float32 ``[E]``.
    """

    fmt: str
    n: int
    k: int
    data: np.ndarray
    scales: Optional[np.ndarray] = None
    biases: Optional[np.ndarray] = None
    tensor_scale: Optional[np.ndarray] = None

    @property
    def num_experts(self) -> int:
        return self.data.shape[0]

    def expert(self, e: int) -> "MatrixSlab":
        sl = slice(e, e + 1)
        return MatrixSlab(
            self.fmt, self.n, self.k, self.data[sl],
            None if self.scales is None else self.scales[sl],
            None if self.biases is None else self.biases[sl],
            None if self.tensor_scale is None else self.tensor_scale[sl])


def draw_matrix(g: np.random.Generator, fmt: str, n: int, k: int, fan_in: int) -> MatrixSlab:
    """Draw one ``[n, k]`` matrix in ``fmt`` (as a one-expert slab)."""
    if fmt in ("f32", "bf16"):
        return MatrixSlab(fmt, n, k, _draw_dense(g, (1, n, k), fan_in, fmt))
    if fmt == "q4_affine_g64":
        if k % 64:
            raise ValueError("q4_affine_g64 needs k % 64 == 0")
        codes = g.integers(0, 16, size=(1, n, k), dtype=np.uint8)
        groups = k // 64
        base = 1.0 / np.sqrt(_Q4_CODE_VAR * fan_in)
        scale = base * g.uniform(0.75, 1.25, size=(1, n, groups))
        bias = -scale * (7.5 + 0.5 * g.standard_normal((1, n, groups)))
        return MatrixSlab(fmt, n, k, _pack_nibbles(codes),
                          scales=scale.astype(np.float16).view(np.uint16),
                          biases=bias.astype(np.float16).view(np.uint16))
    if fmt == "nvfp4":
        if k % 32:
            raise ValueError("nvfp4 needs k % 32 == 0")
        codes = g.integers(0, 16, size=(1, n, k), dtype=np.uint8)
        sc = g.integers(_E4M3_SCALE_CODE_LO, _E4M3_SCALE_CODE_HI + 1, size=(1, n, k // 16),
                        dtype=np.uint8)
        ts = np.array([_NVFP4_TENSOR_SCALE / np.sqrt(fan_in)], dtype=np.float32)
        return MatrixSlab(fmt, n, k, _pack_nibbles(codes), scales=sc, tensor_scale=ts)
    if fmt == "fp8_e4m3":
        if k % 16:
            raise ValueError("fp8_e4m3 needs k % 16 == 0")
        sign = g.integers(0, 2, size=(1, n, k), dtype=np.uint8)
        expo = g.integers(5, 10, size=(1, n, k), dtype=np.uint8)
        mant = g.integers(0, 8, size=(1, n, k), dtype=np.uint8)
        codes = ((sign << np.uint8(7)) | (expo << np.uint8(3)) | mant).astype(np.uint8)
        ts = np.array([1.0 / np.sqrt(_E4M3_DRAWN_MEAN_SQUARE * fan_in)], dtype=np.float32)
        return MatrixSlab(fmt, n, k, codes, tensor_scale=ts)
    if fmt == "mxfp4":
        if k % 32:
            raise ValueError("mxfp4 needs k % 32 == 0")
        codes = g.integers(0, 16, size=(1, n, k), dtype=np.uint8)
        base = 127 + int(np.round(-0.5 * np.log2(_E2M1_MEAN_SQUARE * fan_in)))
        sc = (base + g.integers(-1, 2, size=(1, n, k // 32))).astype(np.uint8)
        return MatrixSlab(fmt, n, k, _pack_nibbles(codes), scales=sc)
    raise ValueError(f"unknown format {fmt!r}")


def _concat(parts: Sequence[MatrixSlab]) -> MatrixSlab:
    p0 = parts[0]
    cat = lambda name: (None if getattr(p0, name) is None
                        else np.concatenate([getattr(p, name) for p in parts], axis=0))
    return MatrixSlab(p0.fmt, p0.n, p0.k, cat("data"), cat("scales"), cat("biases"),
                      cat("tensor_scale"))


def _zeros_like_expert(fmt: str, n: int, k: int) -> MatrixSlab:
    if fmt == "f32":
        return MatrixSlab(fmt, n, k, np.zeros((1, n, k), np.float32))
    if fmt == "bf16":
        return MatrixSlab(fmt, n, k, np.zeros((1, n, k), np.uint16))
    if fmt == "q4_affine_g64":
        z = np.zeros((1, n, k // 64), np.uint16)
        return MatrixSlab(fmt, n, k, np.zeros((1, n, k // 2), np.uint8), scales=z, biases=z.copy())
    if fmt == "nvfp4":
        return MatrixSlab(fmt, n, k, np.zeros((1, n, k // 2), np.uint8),
                          scales=np.zeros((1, n, k // 16), np.uint8),
                          tensor_scale=np.zeros((1,), np.float32))
    if fmt == "mxfp4":
        return MatrixSlab(fmt, n, k, np.zeros((1, n, k // 2), np.uint8),
                          scales=np.zeros((1, n, k // 32), np.uint8))
    if fmt == "fp8_e4m3":
        return MatrixSlab(fmt, n, k, np.zeros((1, n, k), np.uint8),
                          tensor_scale=np.zeros((1,), np.float32))
    raise ValueError(fmt)


KeyFn = Callable[[np.ndarray], np.ndarray]


@dataclass
class SyntheticLayer:
    """Lazily drawn inputs of one MoE layer for ``cfg``.

    Arrays are drawn on first access and cached. ``routed_expert(e, proj)`` draws one expert of
    one projection from its own stream, so the set of experts that is materialised can be
    restricted (``routed(proj, experts=...)`` fills the rest with zero bytes).
    """

    cfg: LayerConfig
    key_fn: Optional[KeyFn] = None
    _cache: dict = field(default_factory=dict, repr=False)

    # ---- small arrays --------------------------------------------------------------------
    def router_w(self) -> np.ndarray:
        if "router" not in self._cache:
            c = self.cfg
            self._cache["router"] = _draw_dense(rng_for(c, TAG_ROUTER), (c.num_experts, c.hidden),
                                                c.hidden, c.x_dtype)
        return self._cache["router"]

    def expert_bias(self) -> Optional[np.ndarray]:
        c = self.cfg
        if not c.has_expert_bias:
            return None
        if "bias" not in self._cache:
            g = rng_for(c, TAG_BIAS)
            self._cache["bias"] = (g.standard_normal(c.num_experts) * np.sqrt(0.1)).astype(
                np.float32)
        return self._cache["bias"]

    def shared_gate_w(self) -> Optional[np.ndarray]:
        c = self.cfg
        if c.shared_kind != "sigmoid_gate":
            return None
        if "sg" not in self._cache:
            self._cache["sg"] = _draw_dense(rng_for(c, TAG_SHARED_GATE), (c.hidden,), c.hidden,
                                            c.x_dtype)
        return self._cache["sg"]

    def x_pool(self) -> np.ndarray:
        """``POOL_ROWS`` activation rows; an m-row input is the first m rows."""
        if "x" not in self._cache:
            self._cache["x"] = np.stack([self._draw_row(r) for r in range(POOL_ROWS)])
        return self._cache["x"]

    def x(self, m: int, offset: int = 0) -> np.ndarray:
        pool = self.x_pool()
        if offset + m > POOL_ROWS:
            raise ValueError("m + offset exceeds the row pool")
        return np.ascontiguousarray(pool[offset:offset + m])

    def _draw_row(self, r: int) -> np.ndarray:
        c = self.cfg
        g = rng_for(c, TAG_X_ROW, r)
        for _ in range(MAX_REDRAWS):
            row = _draw_dense(g, (c.hidden,), 1, c.x_dtype)
            if self.key_fn is None or _gap_ok(self.key_fn(row), c.top_k):
                return row
        raise RuntimeError(f"row {r}: no draw met the selection-gap rule")

    # ---- expert slabs --------------------------------------------------------------------
    def _proj_shape(self, proj: str, inter: int) -> Tuple[int, int, int]:
        h = self.cfg.hidden
        return (inter, h, h) if proj in ("gate", "up") else (h, inter, inter)

    def routed_expert(self, e: int, proj: str) -> MatrixSlab:
        key = ("r", e, proj)
        if key not in self._cache:
            n, k, fan_in = self._proj_shape(proj, self.cfg.moe_inter)
            self._cache[key] = draw_matrix(rng_for(self.cfg, TAG_EXPERT, e, PROJ[proj]),
                                           self.cfg.fmt, n, k, fan_in)
        return self._cache[key]

    def routed(self, proj: str, experts: Optional[Sequence[int]] = None) -> MatrixSlab:
        """All E experts of ``proj`` as one slab; experts outside ``experts`` are zero bytes."""
        E = self.cfg.num_experts
        want = set(range(E)) if experts is None else set(int(e) for e in experts)
        n, k, _ = self._proj_shape(proj, self.cfg.moe_inter)
        parts = [self.routed_expert(e, proj) if e in want else _zeros_like_expert(self.cfg.fmt, n, k)
                 for e in range(E)]
        return _concat(parts)

    def shared(self, proj: str) -> Optional[MatrixSlab]:
        c = self.cfg
        if not c.has_shared:
            return None
        key = ("s", proj)
        if key not in self._cache:
            n, k, fan_in = self._proj_shape(proj, c.shared_inter)
            self._cache[key] = draw_matrix(rng_for(c, TAG_SHARED, PROJ[proj]), c.fmt, n, k, fan_in)
        return self._cache[key]

    def drop_expert_cache(self) -> None:
        for key in [k for k in self._cache if isinstance(k, tuple) and k[0] == "r"]:
            del self._cache[key]


def _gap_ok(keys: np.ndarray, k: int) -> bool:
    s = np.sort(np.asarray(keys, dtype=np.float64))[::-1]
    top = s[: min(k + 1, s.size)]
    return bool(top.size < 2 or np.min(top[:-1] - top[1:]) >= GAP_MIN)


def weight_bytes_per_expert(cfg: LayerConfig, inter: Optional[int] = None) -> int:
    """Bytes of gate+up+down of one expert in ``cfg.fmt`` (storage, scales included)."""
    I = cfg.moe_inter if inter is None else inter
    h = cfg.hidden
    n_el = 3 * I * h
    if cfg.fmt == "f32":
        return 4 * n_el
    if cfg.fmt == "bf16":
        return 2 * n_el
    if cfg.fmt == "q4_affine_g64":
        return n_el // 2 + 4 * (n_el // 64)
    if cfg.fmt == "nvfp4":
        return n_el // 2 + n_el // 16 + 3 * 4
    if cfg.fmt == "mxfp4":
        return n_el // 2 + n_el // 32
    if cfg.fmt == "fp8_e4m3":
        return n_el + 3 * 4
    raise ValueError(cfg.fmt)
