"""Float64 CPU oracle of the decode-time Mixture-of-Experts layer (m = 1..64 rows).

TEST INFRASTRUCTURE ONLY. Nothing in the library imports, links or executes this package. Only
``tests/``, the smoke check in ``__graft_entry__`` and the CPU-baseline leg of ``bench.py`` may
use it. It shares no code, table or constant with the CUDA library: it decodes the packed weight
bytes itself, routes, groups and evaluates every expert in plain numpy float64, row by row, in the
order the steps are described.

What it computes, per row r, with the sources it follows:

1. Router logits ``l = W_r x_r`` (metrale ``forward_bf16_grouped_decode.rs``: the per-row router
   is the first step of the grouped decode, module doc).
2. Selection keys and top-k:
   * softmax routing: key = logit (softmax is monotone, so the order is that of the
     probabilities);
   * sigmoid routing: key = sigmoid(l) + expert_bias when an expert bias is present (iron PR
     "refactor(gemm): split the gemv_q8 grab-bag by family": the biased router selects by the
     biased score and weights by the unbiased one), key = raw logit when the architecture selects
     on raw logits (frink-models ``routed_weight_site.rs`` module doc: Llama 4 takes the top-k of
     the raw logits, the same experts as on the sigmoid probabilities), else sigmoid(l).
   The k largest keys win; equal keys go to the lower expert id; slots are in descending key order.
   The sqrt-softplus router (iron PR, the ``router_sqrtsoftplus`` kernel of the moe family)
   ranks and weights like the sigmoid router with the score sqrt(softplus(l)) = sqrt(log(1+e^l))
   in place of sigmoid(l); the page names the router only, this is the plain reading of its name.
3. Routing weights: softmax probability (over all E) or unbiased sigmoid score of each selected
   expert, divided by their sum when ``norm_topk_prob``, then multiplied by
   ``routed_scaling_factor`` (mlxcel PR "perf(moe): wire lfm2 to the fused decode-MoE kernel":
   sigmoid gating, expert_bias for selection, norm_topk_prob, routed_scaling_factor).
4. Routed-weight site (frink-models ``routed_weight_site.rs``, ``routed_slot``): the slot's
   expert input is x and its output carries w, or, when the weight sits before the FFN (Llama 4),
   the input is w*x and the output carries 1.
5. Expert: ``down(silu(gate(x~)) * up(x~))`` with silu(z) = z * sigmoid(z); with the GeGLU
   activation (metrale ``helpers_a.rs``, ``set_gelu_activation``: the expert activation becomes
   ``gelu_mul``) the gate goes through GELU instead, in its tanh form (the form of the Gemma
   models that page wires it for).
6. Output: the sum over slots (in slot order) of weight * expert output, plus the shared expert,
   scaled by sigmoid(w_sg . x_r) for a sigmoid-gated shared expert (metrale
   ``forward_bf16_grouped_decode.rs``: the blend receives the layer input and the shared expert
   gate weight) or by 1 for a plain one.
7. Grouping of the (row, slot) pairs by expert (metrale ``forward_bf16_grouped_decode.rs``, the
   sort step and its outputs): a stable sort of pair ids p = r*k + s by expert id, the exclusive
   prefix of per-expert counts, the inverse permutation, and the ascending list of experts that
   received at least one pair.

Weight formats decoded here (storage defined by the library's pack helpers; 4-bit data is
``[n, k/2]`` bytes as in metrale ``helpers_a.rs``, ``transpose_experts_gpu``):
 * f32 / bf16: plain row-major ``[n, k]``;
 * 4-bit affine, group 64: ``w = scale * q + bias`` with fp16 scale and bias per 64 elements;
 * NVFP4: E2M1 codes, one E4M3 scale per 16 elements (the NVFP4 scale block of metrale
   ``helpers_a.rs``), one fp32 tensor scale per matrix (its ``weight_scale_2``):
   ``w = e2m1(q) * e4m3(s) * tensor_scale``;
 * FP8: E4M3 codes ``[n, k]`` (one byte per element) and one fp32 scale per expert matrix
   (the FP8 grouped decode of metrale ``forward_fp8_grouped_decode.rs``, whose scale layout
   the pages do not give; read as one scale per matrix): ``w = e4m3(q) * scale``;
 * MXFP4: E2M1 codes, one E8M0 scale per 32 elements (the native MXFP4 scale block of metrale
   ``helpers_a.rs``, the scale-block note of ``transpose_for_prefill_impl``), no tensor scale:
   ``w = e2m1(q) * 2**(s - 127)`` (E8M0 as the OCP Microscaling specification defines it).
Element 2j of a 4-bit row is the low nibble of byte j.

Every function here is pinned by a CPU test against the pages' worked example, closed forms,
library routines or brute force (see ``tests/test_oracle_*.py``).
"""
from __future__ import annotations

from typing import Dict, List, Optional, Sequence, Tuple

import numpy as np

# ---------------------------------------------------------------------------------------------
# Scalar storage formats
# ---------------------------------------------------------------------------------------------


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """bfloat16 storage -> float64 (bf16 is the upper half of an IEEE binary32)."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


def f16_to_f64(bits: np.ndarray) -> np.ndarray:
    """IEEE binary16 storage -> float64."""
    return np.asarray(bits, dtype=np.uint16).view(np.float16).astype(np.float64)


def e2m1_value(code: np.ndarray) -> np.ndarray:
    """FP4 E2M1 code -> value: sign bit 3, exponent bits 2..1 (bias 1), mantissa bit 0.

    Exponent field 0 is subnormal: value = m * 2**-1. Otherwise 2**(e-1) * (1 + m/2).
    """
    c = np.asarray(code, dtype=np.int64)
    s = (c >> 3) & 1
    e = (c >> 1) & 3
    m = c & 1
    mag = np.where(e == 0, 0.5 * m, np.exp2(e - 1.0) * (1.0 + 0.5 * m))
    return np.where(s == 1, -mag, mag)


def e4m3_value(code: np.ndarray) -> np.ndarray:
    """FP8 E4M3 code -> value: sign bit 7, exponent bits 6..3 (bias 7), mantissa bits 2..0.

    Exponent field 0 is subnormal: 2**-6 * m/8. Exponent 15 with mantissa 7 is NaN (no infinity).
    """
    c = np.asarray(code, dtype=np.int64)
    s = (c >> 7) & 1
    e = (c >> 3) & 15
    m = c & 7
    mag = np.where(e == 0, np.exp2(-6.0) * (m / 8.0), np.exp2(e - 7.0) * (1.0 + m / 8.0))
    mag = np.where((e == 15) & (m == 7), np.nan, mag)
    return np.where(s == 1, -mag, mag)


def e8m0_value(code: np.ndarray) -> np.ndarray:
    """E8M0 scale code -> value: an unsigned biased exponent, 2**(code - 127); 0xFF is NaN."""
    c = np.asarray(code, dtype=np.int64)
    return np.where(c == 255, np.nan, np.exp2(c - 127.0))


def unpack_nibbles(packed: np.ndarray, k: int) -> np.ndarray:
    """``[n, k/2]`` bytes -> ``[n, k]`` 4-bit codes; element 2j is the low nibble of byte j."""
    p = np.asarray(packed, dtype=np.uint8)
    n = p.shape[0]
    out = np.empty((n, k), dtype=np.uint8)
    out[:, 0::2] = p & 0x0F
    out[:, 1::2] = p >> 4
    return out


def decode_matrix(slab, e: int = 0) -> np.ndarray:
    """Expert ``e`` of a weight slab -> float64 ``[n, k]``.

    ``slab`` carries ``fmt, n, k, data, scales, biases, tensor_scale`` with expert as the leading
    axis of every array.
    """
    n, k = slab.n, slab.k
    if slab.fmt == "f32":
        return np.asarray(slab.data[e], dtype=np.float32).astype(np.float64)
    if slab.fmt == "bf16":
        return bf16_to_f64(slab.data[e])
    if slab.fmt == "q4_affine_g64":
        q = unpack_nibbles(slab.data[e], k).astype(np.float64)
        scale = np.repeat(f16_to_f64(slab.scales[e]), 64, axis=1)
        bias = np.repeat(f16_to_f64(slab.biases[e]), 64, axis=1)
        return scale * q + bias
    if slab.fmt == "nvfp4":
        v = e2m1_value(unpack_nibbles(slab.data[e], k))
        blk = np.repeat(e4m3_value(slab.scales[e]), 16, axis=1)
        return v * blk * float(np.float32(slab.tensor_scale[e]))
    if slab.fmt == "mxfp4":
        v = e2m1_value(unpack_nibbles(slab.data[e], k))
        return v * np.repeat(e8m0_value(slab.scales[e]), 32, axis=1)
    if slab.fmt == "fp8_e4m3":
        v = e4m3_value(np.asarray(slab.data[e], dtype=np.uint8).reshape(n, k))
        return v * float(np.float32(slab.tensor_scale[e]))
    raise ValueError(f"unknown format {slab.fmt!r}")


def decode_activations(x: np.ndarray, x_dtype: str) -> np.ndarray:
    if x_dtype == "bf16":
        return bf16_to_f64(x)
    if x_dtype == "f32":
        return np.asarray(x, dtype=np.float32).astype(np.float64)
    raise ValueError(x_dtype)


# ---------------------------------------------------------------------------------------------
# Routing
# ---------------------------------------------------------------------------------------------

# Architectures whose routing weight multiplies the routed expert's input (frink-models
# ``routed_weight_site.rs``, ``ROUTED_WEIGHT_BEFORE_FFN``): only Llama 4.
ROUTED_WEIGHT_BEFORE_FFN = ("llama4",)


def weight_before_ffn(arch: str) -> bool:
    return arch in ROUTED_WEIGHT_BEFORE_FFN


def sigmoid(z):
    z = np.asarray(z, dtype=np.float64)
    with np.errstate(over="ignore"):
        return 1.0 / (1.0 + np.exp(-z))


def silu(z):
    """silu(z) = z * sigmoid(z)."""
    z = np.asarray(z, dtype=np.float64)
    return z * sigmoid(z)


def softplus(z):
    """softplus(z) = log(1 + e^z), written as max(z, 0) + log1p(e^-|z|) (no overflow)."""
    z = np.asarray(z, dtype=np.float64)
    return np.maximum(z, 0.0) + np.log1p(np.exp(-np.abs(z)))


def sqrtsoftplus(z):
    """The sqrt-softplus router score: sqrt(softplus(z)) (a positive, increasing score)."""
    return np.sqrt(softplus(z))


def gelu_tanh(z):
    """GELU in its tanh form: z/2 * (1 + tanh(sqrt(2/pi) * (z + 0.044715 z^3)))."""
    z = np.asarray(z, dtype=np.float64)
    return 0.5 * z * (1.0 + np.tanh(np.sqrt(2.0 / np.pi) * (z + 0.044715 * z ** 3)))


def router_score(l, routing: str):
    """Per-expert score of the non-softmax routers: sigmoid or sqrt-softplus of the logit."""
    if routing == "sigmoid":
        return sigmoid(l)
    if routing == "sqrtsoftplus":
        return sqrtsoftplus(l)
    raise ValueError(routing)


def router_logits(x64: np.ndarray, wr64: np.ndarray) -> np.ndarray:
    """``[m, h] x [E, h] -> [m, E]``, one matrix-vector product per row."""
    return np.stack([wr64 @ np.array(row) for row in x64])


def selection_keys(logits_row: np.ndarray, cfg, expert_bias: Optional[np.ndarray]) -> np.ndarray:
    """The per-expert key that top-k ranks (see the module doc, step 2)."""
    l = np.asarray(logits_row, dtype=np.float64)
    if cfg.routing == "softmax":
        return l.copy()
    if cfg.routing not in ("sigmoid", "sqrtsoftplus"):
        raise ValueError(cfg.routing)
    if cfg.select_on_raw_logits:
        return l.copy()
    s = router_score(l, cfg.routing)
    if cfg.has_expert_bias:
        return s + np.asarray(expert_bias, dtype=np.float32).astype(np.float64)
    return s


def select_top_k(keys: Sequence[float], k: int) -> List[int]:
    """Ids of the k largest keys, in descending key order; equal keys -> lower id first."""
    order = sorted(range(len(keys)), key=lambda e: (-float(keys[e]), e))
    return order[:k]


def routing_weights(logits_row: np.ndarray, ids: Sequence[int], cfg) -> np.ndarray:
    """Weights of the selected experts (module doc, step 3)."""
    l = np.asarray(logits_row, dtype=np.float64)
    if cfg.routing == "softmax":
        p = np.exp(l - l.max())
        p /= p.sum()
        w = p[list(ids)]
    else:
        w = router_score(l[list(ids)], cfg.routing)
    if cfg.norm_topk_prob:
        w = w / w.sum()
    return w * float(np.float32(cfg.routed_scaling_factor))


def route_row(logits_row, cfg, expert_bias) -> Tuple[List[int], np.ndarray]:
    ids = select_top_k(selection_keys(logits_row, cfg, expert_bias), cfg.top_k)
    return ids, routing_weights(logits_row, ids, cfg)


def routed_slot(x: np.ndarray, w: float, before_ffn: bool):
    """One slot's expert input and the weight its output carries: ``(x, w)`` or ``(w*x, 1)``."""
    x = np.asarray(x, dtype=np.float64)
    if before_ffn:
        return x * w, 1.0
    return x, w


# ---------------------------------------------------------------------------------------------
# Grouping of (row, slot) pairs by expert
# ---------------------------------------------------------------------------------------------


def group_by_expert(idx: np.ndarray, num_experts: int) -> Dict[str, np.ndarray]:
    """Stable grouping of the pairs p = r*k + s by expert id.

    Returns ``sorted_pairs`` (pair ids ordered by (expert, p)), ``expert_offsets`` (E+1,
    exclusive prefix of counts), ``token_to_perm`` (position of each pair in sorted order),
    ``active`` (ascending ids with a non-zero count) and ``active_count``.
    """
    flat = np.asarray(idx, dtype=np.int64).ravel()
    sorted_pairs = np.argsort(flat, kind="stable")
    counts = np.bincount(flat, minlength=num_experts)
    offsets = np.concatenate([[0], np.cumsum(counts)])
    token_to_perm = np.empty_like(sorted_pairs)
    token_to_perm[sorted_pairs] = np.arange(flat.size)
    active = np.nonzero(counts)[0]
    return {
        "sorted_pairs": sorted_pairs.astype(np.int32),
        "expert_offsets": offsets.astype(np.int32),
        "token_to_perm": token_to_perm.astype(np.int32),
        "active": active.astype(np.int32),
        "active_count": np.int32(active.size),
    }


# ---------------------------------------------------------------------------------------------
# Experts and the layer
# ---------------------------------------------------------------------------------------------


def swiglu_expert(wg: np.ndarray, wu: np.ndarray, wd: np.ndarray, xin: np.ndarray,
                  activation: str = "swiglu") -> np.ndarray:
    """``down(silu(gate(x)) * up(x))`` for one input vector; with ``activation="geglu"`` the gate
    goes through GELU (tanh form) instead of SiLU."""
    xin = np.array(xin, dtype=np.float64)
    g = wg @ xin
    if activation == "swiglu":
        a = silu(g)
    elif activation == "geglu":
        a = gelu_tanh(g)
    else:
        raise ValueError(activation)
    return wd @ (a * (wu @ xin))


class OracleLayer:
    """Float64 view of one layer's inputs, decoding each expert only when it is used.

    ``source`` provides ``cfg``, ``router_w()``, ``expert_bias()``, ``shared_gate_w()``,
    ``routed_expert(e, proj)`` and ``shared(proj)`` returning raw storage arrays / slabs.
    """

    def __init__(self, source, cache_experts: int = 4):
        self.src = source
        self.cfg = source.cfg
        self._router = None
        self._cache: Dict[object, Tuple[np.ndarray, np.ndarray, np.ndarray]] = {}
        self._cache_order: List[object] = []
        self._cache_max = cache_experts

    def router(self) -> np.ndarray:
        if self._router is None:
            self._router = decode_activations(self.src.router_w(), self.cfg.x_dtype)
        return self._router

    def shared_gate(self) -> Optional[np.ndarray]:
        sg = self.src.shared_gate_w()
        return None if sg is None else decode_activations(sg, self.cfg.x_dtype)

    def _remember(self, key, val):
        self._cache[key] = val
        self._cache_order.append(key)
        while len(self._cache_order) > self._cache_max:
            del self._cache[self._cache_order.pop(0)]
        return val

    def expert(self, e: int):
        key = ("r", int(e))
        if key in self._cache:
            return self._cache[key]
        mats = tuple(decode_matrix(self.src.routed_expert(int(e), p), 0)
                     for p in ("gate", "up", "down"))
        return self._remember(key, mats)

    def shared(self):
        key = ("s",)
        if key in self._cache:
            return self._cache[key]
        mats = tuple(decode_matrix(self.src.shared(p), 0) for p in ("gate", "up", "down"))
        return self._remember(key, mats)


def route(layer: OracleLayer, x: np.ndarray):
    """Router logits, top-k ids, weights and the shared gate of every row."""
    cfg = layer.cfg
    x64 = decode_activations(x, cfg.x_dtype)
    logits = router_logits(x64, layer.router())
    bias = layer.src.expert_bias()
    m = x64.shape[0]
    idx = np.zeros((m, cfg.top_k), dtype=np.int32)
    w = np.zeros((m, cfg.top_k), dtype=np.float64)
    for r in range(m):
        ids, wr = route_row(logits[r], cfg, bias)
        idx[r] = ids
        w[r] = wr
    gamma = None
    if cfg.shared_kind == "sigmoid_gate":
        sg = layer.shared_gate()
        gamma = np.array([sigmoid(sg @ np.array(row)) for row in x64])
    return {"x64": x64, "logits": logits, "idx": idx, "w": w, "gamma": gamma}


def moe_forward(layer: OracleLayer, x: np.ndarray, rows: Optional[Sequence[int]] = None):
    """Outputs ``[len(rows), h]`` (float64) of the layer for the rows ``rows`` of ``x``.

    Every row is evaluated on its own: its output does not depend on the other rows. Experts are
    decoded once and applied to every selected slot that uses them; per row the slot outputs are
    summed in slot order, then the shared expert is added.
    """
    cfg = layer.cfg
    rt = route(layer, x)
    x64, idx, w, gamma = rt["x64"], rt["idx"], rt["w"], rt["gamma"]
    m = x64.shape[0]
    rows = list(range(m)) if rows is None else [int(r) for r in rows]
    k = cfg.top_k
    y = {}
    users: Dict[int, List[Tuple[int, int]]] = {}
    for r in rows:
        for s in range(k):
            users.setdefault(int(idx[r, s]), []).append((r, s))
    weight_site = {}
    for e in sorted(users):
        wg, wu, wd = layer.expert(e)
        for r, s in users[e]:
            xin, omega = routed_slot(x64[r], w[r, s], cfg.weight_before_ffn)
            y[(r, s)] = swiglu_expert(wg, wu, wd, xin, cfg.activation)
            weight_site[(r, s)] = omega
    out = np.zeros((len(rows), cfg.hidden), dtype=np.float64)
    for i, r in enumerate(rows):
        acc = np.zeros(cfg.hidden, dtype=np.float64)
        for s in range(k):
            acc = acc + weight_site[(r, s)] * y[(r, s)]
        out[i] = acc
    if cfg.shared_kind in ("plain", "sigmoid_gate") and cfg.shared_inter > 0:
        sg, su, sd = layer.shared()
        for i, r in enumerate(rows):
            g = 1.0 if gamma is None else gamma[r]
            out[i] = out[i] + g * swiglu_expert(sg, su, sd, x64[r], cfg.activation)
    aux = dict(rt)
    aux.update(group_by_expert(idx, cfg.num_experts))
    return out, aux


def selection_key_fn(source):
    """A ``row -> keys`` function for the synthetic generator's selection-gap rule."""
    cfg = source.cfg
    wr = decode_activations(source.router_w(), cfg.x_dtype)
    bias = source.expert_bias()

    def key_fn(row):
        l = wr @ decode_activations(np.asarray(row)[None, :], cfg.x_dtype)[0]
        return selection_keys(l, cfg, bias)

    return key_fn
