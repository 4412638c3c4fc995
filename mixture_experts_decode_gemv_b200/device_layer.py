"""Device copies of a synthetic MoE layer and the C tables that describe them.

``DeviceLayer`` uploads every array of a ``SyntheticLayer`` into CUDA memory (torch tensors, one
slab per projection, expert e at ``e * expert_stride``) and fills the ``moe_cfg`` /
``moe_expert_table`` structs of the C ABI. ``forward`` is a direct call of
``moe_decode_forward``; there is no other implementation.
"""
from __future__ import annotations

from typing import Optional, Sequence

import numpy as np
import torch

from . import binding as B
from .synthetic import LayerConfig, MatrixSlab, SyntheticLayer


def make_cfg(cfg: LayerConfig, out_dtype: str = "f32") -> B.moe_cfg:
    c = B.moe_cfg()
    c.hidden = cfg.hidden
    c.num_experts = cfg.num_experts
    c.top_k = cfg.top_k
    c.moe_inter = cfg.moe_inter
    c.shared_inter = cfg.shared_inter if cfg.has_shared else 0
    c.routing = B.ROUTING_CODES[cfg.routing]
    c.norm_topk_prob = int(cfg.norm_topk_prob)
    c.select_on_raw_logits = int(cfg.select_on_raw_logits)
    c.has_expert_bias = int(cfg.has_expert_bias)
    c.routed_scaling_factor = float(cfg.routed_scaling_factor)
    c.weight_before_ffn = int(cfg.weight_before_ffn)
    c.shared_kind = B.SHARED_CODES[cfg.shared_kind] if cfg.has_shared else B.MOE_SHARED_NONE
    c.x_dtype = B.FORMAT_CODES[cfg.x_dtype]
    c.out_dtype = B.FORMAT_CODES[out_dtype]
    c.activation = B.ACTIVATION_CODES[cfg.activation]
    return c


def _bytes(a: np.ndarray) -> np.ndarray:
    return np.ascontiguousarray(a).view(np.uint8).reshape(-1)


class DeviceSlab:
    """One projection of E experts in device memory."""

    def __init__(self, fmt: str, n: int, k: int, E: int, per_expert, device):
        """``per_expert(e) -> MatrixSlab`` (one expert); uploaded expert by expert."""
        first = per_expert(0)
        self.fmt, self.n, self.k, self.E = fmt, n, k, E
        self.stride = _bytes(first.data).size
        self.sstride = 0 if first.scales is None else _bytes(first.scales).size
        self.packed = torch.empty(E * self.stride, dtype=torch.uint8, device=device)
        self.scales = (torch.empty(E * self.sstride, dtype=torch.uint8, device=device)
                       if first.scales is not None else None)
        self.biases = (torch.empty(E * self.sstride, dtype=torch.uint8, device=device)
                       if first.biases is not None else None)
        self.tscale = (torch.empty(E, dtype=torch.float32, device=device)
                       if first.tensor_scale is not None else None)
        for e in range(E):
            s = first if e == 0 else per_expert(e)
            self.packed[e * self.stride:(e + 1) * self.stride].copy_(
                torch.from_numpy(_bytes(s.data)))
            if self.scales is not None:
                self.scales[e * self.sstride:(e + 1) * self.sstride].copy_(
                    torch.from_numpy(_bytes(s.scales)))
            if self.biases is not None:
                self.biases[e * self.sstride:(e + 1) * self.sstride].copy_(
                    torch.from_numpy(_bytes(s.biases)))
            if self.tscale is not None:
                self.tscale[e:e + 1].copy_(torch.from_numpy(
                    np.asarray(s.tensor_scale, np.float32).reshape(1)))

    def clone(self) -> "DeviceSlab":
        c = DeviceSlab.__new__(DeviceSlab)
        c.__dict__.update(self.__dict__)
        for name in ("packed", "scales", "biases", "tscale"):
            t = getattr(self, name)
            setattr(c, name, None if t is None else t.clone())
        return c

    def matrix(self) -> B.moe_matrix:
        mm = B.moe_matrix()
        mm.format = B.FORMAT_CODES[self.fmt]
        mm.packed = self.packed.data_ptr()
        mm.scales = self.scales.data_ptr() if self.scales is not None else None
        mm.biases = self.biases.data_ptr() if self.biases is not None else None
        mm.tensor_scale = self.tscale.data_ptr() if self.tscale is not None else None
        mm.expert_stride = self.stride
        mm.scale_stride = self.sstride
        return mm

    def nbytes(self) -> int:
        return sum(t.numel() * t.element_size() for t in
                   (self.packed, self.scales, self.biases, self.tscale) if t is not None)


def _dense_to_device(a: Optional[np.ndarray], device):
    if a is None:
        return None
    a = np.ascontiguousarray(a)
    t = torch.from_numpy(a.view(np.int16) if a.dtype == np.uint16 else a)
    return t.to(device)


class DeviceLayer:
    """A ``SyntheticLayer`` resident in device memory plus its C-ABI descriptors."""

    def __init__(self, lay: SyntheticLayer, device="cuda", experts: Optional[Sequence[int]] = None,
                 out_dtype: str = "f32"):
        cfg = lay.cfg
        self.cfg = cfg
        self.device = torch.device(device)
        self.c = make_cfg(cfg, out_dtype)
        self.out_dtype = out_dtype
        self.router_w = _dense_to_device(lay.router_w(), device)
        self.expert_bias = _dense_to_device(lay.expert_bias(), device)
        self.shared_gate_w = _dense_to_device(lay.shared_gate_w(), device)
        want = None if experts is None else set(int(e) for e in experts)
        h, I, S = cfg.hidden, cfg.moe_inter, cfg.shared_inter

        def routed_getter(proj):
            def get(e):
                if want is None or e in want:
                    return lay.routed_expert(e, proj)
                n, k = (I, h) if proj != "down" else (h, I)
                from .synthetic import _zeros_like_expert
                return _zeros_like_expert(cfg.fmt, n, k)
            return get

        self.routed_slabs = {}
        for proj in ("gate", "up", "down"):
            n, k = (I, h) if proj != "down" else (h, I)
            self.routed_slabs[proj] = DeviceSlab(cfg.fmt, n, k, cfg.num_experts,
                                                 routed_getter(proj), device)
        self.shared_slabs = None
        if cfg.has_shared:
            self.shared_slabs = {}
            for proj in ("gate", "up", "down"):
                n, k = (S, h) if proj != "down" else (h, S)
                self.shared_slabs[proj] = DeviceSlab(cfg.fmt, n, k, 1,
                                                     lambda e, p=proj: lay.shared(p), device)
        self._tables()

    def _tables(self):
        self.routed = B.moe_expert_table(self.routed_slabs["gate"].matrix(),
                                         self.routed_slabs["up"].matrix(),
                                         self.routed_slabs["down"].matrix())
        self.shared = None
        if self.shared_slabs is not None:
            self.shared = B.moe_expert_table(self.shared_slabs["gate"].matrix(),
                                             self.shared_slabs["up"].matrix(),
                                             self.shared_slabs["down"].matrix())

    def replica(self) -> "DeviceLayer":
        """A copy of every weight in fresh device memory (same values, other addresses)."""
        r = DeviceLayer.__new__(DeviceLayer)
        r.__dict__.update(self.__dict__)
        r.router_w = self.router_w.clone()
        r.expert_bias = None if self.expert_bias is None else self.expert_bias.clone()
        r.shared_gate_w = None if self.shared_gate_w is None else self.shared_gate_w.clone()
        r.routed_slabs = {k: v.clone() for k, v in self.routed_slabs.items()}
        r.shared_slabs = (None if self.shared_slabs is None
                          else {k: v.clone() for k, v in self.shared_slabs.items()})
        r._tables()
        return r

    def weight_bytes(self) -> int:
        n = sum(s.nbytes() for s in self.routed_slabs.values())
        if self.shared_slabs:
            n += sum(s.nbytes() for s in self.shared_slabs.values())
        return n

    # ---- calls -----------------------------------------------------------------------------
    def workspace_bytes(self, m: int) -> int:
        return B.moe_workspace_bytes(self.c, m)

    def new_workspace(self, m: int, stream=None) -> torch.Tensor:
        nb = self.workspace_bytes(m)
        ws = torch.empty(nb, dtype=torch.uint8, device=self.device)
        B.moe_workspace_init(ws, nb, stream if stream is not None else
                             torch.cuda.current_stream(self.device))
        return ws

    def x_to_device(self, x: np.ndarray) -> torch.Tensor:
        return _dense_to_device(x, self.device)

    def new_out(self, m: int) -> torch.Tensor:
        dt = torch.float32 if self.out_dtype == "f32" else torch.bfloat16
        return torch.empty((m, self.cfg.hidden), dtype=dt, device=self.device)

    def forward(self, x: torch.Tensor, out: torch.Tensor, ws: torch.Tensor, stream=None) -> None:
        m = x.shape[0]
        st = stream if stream is not None else torch.cuda.current_stream(self.device)
        B.moe_decode_forward(self.c, m, x, self.router_w, self.expert_bias, self.routed,
                             self.shared, self.shared_gate_w, out, ws, ws.numel(), st)

    def launches(self, m: int) -> int:
        """Kernel launches one forward call with m rows makes on this device."""
        with torch.cuda.device(self.device):
            return B.moe_decode_launches(self.c, m, self.routed, self.shared)

    def read_routing(self, m: int, ws: torch.Tensor, stream=None):
        st = stream if stream is not None else torch.cuda.current_stream(self.device)
        return B.moe_decode_read_routing(self.c, m, ws, ws.numel(), st)

    def device_status(self, ws: torch.Tensor, stream=None) -> int:
        st = stream if stream is not None else torch.cuda.current_stream(self.device)
        return B.moe_get_device_status(ws, ws.numel(), st)
