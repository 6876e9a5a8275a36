"""Device-memory plumbing around the C ABI: allocate the outputs and workspaces
of the three stages (layer preparation, merge, STE backward) for a list of
layers and build their descriptors. No arithmetic of the method happens here;
every stage runs in libintlora.so.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch

from . import binding as B
from .workloads import LayerSpec, packed_row_bytes


def code_row_bytes(n: int, bits: int) -> int:
    return packed_row_bytes(n, bits, 16)


def out_dtype(spec: LayerSpec) -> torch.dtype:
    variant = 0 if spec.variant == "mul" else 1
    nbytes = B.intlora_merge_out_bytes(variant, spec.w_bits, spec.out_bits)
    return {1: torch.int8, 2: torch.int16, 4: torch.int32}[nbytes]


@dataclass
class LayerState:
    """Device tensors of one layer through the whole path."""
    spec: LayerSpec
    W: torch.Tensor                     # fp32 d x n (input of preparation)
    A: torch.Tensor                     # fp32 d x r
    B: torch.Tensor                     # fp32 r x n
    sigma: torch.Tensor                 # float64 [2]: sigma_W, sigma_R
    w_round: torch.Tensor               # uint8 d x ld
    s: torch.Tensor
    z: torch.Tensor
    out: torch.Tensor                   # P or M
    sbar: torch.Tensor
    zbar: torch.Tensor
    code: torch.Tensor | None = None
    G: torch.Tensor | None = None       # bf16 d x n (STE)
    A16: torch.Tensor | None = None
    B16: torch.Tensor | None = None
    dA: torch.Tensor | None = None
    dB: torch.Tensor | None = None
    extra: dict = field(default_factory=dict)

    def aux_job(self) -> B.AuxJob:
        sp = self.spec
        return B.AuxJob(self.W, sp.seed, sp.stream_id, sp.alpha, sp.w_bits, self.sigma[0:1],
                        self.sigma[1:2], None, self.w_round, self.s, self.z, sp.distribution)

    def layer(self, pass_sigma_r: bool = True) -> B.Layer:
        sp = self.spec
        return B.Layer(self.w_round, sp.n, sp.w_bits, self.s, self.z, self.A, self.B, sp.seed,
                       sp.stream_id, sp.alpha, self.sigma[0:1],
                       self.sigma[1:2] if pass_sigma_r else None, sp.distribution)

    def merge_out(self) -> B.MergeOut:
        return B.MergeOut(self.out, self.sbar, self.zbar if self.spec.variant == "mul" else None,
                          self.code)

    def ste_job(self, masked: bool = False) -> B.SteJob:
        """masked: G is kept only where W_round != z (the layer's own codes)."""
        if masked:
            return B.SteJob(self.G, self.A16, self.B16, self.dA, self.dB, self.w_round,
                            self.spec.w_bits, self.z)
        return B.SteJob(self.G, self.A16, self.B16, self.dA, self.dB)


def allocate(spec: LayerSpec, W, A, Bm, device, G=None, A16=None, B16=None,
             want_code: bool = False) -> LayerState:
    d, n, r = spec.d, spec.n, spec.r
    dev = torch.device(device)
    st = LayerState(
        spec=spec, W=W, A=A, B=Bm,
        sigma=torch.zeros(2, dtype=torch.float64, device=dev),
        w_round=torch.zeros(d, code_row_bytes(n, spec.w_bits), dtype=torch.uint8, device=dev),
        s=torch.zeros(d, dtype=torch.float32, device=dev),
        z=torch.zeros(d, dtype=torch.int32, device=dev),
        out=torch.empty(d, n, dtype=out_dtype(spec), device=dev),
        sbar=torch.zeros(d, dtype=torch.float32, device=dev),
        zbar=torch.zeros(d, dtype=torch.int32, device=dev),
        code=torch.empty(d, n, dtype=torch.uint8, device=dev) if want_code else None,
    )
    if G is not None:
        st.G, st.A16, st.B16 = G, A16, B16
        st.dA = torch.empty(d, r, dtype=torch.float32, device=dev)
        st.dB = torch.empty(r, n, dtype=torch.float32, device=dev)
    return st


def arena(tensors: list[torch.Tensor], device) -> tuple[torch.Tensor, list[torch.Tensor], list[int]]:
    """One device buffer holding copies of `tensors` (each at a 256-byte
    aligned offset), views of it with the tensors' shapes and dtypes, and the
    byte offset of each view: a host mirror of the buffer then moves with one
    copy per direction (or one per contiguous run of views)."""
    offsets, total = [], 0
    for t in tensors:
        offsets.append(total)
        total += (t.numel() * t.element_size() + 255) // 256 * 256
    buf = torch.empty(max(total, 256), dtype=torch.uint8, device=device)
    views = []
    for t, off in zip(tensors, offsets):
        nb = t.numel() * t.element_size()
        v = buf[off:off + nb].view(t.dtype).view(t.shape)
        v.copy_(t)
        views.append(v)
    return buf, views, offsets


def pack_io(states: list[LayerState], device) -> tuple[torch.Tensor, torch.Tensor]:
    """Moves every layer's inputs (W, A, B and the STE operands) into one
    arena and its outputs (merged weights, scales, zero-points, gradients)
    into another; returns (inputs, outputs). A layer's views are contiguous in
    each arena, layers in list order: st.extra["in"] and st.extra["out"] hold
    each layer's [begin, end) byte range. Build the Path afterwards."""
    in_keys = ("W", "A", "B", "G", "A16", "B16")
    out_keys = ("out", "sbar", "zbar", "dA", "dB")
    groups = []
    for tag, keys in (("in", in_keys), ("out", out_keys)):
        slots = [(st, k) for st in states for k in keys if getattr(st, k) is not None]
        buf, views, offsets = arena([getattr(st, k) for st, k in slots], device)
        for (st, k), v, off in zip(slots, views, offsets):
            setattr(st, k, v)
            lo, hi = st.extra.get(tag, (off, off))
            st.extra[tag] = (min(lo, off), max(hi, off + v.numel() * v.element_size()))
        groups.append(buf)
    return groups[0], groups[1]


def workspace(nbytes: int, device) -> torch.Tensor | None:
    if nbytes <= 0:
        return None
    return torch.empty(nbytes, dtype=torch.uint8, device=device)


class Path:
    """The per-layer hot path over a list of layers: preparation (aux + base
    quantization), merge (MUL or SHIFT) and, where requested, the STE
    backward; each stage is one batched call (a handful of launches)."""

    def __init__(self, states: list[LayerState], device, masked_ste: bool = False):
        self.states = states
        self.device = device
        self.masked_ste = masked_ste
        self.mul = [s for s in states if s.spec.variant == "mul"]
        self.shift = [s for s in states if s.spec.variant == "shift"]
        self.ste = [s for s in states if s.G is not None]
        # descriptors are converted to C structs once: the buffers never move
        self.aux_jobs = B.Descriptors(s.aux_job() for s in states)
        self.ws_aux = workspace(B.intlora_gen_aux_workspace_size(self.aux_jobs), device)
        self.ws_merge = workspace(B.intlora_merge_workspace_size(
            [s.layer() for s in states]), device)
        groups = {}
        for s in self.mul:
            groups.setdefault(("mul", s.spec.out_bits), []).append(s)
        for s in self.shift:
            groups.setdefault(("shift", s.spec.out_bits), []).append(s)
        self.merge_groups = [(kind, bits, B.Descriptors(s.layer() for s in sts),
                              B.Descriptors(s.merge_out() for s in sts))
                             for (kind, bits), sts in groups.items()]
        self.ste_jobs = (B.Descriptors(s.ste_job(masked_ste) for s in self.ste)
                         if self.ste else None)
        self.ws_ste = (workspace(B.intlora_ste_workspace_size(self.ste_jobs), device)
                       if self.ste else None)

    def prepare(self, stream=None):
        B.intlora_gen_aux_batched(self.aux_jobs, self.ws_aux, stream)

    def merge(self, stream=None):
        for kind, bits, layers, outs in self.merge_groups:
            if kind == "mul":
                B.intlora_merge_mul_batched(layers, outs, bits, self.ws_merge, stream)
            else:
                B.intlora_merge_shift_batched(layers, outs, bits, self.ws_merge, stream)

    def backward(self, stream=None):
        if self.ste_jobs is not None:
            B.intlora_ste_backward_batched(self.ste_jobs, self.ws_ste, stream)

    def step(self, stream=None):
        self.prepare(stream)
        self.merge(stream)
        self.backward(stream)
