"""Thin ctypes binding of libintlora.so (the C ABI in include/intlora.h).

Argument marshalling only: torch tensors are passed as device pointers and
every step of the computation runs in the library's CUDA kernels. Function
names match the C entry points. Importing works without a GPU; the first call
loads the library and raises ``IntLoRAError``/``OSError`` if it is missing or a
call fails (there is no fallback of any kind).
"""
from __future__ import annotations

import ctypes
import re
from dataclasses import dataclass
from pathlib import Path
from typing import Optional, Sequence

PKG = Path(__file__).resolve().parent
LIB_PATH = PKG / "libintlora.so"
HEADER = PKG.parent / "include" / "intlora.h"

_c_i64, _c_i32, _c_u64, _c_u32 = ctypes.c_int64, ctypes.c_int32, ctypes.c_uint64, ctypes.c_uint32
_c_f32, _c_ptr, _c_size = ctypes.c_float, ctypes.c_void_p, ctypes.c_size_t

DIST_LAPLACE, DIST_GAUSSIAN, DIST_CAUCHY, DIST_STUDENT_T2 = 0, 1, 2, 3   # INTLORA_DIST_*

STATUS = {0: "INTLORA_OK", 1: "INTLORA_ERR_INVALID_ARG", 2: "INTLORA_ERR_UNSUPPORTED",
          3: "INTLORA_ERR_WORKSPACE", 4: "INTLORA_ERR_CUDA", 5: "INTLORA_ERR_TIMEOUT"}


class IntLoRAError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS.get(status, status)}: {message}")
        self.status = status


class intlora_aux_job(ctypes.Structure):
    _fields_ = [("W", _c_ptr), ("d", _c_i64), ("n", _c_i64), ("seed", _c_u64),
                ("stream_id", _c_u32), ("alpha", _c_f32), ("w_bits", _c_i32),
                ("sigma_w_out", _c_ptr), ("sigma_r_out", _c_ptr), ("r_star_out", _c_ptr),
                ("w_round_out", _c_ptr), ("ld_w_out", _c_i64), ("s_out", _c_ptr),
                ("z_out", _c_ptr), ("distribution", _c_i32)]


class intlora_layer(ctypes.Structure):
    _fields_ = [("d", _c_i64), ("n", _c_i64), ("r", _c_i32), ("w_bits", _c_i32),
                ("w_round", _c_ptr), ("ld_w", _c_i64), ("s", _c_ptr), ("z", _c_ptr),
                ("A", _c_ptr), ("B", _c_ptr), ("seed", _c_u64), ("stream_id", _c_u32),
                ("alpha", _c_f32), ("sigma_w", _c_ptr), ("sigma_r", _c_ptr),
                ("distribution", _c_i32)]


class intlora_merge_out(ctypes.Structure):
    _fields_ = [("out", _c_ptr), ("sbar", _c_ptr), ("zbar", _c_ptr), ("code", _c_ptr)]


class intlora_ste_job(ctypes.Structure):
    _fields_ = [("G", _c_ptr), ("A", _c_ptr), ("B", _c_ptr), ("d", _c_i64), ("n", _c_i64),
                ("r", _c_i32), ("dA", _c_ptr), ("dB", _c_ptr), ("mask_codes", _c_ptr),
                ("mask_ld", _c_i64), ("mask_bits", _c_i32), ("mask_z", _c_ptr)]


class intlora_fakequant_job(ctypes.Structure):
    _fields_ = [("q", _c_ptr), ("q_bytes", _c_i32), ("sbar", _c_ptr), ("d", _c_i64), ("n", _c_i64),
                ("w_out", _c_ptr)]


class intlora_linear_job(ctypes.Structure):
    _fields_ = [("X", _c_ptr), ("W", _c_ptr), ("tokens", _c_i64), ("d", _c_i64), ("n", _c_i64),
                ("Y", _c_ptr), ("y_bf16", _c_i32)]


class intlora_train_backward_job(ctypes.Structure):
    _fields_ = [("X", _c_ptr), ("dY", _c_ptr), ("W", _c_ptr), ("A", _c_ptr), ("B", _c_ptr),
                ("tokens", _c_i64), ("d", _c_i64), ("n", _c_i64), ("r", _c_i32),
                ("dX", _c_ptr), ("dA", _c_ptr), ("dB", _c_ptr)]


class intlora_int_gemm_job(ctypes.Structure):
    _fields_ = [("X", _c_ptr), ("x_scale", _c_ptr), ("W", _c_ptr), ("w_scale", _c_ptr),
                ("tokens", _c_i64), ("d", _c_i64), ("n", _c_i64), ("Y", _c_ptr),
                ("y_bf16", _c_i32)]


_P = ctypes.POINTER
_SIGNATURES = {
    "intlora_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "intlora_last_error": (ctypes.c_char_p, []),
    "intlora_version": (ctypes.c_int, []),
    "intlora_device_timeouts": (_c_u32, []),
    "intlora_kernel_launches": (_c_u64, []),
    "intlora_device_status": (ctypes.c_int, []),
    "intlora_selftest_bounded_wait": (ctypes.c_int, [_c_u32, _c_ptr]),
    "intlora_merge_out_bytes": (_c_i32, [_c_i32, _c_i32, _c_i32]),
    "intlora_gen_aux_workspace_size": (_c_size, [_P(intlora_aux_job), _c_i32]),
    "intlora_gen_aux": (ctypes.c_int, [_c_ptr, _c_i64, _c_i64, _c_u64, _c_u32, _c_f32, _c_i32,
                                       _c_ptr, _c_ptr, _c_ptr, _c_ptr, _c_i64, _c_ptr, _c_ptr,
                                       _c_ptr, _c_size, _c_ptr]),
    "intlora_gen_aux_batched": (ctypes.c_int, [_P(intlora_aux_job), _c_i32, _c_ptr, _c_size,
                                               _c_ptr]),
    "intlora_gen_aux_noalloc": (ctypes.c_int, [_c_ptr, _c_i64, _c_i64, _c_u64, _c_u32, _c_f32,
                                               _c_i32, _c_ptr, _c_ptr, _c_ptr, _c_ptr, _c_i64,
                                               _c_ptr, _c_ptr, _c_ptr]),
    "intlora_merge_workspace_size": (_c_size, [_P(intlora_layer), _c_i32]),
    "intlora_merge_mul": (ctypes.c_int, [_P(intlora_layer), _c_i32, _c_ptr, _c_ptr, _c_ptr,
                                         _c_ptr, _c_ptr, _c_size, _c_ptr]),
    "intlora_merge_shift": (ctypes.c_int, [_P(intlora_layer), _c_i32, _c_ptr, _c_ptr, _c_ptr,
                                           _c_ptr, _c_size, _c_ptr]),
    "intlora_merge_mul_batched": (ctypes.c_int, [_P(intlora_layer), _P(intlora_merge_out),
                                                 _c_i32, _c_i32, _c_ptr, _c_size, _c_ptr]),
    "intlora_merge_shift_batched": (ctypes.c_int, [_P(intlora_layer), _P(intlora_merge_out),
                                                   _c_i32, _c_i32, _c_ptr, _c_size, _c_ptr]),
    "intlora_ste_workspace_size": (_c_size, [_P(intlora_ste_job), _c_i32]),
    "intlora_ste_backward": (ctypes.c_int, [_c_ptr, _c_ptr, _c_ptr, _c_i64, _c_i64, _c_i32,
                                            _c_ptr, _c_ptr, _c_ptr, _c_size, _c_ptr]),
    "intlora_ste_backward_batched": (ctypes.c_int, [_P(intlora_ste_job), _c_i32, _c_ptr,
                                                    _c_size, _c_ptr]),
    "intlora_int_planes": (_c_i32, [_c_i64]),
    "intlora_fakequant_bf16": (ctypes.c_int, [_c_ptr, _c_i32, _c_ptr, _c_i64, _c_i64, _c_ptr,
                                              _c_ptr]),
    "intlora_linear_bf16_batched": (ctypes.c_int, [_P(intlora_linear_job), _c_i32, _c_ptr]),
    "intlora_train_backward_workspace_size": (_c_size, [_P(intlora_train_backward_job), _c_i32]),
    "intlora_train_backward_batched": (ctypes.c_int, [_P(intlora_train_backward_job), _c_i32,
                                                      _c_ptr, _c_size, _c_ptr]),
    "intlora_fakequant_bf16_batched": (ctypes.c_int, [_P(intlora_fakequant_job), _c_i32, _c_ptr]),
    "intlora_int_pack": (ctypes.c_int, [_c_ptr, _c_i32, _c_i64, _c_i64, _c_i32, _c_ptr, _c_ptr,
                                        _c_ptr]),
    "intlora_int_gemm_batched": (ctypes.c_int, [_P(intlora_int_gemm_job), _c_i32, _c_i32,
                                                _c_ptr]),
    "intlora_int_gemm": (ctypes.c_int, [_c_ptr, _c_ptr, _c_ptr, _c_ptr, _c_i64, _c_i64, _c_i64,
                                        _c_i32, _c_ptr, _c_ptr]),
}

_lib = None


def lib() -> ctypes.CDLL:
    """Load libintlora.so (fails loudly when it has not been built)."""
    global _lib
    if _lib is None:
        if not LIB_PATH.exists():
            raise OSError(f"{LIB_PATH} is missing: build it with "
                          "`python -m quantized_lora_merge_b200.build`")
        L = ctypes.CDLL(str(LIB_PATH))
        for name, (res, args) in _SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def header_functions() -> list[str]:
    """Names of every function the public header declares."""
    text = HEADER.read_text()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(intlora_[a-z0-9_]+)\s*\(", text)))


def _check(status: int) -> None:
    if status != 0:
        raise IntLoRAError(status, lib().intlora_last_error().decode())


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    return getattr(stream, "cuda_stream", stream)


def _ws(ws):
    if ws is None:
        return None, 0
    return ws.data_ptr(), ws.numel() * ws.element_size()


# ---------------------------------------------------------------------------
# descriptors (torch tensors + scalars)
# ---------------------------------------------------------------------------
@dataclass
class AuxJob:
    W: object
    seed: int
    stream_id: int
    alpha: float
    w_bits: int
    sigma_w: object                 # device float64 scalar (output)
    sigma_r: object                 # device float64 scalar (output)
    r_star: object = None
    w_round: object = None          # uint8 [d, ld]
    s: object = None
    z: object = None
    distribution: int = 0           # INTLORA_DIST_*

    def to_c(self) -> intlora_aux_job:
        d, n = self.W.shape
        ld = self.w_round.shape[1] if self.w_round is not None else 0
        return intlora_aux_job(_ptr(self.W), d, n, self.seed, self.stream_id, self.alpha,
                               self.w_bits, _ptr(self.sigma_w), _ptr(self.sigma_r),
                               _ptr(self.r_star), _ptr(self.w_round), ld, _ptr(self.s),
                               _ptr(self.z), self.distribution)


@dataclass
class Layer:
    w_round: object                 # uint8 [d, ld_w] codes
    n: int
    w_bits: int
    s: object
    z: object
    A: object                       # fp32 [d, r]
    B: object                       # fp32 [r, n]
    seed: int
    stream_id: int
    alpha: float
    sigma_w: object
    sigma_r: object = None
    distribution: int = 0           # INTLORA_DIST_*

    def to_c(self) -> intlora_layer:
        d = self.w_round.shape[0]
        return intlora_layer(d, self.n, self.A.shape[1], self.w_bits, _ptr(self.w_round),
                             self.w_round.shape[1], _ptr(self.s), _ptr(self.z), _ptr(self.A),
                             _ptr(self.B), self.seed, self.stream_id, self.alpha,
                             _ptr(self.sigma_w), _ptr(self.sigma_r), self.distribution)


@dataclass
class MergeOut:
    out: object
    sbar: object
    zbar: object = None
    code: object = None

    def to_c(self) -> intlora_merge_out:
        return intlora_merge_out(_ptr(self.out), _ptr(self.sbar), _ptr(self.zbar),
                                 _ptr(self.code))


@dataclass
class SteJob:
    G: object                       # bf16 [d, n]
    A: object                       # bf16 [d, r]
    B: object                       # bf16 [r, n]
    dA: object                      # fp32 [d, r]
    dB: object                      # fp32 [r, n]
    mask_codes: object = None       # masked STE: W_round uint8 [d, ld] (None: plain STE)
    mask_bits: int = 0
    mask_z: object = None           # int32 [d]

    def to_c(self) -> intlora_ste_job:
        d, n = self.G.shape
        ld = self.mask_codes.shape[1] if self.mask_codes is not None else 0
        return intlora_ste_job(_ptr(self.G), _ptr(self.A), _ptr(self.B), d, n, self.A.shape[1],
                               _ptr(self.dA), _ptr(self.dB), _ptr(self.mask_codes), ld,
                               self.mask_bits, _ptr(self.mask_z))


@dataclass
class IntGemmJob:
    X: object                       # int8 [tokens, n]
    x_scale: object                 # fp32 [tokens]
    W: object                       # int8 [d, planes, n] digit planes
    w_scale: object                 # fp32 [d]
    Y: object                       # fp32 or bf16 [tokens, d]

    def to_c(self) -> intlora_int_gemm_job:
        import torch
        tokens, n = self.X.shape
        return intlora_int_gemm_job(_ptr(self.X), _ptr(self.x_scale), _ptr(self.W),
                                    _ptr(self.w_scale), tokens, self.W.shape[0], n, _ptr(self.Y),
                                    int(self.Y.dtype == torch.bfloat16))


@dataclass
class FakeQuantJob:
    q: object                       # merged integer weights [d, n] (int8/int16/int32)
    sbar: object                    # fp32 [d]
    w_out: object                   # bf16 [d, n]

    def to_c(self) -> intlora_fakequant_job:
        d, n = self.q.shape
        return intlora_fakequant_job(_ptr(self.q), self.q.element_size(), _ptr(self.sbar), d, n,
                                     _ptr(self.w_out))


@dataclass
class LinearJob:
    X: object                       # bf16 [tokens, n]
    W: object                       # bf16 [d, n]
    Y: object                       # fp32 or bf16 [tokens, d]

    def to_c(self) -> intlora_linear_job:
        import torch
        tokens, n = self.X.shape
        return intlora_linear_job(_ptr(self.X), _ptr(self.W), tokens, self.W.shape[0], n,
                                  _ptr(self.Y), int(self.Y.dtype == torch.bfloat16))


@dataclass
class TrainBackwardJob:
    X: object                       # bf16 [tokens, n]
    dY: object                      # bf16 [tokens, d]
    W: object                       # bf16 [d, n] (fake-quantized merged weight)
    A: object                       # bf16 [d, r]
    B: object                       # bf16 [r, n]
    dX: object                      # fp32 [tokens, n]
    dA: object                      # fp32 [d, r]
    dB: object                      # fp32 [r, n]

    def to_c(self) -> intlora_train_backward_job:
        tokens, n = self.X.shape
        d, r = self.A.shape
        return intlora_train_backward_job(_ptr(self.X), _ptr(self.dY), _ptr(self.W), _ptr(self.A),
                                          _ptr(self.B), tokens, d, n, r, _ptr(self.dX),
                                          _ptr(self.dA), _ptr(self.dB))


def _array(struct, items):
    if isinstance(items, Descriptors):
        if items.struct is not struct:
            raise TypeError(f"descriptors of {items.struct.__name__}, expected {struct.__name__}")
        return items.arr
    arr = (struct * max(1, len(items)))()
    for k, it in enumerate(items):
        arr[k] = it.to_c()
    return arr


class Descriptors:
    """A list of descriptors converted to their C structs once, for calls that
    repeat on the same buffers (the per-call conversion of a 128-layer list
    costs milliseconds of Python). Pass it wherever a list is accepted."""

    _STRUCT = {}

    def __init__(self, items):
        items = list(items)
        if not items:
            raise ValueError("empty descriptor list")
        self.struct = self._STRUCT[type(items[0])]
        self.arr = (self.struct * len(items))()
        for k, it in enumerate(items):
            if type(it) is not type(items[0]):
                raise TypeError("mixed descriptor types")
            self.arr[k] = it.to_c()
        self.count = len(items)

    def __len__(self):
        return self.count


Descriptors._STRUCT = {AuxJob: intlora_aux_job, Layer: intlora_layer,
                       MergeOut: intlora_merge_out, SteJob: intlora_ste_job,
                       IntGemmJob: intlora_int_gemm_job, LinearJob: intlora_linear_job,
                       FakeQuantJob: intlora_fakequant_job,
                       TrainBackwardJob: intlora_train_backward_job}


# ---------------------------------------------------------------------------
# entry points (same names as the C ABI)
# ---------------------------------------------------------------------------
def intlora_version() -> int:
    return lib().intlora_version()


def intlora_device_timeouts() -> int:
    """Bounded device waits that gave up since the library was loaded."""
    return lib().intlora_device_timeouts()


def intlora_device_status() -> int:
    """INTLORA_OK, or INTLORA_ERR_TIMEOUT when bounded device waits gave up
    since the last check (synchronizes the device). Returns the status code
    (no exception), so callers can tell the two apart."""
    return lib().intlora_device_status()


def intlora_selftest_bounded_wait(limit_us: int, stream=None) -> None:
    """Enqueues the self-test kernel whose bounded wait runs out."""
    _check(lib().intlora_selftest_bounded_wait(limit_us, _stream(stream)))


def intlora_kernel_launches() -> int:
    """Kernels the library has enqueued since it was loaded (host counter)."""
    return lib().intlora_kernel_launches()


def intlora_merge_out_bytes(variant: int, w_bits: int, out_bits: int) -> int:
    return lib().intlora_merge_out_bytes(variant, w_bits, out_bits)


def intlora_gen_aux_workspace_size(jobs: Sequence[AuxJob]) -> int:
    return lib().intlora_gen_aux_workspace_size(_array(intlora_aux_job, jobs), len(jobs))


def intlora_gen_aux_batched(jobs: Sequence[AuxJob], ws=None, stream=None) -> None:
    p, nb = _ws(ws)
    _check(lib().intlora_gen_aux_batched(_array(intlora_aux_job, jobs), len(jobs), p, nb,
                                         _stream(stream)))


def intlora_gen_aux(job: AuxJob, ws=None, stream=None) -> None:
    c = job.to_c()
    p, nb = _ws(ws)
    _check(lib().intlora_gen_aux(c.W, c.d, c.n, c.seed, c.stream_id, c.alpha, c.w_bits,
                                 c.sigma_w_out, c.sigma_r_out, c.r_star_out, c.w_round_out,
                                 c.ld_w_out, c.s_out, c.z_out, p, nb, _stream(stream)))


def intlora_gen_aux_noalloc(job: AuxJob, stream=None) -> None:
    """Layer preparation with the library's built-in scratch (no workspace)."""
    c = job.to_c()
    _check(lib().intlora_gen_aux_noalloc(c.W, c.d, c.n, c.seed, c.stream_id, c.alpha, c.w_bits,
                                         c.sigma_w_out, c.sigma_r_out, c.r_star_out,
                                         c.w_round_out, c.ld_w_out, c.s_out, c.z_out,
                                         _stream(stream)))


def intlora_merge_workspace_size(layers: Sequence[Layer]) -> int:
    return lib().intlora_merge_workspace_size(_array(intlora_layer, layers), len(layers))


def intlora_merge_mul(layer: Layer, u_bits: int, out: MergeOut, ws=None, stream=None) -> None:
    p, nb = _ws(ws)
    c = layer.to_c()
    _check(lib().intlora_merge_mul(ctypes.byref(c), u_bits, _ptr(out.out), _ptr(out.sbar),
                                   _ptr(out.zbar), _ptr(out.code), p, nb, _stream(stream)))


def intlora_merge_shift(layer: Layer, shift_bits: int, out: MergeOut, ws=None,
                        stream=None) -> None:
    p, nb = _ws(ws)
    c = layer.to_c()
    _check(lib().intlora_merge_shift(ctypes.byref(c), shift_bits, _ptr(out.out), _ptr(out.sbar),
                                     _ptr(out.code), p, nb, _stream(stream)))


def intlora_merge_mul_batched(layers: Sequence[Layer], outs: Sequence[MergeOut], u_bits: int,
                              ws=None, stream=None) -> None:
    p, nb = _ws(ws)
    _check(lib().intlora_merge_mul_batched(_array(intlora_layer, layers),
                                           _array(intlora_merge_out, outs), len(layers), u_bits,
                                           p, nb, _stream(stream)))


def intlora_merge_shift_batched(layers: Sequence[Layer], outs: Sequence[MergeOut],
                                shift_bits: int, ws=None, stream=None) -> None:
    p, nb = _ws(ws)
    _check(lib().intlora_merge_shift_batched(_array(intlora_layer, layers),
                                             _array(intlora_merge_out, outs), len(layers),
                                             shift_bits, p, nb, _stream(stream)))


def intlora_ste_workspace_size(jobs: Sequence[SteJob]) -> int:
    return lib().intlora_ste_workspace_size(_array(intlora_ste_job, jobs), len(jobs))


def intlora_ste_backward(job: SteJob, ws=None, stream=None) -> None:
    c = job.to_c()
    p, nb = _ws(ws)
    _check(lib().intlora_ste_backward(c.G, c.A, c.B, c.d, c.n, c.r, c.dA, c.dB, p, nb,
                                      _stream(stream)))


def intlora_ste_backward_batched(jobs: Sequence[SteJob], ws=None, stream=None) -> None:
    p, nb = _ws(ws)
    _check(lib().intlora_ste_backward_batched(_array(intlora_ste_job, jobs), len(jobs), p, nb,
                                              _stream(stream)))


def intlora_int_planes(max_abs: int) -> int:
    return lib().intlora_int_planes(max_abs)


def intlora_int_pack(q, planes: int, packed, overflow=None, stream=None) -> None:
    """Packs the merged integer weights q (int8/int16/int32 [d, n]) into
    base-128 digit planes packed (int8 [d, planes, n])."""
    d, n = q.shape
    _check(lib().intlora_int_pack(_ptr(q), q.element_size(), d, n, planes, _ptr(packed),
                                  _ptr(overflow), _stream(stream)))


def intlora_int_gemm_batched(jobs: Sequence[IntGemmJob], planes: int, stream=None) -> None:
    _check(lib().intlora_int_gemm_batched(_array(intlora_int_gemm_job, jobs), len(jobs), planes,
                                          _stream(stream)))


def intlora_int_gemm(job: IntGemmJob, planes: int, stream=None) -> None:
    """Single-layer call (fp32 Y; a bf16 Y goes through intlora_int_gemm_batched)."""
    c = job.to_c()
    if c.y_bf16:
        raise TypeError("intlora_int_gemm writes fp32 Y; use intlora_int_gemm_batched for bf16 Y")
    _check(lib().intlora_int_gemm(c.X, c.x_scale, c.W, c.w_scale, c.tokens, c.d, c.n, planes,
                                  c.Y, _stream(stream)))


def intlora_fakequant_bf16(q, sbar, w_out, stream=None) -> None:
    """w_out (bf16 [d, n]) = bf16(fp32(sbar_i) * q_ij) for merged weights q."""
    d, n = q.shape
    _check(lib().intlora_fakequant_bf16(_ptr(q), q.element_size(), _ptr(sbar), d, n, _ptr(w_out),
                                        _stream(stream)))


def intlora_linear_bf16_batched(jobs: Sequence[LinearJob], stream=None) -> None:
    _check(lib().intlora_linear_bf16_batched(_array(intlora_linear_job, jobs), len(jobs),
                                             _stream(stream)))


def intlora_train_backward_workspace_size(jobs: Sequence[TrainBackwardJob]) -> int:
    return lib().intlora_train_backward_workspace_size(_array(intlora_train_backward_job, jobs),
                                                       len(jobs))


def intlora_train_backward_batched(jobs: Sequence[TrainBackwardJob], ws=None, stream=None) -> None:
    p, nb = _ws(ws)
    _check(lib().intlora_train_backward_batched(_array(intlora_train_backward_job, jobs), len(jobs),
                                                p, nb, _stream(stream)))


def intlora_fakequant_bf16_batched(jobs: Sequence[FakeQuantJob], stream=None) -> None:
    _check(lib().intlora_fakequant_bf16_batched(_array(intlora_fakequant_job, jobs), len(jobs),
                                                _stream(stream)))
