"""CPU oracle for the IntLoRA integer low-rank merge (test infrastructure).

TEST INFRASTRUCTURE ONLY: the tests, the repository smoke check and the
CPU-baseline leg of ``bench.py`` import this package; the CUDA library and its
Python binding never do. The arithmetic lives in ``intlora_oracle.c`` (plain
fp64 C, its own Philox4x32-10); this module only builds that file with gcc and
marshals numpy arrays through ctypes. See the C file's header for the sources
each function follows and the readings taken where the pages are silent.

Parity pins: every function here is pinned by ``tests/test_oracle_pins.py``
against something other than itself (an independent Philox implementation,
closed forms, brute-force enumeration, exact rational identities, numpy
matmul). No function is "parity unpinned".
"""
from __future__ import annotations

import ctypes
import hashlib
import os
import subprocess
from pathlib import Path

import numpy as np

_HERE = Path(__file__).resolve().parent
_SRC = _HERE / "intlora_oracle.c"
_LIB_PATH = _HERE / "liboracle.so"
_lib = None

_i64 = ctypes.c_int64
_u64 = ctypes.c_uint64
_u32 = ctypes.c_uint32
_int = ctypes.c_int
_dbl = ctypes.c_double
_ptr = ctypes.c_void_p


def build(force: bool = False) -> Path:
    """Compile the oracle with gcc (-O2, OpenMP, strict IEEE: no fast-math).
    The library is rebuilt whenever the source's hash differs from the one
    recorded beside it (copies of the tree need not keep file times)."""
    digest = hashlib.sha256(_SRC.read_bytes()).hexdigest()
    stamp = _LIB_PATH.with_name(_LIB_PATH.name + ".sha256")
    fresh = _LIB_PATH.exists() and stamp.exists() and stamp.read_text().strip() == digest
    if force or not fresh:
        tmp = _LIB_PATH.with_suffix(f".so.tmp{os.getpid()}")
        cmd = ["gcc", "-std=c11", "-O2", "-fno-fast-math", "-ffp-contract=off", "-fopenmp",
               "-fPIC", "-shared", str(_SRC), "-o", str(tmp), "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB_PATH)
        stamp.write_text(digest + "\n")
    return _LIB_PATH


def _load():
    global _lib
    if _lib is not None:
        return _lib
    lib = ctypes.CDLL(str(build()))
    sig = {
        "orc_philox4x32_10": (None, [_ptr, _ptr, _ptr]),
        "orc_aux_word": (_u32, [_u64, _u32, _i64]),
        "orc_laplace_from_word": (_dbl, [_u32]),
        "orc_aux_block": (None, [_u64, _u32, _i64, _i64, _ptr, _int]),
        "orc_aux_value": (_dbl, [_u64, _u32, _i64, _int]),
        "orc_population_std": (_dbl, [_ptr, _i64]),
        "orc_std_f32": (_dbl, [_ptr, _i64, _i64]),
        "orc_sigma_r": (_dbl, [_i64, _i64, _u64, _u32, _int]),
        "orc_vmc_scale": (_dbl, [_dbl, _dbl, _dbl]),
        "orc_affine_quantize_row": (None, [_ptr, _i64, _int, _ptr, _ptr, _ptr, _ptr, _ptr]),
        "orc_gen_aux": (None, [_ptr, _i64, _i64, _u64, _u32, _dbl, _int, _i64, _i64,
                               _ptr, _ptr, _ptr, _ptr, _ptr, _ptr, _ptr, _ptr, _ptr, _int]),
        "orc_mla_rows": (None, [_ptr, _i64, _ptr, _ptr, _ptr, _ptr, _i64, _i64, _int, _u64,
                                _u32, _dbl, _dbl, _dbl, _i64, _i64, _ptr, _ptr, _int]),
        "orc_merge_mul": (None, [_ptr, _i64, _ptr, _ptr, _ptr, _ptr, _i64, _i64, _int, _u64,
                                 _u32, _dbl, _dbl, _dbl, _int, _i64, _i64, _ptr, _ptr, _ptr,
                                 _ptr, _ptr, _ptr, _ptr, _int]),
        "orc_merge_shift": (None, [_ptr, _i64, _ptr, _ptr, _ptr, _ptr, _i64, _i64, _int, _u64,
                                   _u32, _dbl, _dbl, _dbl, _int, _i64, _i64, _ptr, _ptr, _ptr,
                                   _ptr, _ptr, _int]),
        "orc_shift_quantize_row": (None, [_ptr, _ptr, _i64, _int, _ptr, _ptr, _ptr, _ptr]),
        "orc_ste_backward": (None, [_ptr, _ptr, _ptr, _i64, _i64, _int, _ptr, _ptr]),
        "orc_ste_sampled": (None, [_ptr, _ptr, _ptr, _i64, _i64, _int, _ptr, _i64, _ptr, _i64,
                                   _ptr, _ptr]),
        "orc_quantize_rows": (None, [_ptr, _i64, _u64, _u32, _dbl, _int, _i64, _i64, _ptr, _ptr,
                                     _ptr, _ptr, _ptr, _int]),
        "orc_merge_mul_rows": (None, [_ptr, _i64, _ptr, _ptr, _ptr, _ptr, _i64, _int, _u64, _u32,
                                      _dbl, _int, _i64, _i64, _ptr, _ptr, _ptr, _ptr, _ptr,
                                      _ptr, _int]),
        "orc_int_digits": (_i64, [_ptr, _i64, _i64, _int, _ptr]),
        "orc_fakequant_bf16": (None, [_ptr, _ptr, _i64, _i64, _ptr]),
        "orc_linear_rows": (None, [_ptr, _ptr, _i64, _i64, _i64, _ptr, _i64, _ptr]),
        "orc_int_gemm_rows": (None, [_ptr, _ptr, _ptr, _ptr, _i64, _i64, _i64, _ptr, _i64, _ptr]),
        "orc_num_threads": (_int, []),
        "orc_set_num_threads": (None, [_int]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def _p(a: np.ndarray | None):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle inputs must be C-contiguous"
    return a.ctypes.data


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


# --------------------------------------------------------------------------
# a1: Philox4x32-10 and the Laplace sampler
# --------------------------------------------------------------------------
def philox4x32_10(counter, key) -> np.ndarray:
    ctr = _c(counter, np.uint32)
    k = _c(key, np.uint32)
    out = np.zeros(4, np.uint32)
    _load().orc_philox4x32_10(_p(ctr), _p(k), _p(out))
    return out


def aux_word(seed: int, stream_id: int, e: int) -> int:
    return int(_load().orc_aux_word(seed, stream_id, e))


LAPLACE, GAUSSIAN, CAUCHY, STUDENT_T2 = 0, 1, 2, 3     # auxiliary laws


def aux_value(seed: int, stream_id: int, e: int, dist: int) -> float:
    """Element e of the auxiliary matrix under law `dist`."""
    return float(_load().orc_aux_value(seed, stream_id, e, dist))


def laplace_from_word(x) -> np.ndarray:
    lib = _load()
    xs = np.atleast_1d(np.asarray(x, dtype=np.uint32))
    return np.array([lib.orc_laplace_from_word(int(v)) for v in xs], dtype=np.float64)


def aux_R(d: int, n: int, seed: int, stream_id: int, row_begin: int = 0,
          row_count: int | None = None, dist: int = 0) -> np.ndarray:
    """Rows [row_begin, row_begin+row_count) of the d x n Laplace matrix R."""
    rc = d - row_begin if row_count is None else row_count
    out = np.zeros((rc, n), np.float64)
    _load().orc_aux_block(seed, stream_id, row_begin * n, rc * n, _p(out), dist)
    return out


# --------------------------------------------------------------------------
# a2: sigma and VMC
# --------------------------------------------------------------------------
def population_std(x) -> float:
    a = _c(x, np.float64).ravel()
    return float(_load().orc_population_std(_p(a), a.size))


def std_f32(W) -> float:
    w = _c(W, np.float32)
    d, n = w.shape
    return float(_load().orc_std_f32(_p(w), d, n))


def sigma_r(d: int, n: int, seed: int, stream_id: int, dist: int = 0) -> float:
    return float(_load().orc_sigma_r(d, n, seed, stream_id, dist))


def vmc_scale(sigma_w: float, sigma_r_: float, alpha: float) -> float:
    return float(_load().orc_vmc_scale(sigma_w, sigma_r_, alpha))


# --------------------------------------------------------------------------
# a3 / a6: the affine quantizer of one row
# --------------------------------------------------------------------------
def affine_quantize_row(x, bits: int):
    a = _c(x, np.float64).ravel()
    n = a.size
    scale = np.zeros(1, np.float64)
    zero = np.zeros(1, np.int32)
    codes = np.zeros(n, np.int32)
    pre = np.zeros(n, np.float64)
    zpre = np.zeros(1, np.float64)
    _load().orc_affine_quantize_row(_p(a), n, bits, _p(scale), _p(zero), _p(codes), _p(pre),
                                    _p(zpre))
    return dict(scale=float(scale[0]), zero=int(zero[0]), codes=codes, pre=pre,
                zpre=float(zpre[0]))


# --------------------------------------------------------------------------
# a1-a3: layer preparation
# --------------------------------------------------------------------------
def gen_aux(W, seed: int, stream_id: int, alpha: float, w_bits: int, row_begin: int = 0,
            row_count: int | None = None, want_r_star: bool = False, dist: int = 0) -> dict:
    w = _c(W, np.float32)
    d, n = w.shape
    rc = d - row_begin if row_count is None else row_count
    sw = np.zeros(1, np.float64)
    sr = np.zeros(1, np.float64)
    cc = np.zeros(1, np.float64)
    r_star = np.zeros((rc, n), np.float64) if want_r_star else None
    codes = np.zeros((rc, n), np.int32)
    s = np.zeros(rc, np.float64)
    z = np.zeros(rc, np.int32)
    pre = np.zeros((rc, n), np.float64)
    zpre = np.zeros(rc, np.float64)
    _load().orc_gen_aux(_p(w), d, n, seed, stream_id, alpha, w_bits, row_begin, rc, _p(sw),
                        _p(sr), _p(cc), _p(r_star), _p(codes), _p(s), _p(z), _p(pre), _p(zpre),
                        dist)
    return dict(sigma_w=float(sw[0]), sigma_r=float(sr[0]), c=float(cc[0]), r_star=r_star,
                codes=codes, s=s, z=z, pre=pre, zpre=zpre)


def quantize_rows(W_rows, seed: int, stream_id: int, c: float, w_bits: int,
                  row_begin: int, dist: int = 0) -> dict:
    """Base quantization of rows [row_begin, row_begin + len(W_rows)) of a layer
    from those rows of W alone, with the VMC factor c given (layers too large
    to hold or reduce on the host)."""
    w = _c(W_rows, np.float32)
    rc, n = w.shape
    codes = np.zeros((rc, n), np.int32)
    s = np.zeros(rc, np.float64)
    z = np.zeros(rc, np.int32)
    pre = np.zeros((rc, n), np.float64)
    zpre = np.zeros(rc, np.float64)
    _load().orc_quantize_rows(_p(w), n, seed, stream_id, c, w_bits, row_begin, rc, _p(codes),
                              _p(s), _p(z), _p(pre), _p(zpre), dist)
    return dict(codes=codes, s=s, z=z, pre=pre, zpre=zpre)


# --------------------------------------------------------------------------
# a4-a7: the merges
# --------------------------------------------------------------------------
def _merge_inputs(codes, s, z, A, B):
    cd = _c(codes, np.int32)
    sf = _c(s, np.float32)
    zi = _c(z, np.int32)
    Af = _c(A, np.float32)
    Bf = _c(B, np.float32)
    d, n = cd.shape
    r = Af.shape[1]
    assert Af.shape == (d, r) and Bf.shape == (r, n) and sf.shape == (d,) and zi.shape == (d,)
    return cd, sf, zi, Af, Bf, d, n, r


def mla_rows(codes, s, z, A, B, seed, stream_id, sigma_w, sigma_r_, alpha, row_begin=0,
             row_count=None, dist=0):
    """U and D for the given rows (U * D is the pre-quantization merged weight)."""
    cd, sf, zi, Af, Bf, d, n, r = _merge_inputs(codes, s, z, A, B)
    rc = d - row_begin if row_count is None else row_count
    U = np.zeros((rc, n), np.float64)
    D = np.zeros((rc, n), np.int64)
    _load().orc_mla_rows(_p(cd), n, _p(sf), _p(zi), _p(Af), _p(Bf), d, n, r, seed, stream_id,
                         sigma_w, sigma_r_, alpha, row_begin, rc, _p(U), _p(D), dist)
    return U, D


def merge_mul(codes, s, z, A, B, seed, stream_id, sigma_w, sigma_r_, alpha, u_bits,
              row_begin=0, row_count=None, dist=0) -> dict:
    cd, sf, zi, Af, Bf, d, n, r = _merge_inputs(codes, s, z, A, B)
    rc = d - row_begin if row_count is None else row_count
    U = np.zeros((rc, n), np.float64)
    ur = np.zeros((rc, n), np.int32)
    sbar = np.zeros(rc, np.float64)
    zbar = np.zeros(rc, np.int32)
    P = np.zeros((rc, n), np.int64)
    pre = np.zeros((rc, n), np.float64)
    zpre = np.zeros(rc, np.float64)
    _load().orc_merge_mul(_p(cd), n, _p(sf), _p(zi), _p(Af), _p(Bf), d, n, r, seed, stream_id,
                          sigma_w, sigma_r_, alpha, u_bits, row_begin, rc, _p(U), _p(ur),
                          _p(sbar), _p(zbar), _p(P), _p(pre), _p(zpre), dist)
    return dict(U=U, u_round=ur, sbar=sbar, zbar=zbar, P=P, pre=pre, zpre=zpre)


def merge_mul_rows(codes_rows, s_rows, z_rows, A_rows, B, seed, stream_id, c, u_bits,
                   row_begin, dist=0) -> dict:
    """MUL merge of rows [row_begin, row_begin + len(codes_rows)) from those
    rows' inputs alone, with the VMC factor c given."""
    cd = _c(codes_rows, np.int32)
    sf = _c(s_rows, np.float32)
    zi = _c(z_rows, np.int32)
    Af = _c(A_rows, np.float32)
    Bf = _c(B, np.float32)
    rc, n = cd.shape
    r = Af.shape[1]
    ur = np.zeros((rc, n), np.int32)
    sbar = np.zeros(rc, np.float64)
    zbar = np.zeros(rc, np.int32)
    P = np.zeros((rc, n), np.int64)
    pre = np.zeros((rc, n), np.float64)
    zpre = np.zeros(rc, np.float64)
    _load().orc_merge_mul_rows(_p(cd), n, _p(sf), _p(zi), _p(Af), _p(Bf), n, r, seed, stream_id,
                               c, u_bits, row_begin, rc, _p(ur), _p(sbar), _p(zbar), _p(P),
                               _p(pre), _p(zpre), dist)
    return dict(u_round=ur, sbar=sbar, zbar=zbar, P=P, pre=pre, zpre=zpre)


def shift_quantize_row(U, D, shift_bits: int) -> dict:
    u = _c(U, np.float64).ravel()
    dd = _c(D, np.int64).ravel()
    n = u.size
    sbar = np.zeros(1, np.float64)
    shift = np.zeros(n, np.int32)
    M = np.zeros(n, np.int64)
    pre = np.zeros(n, np.float64)
    _load().orc_shift_quantize_row(_p(u), _p(dd), n, shift_bits, _p(sbar), _p(shift), _p(M),
                                   _p(pre))
    return dict(sbar=float(sbar[0]), shift=shift, M=M, pre=pre)


def merge_shift(codes, s, z, A, B, seed, stream_id, sigma_w, sigma_r_, alpha, shift_bits,
                row_begin=0, row_count=None, dist=0) -> dict:
    cd, sf, zi, Af, Bf, d, n, r = _merge_inputs(codes, s, z, A, B)
    rc = d - row_begin if row_count is None else row_count
    U = np.zeros((rc, n), np.float64)
    sbar = np.zeros(rc, np.float64)
    shift = np.zeros((rc, n), np.int32)
    M = np.zeros((rc, n), np.int64)
    pre = np.zeros((rc, n), np.float64)
    _load().orc_merge_shift(_p(cd), n, _p(sf), _p(zi), _p(Af), _p(Bf), d, n, r, seed, stream_id,
                            sigma_w, sigma_r_, alpha, shift_bits, row_begin, rc, _p(U), _p(sbar),
                            _p(shift), _p(M), _p(pre), dist)
    return dict(U=U, sbar=sbar, shift=shift, M=M, pre=pre)


# --------------------------------------------------------------------------
# a8: STE backward
# --------------------------------------------------------------------------
def ste_backward(G, A, B):
    g = _c(G, np.float64)
    a = _c(A, np.float64)
    b = _c(B, np.float64)
    d, n = g.shape
    r = a.shape[1]
    dA = np.zeros((d, r), np.float64)
    dB = np.zeros((r, n), np.float64)
    _load().orc_ste_backward(_p(g), _p(a), _p(b), d, n, r, _p(dA), _p(dB))
    return dA, dB


def ste_sampled(G_bits, A_bits, B_bits, rows, cols):
    """dA rows and dB columns from bf16 bit patterns (uint16 arrays)."""
    g = _c(G_bits, np.uint16)
    a = _c(A_bits, np.uint16)
    b = _c(B_bits, np.uint16)
    d, n = g.shape
    r = a.shape[1]
    rw = _c(rows, np.int64)
    cl = _c(cols, np.int64)
    dA = np.zeros((rw.size, r), np.float64)
    dB = np.zeros((cl.size, r), np.float64)
    _load().orc_ste_sampled(_p(g), _p(a), _p(b), d, n, r, _p(rw), rw.size, _p(cl), cl.size,
                            _p(dA), _p(dB))
    return dA, dB.T.copy()


# --------------------------------------------------------------------------
# Integer inference GEMM on the merged weights (Y = X W'^T)
# --------------------------------------------------------------------------
def int_planes(max_abs: int) -> int:
    """Base-128 digit planes that hold every integer weight with |w| <= max_abs."""
    for p in (1, 2, 3):
        if max_abs <= 2 ** (7 * p) - 1:
            return p
    return 0


def int_digits(W, planes: int):
    """(digits [d][planes][n] int8, count of weights out of range)."""
    w = _c(W, np.int64)
    d, n = w.shape
    out = np.zeros((d, planes, n), np.int8)
    bad = _load().orc_int_digits(_p(w), d, n, planes, _p(out))
    return out, int(bad)


def int_gemm_rows(X, x_scale, W, w_scale, rows=None):
    """Y rows (fp64) of the integer GEMM for the given token rows (all by default)."""
    x = _c(X, np.int8)
    xs = _c(x_scale, np.float64)
    w = _c(W, np.int64)
    ws = _c(w_scale, np.float64)
    tokens, n = x.shape
    d = w.shape[0]
    rw = _c(np.arange(tokens) if rows is None else rows, np.int64)
    Y = np.zeros((rw.size, d), np.float64)
    _load().orc_int_gemm_rows(_p(x), _p(xs), _p(w), _p(ws), tokens, d, n, _p(rw), rw.size, _p(Y))
    return Y


def ste_mask(codes, z):
    """[D != 0] with D = W_round - z: where the masked STE keeps G."""
    return np.asarray(codes, np.int64) != np.asarray(z, np.int64)[:, None]


def ste_backward_masked(G, A, B, codes, z):
    """Masked STE: dA and dB of G (.) [W_round != z]."""
    return ste_backward(np.asarray(G, np.float64) * ste_mask(codes, z), A, B)


def ste_sampled_masked(G_bits, A_bits, B_bits, codes, z, rows, cols):
    """Sampled rows of dA and columns of dB of the masked STE (bf16 inputs;
    masked elements of G become +0)."""
    g = np.where(ste_mask(codes, z), np.asarray(G_bits, np.uint16), np.uint16(0))
    return ste_sampled(g, A_bits, B_bits, rows, cols)


# --------------------------------------------------------------------------
# Training forward on the merged weights
# --------------------------------------------------------------------------
def fakequant_bf16(Q, sbar):
    """bf16 bit patterns of fp32(sbar_i * Q_ij)."""
    q = _c(Q, np.int64)
    sb = _c(sbar, np.float32)
    d, n = q.shape
    out = np.zeros((d, n), np.uint16)
    _load().orc_fakequant_bf16(_p(q), _p(sb), d, n, _p(out))
    return out


def linear_rows(X_bits, W_bits, rows=None):
    """Y rows (fp64) of X W^T for bf16 patterns X (tokens x n), W (d x n)."""
    x = _c(X_bits, np.uint16)
    w = _c(W_bits, np.uint16)
    tokens, n = x.shape
    d = w.shape[0]
    rw = _c(np.arange(tokens) if rows is None else rows, np.int64)
    Y = np.zeros((rw.size, d), np.float64)
    _load().orc_linear_rows(_p(x), _p(w), tokens, d, n, _p(rw), rw.size, _p(Y))
    return Y


def train_backward(X_bits, dY_bits, W_bits, A_bits, B_bits) -> dict:
    """Backward of one IntLoRA linear Y = X W'^T through the STE, in fp64 from
    bf16 patterns: G = dY^T X (the gradient on W', d x n), dX = dY W'
    (tokens x n), and the STE products dA = G B^T, dB = A^T G."""
    f = lambda b: (np.asarray(b, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    X, dY, W, A, B = (f(b) for b in (X_bits, dY_bits, W_bits, A_bits, B_bits))
    G = dY.T @ X
    dA, dB = ste_backward(G, A, B)
    return dict(G=G, dX=dY @ W, dA=dA, dB=dB)


def num_threads() -> int:
    return int(_load().orc_num_threads())


def set_num_threads(n: int) -> None:
    """OpenMP threads of the oracle's later calls from this thread."""
    _load().orc_set_num_threads(int(n))
