"""The C ABI without a GPU: the library loads, exports every function the
public header declares, and rejects bad arguments on the host with the right
status before any CUDA call (these calls never reach a launch)."""
import ctypes

import pytest

from quantized_lora_merge_b200 import binding as B
from quantized_lora_merge_b200.build import build

FAKE = 0x100000  # 16-byte-aligned dummy address; never dereferenced by validation


@pytest.fixture(scope="module")
def lib():
    build()
    return B.lib()


def test_every_header_function_is_exported(lib):
    names = B.header_functions()
    assert len(names) >= 15
    for name in names:
        assert hasattr(lib, name), f"{name} declared in include/intlora.h but not exported"


def test_status_strings_and_version(lib):
    assert lib.intlora_status_string(0) == b"ok"
    assert lib.intlora_status_string(1) == b"invalid argument"
    assert lib.intlora_status_string(99) == b"unknown status"
    assert lib.intlora_version() >= 100


def test_merge_out_bytes(lib):
    assert lib.intlora_merge_out_bytes(0, 4, 4) == 2     # 15*15 fits int16
    assert lib.intlora_merge_out_bytes(0, 8, 8) == 4     # 255*255 does not
    assert lib.intlora_merge_out_bytes(0, 8, 7) == 2     # 255*127 = 32385
    assert lib.intlora_merge_out_bytes(1, 4, 4) == 1
    assert lib.intlora_merge_out_bytes(1, 8, 4) == 2
    assert lib.intlora_merge_out_bytes(2, 8, 4) == 0


def _aux(**kw):
    j = B.intlora_aux_job(W=FAKE, d=4, n=8, seed=1, stream_id=0, alpha=1.5, w_bits=8,
                          sigma_w_out=FAKE, sigma_r_out=FAKE, r_star_out=None,
                          w_round_out=FAKE, ld_w_out=16, s_out=FAKE, z_out=FAKE)
    for k, v in kw.items():
        setattr(j, k, v)
    return j


@pytest.mark.parametrize("field,value,needle", [
    ("W", None, "W is NULL"),
    ("d", 0, "d and n"),
    ("n", -3, "d and n"),
    ("w_bits", 3, "w_bits"),
    ("alpha", -1.0, "alpha"),
    ("alpha", float("nan"), "alpha"),
    ("sigma_r_out", None, "sigma"),
    ("ld_w_out", 8, "ld_w_out"),
    ("ld_w_out", 24, "ld_w_out"),
    ("W", FAKE + 4, "16-byte"),
    ("s_out", None, "s_out"),
])
def test_gen_aux_rejects(lib, field, value, needle):
    jobs = (B.intlora_aux_job * 1)(_aux(**{field: value}))
    st = lib.intlora_gen_aux_batched(jobs, 1, None, 0, None)
    assert st == 1
    assert needle in lib.intlora_last_error().decode()


def test_gen_aux_4bit_needs_even_n(lib):
    jobs = (B.intlora_aux_job * 1)(_aux(w_bits=4, n=7))
    assert lib.intlora_gen_aux_batched(jobs, 1, None, 0, None) == 1
    assert "even" in lib.intlora_last_error().decode()


def test_gen_aux_workspace_checked(lib):
    jobs = (B.intlora_aux_job * 1)(_aux())
    need = lib.intlora_gen_aux_workspace_size(jobs, 1)
    assert need > 0
    assert lib.intlora_gen_aux_batched(jobs, 1, None, 0, None) == 3
    assert lib.intlora_gen_aux_batched(jobs, 1, FAKE, need - 1, None) == 3


def _layer(**kw):
    l = B.intlora_layer(d=4, n=8, r=4, w_bits=8, w_round=FAKE, ld_w=16, s=FAKE, z=FAKE, A=FAKE,
                        B=FAKE, seed=1, stream_id=0, alpha=1.5, sigma_w=FAKE, sigma_r=FAKE)
    for k, v in kw.items():
        setattr(l, k, v)
    return l


@pytest.mark.parametrize("field,value", [
    ("d", 0), ("r", 0), ("r", 257), ("w_bits", 2), ("w_round", None), ("B", None),
    ("sigma_w", None), ("ld_w", 4), ("w_round", FAKE + 1), ("alpha", -0.5)])
def test_merge_rejects_bad_layer(lib, field, value):
    layer = _layer(**{field: value})
    st = lib.intlora_merge_mul(ctypes.byref(layer), 8, FAKE, FAKE, FAKE, None, None, 0, None)
    assert st == 1, lib.intlora_last_error()


def test_merge_rejects_bad_bits_and_outputs(lib):
    layer = _layer()
    assert lib.intlora_merge_mul(ctypes.byref(layer), 9, FAKE, FAKE, FAKE, None, None, 0, None) == 1
    assert lib.intlora_merge_mul(ctypes.byref(layer), 8, FAKE, FAKE, None, None, None, 0, None) == 1
    assert lib.intlora_merge_shift(ctypes.byref(layer), 6, FAKE, FAKE, None, None, 0, None) == 1
    assert lib.intlora_merge_shift(ctypes.byref(layer), 4, FAKE + 8, FAKE, None, None, 0, None) == 1
    assert lib.intlora_merge_mul(None, 8, FAKE, FAKE, FAKE, None, None, 0, None) == 1


def test_merge_without_sigma_r_needs_workspace(lib):
    layer = _layer(sigma_r=None)
    arr = (B.intlora_layer * 1)(layer)
    need = lib.intlora_merge_workspace_size(arr, 1)
    assert need > 0
    assert lib.intlora_merge_workspace_size((B.intlora_layer * 1)(_layer()), 1) == 0
    st = lib.intlora_merge_mul(ctypes.byref(layer), 8, FAKE, FAKE, FAKE, None, None, 0, None)
    assert st == 3


def test_ste_rejects(lib):
    assert lib.intlora_ste_backward(None, FAKE, FAKE, 4, 8, 4, FAKE, FAKE, None, 0, None) == 1
    assert lib.intlora_ste_backward(FAKE, FAKE, FAKE, 4, 8, 0, FAKE, FAKE, None, 0, None) == 1
    assert lib.intlora_ste_backward(FAKE, FAKE, FAKE, 0, 8, 4, FAKE, FAKE, None, 0, None) == 1
    assert lib.intlora_ste_backward(FAKE + 2, FAKE, FAKE, 4, 8, 4, FAKE, FAKE, None, 0, None) == 1


def test_empty_batches_are_no_ops(lib):
    assert lib.intlora_gen_aux_batched(None, 0, None, 0, None) == 0
    assert lib.intlora_merge_mul_batched(None, None, 0, 8, None, 0, None) == 0
    assert lib.intlora_ste_backward_batched(None, 0, None, 0, None) == 0


# ---------------------------------------------------------------------------
# widened entry points: host-side validation only (no launch is reached)
# ---------------------------------------------------------------------------
def test_int_planes(lib):
    cases = {0: 1, 127: 1, 128: 2, 16383: 2, 16384: 3, 2**21 - 1: 3, 2**21: 0, -1: 0}
    for v, p in cases.items():
        assert lib.intlora_int_planes(v) == p


def test_int_pack_rejects(lib):
    assert lib.intlora_int_pack(FAKE, 3, 4, 16, 1, FAKE, None, None) == 1      # q_bytes
    assert lib.intlora_int_pack(FAKE, 2, 4, 16, 4, FAKE, None, None) == 1      # planes
    assert lib.intlora_int_pack(FAKE, 2, 4, 24, 2, FAKE, None, None) == 1      # n % 16
    assert lib.intlora_last_error() == b"d >= 0, n >= 0 and n % 16 == 0 required"
    assert lib.intlora_int_pack(FAKE, 2, 4, 16, 2, FAKE + 8, None, None) == 1  # alignment
    assert lib.intlora_int_pack(None, 2, 0, 16, 2, None, None, None) == 0      # empty: no-op


def _igjob(**kw):
    j = B.intlora_int_gemm_job(X=FAKE, x_scale=FAKE, W=FAKE, w_scale=FAKE, tokens=4, d=8, n=32, Y=FAKE)
    for k, v in kw.items():
        setattr(j, k, v)
    return (B.intlora_int_gemm_job * 1)(j)


@pytest.mark.parametrize("field,value", [("n", 24), ("X", FAKE + 4), ("Y", None), ("W", None),
                                         ("tokens", 2**31 + 1), ("n", -16)])
def test_int_gemm_rejects(lib, field, value):
    assert lib.intlora_int_gemm_batched(_igjob(**{field: value}), 1, 1, None) == 1


def test_int_gemm_rejects_planes(lib):
    assert lib.intlora_int_gemm_batched(_igjob(), 1, 0, None) == 1
    assert lib.intlora_int_gemm_batched(_igjob(), 1, 4, None) == 1
    assert lib.intlora_int_gemm_batched(_igjob(tokens=0), 1, 1, None) == 0    # empty: no-op


def test_fakequant_and_linear_reject(lib):
    assert lib.intlora_fakequant_bf16(FAKE, 3, FAKE, 4, 8, FAKE, None) == 1
    assert lib.intlora_fakequant_bf16(FAKE, 2, FAKE, 4, 8, FAKE + 2, None) == 1
    assert lib.intlora_fakequant_bf16(FAKE, 2, None, 4, 8, FAKE, None) == 1
    assert lib.intlora_fakequant_bf16(None, 2, None, 0, 8, None, None) == 0   # empty: no-op
    bad_n = (B.intlora_linear_job * 1)(B.intlora_linear_job(X=FAKE, W=FAKE, tokens=4, d=4, n=12, Y=FAKE))
    assert lib.intlora_linear_bf16_batched(bad_n, 1, None) == 1
    no_x = (B.intlora_linear_job * 1)(B.intlora_linear_job(X=None, W=FAKE, tokens=4, d=4, n=16, Y=FAKE))
    assert lib.intlora_linear_bf16_batched(no_x, 1, None) == 1


def test_distribution_is_validated(lib):
    for bad in (-1, 4):
        jobs = (B.intlora_aux_job * 1)(_aux(distribution=bad))
        assert lib.intlora_gen_aux_batched(jobs, 1, None, 0, None) == 1
        assert "distribution" in lib.intlora_last_error().decode()
        layer = _layer(distribution=bad)
        assert lib.intlora_merge_mul(ctypes.byref(layer), 8, FAKE, FAKE, FAKE, None, None, 0, None) == 1


def _ste(**kw):
    j = B.intlora_ste_job(G=FAKE, A=FAKE, B=FAKE, d=4, n=8, r=4, dA=FAKE, dB=FAKE, mask_codes=FAKE,
                          mask_ld=16, mask_bits=4, mask_z=FAKE)
    for k, v in kw.items():
        setattr(j, k, v)
    return (B.intlora_ste_job * 1)(j)


@pytest.mark.parametrize("field,value", [("mask_bits", 5), ("mask_codes", FAKE + 8), ("mask_z", None),
                                         ("mask_ld", 8), ("n", 7)])
def test_masked_ste_rejects(lib, field, value):
    assert lib.intlora_ste_backward_batched(_ste(**{field: value}), 1, None, 0, None) == 1


def test_masked_ste_workspace_size(lib):
    assert lib.intlora_ste_workspace_size(_ste(d=100, n=24), 1) == (100 * 24 * 2 + 255) // 256 * 256
    assert lib.intlora_ste_workspace_size(_ste(mask_codes=None), 1) == 0


def test_header_is_plain_c(tmp_path):
    """include/intlora.h compiles as C11 with warnings as errors, and the
    descriptor layouts accept positional initializers in declared order."""
    import shutil
    import subprocess
    from pathlib import Path
    if shutil.which("gcc") is None:
        pytest.skip("gcc not available")
    inc = Path(__file__).resolve().parents[1] / "include"
    src = tmp_path / "use.c"
    src.write_text(r'''
#include "intlora.h"
int use(void* p) {
  intlora_aux_job a = {0, 4, 8, 1, 0, 1.5f, 4, 0, 0, 0, p, 16, 0, 0, INTLORA_DIST_CAUCHY};
  intlora_layer l = {4, 8, 4, 4, p, 16, 0, 0, 0, 0, 1, 0, 1.5f, 0, 0, INTLORA_DIST_LAPLACE};
  intlora_ste_job s = {p, p, p, 4, 8, 4, 0, 0, p, 16, 4, 0};
  intlora_int_gemm_job g = {0, 0, 0, 0, 1, 1, 16, p, 1};
  intlora_linear_job f = {p, p, 1, 1, 8, p, 0};
  intlora_fakequant_job q = {p, 2, 0, 1, 8, p};
  return (int)(a.distribution + l.distribution + s.mask_bits + g.y_bf16 + f.y_bf16 + q.q_bytes);
}
''')
    res = subprocess.run(["gcc", "-std=c11", "-Wall", "-Wextra", "-Werror", "-c", str(src), "-I", str(inc),
                          "-o", str(tmp_path / "use.o")], capture_output=True, text=True)
    assert res.returncode == 0, res.stderr


def test_selftest_wait_rejects_bad_limits(lib):
    """The bounded-wait self-test validates its limit before launching."""
    assert lib.intlora_selftest_bounded_wait(0, None) == 1
    assert lib.intlora_selftest_bounded_wait(2_000_000, None) == 1
    assert "limit_us" in lib.intlora_last_error().decode()


def test_launch_counter_is_monotonic(lib):
    a = lib.intlora_kernel_launches()
    lib.intlora_merge_out_bytes(0, 8, 8)           # launches nothing
    assert lib.intlora_kernel_launches() == a


def _tb_job(**kw):
    fake = 0x100000
    f = dict(X=fake, dY=fake, W=fake, A=fake, B=fake, tokens=64, d=64, n=128, r=4,
             dX=fake, dA=fake, dB=fake)
    f.update(kw)
    return B.intlora_train_backward_job(**f)


@pytest.mark.parametrize("field,value", [("d", 12), ("n", 0), ("tokens", 0), ("r", 0), ("r", 65),
                                         ("X", None), ("dB", None), ("W", 0x100008)])
def test_train_backward_rejects(lib, field, value):
    job = _tb_job(**{field: value})
    st = lib.intlora_train_backward_batched(ctypes.byref(job), 1, 0x100000, 1 << 30, None)
    assert st == 1, lib.intlora_last_error()


def test_train_backward_workspace_checked(lib):
    job = _tb_job()
    need = lib.intlora_train_backward_workspace_size(ctypes.byref(job), 1)
    assert need > 0 and need % 256 == 0
    assert lib.intlora_train_backward_batched(ctypes.byref(job), 1, None, 0, None) == 3
    assert lib.intlora_train_backward_batched(ctypes.byref(job), 1, 0x100000, need - 1, None) == 3
    assert lib.intlora_train_backward_batched(ctypes.byref(job), 0, None, 0, None) == 0
