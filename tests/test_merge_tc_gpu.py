"""GPU parity of the fused tensor-core merge (A B on tcgen05 into tensor memory,
U parked there, row extrema combined across the CTAs that share a row)
against the CPU oracle, through the C ABI. INTLORA_MERGE_KERNEL=tc sends
every layer the fused kernel takes to it whatever its rank; the shapes cover
one CTA per row (n <= 512, partial last part of tensor memory), groups of 2 to
28 CTAs over the columns, ragged row groups, ranks 1-128 (K padded to 32, 64
and 128) and every code width / output width pair."""
import numpy as np
import pytest

import oracle
from quantized_lora_merge_b200 import binding as B
from quantized_lora_merge_b200 import workloads as wl

from .parity import gpu_merge, spec_for
from .test_parity_gpu import _check_mul, _check_shift, _oracle_prepared

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def fused(monkeypatch):
    monkeypatch.setenv("INTLORA_MERGE_KERNEL", "tc")


FUSED_MUL = [
    # d, n, r, w_bits, u_bits
    (130, 4096, 16, 8, 8),    # Llama width: 8 CTAs per row, int32 products, ragged last row group
    (64, 14336, 16, 8, 8),    # Llama down width: 28 CTAs per row
    (128, 320, 4, 4, 4),      # one CTA per row group, int4 codes, int16 products
    (257, 640, 8, 8, 6),      # 6-bit U (int16 products), three row groups
    (40, 1024, 33, 8, 8),     # rank padded to 64
    (33, 2048, 128, 8, 8),    # rank 128: four K atoms
    (5, 96, 1, 4, 8),         # rank 1, slice of 96 columns
    (70, 8192, 64, 4, 4),     # 16 CTAs per row
    (129, 9216, 16, 8, 8),    # 18 CTAs per row, last row group of one row
]


@pytest.mark.parametrize("d,n,r,w_bits,u_bits", FUSED_MUL)
def test_fused_merge_mul_parity(d, n, r, w_bits, u_bits):
    spec = spec_for(d, n, r, w_bits, "mul", u_bits, sid=500 + d)
    inp = _oracle_prepared(spec)
    got = gpu_merge([spec], [inp])[0]
    _check_mul(spec, inp, got)


FUSED_SHIFT = [
    (96, 3072, 64, 4, 4),     # DiT width: 6 CTAs per row
    (40, 12288, 64, 4, 4),    # DiT fc2 width: 24 CTAs per row
    (129, 512, 16, 8, 4),     # 8-bit base: int16 merged codes
    (3, 64, 7, 4, 2),         # 2-bit shift code
]


@pytest.mark.parametrize("d,n,r,w_bits,shift_bits", FUSED_SHIFT)
def test_fused_merge_shift_parity(d, n, r, w_bits, shift_bits):
    spec = spec_for(d, n, r, w_bits, "shift", shift_bits, sid=600 + d)
    inp = _oracle_prepared(spec)
    got = gpu_merge([spec], [inp])[0]
    _check_shift(spec, inp, got)


def test_fused_batch_of_mixed_geometries():
    """One batched call whose layers need different numbers of CTAs per row
    (several launches sharing the exchange area), with sigma_R reduced on the
    device."""
    specs = [spec_for(d, n, r, 8, "mul", 8, sid=700 + k)
             for k, (d, n, r) in enumerate([(64, 4096, 16), (20, 14336, 16), (130, 320, 8),
                                            (64, 4096, 32), (9, 2048, 16)])]
    inps = [_oracle_prepared(s) for s in specs]
    got = gpu_merge(specs, inps, pass_sigma_r=False)
    for spec, inp, g in zip(specs, inps, got):
        _check_mul(spec, inp, g)


def test_fused_and_row_kernels_agree(monkeypatch):
    """The same layers through the fused kernel and through the row kernels:
    codes differ only where a value sits within the tolerance window of a
    rounding boundary (T from tensor cores vs. fp32 FMAs)."""
    specs = [spec_for(d, n, r, 8, "mul", 8, sid=800 + k)
             for k, (d, n, r) in enumerate([(128, 4096, 16), (64, 14336, 16), (100, 1024, 64)])]
    inps = [_oracle_prepared(s) for s in specs]
    res = {}
    for kernel in ("tc", "rows"):
        monkeypatch.setenv("INTLORA_MERGE_KERNEL", kernel)
        res[kernel] = gpu_merge(specs, inps)
    for x, y in zip(res["tc"], res["rows"]):
        assert np.mean(x["out"] != y["out"]) < 1e-3
        assert np.max(np.abs(x["sbar"] / y["sbar"] - 1)) < 1e-6


def test_fused_without_code_output_and_repeat():
    """Without the optional code output the products are the same, and a
    second call on the same buffers reproduces the first bit for bit."""
    spec = spec_for(96, 4096, 16, 8, "mul", 8, sid=33)
    inp = _oracle_prepared(spec)
    a = gpu_merge([spec], [inp], want_code=False)[0]
    b = gpu_merge([spec], [inp], want_code=True)[0]
    c = gpu_merge([spec], [inp], want_code=True)[0]
    assert np.array_equal(a["out"], b["out"]) and np.array_equal(b["out"], c["out"])
    assert np.array_equal(b["code"], c["code"]) and np.array_equal(b["sbar"], c["sbar"])


@pytest.mark.parametrize("r", [4, 8])
def test_wide_low_rank_rows_route_to_fused(monkeypatch, r):
    """Rows wider than the team kernels take (n > 6144) go to the fused kernel
    at any rank under the default routing (a batch with a narrow layer of the
    same rank beside it): both layers meet the oracle, and the wide one agrees
    with the rows path (A B on the CUDA cores) up to the rounding-boundary
    codes the two ways of forming A B may split differently."""
    specs = [spec_for(70, 8192, r, 8, "mul", 8, sid=90 + r), spec_for(64, 1024, r, 8, "mul", 8, sid=91 + r)]
    inps = [_oracle_prepared(sp) for sp in specs]
    monkeypatch.setenv("INTLORA_MERGE_KERNEL", "auto")
    auto = gpu_merge(specs, inps, batched=True)
    monkeypatch.setenv("INTLORA_MERGE_KERNEL", "rows")
    rows = gpu_merge(specs, inps, batched=True)
    for sp, inp, x, y in zip(specs, inps, auto, rows):
        assert np.mean(x["out"] != y["out"]) < 1e-3
        assert np.max(np.abs(x["sbar"] / y["sbar"] - 1)) < 1e-6
        _check_mul(sp, inp, x)


def test_fused_no_device_wait_gave_up():
    assert B.intlora_device_status() == 0
