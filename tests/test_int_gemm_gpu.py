"""GPU parity of the integer inference GEMM on merged weights (Y = X W'^T with
W' = s_bar Q, Q held as base-128 int8 digit planes) against the oracle,
through the C ABI. Digit packing is integer work: bit-exact. The GEMM's
integer sums are exact on both sides; the GPU then rounds three times in fp32
(sum -> fp32, x_scale * w_scale, the product), so Y agrees within 1e-6
relative (3 * 2^-24 ~ 1.8e-7 is the bound), and bit-exactly where the scales
are 1 and the sums stay below 2^24."""
import numpy as np
import pytest
import torch

import oracle
from quantized_lora_merge_b200 import binding as B
from quantized_lora_merge_b200 import workloads as wl

from .parity import dev, spec_for

pytestmark = pytest.mark.gpu

Y_RTOL = 1e-6


def _t(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to(dev())


def _pack(Q, planes, q_dtype=np.int32):
    q = _t(Q.astype(q_dtype))
    packed = torch.zeros((Q.shape[0], planes, Q.shape[1]), dtype=torch.int8, device=dev())
    ovf = torch.zeros(1, dtype=torch.int32, device=dev())
    B.intlora_int_pack(q, planes, packed, ovf)
    torch.cuda.synchronize()
    return packed, int(ovf.item())


def _gemm(X, xs, packed, ws, planes):
    Xd, xsd, wsd = _t(X), _t(xs), _t(ws)
    Y = torch.full((X.shape[0], packed.shape[0]), float("nan"), device=dev())
    B.intlora_int_gemm(B.IntGemmJob(Xd, xsd, packed, wsd, Y), planes)
    torch.cuda.synchronize()
    return Y.cpu().numpy().astype(np.float64)


def _assert_y(Y, Yo):
    assert np.all(np.isfinite(Y)), "Y has unwritten (NaN) entries"
    rel = np.abs(Y - Yo) / np.maximum(np.abs(Yo), 1e-300)
    rel[(Yo == 0) & (Y == 0)] = 0.0
    assert rel.max(initial=0.0) <= Y_RTOL, f"max rel err {rel.max():.3e}"


# ---------------------------------------------------------------------------
# digit planes
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("q_dtype,planes,bound", [(np.int8, 1, 127), (np.int16, 2, 225),
                                                   (np.int32, 3, 65025), (np.int16, 2, 16383),
                                                   (np.int32, 3, 2**21 - 1), (np.int32, 2, 15)])
def test_pack_bit_exact(q_dtype, planes, bound):
    _, _, Q, _ = wl.int_gemm_host(1, 37, 272, bound, salt=planes)
    Q[0, :4] = [bound, -bound, 0, -1]
    packed, ovf = _pack(Q, planes, q_dtype)
    want, bad = oracle.int_digits(Q, planes)
    assert ovf == 0 and bad == 0
    assert np.array_equal(packed.cpu().numpy(), want)


def test_pack_counts_overflow():
    Q = np.zeros((2, 16), np.int32)
    Q[0, :5] = [128, -129, 127, -128, 5000]
    Q[1, :2] = [16384, -16385]
    for planes in (1, 2):
        packed, ovf = _pack(Q, planes)
        want, bad = oracle.int_digits(Q, planes)
        assert ovf == bad and bad > 0
        assert np.array_equal(packed.cpu().numpy(), want)


# ---------------------------------------------------------------------------
# GEMM
# ---------------------------------------------------------------------------
GEMM_CASES = [  # planes, bound, tokens, d, n: several tiles and ragged tails in every dimension
    (1, 15, 128, 256, 128), (1, 127, 200, 300, 144), (2, 225, 129, 257, 272),
    (3, 65025, 77, 100, 4112), (1, 15, 1, 1, 16), (2, 225, 3, 129, 16), (1, 15, 300, 520, 1040),
    (3, 65025, 256, 64, 256), (2, 255, 513, 130, 384), (1, 15, 140, 1000, 48)]


@pytest.mark.parametrize("planes,bound,tokens,d,n", GEMM_CASES)
def test_int_gemm_parity(planes, bound, tokens, d, n):
    X, xs, Q, ws = wl.int_gemm_host(tokens, d, n, bound)
    packed, ovf = _pack(Q, planes)
    assert ovf == 0
    Y = _gemm(X, xs, packed, ws, planes)
    _assert_y(Y, oracle.int_gemm_rows(X, xs, Q, ws))


@pytest.mark.parametrize("planes,bound,n", [(1, 15, 160), (2, 225, 160), (3, 4000, 16)])
def test_int_gemm_integer_sums_exact(planes, bound, n):
    """Unit scales and |sum| < 2^24: every output is the exact integer sum."""
    X, _, Q, _ = wl.int_gemm_host(130, 260, n, bound, salt=9)
    assert 127 * bound * n < 2**24
    packed, _ = _pack(Q, planes)
    Y = _gemm(X, np.ones(130, np.float32), packed, np.ones(260, np.float32), planes)
    exact = X.astype(np.int64) @ Q.astype(np.int64).T
    assert np.array_equal(Y, exact.astype(np.float64))


def test_int_gemm_on_merged_mul_weights():
    """The oracle's MUL merge of a 4-bit layer (P int, s_bar) through pack and
    GEMM: Y = dequantized activations x merged weights."""
    spec = spec_for(96, 320, 4, 4, sid=31)
    W = wl.host_W(spec)
    g = oracle.gen_aux(W, spec.seed, spec.stream_id, spec.alpha, 4)
    m = oracle.merge_mul(g["codes"], g["s"].astype(np.float32), g["z"], wl.host_A(spec),
                         wl.host_B(spec), spec.seed, spec.stream_id, g["sigma_w"], g["sigma_r"],
                         spec.alpha, 4)
    P = m["P"].astype(np.int32)
    sbar = m["sbar"].astype(np.float32)
    planes = oracle.int_planes(int(np.abs(P).max()))
    X, xs, _, _ = wl.int_gemm_host(200, 96, 320, 1, salt=3)
    packed, ovf = _pack(P, planes, np.int16)
    assert ovf == 0
    Y = _gemm(X, xs, packed, sbar, planes)
    _assert_y(Y, oracle.int_gemm_rows(X, xs, P, sbar))


def test_int_gemm_batched_equals_single_calls():
    shapes = [(1, 15, 200, 300, 144), (1, 15, 64, 640, 256), (1, 15, 1, 17, 32)]
    jobs, singles = [], []
    for k, (planes, bound, tokens, d, n) in enumerate(shapes):
        X, xs, Q, ws = wl.int_gemm_host(tokens, d, n, bound, salt=k)
        packed, _ = _pack(Q, planes)
        singles.append(_gemm(X, xs, packed, ws, planes))
        Y = torch.full((tokens, d), float("nan"), device=dev())
        jobs.append(B.IntGemmJob(_t(X), _t(xs), packed, _t(ws), Y))
    B.intlora_int_gemm_batched(jobs, 1)
    torch.cuda.synchronize()
    for j, s in zip(jobs, singles):
        assert np.array_equal(j.Y.cpu().numpy().astype(np.float64), s)


def test_int_gemm_degenerate_and_invalid():
    X = torch.zeros((5, 0), dtype=torch.int8, device=dev())
    W = torch.zeros((7, 1, 0), dtype=torch.int8, device=dev())
    Y = torch.full((5, 7), 3.0, device=dev())
    xs, ws = torch.ones(5, device=dev()), torch.ones(7, device=dev())
    B.intlora_int_gemm(B.IntGemmJob(X, xs, W, ws, Y), 1)          # n = 0: Y = 0
    torch.cuda.synchronize()
    assert torch.count_nonzero(Y).item() == 0
    Y0 = torch.zeros((0, 7), device=dev())
    B.intlora_int_gemm(B.IntGemmJob(torch.zeros((0, 16), dtype=torch.int8, device=dev()), xs,
                                    torch.zeros((7, 1, 16), dtype=torch.int8, device=dev()), ws,
                                    Y0), 1)
    with pytest.raises(B.IntLoRAError):
        B.intlora_int_gemm(B.IntGemmJob(torch.zeros((5, 24), dtype=torch.int8, device=dev()), xs,
                                        torch.zeros((7, 1, 24), dtype=torch.int8, device=dev()),
                                        ws, Y), 1)
    with pytest.raises(B.IntLoRAError):
        B.intlora_int_gemm(B.IntGemmJob(torch.zeros((5, 16), dtype=torch.int8, device=dev()), xs,
                                        torch.zeros((7, 4, 16), dtype=torch.int8, device=dev()),
                                        ws, Y), 4)


# ---------------------------------------------------------------------------
# full size, sampled rows (the shapes the benchmark times)
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("planes,bound,tokens,d,n", [(1, 15, 4096, 12288, 3072),
                                                     (2, 225, 4096, 1280, 5120),
                                                     (3, 65025, 2048, 4096, 4096)])
def test_int_gemm_full_size_sampled(planes, bound, tokens, d, n):
    Xd, xsd, Qd, wsd = wl.int_gemm_device(tokens, d, n, bound, dev())
    packed = torch.empty((d, planes, n), dtype=torch.int8, device=dev())
    ovf = torch.zeros(1, dtype=torch.int32, device=dev())
    B.intlora_int_pack(Qd, planes, packed, ovf)
    Y = torch.empty((tokens, d), device=dev())
    B.intlora_int_gemm(B.IntGemmJob(Xd, xsd, packed, wsd, Y), planes)
    torch.cuda.synchronize()
    assert ovf.item() == 0
    rows = np.array([0, 1, 127, 128, tokens // 2 + 5, tokens - 1])
    Yo = oracle.int_gemm_rows(Xd.cpu().numpy(), xsd.cpu().numpy().astype(np.float64),
                              Qd.cpu().numpy(), wsd.cpu().numpy().astype(np.float64), rows)
    _assert_y(Y[torch.from_numpy(rows).to(dev())].cpu().numpy().astype(np.float64), Yo)
    assert B.intlora_device_status() == 0


@pytest.mark.parametrize("planes,bound,tokens,d,n", [(1, 15, 200, 304, 144), (2, 225, 129, 257, 272),
                                                     (1, 15, 33, 12, 64)])
def test_int_gemm_bf16_output(planes, bound, tokens, d, n):
    """Y in bf16 (TMA-stored when d % 8 == 0, else stored directly) is the
    fp32 result rounded to nearest even, from the same accumulators."""
    X, xs, Q, ws = wl.int_gemm_host(tokens, d, n, bound, salt=4)
    packed, _ = _pack(Q, planes)
    Xd, xsd, wsd = _t(X), _t(xs), _t(ws)
    Y32 = torch.empty((tokens, d), device=dev())
    Y16 = torch.full((tokens, d), float("nan"), dtype=torch.bfloat16, device=dev())
    B.intlora_int_gemm_batched([B.IntGemmJob(Xd, xsd, packed, wsd, Y32)], planes)
    B.intlora_int_gemm_batched([B.IntGemmJob(Xd, xsd, packed, wsd, Y16)], planes)
    torch.cuda.synchronize()
    assert torch.equal(Y16.view(torch.int16), Y32.to(torch.bfloat16).view(torch.int16))
    _assert_y(Y32.cpu().numpy().astype(np.float64), oracle.int_gemm_rows(X, xs, Q, ws))
