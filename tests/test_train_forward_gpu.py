"""GPU parity of the training forward on merged weights: the fake-quantized
bf16 weight W'_bf16 = bf16(fp32(s_bar_i) Q_ij) (bit-exact: both sides round
the same fp32 product to bf16 with ties to even) and the layer GEMM
Y = X W'^T on the tensor cores (bf16 operands, fp32 accumulation: within the
accumulation bound K 2^-24 sum_j |x_j w_j| of the fp64 oracle)."""
import numpy as np
import pytest
import torch

import oracle
from quantized_lora_merge_b200 import binding as B
from quantized_lora_merge_b200 import workloads as wl

from .parity import dev, spec_for

pytestmark = pytest.mark.gpu


def _t(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to(dev())


def _bf16(bits):
    return _t(bits.view(np.int16)).view(torch.bfloat16)


def _fakequant(Q, sbar, q_dtype):
    w = torch.empty(Q.shape, dtype=torch.bfloat16, device=dev())
    B.intlora_fakequant_bf16(_t(Q.astype(q_dtype)), _t(sbar.astype(np.float32)), w)
    torch.cuda.synchronize()
    return w


def _bits(t):
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def _check_y(Y, Xb, Wb, rows=None):
    Yo = oracle.linear_rows(Xb, Wb, rows)
    xa = np.abs(wl.bf16_bits_to_f32(Xb).astype(np.float64))
    wa = np.abs(wl.bf16_bits_to_f32(Wb).astype(np.float64))
    if rows is not None:
        xa = xa[rows]
    bound = Xb.shape[1] * 2.0**-24 * (xa @ wa.T) + 1e-30
    assert np.all(np.isfinite(Y))
    assert np.all(np.abs(Y - Yo) <= bound), f"max excess {np.max(np.abs(Y - Yo) / bound):.3f}"


@pytest.mark.parametrize("q_dtype,bound", [(np.int8, 15), (np.int16, 225), (np.int32, 65025)])
def test_fakequant_bit_exact(q_dtype, bound):
    rng = np.random.default_rng(bound)
    Q = rng.integers(-bound, bound + 1, (37, 136))
    sbar = rng.uniform(1e-5, 1e-2, 37).astype(np.float32)
    w = _fakequant(Q, sbar, q_dtype)
    assert np.array_equal(_bits(w), oracle.fakequant_bf16(Q, sbar))


@pytest.mark.parametrize("tokens,d,n", [(128, 256, 64), (200, 300, 136), (1, 1, 8), (257, 520, 1032),
                                        (77, 100, 4104), (130, 17, 16)])
def test_linear_bf16_parity(tokens, d, n):
    rng = np.random.default_rng([tokens, d, n])
    Xb = wl.to_bf16_bits(rng.standard_normal((tokens, n)).astype(np.float32))
    Wb = wl.to_bf16_bits((rng.standard_normal((d, n)) * 0.05).astype(np.float32))
    Y = torch.full((tokens, d), float("nan"), device=dev())
    B.intlora_linear_bf16_batched([B.LinearJob(_bf16(Xb), _bf16(Wb), Y)])
    torch.cuda.synchronize()
    _check_y(Y.cpu().numpy().astype(np.float64), Xb, Wb)


def test_forward_on_merged_mul_weights():
    """The oracle's MUL merge of a 4-bit layer: fake-quantized on the GPU
    (bit-exact) and multiplied by bf16 activations."""
    spec = spec_for(96, 320, 4, 4, sid=41)
    W = wl.host_W(spec)
    g = oracle.gen_aux(W, spec.seed, spec.stream_id, spec.alpha, 4)
    m = oracle.merge_mul(g["codes"], g["s"].astype(np.float32), g["z"], wl.host_A(spec),
                         wl.host_B(spec), spec.seed, spec.stream_id, g["sigma_w"], g["sigma_r"],
                         spec.alpha, 4)
    sbar = m["sbar"].astype(np.float32)
    w = _fakequant(m["P"], sbar, np.int16)
    Wb = oracle.fakequant_bf16(m["P"], sbar)
    assert np.array_equal(_bits(w), Wb)
    Xb = wl.to_bf16_bits(np.random.default_rng(5).standard_normal((200, 320)).astype(np.float32))
    Y = torch.empty((200, 96), device=dev())
    B.intlora_linear_bf16_batched([B.LinearJob(_bf16(Xb), w, Y)])
    torch.cuda.synchronize()
    _check_y(Y.cpu().numpy().astype(np.float64), Xb, Wb)


def test_linear_bf16_full_size_sampled():
    """The SD feed-forward shape at 4096 tokens (the benchmark's size)."""
    tokens, d, n = 4096, 5120, 1280
    g = torch.Generator(device=dev())
    g.manual_seed(7)
    X = torch.randn(tokens, n, generator=g, device=dev()).to(torch.bfloat16)
    Wt = (torch.randn(d, n, generator=g, device=dev()) * 0.02).to(torch.bfloat16)
    Y = torch.empty((tokens, d), device=dev())
    B.intlora_linear_bf16_batched([B.LinearJob(X, Wt, Y)])
    torch.cuda.synchronize()
    rows = np.array([0, 1, 127, 128, 2049, tokens - 1])
    Xb, Wb = _bits(X), _bits(Wt)
    _check_y(Y[torch.from_numpy(rows).to(dev())].cpu().numpy().astype(np.float64), Xb, Wb, rows)
    assert B.intlora_device_status() == 0


def test_fakequant_batched_and_ragged():
    """One launch over layers of several widths and code types, ragged rows
    (n % 4 != 0) included."""
    rng = np.random.default_rng(23)
    cases = [(5, 6, np.int16, 225), (9, 50, np.int32, 65025), (16, 64, np.int8, 15),
             (33, 136, np.int16, 225), (1, 2, np.int32, 100)]
    jobs, want = [], []
    for d, n, dt, bound in cases:
        Q = rng.integers(-bound, bound + 1, (d, n))
        sbar = rng.uniform(1e-5, 1e-2, d).astype(np.float32)
        jobs.append(B.FakeQuantJob(_t(Q.astype(dt)), _t(sbar),
                                   torch.empty((d, n), dtype=torch.bfloat16, device=dev())))
        want.append(oracle.fakequant_bf16(Q, sbar))
    B.intlora_fakequant_bf16_batched(jobs)
    torch.cuda.synchronize()
    for j, w in zip(jobs, want):
        assert np.array_equal(_bits(j.w_out), w)


@pytest.mark.parametrize("tokens,d,n", [(200, 304, 136), (77, 100, 64)])
def test_linear_bf16_output(tokens, d, n):
    rng = np.random.default_rng([tokens, d])
    Xb = wl.to_bf16_bits(rng.standard_normal((tokens, n)).astype(np.float32))
    Wb = wl.to_bf16_bits((rng.standard_normal((d, n)) * 0.05).astype(np.float32))
    Y32 = torch.empty((tokens, d), device=dev())
    Y16 = torch.full((tokens, d), float("nan"), dtype=torch.bfloat16, device=dev())
    B.intlora_linear_bf16_batched([B.LinearJob(_bf16(Xb), _bf16(Wb), Y32),
                                   B.LinearJob(_bf16(Xb), _bf16(Wb), Y16)])
    torch.cuda.synchronize()
    assert torch.equal(Y16.view(torch.int16), Y32.to(torch.bfloat16).view(torch.int16))
    _check_y(Y32.cpu().numpy().astype(np.float64), Xb, Wb)
