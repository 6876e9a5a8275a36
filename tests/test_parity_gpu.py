"""GPU parity: every stage of the CUDA path against the CPU oracle on the same
seeded inputs, through the C ABI. Each stage is fed the oracle's inputs, so a
difference in one stage cannot cascade into the next."""
import numpy as np
from dataclasses import replace
import pytest
import torch

import oracle
from quantized_lora_merge_b200 import binding as B
from quantized_lora_merge_b200 import pipeline as P
from quantized_lora_merge_b200 import workloads as wl

from .parity import (STE_RTOL, assert_affine, assert_scale, assert_shift, dev, gpu_gen_aux,
                     gpu_merge, gpu_ste, rel_fro, spec_for)

pytestmark = pytest.mark.gpu


# ---------------------------------------------------------------------------
# a1: Philox + Laplace, materialised through gen_aux with alpha = 0 (R* = R)
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("d,n", [(256, 1024), (37, 50), (3, 6)])
def test_aux_matrix_matches_oracle(d, n):
    spec = spec_for(d, n, 4, 8, alpha=0.0, sid=5)
    W = wl.host_W(spec)
    g = gpu_gen_aux([spec], [W], want_r_star=True)[0]
    R = oracle.aux_R(d, n, spec.seed, spec.stream_id)
    err = np.abs(g["r_star"].astype(np.float64) - R)
    assert np.max(err / np.maximum(1.0, np.abs(R))) < 2e-6
    assert np.array_equal(np.sign(g["r_star"]), np.sign(R))


# ---------------------------------------------------------------------------
# a1-a3: layer preparation
# ---------------------------------------------------------------------------
GEN_SHAPES = [(320, 320, 8), (64, 768, 4), (33, 100, 8), (7, 10, 4), (5, 6, 8), (1, 4, 8),
              (130, 5120, 4), (20, 14336, 8), (9, 2, 4),
              # rows of whole 8-warp sweeps past 6144 columns: tensor-memory parking
              # (7 and 8 sweeps: all in tensor memory; 12 and 14: the rest in shared memory)
              (13, 14336, 4), (70, 12288, 8), (9, 7168, 8), (6, 8192, 4)]


@pytest.mark.parametrize("d,n,w_bits", GEN_SHAPES)
def test_gen_aux_parity(d, n, w_bits):
    spec = spec_for(d, n, 4, w_bits, sid=d + n)
    W = wl.host_W(spec)
    g = gpu_gen_aux([spec], [W])[0]
    o = oracle.gen_aux(W, spec.seed, spec.stream_id, spec.alpha, w_bits)
    assert_scale("sigma_w", g["sigma_w"], o["sigma_w"])
    assert_scale("sigma_r", g["sigma_r"], o["sigma_r"])
    assert_scale("s", g["s"], o["s"])
    assert_affine("W_round", g["codes"], g["z"], o["codes"], o["z"], o["pre"], o["zpre"],
                  2**w_bits - 1)


def test_gen_aux_wide_rows_team_equals_tile(monkeypatch):
    """The tensor-memory-parked team kernel and the row-tile kernels give the
    same codes, scales and zero-points on wide rows (one batch of mixed widths)."""
    specs = [spec_for(d, n, 4, b, sid=60 + k) for k, (d, n, b) in
             enumerate([(21, 14336, 8), (8, 12288, 4), (5, 7168, 8), (12, 4096, 8)])]
    Ws = [wl.host_W(s) for s in specs]
    monkeypatch.setenv("INTLORA_ROW_KERNEL", "tile")
    tile = gpu_gen_aux(specs, Ws, batched=True)
    monkeypatch.setenv("INTLORA_ROW_KERNEL", "auto")
    team = gpu_gen_aux(specs, Ws, batched=True)
    for x, y in zip(team, tile):
        assert np.array_equal(x["codes"], y["codes"])
        assert np.array_equal(x["s"], y["s"]) and np.array_equal(x["z"], y["z"])


def test_gen_aux_batched_equals_single():
    specs = [spec_for(d, n, 4, b, sid=k) for k, (d, n, b) in enumerate(GEN_SHAPES[:5])]
    Ws = [wl.host_W(s) for s in specs]
    a = gpu_gen_aux(specs, Ws, batched=True)
    b = gpu_gen_aux(specs, Ws, batched=False)
    for x, y in zip(a, b):
        assert x["sigma_w"] == y["sigma_w"] and x["sigma_r"] == y["sigma_r"]
        assert np.array_equal(x["codes"], y["codes"]) and np.array_equal(x["s"], y["s"])


# ---------------------------------------------------------------------------
# a4-a7: merges, on the oracle's prepared layers
# ---------------------------------------------------------------------------
def _oracle_prepared(spec):
    W = wl.host_W(spec)
    g = oracle.gen_aux(W, spec.seed, spec.stream_id, spec.alpha, spec.w_bits, dist=spec.distribution)
    return dict(codes=g["codes"], s=g["s"].astype(np.float32), z=g["z"], A=wl.host_A(spec),
                B=wl.host_B(spec), sigma_w=g["sigma_w"], sigma_r=g["sigma_r"])


def _lg2_sbar_bound(spec, inp, qmax):
    """Absolute bound on s_bar from the GPU's fast log2 (absolute error at most
    2^-22 for arguments in [0.5, 2]): each row extremum of U carries
    c ln2 2^-22 of it (|D| >= 1), so s_bar = (u_max - u_min) / qmax carries
    twice that over qmax. Where R* dwarfs W (alpha = 0) this is ~1e-6 of
    s_bar; at the configs' alpha = 1.5 it stays below the 1e-6 bound."""
    c = (inp["sigma_w"] / inp["sigma_r"]) ** spec.alpha
    return 2.0 * c * np.log(2.0) * 2.0**-22 / qmax


def _check_mul(spec, inp, got, lg2_bound=False):
    o = oracle.merge_mul(inp["codes"], inp["s"], inp["z"], inp["A"], inp["B"], spec.seed,
                         spec.stream_id, inp["sigma_w"], inp["sigma_r"], spec.alpha,
                         spec.out_bits, dist=spec.distribution)
    qmax = 2**spec.out_bits - 1
    if lg2_bound:
        err = np.abs(got["sbar"].astype(np.float64) - o["sbar"])
        assert np.all(err <= 1e-6 * np.abs(o["sbar"]) + _lg2_sbar_bound(spec, inp, qmax))
    else:
        assert_scale("s_bar", got["sbar"], o["sbar"])
    assert_affine("U_round", got["code"], got["zbar"], o["u_round"], o["zbar"], o["pre"],
                  o["zpre"], qmax)
    D = inp["codes"].astype(np.int64) - inp["z"][:, None]
    # the products are exactly (U_round - z_bar) * D of the GPU's own codes ...
    assert np.array_equal(got["out"], (got["code"].astype(np.int64) - got["zbar"][:, None]) * D)
    # ... and equal to the oracle's wherever the codes agree
    same = (got["code"] == o["u_round"]) & (got["zbar"] == o["zbar"])[:, None]
    assert np.array_equal(got["out"][same], o["P"][same])
    assert np.all(got["out"][D == 0] == 0)


def _check_shift(spec, inp, got, lg2_bound=False):
    o = oracle.merge_shift(inp["codes"], inp["s"], inp["z"], inp["A"], inp["B"], spec.seed,
                           spec.stream_id, inp["sigma_w"], inp["sigma_r"], spec.alpha,
                           spec.out_bits, dist=spec.distribution)
    if lg2_bound:
        # s_bar = max |U| carries one extremum's error (not two, nor / qmax)
        c = (inp["sigma_w"] / inp["sigma_r"]) ** spec.alpha
        err = np.abs(got["sbar"].astype(np.float64) - o["sbar"])
        assert np.all(err <= 1e-6 * np.abs(o["sbar"]) + c * np.log(2.0) * 2.0**-22)
        # The shift is the nearest integer of x = -log2|U / s_bar|, whose
        # sensitivity to an absolute error e of U is e / (|U| ln 2). The GPU
        # forms U = s + (R* + A B) / D in fp32 with a fast log2 inside R*:
        # e <= 2^-20 (|s| + |U - s| + |U|) (a few roundings of the terms that
        # cancel) + c ln2 2^-22 / |D|. A differing shift is allowed within
        # that window of x around k + 1/2 (plus the usual 1e-5 relative).
        D = inp["codes"].astype(np.float64) - inp["z"][:, None]
        s_i = inp["s"].astype(np.float64)[:, None]
        U = np.asarray(o["U"], np.float64)
        e = 2.0**-20 * (np.abs(s_i) + np.abs(U - s_i) + np.abs(U)) + \
            c * np.log(2.0) * 2.0**-22 / np.maximum(np.abs(D), 1.0)
        x = np.asarray(o["pre"], np.float64)
        g, oc = np.asarray(got["code"], np.int64), np.asarray(o["shift"], np.int64)
        mism = g != oc
        assert np.all(np.abs(g - oc)[mism] == 1)
        frac = x - np.floor(x)
        win = 1e-5 * np.maximum(np.abs(x), 1.0) + e / np.maximum(np.abs(U), 1e-300) / np.log(2.0)
        assert np.all(np.abs(frac - 0.5)[mism] <= win[mism])
    else:
        assert_scale("s_bar", got["sbar"], o["sbar"])
        assert_shift("shift", got["code"], o["shift"], o["pre"], 2**spec.out_bits - 1)
    D = inp["codes"].astype(np.int64) - inp["z"][:, None]
    sign = np.sign(o["U"]).astype(np.int64)
    mag = D >> got["code"].astype(np.int64)
    if lg2_bound:
        # the sign of a U within its error bound of zero is not decided
        sure = np.abs(np.asarray(o["U"], np.float64)) > e
        assert np.array_equal(got["out"][sure], (sign * mag)[sure])
        a = np.abs(got["out"][~sure])
        assert np.all((a == np.abs(mag)[~sure]) | (a == 0))
    else:
        assert np.array_equal(got["out"], sign * mag)
    same = (got["code"] == o["shift"]) & (np.abs(np.asarray(o["U"], np.float64)) > (e if lg2_bound else 0.0))
    assert np.array_equal(got["out"][same], o["M"][same])


MUL_CASES = [
    # d, n, r, w_bits, u_bits
    (320, 320, 4, 8, 8),      # the single 320x320 layer
    (64, 768, 4, 4, 4),       # SD cross-attention shape, int4
    (40, 4096, 16, 8, 8),     # Llama width, cluster of CTAs over the columns
    (24, 14336, 16, 8, 8),    # Llama down-projection width
    (12, 4096, 128, 8, 8),    # rank 128: B streamed through shared memory
    (9, 50, 3, 8, 8),         # ragged: n % 4 != 0, rank not a template
    (130, 5120, 4, 4, 4),     # FF width 4d at d = 1280
    (1, 8, 1, 4, 4),          # single row, rank 1
    (17, 64, 8, 8, 6),        # 6-bit U quantizer (int16 products)
    # ranks 32..64: A B from the tensor cores (tf32 three-term split)
    (100, 1024, 32, 8, 8),
    (129, 256, 33, 8, 8),     # ragged rank (padded to 64) and row block
    (33, 8200, 64, 4, 4),     # wider than the team kernels: row-tile kernels read T
    (7, 100, 48, 4, 4),
    # ranks 65..128: two tensor-core passes over the rank, second product added
    (100, 1024, 96, 8, 8),
    (33, 520, 72, 4, 4),      # second pass of rank 8 (padded to 32)
    (129, 8200, 128, 8, 8),
]


@pytest.mark.parametrize("d,n,r,w_bits,u_bits", MUL_CASES)
def test_merge_mul_parity(d, n, r, w_bits, u_bits):
    spec = spec_for(d, n, r, w_bits, "mul", u_bits, sid=7 + d)
    inp = _oracle_prepared(spec)
    got = gpu_merge([spec], [inp])[0]
    _check_mul(spec, inp, got)


SHIFT_CASES = [
    (32, 3072, 64, 4, 4),     # DiT width, r = 64, 4-bit base, 4-bit shift
    (16, 3072, 128, 4, 4),    # two tensor-core passes
    (16, 12288, 64, 4, 4),    # DiT fc2 width
    (48, 320, 4, 8, 4),       # 8-bit base: int16 merged codes
    (5, 6, 2, 4, 2),          # ragged, 2-bit shift code (clamps at 3)
    (3, 40, 32, 8, 5),
]


@pytest.mark.parametrize("d,n,r,w_bits,shift_bits", SHIFT_CASES)
def test_merge_shift_parity(d, n, r, w_bits, shift_bits):
    spec = spec_for(d, n, r, w_bits, "shift", shift_bits, sid=11 + d)
    inp = _oracle_prepared(spec)
    got = gpu_merge([spec], [inp])[0]
    _check_shift(spec, inp, got)


@pytest.mark.parametrize("variant", ["mul", "shift"])
def test_merge_tensor_core_t_and_cuda_core_t_agree(monkeypatch, variant):
    """The same layers with A B from the tensor cores and from the CUDA cores:
    both meet the oracle, and their codes differ only where a value sits
    within the tolerance window of a rounding boundary."""
    specs = [spec_for(d, n, r, 4, variant, 4, sid=300 + k)
             for k, (d, n, r) in enumerate([(64, 3072, 64), (40, 640, 32), (12, 6400, 64), (24, 1024, 128)])]
    inps = [_oracle_prepared(s) for s in specs]
    res = {}
    for kernel in ("auto", "cuda"):
        monkeypatch.setenv("INTLORA_T_KERNEL", kernel)
        res[kernel] = gpu_merge(specs, inps, batched=True)
        for spec, inp, got in zip(specs, inps, res[kernel]):
            (_check_mul if variant == "mul" else _check_shift)(spec, inp, got)
    for x, y in zip(res["auto"], res["cuda"]):
        assert np.mean(x["out"] != y["out"]) < 1e-3


EDGE_SHAPES = [(130, 4096, 16, 8, 8), (64, 320, 4, 4, 4), (40, 3072, 64, 4, 4)]


@pytest.mark.parametrize("kernel", ["rows", "tc"])
@pytest.mark.parametrize("d,n,r,w_bits,out_bits", EDGE_SHAPES)
@pytest.mark.parametrize("variant", ["mul", "shift"])
def test_merge_with_zero_adapter(monkeypatch, kernel, d, n, r, w_bits, out_bits, variant):
    """A = 0: the zero-initialised low-rank factor every fine-tune starts from
    ([notes] section 1, AQS), so A B = 0 and U = s + R* / D exactly. Through
    both kernel families."""
    monkeypatch.setenv("INTLORA_MERGE_KERNEL", kernel)
    spec = spec_for(d, n, r, w_bits, variant, out_bits if variant == "mul" else 4, sid=900 + d)
    inp = _oracle_prepared(spec)
    inp["A"] = np.zeros_like(inp["A"])
    got = gpu_merge([spec], [inp])[0]
    (_check_mul if variant == "mul" else _check_shift)(spec, inp, got)


@pytest.mark.parametrize("kernel", ["rows", "tc"])
@pytest.mark.parametrize("variant", ["mul", "shift"])
def test_merge_with_alpha_zero(monkeypatch, kernel, variant):
    """alpha = 0: the VMC factor is 1, R* = R ([notes] section 3). R* is then
    ~50x larger than W, and at a row extremum U = s + R*/D cancels to a
    small value: s_bar is checked against the bound the GPU's fast log2
    allows (codes under the usual rule)."""
    monkeypatch.setenv("INTLORA_MERGE_KERNEL", kernel)
    spec = spec_for(96, 4096, 16, 8, variant, 8 if variant == "mul" else 4, sid=77, alpha=0.0)
    inp = _oracle_prepared(spec)
    got = gpu_merge([spec], [inp])[0]
    (_check_mul if variant == "mul" else _check_shift)(spec, inp, got, lg2_bound=True)


@pytest.mark.parametrize("kernel", ["rows", "tc"])
def test_merge_clamps_out_of_range_zero_points(monkeypatch, kernel):
    """Zero-points outside [0, 2^w_bits - 1] are clamped into the code range on
    load (a device-side guard; a valid layer never has them): the merge equals
    the oracle's on the clamped zero-points."""
    monkeypatch.setenv("INTLORA_MERGE_KERNEL", kernel)
    spec = spec_for(64, 2048, 16, 8, "mul", 8, sid=78)
    inp = _oracle_prepared(spec)
    z_bad = inp["z"].copy()
    z_bad[::3] = -7
    z_bad[1::3] = 300
    got = gpu_merge([spec], [dict(inp, z=z_bad)])[0]
    _check_mul(spec, dict(inp, z=np.clip(z_bad, 0, 255)), got)


def test_merge_reduces_sigma_r_on_device_when_not_given():
    spec = spec_for(50, 256, 8, 8, "mul", 8, sid=3)
    inp = _oracle_prepared(spec)
    a = gpu_merge([spec], [inp], pass_sigma_r=True)[0]
    b = gpu_merge([spec], [inp], pass_sigma_r=False)[0]
    _check_mul(spec, inp, b)
    assert np.array_equal(a["sbar"], b["sbar"]) or np.max(np.abs(a["sbar"] / b["sbar"] - 1)) < 1e-6


def test_merge_batched_equals_single():
    specs = [spec_for(d, n, r, wb, "mul", ub, sid=k)
             for k, (d, n, r, wb, ub) in enumerate([(64, 768, 4, 4, 4), (30, 320, 4, 4, 4),
                                                     (130, 5120, 4, 4, 4)])]
    inps = [_oracle_prepared(s) for s in specs]
    a = gpu_merge(specs, inps, batched=True)
    b = gpu_merge(specs, inps, batched=False)
    for x, y in zip(a, b):
        assert np.array_equal(x["out"], y["out"]) and np.array_equal(x["sbar"], y["sbar"])


def test_merge_without_code_output():
    spec = spec_for(20, 128, 4, 8, "mul", 8, sid=2)
    inp = _oracle_prepared(spec)
    a = gpu_merge([spec], [inp], want_code=False)[0]
    b = gpu_merge([spec], [inp], want_code=True)[0]
    assert np.array_equal(a["out"], b["out"])


# ---------------------------------------------------------------------------
# a8: STE backward
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("d,n,r", [(320, 320, 4), (64, 768, 16), (100, 300, 128), (1, 5, 1),
                                   (257, 1030, 33)])
def test_ste_parity(d, n, r):
    spec = spec_for(d, n, r, 8, sid=d)
    Gb = wl.host_G_bits(spec)
    Ab = wl.to_bf16_bits(wl.host_A(spec))
    Bb = wl.to_bf16_bits(wl.host_B(spec))
    dA, dB = gpu_ste(Gb, Ab, Bb)
    G, A, Bm = (wl.bf16_bits_to_f32(x).astype(np.float64) for x in (Gb, Ab, Bb))
    oA, oB = oracle.ste_backward(G, A, Bm)
    assert rel_fro(dA, oA) < STE_RTOL
    assert rel_fro(dB, oB) < STE_RTOL


@pytest.mark.parametrize("d,n,r", [(100, 304, 128), (257, 1032, 33), (129, 136, 1), (1, 8, 4),
                                   (4096, 1024, 64), (130, 4104, 8),
                                   # ranks >= 64: two passes over L2-sized regions (up to
                                   # 16 row blocks x 16 column tiles), reduced into dA, dB
                                   (257, 1032, 96), (130, 4104, 64), (3, 8, 128),
                                   (2100, 2600, 128), (2200, 2056, 64)])
def test_ste_tensor_core_parity(d, n, r):
    """Shapes the tensor-core pass takes (n % 8 == 0, r <= 128): ragged row
    blocks and column tiles, padded ranks (1, 8, 33 -> 16, 16, 48)."""
    spec = spec_for(d, n, r, 8, sid=d + 1)
    Gb = wl.host_G_bits(spec)
    Ab = wl.to_bf16_bits(wl.host_A(spec))
    Bb = wl.to_bf16_bits(wl.host_B(spec))
    dA, dB = gpu_ste(Gb, Ab, Bb)
    G, A, Bm = (wl.bf16_bits_to_f32(x).astype(np.float64) for x in (Gb, Ab, Bb))
    oA, oB = oracle.ste_backward(G, A, Bm)
    assert rel_fro(dA, oA) < STE_RTOL
    assert rel_fro(dB, oB) < STE_RTOL


def test_ste_batched_mixed_ranks_both_kernels(monkeypatch):
    """One batched call over layers of different shapes and ranks, through the
    tensor-core pass and through the CUDA-core kernels: both match the oracle."""
    specs = [spec_for(d, n, r, 8, sid=40 + k) for k, (d, n, r) in
             enumerate([(320, 320, 4), (200, 768, 8), (64, 1280, 16), (384, 256, 2),
                        (96, 512, 64), (40, 136, 128)])]
    host = [(wl.host_G_bits(s), wl.to_bf16_bits(wl.host_A(s)), wl.to_bf16_bits(wl.host_B(s)))
            for s in specs]
    for kernel in ("auto", "cuda"):
        monkeypatch.setenv("INTLORA_STE_KERNEL", kernel)
        jobs = []
        for spec, (Gb, Ab, Bb) in zip(specs, host):
            t = [torch.from_numpy(x.view(np.int16)).to(dev()).view(torch.bfloat16) for x in (Gb, Ab, Bb)]
            jobs.append(B.SteJob(t[0], t[1], t[2],
                                 torch.full((spec.d, spec.r), np.nan, device=dev()),
                                 torch.full((spec.r, spec.n), np.nan, device=dev())))
        B.intlora_ste_backward_batched(jobs)
        torch.cuda.synchronize()
        for job, (Gb, Ab, Bb) in zip(jobs, host):
            G, A, Bm = (wl.bf16_bits_to_f32(x).astype(np.float64) for x in (Gb, Ab, Bb))
            oA, oB = oracle.ste_backward(G, A, Bm)
            assert rel_fro(job.dA.cpu().numpy(), oA) < STE_RTOL, kernel
            assert rel_fro(job.dB.cpu().numpy(), oB) < STE_RTOL, kernel


def test_batches_beyond_one_launch_table():
    """130 layers in one batched call of every stage: the library splits the
    call into chunks of 128 descriptors (and the tensor-core STE into launches
    of 64); every layer still matches its single-layer call and the oracle."""
    specs = [spec_for(8 + 4 * (k % 3), 64 + 16 * (k % 5), 4, 4, "mul", 4, sid=200 + k)
             for k in range(130)]
    Ws = [wl.host_W(s) for s in specs]
    g_b = gpu_gen_aux(specs, Ws, batched=True)
    for k in (0, 64, 127, 128, 129):
        o = oracle.gen_aux(Ws[k], specs[k].seed, specs[k].stream_id, specs[k].alpha, 4)
        assert_scale("sigma_r", g_b[k]["sigma_r"], o["sigma_r"])
        assert_affine("W_round", g_b[k]["codes"], g_b[k]["z"], o["codes"], o["z"], o["pre"],
                      o["zpre"], 15)
    inps = [_oracle_prepared(s) for s in specs]
    a = gpu_merge(specs, inps, batched=True)
    for k in (0, 127, 128, 129):
        b = gpu_merge([specs[k]], [inps[k]], batched=False)[0]
        assert np.array_equal(a[k]["out"], b["out"]) and np.array_equal(a[k]["zbar"], b["zbar"])
    jobs, host = [], []
    for spec in specs:
        Gb, Ab, Bb = (wl.host_G_bits(spec), wl.to_bf16_bits(wl.host_A(spec)),
                      wl.to_bf16_bits(wl.host_B(spec)))
        t = [torch.from_numpy(x.view(np.int16)).to(dev()).view(torch.bfloat16) for x in (Gb, Ab, Bb)]
        jobs.append(B.SteJob(t[0], t[1], t[2], torch.full((spec.d, spec.r), np.nan, device=dev()),
                             torch.full((spec.r, spec.n), np.nan, device=dev())))
        host.append((Gb, Ab, Bb))
    B.intlora_ste_backward_batched(jobs)
    torch.cuda.synchronize()
    for k in (0, 63, 64, 127, 128, 129):
        G, A, Bm = (wl.bf16_bits_to_f32(x).astype(np.float64) for x in host[k])
        oA, oB = oracle.ste_backward(G, A, Bm)
        assert rel_fro(jobs[k].dA.cpu().numpy(), oA) < STE_RTOL
        assert rel_fro(jobs[k].dB.cpu().numpy(), oB) < STE_RTOL


def test_no_device_wait_gave_up():
    """Every bounded wait of the tensor-core kernels finished in time."""
    assert B.intlora_device_status() == 0


def test_batches_with_mixed_seeds():
    """Layers with different Philox keys in one batched call (the library
    launches one group per key) match the oracle and single-layer calls."""
    specs = [spec_for(48, 320, 4, 4, "mul", 4, sid=k, seed=seed)
             for k, seed in enumerate([1, 7, 2**40 + 3])]
    Ws = [wl.host_W(s) for s in specs]
    g_b = gpu_gen_aux(specs, Ws, batched=True)
    g_s = gpu_gen_aux(specs, Ws, batched=False)
    for spec, W, x, y in zip(specs, Ws, g_b, g_s):
        assert np.array_equal(x["codes"], y["codes"]) and x["sigma_r"] == y["sigma_r"]
        o = oracle.gen_aux(W, spec.seed, spec.stream_id, spec.alpha, spec.w_bits)
        assert_scale("sigma_r", x["sigma_r"], o["sigma_r"])
        assert_affine("W_round", x["codes"], x["z"], o["codes"], o["z"], o["pre"], o["zpre"], 15)
    inps = [_oracle_prepared(s) for s in specs]
    a = gpu_merge(specs, inps, batched=True)
    b = gpu_merge(specs, inps, batched=False)
    for spec, inp, x, y in zip(specs, inps, a, b):
        assert np.array_equal(x["out"], y["out"])
        _check_mul(spec, inp, x)


# ---------------------------------------------------------------------------
# auxiliary laws of the ablation (Gaussian, Cauchy, Student-t 2 dof): the
# statistics pass and the row-tile kernels' general-law path
# ---------------------------------------------------------------------------
LAWS = [1, 2, 3]


@pytest.mark.parametrize("dist", LAWS)
@pytest.mark.parametrize("d,n,w_bits", [(64, 768, 4), (33, 100, 8), (7, 10, 4), (5, 6, 8)])
def test_gen_aux_parity_other_laws(dist, d, n, w_bits):
    spec = replace(spec_for(d, n, 4, w_bits, sid=d + n + dist), distribution=dist)
    W = wl.host_W(spec)
    g = gpu_gen_aux([spec], [W], want_r_star=True)[0]
    o = oracle.gen_aux(W, spec.seed, spec.stream_id, spec.alpha, w_bits, want_r_star=True, dist=dist)
    assert_scale("sigma_w", g["sigma_w"], o["sigma_w"])
    assert_scale("sigma_r", g["sigma_r"], o["sigma_r"])
    assert_scale("s", g["s"], o["s"])
    assert_affine("W_round", g["codes"], g["z"], o["codes"], o["z"], o["pre"], o["zpre"],
                  2**w_bits - 1)
    err = np.abs(g["r_star"].astype(np.float64) - o["r_star"])
    assert np.max(err / np.maximum(np.abs(o["r_star"]), 1e-3 * o["c"])) < 2e-6


@pytest.mark.parametrize("dist", LAWS)
@pytest.mark.parametrize("d,n,r,w_bits,bits", [(40, 264, 4, 4, 4), (9, 50, 3, 8, 8), (17, 1024, 16, 8, 8)])
def test_merge_mul_parity_other_laws(dist, d, n, r, w_bits, bits):
    spec = replace(spec_for(d, n, r, w_bits, "mul", bits, sid=3 + d + dist), distribution=dist)
    inp = _oracle_prepared(spec)
    _check_mul(spec, inp, gpu_merge([spec], [inp])[0])


@pytest.mark.parametrize("dist", LAWS)
@pytest.mark.parametrize("d,n,r,w_bits,bits", [(24, 320, 8, 4, 4), (5, 6, 2, 4, 2)])
def test_merge_shift_parity_other_laws(dist, d, n, r, w_bits, bits):
    spec = replace(spec_for(d, n, r, w_bits, "shift", bits, sid=5 + d + dist), distribution=dist)
    inp = _oracle_prepared(spec)
    _check_shift(spec, inp, gpu_merge([spec], [inp])[0])


def test_mixed_laws_in_one_batch():
    """A batch mixing laws is split by law on the host: each layer equals its
    own single-layer result, and sigma_R reduced on the device follows the law."""
    specs = [replace(spec_for(20, 128, 4, 4, "mul", 4, sid=60 + k), distribution=k % 4)
             for k in range(6)]
    inps = [_oracle_prepared(s) for s in specs]
    a = gpu_merge(specs, inps, batched=True, pass_sigma_r=False)
    for k, spec in enumerate(specs):
        b = gpu_merge([spec], [inps[k]], batched=False, pass_sigma_r=False)[0]
        for key in ("out", "sbar", "zbar", "code"):
            assert np.array_equal(a[k][key], b[key]), (spec.distribution, key)
        _check_mul(spec, inps[k], a[k])


# ---------------------------------------------------------------------------
# masked STE: G restricted to D = W_round - z != 0
# ---------------------------------------------------------------------------
def _masked_inputs(spec, w_bits):
    Gb = wl.host_G_bits(spec)
    Ab = wl.to_bf16_bits(wl.host_A(spec))
    Bb = wl.to_bf16_bits(wl.host_B(spec))
    rng = np.random.default_rng([12, spec.stream_id])
    qmax = 2**w_bits - 1
    z = rng.integers(0, qmax + 1, spec.d).astype(np.int32)
    # codes near z so that a sizeable share of D is 0 (1 in 3)
    codes = np.clip(z[:, None] + rng.integers(-1, 2, (spec.d, spec.n)), 0, qmax).astype(np.int32)
    return Gb, Ab, Bb, codes, z


def _gpu_ste_masked(jobs_host, w_bits, with_ws=True):
    jobs = []
    for Gb, Ab, Bb, codes, z in jobs_host:
        d, n = Gb.shape
        r = Ab.shape[1]
        t = [torch.from_numpy(x.view(np.int16)).to(dev()).view(torch.bfloat16) for x in (Gb, Ab, Bb)]
        jobs.append(B.SteJob(t[0], t[1], t[2],
                             torch.full((d, r), np.nan, dtype=torch.float32, device=dev()),
                             torch.full((r, n), np.nan, dtype=torch.float32, device=dev()),
                             torch.from_numpy(wl.pack_codes(codes, w_bits)).to(dev()), w_bits,
                             torch.from_numpy(z).to(dev())))
    # with the workspace: a masked copy of G on the plain (tensor-core) path;
    # without: the CUDA-core kernels mask G as they read it
    ws = P.workspace(B.intlora_ste_workspace_size(jobs), dev()) if with_ws else None
    B.intlora_ste_backward_batched(jobs, ws)
    torch.cuda.synchronize()
    return [(j.dA.cpu().numpy(), j.dB.cpu().numpy()) for j in jobs]


@pytest.mark.parametrize("d,n,r,w_bits", [(320, 320, 4, 4), (200, 768, 8, 8), (64, 1280, 16, 4),
                                          (33, 50, 3, 8), (9, 1032, 33, 4), (1, 8, 1, 8)])
@pytest.mark.parametrize("with_ws", [True, False])
def test_ste_masked_parity(d, n, r, w_bits, with_ws):
    spec = spec_for(d, n, r, w_bits, sid=70 + d)
    h = _masked_inputs(spec, w_bits)
    (dA, dB), = _gpu_ste_masked([h], w_bits, with_ws)
    Gb, Ab, Bb, codes, z = h
    G, A, Bm = (wl.bf16_bits_to_f32(x).astype(np.float64) for x in (Gb, Ab, Bb))
    oA, oB = oracle.ste_backward_masked(G, A, Bm, codes, z)
    assert rel_fro(dA, oA) < STE_RTOL
    assert rel_fro(dB, oB) < STE_RTOL
    if d * n >= 1000:      # the mask matters: the plain STE is far outside the tolerance
        pA, _ = oracle.ste_backward(G, A, Bm)
        assert rel_fro(pA, oA) > 10 * STE_RTOL


def test_ste_masked_and_plain_jobs_in_one_call():
    specs = [spec_for(128, 512, 4, 4, sid=90), spec_for(96, 256, 8, 4, sid=91)]
    hs = [_masked_inputs(s, 4) for s in specs]
    (mA, mB), = _gpu_ste_masked([hs[0]], 4)
    Gb, Ab, Bb, _, _ = hs[1]
    pA, pB = gpu_ste(Gb, Ab, Bb)
    # the same two jobs in one batched call, one masked and one plain
    t0 = [torch.from_numpy(x.view(np.int16)).to(dev()).view(torch.bfloat16) for x in hs[0][:3]]
    t1 = [torch.from_numpy(x.view(np.int16)).to(dev()).view(torch.bfloat16) for x in hs[1][:3]]
    j0 = B.SteJob(t0[0], t0[1], t0[2], torch.empty((128, 4), device=dev()),
                  torch.empty((4, 512), device=dev()),
                  torch.from_numpy(wl.pack_codes(hs[0][3], 4)).to(dev()), 4,
                  torch.from_numpy(hs[0][4]).to(dev()))
    j1 = B.SteJob(t1[0], t1[1], t1[2], torch.empty((96, 8), device=dev()),
                  torch.empty((8, 256), device=dev()))
    B.intlora_ste_backward_batched([j0, j1])
    torch.cuda.synchronize()
    assert rel_fro(j0.dA.cpu().numpy(), mA) < 1e-6 and rel_fro(j0.dB.cpu().numpy(), mB) < 1e-6
    assert rel_fro(j1.dA.cpu().numpy(), pA) < 1e-6 and rel_fro(j1.dB.cpu().numpy(), pB) < 1e-6
