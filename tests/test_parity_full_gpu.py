"""Full-size parity: the configs' real layer shapes, run through the batched
calls exactly as bench.py launches them, checked against the oracle on
sampled rows (and, for the STE, sampled rows of dA and columns of dB), which
the oracle computes one by one. Each stage gets inputs independent of the
CUDA path: preparation gets the seeded W; the merge gets seeded synthetic
prepared layers (codes, scales, zero-points, sigmas); the STE gets seeded G."""
import numpy as np
import pytest
import torch

import oracle
from quantized_lora_merge_b200 import binding as B
from quantized_lora_merge_b200 import pipeline as P
from quantized_lora_merge_b200 import workloads as wl

from .parity import STE_RTOL, assert_affine, assert_scale, assert_shift, rel_fro

pytestmark = pytest.mark.gpu


def _dev():
    return torch.device("cuda", 0)


def _sample_rows(spec, count=6):
    """First and last rows (the last tile is ragged) plus seeded interior rows."""
    rng = np.random.default_rng([9, spec.stream_id])
    rows = {0, spec.d - 1}
    rows.update(int(x) for x in rng.integers(0, spec.d, size=count - 2))
    return sorted(rows)


def _synthetic_prepared(spec):
    """A prepared layer drawn directly (not from any implementation): codes
    uniform over the code range, positive per-row scales, zero-points inside
    the range, and fixed sigmas."""
    rng = np.random.default_rng([7, spec.stream_id])
    qmax = 2**spec.w_bits - 1
    codes = rng.integers(0, qmax + 1, size=(spec.d, spec.n), dtype=np.int64).astype(np.int32)
    s = (rng.uniform(0.5, 1.5, spec.d) * 0.08 / qmax).astype(np.float32)
    z = rng.integers(qmax // 4, 3 * qmax // 4 + 1, size=spec.d).astype(np.int32)
    return dict(codes=codes, s=s, z=z, A=wl.host_A(spec), B=wl.host_B(spec), sigma_w=0.02,
                sigma_r=1.4142)


def _check_prepare(specs):
    dev = _dev()
    states = []
    for spec in specs:
        W = torch.from_numpy(wl.host_W(spec)).to(dev)
        states.append(P.allocate(spec, W, None, None, dev))
    jobs = [st.aux_job() for st in states]
    ws = P.workspace(B.intlora_gen_aux_workspace_size(jobs), dev)
    B.intlora_gen_aux_batched(jobs, ws)
    torch.cuda.synchronize()
    return states


def _verify_prepare(spec, st):
    Wh = wl.host_W(spec)
    rows = _sample_rows(spec)
    sig = st.sigma.cpu().numpy()
    codes = wl.unpack_codes(st.w_round.cpu().numpy(), spec.n, spec.w_bits)
    s = st.s.cpu().numpy()
    z = st.z.cpu().numpy()
    first = True
    for i in rows:
        o = oracle.gen_aux(Wh, spec.seed, spec.stream_id, spec.alpha, spec.w_bits, row_begin=i,
                           row_count=1)
        if first:
            assert_scale("sigma_w", sig[0], o["sigma_w"])
            assert_scale("sigma_r", sig[1], o["sigma_r"])
            first = False
        assert_scale("s", s[i:i + 1], o["s"])
        assert_affine(f"W_round row {i}", codes[i:i + 1], z[i:i + 1], o["codes"], o["z"], o["pre"],
                      o["zpre"], 2**spec.w_bits - 1)


def _run_merge(specs):
    dev = _dev()
    states, inps = [], []
    for spec in specs:
        inp = _synthetic_prepared(spec)
        A = torch.from_numpy(inp["A"]).to(dev)
        Bm = torch.from_numpy(inp["B"]).to(dev)
        st = P.allocate(spec, None, A, Bm, dev, want_code=True)
        st.w_round.copy_(torch.from_numpy(wl.pack_codes(inp["codes"], spec.w_bits)))
        st.s.copy_(torch.from_numpy(inp["s"]))
        st.z.copy_(torch.from_numpy(inp["z"]))
        st.sigma.copy_(torch.tensor([inp["sigma_w"], inp["sigma_r"]], dtype=torch.float64))
        states.append(st)
        inps.append(inp)
    variant, bits = specs[0].variant, specs[0].out_bits
    layers = [st.layer() for st in states]
    outs = [st.merge_out() for st in states]
    ws = P.workspace(B.intlora_merge_workspace_size(layers), dev)   # tensor-core A B at r >= 32
    if variant == "mul":
        B.intlora_merge_mul_batched(layers, outs, bits, ws)
    else:
        B.intlora_merge_shift_batched(layers, outs, bits, ws)
    torch.cuda.synchronize()
    return states, inps


def _verify_merge(spec, st, inp):
    rows = _sample_rows(spec)
    out = st.out.cpu().numpy().astype(np.int64)
    code = st.code.cpu().numpy()
    sbar = st.sbar.cpu().numpy()
    zbar = st.zbar.cpu().numpy()
    for i in rows:
        args = (inp["codes"], inp["s"], inp["z"], inp["A"], inp["B"], spec.seed, spec.stream_id,
                inp["sigma_w"], inp["sigma_r"], spec.alpha, spec.out_bits)
        D = inp["codes"][i].astype(np.int64) - inp["z"][i]
        if spec.variant == "mul":
            o = oracle.merge_mul(*args, row_begin=i, row_count=1)
            assert_scale("s_bar", sbar[i:i + 1], o["sbar"])
            assert_affine(f"U_round row {i}", code[i:i + 1], zbar[i:i + 1], o["u_round"], o["zbar"],
                          o["pre"], o["zpre"], 2**spec.out_bits - 1)
            assert np.array_equal(out[i], (code[i].astype(np.int64) - zbar[i]) * D)
        else:
            o = oracle.merge_shift(*args, row_begin=i, row_count=1)
            assert_scale("s_bar", sbar[i:i + 1], o["sbar"])
            assert_shift(f"shift row {i}", code[i:i + 1], o["shift"], o["pre"], 2**spec.out_bits - 1)
            sign = np.sign(o["U"][0]).astype(np.int64)
            assert np.array_equal(out[i], sign * (D >> code[i].astype(np.int64)))


def _run_and_verify_ste(specs):
    dev = _dev()
    jobs, host = [], []
    for spec in specs:
        Gb = wl.host_G_bits(spec)
        Ab = wl.to_bf16_bits(wl.host_A(spec))
        Bb = wl.to_bf16_bits(wl.host_B(spec))
        t = [torch.from_numpy(x.view(np.int16)).to(dev).view(torch.bfloat16) for x in (Gb, Ab, Bb)]
        jobs.append(B.SteJob(t[0], t[1], t[2],
                             torch.empty(spec.d, spec.r, dtype=torch.float32, device=dev),
                             torch.empty(spec.r, spec.n, dtype=torch.float32, device=dev)))
        host.append((Gb, Ab, Bb))
    B.intlora_ste_backward_batched(jobs)
    torch.cuda.synchronize()
    for spec, job, (Gb, Ab, Bb) in zip(specs, jobs, host):
        rows = np.array(_sample_rows(spec))
        cols = np.array(sorted({0, spec.n - 1} | set(int(x) for x in np.random.default_rng(
            [8, spec.stream_id]).integers(0, spec.n, size=6))))
        oA, oB = oracle.ste_sampled(Gb, Ab, Bb, rows, cols)
        assert rel_fro(job.dA.cpu().numpy()[rows], oA) < STE_RTOL
        assert rel_fro(job.dB.cpu().numpy()[:, cols], oB) < STE_RTOL


# ---------------------------------------------------------------------------
def test_sd_unet_full_batch():
    """All 128 SD-UNet layers in one batched call per stage (the bench step)."""
    specs = wl.sd_unet()
    states = _check_prepare(specs)
    picks = [0, 4, 6, 7, 64, 118, 126, 127]   # every width and linear kind
    for k in picks:
        _verify_prepare(specs[k], states[k])
    del states
    mstates, inps = _run_merge(specs)
    for k in picks:
        _verify_merge(specs[k], mstates[k], inps[k])
    del mstates, inps
    _run_and_verify_ste([specs[k] for k in picks])


def test_llama_shapes_full_size():
    specs = wl.distinct_shapes(wl.llama3_8b(n_layers=1))
    states = _check_prepare(specs)
    for spec, st in zip(specs, states):
        _verify_prepare(spec, st)
    del states
    mstates, inps = _run_merge(specs)
    for spec, st, inp in zip(specs, mstates, inps):
        _verify_merge(spec, st, inp)


def test_dit_shapes_full_size_shift():
    specs = wl.distinct_shapes(wl.dit_3072(n_blocks=1))
    mstates, inps = _run_merge(specs)
    for spec, st, inp in zip(specs, mstates, inps):
        _verify_merge(spec, st, inp)


@pytest.mark.parametrize("r", [4, 16, 128])
def test_rank_sweep_full_size(r):
    specs = [s for s in wl.rank_sweep() if s.r == r]
    mstates, inps = _run_merge(specs)
    for spec, st, inp in zip(specs, mstates, inps):
        _verify_merge(spec, st, inp)
    del mstates, inps
    _run_and_verify_ste(specs)
