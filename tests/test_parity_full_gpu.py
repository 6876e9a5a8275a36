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


# ---------------------------------------------------------------------------
# maximum size: a layer past 2^34 elements, where the Philox block index
# e / 4 needs the counter's high word (rows from 2^20 on, at n = 16384)
# ---------------------------------------------------------------------------
HUGE_D, HUGE_N = 2**20 + 1, 16384           # 2^34 + 16384 elements


def _huge_rows():
    return [0, 12345, 2**19, 2**20 - 1, 2**20]   # the last row lies wholly past 2^34


def test_layer_beyond_2_34_elements():
    dev = _dev()
    if torch.cuda.mem_get_info(dev)[0] < 90 * 2**30:
        pytest.skip("needs ~80 GB of free device memory")
    d, n = HUGE_D, HUGE_N
    assert d * n > 2**34
    # preparation with alpha = 0 (c = 1, no sigma needed on the host): W is a
    # seeded device draw; the sampled rows go to the oracle
    spec = wl.LayerSpec("huge", d, n, 4, 4, "mul", 4, alpha=0.0, stream_id=77)
    g = torch.Generator(device=dev)
    g.manual_seed(2026)
    W = torch.randn(d, n, generator=g, device=dev).mul_(wl.W_STD)
    sigma = torch.zeros(2, dtype=torch.float64, device=dev)
    w_round = torch.zeros(d, P.code_row_bytes(n, 4), dtype=torch.uint8, device=dev)
    s_d = torch.zeros(d, dtype=torch.float32, device=dev)
    z_d = torch.zeros(d, dtype=torch.int32, device=dev)
    job = B.AuxJob(W, spec.seed, spec.stream_id, spec.alpha, 4, sigma[0:1], sigma[1:2], None,
                   w_round, s_d, z_d)
    ws = P.workspace(B.intlora_gen_aux_workspace_size([job]), dev)
    B.intlora_gen_aux_batched([job], ws)
    torch.cuda.synchronize()
    rows = _huge_rows()
    idx = torch.tensor(rows, device=dev)
    W_rows = W[idx].cpu().numpy()
    codes = wl.unpack_codes(w_round[idx].cpu().numpy(), n, 4)
    s, z = s_d[idx].cpu().numpy(), z_d[idx].cpu().numpy()
    sig = sigma.cpu().numpy()
    assert np.all(np.isfinite(sig)) and np.all(sig > 0)
    del W, w_round, s_d, z_d, job, ws
    torch.cuda.empty_cache()
    for k, i in enumerate(rows):
        o = oracle.quantize_rows(W_rows[k:k + 1], spec.seed, spec.stream_id, 1.0, 4, i)
        assert_scale("s", s[k:k + 1], o["s"])
        assert_affine(f"W_round row {i}", codes[k:k + 1], z[k:k + 1], o["codes"], o["z"], o["pre"],
                      o["zpre"], 15)

    # MUL merge with alpha = 1.5 on a seeded synthetic prepared layer
    mspec = wl.LayerSpec("huge", d, n, 4, 4, "mul", 4, alpha=1.5, stream_id=78)
    A = torch.randn(d, 4, generator=g, device=dev).mul_(wl.AB_STD)
    Bm = torch.randn(4, n, generator=g, device=dev).mul_(wl.AB_STD)
    st = P.allocate(mspec, None, A, Bm, dev, want_code=True)
    st.w_round.copy_(torch.randint(0, 256, st.w_round.shape, generator=g, device=dev,
                                   dtype=torch.uint8))
    st.s.copy_(torch.empty(d, device=dev).uniform_(0.5, 1.5, generator=g) * (0.08 / 15))
    st.z.copy_(torch.randint(4, 12, (d,), generator=g, device=dev, dtype=torch.int32))
    sw, sr = 0.02, 1.4142
    st.sigma.copy_(torch.tensor([sw, sr], dtype=torch.float64))
    layers, outs = [st.layer()], [st.merge_out()]
    mws = P.workspace(B.intlora_merge_workspace_size(layers), dev)
    B.intlora_merge_mul_batched(layers, outs, 4, mws)
    torch.cuda.synchronize()
    c = oracle.vmc_scale(sw, sr, 1.5)
    in_codes = wl.unpack_codes(st.w_round[idx].cpu().numpy(), n, 4)
    in_s, in_z = st.s[idx].cpu().numpy(), st.z[idx].cpu().numpy()
    A_rows, B_h = A[idx].cpu().numpy(), Bm.cpu().numpy()
    out = st.out[idx].cpu().numpy().astype(np.int64)
    code = st.code[idx].cpu().numpy()
    sbar, zbar = st.sbar[idx].cpu().numpy(), st.zbar[idx].cpu().numpy()
    del st, mws, A, Bm
    torch.cuda.empty_cache()
    for k, i in enumerate(rows):
        o = oracle.merge_mul_rows(in_codes[k:k + 1], in_s[k:k + 1], in_z[k:k + 1], A_rows[k:k + 1],
                                  B_h, mspec.seed, mspec.stream_id, c, 4, i)
        assert_scale("s_bar", sbar[k:k + 1], o["sbar"])
        assert_affine(f"U_round row {i}", code[k:k + 1], zbar[k:k + 1], o["u_round"], o["zbar"],
                      o["pre"], o["zpre"], 15)
        D = in_codes[k].astype(np.int64) - in_z[k]
        assert np.array_equal(out[k], (code[k].astype(np.int64) - zbar[k]) * D)
