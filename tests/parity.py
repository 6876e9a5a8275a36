"""Helpers for the GPU-vs-oracle parity tests: run one stage of the CUDA path
on host inputs and compare with the oracle under the acceptance rule.

Acceptance (integer codes decided by floating point): at least 99.99% of the
codes are bit-exact; every other code is off by exactly one, and only where
the oracle's fp64 pre-round value lies within 1e-5 * max(|x|, 1) of a rounding
boundary (the GPU decides in fp32, the oracle in fp64). Scales within 1e-6
relative; STE gradients within 1e-3 relative Frobenius (bf16 inputs, fp32
accumulation).
"""
from __future__ import annotations

import numpy as np
import torch

from quantized_lora_merge_b200 import binding as B
from quantized_lora_merge_b200 import pipeline as P
from quantized_lora_merge_b200 import workloads as wl

WINDOW = 1e-5
MIN_EXACT = 0.9999
SCALE_RTOL = 1e-6
STE_RTOL = 1e-3


def dev():
    return torch.device("cuda", 0)


# ---------------------------------------------------------------------------
# comparisons
# ---------------------------------------------------------------------------
def _near_half(x: np.ndarray) -> np.ndarray:
    frac = x - np.floor(x)
    return np.abs(frac - 0.5) <= WINDOW * np.maximum(np.abs(x), 1.0)


def _allowed_mismatches(n: int) -> int:
    """Codes that may differ among n: at most 0.01 % (exactly, in integers),
    so none at all below 10,000 codes."""
    return n // 10000


def assert_scale(name, gpu, ora):
    gpu = np.asarray(gpu, np.float64)
    ora = np.asarray(ora, np.float64)
    rel = np.abs(gpu - ora) / np.maximum(np.abs(ora), 1e-300)
    assert rel.max(initial=0.0) <= SCALE_RTOL, f"{name}: max rel err {rel.max():.3e}"


def assert_affine(name, g_codes, g_zero, o_codes, o_zero, pre, zpre, qmax):
    """Codes of the per-row affine quantizer (W_round or U_round) and their
    zero-points. Rows whose zero-point the two sides decided differently (only
    allowed within the window) are compared on centred codes, clamps aside."""
    g_codes = np.asarray(g_codes, np.int64)
    o_codes = np.asarray(o_codes, np.int64)
    g_zero = np.asarray(g_zero, np.int64)
    o_zero = np.asarray(o_zero, np.int64)
    zmis = g_zero != o_zero
    if zmis.any():
        assert np.all(np.abs(g_zero - o_zero)[zmis] == 1), f"{name}: zero-point off by >1"
        assert np.all(_near_half(np.asarray(zpre)[zmis])), f"{name}: zero-point mismatch off-boundary"
    gc = g_codes - g_zero[:, None]
    oc = o_codes - o_zero[:, None]
    mism = gc != oc
    clamped = (g_codes == 0) | (g_codes == qmax) | (o_codes == 0) | (o_codes == qmax)
    excused = zmis[:, None] & clamped
    hard = mism & ~excused
    n_bad = int(hard.sum())
    assert n_bad <= _allowed_mismatches(gc.size), \
        f"{name}: {n_bad} of {gc.size} codes differ (> {100 * (1 - MIN_EXACT):.2f}%)"
    if n_bad:
        assert np.all(np.abs(gc - oc)[hard] == 1), f"{name}: a code differs by more than one"
        x = np.asarray(pre)[hard]
        assert np.all(_near_half(x)), \
            f"{name}: mismatch away from a rounding boundary at pre-round {x[~_near_half(x)][:5]}"
    return n_bad


def assert_shift(name, g_shift, o_shift, pre, kmax):
    g = np.asarray(g_shift, np.int64)
    o = np.asarray(o_shift, np.int64)
    mism = g != o
    # a clamped oracle shift (t beyond kmax + 1/2) has no boundary to be near
    n_bad = int(mism.sum())
    assert n_bad <= _allowed_mismatches(g.size), f"{name}: {n_bad} shift codes differ"
    if n_bad:
        assert np.all(np.abs(g - o)[mism] == 1), f"{name}: a shift differs by more than one"
        x = np.asarray(pre)[mism]
        assert np.all(_near_half(x)), f"{name}: shift mismatch away from a boundary: {x[:5]}"
    return n_bad


def rel_fro(a, b) -> float:
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


# ---------------------------------------------------------------------------
# GPU stage runners (host numpy in, host numpy out)
# ---------------------------------------------------------------------------
def spec_for(d, n, r, w_bits, variant="mul", out_bits=8, sid=0, alpha=wl.ALPHA, seed=wl.AUX_SEED):
    return wl.LayerSpec(f"t{d}x{n}r{r}", d, n, r, w_bits, variant, out_bits, alpha=alpha,
                        seed=seed, stream_id=sid)


def gpu_gen_aux(specs, Ws, want_r_star=False, batched=True):
    """Run layer preparation; returns per layer a dict of numpy outputs."""
    states, jobs = [], []
    for spec, W in zip(specs, Ws):
        Wd = torch.from_numpy(np.ascontiguousarray(W, np.float32)).to(dev())
        st = P.allocate(spec, Wd, None, None, dev())
        job = st.aux_job()
        if want_r_star:
            job.r_star = torch.empty(spec.d, spec.n, dtype=torch.float32, device=dev())
        states.append(st)
        jobs.append(job)
    if batched:
        ws = P.workspace(B.intlora_gen_aux_workspace_size(jobs), dev())
        B.intlora_gen_aux_batched(jobs, ws)
    else:
        for job in jobs:
            ws = P.workspace(B.intlora_gen_aux_workspace_size([job]), dev())
            B.intlora_gen_aux(job, ws)
    torch.cuda.synchronize()
    res = []
    for spec, st, job in zip(specs, states, jobs):
        sig = st.sigma.cpu().numpy()
        res.append(dict(sigma_w=float(sig[0]), sigma_r=float(sig[1]),
                        codes=wl.unpack_codes(st.w_round.cpu().numpy(), spec.n, spec.w_bits),
                        s=st.s.cpu().numpy(), z=st.z.cpu().numpy(),
                        r_star=job.r_star.cpu().numpy() if want_r_star else None))
    return res


def gpu_merge(specs, inputs, pass_sigma_r=True, batched=True, want_code=True):
    """inputs: per layer dict(codes, s (fp32), z, A, B, sigma_w, sigma_r)."""
    states = []
    for spec, inp in zip(specs, inputs):
        A = torch.from_numpy(np.ascontiguousarray(inp["A"], np.float32)).to(dev())
        Bm = torch.from_numpy(np.ascontiguousarray(inp["B"], np.float32)).to(dev())
        st = P.allocate(spec, None, A, Bm, dev(), want_code=want_code)
        st.w_round.copy_(torch.from_numpy(wl.pack_codes(inp["codes"], spec.w_bits)))
        st.s.copy_(torch.from_numpy(np.asarray(inp["s"], np.float32)))
        st.z.copy_(torch.from_numpy(np.asarray(inp["z"], np.int32)))
        st.sigma.copy_(torch.tensor([inp["sigma_w"], inp["sigma_r"]], dtype=torch.float64))
        states.append(st)
    layers = [st.layer(pass_sigma_r) for st in states]
    outs = [st.merge_out() for st in states]
    variant = specs[0].variant
    bits = specs[0].out_bits
    if batched:
        ws = P.workspace(B.intlora_merge_workspace_size(layers), dev())
        if variant == "mul":
            B.intlora_merge_mul_batched(layers, outs, bits, ws)
        else:
            B.intlora_merge_shift_batched(layers, outs, bits, ws)
    else:
        for layer, out in zip(layers, outs):
            ws = P.workspace(B.intlora_merge_workspace_size([layer]), dev())
            if variant == "mul":
                B.intlora_merge_mul(layer, bits, out, ws)
            else:
                B.intlora_merge_shift(layer, bits, out, ws)
    torch.cuda.synchronize()
    res = []
    for st in states:
        res.append(dict(out=st.out.cpu().numpy().astype(np.int64), sbar=st.sbar.cpu().numpy(),
                        zbar=st.zbar.cpu().numpy(),
                        code=st.code.cpu().numpy() if st.code is not None else None))
    return res


def gpu_ste(Gbits, Abits, Bbits):
    d, n = Gbits.shape
    r = Abits.shape[1]

    def to_bf16(bits):
        return torch.from_numpy(bits.view(np.int16)).to(dev()).view(torch.bfloat16)

    job = B.SteJob(to_bf16(Gbits), to_bf16(Abits), to_bf16(Bbits),
                   torch.full((d, r), np.nan, dtype=torch.float32, device=dev()),
                   torch.full((r, n), np.nan, dtype=torch.float32, device=dev()))
    B.intlora_ste_backward(job)
    torch.cuda.synchronize()
    return job.dA.cpu().numpy(), job.dB.cpu().numpy()
