"""intlora_gen_aux_noalloc: layer preparation for callers that cannot allocate
device memory (their memory manager owns every allocation, or cudaMalloc is not
allowed where they run). The library takes the sigma scratch from a fixed array
of its own instead of a caller workspace. Checked here through the C ABI
against intlora_gen_aux with a caller workspace and against the oracle, on
calls in a row (each reuses the array the previous one left behind), up to
the largest layer it accepts; one row more is refused.

This file is collected last on purpose, so a stop-at-first-failure run has
already run every other test when it gets here."""
import numpy as np
import pytest
import torch

import oracle
from quantized_lora_merge_b200 import binding as B
from quantized_lora_merge_b200 import pipeline as P
from quantized_lora_merge_b200 import workloads as wl

from .parity import assert_affine, assert_scale, spec_for

MAX_ELEMENTS = 4194304   # INTLORA_NOALLOC_MAX_ELEMENTS


def _prepare(spec, W, use_noalloc):
    dev = torch.device("cuda", 0)
    Wd = torch.from_numpy(np.ascontiguousarray(W, np.float32)).to(dev)
    st = P.allocate(spec, Wd, None, None, dev)
    job = st.aux_job()
    if use_noalloc:
        B.intlora_gen_aux_noalloc(job)
    else:
        ws = P.workspace(B.intlora_gen_aux_workspace_size([job]), dev)
        B.intlora_gen_aux(job, ws)
    torch.cuda.synchronize()
    return dict(sigma=st.sigma.cpu().numpy(), w_round=st.w_round.cpu().numpy(),
                s=st.s.cpu().numpy(), z=st.z.cpu().numpy())


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point_on_two_calls():
    torch.cuda.set_device(0)
    # layers back to back: each call reuses the array the previous call left
    # behind, and must not depend on its contents; the last layer has exactly
    # the largest size the entry point accepts
    for spec in (spec_for(320, 320, 4, 8, sid=41), spec_for(1280, 768, 4, 4, sid=42),
                 spec_for(2048, MAX_ELEMENTS // 2048, 4, 8, sid=43)):
        W = wl.host_W(spec)
        ref = _prepare(spec, W, use_noalloc=False)
        got = _prepare(spec, W, use_noalloc=True)
        assert_scale("sigma_w", got["sigma"][0], ref["sigma"][0])
        assert_scale("sigma_r", got["sigma"][1], ref["sigma"][1])
        assert_scale("s", got["s"], ref["s"])
        assert np.array_equal(got["z"], ref["z"])
        assert np.array_equal(got["w_round"], ref["w_round"])
        # and against the oracle, under the same acceptance rule as the rest
        o = oracle.gen_aux(W, spec.seed, spec.stream_id, spec.alpha, spec.w_bits)
        assert_scale("sigma_w", got["sigma"][0], o["sigma_w"])
        assert_scale("sigma_r", got["sigma"][1], o["sigma_r"])
        assert_scale("s", got["s"], o["s"])
        assert_affine("W_round", wl.unpack_codes(got["w_round"], spec.n, spec.w_bits), got["z"],
                      o["codes"], o["z"], o["pre"], o["zpre"], 2**spec.w_bits - 1)


def test_noalloc_rejects_layers_beyond_its_limit():
    """Host-side check: a layer above the stated maximum is refused with a
    clear message before anything is launched (no GPU needed)."""
    lib = B.lib()
    fake = 0x100000
    for d, n in ((2048, 4096), (2049, 2048)):     # twice the limit; one row over it
        assert d * n > MAX_ELEMENTS
        st = lib.intlora_gen_aux_noalloc(fake, d, n, 1, 0, 1.5, 8, fake, fake, None, fake, n,
                                         fake, fake, None)
        assert st == 2                 # INTLORA_ERR_UNSUPPORTED
        msg = lib.intlora_last_error().decode()
        assert str(MAX_ELEMENTS) in msg and "workspace" in msg
    # bad arguments are reported as such, not as a size problem
    st = lib.intlora_gen_aux_noalloc(None, 4, 8, 1, 0, 1.5, 8, fake, fake, None, fake, 16,
                                     fake, fake, None)
    assert st == 1
