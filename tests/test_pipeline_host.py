"""Host-side plumbing of the pipeline (no GPU): the I/O arenas that let the
end-to-end leg move every layer's inputs and outputs with one copy each way."""
import torch

from quantized_lora_merge_b200 import pipeline as P
from quantized_lora_merge_b200 import workloads as wl


def _state(spec):
    d, n, r = spec.d, spec.n, spec.r
    st = P.LayerState(spec=spec, W=torch.randn(d, n), A=torch.randn(d, r), B=torch.randn(r, n),
                      sigma=torch.zeros(2, dtype=torch.float64),
                      w_round=torch.zeros(d, P.code_row_bytes(n, spec.w_bits), dtype=torch.uint8),
                      s=torch.zeros(d), z=torch.zeros(d, dtype=torch.int32),
                      out=torch.zeros(d, n, dtype=torch.int16), sbar=torch.zeros(d),
                      zbar=torch.zeros(d, dtype=torch.int32))
    st.G = torch.randn(d, n).to(torch.bfloat16)
    st.A16, st.B16 = st.A.to(torch.bfloat16), st.B.to(torch.bfloat16)
    st.dA, st.dB = torch.zeros(d, r), torch.zeros(r, n)
    return st


def test_pack_io_keeps_values_aligns_views_and_aliases_the_arenas():
    specs = [wl.LayerSpec("a", 5, 12, 3, 4, "mul", 4, stream_id=0),
             wl.LayerSpec("b", 7, 20, 4, 4, "mul", 4, stream_id=1)]
    states = [_state(s) for s in specs]
    before = [{k: getattr(st, k).clone() for k in ("W", "A", "B", "G", "A16", "B16")}
              for st in states]
    a_in, a_out = P.pack_io(states, "cpu")
    base_in, base_out = a_in.data_ptr(), a_out.data_ptr()
    for st, old in zip(states, before):
        for k, v in old.items():
            t = getattr(st, k)
            assert torch.equal(t, v)
            assert (t.data_ptr() - base_in) % 256 == 0
            assert base_in <= t.data_ptr() < base_in + a_in.numel()
        for k in ("out", "sbar", "zbar", "dA", "dB"):
            t = getattr(st, k)
            assert (t.data_ptr() - base_out) % 256 == 0
            assert base_out <= t.data_ptr() < base_out + a_out.numel()
    # writing through the arena is seen by the layer views
    a_out.fill_(0)
    states[1].sbar.fill_(2.5)
    assert a_out.view(torch.uint8).sum() > 0
    a_out.zero_()
    assert float(states[1].sbar.abs().sum()) == 0.0
