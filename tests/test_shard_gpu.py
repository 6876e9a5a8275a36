"""Layer-sharded whole-model merge through the product path: two ranks (gloo
for the host-side bookkeeping, both on cuda:0, each with its own CUDA context)
split a small model's layers with shard_layers, run preparation, the merge
and the STE backward on their own layers through the C ABI, and rank 0
gathers the results. Layers are independent, so no kernel of one rank waits
on the other; the gathered results equal a single-process run bit for bit
and meet the oracle."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

pytestmark = pytest.mark.gpu


def _model():
    from quantized_lora_merge_b200 import workloads as wl
    shapes = [(64, 4096, 16, 8), (130, 320, 4, 4), (48, 2048, 32, 8), (20, 768, 8, 4), (96, 1024, 16, 8)]
    return [wl.LayerSpec(f"l{k}", d, n, r, wb, "mul", 8 if wb == 8 else 4, stream_id=k, ste=True)
            for k, (d, n, r, wb) in enumerate(shapes)]


def _run_layers(specs):
    """Product path on host numpy inputs: returns per layer (P, s_bar, z_bar,
    W_round codes, dA, dB) as numpy arrays."""
    from quantized_lora_merge_b200 import pipeline as P
    from quantized_lora_merge_b200 import workloads as wl
    dev = torch.device("cuda", 0)
    states = []
    for sp in specs:
        W = torch.from_numpy(wl.host_W(sp)).to(dev)
        A = torch.from_numpy(wl.host_A(sp)).to(dev)
        Bm = torch.from_numpy(wl.host_B(sp)).to(dev)
        bf = lambda bits: torch.from_numpy(bits.view(np.int16)).to(dev).view(torch.bfloat16)  # noqa: E731
        states.append(P.allocate(sp, W, A, Bm, dev, G=bf(wl.host_G_bits(sp)),
                                 A16=bf(wl.to_bf16_bits(wl.host_A(sp))),
                                 B16=bf(wl.to_bf16_bits(wl.host_B(sp)))))
    path = P.Path(states, dev)
    path.step()
    torch.cuda.synchronize()
    return [dict(P=st.out.cpu().numpy(), sbar=st.sbar.cpu().numpy(), zbar=st.zbar.cpu().numpy(),
                 codes=st.w_round.cpu().numpy(), s=st.s.cpu().numpy(), z=st.z.cpu().numpy(),
                 sigma=st.sigma.cpu().numpy(), dA=st.dA.cpu().numpy(), dB=st.dB.cpu().numpy())
            for st in states]


def _worker(rank, world, port, out_q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    try:
        from quantized_lora_merge_b200.sharding import shard_layers
        torch.cuda.set_device(0)
        layers = _model()
        mine = shard_layers([l.numel for l in layers], world)[rank]
        res = _run_layers([layers[k] for k in mine])
        gathered = [None] * world
        dist.all_gather_object(gathered, {k: r for k, r in zip(mine, res)})
        if rank == 0:
            merged = {}
            for part in gathered:
                assert not (set(part) & set(merged))
                merged.update(part)
            out_q.put(merged)
    finally:
        dist.destroy_process_group()


def test_two_rank_sharded_product_path_equals_single_process():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    merged = q.get(timeout=600)
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    layers = _model()
    assert sorted(merged) == list(range(len(layers)))
    single = _run_layers(layers)
    for k in range(len(layers)):
        for key in ("P", "sbar", "zbar", "codes", "s", "z", "sigma", "dA", "dB"):
            assert np.array_equal(merged[k][key], single[k][key]), (k, key)

    # and the sharded results meet the oracle (preparation and merge of two layers)
    import oracle
    from quantized_lora_merge_b200 import workloads as wl
    from .parity import assert_affine, assert_scale
    for k in (0, 2):
        sp = layers[k]
        o = oracle.gen_aux(wl.host_W(sp), sp.seed, sp.stream_id, sp.alpha, sp.w_bits)
        assert_scale("sigma_w", merged[k]["sigma"][0], o["sigma_w"])
        assert_affine("W_round", wl.unpack_codes(merged[k]["codes"], sp.n, sp.w_bits), merged[k]["z"],
                      o["codes"], o["z"], o["pre"], o["zpre"], 2**sp.w_bits - 1)
