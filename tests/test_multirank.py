"""Multi-rank bookkeeping on CPU with gloo (world size 2): layers are sharded
with no collective on the data path, each rank prepares and merges its own
layers (here with the oracle, standing in for the GPU path), and the gathered
results equal a single-rank run. Also the max-over-ranks timing reduction."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from quantized_lora_merge_b200 import workloads as wl
from quantized_lora_merge_b200.sharding import imbalance, shard_layers


def test_shard_layers_properties():
    layers = wl.sd_unet()
    numels = [l.numel for l in layers]
    for world in (1, 2, 3, 4, 8):
        shards = shard_layers(numels, world)
        owned = sorted(k for s in shards for k in s)
        assert owned == list(range(len(layers)))          # each layer exactly once
        assert all(s == sorted(s) for s in shards)
        assert imbalance(numels, shards) < 1.05
    assert shard_layers([5, 3], 4)[2:] == [[], []]
    with pytest.raises(ValueError):
        shard_layers([1], 0)


def _layer_result(spec):
    import oracle
    W = wl.host_W(spec)
    g = oracle.gen_aux(W, spec.seed, spec.stream_id, spec.alpha, spec.w_bits)
    m = oracle.merge_mul(g["codes"], g["s"].astype(np.float32), g["z"], wl.host_A(spec),
                         wl.host_B(spec), spec.seed, spec.stream_id, g["sigma_w"], g["sigma_r"],
                         spec.alpha, spec.out_bits)
    return np.concatenate([m["P"].ravel().astype(np.float64), m["sbar"], [g["sigma_r"]]])


def _small_model():
    return [wl.LayerSpec(f"l{k}", d, n, 4, 4, "mul", 4, stream_id=k)
            for k, (d, n) in enumerate([(16, 32), (8, 64), (24, 16), (4, 40), (12, 12)])]


def _worker(rank, world, port, out_q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        layers = _small_model()
        mine = shard_layers([l.numel for l in layers], world)[rank]
        results = {k: _layer_result(layers[k]) for k in mine}
        gathered = [None] * world
        dist.all_gather_object(gathered, results)
        t = torch.tensor([1.0 + rank], dtype=torch.float64)     # per-rank step time
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        if rank == 0:
            merged = {}
            for part in gathered:
                assert not (set(part) & set(merged))
                merged.update(part)
            out_q.put((merged, float(t.item())))
    finally:
        dist.destroy_process_group()


def test_two_rank_sharded_results_equal_single_rank():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    merged, tmax = q.get(timeout=300)
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    layers = _small_model()
    assert sorted(merged) == list(range(len(layers)))
    for k, spec in enumerate(layers):
        assert np.array_equal(merged[k], _layer_result(spec))
    assert tmax == 2.0


def _e2e_worker(rank, world, port, mem_kb, tmpdir, out_q):
    import datetime
    import sys
    from pathlib import Path
    sys.path.insert(0, str(Path(__file__).resolve().parents[1]))
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    os.environ["LOCAL_WORLD_SIZE"] = "1"
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        mi = Path(tmpdir) / f"meminfo{rank}"
        mi.write_text(f"MemTotal: {2 * mem_kb[rank]} kB\nMemAvailable: {mem_kb[rank]} kB\n")
        ok, why = bench.e2e_allowed(40 << 30, world, torch.device("cpu"), meminfo=str(mi))
        out_q.put((rank, ok, why))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("mem_gib,expect", [((200, 200), True), ((200, 10), False)])
def test_end_to_end_leg_is_skipped_by_every_rank_or_none(tmp_path, mem_gib, expect):
    """bench.py's end-to-end leg holds collectives, so the host-memory check
    is agreed across ranks: one short node makes every rank skip it."""
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    mem_kb = [g << 20 for g in mem_gib]
    procs = [ctx.Process(target=_e2e_worker, args=(r, 2, port, mem_kb, str(tmp_path), q))
             for r in range(2)]
    for p in procs:
        p.start()
    got = dict((r, (ok, why)) for r, ok, why in (q.get(timeout=300) for _ in range(2)))
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    assert got[0][0] == got[1][0] == expect
    if not expect:
        assert "rank(s)" in got[1][1] and "another rank" in got[0][1]
