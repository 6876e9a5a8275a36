#!/usr/bin/env python
"""Benchmark of the IntLoRA merge hot path on B200.

One step = the whole per-layer path over every layer of the workload:
layer preparation (Philox/Laplace R, sigma_W and sigma_R, VMC, base
quantization of W - R*), the merge (MUL for the default workload) and the STE
backward (dA = G B^T, dB = A^T G), each stage one batched call of the C ABI.

Default workload: the 224 linears of a Llama-3-8B-shaped decoder (32 layers:
q, o 4096x4096; k, v 1024x4096; gate, up 14336x4096; down 4096x14336), int8
base codes, rank 16, alpha 1.5, MUL with an 8-bit U quantizer: 6,979,321,856
merged weight elements per step, the largest of the workloads that fits one
GPU (synthetic inputs drawn on the device). `--config sd_unet`, `dit_3072`,
`rank_sweep` and `linear320` select the other workloads. Metric: merged weight
elements per second (whole job); the merge stage's achieved HBM GB/s and its
fraction of the measured copy peak beside it.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
Multi-GPU: one process per GPU under torch.distributed.run; every rank runs its
own copy of the workload (weak scaling; layers are independent, no collective
on the data path), timing is the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time
from pathlib import Path

ROOT = Path(__file__).resolve().parent
sys.path.insert(0, str(ROOT))

METRIC = "merged weight elements/s and achieved HBM GB/s (% of B200 peak), 1 GPU"
UNIT = "elements/s"
NOMINAL_HBM_GBS = 7700.0      # B200 HBM3e nominal (HGX); the measured copy peak is the primary roof
FALLBACK_HBM_GBS = 6650.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", default="llama3_8b")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true",
                    help="skip the integer-GEMM and training-step legs of the default line")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--reference-seconds", type=float, default=150.0,
                    help="--impl reference: oracle seconds over the whole run (warm-up and timed "
                         "steps), split evenly across the steps")
    ap.add_argument("--op", default="step", choices=["step", "int_gemm", "train_forward"],
                    help="step: the merge hot path (default); int_gemm: the integer "
                         "inference GEMM on merged weights")
    ap.add_argument("--planes", type=int, default=1, choices=[1, 2, 3],
                    help="int_gemm: digit planes of the merged weights (1: SHIFT of 4-bit "
                         "codes, 2: MUL of 4-bit codes, 3: MUL of 8-bit codes)")
    ap.add_argument("--tokens", type=int, default=4096)
    ap.add_argument("--y-bf16", action="store_true", help="int_gemm: write Y in bf16")
    ap.add_argument("--dist", type=int, default=0, choices=[0, 1, 2, 3],
                    help="auxiliary law of R for every layer: 0 Laplace (the method's), 1 Gaussian, "
                         "2 Cauchy, 3 Student-t with 2 degrees of freedom (the ablation's laws)")
    ap.add_argument("--rank", type=int, default=0,
                    help="keep only the layers of this LoRA rank (e.g. one point of --config rank_sweep)")
    ap.add_argument("--masked-ste", action="store_true",
                    help="STE backward restricted to D = W_round - z != 0 (the layers' own codes)")
    ap.add_argument("--shard", action="store_true",
                    help="strong scaling: split the model's layers across the ranks (greedy by "
                         "element count) instead of giving every rank its own copy")
    return ap.parse_args()


def peaks():
    p = ROOT / "MEASURED_PEAKS.json"
    if p.exists():
        d = json.loads(p.read_text())
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def workload_desc(name, layers):
    from quantized_lora_merge_b200 import workloads as wl
    l0 = layers[0]
    total = sum(l.numel for l in layers)
    return {
        "workload": f"{name}: {len(layers)} linears, int{l0.w_bits} base codes, r={l0.r}, "
                    f"alpha={l0.alpha}, {l0.variant.upper()} {l0.out_bits}-bit; prepare + merge "
                    f"+ STE backward per step",
        "layers": len(layers),
        "merged_elements_per_step": total,
        "l2": "inputs larger than L2 (fp32 W 4 B/elem + bf16 G 2 B/elem per step, "
              f"{(6 * total) / 1e9:.2f} GB)",
        "data": "synthetic (seeded device draws, shapes of the named model)",
    }


# ---------------------------------------------------------------------------
# algorithmic bytes (unit of work: one merged element)
# ---------------------------------------------------------------------------
def merge_bytes(l):
    code = 0.5 if l.w_bits == 4 else 1.0
    if l.variant == "mul":
        out = 2 if ((2**l.w_bits - 1) * (2**l.out_bits - 1) <= 32767) else 4
        per_row = 4 + 4 + 4 + 4           # s, z in; s_bar, z_bar out
    else:
        out = 1 if l.w_bits <= 7 else 2
        per_row = 4 + 4 + 4
    return l.numel * (code + out) + l.d * per_row + 4 * l.r * (l.d + l.n)


def prepare_bytes(l):
    code = 0.5 if l.w_bits == 4 else 1.0
    # statistics pass reads W; quantization pass reads W and writes codes, s, z
    return l.numel * (4 + 4 + code) + l.d * 8


def merge_ops(l, fused=False):
    """Algorithmic lane operations of the merge kernel, per element x numel:
    Philox4x32-10 share (10 rounds x 4 ops / 4 words = 10), Laplace inverse CDF
    (6: shift, int->float, fma, log2, scale, sign), T = A.B (r FMAs on the
    CUDA cores; none where the tensor cores form it), U (4: add, fma,
    reciprocal multiply, select), row extrema (2), quantize + product (MUL
    5.5: fma, round, clamp x2, sub, half an IMAD; SHIFT 8: abs, exponent,
    mantissa compare, clamps, shift, sign)."""
    quant = 5.5 if l.variant == "mul" else 8.0
    return l.numel * (10 + 6 + (0 if fused else l.r) + 4 + 2 + quant)


ALU_LANES_PER_SM_CLK = 128       # FP32/INT32 lanes per SM per clock on sm_100
NUM_SMS = 148


# sources the fused merge kernel is compiled from (a stored ncu figure is used
# only while they hash to the value recorded beside it)
MERGE_TC_SOURCES = ("merge_tc_kernels.cu", "intlora_device.cuh", "tcgen05_util.cuh", "intlora_kernels.h")
DOMINANT_SOURCES = MERGE_TC_SOURCES


def csrc_hash(sources=None):
    """Hash of the dominant kernel's CUDA sources, so a stored ncu traffic
    figure is only used while the kernel it was taken on is unchanged."""
    import hashlib
    h = hashlib.sha256()
    root = Path(__file__).resolve().parent / "quantized_lora_merge_b200" / "csrc"
    for name in (sources or DOMINANT_SOURCES):
        h.update(name.encode())
        h.update((root / name).read_bytes())
    return h.hexdigest()


def profiled_traffic(name, sources=None, field="dram_bytes_per_launch"):
    """dram__bytes_read.sum + dram__bytes_write.sum (per launch, or per element
    with field="dram_bytes_per_element") from the ncu summary
    profiles/<name>.md, or None when absent or when the kernels have changed
    since it was taken."""
    p = Path(__file__).resolve().parent / "profiles" / f"{name}.md"
    if not p.exists():
        return None
    fields = {}
    for line in p.read_text().splitlines():
        if ":" in line:
            k, v = line.split(":", 1)
            fields[k.strip().strip("-* `")] = v.strip().strip("` ")
    if fields.get("csrc_sha256") != csrc_hash(sources):
        return None
    try:
        return float(fields[field])
    except (KeyError, ValueError):
        return None


def ste_bytes(l):
    # G read once (both products from one pass), A, B, dA, dB
    return l.numel * 2 + l.r * (l.d + l.n) * (2 + 4)


# ---------------------------------------------------------------------------
# clocks
# ---------------------------------------------------------------------------
class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out = ""
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
            except ValueError:
                continue
            for name, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "samples": len(sm), "reasons": sorted(reasons)}


# ---------------------------------------------------------------------------
# CPU oracle baseline (bounded sample of the same workload)
# ---------------------------------------------------------------------------
def oracle_sample(layers, seconds):
    """Run the oracle's whole path (prepare, merge, STE) layer by layer in
    workload order until `seconds` have passed; returns (elements, time)."""
    import numpy as np

    import oracle
    from quantized_lora_merge_b200 import workloads as wl
    done, t_total, names = 0, 0.0, []
    for spec in layers:
        W, A, Bm = wl.host_W(spec), wl.host_A(spec), wl.host_B(spec)
        Gb = wl.host_G_bits(spec)
        A16, B16 = wl.to_bf16_bits(A), wl.to_bf16_bits(Bm)
        t0 = time.perf_counter()
        g = oracle.gen_aux(W, spec.seed, spec.stream_id, spec.alpha, spec.w_bits,
                           dist=spec.distribution)
        s32 = g["s"].astype(np.float32)
        if spec.variant == "mul":
            oracle.merge_mul(g["codes"], s32, g["z"], A, Bm, spec.seed, spec.stream_id,
                             g["sigma_w"], g["sigma_r"], spec.alpha, spec.out_bits,
                             dist=spec.distribution)
        else:
            oracle.merge_shift(g["codes"], s32, g["z"], A, Bm, spec.seed, spec.stream_id,
                               g["sigma_w"], g["sigma_r"], spec.alpha, spec.out_bits,
                               dist=spec.distribution)
        oracle.ste_backward(wl.bf16_bits_to_f32(Gb).astype(np.float64),
                            wl.bf16_bits_to_f32(A16).astype(np.float64),
                            wl.bf16_bits_to_f32(B16).astype(np.float64))
        t_total += time.perf_counter() - t0
        done += spec.numel
        names.append(spec.name)
        if t_total >= seconds:
            break
    return done, t_total, names


def single_core(layers):
    """The oracle on one host thread over the config's smallest layer (whole
    path, repeated until a second has passed), beside the all-core figure."""
    import oracle
    small = min(layers, key=lambda l: l.numel)
    threads = oracle.num_threads()
    oracle.set_num_threads(1)
    done, t, passes = 0, 0.0, 0
    try:
        cores = oracle.num_threads()
        while t < 1.0:
            d, tt, _ = oracle_sample([small], 0.0)
            done, t, passes = done + d, t + tt, passes + 1
    finally:
        oracle.set_num_threads(threads)
    return {"value": done / t, "unit": UNIT, "cores": cores,
            "sample": f"layer {small.name} ({small.d}x{small.n}, the config's smallest) x {passes}, "
                      f"prepare + merge + STE, {t:.1f} s"}


def cpu_baseline(layers, seconds):
    import oracle
    done, t, names = oracle_sample(layers, seconds)
    return {"value": done / t, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"first {len(names)} of {len(layers)} layers in workload order "
                      f"({done} merged elements, prepare + merge + STE, {t:.1f} s)",
            "single_core": single_core(layers)}


# ---------------------------------------------------------------------------
# reference arm: the oracle as it stands on the host cores
# ---------------------------------------------------------------------------
def reference_sample(layers, budget):
    """The per-step sample of the reference arm: whole layers in workload
    order while one still fits the per-step budget (seconds), else a block of
    the first layer's leading rows taken as a layer of its own (whole path,
    sigma over the block), sized by timing a 16-row block. Returns (layers
    to run, description)."""
    from dataclasses import replace
    first = layers[0]
    probe = replace(first, d=min(first.d, 16))
    done, t, _ = oracle_sample([probe], 0.0)
    per_row = t / probe.d
    if per_row * first.d <= budget:
        return layers, "first {count} layers in workload order, prepare + merge + STE"
    rows = max(1, min(first.d, int(budget / per_row)))
    return ([replace(first, d=rows)],
            f"the first {rows} of {first.d} rows of {first.name} ({first.d}x{first.n}) taken as one "
            f"layer, prepare + merge + STE")


def run_reference(args, layers, desc):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    # the whole run's oracle work stays near args.reference_seconds
    budget = args.reference_seconds / max(1, args.steps + args.warmup)
    per_step_seconds = min(20.0, budget)
    sample, what = reference_sample(layers, per_step_seconds)
    for _ in range(args.warmup):
        oracle_sample(sample, per_step_seconds)
    done = t = 0.0
    names = []
    for _ in range(args.steps):
        d, tt, names = oracle_sample(sample, per_step_seconds)
        done += d
        t += tt
    import oracle
    value = done / t
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1000.0 * t / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": desc,
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": oracle.num_threads(),
                             "kind": "oracle",
                             "sample": "each step: " + what.format(count=len(names)),
                             "single_core": single_core(layers)},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------
def main():
    args = parse()
    if args.op == "int_gemm":
        bench_int_gemm(args)
        return
    if args.op == "train_forward":
        bench_train_forward(args)
        return
    from quantized_lora_merge_b200 import workloads as wl
    layers_base = wl.CONFIGS[args.config]()
    if args.rank:
        layers_base = [l for l in layers_base if l.r == args.rank]
        if not layers_base:
            raise SystemExit(f"no layer of rank {args.rank} in {args.config}")
    if args.dist:
        from dataclasses import replace as _replace
        layers_base = [_replace(l, distribution=args.dist) for l in layers_base]
    desc = workload_desc(args.config, layers_base)
    if args.dist:
        desc["auxiliary_law"] = ["laplace", "gaussian", "cauchy", "student_t2"][args.dist]
    if args.masked_ste:
        desc["ste"] = "masked: G kept where W_round != z"
    if args.impl == "reference":
        run_reference(args, layers_base, desc)
        return

    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=device)

    from dataclasses import replace

    from quantized_lora_merge_b200 import build as qbuild
    from quantized_lora_merge_b200 import pipeline as P
    qbuild.build()
    if args.shard:
        # strong scaling: the model's layers are split across the ranks, no
        # collective on the data path
        from quantized_lora_merge_b200.sharding import shard_layers
        if world > len(layers_base):
            raise SystemExit(f"--shard needs at most {len(layers_base)} ranks for this model")
        owned = shard_layers([l.numel for l in layers_base], world)[rank]
        layers = [replace(layers_base[k], ste=True) for k in owned]
    else:
        # weak scaling: every rank owns its own copy of the workload (own R streams)
        layers = [replace(l, stream_id=l.stream_id + 1000 * rank, ste=True) for l in layers_base]

    states = []
    for spec in layers:
        t = wl.device_inputs(spec, device, with_grad=True, salt=rank)
        states.append(P.allocate(spec, t["W"], t["A"], t["B"], device, G=t["G"], A16=t["A16"],
                                 B16=t["B16"]))
    # inputs and outputs each live in one arena, so the end-to-end leg moves
    # them with one host<->device copy per direction
    arena_in, arena_out = P.pack_io(states, device)
    torch.cuda.empty_cache()
    path = P.Path(states, device, masked_ste=args.masked_ste)
    stream = torch.cuda.current_stream(device)

    def barrier():
        if world > 1:
            dist.barrier()

    # warm-up
    for _ in range(max(3, args.warmup)):
        path.step()
    torch.cuda.synchronize(device)

    # timed region: whole steps, plus per-stage events on the launching stream
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    from quantized_lora_merge_b200 import binding as Bnd
    barrier()
    torch.cuda.synchronize(device)
    launches0 = Bnd.intlora_kernel_launches()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for k in range(args.steps):
        ev[k][0].record(stream)
        path.prepare()
        ev[k][1].record(stream)
        path.merge()
        ev[k][2].record(stream)
        path.backward()
        ev[k][3].record(stream)
    t_end.record(stream)
    launches = Bnd.intlora_kernel_launches() - launches0
    torch.cuda.synchronize(device)
    barrier()
    clk = clocks.stop()
    ms_total = t_start.elapsed_time(t_end)
    stage_ms = {name: sum(ev[k][i].elapsed_time(ev[k][i + 1]) for k in range(args.steps))
                / args.steps for i, name in enumerate(["prepare", "merge", "ste_backward"])}
    ms_step = ms_total / args.steps
    if world > 1:
        t = torch.tensor([ms_step], device=device, dtype=torch.float64)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms_step = float(t.item())

    elements = (sum(l.numel for l in layers_base) if args.shard
                else sum(l.numel for l in layers) * world)
    value = elements / (ms_step / 1000.0)
    hbm_peak, peak_kind = peaks()

    per_stage_bytes = {"prepare": sum(prepare_bytes(l) for l in layers),
                       "merge": sum(merge_bytes(l) for l in layers),
                       "ste_backward": sum(ste_bytes(l) for l in layers)}
    stages = {}
    for name, ms in stage_ms.items():
        gbs = per_stage_bytes[name] / (ms / 1000.0) / 1e9
        stages[name] = {"ms": ms, "algorithmic_GB": per_stage_bytes[name] / 1e9,
                        "GB_s": gbs, "frac_of_hbm": gbs / hbm_peak}
    stages["merge"]["elements_per_s"] = sum(l.numel for l in layers) / (stage_ms["merge"] / 1e3)
    # The metric's kernel: the merge stage. Layers of rank >= 16 whose rows are a
    # multiple of 32 columns run on the fused tensor-core merge kernel (one
    # cooperative launch per row width), the rest on the team / row-tile
    # kernels (the library's routing). Its roofline is HBM (algorithmic bytes
    # of W_round, A, B and the outputs); the lane-issue view (modelled
    # operations per element over the SM lane rate at the sampled clock)
    # is reported beside it.
    sm_mhz = clk.get("sm_mhz") or 1965.0
    alu_peak = NUM_SMS * ALU_LANES_PER_SM_CLK * sm_mhz * 1e6 / 1e12          # Top/s
    # the library's routing: the fused kernel from rank 16, and at any rank for
    # rows wider than the team kernels take (6144 columns)
    on_tc = [(not args.dist) and l.n % 32 == 0 and (l.r >= 16 or l.n > 6144) for l in layers]
    fused = all(on_tc)
    alu_achieved = sum(merge_ops(l, f) for l, f in zip(layers, on_tc)) / (stage_ms["merge"] / 1e3) / 1e12
    kernel_name = ("merge_tc_kernel (fused tensor-core merge)" if fused else
                   "merge_tc_kernel (wide rows) + team kernels" if any(on_tc) else
                   "team / row-tile merge kernels" if not args.dist else
                   "merge row-tile kernel (general auxiliary law)")
    traffic = None
    if fused:
        per_el = profiled_traffic(f"merge_tc_kernel_{args.config}", MERGE_TC_SOURCES, "dram_bytes_per_element")
        if per_el is not None:
            traffic = per_el * sum(l.numel for l in layers)

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "strong" if args.shard else "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic", "config": desc,
        "sharding": "layers split across ranks" if args.shard else "one copy of the workload per rank",
        "hbm_GB_s_merge": stages["merge"]["GB_s"],
        "hbm_frac_merge": stages["merge"]["frac_of_hbm"],
        "roofline": {"bound": "hbm", "kernel": kernel_name, "stage": "merge (every launch of the stage)",
                     "achieved": stages["merge"]["GB_s"], "peak": hbm_peak, "unit": "GB/s",
                     "frac": stages["merge"]["frac_of_hbm"],
                     "peak_source": f"{peak_kind} copy bandwidth (MEASURED_PEAKS.json hbm_gbs)",
                     "frac_of_nominal": stages["merge"]["GB_s"] / NOMINAL_HBM_GBS,
                     "nominal_peak": NOMINAL_HBM_GBS,
                     "nominal_source": "B200 HBM3e nominal bandwidth (HGX), secondary reference",
                     "algorithmic_bytes_per_step": per_stage_bytes["merge"],
                     "traffic": traffic,
                     "traffic_unit": "DRAM bytes per step of the stage (ncu bytes per element x elements)",
                     "alu_achieved_Top_s": alu_achieved, "alu_peak_Top_s": alu_peak,
                     "alu_frac_modelled": alu_achieved / alu_peak,
                     "alu_peak_source": f"148 SMs x 128 lanes x measured {sm_mhz:.0f} MHz",
                     "ops_per_element_modelled": merge_ops(layers[0], on_tc[0]) / layers[0].numel},
        "stages": stages,
        "clocks": clk,
        "gpu_launches": launches,
    }

    if not args.no_e2e:
        ok, why = e2e_allowed(arena_in.numel() + arena_out.numel(), world, device)
        if ok:
            line["e2e"] = e2e(states, arena_in, arena_out, device, max(4, min(args.steps, 10)),
                              world, elements, masked_ste=args.masked_ste)
        else:
            line["e2e"] = {"value": None, "unit": UNIT, "unavailable": why}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(layers_base, args.cpu_seconds)
    if not args.no_extra:
        # the next rows of the path, measured on the same GPU after the main
        # workload is released: every rank runs them (no collective inside)
        del path, states, arena_in, arena_out
        torch.cuda.empty_cache()
        launches0 = Bnd.intlora_kernel_launches()
        line["next_int_gemm"] = int_gemm_leg(device, planes=1, tokens=4096, steps=50)
        line["next_train_step"] = train_step_leg(device, tokens=4096, steps=10)
        line["next_legs_gpu_launches"] = Bnd.intlora_kernel_launches() - launches0
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


def int_gemm_leg(device, planes, tokens, steps):
    """Integer inference GEMM on merged weights (the four DiT-3072 block
    linears at `tokens` tokens, merged weights as `planes` int8 digit planes,
    one batched call per step); CUDA-event time, int8 tensor Top/s and the
    fraction of 2 x the measured bf16 dense peak."""
    import torch

    from quantized_lora_merge_b200 import binding as B
    from quantized_lora_merge_b200 import workloads as wl
    bound = wl.INT_GEMM_BOUNDS[GEMM_KIND[planes]]
    jobs, shapes = [], []
    for k, (d, n) in enumerate(GEMM_SHAPES):
        X, xs, Q, ws = wl.int_gemm_device(tokens, d, n, bound, device, salt=k)
        packed = torch.empty((d, planes, n), dtype=torch.int8, device=device)
        B.intlora_int_pack(Q, planes, packed)
        del Q
        jobs.append(B.IntGemmJob(X, xs, packed, ws, torch.empty((tokens, d), device=device)))
        shapes.append((d, n))
    desc = B.Descriptors(jobs)
    for _ in range(3):
        B.intlora_int_gemm_batched(desc, planes)
    stream = torch.cuda.current_stream(device)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(device)
    a.record(stream)
    for _ in range(steps):
        B.intlora_int_gemm_batched(desc, planes)
    b.record(stream)
    torch.cuda.synchronize(device)
    ms = a.elapsed_time(b) / steps
    ops = sum(2 * tokens * d * n * planes for d, n in shapes)
    bf16, kind = bf16_peak_tflops()
    top_s = ops / (ms / 1e3) / 1e12
    del jobs, desc
    torch.cuda.empty_cache()
    return {"workload": f"DiT-3072 block GEMMs at {tokens} tokens, {planes} int8 digit plane(s), fp32 Y",
            "ms": ms, "steps": steps, "tensor_Top_s": top_s, "peak_Top_s": 2.0 * bf16,
            "frac_of_int8_peak": top_s / (2.0 * bf16),
            "peak_source": f"2 x {kind} bf16 dense (nominal int8/bf16 ratio 2)",
            "kernel": "int_gemm_kernel (tcgen05 kind::i8)"}


def train_step_leg(device, tokens, steps):
    """One IntLoRA training step of every SD-UNet linear at `tokens` tokens:
    the MUL merge, the bf16 fake-quantized merged weight, the forward GEMM
    Y = X W'^T and the backward (dX = dY W', dA and dB through the STE
    without the weight gradient in HBM), each one batched call. CUDA-event
    times per stage; bf16 tensor TFLOP/s of the two layer-sized GEMMs
    (forward and dX, 4 tokens d n per layer) against the measured peak."""
    import torch

    from quantized_lora_merge_b200 import binding as B
    from quantized_lora_merge_b200 import pipeline as P
    from quantized_lora_merge_b200 import workloads as wl
    layers = wl.CONFIGS["sd_unet"]()
    states = []
    for spec in layers:
        t = wl.device_inputs(spec, device, with_grad=True, salt=0)
        states.append(P.allocate(spec, t["W"], t["A"], t["B"], device, G=t["G"], A16=t["A16"],
                                 B16=t["B16"]))
    path = P.Path(states, device)
    path.prepare()
    g = torch.Generator(device=device)
    g.manual_seed(17)
    wq = [torch.empty(l.d, l.n, dtype=torch.bfloat16, device=device) for l in layers]
    X = [torch.randn(tokens, l.n, generator=g, device=device).to(torch.bfloat16) for l in layers]
    dY = [(torch.randn(tokens, l.d, generator=g, device=device) * 1e-3).to(torch.bfloat16)
          for l in layers]
    fq = B.Descriptors(B.FakeQuantJob(st.out, st.sbar, w) for st, w in zip(states, wq))
    lin = B.Descriptors(B.LinearJob(x, w, torch.empty(tokens, l.d, dtype=torch.bfloat16,
                                                      device=device))
                        for l, x, w in zip(layers, X, wq))
    bwd_jobs = [B.TrainBackwardJob(x, dy, w, st.A16, st.B16,
                                   torch.empty(tokens, l.n, device=device), st.dA, st.dB)
                for l, st, x, dy, w in zip(layers, states, X, dY, wq)]
    bwd = B.Descriptors(bwd_jobs)
    ws = torch.empty(max(256, B.intlora_train_backward_workspace_size(bwd_jobs)), dtype=torch.uint8,
                     device=device)
    stream = torch.cuda.current_stream(device)

    def step(ev=None):
        path.merge()
        if ev: ev[0].record(stream)
        B.intlora_fakequant_bf16_batched(fq)
        if ev: ev[1].record(stream)
        B.intlora_linear_bf16_batched(lin)
        if ev: ev[2].record(stream)
        B.intlora_train_backward_batched(bwd, ws)
        if ev: ev[3].record(stream)

    for _ in range(3):
        step()
    torch.cuda.synchronize(device)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)]
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for k in range(steps):
        step(evs[k])
    b.record(stream)
    torch.cuda.synchronize(device)
    ms = a.elapsed_time(b) / steps
    fwd_ms = sum(e[1].elapsed_time(e[2]) for e in evs) / steps
    bwd_ms = sum(e[2].elapsed_time(e[3]) for e in evs) / steps
    gemm_flops = sum(4 * tokens * l.d * l.n for l in layers)
    bf16, kind = bf16_peak_tflops()
    tf = gemm_flops / ((fwd_ms + bwd_ms) / 1e3) / 1e12
    del states, path, wq, X, dY, fq, lin, bwd, bwd_jobs, ws
    torch.cuda.empty_cache()
    return {"workload": f"SD-UNet 128 linears at {tokens} tokens: MUL merge + fake-quantization + "
                        f"Y = X W'^T + backward (dX, dA, dB)",
            "ms": ms, "steps": steps, "forward_gemm_ms": fwd_ms, "backward_ms": bwd_ms,
            "gemm_TFLOP_s": tf, "peak_TFLOP_s": bf16, "frac_of_bf16_peak": tf / bf16,
            "peak_source": f"{kind} bf16 dense",
            "note": "TFLOP/s counts the forward and dX GEMMs (4 tokens d n per layer) over the "
                    "forward-GEMM plus backward time; the backward also forms dA and dB"}


def pinned_host(nbytes):
    """Page-locked host buffer of exactly `nbytes` (numpy memory registered
    with the CUDA runtime; torch's pinned allocator would round a 40 GB request
    up to the next power of two). Returns (tensor, release)."""
    import numpy as np
    import torch
    a = np.empty(max(nbytes, 1), dtype=np.uint8)
    rt = torch.cuda.cudart()
    rc = rt.cudaHostRegister(a.ctypes.data, a.nbytes, 0)
    if int(rc) != 0:
        raise RuntimeError(f"cudaHostRegister of {nbytes} bytes failed ({rc})")
    t = torch.from_numpy(a)
    assert t.is_pinned()

    def release():
        rt.cudaHostUnregister(a.ctypes.data)
    return t, release


def host_room(need_bytes, local_ranks, meminfo="/proc/meminfo"):
    """Whether this node's available host memory holds the end-to-end leg's
    pinned arenas for every rank on it (need_bytes each, 10 % margin).
    Returns (ok, reason)."""
    try:
        with open(meminfo) as f:
            avail = next(int(line.split()[1]) * 1024 for line in f if line.startswith("MemAvailable:"))
    except (OSError, StopIteration, ValueError, IndexError):
        return True, ""                 # unknown: let cudaHostRegister decide
    total = need_bytes * max(1, local_ranks)
    if total * 1.1 <= avail:
        return True, ""
    return False, (f"pinned host arenas of {local_ranks} rank(s) x {need_bytes / 1e9:.1f} GB exceed "
                   f"the node's {avail / 1e9:.1f} GB of available host memory")


def e2e_allowed(need_bytes, world, device, meminfo="/proc/meminfo"):
    """Whether the end-to-end leg runs. One rank alone leaves the question to
    cudaHostRegister; several ranks check their node's memory for every
    local rank's arenas (host_room) and agree by a MIN all-reduce, so every
    rank takes the same branch (the leg holds collectives). Returns
    (ok, reason)."""
    if world <= 1:
        return True, ""
    import torch
    import torch.distributed as dist
    ok, why = host_room(need_bytes, int(os.environ.get("LOCAL_WORLD_SIZE", "1")), meminfo)
    f = torch.tensor([1 if ok else 0], device=device, dtype=torch.int32)
    dist.all_reduce(f, op=dist.ReduceOp.MIN)
    agreed = int(f.item()) == 1
    if ok and not agreed:
        why = "another rank's node lacks the host memory for its pinned arenas"
    return agreed, why


def layer_groups(states, budget_bytes=3 << 30):
    """Consecutive runs of layers whose input bytes stay within the budget
    (at least one layer each): the units the end-to-end leg streams."""
    groups, cur, size = [], [], 0
    for st in states:
        lo, hi = st.extra["in"]
        if cur and size + (hi - lo) > budget_bytes:
            groups.append(cur)
            cur, size = [], 0
        cur.append(st)
        size += hi - lo
    if cur:
        groups.append(cur)
    return groups


def e2e(states, arena_in, arena_out, device, steps, world, elements, masked_ste=False):
    """The same step through the public API with HOST buffers: every step
    copies all of its inputs (W, A, B, G and bf16 A, B of every layer, held in
    one pinned host arena) to the device, runs the path and copies every
    merged weight, scale, zero-point and gradient back (one pinned arena).

    The model is streamed as a caller merging it would run it: the layers go
    in consecutive groups of at most ~3 GB of inputs, each group's inputs
    travel host->device on one stream, its three stages run on a second (one
    batched call each) and its results travel device->host on a third, so
    group g+1 goes up while group g computes and group g-1 comes down. The
    device buffers are the ones the device-resident leg uses; every step
    moves all of its bytes both ways inside the timed region."""
    import torch
    import torch.distributed as dist
    from quantized_lora_merge_b200 import pipeline as P
    groups = layer_groups(states)
    paths = [P.Path(g, device, masked_ste=masked_ste) for g in groups]
    rng_in = [(g[0].extra["in"][0], g[-1].extra["in"][1]) for g in groups]
    rng_out = [(g[0].extra["out"][0], g[-1].extra["out"][1]) for g in groups]
    host_in, rel_in = pinned_host(arena_in.numel())
    host_out, rel_out = pinned_host(arena_out.numel())
    host_in.copy_(arena_in)
    h2d = sum(hi - lo for lo, hi in rng_in)
    d2h = sum(hi - lo for lo, hi in rng_out)
    s_h2d, s_run, s_d2h = (torch.cuda.Stream(device) for _ in range(3))
    ng = len(groups)
    copied_in = [torch.cuda.Event() for _ in range(ng)]
    computed = [torch.cuda.Event() for _ in range(ng)]
    copied_out = [torch.cuda.Event() for _ in range(ng)]
    used = [False] * ng

    def one_step():
        for g in range(ng):
            (ilo, ihi), (olo, ohi) = rng_in[g], rng_out[g]
            with torch.cuda.stream(s_h2d):
                if used[g]:
                    s_h2d.wait_event(computed[g])         # the last step has read them
                arena_in[ilo:ihi].copy_(host_in[ilo:ihi], non_blocking=True)
                copied_in[g].record(s_h2d)
            with torch.cuda.stream(s_run):
                s_run.wait_event(copied_in[g])
                if used[g]:
                    s_run.wait_event(copied_out[g])       # the last step's results are home
                paths[g].step(s_run)
                computed[g].record(s_run)
            with torch.cuda.stream(s_d2h):
                s_d2h.wait_event(computed[g])
                host_out[olo:ohi].copy_(arena_out[olo:ohi], non_blocking=True)
                copied_out[g].record(s_d2h)
            used[g] = True

    one_step()                                            # untimed
    torch.cuda.synchronize(device)
    if world > 1:
        dist.barrier()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(s_h2d)
    for _ in range(steps):
        one_step()
    s_d2h.wait_event(copied_out[ng - 1])
    b.record(s_d2h)
    torch.cuda.synchronize(device)
    ms = a.elapsed_time(b) / steps
    rel_in()
    rel_out()
    if world > 1:
        t = torch.tensor([ms], device=device, dtype=torch.float64)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms = float(t.item())
    return {"value": elements / (ms / 1000.0), "unit": UNIT, "ms_per_step": ms,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": steps,
            "pipelined": f"{ng} layer groups per step streamed over 3 streams (pinned host "
                         f"arenas, one copy per group and direction)"}


# ---------------------------------------------------------------------------
# integer inference GEMM on merged weights (--op int_gemm)
# ---------------------------------------------------------------------------
GEMM_METRIC = "integer GEMM on merged weights: tensor ops/s (int8 MMA), 1 GPU"
GEMM_UNIT = "Top/s"
# DiT-3072 block linears (qkv, attention out, fc1, fc2) as (d, n)
GEMM_SHAPES = [(9216, 3072), (3072, 3072), (12288, 3072), (3072, 12288)]
GEMM_KIND = {1: "shift4", 2: "mul4", 3: "mul8"}
GEMM_SOURCES = ("int_gemm_kernels.cu", "tcgen05_util.cuh", "intlora_kernels.h")


def bf16_peak_tflops():
    p = ROOT / "MEASURED_PEAKS.json"
    if p.exists():
        d = json.loads(p.read_text())
        for k in ("bf16_tflops", "bf16_tflops_burst"):
            if k in d:
                return float(d[k]), "measured"
    return 1590.0, "fallback"


def bench_int_gemm(args):
    """One step = the four DiT-3072 block GEMMs Y = X W'^T at `tokens` tokens
    (one batched call): int8 activations x merged integer weights held as
    `planes` int8 digit planes. Metric: int8 tensor ops per second executed
    (2 tokens d n planes per step); algorithmic ops (2 tokens d n) beside it."""
    import torch

    from quantized_lora_merge_b200 import binding as B
    from quantized_lora_merge_b200 import build as qbuild
    from quantized_lora_merge_b200 import workloads as wl
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1 and rank != 0:
        return
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    qbuild.build()
    P, T = args.planes, args.tokens
    bound = wl.INT_GEMM_BOUNDS[GEMM_KIND[P]]
    jobs, host = [], []
    for k, (d, n) in enumerate(GEMM_SHAPES):
        X, xs, Q, ws = wl.int_gemm_device(T, d, n, bound, device, salt=k)
        packed = torch.empty((d, P, n), dtype=torch.int8, device=device)
        B.intlora_int_pack(Q, P, packed)
        del Q
        jobs.append(B.IntGemmJob(X, xs, packed, ws, torch.empty(
            (T, d), dtype=torch.bfloat16 if args.y_bf16 else torch.float32, device=device)))
        host.append((d, n))
    desc_jobs = B.Descriptors(jobs)
    torch.cuda.synchronize(device)
    stream = torch.cuda.current_stream(device)
    tensor_ops = sum(2 * T * d * n * P for d, n in host)
    alg_ops = sum(2 * T * d * n for d, n in host)
    in_bytes = sum(T * n + d * n * P + 4 * (T + d) for d, n in host)
    out_bytes = sum((2 if args.y_bf16 else 4) * T * d for d, n in host)
    for _ in range(max(3, args.warmup)):
        B.intlora_int_gemm_batched(desc_jobs, P)
    torch.cuda.synchronize(device)
    steps = args.steps if args.steps != 1000 else 200
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(device)
    a.record(stream)
    for _ in range(steps):
        B.intlora_int_gemm_batched(desc_jobs, P)
    b.record(stream)
    torch.cuda.synchronize(device)
    clk = clocks.stop()
    ms = a.elapsed_time(b) / steps
    achieved = tensor_ops / (ms / 1e3) / 1e12
    bf16, kind = bf16_peak_tflops()
    peak = 2.0 * bf16                       # int8 dense = 2 x bf16 dense (nominal ratio)
    # end to end: X from pinned host memory, Y back, through the same call
    hx = [torch.empty_like(j.X, device="cpu").pin_memory() for j in jobs]
    hy = [torch.empty_like(j.Y, device="cpu").pin_memory() for j in jobs]
    for h, j in zip(hx, jobs):
        h.copy_(j.X)
    e2e_steps = 5
    ea = torch.cuda.Event(enable_timing=True)
    eb = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(device)
    ea.record(stream)
    for _ in range(e2e_steps):
        for h, j in zip(hx, jobs):
            j.X.copy_(h, non_blocking=True)
        B.intlora_int_gemm_batched(desc_jobs, P)
        for h, j in zip(hy, jobs):
            h.copy_(j.Y, non_blocking=True)
    eb.record(stream)
    torch.cuda.synchronize(device)
    e2e_ms = ea.elapsed_time(eb) / e2e_steps
    line = {
        "metric": GEMM_METRIC, "value": achieved, "unit": GEMM_UNIT, "n_gpus": 1,
        "steps": steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "s8 x s8 -> s32", "data": "synthetic",
        "config": {"workload": f"DiT-3072 block linears (qkv 9216x3072, out 3072x3072, fc1 "
                               f"12288x3072, fc2 3072x12288) at {T} tokens, W'={GEMM_KIND[P]} "
                               f"merged weights as {P} int8 digit plane(s), int8 activations",
                   "tokens": T, "planes": P, "y": "bf16" if args.y_bf16 else "fp32",
                   "l2": f"inputs {in_bytes / 1e6:.0f} MB + outputs {out_bytes / 1e6:.0f} MB per "
                         f"step, larger than L2"},
        "algorithmic_Top_s": alg_ops / (ms / 1e3) / 1e12,
        "roofline": {"bound": "tensor", "kernel": "int_gemm_kernel (tcgen05 kind::i8)",
                     "achieved": achieved, "peak": peak, "unit": "Top/s",
                     "frac": achieved / peak,
                     "peak_source": f"2 x {kind} bf16 dense {bf16:.0f} TFLOP/s (int8/bf16 "
                                    f"nominal ratio 4.5/2.25)",
                     "traffic": profiled_traffic(f"int_gemm_kernel_dit_{GEMM_KIND[P]}",
                                                 GEMM_SOURCES),
                     "traffic_unit": "bytes per launch (one step)"},
        "clocks": clk, "gpu_launches": steps,
        "e2e": {"value": tensor_ops / (e2e_ms / 1e3) / 1e12, "unit": GEMM_UNIT,
                "ms_per_step": e2e_ms,
                "h2d_bytes_per_step": sum(j.X.numel() for j in jobs),
                "d2h_bytes_per_step": sum(j.Y.element_size() * j.Y.numel() for j in jobs)},
    }
    if not args.no_cpu_baseline:
        import numpy as np

        import oracle
        X0, xs0, Q0, ws0 = wl.int_gemm_host(T, *GEMM_SHAPES[0], bound)
        t0 = time.perf_counter()
        rows, done = 0, 0
        while time.perf_counter() - t0 < min(args.cpu_seconds, 10.0) and rows < T:
            oracle.int_gemm_rows(X0, xs0.astype(np.float64), Q0, ws0.astype(np.float64),
                                 np.arange(rows, rows + 4))
            rows += 4
        dt = time.perf_counter() - t0
        done = 2 * rows * GEMM_SHAPES[0][0] * GEMM_SHAPES[0][1]
        line["cpu_baseline"] = {"value": done / dt / 1e12, "unit": "Top/s (algorithmic)",
                                "cores": oracle.num_threads(), "kind": "oracle",
                                "sample": f"{rows} token rows of the qkv GEMM "
                                          f"({GEMM_SHAPES[0][0]}x{GEMM_SHAPES[0][1]}), "
                                          f"exact int64 sums, {dt:.1f} s"}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# training forward on merged weights (--op train_forward)
# ---------------------------------------------------------------------------
def bench_train_forward(args):
    """One step = the training forward of every SD-UNet linear at `tokens`
    tokens: the MUL merge (all layers, one batched call), the bf16
    fake-quantization of the merged weights, and Y = X W'^T for every layer
    (batched bf16 GEMMs on the tensor cores). Metric: GEMM TFLOP/s of the
    whole step (2 tokens d n per layer over the step time)."""
    import torch

    from quantized_lora_merge_b200 import binding as B
    from quantized_lora_merge_b200 import build as qbuild
    from quantized_lora_merge_b200 import pipeline as P
    from quantized_lora_merge_b200 import workloads as wl
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1 and rank != 0:
        return
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    qbuild.build()
    T = args.tokens
    layers = wl.CONFIGS["sd_unet"]()
    states = []
    for spec in layers:
        t = wl.device_inputs(spec, device, salt=0)
        states.append(P.allocate(spec, t["W"], t["A"], t["B"], device))
    path = P.Path(states, device)
    path.prepare()
    g = torch.Generator(device=device)
    g.manual_seed(11)
    wq = [torch.empty(l.d, l.n, dtype=torch.bfloat16, device=device) for l in layers]
    # activations and outputs in bf16 (a training forward's layer outputs)
    lin = B.Descriptors(B.LinearJob(torch.randn(T, l.n, generator=g, device=device).to(torch.bfloat16),
                                    w, torch.empty(T, l.d, dtype=torch.bfloat16, device=device))
                        for l, w in zip(layers, wq))
    stream = torch.cuda.current_stream(device)

    fq = B.Descriptors(B.FakeQuantJob(st.out, st.sbar, w) for st, w in zip(states, wq))

    def step():
        path.merge()
        B.intlora_fakequant_bf16_batched(fq)
        B.intlora_linear_bf16_batched(lin)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize(device)
    steps = args.steps if args.steps != 1000 else 20
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    gemm_ms = 0.0
    torch.cuda.synchronize(device)
    a.record(stream)
    for _ in range(steps):
        path.merge()
        ev[0].record(stream)
        B.intlora_fakequant_bf16_batched(fq)
        ev[1].record(stream)
        B.intlora_linear_bf16_batched(lin)
        ev[2].record(stream)
        ev[2].synchronize()
        gemm_ms += ev[1].elapsed_time(ev[2])
    b.record(stream)
    torch.cuda.synchronize(device)
    clk = clocks.stop()
    ms = a.elapsed_time(b) / steps
    gemm_ms /= steps
    flops = sum(2 * T * l.d * l.n for l in layers)
    bf16, kind = bf16_peak_tflops()
    gemm_tf = flops / (gemm_ms / 1e3) / 1e12
    line = {
        "metric": "training forward on merged weights: GEMM TFLOP/s per step (bf16), 1 GPU",
        "value": flops / (ms / 1e3) / 1e12, "unit": "TFLOP/s", "n_gpus": 1, "steps": steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16 x bf16 -> f32", "data": "synthetic",
        "config": {"workload": f"SD-UNet 128 linears at {T} tokens: MUL merge (4-bit) + bf16 "
                               f"fake-quantization + Y = X W'^T per layer (bf16 X and Y)",
                   "tokens": T},
        "gemm_ms": gemm_ms,
        "roofline": {"bound": "tensor", "kernel": "int_gemm_kernel<0> (tcgen05 kind::f16)",
                     "achieved": gemm_tf, "peak": bf16, "unit": "TFLOP/s", "frac": gemm_tf / bf16,
                     "peak_source": f"{kind} bf16 dense", "traffic": None},
        "clocks": clk,
        "gpu_launches": steps * (2 + (len(layers) + 47) // 48),
    }
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
