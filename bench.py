#!/usr/bin/env python
"""Benchmark of the Krea 2 backbone forward on B200 (sm_100a).

A step is one full backbone forward (every step of the path: RoPE tables, time path, img_in,
28 single-stream blocks, final layer) at 1024^2: batch 1, 512 text + 64x64 = 4096 image
tokens, bf16 with fp32 residual. The metric is algorithmic TFLOP/s (GEMM FLOPs 2*M*N*K of the
projections plus attention FLOPs 4*D*H*S*S_valid over valid keys). The same run also times
the 1024^2 CFG block (batch 2, uncond row with 8 valid text tokens), per-kernel durations with
CUDA events, an end-to-end pass through host buffers, and the CPU oracle on a bounded sample.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl native|reference]

Multi-GPU runs are replicas: each rank runs its own step with no data-path collective; time is
the max over ranks. Under torchrun WORLD_SIZE must equal --gpus; without a launcher, --gpus N > 1
starts the N ranks itself (one process per GPU, rendezvous on 127.0.0.1).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import krea2_inputs as KI  # noqa: E402

METRIC = "Krea2 block fwd bf16 TFLOP/s (% tensor peak); backbone ms/step at 1024²"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.json")
FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ----------------------------------------------------------------------------- work accounting

def block_kernel_work(d: KI.Dims, B: int, T: int, N: int, lengths) -> dict:
    """Algorithmic FLOPs (tensor kernels) or bytes (row kernels) of one block's launches."""
    S = T + N
    M = B * S
    QC = d.qkvg_cols
    valid = [(lengths[b] if T else 0) + N for b in range(B)]
    return {
        "modulation": {"bytes": B * 6 * d.C * 4 * 3},
        "norm1": {"bytes": M * d.C * (4 + 2)},
        "qkv_proj": {"flops": 2 * M * d.C * QC},
        "attention": {"flops": 4 * d.D * d.H * sum(S * v for v in valid)},
        "out_proj_resid": {"flops": 2 * M * d.HD * d.C},
        "norm2": {"bytes": M * d.C * (4 + 2)},
        "gate_up_swiglu": {"flops": 2 * M * d.C * 2 * d.F},
        "down_proj_resid": {"flops": 2 * M * d.F * d.C},
    }


def block_flops(d, B, T, N, lengths) -> float:
    return float(sum(v.get("flops", 0) for v in block_kernel_work(d, B, T, N, lengths).values()))


def backbone_flops(d, B, T, N, lengths) -> float:
    extra = 2 * B * (d.t_dim * d.C + d.C * d.C + d.C * 6 * d.C) + 2 * B * N * d.in_ch * d.C * 2
    return d.n_layers * block_flops(d, B, T, N, lengths) + extra


def oracle_block_flops(d, B, S, R, valid) -> float:
    """FLOPs of one oracle block computing R sampled query rows per batch row (all keys)."""
    M = B * S
    kv = 2 * M * d.C * 2 * d.KVD
    qg = 2 * B * R * d.C * 2 * d.HD
    attn = 4 * d.D * d.H * R * sum(valid)
    out = 2 * B * R * d.HD * d.C
    mlp = 2 * B * R * d.C * 2 * d.F + 2 * B * R * d.F * d.C
    return float(kv + qg + attn + out + mlp)


def peaks() -> dict:
    try:
        with open(PEAKS_FILE) as f:
            p = json.load(f)
        return {"hbm_gbs": p["hbm_gbs"], "bf16_tflops": p["bf16_tflops"],
                "bf16_tflops_sustained": p["bf16_tflops_sustained"], "source": "measured"}
    except (OSError, KeyError, ValueError):
        return dict(FALLBACK, source="fallback")


# Source files that fix each block step's kernel and its launch shape. A recorded DRAM figure
# is only valid while these files are unchanged.
_GEMM_SOURCES = ("gemm_tcgen05.cu", "krea2_device.cuh", "krea2_internal.h")
KERNEL_SOURCES = {
    "qkv_proj": _GEMM_SOURCES, "out_proj_resid": _GEMM_SOURCES, "gate_up_swiglu": _GEMM_SOURCES,
    "down_proj_resid": _GEMM_SOURCES,
    "attention": ("attention_tc.cu", "krea2_device.cuh", "krea2_internal.h"),
}


def kernel_source_hash(kernel: str) -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "flow_matching_stream_b200", "csrc")
    for name in sorted(KERNEL_SOURCES[kernel]):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str):
    """DRAM bytes per launch from a committed ncu summary, if it matches the current kernel sources."""
    try:
        with open(TRAFFIC_FILE) as f:
            rec = json.load(f).get("kernels", {}).get(kernel)
    except (OSError, ValueError):
        return None
    if not rec or kernel not in KERNEL_SOURCES or rec.get("source_hash") != kernel_source_hash(kernel):
        return None
    return rec.get("dram_bytes_per_launch")


def record_traffic(entries) -> None:
    """Store ncu DRAM bytes per launch (read + write) for block steps, stamped with their source hash.

    entries: "kernel=bytes[:profile]" strings, profile naming the summary under profiles/."""
    try:
        with open(TRAFFIC_FILE) as f:
            t = json.load(f)
    except (OSError, ValueError):
        t = {}
    t["_source"] = ("dram__bytes_read.sum + dram__bytes_write.sum per launch from ncu captures at the "
                    "backbone block shape; an entry is valid only while its kernel sources hash to source_hash")
    kernels = t.setdefault("kernels", {})
    for e in entries:
        name, rest = e.split("=", 1)
        nbytes, _, profile = rest.partition(":")
        if name not in KERNEL_SOURCES:
            raise SystemExit(f"unknown block step {name!r}; one of {sorted(KERNEL_SOURCES)}")
        kernels[name] = {"dram_bytes_per_launch": int(nbytes), "source_hash": kernel_source_hash(name)}
        if profile:
            kernels[name]["profile"] = profile
    t.pop("source_hash", None)
    with open(TRAFFIC_FILE, "w") as f:
        json.dump(t, f, indent=1, sort_keys=True)
        f.write("\n")


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        import torch
        self.ident = str(device_index)
        try:
            self.ident = "GPU-" + str(torch.cuda.get_device_properties(device_index).uuid)
        except Exception:
            pass
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-lms", "200", "-i", self.ident], stdout=subprocess.PIPE,
                                         stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=10)
        sm, mx, pw, reasons = [], [], [], set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
                pw.append(float(parts[2]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[3:7]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "power_w_median": float(np.median(pw)) if pw else None, "reasons": sorted(reasons),
                "samples": len(sm)}


# ----------------------------------------------------------------------------- oracle (CPU)

class OracleSample:
    """The CPU oracle (numpy fp32, fp64 softmax) on one block of the backbone workload, computing
    `rows` sampled query rows over all keys. Inputs are generated once; run() is timed."""

    def __init__(self, rows: int):
        from oracle import krea2_oracle as O
        self.O = O
        wl = KI.backbone_1024()
        self.d = d = wl.dims
        self.wl = wl
        self.h = KI.residual(d, wl.B, wl.S)
        self.temb = KI.temb(d, wl.B)
        self.w = KI.block_weights(d, 0)
        self.c, self.s = O.rope_cos_sin(wl.positions(), d.axes, d.theta)
        self.kv = O.key_valid_mask(wl.mask(), wl.B, wl.T, wl.N)
        self.rows = rows
        self.sel = np.linspace(0, wl.S - 1, rows).astype(int)
        valid = [int(self.kv[b].sum()) for b in range(wl.B)]
        self.flops = oracle_block_flops(d, wl.B, wl.S, rows, valid)

    def run(self) -> float:
        d = self.d
        t0 = time.perf_counter()
        self.O.block_forward(self.h, self.temb, self.w, self.c, self.s, self.kv, d.H, d.Hkv, d.D, d.eps,
                             rows=self.sel, dtype=np.float32)
        return time.perf_counter() - t0

    def describe(self, seconds: float) -> str:
        return (f"one block of the 1024^2 backbone workload (S=4608, C=6144), {self.rows} sampled query rows "
                f"over all keys, numpy fp32 + fp64 softmax: {self.flops / 1e9:.0f} GFLOP in {seconds:.2f} s")


def cpu_oracle_sample(rows: int = 4096) -> dict:
    """About 10 s of the oracle on 16 host cores (the GEMM rows dominate; K/V of all keys are
    computed once per sample)."""
    o = OracleSample(rows)
    dt = o.run()
    return {"value": o.flops / dt / 1e12, "unit": "TFLOP/s", "cores": len(os.sched_getaffinity(0)),
            "kind": "oracle", "sample": o.describe(dt)}


# ----------------------------------------------------------------------------- replicas

def max_over_ranks(x: float, world: int, device) -> float:
    """Max of a per-rank number over all ranks (timing is the slowest replica's)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_throughput(world: int, steps: int, flops_per_step: float, ms_max: float) -> float:
    """Whole-job TFLOP/s of `world` replicas that each ran `steps` steps in at most `ms_max` ms."""
    return world * steps * flops_per_step / (ms_max / 1e3) / 1e12


def workload_config(wl: KI.Workload, world: int) -> dict:
    """The `config` object both arms print for the backbone workload."""
    d = wl.dims
    return {"workload": wl.name, "batch": wl.B, "text_tokens": wl.T, "image_tokens": wl.N, "seq_len": wl.S,
            "layers": d.n_layers, "hidden": d.C, "heads": f"{d.H}q/{d.Hkv}kv x {d.D}", "intermediate": d.F,
            "weights": "random-init N(0,1)/sqrt(fan_in), seeded, ~12.2 B params bf16",
            "l2": "inputs larger than L2: 24 GB of block weights stream from HBM every step",
            "parallelism": "replicas" if world > 1 else "single GPU",
            "flops_per_step": backbone_flops(d, wl.B, wl.T, wl.N, wl.lengths)}


# ----------------------------------------------------------------------------- native arm

def run_native(args, rank: int, world: int, local_rank: int) -> None:
    import torch
    import torch.distributed as dist

    import flow_matching_stream_b200 as K2

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=600), device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier(device_ids=[local_rank])

    warmup = max(args.warmup, 3)
    wl = KI.backbone_1024()
    d = wl.dims
    B, T, N, S = wl.B, wl.T, wl.N, wl.S
    dt = torch.bfloat16
    gen = torch.Generator(device=dev).manual_seed(1234 + 0)  # same weights on every replica
    blocks = [K2.BlockWeights.random(d, dt, dev, gen) for _ in range(d.n_layers)]
    mw = K2.ModelWeights(KI.model_weights(d), blocks, dt, dev)

    hidden_h = torch.from_numpy(KI.latents(d, B, N)).to(dt).pin_memory()
    text_h = torch.from_numpy(KI.text_states(d, B, T)).to(dt).pin_memory()
    pos_h = torch.from_numpy(wl.positions()).pin_memory()
    mask_h = torch.from_numpy(wl.mask().astype(np.uint8)).pin_memory()
    t_h = torch.from_numpy(KI.timesteps(B)).pin_memory()
    vel_h = torch.empty(B, N, d.in_ch, dtype=dt).pin_memory()
    hidden, text, pos, mask, tt = (x.to(dev) for x in (hidden_h, text_h, pos_h, mask_h, t_h))
    vel = torch.empty(B, N, d.in_ch, device=dev, dtype=dt)
    ws = torch.empty(K2.workspace_size(d, B, T, N, dt), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def step():
        K2.backbone_forward(d, B, T, N, hidden, text, pos, mask, tt, mw, vel, ws)

    for _ in range(warmup):
        step()
    K2.check_device_error()

    # ---- timed region: K backbone steps, inputs resident in HBM
    clocks = ClockSampler(local_rank)
    clocks.start()
    barrier()
    torch.cuda.synchronize()
    l0 = K2.launch_count()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    launches = K2.launch_count() - l0
    clk = clocks.stop()
    K2.check_device_error()
    ms_total = max_over_ranks(e0.elapsed_time(e1), world, dev)
    flops_step = backbone_flops(d, B, T, N, wl.lengths)
    value = replica_throughput(world, args.steps, flops_step, ms_total)
    ms_step = ms_total / args.steps

    # ---- end to end through host buffers: H2D of the step's inputs, forward, D2H of velocity
    h2d = sum(x.numel() * x.element_size() for x in (hidden_h, text_h, pos_h, mask_h, t_h))
    d2h = vel_h.numel() * vel_h.element_size()

    def e2e_step():
        for dst, src in ((hidden, hidden_h), (text, text_h), (pos, pos_h), (mask, mask_h), (tt, t_h)):
            dst.copy_(src, non_blocking=True)
        step()
        vel_h.copy_(vel, non_blocking=True)

    for _ in range(2):
        e2e_step()
    barrier()
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(args.steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    e2e_value = replica_throughput(world, args.steps, flops_step, e2e_ms)

    # ---- per-kernel durations (CUDA events on the launching stream) at the backbone's block shape
    pk = peaks()
    kernels = traced_block_kernels(K2, torch, d, B, T, N, wl.lengths, blocks[0], dev, reps=max(args.steps, 5))
    dom = max((k for k in kernels if "tflops" in kernels[k]), key=lambda k: kernels[k]["ms"])
    dk = kernels[dom]
    roofline = {"kernel": dom, "bound": "tensor", "achieved": dk["tflops"], "peak": pk["bf16_tflops_sustained"],
                "unit": "TFLOP/s", "frac": dk["tflops"] / pk["bf16_tflops_sustained"],
                "traffic": recorded_traffic(dom), "peak_source": f"{pk['source']} sustained bf16 (kernel timed "
                                                                   f"inside back-to-back blocks)",
                "frac_of_burst": dk["tflops"] / pk["bf16_tflops"]}

    # ---- the 1024^2 CFG block (batch 2: cond all 512 text valid, uncond 8 valid)
    cfg = KI.block_1024_cfg()
    cfg_res = time_block(K2, torch, cfg, dev, args.steps, warmup, pk)

    sampler = time_sampler(K2, torch, d, mw, dev)
    text = time_text_fusion(K2, torch, dev, args.steps)
    sweep = time_attention_sweep(K2, torch, dev, args.steps, pk)
    kv_step = time_kv_cache_step(K2, torch, dev, args.steps, pk)

    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": workload_config(wl, world),
        "backbone_ms_per_step": ms_step,
        "sampler_1024sq": sampler,
        "text_fusion_once_per_prompt": text,
        "attention_sweep": sweep,
        "kv_cache_step_attention": kv_step,
        "pct_of_tensor_peak": {"burst": value / world / pk["bf16_tflops"],
                               "sustained": value / world / pk["bf16_tflops_sustained"]},
        "block_1024sq_cfg": cfg_res,
        "kernels": kernels,
        "roofline": roofline,
        "e2e": {"value": e2e_value, "unit": "TFLOP/s", "ms_per_step": e2e_ms / args.steps,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": int(launches),
        "gpu_launches_per_step": int(launches) // max(args.steps, 1),
        "clocks": clk,
        "peaks": pk,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_oracle_sample()
    # last key: the figures the metric names, compact, so that the end of the line carries them
    line["summary"] = summary(value / world, ms_step, pk, cfg_res, kernels, sweep)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


def _r(x: float, sig: int = 4) -> float:
    return float(f"{x:.{sig}g}")


def summary(tflops_per_gpu: float, ms_step: float, pk: dict, cfg_res: dict, kernels: dict, sweep: list) -> dict:
    """Compact figures for the end of the JSON line: the backbone step, the 1024^2 CFG block
    (config 3) with its per-kernel fractions, attention's in-block share and the attention sweep."""
    cfg_k = cfg_res["kernels"]
    ker = {k: [_r(v["ms"]), _r(v["tflops"] if "tflops" in v else v["gbs"]),
               _r(v["frac_sustained"] if "frac_sustained" in v else v["frac_hbm"], 3)]
           for k, v in cfg_k.items() if k != "modulation"}
    return {
        "backbone_1024sq": {"ms_per_step": _r(ms_step), "tflops": _r(tflops_per_gpu),
                            "frac_burst": _r(tflops_per_gpu / pk["bf16_tflops"], 3),
                            "attention_share": _r(kernels["attention"]["share"], 3),
                            "attention_frac_sustained": _r(kernels["attention"]["frac_sustained"], 3)},
        "block_1024sq_cfg": {"ms": _r(cfg_res["ms_per_block"]), "tflops": _r(cfg_res["tflops"]),
                             "frac_burst": _r(cfg_res["frac_burst"], 3),
                             "frac_sustained": _r(cfg_res["frac_sustained"], 3),
                             "kernels_ms_tflops_or_gbs_frac": ker},
        "attention_sweep_grid_ms_tflops": [[s["grid"], _r(s["ms"]), _r(s["tflops"])] for s in sweep],
        "peaks_source": pk["source"],
    }


def time_sampler(K2, torch, d, mw, dev) -> dict:
    """The device sampling loop (krea2_sample) at 1024^2 for both presets of the pages: 8 steps
    without guidance at mu = 1.15 (distilled) and 28 steps with guidance 4.5 at the resolution mu
    (one batch-2 [cond, uncond] forward per step). Timed eagerly and as a CUDA graph replay."""
    T, gh, gw = 512, 64, 64
    N = gh * gw
    g = torch.Generator(device=dev).manual_seed(9)
    text_c = torch.randn(T, d.C, device=dev, generator=g).to(torch.bfloat16)
    text_u = torch.randn(T, d.C, device=dev, generator=g).to(torch.bfloat16)
    mask_c = torch.ones(T, dtype=torch.uint8, device=dev)
    mask_u = torch.zeros(T, dtype=torch.uint8, device=dev)
    mask_u[:8] = 1  # empty negative prompt: a handful of valid tokens
    pos = torch.from_numpy(KI.position_ids(T, gh, gw)).to(dev)
    lat0 = torch.randn(N, d.in_ch, device=dev, generator=g)
    out = {}
    for name, steps, guidance, mu in (("8_step_distilled", 8, 0.0, 1.15),
                                      ("28_step_cfg_4.5", 28, 4.5, K2.shift_mu(N))):
        sig = K2.sigma_schedule(steps, mu)
        ws = torch.empty(K2.sample_workspace_size(d, T, N, torch.bfloat16, guidance > 0), dtype=torch.uint8,
                         device=dev)
        lat = lat0.clone()

        def run():
            lat.copy_(lat0)
            K2.sample(d, T, N, lat, text_c, text_u, mask_c, mask_u, pos, sig, guidance, mw, ws)

        run()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        run()
        e1.record()
        torch.cuda.synchronize()
        eager = e0.elapsed_time(e1)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            run()
        torch.cuda.synchronize()
        e0.record()
        graph.replay()
        e1.record()
        torch.cuda.synchronize()
        K2.check_device_error()
        replay = e0.elapsed_time(e1)
        finite = bool(torch.isfinite(lat).all().item())
        del graph
        out[name] = {"steps": steps, "guidance": guidance, "mu": mu, "eager_s": eager / 1e3,
                     "graph_replay_s": replay / 1e3, "ms_per_sampler_step": replay / steps,
                     "forwards_per_step": 2 if guidance > 0 else 1, "finite": finite}
    return out


def time_text_fusion(K2, torch, dev, steps: int) -> dict:
    """Text conditioning once per prompt at the pages' sizes: a [cond, uncond] batch of 512 tokens
    x 12 stacked layers x 2560, 2 layerwise + 2 refiner blocks, txt_in to 6144."""
    td = KI.FULL_TEXT
    B, T = 2, 512
    g = torch.Generator(device=dev).manual_seed(13)
    bd = td.block_dims()
    rnd = lambda *sh, sc=1.0: (torch.randn(*sh, device=dev, generator=g) * sc)

    def block():
        C, HD, KVD, F, D = bd.C, bd.HD, bd.KVD, bd.F, bd.D
        return {"wq": rnd(HD, C, sc=C ** -0.5), "wk": rnd(KVD, C, sc=C ** -0.5), "wv": rnd(KVD, C, sc=C ** -0.5),
                "wg": rnd(HD, C, sc=C ** -0.5), "wo": rnd(C, HD, sc=HD ** -0.5), "w_gate": rnd(F, C, sc=C ** -0.5),
                "w_up": rnd(F, C, sc=C ** -0.5), "w_down": rnd(C, F, sc=F ** -0.5), "norm1_w": rnd(C, sc=0.1),
                "norm2_w": rnd(C, sc=0.1), "q_norm_w": rnd(D, sc=0.1), "k_norm_w": rnd(D, sc=0.1)}
    tw = K2.TextWeights({"layerwise": [block() for _ in range(td.n_layerwise)],
                         "refiner": [block() for _ in range(td.n_refiner)], "layer_w": rnd(td.L, sc=td.L ** -0.5),
                         "txt_in_w": rnd(td.C, td.Dt, sc=td.Dt ** -0.5), "txt_in_b": rnd(td.C, sc=0.1)},
                        torch.bfloat16, dev)
    ehs = rnd(B, T, td.L, td.Dt).to(torch.bfloat16)
    mask = torch.ones(B, T, dtype=torch.uint8, device=dev)
    mask[1, 8:] = 0
    out = torch.empty(B, T, td.C, device=dev, dtype=torch.bfloat16)
    ws = torch.empty(K2.text_fusion_workspace_size(td, B, T, torch.bfloat16), dtype=torch.uint8, device=dev)
    for _ in range(2):
        K2.text_fusion(td, B, T, ehs, mask, tw, out, ws)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        K2.text_fusion(td, B, T, ehs, mask, tw, out, ws)
    e1.record()
    torch.cuda.synchronize()
    K2.check_device_error()
    ms = e0.elapsed_time(e1) / steps
    # GEMM FLOPs of the four fusion blocks (B*T*L rows for the layerwise ones) plus txt_in
    per_row = 2 * bd.C * (bd.qkvg_cols + bd.HD + 2 * bd.F + bd.F)
    fl = per_row * (td.n_layerwise * B * T * td.L + td.n_refiner * B * T) + 2 * B * T * td.Dt * td.C
    return {"workload": "text_fusion_2x512x12x2560", "ms": ms, "gemm_tflops": fl / (ms / 1e3) / 1e12}


def time_attention_sweep(K2, torch, dev, steps: int, pk: dict) -> list:
    """The attention-only sweep: 48 q / 12 kv heads x 128 with 512 text tokens (random valid
    length) and 32^2 .. 128^2 image grids, through krea2_gqa_attention (q/k norm + RoPE pass and
    the flash-attention kernel). FLOPs count valid keys only."""
    out = []
    for grid in (32, 64, 96, 128):
        wl = KI.attn_sweep(grid)
        d = wl.dims
        B, T, N, S = wl.B, wl.T, wl.N, wl.S
        g = torch.Generator(device=dev).manual_seed(grid)
        x = torch.randn(B * S, d.qkvg_cols, device=dev, generator=g).to(torch.bfloat16)
        qw = torch.randn(d.D, device=dev, generator=g) * 0.1
        kw = torch.randn(d.D, device=dev, generator=g) * 0.1
        cs = torch.empty(S, d.D // 2, device=dev)
        sn = torch.empty_like(cs)
        K2.rope_tables(d, torch.from_numpy(wl.positions()).to(dev), cs, sn)
        mask = torch.from_numpy(wl.mask().astype(np.uint8)).to(dev)
        o = torch.empty(B * S, d.HD, device=dev, dtype=torch.bfloat16)
        ws = torch.empty(K2.attention_workspace_size(d, B, T, N, torch.bfloat16), dtype=torch.uint8, device=dev)
        run = lambda: K2.gqa_attention(d, B, T, N, x, qw, kw, cs, sn, mask, o, ws)
        for _ in range(3):
            run()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(steps):
            run()
        e1.record()
        torch.cuda.synchronize()
        K2.check_device_error()
        ms = e0.elapsed_time(e1) / steps
        fl = 4.0 * d.D * d.H * S * (wl.lengths[0] + N)
        out.append({"grid": grid, "tokens": S, "valid_text": wl.lengths[0], "ms": ms,
                    "tflops": fl / (ms / 1e3) / 1e12, "frac_burst": fl / (ms / 1e3) / 1e12 / pk["bf16_tflops"]})
        del x, o, ws
    return out


def kv_step_flops(d, Nq: int, valid_keys: int) -> float:
    """Attention FLOPs of Nq new queries over the valid cached + new keys (per batch row)."""
    return 4.0 * d.D * d.H * Nq * valid_keys


def time_kv_cache_step(K2, torch, dev, steps: int, pk: dict) -> dict:
    """One denoising step's attention of the block-causal variant with a key/value cache: the
    prompt (512 text tokens, random valid length) and a 64x64 condition image are cached once;
    each step appends the 64x64 target image's keys and values and runs its 4096 queries over all
    8704 keys (krea2_kv_cache_append + krea2_gqa_attention_kv_cache). FLOPs count valid keys only."""
    wl = KI.backbone_1024()
    d = wl.dims
    T, Ni = wl.T, wl.N
    P, Nq = T + Ni, Ni
    L = P + Nq
    g = torch.Generator(device=dev).manual_seed(31)
    x = torch.randn(L, d.qkvg_cols, device=dev, generator=g).to(torch.bfloat16)
    qw = torch.randn(d.D, device=dev, generator=g) * 0.1
    kw = torch.randn(d.D, device=dev, generator=g) * 0.1
    pos = np.concatenate([KI.position_ids(T, 64, 64), KI.position_ids(0, 64, 64)]).astype(np.float32)
    pos[P:, 0] = 1.0  # the target image sits one step along the first axis
    cs = torch.empty(L, d.D // 2, device=dev)
    sn = torch.empty_like(cs)
    K2.rope_tables(d, torch.from_numpy(pos).to(dev), cs, sn)
    mask = torch.from_numpy(wl.mask().astype(np.uint8)).to(dev)
    kc = torch.empty(1, L, d.KVD, device=dev, dtype=torch.bfloat16)
    vc = torch.empty_like(kc)
    x_prefix, x_new = x[:P].contiguous(), x[P:].contiguous()
    K2.kv_cache_append(d, 1, P, 0, x_prefix, kw, cs[:P], sn[:P], kc, vc)
    o = torch.empty(Nq, d.HD, device=dev, dtype=torch.bfloat16)
    ws = torch.empty(K2.kv_cache_attention_workspace_size(d, 1, Nq, torch.bfloat16), dtype=torch.uint8, device=dev)
    cs_new, sn_new = cs[P:].contiguous(), sn[P:].contiguous()

    def run():
        K2.kv_cache_append(d, 1, Nq, P, x_new, kw, cs_new, sn_new, kc, vc)
        K2.gqa_attention_kv_cache(d, 1, T, L, Nq, x_new, qw, cs_new, sn_new, mask, kc, vc, None, o, ws)

    for _ in range(3):
        run()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        run()
    e1.record()
    torch.cuda.synchronize()
    K2.check_device_error()
    ms = e0.elapsed_time(e1) / steps
    fl = kv_step_flops(d, Nq, int(wl.lengths[0]) + Ni + Nq)
    return {"workload": "block-causal step with cached prompt + 64x64 condition image, 64x64 target",
            "new_tokens": Nq, "keys": L, "valid_text": int(wl.lengths[0]), "ms": ms,
            "tflops": fl / (ms / 1e3) / 1e12, "frac_burst": fl / (ms / 1e3) / 1e12 / pk["bf16_tflops"]}


def traced_block_kernels(K2, torch, d, B, T, N, lengths, bw, dev, reps: int) -> dict:
    S = T + N
    pk = peaks()
    h = torch.randn(B * S, d.C, device=dev)
    temb = torch.randn(B, 6 * d.C, device=dev) * 0.5
    pos = torch.from_numpy(KI.position_ids(T, int(np.sqrt(N)), N // int(np.sqrt(N)))).to(dev)
    cs = torch.empty(S, d.D // 2, device=dev)
    sn = torch.empty_like(cs)
    K2.rope_tables(d, pos, cs, sn)
    mask = torch.from_numpy(KI.mask_from_lengths(T, lengths).astype(np.uint8)).to(dev) if T else None
    ws = torch.empty(K2.workspace_size(d, B, T, N, torch.bfloat16), dtype=torch.uint8, device=dev)
    runs = [[torch.cuda.Event(enable_timing=True) for _ in range(9)] for _ in range(reps)]
    for _ in range(3):
        K2.block_forward(d, B, T, N, h, temb, bw, cs, sn, mask, ws)
    for ev in runs:
        K2.block_forward_traced(d, B, T, N, h, temb, bw, cs, sn, mask, ws, ev)
    torch.cuda.synchronize()
    K2.check_device_error()
    work = block_kernel_work(d, B, T, N, lengths)
    out = {}
    for i, name in enumerate(K2.BLOCK_STEPS):
        ms = float(np.mean([ev[i].elapsed_time(ev[i + 1]) for ev in runs]))
        r = {"ms": ms}
        if "flops" in work[name]:
            r["tflops"] = work[name]["flops"] / (ms / 1e3) / 1e12
            r["frac_sustained"] = r["tflops"] / pk["bf16_tflops_sustained"]
        else:
            r["gbs"] = work[name]["bytes"] / (ms / 1e3) / 1e9
            r["frac_hbm"] = r["gbs"] / pk["hbm_gbs"]
        out[name] = r
    total = sum(v["ms"] for v in out.values())
    for v in out.values():
        v["share"] = v["ms"] / total
    return out


def time_block(K2, torch, wl: KI.Workload, dev, steps: int, warmup: int, pk: dict) -> dict:
    d = wl.dims
    gen = torch.Generator(device=dev).manual_seed(77)
    bw = K2.BlockWeights.random(d, torch.bfloat16, dev, gen)
    B, T, N, S = wl.B, wl.T, wl.N, wl.S
    h = torch.randn(B * S, d.C, device=dev)
    temb = torch.randn(B, 6 * d.C, device=dev) * 0.5
    pos = torch.from_numpy(wl.positions()).to(dev)
    cs = torch.empty(S, d.D // 2, device=dev)
    sn = torch.empty_like(cs)
    K2.rope_tables(d, pos, cs, sn)
    mask = torch.from_numpy(wl.mask().astype(np.uint8)).to(dev)
    ws = torch.empty(K2.workspace_size(d, B, T, N, torch.bfloat16), dtype=torch.uint8, device=dev)
    for _ in range(warmup):
        K2.block_forward(d, B, T, N, h, temb, bw, cs, sn, mask, ws)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        K2.block_forward(d, B, T, N, h, temb, bw, cs, sn, mask, ws)
    e1.record()
    torch.cuda.synchronize()
    K2.check_device_error()
    ms = e0.elapsed_time(e1) / steps
    fl = block_flops(d, B, T, N, wl.lengths)
    tf = fl / (ms / 1e3) / 1e12
    kernels = traced_block_kernels(K2, torch, d, B, T, N, wl.lengths, bw, dev, reps=max(steps, 5))
    return {"workload": wl.name, "ms_per_block": ms, "tflops": tf, "flops": fl,
            "frac_burst": tf / pk["bf16_tflops"], "frac_sustained": tf / pk["bf16_tflops_sustained"],
            "l2": "inputs larger than L2 (868 MB of block weights, ~1 GB of activations)",
            "kernels": kernels}


# ----------------------------------------------------------------------------- reference arm

def run_reference(args, rank: int) -> None:
    """The CPU oracle as the reference arm: each step is a bounded sample of the workload."""
    if rank != 0:
        return
    warmup = max(args.warmup, 3)
    o = OracleSample(rows=128)
    for _ in range(warmup):
        o.run()
    times = [o.run() for _ in range(args.steps)]
    el = float(sum(times))
    value = o.flops * args.steps / el / 1e12
    wl = KI.backbone_1024()
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": warmup, "ms_per_step": el / args.steps * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": workload_config(wl, args.gpus),
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": len(os.sched_getaffinity(0)),
                             "kind": "oracle", "sample": o.describe(el / args.steps)},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- single-kernel cases

KERNEL_CASES = ("gate_up", "qkv", "out_proj", "down", "attention", "norm")


def run_kernel_case(name: str, steps: int) -> None:
    """One kernel at the backbone's block shape (M = 4608 tokens), launched `steps` times.

    Small enough for an ncu capture (< 1 GB on the device, inputs larger than L2)."""
    import torch

    import flow_matching_stream_b200 as K2
    wl = KI.backbone_1024()
    d = wl.dims
    B, T, N, S, M = wl.B, wl.T, wl.N, wl.S, wl.M
    dev = torch.device("cuda", 0)
    g = torch.Generator(device=dev).manual_seed(5)
    bf = torch.bfloat16

    def rnd(*shape, scale=1.0):
        return (torch.randn(*shape, device=dev, generator=g) * scale).to(bf)

    if name in ("gate_up", "qkv", "out_proj", "down"):
        K = d.F if name == "down" else d.C
        Nw = {"gate_up": 2 * d.F, "qkv": d.qkvg_cols, "out_proj": d.C, "down": d.C}[name]
        A, W = rnd(M, K), rnd(Nw, K, scale=K ** -0.5)
        if name in ("out_proj", "down"):
            out = torch.zeros(M, Nw, device=dev)
            gate = torch.randn(B, 6 * d.C, device=dev)
            g_off = (5 if name == "down" else 2) * d.C  # gate_mlp / gate_msa of the modulation
            fn = lambda: K2.linear(K2.KREA2_EPI_RESID, A, W, out, gate=gate.view(-1)[g_off:], rows_per_batch=S,
                                   gate_stride=6 * d.C)
        elif name == "gate_up":
            out = torch.empty(M, d.F, device=dev, dtype=bf)
            fn = lambda: K2.linear(K2.KREA2_EPI_SWIGLU, A, W, out)
        else:
            out = torch.empty(M, Nw, device=dev, dtype=bf)
            fn = lambda: K2.linear(K2.KREA2_EPI_STORE, A, W, out)
        flops = 2.0 * M * Nw * K
    elif name == "attention":
        x = rnd(M, d.qkvg_cols)
        qw = torch.randn(d.D, device=dev) * 0.1
        kw = torch.randn(d.D, device=dev) * 0.1
        cs = torch.empty(S, d.D // 2, device=dev)
        sn = torch.empty_like(cs)
        K2.rope_tables(d, torch.from_numpy(wl.positions()).to(dev), cs, sn)
        mask = torch.from_numpy(wl.mask().astype(np.uint8)).to(dev)
        out = torch.empty(M, d.HD, device=dev, dtype=bf)
        ws = torch.empty(K2.attention_workspace_size(d, B, T, N, bf), dtype=torch.uint8, device=dev)
        fn = lambda: K2.gqa_attention(d, B, T, N, x, qw, kw, cs, sn, mask, out, ws)
        flops = 4.0 * d.D * d.H * S * S
    elif name == "norm":
        h = torch.randn(M, d.C, device=dev)
        nw = torch.randn(d.C, device=dev) * 0.1
        temb = torch.randn(B, 6 * d.C, device=dev)
        table = torch.randn(6, d.C, device=dev) * 0.1
        out = torch.empty(M, d.C, device=dev, dtype=bf)
        fn = lambda: K2.modulated_rmsnorm(d, B, S, h, nw, temb, table, 0, out)
        flops = 0.0
    else:
        raise SystemExit(f"unknown kernel case {name}; choose from {KERNEL_CASES}")
    fn()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        fn()
    e1.record()
    torch.cuda.synchronize()
    K2.check_device_error()
    ms = e0.elapsed_time(e1) / steps
    print(json.dumps({"kernel_case": name, "M": M, "ms": ms, "tflops": flops / (ms / 1e3) / 1e12 if flops else None}))


def main() -> None:
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=("native", "reference"), default="native")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--record-traffic", nargs="+", metavar="STEP=BYTES[:PROFILE]", default=None,
                    help="store ncu DRAM bytes per launch for block steps and exit")
    ap.add_argument("--kernel-case", choices=KERNEL_CASES, default=None,
                    help="run one kernel at the backbone block shape (for profiler captures)")
    args = ap.parse_args()
    if args.record_traffic:
        record_traffic(args.record_traffic)
        return
    if args.kernel_case:
        run_kernel_case(args.kernel_case, args.steps)
        return
    launch = rank_layout(args.gpus, os.environ)
    if launch == "spawn":
        spawn_ranks(args)
        return
    rank, world, local_rank = launch
    if args.impl == "reference":
        run_reference(args, rank)
        return
    run_native(args, rank, world, local_rank)


def rank_layout(gpus: int, env) -> object:
    """(rank, world, local_rank) of this process, or "spawn" when --gpus N > 1 runs without a launcher.

    Under torchrun WORLD_SIZE must equal --gpus: a mismatch would time a different number of
    replicas than the line reports, so it stops the run."""
    if gpus < 1:
        raise SystemExit(f"--gpus must be >= 1, got {gpus}")
    if "WORLD_SIZE" in env:
        world = int(env["WORLD_SIZE"])
        if world != gpus:
            raise SystemExit(f"WORLD_SIZE={world} from the launcher but --gpus {gpus}: they must agree")
        return int(env.get("RANK", "0")), world, int(env.get("LOCAL_RANK", "0"))
    return "spawn" if gpus > 1 else (0, 1, 0)


def _spawned_rank(local_rank: int, args, port: int) -> None:
    os.environ.update(RANK=str(local_rank), LOCAL_RANK=str(local_rank), WORLD_SIZE=str(args.gpus),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    if args.impl == "reference":
        run_reference(args, local_rank)
    else:
        run_native(args, local_rank, args.gpus, local_rank)


def spawn_ranks(args) -> None:
    """One process per GPU on this node, as torchrun would start them (rendezvous on 127.0.0.1)."""
    import socket

    import torch.multiprocessing as mp
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    mp.start_processes(_spawned_rank, args=(args, port), nprocs=args.gpus, start_method="spawn", join=True)


if __name__ == "__main__":
    main()
