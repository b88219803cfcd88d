"""Benchmark of one decode step read from the compressed latent cache.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload I]

A step is the whole hot path over one batch: the latent write of the batch's new tokens
(projection x A, storage into the pages) followed by single-token decode attention over the
full context (K reconstruction on the tensor cores, RoPE, online softmax, latent P.C_v,
split combine and up-projection).  Default workload: the Llama-2-7B-shaped MHA layer with
bf16 latents, batch 8, context 4096.  Metric: KV tokens per second (batch * context / step
time), with the achieved HBM and tensor-core rates of the dominant kernel beside it.

With N > 1 (torchrun) every rank runs its own batch of independent sequences (weak
scaling, no collective on the data path); time is the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import time

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, HERE)

MEASURED_PEAKS = os.path.join(HERE, "MEASURED_PEAKS.json")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# dram bytes per launch of the split kernel from the committed ncu capture of this workload
# (profiles/decode_split_bf16_llama2_b8_ctx4096.md); set to None when the kernel changes
SPLIT_TRAFFIC_BYTES = 146703104  # 143.034112 MB read + 3.668992 MB written

THROTTLE_BITS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
                 0x4: "sw_power_cap", 0x80: "hw_power_brake_slowdown", 0x1: "gpu_idle",
                 0x2: "applications_clocks_setting", 0x100: "display_clock_setting"}


def peaks():
    try:
        with open(MEASURED_PEAKS) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return FALLBACK_PEAKS, "fallback"


class ClockSampler:
    """nvidia-smi clock/throttle samples every 200 ms while the timed region runs."""

    def __init__(self, device_index: int):
        self.proc = None
        self.idx = device_index

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx),
                 "--query-gpu=clocks.sm,clocks.max.sm,power.draw,utilization.gpu,"
                 "clocks_event_reasons.active", "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *a):
        self.out = ""
        if self.proc is not None:
            time.sleep(0.3)
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.out, _ = self.proc.communicate()

    def summary(self):
        sm, mx, reasons = [], None, set()
        for line in (self.out or "").splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 5:
                continue
            try:
                clk, cmax, util = float(parts[0]), float(parts[1]), float(parts[3])
                bits = int(parts[4], 16) if parts[4].startswith("0x") else int(parts[4])
            except ValueError:
                continue
            mx = cmax
            if util > 0:
                sm.append(clk)
                for b, name in THROTTLE_BITS.items():
                    if bits & b and name != "gpu_idle":
                        reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": 0}
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


class OracleDecode:
    """The fp64 oracle's decode of the workload on the host cores (test infrastructure: only
    this CPU-baseline leg of the bench runs it).  Stored latents of the sampled sequences are
    prepared once; the timed work is the oracle's decode attention (reconstruction, RoPE,
    softmax, P.C_v, up-projection) per (sequence, query head)."""

    def __init__(self, workload_index: int, n_seq: int):
        from oracle.workloads import ref_for
        import oracle.starkv_oracle as O
        self.O = O
        self.ref = ref = ref_for(workload_index, False)
        self.w = ref.w
        self.q = ref.queries()
        n_seq = max(1, min(n_seq, self.w["batch"]))  # the workload may hold fewer sequences
        self.seqs = [ref.stored(ref.sequence_latents(b)) for b in range(n_seq)]
        self.cores = (len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity")
                      else os.cpu_count())

    def run(self, b: int, heads) -> float:
        """Decode of sequence b for ``heads``; returns seconds."""
        Ck, Cv = self.seqs[b % len(self.seqs)]
        w, ref = self.w, self.ref
        t0 = time.perf_counter()
        self.O.decode_attention(self.q[b % len(self.seqs)], Ck, Cv, ref.Bk_s, ref.Bv_s,
                                w["rope_theta"], w["n_kv_heads"], heads)
        return time.perf_counter() - t0


def cpu_baseline(workload_index: int, budget_s: float = 12.0):
    """KV tokens/s of the oracle over whole sequences (all heads), repeated for ~budget_s."""
    od = OracleDecode(workload_index, 2)
    w = od.w
    H, L = w["n_q_heads"], w["context"]
    secs, tokens, n = 0.0, 0, 0
    while secs < budget_s:
        secs += od.run(n, list(range(H)))
        tokens += L
        n += 1
    sample = (f"{n} whole sequence(s) of {L} tokens x {H} query heads (2 distinct sequences), "
              f"fp64 NumPy oracle decode; latent storage prepared outside the timing")
    return tokens / secs, secs, od.cores, sample


def run_reference(args, rank, world):
    """The reference arm: the oracle, as it stands, on the host cores.  One step = the decode
    of a bounded slice of the workload (a few query heads of one sequence, sized so that the
    whole run stays within about two minutes); its KV tokens count pro rata of the heads."""
    if rank != 0:
        return
    od = OracleDecode(args.workload, 2)
    w = od.w
    H, L = w["n_q_heads"], w["context"]
    per_head = od.run(0, [0])
    budget = 120.0 / max(1, args.steps + args.warmup)
    n_h = int(max(1, min(H, budget // max(per_head, 1e-6))))
    for i in range(args.warmup):
        od.run(i, [(i + k) % H for k in range(n_h)])
    secs = 0.0
    for i in range(args.steps):
        secs += od.run(i, [(i + k) % H for k in range(n_h)])
    value = args.steps * L * n_h / H / secs
    sample = (f"per step: {n_h} of {H} query heads of one {L}-token sequence (counted as "
              f"{n_h}/{H} of its KV tokens), fp64 NumPy oracle decode")
    line = {
        "impl": "reference", "metric": "compressed-KV decode attention KV tokens/s",
        "value": value, "unit": "KV tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1000 * secs / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": workload_config(w, world),
        "cpu_baseline": {"value": value, "unit": "KV tokens/s", "cores": od.cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "KV tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def workload_config(w, world):
    return {"workload": w["name"], "batch_per_gpu": w["batch"], "global_batch": w["batch"] * world,
            "context": w["context"], "n_q_heads": w["n_q_heads"], "n_kv_heads": w["n_kv_heads"],
            "head_dim": w["head_dim"], "d_model": w["d_model"], "key_rank": w["key_rank"],
            "latent_format": w["fmt"], "parallelism": f"dp{world} (independent sequences)",
            "l2": "flushed between steps (256 MiB write outside the timed events)"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", type=int, default=2)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        run_reference(args, rank, world)
        return

    import torch
    import torch.distributed as dist
    from datetime import timedelta

    from rank_quantized_kv_decode_b200 import api
    from rank_quantized_kv_decode_b200 import dist as D
    from rank_quantized_kv_decode_b200 import workload as W

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
    assert args.warmup >= 3, "at least 3 warm-up steps"

    wl = W.build(args.workload, device=dev, need_down=True)
    w, lay, lc = wl.w, wl.lay, wl.lc
    B, L = w["batch"], w["context"]
    # per-step inputs: the new tokens' hidden rows (written at position L-1) and the queries
    g = np.random.default_rng(1234 + rank)
    xdt = W.x_dtype(w["fmt"])
    x_new = torch.from_numpy(g.standard_normal((B, w["d_model"]), dtype=np.float32)).to(xdt).to(dev)
    seq = torch.arange(B, dtype=torch.int32, device=dev)
    pos = (wl.seq_lens - 1).to(torch.int32)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def call_append():
        api.append(lay, x_new, wl.A_t, seq, pos, wl.block_table, lc.cache, lc.append_ws, lc.status)

    def call_partials():
        api.decode_partials(lay, wl.q, lc.cache, wl.block_table, wl.seq_lens, wl.Bk_t, lc.rope,
                            lc.decode_ws, lc.status)

    def call_combine():
        api.decode_combine(lay, wl.seq_lens, lc.max_pages, wl.Bv, lc.decode_ws, wl.out)

    calls = (call_append, call_partials, call_combine)
    for _ in range(args.warmup):
        flush.fill_(1)
        for c in calls:
            c()
    torch.cuda.synchronize(dev)
    assert lc.status.item() == 0, f"device status {lc.status.item()}"
    # The step's launches replay from CUDA graphs (same kernels, same arguments), so the timed
    # loops are not bound by host-side argument checks and launch latency.  One graph holds
    # the whole step (append, partials, combine: its kernels start with programmatic
    # dependent launch); per-phase graphs time the split kernel on its own.
    step_graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(step_graph):
        for c in calls:
            c()
    graphs = []
    for c in calls:
        g_ = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_):
            c()
        graphs.append(g_)
    for _ in range(3):
        flush.fill_(1)
        step_graph.replay()
        flush.fill_(1)
        for g_ in graphs:
            g_.replay()
    torch.cuda.synchronize(dev)

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    sevs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clocks:
        # (1) whole steps: the throughput
        for i in range(args.steps):
            flush.fill_(i & 0xFF)  # 256 MiB write: L2 holds nothing of the previous step
            evs[i][0].record(stream)
            step_graph.replay()
            evs[i][1].record(stream)
        # (2) the split kernel alone, between the same append and combine
        for i in range(args.steps):
            flush.fill_(i & 0xFF)
            graphs[0].replay()
            sevs[i][0].record(stream)
            graphs[1].replay()
            sevs[i][1].record(stream)
            graphs[2].replay()
        torch.cuda.synchronize(dev)
    step_ms = [e[0].elapsed_time(e[1]) for e in evs]
    split_ms = [e[0].elapsed_time(e[1]) for e in sevs]
    if world > 1:
        dist.barrier()
    # device time of the K steps, max over ranks; every rank processed B sequences
    total_ms = D.max_over_ranks(float(np.sum(step_ms)), dev)
    ms_per_step = total_ms / args.steps
    tokens_per_step = B * L * world
    value = D.aggregate_rate(B * L * args.steps, world, total_ms / 1000.0)

    # end to end through the public API: host inputs (pinned) in, output back to the host
    x_host = x_new.cpu().pin_memory()
    q_host = wl.q.cpu().pin_memory()
    out_host = torch.empty(wl.out.shape, dtype=torch.float32).pin_memory()
    x_dev, q_dev = torch.empty_like(x_new), wl.q
    e2e_evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(args.steps)]

    def e2e_step():
        x_dev.copy_(x_host, non_blocking=True)
        q_dev.copy_(q_host, non_blocking=True)
        api.append(lay, x_dev, wl.A_t, seq, pos, wl.block_table, lc.cache, lc.append_ws, lc.status)
        api.decode_attention(lay, q_dev, lc.cache, wl.block_table, wl.seq_lens, wl.Bk_t, wl.Bv,
                             lc.rope, wl.out, lc.decode_ws, lc.status)
        out_host.copy_(wl.out, non_blocking=True)

    for _ in range(3):
        e2e_step()
    torch.cuda.synchronize(dev)
    for i in range(args.steps):
        flush.fill_(3)
        e2e_evs[i][0].record(stream)
        e2e_step()
        e2e_evs[i][1].record(stream)
    torch.cuda.synchronize(dev)
    e2e_total = D.max_over_ranks(float(np.sum([a.elapsed_time(b) for a, b in e2e_evs])), dev)
    e2e_value = D.aggregate_rate(B * L * args.steps, world, e2e_total / 1000.0)
    h2d = x_host.numel() * x_host.element_size() + q_host.numel() * q_host.element_size()
    d2h = out_host.numel() * out_host.element_size()
    assert lc.status.item() == 0

    # roofline of the dominant kernel (the split kernel: tensor-core bound reconstruction)
    pk, src = peaks()
    split_s = float(np.mean(split_ms)) / 1000.0
    recon_flop = 2.0 * w["key_rank"] * w["n_kv_heads"] * w["head_dim"] * B * L
    tflops = recon_flop / split_s / 1e12
    peak_tc = pk["bf16_tflops"]
    bytes_alg = B * L * lay.token_bytes
    hbm_gbs = bytes_alg / split_s / 1e9
    clk = clocks.summary()
    line = {
        "metric": "compressed-KV decode attention KV tokens/s", "value": value,
        "unit": "KV tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16" if w["fmt"] == "bf16" else w["fmt"],
        "data": "synthetic (seeded latents with the stated singular-value spectra)",
        "config": workload_config(w, world),
        "roofline": {"bound": "tensor", "achieved": tflops, "peak": peak_tc, "unit": "TFLOP/s",
                     "frac": tflops / peak_tc, "traffic": SPLIT_TRAFFIC_BYTES,
                     "peak_source": f"{src} bf16 burst", "kernel": "decode_split_kernel",
                     "peak_sustained": pk.get("bf16_tflops_sustained"),
                     "frac_of_sustained": (tflops / pk["bf16_tflops_sustained"]
                                           if pk.get("bf16_tflops_sustained") else None),
                     "flop_per_launch": recon_flop, "split_ms": split_s * 1000.0,
                     "hbm_achieved_gbs": hbm_gbs, "hbm_peak_gbs": pk["hbm_gbs"],
                     "hbm_frac": hbm_gbs / pk["hbm_gbs"], "hbm_bytes_per_launch": bytes_alg},
        "e2e": {"value": e2e_value, "unit": "KV tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        # pass 1: append (projection + store), split, combine per step; pass 2: the same
        "gpu_launches": 8 * args.steps,
        "clocks": clk,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, dt, cores, sample = cpu_baseline(args.workload)
        line["cpu_baseline"] = {"value": v, "unit": "KV tokens/s", "cores": cores, "kind": "oracle",
                                "sample": sample, "seconds": dt}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
