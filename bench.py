#!/usr/bin/env python
"""Benchmark of the looped-block hot path on B200.

Headline: one looped forward of the 407M-shaped model (d_model 2048, 16 heads
x 128, ffn 8192, INT4 group 128, 2 pre-blocks + 1 shared loop block run L=8,
seq 128, batch 1, final RMSNorm, no logits) per step; value = tokens/s over the
whole job.  Secondary lines (inside the same JSON object) time KV-cached
decode: batch 1 with FP16 KV, batch 8 at context 2048 with INT8 KV, and the
mixed-depth INT3 lanes L=[4,16,32].

Inputs are seeded synthetic weights and token ids.  The model's weights (about
104 MB) fit in the 126 MB L2, so L2 is flushed (a 256 MiB write) before every
timed step; the flush is outside the timed interval.

Multi-GPU: replicas only (each rank runs the same workload on its own GPU, no
data-path collective); value = all ranks' tokens / the slowest rank's time.

`--impl reference` times the CPU oracle instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "looped forward ms & tokens/s (seq=128,L=8; decode tok/s) + % of roofline"
WORKLOAD = ("prefill407m: d_model 2048, 16 heads x 128, SwiGLU ffn 8192, INT4 group 128 fp16 "
            "scales, 2 pre-blocks + shared loop block L=8, seq 128, batch 1, no logits")
FLUSH_BYTES = 256 << 20


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=2000)
    p.add_argument("--warmup", type=int, default=20)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--no-decode", action="store_true", help="skip the decode sub-measurements")
    p.add_argument("--no-cpu-baseline", action="store_true")
    return p.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while running."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None
        self.err = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu_id}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True)
        except OSError as e:
            self.err = str(e)
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        time.sleep(0.15)
        self.out = ""
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.out, _ = self.proc.communicate()

    def summary(self):
        if self.err or not self.out:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [],
                    "note": self.err or "no nvidia-smi samples"}
        sms, mx, reasons, n = [], None, set(), 0
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sms.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            n += 1
            for name, val in zip(names, f[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sms) if sms else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": n}


def gpu_uuid(torch, dev):
    u = str(torch.cuda.get_device_properties(dev).uuid)
    return u if u.startswith("GPU-") else "GPU-" + u


# ----------------------------------------------------------------------------- oracle (CPU)

def oracle_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return max(n)
    except Exception:
        pass
    return os.cpu_count()


def cpu_baseline(seconds: float = 8.0):
    """The oracle as it stands, on the host cores: full seq-128 L=8 forwards
    for about `seconds` (at least 2, after one untimed forward); the cached
    decode step of the batch-1 FP16-KV workload over its first 8 steps (the
    256-token prompt prefill untimed); and the INT4 and INT3 packers on one
    407M block."""
    import numpy as np
    import synthetic as syn
    from oracle import tinyloop_oracle as o
    from oracle.workloads import build_oracle_model
    w = syn.WORKLOADS["prefill407m"]
    om = build_oracle_model("prefill407m")
    ids = syn.prompt_ids(w)
    om.prefill(ids, w.L[0])
    n, t0 = 0, time.perf_counter()
    while n < 2 or time.perf_counter() - t0 < seconds:
        om.prefill(ids, w.L[0])
        n += 1
    dt = time.perf_counter() - t0
    # cached decode: prompt 256 (untimed), then 8 timed steps
    wd = syn.WORKLOADS["decode407m"]
    kv = om.new_kv(wd.L[0], "fp16")
    om.prefill(syn.prompt_ids(wd), wd.L[0], kv=kv)
    steps = syn.decode_ids(wd)
    t1 = time.perf_counter()
    for s in range(8):
        om.decode_step(np.int64(steps[s]), wd.L[0], kv)
    dec_ms = (time.perf_counter() - t1) / 8 * 1e3
    # packers: quantise + pack the five matrices of one block
    wts = syn.block_weights(w.shape, w.seed, "loop")
    pack_ms = {}
    for bits in (4, 3):
        t2 = time.perf_counter()
        o.pack_block(wts, bits, w.group)
        pack_ms[bits] = (time.perf_counter() - t2) * 1e3
    return {"value": round(w.seq * n / dt, 2), "unit": "tokens/s", "cores": oracle_threads(),
            "kind": "oracle",
            "decode_ms_per_step": round(dec_ms, 2),
            "decode_tok_s": round(1e3 / dec_ms, 2),
            "pack_int4_ms_per_block": round(pack_ms[4], 1),
            "pack_int3_ms_per_block": round(pack_ms[3], 1),
            "sample": f"{n} full forwards (seq 128, L=8, fp64 numpy oracle), {dt:.1f} s; "
                      f"8 cached decode steps after a 256-token prompt (batch 1, FP16 KV, "
                      f"L=8); one INT4 and one INT3 pack of a 407M block; model build and "
                      f"prompt prefill untimed"}


def run_reference(args, rank, world):
    """CPU oracle arm: each step is one of the 10 block applications of the
    seq-128 L=8 forward (cycling pre0, pre1, loop x 8 on the inputs that layer
    sees), so K steps are K/10 forwards of work."""
    if rank != 0:
        return
    import numpy as np
    import synthetic as syn
    from oracle import tinyloop_oracle as o
    from oracle.workloads import build_oracle_model
    w = syn.WORKLOADS["prefill407m"]
    L = w.L[0]
    om = build_oracle_model("prefill407m")
    ids = syn.prompt_ids(w)
    trace = []
    om.prefill(ids, L, trace=trace)
    inputs = [om.embed(ids)] + trace[:-1]
    sched = om.schedule(L)
    pos = np.arange(w.seq)

    def step(i):
        layer = i % len(sched)
        blk, h = sched[layer], inputs[layer]
        q, k, v = blk.qkv(h, pos)
        return blk.finish(h, o.causal_attention(q, k, v, pos))

    for i in range(args.warmup):
        step(i)
    t0 = time.perf_counter()
    for i in range(args.steps):
        step(i)
    dt = time.perf_counter() - t0
    layers = len(sched)
    fwd_s = dt / args.steps * layers
    value = round(w.seq / fwd_s, 3)
    sample = (f"{args.steps} block applications = {args.steps / layers:.1f} forwards "
              f"(seq 128, L=8) on the fp64 numpy oracle")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(dt / args.steps * 1e3, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": WORKLOAD, "step": "one block application (1/10 forward)"},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": oracle_threads(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- replicas

def max_over_ranks(t: float, dist, device) -> float:
    """The slowest rank's time (seconds); t itself on a single process."""
    if dist is None:
        return t
    import torch
    tt = torch.tensor([t], dtype=torch.float64, device=device)
    dist.all_reduce(tt, op=dist.ReduceOp.MAX)
    return float(tt.item())


def job_value(units_per_rank: float, world: int, t_max: float) -> float:
    """Whole-job throughput of N independent replicas: every rank's units over
    the slowest rank's time."""
    return units_per_rank * world / t_max


# ----------------------------------------------------------------------------- GPU arm

def source_hash(*files):
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel_file: str, src_files):
    """Per-launch DRAM bytes of a kernel from its committed ncu summary, if the
    summary was taken on the current source (matching hash); else None."""
    path = os.path.join(ROOT, "profiles", kernel_file)
    if not os.path.exists(path):
        return None
    vals = {}
    with open(path) as f:
        for line in f:
            if ":" in line and not line.startswith("#"):
                k, v = line.split(":", 1)
                vals[k.strip()] = v.strip()
    if vals.get("source_sha256_16") != source_hash(*src_files):
        return None
    try:
        return float(vals["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


def run_ours(args, rank, world, dist):
    import numpy as np
    import torch

    from weight_shared_looped_b200 import build as _build
    _build.build()
    import synthetic as syn
    import weight_shared_looped_b200 as tl
    from weight_shared_looped_b200.model import DeviceBlock, DeviceModel

    dev = int(os.environ.get("LOCAL_RANK", 0))
    torch.cuda.set_device(dev)
    pk = peaks()
    w = syn.WORKLOADS["prefill407m"]
    L, seq = w.L[0], w.seq

    def cfg(bits):
        return {"d_model": 2048, "n_heads": 16, "head_dim": 128, "ffn": 8192, "bits": bits,
                "group": 128, "eps": 1e-5, "rope_theta": 10000.0}

    blocks = {n: DeviceBlock(cfg(4), weights=syn.block_weights(w.shape, w.seed, n))
              for n in syn.block_names(w)}
    embed = syn.embedding(w.shape, w.seed)
    gamma_f = syn.final_gain(w.shape, w.seed)
    model = DeviceModel([blocks["pre0"], blocks["pre1"]], blocks["loop"], gamma_f, embed,
                        max_tokens=2048, max_lanes=8, max_ctx=2048 + 64, max_L=32)
    stream = torch.cuda.current_stream()
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    ids = torch.from_numpy(syn.prompt_ids(w).astype(np.int32)).cuda()
    y = torch.empty(seq, 2048, dtype=torch.float32, device="cuda")

    def step():
        model.prefill(ids, L=L, y_out=y)

    def timed(fn, k, warm):
        for _ in range(warm):
            flush.zero_()
            fn()
        torch.cuda.synchronize()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(k)]
        if dist:
            dist.barrier()
        torch.cuda.synchronize()
        for a, b in evs:
            flush.zero_()
            a.record(stream)
            fn()
            b.record(stream)
        torch.cuda.synchronize()
        if dist:
            dist.barrier()
        per = [a.elapsed_time(b) for a, b in evs]
        timed.last_median_ms = statistics.median(per)
        return sum(per) / 1e3   # seconds

    # headline: prefill forward
    for _ in range(max(args.warmup, 3)):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    assert model.sync_status() == tl.TL_OK
    with ClockSampler(gpu_uuid(torch, dev)) as clk, torch.cuda.nvtx.range("prefill"):
        t = timed(step, args.steps, 0)
    assert model.sync_status() == tl.TL_OK
    median_ms = max_over_ranks(timed.last_median_ms, dist, "cuda")
    t = max_over_ranks(t, dist, "cuda")
    value = job_value(seq * args.steps, world, t)
    ms_per_step = t / args.steps * 1e3
    n_layers = 2 + L
    launches_per_fwd = 2 + 8 * n_layers   # embed, final norm; per layer norm, QKV, RoPE+KV, attention, O, norm, gate|up+SwiGLU, down

    # e2e: host (pinned) ids in, host y out, through the C-ABI call
    ids_h = torch.from_numpy(syn.prompt_ids(w).astype(np.int32)).pin_memory()
    y_h = torch.empty(seq, 2048, dtype=torch.float32).pin_memory()
    k_e2e = max(10, min(args.steps, 500))
    t_e2e = max_over_ranks(timed(lambda: model.prefill(ids_h, L=L, y_out=y_h), k_e2e, 3), dist,
                           "cuda")
    e2e = {"value": round(job_value(seq * k_e2e, world, t_e2e), 1), "unit": "tokens/s",
           "h2d_bytes_per_step": ids_h.numel() * 4, "d2h_bytes_per_step": y_h.numel() * 4}

    # roofline of the dominant kernel: the gate|up GEMM launch (N 16384, K 2048, T 128)
    xg = torch.randn(seq, 2048, device="cuda").half()
    wg = torch.cat([blocks["loop"].t["w_gate"], blocks["loop"].t["w_up"]])
    sg = torch.cat([blocks["loop"].t["s_gate"], blocks["loop"].t["s_up"]])
    yg = torch.empty(seq, 16384, dtype=torch.float32, device="cuda")
    ws_b = tl.tl_linear_workspace_bytes(16384, 2048, seq)
    wsg = torch.empty(max(ws_b, 1), dtype=torch.uint8, device="cuda")
    flops = 2.0 * seq * 16384 * 2048
    # isolated: one launch per event pair, L2 flushed before each (includes the
    # launch latency of a single kernel)
    k_iso = 200
    t_iso = timed(lambda: tl.tl_linear(wg, sg, 16384, 2048, 128, xg, yg, wsg), k_iso, 5)
    # steady state: back-to-back launches captured in a CUDA graph, rotating
    # over 8 copies of the weights (8 x 17.3 MB > the 126 MB L2, so every
    # launch streams its weights from HBM), one event pair around 2 x 200
    wgs = [wg.clone() for _ in range(8)]
    sgs = [sg.clone() for _ in range(8)]

    def gemm_chain():
        for _ in range(25):
            for c in range(8):
                tl.tl_linear(wgs[c], sgs[c], 16384, 2048, 128, xg, yg, wsg)

    gemm_chain()
    torch.cuda.synchronize()
    gg = torch.cuda.CUDAGraph()
    with torch.cuda.graph(gg):
        gemm_chain()
    gg.replay()
    torch.cuda.synchronize()
    ea, eb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    ea.record(stream)
    gg.replay()
    gg.replay()
    eb.record(stream)
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    k_gemm = 400
    t_gemm = ea.elapsed_time(eb) / 1e3
    del gg
    achieved = flops * k_gemm / t_gemm / 1e12
    roof = {"bound": "tensor", "achieved": round(achieved, 2), "peak": pk["bf16_tflops"],
            "unit": "TFLOP/s", "frac": round(achieved / pk["bf16_tflops"], 4),
            "traffic": ncu_traffic("gemm_w4_tc_gateup_T128.md",
                                   ["weight_shared_looped_b200/csrc/gemm_tc.cu"]),
            "kernel": "gemm_w4_tc_kernel<128> (gate|up, N 16384, K 2048, T 128; 400 back-to-back "
                      "launches over 8 weight copies larger than L2)",
            "peak_kind": f"bf16 dense burst, {pk['source']} (fp16 operands run at the same rate)",
            "us_per_launch": round(t_gemm / k_gemm * 1e6, 2),
            "us_per_launch_isolated": round(t_iso / k_iso * 1e6, 2),
            "forward_tflops": round(172.5e9 * args.steps / (t / world) / 1e12, 2),
            "forward_frac": round(172.5e9 * args.steps / (t / world) / 1e12 / pk["bf16_tflops"], 4)}

    l2 = l2_probe(tl, torch, dist)
    decode = None
    if not args.no_decode:
        decode = run_decode(model, blocks, syn, tl, torch, np, flush, timed, dist, world, pk,
                            cfg, l2["gbs"])

    line = {"metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4),
            "ms_per_step_median": round(median_ms, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "fp16",
            "data": "synthetic",
            "config": {"workload": WORKLOAD, "l2": "flushed before every timed step (256 MiB write)",
                       "parallelism": "replicas" if world > 1 else "single",
                       "graphs": "one CUDA graph per (seq, L)"},
            "roofline": roof, "e2e": e2e, "gpu_launches": launches_per_fwd * args.steps,
            "l2_probe": l2,
            "clocks": clk.summary()}
    if decode is not None:
        line["decode"] = decode
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline()
    elif rank == 0:
        line["cpu_baseline"] = None
    model.close()
    return line


def l2_probe(tl, torch, dist, mib: int = 32, passes: int = 64):
    """L2 read bandwidth: tl_read_probe over a buffer well inside the L2 (one
    untimed pass makes it resident), timed with CUDA events on the launching
    stream, best of 5."""
    buf = torch.empty(mib << 20, dtype=torch.uint8, device="cuda")
    buf.fill_(1)
    sink = torch.zeros(2, dtype=torch.int32, device="cuda")
    stream = torch.cuda.current_stream()
    tl.tl_read_probe(buf, 1, sink)
    best = None
    for _ in range(5):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        tl.tl_read_probe(buf, passes, sink)
        b.record(stream)
        torch.cuda.synchronize()
        t = a.elapsed_time(b) / 1e3
        best = t if best is None else min(best, t)
    assert int(sink[1].item()) == passes
    best = max_over_ranks(best, dist, "cuda")
    gbs = (mib << 20) * passes / best / 1e9
    return {"gbs": round(gbs, 1), "bytes": mib << 20, "passes": passes,
            "how": "tl_read_probe (128-bit loads over every SM) on an L2-resident buffer, "
                   "CUDA events, best of 5"}


def block_bytes(tl, bits: int, d: int = 2048, f: int = 8192, group: int = 128) -> int:
    """Packed bytes (codes + fp16 scales) of one block, from the library's
    own size query."""
    total = 0
    for n, k in ((3 * d, d), (d, d), (f, d), (f, d), (d, f)):
        c, sc = tl.tl_packed_bytes(n, k, bits, group)
        total += c + sc
    return total


def decode_roofline(t_step, hbm_bytes, l2_bytes, hbm_gbs, l2_gbs):
    """The decode roofline: t = HBM bytes / HBM bandwidth + L2 bytes / L2
    bandwidth (the loop block's re-reads within a step come from L2)."""
    t_roof = hbm_bytes / (hbm_gbs * 1e9) + l2_bytes / (l2_gbs * 1e9)
    return {"hbm_bytes_per_step": int(hbm_bytes), "l2_bytes_per_step": int(l2_bytes),
            "roofline_us": round(t_roof * 1e6, 2),
            "frac_roofline": round(t_roof / t_step, 4),
            "frac_hbm": round(hbm_bytes / t_step / 1e9 / hbm_gbs, 4)}


def loop_read_bytes(tl, blk) -> int:
    """Bytes the decode kernels read per application of an INT3 block: its
    canonical 10-codes-per-word rows and fp16 scales (read natively)."""
    return block_bytes(tl, 3)


def run_spec(model, kv, w, torch, np, dist, world, K=4, L_draft=2, L_verify=8, n_steps=24):
    """Greedy self-speculative steps (K drafts at L_draft, one verify extend of
    K + 1 tokens at L_verify) from the 256-token prompt, against plain greedy
    decoding (one-token extend at L_verify + head) from the same state.  Each
    speculative step synchronises once (acceptance is decided on the host), so
    both loops are timed with CUDA events around the whole loop."""
    import synthetic as syn
    stream = torch.cuda.current_stream()
    base = w.seq
    tok0 = int(syn.decode_ids(w)[0])

    def spec_loop():
        kv.set_position(0, base)
        tok, n_tok = tok0, 0
        for _ in range(n_steps):
            out = model.spec_step(kv, tok, K=K, L_draft=L_draft, L_verify=L_verify)
            n_tok += len(out)
            tok = out[-1]
        return n_tok

    def greedy_loop(n):
        kv.set_position(0, base)
        tok = torch.tensor([tok0], dtype=torch.int32, device="cuda")
        for _ in range(n):
            y = model.extend(kv, tok, L=L_verify)
            tok = model.greedy_head(y)

    spec_loop()          # warm the graphs
    greedy_loop(2)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    n_tok = spec_loop()
    b.record(stream)
    torch.cuda.synchronize()
    t_spec = max_over_ranks(a.elapsed_time(b) / 1e3, dist, "cuda")
    a.record(stream)
    greedy_loop(n_tok)
    b.record(stream)
    torch.cuda.synchronize()
    t_greedy = max_over_ranks(a.elapsed_time(b) / 1e3, dist, "cuda")
    return {"tok_s": round(n_tok * world / t_spec, 1),
            "greedy_tok_s": round(n_tok * world / t_greedy, 1),
            "tokens_per_step": round(n_tok / n_steps, 3),
            "acceptance": round((n_tok - n_steps) / (n_steps * K), 4),
            "K": K, "L_draft": L_draft, "L_verify": L_verify, "steps": n_steps,
            "workload": "batch 1, FP16 KV, after the 256-token prompt; greedy tokens through the "
                        "tied fp16 embedding (50257 x 2048); synthetic random weights, so the "
                        "acceptance is what such weights give, not a trained model's"}


def run_b1_variants(model, blocks, w, syn, tl, torch, np, timed, dist, world, cfg, hbm, l2_gbs,
                    blk_bytes, kv_bytes, ids_t):
    """B = 1 decode (prompt 256, 128 steps, L = 8, FP16 KV) with loop-block
    weight variants; the bytes per step count each variant's first read from
    HBM and its further reads from L2."""
    from weight_shared_looped_b200.model import DeviceBlock, DeviceModel
    out = {}
    wl = syn.block_weights(w.shape, w.seed, "loop")
    signed = DeviceBlock(cfg(4), weights=wl, sign=True)
    low = DeviceBlock(cfg(3), weights=wl)
    sign_bytes = sum(tl.tl_sign_bits_bytes(n, k) for n, k in
                     ((3 * 2048, 2048), (2048, 2048), (8192, 2048), (8192, 2048), (2048, 8192)))
    low_bytes = block_bytes(tl, 3)
    cases = {
        # iterations 1, 3, 5, 7 also read the sign bits
        "b1_cross_iter": (signed, [], True, 3 * blk_bytes + sign_bytes + kv_bytes,
                          7 * blk_bytes + 3 * sign_bytes),
        # iterations 0-3 read the INT3 copy, 4-7 the INT4 block
        "b1_dual_bit_int3_int4": (blocks["loop"], [low] * 4, False,
                                  3 * blk_bytes + low_bytes + kv_bytes,
                                  3 * blk_bytes + 3 * low_bytes),
    }
    dids = [ids_t(syn.decode_ids(w)[i:i + 1]) for i in range(w.steps)]
    # store-h KV: the cache keeps the fp16 QKV-input rows, each step rebuilds K
    # and V with the quantised-weight GEMM (its weight reads: W_k, W_v rows)
    qkv_kv_bytes = 2 * (2048 * 2048 // 2 + 2048 * 16 * 2)
    avg_ctx = w.seq + (w.steps + 1) / 2
    bucket_rows = sum(min(w.max_ctx, (p + 127) // 128 * 128) for p in range(w.seq, w.seq + w.steps)) / w.steps
    cases["b1_store_h"] = (blocks["loop"], [], False, 3 * blk_bytes + kv_bytes / 2,
                           7 * blk_bytes + 10 * qkv_kv_bytes, "h",
                           round(10 * bucket_rows * 2 * 2048 * 2048 * 2 / 1e9, 2))
    for name, case in cases.items():
        loop_blk, variants, cross, hbm_b, l2_b = case[:5]
        kv_dtype = case[5] if len(case) > 5 else "fp16"
        m = DeviceModel([blocks["pre0"], blocks["pre1"]], loop_blk, syn.final_gain(w.shape, w.seed),
                        syn.embedding(w.shape, w.seed), max_tokens=w.seq, max_lanes=1,
                        max_ctx=w.max_ctx, max_L=8)
        m.set_cross_iter(cross)
        m.set_iteration_blocks(variants)
        kv = m.new_kv([8], max_ctx=w.max_ctx, dtype=kv_dtype)
        m.prefill(ids_t(syn.prompt_ids(w)), L=8, kv=kv, lane=0)
        y1 = torch.empty(1, 2048, dtype=torch.float32, device="cuda")
        it = iter(range(10 ** 9))

        def dstep():
            m.decode(kv, dids[next(it) % w.steps], L_per_lane=[8], y_out=y1)

        dstep()
        kv.set_position(0, w.seq)
        it = iter(range(10 ** 9))
        t = max_over_ranks(timed(dstep, w.steps, 0), dist, "cuda")
        out[name] = {"tok_s": round(w.steps * world / t, 1),
                     "ms_per_step": round(t / w.steps * 1e3, 4),
                     "ms_per_step_median": round(timed.last_median_ms, 4),
                     **decode_roofline(t / w.steps, hbm_b, l2_b, hbm, l2_gbs),
                     "workload": "prompt 256 + 128 steps, L=8, FP16 KV, batch 1"}
        if kv_dtype == "h":
            out[name]["workload"] = ("prompt 256 + 128 steps, L=8, store-h cache (fp16 QKV-input "
                                     "rows; K and V of every position below the step's 128-"
                                     "position bucket rebuilt every step), batch 1")
            out[name]["rebuild_gflop_per_step"] = case[6]
            out[name]["cache_bytes"] = tl.tl_kv_bytes(m.handle, w.max_ctx, [8], tl.TL_KV_H)
            out[name]["cache_bytes_fp16_kv"] = tl.tl_kv_bytes(m.handle, w.max_ctx, [8],
                                                              tl.TL_KV_FP16)
        kv.close()
        m.close()
        torch.cuda.synchronize()
    signed.close()
    low.close()
    return out


def run_decode(model, blocks, syn, tl, torch, np, flush, timed, dist, world, pk, cfg, l2_gbs):
    """KV-cached decode throughput: B=1 FP16 KV (prompt 256, 128 steps), B=8
    INT8 KV at context 2048 (64 steps), mixed-depth INT3 lanes (ctx 1024, 32
    steps).  Each timed step is one tl_decode_step; caches are filled by GPU
    prefill of seeded prompt ids.  L2 is flushed before every step, so each
    step reads the model's weights once from HBM; the loop block's further
    iterations re-read them from L2."""
    from weight_shared_looped_b200.model import DeviceBlock, DeviceModel
    out = {}
    hbm = pk["hbm_gbs"]
    blk_bytes = block_bytes(tl, 4)

    def ids_t(x):
        return torch.from_numpy(np.ascontiguousarray(x, dtype=np.int32)).cuda()

    def max_t(t):
        return max_over_ranks(t, dist, "cuda")

    # B = 1, FP16 KV, prompt 256 -> 384
    w = syn.WORKLOADS["decode407m"]
    kv = model.new_kv([8], max_ctx=w.max_ctx)
    model.prefill(ids_t(syn.prompt_ids(w)), L=8, kv=kv, lane=0)
    dids = [ids_t(syn.decode_ids(w)[i:i + 1]) for i in range(w.steps)]
    it = iter(range(10 ** 9))
    y1 = torch.empty(1, 2048, dtype=torch.float32, device="cuda")

    def dstep():
        model.decode(kv, dids[next(it) % w.steps], L_per_lane=[8], y_out=y1)

    # warm the graph, then rewind the cache so every timed step is at 256..383
    dstep()
    kv.set_position(0, w.seq)
    it = iter(range(10 ** 9))
    with torch.cuda.nvtx.range("decode_b1"):
        t = max_t(timed(dstep, w.steps, 0))
    med = timed.last_median_ms
    avg_ctx = w.seq + (w.steps + 1) / 2
    kv_bytes = 10 * avg_ctx * 2048 * 2 * 2
    out["b1_fp16kv"] = {"tok_s": round(w.steps * world / t, 1),
                        "ms_per_step": round(t / w.steps * 1e3, 4),
                        "ms_per_step_median": round(med, 4),
                        **decode_roofline(t / w.steps, 3 * blk_bytes + kv_bytes, 7 * blk_bytes,
                                          hbm, l2_gbs),
                        "workload": "prompt 256 + 128 steps, L=8, FP16 KV, batch 1"}

    # the same B = 1 workload with per-iteration weight variants of the loop
    # block ("Current Status", architecture-unique features table): cross-
    # iteration rounding (odd iterations add the sign-of-frac bits) and the
    # dual-bit swap (an INT3 copy for iterations 0-3, the INT4 block for 4-7)
    out.update(run_b1_variants(model, blocks, w, syn, tl, torch, np, timed, dist, world, cfg,
                               hbm, l2_gbs, blk_bytes, kv_bytes, ids_t))

    # self-speculative decode on the same cache ("Current Status", self-speculative
    # row: L=2 draft, L=8 verify, same weights): greedy tokens through the tied
    # embedding head; draft + verify throughput, acceptance, and plain greedy
    # decode with the same head for comparison
    out["spec_L2_L8"] = run_spec(model, kv, w, torch, np, dist, world)
    kv.close()
    torch.cuda.synchronize()
    kv = None

    # B = 8, INT8 KV, context 2048 -> 2112
    w = syn.WORKLOADS["longctx_int8"]
    kv = model.new_kv(list(w.L), max_ctx=w.max_ctx, dtype="int8")
    for b in range(8):
        model.prefill(ids_t(syn.token_ids(w.seq, w.seed, f"ctxprompt.lane{b}")), L=8, kv=kv,
                      lane=b)
    ids8 = [ids_t(np.array([syn.decode_ids(w, b)[s] for b in range(8)])) for s in range(w.steps)]
    y8 = torch.empty(8, 2048, dtype=torch.float32, device="cuda")
    it2 = iter(range(10 ** 9))

    def dstep8():
        model.decode(kv, ids8[next(it2) % w.steps], L_per_lane=list(w.L), y_out=y8)

    dstep8()
    for b in range(8):
        kv.set_position(b, w.seq)
    with torch.cuda.nvtx.range("decode_b8"):
        t = max_t(timed(dstep8, w.steps, 0))
    med = timed.last_median_ms
    avg_ctx = w.seq + (w.steps + 1) / 2
    kv_bytes = 8 * 10 * avg_ctx * 16 * (2 * 128 + 2 * 2)
    out["b8_int8kv_ctx2048"] = {"tok_s": round(8 * w.steps * world / t, 1),
                                "ms_per_step": round(t / w.steps * 1e3, 4),
                                "ms_per_step_median": round(med, 4),
                                **decode_roofline(t / w.steps, 3 * blk_bytes + kv_bytes,
                                                  7 * blk_bytes, hbm, l2_gbs),
                                "workload": "batch 8, context 2048 + 64 steps, L=8, INT8 KV"}
    kv.close()
    torch.cuda.synchronize()

    # mixed-depth INT3 loop block, lanes L = [4, 16, 32], context 1024
    w = syn.WORKLOADS["mixed_int3"]
    loop3 = DeviceBlock(cfg(3), weights=syn.block_weights(w.shape, w.seed, "loop"))
    m3 = DeviceModel([blocks["pre0"], blocks["pre1"]], loop3, syn.final_gain(w.shape, w.seed),
                     syn.embedding(w.shape, w.seed), max_tokens=1024, max_lanes=3,
                     max_ctx=w.max_ctx, max_L=32)
    kv = m3.new_kv(list(w.L), max_ctx=w.max_ctx)
    for b in range(3):
        m3.prefill(ids_t(syn.prompt_ids(w, b)), L=w.L[b], kv=kv, lane=b)
    ids3 = [ids_t(np.array([syn.decode_ids(w, b)[s] for b in range(3)])) for s in range(w.steps)]
    y3 = torch.empty(3, 2048, dtype=torch.float32, device="cuda")
    it3 = iter(range(10 ** 9))

    def dstep3():
        m3.decode(kv, ids3[next(it3) % w.steps], L_per_lane=list(w.L), y_out=y3)

    dstep3()
    for b in range(3):
        kv.set_position(b, w.seq)
    with torch.cuda.nvtx.range("decode_b3"):
        t = max_t(timed(dstep3, w.steps, 0))
    med = timed.last_median_ms
    avg_ctx = w.seq + (w.steps + 1) / 2
    slots = sum(2 + L for L in w.L)
    kv_bytes = slots * avg_ctx * 2048 * 2 * 2
    loop_bytes = loop_read_bytes(tl, loop3)
    out["b3_int3_mixedL"] = {"tok_s": round(3 * w.steps * world / t, 1),
                             "ms_per_step": round(t / w.steps * 1e3, 4),
                             "ms_per_step_median": round(med, 4),
                             **decode_roofline(t / w.steps, 2 * blk_bytes + loop_bytes + kv_bytes,
                                               (max(w.L) - 1) * loop_bytes, hbm, l2_gbs),
                             "loop_block_bytes_read": loop_bytes,
                             "workload": "lanes L=[4,16,32], INT3 loop block, context 1024 + "
                                         "32 steps, FP16 KV"}
    kv.close()
    m3.close()
    loop3.close()
    return out


def main():
    args = parse()
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    dist = None
    if world > 1:
        import datetime
        import torch
        import torch.distributed as tdist
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", 0)))
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        dist = tdist
    line = run_ours(args, rank, world, dist)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
