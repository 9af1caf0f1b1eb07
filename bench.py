"""Benchmark of the gated delta rule hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = chunked prefill (gdn_chunk_fwd) + the sigmoid-gate zero-centred RMSNorm
epilogue (gdn_gate_norm) over one batch of the prefill workload; the same step as one
library call (gdn_chunk_fwd_gated: y into o, then the gate-norm in place) is timed beside
it under "fused_step". The workload: 4 sequences x 4096
tokens, H = 16, d_k = d_v = 128, chunk 64, bf16 q/k/v, fp32 state. Inputs are seeded
synthetic draws (workloads/), resident in HBM before the timed region; q, k, v and z
(256 MiB) exceed the 126 MB L2, so no flush is needed between steps.

The decode step (256 sequences x 32 heads, d = 128, 537 MB fp32 state in HBM) is timed
separately and reported under "decode"; the featurisation step in front of the prefill
(gdn_featurize on the prefill workload's shape) under "featurize"; the prefill alone on
the long-context workload (one 65,536-token sequence, H = 32, S0 != 0) and on the packed
variable-length batch (8 sequences, H = 16) under "prefill_long" and "prefill_varlen".

Multi-GPU (torchrun, one process per GPU): every rank runs its own independent batch
(the chains do not interact), so scaling is weak and the data path has no collective;
timing is the max over ranks of the device-timed region.

--impl reference runs the fp64 CPU oracle on the host cores (rank 0 only) on bounded
samples of the same workload; it is the slow reference arm, not a target.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "GDN prefill tokens/s + % tensor peak; decode-step state GB/s vs HBM peak"
UNIT = "tokens/s"
WORKLOAD = ("prefill bf16: 4 seqs x 4096 tokens, H=16, d_k=d_v=128, chunk 64, fp32 state, "
            "bf16 y, then sigmoid-gate zero-centred RMSNorm (bf16 z and o)")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
KERNEL_SOURCES = ["gated_deltanet_05_b200/csrc/gdn_chunk_sm100.cuh",
                  "gated_deltanet_05_b200/csrc/sm100_ptx.cuh"]


def flops_per_token_head(chunk: int, d: int) -> float:
    """Canonical chunked-form FLOPs per (token, head), full C x C tiles: five C x d
    products at 2Cd (K K^T, Q K^T, T K, T V, P U~), three d x d products at 2d^2
    (W S, Q S, state update) and the C x C solve at C^2/3."""
    return 10.0 * chunk * d + 6.0 * d * d + chunk * chunk / 3.0


def prefill_bytes_per_token_head(in_elem: int, y_elem: int, d: int) -> float:
    """Minimal HBM bytes per (token, head): read q, k, v (3 d in_elem), write y (d y_elem),
    read log_alpha and beta (8 bytes)."""
    return 3 * in_elem * d + y_elem * d + 8.0


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic():
    """DRAM bytes per launch of the prefill kernel from the committed ncu summary, if it
    was taken on the current kernel source (else None)."""
    path = os.path.join(ROOT, "profiles", "chunk_fwd_bf16_prefill.json")
    try:
        with open(path) as f:
            rec = json.load(f)
    except (OSError, ValueError):
        return None
    if rec.get("kernel_source_hash") != kernel_source_hash():
        return None
    return rec.get("dram_bytes_per_launch")


class ClockSampler:
    """nvidia-smi clocks and throttle reasons, sampled in the background."""

    QUERY = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.file = None

    def start(self):
        try:
            self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=self.file, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        return self

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.12)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.file.flush()
        self.file.seek(0)
        rows = [r.split(", ") for r in self.file.read().strip().splitlines() if r.strip()]
        os.unlink(self.file.name)
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            if len(r) < 10:
                continue
            try:
                sm.append(float(r[2]))
                mx = float(r[3])
            except ValueError:
                continue
            for n, val in zip(names, r[6:10]):
                if val.strip().lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def dist_setup(args):
    import torch
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus and "WORLD_SIZE" in os.environ:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if args.impl == "ours" else "gloo"
        if args.impl == "ours":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
        pg = dist
    elif args.impl == "ours":
        torch.cuda.set_device(local)
    return rank, world, local, pg


def max_over_ranks(pg, value: float, device):
    if pg is None:
        return value
    import torch
    t = torch.tensor([value], dtype=torch.float64, device=device)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return float(t.item())


def barrier(pg, device=None):
    if pg is not None:
        if device is not None:
            pg.barrier(device_ids=[device.index])
        else:
            pg.barrier()


# ------------------------------------------------------------------------------ CPU oracle
def oracle_sample(inp, seq_heads, n_threads=0):
    """Run the fp64 oracle on the given (sequence, head) chains of a prefill input;
    returns (token-heads processed, seconds, threads used)."""
    import numpy as np
    import torch

    import oracle
    seqs = sorted({s for s, _ in seq_heads})
    heads = sorted({h for _, h in seq_heads})
    cu = inp["cu_seqlens"].tolist()
    idx = torch.from_numpy(np.concatenate([np.arange(cu[s], cu[s + 1]) for s in seqs]))
    hs = torch.tensor(heads)
    sel = {k: inp[k].index_select(0, idx).index_select(1, hs)
           for k in ("q", "k", "v", "log_alpha", "beta")}
    lens = [cu[s + 1] - cu[s] for s in seqs]
    cu_sub = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    t0 = time.perf_counter()
    _, _, used = oracle.recurrent(sel["q"], sel["k"], sel["v"], sel["log_alpha"], sel["beta"],
                                  cu_sub, n_threads=n_threads)
    dt = time.perf_counter() - t0
    return int(sum(lens)) * len(heads), dt, used


def run_reference(args, rank, world, pg):
    if rank != 0:
        return
    import workloads as W
    w = W.WORKLOADS["prefill"]
    inp = W.make_prefill_inputs(w, with_gate=False)
    cores = os.cpu_count() or 1
    H = w.H
    n_seq = len(w.lengths)
    # one step = one bounded sample: `cores` chains (whole sequences), rotating over the batch
    chains = [(s, h) for h in range(H) for s in range(n_seq)]
    per_step = max(1, min(cores, len(chains)))
    done, elapsed, used = 0, 0.0, 1
    for i in range(args.warmup + args.steps):
        pick = [chains[(i * per_step + j) % len(chains)] for j in range(per_step)]
        # a square sample: every listed sequence with every listed head
        seqs = sorted({s for s, _ in pick})
        heads = sorted({h for _, h in pick})
        n_th, dt, used = oracle_sample(inp, [(s, h) for s in seqs for h in heads])
        if i >= args.warmup:
            done += n_th
            elapsed += dt
    th_per_s = done / elapsed
    value = th_per_s / H
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * elapsed / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD, "global_batch": 4, "seq_len": 4096, "heads": 16,
                   "parallelism": "host threads"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": used, "kind": "oracle",
                         "sample": f"per step: whole 4096-token chains of the prefill workload, "
                                   f"{per_step} (sequence, head) pairs; {done} token-heads timed"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------------------ our arm
def run_ours(args, rank, world, local, pg):
    import torch

    import gated_deltanet_05_b200 as gdn
    import workloads as W

    device = torch.device("cuda", local)
    w = W.WORKLOADS["prefill"]
    H, d, C = w.H, w.d_k, w.chunk
    inp = W.make_prefill_inputs(w, seed=w.seed + 1000 * rank)
    n_tok = int(inp["cu_seqlens"][-1])
    dev = {k: (v.to(device) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    cu_host = inp["cu_seqlens"]
    y = torch.empty((n_tok, H, d), dtype=torch.bfloat16, device=device)
    o = torch.empty((n_tok, H, d), dtype=torch.bfloat16, device=device)
    stream = torch.cuda.current_stream(device)

    def step(ev=None):
        # the whole hot path: chunked prefill (bf16 y), then the gate-norm epilogue
        if ev is not None:
            ev[0].record(stream)
        gdn.chunk_fwd(dev["q"], dev["k"], dev["v"], dev["log_alpha"], dev["beta"],
                      dev["cu_seqlens"], chunk=C, cu_seqlens_host=cu_host, out=y,
                      final_state=True)
        if ev is not None:
            ev[1].record(stream)
        gdn.gate_norm(y, dev["z"], dev["w_norm"], out=o)
        if ev is not None:
            ev[2].record(stream)

    def fused_step(ev):
        ev[0].record(stream)
        gdn.chunk_fwd_gated(dev["q"], dev["k"], dev["v"], dev["log_alpha"], dev["beta"],
                            dev["cu_seqlens"], dev["z"], dev["w_norm"], chunk=C,
                            cu_seqlens_host=cu_host, out=o, final_state=True)
        ev[1].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(device)
    status = gdn.device_error(device)
    if status != "GDN_OK":
        raise SystemExit(f"device error after warm-up: {status}")

    # timed region: K steps, per-kernel events inside
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(local).start()
    time.sleep(0.2)
    barrier(pg, device)
    torch.cuda.synchronize(device)
    t_start.record(stream)
    for i in range(args.steps):
        step(evs[i])
    t_end.record(stream)
    torch.cuda.synchronize(device)
    barrier(pg, device)
    clocks = sampler.stop()
    elapsed_ms = t_start.elapsed_time(t_end)
    elapsed_ms = max_over_ranks(pg, elapsed_ms, device)
    chunk_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    gn_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
    # the same step as one gdn_chunk_fwd_gated call (y into o, then the gate-norm in place)
    fevs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(20)]
    for e in fevs:
        fused_step(e)
    torch.cuda.synchronize(device)
    fused_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in fevs)
    ms_per_step = elapsed_ms / args.steps
    tokens_per_step = n_tok * world
    value = tokens_per_step / (ms_per_step * 1e-3)

    peaks, peak_kind = load_peaks()
    token_heads = n_tok * H
    flops = flops_per_token_head(C, d) * token_heads
    algo_bytes = prefill_bytes_per_token_head(2, 2, d) * token_heads + len(w.lengths) * H * d * d * 4
    chunk_s = chunk_ms * 1e-3
    tflops = flops / chunk_s / 1e12
    gbs = algo_bytes / chunk_s / 1e9
    t_tensor = flops / (peaks["bf16_tflops"] * 1e12)
    t_hbm = algo_bytes / (peaks["hbm_gbs"] * 1e9)
    roofline = {
        "kernel": "gdn::sm100::chunk_fwd_bf16_kernel",
        "bound": "hbm" if t_hbm >= t_tensor else "tensor",
        "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
        "frac": gbs / peaks["hbm_gbs"], "peak_source": f"{peak_kind} hbm_gbs",
        "traffic": profiled_traffic(),
        "algorithmic_bytes_per_launch": algo_bytes,
        "launch_ms": chunk_ms,
        "tensor": {"achieved": tflops, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                   "frac": tflops / peaks["bf16_tflops"],
                   "peak_source": f"{peak_kind} bf16_tflops (burst)",
                   "flops_per_launch": flops,
                   "flops_per_token_head": flops_per_token_head(C, d)},
    }
    gn_bytes = (2 + 2 + 2) * n_tok * H * d + 4 * d          # y, z and o bf16
    gate_norm_obj = {"launch_ms": gn_ms, "achieved": gn_bytes / (gn_ms * 1e-3) / 1e9,
                     "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": gn_bytes / (gn_ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
                     "bytes_per_launch": gn_bytes}
    fused = {"ms_per_step": fused_ms,
             "note": "the same step as one gdn_chunk_fwd_gated call (two launches: y into o, then "
                     "the gate-norm in place on o), 20 steps"}

    shapes = {} if args.no_shapes else {
        "long": bench_prefill_shape(args, "long", device, peaks, peak_kind, pg, rank),
        "varlen": bench_prefill_shape(args, "varlen", device, peaks, peak_kind, pg, rank)}
    decode = None if args.no_decode else bench_decode(args, device, peaks, peak_kind, pg)
    qsa = None if args.no_shapes else bench_qsa(args, device, peaks, pg, rank)
    featurize = bench_featurize(args, device, peaks, peak_kind, pg, rank)
    backward = bench_backward(args, inp, device, pg) if world == 1 else None
    e2e = bench_e2e(args, inp, device, pg, world)

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded draws: L2-normalised q,k ~ N(0,1); v ~ N(0,1); "
                "beta = sigmoid(N(0,1)); log alpha = -exp(A) softplus(N(0,1)), A ~ U(-1,1))",
        "config": {"workload": WORKLOAD, "global_batch": 4 * world, "seq_len": 4096,
                   "heads": H, "d_k": d, "d_v": d, "chunk": C, "parallelism": f"dp{world}",
                   "l2": "no flush: q, k, v, z are 256 MiB per step, above the 126 MB L2"},
        "roofline": roofline,
        "prefill_long": shapes.get("long"),
        "prefill_varlen": shapes.get("varlen"),
        "gate_norm": gate_norm_obj,
        "fused_step": fused,
        "decode": decode,
        "featurize": featurize,
        "qsa_indexer": qsa,
        "backward": backward,
        "e2e": e2e,
        "gpu_launches": 2 * args.steps,
        "clocks": clocks,
    }
    if rank == 0 and not args.no_cpu_baseline and world == 1:
        line["cpu_baseline"] = cpu_baseline(inp, H)
    if rank == 0:
        print(json.dumps(line), flush=True)


def bench_prefill_shape(args, name, device, peaks, peak_kind, pg, rank):
    """gdn_chunk_fwd alone (bf16 y, S_T written) on another prefill workload: "long" (one
    65,536-token sequence, H = 32, S0 != 0, A ~ U(-3, 1)) or "varlen" (8 packed sequences
    of U[512, 8192] tokens, H = 16). Roofline bytes per launch: q, k, v, y in bf16 and the
    fp32 gates per token-head, plus S_T (and S0 when present) per chain."""
    import torch

    import gated_deltanet_05_b200 as gdn
    import workloads as W
    w = W.WORKLOADS[name]
    inp = W.make_prefill_inputs(w, with_gate=False, seed=w.seed + 1000 * rank)
    dev = {k: (v.to(device) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    n_tok = int(inp["cu_seqlens"][-1])
    n_seq = inp["cu_seqlens"].numel() - 1
    H, d, C = w.H, w.d_k, w.chunk
    y = torch.empty((n_tok, H, d), dtype=torch.bfloat16, device=device)
    S_T = torch.empty((n_seq, H, d, d), dtype=torch.float32, device=device)
    cu_host = inp["cu_seqlens"]
    stream = torch.cuda.current_stream(device)

    def run():
        gdn.chunk_fwd(dev["q"], dev["k"], dev["v"], dev["log_alpha"], dev["beta"], dev["cu_seqlens"],
                      S0=dev.get("S0"), chunk=C, cu_seqlens_host=cu_host, out=y, state_out=S_T)

    for _ in range(max(3, args.warmup)):
        run()
    torch.cuda.synchronize(device)
    reps = 10
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    barrier(pg, device)
    a.record(stream)
    for _ in range(reps):
        run()
    b.record(stream)
    torch.cuda.synchronize(device)
    status = gdn.device_error(device)
    if status != "GDN_OK":
        raise SystemExit(f"device error in the {name} prefill leg: {status}")
    ms = max_over_ranks(pg, a.elapsed_time(b), device) / reps
    token_heads = n_tok * H
    n_states = (2 if dev.get("S0") is not None else 1) * n_seq * H
    algo_bytes = prefill_bytes_per_token_head(2, 2, d) * token_heads + n_states * d * d * 4
    flops = flops_per_token_head(C, d) * token_heads
    gbs = algo_bytes / (ms * 1e-3) / 1e9
    tflops = flops / (ms * 1e-3) / 1e12
    return {"workload": f"{name} bf16: {n_seq} seq(s), {n_tok} tokens, H={H}, d={d}, chunk {C}, "
                        f"bf16 y" + (", S0 != 0" if dev.get("S0") is not None else ""),
            "chains": n_seq * H, "launch_ms": ms, "tokens_per_s": n_tok / (ms * 1e-3),
            "bytes_per_launch": algo_bytes, "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": gbs / peaks["hbm_gbs"], "peak_source": f"{peak_kind} hbm_gbs",
            "tensor": {"achieved": tflops, "unit": "TFLOP/s", "frac": tflops / peaks["bf16_tflops"],
                       "flops_per_launch": flops},
            "launches": reps, "l2": "inputs above the 126 MB L2"}


def bench_qsa(args, device, peaks, pg, rank):
    """The QSA compressed indexer (gdn_qsa_indexer: vectors, tensor-core scores, top-K) on
    one 16,384-token sequence, Hq = 4, r = 4, K = 2048, bf16. The score FLOPs count every
    visible (token, block) pair: 2 * 128 * Hq per pair."""
    import torch

    import gated_deltanet_05_b200 as gdn
    import workloads as W
    cfg = W.QSA_WORKLOAD
    inp = W.make_qsa_inputs(cfg["lengths"], cfg["Hq"], cfg["dtype"], seed=cfg["seed"] + 1000 * rank)
    d = {k: inp[k].to(device) for k in ("qx", "kx", "wq", "wk", "cu_seqlens")}
    r, K, Hq = cfg["r"], cfg["K"], cfg["Hq"]
    n = int(inp["cu_seqlens"][-1])
    nb = n // r
    kb = -(-K // r)
    out = (torch.empty((n, nb), dtype=torch.float32, device=device),
           torch.empty((n, kb), dtype=torch.int32, device=device))
    stream = torch.cuda.current_stream(device)

    def run():
        gdn.qsa_indexer(d["qx"], d["kx"], d["wq"], d["wk"], d["cu_seqlens"], r=r, K=K,
                        cu_seqlens_host=inp["cu_seqlens"], out=out)

    for _ in range(max(3, args.warmup)):
        run()
    torch.cuda.synchronize(device)
    reps = 20
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    barrier(pg, device)
    a.record(stream)
    for _ in range(reps):
        run()
    b.record(stream)
    torch.cuda.synchronize(device)
    status = gdn.device_error(device)
    if status != "GDN_OK":
        raise SystemExit(f"device error in the QSA leg: {status}")
    ms = max_over_ranks(pg, a.elapsed_time(b), device) / reps
    pairs = sum(min(nb, (i + 1) // r) for i in range(n))
    flops = 2.0 * 128 * Hq * pairs
    return {"workload": f"QSA indexer bf16: 1 seq x {n} tokens, Hq={Hq}, d=128, r={r}, K={K} (K_B={kb})",
            "kernels": "qsa_setup, qsa_vectors, qsa_scores_tc (tcgen05), qsa_topk",
            "ms_per_call": ms, "tokens_per_s": n / (ms * 1e-3), "visible_pairs": pairs,
            "score_flops": flops, "score_tflops_over_call": flops / (ms * 1e-3) / 1e12,
            "score_bytes_written": 4 * pairs, "launches": reps}


def bench_decode(args, device, peaks, peak_kind, pg):
    """Decode step: 256 sequences x 32 heads, d = 128, fp32 state resident in HBM."""
    import torch

    import gated_deltanet_05_b200 as gdn
    import workloads as W
    w = W.WORKLOADS["decode"]
    n, H, d = w.n_seq_decode, w.H, w.d_k
    n_inputs = 8                                    # distinct staged steps, cycled
    staged = []
    for s in range(n_inputs):
        x = W.make_decode_inputs(w, s)
        staged.append({k: v.to(device) for k, v in x.items()})
    S = torch.zeros((n, H, d, d), dtype=torch.float32, device=device)
    y = torch.empty((n, H, d), dtype=torch.float32, device=device)
    stream = torch.cuda.current_stream(device)

    def one(i):
        x = staged[i % n_inputs]
        gdn.decode_step(x["q"], x["k"], x["v"], x["alpha"], x["beta"], S, out=y)

    for i in range(max(3, args.warmup)):
        one(i)
    torch.cuda.synchronize(device)
    steps = max(args.steps, 50)
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    barrier(pg, device)
    a.record(stream)
    for i in range(steps):
        one(i)
    b.record(stream)
    torch.cuda.synchronize(device)
    ms = max_over_ranks(pg, a.elapsed_time(b), device) / steps
    state_bytes = n * H * d * d * 4
    step_bytes = 2 * state_bytes + n * H * (3 * d * 4 + d * 4 + 8)
    gbs = step_bytes / (ms * 1e-3) / 1e9

    # several tokens per call (next_n = 4): one pass over the state for 4 tokens
    nt = 4
    staged_t = []
    for s_ in range(4):
        xs = [W.make_decode_inputs(w, 1000 + s_ * nt + i) for i in range(nt)]
        staged_t.append({key: torch.stack([x[key] for x in xs], 1).contiguous().to(device)
                         for key in ("q", "k", "v", "alpha", "beta")})
    y_t = torch.empty((n, nt, H, d), dtype=torch.float32, device=device)

    def multi(i):
        x = staged_t[i % len(staged_t)]
        gdn.decode_tokens(x["q"], x["k"], x["v"], x["alpha"], x["beta"], S, out=y_t)

    for i in range(max(3, args.warmup)):
        multi(i)
    torch.cuda.synchronize(device)
    barrier(pg, device)
    a.record(stream)
    for i in range(steps):
        multi(i)
    b.record(stream)
    torch.cuda.synchronize(device)
    ms_t = max_over_ranks(pg, a.elapsed_time(b), device) / steps
    call_bytes = 2 * state_bytes + nt * n * H * (3 * d * 4 + d * 4 + 8)
    gbs_t = call_bytes / (ms_t * 1e-3) / 1e9
    status = gdn.device_error(device)
    if status != "GDN_OK":
        raise SystemExit(f"device error in the decode leg: {status}")
    return {"workload": "decode fp32 state: 256 seqs x H=32, d_k=d_v=128, one token per step",
            "ms_per_step": ms, "tokens_per_s": n / (ms * 1e-3), "bytes_per_step": step_bytes,
            "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": gbs / peaks["hbm_gbs"], "peak_source": f"{peak_kind} hbm_gbs",
            "steps": steps, "l2": "state 537 MB > L2",
            "tokens_4": {"kernel": "gdn::decode_tokens_kernel", "tokens_per_call": nt,
                         "ms_per_call": ms_t, "tokens_per_s": n * nt / (ms_t * 1e-3),
                         "bytes_per_call": call_bytes, "achieved": gbs_t, "unit": "GB/s",
                         "frac": gbs_t / peaks["hbm_gbs"]}}


def bench_featurize(args, device, peaks, peak_kind, pg, rank):
    """The featurisation step in front of the prefill (short conv, SiLU, L2 norm, gates)
    on the prefill workload's shape: 4 x 4096 tokens, H = 16, d = 128, bf16 streams."""
    import torch

    import gated_deltanet_05_b200 as gdn
    import workloads as W
    w = W.WORKLOADS["prefill"]
    inp = W.make_featurize_inputs(w, seed=w.seed + 7 + 1000 * rank)
    keys = ("xq", "xk", "xv", "conv_q", "conv_k", "conv_v", "beta_logit", "alpha_logit", "A",
            "b_alpha", "cu_seqlens")
    dev = [inp[k].to(device) for k in keys]
    n_tok, H, d = inp["xq"].shape
    cu_host = inp["cu_seqlens"]
    out = (torch.empty_like(dev[0]), torch.empty_like(dev[1]), torch.empty_like(dev[2]),
           torch.empty((n_tok, H), dtype=torch.float32, device=device),
           torch.empty((n_tok, H), dtype=torch.float32, device=device))
    stream = torch.cuda.current_stream(device)
    for _ in range(max(3, args.warmup)):
        gdn.featurize(*dev, cu_seqlens_host=cu_host, out=out)
    torch.cuda.synchronize(device)
    steps = max(args.steps, 20)
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    barrier(pg, device)
    a.record(stream)
    for _ in range(steps):
        gdn.featurize(*dev, cu_seqlens_host=cu_host, out=out)
    b.record(stream)
    torch.cuda.synchronize(device)
    status = gdn.device_error(device)
    if status != "GDN_OK":
        raise SystemExit(f"device error in the featurisation leg: {status}")
    ms = max_over_ranks(pg, a.elapsed_time(b), device) / steps
    # read x (3 streams) + 2 logits, write q, k, v + beta, log alpha; plus the weights
    step_bytes = n_tok * H * 2 * (3 * d * 2 + 2 * 4) + 3 * H * d * 4 * 4 + 2 * H * 4
    gbs = step_bytes / (ms * 1e-3) / 1e9
    return {"workload": "featurisation bf16: 4 seqs x 4096 tokens, H=16, d=128, conv width 4",
            "kernel": "gdn::featurize_kernel (2 launches)", "launch_ms": ms,
            "bytes_per_launch": step_bytes, "achieved": gbs, "peak": peaks["hbm_gbs"],
            "unit": "GB/s", "frac": gbs / peaks["hbm_gbs"], "peak_source": f"{peak_kind} hbm_gbs",
            "steps": steps, "l2": "inputs 192 MiB > L2"}


def bench_backward(args, inp, device, pg):
    """The backward (gdn_backward) on the prefill workload, a few launches. Guarded: a
    failure here is reported in the line instead of ending the run."""
    import torch

    import gated_deltanet_05_b200 as gdn
    try:
        dev = {k: inp[k].to(device) for k in ("q", "k", "v", "log_alpha", "beta", "cu_seqlens", "z")}
        dy = dev["z"]                           # any bf16 [N, H, d_v] cotangent
        cu_host = inp["cu_seqlens"]
        run = lambda: gdn.backward(dev["q"], dev["k"], dev["v"], dev["log_alpha"], dev["beta"],
                                   dev["cu_seqlens"], dy, cu_seqlens_host=cu_host)
        run()
        torch.cuda.synchronize(device)
        reps = 3
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        barrier(pg, device)
        a.record()
        for _ in range(reps):
            run()
        b.record()
        torch.cuda.synchronize(device)
        ms = max_over_ranks(pg, a.elapsed_time(b), device) / reps
        status = gdn.device_error(device)
        n_tok = inp["q"].shape[0]
        # products of the chunked backward per (chain, 64-token chunk), full C x C tiles:
        # 24 C^2 d + 16 C d^2 FLOP (prep [K; Q] K^T and W: 6 C^2 d; state chain forward
        # T V, W S, K^T U~: 2 C^2 d + 4 C d^2; state adjoints P^T dY, K dS', Q^T dY, W^T dU~:
        # 2 C^2 d + 6 C d^2; sums over v T^T dU~, dY U~^T, X U~^T, dU~ S^T, U~ dS'^T, dY S^T:
        # 6 C^2 d + 6 C d^2; dq/dk T^T dW, (dP o Gamma) K, (dP o Gamma)^T Q, (dA + dA^T) K: 8 C^2 d)
        C, d, H = 64, inp["q"].shape[2], inp["q"].shape[1]
        lens = (inp["cu_seqlens"][1:] - inp["cu_seqlens"][:-1]).tolist()
        n_cc = H * sum(-(-L // C) for L in lens)
        flops = n_cc * (24 * C * C * d + 16 * C * d * d)
        tf = flops / (ms * 1e-3) / 1e12
        # the products run as tf32 mma.sync with a two-part operand split (three tensor-core
        # products per product); peak: dense tf32 = measured bf16 x the nominal 1.1 / 2.25
        peaks, kind = load_peaks()
        peak_tf32 = peaks["bf16_tflops"] * 1.1 / 2.25
        fma_peak = 148 * 128 * 2 * 1.965e9 / 1e12
        return {"kernel": "gdn::bwdc chunked backward (prep, fwd, state, vpart, kpart; tf32x3 mma.sync)",
                "ms_per_launch": ms, "tokens_per_s": n_tok / (ms * 1e-3), "launches": reps, "status": status,
                "workload": "prefill shape: 4 x 4096 tokens, H=16, d=128, bf16 inputs",
                "roofline": {"bound": "tensor", "achieved": tf, "peak": peak_tf32, "unit": "TFLOP/s",
                             "frac": tf / peak_tf32, "peak_source": f"{kind} bf16_tflops x 1.1/2.25 (tf32)",
                             "flops_per_launch": flops, "tensor_products_per_product": "3, or 2 (1) with one (two) bf16 input operands",
                             "fp32_fma_peak": fma_peak, "fp32_fma_frac": tf / fma_peak}}
    except Exception as exc:                      # reported, not raised
        return {"error": f"{type(exc).__name__}: {exc}"[:300]}


def bench_e2e(args, inp, device, pg, world):
    """Same step through the public API with the inputs in pinned host memory: H2D copy of
    q, k, v, log_alpha, beta, z every step, D2H read of the output o. Steps are pipelined
    over three streams and two device buffer sets: step i's inputs go up while step i - 1
    computes and step i - 2's output comes down (H2D and D2H use separate copy engines)."""
    import torch

    import gated_deltanet_05_b200 as gdn
    H, C = inp["H"], inp["chunk"]
    host = {k: inp[k].pin_memory() for k in ("q", "k", "v", "log_alpha", "beta", "z")}
    w_dev = inp["w_norm"].to(device)
    cu_host = inp["cu_seqlens"]
    cu_dev = cu_host.to(device)
    dev = [{k: torch.empty_like(v, device=device) for k, v in host.items()} for _ in range(2)]
    outs = [None, None]
    o_host = [torch.empty(inp["v"].shape, dtype=inp["v"].dtype).pin_memory() for _ in range(2)]
    s_in = torch.cuda.Stream(device)
    s_cmp = torch.cuda.Stream(device)
    s_out = torch.cuda.Stream(device)
    done_cmp = [torch.cuda.Event(), torch.cuda.Event()]   # buffer set free again
    done_out = [torch.cuda.Event(), torch.cuda.Event()]   # output buffer read back
    h2d = sum(v.numel() * v.element_size() for v in host.values())
    d2h = o_host[0].numel() * o_host[0].element_size()
    first = [True, True]

    def step(i):
        j = i & 1
        with torch.cuda.stream(s_in):
            if not first[j]:
                s_in.wait_event(done_cmp[j])      # step i - 2 has finished reading this set
            for k in host:
                dev[j][k].copy_(host[k], non_blocking=True)
            up = torch.cuda.Event()
            up.record(s_in)
        with torch.cuda.stream(s_cmp):
            s_cmp.wait_event(up)
            if not first[j]:
                s_cmp.wait_event(done_out[j])     # step i - 2's output has been read back
            d = dev[j]
            y, _ = gdn.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], cu_dev,
                                 chunk=C, cu_seqlens_host=cu_host, y_dtype=torch.bfloat16)
            outs[j] = gdn.gate_norm(y, d["z"], w_dev, out_dtype=torch.bfloat16)
            done_cmp[j].record(s_cmp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(done_cmp[j])
            o_host[j].copy_(outs[j], non_blocking=True)
            done_out[j].record(s_out)
        first[j] = False

    for i in range(2):
        step(i)
    torch.cuda.synchronize(device)
    steps = max(1, min(args.steps, 20))
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    barrier(pg, device)
    a.record(s_in)
    for i in range(steps):
        step(i)
    s_in.wait_stream(s_out)
    b.record(s_in)
    torch.cuda.synchronize(device)
    ms = max_over_ranks(pg, a.elapsed_time(b), device) / steps
    n_tok = inp["q"].shape[0]
    return {"value": n_tok * world / (ms * 1e-3), "unit": UNIT, "ms_per_step": ms,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": steps,
            "pipelined": "3 streams, 2 device buffer sets: H2D of step i, compute of i - 1, D2H of i - 2"}


def cpu_baseline(inp, H, min_seconds=10.0, max_reps=12):
    """The fp64 oracle on the host cores over a bounded sample of the same workload: every
    (sequence, head) chain of the batch, repeated until about min_seconds of CPU time."""
    n_seq = inp["cu_seqlens"].numel() - 1
    pairs = [(s, h) for s in range(n_seq) for h in range(H)]
    done, elapsed, reps, used = 0, 0.0, 0, 1
    while reps < max_reps and (reps == 0 or elapsed < min_seconds):
        n_th, dt, used = oracle_sample(inp, pairs)
        done += n_th
        elapsed += dt
        reps += 1
    return {"value": done / elapsed / H, "unit": UNIT, "cores": used, "kind": "oracle",
            "sample": f"all {len(pairs)} (sequence, head) chains of the prefill workload, "
                      f"{reps} pass(es): {done} token-heads in {elapsed:.1f} s; "
                      f"tokens/s = token-heads/s / H"}


def run_case(args):
    """A few launches of one kernel on a named shape, nothing else (for ncu captures):
    --case prefill:S,T,H   (bf16, d=128, chunk 64, bf16 y)
    --case prefill_gated:S,T,H (the same with the fused gate-norm, bf16 z and o)
    --case decode:N        (N sequences x 32 heads, d=128, fp32 state)
    --case gate_norm:R     (R rows of d_v = 128: bf16 y, z and o, as in the bench step)
    --case featurize:S,T,H (bf16, d=128, conv width 4)
    --case decode_tokens:N,T (N sequences x 32 heads, d=128, T tokens per call)
    --case qsa:N           (the QSA indexer on one N-token sequence, Hq=4, r=4, K=2048, bf16)
    --case backward:S,T,H  (gdn_backward, bf16 inputs, d=128, a bf16 cotangent of y)"""
    import torch

    import gated_deltanet_05_b200 as gdn
    import workloads as W
    kind, _, shape = args.case.partition(":")
    dims = [int(x) for x in shape.split(",")] if shape else []
    torch.cuda.set_device(0)
    if kind == "prefill":
        n_seq, T, H = dims
        w = W.Workload("case", "bf16", (T,) * n_seq, H, 128, 128, 64, seed=1)
        inp = W.make_prefill_inputs(w, with_gate=False)
        d = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
        for _ in range(args.reps):
            gdn.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["cu_seqlens"],
                          cu_seqlens_host=inp["cu_seqlens"], y_dtype=torch.bfloat16)
    elif kind == "prefill_gated":
        n_seq, T, H = dims
        w = W.Workload("case", "bf16", (T,) * n_seq, H, 128, 128, 64, seed=1)
        inp = W.make_prefill_inputs(w)
        d = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
        for _ in range(args.reps):
            gdn.chunk_fwd_gated(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["cu_seqlens"],
                                d["z"], d["w_norm"], cu_seqlens_host=inp["cu_seqlens"])
    elif kind == "decode":
        (n,) = dims
        x = {k: v.cuda() for k, v in W.make_decode_inputs(W.WORKLOADS["decode"], 0, n_seq=n).items()}
        S = torch.zeros(n, 32, 128, 128, device="cuda")
        for _ in range(args.reps):
            gdn.decode_step(x["q"], x["k"], x["v"], x["alpha"], x["beta"], S)
    elif kind == "decode_tokens":
        n, nt = dims
        w = W.WORKLOADS["decode"]
        xs = [W.make_decode_inputs(w, i, n_seq=n) for i in range(nt)]
        x = {key: torch.stack([xi[key] for xi in xs], 1).contiguous().cuda()
             for key in ("q", "k", "v", "alpha", "beta")}
        S = torch.zeros(n, 32, 128, 128, device="cuda")
        for _ in range(args.reps):
            gdn.decode_tokens(x["q"], x["k"], x["v"], x["alpha"], x["beta"], S)
    elif kind == "gate_norm":
        (rows,) = dims
        g = torch.Generator().manual_seed(0)
        y = torch.randn(rows, 128, generator=g).to(torch.bfloat16).cuda()
        z = torch.randn(rows, 128, generator=g).to(torch.bfloat16).cuda()
        wn = (torch.randn(128, generator=g) * 0.02).cuda()
        for _ in range(args.reps):
            gdn.gate_norm(y, z, wn, out_dtype=torch.bfloat16)
    elif kind == "qsa":
        (n,) = dims
        inp = W.make_qsa_inputs((n,), 4, "bf16", seed=5)
        d = {k: inp[k].cuda() for k in ("qx", "kx", "wq", "wk", "cu_seqlens")}
        for _ in range(args.reps):
            gdn.qsa_indexer(d["qx"], d["kx"], d["wq"], d["wk"], d["cu_seqlens"], r=4, K=2048,
                            cu_seqlens_host=inp["cu_seqlens"])
    elif kind == "featurize":
        n_seq, T, H = dims
        w = W.Workload("case", "bf16", (T,) * n_seq, H, 128, 128, 64, seed=1)
        inp = W.make_featurize_inputs(w)
        keys = ("xq", "xk", "xv", "conv_q", "conv_k", "conv_v", "beta_logit", "alpha_logit", "A",
                "b_alpha", "cu_seqlens")
        dev = [inp[k].cuda() for k in keys]
        for _ in range(args.reps):
            gdn.featurize(*dev, cu_seqlens_host=inp["cu_seqlens"])
    elif kind == "backward":
        n_seq, T, H = dims
        w = W.Workload("case", "bf16", (T,) * n_seq, H, 128, 128, 64, seed=1)
        inp = W.make_prefill_inputs(w)
        d = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
        for _ in range(args.reps):
            gdn.backward(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["cu_seqlens"], d["z"],
                         cu_seqlens_host=inp["cu_seqlens"])
    else:
        raise SystemExit(f"unknown case {args.case}")
    torch.cuda.synchronize()
    status = gdn.device_error()
    print(f"case {args.case} x{args.reps}: {status}")
    if status != "GDN_OK":
        raise SystemExit(1)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-shapes", action="store_true", help="skip the long and varlen prefill legs")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--case", default=None, help="profiling case, e.g. prefill:4,4096,16")
    ap.add_argument("--reps", type=int, default=3)
    args = ap.parse_args()
    if args.case:
        run_case(args)
        return
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    rank, world, local, pg = dist_setup(args)
    try:
        if args.impl == "reference":
            run_reference(args, rank, world, pg)
        else:
            run_ours(args, rank, world, local, pg)
    finally:
        if pg is not None:
            pg.destroy_process_group()


if __name__ == "__main__":
    main()
