"""Benchmark of the Gated Delta Rule-2 hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = one ``gdn2_chunk_fwd`` over the 1.3B-layer workload (B=4, T=2048,
H=16, d_k=d_v=128, chunk 64, bf16 inputs, fp32 state, seeded synthetic data).
``value`` is tokens/s over all ranks (each rank runs its own batch; no
collective on the data path: weak scaling).  The same JSON line carries the
decode measurement (256 x 16 heads, 1024 single-token steps replayed from one
CUDA graph) as ``decode_step``, the block prologue and epilogue around the mixer
(``block_prologue``, ``block_epilogue``), the backward on the same workload
(``chunk_bwd``), the long-context workload with a sequence-length sweep
(``long_context``), the packed workload with its three gate variants (``varlen``),
the step sustained for about 0.5 s with its own clock samples (``sustained``), the
roofline of the chunk forward (its two kernels overlap, so the call is the unit),
the CPU oracle baseline, the end-to-end number through host buffers, and clocks.

``--impl reference`` times the fp64 CPU oracle (the only reference that
exists for this method) on a bounded sample of the same workload.
"""
import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

import gdn2_workloads as W  # noqa: E402

TOK = ("q", "k", "v", "alpha", "b", "w")
METRIC = "gdn2_chunk_fwd tokens/s and % bf16 TC peak; decode_step HBM GB/s (1 B200)"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ---------------------------------------------------------------- algorithmic work

def chunk_bytes(wl, tokens, n_seq):
    """Bytes the method must move: inputs + output in the token dtype, S0 read + S_T written in fp32."""
    es = 2 if wl.dtype == "bf16" else 4
    per_token_head = es * (4 * wl.dk + 2 * wl.dv) + es * wl.dv
    return tokens * wl.H * per_token_head + 2 * n_seq * wl.H * wl.dk * wl.dv * 4


def chunk_flops(wl, tokens):
    """Flops per token-head: the three d_k x d_v products (W S, K_hat^T Delta, Q_hat S) and the
    chunk-local triangular maps (erase interaction, solve, causal read)."""
    C = wl.chunk
    return tokens * wl.H * (6 * wl.dk * wl.dv + C * (3 * wl.dk + 2 * wl.dv))


def decode_bytes(wl):
    """Per step: the fp32 state read once and written once, plus the token inputs and o."""
    heads = wl.B * wl.H
    return heads * (2 * wl.dk * wl.dv * 4 + 2 * (4 * wl.dk + 2 * wl.dv) + 2 * wl.dv)


# ---------------------------------------------------------------- helpers

def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def traffic_record(kernel):
    """DRAM bytes per launch from a committed ncu summary, if the kernel source has not changed since."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f).get(kernel)
    if not rec:
        return None
    src = os.path.join(ROOT, rec["source"])
    if not os.path.exists(src) or hashlib.sha256(open(src, "rb").read()).hexdigest() != rec["source_sha256"]:
        return None
    return rec


class ClockSampler:
    """Polls SM clock and throttle reasons through NVML on a background thread."""

    REASONS = {  # NVML clocks-event reason bits
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
        0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
        0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting",
    }

    def __init__(self, device_index, period_s=0.0002):
        self.samples, self.period, self._stop = [], period_s, threading.Event()
        self.ok = False
        self.max_mhz = None
        try:
            import pynvml
            pynvml.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            try:
                self.h = pynvml.nvmlDeviceGetHandleByUUID(("GPU-" + uuid) if not uuid.startswith("GPU-") else uuid)
            except Exception:
                self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # noqa: BLE001
            self.err = repr(e)

    def _run(self):
        while not self._stop.is_set():
            try:
                mhz = self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM)
                rs = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                self.samples.append((time.perf_counter(), mhz, rs))
            except Exception:  # noqa: BLE001
                pass
            time.sleep(self.period)

    def start(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def stop(self):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self, t0, t1):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "note": "NVML unavailable"}
        inside = [s for s in self.samples if t0 <= s[0] <= t1]
        note = "sampled during the timed region"
        if len(inside) < 3:
            inside, note = self.samples, "timed region shorter than the sampling period; warm-up + timed window"
        reasons = set()
        for _, _, rs in inside:
            for bit, name in self.REASONS.items():
                if rs & bit and name != "gpu_idle":
                    reasons.add(name)
        mhz = [m for _, m, _ in inside]
        return {"sm_mhz": statistics.median(mhz) if mhz else None, "sm_max_mhz": self.max_mhz,
                "reasons": sorted(reasons), "samples": len(inside), "note": note}


def init_dist():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return ws, rank, local


def barrier(ws):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x, ws, device):
    if ws == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ---------------------------------------------------------------- reference arm (the fp64 oracle)

def oracle_sample(wl, seed, seqs, heads):
    """CPU inputs of a bounded sample of the workload: ``seqs`` sequences x ``heads`` heads."""
    d = [W.sequence_inputs(wl, n, device="cpu", seed=seed) for n in range(seqs)]
    x = {n: torch.stack([s[n][:, :heads] for s in d]).double().numpy() for n in TOK}
    S0 = torch.stack([s["S0"][:heads] for s in d]).double().numpy()
    return x, S0


def time_oracle(wl, seed, seqs, heads, reps=1):
    import oracle
    x, S0 = oracle_sample(wl, seed, seqs, heads)
    t0 = time.perf_counter()
    for _ in range(reps):
        oracle.recurrent(*[x[n] for n in TOK], S0=S0)
    dt = time.perf_counter() - t0
    tokens = seqs * wl.T * reps
    return tokens, dt, oracle.max_threads()


def run_reference(args, ws, rank):
    if rank != 0:
        return 0
    wl = W.WORKLOADS["layer_1p3b"]
    seqs, heads = 1, wl.H   # one sequence (2048 tokens) of the batch, all 16 heads, per step
    for _ in range(args.warmup):
        time_oracle(wl, 0, seqs, heads)
    total_tok, total_t, cores = 0, 0.0, 1
    for _ in range(args.steps):
        tok, dt, cores = time_oracle(wl, 0, seqs, heads)
        total_tok += tok
        total_t += dt
    value = total_tok / total_t
    sample = f"{seqs} sequence x {wl.T} tokens x {heads} heads of the layer_1p3b batch per step"
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total_t / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": {"workload": "layer_1p3b", "B": wl.B, "T": wl.T, "H": wl.H,
                                        "d_k": wl.dk, "d_v": wl.dv, "chunk": wl.chunk},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------- our arm

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-block", action="store_true", help="skip the block prologue/epilogue measurement")
    ap.add_argument("--no-bwd", action="store_true", help="skip the backward measurement")
    ap.add_argument("--no-workloads", action="store_true",
                    help="skip the long-context, sequence-length sweep and packed-varlen measurements")
    ap.add_argument("--profile-case", choices=["chunk", "decode", "block", "bwd", "bwd_small"],
                    help="run one warm-up and one measured launch of that kernel on its full workload, for ncu")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    ws, rank, local = init_dist()
    if args.impl == "reference":
        return run_reference(args, ws, rank)
    if args.profile_case:
        return profile_case(args.profile_case)

    import gated_delta_rule_131_b200 as gdn2
    gdn2.lib()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    wl = W.WORKLOADS["layer_1p3b"]
    tokens = wl.B * wl.T

    # this rank's shard of a global batch of ws x B sequences (each sequence has its own seeded
    # generator); two independent input sets, 2 x 235 MB > L2, alternated between steps
    mine = W.shard(wl.B * ws, ws, rank)
    sets = [W.chunk_inputs(wl, device=dev, seed=i, indices=mine) for i in range(2)]
    o = torch.empty(wl.B, wl.T, wl.H, wl.dv, device=dev, dtype=torch.bfloat16)
    ST = torch.empty(wl.B, wl.H, wl.dk, wl.dv, device=dev, dtype=torch.float32)
    stream = torch.cuda.current_stream(dev)

    def step(i):
        d = sets[i % 2]
        gdn2.chunk_fwd(*[d[n] for n in TOK], S0=d["S0"], o=o, S_T=ST, stream=stream)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize(dev)

    clocks = ClockSampler(local).start()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    launches0 = gdn2.launch_count()
    barrier(ws)
    torch.cuda.synchronize(dev)
    t_wall0 = time.perf_counter()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for i in range(args.steps):
        ev[i][0].record(stream)
        step(i)
        ev[i][1].record(stream)
    end.record(stream)
    torch.cuda.synchronize(dev)
    barrier(ws)
    t_wall1 = time.perf_counter()
    launches = gdn2.launch_count() - launches0
    clocks.stop()
    elapsed_ms = max_over_ranks(start.elapsed_time(end), ws, dev)
    launch_ms = [a.elapsed_time(b) for a, b in ev]
    avg_launch_ms = statistics.mean(launch_ms)

    value = ws * tokens * args.steps / (elapsed_ms / 1e3)
    pk, pk_kind = peaks()
    alg_bytes = chunk_bytes(wl, tokens, wl.B)
    alg_flops = chunk_flops(wl, tokens)
    achieved_gbs = alg_bytes / (avg_launch_ms / 1e3) / 1e9
    tflops = alg_flops / (avg_launch_ms / 1e3) / 1e12
    kernel_name = "chunk_fwd"
    tr = traffic_record(kernel_name)
    roofline = {"bound": "hbm", "achieved": achieved_gbs, "peak": pk["hbm_gbs"], "unit": "GB/s",
                "frac": achieved_gbs / pk["hbm_gbs"], "traffic": tr["dram_bytes_per_launch"] if tr else None,
                "kernel": tr["kernel"] if tr else kernel_name, "peak_source": pk_kind,
                "algorithmic_bytes_per_launch": alg_bytes, "avg_launch_ms": avg_launch_ms}
    tensor = {"achieved": tflops, "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
              "frac": tflops / pk["bf16_tflops"], "algorithmic_flops_per_launch": alg_flops,
              "note": "algorithmic flops (not padded MMA work) over the bf16 dense burst peak"}

    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": elapsed_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": "layer_1p3b", "B": wl.B, "T": wl.T, "H": wl.H, "d_k": wl.dk,
                   "d_v": wl.dv, "chunk": wl.chunk, "state": "fp32", "parallelism": f"replicas x{ws}",
                   "l2": "inputs larger than L2: two 235 MB input sets alternated between steps"},
        "roofline": roofline, "tensor": tensor, "gpu_launches": launches,
        "clocks": clocks.summary(t_wall0, t_wall1),
    }

    # ------------------------------------------------------------ decode: 1024 steps in one graph
    if not args.no_decode:
        line["decode_step"] = bench_decode(gdn2, dev, stream, pk, pk_kind)
        line["gpu_launches_decode"] = line["decode_step"].pop("launches")
    # ------------------------------------------------------------ block prologue / epilogue around the mixer
    if not args.no_block:
        line.update(bench_block(gdn2, dev, stream, pk, pk_kind))
    if not args.no_bwd:
        line["chunk_bwd"] = bench_bwd(gdn2, dev, stream, pk, pk_kind)
    if not args.no_workloads:
        line["long_context"] = bench_long_context(gdn2, dev, stream, pk, pk_kind)
        line["varlen"] = bench_varlen(gdn2, dev, stream, pk, pk_kind)
    # ------------------------------------------------------------ the headline step, sustained for ~0.5 s
    line["sustained"] = bench_sustained(step, dev, stream, local, len(ev))

    # ------------------------------------------------------------ end to end through host buffers
    line["e2e"] = bench_e2e(gdn2, wl, sets[0], dev, stream, ws, tokens)

    # ------------------------------------------------------------ CPU oracle baseline
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        tok, dt, cores = time_oracle(wl, 0, wl.B, wl.H)
        line["cpu_baseline"] = {"value": tok / dt, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                                "sample": f"the whole layer_1p3b batch ({wl.B} x {wl.T} tokens x {wl.H} heads), "
                                          f"one pass, {dt:.1f} s"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if ws > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


def profile_case(which):
    """Two launches (warm-up + measured) of one kernel on its full workload; nothing else is timed."""
    import gated_delta_rule_131_b200 as gdn2
    dev = torch.device("cuda", 0)
    if which == "chunk":
        wl = W.WORKLOADS["layer_1p3b"]
        d = W.chunk_inputs(wl, device=dev, seed=0)
        for _ in range(2):
            gdn2.chunk_fwd(*[d[n] for n in TOK], S0=d["S0"])
    elif which in ("bwd", "bwd_small"):
        wl = W.WORKLOADS["layer_1p3b"]
        if which == "bwd_small":  # 4 x 512 tokens: the layer's 512 CTAs and occupancy, about 0.4 GB on the device
            wl = W.Workload("bwd_small", B=4, T=512, H=16, dk=128, dv=128)
        d = W.chunk_inputs(wl, device=dev, seed=0)
        gen = torch.Generator(device="cpu").manual_seed(1000)
        dO = torch.randn(d["q"].shape[:-1] + (wl.dv,), generator=gen).to(dev, torch.bfloat16)
        dST = torch.randn(d["S0"].shape, generator=gen).to(dev) * 0.1
        for _ in range(2):
            gdn2.chunk_bwd(*[d[n] for n in TOK], dO, S0=d["S0"], dS_T=dST)
    elif which == "block":
        wl = W.WORKLOADS["layer_1p3b"]
        d = W.block_inputs(wl, device=dev, seed=0, conv_len=4)
        for _ in range(2):
            gdn2.block_prologue(*[d[n] for n in ("xq", "xk", "xv", "xa", "xb", "xw", "conv_q", "conv_k", "conv_v")])
            gdn2.block_epilogue(d["xv"], d["z"], d["norm_weight"])
    else:
        wl = W.WORKLOADS["decode"]
        S = W.decode_state(wl, device=dev, seed=0)
        for s in range(2):
            t = W.decode_token_inputs(wl, s, device=dev, seed=0)
            gdn2.decode_step(*[t[n] for n in TOK], S=S)
    torch.cuda.synchronize(dev)
    print(f"profile case {which}: ok", flush=True)
    return 0


def bench_decode(gdn2, dev, stream, pk, pk_kind):
    wl = W.WORKLOADS["decode"]
    S = W.decode_state(wl, device=dev, seed=0)
    steps = wl.decode_steps
    toks = [W.decode_token_inputs(wl, s, device=dev, seed=0) for s in range(steps)]
    outs = torch.empty(steps, wl.B, wl.H, wl.dv, device=dev, dtype=torch.bfloat16)
    # eager warm-up, then capture the 1024 launches into one graph
    for s in range(3):
        gdn2.decode_step(*[toks[s][n] for n in TOK], S=S, o=outs[s], stream=stream)
    torch.cuda.synchronize(dev)
    g = torch.cuda.CUDAGraph()
    cap = torch.cuda.Stream(dev)
    c0 = gdn2.launch_count()
    with torch.cuda.graph(g, stream=cap):
        for s in range(steps):
            gdn2.decode_step(*[toks[s][n] for n in TOK], S=S, o=outs[s], stream=cap)
    per_replay = gdn2.launch_count() - c0
    g.replay()
    torch.cuda.synchronize(dev)
    reps = 3
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    rs = torch.cuda.current_stream(dev)
    a.record(rs)
    for _ in range(reps):
        g.replay()
    b.record(rs)
    torch.cuda.synchronize(dev)
    ms = a.elapsed_time(b)
    per_step_ms = ms / (reps * steps)
    bytes_step = decode_bytes(wl)
    gbs = bytes_step / (per_step_ms / 1e3) / 1e9
    tr = traffic_record("decode_step")
    del g
    return {"value": gbs, "unit": "GB/s", "workload": "decode", "B": wl.B, "H": wl.H, "d_k": wl.dk,
            "d_v": wl.dv, "steps_per_graph": steps, "graph_replays": reps, "us_per_step": per_step_ms * 1e3,
            "tokens_per_s": wl.B / (per_step_ms / 1e3),
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": pk["hbm_gbs"], "unit": "GB/s",
                         "frac": gbs / pk["hbm_gbs"], "traffic": tr["dram_bytes_per_launch"] if tr else None,
                         "peak_source": pk_kind, "algorithmic_bytes_per_launch": bytes_step},
            "launches": per_replay * reps}


def block_bytes(wl, tokens, conv_len=4):
    """Algorithmic bytes of the block prologue and epilogue (every element read and written once)."""
    e = 2 if wl.dtype == "bf16" else 4
    th = tokens * wl.H
    # six pre-activations in, six outputs out; plus the fp32 taps of the three paths, [H*d, K] each
    pro = th * 2 * (4 * wl.dk + 2 * wl.dv) * e + conv_len * wl.H * (2 * wl.dk + wl.dv) * 4
    epi = th * 3 * wl.dv * e + wl.dv * 4
    return pro, epi


def bench_block(gdn2, dev, stream, pk, pk_kind, reps=20):
    """The block prologue and epilogue around the mixer on the 1.3B-layer shape (4 taps)."""
    wl = W.WORKLOADS["layer_1p3b"]
    tokens = wl.B * wl.T
    d = W.block_inputs(wl, device=dev, seed=0, conv_len=4)
    pre = [d[n] for n in ("xq", "xk", "xv", "xa", "xb", "xw", "conv_q", "conv_k", "conv_v")]
    o = d["xv"]
    y = torch.empty_like(o)
    pro_b, epi_b = block_bytes(wl, tokens)
    out = {}
    for name, fn, nbytes in (("block_prologue", lambda: gdn2.block_prologue(*pre, stream=stream), pro_b),
                             ("block_epilogue", lambda: gdn2.block_epilogue(o, d["z"], d["norm_weight"], y=y,
                                                                            stream=stream), epi_b)):
        for _ in range(3):
            fn()
        torch.cuda.synchronize(dev)
        c0 = gdn2.launch_count()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
        for a, b in ev:
            a.record(stream)
            fn()
            b.record(stream)
        torch.cuda.synchronize(dev)
        ms = statistics.median(a.elapsed_time(b) for a, b in ev)
        gbs = nbytes / (ms / 1e3) / 1e9
        tr = traffic_record(name)
        out[name] = {"value": gbs, "unit": "GB/s", "workload": "layer_1p3b", "conv_len": 4,
                     "us_per_call": ms * 1e3, "launches": gdn2.launch_count() - c0,
                     "roofline": {"bound": "hbm", "achieved": gbs, "peak": pk["hbm_gbs"], "unit": "GB/s",
                                  "frac": gbs / pk["hbm_gbs"],
                                  "traffic": tr["dram_bytes_per_launch"] if tr else None, "peak_source": pk_kind,
                                  "algorithmic_bytes_per_launch": nbytes}}
    return out


def bwd_bytes(wl, tokens, nseq):
    """Algorithmic bytes of one backward call: the six forward inputs and dL/do read, the six
    gradients written (bf16), and S0, dL/dS_T read and dS0 written (fp32)."""
    e = 2 if wl.dtype == "bf16" else 4
    th = tokens * wl.H
    return th * (2 * (4 * wl.dk + 2 * wl.dv) + wl.dv) * e + 3 * nseq * wl.H * wl.dk * wl.dv * 4


def bench_bwd(gdn2, dev, stream, pk, pk_kind, reps=5):
    """gdn2_chunk_bwd on the 1.3B-layer workload (seeded dL/do and dL/dS_T)."""
    wl = W.WORKLOADS["layer_1p3b"]
    tokens = wl.B * wl.T
    d = W.chunk_inputs(wl, device=dev, seed=0)
    gen = torch.Generator(device="cpu").manual_seed(1000)
    dO = torch.randn(d["q"].shape[:-1] + (wl.dv,), generator=gen).to(dev, torch.bfloat16)
    dST = torch.randn(d["S0"].shape, generator=gen).to(dev) * 0.1
    fn = lambda: gdn2.chunk_bwd(*[d[n] for n in TOK], dO, S0=d["S0"], dS_T=dST, stream=stream)
    for _ in range(3):
        fn()
    torch.cuda.synchronize(dev)
    c0 = gdn2.launch_count()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
    for a, b in ev:
        a.record(stream)
        fn()
        b.record(stream)
    torch.cuda.synchronize(dev)
    ms = statistics.median(a.elapsed_time(b) for a, b in ev)
    nbytes = bwd_bytes(wl, tokens, wl.B)
    gbs = nbytes / (ms / 1e3) / 1e9
    tr = traffic_record("chunk_bwd")
    return {"value": tokens / (ms / 1e3), "unit": "tokens/s", "workload": "layer_1p3b", "ms_per_call": ms,
            "launches": gdn2.launch_count() - c0,
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": pk["hbm_gbs"], "unit": "GB/s",
                         "frac": gbs / pk["hbm_gbs"], "traffic": tr["dram_bytes_per_launch"] if tr else None,
                         "peak_source": pk_kind, "algorithmic_bytes_per_launch": nbytes,
                         "note": "issue- and latency-bound SIMT kernel (about 860 instructions per warp and token)"}}


def time_calls(fn, dev, stream, reps):
    """Median CUDA-event time (ms) of ``reps`` calls of ``fn`` on ``stream``, after three warm-up calls."""
    for _ in range(3):
        fn()
    torch.cuda.synchronize(dev)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
    for a, b in ev:
        a.record(stream)
        fn()
        b.record(stream)
    torch.cuda.synchronize(dev)
    return statistics.median(a.elapsed_time(b) for a, b in ev)


def chunk_entry(gdn2, wl, d, dev, stream, pk, pk_kind, reps):
    """tokens/s and HBM roofline of one chunk_fwd call on the inputs ``d`` of workload ``wl``."""
    lens = d["lengths"]
    tokens = sum(lens)
    fn = lambda: gdn2.chunk_fwd(*[d[n] for n in TOK], S0=d["S0"], cu_seqlens=d["cu_seqlens"], stream=stream)
    c0 = gdn2.launch_count()
    ms = time_calls(fn, dev, stream, reps)
    launches = (gdn2.launch_count() - c0) // (reps + 3)
    nbytes = chunk_bytes(wl, tokens, len(lens))
    gbs = nbytes / (ms / 1e3) / 1e9
    return {"value": tokens / (ms / 1e3), "unit": "tokens/s", "workload": wl.name, "tokens": tokens,
            "B": len(lens), "H": wl.H, "d_k": wl.dk, "d_v": wl.dv, "us_per_call": ms * 1e3,
            "launches_per_call": launches,
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": pk["hbm_gbs"], "unit": "GB/s",
                         "frac": gbs / pk["hbm_gbs"], "traffic": None, "peak_source": pk_kind,
                         "algorithmic_bytes_per_launch": nbytes}}


def bench_long_context(gdn2, dev, stream, pk, pk_kind):
    """The long-context workload (B=1, H=16, T=65536, retention-biased decay), and the pages' claim of
    near-flat throughput as sequences grow: tokens/s at a fixed 131,072 tokens x 16 heads per call,
    split into sequences of 2048 ... 65536 tokens.  ``flat_scaling`` = tokens/s at T = 65536 over
    tokens/s at T = 2048 (1.0 is perfectly flat)."""
    wl = W.WORKLOADS["long_context"]
    d = W.chunk_inputs(wl, device=dev, seed=0)
    out = chunk_entry(gdn2, wl, d, dev, stream, pk, pk_kind, reps=10)
    del d
    sweep = []
    total = 131072
    for T in (2048, 8192, 32768, 65536):
        wls = W.scaled(W.WORKLOADS["layer_1p3b"], name=f"seq_{T}", B=total // T, T=T)
        ds = W.chunk_inputs(wls, device=dev, seed=0)
        e = chunk_entry(gdn2, wls, ds, dev, stream, pk, pk_kind, reps=10)
        sweep.append({"B": wls.B, "T": T, "tokens_per_s": e["value"], "us_per_call": e["us_per_call"],
                      "roofline_frac": e["roofline"]["frac"]})
        del ds
    out["seq_sweep"] = sweep
    out["flat_scaling"] = sweep[-1]["tokens_per_s"] / sweep[0]["tokens_per_s"]
    out["flat_scaling_note"] = ("tokens/s at 2 x 65536 tokens over 64 x 2048 tokens, 16 heads, d = 128, bf16; "
                                "same 131,072 tokens per call")
    return out


def bench_varlen(gdn2, dev, stream, pk, pk_kind):
    """The packed workload (32 sequences, lengths uniform in [1, 8192], H=32, d_v=256) with its three
    gate variants: per-channel b and w, the KDA case and the Gated DeltaNet case."""
    out = {}
    for name in ("varlen", "varlen_kda", "varlen_gdn"):
        wl = W.WORKLOADS[name]
        d = W.chunk_inputs(wl, device=dev, seed=0)
        out[wl.variant] = chunk_entry(gdn2, wl, d, dev, stream, pk, pk_kind, reps=5)
        del d
    return out


def bench_sustained(step, dev, stream, device_index, first, seconds=0.5):
    """The headline step repeated back to back for about ``seconds`` (after the timed steps), with its
    own clock samples: the clocks the step runs at under sustained load."""
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    step(first)
    b.record(stream)
    torch.cuda.synchronize(dev)
    n = max(10, int(seconds / max(a.elapsed_time(b) / 1e3, 1e-6)))
    clocks = ClockSampler(device_index).start()
    t0 = time.perf_counter()
    a.record(stream)
    for i in range(n):
        step(first + i)
    b.record(stream)
    torch.cuda.synchronize(dev)
    t1 = time.perf_counter()
    clocks.stop()
    ms = a.elapsed_time(b)
    return {"steps": n, "ms_per_step": ms / n, "seconds": ms / 1e3, "clocks": clocks.summary(t0, t1)}


def bench_e2e(gdn2, wl, d, dev, stream, ws, tokens, steps=6):
    """chunk_fwd through the public call with pinned host buffers.  Every step copies its inputs and
    S0 host -> device, calls chunk_fwd and reads o and S_T back to the host, all inside the timed
    region.  Steps are pipelined over two device buffer sets and three streams (copy in, the call,
    copy out): one step's input copy overlaps the previous step's call and readback, as a serving
    loop would run them.  A buffer set is refilled only after the call that read it has finished,
    and its outputs are overwritten only after their readback."""
    host = {n: d[n].cpu().pin_memory() for n in TOK}
    host["S0"] = d["S0"].cpu().pin_memory()
    nbuf = 2
    dev_in = [{n: torch.empty_like(d[n]) for n in host} for _ in range(nbuf)]
    dev_out = [(torch.empty(wl.B, wl.T, wl.H, wl.dv, dtype=torch.bfloat16, device=dev),
                torch.empty(wl.B, wl.H, wl.dk, wl.dv, dtype=torch.float32, device=dev)) for _ in range(nbuf)]
    host_out = [(torch.empty(wl.B, wl.T, wl.H, wl.dv, dtype=torch.bfloat16).pin_memory(),
                 torch.empty(wl.B, wl.H, wl.dk, wl.dv, dtype=torch.float32).pin_memory()) for _ in range(nbuf)]
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = sum(t.numel() * t.element_size() for t in host_out[0])
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)

    def run(n):
        ev_call = [torch.cuda.Event() for _ in range(n)]
        ev_back = [torch.cuda.Event() for _ in range(n)]
        for k in range(n):
            b = k % nbuf
            if k >= nbuf:
                s_in.wait_event(ev_call[k - nbuf])  # the call that read this buffer set is done
            with torch.cuda.stream(s_in):
                for name, t in host.items():
                    dev_in[b][name].copy_(t, non_blocking=True)
            ev_copied = torch.cuda.Event()
            ev_copied.record(s_in)
            stream.wait_event(ev_copied)
            if k >= nbuf:
                stream.wait_event(ev_back[k - nbuf])  # this buffer set's outputs were read back
            gdn2.chunk_fwd(*[dev_in[b][name] for name in TOK], S0=dev_in[b]["S0"], o=dev_out[b][0],
                           S_T=dev_out[b][1], stream=stream)
            ev_call[k].record(stream)
            s_out.wait_event(ev_call[k])
            with torch.cuda.stream(s_out):
                host_out[b][0].copy_(dev_out[b][0], non_blocking=True)
                host_out[b][1].copy_(dev_out[b][1], non_blocking=True)
            ev_back[k].record(s_out)
        return ev_back[-1]

    run(2)
    torch.cuda.synchronize(dev)
    barrier(ws)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(s_in)
    last = run(steps)
    s_out.wait_event(last)
    b.record(s_out)
    torch.cuda.synchronize(dev)
    barrier(ws)
    ms = max_over_ranks(a.elapsed_time(b), ws, dev)
    return {"value": ws * tokens * steps / (ms / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "steps": steps,
            "pipelined": "two device buffer sets; copy-in, call and copy-out streams overlap across steps"}


if __name__ == "__main__":
    sys.exit(main())
