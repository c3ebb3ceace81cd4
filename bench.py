"""Benchmark of the ODA decode hot path on B200 (one JSON line on rank 0).

Workload (default): Qwen3-8B-shaped attention, 36 layers, 32 query / 8 KV heads, head_dim 128,
context 131072, batch 4, flags Bernoulli(0.125) per sequence-step, recall head (D = 4096)
still run.  A step = local pass (36 layers), recall head, conditional full retry of the
flagged sequences, commit, for the whole batch.  Inputs: seeded synthetic data (bf16 K/V/q
~ N(0,1)), the 77 GB cache resident in HBM (larger than L2, no flush needed).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

--gpus N > 1 runs under torchrun as N independent replicas (one batch per GPU, no
collective on the data path); timing is the max over ranks.  --impl reference times the
CPU oracle (the plain fp64 restatement in oracle/) on the host cores over a bounded sample
of the same workload.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "ODA decode-attn steps/s + % of HBM peak, 128K ctx, 12.5% recall, 1 B200"

# DRAM bytes (read + write) of one full-set attention launch from an ncu capture of the
# 32K-context, 2-layer profiling workload (4 flagged sequences x 32768 cached tokens); the bench
# scales it to its own launches by cached tokens processed.  Valid only for the kernel source it
# was taken from (first 16 hex digits of the file's SHA-256).
NCU_FULL_KERNEL_TRAFFIC = {"attention_cu_sha256": "00d69c2bf934804c", "bytes": 540707072,
                           "cached_tokens": 4 * 32768}
UNIT = "steps/s"
FALLBACK_HBM_GBS = 6650.0
NOMINAL_HBM_GBS = 8000.0   # B200 HBM3e specification; `frac` uses the measured copy peak


def traffic_per_token():
    """ncu DRAM bytes per cached token of one full-set launch, or None if the kernel changed."""
    import hashlib
    path = os.path.join(ROOT, "conditional_sparse_attention_b200", "csrc", "attention.cu")
    try:
        sha = hashlib.sha256(open(path, "rb").read()).hexdigest()[:16]
    except OSError:
        return None
    t = NCU_FULL_KERNEL_TRAFFIC
    return t["bytes"] / t["cached_tokens"] if sha == t["attention_cu_sha256"] else None


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


# ---------------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi sampling during the timed region (SM clock, max, throttle reasons)."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.th = threading.Thread(target=self._read, daemon=True)
            self.th.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for nm, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------------------ accounting
KV_BYTES_PER_TOKEN_HEAD = {"bf16": 128 * 2 * 2,       # K and V rows, bf16
                           "fp8": 128 * 2 + 2 * 4}     # K and V e4m3 codes + two fp32 scales


def hybrid_state_bytes(wl) -> int:
    """Recurrent + conv state of one sequence over all linear-recurrent layers (fp32)."""
    from workload import configs
    n = len(wl.gdn_layers)
    return n * (configs.GDN_HEADS * configs.GDN_DIM * configs.GDN_DIM +
                configs.CONV_TAPS * configs.CONV_WIDTH) * 4


def step_bytes(wl, pos_list, flags, kv="bf16"):
    """Algorithmic bytes of one step: local KV + flagged full KV + head weights; hybrid stacks add
    the recurrent state each pass reads and writes (the local pass for every sequence, the retry
    for flagged ones; with ping-pong state buffers nothing is snapshotted or restored)."""
    from workload import inputs
    per_tok = wl.Hkv * KV_BYTES_PER_TOKEN_HEAD[kv]
    st = hybrid_state_bytes(wl) if wl.hybrid else 0
    b = 0
    for bi, t in enumerate(pos_list):
        b += min(t, wl.sinks + wl.window) * per_tok * wl.L + 2 * st
        if flags[bi]:
            b += t * per_tok * wl.L + 2 * st
    return b + inputs.head_param_count(wl.D) * 4


def head_launches(wl) -> int:
    """The recall head is one cooperative launch for up to 8 sequences (D a multiple of 1024,
    at least 128 SMs), else six phase launches."""
    return 1 if wl.B <= 8 and wl.D % 1024 == 0 else 6


def kernel_launches(wl, any_flag: bool) -> int:
    # local layers, glue, head, set-cond, commit (hybrid stacks: no snapshot or restore copies)
    n = wl.L + (wl.n_layers - wl.L) + 1 + head_launches(wl) + 1 + 1
    if any_flag:
        n += wl.n_layers + 1
    return n


# ------------------------------------------------------------------- multi-rank
def replica_workload(wl, rank: int, world: int):
    """Replicas only: every rank decodes its own batch (a distinct seed), no data exchange."""
    return wl if world <= 1 else wl.replace(seed=wl.seed + 1000 * rank, name=f"{wl.name}_r{rank}")


def max_over_ranks(ms: float, world: int, device=None) -> float:
    """Device-timed milliseconds, maximised over ranks (all ranks call this in the same order)."""
    if world <= 1:
        return float(ms)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(ms)], dtype=torch.float64,
                     device=device if dist.get_backend() == "nccl" else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# --------------------------------------------------------------------- oracle sample
def timed_steps(W: int, K: int) -> list:
    """Step indices whose inputs the K timed steps of the GPU arm use (after the first step and
    W warm-up steps, cycling through W + K stored step inputs)."""
    n_store = W + K
    return [(1 + W + i) % n_store for i in range(K)]


class OracleStepSample:
    """The CPU oracle's cost of one decode step of the workload, composed from timed parts.

    Each part is one call of the oracle exactly as its decode step (oracle.step.run_pass)
    makes it, on sequence 0 / attention layer 0 of the workload's step-0 inputs:
      * local attention of one (sequence, layer) over S^L, all KV heads;
      * full attention of one (sequence, layer) over S^F, all KV heads;
      * one recall-head score (the oracle scores sequence by sequence).
    A step costs L*B local calls, one full call per flagged (sequence, layer) and B head
    scores; the flags are the workload's seeded schedule for the GPU arm's timed steps (the
    head's own gate where the workload routes on the head, counted at the workload's expected
    rate).  Full calls are scaled from sequence 0's context to each flagged sequence's by the
    cached tokens, the only size that changes their work; so are the local calls, because the
    oracle's decode step hands every call the whole cache of its sequence.  Inputs are generated
    once, outside the timed region."""

    def __init__(self, wl, W: int, K: int):
        import numpy as np
        from workload import inputs
        self.wl = wl
        self.t = wl.ctx[0] + 1
        q, kn, vn = inputs.step_qkv(wl, 0, wl.attn_layers[0], 0)
        self.q, self.kn, self.vn = q[0], kn[0], vn[0]
        self.kc = inputs.cache_tokens(wl, "k", 0, 0, self.t - 1)
        self.vc = inputs.cache_tokens(wl, "v", 0, 0, self.t - 1)
        self.P = inputs.head_weights(wl)
        self.e = inputs.emb(wl, 0).astype(np.float64)[0]
        self.hp = inputs.h_prev0(wl).astype(np.float64)[0]
        # flagged (sequence, step) pairs of the timed steps -> full calls per step, in units of
        # sequence 0's context
        if wl.routing == "bernoulli":
            steps = timed_steps(W, K)
            fl = np.array([inputs.schedule(wl, s) for s in steps])
        else:
            fl = np.full((1, wl.B), 0.4)
        rel = np.array([(c + 1) / self.t for c in wl.ctx])
        self.full_units = float((fl * rel[None, :]).sum(axis=1).mean())
        self.local_units = float(rel.sum())
        self.flagged_per_step = float(fl.sum(axis=1).mean())

    def run(self) -> dict:
        """Seconds of each part (one timed call each)."""
        import numpy as np
        from oracle.attention import attend_bits
        from oracle.head import recall_head
        from oracle.sets import full_set, local_set
        wl, t = self.wl, self.t
        t0 = time.perf_counter()
        o_l = attend_bits(self.q, self.kc, self.vc, self.kn, self.vn, local_set(t, wl.sinks, wl.window))
        t1 = time.perf_counter()
        o_f = attend_bits(self.q, self.kc, self.vc, self.kn, self.vn, full_set(t))
        t2 = time.perf_counter()
        sc = recall_head(self.P, self.hp, self.e, self.e)
        t3 = time.perf_counter()
        assert np.isfinite(o_l).all() and np.isfinite(o_f).all() and np.isfinite(sc)
        return {"local_s": t1 - t0, "full_s": t2 - t1, "head_s": t3 - t2}

    def step_seconds(self, part: dict) -> float:
        wl = self.wl
        return (wl.L * self.local_units * part["local_s"] + wl.L * self.full_units * part["full_s"] +
                wl.B * part["head_s"])

    def describe(self, part: dict) -> str:
        wl = self.wl
        return (f"fp64 oracle, one call of each part as its decode step makes it (sequence 0, "
                f"attention layer 0, all {wl.Hkv} KV heads, t={self.t}): local attention "
                f"{part['local_s']:.3f} s, full attention {part['full_s']:.3f} s, recall-head score "
                f"{part['head_s']:.3f} s; step = {wl.L}x{wl.B} local + {wl.L}x"
                f"{self.flagged_per_step:.3f} full (the schedule's flagged sequences per timed "
                f"step) + {wl.B} head scores = {self.step_seconds(part):.1f} s")


def cpu_cores() -> int:
    return len(os.sched_getaffinity(0))


def workload_config(wl, world: int, eager: bool, kv: str = "bf16") -> dict:
    """The `config` object of both arms' JSON lines (the workload and how the GPU arm runs it)."""
    n_pages = sum((c + 1 + 15) // 16 for c in wl.ctx)
    cache_gb = n_pages * 16 * wl.Hkv * KV_BYTES_PER_TOKEN_HEAD[kv] * wl.L / 1e9
    return {"workload": wl.name, "B": wl.B, "layers": wl.L, "Hq": wl.Hq, "Hkv": wl.Hkv,
            "head_dim": 128, "ctx": wl.ctx[0] if len(set(wl.ctx)) == 1 else
            f"{min(wl.ctx)}..{max(wl.ctx)}",
            "recall_rate": (wl.rates[0] if len(set(wl.rates)) == 1 else
                            f"{min(wl.rates):.3f}..{max(wl.rates):.3f}") if wl.rates else None,
            "page_tokens": 16, "kv_cache": kv, "parallelism": f"replicas{world}",
            "l2": f"inputs larger than L2 ({cache_gb:.0f} GB resident KV cache), no flush",
            "launch": "eager" if eager else "cuda-graph with conditional IF node"}


def run_reference(args, wl, rank, world):
    if rank != 0:
        return
    smp = OracleStepSample(wl, args.warmup, args.steps)
    vals, parts = [], []
    for i in range(args.warmup + args.steps):
        part = smp.run()
        if i >= args.warmup:
            parts.append(part)
            vals.append(1.0 / smp.step_seconds(part))
    value = statistics.median(vals)
    mid = parts[vals.index(sorted(vals)[len(vals) // 2])]
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1000.0 / value, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(wl, world, args.eager, args.kv),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cpu_cores(), "kind": "oracle",
                             "sample": smp.describe(mid) + f"; median of {args.steps} samples"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------------ GPU arm
def time_layer_kernels(dec, mode: int, flag, reps: int = 3) -> float:
    """Average device milliseconds of one attention launch: a graph holding one launch per
    layer (local: mode 0, full: mode 1 with the given flags) replayed ``reps`` times."""
    import torch
    from conditional_sparse_attention_b200 import oda
    s = dec.stream
    wl = dec.wl
    torch.cuda.synchronize(dec.device)
    oda.oda_graph_begin(s)
    for a in range(wl.L):
        if mode == 0:
            dec._attend_local(dec.ctx, dec.layers[a], dec.page_table, dec.pos, dec.sv["q"][0, a],
                              dec.sv["k"][0, a], dec.sv["v"][0, a], dec.o[0, a], s)
        else:
            dec._attend_full(dec.ctx, dec.layers[a], dec.page_table, dec.pos, flag,
                             dec.sv["q"][1, a], dec.sv["k"][1, a], dec.sv["v"][1, a],
                             dec.o[1, a], s)
    g = oda.oda_graph_end(s)
    g.launch(s)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s)
    for _ in range(reps):
        g.launch(s)
    e1.record(s)
    e1.synchronize()
    g.close()
    return e0.elapsed_time(e1) / (reps * wl.L)


def time_head(dec, reps: int = 5) -> float:
    """Average device milliseconds of one recall-head score (its launch or launches, as a graph)."""
    import torch
    from conditional_sparse_attention_b200 import oda
    s = dec.stream
    torch.cuda.synchronize(dec.device)
    oda.oda_graph_begin(s)
    oda.oda_recall_score(dec.ctx, dec.head_w, dec.h_prev, dec.sv["emb"], dec.h[0],
                         dec.sv["sched"] if dec.routing_scheduled else None, dec.score, dec.flag,
                         dec.any_flag, s)
    g = oda.oda_graph_end(s)
    g.launch(s)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s)
    for _ in range(reps):
        g.launch(s)
    e1.record(s)
    e1.synchronize()
    g.close()
    return e0.elapsed_time(e1) / reps


def run_kernel_only(args, wl, local_rank):
    """Profiling mode: set up the workload, stage step 0, launch one kernel ``--kernel-reps``
    times (full: the full-set attention with every sequence flagged; local: the local-set
    attention; head: the recall head on the local hidden state) and exit."""
    import torch
    from conditional_sparse_attention_b200 import oda
    from conditional_sparse_attention_b200.engine import OdaDecoder
    dev = torch.device("cuda", local_rank)
    if args.kernel_only == "bbstep":
        # whole-model steps of the synthetic backbone, issued kernel by kernel (a profiler lists
        # every launch; graphs with conditional nodes hide theirs)
        from workload import configs
        if not wl.backbone:   # default: the whole 28-layer model at 4K context
            wl = configs.bb_qwen3_1p7b(ctx=4096)
        dec = OdaDecoder(wl, device=dev, capacity_steps=args.kernel_reps + 2)
        for r in range(args.kernel_reps):
            dec.step(dec.make_step_buffer(r))
        dec.synchronize()
        print(json.dumps({"kernel_only": "bbstep", "workload": wl.name, "steps": args.kernel_reps,
                          "device_error": dec.device_error()}), flush=True)
        dec.close()
        return
    dec = OdaDecoder(wl, device=dev, capacity_steps=4, kv_format=args.kv)
    dec.stage(dec.make_step_buffer(0))
    dec.synchronize()
    ones = torch.ones(wl.B, dtype=torch.int32, device=dev)
    if args.kernel_only == "grad":
        # one training step of the recall head on the step's inputs, with synthetic next-token
        # probabilities of the two passes (every position valid)
        grads = {k: torch.empty_like(v) for k, v in dec.head_params.items()}
        gw = oda.head_grads(grads)
        p_full = torch.linspace(0.2, 0.8, wl.B, device=dev)
        p_local = torch.linspace(0.7, 0.1, wl.B, device=dev)
        loss = torch.zeros(1, device=dev)
        q = torch.zeros(wl.B, device=dev)
        y = torch.zeros(wl.B, device=dev)
        ws = torch.empty(oda.oda_recall_grad_workspace_bytes(wl.B, wl.D), dtype=torch.uint8,
                         device=dev)

        def grad_step(d):
            oda.oda_recall_grad(d.head_w, gw, wl.B, wl.D, d.h_prev, d.sv["emb"], d.h[0], p_full,
                                p_local, ones, 0.01, loss, q, y, ws, d.stream)
    for r in range(args.kernel_reps):
        a = r % wl.L
        if args.kernel_only == "full":
            dec._attend_full(dec.ctx, dec.layers[a], dec.page_table, dec.pos, ones,
                             dec.sv["q"][1, a], dec.sv["k"][1, a], dec.sv["v"][1, a],
                             dec.o[1, a], dec.stream)
        elif args.kernel_only == "local":
            dec._attend_local(dec.ctx, dec.layers[a], dec.page_table, dec.pos, dec.sv["q"][0, a],
                              dec.sv["k"][0, a], dec.sv["v"][0, a], dec.o[0, a], dec.stream)
        elif args.kernel_only == "head":
            oda.oda_recall_score(dec.ctx, dec.head_w, dec.h_prev, dec.sv["emb"], dec.h[0],
                                 dec.sv["sched"] if dec.routing_scheduled else None, dec.score,
                                 dec.flag, dec.any_flag, dec.stream)
        else:
            grad_step(dec)
    dec.synchronize()
    err = dec.device_error()
    print(json.dumps({"kernel_only": args.kernel_only, "workload": wl.name, "kv": args.kv,
                      "launches": args.kernel_reps, "device_error": err}), flush=True)
    dec.close()

SWEEP_CTX = (4096, 16384, 32768, 65536, 131072)
SWEEP_RHO = (0.0, 0.125, 0.25, 0.5, 1.0)


def run_sweep(args, wl0, local_rank):
    """Recall-rate x context sweep of the decode step on the workload's shapes (batch, heads,
    layers).  Per context: the whole step (local pass, head, conditional full retry, commit; CUDA
    graph) at each recall rate, with Bernoulli flags drawn per (sequence, step), and, as the
    always-full reference, the full-set attention of every sequence and layer (kernels alone: no
    local pass, no head).  One JSON line per point, then one summary line."""
    import torch
    from conditional_sparse_attention_b200.engine import OdaDecoder, fill_step_inputs
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    W, K = args.warmup, args.steps
    per = W + K
    points = []
    for ctx in SWEEP_CTX:
        wl = wl0.replace(name=f"{wl0.name}_sweep_ctx{ctx}", ctx=(ctx,) * wl0.B, routing="bernoulli",
                         rates=(0.0,) * wl0.B, steps=per * len(SWEEP_RHO))
        dec = OdaDecoder(wl, device=dev, capacity_steps=per * len(SWEEP_RHO) + 4)
        dec.capture()
        step = 0
        ones = torch.ones(wl.B, dtype=torch.int32, device=dev)
        full_ms = None
        for rho in SWEEP_RHO:
            wr = wl.replace(rates=(rho,) * wl.B)   # same inputs, the schedule drawn at rate rho
            bufs = []
            for i in range(per):
                buf = torch.zeros(dec.layout.nbytes, dtype=torch.uint8, device=dev)
                fill_step_inputs(wr, step + i, dec.layout.views(buf))
                bufs.append(buf)
            for i in range(W):
                dec.step(bufs[i])
            flags = torch.zeros((K, wl.B), dtype=torch.int32, device=dev)
            dec.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            with torch.cuda.stream(dec.stream):
                e0.record(dec.stream)
                for i in range(K):
                    dec.step(bufs[W + i])
                    flags[i].copy_(dec.flag, non_blocking=True)
                e1.record(dec.stream)
            e1.synchronize()
            step += per
            step_ms = e0.elapsed_time(e1) / K
            if full_ms is None:
                full_ms = time_layer_kernels(dec, 1, ones, reps=2) * wl.L
            pt = {"sweep": True, "ctx": ctx, "rho": rho, "realized_rho": float(flags.float().mean()),
                  "oda_step_ms": step_ms, "always_full_attention_ms": full_ms,
                  "oda_over_full": step_ms / full_ms, "steps": K, "warmup": W,
                  "device_error": dec.device_error()}
            points.append(pt)
            print(json.dumps(pt), flush=True)
        dec.close()
        del dec, bufs
        torch.cuda.empty_cache()
    # per context: the largest swept rate at which the whole ODA step is still faster than the
    # always-full attention kernels alone
    cross = {}
    for ctx in SWEEP_CTX:
        ok = [p["rho"] for p in points if p["ctx"] == ctx and p["oda_step_ms"] < p["always_full_attention_ms"]]
        cross[str(ctx)] = max(ok) if ok else None
    print(json.dumps({"sweep_summary": True, "workload": wl0.name, "B": wl0.B, "layers": wl0.L,
                      "max_rho_where_oda_is_faster": cross}), flush=True)


BB_CTX = (4096, 16384, 32768, 65536, 131072)
BB_RHO = (0.0, 0.125, 0.5, 1.0)


def run_backbone(args, local_rank):
    """Whole-model decode steps of the synthetic Qwen3-1.7B-shaped model (batch 1): every layer's
    projections and attention, the recall head, the conditional full pass, the commit and the LM
    head - the scope of the method notes' throughput measurement (§3.3) - at each context and
    recall rate, beside the always-full model (full attention everywhere, no head).  Per point:
    the first step including graph capture and the warm median; one JSON line per point, then a
    summary with the speed-up over always-full at each context."""
    import torch
    from conditional_sparse_attention_b200 import oda
    from conditional_sparse_attention_b200.engine import OdaDecoder, fill_step_inputs
    from workload import configs
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    W, K = args.warmup, args.steps
    hbm, peak_src = peaks()
    ctxs = BB_CTX if args.backbone_ctx is None else tuple(int(c) for c in args.backbone_ctx.split(","))
    out = []
    for ctx in ctxs:
        wl0 = configs.bb_qwen3_1p7b(ctx=ctx)
        per = W + K
        total = per * (len(BB_RHO) + 2) + 8
        wl = wl0.replace(steps=total)
        dec = OdaDecoder(wl, device=dev, capacity_steps=total, bb_fused=not args.bb_separate)
        weight_bytes = dec.backbone_bytes()
        lm_bytes = wl.vocab * wl.D * 2
        head_bytes = __import__("workload.inputs", fromlist=["x"]).head_param_count(wl.D) * 4
        per_tok = wl.Hkv * KV_BYTES_PER_TOKEN_HEAD["bf16"]
        t0 = time.perf_counter()
        dec.capture()
        dec.step(dec.make_step_buffer(0))
        dec.synchronize()
        first_ms = (time.perf_counter() - t0) * 1e3
        step = 1
        res = {"ctx": ctx, "first_step_ms_incl_capture": first_ms}
        for rho in BB_RHO:
            wr = wl.replace(rates=(rho,) * wl.B)
            bufs = []
            for i in range(per):
                buf = torch.zeros(dec.layout.nbytes, dtype=torch.uint8, device=dev)
                fill_step_inputs(wr, step + i, dec.layout.views(buf))
                bufs.append(buf)
            for i in range(W):
                dec.step(bufs[i])
            flags = torch.zeros((K, wl.B), dtype=torch.int32, device=dev)
            dec.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            with torch.cuda.stream(dec.stream):
                e0.record(dec.stream)
                for i in range(K):
                    dec.step(bufs[W + i])
                    flags[i].copy_(dec.flag, non_blocking=True)
                e1.record(dec.stream)
            e1.synchronize()
            step += per
            ms = e0.elapsed_time(e1) / K
            f = flags.float().mean().item()
            t = ctx + step
            bytes_step = (weight_bytes * (1 + f) + lm_bytes + head_bytes +
                          wl.L * min(t, wl.sinks + wl.window) * per_tok + f * wl.L * t * per_tok)
            res[f"rho_{rho}"] = {"ms_per_step": ms, "tokens_per_s": wl.B * 1e3 / ms,
                                 "realized_rho": f, "gb_per_step": bytes_step / 1e9,
                                 "achieved_gbs": bytes_step / (ms * 1e-3) / 1e9}
        # always-full model: its own graph
        s_ = dec.stream
        torch.cuda.synchronize(dev)
        oda.oda_graph_begin(s_)
        dec.issue_always_full()
        g = oda.oda_graph_end(s_)
        for _ in range(W):
            g.launch(s_)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(s_)
        for _ in range(K):
            g.launch(s_)
        e1.record(s_)
        e1.synchronize()
        g.close()
        ms_full = e0.elapsed_time(e1) / K
        t = ctx + step + W + K
        full_bytes = weight_bytes + lm_bytes + wl.L * t * per_tok
        res["always_full"] = {"ms_per_step": ms_full, "tokens_per_s": wl.B * 1e3 / ms_full,
                              "gb_per_step": full_bytes / 1e9,
                              "achieved_gbs": full_bytes / (ms_full * 1e-3) / 1e9}
        res["speedup_at_rho_0.125"] = ms_full / res["rho_0.125"]["ms_per_step"]
        res["device_error"] = dec.device_error()
        res["backbone_weight_gb"] = weight_bytes / 1e9
        print(json.dumps({"backbone_sweep": True, "workload": wl0.name, **res}), flush=True)
        out.append(res)
        dec.close()
        del dec
        torch.cuda.empty_cache()
    print(json.dumps({"backbone_summary": True, "model": "synthetic Qwen3-1.7B-shaped, batch 1",
                      "peak_gbs": hbm, "peak_source": peak_src,
                      "speedup_over_always_full_at_rho_0.125": {str(r["ctx"]): r["speedup_at_rho_0.125"] for r in out},
                      "tokens_per_s_at_rho_0.125": {str(r["ctx"]): r["rho_0.125"]["tokens_per_s"] for r in out},
                      "always_full_tokens_per_s": {str(r["ctx"]): r["always_full"]["tokens_per_s"] for r in out}}),
          flush=True)


def run_ours(args, wl, rank, world, local_rank):
    import torch
    from conditional_sparse_attention_b200 import oda
    from conditional_sparse_attention_b200.engine import OdaDecoder
    from workload import inputs as inputs_mod

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    wl = replica_workload(wl, rank, world)
    W, K = args.warmup, args.steps
    n_e2e = K if args.e2e else 0
    cap = W + K + W + n_e2e + 24   # + the unflagged / one-flag probes (2 x 9 steps)
    t_setup = time.perf_counter()
    dec = OdaDecoder(wl, device=dev, capacity_steps=cap, kv_format=args.kv)
    n_store = min(cap, W + K)
    store = [dec.make_step_buffer(s) for s in range(n_store)]
    torch.cuda.synchronize(dev)
    setup_s = time.perf_counter() - t_setup

    # first step including graph capture (the pages' "first request" includes capture)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    tf = time.perf_counter()
    if not args.eager:
        dec.capture()
    dec.stage(store[0])
    dec.launch()
    dec.synchronize()
    first_ms = (time.perf_counter() - tf) * 1000.0
    step_idx = 1
    for _ in range(W):
        dec.step(store[step_idx % n_store])
        step_idx += 1
    dec.synchronize()

    # ---------------- timed region: K steps, device-timed with events on the launching stream
    sampler = ClockSampler(local_rank) if rank == 0 else None
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    if sampler:
        sampler.start()
        time.sleep(0.3)
    flags_log, pos_log = [], []
    pos_before = dec.pos.clone()
    flag_hist = torch.zeros((K, wl.B), dtype=torch.int32, device=dev)
    pos_hist = torch.zeros((K, wl.B), dtype=torch.int32, device=dev)
    with torch.cuda.stream(dec.stream):
        ev0.record(dec.stream)
        for i in range(K):
            pos_hist[i].copy_(dec.pos, non_blocking=True)
            dec.step(store[step_idx % n_store])
            flag_hist[i].copy_(dec.flag, non_blocking=True)
            step_idx += 1
        ev1.record(dec.stream)
    torch.cuda.synchronize(dev)
    clocks = sampler.stop() if sampler else None
    if world > 1:
        torch.distributed.barrier()
    elapsed_ms = max_over_ranks(ev0.elapsed_time(ev1), world, dev)
    flags = flag_hist.cpu().numpy()
    poss = pos_hist.cpu().numpy()
    total_bytes = sum(step_bytes(wl, poss[i].tolist(), flags[i].tolist(), args.kv) for i in range(K))
    realized_rate = float(flags.mean())
    launches = sum(kernel_launches(wl, bool(flags[i].any())) for i in range(K))

    # ---------------- per-kernel timing: each attention kernel replayed as a graph of one launch
    # per layer (no host gaps), CUDA events on the launching stream
    hbm, peak_src = peaks()
    per_tok = wl.Hkv * KV_BYTES_PER_TOKEN_HEAD[args.kv]
    pos_now = dec.pos.cpu().numpy()
    pats = {}
    for f in flags:
        if f.any():
            key = tuple(int(x) for x in f)
            pats[key] = pats.get(key, 0) + 1
    if not pats:
        pats = {tuple([1] + [0] * (wl.B - 1)): 1}
    full_bytes = full_ms = 0.0
    n_full = 0
    for pat, count in pats.items():
        ft = torch.tensor(pat, dtype=torch.int32, device=dev)
        ms = time_layer_kernels(dec, 1, ft, reps=2)
        full_ms += count * ms
        full_bytes += count * sum(int(pos_now[b]) * per_tok for b in range(wl.B) if pat[b])
        n_full += 2 * wl.L
    full_gbs = full_bytes / (full_ms * 1e-3) / 1e9
    tpt = traffic_per_token() if args.kv == "bf16" else None
    n_pat_launches = sum(pats.values())
    full_traffic = (tpt * (full_bytes / per_tok) / n_pat_launches) if tpt else None
    loc_ms = time_layer_kernels(dec, 0, None, reps=3)
    head_ms = time_head(dec, reps=5)
    head_bytes = inputs_mod.head_param_count(wl.D) * 4
    loc_bytes = sum(min(int(pos_now[b]), wl.sinks + wl.window) * per_tok for b in range(wl.B))
    loc_gbs = loc_bytes / (loc_ms * 1e-3) / 1e9
    n_flagged_steps = sum(1 for f in flags if f.any())
    att_bytes = wl.L * (K * loc_bytes + (full_bytes if n_flagged_steps else 0.0))
    att_ms = wl.L * (K * loc_ms + (full_ms if n_flagged_steps else 0.0))
    att_gbs = att_bytes / (att_ms * 1e-3) / 1e9
    att_us_per_step = att_ms * 1e3 / K

    # ---------------- end to end: pinned host inputs -> H2D, step, D2H of the results
    e2e = e2e_detail = None
    if args.e2e:
        host = [b.cpu().pin_memory() for b in store]
        out_r = torch.empty(dec.results.numel(), dtype=torch.float32).pin_memory()
        # the same step inputs (and so the same scheduled flags) as the device-timed loop
        for i in range(2):
            dec.step(host[(W - 1 + i) % n_store])
        dec.synchronize()
        if world > 1:
            torch.distributed.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(dec.stream):
            e0.record(dec.stream)
            dec.copy_stream.wait_event(e0)   # every upload of the timed steps starts after e0
            h0 = time.perf_counter()
            for i in range(n_e2e):
                dec.step(host[(1 + W + i) % n_store])
                dec.read_results(out_r)   # h_prev, score and flags in one device-to-host copy
            host_issue_s = time.perf_counter() - h0
            e1.record(dec.stream)
        torch.cuda.synchronize(dev)
        e_ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
        e2e = {"value": world * n_e2e / (e_ms * 1e-3), "unit": UNIT,
               "h2d_bytes_per_step": dec.layout.nbytes,
               "d2h_bytes_per_step": out_r.numel() * 4}
        # the copies alone, for reading the end-to-end number: uploads back to back on the copy
        # stream, and the read-backs on the step stream
        c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(dec.copy_stream):
            c0.record(dec.copy_stream)
            for i in range(n_e2e):
                dec.staging[i % 2].copy_(host[(1 + W + i) % n_store], non_blocking=True)
            c1.record(dec.copy_stream)
        c1.synchronize()
        d0, d1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(dec.stream):
            d0.record(dec.stream)
            for i in range(n_e2e):
                dec.read_results(out_r)
            d1.record(dec.stream)
        d1.synchronize()
        e2e_detail = {"upload_us_per_step": c0.elapsed_time(c1) * 1e3 / n_e2e,
                      "upload_gbs": dec.layout.nbytes * n_e2e / (c0.elapsed_time(c1) * 1e-3) / 1e9,
                      "readback_us_per_step": d0.elapsed_time(d1) * 1e3 / n_e2e,
                      "host_issue_us_per_step": host_issue_s * 1e6 / n_e2e,
                      "step_us": e_ms * 1e3 / n_e2e}
    # ---------------- a step with no flagged sequence (the IF node skips the retry): what the
    # local pass and the head leave to the glue (hidden-state sums, commit, condition node)
    quiet = dec.make_step_buffer(0)
    dec.layout.views(quiet)["sched"].zero_()
    if dec.routing_scheduled:
        n_probe = 8

        def probe_us(buf):
            """Device time per step of n_probe steps on one buffer; a sleep kernel ahead of the
            first event keeps the host's issue of the steps out of the interval."""
            dec.step(buf)
            dec.synchronize()
            p0, p1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            with torch.cuda.stream(dec.stream):
                torch.cuda._sleep(4_000_000)
                p0.record(dec.stream)
                for _ in range(n_probe):
                    dec.step(buf)
                p1.record(dec.stream)
            p1.synchronize()
            return p0.elapsed_time(p1) * 1e3 / n_probe

        quiet_us = probe_us(quiet)
        # the step-input staging copy alone (device to device, in the step stream); a sleep
        # kernel ahead of the copies keeps the host's issue time out of the interval
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(dec.stream):
            torch.cuda._sleep(4_000_000)
            s0.record(dec.stream)
            for i in range(8):
                dec.stage(store[i % n_store])
            s1.record(dec.stream)
        s1.synchronize()
        stage_us = s0.elapsed_time(s1) * 1e3 / 8
        step_detail = {"unflagged_step_us": quiet_us, "local_pass_us": loc_ms * 1e3 * wl.L,
                       "head_us": head_ms * 1e3, "staging_copy_us": stage_us,
                       "glue_us": quiet_us - loc_ms * 1e3 * wl.L - head_ms * 1e3 - stage_us}
        # a step with exactly one flagged sequence: its extra time over the unflagged step is the
        # retry of one sequence (every layer's full-set attention, the retry's hidden-state
        # glue and the conditional's launch)
        one = dec.make_step_buffer(0)
        ov = dec.layout.views(one)["sched"]
        ov.zero_()
        ov[0] = 1
        one_us = probe_us(one)
        rho = statistics.mean(wl.rates) if wl.rates else 0.0
        retry_us = one_us - quiet_us
        norm_us = quiet_us + rho * wl.B * retry_us
        rate_normalized = {"value": 1e6 / norm_us, "unit": UNIT, "rho": rho,
                           "unflagged_step_us": quiet_us, "one_flag_step_us": one_us,
                           "retry_us_per_sequence": retry_us,
                           "formula": "1 / (unflagged step + rho * B * (one-flag step - unflagged step))"}
    else:
        step_detail = None
        rate_normalized = None
    err = dec.device_error()

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        smp = OracleStepSample(wl, W, K)
        part = smp.run()
        cpu = {"value": 1.0 / smp.step_seconds(part), "unit": UNIT, "cores": cpu_cores(),
               "kind": "oracle", "sample": smp.describe(part)}

    if rank == 0:
        value = world * K / (elapsed_ms * 1e-3)
        step_gbs = total_bytes / (elapsed_ms * 1e-3) / 1e9
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K,
            "warmup": W, "ms_per_step": elapsed_ms / K, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if args.kv == "bf16" else "fp8",
            "data": "synthetic",
            "config": workload_config(wl, world, args.eager, args.kv),
            "roofline": {"bound": "hbm", "achieved": full_gbs, "peak": hbm, "unit": "GB/s",
                         "frac": full_gbs / hbm, "frac_of_nominal": full_gbs / NOMINAL_HBM_GBS,
                         "traffic": full_traffic,
                         "algorithmic_bytes_per_launch": full_bytes / n_pat_launches,
                         "kernel": f"attn_full_kernel<{args.kv} pages> (full set, flagged sequences)",
                         "peak_source": peak_src, "launches_timed": n_full,
                         "us_per_launch": full_ms * 1000.0 / sum(pats.values()),
                         "flag_patterns": {"".join(map(str, k)): v for k, v in pats.items()}},
            "step_roofline": {"algorithmic_gb_per_step": total_bytes / K / 1e9,
                              "achieved_gbs": step_gbs, "frac": step_gbs / hbm,
                              "frac_of_nominal": step_gbs / NOMINAL_HBM_GBS},
            "local_kernel": {"achieved_gbs": loc_gbs, "frac": loc_gbs / hbm,
                             "us_per_launch": loc_ms * 1000.0},
            # both attention kernels over the timed steps: K local passes and the full-set
            # launches of the realised flag patterns (one per layer of a flagged step)
            "attention_kernels": {"achieved_gbs": att_gbs, "frac": att_gbs / hbm,
                                  "frac_of_nominal": att_gbs / NOMINAL_HBM_GBS,
                                  "us_per_step": att_us_per_step},
            "recall_head": {"us_per_score": head_ms * 1000.0,
                            "achieved_gbs": head_bytes / (head_ms * 1e-3) / 1e9,
                            "frac": head_bytes / (head_ms * 1e-3) / 1e9 / hbm},
            "realized_recall_rate": realized_rate,
            "first_step_ms_incl_capture": first_ms, "setup_s": setup_s,
            "gpu_launches": launches, "device_error": err,
            "clocks": clocks, "e2e": e2e, "e2e_detail": e2e_detail, "step_detail": step_detail,
            "rate_normalized": rate_normalized,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    dec.close()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=32)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="cfg2")
    ap.add_argument("--kv", choices=["bf16", "fp8"], default="bf16",
                    help="KV cache page format (fp8: e4m3 codes with per-row fp32 scales)")
    ap.add_argument("--no-e2e", dest="e2e", action="store_false")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--eager", action="store_true",
                    help="issue every step's kernels directly instead of replaying a CUDA graph "
                         "(profilers cannot see kernel nodes of graphs with conditional nodes)")
    ap.add_argument("--kernel-only", choices=["full", "local", "head", "grad", "bbstep"], default=None,
                    help="profiling mode: launch one kernel (full or local attention, the recall "
                         "head) or one recall-head training step --kernel-reps times and exit")
    ap.add_argument("--kernel-reps", type=int, default=3)
    ap.add_argument("--sweep", action="store_true",
                    help="recall-rate x context sweep of the step against always-full attention")
    ap.add_argument("--backbone", action="store_true",
                    help="whole-model steps of the synthetic Qwen3-1.7B-shaped model (projections, "
                         "attention, head, retry, commit, LM head) at 4K..128K against always-full")
    ap.add_argument("--bb-separate", action="store_true",
                    help="--backbone: separate o_proj / MLP / QKV launches instead of the fused one")
    ap.add_argument("--backbone-ctx", default=None,
                    help="comma-separated contexts for --backbone (default 4K,16K,32K,64K,128K)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    from workload import configs
    wl = configs.get(args.workload)
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, wl, rank, world)
        return
    if args.kernel_only:
        run_kernel_only(args, wl, local_rank)
        return
    if args.sweep:
        run_sweep(args, wl, local_rank)
        return
    if args.backbone:
        run_backbone(args, local_rank)
        return
    import torch
    if world > 1:
        import datetime
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        run_ours(args, wl, rank, world, local_rank)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
