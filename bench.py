#!/usr/bin/env python
"""Decode throughput of the Qwen2-1.5B-shaped decoder on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One JSON line on stdout (rank 0).  A "step" is one greedy decode step of the
whole hot path (embedding, 28 decoder layers, final norm, lm_head, argmax)
for every sequence of the batch.  Workload (default): the full 28-layer
Qwen2-1.5B shape, random-init bf16 weights, batch 1, a 512-token prompt of
uniform random ids prefilled first (timed separately), then the timed decode
steps (context 512 + warmup + steps).  Per step the kernels stream all
3.09 GB of weights, far more than the 126 MB L2, so no L2 flush is needed.
At batch 1 the step is one kernel launch (the streaming step), so the
roofline object (`roofline`) is that kernel's: the step's algorithmic bytes
over its event-timed launch, with the DRAM traffic recorded under
`profiles/` while its sources are unchanged.  Extra keys report the phases
of that launch (`phases_us`: critical-path time per phase, from the
kernel's own global-timer stamps), the other decode paths' step times
(`paths_ms`), batch 64 at 4096 context (`b64`, KV filled with N(0,1), with a
per-kernel-class breakdown), the 512-token prefill (`prefill`), the
32768-token prefill (`prefill_long`), the tcgen05 GEMM on the prefill linears
at 4096 tokens (the model's prefill chunk, first) and 32768 tokens
(`prefill_gemms`, fraction of the measured bf16 peak), the tcgen05 prefill
attention on the 32768-token prompt's last chunk (`prefill_attention`: 4096
query rows over 32768 keys, causal FLOPs over the measured bf16 peak), the
host-buffer entry
point end to end (`e2e`), SM clocks during the timed region (`clocks`) and
the CPU oracle baseline (`cpu_baseline`).  Fractions of HBM are given against
the measured copy bandwidth (`frac`) and against the ~8 TB/s datasheet
figure (`frac_vs_8tbs`).

Multi-GPU: replicas (`--gpus N` under torchrun): every rank decodes its own
sequences, no data-path collective; the time is the max over ranks.
"""

from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

import synth  # noqa: E402

METRIC = "decode tok/s (Qwen2-1.5B shape, bf16, B=1/64); achieved HBM GB/s vs peak"
WORKLOAD = "qwen2-1.5b-b1-prompt512-decode128"
WORKLOAD_B64 = "qwen2-1.5b-b64-ctx4096-decode32"
WORKLOAD_LONG = "qwen2-1.5b-b1-prompt32768-decode64"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
DATASHEET_HBM_GBS = 8000.0  # B200 HBM3e, datasheet


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


# ------------------------------------------------------------ distributed

class Dist:
    def __init__(self):
        self.rank = int(os.environ.get("RANK", "0"))
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.pg = None

    def init(self, use_cuda: bool):
        if self.world > 1:
            import torch.distributed as dist
            kw = dict(timeout=datetime.timedelta(seconds=300))
            if use_cuda:
                torch.cuda.set_device(self.local)
                dist.init_process_group("nccl", device_id=torch.device(f"cuda:{self.local}"), **kw)
            else:
                dist.init_process_group("gloo", **kw)
            self.pg = dist
        elif use_cuda:
            torch.cuda.set_device(self.local)

    def barrier(self):
        if self.pg:
            self.pg.barrier()

    def max(self, x: float) -> float:
        if not self.pg:
            return x
        dev = f"cuda:{self.local}" if torch.cuda.is_available() else "cpu"
        t = torch.tensor([x], dtype=torch.float64, device=dev)
        self.pg.all_reduce(t, op=self.pg.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.pg:
            self.pg.destroy_process_group()


# ------------------------------------------------------------------ clocks

class Clocks:
    """nvidia-smi sampling of SM clocks and throttle reasons during timed work."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits", "-lms", "100",
                 "-i", str(self.idx)], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        rows = []
        if self.path and os.path.exists(self.path):
            for line in open(self.path):
                f = [x.strip() for x in line.split(",")]
                if len(f) >= 8:
                    rows.append(f)
            os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[4 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


# ------------------------------------------------------- byte accounting

def layer_weight_bytes(s) -> int:
    es = 2 if s.dtype == "bf16" else 4
    qkvd = s.q_dim + 2 * s.kv_dim
    return es * (qkvd * s.hidden + qkvd + s.hidden * s.q_dim + 3 * s.intermediate * s.hidden + 2 * s.hidden)


def decode_step_bytes(s, batch: int, ctx: float) -> float:
    """Algorithmic HBM bytes of one decode step: every weight once (the
    embedding table only for the rows read), the KV of every visible position
    of every sequence read once, the new K/V written."""
    es = 2 if s.dtype == "bf16" else 4
    kv_per_pos = 2 * s.n_layers * s.kv_dim * es
    w = s.n_layers * layer_weight_bytes(s) + es * (s.vocab * s.hidden + s.hidden)
    return w + batch * (ctx + 1) * kv_per_pos + batch * s.hidden * es


# The source files each profiled kernel is built from: a recorded DRAM
# traffic figure stands only while these are unchanged.
KERNEL_SOURCES = {
    "gate_up": ["decode.cu", "decode.h", "common.cuh", "tma.h", "kernels.h"],
    "stream_step": ["sdecode.cu", "sdecode.h", "common.cuh", "tma.h", "pdecode.h"],
}


def kernel_src_hash(kernel: str = "gate_up") -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "qwen2_decode_step_b200", "csrc")
    for fn in KERNEL_SOURCES[kernel]:
        h.update(open(os.path.join(csrc, fn), "rb").read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str, workload: str):
    """Per-launch DRAM bytes from a committed ncu summary, if it was taken on
    the current kernel sources (else None)."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p))
    e = d.get(f"{kernel}@{workload}")
    if not e or e.get("src_hash") != kernel_src_hash(kernel):
        return None
    return e.get("dram_bytes_per_launch")


# --------------------------------------------------------------- oracle leg

def oracle_decode_sample(max_seconds: float, max_substeps: int, seed: int = 1003):
    """Times the CPU oracle on a bounded sample of the B=1 decode step of the
    full Qwen2-1.5B shape at context 512: a sub-step is one full-size decoder
    layer (decode of one token against 512 cached positions) plus 1/28 of the
    lm_head rows; 28 sub-steps are one token's work.  Returns (tok/s, sample
    description, sub-steps run)."""
    import oracle
    shape = synth.QWEN2_1P5B_ONE_LAYER
    w = {k: synth.weight(shape, k[0], k[1], seed) for k in shape.weight_shapes()
         if k[0] not in ("embed", "lm_head")}
    om = oracle.OracleModel(shape, max_seq=600)
    om.load(w)
    k, v = synth.kv_fill(shape, 512, seed, 0, 0)
    ok, ov = om.kv(0, 0)
    ok[:512] = k
    ov[:512] = v
    x = synth.hidden_input(shape, 1, seed)
    rows = (synth.QWEN2_1P5B.vocab + 27) // 28
    lm = synth.normal((rows, shape.hidden), 0.02, 99, "bf16")
    h = synth.normal((1, shape.hidden), 1.0, 98, "bf16")
    spent, n = 0.0, 0
    while n < max_substeps and (spent < max_seconds or n == 0):
        om.set_len(0, 512)
        t0 = time.perf_counter()
        om.forward_hidden(0, x)
        oracle.linear(h, lm, None, out_dtype=torch.float32)
        spent += time.perf_counter() - t0
        n += 1
    per_token = spent / n * 28
    desc = (f"{n} sub-steps; each = one full-size Qwen2-1.5B decoder layer decoding 1 token at "
            f"context 512 + lm_head GEMV over {rows} of {synth.QWEN2_1P5B.vocab} vocab rows (1/28); "
            f"28 sub-steps = one decode step (tok/s = 1 / (28 x mean sub-step time))")
    return 1.0 / per_token, desc, n


def run_reference(args, dist: Dist):
    """The oracle arm: the plain CPU oracle, as it stands, on the host cores."""
    dist.init(use_cuda=False)
    if dist.rank != 0:
        dist.close()
        return
    import oracle
    oracle.lib()
    # warm-up sub-steps (untimed), then K timed sub-steps bounded to a few minutes
    oracle_decode_sample(0.0, max(1, min(args.warmup, 3)))
    t0 = time.perf_counter()
    tps, desc, n = oracle_decode_sample(max_seconds=min(120.0, 1.5 * args.steps),
                                        max_substeps=args.steps)
    wall = time.perf_counter() - t0
    # A step of this arm is one sub-step (one layer of the token plus 1/28 of the
    # lm_head), so ms_per_step x steps is the arm's timed run.
    line = {
        "impl": "reference", "metric": METRIC, "value": tps, "unit": "tok/s", "n_gpus": args.gpus,
        "steps": n, "substeps_per_token": 28, "warmup": args.warmup,
        "ms_per_step": 1000.0 / tps / 28, "ms_per_token": 1000.0 / tps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64 (bf16 storage)", "data": "synthetic",
        "config": {"workload": WORKLOAD, "batch": 1, "context": 512, "sampled": True},
        "cpu_baseline": {"value": tps, "unit": "tok/s", "cores": 1, "kind": "oracle", "sample": desc},
        "e2e": {"value": tps, "unit": "tok/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "wall_s": wall,
    }
    print(json.dumps(line), flush=True)
    dist.close()


# ----------------------------------------------------------------- our arm

def cuda_time(fn, n: int) -> float:
    """ms of n calls of fn, CUDA events on the current stream."""
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    s.record()
    for _ in range(n):
        fn()
    e.record()
    torch.cuda.synchronize()
    return s.elapsed_time(e)


def run_ours(args, dist: Dist):
    import qwen2_decode_step_b200 as q2
    dist.init(use_cuda=True)
    dev = torch.cuda.current_device()
    shape = synth.QWEN2_1P5B
    wl = synth.WORKLOADS[WORKLOAD]
    seed = wl["seed"] + 100 * dist.rank
    prompt_len = wl["prompt"]
    b64 = not args.no_b64
    max_batch = 64 if b64 else 1
    past64 = synth.WORKLOADS[WORKLOAD_B64]["past"]
    max_seq = max(prompt_len + args.warmup + args.steps + 128, (past64 + args.b64_steps + 16) if b64 else 0)
    model = q2.Model(shape, max_seq=max_seq, max_batch=max_batch)
    for key in shape.weight_shapes():  # drawn on the GPU tensor by tensor, copied in, freed
        t = synth.weight(shape, key[0], key[1], seed, device="cuda")
        model.load_weight(key[0], key[1], t)
        del t
    torch.cuda.synchronize()

    # ---- prefill (load and generate are timed apart)
    ids = synth.prompt_ids(shape, prompt_len, seed, device="cuda")
    model.prefill(ids, [prompt_len])
    model.reset_kv()
    torch.cuda.synchronize()
    pre_ms = cuda_time(lambda: model.prefill(ids, [prompt_len]), 1)
    model.reset_kv()
    nxt = model.prefill(ids, [prompt_len])

    clocks = Clocks(dev)
    # ---- B = 1 decode: warm-up, then K timed steps
    bufs = [nxt.clone(), torch.empty_like(nxt)]
    for i in range(args.warmup):
        model.decode_step(bufs[i % 2], out=bufs[(i + 1) % 2])
    cur = args.warmup % 2
    clocks.start()
    dist.barrier()
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.nvtx.range_push("decode")  # lets ncu select exactly the timed steps
    s.record()
    for i in range(args.steps):
        model.decode_step(bufs[(cur + i) % 2], out=bufs[(cur + i + 1) % 2])
    e.record()
    torch.cuda.nvtx.range_pop()
    torch.cuda.synchronize()
    dist.barrier()
    ms = dist.max(s.elapsed_time(e))
    ms_step = ms / args.steps
    ctx_mean = prompt_len + args.warmup + (args.steps - 1) / 2.0
    step_bytes = decode_step_bytes(shape, 1, ctx_mean)

    # ---- inside the same decode step: with one launch per step (the streaming
    # step), the critical-path time of each phase from the kernel's own
    # global-timer stamps and the launch by CUDA events; otherwise each kernel
    # class by events around its launches (serialised, isolated)
    last = bufs[(cur + args.steps) % 2]
    ktimes, kernels_per_step = model.time_kernels(last, steps=min(args.steps, 20))

    # ---- the other decode paths of batch 1 on the same model (context)
    paths_ms = {}
    for path in ("kernels", "persistent"):
        try:
            model.set_decode_path(path)
        except q2.Q2Error:
            continue
        pb = [last.clone(), torch.empty_like(last)]
        for i in range(3):
            model.decode_step(pb[i % 2], out=pb[(i + 1) % 2])
        n_p = 10
        paths_ms[path] = dist.max(cuda_time_b64(model, pb, n_p)) / n_p
    model.set_decode_path("auto")
    model.set_seq_len(0, prompt_len + args.warmup + args.steps)

    # ---- e2e: the public host-buffer entry point, H2D ids + D2H next each step
    ids_h = torch.empty(1, dtype=torch.int64).pin_memory()
    out_h = torch.empty(1, dtype=torch.int64).pin_memory()
    ids_h.copy_(last.cpu())
    for _ in range(3):
        model.decode_step_host(ids_h, out_h)
        ids_h.copy_(out_h)
    dist.barrier()

    def e2e_step():
        model.decode_step_host(ids_h, out_h)
        ids_h.copy_(out_h)
    e2e_n = max(1, min(args.steps, 100))
    e2e_ms = dist.max(cuda_time(e2e_step, e2e_n)) / e2e_n

    # ---- batch 64 at 4096 context (KV N(0,1), kernel-only fill)
    b64_line = None
    if b64:
        B = 64
        for l in range(shape.n_layers):
            for b in range(B):
                k, v = synth.kv_fill(shape, past64, seed, l, b, device="cuda")
                gk, gv = model.kv_cache(l, b)
                gk[:, :past64].copy_(k.permute(1, 0, 2))
                gv[:, :past64].copy_(v.permute(1, 0, 2))
        torch.cuda.synchronize()
        for b in range(B):
            model.set_seq_len(b, past64)
        ids64 = synth.uniform_ids(B, shape.vocab, seed + 7, device="cuda")
        b64bufs = [ids64, torch.empty_like(ids64)]
        for i in range(3):
            model.decode_step(b64bufs[i % 2], out=b64bufs[(i + 1) % 2])
        n64 = args.b64_steps
        dist.barrier()
        ms64 = dist.max(cuda_time_b64(model, b64bufs, n64)) / n64
        ctx64 = past64 + 3 + (n64 - 1) / 2.0
        bytes64 = decode_step_bytes(shape, B, ctx64)
        # per kernel class inside the batch-64 step (events around each launch:
        # serialised, isolated times), with the HBM rate of the classes whose
        # bytes are known from the shapes
        k64, kps64 = model.time_kernels(b64bufs[n64 % 2], steps=3)
        H, I, qkvd = shape.hidden, shape.intermediate, shape.q_dim + 2 * shape.kv_dim
        cls_bytes = {"qkv": 2 * (qkvd * H + B * (H + qkvd)), "o": 2 * (H * shape.q_dim + B * 2 * H),
                     "gate_up": 2 * (2 * I * H + B * (H + I)), "down": 2 * (H * I + B * (I + 2 * H)),
                     "lm_head": 2 * shape.vocab * H + 4 * B * shape.vocab,
                     "attn": B * (past64 + 3 + n64 / 2.0) * 2 * shape.kv_dim * 2}
        breakdown = {}
        for k, (mean_ms, per) in k64.items():
            if not per:
                continue
            e = {"mean_ms": round(mean_ms, 5), "per_step": per}
            if k in cls_bytes and mean_ms > 0:
                e["gbs"] = round(cls_bytes[k] / (mean_ms / 1e3) / 1e9, 1)
                e["frac"] = round(e["gbs"] / float(peaks()[0]["hbm_gbs"]), 3)
            breakdown[k] = e
        b64_line = {"workload": WORKLOAD_B64, "batch": B, "value": B * dist.world / (ms64 / 1e3),
                    "unit": "tok/s", "ms_per_step": ms64, "steps": n64,
                    "achieved_gbs": bytes64 / (ms64 / 1e3) / 1e9, "bytes_per_step": bytes64,
                    "frac": bytes64 / (ms64 / 1e3) / 1e9 / float(peaks()[0]["hbm_gbs"]),
                    "kernels_ms": {"timing": "CUDA events around each launch of a replayed step "
                                             "(serialised, isolated: they do not add up to the step)",
                                   "by_class": breakdown, "kernels_per_step": kps64}}
    clk = clocks.stop()

    pk, pk_kind = peaks()
    hbm = float(pk["hbm_gbs"])
    gemms = None
    long_line = None
    if not args.no_long_prefill:
        wl_long = synth.WORKLOADS[WORKLOAD_LONG]
        long_line = long_prefill(shape, wl_long["seed"] + 100 * dist.rank, wl_long["prompt"])
    attn_rate = None
    if not args.no_long_prefill:
        attn_rate = prefill_attention_rate(shape, float(pk["bf16_tflops"]))
        attn_rate["peak_kind"] = pk_kind
    if not args.no_prefill_gemms:
        gemms = {str(t): prefill_gemm_rates(shape, t, float(pk["bf16_tflops"]))
                 for t in (int(x) for x in args.prefill_gemm_tokens.split(","))}
    step_gbs = step_bytes / (ms_step / 1e3) / 1e9
    if kernels_per_step == 1:
        # one launch per step: that kernel is the roofline's subject
        launch_ms = ktimes["step"][0]
        achieved = step_bytes / (launch_ms / 1e3) / 1e9 if launch_ms > 0 else None
        roofline = {"kernel": "sdecode_kernel (batch-1 streaming step, one launch per step)",
                    "bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s",
                    "frac": (achieved / hbm) if achieved else None,
                    "frac_vs_8tbs": (achieved / DATASHEET_HBM_GBS) if achieved else None,
                    "traffic": recorded_traffic("stream_step", WORKLOAD),
                    "bytes_per_launch": step_bytes, "mean_launch_ms": launch_ms, "peak_kind": pk_kind}
        kernel_times = {"phases_us": {k: round(v[0] * 1e3, 3) for k, v in ktimes.items()
                                      if v[1] and k != "step"},
                        "phases_timing": "critical path per phase instance inside the one launch "
                                         "(latest end of the phase minus latest end of the phase "
                                         "before, global-timer stamps)"}
    else:
        gu_ms, gu_n = ktimes["gate_up"]
        gu_bytes = 2 * shape.intermediate * shape.hidden * 2 + shape.hidden * 2 + 2 * shape.intermediate * 2
        achieved = gu_bytes / (gu_ms / 1e3) / 1e9 if gu_ms > 0 else None
        roofline = {"kernel": "gate_up", "bound": "hbm", "achieved": achieved, "peak": hbm,
                    "unit": "GB/s", "frac": (achieved / hbm) if achieved else None,
                    "frac_vs_8tbs": (achieved / DATASHEET_HBM_GBS) if achieved else None,
                    "traffic": recorded_traffic("gate_up", WORKLOAD),
                    "bytes_per_launch": gu_bytes, "mean_launch_ms": gu_ms, "peak_kind": pk_kind}
        kernel_times = {"kernels_ms": {k: {"mean_ms": round(v[0], 5), "per_step": v[1]}
                                       for k, v in ktimes.items() if v[1]},
                        "kernels_timing": "CUDA events around each launch of a replayed step "
                                          "(serialised, isolated: they do not add up to the step)"}
    line = {
        "metric": METRIC,
        "value": 1 * dist.world / (ms_step / 1e3),
        "unit": "tok/s",
        "n_gpus": dist.world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (random-init bf16 weights, uniform random prompt ids)",
        "config": {"workload": WORKLOAD, "batch": 1, "prompt": prompt_len,
                   "context": f"{prompt_len + args.warmup}..{prompt_len + args.warmup + args.steps}",
                   "l2": "no flush: each step streams 3.09 GB of weights (> 126 MB L2)",
                   "parallelism": f"replicas x{dist.world}"},
        "step_roofline": {"bytes_per_step": step_bytes, "achieved_gbs": step_gbs,
                          "peak_gbs": hbm, "frac": step_gbs / hbm, "frac_vs_8tbs": step_gbs / DATASHEET_HBM_GBS,
                          "peak_kind": pk_kind},
        "roofline": roofline,
        **kernel_times,
        "paths_ms": paths_ms,
        "gpu_launches": kernels_per_step * args.steps,
        "kernels_per_step": kernels_per_step,
        "prefill": {"tokens": prompt_len, "ms": pre_ms, "tok_s": prompt_len / (pre_ms / 1e3)},
        "prefill_long": long_line,
        "prefill_attention": attn_rate,
        "prefill_gemms": gemms and {"tokens": args.prefill_gemm_tokens,
                                    "peak_tflops": float(pk["bf16_tflops"]), "peak_kind": pk_kind,
                                    "kernel": "tc_gemm_kernel (tcgen05, TMEM)", "by_tokens": gemms},
        "e2e": {"value": 1 * dist.world / (e2e_ms / 1e3), "unit": "tok/s", "h2d_bytes_per_step": 8,
                "d2h_bytes_per_step": 8, "ms_per_step": e2e_ms,
                "api": "q2_model_decode_step_host (pinned host ids -> host next)"},
        "b64": b64_line,
        "clocks": clk,
    }
    model.close()
    if dist.rank == 0 and dist.world == 1 and not args.no_cpu_baseline:
        tps, desc, n = oracle_decode_sample(max_seconds=args.cpu_seconds, max_substeps=10_000)
        line["cpu_baseline"] = {"value": tps, "unit": "tok/s", "cores": 1, "kind": "oracle",
                                "sample": desc}
    if dist.rank == 0:
        print(json.dumps(line), flush=True)
    dist.close()


def prefill_gemm_rates(shape, tokens: int, peak_tflops: float, reps: int = 10):
    """The tcgen05 GEMM on the prefill linears of one `tokens`-token chunk
    (synthetic bf16 operands resident on the device), timed with CUDA events
    on the current stream: TFLOP/s and the fraction of the measured bf16 peak."""
    import qwen2_decode_step_b200 as q2
    H, I, qkvd = shape.hidden, shape.intermediate, shape.q_dim + 2 * shape.kv_dim
    g = torch.Generator(device="cuda")
    g.manual_seed(4242)
    out = {}
    for name, N, K in (("qkv", qkvd, H), ("o", H, shape.q_dim), ("gate_up", 2 * I, H), ("down", H, I)):
        x = torch.randn(tokens, K, device="cuda", generator=g).bfloat16()
        w = (torch.randn(N, K, device="cuda", generator=g) * 0.02).bfloat16()
        y = torch.empty(tokens, N, device="cuda", dtype=torch.bfloat16)
        for _ in range(3):
            q2.q2_linear(y, x, w)
        ms = cuda_time(lambda: q2.q2_linear(y, x, w), reps) / reps
        tf = 2.0 * tokens * N * K / (ms / 1e3) / 1e12
        out[name] = {"M": tokens, "N": N, "K": K, "ms": ms, "tflops": tf, "frac": tf / peak_tflops}
        del x, w, y
    q2.q2_check_device_error()
    return out


def prefill_attention_rate(shape, peak_tflops: float, S: int = 4096, T: int = 32768, reps: int = 10):
    """The tcgen05 prefill attention through q2_self_attention on the last
    S-row chunk of a T-token prompt (synthetic N(0,1) bf16 q/k/v resident on
    the device; q, k, v and out are ~59 MB for the Qwen2-1.5B shape, under
    the 126 MB L2, so a 256 MB buffer is written before every call): reps
    back-to-back (write, call) pairs timed with CUDA events on the current
    stream, minus reps writes alone timed the same way (the host's per-call
    work overlaps the device's as in a prefill).  FLOPs: QK^T and PV,
    4 * nh * hd per visible (row, key) pair, causal."""
    import qwen2_decode_step_b200 as q2
    nh, nkv, hd = shape.n_heads, shape.n_kv_heads, shape.head_dim
    g = torch.Generator(device="cuda")
    g.manual_seed(4343)
    q = torch.randn(S, nh, hd, device="cuda", generator=g).bfloat16()
    k = torch.randn(T, nkv, hd, device="cuda", generator=g).bfloat16()
    v = torch.randn(T, nkv, hd, device="cuda", generator=g).bfloat16()
    out = torch.empty(S, nh, hd, device="cuda", dtype=torch.bfloat16)
    scale = 1.0 / math.sqrt(hd)
    for _ in range(3):
        q2.q2_self_attention(out, q, k, v, scale)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")

    def flushed_call():
        flush.fill_(1)
        q2.q2_self_attention(out, q, k, v, scale)

    flushed_call()
    ms = (cuda_time(flushed_call, reps) - cuda_time(lambda: flush.fill_(1), reps)) / reps
    del flush
    q2.q2_check_device_error()
    pairs = S * (T - S) + S * (S + 1) // 2
    tf = 4.0 * nh * hd * pairs / (ms / 1e3) / 1e12
    return {"workload": f"{S} query rows over {T} keys (the {T}-token prompt's last chunk), "
                        f"{nh} heads / {nkv} kv heads, hd {hd}",
            "kernel": "attn_tc_kernel (tcgen05, TMEM)",
            "l2": "256 MB written before every call; the writes' own time subtracted",
            "ms": ms, "tflops": tf, "frac": tf / peak_tflops}


def long_prefill(shape, seed: int, tokens: int, decode_steps: int = 64):
    """Prefill of one `tokens`-token prompt on a fresh batch-1 model (weights
    drawn on the device), timed with CUDA events after one untimed run; then
    `decode_steps` greedy decode steps over that cache (3 untimed first),
    timed the same way."""
    import qwen2_decode_step_b200 as q2
    m = q2.Model(shape, max_seq=tokens + decode_steps + 8, max_batch=1)
    for key in shape.weight_shapes():
        t = synth.weight(shape, key[0], key[1], seed, device="cuda")
        m.load_weight(key[0], key[1], t)
        del t
    ids = synth.prompt_ids(shape, tokens, seed, device="cuda")
    m.prefill(ids, [tokens])
    m.reset_kv()
    ms = cuda_time(lambda: m.prefill(ids, [tokens]), 1)
    m.reset_kv()
    nxt = m.prefill(ids, [tokens])
    bufs = [nxt.clone(), torch.empty_like(nxt)]
    for i in range(3):
        m.decode_step(bufs[i % 2], out=bufs[(i + 1) % 2])
    n = max(1, decode_steps - 3)
    dms = cuda_time_b64(m, [bufs[1], bufs[0]], n) / n
    m.check_error()
    m.close()
    ctx = tokens + 3 + (n - 1) / 2.0
    dbytes = decode_step_bytes(shape, 1, ctx)
    hbm = float(peaks()[0]["hbm_gbs"])
    return {"workload": WORKLOAD_LONG, "tokens": tokens, "ms": ms, "tok_s": tokens / (ms / 1e3),
            "decode": {"steps": n, "context": f"{tokens + 3}..{tokens + 3 + n - 1}", "ms_per_step": dms,
                       "tok_s": 1.0 / (dms / 1e3), "bytes_per_step": dbytes,
                       "achieved_gbs": dbytes / (dms / 1e3) / 1e9, "frac": dbytes / (dms / 1e3) / 1e9 / hbm}}


def cuda_time_b64(model, bufs, n):
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    s.record()
    for i in range(n):
        model.decode_step(bufs[i % 2], out=bufs[(i + 1) % 2])
    e.record()
    torch.cuda.synchronize()
    return s.elapsed_time(e)


PROFILE_CASES = ("stream-small", "stream-full", "gemm4096", "attn-chunk", "b64-layer")


def run_profile_case(case: str):
    """A small, self-contained run of one kernel's workload for ncu captures
    (the summaries under profiles/ name these commands).  Prints one line of
    what ran; no timing is reported."""
    import dataclasses
    import qwen2_decode_step_b200 as q2
    torch.cuda.init()
    shape = synth.QWEN2_1P5B
    if case in ("stream-small", "stream-full"):
        # batch-1 streaming steps after a 512-token prompt: 4 layers and a
        # 32000-row vocabulary (0.47 GB of weights, above L2), or the full model
        if case == "stream-small":
            shape = dataclasses.replace(shape, n_layers=4, vocab=32000)
        seed = synth.WORKLOADS[WORKLOAD]["seed"]
        m = q2.Model(shape, max_seq=640, max_batch=1)
        for key in shape.weight_shapes():
            t = synth.weight(shape, key[0], key[1], seed, device="cuda")
            m.load_weight(key[0], key[1], t)
            del t
        m.set_decode_path("stream")
        m.set_graphs(False)
        nxt = m.prefill(synth.prompt_ids(shape, 512, seed, device="cuda"), [512])
        torch.cuda.synchronize()
        torch.cuda.nvtx.range_push("decode")
        for _ in range(6):
            nxt = m.decode_step(nxt)
        torch.cuda.synchronize()
        torch.cuda.nvtx.range_pop()
        m.check_error()
        m.close()
        print(f"{case}: {shape.n_layers} layers, 6 streaming steps at context 512..517")
    elif case == "gemm4096":
        out = prefill_gemm_rates(shape, 4096, 1.0, reps=1)
        print("gemm4096: the q/k/v, o, gate/up and down linears at M = 4096 (3 warm-up + 1 call each):",
              {k: (v["N"], v["K"]) for k, v in out.items()})
    elif case == "attn-chunk":
        # the last 4096-row chunk of the 32768-token prompt: rows at positions
        # 28672.. over 32768 keys, K/V token-major (the operator's layout)
        import math
        S, T, nh, nkv, hd = 4096, 32768, shape.n_heads, shape.n_kv_heads, shape.head_dim
        q = synth.normal((S, nh, hd), 1.0, 11, "bf16").cuda()
        k = synth.normal((T, nkv, hd), 1.0, 12, "bf16").cuda()
        v = synth.normal((T, nkv, hd), 1.0, 13, "bf16").cuda()
        o = torch.empty((S, nh, hd), dtype=torch.bfloat16, device="cuda")
        for _ in range(3):
            q2.q2_self_attention(o, q, k, v, 1.0 / math.sqrt(hd))
        torch.cuda.synchronize()
        q2.q2_check_device_error()
        print(f"attn-chunk: {S} query rows x {T} keys, {nh} heads / {nkv} kv heads, 3 calls")
    elif case == "b64-layer":
        # one full-size decoder layer at batch 64 over 4096 cached positions
        one = dataclasses.replace(shape, n_layers=1)
        wl = synth.WORKLOADS[WORKLOAD_B64]
        B, past = wl["batch"], wl["past"]
        m = q2.Model(one, max_seq=past + 16, max_batch=B)
        for key in one.weight_shapes():
            t = synth.weight(one, key[0], key[1], wl["seed"], device="cuda")
            m.load_weight(key[0], key[1], t)
            del t
        for b in range(B):
            kk, vv = synth.kv_fill(one, past, wl["seed"], 0, b, device="cuda")
            gk, gv = m.kv_cache(0, b)
            gk[:, :past].copy_(kk.permute(1, 0, 2))
            gv[:, :past].copy_(vv.permute(1, 0, 2))
            m.set_seq_len(b, past)
        m.set_graphs(False)
        ids = synth.uniform_ids(B, one.vocab, wl["seed"] + 7, device="cuda")
        torch.cuda.synchronize()
        torch.cuda.nvtx.range_push("decode")
        for _ in range(4):
            ids = m.decode_step(ids)
        torch.cuda.synchronize()
        torch.cuda.nvtx.range_pop()
        m.check_error()
        m.close()
        print(f"b64-layer: one decoder layer + head, batch {B}, context {past}..{past + 3}, 4 steps")


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--b64-steps", type=int, default=32)
    ap.add_argument("--no-b64", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-prefill-gemms", action="store_true")
    ap.add_argument("--no-long-prefill", action="store_true",
                    help="skip the 32768-token prefill timing")
    ap.add_argument("--prefill-gemm-tokens", default="4096,32768",
                    help="token counts at which the prefill linears are timed: the model's prefill "
                         "chunk (4096) and the whole 32768-token prompt as one product")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--profile", choices=PROFILE_CASES,
                    help="run one small kernel workload for an ncu capture and exit (no bench line)")
    args = ap.parse_args()
    if args.profile:
        run_profile_case(args.profile)
        return
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    dist = Dist()
    if args.impl == "reference":
        run_reference(args, dist)
    else:
        run_ours(args, dist)


if __name__ == "__main__":
    main()
