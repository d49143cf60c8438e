#!/usr/bin/env python
"""Benchmark of the JetBlock token mixer on B200.

Headline step (the `value` of the JSON line): one serving iteration of the
mixer on 2B shapes (H=12, dk=96, dv=256, d_model=1536, bf16 inputs, float32
state):
  prefill  one jet_jetblock_prefill call over one new 4096-token sequence
           (zero initial state): the kernel generator, then the chunked GDN
           prefill with the dynamic conv folded into its chunk preparation;
  decode   generator+conv with history (T=1) and the GDN decode step for 256
           running sequences, one token each; the state advances in place from
           step to step (64 pre-drawn token sets, cycled).
Tokens per step = 4096 + 256. Every rank runs its own copy of this work
(independent shards, no collective on the data path): weak scaling.

The same line carries the other stated workloads under "configs", each
timed on the device, end to end from pinned host buffers, against its
roofline, and beside a bounded sample on the float64 oracle:
  prefill_4b_t65536   one 65536-token prefill on 4B shapes (H=16, dk=128)
  prefill_2b_t262144  one 262144-token prefill on 2B shapes
  decode_2b_after_t262144  256 decode steps at B=1 continuing that prefill
  decode_4b_b{1,16,64,256,1024}  the 4B decode sweep
  prefill_2b_t262144_seqpar  (N > 1 only) the 262144-token prompt split into
                      N token ranges, one per GPU (strong scaling)
Their inputs use the block-seeded variant of the recipe (synth
prefill_inputs_blocked / decode_inputs_blocked) so that multi-GB draws take
seconds.

Prints one JSON line (rank 0). `--impl reference` times the float64 CPU
oracle on the headline workload instead (bounded sample per step).
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

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

PREFILL = synth.CONFIGS["prefill_2b_t4096"]
DECODE = synth.CONFIGS["decode_2b_b256"]
TOKENS_PER_STEP = PREFILL.B * PREFILL.T + DECODE.B
METRIC = "JetBlock prefill & decode tokens/s (2B/4B shapes); % of HBM/BF16 roofline"
WORKLOAD = ("mixed serving step on 2B JetBlock shapes: prefill of one 4096-token sequence "
            "(prefill_2b_t4096) + one decode token for each of 256 sequences (decode_2b_b256)")
CHUNK = 64
L2_BYTES = 126 * (1 << 20)


PEAK_SOURCE = {"measured": "measured (MEASURED_PEAKS.json hbm_gbs: a copy kernel timed alone on a B200)",
               "fallback": "fallback (no MEASURED_PEAKS.json: 6650 GB/s and 1590 TFLOP/s, an earlier "
                           "B200 measurement)"}


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return dict(hbm_gbs=d["hbm_gbs"], bf16_tflops=d["bf16_tflops"],
                    bf16_tflops_sustained=d.get("bf16_tflops_sustained", d["bf16_tflops"]), source="measured")
    return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0, source="fallback")


# ------------------------------------------------------------------ algorithmic traffic
def prefill_model(s, B=None, T=None):
    """Algorithmic bytes and flops of a prefill of B sequences x T tokens.
    "bytes" is the per-unit count of the scope table: K1 (x, v read, v' written)
    + K2 (q, k, v', g, beta read, o written, final state written), every input
    read once and every output written once. "bytes_fused" is the minimum of the
    one-call form, where v' never leaves the chip."""
    B = s.B if B is None else B
    T = s.T if T is None else T
    e = 2 if s.dtype == "bf16" else 4
    N = B * T
    w = (s.D * 32 + 32 * s.H * 4) * e
    k1 = N * (s.D * e + 2 * s.H * s.dv * e) + w
    k2 = N * s.H * (2 * s.dk * e + 2 * s.dv * e + 8) + B * s.H * s.dv * s.dk * 4
    fused = N * (s.D * e + s.H * (2 * s.dk * e + 2 * s.dv * e + 8)) + B * s.H * s.dv * s.dk * 4 + w
    gen_flops = N * (2 * s.D * 32 + 2 * 32 * s.H * 4 + 8 * s.H * s.dv)
    gdn_flops = N * s.H * (2 * CHUNK * (3 * s.dk + 2 * s.dv) + 6 * s.dk * s.dv + CHUNK * CHUNK / 3)
    return dict(bytes=k1 + k2, bytes_fused=fused, flops=gen_flops + gdn_flops,
                bytes_k1=k1, bytes_k2=k2, flops_k1=gen_flops, flops_k2=gdn_flops)


def decode_model(s, B=None):
    """Algorithmic bytes and flops of one decode step of B sequences: K1 with T=1
    (x, v read, v' written, history read and written) and K3 (state read and
    written, token vectors)."""
    B = s.B if B is None else B
    e = 2 if s.dtype == "bf16" else 4
    k1 = B * (s.D * e + 2 * s.H * s.dv * e + 2 * 3 * s.H * s.dv * e) + (s.D * 32 + 32 * s.H * 4) * e
    k3 = B * s.H * (2 * s.dv * s.dk * 4 + 2 * s.dk * e + 2 * s.dv * e + 8)
    return dict(bytes=k1 + k3, bytes_k1=k1, bytes_k3=k3,
                flops=B * (2 * s.D * 32 + 8 * s.H * s.dv) + B * s.H * 7 * s.dk * s.dv,
                flops_k1=B * (2 * s.D * 32 + 8 * s.H * s.dv), flops_k3=B * s.H * 7 * s.dk * s.dv)


def roofline_us(nbytes, flops, pk):
    return 1e6 * max(nbytes / (pk["hbm_gbs"] * 1e9), flops / (pk["bf16_tflops"] * 1e12))


def model_bytes():
    """Algorithmic bytes (and flops) of each library call of the headline step."""
    p, d = prefill_model(PREFILL), decode_model(DECODE)
    return {
        "jetblock_prefill": dict(bytes=p["bytes"], bytes_fused=p["bytes_fused"], flops=p["flops"]),
        "genconv_decode": dict(bytes=d["bytes_k1"], flops=d["flops_k1"]),
        "gdn_decode": dict(bytes=d["bytes_k3"], flops=d["flops_k3"]),
    }


def csrc_digest(files):
    """Digest of the kernel sources a measurement depends on."""
    h = hashlib.sha256()
    d = os.path.join(ROOT, "linear_attention_lm_gen_b200", "csrc")
    for f in sorted(files):
        h.update(f.encode())
        h.update(open(os.path.join(d, f), "rb").read())
    return h.hexdigest()[:16]


def ncu_traffic(call: str):
    """DRAM bytes per call (read + write, summed over its launches) from a
    committed ncu summary, only if it was taken on the current sources."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    ent = json.load(open(p)).get(call)
    if not ent or ent.get("sources_sha") != csrc_digest(ent.get("sources", [])):
        return None
    return ent.get("dram_bytes_per_launch")


# ------------------------------------------------------------------ clocks
class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.proc = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu=timestamp,{self.FIELDS}", "--format=csv,noheader,nounits",
                 "-i", str(index), "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self, t0: float, t1: float):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=10)
        rows = []
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                ts = time.mktime(time.strptime(parts[0].split(".")[0], "%Y/%m/%d %H:%M:%S"))
                rows.append((ts, float(parts[1]), float(parts[2]), parts[4:9]))
            except ValueError:
                continue
        inside = [r for r in rows if t0 - 1.0 <= r[0] <= t1 + 1.0] or rows
        if not inside:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
        names = ["active_mask", "hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in inside for i in range(1, 5) if r[3][i].lower().startswith("active")})
        return {"sm_mhz": statistics.median(r[1] for r in inside), "sm_max_mhz": max(r[2] for r in inside),
                "reasons": reasons, "samples": len(inside)}


def as_torch(a):
    import torch
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(a))


# ------------------------------------------------------------------ the headline workload
class Workload:
    def __init__(self, device, seed: int):
        import torch
        import linear_attention_lm_gen_b200 as jet
        self.torch, self.jet, self.dev = torch, jet, device
        p = synth.prefill_inputs(PREFILL, seed=seed)
        d = synth.decode_inputs(DECODE, seed=seed + 1)
        self.host_p = {k: as_torch(v).pin_memory() for k, v in p.items() if isinstance(v, np.ndarray)}
        self.host_d = {k: as_torch(v).pin_memory() for k, v in d.items() if isinstance(v, np.ndarray)}
        # two device copies of the prefill inputs (the end-to-end pass copies the
        # next step's inputs in while the current step runs)
        self.pb = [{k: v.to(device) for k, v in self.host_p.items()} for _ in range(2)]
        self.d = {k: v.to(device) for k, v in self.host_d.items()}
        P, Dc = PREFILL, DECODE
        bf = torch.bfloat16
        self.ob = [torch.empty((P.B, P.T, P.H, P.dv), device=device, dtype=bf) for _ in range(2)]
        self.S_out = torch.empty((P.B, P.H, P.dv, P.dk), device=device, dtype=torch.float32)
        self.S = self.d["S0"].clone()
        self.hist = [self.d["hist"].clone(), torch.empty_like(self.d["hist"])]
        self.vc_d = torch.empty((Dc.B, 1, Dc.H, Dc.dv), device=device, dtype=bf)
        self.odb = [torch.empty((Dc.B, Dc.H, Dc.dv), device=device, dtype=bf) for _ in range(2)]
        ws = jet.jet_jetblock_prefill_workspace_size(P.B, P.T, P.H, P.dk, P.dv)
        self.ws = torch.empty(max(ws, 16), device=device, dtype=torch.uint8)
        # pinned host buffers for the end-to-end pass
        self.h_o = [torch.empty(self.ob[0].shape, dtype=bf).pin_memory() for _ in range(2)]
        self.h_o_d = [torch.empty(self.odb[0].shape, dtype=bf).pin_memory() for _ in range(2)]

    # the library calls of one step, in order (each timed between two events)
    CALLS = ("jetblock_prefill", "genconv_decode", "gdn_decode")

    def step(self, stream, i: int, ev=None, counts=None, buf: int = 0):
        jet, p, d = self.jet, self.pb[buf], self.d
        o, o_d = self.ob[buf], self.odb[buf]

        def mark(j):
            if ev is not None:
                ev[j].record(stream)
            if counts is not None:
                counts.append(jet.jet_launch_count())
        mark(0)
        # prefill: generator, then the GDN prefill with the conv folded into its chunks (one call)
        jet.jet_jetblock_prefill(p["x"], p["W1"], p["W2"], p["q"], p["k"], p["v"], p["g"], p["beta"], None, None,
                                 None, o, self.S_out, self.ws, stream=stream)
        mark(1)
        s = i % DECODE.steps
        hin, hout = self.hist[i % 2], self.hist[(i + 1) % 2]
        # decode: generator + conv with the history (T = 1), then the state update
        jet.jet_dyn_conv_v(d["x"][s][:, None], d["W1"], d["W2"], d["v"][s][:, None], hin, self.vc_d, hout,
                           stream=stream)
        mark(2)
        jet.jet_gdn_decode_step(d["q"][s], d["k"][s], self.vc_d[:, 0], d["g"][s], d["beta"][s], self.S, o_d,
                                stream=stream)
        mark(3)

    def h2d(self, i: int, buf: int) -> int:
        """Copy one step's inputs from pinned host memory (current stream); returns bytes."""
        n = 0
        p = self.pb[buf]
        for k in ("x", "q", "k", "v", "g", "beta"):
            p[k].copy_(self.host_p[k], non_blocking=True)
            n += p[k].numel() * p[k].element_size()
        s = i % DECODE.steps
        for k in ("x", "q", "k", "v", "g", "beta"):
            self.d[k][s].copy_(self.host_d[k][s], non_blocking=True)
            n += self.d[k][s].numel() * self.d[k][s].element_size()
        return n

    def d2h(self, buf: int) -> int:
        """Read one step's outputs back into pinned host memory (current stream); returns bytes."""
        self.h_o[buf].copy_(self.ob[buf], non_blocking=True)
        self.h_o_d[buf].copy_(self.odb[buf], non_blocking=True)
        return self.ob[buf].numel() * 2 + self.odb[buf].numel() * 2


# ------------------------------------------------------------------ CPU oracle legs
def oracle_step(orc, p64, d64, frac: float = 1.0, dstep: int = 0):
    """The headline workload on the float64 oracle; `frac` < 1 takes the first frac
    of the prefill tokens and of the decode sequences (same mix). Returns tokens done."""
    Tp = max(1, int(round(PREFILL.T * frac)))
    Bd = max(1, int(round(DECODE.B * frac)))
    sl = lambda a: a[:, :Tp]
    orc.jetblock_prefill(sl(p64["x"]), p64["W1"], p64["W2"], sl(p64["q"]), sl(p64["k"]), sl(p64["v"]),
                         sl(p64["g"]), sl(p64["beta"]))
    s = dstep % DECODE.steps
    one = lambda a: a[s:s + 1, :Bd]
    orc.jetblock_decode(one(d64["x"]), d64["W1"], d64["W2"], one(d64["q"]), one(d64["k"]), one(d64["v"]),
                        one(d64["g"]), one(d64["beta"]), d64["S0"][:Bd], d64["hist"][:Bd])
    return Tp * PREFILL.B + Bd


def f64_inputs(inp):
    return {k: synth.to_f64(v, inp["dtype"]) if v.dtype == np.uint16 else v.astype(np.float64)
            for k, v in inp.items() if isinstance(v, np.ndarray)}


def oracle_inputs(seed: int):
    return (f64_inputs(synth.prefill_inputs(PREFILL, seed=seed)),
            f64_inputs(synth.decode_inputs(DECODE, seed=seed + 1)))


def cpu_baseline(seed: int, budget_s: float = 15.0):
    import oracle
    orc = oracle.get()
    p64, d64 = oracle_inputs(seed)
    t0 = time.perf_counter()
    tokens, reps = 0, 0
    while True:
        tokens += oracle_step(orc, p64, d64, 1.0, reps)
        reps += 1
        if time.perf_counter() - t0 > budget_s:
            break
    dt = time.perf_counter() - t0
    return {"value": tokens / dt, "unit": "tokens/s", "cores": orc.num_threads(), "kind": "oracle",
            "sample": f"{reps} full step(s) of the same workload (4096-token prefill + one decode token "
                      f"for each of 256 sequences) on the float64 oracle, {dt:.1f} s"}


def cpu_prefill_sample(s, inp, budget_s: float):
    """The oracle on consecutive 1024-token pieces of sequence 0 of a prefill
    workload (each piece continues the state and history of the last), until
    the budget is spent."""
    import oracle
    orc = oracle.get()
    dt_ = inp["dtype"]
    W1, W2 = synth.to_f64(inp["W1"], dt_), synth.to_f64(inp["W2"], dt_)
    S, hist, done = None, None, 0
    t0 = time.perf_counter()
    while done < s.T and time.perf_counter() - t0 < budget_s:
        sl = lambda k: synth.to_f64(inp[k][:1, done:done + 1024], dt_) if inp[k].dtype == np.uint16 \
            else inp[k][:1, done:done + 1024].astype(np.float64)
        r = orc.jetblock_prefill(sl("x"), W1, W2, sl("q"), sl("k"), sl("v"), sl("g"), sl("beta"), S, hist)
        S, hist = r["S"], r["hist"]
        done += sl("x").shape[1]
    el = time.perf_counter() - t0
    return {"value": done / el, "unit": "tokens/s", "cores": orc.num_threads(), "kind": "oracle",
            "sample": f"the first {done} tokens of sequence 0 in 1024-token pieces on the float64 oracle, {el:.1f} s"}


def cpu_decode_sample(s, inp, budget_s: float, seqs: int = 16):
    """The oracle on decode steps of the first `seqs` sequences until the budget is spent."""
    import oracle
    orc = oracle.get()
    d = f64_inputs({k: (v[:, :seqs] if k in ("x", "q", "k", "v", "g", "beta") else
                        (v[:seqs] if k in ("S0", "hist") else v)) if isinstance(v, np.ndarray) else v
                    for k, v in inp.items()})
    B = d["x"].shape[1]
    S, h, n = d["S0"], d["hist"], 0
    t0 = time.perf_counter()
    while time.perf_counter() - t0 < budget_s:
        st = n % d["x"].shape[0]
        one = lambda a: a[st:st + 1]
        r = orc.jetblock_decode(one(d["x"]), d["W1"], d["W2"], one(d["q"]), one(d["k"]), one(d["v"]), one(d["g"]),
                                one(d["beta"]), S, h)
        S, h = r["S"], r["hist"]
        n += 1
    el = time.perf_counter() - t0
    return {"value": n * B / el, "unit": "tokens/s", "cores": orc.num_threads(), "kind": "oracle",
            "sample": f"{n} decode step(s) of {B} sequence(s) on the float64 oracle, {el:.1f} s"}


# ------------------------------------------------------------------ multi-rank plumbing
class Ranks:
    """One process per GPU (torchrun sets RANK / LOCAL_RANK / WORLD_SIZE). The
    path shards without any exchange: every rank runs the same per-GPU
    workload on its own inputs (weak scaling); the only collectives are the
    barriers around the timed regions and the max over ranks of their durations."""

    def __init__(self, env=None):
        env = os.environ if env is None else env
        self.world = int(env.get("WORLD_SIZE", "1"))
        self.rank = int(env.get("RANK", "0"))
        self.local = int(env.get("LOCAL_RANK", "0"))

    def seed(self, base: int) -> int:
        return base + 17 * self.rank              # distinct synthetic inputs per rank

    def max_over_ranks(self, x: float, device=None) -> float:
        if self.world == 1:
            return x
        import torch
        import torch.distributed as dist
        t = torch.tensor([x], dtype=torch.float64, device=device)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())

    def value(self, tokens_per_rank_per_step: int, steps: int, ms_max: float) -> float:
        """Whole-job tokens/s: every rank's tokens over the slowest rank's time."""
        return tokens_per_rank_per_step * self.world * steps / (ms_max * 1e-3)


def run_reference(args):
    if Ranks().rank != 0:                       # rank 0 alone runs the oracle; the others exit
        return 0
    import oracle
    orc = oracle.get()
    p64, d64 = oracle_inputs(args.seed)
    t0 = time.perf_counter()
    oracle_step(orc, p64, d64, 1.0, 0)
    full = time.perf_counter() - t0
    frac = min(1.0, 150.0 / max(1e-9, full * (args.steps + args.warmup)))
    for i in range(args.warmup):
        oracle_step(orc, p64, d64, frac, i)
    t0 = time.perf_counter()
    tokens = 0
    for i in range(args.steps):
        tokens += oracle_step(orc, p64, d64, frac, i)
    dt = time.perf_counter() - t0
    value = tokens / dt
    sample = (f"each step: the first {frac:.3f} of the workload's prefill tokens and decode sequences "
              f"(same 16:1 mix) on the float64 oracle")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * dt / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": WORKLOAD, "tokens_per_step_full": TOKENS_PER_STEP, "sample_fraction": frac},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": orc.num_threads(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ the other stated workloads
class Timer:
    """Per-step events on one stream, L2 flushed between steps when asked (the
    flush runs between the events, outside the timed work)."""

    def __init__(self, torch, device, stream, flush: bool):
        self.torch, self.stream = torch, stream
        self.scrub = torch.empty(2 * L2_BYTES // 4, device=device, dtype=torch.float32) if flush else None

    def run(self, fn, steps: int, warmup: int):
        torch = self.torch
        with torch.cuda.stream(self.stream):
            for i in range(warmup):
                fn(i)
            ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
            for i in range(steps):
                if self.scrub is not None:
                    self.scrub.fill_(float(i))
                ev[i][0].record(self.stream)
                fn(warmup + i)
                ev[i][1].record(self.stream)
        self.stream.synchronize()
        return [a.elapsed_time(b) for a, b in ev]          # ms per step


def host_pinned(inp, keys):
    return {k: as_torch(inp[k]).pin_memory() for k in keys}


def measure_prefill_config(ctx, name: str, steps: int, warmup: int, keep: bool = False):
    """One jet_jetblock_prefill call over the whole prompt per step."""
    torch, jet, dev, stream, rk, pk = ctx["torch"], ctx["jet"], ctx["dev"], ctx["stream"], ctx["rk"], ctx["pk"]
    s = synth.CONFIGS[name]
    inp = synth.prefill_inputs_blocked(s, seed=ctx["seed"])
    keys = ("x", "q", "k", "v", "g", "beta")
    host = host_pinned(inp, keys + ("W1", "W2"))
    d = {k: v.to(dev) for k, v in host.items()}
    o = torch.empty((s.B, s.T, s.H, s.dv), device=dev, dtype=torch.bfloat16)
    S = torch.empty((s.B, s.H, s.dv, s.dk), device=dev, dtype=torch.float32)
    hist = torch.empty((s.B, 3, s.H, s.dv), device=dev, dtype=torch.bfloat16)
    ws = torch.empty(max(16, jet.jet_jetblock_prefill_workspace_size(s.B, s.T, s.H, s.dk, s.dv)), device=dev,
                     dtype=torch.uint8)
    call = lambda i: jet.jet_jetblock_prefill(d["x"], d["W1"], d["W2"], d["q"], d["k"], d["v"], d["g"], d["beta"],
                                              None, hist, None, o, S, ws, stream=stream)
    ctx["barrier"]()
    ms = Timer(torch, dev, stream, flush=False).run(call, steps, warmup)      # inputs are GBs: larger than L2
    t = rk.max_over_ranks(statistics.median(ms), dev)
    # end to end: the step's inputs copied in from pinned memory and o read back, every step
    h_o = torch.empty(o.shape, dtype=torch.bfloat16).pin_memory()
    h2d = sum(host[k].numel() * host[k].element_size() for k in keys)
    d2h = o.numel() * 2

    def e2e(i):
        for k in keys:
            d[k].copy_(host[k], non_blocking=True)
        call(i)
        h_o.copy_(o, non_blocking=True)
    ctx["barrier"]()
    e_ms = rk.max_over_ranks(statistics.median(Timer(torch, dev, stream, False).run(e2e, max(2, steps // 2), 1)),
                             dev)
    m = prefill_model(s)
    tok = s.B * s.T
    r_us = roofline_us(m["bytes"], m["flops"], pk)
    out = {"workload": f"one jet_jetblock_prefill call over {s.B} x {s.T} tokens (H={s.H}, dk={s.dk}, dv={s.dv}, "
                       f"d_model={s.D}, bf16, float32 state, zero initial state)",
           "tokens_per_s": rk.world * tok / (t * 1e-3), "us_per_call": t * 1e3, "steps": steps, "warmup": warmup,
           "l2": "inputs larger than L2 (no flush needed)",
           "roofline": {"bound": "hbm" if m["bytes"] / pk["hbm_gbs"] > m["flops"] / (pk["bf16_tflops"] * 1e3)
                        else "tensor", "algorithmic_bytes": m["bytes"], "algorithmic_flops": m["flops"],
                        "achieved": m["bytes"] / (t * 1e-3) / 1e9, "peak": pk["hbm_gbs"], "unit": "GB/s",
                        "roofline_us": r_us, "frac": r_us / (t * 1e3),
                        "frac_vs_fused_bytes": 1e6 * m["bytes_fused"] / (pk["hbm_gbs"] * 1e9) / (t * 1e3)},
           "e2e": {"value": rk.world * tok / (e_ms * 1e-3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                   "d2h_bytes_per_step": d2h, "ms_per_step": e_ms}}
    kept = dict(S=S, hist=hist, W1=d["W1"], W2=d["W2"]) if keep else None
    del d, o, ws
    return out, inp, kept


def measure_decode_after(ctx, name: str, kept, reps: int):
    """s.steps decode steps at B=1 continuing the long prefill (its state and
    history), jet_jetblock_decode_step per step, captured once in a CUDA graph
    and replayed; a replay is one timed iteration (L2 flushed between replays)."""
    torch, jet, dev, stream, rk, pk = ctx["torch"], ctx["jet"], ctx["dev"], ctx["stream"], ctx["rk"], ctx["pk"]
    s = synth.CONFIGS[name]
    n = s.steps
    inp = synth.decode_inputs_blocked(s.with_(B=1), seed=ctx["seed"] + 5, steps=n)
    keys = ("x", "q", "k", "v", "g", "beta")
    host = host_pinned(inp, keys)
    d = {k: v.to(dev) for k, v in host.items()}
    S, W1, W2 = kept["S"], kept["W1"], kept["W2"]
    hb = [kept["hist"], torch.empty_like(kept["hist"])]
    o = torch.empty((n, 1, s.H, s.dv), device=dev, dtype=torch.bfloat16)
    taps = torch.empty((n, 1, s.H, 4), device=dev, dtype=torch.float32)

    def steps_fn():
        for t in range(n):
            jet.jet_jetblock_decode_step(d["x"][t], W1, W2, d["q"][t], d["k"][t], d["v"][t], hb[t % 2],
                                         hb[(t + 1) % 2], d["g"][t], d["beta"][t], S, o[t], taps[t], stream=stream)
    with torch.cuda.stream(stream):
        steps_fn()                                   # warm-up outside the graph
    stream.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        steps_fn()
    ctx["barrier"]()
    ms = Timer(torch, dev, stream, flush=True).run(lambda i: graph.replay(), reps, 3)
    t = rk.max_over_ranks(statistics.median(ms), dev)
    h_o = torch.empty(o.shape, dtype=torch.bfloat16).pin_memory()
    h2d = sum(host[k].numel() * host[k].element_size() for k in keys)

    def e2e(i):
        for k in keys:
            d[k].copy_(host[k], non_blocking=True)
        graph.replay()
        h_o.copy_(o, non_blocking=True)
    e_ms = rk.max_over_ranks(statistics.median(Timer(torch, dev, stream, True).run(e2e, max(2, reps // 2), 1)), dev)
    del graph
    m = decode_model(s, 1)
    us_step = t * 1e3 / n
    r_us = roofline_us(m["bytes"], m["flops"], pk)
    return {"workload": f"{n} decode steps at B=1 (2 launches each: generator, then conv + history shift + update "
                        f"in one pass over S) continuing the {s.T}-token prefill, as one CUDA graph",
            "tokens_per_s": rk.world * n / (t * 1e-3), "us_per_step": us_step, "replays": reps,
            "l2": "flushed between replays; within a replay the 1.2 MB state stays in L2 from step to step",
            "roofline": {"bound": "hbm", "algorithmic_bytes_per_step": m["bytes"], "roofline_us_per_step": r_us,
                         "frac": r_us / us_step, "achieved": m["bytes"] / (us_step * 1e-6) / 1e9,
                         "peak": pk["hbm_gbs"], "unit": "GB/s",
                         "note": "launch-latency bound: 2.4 MB per step is 0.37 us of HBM time"},
            "e2e": {"value": rk.world * n / (e_ms * 1e-3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": o.numel() * 2, "ms_per_step": e_ms}}, inp


def measure_decode_config(ctx, name: str, steps: int, warmup: int, token_sets: int = 8):
    """One decode step for every sequence per step: the generator + conv launch
    (T=1, with history) and the state update, the two calls of the headline step."""
    torch, jet, dev, stream, rk, pk = ctx["torch"], ctx["jet"], ctx["dev"], ctx["stream"], ctx["rk"], ctx["pk"]
    s = synth.CONFIGS[name]
    inp = synth.decode_inputs_blocked(s, seed=ctx["seed"] + 3, steps=token_sets)
    keys = ("x", "q", "k", "v", "g", "beta")
    host = host_pinned(inp, keys + ("W1", "W2", "S0", "hist"))
    d = {k: v.to(dev) for k, v in host.items()}
    S = d["S0"]
    hb = [d["hist"], torch.empty_like(d["hist"])]
    vc = torch.empty((s.B, 1, s.H, s.dv), device=dev, dtype=torch.bfloat16)
    o = torch.empty((s.B, s.H, s.dv), device=dev, dtype=torch.bfloat16)

    def call(i):
        st = i % token_sets
        jet.jet_dyn_conv_v(d["x"][st][:, None], d["W1"], d["W2"], d["v"][st][:, None], hb[i % 2], vc, hb[(i + 1) % 2],
                           stream=stream)
        jet.jet_gdn_decode_step(d["q"][st], d["k"][st], vc[:, 0], d["g"][st], d["beta"][st], S, o, stream=stream)
    m = decode_model(s)
    flush = m["bytes"] < L2_BYTES
    ctx["barrier"]()
    ms = Timer(torch, dev, stream, flush=flush).run(call, steps, warmup)
    t = rk.max_over_ranks(statistics.median(ms), dev)
    h_o = torch.empty(o.shape, dtype=torch.bfloat16).pin_memory()

    def e2e(i):
        st = i % token_sets
        for k in keys:
            d[k][st].copy_(host[k][st], non_blocking=True)
        call(i)
        h_o.copy_(o, non_blocking=True)
    e_ms = rk.max_over_ranks(statistics.median(Timer(torch, dev, stream, flush).run(e2e, max(3, steps // 2), 2)), dev)
    h2d = sum(host[k][0].numel() * host[k][0].element_size() for k in keys)
    r_us = roofline_us(m["bytes"], m["flops"], pk)
    del d, S, hb
    return {"workload": f"one decode token for each of {s.B} sequences on 4B shapes (H={s.H}, dk={s.dk}, "
                        f"dv={s.dv}, d_model={s.D}); generator + conv launch, then the state update",
            "tokens_per_s": rk.world * s.B / (t * 1e-3), "us_per_step": t * 1e3, "steps": steps, "warmup": warmup,
            "l2": "flushed between steps" if flush else "state larger than L2 (no flush needed)",
            "roofline": {"bound": "hbm", "algorithmic_bytes": m["bytes"], "roofline_us": r_us,
                         "achieved": m["bytes"] / (t * 1e-3) / 1e9, "peak": pk["hbm_gbs"], "unit": "GB/s",
                         "frac": r_us / (t * 1e3)},
            "e2e": {"value": rk.world * s.B / (e_ms * 1e-3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": o.numel() * 2, "ms_per_step": e_ms}}, inp


def measure_seqpar(ctx, name: str, steps: int, warmup: int):
    """One prompt split into N token ranges, one per rank (strong scaling):
    each rank runs its range, the ranks all-gather the conv halos and the
    (end state, transition) pairs over NCCL, compose the start states and
    correct their outputs (seqpar.sequence_parallel_prefill)."""
    torch, jet, dev, stream, rk, pk = ctx["torch"], ctx["jet"], ctx["dev"], ctx["stream"], ctx["rk"], ctx["pk"]
    from linear_attention_lm_gen_b200 import seqpar
    s = synth.CONFIGS[name]
    Tr = s.T // rk.world
    inp = synth.prefill_inputs_blocked(s.with_(T=Tr), seed=ctx["seed"] + 1000 * rk.rank)
    d = {k: as_torch(v).to(dev) for k, v in inp.items() if isinstance(v, np.ndarray)}
    call = lambda i: seqpar.sequence_parallel_prefill(d["x"], d["W1"], d["W2"], d["q"], d["k"], d["v"], d["g"],
                                                      d["beta"])
    ctx["barrier"]()
    ms = Timer(torch, dev, stream, flush=False).run(call, steps, warmup)
    t = rk.max_over_ranks(statistics.median(ms), dev)
    m = prefill_model(s)
    r_us = roofline_us(m["bytes"], m["flops"], pk) / rk.world
    return {"workload": f"one {s.T}-token prefill on 2B shapes split into {rk.world} ranges of {Tr} tokens, one per "
                        f"GPU: range pass, all-gather of the conv halos and the (E, A) pairs over NCCL, compose, "
                        f"output correction",
            "scaling": "strong", "tokens_per_s": s.T / (t * 1e-3), "us_per_call": t * 1e3, "steps": steps,
            "warmup": warmup, "exchange_bytes_per_rank": (s.H * s.dv * s.dk + s.H * s.dk * s.dk) * 4 + 3 * s.H * s.dv * 2,
            "roofline": {"bound": "hbm", "roofline_us": r_us, "frac": r_us / (t * 1e3),
                         "note": "the whole prompt's algorithmic bytes over N GPUs' HBM"}}


def varlen_lengths(n: int = 16, seed: int = 5, lo: int = 1, hi: int = 4096):
    """A mixed serving batch: n prompt lengths drawn log-uniform in [lo, hi]
    (seeded), the longest and shortest always present."""
    rng = np.random.default_rng(seed)
    lens = np.exp(rng.uniform(np.log(lo), np.log(hi), n - 2)).astype(int).clip(lo, hi).tolist()
    return [hi] + lens + [lo]


def measure_varlen_config(ctx, steps: int, warmup: int):
    """A serving round of prompts of mixed lengths on 2B shapes: one
    jet_jetblock_prefill_varlen call over the packed batch, against one
    jet_jetblock_prefill call per prompt on the same inputs."""
    torch, jet, dev, stream, rk, pk = ctx["torch"], ctx["jet"], ctx["dev"], ctx["stream"], ctx["rk"], ctx["pk"]
    s = PREFILL
    lens = varlen_lengths()
    n, total = len(lens), sum(lens)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    inp = synth.prefill_inputs_blocked(s.with_(B=1, T=total), seed=ctx["seed"] + 7)
    keys = ("x", "q", "k", "v", "g", "beta")
    host = {k: as_torch(inp[k][0]).pin_memory() for k in keys}
    d = {k: v.to(dev) for k, v in host.items()}
    W1, W2 = as_torch(inp["W1"]).to(dev), as_torch(inp["W2"]).to(dev)
    o = torch.empty((total, s.H, s.dv), device=dev, dtype=torch.bfloat16)
    S = torch.empty((n, s.H, s.dv, s.dk), device=dev, dtype=torch.float32)
    hist = torch.empty((n, 3, s.H, s.dv), device=dev, dtype=torch.bfloat16)
    ws = torch.empty(max(16, jet.jet_jetblock_prefill_varlen_workspace_size(cu, s.H, s.dk, s.dv)), device=dev,
                     dtype=torch.uint8)
    call = lambda i: jet.jet_jetblock_prefill_varlen(d["x"], W1, W2, d["q"], d["k"], d["v"], d["g"], d["beta"], cu,
                                                     None, hist, None, o, S, ws, stream=stream)
    ws1 = torch.empty(max(16, max(jet.jet_jetblock_prefill_workspace_size(1, T, s.H, s.dk, s.dv) for T in lens)),
                      device=dev, dtype=torch.uint8)
    one = lambda key, a, b: d[key][a:b].unsqueeze(0)

    def per_prompt(i):
        for j in range(n):
            a, b = int(cu[j]), int(cu[j + 1])
            jet.jet_jetblock_prefill(one("x", a, b), W1, W2, one("q", a, b), one("k", a, b), one("v", a, b),
                                     one("g", a, b), one("beta", a, b), None, hist[j:j + 1], None,
                                     o[a:b].unsqueeze(0), S[j:j + 1], ws1, stream=stream)
    ctx["barrier"]()
    timer = Timer(torch, dev, stream, flush=True)          # the batch is ~0.3 GB: flush L2 between steps
    t = rk.max_over_ranks(statistics.median(timer.run(call, steps, warmup)), dev)
    t_loop = rk.max_over_ranks(statistics.median(timer.run(per_prompt, steps, warmup)), dev)
    h_o = torch.empty(o.shape, dtype=torch.bfloat16).pin_memory()
    h2d = sum(host[k].numel() * host[k].element_size() for k in keys)

    def e2e(i):
        for k in keys:
            d[k].copy_(host[k], non_blocking=True)
        call(i)
        h_o.copy_(o, non_blocking=True)
    ctx["barrier"]()
    e_ms = rk.max_over_ranks(statistics.median(timer.run(e2e, max(2, steps // 2), 1)), dev)
    m = prefill_model(s, B=1, T=total)
    nbytes = m["bytes"] + (n - 1) * s.H * s.dv * s.dk * 4          # one final state per prompt
    r_us = roofline_us(nbytes, m["flops"], pk)
    return {"workload": f"one jet_jetblock_prefill_varlen call over {n} prompts of lengths {lens} ({total} tokens) "
                        f"packed along the token axis (2B shapes: H={s.H}, dk={s.dk}, dv={s.dv}, d_model={s.D}, "
                        f"bf16, zero initial states)",
            "tokens_per_s": rk.world * total / (t * 1e-3), "us_per_call": t * 1e3, "steps": steps, "warmup": warmup,
            "l2": "flushed between steps",
            "one_call_per_prompt": {"tokens_per_s": rk.world * total / (t_loop * 1e-3), "us_per_round": t_loop * 1e3,
                                    "calls": n},
            "roofline": {"bound": "hbm", "algorithmic_bytes": nbytes, "achieved": nbytes / (t * 1e-3) / 1e9,
                         "peak": pk["hbm_gbs"], "unit": "GB/s", "roofline_us": r_us, "frac": r_us / (t * 1e3)},
            "e2e": {"value": rk.world * total / (e_ms * 1e-3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": o.numel() * 2, "ms_per_step": e_ms}}, inp, s.with_(B=1, T=total)


def layer_weights(s, seed: int):
    """Seeded bf16 layer weights ~ N(0, 1/fan_in) on 2B/4B shapes, gamma = 1 + 0.1 N(0, 1)."""
    rng = np.random.Generator(np.random.PCG64([seed, 11]))
    bf = lambda *shape: synth.jetblock._draw(rng, shape, "bf16", scale=1.0 / np.sqrt(shape[0]))
    D, H, dk, dv = s.D, s.H, s.dk, s.dv
    w = dict(Wq=bf(D, H * dk), Wk=bf(D, H * dk), Wv=bf(D, H * dv), Wg=bf(D, H), Wb=bf(D, H), Wz=bf(D, H * dv),
             Wo=bf(H * dv, D), W1=bf(D, 32), W2=bf(32, H * 4))
    w["gamma"] = (1.0 + 0.1 * rng.standard_normal(dv)).astype(np.float32)
    return w


LAYER_ORDER = ("Wq", "Wk", "Wv", "Wg", "Wb", "Wz", "Wo", "gamma", "W1", "W2")


def layer_model(s, B: int, T: int):
    """Algorithmic flops and bytes of the layer over B x T tokens: the seven GEMMs and the mixer's
    flops; bytes of the fused minimum (x in, y out, every weight once, final state and history out)."""
    N = B * T
    D, H, dk, dv = s.D, s.H, s.dk, s.dv
    proj = 2 * H * dk + 2 * H * dv + 2 * H
    flops = 2 * N * D * proj + 2 * N * H * dv * D
    if T > 1:
        flops += prefill_model(s, B=B, T=T)["flops"]
    else:
        flops += decode_model(s, B=B)["flops"]
    weights = 2 * (D * proj + H * dv * D + D * 32 + 32 * H * 4) + 4 * dv
    state = B * H * dv * dk * 4 * (1 if T > 1 else 2) + B * 3 * H * dv * 2 * 2
    return dict(flops=flops, bytes=2 * N * D * 2 + weights + state)


def measure_layer_config(ctx, name: str, T: int, steps: int, warmup: int):
    """The JetBlock layer (jet_jetblock_layer): prefill of T tokens, or (T = 1) one decode step of B
    sequences with the state advanced in place."""
    torch, jet, dev, stream, rk, pk = ctx["torch"], ctx["jet"], ctx["dev"], ctx["stream"], ctx["rk"], ctx["pk"]
    s = synth.CONFIGS[name]
    B = s.B
    w = layer_weights(s, ctx["seed"])
    g = {k: as_torch(v).to(dev) for k, v in w.items()}
    x_np = synth.jetblock._draw(np.random.Generator(np.random.PCG64([ctx["seed"], 12])), (B, T, s.D), "bf16")
    xh = as_torch(x_np).pin_memory()
    x = xh.to(dev)
    S = torch.zeros((B, s.H, s.dv, s.dk), device=dev, dtype=torch.float32)
    hist = [torch.zeros((B, 3, s.H, s.dv), device=dev, dtype=torch.bfloat16) for _ in range(2)]
    y = torch.empty((B, T, s.D), device=dev, dtype=torch.bfloat16)
    ws = torch.empty(max(16, jet.jet_jetblock_layer_workspace_size(B, T, s.D, s.H, s.dk, s.dv)), device=dev,
                     dtype=torch.uint8)
    decode = T == 1

    def call(i):
        if decode:      # one more token per sequence: the state advances in place
            jet.jet_jetblock_layer(x, *[g[k] for k in LAYER_ORDER], hist_in=hist[i % 2], hist_out=hist[(i + 1) % 2],
                                   S0=S, S_out=S, y=y, workspace=ws, stream=stream)
        else:           # the same prompt from a zero state every step
            jet.jet_jetblock_layer(x, *[g[k] for k in LAYER_ORDER], hist_out=hist[0], S_out=S, y=y, workspace=ws,
                                   stream=stream)
    m = layer_model(s, B, T)
    flush = not decode              # the prefill's inputs and weights fit in L2; the decode state does not
    ctx["barrier"]()
    t = rk.max_over_ranks(statistics.median(Timer(torch, dev, stream, flush=flush).run(call, steps, warmup)), dev)
    hy = torch.empty(y.shape, dtype=torch.bfloat16).pin_memory()

    def e2e(i):
        x.copy_(xh, non_blocking=True)
        call(i)
        hy.copy_(y, non_blocking=True)
    e_ms = rk.max_over_ranks(statistics.median(Timer(torch, dev, stream, flush).run(e2e, max(3, steps // 2), 2)), dev)
    tok = B * T
    r_us = roofline_us(m["bytes"], m["flops"], pk)
    bound = "hbm" if m["bytes"] / pk["hbm_gbs"] > m["flops"] / (pk["bf16_tflops"] * 1e3) else "tensor"
    what = (f"one decode token for each of {B} sequences" if decode else f"a {T}-token prompt") + \
        f" through jet_jetblock_layer on {name[:2].upper()} shapes (H={s.H}, dk={s.dk}, dv={s.dv}, d_model={s.D}): " \
        f"projections (cuBLAS), gates, the mixer, per-head RMSNorm and SiLU gate, output projection"
    out = {"workload": what, "tokens_per_s": rk.world * tok / (t * 1e-3), "us_per_call": t * 1e3, "steps": steps,
           "warmup": warmup, "l2": "flushed between steps" if flush else "state larger than L2 (no flush needed)",
           "roofline": {"bound": bound, "algorithmic_bytes": m["bytes"], "algorithmic_flops": m["flops"],
                        "achieved": (m["flops"] / (t * 1e-3) / 1e12) if bound == "tensor"
                        else m["bytes"] / (t * 1e-3) / 1e9,
                        "peak": pk["bf16_tflops"] if bound == "tensor" else pk["hbm_gbs"],
                        "unit": "TFLOP/s" if bound == "tensor" else "GB/s", "roofline_us": r_us,
                        "frac": r_us / (t * 1e3)},
           "e2e": {"value": rk.world * tok / (e_ms * 1e-3), "unit": "tokens/s",
                   "h2d_bytes_per_step": xh.numel() * 2, "d2h_bytes_per_step": y.numel() * 2, "ms_per_step": e_ms}}
    del g, S, ws
    return out, w, x_np


def cpu_layer_sample(s, w, x, budget_s: float, decode: bool):
    """The oracle's layer on the first tokens (prefill: pieces of 256 continuing the state) or on the
    first sequences (decode) of the workload, until the budget is spent."""
    import oracle
    from oracle import layer as olayer
    orc = oracle.get()
    f = {k: (synth.to_f64(v, "bf16") if v.dtype == np.uint16 else v.astype(np.float64)) for k, v in w.items()}
    args = [f[k] for k in LAYER_ORDER]
    xf = synth.to_f64(x, "bf16")
    done, t0 = 0, time.perf_counter()
    if decode:
        H, dv, dk = s.H, s.dv, s.dk
        while done < xf.shape[0] and time.perf_counter() - t0 < budget_s:
            xs = xf[done:done + 4, 0][None]                    # [1 step, 4 sequences, D]
            n = xs.shape[1]
            olayer.layer_decode(orc, xs, *args, np.zeros((n, H, dv, dk)), np.zeros((n, 3, H, dv)))
            done += n
        what = f"one decode step of the first {done} sequences"
    else:
        S, hist = None, None
        while done < xf.shape[1] and time.perf_counter() - t0 < budget_s:
            r = olayer.layer_prefill(orc, xf[:1, done:done + 256], *args, S, hist)
            S, hist = r["S"], r["hist"]
            done += min(256, xf.shape[1] - done)
        what = f"the first {done} tokens of the prompt in 256-token pieces"
    el = time.perf_counter() - t0
    return {"value": done / el, "unit": "tokens/s", "cores": orc.num_threads(), "kind": "oracle",
            "sample": f"{what} on the float64 oracle of the layer, {el:.1f} s"}


def run_configs(ctx, args):
    out = {}
    if ctx["rk"].world > 1:
        out["prefill_2b_t262144_seqpar"] = measure_seqpar(ctx, "prefill_2b_t262144", steps=5, warmup=3)
        ctx["torch"].cuda.empty_cache()
    cpu = not args.no_cpu_baseline and ctx["rk"].rank == 0
    budget = args.cpu_budget_config
    for lname, T in (("prefill_2b_t4096", 4096), ("decode_2b_b256", 1)):
        r, w, x = measure_layer_config(ctx, lname, T, steps=10 if T > 1 else 20, warmup=3)
        if cpu:
            r["cpu_baseline"] = cpu_layer_sample(synth.CONFIGS[lname], w, x, budget / 2, decode=T == 1)
        out["jetblock_layer_" + ("2b_t4096" if T > 1 else "2b_decode_b256")] = r
        ctx["torch"].cuda.empty_cache()
    r, inp, sp = measure_varlen_config(ctx, steps=10, warmup=3)
    if cpu:     # the oracle's cost per token does not depend on where the prompts are cut
        r["cpu_baseline"] = cpu_prefill_sample(sp, inp, budget / 2)
    out["prefill_2b_varlen_mixed"] = r
    del inp
    for name in ("prefill_4b_t65536", "prefill_2b_t262144"):
        long_ = name == "prefill_2b_t262144"
        r, inp, kept = measure_prefill_config(ctx, name, steps=5 if long_ else 10, warmup=3, keep=long_)
        if cpu:
            r["cpu_baseline"] = cpu_prefill_sample(synth.CONFIGS[name], inp, budget)
        out[name] = r
        del inp
        if long_:
            r, dinp = measure_decode_after(ctx, name, kept, reps=5)
            if cpu:
                r["cpu_baseline"] = cpu_decode_sample(synth.CONFIGS[name].with_(B=1), dinp, budget, seqs=1)
            out["decode_2b_after_t262144"] = r
            del kept
        ctx["torch"].cuda.empty_cache()
    for b in (1, 16, 64, 256, 1024):
        name = f"decode_4b_b{b}"
        r, inp = measure_decode_config(ctx, name, steps=20, warmup=3)
        if cpu:
            r["cpu_baseline"] = cpu_decode_sample(synth.CONFIGS[name], inp, budget / 3)
        out[name] = r
        ctx["torch"].cuda.empty_cache()
    return out


# ------------------------------------------------------------------ main GPU arm
def run_jet(args):
    import torch
    import torch.distributed as dist
    from linear_attention_lm_gen_b200 import build as jbuild

    rk = Ranks()
    world, rank, local = rk.world, rk.rank, rk.local
    if world != args.gpus:
        print(f"WORLD_SIZE={world} but --gpus {args.gpus}", file=sys.stderr)
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=device)

    jbuild.build()
    import linear_attention_lm_gen_b200 as jet
    jet.load_library()
    wl = Workload(device, seed=rk.seed(args.seed))
    stream = torch.cuda.Stream(device)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(device)

    def max_over_ranks(x: float) -> float:
        return rk.max_over_ranks(x, device)

    counts = []
    with torch.cuda.stream(stream):
        for i in range(args.warmup):
            wl.step(stream, i, counts=counts if i == args.warmup - 1 else None)
    per_call_launches = np.diff(np.array(counts))   # kernel launches behind each call of a step
    if jet.jet_device_error(stream) != 0:
        raise RuntimeError("device error word set after warm-up")

    # ---- device-resident timed pass: events only around the K steps. Each
    # launch starts while the one before it drains (programmatic dependent
    # launch); an event between two calls would end that overlap, so the
    # per-call times come from a second pass of the same K steps below.
    ncall = len(Workload.CALLS)
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local)
    time.sleep(0.3)
    barrier()
    n0 = jet.jet_launch_count()
    t_wall0 = time.time()
    with torch.cuda.stream(stream):
        start.record(stream)
        for i in range(args.steps):
            wl.step(stream, args.warmup + i)
        stop.record(stream)
    barrier()
    t_wall1 = time.time()
    launches = jet.jet_launch_count() - n0
    clk = clocks.stop(t_wall0, t_wall1)
    ms = max_over_ranks(start.elapsed_time(stop))
    if jet.jet_device_error(stream) != 0:
        raise RuntimeError("device error word set in the timed region")
    # ---- the same K steps with an event between every two calls: time per call
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(ncall + 1)] for _ in range(args.steps)]
    barrier()
    with torch.cuda.stream(stream):
        for i in range(args.steps):
            wl.step(stream, args.warmup + args.steps + i, evs[i])
    barrier()
    per_call = np.zeros(ncall)
    for e in evs:
        for j in range(ncall):
            per_call[j] += e[j].elapsed_time(e[j + 1])
    per_call /= args.steps                      # ms per call
    per_call = np.array([max_over_ranks(x) for x in per_call])
    if jet.jet_device_error(stream) != 0:
        raise RuntimeError("device error word set in the per-call pass")

    # ---- end-to-end pass: host inputs in, results out, through the same calls.
    # Every step copies its own inputs from pinned host memory and reads its
    # outputs back; the copies of step i+1's inputs and of step i-1's outputs
    # run on their own streams while step i computes (double-buffered).
    barrier()
    e_start, e_stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s_in, s_out = torch.cuda.Stream(device), torch.cuda.Stream(device)
    in_ready = [torch.cuda.Event() for _ in range(2)]
    comp_done = [torch.cuda.Event() for _ in range(2)]
    out_done = [torch.cuda.Event() for _ in range(2)]
    h2d = d2h = 0
    e_start.record(stream)
    s_in.wait_event(e_start)
    for i in range(args.steps):
        j = i % 2
        with torch.cuda.stream(s_in):
            if i >= 2:
                s_in.wait_event(comp_done[j])          # step i-2 has consumed buffer j
            h2d = wl.h2d(args.warmup + 2 * args.steps + i, j)
            in_ready[j].record(s_in)
        stream.wait_event(in_ready[j])
        if i >= 2:
            stream.wait_event(out_done[j])             # step i-2's outputs have been read back
        with torch.cuda.stream(stream):
            wl.step(stream, args.warmup + 2 * args.steps + i, buf=j)
        comp_done[j].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(comp_done[j])
            d2h = wl.d2h(j)
            out_done[j].record(s_out)
    for j in range(min(2, args.steps)):
        stream.wait_event(out_done[j])
    e_stop.record(stream)
    barrier()
    e_ms = max_over_ranks(e_start.elapsed_time(e_stop))
    del wl

    pk = peaks()
    configs = None
    if not args.no_configs:
        ctx = dict(torch=torch, jet=jet, dev=device, stream=stream, rk=rk, pk=pk, seed=rk.seed(args.seed + 100),
                   barrier=barrier)
        configs = run_configs(ctx, args)

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0

    mb = model_bytes()
    names = list(Workload.CALLS)
    calls = {}
    for j, n in enumerate(names):
        t = per_call[j] * 1e-3
        gbs = mb[n]["bytes"] / t / 1e9
        r_us = roofline_us(mb[n]["bytes"], mb[n]["flops"], pk)
        calls[n] = {"us_per_call": per_call[j] * 1e3, "kernels_per_call": int(per_call_launches[j]),
                    "algorithmic_bytes": mb[n]["bytes"], "algorithmic_flops": mb[n]["flops"], "achieved_gbs": gbs,
                    "hbm_frac": gbs / pk["hbm_gbs"], "roofline_us": r_us, "roofline_frac": r_us / (per_call[j] * 1e3)}
    calls["jetblock_prefill"]["algorithmic_bytes_fused"] = mb["jetblock_prefill"]["bytes_fused"]
    calls["jetblock_prefill"]["roofline_frac_vs_fused_bytes"] = \
        roofline_us(mb["jetblock_prefill"]["bytes_fused"], 0, pk) / (per_call[0] * 1e3)
    # the headline roofline is that of the call with the largest share of the step
    dom = names[int(np.argmax(per_call))]
    value = rk.value(TOKENS_PER_STEP, args.steps, ms)
    prefill_ms = per_call[0]
    decode_ms = per_call[1] + per_call[2]
    roof_step_us = sum(c["roofline_us"] for c in calls.values())
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded numpy PCG64; shapes of the 2B/4B JetBlock)",
        "config": {"workload": WORKLOAD, "tokens_per_step_per_gpu": TOKENS_PER_STEP,
                   "prefill": {"B": PREFILL.B, "T": PREFILL.T, "H": PREFILL.H, "dk": PREFILL.dk, "dv": PREFILL.dv,
                               "d_model": PREFILL.D, "chunk": CHUNK, "initial_state": "zero"},
                   "decode": {"B": DECODE.B, "H": DECODE.H, "dk": DECODE.dk, "dv": DECODE.dv, "d_model": DECODE.D,
                              "state": "float32, advanced in place every step", "token_sets": DECODE.steps},
                   "l2": "inputs larger than L2: 608 MB of decode state streamed per step (L2 126 MB)",
                   "parallelism": f"dp{world} (independent shard per GPU, no collective on the data path)"},
        "roofline": {"bound": "hbm", "kernel": dom, "achieved": calls[dom]["achieved_gbs"], "peak": pk["hbm_gbs"],
                     "unit": "GB/s", "frac": calls[dom]["hbm_frac"], "traffic": ncu_traffic(dom),
                     "peak_source": PEAK_SOURCE[pk["source"]],
                     "note": "the call with the largest share of the step; achieved = the scope table's "
                             "algorithmic bytes of the call / its event time in the per-call pass"},
        "ms_per_step_per_call_pass": float(sum(per_call)),
        "roofline_by_phase": {
            "prefill": {"call": "jetblock_prefill", "frac": calls["jetblock_prefill"]["roofline_frac"],
                        "frac_vs_fused_bytes": calls["jetblock_prefill"]["roofline_frac_vs_fused_bytes"]},
            "decode": {"calls": ["genconv_decode", "gdn_decode"],
                       "frac": (calls["genconv_decode"]["roofline_us"] + calls["gdn_decode"]["roofline_us"])
                       / (decode_ms * 1e3),
                       "gdn_decode_kernel_frac": calls["gdn_decode"]["roofline_frac"]}},
        "step_roofline": {"roofline_us": roof_step_us, "measured_us": 1e3 * ms / args.steps,
                          "frac": roof_step_us / (1e3 * ms / args.steps)},
        "phases": {
            "prefill": {"tokens_per_s": PREFILL.T / (prefill_ms * 1e-3), "us": prefill_ms * 1e3,
                        "roofline_us": calls["jetblock_prefill"]["roofline_us"]},
            "decode": {"tokens_per_s": DECODE.B / (decode_ms * 1e-3), "us": decode_ms * 1e3,
                       "roofline_us": calls["genconv_decode"]["roofline_us"] + calls["gdn_decode"]["roofline_us"]}},
        "calls": calls,
        "gpu_launches": int(launches),
        "clocks": clk,
        "e2e": {"value": TOKENS_PER_STEP * world * args.steps / (e_ms * 1e-3), "unit": "tokens/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e_ms / args.steps},
    }
    for ph in line["phases"].values():
        ph["roofline_frac"] = ph["roofline_us"] / ph["us"]
    if configs is not None:
        line["configs"] = configs
    if not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(args.seed, args.cpu_budget)
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="jet", choices=["jet", "reference"])
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-configs", action="store_true", help="time the headline step only")
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--cpu-budget-config", type=float, default=3.0)
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)        # at least 3 untimed warm-up steps
    if args.impl == "reference":
        return run_reference(args)
    return run_jet(args)


if __name__ == "__main__":
    sys.exit(main())
