#!/usr/bin/env python
"""Benchmark of the KDA hot path on B200.

Step = one chunked prefill (tensor-core kernel) of the mid-size prefill
workload: B=4, T=8192, H=16, dk=dv=128, bf16 q/k/v, fp32 log_alpha and beta,
N(0, 0.1^2) fp32 initial state, chunk C=64 (inputs resident in HBM).
Metric: tokens/s (positions B*T per second, all heads). The same JSON line
carries the decode-step workload (B=256 sequences, H=32, d=128, fp32 state
[256,32,128,128] updated in place, bf16 inputs, fresh inputs every step) as
state-update GB/s, the packed variable-length prefill (64 sequences of
log-uniform length in [128, 32768], H=32) and the long-context workload (one
T=1,048,576 H=32 prefill, then 512 single-sequence decode steps replayed
from a CUDA graph), each with its roofline fraction; the other gate forms,
the fused input prologue and multi-token decode ("forms"); the backward of
the prefill workload ("backward", --backward-tokens N for the first N tokens
of each sequence); and the end-to-end step through the public API from
pinned host buffers, steps pipelined over three streams ("e2e").

  python bench.py [--gpus N --steps K --warmup W]        # this library
  python bench.py --impl reference [...]                 # the fp64 CPU oracle

With N > 1 (torchrun, one process per GPU) every rank runs its own copy of
the workload (independent sequences: no data-path collective); the time is
the max over ranks and the value counts the tokens of all ranks.
"""
import argparse
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

METRIC = "KDA prefill tokens/s & decode state GB/s (fraction of B200 roofline), 1 GPU"
PREFILL = dict(B=4, T=8192, H=16, dk=128, dv=128, chunk=64, init_std=0.1)
DECODE = dict(B=256, H=32, dk=128, dv=128, std=0.05)
VARLEN = dict(H=32)
LONG = dict(T=1 << 20, H=32, decode_steps=512)
BYTES_PER_HEAD_TOKEN = 3 * 256 + 512 + 4 + 256        # q,k,v + log_alpha + beta + o
FLOPS_PER_HEAD_TOKEN = 6 * 128 * 128 + 2 * 64 * (3 * 128 + 2 * 128)   # dense tiles, C = 64
PROFILE = os.path.join(ROOT, "profiles", "chunk64_prefill_b4_t8192_h16.txt")
KERNEL_SRC = os.path.join(ROOT, "gated_delta_rule_61_b200", "csrc", "kda_chunk.cu")
DECODE_PROFILE = os.path.join(ROOT, "profiles", "decode_step_b256_h32.txt")
VARLEN_PROFILE = os.path.join(ROOT, "profiles", "chunk64_varlen_64seq_h32.txt")
DECODE_SRC = os.path.join(ROOT, "gated_delta_rule_61_b200", "csrc", "kda_decode.cu")


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), "measured"
    except Exception:
        return 6650.0, 1590.0, "fallback"


def sustained_tflops():
    """The bf16 GEMM peak measured under the power cap over seconds (the
    denominator for a kernel timed inside a long loop), or the fallback."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops_sustained"])
    except Exception:
        return 1400.0


def code_hash(path):
    """sha256 (first 16 hex digits) of a CUDA source with comments and
    whitespace removed: a comment edit keeps it, a code change does not."""
    import re
    text = open(path).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    text = re.sub(r"\s+", "", text)
    return hashlib.sha256(text.encode()).hexdigest()[:16]


def kernel_traffic(profile=PROFILE, src=KERNEL_SRC):
    """dram bytes per launch from a committed ncu summary, if it was taken on
    the current kernel code (else None)."""
    try:
        text = open(profile).read()
        fields = dict(line.split(":", 1) for line in text.splitlines() if ":" in line)
        if fields.get("kernel_code_sha256_16", "").strip() != code_hash(src):
            return None
        return int(fields["dram_bytes_per_launch"].strip())
    except Exception:
        return None


class ClockSampler:
    """nvidia-smi clock/throttle samples every 50 ms during the timed regions."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        self.p = None

    def __enter__(self):
        try:
            self.p = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.Q,
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.p = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        if self.p is not None:
            self.p.terminate()
            try:
                self.p.wait(timeout=5)
            except Exception:
                self.p.kill()

    def summary(self):
        try:
            self.f.seek(0)
            rows = [r.split(",") for r in self.f.read().strip().splitlines() if r.strip()]
        except Exception:
            rows = []
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        sm = [float(r[1]) for r in rows if r[1].strip().replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].strip().replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if "Active" in v
                          and "Not" not in v})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows)}


def dist_setup(n_gpus, backend="nccl"):
    """Rank layout from the torchrun environment; joins the process group when
    there is more than one rank (NCCL on the GPUs; gloo for the CPU tests)."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        if backend == "nccl":
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                    device_id=torch.device("cuda", local))
        else:
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def max_over_ranks(x, world, device="cuda"):
    """The job's time is the slowest rank's: one all-reduce of a scalar."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world, sync_cuda=True):
    import torch
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    if sync_cuda:
        torch.cuda.synchronize()


def job_value(world, units_per_rank, ms_per_step):
    """Whole-job throughput: every rank processes units_per_rank per step
    (independent replicas), the step takes the slowest rank's time."""
    return world * units_per_rank / (ms_per_step * 1e-3)


def rank0_print(rank, line):
    """The JSON line comes from rank 0 alone."""
    if rank == 0:
        print(json.dumps(line), flush=True)


def _oracle_sample(n_tok, seed=0):
    import torch
    from gated_delta_rule_61_b200.inputs import prefill_inputs
    P = PREFILL
    return prefill_inputs(P["B"], n_tok, P["H"], P["dk"], P["dv"], dtype=torch.bfloat16,
                          seed=seed, init_std=P["init_std"])


def _oracle_run(inp, cores):
    import oracle
    t0 = time.perf_counter()
    oracle.kda_forward(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"],
                       init_state=inp["init_state"], n_threads=cores)
    return time.perf_counter() - t0


def _oracle_tokens_for(budget_s, cores):
    """Tokens per chain (all B*H chains) the oracle covers in about budget_s."""
    cal = 32
    dt = _oracle_run(_oracle_sample(cal), cores)
    return int(max(cal, min(PREFILL["T"], cal * budget_s / max(dt, 1e-6))))


def cpu_oracle_prefill(budget_s=12.0, seed=0):
    """Time the fp64 oracle on a bounded sample of the prefill workload: all
    B*H chains over their first n_tok tokens, n_tok sized to about budget_s
    seconds from a short calibration run."""
    import oracle
    cores = oracle.default_threads()
    n_tok = _oracle_tokens_for(budget_s, cores)
    dt = _oracle_run(_oracle_sample(n_tok, seed), cores)
    return PREFILL["B"] * n_tok / dt, cores, n_tok, dt


def bench_reference(args):
    """The fp64 oracle as the reference arm: rank 0 only, each step a bounded
    sample of the workload sized so the whole run takes about two minutes."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    cores = oracle.default_threads()
    per_step = max(0.05, min(args.ref_budget, 120.0 / (args.steps + args.warmup)))
    n_tok = _oracle_tokens_for(per_step, cores)
    inp = _oracle_sample(n_tok)
    for _ in range(args.warmup):
        _oracle_run(inp, cores)
    times = [_oracle_run(inp, cores) for _ in range(args.steps)]
    total = sum(times)
    P = PREFILL
    value = P["B"] * n_tok * args.steps / total
    sample = ("all %d (batch, head) chains, first %d of %d tokens per step, fp64 oracle"
              % (P["B"] * P["H"], n_tok, P["T"]))
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * P["B"] * P["T"] / value, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": "KDA prefill B=4 T=8192 H=16 dk=dv=128 bf16 q/k/v, fp32 "
                                   "gates and state, chunk C=64 (per GPU)",
                       "global_batch": P["B"], "seq_len": P["T"], "heads": P["H"],
                       "parallelism": "replicas"},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0},
            "gpu_launches": 0}
    rank0_print(rank, line)


def _time_calls(fn, n, stream):
    """Mean device time (ms) of n back-to-back calls, CUDA events on `stream`."""
    import torch
    fn()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    a.record(stream)
    for _ in range(n):
        fn()
    b.record(stream)
    torch.cuda.synchronize()
    return a.elapsed_time(b) / n


def bench_backward(args, dev, stream, hbm, world, inp):
    """Backward of the prefill workload (gradients of every input and the
    initial state from dL/do and dL/dS_final); --backward-tokens takes the
    first N tokens of each sequence instead of all of them."""
    import torch
    from gated_delta_rule_61_b200 import kda
    P = PREFILL
    T = min(args.backward_tokens, P["T"]) if args.backward_tokens > 0 else P["T"]
    x = {n: inp[n][:, :T].contiguous() for n in ("q", "k", "v", "log_alpha", "beta")}
    x["init_state"] = inp["init_state"]
    head_tokens = P["B"] * T * P["H"]
    state_bytes = 2 * P["B"] * P["H"] * P["dk"] * P["dv"] * 4
    g = torch.Generator(device=dev).manual_seed(78)
    d_o = torch.randn(x["v"].shape, device=dev, generator=g).to(x["v"].dtype)
    d_fin = torch.randn(x["init_state"].shape, device=dev, generator=g)
    need = kda.lib().kda_backward_workspace_bytes(P["B"], P["B"] * T, P["H"], P["dk"], P["dv"])
    ws = torch.empty(need, dtype=torch.uint8, device=dev)
    ms = _time_calls(lambda: kda.backward(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"],
                                          d_o, init_state=x["init_state"], d_final=d_fin,
                                          workspace=ws, stream=stream), 2, stream)
    # bytes: the forward inputs read twice (checkpoint pass and block
    # recomputation), d_o, the fp32 gradients written, states
    per = 2 * (3 * 256 + 512 + 4) + 256 + 4 * (3 * 128 + 128 + 1)
    gbs = (head_tokens * per + 3 * state_bytes) / (ms * 1e-3) / 1e9
    out = {"workload": "KDA backward of B=%d T=%d H=%d d=128 bf16 (token-recurrent, "
                       "checkpoints every 16 tokens)" % (P["B"], T, P["H"]),
           "ms_per_call": ms, "tokens_per_s": world * P["B"] * T / (ms * 1e-3),
           "roofline": {"bound": "latency (serial token chain)", "achieved": gbs,
                        "peak": hbm, "unit": "GB/s", "frac": gbs / hbm}}
    # the same through the input prologue (raw q/k projections, beta and gate
    # logits; the gradients are with respect to those)
    raw = {n: torch.randn(x[n].shape, device=dev, generator=g).to(x[n].dtype) for n in ("q", "k")}
    raw["beta"] = torch.randn(x["beta"].shape, device=dev, generator=g)
    raw["log_alpha"] = torch.randn(x["log_alpha"].shape, device=dev, generator=g) + 3.0
    ms_raw = _time_calls(lambda: kda.backward(raw["q"], raw["k"], x["v"], raw["log_alpha"],
                                              raw["beta"], d_o, init_state=x["init_state"],
                                              d_final=d_fin, workspace=ws, raw_qk=True,
                                              raw_beta=True, raw_gate=True, stream=stream),
                         2, stream)
    out["raw_inputs_ms_per_call"] = ms_raw
    del d_o, d_fin, ws, x, raw
    torch.cuda.empty_cache()
    return out


def bench_forms(args, dev, stream, hbm, world, inp, dec):
    """The other gate forms (one decay per token, none), the fused input
    prologue (raw q/k projections, beta and gate logits) and multi-token
    decode, each on the workload of its base entry point, with its own
    algorithmic bytes."""
    import torch
    from gated_delta_rule_61_b200 import kda
    from gated_delta_rule_61_b200.inputs import decode_inputs, decode_state
    P, D = PREFILL, DECODE
    out = {}
    head_tokens = P["B"] * P["T"] * P["H"]
    state_bytes = 2 * P["B"] * P["H"] * P["dk"] * P["dv"] * 4
    o = torch.empty_like(inp["v"])
    fs = torch.empty_like(inp["init_state"])
    g = torch.Generator(device=dev).manual_seed(77)
    gate_inputs = {
        "scalar": (torch.nn.functional.logsigmoid(
            torch.randn(P["B"], P["T"], P["H"], device=dev, generator=g) + 3.0), 4),
        "none": (None, 0),
    }
    for gate, (la, la_bytes) in gate_inputs.items():
        ms = _time_calls(lambda: kda.prefill(inp["q"], inp["k"], inp["v"], la, inp["beta"],
                                             init_state=inp["init_state"], chunk=64, gate=gate,
                                             o=o, final_state=fs, stream=stream), 10, stream)
        per = 3 * 256 + la_bytes + 4 + 256
        gbs = (head_tokens * per + state_bytes) / (ms * 1e-3) / 1e9
        out["prefill_gate_" + gate] = {
            "ms_per_call": ms, "tokens_per_s": world * P["B"] * P["T"] / (ms * 1e-3),
            "bytes_per_head_token": per,
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s",
                         "frac": gbs / hbm}}
    # raw projections: q, k ~ N(0, 1) unnormalised, beta and gate logits
    raw = {n: torch.randn(inp[n].shape, device=dev, generator=g).to(inp[n].dtype)
           for n in ("q", "k")}
    raw["beta"] = torch.randn(inp["beta"].shape, device=dev, generator=g)
    raw["log_alpha"] = torch.randn(inp["log_alpha"].shape, device=dev, generator=g) + 3.0
    ms = _time_calls(lambda: kda.prefill(raw["q"], raw["k"], inp["v"], raw["log_alpha"],
                                         raw["beta"], init_state=inp["init_state"], chunk=64,
                                         raw_qk=True, raw_beta=True, raw_gate=True, o=o,
                                         final_state=fs, stream=stream), 10, stream)
    gbs = (head_tokens * BYTES_PER_HEAD_TOKEN + state_bytes) / (ms * 1e-3) / 1e9
    out["prefill_raw_inputs"] = {
        "ms_per_call": ms, "tokens_per_s": world * P["B"] * P["T"] / (ms * 1e-3),
        "bytes_per_head_token": BYTES_PER_HEAD_TOKEN,
        "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s",
                     "frac": gbs / hbm}}
    del raw
    # decode forms and multi-token decode at B=256, H=32
    S = decode_state(D["B"], D["H"], D["dk"], D["dv"], std=D["std"], seed=17, device=dev)
    heads = D["B"] * D["H"]
    sbytes = 2 * D["dk"] * D["dv"] * 4
    d1 = decode_inputs(D["B"], D["H"], D["dk"], D["dv"], dtype=torch.bfloat16, seed=17,
                       device=dev)
    la_s = torch.nn.functional.logsigmoid(torch.randn(D["B"], D["H"], device=dev,
                                                      generator=g) + 3.0)
    od = torch.empty(D["B"], D["H"], D["dv"], dtype=torch.bfloat16, device=dev)
    for name, la, per_la, kw in (("decode_gate_scalar", la_s, 4, dict(gate="scalar")),
                                 ("decode_raw_inputs", d1["log_alpha"], 512,
                                  dict(raw_qk=True, raw_beta=True, raw_gate=True))):
        q1, k1, v1 = (d1[n][:, None] for n in ("q", "k", "v"))
        la1 = la[:, None]
        b1 = d1["beta"][:, None]
        ms = _time_calls(lambda: kda.decode(q1, k1, v1, la1, b1, S, o=od[:, None], stream=stream,
                                            **kw), 50, stream)
        per = sbytes + 3 * 256 + per_la + 4 + 256
        gbs = heads * per / (ms * 1e-3) / 1e9
        out[name] = {"us_per_step": ms * 1e3, "bytes_per_head_step": per,
                     "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s",
                                  "frac": gbs / hbm}}
    single_us = dec["ms_per_step"] * 1e3 if dec else None
    multi = {}
    for T in (2, 4, 8, 16):
        x = {n: torch.randn(D["B"], T, D["H"], D["dk"], device=dev, generator=g).to(torch.bfloat16)
             for n in ("q", "k", "v")}
        for n in ("q", "k"):
            x[n] = (x[n].float() / x[n].float().norm(dim=-1, keepdim=True)).to(torch.bfloat16)
        la = torch.nn.functional.logsigmoid(torch.randn(D["B"], T, D["H"], D["dk"], device=dev,
                                                        generator=g) + 3.0)
        b = torch.sigmoid(torch.randn(D["B"], T, D["H"], device=dev, generator=g))
        om = torch.empty(D["B"], T, D["H"], D["dv"], dtype=torch.bfloat16, device=dev)
        ms = _time_calls(lambda: kda.decode(x["q"], x["k"], x["v"], la, b, S, o=om,
                                            stream=stream), 20, stream)
        per = sbytes + T * BYTES_PER_HEAD_TOKEN
        gbs = heads * per / (ms * 1e-3) / 1e9
        multi["T%d" % T] = {
            "us_per_call": ms * 1e3, "tokens_per_s": world * D["B"] * T / (ms * 1e-3),
            "vs_single_steps": (T * single_us / (ms * 1e3)) if single_us else None,
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s",
                         "frac": gbs / hbm}}
    out["decode_multi_token"] = {
        "workload": "B=256 H=32 d=128, T tokens per sequence per call, state in place",
        **multi}
    del S
    torch.cuda.empty_cache()
    return out


def bench_ours(args):
    import torch
    from gated_delta_rule_61_b200 import kda
    from gated_delta_rule_61_b200.inputs import decode_inputs, decode_state, prefill_inputs
    world, rank, local = dist_setup(args.gpus)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    P, D = PREFILL, DECODE
    hbm, bf16_tf, peak_kind = peaks()

    # ---------------- prefill (the headline step) ----------------
    inp = prefill_inputs(P["B"], P["T"], P["H"], P["dk"], P["dv"], dtype=torch.bfloat16,
                         seed=1000 + rank, init_std=P["init_std"], device=dev)
    o = torch.empty_like(inp["v"])
    fs = torch.empty_like(inp["init_state"])
    stream = torch.cuda.current_stream(dev)

    def step():
        kda.prefill(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"],
                    init_state=inp["init_state"], chunk=P["chunk"], o=o, final_state=fs,
                    stream=stream)

    for _ in range(args.warmup):
        step()
    barrier(world)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    clk = ClockSampler(local).__enter__()
    if True:
        barrier(world)
        t_start = torch.cuda.Event(enable_timing=True)
        t_end = torch.cuda.Event(enable_timing=True)
        t_start.record(stream)
        for i in range(args.steps):
            ev[i][0].record(stream)
            step()
            ev[i][1].record(stream)
        t_end.record(stream)
        barrier(world)
    total_ms = max_over_ranks(t_start.elapsed_time(t_end), world)
    kernel_ms = statistics.mean(a.elapsed_time(b) for a, b in ev)
    ms_per_step = total_ms / args.steps
    tokens = P["B"] * P["T"]
    value = job_value(world, tokens, ms_per_step)
    head_tokens = tokens * P["H"]
    state_bytes = 2 * P["B"] * P["H"] * P["dk"] * P["dv"] * 4
    alg_bytes = head_tokens * BYTES_PER_HEAD_TOKEN + state_bytes
    achieved_gbs = alg_bytes / (kernel_ms * 1e-3) / 1e9
    traffic = kernel_traffic()
    tflops = head_tokens * FLOPS_PER_HEAD_TOKEN / (kernel_ms * 1e-3) / 1e12
    st, detail = kda.device_status()
    if st != kda.KDA_OK:
        raise RuntimeError("device status %d (detail %d) after the timed region" % (st, detail))

    # ---------------- decode (second half of the metric) ----------------
    dec = None
    if not args.no_decode:
        S = decode_state(D["B"], D["H"], D["dk"], D["dv"], std=D["std"], seed=7 + rank,
                         device=dev)
        n_in = min(args.decode_steps, 1000)
        steps_in = [decode_inputs(D["B"], D["H"], D["dk"], D["dv"], dtype=torch.bfloat16,
                                  seed=7 + rank, step=i, device=dev) for i in range(n_in)]
        od = torch.empty(D["B"], D["H"], D["dv"], dtype=torch.bfloat16, device=dev)

        def dstep(i):
            d = steps_in[i % n_in]
            kda.decode_step(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], S, o=od,
                            stream=stream)

        for i in range(args.warmup):
            dstep(i)
        barrier(world)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for i in range(args.decode_steps):
            dstep(i)
        b.record(stream)
        barrier(world)
        dms = max_over_ranks(a.elapsed_time(b), world) / args.decode_steps
        per_step_bytes = D["B"] * D["H"] * (2 * D["dk"] * D["dv"] * 4 + BYTES_PER_HEAD_TOKEN)
        gbs = world * per_step_bytes / (dms * 1e-3) / 1e9
        dec = {"value": gbs, "unit": "GB/s", "ms_per_step": dms, "steps": args.decode_steps,
               "tokens_per_s": world * D["B"] / (dms * 1e-3),
               "workload": "KDA decode B=256 H=32 dk=dv=128, fp32 state in place, bf16 inputs",
               "roofline": {"bound": "hbm", "achieved": gbs / world, "peak": hbm,
                            "unit": "GB/s", "frac": gbs / world / hbm,
                            "traffic": kernel_traffic(DECODE_PROFILE, DECODE_SRC),
                            "peak_kind": peak_kind}}
        del steps_in, S
    # ---------------- packed variable-length prefill ----------------
    var = None
    if not args.no_varlen:
        from gated_delta_rule_61_b200.inputs import varlen_lengths
        lengths = varlen_lengths(args.varlen_seqs, 128, args.varlen_max, seed=0)
        vin = prefill_inputs(1, 0, VARLEN["H"], 128, 128, dtype=torch.bfloat16, seed=2000 + rank,
                             init_std=0.1, lengths=lengths, device=dev)
        vo = torch.empty_like(vin["v"])
        vs = torch.empty_like(vin["init_state"])
        ws = torch.empty(kda.workspace_bytes(len(lengths), VARLEN["H"], 128, 128, kda.KDA_BF16, 64,
                                             True), dtype=torch.uint8, device=dev)

        def vstep():
            kda.prefill(vin["q"], vin["k"], vin["v"], vin["log_alpha"], vin["beta"],
                        init_state=vin["init_state"], cu_seqlens=vin["cu_seqlens"], chunk=64,
                        o=vo, final_state=vs, workspace=ws, stream=stream)

        vstep()
        barrier(world)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        n_v = 3
        a.record(stream)
        for _ in range(n_v):
            vstep()
        b.record(stream)
        barrier(world)
        vms = max_over_ranks(a.elapsed_time(b), world) / n_v
        t_tot = sum(lengths)
        vbytes = t_tot * VARLEN["H"] * BYTES_PER_HEAD_TOKEN + 2 * len(lengths) * VARLEN["H"] * 128 * 128 * 4
        vgbs = vbytes / (vms * 1e-3) / 1e9
        var = {"value": world * t_tot / (vms * 1e-3), "unit": "tokens/s", "ms_per_step": vms,
               "workload": "KDA packed varlen prefill: %d sequences log-uniform in [128, %d] "
                           "(%d tokens, longest %d), H=32, d=128, bf16, C=64"
                           % (len(lengths), args.varlen_max, t_tot, max(lengths)),
               "roofline": {"bound": "hbm", "achieved": vgbs, "peak": hbm, "unit": "GB/s",
                            "frac": vgbs / hbm, "traffic": kernel_traffic(VARLEN_PROFILE),
                            "peak_kind": peak_kind},
               "gpu_launches_per_step": 2}
        del vin, vo, vs
    # ---------------- long context: one 1M-token prefill, then graph-replayed decode ----------------
    lng = None
    if not args.no_long:
        L = dict(LONG)
        if args.long_tokens:
            L["T"] = args.long_tokens
        lin = prefill_inputs(1, L["T"], L["H"], 128, 128, dtype=torch.bfloat16, seed=4000 + rank,
                             device=dev)
        lo = torch.empty_like(lin["v"])
        ls = torch.empty(1, L["H"], 128, 128, dtype=torch.float32, device=dev)

        def lstep():
            kda.prefill(lin["q"], lin["k"], lin["v"], lin["log_alpha"], lin["beta"], chunk=64,
                        o=lo, final_state=ls, stream=stream)

        lstep()
        barrier(world)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        n_l = 3
        a.record(stream)
        for _ in range(n_l):
            lstep()
        b.record(stream)
        barrier(world)
        lms = max_over_ranks(a.elapsed_time(b), world) / n_l
        lbytes = L["T"] * L["H"] * BYTES_PER_HEAD_TOKEN + L["H"] * 128 * 128 * 4
        lgbs = lbytes / (lms * 1e-3) / 1e9
        del lin, lo
        # decode from the prefill's final state: B=1, so a step is a few microseconds
        # and launch overhead matters; the steps are captured once in a CUDA graph
        n_d = L["decode_steps"]
        dins = [decode_inputs(1, L["H"], 128, 128, dtype=torch.bfloat16, seed=4000 + rank,
                              step=i, device=dev) for i in range(n_d)]
        dout = torch.empty(n_d, 1, L["H"], 128, dtype=torch.bfloat16, device=dev)
        s_work = ls.clone()
        graph = torch.cuda.CUDAGraph()
        cap = torch.cuda.Stream(dev)
        cap.wait_stream(stream)
        with torch.cuda.graph(graph, stream=cap):
            for i, d in enumerate(dins):
                kda.decode_step(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], s_work,
                                o=dout[i], stream=cap)
        stream.wait_stream(cap)
        for _ in range(args.warmup):
            s_work.copy_(ls)
            graph.replay()
        barrier(world)
        ev_d = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                for _ in range(n_l)]
        for a, b in ev_d:
            s_work.copy_(ls)       # every replay starts from the prefill's final state
            a.record(stream)
            graph.replay()
            b.record(stream)
        barrier(world)
        gms = max_over_ranks(statistics.mean(a.elapsed_time(b) for a, b in ev_d), world)
        dus = gms * 1e3 / n_d
        dbytes = L["H"] * (2 * 128 * 128 * 4 + BYTES_PER_HEAD_TOKEN)
        lng = {"value": world * L["T"] / (lms * 1e-3), "unit": "tokens/s", "ms_per_step": lms,
               "workload": "KDA long-context prefill B=1 T=%d H=32 d=128 bf16, C=64, zero "
                           "initial state; then %d decode steps (CUDA graph)" % (L["T"], n_d),
               "roofline": {"bound": "hbm", "achieved": lgbs, "peak": hbm, "unit": "GB/s",
                            "frac": lgbs / hbm, "traffic": None, "peak_kind": peak_kind},
               "decode": {"us_per_step": dus, "steps": n_d, "unit": "GB/s",
                          "value": dbytes / (dus * 1e-6) / 1e9,
                          "frac": dbytes / (dus * 1e-6) / 1e9 / hbm}}
        del graph, dins, dout, s_work, ls
        torch.cuda.empty_cache()
    # ---------------- gate forms, fused prologue, multi-token decode ----------------
    forms = None
    if not args.no_forms:
        forms = bench_forms(args, dev, stream, hbm, world, inp, dec)
    bwd = None
    if not args.no_backward:
        bwd = bench_backward(args, dev, stream, hbm, world, inp)
    clk.__exit__(None, None, None)

    # ---------------- end to end through the public API (host buffers) ----------------
    e2e = None
    if not args.no_e2e:
        host = {k: (v.cpu().pin_memory() if v is not None else None) for k, v in inp.items()}
        o_h = torch.empty(o.shape, dtype=o.dtype).pin_memory()
        s_h = torch.empty(fs.shape, dtype=fs.dtype).pin_memory()
        h2d = sum(v.numel() * v.element_size() for v in host.values() if v is not None)
        d2h = o_h.numel() * o_h.element_size() + s_h.numel() * s_h.element_size()

        # Every step: its inputs from pinned host memory, one public call, its
        # results back to the host. Steps are pipelined over three streams with
        # two sets of device buffers, so one step's device-to-host copy and
        # call overlap the next step's host-to-device copy (PCIe carries both
        # directions at once); each step's copies still run in full inside the
        # timed region. (Splitting one step into per-sequence calls on three
        # streams was measured slower: the per-sequence launches run in a
        # slower ring shape.)
        s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        dbuf = [{k: (torch.empty_like(v, device=dev) if v is not None else None)
                 for k, v in host.items()} for _ in range(2)]
        obuf = [(torch.empty_like(o), torch.empty_like(fs)) for _ in range(2)]
        ev = {n: [torch.cuda.Event() for _ in range(2)] for n in ("h2d", "call", "d2h")}
        used = [False, False]

        def e2e_step(i):
            j = i % 2
            with torch.cuda.stream(s_in):
                if used[j]:
                    s_in.wait_event(ev["call"][j])   # the call two steps back read these
                for k, v in host.items():
                    if v is not None:
                        dbuf[j][k].copy_(v, non_blocking=True)
                ev["h2d"][j].record(s_in)
            stream.wait_event(ev["h2d"][j])
            if used[j]:
                stream.wait_event(ev["d2h"][j])     # its results were copied out
            g = dbuf[j]
            kda.prefill(g["q"], g["k"], g["v"], g["log_alpha"], g["beta"],
                        init_state=g["init_state"], chunk=P["chunk"], o=obuf[j][0],
                        final_state=obuf[j][1], stream=stream)
            ev["call"][j].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev["call"][j])
                o_h.copy_(obuf[j][0], non_blocking=True)
                s_h.copy_(obuf[j][1], non_blocking=True)
                ev["d2h"][j].record(s_out)
            used[j] = True

        e2e_step(0)
        e2e_step(1)
        torch.cuda.synchronize(dev)
        barrier(world)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        n_e2e = max(1, min(args.steps, 8))
        a.record(s_in)
        for i in range(n_e2e):
            e2e_step(i)
        b.record(s_out)
        torch.cuda.synchronize(dev)
        barrier(world)
        ems = max_over_ranks(a.elapsed_time(b), world) / n_e2e
        e2e = {"value": world * tokens / (ems * 1e-3), "unit": "tokens/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": ems}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        tok_s, cores, n_tok, dt = cpu_oracle_prefill(budget_s=args.cpu_budget)
        cpu = {"value": tok_s, "unit": "tokens/s", "cores": cores, "kind": "oracle",
               "sample": "all %d (batch, head) chains, first %d of %d tokens (%.1f s)"
                         % (P["B"] * P["H"], n_tok, P["T"], dt)}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": "KDA prefill B=4 T=8192 H=16 dk=dv=128 bf16 q/k/v, fp32 "
                                   "gates and state, chunk C=64 (per GPU)",
                       "global_batch": P["B"] * world, "seq_len": P["T"], "heads": P["H"],
                       "parallelism": "replicas (dp%d)" % world,
                       "l2": "inputs larger than L2 (%.0f MB read per step)" % (alg_bytes / 1e6)},
            "roofline": {"bound": "hbm", "achieved": achieved_gbs, "peak": hbm,
                         "unit": "GB/s", "frac": achieved_gbs / hbm, "traffic": traffic,
                         "peak_kind": peak_kind, "kernel_ms": kernel_ms,
                         "tensor": {"achieved_tflops": tflops, "peak_tflops": bf16_tf,
                                    "frac": tflops / bf16_tf,
                                    "peak_tflops_sustained": sustained_tflops(),
                                    "frac_sustained": tflops / sustained_tflops()}},
            "decode": dec, "varlen": var, "long": lng, "forms": forms, "backward": bwd, "e2e": e2e,
            "cpu_baseline": cpu,
            "gpu_launches": args.steps, "clocks": clk.summary(),
        }
        rank0_print(rank, line)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=60)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--decode-steps", type=int, default=1000)
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-varlen", action="store_true")
    ap.add_argument("--no-long", action="store_true")
    ap.add_argument("--long-tokens", type=int, default=0,
                    help="tokens of the long-context prefill (default: the full workload)")
    ap.add_argument("--no-forms", action="store_true")
    ap.add_argument("--no-backward", action="store_true")
    ap.add_argument("--backward-tokens", type=int, default=0,
                    help="backward over the first N tokens of each sequence (default: all)")
    ap.add_argument("--varlen-seqs", type=int, default=64,
                    help="packed sequences of the varlen workload (a smaller case for profiling)")
    ap.add_argument("--varlen-max", type=int, default=32768,
                    help="longest sequence of the varlen workload")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=12.0)
    ap.add_argument("--ref-budget", type=float, default=8.0)
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        bench_reference(args)
    else:
        bench_ours(args)


if __name__ == "__main__":
    main()
