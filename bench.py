#!/usr/bin/env python
"""Benchmark: PKM layer forward tokens/s on B200, with the roofline fraction.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step is one pkm_forward over one batch of the 1024^2-slot workload (B = 16384
tokens, d_model = 1024, H = 4, dq = 512, n = 1024, k = 32, v = 1024, bf16 inputs,
fp32 scores and accumulation) with every input resident in HBM. L2 is flushed (a
256 MiB write) before every timed step, outside the step's CUDA-event bracket.
Under torchrun each rank runs the same workload on its own GPU with no collective
on the data path (weak scaling); the reported time is the max over ranks.

Rank 0 prints one JSON line. Besides the throughput it carries the roofline of the
dominant kernel (stage times come from CUDA events the library records between its
launches on the launching stream), the whole-step roofline, an end-to-end figure
through the same call with host buffers, the oracle timed on this host's cores, the
SM clocks sampled during the timed loop, and sub-objects for the 512^2 forward
(c512), the value backward and the full backward on its picks (backward,
backward_full), a training step with BatchNorm on batch statistics (train), the
small-batch latency on the 1024^2 layer (small_batch) and the wide layer (wide).

    python bench.py --part NAME          # one sub-object alone (for profiling)
    python bench.py --tokens B           # the main workload on its first B tokens
    python bench.py --part latency --tokens B   # B-token calls through the default
                                                # choice only (for profiling)

``--impl reference`` times the fp64 CPU oracle instead (a bounded sample of the
same workload per step) and prints the same metric with "impl": "reference".
"""
from __future__ import annotations

import argparse
import ctypes
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "PKM forward tokens/sec at 512² and 1024² slots (H=4,k=32); % of roofline"
UNIT = "tokens/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
FLUSH_BYTES = 256 << 20

# DRAM bytes (read + write) of one launch of the dominant kernel, from an ncu capture,
# keyed by (kernel_sha(), workload, tokens); reported as null once the kernel's source
# has changed since the capture.
TRAFFIC = {
    # c1024 at 4096 tokens: dram read 956.5 MB + write 7.8 MB, scaled x4 to the
    # 16384-token launch (the gather's traffic grows with the tokens). Captured at
    # source hash ab6394527d8d2580; the file's header comment changed since, not the
    # kernel.
    ("418f99fd39fed721", "c1024", 16384): 3.857e9,
}


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def workload_desc(w) -> str:
    return ("%s: B=%d tokens, d_model=%d, H=%d, dq=%d, n=%d (%d slots), k=%d, v=%d, %s"
            % (w.name, w.B, w.d_model, w.H, w.dq, w.n, w.n * w.n, w.k, w.v, w.dtype))


def per_token_bytes(w):
    """Algorithmic HBM bytes per token of the select+gather kernel: the H*k gathered
    value rows, the per-half lists read, the out row and idx/weight/score written."""
    esz = 2 if w.dtype == "bf16" else 4
    return w.H * w.k * w.v * esz + w.v * 4 + w.H * 2 * w.k * 8 + w.H * w.k * 12


def small_call_bytes(w, B):
    """Compulsory HBM bytes of one small-batch forward call of B tokens: W_q and the
    sub-keys read once, x in, the B*H*k value rows, out, indices and weights out."""
    esz = 2 if w.dtype == "bf16" else 4
    return (w.H * w.dq * w.d_model * esz + w.H * 2 * w.n * (w.dq // 2) * esz
            + B * w.d_model * esz + B * w.H * w.k * w.v * esz + B * w.v * 4
            + B * w.H * w.k * 8)


def gemm_flops_per_token(w):
    """Query projection + per-half scoring, as the method defines them."""
    return 2 * w.d_model * w.H * w.dq + 2 * w.H * 2 * w.n * (w.dq // 2)


def max_over_ranks(x: float, world: int, device) -> float:
    """Largest value of x over all ranks (the slowest rank sets a step's time)."""
    if world <= 1:
        return float(x)
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# --------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.proc = None
        self.path = None
        try:
            props = torch.cuda.get_device_properties(device_index)
            uuid = str(getattr(props, "uuid", "") or "")
            sel = ("GPU-" + uuid) if uuid and not uuid.startswith("GPU-") else uuid
            if not sel:
                vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
                sel = vis.split(",")[device_index] if vis else str(device_index)
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.out = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", sel, "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=self.out, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.out.close()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        smax = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i] == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": reasons, "samples": len(rows)}


# ---------------------------------------------------------------- CPU oracle
def time_oracle(w, L, budget_s: float, max_tokens: int, chunk: int = 256):
    """Oracle forward on consecutive chunks of the workload's tokens until the time
    budget or max_tokens is reached. Returns (tokens/s, tokens, seconds, threads)."""
    import oracle
    threads = os.cpu_count() or 1
    done, spent = 0, 0.0
    while done < max_tokens and spent < budget_s:
        m = min(chunk, max_tokens - done)
        Ls = dict(L)
        Ls["x"] = L["x"][done:done + m]
        t0 = time.perf_counter()
        oracle.forward(Ls, w.H, w.dq, w.n, w.k, threads=threads)
        spent += time.perf_counter() - t0
        done += m
    return done / spent, done, spent, threads


# ---------------------------------------------------------------- reference
def run_reference(args, rank, world):
    if rank != 0:
        return
    import oracle  # noqa: F401  (builds the oracle library on first use)
    w = synth.WORKLOADS[args.workload]
    L = synth.make_layer(w)
    # Size each step's sample so the whole run stays within about two minutes.
    rate, _, _, threads = time_oracle(w, L, budget_s=2.0, max_tokens=min(w.B, 512), chunk=128)
    per_step = max(64, min(w.B, int(rate * 120.0 / max(1, args.steps + args.warmup))))
    per_step = (per_step // 64) * 64
    times = []
    for s in range(args.warmup + args.steps):
        r, toks, sec, threads = time_oracle(w, L, budget_s=1e9, max_tokens=per_step,
                                            chunk=per_step)
        if s >= args.warmup:
            times.append(sec)
    mean = statistics.mean(times)
    value = per_step / mean
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": mean * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded, shapes of the pages' setups)",
        "config": {"workload": workload_desc(w), "sample_tokens_per_step": per_step,
                   "parallelism": "host cores, rank 0 only"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": "first %d of the %d tokens per step" % (per_step, w.B)},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------- our arm
def kernel_sha() -> str:
    """Hash of the gather kernel's source (its file and the selection header)."""
    h = hashlib.sha256()
    for name in ("pkm_select_gather.cu", "pkm_select.cuh"):
        with open(os.path.join(ROOT, "product_key_memory_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def run_ours(args, rank, world, local_rank):
    import torch.distributed as dist
    import product_key_memory_b200 as P

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    w = synth.WORKLOADS[args.workload]
    L = synth.make_layer(w)
    if args.tokens is not None:
        if not 1 <= args.tokens <= w.B:
            raise SystemExit("--tokens must be in [1, %d]" % w.B)
        w = w.with_tokens(args.tokens)
        L["x"] = L["x"][:args.tokens].contiguous()
    d = {k: v.to(dev) for k, v in L.items()}
    B = w.B
    out = torch.empty(B, w.v, dtype=torch.float32, device=dev)
    idx = torch.empty(B, w.H, w.k, dtype=torch.int32, device=dev)
    wts = torch.empty(B, w.H, w.k, dtype=torch.float32, device=dev)
    scs = torch.empty(B, w.H, w.k, dtype=torch.float32, device=dev)
    shape = P.make_shape(B, w.d_model, w.H, w.dq, w.n, w.k, w.v, w.torch_dtype)
    ws = P.alloc_workspace(shape, False, dev)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def fwd(x=None):
        P.pkm_forward(d["x"] if x is None else x, d["W_q"], d["bn_mean"], d["bn_var"],
                      d["bn_gamma"], d["bn_beta"], d["subkeys"], d["values"], k=w.k, out=out,
                      indices=idx, weights=wts, scores=scs, workspace=ws)

    def barrier():
        if world > 1:
            dist.barrier()

    for s in range(args.warmup):
        flush.fill_(s & 0xff)
        fwd()
    if P.pkm_device_status(ws) != 0:
        raise RuntimeError("device status after warm-up: %s" % P.pkm_status_string(-5))
    P.pkm_trace_enable(True)
    P.pkm_trace_read(0)
    P.pkm_trace_read(1)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    sampler = ClockSampler(local_rank) if rank == 0 else None
    barrier()
    torch.cuda.synchronize(dev)
    for s in range(args.steps):
        flush.fill_((s + 1) & 0xff)
        ev[s][0].record(stream)
        fwd()
        ev[s][1].record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    clocks = sampler.stop() if sampler else None
    stage_ms, calls, launches = P.pkm_trace_read(0)
    P.pkm_trace_enable(False)
    step_ms = [a.elapsed_time(b) for a, b in ev]
    total_ms = max_over_ranks(sum(step_ms), world, dev)
    if P.pkm_device_status(ws) != 0:
        raise RuntimeError("device status after timing: %s" % P.pkm_status_string(-5))
    value = world * args.steps * B / (total_ms / 1e3)
    distinct = int(P.pkm_slot_usage(idx, w.n).item())
    usage = {"distinct_slots": distinct, "slots": w.n * w.n, "fraction": distinct / (w.n * w.n),
             "picks": B * w.H * w.k}
    ms_per_step = total_ms / args.steps

    pk, pk_kind = peaks()
    hbm = float(pk["hbm_gbs"])
    bf16 = float(pk["bf16_tflops"])
    stage_avg = [m / max(1, calls) for m in stage_ms[:3]]
    call_avg = stage_ms[3] / max(1, calls)
    names = ["query_network", "subkey_scores_topk", "select_softmax_gather"]
    dom = max(range(3), key=lambda i: stage_avg[i])
    F = w.H * w.dq
    if dom == 2:
        alg = per_token_bytes(w) * B
        achieved = alg / (stage_avg[2] * 1e-3) / 1e9
        sha = kernel_sha()
        tr = TRAFFIC.get((sha, w.name, B))
        roof = {"kernel": names[2], "bound": "hbm", "achieved": achieved, "peak": hbm,
                "unit": "GB/s", "frac": achieved / hbm, "traffic": tr,
                "algorithmic_bytes_per_launch": alg, "ms_per_launch": stage_avg[2],
                "peak_kind": pk_kind}
    else:
        fl = (2 * B * w.d_model * F) if dom == 0 else (2 * B * w.H * 2 * w.n * (w.dq // 2))
        achieved = fl / (stage_avg[dom] * 1e-3) / 1e12
        roof = {"kernel": names[dom], "bound": "tensor", "achieved": achieved, "peak": bf16,
                "unit": "TFLOP/s", "frac": achieved / bf16, "traffic": None,
                "algorithmic_flops_per_launch": fl, "ms_per_launch": stage_avg[dom],
                "peak_kind": pk_kind}
    t_mem = w.H * w.k * w.v * (2 if w.dtype == "bf16" else 4) * B / (hbm * 1e9)
    t_gemm = gemm_flops_per_token(w) * B / (bf16 * 1e12)
    t_roof_ms = max(t_mem, t_gemm) * 1e3
    # Compulsory I/O besides the gathered rows: x in, W_q and the sub-keys, out,
    # indices and weights out.
    esz = 2 if w.dtype == "bf16" else 4
    secondary = (B * w.d_model * esz + F * w.d_model * esz + w.H * w.n * w.dq * esz
                 + B * w.v * 4 + B * w.H * w.k * 8)
    step_roof = {"t_roof_ms": t_roof_ms, "t_step_ms": ms_per_step, "frac": t_roof_ms / ms_per_step,
                 "secondary_io_bytes": secondary,
                 "secondary_io_share": secondary / (w.H * w.k * w.v * esz * B),
                 "bound": "hbm" if t_mem >= t_gemm else "tensor",
                 "stage_ms": dict(zip(names, stage_avg)), "call_ms": call_avg,
                 "peak_kind": pk_kind}

    # ---- end to end through pkm_forward with host buffers, pipelined like a serving
    # loop: step i+1's input copy (pinned host -> device) and step i-1's result read
    # (device -> pinned host) overlap step i's forward on three streams, with device
    # tensors double-buffered. The result read back is `out`; indices and weights stay
    # on the device for the backward.
    x_h = L["x"].pin_memory()
    out_h = [torch.empty(out.shape, dtype=out.dtype).pin_memory() for _ in range(2)]
    x_d = [torch.empty_like(d["x"]) for _ in range(2)]
    out_d = [out, torch.empty_like(out)]
    idx_d = [idx, torch.empty_like(idx)]
    w_d = [wts, torch.empty_like(wts)]
    s_in, s_cmp, s_out = (torch.cuda.Stream(dev) for _ in range(3))

    def e2e_run(steps):
        ev_in = [torch.cuda.Event() for _ in range(steps)]
        ev_cmp = [torch.cuda.Event() for _ in range(steps)]
        ev_out = [torch.cuda.Event() for _ in range(steps)]
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(s_in)
        for i in range(steps):
            b = i & 1
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(ev_cmp[i - 2])      # x_d[b] no longer read
                x_d[b].copy_(x_h, non_blocking=True)
                ev_in[i].record(s_in)
            with torch.cuda.stream(s_cmp):
                s_cmp.wait_event(ev_in[i])
                if i >= 2:
                    s_cmp.wait_event(ev_out[i - 2])     # out_d[b] already read back
                P.pkm_forward(x_d[b], d["W_q"], d["bn_mean"], d["bn_var"], d["bn_gamma"],
                              d["bn_beta"], d["subkeys"], d["values"], k=w.k, out=out_d[b],
                              indices=idx_d[b], weights=w_d[b], want_scores=False,
                              workspace=ws, stream=s_cmp)
                ev_cmp[i].record(s_cmp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_cmp[i])
                out_h[b].copy_(out_d[b], non_blocking=True)
                ev_out[i].record(s_out)
        t1.record(s_out)
        torch.cuda.synchronize(dev)
        return t0.elapsed_time(t1)

    e2e_run(3)
    barrier()
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks(e2e_run(args.steps), world, dev)
    e2e = {"value": world * args.steps * B / (e2e_ms / 1e3), "unit": UNIT,
           "h2d_bytes_per_step": x_h.numel() * x_h.element_size(),
           "d2h_bytes_per_step": out_h[0].numel() * out_h[0].element_size(),
           "ms_per_step": e2e_ms / args.steps,
           "pipelining": "copy-in, forward and copy-out of consecutive steps overlap"}
    launches_e2e = P.pkm_trace_read(0)[2]

    extra = {}
    if not args.no_extras:
        del d, x_d
        torch.cuda.empty_cache()
        extra = run_c512_and_backward(args, dev, P, hbm, bf16, stream, world, barrier)

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": w.dtype,
        "data": "synthetic (seeded; shapes and distributions of the pages' 1024^2-slot setup)",
        "config": {"workload": workload_desc(w), "global_batch": B * world,
                   "seq_len": None, "parallelism": "dp%d (independent replicas)" % world,
                   "l2": "flushed before every timed step (256 MiB write, outside the bracket)"},
        "roofline": roof, "step_roofline": step_roof, "e2e": e2e, "slot_usage": usage,
        # Keys scored per (token, head): the product search scores both codebooks
        # (2n) and the pruned candidate pairs, the flat search every one of n^2 keys.
        "search_cost": {"product": 2 * w.n + pruned_pairs(w.k), "flat": w.n * w.n,
                        "flat_over_product": w.n * w.n / (2 * w.n + pruned_pairs(w.k))},
        "gpu_launches": launches, "gpu_launches_e2e": launches_e2e,
        "clocks": clocks,
    }
    line.update(extra)
    if rank == 0 and world == 1 and not args.no_extras:
        budget = float(os.environ.get("PKM_CPU_BASELINE_S", "15"))
        rate, toks, sec, threads = time_oracle(w, L, budget_s=budget, max_tokens=B)
        line["cpu_baseline"] = {"value": rate, "unit": UNIT, "cores": threads, "kind": "oracle",
                                "sample": "first %d of the %d tokens (%.1f s)" % (toks, B, sec)}
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_c512_and_backward(args, dev, P, hbm, bf16, stream, world, barrier,
                          parts=("c512", "backward", "backward_full", "train", "latency",
                                 "wide")):
    """512^2-slot forward (the metric's other memory size), the value backward and the
    full backward on its picks, and the wide 1024^2-slot layer (H = 8, v = 1600).
    `parts` selects the measurements (the c512 forward always runs: it makes the
    picks)."""
    w = synth.WORKLOADS["c512"]
    L = synth.make_layer(w)
    d = {k: v.to(dev) for k, v in L.items()}
    B = w.B
    out = torch.empty(B, w.v, dtype=torch.float32, device=dev)
    idx = torch.empty(B, w.H, w.k, dtype=torch.int32, device=dev)
    wts = torch.empty(B, w.H, w.k, dtype=torch.float32, device=dev)
    shape = P.make_shape(B, w.d_model, w.H, w.dq, w.n, w.k, w.v, w.torch_dtype)
    ws = P.alloc_workspace(shape, False, dev)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def fwd():
        # Reads the current bindings of d, w, out, idx, wts and ws in this function.
        P.pkm_forward(d["x"], d["W_q"], d["bn_mean"], d["bn_var"], d["bn_gamma"], d["bn_beta"],
                      d["subkeys"], d["values"], k=w.k, out=out, indices=idx, weights=wts,
                      want_scores=False, workspace=ws)

    def timed(fn, steps):
        ms = []
        for s in range(steps):
            flush.fill_(s & 0xff)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            ms.append((a, b))
        torch.cuda.synchronize(dev)
        return sum(a.elapsed_time(b) for a, b in ms) / steps

    for _ in range(max(3, args.warmup)):
        fwd()
    barrier()
    P.pkm_trace_enable(True)
    P.pkm_trace_read(0)
    fwd_ms = timed(fwd, args.steps)
    stage_ms, calls, _ = P.pkm_trace_read(0)
    t_roof = max(w.H * w.k * w.v * 2 * B / (hbm * 1e9), gemm_flops_per_token(w) * B / (bf16 * 1e12))
    res = {}
    if "c512" in parts:
        res["c512"] = {"workload": workload_desc(w), "value": world * B / (fwd_ms / 1e3),
                       "unit": UNIT, "ms_per_step": fwd_ms,
                       "step_roofline_frac": t_roof * 1e3 / fwd_ms,
                       "stage_ms": [m / max(1, calls) for m in stage_ms[:3]]}

    # Backward on the c512 picks: grad_out ~ N(0, 1) bf16 [4096][1024].
    gout = synth.make_grad_out(w).to(dev)
    gv = torch.zeros(w.n * w.n, w.v, dtype=torch.float32, device=dev)
    gs = torch.empty(B, w.H, w.k, dtype=torch.float32, device=dev)
    bshape = P.make_shape(B, 0, w.H, 0, w.n, w.k, w.v, w.torch_dtype)
    bws = P.alloc_workspace(bshape, True, dev)

    def bwd():
        P.pkm_backward_values(d["values"], idx, wts, gout, gv, gs, w.n, workspace=bws)

    uniq = int(torch.unique(idx).numel())
    picks = idx.numel()
    bytes_alg = picks * w.v * 2 + B * w.v * 2 + picks * 8 + 2 * uniq * w.v * 4
    if "backward" in parts:
        for _ in range(max(3, args.warmup)):
            bwd()
        P.pkm_trace_read(1)
        bwd_ms = timed(bwd, args.steps)
        bstage, bcalls, _ = P.pkm_trace_read(1)
        res["backward"] = {
            "workload": "bwd512: value backward on the c512 picks, grad_out bf16 [4096][1024]",
            "value": world * B / (bwd_ms / 1e3), "unit": UNIT, "ms_per_step": bwd_ms,
            "unique_rows": uniq, "picks": picks,
            "algorithmic_bytes": bytes_alg, "achieved_gbs": bytes_alg / (bwd_ms * 1e-3) / 1e9,
            "frac_of_hbm": bytes_alg / (bwd_ms * 1e-3) / 1e9 / hbm,
            "stage_ms": [m / max(1, bcalls) for m in bstage[:2]]}
        # The same call on skewed picks: every pick from 40 of the 262,144 slots (about
        # 13,000 picks per touched row), the case a per-pick atomic scatter serialises on.
        hidx, hw = synth.random_selection(B, w.H, w.k, w.n * w.n, seed=77, hot_rows=40)
        hidx, hw = hidx.to(dev), hw.to(dev)

        def bwd_hot():
            P.pkm_backward_values(d["values"], hidx, hw, gout, gv, gs, w.n, workspace=bws)

        for _ in range(max(3, args.warmup)):
            bwd_hot()
        hot_ms = timed(bwd_hot, args.steps)
        res["backward"]["skewed"] = {
            "picks_from_slots": 40, "ms_per_step": hot_ms,
            "value": world * B / (hot_ms / 1e3), "unit": UNIT,
            "vs_uniform": hot_ms / bwd_ms}
    P.pkm_trace_enable(False)

    # Full backward on the same picks: every gradient of the layer (x, W_q, BatchNorm
    # affine, sub-keys, values, kept scores).
    F = w.H * w.dq
    fws = torch.empty(int(P.lib().pkm_workspace_size(ctypes.byref(shape), 3)), dtype=torch.uint8,
                      device=dev)
    grads = {"x": torch.empty(B, w.d_model, device=dev), "W_q": torch.empty(F, w.d_model, device=dev),
             "bn_gamma": torch.empty(F, device=dev), "bn_beta": torch.empty(F, device=dev),
             "subkeys": torch.empty(w.H, 2, w.n, w.dq // 2, device=dev), "values": gv, "scores": gs}

    def bwd_full():
        P.pkm_backward(d["x"], d["W_q"], d["bn_mean"], d["bn_var"], d["bn_gamma"], d["bn_beta"],
                       d["subkeys"], d["values"], idx, wts, gout, grads, workspace=fws)

    if "backward_full" in parts:
        for _ in range(max(3, args.warmup)):
            bwd_full()
        full_ms = timed(bwd_full, args.steps)
        full_bytes = (bytes_alg + B * w.d_model * (2 + 4) + F * w.d_model * (2 + 4)
                      + w.H * w.n * w.dq * (2 + 4))
        full_flops = 3 * 2 * B * F * w.d_model     # x W_q^T again, dL/dx, dL/dW_q
        t_mem, t_gemm = full_bytes / (hbm * 1e9), full_flops / (bf16 * 1e12)
        res["backward_full"] = {
            "workload": "bwd512 full: every gradient of the c512 layer on its picks",
            "value": world * B / (full_ms / 1e3), "unit": UNIT, "ms_per_step": full_ms,
            "algorithmic_bytes": full_bytes, "gemm_flops": full_flops,
            "step_roofline_frac": max(t_mem, t_gemm) * 1e3 / full_ms}
    if "latency" in parts:
        res["small_batch"] = run_latency(args, dev, P, with_wide="wide" not in parts)
    if "train" in parts:
        # One training step of the layer with BatchNorm in training mode: the forward
        # on batch statistics (running statistics updated), then the full backward
        # through them.
        tws = torch.empty(int(P.lib().pkm_workspace_size(ctypes.byref(shape), 4)),
                          dtype=torch.uint8, device=dev)
        rm, rv = d["bn_mean"].clone(), d["bn_var"].clone()
        bm = torch.empty(F, device=dev)
        bv = torch.empty(F, device=dev)
        scs = torch.empty(B, w.H, w.k, dtype=torch.float32, device=dev)

        def fwd_train():
            rc = P.lib().pkm_forward_train(
                ctypes.byref(shape), P._ptr(d["x"]), P._ptr(d["W_q"]), P._ptr(rm), P._ptr(rv),
                P._ptr(d["bn_gamma"]), P._ptr(d["bn_beta"]), ctypes.c_float(0.1),
                P._ptr(d["subkeys"]), P._ptr(d["values"]), P._ptr(out), P._ptr(idx),
                P._ptr(wts), P._ptr(scs), P._ptr(bm), P._ptr(bv), P._ptr(tws), tws.numel(),
                P._stream(None))
            if rc != 0:
                raise RuntimeError("pkm_forward_train: %s" % P.pkm_status_string(rc))

        def bwd_train():
            P.pkm_backward(d["x"], d["W_q"], bm, bv, d["bn_gamma"], d["bn_beta"], d["subkeys"],
                           d["values"], idx, wts, gout, grads, workspace=fws, bn_training=True)

        def train_step():
            fwd_train()
            bwd_train()

        for _ in range(max(3, args.warmup)):
            train_step()
        ftr_ms = timed(fwd_train, args.steps)
        step_ms = timed(train_step, args.steps)
        res["train"] = {
            "workload": "c512 training step: forward on batch statistics + full backward "
                        "through them, B=4096",
            "value": world * B / (step_ms / 1e3), "unit": UNIT, "ms_per_step": step_ms,
            "forward_train_ms": ftr_ms, "backward_train_ms": step_ms - ftr_ms}
        del tws
    del d, gv, gout, bws, ws, fws, grads
    torch.cuda.empty_cache()
    if "wide" not in parts:
        return res

    # The wide layer: d_model 1600, H = 8, 1024^2 slots, v = 1600 (3.4 GB table).
    w = synth.WORKLOADS["wide"]
    L = synth.make_layer(w)
    d = {k: v.to(dev) for k, v in L.items()}
    del L
    B = w.B
    out = torch.empty(B, w.v, dtype=torch.float32, device=dev)
    idx = torch.empty(B, w.H, w.k, dtype=torch.int32, device=dev)
    wts = torch.empty(B, w.H, w.k, dtype=torch.float32, device=dev)
    shape = P.make_shape(B, w.d_model, w.H, w.dq, w.n, w.k, w.v, w.torch_dtype)
    ws = P.alloc_workspace(shape, False, dev)
    for _ in range(max(3, args.warmup)):
        fwd()
    barrier()
    P.pkm_trace_enable(True)
    P.pkm_trace_read(0)
    fwd_ms = timed(fwd, args.steps)
    stage_ms, calls, _ = P.pkm_trace_read(0)
    P.pkm_trace_enable(False)
    t_mem = w.H * w.k * w.v * 2 * B / (hbm * 1e9)
    t_gemm = gemm_flops_per_token(w) * B / (bf16 * 1e12)
    res["wide"] = {"workload": workload_desc(w), "value": world * B / (fwd_ms / 1e3),
                   "unit": UNIT, "ms_per_step": fwd_ms,
                   "step_roofline_frac": max(t_mem, t_gemm) * 1e3 / fwd_ms,
                   "stage_ms": [m / max(1, calls) for m in stage_ms[:3]],
                   "gather_gbs": per_token_bytes(w) * B / (stage_ms[2] / max(1, calls) * 1e-3) / 1e9}
    if "small_batch" in res:
        res["small_batch"].update(latency_table(args, dev, P, "wide", d, WIDE_LATENCY_B))
    return res


def pruned_pairs(k: int) -> int:
    """Candidate pairs (a, b) of the two sorted per-half lists with (a+1)(b+1) <= k."""
    return sum(k // (a + 1) for a in range(k))


# Batch sizes of the latency table: both sides of the automatic cut-off between the
# small-batch kernels and the tensor-core path (384 tokens with H = 4, 240 with H = 8).
C1024_LATENCY_B = (1, 4, 8, 16, 32, 64, 96, 128, 192, 256, 384, 448)
WIDE_LATENCY_B = (64, 128, 192, 240, 256)


def latency_table(args, dev, P, wname, d, Bs, paths=("auto", "small_fused", "small_split", "tc")):
    """Forward latency of a few tokens on the layer d (device tensors of workload
    wname), caches warm (one token touches H*k value rows). Each batch size through the
    default choice, each small-batch form forced (the single cooperative kernel
    "small_fused", the three kernels "small_split") and the large-batch tensor-core
    kernels ("tc"): the data behind the cut-offs. Two timings per entry, CUDA events
    around many calls issued back to back: "B=..": 10 calls captured in a CUDA graph,
    replayed 20 times (the device's time per call, as a serving loop that replays
    graphs sees it); "B=.. stream": 200 calls launched one by one from Python, which
    on a slow host measures the host's launch time instead."""
    w0 = synth.WORKLOADS[wname]
    res = {}
    # The GPU's clocks ramp up under load: ~0.2 s of large-batch forwards first, so the
    # first measured entry is not taken at idle clocks.
    x = d["x"].contiguous()
    t_end = time.time() + 0.2
    while time.time() < t_end:
        P.pkm_forward(x, d["W_q"], d["bn_mean"], d["bn_var"], d["bn_gamma"], d["bn_beta"],
                      d["subkeys"], d["values"], k=w0.k, want_scores=False)
        torch.cuda.synchronize(dev)
    side = torch.cuda.Stream(dev)
    for path in paths:
        for B in Bs:
            x = d["x"][:B].contiguous()
            out = torch.empty(B, w0.v, device=dev)
            idx = torch.empty(B, w0.H, w0.k, dtype=torch.int32, device=dev)
            wts = torch.empty(B, w0.H, w0.k, device=dev)
            with P.options(path=path):
                shape = P.make_shape(B, w0.d_model, w0.H, w0.dq, w0.n, w0.k, w0.v,
                                     w0.torch_dtype)
                ws = P.alloc_workspace(shape, False, dev)

                def call():
                    P.pkm_forward(x, d["W_q"], d["bn_mean"], d["bn_var"], d["bn_gamma"],
                                  d["bn_beta"], d["subkeys"], d["values"], k=w0.k, out=out,
                                  indices=idx, weights=wts, want_scores=False, workspace=ws)

                for _ in range(max(3, args.warmup) * 4):
                    call()
                torch.cuda.synchronize(dev)
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                n = 200
                a.record()
                for _ in range(n):
                    call()
                b.record()
                torch.cuda.synchronize(dev)
                stream_us = a.elapsed_time(b) / n * 1e3
                side.wait_stream(torch.cuda.current_stream(dev))
                with torch.cuda.stream(side):
                    call()
                torch.cuda.current_stream(dev).wait_stream(side)
                torch.cuda.synchronize(dev)
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g):
                    for _ in range(10):
                        call()
                g.replay()
                torch.cuda.synchronize(dev)
                a.record()
                for _ in range(20):
                    g.replay()
                b.record()
                torch.cuda.synchronize(dev)
                graph_us = a.elapsed_time(b) / 200 * 1e3
                del g
            key = ("" if wname == "c1024" else wname + " ") + "B=%d" % B
            key += "" if path == "auto" else " " + path
            res[key] = graph_us
            res[key + " stream"] = stream_us
    return res


def run_latency(args, dev, P, with_wide=False):
    """Small-batch latency on the 1024^2-slot layer (1 to 448 tokens). The wide layer's
    entries are added where that layer is built (run_c512_and_backward), or here when
    with_wide is set (the latency part run alone)."""
    w0 = synth.WORKLOADS["c1024"]
    if args.part == "latency" and args.tokens is not None:
        # One batch size through the default choice only (profiling).
        L = synth.make_layer(w0.with_(B=args.tokens))
        d = {k: v.to(dev) for k, v in L.items()}
        return latency_table(args, dev, P, "c1024", d, (args.tokens,), paths=("auto",))
    L = synth.make_layer(w0.with_(B=max(C1024_LATENCY_B)))
    d = {k: v.to(dev) for k, v in L.items()}
    res = {"workload": "c1024 layer (1024^2 slots, H=4, k=32, v=1024, bf16) and the wide "
                       "layer (d_model 1600, H=8, v=1600), B tokens per call",
           "unit": "us per call",
           "timing": "plain keys: 10 calls in a CUDA graph replayed 20 times (device time "
                     "per call); '... stream' keys: 200 calls launched one by one"}
    res.update(latency_table(args, dev, P, "c1024", d, C1024_LATENCY_B))
    # The time those bytes take at the HBM copy peak, next to the measured time.
    hbm = float(peaks()[0]["hbm_gbs"])
    res["byte_floor_us"] = {"B=%d" % B: small_call_bytes(w0, B) / (hbm * 1e3)
                            for B in (1, 64)}
    del d, L
    if with_wide:
        L = synth.make_layer(synth.WORKLOADS["wide"].with_(B=max(WIDE_LATENCY_B)))
        d = {k: v.to(dev) for k, v in L.items()}
        del L
        res.update(latency_table(args, dev, P, "wide", d, WIDE_LATENCY_B))
    return res


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="c1024", choices=sorted(synth.WORKLOADS))
    ap.add_argument("--tokens", type=int, default=None,
                    help="tokens per step instead of the workload's (the first B rows of "
                         "its seeded input; for profiling a smaller case of the same layer)")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the c512 / backward / CPU-oracle measurements")
    ap.add_argument("--part", default=None,
                    choices=["c512", "backward", "backward_full", "train", "latency", "wide"],
                    help="run only this sub-measurement and print its JSON object "
                         "(for profiling one kernel family; not a bench line)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if args.part is not None:
        import product_key_memory_b200 as P
        dev = torch.device("cuda", local_rank)
        torch.cuda.set_device(dev)
        pk, _ = peaks()
        res = run_c512_and_backward(args, dev, P, float(pk["hbm_gbs"]), float(pk["bf16_tflops"]),
                                    torch.cuda.current_stream(dev), 1, lambda: None,
                                    parts=(args.part,))
        print(json.dumps(res), flush=True)
        return
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local_rank))
    try:
        run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
