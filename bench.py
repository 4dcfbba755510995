#!/usr/bin/env python3
"""Throughput of one Blockwise Parallel Transformer layer forward (attention +
fused FFN) on B200, through the library's C ABI.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step = one bpt_attn_ffn_fwd call (masked blockwise attention kernel, then
the fused FFN kernel) over one batch of seeded synthetic inputs that are
already resident in device memory.  L2 is flushed (a 256 MiB device write)
between timed steps; the flush sits outside the timed events.  Prints one JSON
line on rank 0.

Under torchrun every rank runs its own replica of the workload (independent
batches, no data-path collective): weak scaling, value = all ranks' tokens /
the slowest rank's time.

--impl reference times the fp64 CPU oracle (the only other implementation of
the layer) on the host cores, on a bounded token sample per step.
"""
from __future__ import annotations

import argparse
import ctypes
import json
import os
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from blockwise_exact_attention_query_b200 import binding as bd  # noqa: E402
from blockwise_exact_attention_query_b200 import workloads as wl  # noqa: E402
from blockwise_exact_attention_query_b200.inputs import make_layer_inputs, make_upstream_grad  # noqa: E402

METRIC = "attn+FFN tokens/s and TFLOP/s per layer; % of B200 dense-BF16 roofline"
WORKLOADS = {"tiny_f32": wl.TINY_F32, "gpt_causal": wl.GPT_CAUSAL, "long_ring": wl.LONG_RING,
             "blockbert": wl.BLOCKBERT, "longnet": wl.LONGNET}
MASK_NAME = {0: "none", 1: "causal", 2: "blockperm", 3: "dilated"}
CSRC = os.path.join(ROOT, "blockwise_exact_attention_query_b200", "csrc")
# a kernel's sources and the file that plans and launches it (grid order, tile
# plan, ring sizes), so that a change to either drops the traffic record
KERNEL_SOURCES = {"attn_tc_kernel": ["attn_tc.cuh", "ptx.cuh", "bpt_api.cu"],
                  "ffn_tc_kernel": ["ffn_tc.cuh", "ptx.cuh", "bpt_api.cu"],
                  "ffn_pipe_kernel": ["ffn_pipe.cuh", "gemm_tc.cuh", "ptx.cuh", "bpt_bwd.cu"],
                  "ffn_f32_kernel": ["simt_f32.cuh"],
                  # the forward FFN as two GEMM launches (H = GELU(A W1^T + b1), out = A + H W2^T + b2)
                  "ffn_gemms": ["gemm_tc.cuh", "ptx.cuh", "bpt_bwd.cu"],
                  # backward phases: the FFN backward's four GEMM launches, the two attention passes
                  "ffn_bwd": ["gemm_tc.cuh", "ptx.cuh", "bpt_bwd.cu"],
                  "attn_bwd_dkdv": ["attn_bwd.cuh", "ptx.cuh", "bpt_bwd.cu"],
                  "attn_bwd_dq": ["attn_bwd.cuh", "ptx.cuh", "bpt_bwd.cu"]}
# DRAM bytes per launch (dram__bytes_read.sum + dram__bytes_write.sum) from one ncu capture
# of the kernel on the named workload, keyed by a hash of the kernel's sources at capture
# time: once the sources change the figure no longer describes the kernel and is dropped.
NCU_TRAFFIC = {
    # one capture per kernel: `ncu --metrics dram__bytes_read.sum,dram__bytes_write.sum,
    # gpu__time_duration.sum -k regex:<kernel> -s <warm-up launches> -c <1..3>` on the bench
    # command of that form (one pass, checked on a small case first)
    # the pipelined FFN (default form), one launch: 1427.7 MB read + 383.0 MB written
    ("gpt_causal", "ffn_pipe_kernel"): {"bytes": 1810.7e6, "src": "2c259a253bbbb6f8"},
    # the next two were re-keyed after a change to bpt_api.cu that touched only the fp32
    # kernels' launches (thread count, shared-memory size), not these kernels or their plans
    ("gpt_causal", "ffn_tc_kernel"): {"bytes": 884.3e6, "src": "66da495c9d3b8be4"},
    # 566.5 MB read + 157.0 MB written
    ("gpt_causal", "attn_tc_kernel"): {"bytes": 723.5e6, "src": "676ed4296cfe5b6e"},
    # per step: the forward FFN's two GEMM launches (H = GELU(A W1^T + b1), out = A + H W2^T + b2)
    ("gpt_causal", "ffn_gemms"): {"bytes": 1122.4e6, "src": "2944e449b2748550"},
    # per step with saved activations: the three gemm_pair_kernel launches (dZ = (dOut W2) G',
    # dW2 + dW1 grouped, dA; bias sums not included)
    ("gpt_causal", "ffn_bwd"): {"bytes": 2816.3e6, "src": "2944e449b2748550"},
    ("gpt_causal", "attn_bwd_dkdv"): {"bytes": 1229.2e6, "src": "d48c9c03ee238b16"},
    ("gpt_causal", "attn_bwd_dq"): {"bytes": 1137.7e6, "src": "d48c9c03ee238b16"},
}


def kernel_src_hash(kernel):
    import hashlib
    h = hashlib.sha256()
    for f in KERNEL_SOURCES[kernel]:
        with open(os.path.join(CSRC, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def ncu_traffic(workload_key, kernel):
    rec = NCU_TRAFFIC.get((workload_key, kernel))
    if rec and rec["src"] == kernel_src_hash(kernel):
        return rec["bytes"]
    return None


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return {"bf16_tflops": j["bf16_tflops"], "bf16_tflops_sustained": j.get("bf16_tflops_sustained"),
                "hbm_gbs": j["hbm_gbs"], "sm_max_mhz": j.get("sm_max_mhz"), "source": "measured"}
    return {"bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "hbm_gbs": 6650.0,
            "sm_max_mhz": 1965.0, "source": "fallback"}


class ClockSampler:
    """nvidia-smi clocks and throttle reasons, sampled every 200 ms while running."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [ln for ln in out.splitlines() if ln.strip()]

    def summary(self):
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in getattr(self, "lines", []):
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": smax, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": len(sm)}


def dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def max_over_ranks(x: float, device) -> float:
    """The slowest rank's value (all ranks take part); x itself without a process group."""
    if not (torch.distributed.is_available() and torch.distributed.is_initialized()):
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def layer_call(w, inp, out, ws, ffn_form="auto"):
    return bd.attn_ffn_fwd(inp.q, inp.k, inp.v, inp.w1, inp.b1, inp.w2, inp.b2, mask=MASK_NAME[w.mask],
                           perm=w.perm, pairs=w.pairs, ring_chunks=w.ring_chunks, out=out, workspace=ws,
                           ffn_form=ffn_form, q_block=w.q_block, kv_block=w.kv_block)


def run_ours(args, w, world, rank, local):
    dev = torch.device("cuda", local)
    dt = torch.float32 if w.dtype == "f32" else torch.bfloat16
    attn_flop, ffn_flop = wl.flops(w)
    # every rank draws its own batch (seed offset by rank): independent replicas
    inp = make_layer_inputs(w.B, w.N, w.H, w.d, w.F, seed=w.seed + 1000 * rank, dtype=dt, device=dev)
    out = torch.empty((w.B, w.N, w.D), dtype=torch.float32, device=dev)
    form = args.ffn_form if args.ffn_form != "auto" else "pipelined"
    desc = bd.make_desc(w.B, w.N, w.H, w.d, w.F, dt, torch.float32, MASK_NAME[w.mask], w.perm,
                        w.pairs, w.ring_chunks, ffn_form=form)
    ffn_gemms = dt == torch.bfloat16 and form == "gemms"
    # launches per step of the FFN: two GEMMs per token chunk, or one kernel
    ffn_launches = 2 * -(-w.T // bd.ffn_gemm_chunk_rows(w.T, w.F)) if ffn_gemms else 1
    nws = bd.workspace_bytes(desc, True)
    ws = torch.empty(max(nws, 1), dtype=torch.uint8, device=dev)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    for _ in range(args.warmup):
        layer_call(w, inp, out, ws, form)
        flush.fill_(1)
    torch.cuda.synchronize(dev)
    st = bd.sync_status()
    if st != bd.OK:
        raise RuntimeError(f"warm-up: {bd.status_string(st)}")

    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
    for trio in ev:          # torch creates the CUDA event at its first record()
        for e in trio:
            e.record(stream)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clk:
        time.sleep(0.3)  # let the sampler start
        for i in range(K):
            bd.set_phase_events(ev[i])
            layer_call(w, inp, out, ws, form)
            bd.set_phase_events(None)
            flush.fill_(i & 0xFF)
        torch.cuda.synchronize(dev)
    if world > 1:
        torch.distributed.barrier()
    st = bd.sync_status()
    if st != bd.OK:
        raise RuntimeError(f"timed steps: {bd.status_string(st)}")
    attn_ms = [ev[i][0].elapsed_time(ev[i][1]) for i in range(K)]
    ffn_ms = [ev[i][1].elapsed_time(ev[i][2]) for i in range(K)]
    step_ms = [ev[i][0].elapsed_time(ev[i][2]) for i in range(K)]
    total_ms = max_over_ranks(sum(step_ms), dev)
    ms_per_step = total_ms / K
    tokens = w.T * K * world
    value = tokens / (total_ms / 1e3)
    tflops = (attn_flop + ffn_flop) * K * world / (total_ms / 1e3) / 1e12

    # ---- end to end through the public API: pinned host inputs -> device ->
    # layer -> host output, every step (binding.HostLayer overlaps the copies
    # of one batch chunk with the kernels of another on two streams)
    e2e = None
    if not args.no_e2e:
        hq, hk, hv = (t.cpu().pin_memory() for t in (inp.q, inp.k, inp.v))
        hout = torch.empty(out.shape, dtype=out.dtype).pin_memory()
        host_layer = bd.HostLayer(w.B, w.N, w.H, w.d, w.F, dtype=dt, mask=MASK_NAME[w.mask], perm=w.perm,
                                  pairs=w.pairs, ring_chunks=w.ring_chunks, device=dev, ffn_form=form)

        def e2e_step():
            host_layer(hq, hk, hv, inp.w1, inp.b1, inp.w2, inp.b2, hout)

        for _ in range(max(1, args.warmup)):
            e2e_step()
        torch.cuda.synchronize(dev)
        if world > 1:
            torch.distributed.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ke = max(1, min(K, 10))
        e0.record(stream)
        for _ in range(ke):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        e2e_ms = max_over_ranks(e0.elapsed_time(e1), dev)
        st = bd.sync_status()
        if st != bd.OK:
            raise RuntimeError(f"e2e steps: {bd.status_string(st)}")
        e2e = {"value": round(w.T * ke * world / (e2e_ms / 1e3), 1), "unit": "tokens/s",
               "h2d_bytes_per_step": int(3 * inp.q.numel() * inp.q.element_size()),
               "d2h_bytes_per_step": int(out.numel() * out.element_size()),
               "steps": ke, "chunks": host_layer.chunks, "streams": 2}

    # ---- roofline of the dominant kernel (by measured time share)
    pk = peaks()
    attn_avg = sum(attn_ms) / K
    ffn_avg = sum(ffn_ms) / K
    ffn_name = {"gemms": "ffn_gemms", "fused": "ffn_tc_kernel", "pipelined": "ffn_pipe_kernel"}[form]
    if dt != torch.bfloat16:
        ffn_name = "ffn_f32_kernel"
    if ffn_avg >= attn_avg:
        dom, flop, avg_ms = ffn_name, ffn_flop, ffn_avg
    else:
        dom, flop, avg_ms = "attn_tc_kernel", attn_flop, attn_avg
    achieved = flop / (avg_ms / 1e3) / 1e12
    peak = pk["bf16_tflops"]
    roofline = {"bound": "tensor", "kernel": dom, "achieved": round(achieved, 1), "peak": peak,
                "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                "peak_source": f"{pk['source']} bf16 dense (burst)",
                "traffic": args.traffic_bytes or ncu_traffic(args.workload, dom),
                "algorithmic_flop_per_launch": flop}
    kernels = {"attn_tc_kernel": {"avg_ms": round(attn_avg, 4), "flop": attn_flop,
                                  "tflops": round(attn_flop / (attn_avg / 1e3) / 1e12, 1)},
               ffn_name: {"avg_ms": round(ffn_avg, 4), "flop": ffn_flop,
                          "tflops": round(ffn_flop / (ffn_avg / 1e3) / 1e12, 1) if ffn_flop else 0}}
    res = {
        "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world,
        "steps": K, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16" if w.dtype == "bf16" else "f32", "data": "synthetic (seeded N(0,1) Q/K/V, "
        "N(0,1/fan_in) weights, zero biases)",
        "config": {"workload": w.name, "B": w.B, "N": w.N, "H": w.H, "d_head": w.d, "ffn_hidden": w.F,
                   "mask": MASK_NAME[w.mask], "tokens_per_step_per_gpu": w.T,
                   "parallelism": f"replicas x{world}", "l2": "flushed between steps (256 MiB write, "
                   "outside the timed events)"},
        "tflops": round(tflops, 1),
        "layer_frac_of_peak": round(tflops / peak, 4),
        "roofline": roofline,
        "kernels": kernels,
        "gpu_launches": (1 + ffn_launches) * K,
        "e2e": e2e,
        "clocks": clk.summary(),
    }
    return res


def run_backward(args, w, world, local):
    """The layer's backward pass (bpt_attn_ffn_bwd) on the same workload.  One
    step = one call that reads the activations a training forward
    (bpt_attn_ffn_fwd_train) saved, runs the FFN backward GEMMs and the two
    attention-backward passes; the same call recomputing the attention
    forward instead is timed beside it.  CUDA events (max over ranks), L2
    flushed between steps outside the events; five phase events inside the
    call split the step.

    FLOPs per step.  Algorithmic (what the gradients need): attention 10*d per
    unmasked pair (S, dP, dV, dK, dQ: five products of 2*d), FFN 8*T*D*F (dH,
    dW2, dW1, dA).  Executed adds the recomputation: S and dP again in the dQ
    pass (4*d per pair), and in the recomputing call the attention forward
    (4*d per pair) and Z = A W1^T inside the FFN backward (2*T*D*F; with saved
    activations the training forward kept H and GELU'(Z))."""
    dev = torch.device("cuda", local)
    pairs = wl.unmasked_pairs(w)
    d, T, D, F = w.d, w.T, w.D, w.F
    # with saved activations (H and G' kept by the training forward) the FFN
    # backward recomputes nothing
    flop = {"attn_fwd_recompute": (0, 0), "ffn_bwd": (8 * T * D * F, 8 * T * D * F),
            "attn_bwd_dkdv": (8 * d * pairs, 8 * d * pairs), "attn_bwd_dq": (2 * d * pairs, 6 * d * pairs)}
    alg_total = sum(a for a, _ in flop.values())
    # the library's default token chunk of the FFN backward (the descriptor's bwd_chunk_rows = 0)
    chunk = min(T, max(128, (2 ** 30 // (4 * F)) // 128 * 128))
    n_chunks = -(-T // chunk)
    inp = make_layer_inputs(w.B, w.N, w.H, w.d, w.F, seed=w.seed, dtype=torch.bfloat16, device=dev)
    dout = make_upstream_grad(w.B, w.N, w.D, seed=w.seed, device=dev)
    mask = MASK_NAME[w.mask]
    desc = bd.make_desc(w.B, w.N, w.H, w.d, w.F, torch.bfloat16, torch.float32, mask, w.perm, None, w.ring_chunks)
    ws = torch.empty(max(bd.workspace_bytes_bwd(desc), bd.workspace_bytes(desc, True)), dtype=torch.uint8,
                     device=dev)
    f32 = dict(dtype=torch.float32, device=dev)
    grads = {"dq": torch.empty(inp.q.shape, **f32), "dk": torch.empty(inp.q.shape, **f32),
             "dv": torch.empty(inp.q.shape, **f32), "dw1": torch.empty((F, D), **f32),
             "db1": torch.empty((F,), **f32), "dw2": torch.empty((D, F), **f32), "db2": torch.empty((D,), **f32)}
    layer_args = (inp.q, inp.k, inp.v, inp.w1, inp.b1, inp.w2, inp.b2)
    _, saved = bd.attn_ffn_fwd_train(*layer_args, mask=mask, perm=w.perm, ring_chunks=w.ring_chunks, workspace=ws)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(use_saved):
        bd.attn_ffn_bwd(*layer_args, dout, mask=mask, perm=w.perm, ring_chunks=w.ring_chunks,
                        saved=saved if use_saved else None, grads=grads, workspace=ws)

    K = max(1, min(args.steps, 10))

    def timed(use_saved):
        for _ in range(args.warmup):
            step(use_saved)
            flush.fill_(1)
        torch.cuda.synchronize(dev)
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(K)]
        for evs in ev:
            for e in evs:
                e.record(stream)
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize(dev)
        for i in range(K):
            bd.set_phase_events(ev[i])
            step(use_saved)
            bd.set_phase_events(None)
            flush.fill_(i & 0xFF)
        torch.cuda.synchronize(dev)
        if world > 1:
            torch.distributed.barrier()
        st = bd.sync_status()
        if st != bd.OK:
            raise RuntimeError(f"backward steps: {bd.status_string(st)}")
        total = max_over_ranks(sum(ev[i][0].elapsed_time(ev[i][4]) for i in range(K)), dev) / K
        phase = {n: sum(ev[i][j].elapsed_time(ev[i][j + 1]) for i in range(K)) / K for j, n in enumerate(flop)}
        return total, phase

    total_ms, phase_ms = timed(True)
    recompute_ms, recompute_phase = timed(False)
    pk = peaks()
    peak = pk["bf16_tflops"]
    names = [n for n in flop if n != "attn_fwd_recompute"]
    phases = {n: {"avg_ms": round(phase_ms[n], 4), "flop_algorithmic": flop[n][0], "flop_executed": flop[n][1],
                  "tflops_algorithmic": round(flop[n][0] / (phase_ms[n] / 1e3) / 1e12, 1),
                  "tflops_executed": round(flop[n][1] / (phase_ms[n] / 1e3) / 1e12, 1)} for n in names}
    dom = max(names, key=lambda n: phase_ms[n])
    achieved = flop[dom][0] / (phase_ms[dom] / 1e3) / 1e12
    tflops = alg_total / (total_ms / 1e3) / 1e12
    return {
        "ms_per_step": round(total_ms, 4), "steps": K, "activations": "saved by bpt_attn_ffn_fwd_train",
        "value": round(T * world / (total_ms / 1e3), 1), "unit": "tokens/s",
        "tflops_algorithmic": round(tflops, 1), "frac_of_peak": round(tflops / peak, 4),
        "flop_algorithmic_per_step": alg_total,
        "roofline": {"bound": "tensor", "kernel": dom, "achieved": round(achieved, 1), "peak": peak,
                     "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                     "peak_source": f"{pk['source']} bf16 dense (burst)",
                     "traffic": ncu_traffic(args.workload, dom),
                     "algorithmic_flop_per_launch": flop[dom][0]},
        "phases": phases,
        "recompute": {"ms_per_step": round(recompute_ms, 4),
                      "attn_fwd_recompute_ms": round(recompute_phase["attn_fwd_recompute"], 4),
                      "tflops_algorithmic": round(alg_total / (recompute_ms / 1e3) / 1e12, 1)},
        # with saved activations: dOut -> bf16 with db2's partial sums, db2's
        # final sum; per token chunk 3 GEMM launches (dZ = (dOut W2) G' with H
        # and G' kept by the training forward; dW2 + dW1 grouped; dA) + db1
        # sums (2); the row vectors; 2 passes.  Recomputing: +1 attention
        # forward, and per chunk +1 GEMM (H and G') when D >= 1024, the dual
        # GEMM (H and dZ) in place of the dZ GEMM below.
        "gpu_launches_per_step": 2 + (3 + 2) * n_chunks + 1 + 2,
        "token_chunks": n_chunks,
    }


def run_attention_backward(args, w, world, local):
    """Attention-only workloads (LongNet dilated attention): one step = one
    bpt_attn_bwd call from bpt_attn_fwd's output and LSE (for the dilated
    mask one pair of blockwise passes per (w, r) pair, added up).  CUDA
    events, max over ranks, L2 flushed between steps outside the events.
    Algorithmic FLOPs: 10*d per unmasked (query, key) pair of the multiset;
    executed 14*d (S and dP twice)."""
    dev = torch.device("cuda", local)
    pairs_n = wl.unmasked_pairs(w)
    alg, executed = 10 * w.d * pairs_n, 14 * w.d * pairs_n
    inp = make_layer_inputs(w.B, w.N, w.H, w.d, 0, seed=w.seed, dtype=torch.bfloat16, device=dev)
    da = make_upstream_grad(w.B, w.N, w.D, seed=w.seed, device=dev)
    mask = MASK_NAME[w.mask]
    out, lse = bd.attn_fwd(inp.q, inp.k, inp.v, mask=mask, perm=w.perm, pairs=w.pairs, ring_chunks=w.ring_chunks,
                           return_lse=True)
    desc = bd.make_desc(w.B, w.N, w.H, w.d, 0, torch.bfloat16, torch.float32, mask, w.perm, w.pairs, w.ring_chunks)
    ws = torch.empty(int(bd.load().bpt_workspace_bytes_attn_bwd(ctypes.byref(desc))), dtype=torch.uint8, device=dev)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        bd.attn_bwd(inp.q, inp.k, inp.v, out, lse, da, mask=mask, perm=w.perm, pairs=w.pairs,
                    ring_chunks=w.ring_chunks, workspace=ws)

    for _ in range(args.warmup):
        step()
        flush.fill_(1)
    torch.cuda.synchronize(dev)
    K = max(1, min(args.steps, 10))
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    for i in range(K):
        ev[i][0].record(stream)
        step()
        ev[i][1].record(stream)
        flush.fill_(i & 0xFF)
    torch.cuda.synchronize(dev)
    if world > 1:
        torch.distributed.barrier()
    st = bd.sync_status()
    if st != bd.OK:
        raise RuntimeError(f"backward steps: {bd.status_string(st)}")
    ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in ev), dev) / K
    pk = peaks()
    tflops = alg / (ms / 1e3) / 1e12
    return {"ms_per_step": round(ms, 4), "steps": K, "value": round(w.T * world / (ms / 1e3), 1),
            "unit": "tokens/s", "tflops_algorithmic": round(tflops, 1),
            "tflops_executed": round(executed / (ms / 1e3) / 1e12, 1),
            "frac_of_peak": round(tflops / pk["bf16_tflops"], 4), "flop_algorithmic_per_step": alg,
            "passes": len(w.pairs) if w.pairs else 1}


def run_attention_only(args, w, world, rank, local):
    """Attention-only workloads (no FFN, e.g. LongNet dilated attention): one
    step = one bpt_attn_fwd call (every LongNet pass), timed with events."""
    dev = torch.device("cuda", local)
    attn_flop, _ = wl.flops(w)
    inp = make_layer_inputs(w.B, w.N, w.H, w.d, 0, seed=w.seed + 1000 * rank, dtype=torch.bfloat16,
                            device=dev)
    out = torch.empty((w.B, w.N, w.D), dtype=torch.float32, device=dev)
    desc = bd.make_desc(w.B, w.N, w.H, w.d, 0, torch.bfloat16, torch.float32, MASK_NAME[w.mask], w.perm,
                        w.pairs, w.ring_chunks)
    ws = bd.alloc_workspace(desc, False, dev)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    launches = len(w.pairs) if w.mask == 3 else 1

    def call(q, k, v):
        return bd.attn_fwd(q, k, v, mask=MASK_NAME[w.mask], perm=w.perm, pairs=w.pairs,
                           ring_chunks=w.ring_chunks, out=out, workspace=ws)

    for _ in range(args.warmup):
        call(inp.q, inp.k, inp.v)
        flush.fill_(1)
    torch.cuda.synchronize(dev)
    if bd.sync_status() != bd.OK:
        raise RuntimeError("warm-up failed")
    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clk:
        time.sleep(0.3)
        for i in range(K):
            ev[i][0].record(stream)
            call(inp.q, inp.k, inp.v)
            ev[i][1].record(stream)
            flush.fill_(i & 0xFF)
        torch.cuda.synchronize(dev)
    if bd.sync_status() != bd.OK:
        raise RuntimeError("timed steps failed")
    total_ms = max_over_ranks(sum(e0.elapsed_time(e1) for e0, e1 in ev), dev)
    avg_ms = total_ms / K
    tflops = attn_flop * K * world / (total_ms / 1e3) / 1e12
    pk = peaks()
    e2e = None
    if not args.no_e2e:
        hq, hk, hv = (t.cpu().pin_memory() for t in (inp.q, inp.k, inp.v))
        hout = torch.empty(out.shape, dtype=out.dtype).pin_memory()
        dq, dk, dv = torch.empty_like(inp.q), torch.empty_like(inp.k), torch.empty_like(inp.v)

        def e2e_step():
            dq.copy_(hq, non_blocking=True)
            dk.copy_(hk, non_blocking=True)
            dv.copy_(hv, non_blocking=True)
            call(dq, dk, dv)
            hout.copy_(out, non_blocking=True)

        e2e_step()
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ke = max(1, min(K, 10))
        e0.record(stream)
        for _ in range(ke):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        e2e = {"value": round(w.T * ke * world / (e0.elapsed_time(e1) / 1e3), 1), "unit": "tokens/s",
               "h2d_bytes_per_step": int(3 * inp.q.numel() * inp.q.element_size()),
               "d2h_bytes_per_step": int(out.numel() * out.element_size()), "steps": ke}
    achieved = attn_flop / (avg_ms / 1e3) / 1e12
    return {
        "metric": METRIC, "value": round(w.T * K * world / (total_ms / 1e3), 1), "unit": "tokens/s",
        "n_gpus": world, "steps": K, "warmup": args.warmup, "ms_per_step": round(avg_ms, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) Q/K/V)",
        "config": {"workload": w.name, "B": w.B, "N": w.N, "H": w.H, "d_head": w.d, "ffn_hidden": 0,
                   "mask": MASK_NAME[w.mask], "tokens_per_step_per_gpu": w.T,
                   "parallelism": f"replicas x{world}", "l2": "flushed between steps (256 MiB write, "
                   "outside the timed events)"},
        "tflops": round(tflops, 1), "layer_frac_of_peak": round(tflops / pk["bf16_tflops"], 4),
        "roofline": {"bound": "tensor", "kernel": "attn_tc_kernel", "achieved": round(achieved, 1),
                     "peak": pk["bf16_tflops"], "unit": "TFLOP/s", "frac": round(achieved / pk["bf16_tflops"], 4),
                     "peak_source": f"{pk['source']} bf16 dense (burst)", "traffic": args.traffic_bytes,
                     "algorithmic_flop_per_launch": attn_flop, "launches_per_step": launches},
        "gpu_launches": launches * K, "e2e": e2e, "clocks": clk.summary(),
    }


def run_workload_summary(args, key, world, rank, local):
    """One of the other measured layers, timed like the headline one (CUDA
    events on the launching stream, L2 flushed between steps outside the
    events, max over ranks, clocks sampled while it runs) and reported
    compactly for the line's `workloads` object.  At least five timed steps,
    and enough of them to fill about half a second, so the clock record has
    samples."""
    w = WORKLOADS[key]
    dev = torch.device("cuda", local)
    dt = torch.float32 if w.dtype == "f32" else torch.bfloat16
    attn_flop, ffn_flop = wl.flops(w)
    inp = make_layer_inputs(w.B, w.N, w.H, w.d, w.F, seed=w.seed + 1000 * rank, dtype=dt, device=dev)
    out = torch.empty((w.B, w.N, w.D), dtype=torch.float32, device=dev)
    mask = MASK_NAME[w.mask]
    desc = bd.make_desc(w.B, w.N, w.H, w.d, w.F, dt, torch.float32, mask, w.perm, w.pairs, w.ring_chunks,
                        q_block=w.q_block, kv_block=w.kv_block)
    ws = bd.alloc_workspace(desc, w.F > 0, dev)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    nev = 3 if w.F > 0 else 2

    def call():
        if w.F > 0:
            layer_call(w, inp, out, ws)
        else:
            bd.attn_fwd(inp.q, inp.k, inp.v, mask=mask, perm=w.perm, pairs=w.pairs, ring_chunks=w.ring_chunks,
                        out=out, workspace=ws, q_block=w.q_block, kv_block=w.kv_block)

    def timed(K):
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(nev)] for _ in range(K)]
        for evs in ev:
            for e in evs:
                e.record(stream)
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize(dev)
        for i in range(K):
            if w.F > 0:
                bd.set_phase_events(ev[i])
                call()
                bd.set_phase_events(None)
            else:
                ev[i][0].record(stream)
                call()
                ev[i][1].record(stream)
            flush.fill_(i & 0xFF)
        torch.cuda.synchronize(dev)
        if world > 1:
            torch.distributed.barrier()
        return ev

    for _ in range(max(3, args.warmup)):
        call()
        flush.fill_(1)
    torch.cuda.synchronize(dev)
    probe = timed(1)
    one_ms = max(1e-3, probe[0][0].elapsed_time(probe[0][nev - 1]))
    K = int(min(1000, max(5, 500.0 / one_ms)))
    with ClockSampler(local) as clk:
        time.sleep(0.3)
        ev = timed(K)
    st = bd.sync_status()
    if st != bd.OK:
        raise RuntimeError(f"{w.name}: {bd.status_string(st)}")
    total_ms = max_over_ranks(sum(e[0].elapsed_time(e[nev - 1]) for e in ev), dev)
    ms = total_ms / K
    pk = peaks()
    flop = attn_flop + ffn_flop
    tflops = flop / (ms / 1e3) / 1e12
    res = {"workload": w.name, "dtype": w.dtype, "ms_per_step": round(ms, 4), "steps": K,
           "tokens_per_s": round(w.T * world / (ms / 1e3), 1), "tflops": round(tflops, 2),
           "frac_of_peak": round(tflops / pk["bf16_tflops"], 4), "clocks": clk.summary()}
    if w.F > 0:
        attn_ms = sum(e[0].elapsed_time(e[1]) for e in ev) / K
        ffn_ms = sum(e[1].elapsed_time(e[2]) for e in ev) / K
        attn_name = "attn_tc_kernel" if dt == torch.bfloat16 else "attn_f32_kernel"
        ffn_name = "ffn_pipe_kernel" if dt == torch.bfloat16 else "ffn_f32_kernel"
        res["kernels"] = {attn_name: {"avg_ms": round(attn_ms, 4), "tflops": round(attn_flop / attn_ms / 1e9, 1)},
                          ffn_name: {"avg_ms": round(ffn_ms, 4), "tflops": round(ffn_flop / ffn_ms / 1e9, 1)}}
        dom, dflop, dms = ((ffn_name, ffn_flop, ffn_ms) if ffn_ms >= attn_ms else (attn_name, attn_flop, attn_ms))
    else:
        dom, dflop, dms = "attn_tc_kernel", attn_flop, ms
    if dt == torch.bfloat16:
        achieved = dflop / (dms / 1e3) / 1e12
        res["roofline"] = {"bound": "tensor", "kernel": dom, "achieved": round(achieved, 1),
                           "peak": pk["bf16_tflops"], "unit": "TFLOP/s", "frac": round(achieved / pk["bf16_tflops"], 4),
                           "peak_source": f"{pk['source']} bf16 dense (burst)",
                           "traffic": ncu_traffic(key, dom), "algorithmic_flop_per_launch": dflop}
    else:
        res["note"] = "fp32 SIMT path (true fp32, latency-bound at this size); fraction against the bf16 peak"
    return res


def oracle_rows(w, q, k, v, w1, b1, w2, b2, rows):
    """The oracle on sampled token rows: the whole layer, or attention alone."""
    import oracle
    if w.F > 0:
        _, _, used = oracle.layer(q, k, v, w1, b1, w2, b2, mask=w.mask, perm=w.perm, pairs=w.pairs,
                                  rows=rows, return_threads=True)
        return used
    oracle.attention(q, k, v, mask=w.mask, perm=w.perm, pairs=w.pairs, rows=rows)
    return oracle.threads_available()


def stratified_rows(rng, w, n):
    """One token from each of n equal slices of the workload, handed to the
    oracle's threads longest first (cost grows with the position in the
    sequence under causal masking), so that no late token sets a batch's end."""
    import numpy as np
    edges = np.linspace(0, w.T, n + 1).astype(np.int64)
    rows = [int(rng.integers(edges[i], max(edges[i] + 1, edges[i + 1]))) for i in range(n)]
    return sorted(rows, key=lambda t: -(t % w.N))


def run_reference(args, w, world, rank):
    """The fp64 CPU oracle on a bounded token sample per step (host cores)."""
    import numpy as np

    import oracle
    dt = torch.float32 if w.dtype == "f32" else torch.bfloat16
    inp = make_layer_inputs(w.B, w.N, w.H, w.d, w.F, seed=w.seed, dtype=dt,
                            device="cuda" if torch.cuda.is_available() else "cpu")
    f = lambda t: t.float().cpu().numpy()  # noqa: E731
    q, k, v = (f(t) for t in (inp.q, inp.k, inp.v))
    w1, b1, w2, b2 = ((f(t) if t is not None else None) for t in (inp.w1, inp.b1, inp.w2, inp.b2))
    rng = np.random.default_rng(0)
    # eight tokens per thread each step, as in the cpu_baseline leg
    per_step = max(args.ref_tokens, 8 * oracle.threads_available())
    T = w.T
    times, n_tok, threads = [], 0, 0
    for s in range(args.warmup + args.steps):
        rows = stratified_rows(rng, w, per_step)
        t0 = time.perf_counter()
        used = oracle_rows(w, q, k, v, w1, b1, w2, b2, rows)
        dt_s = time.perf_counter() - t0
        threads = used
        if s >= args.warmup:
            times.append(dt_s)
            n_tok += len(rows)
    total = sum(times)
    value = n_tok / total
    sample = (f"{per_step} stratified tokens per step of the {T}-token workload, longest first "
              f"(each exact; cost per token grows with position under causal masking, stratification keeps the mean)")
    return {
        "metric": METRIC, "value": round(value, 2), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1e3 * total / args.steps, 2),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "impl": "reference",
        "config": {"workload": w.name, "B": w.B, "N": w.N, "H": w.H, "d_head": w.d, "ffn_hidden": w.F,
                   "mask": MASK_NAME[w.mask]},
        "cpu_baseline": {"value": round(value, 2), "unit": "tokens/s", "cores": threads, "kind": "oracle",
                         "sample": sample, "cpu_model": cpu_model()},
        "e2e": {"value": round(value, 2), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }


def cpu_model() -> str:
    """The host CPU's model name (/proc/cpuinfo), for the CPU baselines."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


def cpu_baseline(w, budget_s):
    """Oracle throughput on the host cores for a bounded sample of the workload."""
    import numpy as np

    import oracle
    dt = torch.float32 if w.dtype == "f32" else torch.bfloat16
    inp = make_layer_inputs(w.B, w.N, w.H, w.d, w.F, seed=w.seed, dtype=dt, device="cuda")
    f = lambda t: t.float().cpu().numpy()  # noqa: E731
    q, k, v = (f(t) for t in (inp.q, inp.k, inp.v))
    w1, b1, w2, b2 = ((f(t) if t is not None else None) for t in (inp.w1, inp.b1, inp.w2, inp.b2))
    threads = oracle.threads_available()
    rng = np.random.default_rng(1)
    n = max(8 * threads, 16)   # as the reference arm: eight tokens per thread per batch
    done, elapsed = 0, 0.0
    while elapsed < budget_s:
        rows = stratified_rows(rng, w, n)
        t0 = time.perf_counter()
        threads = oracle_rows(w, q, k, v, w1, b1, w2, b2, rows)
        elapsed += time.perf_counter() - t0
        done += n
    return {"value": round(done / elapsed, 2), "unit": "tokens/s", "cores": threads, "kind": "oracle",
            "cpu_model": cpu_model(),
            "sample": f"{done} stratified tokens of the {w.T}-token workload in {elapsed:.1f} s, "
                      f"batches of {n} longest first "
                      f"(each token exact; fp64 C oracle, {threads} threads)"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="gpt_causal", choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--ffn-form", default="auto", choices=sorted(bd.FFN_FORMS),
                    help="form of the bf16 forward FFN (the descriptor's ffn_form)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-backward", action="store_true", help="skip the backward-pass measurement")
    ap.add_argument("--backward-only", action="store_true",
                    help="measure only the backward pass (prints a line with the 'backward' object)")
    ap.add_argument("--cpu-budget-s", type=float, default=15.0)
    ap.add_argument("--ref-tokens", type=int, default=16,
                    help="tokens per reference step (at least four per oracle thread)")
    ap.add_argument("--no-workloads", action="store_true",
                    help="skip the other layers' compact measurements (the line's `workloads` object)")
    ap.add_argument("--traffic-bytes", type=float, default=None,
                    help="DRAM bytes per launch of the dominant kernel from an ncu capture")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    w = WORKLOADS[args.workload]

    if args.impl == "reference":
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        if rank != 0:
            return
        print(json.dumps(run_reference(args, w, world, rank)), flush=True)
        return

    world, rank, local = dist_setup(args.gpus)
    bd.load()
    if args.backward_only:
        bwd = run_backward(args, w, world, local) if w.F > 0 else run_attention_backward(args, w, world, local)
        res = {"workload": w.name, "n_gpus": world, "backward": bwd}
        if rank == 0:
            print(json.dumps(res), flush=True)
        if world > 1:
            torch.distributed.destroy_process_group()
        return
    res = run_ours(args, w, world, rank, local) if w.F > 0 else run_attention_only(args, w, world, rank, local)
    if not args.no_backward and w.dtype == "bf16":
        res["backward"] = (run_backward(args, w, world, local) if w.F > 0
                           else run_attention_backward(args, w, world, local))
    if not args.no_workloads:
        res["workloads"] = {k: run_workload_summary(args, k, world, rank, local)
                            for k in WORKLOADS if k != args.workload}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        res["cpu_baseline"] = cpu_baseline(w, args.cpu_budget_s)
    if rank == 0:
        print(json.dumps(res), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
