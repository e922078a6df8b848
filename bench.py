#!/usr/bin/env python
"""Benchmark of the Longformer attention forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload base_bf16]

One step = one forward pass of the whole attention (mask pass, global-token
gathers, the fused band + global-row tensor-core kernel and the split
combine) over one batch of the workload, inputs resident in HBM.  The timed
region is K steps between a barrier + synchronize on both sides, timed with
CUDA events on the launching stream; the max over ranks is reported.  The
inputs rotate over several buffer sets whose total exceeds the L2 cache, so
no step reads another step's inputs out of L2.

Metric: attended scores per second (and TFLOP/s at 4 * head_dim FLOP per
attended pair), whole job.  Multi-GPU (torchrun): every rank runs its own
copy of the workload (independent batches, no collective on the data path):
weak scaling.

--impl reference times the CPU oracle (oracle/, float64, OpenMP) on a
bounded sample of the same workload -- the only reference implementation
this project has (the pages publish no code to install).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from sparse_sliding_window_b200 import synth  # noqa: E402

METRIC = "attended scores/s and TFLOP/s at n=4096 w=512 bf16; % of B200 roofline"
UNIT = "scores/s"


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        j = json.load(open(path))
        return dict(hbm=float(j["hbm_gbs"]), bf16=float(j["bf16_tflops"]),
                    bf16_sus=float(j.get("bf16_tflops_sustained", j["bf16_tflops"])), src="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sus=1400.0, src="fallback")


def algorithmic_bytes(wl, mask) -> int:
    """Bytes one forward must move at least, per sequence b and head:
    Q_s, K_s, V_s read at the valid rows (mask != 0; a padding row is never
    a query nor a key), Q_g read at the global rows, K_g and V_g read at the
    valid rows only when the sequence has a global token (nothing else reads
    them), O (every row, zeros at padding) and the fp32 log-normaliser
    written, and the int32 mask read once."""
    eb = 4 if wl.dtype == "f32" else 2
    row = wl.head_dim * eb
    total = mask.size * 4
    for b in range(mask.shape[0]):
        nvalid = int((mask[b] != 0).sum())
        ng = int((mask[b] == 2).sum())
        per_head = 3 * nvalid * row + ng * row + (2 * nvalid * row if ng else 0)
        per_head += wl.n * row + wl.n * 4
        total += wl.H * per_head
    return total


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 200 ms."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, dev_uuid=None):
        self.proc = None
        self.out = None
        self.uuid = dev_uuid

    def start(self):
        try:
            cmd = ["nvidia-smi", "--query-gpu=" + self.Q, "--format=csv,noheader,nounits", "-lms", "200"]
            if self.uuid:
                cmd += ["-i", self.uuid]
            self.out = open(os.path.join("/tmp", "lf_clocks_%d.csv" % os.getpid()), "w+")
            self.proc = subprocess.Popen(cmd, stdout=self.out, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.out.seek(0)
        rows = [l.strip().split(",") for l in self.out if l.strip()]
        self.out.close()
        try:
            os.remove(self.out.name)
        except OSError:
            pass
        sm, mx, reasons, pw = [], [], set(), []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            try:
                sm.append(float(r[1]))
                mx.append(float(r[2]))
                pw.append(float(r[3]))
                for k, nm in enumerate(names):
                    if r[5 + k].strip().lower() == "active":
                        reasons.add(nm)
            except (ValueError, IndexError):
                continue
        if not sm:
            return None
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": float(max(mx)),
                "power_w_max": float(max(pw)) if pw else None, "reasons": sorted(reasons),
                "samples": len(sm), "window": "warm-up and timed region"}


def max_over_ranks(value: float, world: int, device=None) -> float:
    """The largest of the per-rank values (device timings are reported as the
    slowest rank).  Uses the default process group when world > 1."""
    if world <= 1:
        return float(value)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank: int, world: int, ms_per_step: float) -> float:
    """Whole-job units per second: every rank processes its own replica of
    the workload (weak scaling); the step time is the slowest rank's."""
    return units_per_rank * world / (ms_per_step * 1e-3)


# DRAM traffic of the main forward kernel per launch, from the ncu captures
# summarised under profiles/; reported only while the kernel sources are the
# ones that were profiled (their sha256 prefix), else null.
PROFILED_TRAFFIC = {"base_bf16": {"bytes": 31919872, "sha": "e3273b3afd2a8e39"}}


def kernel_traffic(workload: str):
    import hashlib
    rec = PROFILED_TRAFFIC.get(workload)
    if not rec:
        return None
    h = hashlib.sha256()
    for f in ("lf_tc.cu", "lf_ptx.cuh", "lf_common.cuh"):
        h.update(open(os.path.join(ROOT, "sparse_sliding_window_b200", "csrc", f), "rb").read())
    return rec["bytes"] if h.hexdigest()[:16] == rec["sha"] else None


def _dist():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def resolve_world(gpus: int, env=None):
    """The rank layout for ``--gpus N``.  Under a launcher (torchrun sets
    WORLD_SIZE) N must equal the world size.  Without one, N = 1 runs here
    and N > 1 returns None: the caller relaunches itself with one process
    per GPU (``launch_command``).  Returns (world, rank, local_rank)."""
    env = os.environ if env is None else env
    if gpus < 1:
        raise SystemExit("bench.py: --gpus must be >= 1 (got %d)" % gpus)
    if "WORLD_SIZE" in env:
        world = int(env["WORLD_SIZE"])
        if world != gpus:
            raise SystemExit("bench.py: --gpus %d but the launcher started %d ranks" % (gpus, world))
        return world, int(env.get("RANK", "0")), int(env.get("LOCAL_RANK", "0"))
    if gpus == 1:
        return 1, 0, 0
    return None


def launch_command(gpus: int, argv):
    """torchrun command that reruns this script with one rank per GPU (local
    rendezvous on 127.0.0.1)."""
    return [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
            "--nproc-per-node", str(gpus), "--master-addr", "127.0.0.1", "--master-port",
            str(29500 + os.getpid() % 1000), os.path.abspath(__file__)] + list(argv)


def rank_step_time(local_ms: float, world: int, device=None) -> float:
    """Cross-rank part of a timed region: every rank has timed its own K
    steps on its device; after a barrier the slowest rank's time is the
    job's step time (the same on every rank)."""
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    return max_over_ranks(local_ms, world, device)


def run_reference(args, wl):
    """The CPU oracle on a bounded sample (whole heads) of the workload."""
    ws, rank, _ = _dist()
    if rank != 0:
        return 0
    import oracle
    oracle.build()
    inp = synth.make_inputs(wl)
    f = {k: synth.as_float64(v, wl.dtype) for k, v in inp.items() if k not in ("mask", "dilation")}
    scale = 1.0 / math.sqrt(wl.head_dim)
    head = (0, 0)
    pairs = oracle.count_pairs(wl.n, wl.r, wl.dilation[0], wl.causal, inp["mask"][0])

    def step():
        b, h = head
        oracle.fwd_head(wl.r, wl.dilation[h], wl.causal, scale, inp["mask"][b], f["qs"][b, h],
                        f["ks"][b, h], f["vs"][b, h], f["qg"][b, h], f["kg"][b, h], f["vg"][b, h])

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = (time.perf_counter() - t0) / args.steps
    v = pairs / dt
    sample = "one (b,h) head of %s per step (%d of %d heads)" % (wl.name, 1, wl.B * wl.H)
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": ws,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": wl.name, "B": wl.B, "H": wl.H, "n": wl.n,
                                            "window": 2 * wl.r, "head_dim": wl.head_dim},
            "cpu_baseline": {"value": v, "unit": UNIT, "cores": oracle.threads(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def cpu_baseline(wl, budget_s=10.0):
    """The oracle as it stands, timed on the host cores over whole heads of
    the workload, cycling over them until ~budget_s seconds of work (rank 0,
    N = 1 only)."""
    import oracle
    oracle.build()
    inp = synth.make_inputs(wl)
    f = {k: synth.as_float64(v, wl.dtype) for k, v in inp.items() if k not in ("mask", "dilation")}
    scale = 1.0 / math.sqrt(wl.head_dim)
    heads = [(b, h) for b in range(wl.B) for h in range(wl.H)]
    npairs = {}
    done, pairs, t_total = 0, 0, 0.0
    while t_total < budget_s:
        b, h = heads[done % len(heads)]
        t0 = time.perf_counter()
        oracle.fwd_head(wl.r, wl.dilation[h], wl.causal, scale, inp["mask"][b], f["qs"][b, h],
                        f["ks"][b, h], f["vs"][b, h], f["qg"][b, h], f["kg"][b, h], f["vg"][b, h])
        t_total += time.perf_counter() - t0
        if (b, h) not in npairs:
            npairs[(b, h)] = oracle.count_pairs(wl.n, wl.r, wl.dilation[h], wl.causal, inp["mask"][b])
        pairs += npairs[(b, h)]
        done += 1
    return {"value": pairs / t_total, "unit": UNIT, "cores": oracle.threads(), "kind": "oracle",
            "sample": "%d head forwards (cycling over the %d (b,h) heads of %s), float64, %.1f s" % (
                done, len(heads), wl.name, t_total)}


def time_backward(att, d, wl, pairs, world, steps, warmup, dev, stream):
    """Time lf_attn_bwd (six gradients) on the forward's outputs; reported
    beside the forward metric (algorithmic 8 * head_dim FLOP per pair)."""
    import torch
    from sparse_sliding_window_b200 import lf_attn as L
    g = d.get("do")
    if g is None:
        g = torch.randn_like(d["qs"])
    if att.ws_b is None:
        att.ws_b = L.workspace(att.p, True, dev)
    grads = [torch.empty_like(d["qs"]) for _ in range(6)]

    def bstep():
        L.lf_attn_bwd(att.p, d["qs"], d["ks"], d["vs"], d["qg"], d["kg"], d["vg"], d["mask"], d["o"],
                      d["lse"], g, *grads, att.ws_b)

    for _ in range(max(3, warmup // 4)):
        bstep()
    torch.cuda.synchronize(dev)
    att.status(bwd=True)
    k = max(3, min(steps, 20))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        torch.distributed.barrier()
    e0.record(stream)
    for _ in range(k):
        bstep()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    att.status(bwd=True)
    ms = rank_step_time(e0.elapsed_time(e1) / k, world, dev)
    kinds = ("CUDA-core backward (delta, dQ, dK_s/dV_s, dK_g/dV_g)" if wl.dtype == "f32" else
             "tensor-core dQ and dK/dV band kernels + CUDA-core global-token parts")
    pk = _peaks()
    tfl = 8.0 * wl.head_dim * pairs * world / (ms * 1e-3) / 1e12
    return {"ms_per_step": ms, "steps": k, "kernels": kinds, "launch": "eager",
            "tflops_algorithmic": tfl, "tensor_frac_sustained": tfl / pk["bf16_sus"],
            "scores_per_s": pairs * world / (ms * 1e-3)}


def decode_numbers(wl, steps, warmup, dev):
    """Decode step of a causal workload: one new token per sequence against
    the full-length cache (every head), timed on the device over CUDA-graph
    replays.  HBM-bound: the window's key and value rows are read once per
    head.  Returns the numbers and the roofline."""
    import torch
    from sparse_sliding_window_b200 import lf_attn as L
    assert wl.causal, "the decode step is the causal window"
    inp = synth.make_inputs(wl, with_do=False)

    def dev_t(a):
        return _host_tensor(a, wl.dtype).to(dev)
    kc, vc = dev_t(inp["ks"]), dev_t(inp["vs"])
    q = dev_t(np.ascontiguousarray(inp["qs"][:, :, -1]))
    lens = torch.full((wl.B,), wl.n, dtype=torch.int32, device=dev)
    o = torch.empty_like(q)
    lse = torch.empty((wl.B, wl.H), dtype=torch.float32, device=dev)
    p = L.make_params(wl.B, wl.H, wl.n, wl.r, wl.dilation, True, 0.0,
                      {"bf16": L.LF_BF16, "f16": L.LF_F16, "f32": L.LF_F32}[wl.dtype])
    for _ in range(max(3, warmup)):
        L.lf_attn_decode(p, q, kc, vc, lens, o, lse)
    torch.cuda.synchronize(dev)
    # a serving loop replays the step from a CUDA graph: the host launches
    # nothing per token, so the device time per step is what is measured
    # (a per-call Python launch loop would time the host instead)
    per_graph = 32
    side = torch.cuda.Stream(dev)
    side.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(side):
        L.lf_attn_decode(p, q, kc, vc, lens, o, lse)
    torch.cuda.current_stream(dev).wait_stream(side)
    torch.cuda.synchronize(dev)
    gr = torch.cuda.CUDAGraph()
    with torch.cuda.graph(gr):
        for _ in range(per_graph):
            L.lf_attn_decode(p, q, kc, vc, lens, o, lse)
    reps = max(1, steps // per_graph)
    for _ in range(3):
        gr.replay()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        gr.replay()
    e1.record()
    torch.cuda.synchronize(dev)
    ms = e0.elapsed_time(e1) / (reps * per_graph)
    del gr
    eb = 4 if wl.dtype == "f32" else 2
    keys = sum(min(wl.r, (wl.n - 1) // d) + 1 for d in wl.dilation) * wl.B
    nbytes = keys * 2 * 64 * eb + 2 * wl.B * wl.H * 64 * eb + wl.B * wl.H * 4
    pk = _peaks()
    return {"ms_per_step": ms, "tokens_per_s": wl.B / (ms * 1e-3), "steps_timed": reps * per_graph,
            "launch": "cuda_graph",
            "roofline": {"bound": "hbm", "achieved": nbytes / (ms * 1e-3) / 1e9, "peak": pk["hbm"],
                         "unit": "GB/s", "frac": nbytes / (ms * 1e-3) / 1e9 / pk["hbm"],
                         "traffic": None, "algorithmic_bytes": nbytes,
                         "note": "CUDA-graph replay of 32 steps; a step still includes the device-side launch gap"}}


def projection_numbers(wl, steps, warmup, dev):
    """The projections around one attention layer of the workload's shape,
    each GEMM timed by CUDA events the library records around its kernel,
    with L2 flushed (a 256 MB write) before every timed call:
      in:  hidden [B, n, d_model] -> Q_s, K_s, V_s, K_g, V_g (one call, N = 5 d_model)
      qg:  Q_g at the sequence's global tokens only (row gather + GEMM)
      out: heads [B, H, n, 64] -> [B, n, d_model]
    FLOPs are 2 M N K of the rows computed."""
    import torch
    from sparse_sliding_window_b200 import lf_attn as L
    B, n, H = wl.B, wl.n, wl.H
    D = H * wl.head_dim
    tdt = torch.float16 if wl.dtype == "f16" else torch.bfloat16
    g = torch.Generator(device=dev).manual_seed(1234)

    def rnd(*shape, scale=1.0):
        return (torch.randn(*shape, device=dev, generator=g) * scale).to(tdt)

    x = rnd(B, n, D)
    w_in, b_in = rnd(5 * D, D, scale=D ** -0.5), rnd(5 * D, scale=0.1)
    w_qg, b_qg = rnd(D, D, scale=D ** -0.5), rnd(D, scale=0.1)
    w_out, b_out = rnd(D, D, scale=D ** -0.5), rnd(D, scale=0.1)
    o = rnd(B, H, n, wl.head_dim)
    outs = [torch.empty(B, H, n, wl.head_dim, device=dev, dtype=tdt) for _ in range(6)]
    y = torch.empty(B, n, D, device=dev, dtype=tdt)
    mask = torch.from_numpy(synth.build_mask(wl)).to(dev)
    ng = int((mask == 2).sum(dim=1).max().item())
    p = L.make_proj_params(B, n, H, L.LF_BF16 if wl.dtype != "f16" else L.LF_F16)
    ws = L.proj_workspace(p, max(ng, 1))
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    calls = {
        "in": (lambda: L.lf_proj_in(p, x, w_in, b_in, outs[:5], ws), 2.0 * B * n * 5 * D * D),
        "out": (lambda: L.lf_proj_out(p, o, w_out, b_out, y, ws), 2.0 * B * n * D * D),
    }
    if ng > 0:
        calls["qg"] = (lambda: L.lf_proj_in(p, x, w_qg, b_qg, outs[5:], ws, rows_mask=mask,
                                            rows_code=2, max_rows=ng),
                       2.0 * int((mask == 2).sum().item()) * D * D)
    a, c = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    c.record()
    pk = _peaks()
    res = {}
    for name, (fn, flops) in calls.items():
        for _ in range(max(3, warmup)):
            fn()
        torch.cuda.synchronize(dev)
        ts = []
        for _ in range(max(5, min(steps, 50))):
            flush.zero_()
            L.lf_proj_set_timing_events(a, c)
            fn()
            L.lf_proj_set_timing_events(None, None)
            torch.cuda.synchronize(dev)
            ts.append(a.elapsed_time(c) * 1e-3)
        L.lf_attn_status(ws)
        ts.sort()
        t = ts[len(ts) // 2]
        res[name] = {"kernel_us": t * 1e6, "tflops": flops / t * 1e-12,
                     "frac": flops / t * 1e-12 / pk["bf16"], "flops": flops}
    res["peak_tflops"] = pk["bf16"]
    res["peak_source"] = pk["src"]
    res["shape"] = {"B": B, "n": n, "d_model": D, "heads": H, "global_rows": int((mask == 2).sum().item())}
    res["timing"] = "median over calls, CUDA events around each GEMM kernel, L2 flushed before each"
    return res


def cross_numbers(steps, warmup, dev, B=2, H=16, Lq=1024, Lk=16384):
    """LED decoder cross-attention (the pages' 16K-token encoder output,
    1024 decoder positions, 16 heads, two sequences): lf_attn_cross_fwd,
    kernel by the library's CUDA events, step (setup + kernel + merge) by
    events around the call; inputs rotate over enough sets to exceed L2.
    4 * 64 FLOP per (query, key) pair."""
    import torch
    from sparse_sliding_window_b200 import lf_attn as L
    g = torch.Generator(device=dev).manual_seed(99)
    set_bytes = B * H * (Lq + 2 * Lk) * 64 * 2
    nsets = max(2, int(2 * torch.cuda.get_device_properties(dev).L2_cache_size // set_bytes) + 1)
    sets = [[torch.randn(B, H, L_, 64, device=dev, generator=g).bfloat16() for L_ in (Lq, Lk, Lk)]
            for _ in range(nsets)]
    km = torch.ones(B, Lk, dtype=torch.int32, device=dev)
    o = torch.empty(B, H, Lq, 64, device=dev, dtype=torch.bfloat16)
    lse = torch.empty(B, H, Lq, device=dev)
    p = L.make_cross_params(B, H, Lq, Lk, L.LF_BF16)
    ws = L.cross_workspace(p, device=dev)
    for i in range(max(3, warmup)):
        L.lf_attn_cross_fwd(p, *sets[i % nsets], km, o, lse, ws)
    torch.cuda.synchronize(dev)
    a, c = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    c.record()
    kt, st = [], []
    for i in range(max(5, min(steps, 30))):
        L.lf_attn_set_timing_events(a, c)
        s0.record()
        L.lf_attn_cross_fwd(p, *sets[i % nsets], km, o, lse, ws)
        s1.record()
        L.lf_attn_set_timing_events(None, None)
        torch.cuda.synchronize(dev)
        kt.append(a.elapsed_time(c) * 1e-3)
        st.append(s0.elapsed_time(s1) * 1e-3)
    L.lf_attn_status(ws)
    kt.sort()
    st.sort()
    flops = 4.0 * 64 * B * H * Lq * Lk
    pk = _peaks()
    return {"shape": {"B": B, "H": H, "Lq": Lq, "Lk": Lk}, "kernel_us": kt[len(kt) // 2] * 1e6,
            "step_us": st[len(st) // 2] * 1e6, "tflops_kernel": flops / kt[len(kt) // 2] * 1e-12,
            "tflops_step": flops / st[len(st) // 2] * 1e-12,
            "frac_kernel": flops / kt[len(kt) // 2] * 1e-12 / pk["bf16"], "peak_tflops": pk["bf16"],
            "peak_source": pk["src"], "l2": "inputs rotate over %d sets" % nsets}


def run_decode(args, wl):
    import torch
    dev = torch.device("cuda", 0)
    d = decode_numbers(wl, args.steps, args.warmup, dev)
    line = {"metric": "decode tokens/s (causal window, one new token per sequence, all heads)",
            "value": d["tokens_per_s"], "unit": "tokens/s", "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": d["ms_per_step"], "higher_is_better": True,
            "dtype": wl.dtype, "steps_timed": d["steps_timed"], "data": "synthetic",
            "config": {"workload": wl.name + " decode", "B": wl.B, "H": wl.H, "cache_len": wl.n,
                       "window_one_sided": wl.r, "dilation": wl.dilation},
            "roofline": d["roofline"]}
    print(json.dumps(line), flush=True)
    return 0


def _host_tensor(a, dtype):
    import torch
    if dtype == "bf16":
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(a))


NAMES = ["qs", "ks", "vs", "qg", "kg", "vg"]


def measure(wl, kern, steps, warmup, world, dev, stream, graph=True, e2e=False,
            min_warm_seconds=0.0, sampler=None):
    """One workload's forward on this rank: attended pairs (the library's
    pair counter), the CUDA-graph and eager step times over input sets that
    rotate through more than the L2 cache, the main kernel's time from CUDA
    events the library records around it on its stream, the roofline of
    that kernel, and optionally the end-to-end time through the public API
    with host buffers.  Timed regions end with a barrier and the max over
    ranks."""
    import torch
    from sparse_sliding_window_b200 import lf_attn as L
    inp = synth.make_inputs(wl, with_do=wl.backward)
    mask_np = inp["mask"]
    ng = int((mask_np == 2).sum(axis=1).max())
    att = L.LongformerAttention(wl.B, wl.H, wl.n, wl.r, wl.dilation, wl.causal, dtype=wl.dtype,
                                max_global=ng, kernel=kern, device=dev)
    host = {k: _host_tensor(inp[k], wl.dtype).pin_memory() for k in NAMES}
    host["mask"] = torch.from_numpy(mask_np).pin_memory()
    set_bytes = sum(host[k].numel() * host[k].element_size() for k in NAMES)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    nsets = max(2, int(math.ceil(1.5 * l2 / max(set_bytes, 1))) + 1)
    sets = []
    for s in range(nsets):
        d = {k: host[k].to(dev, non_blocking=False) for k in NAMES + ["mask"]}
        d["o"] = torch.empty_like(d["qs"])
        d["lse"] = torch.empty(d["qs"].shape[:3], dtype=torch.float32, device=dev)
        sets.append(d)
    if wl.backward:
        sets[0]["do"] = _host_tensor(inp["do"], wl.dtype).to(dev)
    torch.cuda.synchronize(dev)
    pairs = int(att.count_pairs(sets[0]["mask"]).sum().item())
    att.status()

    def step(i):
        d = sets[i % nsets]
        att.fwd(d["qs"], d["ks"], d["vs"], d["qg"], d["kg"], d["vg"], d["mask"], d["o"], d["lse"])

    if sampler is not None:
        sampler.start()
    i = 0
    t_start = time.time()
    while i < warmup or time.time() - t_start < min_warm_seconds:
        step(i)
        i += 1
        if i % 64 == 0:
            torch.cuda.synchronize(dev)
    torch.cuda.synchronize(dev)
    att.status()
    # eager steps, with the kernel events of every step
    kev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(steps)]
    for a, b in kev:  # create the CUDA events; the library re-records them
        a.record(stream)
        b.record(stream)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    launches0 = L.lf_attn_launch_count()
    e0.record(stream)
    for k in range(steps):
        L.lf_attn_set_timing_events(*kev[k])
        step(i + k)
    e1.record(stream)
    L.lf_attn_set_timing_events(None, None)
    torch.cuda.synchronize(dev)
    launches = L.lf_attn_launch_count() - launches0
    clocks = sampler.stop() if sampler is not None else None
    att.status()
    t_ms = rank_step_time(e0.elapsed_time(e1), world, dev)
    k_ms = rank_step_time(float(np.mean([a.elapsed_time(b) for a, b in kev])), world, dev)
    ms_step_eager = t_ms / steps
    ms_step = ms_step_eager
    if graph:
        # the same steps replayed from CUDA graphs (one per input set): the
        # library's launches are captured once, replays skip host launch cost
        graphs = []
        for sidx in range(nsets):
            side = torch.cuda.Stream(dev)
            side.wait_stream(stream)
            with torch.cuda.stream(side):
                step(sidx)
            stream.wait_stream(side)
            gr = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gr):
                step(sidx)
            graphs.append(gr)
        for k in range(max(3, warmup)):
            graphs[k % nsets].replay()
        torch.cuda.synchronize(dev)
        g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize(dev)
        g0.record(stream)
        for k in range(steps):
            graphs[k % nsets].replay()
        g1.record(stream)
        torch.cuda.synchronize(dev)
        ms_step = rank_step_time(g0.elapsed_time(g1), world, dev) / steps
        att.status()
        del graphs
    flops = 4.0 * wl.head_dim * pairs
    pk = _peaks()
    abytes = algorithmic_bytes(wl, mask_np)
    t_flop = flops / (pk["bf16"] * 1e12)
    t_byte = abytes / (pk["hbm"] * 1e9)
    k_s = k_ms * 1e-3
    if t_byte >= t_flop:
        roof = {"bound": "hbm", "achieved": abytes / k_s / 1e9, "peak": pk["hbm"], "unit": "GB/s"}
    else:
        roof = {"bound": "tensor", "achieved": flops / k_s / 1e12, "peak": pk["bf16"], "unit": "TFLOP/s"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["traffic"] = kernel_traffic(wl.name) if kern != 1 else None
    roof["peak_source"] = pk["src"]
    roof["kernel_ms"] = k_ms
    roof["algorithmic_bytes"] = abytes
    roof["algorithmic_flops"] = flops
    roof["tensor_view"] = {"achieved_tflops": flops / k_s / 1e12, "peak": pk["bf16"],
                           "frac": flops / k_s / 1e12 / pk["bf16"]}
    roof["step_frac"] = max(t_flop, t_byte) / (ms_step * 1e-3)
    roof["timed_on"] = "eager launches, events around the kernel on its stream"
    out = {"wl": wl, "pairs": pairs, "ng": ng, "nsets": nsets, "set_bytes": set_bytes, "l2": l2,
           "ms_step": ms_step, "ms_step_eager": ms_step_eager, "kernel_ms": k_ms,
           "launches_per_step": launches / steps, "launches": launches, "roofline": roof,
           "clocks": clocks, "scores_per_s": job_throughput(pairs, world, ms_step),
           "tflops": flops * world / (ms_step * 1e-3) / 1e12, "att": att, "sets": sets}
    if e2e:
        # end-to-end through the public API: H2D of the step's inputs from
        # pinned host memory, the forward, D2H of the output
        o_host = torch.empty(sets[0]["o"].shape, dtype=sets[0]["o"].dtype).pin_memory()
        d = sets[0]
        for _ in range(3):
            for k in NAMES + ["mask"]:
                d[k].copy_(host[k], non_blocking=True)
            att.fwd(d["qs"], d["ks"], d["vs"], d["qg"], d["kg"], d["vg"], d["mask"], d["o"], d["lse"])
            o_host.copy_(d["o"], non_blocking=True)
        torch.cuda.synchronize(dev)
        ee0, ee1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e2e_steps = max(3, min(steps, 50))
        ee0.record(stream)
        for _ in range(e2e_steps):
            for k in NAMES + ["mask"]:
                d[k].copy_(host[k], non_blocking=True)
            att.fwd(d["qs"], d["ks"], d["vs"], d["qg"], d["kg"], d["vg"], d["mask"], d["o"], d["lse"])
            o_host.copy_(d["o"], non_blocking=True)
        ee1.record(stream)
        torch.cuda.synchronize(dev)
        e2e_ms = rank_step_time(ee0.elapsed_time(ee1) / e2e_steps, world, dev)
        out["e2e"] = {"value": job_throughput(pairs, world, e2e_ms), "unit": UNIT,
                      "h2d_bytes_per_step": int(set_bytes + host["mask"].numel() * 4),
                      "d2h_bytes_per_step": int(o_host.numel() * o_host.element_size()),
                      "ms_per_step": e2e_ms}
    return out


def summary(m):
    """The per-workload numbers reported beside the headline line."""
    wl, r = m["wl"], m["roofline"]
    return {"step_ms": m["ms_step"], "step_ms_eager": m["ms_step_eager"], "kernel_ms": m["kernel_ms"],
            "scores_per_s": m["scores_per_s"], "tflops": m["tflops"],
            "attended_pairs": m["pairs"], "dtype": wl.dtype,
            "roofline": {"bound": r["bound"], "achieved": r["achieved"], "peak": r["peak"],
                         "unit": r["unit"], "frac": r["frac"], "step_frac": r["step_frac"],
                         "algorithmic_bytes": r["algorithmic_bytes"], "traffic": r["traffic"],
                         "tensor_frac": r["tensor_view"]["frac"]},
            "gpu_launches_per_step": m["launches_per_step"],
            "config": {"B": wl.B, "H": wl.H, "n": wl.n, "window": 2 * wl.r,
                       "dilation": sorted(set(wl.dilation)), "causal": wl.causal,
                       "global_tokens_per_seq": m["ng"]}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="base_bf16", choices=sorted(synth.WORKLOADS))
    ap.add_argument("--kernel", default="auto", choices=["auto", "simt", "tc"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--min-warm-seconds", type=float, default=1.0)
    ap.add_argument("--no-graph", action="store_true",
                    help="time eager launches only (default: also replay each step from a CUDA graph)")
    ap.add_argument("--decode", action="store_true",
                    help="time the causal-window decode step instead (causal workloads)")
    ap.add_argument("--bwd", action="store_true",
                    help="also time the backward (default for workloads with a backward)")
    ap.add_argument("--no-others", action="store_true",
                    help="skip the other workloads reported under 'workloads'")
    ap.add_argument("--proj", action="store_true",
                    help="time only the projection GEMMs around the layer (one JSON line)")
    ap.add_argument("--cross", action="store_true",
                    help="time only the LED decoder cross-attention (one JSON line)")
    args = ap.parse_args()
    wl = synth.WORKLOADS[args.workload]
    layout = resolve_world(args.gpus)
    if layout is None:
        # --gpus N > 1 without a launcher: one process per GPU under torchrun
        return subprocess.call(launch_command(args.gpus, sys.argv[1:]))
    if args.impl == "reference":
        return run_reference(args, wl)

    import torch
    from sparse_sliding_window_b200 import lf_attn as L

    if args.decode:
        return run_decode(args, wl)
    if args.cross:
        cr = cross_numbers(args.steps, args.warmup, torch.device("cuda", 0))
        print(json.dumps({"metric": "LED decoder cross-attention TFLOP/s (1024 queries x 16384 keys, 16 heads, B 2)",
                          "value": cr["tflops_step"], "unit": "TFLOP/s", "n_gpus": 1, "steps": args.steps,
                          "warmup": args.warmup, "ms_per_step": cr["step_us"] * 1e-3, "higher_is_better": True,
                          "dtype": "bf16", "data": "synthetic", "config": {"workload": "led decoder cross-attention"},
                          "cross_attention": cr}), flush=True)
        return 0
    if args.proj:
        pr = projection_numbers(wl, args.steps, args.warmup, torch.device("cuda", 0))
        tot_f = sum(v["flops"] for k, v in pr.items() if isinstance(v, dict) and "flops" in v)
        tot_t = sum(v["kernel_us"] for k, v in pr.items() if isinstance(v, dict) and "flops" in v)
        print(json.dumps({"metric": "projection GEMM TFLOP/s (input, global-row and output projections)",
                          "value": tot_f / tot_t * 1e-6, "unit": "TFLOP/s", "n_gpus": 1,
                          "steps": args.steps, "warmup": args.warmup, "ms_per_step": tot_t * 1e-3,
                          "higher_is_better": True, "dtype": wl.dtype, "data": "synthetic",
                          "config": {"workload": wl.name + " projections"}, "projections": pr}),
              flush=True)
        return 0
    world, rank, local = layout
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    kern = {"auto": L.LF_KERNEL_AUTO, "simt": L.LF_KERNEL_SIMT, "tc": L.LF_KERNEL_TC}[args.kernel]

    sampler = ClockSampler(getattr(torch.cuda.get_device_properties(dev), "uuid", None) and
                           "GPU-" + str(torch.cuda.get_device_properties(dev).uuid))
    m = measure(wl, kern, args.steps, args.warmup, world, dev, stream, graph=not args.no_graph,
                e2e=True, min_warm_seconds=args.min_warm_seconds, sampler=sampler)
    pairs = m["pairs"]
    line = {"metric": METRIC, "value": m["scores_per_s"], "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": m["ms_step"],
            "ms_per_step_eager": m["ms_step_eager"],
            "launch": "eager" if args.no_graph else "cuda_graph", "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": wl.dtype, "data": "synthetic",
            "config": {"workload": wl.name, "B": wl.B, "H": wl.H, "n": wl.n, "window": 2 * wl.r,
                       "head_dim": wl.head_dim, "dilation": sorted(set(wl.dilation)),
                       "causal": wl.causal, "global_tokens_per_seq": m["ng"], "kernel": args.kernel,
                       "l2": "inputs rotate over %d buffer sets (%.0f MB > L2 %.0f MB)" % (
                           m["nsets"], m["nsets"] * m["set_bytes"] / 1e6, m["l2"] / 1e6),
                       "parallelism": "replicas x%d" % world if world > 1 else "1 GPU"},
            "tflops": m["tflops"], "attended_pairs_per_step": pairs * world,
            "roofline": m["roofline"], "clocks": m["clocks"], "gpu_launches": int(m["launches"]),
            "e2e": m["e2e"]}
    if args.bwd or wl.backward:
        line["backward"] = time_backward(m["att"], m["sets"][0], wl, pairs, world, args.steps,
                                         args.warmup, dev, stream)
    del m
    if world == 1 and args.kernel != "simt":
        line["projections"] = projection_numbers(wl, args.steps, args.warmup, dev)
        line["cross_attention"] = cross_numbers(args.steps, args.warmup, dev)
    if not args.no_others and args.kernel != "simt":
        # every other workload, driver-observed beside the headline: its
        # forward step / main kernel / roofline, the backward where it has
        # one, and the decode step of the causal one
        others = {}
        ksteps, kwarm = max(3, min(args.steps, 30)), max(3, min(args.warmup, 5))
        for name in sorted(synth.WORKLOADS):
            if name == wl.name:
                continue
            owl = synth.WORKLOADS[name]
            om = measure(owl, kern, ksteps, kwarm, world, dev, stream, graph=not args.no_graph)
            entry = summary(om)
            entry["steps"] = ksteps
            if owl.backward:
                entry["backward"] = time_backward(om["att"], om["sets"][0], owl, om["pairs"], world,
                                                  ksteps, kwarm, dev, stream)
            if owl.causal:
                entry["decode"] = decode_numbers(owl, 256, 3, dev)
            others[name] = entry
            del om
            torch.cuda.empty_cache()
        line["workloads"] = others
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(wl)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
