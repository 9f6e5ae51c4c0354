"""Benchmark of the sparse-MoE FFN layer forward on B200 (one process per GPU).

python bench.py --gpus N --steps K --warmup W [--impl ours|reference] [--workload NAME]

A step is one moe_layer_forward (route + permute + SwiGLU experts + shared
experts + combine) over one batch of synthetic tokens whose inputs are already
resident in HBM. The default workload is the DeepSeek-V3-shaped prefill layer
(n = 16384 tokens, d = 7168, 256 routed experts + 1 shared, sigmoid scores with
a selection bias, 8 groups of 32 keep 4, top-8, I = 2048, bf16), the largest
of the layer shapes that fits one GPU. Ranks are
independent replicas (weak scaling, no collective on the data path); the time
is the maximum over ranks of the CUDA-event time of K steps.

The reference arm (--impl reference) times the fp64 CPU oracle on the host
cores on a bounded token sample of the same workload.

--gpus N run as a plain command starts N ranks itself (torch.distributed.run,
one process per GPU); launched by torch.distributed.run it is one of them.

--ep R times the expert-parallel layer (moe_ep_layer_forward) of a group of R
ranks: the workload's tokens split evenly over the ranks, rank q owning experts
[q E/R, (q+1) E/R). With --gpus R (one process per GPU) the ranks exchange rows
over CUDA IPC peer mappings with flag barriers between the steps; as a single
process the group is emulated on one GPU, every rank's exchange buffers in its
memory and the steps of all ranks in stream order.
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
sys.path.insert(0, ROOT)

METRIC = "MoE layer tokens/s (route+permute+SwiGLU+combine) and % of roofline, 1 B200"
L2_BYTES = 126 * 1024 * 1024


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return p["hbm_gbs"], p["bf16_tflops"], p.get("bf16_tflops_sustained"), "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


def _dist():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def reduce_max(x: float, world: int, device="cpu") -> float:
    """Maximum of a per-rank scalar over all ranks (every rank gets it)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist

    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(tokens_per_rank: int, steps: int, world: int, ms_total_max: float) -> float:
    """Whole-job tokens/s: every rank processes its own batch (replicas), time = slowest rank."""
    return world * tokens_per_rank * steps / (ms_total_max / 1e3)


def layer_work(w, kept_slots, active_experts):
    """Algorithmic FLOPs and bytes of one layer forward."""
    b = 4 if w.dtype == "f32" else 2       # activations and router weight (bf16 for the FP8 experts)
    bw = 1 + 1 / 16384 if w.dtype == "fp8" else b  # expert weights: E4M3 codes plus one scale byte per 128 x 128
    d, I, E, n = w.d_model, w.moe_intermediate_size, w.n_routed, w.n
    flops = 2 * n * E * d + 6 * kept_slots * d * I + 6 * n * d * w.I_s
    bytes_ = E * d * b + active_experts * 3 * d * I * bw + 3 * d * w.I_s * bw + 2 * n * d * b
    return flops, bytes_


def _ceil(a, b):
    return -(-a // b)


def _router_splits(w, n=None):
    """Split-K factor of the two-kernel router's logits GEMM for a batch of n tokens (router_splits in
    csrc/api.cu)."""
    n = w.n if n is None else n
    if w.dtype == "f32":
        return 1
    tiles = _ceil(n, 128) * _ceil(w.n_routed, 256)
    if tiles >= 74:
        return 1
    num_kb = _ceil(w.d_model, 64)
    ld = _ceil(w.n_routed, 4) * 4
    s = max(1, min(148 // tiles, (4 << 20) // (n * ld * 4), 32, num_kb))
    return _ceil(num_kb, _ceil(num_kb, s))


def _fp8_gemm_launches(rows, groups):
    """Kernels of one FP8 expert GEMM: SM-pair tiles lay out the B scale words first."""
    if rows <= 16 * groups:
        return 1  # 32-row short tiles
    return 2 if rows // groups >= 128 else 1


def _router_launches(w, n):
    """Kernels of this library's router (route_impl in csrc/api.cu) on a batch of n tokens, with the
    histogram and scan of its expert counts."""
    bf16_act = w.dtype != "f32"
    if bf16_act and w.cap_policy == "none" and n >= 2048 and w.top_k <= 8:
        k = 4  # one-pass router, first binary64 pass over its queue, refinement, second pass
    else:
        k = 2 if _router_splits(w, n) > 1 else 1  # logits GEMM (+ sum of the split-K partials)
        k += 3 if bf16_act and w.d_model % 8 == 0 else 1  # first pass, refinement, second pass
        if w.cap_policy != "none":
            k += 2  # capacity + gates
    return k + 2  # histogram + scan


def _ffn_launches(w, rows, groups):
    """Kernels of the expert FFN over `rows` permuted rows in `groups` experts (ffn_impl / ffn_fp8)."""
    if w.dtype == "fp8":
        return 2 + 2 * _fp8_gemm_launches(rows, groups)  # quantise x and h, GEMM1, GEMM2
    return 2  # GEMM1 (SwiGLU) + GEMM2


def launches_per_step(w):
    """Kernels of this library launched by one moe_layer_forward (the choices of csrc/api.cu)."""
    n = _router_launches(w, w.n)  # the permutation reuses the histogram and scan
    n += 1 if w.dtype == "fp8" else 2  # scatter (+ row copy; the FP8 quantiser gathers the rows)
    n += _ffn_launches(w, w.n * w.top_k, w.n_routed)
    if w.n_shared:
        n += _ffn_launches(w, w.n, 1)
    n += 1  # combine
    return n


def _sources_sha():
    """Hash of the sources of the dominant kernel (the tensor-core grouped GEMM)."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "top_routing_expert_router_b200", "csrc")
    for fn in ("gemm_tc.cu", "ptx.cuh", "common.cuh"):
        with open(os.path.join(csrc, fn), "rb") as f:
            h.update(fn.encode() + f.read())
    return h.hexdigest()[:16]


def _traffic(kernel_key, workload):
    """DRAM bytes per launch from the committed ncu summary, if it matches the current sources."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            t = json.load(f)
        e = t[kernel_key][workload]
        if e.get("sources_sha") == _sources_sha():
            return e["bytes_per_launch"]
    except Exception:
        pass
    return None


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.out = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"], stdout=self.out,
                                         stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        if self.proc:
            self.proc.terminate()
            self.proc.wait(timeout=10)

    def summary(self):
        self.out.flush()
        self.out.seek(0)
        rows = [r.split(",") for r in self.out.read().strip().splitlines() if r.count(",") >= 8]
        os.unlink(self.out.name)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        sm = [float(r[1]) for r in rows if r[1].strip().replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].strip().replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if "Active" in r[5 + i] and "Not" not in r[5 + i]})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


def run_ours(args):
    import torch
    import torch.distributed as dist

    import top_routing_expert_router_b200 as moe
    from synth import workloads as W

    world, rank, local = _dist()
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta

        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local))
    w = W.get(args.workload)
    dev = W.device_inputs(w, seed=rank, device=f"cuda:{local}")
    cfg = moe.make_config(dtype=w.dtype, **w.cfg_fields())
    n = w.n
    ws = torch.empty(moe.moe_workspace_size(cfg, n), dtype=torch.uint8, device="cuda")
    y = torch.empty((n, w.d_model), dtype=dev["x"].dtype, device="cuda")
    counts = torch.empty(w.n_routed, dtype=torch.int32, device="cuda")
    diag = torch.zeros(8, dtype=torch.int32, device="cuda")
    if w.dtype == "fp8":
        mats = ("gate", "up", "down")
        scales = {k: dev["w_%s_s" % k] for k in mats}
        scales.update({"ws_" + k: dev["ws_%s_s" % k] for k in mats if "ws_%s_s" % k in dev})
        weights = moe.make_weights(dev["w_r"], dev["w_gate_q"], dev["w_up_q"], dev["w_down_q"], dev.get("ws_gate_q"),
                                   dev.get("ws_up_q"), dev.get("ws_down_q"), dev.get("bias"), scales=scales)
    else:
        weights = moe.make_weights(dev["w_r"], dev["w_gate"], dev["w_up"], dev["w_down"], dev.get("ws_gate"),
                                   dev.get("ws_up"), dev.get("ws_down"), dev.get("bias"))
    stream = torch.cuda.current_stream()
    s = stream.cuda_stream

    def step():
        moe.moe_layer_forward(cfg, n, dev["x"], weights, y, ws, counts=counts, diag=diag, stream=s)

    for _ in range(args.warmup):
        step()
    st = moe.moe_sync_status(ws, s)
    if st != moe.MOE_OK:
        raise RuntimeError(f"device status after warm-up: {moe.moe_status_string(st)}")

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    phys = os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",")
    gpu_index = phys[local] if len(phys) > local and phys[local] != "" else str(local)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    # one event after each step as well: the per-step times show the power cap taking the clocks down
    step_ev = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    with ClockSampler(gpu_index) as clk:
        barrier()
        ev0.record(stream)
        for i in range(args.steps):
            step()
            step_ev[i].record(stream)
        ev1.record(stream)
        barrier()
    ms_total = reduce_max(ev0.elapsed_time(ev1), world, "cuda")
    ms_step = ms_total / args.steps
    step_ms = [round((ev0 if i == 0 else step_ev[i - 1]).elapsed_time(step_ev[i]), 3) for i in range(args.steps)]
    value = job_throughput(n, args.steps, world, ms_total)
    clocks = clk.summary()

    # Stage times through the staged entry points (same kernels), events on the launching stream.
    nk = n * w.top_k
    idx = torch.empty((n, w.top_k), dtype=torch.int32, device="cuda")
    tw = torch.empty((n, w.top_k), dtype=torch.float32, device="cuda")
    offs = torch.empty(w.n_routed + 1, dtype=torch.int32, device="cuda")
    perm = torch.empty(nk, dtype=torch.int32, device="cuda")
    dest = torch.empty((n, w.top_k), dtype=torch.int32, device="cuda")
    xp = torch.empty((nk, w.d_model), dtype=dev["x"].dtype, device="cuda")
    eo = torch.empty((nk, w.d_model), dtype=dev["x"].dtype, device="cuda")
    stages = {
        "route": lambda: moe.moe_route(cfg, n, dev["x"], weights, idx, tw, counts, diag, ws, s),
        "permute": lambda: moe.moe_permute(cfg, n, dev["x"], idx, offs, perm, dest, xp, ws, s),
        "expert_ffn": lambda: moe.moe_expert_ffn(cfg, n, xp, offs, weights, eo, ws, s),
        "combine": lambda: moe.moe_combine(cfg, n, eo, dest, tw, dev["x"], weights, y, ws, s),
    }
    reps = max(3, min(args.steps, 20))
    stage_ms = {}
    for name, fn in stages.items():
        fn()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        a.record(stream)
        for _ in range(reps):
            fn()
        b.record(stream)
        torch.cuda.synchronize()
        stage_ms[name] = a.elapsed_time(b) / reps
    st = moe.moe_sync_status(ws, s)
    if st != moe.MOE_OK:
        raise RuntimeError(f"device status: {moe.moe_status_string(st)}")
    dg = dict(zip(moe.DIAG_FIELDS, diag.cpu().tolist()))
    cnt = counts.cpu()
    kept = int(cnt.sum())
    active = int((cnt > 0).sum())
    flops, bytes_ = layer_work(w, kept, active)

    # End to end through the public API with host buffers: every step copies its x in from pinned
    # host memory and its y out to pinned host memory. The copies run on a copy stream with two
    # device buffers of each, so step i+1's input and step i-1's output move while step i computes
    # (the pipelining a serving loop would use); every byte still crosses the bus inside the timed region.
    x_host = dev["x"].cpu().pin_memory()
    y_host = [torch.empty_like(y, device="cpu").pin_memory() for _ in range(2)]
    xbuf = [dev["x"], torch.empty_like(dev["x"])]
    ybuf = [y, torch.empty_like(y)]
    h2d, d2h = torch.cuda.Stream(), torch.cuda.Stream()  # one per direction: neither copy waits behind the other
    ev = lambda: torch.cuda.Event()
    x_ready, y_done, out_done = [ev(), ev()], [ev(), ev()], [ev(), ev()]
    e2e_steps = max(3, min(args.steps, 20))
    barrier()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    h2d.wait_event(a)
    d2h.wait_event(a)
    for i in range(e2e_steps):
        k = i % 2
        with torch.cuda.stream(h2d):
            if i >= 2:
                h2d.wait_event(y_done[k])  # step i-2 has finished reading xbuf[k]
            xbuf[k].copy_(x_host, non_blocking=True)
            x_ready[k].record(h2d)
        stream.wait_event(x_ready[k])
        if i >= 2:
            stream.wait_event(out_done[k])  # ybuf[k] of step i-2 has been copied out
        moe.moe_layer_forward(cfg, n, xbuf[k], weights, ybuf[k], ws, counts=counts, diag=diag, stream=s)
        y_done[k].record(stream)
        with torch.cuda.stream(d2h):
            d2h.wait_event(y_done[k])
            y_host[k].copy_(ybuf[k], non_blocking=True)
            out_done[k].record(d2h)
    for k in range(2):
        stream.wait_event(out_done[k])
    b.record(stream)
    barrier()
    e2e_ms = reduce_max(a.elapsed_time(b) / e2e_steps, world, "cuda")
    if not torch.equal(y_host[(e2e_steps - 1) % 2], y.cpu()):
        raise RuntimeError("end-to-end output differs from the device-resident run")
    bpe = dev["x"].element_size()

    hbm, tf_burst, tf_sust, peak_kind = _peaks()
    peak_dtype = "bf16"
    if w.dtype == "fp8":  # E4M3 contraction: the measured bf16 peak times the nominal FP8/bf16 ratio (4.5 / 2.25)
        tf_burst, tf_sust, peak_dtype = 2 * tf_burst, 2 * tf_sust if tf_sust else None, "bf16 x 2 (nominal fp8/bf16) for fp8"
    ffn_flops = 6.0 * kept * w.d_model * w.moe_intermediate_size
    achieved = ffn_flops / (stage_ms["expert_ffn"] / 1e3) / 1e12
    t_roof = max(flops / (tf_burst * 1e12), bytes_ / (hbm * 1e9))
    out = {
        "metric": METRIC,
        "value": value,
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "e4m3 x e4m3 -> f32 (bf16 activations)" if w.dtype == "fp8" else w.dtype,
        "data": "synthetic (seeded counter-based generator; Irwin-Hall normals)",
        "config": {"workload": w.name, "n_tokens": n, "d_model": w.d_model, "n_routed": w.n_routed,
                   "top_k": w.top_k, "moe_intermediate_size": w.moe_intermediate_size, "n_shared": w.n_shared,
                   "score_fn": w.score_fn, "cap_policy": w.cap_policy, "parallelism": f"replicas x{world}",
                   "l2": f"inputs larger than L2: {active} experts x {3 * w.d_model * w.moe_intermediate_size * (1 if w.dtype == 'fp8' else bpe) / 1e6:.0f} MB of weights streamed per step"},
        "roofline": {"bound": "tensor", "kernel": "moe_expert_ffn (grouped SwiGLU GEMM1 + down GEMM2)",
                     "achieved": achieved, "peak": tf_burst, "unit": "TFLOP/s", "frac": achieved / tf_burst,
                     "peak_kind": f"{peak_kind} {peak_dtype} burst", "frac_of_sustained": achieved / tf_sust if tf_sust else None,
                     "flops_per_launch": ffn_flops, "traffic": _traffic("expert_ffn", w.name)},
        "layer_roofline": {"flops": flops, "bytes": bytes_, "t_roof_ms": t_roof * 1e3,
                           "frac": t_roof * 1e3 / ms_step, "active_experts": active, "kept_slots": kept},
        "stages_ms": stage_ms,
        "step_ms": step_ms,
        "diag": dg,
        "e2e": {"value": world * n / (e2e_ms / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": n * w.d_model * bpe,
                "d2h_bytes_per_step": n * w.d_model * bpe, "ms_per_step": e2e_ms},
        "gpu_launches": launches_per_step(w) * args.steps,
        "clocks": clocks,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(w, args.cpu_sample or default_cpu_sample(w))
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(out), flush=True)


NVLINK_GBS = 770.0  # measured peer copy per direction per GPU on this kind of node (NVLink 5)


def _split(n, world):
    return [n // world + (1 if q < n % world else 0) for q in range(world)]


def ep_group_plan(n, E, k, world, rank):
    """One rank of an expert-parallel group over a batch of n tokens: its token slice, the experts it
    owns and the receive-buffer rows every rank allocates (a token holds at most min(k, E / world) of
    one owner's experts)."""
    splits = _split(n, world)
    first = sum(splits[:rank])
    Eq = E // world
    return dict(tokens=(first, first + splits[rank]), experts=(rank * Eq, (rank + 1) * Eq),
                recv_rows=max(1, n * min(k, Eq)), splits=splits)


def _ep_rank_weights(moe, w, dev, q, world):
    Eq = w.n_routed // world
    sl = slice(q * Eq, (q + 1) * Eq)
    if w.dtype == "fp8":
        mats = ("gate", "up", "down")
        scales = {k: dev["w_%s_s" % k][sl] for k in mats}
        scales.update({"ws_" + k: dev["ws_%s_s" % k] for k in mats if "ws_%s_s" % k in dev})
        return moe.make_weights(dev["w_r"], dev["w_gate_q"][sl], dev["w_up_q"][sl], dev["w_down_q"][sl],
                                dev.get("ws_gate_q"), dev.get("ws_up_q"), dev.get("ws_down_q"), dev.get("bias"),
                                scales=scales)
    return moe.make_weights(dev["w_r"], dev["w_gate"][sl], dev["w_up"][sl], dev["w_down"][sl], dev.get("ws_gate"),
                            dev.get("ws_up"), dev.get("ws_down"), dev.get("bias"))


def ep_launches_per_rank(w, n_rank, world, barriers):
    """Kernels of this library one rank launches in one moe_ep_layer_forward over its n_rank tokens
    (ep_forward in csrc/api.cu). The owned experts' row count is taken as the group's average,
    n k / world over E / world experts. With one process per GPU (barriers) the rank also launches
    the flag barrier after each of the four steps."""
    n = _router_launches(w, n_rank)  # route, histogram + scan of the counts
    n += 3  # local stable permutation: histogram + scan + scatter (no local row gather)
    n += 2  # count publish, row push
    n += _ffn_launches(w, _ceil(w.n * w.top_k, world), max(1, w.n_routed // world))
    if w.n_shared:
        n += _ffn_launches(w, n_rank, 1)
    n += 1  # combine
    if barriers:
        n += 4
    return n


def run_ep(args):
    import torch

    import top_routing_expert_router_b200 as moe
    from synth import workloads as W

    world, rank, _ = _dist()
    if world > 1:
        raise SystemExit("--ep emulates the whole group on one GPU: run it as a single process")
    R = args.ep
    torch.cuda.set_device(0)
    w = W.get(args.workload)
    dev = W.device_inputs(w, device="cuda")
    cfg = moe.make_config(dtype=w.dtype, **w.cfg_fields())
    n, d, E, k = w.n, w.d_model, w.n_routed, w.top_k
    Eq = E // R
    splits = _split(n, R)
    first = [sum(splits[:q]) for q in range(R + 1)]
    recv_rows = moe.moe_ep_recv_rows_bound(cfg, R, splits)
    x = dev["x"]
    bufs = dict(recv_x=[torch.empty((recv_rows, d), dtype=x.dtype, device="cuda") for _ in range(R)],
                recv_out=[torch.empty((recv_rows, d), dtype=x.dtype, device="cuda") for _ in range(R)],
                counts=[torch.zeros((R, E), dtype=torch.int32, device="cuda") for _ in range(R)])
    group = moe.make_ep_group(recv_rows, **bufs)
    y = torch.empty_like(x)
    idx = torch.empty((n, k), dtype=torch.int32, device="cuda")
    ranks = [dict(n=splits[q], x=x[first[q]:first[q + 1]], y=y[first[q]:first[q + 1]],
                  topk_idx=idx[first[q]:first[q + 1]], weights=_ep_rank_weights(moe, w, dev, q, R),
                  ws=torch.empty(moe.moe_ep_workspace_size(cfg, R, splits[q], recv_rows), dtype=torch.uint8,
                                 device="cuda")) for q in range(R)]
    stream = torch.cuda.current_stream()
    s = stream.cuda_stream

    def step(xin=None, yout=None):
        rs = ranks
        if xin is not None:
            rs = [dict(r, x=xin[first[q]:first[q + 1]], y=yout[first[q]:first[q + 1]]) for q, r in enumerate(ranks)]
        moe.moe_ep_layer_forward(cfg, group, 0, rs, stream=s)

    for _ in range(args.warmup):
        step()
    for r in ranks:
        st = moe.moe_sync_status(r["ws"], s)
        if st != moe.MOE_OK:
            raise RuntimeError(f"device status after warm-up: {moe.moe_status_string(st)}")
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(os.environ.get("CUDA_VISIBLE_DEVICES", "0").split(",")[0] or "0") as clk:
        torch.cuda.synchronize()
        ev0.record(stream)
        for _ in range(args.steps):
            step()
        ev1.record(stream)
        torch.cuda.synchronize()
    ms_step = ev0.elapsed_time(ev1) / args.steps
    clocks = clk.summary()

    # Exchange volume: slot rows whose expert lives on another rank cross NVLink twice (token row
    # out, expert output back); the busiest rank bounds the time.
    owner = (idx.cpu() // Eq).numpy()
    src = __import__("numpy").repeat(__import__("numpy").arange(R), splits)[:, None]
    bpe = x.element_size()
    remote = (owner != src) & (idx.cpu().numpy() >= 0)
    sent = [int(remote[first[q]:first[q + 1]].sum()) for q in range(R)]
    recvd = [int((remote & (owner == q)).sum()) for q in range(R)]
    busiest = max(max(sent), max(recvd)) * d * bpe
    nvlink_ms = 2 * busiest / (NVLINK_GBS * 1e9) * 1e3  # dispatch + combine, each one direction per rank

    # Owned-expert FFN of every rank over the rows it received (the same kernels as in the layer).
    tables = bufs["counts"][0].cpu()
    col = tables.sum(0)
    ffn_cfg = moe.make_config(dtype=w.dtype, **{**w.cfg_fields(), "n_routed": Eq, "top_k": 1, "n_shared": 0,
                                                "n_group": 1, "topk_group": 1, "score_fn": "softmax",
                                                "renormalize": False, "routed_scaling_factor": 1.0})
    ffn_ws = torch.empty(moe.moe_workspace_size(ffn_cfg, recv_rows), dtype=torch.uint8, device="cuda")
    offs = []
    for q in range(R):
        c = col[q * Eq:(q + 1) * Eq]
        offs.append(torch.cat([torch.zeros(1, dtype=torch.int64), c.cumsum(0)]).to(torch.int32).cuda())
    reps = max(3, min(args.steps, 10))
    for q in range(R):
        moe.moe_expert_ffn(ffn_cfg, recv_rows, bufs["recv_x"][q], offs[q], ranks[q]["weights"], bufs["recv_out"][q],
                           ffn_ws, s)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    a.record(stream)
    for _ in range(reps):
        for q in range(R):
            moe.moe_expert_ffn(ffn_cfg, recv_rows, bufs["recv_x"][q], offs[q], ranks[q]["weights"],
                               bufs["recv_out"][q], ffn_ws, s)
    b.record(stream)
    torch.cuda.synchronize()
    ffn_ms = a.elapsed_time(b) / reps
    if moe.moe_sync_status(ffn_ws, s) != moe.MOE_OK:
        raise RuntimeError("device status after the expert FFN")
    kept = int(col.sum())
    ffn_flops = 6.0 * kept * d * w.moe_intermediate_size

    # End to end: every step copies x in from pinned host memory and y out to pinned host memory.
    x_host = x.cpu().pin_memory()
    y_host = torch.empty_like(y, device="cpu").pin_memory()
    xd, yd = torch.empty_like(x), torch.empty_like(y)
    e2e_steps = max(3, min(args.steps, 10))
    torch.cuda.synchronize()
    a.record(stream)
    for _ in range(e2e_steps):
        xd.copy_(x_host, non_blocking=True)
        step(xd, yd)
        y_host.copy_(yd, non_blocking=True)
    b.record(stream)
    torch.cuda.synchronize()
    e2e_ms = a.elapsed_time(b) / e2e_steps
    if not torch.equal(y_host, y.cpu()):
        raise RuntimeError("end-to-end output differs from the device-resident run")

    hbm, tf_burst, tf_sust, peak_kind = _peaks()
    peak_dtype = "bf16"
    if w.dtype == "fp8":
        tf_burst, tf_sust, peak_dtype = 2 * tf_burst, 2 * tf_sust if tf_sust else None, "bf16 x 2 (nominal fp8/bf16) for fp8"
    achieved = ffn_flops / (ffn_ms / 1e3) / 1e12
    out = {
        "metric": METRIC, "value": n / (ms_step / 1e3), "unit": "tokens/s", "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "e4m3 x e4m3 -> f32 (bf16 activations)" if w.dtype == "fp8" else w.dtype,
        "data": "synthetic (seeded counter-based generator; Irwin-Hall normals)",
        "config": {"workload": w.name, "n_tokens": n, "tokens_per_rank": splits,
                   "parallelism": f"ep{R} emulated on 1 GPU (every rank's buffers local, ranks in stream order)",
                   "recv_rows": recv_rows,
                   "l2": "inputs larger than L2: every expert's weights streamed per step"},
        "roofline": {"bound": "tensor", "kernel": "owned-expert FFN of every rank (grouped SwiGLU GEMM1 + GEMM2)",
                     "achieved": achieved, "peak": tf_burst, "unit": "TFLOP/s", "frac": achieved / tf_burst,
                     "peak_kind": f"{peak_kind} {peak_dtype} burst", "flops_per_launch": ffn_flops,
                     "traffic": None},
        "exchange": {"remote_slots_sent_per_rank": sent, "remote_slots_received_per_rank": recvd,
                     "busiest_rank_bytes_each_way": busiest, "nvlink_gbs": NVLINK_GBS,
                     "projected_nvlink_ms_dispatch_plus_combine": nvlink_ms,
                     "layer_minus_ffn_ms": ms_step - ffn_ms},
        "e2e": {"value": n / (e2e_ms / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": n * d * bpe,
                "d2h_bytes_per_step": n * d * bpe, "ms_per_step": e2e_ms},
        "gpu_launches": sum(ep_launches_per_rank(w, nq, R, False) for nq in splits) * args.steps,
        "clocks": clocks,
    }
    print(json.dumps(out), flush=True)


def _expert_bytes(w):
    """Bytes of one routed expert's three matrices in the workload's dtype."""
    per = 1 if w.dtype == "fp8" else (4 if w.dtype == "f32" else 2)
    return 3 * w.d_model * w.moe_intermediate_size * per


def default_cpu_sample(w):
    """Tokens in the oracle's timed sample: 16, fewer where the experts that many tokens reach would
    need more than about 4 GB of host weights (the sample's experts are generated on the host)."""
    if w.n_routed * _expert_bytes(w) <= 4e9:
        return min(16, w.n)
    return max(1, min(16, w.n, int(4e9 // (w.top_k * _expert_bytes(w)))))


def run_ep_dist(args):
    """Expert parallelism with one process per GPU (launched by torch.distributed.run, WORLD_SIZE = R):
    rank q owns experts [q E/R, (q+1) E/R) and routes its slice of the batch; the exchange buffers are
    mapped between the processes with CUDA IPC records exchanged through the process group, and the
    library's flag barriers (bounded waits) separate the steps of each layer call."""
    from datetime import timedelta

    import torch
    import torch.distributed as dist

    import top_routing_expert_router_b200 as moe
    from synth import workloads as W

    world, rank, local = _dist()
    if world != args.ep:
        raise SystemExit(f"--ep {args.ep} with {world} processes: launch one process per rank")
    if torch.cuda.device_count() <= local:
        raise SystemExit("one GPU per rank: ranks that wait on one another must not share a GPU")
    torch.cuda.set_device(local)
    dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local))
    w = W.get(args.workload)
    dev = W.device_inputs(w, device=f"cuda:{local}")  # seed 0 on every rank: one batch, split below
    cfg = moe.make_config(dtype=w.dtype, **w.cfg_fields())
    plan = ep_group_plan(w.n, w.n_routed, w.top_k, world, rank)
    t0, t1 = plan["tokens"]
    n_mine, d, R = t1 - t0, w.d_model, world
    recv_rows = plan["recv_rows"]
    x = dev["x"][t0:t1]
    local_bufs = dict(recv_x=torch.empty((recv_rows, d), dtype=x.dtype, device="cuda"),
                      recv_out=torch.empty((recv_rows, d), dtype=x.dtype, device="cuda"),
                      counts=torch.zeros((R, w.n_routed), dtype=torch.int32, device="cuda"),
                      flags=torch.zeros(R + 1, dtype=torch.int32, device="cuda"))
    torch.cuda.synchronize()

    def gather(obj):
        out = [None] * world
        dist.all_gather_object(out, obj)
        return out

    peers = moe.ep_open_peers(local_bufs, rank, world, gather)
    group = moe.make_ep_group(recv_rows, peers["recv_x"], peers["recv_out"], peers["counts"], peers["flags"])
    y = torch.empty_like(x)
    mine = dict(n=n_mine, x=x, y=y, weights=_ep_rank_weights(moe, w, dev, rank, R),
                ws=torch.empty(moe.moe_ep_workspace_size(cfg, R, n_mine, recv_rows), dtype=torch.uint8,
                               device="cuda"))
    stream = torch.cuda.current_stream()
    s = stream.cuda_stream

    def step(xin=None, yout=None):
        r = mine if xin is None else dict(mine, x=xin, y=yout)
        moe.moe_ep_layer_forward(cfg, group, rank, [r], stream=s)

    try:
        for _ in range(args.warmup):
            step()
        st = moe.moe_sync_status(mine["ws"], s)
        if st != moe.MOE_OK:
            raise RuntimeError(f"rank {rank}: device status after warm-up: {moe.moe_status_string(st)}")
        # the split layer computes what the single-device layer computes on this rank's tokens
        full_w = _ep_rank_weights(moe, w, dev, 0, 1)
        ref = torch.empty_like(y)
        ws1 = torch.empty(moe.moe_workspace_size(cfg, n_mine), dtype=torch.uint8, device="cuda")
        moe.moe_layer_forward(cfg, n_mine, x, full_w, ref, ws1, stream=s)
        torch.cuda.synchronize()
        same = bool(torch.equal(ref.view(torch.int16), y.view(torch.int16)))
        del ws1, ref
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        phys = os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",")
        with ClockSampler(phys[local] if len(phys) > local and phys[local] != "" else str(local)) as clk:
            dist.barrier()
            torch.cuda.synchronize()
            ev0.record(stream)
            for _ in range(args.steps):
                step()
            ev1.record(stream)
            torch.cuda.synchronize()
            dist.barrier()
        ms_total = reduce_max(ev0.elapsed_time(ev1), world, "cuda")
        clocks = clk.summary()
        st = moe.moe_sync_status(mine["ws"], s)
        # end to end: this rank's token rows in from pinned host memory, its outputs back
        x_host = x.cpu().pin_memory()
        y_host = torch.empty_like(y, device="cpu").pin_memory()
        xd, yd = torch.empty_like(x), torch.empty_like(y)
        e2e_steps = max(3, min(args.steps, 10))
        dist.barrier()
        torch.cuda.synchronize()
        ev0.record(stream)
        for _ in range(e2e_steps):
            xd.copy_(x_host, non_blocking=True)
            step(xd, yd)
            y_host.copy_(yd, non_blocking=True)
        ev1.record(stream)
        torch.cuda.synchronize()
        e2e_ms = reduce_max(ev0.elapsed_time(ev1) / e2e_steps, world, "cuda")
        ok_all = gather(dict(rank=rank, status=int(st), same=same))
    finally:
        torch.cuda.synchronize()
        dist.barrier()
        for name, addrs in peers.items():
            for q, a in enumerate(addrs):
                if q != rank:
                    moe.moe_ep_close_handle(a)
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        bpe = x.element_size()
        out = {
            "metric": METRIC, "value": w.n * args.steps / (ms_total / 1e3), "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_total / args.steps,
            "higher_is_better": True, "scaling": "strong", "vs_baseline": None,
            "dtype": "e4m3 x e4m3 -> f32 (bf16 activations)" if w.dtype == "fp8" else w.dtype,
            "data": "synthetic (seeded counter-based generator; Irwin-Hall normals)",
            "config": {"workload": w.name, "n_tokens": w.n, "tokens_per_rank": plan["splits"],
                       "parallelism": f"ep{world}, one process per GPU (CUDA IPC peer buffers, flag barriers)",
                       "recv_rows": recv_rows, "l2": "inputs larger than L2: every expert's weights streamed per step"},
            "ranks": ok_all,
            "e2e": {"value": w.n / (e2e_ms / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": w.n * d * bpe,
                    "d2h_bytes_per_step": w.n * d * bpe, "ms_per_step": e2e_ms},
            "gpu_launches": sum(ep_launches_per_rank(w, nq, world, True) for nq in plan["splits"]) * args.steps,
            "clocks": clocks,
        }
        print(json.dumps(out), flush=True)


def _oracle_inputs(w, tokens):
    """Host inputs of the oracle's sample: the first `tokens` rows of x, the router, the shared
    experts, and the routed experts those tokens reach. The other routed experts' matrices are
    zero-filled arrays the oracle never reads (their pages are never touched), so the sample of a
    256-expert layer does not hold every expert in host memory."""
    import numpy as np

    from oracle import oracle as O
    from synth import workloads as W

    specs = w.tensor_specs()
    small = ["w_r"] + (["bias"] if w.bias_range else [])
    shared = ["ws_gate", "ws_up", "ws_down"] if w.n_shared else []
    routed = ["w_gate", "w_up", "w_down"]
    if w.dtype == "fp8":
        shared = [m + sfx for m in shared for sfx in ("_q", "_s")]
        routed = [m + sfx for m in routed for sfx in ("_q", "_s")]
    inp = W.host_inputs(w, names=small + shared)
    inp["x"] = W.host_rows(w, "x", range(tokens))
    idx, _, _, _ = O.route_capacity(O.Cfg(**w.cfg_fields()), O.router_logits(inp["x"], inp["w_r"]), inp.get("bias"))
    used = sorted({int(e) for e in idx.ravel() if e >= 0})
    for nm in routed:
        shape, dt = specs[nm][0], specs[nm][5]
        a = np.zeros(shape, {"u8": np.uint8, "f32": np.float32}.get(dt, np.uint16))
        if used:
            a[used] = W.host_rows(w, nm, used)
        inp[nm] = a
    return inp


def _oracle_time(w, inp, tokens):
    """Seconds the oracle layer takes on the first `tokens` rows of the sample."""
    from oracle import oracle as O

    cfg = O.Cfg(**w.cfg_fields())
    t0 = time.perf_counter()
    if w.dtype == "fp8":
        w8 = {k: (inp["w_%s_q" % k], inp["w_%s_s" % k]) for k in ("gate", "up", "down")}
        ws8 = {k: (inp["ws_%s_q" % k], inp["ws_%s_s" % k]) for k in ("gate", "up", "down")} if w.n_shared else None
        O.layer_fp8(cfg, inp["x"][:tokens], inp["w_r"], inp.get("bias"), w8, ws8)
    else:
        O.layer(cfg, inp["x"][:tokens], inp["w_r"], inp["w_gate"], inp["w_up"], inp["w_down"], inp.get("bias"),
                inp.get("ws_gate"), inp.get("ws_up"), inp.get("ws_down"))
    return time.perf_counter() - t0


def _cores():
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count()


CPU_BASELINE_MIN_S = 10.0   # CPU work the baseline's figure rests on
CPU_BASELINE_MAX_PASSES = 20


def cpu_baseline(w, tokens):
    """The oracle layer timed on the first `tokens` tokens of the workload (a bounded sample whose
    experts fit in host memory), in passes over that same sample until about 10 s of CPU work have
    been timed (at most 20 passes)."""
    inp = _oracle_inputs(w, tokens)
    secs = []
    while sum(secs) < CPU_BASELINE_MIN_S and len(secs) < CPU_BASELINE_MAX_PASSES:
        secs.append(_oracle_time(w, inp, tokens))
    total = sum(secs)
    return {"value": tokens * len(secs) / total, "unit": "tokens/s",
            "cores": int(os.environ.get("OMP_NUM_THREADS", _cores())), "kind": "oracle",
            "sample": f"fp64 oracle layer (routing of the sample as its own batch, experts, combine) on the first "
                      f"{tokens} tokens of {w.name}, {len(secs)} passes: {total:.1f} s"}


def run_reference(args):
    from synth import workloads as W

    world, rank, _ = _dist()
    if rank != 0:
        return
    w = W.get(args.workload)
    tokens = args.ref_sample
    inp = _oracle_inputs(w, tokens)
    for _ in range(args.warmup):
        _oracle_time(w, inp, 1)
    secs = [_oracle_time(w, inp, tokens) for _ in range(args.steps)]
    total = sum(secs)
    value = tokens * args.steps / total
    cores = int(os.environ.get("OMP_NUM_THREADS", _cores()))
    out = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": total / args.steps * 1e3,
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
           "data": "synthetic", "config": {"workload": w.name, "n_tokens_sampled_per_step": tokens},
           "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                            "sample": f"fp64 oracle layer on {tokens} tokens of {w.name} per step (inputs generated before timing)"},
           "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="deepseek_v3_prefill")
    ap.add_argument("--cpu-sample", type=int, default=0,
                    help="tokens in the oracle's timed sample (0: 16, fewer for layers whose sampled experts "
                         "would need more than about 4 GB of host weights)")
    ap.add_argument("--ref-sample", type=int, default=1, help="tokens per step of the reference (oracle) arm")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--ep", type=int, default=0, help="expert-parallel group of this many ranks, emulated on one GPU")
    ap.add_argument("--timeout", type=int, default=900, help="limit (s) of a self-launched multi-rank run")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("at least 3 warm-up steps")
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        sys.exit(launch_ranks(args.gpus, args.timeout))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if args.impl == "reference":
        run_reference(args)
    elif args.ep > 1 and world > 1:
        run_ep_dist(args)
    elif args.ep > 1:
        run_ep(args)
    else:
        run_ours(args)


def launch_ranks(n, limit_s, script=None, argv=None):
    """Run `script argv` (default: this command) as n ranks, one process per GPU, under
    torch.distributed.run on this node (rendezvous on 127.0.0.1); returns its exit status.
    `timeout -k 60` bounds the whole run."""
    import socket

    sock = socket.socket()
    sock.bind(("127.0.0.1", 0))
    port = sock.getsockname()[1]
    sock.close()
    cmd = ["timeout", "-k", "60", str(limit_s), sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
           f"--nproc-per-node={n}", "--master-addr", "127.0.0.1", "--master-port", str(port),
           script or os.path.abspath(__file__), *(sys.argv[1:] if argv is None else argv)]
    return subprocess.call(cmd)


if __name__ == "__main__":
    main()
