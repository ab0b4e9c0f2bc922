#!/usr/bin/env python
"""CSA2 layer-group benchmark on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config 4] [--impl ours|reference]

A step is one pass of the layer group of the chosen workload (default: the
1M-context hierarchical decode group, F + 3 Reindex + 4 Reuse, batch 8) over
one batch of queries, with the KV cache and indexer keys resident in HBM.

Timing (ours): every layer runs after an L2 flush (a 2x-L2 write outside the
layer's event window, standing in for the FFN/MoE weights that stream between
attention layers); a step's time is the sum of its per-layer CUDA-event times.
`value` = queries of all ranks / max over ranks of that time.  Also reported:
the same group back to back without flushes ("warm"), an end-to-end number
through the public API with pinned host buffers and the copies inside the
timed region ("e2e"), the dominant kernel's roofline from live per-kernel
event timing, the SM clocks sampled during the timed region, and the CPU
oracle on a bounded sample ("cpu_baseline").

--impl reference times the float64 CPU oracle on the same workload, the GPU
arm's whole batch per step (a spread sample of 8 queries for the 4096-query
prefill), on rank 0 only.

Multi-GPU (torchrun): every rank runs its own replica of the workload; the
path has no data-path collective (sequences are independent).
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "CSA2 decode queries/s per layer group at 1M ctx; achieved HBM TB/s vs peak"
UNIT = "queries/s"
L2_BYTES = 126 * 2 ** 20
FALLBACK_HBM_GBS = 6650.0
REF_MAX_BATCH = 64        # largest batch the reference arm runs whole per step
REF_SAMPLE = 8            # queries per reference step of a larger batch (prefill)


# ---------------------------------------------------------------------------- ranks

def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def dist_init(world, backend):
    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300))


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def reduce_max(x: float, world: int, device=None) -> float:
    """Max of a float over all ranks (identity with one rank)."""
    if world == 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ---------------------------------------------------------------------------- clocks

CLOCK_FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,utilization.gpu,clocks_event_reasons.active,"
                "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
REASON_COLS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")


class ClockSampler:
    """nvidia-smi sampling every 200 ms while the timed region runs."""

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={CLOCK_FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 10:
                continue
            try:
                rows.append({"sm": float(parts[1]), "max": float(parts[2]), "util": float(parts[4]),
                             "reasons": {c: ("Not" not in parts[6 + i]) for i, c in enumerate(REASON_COLS)}})
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        load = [r for r in rows if r["util"] > 0] or rows
        reasons = sorted({c for r in load for c, on in r["reasons"].items() if on})
        return {"sm_mhz": statistics.median(r["sm"] for r in load),
                "sm_max_mhz": max(r["max"] for r in rows), "reasons": reasons,
                "samples": len(rows), "samples_under_load": len(load)}


# ---------------------------------------------------------------------------- peaks, traffic

def measured_hbm_gbs():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


def measured_tflops(launch_s):
    """Dense bf16 tensor peak: the burst figure for a launch shorter than 1 ms,
    the sustained (power-capped) one for longer launches."""
    key = "bf16_tflops_sustained" if launch_s >= 1e-3 else "bf16_tflops"
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)[key]), f"measured (MEASURED_PEAKS.json {key})"
    except (OSError, KeyError, ValueError):
        return (1400.0 if launch_s >= 1e-3 else 1590.0), "fallback (pool's earlier measurement)"


def source_digest(*names) -> str:
    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(ROOT, "kv_cache_csa2_b200", "csrc", n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:12]


# kernel kind -> (source files whose digest must match the profile, profile summary)
PROFILED_SOURCES = {
    "index_scores": (("index_scores.cu", "index_scores_tc.cu"), "profiles/index_scores_c4.md"),
    "attn": (("attn_tc.cu", "attn_common.cuh", "sm100.cuh", "common.cuh"), "profiles/attn_c4.md"),
    "topk": (("topk.cu", "topk_multi.cu", "topk_cta.cu", "topk_cluster.cu"), "profiles/topk_c4.md"),
    "index_pool": (("index_scores.cu", "index_scores_tc.cu"), "profiles/index_pool_c4.md"),
}


# the workload the committed summaries were captured on (traffic per launch
# depends on the workload's sizes)
PROFILED_WORKLOAD = "c4_hier_decode_f_3ri_4u_1m"


def ncu_traffic(kind, workload):
    """DRAM bytes per launch for `kind` from the committed ncu summary, or None
    when there is none, it was taken on another workload, or the kernel
    source changed since it was taken."""
    if kind not in PROFILED_SOURCES or workload != PROFILED_WORKLOAD:
        return None
    srcs, path = PROFILED_SOURCES[kind]
    try:
        text = open(os.path.join(ROOT, path)).read()
    except OSError:
        return None
    m = re.search(r"traffic_bytes_per_launch:\s*([0-9.eE+]+)\s+source_digest:\s*([0-9a-f]+)", text)
    if not m or m.group(2) != source_digest(*srcs):
        return None
    return float(m.group(1))


# ---------------------------------------------------------------------------- algorithmic bytes

def algorithmic_bytes(wl):
    """Bytes the method must move in one step, per kernel kind: the inputs it
    has to read and the outputs it has to write (indexer keys of the scored
    entries, gathered KV rows, q / w / out / lse / top-k / pool).  Score
    intermediates are not counted.  Returns {kind: (bytes per step, launches
    per step)}."""
    rows = wl.B * wl.Q
    qidx = rows * wl.Hi * (wl.d * 2 + 4)            # indexer q (bf16) + w (f32)
    kv_row = wl.D * 2 if not wl.kv_fp4 else wl.D // 2 + wl.D // 16
    out = {}
    n_sel = sum(1 for m in wl.modes if m != "reuse")
    n_full = sum(1 for m in wl.modes if m == "full")
    n_re = n_sel - n_full
    dense = n_full * (wl.B * wl.N * wl.d * 2 + qidx)
    if n_re and wl.P == 0:
        dense += n_re * (wl.B * wl.N * wl.d * 2 + qidx)
    out["index_scores"] = (dense, n_full + (n_re if wl.P == 0 else 0))
    if wl.P and n_re:
        out["index_pool"] = (n_re * (rows * wl.P * (wl.d * 2 + 4) + qidx), n_re)
    attn = wl.n_layers * (rows * wl.k * (kv_row + 4) + rows * wl.Ha * (wl.D * 2 * 2 + 4))
    attn += wl.n_layers * wl.B * wl.swa * wl.D * 2          # each layer's window rows
    out["attn"] = (attn, wl.n_layers)
    if wl.compress_new_tokens:        # raw tokens c (bf16) and z (f32) in, entries (bf16) out
        t_in = wl.compress_new_tokens + (wl.m if wl.halo else 0)
        n_new = wl.compress_new_tokens // wl.m
        out["compress"] = (wl.B * (t_in * wl.D * 6 + n_new * wl.D * 2) + 2 * wl.m * wl.D * 4, 1)
    return out


def algorithmic_flops(wl):
    """Tensor-core work the method must do in one step, per kernel kind: the
    indexer's q.k products over the scored entries (Full: every visible entry,
    causal in prefill; Reindex: the pool) and attention's two products over
    the selected rows.  {kind: flops per step}."""
    import numpy as np
    from kv_cache_csa2_b200.configs import n_visible
    rows = wl.B * wl.Q
    nv = n_visible(wl)
    visible = int(np.asarray(nv, dtype=np.int64).sum()) if nv is not None else rows * wl.N
    n_full = sum(1 for m in wl.modes if m == "full")
    n_re = sum(1 for m in wl.modes if m == "reindex")
    per = 2 * wl.Hi * wl.d
    out = {"index_scores": per * visible * (n_full + (n_re if wl.P == 0 else 0))}
    if wl.P and n_re:
        out["index_pool"] = per * rows * wl.P * n_re
    out["attn"] = wl.n_layers * rows * (wl.k + wl.swa) * wl.Ha * wl.D * 4
    return out


def kernel_min_bytes(wl):
    """Per kind, what one launch of that kernel must at least move (for the
    kernels whose inputs are intermediates, e.g. top-k reading the scores, this
    is not part of the group's algorithmic bytes).  {kind: bytes per step}."""
    rows = wl.B * wl.Q
    alg = {k: v[0] for k, v in algorithmic_bytes(wl).items()}
    n_full = sum(1 for m in wl.modes if m == "full")
    n_re = sum(1 for m in wl.modes if m == "reindex")
    L_full = wl.N
    topk = n_full * rows * (L_full * 4 + (wl.k + wl.P) * 4) * (2 if wl.P else 1)
    topk += n_re * rows * ((wl.P if wl.P else wl.N) * 4 + wl.k * 4)
    alg["topk"] = topk
    return alg


# ---------------------------------------------------------------------------- ours

def device_inputs(wl, inp, torch, device):
    import numpy as np

    def bf(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(device)

    d = {"kv": bf(inp["kv"]), "index_k": bf(inp["index_k"]),
         "n_visible": torch.from_numpy(inp["n_visible"]).to(device) if inp["n_visible"] is not None else None,
         "layers": []}
    for L in inp["layers"]:
        e = {"q_attn": bf(L["q_attn"])}
        if "win" in L:
            e["swa"] = (bf(L["win"]), torch.from_numpy(L["win_end"]).to(device), wl.swa)
        if "q_index" in L:
            e["q_index"] = bf(L["q_index"])
            e["w_index"] = torch.from_numpy(L["w_index"]).to(device)
        d["layers"].append(e)
    return d


def run_ours(args, wl, world, rank, local):
    import torch
    import kv_cache_csa2_b200 as K
    from kv_cache_csa2_b200 import inputs as I

    if not torch.cuda.is_available():
        raise SystemExit("bench.py: no CUDA device")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist_init(world, "nccl")
    K.lib()
    inp = I.make_inputs(wl, seed=args.seed)
    D = device_inputs(wl, inp, torch, dev)
    kv, kv_scales = D["kv"], None
    compress = None
    if wl.compress_new_tokens:
        # the newest entries are compressed from raw tokens inside every step
        # (row a1), appended after the cached entries of the KV buffer
        n_cached = inp["kv"].shape[1]
        kv = torch.empty(wl.B, wl.N, wl.D, dtype=torch.bfloat16, device=dev)
        kv[:, :n_cached] = D["kv"]
        del D["kv"]
        bf = lambda bits: torch.from_numpy(bits.view("int16")).view(torch.bfloat16).to(dev)  # noqa: E731
        D["c"], D["z"] = bf(inp["c"]), torch.from_numpy(inp["z"]).to(dev)
        D["bias"] = torch.from_numpy(inp["bias"]).to(dev)
        tail = kv[:, n_cached:]

        def compress():
            K.csa2_compress(D["c"], D["z"], D["bias"], wl.m, has_left_halo=wl.halo, out=tail,
                            out_batch_stride=wl.N * wl.D)
    if wl.kv_fp4:
        kv, kv_scales = K.csa2_fp4_pack(D["kv"])
    modes = [{"full": K.FULL, "reindex": K.REINDEX, "reuse": K.REUSE}[m] for m in wl.modes]
    g = K.Group(wl.B, wl.Q, wl.N, wl.D, wl.Ha, wl.Hi, wl.d, wl.k, modes, P=wl.P, scale=wl.attn_scale,
                kv_fmt=K.KV_FP4 if wl.kv_fp4 else K.KV_BF16)
    outs = [torch.empty(wl.B, wl.Q, wl.Ha, wl.D, dtype=torch.bfloat16, device=dev) for _ in wl.modes]
    lses = [torch.empty(wl.B, wl.Q, wl.Ha, dtype=torch.float32, device=dev) for _ in wl.modes]
    kws = []
    for i, mode in enumerate(wl.modes):
        L = D["layers"][i]
        kw = {}
        if mode == "full":
            kw = dict(kv=kv, kv_scales=kv_scales, index_k=D["index_k"], n_visible=D["n_visible"])
        elif mode == "reindex":
            kw = dict(n_visible=D["n_visible"])
        if mode != "reuse":
            kw.update(q_index=L["q_index"], w_index=L["w_index"])
        kws.append(kw)

    def layer(i):
        if i == 0 and compress is not None:
            compress()
        g.layer(i, D["layers"][i]["q_attn"], outs[i], lses[i], swa=D["layers"][i].get("swa"), **kws[i])

    flush_buf = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)

    def flush():
        flush_buf.fill_(1.0)

    n_layers = wl.n_layers
    for _ in range(args.warmup):
        for i in range(n_layers):
            flush()
            layer(i)
    torch.cuda.synchronize()
    K.csa2_device_error()
    # each layer's calls into the library, captured once as a CUDA graph (the
    # library launches on the capturing stream); replays carry no host work
    graphs, graph_note = None, "each layer replayed as a CUDA graph of its library calls"
    if not args.eager:
        try:
            graphs = []
            for i in range(n_layers):
                gph = torch.cuda.CUDAGraph()
                with torch.cuda.graph(gph):
                    layer(i)
                graphs.append(gph)
            torch.cuda.synchronize()
        except Exception as e:                      # report and time eagerly instead
            graphs, graph_note = None, f"eager launches (graph capture failed: {e})"
    else:
        graph_note = "eager launches"

    def run_layer(i):
        if graphs is not None:
            graphs[i].replay()
        else:
            layer(i)

    # ---- cold: flush before every layer, per-layer events
    for _ in range(args.warmup):
        for i in range(n_layers):
            flush()
            run_layer(i)
    torch.cuda.synchronize()
    ev = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(n_layers)] for _ in range(args.steps)]
    sampler = ClockSampler(local)
    barrier(world)
    torch.cuda.synchronize()
    sampler.start()
    t0 = time.perf_counter()
    for s in range(args.steps):
        for i in range(n_layers):
            flush()
            ev[s][i][0].record()
            run_layer(i)
            ev[s][i][1].record()
    torch.cuda.synchronize()
    barrier(world)
    wall = time.perf_counter() - t0
    clocks = sampler.stop()
    K.csa2_device_error()
    step_ms = [sum(a.elapsed_time(b) for a, b in ev[s]) for s in range(args.steps)]
    layer_ms = [statistics.mean(ev[s][i][0].elapsed_time(ev[s][i][1]) for s in range(args.steps))
                for i in range(n_layers)]
    ms_local = statistics.mean(step_ms)
    ms = reduce_max(ms_local, world, dev)
    queries = world * wl.B * wl.Q
    value = queries / (ms / 1e3)

    # ---- per-kernel device times over the same K steps (eager launches, each
    # bracketed by events on its own stream by the library)
    K.reset_launch_counts()
    K.timing_reset()
    K.timing_enable(True)
    for s in range(args.steps):
        for i in range(n_layers):
            flush()
            layer(i)
    torch.cuda.synchronize()
    K.timing_enable(False)
    launches = K.launch_counts()
    ktimes = K.kernel_times()
    K.csa2_device_error()

    # ---- warm: the group back to back
    for _ in range(args.warmup):
        for i in range(n_layers):
            run_layer(i)
    barrier(world)
    torch.cuda.synchronize()
    w0, w1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    w0.record()
    for _ in range(args.steps):
        for i in range(n_layers):
            run_layer(i)
    w1.record()
    torch.cuda.synchronize()
    warm_ms = reduce_max(w0.elapsed_time(w1) / args.steps, world, dev)
    graphs = None

    # ---- e2e: host inputs -> API -> host outputs, copies inside the timed region.
    # Layer i's inputs go up on a copy stream ahead of the compute, layer i's
    # outputs come back on another while layer i+1 computes (a step starts
    # after the previous step's compute and copies).
    h_in, d_in = [[] for _ in range(n_layers)], [[] for _ in range(n_layers)]
    if compress is not None:          # the step's raw tokens go up with the first layer's queries
        for key in ("c", "z"):
            h_in[0].append(D[key].cpu().pin_memory())
            d_in[0].append(D[key])
    for i in range(n_layers):
        for key in ("q_attn", "q_index", "w_index"):
            t = D["layers"][i].get(key)
            if t is not None:
                h_in[i].append(t.cpu().pin_memory())
                d_in[i].append(t)
    h_out = [[outs[i].cpu().pin_memory(), lses[i].cpu().pin_memory()] for i in range(n_layers)]
    d_out = [[outs[i], lses[i]] for i in range(n_layers)]
    bi = sum(t.numel() * t.element_size() for ts in h_in for t in ts)
    bo = sum(t.numel() * t.element_size() for ts in h_out for t in ts)
    comp = torch.cuda.current_stream()
    s_up, s_down = torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(n_layers)]
    ev_done = [torch.cuda.Event() for _ in range(n_layers)]

    def e2e_step():
        s_up.wait_stream(comp)                   # the previous step no longer reads the inputs
        comp.wait_stream(s_down)                 # nor are its outputs still being read back
        with torch.cuda.stream(s_up):
            for i in range(n_layers):
                for h, d in zip(h_in[i], d_in[i]):
                    d.copy_(h, non_blocking=True)
                ev_in[i].record(s_up)
        for i in range(n_layers):
            comp.wait_event(ev_in[i])
            layer(i)
            ev_done[i].record(comp)
            s_down.wait_event(ev_done[i])
            with torch.cuda.stream(s_down):
                for h, d in zip(h_out[i], d_out[i]):
                    h.copy_(d, non_blocking=True)
        comp.wait_stream(s_down)                 # the step ends when its outputs are on the host

    for _ in range(args.warmup):
        e2e_step()
    barrier(world)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        e2e_step()
    e1.record()
    torch.cuda.synchronize()
    e2e_ms = reduce_max(e0.elapsed_time(e1) / args.steps, world, dev)
    g.close()

    # ---- roofline of the dominant kernel (largest device time in the cold region)
    hbm, peak_src = measured_hbm_gbs()
    alg = algorithmic_bytes(wl)
    per_kind = {k: v for k, v in ktimes.items() if v[1] > 0}
    dom = max(per_kind, key=lambda k: per_kind[k][0]) if per_kind else None
    roof = None
    if dom is not None:
        tot_ms, n = per_kind[dom]
        avg_s = tot_ms / n / 1e3
        per_step = n / args.steps
        bytes_per_launch = kernel_min_bytes(wl).get(dom, 0) / max(per_step, 1)
        flops_per_launch = algorithmic_flops(wl).get(dom, 0) / max(per_step, 1)
        tflops, tf_src = measured_tflops(avg_s)
        # the bound is whichever of the two ideal times is longer
        tensor = flops_per_launch / (tflops * 1e12) > bytes_per_launch / (hbm * 1e9)
        if tensor:
            achieved = flops_per_launch / avg_s / 1e12 if avg_s > 0 else 0.0
            roof = {"kernel": dom, "bound": "tensor", "achieved": round(achieved, 1), "peak": tflops,
                    "unit": "TFLOP/s", "frac": round(achieved / tflops, 4), "traffic": ncu_traffic(dom, wl.name),
                    "algorithmic_flops_per_launch": int(flops_per_launch),
                    "algorithmic_bytes_per_launch": int(bytes_per_launch), "peak_source": tf_src}
        else:
            achieved = bytes_per_launch / avg_s / 1e9 if avg_s > 0 else 0.0
            roof = {"kernel": dom, "bound": "hbm", "achieved": round(achieved, 1), "peak": hbm,
                    "unit": "GB/s", "frac": round(achieved / hbm, 4), "traffic": ncu_traffic(dom, wl.name),
                    "algorithmic_bytes_per_launch": int(bytes_per_launch),
                    "peak_source": f"{peak_src} (MEASURED_PEAKS.json hbm_gbs)" if peak_src == "measured"
                    else "fallback 6650 GB/s"}
        roof.update(avg_launch_us=round(avg_s * 1e6, 2), launches=n)
    kernels = {k: {"total_ms": round(v[0], 4), "launches": v[1],
                   "avg_us": round(v[0] / v[1] * 1e3, 2)} for k, v in per_kind.items()}
    total_alg = sum(v[0] for v in alg.values())
    res = {
        "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1)/U(0,1) inputs of the workload's shapes)",
        "config": {"workload": wl.name, "B": wl.B, "Q": wl.Q, "L": wl.L, "m": wl.m, "N": wl.N, "swa": wl.swa,
                   "D": wl.D, "Ha": wl.Ha, "Hi": wl.Hi, "d": wl.d, "k": wl.k, "P": wl.P,
                   "modes": ",".join(wl.modes), "kv": "fp4" if wl.kv_fp4 else "bf16",
                   "l2": "flushed before every layer (2x L2 write outside the layer's events); "
                         "ms_per_step = sum of per-layer CUDA-event times",
                   "launch": graph_note,
                   "parallelism": f"replicas x{world}"},
        "group_bytes": int(total_alg),
        "group_achieved_gbs": round(total_alg / (ms_local / 1e3) / 1e9, 1),
        "group_frac_of_hbm": round(total_alg / (ms_local / 1e3) / 1e9 / hbm, 4),
        "layer_ms": [round(x, 4) for x in layer_ms],
        "warm": {"ms_per_step": round(warm_ms, 4), "value": round(queries / (warm_ms / 1e3), 1),
                 "note": "same group back to back, no L2 flush"},
        "e2e": {"value": round(queries / (e2e_ms / 1e3), 1), "unit": UNIT,
                "h2d_bytes_per_step": bi, "d2h_bytes_per_step": bo,
                "note": "per step: pinned-host -> device copy of every layer's queries and head "
                        "weights, the group through the C ABI, device -> pinned-host copy of every "
                        "layer's output and lse, on two copy streams that overlap the other "
                        "layers' compute; KV cache and indexer keys stay resident"},
        "roofline": roof,
        "kernels": kernels,
        "gpu_launches": int(sum(launches.values())),
        "gpu_launches_note": "library kernel launches over the K timed steps (counted on the eager pass "
                             "that times each kernel; the graph replays launch the same kernels)",
        "clocks": clocks,
        "wall_s_timed_region": round(wall, 4),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        res["cpu_baseline"] = cpu_baseline(wl, inp, budget_s=args.cpu_budget)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    return res


# ---------------------------------------------------------------------------- oracle (CPU)

def oracle_queries(wl, inp, queries):
    """Run the oracle's layer group for the listed (b, q) queries (each
    sequence's raw tokens compressed once per call); returns seconds."""
    import numpy as np
    import oracle as O
    from kv_cache_csa2_b200 import inputs as I

    t0 = time.perf_counter()
    n_cached = inp["kv"].shape[1]
    new_of = {}
    for b, t in queries:
        kb = inp["kv"][b:b + 1]
        if wl.compress_new_tokens and b not in new_of:   # the newest entries come from raw tokens
            _, new_of[b] = O.compress(O.bf16_bits_to_float(inp["c"][b:b + 1]),
                                      inp["z"][b:b + 1].astype(np.float64),
                                      inp["bias"].astype(np.float64), wl.m, wl.halo)
        new = new_of.get(b)

        def rows(_, ids, kb=kb, new=new):
            ids = np.asarray(ids)
            r = np.empty((len(ids), wl.D))
            old = ids < n_cached
            r[old] = O.bf16_bits_to_float(kb[0, ids[old]])
            if (~old).any():
                r[~old] = new[0, ids[~old] - n_cached]
            return O.fp4_unpack(*O.fp4_pack(r)) if wl.kv_fp4 else r

        layers = []
        for L in inp["layers"]:
            d = {"q_attn": O.bf16_bits_to_float(L["q_attn"][b:b + 1, t:t + 1])}
            if "win" in L:
                d["swa"] = (O.bf16_bits_to_float(L["win"][b:b + 1]), L["win_end"][b:b + 1, t:t + 1], wl.swa)
            if "q_index" in L:
                d["q_index"] = O.bf16_bits_to_float(L["q_index"][b:b + 1, t:t + 1])
                d["w_index"] = L["w_index"][b:b + 1, t:t + 1].astype(np.float64)
            layers.append(d)
        nv = inp["n_visible"][b:b + 1, t:t + 1] if inp["n_visible"] is not None else None
        O.run_group(list(wl.modes), layers, rows, I.bf16_bits_to_f32(inp["index_k"][b:b + 1]), wl.k,
                    wl.attn_scale, pool_size=wl.P, n_visible=nv)
    return time.perf_counter() - t0


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        return max((i.get("num_threads", 1) for i in threadpool_info()), default=1)
    except Exception:
        return os.cpu_count() or 1


def cpu_baseline(wl, inp, budget_s=20.0):
    qs = [(b, t) for b in range(wl.B) for t in range(wl.Q)]
    done, spent = 0, 0.0
    while done < len(qs) and spent < budget_s:
        spent += oracle_queries(wl, inp, [qs[done]])
        done += 1
    return {"value": round(done / spent, 3), "unit": UNIT, "cores": os.cpu_count() or 1,
            "blas_threads": blas_threads(), "kind": "oracle",
            "sample": f"{done} of the workload's {len(qs)} queries, each through the whole layer group "
                      f"(float64 numpy oracle), {spent:.1f} s"}


def run_reference(args, wl, world, rank):
    if rank != 0:
        return None
    from kv_cache_csa2_b200 import inputs as I
    inp = I.make_inputs(wl, seed=args.seed)
    qs = [(b, t) for b in range(wl.B) for t in range(wl.Q)]
    # a step is the GPU arm's whole batch when it has at most REF_MAX_BATCH
    # queries (every decode workload), else REF_SAMPLE queries spread over it
    if len(qs) <= REF_MAX_BATCH:
        per_step, same = len(qs), True
    else:
        per_step, same = REF_SAMPLE, False
    stride = max(1, len(qs) // per_step)
    for i in range(args.warmup):            # warm-up: one query each (untimed)
        oracle_queries(wl, inp, [qs[i % len(qs)]])
    spent, done = 0.0, 0
    for i in range(args.steps):
        batch = [qs[(i + j * stride) % len(qs)] for j in range(per_step)]
        spent += oracle_queries(wl, inp, batch)
        done += len(batch)
    value = done / spent
    cores = os.cpu_count() or 1
    sample = (f"{args.steps} steps of {per_step} queries, each through the whole layer group "
              f"(float64 numpy oracle){'' if same else f'; the workload has {len(qs)} queries per step'}")
    return {"impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": UNIT,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(spent / args.steps * 1e3, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded N(0,1)/U(0,1) inputs of the workload's shapes)",
            "config": {"workload": wl.name, "B": wl.B, "Q": wl.Q, "L": wl.L, "N": wl.N, "D": wl.D,
                       "k": wl.k, "P": wl.P, "modes": ",".join(wl.modes),
                       "sample_per_step": f"{per_step} queries" + (" (the whole batch)" if same else "")},
            "cpu_baseline": {"value": round(value, 3), "unit": UNIT, "cores": cores,
                             "blas_threads": blas_threads(), "kind": "oracle", "sample": sample},
            "e2e": {"value": round(value, 3), "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


# ---------------------------------------------------------------------------- kernel cases

KERNEL_CASES = ("attn", "full", "reindex", "attn_swa", "dense", "compress_hca", "full_fp4",
                "reindex_fp4", "fused_prefill", "fused_small", "attn_prefill")


def run_kernel_case(name, reps=4, timed=False):
    """One library call on seeded synthetic inputs of one workload's shapes,
    `reps` times (the short program the ncu captures use; prints one JSON
    line).  With `timed`, each call runs after an L2 flush, bracketed by CUDA
    events on the launching stream, and the line carries the median time and
    the algorithmic bytes and flops of one call with their roofline fraction.
      attn           csa2_sparse_attn, 8 queries x 64 heads x 512, k = 2048
      full           csa2_index_topk(FULL) over 8 x 262144 entries, pool 16384 + top 2048
      reindex        csa2_index_topk(REINDEX) inside a 16384-slot pool, top 2048
      attn_swa       attn plus each query's 128-row sliding window (csa2_sparse_attn_swa)
      dense          HCA attention: 8 queries over 8192 entries (1M tokens / 128)
      compress_hca   HCA compression of 8 x 8192 tokens into groups of 128 (D = 512)
      full_fp4       full with the FP4 indexer (FP4 q and K, bf16 scores)
      reindex_fp4    reindex with the FP4 indexer
      fused_prefill  csa2_index_topk(FULL) of a 4096-query prefill chunk over 262144
                     entries, top 2048: the fused indexer + streaming top-k
      fused_small    the fused indexer on 592 queries (one 4-query group per SM) over 65536
                     entries, top 2048 (the size its ncu capture uses)
      attn_prefill   csa2_sparse_attn of the same chunk: 4096 queries x 64 heads x 512,
                     k = 2048 of 262144 entries each"""
    import torch
    import kv_cache_csa2_b200 as K
    g = torch.Generator(device="cuda").manual_seed(0)
    B, D, Ha, k_sel = 8, 512, 64, 2048
    flops, nbytes = 0.0, 0.0

    def randn(*shape, std=1.0):
        return (torch.randn(*shape, device="cuda", generator=g) * std).to(torch.bfloat16)

    def sel_ids(N, k):
        return torch.stack([torch.sort(torch.randperm(N, device="cuda", generator=g)[:k])[0]
                            for _ in range(B)]).view(B, 1, k).to(torch.int32)

    if name in ("attn", "attn_swa"):
        N = 32768
        kv, q, topk = randn(B, N, D), randn(B, 1, Ha, D), sel_ids(N, k_sel)
        nbytes = B * k_sel * (D * 2 + 4) + B * Ha * (D * 4 + 4)
        flops = 4.0 * B * k_sel * Ha * D
        if name == "attn":
            call = lambda: K.csa2_sparse_attn(q, kv, topk, D ** -0.5)  # noqa: E731
        else:
            win = randn(B, 128, D)
            we = torch.full((B, 1), 128, dtype=torch.int32, device="cuda")
            nbytes += B * 128 * D * 2
            flops += 4.0 * B * 128 * Ha * D
            call = lambda: K.csa2_sparse_attn_swa(q, kv, topk, D ** -0.5, win, we, 128)  # noqa: E731
    elif name == "attn_prefill":
        Q, N = 4096, 262144
        kv, q = randn(1, N, D), randn(1, Q, Ha, D)
        topk = torch.stack([torch.sort(torch.randperm(N, device="cuda", generator=g)[:k_sel])[0]
                            for _ in range(Q)]).view(1, Q, k_sel).to(torch.int32)
        nbytes = Q * k_sel * (D * 2 + 4) + Q * Ha * (D * 4 + 4)
        flops = 4.0 * Q * k_sel * Ha * D
        call = lambda: K.csa2_sparse_attn(q, kv, topk, D ** -0.5)  # noqa: E731
    elif name == "dense":
        N = 8192
        kv, q = randn(B, N, D), randn(B, 1, Ha, D)
        nbytes = B * N * D * 2 + B * Ha * (D * 4 + 4)
        flops = 4.0 * B * N * Ha * D
        call = lambda: K.csa2_dense_attn(q, kv, D ** -0.5)  # noqa: E731
    elif name == "compress_hca":
        T, m = 8192, 128
        c = randn(B, T, D)
        z = torch.randn(B, T, D, device="cuda", generator=g)
        bias = torch.randn(m, D, device="cuda", generator=g)
        nbytes = B * T * D * 6 + B * (T // m) * D * 2 + m * D * 4
        call = lambda: K.csa2_compress_hca(c, z, bias, m)  # noqa: E731
    elif name == "fused_small":
        Q, N = 592, 65536
        q = randn(1, Q, 64, 128)
        w = torch.randn(1, Q, 64, device="cuda", generator=g)
        kk = randn(1, N, 128)
        flops = 2.0 * 64 * 128 * Q * N
        nbytes = N * 128 * 2 + Q * 64 * (128 * 2 + 4) + Q * k_sel * 4
        call = lambda: K.csa2_index_topk(K.FULL, q, w, kk, k_sel)  # noqa: E731
    elif name == "fused_prefill":
        Q, N = 4096, 262144
        q = randn(1, Q, 64, 128)
        w = torch.randn(1, Q, 64, device="cuda", generator=g)
        kk = randn(1, N, 128)
        nv = torch.arange(N - Q + 1, N + 1, dtype=torch.int32, device="cuda").view(1, Q)
        flops = 2.0 * 64 * 128 * float(nv.sum().item())
        nbytes = N * 128 * 2 + Q * 64 * (128 * 2 + 4) + Q * k_sel * 4
        call = lambda: K.csa2_index_topk(K.FULL, q, w, kk, k_sel, n_visible=nv)  # noqa: E731
    else:
        N, P = 262144, 16384
        fp4 = name.endswith("_fp4")
        q = randn(B, 1, 64, 128, std=1 / 11.3)
        w = torch.rand(B, 1, 64, device="cuda", generator=g)
        kk = randn(B, N, 128, std=1 / 11.3)
        row = 128 // 2 + 128 // 16 if fp4 else 128 * 2
        pool = sel_ids(N, P) if name.startswith("reindex") else None
        scored = B * (P if pool is not None else N)
        nbytes = scored * (row + (4 if pool is not None else 0)) + B * k_sel * 4 + (B * P * 4 if pool is None else 0)
        flops = 2.0 * scored * 64 * 128
        if fp4:
            qc, qs = K.csa2_fp4_pack(q)
            kc, ks = K.csa2_fp4_pack(kk)
            if pool is None:
                call = lambda: K.csa2_index_topk_fp4(K.FULL, qc, qs, w, kc, ks, k_sel, pool_size=P)  # noqa: E731
            else:
                call = lambda: K.csa2_index_topk_fp4(K.REINDEX, qc, qs, w, kc, ks, k_sel, pool_in=pool)  # noqa: E731
        elif pool is None:
            call = lambda: K.csa2_index_topk(K.FULL, q, w, kk, k_sel, pool_size=P)  # noqa: E731
        else:
            call = lambda: K.csa2_index_topk(K.REINDEX, q, w, kk, k_sel, pool_in=pool)  # noqa: E731
    res = {"kernel_case": name, "reps": reps, "ok": True}
    if not timed:
        for _ in range(reps):
            call()
        torch.cuda.synchronize()
        K.csa2_device_error()
        return res
    flush_buf = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device="cuda")
    for _ in range(3):
        flush_buf.fill_(1.0)
        call()
    times = []
    for _ in range(reps):
        flush_buf.fill_(1.0)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        call()
        e1.record()
        e1.synchronize()
        times.append(e0.elapsed_time(e1))
    K.csa2_device_error()
    t = statistics.median(times) / 1e3
    hbm, _ = measured_hbm_gbs()
    tflops, tsrc = measured_tflops(t)
    res.update(us=round(t * 1e6, 2), algorithmic_bytes=int(nbytes), algorithmic_flops=int(flops),
               achieved_gbs=round(nbytes / t / 1e9, 1), achieved_tflops=round(flops / t / 1e12, 2),
               hbm_frac=round(nbytes / t / 1e9 / hbm, 4), tensor_frac=round(flops / t / 1e12 / tflops, 4),
               tensor_peak=tflops, tensor_peak_source=tsrc,
               l2="flushed before every call (2x L2 write outside the events)")
    return res


# ---------------------------------------------------------------------------- main

def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", type=int, default=4, choices=[1, 2, 3, 4, 5, 6])
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--cpu-budget", type=float, default=20.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--eager", action="store_true", help="launch layers eagerly instead of CUDA graphs")
    ap.add_argument("--kernel-case", choices=KERNEL_CASES,
                    help="run one library call of a workload 4 times and exit (for ncu captures)")
    ap.add_argument("--timed", action="store_true",
                    help="with --kernel-case: time --steps calls (L2 flushed before each) and report "
                         "the median with its roofline fraction")
    args = ap.parse_args(argv)
    if args.kernel_case:
        reps = args.steps if args.timed else 4
        print(json.dumps(run_kernel_case(args.kernel_case, reps=reps, timed=args.timed)), flush=True)
        return
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    from kv_cache_csa2_b200.configs import CONFIGS
    wl = CONFIGS[args.config]
    world, rank, local = dist_env()
    if args.impl == "reference":
        res = run_reference(args, wl, world, rank)
    else:
        res = run_ours(args, wl, world, rank, local)
    if rank == 0 and res is not None:
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
