#!/usr/bin/env python
"""Decode throughput of the ARKV tri-state KV-cache path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl arkv|reference]

A step is one decode step of the whole attention stack: for every layer, append +
mixed-precision attention (arkv_decode_attn), score update (arkv_score_update),
and the tier reassignment (arkv_reassign) on every reassign_interval-th step.  The
score update and reassignment of a layer run on a side stream (layers dealt round
robin over --streams - 1 of them), beside the next layers' attention; the layer's next
attention call waits for them.
Each GPU runs its own replica of the workload (independent sequences; no
collective on the data path), so `value` is the tokens/s of all ranks together
("scaling": "weak").  Inputs are synthetic and seeded; each step streams the whole
compressed cache (GBs, far above the 126 MB L2), so no L2 flush is needed.
"""
from __future__ import annotations

import argparse
import csv
import io
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from mixed_precision_kv_arkv_b200 import workloads  # noqa: E402

METRIC = "decode tokens/s & HBM GB/s (% of peak), tri-state KV attention, 8B shape 32K"
FALLBACK_HBM_GBS = 6650.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=128)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default=workloads.LLAMA3_8B.name, choices=sorted(workloads.BY_NAME))
    ap.add_argument("--impl", default="arkv", choices=["arkv", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--streams", type=int, default=5,
                    help="S >= 2: score updates and reassignments on S - 1 side streams (layer l on side "
                         "stream l mod (S - 1)) beside the next layers' attention; 1: everything on one stream")
    ap.add_argument("--no-early-start", action="store_true",
                    help="launch every attention call with early_start = 0 (it waits for the previous "
                         "kernel before reading its cache)")
    ap.add_argument("--layers", type=int, default=None,
                    help="run only this many layers of the workload (profiling a smaller case)")
    return ap.parse_args()


# ------------------------------------------------------------------ helpers
def hbm_peak():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def max_over_ranks(x: float, device, world: int) -> float:
    """The largest of every rank's x (the job's time is its slowest rank's); x itself
    when there is one rank."""
    if world <= 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tokens_per_s(batch: int, steps: int, world: int, ms: float) -> float:
    """Whole-job decode throughput: every rank decodes `batch` sequences per step
    (independent replicas), timed by the slowest rank."""
    return batch * steps * world / (ms * 1e-3)


# kernels one decode step of one layer launches: decode_attn_kernel (arkv_decode_attn,
# the split merge included) and score_update_kernel (arkv_score_update);
# arkv_reassign adds reassign_kernel every reassignment interval
KERNELS_PER_LAYER_STEP = 2


def kernel_traffic(kernel_file: str):
    """DRAM bytes (read + write) of one arkv_decode_attn call -- its attention and
    merge kernels -- from the committed ncu summary, if it was taken on the current
    kernel source (else None)."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "decode_attn_traffic.txt")
    src = os.path.join(ROOT, "mixed_precision_kv_arkv_b200", "csrc", kernel_file)
    try:
        kv = dict(line.split(":", 1) for line in open(path) if ":" in line)
        sha = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
        if kv.get("kernel_src_sha256_16", "").strip() != sha:
            return None
        return float(kv["dram_bytes_per_launch_scaled"].strip())
    except Exception:
        return None


class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, local_rank: int):
        vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
        ids = [v.strip() for v in vis.split(",") if v.strip()]
        self.index = ids[local_rank] if local_rank < len(ids) else str(local_rank)
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.first = self.proc.stdout.readline()     # sampling has started
        except Exception:
            self.proc = None
            self.first = ""
        return self

    def __exit__(self, *exc):
        self.out = ""
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()
            self.out = self.out or ""
        return False

    def summary(self):
        rows = [r for r in csv.reader(io.StringIO(self.out or "")) if len(r) >= 9]
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        sm = [float(r[1]) for r in rows if r[1].strip().replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].strip().replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].strip() == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons, "samples": len(rows)}


# ------------------------------------------------------------------ CPU baseline (the oracle)
class OracleSampler:
    """The oracle on a bounded sample of the workload: some rows of layer 0, set up
    once (prefill + initial reassignment, untimed), then timed decode steps
    (attention + score update, and the reassignment on its steps)."""

    def __init__(self, wl, rows=(0,)):
        from threadpoolctl import threadpool_info
        from mixed_precision_kv_arkv_b200 import inputs
        from oracle import arkv as A

        self.wl, self.rows, self.inputs = wl, list(rows), inputs
        pre = inputs.layer_prefill(wl, 0, 0, seqs=sorted({r // wl.hkv for r in rows}),
                                   kv_heads=sorted({r % wl.hkv for r in rows}))
        f = inputs.bf16_to_f64
        self.lay = A.OracleLayer(wl.batch, wl.hq, wl.hkv, wl.head_dim, wl.window, wl.n_obs,
                                 wl.budget_frac, wl.gamma, pre["ctx_len"], rows=self.rows,
                                 fmt=wl.quant_format)
        self.lay.prefill(f(pre["k"]), f(pre["v"]), f(pre["q_obs"]))
        self.r = wl.oq_ratio if wl.oq_ratio is not None else wl.r_bar
        self.lay.initial_reassign(self.r)
        self.t = 0
        self.threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])

    def step(self) -> float:
        """One timed decode step of the sampled rows; seconds per row-step."""
        wl, f = self.wl, self.inputs.bf16_to_f64
        d = self.inputs.decode_inputs(wl, 0, self.t)
        t0 = time.perf_counter()
        self.lay.decode_step(self.t, f(d["q"]), f(d["k_new"]), f(d["v_new"]))
        if (self.t + 1) % wl.reassign_interval == 0:
            self.lay.reassign(self.t, self.r)
        dt = time.perf_counter() - t0
        self.t += 1
        return dt / len(self.rows)

    def describe(self, n_steps):
        wl = self.wl
        return (f"oracle on row(s) {self.rows} of layer 0 ({wl.name}), {n_steps} decode steps "
                f"incl. reassignments every {wl.reassign_interval}; time per row-step scaled to "
                f"{wl.layers} layers x {wl.rows} rows")


def cpu_baseline_from_state(wl, lay0, ctx_np, t_next, o_dev, seconds, decode_step_dev):
    """The oracle on the benchmarked data: row 0 of layer 0 is read back from the device
    after the timed passes and loaded into the oracle; one decode step is then run on
    both (the device's step outside any timed region) and compared -- attention output
    and scores -- and the oracle goes on alone for timed steps, first on every core,
    then on one thread."""
    import numpy as np
    import torch
    from threadpoolctl import threadpool_info, threadpool_limits
    from mixed_precision_kv_arkv_b200 import inputs
    from oracle import arkv as A

    c, rid, D, G = lay0["cache"], 0, wl.head_dim, wl.group
    n0 = int(ctx_np[0])
    n16, n8 = int(c.n_bf16[rid]), int(c.n_fp8[rid])
    f = inputs.bf16_to_f64
    to_u16 = lambda t: t.view(torch.int16).cpu().numpy().view(np.uint16)
    pos = np.concatenate([c.pos16[rid, :n16].cpu().numpy(), c.pos8[rid, :n8].cpu().numpy()]).astype(np.int64)
    order = np.argsort(pos, kind="stable")
    cat = lambda a, b: np.concatenate([a, b])[order]
    zeros16 = np.zeros((n8, D), np.uint16)
    row = A.Row(D=D, pos=pos[order], orig=cat(np.ones(n16, bool), np.zeros(n8, bool)),
                kf=f(cat(to_u16(c.k16[rid, :n16]), zeros16)), vf=f(cat(to_u16(c.v16[rid, :n16]), zeros16)),
                kc=cat(np.zeros((n16, D), np.uint8), c.k8[rid, :n8].cpu().numpy()),
                vc=cat(np.zeros((n16, D), np.uint8), c.v8[rid, :n8].cpu().numpy()),
                sk=cat(np.ones(n16, np.float32), c.sk[rid, :n8].cpu().numpy()),
                sv=cat(np.ones(n16, np.float32), c.sv[rid, :n8].cpu().numpy()),
                mu=cat(c.mu16[rid, :n16].cpu().numpy(), c.mu8[rid, :n8].cpu().numpy()),
                m2=cat(c.m2_16[rid, :n16].cpu().numpy(), c.m2_8[rid, :n8].cpu().numpy()),
                fmt=wl.quant_format)
    # Welford counts after step t_next - 1: the observations the token has had
    p_ = row.pos
    row.cnt = np.where(p_ < n0, np.minimum(wl.n_obs, n0 - p_) + t_next, t_next - (p_ - n0)).astype(np.int64)

    dec = lay0["dec"]
    host = {k: dec[k].view(torch.int16).cpu().numpy().view(np.uint16) for k in ("q", "k_new", "v_new")}
    n_in = host["q"].shape[0]

    def oracle_step(t):
        i = t % n_in
        row.append(n0 + t, f(host["k_new"][i, 0, 0]), f(host["v_new"][i, 0, 0]))
        o, _ = A.decode_row(row, f(host["q"][i, 0, :G]))
        if (t + 1) % wl.reassign_interval == 0:
            A.reassign_row(row, n0 + t + 1, wl.window, wl.budget_frac, lay0["r"], wl.gamma)
        return o

    # the step both sides take from the same state
    decode_step_dev(t_next)
    if torch.cuda.is_available():
        torch.cuda.synchronize()
    t0 = time.perf_counter()
    o_ref = oracle_step(t_next)
    first = time.perf_counter() - t0
    o_gpu = o_dev[0, 0, :G].cpu().numpy().astype(np.float64)
    o_rel = float((np.abs(o_gpu - o_ref).max(axis=-1) / np.abs(o_ref).max(axis=-1)).max())
    check = {"o_rel": o_rel}
    if (t_next + 1) % wl.reassign_interval != 0:   # scores of the same tokens on both sides
        n16, n8 = int(c.n_bf16[rid]), int(c.n_fp8[rid])
        pos2 = np.concatenate([c.pos16[rid, :n16].cpu().numpy(), c.pos8[rid, :n8].cpu().numpy()]).astype(np.int64)
        o2 = np.argsort(pos2, kind="stable")
        mu = np.concatenate([c.mu16[rid, :n16].cpu().numpy(), c.mu8[rid, :n8].cpu().numpy()])[o2]
        m2 = np.concatenate([c.m2_16[rid, :n16].cpu().numpy(), c.m2_8[rid, :n8].cpu().numpy()])[o2]
        same = np.array_equal(pos2[o2], row.pos)
        check["positions_equal"] = bool(same)
        if same:
            s_ref = A.heavy_hitter_score(row.mu, row.m2, row.cnt, wl.gamma)
            s_gpu = A.heavy_hitter_score(mu, m2, row.cnt, wl.gamma)
            check["s_rel"] = float(np.max(np.abs(s_gpu - s_ref) / (np.abs(s_ref) + 1e-300)))
    check["tolerance"] = {"o_rel": 2e-3, "s_rel": 1e-5}
    check["ok"] = bool(o_rel <= 2e-3 and check.get("s_rel", 0.0) <= 1e-5 and check.get("positions_equal", True))

    def timed_steps(t, budget):
        per = [first] if t == t_next + 1 else []
        spent = sum(per)
        while len(per) < wl.reassign_interval or spent < budget:
            a = time.perf_counter()
            oracle_step(t)
            per.append(time.perf_counter() - a)
            spent += per[-1]
            t += 1
        return per, t

    all_threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    per_all, t = timed_steps(t_next + 1, seconds / 2)
    with threadpool_limits(limits=1):
        per_one, t = timed_steps(t, seconds / 2)
    scale = wl.rows * wl.layers                       # row-steps in one decode step of the stack
    v_all = wl.batch / (statistics.mean(per_all) * scale)
    v_one = wl.batch / (statistics.mean(per_one) * scale)
    return {"value": v_all, "unit": "tokens/s", "cores": all_threads, "nproc": os.cpu_count(),
            "kind": "oracle",
            "single_thread": {"value": v_one, "unit": "tokens/s", "cores": 1},
            "sample": (f"oracle on row 0 of layer 0 ({wl.name}) from the benchmarked device state after "
                       f"{t_next} decode steps: {len(per_all)} steps on {all_threads} threads, then "
                       f"{len(per_one)} on 1 thread, reassignments every {wl.reassign_interval}; time per "
                       f"row-step scaled to {wl.layers} layers x {wl.rows} rows (extrapolated)"),
            "extrapolated": True,
            "check_on_benchmarked_state": check}


def run_reference(args, wl, rank):
    if rank != 0:
        return
    smp = OracleSampler(wl)
    per = []
    for i in range(args.warmup + args.steps):
        x = smp.step()
        if i >= args.warmup:
            per.append(x)
    step_s = statistics.mean(per) * wl.rows * wl.layers
    value = wl.batch / step_s
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": step_s * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_of(wl),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": smp.threads,
                             "nproc": os.cpu_count(), "kind": "oracle", "sample": smp.describe(len(per)),
                             "extrapolated": True},
            "extrapolated": True,
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def config_of(wl, streams=5, early=None):
    return {"workload": wl.name, "layers": wl.layers, "batch": wl.batch, "hq": wl.hq, "hkv": wl.hkv,
            "head_dim": wl.head_dim, "n_ctx": wl.n_ctx, "n_ctx_min": wl.n_ctx_min,
            "budget_frac": wl.budget_frac, "oq_ratio": wl.oq_ratio if wl.oq_ratio is not None
            else f"per layer from prefill stats (r_bar {wl.r_bar})", "window": wl.window,
            "gamma": wl.gamma, "reassign_interval": wl.reassign_interval, "quant_format": wl.quant_format,
            "streams": (f"score update and reassignment on {streams - 1} side stream(s), layers round robin"
                        if streams >= 2 else "one stream"),
            "l2": "no flush: every step streams the whole compressed cache, far above L2",
            "early_start": (wl.layers >= 3) if early is None else bool(early)}


# ------------------------------------------------------------------ GPU arm
def run_arkv(args, wl, rank, world, local_rank):
    import numpy as np
    import torch
    import torch.distributed as dist
    from mixed_precision_kv_arkv_b200 import abi, build, inputs
    from mixed_precision_kv_arkv_b200.cache import LayerCache, Workspace, make_cfg, stream_ptr

    build.build()
    abi.lib()
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    s = stream_ptr()
    L, B, Hq, Hkv, D = wl.layers, wl.batch, wl.hq, wl.hkv, wl.head_dim
    K, W = args.steps, args.warmup
    passes = 1 + (0 if args.no_e2e else 1) + 1          # value, e2e, per-call kernel timing
    total_steps = W + passes * K
    ctx_np = inputs.ctx_lengths(wl, 0)
    n_max = int(ctx_np.max()) + total_steps + 1        # + the step the CPU baseline checks
    ctx = torch.from_numpy(ctx_np).to(dev)

    # ---------- prefill statistics of every layer, then the per-layer Original share
    probe = make_cfg(B, Hq, Hkv, D, wl.window, wl.n_obs, wl.gamma, wl.budget_frac, 1, 1, wl.quant_format)
    # consecutive attention calls on the main stream belong to different layers, so with
    # three or more layers each may read its cache before the previous kernel ends
    early = L >= 3 and not args.no_early_start
    ws_pre = Workspace(abi.arkv_workspace_bytes(probe, abi.ARKV_WS_PREFILL, wl.n_ctx), dev)
    stats = torch.zeros((L, 3), dtype=torch.float64, device=dev)
    mu0 = torch.zeros((wl.rows, wl.n_ctx), dtype=torch.float64, device=dev)
    m20 = torch.zeros_like(mu0)
    seed = rank
    for l in range(L):
        pre = inputs.layer_prefill_torch(wl, l, dev, seed, ctx_np)
        abi.arkv_prefill_stats(probe, pre["q_obs"].data_ptr(), pre["k"].data_ptr(), wl.n_ctx,
                               ctx.data_ptr(), stats[l].data_ptr(), None, mu0.data_ptr(),
                               m20.data_ptr(), ws_pre.ptr, ws_pre.nbytes, s)
        del pre
    st_host = stats.cpu().numpy()
    if wl.oq_ratio is not None:
        r = np.full(L, wl.oq_ratio, np.float32)
    else:
        r = np.zeros(L, np.float32)
        abi.arkv_oq_ratio(st_host.ctypes.data, L, wl.r_bar, r.ctypes.data)

    # ---------- per-layer caches: capacities, initial pack
    layers = []
    for l in range(L):
        # K slots beyond the workload's need: the pipelined kernel pass appends K tokens
        # with no reassignment between (its appends are rolled back afterwards)
        cap_o, cap_q = abi.arkv_row_capacity(probe, n_max, float(r[l]), wl.reassign_interval + K)
        cfg = make_cfg(B, Hq, Hkv, D, wl.window, wl.n_obs, wl.gamma, wl.budget_frac, cap_o, cap_q,
                       wl.quant_format, early_start=early)
        cache = LayerCache(cfg, dev)
        pre = inputs.layer_prefill_torch(wl, l, dev, seed, ctx_np)
        abi.arkv_prefill_stats(cfg, pre["q_obs"].data_ptr(), pre["k"].data_ptr(), wl.n_ctx,
                               ctx.data_ptr(), stats[l].data_ptr(), None, mu0.data_ptr(),
                               m20.data_ptr(), ws_pre.ptr, ws_pre.nbytes, s)
        abi.arkv_quantize_pack(cfg, float(r[l]), pre["k"].data_ptr(), pre["v"].data_ptr(), wl.n_ctx,
                               ctx.data_ptr(), mu0.data_ptr(), m20.data_ptr(), cache.c, None,
                               ws_pre.ptr, ws_pre.nbytes, s)
        dec = inputs.decode_inputs_torch(wl, pre["u"], total_steps + 1, dev, seed, l)
        layers.append({"cfg": cfg, "cache": cache, "r": float(r[l]), "dec": dec,
                       "ws_d": Workspace(abi.arkv_workspace_bytes(cfg, abi.ARKV_WS_DECODE), dev),
                       "ws_r": Workspace(abi.arkv_workspace_bytes(cfg, abi.ARKV_WS_REASSIGN), dev)})
        del pre
    del ws_pre, mu0, m20
    torch.cuda.synchronize()
    status = sum(int(x["cache"].status.item()) for x in layers)
    assert status == 0, f"cache status {status} after pack"
    o = torch.zeros((L, B, Hq, D), dtype=torch.float32, device=dev)
    launches = {"n": 0}

    # The score update and reassignment of layer l run on side stream l mod (S - 1): the
    # next layer's attention does not wait for them (in a model, the next layer's query
    # needs only this layer's output), and the reassignments of a reassignment step, one
    # row per CTA, run side by side on several streams instead of one after another.
    # The next call on layer l's cache waits for them.
    sides = [torch.cuda.Stream(device=dev) for _ in range(max(args.streams - 1, 0))]
    pending = {}                                             # layer -> event after its side work

    def settle(l):
        ev_done = pending.pop(l, None)
        if ev_done is not None:
            torch.cuda.current_stream().wait_event(ev_done)

    def join():
        for l in list(pending):
            settle(l)

    def layer_step(l, t, q=None, kn=None, vn=None, ev=None):
        x = layers[l]
        cfg, c = x["cfg"], x["cache"].c
        q = x["dec"]["q"][t] if q is None else q
        kn = x["dec"]["k_new"][t] if kn is None else kn
        vn = x["dec"]["v_new"][t] if vn is None else vn
        settle(l)
        main = torch.cuda.current_stream()
        if ev is not None:
            ev[0].record(main)
        abi.arkv_decode_attn(cfg, t, q.data_ptr(), kn.data_ptr(), vn.data_ptr(), ctx.data_ptr(), c,
                             o[l].data_ptr(), x["ws_d"].ptr, x["ws_d"].nbytes, main.cuda_stream)
        if ev is not None:
            ev[1].record(main)
        side = sides[l % len(sides)] if sides else None
        aux = side if side is not None else main
        if side is not None:
            attended = torch.cuda.Event()
            attended.record(main)
            side.wait_event(attended)
        abi.arkv_score_update(cfg, t, ctx.data_ptr(), c, x["ws_d"].ptr, x["ws_d"].nbytes, aux.cuda_stream)
        launches["n"] += KERNELS_PER_LAYER_STEP
        if (t + 1) % wl.reassign_interval == 0:
            abi.arkv_reassign(cfg, t, x["r"], ctx.data_ptr(), c, None, x["ws_r"].ptr, x["ws_r"].nbytes,
                              aux.cuda_stream)
            launches["n"] += 1
        if side is not None:
            done = torch.cuda.Event()
            done.record(side)
            pending[l] = done

    for t in range(W):                                       # warm-up, eager
        for l in range(L):
            layer_step(l, t)
    join()
    torch.cuda.synchronize()

    def capture(t0, nsteps, body):
        graphs, t = [], t0
        while t < t0 + nsteps:
            n = min(wl.reassign_interval - (t % wl.reassign_interval), t0 + nsteps - t)
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                for tt in range(t, t + n):
                    body(tt)
                join()                                       # the side stream rejoins the capture
            graphs.append(g)
            t += n
        return graphs

    # ---------- pass 1: device-timed value
    t_value = W
    g_value = capture(t_value, K, lambda tt: [layer_step(l, tt) for l in range(L)])
    launches["n"] = 0
    for tt in range(t_value, t_value + K):
        for l in range(L):
            launches["n"] += KERNELS_PER_LAYER_STEP + (1 if (tt + 1) % wl.reassign_interval == 0 else 0)
    gpu_launches = launches["n"]

    # ---------- pass 2: end to end through host buffers
    t_e2e = W + K
    h2d = d2h = 0
    if not args.no_e2e:
        qh = torch.stack([x["dec"]["q"][t_e2e:t_e2e + K] for x in layers], 1).cpu().pin_memory()
        kh = torch.stack([x["dec"]["k_new"][t_e2e:t_e2e + K] for x in layers], 1).cpu().pin_memory()
        vh = torch.stack([x["dec"]["v_new"][t_e2e:t_e2e + K] for x in layers], 1).cpu().pin_memory()
        oh = torch.empty((K, L, B, Hq, D), dtype=torch.float32).pin_memory()
        qd, kd, vd = (torch.empty_like(qh[0], device=dev), torch.empty_like(kh[0], device=dev),
                      torch.empty_like(vh[0], device=dev))
        h2d = qh[0].numel() * 2 + kh[0].numel() * 2 + vh[0].numel() * 2
        d2h = oh[0].numel() * 4

        # the host transfers go through arkv_copy_async (a kernel reading and writing the
        # page-locked buffers), so the captured step has no copy-engine node between its
        # kernels; one call per buffer before the capture checks each buffer.  One copy per
        # buffer and direction per step, on the main stream: per-layer copies on side
        # streams were slower, because the attention calls then wait on events between
        # them and lose their programmatic early launch
        def transfers(i):
            st = torch.cuda.current_stream().cuda_stream
            for dd, hh in ((qd, qh[i]), (kd, kh[i]), (vd, vh[i])):
                abi.arkv_copy_async(dd.data_ptr(), hh.data_ptr(), dd.numel() * dd.element_size(), st)

        def result(i):
            abi.arkv_copy_async(oh[i].data_ptr(), o.data_ptr(), o.numel() * o.element_size(),
                                torch.cuda.current_stream().cuda_stream)
        for i in range(K):
            transfers(i)
            result(i)
        torch.cuda.synchronize()

        def e2e_body(tt):
            i = tt - t_e2e
            transfers(i)
            for l in range(L):
                layer_step(l, tt, qd[l], kd[l], vd[l])
            result(i)
        g_e2e = capture(t_e2e, K, e2e_body)

    # ---------- pass 3: the decode kernel timed by events on its stream
    t_k = W + (passes - 1) * K
    evs = [(torch.cuda.Event(enable_timing=True, external=True),
            torch.cuda.Event(enable_timing=True, external=True)) for _ in range(K * L)]
    counts = torch.zeros((K, L, 2, wl.rows), dtype=torch.int32, device=dev)

    def k_body(tt):
        i = tt - t_k
        for l in range(L):
            settle(l)
            counts[i, l, 0].copy_(layers[l]["cache"].n_bf16)
            counts[i, l, 1].copy_(layers[l]["cache"].n_fp8)
            layer_step(l, tt, ev=evs[i * L + l])
    g_k = capture(t_k, K, k_body)

    # ---------- pass 4: the attention calls alone, K steps of L back-to-back launches on
    # one stream (each may overlap the tail of the one before it), timed as a whole;
    # replayed on the state pass 3 leaves, and rolled back afterwards (n_bf16 restored)
    def pipe_body(tt):
        for l in range(L):
            x = layers[l]
            abi.arkv_decode_attn(x["cfg"], tt, x["dec"]["q"][tt].data_ptr(), x["dec"]["k_new"][tt].data_ptr(),
                                 x["dec"]["v_new"][tt].data_ptr(), ctx.data_ptr(), x["cache"].c,
                                 o[l].data_ptr(), x["ws_d"].ptr, x["ws_d"].nbytes,
                                 torch.cuda.current_stream().cuda_stream)
    g_pipe = capture(t_k, K, pipe_body)

    def timed(graphs):
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for g in graphs:
            g.replay()
        b.record()
        torch.cuda.synchronize()
        return max_over_ranks(a.elapsed_time(b), dev, world)

    with ClockSampler(local_rank) as clk:
        ms_value = timed(g_value)
        ms_e2e = timed(g_e2e) if not args.no_e2e else None
        # the last step's outputs, as copied to host memory, against the device buffer
        # they were copied from (no pass has written it since)
        e2e_copied = bool(torch.equal(oh[K - 1], o.cpu())) if not args.no_e2e else None
        timed(g_k)
        join()
        saved = [(x["cache"].n_bf16.clone(), x["cache"].n_fp8.clone()) for x in layers]
        torch.cuda.synchronize()
        ms_pipe = timed(g_pipe)
        for x, (n16, n8) in zip(layers, saved):
            x["cache"].n_bf16.copy_(n16)
    torch.cuda.synchronize()
    outputs_finite = bool(torch.isfinite(o).all())            # every layer's output of the last step
    clocks = clk.summary()
    clocks["window"] = "sampled every 50 ms across the four timed passes"
    io_bytes = B * Hq * D * 2 + B * Hq * D * 4 + 2 * B * Hkv * D * 2
    # per-call timing (pass 3): events around each launch inside the full step
    k1_ms = [a.elapsed_time(b) for a, b in evs]
    cn = counts.cpu().numpy().astype(np.int64)               # [K, L, 2, rows] before each launch
    per_row = (cn[:, :, 0] + 1) * 4 * D + cn[:, :, 1] * (2 * D + 8)
    alg_bytes = per_row.sum(-1) + io_bytes                   # [K, L]
    achieved_iso = float(alg_bytes.sum() / (sum(k1_ms) * 1e-3) / 1e9)
    # pipelined timing (pass 4): launch i of layer l sees n_bf16 = saved + i
    n16_0 = np.stack([n16.cpu().numpy() for n16, _ in saved]).astype(np.int64)      # [L, rows]
    n8_0 = np.stack([n8.cpu().numpy() for _, n8 in saved]).astype(np.int64)
    steps_i = np.arange(K, dtype=np.int64)[:, None, None]
    pipe_row = (n16_0[None] + steps_i + 1) * 4 * D + n8_0[None] * (2 * D + 8)       # [K, L, rows]
    pipe_bytes = pipe_row.sum(-1) + io_bytes
    ms_per_pipe = ms_pipe / (K * L)
    achieved = float(pipe_bytes.sum() / (ms_pipe * 1e-3) / 1e9)
    peak, peak_kind = hbm_peak()
    step_bytes = float(alg_bytes.sum(-1).mean())

    status = sum(int(x["cache"].status.item()) for x in layers)
    value = job_tokens_per_s(B, K, world, ms_value)
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": K,
        "warmup": W, "ms_per_step": ms_value / K, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic", "config": config_of(wl, args.streams, early),
        "hbm_gbs_step": step_bytes / (ms_value / K * 1e-3) / 1e9,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": kernel_traffic("decode_attn.cu"),
                     "kernel": f"arkv_decode_attn call: decode_attn_kernel<{D}> (split merge fused)",
                     "peak_source": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs)" if peak_kind == "measured"
                     else "fallback 6650 GB/s",
                     "timing": f"CUDA events around {K} x {L} back-to-back launches on one stream "
                               f"(early_start={int(early)}), per-launch mean",
                     "bytes_per_launch": float(pipe_bytes.mean()),
                     "ms_per_launch": ms_per_pipe,
                     "isolated": {"timing": "CUDA events around each launch inside the full step "
                                            "(score updates on the side stream running beside it)",
                                  "achieved": achieved_iso, "frac": achieved_iso / peak,
                                  "bytes_per_launch": float(alg_bytes.mean()),
                                  "ms_per_launch": statistics.mean(k1_ms)}},
        "gpu_launches": gpu_launches,
        "clocks": clocks,
        "oq_ratio_per_layer": [round(float(x), 4) for x in r],
        "cache_status": status,
        "outputs_finite": outputs_finite,
    }
    if not args.no_e2e:
        line["e2e"] = {"value": job_tokens_per_s(B, K, world, ms_e2e), "unit": "tokens/s",
                       "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                       "ms_per_step": ms_e2e / K,
                       "transfers": "arkv_copy_async, one per buffer and direction per step, on the "
                                    "attention stream",
                       "outputs_copied": e2e_copied}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline_from_state(wl, layers[0], ctx_np, total_steps, o, args.cpu_seconds,
                                                       lambda t: (layer_step(0, t), join()))
    if rank == 0:
        print(json.dumps(line), flush=True)
    del g_value, g_k, g_pipe
    if not args.no_e2e:
        del g_e2e


def main():
    args = parse()
    wl = workloads.BY_NAME[args.workload]
    if args.layers is not None:
        wl = wl.with_(layers=args.layers)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, wl, rank)
        return
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    try:
        run_arkv(args, wl, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.barrier()
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
