"""Benchmark of the fused KV-cache step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload single_bf16|verify_bf16|long_bf16|batch_bf16]

Prints ONE JSON line on rank 0.  A step is one pass of the whole hot path over
one batch of synthetic input: for a fused-step workload the projection/RoPE/
cache-scatter kernel then the full-cache attention; for the verify workload
the verify pass plus the acceptance reduction.  Inputs are resident in HBM
when the timed region starts; L2 is flushed (a 512 MB write) before every
timed step, and each step is timed with CUDA events on the launching stream.
Under torchrun every rank runs its own sequences (weak scaling, no data-path
collective); the time is the max over ranks.

--impl reference times the fp64 CPU oracle (the only reference this method
has) on the host cores, on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import workloads as W  # noqa: E402

L2_FLUSH_BYTES = 512 << 20
DEFAULT_WORKLOAD = "batch_bf16"
SWEEP_BATCHES = (1, 2, 4, 8, 16, 32, 64)
FALLBACK_HBM_GBS = 6650.0
NOMINAL_HBM_GBS = 8000.0  # B200 HBM3e, nominal


# ------------------------------------------------------------------ helpers

def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def workload_desc(name, cfg):
    if cfg["kind"] == "fused":
        return (f"{name}: fused step B={cfg['B']} N={cfg['N']} D={cfg['D']} H={cfg['H']} "
                f"dh={cfg['dh']} |Q|={cfg['n_track'] + cfg['beta_m']} ({cfg['n_track']} tracked + "
                f"{cfg['beta_m']} front masks) {cfg['dtype']}")
    R = cfg["n_tv"] + 2 * cfg["n_s"]
    return (f"{name}: verify pass + acceptance B={cfg['B']} N={cfg['N']} D={cfg['D']} "
            f"H={cfg['H']} dh={cfg['dh']} R={R} ({cfg['n_tv']} T_v + {cfg['n_s']} draft + "
            f"{cfg['n_s']} mask rows) V={cfg['vocab']} {cfg['dtype']}")


def workload_with_overrides(args):
    """The named workload, with --batch / --seq-len applied (name suffixed)."""
    cfg = dict(W.CONFIGS[args.workload])
    name = args.workload
    if args.batch is not None:
        cfg["B"] = args.batch
        name += f"@B{args.batch}"
    if args.seq_len is not None:
        gen = cfg["N"] - cfg["n_prompt"]
        if args.seq_len <= gen:
            gen = args.seq_len // 2
        cfg["N"], cfg["n_prompt"] = args.seq_len, args.seq_len - gen
        name += f"@N{args.seq_len}"
    return cfg, name


def bench_config(name, cfg, world):
    """The workload a line measures; the same dict in both arms of the bench."""
    return {"workload": workload_desc(name, cfg),
            "l2": "GPU arm: flushed before every timed step (512 MB write); host arm: n/a",
            "parallelism": f"replicas x{world} (sequences sharded over ranks, no collective)"}


def algorithmic_bytes(cfg):
    """Bytes each kernel must move at least (per launch), by its definition.

    projection: W_qkv + the gathered rows x[Q] + new k, v written to the cache
                + rotated q written for the attention;
    attention:  the whole K, V cache of every sequence (plus side slots)
                + q read + output written;
    accept:     the logits."""
    e = 2 if cfg["dtype"] == "bf16" else 4
    B, N, D, H, dh = cfg["B"], cfg["N"], cfg["D"], cfg["H"], cfg["dh"]
    E = H * dh
    rows = cfg["n_track"] + cfg["beta_m"] if cfg["kind"] == "fused" else cfg["n_tv"] + 2 * cfg["n_s"]
    M = B * rows
    side = B * H * cfg.get("n_s", 0) * dh * e * 2 if cfg["kind"] == "verify" else 0
    proj = 3 * E * D * e + M * D * e + 2 * M * E * e + M * E * e
    attn = 2 * B * H * N * dh * e + side + M * E * e + M * E * e
    out = {"proj": proj, "attn": attn}
    if cfg["kind"] == "verify":
        out["accept"] = M * cfg["vocab"] * 4
    return out, rows


L2_BYTES = 126 * 1024 * 1024


def resident_bytes(cfg):
    """W_qkv and the K, V caches: the state every step reads from HBM."""
    e = 2 if cfg["dtype"] == "bf16" else 4
    B, N, D, H, dh = cfg["B"], cfg["N"], cfg["D"], cfg["H"], cfg["dh"]
    return 3 * H * dh * D * e + 2 * B * H * N * dh * e


def step_bytes_min(cfg):
    """Bytes one whole step must move at least, by the method's definition: W_qkv,
    the rows x[Q], the K, V of the cache slots the step does not write, the new
    k, v (cache and side slots), the side slots read back, and the output (plus
    the logits for a verify pass and its acceptance).  Unlike the per-kernel sum,
    it counts neither the rotated q staged between the two kernels nor the
    attention's re-read of the slots just written."""
    e = 2 if cfg["dtype"] == "bf16" else 4
    B, N, D, H, dh = cfg["B"], cfg["N"], cfg["D"], cfg["H"], cfg["dh"]
    E = H * dh
    if cfg["kind"] == "fused":
        rows = cfg["n_track"] + cfg["beta_m"]
        cache_rows, side_rows = rows, 0
    else:
        rows = cfg["n_tv"] + 2 * cfg["n_s"]
        cache_rows, side_rows = cfg["n_tv"] + cfg["n_s"], cfg["n_s"]
    M = B * rows
    total = (3 * E * D * e + M * D * e + 2 * B * H * (N - cache_rows) * dh * e
             + 2 * M * E * e + 2 * B * side_rows * E * e + M * E * e)
    if cfg["kind"] == "verify":
        total += M * cfg["vocab"] * 4
    return total


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while running."""
    NAMES = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
             0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, device_index):
        self.samples = []
        self.ok = False
        self.max_mhz = None
        try:
            import pynvml
            pynvml.nvmlInit()
            h = None
            try:
                uuid = str(torch.cuda.get_device_properties(device_index).uuid)
                if not uuid.startswith("GPU-"):
                    uuid = "GPU-" + uuid
                h = pynvml.nvmlDeviceGetHandleByUUID(uuid)
            except Exception:
                h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.h, self.nv = h, pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
            self.reasons_fn = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                getattr(pynvml, "nvmlDeviceGetCurrentClocksThrottleReasons")
            self.ok = True
        except Exception as e:  # no NVML: report it
            self.err = repr(e)
        self._stop = threading.Event()

    def _run(self):
        while not self._stop.is_set():
            try:
                mhz = self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM)
                rs = self.reasons_fn(self.h)
                self.samples.append((time.perf_counter(), mhz, rs))
            except Exception:
                pass
            time.sleep(0.002)

    def start(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()

    def stop(self):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self, t0, t1):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "note": "NVML unavailable"}
        inside = [s for s in self.samples if t0 <= s[0] <= t1] or self.samples[-3:]
        mhz = [s[1] for s in inside]
        bits = 0
        for s in inside:
            bits |= int(s[2])
        return {"sm_mhz": statistics.median(mhz) if mhz else None, "sm_max_mhz": self.max_mhz,
                "reasons": sorted(n for b, n in self.NAMES.items() if bits & b),
                "samples": len(inside)}


def traffic_for(kernel_key):
    """Per-launch DRAM bytes of a kernel from a committed ncu summary, or None when
    the summary is missing or the kernel source changed since the capture."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p)).get(kernel_key)
    if not d:
        return None
    src = os.path.join(ROOT, d["source"])
    if not os.path.exists(src):
        return None
    h = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    return d["bytes_per_launch"] if h == d["source_sha256_16"] else None


# ------------------------------------------------------------------ our arm

def run_ours(args, world, rank, local, cfg=None, name=None, with_e2e=True):
    import kv_cache_attention_fdllm_b200 as F
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    name = name or args.workload
    cfg = cfg or W.CONFIGS[args.workload]
    B = cfg["B"]
    seqs = F.rank_sequences(B, rank)  # each rank owns its own sequences
    rope_base = cfg["rope_base"]
    verify = cfg["kind"] == "verify"
    if verify:
        host = W.verify_inputs(cfg, seqs=seqs)
        acc = W.accept_inputs(cfg, seqs=seqs)
    else:
        host = W.fused_inputs(cfg, seqs=seqs)
    d = W.to_device(host, dev)
    dt = d["w_qkv"].dtype
    H, dh, N, D = cfg["H"], cfg["dh"], cfg["N"], cfg["D"]
    if verify:
        R = cfg["n_tv"] + 2 * cfg["n_s"]
        S_max = cfg["n_s"]
        ws = F.alloc_workspace(F.fdllm_verify_step_workspace_bytes(B, N, D, H, dh, R, S_max, dt), dev)
        q = torch.empty((B, R, H, dh), dtype=dt, device=dev)
        out = torch.empty((B, R, H * dh), dtype=dt, device=dev)
        ad = W.to_device(acc, dev)
        V = cfg["vocab"]
        ws_a = F.alloc_workspace(F.fdllm_accept_workspace_bytes(B, R, V), dev)
        top1 = torch.empty((B, R), dtype=torch.int32, device=dev)
        conf = torch.empty((B, R), dtype=torch.float32, device=dev)
        flags = torch.empty((B, R), dtype=torch.uint8, device=dev)
        n_acc = torch.empty((B,), dtype=torch.int32, device=dev)
        rows = R
    else:
        nq = cfg["n_track"] + cfg["beta_m"]
        ws = F.alloc_workspace(F.fdllm_fused_step_workspace_bytes(B, N, D, H, dh, nq, dt), dev)
        q = torch.empty((B, nq, H, dh), dtype=dt, device=dev)
        out = torch.empty((B, nq, H * dh), dtype=dt, device=dev)
        rows = nq

    def stage_proj():
        if verify:
            F.fdllm_verify_qkv_rope_scatter(d["x_rows"], d["pos"], d["view"], d["w_qkv"],
                                            d["k_cache"], d["v_cache"], d["k_side"], d["v_side"],
                                            q, ws, rope_base=rope_base)
        else:
            F.fdllm_qkv_rope_scatter(d["x"], d["q_idx"], d["w_qkv"], d["k_cache"], d["v_cache"], q,
                                     ws, rope_base=rope_base)

    def stage_attn():
        if verify:
            F.fdllm_verify_attend(q, d["pos"], d["view"], d["rank"], d["k_cache"], d["v_cache"],
                                  d["k_side"], d["v_side"], out, ws)
        else:
            F.fdllm_attend(q, d["k_cache"], d["v_cache"], out, ws)

    def stage_accept():
        F.fdllm_accept(ad["logits"], ad["kind"], ad["ref_tok"], ad["rank"], top1, conf, flags,
                       n_acc, ws_a, eps=0.9, gamma=0.8)

    stages = [("proj", stage_proj), ("attn", stage_attn)] + ([("accept", stage_accept)] if verify else [])
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def full_step():
        # the public calls a user makes: one fused step (or verify pass + acceptance),
        # whose kernels overlap through programmatic dependent launch
        if verify:
            F.fdllm_verify_step(d["x_rows"], d["pos"], d["view"], d["rank"], d["w_qkv"],
                                d["k_cache"], d["v_cache"], d["k_side"], d["v_side"], out, ws,
                                rope_base=rope_base)
            stage_accept()
        else:
            F.fdllm_fused_step(d["x"], d["q_idx"], d["w_qkv"], d["k_cache"], d["v_cache"], out, ws,
                               rope_base=rope_base)

    def one_step(evs):
        # the same kernels one stage at a time, an event between stages
        evs[0].record()
        for i, (_, fn) in enumerate(stages):
            fn()
            evs[i + 1].record()

    # warm-up (untimed)
    for _ in range(args.warmup):
        flush.fill_(1)
        full_step()
        flush.fill_(1)
        one_step([torch.cuda.Event(enable_timing=True) for _ in range(len(stages) + 1)])
    torch.cuda.synchronize()
    if F.fdllm_get_status(ws) != F.OK:
        raise RuntimeError("device status set during warm-up")

    step_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(args.steps)]
    sampler = ClockSampler(dev.index)
    sampler.start()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    launches0 = F.lib().fdllm_launch_count()
    t0 = time.perf_counter()
    # a long write first lets the host queue the timed steps ahead of the GPU
    torch.empty(4 * L2_FLUSH_BYTES, dtype=torch.uint8, device=dev).fill_(0)
    for k in range(args.steps):
        flush.fill_(k & 0xff)
        step_ev[k][0].record()
        full_step()
        step_ev[k][1].record()
    torch.cuda.synchronize()
    t1 = time.perf_counter()
    launches = F.lib().fdllm_launch_count() - launches0
    if world > 1:
        torch.distributed.barrier()
    sampler.stop()
    step_ms = [a.elapsed_time(b) for a, b in step_ev]

    # per-stage times (roofline of the dominant kernel), in a pass of their own
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(len(stages) + 1)]
           for _ in range(args.steps)]
    for k in range(args.steps):
        flush.fill_(k & 0xff)
        one_step(evs[k])
    torch.cuda.synchronize()
    if F.fdllm_get_status(ws) != F.OK:
        raise RuntimeError("device status set during the timed steps")
    stage_ms = {name: [evs[k][i].elapsed_time(evs[k][i + 1]) for k in range(args.steps)]
                for i, (name, _) in enumerate(stages)}
    mean_step = F.max_over_ranks(sum(step_ms) / len(step_ms), dev)
    tokens_per_step = B * rows * world

    # ---------------- end to end through the public call with host buffers: every
    # step copies its inputs from pinned host memory (the rows the step reads and
    # their indices; for a verify pass also its metadata and the logits) and reads
    # its results back; W and the caches are the resident state the step updates
    e2e = None
    if with_e2e:
        nbytes = lambda ts: int(sum(t.numel() * t.element_size() for t in ts))  # noqa: E731
        ws_e = F.alloc_workspace(ws.numel(), dev)
        if verify:
            hin = {k: host[k] for k in ("x_rows", "pos", "view", "rank")}
            hin.update({"logits": acc["logits"], "kind": acc["kind"], "ref_tok": acc["ref_tok"]})
            ws_ea = F.alloc_workspace(ws_a.numel(), dev)
            outs = [out, top1, conf, flags, n_acc]
        else:
            # x[Q]: row i of sequence b is x[b, q_idx[b, i]], gathered once on the host
            qi = host["q_idx"].long()
            hin = {"x_rows": torch.stack([host["x"][b, qi[b]] for b in range(B)]).contiguous(),
                   "q_idx": host["q_idx"]}
            outs = [out]
        pin = {k: v.pin_memory() for k, v in hin.items()}
        dbuf = {k: torch.empty(v.shape, dtype=v.dtype, device=dev) for k, v in pin.items()}
        outs_h = [torch.empty(o.shape, dtype=o.dtype).pin_memory() for o in outs]

        def e2e_call(dbuf, outs, stream):
            # the public calls of one step on `stream`, from the device copies of its inputs
            if verify:
                o, tp, cf, fl, na = outs
                F.fdllm_verify_step(dbuf["x_rows"], dbuf["pos"], dbuf["view"], dbuf["rank"],
                                    d["w_qkv"], d["k_cache"], d["v_cache"], d["k_side"],
                                    d["v_side"], o, ws_e, rope_base=rope_base, stream=stream)
                F.fdllm_accept(dbuf["logits"], dbuf["kind"], dbuf["ref_tok"], dbuf["rank"], tp,
                               cf, fl, na, ws_ea, eps=0.9, gamma=0.8, stream=stream)
            else:
                F.fdllm_fused_step_rows(dbuf["x_rows"], dbuf["q_idx"], d["w_qkv"], d["k_cache"],
                                        d["v_cache"], outs[0], ws_e, rope_base=rope_base,
                                        stream=stream)

        n_e2e = max(3, args.steps // 4)
        # When the resident state (W and the caches) exceeds L2 the steps need no
        # flush between them, and they run as a pipeline: step k+1's inputs go up
        # and step k-1's results come back on two copy streams while step k
        # computes, with two sets of device buffers.  Every step's copies stay
        # inside the timed region.  Otherwise each step is timed alone, after an
        # L2 flush outside its events.
        pipelined = resident_bytes(cfg) > L2_BYTES
        if pipelined:
            dbufs = [dbuf, {k: torch.empty_like(v) for k, v in dbuf.items()}]
            outs2 = [outs, [torch.empty_like(o) for o in outs]]
            outs_h2 = [outs_h, [torch.empty(o.shape, dtype=o.dtype).pin_memory() for o in outs]]
            s_c = torch.cuda.current_stream(dev)
            s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)

            def e2e_run(nsteps, start=None):
                ev_in = [torch.cuda.Event() for _ in range(nsteps)]
                ev_c = [torch.cuda.Event() for _ in range(nsteps)]
                ev_out = [torch.cuda.Event() for _ in range(nsteps)]
                if start is not None:
                    start.record(s_c)
                s_in.wait_stream(s_c)
                s_out.wait_stream(s_c)
                for k in range(nsteps):
                    b = k % 2
                    with torch.cuda.stream(s_in):
                        if k >= 2:
                            s_in.wait_event(ev_c[k - 2])  # buffer set b is read by step k-2
                        for key in pin:
                            dbufs[b][key].copy_(pin[key], non_blocking=True)
                        ev_in[k].record(s_in)
                    s_c.wait_event(ev_in[k])
                    if k >= 2:
                        s_c.wait_event(ev_out[k - 2])  # output set b is read back by step k-2
                    e2e_call(dbufs[b], outs2[b], s_c)
                    ev_c[k].record(s_c)
                    with torch.cuda.stream(s_out):
                        s_out.wait_event(ev_c[k])
                        for oh, o in zip(outs_h2[b], outs2[b]):
                            oh.copy_(o, non_blocking=True)
                        ev_out[k].record(s_out)
                s_c.wait_stream(s_in)
                s_c.wait_stream(s_out)

            e2e_run(args.warmup)
            torch.cuda.synchronize()
            if world > 1:
                torch.distributed.barrier()
            ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e2e_run(n_e2e, start=ev0)
            ev1.record(s_c)
            torch.cuda.synchronize()
            e2e_ms = F.max_over_ranks(ev0.elapsed_time(ev1) / n_e2e, dev)
        else:
            e2e_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                      for _ in range(n_e2e)]
            for i in range(args.warmup + len(e2e_ev)):
                flush.fill_(2)
                ev = e2e_ev[i - args.warmup] if i >= args.warmup else None
                if ev:
                    ev[0].record()
                for k in pin:
                    dbuf[k].copy_(pin[k], non_blocking=True)
                e2e_call(dbuf, outs, None)
                for oh, o in zip(outs_h, outs):
                    oh.copy_(o, non_blocking=True)
                if ev:
                    ev[1].record()
            torch.cuda.synchronize()
            e2e_ms = F.max_over_ranks(sum(a.elapsed_time(b) for a, b in e2e_ev) / len(e2e_ev), dev)
        e2e = {"value": tokens_per_step / (e2e_ms / 1e3),
               "unit": "query-tokens/s" if not verify else "query-rows/s",
               "h2d_bytes_per_step": nbytes(pin.values()),
               "d2h_bytes_per_step": nbytes(outs_h),
               "ms_per_step": e2e_ms,
               "pipelined": pipelined,
               "l2": ("resident W and caches exceed L2: no flush; the steps overlap their copies "
                      "with the neighbouring steps' compute") if pipelined else
                     "flushed before every step, outside its events",
               "path": ("pinned host x_rows, pos, view, rank, logits, kind, ref_tok -> "
                        "fdllm_verify_step + fdllm_accept -> pinned host out, top1, conf, flags, "
                        "n_accept") if verify else
                       "pinned host x[Q] rows, q_idx -> fdllm_fused_step_rows -> pinned host out"}

    # ---------------- roofline of the dominant kernel
    peak, peak_kind = measured_peaks()
    alg, rows = algorithmic_bytes(cfg)
    stage_mean = {k: sum(v) / len(v) for k, v in stage_ms.items()}
    dom = max(stage_mean, key=stage_mean.get)
    achieved = alg[dom] / (stage_mean[dom] / 1e3) / 1e9
    step_bytes = step_bytes_min(cfg)
    # what the stage call launches, timed together by the events around it
    # the library projects 128 rows and more on CTA pairs, fewer on single CTAs
    proj_k = "proj_pair_kernel" if B * rows >= 128 else "proj_tc_kernel"
    kernels = {"proj": proj_k if verify else "proj_prep_kernel + " + proj_k,
               "attn": "attn_tc_kernel", "accept": "accept_kernel"}
    if cfg["dtype"] != "bf16":
        kernels = {"proj": "proj_simt kernels", "attn": "attn_simt", "accept": "accept_kernel"}
    roofline = {"bound": "hbm", "kernel": kernels[dom], "stage": dom, "achieved": achieved, "peak": peak,
                "unit": "GB/s", "frac": achieved / peak, "peak_source": f"{peak_kind} hbm_gbs",
                "algorithmic_bytes_per_launch": alg[dom],
                "traffic": traffic_for(f"{name}:{dom}"),
                "ms_per_launch": stage_mean[dom]}

    res = {
        "metric": "fused-step query-tokens/s" if not verify else "verify-pass query-rows/s",
        "value": tokens_per_step / (mean_step / 1e3),
        "unit": "query-tokens/s" if not verify else "query-rows/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": mean_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": cfg["dtype"], "data": "synthetic",
        "config": bench_config(name, cfg, world),
        "hbm_gbs_step": step_bytes / (mean_step / 1e3) / 1e9,
        "step_roofline_frac": step_bytes / (mean_step / 1e3) / 1e9 / peak,
        "step_roofline_frac_nominal": step_bytes / (mean_step / 1e3) / 1e9 / NOMINAL_HBM_GBS,
        "stage_ms": stage_mean,
        "roofline": roofline,
        "e2e": e2e,
        "gpu_launches": int(launches),
        "clocks": sampler.summary(t0, t1),
    }
    return res


# ------------------------------------------------------------------ oracle leg

def oracle_step_fn(cfg, seqs):
    """One oracle pass over the given sequences of the workload (inputs prepared)."""
    import oracle as O
    H, dh, base = cfg["H"], cfg["dh"], cfg["rope_base"]
    f = O.to_f64
    if cfg["kind"] == "fused":
        inp = W.fused_inputs(cfg, seqs=seqs)
        a = (f(inp["x"]), inp["q_idx"].numpy(), f(inp["w_qkv"]), base, f(inp["k_cache"]),
             f(inp["v_cache"]), H, dh, cfg["dtype"])
        return lambda: O.fused_step(*a), len(seqs) * inp["q_idx"].shape[1]
    inp = W.verify_inputs(cfg, seqs=seqs)
    acc = W.accept_inputs(cfg, seqs=seqs)
    a = (f(inp["x_rows"]), inp["pos"].numpy(), inp["view"].numpy(), inp["rank"].numpy(),
         f(inp["w_qkv"]), base, f(inp["k_cache"]), f(inp["v_cache"]), f(inp["k_side"]),
         f(inp["v_side"]), H, dh, cfg["dtype"])
    la = (acc["logits"].numpy().astype(np.float64), acc["kind"].numpy(), acc["ref_tok"].numpy(),
          acc["rank"].numpy(), 0.9, 0.8)

    def step():
        O.verify_step(*a)
        O.accept(*la)
    return step, len(seqs) * inp["pos"].shape[1]


def cpu_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


def time_oracle(cfg, budget_s, max_reps, warmup=0):
    """Times the oracle as it stands on one sequence of the workload (a bounded sample).

    Inputs are generated and converted once; each timed step is one whole oracle pass.
    Returns (units/s, timed steps, units per step, seconds per step list)."""
    step, units = oracle_step_fn(cfg, [0])
    for _ in range(warmup):
        step()
    per = []
    while len(per) < max_reps and (not per or sum(per) < budget_s):
        t0 = time.perf_counter()
        step()
        per.append(time.perf_counter() - t0)
    return units * len(per) / sum(per), len(per), units, per


def run_reference(args, world, rank):
    cfg = W.CONFIGS[args.workload]
    budget = float(os.environ.get("FDLLM_ORACLE_BUDGET_S", "60"))
    # the warm-up is capped at one pass: it only pages in the numpy code paths
    _, _, units, per_step = time_oracle(cfg, budget, max(1, args.steps), warmup=min(1, args.warmup))
    mean = sum(per_step) / len(per_step)
    value = units / mean
    unit = "query-tokens/s" if cfg["kind"] == "fused" else "query-rows/s"
    sample = (f"one sequence (b=0) of {args.workload} per step: {units} query rows, the whole "
              f"fp64 oracle step (projection, RoPE, cache write, full-cache attention"
              + (", verify masks, acceptance over V logits" if cfg["kind"] == "verify" else "") + ")")
    return {"impl": "reference", "metric": "fused-step query-tokens/s" if cfg["kind"] == "fused"
            else "verify-pass query-rows/s", "value": value, "unit": unit, "n_gpus": world,
            "steps": len(per_step), "warmup": min(1, args.warmup), "ms_per_step": mean * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": bench_config(args.workload, cfg, world),
            "cpu_baseline": {"value": value, "unit": unit, "cores": cpu_threads(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


# ------------------------------------------------------------------ main

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD,
                    choices=[k for k in W.CONFIGS if k != "tiny_fp32"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true", help="skip the end-to-end pass")
    ap.add_argument("--batch", type=int, default=None,
                    help="override the workload's batch B (a smaller case of the same kernels, "
                         "e.g. for a profiler capture)")
    ap.add_argument("--seq-len", type=int, default=None,
                    help="override the workload's cache length N (the generated block stays "
                         "at the end; the prompt shrinks)")
    ap.add_argument("--sweep-batch", action="store_true",
                    help="batch scaling study: the single-sequence shape (N = 512 prompt + 512 "
                         "generated, |Q| = 32) at B = 1..64 per GPU, one JSON line per B")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    world, rank, local = dist_env()

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args, world, rank)), flush=True)
        return

    if world > 1:
        torch.distributed.init_process_group(
            "nccl", device_id=torch.device("cuda", local),
            timeout=__import__("datetime").timedelta(seconds=120))
    try:
        if args.sweep_batch:
            for B in SWEEP_BATCHES:
                cfg = dict(W.CONFIGS["single_bf16"], B=B, seed=6)
                r = run_ours(args, world, rank, local, cfg=cfg, name=f"sweep_B{B}", with_e2e=False)
                if rank == 0:
                    print(json.dumps({"sweep": "batch", "B_per_gpu": B, "n_gpus": world,
                                      "value": r["value"], "unit": r["unit"],
                                      "ms_per_step": r["ms_per_step"],
                                      "hbm_gbs_step": r["hbm_gbs_step"],
                                      "step_roofline_frac": r["step_roofline_frac"],
                                      "stage_ms": r["stage_ms"], "clocks": r["clocks"],
                                      "config": r["config"]}), flush=True)
            return
        cfg, name = workload_with_overrides(args)
        res = run_ours(args, world, rank, local, cfg=cfg, name=name, with_e2e=not args.no_e2e)
        if rank == 0 and world == 1 and not args.no_cpu_baseline:
            v, reps, units, _ = time_oracle(cfg, float(os.environ.get("FDLLM_ORACLE_BUDGET_S", "15")), 50)
            res["cpu_baseline"] = {
                "value": v, "unit": res["unit"], "cores": cpu_threads(), "kind": "oracle",
                "sample": f"{reps} oracle step(s) of one sequence (b=0) of {args.workload}, "
                          f"{units} query rows each, fp64 numpy"}
        if rank == 0:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
