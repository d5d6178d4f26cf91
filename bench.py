#!/usr/bin/env python
"""Throughput of the gated ReLU linear-attention token mixer on B200.

One step = the whole operator (state reduction, combine, apply) over one synthetic
720p/5s-shaped problem (B=1, H=32, d=128, 21 x 45 x 80 latent grid, N = 75,600) already
resident in HBM.  Prints one JSON line.  Multi-GPU runs (torchrun) give every rank its own
problem (weak scaling, no collective on the data path); the time is the max over ranks.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "gated linear-attn tokens·heads/s at 720p shapes; % of B200 HBM roofline"
UNIT = "tokens*heads/s"
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
KERNEL_SOURCES = {
    "apply_tc_kernel": "gated_linear_attention_relu_b200/csrc/apply_tc.cuh",
    "state_tc_kernel": "gated_linear_attention_relu_b200/csrc/state_tc.cuh",
}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default="720p_5s")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--simt", action="store_true", help="force the CUDA-core kernels")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="CPU work of the oracle baseline")
    ap.add_argument("--gated", action="store_true",
                    help="full gated form: write gate beta [B,H,N] and RMSNorm before the output gate")
    ap.add_argument("--causal", action="store_true",
                    help="token-causal operator (token n reads tokens 0..n) on a bidirectional workload's shape")
    ap.add_argument("--backward", action="store_true",
                    help="gradients (dQ, dK, dV, dG from dO; with --gated also dbeta, dgamma) of the "
                         "workload's form, bidirectional or block-causal")
    ap.add_argument("--saved-state", action="store_true",
                    help="with --backward: gradients from the states the forward pass returned "
                         "(la_backward_saved), as a training step keeps them, instead of reducing them again")
    ap.add_argument("--stream", action="store_true",
                    help="block-causal workloads: one la_block_step call per block on a carried cache, "
                         "as a block-autoregressive generator runs")
    return ap.parse_args()


def measured_hbm():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            v = float(json.load(f)["hbm_gbs"])
        return v, "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def kernel_traffic(name):
    """DRAM bytes per launch of `name` from the committed ncu summary, if the kernel source is
    unchanged since the capture (else None)."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)[name]
        src = os.path.join(ROOT, KERNEL_SOURCES[name])
        sha = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
        if rec.get("source_sha") != sha:
            return None, rec
        return rec, rec
    except Exception:
        return None, None


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while the timed region runs."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
               0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown", 0x100: "display_clocks"}

    def __init__(self, index, period=0.001):
        self.samples, self.reasons, self.ok = [], set(), False
        self.mem = []
        self.period, self._stop = period, threading.Event()
        try:
            import pynvml

            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # clocks are reported as unavailable
            self.err = str(e)

    def _run(self):
        nv = self.nv
        get_r = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                self.mem.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_MEM))
                r = get_r(self.h)
                for bit, name in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "note": "NVML unavailable"}
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons - {"gpu_idle"}),
                "samples": len(self.samples),
                "mem_mhz": statistics.median(self.mem) if self.mem else None}


def oracle_sample(w, seconds, steps=None, warmup=0, mode="forward"):
    """Time the fp64 oracle on one head of the workload (all its tokens): token*heads/s.

    ``mode`` picks the oracle of what the GPU run measures: "forward" (bidirectional or
    block-causal, as the workload says), "gated" (write gate and RMSNorm), "causal"
    (token-causal), "backward" (gradients, bidirectional or block-causal) or "backward_gated"
    (gradients of the gated form)."""
    import numpy as np

    import oracle as orc
    from gated_linear_attention_relu_b200 import workloads as wl

    one = w.with_(B=1, H=1)
    Q, K, V, G = (t.float().numpy().astype(np.float64)[0, 0] for t in wl.generate(one, "cpu"))
    pos = orc.grid_positions(w.T, w.Hh, w.W)
    if mode in ("gated", "backward_gated"):
        beta, gamma = (t.float().numpy().astype(np.float64) for t in wl.generate_gates(one, "cpu"))
        beta = beta[0, 0]
    if mode in ("backward", "backward_gated"):
        dO = wl.generate_grad(one, "cpu").float().numpy().astype(np.float64)[0, 0]
    # The token-causal oracle walks rows one by one in Python: time it on a fixed sample of rows
    # (it still carries the state over every token).
    rows = np.sort(np.random.default_rng(0).choice(w.N, size=min(w.N, 2000), replace=False)) \
        if mode == "causal" else None

    def run():
        if mode == "causal":
            orc.tokencausal_rows(Q, K, V, G, pos, w.bands, w.rope_base, w.eps, rows=rows)
        elif mode == "backward" and w.block_frames <= 0:
            orc.head_backward(Q, K, V, G, dO, pos, w.bands, w.rope_base, w.eps)
        elif mode in ("backward", "backward_gated"):
            gated = mode == "backward_gated"
            orc.head_backward_gated(Q, K, V, G, dO, pos, w.bands, w.rope_base, w.eps, block_frames=w.block_frames,
                                    beta=beta if gated else None, rms=(gamma, 1e-6) if gated else None)
        elif mode == "gated":
            orc.forward_positions(Q, K, V, G, pos, w.bands, w.rope_base, w.eps, beta=beta, rms=(gamma, 1e-6))
        elif w.block_frames > 0:
            Sb, zb = orc.block_states(K, V, pos, w.bands, w.rope_base, w.block_frames)
            Si, zi = np.cumsum(Sb, 0), np.cumsum(zb, 0)
            blk = orc.block_of_tokens(pos, w.block_frames)
            for b in range(Si.shape[0]):
                sel = blk == b
                orc.head_apply(Q[sel], G[sel], Si[b], zi[b], pos[sel], w.bands, w.rope_base, w.eps)
        else:
            S, z = orc.head_state(K, V, pos, w.bands, w.rope_base)
            orc.head_apply(Q, G, S, z, pos, w.bands, w.rope_base, w.eps)

    for _ in range(warmup):
        run()
    times = []
    t_all = time.perf_counter()
    while True:
        t0 = time.perf_counter()
        run()
        times.append(time.perf_counter() - t0)
        if steps is not None and len(times) >= steps:
            break
        if steps is None and time.perf_counter() - t_all >= seconds:
            break
    threads = os.cpu_count()
    try:
        from threadpoolctl import threadpool_info

        threads = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        pass
    per_run = len(rows) if rows is not None else w.N
    value = per_run * len(times) / sum(times)
    return value, threads, times


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    from gated_linear_attention_relu_b200 import workloads as wl

    w = wl.WORKLOADS[args.workload]
    mode = "causal" if args.causal else ("backward" if args.backward else ("gated" if args.gated else "forward"))
    if args.backward and args.gated:
        mode = "backward_gated"
    value, cores, times = oracle_sample(w, 0, steps=max(1, args.steps), warmup=max(0, args.warmup), mode=mode)
    sample = (f"one head of {w.name} ({f'{min(w.N, 2000)} sampled outputs' if mode == 'causal' else f'all {w.N} tokens'}), "
              f"fp64 numpy oracle ({mode}), per step")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": len(times), "warmup": args.warmup, "ms_per_step": 1e3 * sum(times) / len(times),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": config_of(w, args.gpus),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def config_of(w, n):
    return {"workload": w.name, "B": w.B, "H": w.H, "grid_T_Hh_W": [w.T, w.Hh, w.W], "N": w.N, "d": w.d,
            "rope_bands": list(w.bands), "block_frames": w.block_frames, "global_batch": w.B * n,
            "seq_len": w.N, "parallelism": f"dp{n}" if n > 1 else "single",
            "l2": f"inputs {w.min_bytes * 4 / 5 / 1e9:.2f} GB > 126 MB L2 (no flush)"}


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)

    import torch

    import gated_linear_attention_relu_b200 as la
    from gated_linear_attention_relu_b200 import dist as ldist
    from gated_linear_attention_relu_b200 import workloads as wl

    rank, local, world = ldist.env_rank()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    ldist.init("nccl")
    w = wl.WORKLOADS[args.workload]
    p = la.Problem.from_workload(w, force_simt=args.simt, token_causal=args.causal)
    la.load()

    Q, K, V, G = wl.generate(w, dev, seed=w.seed + 1000 * rank)
    O = torch.empty_like(Q)
    ws, _ = la.workspace(p, dev)
    stream = torch.cuda.current_stream()
    S_incl = z_incl = None
    if w.block_frames > 0:
        S_incl = torch.empty((w.B, w.H, w.nblk, w.d, w.d), dtype=torch.float32, device=dev)
        z_incl = torch.empty((w.B, w.H, w.nblk, w.d), dtype=torch.float32, device=dev)
    gates = {}
    if args.gated:
        beta, gamma = wl.generate_gates(w, dev, seed=w.seed + 7 + 1000 * rank)
        gates = dict(beta=beta, gamma=gamma, rms_norm=True, norm_eps=1e-6)
    if args.stream and w.block_frames <= 0:
        raise SystemExit("--stream needs a block-causal workload")

    if args.backward:
        if args.causal or args.stream:
            raise SystemExit("--backward takes no --causal or --stream")
        dO = wl.generate_grad(w, dev, seed=w.seed + 11 + 1000 * rank)
        grads = tuple(torch.empty_like(Q) for _ in range(4))
        saved = {}
        if args.saved_state:
            # The states the forward pass computes (outside the timed region, as in a training step).
            _, S_sv, z_sv = la.forward_gated(p, Q, K, V, G, ws=ws, return_states=True, **gates)
            saved = dict(S=S_sv, z=z_sv)
    elif args.saved_state:
        raise SystemExit("--saved-state goes with --backward")
    if args.stream:
        # One block per call pair, on contiguous per-block tensors cut out before timing (a
        # generator produces each block's tensors as it goes).
        HW = w.Hh * w.W
        blocks = []
        for t0 in range(0, w.T, w.block_frames):
            t1 = min(w.T, t0 + w.block_frames)
            sl = slice(t0 * HW, t1 * HW)
            pb = la.Problem.from_workload(w, T=t1 - t0, block_frames=0, t0=t0)
            blocks.append((pb, [x[:, :, sl].contiguous() for x in (Q, K, V, G)], torch.empty_like(Q[:, :, sl])))
        ws_s, _ = la.workspace(blocks[0][0], dev)
        S_c = torch.empty((w.B, w.H, w.d, w.d), dtype=torch.float32, device=dev)
        z_c = torch.empty((w.B, w.H, w.d), dtype=torch.float32, device=dev)
        counter = {"launches": 0}

        def forward_plain():
            S_c.zero_()
            z_c.zero_()
            n = 0
            for pb, (qb, kb, vb, gb), ob in blocks:
                la.block_step(pb, qb, kb, vb, gb, S_c, z_c, O=ob, ws=ws_s)
                n += la.last_launch_count()
            counter["launches"] = n
    elif args.backward:
        counter = {"launches": 0}

        def forward_plain():
            la.backward(p, Q, K, V, G, dO, grads=grads, ws=ws, **gates, **saved)
            counter["launches"] = la.last_launch_count()
    elif args.causal:
        if w.block_frames > 0 or args.gated:
            raise SystemExit("--causal takes a bidirectional workload and no --gated")

        def forward_plain():
            la.forward_tokencausal(p, Q, K, V, G, O=O, ws=ws)
    else:
        def forward_plain():
            if args.gated:
                la.forward_gated(p, Q, K, V, G, O=O, ws=ws, S_incl=S_incl, z_incl=z_incl, **gates)
            elif w.block_frames > 0:
                la.forward_blockcausal(p, Q, K, V, G, O=O, ws=ws, S_incl=S_incl, z_incl=z_incl)
            else:
                la.forward_bidir(p, Q, K, V, G, O=O, ws=ws)

    # Marker events around each kernel of each timed step; recorded once here so their CUDA
    # handles exist before the timed region.
    nmark = 6
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(nmark)] for _ in range(args.steps)]
    for row in evs:
        for e in row:
            e.record(stream)
    whole_step = args.stream or args.backward  # no per-kernel events for these
    if not whole_step:
        for _ in range(max(3, args.warmup)):
            la.forward_marked(p, Q, K, V, G, O, ws, evs[0], S_incl, z_incl, **gates)
        launches_per_step = la.last_launch_count()
    torch.cuda.synchronize()
    assert la.device_error() == 0, "device-side error during warm-up"

    for _ in range(max(3, args.warmup)):
        forward_plain()
    torch.cuda.synchronize()
    if whole_step:
        launches_per_step = counter["launches"]

    # Timed region (the headline): K steps of the public forward call, bracketed by a barrier and
    # a synchronize on both sides.  No events sit between the kernels of a step, so each kernel
    # may start early (programmatic dependent launch) as it does for a user.
    ldist.barrier(dev)
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        start.record(stream)
        for k in range(args.steps):
            forward_plain()
        end.record(stream)
        torch.cuda.synchronize()
    ldist.barrier(dev)
    t_ms = start.elapsed_time(end)
    t_max = ldist.max_over_ranks(t_ms, dev)
    assert la.device_error() == 0, "device-side error in the timed region"

    # Second timed region, same K steps with an event before and after every kernel: the
    # per-kernel durations and the dominant kernel's roofline come from here.  (An event between
    # two kernels keeps the second from starting early, so these steps run a little longer.)
    marked_ms = None
    if not whole_step:
        ldist.barrier(dev)
        torch.cuda.synchronize()
        m_start, m_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        m_start.record(stream)
        for k in range(args.steps):
            la.forward_marked(p, Q, K, V, G, O, ws, evs[k], S_incl, z_incl, **gates)
        m_end.record(stream)
        torch.cuda.synchronize()
        ldist.barrier(dev)
        marked_ms = m_start.elapsed_time(m_end) / args.steps
        assert la.device_error() == 0, "device-side error in the marked region"

    elem = w.elem_bytes
    th = w.B * w.H * w.N
    peak, peak_kind = measured_hbm()
    value = world * th * args.steps / (t_max * 1e-3)
    ms_per_step = t_max / args.steps
    # bytes_min: Q, K, V, G read once and O written once (+ the write gate when gated); the
    # backward pass reads Q, K, V, G, dO and writes dQ, dK, dV, dG (+ reads beta, writes dbeta).
    min_bytes = w.min_bytes + (th * elem if args.gated else 0)
    if args.backward:
        min_bytes = 9 * th * w.d * elem + (2 * th * elem if args.gated else 0)
    roof_all = min_bytes / (ms_per_step * 1e-3) / 1e9

    if whole_step:
        # No events sit between these kernels, so the roofline is the whole step's.
        kernels, alg, achieved, traffic = {}, min_bytes, roof_all, None
        dominant = "whole step (per-block calls)" if args.stream else f"whole step ({launches_per_step} kernels)"
    else:
        # Per-kernel durations inside the timed steps of the second region.
        tc = not args.simt and w.d == 128 and w.dtype == "bf16"
        if args.causal:
            names = ["rope_table_kernel", "state_tc_kernel", "start_kernel", "causal_tc_kernel"]
        elif tc and w.nblk > 1:
            names = ["rope_table_kernel", "state_tc_kernel", "blocksum_kernel", "prefix_kernel", "apply_tc_kernel"]
        elif tc:
            names = ["rope_table_kernel", "state_tc_kernel", "combine_kernel", "apply_tc_kernel"]
        else:
            names = ["state_simt_kernel", "combine_kernel", "apply_simt_kernel"]
        assert len(names) == launches_per_step, (names, launches_per_step)
        per = {n: [] for n in names}
        for k in range(args.steps):
            for i, n in enumerate(names):
                per[n].append(evs[k][i].elapsed_time(evs[k][i + 1]))
        kern_ms = {n: sum(v) / len(v) for n, v in per.items()}
        tot = sum(kern_ms.values())
        # the token-causal kernel reads Q, K, V, G and writes O; the apply kernel reads Q, G, writes O
        state_name = next(n for n in names if n.startswith("state_"))
        alg_bytes = {state_name: (2 * w.d + (1 if args.gated else 0)) * th * elem,
                     names[-1]: (5 if args.causal else 3) * th * w.d * elem}
        dominant = max((n for n in names if n in alg_bytes), key=lambda n: kern_ms[n])
        alg = alg_bytes[dominant]
        achieved = alg / (kern_ms[dominant] * 1e-3) / 1e9
        traffic_rec, _ = kernel_traffic(dominant)
        traffic = None
        if traffic_rec is not None and traffic_rec.get("workload") == w.name and not args.gated:
            traffic = traffic_rec.get("bytes_per_launch")
        kernels = {n: {"ms": kern_ms[n], "share": kern_ms[n] / tot if tot else None} for n in names}

    config = config_of(w, world)
    if args.gated:
        config["gated"] = "write gate beta [B,H,N] + RMSNorm (gamma [d]) before the output gate"
    if args.backward:
        config["mode"] = ("backward: dQ, dK, dV, dG" + (", dbeta, dgamma" if args.gated else "") +
                          (" from dO and the forward's saved states (la_backward_saved)" if args.saved_state
                           else " from dO (recomputes the forward state)"))
    if args.causal:
        config["mode"] = "token-causal (token n reads tokens 0..n; K and V are read by both passes)"
    if args.stream:
        config["stream"] = f"{len(blocks)} blocks, one la_block_step per block on a carried cache"
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": w.dtype, "data": "synthetic (seeded N(0,1) inputs of the workload's shape)",
        "config": config,
        "hbm_roofline_frac_8tbs": roof_all / NOMINAL_HBM_GBS,
        "hbm_roofline_frac_measured": roof_all / peak,
        "achieved_gbs_whole_step": roof_all,
        "roofline": {"bound": "hbm", "kernel": dominant, "achieved": achieved, "peak": peak,
                     "peak_kind": peak_kind, "unit": "GB/s", "frac": achieved / peak, "traffic": traffic,
                     "algorithmic_bytes_per_launch": alg},
        "kernels": kernels,
        "kernels_region": {"ms_per_step": marked_ms, "note": "second timed region, events around every kernel"},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clk.summary(),
    }
    if line["clocks"].get("sm_mhz"):
        # Clock-normalised step time: ms per step x median SM MHz (compare runs at different clocks).
        line["clocks"]["ms_per_step_x_sm_mhz"] = ms_per_step * line["clocks"]["sm_mhz"]

    if not args.no_e2e and args.stream:
        line["e2e"] = e2e_stream(la, w, blocks, ws_s, S_c, z_c, dev, args, ldist, world)
    elif not args.no_e2e:
        line["e2e"] = e2e(la, p, w, Q, K, V, G, O, ws, dev, args, ldist, world, gates, causal=args.causal,
                          dO=dO if args.backward else None, grads=grads if args.backward else None,
                          saved=saved if args.backward else None)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        mode = "causal" if args.causal else ("backward" if args.backward else ("gated" if args.gated else "forward"))
        if args.backward and args.gated:
            mode = "backward_gated"
        v, cores, times = oracle_sample(w, args.cpu_seconds, mode=mode)
        line["cpu_baseline"] = {"value": v, "unit": UNIT, "cores": cores, "kind": "oracle",
                                "sample": f"one head of {w.name} ({f'{min(w.N, 2000)} sampled outputs' if mode == 'causal' else f'all {w.N} tokens'}), "
                                          f"{len(times)} runs, fp64 numpy oracle ({mode})"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    ldist.finalize()
    return 0


def e2e_stream(la, w, blocks, ws, S_c, z_c, dev, args, ldist, world):
    """End to end for block-autoregressive generation through la_block_step: a step is one video.
    Each block's Q, K, V, G come from pinned host memory (as a generator would hand them over) and
    the block's O goes back to the host; block j+1's inputs cross the host link while block j
    computes (two device buffer sets, copies in on one stream, the operator on the current stream,
    copies out on a third)."""
    import torch

    hosts = [[t.cpu().pin_memory() for t in ins] for _, ins, _ in blocks]
    ohost = [torch.empty(o.shape, dtype=o.dtype).pin_memory() for _, _, o in blocks]
    # two device sets per block length (a last block may be shorter), contiguous [B, H, n, d]
    sets = {}
    for _, ins, o in blocks:
        n = o.shape[2]
        if n not in sets:
            sets[n] = ([[torch.empty_like(t) for t in ins] for _ in range(2)], [torch.empty_like(o) for _ in range(2)])
    cur = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_done = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    used = [False, False]
    nb = len(blocks)

    def video():
        S_c.zero_()
        z_c.zero_()
        for j, (pb, _, o) in enumerate(blocks):
            k = j & 1
            dsets, osets = sets[o.shape[2]]
            with torch.cuda.stream(s_in):
                if used[k]:
                    s_in.wait_event(ev_done[k])  # block j-2's operator has read set k
                for hsrc, dst in zip(hosts[j], dsets[k]):
                    dst.copy_(hsrc, non_blocking=True)
                ev_in[k].record(s_in)
            cur.wait_event(ev_in[k])
            if used[k]:
                cur.wait_event(ev_out[k])  # block j-2's output has left set k
            d = dsets[k]
            la.block_step(pb, d[0], d[1], d[2], d[3], S_c, z_c, O=osets[k], ws=ws)
            ev_done[k].record(cur)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_done[k])
                ohost[j].copy_(osets[k], non_blocking=True)
                ev_out[k].record(s_out)
            used[k] = True

    video()
    torch.cuda.synchronize()
    ldist.barrier(dev)
    steps = max(3, min(args.steps, 10))
    st, en = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    st.record(cur)
    s_in.wait_stream(cur)
    s_out.wait_stream(cur)
    for _ in range(steps):
        video()
    cur.wait_stream(s_in)
    cur.wait_stream(s_out)
    en.record(cur)
    torch.cuda.synchronize()
    t = ldist.max_over_ranks(st.elapsed_time(en), dev)
    h2d = sum(x.numel() * x.element_size() for hb in hosts for x in hb)
    d2h = sum(x.numel() * x.element_size() for x in ohost)
    return {"value": world * w.B * w.H * w.N * steps / (t * 1e-3), "unit": UNIT, "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "steps": steps,
            "pipelined": f"{nb} la_block_step calls per video; block j+1 copied in while block j computes"}


def e2e(la, p, w, Q, K, V, G, O, ws, dev, args, ldist, world, gates=None, causal=False, dO=None, grads=None,
        saved=None):
    """Same metric through the public API with the inputs in pinned host memory: every step
    copies the step's inputs host->device (Q, K, V, G, and the write gate when gated, or dO for
    the backward pass, with the forward's states when it starts from them), runs the operator and
    copies its outputs (O, or dQ, dK, dV, dG)
    device->host.  Steps are pipelined the way a caller streaming batches would run them: two
    device copies of the inputs and of the outputs, the host->device copies on one stream, the
    operator on the current stream and the device->host copies on a third, so step k+1's inputs
    and step k-1's outputs cross the host link while step k computes (each copy engine works one
    direction)."""
    import torch

    gates = gates or {}
    if dO is not None:
        saved = saved or {}
        extra = ([("beta", gates["beta"])] if "beta" in gates else []) + sorted(saved.items())
        srcs0 = [Q, K, V, G, dO] + [t for _, t in extra]
        outs0 = list(grads)

        def run(d, o):
            g = dict(gates)
            g.update({name: d[5 + i] for i, (name, _) in enumerate(extra)})
            la.backward(p, d[0], d[1], d[2], d[3], d[4], grads=tuple(o), ws=ws, **g)
    else:
        srcs0 = [Q, K, V, G] + ([gates["beta"]] if "beta" in gates else [])
        outs0 = [O]

        def run(d, o):
            if gates:
                g = dict(gates)
                if len(d) > 4:
                    g["beta"] = d[4]
                la.forward_gated(p, d[0], d[1], d[2], d[3], O=o[0], ws=ws, **g)
            elif causal:
                la.forward_tokencausal(p, d[0], d[1], d[2], d[3], O=o[0], ws=ws)
            else:
                la.forward(p, d[0], d[1], d[2], d[3], O=o[0], ws=ws)

    hosts = [t.cpu().pin_memory() for t in srcs0]
    dsets = [srcs0, [torch.empty_like(t) for t in srcs0]]
    osets = [outs0, [torch.empty_like(t) for t in outs0]]
    ohost = [[torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in outs0] for _ in range(2)]
    steps = max(3, min(args.steps, 10))
    cur = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_done = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    used = [False, False]

    def step(k):
        j = k & 1
        with torch.cuda.stream(s_in):
            if used[j]:
                s_in.wait_event(ev_done[j])  # the operator of step k-2 has read this input set
            for hsrc, dst in zip(hosts, dsets[j]):
                dst.copy_(hsrc, non_blocking=True)
            ev_in[j].record(s_in)
        cur.wait_event(ev_in[j])
        if used[j]:
            cur.wait_event(ev_out[j])  # step k-2's outputs have left these buffers
        run(dsets[j], osets[j])
        ev_done[j].record(cur)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_done[j])
            for hdst, src in zip(ohost[j], osets[j]):
                hdst.copy_(src, non_blocking=True)
            ev_out[j].record(s_out)
        used[j] = True

    for k in range(2):
        step(k)
    torch.cuda.synchronize()
    ldist.barrier(dev)
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record(cur)
    s_in.wait_stream(cur)
    s_out.wait_stream(cur)
    for k in range(steps):
        step(k)
    cur.wait_stream(s_in)
    cur.wait_stream(s_out)
    e.record(cur)
    torch.cuda.synchronize()
    t = ldist.max_over_ranks(s.elapsed_time(e), dev)
    th = w.B * w.H * w.N
    h2d = sum(x.numel() * x.element_size() for x in srcs0)
    d2h = sum(x.numel() * x.element_size() for x in outs0)
    return {"value": world * th * steps / (t * 1e-3), "unit": UNIT, "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "steps": steps,
            "pipelined": "two input and output buffers; copies in, operator and copies out on three streams"}


if __name__ == "__main__":
    sys.exit(main())
