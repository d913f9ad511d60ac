"""Benchmark: SWA∥RMA decode tok/s at B=512 over 8 layers, commits/s, % of HBM roofline.

Workload (per GPU; weak scaling over GPUs, no data-path collective): 512
sequences, 8 SWA∥RMA layers, state seeded at position 32768 with window and
bank full and pending fill U{0..255} per sequence (36 GiB of BF16 K/V, far
above the 126 MB L2, so no flush is needed between steps).  One step = one
token for every sequence through all 8 layers (projections, scores, norm +
RoPE, window write, pending append, both reads, o_proj, device-decided commits)
plus the metadata advance.  Over 256 steps every sequence commits once.

Usage: python bench.py [--gpus N --steps K --warmup W] [--impl reference]
Under torchrun each rank runs its own replica on its own GPU; rank 0 prints
one JSON line with the whole-job throughput (max time over ranks).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "SWA∥RMA decode tok/s (B=512, 8 layers) + commits/s; % of B200 HBM roofline"
WORKLOAD = "decode_b512_l8_t32768"
B, LAYERS, T0 = 512, 8, 32768
ROW = 1024  # bytes of one K row + one V row


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=256)
    ap.add_argument("--warmup", type=int, default=4)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer pass")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-commit-bench", action="store_true")
    ap.add_argument("--no-prefill-bench", action="store_true")
    ap.add_argument("--no-rma-off", action="store_true",
                    help="skip the decode pass with the RMA switched off (the ablation)")
    ap.add_argument("--no-graph", action="store_true",
                    help="skip the CUDA-graph pass (one captured graph per decode step)")
    ap.add_argument("--no-pool", action="store_true",
                    help="skip the pooled-layout A/B (decode steps and commits)")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the B=1 (one layer) and B=64 (8 layers) decode configurations")
    ap.add_argument("--prefill-chunks", type=int, default=512,
                    help="256-token chunks of the prefill stream (512 = 131072 tokens)")
    ap.add_argument("--kernel", default="step",
                    choices=["step", "attend", "commit", "prefill", "score", "layer"],
                    help="step: the benchmark; attend/commit: one kernel alone at --batch "
                         "sequences; score: the scorer on --batch tokens; prefill: "
                         "--prefill-chunks chunks of one layer; layer: one decode layer "
                         "call at --batch sequences (profiling drivers)")
    ap.add_argument("--batch", type=int, default=256)
    ap.add_argument("--sweep", action="store_true",
                    help="layer-level batch sweep B = 1..512 (one JSON line per batch size)")
    return ap.parse_args()


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """SM clocks and throttle reasons sampled during the timed region: NVML read
    every 10 ms from a host thread (read-only queries), else nvidia-smi every
    200 ms.  Samples outside the timed windows (begin/end) are ignored."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    # NVML clock event reason bits
    REASON_BITS = {"sw_power_cap": 0x4, "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20,
                   "hw_thermal_slowdown": 0x40}

    def __init__(self, gpu_index, device=None):
        self.idx = gpu_index
        self.device = device
        self.proc = None
        self.nvml = None
        self.samples = []  # (host time, sm MHz, max sm MHz, set of reasons)
        self.lines = []    # (host time, nvidia-smi line)
        self.windows = []  # [t0, t1] spans of timed work
        self.stop_flag = False

    def begin(self):
        self.windows.append([time.monotonic(), None])

    def end(self):
        self.windows[-1][1] = time.monotonic()

    def _nvml_handle(self):
        import pynvml
        pynvml.nvmlInit()
        try:
            import torch
            uuid = str(torch.cuda.get_device_properties(self.device).uuid)
            return pynvml, pynvml.nvmlDeviceGetHandleByUUID(
                uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
        except Exception:
            return pynvml, pynvml.nvmlDeviceGetHandleByIndex(self.idx)

    def start(self):
        try:
            self.nvml = self._nvml_handle()
            self.th = threading.Thread(target=self._poll_nvml, daemon=True)
            self.th.start()
            return
        except Exception:
            self.nvml = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.th = threading.Thread(target=self._read, daemon=True)
            self.th.start()
        except Exception:
            self.proc = None

    def _poll_nvml(self):
        pynvml, h = self.nvml
        smax = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
        while not self.stop_flag:
            t = time.monotonic()
            if self.windows and self.windows[-1][1] is None:
                try:
                    sm = pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
                    bits = pynvml.nvmlDeviceGetCurrentClocksThrottleReasons(h)
                    rs = {n for n, b in self.REASON_BITS.items() if bits & b}
                    self.samples.append((t, float(sm), float(smax), rs))
                except Exception:
                    pass
            time.sleep(0.01)

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.monotonic(), line.strip()))

    def _timed(self, t):
        return any(a <= t <= (b if b is not None else float("inf")) for a, b in self.windows)

    def stop(self):
        if self.nvml:
            self.stop_flag = True
            self.th.join(timeout=5)
            sm = [x[1] for x in self.samples if self._timed(x[0])]
            smax = [x[2] for x in self.samples if self._timed(x[0])]
            reasons = set()
            for x in self.samples:
                if self._timed(x[0]):
                    reasons |= x[3]
            return {"sm_mhz": statistics.median(sm) if sm else None,
                    "sm_max_mhz": max(smax) if smax else None, "reasons": sorted(reasons),
                    "samples": len(sm), "source": "NVML, every 10 ms in the timed loops"}
        if not self.proc:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["clock query unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for t, ln in self.lines:
            if self.windows and not self._timed(t):
                continue
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None, "reasons": sorted(reasons),
                "samples": len(sm), "source": "nvidia-smi, every 200 ms"}


# ------------------------------------------------------------ multi-rank

def reduce_max(value: float, device) -> float:
    """Max of a float over all ranks (identity without a process group).  Every
    rank calls it at the same points, in warm-up, timing and error paths alike."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_tokens_per_s(world: int, batch: int, steps: int, max_ms: float) -> float:
    """Weak scaling: every rank decodes its own batch; the job's rate uses the
    slowest rank's time."""
    return world * batch * steps / (max_ms / 1e3)


# --------------------------------------------------------------- our arm

def algorithmic_read_bytes(fills, steps_from, steps):
    """State bytes the reads of one layer must touch, summed over the given steps:
    per (sequence, group) 1024 window rows + 1024 bank rows + (pending + 1) rows,
    K and V, plus q (2 branches x 4 heads x 512 B) and o (2 x 4 x 1 KiB FP32)."""
    tot = 0
    for s in range(steps_from, steps_from + steps):
        for f in fills:
            p = (f + s) % 256
            tot += 4 * ((1024 + 1024 + p + 1) * ROW + 2 * 4 * 512 + 2 * 4 * 1024)
    return tot


def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    import sliding_window_anchor_b200 as sab
    from synth import workloads as wl

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    seed = wl.seed_of(wl.DECODE_B512)
    weights = [sab.LayerWeights.from_dict(wl.make_weights(seed, l, device=dev))
               for l in range(LAYERS)]
    wdicts = [w.t for w in weights]
    st = sab.State(B, LAYERS, device=dev)

    def normrope(x, g, pos):
        return sab.qk_norm_rope(x.contiguous(), g, pos.to(torch.int32).contiguous())

    fills = wl.seed_state(st.arrays(), range(B), LAYERS, T0, "uniform", seed, wdicts, normrope,
                          device=dev).cpu().tolist()
    ids = torch.arange(B, dtype=torch.int32, device=dev)
    ws = torch.empty(sab.decode_workspace_bytes(B), dtype=torch.uint8, device=dev)
    total = args.warmup + args.steps
    n_x = min(total, 64)  # distinct per-step inputs, resident before timing
    xs = [[wl.make_x(seed, l, s, range(B), device=dev) for l in range(LAYERS)] for s in range(n_x)]
    outs = [torch.empty(B, 2560, dtype=torch.bfloat16, device=dev) for _ in range(LAYERS)]
    stream = torch.cuda.current_stream(dev)

    def step(s):
        for l in range(LAYERS):
            sab.swa_rma_decode(st, weights[l], l, ids, xs[s % n_x][l], out=outs[l], ws=ws)
        sab.advance(st, ids)

    for s in range(args.warmup):
        step(s)
    torch.cuda.synchronize(dev)
    if sab.last_device_error(st) != 0:
        raise RuntimeError("device error during warm-up")
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    sab.profile_read(reset=True)
    sab.profile_enable(True)
    clocks = ClockSampler(local_rank, dev)
    clocks.start()
    n0 = sab.launch_count()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.nvtx.range_push("timed_eager" if not args.no_graph else "timed")
    clocks.begin()
    e0.record(stream)
    for s in range(args.warmup, total):
        step(s)
    e1.record(stream)
    torch.cuda.nvtx.range_pop()
    torch.cuda.synchronize(dev)
    clocks.end()
    ms = e0.elapsed_time(e1)
    launches = sab.launch_count() - n0
    sab.profile_enable(False)
    attend_ms, attend_n = sab.profile_read(reset=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    err = sab.last_device_error(st)
    if err != 0:
        raise RuntimeError(f"device error {err} in the timed region")
    commits = sum(1 for f in fills for s in range(args.warmup, total) if (f + s) % 256 == 255)

    graph = None
    if not args.no_graph:
        # the same steps replayed from CUDA graphs: one graph per distinct input buffer,
        # each holding a whole step (8 layers, device-gated commits, the advance)
        stream_g = torch.cuda.Stream(dev)
        graphs = []
        n_launch0 = sab.launch_count()
        for s in range(n_x):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream_g):
                step(s)
            graphs.append(g)
        per_step = (sab.launch_count() - n_launch0) // n_x
        for s in range(args.warmup):
            graphs[s % n_x].replay()
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)
        g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.nvtx.range_push("timed")
        clocks.begin()
        g0.record(stream)
        for s in range(args.warmup, total):
            graphs[s % n_x].replay()
        g1.record(stream)
        torch.cuda.nvtx.range_pop()
        torch.cuda.synchronize(dev)
        clocks.end()
        if sab.last_device_error(st) != 0:
            raise RuntimeError("device error in the graph pass")
        gms = reduce_max(g0.elapsed_time(g1), dev)
        graph = {"ms": gms, "launches_per_step": per_step}
        del graphs
    clk = clocks.stop()  # samples taken during the eager and the graph timed loops

    e2e = None
    if not args.no_e2e:
        # the same steps through the C ABI from pinned host buffers: every step's
        # inputs (all layers' x) go host -> device and its outputs (all layers')
        # device -> host inside the timed region.  Copies run on their own streams,
        # double-buffered, so step s+1's upload and step s's download overlap the
        # compute of the neighbouring steps; events order every buffer reuse.
        hx = [torch.empty(LAYERS, B, 2560, dtype=torch.bfloat16, pin_memory=True)
              for _ in range(2)]
        for i in range(2):
            for l in range(LAYERS):
                hx[i][l].copy_(xs[i][l])
        hout = [torch.empty(LAYERS, B, 2560, dtype=torch.bfloat16, pin_memory=True)
                for _ in range(2)]
        dx = [torch.empty(LAYERS, B, 2560, dtype=torch.bfloat16, device=dev) for _ in range(2)]
        dout = [torch.empty(LAYERS, B, 2560, dtype=torch.bfloat16, device=dev)
                for _ in range(2)]
        s_h2d, s_d2h = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        h2d_done = [torch.cuda.Event() for _ in range(2)]
        comp_done = [torch.cuda.Event() for _ in range(2)]
        d2h_done = [torch.cuda.Event() for _ in range(2)]
        k_e2e = min(args.steps, 64)

        def e2e_step(b):
            for l in range(LAYERS):
                sab.swa_rma_decode(st, weights[l], l, ids, dx[b][l], out=dout[b][l], ws=ws)
            sab.advance(st, ids)

        # unless --no-graph, each buffer's step is replayed from a captured CUDA graph
        # of the same calls (the production path); the copies stay outside it
        e2e_graphs = None
        if not args.no_graph:
            stream_g = torch.cuda.Stream(dev)
            e2e_graphs = []
            for b in range(2):
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g, stream=stream_g):
                    e2e_step(b)
                e2e_graphs.append(g)
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record(stream)
        s_h2d.wait_event(f0)
        for s in range(k_e2e):
            b = s % 2
            if s >= 2:
                s_h2d.wait_event(comp_done[b])  # step s-2 has read dx[b]
            with torch.cuda.stream(s_h2d):
                dx[b].copy_(hx[b], non_blocking=True)
            h2d_done[b].record(s_h2d)
            stream.wait_event(h2d_done[b])
            if s >= 2:
                stream.wait_event(d2h_done[b])  # step s-2's outputs have left dout[b]
            if e2e_graphs is not None:
                e2e_graphs[b].replay()
            else:
                e2e_step(b)
            comp_done[b].record(stream)
            s_d2h.wait_event(comp_done[b])
            with torch.cuda.stream(s_d2h):
                hout[b].copy_(dout[b], non_blocking=True)
            d2h_done[b].record(s_d2h)
        for b in range(2):
            stream.wait_event(d2h_done[b])
        f1.record(stream)
        torch.cuda.synchronize(dev)
        e2e_ms = reduce_max(f0.elapsed_time(f1), dev)
        nbytes = LAYERS * B * 2560 * 2
        e2e = {"value": whole_job_tokens_per_s(world, B, k_e2e, e2e_ms), "unit": "tok/s",
               "h2d_bytes_per_step": nbytes, "d2h_bytes_per_step": nbytes, "steps": k_e2e,
               "copies": "pinned host buffers, own streams, double-buffered",
               "launch": "one CUDA graph per step" if e2e_graphs is not None else "eager"}
        del e2e_graphs


    rma_off = None
    if not args.no_rma_off:
        # the pages' ablation: the same decode with every RMA module off (window read only)
        k_off = min(args.steps, 64)
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
        sab.profile_read(reset=True)
        sab.profile_enable(True)
        r0, r1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        r0.record(stream)
        for s in range(k_off):
            for l in range(LAYERS):
                sab.swa_rma_decode(st, weights[l], l, ids, xs[s % n_x][l], out=outs[l], ws=ws,
                                   rma_off=True)
            sab.advance(st, ids, rma_off=True)
        r1.record(stream)
        torch.cuda.synchronize(dev)
        sab.profile_enable(False)
        off_attend_ms, off_attend_n = sab.profile_read(reset=True)
        if sab.last_device_error(st) != 0:
            raise RuntimeError("device error in the RMA-off pass")
        off_ms = reduce_max(r0.elapsed_time(r1), dev)
        # per (sequence, group): 1024 window rows (K + V), q_swa (4 x 512 B), o (4 x 1 KiB)
        alg = B * 4 * (1024 * ROW + 4 * 512 + 4 * 1024)
        hbm, kind = peaks()
        per = off_attend_ms / max(off_attend_n, 1)
        rma_off = {"value": whole_job_tokens_per_s(world, B, k_off, off_ms),
                   "ms_per_step": off_ms / k_off, "steps": k_off,
                   "attend_avg_launch_ms": per,
                   "attend_frac": alg / (per / 1e3) / 1e9 / hbm if per > 0 else None,
                   "attend_alg_bytes_per_launch": alg,
                   "note": "ER_FLAG_RMA_OFF, eager: o_rma = 0, no score, append or commit"}

    ms = reduce_max(ms, dev)
    pool_ab = None
    if not args.no_pool and rank == 0:
        pool_ab = pooled_ab(st, weights, ids, xs, dev)  # before the commit workload replaces the state
    cm = None
    if not args.no_commit_bench and rank == 0:
        # the commit microbench reuses the decode state's memory (B=512 x 8 layers)
        cm = commit_microbench(st, dev)
    pf = None
    if not args.no_prefill_bench and rank == 0:
        pf = prefill_bench(dev, args.prefill_chunks)
    cfgs = None
    if not args.no_configs and rank == 0:
        cfgs = {r["workload"]: r for r in (decode_config_bench(dev, wl.DECODE_B1),
                                           decode_config_bench(dev, wl.DECODE_B64))}
    return dict(ms=ms, launches=launches, clocks=clk, attend_ms=attend_ms, attend_n=attend_n,
                fills=fills, commits=commits, e2e=e2e, commit_microbench=cm, prefill=pf,
                graph=graph, rma_off=rma_off, configs=cfgs, pool=pool_ab)


# ------------------------------------------------------- commit microbench

def commit_microbench(st, dev, reps=3):
    """Times er_rma_commit(layer=-1) over every sequence: B x 8 layers x 4 groups
    independent top-1024-of-1280 merges of the commit workload.  Every repetition
    is a fresh workload (scores N(0,1) with ~5% exact ties, bank and pending full;
    synth.workloads.seed_commit_workload), the first one untimed.  Algorithmic bytes
    per merge: the 1280 keys (score + position, 8 B each) read, plus each moved
    record's K and V row read and written (2 x 1 KiB) with its score and position
    (2 x 8 B).  The same seeds are checked bit-exact against the oracle by
    tests/test_gpu_steps.py::test_commit_full_size_workload_matches_oracle."""
    import torch
    import sliding_window_anchor_b200 as sab
    from synth import workloads as wl
    seed = wl.seed_of(wl.COMMIT)
    ids = torch.arange(st.s_max, dtype=torch.int32, device=dev)
    merges = st.s_max * st.n_layers * 4
    times, moved = [], []
    for rep in range(reps + 1):
        wl.seed_commit_workload(st.arrays(), range(st.s_max), st.n_layers, T0, seed, rep, dev)
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        sab.rma_commit(st, -1, ids)
        e1.record()
        torch.cuda.synchronize(dev)
        if sab.last_device_error(st) != 0:
            raise RuntimeError("device error in the commit microbench")
        if rep > 0:  # the first repetition is the warm-up
            times.append(e0.elapsed_time(e1))
            moved.append(int((st.bank_pos >= T0).sum()))  # pending positions are T0..T0+255
    i = sorted(range(reps), key=lambda k: times[k])[reps // 2]
    ms, m = times[i], moved[i]
    alg = merges * 1280 * 8 + m * (2 * 1024 + 16)
    hbm, kind = peaks()
    return {"workload": f"commit_b{st.s_max}_l{st.n_layers}", "merges": merges, "ms": ms,
            "merges_per_s": merges / (ms / 1e3),
            "sequence_commits_per_s": st.s_max / (ms / 1e3),
            "moved_records": m, "moved_per_merge": m / merges, "alg_bytes": alg,
            "achieved_gbs": alg / (ms / 1e3) / 1e9,
            "frac": alg / (ms / 1e3) / 1e9 / hbm, "peak_gbs": hbm, "peak_kind": kind,
            "reps": reps, "note": "median of the timed repetitions, each a freshly seeded "
                                  "workload (i.i.d. scores, ~5% ties)"}


def pooled_ab(st, weights, ids, xs, dev, steps=32, reps=3):
    """The pooled anchor layout (ER_STATE_POOL, a commit that moves no K/V row)
    against the plain one, measured on the same work: (1) decode steps of the
    decode workload, each layout starting from the same records, replayed from
    CUDA graphs; (2) the commit microbench, each repetition's workload copied
    into the pooled layout (identical records and keys)."""
    import torch
    import sliding_window_anchor_b200 as sab
    from synth import workloads as wl
    B, L = st.s_max, st.n_layers
    n_x = len(xs)
    ws = torch.empty(sab.decode_workspace_bytes(B), dtype=torch.uint8, device=dev)
    outs = [torch.empty(B, 2560, dtype=torch.bfloat16, device=dev) for _ in range(L)]
    stream = torch.cuda.current_stream(dev)
    pool = sab.State(B, L, device=dev, pool=True)
    pool.pool_from_plain(st)
    res = {}
    for name, state in (("pooled", pool), ("plain", st)):
        def step(s, state=state):
            for l in range(L):
                sab.swa_rma_decode(state, weights[l], l, ids, xs[s % n_x][l], out=outs[l], ws=ws)
            sab.advance(state, ids)
        step(0)  # the stream's side resources exist before capture
        torch.cuda.synchronize(dev)
        stream_g = torch.cuda.Stream(dev)
        graphs = []
        for s in range(n_x):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream_g):
                step(s)
            graphs.append(g)
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for s in range(steps):
            graphs[(s + 1) % n_x].replay()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        del graphs
        if sab.last_device_error(state) != 0:
            raise RuntimeError(f"device error in the {name} decode pass")
        ms = e0.elapsed_time(e1) / steps
        res[name] = {"ms_per_step": ms, "tok_per_s": B / (ms / 1e3)}
    # the commit microbench in both layouts on the same workloads
    seed = wl.seed_of(wl.COMMIT)
    merges = B * L * 4
    t_plain, t_pool, moved = [], [], []
    snap_keys = None
    for rep in range(reps + 1):
        wl.seed_commit_workload(st.arrays(), range(B), L, T0, seed, rep, dev)
        pool.pool_from_plain(st)
        torch.cuda.synchronize(dev)
        for name, state, acc in (("pooled", pool, t_pool), ("plain", st, t_plain)):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            sab.rma_commit(state, -1, ids)
            e1.record()
            torch.cuda.synchronize(dev)
            if sab.last_device_error(state) != 0:
                raise RuntimeError(f"device error in the {name} commit")
            if rep > 0:
                acc.append(e0.elapsed_time(e1))
        if rep > 0:
            moved.append(int((st.bank_pos >= T0).sum()))
    med = lambda v: sorted(v)[len(v) // 2]
    hbm, kind = peaks()
    m = med(moved)
    # bytes a pooled merge must touch: the 1280 keys read, the evicted slots'
    # position and score written, the 256-entry slot list written (no K/V row)
    pool_alg = merges * (1280 * 8 + (m / merges) * 8 + 256 * 4)
    plain_alg = merges * 1280 * 8 + m * (2 * 1024 + 16)
    res["commit"] = {
        "workload": f"commit_b{B}_l{L}", "merges": merges, "moved_records_plain": m,
        "plain_ms": med(t_plain), "pooled_ms": med(t_pool),
        "plain_merges_per_s": merges / (med(t_plain) / 1e3),
        "pooled_merges_per_s": merges / (med(t_pool) / 1e3),
        "plain_alg_bytes": plain_alg, "pooled_alg_bytes": pool_alg,
        "pooled_frac": pool_alg / (med(t_pool) / 1e3) / 1e9 / hbm, "peak_kind": kind}
    res["note"] = ("decode: both layouts from the same records, the same inputs, graph-replayed; "
                   "the pooled read takes all 1280 pool slots per group (free and later ones "
                   "masked) where the plain one takes the bank and the filled pending slots")
    del pool
    torch.cuda.empty_cache()
    return res


def prefill_attention_flops(t0: int, T: int, c: int, p0: int) -> int:
    """Algorithmic FLOPs of one chunk's two reads (QKᵀ and PV, 2 FLOP per
    multiply-add, 16 heads, head dim 256): query i at position t0+i reads
    min(t0+i, 1023)+1 window keys and c + p0 + i + 1 anchors."""
    keys = 0
    for i in range(T):
        keys += min(t0 + i, 1023) + 1 + c + p0 + i + 1
    return keys * 16 * 256 * 2 * 2


def prefill_bench(dev, chunks: int, layers: int = LAYERS, warm_chunks: int = 2,
                  graph: bool = True):
    """Chunked prefill of one stream from position 0 in 256-token chunks through
    `layers` layers (every 4096th token scaled by 4), inputs resident before
    timing.  Returns tokens/s over the whole stream and the attention share."""
    import torch
    import sliding_window_anchor_b200 as sab
    from synth import workloads as wl
    seed = wl.seed_of(wl.PREFILL)
    T = 256
    weights = [sab.LayerWeights.from_dict(wl.make_weights(seed, l, device=dev))
               for l in range(layers)]
    st = sab.State(1, layers, device=dev)
    ws = torch.empty(sab.prefill_workspace_bytes(T), dtype=torch.uint8, device=dev)
    outs = [torch.empty(T, 2560, dtype=torch.bfloat16, device=dev) for _ in range(layers)]
    xs = [[wl.make_x(seed, l, c, range(T), device=dev, big_every=4096, first_pos=c * T)
           for l in range(layers)] for c in range(chunks)]
    stream = torch.cuda.current_stream(dev)
    seq0 = torch.zeros(1, dtype=torch.int32, device=dev)

    def run(c0, c1):
        for c in range(c0, c1):
            for l in range(layers):
                sab.swa_rma_prefill_chunk(st, weights[l], l, 0, xs[c][l], out=outs[l], ws=ws)
            sab.advance(st, seq0, T)

    # warm-up on a scratch copy of the stream start, then restart from position 0
    run(0, min(warm_chunks, chunks))
    torch.cuda.synchronize(dev)
    sab.state_init(st, seq0)
    torch.cuda.synchronize(dev)
    n0 = sab.launch_count()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    h0 = time.perf_counter()
    e0.record(stream)
    run(0, chunks)
    e1.record(stream)
    host_ms = (time.perf_counter() - h0) * 1e3  # submission time on the host
    torch.cuda.synchronize(dev)
    launches = sab.launch_count() - n0
    if sab.last_device_error(st) != 0:
        raise RuntimeError("device error in the prefill bench")
    ms = e0.elapsed_time(e1)
    # the prefill reads' own time: a second eager pass with events around each
    # read launch (the events cost host time, so this pass is not the one timed)
    sab.state_init(st, seq0)
    torch.cuda.synchronize(dev)
    sab.profile_read(reset=True)
    sab.profile_enable(True)
    run(0, chunks)
    torch.cuda.synchronize(dev)
    sab.profile_enable(False)
    attn_ms, attn_n = sab.profile_read(reset=True)
    if sab.last_device_error(st) != 0:
        raise RuntimeError("device error in the prefill bench")
    graph_ms = None
    if graph:
        # the same stream replayed from CUDA graphs, one per chunk (all layers + advance)
        stream_g = torch.cuda.Stream(dev)
        graphs = []
        for c in range(chunks):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream_g):
                run(c, c + 1)
            graphs.append(g)
        sab.state_init(st, seq0)
        torch.cuda.synchronize(dev)
        g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        g0.record(stream)
        for g in graphs:
            g.replay()
        g1.record(stream)
        torch.cuda.synchronize(dev)
        if sab.last_device_error(st) != 0:
            raise RuntimeError("device error in the prefill graph pass")
        graph_ms = g0.elapsed_time(g1)
        del graphs
    # attention FLOPs: bank and pending counts follow from the commit rule (every
    # 256 tokens the block commits into a bank capped at 1024)
    flops = 0
    for c in range(chunks):
        t0 = c * T
        bank = min(1024, t0)
        flops += prefill_attention_flops(t0, T, bank, 0)
    flops *= layers
    return {"workload": f"prefill_l{layers}_{chunks * T}tok_c256", "tokens": chunks * T,
            "layers": layers, "ms": ms, "tok_per_s": chunks * T / (ms / 1e3),
            "ms_per_chunk_layer": ms / (chunks * layers), "gpu_launches": launches,
            "attention_ms": attn_ms, "attention_launches": attn_n,
            "attention_tflops": flops / (attn_ms / 1e3) / 1e12 if attn_ms > 0 else None,
            "attention_flops": flops, "host_submit_ms": host_ms,
            "graph": None if graph_ms is None else {
                "ms": graph_ms, "tok_per_s": chunks * T / (graph_ms / 1e3),
                "note": "same chunks replayed from one captured CUDA graph per chunk"}}


# bytes every decode layer step reads from the weights: the fused q/k/v + W1-term
# matrix (13056 x 2560 BF16), W_o (2560 x 4096 BF16), W2 and the four gains
WEIGHT_BYTES_PER_LAYER = 13056 * 2560 * 2 + 2560 * 4096 * 2 + 4 * 256 * 4 + 4 * 256 * 2


def decode_config_bench(dev, workload: str, n_x: int = 16, warmup: int = 3):
    """One named decode workload end to end on the device: its state
    seeded as the tests seed it, then all of its steps (a1-a7 per layer, device-
    gated commits, the advance) replayed from CUDA graphs (one per distinct input
    buffer, inputs resident).  Reports tok/s, ms/step and the fraction of the byte
    floor (every layer step reads its weights once and its state rows once, at the
    measured HBM bandwidth); an eager pass times the read kernel's launches."""
    import torch
    import sliding_window_anchor_b200 as sab
    from synth import workloads as wl
    cfg, seed = wl.CONFIGS[workload], wl.seed_of(workload)
    Bc, L, steps, t0 = cfg["B"], cfg["n_layers"], cfg["steps"], cfg["t0"]
    weights = [sab.LayerWeights.from_dict(wl.make_weights(seed, l, device=dev))
               for l in range(L)]
    st = sab.State(Bc, L, device=dev)

    def normrope(x, g, pos):
        return sab.qk_norm_rope(x.contiguous(), g, pos.to(torch.int32).contiguous())

    fills = wl.seed_state(st.arrays(), range(Bc), L, t0, cfg["pend"], seed,
                          [w.t for w in weights], normrope, device=dev).cpu().tolist()
    snap = st.blob.clone()
    ids = torch.arange(Bc, dtype=torch.int32, device=dev)
    ws = torch.empty(sab.decode_workspace_bytes(Bc), dtype=torch.uint8, device=dev)
    n_x = min(n_x, steps)
    xs = [[wl.make_x(seed, l, s, range(Bc), device=dev) for l in range(L)] for s in range(n_x)]
    outs = [torch.empty(Bc, 2560, dtype=torch.bfloat16, device=dev) for _ in range(L)]
    stream = torch.cuda.current_stream(dev)

    def step(s):
        for l in range(L):
            sab.swa_rma_decode(st, weights[l], l, ids, xs[s % n_x][l], out=outs[l], ws=ws)
        sab.advance(st, ids)

    # eager pass over the first steps: the read kernel's own launches, timed
    for s in range(warmup):
        step(s)
    torch.cuda.synchronize(dev)
    k_eager = min(steps, 32)
    sab.profile_read(reset=True)
    sab.profile_enable(True)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for s in range(k_eager):
        step(s)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    sab.profile_enable(False)
    a_ms, a_n = sab.profile_read(reset=True)
    eager_ms = e0.elapsed_time(e1)
    a_alg = algorithmic_read_bytes(fills, warmup, k_eager) * L
    # the whole configuration from its seeded start, replayed from graphs
    st.blob.copy_(snap)
    stream_g = torch.cuda.Stream(dev)
    graphs = []
    for s in range(n_x):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream_g):
            step(s)
        graphs.append(g)
    st.blob.copy_(snap)  # capture launches nothing; restore anyway
    torch.cuda.synchronize(dev)
    g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    g0.record(stream)
    for s in range(steps):
        graphs[s % n_x].replay()
    g1.record(stream)
    torch.cuda.synchronize(dev)
    del graphs
    if sab.last_device_error(st) != 0:
        raise RuntimeError(f"device error in the {workload} bench")
    ms = g0.elapsed_time(g1)
    hbm, kind = peaks()
    state_bytes = algorithmic_read_bytes(fills, 0, steps) * L
    floor_bytes = state_bytes + steps * L * WEIGHT_BYTES_PER_LAYER
    floor_ms = floor_bytes / (hbm * 1e9) * 1e3
    commits = sum(1 for f in fills for s in range(steps) if (f + s) % 256 == 255)
    per_read = a_ms / a_n if a_n else None
    return {"workload": cfg["name"], "B": Bc, "layers": L, "t0": t0, "steps": steps,
            "tok_per_s": Bc * steps / (ms / 1e3), "ms_per_step": ms / steps,
            "ms_per_layer_step": ms / (steps * L), "commits": commits,
            "floor_ms_per_step": floor_ms / steps, "floor_frac": floor_ms / ms,
            "floor_bytes_per_step": floor_bytes / steps,
            "eager_ms_per_step": eager_ms / k_eager,
            "attend_avg_launch_ms": per_read,
            "attend_frac": (a_alg / a_n) / (per_read / 1e3) / 1e9 / hbm if a_n else None,
            "peak_gbs": hbm, "peak_kind": kind,
            "launch": "one CUDA graph per step (inputs resident, %d buffers)" % n_x}


SWEEP_BATCHES = (1, 2, 4, 8, 16, 32, 64, 96, 128, 160, 192, 224, 256, 288, 320, 352, 384, 448,
                 512)


def batch_sweep(dev, batches=SWEEP_BATCHES, steps: int = 32, warmup: int = 4):
    """One SWA∥RMA layer's decode step (a1–a7 + advance) at each batch size, on
    the decode workload (t0 = 32768, window and bank full, pending fill
    U{0..255}).  Throughput from the steps replayed out of CUDA graphs (one per
    input buffer); the read kernel's GB/s from an eager pass with its launches
    timed by CUDA events, over the algorithmic bytes of the rows it must read."""
    import torch
    import sliding_window_anchor_b200 as sab
    from synth import workloads as wl
    seed = wl.seed_of(wl.DECODE_B512)
    bmax = max(batches)
    w = sab.LayerWeights.from_dict(wl.make_weights(seed, 0, device=dev))
    st = sab.State(bmax, 1, device=dev)

    def normrope(x, g, pos):
        return sab.qk_norm_rope(x.contiguous(), g, pos.to(torch.int32).contiguous())

    fills = wl.seed_state(st.arrays(), range(bmax), 1, T0, "uniform", seed, [w.t], normrope,
                          device=dev).cpu().tolist()
    done = [0] * bmax  # steps each sequence has taken
    hbm, kind = peaks()
    stream = torch.cuda.current_stream(dev)
    n_x = 8
    rows = []
    for B in batches:
        ids = torch.arange(B, dtype=torch.int32, device=dev)
        ws = torch.empty(sab.decode_workspace_bytes(B), dtype=torch.uint8, device=dev)
        xs = [wl.make_x(seed, 0, s, range(B), device=dev) for s in range(n_x)]
        out = torch.empty(B, 2560, dtype=torch.bfloat16, device=dev)

        def step(s):
            sab.swa_rma_decode(st, w, 0, ids, xs[s % n_x], out=out, ws=ws)
            sab.advance(st, ids)

        def took(k):
            for b in range(B):
                done[b] += k

        for s in range(warmup):
            step(s)
        took(warmup)
        # eager pass: the read kernel's launches timed
        alg = 0
        for s in range(steps):
            for b in range(B):
                p = (fills[b] + done[b] + s) % 256
                alg += 4 * ((1024 + 1024 + p + 1) * ROW + 2 * 4 * 512 + 2 * 4 * 1024)
        torch.cuda.synchronize(dev)
        sab.profile_read(reset=True)
        sab.profile_enable(True)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for s in range(steps):
            step(s)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        sab.profile_enable(False)
        a_ms, a_n = sab.profile_read(reset=True)
        eager_ms = e0.elapsed_time(e1)
        took(steps)
        # graph pass
        stream_g = torch.cuda.Stream(dev)
        graphs = []
        for s in range(n_x):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream_g):
                step(s)
            graphs.append(g)
        for s in range(warmup):
            graphs[s % n_x].replay()
        took(warmup)
        torch.cuda.synchronize(dev)
        g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        g0.record(stream)
        for s in range(steps):
            graphs[s % n_x].replay()
        g1.record(stream)
        torch.cuda.synchronize(dev)
        took(steps)
        del graphs
        if sab.last_device_error(st) != 0:
            raise RuntimeError(f"device error in the sweep at B={B}")
        g_ms = g0.elapsed_time(g1)
        attend_gbs = (alg / steps) / (a_ms / a_n / 1e3) / 1e9 if a_n else None
        row = {"workload": "decode_layer_t32768", "B": B, "layers": 1, "steps": steps,
               "tok_per_s": B * steps / (g_ms / 1e3), "ms_per_step": g_ms / steps,
               "eager_ms_per_step": eager_ms / steps,
               "attend_ms": a_ms / a_n if a_n else None, "attend_gbs": attend_gbs,
               "attend_frac": attend_gbs / hbm if attend_gbs else None, "peak_kind": kind}
        print(json.dumps(row), flush=True)
        rows.append(row)
    return rows


def single_kernel(args):
    """Profiling driver: one kernel alone on a --batch workload, three launches."""
    import torch
    import synth
    import sliding_window_anchor_b200 as sab
    from synth import workloads as wl
    dev = torch.device("cuda", 0)
    B = args.batch
    if args.kernel == "attend":
        seed = 5
        w = wl.make_weights(seed, 0, device=dev)
        st = sab.State(B, 1)
        nr = lambda x, g, p: sab.qk_norm_rope(x.contiguous(), g, p.to(torch.int32).contiguous())
        fills = wl.seed_state(st.arrays(), range(B), 1, T0, "uniform", seed, [w], nr, device=dev)
        q1 = synth.normal((B, 16, 256), seed, 900, torch.bfloat16, dev)
        q2 = synth.normal((B, 16, 256), seed, 901, torch.bfloat16, dev)
        ids = torch.arange(B, dtype=torch.int32, device=dev)
        ws = torch.empty(sab.attend_workspace_bytes(B), dtype=torch.uint8, device=dev)
        ms = []
        for _ in range(7):  # the first is a warm-up
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            sab.swa_rma_attend(st, 0, ids, q1, q2, ws=ws)
            e1.record()
            torch.cuda.synchronize()
            ms.append(e0.elapsed_time(e1))
        alg = sum(4 * ((2048 + int(f) + 1) * ROW + 2 * 4 * 512 + 2 * 4 * 1024)
                  for f in fills.tolist())
        if sab.last_device_error(st) != 0:
            raise RuntimeError("device error")
        med = sorted(ms[1:])[len(ms[1:]) // 2]
        out = {"kernel": "k_attend", "batch": B, "layers": 1, "ms": med,
               "ms_launches": [round(m, 4) for m in ms[1:]], "alg_bytes": alg,
               "gbs": alg / (med / 1e3) / 1e9,
               "note": "median of 6 calls after a warm-up; each call's events include its "
                       "host-side setup (tensor maps, the work-counter reset)"}
    elif args.kernel == "score":
        w = sab.LayerWeights.from_dict(wl.make_weights(5, 0, device=dev))
        x = synth.normal((B, 2560), 5, synth.MISC, torch.bfloat16, dev)
        ws = torch.empty(sab.score_workspace_bytes(B), dtype=torch.uint8, device=dev)
        ms = []
        for _ in range(3):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            sab.rma_score(w, x, ws=ws)
            e1.record()
            torch.cuda.synchronize()
            ms.append(e0.elapsed_time(e1))
        flops = 3 * B * 2560 * 256 * 2  # the three BF16 terms of W1 on the tensor cores
        out = {"kernel": "k_score_tc", "batch": B, "ms": ms[-1], "tc_flops": flops,
               "tflops": flops / (ms[-1] / 1e3) / 1e12}
    elif args.kernel == "prefill":
        out = {"kernel": "prefill", **prefill_bench(dev, args.prefill_chunks, layers=1,
                                                    warm_chunks=1)}
    elif args.kernel == "layer":
        # the decode workload's state for one layer (t0 = 32768, pending U{0..255})
        seed = wl.seed_of(wl.DECODE_B512)
        w = sab.LayerWeights.from_dict(wl.make_weights(seed, 0, device=dev))
        st = sab.State(B, 1, device=dev)
        nr = lambda x, g, p: sab.qk_norm_rope(x.contiguous(), g, p.to(torch.int32).contiguous())
        wl.seed_state(st.arrays(), range(B), 1, T0, "uniform", seed, [w.t], nr, device=dev)
        ids = torch.arange(B, dtype=torch.int32, device=dev)
        ws = torch.empty(sab.decode_workspace_bytes(B), dtype=torch.uint8, device=dev)
        xs = [wl.make_x(seed, 0, s, range(B), device=dev) for s in range(2)]
        y = torch.empty(B, 2560, dtype=torch.bfloat16, device=dev)
        ms = []
        for i in range(7):  # the first is a warm-up
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            sab.swa_rma_decode(st, w, 0, ids, xs[i % 2], out=y, ws=ws)
            e1.record()
            sab.advance(st, ids)
            torch.cuda.synchronize()
            ms.append(e0.elapsed_time(e1))
        if sab.last_device_error(st) != 0:
            raise RuntimeError("device error")
        med = sorted(ms[1:])[len(ms[1:]) // 2]
        out = {"kernel": "layer", "batch": B, "layers": 1, "ms": med,
               "ms_calls": [round(m, 4) for m in ms[1:]],
               "note": "one decode layer call (a1-a7) per timed region, eager; median of 6"}
    else:
        st = sab.State(B, LAYERS)
        r = commit_microbench(st, dev, reps=2)
        out = {"kernel": "k_commit", "batch": B, **r}
    print(json.dumps(out), flush=True)


# ------------------------------------------------------------ CPU oracle

def oracle_tokens_per_s(budget_s=12.0, max_threads=8):
    """The oracle as it stands on the host cores: whole decode steps (8 layers) of
    independent sequences of the same workload, one sequence per thread."""
    from concurrent.futures import ThreadPoolExecutor

    import oracle
    from synth import workloads as wl

    seed = wl.seed_of(wl.DECODE_B512)
    threads = max(1, min(max_threads, os.cpu_count() or 1))
    ows = []
    for l in range(LAYERS):
        w = wl.make_weights(seed, l)
        ows.append((oracle.OracleWeights(w["w_qkv"], w["w_o"], w["q_norm_swa"], w["k_norm_swa"],
                                         w["q_norm_rma"], w["k_norm_rma"], w["w1"], w["w2"]), w))
    wdicts = [w for _, w in ows]
    states = []
    for i in range(threads):
        ost = oracle.OracleState(1, LAYERS)
        arrays = {n: getattr(ost, n) for n in oracle.OracleState.ARRAYS}
        wl.seed_state(arrays, [i], LAYERS, T0, "uniform", seed, wdicts, oracle.norm_rope)
        states.append(ost)
    xs = [[wl.make_x(seed, l, s, [i])[0] for l in range(LAYERS)] for i in range(threads)
          for s in range(1)]
    deadline = time.time() + budget_s
    counts = [0] * threads

    def work(i):
        while time.time() < deadline:
            for l in range(LAYERS):
                states[i].decode_layer(ows[l][0], l, 0, xs[i][l])
            states[i].advance(0)
            counts[i] += 1

    t0 = time.time()
    with ThreadPoolExecutor(threads) as ex:
        list(ex.map(work, range(threads)))
    dt = time.time() - t0
    return sum(counts) / dt, threads, sum(counts), dt


def oracle_merges_per_s(budget_s=4.0):
    """The oracle's commit (a full sort of the 1280 records, then the moves) on the
    commit workload, one thread: one sequence x 8 layers x 4 groups per call, each a
    freshly seeded repetition (as the GPU microbench seeds them)."""
    import oracle
    from synth import workloads as wl
    seed = wl.seed_of(wl.COMMIT)
    ost = oracle.OracleState(1, LAYERS)
    arrays = {n: getattr(ost, n) for n in oracle.OracleState.ARRAYS}
    merges, spent, rep = 0, 0.0, 0
    while spent < budget_s:
        wl.seed_commit_workload(arrays, [rep % 512], LAYERS, T0, seed, rep, "cpu")
        t0 = time.time()
        ost.commit(-1, 0)
        spent += time.time() - t0
        merges += LAYERS * 4
        rep += 1
    return merges / spent, merges, spent


def workload_config(world: int, launch: str) -> dict:
    """The workload both arms report (the reference arm's launch is the host)."""
    return {"workload": WORKLOAD, "B": B, "layers": LAYERS, "t0": T0,
            "pending_fill": "U{0..255}", "state_gib_per_gpu": 36.0,
            "l2": "inputs larger than L2 (36 GiB state per GPU), no flush",
            "parallelism": f"replicas x{world}", "launch": launch}


def reference_arm(args, rank, world):
    if rank != 0:
        return
    budget = max(3.0, min(60.0, 2.0 * (args.steps + args.warmup)))
    v, cores, toks, dt = oracle_tokens_per_s(budget_s=min(budget, 30.0))
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "tok/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": None,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": workload_config(world, "the oracle on the host cores"),
            "cpu_baseline": {"value": v, "unit": "tok/s", "cores": cores, "kind": "oracle",
                             "sample": f"{toks} whole 8-layer decode steps of {cores} sequences "
                                       f"of the workload in {dt:.1f} s"},
            "e2e": {"value": v, "unit": "tok/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ main

def main():
    args = parse()
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local_rank = int(os.environ.get("LOCAL_RANK", 0))
    if args.impl == "reference":
        reference_arm(args, rank, world)
        return
    if args.sweep:
        import torch
        batch_sweep(torch.device("cuda", 0))
        return
    if args.kernel != "step":
        single_kernel(args)
        return
    import torch
    import torch.distributed as dist
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=600),
                                device_id=torch.device("cuda", local_rank))
    r = run_ours(args, rank, world, local_rank)
    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return
    hbm, peak_kind = peaks()
    fills = r["fills"]
    alg = algorithmic_read_bytes(fills, args.warmup, args.steps) * LAYERS
    n_launch = max(r["attend_n"], 1)
    per_launch = alg / (args.steps * LAYERS)
    avg_ms = r["attend_ms"] / n_launch
    achieved = per_launch / (avg_ms / 1e3) / 1e9
    traffic = None
    tpath = os.path.join(ROOT, "profiles", "attend_traffic.json")
    if os.path.exists(tpath):
        # DRAM traffic from the committed ncu capture; null once the kernel source has changed
        import hashlib
        rec = json.load(open(tpath))
        src = os.path.join(ROOT, rec["source"])
        if hashlib.sha256(open(src, "rb").read()).hexdigest() == rec.get("source_sha256"):
            traffic = rec.get("bytes_per_launch_full")
    cpu = None
    if not args.no_cpu_baseline and world == 1:
        v, cores, toks, dt = oracle_tokens_per_s(budget_s=12.0)
        v1, _, toks1, dt1 = oracle_tokens_per_s(budget_s=6.0, max_threads=1)
        mps, merges, mdt = oracle_merges_per_s(budget_s=4.0)
        cpu = {"value": v, "unit": "tok/s", "cores": cores, "kind": "oracle",
               "sample": f"{toks} whole 8-layer decode steps of {cores} sequences of the "
                         f"workload in {dt:.1f} s",
               "single_thread": {"value": v1, "unit": "tok/s", "cores": 1,
                                 "sample": f"{toks1} whole 8-layer decode steps of one "
                                           f"sequence in {dt1:.1f} s"},
               "commit": {"value": mps, "unit": "merges/s", "cores": 1,
                          "sample": f"{merges} merges of the commit workload (top 1024 of "
                                    f"1280 by full sort, then the moves) in {mdt:.1f} s"}}
    # headline: the steps replayed from CUDA graphs when that pass ran, else the eager pass
    g = r["graph"]
    head_ms = g["ms"] if g else r["ms"]
    step_bytes = alg / args.steps + LAYERS * WEIGHT_BYTES_PER_LAYER
    head_launches = g["launches_per_step"] * args.steps if g else r["launches"]
    secs = head_ms / 1e3
    line = {
        "metric": METRIC, "value": whole_job_tokens_per_s(world, B, args.steps, head_ms),
        "unit": "tok/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": head_ms / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": workload_config(world, "one CUDA graph per step" if g else "eager"),
        "commits_per_s": world * r["commits"] / secs,
        "merges_per_s": world * r["commits"] * LAYERS * 4 / secs,
        "roofline": {"bound": "hbm", "kernel": "k_attend", "achieved": achieved, "peak": hbm,
                     "peak_kind": peak_kind, "unit": "GB/s", "frac": achieved / hbm,
                     "traffic": traffic, "alg_bytes_per_launch": per_launch,
                     "avg_launch_ms": avg_ms, "launches": r["attend_n"],
                     "above_peak": achieved > hbm,
                     "peak_test": "a read+write device copy (b.copy_(a), 1 Gi BF16 elements); "
                                  "a read-only stream can exceed it",
                     "step": {"bytes": step_bytes, "ms": head_ms / args.steps,
                              "achieved": step_bytes / (head_ms / args.steps / 1e3) / 1e9,
                              "frac": step_bytes / (head_ms / args.steps / 1e3) / 1e9 / hbm,
                              "note": "the whole step: state rows of all reads plus every "
                                      "layer's weights, over the step time"}},
        "cpu_baseline": cpu,
        "e2e": r["e2e"],
        "gpu_launches": head_launches,
        "clocks": r["clocks"],
        "commit_microbench": r["commit_microbench"],
        "prefill": r["prefill"],
        "rma_off": r["rma_off"],
        "configs": r["configs"],
        "pooled_layout": r["pool"],
        "eager": {"value": whole_job_tokens_per_s(world, B, args.steps, r["ms"]),
                  "ms_per_step": r["ms"] / args.steps, "gpu_launches": r["launches"],
                  "note": "the same steps launched call by call through the binding; "
                          "roofline timing comes from this pass"},
    }
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
