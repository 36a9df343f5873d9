#!/usr/bin/env python
"""Benchmark of the mHC decode boundary on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--no-sweep]

A boundary is one decode attention-side boundary at rows=32, H=7168,
hc_mult=4 with 8 bf16 TP-partials, an MXFP8 layer input (swizzled 128x4
scales) and the next coefficients (20 Sinkhorn iterations): the partial sum,
post-mix, collapse + RMSNorm + MXFP8 and coefficient steps in two launches
chained by programmatic dependent launch (a streaming kernel and a tail). A
step is one replay of a CUDA graph of 240 such boundaries, one after the other
on one stream, over enough distinct buffer sets (inputs, weights and outputs;
27 sets, ~0.29 GB, at rows 32) that each set is touched again only after more
than twice the 126 MB L2 of other traffic: every boundary reads HBM, not L2.
Steps are timed with CUDA events on the launching stream; the metric is
microseconds per boundary (lower is better) and the achieved HBM GB/s of the
algorithmic bytes (each input read once, each output written once).

Also reported on the same JSON line: the rows sweep 1..128 of the same boundary,
one decode step of the layer loop (61 layers: 123 chained boundaries), the
end-to-end time through the C ABI with host buffers (copies included), the CPU
oracle on the machine's host cores, and the SM clocks sampled during the timed region.

With --gpus N > 1 (one process per GPU under torchrun) every rank runs its own
replica of the workload (the boundary has no exchange step on one GPU's decode
batch); the value is the aggregate time per boundary, max over ranks.

--impl reference times the CPU oracle (the float64 restatement of the method)
as the reference arm, on rank 0 only.
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

import torch  # noqa: E402

ROWS, HIDDEN, HC, PARTIALS = 32, 7168, 4, 8
L2_BYTES = 126 * 1024 * 1024
FALLBACK_HBM_GBS = 6650.0
METRIC = "µs/boundary and achieved HBM GB/s (% of B200 peak) at rows 1–128, H=7168, n=4"


def boundary_bytes(R, H=HIDDEN, n=HC, P=PARTIALS, mxfp8=True, coeff=True, scale_bytes=None):
    """Algorithmic bytes of one partial-sum boundary: each input read once, each output written once."""
    C = 2 * n + n * n
    b = P * R * H * 2            # partials
    b += R * n * H * 2 * 2       # residual in + out
    b += R * (2 * n + n * n) * 4  # post, comb, pre
    b += H * 2 + R * H * 2       # norm_weight, layer_input
    if coeff:
        b += n * H * C * 4 + (3 + C) * 4 + R * (2 * n + n * n) * 4  # fn, scale, base; coefficients out
    if mxfp8:
        b += R * H + (scale_bytes if scale_bytes is not None else ((R + 127) // 128 * 128) * ((H // 32 + 3) // 4 * 4))
    return b


def sets_for(R):
    """Distinct buffer sets so that one pass over them moves more than twice the L2 size."""
    return max(4, -(-int(2.2 * L2_BYTES) // boundary_bytes(R)))


def load_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def load_traffic():
    """DRAM bytes per launch of the boundary kernel from the committed ncu summary,
    or None when the kernel sources changed since it was taken."""
    from mhc_residual_stream_b200 import build
    p = os.path.join(ROOT, "profiles", "boundary_kernel_traffic.json")
    try:
        with open(p) as f:
            t = json.load(f)
        if t.get("source_sha256") == build.source_digest():
            return t.get("dram_bytes_per_launch")
    except Exception:
        pass
    return None


# ---------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi samples of this GPU's clocks and throttle reasons while running."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device):
        self.samples = []
        self.proc = None
        try:
            uuid = str(torch.cuda.get_device_properties(device).uuid)
            self.ident = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
        except Exception:
            self.ident = None

    def start(self):
        if self.ident is None:
            return
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.ident, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) >= 8:
                self.samples.append(parts)

    def stop(self):
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.thread.join(timeout=5)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        sm = [float(s[0]) for s in self.samples if s[0].replace(".", "").isdigit()]
        mx = [float(s[1]) for s in self.samples if s[1].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for s in self.samples for i in range(4) if s[4 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(self.samples)}


# ---------------------------------------------------------------- our arm

# fn is packed once, at weight-load time, into the projection's bf16-term tiles
# (mhc_projection_pack); --unpacked-fn times the kernels splitting fp32 fn per call
PACK_FN = True


class BoundarySet:
    """Device buffers of one boundary of the benchmark workload."""

    def __init__(self, R, seed, device, mxfp8=True):
        from mhc_residual_stream_b200 import mhc as M
        from mhc_residual_stream_b200 import synthetic as S
        d = S.draw_boundary(R, HIDDEN, n=HC, partials=PARTIALS, seed=seed)
        self.host = d
        self.partials = d["partials"].to(device)
        self.residual = d["residual"].to(device)
        self.post = d["post"].to(device)
        self.comb = d["comb"].to(device)
        self.pre = d["pre"].to(device)
        self.norm_weight = d["norm_weight"].to(device)
        self.coeffs = M.Coeffs.from_weights(d["coeff"], device, packed=PACK_FN)
        if PACK_FN:
            self.coeffs.fn = None  # the kernels read the packed form only
        self.residual_out = torch.empty_like(self.residual)
        self.layer_input = torch.empty(R, HIDDEN, dtype=torch.bfloat16, device=device)
        self.q_data = torch.empty(R, HIDDEN, dtype=torch.uint8, device=device) if mxfp8 else None
        self.q_scale = (torch.empty(M.mhc_mxfp8_scale_bytes(R, HIDDEN, True), dtype=torch.uint8, device=device)
                        if mxfp8 else None)
        self.post_out = torch.empty_like(self.post)
        self.comb_out = torch.empty_like(self.comb)
        self.pre_out = torch.empty_like(self.pre)

    def launch(self, ws, stream=None):
        from mhc_residual_stream_b200 import mhc as M
        M.mhc_boundary_post_pre(self.partials, self.residual, self.post, self.comb, self.pre, self.norm_weight,
                                1e-6, self.coeffs, self.residual_out, layer_input=self.layer_input,
                                mxfp8=None if self.q_data is None else (self.q_data, self.q_scale, True),
                                post_out=self.post_out, comb_out=self.comb_out, pre_out=self.pre_out,
                                workspace=ws, stream=stream)


def capture(fn, n):
    """A CUDA graph of n calls of fn(i)."""
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        fn(0)  # a launch outside the capture on the capture's stream (initialisation)
    torch.cuda.current_stream().wait_stream(s)
    with torch.cuda.graph(g):
        for i in range(n):
            fn(i)
    return g


GRAPH_LEN = 240  # boundaries per step (one graph replay)


def step_graph(sets, ws, graph_len=GRAPH_LEN):
    """The step: a CUDA graph of graph_len boundaries rotating over `sets`."""
    nset = len(sets)
    return capture(lambda i: sets[i % nset].launch(ws), graph_len)


def run_timed(graph, steps, warmup, sampler=None):
    """`warmup` untimed replays, then the elapsed ms of `steps` replays on the launching stream."""
    for _ in range(warmup):
        graph.replay()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    if sampler:
        sampler.start()
        time.sleep(0.3)
    torch.cuda._sleep(2_000_000)  # keep the GPU busy while the replays are queued behind the start event
    start.record()
    for _ in range(steps):
        graph.replay()
    end.record()
    torch.cuda.synchronize()
    if sampler:
        sampler.stop()
    return start.elapsed_time(end)


def launch_floor_us(reps=20, graph_len=240):
    """Device time of one empty kernel as a CUDA-graph node (the launch floor): a
    graph of graph_len zero-length spin kernels, median over reps replays."""
    g = capture(lambda i: torch.cuda._sleep(0), graph_len)
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    times = []
    for _ in range(reps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        g.replay()
        b.record()
        torch.cuda.synchronize()
        times.append(a.elapsed_time(b) * 1000.0 / graph_len)
    return statistics.median(times)


E2E_INPUTS = ("partials", "residual", "post", "comb", "pre")
E2E_OUTPUTS = ("residual_out", "layer_input", "q_data", "q_scale", "post_out", "comb_out", "pre_out")


def _arena_views(like, keys, buf):
    """Views of the uint8 buffer `buf` shaped like `like`'s tensors `keys`, each 256-byte aligned."""
    views, off = {}, 0
    for k in keys:
        t = getattr(like, k)
        nb = t.numel() * t.element_size()
        views[k] = buf[off:off + nb].view(t.dtype).view(t.shape)
        off += (nb + 255) // 256 * 256
    return views


def _arena_bytes(like, keys):
    return sum((getattr(like, k).numel() * getattr(like, k).element_size() + 255) // 256 * 256 for k in keys)


def e2e_time(bset, ws, steps, device):
    """Per boundary through the C ABI with host buffers. Every step copies its inputs
    (partials, streams, mixes) from one pinned host staging buffer to the device,
    runs the boundary, and copies every output back into a pinned host buffer, all
    inside the timed region. The inputs and outputs of a step live in one device
    buffer each (two slots, used by alternate steps), so a step is one host-to-device
    copy, the two kernels and one device-to-host copy; the copies run on their own
    streams, so the next step's upload overlaps this step's boundary and download.
    The weights stay resident, as they would in a model. Median of three timed runs;
    also returns the last step's downloaded outputs (views of the host buffer)."""
    import copy
    nin, nout = _arena_bytes(bset, E2E_INPUTS), _arena_bytes(bset, E2E_OUTPUTS)
    h_in = torch.empty(nin, dtype=torch.uint8).pin_memory()
    for k, v in _arena_views(bset, E2E_INPUTS, h_in).items():
        v.copy_(getattr(bset, k).cpu())
    h_out = torch.empty(nout, dtype=torch.uint8).pin_memory()
    slots = []
    for _ in range(2):
        b = copy.copy(bset)
        d_in = torch.empty(nin, dtype=torch.uint8, device=device)
        d_out = torch.empty(nout, dtype=torch.uint8, device=device)
        for keys, buf in ((E2E_INPUTS, d_in), (E2E_OUTPUTS, d_out)):
            for k, v in _arena_views(bset, keys, buf).items():
                setattr(b, k, v)
        slots.append((b, d_in, d_out))
    main = torch.cuda.current_stream()
    s_in, s_run, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    in_done = [torch.cuda.Event() for _ in range(2)]
    run_done = [torch.cuda.Event() for _ in range(2)]
    out_done = [torch.cuda.Event() for _ in range(2)]
    for ev in run_done + out_done:
        ev.record(main)
    for st in (s_in, s_run, s_out):
        st.wait_stream(main)

    def step(i):
        j = i & 1
        b, d_in, d_out = slots[j]
        s_in.wait_event(run_done[j])  # the slot's inputs are free again
        with torch.cuda.stream(s_in):
            d_in.copy_(h_in, non_blocking=True)
        in_done[j].record(s_in)
        s_run.wait_event(in_done[j])
        s_run.wait_event(out_done[j])  # the slot's outputs have been read out
        with torch.cuda.stream(s_run):
            b.launch(ws)
        run_done[j].record(s_run)
        s_out.wait_event(run_done[j])
        with torch.cuda.stream(s_out):
            h_out.copy_(d_out, non_blocking=True)
        out_done[j].record(s_out)

    for i in range(100):  # warm-up: the first copies from freshly pinned pages are slower
        step(i)
    torch.cuda.synchronize()
    runs = []
    for _ in range(3):  # the host's PCIe is shared with other jobs: the median of three runs
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        start.record(main)
        for st in (s_in, s_run, s_out):
            st.wait_stream(main)
        for i in range(steps):
            step(i)
        for st in (s_in, s_run, s_out):
            main.wait_stream(st)
        end.record(main)
        torch.cuda.synchronize()
        runs.append(start.elapsed_time(end) * 1000.0 / steps)
    return statistics.median(runs), nin, nout, _arena_views(bset, E2E_OUTPUTS, h_out)


def cpu_baseline(budget_s=12.0):
    """The oracle (float64, as it stands) on the benchmark boundary, on this host's cores."""
    import threadpoolctl
    import oracle as O
    from mhc_residual_stream_b200 import synthetic as S
    d = S.draw_boundary(ROWS, HIDDEN, n=HC, partials=PARTIALS, seed=2032)
    f = {k: d[k].double().numpy() for k in ("partials", "residual", "post", "comb", "pre", "norm_weight")}
    cw = {k: (v.double().numpy() if isinstance(v, torch.Tensor) else v) for k, v in d["coeff"].as_dict().items()}
    cores = len(os.sched_getaffinity(0))
    blas = max([i.get("num_threads", 1) for i in threadpoolctl.threadpool_info()] + [1])
    times = []
    t_end = time.perf_counter() + budget_s
    while True:
        t0 = time.perf_counter()
        O.boundary(partials=f["partials"], residual=f["residual"], post=f["post"], comb=f["comb"], pre=f["pre"],
                   norm_weight=f["norm_weight"], norm_eps=1e-6, coeff=cw, mxfp8=True, swizzled=True)
        times.append(time.perf_counter() - t0)
        if time.perf_counter() > t_end or len(times) >= 200:
            break
    us = statistics.median(times) * 1e6
    one = []  # the same on one thread
    with threadpoolctl.threadpool_limits(limits=1):
        t_end = time.perf_counter() + budget_s / 2
        while True:
            t0 = time.perf_counter()
            O.boundary(partials=f["partials"], residual=f["residual"], post=f["post"], comb=f["comb"],
                       pre=f["pre"], norm_weight=f["norm_weight"], norm_eps=1e-6, coeff=cw, mxfp8=True,
                       swizzled=True)
            one.append(time.perf_counter() - t0)
            if time.perf_counter() > t_end or len(one) >= 100:
                break
    return {"value": round(us, 1), "unit": "µs/boundary", "cores": cores, "kind": "oracle",
            "single_thread_value": round(statistics.median(one) * 1e6, 1),
            "sample": f"{len(times)} full boundaries (rows 32, H 7168, n 4, P 8, MXFP8, coefficients), median; "
                      f"numpy float64 on {cores} available cores (BLAS threads {blas}); single_thread_value: "
                      f"{len(one)} more on 1 thread"}


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    return world, rank, local


def max_over_ranks(x, world):
    """Largest value over the ranks (every rank gets it); device-timed numbers use this."""
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_us_per_boundary(ms_max, steps, world):
    """Whole-job time per boundary: the slowest rank's elapsed time over all ranks' boundaries."""
    return ms_max * 1000.0 / (steps * world)


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def ours(args):
    from mhc_residual_stream_b200 import build
    from mhc_residual_stream_b200 import mhc as M
    world, rank, local = dist_setup(args)
    build.build()
    M.lib()
    device = torch.device("cuda", local if world > 1 else torch.cuda.current_device())
    torch.cuda.set_device(device)
    peak, peak_kind = load_peak()

    nsets = sets_for(ROWS)
    sets = [BoundarySet(ROWS, 900000 + 97 * i + 1000 * rank, device) for i in range(nsets)]
    ws = M.new_workspace(ROWS, HIDDEN, HC, device)
    set_bytes = sum(t.numel() * t.element_size() for s in sets[:1] for t in
                    (s.partials, s.residual, s.coeffs.fn if s.coeffs.fn is not None else s.coeffs.fn_packed,
                     s.residual_out, s.layer_input, s.q_data))
    assert set_bytes * nsets > 2 * L2_BYTES
    graph = step_graph(sets, ws)
    sampler = ClockSampler(device) if rank == 0 else None
    barrier(world)
    ms = run_timed(graph, args.steps, args.warmup, sampler)
    ms = max_over_ranks(ms, world)
    st = M.mhc_get_device_status(ws)
    if st != M.OK:
        raise RuntimeError(f"device status {M.STATUS_NAMES[st]}")
    boundaries = args.steps * GRAPH_LEN
    us_per = aggregate_us_per_boundary(ms, boundaries, world)
    us_kernel = ms * 1000.0 / boundaries                 # per launch on one GPU
    bpb = boundary_bytes(ROWS)
    achieved = bpb / (us_kernel * 1e-6) / 1e9

    result = {
        "metric": METRIC, "value": round(us_per, 4), "unit": "µs/boundary", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms / args.steps, 6),
        "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded; decode attention-side boundary inputs, no trained weights)",
        "config": {"workload": "decode attention-side boundary: rows 32, H 7168, hc_mult 4, 8 bf16 partials, "
                               "MXFP8 layer input (swizzled 128x4), coefficients with 20 Sinkhorn iterations",
                   "rows": ROWS, "hidden": HIDDEN, "hc_mult": HC, "partials": PARTIALS,
                   "step": f"one CUDA-graph replay of {GRAPH_LEN} boundaries on one stream "
                           f"({boundaries} boundaries timed)",
                   "l2": f"inputs larger than L2: {nsets} rotating buffer sets, {set_bytes * nsets / 1e6:.0f} MB; "
                         "a set is reused only after more than twice the L2 size of other traffic",
                   "timing": "CUDA events on the launching stream around the timed replays",
                   "fn": ("packed once at weight load (mhc_projection_pack)" if PACK_FN
                          else "fp32, split into bf16 terms in every call"),
                   "parallelism": f"replicas x{world}"},
        "gb_per_s": round(achieved * world, 1),
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(achieved / peak, 4), "frac_of_nominal_8000": round(achieved / 8000.0, 4),
                     "traffic": load_traffic(),
                     "algorithmic_bytes": bpb, "peak_kind": f"{peak_kind} (copy bandwidth)",
                     "kernel": "boundary_kernel<4, partials> + boundary_tail_kernel<4>: the two launches "
                               "of one boundary, timed together (CUDA events around graph replays); traffic "
                               "is the streaming kernel's DRAM bytes per launch (the tail reads L2)"},
        "gpu_launches": 2 * boundaries,
    }
    if sampler is not None:
        result["clocks"] = sampler.summary()
    lf = launch_floor_us()
    result["launch_floor"] = {"us_per_kernel": round(lf, 3), "kernels_per_boundary": 2,
                              "us_per_boundary": round(2 * lf, 3),
                              "how": "CUDA graph of 240 empty kernels (torch.cuda._sleep(0)), median of 20 replays"}

    if not args.no_sweep:
        sweep = {}
        for R in (1, 2, 4, 8, 16, 32, 64, 128):
            ss = [BoundarySet(R, 800000 + 131 * i + R, device) for i in range(sets_for(R))]
            wsr = M.new_workspace(R, HIDDEN, HC, device)
            gr = step_graph(ss, wsr)
            reps = max(3, min(args.steps, 100))
            msr = run_timed(gr, reps, 3)
            if M.mhc_get_device_status(wsr) != M.OK:
                raise RuntimeError(f"rows {R}: device status")
            us = msr * 1000.0 / (reps * GRAPH_LEN)
            gbs = boundary_bytes(R) / (us * 1e-6) / 1e9
            sweep[str(R)] = {"us": round(us, 3), "gb_per_s": round(gbs, 1), "frac": round(gbs / peak, 4),
                             "algorithmic_bytes": boundary_bytes(R), "sets": len(ss)}
            del ss, gr
        result["rows_sweep"] = sweep
        # one decode step: the 123 chained boundaries of the 61-layer loop at rows 32
        from mhc_residual_stream_b200.decode import DecodeLoop
        loop = DecodeLoop(rows=ROWS, device=str(device), pack_fn=PACK_FN)
        g = capture(lambda i: loop.run(), 1)
        for _ in range(3):
            g.replay()
        torch.cuda.synchronize()
        reps = 20
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda._sleep(2_000_000)
        start.record()
        for _ in range(reps):
            g.replay()
        end.record()
        torch.cuda.synchronize()
        us_step = start.elapsed_time(end) * 1000.0 / reps
        lb = loop.algorithmic_bytes()
        result["decode_step"] = {"boundaries": len(loop.steps), "us": round(us_step, 2),
                                 "us_per_boundary": round(us_step / len(loop.steps), 3),
                                 "gb_per_s": round(lb / (us_step * 1e-6) / 1e9, 1), "algorithmic_bytes": lb}
        if M.mhc_get_device_status(loop.workspace) != M.OK:
            raise RuntimeError("decode loop device status")

    e2e_us, h2d, d2h, _ = e2e_time(sets[0], ws, 200, device)
    e2e_us = max_over_ranks(e2e_us, world) / world
    result["e2e"] = {"value": round(e2e_us, 2), "unit": "µs/boundary", "h2d_bytes_per_step": h2d,
                     "d2h_bytes_per_step": d2h}
    if rank == 0 and world == 1 and not args.no_cpu:
        result["cpu_baseline"] = cpu_baseline()
    barrier(world)
    if rank == 0:
        print(json.dumps(result), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def reference(args):
    """The reference arm: the CPU oracle, on rank 0 only, on this machine's host cores."""
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return
    import threadpoolctl
    import oracle as O
    from mhc_residual_stream_b200 import synthetic as S
    d = S.draw_boundary(ROWS, HIDDEN, n=HC, partials=PARTIALS, seed=2032)
    f = {k: d[k].double().numpy() for k in ("partials", "residual", "post", "comb", "pre", "norm_weight")}
    cw = {k: (v.double().numpy() if isinstance(v, torch.Tensor) else v) for k, v in d["coeff"].as_dict().items()}

    def step():
        O.boundary(partials=f["partials"], residual=f["residual"], post=f["post"], comb=f["comb"], pre=f["pre"],
                   norm_weight=f["norm_weight"], norm_eps=1e-6, coeff=cw, mxfp8=True, swizzled=True)

    for _ in range(min(args.warmup, 3)):
        step()
    budget = 90.0
    t0 = time.perf_counter()
    done = 0
    while done < args.steps:
        step()
        done += 1
        if time.perf_counter() - t0 > budget:
            break
    el = time.perf_counter() - t0
    us = el * 1e6 / done
    cores = len(os.sched_getaffinity(0))
    sample = (f"{done} of {args.steps} requested boundaries timed (bounded at {budget:.0f} s); "
              "full rows-32 boundary each")
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": round(us, 1), "unit": "µs/boundary",
        "n_gpus": world, "steps": done, "warmup": min(args.warmup, 3), "ms_per_step": round(us / 1000, 3),
        "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded)",
        "config": {"workload": "decode attention-side boundary: rows 32, H 7168, hc_mult 4, 8 bf16 partials, "
                               "MXFP8 layer input (swizzled 128x4), coefficients with 20 Sinkhorn iterations",
                   "rows": ROWS, "hidden": HIDDEN, "hc_mult": HC, "partials": PARTIALS},
        "cpu_baseline": {"value": round(us, 1), "unit": "µs/boundary", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(us, 1), "unit": "µs/boundary", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


def phases(args):
    """Per-phase clock stamps of chained boundaries (a stamped copy of the library,
    built into a temporary directory): one markdown table row per row count."""
    from mhc_residual_stream_b200 import mhc as M
    from mhc_residual_stream_b200 import phase_stamps as PS
    M.LIB_PATH = PS.build_stamped()
    L = M.lib()
    device = torch.device("cuda", 0)
    G = HIDDEN // 64
    keys = [k for k, _ in PS.PHASES]
    print("| rows | µs / boundary (stamped copy) | " + " | ".join(keys) + " |")
    print("|---" * (len(keys) + 2) + "|")
    for R in args.phases:
        sets = [BoundarySet(R, 500 + i, device) for i in range(sets_for(R))]
        if args.shared_inputs:  # every boundary reads set 0's inputs and weights, which stay in L2
            for s in sets[1:]:
                s.partials, s.residual, s.coeffs = sets[0].partials, sets[0].residual, sets[0].coeffs
                s.post, s.comb, s.pre, s.norm_weight = sets[0].post, sets[0].comb, sets[0].pre, sets[0].norm_weight
        ws = M.new_workspace(R, HIDDEN, HC, device)
        graph = step_graph(sets, ws)
        run_timed(graph, 3, args.warmup)
        PS.reset(L)  # every block's ring starts with the timed replays
        ms = run_timed(graph, args.steps, 0)
        if M.mhc_get_device_status(ws) != M.OK:
            raise RuntimeError(f"rows {R}: device status")
        S, T = PS.read(L)
        ph = PS.summary(S, T, G)
        us = ms * 1000.0 / (args.steps * GRAPH_LEN)
        print(f"| {R} | {us:.2f} | " + " | ".join("-" if ph[k] is None else f"{ph[k] / 1000:.2f}" for k in keys) + " |",
              flush=True)
        del sets, graph


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100, help=f"timed steps (graph replays of {GRAPH_LEN} boundaries)")
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--no-sweep", action="store_true", help="skip the rows sweep and the decode-loop step")
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU oracle baseline")
    ap.add_argument("--unpacked-fn", action="store_true",
                    help="pass fp32 fn (split into bf16 terms in every call) instead of the packed form")
    ap.add_argument("--phases", type=int, nargs="+", metavar="ROWS",
                    help="instead of the benchmark: per-phase clock stamps (µs after the streaming kernel's "
                         "wait) of chained boundaries at these row counts, from a stamped copy of the library")
    ap.add_argument("--shared-inputs", action="store_true",
                    help="with --phases: every boundary reads the same inputs and weights, so that they stay in L2 "
                         "(a bound on what the HBM traffic costs; not a benchmark of the workload)")
    args = ap.parse_args()
    global PACK_FN
    PACK_FN = not args.unpacked_fn
    if args.warmup < 3:
        args.warmup = 3
    if args.phases:
        phases(args)
    elif args.impl == "reference":
        reference(args)
    else:
        ours(args)


if __name__ == "__main__":
    main()
