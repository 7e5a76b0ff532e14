"""Benchmark of the quantized-linear hot path on B200.

Headline workload (one step): the decode / MTP / verify MLP projections of a
27B-class decoder layer -- gate+up 34816x5120 in Q4 group-64 then down
5120x17408 in Q5 group-64 (FP16 scales), BF16 activations ~N(0,1) with 0.5%
outlier channels, weights ~N(0,0.02) with 1% outlier rows -- at T = 1, 4, 17
and 33 tokens: eight qlin_gemv calls.  The metric is weight-streaming GB/s:
algorithmic bytes (packed codes + high bits + scales + x + y) over device time.

Other rows of the path are measured in the same run and reported under
"rows": packing, MXFP8 decode, the Q8 group-32 and FP8-row head GEMVs, the
activation quantizer, the int8 prefill GEMM (2048 tokens) and the one-layer
prefill sweep (T = 512, 1792, 8192) with the GDN a/b BF16 projection.

python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
Under torchrun every rank runs the same workload independently (replicas, no
collective in the data path); timing is the max over ranks.
"""
import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

T_LIST = (1, 4, 17, 33)
GATE_UP = (34816, 5120)
DOWN = (5120, 17408)
# Weight copies: the step's call pair at T_LIST[i] (gate+up then down) uses
# copy i, so a matrix is read again only after the other seven calls of the
# step (3 x 153.2 + 58.5 = 518 MB of other weights, 4x the 126 MB L2).
L2_COPIES = len(T_LIST)
L2_BYTES = 126 * 1024 * 1024
NOMINAL_HBM_GBS = 8000.0  # the ~8 TB/s HBM3e figure the GEMV target is stated against
METRIC = "GEMV weight GB/s & % HBM peak (T=1..33); prefill int8 TOPS & % peak"


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--no-rows", action="store_true", help="skip the per-row measurements")
    p.add_argument("--cpu-seconds", type=float, default=12.0, help="target CPU work of the oracle sample")
    p.add_argument("--case", default=None,
                   help="run one kernel case only (for profilers): gemv:<q3|q4|q5|q6|q8|fp8|bf16>:<N>x<K>:T<t> "
                        "or gemm_fp8:<N>x<K>:T<t> "
                        "or gemm_a8:<q3|q4|q5|q6>:<N>x<K>:T<t> or quantize:<T>x<K> or decode:<R>x<C>")
    return p.parse_args()


def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), float(d.get("bf16_tflops_sustained", 0)), "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


# ---------------------------------------------------------------------------
# distributed plumbing (replicas)
# ---------------------------------------------------------------------------
class Dist:
    def __init__(self, n):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.pg = None
        if self.world > 1:
            import datetime
            import torch.distributed as dist
            backend = "nccl" if torch.cuda.is_available() else "gloo"
            if torch.cuda.is_available():
                torch.cuda.set_device(self.local)
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
            self.pg = dist

    def barrier(self):
        if self.pg:
            self.pg.barrier()

    def max(self, v):
        if not self.pg:
            return v
        dev = "cuda" if torch.cuda.is_available() else "cpu"
        t = torch.tensor([v], dtype=torch.float64, device=dev)
        self.pg.all_reduce(t, op=self.pg.ReduceOp.MAX)
        return float(t.item())

    def sum(self, v):
        if not self.pg:
            return v
        dev = "cuda" if torch.cuda.is_available() else "cpu"
        t = torch.tensor([v], dtype=torch.float64, device=dev)
        self.pg.all_reduce(t, op=self.pg.ReduceOp.SUM)
        return float(t.item())

    def close(self):
        if self.pg:
            self.pg.destroy_process_group()


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------
class Clocks:
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        try:
            self.index = "GPU-" + str(torch.cuda.get_device_properties(device_index).uuid)
        except Exception:
            self.index = str(device_index)
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=self.fh, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if not self.proc:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.fh.close()
        sm, mx, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    mx = max(mx, float(parts[2]))
                except ValueError:
                    continue
                for nm, val in zip(names, parts[5:9]):
                    if val.lower().startswith("active"):
                        reasons.add(nm)
        os.unlink(self.path)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------------
# workload construction (on the device, seeded)
# ---------------------------------------------------------------------------
def packed(q, synth, fmt, n, k, seed, dev, allow_a8=False):
    w = synth.weights_f32(n, k, seed=seed, device=dev)
    pw = q.PackedWeights(fmt, n, k, device=dev, allow_a8=allow_a8)
    q.qlin_pack_weights(q.SRC_F32, w, pw)
    del w
    return pw


def measured_traffic(key):
    """DRAM bytes (read + write) per launch from an ncu capture summarised in
    profiles/traffic.json; None when the kernel source changed since then."""
    import hashlib
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            entry = json.load(f)[key]
        h = hashlib.sha256()
        for rel in entry["sources"]:
            with open(os.path.join(ROOT, rel), "rb") as f:
                h.update(f.read())
        if h.hexdigest() != entry["sources_sha256"]:
            return None
        return entry["dram_bytes_per_launch"]
    except Exception:
        return None


def gemv_bytes(pw, t):
    return pw.bytes() + 2 * t * pw.k + 2 * t * pw.n


def sleep_ahead(n_calls):
    """Hold the stream in a device-side spin (~0.1 ms per call about to be
    queued) so the host queues every following launch before the device gets
    to it: the device then runs them back to back and events around each one
    time the kernel, not the host's launch overhead."""
    torch.cuda._sleep(int(2e5 * max(1, n_calls)))


class Timer:
    """CUDA events on the launching stream around each call."""

    def __init__(self):
        self.pairs = []

    def run(self, fn):
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record()
        fn()
        e.record()
        self.pairs.append((s, e))

    def total_ms(self):
        return sum(s.elapsed_time(e) for s, e in self.pairs)


def count_our_launches(fn):
    """Number of kernels from libqlin (namespace qlin) that one call of fn launches."""
    from torch.profiler import ProfilerActivity, profile
    torch.cuda.synchronize()
    with profile(activities=[ProfilerActivity.CUDA]) as prof:
        fn()
        torch.cuda.synchronize()
    n = 0
    for ev in prof.events():
        if ev.device_type.name == "CUDA" and "qlin" in ev.name:
            n += 1
    return n


def run_ours(args, dist):
    import quantized_weight_linear_qlin_b200 as q
    import synth
    from quantized_weight_linear_qlin_b200 import _build
    _build.build()
    q.lib()
    dev = torch.device("cuda", dist.local)
    torch.cuda.set_device(dev)
    hbm, bf16_tf, bf16_tf_sus, peak_kind = measured_peaks()

    # ---- headline workload: decode MLP, Q4 gate+up then Q5 down, rotating copies
    copies = []
    for c in range(L2_COPIES):
        gu = packed(q, synth, q.Q4_G64, *GATE_UP, synth.seed_for(1, 10 + c), dev)
        dn = packed(q, synth, q.Q5_G64, *DOWN, synth.seed_for(1, 20 + c), dev)
        copies.append((gu, dn))
    xs_gu = {t: synth.activations_bf16(t, GATE_UP[1], seed=synth.seed_for(1, 30 + t), device=dev) for t in T_LIST}
    xs_dn = {t: synth.activations_bf16(t, DOWN[1], seed=synth.seed_for(1, 60 + t), device=dev) for t in T_LIST}
    ys_gu = {t: torch.empty(t, GATE_UP[0], dtype=torch.bfloat16, device=dev) for t in T_LIST}
    ys_dn = {t: torch.empty(t, DOWN[0], dtype=torch.bfloat16, device=dev) for t in T_LIST}
    ws = q.Workspace(dev)
    for gu, dn in copies:
        for t in T_LIST:
            ws.ensure(q.qlin_gemv_workspace_bytes(gu, t))
            ws.ensure(q.qlin_gemv_workspace_bytes(dn, t))
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    step_bytes = sum(gemv_bytes(copies[0][0], t) + gemv_bytes(copies[0][1], t) for t in T_LIST)
    gu_b, dn_b = copies[0][0].bytes(), copies[0][1].bytes()
    reuse_mb = min((L2_COPIES - 1) * (gu_b + dn_b) + dn_b, (L2_COPIES - 1) * (gu_b + dn_b) + gu_b) / 1e6
    launches_per_call = {}

    def step(i, timer=None):
        for ti, t in enumerate(T_LIST):
            gu, dn = copies[ti]
            for pw, x, y in ((gu, xs_gu[t], ys_gu[t]), (dn, xs_dn[t], ys_dn[t])):
                f = (lambda pw=pw, x=x, y=y: q.qlin_gemv(pw, x, y, q.OUT_BF16, workspace=ws, dev_status=status))
                if timer:
                    timer.run(f)
                else:
                    f()

    clocks = Clocks(dist.local)
    clocks.start()  # sampling covers the warm-up (at least ~1 s of this load) and the timed region
    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    # one CUDA graph holds a whole step (8 launches), so the timed region is
    # device work only
    cap = torch.cuda.Stream()
    cap.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=cap):
        step(0)
    torch.cuda.synchronize()
    t_settle = time.perf_counter()
    i = 0
    while time.perf_counter() - t_settle < 1.0:
        graph.replay()
        i += 1
        if i % 50 == 0:
            torch.cuda.synchronize()
    torch.cuda.synchronize()
    dist.barrier()
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record()
    for i in range(args.steps):
        graph.replay()
    end.record()
    torch.cuda.synchronize()
    dist.barrier()
    clk = clocks.stop()
    ms = dist.max(start.elapsed_time(end))
    # per-call event timing pass (same work, used for the kernel roofline):
    # direct calls queued behind a device spin, events around each call
    timer = Timer()
    sleep_ahead(args.steps * 2 * len(T_LIST))
    for i in range(args.steps):
        step(i, timer)
    torch.cuda.synchronize()
    call_ms = timer.total_ms() / args.steps
    # host time of one qlin_gemv call through the binding (calls queued behind
    # a device spin, no events)
    n_host = 4 * args.steps * 2 * len(T_LIST)
    sleep_ahead(n_host)
    t_host = time.perf_counter()
    for i in range(4 * args.steps):
        step(i)
    host_us_per_call = (time.perf_counter() - t_host) / n_host * 1e6
    torch.cuda.synchronize()
    del graph
    assert status.item() == 0, "device wait timed out"

    ms_per_step = ms / args.steps
    total_units = dist.sum(step_bytes * args.steps)
    value = total_units / (ms / 1e3) / 1e9

    # launches of our kernels in one step, counted by the CUDA profiler
    launches = count_our_launches(lambda: step(0)) * args.steps

    # ---- e2e: through the public API with pinned host buffers.  Each step's
    # eight activation tensors go up in one host-to-device copy and its eight
    # results come back in one device-to-host copy, each direction on a copy
    # stream of its own (the two directions run at once): the inputs of step
    # i+1 (double-buffered) move while step i computes, and the results of
    # step i while step i+1 computes, as a serving loop would overlap them.
    xs_list = [x for t in T_LIST for x in (xs_gu[t], xs_dn[t])]
    ys_list = [y for t in T_LIST for y in (ys_gu[t], ys_dn[t])]
    hx_all = torch.cat([x.reshape(-1) for x in xs_list]).cpu().pin_memory()
    n_y = sum(y.numel() for y in ys_list)
    dx_all = [torch.empty_like(hx_all, device=dev) for _ in range(2)]
    dy_all = [torch.empty(n_y, dtype=torch.bfloat16, device=dev) for _ in range(2)]
    hy_all = torch.empty(n_y, dtype=torch.bfloat16).pin_memory()

    def views(flat, shapes):
        out, o = [], 0
        for shp in shapes:
            n = shp[0] * shp[1]
            out.append(flat[o:o + n].view(shp))
            o += n
        return out
    dxv = [views(b, [tuple(x.shape) for x in xs_list]) for b in dx_all]
    dyv = [views(b, [tuple(y.shape) for y in ys_list]) for b in dy_all]
    h2d = hx_all.numel() * 2
    d2h = hy_all.numel() * 2
    main = torch.cuda.current_stream()
    up, down = torch.cuda.Stream(), torch.cuda.Stream()
    h2d_done = [torch.cuda.Event() for _ in range(2)]
    comp_done = [torch.cuda.Event() for _ in range(2)]
    d2h_done = [torch.cuda.Event() for _ in range(2)]

    def e2e_run(n):
        up.wait_stream(main)
        down.wait_stream(main)
        for i in range(n):
            b = i & 1
            if i >= 2:
                up.wait_event(comp_done[b])  # step i-2 has read input buffer b
            with torch.cuda.stream(up):
                dx_all[b].copy_(hx_all, non_blocking=True)
            h2d_done[b].record(up)
            main.wait_event(h2d_done[b])
            if i >= 2:
                main.wait_event(d2h_done[b])  # step i-2's results have left output buffer b
            for ti, t in enumerate(T_LIST):
                gu, dn = copies[ti]
                q.qlin_gemv(gu, dxv[b][2 * ti], dyv[b][2 * ti], q.OUT_BF16, workspace=ws)
                q.qlin_gemv(dn, dxv[b][2 * ti + 1], dyv[b][2 * ti + 1], q.OUT_BF16, workspace=ws)
            comp_done[b].record(main)
            down.wait_event(comp_done[b])
            with torch.cuda.stream(down):
                hy_all.copy_(dy_all[b], non_blocking=True)
            d2h_done[b].record(down)
        main.wait_stream(up)
        main.wait_stream(down)

    e2e_run(args.warmup)
    torch.cuda.synchronize()
    dist.barrier()
    s2, e2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s2.record()
    e2e_run(args.steps)
    e2.record()
    torch.cuda.synchronize()
    e2e_ms = dist.max(s2.elapsed_time(e2))
    e2e_value = dist.sum(step_bytes * args.steps) / (e2e_ms / 1e3) / 1e9

    # dominant kernel of the step: the kernel instantiation with the largest
    # summed device time over the step's 8 calls (call j of a step: matrix
    # j % 2 = gate+up / down, T = T_LIST[j // 2])
    groups = {}
    for j in range(2 * len(T_LIST)):
        t = T_LIST[j // 2]
        fmt = "Q4_G64" if j % 2 == 0 else "Q5_G64"
        kern = (f"gemv_sm_kernel<{fmt}, 1>" if t == 1 else
                f"gemv_tc_kernel<{fmt}, {16 if t <= 16 else 32 if t <= 32 else 48 if t <= 48 else 64}>")
        ms_j = sum(timer.pairs[8 * i + j][0].elapsed_time(timer.pairs[8 * i + j][1])
                   for i in range(args.steps)) / args.steps
        g = groups.setdefault(kern, {"ms": 0.0, "bytes": 0, "calls": []})
        g["ms"] += ms_j
        g["bytes"] += gemv_bytes(copies[0][j % 2], t)
        g["calls"].append(("gate+up 34816x5120" if j % 2 == 0 else "down 5120x17408") + f" T={t}")
    dom_kern, dom = max(groups.items(), key=lambda kv: kv[1]["ms"])
    achieved = dom["bytes"] / (dom["ms"] / 1e3) / 1e9
    traffic = measured_traffic(dom_kern)
    out = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "GB/s",
        "n_gpus": dist.world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_per_step, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "q4/q5 codes x bf16 -> f32 accumulate",
        "data": "synthetic (seeded; weights N(0,0.02) with 1% outlier rows x8, x N(0,1) with 0.5% outlier channels x20)",
        "config": {
            "workload": "decode MLP GEMV: gate+up 34816x5120 Q4G64 then down 5120x17408 Q5G64, T in {1,4,17,33}",
            "calls_per_step": 2 * len(T_LIST),
            "bytes_per_step": step_bytes,
            "l2": (f"{L2_COPIES} weight copies, copy i for the call pair at T_LIST[i]: a matrix is re-read "
                   f"after {reuse_mb:.0f} MB of other weights ({reuse_mb * 1e6 / L2_BYTES:.1f}x the 126 MB L2)"),
            "parallelism": f"replicas x{dist.world}",
            "timed_region": "CUDA graph replay of the step's 8 launches",
        },
        "roofline": {
            "bound": "hbm", "kernel": dom_kern + ": " + ", ".join(dom["calls"]),
            "timing": "CUDA events around each call, calls queued behind a device spin",
            "algorithmic_bytes_per_launch": dom["bytes"] / len(dom["calls"]),
            "share_of_step": round(dom["ms"] / call_ms, 3),
            "achieved": round(achieved, 1), "peak": hbm, "peak_kind": f"{peak_kind} HBM copy GB/s",
            "unit": "GB/s", "frac": round(achieved / hbm, 4), "traffic": traffic,
            "peak_nominal": NOMINAL_HBM_GBS, "frac_nominal": round(achieved / NOMINAL_HBM_GBS, 4),
            "step_achieved_all_8_calls": round(step_bytes / (call_ms / 1e3) / 1e9, 1),
        },
        "e2e": {"value": round(e2e_value, 2), "unit": "GB/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "host_us_per_call": round(host_us_per_call, 1)},
        "gpu_launches": launches,
        "clocks": clk,
    }
    return out, dict(q=q, synth=synth, dev=dev, hbm=hbm, copies=copies, ws=ws, bf16_tf=bf16_tf)


# ---------------------------------------------------------------------------
# per-row measurements (outside the headline timed region)
# ---------------------------------------------------------------------------
def time_fn(fn, iters=10, warm=3, flush=None):
    """Average device time of one call: the calls are queued behind a device
    spin, each after an L2 flush when one is given, events around each call."""
    for _ in range(warm):
        fn()
    torch.cuda.synchronize()
    timer = Timer()
    sleep_ahead(iters)
    for _ in range(iters):
        if flush is not None:
            flush()
        timer.run(fn)
    torch.cuda.synchronize()
    return timer.total_ms() / iters


def measure_rows(ctx):
    q, synth, dev, hbm = ctx["q"], ctx["synth"], ctx["dev"], ctx["hbm"]
    rows = {}
    l2_buf = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)

    def flush():
        l2_buf.zero_()

    ws = ctx["ws"]
    # pack (offline converter step) of gate+up from FP32
    w = synth.weights_f32(*GATE_UP, seed=1, device=dev)
    pw = q.PackedWeights(q.Q4_G64, *GATE_UP, device=dev)
    ms = time_fn(lambda: q.qlin_pack_weights(q.SRC_F32, w, pw), iters=3, warm=1)
    rows["pack_q4_gate_up_from_f32"] = {"ms": round(ms, 3), "GB/s": round((w.numel() * 4 + pw.bytes()) / ms / 1e6, 1)}
    del w, pw
    # MXFP8 decode 5120x17408
    words, sc = synth.mxfp8_source(5120, 17408, seed=2, device=dev)
    out = torch.empty(5120, 17408, dtype=torch.int16, device=dev)
    ms = time_fn(lambda: q.qlin_decode_mxfp8(words, sc, 5120, 17408, out), flush=flush)
    b = words.numel() * 4 + sc.numel() + out.numel() * 2
    rows["decode_mxfp8_5120x17408"] = {"ms": round(ms, 4), "GB/s": round(b / ms / 1e6, 1),
                                       "frac_hbm": round(b / ms / 1e6 / hbm, 3)}
    del words, sc, out
    # Q8 group-32 GEMV 5120x5120, and the 152064x5120 output head as row-scaled
    # FP8 and as Q8 group-32 across T = 1..64 (the pages' FP8-vs-Q8 head crossover)
    head_ts = (1, 17, 33, 48, 64)
    for name, fmt, n, k, ts in (("gemv_q8_5120x5120", q.Q8_G32, 5120, 5120, T_LIST),
                                ("gemv_fp8_head_152064x5120", q.FP8_ROW, 152064, 5120, head_ts),
                                ("gemv_q8_head_152064x5120", q.Q8_G32, 152064, 5120, head_ts)):
        pw = packed(q, synth, fmt, n, k, 3, dev)
        res = {}
        for t in ts:
            x = synth.activations_bf16(t, k, seed=4, device=dev)
            y = torch.empty(t, n, dtype=torch.bfloat16, device=dev)
            ws.ensure(q.qlin_gemv_workspace_bytes(pw, t))
            ms = time_fn(lambda: q.qlin_gemv(pw, x, y, q.OUT_BF16, workspace=ws), flush=flush)
            gbs = gemv_bytes(pw, t) / ms / 1e6
            res[f"T={t}"] = {"us": round(ms * 1e3, 1), "GB/s": round(gbs, 1), "frac_hbm": round(gbs / hbm, 3),
                              "frac_nominal_8tbs": round(gbs / NOMINAL_HBM_GBS, 3)}
        rows[name] = res
        del pw
    # which head format is faster at each T (time per call)
    fp8h, q8h = rows["gemv_fp8_head_152064x5120"], rows["gemv_q8_head_152064x5120"]
    rows["head_faster_format"] = {tk: ("fp8_row" if fp8h[tk]["us"] <= q8h[tk]["us"] else "q8_g32")
                                  for tk in fp8h if tk in q8h}
    # headline matrices per T (kernel view)
    gu, dn = ctx["copies"][0]
    for name, pw in (("gemv_q4_gate_up", gu), ("gemv_q5_down", dn)):
        res = {}
        for t in T_LIST:
            x = synth.activations_bf16(t, pw.k, seed=5, device=dev)
            y = torch.empty(t, pw.n, dtype=torch.bfloat16, device=dev)
            ms = time_fn(lambda: q.qlin_gemv(pw, x, y, q.OUT_BF16, workspace=ws), flush=flush)
            gbs = gemv_bytes(pw, t) / ms / 1e6
            res[f"T={t}"] = {"us": round(ms * 1e3, 1), "GB/s": round(gbs, 1), "frac_hbm": round(gbs / hbm, 3),
                              "frac_nominal_8tbs": round(gbs / NOMINAL_HBM_GBS, 3)}
        rows[name] = res
    # the Q3 / Q6 group-64 widths at the MLP shapes (decode GEMV)
    for name, fmt, (n, k) in (("gemv_q3_gate_up", q.Q3_G64, GATE_UP), ("gemv_q6_down", q.Q6_G64, DOWN)):
        pw = packed(q, synth, fmt, n, k, 16, dev, allow_a8=True)
        res = {}
        for t in T_LIST:
            x = synth.activations_bf16(t, k, seed=5, device=dev)
            y = torch.empty(t, n, dtype=torch.bfloat16, device=dev)
            ws.ensure(q.qlin_gemv_workspace_bytes(pw, t))
            ms = time_fn(lambda: q.qlin_gemv(pw, x, y, q.OUT_BF16, workspace=ws), flush=flush)
            gbs = gemv_bytes(pw, t) / ms / 1e6
            res[f"T={t}"] = {"us": round(ms * 1e3, 1), "GB/s": round(gbs, 1), "frac_hbm": round(gbs / hbm, 3),
                             "frac_nominal_8tbs": round(gbs / NOMINAL_HBM_GBS, 3)}
        rows[name] = res
        del pw
    # activation quantizer, T=2048 x 17408
    x = synth.activations_bf16(2048, 17408, seed=6, device=dev)
    xq = torch.empty(2048, 17408, dtype=torch.int8, device=dev)
    xs = torch.empty(2048, 17408 // 64, dtype=torch.float32, device=dev)
    ms = time_fn(lambda: q.qlin_quantize_act(x, xq, xs), flush=flush)
    b = x.numel() * 2 + xq.numel() + xs.numel() * 4
    rows["quantize_act_2048x17408"] = {"us": round(ms * 1e3, 1), "GB/s": round(b / ms / 1e6, 1),
                                       "frac_hbm": round(b / ms / 1e6 / hbm, 3)}
    del x, xq, xs
    # int8 peak on this machine (cuBLASLt int8 GEMM, the denominator only)
    try:
        a = torch.randint(-127, 127, (8192, 8192), dtype=torch.int8, device=dev)
        bm = torch.randint(-127, 127, (8192, 8192), dtype=torch.int8, device=dev).t()
        ms = time_fn(lambda: torch._int_mm(a, bm), iters=10)
        int8_peak = 2 * 8192 ** 3 / ms / 1e9
        del a, bm
    except Exception as e:  # pragma: no cover
        int8_peak = None
        rows["int8_peak_error"] = str(e)[:200]
    rows["int8_peak_tops_measured_torch_int_mm_8192"] = round(int8_peak, 1) if int8_peak else None
    peak = int8_peak or 4500.0
    # int8 prefill GEMM, 2048 tokens (fused quantizer)
    res = {}
    for name, fmt, (n, k) in (("gate_up_q4", q.Q4_G64, GATE_UP), ("down_q5", q.Q5_G64, DOWN),
                              ("gate_up_q3", q.Q3_G64, GATE_UP), ("down_q6", q.Q6_G64, DOWN)):
        pw = packed(q, synth, fmt, n, k, 7, dev, allow_a8=True)
        x = synth.activations_bf16(2048, k, seed=8, device=dev)
        y = torch.empty(2048, n, dtype=torch.bfloat16, device=dev)
        ws.ensure(q.qlin_gemm_a8_workspace_bytes(2048, n, k))
        ms = time_fn(lambda: q.qlin_gemm_a8(pw, y, x=x, workspace=ws), iters=5, flush=flush)
        tops = 2 * 2048 * n * k / ms / 1e9
        res[name] = {"ms": round(ms, 3), "TOPS": round(tops, 1), "frac_int8_peak": round(tops / peak, 3)}
        del pw, x, y
    rows["gemm_a8_T2048"] = res
    # one-layer prefill sweep
    layer = (("q", 6144, 5120, q.Q4_G64), ("k", 1024, 5120, q.Q4_G64), ("v", 1024, 5120, q.Q4_G64),
             ("o", 5120, 6144, q.Q4_G64), ("gate", 17408, 5120, q.Q4_G64), ("up", 17408, 5120, q.Q4_G64),
             ("down", 5120, 17408, q.Q5_G64))
    pws = {nm: packed(q, synth, fmt, n, k, 9, dev, allow_a8=True) for nm, n, k, fmt in layer}
    gdn = packed(q, synth, q.BF16, 96, 5120, 10, dev)
    sweep = {}
    for t in (512, 1792, 8192):
        xin = {k: synth.activations_bf16(t, k, seed=11, device=dev) for k in (5120, 6144, 17408)}
        ys = {nm: torch.empty(t, n, dtype=torch.bfloat16, device=dev) for nm, n, k, fmt in layer}
        for nm, n, k, fmt in layer:
            ws.ensure(q.qlin_gemm_a8_workspace_bytes(t, n, k))

        def layer_fn():
            for nm, n, k, fmt in layer:
                q.qlin_gemm_a8(pws[nm], ys[nm], x=xin[k], workspace=ws)
        ms = time_fn(layer_fn, iters=3, warm=1, flush=flush)
        ops = sum(2 * t * n * k for nm, n, k, fmt in layer)
        yg = torch.empty(t, 96, dtype=torch.bfloat16, device=dev)
        ws.ensure(q.qlin_gemv_workspace_bytes(gdn, t))
        gms = time_fn(lambda: q.qlin_gemv(gdn, xin[5120], yg, q.OUT_BF16, workspace=ws), iters=3, warm=1,
                      flush=flush)
        sweep[f"T={t}"] = {"ms": round(ms, 3), "TOPS": round(ops / ms / 1e9, 1),
                           "frac_int8_peak": round(ops / ms / 1e9 / peak, 3),
                           "tok_per_s_linear_only": round(t / ms * 1e3, 1),
                           "gdn_ab_bf16_us": round(gms * 1e3, 1),
                           "gdn_ab_GB/s": round((t * 5120 * 2 + 96 * 5120 * 2 + t * 96 * 2) / gms / 1e6, 1),
                           "gdn_ab_frac_hbm": round((t * 5120 * 2 + 96 * 5120 * 2 + t * 96 * 2) / gms / 1e6 / hbm, 3)}
    rows["prefill_layer_sweep"] = sweep
    del pws, gdn
    rows.update(measure_fp8_route(ctx, flush))
    return rows


def measure_fp8_route(ctx, flush):
    """The FP8-activation route (row-FP8 weights x per-token E4M3 activations,
    quantizer fused into the call): the output head at decode sizes (weight
    GB/s) and three prefill projections (TFLOP/s against the FP8 dense peak,
    taken as 2x the measured BF16 GEMM peak: the nominal FP8/BF16 ratio)."""
    q, synth, dev, hbm, ws = ctx["q"], ctx["synth"], ctx["dev"], ctx["hbm"], ctx["ws"]
    fp8_peak = 2.0 * ctx["bf16_tf"]
    rows = {}
    pw = packed(q, synth, q.FP8_ROW, 152064, 5120, 12, dev)
    res = {}
    for t in (1, 33):
        x = synth.activations_bf16(t, 5120, seed=13, device=dev)
        y = torch.empty(t, 152064, dtype=torch.bfloat16, device=dev)
        ws.ensure(q.qlin_gemm_fp8_workspace_bytes(t, 5120))
        ms = time_fn(lambda: q.qlin_gemm_fp8(pw, y, x=x, workspace=ws), flush=flush)
        gbs = gemv_bytes(pw, t) / ms / 1e6
        res[f"T={t}"] = {"us": round(ms * 1e3, 1), "GB/s": round(gbs, 1), "frac_hbm": round(gbs / hbm, 3),
                         "frac_nominal_8tbs": round(gbs / NOMINAL_HBM_GBS, 3)}
    rows["gemm_fp8_head_152064x5120"] = res
    del pw
    res = {}
    for name, n, k, t in (("q_6144x5120_T8192", 6144, 5120, 8192), ("gate_up_34816x5120_T2048", 34816, 5120, 2048),
                          ("down_5120x17408_T2048", 5120, 17408, 2048)):
        pw = packed(q, synth, q.FP8_ROW, n, k, 14, dev)
        x = synth.activations_bf16(t, k, seed=15, device=dev)
        y = torch.empty(t, n, dtype=torch.bfloat16, device=dev)
        ws.ensure(q.qlin_gemm_fp8_workspace_bytes(t, k))
        ms = time_fn(lambda: q.qlin_gemm_fp8(pw, y, x=x, workspace=ws), iters=5, flush=flush)
        tf = 2.0 * t * n * k / ms / 1e9
        res[name] = {"ms": round(ms, 4), "TFLOP/s": round(tf, 1), "frac_fp8_peak": round(tf / fp8_peak, 3)}
        del pw, x, y
    res["fp8_peak_tflops"] = round(fp8_peak, 1)
    rows["gemm_fp8_prefill"] = res
    return rows


# ---------------------------------------------------------------------------
# CPU baseline: the oracle on the host cores, bounded sample
# ---------------------------------------------------------------------------
def cpu_baseline(target_s):
    """The oracle as it stands on the host cores, on a bounded sample of the
    headline step (leading rows of both matrices at every T): once with the
    rows split over every available core, once on a single thread; the
    multi-threaded figure is the line's value."""
    import numpy as np

    import oracle
    import synth
    cores = oracle.cores_available()
    frac_rows = 64
    gu_w = synth.weights_f32(frac_rows, GATE_UP[1], seed=synth.seed_for(1, 10))
    dn_w = synth.weights_f32(frac_rows, DOWN[1], seed=synth.seed_for(1, 20))
    pgu = oracle.pack(oracle.Q4_G64, gu_w.numpy())
    pdn = oracle.pack(oracle.Q5_G64, dn_w.numpy())
    xg = {t: synth.activations_bf16(t, GATE_UP[1], seed=synth.seed_for(1, 30 + t)).view(torch.int16).numpy().view(np.uint16) for t in T_LIST}
    xd = {t: synth.activations_bf16(t, DOWN[1], seed=synth.seed_for(1, 60 + t)).view(torch.int16).numpy().view(np.uint16) for t in T_LIST}

    def pbytes(p):
        return sum(a.nbytes for a in (p["codes"], p["hibits"], p["scales"]) if a is not None)

    def one(nthreads):
        b = 0
        for t in T_LIST:
            oracle.gemv(pgu, xg[t], nthreads=nthreads, with_bound=False)
            oracle.gemv(pdn, xd[t], nthreads=nthreads, with_bound=False)
            b += pbytes(pgu) + 2 * t * GATE_UP[1] + 2 * t * frac_rows
            b += pbytes(pdn) + 2 * t * DOWN[1] + 2 * t * frac_rows
        return b

    def timed(nthreads, seconds):
        t0 = time.perf_counter()
        one(nthreads)
        dt = time.perf_counter() - t0
        reps = max(1, int(seconds / max(dt, 1e-3)))
        t0 = time.perf_counter()
        tot = sum(one(nthreads) for _ in range(reps))
        dt = time.perf_counter() - t0
        return tot / dt / 1e9, reps, dt

    v, reps, dt = timed(cores, 0.6 * target_s)
    v1, reps1, dt1 = timed(1, 0.4 * target_s)
    sample = f"{frac_rows} leading rows of each headline matrix at T in {list(T_LIST)}"
    return {"value": round(v, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
            "sample": f"{sample}, {reps} repetitions ({dt:.1f} s), rows split over {cores} threads",
            "single_thread": {"value": round(v1, 4), "unit": "GB/s", "cores": 1,
                              "sample": f"{sample}, {reps1} repetitions ({dt1:.1f} s), one thread"}}


def run_case(args):
    """One kernel case, W warm-up + K timed calls; prints a short JSON line."""
    import quantized_weight_linear_qlin_b200 as q
    import synth
    from quantized_weight_linear_qlin_b200 import _build
    _build.build()
    dev = torch.device("cuda", 0)
    fmts = {"q4": q.Q4_G64, "q5": q.Q5_G64, "q8": q.Q8_G32, "fp8": q.FP8_ROW, "bf16": q.BF16,
            "q3": q.Q3_G64, "q6": q.Q6_G64}
    parts = args.case.split(":")
    kind = parts[0]
    ws = q.Workspace(dev)
    if kind in ("gemv", "gemm_a8"):
        fmt = fmts[parts[1]]
        n, k = (int(v) for v in parts[2].split("x"))
        t = int(parts[3][1:])
        pw = packed(q, synth, fmt, n, k, 1, dev, allow_a8=kind == "gemm_a8")
        x = synth.activations_bf16(t, k, seed=2, device=dev)
        y = torch.empty(t, n, dtype=torch.bfloat16, device=dev)
        if kind == "gemv":
            ws.ensure(q.qlin_gemv_workspace_bytes(pw, t))
            fn = lambda: q.qlin_gemv(pw, x, y, q.OUT_BF16, workspace=ws)  # noqa: E731
            units, unit = gemv_bytes(pw, t), "GB/s"
        else:
            ws.ensure(q.qlin_gemm_a8_workspace_bytes(t, n, k))
            fn = lambda: q.qlin_gemm_a8(pw, y, x=x, workspace=ws)  # noqa: E731
            units, unit = 2 * t * n * k, "TOPS"
    elif kind == "gemm_fp8":
        n, k = (int(v) for v in parts[1].split("x"))
        t = int(parts[2][1:])
        pw = packed(q, synth, q.FP8_ROW, n, k, 1, dev)
        x = synth.activations_bf16(t, k, seed=2, device=dev)
        y = torch.empty(t, n, dtype=torch.bfloat16, device=dev)
        ws.ensure(q.qlin_gemm_fp8_workspace_bytes(t, k))
        fn = lambda: q.qlin_gemm_fp8(pw, y, x=x, workspace=ws)  # noqa: E731
        units, unit = 2 * t * n * k, "TFLOP/s"
    elif kind == "quantize":
        t, k = (int(v) for v in parts[1].split("x"))
        x = synth.activations_bf16(t, k, seed=2, device=dev)
        xq = torch.empty(t, k, dtype=torch.int8, device=dev)
        xs = torch.empty(t, k // 64, dtype=torch.float32, device=dev)
        fn = lambda: q.qlin_quantize_act(x, xq, xs)  # noqa: E731
        units, unit = t * k * 2 + t * k + t * (k // 64) * 4, "GB/s"
    elif kind == "decode":
        r, c = (int(v) for v in parts[1].split("x"))
        words, sc = synth.mxfp8_source(r, c, seed=2, device=dev)
        out = torch.empty(r, c, dtype=torch.int16, device=dev)
        fn = lambda: q.qlin_decode_mxfp8(words, sc, r, c, out)  # noqa: E731
        units, unit = r * c + r * (c // 32) + 2 * r * c, "GB/s"
    else:
        raise SystemExit(f"unknown case {args.case}")
    l2_buf = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    ms = time_fn(fn, iters=args.steps, warm=args.warmup, flush=l2_buf.zero_)
    per_ms = 1e6 if unit == "GB/s" else 1e9
    print(json.dumps({"case": args.case, "ms": round(ms, 5), unit: round(units / ms / per_ms, 2)}))


def main():
    args = parse()
    if args.case:
        run_case(args)
        return
    dist = Dist(args.gpus)
    if args.impl == "reference":
        if dist.rank != 0:
            dist.close()
            return
        cb = None
        t0 = time.perf_counter()
        vals = []
        for _ in range(args.warmup + args.steps):
            cb = cpu_baseline(max(0.5, 60.0 / max(1, args.warmup + args.steps)))
            vals.append(cb["value"])
        v = statistics.median(vals[args.warmup:] or vals)
        cb["value"] = v
        out = {"impl": "reference", "metric": METRIC, "value": v, "unit": "GB/s", "n_gpus": 1,
               "steps": args.steps, "warmup": args.warmup, "higher_is_better": True, "scaling": "weak",
               "vs_baseline": None, "dtype": "f64 oracle (scalar C++)", "data": "synthetic",
               "config": {"workload": "decode MLP GEMV: gate+up 34816x5120 Q4G64 then down 5120x17408 Q5G64, T in {1,4,17,33} (row sample)"},
               "cpu_baseline": cb, "e2e": {"value": v, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
               "wall_s": round(time.perf_counter() - t0, 1)}
        print(json.dumps(out))
        dist.close()
        return
    out, ctx = run_ours(args, dist)
    if dist.rank == 0:
        if not args.no_rows:
            # the per-row measurements come after the headline; a failure there
            # is reported in the line instead of losing it
            try:
                out["rows"] = measure_rows(ctx)
            except Exception as e:  # pragma: no cover
                out["rows"] = {"error": f"{type(e).__name__}: {e}"[:300]}
        out["cpu_baseline"] = cpu_baseline(args.cpu_seconds)
        print(json.dumps(out))
    dist.barrier()
    dist.close()


if __name__ == "__main__":
    main()
