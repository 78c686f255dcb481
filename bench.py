"""Benchmark of the fused-dequant low-bit GEMM path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload w4a16_sweep|moe|mxfp4|nvfp4|tiny|mxfp4_a16|w3a16|w2a16|w8a16|mxint4_a16]
                    [--sweep-only]

Default workload (one "step"): the dense W4A16 M-sweep, M in {1, 4, 16, 64,
256, 1024, 4096} for (K, N) = (7168, 18432) and (18432, 7168), symmetric
INT4, group 128, fp16 scales, bf16 activations: 14 GEMMs through the C ABI.
`value` is the sweep's aggregate TFLOP/s (total FLOPs / total time).  The
same line then carries the rest of the metric, each timed the same way with
its own roofline: the W4A8-MXFP4 GEMMs (`mxfp4_a8`), the NVFP4 W4A4 GEMMs
(`nvfp4`), the MoE layer (`moe`, tok/s) and the tiny dense case (`tiny`,
microseconds); --sweep-only leaves them out.

Other workloads (--workload) print their own line: each of those, and the
other weight formats on the W4A16 kernels.

Timing: W untimed warm-up steps, then K steps bracketed by a barrier and a
device synchronize, timed with CUDA events on the launching stream; weight
blobs rotate over several copies whose total exceeds 3x the L2 size, so
every GEMM streams its weights from HBM.  Under torchrun every rank runs an
independent replica (the path has no exchange step) and the time is the
maximum over ranks.

--impl reference times the CPU oracle (the method's plain fp64 definition)
on a bounded sample of the same workload on the host cores.
"""

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "W4A16/FP4 GEMM TFLOP/s and HBM GB/s vs roofline (1 B200), M=1..8192; MoE tok/s"
SWEEP_M = (1, 4, 16, 64, 256, 1024, 4096)
SWEEP_KN = ((7168, 18432), (18432, 7168))
GROUP = 128


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# DRAM bytes (read + write) per launch of the sweep GEMMs, from one ncu
# capture of the bench's first warm-up step (cold caches), recorded in
# profiles/traffic_w4a16_sweep.md with the commit it ran on.  The capture
# holds for the kernel sources it ran (TRAFFIC_SOURCES, a fingerprint of
# csrc/ and include/): once they change, `traffic` reads null until the
# capture is taken again.
TRAFFIC_COMMIT = "da1bb90"
# sources since the capture differ only in comments (the register path's
# documentation in include/hq.h and csrc/w4a16_reg.cu)
TRAFFIC_SOURCES = "801df59bbb0197d2"
TRAFFIC_BYTES = {
    (1, 7168, 18432): 68638976,
    (4, 7168, 18432): 68249856,
    (16, 7168, 18432): 68398592,
    (64, 7168, 18432): 71147008,
    (256, 7168, 18432): 75643648,
    (1024, 7168, 18432): 158340864,
    (4096, 7168, 18432): 422855936,
    (1, 18432, 7168): 68249344,
    (4, 18432, 7168): 68308480,
    (16, 18432, 7168): 68766208,
    (64, 18432, 7168): 74269440,
    (256, 18432, 7168): 85654528,
    (1024, 18432, 7168): 199288832,
    (4096, 18432, 7168): 710096640,
}


def kernel_sources_fingerprint():
    """sha256 (first 16 hex digits) of the library's sources, in name order."""
    import glob
    import hashlib
    files = sorted(glob.glob(os.path.join(ROOT, "quantized_gemm_bit_b200", "csrc", "*")))
    files.append(os.path.join(ROOT, "include", "hq.h"))
    h = hashlib.sha256()
    for f in files:
        h.update(os.path.basename(f).encode())
        with open(f, "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def w4a16_bytes(m, k, n):
    """Algorithmic bytes of one W4A16 GEMM: packed codes (K*N/2) + fp16
    scales (2*N*K/128) + bf16 A (2*M*K) + bf16 C (2*M*N), each once."""
    return k * n // 2 + 2 * n * (k // GROUP) + 2 * m * k + 2 * m * n


def w4a16_flops(m, k, n):
    return 2.0 * m * k * n


class Clocks:
    """Samples nvidia-smi every 50 ms while the timed region runs (the
    sampler starts half a second early; idle samples below half the peak
    clock are left out of the median)."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.dev = device_index
        self.proc = None
        # the raw samples go to $HQ_CLOCKS_DIR (default: the system temp
        # directory); the line printed carries their summary
        import tempfile
        out_dir = os.environ.get("HQ_CLOCKS_DIR", tempfile.gettempdir())
        self.path = os.path.join(out_dir, f"hq_clocks_rank{device_index}.csv")

    def __enter__(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.dev), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=self.f, stderr=subprocess.DEVNULL)
            time.sleep(0.5)   # let the sampler start before the timed region
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.f.close()

    def summary(self):
        if self.proc is None or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        sm, smax, reasons = [], None, set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    smax = float(parts[2])
                except ValueError:
                    continue
                for nm, v in zip(names, parts[5:9]):
                    if v.lower() == "active":
                        reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": smax, "reasons": sorted(reasons)}
        loaded = [x for x in sm if x > 0.5 * max(sm)] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------- distributed

def dist_init():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x, world):
    """The largest of the ranks' values (times are reported as the slowest
    rank's).  NCCL reduces on the device; a gloo group (CPU tests) on the host."""
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ---------------------------------------------------------------- W4A16 sweep

def setup_w4a16_sweep(l2_bytes):
    from quantized_gemm_bit_b200 import hq, synth
    dev = "cuda"
    shapes = []
    for si, (k, n) in enumerate(SWEEP_KN):
        q, s, _ = synth.w4a16_weights(n, k, GROUP, False, seed=1000 + si)
        d = hq.hq_quant_desc_init(hq.HQ_FMT_INT4, n, k, GROUP, 0, 1)
        blob = torch.from_numpy(hq.hq_pack_weights(d, q, s, None)).to(dev)
        copies = max(2, int(np.ceil(3 * l2_bytes / blob.numel())) + 1)
        blobs = [blob] + [blob.clone() for _ in range(copies - 1)]
        acts, outs, wss, host_a, host_c = [], [], [], [], []
        for m in SWEEP_M:
            a = synth.bf16_normal(m, k, seed=1000 + m).to(dev)
            acts.append(a)
            outs.append(torch.empty(m, n, dtype=torch.bfloat16, device=dev))
            wss.append(torch.zeros(max(256, hq.hq_workspace_size(d, m)), dtype=torch.uint8, device=dev))
            host_a.append(a.cpu().pin_memory())
            host_c.append(torch.empty(m, n, dtype=torch.bfloat16).pin_memory())
        shapes.append(dict(k=k, n=n, d=d, blobs=blobs, acts=acts, outs=outs, wss=wss, host_a=host_a,
                           host_c=host_c))
    return shapes


def run_w4a16_sweep(args, rank, world, peaks):
    from quantized_gemm_bit_b200 import hq
    props = torch.cuda.get_device_properties(torch.cuda.current_device())
    l2 = getattr(props, "L2_cache_size", 126 * 2 ** 20)
    shapes = setup_w4a16_sweep(l2)
    stream = torch.cuda.current_stream()
    gemms = [(si, mi) for si in range(len(shapes)) for mi in range(len(SWEEP_M))]
    counter = [0]

    def one_step(e2e=False):
        # the user's call path: one C-ABI call per GEMM from Python
        for (si, mi) in gemms:
            sh = shapes[si]
            blob = sh["blobs"][counter[0] % len(sh["blobs"])]
            counter[0] += 1
            m = SWEEP_M[mi]
            if e2e:
                sh["acts"][mi].copy_(sh["host_a"][mi], non_blocking=True)
            hq.hq_gemm_w4a16(sh["d"], blob, sh["acts"][mi], m, sh["outs"][mi], sh["wss"][mi], stream=stream)
            if e2e:
                sh["host_c"][mi].copy_(sh["outs"][mi], non_blocking=True)

    # correctness guard: the device status must be clean after warm-up
    for _ in range(args.warmup):
        one_step()
    torch.cuda.synchronize()
    for sh in shapes:
        for ws in sh["wss"]:
            st = hq.hq_check_device_status(ws)
            if st != hq.HQ_OK:
                raise RuntimeError(f"device status after warm-up: {hq.status_string(st)}")

    # ---- device-resident timed region (CUDA graphs, see _time_launches): in
    # graph c, GEMM mi of a shape reads weight copy (c + mi) mod ncopy, so the
    # GEMMs of a step never share a copy and a GEMM's back-to-back launches
    # (c = 0, 1, ...) never repeat one
    ncopy = len(shapes[0]["blobs"])
    launches = []
    for (si, mi) in gemms:
        def f(c, si=si, mi=mi):
            sh = shapes[si]
            blob = sh["blobs"][(c + mi) % len(sh["blobs"])]
            hq.hq_gemm_w4a16(sh["d"], blob, sh["acts"][mi], SWEEP_M[mi], sh["outs"][mi], sh["wss"][mi])
        launches.append(f)
    with Clocks(torch.cuda.current_device()) as clk:
        ms, per = _time_launches(launches, args.steps, args.warmup, world, ncopy=ncopy)
    per_launch_us = dict(zip(gemms, per))
    for sh in shapes:
        for ws in sh["wss"]:
            st = hq.hq_check_device_status(ws)
            if st != hq.HQ_OK:
                raise RuntimeError(f"device status after the timed region: {hq.status_string(st)}")

    # ---- end-to-end through the C ABI with host buffers (pinned), copies inside
    for _ in range(max(1, args.warmup // 2)):
        one_step(e2e=True)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(args.steps):
        one_step(e2e=True)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world)

    flops_step = sum(w4a16_flops(m, sh["k"], sh["n"]) for sh in shapes for m in SWEEP_M)
    bytes_step = sum(w4a16_bytes(m, sh["k"], sh["n"]) for sh in shapes for m in SWEEP_M)
    value = flops_step * args.steps * world / (ms * 1e-3) / 1e12
    e2e_value = flops_step * args.steps * world / (e2e_ms * 1e-3) / 1e12
    h2d = sum(m * sh["k"] * 2 for sh in shapes for m in SWEEP_M)
    d2h = sum(m * sh["n"] * 2 for sh in shapes for m in SWEEP_M)

    sweep = []
    for (si, mi) in gemms:
        sh = shapes[si]
        m = SWEEP_M[mi]
        us = per_launch_us[(si, mi)]
        fl = w4a16_flops(m, sh["k"], sh["n"])
        by = w4a16_bytes(m, sh["k"], sh["n"])
        tf = fl / (us * 1e-6) / 1e12
        gb = by / (us * 1e-6) / 1e9
        ridge = peaks["bf16_tflops"] * 1e3 / peaks["hbm_gbs"]        # flop per byte
        bound = "hbm" if fl / by < ridge else "tensor"
        frac = gb / peaks["hbm_gbs"] if bound == "hbm" else tf / peaks["bf16_tflops"]
        sweep.append(dict(m=m, k=sh["k"], n=sh["n"], us=round(us, 2), tflops=round(tf, 1), gbs=round(gb, 1),
                          bound=bound, frac=round(frac, 3)))

    def roof(entries, bound):
        # the dominant launch class: time-weighted over the given launches
        t = sum(e["us"] for e in entries)
        keys = [(e["m"], e["k"], e["n"]) for e in entries]
        fresh = TRAFFIC_SOURCES is not None and TRAFFIC_SOURCES == kernel_sources_fingerprint()
        traffic = (round(sum(TRAFFIC_BYTES[x] for x in keys) / len(keys))
                   if fresh and all(x in TRAFFIC_BYTES for x in keys) else None)
        tinfo = dict(traffic_commit=TRAFFIC_COMMIT, traffic_sources=TRAFFIC_SOURCES,
                     sources=kernel_sources_fingerprint())
        algo = round(sum(w4a16_bytes(*x) for x in keys) / len(keys))
        if bound == "hbm":
            ach = sum(w4a16_bytes(e["m"], e["k"], e["n"]) for e in entries) / (t * 1e-6) / 1e9
            return dict(bound="hbm", achieved=round(ach, 1), peak=peaks["hbm_gbs"], unit="GB/s",
                        frac=round(ach / peaks["hbm_gbs"], 3), traffic=traffic, algorithmic_bytes=algo,
                        launches=[f"M={e['m']},K={e['k']},N={e['n']}" for e in entries],
                        peak_source=_peak_src(peaks, "hbm"), **tinfo)
        ach = sum(w4a16_flops(e["m"], e["k"], e["n"]) for e in entries) / (t * 1e-6) / 1e12
        return dict(bound="tensor", achieved=round(ach, 1), peak=peaks["bf16_tflops"], unit="TFLOP/s",
                    frac=round(ach / peaks["bf16_tflops"], 3), traffic=traffic, algorithmic_bytes=algo,
                    launches=[f"M={e['m']},K={e['k']},N={e['n']}" for e in entries],
                    peak_source=_peak_src(peaks, "bf16"), **tinfo)

    big = [e for e in sweep if e["m"] == 4096]
    small = [e for e in sweep if e["m"] <= 16]
    clocks = clk.summary()
    line = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms / args.steps, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16 x int4 (fp32 accumulate)",
        "data": "synthetic (seeded; uniform int4 codes, fp16 scales 0.002+0.01|N(0,1)|, bf16 N(0,1) activations)",
        "config": {
            "workload": "dense W4A16 M-sweep: M in {1,4,16,64,256,1024,4096} x (K,N) in {(7168,18432),"
                        "(18432,7168)}, symmetric INT4, group 128",
            "gemms_per_step": len(gemms),
            "l2": f"weights rotate over {len(shapes[0]['blobs'])} copies per shape (>3x L2), no flush",
            "launch": "CUDA graphs: one per step (the 14 C-ABI calls, captured once per weight-copy rotation); "
                      "per-launch times from graphs of back-to-back launches of each GEMM",
            "parallelism": f"replicas x{world}",
        },
        "roofline": roof(big, "tensor"),
        "roofline_small_m": roof(small, "hbm"),
        "sweep": sweep,
        "e2e": {"value": round(e2e_value, 2), "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        "gpu_launches": len(gemms) * args.steps,
        "clocks": clocks,
        "algorithmic_bytes_per_step": bytes_step,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline_w4a16(budget_s=args.cpu_budget)
    return line


# ---------------------------------------------------------------- other workloads

FP8_RATIO, FP4_RATIO = 2.0, 4.0   # nominal dense peaks relative to bf16 (4.5 / 9 vs 2.25 PF)


def _peak_src(peaks, kind):
    """Where a roofline denominator comes from."""
    src = peaks["source"]
    return {"hbm": f"{src} copy bandwidth (burst)",
            "bf16": f"{src} cuBLAS bf16 8192^3 (burst)",
            "fp8": f"{src} cuBLAS bf16 (burst) x nominal fp8/bf16 ratio 2 (4.5 / 2.25 PFLOP/s)",
            "fp4": f"{src} cuBLAS bf16 (burst) x nominal fp4/bf16 ratio 4 (9 / 2.25 PFLOP/s)"}[kind]


def _bound(flops, nbytes, tensor_peak_tflops, peaks):
    """Which roofline a launch sits under (its arithmetic intensity against
    the ridge point) and its fraction of that roofline."""
    ridge = tensor_peak_tflops * 1e3 / peaks["hbm_gbs"]     # flop per byte
    return {"bound": "hbm" if flops / nbytes < ridge else "tensor"}


def _capture(fns, side):
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=side):
        for f in fns:
            f()
    return g


def _time_launches(launches, steps, warmup, world, ncopy=1):
    """Time `launches` (callables f(c) issuing C-ABI calls on the current
    stream; c = weight-copy index) through CUDA graphs, so host launch cost
    never starves the GPU.
      * steps: graph c holds every launch with copy c; step i replays graph
        i % ncopy; the K timed steps sit between two events (barrier and
        synchronize on both sides);
      * per launch: one graph of R = max(ncopy, 4) back-to-back launches of
        it (copies rotating), replayed three times between two events while
        a fourth replay queued before them keeps the GPU busy; the mean
        duration includes the launch gaps inside the graph.  Each launch is
        timed alone: the GPU idles for 0.2 s first, so a small GEMM is not
        measured at the clocks the power cap left after a large one.
    Returns (total ms over `steps`, per-launch mean microseconds)."""
    stream = torch.cuda.current_stream()
    for i in range(max(1, warmup)):        # host-side first-call setup happens here, outside capture
        for f in launches:
            f(i % ncopy)
    torch.cuda.synchronize()
    side = torch.cuda.Stream()
    side.wait_stream(stream)
    graphs = [_capture([(lambda f=f, c=c: f(c)) for f in launches], side) for c in range(ncopy)]
    stream.wait_stream(side)
    for i in range(warmup):
        graphs[i % ncopy].replay()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    t0.record(stream)
    for i in range(steps):
        graphs[i % ncopy].replay()
    t1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    ms = max_over_ranks(t0.elapsed_time(t1), world)
    del graphs
    per = []
    reps = max(ncopy, 4)
    for f in launches:
        side.wait_stream(stream)
        g = _capture([(lambda f=f, c=c: f(c % ncopy)) for c in range(reps)], side)
        stream.wait_stream(side)
        g.replay()
        torch.cuda.synchronize()
        time.sleep(0.2)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        g.replay()                      # keeps the GPU busy while the timed replays are queued
        a.record(stream)
        for _ in range(3):
            g.replay()
        b.record(stream)
        torch.cuda.synchronize()
        per.append(a.elapsed_time(b) * 1e3 / (3 * reps))
        del g
    return ms, per


def run_mxfp4(args, rank, world, peaks):
    """W4A8-MXFP4: M in {16, 256, 4096}, K = N = 7168."""
    from quantized_gemm_bit_b200 import hq, synth
    k = n = 7168
    codes, e8 = synth.mxfp4_weights(n, k, seed=2000)
    d = hq.hq_quant_desc_init(hq.HQ_FMT_MXFP4, n, k, 32, 0, 1)
    blob = torch.from_numpy(hq.hq_pack_weights(d, codes, e8)).cuda()
    props = torch.cuda.get_device_properties(torch.cuda.current_device())
    l2 = getattr(props, "L2_cache_size", 126 * 2 ** 20)
    ncopy_w = max(2, int(np.ceil(3 * l2 / blob.numel())) + 1)
    blobs = [blob] + [blob.clone() for _ in range(ncopy_w - 1)]
    launches, rows = [], []
    for m in (16, 256, 4096):
        x = synth.bf16_normal(m, k, seed=2000 + m).cuda()
        q = torch.empty(m, k, dtype=torch.uint8, device="cuda")
        sc = torch.empty(m, dtype=torch.float32, device="cuda")
        hq.hq_quantize_fp8_rows(x, m, k, q, sc)
        c = torch.empty(m, n, dtype=torch.bfloat16, device="cuda")
        ws = torch.zeros(max(256, hq.hq_workspace_size(d, m)), dtype=torch.uint8, device="cuda")

        def f(cp, j=len(launches), m=m, q=q, sc=sc, c=c, ws=ws):
            hq.hq_gemm_mxfp4_a8(d, blobs[(cp * 3 + j) % len(blobs)], q, sc, m, c, ws)
        launches.append(f)
        rows.append(m)
    ncopy = len(blobs) // np.gcd(len(blobs), 3)      # graphs until every copy has served every launch
    ms, per = _time_launches(launches, args.steps, args.warmup, world, ncopy=int(ncopy))
    peak = peaks["bf16_tflops"] * FP8_RATIO
    out = []
    for m, us in zip(rows, per):
        fl = 2.0 * m * n * k
        by = n * k // 2 + n * k // 32 + m * k + 4 * m + 2 * m * n
        out.append(dict(m=m, k=k, n=n, us=round(us, 2), tflops=round(fl / us / 1e6, 1), gbs=round(by / us / 1e3, 1),
                        frac_fp8_peak=round(fl / us / 1e6 / peak, 3), frac_hbm=round(by / us / 1e3 / peaks["hbm_gbs"], 3),
                        **_bound(fl, by, peak, peaks)))
    flops = sum(2.0 * m * n * k for m in rows)
    big = out[-1]
    return {"workload": "W4A8-MXFP4 GEMM, M in {16,256,4096}, K=N=7168", "value": round(flops * args.steps * world
            / (ms * 1e-3) / 1e12, 2), "unit": "TFLOP/s", "ms_per_step": round(ms / args.steps, 4),
            "peak_fp8_tflops": round(peak, 1), "peak_source": _peak_src(peaks, "fp8"),
            "roofline": dict(bound="tensor", launch="M=4096", achieved=big["tflops"], peak=round(peak, 1),
                             unit="TFLOP/s", frac=big["frac_fp8_peak"], peak_source=_peak_src(peaks, "fp8")),
            "roofline_small_m": dict(bound="hbm", launch="M=16", achieved=out[0]["gbs"], peak=peaks["hbm_gbs"],
                                     unit="GB/s", frac=out[0]["frac_hbm"], peak_source=_peak_src(peaks, "hbm")),
            "gpu_launches": len(rows) * args.steps, "detail": out}


def _run_w16_format(args, world, peaks, fmt):
    """Another weight format on the W4A16 kernels (bf16 activations):
    M in {16, 64, 256, 4096}, K=7168, N=18432.  fmt "mxfp4_a16": e2m1 codes
    with an E8M0 scale per 32 K; "w3a16" / "w2a16": INT3 / INT2 codes with
    an fp16 scale per 128 K (symmetric)."""
    from quantized_gemm_bit_b200 import hq, synth
    k, n = 7168, 18432
    if fmt == "mxfp4_a16":
        codes, e8 = synth.mxfp4_weights(n, k, seed=6000)
        d = hq.hq_quant_desc_init(hq.HQ_FMT_MXFP4_A16, n, k, 32, 0, 1)
        blob = torch.from_numpy(hq.hq_pack_weights(d, codes, e8)).cuda()
        wbytes = n * k // 2 + n * k // 32
        name, dt = "MXFP4 weights x bf16 activations", "bf16 x e2m1 (fp32 accumulate)"
    elif fmt == "w3a16":
        q, sc, _ = synth.w3a16_weights(n, k, 128, False, seed=7000)
        d = hq.hq_quant_desc_init(hq.HQ_FMT_INT3, n, k, 128, 0, 1)
        blob = torch.from_numpy(hq.hq_pack_weights(d, q, sc)).cuda()
        wbytes = 3 * n * k // 8 + 2 * n * (k // GROUP)
        name, dt = "INT3 weights (group 128) x bf16 activations", "bf16 x int3 (fp32 accumulate)"
    elif fmt == "w8a16":
        q, sc, _ = synth.w8a16_weights(n, k, 128, False, seed=7800)
        d = hq.hq_quant_desc_init(hq.HQ_FMT_INT8, n, k, 128, 0, 1)
        blob = torch.from_numpy(hq.hq_pack_weights(d, q, sc)).cuda()
        wbytes = n * k + 2 * n * (k // GROUP)
        name, dt = "INT8 weights (group 128) x bf16 activations", "bf16 x int8 (fp32 accumulate)"
    elif fmt == "mxint4_a16":
        codes, e8 = synth.mxint4_weights(n, k, seed=7900)
        d = hq.hq_quant_desc_init(hq.HQ_FMT_MXINT4, n, k, 32, 0, 1)
        blob = torch.from_numpy(hq.hq_pack_weights(d, codes, e8)).cuda()
        wbytes = n * k // 2 + n * k // 32
        name, dt = "MXINT4 weights x bf16 activations", "bf16 x int4 e8m0-scaled (fp32 accumulate)"
    else:
        q, sc, _ = synth.w2a16_weights(n, k, 128, False, seed=7500)
        d = hq.hq_quant_desc_init(hq.HQ_FMT_INT2, n, k, 128, 0, 1)
        blob = torch.from_numpy(hq.hq_pack_weights(d, q, sc)).cuda()
        wbytes = n * k // 4 + 2 * n * (k // GROUP)
        name, dt = "INT2 weights (group 128) x bf16 activations", "bf16 x int2 (fp32 accumulate)"
    props = torch.cuda.get_device_properties(torch.cuda.current_device())
    l2 = getattr(props, "L2_cache_size", 126 * 2 ** 20)
    ms_list = (16, 64, 256, 4096)
    ncopy_w = max(2, int(np.ceil(3 * l2 / blob.numel())) + 1)
    blobs = [blob] + [blob.clone() for _ in range(ncopy_w - 1)]
    launches = []
    for j, m in enumerate(ms_list):
        a = synth.bf16_normal(m, k, seed=6001 + m).cuda()
        c = torch.empty(m, n, dtype=torch.bfloat16, device="cuda")
        ws = torch.zeros(max(256, hq.hq_workspace_size(d, m)), dtype=torch.uint8, device="cuda")

        def f(cp, j=j, m=m, a=a, c=c, ws=ws):
            hq.hq_gemm_w4a16(d, blobs[(cp * len(ms_list) + j) % len(blobs)], a, m, c, ws)
        launches.append(f)
    ncopy = len(blobs) // np.gcd(len(blobs), len(ms_list))
    ms, per = _time_launches(launches, args.steps, args.warmup, world, ncopy=int(ncopy))
    out = []
    for m, us in zip(ms_list, per):
        fl = 2.0 * m * n * k
        by = wbytes + 2 * m * k + 2 * m * n
        out.append(dict(m=m, k=k, n=n, us=round(us, 2), tflops=round(fl / us / 1e6, 1), gbs=round(by / us / 1e3, 1),
                        frac_hbm=round(by / us / 1e3 / peaks["hbm_gbs"], 3),
                        frac_bf16_peak=round(fl / us / 1e6 / peaks["bf16_tflops"], 3)))
    flops = sum(2.0 * m * n * k for m in ms_list)
    return {"workload": f"{name} (W4A16 kernels), M in {{16,64,256,4096}}, K=7168, N=18432",
            "value": round(flops * args.steps * world / (ms * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
            "ms_per_step": round(ms / args.steps, 4), "dtype": dt, "detail": out}


def run_mxfp4_a16(args, rank, world, peaks):
    return _run_w16_format(args, world, peaks, "mxfp4_a16")


def run_w3a16(args, rank, world, peaks):
    return _run_w16_format(args, world, peaks, "w3a16")


def run_w2a16(args, rank, world, peaks):
    return _run_w16_format(args, world, peaks, "w2a16")


def run_w8a16(args, rank, world, peaks):
    return _run_w16_format(args, world, peaks, "w8a16")


def run_mxint4_a16(args, rank, world, peaks):
    return _run_w16_format(args, world, peaks, "mxint4_a16")


def run_nvfp4(args, rank, world, peaks):
    """NVFP4 W4A4: 8192^3 and M=16384, K=7168, N=18432 (inputs quantized from
    bf16 N(0,1) draws on the GPU by the library's own quantizer)."""
    from quantized_gemm_bit_b200 import hq, synth
    launches, shapes = [], []
    for si, (m, n, k) in enumerate(((8192, 8192, 8192), (16384, 18432, 7168))):
        def quant(rows, seed):
            x = synth.bf16_normal(rows, k, seed).cuda()
            codes = torch.empty(rows, k // 2, dtype=torch.uint8, device="cuda")
            sf = torch.empty(rows, k // 16, dtype=torch.uint8, device="cuda")
            g = torch.empty(1, dtype=torch.float32, device="cuda")
            wsq = torch.zeros(hq.hq_quantize_nvfp4_workspace_size(rows, k), dtype=torch.uint8, device="cuda")
            hq.hq_quantize_nvfp4(x, rows, k, codes, sf, g, wsq)
            return codes, sf, g
        wc, wsf, wg = quant(n, 4000 + si)
        ac, asf, ag = quant(m, 4100 + si)
        d = hq.hq_quant_desc_init(hq.HQ_FMT_NVFP4, n, k, 16, 0, 1)
        blob = torch.from_numpy(hq.hq_pack_weights(d, wc.cpu(), wsf.cpu(), None, float(wg.item()))).cuda()
        c = torch.empty(m, n, dtype=torch.bfloat16, device="cuda")
        ws = torch.zeros(max(256, hq.hq_workspace_size(d, m)), dtype=torch.uint8, device="cuda")
        a_g = float(ag.item())

        def f(cp, m=m, d=d, blob=blob, ac=ac, asf=asf, a_g=a_g, c=c, ws=ws):
            hq.hq_gemm_nvfp4(d, blob, ac, asf, a_g, m, c, ws)
        launches.append(f)
        shapes.append((m, n, k))
    ms, per = _time_launches(launches, args.steps, args.warmup, world)
    peak = peaks["bf16_tflops"] * FP4_RATIO
    out = []
    for (m, n, k), us in zip(shapes, per):
        fl = 2.0 * m * n * k
        # codes + E4M3 block scales of both operands, the weights' tensor scale, bf16 C
        by = (m + n) * k // 2 + (m + n) * k // 16 + 16 + 2 * m * n
        out.append(dict(m=m, k=k, n=n, us=round(us, 2), tflops=round(fl / us / 1e6, 1), gbs=round(by / us / 1e3, 1),
                        frac_fp4_peak=round(fl / us / 1e6 / peak, 3), **_bound(fl, by, peak, peaks)))
    flops = sum(2.0 * m * n * k for m, n, k in shapes)
    t_all = sum(e["us"] for e in out)
    ach = flops / (t_all * 1e-6) / 1e12
    return {"workload": "NVFP4 W4A4 GEMM, 8192^3 and M=16384 K=7168 N=18432", "value": round(
            flops * args.steps * world / (ms * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
            "ms_per_step": round(ms / args.steps, 4), "peak_fp4_tflops": round(peak, 1),
            "peak_source": _peak_src(peaks, "fp4"),
            "roofline": dict(bound="tensor", launch="both shapes (time-weighted)", achieved=round(ach, 1),
                             peak=round(peak, 1), unit="TFLOP/s", frac=round(ach / peak, 3),
                             peak_source=_peak_src(peaks, "fp4")),
            "gpu_launches": 2 * len(shapes) * args.steps, "detail": out}


def run_moe(args, rank, world, peaks):
    """MoE layer over the grouped W4A16 GEMMs: 256 experts, top-8, hidden
    7168, intermediate 2048 (gate+up N=4096, down K=2048), T in
    {64, 1024, 8192}: route (top-k + softmax weights) + permute/gather +
    gate_up with SwiGLU in its epilogue + down + weighted combine."""
    from quantized_gemm_bit_b200 import hq, synth
    E, TOPK, H, I = 256, 8, 7168, 2048
    mats = {}
    for name, (n, k, seed) in {"gate_up": (2 * I, H, 3000), "down": (H, I, 3010)}.items():
        q, s, _ = synth.w4a16_weights(n, k, 128, False, seed=seed, experts=E)
        d = hq.hq_quant_desc_init(hq.HQ_FMT_INT4, n, k, 128, 0, E)
        # gate+up in the gated row order: SwiGLU runs in that GEMM's epilogue
        pack = hq.hq_pack_weights_gated if name == "gate_up" else hq.hq_pack_weights
        mats[name] = (d, torch.from_numpy(pack(d, q, s, None)).cuda(), n, k)
        del q, s
    detail, launches, meta = [], [], []
    for t in (64, 1024, 8192):
        logits = synth.router_logits(t, E, seed=3001).cuda()
        x = synth.bf16_normal(t, H, seed=3002).cuda()
        ids = torch.empty(t, TOPK, dtype=torch.int32, device="cuda")
        wts = torch.empty(t, TOPK, dtype=torch.float32, device="cuda")
        src = torch.empty(t * TOPK, dtype=torch.int32, device="cuda")
        off = torch.empty(E + 1, dtype=torch.int32, device="cuda")
        xs = torch.empty(t * TOPK, H, dtype=torch.bfloat16, device="cuda")
        pws = torch.zeros(hq.hq_moe_permute_workspace_size(t, TOPK, E), dtype=torch.uint8, device="cuda")
        h = torch.empty(t * TOPK, I, dtype=torch.bfloat16, device="cuda")
        c2 = torch.empty(t * TOPK, H, dtype=torch.bfloat16, device="cuda")
        out = torch.empty(t, H, dtype=torch.bfloat16, device="cuda")
        d1, w1, _, _ = mats["gate_up"]
        d2, w2, _, _ = mats["down"]
        ws1 = torch.zeros(max(256, hq.hq_workspace_size(d1, t * TOPK)), dtype=torch.uint8, device="cuda")
        ws2 = torch.zeros(max(256, hq.hq_workspace_size(d2, t * TOPK)), dtype=torch.uint8, device="cuda")
        wsc = torch.zeros(hq.hq_moe_combine_workspace_size(t, TOPK), dtype=torch.uint8, device="cuda")

        def route(cp, t=t, logits=logits, ids=ids, wts=wts, src=src, off=off, x=x, xs=xs, pws=pws):
            hq.hq_moe_topk_softmax(logits, t, E, TOPK, ids, wts)
            hq.hq_moe_permute(ids, t, TOPK, E, src, off, pws, a=x, hidden=H, a_sorted=xs)

        def g1(cp, t=t, xs=xs, off=off, h=h, ws1=ws1):
            hq.hq_grouped_gemm_moe_swiglu(d1, w1, xs, off, t * TOPK, h, ws1)

        def g2(cp, t=t, h=h, off=off, c2=c2, ws2=ws2):
            hq.hq_grouped_gemm_moe(d2, w2, h, off, t * TOPK, c2, ws2)

        def comb(cp, t=t, c2=c2, src=src, wts=wts, out=out, wsc=wsc):
            hq.hq_moe_combine(c2, src, wts, t, TOPK, H, out, wsc)
        launches += [route, g1, g2, comb]
        meta.append((t, off, (ws1, ws2, wsc, pws)))
    ms, per = _time_launches(launches, args.steps, args.warmup, world)
    for (_, _, wss) in meta:
        for ws in wss:
            st = hq.hq_check_device_status(ws)
            if st != hq.HQ_OK:
                raise RuntimeError(f"device status after the MoE timing: {hq.status_string(st)}")
    tok_total = 0
    for i, (t, off, _) in enumerate(meta):
        r_us, g1_us, g2_us, c_us = per[4 * i: 4 * i + 4]
        offs = off.cpu().numpy()
        active = int((offs[1:] > offs[:-1]).sum())
        wbytes = active * (2 * I * H // 2 + 2 * I * (H // 128) * 2 + H * I // 2 + H * (I // 128) * 2)
        fl = 2.0 * t * TOPK * H * 3 * I
        gemm_us = g1_us + g2_us
        layer_us = r_us + g1_us + g2_us + c_us
        detail.append(dict(tokens=t, active_experts=active, route_permute_us=round(r_us, 2),
                           gate_up_swiglu_us=round(g1_us, 2), down_us=round(g2_us, 2),
                           combine_us=round(c_us, 2), tok_per_s=round(t / (layer_us * 1e-6), 1),
                           tok_per_s_gemms=round(t / (gemm_us * 1e-6), 1), tflops=round(fl / gemm_us / 1e6, 1),
                           weight_gbs=round(wbytes / gemm_us / 1e3, 1),
                           frac_hbm=round(wbytes / gemm_us / 1e3 / peaks["hbm_gbs"], 3)))
        tok_total += t
    # value: tokens of all three batches per step over the whole step (every
    # launch of the layer); the detail gives each batch alone
    small = [x for x in detail if x["tokens"] <= 1024]
    gb_small = sum(x["weight_gbs"] * (x["gate_up_swiglu_us"] + x["down_us"]) for x in small) / sum(
        x["gate_up_swiglu_us"] + x["down_us"] for x in small)
    big = [x for x in detail if x["tokens"] == 8192][0]
    return {"workload": "MoE layer over grouped W4A16 GEMMs: 256 experts, top-8, hidden 7168, intermediate 2048 "
                        "(gate+up N=4096, down K=2048), T in {64,1024,8192}; one step = route (top-k + softmax "
                        "weights) + permute/gather + gate_up with fused SwiGLU + down + weighted combine for each T",
            "value": round(tok_total * args.steps * world / (ms * 1e-3), 1), "unit": "tok/s",
            "ms_per_step": round(ms / args.steps, 4),
            "roofline": dict(bound="tensor", launch="T=8192 gate_up + down", achieved=big["tflops"],
                             peak=peaks["bf16_tflops"], unit="TFLOP/s",
                             frac=round(big["tflops"] / peaks["bf16_tflops"], 3), peak_source=_peak_src(peaks, "bf16")),
            "roofline_small_t": dict(bound="hbm", launch="T=64 and T=1024 gate_up + down (active-expert weights)",
                                     achieved=round(gb_small, 1), peak=peaks["hbm_gbs"], unit="GB/s",
                                     frac=round(gb_small / peaks["hbm_gbs"], 3), peak_source=_peak_src(peaks, "hbm")),
            "gpu_launches": 9 * len(detail) * args.steps, "detail": detail}


def run_tiny(args, rank, world, peaks):
    """Dense W4A16 tiny: M=16, K=N=1024, asymmetric INT4 (zero points),
    group 128: a latency-bound launch, reported in microseconds."""
    from quantized_gemm_bit_b200 import hq, synth
    m, n, k = 16, 1024, 1024
    q, s, z = synth.w4a16_weights(n, k, GROUP, True, seed=0)
    d = hq.hq_quant_desc_init(hq.HQ_FMT_INT4, n, k, GROUP, 1, 1)
    blob = torch.from_numpy(hq.hq_pack_weights(d, q, s, z)).cuda()
    a = synth.bf16_normal(m, k, seed=1).cuda()
    c = torch.empty(m, n, dtype=torch.bfloat16, device="cuda")
    ws = torch.zeros(max(256, hq.hq_workspace_size(d, m)), dtype=torch.uint8, device="cuda")

    def f(cp):
        hq.hq_gemm_w4a16(d, blob, a, m, c, ws)
    ms, per = _time_launches([f], args.steps, args.warmup, world)
    st = hq.hq_check_device_status(ws)
    if st != hq.HQ_OK:
        raise RuntimeError(f"device status after the tiny timing: {hq.status_string(st)}")
    by = k * n // 2 + 2 * n * (k // GROUP) + n * (k // GROUP) + 2 * m * k + 2 * m * n
    us = per[0]
    return {"workload": "dense W4A16 tiny: M=16, K=N=1024, asymmetric INT4 group 128 (weights stay in L2)",
            "value": round(us, 2), "unit": "us per launch", "higher_is_better": False,
            "ms_per_step": round(ms / args.steps, 4), "gbs": round(by / us / 1e3, 1),
            "algorithmic_bytes": by, "gpu_launches": args.steps}


# ---------------------------------------------------------------- CPU oracle

def cpu_baseline_w4a16(budget_s=20.0):
    """Time the fp64 oracle on a bounded sample of the sweep: for each shape,
    dequantize W once and multiply 16 activation rows (the M=16 point)."""
    from oracle import gemm as G
    from oracle import formats as F
    from quantized_gemm_bit_b200 import synth
    flops, secs = 0.0, 0.0
    for si, (k, n) in enumerate(SWEEP_KN):
        q, s, _ = synth.w4a16_weights(n, k, GROUP, False, seed=1000 + si)
        a = synth.bf16_normal(16, k, seed=1016)
        bits = a.view(torch.int16).numpy().view(np.uint16)
        t = time.perf_counter()
        G.w4a16_ref(bits, q.numpy(), s.numpy(), None, GROUP)
        secs += time.perf_counter() - t
        flops += w4a16_flops(16, k, n)
        if secs > budget_s:
            break
    cores = torch.get_num_threads()
    return {"value": round(flops / secs / 1e12, 6), "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
            "sample": "M=16 rows of both sweep shapes (K,N)=(7168,18432),(18432,7168): full fp64 dequant "
                      f"of W + fp64 matmul, {secs:.1f} s"}


def run_reference(args, rank, world):
    if rank != 0:
        return None
    cb = cpu_baseline_w4a16(budget_s=args.cpu_budget)
    secs = []
    for _ in range(args.warmup):
        cpu_baseline_w4a16(budget_s=args.cpu_budget)
    t = time.perf_counter()
    for _ in range(args.steps):
        cpu_baseline_w4a16(budget_s=args.cpu_budget)
    el = time.perf_counter() - t
    flops = sum(w4a16_flops(16, k, n) for k, n in SWEEP_KN)
    value = flops * args.steps / el / 1e12
    secs.append(el)
    return {
        "impl": "reference",
        "metric": METRIC,
        "value": round(value, 6),
        "unit": "TFLOP/s",
        "n_gpus": 1,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(el / args.steps * 1e3, 2),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic (seeded)",
        "config": {"workload": "dense W4A16 M-sweep, bounded sample: the M=16 point of both (K,N) shapes",
                   "parallelism": "host cores"},
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": cb["cores"], "kind": "oracle",
                         "sample": cb["sample"]},
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="w4a16_sweep",
                    choices=["w4a16_sweep", "mxfp4", "mxfp4_a16", "w3a16", "w2a16", "w8a16", "mxint4_a16", "nvfp4", "moe",
                             "tiny"])
    ap.add_argument("--cpu-budget", type=float, default=20.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--sweep-only", action="store_true",
                    help="default workload: time the W4A16 sweep alone, without the FP4, MoE and tiny lines")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        line = run_reference(args, rank, int(os.environ.get("WORLD_SIZE", "1")))
        if line is not None:
            print(json.dumps(line), flush=True)
        return

    rank, world, _ = dist_init()
    from quantized_gemm_bit_b200.build import build
    if rank == 0:
        build()
    barrier(world)
    peaks = load_peaks()
    if args.workload == "w4a16_sweep":
        line = run_w4a16_sweep(args, rank, world, peaks)
        if not args.sweep_only:
            # the rest of the metric, each with its own roofline: the
            # block-scaled GEMMs, the MoE layer and the tiny dense case
            for key, fn in (("mxfp4_a8", run_mxfp4), ("nvfp4", run_nvfp4), ("moe", run_moe), ("tiny", run_tiny)):
                torch.cuda.empty_cache()
                line[key] = fn(args, rank, world, peaks)
    else:
        fn = {"mxfp4": run_mxfp4, "mxfp4_a16": run_mxfp4_a16, "w3a16": run_w3a16, "w2a16": run_w2a16,
              "w8a16": run_w8a16, "mxint4_a16": run_mxint4_a16, "nvfp4": run_nvfp4, "moe": run_moe,
              "tiny": run_tiny}[args.workload]
        line = {"metric": METRIC, "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                "higher_is_better": True, "scaling": "weak", "data": "synthetic (seeded)"}
        line.update(fn(args, rank, world, peaks))
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
