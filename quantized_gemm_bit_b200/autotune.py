"""Offline autotuning of the launch plan for one GEMM shape, through the C ABI.

The pages separate the quantization description from the execution choices
(token tile, K split, MMA variant) and leave the choice to heuristics, with
tuning on the roadmap ("Humming: open-source kernel library for quantized
inference", summary paragraph 3 and key points).  This sweeps those choices
for one shape on the GPU at hand:

    python -m quantized_gemm_bit_b200.autotune --kind w4a16 --m 16 --k 7168 --n 18432
    python -m quantized_gemm_bit_b200.autotune --kind mxfp4 --m 256 --k 7168 --n 7168
    python -m quantized_gemm_bit_b200.autotune --kind mxfp4_a16 --m 16 --k 7168 --n 18432
    python -m quantized_gemm_bit_b200.autotune --kind w3a16 --m 16 --k 7168 --n 18432
    python -m quantized_gemm_bit_b200.autotune --kind moe --m 1024 --k 7168 --n 4096

Every candidate `hq_tuning` (and the library's own choice, `None`) runs as a
CUDA graph of back-to-back launches over weight copies rotating across more
than 3x L2, timed with CUDA events; candidates the library refuses are
skipped, and a candidate whose run records a device-side error is an error.
The result is a table sorted by time plus the best tuning and its speed-up
over the library's choice: one entry of a per-shape heuristic table.  With
--table PATH the entry is merged into a JSON table file, which load_table()
installs in the library (hq_tuning_table_set): calls of that shape that pass
no tuning then run the table's plan.

    python -m quantized_gemm_bit_b200.autotune --kind w4a16 --m 16 --table tuning.json --m-range 1,16
"""

import argparse
import json
import os

import torch

from . import hq, synth

TILES = (16, 32, 64, 128, 256)


STAGES = (0, 2, 4)


def candidates(kind, m):
    """Tunings worth trying at m rows: token tiles up to twice the rows
    (at least 16), K splits 0 (the library's choice) to 3, pipeline stages
    in flight (0 = the kernel's whole ring, 2, 4), for the W4A16 kernels
    with INT4, INT3, INT2 or INT8 weights both weight variants (the MX
    formats have only the rescaled one), and for the block-scaled GEMMs
    with 128/256-token tiles one CTA per weight tile or CTA pairs."""
    cap = max(16, 2 * m)
    tiles = [t for t in TILES if t <= cap] or [16]
    variants = ((1, 2) if kind in ("w4a16", "moe", "w3a16", "w2a16", "w8a16")
                else (1,) if kind in ("mxfp4_a16", "mxint4_a16") else (0,))
    splits = (0,) if kind == "moe" else (0, 1, 2, 3)
    out = [None]
    for t in tiles:
        for s in splits:
            for v in variants:
                if v == 2 and t > 64:
                    continue
                for st in STAGES:
                    out.append(hq.Tuning(tile_m=t, split_k=s, variant=v, stages=st))
    # block-scaled 128/256-token whole tiles: one CTA per weight tile, or
    # CTA pairs (the library's choice at 256 picks either)
    if kind in ("mxfp4", "nvfp4"):
        for t in (x for x in tiles if x >= 128):
            for g in (1, 2):
                for st in STAGES:
                    out.append(hq.Tuning(tile_m=t, cta_group=g, stages=st))
    return out


def _describe(t):
    return ("library" if t is None
            else f"tile_m={t.tile_m} split_k={t.split_k} variant={t.variant} stages={t.stages}"
                 + (f" cta_group={t.cta_group}" if t.cta_group else ""))


def _tuning_dict(t):
    return {f: int(getattr(t, f)) for f, _ in hq.Tuning._fields_}


def table_entry(d, m_min, m_max, t):
    """One entry of the per-shape table (a dict, as the JSON file holds it)."""
    return {"fmt": int(d.fmt), "n": int(d.n), "k": int(d.k), "num_experts": int(d.num_experts),
            "m_min": int(m_min), "m_max": int(m_max), "tuning": _tuning_dict(t)}


def merge_table(path, entry):
    """Add `entry` to the JSON table at `path`, replacing an entry of the
    same shape and m range."""
    table = {"entries": []}
    if os.path.exists(path):
        with open(path) as f:
            table = json.load(f)
    key = lambda e: (e["fmt"], e["n"], e["k"], e["num_experts"], e["m_min"], e["m_max"])
    table["entries"] = [e for e in table["entries"] if key(e) != key(entry)] + [entry]
    with open(path, "w") as f:
        json.dump(table, f, indent=1)
    return table


def load_table(path):
    """Install the JSON table at `path` in the library (hq_tuning_table_set)."""
    with open(path) as f:
        table = json.load(f)
    hq.hq_tuning_table_set(table["entries"])
    return table


def _time(fn, ncopy, reps=3):
    """Mean microseconds per call of fn(copy) in a CUDA graph of max(ncopy, 4)
    back-to-back calls, replayed `reps` times after one warm replay."""
    r = max(ncopy, 4)
    for i in range(2):
        fn(i % ncopy)
    torch.cuda.synchronize()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=side):
        for i in range(r):
            fn(i % ncopy)
    torch.cuda.current_stream().wait_stream(side)
    g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    g.replay()
    e0.record()
    for _ in range(reps):
        g.replay()
    e1.record()
    torch.cuda.synchronize()
    del g
    return e0.elapsed_time(e1) * 1e3 / (reps * r)


def _copies(blob):
    l2 = getattr(torch.cuda.get_device_properties(torch.cuda.current_device()), "L2_cache_size", 126 << 20)
    n = max(2, -(-3 * l2 // blob.numel()) + 1)
    return [blob] + [blob.clone() for _ in range(n - 1)]


def _setup(kind, m, n, k, experts, topk, dev):
    """Seeded synthetic inputs of the shape and a call(tuning, copy, c, ws)."""
    if kind == "w4a16":
        q, s, _ = synth.w4a16_weights(n, k, 128, False, seed=1000)
        d = hq.hq_quant_desc_init(hq.HQ_FMT_INT4, n, k, 128, 0, 1)
        blobs = _copies(torch.from_numpy(hq.hq_pack_weights(d, q, s, None)).to(dev))
        a = synth.bf16_normal(m, k, seed=1001).to(dev)
        rows = m

        def call(t, i, c, ws):
            hq.hq_gemm_w4a16(d, blobs[i], a, m, c, ws, t)
    elif kind in ("w3a16", "w2a16", "w8a16"):
        if kind == "w3a16":
            q, s, _ = synth.w3a16_weights(n, k, 128, False, seed=7000)
            d = hq.hq_quant_desc_init(hq.HQ_FMT_INT3, n, k, 128, 0, 1)
        elif kind == "w8a16":
            q, s, _ = synth.w8a16_weights(n, k, 128, False, seed=7800)
            d = hq.hq_quant_desc_init(hq.HQ_FMT_INT8, n, k, 128, 0, 1)
        else:
            q, s, _ = synth.w2a16_weights(n, k, 128, False, seed=7500)
            d = hq.hq_quant_desc_init(hq.HQ_FMT_INT2, n, k, 128, 0, 1)
        blobs = _copies(torch.from_numpy(hq.hq_pack_weights(d, q, s, None)).to(dev))
        a = synth.bf16_normal(m, k, seed=7001).to(dev)
        rows = m

        def call(t, i, c, ws):
            hq.hq_gemm_w4a16(d, blobs[i], a, m, c, ws, t)
    elif kind in ("mxfp4_a16", "mxint4_a16"):
        mxi = kind == "mxint4_a16"
        codes, e8 = (synth.mxint4_weights if mxi else synth.mxfp4_weights)(n, k, seed=6000)
        d = hq.hq_quant_desc_init(hq.HQ_FMT_MXINT4 if mxi else hq.HQ_FMT_MXFP4_A16, n, k, 32, 0, 1)
        blobs = _copies(torch.from_numpy(hq.hq_pack_weights(d, codes, e8)).to(dev))
        a = synth.bf16_normal(m, k, seed=6001).to(dev)
        rows = m

        def call(t, i, c, ws):
            hq.hq_gemm_w4a16(d, blobs[i], a, m, c, ws, t)
    elif kind == "mxfp4":
        codes, e8 = synth.mxfp4_weights(n, k, seed=2000)
        d = hq.hq_quant_desc_init(hq.HQ_FMT_MXFP4, n, k, 32, 0, 1)
        blobs = _copies(torch.from_numpy(hq.hq_pack_weights(d, codes, e8)).to(dev))
        # E4M3 activations from the library's own per-token quantizer
        x = synth.bf16_normal(m, k, seed=2001).to(dev)
        aq = torch.empty(m, k, dtype=torch.uint8, device=dev)
        asc = torch.empty(m, dtype=torch.float32, device=dev)
        hq.hq_quantize_fp8_rows(x, m, k, aq, asc)
        rows = m

        def call(t, i, c, ws):
            hq.hq_gemm_mxfp4_a8(d, blobs[i], aq, asc, m, c, ws, t)
    elif kind == "nvfp4":
        def quant(r, seed):
            x = synth.bf16_normal(r, k, seed).to(dev)
            codes = torch.empty(r, k // 2, dtype=torch.uint8, device=dev)
            sf = torch.empty(r, k // 16, dtype=torch.uint8, device=dev)
            g = torch.empty(1, dtype=torch.float32, device=dev)
            wsq = torch.zeros(hq.hq_quantize_nvfp4_workspace_size(r, k), dtype=torch.uint8, device=dev)
            hq.hq_quantize_nvfp4(x, r, k, codes, sf, g, wsq)
            return codes, sf, float(g.item())
        wc, wsf, wg = quant(n, 4000)
        ac, asf, ag = quant(m, 4100)
        d = hq.hq_quant_desc_init(hq.HQ_FMT_NVFP4, n, k, 16, 0, 1)
        blobs = _copies(torch.from_numpy(hq.hq_pack_weights(d, wc.cpu(), wsf.cpu(), None, wg)).to(dev))
        rows = m

        def call(t, i, c, ws):
            hq.hq_gemm_nvfp4(d, blobs[i], ac, asf, ag, m, c, ws, t)
    elif kind == "moe":
        # m = tokens routed top-k over `experts`; the grouped GEMM runs on the
        # m * topk expert-sorted rows
        q, s, _ = synth.w4a16_weights(n, k, 128, False, seed=3000, experts=experts)
        d = hq.hq_quant_desc_init(hq.HQ_FMT_INT4, n, k, 128, 0, experts)
        blobs = [torch.from_numpy(hq.hq_pack_weights(d, q, s, None)).to(dev)]
        logits = synth.router_logits(m, experts, seed=3001).to(dev)
        ids = torch.empty(m, topk, dtype=torch.int32, device=dev)
        src = torch.empty(m * topk, dtype=torch.int32, device=dev)
        off = torch.empty(experts + 1, dtype=torch.int32, device=dev)
        pws = torch.zeros(hq.hq_moe_permute_workspace_size(m, topk, experts), dtype=torch.uint8, device=dev)
        hq.hq_moe_topk(logits, m, experts, topk, ids)
        hq.hq_moe_permute(ids, m, topk, experts, src, off, pws)
        rows = m * topk
        a = synth.bf16_normal(rows, k, seed=3002).to(dev)

        def call(t, i, c, ws):
            hq.hq_grouped_gemm_moe(d, blobs[i], a, off, rows, c, ws, t)
    else:
        raise ValueError(kind)
    return d, rows, len(blobs), call


def autotune(kind, m, n, k, experts=256, topk=8, tunings=None, dev="cuda"):
    """Times every candidate tuning; returns (rows sorted by time, best row,
    the library's row).  A row is {"tuning": ..., "us": ..., "desc": ...}."""
    d, rows, ncopy, call = _setup(kind, m, n, k, experts, topk, dev)
    c = torch.empty(rows, n, dtype=torch.bfloat16, device=dev)
    results = []
    for t in (candidates(kind, m) if tunings is None else tunings):
        try:
            ws = torch.zeros(max(256, hq.hq_workspace_size(d, rows, t)), dtype=torch.uint8, device=dev)
            us = _time(lambda i: call(t, i, c, ws), ncopy)
        except hq.HQError:
            continue                      # refused by the library: not a valid plan here
        st = hq.hq_check_device_status(ws)
        if st != hq.HQ_OK:
            raise RuntimeError(f"{_describe(t)}: device status {hq.status_string(st)}")
        results.append({"tuning": t, "us": us, "desc": _describe(t)})
    results.sort(key=lambda r: r["us"])
    library = next(r for r in results if r["tuning"] is None)
    return results, results[0], library, d, rows


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--kind", default="w4a16",
                    choices=["w4a16", "w3a16", "w2a16", "w8a16", "mxfp4_a16", "mxint4_a16", "mxfp4", "nvfp4", "moe"])
    ap.add_argument("--m", type=int, default=16, help="rows (tokens for --kind moe)")
    ap.add_argument("--k", type=int, default=7168)
    ap.add_argument("--n", type=int, default=18432)
    ap.add_argument("--experts", type=int, default=256)
    ap.add_argument("--topk", type=int, default=8)
    ap.add_argument("--table", default=None, help="merge the best tuning into this JSON table file")
    ap.add_argument("--m-range", default=None, help="lo,hi: the rows the table entry applies to (default m,m)")
    a = ap.parse_args(argv)
    from .build import build
    build()
    results, best, library, d, rows = autotune(a.kind, a.m, a.n, a.k, a.experts, a.topk)
    for r in results:
        print(f"{r['us']:10.2f} us  {r['desc']}")
    t = best["tuning"]
    print(json.dumps({"kind": a.kind, "m": a.m, "n": a.n, "k": a.k,
                      "best": None if t is None else _tuning_dict(t),
                      "best_us": round(best["us"], 2), "library_us": round(library["us"], 2),
                      "speedup_over_library": round(library["us"] / best["us"], 3)}))
    if a.table and t is not None:
        lo, hi = (rows, rows) if a.m_range is None else (int(x) for x in a.m_range.split(","))
        merge_table(a.table, table_entry(d, lo, hi, t))


if __name__ == "__main__":
    main()
