"""Run one GEMM configuration a few times through the C ABI, for profilers.

    python -m quantized_gemm_bit_b200.profile_case --kind w4a16 --m 16 --k 7168 --n 18432 --iters 3
    python -m quantized_gemm_bit_b200.profile_case --kind nvfp4 --m 8192 --k 8192 --n 8192 --iters 2
    python -m quantized_gemm_bit_b200.profile_case --kind w3a16 --m 16 --k 7168 --n 18432 --iters 3

Inputs are the seeded synthetic workload tensors; the device status is
checked at the end (non-zero exit on any error).  Used to capture ncu
profiles of single kernels on small, self-terminating cases.
"""

import argparse
import sys

import torch

from . import hq, synth
from .build import build


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--kind", default="w4a16",
                    choices=["w4a16", "w3a16", "w2a16", "w8a16", "mxfp4_a16", "mxint4_a16", "moe", "moe_swiglu",
                             "mxfp4", "nvfp4"])
    ap.add_argument("--m", type=int, default=16)
    ap.add_argument("--k", type=int, default=7168)
    ap.add_argument("--n", type=int, default=18432)
    ap.add_argument("--experts", type=int, default=256)
    ap.add_argument("--topk", type=int, default=8)
    ap.add_argument("--iters", type=int, default=3)
    ap.add_argument("--asym", action="store_true")
    ap.add_argument("--tile-m", type=int, default=0)
    ap.add_argument("--split-k", type=int, default=0)
    ap.add_argument("--variant", type=int, default=0)
    ap.add_argument("--stages", type=int, default=0)
    ap.add_argument("--cta-group", type=int, default=0, help="block-scaled: 1 = one CTA per tile, 2 = CTA pairs")
    a = ap.parse_args(argv)
    build()
    dev = "cuda"
    tuning = (hq.Tuning(tile_m=a.tile_m, split_k=a.split_k, variant=a.variant, stages=a.stages,
                        cta_group=a.cta_group)
              if (a.tile_m or a.split_k or a.variant or a.stages or a.cta_group) else None)
    if a.kind in ("mxfp4", "nvfp4"):
        ws = None
        if a.kind == "mxfp4":
            codes, e8 = synth.mxfp4_weights(a.n, a.k, seed=2000)
            d = hq.hq_quant_desc_init(hq.HQ_FMT_MXFP4, a.n, a.k, 32, 0, 1)
            blob = torch.from_numpy(hq.hq_pack_weights(d, codes, e8)).to(dev)
            x = synth.bf16_normal(a.m, a.k, seed=2001).to(dev)
            xq = torch.empty(a.m, a.k, dtype=torch.uint8, device=dev)
            xs = torch.empty(a.m, dtype=torch.float32, device=dev)
            hq.hq_quantize_fp8_rows(x, a.m, a.k, xq, xs)
            run = lambda c, ws: hq.hq_gemm_mxfp4_a8(d, blob, xq, xs, a.m, c, ws, tuning)
        else:
            def quant(rows, seed):
                x = synth.bf16_normal(rows, a.k, seed).to(dev)
                codes = torch.empty(rows, a.k // 2, dtype=torch.uint8, device=dev)
                sf = torch.empty(rows, a.k // 16, dtype=torch.uint8, device=dev)
                g = torch.empty(1, dtype=torch.float32, device=dev)
                wsq = torch.zeros(hq.hq_quantize_nvfp4_workspace_size(rows, a.k), dtype=torch.uint8, device=dev)
                hq.hq_quantize_nvfp4(x, rows, a.k, codes, sf, g, wsq)
                return codes, sf, g
            wc, wsf, wg = quant(a.n, 4000)
            ac, asf, ag = quant(a.m, 4100)
            d = hq.hq_quant_desc_init(hq.HQ_FMT_NVFP4, a.n, a.k, 16, 0, 1)
            blob = torch.from_numpy(hq.hq_pack_weights(d, wc.cpu(), wsf.cpu(), None, float(wg.item()))).to(dev)
            a_g = float(ag.item())
            run = lambda c, ws: hq.hq_gemm_nvfp4(d, blob, ac, asf, a_g, a.m, c, ws, tuning)
        c = torch.empty(a.m, a.n, dtype=torch.bfloat16, device=dev)
        ws = torch.zeros(max(256, hq.hq_workspace_size(d, a.m, tuning)), dtype=torch.uint8, device=dev)
        for _ in range(a.iters):
            run(c, ws)
    elif a.kind in ("w4a16", "w3a16", "w2a16", "w8a16", "mxfp4_a16", "mxint4_a16"):
        # the W4A16 kernels with INT4, INT3, INT2, INT8, MXFP4 or MXINT4 weights
        if a.kind == "w4a16":
            q, s, z = synth.w4a16_weights(a.n, a.k, 128, a.asym, seed=1000)
            d = hq.hq_quant_desc_init(hq.HQ_FMT_INT4, a.n, a.k, 128, int(a.asym), 1)
            blob = torch.from_numpy(hq.hq_pack_weights(d, q, s, z)).to(dev)
        elif a.kind == "w3a16":
            q, s, z = synth.w3a16_weights(a.n, a.k, 128, a.asym, seed=7000)
            d = hq.hq_quant_desc_init(hq.HQ_FMT_INT3, a.n, a.k, 128, int(a.asym), 1)
            blob = torch.from_numpy(hq.hq_pack_weights(d, q, s, z)).to(dev)
        elif a.kind == "w2a16":
            q, s, z = synth.w2a16_weights(a.n, a.k, 128, a.asym, seed=7500)
            d = hq.hq_quant_desc_init(hq.HQ_FMT_INT2, a.n, a.k, 128, int(a.asym), 1)
            blob = torch.from_numpy(hq.hq_pack_weights(d, q, s, z)).to(dev)
        elif a.kind == "w8a16":
            q, s, z = synth.w8a16_weights(a.n, a.k, 128, a.asym, seed=7800)
            d = hq.hq_quant_desc_init(hq.HQ_FMT_INT8, a.n, a.k, 128, int(a.asym), 1)
            blob = torch.from_numpy(hq.hq_pack_weights(d, q, s, z)).to(dev)
        elif a.kind == "mxint4_a16":
            codes, e8 = synth.mxint4_weights(a.n, a.k, seed=7900)
            d = hq.hq_quant_desc_init(hq.HQ_FMT_MXINT4, a.n, a.k, 32, 0, 1)
            blob = torch.from_numpy(hq.hq_pack_weights(d, codes, e8)).to(dev)
        else:
            codes, e8 = synth.mxfp4_weights(a.n, a.k, seed=6000)
            d = hq.hq_quant_desc_init(hq.HQ_FMT_MXFP4_A16, a.n, a.k, 32, 0, 1)
            blob = torch.from_numpy(hq.hq_pack_weights(d, codes, e8)).to(dev)
        x = synth.bf16_normal(a.m, a.k, seed=1001).to(dev)
        c = torch.empty(a.m, a.n, dtype=torch.bfloat16, device=dev)
        ws = torch.zeros(max(256, hq.hq_workspace_size(d, a.m, tuning)), dtype=torch.uint8, device=dev)
        for _ in range(a.iters):
            hq.hq_gemm_w4a16(d, blob, x, a.m, c, ws, tuning)
    else:
        t, e, k_top = a.m, a.experts, a.topk
        q, s, _ = synth.w4a16_weights(a.n, a.k, 128, False, seed=3000, experts=e)
        d = hq.hq_quant_desc_init(hq.HQ_FMT_INT4, a.n, a.k, 128, 0, e)
        gated = a.kind == "moe_swiglu"       # gate+up weights in the gated order, SwiGLU in the epilogue
        blob = torch.from_numpy((hq.hq_pack_weights_gated if gated else hq.hq_pack_weights)(d, q, s, None)).to(dev)
        logits = synth.router_logits(t, e, seed=3001).to(dev)
        x = synth.bf16_normal(t, a.k, seed=3002).to(dev)
        ids = torch.empty(t, k_top, dtype=torch.int32, device=dev)
        src = torch.empty(t * k_top, dtype=torch.int32, device=dev)
        off = torch.empty(e + 1, dtype=torch.int32, device=dev)
        xs = torch.empty(t * k_top, a.k, dtype=torch.bfloat16, device=dev)
        c = torch.empty(t * k_top, a.n // 2 if gated else a.n, dtype=torch.bfloat16, device=dev)
        pws = torch.zeros(hq.hq_moe_permute_workspace_size(t, k_top, e), dtype=torch.uint8, device=dev)
        ws = torch.zeros(max(256, hq.hq_workspace_size(d, t * k_top, tuning)), dtype=torch.uint8, device=dev)
        for _ in range(a.iters):
            hq.hq_moe_topk(logits, t, e, k_top, ids)
            hq.hq_moe_permute(ids, t, k_top, e, src, off, pws, a=x, hidden=a.k, a_sorted=xs)
            if gated:
                hq.hq_grouped_gemm_moe_swiglu(d, blob, xs, off, t * k_top, c, ws, tuning)
            else:
                hq.hq_grouped_gemm_moe(d, blob, xs, off, t * k_top, c, ws, tuning)
        st = hq.hq_check_device_status(pws)
        if st != hq.HQ_OK:
            print("device status", hq.status_string(st))
            return 1
    torch.cuda.synchronize()
    st = hq.hq_check_device_status(ws)
    if st != hq.HQ_OK:
        print("device status", hq.status_string(st))
        return 1
    print("ok")
    return 0


if __name__ == "__main__":
    sys.exit(main())
