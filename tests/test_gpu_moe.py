"""GPU parity of the MoE path through the C ABI: top-k routing and the
expert-sorted permutation are bit-exact against the oracle; the grouped
W4A16 GEMM matches the fp64 oracle within the GEMM tolerance, in full on a
reduced configuration and on sampled rows/columns at the full workload
(256 experts, top-8, hidden 7168, gate+up N=4096, down K=2048)."""

import numpy as np
import pytest
import torch

from gpu_helpers import check_gemm, workspace
from oracle import formats as F
from oracle import gemm as G
from oracle import moe as R
from quantized_gemm_bit_b200 import hq, synth
from quantized_gemm_bit_b200.build import build

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _setup():
    build()
    torch.cuda.init()


def _bits(a):
    return a.view(torch.int16).numpy().view(np.uint16)


def gpu_route(logits, k):
    t, e = logits.shape
    ids = torch.empty(t, k, dtype=torch.int32, device=DEV)
    hq.hq_moe_topk(logits.to(DEV), t, e, k, ids)
    return ids


def gpu_permute(ids, e, a=None):
    t, k = ids.shape
    src = torch.full((t * k,), -1, dtype=torch.int32, device=DEV)
    off = torch.full((e + 1,), -1, dtype=torch.int32, device=DEV)
    ws = workspace(hq.hq_moe_permute_workspace_size(t, k, e))
    a_sorted = None
    if a is not None:
        a_sorted = torch.empty(t * k, a.shape[1], dtype=torch.bfloat16, device=DEV)
    hq.hq_moe_permute(ids, t, k, e, src, off, ws, a=None if a is None else a.to(DEV),
                      hidden=0 if a is None else a.shape[1], a_sorted=a_sorted)
    st = hq.hq_check_device_status(ws)
    return src, off, a_sorted, st


@pytest.mark.parametrize("t", [1, 64, 1024, 8192])
def test_topk_bit_exact(t):
    logits = synth.router_logits(t, 256, seed=3001 + t)
    ids = gpu_route(logits, 8).cpu().numpy()
    assert np.array_equal(ids, R.topk_by_logit(logits.numpy(), 8))


def test_topk_ties_go_to_lower_index():
    logits = torch.zeros(5, 40)
    logits[1, 7] = 1.0
    logits[2, ::3] = -1.0
    logits[3] = torch.arange(40).float() % 4
    ids = gpu_route(logits, 6).cpu().numpy()
    assert np.array_equal(ids, R.topk_by_logit(logits.numpy(), 6))


@pytest.mark.parametrize("t,e,k", [(1, 256, 8), (64, 256, 8), (1000, 256, 8), (8192, 256, 8), (37, 5, 3)])
def test_permute_and_gather_bit_exact(t, e, k):
    logits = synth.router_logits(t, e, seed=4000 + t)
    ids = R.topk_by_logit(logits.numpy(), k)
    hidden = 64
    a = synth.bf16_normal(t, hidden, seed=4100 + t)
    src, off, a_sorted, st = gpu_permute(torch.from_numpy(ids).to(DEV), e, a)
    assert st == hq.HQ_OK
    counts, off_ref, src_ref = R.permute(ids, e)
    assert np.array_equal(off.cpu().numpy(), off_ref)
    assert np.array_equal(src.cpu().numpy(), src_ref)
    ref_rows = R.gather_rows(_bits(a), src_ref, k)
    assert np.array_equal(_bits(a_sorted.cpu()), ref_rows)


def test_permute_duplicates_empty_experts_and_bad_ids():
    ids = torch.tensor([[3, 3], [0, 3], [1, 1]], dtype=torch.int32)
    src, off, _, st = gpu_permute(ids.to(DEV), 6)
    assert st == hq.HQ_OK
    _, off_ref, src_ref = R.permute(ids.numpy(), 6)
    assert np.array_equal(off.cpu().numpy(), off_ref)
    assert np.array_equal(src.cpu().numpy(), src_ref)
    bad = torch.tensor([[0, 9]], dtype=torch.int32)
    _, _, _, st = gpu_permute(bad.to(DEV), 6)
    assert st == hq.HQ_ERR_DEVICE_BAD_OFFSETS


def _grouped(desc, blob, a_sorted, off, rows, n, tuning=None):
    c = torch.empty(rows, n, dtype=torch.bfloat16, device=DEV)
    ws = workspace(hq.hq_workspace_size(desc, rows, tuning))
    hq.hq_grouped_gemm_moe(desc, blob, a_sorted, off, rows, c, ws, tuning)
    assert hq.hq_check_device_status(ws) == hq.HQ_OK
    return c


@pytest.mark.parametrize("tile_m,variant", [(0, 0), (16, 0), (32, 0), (64, 0), (128, 0), (16, 2), (32, 2), (64, 2)])
def test_grouped_reduced_config_full_output(tile_m, variant):
    e, n, k, t, topk = 8, 256, 512, 40, 2
    q, s, _ = synth.w4a16_weights(n, k, 128, False, seed=5000, experts=e)
    d = hq.hq_quant_desc_init(hq.HQ_FMT_INT4, n, k, 128, 0, e)
    blob = torch.from_numpy(hq.hq_pack_weights(d, q, s, None)).to(DEV)
    logits = synth.router_logits(t, e, seed=5001)
    logits[:, 5] = -100.0                      # expert 5 never chosen: an empty group
    ids = R.topk_by_logit(logits.numpy(), topk)
    a = synth.bf16_normal(t, k, seed=5002)
    src, off, a_sorted, st = gpu_permute(torch.from_numpy(ids).to(DEV), e, a)
    assert st == hq.HQ_OK
    tuning = hq.Tuning(tile_m=tile_m, variant=variant) if (tile_m or variant) else None
    c = _grouped(d, blob, a_sorted, off, t * topk, n, tuning)
    _, ref = G.grouped_w4a16_ref(_bits(a_sorted.cpu()), off.cpu().numpy(), q.numpy(), s.numpy(), None, 128)
    check_gemm(c, ref, k, f"grouped tile_m={tile_m} variant={variant}")


def test_grouped_bad_offsets_are_reported():
    e, n, k = 4, 128, 256
    q, s, _ = synth.w4a16_weights(n, k, 128, False, seed=5100, experts=e)
    d = hq.hq_quant_desc_init(hq.HQ_FMT_INT4, n, k, 128, 0, e)
    blob = torch.from_numpy(hq.hq_pack_weights(d, q, s, None)).to(DEV)
    a = synth.bf16_normal(10, k, seed=5101).to(DEV)
    off = torch.tensor([0, 6, 3, 8, 10], dtype=torch.int32, device=DEV)   # not monotone
    c = torch.zeros(10, n, dtype=torch.bfloat16, device=DEV)
    ws = workspace(hq.hq_workspace_size(d, 10))
    hq.hq_grouped_gemm_moe(d, blob, a, off, 10, c, ws)
    assert hq.hq_check_device_status(ws) == hq.HQ_ERR_DEVICE_BAD_OFFSETS
    assert int(c.float().abs().sum()) == 0                               # nothing written


_FULL = {}


def _full_weights(which):
    """256 experts; gate+up: N=4096, K=7168; down: N=7168, K=2048."""
    if which not in _FULL:
        n, k, seed = (4096, 7168, 3000) if which == "gate_up" else (7168, 2048, 3010)
        q, s, _ = synth.w4a16_weights(n, k, 128, False, seed=seed, experts=256)
        d = hq.hq_quant_desc_init(hq.HQ_FMT_INT4, n, k, 128, 0, 256)
        blob = torch.from_numpy(hq.hq_pack_weights(d, q, s, None)).to(DEV)
        _FULL[which] = (d, blob, q.numpy(), s.numpy(), n, k)
    return _FULL[which]


@pytest.mark.parametrize("t", [64, 1024, 8192])
@pytest.mark.parametrize("which", ["gate_up", "down"])
def test_grouped_full_size_sampled(t, which):
    d, blob, q, s, n, k = _full_weights(which)
    logits = synth.router_logits(t, 256, seed=3001)
    ids = gpu_route(logits, 8)
    if which == "gate_up":
        a = synth.bf16_normal(t, k, seed=3002)
        src, off, a_sorted, st = gpu_permute(ids, 256, a)
        assert st == hq.HQ_OK
    else:
        src, off, _, st = gpu_permute(ids, 256)
        assert st == hq.HQ_OK
        a_sorted = synth.bf16_normal(t * 8, k, seed=3003).to(DEV)
    rows_total = t * 8
    c = _grouped(d, blob, a_sorted, off, rows_total, n)
    offs = off.cpu().numpy()
    rng = np.random.default_rng(t)
    rows = []
    for ex in range(256):
        lo, hi = offs[ex], offs[ex + 1]
        if hi > lo:
            rows.extend({lo, hi - 1, int(rng.integers(lo, hi))})
    rows = np.array(sorted(set(rows)))
    cols = np.array(sorted({c0 for nt in range(n // 128) for c0 in (nt * 128, nt * 128 + 127,
                                                                     nt * 128 + int(rng.integers(0, 128)))}))
    a_rows = _bits(a_sorted[torch.from_numpy(rows).to(DEV)].cpu())
    expert_of = np.searchsorted(offs, rows, side="right") - 1
    ref = np.zeros((len(rows), len(cols)))
    for ex in np.unique(expert_of):
        sel = np.nonzero(expert_of == ex)[0]
        w = G.w4a16_dequant(q[ex], s[ex], None, 128, rows=cols)
        ref[sel] = F.bf16_bits_to_f64(a_rows[sel]) @ w.T
    got = c[torch.from_numpy(rows).to(DEV)][:, torch.from_numpy(cols).to(DEV)]
    check_gemm(got, ref, k, f"moe {which} t={t}")
