"""GPU test of hq_gemm_w4a16_static, the W4A16 entry point that allocates
nothing (its scratch is a fixed array inside the library, for callers that
cannot allocate device memory while they run a layer).

It must give the same result as hq_gemm_w4a16 with a caller workspace, on
two calls in a row (the second call reuses the array the first one left
behind), for every weight format of the W4A16 kernels; where the workspace
entry point's plan would not fit the array, it must still match the
oracle.  Kept in its own file, collected last."""

import ctypes

import numpy as np
import pytest
import torch

from gpu_helpers import check_gemm, workspace
from oracle import gemm as G
from quantized_gemm_bit_b200 import hq, synth
from quantized_gemm_bit_b200.build import build

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _setup():
    build()
    torch.cuda.init()


def _call_static(d, blob, a, m, c, tuning=None):
    L = hq.lib()
    st = L.hq_gemm_w4a16_static(ctypes.byref(d), blob.data_ptr(), a.data_ptr(), int(m), c.data_ptr(),
                                hq._tuning(tuning), torch.cuda.current_stream().cuda_stream)
    return st


def _weights(fmt, n, k, asym, seed):
    """Canonical weights, descriptor, packed blob and the oracle's function
    for one format (asym: zero points, where the format has them)."""
    if fmt == hq.HQ_FMT_MXFP4_A16:
        codes, e8 = synth.mxfp4_weights(n, k, seed=seed)
        d = hq.hq_quant_desc_init(fmt, n, k, 32, 0, 1)
        blob = torch.from_numpy(hq.hq_pack_weights(d, codes, e8)).to(DEV)
        return d, blob, lambda bits: G.mxfp4_a16_ref(bits, codes.numpy(), e8.numpy())
    make, ref = {hq.HQ_FMT_INT4: (synth.w4a16_weights, G.w4a16_ref), hq.HQ_FMT_INT3: (synth.w3a16_weights, G.w3a16_ref),
                 hq.HQ_FMT_INT2: (synth.w2a16_weights, G.w2a16_ref)}[fmt]
    q, s, z = make(n, k, 128, asym, seed)
    d = hq.hq_quant_desc_init(fmt, n, k, 128, int(asym), 1)
    blob = torch.from_numpy(hq.hq_pack_weights(d, q, s, z)).to(DEV)
    return d, blob, lambda bits: ref(bits, q.numpy(), s.numpy(), None if z is None else z.numpy(), 128)


def _bits(a):
    return a.cpu().view(torch.int16).numpy().view(np.uint16)


@pytest.mark.parametrize("fmt,m,n,k,asym", [
    (hq.HQ_FMT_INT4, 16, 7168, 18432, False),   # stream-K: partial sums and tile counters live in the scratch array
    (hq.HQ_FMT_INT4, 5, 640, 384, True),        # stream-K with three units per CTA
    (hq.HQ_FMT_INT4, 64, 18432, 7168, False),   # whole tiles (scratch holds only the error word)
    (hq.HQ_FMT_INT3, 5, 640, 384, True),        # the other weight formats of the W4A16 kernels, K split
    (hq.HQ_FMT_INT2, 5, 640, 384, True),
    (hq.HQ_FMT_MXFP4_A16, 5, 640, 384, False),
])
def test_static_scratch_matches_workspace_entry_point(fmt, m, n, k, asym):
    d, blob, oracle_fn = _weights(fmt, n, k, asym, 9000 + m + fmt)
    a = synth.bf16_normal(m, k, seed=9001 + m).to(DEV)
    via_ws = torch.empty(m, n, dtype=torch.bfloat16, device=DEV)
    ws = workspace(hq.hq_workspace_size(d, m))
    hq.hq_gemm_w4a16(d, blob, a, m, via_ws, ws)
    assert hq.hq_check_device_status(ws) == hq.HQ_OK
    ref = oracle_fn(_bits(a))
    for call in range(2):
        c = torch.full((m, n), float("nan"), dtype=torch.bfloat16, device=DEV)
        assert _call_static(d, blob, a, m, c) == hq.HQ_OK
        torch.cuda.synchronize()
        check_gemm(c, ref, k, f"static scratch fmt={fmt} call {call}")
        assert torch.equal(c, via_ws)      # same launch plan, same bits as the workspace entry point
    assert hq.hq_static_check_device_status() == hq.HQ_OK


def test_static_scratch_runs_whole_tiles_when_the_split_tail_does_not_fit():
    """M=2048, N=7168: 448 256-token tiles, three full waves and a ragged
    one, which hq_gemm_w4a16 runs as whole tiles plus a split-K tail whose
    partial sums (about 39 MB) exceed the array; the allocation-free entry
    point runs whole tiles instead (another plan, so it is checked against
    the oracle, twice)."""
    m, n, k = 2048, 7168, 512
    d, blob, oracle_fn = _weights(hq.HQ_FMT_INT4, n, k, True, 9100)
    assert hq.hq_workspace_size(d, m) > (16 << 20)
    a = synth.bf16_normal(m, k, seed=9101).to(DEV)
    ref = oracle_fn(_bits(a))
    for call in range(2):
        c = torch.full((m, n), float("nan"), dtype=torch.bfloat16, device=DEV)
        assert _call_static(d, blob, a, m, c) == hq.HQ_OK
        torch.cuda.synchronize()
        check_gemm(c, ref, k, f"static scratch whole-tile fallback call {call}")
    assert hq.hq_static_check_device_status() == hq.HQ_OK


def test_static_scratch_rejects_plans_beyond_its_size():
    # a 256-token tile split over all SMs needs far more than 16 MiB
    m, n, k = 1024, 7168, 18432
    d = hq.hq_quant_desc_init(hq.HQ_FMT_INT4, n, k, 128, 0, 1)
    blob = torch.zeros(hq.hq_packed_size(d), dtype=torch.uint8, device=DEV)
    a = torch.zeros(m, k, dtype=torch.bfloat16, device=DEV)
    c = torch.zeros(m, n, dtype=torch.bfloat16, device=DEV)
    t = hq.Tuning(tile_m=256, split_k=3)
    assert _call_static(d, blob, a, m, c, t) == hq.HQ_ERR_WORKSPACE_TOO_SMALL
