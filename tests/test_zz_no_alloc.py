"""GPU test of hq_gemm_w4a16_static, the W4A16 entry point that allocates
nothing (its scratch is a fixed array inside the library, for callers that
cannot allocate device memory while they run a layer).

It must give the same result as hq_gemm_w4a16 with a caller workspace, on
two calls in a row (the second call reuses the array the first one left
behind).  Kept in its own file, collected last."""

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


@pytest.mark.parametrize("m,n,k,asym", [
    (16, 7168, 18432, False),    # stream-K: partial sums and tile counters live in the scratch array
    (5, 640, 384, True),         # stream-K with three units per CTA
    (64, 18432, 7168, False),    # whole tiles (scratch holds only the error word)
])
def test_static_scratch_matches_workspace_entry_point(m, n, k, asym):
    q, s, z = synth.w4a16_weights(n, k, 128, asym, seed=9000 + m)
    a = synth.bf16_normal(m, k, seed=9001 + m).to(DEV)
    d = hq.hq_quant_desc_init(hq.HQ_FMT_INT4, n, k, 128, int(asym), 1)
    blob = torch.from_numpy(hq.hq_pack_weights(d, q, s, z)).to(DEV)
    via_ws = torch.empty(m, n, dtype=torch.bfloat16, device=DEV)
    ws = workspace(hq.hq_workspace_size(d, m))
    hq.hq_gemm_w4a16(d, blob, a, m, via_ws, ws)
    assert hq.hq_check_device_status(ws) == hq.HQ_OK
    ref = G.w4a16_ref(a.cpu().view(torch.int16).numpy().view(np.uint16), q.numpy(), s.numpy(),
                      None if z is None else z.numpy(), 128)
    for call in range(2):
        c = torch.full((m, n), float("nan"), dtype=torch.bfloat16, device=DEV)
        assert _call_static(d, blob, a, m, c) == hq.HQ_OK
        torch.cuda.synchronize()
        check_gemm(c, ref, k, f"static scratch call {call}")
        assert torch.equal(c, via_ws)      # same launch plan, same bits as the workspace entry point


def test_static_scratch_rejects_plans_beyond_its_size():
    # a 256-token tile split over all SMs needs far more than 16 MiB
    m, n, k = 1024, 7168, 18432
    d = hq.hq_quant_desc_init(hq.HQ_FMT_INT4, n, k, 128, 0, 1)
    blob = torch.zeros(hq.hq_packed_size(d), dtype=torch.uint8, device=DEV)
    a = torch.zeros(m, k, dtype=torch.bfloat16, device=DEV)
    c = torch.zeros(m, n, dtype=torch.bfloat16, device=DEV)
    t = hq.Tuning(tile_m=256, split_k=3)
    assert _call_static(d, blob, a, m, c, t) == hq.HQ_ERR_WORKSPACE_TOO_SMALL
