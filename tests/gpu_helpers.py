"""Shared helpers for the GPU parity tests: tolerance checks written out
from the stated bars, workspace allocation and tile-covering row samples."""

import os

import numpy as np
import torch

from quantized_gemm_bit_b200 import hq

# GEMM tolerance: relative Frobenius error <= 5e-3 and, per element,
# |err| <= 1e-2*|ref| + 2e-3*sqrt(K)*rms(ref).
REL_FRO = 5e-3
ELEM_REL = 1e-2
ELEM_ABS = 2e-3


def check_gemm(c_bf16, ref, k, what="", gemms=1):
    """GEMM output against the oracle.  `gemms` > 1 for a result that carries
    the errors of that many GEMMs in a row (a chain, checked against the
    oracle's own chain): the bars add up, so both scale by `gemms`."""
    c = c_bf16.float().double().cpu().numpy() if isinstance(c_bf16, torch.Tensor) else np.asarray(c_bf16)
    ref = np.asarray(ref, dtype=np.float64)
    assert c.shape == ref.shape, (c.shape, ref.shape)
    assert np.all(np.isfinite(c)), what
    err = c - ref
    nref = np.linalg.norm(ref)
    rel = np.linalg.norm(err) / nref if nref > 0 else np.linalg.norm(err)
    rms = np.sqrt(np.mean(ref ** 2))
    bound = gemms * (ELEM_REL * np.abs(ref) + ELEM_ABS * np.sqrt(k) * rms)
    worst = np.max(np.abs(err) - bound)
    log = os.environ.get("HQ_PARITY_LOG")
    if log:   # one line per check: label, rel Frobenius, worst |err| / element bound
        with open(log, "a") as f:
            f.write(f"{what}\t{rel:.3e}\t{np.max(np.abs(err) / np.maximum(bound, 1e-300)):.3e}\n")
    assert rel <= gemms * REL_FRO, f"{what}: rel Frobenius {rel:.3e}"
    assert worst <= 0, f"{what}: element bound exceeded by {worst:.3e}"
    return rel


def workspace(nbytes, device="cuda"):
    # torch's caching allocator returns 512-byte aligned blocks
    ws = torch.zeros(max(256, nbytes), dtype=torch.uint8, device=device)
    assert ws.data_ptr() % 256 == 0
    return ws


def tile_rows(m, tile, rng, per_tile=2):
    """First and last row of every `tile`-row tile plus a few random rows."""
    rows = set()
    for t0 in range(0, m, tile):
        t1 = min(m, t0 + tile) - 1
        rows.update({t0, t1})
        rows.update(rng.integers(t0, t1 + 1, size=per_tile).tolist())
    return np.array(sorted(rows))


def check_swiglu(h_bf16, gate_up_ref, inter, k, what=""):
    """Output of the gate+up GEMM with the fused SwiGLU epilogue against the
    oracle's fp64 gate and up values (one GEMM's output, so the GEMM's
    relative Frobenius bar), and per element the GEMM element bound carried
    through h = silu(g) * u to first order,
        |err_h| <= |silu'(g) u| B + |silu(g)| B + 2^-8 |h|,
    B = 1e-2 |ref| + 2e-3 sqrt(K) rms(ref) taken for g and u, plus the
    bf16 rounding of h."""
    h = h_bf16.float().double().cpu().numpy() if isinstance(h_bf16, torch.Tensor) else np.asarray(h_bf16)
    gu = np.asarray(gate_up_ref, dtype=np.float64)
    g, u = gu[:, :inter], gu[:, inter:2 * inter]
    sig = 1.0 / (1.0 + np.exp(-g))
    ref = g * sig * u
    dsilu = sig * (1.0 + g * (1.0 - sig))
    rms = np.sqrt(np.mean(gu ** 2))
    bg = ELEM_REL * np.abs(g) + ELEM_ABS * np.sqrt(k) * rms
    bu = ELEM_REL * np.abs(u) + ELEM_ABS * np.sqrt(k) * rms
    bound = np.abs(dsilu * u) * bg + np.abs(g * sig) * bu + 2.0 ** -8 * np.abs(ref)
    assert h.shape == ref.shape and np.all(np.isfinite(h)), what
    err = h - ref
    rel = np.linalg.norm(err) / np.linalg.norm(ref)
    log = os.environ.get("HQ_PARITY_LOG")
    if log:
        with open(log, "a") as f:
            f.write(f"{what}\t{rel:.3e}\t{np.max(np.abs(err) / np.maximum(bound, 1e-300)):.3e}\n")
    assert rel <= REL_FRO, f"{what}: rel Frobenius {rel:.3e}"
    worst = np.max(np.abs(err) - bound)
    assert worst <= 0, f"{what}: element bound exceeded by {worst:.3e}"
    return rel
