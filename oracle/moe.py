"""MoE routing and expert-sorted permutation (test infrastructure).

The pages name a "Grouped" MoE path ("Humming: open-source kernel library
for quantized inference", summary, fifth paragraph: the grouped MoE path on
B300; Humming news page, comparison table row "MoE W4A16, B300, large
batch").  They do not describe routing; the workload fixes top-8 of 256
experts from a softmax over router logits, with tokens permuted into
expert-sorted order and per-expert row offsets.

Readings (the pages are silent):
  * top-k by probability equals top-k by logit (softmax is monotone), so
    selection is done on the logits, exactly, without exp rounding;
  * ties go to the lower expert index; slots within a token are ordered by
    descending logit (ties: lower index first);
  * the sorted order is (expert ascending, flattened slot index t*k+j
    ascending), which is unique and therefore bit-exactly checkable;
  * the layer around the two grouped GEMMs is the usual gated MoE feed-
    forward: the gate+up GEMM's N = 2I columns are the gate (first I) and
    the up projection (last I), h = silu(gate) * up with
    silu(x) = x / (1 + exp(-x)); the down GEMM's rows are un-permuted and
    summed per token with the softmax probabilities of the selected
    experts as weights (over all E experts, not renormalised over the k).
"""

import numpy as np

from .formats import bf16_bits_to_f64


def topk_by_logit(logits, k):
    """logits fp32 [T, E] -> expert ids int32 [T, k], descending logit,
    ties to the lower expert index."""
    l = np.asarray(logits, dtype=np.float32)
    t, e = l.shape
    order = np.argsort(-l.astype(np.float64), axis=1, kind="stable")
    return order[:, :k].astype(np.int32)


def softmax_topk_weights(logits, ids):
    """Softmax probabilities (fp64) of the selected experts, not
    renormalised: the combine weights."""
    l = np.asarray(logits, dtype=np.float64)
    p = np.exp(l - l.max(axis=1, keepdims=True))
    p /= p.sum(axis=1, keepdims=True)
    return np.take_along_axis(p, np.asarray(ids, dtype=np.int64), axis=1)


def permute(topk_ids, num_experts):
    """topk ids [T, k] -> (counts [E], offsets [E+1], sorted_src [T*k]).

    counts[e]  = number of slots routed to e;
    offsets    = exclusive prefix sum of counts, offsets[E] = T*k;
    sorted_src = flattened slot indices t*k+j ordered by (expert, t*k+j).
    """
    ids = np.asarray(topk_ids, dtype=np.int64).ravel()
    counts = np.bincount(ids, minlength=num_experts).astype(np.int32)
    offsets = np.zeros(num_experts + 1, dtype=np.int32)
    offsets[1:] = np.cumsum(counts)
    # explicit (expert, slot) ordering: build buckets slot by slot
    buckets = [[] for _ in range(num_experts)]
    for slot, e in enumerate(ids.tolist()):
        buckets[e].append(slot)
    sorted_src = np.array([s for b in buckets for s in b], dtype=np.int32)
    return counts, offsets, sorted_src


def gather_rows(a, sorted_src, k):
    """A_sorted[i] = A[sorted_src[i] // k] (a bit copy of the bf16 row)."""
    src_tok = np.asarray(sorted_src, dtype=np.int64) // k
    return np.asarray(a)[src_tok]


def silu_mul(gate_up_bf16_bits, inter):
    """SwiGLU of the gate+up output: bf16 bits [rows, 2*inter] ->
    fp64 [rows, inter], h = silu(g) * u, g = columns [0, inter),
    u = columns [inter, 2*inter), silu(x) = x / (1 + exp(-x))."""
    x = bf16_bits_to_f64(gate_up_bf16_bits)
    g, u = x[:, :inter], x[:, inter:2 * inter]
    with np.errstate(over="ignore"):
        return g / (1.0 + np.exp(-g)) * u


def silu_mul_f64(gate_up, inter):
    """SwiGLU on unrounded gate+up values: fp64 [rows, 2*inter] -> fp64
    [rows, inter], h = silu(g) * u as in silu_mul (the form the GEMM with
    the fused SwiGLU epilogue computes: no bf16 rounding of g and u)."""
    x = np.asarray(gate_up, dtype=np.float64)
    g, u = x[:, :inter], x[:, inter:2 * inter]
    with np.errstate(over="ignore"):
        return g / (1.0 + np.exp(-g)) * u


def combine(y_sorted_bf16_bits, sorted_src, weights, k):
    """Un-permute and weigh the down GEMM's output: bf16 bits
    [T*k, H] in expert-sorted order -> fp64 [T, H],
    out[t] = sum_j weights[t, j] * Y[p(t, j)] where sorted_src[p] = t*k + j."""
    y = bf16_bits_to_f64(y_sorted_bf16_bits)
    src = np.asarray(sorted_src, dtype=np.int64)
    w = np.asarray(weights, dtype=np.float64)
    t = len(src) // k
    pos = np.empty(len(src), dtype=np.int64)
    pos[src] = np.arange(len(src))            # position of every flattened slot
    out = np.zeros((t, y.shape[1]))
    for j in range(k):
        out += w[:, j:j + 1] * y[pos[np.arange(t) * k + j]]
    return out
