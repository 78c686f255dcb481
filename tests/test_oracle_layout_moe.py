"""Pins for the oracle's packed-layout formulas and MoE routing."""

import itertools

import numpy as np

from oracle import formats as F
from oracle import layout as L
from oracle import moe as R
from quantized_gemm_bit_b200 import synth


def test_w4a16_layout_is_a_bijection():
    for n, k, asym in ((128, 256, False), (200, 384, True)):
        nn, kk = np.meshgrid(np.arange(n), np.arange(k), indexing="ij")
        byte, nib = L.w4a16_code_byte_and_nibble(nn.ravel(), kk.ravel(), k, asym)
        slot = byte * 2 + nib
        assert len(np.unique(slot)) == n * k
        total = L.w4a16_packed_bytes(n, k, asym)
        assert slot.max() < 2 * total
        # codes, scales and zeros never overlap
        ng, gg = np.meshgrid(np.arange(n), np.arange(k // 128), indexing="ij")
        sb = L.w4a16_scale_byte(ng.ravel(), gg.ravel(), k, asym)
        used = set(byte.tolist())
        assert not (used & set(sb.tolist())) and not (used & set((sb + 1).tolist()))
        if asym:
            zb = L.w4a16_zero_byte(ng.ravel(), gg.ravel(), k)
            assert not (used & set(zb.tolist())) and not (set(zb.tolist()) & set(sb.tolist()))


def test_w4a16_pack_unpack_roundtrip():
    for asym in (False, True):
        q, s, z = synth.w4a16_weights(136, 256, 128, asym, seed=51)
        blob = L.w4a16_pack(q.numpy(), s.numpy(), None if z is None else z.numpy())
        assert blob.size == L.w4a16_packed_bytes(136, 256, asym)
        codes, s2, z2 = L.w4a16_unpack(blob, 136, 256, asym)
        assert np.array_equal(codes, F.int4_unpack_words(q.numpy()))
        assert np.array_equal(s2.view(np.uint16), s.numpy().view(np.uint16))
        if asym:
            assert np.array_equal(z2, z.numpy())
        # padding rows 136..255 of the second tile stay zero
        nt_bytes = 2 * L.w4a16_record_bytes(asym)
        rec = L.w4a16_record_bytes(asym)
        tile1 = blob[nt_bytes:].reshape(2, rec)
        codes1 = tile1[:, :8192].reshape(2, 4, 128, 16)
        assert np.all(codes1[:, :, 8:, :] == 0)


def test_w4a16_layout_small_hand_example():
    """Code q[n=1, k=3] (chunk 0, word 0, element 3 -> nibble 5) lands at
    byte (0*128 + 1)*16 + 0*4 + 2, high nibble; q[0, 33] (chunk 1, word 0,
    element 1 -> nibble 4) at byte (1*128 + 0)*16 + 2, low nibble."""
    b, nib = L.w4a16_code_byte_and_nibble(1, 3, 128, False)
    assert (int(b), int(nib)) == (18, 1)
    b, nib = L.w4a16_code_byte_and_nibble(0, 33, 128, False)
    assert (int(b), int(nib)) == (2050, 0)


def test_topk_by_logit_brute_force():
    rng = np.random.default_rng(61)
    logits = rng.standard_normal((40, 8)).astype(np.float32)
    logits[3, 2] = logits[3, 5]                          # a tie
    ids = R.topk_by_logit(logits, 3)
    for t in range(40):
        ranked = sorted(range(8), key=lambda e: (-float(logits[t, e]), e))
        assert list(ids[t]) == ranked[:3]


def test_topk_set_invariants_full_size():
    logits = synth.router_logits(64, 256, seed=3001).numpy()
    ids = R.topk_by_logit(logits, 8)
    for t in range(64):
        sel = set(ids[t].tolist())
        assert len(sel) == 8
        rest = [e for e in range(256) if e not in sel]
        assert logits[t, list(sel)].min() >= logits[t, rest].max()


def test_permute_invariants_and_brute_force():
    rng = np.random.default_rng(62)
    for t, e, k in ((5, 8, 2), (33, 16, 4), (64, 256, 8)):
        logits = rng.standard_normal((t, e)).astype(np.float32)
        ids = R.topk_by_logit(logits, k)
        counts, off, src = R.permute(ids, e)
        assert off[0] == 0 and off[-1] == t * k and np.all(np.diff(off) == counts)
        assert sorted(src.tolist()) == list(range(t * k))
        flat = ids.ravel()
        for ex in range(e):
            seg = src[off[ex]:off[ex + 1]]
            assert np.all(flat[seg] == ex)
            assert np.all(np.diff(seg // k) > 0)          # token strictly increasing
        # brute force: sort all (expert, slot) pairs
        pairs = sorted((int(flat[s]), s) for s in range(t * k))
        assert [p[1] for p in pairs] == src.tolist()


def test_permute_handles_empty_experts_and_duplicates():
    ids = np.array([[3, 3], [0, 3]], dtype=np.int32)      # duplicates allowed
    counts, off, src = R.permute(ids, 5)
    assert counts.tolist() == [1, 0, 0, 3, 0]
    assert off.tolist() == [0, 1, 1, 1, 4, 4]
    assert src.tolist() == [2, 0, 1, 3]


def test_gather_rows():
    a = np.arange(12, dtype=np.uint16).reshape(4, 3)
    src = np.array([5, 0, 7, 2], dtype=np.int32)
    out = R.gather_rows(a, src, 2)
    assert np.array_equal(out, a[[2, 0, 3, 1]])


def test_synth_distributions():
    q, s, z = synth.w4a16_weights(256, 1024, 128, True, seed=0)
    codes = F.int4_unpack_words(q.numpy())
    hist = np.bincount(codes.ravel(), minlength=16) / codes.size
    assert np.all(np.abs(hist - 1 / 16) < 0.005)
    sv = s.numpy().astype(np.float64)
    assert sv.min() >= 0.002 - 1e-6 and abs(sv.mean() - (0.002 + 0.01 * np.sqrt(2 / np.pi))) < 5e-4
    assert z.numpy().max() == 15 and z.numpy().min() == 0
    codes, e8 = synth.mxfp4_weights(64, 1024, seed=2)
    assert set(np.unique(e8.numpy()).tolist()) == set(range(119, 126))
    assert list(itertools.islice(range(3), 1)) == [0]


# ---------------------------------------------------------------- MoE layer: SwiGLU and combine

def _bf16(x):
    return F.f32_to_bf16_bits_rne(np.asarray(x, dtype=np.float32))


def test_silu_mul_against_logistic_function_and_identities():
    """silu(g) * u against scipy's logistic function (a routine the oracle
    does not call), the identity silu(x) - silu(-x) = x, silu(0) = 0, the
    tails silu(x) -> x and silu(-x) -> -0, and the column split (gate first)."""
    from scipy.special import expit
    rng = np.random.default_rng(5)
    g = rng.normal(0, 4, (6, 8))
    u = rng.normal(0, 1, (6, 8))
    x = np.concatenate([_bf16(g), _bf16(u)], axis=1)
    gb, ub = F.bf16_bits_to_f64(x[:, :8]), F.bf16_bits_to_f64(x[:, 8:])
    h = R.silu_mul(x, 8)
    assert np.allclose(h, gb * expit(gb) * ub, rtol=1e-14, atol=0)
    ones = np.concatenate([x[:, :8], _bf16(np.ones((6, 8)))], axis=1)
    neg = np.concatenate([_bf16(-gb), _bf16(np.ones((6, 8)))], axis=1)
    assert np.allclose(R.silu_mul(ones, 8) - R.silu_mul(neg, 8), gb, rtol=0, atol=1e-12)
    edge = np.concatenate([_bf16([[0.0, 200.0, -200.0, 1.0]]), _bf16([[3.0, 1.0, 1.0, 0.0]])], axis=1)
    he = R.silu_mul(edge, 4)[0]
    assert he[0] == 0.0 and he[1] == 200.0 and -1e-80 < he[2] <= 0.0 and he[3] == 0.0
    # the gate is the first half: swapping the halves changes the result
    swapped = np.concatenate([x[:, 8:], x[:, :8]], axis=1)
    assert not np.allclose(R.silu_mul(swapped, 8), h)


def _combine_brute(y_bits, src, w, k):
    y = F.bf16_bits_to_f64(y_bits)
    t = len(src) // k
    out = [[0.0] * y.shape[1] for _ in range(t)]
    for p, slot in enumerate(src):
        tok, j = divmod(int(slot), k)
        for c in range(y.shape[1]):
            out[tok][c] += float(w[tok][j]) * y[p][c]
    return np.array(out)


def test_combine_brute_force_one_hot_and_linearity():
    rng = np.random.default_rng(6)
    t, e, k, h = 7, 9, 3, 5
    ids = R.topk_by_logit(rng.normal(size=(t, e)).astype(np.float32), k)
    _, _, src = R.permute(ids, e)
    y = _bf16(rng.normal(size=(t * k, h)))
    w = rng.random((t, k)).astype(np.float32)
    out = R.combine(y, src, w, k)
    assert np.allclose(out, _combine_brute(y, src, w, k), rtol=1e-15, atol=1e-15)
    # one-hot weights pick slot j of each token, un-permuted
    for j in range(k):
        oh = np.zeros((t, k), dtype=np.float32)
        oh[:, j] = 1.0
        pos = {int(s): p for p, s in enumerate(src)}
        want = F.bf16_bits_to_f64(y[[pos[tok * k + j] for tok in range(t)]])
        assert np.array_equal(R.combine(y, src, oh, k), want)
    w2 = rng.random((t, k)).astype(np.float32)
    wsum = w.astype(np.float64) + w2.astype(np.float64)
    assert np.allclose(R.combine(y, src, wsum, k), out + R.combine(y, src, w2, k), rtol=1e-12, atol=1e-12)


def test_softmax_topk_weights_properties():
    """Over all experts the probabilities sum to 1; ratios are exp of logit
    differences; the selected ones are the k largest, in slot order."""
    rng = np.random.default_rng(7)
    logits = rng.normal(size=(5, 16)).astype(np.float32)
    all_ids = np.tile(np.arange(16), (5, 1))
    assert np.allclose(R.softmax_topk_weights(logits, all_ids).sum(axis=1), 1.0, rtol=1e-14)
    ids = R.topk_by_logit(logits, 4)
    w = R.softmax_topk_weights(logits, ids)
    l64 = logits.astype(np.float64)
    for tkn in range(5):
        for a, b in itertools.combinations(range(4), 2):
            ratio = np.exp(l64[tkn, ids[tkn, a]] - l64[tkn, ids[tkn, b]])
            assert np.isclose(w[tkn, a] / w[tkn, b], ratio, rtol=1e-12)
        assert np.all(np.diff(w[tkn]) <= 0)
    assert np.all(w.sum(axis=1) < 1.0)       # not renormalised over the k selected


def test_silu_mul_f64_matches_the_bf16_form_and_the_logistic_function():
    """The unrounded SwiGLU (for the fused epilogue) is the same function:
    on bf16-representable inputs it equals silu_mul exactly, and on any
    inputs g * expit(g) * u (scipy)."""
    from scipy.special import expit
    rng = np.random.default_rng(8)
    g = rng.normal(0, 3, (5, 16))
    u = rng.normal(0, 1, (5, 16))
    x = np.concatenate([_bf16(g), _bf16(u)], axis=1)
    assert np.array_equal(R.silu_mul_f64(F.bf16_bits_to_f64(x), 16), R.silu_mul(x, 16))
    h = R.silu_mul_f64(np.concatenate([g, u], axis=1), 16)
    assert np.allclose(h, g * expit(g) * u, rtol=1e-14, atol=0)


def test_gated_row_order_hand_example_and_bijection():
    """Packed row p of the gated order: gate rows in lanes 0-15 of every
    32-row quarter, the up rows of the same features in lanes 16-31."""
    src = L.gated_source_rows(256)            # I = 128
    assert src[0] == 0 and src[15] == 15      # tile 0, quarter 0: gate 0..15
    assert src[16] == 128 and src[31] == 143  # ... then up 0..15
    assert src[32] == 16 and src[48] == 144   # quarter 1: features 16..31
    assert src[127] == 128 + 63               # tile 0 ends with up feature 63
    assert src[128] == 64 and src[144] == 192  # tile 1: features 64..127
    assert np.array_equal(np.sort(src), np.arange(256))
    big = L.gated_source_rows(4096)
    assert np.array_equal(np.sort(big), np.arange(4096))
    # every tile covers 64 gate features and the same 64 up features
    for j in range(4096 // 128):
        t = big[128 * j:128 * (j + 1)]
        assert np.array_equal(np.sort(t[t < 2048]), np.arange(64 * j, 64 * j + 64))
        assert np.array_equal(np.sort(t[t >= 2048]) - 2048, np.arange(64 * j, 64 * j + 64))
