"""Pins of the oracle's cross-attention (README, "Cross-attention" and
"Encoder-decoder model and generation") against what the pages and the
mathematics fix, independently of the cross-attention code itself."""
import numpy as np

from oracle import dark_oracle as O


def _inputs(seed, B=2, H=2, Lq=6, Lk=9, d=8, r=8, m=32):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, H, Lq, d))
    k = rng.standard_normal((B, H, Lk, d))
    v = rng.standard_normal((B, H, Lk, d))
    omega = rng.standard_normal((1, m, r))
    geom = np.eye(r, d)[None] + 0.1 * rng.standard_normal((H, r, d))
    return q, k, v, omega, geom


def test_equals_noncausal_self_attention_form():
    # same number of queries and keys: the pairwise cross-attention sums equal
    # the associative non-causal form Phi(Q) (Phi(K)^T V) / Phi(Q) (Phi(K)^T 1)
    q, k, v, om, gm = _inputs(1, Lq=7, Lk=7)
    mask = np.array([[1, 1, 0, 1, 1, 1, 0], [1, 0, 1, 1, 1, 1, 1]], np.uint8)
    got, kv, z = O.cross_attention(q, k, v, om, gm, context_mask=mask)
    ref, kv_r, z_r = O.attention(q, k, v, om, gm, key_mask=mask, causal=False)
    assert np.abs(got - ref).max() <= 1e-12 * np.abs(ref).max()
    assert np.abs(kv - kv_r).max() <= 1e-12 * np.abs(kv_r).max()
    assert np.abs(z - z_r).max() <= 1e-12 * np.abs(z_r).max()


def test_context_permutation_invariance():
    q, k, v, om, gm = _inputs(2)
    mask = np.array([[1, 1, 1, 0, 1, 1, 0, 1, 1], [1] * 9], np.uint8)
    perm = np.random.default_rng(3).permutation(k.shape[2])
    a, _, _ = O.cross_attention(q, k, v, om, gm, context_mask=mask)
    b, _, _ = O.cross_attention(q, k[:, :, perm], v[:, :, perm], om, gm, context_mask=mask[:, perm])
    assert np.abs(a - b).max() <= 1e-12 * np.abs(a).max()


def test_masked_context_positions_do_not_matter():
    q, k, v, om, gm = _inputs(4)
    mask = np.array([[1, 0, 1, 1, 0, 1, 1, 1, 1], [0, 1, 1, 1, 1, 1, 1, 1, 0]], np.uint8)
    a, _, _ = O.cross_attention(q, k, v, om, gm, context_mask=mask)
    k2, v2 = k.copy(), v.copy()
    k2[mask[:, None, :].repeat(2, 1) == 0] = 50.0
    v2[mask[:, None, :].repeat(2, 1) == 0] = -7.0
    b, _, _ = O.cross_attention(q, k2, v2, om, gm, context_mask=mask)
    assert np.abs(a - b).max() == 0.0


def test_query_mask_zeroes_rows_and_keeps_the_rest():
    q, k, v, om, gm = _inputs(5)
    qm = np.array([[1, 0, 1, 1, 1, 0], [1, 1, 1, 1, 1, 1]], np.uint8)
    a, _, _ = O.cross_attention(q, k, v, om, gm)
    b, _, _ = O.cross_attention(q, k, v, om, gm, query_mask=qm)
    dead = qm[:, None, :, None].repeat(2, 1) == 0
    assert np.all(b[np.broadcast_to(dead, b.shape)] == 0.0)
    assert np.abs(a - b)[~np.broadcast_to(dead, b.shape)].max() == 0.0


def test_outputs_are_convex_combinations_of_valid_context_values():
    q, k, v, om, gm = _inputs(6, Lk=11)
    mask = np.ones((2, 11), np.uint8)
    mask[0, 3:7] = 0
    out, _, _ = O.cross_attention(q, k, v, om, gm, context_mask=mask)
    for b in range(2):
        sel = mask[b] != 0
        lo = v[b][:, sel].min(axis=1)
        hi = v[b][:, sel].max(axis=1)
        assert np.all(out[b] >= lo[:, None, :] - 1e-12)
        assert np.all(out[b] <= hi[:, None, :] + 1e-12)


def test_decode_against_the_summary_equals_one_query_cross_attention():
    q, k, v, om, gm = _inputs(7, Lq=3)
    mask = np.array([[1, 1, 1, 1, 0, 1, 1, 1, 1], [1, 1, 0, 1, 1, 1, 1, 1, 1]], np.uint8)
    full, kv, z = O.cross_attention(q, k, v, om, gm, context_mask=mask)
    for i in range(3):
        step = O.cross_decode_step(kv, z, q[:, :, i], om, gm)
        assert np.abs(step - full[:, :, i]).max() <= 1e-12 * np.abs(full).max()
    # the summary is left as it was
    kv0, z0 = kv.copy(), z.copy()
    O.cross_decode_step(kv, z, q[:, :, 0], om, gm)
    assert np.array_equal(kv, kv0) and np.array_equal(z, z0)


def test_empty_context_gives_zero_rows():
    q, k, v, om, gm = _inputs(8)
    out, kv, z = O.cross_attention(q, k, v, om, gm, context_mask=np.zeros((2, 9), np.uint8))
    assert np.all(out == 0.0) and np.all(kv == 0.0) and np.all(z == 0.0)
