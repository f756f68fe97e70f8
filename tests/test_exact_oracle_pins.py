"""Pins of the oracle's exact learned-kernel attention (README, "Attention modes")
against an independent softmax-attention routine (torch fp64 scaled dot-product
attention), an invariance of the kernel and the random-feature estimator's limit."""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import dark_oracle as O


def _inputs(seed, B=2, H=2, L=9, d=8, r=6):
    rng = np.random.default_rng(seed)
    q, k, v = (rng.standard_normal((B, H, L, d)) for _ in range(3))
    geom = np.eye(r, d)[None] + 0.3 * rng.standard_normal((H, r, d))
    return q, k, v, geom


@pytest.mark.parametrize("causal", [False, True])
def test_matches_torch_sdpa_on_projected_tokens(causal):
    q, k, v, gm = _inputs(1)
    mask = np.array([[1, 1, 0, 1, 1, 1, 0, 1, 1], [0, 1, 1, 1, 1, 0, 1, 1, 1]], np.uint8)
    got = O.exact_attention(q, k, v, gm, key_mask=mask, causal=causal)
    B, H, L, d = q.shape
    s = d ** -0.25
    tq, tk, tv = (torch.tensor(x) for x in (q, k, v))
    tg = torch.tensor(gm)
    u = torch.einsum("bhld,hrd->bhlr", tq * s, tg)
    w = torch.einsum("bhld,hrd->bhlr", tk * s, tg)
    keep = torch.tensor(mask != 0)[:, None, None, :].expand(B, H, L, L)
    if causal:
        keep = keep & torch.ones(L, L, dtype=torch.bool).tril()
    ref = F.scaled_dot_product_attention(u, w, tv, attn_mask=keep, scale=1.0).numpy()
    seen = keep.any(-1).numpy()
    assert np.abs(got[seen] - ref[seen]).max() <= 1e-12
    assert np.all(got[~seen] == 0.0)


def test_identity_geometry_is_standard_attention():
    q, k, v, _ = _inputs(2, r=8)
    eye = np.eye(8)[None]
    got = O.exact_attention(q, k, v, eye)
    ref = F.scaled_dot_product_attention(*(torch.tensor(x) for x in (q, k, v))).numpy()
    assert np.abs(got - ref).max() <= 1e-12


def test_invariant_to_rotating_the_geometry():
    q, k, v, gm = _inputs(3)
    u, _ = np.linalg.qr(np.random.default_rng(4).standard_normal((6, 6)))
    a = O.exact_attention(q, k, v, gm, causal=True)
    b = O.exact_attention(q, k, v, np.einsum("ij,hjd->hid", u, gm), causal=True)
    assert np.abs(a - b).max() <= 1e-12


def test_random_features_converge_to_the_exact_kernel():
    q, k, v, gm = _inputs(5, B=1, H=1, L=6, d=4, r=4)
    q, k = 0.5 * q, 0.5 * k
    ref = O.exact_attention(q, k, v, gm)
    errs = []
    for m in (256, 65536):
        om = np.random.default_rng(6).standard_normal((1, m, 4))
        est, _, _ = O.attention(q, k, v, om, gm)
        errs.append(np.abs(est - ref).max())
    assert errs[1] < 0.05 and errs[1] < errs[0] / 4


def test_cross_form_and_query_mask():
    # queries over a separate context: equal to the self-attention form when the
    # context is the same tokens; a masked query row is zero, the rest unchanged
    q, k, v, gm = _inputs(7)
    mask = np.array([[1, 1, 0, 1, 1, 1, 1, 1, 0], [1] * 9], np.uint8)
    a = O.exact_attention(q, k, v, gm, key_mask=mask)
    qm = np.array([[1, 0, 1, 1, 1, 1, 1, 1, 1], [1, 1, 1, 0, 0, 1, 1, 1, 1]], np.uint8)
    b = O.exact_attention(q, k, v, gm, key_mask=mask, query_mask=qm)
    dead = np.broadcast_to((qm == 0)[:, None, :, None], a.shape)
    assert np.all(b[dead] == 0.0) and np.array_equal(a[~dead], b[~dead])
    # a longer context: rows against torch SDPA with the key mask as attn_mask
    rng = np.random.default_rng(8)
    k2, v2 = rng.standard_normal((2, 2, 13, 8)), rng.standard_normal((2, 2, 13, 8))
    cm = np.ones((2, 13), np.uint8)
    cm[0, 4:7] = 0
    got = O.exact_attention(q, k2, v2, gm, key_mask=cm)
    s = 8 ** -0.25
    tg = torch.tensor(gm)
    u = torch.einsum("bhld,hrd->bhlr", torch.tensor(q) * s, tg)
    w = torch.einsum("bhld,hrd->bhlr", torch.tensor(k2) * s, tg)
    keep = torch.tensor(cm != 0)[:, None, None, :].expand(2, 2, 9, 13)
    ref = F.scaled_dot_product_attention(u, w, torch.tensor(v2), attn_mask=keep, scale=1.0)
    assert np.abs(got - ref.numpy()).max() <= 1e-12


def test_auto_policy():
    assert O.uses_exact(1024, 1024) and not O.uses_exact(1025, 1024)
    assert not O.uses_exact(16, 0)
