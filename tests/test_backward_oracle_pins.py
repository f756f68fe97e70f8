"""Pins of the oracle's backward pass (gradients of PRF attention with respect to
q, k, v and the geometry M; README, "Kernel": M is learned) against what the
mathematics fixes, independently of the oracle's own chain rule:

* central finite differences of the pinned forward, entry by entry;
* reverse-mode autograd (torch, fp64) over a different formulation of the same
  function: the explicit L x L matrix of kernel estimates, row-normalised;
* closed forms: dv = A^T dout with A the row-normalised matrix of kernel
  estimates; one token gives dv = dout and no other gradient;
* invariants: shared geometry collects the per-head gradients, a batch row with
  no valid key has zero gradients.
"""
import numpy as np
import pytest
import torch

from oracle import dark_oracle as O


def _inputs(seed, B=2, H=2, L=7, d=4, r=3, m=5, heads_geom=2, heads_omega=1):
    rng = np.random.default_rng(seed)
    q = 0.8 * rng.standard_normal((B, H, L, d))
    k = 0.8 * rng.standard_normal((B, H, L, d))
    v = rng.standard_normal((B, H, L, d))
    g = rng.standard_normal((B, H, L, d))
    omega = rng.standard_normal((heads_omega, m, r))
    geom = np.eye(r, d)[None] + 0.3 * rng.standard_normal((heads_geom, r, d))
    return q, k, v, omega, geom, g


def _loss(q, k, v, omega, geom, g, mask, causal):
    out, _, _ = O.attention(q, k, v, omega, geom, key_mask=mask, causal=causal)
    return float((out * g).sum())


def _fd(f, x, eps=1e-6):
    grad = np.zeros_like(x)
    it = np.nditer(x, flags=["multi_index"])
    for _ in it:
        i = it.multi_index
        x0 = x[i]
        x[i] = x0 + eps
        fp = f()
        x[i] = x0 - eps
        fm = f()
        x[i] = x0
        grad[i] = (fp - fm) / (2 * eps)
    return grad


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("heads", [(1, 2), (2, 1), (2, 2)])
def test_gradients_match_finite_differences(causal, heads):
    ho, hg = heads
    q, k, v, om, gm, g = _inputs(10 + ho + 3 * hg + causal, heads_geom=hg, heads_omega=ho)
    mask = np.array([[1, 1, 0, 1, 1, 1, 1], [0, 1, 1, 1, 0, 1, 1]], np.uint8)
    dq, dk, dv, dgm = O.attention_backward(q, k, v, om, gm, g, key_mask=mask, causal=causal)

    def f():
        return _loss(q, k, v, om, gm, g, mask, causal)

    for got, x in ((dq, q), (dk, k), (dv, v), (dgm, gm)):
        ref = _fd(f, x)
        assert np.abs(got - ref).max() <= 1e-6 * max(1.0, np.abs(ref).max()), np.abs(got - ref).max()


def _torch_quadratic(q, k, v, omega, geom, mask, causal):
    """out_i = sum_j K_ij v_j / sum_j K_ij with K_ij = phi(q_i) . phi(k_j) over the
    valid keys (and j <= i when causal): the L x L form, in torch fp64."""
    B, H, L, d = q.shape
    s = d ** -0.25
    outs = []
    for b in range(B):
        rows = []
        for h in range(H):
            om = omega[0] if omega.shape[0] == 1 else omega[h]
            gm = geom[0] if geom.shape[0] == 1 else geom[h]

            def phi(x):
                u = (x * s) @ gm.T
                return torch.exp(u @ om.T - 0.5 * (u * u).sum(-1, keepdim=True)) / om.shape[0] ** 0.5

            kmat = phi(q[b, h]) @ phi(k[b, h]).T
            keep = torch.as_tensor(mask[b] != 0)[None, :].expand(L, L)
            if causal:
                keep = keep & torch.ones(L, L, dtype=torch.bool).tril()
            kmat = torch.where(keep, kmat, torch.zeros_like(kmat))
            den = kmat.sum(-1, keepdim=True)
            rows.append(torch.where(den > 0, (kmat @ v[b, h]) / torch.where(den > 0, den, 1.0),
                                    torch.zeros_like(q[b, h])))
        outs.append(torch.stack(rows))
    return torch.stack(outs)


@pytest.mark.parametrize("causal", [False, True])
def test_gradients_match_autograd_of_the_quadratic_form(causal):
    q, k, v, om, gm, g = _inputs(3, B=2, H=3, L=40, d=8, r=8, m=16, heads_geom=3, heads_omega=3)
    mask = np.ones((2, 40), np.uint8)
    mask[1, 25:] = 0
    mask[0, 0] = 0
    tq, tk, tv, tgm = (torch.tensor(x, requires_grad=True) for x in (q, k, v, gm))
    out = _torch_quadratic(tq, tk, tv, torch.tensor(om), tgm, mask, causal)
    (out * torch.tensor(g)).sum().backward()
    dq, dk, dv, dgm = O.attention_backward(q, k, v, om, gm, g, key_mask=mask, causal=causal)
    for got, ref in ((dq, tq.grad), (dk, tk.grad), (dv, tv.grad), (dgm, tgm.grad)):
        ref = ref.numpy()
        assert np.abs(got - ref).max() <= 1e-10 * np.abs(ref).max()


def test_shared_geometry_collects_the_per_head_gradients():
    q, k, v, om, gm, g = _inputs(4, H=3, heads_geom=1)
    per_head = np.repeat(gm, 3, axis=0)
    _, _, _, shared = O.attention_backward(q, k, v, om, gm, g, causal=True)
    _, _, _, split = O.attention_backward(q, k, v, om, per_head, g, causal=True)
    assert np.abs(shared[0] - split.sum(axis=0)).max() <= 1e-12 * np.abs(shared).max()


def test_rows_without_visible_keys_have_zero_gradients():
    q, k, v, om, gm, g = _inputs(5)
    mask = np.array([[0, 0, 0, 0, 0, 0, 0], [0, 0, 1, 1, 1, 1, 1]], np.uint8)
    dq, dk, dv, _ = O.attention_backward(q, k, v, om, gm, g, key_mask=mask, causal=True)
    assert np.all(dq[0] == 0) and np.all(dk[0] == 0) and np.all(dv[0] == 0)
    # causal: queries before the first valid key see nothing; masked keys get nothing
    assert np.all(dq[1, :, :2] == 0)
    assert np.all(dk[1, :, :2] == 0) and np.all(dv[1, :, :2] == 0)
    assert np.abs(dq[1, :, 2:]).max() > 0


@pytest.mark.parametrize("causal", [False, True])
def test_value_gradient_is_the_transposed_attention_matrix(causal):
    # out = A v with A the row-normalised matrix of kernel estimates over the
    # visible keys, so dv = A^T dout exactly (a closed form, from the L x L matrix)
    q, k, v, om, gm, g = _inputs(11, L=12, heads_geom=2, heads_omega=1)
    mask = np.ones((2, 12), np.uint8)
    mask[1, [2, 7]] = 0
    _, _, dv, _ = O.attention_backward(q, k, v, om, gm, g, key_mask=mask, causal=causal)
    for b in range(2):
        for h in range(2):
            phq = O.feature_map(q[b, h], om[0], gm[h])
            phk = O.feature_map(k[b, h], om[0], gm[h])
            kmat = phq @ phk.T
            kmat[:, mask[b] == 0] = 0.0
            if causal:
                kmat = np.tril(kmat)
            a = kmat / kmat.sum(axis=1, keepdims=True)
            ref = a.T @ g[b, h]
            assert np.abs(dv[b, h] - ref).max() <= 1e-12 * np.abs(ref).max()


def test_single_token_closed_form():
    # one token: out = v exactly, so dv = dout and every other gradient is zero
    q, k, v, om, gm, g = _inputs(12, L=1)
    dq, dk, dv, dgm = O.attention_backward(q, k, v, om, gm, g, causal=True)
    assert np.abs(dv - g).max() <= 1e-12
    scale = np.abs(g).max()
    for x in (dq, dk, dgm):
        assert np.abs(x).max() <= 1e-12 * scale
