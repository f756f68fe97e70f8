"""Full-size parity: every workload at its full size, through the same C-ABI
call bench.py times, checked on sampled output rows against the oracle's
one-row definition, plus a property that holds at any size (every output lies
within the per-column range of the visible valid values, since the weights are
positive and normalised)."""
import numpy as np
import pytest
import torch

from oracle import dark_oracle as O
from random_feature_linear_b200 import synth

from gpu_run import forward, to_dev

pytestmark = pytest.mark.gpu
TOL_BF16 = 2e-2


@pytest.fixture(scope="module")
def D(cuda_ok):
    from random_feature_linear_b200 import dark
    return dark


def _sample_rows(L, valid_len, rng, n=6):
    rows = {0, 1, L - 1, max(0, valid_len - 1), min(L - 1, valid_len)}
    rows |= set(rng.integers(0, L, n).tolist())
    return sorted(r for r in rows if 0 <= r < L)


def _check_rows(w, inp, got, heads, rng):
    worst = 0.0
    for (b, h) in heads:
        vl = w.L if w.lengths is None else w.lengths[b]
        rows = _sample_rows(w.L, vl, rng)
        ref = O.attention_rows(inp["q"], inp["k"], inp["v"], inp["omega"], inp["geom"],
                               inp["mask"], w.causal, b, h, rows)
        worst = max(worst, float(np.abs(got[b, h, rows] - ref).max()))
    return worst


def _check_convex(w, inp, got):
    """Causal: running min/max of the valid values up to each row; non-causal: over all."""
    v = inp["v"].astype(np.float32)
    got = got.astype(np.float32)
    mask = np.ones((w.B, w.L), bool) if inp["mask"] is None else inp["mask"] != 0
    big = np.where(mask[:, None, :, None], v, np.inf)
    small = np.where(mask[:, None, :, None], v, -np.inf)
    if w.causal:
        lo = np.minimum.accumulate(big, axis=2)
        hi = np.maximum.accumulate(small, axis=2)
    else:
        lo = np.broadcast_to(big.min(axis=2, keepdims=True), v.shape)
        hi = np.broadcast_to(small.max(axis=2, keepdims=True), v.shape)
    has = np.isfinite(lo)
    assert np.all(got[~has] == 0)
    assert np.all(got[has] >= lo[has] - TOL_BF16) and np.all(got[has] <= hi[has] + TOL_BF16)


@pytest.mark.parametrize("cfg", [2, 3, 4, 5])
def test_full_size_forward(D, cuda_ok, cfg):
    w = synth.WORKLOADS[cfg]
    inp = synth.make_inputs(w)
    res = forward(D, w, inp, cuda_ok, with_state=(cfg == 5))
    assert res["status"] == 0
    got = res["out"]
    assert np.all(np.isfinite(got))
    rng = np.random.default_rng(cfg)
    bh = [(b, h) for b in range(w.B) for h in range(w.H)]
    heads = [bh[i] for i in sorted(set([0, len(bh) - 1] + rng.integers(0, len(bh), 2).tolist()))]
    err = _check_rows(w, inp, got, heads, rng)
    assert err <= TOL_BF16, err
    _check_convex(w, inp, got)
    if cfg == 5:
        # prefill state of sampled heads: Phi(K)^T V and Phi(K)^T 1 over all keys
        for (b, h) in heads:
            phk = O.feature_map(inp["k"][b, h], inp["omega"][0], inp["geom"][h])
            kv = phk.T @ inp["v"][b, h].astype(np.float64)
            z = phk.sum(axis=0)
            assert np.abs(res["kv"][b, h] - kv).max() <= TOL_BF16 * np.abs(kv).max()
            assert np.abs(res["z"][b, h] - z).max() <= TOL_BF16 * np.abs(z).max()
        # two decode steps on the full batch, checked on the sampled heads
        stream = synth.decode_stream(w, 2)
        kvs = {hd: None for hd in heads}
        for t in range(2):
            q, k, v = (to_dev(stream[nm][t], torch.bfloat16, cuda_ok) for nm in ("q", "k", "v"))
            out = torch.empty_like(q)
            D.dark_decode_step(res["proj"], res["state"], q, k, v, out)
            torch.cuda.synchronize()
            o = out.double().cpu().numpy()
            for (b, h) in heads:
                if kvs[(b, h)] is None:
                    phk = O.feature_map(inp["k"][b, h], inp["omega"][0], inp["geom"][h])
                    kvs[(b, h)] = (phk.T @ inp["v"][b, h].astype(np.float64), phk.sum(axis=0))
                kv, z = kvs[(b, h)]
                ro, kv2, z2 = O.decode_step(kv[None, None], z[None, None], stream["q"][t][b:b + 1, h:h + 1],
                                            stream["k"][t][b:b + 1, h:h + 1], stream["v"][t][b:b + 1, h:h + 1],
                                            inp["omega"], inp["geom"][h:h + 1])
                kvs[(b, h)] = (kv2[0, 0], z2[0, 0])
                assert np.abs(o[b, h] - ro[0, 0]).max() <= TOL_BF16
