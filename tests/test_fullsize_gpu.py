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


def test_full_size_decode_1024_steps(D, cuda_ok):
    # Workload 5 as specified: a 4096-token causal prefill of the whole batch
    # (B64 H8 d64 m256) followed by 1024 single-token decode steps of the whole
    # batch through the C ABI. Every step's output on sampled heads is compared
    # with the oracle's decode recurrence continued from its own prefill state
    # (README, "Encoder-decoder model and generation": update, then emit), and
    # the final fp32 state (kv, z) with the oracle's, relative to its largest
    # entry, so that drift of the carried state over 1024 updates is checked.
    w = synth.WORKLOADS[5]
    steps = 1024
    inp = synth.make_inputs(w)
    res = forward(D, w, inp, cuda_ok, with_state=True)
    assert res["status"] == 0
    stream = synth.decode_stream(w, steps)
    sq, sk, sv = (to_dev(stream[nm], torch.bfloat16, cuda_ok) for nm in ("q", "k", "v"))
    outs = torch.empty_like(sq)
    status = torch.zeros(1, dtype=torch.int32, device=cuda_ok)
    for t in range(steps):
        D.dark_decode_step(res["proj"], res["state"], sq[t], sk[t], sv[t], outs[t],
                           dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    got = outs.double().cpu().numpy()                        # [steps, B, H, d]
    assert np.all(np.isfinite(got))
    kv_end = res["state_tensors"][0].double().cpu().numpy()
    z_end = res["state_tensors"][1].double().cpu().numpy()
    rng = np.random.default_rng(55)
    bh = [(b, h) for b in range(w.B) for h in range(w.H)]
    heads = [bh[i] for i in sorted(set([0, len(bh) - 1] + rng.integers(0, len(bh), 2).tolist()))]
    for (b, h) in heads:
        gm = inp["geom"][h:h + 1]
        phk = O.feature_map(inp["k"][b, h], inp["omega"][0], inp["geom"][h])
        kv = (phk.T @ inp["v"][b, h].astype(np.float64))[None, None]
        z = phk.sum(axis=0)[None, None]
        worst = 0.0
        for t in range(steps):
            sl = (slice(b, b + 1), slice(h, h + 1))
            ro, kv, z = O.decode_step(kv, z, stream["q"][t][sl], stream["k"][t][sl],
                                      stream["v"][t][sl], inp["omega"], gm)
            worst = max(worst, float(np.abs(got[t, b, h] - ro[0, 0]).max()))
        assert worst <= TOL_BF16, (b, h, worst)
        # the same bar as the prefill state above (bf16 feature operands)
        assert np.abs(kv_end[b, h] - kv[0, 0]).max() <= TOL_BF16 * np.abs(kv).max(), (b, h)
        assert np.abs(z_end[b, h] - z[0, 0]).max() <= TOL_BF16 * np.abs(z).max(), (b, h)
