"""Parity of the CUDA forward path (through the C ABI) with the fp64 oracle."""
import numpy as np
import pytest
import torch

from oracle import dark_oracle as O
from random_feature_linear_b200 import synth

from gpu_run import check, forward

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def D(cuda_ok):
    from random_feature_linear_b200 import dark
    return dark


def _oracle(inp, causal):
    return O.attention(inp["q"], inp["k"], inp["v"], inp["omega"], inp["geom"],
                       key_mask=inp["mask"], causal=causal)


# Small versions of the five workload recipes: several 128-token tiles plus a
# ragged tail, so every tile kind and the tail path run.
SMALL = {
    "c1": synth.WORKLOADS[1],
    "c1-causal": synth.WORKLOADS[1].with_sizes(causal=True, L=300, B=2, H=2),
    "c1-masked": synth.WORKLOADS[1].with_sizes(L=200, B=2, lengths=(200, 77)),
    "c2": synth.WORKLOADS[2].with_sizes(H=2, L=300, lengths=(300, 217)),
    "c3": synth.WORKLOADS[3].with_sizes(H=3, L=700),
    "c4": synth.WORKLOADS[4].with_sizes(B=1, H=2, L=300),
    "c5-prefill": synth.WORKLOADS[5].with_sizes(B=3, H=2, L=333),
    "c2-noncausal": synth.WORKLOADS[2].with_sizes(H=2, L=260, lengths=(260, 131), causal=False),
    "c3-causal": synth.WORKLOADS[3].with_sizes(H=2, L=385, causal=True),
    # wide heads (two-launch tensor-core path): key mask, ragged tails, other d/m/r
    "c4-masked": synth.WORKLOADS[4].with_sizes(B=2, H=1, L=260, lengths=(260, 100)),
    "wide-d128-m256": synth.WORKLOADS[4].with_sizes(B=2, H=2, L=270, d=128, r=128, m=256,
                                                      lengths=(270, 150)),
    # other (m, r) instances of the d = 64 tensor-core kernels
    "c2-m128-r48": synth.WORKLOADS[2].with_sizes(H=2, L=300, lengths=(300, 211), m=128, r=48),
    "c3-m128-r16": synth.WORKLOADS[3].with_sizes(H=3, L=700, m=128, r=16),
    "c3-r64": synth.WORKLOADS[3].with_sizes(H=2, L=520, r=64),
    "c2-noncausal-r48": synth.WORKLOADS[2].with_sizes(H=2, L=390, lengths=(390, 260), r=48,
                                                      causal=False),
    "wide-d128-m128-shared": synth.WORKLOADS[4].with_sizes(B=1, H=3, L=140, d=128, r=64, m=128,
                                                             per_head_geom=False),
}


@pytest.mark.parametrize("name", list(SMALL))
def test_forward_matches_oracle(D, cuda_ok, name):
    w = SMALL[name]
    inp = synth.make_inputs(w)
    res = forward(D, w, inp, cuda_ok, with_state=True)
    assert res["status"] == 0
    out, kv, z = _oracle(inp, w.causal)
    check(w, res["out"], out)
    # state over all valid keys: relative to the largest entry of each head
    for got, ref in ((res["kv"], kv), (res["z"], z)):
        scale = np.abs(ref).reshape(ref.shape[0], ref.shape[1], -1).max(axis=2)
        err = np.abs(got - ref).reshape(scale.shape + (-1,)).max(axis=2) / scale
        assert err.max() <= (1e-4 if w.dtype == "f32" else 2e-2), err.max()


@pytest.mark.parametrize("recipe", ["c2", "wide-d128", "c3"])
def test_strided_inputs(D, cuda_ok, recipe):
    # q, k, v interleaved as [B][L][3][H][d] and out as [B][L][H][d]
    w = {"c2": synth.WORKLOADS[2].with_sizes(H=2, L=200, lengths=(200, 150)),
         "wide-d128": synth.WORKLOADS[4].with_sizes(B=2, H=2, L=150, d=128, r=128, m=256,
                                                    lengths=(150, 90)),
         "c3": synth.WORKLOADS[3].with_sizes(H=2, L=300)}[recipe]
    inp = synth.make_inputs(w)
    res = forward(D, w, inp, cuda_ok, strided=True)
    assert res["status"] == 0
    out, _, _ = _oracle(inp, w.causal)
    check(w, res["out"], out)


@pytest.mark.parametrize("name", ["c1-causal", "c2", "c3", "c4-masked", "wide-d128-m256",
                                  "wide-d128-m128-shared"])
def test_stabiliser_changes_nothing(D, cuda_ok, name):
    w = SMALL[name]
    inp = synth.make_inputs(w)
    flags = (D.DARK_CAUSAL if w.causal else 0) | D.DARK_STABILISE
    res = forward(D, w, inp, cuda_ok, flags=flags, with_state=True)
    assert res["status"] == 0
    out, kv, z = _oracle(inp, w.causal)
    check(w, res["out"], out)
    # the stabilised state is the true one times 2^{-shift}
    sc = np.exp2(-res["shift"])[:, :, None]
    zs = z * sc
    assert np.abs(res["z"] - zs).max() <= 2e-2 * np.abs(zs).max()


def _query_exponent_max(inp):
    """Largest base-2 query exponent max_j log2(e) (omega_j . M q~) over all
    heads and tokens (the oracle's feature exponent without the key terms)."""
    d = inp["q"].shape[-1]
    top = 0.0
    for h in range(inp["q"].shape[1]):
        wtop = np.log2(np.e) * d ** -0.25 * (inp["omega"][0].astype(np.float64)
                                             @ inp["geom"][h % inp["geom"].shape[0]]
                                             .astype(np.float64))
        qh = inp["q"][:, h].astype(np.float64).reshape(-1, d)
        top = max(top, float((qh @ wtop.T).max()))
    return top


@pytest.mark.parametrize("recipe", ["f32-causal", "bf16-causal", "bf16-noncausal",
                                    "bf16-wide-d256", "bf16-wide-d128"])
def test_stabiliser_avoids_overflow(D, cuda_ok, recipe):
    # Queries scaled so that their largest exponent is ~2^138 (by 6 for the
    # d = 64 recipes): that overflows fp32 unless the per-query constant is
    # subtracted (key exponents are bounded by |omega_j|^2 / 2 and stay in
    # range). Without the flag the device reports a non-finite output; with it
    # the result matches the oracle. fp32 runs the FFMA kernels, bf16 the
    # tensor-core kernels (d = 64, and the wide-head pair for d = 128, 256).
    w = {"f32-causal": synth.WORKLOADS[1].with_sizes(L=130, causal=True),
         "bf16-causal": synth.WORKLOADS[2].with_sizes(H=2, L=260, lengths=(260, 199)),
         "bf16-noncausal": synth.WORKLOADS[3].with_sizes(H=2, L=300),
         "bf16-wide-d256": synth.WORKLOADS[4].with_sizes(B=1, H=2, L=300, lengths=(300,)),
         "bf16-wide-d128": synth.WORKLOADS[4].with_sizes(B=2, H=2, L=270, d=128, r=128, m=256,
                                                          lengths=(270, 150))}[recipe]
    inp = synth.make_inputs(w)
    scale = 6.0 if w.d == 64 else 138.0 / _query_exponent_max(inp)
    q = inp["q"] * scale
    if w.dtype == "bf16":
        # the device reads bf16 tokens: give the oracle the same rounded values
        q = torch.from_numpy(q).to(torch.bfloat16).double().numpy()
    inp = dict(inp, q=q)
    causal = D.DARK_CAUSAL if w.causal else 0
    res = forward(D, w, inp, cuda_ok, flags=causal)
    assert res["status"] == D.DARK_ERR_NUMERIC
    res = forward(D, w, inp, cuda_ok, flags=causal | D.DARK_STABILISE)
    assert res["status"] == 0
    out, _, _ = _oracle(inp, w.causal)
    if w.dtype == "f32":
        check(w, res["out"], out)
    else:
        # bf16 tokens meet an fp16 W' (each entry within 2^-11 of itself), so
        # the base-2 query exponent j of token i moves by at most
        # 2^-11 sum_t |W'_jt q_it|: about 0.1 at these 2^138 exponents. A
        # convex mix whose feature weights move by the factor 2^(+-de) moves by
        # at most 2 ln2 de max|v|; that bound, over the usual 2e-2, is the
        # tolerance here.
        d = inp["q"].shape[-1]
        de = 0.0
        for h in range(w.H):
            wtop = np.log2(np.e) * d ** -0.25 * (inp["omega"][0].astype(np.float64)
                                                 @ inp["geom"][h % inp["geom"].shape[0]]
                                                 .astype(np.float64))
            qh = np.abs(inp["q"][:, h].astype(np.float64)).reshape(-1, d)
            de = max(de, 2.0 ** -11 * float((qh @ np.abs(wtop).T).max()))
        tol = 2e-2 + 2 * np.log(2) * de * float(np.abs(inp["v"]).max())
        assert np.all(np.isfinite(res["out"]))
        err = float(np.abs(res["out"] - out).max())
        assert err <= tol, (err, tol, de)


def test_rows_without_valid_keys_are_zero(D, cuda_ok):
    w = synth.WORKLOADS[2].with_sizes(H=2, L=257, lengths=(0, 3))
    inp = synth.make_inputs(w)
    res = forward(D, w, inp, cuda_ok)
    assert res["status"] == 0
    out, _, _ = _oracle(inp, True)
    assert np.all(res["out"][0] == 0)
    check(w, res["out"], out)


@pytest.mark.parametrize("L", [1, 2, 127, 128, 129])
def test_short_sequences(D, cuda_ok, L):
    for base in (synth.WORKLOADS[2].with_sizes(H=2, lengths=None), synth.WORKLOADS[3].with_sizes(H=2)):
        w = base.with_sizes(L=L)
        inp = synth.make_inputs(w)
        res = forward(D, w, inp, cuda_ok)
        out, _, _ = _oracle(inp, w.causal)
        check(w, res["out"], out)


def test_shared_and_per_head_geometry_agree_when_equal(D, cuda_ok):
    w = synth.WORKLOADS[2].with_sizes(H=3, L=150, lengths=None)
    inp = synth.make_inputs(w)
    shared = dict(inp, geom=inp["geom"][:1])
    tiled = dict(inp, geom=np.repeat(inp["geom"][:1], 3, axis=0))
    a = forward(D, w, shared, cuda_ok)["out"]
    b = forward(D, w, tiled, cuda_ok)["out"]
    np.testing.assert_array_equal(a, b)


def test_workspace_reuse_is_deterministic(D, cuda_ok):
    w = SMALL["c2"]
    inp = synth.make_inputs(w)
    r1 = forward(D, w, inp, cuda_ok)
    r2 = forward(D, w, inp, cuda_ok, ws=r1["ws"])
    np.testing.assert_array_equal(r1["out"], r2["out"])
    assert r1["ws"][:256].count_nonzero().item() == 0
