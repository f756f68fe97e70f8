"""Parity of the streaming decode step (through the C ABI) with the fp64 oracle."""
import numpy as np
import pytest
import torch

from oracle import dark_oracle as O
from random_feature_linear_b200 import synth

from gpu_run import check, forward, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def D(cuda_ok):
    from random_feature_linear_b200 import dark
    return dark


def _decode_run(D, dev, w, inp, stream, steps, stabilise=False, valid=None):
    flags = D.DARK_CAUSAL | (D.DARK_STABILISE if stabilise else 0)
    res = forward(D, w, inp, dev, flags=flags, with_state=True)
    assert res["status"] == 0
    proj, st = res["proj"], res["state"]
    tdt = D.torch_dtype(proj.dtype)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    outs = []
    for t in range(steps):
        q, k, v = (to_dev(stream[nm][t], tdt, dev) for nm in ("q", "k", "v"))
        out = torch.empty_like(q)
        vt = None if valid is None else torch.from_numpy(valid[t]).to(dev)
        D.dark_decode_step(proj, st, q, k, v, out, valid=vt, dev_status=status)
        outs.append(out.double().cpu().numpy())
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return outs, res


def _oracle_decode(inp, stream, steps, valid=None):
    _, kv, z = O.attention(inp["q"], inp["k"], inp["v"], inp["omega"], inp["geom"],
                           key_mask=inp["mask"], causal=True)
    outs = []
    for t in range(steps):
        o, kv, z = O.decode_step(kv, z, stream["q"][t], stream["k"][t], stream["v"][t],
                                 inp["omega"], inp["geom"], valid=None if valid is None else valid[t])
        outs.append(o)
    return outs


@pytest.mark.parametrize("stabilise", [False, True])
def test_decode_after_prefill(D, cuda_ok, stabilise):
    w = synth.WORKLOADS[5].with_sizes(B=3, H=2, L=333)
    inp = synth.make_inputs(w)
    stream = synth.decode_stream(w, 6)
    got, _ = _decode_run(D, cuda_ok, w, inp, stream, 6, stabilise=stabilise)
    ref = _oracle_decode(inp, stream, 6)
    for g, r in zip(got, ref):
        check(w, g[:, :, None], r[:, :, None])


def test_decode_with_invalid_tokens(D, cuda_ok):
    w = synth.WORKLOADS[5].with_sizes(B=4, H=2, L=130)
    inp = synth.make_inputs(w)
    stream = synth.decode_stream(w, 4)
    valid = np.array([[1, 0, 1, 1], [0, 0, 1, 0], [1, 1, 1, 1], [1, 0, 0, 1]], np.uint8)
    got, _ = _decode_run(D, cuda_ok, w, inp, stream, 4, valid=valid)
    ref = _oracle_decode(inp, stream, 4, valid=valid)
    for g, r in zip(got, ref):
        check(w, g[:, :, None], r[:, :, None])


def test_decode_fp32(D, cuda_ok):
    w = synth.WORKLOADS[1].with_sizes(B=2, H=2, L=70, causal=True)
    inp = synth.make_inputs(w)
    stream = synth.decode_stream(w, 3)
    got, _ = _decode_run(D, cuda_ok, w, inp, stream, 3)
    ref = _oracle_decode(inp, stream, 3)
    for g, r in zip(got, ref):
        check(w, g[:, :, None], r[:, :, None])


def test_decode_from_empty_state_returns_first_value(D, cuda_ok):
    w = synth.WORKLOADS[5].with_sizes(B=2, H=2, L=1)
    inp = synth.make_inputs(w)
    dev = cuda_ok
    omega = torch.from_numpy(inp["omega"]).to(dev)
    geom = torch.from_numpy(inp["geom"]).to(dev)
    proj, _wb = D.dark_make_projection(omega, geom, 2, D.DARK_BF16)
    st, tens = D.make_state(proj, 2, 2, dev)
    D.dark_state_init(proj, st)
    s = synth.decode_stream(w, 1)
    q, k, v = (to_dev(s[nm][0], torch.bfloat16, dev) for nm in ("q", "k", "v"))
    out = torch.empty_like(q)
    D.dark_decode_step(proj, st, q, k, v, out)
    torch.cuda.synchronize()
    assert torch.equal(out, v)


def test_redraw_makes_state_stale(D, cuda_ok):
    w = synth.WORKLOADS[5].with_sizes(B=2, H=2, L=64)
    inp = synth.make_inputs(w)
    res = forward(D, w, inp, cuda_ok, with_state=True)
    dev = cuda_ok
    omega = torch.from_numpy(inp["omega"]).to(dev)
    geom = torch.from_numpy(inp["geom"]).to(dev)
    proj2, _wb = D.dark_make_projection(omega, geom, 2, D.DARK_BF16)
    assert proj2.generation != res["proj"].generation
    q = torch.zeros(2, 2, 64, dtype=torch.bfloat16, device=dev)
    with pytest.raises(D.DarkError) as ei:
        D.dark_decode_step(proj2, res["state"], q, q, q, torch.empty_like(q))
    assert ei.value.status == D.DARK_ERR_STALE_STATE
    # the old projection still accepts it
    D.dark_decode_step(res["proj"], res["state"], q, q, q, torch.empty_like(q))
    torch.cuda.synchronize()


def test_decode_shared_projection(D, cuda_ok):
    # one W' for all heads (shared Omega and M)
    w = synth.WORKLOADS[5].with_sizes(B=5, H=3, L=140, per_head_geom=False)
    inp = synth.make_inputs(w)
    stream = synth.decode_stream(w, 3)
    got, _ = _decode_run(D, cuda_ok, w, inp, stream, 3)
    ref = _oracle_decode(inp, stream, 3)
    for g, r in zip(got, ref):
        check(w, g[:, :, None], r[:, :, None])


@pytest.mark.parametrize("dims", [(128, 256, 128), (256, 512, 256)])
def test_decode_after_wide_prefill(D, cuda_ok, dims):
    # prefill on the wide-head path (state carried in TMEM value blocks), then
    # decode; at d=128 W' (96 KB) is read from L2, at d=256 as well (384 KB)
    d, m, r = dims
    w = synth.WORKLOADS[4].with_sizes(B=1, H=2, L=200, d=d, r=r, m=m)
    inp = synth.make_inputs(w)
    stream = synth.decode_stream(w, 3)
    got, _ = _decode_run(D, cuda_ok, w, inp, stream, 3)
    ref = _oracle_decode(inp, stream, 3)
    for g, r_ in zip(got, ref):
        check(w, g[:, :, None], r_[:, :, None])


def test_decode_staged_projection_small_m(D, cuda_ok):
    # m=128, r=32, d=64: W' (20 KB) staged in shared memory, 3 passes of rows
    w = synth.WORKLOADS[5].with_sizes(B=2, H=3, L=150, m=128, r=32)
    inp = synth.make_inputs(w)
    stream = synth.decode_stream(w, 4)
    got, _ = _decode_run(D, cuda_ok, w, inp, stream, 4)
    ref = _oracle_decode(inp, stream, 4)
    for g, r_ in zip(got, ref):
        check(w, g[:, :, None], r_[:, :, None])


@pytest.mark.parametrize("per_head,B", [(True, 41), (False, 41), (True, 40), (False, 40)],
                         ids=["per-head-geometry-odd", "shared-geometry-odd",
                              "per-head-geometry-even", "shared-geometry-even"])
def test_decode_many_heads(D, cuda_ok, per_head, B):
    # More heads than twice the SM count, with invalid tokens in some batch rows:
    # an even batch runs two batch rows per block (the second row's state through
    # shared memory), an odd one a row per block
    w = synth.WORKLOADS[5].with_sizes(B=B, H=8, L=130, per_head_geom=per_head)
    inp = synth.make_inputs(w)
    steps = 3
    stream = synth.decode_stream(w, steps)
    rng = np.random.default_rng(5)
    valid = (rng.random((steps, w.B)) > 0.2).astype(np.uint8)
    got, res = _decode_run(D, cuda_ok, w, inp, stream, steps, valid=valid)
    ref = _oracle_decode(inp, stream, steps, valid=valid)
    for g, r in zip(got, ref):
        check(w, g[:, :, None], r[:, :, None])
    # the state after the steps: the oracle's recurrence over prefill and steps
    _, kv, z = O.attention(inp["q"], inp["k"], inp["v"], inp["omega"], inp["geom"],
                           key_mask=inp["mask"], causal=True)
    for t in range(steps):
        _, kv, z = O.decode_step(kv, z, stream["q"][t], stream["k"][t], stream["v"][t],
                                 inp["omega"], inp["geom"], valid=valid[t])
    kv_g = res["state_tensors"][0].double().cpu().numpy()
    z_g = res["state_tensors"][1].double().cpu().numpy()
    for got_s, ref_s in ((kv_g, kv), (z_g, z)):
        scale = np.abs(ref_s).reshape(w.B, w.H, -1).max(axis=2)
        err = np.abs(got_s - ref_s).reshape(w.B, w.H, -1).max(axis=2) / scale
        assert err.max() <= 2e-2, err.max()
