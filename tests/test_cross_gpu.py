"""Parity of cross-attention (queries over a separate context) and of decoding
against a fixed context summary, through the C ABI, with the fp64 oracle."""
import numpy as np
import pytest
import torch

from oracle import dark_oracle as O
from random_feature_linear_b200 import synth

from gpu_run import check, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def D(cuda_ok):
    from random_feature_linear_b200 import dark
    return dark


def _inputs(w, Lq, Lk, q_len=None, ctx_len=None):
    """Queries from the recipe at length Lq, context keys/values at length Lk
    (same Omega and M); masks from per-batch valid lengths (tail padded)."""
    iq = synth.make_inputs(w.with_sizes(L=Lq, lengths=None))
    ik = synth.make_inputs(w.with_sizes(L=Lk, lengths=None), salt=1)
    qm = None if q_len is None else (np.arange(Lq)[None] < np.asarray(q_len)[:, None]).astype(np.uint8)
    cm = None if ctx_len is None else (np.arange(Lk)[None] < np.asarray(ctx_len)[:, None]).astype(np.uint8)
    return dict(q=iq["q"], k=ik["k"], v=ik["v"], omega=iq["omega"], geom=iq["geom"], qm=qm, cm=cm)


def _run(D, dev, w, x, flags=0, strided=False, with_state=True):
    dt = D.DARK_BF16 if w.dtype == "bf16" else D.DARK_F32
    tdt = D.torch_dtype(dt)
    proj, wbuf = D.dark_make_projection(torch.from_numpy(x["omega"]).to(dev),
                                        torch.from_numpy(x["geom"]).to(dev), w.H, dt)
    B, H, Lq, d = x["q"].shape
    Lk = x["k"].shape[2]
    qs = kvs = os_ = None
    if strided:
        # queries and output as [B][L][H][d]; keys and values interleaved [B][L][2][H][d]
        qt = to_dev(x["q"], tdt, dev).permute(0, 2, 1, 3).contiguous()
        q = qt.permute(0, 2, 1, 3)
        kv = torch.empty(B, Lk, 2, H, d, dtype=tdt, device=dev)
        kv[:, :, 0] = to_dev(x["k"], tdt, dev).permute(0, 2, 1, 3)
        kv[:, :, 1] = to_dev(x["v"], tdt, dev).permute(0, 2, 1, 3)
        k, v = kv[:, :, 0], kv[:, :, 1]
        qs, kvs = (Lq * H * d, d, H * d), (Lk * 2 * H * d, d, 2 * H * d)
        out_t = torch.full((B, Lq, H, d), float("nan"), dtype=tdt, device=dev)
        os_ = (Lq * H * d, d, H * d)
        out = out_t
    else:
        q, k, v = (to_dev(x[n], tdt, dev) for n in ("q", "k", "v"))
        out = torch.full((B, H, Lq, d), float("nan"), dtype=tdt, device=dev)
    qm = None if x["qm"] is None else torch.from_numpy(x["qm"]).to(dev)
    cm = None if x["cm"] is None else torch.from_numpy(x["cm"]).to(dev)
    st, st_t = D.make_state(proj, B, H, dev, stabilised=bool(flags & D.DARK_STABILISE)) \
        if with_state else (None, None)
    ws = D.alloc_cross_workspace(proj, B, H, Lq, Lk, flags, dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    D.dark_cross_attention_fwd(proj, q, k, v, out, B, H, Lq, Lk, query_mask=qm, context_mask=cm,
                               flags=flags, context_out=st, ws=ws, dev_status=status,
                               q_strides=qs, kv_strides=kvs, out_strides=os_)
    torch.cuda.synchronize()
    assert int(status.item()) == 0, D.dark_status_string(int(status.item()))
    o = out.permute(0, 2, 1, 3) if strided else out
    return dict(out=o.double().cpu().numpy(), proj=proj, wbuf=wbuf, state=st, st_t=st_t)


def _oracle(x):
    return O.cross_attention(x["q"], x["k"], x["v"], x["omega"], x["geom"], query_mask=x["qm"],
                             context_mask=x["cm"])


CASES = {
    # tensor-core path (bf16, d = 64, m in {128, 256}, r a multiple of 16 up to 64)
    "tc-ragged-masked": (synth.WORKLOADS[2].with_sizes(H=2), 200, 333, (200, 150), (333, 260)),
    "tc-short-context": (synth.WORKLOADS[3].with_sizes(H=2), 390, 70, None, None),
    "tc-long-context": (synth.WORKLOADS[2].with_sizes(B=1, H=3), 65, 700, None, (610,)),
    # SIMT path: fp32 I/O, and a shape the tensor-core kernels do not take
    "simt-fp32": (synth.WORKLOADS[1].with_sizes(B=2, H=2), 70, 150, (70, 33), (150, 97)),
    "simt-d128": (synth.WORKLOADS[4].with_sizes(B=1, H=2, d=128, r=32, m=128), 90, 130, None, None),
}


@pytest.mark.parametrize("name", list(CASES))
def test_cross_attention_matches_oracle(D, cuda_ok, name):
    w, Lq, Lk, ql, cl = CASES[name]
    x = _inputs(w, Lq, Lk, ql, cl)
    res = _run(D, cuda_ok, w, x)
    out, kv, z = _oracle(x)
    check(w, res["out"], out)
    if x["qm"] is not None:
        dead = np.broadcast_to((x["qm"] == 0)[:, None, :, None], out.shape)
        assert np.all(res["out"][dead] == 0.0)
    st_kv = res["st_t"][0].double().cpu().numpy()
    st_z = res["st_t"][1].double().cpu().numpy()
    tol = 1e-4 if w.dtype == "f32" else 2e-2
    for got, ref in ((st_kv, kv), (st_z, z)):
        scale = np.abs(ref).reshape(ref.shape[0], ref.shape[1], -1).max(axis=2)
        err = np.abs(got - ref).reshape(scale.shape + (-1,)).max(axis=2) / scale
        assert err.max() <= tol, err.max()


@pytest.mark.parametrize("name", ["tc-ragged-masked", "simt-fp32"])
def test_cross_attention_strided(D, cuda_ok, name):
    w, Lq, Lk, ql, cl = CASES[name]
    x = _inputs(w, Lq, Lk, ql, cl)
    res = _run(D, cuda_ok, w, x, strided=True, with_state=False)
    check(w, res["out"], _oracle(x)[0])


def test_cross_attention_stabilised(D, cuda_ok):
    w, Lq, Lk, ql, cl = CASES["tc-ragged-masked"]
    x = _inputs(w, Lq, Lk, ql, cl)
    res = _run(D, cuda_ok, w, x, flags=D.DARK_STABILISE, with_state=False)
    check(w, res["out"], _oracle(x)[0])


def test_empty_context_and_single_tokens(D, cuda_ok):
    w = synth.WORKLOADS[2].with_sizes(B=2, H=1)
    x = _inputs(w, 5, 9, None, (0, 9))
    res = _run(D, cuda_ok, w, x, with_state=False)
    assert np.all(res["out"][0] == 0.0)
    check(w, res["out"], _oracle(x)[0])
    x1 = _inputs(w, 1, 1)
    res1 = _run(D, cuda_ok, w, x1, with_state=False)
    check(w, res1["out"], _oracle(x1)[0])


@pytest.mark.parametrize("name", ["tc-ragged-masked", "simt-fp32"])
def test_cross_decode_against_the_summary(D, cuda_ok, name):
    w, Lq, Lk, ql, cl = CASES[name]
    x = _inputs(w, Lq, Lk, ql, cl)
    res = _run(D, cuda_ok, w, x)
    proj, st, st_t = res["proj"], res["state"], res["st_t"]
    kv0, z0 = st_t[0].clone(), st_t[1].clone()
    stream = synth.decode_stream(w, 3)
    tdt = D.torch_dtype(proj.dtype)
    status = torch.zeros(1, dtype=torch.int32, device=cuda_ok)
    _, kv, z = _oracle(x)
    for t in range(3):
        q = to_dev(stream["q"][t], tdt, cuda_ok)
        out = torch.empty_like(q)
        D.dark_cross_decode_step(proj, st, q, out, dev_status=status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        ref = O.cross_decode_step(kv, z, stream["q"][t], x["omega"], x["geom"])
        check(w, out.double().cpu().numpy()[:, :, None], ref[:, :, None])
    # the summary is read only
    assert torch.equal(st_t[0], kv0) and torch.equal(st_t[1], z0)
