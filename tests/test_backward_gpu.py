"""Parity of the backward pass (dq, dk, dv and the geometry gradient) through the
C ABI with the fp64 oracle, on seeded synthetic inputs.

Tolerances (per (batch, head), relative to the largest reference entry): fp32
I/O 1e-4 (fp32 arithmetic throughout); bf16 I/O 8e-3 for dq, dk, dv and the
geometry gradient: the bf16 path runs every contraction on the tensor cores
with tf32 operands (10 explicit mantissa bits, unit roundoff 2^-11) and fp32
accumulation, and rounding dq, dk, dv to bf16 moves each entry by up to 2^-9
of itself. A numpy emulation of that arithmetic on the causal workload gives
about 1.5e-3 for the gradients.
"""
import numpy as np
import pytest
import torch

from oracle import dark_oracle as O
from random_feature_linear_b200 import synth

from gpu_run import to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def D(cuda_ok):
    from random_feature_linear_b200 import dark
    return dark


def run_backward(D, w, inp, dout, dev, flags, strided=False):
    dt = D.DARK_BF16 if w.dtype == "bf16" else D.DARK_F32
    tdt = D.torch_dtype(dt)
    omega = torch.from_numpy(np.ascontiguousarray(inp["omega"])).to(dev)
    geom = torch.from_numpy(np.ascontiguousarray(inp["geom"])).to(dev)
    B, H, L, d = inp["q"].shape
    xs = gs = ds = None
    if strided:
        # q, k, v interleaved [B][L][3][H][d]; dout and the gradients [B][L][H][d]
        packed = torch.empty(B, L, 3, H, d, dtype=tdt, device=dev)
        for i, nm in enumerate(("q", "k", "v")):
            packed[:, :, i] = to_dev(inp[nm], tdt, dev).permute(0, 2, 1, 3)
        q, k, v = packed[:, :, 0], packed[:, :, 1], packed[:, :, 2]
        xs = (L * 3 * H * d, d, 3 * H * d)
        g = to_dev(dout, tdt, dev).permute(0, 2, 1, 3).contiguous()
        gs = ds = (L * H * d, d, H * d)
        grads = [torch.full((B, L, H, d), float("nan"), dtype=tdt, device=dev) for _ in range(3)]
    else:
        q, k, v = (to_dev(inp[nm], tdt, dev) for nm in ("q", "k", "v"))
        g = to_dev(dout, tdt, dev)
        grads = [torch.full((B, H, L, d), float("nan"), dtype=tdt, device=dev) for _ in range(3)]
    mask = None if inp["mask"] is None else torch.from_numpy(inp["mask"]).to(dev)
    dgeom = torch.full(tuple(geom.shape), float("nan"), dtype=torch.float32, device=dev)
    ws = D.alloc_bwd_workspace(omega, geom, B, H, L, dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    D.dark_attention_bwd(omega, geom, q, k, v, g, *grads, B, H, L, dt, key_mask=mask,
                         flags=flags, dgeom=dgeom, ws=ws, dev_status=status, qkv_strides=xs,
                         dout_strides=gs, grad_strides=ds)
    torch.cuda.synchronize()
    assert int(status.item()) == 0, D.dark_status_string(int(status.item()))
    out = [t.permute(0, 2, 1, 3) if strided else t for t in grads]
    return [t.double().cpu().numpy() for t in out] + [dgeom.double().cpu().numpy()]


def rel_per_head(got, ref):
    B, H = ref.shape[:2]
    worst = 0.0
    for b in range(B):
        for h in range(H):
            den = max(np.abs(ref[b, h]).max(), 1e-30)
            worst = max(worst, np.abs(got[b, h] - ref[b, h]).max() / den)
    return worst


def check_grads(w, got, ref):
    tol = 1e-4 if w.dtype == "f32" else 8e-3
    for name, g, r in zip(("dq", "dk", "dv"), got[:3], ref[:3]):
        assert np.all(np.isfinite(g)), name
        err = rel_per_head(g, r)
        assert err <= tol, f"{name}: relative error {err:.3e} > {tol}"
    dg, rg = got[3], ref[3]
    assert np.all(np.isfinite(dg))
    err = max(np.abs(dg[i] - rg[i]).max() / np.abs(rg[i]).max() for i in range(rg.shape[0]))
    assert err <= tol, f"dgeom: relative error {err:.3e} > {tol}"


SMALL = {
    "f32-noncausal-masked": synth.WORKLOADS[1].with_sizes(B=2, H=2, L=150, lengths=(150, 101)),
    "f32-causal-masked": synth.WORKLOADS[1].with_sizes(B=2, H=2, L=150, causal=True,
                                                       lengths=(150, 101)),
    "bf16-causal-c2": synth.WORKLOADS[2].with_sizes(H=2, L=200, lengths=(200, 150)),
    "bf16-noncausal-c3": synth.WORKLOADS[3].with_sizes(H=2, L=300),
    "bf16-causal-d128": synth.WORKLOADS[4].with_sizes(B=1, H=2, L=130, d=128, r=128, m=256),
    "f32-causal-d256": synth.WORKLOADS[4].with_sizes(B=1, H=1, L=70, d=256, r=64, m=128,
                                                      dtype="f32"),
    "f32-one-tile": synth.WORKLOADS[1].with_sizes(B=1, H=1, L=64, causal=True),
    "bf16-causal-ragged44": synth.WORKLOADS[2].with_sizes(H=2, L=300, lengths=(300, 217)),
}


def _ref(w, inp, dout, causal):
    return O.attention_backward(inp["q"], inp["k"], inp["v"], inp["omega"], inp["geom"], dout,
                                key_mask=inp["mask"], causal=causal)


@pytest.mark.parametrize("name", list(SMALL))
def test_backward_matches_oracle(D, cuda_ok, name):
    w = SMALL[name]
    inp = synth.make_inputs(w)
    dout = synth.make_cotangent(w)
    flags = D.DARK_CAUSAL if w.causal else 0
    got = run_backward(D, w, inp, dout, cuda_ok, flags)
    check_grads(w, got, _ref(w, inp, dout, w.causal))


@pytest.mark.parametrize("name", ["f32-causal-masked", "bf16-causal-c2", "bf16-noncausal-c3"])
def test_backward_stabilised(D, cuda_ok, name):
    w = SMALL[name]
    inp = synth.make_inputs(w)
    dout = synth.make_cotangent(w)
    flags = (D.DARK_CAUSAL if w.causal else 0) | D.DARK_STABILISE
    got = run_backward(D, w, inp, dout, cuda_ok, flags)
    check_grads(w, got, _ref(w, inp, dout, w.causal))


@pytest.mark.parametrize("name", ["bf16-causal-c2", "f32-noncausal-masked"])
def test_backward_strided(D, cuda_ok, name):
    w = SMALL[name]
    inp = synth.make_inputs(w)
    dout = synth.make_cotangent(w)
    flags = D.DARK_CAUSAL if w.causal else 0
    got = run_backward(D, w, inp, dout, cuda_ok, flags, strided=True)
    check_grads(w, got, _ref(w, inp, dout, w.causal))


def test_backward_per_head_omega_shared_geometry(D, cuda_ok):
    # Omega drawn per head, M shared: the geometry gradient collects every head
    w = synth.WORKLOADS[1].with_sizes(B=2, H=3, L=100, causal=True, lengths=(100, 77))
    inp = synth.make_inputs(w)
    inp["omega"] = np.stack([synth.draw_omega(np.random.default_rng(40 + h), w.m, w.r, "orthogonal")
                             for h in range(w.H)]).astype(np.float32)
    dout = synth.make_cotangent(w)
    got = run_backward(D, w, inp, dout, cuda_ok, D.DARK_CAUSAL)
    check_grads(w, got, _ref(w, inp, dout, True))


def test_backward_single_token(D, cuda_ok):
    # one token: the output is v exactly, so dv = dout and q, k and M get no
    # gradient (the oracle's are rounding noise around zero)
    w = synth.WORKLOADS[1].with_sizes(B=2, H=1, L=1, causal=True)
    inp = synth.make_inputs(w)
    dout = synth.make_cotangent(w)
    got = run_backward(D, w, inp, dout, cuda_ok, D.DARK_CAUSAL)
    scale = np.abs(dout).max()
    assert np.abs(got[2] - dout).max() <= 1e-5 * scale
    for g in (got[0], got[1], got[3]):
        assert np.abs(g).max() <= 1e-4 * scale


def test_backward_takes_tensor_strides(D, cuda_ok):
    # Omega drawn as a transposed (non-contiguous) array and q, k, v passed as
    # [B][L][H][d] permuted views without explicit strides: the binding hands the
    # kernels the tensors' own strides and a dense Omega
    w = SMALL["bf16-causal-c2"]
    inp = synth.make_inputs(w)
    dout = synth.make_cotangent(w)
    assert not inp["omega"].flags["C_CONTIGUOUS"]
    dev = cuda_ok
    omega = torch.from_numpy(inp["omega"]).to(dev)
    assert not omega.is_contiguous()
    geom = torch.from_numpy(inp["geom"]).to(dev)
    q, k, v, g = (to_dev(x, torch.bfloat16, dev).permute(0, 2, 1, 3).contiguous().permute(0, 2, 1, 3)
                  for x in (inp["q"], inp["k"], inp["v"], dout))
    grads = [torch.empty_like(q) for _ in range(3)]
    dgeom = torch.empty(tuple(geom.shape), dtype=torch.float32, device=dev)
    ws = D.alloc_bwd_workspace(omega, geom, w.B, w.H, w.L, dev)
    D.dark_attention_bwd(omega, geom, q, k, v, g, *grads, w.B, w.H, w.L, D.DARK_BF16,
                         key_mask=torch.from_numpy(inp["mask"]).to(dev), flags=D.DARK_CAUSAL,
                         dgeom=dgeom, ws=ws)
    torch.cuda.synchronize()
    got = [t.double().cpu().numpy() for t in grads] + [dgeom.double().cpu().numpy()]
    check_grads(w, got, _ref(w, inp, dout, True))


def test_backward_empty_rows(D, cuda_ok):
    # batch row 0 has no valid key: every gradient of that row is zero
    w = synth.WORKLOADS[2].with_sizes(H=2, L=90, lengths=(0, 90))
    inp = synth.make_inputs(w)
    dout = synth.make_cotangent(w)
    got = run_backward(D, w, inp, dout, cuda_ok, D.DARK_CAUSAL)
    for g in got[:3]:
        assert np.all(g[0] == 0.0)
    ref = _ref(w, inp, dout, True)
    check_grads(w, [g[1:] for g in got[:3]] + [got[3]], [r[1:] for r in ref[:3]] + [ref[3]])


def test_backward_full_size_sampled_heads(D, cuda_ok):
    # the causal masked workload at full size (B2 H8 L2048 d64 r64 m256); heads 0
    # and 7 (both batch rows) checked against the oracle run on those heads alone
    w = synth.WORKLOADS[2]
    inp = synth.make_inputs(w)
    dout = synth.make_cotangent(w)
    got = run_backward(D, w, inp, dout, cuda_ok, D.DARK_CAUSAL)
    for h in (0, 7):
        sl = (slice(None), slice(h, h + 1))
        ref = O.attention_backward(inp["q"][sl], inp["k"][sl], inp["v"][sl], inp["omega"],
                                   inp["geom"][h:h + 1], dout[sl], key_mask=inp["mask"],
                                   causal=True)
        check_grads(w, [g[sl] for g in got[:3]] + [got[3][h:h + 1]], ref)
