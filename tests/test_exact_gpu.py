"""Parity of the exact learned-kernel mode (DARK_EXACT) with the oracle's exact
attention, through the C ABI: self- and cross-attention, masks, strides, the
no-allocation entry point and the full causal workload on sampled heads."""
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


CASES = {
    "bf16-causal-c2": synth.WORKLOADS[2].with_sizes(H=2, L=200, lengths=(200, 150)),
    "bf16-noncausal-c3": synth.WORKLOADS[3].with_sizes(H=2, L=300),
    "f32-noncausal-masked": synth.WORKLOADS[1].with_sizes(B=2, H=2, L=150, lengths=(150, 97)),
    "f32-causal": synth.WORKLOADS[1].with_sizes(B=1, H=2, L=130, causal=True),
    "bf16-causal-d128": synth.WORKLOADS[4].with_sizes(B=1, H=2, L=130, d=128, r=128, m=256),
    # d = 128 on the tensor cores: r = 64 (one projection block), key masks
    # and a ragged last tile over three 128-token tiles
    "bf16-noncausal-d128-r64": synth.WORKLOADS[3].with_sizes(H=2, L=300, d=128, r=64, m=128),
    "bf16-causal-d128-masked": synth.WORKLOADS[2].with_sizes(H=2, L=300, lengths=(300, 211),
                                                             d=128, r=96, m=256),
    "f32-causal-d256": synth.WORKLOADS[4].with_sizes(B=1, H=1, L=70, d=256, r=64, m=128,
                                                      dtype="f32"),
    # six query tiles on a few heads: the key ranges are split across CTAs and
    # the splits' partial results combined
    "bf16-causal-split": synth.WORKLOADS[2].with_sizes(H=2, L=700, lengths=(700, 517)),
    "bf16-single-token": synth.WORKLOADS[2].with_sizes(H=1, L=1, lengths=(1, 1)),
    "bf16-empty-row": synth.WORKLOADS[2].with_sizes(H=1, L=90, lengths=(0, 90)),
}


def _flags(D, w):
    return D.DARK_EXACT | (D.DARK_CAUSAL if w.causal else 0)


def _ref(inp, causal):
    return O.exact_attention(inp["q"], inp["k"], inp["v"], inp["geom"], key_mask=inp["mask"],
                             causal=causal)


@pytest.mark.parametrize("name", list(CASES))
def test_exact_matches_oracle(D, cuda_ok, name):
    w = CASES[name]
    inp = synth.make_inputs(w)
    res = forward(D, w, inp, cuda_ok, flags=_flags(D, w))
    assert res["status"] == 0
    check(w, res["out"], _ref(inp, w.causal))


@pytest.mark.parametrize("name", ["bf16-causal-c2", "f32-noncausal-masked",
                                  "bf16-causal-d128-masked"])
def test_exact_strided(D, cuda_ok, name):
    w = CASES[name]
    inp = synth.make_inputs(w)
    res = forward(D, w, inp, cuda_ok, flags=_flags(D, w), strided=True)
    assert res["status"] == 0
    check(w, res["out"], _ref(inp, w.causal))


def test_exact_rejects_a_state_output(D, cuda_ok):
    w = CASES["bf16-causal-c2"]
    inp = synth.make_inputs(w)
    with pytest.raises(D.DarkError) as ei:
        forward(D, w, inp, cuda_ok, flags=_flags(D, w), with_state=True)
    assert ei.value.status == D.DARK_ERR_INVALID_ARG


def test_exact_no_alloc_entry_point(D, cuda_ok):
    w = CASES["bf16-causal-c2"]
    inp = synth.make_inputs(w)
    proj, _wbuf = D.dark_make_projection(torch.from_numpy(inp["omega"]).to(cuda_ok),
                                         torch.from_numpy(inp["geom"]).to(cuda_ok), w.H,
                                         D.DARK_BF16)
    q, k, v = (to_dev(inp[n], torch.bfloat16, cuda_ok) for n in ("q", "k", "v"))
    out = torch.empty_like(q)
    D.dark_attention_fwd_noalloc(proj, q, k, v, out, w.B, w.H, w.L,
                                 key_mask=torch.from_numpy(inp["mask"]).to(cuda_ok),
                                 flags=_flags(D, w))
    torch.cuda.synchronize()
    check(w, out.double().cpu().numpy(), _ref(inp, True))


def test_exact_cross_attention(D, cuda_ok):
    # 90 queries over 230 context tokens with both masks
    w = synth.WORKLOADS[2].with_sizes(H=2)
    iq = synth.make_inputs(w.with_sizes(L=90, lengths=None))
    ik = synth.make_inputs(w.with_sizes(L=230, lengths=None), salt=1)
    qm = (np.arange(90)[None] < np.array([90, 61])[:, None]).astype(np.uint8)
    cm = (np.arange(230)[None] < np.array([230, 170])[:, None]).astype(np.uint8)
    dev = cuda_ok
    proj, _wbuf = D.dark_make_projection(torch.from_numpy(iq["omega"]).to(dev),
                                         torch.from_numpy(iq["geom"]).to(dev), w.H, D.DARK_BF16)
    q = to_dev(iq["q"], torch.bfloat16, dev)
    k, v = (to_dev(ik[n], torch.bfloat16, dev) for n in ("k", "v"))
    out = torch.full_like(q, float("nan"))
    ws = D.alloc_cross_workspace(proj, w.B, w.H, 90, 230, D.DARK_EXACT, dev)
    D.dark_cross_attention_fwd(proj, q, k, v, out, w.B, w.H, 90, 230,
                               query_mask=torch.from_numpy(qm).to(dev),
                               context_mask=torch.from_numpy(cm).to(dev), flags=D.DARK_EXACT,
                               ws=ws)
    torch.cuda.synchronize()
    ref = O.exact_attention(iq["q"], ik["k"], ik["v"], iq["geom"], key_mask=cm, query_mask=qm)
    check(w, out.double().cpu().numpy(), ref)


def test_exact_full_size_sampled_heads(D, cuda_ok):
    w = synth.WORKLOADS[2]
    inp = synth.make_inputs(w)
    res = forward(D, w, inp, cuda_ok, flags=_flags(D, w))
    assert res["status"] == 0
    for h in (0, 5):
        sl = (slice(None), slice(h, h + 1))
        ref = O.exact_attention(inp["q"][sl], inp["k"][sl], inp["v"][sl], inp["geom"][h:h + 1],
                                key_mask=inp["mask"], causal=True)
        check(w, res["out"][sl], ref)
