"""Parity of the device projection sampler with the oracle's (same generator,
written independently on each side), reproducibility, and a forward pass on a
device-sampled projection."""
import numpy as np
import pytest
import torch

from oracle import dark_oracle as O
from oracle import dark_sampler as S
from random_feature_linear_b200 import synth

from gpu_run import check, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def D(cuda_ok):
    from random_feature_linear_b200 import dark
    return dark


CASES = [
    # (seed, draw, heads, m, r, orthogonal)
    (7, 0, 1, 256, 64, True),          # the causal workload's shape
    (7, 3, 2, 20, 8, True),            # two heads, partial last block
    (123, 1, 1, 512, 256, True),       # the large-head workload's shape
    (5, 0, 1, 3, 1, True),             # r = 1
    (2**63 + 5, 2**40, 3, 64, 64, False),
    (11, 2, 2, 100, 30, False),        # element count not a multiple of 4
]


@pytest.mark.parametrize("case", CASES)
def test_sampler_matches_oracle(D, cuda_ok, case):
    seed, draw, heads, m, r, orth = case
    om = torch.full((heads, m, r), float("nan"), dtype=torch.float32, device=cuda_ok)
    D.dark_sample_omega(seed, draw, om, orthogonal=orth)
    torch.cuda.synchronize()
    got = om.double().cpu().numpy()
    ref = S.sample_omega(seed, draw, heads, m, r, orth)
    assert np.all(np.isfinite(got))
    assert np.abs(got - ref).max() <= 1e-6 * max(1.0, np.abs(ref).max())


def test_sampler_is_reproducible_and_draws_differ(D, cuda_ok):
    a, b, c = (torch.empty(1, 256, 64, dtype=torch.float32, device=cuda_ok) for _ in range(3))
    D.dark_sample_omega(7, 0, a)
    D.dark_sample_omega(7, 0, b)
    D.dark_sample_omega(7, 1, c)
    torch.cuda.synchronize()
    assert torch.equal(a, b)
    assert (a - c).abs().max().item() > 0.5


def test_forward_on_a_sampled_projection(D, cuda_ok):
    # Omega sampled on the device, then the causal masked forward; the oracle uses
    # its own draw of the same (seed, draw), rounded to fp32 like the device's
    w = synth.WORKLOADS[2].with_sizes(H=2, L=200, lengths=(200, 150))
    inp = synth.make_inputs(w)
    om = torch.empty(1, w.m, w.r, dtype=torch.float32, device=cuda_ok)
    D.dark_sample_omega(2024, 0, om)
    geom = torch.from_numpy(inp["geom"]).to(cuda_ok)
    proj, _wbuf = D.dark_make_projection(om, geom, w.H, D.DARK_BF16)
    q, k, v = (to_dev(inp[n], torch.bfloat16, cuda_ok) for n in ("q", "k", "v"))
    out = torch.empty_like(q)
    mask = torch.from_numpy(inp["mask"]).to(cuda_ok)
    ws = D.alloc_workspace(proj, w.B, w.H, w.L, D.DARK_CAUSAL, cuda_ok)
    D.dark_attention_fwd(proj, q, k, v, out, w.B, w.H, w.L, key_mask=mask, flags=D.DARK_CAUSAL,
                         ws=ws)
    torch.cuda.synchronize()
    om_ref = S.sample_omega(2024, 0, 1, w.m, w.r, True).astype(np.float32)
    ref, _, _ = O.attention(inp["q"], inp["k"], inp["v"], om_ref, inp["geom"],
                            key_mask=inp["mask"], causal=True)
    check(w, out.double().cpu().numpy(), ref)
