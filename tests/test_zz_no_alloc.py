"""dark_attention_fwd_noalloc against dark_attention_fwd (GPU, through the C ABI).

The no-allocation entry point serves callers that cannot call cudaMalloc (a
runtime that hands the library only the tensors of the call, or an allocator
that refuses extra allocations): its scratch is a fixed array inside the
library. It must give the same results as the workspace entry point, and the
fp64 oracle's within the forward tolerances, call after call, even though every
call reuses the same scratch. This file is collected last so that a run
stopping at its first failure has run everything else before it.
"""
import numpy as np
import pytest
import torch

from oracle import dark_oracle as O
from random_feature_linear_b200 import synth

from gpu_run import check

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def D(cuda_ok):
    from random_feature_linear_b200 import dark
    return dark


def _run(D, dev, w, inp, noalloc):
    omega = torch.from_numpy(inp["omega"]).to(dev)
    geom = torch.from_numpy(inp["geom"]).to(dev)
    dt = D.DARK_BF16 if w.dtype == "bf16" else D.DARK_F32
    tdt = D.torch_dtype(dt)
    proj, wbuf = D.dark_make_projection(omega, geom, w.H, dt)
    q, k, v = (torch.from_numpy(inp[n]).to(dev).to(tdt) for n in ("q", "k", "v"))
    mask = None if inp["mask"] is None else torch.from_numpy(inp["mask"]).to(dev)
    out = torch.full_like(q, float("nan"))
    flags = D.DARK_CAUSAL if w.causal else 0
    st, st_t = D.make_state(proj, w.B, w.H, dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    if noalloc:
        D.dark_attention_fwd_noalloc(proj, q, k, v, out, w.B, w.H, w.L, key_mask=mask,
                                     flags=flags, state_out=st, dev_status=status)
    else:
        ws = D.alloc_workspace(proj, w.B, w.H, w.L, flags, dev)
        D.dark_attention_fwd(proj, q, k, v, out, w.B, w.H, w.L, key_mask=mask, flags=flags,
                             state_out=st, ws=ws, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return out.double().cpu().numpy(), st_t[0].double().cpu().numpy(), st_t[1].double().cpu().numpy()


CASES = [
    synth.WORKLOADS[2].with_sizes(H=2, L=300, lengths=(300, 217)),        # causal, tensor cores
    synth.WORKLOADS[3].with_sizes(H=3, L=700),                            # non-causal, tensor cores
    synth.WORKLOADS[1],                                                   # fp32, SIMT kernels
]


@pytest.mark.parametrize("w", CASES, ids=["causal-bf16", "noncausal-bf16", "noncausal-fp32"])
def test_noalloc_matches_workspace_entry_twice(D, cuda_ok, w):
    # two calls in a row with different inputs: the shared scratch keeps the
    # previous call's contents and must not leak into the next result
    for salt in (0, 1):
        inp = synth.make_inputs(w, salt=salt)
        ref, kv_ref, z_ref = _run(D, cuda_ok, w, inp, noalloc=False)
        got, kv, z = _run(D, cuda_ok, w, inp, noalloc=True)
        assert np.all(np.isfinite(got))
        if w.dtype == "f32":
            den = np.abs(ref).reshape(w.B, w.H, -1).max(axis=2)[:, :, None, None]
            assert (np.abs(got - ref) / den).max() <= 1e-4
        else:
            assert np.abs(got - ref).max() <= 2e-2
        np.testing.assert_allclose(kv, kv_ref, rtol=1e-4, atol=1e-6 * np.abs(kv_ref).max())
        np.testing.assert_allclose(z, z_ref, rtol=1e-4, atol=1e-6 * np.abs(z_ref).max())
        # and the fp64 oracle on the same inputs
        want, _, _ = O.attention(inp["q"], inp["k"], inp["v"], inp["omega"], inp["geom"],
                                 key_mask=inp["mask"], causal=w.causal)
        check(w, got, want)


def test_noalloc_rejects_calls_beyond_its_scratch(D, cuda_ok):
    w = synth.WORKLOADS[2].with_sizes(B=1, H=1, L=64, lengths=None)
    inp = synth.make_inputs(w)
    omega = torch.from_numpy(inp["omega"]).to(cuda_ok)
    geom = torch.from_numpy(inp["geom"]).to(cuda_ok)
    proj, _wb = D.dark_make_projection(omega, geom, 1, D.DARK_BF16)
    # a strided layout the tensor-core path refuses forces the generic path, whose
    # feature maps for this length need far more than the fixed scratch
    L = 1 << 16
    big = torch.zeros(2, 1, L, 64 + 4, dtype=torch.bfloat16, device=cuda_ok)
    q = big[..., :64]
    need = D.dark_attention_workspace_bytes(proj, 2, 1, L, 0)
    assert need > D.dark_noalloc_scratch_bytes()
    with pytest.raises(D.DarkError) as ei:
        D.dark_attention_fwd_noalloc(proj, q, q, q, torch.empty(2, 1, L, 64, dtype=torch.bfloat16,
                                                                device=cuda_ok), 2, 1, L,
                                     qkv_strides=(L * 68, L * 68, 68))
    assert ei.value.status == D.DARK_ERR_UNSUPPORTED
