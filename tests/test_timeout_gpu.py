"""The device time-out path of the tensor-core kernels (GPU, through the C ABI).

Every wait of a tensor-core kernel on another part of the GPU is bounded; a
wait that runs out records DARK_ERR_TIMEOUT in the caller's status word, waits
(bounded) for the CTA's own copies and MMAs still in flight, frees its TMEM and
returns. The testing hook dark_set_test_stall_cycles makes every tensor-core
kernel first wait on a barrier that nothing completes, so that this path runs
deterministically without any fault: the call must report DARK_ERR_TIMEOUT,
and the next call on the same context (hook off) must match the oracle.
"""
import numpy as np
import pytest
import torch

from oracle import dark_oracle as O
from random_feature_linear_b200 import synth

from gpu_run import check, forward

pytestmark = pytest.mark.gpu

CASES = {
    # causal d64 with few heads: key-state launch and the chunk kernel
    "causal-d64": (synth.WORKLOADS[2].with_sizes(H=2, L=300, lengths=(300, 217)), 0),
    # non-causal d64: key states, reduction, query tiles
    "noncausal-d64": (synth.WORKLOADS[3].with_sizes(H=3, L=400), 0),
    # wide heads: features launch and value launch
    "wide-d128": (synth.WORKLOADS[4].with_sizes(B=1, H=2, L=260, d=128, r=128, m=256), 0),
    # exact mode on the tensor cores
    "exact-d64": (synth.WORKLOADS[2].with_sizes(H=2, L=260, lengths=(260, 200)), 4),
}


@pytest.fixture(scope="module")
def D(cuda_ok):
    from random_feature_linear_b200 import dark
    yield dark
    dark.dark_set_test_stall_cycles(0)


@pytest.mark.parametrize("name", list(CASES))
def test_stalled_wait_reports_timeout_and_context_survives(D, cuda_ok, name):
    w, extra = CASES[name]
    inp = synth.make_inputs(w)
    flags = (D.DARK_CAUSAL if w.causal else 0) | (D.DARK_EXACT if extra & 4 else 0)
    try:
        D.dark_set_test_stall_cycles(20000)
        res = forward(D, w, inp, cuda_ok, flags=flags)
    finally:
        D.dark_set_test_stall_cycles(0)
    assert res["status"] == D.DARK_ERR_TIMEOUT, D.dark_status_string(res["status"])
    # the same context keeps working, with the hook off
    res = forward(D, w, inp, cuda_ok, flags=flags)
    assert res["status"] == 0, D.dark_status_string(res["status"])
    if flags & D.DARK_EXACT:
        ref = O.exact_attention(inp["q"], inp["k"], inp["v"], inp["geom"], key_mask=inp["mask"],
                                causal=w.causal)
    else:
        ref = O.attention(inp["q"], inp["k"], inp["v"], inp["omega"], inp["geom"],
                          key_mask=inp["mask"], causal=w.causal)[0]
    check(w, res["out"], ref)
