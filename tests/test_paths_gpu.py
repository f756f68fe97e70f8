"""Which kernels a call runs: each case launches one call in a fresh process
under the CUDA profiler (CUPTI records kernels in the first profiling session
of a process only) and checks the library's kernels in its launch list, so that
a shape meant for the tensor cores cannot pass its parity tests on the FFMA
kernels unnoticed."""
import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

_SCRIPT = r'''
import json, sys
import numpy as np, torch
from torch.profiler import ProfilerActivity, profile
from random_feature_linear_b200 import dark as D, synth
case = sys.argv[1]
dev = torch.device("cuda", 0)
def kernels(fn):
    fn(); torch.cuda.synchronize()
    with profile(activities=[ProfilerActivity.CUDA]) as prof:
        fn(); torch.cuda.synchronize()
    names = [e.name for e in prof.events() if e.device_type == torch.autograd.DeviceType.CUDA]
    return sorted(set(n for n in names if "dark::" in n))
if case.startswith("bwd"):
    w = synth.WORKLOADS[2].with_sizes(H=2, L=300, lengths=(300, 217))
    inp = synth.make_inputs(w)
    dout = synth.make_cotangent(w)
    omega = torch.from_numpy(np.ascontiguousarray(inp["omega"])).to(dev)
    geom = torch.from_numpy(np.ascontiguousarray(inp["geom"])).to(dev)
    q, k, v, g = (torch.from_numpy(np.ascontiguousarray(x)).to(dev).to(torch.bfloat16)
                  for x in (inp["q"], inp["k"], inp["v"], dout))
    grads = [torch.empty_like(q) for _ in range(3)]
    dgeom = torch.empty(tuple(geom.shape), dtype=torch.float32, device=dev)
    ws = D.alloc_bwd_workspace(omega, geom, w.B, w.H, w.L, dev)
    flags = D.DARK_CAUSAL | (D.DARK_STABILISE if case == "bwd-stab" else 0)
    mask = torch.from_numpy(inp["mask"]).to(dev)
    fn = lambda: D.dark_attention_bwd(omega, geom, q, k, v, g, *grads, w.B, w.H, w.L, D.DARK_BF16,
                                      key_mask=mask, flags=flags, dgeom=dgeom, ws=ws)
elif case.startswith("fwd") or case.startswith("exact"):
    w = {"fwd-stab-causal": synth.WORKLOADS[2].with_sizes(H=2, L=300, lengths=(300, 217)),
         "fwd-stab-noncausal": synth.WORKLOADS[3].with_sizes(H=2, L=300),
         "fwd-stab-wide": synth.WORKLOADS[4].with_sizes(B=1, H=2, L=300, lengths=(300,)),
         "exact-d64": synth.WORKLOADS[2].with_sizes(H=2, L=300, lengths=(300, 217)),
         "exact-d128": synth.WORKLOADS[2].with_sizes(H=2, L=300, lengths=(300, 217), d=128,
                                                     r=128)}[case]
    inp = synth.make_inputs(w)
    omega = torch.from_numpy(inp["omega"]).to(dev)
    geom = torch.from_numpy(inp["geom"]).to(dev)
    proj, _wb = D.dark_make_projection(omega, geom, w.H, D.DARK_BF16)
    q, k, v = (torch.from_numpy(inp[n]).to(dev).to(torch.bfloat16) for n in ("q", "k", "v"))
    out = torch.empty_like(q)
    mask = None if inp["mask"] is None else torch.from_numpy(inp["mask"]).to(dev)
    flags = (D.DARK_CAUSAL if w.causal else 0) | (
        D.DARK_EXACT if case.startswith("exact") else D.DARK_STABILISE)
    ws = D.alloc_workspace(proj, w.B, w.H, w.L, flags, dev)
    fn = lambda: D.dark_attention_fwd(proj, q, k, v, out, w.B, w.H, w.L, key_mask=mask,
                                      flags=flags, ws=ws)
print(json.dumps(kernels(fn)))
'''


def launched(case: str) -> list:
    p = subprocess.run([sys.executable, "-c", _SCRIPT, case], cwd=ROOT, capture_output=True,
                       text=True, timeout=600)
    assert p.returncode == 0, p.stderr[-3000:]
    return json.loads(p.stdout.strip().splitlines()[-1])


@pytest.mark.parametrize("case", ["bwd", "bwd-stab"])
def test_bf16_backward_runs_on_tensor_cores(cuda_ok, case):
    names = launched(case)
    for kernel in ("tbf_features_kernel", "tbf_state_kernel", "tbf_pass_kernel", "tbf_dx_kernel",
                   "tbf_dw_kernel"):
        assert any(kernel in n for n in names), (kernel, names)
    assert not any("pass_kernel<" in n and "tbf_" not in n for n in names), names


@pytest.mark.parametrize("case,kernel", [("fwd-stab-causal", "causal_kernel"),
                                         ("fwd-stab-noncausal", "queries_kernel")])
def test_stabilised_forward_runs_on_tensor_cores(cuda_ok, case, kernel):
    # DARK_STABILISE on bf16 d = 64: the key-constant pass runs in keys_kernel,
    # the attention in the tensor-core kernels; none of the FFMA kernels
    names = launched(case)
    assert any(kernel in n for n in names), names
    assert any("keys_kernel" in n for n in names), names
    assert not any(("out_kernel" in n or "scan_kernel" in n) for n in names), names


@pytest.mark.parametrize("case", ["exact-d64", "exact-d128"])
def test_bf16_exact_runs_on_tensor_cores(cuda_ok, case):
    names = launched(case)
    assert any("exact_tc_kernel" in n for n in names), names
    assert not any("exact_attn_kernel" in n for n in names), names


def test_stabilised_wide_forward_runs_on_tensor_cores(cuda_ok):
    # DARK_STABILISE at d = 256: the statistics pass and the stabilised pass of
    # features_kernel, then values_kernel; none of the FFMA kernels
    names = launched("fwd-stab-wide")
    assert sum("features_kernel<256, 512, 256" in n for n in names) == 2, names
    assert any("values_kernel" in n for n in names), names
    assert not any(("out_kernel" in n or "scan_kernel" in n or "chunk_state_kernel" in n)
                   for n in names), names
