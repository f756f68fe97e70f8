"""The bench's algorithmic work counts (the roofline numerators) against figures
derived independently from the workloads' shapes, and hand counts at tiny sizes."""
import pytest

import bench
from random_feature_linear_b200 import synth


@pytest.mark.parametrize("cfg,flops,mbytes", [
    (2, 4.60e9, 16.8),     # causal masked, B2 H8 L2048 d64 r64 m256
    (3, 3.57e10, 134.2),   # non-causal, B1 H16 L16384 d64 r32 m256
    (4, 3.10e11, 536.9),   # causal, B4 H8 L8192 d256 r256 m512
])
def test_forward_work_counts(cfg, flops, mbytes):
    w = synth.WORKLOADS[cfg]
    assert bench.alg_flops(w) == pytest.approx(flops, rel=2e-3)
    assert bench.alg_bytes(w) / 1e6 == pytest.approx(mbytes, rel=2e-3)


def test_decode_bytes_are_the_state_read_and_written():
    w = synth.WORKLOADS[5]
    state = 2 * w.B * w.H * w.m * (w.d + 1) * 4          # fp32 (KV, z), read and written
    assert state / 1e6 == pytest.approx(68.2, rel=2e-3)
    assert bench.decode_bytes(w) >= state and bench.decode_bytes(w) - state < 0.3e6


def test_exact_and_backward_counts_by_hand():
    w = synth.WORKLOADS[1].with_sizes(B=1, H=1, L=4, d=8, r=2, m=3, causal=True)
    # exact: projections 2 * 2 * L d r, then 10 visible pairs x 2 (r + d)
    assert bench.exact_flops(w) == 2 * 2 * 4 * 8 * 2 + 10 * 2 * (2 + 8)
    # backward: features 2Ldm + 2Ld(m+r); five 2Lm(d+1); dx 2Ldm + 2Ld(m+r) + 2Ldr;
    # dW' 4L(m+r)d
    L, d, r, m = 4, 8, 2, 3
    by_hand = (2 * L * d * m + 2 * L * d * (m + r) + 5 * 2 * L * m * (d + 1)
               + 2 * L * d * m + 2 * L * d * (m + r) + 2 * L * d * r + 4 * L * (m + r) * d)
    assert bench.bwd_flops(w) == by_hand
