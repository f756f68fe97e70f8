"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every entry point declared in include/dark.h, and rejects bad arguments before
anything is enqueued."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def D():
    from random_feature_linear_b200 import build
    build.build()
    from random_feature_linear_b200 import dark
    return dark


def _declared():
    src = open(os.path.join(ROOT, "include", "dark.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(dark_[a-z_]+)\s*\(", src)))


def test_every_declared_symbol_is_exported(D):
    names = _declared()
    assert "dark_attention_fwd" in names and "dark_decode_step" in names
    lib = ctypes.CDLL(D.library_path())
    for n in names:
        assert hasattr(lib, n), n
    assert set(D.EXPORTS) <= set(names)


def test_version_and_status_strings(D):
    hdr = open(os.path.join(ROOT, "include", "dark.h")).read()
    assert D.dark_abi_version() == int(re.search(r"#define DARK_ABI_VERSION (\d+)", hdr).group(1))
    for s in range(7):
        assert D.dark_status_string(s).startswith("DARK_")
    assert "unknown" in D.dark_status_string(99)


def test_projection_bytes(D):
    assert D.dark_projection_bytes(8, 256, 64, 64, D.DARK_BF16) == 8 * 320 * 64 * 2
    assert D.dark_projection_bytes(1, 64, 64, 64, D.DARK_F32) == 128 * 64 * 4
    assert D.dark_projection_bytes(0, 64, 64, 64, D.DARK_F32) == 0


def _fake_proj(D, **kw):
    p = D.dark_projection()
    p.heads, p.m, p.r, p.d, p.dtype, p.generation, p.w = 1, 64, 64, 64, D.DARK_BF16, 7, 0x1000
    for k, v in kw.items():
        setattr(p, k, v)
    return p


def test_make_projection_rejects_bad_arguments(D):
    lib = D._lib
    out = D.dark_projection()
    f = 0x1000
    # null pointers, head counts not in {1, H}, bad dtype, unsupported sizes, short buffer
    assert lib.dark_make_projection(None, 1, f, 1, 8, 64, 64, 64, 1, f, 1 << 20, None, ctypes.byref(out)) == 1
    assert lib.dark_make_projection(f, 3, f, 1, 8, 64, 64, 64, 1, f, 1 << 20, None, ctypes.byref(out)) == 1
    assert lib.dark_make_projection(f, 1, f, 1, 8, 64, 64, 64, 7, f, 1 << 20, None, ctypes.byref(out)) == 1
    assert lib.dark_make_projection(f, 1, f, 1, 8, 64, 64, 66, 1, f, 1 << 20, None, ctypes.byref(out)) == 2
    assert lib.dark_make_projection(f, 1, f, 1, 8, 2048, 64, 64, 1, f, 1 << 30, None, ctypes.byref(out)) == 2
    assert lib.dark_make_projection(f, 1, f, 1, 8, 64, 64, 64, 1, f, 100, None, ctypes.byref(out)) == 1
    assert lib.dark_make_projection(f, 1, f, 1, 8, 64, 64, 64, 1, f + 2, 1 << 20, None, ctypes.byref(out)) == 1


def test_forward_rejects_bad_arguments(D):
    lib = D._lib
    f = 0x10000
    p = _fake_proj(D)
    args = lambda **kw: dict(dict(q=f, k=f, v=f, o=f, B=2, H=1, L=16, flags=0, ws=f, wsb=1 << 30), **kw)

    def call(a, proj=p):
        return lib.dark_attention_fwd(ctypes.byref(proj), a["q"], a["k"], a["v"], a["o"], None, None,
                                      a["B"], a["H"], a["L"], None, a["flags"], None, a["ws"], a["wsb"],
                                      None, None)
    assert call(args(q=None)) == 1
    assert call(args(B=0)) == 1
    assert call(args(L=-3)) == 1
    assert call(args(flags=8)) == 1
    assert call(args(ws=None)) == 1
    assert call(args(ws=f + 16)) == 1                 # not 256-byte aligned
    assert call(args(H=3), _fake_proj(D, heads=2)) == 1
    assert call(args(), _fake_proj(D, d=66)) == 2
    assert call(args(), _fake_proj(D, w=0x1002)) == 1  # W' not 16-byte aligned
    assert call(args(wsb=16)) == 1                    # workspace too small
    st = D.dark_state(f, f, None, 2, 1, 32, 64, 0)     # m mismatch
    assert lib.dark_attention_fwd(ctypes.byref(p), f, f, f, f, None, None, 2, 1, 16, None, 0,
                                  ctypes.byref(st), f, 1 << 30, None, None) == 1
    st = D.dark_state(f, f, None, 2, 1, 64, 64, 0)     # stabilised state without shift
    assert lib.dark_attention_fwd(ctypes.byref(p), f, f, f, f, None, None, 2, 1, 16, None, 2,
                                  ctypes.byref(st), f, 1 << 30, None, None) == 1


def test_decode_rejects_stale_state_before_launch(D):
    lib = D._lib
    f = 0x10000
    p = _fake_proj(D, generation=5)
    st = D.dark_state(f, f, None, 2, 1, 64, 64, 4)
    assert lib.dark_decode_step(ctypes.byref(p), ctypes.byref(st), f, f, f, f, None, None, None) == 3
    st = D.dark_state(f, f, None, 2, 1, 64, 32, 5)     # d mismatch
    assert lib.dark_decode_step(ctypes.byref(p), ctypes.byref(st), f, f, f, f, None, None, None) == 1
    st = D.dark_state(f + 4, f, None, 2, 1, 64, 64, 5)  # kv not 16-byte aligned
    assert lib.dark_decode_step(ctypes.byref(p), ctypes.byref(st), f, f, f, f, None, None, None) == 1


def test_workspace_query(D):
    p = _fake_proj(D, m=256, d=64, heads=8)
    n1 = D.dark_attention_workspace_bytes(p, 2, 8, 2048, D.DARK_CAUSAL)
    n2 = D.dark_attention_workspace_bytes(p, 2, 8, 4096, D.DARK_CAUSAL)
    assert n1 >= 256 and n2 > n1
    assert D.dark_attention_workspace_bytes(p, 0, 8, 2048, 0) == 0


def test_cross_attention_rejects_bad_arguments(D):
    lib = D._lib
    f = 0x10000
    p = _fake_proj(D)

    def call(q=f, Lq=16, k=f, v=f, Lk=40, o=f, B=2, H=1, flags=0, ws=f, wsb=1 << 30, ctx=None):
        return lib.dark_cross_attention_fwd(ctypes.byref(p), q, None, Lq, None, k, v, None, Lk,
                                            None, o, None, B, H, flags, ctx, ws, wsb, None, None)

    assert call(flags=D.DARK_CAUSAL) == 1            # no causal cross-attention
    assert call(Lq=0) == 1 and call(Lk=0) == 1 and call(B=0) == 1
    assert call(q=None) == 1 and call(k=None) == 1 and call(o=None) == 1
    assert call(ws=None) == 1 and call(ws=f + 8) == 1
    assert call(flags=8) == 1
    st = D.dark_state(f, f, None, 2, 1, 64, 32, 0)      # d mismatch
    assert call(ctx=ctypes.byref(st)) == 1
    # workspace: none for causal, some for valid sizes, growing with the context
    assert D.dark_cross_attention_workspace_bytes(p, 2, 1, 16, 40, D.DARK_CAUSAL) == 0
    small = D.dark_cross_attention_workspace_bytes(p, 2, 1, 16, 40, 0)
    big = D.dark_cross_attention_workspace_bytes(p, 2, 1, 16, 4000, 0)
    assert 0 < small < big


def test_cross_decode_rejects_stale_and_bad_arguments(D):
    lib = D._lib
    f = 0x10000
    p = _fake_proj(D)
    st = D.dark_state(f, f, None, 2, 1, 64, 64, p.generation)
    assert lib.dark_cross_decode_step(ctypes.byref(p), None, f, f, None, None) == 1
    assert lib.dark_cross_decode_step(ctypes.byref(p), ctypes.byref(st), None, f, None, None) == 1
    stale = D.dark_state(f, f, None, 2, 1, 64, 64, p.generation + 1)
    assert lib.dark_cross_decode_step(ctypes.byref(p), ctypes.byref(stale), f, f, None, None) == 3


def test_backward_rejects_bad_arguments(D):
    lib = D._lib
    f = 0x10000
    need = D.dark_attention_bwd_workspace_bytes(1, 2, 64, 32, 64, 2, 2, 100)

    def call(om=f, ho=1, gm=f, hg=2, m=64, r=32, d=64, dt=D.DARK_BF16, q=f, g=f, B=2, H=2, L=100,
             flags=0, dq=f, ws=f, wsb=need, strides=None):
        return lib.dark_attention_bwd(om, ho, gm, hg, m, r, d, dt, q, f, f, strides, g, None, B, H,
                                      L, None, flags, dq, f, f, None, None, ws, wsb, None, None)

    assert call(om=None) == 1 and call(gm=None) == 1 and call(q=None) == 1
    assert call(g=None) == 1 and call(dq=None) == 1 and call(ws=None) == 1
    assert call(ho=3) == 1 and call(hg=0) == 1            # heads must be 1 or H
    assert call(B=0) == 1 and call(L=0) == 1
    assert call(flags=4) == 1 and call(dt=7) == 1
    assert call(d=6) == 2 and call(m=4096) == 2           # outside the library's sizes
    assert call(ws=f + 64) == 1 and call(wsb=need - 1) == 1
    assert call(strides=(ctypes.c_int64 * 3)(-1, 64, 64)) == 1
    assert call(B=300, H=300, hg=1, wsb=1 << 62) == 2      # grid bound on B*H
    # workspace size: zero for bad sizes, growing with L
    assert D.dark_attention_bwd_workspace_bytes(1, 2, 64, 32, 64, 0, 2, 100) == 0
    assert need < D.dark_attention_bwd_workspace_bytes(1, 2, 64, 32, 64, 2, 2, 1000)


def test_redraw_schedule_matches_oracle(D):
    # random sequences of forwards (training or evaluation), manual and forced
    # redraws, fix and unfix: the library's schedule and the oracle's take the
    # same decisions
    import random

    from oracle import dark_sampler as S
    rng = random.Random(5)
    for trial in range(40):
        interval = rng.choice([None, 1, 2, 3, 5])
        det = rng.random() < 0.2
        lib, ref = D.RedrawSchedule(9, interval, det), S.RedrawSchedule(9, interval, det)
        for _ in range(60):
            op = rng.randrange(6)
            if op <= 2:
                tr = op != 2
                assert lib.forward(tr) == ref.forward(tr)
            elif op == 3:
                f = rng.random() < 0.3
                assert lib.redraw(f) == ref.redraw(f)
            elif op == 4:
                lib.fix()
                ref.fix()
            else:
                lib.unfix()
                ref.unfix()
            assert lib.draw == ref.draw


def test_sampler_rejects_bad_arguments(D):
    lib = D._lib
    f = 0x10000
    need = D.dark_sample_omega_workspace_bytes(1, 256, 64, True)
    assert need > 0 and D.dark_sample_omega_workspace_bytes(1, 256, 64, False) == 0
    assert lib.dark_sample_omega(1, 0, 1, 256, 64, 1, None, f, need, None) == 1
    assert lib.dark_sample_omega(1, 0, 1, 256, 64, 1, f + 2, f, need, None) == 1
    assert lib.dark_sample_omega(1, 0, 0, 256, 64, 1, f, f, need, None) == 1
    assert lib.dark_sample_omega(1, 0, 1, 256, 64, 1, f, None, need, None) == 1
    assert lib.dark_sample_omega(1, 0, 1, 256, 64, 1, f, f, need - 8, None) == 1
    assert lib.dark_sample_omega(1, 0, 1, 256, 64, 1, f, f + 16, need, None) == 1
    assert lib.dark_sample_omega(1, 0, 1, 256, 512, 1, f, f, 1 << 40, None) == 2
    assert lib.dark_sample_omega(1, 0, 1, 4096, 64, 0, f, None, 0, None) == 2


def test_binding_takes_strides_from_the_tensors(D):
    import torch
    x = torch.zeros(2, 3, 5, 8)
    assert list(D._strides(None, x)) == [120, 40, 8]
    # a [B][L][H][d] buffer viewed as [B][H][L][d]
    y = torch.zeros(2, 5, 3, 8).permute(0, 2, 1, 3)
    assert list(D._strides(None, y, y)) == [120, 8, 24]
    # explicit strides win
    assert list(D._strides((1, 2, 3), x)) == [1, 2, 3]
    with pytest.raises(ValueError):
        D._strides(None, x, y)                     # q, k, v must share one layout
    with pytest.raises(ValueError):
        D._strides(None, torch.zeros(2, 3, 8, 5).transpose(2, 3))   # d must be innermost
    with pytest.raises(ValueError):
        D._dense(torch.zeros(4, 6)[:, ::2], "mask")  # arrays without strides must be dense
    assert D._dense(None, "mask") is None
