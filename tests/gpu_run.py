"""Runs the CUDA path through the C ABI on seeded synthetic inputs (test helper)."""
from __future__ import annotations

import numpy as np
import torch

from random_feature_linear_b200 import synth


def dtype_code(D, w: synth.Workload) -> int:
    return D.DARK_BF16 if w.dtype == "bf16" else D.DARK_F32


def to_dev(x, tdt, dev):
    return torch.from_numpy(np.ascontiguousarray(x)).to(dev).to(tdt)


def forward(D, w: synth.Workload, inp: dict, dev, flags=None, with_state=False, strided=False,
            ws=None):
    """Returns dict(out=fp64 numpy, kv, z, shift, status, proj, tensors...)."""
    dt = dtype_code(D, w)
    tdt = D.torch_dtype(dt)
    omega = torch.from_numpy(inp["omega"]).to(dev)
    geom = torch.from_numpy(inp["geom"]).to(dev)
    proj, wbuf = D.dark_make_projection(omega, geom, w.H, dt)
    if flags is None:
        flags = D.DARK_CAUSAL if w.causal else 0
    B, H, L, d = inp["q"].shape
    qkv_strides = None
    if strided:
        # q, k, v interleaved as [B][L][3][H][d] (a fused projection's layout)
        packed = torch.empty(B, L, 3, H, d, dtype=tdt, device=dev)
        for i, nm in enumerate(("q", "k", "v")):
            packed[:, :, i] = to_dev(inp[nm], tdt, dev).permute(0, 2, 1, 3)
        q, k, v = packed[:, :, 0], packed[:, :, 1], packed[:, :, 2]
        qkv_strides = (L * 3 * H * d, d, 3 * H * d)
        out = torch.empty(B, L, H, d, dtype=tdt, device=dev)
        out_strides = (L * H * d, d, H * d)
    else:
        q, k, v = (to_dev(inp[nm], tdt, dev) for nm in ("q", "k", "v"))
        out = torch.full((B, H, L, d), float("nan"), dtype=tdt, device=dev)
        out_strides = None
    mask = None if inp["mask"] is None else torch.from_numpy(inp["mask"]).to(dev)
    st, st_t = (None, None)
    if with_state:
        st, st_t = D.make_state(proj, B, H, dev, stabilised=bool(flags & D.DARK_STABILISE))
    if ws is None:
        ws = D.alloc_workspace(proj, B, H, L, flags, dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    D.dark_attention_fwd(proj, q, k, v, out, B, H, L, key_mask=mask, flags=flags, state_out=st,
                         ws=ws, dev_status=status, qkv_strides=qkv_strides,
                         out_strides=out_strides)
    torch.cuda.synchronize()
    o = out.permute(0, 2, 1, 3) if strided else out
    res = dict(out=o.double().cpu().numpy(), status=int(status.item()), proj=proj, wbuf=wbuf,
               ws=ws, state=st)
    if with_state:
        res["kv"] = st_t[0].double().cpu().numpy()
        res["z"] = st_t[1].double().cpu().numpy()
        res["shift"] = None if st_t[2] is None else st_t[2].double().cpu().numpy()
        res["state_tensors"] = st_t
    return res


def rel_err_per_head(got, ref):
    """max |g - o| / max |o| over each (b, h)."""
    B, H = ref.shape[:2]
    worst = 0.0
    for b in range(B):
        for h in range(H):
            den = np.abs(ref[b, h]).max()
            worst = max(worst, np.abs(got[b, h] - ref[b, h]).max() / max(den, 1e-30))
    return worst


def check(w: synth.Workload, got, ref):
    """Tolerances: fp32 I/O max relative error <= 1e-4 (per head, normalised by
    max |out|); bf16 I/O max absolute error <= 2e-2 on unit-variance V."""
    assert np.all(np.isfinite(got))
    if w.dtype == "f32":
        err = rel_err_per_head(got, ref)
        assert err <= 1e-4, f"fp32 relative error {err:.3e}"
    else:
        err = np.abs(got - ref).max()
        assert err <= 2e-2, f"bf16 absolute error {err:.3e}"
    return err
