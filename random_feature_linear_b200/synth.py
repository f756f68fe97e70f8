"""Seeded synthetic inputs for DARKformer random-feature attention.

This module only draws random numbers and lays them out. It holds none of the
method's arithmetic (no feature map, no projection product, no attention), so
both the fp64 CPU oracle and the CUDA path can consume its arrays without
sharing any computation.

The random projection Omega is drawn here and handed to both sides as an input:
the DARKformer README (section "Self-attention") names two families,
independent Gaussian features (``orthogonal_features=False``) and the default
orthogonal Gaussian blocks; the README (section "Kernel") fixes
omega_j ~ N(0, I) in R^r.

Seeds: every tensor of workload ``cfg`` comes from
``numpy.random.default_rng(1000 * cfg + tid)`` with tid = 1 Omega, 2 M,
3 Q, 4 K, 5 V, 6 the decode token stream. All draws are fp64, cast to fp32,
then rounded to bfloat16 (round-to-nearest-even) for bf16 workloads.
"""
from __future__ import annotations

import dataclasses
import numpy as np

TID_OMEGA, TID_GEOM, TID_Q, TID_K, TID_V, TID_STREAM, TID_GRAD = 1, 2, 3, 4, 5, 6, 7


@dataclasses.dataclass(frozen=True)
class Workload:
    """Shape and distribution recipe of one synthetic workload."""
    cfg: int
    name: str
    B: int
    H: int
    L: int
    d: int
    r: int
    m: int
    dtype: str                 # "f32" or "bf16": the I/O type of q, k, v, out
    causal: bool
    features: str              # "iid" or "orthogonal"
    geom: str                  # "identity+noise" or "gaussian"
    geom_sigma: float          # std of the noise (identity+noise) or of the entries
    per_head_geom: bool        # one M per head (True) or one shared M (False)
    qk: str                    # "normal" or "anisotropic"
    qk_scale: tuple = (1.0, 1.0)   # (lo, hi) of the log-spaced per-dim scales
    lengths: tuple | None = None   # valid length per batch row (tail padded); None = all valid
    decode_steps: int = 0

    @property
    def tokens(self) -> int:
        return self.B * self.H * self.L

    def with_sizes(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS = {
    1: Workload(1, "tiny non-causal fp32 (B1 H1 L256 d64 r64 m64, iid features)",
                B=1, H=1, L=256, d=64, r=64, m=64, dtype="f32", causal=False,
                features="iid", geom="identity+noise", geom_sigma=0.1,
                per_head_geom=False, qk="normal"),
    2: Workload(2, "causal masked bf16 (B2 H8 L2048 d64 r64 m256, lengths 2048/1500)",
                B=2, H=8, L=2048, d=64, r=64, m=256, dtype="bf16", causal=True,
                features="orthogonal", geom="identity+noise", geom_sigma=0.05,
                per_head_geom=True, qk="normal", lengths=(2048, 1500)),
    3: Workload(3, "long non-causal bf16 (B1 H16 L16384 d64 r32 shared M, m256)",
                B=1, H=16, L=16384, d=64, r=32, m=256, dtype="bf16", causal=False,
                features="orthogonal", geom="gaussian", geom_sigma=1.0 / 8.0,
                per_head_geom=False, qk="anisotropic", qk_scale=(0.1, 3.0)),
    4: Workload(4, "large-head causal bf16 (B4 H8 L8192 d256 r256 m512)",
                B=4, H=8, L=8192, d=256, r=256, m=512, dtype="bf16", causal=True,
                features="orthogonal", geom="identity+noise", geom_sigma=0.02,
                per_head_geom=True, qk="anisotropic", qk_scale=(0.05, 3.0)),
    5: Workload(5, "streaming decode bf16 I/O, fp32 state (B64 H8 d64 r64 m256, 4096 prefill + 1024 steps)",
                B=64, H=8, L=4096, d=64, r=64, m=256, dtype="bf16", causal=True,
                features="orthogonal", geom="identity+noise", geom_sigma=0.05,
                per_head_geom=True, qk="normal", decode_steps=1024),
}


def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to the nearest bfloat16 (ties to even); returns fp32."""
    a = np.ascontiguousarray(x, dtype=np.float32)
    u = a.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000
    return u.astype(np.uint32).view(np.float32).reshape(a.shape)


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """The upper 16 bits of fp32 values that are already bf16-representable."""
    a = np.ascontiguousarray(x, dtype=np.float32)
    return (a.view(np.uint32) >> 16).astype(np.uint16)


def _rng(w: Workload, tid: int, salt: int = 0) -> np.random.Generator:
    return np.random.default_rng(1000 * w.cfg + tid + 100_000 * salt)


def draw_omega(rng: np.random.Generator, m: int, r: int, kind: str) -> np.ndarray:
    """m x r feature matrix: iid N(0,1) rows, or stacked orthogonal blocks.

    Orthogonal blocks: for each block of r rows draw G ~ N(0,1)^{r x r}, take its
    QR factorisation, fix the column signs with sign(diag R) (Haar measure),
    and give each row the norm of a fresh N(0, I_r) vector (a chi(r) draw), so
    that every row is still marginally N(0, I_r). A final partial block keeps
    its first rows.
    """
    if kind == "iid":
        return rng.standard_normal((m, r))
    if kind != "orthogonal":
        raise ValueError(kind)
    blocks = []
    for _ in range((m + r - 1) // r):
        g = rng.standard_normal((r, r))
        qm, rm = np.linalg.qr(g)
        qm = qm * np.sign(np.diag(rm))[None, :]
        norms = np.linalg.norm(rng.standard_normal((r, r)), axis=1)
        blocks.append(qm.T * norms[:, None])     # rows of Q^T are orthonormal
    return np.concatenate(blocks, axis=0)[:m]


def _draw_geom(rng, w: Workload, heads: int) -> np.ndarray:
    if w.geom == "identity+noise":
        eye = np.eye(w.r, w.d)
        return eye[None] + w.geom_sigma * rng.standard_normal((heads, w.r, w.d))
    if w.geom == "gaussian":
        return w.geom_sigma * rng.standard_normal((heads, w.r, w.d))
    raise ValueError(w.geom)


def _draw_qk(rng, w: Workload, shape) -> np.ndarray:
    g = rng.standard_normal(shape)
    if w.qk == "normal":
        return g
    s = np.geomspace(w.qk_scale[0], w.qk_scale[1], w.d)   # both endpoints, dimension order
    return g * s


def _io(w: Workload, x: np.ndarray) -> np.ndarray:
    x32 = x.astype(np.float32)
    return round_bf16(x32) if w.dtype == "bf16" else x32


def make_inputs(w: Workload, salt: int = 0) -> dict:
    """All inputs of one workload as numpy arrays (fp32; bf16-exact where bf16).

    Returns omega [1, m, r], geom [H_M, r, d], q/k/v [B, H, L, d] and
    mask [B, L] uint8 (1 = valid) or None.
    """
    omega = draw_omega(_rng(w, TID_OMEGA, salt), w.m, w.r, w.features)[None].astype(np.float32)
    geom = _draw_geom(_rng(w, TID_GEOM, salt), w, w.H if w.per_head_geom else 1).astype(np.float32)
    shape = (w.B, w.H, w.L, w.d)
    q = _io(w, _draw_qk(_rng(w, TID_Q, salt), w, shape))
    k = _io(w, _draw_qk(_rng(w, TID_K, salt), w, shape))
    v = _io(w, _rng(w, TID_V, salt).standard_normal(shape))
    mask = None
    if w.lengths is not None:
        if len(w.lengths) != w.B:
            raise ValueError("one valid length per batch row")
        mask = np.zeros((w.B, w.L), np.uint8)
        for b, n in enumerate(w.lengths):
            mask[b, :n] = 1
    return dict(omega=omega, geom=geom, q=q, k=k, v=v, mask=mask)


def make_cotangent(w: Workload, salt: int = 0) -> np.ndarray:
    """Upstream gradient dout ~ N(0, 1) of the attention output, [B, H, L, d]
    (bf16-exact where the workload's I/O is bf16)."""
    return _io(w, _rng(w, TID_GRAD, salt).standard_normal((w.B, w.H, w.L, w.d)))


def decode_stream(w: Workload, steps: int, salt: int = 0) -> dict:
    """Token stream for the decode workload: q_t, k_t, v_t ~ N(0,1), [steps, B, H, d]."""
    rng = _rng(w, TID_STREAM, salt)
    shape = (steps, w.B, w.H, w.d)
    q = _io(w, rng.standard_normal(shape))
    k = _io(w, rng.standard_normal(shape))
    v = _io(w, rng.standard_normal(shape))
    return dict(q=q, k=k, v=v)
