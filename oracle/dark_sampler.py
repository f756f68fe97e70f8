"""fp64 CPU oracle of the projection sampler: Omega drawn from a counter-based
generator, independent Gaussian features or orthogonal Gaussian blocks, and the
redraw lifecycle.

TEST INFRASTRUCTURE ONLY. Only ``tests/`` and ``__graft_entry__.smoke()`` may
import or run this module; it imports nothing from the product and shares no
code with the CUDA path.

Sources:
* DARKformer README ("Data-Aware Random Feature Kernels for Transformers"),
  section "Self-attention": ``orthogonal_features`` chooses orthogonal Gaussian
  blocks (default) or independent Gaussian features; omega_j ~ N(0, I) (section
  "Kernel"). Section "Projection lifecycle": a projection is kept until it is
  redrawn; with a redraw interval a new draw falls due once that many training
  forwards have run, and forwards outside training are not counted; a fixed
  projection refuses redraws unless one is forced; a seed reproduces the draws.
* Philox4x64-10: Salmon, Moraes, Dror and Shaw, "Parallel random numbers: as easy
  as 1, 2, 3" (SC 2011): ten rounds of two 64 x 64 -> 128-bit multiplies with the
  round constants below and a Weyl-sequence key schedule.
* Box-Muller (1958): two uniforms give two independent N(0, 1) values.

The sampler's layout (a library choice; the pages fix no generator):
* key = (seed, draw): draw counts the redraws of one projection;
* the Gaussian stream of head h and purpose s (0: the features or the block
  matrices G, 1: the vectors whose norms scale the orthogonal rows) has element e
  from word e % 4 of Philox block counter (e // 4, h, s, 0); words (0, 1) and
  (2, 3) form Box-Muller pairs with u1 = 1 - u(x_a), u2 = u(x_b), u(x) =
  (x >> 11) * 2^-53;
* independent features: Omega_h[j, i] = z(h, 0, j r + i);
* orthogonal blocks: block b is G[i, k] = z(h, 0, b r^2 + i r + k); its QR
  factorisation with a positive diagonal of R gives Q; row i of the block is
  ||(z(h, 1, b r^2 + i r + k))_k|| * Q[:, i]; a final partial block keeps its
  first rows.
"""
from __future__ import annotations

import math

import numpy as np

MASK64 = (1 << 64) - 1
PHILOX_M = (0xD2E7470EE14C6C93, 0xCA5A826395121157)
PHILOX_W = (0x9E3779B97F4A7C15, 0xBB67AE8584CAA73B)


def philox4x64(counter, key, rounds: int = 10) -> list[int]:
    """One Philox4x64 block: four 64-bit words from a 4-word counter and 2-word key."""
    c0, c1, c2, c3 = (int(x) & MASK64 for x in counter)
    k0, k1 = (int(x) & MASK64 for x in key)
    for _ in range(rounds):
        p0 = PHILOX_M[0] * c0
        p1 = PHILOX_M[1] * c2
        c0, c1, c2, c3 = ((p1 >> 64) ^ c1 ^ k0) & MASK64, p1 & MASK64, \
                         ((p0 >> 64) ^ c3 ^ k1) & MASK64, p0 & MASK64
        k0 = (k0 + PHILOX_W[0]) & MASK64
        k1 = (k1 + PHILOX_W[1]) & MASK64
    return [c0, c1, c2, c3]


def uniform53(x: int) -> float:
    """[0, 1) from the top 53 bits of a 64-bit word."""
    return (x >> 11) * 2.0 ** -53


def gaussians(seed: int, draw: int, head: int, purpose: int, n: int) -> np.ndarray:
    """The first n values of the Gaussian stream (seed, draw, head, purpose)."""
    out = np.empty(((n + 3) // 4) * 4)
    for blk in range((n + 3) // 4):
        x = philox4x64((blk, head, purpose, 0), (seed, draw))
        for p in range(2):
            u1 = 1.0 - uniform53(x[2 * p])
            u2 = uniform53(x[2 * p + 1])
            rho = math.sqrt(-2.0 * math.log(u1))
            out[4 * blk + 2 * p] = rho * math.cos(2.0 * math.pi * u2)
            out[4 * blk + 2 * p + 1] = rho * math.sin(2.0 * math.pi * u2)
    return out[:n]


def sample_omega(seed: int, draw: int, heads: int, m: int, r: int,
                 orthogonal: bool) -> np.ndarray:
    """Omega [heads, m, r] in fp64 (the CUDA sampler rounds it to fp32)."""
    omega = np.empty((heads, m, r))
    nblk = (m + r - 1) // r
    for h in range(heads):
        if not orthogonal:
            omega[h] = gaussians(seed, draw, h, 0, m * r).reshape(m, r)
            continue
        g_all = gaussians(seed, draw, h, 0, nblk * r * r).reshape(nblk, r, r)
        n_all = gaussians(seed, draw, h, 1, nblk * r * r).reshape(nblk, r, r)
        rows = []
        for b in range(nblk):
            q, rr = np.linalg.qr(g_all[b])
            q = q * np.sign(np.diag(rr))[None, :]      # the factorisation with diag(R) > 0
            norms = np.linalg.norm(n_all[b], axis=1)
            rows.append(q.T * norms[:, None])
        omega[h] = np.concatenate(rows, axis=0)[:m]
    return omega


class RedrawSchedule:
    """The projection lifecycle of the README's "Projection lifecycle" section.

    interval None: no scheduled redraws. With a positive interval a redraw falls
    due once that many training forwards have run; it happens at the start of the
    next training forward, which uses the new draw. Forwards outside training are
    not counted. While fixed, a scheduled
    redraw that falls due is dropped (the interval restarts) and ordinary manual
    redraws are ignored; a forced manual redraw happens once. Any redraw restarts
    the interval. ``deterministic`` fixes the projection at construction.
    """

    def __init__(self, seed: int, interval: int | None = None, deterministic: bool = False):
        self.seed = seed
        self.draw = 0
        self.interval = interval
        self.count = 0
        self.fixed = deterministic

    def forward(self, training: bool) -> bool:
        """Called at the start of a forward; True if a redraw happened first."""
        redrew = False
        if training and self.interval is not None and self.count >= self.interval:
            self.count = 0
            if not self.fixed:
                self.draw += 1
                redrew = True
        if training:
            self.count += 1
        return redrew

    def redraw(self, force: bool = False) -> bool:
        if self.fixed and not force:
            return False
        self.draw += 1
        self.count = 0
        return True

    def fix(self) -> None:
        self.fixed = True

    def unfix(self) -> None:
        self.fixed = False
