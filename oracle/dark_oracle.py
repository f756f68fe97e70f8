"""fp64 CPU oracle for DARKformer positive-random-feature (PRF) attention.

TEST INFRASTRUCTURE ONLY. Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / reference legs of ``bench.py`` may import or run this module.
The product path (the C-ABI library and its Python binding) never calls it, and
this module imports nothing from the product: it shares no code with the CUDA
path. Inputs arrive as plain arrays; the random projection Omega is an input.

Source of every formula: the DARKformer README ("Data-Aware Random Feature
Kernels for Transformers", darkformer-pytorch 0.1.0 package description):

* section "Kernel": Sigma = M^T M, kappa(q, k) = exp(q^T Sigma k); the public
  modules scale both q and k by d_h^{-1/4}; the positive random feature map is
  phi(x; omega_j) = m^{-1/2} exp(omega_j^T M x - 1/2 x^T Sigma x) with
  omega_j ~ N(0, I); attention is Phi(Q)(Phi(K)^T V) / Phi(Q)(Phi(K)^T 1).
* section "Self-attention": a boolean B x L mask marks valid tokens; in causal
  attention a key must be both valid and not later than the query.
* section "Encoder-decoder model and generation": in linear mode the prompt is
  processed once and recurrent statistics (Phi(K)^T V, Phi(K)^T 1) are then
  updated per appended token; decoder cross-attention summarises the encoded
  source once per layer.
* section "Cross-attention": queries attend over a separate context; query and
  context masks are separate; there is no causal option.

Readings where the pages are silent (each is listed with its reason in the
design notes of this repository):

* omega_j lives in R^r (it multiplies M x, and M is r x d).
* "x" inside phi is the d^{-1/4}-scaled vector.
* causal attention includes the diagonal (key i is visible to query i).
* the mask acts on keys only; a query row with no visible valid key has a zero
  denominator and its output is defined as 0.
* decode: the new key/value pair is added to the state first, then the output
  for the new query is emitted (the same inclusive rule as causal prefill).
* cross-attention: the context mask drops context positions; a masked query
  row outputs 0 (the pages do not say what the query mask does).

Everything is computed in fp64 with plain numpy; bf16/fp32 inputs are upcast
exactly. Parity of every function here is pinned by ``tests/test_oracle_pins.py``
(Monte Carlo against the closed-form kernel, the Performer special case,
brute-force L x L forms, convexity, invariances, decode consistency and a
hand-derived worked example).
"""
from __future__ import annotations

import numpy as np


def _f64(x) -> np.ndarray:
    return np.asarray(x, dtype=np.float64)


def _head(arr: np.ndarray, h: int) -> np.ndarray:
    """Per-head slice of a [H_x, ...] parameter stack with H_x in {1, H}."""
    return arr[0] if arr.shape[0] == 1 else arr[h]


def kernel_matrix(geom: np.ndarray) -> np.ndarray:
    """Sigma = M^T M (README, "Kernel")."""
    m = _f64(geom)
    return m.T @ m


def feature_map(x, omega, geom) -> np.ndarray:
    """phi_Sigma(x; omega_j) for every row of x (README, "Kernel").

    x: [..., d] unscaled tokens; omega: [m, r]; geom (M): [r, d].
    Returns [..., m] = m^{-1/2} exp(omega_j^T M x~ - 1/2 x~^T Sigma x~),
    with x~ = d^{-1/4} x.
    """
    x = _f64(x)
    omega = _f64(omega)
    geom = _f64(geom)
    d = x.shape[-1]
    m = omega.shape[0]
    xs = x * d ** -0.25
    sigma = kernel_matrix(geom)
    quad = 0.5 * np.einsum("...i,ij,...j->...", xs, sigma, xs)
    lin = (xs @ geom.T) @ omega.T            # omega_j^T (M x~)
    return np.exp(lin - quad[..., None]) / np.sqrt(m)


def feature_exponents(x, omega, geom) -> np.ndarray:
    """The natural-log exponents of feature_map without the m^{-1/2} factor."""
    x = _f64(x)
    d = x.shape[-1]
    xs = x * d ** -0.25
    quad = 0.5 * np.einsum("...i,ij,...j->...", xs, kernel_matrix(geom), xs)
    return (xs @ _f64(geom).T) @ _f64(omega).T - quad[..., None]


def _ratio(num: np.ndarray, den: np.ndarray) -> np.ndarray:
    out = np.zeros_like(num)
    ok = den > 0
    out[ok] = num[ok] / den[ok, None]
    return out


def attention(q, k, v, omega, geom, key_mask=None, causal=False):
    """Full forward pass of PRF attention for every (batch, head).

    q, k, v: [B, H, L, d]; omega: [H_o, m, r]; geom: [H_m, r, d] (H_o, H_m in
    {1, H}); key_mask: [B, L] (nonzero = valid) or None.

    Non-causal (README, "Kernel"): S = Phi(K)^T V and z = Phi(K)^T 1 over the
    valid keys, out = Phi(Q) S / Phi(Q) z.
    Causal (README, "Self-attention" and "generation"): the recurrence in token
    order -- add key i to (S, z) if it is valid, then emit query i.

    Returns (out [B, H, L, d], kv [B, H, m, d], z [B, H, m]) where (kv, z) is
    the state after the last token.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, L, d = q.shape
    m = omega.shape[1]
    out = np.zeros((B, H, L, d))
    kv = np.zeros((B, H, m, d))
    zz = np.zeros((B, H, m))
    for b in range(B):
        valid = np.ones(L, bool) if key_mask is None else np.asarray(key_mask[b]) != 0
        for h in range(H):
            om, gm = _head(omega, h), _head(geom, h)
            phq = feature_map(q[b, h], om, gm)
            phk = feature_map(k[b, h], om, gm) * valid[:, None]
            if not causal:
                s = phk.T @ v[b, h]
                z = phk.sum(axis=0)
                out[b, h] = _ratio(phq @ s, phq @ z)
            else:
                s = np.zeros((m, d))
                z = np.zeros(m)
                for i in range(L):
                    if valid[i]:
                        s += np.outer(phk[i], v[b, h, i])
                        z += phk[i]
                    den = phq[i] @ z
                    out[b, h, i] = (phq[i] @ s) / den if den > 0 else 0.0
            kv[b, h] = s
            zz[b, h] = z
    return out, kv, zz


def attention_rows(q, k, v, omega, geom, key_mask, causal, b, h, rows):
    """Selected output rows of one (batch, head), each from its own definition.

    out_i = sum_j kappa_hat(q_i, k_j) v_j / sum_j kappa_hat(q_i, k_j), where
    kappa_hat(q, k) = phi(q) . phi(k) and j runs over the valid keys (j <= i
    when causal). Used to check large workloads on sampled rows.
    """
    om, gm = _head(omega, h), _head(geom, h)
    kk = _f64(k[b, h])
    vv = _f64(v[b, h])
    L = kk.shape[0]
    valid = np.ones(L, bool) if key_mask is None else np.asarray(key_mask[b]) != 0
    phk = feature_map(kk, om, gm)
    res = np.zeros((len(rows), vv.shape[1]))
    for n, i in enumerate(rows):
        phq = feature_map(_f64(q[b, h, i]), om, gm)
        sel = valid.copy()
        if causal:
            sel[i + 1:] = False
        w = phk[sel] @ phq
        den = w.sum()
        res[n] = (w @ vv[sel]) / den if den > 0 else 0.0
    return res


def decode_step(kv, z, q_t, k_t, v_t, omega, geom, valid=None):
    """One streaming decode step for every (batch, head).

    kv: [B, H, m, d], z: [B, H, m] (the recurrent statistics Phi(K)^T V and
    Phi(K)^T 1); q_t, k_t, v_t: [B, H, d]; valid: [B] or None.
    The new key is added first (if valid), then the output is emitted.
    Returns (out_t [B, H, d], kv', z').
    """
    kv = _f64(kv).copy()
    z = _f64(z).copy()
    q_t, k_t, v_t = _f64(q_t), _f64(k_t), _f64(v_t)
    B, H, d = q_t.shape
    out = np.zeros((B, H, d))
    for b in range(B):
        ok = True if valid is None else bool(valid[b])
        for h in range(H):
            om, gm = _head(omega, h), _head(geom, h)
            if ok:
                pk = feature_map(k_t[b, h], om, gm)
                kv[b, h] += np.outer(pk, v_t[b, h])
                z[b, h] += pk
            pq = feature_map(q_t[b, h], om, gm)
            den = pq @ z[b, h]
            out[b, h] = (pq @ kv[b, h]) / den if den > 0 else 0.0
    return out, kv, z


def cross_attention(q, k, v, omega, geom, query_mask=None, context_mask=None):
    """Cross-attention of queries over a separate context (README,
    "Cross-attention": separate query and context masks, no causal option).

    q: [B, H, Lq, d]; k, v: [B, H, Lk, d]; query_mask: [B, Lq]; context_mask:
    [B, Lk] (nonzero = valid, None = all valid). out_i = sum_j kappa_hat(q_i, k_j)
    v_j / sum_j kappa_hat(q_i, k_j) over the valid context positions j, written
    out pair by pair; a masked query row, or one whose denominator is zero,
    outputs 0. Returns (out [B, H, Lq, d], kv [B, H, m, d], z [B, H, m]), the
    context summary Phi(K)^T V and Phi(K)^T 1 that a decoder reuses at every step.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, Lq, d = q.shape
    Lk = k.shape[2]
    m = omega.shape[1]
    out = np.zeros((B, H, Lq, d))
    kv = np.zeros((B, H, m, d))
    zz = np.zeros((B, H, m))
    for b in range(B):
        ctx = np.ones(Lk, bool) if context_mask is None else np.asarray(context_mask[b]) != 0
        qry = np.ones(Lq, bool) if query_mask is None else np.asarray(query_mask[b]) != 0
        for h in range(H):
            om, gm = _head(omega, h), _head(geom, h)
            phq = feature_map(q[b, h], om, gm)
            phk = feature_map(k[b, h], om, gm)
            for i in range(Lq):
                if not qry[i]:
                    continue
                num = np.zeros(d)
                den = 0.0
                for j in range(Lk):
                    if ctx[j]:
                        w = float(phq[i] @ phk[j])
                        num += w * v[b, h, j]
                        den += w
                out[b, h, i] = num / den if den > 0 else 0.0
            kv[b, h] = (phk * ctx[:, None]).T @ v[b, h]
            zz[b, h] = (phk * ctx[:, None]).sum(axis=0)
    return out, kv, zz


def cross_decode_step(kv, z, q_t, omega, geom):
    """One decoder step of cross-attention against a fixed context summary
    (README, "Encoder-decoder model and generation": each layer's decoder reuses
    one summary of the encoder output): out_t = phi(q_t)^T kv / phi(q_t)^T z; the
    summary is not changed. q_t: [B, H, d]; kv: [B, H, m, d]; z: [B, H, m]."""
    kv, z, q_t = _f64(kv), _f64(z), _f64(q_t)
    B, H, d = q_t.shape
    out = np.zeros((B, H, d))
    for b in range(B):
        for h in range(H):
            pq = feature_map(q_t[b, h], _head(omega, h), _head(geom, h))
            den = pq @ z[b, h]
            out[b, h] = (pq @ kv[b, h]) / den if den > 0 else 0.0
    return out


def exponent_range(x, omega, geom):
    """(min, max) natural-log exponent of phi over x, m^{-1/2} included."""
    e = feature_exponents(x, omega, geom) - 0.5 * np.log(np.asarray(omega).shape[0])
    return float(e.min()), float(e.max())


def attention_backward(q, k, v, omega, geom, dout, key_mask=None, causal=False):
    """Gradients of sum(dout * attention(q, k, v, omega, geom, key_mask, causal))
    with respect to q, k, v and the geometry M (README, "Kernel": M is the
    learned factor of Sigma = M^T M; Omega is a fixed draw and gets none).

    The chain rule of the forward above, step by step for each (batch, head):
      S_i, z_i  = the key statistics query i sees (all valid keys, or the
                  valid keys j <= i when causal);
      num_i = phi(q_i) S_i, den_i = phi(q_i) . z_i, o_i = num_i / den_i;
      w_i = g_i / den_i, c_i = (g_i . o_i) / den_i (zero when den_i = 0);
      dphi(q_i) = S_i w_i - z_i c_i;
      dS_j = sum over the queries i that see key j of phi(q_i) w_i^T,
      dz_j = -sum of phi(q_i) c_i over the same queries;
      dv_j = dS_j^T phi(k_j), dphi(k_j) = dS_j v_j + dz_j (valid keys only).
    Through phi(x)_j = m^{-1/2} exp(omega_j . u - |u|^2 / 2), u = M x~, x~ = d^{-1/4} x:
      a_j = dphi_j phi_j;  du = Omega^T a - (sum_j a_j) u;
      dx = d^{-1/4} M^T du;  dM += du x~^T.
    q, k, v, dout: [B, H, L, d]; omega: [H_o, m, r]; geom: [H_m, r, d].
    Returns (dq, dk, dv [B, H, L, d], dgeom [H_m, r, d]), dgeom summed over
    batches and over the heads that share it.
    """
    q, k, v, g_all = _f64(q), _f64(k), _f64(v), _f64(dout)
    omega, geom = _f64(omega), _f64(geom)
    B, H, L, d = q.shape
    m = omega.shape[1]
    s = d ** -0.25
    dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    dgeom = np.zeros_like(geom)
    for b in range(B):
        valid = np.ones(L, bool) if key_mask is None else np.asarray(key_mask[b]) != 0
        for h in range(H):
            om, gm = _head(omega, h), _head(geom, h)
            phq = feature_map(q[b, h], om, gm)
            phk = feature_map(k[b, h], om, gm) * valid[:, None]
            vv, g = v[b, h], g_all[b, h]
            contrib = np.einsum("jf,je->jfe", phk, vv)          # phi(k_j) v_j^T
            if causal:
                S = np.cumsum(contrib, axis=0)                  # S_i over keys j <= i
                z = np.cumsum(phk, axis=0)
            else:
                S = np.broadcast_to(contrib.sum(axis=0), (L, m, d))
                z = np.broadcast_to(phk.sum(axis=0), (L, m))
            num = np.einsum("if,ife->ie", phq, S)
            den = np.einsum("if,if->i", phq, z)
            ok = den > 0
            safe = np.where(ok, den, 1.0)
            o = np.where(ok[:, None], num / safe[:, None], 0.0)
            w = np.where(ok[:, None], g / safe[:, None], 0.0)
            c = np.where(ok, np.einsum("ie,ie->i", g, o) / safe, 0.0)
            dphq = np.einsum("ife,ie->if", S, w) - z * c[:, None]
            gq = np.einsum("if,ie->ife", phq, w)                # phi(q_i) w_i^T
            gz = -phq * c[:, None]
            if causal:
                # key j is seen by the queries i >= j: suffix sums
                dS = np.cumsum(gq[::-1], axis=0)[::-1]
                dz = np.cumsum(gz[::-1], axis=0)[::-1]
            else:
                dS = np.broadcast_to(gq.sum(axis=0), (L, m, d))
                dz = np.broadcast_to(gz.sum(axis=0), (L, m))
            dv[b, h] = np.einsum("jfe,jf->je", dS, phk) * valid[:, None]
            dphk = (np.einsum("jfe,je->jf", dS, vv) + dz) * valid[:, None]
            ghm = np.zeros_like(gm)
            for x, dph, ph, dst in ((q[b, h], dphq, phq, dq), (k[b, h], dphk, phk, dk)):
                xs = x * s
                u = xs @ gm.T
                a = dph * ph
                du = a @ om - a.sum(axis=1, keepdims=True) * u
                dst[b, h] = s * (du @ gm)
                ghm += du.T @ xs
            dgeom[0 if geom.shape[0] == 1 else h] += ghm
    return dq, dk, dv, dgeom


def exact_attention(q, k, v, geom, key_mask=None, causal=False, query_mask=None):
    """The learned kernel evaluated exactly (README, "Attention modes": in the
    exact mode M acts on queries and keys and ordinary softmax attention with
    scaled scores follows): out_i = sum_j softmax_j(u_i . w_j) v_j with u = M q~, w = M k~,
    x~ = d^{-1/4} x, so the scores are q^T Sigma k / sqrt(d), over the valid keys
    (and j <= i when causal). A row with no visible key, or a masked query row,
    outputs 0.

    q: [B, H, Lq, d]; k, v: [B, H, Lk, d] (Lk = Lq when causal); geom: [H_m, r, d];
    key_mask: [B, Lk] or None; query_mask: [B, Lq] or None.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, Lq, d = q.shape
    Lk = k.shape[2]
    out = np.zeros((B, H, Lq, d))
    s = d ** -0.25
    for b in range(B):
        valid = np.ones(Lk, bool) if key_mask is None else np.asarray(key_mask[b]) != 0
        live = np.ones(Lq, bool) if query_mask is None else np.asarray(query_mask[b]) != 0
        for h in range(H):
            gm = _f64(_head(geom, h))
            u = (q[b, h] * s) @ gm.T
            w = (k[b, h] * s) @ gm.T
            scores = u @ w.T
            keep = np.broadcast_to(valid[None, :], (Lq, Lk)).copy()
            if causal:
                keep &= np.tril(np.ones((Lq, Lk), bool))
            for i in range(Lq):
                if not live[i] or not keep[i].any():
                    continue
                z = scores[i][keep[i]]
                p = np.exp(z - z.max())
                out[b, h, i] = (p / p.sum()) @ v[b, h][keep[i]]
    return out


def uses_exact(L: int, exact_threshold: int) -> bool:
    """Auto mode (README, "Attention modes"): the exact mode for sequences up
    to the threshold length, random features for longer ones."""
    return exact_threshold > 0 and L <= exact_threshold
