"""Pins of the fp64 oracle against what the DARKformer README and mathematics fix.

None of these re-types the oracle's formula and compares it with itself. Each
pin checks the oracle against an independent fact:

* the closed-form kernel the features estimate, exp(q^T Sigma k / sqrt(d_h))
  (README "Kernel"), with the Gaussian moment generating function giving the
  estimator's exact variance;
* Performer positive features, the special case M = I (README "Kernel" states
  DARKformer follows the Performer positive feature formulation);
* the explicit L x L form of normalised attention (associativity);
* brute-force causal / masked L x L forms;
* convexity of the output (positive weights);
* the m -> infinity limit, exact softmax attention with the learned kernel;
* invariances and decode/prefill consistency;
* a hand-derived two-token worked example (tests/golden).

Planted mistakes (mutants of the feature map) must fail the pins.
"""
import json
import os

import numpy as np
import pytest

from oracle import dark_oracle as O
from random_feature_linear_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------- helpers ---

def _closed_form_kernel(q, k, geom):
    """exp(q^T Sigma k / sqrt(d)), Sigma = M^T M -- README "Kernel"."""
    d = q.shape[-1]
    sig = geom.T @ geom
    return np.exp(q @ sig @ k / np.sqrt(d))


def _closed_form_var(q, k, geom):
    """Variance of one feature product X = m phi_j(q) phi_j(k), omega ~ N(0, I).

    With u = M q~, v = M k~ (x~ = d^{-1/4} x): X = exp(omega.(u+v) - |u|^2/2 - |v|^2/2);
    the Gaussian MGF gives E X = exp(u.v), E X^2 = exp(2|u+v|^2 - |u|^2 - |v|^2).
    """
    d = q.shape[-1]
    u = geom @ (q * d ** -0.25)
    v = geom @ (k * d ** -0.25)
    ex2 = np.exp(2 * (u + v) @ (u + v) - u @ u - v @ v)
    return ex2 - np.exp(2 * u @ v)


def mc_pin(feature_fn, seeds=range(8), ms=(64, 256, 1024, 4096, 16384, 65536)):
    """Checks feature_fn against the closed-form kernel. Returns (ok, slope)."""
    rng = np.random.default_rng(7)
    d, r = 6, 6
    geom = np.eye(r, d) + 0.4 * rng.standard_normal((r, d))      # square, non-symmetric
    q = 0.45 * rng.standard_normal(d)
    k = 0.45 * rng.standard_normal(d)
    exact = _closed_form_kernel(q, k, geom)
    sd1 = np.sqrt(_closed_form_var(q, k, geom))
    ok = True
    rms = []
    for m in ms:
        errs = []
        for s in seeds:
            omega = np.random.default_rng(1000 + s).standard_normal((m, r))
            est = feature_fn(q, omega, geom) @ feature_fn(k, omega, geom)
            errs.append(est - exact)
            if abs(est - exact) > 5 * sd1 / np.sqrt(m):
                ok = False
        rms.append(np.sqrt(np.mean(np.square(errs))))
    slope = np.polyfit(np.log(ms), np.log(rms), 1)[0]
    return ok and abs(slope + 0.5) < 0.2, slope


# ------------------------------------------------------------- the pins ---

def test_mc_converges_to_closed_form_kernel():
    ok, slope = mc_pin(O.feature_map)
    assert ok, f"Monte Carlo pin failed (slope {slope:.3f})"


@pytest.mark.parametrize("mutant", [
    "no_half", "plus_norm", "no_dscale", "transposed_sigma", "no_sqrt_m", "scale_sqrt_d"])
def test_planted_mistakes_fail_the_mc_pin(mutant):
    def fm(x, omega, geom):
        x = np.asarray(x, float)
        d = x.shape[-1]
        m = omega.shape[0]
        xs = x * d ** -0.25
        quad_coef = 0.5
        sig = geom.T @ geom
        if mutant == "no_half":
            quad_coef = 1.0
        if mutant == "plus_norm":
            quad_coef = -0.5
        if mutant == "no_dscale":
            xs = x
        if mutant == "scale_sqrt_d":
            xs = x * d ** -0.5
        if mutant == "transposed_sigma":
            sig = geom @ geom.T
        quad = quad_coef * xs @ sig @ xs
        val = np.exp((xs @ geom.T) @ omega.T - quad)
        return val if mutant == "no_sqrt_m" else val / np.sqrt(m)
    ok, _ = mc_pin(fm, seeds=range(3), ms=(4096, 65536))
    assert not ok, f"mutant {mutant} was not caught"


def test_performer_positive_features_special_case():
    # M = I, r = d: Performer's positive random features exp(w^T x - |x|^2 / 2) / sqrt(m)
    # applied to x = d^{-1/4} x_raw.
    rng = np.random.default_rng(3)
    d, m = 16, 40
    omega = rng.standard_normal((m, d))
    x = rng.standard_normal((5, d))
    xs = x / d ** 0.25
    performer = np.exp(xs @ omega.T - 0.5 * np.sum(xs * xs, axis=1, keepdims=True)) / np.sqrt(m)
    got = O.feature_map(x, omega, np.eye(d))
    np.testing.assert_allclose(got, performer, rtol=1e-13, atol=0)


def test_worked_example_golden():
    g = json.load(open(os.path.join(GOLDEN, "two_token_worked_example.json")))
    om = np.array(g["omega"])[None]
    gm = np.array(g["geom"])[None]
    q = np.array(g["q"]).reshape(1, 1, 2, 1)
    k = np.array(g["k"]).reshape(1, 1, 2, 1)
    v = np.array(g["v"]).reshape(1, 1, 2, 1)
    phq = O.feature_map(q[0, 0], om[0], gm[0])
    phk = O.feature_map(k[0, 0], om[0], gm[0])
    np.testing.assert_allclose(phq @ phk.T, np.array(g["weights"]), rtol=1e-14)
    out, _, _ = O.attention(q, k, v, om, gm, causal=False)
    np.testing.assert_allclose(out[0, 0, :, 0], g["out_noncausal"], rtol=1e-14)
    out, _, _ = O.attention(q, k, v, om, gm, causal=True)
    np.testing.assert_allclose(out[0, 0, :, 0], g["out_causal"], rtol=1e-14)
    out, _, _ = O.attention(q, k, v, om, gm, key_mask=np.array([[1, 0]]), causal=False)
    np.testing.assert_allclose(out[0, 0, :, 0], g["out_noncausal_key2_masked"], rtol=1e-14)


def _small(seed=0, B=2, H=3, L=37, d=8, r=5, m=24, per_head=True):
    rng = np.random.default_rng(seed)
    omega = rng.standard_normal((1, m, r))
    geom = np.eye(r, d)[None] + 0.3 * rng.standard_normal((H if per_head else 1, r, d))
    q, k, v = (rng.standard_normal((B, H, L, d)) for _ in range(3))
    mask = (rng.random((B, L)) > 0.3).astype(np.uint8)
    return omega, geom, q, k, v, mask


def _brute(q, k, v, omega, geom, mask, causal):
    """Explicit L x L normalised attention: A = Phi_Q Phi_K^T, masked, row-normalised."""
    B, H, L, d = q.shape
    out = np.zeros_like(q)
    for b in range(B):
        for h in range(H):
            om = omega[0] if omega.shape[0] == 1 else omega[h]
            gm = geom[0] if geom.shape[0] == 1 else geom[h]
            a = O.feature_map(q[b, h], om, gm) @ O.feature_map(k[b, h], om, gm).T
            if mask is not None:
                a = a * (mask[b] != 0)[None, :]
            if causal:
                a = np.tril(a)
            den = a.sum(axis=1)
            good = den > 0
            out[b, h][good] = (a @ v[b, h])[good] / den[good, None]
    return out


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("masked", [False, True])
def test_associative_equals_explicit_lxl(causal, masked):
    omega, geom, q, k, v, mask = _small(seed=int(causal) + 2 * int(masked))
    mask = mask if masked else None
    out, _, _ = O.attention(q, k, v, omega, geom, key_mask=mask, causal=causal)
    ref = _brute(q, k, v, omega, geom, mask, causal)
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-12)


def test_rows_match_full_forward():
    omega, geom, q, k, v, mask = _small(seed=5)
    for causal in (False, True):
        out, _, _ = O.attention(q, k, v, omega, geom, key_mask=mask, causal=causal)
        rows = [0, 3, 17, 36]
        got = O.attention_rows(q, k, v, omega, geom, mask, causal, 1, 2, rows)
        np.testing.assert_allclose(got, out[1, 2, rows], rtol=1e-12, atol=1e-13)


def test_state_is_total_sum_over_valid_keys():
    omega, geom, q, k, v, mask = _small(seed=6)
    for causal in (False, True):
        _, kv, z = O.attention(q, k, v, omega, geom, key_mask=mask, causal=causal)
        for b in range(2):
            for h in range(3):
                phk = O.feature_map(k[b, h], omega[0], geom[h])[mask[b] != 0]
                np.testing.assert_allclose(kv[b, h], phk.T @ v[b, h][mask[b] != 0], rtol=1e-12)
                np.testing.assert_allclose(z[b, h], phk.sum(0), rtol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_convexity(causal):
    omega, geom, q, k, v, mask = _small(seed=9, L=29)
    out, _, _ = O.attention(q, k, v, omega, geom, key_mask=mask, causal=causal)
    for b in range(2):
        for h in range(3):
            for i in range(29):
                sel = mask[b] != 0
                if causal:
                    sel = sel & (np.arange(29) <= i)
                if not sel.any():
                    assert np.all(out[b, h, i] == 0)
                    continue
                lo = v[b, h][sel].min(axis=0) - 1e-12
                hi = v[b, h][sel].max(axis=0) + 1e-12
                assert np.all(out[b, h, i] >= lo) and np.all(out[b, h, i] <= hi)


def test_row_without_valid_key_is_zero():
    omega, geom, q, k, v, mask = _small(seed=10)
    mask[0, :] = 0
    mask[1, :5] = 0
    out, kv, z = O.attention(q, k, v, omega, geom, key_mask=mask, causal=True)
    assert np.all(out[0] == 0) and np.all(kv[0] == 0) and np.all(z[0] == 0)
    assert np.all(out[1, :, :5] == 0)
    assert np.all(np.abs(out[1, :, 5]) > 0)


def test_softmax_limit():
    # m -> infinity: normalised PRF attention -> softmax attention with scores
    # q~^T Sigma k~ = (M q~).(M k~)  (README "Kernel": the estimator approximates kappa).
    rng = np.random.default_rng(11)
    L, d, r = 6, 4, 4
    geom = np.eye(r, d) + 0.2 * rng.standard_normal((r, d))
    q = 0.6 * rng.standard_normal((1, 1, L, d))
    k = 0.6 * rng.standard_normal((1, 1, L, d))
    v = rng.standard_normal((1, 1, L, d))
    s = (q[0, 0] @ geom.T @ geom @ k[0, 0].T) / np.sqrt(d)
    p = np.exp(s - s.max(axis=1, keepdims=True))
    exact = (p / p.sum(axis=1, keepdims=True)) @ v[0, 0]
    errs = []
    for m in (256, 4096, 65536):
        e = []
        for seed in range(4):
            omega = np.random.default_rng(seed).standard_normal((1, m, r))
            out, _, _ = O.attention(q, k, v, omega, geom[None])
            e.append(np.abs(out[0, 0] - exact).max())
        errs.append(np.mean(e))
    assert errs[-1] < 0.03
    assert errs[0] > 4 * errs[-1]


def test_mask_and_permutation_invariance():
    omega, geom, q, k, v, mask = _small(seed=12)
    rng = np.random.default_rng(0)
    for causal in (False, True):
        out, _, _ = O.attention(q, k, v, omega, geom, key_mask=mask, causal=causal)
        k2, v2 = k.copy(), v.copy()
        bad = mask == 0
        for b in range(2):
            k2[b, :, bad[b]] = 50 * rng.standard_normal(k2[b, :, bad[b]].shape)
            v2[b, :, bad[b]] = 1e3
        out2, _, _ = O.attention(q, k2, v2, omega, geom, key_mask=mask, causal=causal)
        np.testing.assert_allclose(out2, out, rtol=1e-12, atol=1e-12)
    perm = rng.permutation(37)
    out, _, _ = O.attention(q, k, v, omega, geom, key_mask=mask)
    out_p, _, _ = O.attention(q, k[:, :, perm], v[:, :, perm], omega, geom, key_mask=mask[:, perm])
    np.testing.assert_allclose(out_p, out, rtol=1e-12, atol=1e-12)


def test_decode_continues_causal_prefill():
    omega, geom, q, k, v, mask = _small(seed=13, L=30)
    T = 22
    full, _, _ = O.attention(q, k, v, omega, geom, key_mask=mask, causal=True)
    _, kv, z = O.attention(q[:, :, :T], k[:, :, :T], v[:, :, :T], omega, geom,
                           key_mask=mask[:, :T], causal=True)
    for t in range(T, 30):
        out_t, kv, z = O.decode_step(kv, z, q[:, :, t], k[:, :, t], v[:, :, t], omega, geom,
                                     valid=mask[:, t])
        np.testing.assert_allclose(out_t, full[:, :, t], rtol=1e-11, atol=1e-12)


def test_orthogonal_blocks_structure_and_unbiasedness():
    rng = np.random.default_rng(21)
    r, m = 8, 20
    om = synth.draw_omega(rng, m, r, "orthogonal")
    assert om.shape == (m, r)
    for blk in (om[:8], om[8:16]):
        g = blk @ blk.T
        np.testing.assert_allclose(g - np.diag(np.diag(g)), 0, atol=1e-10)
    # unbiased estimator of the closed-form kernel, no more spread than iid
    d = r
    geom = np.eye(r) + 0.3 * np.random.default_rng(1).standard_normal((r, d))
    q = 0.4 * np.random.default_rng(2).standard_normal(d)
    k = 0.4 * np.random.default_rng(3).standard_normal(d)
    exact = _closed_form_kernel(q, k, geom)
    mm = 64
    est_o, est_i = [], []
    for s in range(400):
        g = np.random.default_rng(5000 + s)
        omo = synth.draw_omega(g, mm, r, "orthogonal")
        omi = synth.draw_omega(g, mm, r, "iid")
        est_o.append(O.feature_map(q, omo, geom) @ O.feature_map(k, omo, geom))
        est_i.append(O.feature_map(q, omi, geom) @ O.feature_map(k, omi, geom))
    est_o, est_i = np.array(est_o), np.array(est_i)
    assert abs(est_o.mean() - exact) < 5 * est_o.std() / np.sqrt(len(est_o))
    assert est_o.var() <= 1.1 * est_i.var()


def test_synth_bf16_rounding_matches_torch():
    torch = pytest.importorskip("torch")
    x = np.random.default_rng(0).standard_normal(100_000).astype(np.float32) * 37
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float32).numpy()
    np.testing.assert_array_equal(synth.round_bf16(x), ref)


def test_workload_recipes():
    w = synth.WORKLOADS[2].with_sizes(L=64, lengths=(64, 40))
    inp = synth.make_inputs(w)
    assert inp["q"].shape == (2, 8, 64, 64) and inp["geom"].shape == (8, 64, 64)
    assert inp["mask"].sum(axis=1).tolist() == [64, 40]
    np.testing.assert_array_equal(synth.round_bf16(inp["q"]), inp["q"])
    w3 = synth.WORKLOADS[3].with_sizes(L=32)
    inp3 = synth.make_inputs(w3)
    assert inp3["geom"].shape == (1, 32, 64)
    # the per-dim scale grows along d
    sd = inp3["q"].reshape(-1, 64).std(axis=0)
    assert sd[-1] > 10 * sd[0]


def test_exponents_stay_in_range_for_workloads():
    # Overflow check of the feature exponents (natural log) for the five recipes,
    # on a sample of tokens: far from fp32/bf16 overflow (88.7) and underflow.
    for cfg in (1, 2, 3, 4, 5):
        w = synth.WORKLOADS[cfg]
        w = w.with_sizes(L=64, B=1, lengths=None)
        inp = synth.make_inputs(w)
        lo, hi = O.exponent_range(inp["k"][0, 0], inp["omega"][0], inp["geom"][0])
        assert -80 < lo and hi < 40, (cfg, lo, hi)


def test_feature_exponents_hand_values():
    # README, "Kernel": the exponent of phi_j(x) is omega_j^T M x~ - 1/2 |M x~|^2
    # (x~ = d^{-1/4} x) and phi carries the factor m^{-1/2}. Hand-derived cases:
    # (1) the two-token example (d = r = 1, M = 1, Omega = [1; -1]): x = 1 gives
    #     [1 - 1/2, -1 - 1/2], x = -1 gives [-3/2, 1/2], x = -1/2 gives [-5/8, 3/8].
    g = json.load(open(os.path.join(GOLDEN, "two_token_worked_example.json")))
    om, gm = np.array(g["omega"]), np.array(g["geom"])
    x = np.array([[1.0], [-1.0], [-0.5]])
    e = O.feature_exponents(x, om, gm)
    np.testing.assert_allclose(e, [[0.5, -1.5], [-1.5, 0.5], [-0.625, 0.375]], atol=1e-15)
    lo, hi = O.exponent_range(x, om, gm)
    assert abs(lo - (-1.5 - 0.5 * np.log(2))) < 1e-15 and abs(hi - (0.5 - 0.5 * np.log(2))) < 1e-15
    # (2) d = r = 4 so that d^{-1/4} = 2^{-1/2} matters, M = 2 I: x = (sqrt 2, 0, 0, 0)
    #     gives x~ = e_1, M x~ = 2 e_1 and 1/2 |M x~|^2 = 2; omega = e_1, e_2, -e_1
    #     and 3 e_1 + e_4 give exponents 2 - 2, 0 - 2, -2 - 2 and 6 - 2.
    om4 = np.array([[1.0, 0, 0, 0], [0, 1.0, 0, 0], [-1.0, 0, 0, 0], [3.0, 0, 0, 1.0]])
    x4 = np.array([[np.sqrt(2.0), 0, 0, 0]])
    e4 = O.feature_exponents(x4, om4, 2.0 * np.eye(4))
    np.testing.assert_allclose(e4, [[0.0, -2.0, -4.0, 4.0]], atol=1e-14)
    lo4, hi4 = O.exponent_range(x4, om4, 2.0 * np.eye(4))
    assert abs(lo4 - (-4.0 - np.log(2))) < 1e-14 and abs(hi4 - (4.0 - np.log(2))) < 1e-14
    # (3) low rank, r = 2 < d = 4: M x~ keeps two coordinates only
    gm2 = np.array([[1.0, 1.0, 0, 0], [0, 0, 2.0, 0]])
    x2 = np.array([[2.0, 0.0, 1.0, 5.0]]) * np.sqrt(2.0)      # x~ = (2, 0, 1, 5)
    om2 = np.array([[1.0, 0.0], [0.0, -1.0]])
    # M x~ = (2, 2), 1/2 |M x~|^2 = 4; exponents 2 - 4 and -2 - 4
    np.testing.assert_allclose(O.feature_exponents(x2, om2, gm2), [[-2.0, -6.0]], atol=1e-14)


def test_feature_exponents_agree_with_feature_map():
    # exponent_range bounds log(phi) itself: the log of the pinned feature map
    # (times sqrt(m) for the exponents) on random recipes, with per-head geometry
    rng = np.random.default_rng(11)
    for d, r, m in ((64, 64, 256), (64, 32, 128), (16, 8, 8)):
        x = rng.standard_normal((50, d))
        om = rng.standard_normal((m, r))
        gm = np.eye(r, d) + 0.1 * rng.standard_normal((r, d))
        phi = O.feature_map(x, om, gm)
        np.testing.assert_allclose(O.feature_exponents(x, om, gm), np.log(phi * np.sqrt(m)),
                                   rtol=0, atol=1e-12)
        lo, hi = O.exponent_range(x, om, gm)
        assert abs(lo - np.log(phi).min()) < 1e-12 and abs(hi - np.log(phi).max()) < 1e-12
