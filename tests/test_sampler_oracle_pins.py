"""Pins of the oracle's projection sampler against what fixes it independently:
numpy's own Philox4x64-10 bit generator, the normal distribution, the algebra of
the QR factorisation, and the lifecycle rules of the README's "Projection
lifecycle" section."""
import numpy as np
from scipy import stats

from oracle import dark_sampler as S


def test_philox_matches_numpy_bit_generator():
    # numpy's Philox advances its counter before each block: block n of numpy's
    # stream is the function at counter n + 1
    for key in ((7, 3), (0, 0), (2**64 - 1, 12345), (0xDEADBEEF, 2**63)):
        bg = np.random.Philox(key=np.array(key, dtype=np.uint64),
                              counter=np.array([0, 0, 0, 0], dtype=np.uint64))
        raw = bg.random_raw(4 * 6)
        for n in range(6):
            assert S.philox4x64((n + 1, 0, 0, 0), key) == [int(x) for x in raw[4 * n:4 * n + 4]]
    # higher counter words: numpy carries into them
    start = [2**64 - 2, 5, 9, 1]
    bg = np.random.Philox(key=np.array([1, 2], dtype=np.uint64),
                          counter=np.array(start, dtype=np.uint64))
    raw = bg.random_raw(8)
    assert S.philox4x64((2**64 - 1, 5, 9, 1), (1, 2)) == [int(x) for x in raw[:4]]
    assert S.philox4x64((0, 6, 9, 1), (1, 2)) == [int(x) for x in raw[4:8]]


def test_uniform_range():
    assert S.uniform53(0) == 0.0
    assert S.uniform53(2**64 - 1) == 1.0 - 2.0 ** -53


def test_gaussian_stream_is_standard_normal():
    z = S.gaussians(11, 0, 0, 0, 40000)
    assert stats.kstest(z, "norm").pvalue > 1e-3
    assert abs(z.mean()) < 4 / np.sqrt(z.size)
    assert abs(z.var() - 1) < 4 * np.sqrt(2 / z.size)
    # the two values of a Box-Muller pair and neighbouring pairs are uncorrelated
    assert abs(np.corrcoef(z[0::2], z[1::2])[0, 1]) < 4 / np.sqrt(z.size / 2)
    # streams of other heads, purposes, draws and seeds differ
    base = S.gaussians(11, 0, 0, 0, 64)
    for other in (S.gaussians(11, 0, 1, 0, 64), S.gaussians(11, 0, 0, 1, 64),
                  S.gaussians(11, 1, 0, 0, 64), S.gaussians(12, 0, 0, 0, 64)):
        assert np.abs(base - other).max() > 0.1


def test_iid_features_are_the_stream():
    om = S.sample_omega(5, 2, 2, 24, 8, orthogonal=False)
    for h in range(2):
        assert np.array_equal(om[h].ravel(), S.gaussians(5, 2, h, 0, 24 * 8))


def test_orthogonal_blocks():
    seed, draw, m, r = 9, 1, 20, 8          # two full blocks and a partial one
    om = S.sample_omega(seed, draw, 1, m, r, orthogonal=True)[0]
    g_all = S.gaussians(seed, draw, 0, 0, 3 * r * r).reshape(3, r, r)
    n_all = S.gaussians(seed, draw, 0, 1, 3 * r * r).reshape(3, r, r)
    for b in range(3):
        rows = om[b * r:(b + 1) * r]
        k = rows.shape[0]
        norms = np.linalg.norm(n_all[b], axis=1)[:k]
        # row norms are the chi draws; rows of a block are mutually orthogonal
        assert np.allclose(np.linalg.norm(rows, axis=1), norms, rtol=1e-12)
        gram = rows @ rows.T
        assert np.abs(gram - np.diag(np.diag(gram))).max() < 1e-12 * gram.max()
        # the unit rows are the leading columns of the Q of G = Q R with diag(R) > 0:
        # Q^T G is upper triangular with a positive diagonal
        qt = rows / norms[:, None]
        rr = qt @ g_all[b]
        assert np.abs(np.tril(rr, -1)).max() < 1e-12 * np.abs(rr).max()
        assert np.all(np.diag(rr)[:k] > 0)
    # the partial block is the prefix of the full one
    full = S.sample_omega(seed, draw, 1, 24, r, orthogonal=True)[0]
    assert np.array_equal(full[:m], om)


def test_redraw_schedule_rules():
    s = S.RedrawSchedule(seed=7, interval=3)
    draws = []
    for _ in range(7):
        s.forward(training=True)
        draws.append(s.draw)
    assert draws == [0, 0, 0, 1, 1, 1, 2]
    # forwards outside training are not counted
    s2 = S.RedrawSchedule(seed=7, interval=2)
    seq = [s2.forward(t) for t in (True, False, False, True, True)]
    assert seq == [False, False, False, False, True] and s2.draw == 1
    # no interval: never scheduled; manual redraws advance the draw
    s3 = S.RedrawSchedule(seed=1)
    assert not any(s3.forward(True) for _ in range(10)) and s3.draw == 0
    assert s3.redraw() and s3.draw == 1
    # fixed: scheduled and manual redraws are dropped, force overrides once
    s4 = S.RedrawSchedule(seed=1, interval=1)
    s4.fix()
    assert not any(s4.forward(True) for _ in range(5)) and s4.draw == 0
    assert not s4.redraw() and s4.draw == 0
    assert s4.redraw(force=True) and s4.draw == 1
    assert not s4.redraw() and s4.draw == 1
    s4.unfix()
    s4.forward(True)
    assert s4.forward(True) and s4.draw == 2
    # deterministic: fixed at construction
    s5 = S.RedrawSchedule(seed=1, interval=1, deterministic=True)
    assert not any(s5.forward(True) for _ in range(4)) and s5.draw == 0
