"""The token sample that the full-size parity test checks against the oracle
(tests/test_gpu_parity.py::full_size_sample), on synthetic routings: every token of the four
least-loaded active experts, a token in every 128-row m-tile of every active expert (its
first row) and each expert's last row, and a seeded random subset."""
import numpy as np

from test_gpu_parity import N_RANDOM_TOKENS, full_size_sample


def _routing(T, E, k, seed, skew=0.0):
    rng = np.random.default_rng(seed)
    p = np.arange(1, E + 1, dtype=np.float64) ** -skew if skew else np.ones(E)
    p /= p.sum()
    return np.stack([rng.choice(E, size=k, replace=False, p=p) for _ in range(T)]).astype(np.int32)


def _check(idx, T, E):
    toks = full_size_sample(idx, T, E)
    assert np.all(np.diff(toks) > 0) and toks.min() >= 0 and toks.max() < T
    chosen = set(toks.tolist())
    counts = np.bincount(idx.reshape(-1), minlength=E)
    active = np.nonzero(counts)[0]
    rare = active[np.argsort(counts[active], kind="stable")][:4]
    for e in rare:
        rows = np.nonzero((idx == e).any(axis=1))[0]
        assert set(rows.tolist()) <= chosen
    for e in active:
        rows = np.nonzero((idx == e).any(axis=1))[0]     # row order = ascending token id
        for m in range(0, len(rows), 128):
            assert rows[m] in chosen                     # the first row of every m-tile
        assert rows[-1] in chosen                        # the last, partial m-tile
    assert len(toks) >= min(T, N_RANDOM_TOKENS)
    return toks


def test_sample_covers_every_tile_of_a_balanced_routing():
    _check(_routing(8192, 8, 2, 1), 8192, 8)


def test_sample_covers_every_tile_of_a_skewed_routing():
    _check(_routing(4096, 256, 8, 2, skew=1.2), 4096, 256)


def test_sample_of_a_small_batch_is_the_whole_batch():
    toks = _check(_routing(64, 256, 8, 3, skew=1.2), 64, 256)
    assert len(toks) == 64
