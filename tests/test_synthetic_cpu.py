"""The synthetic input recipe: seeded prompts with the stated distributions
and model shapes whose parameter counts match the names they carry."""
import numpy as np
import pytest
import scipy.stats

import synthetic as syn


def test_zipf_prompt_frequencies():
    V = 1000
    ids = syn.zipf_prompt(200_000, V, seed=3)
    k = np.arange(1, V + 1, dtype=np.float64)
    p = k ** -1.1 / (k ** -1.1).sum()
    counts = np.bincount(ids, minlength=V)[:20]
    exp = p[:20] * len(ids)
    # the 20 most likely ids, plus the rest as one cell
    obs = np.append(counts, len(ids) - counts.sum())
    expc = np.append(exp, len(ids) - exp.sum())
    assert scipy.stats.chisquare(obs, expc).pvalue > 0.001
    assert np.array_equal(ids[:50], syn.zipf_prompt(200_000, V, seed=3)[:50])


def test_copy_prompt_fraction_and_spans():
    ids, frac = syn.copy_prompt(4096, 49152, seed=1)
    assert len(ids) == 4096 and 0.38 <= frac <= 0.45
    # copied spans repeat earlier text: a span of length L (16..64) repeats
    # L - 15 of its 16-grams, so about 40 % x 25/40 of the positions do
    seen, repeats = set(), 0
    for t in range(16, len(ids) + 1):
        g = tuple(ids[t - 16:t].tolist())
        repeats += g in seen
        seen.add(g)
    assert repeats > 0.15 * len(ids)
    fresh = syn.zipf_prompt(4096, 49152, seed=1)
    seen, rep_fresh = set(), 0
    for t in range(16, len(fresh) + 1):
        g = tuple(fresh[t - 16:t].tolist())
        rep_fresh += g in seen
        seen.add(g)
    assert rep_fresh < 0.01 * len(fresh)


def test_sweep_rows_ranges():
    d, l = syn.sweep_rows(64)
    assert d.min() >= 1 and d.max() <= 4 and l.min() >= 256 and l.max() <= 8192


@pytest.mark.parametrize("name,billions", [("ouro14", 1.4), ("ouro26", 2.6), ("huginn35", 3.5)])
def test_parameter_counts_match_the_names(name, billions):
    cfg = syn.MODELS[name]
    n = sum(int(np.prod(shape)) for _, shape, _, _ in syn.tensor_specs(cfg))
    assert abs(n / 1e9 - billions) / billions < 0.12, n
