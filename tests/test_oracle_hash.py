"""Pins for the oracle's random draws: hash, time draw, corruption.

Each check is against something other than the oracle's own code: published
SplitMix64 vectors, a sequential re-derivation of the generator, the page's
probability formula evaluated in exact rational arithmetic, binomial and
chi-square statistics, and layout invariances.
"""
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
from conftest import GOLDEN

M64 = (1 << 64) - 1


def _golden():
    outs, buckets = [], []
    with open(os.path.join(GOLDEN, "splitmix64_vectors.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            tok = line.split()
            if tok[0] == "out":
                outs.append((int(tok[1]), int(tok[2]), int(tok[3])))
            elif tok[0] == "buckets":
                buckets.append((int(tok[1]), int(tok[2]), int(tok[3]), [int(x) for x in tok[4:]]))
    return outs, buckets


def test_splitmix64_published_vectors():
    outs, _ = _golden()
    assert len(outs) >= 8
    for seed, k, want in outs:
        assert oracle.splitmix64_at(seed, k) == want


def test_splitmix64_published_bucket_counts():
    _, buckets = _golden()
    for seed, n, b, counts in buckets:
        got = [0] * b
        for k in range(n):
            got[int(oracle.splitmix64_at(seed, k) / 2.0 ** 64 * b)] += 1
        assert got == counts


def _sequential_stream(seed, n):
    """SplitMix64 written as the stateful generator of the paper: advance the
    state by gamma, then finalise.  Independent of the oracle's direct
    counter-indexed formula."""
    out = np.empty(n, dtype=np.uint64)
    state = np.uint64(seed)
    gamma = np.uint64(0x9E3779B97F4A7C15)
    with np.errstate(over="ignore"):
        for i in range(n):
            state = state + gamma
            z = state
            z = (z ^ (z >> np.uint64(30))) * np.uint64(0xBF58476D1CE4E5B9)
            z = (z ^ (z >> np.uint64(27))) * np.uint64(0x94D049BB133111EB)
            out[i] = z ^ (z >> np.uint64(31))
    return out


@pytest.mark.parametrize("seed", [0, 7, 2 ** 63 + 5])
def test_direct_index_equals_sequential_stepping(seed):
    seq = _sequential_stream(seed, 20000)
    direct = np.array([oracle.splitmix64_at(seed, k) for k in range(20000)], dtype=np.uint64)
    assert np.array_equal(seq, direct)


def test_counter_layout():
    assert oracle.counter(0, 0, 0) == 0
    assert oracle.counter(1, 0, 0) == 1 << 56
    assert oracle.counter(2, 3, 5) == (2 << 56) | (3 << 32) | 5
    assert oracle.counter(1, (1 << 24) - 1, (1 << 32) - 1) == (1 << 56) | (((1 << 24) - 1) << 32) | ((1 << 32) - 1)


def test_u24_uniform_chi_square():
    n, bins = 200000, 64
    draws = np.array([oracle.splitmix64_at(11, oracle.counter(1, 0, k)) >> 40 for k in range(n)])
    assert draws.min() >= 0 and draws.max() < 1 << 24
    counts = np.bincount(draws * bins >> 24, minlength=bins)
    e = n / bins
    chi2 = ((counts - e) ** 2 / e).sum()
    # chi-square with 63 dof: mean 63, sd ~11.2; 63 + 6 sd is far in the tail
    assert chi2 < 63 + 6 * 11.2


# --------------------------------------------------------------------------
# t and p  ("LLaDA-8B-MDLM-LoRA", Training table, row "Objective";
#           "diffusiongemma-26B-A4B-it-ALWAYS-THINK", Finetuning notes)
# --------------------------------------------------------------------------
def _exact_p(t: float, eps: float) -> Fraction:
    return (1 - Fraction(eps)) * Fraction(t) + Fraction(eps)


def test_absorbing_p_follows_formula_within_fp32_rounding():
    eps = 1e-3
    t, p = oracle.sample_t(123, 4096, oracle.ABSORBING, eps)
    eps32 = float(np.float32(eps))
    for ti, pi in zip(t[:512], p[:512]):
        # t is a multiple of 2^-24 in [0,1)
        assert 0.0 <= ti < 1.0 and float(ti) * 2 ** 24 == int(float(ti) * 2 ** 24)
        exact = _exact_p(float(ti), eps32)
        # three fp32 roundings -> within 2 ulp of the exact value
        ulp = np.spacing(np.float32(pi))
        assert abs(Fraction(float(pi)) - exact) <= 2 * Fraction(float(ulp))
    assert (p >= np.float32(eps)).all() and (p < 1.0).all()
    # t ~ U(0,1): mean and variance of 4096 draws
    assert abs(t.mean() - 0.5) < 5 * np.sqrt(1 / 12 / 4096)
    assert abs(t.var() - 1 / 12) < 0.01


def test_uniform_t_in_eps_one():
    eps = 1e-3
    t, p = oracle.sample_t(5, 4096, oracle.UNIFORM, eps)
    assert np.array_equal(t, p)
    assert (t >= np.float32(eps)).all() and (t < 1.0).all()
    assert abs(t.mean() - (1 + eps) / 2) < 5 * np.sqrt(1 / 12 / 4096)


def test_p_floor_and_ceiling_exhaustive():
    """Over all 2^24 values of u: p(0) = eps exactly, p monotone, p < 1
    (so 1/p is bounded and the corruption threshold stays below 2^24)."""
    eps = np.float32(1e-3)
    c1 = np.float32(1.0) - eps
    u = np.arange(1 << 24, dtype=np.float32) * np.float32(2.0 ** -24)
    p = (c1 * u).astype(np.float32) + eps
    assert p.dtype == np.float32
    assert p[0] == eps
    assert (np.diff(p) >= 0).all()
    assert p[-1] < 1.0
    # the oracle's draws are members of this table
    t, po = oracle.sample_t(99, 2000, oracle.ABSORBING, 1e-3)
    idx = (t.astype(np.float64) * 2 ** 24).astype(np.int64)
    assert np.array_equal(p[idx], po)


def test_time_draw_is_stream_zero_of_the_unit():
    """t of unit u is u24 of the hash at counter (stream 0, unit u, position
    0), from the published generator and the counter layout pinned above."""
    for mode in (oracle.ABSORBING, oracle.UNIFORM):
        t, _ = oracle.sample_t(2024, 300, mode, 1e-3)
        u = np.array([oracle.splitmix64_at(2024, oracle.counter(0, k, 0)) >> 40 for k in range(300)],
                     np.float64) * 2.0 ** -24
        if mode == oracle.ABSORBING:
            assert np.array_equal(t.astype(np.float64), u)
        else:   # t = fl(fl((1 - eps) u) + eps), monotone in u
            order = np.argsort(u, kind="stable")
            assert (np.diff(t[order]) >= 0).all()
            c1 = np.float32(1.0) - np.float32(1e-3)
            assert np.array_equal(t, (c1 * u.astype(np.float32)).astype(np.float32) + np.float32(1e-3))


def test_time_draw_depends_on_seed_and_unit_only():
    t1, _ = oracle.sample_t(42, 10, oracle.ABSORBING, 1e-3)
    t2, _ = oracle.sample_t(42, 20, oracle.ABSORBING, 1e-3)
    t3, _ = oracle.sample_t(43, 10, oracle.ABSORBING, 1e-3)
    assert np.array_equal(t1, t2[:10])
    assert not np.array_equal(t1, t3)


# --------------------------------------------------------------------------
# corruption
# --------------------------------------------------------------------------
@pytest.mark.parametrize("pval", [1e-3, 0.1, 0.5, 0.9, 0.999])
def test_mask_fraction_binomial(pval):
    n = 1 << 20
    lay = oracle.Layout(1, n, None, None)
    clean = np.zeros(n, np.int32)
    p = np.array([pval], np.float32)
    noisy, corr = oracle.corrupt(lay, clean, p, oracle.ABSORBING, 7, 8, seed=3)
    frac = corr.mean()
    sd = np.sqrt(pval * (1 - pval) / n)
    assert abs(frac - pval) < 5 * sd + 1e-9
    assert np.array_equal(noisy[corr == 1], np.full(int(corr.sum()), 7, np.int32))
    assert np.array_equal(noisy[corr == 0], clean[corr == 0])


def test_corruption_threshold_is_strict_and_exact():
    """corrupted iff u24 < p * 2^24: recompute u24 from the published
    generator via the sequential stream and compare token by token."""
    n = 5000
    lay = oracle.Layout(1, n, None, None)
    p = np.array([0.37], np.float32)
    _, corr = oracle.corrupt(lay, np.zeros(n, np.int32), p, oracle.ABSORBING, 1, 2, seed=77)
    thr = Fraction(float(p[0])) * 2 ** 24
    base = oracle.counter(1, 0, 0)
    for i in range(n):
        u24 = oracle.splitmix64_at(77, base + i) >> 40
        assert corr[i] == (1 if u24 < thr else 0)


def test_corruption_threshold_equality_is_not_corrupted():
    """A token whose draw equals p * 2^24 exactly is not corrupted (strict
    compare): p is set to k / 2^24 for the k one token drew, exact in fp32."""
    n = 4000
    base = oracle.counter(1, 0, 0)
    u24 = np.array([oracle.splitmix64_at(91, base + i) >> 40 for i in range(n)], np.int64)
    i0 = int(np.argmax(u24 > 0))
    k = int(u24[i0])
    p = np.array([k * 2.0 ** -24], np.float32)
    assert float(p[0]) * 2 ** 24 == k
    lay = oracle.Layout(1, n, None, None)
    _, corr = oracle.corrupt(lay, np.zeros(n, np.int32), p, oracle.ABSORBING, 1, 2, seed=91)
    assert corr[i0] == 0
    assert np.array_equal(corr, (u24 < k).astype(np.uint8))


def test_uniform_replacement_histogram_and_rate():
    V = 97
    n = 1 << 18
    lay = oracle.Layout(1, n, None, None)
    clean = np.full(n, 5, np.int32)
    t = np.array([0.6], np.float32)
    noisy, corr = oracle.corrupt(lay, clean, t, oracle.UNIFORM, -1, V, seed=9)
    frac = corr.mean()
    assert abs(frac - 0.6) < 5 * np.sqrt(0.6 * 0.4 / n)
    r = noisy[corr == 1]
    assert r.min() >= 0 and r.max() < V
    counts = np.bincount(r, minlength=V)
    e = r.shape[0] / V
    chi2 = ((counts - e) ** 2 / e).sum()
    assert chi2 < 96 + 6 * np.sqrt(2 * 96)
    # replacement equal to the clean id is kept (it is still "corrupted")
    assert (r == 5).sum() > 0
    assert np.array_equal(noisy[corr == 0], clean[corr == 0])


def test_replacement_multiply_shift_bounds():
    """r = ((h >> 32) * V) >> 32 lies in [0, V) for extreme h and large V."""
    V = 262144
    n = 4096
    lay = oracle.Layout(1, n, None, None)
    noisy, corr = oracle.corrupt(lay, np.zeros(n, np.int32), np.array([0.999], np.float32),
                                 oracle.UNIFORM, -1, V, seed=1)
    r = noisy[corr == 1]
    assert r.min() >= 0 and r.max() < V
    base = oracle.counter(2, 0, 0)
    for i in np.nonzero(corr)[0][:200]:
        h = oracle.splitmix64_at(1, base + int(i))
        assert noisy[i] == ((h >> 32) * V) >> 32


def test_pads_never_corrupted():
    n = 4096
    pad = np.zeros(n, np.uint8)
    pad[3000:] = 1
    lay = oracle.Layout(1, n, None, pad)
    clean = np.arange(n, dtype=np.int32) % 50
    noisy, corr = oracle.corrupt(lay, clean, np.array([0.999], np.float32),
                                 oracle.ABSORBING, 99, 100, seed=4)
    assert corr[3000:].sum() == 0
    assert np.array_equal(noisy[3000:], clean[3000:])
    assert corr[:3000].mean() > 0.99


def test_packing_invariance_of_corruption():
    """Positions restart at document boundaries ("Native diffusion
    language-model training", Packed training), so a document's corruption
    is the same packed (cu_seqlens) or padded into its own row."""
    lens = [5, 17, 40, 1, 33]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    T = int(cu[-1])
    rng = np.random.default_rng(0)
    clean_packed = rng.integers(0, 1000, T).astype(np.int32)
    p = np.array([0.3, 0.5, 0.7, 0.9, 0.2], np.float32)
    lay_p = oracle.Layout(len(lens), 0, cu, None)
    noisy_p, corr_p = oracle.corrupt(lay_p, clean_packed, p, oracle.UNIFORM, -1, 1000, seed=12)
    Lmax = max(lens)
    clean_d = np.zeros(len(lens) * Lmax, np.int32)
    pad = np.ones(len(lens) * Lmax, np.uint8)
    for u, l in enumerate(lens):
        clean_d[u * Lmax:u * Lmax + l] = clean_packed[cu[u]:cu[u + 1]]
        pad[u * Lmax:u * Lmax + l] = 0
    lay_d = oracle.Layout(len(lens), Lmax, None, pad)
    noisy_d, corr_d = oracle.corrupt(lay_d, clean_d, p, oracle.UNIFORM, -1, 1000, seed=12)
    for u, l in enumerate(lens):
        assert np.array_equal(corr_p[cu[u]:cu[u + 1]], corr_d[u * Lmax:u * Lmax + l])
        assert np.array_equal(noisy_p[cu[u]:cu[u + 1]], noisy_d[u * Lmax:u * Lmax + l])


def test_inconsistent_layout_rejected():
    cu = np.array([0, 5, 3], np.int32)  # not monotone: token 3 lies in unit 0
    lay = oracle.Layout(2, 0, cu, None)
    # cu[-1] = 3 tokens, all inside unit 0 -> consistent for those tokens;
    # a layout whose tokens fall outside every unit is rejected:
    cu2 = np.array([1, 2, 4], np.int32)
    lay2 = oracle.Layout(2, 0, cu2, None)
    with pytest.raises(ValueError):
        oracle.corrupt(lay2, np.zeros(4, np.int32), np.array([0.5, 0.5], np.float32),
                       oracle.ABSORBING, 0, 2, seed=0)
    oracle.corrupt(lay, np.zeros(3, np.int32), np.array([0.5, 0.5], np.float32),
                   oracle.ABSORBING, 0, 2, seed=0)
