"""Pins of the oracle's typed-decision losses ("Native diffusion language-model
training", Typed-decision training and Labels): candidate-restricted CE,
full-vocabulary CE over the answer tokens, and the Brier term over the
restricted distribution, for hard, dist and set labels, with hard-label
smoothing -- each checked against something other than the oracle itself:
closed forms, a textbook cross-entropy (torch CPU, float64), central finite
differences, and identities between the label kinds.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from oracle import DIST, HARD, LABEL_BOTH, LABEL_FULL, LABEL_RESTRICTED, SET


def one_slot(z, a, kind, val, **kw):
    z = np.asarray(z, np.float64)[None, :]
    a = np.asarray(a, np.int32)
    return oracle.decision_loss(z, z.shape[1], None, np.array([0, a.size], np.int64), a,
                                np.array([kind]), np.asarray(val, np.float64), **kw)


def onehot(K, g):
    v = np.zeros(K)
    v[g] = 1.0
    return v


@pytest.mark.parametrize("K,V", [(2, 7), (5, 50), (26, 1000)])
def test_equal_logits(K, V):
    """All logits equal: the restricted softmax is uniform (CE_res = ln K for
    any target that sums to one), the full softmax is uniform (CE_full =
    ln V), and the Brier score is sum_k (1/K - y_k)^2."""
    z = np.full(V, 0.37)
    a = np.arange(3, 3 + K)
    rng = np.random.default_rng(K)
    pi = rng.dirichlet(np.ones(K))
    S = np.zeros(K)
    S[rng.choice(K, size=max(1, K // 2), replace=False)] = 1.0
    for kind, val, y in ((HARD, onehot(K, K - 1), onehot(K, K - 1)), (DIST, pi, pi), (SET, S, S / S.sum())):
        r = one_slot(z, a, kind, val, brier_weight=0.1)
        assert r["ce_res"][0] == pytest.approx(math.log(K), rel=1e-13, abs=1e-14)
        assert r["ce_full"][0] == pytest.approx(math.log(V), rel=1e-13)
        assert r["brier"][0] == pytest.approx(((1.0 / K - y) ** 2).sum(), rel=1e-12, abs=1e-15)
        assert r["loss"] == pytest.approx(math.log(K) + math.log(V) + 0.1 * r["brier"][0], rel=1e-13)
    # a hard label's Brier score at uniform prediction: (K - 1) / K
    assert one_slot(z, a, HARD, onehot(K, 0))["brier"][0] == pytest.approx((K - 1) / K, rel=1e-13)


@pytest.mark.parametrize("c", [0.5, 3.0, 60.0])
def test_one_spike_closed_forms(c):
    """Logit c on the gold answer, 0 on every other token: r_g = e^c / (e^c +
    K - 1), CE_res = -ln r_g, CE_full = ln(e^c + V - 1) - c, Brier =
    (1 - r_g)^2 K / (K - 1); a confident right answer (c = 60) has Brier 0."""
    K, V, g = 4, 300, 2
    z = np.zeros(V)
    a = np.array([10, 20, 30, 40])
    z[a[g]] = c
    r = one_slot(z, a, HARD, onehot(K, g))
    rg = math.exp(c) / (math.exp(c) + K - 1)
    assert r["ce_res"][0] == pytest.approx(-math.log(rg), rel=1e-12, abs=1e-24)
    assert r["ce_full"][0] == pytest.approx(math.log(math.exp(c) + V - 1) - c, rel=1e-12, abs=1e-24)
    assert r["brier"][0] == pytest.approx((1 - rg) ** 2 * K / (K - 1), rel=1e-12, abs=1e-40)
    if c == 60.0:
        assert r["brier"][0] < 1e-40 and r["ce_res"][0] < 1e-20


def test_all_tokens_as_candidates_is_textbook_cross_entropy():
    """K = V with the answer tokens = the whole vocabulary: the restricted
    and the full CE are both the textbook cross-entropy (torch, float64),
    hard and soft targets alike."""
    V = 64
    rng = np.random.default_rng(1)
    z = rng.standard_normal(V) * 2
    a = rng.permutation(V)
    pi = rng.dirichlet(np.ones(V))
    zt = torch.from_numpy(z)[None]
    for kind, val in ((HARD, onehot(V, 17)), (DIST, pi)):
        r = one_slot(z, a, kind, val)
        target = torch.zeros(1, V, dtype=torch.float64)
        target[0, torch.from_numpy(a)] = torch.from_numpy(val)
        want = float(torch.nn.functional.cross_entropy(zt, target))
        assert r["ce_res"][0] == pytest.approx(want, rel=1e-12)
        assert r["ce_full"][0] == pytest.approx(want, rel=1e-12)


def _random_batch(seed, n=5, V=23, Kmax=6):
    rng = np.random.default_rng(seed)
    off = [0]
    ids, kinds, vals = [], [], []
    for i in range(n):
        K = int(rng.integers(1 if i == 0 else 2, Kmax + 1))
        ids.append(rng.choice(V, size=K, replace=False))
        kind = [HARD, DIST, SET][i % 3]
        if kind == HARD:
            v = onehot(K, int(rng.integers(K)))
        elif kind == DIST:
            v = rng.dirichlet(np.ones(K))
            v[int(rng.integers(K))] = 0.0           # a zero entry is valid
            v /= v.sum()
        else:
            v = np.zeros(K)
            v[rng.choice(K, size=int(rng.integers(1, K + 1)), replace=False)] = 1.0
        kinds.append(kind)
        vals.append(v)
        off.append(off[-1] + K)
    z = rng.standard_normal((n + 3, V)) * 1.5
    rows = rng.choice(n + 3, size=n, replace=False)
    return (z, V, rows, np.array(off, np.int64), np.concatenate(ids).astype(np.int32), np.array(kinds),
            np.concatenate(vals))


@pytest.mark.parametrize("label_softmax", [LABEL_RESTRICTED, LABEL_FULL, LABEL_BOTH])
@pytest.mark.parametrize("brier_weight,smoothing", [(0.1, 0.0), (0.7, 0.2)])
def test_gradient_central_differences(label_softmax, brier_weight, smoothing):
    """dlogits is the derivative of the loss (times grad_scale): central
    differences in double on every logit of every slot row."""
    z, V, rows, off, ids, kinds, vals = _random_batch(3)
    kw = dict(label_softmax=label_softmax, brier_weight=brier_weight, smoothing=smoothing)
    r = oracle.decision_loss(z, V, rows, off, ids, kinds, vals, grad_scale=1.7, **kw)
    h = 1e-6
    for i, row in enumerate(rows):
        for v in range(V):
            zp = z.copy()
            zp[row, v] += h
            zm = z.copy()
            zm[row, v] -= h
            fd = (oracle.decision_loss(zp, V, rows, off, ids, kinds, vals, **kw)["loss"]
                  - oracle.decision_loss(zm, V, rows, off, ids, kinds, vals, **kw)["loss"]) / (2 * h)
            assert r["dlogits"][i, v] == pytest.approx(1.7 * fd, abs=1e-8)


def test_gradient_rows_sum_to_zero_and_shift_invariance():
    """Every term is invariant to adding a constant to a row's logits, so
    each gradient row sums to zero; a shifted batch gives the same loss and
    gradient."""
    z, V, rows, off, ids, kinds, vals = _random_batch(4, n=7)
    r = oracle.decision_loss(z, V, rows, off, ids, kinds, vals, smoothing=0.1)
    assert np.abs(r["dlogits"].sum(1)).max() < 1e-15
    r2 = oracle.decision_loss(z + 11.25, V, rows, off, ids, kinds, vals, smoothing=0.1)
    assert r2["loss"] == pytest.approx(r["loss"], rel=1e-12)
    np.testing.assert_allclose(r2["dlogits"], r["dlogits"], atol=1e-15)


def test_label_kinds_agree_where_they_coincide():
    """A dist label that is one-hot, and a one-element set, are the hard
    label; a set is the dist that is uniform over it."""
    rng = np.random.default_rng(5)
    V, K, g = 40, 6, 4
    z = rng.standard_normal(V)
    a = rng.choice(V, K, replace=False)
    hard = one_slot(z, a, HARD, onehot(K, g))
    for kind in (DIST, SET):
        o = one_slot(z, a, kind, onehot(K, g))
        assert o["loss"] == pytest.approx(hard["loss"], rel=1e-14)
        np.testing.assert_allclose(o["dlogits"], hard["dlogits"], atol=1e-16)
    S = np.array([1.0, 0, 1, 1, 0, 0])
    s = one_slot(z, a, SET, S)
    d = one_slot(z, a, DIST, S / 3)
    assert s["loss"] == pytest.approx(d["loss"], rel=1e-14)


def test_hard_label_smoothing():
    """Smoothing eps mixes the one-hot CE target with the uniform one over
    the K answers: CE(eps) = (1 - eps) CE(one-hot) + eps * mean_k(-log r_k)
    (restricted) and the same with -log P(a_k) (full); the Brier target is
    unchanged; eps = 0 is the plain hard label."""
    rng = np.random.default_rng(6)
    V, K, g, eps = 30, 5, 1, 0.15
    z = rng.standard_normal(V) * 2
    a = rng.choice(V, K, replace=False)
    plain = one_slot(z, a, HARD, onehot(K, g))
    sm = one_slot(z, a, HARD, onehot(K, g), smoothing=eps)
    c = z[a]
    log_r = c - (c.max() + np.log(np.exp(c - c.max()).sum()))
    log_p = c - (z.max() + np.log(np.exp(z - z.max()).sum()))
    assert sm["ce_res"][0] == pytest.approx((1 - eps) * plain["ce_res"][0] + eps * (-log_r).mean(), rel=1e-13)
    assert sm["ce_full"][0] == pytest.approx((1 - eps) * plain["ce_full"][0] + eps * (-log_p).mean(), rel=1e-13)
    assert sm["brier"][0] == plain["brier"][0]
    zero = one_slot(z, a, HARD, onehot(K, g), smoothing=0.0)
    assert zero["loss"] == plain["loss"]


def test_label_softmax_selects_terms_and_loss_is_the_slot_mean():
    """both = restricted + full (Brier once); the loss is the mean over the
    label slots of each slot's terms."""
    z, V, rows, off, ids, kinds, vals = _random_batch(7, n=6)
    kw = dict(brier_weight=0.1)
    both = oracle.decision_loss(z, V, rows, off, ids, kinds, vals, label_softmax=LABEL_BOTH, **kw)
    res = oracle.decision_loss(z, V, rows, off, ids, kinds, vals, label_softmax=LABEL_RESTRICTED, **kw)
    full = oracle.decision_loss(z, V, rows, off, ids, kinds, vals, label_softmax=LABEL_FULL, **kw)
    n = len(rows)
    assert both["loss"] == pytest.approx(res["loss"] + full["loss"] - 0.1 * both["brier"].mean(), rel=1e-13)
    assert res["loss"] == pytest.approx((res["ce_res"] + 0.1 * res["brier"]).sum() / n, rel=1e-13)
    assert full["loss"] == pytest.approx((full["ce_full"] + 0.1 * full["brier"]).sum() / n, rel=1e-13)
    assert both["slot_loss"].sum() == pytest.approx(both["loss"], rel=1e-14)
    # restricted-only: nothing outside the answer tokens gets a gradient
    outside = np.ones((n, V), bool)
    for i in range(n):
        outside[i, ids[off[i]:off[i + 1]]] = False
    assert (res["dlogits"][outside] == 0).all()


def test_bf16_rows_decode_like_their_values():
    """bf16 bit patterns and the same values in float64 give the same loss."""
    z, V, rows, off, ids, kinds, vals = _random_batch(8)
    zb = torch.from_numpy(z).to(torch.bfloat16)
    bits = zb.view(torch.int16).numpy().view(np.uint16)
    a = oracle.decision_loss(bits, V, rows, off, ids, kinds, vals)
    b = oracle.decision_loss(zb.double().numpy(), V, rows, off, ids, kinds, vals)
    assert a["loss"] == b["loss"]
    np.testing.assert_array_equal(a["dlogits"], b["dlogits"])


def test_invalid_labels_are_refused():
    z = np.zeros(10)
    with pytest.raises(ValueError):
        one_slot(z, [1, 2, 2], HARD, onehot(3, 0))          # duplicate answer token
    with pytest.raises(ValueError):
        one_slot(z, [1, 12], HARD, onehot(2, 0))            # outside the vocabulary
    with pytest.raises(ValueError):
        one_slot(z, [1, 2], HARD, [1.0, 1.0])               # two gold answers
    with pytest.raises(ValueError):
        one_slot(z, [1, 2], SET, [0.0, 0.0])                # empty set
    with pytest.raises(ValueError):
        one_slot(z, [1, 2], DIST, [1.5, -0.5])              # negative probability


def test_single_answer_question():
    """K = 1: the restricted softmax is certain (CE_res = 0, Brier = 0 for
    any label), the full CE is the plain CE of that token."""
    z = np.array([0.3, -1.2, 2.0, 0.1])
    for kind in (HARD, DIST, SET):
        r = one_slot(z, [2], kind, [1.0])
        assert r["ce_res"][0] == 0.0 and r["brier"][0] == 0.0
        assert r["ce_full"][0] == pytest.approx(math.log(np.exp(z).sum()) - 2.0, rel=1e-14)
