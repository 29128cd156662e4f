"""Pins for the oracle's loss, gradient and reductions.

Checked against: closed forms (all-zero logits give ln V, a single spike
gives ln(e^c + V - 1) - c), a textbook log-softmax routine (torch CPU fp64,
an independent library implementation), central finite differences,
layout invariances and the pages' statements of the objectives:
  "LLaDA-8B-MDLM-LoRA", Training table, row "Objective";
  "Native diffusion language-model training", model table, Packed training,
  Adapters/merging (Cut Cross Entropy);
  "diffusiongemma-26B-A4B-it-ALWAYS-THINK", Finetuning notes.
"""
import math

import numpy as np
import pytest
import torch

import oracle


def bf16_bits_of(x: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(torch.bfloat16) \
        .view(torch.int16).numpy().view(np.uint16)


def torch_ce(logits_f64: np.ndarray, targets: np.ndarray) -> np.ndarray:
    return torch.nn.functional.cross_entropy(
        torch.from_numpy(logits_f64), torch.from_numpy(targets.astype(np.int64)),
        reduction="none").numpy()


# --------------------------------------------------------------------------
# per-row CE
# --------------------------------------------------------------------------
@pytest.mark.parametrize("V", [2, 8, 1000, 126464])
def test_all_zero_logits_give_ln_v(V):
    logits = np.zeros((3, V), np.uint16)          # bf16 +0.0
    lse, ce = oracle.ce_rows(logits, V, np.arange(3), np.array([0, V // 2, V - 1]))
    assert np.allclose(ce, math.log(V), rtol=0, atol=1e-12)
    assert np.allclose(lse, math.log(V), rtol=0, atol=1e-12)


@pytest.mark.parametrize("c", [4.0, -2.5, 30.0])
def test_single_spike_closed_form(c):
    V = 4096
    x = np.zeros((1, V), np.float32)
    x[0, 17] = c
    _, ce = oracle.ce_rows(bf16_bits_of(x), V, np.array([0]), np.array([17]))
    want = math.log(math.exp(c) + V - 1) - c
    assert abs(ce[0] - want) < 1e-12 * max(1.0, abs(want))
    # a different target: ce = lse - 0
    _, ce2 = oracle.ce_rows(bf16_bits_of(x), V, np.array([0]), np.array([3]))
    assert abs(ce2[0] - math.log(math.exp(c) + V - 1)) < 1e-12 * max(1.0, c)


def test_ce_matches_textbook_log_softmax():
    rng = np.random.default_rng(1)
    V, R = 3001, 37
    x32 = (rng.standard_normal((R, V)) * 3).astype(np.float32)
    bits = bf16_bits_of(x32)
    x = oracle.bf16_to_f64(bits)
    tg = rng.integers(0, V, R)
    _, ce = oracle.ce_rows(bits, V, np.arange(R), tg)
    assert np.allclose(ce, torch_ce(x, tg), rtol=1e-13, atol=1e-12)
    # f64 entry point on the decoded matrix gives the same
    _, ce64 = oracle.ce_rows(x, V, np.arange(R), tg)
    assert np.allclose(ce, ce64, rtol=0, atol=1e-13)


def test_ce_respects_row_stride():
    rng = np.random.default_rng(2)
    V, ld, R = 100, 128, 5
    x = (rng.standard_normal((R, ld)) * 2).astype(np.float32)
    x[:, V:] = 1e4                                  # must be ignored
    bits = bf16_bits_of(x)
    tg = np.array([0, 1, 50, 98, 99])
    _, ce = oracle.ce_rows(bits, V, np.arange(R), tg)
    ref = torch_ce(oracle.bf16_to_f64(bits)[:, :V], tg)
    assert np.allclose(ce, ref, rtol=1e-13, atol=1e-12)


def test_bf16_decode_exact():
    vals = np.array([0.0, -0.0, 1.0, -2.0, 0.1, 3.0e38, 1e-40], np.float32)
    dec = oracle.bf16_to_f64(bf16_bits_of(vals))
    ref = torch.from_numpy(vals).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(dec, ref)


# --------------------------------------------------------------------------
# gradient
# --------------------------------------------------------------------------
def test_gradient_rows_sum_to_zero_and_signs():
    rng = np.random.default_rng(3)
    V, R = 5000, 8
    bits = bf16_bits_of((rng.standard_normal((R, V)) * 3).astype(np.float32))
    tg = rng.integers(0, V, R)
    lse, _ = oracle.ce_rows(bits, V, np.arange(R), tg)
    coef = rng.uniform(0.1, 5.0, R)
    g = oracle.grad_rows(bits, V, np.arange(R), tg, coef, lse)
    assert np.abs(g.sum(axis=1)).max() < 1e-12 * V
    for r in range(R):
        assert g[r, tg[r]] < 0
        others = np.delete(g[r], tg[r])
        assert (others >= 0).all()


def _absorbing_loss_f64(x: np.ndarray, layout, clean, corr, p, align):
    plan = oracle.plan_diffusion(layout, clean, corr, p, oracle.ABSORBING, align)
    tr = oracle.term(x, x.shape[1], plan)
    loss, _ = oracle.reduce_units(layout.n_units, tr)
    return loss, tr


@pytest.mark.parametrize("align", [oracle.ALIGNED, oracle.SHIFTED])
def test_finite_differences_absorbing(align):
    """d loss / d logits from the oracle vs central differences of the
    oracle's own loss function, B=2 L=4 V=8 in double."""
    rng = np.random.default_rng(4)
    B, L, V = 2, 4, 8
    lay = oracle.Layout(B, L, None, None)
    x = rng.standard_normal((B * L, V)) * 2
    clean = rng.integers(0, V - 1, B * L).astype(np.int32)
    corr = np.array([1, 0, 1, 1, 0, 1, 1, 1], np.uint8)
    p = np.array([0.3, 0.8], np.float32)
    loss, tr = _absorbing_loss_f64(x, lay, clean, corr, p, align)
    g = oracle.term_grad(x, V, tr, np.arange(B * L), grad_scale=1.0)
    h = 1e-6
    fd = np.zeros_like(x)
    for i in range(B * L):
        for v in range(V):
            xp = x.copy(); xp[i, v] += h
            xm = x.copy(); xm[i, v] -= h
            fd[i, v] = (_absorbing_loss_f64(xp, lay, clean, corr, p, align)[0]
                        - _absorbing_loss_f64(xm, lay, clean, corr, p, align)[0]) / (2 * h)
    assert np.abs(fd - g).max() < 1e-7


def test_grad_scale_multiplies_gradient_only():
    rng = np.random.default_rng(5)
    lay = oracle.Layout(1, 16, None, None)
    x = rng.standard_normal((16, 11))
    clean = rng.integers(0, 10, 16).astype(np.int32)
    corr = np.ones(16, np.uint8)
    p = np.array([0.5], np.float32)
    loss, tr = _absorbing_loss_f64(x, lay, clean, corr, p, oracle.ALIGNED)
    g1 = oracle.term_grad(x, 11, tr, np.arange(16), 1.0)
    g3 = oracle.term_grad(x, 11, tr, np.arange(16), 3.0)
    assert np.allclose(g3, 3 * g1, rtol=1e-15, atol=0)


# --------------------------------------------------------------------------
# weighting, normaliser, alignment
# --------------------------------------------------------------------------
def test_all_masked_p_one_is_mean_textbook_ce():
    """With every token masked and p = 1 the weight is 1/N: the loss is the
    textbook mean CE over all tokens."""
    rng = np.random.default_rng(6)
    B, L, V = 3, 20, 257
    lay = oracle.Layout(B, L, None, None)
    x = rng.standard_normal((B * L, V)) * 3
    clean = rng.integers(0, V, B * L).astype(np.int32)
    loss, _ = _absorbing_loss_f64(x, lay, clean, np.ones(B * L, np.uint8),
                                  np.ones(B, np.float32), oracle.ALIGNED)
    assert abs(loss - torch_ce(x, clean).mean()) < 1e-12


def test_inverse_p_weight_and_non_pad_normaliser():
    """[LLaDA]: CE on masked tokens divided by the mask probability; the sum
    is normalised by the number of non-pad tokens (N), not by the number of
    masked tokens."""
    rng = np.random.default_rng(7)
    L, V = 10, 33
    pad = np.zeros(L, np.uint8); pad[8:] = 1
    lay = oracle.Layout(1, L, None, pad)
    x = rng.standard_normal((L, V))
    clean = rng.integers(0, V, L).astype(np.int32)
    corr = np.array([1, 0, 0, 1, 0, 0, 0, 1, 0, 0], np.uint8)
    p = np.array([0.25], np.float32)
    loss, _ = _absorbing_loss_f64(x, lay, clean, corr, p, oracle.ALIGNED)
    ce = torch_ce(x, clean)
    want = (ce[0] + ce[3] + ce[7]) / float(p[0]) / 8
    assert abs(loss - want) < 1e-12


def test_expected_absorbing_loss_on_zero_logits_is_ln_v():
    """All-zero logits: ce = ln V per scored row, loss = ln V * sum(1/p)/N;
    since E[1{masked}/p] = 1 the loss averages to ln V over many draws."""
    V, B, L = 64, 64, 256
    lay = oracle.Layout(B, L, None, None)
    x = np.zeros((B * L, V), np.uint16)
    clean = np.zeros(B * L, np.int32)
    losses = []
    for seed in range(20):
        t, p = oracle.sample_t(seed, B, oracle.ABSORBING, 1e-3)
        _, corr = oracle.corrupt(lay, clean, p, oracle.ABSORBING, V - 1, V, seed)
        plan = oracle.plan_diffusion(lay, clean, corr, p, oracle.ABSORBING, oracle.ALIGNED)
        tr = oracle.term(x, V, plan)
        loss, _ = oracle.reduce_units(B, tr)
        # exact closed form given the mask
        scored = plan.target >= 0
        closed = math.log(V) * (1.0 / p[plan.unit[scored]].astype(np.float64)).sum() / (B * L)
        assert abs(loss - closed) < 1e-12 * closed
        losses.append(loss)
    assert abs(np.mean(losses) / math.log(V) - 1.0) < 0.05


def test_shifted_indexing_spike():
    """Dream-style shifted logits: row i scores token i+1.  A spike at
    clean[i+1] in row i gives a small shifted loss and a large aligned one;
    each unit's last row is unscored."""
    B, L, V = 2, 12, 50
    lay = oracle.Layout(B, L, None, None)
    rng = np.random.default_rng(8)
    clean = rng.integers(0, V, B * L).astype(np.int32)
    x = np.zeros((B * L, V))
    for i in range(B * L - 1):
        x[i, clean[i + 1]] = 20.0
    corr = np.ones(B * L, np.uint8)
    p = np.ones(B, np.float32)
    ls, trs = _absorbing_loss_f64(x, lay, clean, corr, p, oracle.SHIFTED)
    la, _ = _absorbing_loss_f64(x, lay, clean, corr, p, oracle.ALIGNED)
    assert ls < 1e-6          # each scored row: ln(e^20 + V - 1) - 20 ~ 1e-7
    assert la > 1.0
    assert trs.plan.target[L - 1] == -1 and trs.plan.target[2 * L - 1] == -1
    assert (trs.plan.target[:L - 1] == clean[1:L]).all()
    assert (trs.plan.target[L:2 * L - 1] == clean[L + 1:]).all()


def test_shifted_row_needs_corrupted_target():
    B, L, V = 1, 6, 9
    lay = oracle.Layout(B, L, None, None)
    clean = np.arange(L, dtype=np.int32)
    corr = np.array([1, 0, 1, 0, 0, 1], np.uint8)
    plan = oracle.plan_diffusion(lay, clean, corr, np.array([0.5], np.float32),
                                 oracle.ABSORBING, oracle.SHIFTED)
    assert list(plan.target) == [-1, 2, -1, -1, 5, -1]


# --------------------------------------------------------------------------
# uniform noise + encoder AR
# --------------------------------------------------------------------------
def test_uniform_lambda_zero_is_canvas_mean():
    rng = np.random.default_rng(9)
    B, C, P, V = 2, 8, 4, 31
    canvas = oracle.Layout(B, C, None, None)
    enc = oracle.Layout(B, P + C, None, None)
    full = rng.integers(0, V, (B, P + C)).astype(np.int32)
    cclean = full[:, P:].reshape(-1).copy()
    xc = rng.standard_normal((B * C, V))
    xe = rng.standard_normal((B * (P + C), V))
    loss, unit, tc, te = oracle.loss_uniform(canvas, xc, cclean, enc, xe, full.reshape(-1), V, 0.0)
    assert abs(loss - torch_ce(xc, cclean).mean()) < 1e-12
    assert abs(unit.sum() - loss) < 1e-12


def test_encoder_term_is_plain_causal_ce():
    rng = np.random.default_rng(10)
    B, C, P, V = 3, 5, 7, 41
    canvas = oracle.Layout(B, C, None, None)
    enc = oracle.Layout(B, P + C, None, None)
    full = rng.integers(0, V, (B, P + C)).astype(np.int32)
    xc = np.zeros((B * C, V))                      # canvas term = ln V exactly
    xe = rng.standard_normal((B * (P + C), V)) * 2
    lam = 0.7
    loss, _, tc, te = oracle.loss_uniform(canvas, xc, full[:, P:].reshape(-1).copy(), enc, xe,
                                          full.reshape(-1), V, lam)
    xe3 = xe.reshape(B, P + C, V)
    causal = torch.nn.functional.cross_entropy(
        torch.from_numpy(xe3[:, :-1].reshape(-1, V)),
        torch.from_numpy(full[:, 1:].reshape(-1).astype(np.int64))).item()
    assert abs(loss - (math.log(V) + lam * causal)) < 1e-12


def test_encoder_term_with_pads_brute_force():
    """Encoder sequences with trailing pads: the term is the mean textbook CE
    over exactly the next-token pairs whose target is a real token of the
    same sequence, enumerated here one by one."""
    rng = np.random.default_rng(11)
    B, S, V = 3, 9, 23
    lengths = (9, 4, 1)                      # real tokens per sequence, then pads
    pad = np.zeros(B * S, np.uint8)
    for b, n in enumerate(lengths):
        pad[b * S + n:(b + 1) * S] = 1
    enc = oracle.Layout(B, S, None, pad)
    ids = rng.integers(0, V, B * S).astype(np.int32)
    x = rng.standard_normal((B * S, V)) * 2
    rows, tgts = [], []
    for b in range(B):
        for i in range(S - 1):
            if i + 1 < lengths[b]:
                rows.append(b * S + i)
                tgts.append(ids[b * S + i + 1])
    want = torch.nn.functional.cross_entropy(torch.from_numpy(x[rows]),
                                             torch.from_numpy(np.array(tgts, np.int64))).item()
    lam = 1.3
    tr = oracle.term(x, V, oracle.plan_encoder(enc, ids, lam))
    assert sorted(tr.rows.tolist()) == rows
    assert abs(tr.row_loss.sum() - lam * want) < 1e-12


# --------------------------------------------------------------------------
# uniform noise: 1/(1-t) time weighting with a cap, per-example mean
# --------------------------------------------------------------------------
def _canvas_case(seed, B=3, C=6, V=37, pads=None):
    rng = np.random.default_rng(seed)
    pad = None
    if pads is not None:
        pad = np.zeros(B * C, np.uint8)
        for b, n in enumerate(pads):
            pad[b * C + n:(b + 1) * C] = 1
    canvas = oracle.Layout(B, C, None, pad)
    clean = rng.integers(0, V, B * C).astype(np.int32)
    x = rng.standard_normal((B * C, V)) * 2
    t = np.array([0.2, 0.55, 0.9][:B], np.float32)
    return canvas, clean, x, t, V


def _canvas_loss(canvas, clean, x, t, V, tw, clip, red):
    plan = oracle.plan_diffusion(canvas, clean, None, t, oracle.UNIFORM, oracle.ALIGNED, tw, clip, red)
    tr = oracle.term(x, V, plan)
    return oracle.reduce_units(canvas.n_units, tr)[0], tr


def test_rhine_cap_one_is_the_plain_mean():
    """1/(1-t) >= 1, so a cap of 1 leaves every weight at 1: the plain token
    mean exactly (a cap applied the wrong way would not)."""
    case = _canvas_case(21)
    plain, _ = _canvas_loss(*case, oracle.NO_TIME_WEIGHT, 0.0, oracle.TOKEN_MEAN)
    capped, _ = _canvas_loss(*case, oracle.INV_ONE_MINUS_T, 1.0, oracle.TOKEN_MEAN)
    assert abs(capped - plain) < 1e-12
    canvas, clean, x, t, V = case
    assert abs(plain - torch_ce(x, clean).mean()) < 1e-12


def test_rhine_single_example_scales_by_inverse_one_minus_t():
    canvas, clean, x, t, V = _canvas_case(22, B=1)
    plain, _ = _canvas_loss(canvas, clean, x, t, V, oracle.NO_TIME_WEIGHT, 0.0, oracle.TOKEN_MEAN)
    for red in (oracle.TOKEN_MEAN, oracle.EXAMPLE_MEAN):
        w, _ = _canvas_loss(canvas, clean, x, t, V, oracle.INV_ONE_MINUS_T, 0.0, red)
        assert abs(w - plain / (1.0 - float(t[0]))) < 1e-12 * abs(w)
    # a cap below 1/(1-t) = 1.25 takes over
    w, _ = _canvas_loss(canvas, clean, x, t, V, oracle.INV_ONE_MINUS_T, 1.1, oracle.TOKEN_MEAN)
    assert abs(w - plain * 1.1) < 1e-12 * abs(w)


def test_example_mean_equal_lengths_is_token_mean_and_unequal_is_not():
    case = _canvas_case(23)
    tok, _ = _canvas_loss(*case, oracle.NO_TIME_WEIGHT, 0.0, oracle.TOKEN_MEAN)
    ex, _ = _canvas_loss(*case, oracle.NO_TIME_WEIGHT, 0.0, oracle.EXAMPLE_MEAN)
    assert abs(tok - ex) < 1e-12
    # examples of 6, 2 and 4 canvas tokens: the mean of the three per-example
    # means, each a textbook CE mean over that example's rows
    canvas, clean, x, t, V = _canvas_case(23, pads=(6, 2, 4))
    ex, tr = _canvas_loss(canvas, clean, x, t, V, oracle.NO_TIME_WEIGHT, 0.0, oracle.EXAMPLE_MEAN)
    ce = torch_ce(x, clean).reshape(3, 6)
    want = (ce[0, :6].mean() + ce[1, :2].mean() + ce[2, :4].mean()) / 3
    assert abs(ex - want) < 1e-12
    tok, _ = _canvas_loss(canvas, clean, x, t, V, oracle.NO_TIME_WEIGHT, 0.0, oracle.TOKEN_MEAN)
    assert abs(tok - (ce[0, :6].sum() + ce[1, :2].sum() + ce[2, :4].sum()) / 12) < 1e-12
    assert abs(tok - ex) > 1e-3


def test_rhine_example_mean_on_zero_logits_closed_form():
    """All-zero logits: every CE is ln V, so the loss is ln V times the mean
    over examples of min(1/(1-t), cap)."""
    canvas, clean, x, t, V = _canvas_case(24, pads=(6, 3, 1))
    x = np.zeros_like(x)
    loss, _ = _canvas_loss(canvas, clean, x, t, V, oracle.INV_ONE_MINUS_T, 4.0, oracle.EXAMPLE_MEAN)
    f = [min(1.0 / (1.0 - float(tt)), 4.0) for tt in t]     # 1.25, 2.22.., 10 -> 4
    assert abs(loss - math.log(V) * sum(f) / 3) < 1e-12


def test_example_mean_skips_examples_without_scored_rows():
    canvas, clean, x, t, V = _canvas_case(25, pads=(6, 0, 3))
    ex, _ = _canvas_loss(canvas, clean, x, t, V, oracle.NO_TIME_WEIGHT, 0.0, oracle.EXAMPLE_MEAN)
    ce = torch_ce(x, clean).reshape(3, 6)
    assert abs(ex - (ce[0].mean() + ce[2, :3].mean()) / 2) < 1e-12


# --------------------------------------------------------------------------
# packed documents
# --------------------------------------------------------------------------
def test_packing_invariance_of_unit_sums():
    """The same documents packed with cu_seqlens or padded into rows with a
    pad mask give the same corruption, the same per-document sums and the
    same total (N = non-pad tokens in both)."""
    lens = [3, 17, 9, 1, 30]
    V = 61
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    T = int(cu[-1])
    rng = np.random.default_rng(11)
    clean_p = rng.integers(0, V - 1, T).astype(np.int32)
    xp = rng.standard_normal((T, V)) * 2
    lay_p = oracle.Layout(len(lens), 0, cu, None)
    Lmax = max(lens)
    clean_d = np.zeros(len(lens) * Lmax, np.int32)
    pad = np.ones(len(lens) * Lmax, np.uint8)
    xd = np.zeros((len(lens) * Lmax, V))
    for u, l in enumerate(lens):
        clean_d[u * Lmax:u * Lmax + l] = clean_p[cu[u]:cu[u + 1]]
        pad[u * Lmax:u * Lmax + l] = 0
        xd[u * Lmax:u * Lmax + l] = xp[cu[u]:cu[u + 1]]
    lay_d = oracle.Layout(len(lens), Lmax, None, pad)
    _, p = oracle.sample_t(3, len(lens), oracle.ABSORBING, 1e-3)
    for align in (oracle.ALIGNED, oracle.SHIFTED):
        _, cp = oracle.corrupt(lay_p, clean_p, p, oracle.ABSORBING, V - 1, V, 5)
        _, cd = oracle.corrupt(lay_d, clean_d, p, oracle.ABSORBING, V - 1, V, 5)
        lp, trp = _absorbing_loss_f64(xp, lay_p, clean_p, cp, p, align)
        ld, trd = _absorbing_loss_f64(xd, lay_d, clean_d, cd, p, align)
        _, up = oracle.reduce_units(len(lens), trp)
        _, ud = oracle.reduce_units(len(lens), trd)
        assert np.allclose(up, ud, rtol=1e-14, atol=1e-15)
        assert abs(lp - ld) < 1e-13


# --------------------------------------------------------------------------
# fused lm_head
# --------------------------------------------------------------------------
@pytest.mark.parametrize("align", [oracle.ALIGNED, oracle.SHIFTED])
def test_linear_equals_unfused_on_materialised_logits(align):
    rng = np.random.default_rng(12)
    T, D, V = 64, 64, 1000
    lens = [10, 30, 24]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    lay = oracle.Layout(3, 0, cu, None)
    H = bf16_bits_of(rng.standard_normal((T, D)).astype(np.float32))
    W = bf16_bits_of((rng.standard_normal((V, D)) * 0.02).astype(np.float32))
    clean = rng.integers(0, V - 1, T).astype(np.int32)
    _, p = oracle.sample_t(1, 3, oracle.ABSORBING, 1e-3)
    _, corr = oracle.corrupt(lay, clean, p, oracle.ABSORBING, V - 1, V, 2)
    out = oracle.linear_loss(lay, H, W, clean, corr, p, grad_scale=2.0, align=align)
    Z = oracle.bf16_to_f64(H) @ oracle.bf16_to_f64(W).T
    loss, tr = _absorbing_loss_f64(Z, lay, clean, corr, p, align)
    assert abs(out["loss"] - loss) < 1e-12 * max(1, loss)
    dZ = oracle.term_grad(Z, V, tr, np.arange(T), grad_scale=2.0)
    assert np.allclose(out["dH"], dZ @ oracle.bf16_to_f64(W), rtol=1e-10, atol=1e-14)
    assert np.allclose(out["dW"], dZ.T @ oracle.bf16_to_f64(H), rtol=1e-10, atol=1e-14)
    unscored = np.ones(T, bool); unscored[out["rows"]] = False
    assert (out["dH"][unscored] == 0).all()


def test_linear_finite_differences():
    """dH and dW against central differences of the fused loss (catches a
    transposed or missing operand)."""
    rng = np.random.default_rng(13)
    T, D, V = 6, 4, 7
    lay = oracle.Layout(1, T, None, None)
    Hf = rng.standard_normal((T, D))
    Wf = rng.standard_normal((V, D)) * 0.5
    clean = rng.integers(0, V, T).astype(np.int32)
    corr = np.array([1, 1, 0, 1, 0, 1], np.uint8)
    p = np.array([0.4], np.float32)

    def loss_of(Hm, Wm):
        Z = Hm @ Wm.T
        return _absorbing_loss_f64(Z, lay, clean, corr, p, oracle.ALIGNED)

    loss, tr = loss_of(Hf, Wf)
    dZ = oracle.term_grad(Hf @ Wf.T, V, tr, np.arange(T), 1.0)
    dH, dW = dZ @ Wf, dZ.T @ Hf
    h = 1e-6
    for (M, G, which) in ((Hf, dH, 0), (Wf, dW, 1)):
        fd = np.zeros_like(M)
        for idx in np.ndindex(*M.shape):
            Mp = M.copy(); Mp[idx] += h
            Mm = M.copy(); Mm[idx] -= h
            lp = loss_of(Mp, Wf)[0] if which == 0 else loss_of(Hf, Mp)[0]
            lm = loss_of(Mm, Wf)[0] if which == 0 else loss_of(Hf, Mm)[0]
            fd[idx] = (lp - lm) / (2 * h)
        assert np.abs(fd - G).max() < 1e-7
    # the oracle's fused entry on the same (bf16-representable) inputs
    Hb = bf16_bits_of(Hf.astype(np.float32)); Wb = bf16_bits_of(Wf.astype(np.float32))
    out = oracle.linear_loss(lay, Hb, Wb, clean, corr, p)
    Hq, Wq = oracle.bf16_to_f64(Hb), oracle.bf16_to_f64(Wb)
    lq, trq = loss_of(Hq, Wq)
    dZq = oracle.term_grad(Hq @ Wq.T, V, trq, np.arange(T), 1.0)
    assert abs(out["loss"] - lq) < 1e-12
    assert np.allclose(out["dH"], dZq @ Wq, atol=1e-13)
    assert np.allclose(out["dW"], dZq.T @ Hq, atol=1e-13)


def test_linear_rows_spot_check_matches_full():
    rng = np.random.default_rng(14)
    T, D, V = 48, 32, 300
    lay = oracle.Layout(2, 24, None, None)
    H = bf16_bits_of(rng.standard_normal((T, D)).astype(np.float32))
    W = bf16_bits_of((rng.standard_normal((V, D)) * 0.1).astype(np.float32))
    clean = rng.integers(0, V, T).astype(np.int32)
    _, p = oracle.sample_t(4, 2, oracle.ABSORBING, 1e-3)
    _, corr = oracle.corrupt(lay, clean, p, oracle.ABSORBING, V - 1, V, 4)
    full = oracle.linear_loss(lay, H, W, clean, corr, p, grad_scale=0.5)
    rows = full["rows"][::3]
    spot = oracle.linear_rows(lay, H, W, clean, corr, p, rows, grad_scale=0.5)
    pos = np.searchsorted(full["rows"], rows)
    assert np.allclose(spot["ce"], full["ce"][pos], rtol=1e-14)
    assert np.allclose(spot["dH"], full["dH"][rows], rtol=1e-12, atol=1e-15)


# --------------------------------------------------------------------------
# fused lm_head, uniform noise (canvas term + encoder AR term, one head)
# --------------------------------------------------------------------------
def _uniform_linear_case(seed, D=64, V=1000):
    rng = np.random.default_rng(seed)
    lens = [10, 30, 24]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    canvas = oracle.Layout(3, 0, cu, None)
    Le = 40                                   # encoder: dense [3, 40] with trailing pads
    pad = np.zeros(3 * Le, np.uint8)
    for u, n in enumerate((40, 33, 2)):
        pad[u * Le + n:(u + 1) * Le] = 1
    enc = oracle.Layout(3, Le, None, pad)
    H = bf16_bits_of(rng.standard_normal((64, D)).astype(np.float32))
    He = bf16_bits_of(rng.standard_normal((3 * Le, D)).astype(np.float32))
    W = bf16_bits_of((rng.standard_normal((V, D)) * 0.05).astype(np.float32))
    clean = rng.integers(0, V, 64).astype(np.int32)
    eclean = rng.integers(0, V, 3 * Le).astype(np.int32)
    return canvas, enc, H, He, W, clean, eclean


@pytest.mark.parametrize("align", [oracle.ALIGNED, oracle.SHIFTED])
def test_linear_uniform_equals_unfused_on_materialised_logits(align):
    """The fused uniform loss equals the unfused two-term loss on Z = H W^T
    and Ze = He W^T (double), with dH = dZ W, dHe = dZe W and dW the sum of
    both terms' dZ^T H."""
    canvas, enc, H, He, W, clean, eclean = _uniform_linear_case(21)
    V = W.shape[0]
    lam, g = 0.7, 1.5
    out = oracle.linear_loss_uniform(canvas, H, W, clean, enc, He, eclean, lam, align, grad_scale=g)
    Hd, Hed, Wd = oracle.bf16_to_f64(H), oracle.bf16_to_f64(He), oracle.bf16_to_f64(W)
    Z, Ze = Hd @ Wd.T, Hed @ Wd.T
    loss, unit, tc, te = oracle.loss_uniform(canvas, Z, clean, enc, Ze, eclean, V, lam, align)
    assert abs(out["loss"] - loss) < 1e-12 * max(1.0, loss)
    assert np.allclose(out["unit_loss"], unit, rtol=1e-12, atol=1e-15)
    dZ = oracle.term_grad(Z, V, tc, np.arange(64), g)
    dZe = oracle.term_grad(Ze, V, te, np.arange(120), g)
    assert np.allclose(out["dH"], dZ @ Wd, rtol=1e-10, atol=1e-14)
    assert np.allclose(out["dHe"], dZe @ Wd, rtol=1e-10, atol=1e-14)
    assert np.allclose(out["dW"], dZ.T @ Hd + dZe.T @ Hed, rtol=1e-10, atol=1e-14)
    # rows with no target: the last row of each unit when shifted (canvas),
    # the last non-pad token of each unit and every pad row (encoder)
    n_c = 64 - (3 if align == oracle.SHIFTED else 0)
    assert out["rows"].shape[0] == n_c and out["enc_rows"].shape[0] == 39 + 32 + 1
    unscored = np.ones(120, bool); unscored[out["enc_rows"]] = False
    assert (out["dHe"][unscored] == 0).all()


def test_linear_uniform_finite_differences():
    """d loss / d(H, He, W) of the two-term loss against central differences
    (a transposed operand or a dropped encoder share of dW fails)."""
    rng = np.random.default_rng(22)
    D, V = 3, 5
    canvas = oracle.Layout(1, 4, None, None)
    enc = oracle.Layout(1, 5, None, None)
    Hf = rng.standard_normal((4, D))
    Hef = rng.standard_normal((5, D))
    Wf = rng.standard_normal((V, D)) * 0.5
    clean = rng.integers(0, V, 4).astype(np.int32)
    eclean = rng.integers(0, V, 5).astype(np.int32)
    lam = 0.3

    def loss_of(Hm, Hem, Wm):
        return oracle.loss_uniform(canvas, Hm @ Wm.T, clean, enc, Hem @ Wm.T, eclean, V, lam)

    loss, _, tc, te = loss_of(Hf, Hef, Wf)
    dZ = oracle.term_grad(Hf @ Wf.T, V, tc, np.arange(4), 1.0)
    dZe = oracle.term_grad(Hef @ Wf.T, V, te, np.arange(5), 1.0)
    grads = (dZ @ Wf, dZe @ Wf, dZ.T @ Hf + dZe.T @ Hef)
    h = 1e-6
    args = [Hf, Hef, Wf]
    for which, G in enumerate(grads):
        fd = np.zeros_like(args[which])
        for idx in np.ndindex(*fd.shape):
            ap = [a.copy() for a in args]; ap[which][idx] += h
            am = [a.copy() for a in args]; am[which][idx] -= h
            fd[idx] = (loss_of(*ap)[0] - loss_of(*am)[0]) / (2 * h)
        assert np.abs(fd - G).max() < 1e-7
    # the oracle's fused entry on the same inputs rounded to bf16
    Hb, Heb, Wb = (bf16_bits_of(a.astype(np.float32)) for a in (Hf, Hef, Wf))
    out = oracle.linear_loss_uniform(canvas, Hb, Wb, clean, enc, Heb, eclean, lam)
    Hq, Heq, Wq = (oracle.bf16_to_f64(a) for a in (Hb, Heb, Wb))
    lq, _, tcq, teq = loss_of(Hq, Heq, Wq)
    dZq = oracle.term_grad(Hq @ Wq.T, V, tcq, np.arange(4), 1.0)
    dZeq = oracle.term_grad(Heq @ Wq.T, V, teq, np.arange(5), 1.0)
    assert abs(out["loss"] - lq) < 1e-12
    assert np.allclose(out["dH"], dZq @ Wq, atol=1e-13)
    assert np.allclose(out["dHe"], dZeq @ Wq, atol=1e-13)
    assert np.allclose(out["dW"], dZq.T @ Hq + dZeq.T @ Heq, atol=1e-13)


def test_linear_uniform_without_encoder_is_lambda_zero():
    canvas, enc, H, He, W, clean, eclean = _uniform_linear_case(23, D=32, V=300)
    a = oracle.linear_loss_uniform(canvas, H, W, clean, None, None, None, 0.0)
    b = oracle.linear_loss_uniform(canvas, H, W, clean, enc, He, eclean, 0.0)
    assert a["loss"] == b["loss"]
    assert np.array_equal(a["dH"], b["dH"]) and np.array_equal(a["dW"], b["dW"])
    assert (b["dHe"] == 0).all()
    # every canvas row is scored with weight 1/64 (aligned, no pads)
    assert a["rows"].shape[0] == 64 and np.allclose(a["plan"].weight, 1 / 64)


def test_linear_rows_plan_spot_check_matches_full():
    canvas, enc, H, He, W, clean, eclean = _uniform_linear_case(24, D=32, V=300)
    full = oracle.linear_loss_uniform(canvas, H, W, clean, enc, He, eclean, 0.5, oracle.SHIFTED, 0.25)
    rows = full["enc_rows"][::5]
    spot = oracle.linear_rows_plan(full["enc_plan"], He, W, rows, 0.25)
    pos = np.searchsorted(full["enc_rows"], rows)
    assert np.allclose(spot["ce"], full["enc_ce"][pos], rtol=1e-14)
    assert np.allclose(spot["dH"], full["dHe"][rows], rtol=1e-12, atol=1e-15)
    rows = full["rows"][1::4]
    spot = oracle.linear_rows_plan(full["plan"], H, W, rows, 0.25)
    assert np.allclose(spot["dH"], full["dH"][rows], rtol=1e-12, atol=1e-15)
