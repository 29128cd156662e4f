"""The oracle's pins catch plausible mistakes.

Each case plants one mistake in the oracle -- on the CPU, by wrapping one of
its functions for the duration of the test -- then runs every pin of the
oracle's test modules against the mutated oracle and requires at least one
pin to fail.  The mistakes are the kind a reader could make writing the
oracle from the pages: a dropped term or factor, a wrong sign, an index off
by one, an operand or a share left out.  A mutation no pin notices would mean
a part of the oracle that nothing independent checks.
"""
import inspect
import itertools

import numpy as np
import pytest

import oracle
import test_oracle_decision as decision_pins
import test_oracle_hash as hash_pins
import test_oracle_loss as loss_pins


def _expand(fn):
    """Keyword sets of a pin's parametrize marks (one empty set if none)."""
    marks = [m for m in getattr(fn, "pytestmark", []) if m.name == "parametrize"]
    grids = []
    for m in marks:
        names = m.args[0].split(",") if isinstance(m.args[0], str) else list(m.args[0])
        names = [n.strip() for n in names]
        grids.append([dict(zip(names, v if len(names) > 1 else (v,))) for v in m.args[1]])
    for combo in itertools.product(*grids):
        kw = {}
        for c in combo:
            kw.update(c)
        yield kw


def _failing_pins(*modules):
    failed = []
    for mod in modules:
        for name, fn in inspect.getmembers(mod, inspect.isfunction):
            if not name.startswith("test_") or fn.__module__ != mod.__name__:
                continue
            for kw in _expand(fn):
                try:
                    fn(**kw)
                except Exception as e:          # AssertionError, or the mutation broke a shape
                    failed.append(f"{name}{kw if kw else ''}: {type(e).__name__}")
                    break
    return failed


def _wrap(monkeypatch, name, make):
    real = getattr(oracle, name)
    monkeypatch.setattr(oracle, name, make(real))


# ---- mistakes in the per-row CE and gradient ------------------------------
def m_ce_without_target_logit(real):
    def f(logits, vocab, rows, targets):
        lse, ce = real(logits, vocab, rows, targets)
        return lse, lse                          # ce = lse: the target logit dropped
    return f


def m_ce_target_off_by_one(real):
    def f(logits, vocab, rows, targets):
        return real(logits, vocab, rows, (np.asarray(targets) + 1) % vocab)
    return f


def m_grad_sign(real):
    def f(logits, vocab, rows, targets, coef, lse):
        return -real(logits, vocab, rows, targets, coef, lse)
    return f


def m_grad_without_onehot(real):
    def f(logits, vocab, rows, targets, coef, lse):
        g = real(logits, vocab, rows, targets, coef, lse)
        if g.shape[0]:
            g[np.arange(g.shape[0]), np.asarray(targets)] += np.asarray(coef, np.float64)
        return g
    return f


def m_bf16_low_bit(real):
    def f(a):
        return real(np.asarray(a, np.uint16) & np.uint16(0xFFFE))
    return f


# ---- mistakes in the row plan and the weights -----------------------------
def m_absorbing_without_inverse_p(real):
    def f(layout, clean, corrupted, p, mode, align, *a, **kw):
        plan = real(layout, clean, corrupted, p, mode, align, *a, **kw)
        if mode == oracle.ABSORBING:
            s = plan.target >= 0
            plan.weight[s] *= p[plan.unit[s]].astype(np.float64)
        return plan
    return f


def m_normaliser_plus_one(real):
    def f(layout, clean, corrupted, p, mode, align, *a, **kw):
        plan = real(layout, clean, corrupted, p, mode, align, *a, **kw)
        if mode == oracle.ABSORBING:
            N = int(layout.nonpad().sum())
            plan.weight *= N / (N + 1.0)
        return plan
    return f


def m_shift_forgotten(real):
    def f(layout, clean, corrupted, p, mode, align, *a, **kw):
        plan = real(layout, clean, corrupted, p, mode, align, *a, **kw)
        if align == oracle.SHIFTED:
            s = np.nonzero(plan.target >= 0)[0]
            plan.target[s] = np.asarray(clean)[s]  # scores token i instead of i + 1
        return plan
    return f


def m_encoder_without_lambda(real):
    def f(layout, clean, lam):
        plan = real(layout, clean, lam)
        if lam != 0:
            plan.weight /= lam
        return plan
    return f


def m_encoder_crosses_units(real):
    def f(layout, clean, lam):
        plan = real(layout, clean, lam)
        n = layout.n_tokens
        nonpad = layout.nonpad()
        leak = [i for i in range(n - 1) if plan.target[i] < 0 and nonpad[i + 1]]
        if leak:
            cnt = int((plan.target >= 0).sum()) + len(leak)
            plan.target[leak] = np.asarray(clean)[np.asarray(leak) + 1]
            plan.weight[:] = 0.0
            plan.weight[plan.target >= 0] = lam / cnt
        return plan
    return f


def m_reduce_wrong_unit(real):
    def f(n_units, *terms):
        unit_loss = np.zeros(n_units, np.float64)
        for tr in terms:
            np.add.at(unit_loss, (tr.plan.unit + 1) % max(n_units, 1), tr.row_loss)
        return float(unit_loss.sum()), unit_loss
    return f


def m_rhine_cap_ignored(real):
    def f(layout, clean, corrupted, p, mode, align, time_weighting=oracle.NO_TIME_WEIGHT, weight_clip=0.0,
          reduction=oracle.TOKEN_MEAN):
        return real(layout, clean, corrupted, p, mode, align, time_weighting, 0.0, reduction)
    return f


def m_example_mean_over_all_examples(real):
    def f(layout, clean, corrupted, p, mode, align, time_weighting=oracle.NO_TIME_WEIGHT, weight_clip=0.0,
          reduction=oracle.TOKEN_MEAN):
        plan = real(layout, clean, corrupted, p, mode, align, time_weighting, weight_clip, reduction)
        if reduction == oracle.EXAMPLE_MEAN and layout.n_units > 0:
            b_eff = len(set(plan.unit[plan.target >= 0].tolist()))
            plan.weight *= b_eff / layout.n_units
        return plan
    return f


def m_rhine_inverse_t(real):
    def f(layout, clean, corrupted, p, mode, align, time_weighting=oracle.NO_TIME_WEIGHT, weight_clip=0.0,
          reduction=oracle.TOKEN_MEAN):
        plan = real(layout, clean, corrupted, p, mode, align, time_weighting, weight_clip, reduction)
        if time_weighting == oracle.INV_ONE_MINUS_T:
            t = p.astype(np.float64)
            right = 1.0 / (1.0 - t)
            wrong = 1.0 / t
            if weight_clip > 0:
                right, wrong = np.minimum(right, weight_clip), np.minimum(wrong, weight_clip)
            s = plan.target >= 0
            plan.weight[s] *= (wrong / right)[plan.unit[s]]
        return plan
    return f


def m_encoder_scores_pads(real):
    def f(layout, clean, lam):
        plan = real(layout, clean, lam)
        unit = layout.unit_of_token()
        nonpad = layout.nonpad()
        extra = [i for i in range(layout.n_tokens - 1)
                 if plan.target[i] < 0 and unit[i + 1] == unit[i] and not nonpad[i + 1]]
        if extra:
            plan.target[extra] = np.asarray(clean)[np.asarray(extra) + 1]
            cnt = int((plan.target >= 0).sum())
            plan.weight[:] = 0.0
            plan.weight[plan.target >= 0] = lam / cnt
        return plan
    return f


# ---- mistakes in the fused head -------------------------------------------
def m_linear_dw_dropped(real):
    def f(plan, H, W, grad_scale, want_grads, keep_dz=False):
        out = real(plan, H, W, grad_scale, want_grads, keep_dz)
        return out[:5] + ((None if out[5] is None else np.zeros_like(out[5])),) + out[6:]
    return f


def m_linear_dh_on_wrong_rows(real):
    def f(plan, H, W, grad_scale, want_grads, keep_dz=False):
        rows, lse, ce, row_loss, dH, dW, dZ = real(plan, H, W, grad_scale, want_grads, keep_dz)
        if dH is not None and rows.size > 1:
            dH[rows] = dH[rows[::-1]]              # gradients land on the wrong rows
        return rows, lse, ce, row_loss, dH, dW, dZ
    return f


def m_linear_uniform_encoder_dw_dropped(real):
    def f(canvas, H, W, canvas_clean, encoder, He, enc_clean, lam, *a, **kw):
        out = real(canvas, H, W, canvas_clean, encoder, He, enc_clean, lam, *a, **kw)
        if encoder is not None and "dW" in out:
            alone = real(canvas, H, W, canvas_clean, None, None, None, lam, *a, **kw)
            out["dW"] = alone["dW"]
        return out
    return f


# ---- mistakes in the time draw and the corruption --------------------------
def m_p_without_eps_floor(real):
    def f(seed, n_units, mode, eps):
        t, p = real(seed, n_units, mode, eps)
        return (t, t.copy()) if mode == oracle.ABSORBING else (t, p)
    return f


def m_pads_corrupted(real):
    def f(layout, clean, p, mode, mask_id, vocab, seed):
        noisy, corr = real(layout, clean, p, mode, mask_id, vocab, seed)
        if layout.pad_mask is not None:
            pad = np.asarray(layout.pad_mask).astype(bool)
            corr = corr.copy()
            corr[pad] = 1
        return noisy, corr
    return f


def m_counter_fields_swapped(real):
    def f(stream, unit, pos):
        return real(stream, pos, unit) if pos < (1 << 24) else real(stream, unit, pos)
    return f


MUTATIONS = [
    ("ce_rows", m_ce_without_target_logit, (loss_pins,)),
    ("ce_rows", m_ce_target_off_by_one, (loss_pins,)),
    ("grad_rows", m_grad_sign, (loss_pins,)),
    ("grad_rows", m_grad_without_onehot, (loss_pins,)),
    ("bf16_to_f64", m_bf16_low_bit, (loss_pins,)),
    ("plan_diffusion", m_absorbing_without_inverse_p, (loss_pins,)),
    ("plan_diffusion", m_normaliser_plus_one, (loss_pins,)),
    ("plan_diffusion", m_shift_forgotten, (loss_pins,)),
    ("plan_encoder", m_encoder_without_lambda, (loss_pins,)),
    ("plan_encoder", m_encoder_crosses_units, (loss_pins,)),
    ("reduce_units", m_reduce_wrong_unit, (loss_pins,)),
    ("plan_diffusion", m_rhine_cap_ignored, (loss_pins,)),
    ("plan_diffusion", m_example_mean_over_all_examples, (loss_pins,)),
    ("plan_diffusion", m_rhine_inverse_t, (loss_pins,)),
    ("plan_encoder", m_encoder_scores_pads, (loss_pins,)),
    ("_linear_term", m_linear_dw_dropped, (loss_pins,)),
    ("_linear_term", m_linear_dh_on_wrong_rows, (loss_pins,)),
    ("linear_loss_uniform", m_linear_uniform_encoder_dw_dropped, (loss_pins,)),
    ("sample_t", m_p_without_eps_floor, (hash_pins, loss_pins)),
    ("corrupt", m_pads_corrupted, (hash_pins,)),
    ("counter", m_counter_fields_swapped, (hash_pins,)),
]


@pytest.mark.parametrize("target,mutation,modules", MUTATIONS,
                         ids=[m[1].__name__[2:] for m in MUTATIONS])
def test_a_planted_mistake_fails_a_pin(monkeypatch, target, mutation, modules):
    _wrap(monkeypatch, target, mutation)
    failed = _failing_pins(*modules)
    assert failed, f"no pin notices the mistake {mutation.__name__[2:]} in oracle.{target}"


def test_control_every_pin_passes_on_the_unmutated_oracle():
    assert _failing_pins(loss_pins, hash_pins, decision_pins) == []


# ---- mistakes in the typed-decision losses ---------------------------------
# Each case copies the source of one oracle function, makes one textual
# change, compiles the copy with the oracle module's globals and puts it in
# the function's place for the duration of the test.
PY_MUTATIONS = [
    ("decision_loss", "full_ce_over_the_answers_only",
     "ce_full[i] = -(q * (c - lse)).sum()", "ce_full[i] = -(q * (c - lse_r)).sum()"),
    ("decision_loss", "brier_on_the_full_softmax",
     "brier[i] = ((r - y) ** 2).sum()", "brier[i] = ((P[a] - y) ** 2).sum()"),
    ("decision_loss", "restricted_gradient_sign", "g[a] += Q * r - q", "g[a] -= Q * r - q"),
    ("decision_loss", "full_gradient_without_onehot", "g[a] -= q\n", "g[a] -= 0.0 * q\n"),
    ("decision_loss", "brier_gradient_without_its_mean",
     "g[a] += brier_weight * 2.0 * r * (d - (r * d).sum())", "g[a] += brier_weight * 2.0 * r * d"),
    ("decision_loss", "brier_weight_dropped",
     "per_slot = (ce_res * use_res + ce_full * use_full + brier_weight * brier) * w",
     "per_slot = (ce_res * use_res + ce_full * use_full + brier) * w"),
    ("decision_loss", "sum_over_slots_not_mean", "w = 1.0 / n if n > 0 else 0.0", "w = 1.0"),
    ("decision_targets", "smoothing_not_spread_over_the_answers",
     "q = (1.0 - smoothing) * y + smoothing / K", "q = (1.0 - smoothing) * y + smoothing"),
    ("decision_targets", "smoothing_applied_to_brier",
     "y = val.copy()\n        q = (1.0 - smoothing) * y + smoothing / K",
     "y = (1.0 - smoothing) * val + smoothing / K\n        q = y.copy()"),
    ("decision_targets", "set_target_not_normalised", "y = val / val.sum()", "y = val.copy()"),
]


@pytest.mark.parametrize("fn,old,new", [m[::2][:1] + m[2:] for m in PY_MUTATIONS],
                         ids=[m[1] for m in PY_MUTATIONS])
def test_a_planted_mistake_in_the_decision_oracle_fails_a_pin(monkeypatch, fn, old, new):
    import textwrap
    src = textwrap.dedent(inspect.getsource(getattr(oracle, fn)))
    assert src.count(old) == 1, old
    ns = dict(vars(oracle))
    exec(compile(src.replace(old, new), f"<mutated {fn}>", "exec"), ns)
    monkeypatch.setattr(oracle, fn, ns[fn])
    failed = _failing_pins(decision_pins)
    assert failed, f"no pin notices the change {old!r} -> {new!r} in oracle.{fn}"


# ---- mistakes in the C part of the oracle ---------------------------------
# Each case copies the oracle's C source, makes one textual change, compiles
# the copy into the test's temporary directory and points the oracle at it;
# the oracle's own source and library are not touched.
C_MUTATIONS = [
    ("splitmix_gamma", "#define DLMO_GAMMA 0x9E3779B97F4A7C15ULL", "#define DLMO_GAMMA 0x9E3779B97F4A7C17ULL"),
    ("finaliser_shift", "z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;", "z = (z ^ (z >> 29)) * 0xBF58476D1CE4E5B9ULL;"),
    ("u24_cut", "return (uint32_t)(h >> 40);", "return (uint32_t)(h >> 41);"),
    ("threshold_not_strict", "int c = (float)u24_of(h1) < thr;", "int c = (float)u24_of(h1) <= thr;"),
    ("replacement_shift", "(uint64_t)(uint32_t)vocab) >> 32);", "(uint64_t)(uint32_t)vocab) >> 31);"),
    ("uniform_t_without_floor", "else           { t[u] = v; p[u] = v; }", "else           { t[u] = x; p[u] = v; }"),
    ("time_draw_stream", "dlmo_counter(0, (uint32_t)u, 0)", "dlmo_counter(1, (uint32_t)u, 0)"),
    ("lse_without_max", "return m + log(s);", "return log(s);"),
    ("bf16_decode_shift", "uint32_t w = (uint32_t)b << 16;", "uint32_t w = (uint32_t)b << 15;"),
    ("grad_bf16_onehot_sign", "o[v] = coef[k] * (exp(buf[v] - lse[k]) - (v == targets[k] ? 1.0 : 0.0));",
     "o[v] = coef[k] * (exp(buf[v] - lse[k]) + (v == targets[k] ? 1.0 : 0.0));"),
    ("grad_f64_onehot_sign", "o[v] = coef[k] * (exp(x[v] - lse[k]) - (v == targets[k] ? 1.0 : 0.0));",
     "o[v] = coef[k] * (exp(x[v] - lse[k]) + (v == targets[k] ? 1.0 : 0.0));"),
    ("pads_not_skipped", "if (pad_mask && pad_mask[i])", "if (0 && pad_mask)"),
    ("document_bound", "if (i >= cu[u] && i < cu[u + 1])", "if (i >= cu[u] && i <= cu[u + 1])"),
]


@pytest.mark.parametrize("old,new", [m[1:] for m in C_MUTATIONS], ids=[m[0] for m in C_MUTATIONS])
def test_a_planted_mistake_in_the_c_oracle_fails_a_pin(monkeypatch, tmp_path, old, new):
    import subprocess
    src = open(oracle._build.SRC).read()
    assert src.count(old) == 1, old
    mutated = tmp_path / "dlm_oracle_mutated.c"
    mutated.write_text(src.replace(old, new))
    lib = tmp_path / "liboracle_mutated.so"
    subprocess.run(["gcc", "-O2", "-std=c99", "-fopenmp", "-ffp-contract=off", "-fno-fast-math", "-shared",
                    "-fPIC", "-o", str(lib), str(mutated), "-lm"], check=True)
    monkeypatch.setattr(oracle._build, "build", lambda *a, **kw: str(lib))
    monkeypatch.setattr(oracle, "_lib", None)
    failed = _failing_pins(loss_pins, hash_pins)
    assert failed, f"no pin notices the change {old!r} -> {new!r}"
