"""CPU oracle for the diffusion-LM noising-plus-loss path.

TEST INFRASTRUCTURE ONLY.  Only the test suite, the package entry point's
``smoke()`` check and the CPU-baseline leg of ``bench.py`` may import this
module.  The product path never does, and this module imports nothing from
the product package: the two share no code.  The only module both sides use
is ``dlm_inputs`` (seeded synthetic inputs; none of the method's arithmetic).

Scalar loops (hash, corruption, per-row CE in double) are in
``dlm_oracle.c``; this file orchestrates them and holds the row plan, the
weights and the reductions, written in numpy float64.

Sources (page title, section):
  [LLaDA]   "LLaDA-8B-MDLM-LoRA", Training table, row "Objective".
  [Axolotl] "Native diffusion language-model training": model table
            (noise, alignment, objective per model); "Packed training";
            "Adapters, merging and inference" (Cut Cross Entropy: full-vocab
            CE from hidden states, aligned targets, plain linear head).
  [Gemma]   "diffusiongemma-26B-A4B-it-ALWAYS-THINK", Finetuning notes.

Readings where the pages are silent (each listed in the design notes):
  * loss normaliser for absorbing noise = number of non-pad tokens N;
  * shifted rows: row i scores token i+1 of the same unit; each unit's last
    row is unscored; position 0 may be corrupted but no row scores it;
  * uniform canvas: every non-pad canvas target is scored, mean over them;
  * encoder AR: row i scores token i+1 of the same unit, mean over pairs;
  * the softmax runs over the whole vocabulary, mask-id column included.

Pins: every function here is checked, in ``tests/test_oracle_*.py``, against
something other than itself (published SplitMix64 vectors, a sequential
re-derivation, closed forms, finite differences, a textbook log-softmax,
binomial/chi-square statistics).  The end-to-end loss value has no worked
example on the pages: parity unpinned for the whole-pipeline number itself
(its parts are pinned).
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional

import numpy as np

from . import build as _build

ABSORBING, UNIFORM = 0, 1
ALIGNED, SHIFTED = 0, 1
# uniform-noise objective options ([Gemma] "Rhine objectives", page
# "Native diffusion language-model training", Objective and recurrence options)
NO_TIME_WEIGHT, INV_ONE_MINUS_T = 0, 1
TOKEN_MEAN, EXAMPLE_MEAN = 0, 1

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        u64, i64, i32, f32 = ctypes.c_uint64, ctypes.c_int64, ctypes.c_int32, ctypes.c_float
        vp = ctypes.c_void_p
        L.dlmo_splitmix64_at.restype = u64
        L.dlmo_splitmix64_at.argtypes = [u64, u64]
        L.dlmo_counter.restype = u64
        L.dlmo_counter.argtypes = [ctypes.c_uint32, ctypes.c_uint32, ctypes.c_uint32]
        L.dlmo_sample_t.restype = None
        L.dlmo_sample_t.argtypes = [u64, i32, i32, f32, vp, vp]
        L.dlmo_corrupt.restype = ctypes.c_int
        L.dlmo_corrupt.argtypes = [i32, i32, vp, vp, i64, vp, vp, i32, i32, i32, u64, vp, vp]
        for name in ("dlmo_ce_rows_bf16", "dlmo_ce_rows_f64"):
            f = getattr(L, name)
            f.restype = None
            f.argtypes = [vp, i64, i32, i64, vp, vp, vp, vp]
        for name in ("dlmo_grad_rows_bf16", "dlmo_grad_rows_f64"):
            f = getattr(L, name)
            f.restype = None
            f.argtypes = [vp, i64, i32, i64, vp, vp, vp, vp, vp]
        L.dlmo_bf16_to_f64.restype = None
        L.dlmo_bf16_to_f64.argtypes = [vp, i64, vp]
        _lib = L
    return _lib


def _p(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


# --------------------------------------------------------------------------
# Layout of tokens into units (sequences or packed documents)
# --------------------------------------------------------------------------
@dataclass
class Layout:
    """n_units sequences of seq_len tokens (cu_seqlens None), or n_units
    packed documents delimited by cu_seqlens [n_units+1]; pad_mask [n_tokens]
    with 1 = pad, or None."""
    n_units: int
    seq_len: int
    cu_seqlens: Optional[np.ndarray]
    pad_mask: Optional[np.ndarray]

    @property
    def n_tokens(self) -> int:
        if self.cu_seqlens is None:
            return self.n_units * self.seq_len
        return int(self.cu_seqlens[-1])

    def unit_of_token(self) -> np.ndarray:
        n = self.n_tokens
        if self.cu_seqlens is None:
            return np.arange(n, dtype=np.int64) // self.seq_len
        unit = np.empty(n, dtype=np.int64)
        cu = self.cu_seqlens
        for u in range(self.n_units):
            unit[cu[u]:cu[u + 1]] = u
        return unit

    def nonpad(self) -> np.ndarray:
        if self.pad_mask is None:
            return np.ones(self.n_tokens, dtype=bool)
        return self.pad_mask == 0


# --------------------------------------------------------------------------
# Hash, time draw, corruption  (C loops)
# --------------------------------------------------------------------------
def splitmix64_at(seed: int, counter: int) -> int:
    return int(lib().dlmo_splitmix64_at(seed, counter))


def counter(stream: int, unit: int, pos: int) -> int:
    return int(lib().dlmo_counter(stream, unit, pos))


def sample_t(seed: int, n_units: int, mode: int, eps: float):
    """[LLaDA] absorbing: t ~ U(0,1), p = (1-eps) t + eps.
    [Gemma] uniform: t ~ U(eps,1), p = t.  Returns float32 (t, p)."""
    t = np.zeros(n_units, np.float32)
    p = np.zeros(n_units, np.float32)
    lib().dlmo_sample_t(seed, n_units, mode, ctypes.c_float(eps), _p(t), _p(p))
    return t, p


def corrupt(layout: Layout, clean: np.ndarray, p: np.ndarray, mode: int,
            mask_id: int, vocab: int, seed: int):
    """[LLaDA]/[Gemma] seeded corruption; returns (noisy int32, corrupted uint8)."""
    clean = np.ascontiguousarray(clean, np.int32)
    p = np.ascontiguousarray(p, np.float32)
    n = layout.n_tokens
    noisy = np.zeros(n, np.int32)
    corr = np.zeros(n, np.uint8)
    cu = None if layout.cu_seqlens is None else np.ascontiguousarray(layout.cu_seqlens, np.int32)
    pm = None if layout.pad_mask is None else np.ascontiguousarray(layout.pad_mask, np.uint8)
    rc = lib().dlmo_corrupt(layout.n_units, layout.seq_len, _p(cu), _p(pm), n, _p(clean),
                            _p(p), mode, mask_id, vocab, seed, _p(noisy), _p(corr))
    if rc != 0:
        raise ValueError("inconsistent layout")
    return noisy, corr


# --------------------------------------------------------------------------
# Row plan: which logits row is scored, against which target, with what weight
# --------------------------------------------------------------------------
@dataclass
class RowPlan:
    target: np.ndarray   # int64 [rows], -1 = unscored
    unit: np.ndarray     # int64 [rows]
    weight: np.ndarray   # float64 [rows], 0 on unscored rows


def plan_diffusion(layout: Layout, clean: np.ndarray, corrupted: Optional[np.ndarray],
                   p: Optional[np.ndarray], mode: int, align: int,
                   time_weighting: int = NO_TIME_WEIGHT, weight_clip: float = 0.0,
                   reduction: int = TOKEN_MEAN) -> RowPlan:
    """Diffusion term.  Row i scores token j = i (aligned) or j = i+1 of the
    same unit (shifted; [Axolotl] model table: Dream's logit i predicts token
    i+1).  The target must be a non-pad token; absorbing noise additionally
    requires it to be corrupted ([LLaDA]: CE on masked tokens).
      absorbing: weight = 1 / (p_unit * N), N = non-pad tokens in the call.
      uniform:   weight = f_unit / (number of scored canvas rows)  (mean, [Gemma]),
                 or, with reduction EXAMPLE_MEAN, f_unit / (B' * n_unit): the
                 mean over each example's scored rows, then over the B'
                 examples that have any ([Axolotl] Objective options:
                 objective_reduction example_mean).
                 f_unit = 1, or with time weighting INV_ONE_MINUS_T
                 min(1 / (1 - t_unit), clip) (no cap when clip <= 0), t = p for
                 uniform noise ([Axolotl]: Rhine objectives, rhine_weight_clip
                 caps the 1 / (1 - t) weights).
    """
    n = layout.n_tokens
    unit = layout.unit_of_token()
    nonpad = layout.nonpad()
    target = np.full(n, -1, np.int64)
    weight = np.zeros(n, np.float64)
    if align == ALIGNED:
        j = np.arange(n)
        ok = nonpad.copy()
    else:
        j = np.arange(n) + 1
        ok = np.zeros(n, bool)
        ok[:-1] = (unit[1:] == unit[:-1]) & nonpad[1:]
        j = np.minimum(j, n - 1)
    if mode == ABSORBING:
        ok &= corrupted[j].astype(bool)
    target[ok] = clean[j[ok]]
    if mode == ABSORBING:
        N = int(nonpad.sum())
        if N > 0:
            weight[ok] = 1.0 / (p[unit[ok]].astype(np.float64) * N)
    else:
        f = np.ones(n, np.float64)
        if time_weighting == INV_ONE_MINUS_T:
            fu = 1.0 / (1.0 - p.astype(np.float64))
            if weight_clip > 0:
                fu = np.minimum(fu, float(weight_clip))
            f = fu[unit]
        if reduction == TOKEN_MEAN:
            cnt = int(ok.sum())
            if cnt > 0:
                weight[ok] = f[ok] / cnt
        else:
            n_u = np.bincount(unit[ok], minlength=layout.n_units)
            b_eff = int((n_u > 0).sum())
            if b_eff > 0:
                weight[ok] = f[ok] / (b_eff * n_u[unit[ok]])
    return RowPlan(target, unit, weight)


def plan_encoder(layout: Layout, clean: np.ndarray, lam: float) -> RowPlan:
    """[Gemma] encoder AR term: plain causal next-token CE over the clean full
    sequence.  Row i scores token i+1 of the same unit (non-pad); weight =
    lam / (number of such pairs)."""
    n = layout.n_tokens
    unit = layout.unit_of_token()
    nonpad = layout.nonpad()
    ok = np.zeros(n, bool)
    ok[:-1] = (unit[1:] == unit[:-1]) & nonpad[1:]
    target = np.full(n, -1, np.int64)
    target[:-1][ok[:-1]] = clean[1:][ok[:-1]]
    weight = np.zeros(n, np.float64)
    cnt = int(ok.sum())
    if cnt > 0:
        weight[ok] = lam / cnt
    return RowPlan(target, unit, weight)


# --------------------------------------------------------------------------
# Per-row CE and gradient over a logits matrix (C loops, double)
# --------------------------------------------------------------------------
def ce_rows(logits: np.ndarray, vocab: int, rows: np.ndarray, targets: np.ndarray):
    """(lse, ce) in double for the listed rows.  `logits` is a 2-D uint16
    array of bf16 bit patterns [rows_total, ld] or a 2-D float64 array."""
    rows = np.ascontiguousarray(rows, np.int64)
    targets = np.ascontiguousarray(targets, np.int32)
    n = rows.shape[0]
    lse = np.zeros(n, np.float64)
    ce = np.zeros(n, np.float64)
    if n == 0:
        return lse, ce
    assert logits.flags.c_contiguous
    ld = logits.shape[1]
    if logits.dtype == np.uint16:
        lib().dlmo_ce_rows_bf16(_p(logits), ld, vocab, n, _p(rows), _p(targets), _p(lse), _p(ce))
    elif logits.dtype == np.float64:
        lib().dlmo_ce_rows_f64(_p(logits), ld, vocab, n, _p(rows), _p(targets), _p(lse), _p(ce))
    else:
        raise TypeError(logits.dtype)
    return lse, ce


def grad_rows(logits: np.ndarray, vocab: int, rows: np.ndarray, targets: np.ndarray,
              coef: np.ndarray, lse: np.ndarray) -> np.ndarray:
    """coef_k * (softmax(row_k) - onehot(target_k)) in double, [n, vocab]."""
    rows = np.ascontiguousarray(rows, np.int64)
    targets = np.ascontiguousarray(targets, np.int32)
    coef = np.ascontiguousarray(coef, np.float64)
    lse = np.ascontiguousarray(lse, np.float64)
    n = rows.shape[0]
    out = np.zeros((n, vocab), np.float64)
    if n == 0:
        return out
    ld = logits.shape[1]
    if logits.dtype == np.uint16:
        lib().dlmo_grad_rows_bf16(_p(logits), ld, vocab, n, _p(rows), _p(targets), _p(coef),
                                  _p(lse), _p(out))
    else:
        lib().dlmo_grad_rows_f64(_p(logits), ld, vocab, n, _p(rows), _p(targets), _p(coef),
                                 _p(lse), _p(out))
    return out


def bf16_to_f64(a: np.ndarray) -> np.ndarray:
    a = np.ascontiguousarray(a, np.uint16)
    out = np.empty(a.shape, np.float64)
    lib().dlmo_bf16_to_f64(_p(a), a.size, _p(out))
    return out


# --------------------------------------------------------------------------
# The loss over one logits tensor, and the two-term uniform loss
# --------------------------------------------------------------------------
@dataclass
class TermResult:
    plan: RowPlan
    rows: np.ndarray      # scored row indices
    lse: np.ndarray       # per scored row
    ce: np.ndarray        # per scored row
    row_loss: np.ndarray  # [rows_total] weight * ce, 0 on unscored rows


def term(logits: np.ndarray, vocab: int, plan: RowPlan) -> TermResult:
    rows = np.nonzero(plan.target >= 0)[0]
    lse, ce = ce_rows(logits, vocab, rows, plan.target[rows])
    row_loss = np.zeros(plan.target.shape[0], np.float64)
    row_loss[rows] = plan.weight[rows] * ce
    return TermResult(plan, rows, lse, ce, row_loss)


def reduce_units(n_units: int, *terms: TermResult):
    """Per-unit sums of weight*ce (per-example reduction, [Axolotl]
    "Objective and recurrence options") and the total loss."""
    unit_loss = np.zeros(n_units, np.float64)
    for tr in terms:
        np.add.at(unit_loss, tr.plan.unit, tr.row_loss)
    return float(unit_loss.sum()), unit_loss


def term_grad(logits: np.ndarray, vocab: int, tr: TermResult, rows: np.ndarray,
              grad_scale: float) -> np.ndarray:
    """dlogits for the listed rows (scored or not), double [len(rows), vocab]:
    grad_scale * weight * (softmax - onehot) on scored rows, exact zeros else."""
    rows = np.asarray(rows, np.int64)
    out = np.zeros((rows.shape[0], vocab), np.float64)
    scored = tr.plan.target[rows] >= 0
    if scored.any():
        sel = rows[scored]
        # lse of the selected rows, looked up from the scored list
        pos = np.searchsorted(tr.rows, sel)
        lse = tr.lse[pos]
        coef = grad_scale * tr.plan.weight[sel]
        out[scored] = grad_rows(logits, vocab, sel, tr.plan.target[sel], coef, lse)
    return out


def loss_absorbing(layout: Layout, logits: np.ndarray, vocab: int, clean: np.ndarray,
                   corrupted: np.ndarray, p: np.ndarray, align: int):
    plan = plan_diffusion(layout, clean, corrupted, p, ABSORBING, align)
    tr = term(logits, vocab, plan)
    loss, unit_loss = reduce_units(layout.n_units, tr)
    return loss, unit_loss, tr


def loss_uniform(canvas: Layout, logits: np.ndarray, canvas_clean: np.ndarray,
                 encoder: Layout, enc_logits: np.ndarray, enc_clean: np.ndarray,
                 vocab: int, lam: float, align: int = ALIGNED, p: Optional[np.ndarray] = None,
                 time_weighting: int = NO_TIME_WEIGHT, weight_clip: float = 0.0,
                 reduction: int = TOKEN_MEAN):
    """[Gemma] total = canvas CE (mean; optionally time-weighted and/or the
    mean of per-example means, see plan_diffusion) + lam * encoder AR CE
    (mean over next-token pairs)."""
    pc = plan_diffusion(canvas, canvas_clean, None, p, UNIFORM, align, time_weighting, weight_clip, reduction)
    pe = plan_encoder(encoder, enc_clean, lam)
    tc = term(logits, vocab, pc)
    te = term(enc_logits, vocab, pe)
    loss, unit_loss = reduce_units(canvas.n_units, tc, te)
    return loss, unit_loss, tc, te


# --------------------------------------------------------------------------
# Fused lm_head (Cut Cross Entropy style): logits = H W^T never rounded
# --------------------------------------------------------------------------
def linear_logits(H_rows: np.ndarray, W: np.ndarray, chunk: int = 16384) -> np.ndarray:
    """Z = H_rows W^T in double from bf16 inputs (library matmul as one step).
    H_rows: uint16 [n, D] (bf16 bits); W: uint16 [V, D]."""
    Hd = bf16_to_f64(H_rows)
    V = W.shape[0]
    Z = np.empty((Hd.shape[0], V), np.float64)
    for v0 in range(0, V, chunk):
        Wd = bf16_to_f64(W[v0:v0 + chunk])
        Z[:, v0:v0 + chunk] = Hd @ Wd.T
    return Z


def linear_loss(layout: Layout, H: np.ndarray, W: np.ndarray, clean: np.ndarray,
                corrupted: np.ndarray, p: np.ndarray, grad_scale: float = 1.0,
                want_grads: bool = True, align: int = ALIGNED, keep_dz: bool = False):
    """[Axolotl] CCE path, absorbing noise.  The rows of H that score a
    target (aligned: row i scores token i, as CCE does on the page; shifted:
    row i scores token i+1 of the same unit, the unfused loss's Dream
    reading carried over) form Z = H_M W^T in double; CE and weights as for
    the unfused loss; dZ = grad_scale * w * (softmax - onehot); dH_M = dZ W,
    dW = dZ^T H_M, other rows of dH exactly zero.  keep_dz: also return dZ
    ([scored rows, V], double) for the tests' error scales."""
    plan = plan_diffusion(layout, clean, corrupted, p, ABSORBING, align)
    rows, lse, ce, row_loss, dH, dW, dZ = _linear_term(plan, H, W, grad_scale, want_grads, keep_dz)
    unit_loss = np.zeros(layout.n_units, np.float64)
    np.add.at(unit_loss, plan.unit, row_loss)
    out = dict(loss=float(unit_loss.sum()), unit_loss=unit_loss, rows=rows, lse=lse, ce=ce, plan=plan)
    if want_grads:
        out.update(dH=dH, dW=dW)
    if keep_dz:
        out.update(dZ=dZ)
    return out


def linear_rows(layout: Layout, H: np.ndarray, W: np.ndarray, clean: np.ndarray,
                corrupted: np.ndarray, p: np.ndarray, sample_rows: np.ndarray,
                grad_scale: float = 1.0, align: int = ALIGNED):
    """Full-size spot check: for a few scored rows only, their CE, weight*ce
    and their row of dH (which needs only that row's own softmax)."""
    plan = plan_diffusion(layout, clean, corrupted, p, ABSORBING, align)
    out = linear_rows_plan(plan, H, W, sample_rows, grad_scale)
    out["plan"] = plan
    return out


def _linear_term(plan: RowPlan, H: np.ndarray, W: np.ndarray, grad_scale: float, want_grads: bool,
                 keep_dz: bool = False):
    """One term of a fused-head loss: the scored rows of H (by `plan`) form
    Z = H_M W^T in double; returns (rows, lse, ce, row_loss, dH, dW, dZ), dH
    over all rows of H (zeros on unscored rows), dW = dZ^T H_M ([V, D]), dZ
    only when keep_dz (else None)."""
    rows = np.nonzero(plan.target >= 0)[0]
    V, D = W.shape
    Z = linear_logits(H[rows], W)
    local = np.arange(rows.shape[0], dtype=np.int64)
    lse, ce = ce_rows(Z, V, local, plan.target[rows])
    row_loss = np.zeros(plan.target.shape[0], np.float64)
    row_loss[rows] = plan.weight[rows] * ce
    dH = dW = None
    if want_grads:
        dZ = grad_rows(Z, V, local, plan.target[rows], grad_scale * plan.weight[rows], lse)
        del Z
        Hd = bf16_to_f64(H[rows])
        dH = np.zeros((H.shape[0], D), np.float64)
        dW = np.zeros((V, D), np.float64)
        for v0 in range(0, V, 16384):
            Wd = bf16_to_f64(W[v0:v0 + 16384])
            dH[rows] += dZ[:, v0:v0 + 16384] @ Wd
            dW[v0:v0 + 16384] = dZ[:, v0:v0 + 16384].T @ Hd
        if not keep_dz:
            dZ = None
    else:
        dZ = None
    return rows, lse, ce, row_loss, dH, dW, dZ


def linear_loss_uniform(canvas: Layout, H: np.ndarray, W: np.ndarray, canvas_clean: np.ndarray,
                        encoder: Optional[Layout], He: Optional[np.ndarray],
                        enc_clean: Optional[np.ndarray], lam: float, align: int = ALIGNED,
                        grad_scale: float = 1.0, want_grads: bool = True, keep_dz: bool = False):
    """[Gemma] uniform-noise objective through a plain linear head, without a
    logits tensor ([Axolotl] Cut Cross Entropy carried to uniform noise):
    canvas term = mean CE of every non-pad canvas target (row i scores token
    i, or token i+1 of the same unit when shifted) on Z = H W^T; encoder term
    = lam * mean next-token CE over the clean full sequence on Ze = He W^T.
    dH, dHe = dZ W, dZe W (zeros on unscored rows); dW = dZ^T H_M + dZe^T He_M,
    one shared head.  H, He, W: uint16 bf16 bits [T, D], [Te, D], [V, D].
    keep_dz: also return dZ and dZe (double, [scored rows, V] per term)."""
    pc = plan_diffusion(canvas, canvas_clean, None, None, UNIFORM, align)
    tc = _linear_term(pc, H, W, grad_scale, want_grads, keep_dz)
    terms = [(pc, tc)]
    if encoder is not None:
        pe = plan_encoder(encoder, enc_clean, lam)
        terms.append((pe, _linear_term(pe, He, W, grad_scale, want_grads, keep_dz)))
    unit_loss = np.zeros(canvas.n_units, np.float64)
    for plan, t in terms:
        np.add.at(unit_loss, plan.unit, t[3])
    out = dict(loss=float(unit_loss.sum()), unit_loss=unit_loss, rows=tc[0], ce=tc[2], plan=pc)
    if encoder is not None:
        out.update(enc_rows=terms[1][1][0], enc_ce=terms[1][1][2], enc_plan=terms[1][0])
    if want_grads:
        out.update(dH=tc[4], dW=tc[5] + (terms[1][1][5] if encoder is not None else 0.0))
        if encoder is not None:
            out.update(dHe=terms[1][1][4])
    if keep_dz:
        out.update(dZ=tc[6], dZe=terms[1][1][6] if encoder is not None else None)
    return out


def linear_rows_plan(plan: RowPlan, H: np.ndarray, W: np.ndarray, sample_rows: np.ndarray,
                     grad_scale: float = 1.0):
    """Full-size spot check for any row plan (uniform canvas, encoder AR):
    for a few scored rows, their CE, weight*ce and their row of dH."""
    sample_rows = np.asarray(sample_rows, np.int64)
    assert (plan.target[sample_rows] >= 0).all()
    V, D = W.shape
    Z = linear_logits(H[sample_rows], W)
    local = np.arange(sample_rows.shape[0], dtype=np.int64)
    tgt = plan.target[sample_rows]
    lse, ce = ce_rows(Z, V, local, tgt)
    dZ = grad_rows(Z, V, local, tgt, grad_scale * plan.weight[sample_rows], lse)
    dH = np.zeros((sample_rows.shape[0], D), np.float64)
    for v0 in range(0, V, 16384):
        dH += dZ[:, v0:v0 + 16384] @ bf16_to_f64(W[v0:v0 + 16384])
    return dict(ce=ce, lse=lse, weighted=plan.weight[sample_rows] * ce, dH=dH)


# --------------------------------------------------------------------------
# Typed-decision losses at label slots ([Axolotl] "Typed-decision training",
# "Labels"; "Adapters, merging and inference": the restricted-label and Brier
# terms are computed over the allowed answers)
# --------------------------------------------------------------------------
HARD, DIST, SET = 0, 1, 2                       # label kinds
LABEL_RESTRICTED, LABEL_FULL, LABEL_BOTH = 1, 2, 3   # labels.label_softmax


def decision_targets(kind: int, val: np.ndarray, smoothing: float):
    """The CE target q and the Brier target y of one label over its K
    alternatives, in double.  `val` holds one value per alternative:
    hard -- 1 at the gold index, 0 elsewhere; dist -- the probabilities;
    set -- 1 for each allowed index, 0 elsewhere.
      hard: y = one-hot; q = (1 - smoothing) one-hot + smoothing / K
            (hard_label_smoothing spreads that fraction of the one-hot CE
            target uniformly over the question's K answer tokens; the Brier
            target is unchanged);
      dist: q = y = the probabilities as given;
      set:  q = y = uniform over the allowed indexes (reading: each allowed
            answer equally right)."""
    val = np.asarray(val, np.float64)
    K = val.shape[0]
    if K < 1:
        raise ValueError("a question has at least one alternative")
    if kind == HARD:
        if not (np.count_nonzero(val) == 1 and ((val == 0.0) | (val == 1.0)).all()):
            raise ValueError("hard label: exactly one 1, zeros elsewhere")
        y = val.copy()
        q = (1.0 - smoothing) * y + smoothing / K
    elif kind == DIST:
        if not (np.isfinite(val).all() and (val >= 0).all()):
            raise ValueError("dist label: finite, non-negative probabilities")
        y = val.copy()
        q = val.copy()
    elif kind == SET:
        if not (((val == 0.0) | (val == 1.0)).all() and val.sum() >= 1):
            raise ValueError("set label: a non-empty 0/1 membership")
        y = val / val.sum()
        q = y.copy()
    else:
        raise ValueError(f"label kind {kind}")
    return q, y


def decision_loss(logits: np.ndarray, vocab: int, slot_rows: Optional[np.ndarray], cand_off: np.ndarray,
                  cand_ids: np.ndarray, kind: np.ndarray, val: np.ndarray,
                  label_softmax: int = LABEL_BOTH, brier_weight: float = 0.1, smoothing: float = 0.0,
                  grad_scale: float = 1.0):
    """Typed-decision loss over n label slots, each one logits row z (bf16
    bits uint16 [rows, ld] or float64) and its question's K answer tokens
    a_0..a_{K-1} (distinct ids; cand_ids[cand_off[i]:cand_off[i+1]]):
      r = softmax over the K candidate logits z[a_k] (candidate-restricted);
      P = softmax over the whole vocabulary;
      CE_res  = -sum_k q_k log r_k            (label_softmax restricted/both)
      CE_full = -sum_k q_k log P(a_k)         (label_softmax full/both; the
                full-vocabulary softmax still penalises probability outside
                the valid answers)
      Brier   = sum_k (r_k - y_k)^2,  weighted by brier_weight (0.1 on the
                page), over the restricted distribution
      loss    = (1/n) sum over slots of the selected terms (reading: the mean
                over label slots).
    Returns loss, the per-slot contribution (its terms / n), the three terms
    per slot, and dlogits = grad_scale * d loss / dz ([n, vocab], double)."""
    n = int(cand_off.shape[0]) - 1
    rows = np.arange(n) if slot_rows is None else np.asarray(slot_rows, np.int64)
    if logits.dtype == np.uint16:
        z_all = bf16_to_f64(np.ascontiguousarray(logits[rows, :vocab]))
    else:
        z_all = np.asarray(logits[rows, :vocab], np.float64)
    use_res = label_softmax in (LABEL_RESTRICTED, LABEL_BOTH)
    use_full = label_softmax in (LABEL_FULL, LABEL_BOTH)
    ce_res = np.zeros(n)
    ce_full = np.zeros(n)
    brier = np.zeros(n)
    grad = np.zeros((n, vocab))
    w = 1.0 / n if n > 0 else 0.0
    for i in range(n):
        z = z_all[i]
        a = np.asarray(cand_ids[cand_off[i]:cand_off[i + 1]], np.int64)
        if a.size == 0 or np.unique(a).size != a.size or a.min() < 0 or a.max() >= vocab:
            raise ValueError(f"slot {i}: answer tokens must be distinct ids in [0, vocab)")
        q, y = decision_targets(int(kind[i]), val[cand_off[i]:cand_off[i + 1]], smoothing)
        Q = q.sum()
        # full-vocabulary softmax
        m = z.max()
        lse = m + np.log(np.exp(z - m).sum())
        P = np.exp(z - lse)
        # candidate-restricted softmax
        c = z[a]
        cm = c.max()
        lse_r = cm + np.log(np.exp(c - cm).sum())
        r = np.exp(c - lse_r)
        ce_res[i] = -(q * (c - lse_r)).sum()
        ce_full[i] = -(q * (c - lse)).sum()
        brier[i] = ((r - y) ** 2).sum()
        g = np.zeros(vocab)
        if use_full:                      # d CE_full / dz_v = Q P_v - q(v)
            g += Q * P
            g[a] -= q
        if use_res:                       # d CE_res / dz_{a_k} = Q r_k - q_k
            g[a] += Q * r - q
        # d Brier / dz_{a_j} = 2 r_j ((r_j - y_j) - sum_k r_k (r_k - y_k))
        d = r - y
        g[a] += brier_weight * 2.0 * r * (d - (r * d).sum())
        grad[i] = grad_scale * w * g
    per_slot = (ce_res * use_res + ce_full * use_full + brier_weight * brier) * w
    return dict(loss=float(per_slot.sum()), slot_loss=per_slot, ce_res=ce_res, ce_full=ce_full,
                brier=brier, dlogits=grad)
