"""GPU parity of the typed-decision losses at label slots against the CPU
oracle ("Native diffusion language-model training", Typed-decision training
and Labels): loss within 1e-5 relative, every slot's share, and the bf16
gradient of every logit -- on the full 128-slot workload, on ragged
vocabularies and row strides (the scalar path), with 128 answers per
question, a slot-row indirection, every label_softmax setting, smoothing,
and slots whose labels the kernel must refuse.

Both kernel paths are covered: the cluster path (one cluster of CTAs per
slot, 16-byte aligned rows) and the three-kernel path (any row stride).

Gradient bar: entries away from the answer tokens are g w Q P_v, one
product rounded to bf16 -- the gradient bar of the other losses (2e-3
absolute and within one bf16 ulp of the rounded exact value).  The K
answer-token entries add up to five fp32 terms of size up to |g w| (Q +
2 + 4 b) that may cancel, so their bar is one bf16 ulp plus 2^-20 of that
size (fp32 rounding of the terms).
"""
import numpy as np
import pytest
import torch

import dlm_inputs as di
import oracle
from parity import assert_grad_close, assert_loss_close, bf16_ulp, gpu_bf16_to_f64

pytestmark = pytest.mark.gpu

dlm = pytest.importorskip("diffusion_lm_loss_b200")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dlm.lib()


def _batch(seed, n, V, kmax, kinds=(0, 1, 2), kmin=1):
    rng = np.random.default_rng(seed)
    off = [0]
    ids, kind, vals = [], [], []
    for i in range(n):
        K = int(rng.integers(kmin, kmax + 1))
        ids.append(rng.choice(V, size=K, replace=False))
        k = kinds[i % len(kinds)]
        if k == oracle.HARD:
            v = np.zeros(K, np.float32)
            v[rng.integers(K)] = 1.0
        elif k == oracle.DIST:
            v = rng.dirichlet(np.ones(K))
            if K > 2:
                v[rng.integers(K)] = 0.0            # a zero entry is a valid probability
            v = (v / v.sum()).astype(np.float32)
        else:
            v = np.zeros(K, np.float32)
            v[rng.choice(K, size=int(rng.integers(1, K + 1)), replace=False)] = 1.0
        kind.append(k)
        vals.append(v)
        off.append(off[-1] + K)
    return (np.array(off, np.int32), np.concatenate(ids).astype(np.int32), np.array(kind, np.int32),
            np.concatenate(vals).astype(np.float32))


def _dev(*arrays):
    return [torch.from_numpy(np.ascontiguousarray(a)).cuda() for a in arrays]


def _check(out, ref, off, ids, kinds_used, grad_scale, brier_w, n, V, label_softmax):
    assert_loss_close(float(out.loss.item()), ref["loss"])
    sl = out.slot_loss.cpu().numpy()[:n].astype(np.float64)
    np.testing.assert_allclose(sl, ref["slot_loss"], rtol=1e-5, atol=1e-7 * abs(ref["loss"]))
    g = gpu_bf16_to_f64(out.dlogits)[:, :V]
    exact = ref["dlogits"]
    cand = np.zeros((n, V), bool)
    for i in range(n):
        cand[i, ids[off[i]:off[i + 1]]] = True
    # away from the answer tokens: one rounded product
    assert_grad_close(np.where(cand, 0.0, g), np.where(cand, 0.0, exact), "dlogits (dense part)")
    # at the answer tokens: a few fp32 terms that may cancel
    Qmax = 1.0 + 1e-4
    size = abs(grad_scale) / n * (2 * Qmax + 2 + 4 * brier_w)
    err = np.abs(g[cand] - exact[cand])
    tol = bf16_ulp(np.maximum(np.abs(g[cand]), np.abs(exact[cand]))) + 2.0 ** -20 * size
    assert (err <= tol).all(), f"dlogits at answer tokens: max err {err.max():.3e}, worst tol {tol[np.argmax(err - tol)]:.3e}"


@pytest.mark.parametrize("label_softmax", [oracle.LABEL_BOTH, oracle.LABEL_RESTRICTED, oracle.LABEL_FULL])
def test_decision_full_workload(label_softmax):
    """The 128-slot workload (K in [2, 26] from one codebook, V = 126,464,
    16-byte path, three CTAs per row) against the oracle, every gradient
    element."""
    spec = di.WORKLOADS["dec_s128_k26_v126464"]
    case = di.make_case(spec, "cuda")
    e = case.extra
    out = dlm.decision_loss_fwd_bwd(case.logits, spec.vocab, e["cand_off"], e["cand_ids"], e["kind"], e["val"],
                                    label_softmax=label_softmax, brier_weight=0.1, hard_label_smoothing=0.05)
    torch.cuda.synchronize()
    assert out.device_status() == 0
    off, ids = e["cand_off"].cpu().numpy(), e["cand_ids"].cpu().numpy()
    ref = oracle.decision_loss(di.bf16_bits(case.logits), spec.vocab, None, off, ids, e["kind"].cpu().numpy(),
                               e["val"].cpu().numpy(), label_softmax=label_softmax, brier_weight=0.1,
                               smoothing=0.05)
    _check(out, ref, off, ids, None, 1.0, 0.1, spec.n_units, spec.vocab, label_softmax)


@pytest.mark.parametrize("n,V,kmin,kmax,ld_pad,seed", [
    (37, 5003, 1, 128, 3, 0),     # ragged V and row stride: three kernels, scalar loads; 1 to 128 answers
    (5, 126464, 2, 26, 0, 1),     # few slots: clusters of 8 CTAs per row
    (300, 2048, 2, 8, 0, 2),      # many slots, one CTA per row
    (3, 16, 16, 16, 0, 3),        # every token of the vocabulary an answer
    (4, 300000, 2, 26, 0, 4),     # long rows: clusters of 8 CTAs of 37,500 columns
    (6, 8192, 33, 128, 0, 5),     # the cluster path with more than one group of 32 answers
    (1024, 65536, 2, 26, 0, 8),   # clusters of 2 (rows in flight kept within L2), several waves
])
def test_decision_elementwise(n, V, kmin, kmax, ld_pad, seed):
    off, ids, kind, val = _batch(seed, n, V, kmax, kmin=kmin)
    gen = torch.Generator(device="cuda")
    gen.manual_seed(seed)
    base = (torch.randn((n, V + ld_pad), generator=gen, device="cuda") * 2.5).to(torch.bfloat16)
    logits = base[:, :V] if ld_pad else base
    d_off, d_ids, d_kind, d_val = _dev(off, ids, kind, val)
    out = dlm.decision_loss_fwd_bwd(logits, V, d_off, d_ids, d_kind, d_val, brier_weight=0.3,
                                    hard_label_smoothing=0.1, grad_scale=-0.75)
    torch.cuda.synchronize()
    assert out.device_status() == 0
    ref = oracle.decision_loss(di.bf16_bits(logits), V, None, off, ids, kind, val, brier_weight=0.3,
                               smoothing=0.1, grad_scale=-0.75)
    _check(out, ref, off, ids, None, -0.75, 0.3, n, V, oracle.LABEL_BOTH)


def test_decision_slot_rows_indirection():
    """Slots reading rows of a larger logits tensor (slot_rows) give the
    same results as the same rows passed compactly."""
    n, V = 24, 4096
    off, ids, kind, val = _batch(4, n, V, 26)
    gen = torch.Generator(device="cuda")
    gen.manual_seed(4)
    big = (torch.randn((200, V), generator=gen, device="cuda") * 3).to(torch.bfloat16)
    rows = torch.randperm(200, generator=torch.Generator().manual_seed(1))[:n].to(torch.int64)
    d_off, d_ids, d_kind, d_val = _dev(off, ids, kind, val)
    a = dlm.decision_loss_fwd_bwd(big, V, d_off, d_ids, d_kind, d_val, slot_rows=rows.cuda())
    b = dlm.decision_loss_fwd_bwd(big[rows.cuda()].contiguous(), V, d_off, d_ids, d_kind, d_val)
    torch.cuda.synchronize()
    assert a.loss.item() == b.loss.item()
    assert torch.equal(a.dlogits.view(torch.int16), b.dlogits.view(torch.int16))
    ref = oracle.decision_loss(di.bf16_bits(big), V, rows.numpy(), off, ids, kind, val)
    _check(a, ref, off, ids, None, 1.0, 0.1, n, V, oracle.LABEL_BOTH)


def test_decision_invalid_slots_are_flagged_and_skipped():
    """An answer id outside the vocabulary, a repeated answer id and a hard
    label with two golds: status bits, zero loss share and zero gradient
    rows for those slots; the other slots are unaffected (the mean still
    divides by every slot)."""
    n, V = 12, 3000
    off, ids, kind, val = _batch(5, n, V, 10, kmin=3)
    good = np.ones(n, bool)
    ids_bad = ids.copy()
    ids_bad[off[2]] = V + 5                          # slot 2: id outside [0, V)
    ids_bad[off[5] + 1] = ids_bad[off[5]]            # slot 5: repeated answer
    val_bad = val.copy()
    h = int(np.nonzero(kind == oracle.HARD)[0][-1])  # a hard slot: two golds
    val_bad[off[h]:off[h + 1]] = 0.0
    val_bad[off[h]:off[h] + 2] = 1.0
    for s in (2, 5, h):
        good[s] = False
    gen = torch.Generator(device="cuda")
    gen.manual_seed(5)
    logits = (torch.randn((n, V), generator=gen, device="cuda") * 2).to(torch.bfloat16)
    out = dlm.decision_loss_fwd_bwd(logits, V, *_dev(off, ids_bad, kind, val_bad))
    torch.cuda.synchronize()
    st = out.device_status()
    assert st & dlm.DEV_BAD_TOKEN_ID and st & dlm.DEV_BAD_LABEL
    g = out.dlogits.float().cpu()
    sl = out.slot_loss.cpu().numpy()[:n]
    for s in np.nonzero(~good)[0]:
        assert sl[s] == 0.0 and bool((g[s] == 0).all())
    # the valid slots alone, with the mean over all n slots
    keep = np.nonzero(good)[0]
    ref = oracle.decision_loss(di.bf16_bits(logits), V, keep, np.concatenate([[0], np.cumsum(np.diff(off)[keep])]),
                               np.concatenate([ids[off[i]:off[i + 1]] for i in keep]), kind[keep],
                               np.concatenate([val[off[i]:off[i + 1]] for i in keep]))
    scale = len(keep) / n
    assert_loss_close(float(out.loss.item()), ref["loss"] * scale)
    np.testing.assert_allclose(sl[keep], ref["slot_loss"] * scale, rtol=1e-5)
    # a call after the failing one starts from a clean status word
    out2 = dlm.decision_loss_fwd_bwd(logits, V, *_dev(off, ids, kind, val), out=out)
    assert out2.device_status() == 0


def test_decision_repeated_ids_across_answer_groups():
    """Repeated answer ids found wherever they sit among K = 70 answers
    (the label warp holds answers k, k + 32, k + 64 per lane): across two
    groups of 32, inside the second group and inside the third.  Those
    slots are refused (DEV_BAD_LABEL, zero share and gradient), the valid
    one matches the oracle -- on both kernel paths."""
    n, V, K = 4, 4096, 70
    rng = np.random.default_rng(11)
    off = np.arange(0, (n + 1) * K, K, dtype=np.int32)
    ids = np.concatenate([rng.choice(V, size=K, replace=False) for _ in range(n)]).astype(np.int32)
    kind = np.full(n, oracle.DIST, np.int32)
    val = np.concatenate([rng.dirichlet(np.ones(K)) for _ in range(n)]).astype(np.float32)
    ids[off[1] + 40] = ids[off[1] + 3]          # across groups 0 and 1
    ids[off[2] + 50] = ids[off[2] + 33]         # inside group 1
    ids[off[3] + 69] = ids[off[3] + 64]         # inside group 2
    gen = torch.Generator(device="cuda")
    gen.manual_seed(11)
    for ld_pad in (0, 3):
        base = (torch.randn((n, V + ld_pad), generator=gen, device="cuda") * 2).to(torch.bfloat16)
        logits = base[:, :V] if ld_pad else base
        out = dlm.decision_loss_fwd_bwd(logits, V, *_dev(off, ids, kind, val))
        torch.cuda.synchronize()
        assert out.device_status() == dlm.DEV_BAD_LABEL
        g = out.dlogits.float().cpu()
        sl = out.slot_loss.cpu().numpy()[:n]
        for s_ in (1, 2, 3):
            assert sl[s_] == 0.0 and bool((g[s_] == 0).all())
        ref = oracle.decision_loss(di.bf16_bits(logits), V, np.array([0]), off[:2], ids[:K], kind[:1], val[:K])
        assert_loss_close(float(out.loss.item()), ref["loss"] / n)
        np.testing.assert_allclose(sl[0], ref["slot_loss"][0] / n, rtol=1e-5)


def test_decision_most_slots_one_call():
    """DLM_DECISION_MAX_SLOTS label slots in one call (the cluster grid's
    y extent at its limit; one CTA per slot of V = 64), with one- to
    four-answer questions, against the oracle element by element; one slot
    more is refused before anything runs."""
    n, V = dlm.DECISION_MAX_SLOTS, 64
    off, ids, kind, val = _batch(12, n, V, 4, kmin=1)
    gen = torch.Generator(device="cuda")
    gen.manual_seed(12)
    logits = (torch.randn((n + 1, V), generator=gen, device="cuda") * 2).to(torch.bfloat16)
    out = dlm.decision_loss_fwd_bwd(logits[:n], V, *_dev(off, ids, kind, val))
    torch.cuda.synchronize()
    assert out.device_status() == 0
    ref = oracle.decision_loss(di.bf16_bits(logits[:n]), V, None, off, ids, kind, val)
    _check(out, ref, off, ids, None, 1.0, 0.1, n, V, oracle.LABEL_BOTH)
    off2 = np.concatenate([off, [off[-1] + 1]]).astype(np.int32)
    ids2 = np.concatenate([ids, [0]]).astype(np.int32)
    with pytest.raises(dlm.DlmError):
        dlm.decision_loss_fwd_bwd(logits, V, *_dev(off2, ids2, np.concatenate([kind, [oracle.HARD]]).astype(np.int32),
                                                   np.concatenate([val, [1.0]]).astype(np.float32)))


def test_decision_concurrent_streams():
    """Calls with their own workspaces on two streams at once (one of them
    a multi-wave call, the other the one-wave kernel) give the serial
    results bit for bit."""
    base = di.WORKLOADS["dec_s128_k26_v126464"]
    specs = [base, base.scaled(n_units=700)]
    cases = [di.make_case(sp, "cuda", seed=20 + i) for i, sp in enumerate(specs)]

    def run(i):
        e = cases[i].extra
        return dlm.decision_loss_fwd_bwd(cases[i].logits, specs[i].vocab, e["cand_off"], e["cand_ids"], e["kind"],
                                         e["val"])

    serial = [run(0), run(1)]
    torch.cuda.synchronize()
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    conc = [None, None]
    for _ in range(3):
        for i, st in enumerate(streams):
            with torch.cuda.stream(st):
                conc[i] = run(i)
        torch.cuda.synchronize()
        for a, b in zip(serial, conc):
            assert torch.equal(a.loss, b.loss)
            assert torch.equal(a.dlogits.view(torch.int16), b.dlogits.view(torch.int16))
            assert b.device_status() == 0


def test_decision_no_slots_and_reproducible():
    V = 1024
    z = torch.zeros((0, V), dtype=torch.bfloat16, device="cuda")
    out = dlm.decision_loss_fwd_bwd(z, V, *_dev(np.zeros(1, np.int32), np.zeros(0, np.int32),
                                                np.zeros(0, np.int32), np.zeros(0, np.float32)))
    torch.cuda.synchronize()
    assert float(out.loss.item()) == 0.0 and out.device_status() == 0
    spec = di.WORKLOADS["dec_s128_k26_v126464"]
    case = di.make_case(spec, "cuda")
    e = case.extra
    a = dlm.decision_loss_fwd_bwd(case.logits, spec.vocab, e["cand_off"], e["cand_ids"], e["kind"], e["val"])
    b = dlm.decision_loss_fwd_bwd(case.logits, spec.vocab, e["cand_off"], e["cand_ids"], e["kind"], e["val"])
    torch.cuda.synchronize()
    assert a.loss.item() == b.loss.item()
    assert torch.equal(a.dlogits.view(torch.int16), b.dlogits.view(torch.int16))


def test_decision_rows_and_offsets_outside_their_arrays_are_refused():
    """A slot row outside the logits tensor, and answer offsets that leave
    the answer arrays (device data the host cannot check): DEV_BAD_LAYOUT,
    those slots skipped, the others unaffected -- on both kernel paths."""
    n, V = 10, 4096
    off, ids, kind, val = _batch(6, n, V, 12, kmin=2)
    gen = torch.Generator(device="cuda")
    gen.manual_seed(6)
    for ld_pad in (0, 3):                       # the cluster path, then the three-kernel path
        base = (torch.randn((16, V + ld_pad), generator=gen, device="cuda") * 2).to(torch.bfloat16)
        logits = base[:, :V] if ld_pad else base
        rows = np.arange(n, dtype=np.int64)
        rows[3] = 16                            # one past the last row
        bad_off = off.copy()
        bad_off[8] = off[8] + 1000              # slot 7 ends and slot 8 starts beyond the answer arrays
        out = dlm.decision_loss_fwd_bwd(logits, V, *_dev(bad_off, ids, kind, val),
                                        slot_rows=torch.from_numpy(rows).cuda())
        torch.cuda.synchronize()
        st = out.device_status()
        assert st & dlm.DEV_BAD_LAYOUT, st
        g = out.dlogits.float().cpu()
        sl = out.slot_loss.cpu().numpy()[:n]
        for s_ in (3, 7, 8):
            assert sl[s_] == 0.0 and bool((g[s_] == 0).all())
        keep = np.array([i for i in range(n) if i not in (3, 7, 8)])
        ref = oracle.decision_loss(di.bf16_bits(logits), V, rows[keep],
                                   np.concatenate([[0], np.cumsum(np.diff(off)[keep])]),
                                   np.concatenate([ids[off[i]:off[i + 1]] for i in keep]), kind[keep],
                                   np.concatenate([val[off[i]:off[i + 1]] for i in keep]))
        assert_loss_close(float(out.loss.item()), ref["loss"] * len(keep) / n)


def test_decision_graph_replays_and_dirty_workspace():
    """Nothing in the workspace needs zeroing between calls: a workspace
    full of garbage, the same workspace reused by calls of another shape,
    and a CUDA graph of the call replayed several times all give the direct
    call's loss bit for bit and a clean status word."""
    spec = di.WORKLOADS["dec_s128_k26_v126464"].scaled(n_units=40)
    case = di.make_case(spec, "cuda")
    e = case.extra
    args = (case.logits, spec.vocab, e["cand_off"], e["cand_ids"], e["kind"], e["val"])
    ref = dlm.decision_loss_fwd_bwd(*args)
    torch.cuda.synchronize()
    want = ref.loss.item()
    # garbage in the whole workspace, the ticket included
    ref.workspace.fill_(0xA5)
    ref.loss.fill_(float("nan"))
    again = dlm.decision_loss_fwd_bwd(*args, out=ref)
    torch.cuda.synchronize()
    assert again.loss.item() == want and again.device_status() == 0
    # the same workspace between calls of another shape (other CTA counts)
    small = di.WORKLOADS["dec_s128_k26_v126464"].scaled(n_units=7)
    sc = di.make_case(small, "cuda", seed=9)
    se = sc.extra
    ws = ref.workspace
    o2 = dlm.DecisionOut(torch.empty(1, device="cuda"), torch.empty(7, device="cuda"),
                         torch.empty((7, small.vocab), dtype=torch.bfloat16, device="cuda"), ws)
    s_ref = dlm.decision_loss_fwd_bwd(sc.logits, small.vocab, se["cand_off"], se["cand_ids"], se["kind"], se["val"])
    dlm.decision_loss_fwd_bwd(sc.logits, small.vocab, se["cand_off"], se["cand_ids"], se["kind"], se["val"], out=o2)
    again = dlm.decision_loss_fwd_bwd(*args, out=ref)
    torch.cuda.synchronize()
    assert o2.loss.item() == s_ref.loss.item() and again.loss.item() == want
    # a graph of the call, replayed
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        dlm.decision_loss_fwd_bwd(*args, out=ref)
    for _ in range(3):
        ref.loss.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        assert ref.loss.item() == want and ref.device_status() == 0
