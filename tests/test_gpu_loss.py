"""GPU parity of the weighted CE forward + backward against the CPU oracle.

Element-by-element at sizes the oracle finishes in seconds (more rows than
CTAs, ragged vocabularies, packed documents, pads, empty documents); at the full
workload sizes, in the launch configuration the benchmark times: the total
loss and every per-unit sum over all rows, and the gradient on sampled rows.
"""
import numpy as np
import pytest
import torch

import dlm_inputs as di
import oracle
from parity import (assert_grad_close, assert_loss_close, assert_units_close, gpu_bf16_to_f64)

pytestmark = pytest.mark.gpu

dlm = pytest.importorskip("diffusion_lm_loss_b200")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dlm.lib()


def _bits(t: torch.Tensor) -> np.ndarray:
    return di.bf16_bits(t)


def _sample_rows(n_rows, unit_len, k=48, seed=0):
    rng = np.random.default_rng(seed)
    fixed = [0, 1, n_rows - 1, n_rows - 2]
    if unit_len:
        fixed += [unit_len - 1, unit_len, min(n_rows - 1, 2 * unit_len - 1)]
    extra = rng.choice(n_rows, size=min(k, n_rows), replace=False)
    return np.unique(np.clip(np.array(fixed + list(extra)), 0, n_rows - 1))


def run_absorbing(spec, logits, clean, *, n_units, seq_len, cu=None, pad=None, seed=0,
                  grad_rows=None, grad_scale=1.0, p_override=None):
    """GPU: sample_t -> corrupt -> loss.  Oracle: the same from the same
    inputs.  Compares everything; grads on `grad_rows` (None = all rows)."""
    dev = torch.device("cuda")
    V = spec.vocab
    n = clean.shape[0]
    cu_d = cu.to(dev) if cu is not None else None
    pad_d = pad.to(dev) if pad is not None else None
    lay = dlm.make_layout(n_units, seq_len, cu_d, pad_d, n_tokens=n)
    clean_d = clean.to(dev)
    logits_d = logits.to(dev)
    if p_override is None:
        t, p = dlm.sample_t(seed, n_units, oracle.ABSORBING, spec.eps)
    else:
        p = p_override.to(dev)
    noisy, corr = dlm.corrupt(lay, clean_d, p, oracle.ABSORBING, spec.mask_id, V, seed)
    out = dlm.loss_fwd_bwd(lay, logits_d, V, clean_d, corr, p, oracle.ABSORBING, spec.align,
                           grad_scale=grad_scale)
    torch.cuda.synchronize()
    assert out.device_status() == 0

    cu_np = cu.cpu().numpy() if cu is not None else None
    pad_np = pad.cpu().numpy() if pad is not None else None
    lay_o = oracle.Layout(n_units, seq_len, cu_np, pad_np)
    clean_np = clean.cpu().numpy()
    if p_override is None:
        _, p_o = oracle.sample_t(seed, n_units, oracle.ABSORBING, spec.eps)
        assert np.array_equal(p.cpu().numpy().view(np.uint32), p_o.view(np.uint32))
    else:
        p_o = p_override.cpu().numpy()
    _, corr_o = oracle.corrupt(lay_o, clean_np, p_o, oracle.ABSORBING, spec.mask_id, V, seed)
    assert np.array_equal(corr.cpu().numpy(), corr_o)
    x = _bits(logits)
    loss_o, unit_o, tr = oracle.loss_absorbing(lay_o, x, V, clean_np, corr_o, p_o, spec.align)
    assert_loss_close(float(out.loss.item()), loss_o)
    assert_units_close(out.unit_loss.cpu().numpy()[:n_units], unit_o, loss_o)
    rows = np.arange(n) if grad_rows is None else np.asarray(grad_rows)
    g_o = oracle.term_grad(x, V, tr, rows, grad_scale)
    g = gpu_bf16_to_f64(out.dlogits[torch.from_numpy(rows).to(dev), :V])
    assert_grad_close(g, g_o)
    return out, tr


# --------------------------------------------------------------------------
# absorbing, aligned / shifted
# --------------------------------------------------------------------------
def test_tiny_absorbing_full():
    spec = di.WORKLOADS["abs_b2_l64_v1024"]
    case = di.make_case(spec, "cpu")
    for seed in (0, 1, 2, 3):
        run_absorbing(spec, case.logits, case.clean, n_units=2, seq_len=64, seed=seed)


def test_llada_like_mid_size_elementwise():
    """L=256 rows of V=126464 (more rows than CTAs in flight at once), every element checked."""
    spec = di.WORKLOADS["abs_b1_l4096_v126464"].scaled(seq_len=256)
    case = di.make_case(spec, "cuda")
    run_absorbing(spec, case.logits, case.clean, n_units=1, seq_len=256, seed=0)
    run_absorbing(spec, case.logits, case.clean, n_units=1, seq_len=256, seed=5, grad_scale=0.25)


def test_llada_like_full_size():
    spec = di.WORKLOADS["abs_b1_l4096_v126464"]
    case = di.make_case(spec, "cuda")
    for seed in (0, 11):
        run_absorbing(spec, case.logits, case.clean, n_units=1, seq_len=4096, seed=seed,
                      grad_rows=_sample_rows(4096, 4096, seed=seed))


@pytest.mark.parametrize("units,align", [(5, oracle.ALIGNED), (5, oracle.SHIFTED), (33, oracle.ALIGNED)])
def test_many_rows_plan_slices(units, align):
    """Sequences of 4,000 rows split over the plan's CTAs: 20,000 rows (every
    CTA keeps its slice in shared memory) and 132,000 rows (more than the
    eight CTAs keep, so the list comes from the re-classifying pass)."""
    spec = di.WORKLOADS["abs_b1_l4096_v126464"].scaled(vocab=4096, mask_id=4095, ids_high=4000, n_units=units,
                                                       seq_len=4000, spike=0.0, align=align)
    case = di.make_case(spec, "cuda")
    run_absorbing(spec, case.logits, case.clean, n_units=units, seq_len=4000, seed=7,
                  grad_rows=_sample_rows(units * 4000, 4000, seed=7))


def test_dream_like_shifted_mid_size_elementwise():
    spec = di.WORKLOADS["shift_b8_l2048_v152064"].scaled(n_units=3, seq_len=100)
    case = di.make_case(spec, "cuda")
    out, tr = run_absorbing(spec, case.logits, case.clean, n_units=3, seq_len=100, seed=2)
    assert (tr.plan.target[[99, 199, 299]] == -1).all()


def test_dream_like_shifted_full_size():
    spec = di.WORKLOADS["shift_b8_l2048_v152064"]
    case = di.make_case(spec, "cuda")
    run_absorbing(spec, case.logits, case.clean, n_units=8, seq_len=2048, seed=0,
                  grad_rows=_sample_rows(8 * 2048, 2048))


@pytest.mark.parametrize("V,ld", [(1003, 1003), (1000, 1010), (5000, 5000), (8192, 8200),
                                  (40000, 40000), (262144, 262144), (1048576, 1048576), (1000003, 1000003)])
def test_vocab_and_stride_variants(V, ld):
    """Ragged vocabularies (general kernel), padded row strides (columns past
    V untouched), the largest cluster split, and rows of about a million
    columns (2 MB each: the rows in flight no longer fit in L2) on both
    kernels."""
    spec = di.WORKLOADS["abs_b2_l64_v1024"].scaled(vocab=V, mask_id=V - 1, ids_high=V - 2,
                                                   n_units=2, seq_len=24, std=3.0)
    case = di.make_case(spec.scaled(vocab=ld), "cuda")      # draw [rows, ld], use the first V
    logits = case.logits
    dev = torch.device("cuda")
    lay = dlm.make_layout(2, 24)
    clean = case.clean.clamp(max=V - 2)
    t, p = dlm.sample_t(4, 2, oracle.ABSORBING, 1e-3)
    _, corr = dlm.corrupt(lay, clean, p, oracle.ABSORBING, V - 1, V, 4)
    sentinel = torch.full_like(logits, 7.0)
    out = dlm.LossOut(torch.empty(1, device=dev), torch.empty(2, device=dev), sentinel, None,
                      torch.empty(dlm.loss_workspace_size(lay), dtype=torch.uint8, device=dev))
    dlm.loss_fwd_bwd(lay, logits, V, clean, corr, p, oracle.ABSORBING, oracle.ALIGNED, out=out)
    torch.cuda.synchronize()
    if ld > V:
        assert bool((out.dlogits[:, V:] == 7.0).all())
    x = _bits(logits)
    lay_o = oracle.Layout(2, 24, None, None)
    _, p_o = oracle.sample_t(4, 2, oracle.ABSORBING, 1e-3)
    _, corr_o = oracle.corrupt(lay_o, clean.cpu().numpy(), p_o, oracle.ABSORBING, V - 1, V, 4)
    loss_o, unit_o, tr = oracle.loss_absorbing(lay_o, x, V, clean.cpu().numpy(), corr_o, p_o,
                                               oracle.ALIGNED)
    assert_loss_close(float(out.loss.item()), loss_o)
    g_o = oracle.term_grad(x, V, tr, np.arange(48), 1.0)
    assert_grad_close(gpu_bf16_to_f64(out.dlogits[:, :V]), g_o)


def test_packed_documents_with_pads_and_empty_docs():
    """Packed varlen layout (cu_seqlens), pads inside documents and empty
    documents; both alignments."""
    rng = np.random.default_rng(1)
    lens = [50, 0, 300, 17, 1, 0, 400, 256]
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32)
    T = int(cu[-1])
    spec = di.WORKLOADS["abs_b1_l4096_v126464"].scaled(vocab=32768, mask_id=32767, ids_high=32000)
    case = di.make_case(spec.scaled(seq_len=T), "cuda")
    pad = torch.from_numpy((rng.random(T) < 0.1).astype(np.uint8))
    for align in (oracle.ALIGNED, oracle.SHIFTED):
        run_absorbing(spec.scaled(align=align), case.logits, case.clean, n_units=len(lens),
                      seq_len=0, cu=cu, pad=pad, seed=3)


def test_packed_geometric_documents():
    """The packed-document shape of the fused-head workload, through the
    unfused loss on materialised logits (V = 32000)."""
    spec = di.WORKLOADS["lin_t16384_d4096_v126464"].scaled(n_tokens_packed=2048)
    c = di.make_case(spec, "cpu", with_tensors=False)
    lspec = di.WORKLOADS["abs_b1_l4096_v126464"].scaled(vocab=32000, mask_id=31999, ids_high=31000,
                                                        seq_len=2048, spike=0.0)
    lc = di.make_case(lspec, "cuda")
    run_absorbing(lspec, lc.logits, lc.clean, n_units=c.n_units, seq_len=0, cu=c.cu_seqlens, seed=9)


# --------------------------------------------------------------------------
# edge cases
# --------------------------------------------------------------------------
def test_no_scored_rows_gives_zero_loss_and_zero_grads():
    spec = di.WORKLOADS["abs_b1_l4096_v126464"].scaled(seq_len=64)
    case = di.make_case(spec, "cuda")
    p = torch.full((1,), 1e-9, dtype=torch.float32)      # threshold below every draw's chance
    dev = torch.device("cuda")
    lay = dlm.make_layout(1, 64)
    corr = torch.zeros(64, dtype=torch.uint8, device=dev)
    out = dlm.loss_fwd_bwd(lay, case.logits, spec.vocab, case.clean, corr, p.to(dev))
    torch.cuda.synchronize()
    assert float(out.loss.item()) == 0.0
    assert bool((out.dlogits == 0).all())


def test_all_rows_scored_p_one_is_mean_ce():
    spec = di.WORKLOADS["abs_b1_l4096_v126464"].scaled(seq_len=128)
    case = di.make_case(spec, "cuda")
    dev = torch.device("cuda")
    lay = dlm.make_layout(1, 128)
    corr = torch.ones(128, dtype=torch.uint8, device=dev)
    p = torch.ones(1, dtype=torch.float32, device=dev)
    out = dlm.loss_fwd_bwd(lay, case.logits, spec.vocab, case.clean, corr, p)
    ref = torch.nn.functional.cross_entropy(case.logits.double(), case.clean.long()).item()
    assert abs(float(out.loss.item()) - ref) <= 1e-5 * ref


def test_empty_input():
    dev = torch.device("cuda")
    lay = dlm.make_layout(2, 0)
    logits = torch.empty((0, 4096), dtype=torch.bfloat16, device=dev)
    clean = torch.empty(0, dtype=torch.int32, device=dev)
    corr = torch.empty(0, dtype=torch.uint8, device=dev)
    p = torch.full((2,), 0.5, device=dev)
    out = dlm.loss_fwd_bwd(lay, logits, 4096, clean, corr, p)
    torch.cuda.synchronize()
    assert float(out.loss.item()) == 0.0
    assert out.unit_loss.cpu().tolist() == [0.0, 0.0]


@pytest.mark.parametrize("V", [126464, 1000])
def test_keep_unscored_rows_leaves_them_untouched(V):
    """keep_unscored_rows: scored rows as usual, every other row of dlogits
    keeps what the caller put there (fast kernel and general kernel)."""
    spec = di.WORKLOADS["abs_b1_l4096_v126464"].scaled(vocab=V, mask_id=V - 1, ids_high=V - 2, seq_len=96,
                                                       spike=0.0)
    case = di.make_case(spec, "cuda")
    dev = torch.device("cuda")
    lay = dlm.make_layout(1, 96)
    t, p = dlm.sample_t(6, 1)
    _, corr = dlm.corrupt(lay, case.clean, p, oracle.ABSORBING, spec.mask_id, V, 6)
    opts = dlm.LossOptions(keep_unscored_rows=1)
    sentinel = 0x3F80                                        # bf16 1.0
    out = dlm.loss_fwd_bwd(lay, case.logits, V, case.clean, corr, p, options=opts)
    out.dlogits.view(torch.int16).fill_(sentinel)
    out = dlm.loss_fwd_bwd(lay, case.logits, V, case.clean, corr, p, options=opts, out=out)
    torch.cuda.synchronize()
    assert out.device_status() == 0
    lay_o = oracle.Layout(1, 96, None, None)
    _, p_o = oracle.sample_t(6, 1, oracle.ABSORBING, 1e-3)
    _, corr_o = oracle.corrupt(lay_o, case.clean.cpu().numpy(), p_o, oracle.ABSORBING, spec.mask_id, V, 6)
    x = di.bf16_bits(case.logits)
    loss_o, unit_o, tr = oracle.loss_absorbing(lay_o, x, V, case.clean.cpu().numpy(), corr_o, p_o, oracle.ALIGNED)
    assert_loss_close(float(out.loss.item()), loss_o)
    scored = tr.rows
    assert 0 < scored.size < 96
    assert_grad_close(gpu_bf16_to_f64(out.dlogits[torch.from_numpy(scored).to(dev)]),
                      oracle.term_grad(x, V, tr, scored, 1.0))
    unscored = np.setdiff1d(np.arange(96), scored)
    bits = out.dlogits.view(torch.int16)[torch.from_numpy(unscored).to(dev)].cpu().numpy()
    assert (bits == sentinel).all()


@pytest.mark.parametrize("V,align", [(126464, oracle.ALIGNED), (152064, oracle.SHIFTED), (1000, oracle.ALIGNED)])
def test_every_gradient_element_is_written(V, align):
    """Outputs poisoned with NaN before the call: afterwards no element of
    dlogits may still hold the poison (scored rows get the gradient, all
    others zeros)."""
    spec = di.WORKLOADS["abs_b1_l4096_v126464"].scaled(vocab=V, mask_id=V - 1, ids_high=V - 2, n_units=3,
                                                       seq_len=70, spike=0.0, align=align)
    case = di.make_case(spec, "cuda")
    lay = dlm.make_layout(3, 70)
    t, p = dlm.sample_t(9, 3)
    _, corr = dlm.corrupt(lay, case.clean, p, oracle.ABSORBING, spec.mask_id, V, 9)
    out = dlm.loss_fwd_bwd(lay, case.logits, V, case.clean, corr, p, oracle.ABSORBING, align)
    out.dlogits.fill_(float("nan"))
    out = dlm.loss_fwd_bwd(lay, case.logits, V, case.clean, corr, p, oracle.ABSORBING, align, out=out)
    torch.cuda.synchronize()
    assert out.device_status() == 0
    assert not bool(torch.isnan(out.dlogits).any())


def test_every_gradient_element_is_written_uniform():
    spec = di.WORKLOADS["unif_b4_p512_c1024_v262144"].scaled(n_units=2, prefix=8, seq_len=24)
    case = di.make_case(spec, "cuda")
    B, C, P, V = 2, 24, 8, spec.vocab
    lay = dlm.make_layout(B, C)
    enc_lay = dlm.make_layout(B, P + C)
    t, p = dlm.sample_t(2, B, oracle.UNIFORM, spec.eps)
    _, corr = dlm.corrupt(lay, case.clean, p, oracle.UNIFORM, -1, V, 2)
    kw = dict(enc_layout=enc_lay, enc_logits=case.enc_logits, enc_ids=case.enc_clean, enc_ar_weight=1.0)
    out = dlm.loss_fwd_bwd(lay, case.logits, V, case.clean, corr, p, oracle.UNIFORM, oracle.ALIGNED, **kw)
    out.dlogits.fill_(float("nan"))
    out.enc_dlogits.fill_(float("nan"))
    out = dlm.loss_fwd_bwd(lay, case.logits, V, case.clean, corr, p, oracle.UNIFORM, oracle.ALIGNED, out=out,
                           **kw)
    torch.cuda.synchronize()
    assert not bool(torch.isnan(out.dlogits).any())
    assert not bool(torch.isnan(out.enc_dlogits).any())


def test_concurrent_calls_on_two_streams_match_serial():
    """Two loss calls with their own workspaces, in flight together on two
    streams, give bit-identical results to the same calls run one after
    the other: the library keeps no state between calls."""
    specs = [di.WORKLOADS["abs_b1_l4096_v126464"].scaled(seq_len=512),
             di.WORKLOADS["shift_b8_l2048_v152064"].scaled(n_units=2, seq_len=300)]
    cases = [di.make_case(sp, "cuda") for sp in specs]
    lays = [dlm.make_layout(sp.n_units, sp.seq_len) for sp in specs]

    def run(i, seed):
        sp, cs, lay = specs[i], cases[i], lays[i]
        t, p = dlm.sample_t(seed, sp.n_units)
        _, corr = dlm.corrupt(lay, cs.clean, p, oracle.ABSORBING, sp.mask_id, sp.vocab, seed)
        return dlm.loss_fwd_bwd(lay, cs.logits, sp.vocab, cs.clean, corr, p, oracle.ABSORBING, sp.align)

    serial = [run(0, 3), run(1, 4)]
    torch.cuda.synchronize()
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    conc = [None, None]
    for rep in range(3):
        for i, st in enumerate(streams):
            with torch.cuda.stream(st):
                conc[i] = run(i, 3 + i)
        torch.cuda.synchronize()
        for a, b in zip(serial, conc):
            assert torch.equal(a.loss, b.loss)
            assert torch.equal(a.dlogits.view(torch.int16), b.dlogits.view(torch.int16))


def test_bad_target_id_is_flagged_and_row_skipped():
    spec = di.WORKLOADS["abs_b1_l4096_v126464"].scaled(seq_len=64)
    case = di.make_case(spec, "cuda")
    dev = torch.device("cuda")
    clean = case.clean.clone()
    clean[5] = spec.vocab + 3
    lay = dlm.make_layout(1, 64)
    corr = torch.ones(64, dtype=torch.uint8, device=dev)
    p = torch.ones(1, dtype=torch.float32, device=dev)
    out = dlm.loss_fwd_bwd(lay, case.logits, spec.vocab, clean, corr, p)
    assert out.device_status() & dlm.DEV_BAD_TOKEN_ID
    assert bool((out.dlogits[5] == 0).all())
    assert bool((out.dlogits[6] != 0).any())


def test_bad_cu_seqlens_is_flagged_not_faulting():
    spec = di.WORKLOADS["abs_b1_l4096_v126464"].scaled(seq_len=64)
    case = di.make_case(spec, "cuda")
    dev = torch.device("cuda")
    cu = torch.tensor([0, 40, 10, 64], dtype=torch.int32, device=dev)
    lay = dlm.make_layout(3, 0, cu, None, n_tokens=64)
    corr = torch.ones(64, dtype=torch.uint8, device=dev)
    p = torch.ones(3, dtype=torch.float32, device=dev)
    out = dlm.loss_fwd_bwd(lay, case.logits, spec.vocab, case.clean, corr, p)
    assert out.device_status() & dlm.DEV_BAD_LAYOUT


def test_bitwise_reproducible():
    spec = di.WORKLOADS["abs_b1_l4096_v126464"].scaled(seq_len=512)
    case = di.make_case(spec, "cuda")
    dev = torch.device("cuda")
    lay = dlm.make_layout(1, 512)
    t, p = dlm.sample_t(1, 1)
    _, corr = dlm.corrupt(lay, case.clean, p, oracle.ABSORBING, spec.mask_id, spec.vocab, 1)
    a = dlm.loss_fwd_bwd(lay, case.logits, spec.vocab, case.clean, corr, p)
    b = dlm.loss_fwd_bwd(lay, case.logits, spec.vocab, case.clean, corr, p)
    torch.cuda.synchronize()
    assert a.loss.item() == b.loss.item()
    assert torch.equal(a.dlogits.view(torch.int16), b.dlogits.view(torch.int16))
    assert torch.equal(a.unit_loss, b.unit_loss)


# --------------------------------------------------------------------------
# uniform noise + encoder AR term
# --------------------------------------------------------------------------
def run_uniform(spec, case, *, seed=0, grad_rows=None, enc_grad_rows=None, lam=None,
                align=oracle.ALIGNED, grad_scale=1.0, opts=None, canvas_pad=None):
    """opts: (time weighting, cap, reduction) for dlm_loss_fwd_bwd_ex;
    canvas_pad: uint8 [B*C] pad mask of the canvas (examples of unequal
    length)."""
    dev = torch.device("cuda")
    B, C, P, V = spec.n_units, spec.seq_len, spec.prefix, spec.vocab
    lam = spec.enc_ar_weight if lam is None else lam
    pad_d = torch.from_numpy(canvas_pad).to(dev) if canvas_pad is not None else None
    lay = dlm.make_layout(B, C, None, pad_d)
    enc_lay = dlm.make_layout(B, P + C)
    clean = case.clean.to(dev)
    enc_clean = case.enc_clean.to(dev)
    t, p = dlm.sample_t(seed, B, oracle.UNIFORM, spec.eps)
    noisy, corr = dlm.corrupt(lay, clean, p, oracle.UNIFORM, -1, V, seed)
    options = dlm.LossOptions(*opts) if opts is not None else None
    out = dlm.loss_fwd_bwd(lay, case.logits.to(dev), V, clean, corr, p, oracle.UNIFORM, align,
                           enc_layout=enc_lay, enc_logits=case.enc_logits.to(dev),
                           enc_ids=enc_clean, enc_ar_weight=lam, grad_scale=grad_scale, options=options)
    torch.cuda.synchronize()
    assert out.device_status() == 0
    # oracle
    _, p_o = oracle.sample_t(seed, B, oracle.UNIFORM, spec.eps)
    assert np.array_equal(p.cpu().numpy().view(np.uint32), p_o.view(np.uint32))
    lay_o = oracle.Layout(B, C, None, canvas_pad)
    noisy_o, corr_o = oracle.corrupt(lay_o, case.clean.cpu().numpy(), p_o, oracle.UNIFORM, -1, V, seed)
    assert np.array_equal(corr.cpu().numpy(), corr_o)
    assert np.array_equal(noisy.cpu().numpy(), noisy_o)
    xc, xe = _bits(case.logits), _bits(case.enc_logits)
    tw, clip, red = opts if opts is not None else (oracle.NO_TIME_WEIGHT, 0.0, oracle.TOKEN_MEAN)
    loss_o, unit_o, tc, te = oracle.loss_uniform(lay_o, xc, case.clean.cpu().numpy(),
                                                 oracle.Layout(B, P + C, None, None), xe,
                                                 case.enc_clean.cpu().numpy(), V, lam, align, p_o,
                                                 tw, clip, red)
    assert_loss_close(float(out.loss.item()), loss_o)
    assert_units_close(out.unit_loss.cpu().numpy()[:B], unit_o, loss_o)
    rows = np.arange(B * C) if grad_rows is None else np.asarray(grad_rows)
    erows = np.arange(B * (P + C)) if enc_grad_rows is None else np.asarray(enc_grad_rows)
    assert_grad_close(gpu_bf16_to_f64(out.dlogits[torch.from_numpy(rows).to(dev)]),
                      oracle.term_grad(xc, V, tc, rows, grad_scale), "canvas dlogits")
    assert_grad_close(gpu_bf16_to_f64(out.enc_dlogits[torch.from_numpy(erows).to(dev)]),
                      oracle.term_grad(xe, V, te, erows, grad_scale), "encoder dlogits")
    return out


def test_gemma_like_uniform_mid_size_elementwise():
    spec = di.WORKLOADS["unif_b4_p512_c1024_v262144"].scaled(n_units=2, prefix=8, seq_len=32)
    case = di.make_case(spec, "cuda")
    run_uniform(spec, case, seed=0)
    run_uniform(spec, case, seed=1, lam=0.0)
    run_uniform(spec, case, seed=2, lam=0.3, align=oracle.SHIFTED, grad_scale=2.0)


def _canvas_pad(B, C, lengths):
    pad = np.zeros(B * C, np.uint8)
    for b, n in enumerate(lengths):
        pad[b * C + n:(b + 1) * C] = 1
    return pad


@pytest.mark.parametrize("opts", [(oracle.INV_ONE_MINUS_T, 3.0, oracle.EXAMPLE_MEAN),
                                  (oracle.INV_ONE_MINUS_T, 0.0, oracle.TOKEN_MEAN),
                                  (oracle.NO_TIME_WEIGHT, 0.0, oracle.EXAMPLE_MEAN)])
def test_gemma_like_rhine_objective_options(opts):
    """1/(1-t) time weighting with and without a cap, and the mean of
    per-example canvas means, on examples of 32, 20 and 7 canvas tokens."""
    spec = di.WORKLOADS["unif_b4_p512_c1024_v262144"].scaled(n_units=3, prefix=8, seq_len=32)
    case = di.make_case(spec, "cuda")
    run_uniform(spec, case, seed=4, opts=opts, canvas_pad=_canvas_pad(3, 32, (32, 20, 7)))


def test_example_mean_skips_an_example_without_canvas_rows_general_path():
    spec = di.WORKLOADS["unif_b4_p512_c1024_v262144"].scaled(n_units=3, prefix=4, seq_len=16, vocab=1000,
                                                             ids_high=999)
    case = di.make_case(spec, "cuda")
    run_uniform(spec, case, seed=5, opts=(oracle.INV_ONE_MINUS_T, 2.0, oracle.EXAMPLE_MEAN),
                canvas_pad=_canvas_pad(3, 16, (16, 0, 5)), lam=0.5)


def test_gemma_like_uniform_small_vocab_general_path():
    spec = di.WORKLOADS["unif_b4_p512_c1024_v262144"].scaled(vocab=3001, ids_high=3000, n_units=3,
                                                             prefix=5, seq_len=20)
    case = di.make_case(spec, "cuda")
    run_uniform(spec, case, seed=4)


def test_gemma_like_uniform_full_size():
    spec = di.WORKLOADS["unif_b4_p512_c1024_v262144"]
    case = di.make_case(spec, "cuda")
    run_uniform(spec, case, seed=0, grad_rows=_sample_rows(4 * 1024, 1024, k=24),
                enc_grad_rows=_sample_rows(4 * 1536, 1536, k=24))
