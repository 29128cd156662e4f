"""The torch.autograd.Function wrappers of the four losses: loss.backward()
hands over exactly the gradients of the direct calls (bit for bit: the
upstream gradient of the loss itself is 1, and the library's rescale then
touches nothing); a scaled loss scales them in the library (each element
bf16(g x), the same rounding torch's own bf16 product gives); a frozen head
gets no weight gradient; and the gradients match the oracle."""
import numpy as np
import pytest
import torch

import dlm_inputs as di
import oracle
from parity import assert_grad_close, assert_loss_close

pytestmark = pytest.mark.gpu

dlm = pytest.importorskip("diffusion_lm_loss_b200")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dlm.lib()


def _same_bits(a, b):
    return torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_scale_kernel_one_is_untouched_other_factors_round_like_torch():
    gen = torch.Generator(device="cuda")
    gen.manual_seed(0)
    x = (torch.randn((37, 1003), generator=gen, device="cuda") * 5).to(torch.bfloat16)
    for shape_view in (x, x[:, :1000], x.reshape(-1)):
        y = shape_view.clone()
        dlm.scale_bf16_(y, torch.ones(1, device="cuda"))
        assert _same_bits(y, shape_view)
        for g in (0.37, -2.5, 0.0):
            y = shape_view.clone()
            dlm.scale_bf16_(y, torch.full((1,), g, device="cuda"))
            want = (shape_view.float() * g).to(torch.bfloat16)
            assert _same_bits(y, want)


def _loss_inputs(seed=0):
    spec = di.WORKLOADS["abs_b1_l4096_v126464"].scaled(seq_len=256, n_units=2)
    case = di.make_case(spec, "cuda", seed=seed)
    lay = dlm.make_layout(2, 256)
    t, p = dlm.sample_t(seed, 2)
    _, corr = dlm.corrupt(lay, case.clean, p, dlm.ABSORBING, spec.mask_id, spec.vocab, seed)
    return spec, case, lay, p, corr


def test_diffusion_loss_autograd():
    spec, case, lay, p, corr = _loss_inputs()
    direct = dlm.loss_fwd_bwd(lay, case.logits, spec.vocab, case.clean, corr, p)
    logits = case.logits.clone().requires_grad_(True)
    loss = dlm.diffusion_loss(lay, logits, spec.vocab, case.clean, corr, p)
    loss.backward()
    assert loss.item() == direct.loss.item()
    assert _same_bits(logits.grad, direct.dlogits)
    # a scaled loss: the library multiplies the kept gradient
    logits.grad = None
    (dlm.diffusion_loss(lay, logits, spec.vocab, case.clean, corr, p) * 3.0).backward()
    assert _same_bits(logits.grad, (direct.dlogits.float() * 3.0).to(torch.bfloat16))
    # and against the oracle
    lay_o = oracle.Layout(2, 256, None, None)
    _, p_o = oracle.sample_t(0, 2, oracle.ABSORBING, spec.eps)
    _, corr_o = oracle.corrupt(lay_o, case.clean.cpu().numpy(), p_o, oracle.ABSORBING, spec.mask_id, spec.vocab, 0)
    x = di.bf16_bits(case.logits)
    loss_o, _, tr = oracle.loss_absorbing(lay_o, x, spec.vocab, case.clean.cpu().numpy(), corr_o, p_o, oracle.ALIGNED)
    assert_loss_close(loss.item(), loss_o)
    g_o = oracle.term_grad(x, spec.vocab, tr, np.arange(512), 1.0)
    assert_grad_close(direct.dlogits.float().cpu().double().numpy(), g_o)


def test_diffusion_loss_autograd_uniform_two_inputs():
    spec = di.WORKLOADS["unif_b4_p512_c1024_v262144"].scaled(n_units=2, seq_len=64, prefix=32, vocab=4096,
                                                              ids_high=4095)
    case = di.make_case(spec, "cuda", seed=3)
    lay, enc = dlm.make_layout(2, 64), dlm.make_layout(2, 96)
    direct = dlm.loss_fwd_bwd(lay, case.logits, 4096, case.clean, None, None, dlm.UNIFORM, dlm.ALIGNED,
                              enc_layout=enc, enc_logits=case.enc_logits, enc_ids=case.enc_clean, enc_ar_weight=0.5)
    a = case.logits.clone().requires_grad_(True)
    b = case.enc_logits.clone().requires_grad_(True)
    dlm.diffusion_loss(lay, a, 4096, case.clean, None, None, dlm.UNIFORM, dlm.ALIGNED, enc_layout=enc,
                       enc_logits=b, enc_ids=case.enc_clean, enc_ar_weight=0.5).backward()
    assert _same_bits(a.grad, direct.dlogits) and _same_bits(b.grad, direct.enc_dlogits)


def test_linear_losses_autograd_and_frozen_head():
    spec = di.WORKLOADS["lin_t16384_d4096_v126464"].scaled(n_tokens_packed=512, d_model=256, vocab=8192,
                                                           ids_high=8000, mask_id=8191)
    case = di.make_case(spec, "cuda")
    lay = dlm.make_layout(case.n_units, 0, case.cu_seqlens, None, n_tokens=512)
    t, p = dlm.sample_t(1, case.n_units)
    _, corr = dlm.corrupt(lay, case.clean, p, dlm.ABSORBING, spec.mask_id, spec.vocab, 1)
    direct = dlm.linear_loss_fwd_bwd(lay, case.hidden, case.weight, case.clean, corr, p)
    h = case.hidden.clone().requires_grad_(True)
    w = case.weight.clone().requires_grad_(True)
    loss = dlm.linear_diffusion_loss(lay, h, w, case.clean, corr, p)
    (loss * 0.5).backward()
    assert loss.item() == direct.loss.item()
    assert _same_bits(h.grad, (direct.d_hidden.float() * 0.5).to(torch.bfloat16))
    assert _same_bits(w.grad, (direct.d_weight.float() * 0.5).to(torch.bfloat16))
    h2 = case.hidden.clone().requires_grad_(True)
    dlm.linear_diffusion_loss(lay, h2, case.weight, case.clean, corr, p).backward()
    assert _same_bits(h2.grad, direct.d_hidden) and case.weight.grad is None
    # uniform noise through the head
    us = di.WORKLOADS["lin_unif_b4_p512_c1024_d4096_v262144"].scaled(n_units=2, seq_len=64, prefix=32, d_model=128,
                                                                     vocab=4096, ids_high=4095)
    uc = di.make_case(us, "cuda", seed=2)
    ul, ue = dlm.make_layout(2, 64), dlm.make_layout(2, 96)
    ud = dlm.linear_loss_uniform_fwd_bwd(ul, uc.hidden, uc.weight, uc.clean, ue, uc.enc_hidden, uc.enc_clean,
                                         enc_ar_weight=1.0)
    hh = uc.hidden.clone().requires_grad_(True)
    he = uc.enc_hidden.clone().requires_grad_(True)
    ww = uc.weight.clone().requires_grad_(True)
    dlm.linear_uniform_loss(ul, hh, ww, uc.clean, ue, he, uc.enc_clean, 1.0).backward()
    assert _same_bits(hh.grad, ud.d_hidden) and _same_bits(he.grad, ud.d_enc_hidden)
    assert _same_bits(ww.grad, ud.d_weight)


def test_decision_loss_autograd():
    spec = di.WORKLOADS["dec_s128_k26_v126464"]
    case = di.make_case(spec, "cuda")
    e = case.extra
    direct = dlm.decision_loss_fwd_bwd(case.logits, spec.vocab, e["cand_off"], e["cand_ids"], e["kind"], e["val"])
    z = case.logits.clone().requires_grad_(True)
    loss = dlm.decision_loss(z, spec.vocab, e["cand_off"], e["cand_ids"], e["kind"], e["val"])
    (-2.0 * loss).backward()
    assert loss.item() == direct.loss.item()
    assert _same_bits(z.grad, (direct.dlogits.float() * -2.0).to(torch.bfloat16))
