"""GPU parity of the fused lm_head + loss (tensor-core path) against the CPU
oracle ("Native diffusion language-model training", Adapters, merging and
inference: Cut Cross Entropy -- aligned absorbing loss from hidden states).

Element by element at sizes the oracle finishes in seconds (ragged vocabulary
tiles, d_model below one output tile, several backward vocabulary chunks);
at the full packed-document size: per-document sums of short documents, dH
rows of sampled masked tokens, and identities that hold at any size:
<dW, W> = <dH, H> (both equal sum_{m,v} dZ[m,v] Z[m,v]) and sum_v dW[v,:] = 0.
"""
import numpy as np
import pytest
import torch

import dlm_inputs as di
import oracle
from parity import assert_loss_close, assert_units_close

pytestmark = pytest.mark.gpu

dlm = pytest.importorskip("diffusion_lm_loss_b200")

# dH, dW are bf16 outputs of fp32 sums over D (dH) or M (dW) products: the
# bar is a relative Frobenius error against the double-precision oracle.
GRAD_REL_FRO = 5e-3


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dlm.lib()


def rel_fro(a, b):
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def run_linear(spec, case, seed=0, grad_scale=1.0, want_dw=True, align=oracle.ALIGNED):
    dev = torch.device("cuda")
    T = case.n_tokens
    lay = dlm.make_layout(case.n_units, case.seq_len, case.cu_seqlens.to(dev) if case.cu_seqlens is not None else None,
                          None, n_tokens=T)
    clean = case.clean.to(dev)
    t, p = dlm.sample_t(seed, case.n_units, oracle.ABSORBING, spec.eps)
    _, corr = dlm.corrupt(lay, clean, p, oracle.ABSORBING, spec.mask_id, spec.vocab, seed)
    out = dlm.linear_loss_fwd_bwd(lay, case.hidden.to(dev), case.weight.to(dev), clean, corr, p,
                                  grad_scale=grad_scale, want_d_weight=want_dw, align=align)
    torch.cuda.synchronize()
    assert out.device_status() == 0
    cu = case.cu_seqlens.cpu().numpy() if case.cu_seqlens is not None else None
    lay_o = oracle.Layout(case.n_units, case.seq_len, cu, None)
    _, p_o = oracle.sample_t(seed, case.n_units, oracle.ABSORBING, spec.eps)
    _, corr_o = oracle.corrupt(lay_o, case.clean.cpu().numpy(), p_o, oracle.ABSORBING, spec.mask_id,
                               spec.vocab, seed)
    assert np.array_equal(corr.cpu().numpy(), corr_o)
    return out, lay_o, p_o, corr_o


@pytest.mark.parametrize("T,D,V,seed", [(64, 64, 1000, 4), (700, 128, 4104, 5), (2048, 256, 20000, 6)])
def test_linear_shifted_elementwise(T, D, V, seed):
    """Shifted targets through the fused head: hidden state i scores token
    i+1 of its document (the unfused loss's Dream alignment)."""
    spec = di.WORKLOADS["lin_t16384_d4096_v126464"].scaled(n_tokens_packed=T, d_model=D, vocab=V,
                                                           ids_high=V - 2, mask_id=V - 1, doc_mean=50.0)
    case = di.make_case(spec, "cuda")
    out, lay_o, p_o, corr_o = run_linear(spec, case, seed=seed, grad_scale=0.75, align=oracle.SHIFTED)
    H = di.bf16_bits(case.hidden)
    W = di.bf16_bits(case.weight)
    ref = oracle.linear_loss(lay_o, H, W, case.clean.cpu().numpy(), corr_o, p_o, grad_scale=0.75,
                             align=oracle.SHIFTED)
    assert_loss_close(float(out.loss.item()), ref["loss"])
    assert_units_close(out.unit_loss.cpu().numpy()[:case.n_units], ref["unit_loss"], ref["loss"])
    dH = out.d_hidden.double().cpu().numpy()
    dW = out.d_weight.double().cpu().numpy()
    assert rel_fro(dH, ref["dH"]) < GRAD_REL_FRO
    assert rel_fro(dW, ref["dW"]) < GRAD_REL_FRO
    unscored = np.ones(T, bool)
    unscored[ref["rows"]] = False
    assert (dH[unscored] == 0).all()


def test_linear_pads_negative_scale_no_dw():
    """Padded tokens (never scored, not counted in N), a negative gradient
    scale, and d_weight skipped."""
    T, D, V = 640, 128, 4096
    spec = di.WORKLOADS["lin_t16384_d4096_v126464"].scaled(n_tokens_packed=T, d_model=D, vocab=V,
                                                           ids_high=V - 2, mask_id=V - 1, doc_mean=60.0)
    case = di.make_case(spec, "cuda")
    dev = torch.device("cuda")
    rng = np.random.default_rng(8)
    pad = (rng.random(T) < 0.15).astype(np.uint8)
    lay = dlm.make_layout(case.n_units, 0, case.cu_seqlens, torch.from_numpy(pad).to(dev), n_tokens=T)
    t, p = dlm.sample_t(8, case.n_units)
    _, corr = dlm.corrupt(lay, case.clean, p, oracle.ABSORBING, spec.mask_id, V, 8)
    out = dlm.linear_loss_fwd_bwd(lay, case.hidden, case.weight, case.clean, corr, p, grad_scale=-0.5,
                                  want_d_weight=False)
    torch.cuda.synchronize()
    assert out.device_status() == 0 and out.d_weight is None
    lay_o = oracle.Layout(case.n_units, 0, case.cu_seqlens.cpu().numpy(), pad)
    _, p_o = oracle.sample_t(8, case.n_units, oracle.ABSORBING, spec.eps)
    _, corr_o = oracle.corrupt(lay_o, case.clean.cpu().numpy(), p_o, oracle.ABSORBING, spec.mask_id, V, 8)
    assert np.array_equal(corr.cpu().numpy(), corr_o)
    assert not corr_o[pad == 1].any()
    ref = oracle.linear_loss(lay_o, di.bf16_bits(case.hidden), di.bf16_bits(case.weight),
                             case.clean.cpu().numpy(), corr_o, p_o, grad_scale=-0.5)
    assert_loss_close(float(out.loss.item()), ref["loss"])
    assert rel_fro(out.d_hidden.double().cpu().numpy(), ref["dH"]) < GRAD_REL_FRO


@pytest.mark.parametrize("T,D,V,seed", [(64, 64, 1000, 0), (512, 256, 4096, 1), (300, 128, 2056, 2),
                                        (2048, 512, 40000, 3)])
def test_linear_elementwise(T, D, V, seed):
    spec = di.WORKLOADS["lin_t16384_d4096_v126464"].scaled(n_tokens_packed=T, d_model=D, vocab=V,
                                                           ids_high=V - 2, mask_id=V - 1, doc_mean=50.0)
    case = di.make_case(spec, "cuda")
    out, lay_o, p_o, corr_o = run_linear(spec, case, seed=seed, grad_scale=0.5)
    H = di.bf16_bits(case.hidden)
    W = di.bf16_bits(case.weight)
    ref = oracle.linear_loss(lay_o, H, W, case.clean.cpu().numpy(), corr_o, p_o, grad_scale=0.5)
    assert_loss_close(float(out.loss.item()), ref["loss"])
    assert_units_close(out.unit_loss.cpu().numpy()[:case.n_units], ref["unit_loss"], ref["loss"])
    dH = out.d_hidden.double().cpu().numpy()
    dW = out.d_weight.double().cpu().numpy()
    assert rel_fro(dH, ref["dH"]) < GRAD_REL_FRO
    assert rel_fro(dW, ref["dW"]) < GRAD_REL_FRO
    unscored = np.ones(T, bool)
    unscored[ref["rows"]] = False
    assert (dH[unscored] == 0).all()


def test_linear_no_masked_rows():
    spec = di.WORKLOADS["lin_t16384_d4096_v126464"].scaled(n_tokens_packed=256, d_model=128, vocab=1024,
                                                           ids_high=1000, mask_id=1023)
    case = di.make_case(spec, "cuda")
    dev = torch.device("cuda")
    lay = dlm.make_layout(case.n_units, 0, case.cu_seqlens.to(dev), None, n_tokens=256)
    corr = torch.zeros(256, dtype=torch.uint8, device=dev)
    p = torch.full((case.n_units,), 0.5, device=dev)
    out = dlm.linear_loss_fwd_bwd(lay, case.hidden, case.weight, case.clean, corr, p)
    torch.cuda.synchronize()
    assert float(out.loss.item()) == 0.0
    assert bool((out.d_hidden == 0).all()) and bool((out.d_weight == 0).all())


def test_linear_matches_unfused_gpu_path_on_materialised_logits():
    """Same loss through the fused head and through dlm_loss_fwd_bwd on
    logits = H W^T (fp32, rounded to bf16): agree to the bf16 rounding of the
    materialised logits."""
    spec = di.WORKLOADS["lin_t16384_d4096_v126464"].scaled(n_tokens_packed=256, d_model=256, vocab=8192,
                                                           ids_high=8000, mask_id=8191)
    case = di.make_case(spec, "cuda")
    out, lay_o, p_o, corr_o = run_linear(spec, case, seed=5)
    dev = torch.device("cuda")
    logits = (case.hidden.float() @ case.weight.float().T).to(torch.bfloat16)
    lay = dlm.make_layout(case.n_units, 0, case.cu_seqlens.to(dev), None, n_tokens=256)
    p = torch.from_numpy(p_o).to(dev)
    corr = torch.from_numpy(corr_o).to(dev)
    ref = dlm.loss_fwd_bwd(lay, logits, 8192, case.clean, corr, p)
    torch.cuda.synchronize()
    assert abs(float(out.loss.item()) - float(ref.loss.item())) < 2e-3 * abs(float(ref.loss.item()))


def test_linear_bitwise_reproducible():
    spec = di.WORKLOADS["lin_t16384_d4096_v126464"].scaled(n_tokens_packed=512, d_model=256, vocab=20000,
                                                           ids_high=19000, mask_id=19999)
    case = di.make_case(spec, "cuda")
    a, *_ = run_linear(spec, case, seed=7)
    b, *_ = run_linear(spec, case, seed=7)
    assert a.loss.item() == b.loss.item()
    assert torch.equal(a.d_hidden.view(torch.int16), b.d_hidden.view(torch.int16))
    assert torch.equal(a.d_weight.view(torch.int16), b.d_weight.view(torch.int16))


def test_linear_full_size():
    spec = di.WORKLOADS["lin_t16384_d4096_v126464"]
    case = di.make_case(spec, "cuda")
    out, lay_o, p_o, corr_o = run_linear(spec, case, seed=0)
    H = di.bf16_bits(case.hidden)
    W = di.bf16_bits(case.weight)
    clean = case.clean.cpu().numpy()
    plan = oracle.plan_diffusion(lay_o, clean, corr_o, p_o, oracle.ABSORBING, oracle.ALIGNED)
    scored = np.nonzero(plan.target >= 0)[0]
    M = scored.shape[0]
    assert 0.3 * 16384 < M < 0.7 * 16384
    # dH on sampled masked rows (each needs only its own row's softmax)
    rng = np.random.default_rng(0)
    sample = np.sort(rng.choice(scored, size=12, replace=False))
    spot = oracle.linear_rows(lay_o, H, W, clean, corr_o, p_o, sample)
    dH = out.d_hidden.double().cpu().numpy()
    assert rel_fro(dH[sample], spot["dH"]) < GRAD_REL_FRO
    # per-document sums of the shortest documents (every masked row of the doc)
    cu = case.cu_seqlens.cpu().numpy()
    lens = np.diff(cu)
    unit_gpu = out.unit_loss.cpu().numpy()
    for u in np.argsort(lens)[:3]:
        rows = scored[(scored >= cu[u]) & (scored < cu[u + 1])]
        want = 0.0 if rows.size == 0 else float(
            oracle.linear_rows(lay_o, H, W, clean, corr_o, p_o, rows)["weighted"].sum())
        assert abs(unit_gpu[u] - want) <= 1e-5 * max(abs(want), 1e-12) + 1e-9
    # unscored rows of dH are exact zeros
    un = np.setdiff1d(np.arange(16384), scored)
    assert (dH[un[:200]] == 0).all()
    # identities at any size
    dW = out.d_weight.double()
    Wd = case.weight.double()
    Hd = case.hidden.double()
    lhs = float((dW * Wd).sum())
    rhs = float((out.d_hidden.double() * Hd).sum())
    assert abs(lhs - rhs) <= 2e-3 * max(abs(lhs), abs(rhs))
    colsum = dW.sum(0).abs().max().item()
    assert colsum <= 1e-2 * dW.abs().sum(0).max().item()
