"""GPU parity of the fused lm_head + loss (tensor-core path) against the CPU
oracle ("Native diffusion language-model training", Adapters, merging and
inference: Cut Cross Entropy -- aligned absorbing loss from hidden states).

Loss within 1e-5 relative, every per-unit sum, and dH and dW element by
element (the bar for a bf16 sum of products whose one operand was rounded
to bf16, in parity.py), at sizes the oracle finishes in seconds (ragged
vocabulary tiles, d_model below one output tile, several backward
vocabulary chunks) and at the full sizes of both fused-head workloads
(packed documents T=16,384, D=4,096, V=126,464; DiffusionGemma-like canvas
and encoder, V=262,144), plus identities that hold at any size:
<dW, W> = <dH, H> (both equal sum_{m,v} dZ[m,v] Z[m,v]) and sum_v dW[v,:] = 0.
"""
import numpy as np
import pytest
import torch

import dlm_inputs as di
import oracle
from parity import assert_bf16_sum_close, assert_loss_close, assert_units_close, product_rms_scale

pytestmark = pytest.mark.gpu

dlm = pytest.importorskip("diffusion_lm_loss_b200")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dlm.lib()


def _host_f32(t):
    """A bf16 device tensor as a float32 numpy array (exact: every bf16
    value is a float32 value; half the host memory of float64)."""
    return t.detach().float().cpu().numpy()


def assert_fused_grads(ref, W, terms, dW_gpu):
    """dH of every term element by element on its scored rows and exact
    zeros on all other rows; dW element by element.  terms: (name, gpu dH
    [rows, D] device tensor, H [rows, D] device tensor, oracle key of dH,
    oracle key of the scored rows, oracle key of dZ).  Returns the relative
    Frobenius errors, for reports."""
    Wd = _host_f32(W)
    fro = {}
    s2_dw = None
    for name, g, H, k_dh, k_rows, k_dz in terms:
        rows, dZ = ref[k_rows], ref[k_dz]
        gd = _host_f32(g)
        fro[name] = assert_bf16_sum_close(gd[rows], ref[k_dh][rows], product_rms_scale(dZ, Wd), name)
        un = np.ones(gd.shape[0], bool)
        un[rows] = False
        assert (gd[un] == 0).all(), f"{name}: nonzero rows where nothing is scored"
        del gd
        if dW_gpu is not None:
            s = product_rms_scale(dZ, _host_f32(H)[rows], transpose_a=True)
            s2_dw = s * s if s2_dw is None else s2_dw + s * s
            del s
    if dW_gpu is not None:
        fro["dW"] = assert_bf16_sum_close(_host_f32(dW_gpu), ref["dW"], np.sqrt(s2_dw), "dW")
    return fro


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
                             align=oracle.SHIFTED, keep_dz=True)
    assert_loss_close(float(out.loss.item()), ref["loss"])
    assert_units_close(out.unit_loss.cpu().numpy()[:case.n_units], ref["unit_loss"], ref["loss"])
    assert_fused_grads(ref, case.weight, [("dH", out.d_hidden, case.hidden, "dH", "rows", "dZ")], out.d_weight)


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
                             case.clean.cpu().numpy(), corr_o, p_o, grad_scale=-0.5, keep_dz=True)
    assert_loss_close(float(out.loss.item()), ref["loss"])
    assert_fused_grads(ref, case.weight, [("dH", out.d_hidden, case.hidden, "dH", "rows", "dZ")], None)


@pytest.mark.parametrize("T,D,V,seed", [(64, 64, 1000, 0), (512, 256, 4096, 1), (300, 128, 2056, 2),
                                        (2048, 512, 40000, 3)])
def test_linear_elementwise(T, D, V, seed):
    spec = di.WORKLOADS["lin_t16384_d4096_v126464"].scaled(n_tokens_packed=T, d_model=D, vocab=V,
                                                           ids_high=V - 2, mask_id=V - 1, doc_mean=50.0)
    case = di.make_case(spec, "cuda")
    out, lay_o, p_o, corr_o = run_linear(spec, case, seed=seed, grad_scale=0.5)
    H = di.bf16_bits(case.hidden)
    W = di.bf16_bits(case.weight)
    ref = oracle.linear_loss(lay_o, H, W, case.clean.cpu().numpy(), corr_o, p_o, grad_scale=0.5, keep_dz=True)
    assert_loss_close(float(out.loss.item()), ref["loss"])
    assert_units_close(out.unit_loss.cpu().numpy()[:case.n_units], ref["unit_loss"], ref["loss"])
    assert_fused_grads(ref, case.weight, [("dH", out.d_hidden, case.hidden, "dH", "rows", "dZ")], out.d_weight)


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


def _identities(dW, W, pairs):
    """<dW, W> = sum over terms <dH, H> (both are sum_{m,v} dZ[m,v] Z[m,v]),
    and sum_v dW[v, :] = 0 (each row of dZ sums to zero)."""
    dWd = dW.double()
    lhs = float((dWd * W.double()).sum())
    rhs = sum(float((g.double() * H.double()).sum()) for g, H in pairs)
    assert abs(lhs - rhs) <= 2e-3 * max(abs(lhs), abs(rhs))
    colsum = dWd.sum(0).abs().max().item()
    assert colsum <= 1e-2 * dWd.abs().sum(0).max().item()


def _need_host_memory(gb: float):
    """The full-size comparisons run the oracle in double on the host (the
    logits, their softmax and dW of a 1-4 GB head); on a host with less free
    memory they are skipped rather than driving the machine out of memory."""
    import psutil
    avail = psutil.virtual_memory().available / 1e9
    if avail < gb:
        pytest.skip(f"the full-size oracle comparison needs ~{gb:.0f} GB of free host memory, {avail:.0f} GB free")


def test_linear_full_size():
    """The packed-document fused-head workload at full size (T=16,384,
    D=4,096, V=126,464, ~7,800 masked rows) against the oracle run in full:
    the loss within 1e-5 relative, every per-document sum, dH on every
    masked row and every element of dW."""
    _need_host_memory(40.0)
    spec = di.WORKLOADS["lin_t16384_d4096_v126464"]
    case = di.make_case(spec, "cuda")
    out, lay_o, p_o, corr_o = run_linear(spec, case, seed=0)
    ref = oracle.linear_loss(lay_o, di.bf16_bits(case.hidden), di.bf16_bits(case.weight),
                             case.clean.cpu().numpy(), corr_o, p_o, keep_dz=True)
    M = ref["rows"].shape[0]
    assert 0.3 * 16384 < M < 0.7 * 16384
    assert_loss_close(float(out.loss.item()), ref["loss"])
    assert_units_close(out.unit_loss.cpu().numpy()[:case.n_units], ref["unit_loss"], ref["loss"])
    fro = assert_fused_grads(ref, case.weight, [("dH", out.d_hidden, case.hidden, "dH", "rows", "dZ")],
                             out.d_weight)
    print(f"full-size fused head: M={M}, relative Frobenius errors {fro}")
    _identities(out.d_weight, case.weight, [(out.d_hidden, case.hidden)])


# --------------------------------------------------------------------------
# uniform noise through the fused head: canvas term + encoder AR term
# ("diffusiongemma-26B-A4B-it-ALWAYS-THINK", Finetuning notes)
# --------------------------------------------------------------------------
def run_linear_uniform(spec, case, lam, align=oracle.ALIGNED, grad_scale=1.0, want_dw=True,
                       canvas_pad=None, enc_pad=None, with_encoder=True):
    dev = torch.device("cuda")
    B, C, P = case.n_units, case.seq_len, spec.prefix
    cp = torch.from_numpy(canvas_pad).to(dev) if canvas_pad is not None else None
    ep = torch.from_numpy(enc_pad).to(dev) if enc_pad is not None else None
    lay = dlm.make_layout(B, C, None, cp)
    enc = dlm.make_layout(B, P + C, None, ep) if with_encoder else None
    out = dlm.linear_loss_uniform_fwd_bwd(
        lay, case.hidden, case.weight, case.clean, enc, case.enc_hidden if with_encoder else None,
        case.enc_clean if with_encoder else None, enc_ar_weight=lam, align=align, grad_scale=grad_scale,
        want_d_weight=want_dw)
    torch.cuda.synchronize()
    assert out.device_status() == 0
    lay_o = oracle.Layout(B, C, None, canvas_pad)
    enc_o = oracle.Layout(B, P + C, None, enc_pad) if with_encoder else None
    ref = oracle.linear_loss_uniform(
        lay_o, di.bf16_bits(case.hidden), di.bf16_bits(case.weight), case.clean.cpu().numpy(), enc_o,
        di.bf16_bits(case.enc_hidden) if with_encoder else None,
        case.enc_clean.cpu().numpy() if with_encoder else None, lam, align, grad_scale=grad_scale,
        want_grads=True, keep_dz=True)
    return out, ref


def UNIFORM_TERMS(out, case):
    """The canvas and the encoder term of a fused uniform call, for
    assert_fused_grads."""
    return [("dH", out.d_hidden, case.hidden, "dH", "rows", "dZ"),
            ("dHe", out.d_enc_hidden, case.enc_hidden, "dHe", "enc_rows", "dZe")]


def _uniform_spec(B, C, P, D, V):
    return di.WORKLOADS["lin_unif_b4_p512_c1024_d4096_v262144"].scaled(
        n_units=B, seq_len=C, prefix=P, d_model=D, vocab=V, ids_high=V - 1)


@pytest.mark.parametrize("B,C,P,D,V,align,seed", [
    (2, 40, 24, 64, 1000, oracle.ALIGNED, 0),       # ragged vocabulary tile, one row tile
    (3, 300, 197, 128, 4104, oracle.SHIFTED, 1),    # ~2,400 rows: ten paired row tiles, ragged
    (4, 256, 128, 256, 20000, oracle.ALIGNED, 2),   # two backward vocabulary chunks
])
def test_linear_uniform_elementwise(B, C, P, D, V, align, seed):
    spec = _uniform_spec(B, C, P, D, V)
    case = di.make_case(spec, "cuda", seed=seed)
    out, ref = run_linear_uniform(spec, case, lam=0.8, align=align, grad_scale=0.5)
    assert_loss_close(float(out.loss.item()), ref["loss"])
    assert_units_close(out.unit_loss.cpu().numpy()[:B], ref["unit_loss"], ref["loss"])
    # element by element; rows with no target are exact zeros (each unit's
    # last canvas row when shifted, each unit's last encoder row)
    assert_fused_grads(ref, case.weight, UNIFORM_TERMS(out, case), out.d_weight)
    assert ref["enc_rows"].shape[0] == B * (P + C - 1)


def test_linear_uniform_pads_without_encoder_no_dw():
    """Padded canvas tokens are never scored; no encoder term; d_weight
    skipped; negative gradient scale."""
    B, C, D, V = 3, 200, 128, 4096
    spec = _uniform_spec(B, C, 0, D, V)
    case = di.make_case(spec, "cuda", seed=3)
    pad = np.zeros(B * C, np.uint8)
    for b, n in enumerate((200, 151, 9)):
        pad[b * C + n:(b + 1) * C] = 1
    out, ref = run_linear_uniform(spec, case, lam=1.0, grad_scale=-0.25, want_dw=False, canvas_pad=pad,
                                  with_encoder=False)
    assert out.d_weight is None and out.d_enc_hidden is None
    assert_loss_close(float(out.loss.item()), ref["loss"])
    assert_fused_grads(ref, case.weight, UNIFORM_TERMS(out, case)[:1], None)
    assert (out.d_hidden[torch.from_numpy(pad).cuda().bool()] == 0).all()


def test_linear_uniform_encoder_pads():
    """Padded encoder positions: neither scored nor a target."""
    B, C, P, D, V = 2, 96, 64, 64, 2048
    spec = _uniform_spec(B, C, P, D, V)
    case = di.make_case(spec, "cuda", seed=4)
    epad = np.zeros(B * (P + C), np.uint8)
    epad[(P + C) - 30:(P + C)] = 1          # unit 0 ends 30 tokens early
    out, ref = run_linear_uniform(spec, case, lam=2.0, enc_pad=epad)
    assert_loss_close(float(out.loss.item()), ref["loss"])
    assert_units_close(out.unit_loss.cpu().numpy()[:B], ref["unit_loss"], ref["loss"])
    assert_fused_grads(ref, case.weight, UNIFORM_TERMS(out, case), out.d_weight)
    assert ref["enc_rows"].shape[0] == (P + C - 31) + (P + C - 1)


def test_linear_uniform_matches_unfused_gpu_path_on_materialised_logits():
    """The fused uniform call and dlm_loss_fwd_bwd (uniform, with the
    encoder term) on logits = H W^T rounded to bf16 agree to that rounding."""
    B, C, P, D, V = 2, 128, 64, 256, 8192
    spec = _uniform_spec(B, C, P, D, V)
    case = di.make_case(spec, "cuda", seed=5)
    dev = torch.device("cuda")
    lay = dlm.make_layout(B, C)
    enc = dlm.make_layout(B, P + C)
    fused = dlm.linear_loss_uniform_fwd_bwd(lay, case.hidden, case.weight, case.clean, enc, case.enc_hidden,
                                            case.enc_clean, enc_ar_weight=0.5)
    logits = (case.hidden.float() @ case.weight.float().T).to(torch.bfloat16)
    enc_logits = (case.enc_hidden.float() @ case.weight.float().T).to(torch.bfloat16)
    p = torch.ones(B, dtype=torch.float32, device=dev)
    corr = torch.ones(B * C, dtype=torch.uint8, device=dev)
    ref = dlm.loss_fwd_bwd(lay, logits, V, case.clean, corr, p, oracle.UNIFORM, oracle.ALIGNED,
                           enc_layout=enc, enc_logits=enc_logits, enc_ids=case.enc_clean, enc_ar_weight=0.5)
    torch.cuda.synchronize()
    a, b = float(fused.loss.item()), float(ref.loss.item())
    assert abs(a - b) < 2e-3 * abs(b)


def test_linear_uniform_full_size():
    """DiffusionGemma-like shapes (B=4, prefix 512 + canvas 1024, D=4,096,
    V=262,144; 10,236 scored rows) against the oracle run in full: the loss
    within 1e-5 relative, the per-unit sums, dH and dH_enc on every row and
    every element of dW (the sum of both terms' contributions)."""
    _need_host_memory(72.0)
    spec = di.WORKLOADS["lin_unif_b4_p512_c1024_d4096_v262144"]
    case = di.make_case(spec, "cuda")
    B, C, P = 4, 1024, 512
    out, ref = run_linear_uniform(spec, case, lam=1.0)
    assert ref["rows"].shape[0] + ref["enc_rows"].shape[0] == B * C + B * (P + C - 1)
    assert_loss_close(float(out.loss.item()), ref["loss"])
    assert_units_close(out.unit_loss.cpu().numpy()[:B], ref["unit_loss"], ref["loss"])
    fro = assert_fused_grads(ref, case.weight, UNIFORM_TERMS(out, case), out.d_weight)
    print(f"full-size fused head, uniform noise: relative Frobenius errors {fro}")
    _identities(out.d_weight, case.weight, [(out.d_hidden, case.hidden), (out.d_enc_hidden, case.enc_hidden)])
