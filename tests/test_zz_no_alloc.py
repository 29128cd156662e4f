"""dlm_loss_fwd_bwd_static: the loss for callers that may not allocate device
memory (they are handed only their inputs and outputs, e.g. a plugin inside a
program that owns all GPU memory), so they cannot pass a workspace.  Its
scratch is a fixed array inside the library.

Called through the C ABI (ctypes), twice in a row, and compared with
dlm_loss_fwd_bwd on the same inputs: the two run the same kernels, so the
results must agree within the parity tolerances (loss 1e-5 relative, bf16
gradients 2e-3 absolute).  The file is named so pytest collects it last; it
also passes on its own in a fresh process.
"""
import ctypes

import pytest
import torch

import dlm_inputs as di

pytestmark = pytest.mark.gpu

dlm = pytest.importorskip("diffusion_lm_loss_b200")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dlm.lib()


def _static_call(L, lay, logits, V, clean, corr, p, mode, align, loss, unit, dlogits,
                 enc_lay=None, enc_logits=None, enc_ids=None, lam=0.0):
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return L.dlm_loss_fwd_bwd_static(
        ctypes.byref(lay), logits.data_ptr(), logits.stride(0), V, clean.data_ptr(),
        corr.data_ptr() if corr is not None else None, p.data_ptr() if p is not None else None,
        mode, align, ctypes.byref(enc_lay) if enc_lay is not None else None,
        enc_logits.data_ptr() if enc_logits is not None else None,
        enc_logits.stride(0) if enc_logits is not None else 0,
        enc_ids.data_ptr() if enc_ids is not None else None, lam, 1.0, loss.data_ptr(), unit.data_ptr(),
        dlogits.data_ptr(), None, stream)


@pytest.mark.parametrize("key,L_len", [("abs_b1_l4096_v126464", 512), ("shift_b8_l2048_v152064", 64),
                                       ("abs_b2_l64_v1024", 64)])
def test_static_entry_matches_workspace_entry_twice(key, L_len):
    spec = di.WORKLOADS[key].scaled(seq_len=L_len)
    case = di.make_case(spec, "cuda")
    L = dlm.lib()
    dev = torch.device("cuda")
    B, V = spec.n_units, spec.vocab
    lay = dlm.make_layout(B, L_len)
    for call, seed in enumerate((21, 22)):
        t, p = dlm.sample_t(seed, B, spec.mode, spec.eps)
        _, corr = dlm.corrupt(lay, case.clean, p, spec.mode, spec.mask_id, V, seed)
        ref = dlm.loss_fwd_bwd(lay, case.logits, V, case.clean, corr, p, spec.mode, spec.align)
        loss = torch.full((1,), float("nan"), device=dev)
        unit = torch.full((B,), float("nan"), device=dev)
        dl = torch.full_like(case.logits, 3.0)
        rc = _static_call(L, lay, case.logits, V, case.clean, corr, p, spec.mode, spec.align, loss, unit, dl)
        assert rc == 0, (call, dlm.STATUS.get(rc, rc))
        torch.cuda.synchronize()
        lo, lr = float(loss.item()), float(ref.loss.item())
        assert abs(lo - lr) <= 1e-5 * abs(lr), (call, lo, lr)
        assert torch.allclose(unit, ref.unit_loss[:B], rtol=1e-5, atol=1e-7)
        assert float((dl.float() - ref.dlogits.float()).abs().max()) <= 2e-3


def test_static_entry_uniform_with_encoder():
    spec = di.WORKLOADS["unif_b4_p512_c1024_v262144"].scaled(n_units=2, prefix=8, seq_len=24)
    case = di.make_case(spec, "cuda")
    L = dlm.lib()
    dev = torch.device("cuda")
    lay = dlm.make_layout(2, 24)
    enc_lay = dlm.make_layout(2, 32)
    t, p = dlm.sample_t(5, 2, spec.mode, spec.eps)
    _, corr = dlm.corrupt(lay, case.clean, p, spec.mode, -1, spec.vocab, 5)
    ref = dlm.loss_fwd_bwd(lay, case.logits, spec.vocab, case.clean, corr, p, spec.mode, spec.align,
                           enc_layout=enc_lay, enc_logits=case.enc_logits, enc_ids=case.enc_clean,
                           enc_ar_weight=1.0)
    for _ in range(2):
        loss = torch.empty(1, device=dev)
        unit = torch.empty(2, device=dev)
        dl = torch.empty_like(case.logits)
        stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
        edl = torch.empty_like(case.enc_logits)
        rc = L.dlm_loss_fwd_bwd_static(ctypes.byref(lay), case.logits.data_ptr(), spec.vocab, spec.vocab,
                                       case.clean.data_ptr(), corr.data_ptr(), p.data_ptr(), spec.mode,
                                       spec.align, ctypes.byref(enc_lay), case.enc_logits.data_ptr(),
                                       spec.vocab, case.enc_clean.data_ptr(), 1.0, 1.0, loss.data_ptr(),
                                       unit.data_ptr(), dl.data_ptr(), edl.data_ptr(), stream)
        assert rc == 0
        torch.cuda.synchronize()
        assert abs(float(loss.item()) - float(ref.loss.item())) <= 1e-5 * abs(float(ref.loss.item()))
        assert float((dl.float() - ref.dlogits.float()).abs().max()) <= 2e-3
        assert float((edl.float() - ref.enc_dlogits.float()).abs().max()) <= 2e-3


def test_static_entry_refuses_problems_beyond_its_scratch():
    L = dlm.lib()
    dev = torch.device("cuda")
    big = dlm.make_layout(1, 1 << 20)          # one million rows: needs ~20 MB of scratch
    dummy = torch.empty(16, dtype=torch.int32, device=dev)
    rc = L.dlm_loss_fwd_bwd_static(ctypes.byref(big), dummy.data_ptr(), 4096, 4096, dummy.data_ptr(),
                                   dummy.data_ptr(), dummy.data_ptr(), 0, 0, None, None, 0, None, 0.0, 1.0,
                                   dummy.data_ptr(), None, dummy.data_ptr(), None, None)
    assert rc == 3   # DLM_ERR_WORKSPACE_TOO_SMALL, nothing enqueued
