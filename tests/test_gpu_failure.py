"""Failure detection and less common branches, on the GPU.

* The bounded on-chip wait: a kernel waits on a barrier phase nothing
  completes; it must give up after its limit, flag DLM_DEV_WAIT_TIMEOUT and
  leave the context usable (no trap, no fault, no hang).
* Data-dependent errors of the fused head (bad ids) are flagged, not faults.
* Negative gradient scale (the exponent-folding shortcut does not apply) and
  dense sequences with padding, against the oracle.
"""
import ctypes
import time

import numpy as np
import pytest
import torch

import dlm_inputs as di
import oracle
from parity import assert_grad_close, assert_loss_close, assert_units_close, gpu_bf16_to_f64

pytestmark = pytest.mark.gpu

dlm = pytest.importorskip("diffusion_lm_loss_b200")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dlm.lib()


def test_bounded_wait_gives_up_and_context_survives():
    L = dlm.lib()
    dev = torch.device("cuda")
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    assert L.dlm_selftest_bounded_wait(20_000_000, status.data_ptr(), stream) == 0   # 20 ms
    torch.cuda.synchronize()
    dt = time.perf_counter() - t0
    assert int(status.item()) & dlm.DEV_WAIT_TIMEOUT
    assert 0.015 < dt < 5.0
    # the context still works: a normal loss call afterwards
    spec = di.WORKLOADS["abs_b2_l64_v1024"]
    case = di.make_case(spec, "cuda")
    lay = dlm.make_layout(2, 64)
    t, p = dlm.sample_t(0, 2)
    _, corr = dlm.corrupt(lay, case.clean, p, oracle.ABSORBING, spec.mask_id, spec.vocab, 0)
    out = dlm.loss_fwd_bwd(lay, case.logits, spec.vocab, case.clean, corr, p)
    torch.cuda.synchronize()
    assert np.isfinite(float(out.loss.item())) and out.device_status() == 0


@pytest.mark.parametrize("g", [-0.5, 0.0])
def test_negative_and_zero_grad_scale(g):
    spec = di.WORKLOADS["abs_b1_l4096_v126464"].scaled(seq_len=128)
    case = di.make_case(spec, "cuda")
    lay = dlm.make_layout(1, 128)
    t, p = dlm.sample_t(3, 1)
    _, corr = dlm.corrupt(lay, case.clean, p, oracle.ABSORBING, spec.mask_id, spec.vocab, 3)
    out = dlm.loss_fwd_bwd(lay, case.logits, spec.vocab, case.clean, corr, p, grad_scale=g)
    torch.cuda.synchronize()
    lay_o = oracle.Layout(1, 128, None, None)
    _, p_o = oracle.sample_t(3, 1, oracle.ABSORBING, 1e-3)
    _, corr_o = oracle.corrupt(lay_o, case.clean.cpu().numpy(), p_o, oracle.ABSORBING, spec.mask_id,
                               spec.vocab, 3)
    x = di.bf16_bits(case.logits)
    loss_o, unit_o, tr = oracle.loss_absorbing(lay_o, x, spec.vocab, case.clean.cpu().numpy(), corr_o, p_o,
                                               oracle.ALIGNED)
    assert_loss_close(float(out.loss.item()), loss_o)
    assert_grad_close(gpu_bf16_to_f64(out.dlogits), oracle.term_grad(x, spec.vocab, tr, np.arange(128), g))


@pytest.mark.parametrize("align", [oracle.ALIGNED, oracle.SHIFTED])
def test_dense_sequences_with_padding(align):
    """Dense [B, L] layout with trailing pads: N counts the non-pad tokens,
    pads are never corrupted or scored."""
    B, L = 3, 200
    spec = di.WORKLOADS["abs_b1_l4096_v126464"].scaled(vocab=16384, mask_id=16383, ids_high=16000,
                                                       n_units=B, seq_len=L, spike=0.0)
    case = di.make_case(spec, "cuda")
    dev = torch.device("cuda")
    pad = np.zeros(B * L, np.uint8)
    for b, n in enumerate((200, 150, 37)):
        pad[b * L + n:(b + 1) * L] = 1
    pad_d = torch.from_numpy(pad).to(dev)
    lay = dlm.make_layout(B, L, None, pad_d)
    t, p = dlm.sample_t(8, B)
    _, corr = dlm.corrupt(lay, case.clean, p, oracle.ABSORBING, spec.mask_id, spec.vocab, 8)
    out = dlm.loss_fwd_bwd(lay, case.logits, spec.vocab, case.clean, corr, p, oracle.ABSORBING, align)
    torch.cuda.synchronize()
    assert out.device_status() == 0
    lay_o = oracle.Layout(B, L, None, pad)
    _, p_o = oracle.sample_t(8, B, oracle.ABSORBING, 1e-3)
    _, corr_o = oracle.corrupt(lay_o, case.clean.cpu().numpy(), p_o, oracle.ABSORBING, spec.mask_id,
                               spec.vocab, 8)
    assert np.array_equal(corr.cpu().numpy(), corr_o)
    x = di.bf16_bits(case.logits)
    loss_o, unit_o, tr = oracle.loss_absorbing(lay_o, x, spec.vocab, case.clean.cpu().numpy(), corr_o, p_o, align)
    assert_loss_close(float(out.loss.item()), loss_o)
    assert_units_close(out.unit_loss.cpu().numpy()[:B], unit_o, loss_o)
    assert_grad_close(gpu_bf16_to_f64(out.dlogits), oracle.term_grad(x, spec.vocab, tr, np.arange(B * L), 1.0))


def test_linear_bad_target_is_flagged_and_skipped():
    spec = di.WORKLOADS["lin_t16384_d4096_v126464"].scaled(n_tokens_packed=256, d_model=128, vocab=2048,
                                                           ids_high=2000, mask_id=2047)
    case = di.make_case(spec, "cuda")
    dev = torch.device("cuda")
    clean = case.clean.clone()
    clean[7] = 5000                       # outside [0, V)
    lay = dlm.make_layout(case.n_units, 0, case.cu_seqlens, None, n_tokens=256)
    corr = torch.ones(256, dtype=torch.uint8, device=dev)
    p = torch.ones(case.n_units, dtype=torch.float32, device=dev)
    out = dlm.linear_loss_fwd_bwd(lay, case.hidden, case.weight, clean, corr, p)
    assert out.device_status() & dlm.DEV_BAD_TOKEN_ID
    assert bool((out.d_hidden[7] == 0).all())
    assert bool((out.d_hidden[8] != 0).any())
