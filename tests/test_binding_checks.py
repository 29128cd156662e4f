"""Argument checks of the Python binding (no GPU needed).

The C ABI receives bare pointers, so it cannot see that a buffer is shorter
than the layout says; the binding checks every tensor's dtype, then its size,
then its device, before any pointer reaches the library.  These tests pass CPU
tensors: a tensor of the wrong size must be refused for its size (before the
device check), one of the right size only for being on the CPU.
"""
import pytest
import torch

import diffusion_lm_loss_b200 as dlm

bf16 = torch.bfloat16


def _cpu_only(fn):
    with pytest.raises(ValueError, match="must be a CUDA tensor"):
        fn()


def test_make_layout_sizes():
    with pytest.raises(ValueError, match="cu_seqlens: needs at least 4"):
        dlm.make_layout(3, 0, torch.zeros(3, dtype=torch.int32), n_tokens=10)
    with pytest.raises(ValueError, match="pad_mask: needs at least 20"):
        dlm.make_layout(2, 10, None, torch.zeros(19, dtype=torch.uint8))
    with pytest.raises(TypeError, match="pad_mask"):
        dlm.make_layout(2, 10, None, torch.zeros(20, dtype=torch.bool))
    with pytest.raises(ValueError, match="non-negative"):
        dlm.make_layout(-1, 10)
    _cpu_only(lambda: dlm.make_layout(2, 10, None, torch.zeros(20, dtype=torch.uint8)))


def test_corrupt_sizes():
    lay = dlm.make_layout(2, 8)
    with pytest.raises(ValueError, match="clean_ids: needs at least 16"):
        dlm.corrupt(lay, torch.zeros(15, dtype=torch.int32), torch.zeros(2))
    with pytest.raises(ValueError, match="p: needs at least 2"):
        dlm.corrupt(lay, torch.zeros(16, dtype=torch.int32), torch.zeros(1))
    _cpu_only(lambda: dlm.corrupt(lay, torch.zeros(16, dtype=torch.int32), torch.zeros(2)))


def test_loss_sizes_and_dtypes():
    lay = dlm.make_layout(2, 8)
    V = 100
    logits = torch.zeros(16, V, dtype=bf16)
    ids = torch.zeros(16, dtype=torch.int32)
    corr = torch.zeros(16, dtype=torch.uint8)
    p = torch.zeros(2)
    with pytest.raises(ValueError, match="logits: needs at least 16 rows"):
        dlm.loss_fwd_bwd(lay, logits[:15], V, ids, corr, p)
    with pytest.raises(ValueError, match="logits: needs at least 101 columns"):
        dlm.loss_fwd_bwd(lay, logits, V + 1, ids, corr, p)
    with pytest.raises(ValueError, match="unit column stride"):
        dlm.loss_fwd_bwd(lay, torch.zeros(V, 16, dtype=bf16).t(), V, ids, corr, p)
    with pytest.raises(ValueError, match="clean_ids: needs at least 16"):
        dlm.loss_fwd_bwd(lay, logits, V, ids[:8], corr, p)
    with pytest.raises(ValueError, match="corrupted: required"):
        dlm.loss_fwd_bwd(lay, logits, V, ids, None, p)       # absorbing noise needs the mask
    with pytest.raises(TypeError, match="corrupted"):
        dlm.loss_fwd_bwd(lay, logits, V, ids, corr.bool(), p)
    with pytest.raises(TypeError, match="p: expected torch.float32"):
        dlm.loss_fwd_bwd(lay, logits, V, ids, corr, p.double())
    with pytest.raises(ValueError, match="enc_logits needs enc_layout"):
        dlm.loss_fwd_bwd(lay, logits, V, ids, corr, p, dlm.UNIFORM, enc_logits=logits, enc_ids=ids)
    enc = dlm.make_layout(2, 12)
    with pytest.raises(ValueError, match="enc_logits: needs at least 24 rows"):
        dlm.loss_fwd_bwd(lay, logits, V, ids, corr, p, dlm.UNIFORM, enc_layout=enc, enc_logits=logits,
                         enc_ids=torch.zeros(24, dtype=torch.int32))
    with pytest.raises(ValueError, match="enc_ids: needs at least 24"):
        dlm.loss_fwd_bwd(lay, logits, V, ids, corr, p, dlm.UNIFORM, enc_layout=enc,
                         enc_logits=torch.zeros(24, V, dtype=bf16), enc_ids=ids)
    # uniform noise needs neither the mask nor p
    _cpu_only(lambda: dlm.loss_fwd_bwd(lay, logits, V, ids, None, None, dlm.UNIFORM))
    _cpu_only(lambda: dlm.loss_fwd_bwd(lay, logits, V, ids, corr, p))


def test_gradient_buffer_keeps_the_row_stride():
    """A gradient is written with its input's row stride: for logits that are
    a column slice of a wider buffer, the allocated gradient must have the
    same strides (a contiguous copy of the shape would be overrun)."""
    base = torch.zeros(4, 10, dtype=bf16)
    view = base[:, :7]
    g = dlm._like_rows(view)
    assert g.shape == view.shape and g.stride() == (10, 1)
    assert torch.empty_like(view).stride() == (7, 1)       # what a plain copy of the shape gives
    z = dlm._like_rows(view, zero=True)
    assert bool((z == 0).all())
    # a caller-supplied buffer of the right shape but another row stride is refused
    with pytest.raises(ValueError, match="row stride 10"):
        dlm._check_grad(torch.zeros(4, 7, dtype=bf16), view, "out.dlogits")
    with pytest.raises(ValueError, match="shape"):
        dlm._check_grad(torch.zeros(3, 10, dtype=bf16)[:, :7], view, "out.dlogits")


def test_reused_outputs_are_checked():
    lay = dlm.make_layout(2, 8)
    V = 64
    logits = torch.zeros(16, V, dtype=bf16)
    ids = torch.zeros(16, dtype=torch.int32)
    corr = torch.zeros(16, dtype=torch.uint8)
    p = torch.zeros(2)
    ws = torch.zeros(1024, dtype=torch.uint8)
    bad = dlm.LossOut(torch.zeros(1), torch.zeros(1), torch.zeros(16, V, dtype=bf16), None, ws)
    with pytest.raises(ValueError, match="out.unit_loss: needs at least 2"):
        dlm.loss_fwd_bwd(lay, logits, V, ids, corr, p, out=bad)
    bad = dlm.LossOut(torch.zeros(1), torch.zeros(2), torch.zeros(8, V, dtype=bf16), None, ws)
    with pytest.raises(ValueError, match="out.dlogits"):
        dlm.loss_fwd_bwd(lay, logits, V, ids, corr, p, out=bad)


def test_linear_sizes():
    lay = dlm.make_layout(2, 8)
    H = torch.zeros(16, 64, dtype=bf16)
    W = torch.zeros(128, 64, dtype=bf16)
    ids = torch.zeros(16, dtype=torch.int32)
    corr = torch.zeros(16, dtype=torch.uint8)
    p = torch.zeros(2)
    with pytest.raises(ValueError, match="hidden: needs at least 16 rows"):
        dlm.linear_loss_fwd_bwd(lay, H[:12], W, ids, corr, p)
    with pytest.raises(ValueError, match="share d_model"):
        dlm.linear_loss_fwd_bwd(lay, H, torch.zeros(128, 32, dtype=bf16), ids, corr, p)
    with pytest.raises(ValueError, match="must be contiguous"):
        dlm.linear_loss_fwd_bwd(lay, torch.zeros(64, 16, dtype=bf16).t(), W, ids, corr, p)
    with pytest.raises(ValueError, match="corrupted: needs at least 16"):
        dlm.linear_loss_fwd_bwd(lay, H, W, ids, corr[:3], p)
    _cpu_only(lambda: dlm.linear_loss_fwd_bwd(lay, H, W, ids, corr, p))
    enc = dlm.make_layout(2, 12)
    with pytest.raises(ValueError, match="enc_hidden: required"):
        dlm.linear_loss_uniform_fwd_bwd(lay, H, W, ids, enc, None, torch.zeros(24, dtype=torch.int32))
    with pytest.raises(ValueError, match="enc_hidden: needs at least 1536"):
        dlm.linear_loss_uniform_fwd_bwd(lay, H, W, ids, enc, torch.zeros(20, 64, dtype=bf16),
                                        torch.zeros(24, dtype=torch.int32))
    with pytest.raises(ValueError, match="enc_ids: needs at least 24"):
        dlm.linear_loss_uniform_fwd_bwd(lay, H, W, ids, enc, torch.zeros(24, 64, dtype=bf16),
                                        torch.zeros(20, dtype=torch.int32))
    _cpu_only(lambda: dlm.linear_loss_uniform_fwd_bwd(lay, H, W, ids, enc, torch.zeros(24, 64, dtype=bf16),
                                                      torch.zeros(24, dtype=torch.int32)))


def test_fused_head_workspace_is_1024_byte_aligned():
    for n in (1, 1000, 4096, 123457):
        ws = dlm._aligned_workspace(n, "cpu")
        assert ws.numel() == n and ws.dtype == torch.uint8 and ws.is_contiguous()
        assert ws.data_ptr() % 1024 == 0


# --------------------------------------------------------------------------
# valid calls get past every host-side check: the binding's (device check
# stubbed out) and the library's, and stop only at the library's own check
# for a B200, which fails here without a device
# --------------------------------------------------------------------------
@pytest.fixture
def host_only(monkeypatch):
    from diffusion_lm_loss_b200 import build as dlm_build
    dlm_build.build()
    monkeypatch.setattr(dlm, "_on_cuda", lambda **kw: None)
    monkeypatch.setattr(dlm, "_stream", lambda: None)


def _stops_at_device_check(fn):
    with pytest.raises(dlm.DlmError) as e:
        fn()
    assert e.value.code in (2, 4), e.value      # DLM_ERR_UNSUPPORTED / DLM_ERR_CUDA, nothing earlier


def test_valid_loss_calls_pass_host_checks(host_only):
    V = 1000
    lay = dlm.make_layout(2, 24)
    logits = torch.zeros(48, V, dtype=bf16)
    ids = torch.zeros(48, dtype=torch.int32)
    corr = torch.zeros(48, dtype=torch.uint8)
    p = torch.full((2,), 0.5)
    _stops_at_device_check(lambda: dlm.corrupt(lay, ids, p, dlm.ABSORBING, V - 1, V, 0))
    _stops_at_device_check(lambda: dlm.loss_fwd_bwd(lay, logits, V, ids, corr, p))
    # padded row stride: logits a column slice of a wider buffer, own gradient buffer reused
    wide = torch.zeros(48, 1010, dtype=bf16)
    out = dlm.LossOut(torch.zeros(1), torch.zeros(2), dlm._like_rows(wide[:, :V]), None,
                      dlm._aligned_workspace(dlm.loss_workspace_size(lay), "cpu", 256))
    _stops_at_device_check(lambda: dlm.loss_fwd_bwd(lay, wide[:, :V], V, ids, corr, p, out=out))
    # uniform noise with the encoder term and the objective options
    enc = dlm.make_layout(2, 32)
    kw = dict(enc_layout=enc, enc_logits=torch.zeros(64, V, dtype=bf16),
              enc_ids=torch.zeros(64, dtype=torch.int32), enc_ar_weight=1.0)
    _stops_at_device_check(lambda: dlm.loss_fwd_bwd(lay, logits, V, ids, None, None, dlm.UNIFORM, **kw))
    opts = dlm.LossOptions(dlm.TIME_WEIGHT_INV_ONE_MINUS_T, 10.0, dlm.REDUCE_EXAMPLE_MEAN)
    _stops_at_device_check(lambda: dlm.loss_fwd_bwd(lay, logits, V, ids, corr, p, dlm.UNIFORM, options=opts,
                                                    **kw))
    # empty input
    empty = dlm.make_layout(2, 0)
    _stops_at_device_check(lambda: dlm.loss_fwd_bwd(empty, torch.zeros(0, 4096, dtype=bf16), 4096,
                                                    torch.zeros(0, dtype=torch.int32),
                                                    torch.zeros(0, dtype=torch.uint8), p))


def test_valid_fused_head_calls_pass_host_checks(host_only):
    D, V = 64, 1024
    lay = dlm.make_layout(2, 24)
    H = torch.zeros(48, D, dtype=bf16)
    W = torch.zeros(V, D, dtype=bf16)
    ids = torch.zeros(48, dtype=torch.int32)
    corr = torch.zeros(48, dtype=torch.uint8)
    p = torch.full((2,), 0.5)
    for align in (dlm.ALIGNED, dlm.SHIFTED):
        _stops_at_device_check(lambda: dlm.linear_loss_fwd_bwd(lay, H, W, ids, corr, p, align=align))
    _stops_at_device_check(lambda: dlm.linear_loss_fwd_bwd(lay, H, W, ids, corr, p, want_d_weight=False))
    enc = dlm.make_layout(2, 40)
    He = torch.zeros(80, D, dtype=bf16)
    eids = torch.zeros(80, dtype=torch.int32)
    _stops_at_device_check(lambda: dlm.linear_loss_uniform_fwd_bwd(lay, H, W, ids, enc, He, eids, 0.5))
    _stops_at_device_check(lambda: dlm.linear_loss_uniform_fwd_bwd(lay, H, W, ids, align=dlm.SHIFTED,
                                                                   want_d_weight=False))
