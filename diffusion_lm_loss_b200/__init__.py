"""Python binding of the B200 diffusion-LM noising-plus-loss library.

Argument marshalling only: every step runs in the CUDA kernels of
``libdlm.so`` (built from ``csrc/`` for sm_100a); torch provides device
memory and streams.  There is no CPU fallback -- importing this module
without the built library, or calling it on a non-sm_100 device, raises.

Two layers:
  * ``lib()``: the raw C ABI through ctypes, functions named as in
    ``include/dlm.h`` (``dlm_sample_t``, ``dlm_corrupt``,
    ``dlm_loss_fwd_bwd``, ``dlm_linear_loss_fwd_bwd``, ...);
  * tensor helpers with the same names minus the prefix (``sample_t``,
    ``corrupt``, ``loss_fwd_bwd``, ``linear_loss_fwd_bwd``,
    ``linear_loss_uniform_fwd_bwd``, ``decision_loss_fwd_bwd``) that check every tensor argument's
    dtype, size against the layout and device, allocate outputs and
    workspace with torch on the current device and call the ABI on the
    current torch stream;
  * ``torch.autograd.Function`` wrappers of the four losses
    (``diffusion_loss``, ``linear_diffusion_loss``,
    ``linear_uniform_loss``, ``decision_loss``): the forward runs the fused
    forward + backward call and keeps its gradients; the backward hands them
    over, multiplied by the upstream gradient in the library
    (``dlm_scale_bf16``, which does nothing when that gradient is 1).
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libdlm.so")

ABSORBING, UNIFORM = 0, 1
ALIGNED, SHIFTED = 0, 1
TIME_WEIGHT_NONE, TIME_WEIGHT_INV_ONE_MINUS_T = 0, 1
REDUCE_TOKEN_MEAN, REDUCE_EXAMPLE_MEAN = 0, 1

DEV_BAD_TOKEN_ID = 0x1
DEV_BAD_LAYOUT = 0x2
DEV_WAIT_TIMEOUT = 0x4
DEV_BAD_LABEL = 0x8

LABEL_HARD, LABEL_DIST, LABEL_SET = 0, 1, 2
LABEL_SOFTMAX_RESTRICTED, LABEL_SOFTMAX_FULL, LABEL_SOFTMAX_BOTH = 1, 2, 3
DECISION_MAX_ANSWERS = 128
DECISION_MAX_SLOTS = 65535

STATUS = {0: "DLM_OK", 1: "DLM_ERR_INVALID_ARGUMENT", 2: "DLM_ERR_UNSUPPORTED",
          3: "DLM_ERR_WORKSPACE_TOO_SMALL", 4: "DLM_ERR_CUDA"}

# every symbol include/dlm.h declares
EXPORTS = ("dlm_status_string", "dlm_last_cuda_error", "dlm_version", "dlm_sample_t", "dlm_corrupt",
           "dlm_loss_workspace_size", "dlm_loss_fwd_bwd", "dlm_loss_fwd_bwd_ex", "dlm_loss_fwd_bwd_static",
           "dlm_linear_loss_workspace_size",
           "dlm_linear_loss_fwd_bwd", "dlm_linear_loss_fwd_bwd_ex", "dlm_linear_loss_uniform_workspace_size",
           "dlm_linear_loss_uniform_fwd_bwd", "dlm_decision_workspace_size", "dlm_decision_loss_fwd_bwd",
           "dlm_scale_bf16", "dlm_get_device_status", "dlm_selftest_bounded_wait",
           "dlm_test_skip_device_check")


class DlmError(RuntimeError):
    def __init__(self, code: int, where: str, detail: str = ""):
        super().__init__(f"{where}: {STATUS.get(code, code)}" + (f" [{detail}]" if detail else ""))
        self.code = code


class LossOptions(ctypes.Structure):
    """dlm_loss_options_t: uniform-noise objective options."""
    _fields_ = [("struct_size", ctypes.c_uint32), ("time_weighting", ctypes.c_int32),
                ("weight_clip", ctypes.c_float), ("reduction", ctypes.c_int32),
                ("keep_unscored_rows", ctypes.c_int32)]

    def __init__(self, time_weighting=TIME_WEIGHT_NONE, weight_clip=0.0, reduction=REDUCE_TOKEN_MEAN,
                 keep_unscored_rows=0):
        super().__init__(ctypes.sizeof(LossOptions), time_weighting, weight_clip, reduction,
                         keep_unscored_rows)


class Layout(ctypes.Structure):
    """dlm_layout_t: n_units sequences of seq_len tokens (cu_seqlens NULL) or
    n_units packed documents (cu_seqlens [n_units+1] int32 on the device);
    pad_mask [n_tokens] uint8 on the device (1 = pad) or NULL."""
    _fields_ = [("n_units", ctypes.c_int32), ("seq_len", ctypes.c_int32),
                ("n_tokens", ctypes.c_int64), ("cu_seqlens", ctypes.c_void_p),
                ("pad_mask", ctypes.c_void_p)]


def make_layout(n_units: int, seq_len: int = 0, cu_seqlens: Optional[torch.Tensor] = None,
                pad_mask: Optional[torch.Tensor] = None, n_tokens: Optional[int] = None) -> Layout:
    """A dlm_layout_t over device tensors.  The layout holds references to
    cu_seqlens and pad_mask, whose device pointers it carries, so they stay
    allocated as long as the layout is in use."""
    if n_units < 0 or seq_len < 0 or (n_tokens is not None and n_tokens < 0):
        raise ValueError("n_units, seq_len and n_tokens must be non-negative")
    if cu_seqlens is not None:
        _check(cu_seqlens, torch.int32, "cu_seqlens", min_numel=n_units + 1)
        if n_tokens is None:
            raise ValueError("packed layouts need n_tokens (cu_seqlens lives on the device)")
        cu = cu_seqlens.data_ptr()
    else:
        cu = None
        n_tokens = n_units * seq_len if n_tokens is None else n_tokens
    pm = None
    if pad_mask is not None:
        _check(pad_mask, torch.uint8, "pad_mask", min_numel=n_tokens)
        pm = pad_mask.data_ptr()
    _on_cuda(cu_seqlens=cu_seqlens, pad_mask=pad_mask)
    lay = Layout(n_units, seq_len, n_tokens, cu, pm)
    lay._tensors = (cu_seqlens, pad_mask)
    return lay


_lib = None


def lib():
    """The loaded C ABI (ctypes), with argument and return types declared."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is not built: run python -m diffusion_lm_loss_b200.build "
                          "(there is no CPU fallback)")
    L = ctypes.CDLL(LIB_PATH)
    vp, i32, i64, u64, f32, sz = (ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_uint64,
                                  ctypes.c_float, ctypes.c_size_t)
    lp = ctypes.POINTER(Layout)
    L.dlm_status_string.restype = ctypes.c_char_p
    L.dlm_status_string.argtypes = [ctypes.c_int]
    L.dlm_last_cuda_error.restype = ctypes.c_char_p
    L.dlm_last_cuda_error.argtypes = []
    L.dlm_version.restype = ctypes.c_int
    L.dlm_version.argtypes = []
    L.dlm_sample_t.restype = ctypes.c_int
    L.dlm_sample_t.argtypes = [u64, i32, i32, f32, vp, vp, vp]
    L.dlm_corrupt.restype = ctypes.c_int
    L.dlm_corrupt.argtypes = [lp, vp, vp, i32, i32, i32, u64, vp, vp, vp, vp]
    L.dlm_loss_workspace_size.restype = sz
    L.dlm_loss_workspace_size.argtypes = [lp, lp]
    L.dlm_loss_fwd_bwd.restype = ctypes.c_int
    L.dlm_loss_fwd_bwd.argtypes = [lp, vp, i64, i32, vp, vp, vp, i32, i32, lp, vp, i64, vp, f32,
                                   f32, vp, vp, vp, vp, vp, sz, vp]
    L.dlm_loss_fwd_bwd_ex.restype = ctypes.c_int
    L.dlm_loss_fwd_bwd_ex.argtypes = [lp, vp, i64, i32, vp, vp, vp, i32, i32, lp, vp, i64, vp, f32,
                                      f32, ctypes.POINTER(LossOptions), vp, vp, vp, vp, vp, sz, vp]
    L.dlm_loss_fwd_bwd_static.restype = ctypes.c_int
    L.dlm_loss_fwd_bwd_static.argtypes = [lp, vp, i64, i32, vp, vp, vp, i32, i32, lp, vp, i64, vp, f32,
                                          f32, vp, vp, vp, vp, vp]
    L.dlm_linear_loss_workspace_size.restype = sz
    L.dlm_linear_loss_workspace_size.argtypes = [lp, i32, i32]
    L.dlm_linear_loss_fwd_bwd.restype = ctypes.c_int
    L.dlm_linear_loss_fwd_bwd.argtypes = [lp, vp, vp, i32, i32, vp, vp, vp, f32, vp, vp, vp, vp,
                                          vp, sz, vp]
    L.dlm_linear_loss_fwd_bwd_ex.restype = ctypes.c_int
    L.dlm_linear_loss_fwd_bwd_ex.argtypes = [lp, vp, vp, i32, i32, vp, vp, vp, i32, f32, vp, vp, vp, vp,
                                             vp, sz, vp]
    L.dlm_linear_loss_uniform_workspace_size.restype = sz
    L.dlm_linear_loss_uniform_workspace_size.argtypes = [lp, lp, i32, i32]
    L.dlm_linear_loss_uniform_fwd_bwd.restype = ctypes.c_int
    L.dlm_linear_loss_uniform_fwd_bwd.argtypes = [lp, vp, lp, vp, vp, vp, i32, i32, vp, i32, f32, f32,
                                                  vp, vp, vp, vp, vp, vp, sz, vp]
    L.dlm_decision_workspace_size.restype = sz
    L.dlm_decision_workspace_size.argtypes = [i32, i32]
    L.dlm_decision_loss_fwd_bwd.restype = ctypes.c_int
    L.dlm_decision_loss_fwd_bwd.argtypes = [i32, vp, i64, i64, i32, vp, vp, i64, vp, vp, vp, i32, f32, f32, f32, vp,
                                            vp, vp, i64, vp, sz, vp]
    L.dlm_scale_bf16.restype = ctypes.c_int
    L.dlm_scale_bf16.argtypes = [vp, i64, i64, i64, vp, vp]
    L.dlm_test_skip_device_check.restype = ctypes.c_int
    L.dlm_test_skip_device_check.argtypes = [i32]
    L.dlm_selftest_bounded_wait.restype = ctypes.c_int
    L.dlm_selftest_bounded_wait.argtypes = [u64, vp, vp]
    L.dlm_get_device_status.restype = ctypes.c_int
    L.dlm_get_device_status.argtypes = [vp, ctypes.POINTER(ctypes.c_uint32), vp]
    _lib = L
    return L


def _check(t: Optional[torch.Tensor], dtype, name: str, min_numel: Optional[int] = None,
           min_rows: Optional[int] = None, min_cols: Optional[int] = None):
    """A tensor argument before its pointer goes to the library: dtype and
    size (the C ABI sees only pointers, so a buffer shorter than the layout
    says would be read or written out of bounds on the device).  The device
    is checked afterwards, for all arguments of a call together (_on_cuda).
    min_numel: a contiguous buffer of at least that many elements; min_rows /
    min_cols: a 2-D tensor with unit column stride and at least that many rows
    / columns."""
    if t is None:
        raise ValueError(f"{name}: required")
    if t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if min_numel is not None:
        if not t.is_contiguous():
            raise ValueError(f"{name}: must be contiguous")
        if t.numel() < min_numel:
            raise ValueError(f"{name}: needs at least {min_numel} elements, has {t.numel()}")
    if min_rows is not None or min_cols is not None:
        if t.dim() != 2 or (t.shape[1] > 1 and t.stride(1) != 1):
            raise ValueError(f"{name}: must be 2-D with unit column stride, got shape {tuple(t.shape)}")
        if min_rows is not None and t.shape[0] < min_rows:
            raise ValueError(f"{name}: needs at least {min_rows} rows, has {t.shape[0]}")
        if min_cols is not None and t.shape[1] < min_cols:
            raise ValueError(f"{name}: needs at least {min_cols} columns, has {t.shape[1]}")


def _on_cuda(**tensors):
    """Every tensor argument of a call (None = not given) on one CUDA device."""
    dev = None
    for name, t in tensors.items():
        if t is None:
            continue
        if not t.is_cuda:
            raise ValueError(f"{name}: must be a CUDA tensor (there is no CPU path)")
        if dev is None:
            dev = t.device
        elif t.device != dev:
            raise ValueError(f"{name}: on {t.device}, the other arguments on {dev}")


def _like_rows(t: torch.Tensor, zero: bool = False) -> torch.Tensor:
    """A buffer with t's shape and strides (a gradient is written with the
    row stride of its input, which may be wider than the row)."""
    out = torch.empty_strided(t.shape, t.stride(), dtype=t.dtype, device=t.device)
    return out.zero_() if zero else out


def _check_grad(g: Optional[torch.Tensor], like: torch.Tensor, name: str):
    """A caller-supplied gradient buffer: same dtype, shape and row stride as
    the input it is the gradient of."""
    _check(g, like.dtype, name)
    if tuple(g.shape) != tuple(like.shape) or (like.dim() == 2 and g.stride(0) != like.stride(0)):
        raise ValueError(f"{name}: must have the shape {tuple(like.shape)} and row stride "
                         f"{like.stride(0)} of its input")


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else t.data_ptr()


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _ok(code: int, where: str):
    if code != 0:
        detail = lib().dlm_last_cuda_error().decode() if code == 4 else ""
        raise DlmError(code, where, detail)


def _check_out(loss: torch.Tensor, unit_loss: Optional[torch.Tensor], layout: Layout,
               workspace: torch.Tensor):
    """The scalar outputs and the workspace of a reused result object (the
    library itself checks the workspace's size against the call)."""
    _check(loss, torch.float32, "out.loss", min_numel=1)
    if unit_loss is not None:
        _check(unit_loss, torch.float32, "out.unit_loss", min_numel=layout.n_units)
    _check(workspace, torch.uint8, "out.workspace", min_numel=0)


def _bits(t: torch.Tensor) -> torch.Tensor:
    return t.view(torch.int16) if t.dtype == torch.bfloat16 else t


# --------------------------------------------------------------------------
# tensor helpers
# --------------------------------------------------------------------------
def sample_t(seed: int, n_units: int, mode: int = ABSORBING, eps: float = 1e-3,
             device=None):
    """(t, p): float32 [n_units] on the current (or given) CUDA device."""
    dev = torch.device("cuda") if device is None else torch.device(device)
    t = torch.empty(n_units, dtype=torch.float32, device=dev)
    p = torch.empty(n_units, dtype=torch.float32, device=dev)
    _ok(lib().dlm_sample_t(seed, n_units, mode, eps, _ptr(t), _ptr(p), _stream()), "dlm_sample_t")
    return t, p


def corrupt(layout: Layout, clean_ids: torch.Tensor, p: torch.Tensor, mode: int = ABSORBING,
            mask_id: int = 0, vocab: int = 0, seed: int = 0,
            dev_status: Optional[torch.Tensor] = None):
    """(noisy int32, corrupted uint8), same length as clean_ids."""
    _check(clean_ids, torch.int32, "clean_ids", min_numel=layout.n_tokens)
    _check(p, torch.float32, "p", min_numel=layout.n_units)
    if dev_status is not None and (dev_status.dtype not in (torch.int32, torch.uint32) or dev_status.numel() < 1):
        raise ValueError("dev_status: an int32 / uint32 tensor of at least one element")
    _on_cuda(clean_ids=clean_ids, p=p, dev_status=dev_status)
    noisy = torch.empty_like(clean_ids)
    corr = torch.empty(clean_ids.shape, dtype=torch.uint8, device=clean_ids.device)
    _ok(lib().dlm_corrupt(ctypes.byref(layout), _ptr(clean_ids), _ptr(p), mode, mask_id, vocab, seed,
                          _ptr(noisy), _ptr(corr), _ptr(dev_status), _stream()), "dlm_corrupt")
    return noisy, corr


@dataclass
class LossOut:
    loss: torch.Tensor            # float32 [1]
    unit_loss: torch.Tensor       # float32 [n_units]
    dlogits: torch.Tensor         # bf16, logits' shape
    enc_dlogits: Optional[torch.Tensor]
    workspace: torch.Tensor       # uint8; holds the device status word

    def device_status(self) -> int:
        return device_status(self.workspace)


def loss_workspace_size(layout: Layout, enc_layout: Optional[Layout] = None) -> int:
    return int(lib().dlm_loss_workspace_size(ctypes.byref(layout),
                                             ctypes.byref(enc_layout) if enc_layout else None))


def loss_fwd_bwd(layout: Layout, logits: torch.Tensor, vocab: int, clean_ids: torch.Tensor,
                 corrupted: Optional[torch.Tensor], p: Optional[torch.Tensor],
                 mode: int = ABSORBING, align: int = ALIGNED,
                 enc_layout: Optional[Layout] = None, enc_logits: Optional[torch.Tensor] = None,
                 enc_ids: Optional[torch.Tensor] = None, enc_ar_weight: float = 1.0,
                 grad_scale: float = 1.0, out: Optional[LossOut] = None,
                 options: Optional[LossOptions] = None) -> LossOut:
    """Weighted CE forward + backward (see dlm_loss_fwd_bwd).  logits: bf16
    [rows, ld] (2-D, row stride ld >= vocab).  Reuses the buffers of `out`
    when given (no allocation)."""
    T = layout.n_tokens
    _check(logits, torch.bfloat16, "logits", min_rows=T, min_cols=vocab)
    _check(clean_ids, torch.int32, "clean_ids", min_numel=T)
    if corrupted is not None or (mode == ABSORBING and T > 0):
        _check(corrupted, torch.uint8, "corrupted", min_numel=T)
    if p is not None:
        _check(p, torch.float32, "p", min_numel=layout.n_units)
    ld = logits.stride(0)
    enc_ld = 0
    if enc_logits is not None:
        if enc_layout is None:
            raise ValueError("enc_logits needs enc_layout")
        _check(enc_logits, torch.bfloat16, "enc_logits", min_rows=enc_layout.n_tokens, min_cols=vocab)
        _check(enc_ids, torch.int32, "enc_ids", min_numel=enc_layout.n_tokens)
        enc_ld = enc_logits.stride(0)
    if out is not None:
        _check_out(out.loss, out.unit_loss, layout, out.workspace)
        _check_grad(out.dlogits, logits, "out.dlogits")
        if enc_logits is not None:
            _check_grad(out.enc_dlogits, enc_logits, "out.enc_dlogits")
    o = out if out is not None else LossOut(None, None, None, None, None)
    _on_cuda(logits=logits, clean_ids=clean_ids, corrupted=corrupted, p=p, enc_logits=enc_logits,
             enc_ids=enc_ids, loss=o.loss, unit_loss=o.unit_loss, workspace=o.workspace, dlogits=o.dlogits,
             enc_dlogits=o.enc_dlogits if enc_logits is not None else None)
    dev = logits.device
    keep = options is not None and options.keep_unscored_rows
    if out is None:
        ws = _aligned_workspace(loss_workspace_size(layout, enc_layout), dev, 256)
        # rows the call leaves untouched must start as zeros
        out = LossOut(torch.empty(1, dtype=torch.float32, device=dev),
                      torch.empty(max(layout.n_units, 1), dtype=torch.float32, device=dev),
                      _like_rows(logits, keep),
                      _like_rows(enc_logits, keep) if enc_logits is not None else None, ws)
    if options is None:
        _ok(lib().dlm_loss_fwd_bwd(
            ctypes.byref(layout), _ptr(logits), ld, vocab, _ptr(clean_ids), _ptr(corrupted), _ptr(p),
            mode, align, ctypes.byref(enc_layout) if enc_layout is not None else None,
            _ptr(enc_logits), enc_ld, _ptr(enc_ids), enc_ar_weight, grad_scale, _ptr(out.loss),
            _ptr(out.unit_loss), _ptr(out.dlogits), _ptr(out.enc_dlogits), _ptr(out.workspace),
            out.workspace.numel(), _stream()), "dlm_loss_fwd_bwd")
    else:
        _ok(lib().dlm_loss_fwd_bwd_ex(
            ctypes.byref(layout), _ptr(logits), ld, vocab, _ptr(clean_ids), _ptr(corrupted), _ptr(p),
            mode, align, ctypes.byref(enc_layout) if enc_layout is not None else None,
            _ptr(enc_logits), enc_ld, _ptr(enc_ids), enc_ar_weight, grad_scale, ctypes.byref(options),
            _ptr(out.loss), _ptr(out.unit_loss), _ptr(out.dlogits), _ptr(out.enc_dlogits),
            _ptr(out.workspace), out.workspace.numel(), _stream()), "dlm_loss_fwd_bwd_ex")
    return out


@dataclass
class LinearOut:
    loss: torch.Tensor
    unit_loss: torch.Tensor
    d_hidden: torch.Tensor
    d_weight: Optional[torch.Tensor]
    workspace: torch.Tensor
    d_enc_hidden: Optional[torch.Tensor] = None

    def device_status(self) -> int:
        return device_status(self.workspace)


def _aligned_workspace(nbytes: int, device, align: int = 1024) -> torch.Tensor:
    """A uint8 workspace whose first byte is `align`-byte aligned (the loss
    needs 256, the fused head 1024; the caching allocator guarantees 512 and
    other allocators less): a slice of a slightly larger buffer, which the
    slice keeps alive."""
    buf = torch.empty(nbytes + align - 1, dtype=torch.uint8, device=device)
    off = (-buf.data_ptr()) % align
    return buf[off:off + nbytes]


def _check_head(layout: Layout, hidden: torch.Tensor, weight: torch.Tensor):
    """hidden [n_tokens, D] and weight [V, D], contiguous bf16; returns (T, D, V)."""
    T = layout.n_tokens
    _check(hidden, torch.bfloat16, "hidden", min_numel=0)
    _check(weight, torch.bfloat16, "weight", min_numel=0)
    if hidden.dim() != 2 or weight.dim() != 2 or hidden.shape[1] != weight.shape[1]:
        raise ValueError("hidden [tokens, d_model] and weight [vocab, d_model] must share d_model")
    if hidden.shape[0] < T:
        raise ValueError(f"hidden: needs at least {T} rows, has {hidden.shape[0]}")
    return T, int(hidden.shape[1]), int(weight.shape[0])


def linear_loss_workspace_size(layout: Layout, d_model: int, vocab: int) -> int:
    return int(lib().dlm_linear_loss_workspace_size(ctypes.byref(layout), d_model, vocab))


def linear_loss_fwd_bwd(layout: Layout, hidden: torch.Tensor, weight: torch.Tensor,
                        clean_ids: torch.Tensor, corrupted: torch.Tensor, p: torch.Tensor,
                        grad_scale: float = 1.0, want_d_weight: bool = True,
                        out: Optional[LinearOut] = None, align: int = ALIGNED) -> LinearOut:
    """Fused lm_head + absorbing loss (see dlm_linear_loss_fwd_bwd; align =
    SHIFTED goes through dlm_linear_loss_fwd_bwd_ex)."""
    T, D, V = _check_head(layout, hidden, weight)
    _check(clean_ids, torch.int32, "clean_ids", min_numel=T)
    _check(corrupted, torch.uint8, "corrupted", min_numel=T)
    _check(p, torch.float32, "p", min_numel=layout.n_units)
    if out is not None:
        _check_out(out.loss, out.unit_loss, layout, out.workspace)
        _check_grad(out.d_hidden, hidden, "out.d_hidden")
        if out.d_weight is not None:
            _check_grad(out.d_weight, weight, "out.d_weight")
    o = out if out is not None else LinearOut(None, None, None, None, None)
    _on_cuda(hidden=hidden, weight=weight, clean_ids=clean_ids, corrupted=corrupted, p=p, loss=o.loss,
             unit_loss=o.unit_loss, workspace=o.workspace, d_hidden=o.d_hidden, d_weight=o.d_weight)
    dev = hidden.device
    if out is None:
        ws = _aligned_workspace(linear_loss_workspace_size(layout, D, V), dev)
        out = LinearOut(torch.empty(1, dtype=torch.float32, device=dev),
                        torch.empty(max(layout.n_units, 1), dtype=torch.float32, device=dev),
                        torch.empty_like(hidden),
                        torch.empty_like(weight) if want_d_weight else None, ws)
    if align == ALIGNED:
        _ok(lib().dlm_linear_loss_fwd_bwd(
            ctypes.byref(layout), _ptr(hidden), _ptr(weight), D, V, _ptr(clean_ids), _ptr(corrupted),
            _ptr(p), grad_scale, _ptr(out.loss), _ptr(out.unit_loss), _ptr(out.d_hidden),
            _ptr(out.d_weight), _ptr(out.workspace), out.workspace.numel(), _stream()),
            "dlm_linear_loss_fwd_bwd")
    else:
        _ok(lib().dlm_linear_loss_fwd_bwd_ex(
            ctypes.byref(layout), _ptr(hidden), _ptr(weight), D, V, _ptr(clean_ids), _ptr(corrupted),
            _ptr(p), align, grad_scale, _ptr(out.loss), _ptr(out.unit_loss), _ptr(out.d_hidden),
            _ptr(out.d_weight), _ptr(out.workspace), out.workspace.numel(), _stream()),
            "dlm_linear_loss_fwd_bwd_ex")
    return out


def linear_loss_uniform_workspace_size(layout: Layout, enc_layout: Optional[Layout], d_model: int,
                                       vocab: int) -> int:
    enc = ctypes.byref(enc_layout) if enc_layout is not None else None
    return int(lib().dlm_linear_loss_uniform_workspace_size(ctypes.byref(layout), enc, d_model, vocab))


def linear_loss_uniform_fwd_bwd(layout: Layout, hidden: torch.Tensor, weight: torch.Tensor,
                                clean_ids: torch.Tensor, enc_layout: Optional[Layout] = None,
                                enc_hidden: Optional[torch.Tensor] = None,
                                enc_ids: Optional[torch.Tensor] = None, enc_ar_weight: float = 1.0,
                                align: int = ALIGNED, grad_scale: float = 1.0, want_d_weight: bool = True,
                                out: Optional[LinearOut] = None) -> LinearOut:
    """Fused lm_head + uniform-noise loss with the optional encoder
    next-token term (see dlm_linear_loss_uniform_fwd_bwd)."""
    T, D, V = _check_head(layout, hidden, weight)
    _check(clean_ids, torch.int32, "clean_ids", min_numel=T)
    if enc_layout is not None:
        Te = enc_layout.n_tokens
        _check(enc_hidden, torch.bfloat16, "enc_hidden", min_numel=Te * D)
        if enc_hidden.dim() != 2 or enc_hidden.shape[1] != D:
            raise ValueError("enc_hidden must be [enc_tokens, d_model]")
        _check(enc_ids, torch.int32, "enc_ids", min_numel=Te)
    if out is not None:
        _check_out(out.loss, out.unit_loss, layout, out.workspace)
        _check_grad(out.d_hidden, hidden, "out.d_hidden")
        if out.d_weight is not None:
            _check_grad(out.d_weight, weight, "out.d_weight")
        if enc_layout is not None:
            _check_grad(out.d_enc_hidden, enc_hidden, "out.d_enc_hidden")
    o = out if out is not None else LinearOut(None, None, None, None, None)
    _on_cuda(hidden=hidden, weight=weight, clean_ids=clean_ids, enc_hidden=enc_hidden, enc_ids=enc_ids,
             loss=o.loss, unit_loss=o.unit_loss, workspace=o.workspace, d_hidden=o.d_hidden,
             d_weight=o.d_weight, d_enc_hidden=o.d_enc_hidden if enc_layout is not None else None)
    dev = hidden.device
    if out is None:
        ws = _aligned_workspace(linear_loss_uniform_workspace_size(layout, enc_layout, D, V), dev)
        out = LinearOut(torch.empty(1, dtype=torch.float32, device=dev),
                        torch.empty(max(layout.n_units, 1), dtype=torch.float32, device=dev),
                        torch.empty_like(hidden),
                        torch.empty_like(weight) if want_d_weight else None, ws,
                        torch.empty_like(enc_hidden) if enc_layout is not None else None)
    enc = ctypes.byref(enc_layout) if enc_layout is not None else None
    _ok(lib().dlm_linear_loss_uniform_fwd_bwd(
        ctypes.byref(layout), _ptr(hidden), enc, _ptr(enc_hidden), _ptr(enc_ids), _ptr(weight), D, V,
        _ptr(clean_ids), align, enc_ar_weight, grad_scale, _ptr(out.loss), _ptr(out.unit_loss),
        _ptr(out.d_hidden), _ptr(out.d_enc_hidden), _ptr(out.d_weight), _ptr(out.workspace),
        out.workspace.numel(), _stream()),
        "dlm_linear_loss_uniform_fwd_bwd")
    return out


@dataclass
class DecisionOut:
    loss: torch.Tensor            # float32 [1]
    slot_loss: torch.Tensor       # float32 [n_slots]: each slot's share of the loss
    dlogits: torch.Tensor         # bf16 [n_slots, vocab]: row i = slot i
    workspace: torch.Tensor       # uint8; holds the device status word

    def device_status(self) -> int:
        return device_status(self.workspace)


def decision_workspace_size(n_slots: int, vocab: int) -> int:
    return int(lib().dlm_decision_workspace_size(n_slots, vocab))


def decision_loss_fwd_bwd(logits: torch.Tensor, vocab: int, cand_off: torch.Tensor, cand_ids: torch.Tensor,
                          label_kind: torch.Tensor, label_val: torch.Tensor,
                          slot_rows: Optional[torch.Tensor] = None,
                          label_softmax: int = LABEL_SOFTMAX_BOTH, brier_weight: float = 0.1,
                          hard_label_smoothing: float = 0.0, grad_scale: float = 1.0,
                          out: Optional[DecisionOut] = None) -> DecisionOut:
    """Typed-decision losses at label slots (see dlm_decision_loss_fwd_bwd).
    logits: bf16 [rows, ld]; slot i reads row slot_rows[i] (int64), or row i
    when slot_rows is None.  cand_off int32 [n_slots + 1]; cand_ids int32 and
    label_val float32 of the same length; label_kind int32 [n_slots].  Rows
    and offsets that leave these arrays (device data) are refused by the
    kernels (DEV_BAD_LAYOUT)."""
    n = int(cand_off.numel()) - 1
    if n < 0:
        raise ValueError("cand_off: needs n_slots + 1 entries")
    _check(cand_off, torch.int32, "cand_off", min_numel=n + 1)
    _check(label_kind, torch.int32, "label_kind", min_numel=n)
    _check(cand_ids, torch.int32, "cand_ids", min_numel=0)
    _check(label_val, torch.float32, "label_val", min_numel=cand_ids.numel())
    rows_needed = n
    if slot_rows is not None:
        _check(slot_rows, torch.int64, "slot_rows", min_numel=n)
        rows_needed = 1
    _check(logits, torch.bfloat16, "logits", min_rows=rows_needed if n > 0 else 0, min_cols=vocab)
    if out is not None:
        _check(out.loss, torch.float32, "out.loss", min_numel=1)
        _check(out.slot_loss, torch.float32, "out.slot_loss", min_numel=n)
        _check(out.dlogits, torch.bfloat16, "out.dlogits", min_rows=n, min_cols=vocab)
        _check(out.workspace, torch.uint8, "out.workspace", min_numel=0)
    o = out if out is not None else DecisionOut(None, None, None, None)
    _on_cuda(logits=logits, cand_off=cand_off, cand_ids=cand_ids, label_kind=label_kind, label_val=label_val,
             slot_rows=slot_rows, loss=o.loss, slot_loss=o.slot_loss, dlogits=o.dlogits, workspace=o.workspace)
    dev = logits.device
    if out is None:
        out = DecisionOut(torch.empty(1, dtype=torch.float32, device=dev),
                          torch.empty(max(n, 1), dtype=torch.float32, device=dev),
                          torch.empty((n, vocab), dtype=torch.bfloat16, device=dev),
                          _aligned_workspace(decision_workspace_size(n, vocab), dev, 256))
    _ok(lib().dlm_decision_loss_fwd_bwd(
        n, _ptr(logits), max(int(logits.shape[0]), 1), logits.stride(0), vocab, _ptr(slot_rows), _ptr(cand_off),
        int(cand_ids.numel()), _ptr(cand_ids),
        _ptr(label_kind), _ptr(label_val), label_softmax, brier_weight, hard_label_smoothing, grad_scale,
        _ptr(out.loss), _ptr(out.slot_loss), _ptr(out.dlogits), out.dlogits.stride(0), _ptr(out.workspace),
        out.workspace.numel(), _stream()), "dlm_decision_loss_fwd_bwd")
    return out


def device_status(workspace: torch.Tensor) -> int:
    """Device status word of a loss workspace (synchronises the stream)."""
    v = ctypes.c_uint32(0)
    _ok(lib().dlm_get_device_status(_ptr(workspace), ctypes.byref(v), _stream()),
        "dlm_get_device_status")
    return int(v.value)


# --------------------------------------------------------------------------
# autograd wrappers
# --------------------------------------------------------------------------
def scale_bf16_(x: torch.Tensor, scale: torch.Tensor) -> torch.Tensor:
    """x *= scale in place on the device (see dlm_scale_bf16); scale is a
    one-element float32 device tensor.  x: bf16, 1-D or 2-D with unit column
    stride."""
    _check(scale, torch.float32, "scale", min_numel=1)
    _check(x, torch.bfloat16, "x")
    x2 = x.view(1, -1) if x.dim() == 1 else x
    if x2.dim() != 2 or (x2.shape[1] > 1 and x2.stride(1) != 1):
        raise ValueError("x: 1-D contiguous or 2-D with unit column stride")
    _on_cuda(x=x, scale=scale)
    _ok(lib().dlm_scale_bf16(_ptr(x2), x2.shape[0], x2.shape[1], x2.stride(0) if x2.shape[0] > 1 else x2.shape[1],
                             _ptr(scale), _stream()), "dlm_scale_bf16")
    return x


def _upstream(grad: torch.Tensor) -> torch.Tensor:
    return grad.detach().reshape(1).to(torch.float32).contiguous()


class _DiffusionLossFn(torch.autograd.Function):
    @staticmethod
    def forward(ctx, logits, enc_logits, layout, vocab, clean_ids, corrupted, p, mode, align, enc_layout,
                enc_ids, enc_ar_weight, options):
        out = loss_fwd_bwd(layout, logits, vocab, clean_ids, corrupted, p, mode, align, enc_layout=enc_layout,
                           enc_logits=enc_logits, enc_ids=enc_ids, enc_ar_weight=enc_ar_weight, options=options)
        ctx.grads = (out.dlogits, out.enc_dlogits)
        ctx.out = out
        return out.loss.view(())

    @staticmethod
    def backward(ctx, grad):
        g = _upstream(grad)
        d, de = ctx.grads
        ctx.grads = None
        scale_bf16_(d, g)
        if de is not None:
            scale_bf16_(de, g)
        return (d, de) + (None,) * 11


def diffusion_loss(layout: Layout, logits: torch.Tensor, vocab: int, clean_ids: torch.Tensor,
                   corrupted: Optional[torch.Tensor], p: Optional[torch.Tensor], mode: int = ABSORBING,
                   align: int = ALIGNED, enc_layout: Optional[Layout] = None,
                   enc_logits: Optional[torch.Tensor] = None, enc_ids: Optional[torch.Tensor] = None,
                   enc_ar_weight: float = 1.0, options: Optional[LossOptions] = None) -> torch.Tensor:
    """The loss of dlm_loss_fwd_bwd as a differentiable scalar of `logits`
    (and `enc_logits`).  The forward computes the gradient too and keeps it
    (memory of one logits tensor) until backward hands it to autograd.
    Logits are [rows, vocab] here (the gradient has their shape)."""
    for t, name in ((logits, "logits"), (enc_logits, "enc_logits")):
        if t is not None and (t.dim() != 2 or t.shape[1] != vocab):
            raise ValueError(f"{name}: [rows, vocab]")
    return _DiffusionLossFn.apply(logits, enc_logits, layout, vocab, clean_ids, corrupted, p, mode, align,
                                  enc_layout, enc_ids, enc_ar_weight, options)


class _LinearLossFn(torch.autograd.Function):
    @staticmethod
    def forward(ctx, hidden, weight, layout, clean_ids, corrupted, p, align):
        out = linear_loss_fwd_bwd(layout, hidden, weight, clean_ids, corrupted, p,
                                  want_d_weight=weight.requires_grad, align=align)
        ctx.grads = (out.d_hidden, out.d_weight)
        ctx.out = out
        return out.loss.view(())

    @staticmethod
    def backward(ctx, grad):
        g = _upstream(grad)
        dh, dw = ctx.grads
        ctx.grads = None
        scale_bf16_(dh, g)
        if dw is not None:
            scale_bf16_(dw, g)
        return (dh, dw) + (None,) * 5


def linear_diffusion_loss(layout: Layout, hidden: torch.Tensor, weight: torch.Tensor, clean_ids: torch.Tensor,
                          corrupted: torch.Tensor, p: torch.Tensor, align: int = ALIGNED) -> torch.Tensor:
    """The loss of dlm_linear_loss_fwd_bwd as a differentiable scalar of
    `hidden` and `weight` (dW is skipped when weight does not require a
    gradient, e.g. a frozen head)."""
    return _LinearLossFn.apply(hidden, weight, layout, clean_ids, corrupted, p, align)


class _LinearUniformLossFn(torch.autograd.Function):
    @staticmethod
    def forward(ctx, hidden, enc_hidden, weight, layout, clean_ids, enc_layout, enc_ids, enc_ar_weight, align):
        out = linear_loss_uniform_fwd_bwd(layout, hidden, weight, clean_ids, enc_layout, enc_hidden, enc_ids,
                                          enc_ar_weight=enc_ar_weight, align=align,
                                          want_d_weight=weight.requires_grad)
        ctx.grads = (out.d_hidden, out.d_enc_hidden, out.d_weight)
        ctx.out = out
        return out.loss.view(())

    @staticmethod
    def backward(ctx, grad):
        g = _upstream(grad)
        grads = ctx.grads
        ctx.grads = None
        for t in grads:
            if t is not None:
                scale_bf16_(t, g)
        return grads + (None,) * 6


def linear_uniform_loss(layout: Layout, hidden: torch.Tensor, weight: torch.Tensor, clean_ids: torch.Tensor,
                        enc_layout: Optional[Layout] = None, enc_hidden: Optional[torch.Tensor] = None,
                        enc_ids: Optional[torch.Tensor] = None, enc_ar_weight: float = 1.0,
                        align: int = ALIGNED) -> torch.Tensor:
    """The loss of dlm_linear_loss_uniform_fwd_bwd as a differentiable
    scalar of `hidden`, `enc_hidden` and `weight`."""
    return _LinearUniformLossFn.apply(hidden, enc_hidden, weight, layout, clean_ids, enc_layout, enc_ids,
                                      enc_ar_weight, align)


class _DecisionLossFn(torch.autograd.Function):
    @staticmethod
    def forward(ctx, logits, vocab, cand_off, cand_ids, label_kind, label_val, label_softmax, brier_weight,
                hard_label_smoothing):
        out = decision_loss_fwd_bwd(logits, vocab, cand_off, cand_ids, label_kind, label_val,
                                    label_softmax=label_softmax, brier_weight=brier_weight,
                                    hard_label_smoothing=hard_label_smoothing)
        ctx.grads = out.dlogits
        ctx.out = out
        return out.loss.view(())

    @staticmethod
    def backward(ctx, grad):
        d = ctx.grads
        ctx.grads = None
        scale_bf16_(d, _upstream(grad))
        return (d,) + (None,) * 8


def decision_loss(logits: torch.Tensor, vocab: int, cand_off: torch.Tensor, cand_ids: torch.Tensor,
                  label_kind: torch.Tensor, label_val: torch.Tensor, label_softmax: int = LABEL_SOFTMAX_BOTH,
                  brier_weight: float = 0.1, hard_label_smoothing: float = 0.0) -> torch.Tensor:
    """The typed-decision loss of dlm_decision_loss_fwd_bwd as a
    differentiable scalar of `logits` ([n_slots, vocab], one row per label
    slot)."""
    if logits.dim() != 2 or tuple(logits.shape) != (cand_off.numel() - 1, vocab):
        raise ValueError("logits: [n_slots, vocab], one row per label slot")
    return _DecisionLossFn.apply(logits, vocab, cand_off, cand_ids, label_kind, label_val, label_softmax,
                                 brier_weight, hard_label_smoothing)
