"""CUDA failures turned into status codes, on a host without a usable GPU.

With the library's device check skipped (the dlm_test_skip_device_check test
hook), every entry point goes on to its own CUDA calls; on a host where the
CUDA runtime finds no device those calls fail, and each entry point must
return DLM_ERR_CUDA with a message naming the step that failed -- no crash,
no hang -- and keep working for the next call.  The failure is made on the
host (a runtime without a device), never on a GPU: the tests run only where
neither the CUDA driver nor torch can reach a device (decided without calling
the library, so nothing is launched), and skip everywhere else.  The pointers
below are fake device addresses that the host code never dereferences.
"""
import ctypes

import pytest

import diffusion_lm_loss_b200 as dlm
from diffusion_lm_loss_b200 import build as dlm_build

DLM_ERR_INVALID_ARGUMENT, DLM_ERR_CUDA = 1, 4
WS = 1 << 20               # a fake, 1024-byte aligned workspace address


def _a_device_may_be_usable() -> bool:
    """True unless neither the CUDA driver nor torch can see a device.  Decided
    without the library, so that nothing is launched: on a host with a device,
    a call with the fake pointers below would write to them."""
    import torch
    if torch.cuda.is_available() or torch.cuda.device_count() > 0:
        return True
    try:
        cu = ctypes.CDLL("libcuda.so.1")
    except OSError:
        return False                        # no driver: no device can be reached
    n = ctypes.c_int(0)
    if cu.cuInit(0) != 0:
        return False
    return cu.cuDeviceGetCount(ctypes.byref(n)) != 0 or n.value > 0


@pytest.fixture(scope="module")
def L():
    if _a_device_may_be_usable():
        pytest.skip("a CUDA device may be usable here: the hook must not run with fake pointers")
    dlm_build.build()
    lib = dlm.lib()
    assert lib.dlm_test_skip_device_check(1) == 0
    yield lib
    assert lib.dlm_test_skip_device_check(0) == 0


def _fails_at(L, rc, step):
    msg = L.dlm_last_cuda_error().decode()
    assert rc == DLM_ERR_CUDA, (rc, msg)
    assert msg.startswith(step), msg


def test_every_entry_point_reports_its_cuda_failure(L):
    lay = dlm.Layout(2, 24, 48, None, None)
    enc = dlm.Layout(2, 32, 64, None, None)
    ws_l = L.dlm_loss_workspace_size(ctypes.byref(lay), None)
    ws_e = L.dlm_loss_workspace_size(ctypes.byref(lay), ctypes.byref(enc))
    ws_h = L.dlm_linear_loss_workspace_size(ctypes.byref(lay), 64, 1024)
    ws_u = L.dlm_linear_loss_uniform_workspace_size(ctypes.byref(lay), ctypes.byref(enc), 64, 1024)
    lp = ctypes.byref(lay)
    for _ in range(2):      # a second round: nothing is left broken by the first
        _fails_at(L, L.dlm_sample_t(1, 4, 0, 1e-3, 256, 512, None), "k_sample_t launch")
        _fails_at(L, L.dlm_corrupt(lp, 256, 512, 0, 999, 1000, 7, 1024, 2048, None, None), "k_corrupt launch")
        _fails_at(L, L.dlm_loss_fwd_bwd(lp, 4096, 1000, 1000, 256, 512, 768, 0, 0, None, None, 0, None,
                                        1.0, 1.0, 1024, 1280, 8192, None, WS, ws_l, None), "k_plan")
        _fails_at(L, L.dlm_loss_fwd_bwd(lp, 4096, 4096, 4096, 256, None, None, 1, 0, ctypes.byref(enc), 8192,
                                        4096, 512, 1.0, 1.0, 1024, 1280, 16384, 32768, WS, ws_e, None), "k_plan")
        _fails_at(L, L.dlm_loss_fwd_bwd_ex(lp, 4096, 1000, 1000, 256, 512, 768, 0, 0, None, None, 0, None,
                                           1.0, 1.0, None, 1024, 1280, 8192, None, WS, ws_l, None), "k_plan")
        _fails_at(L, L.dlm_loss_fwd_bwd_static(lp, 4096, 1000, 1000, 256, 512, 768, 0, 0, None, None, 0,
                                               None, 1.0, 1.0, 1024, 1280, 8192, None, None), "cudaGetSymbolAddress(scratch)")
        _fails_at(L, L.dlm_linear_loss_fwd_bwd(lp, 4096, 8192, 64, 1024, 256, 512, 768, 1.0, 1024, 1280,
                                               16384, 32768, WS, ws_h, None), "k_plan")
        _fails_at(L, L.dlm_linear_loss_fwd_bwd_ex(lp, 4096, 8192, 64, 1024, 256, 512, 768, 1, 1.0, 1024,
                                                  1280, 16384, 32768, WS, ws_h, None), "k_plan")
        _fails_at(L, L.dlm_linear_loss_uniform_fwd_bwd(lp, 4096, ctypes.byref(enc), 8192, 512, 16384, 64,
                                                       1024, 256, 0, 1.0, 1.0, 1024, 1280, 32768, 65536,
                                                       None, WS, ws_u, None), "k_plan")
        ws_d = L.dlm_decision_workspace_size(4, 1024)
        dec = [4, 4096, 4, 1024, 1024, None, 256, 8, 512, 768, 1024, 3, 0.1, 0.0, 1.0, 1280, None, 8192, 1024,
               WS, ws_d, None]
        _fails_at(L, L.dlm_decision_loss_fwd_bwd(*dec), "k_dec_cluster launch")          # 16-byte rows
        dec_g = list(dec); dec_g[3] = 1025
        _fails_at(L, L.dlm_decision_loss_fwd_bwd(*dec_g), "k_dec_partial launch")      # any row stride
        dec_0 = list(dec); dec_0[0] = 0
        _fails_at(L, L.dlm_decision_loss_fwd_bwd(*dec_0), "status reset")              # no slots
        _fails_at(L, L.dlm_scale_bf16(4096, 4, 64, 64, 256, None), "k_scale_bf16 launch")
        _fails_at(L, L.dlm_selftest_bounded_wait(1000, 256, None), "k_selftest_wait launch")
        _fails_at(L, L.dlm_get_device_status(WS, ctypes.byref(ctypes.c_uint32()), None),
                  "dlm_get_device_status")


def test_argument_errors_still_come_first(L):
    """With the device check skipped, a bad argument is still refused before
    any CUDA call (the message of the last CUDA failure is left as it was)."""
    lay = dlm.Layout(2, 24, 48, None, None)
    L.dlm_sample_t(1, 4, 0, 1e-3, 256, 512, None)
    before = L.dlm_last_cuda_error().decode()
    assert L.dlm_sample_t(1, 4, 0, 1e-3, None, 512, None) == DLM_ERR_INVALID_ARGUMENT
    assert L.dlm_loss_fwd_bwd(ctypes.byref(lay), 4096, 1000, 1000, 256, 512, 768, 0, 7, None, None, 0, None,
                              1.0, 1.0, 1024, 1280, 8192, None, WS, 1 << 30, None) == DLM_ERR_INVALID_ARGUMENT
    assert L.dlm_last_cuda_error().decode() == before


def test_hook_values(L):
    assert L.dlm_test_skip_device_check(2) == DLM_ERR_INVALID_ARGUMENT
    assert L.dlm_test_skip_device_check(-1) == DLM_ERR_INVALID_ARGUMENT
    assert L.dlm_test_skip_device_check(1) == 0
