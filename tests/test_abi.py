"""The C-ABI library loads and exports every symbol include/dlm.h declares;
host-side argument checks reject bad calls before anything touches a GPU
(no compute calls here: these run without a device)."""
import ctypes
import os
import re

import pytest

from conftest import ROOT

import diffusion_lm_loss_b200 as dlm
from diffusion_lm_loss_b200 import build as dlm_build


@pytest.fixture(scope="module")
def L():
    dlm_build.build()
    return dlm.lib()


def declared_functions():
    src = open(os.path.join(ROOT, "include", "dlm.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(dlm_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_four_path_calls():
    names = declared_functions()
    for n in ("dlm_sample_t", "dlm_corrupt", "dlm_loss_fwd_bwd", "dlm_linear_loss_fwd_bwd"):
        assert n in names


def test_every_declared_symbol_is_exported(L):
    names = declared_functions()
    assert set(names) == set(dlm.EXPORTS)
    for n in names:
        assert hasattr(L, n), n
    # nothing else leaks out of the library (hidden visibility)
    out = os.popen(f"nm -D --defined-only {dlm.LIB_PATH}").read()
    exported = set(re.findall(r"\bT (dlm_[a-z0-9_]+)", out))
    assert exported == set(names)


def test_status_strings_and_version(L):
    assert L.dlm_status_string(0) == b"DLM_OK"
    assert L.dlm_status_string(3) == b"DLM_ERR_WORKSPACE_TOO_SMALL"
    assert L.dlm_status_string(99) == b"DLM_ERR_UNKNOWN"
    assert L.dlm_version() >= 100


def test_host_side_rejections(L):
    # these all fail argument validation before any device query or launch
    assert L.dlm_sample_t(0, -1, 0, 1e-3, None, None, None) == 1
    assert L.dlm_sample_t(0, 4, 7, 1e-3, None, None, None) == 1
    assert L.dlm_sample_t(0, 4, 0, 1.5, None, None, None) == 1
    assert L.dlm_sample_t(0, 0, 0, 1e-3, None, None, None) == 0           # no-op
    bad = dlm.Layout(2, 10, 21, None, None)                              # 2*10 != 21
    assert L.dlm_corrupt(ctypes.byref(bad), None, None, 0, 0, 0, 0, None, None, None, None) == 1
    lay = dlm.Layout(2, 10, 20, None, None)
    assert L.dlm_corrupt(ctypes.byref(lay), None, None, 0, 0, 0, 0, None, None, None, None) == 1
    # loss: ld < vocab, bad mode, encoder with absorbing noise, small workspace
    args = [ctypes.byref(lay), 16, 32, 32, 16, 16, 16, 0, 0, None, None, 0, None, 0.0, 1.0, 16,
            None, 16, None, 256, 1 << 20, None]
    a = list(args); a[2] = 16
    assert L.dlm_loss_fwd_bwd(*a) == 1                                    # ld < vocab
    a = list(args); a[7] = 5
    assert L.dlm_loss_fwd_bwd(*a) == 1                                    # mode
    a = list(args); a[8] = 9
    assert L.dlm_loss_fwd_bwd(*a) == 1                                    # align
    a = list(args); a[10] = 16
    assert L.dlm_loss_fwd_bwd(*a) == 1                                    # encoder w/ absorbing
    a = list(args); a[20] = 4
    assert L.dlm_loss_fwd_bwd(*a) == 3                                    # workspace too small
    a = list(args); a[19] = 100
    assert L.dlm_loss_fwd_bwd(*a) == 1                                    # misaligned workspace
    # objective options: only for uniform noise, known values, a full struct,
    # time weighting needs p
    def ex(opts, mode=1, p=16):
        a = list(args)
        a[6] = p
        a[7] = mode
        a.insert(15, ctypes.byref(opts) if opts is not None else None)
        return L.dlm_loss_fwd_bwd_ex(*a)
    assert ex(dlm.LossOptions(dlm.TIME_WEIGHT_INV_ONE_MINUS_T, 2.0), mode=0) == 1   # absorbing
    assert ex(dlm.LossOptions(reduction=dlm.REDUCE_EXAMPLE_MEAN), mode=0) == 1
    assert ex(dlm.LossOptions(time_weighting=7)) == 1
    assert ex(dlm.LossOptions(reduction=5)) == 1
    short = dlm.LossOptions(dlm.TIME_WEIGHT_INV_ONE_MINUS_T)
    short.struct_size = 8
    assert ex(short) == 1
    assert ex(dlm.LossOptions(dlm.TIME_WEIGHT_INV_ONE_MINUS_T), p=None) == 1          # no p
    assert ex(dlm.LossOptions(weight_clip=float("nan"))) == 1
    assert ex(dlm.LossOptions(keep_unscored_rows=2)) == 1
    old16 = dlm.LossOptions(keep_unscored_rows=2)    # a 16-byte struct: the field is not read
    old16.struct_size = 16
    assert ex(old16) != 1
    # fused head: alignment must be aligned or shifted
    lin = dlm.Layout(1, 64, 64, None, None)
    assert L.dlm_linear_loss_fwd_bwd_ex(ctypes.byref(lin), 16, 16, 64, 1024, 16, 16, 16, 7, 1.0, 16, None,
                                        16, None, 1024, 1 << 30, None) == 1
    # bounded-wait self-test: no status word, zero or over-long limit
    assert L.dlm_selftest_bounded_wait(10, None, None) == 1
    assert L.dlm_selftest_bounded_wait(0, 16, None) == 1
    assert L.dlm_selftest_bounded_wait(20_000_000_000, 16, None) == 1


def test_linear_uniform_rejections(L):
    """Host-side checks of dlm_linear_loss_uniform_fwd_bwd: each bad argument
    returns DLM_ERR_INVALID_ARGUMENT (or WORKSPACE_TOO_SMALL) before anything
    is enqueued (no GPU is touched)."""
    can = dlm.Layout(2, 32, 64, None, None)
    enc = dlm.Layout(2, 48, 96, None, None)
    need = L.dlm_linear_loss_uniform_workspace_size(ctypes.byref(can), ctypes.byref(enc), 64, 1024)

    def call(layout=can, hidden=16, enc_layout=enc, enc_hidden=16, enc_ids=16, d_model=64, vocab=1024,
             clean=16, align=0, d_hidden=16, d_enc_hidden=16, ws=1024, ws_bytes=need):
        e = ctypes.byref(enc_layout) if enc_layout is not None else None
        return L.dlm_linear_loss_uniform_fwd_bwd(ctypes.byref(layout), hidden, e, enc_hidden, enc_ids, 16,
                                                 d_model, vocab, clean, align, 1.0, 1.0, 16, None, d_hidden,
                                                 d_enc_hidden, None, ws, ws_bytes, None)
    assert call(align=2) == 1
    assert call(d_model=96) == 1                                  # d_model % 64
    assert call(vocab=1020) == 1                                  # vocab % 8
    assert call(enc_layout=dlm.Layout(3, 32, 96, None, None)) == 1  # unit counts differ
    assert call(enc_hidden=None) == 1
    assert call(enc_ids=None) == 1
    assert call(d_enc_hidden=None) == 1
    assert call(enc_hidden=24) == 1                               # not 16-byte aligned
    assert call(clean=None) == 1
    assert call(d_hidden=None) == 1
    assert call(ws=512) == 1                                      # workspace not 1024-aligned
    assert call(ws_bytes=need - 1) == 3                           # DLM_ERR_WORKSPACE_TOO_SMALL
    # without the encoder term the workspace is that of the canvas rows alone;
    # with it, that of canvas + encoder rows
    alone = L.dlm_linear_loss_uniform_workspace_size(ctypes.byref(can), None, 64, 1024)
    assert alone == L.dlm_linear_loss_workspace_size(ctypes.byref(can), 64, 1024)
    both = dlm.Layout(2, 80, 160, None, None)
    assert need == L.dlm_linear_loss_workspace_size(ctypes.byref(both), 64, 1024)
    # rows whose 256-row padding would overflow an int: no workspace size
    huge = dlm.Layout(1, 0, (1 << 31) - 200, None, None)
    assert L.dlm_linear_loss_workspace_size(ctypes.byref(huge), 64, 1024) == 0
    assert L.dlm_linear_loss_uniform_workspace_size(ctypes.byref(huge), None, 64, 1024) == 0
    half = dlm.Layout(1, 0, 1 << 30, None, None)
    assert L.dlm_linear_loss_uniform_workspace_size(ctypes.byref(half), ctypes.byref(half), 64, 1024) == 0


def test_decision_and_scale_rejections(L):
    """dlm_decision_loss_fwd_bwd and dlm_scale_bf16 refuse bad arguments
    before any device query or launch."""
    n, V = 4, 1024
    ws = L.dlm_decision_workspace_size(n, V)
    assert ws > 0
    assert L.dlm_decision_workspace_size(dlm.DECISION_MAX_SLOTS, V) > 0
    assert L.dlm_decision_workspace_size(dlm.DECISION_MAX_SLOTS + 1, V) == 0
    assert L.dlm_decision_workspace_size(-1, V) == 0
    assert L.dlm_decision_workspace_size(n, 0) == 0
    # n_slots, logits, n_rows, ld, vocab, slot_rows, cand_off, n_cands, cand_ids, kind, val,
    # label_softmax, brier, smoothing, grad_scale, loss, slot_loss, dlogits, ld_out, ws, ws_bytes, stream
    args = [n, 4096, n, V, V, None, 256, 8, 512, 768, 1024, dlm.LABEL_SOFTMAX_BOTH, 0.1, 0.0, 1.0, 1280,
            None, 8192, V, 1 << 20, ws, None]

    def rc(**kw):
        a = list(args)
        for k, v in kw.items():
            a[int(k[1:])] = v
        return L.dlm_decision_loss_fwd_bwd(*a)

    assert rc(a0=dlm.DECISION_MAX_SLOTS + 1) == 1         # too many slots
    assert rc(a0=-1) == 1
    assert rc(a4=0) == 1                                  # vocab
    assert rc(a3=V - 1) == 1                              # ld < vocab
    assert rc(a18=V - 1) == 1                             # ld_out < vocab
    assert rc(a2=0) == 1                                  # no rows
    assert rc(a2=n - 1) == 1                              # fewer rows than slots, no slot_rows
    assert rc(a7=-1) == 1                                 # n_cands
    assert rc(a11=0) == 1 and rc(a11=4) == 1              # label_softmax
    assert rc(a12=-0.5) == 1 and rc(a12=float("inf")) == 1   # brier weight
    assert rc(a13=1.5) == 1 and rc(a13=-0.1) == 1         # smoothing
    assert rc(a14=float("nan")) == 1                      # grad_scale
    assert rc(a15=None) == 1 and rc(a19=None) == 1        # loss, workspace
    assert rc(a1=None) == 1 and rc(a6=None) == 1 and rc(a17=None) == 1
    assert rc(a19=(1 << 20) + 4) == 1                     # misaligned workspace
    assert rc(a20=ws - 1) == 3                            # workspace too small
    # scale: rows, cols, ld, scale
    assert L.dlm_scale_bf16(4096, -1, 64, 64, 256, None) == 1
    assert L.dlm_scale_bf16(4096, 4, 64, 63, 256, None) == 1
    assert L.dlm_scale_bf16(4096, 4, 64, 64, None, None) == 1
    assert L.dlm_scale_bf16(None, 4, 64, 64, 256, None) == 1
    assert L.dlm_scale_bf16(None, 0, 64, 64, 256, None) == 0   # empty: nothing to do


def test_workspace_size_grows_with_rows(L):
    a = dlm.Layout(1, 4096, 4096, None, None)
    b = dlm.Layout(1, 8192, 8192, None, None)
    sa = L.dlm_loss_workspace_size(ctypes.byref(a), None)
    sb = L.dlm_loss_workspace_size(ctypes.byref(b), None)
    assert sa > 4096 * 16 and sb > sa and sa % 256 == 0


def test_header_is_plain_c_and_links(L, tmp_path):
    """include/dlm.h compiles as pedantic C99 and as C++, and a C program
    links against the library and calls it (no GPU call: the version)."""
    import shutil
    import subprocess
    cc = shutil.which("gcc")
    if cc is None:
        pytest.skip("no C compiler")
    src = tmp_path / "use_dlm.c"
    src.write_text(
        '#include "dlm.h"\n'
        'int main(void) {\n'
        '    dlm_loss_options_t o = {sizeof(o), DLM_TIME_WEIGHT_NONE, 0.f, DLM_REDUCE_TOKEN_MEAN, 0};\n'
        '    dlm_layout_t l = {1, 4, 4, 0, 0};\n'
        '    (void)o; (void)l;\n'
        '    return dlm_version() == %d ? 0 : 1;\n'
        '}\n' % L.dlm_version())
    inc = os.path.join(ROOT, "include")
    libdir = os.path.dirname(dlm.LIB_PATH)
    exe = tmp_path / "use_dlm"
    subprocess.run([cc, "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I", inc, str(src),
                    "-L", libdir, "-ldlm", "-Wl,-rpath," + libdir, "-o", str(exe)], check=True)
    subprocess.run(["g++", "-std=c++17", "-Wall", "-Wextra", "-Werror", "-I", inc, "-x", "c++", "-fsyntax-only",
                    str(src)], check=True)
    assert subprocess.run([str(exe)]).returncode == 0


def test_binding_refuses_cpu_tensors():
    import torch
    with pytest.raises((ValueError, TypeError)):
        dlm.corrupt(dlm.Layout(1, 4, 4, None, None), torch.zeros(4, dtype=torch.int32),
                    torch.zeros(1, dtype=torch.float32))


def test_oracle_and_product_share_no_code():
    """Neither side imports the other; the oracle has no CUDA, the package no
    oracle."""
    pkg = os.path.join(ROOT, "diffusion_lm_loss_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                txt = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in txt and "from oracle" not in txt and "dlm_oracle" not in txt
    for f in os.listdir(os.path.join(ROOT, "oracle")):
        if f.endswith((".py", ".c")):
            txt = open(os.path.join(ROOT, "oracle", f)).read()
            assert "diffusion_lm_loss_b200" not in txt and "dlm.h" not in txt
    # the seeded input module both sides use imports neither of them
    for f in os.listdir(os.path.join(ROOT, "dlm_inputs")):
        if f.endswith(".py"):
            txt = open(os.path.join(ROOT, "dlm_inputs", f)).read()
            for name in ("oracle", "diffusion_lm_loss_b200"):
                assert f"import {name}" not in txt and f"from {name}" not in txt
