"""GPU parity of the time draw and the corruption against the CPU oracle:
bit-exact t, p, masks and replacement ids, through the C ABI."""
import numpy as np
import pytest
import torch

import dlm_inputs as di
import oracle

pytestmark = pytest.mark.gpu

dlm = pytest.importorskip("diffusion_lm_loss_b200")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dlm.lib()


@pytest.mark.parametrize("mode", [oracle.ABSORBING, oracle.UNIFORM])
@pytest.mark.parametrize("n_units,seed,eps", [(1, 0, 1e-3), (8, 3, 1e-3), (5000, 2 ** 40 + 7, 0.05),
                                             (1 << 16, 12345, 0.0)])
def test_sample_t_bit_exact(mode, n_units, seed, eps):
    t, p = dlm.sample_t(seed, n_units, mode, eps)
    to, po = oracle.sample_t(seed, n_units, mode, eps)
    assert np.array_equal(t.cpu().numpy().view(np.uint32), to.view(np.uint32))
    assert np.array_equal(p.cpu().numpy().view(np.uint32), po.view(np.uint32))


def _corrupt_both(n_units, seq_len, cu, pad, clean, p, mode, mask_id, vocab, seed):
    dev = torch.device("cuda")
    n = clean.shape[0]
    cu_d = torch.from_numpy(cu).to(dev) if cu is not None else None
    pad_d = torch.from_numpy(pad).to(dev) if pad is not None else None
    lay = dlm.make_layout(n_units, seq_len, cu_d, pad_d, n_tokens=n)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    noisy, corr = dlm.corrupt(lay, torch.from_numpy(clean).to(dev), torch.from_numpy(p).to(dev),
                              mode, mask_id, vocab, seed, dev_status=status)
    no, co = oracle.corrupt(oracle.Layout(n_units, seq_len, cu, pad), clean, p, mode, mask_id,
                            vocab, seed)
    return noisy.cpu().numpy(), corr.cpu().numpy(), no, co, int(status.item())


@pytest.mark.parametrize("key", [k for k, s in di.WORKLOADS.items() if s.kind != "decision"])   # label slots are not corrupted
def test_corrupt_bit_exact_on_every_workload_shape(key):
    spec = di.WORKLOADS[key]
    case = di.make_case(spec, "cpu", with_tensors=False)
    mode = spec.mode
    eps = spec.eps
    for seed in (0, 1, 987654321):
        _, p = oracle.sample_t(seed, case.n_units, mode, eps)
        cu = case.cu_seqlens.numpy() if case.cu_seqlens is not None else None
        g_noisy, g_corr, o_noisy, o_corr, st = _corrupt_both(
            case.n_units, case.seq_len, cu, None, case.clean.numpy(), p, mode,
            spec.mask_id, spec.vocab, seed)
        assert st == 0
        assert np.array_equal(g_corr, o_corr)
        assert np.array_equal(g_noisy, o_noisy)


def test_corrupt_pads_docs_and_empty_documents():
    rng = np.random.default_rng(0)
    lens = [7, 0, 130, 1, 0, 600, 33]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    T = int(cu[-1])
    clean = rng.integers(0, 50000, T).astype(np.int32)
    pad = (rng.random(T) < 0.2).astype(np.uint8)
    p = rng.uniform(0.001, 1.0, len(lens)).astype(np.float32)
    for mode in (oracle.ABSORBING, oracle.UNIFORM):
        g_noisy, g_corr, o_noisy, o_corr, st = _corrupt_both(len(lens), 0, cu, pad, clean, p, mode,
                                                              50000, 50001, 77)
        assert st == 0
        assert np.array_equal(g_corr, o_corr) and np.array_equal(g_noisy, o_noisy)
        assert g_corr[pad == 1].sum() == 0


def test_corrupt_threshold_edges():
    """p exactly at the floor and just below 1: the strict fp32 compare."""
    n = 1 << 16
    clean = np.arange(n, dtype=np.int32) % 1000
    for pv in (np.float32(1e-3), np.nextafter(np.float32(1.0), np.float32(0)), np.float32(0.5)):
        p = np.array([pv], np.float32)
        g_noisy, g_corr, o_noisy, o_corr, _ = _corrupt_both(1, n, None, None, clean, p,
                                                            oracle.ABSORBING, 1000, 1001, 5)
        assert np.array_equal(g_corr, o_corr) and np.array_equal(g_noisy, o_noisy)


def test_corrupt_draw_exactly_on_the_threshold():
    """A token whose 24-bit draw equals p * 2^24 stays clean, on the GPU as in
    the oracle (strict compare): p = k / 2^24 for the k one token drew."""
    n = 4000
    base = oracle.counter(1, 0, 0)
    u24 = np.array([oracle.splitmix64_at(91, base + i) >> 40 for i in range(n)], np.int64)
    i0 = int(np.argmax(u24 > 0))
    p = np.array([int(u24[i0]) * 2.0 ** -24], np.float32)
    clean = np.zeros(n, np.int32)
    g_noisy, g_corr, o_noisy, o_corr, st = _corrupt_both(1, n, None, None, clean, p, oracle.ABSORBING, 1, 2, 91)
    assert st == 0 and g_corr[i0] == 0 and o_corr[i0] == 0
    assert np.array_equal(g_corr, o_corr) and np.array_equal(g_noisy, o_noisy)


def test_corrupt_flags_bad_cu_seqlens():
    cu = np.array([0, 10, 4, 20], np.int32)       # not non-decreasing
    clean = np.zeros(20, np.int32)
    p = np.full(3, 0.5, np.float32)
    dev = torch.device("cuda")
    lay = dlm.make_layout(3, 0, torch.from_numpy(cu).to(dev), None, n_tokens=20)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    dlm.corrupt(lay, torch.from_numpy(clean).to(dev), torch.from_numpy(p).to(dev),
                oracle.ABSORBING, 1, 2, 0, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) & dlm.DEV_BAD_LAYOUT
