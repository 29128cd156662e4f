"""Host checks of the seeded synthetic-input generator (no method arithmetic)."""
import numpy as np
import torch

import dlm_inputs as di


def test_doc_lengths_cover_total_and_respect_bounds():
    g = torch.Generator(); g.manual_seed(5)
    lens = di.doc_lengths(16384, 296.0, 16, 4096, g)
    assert sum(lens) == 16384
    assert all(16 <= l <= 4096 for l in lens[:-1])
    assert lens[-1] >= 16
    # mean in the right range for a geometric(mean 296) clamped below at 16
    assert 150 < sum(lens) / len(lens) < 500


def test_same_seed_same_case():
    spec = di.WORKLOADS["abs_b2_l64_v1024"]
    a = di.make_case(spec, "cpu")
    b = di.make_case(spec, "cpu")
    assert torch.equal(a.clean, b.clean) and torch.equal(a.logits.view(torch.int16), b.logits.view(torch.int16))
    c = di.make_case(spec, "cpu", seed=1)
    assert not torch.equal(a.clean, c.clean)


def test_shapes_and_ranges():
    s = di.WORKLOADS["abs_b1_l4096_v126464"].scaled(seq_len=64)
    c = di.make_case(s, "cpu")
    assert c.logits.shape == (64, 126464) and c.logits.dtype == torch.bfloat16
    assert int(c.clean.min()) >= 0 and int(c.clean.max()) <= s.ids_high
    # the clean token's logit carries the +4 spike: it is the row maximum most of the time
    hits = (c.logits.float().argmax(1) == c.clean.long()).float().mean()
    assert hits < 1.0  # N(0,3) noise over 126k columns usually exceeds +4
    u = di.WORKLOADS["unif_b4_p512_c1024_v262144"].scaled(prefix=8, seq_len=16, vocab=1000, ids_high=999)
    cu = di.make_case(u, "cpu")
    assert cu.enc_clean.shape == (4 * 24,) and cu.clean.shape == (4 * 16,)
    assert torch.equal(cu.enc_clean.view(4, 24)[:, 8:].reshape(-1), cu.clean)
    assert cu.logits.shape == (64, 1000) and cu.enc_logits.shape == (96, 1000)
    l = di.WORKLOADS["lin_t16384_d4096_v126464"].scaled(n_tokens_packed=512, d_model=64, vocab=1000,
                                                        ids_high=990, mask_id=991)
    cl = di.make_case(l, "cpu")
    assert int(cl.cu_seqlens[-1]) == 512 and cl.hidden.shape == (512, 64) and cl.weight.shape == (1000, 64)


def test_decision_workload_recipe():
    """The typed-decision draws: K in [2, k_max] answers per slot, the first
    K codebook tokens, distinct ids inside the vocabulary, valid labels of
    every kind, and the same draw for the same seed."""
    spec = di.WORKLOADS["dec_s128_k26_v126464"].scaled(n_units=40, vocab=5000, ids_high=4999)
    a = di.make_case(spec, "cpu")
    b = di.make_case(spec, "cpu")
    e = a.extra
    off, ids, kind, val = (e[k].numpy() for k in ("cand_off", "cand_ids", "kind", "val"))
    assert off[0] == 0 and (np.diff(off) >= 2).all() and (np.diff(off) <= spec.k_max).all()
    assert ids.min() >= 0 and ids.max() < spec.vocab
    longest = int(np.argmax(np.diff(off)))
    book = ids[off[longest]:off[longest + 1]]
    for i in range(spec.n_units):
        seg = ids[off[i]:off[i + 1]]
        assert len(np.unique(seg)) == len(seg) and np.array_equal(seg, book[:len(seg)])
        v = val[off[i]:off[i + 1]]
        if kind[i] == di.HARD:
            assert (v == 1).sum() == 1 and ((v == 0) | (v == 1)).all()
        elif kind[i] == di.DIST:
            assert (v >= 0).all() and abs(v.sum() - 1) < 1e-4
        else:
            assert (v == 1).sum() >= 1 and ((v == 0) | (v == 1)).all()
    assert set(kind.tolist()) == {di.HARD, di.DIST, di.SET}
    assert torch.equal(a.logits, b.logits) and torch.equal(a.extra["val"], b.extra["val"])
    assert tuple(a.logits.shape) == (40, 5000)
