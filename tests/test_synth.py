"""The seeded input generators: deterministic, index-addressable, and drawing
the distributions the workloads name (fp16 N(0, 0.02) master weights with a
0.1% rate of +-0.2 outliers where asked, bf16 N(0, 1) activations, top-k
routing with softmax-renormalised weights)."""
import numpy as np
import torch

import synth


def test_counter_generator_is_index_addressable():
    wl = synth.WORKLOADS[2]
    full = synth.expert_weights(wl, 3, 1000, 5000)
    idx = torch.tensor([1000, 1001, 3333, 5999])
    assert torch.equal(synth.expert_weights_at(wl, 3, idx), full[idx - 1000])
    again = synth.expert_weights(wl, 3, 1000, 5000)
    assert torch.equal(full, again)
    other = synth.expert_weights(wl, 4, 1000, 5000)
    assert not torch.equal(full, other)


def test_uniform_high_indices():
    u = synth.uniform_u32(7, 1, (1 << 32) - 4, 4)
    assert u.dtype == torch.int64 and int(u.min()) >= 0 and int(u.max()) < (1 << 32)
    v = synth.uniform_u32_at(7, 1, torch.tensor([(1 << 32) - 1], dtype=torch.int64))
    assert int(v[0]) == int(u[3])


def test_weight_distribution():
    wl = synth.WORKLOADS[1]
    w = synth.expert_weights(wl, 0).double()
    assert abs(w.mean().item()) < 5e-4
    assert abs(w.std().item() - 0.02) < 3e-4
    wl2 = synth.WORKLOADS[2]
    w2 = synth.expert_weights(wl2, 0, 0, 1 << 22).double()
    frac = (w2.abs() > 0.19).double().mean().item()
    assert 0.0008 < frac < 0.0012
    assert w2.abs().max().item() == float(np.float16(0.2))


def test_activation_distribution():
    wl = synth.WORKLOADS[4]
    x = synth.activations(wl, T=256)
    assert x.dtype == torch.bfloat16 and x.shape == (256, wl.H)
    assert abs(x.double().std().item() - 1.0) < 0.01


def test_topk_routing():
    logits = np.array([[0.1, 0.5, 0.5, -1.0], [2.0, 1.0, 0.0, 3.0]])
    ids, w = synth.topk_route(logits, 2)
    assert ids.tolist() == [[1, 2], [3, 0]]       # ties -> lower expert id
    assert np.allclose(w.sum(1), 1.0)
    assert np.allclose(w[0], [0.5, 0.5])
    e = np.exp(np.array([3.0, 2.0]) - 3.0)
    assert np.allclose(w[1], e / e.sum())


def test_zipf_skew_and_schedule():
    wl = synth.WORKLOADS[3]
    p = synth.importance(wl)
    assert abs(p.sum() - 1.0) < 1e-12
    assert abs(p.max() - 1.0 / sum(r ** -1.1 for r in range(1, 129))) < 1e-12
    ids, _ = synth.routing(wl)
    counts = np.bincount(ids.ravel(), minlength=wl.E)
    assert counts.max() >= 40   # the top expert is picked by most tokens
    sch = synth.schedule(synth.WORKLOADS[5])
    assert len(sch) == 20 and [k for k, _ in sch[::2]] == ["decode"] * 10
    assert [a for _, a in sch[1::2]] == synth.REPAGE_AVG_BITS
