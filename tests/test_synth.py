"""CPU checks of the synthetic input generator and forced routings."""
import numpy as np
import pytest


def _f32(bits):
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def test_generator_is_deterministic_and_keyed(syn):
    w = syn.WORKLOADS["tiny"]
    a = syn.codes_host(w, 0, 1, syn.GATE)
    assert (a == syn.codes_host(w, 0, 1, syn.GATE)).all()
    assert (a != syn.codes_host(w, 0, 2, syn.GATE)).any()
    assert (a != syn.codes_host(w, 1, 1, syn.GATE)).any()
    assert (syn.codes_host(w, 0, 1, syn.UP) != a).any()
    assert (syn.x_host(w, 0) != syn.x_host(w, 1)).any()


def test_codes_cover_their_range(syn):
    w = syn.WORKLOADS["tiny"]
    c4 = syn.codes_host(w, 0, 0, syn.DOWN)
    assert c4.max() == 15 and c4.min() == 0
    c2 = syn.codes_host(w.with_(bits_routed=2), 0, 0, syn.DOWN)
    assert c2.max() == 3 and c2.min() == 0
    c3 = syn.codes_host(w.with_(bits_routed=3), 0, 0, syn.DOWN)
    assert c3.max() == 7 and c3.min() == 0
    # low bits of the same draws
    assert ((c4 & 3) == c2).all() and ((c4 & 7) == c3).all()
    counts = np.bincount(c4.ravel(), minlength=16) / c4.size
    assert np.abs(counts - 1 / 16).max() < 0.01


def test_distributions(syn):
    w = syn.WORKLOADS["layer4"]
    s = _f32(syn.scale_host(w, 0, 3, syn.GATE)).astype(np.float64)
    assert s.min() >= 0.005 * (1 - 2 ** -8) and s.max() <= 0.02 * (1 + 2 ** -8)
    assert abs(s.mean() - 0.0125) < 2e-4
    b = _f32(syn.bias_host(w, 0, 3, syn.GATE)).astype(np.float64)
    assert abs(b.mean()) < 2e-4 and abs(b.std() - 0.01) < 3e-4
    x = _f32(syn.x_host(w, 5, 8)).astype(np.float64)
    assert abs(x.mean()) < 0.02 and abs(x.std() - 1.0) < 0.02
    r = _f32(syn.router_host(w.with_(E=64), 0)).astype(np.float64)
    assert abs(r.std() - 0.02) < 5e-4


def test_overlap_routing_statistic(syn):
    r = syn.overlap_routing(E=512, K=4, tokens=256, layers=24, p=0.27, seed=0)
    assert r.shape == (256, 24, 4)
    assert r.min() >= 0 and r.max() < 512
    for t in range(0, 256, 17):
        for l in range(24):
            assert len(set(r[t, l].tolist())) == 4
    ov = syn.measured_overlap(r)
    assert abs(ov - 0.27) < 0.02, ov


def test_zipf_routing(syn):
    r = syn.zipf_routing(E=512, K=4, B=32, steps=50, s=1.1, seed=0)
    assert r.shape == (50, 32, 4)
    for st in range(50):
        for b in range(32):
            assert len(set(r[st, b].tolist())) == 4
    distinct = [len(set(r[st].ravel().tolist())) for st in range(50)]
    assert 40 < np.mean(distinct) < 90
    # popularity is skewed: the most used expert is far above uniform
    counts = np.bincount(r.ravel(), minlength=512)
    assert counts.max() > 10 * counts.sum() / 512
