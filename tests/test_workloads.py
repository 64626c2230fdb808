"""The seeded input recipe (host only, small grids of each workload's recipe):
deterministic draws, the stated shapes and types, Q and K sharing one smooth
positional field per head while V does not, and the sink and near-uniform
heads of the stress workload."""
import math

import numpy as np
import torch

from block_sparse_attention_softmax_b200.workloads import (
    FLAT_HEAD_FRAC, FLAT_Q_GAIN, POS_AMPLITUDE, SINK_GAIN, SINK_KEYS, WORKLOADS, make_inputs)


def _small(name, grid=(3, 6, 8)):
    return WORKLOADS[name].with_n(grid)


def test_draws_are_seeded_and_shaped():
    wl = _small("wan14b_720p")
    a, b = make_inputs(wl), make_inputs(wl)
    for key in ("q", "k", "v", "alpha"):
        assert torch.equal(a[key], b[key]), key
    c = make_inputs(wl, seed=wl.seed + 1)
    assert not torch.equal(a["q"], c["q"])
    for key in ("q", "k", "v"):
        t = a[key]
        assert t.shape == (wl.B, wl.H, wl.N, wl.d) and t.dtype == torch.bfloat16 and t.is_contiguous()
    al = a["alpha"]
    assert al.shape == (wl.H, wl.d) and al.dtype == torch.float32
    assert float(al.min()) >= 0.0 and float(al.max()) < 1.0
    assert make_inputs(_small("wan13b_480p"))["alpha"] is None


def test_q_and_k_share_the_positional_field():
    """Q = Z_q + A P and K = Z_k + A P with unit-variance P: corr(Q, K) is
    A^2 / (1 + A^2) per element, V is independent of both."""
    wl = _small("wan13b_480p", (7, 10, 12))
    x = make_inputs(wl)
    q, k, v = (x[n].float().reshape(-1).numpy() for n in ("q", "k", "v"))
    want = POS_AMPLITUDE ** 2 / (1.0 + POS_AMPLITUDE ** 2)
    assert abs(np.corrcoef(q, k)[0, 1] - want) < 0.05
    assert abs(np.corrcoef(q, v)[0, 1]) < 0.02
    assert abs(q.var() - (1.0 + POS_AMPLITUDE ** 2)) < 0.3
    assert abs(v.var() - 1.0) < 0.05
    # i.i.d. workload: no shared component
    t = make_inputs(WORKLOADS["tiny"])
    assert abs(np.corrcoef(t["q"].float().reshape(-1), t["k"].float().reshape(-1))[0, 1]) < 0.02


def test_sink_keys_and_near_uniform_heads():
    wl = _small("sink_skew", (3, 6, 8))
    x = make_inputs(wl)
    flat = x["flat_heads"]
    assert len(flat) == round(FLAT_HEAD_FRAC * wl.H)
    base = math.sqrt(1.0 + POS_AMPLITUDE ** 2)             # per-element std of Q and K
    for h in range(wl.H):
        kn = x["k"][0, h].float().norm(dim=1)
        top = torch.topk(kn, SINK_KEYS + 1).values
        # exactly SINK_KEYS keys carry the gain
        assert float(top[SINK_KEYS - 1]) > 0.5 * SINK_GAIN * base * math.sqrt(wl.d)
        assert float(top[SINK_KEYS]) < 2.0 * base * math.sqrt(wl.d)
        q_std = float(x["q"][0, h].float().std())
        if h in flat:
            assert abs(q_std - FLAT_Q_GAIN * base) < 0.2 * FLAT_Q_GAIN * base
        else:
            assert abs(q_std - base) < 0.2 * base
