"""The seeded input recipe (CPU only): reproducible seeds, shapes and dtypes,
the stated distributions, and the Zipf workload's skew and empty experts."""
import numpy as np
import torch

import oracle
from combine_top_route_counting_b200 import inputs


def test_generators_are_seeded_and_shaped():
    w = inputs.WORKLOADS["tiny"]
    a, b = inputs.make_logits(w), inputs.make_logits(w)
    assert torch.equal(a, b) and a.shape == (w.n_tokens, w.E) and a.dtype == torch.float32
    x = inputs.make_x(w)
    assert torch.equal(x, inputs.make_x(w)) and x.shape == (w.n_tokens, w.H)
    assert x.dtype == torch.bfloat16
    W1, W3, W2 = inputs.make_weights(w)
    assert W1.shape == (w.E, w.H, w.I) and W3.shape == (w.E, w.H, w.I) and W2.shape == (w.E, w.I, w.H)
    assert not torch.equal(W1, W3)                     # separate streams
    d = inputs.make_dout(w)
    assert d.shape == (w.n_tokens, w.H) and not torch.equal(d, x)
    # different workloads draw different numbers
    assert not torch.equal(inputs.make_logits(inputs.WORKLOADS["tiny_bwd"])[:4, :4], a[:4, :4])


def test_distributions_match_the_recipe():
    w = inputs.WORKLOADS["mid"]
    lg = inputs.make_logits(w)
    assert abs(lg.mean().item()) < 0.01 and abs(lg.std().item() - 1) < 0.01
    x = inputs.make_x(w).float()
    assert abs(x.std().item() - 1) < 0.01
    W1, _, W2 = inputs.make_weights(w)
    assert abs(W1.float().std().item() - 0.02) < 2e-4 and abs(W2.float().std().item() - 0.02) < 2e-4


def test_uniform_ids_are_distinct_per_token():
    ids = inputs.make_ids_uniform(3, 200, 40, 8, seed=1).numpy()
    assert ids.shape == (3, 200, 8) and ids.min() >= 0 and ids.max() < 40
    flat = ids.reshape(-1, 8)
    assert all(len(set(r)) == 8 for r in flat)
    counts = np.bincount(flat.reshape(-1), minlength=40)
    assert counts.min() > 0.6 * counts.mean()          # roughly uniform


def test_zipf_workload_skew_and_empty_experts():
    w = inputs.WORKLOADS["zipf"]
    ids, _, _ = oracle.route_topk(inputs.make_logits(w), w.k)
    counts = np.sort(np.bincount(ids.reshape(-1), minlength=w.E))[::-1]
    share = counts / ids.size
    assert 0.09 < share[0] < 0.14                       # ~11.5 % on the top expert
    assert 0.27 < share[:4].sum() < 0.36                # ~31.6 % on the top 4
    empty = inputs.empty_experts(w)
    assert len(empty) == w.n_empty == 8
    assert not np.isin(ids, empty).any()
    assert (counts[-8:] == 0).all()
