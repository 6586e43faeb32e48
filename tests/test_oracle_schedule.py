"""Pins for the oracle's schedule Phi (CPU only).

The oracle's counting sort is checked against (a) schedules worked by hand
from the placement formula, (b) two other oracle placements computed in a
different way (closed form with a sequential rank scan; explicit round-robin
queue simulation), (c) a pure-Python round-robin written here, independently,
on exhaustive tiny inputs and random small ones, (d) the invariants the pages
fix, and (e) the pages' worked numbers.
"""
import itertools
import json
import os

import numpy as np
import pytest

import oracle
from combine_top_route_counting_b200 import inputs

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def py_round_robin(ids, P, N, k, E, pad):
    """Independent restatement: per expert, visit peers 0..P-1 in rounds, taking the
    next route (ascending q) of every peer that still has one; pad with (-1,-1)."""
    R = N * k
    per = [[[] for _ in range(P)] for _ in range(E)]
    for r in range(P):
        for q in range(R):
            per[ids[r][q // k][q % k]][r].append(q)
    phi, offsets = [], []
    route_row = np.zeros((P, N, k), np.int64)
    for l in range(E):
        offsets.append(len(phi))
        queues = [list(per[l][r]) for r in range(P)]
        while any(queues):
            for r in range(P):
                if queues[r]:
                    q = queues[r].pop(0)
                    route_row[r, q // k, q % k] = len(phi)
                    phi.append((r, q // k))
        while (len(phi) - offsets[-1]) % pad:
            phi.append((-1, -1))
    offsets.append(len(phi))
    return np.array(phi, np.int64).reshape(-1, 2), np.array(offsets), route_row


def check_invariants(s, ids, P, N, k, E, pad):
    phi, off, cnt, rr = s["phi"], s["offsets"], s["counts"], s["route_row"]
    ids = np.asarray(ids).reshape(P, N, k)
    T = np.zeros(E, np.int64)
    for l in range(E):
        T[l] = (ids == l).sum()
        assert cnt[l].sum() == T[l]
        for r in range(P):
            assert cnt[l, r] == (ids[r] == l).sum()
    Tp = (T + pad - 1) // pad * pad
    assert (Tp % pad == 0).all()
    assert off[0] == 0 and (np.diff(off) == Tp).all(), "offsets = prefix sums of padded totals"
    assert phi.shape[0] == off[E]
    # every route appears exactly once, at its route_row, and nothing else is non-pad
    seen = np.zeros(phi.shape[0], np.int64)
    for r in range(P):
        for i in range(N):
            for j in range(k):
                row = rr[r, i, j]
                l = ids[r, i, j]
                assert off[l] <= row < off[l] + T[l]
                assert tuple(phi[row]) == (r, i)
                seen[row] += 1
    for l in range(E):
        assert (seen[off[l]:off[l] + T[l]] == 1).all()
        assert (seen[off[l] + T[l]:off[l + 1]] == 0).all()
        assert (phi[off[l] + T[l]:off[l + 1]] == -1).all()
        # rows of one peer inside a segment appear in ascending (token, slot)
        seg = phi[off[l]:off[l] + T[l]]
        for r in range(P):
            toks = seg[seg[:, 0] == r][:, 1]
            assert (np.diff(toks) >= 0).all()
    assert s["reads"] == 2 * P * N * k, "each route is read twice: count and scatter"


def test_handworked_golden():
    cases = json.load(open(os.path.join(GOLD, "schedule_handworked.json")))["cases"]
    for c in cases:
        P, N, k, E, pad = c["P"], c["N"], c["k"], c["E"], c["pad"]
        ids = np.array(c["ids"], np.int32)
        s = oracle.schedule(ids, P, N, k, E, pad)
        assert s["phi"].tolist() == c["phi"]
        assert s["offsets"].tolist() == c["offsets"]
        assert s["counts"].tolist() == c["counts"]
        assert s["route_row"].tolist() == c["route_row"]
        check_invariants(s, ids, P, N, k, E, pad)


def _three_way(ids, P, N, k, E, pad):
    s = oracle.schedule(ids, P, N, k, E, pad)
    off_c, rr_c = oracle.place_closed_form(ids, P, N, k, E, pad)
    off_q, rr_q, phi_q = oracle.place_queue_sim(ids, P, N, k, E, pad)
    assert (s["offsets"] == off_c).all() and (s["offsets"] == off_q).all()
    assert (s["route_row"] == rr_c).all() and (s["route_row"] == rr_q).all()
    assert (s["phi"] == phi_q).all()
    return s


@pytest.mark.parametrize("P,N,k,E", [(2, 2, 1, 3), (3, 2, 1, 2), (1, 3, 1, 3), (2, 1, 2, 3)])
def test_exhaustive_tiny(P, N, k, E):
    """All id patterns of tiny shapes: counting sort == closed form == queue sim == python."""
    per_token = [p for p in itertools.permutations(range(E), k)]
    n = 0
    for combo in itertools.product(per_token, repeat=P * N):
        ids = np.array(combo, np.int32).reshape(P, N, k)
        for pad in (1, 2, 4):
            s = _three_way(ids, P, N, k, E, pad)
            phi, off, rr = py_round_robin(ids.tolist(), P, N, k, E, pad)
            assert (s["phi"] == phi).all() and (s["offsets"] == off).all()
            assert (s["route_row"] == rr).all()
            check_invariants(s, ids, P, N, k, E, pad)
        n += 1
    assert n == len(per_token) ** (P * N)


def test_sweep_945_three_way():
    """The randomized sweep (P 1..8, E 1..64, N 1..512, k 1..min(8,E)), pad 256."""
    n = 0
    for P, N, E, k, ids in inputs.sweep_cases():
        _three_way(ids.numpy(), P, N, k, E, 256)
        n += 1
    assert n == 945


def test_sweep_python_and_invariants():
    for c, (P, N, E, k, ids) in enumerate(inputs.sweep_cases(n_cases=60, seed=7, max_N=48)):
        idn = ids.numpy()
        s = oracle.schedule(idn, P, N, k, E, 256)
        phi, off, rr = py_round_robin(idn.tolist(), P, N, k, E, 256)
        assert (s["phi"] == phi).all() and (s["offsets"] == off).all()
        assert (s["route_row"] == rr).all()
        check_invariants(s, idn, P, N, k, E, 256)


def test_chunking_does_not_change_phi():
    """More routes than logical threads (chunks of several routes per thread) and
    fewer: the result must equal the round-robin definition either way."""
    for (P, N, k, E) in [(2, 700, 3, 5), (3, 1500, 1, 4), (1, 5, 2, 2)]:
        ids = inputs.make_ids_uniform(P, N, E, k, seed=P * 1000 + N).numpy()
        s = oracle.schedule(ids, P, N, k, E, 256)
        phi, off, rr = py_round_robin(ids.tolist(), P, N, k, E, 256)
        assert (s["phi"] == phi).all() and (s["route_row"] == rr).all()


def test_empty_and_degenerate():
    # no tokens: every segment is empty
    ids = np.zeros((3, 0, 2), np.int32)
    s = oracle.schedule(ids, 3, 0, 2, 4, 256)
    assert s["offsets"].tolist() == [0, 0, 0, 0, 0] and s["phi"].shape == (0, 2)
    # one expert takes everything
    ids = np.zeros((2, 300, 1), np.int32)
    s = oracle.schedule(ids, 2, 300, 1, 1, 256)
    assert s["offsets"].tolist() == [0, 768]
    assert s["phi"][:600:2, 0].tolist() == [0] * 300  # peers alternate
    assert s["phi"][1:600:2, 0].tolist() == [1] * 300
    check_invariants(s, ids, 2, 300, 1, 1, 256)
    # k = E: every token uses every expert
    ids = np.tile(np.arange(3, dtype=np.int32)[::-1], (1, 4, 1)).reshape(1, 4, 3)
    s = oracle.schedule(ids, 1, 4, 3, 3, 256)
    check_invariants(s, ids, 1, 4, 3, 3, 256)
    # an out-of-range id is rejected
    with pytest.raises(ValueError):
        oracle.schedule(np.array([[[5]]], np.int32), 1, 1, 1, 2, 256)


def test_worked_numbers_route_reads_and_counters():
    w = json.load(open(os.path.join(GOLD, "worked_numbers.json")))["route_reads"]
    wl = inputs.WORKLOADS["sched"]
    assert (wl.P, wl.N, wl.E, wl.k) == (w["P"], w["tokens_per_peer"], w["E"], w["k"])
    ids = inputs.make_sched_ids(wl).numpy()
    s = oracle.schedule(ids, wl.P, wl.N, wl.k, wl.E, 256)
    R = wl.N * wl.k
    assert s["reads"] == w["new_reads"] == 2 * wl.P * R
    assert s["threads"] == w["threads_per_peer"]
    # counters of one destination rank: its E/P local experts x P peers x 1024 threads
    assert s["counter_words"] // wl.P == w["counters_per_rank"] == wl.E * 1024
    # the old per-(expert, peer) rescanning scheduler: R*(2E + P) reads
    assert R * (2 * wl.E + wl.P) == w["old_reads"]
    assert w["old_reads"] // w["new_reads"] == w["cut"]
    check_invariants_light(s, ids, wl)


def check_invariants_light(s, ids, wl):
    P, N, k, E = wl.P, wl.N, wl.k, wl.E
    phi, off, rr = s["phi"], s["offsets"], s["route_row"]
    assert ((np.diff(off)) % 256 == 0).all()
    flat = rr.reshape(-1)
    assert len(np.unique(flat)) == flat.size, "every route has its own row"
    r_idx = np.repeat(np.arange(P), N * k)
    i_idx = np.tile(np.repeat(np.arange(N), k), P)
    assert (phi[flat, 0] == r_idx).all() and (phi[flat, 1] == i_idx).all()
    nonpad = (phi[:, 0] >= 0).sum()
    assert nonpad == P * N * k


def test_wave_floor():
    w = json.load(open(os.path.join(GOLD, "worked_numbers.json")))["wave_floor"]
    assert oracle.wave_floor(w["H"], w["I"], w["C"]) == w["T_min"]
    assert min(2 * w["I"], w["H"]) == w["min_2I_H"]
    # floors of the other workloads; the bound is the smallest T meeting both tile counts
    for H, I in [(256, 128), (2048, 1024), (7168, 2048)]:
        T = oracle.wave_floor(H, I, 148)
        assert T * 2 * I >= 2 * 148 * 128 * 256 and T * H >= 2 * 148 * 128 * 256
        assert (T - 1) * min(2 * I, H) < 2 * 148 * 128 * 256
    assert oracle.wave_floor(256, 128, 148) == 37888
    assert oracle.wave_floor(2048, 1024, 148) == 4736
