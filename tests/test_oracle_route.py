"""Pins of the oracle's router against brute force, a library top-k and
invariants (TransformerEngine PR "DeepSeekV3Layer", Description, DeepSeekV3MoE
bullet: sigmoid router, aux-loss-free bias, grouped top-k)."""

import itertools
import math
import os

import numpy as np
import pytest

from oracle import moe_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def brute_route(logits, bias, G, g, k, rsf):
    """Enumerate every group subset and every expert subset; keep the best sum.

    A group's score is the best pair sum inside it; the kept groups are the
    g-subset with the largest total score; the experts are the k-subset of the
    kept groups' experts with the largest total biased score.  The first
    subset in lexicographic order wins a tie, which prefers lower indices.
    """
    T, E = logits.shape
    gs = E // G
    sets, gates = [], []
    for t in range(T):
        s = [1.0 / (1.0 + math.exp(-float(l))) for l in logits[t]]
        b = [s[e] + float(bias[e]) for e in range(E)]
        gsc = [max(b[i] + b[j] for i, j in itertools.combinations(range(q * gs, (q + 1) * gs), 2))
               for q in range(G)]
        best = None
        for sub in itertools.combinations(range(G), g):
            v = sum(gsc[q] for q in sub)
            if best is None or v > best[0]:
                best = (v, sub)
        elig = [e for q in best[1] for e in range(q * gs, (q + 1) * gs)]
        bestE = None
        for sub in itertools.combinations(elig, k):
            v = sum(b[e] for e in sub)
            if bestE is None or v > bestE[0]:
                bestE = (v, sub)
        chosen = list(bestE[1])
        tot = sum(s[e] for e in chosen)
        sets.append(chosen)
        gates.append({e: s[e] / tot * rsf for e in chosen})
    return sets, gates


@pytest.mark.parametrize("E,G,g,k", [(8, 4, 2, 2), (12, 3, 2, 3), (16, 4, 2, 4), (8, 2, 1, 3)])
def test_route_matches_brute_force(E, G, g, k):
    rng = np.random.default_rng(1000 + E * 31 + G * 7 + g * 3 + k)
    n = 0
    for trial in range(60):
        T = 5
        logits = rng.normal(0, 1.0, (T, E))
        bias = rng.uniform(-0.1, 0.1, E)
        r = O.route(logits, bias, G, g, k, 2.5)
        sets, gates = brute_route(logits, bias, G, g, k, 2.5)
        for t in range(T):
            assert sorted(r["idx"][t].tolist()) == sorted(sets[t])
            for j, e in enumerate(r["idx"][t]):
                assert abs(r["w"][t, j] - gates[t][int(e)]) <= 1e-12
            n += 1
    assert n == 300


def test_route_ties_go_to_lower_index():
    # Exact ties in b between experts and between groups.
    E, G, g, k = 8, 4, 2, 2
    logits = np.zeros((3, E))
    bias = np.zeros(E)
    # token 0: all equal -> groups 0,1 and experts 0,1
    # token 1: experts 5 and 7 tie for the top; groups 2 and 3 tie
    logits[1, 5] = logits[1, 7] = 2.0
    # token 2: expert 6 best, then a tie between 1 and 2 (groups 0 and 1)
    logits[2, 6] = 3.0
    logits[2, 1] = logits[2, 2] = 1.0
    r = O.route(logits, bias, G, g, k, 1.0)
    sets, _ = brute_route(logits, bias, G, g, k, 1.0)
    assert r["idx"][0].tolist() == [0, 1]
    assert r["idx"][1].tolist() == [5, 7]
    assert r["idx"][2].tolist() == [6, 1]
    for t in range(3):
        assert sorted(r["idx"][t].tolist()) == sorted(sets[t])


def test_single_group_is_plain_topk():
    rng = np.random.default_rng(7)
    T, E, k = 200, 64, 6
    logits = rng.normal(0, 1, (T, E))
    bias = rng.uniform(-0.1, 0.1, E)
    r = O.route(logits, bias, 1, 1, k, 2.5)
    b = 1.0 / (1.0 + np.exp(-logits)) + bias
    ref = np.argsort(-b, axis=1)[:, :k]
    assert np.array_equal(r["idx"], ref)


def test_route_invariants_large():
    rng = np.random.default_rng(11)
    T, E, G, g, k, rsf = 512, 256, 8, 4, 8, 2.5
    logits = rng.normal(0, 1, (T, E))
    bias = rng.uniform(-0.1, 0.1, E)
    r = O.route(logits, bias, G, g, k, rsf)
    idx, w, b = r["idx"], r["w"], r["b"]
    assert np.all(np.abs(w.sum(axis=1) - rsf) <= 1e-12)
    gs = E // G
    for t in range(T):
        sel = idx[t]
        assert len(set(sel.tolist())) == k
        grp = b[t].reshape(G, gs)
        gscore = np.sort(grp, axis=1)[:, -2:].sum(axis=1)
        kept = set(np.argsort(-gscore, kind="stable")[:g].tolist())
        assert all(int(e) // gs in kept for e in sel)
        elig = [e for q in kept for e in range(q * gs, (q + 1) * gs)]
        rest = [e for e in elig if e not in set(sel.tolist())]
        assert b[t, sel].min() >= b[t, rest].max()
        # listed by b descending
        assert np.all(np.diff(b[t, sel]) <= 0)


def test_gates_use_unbiased_scores():
    # A large bias changes the selection but not the gate ratio.
    logits = np.array([[0.0, 1.0, 2.0, 3.0]])
    bias = np.array([10.0, 0.0, 0.0, 0.0])
    r = O.route(logits, bias, 1, 1, 2, 1.0)
    assert r["idx"][0].tolist() == [0, 3]
    s0, s3 = 0.5, 1.0 / (1.0 + math.exp(-3.0))
    assert abs(r["w"][0, 0] - s0 / (s0 + s3)) < 1e-15


def test_margins_match_brute_force():
    rng = np.random.default_rng(5)
    T, E, G, g, k = 50, 16, 4, 2, 4
    logits = rng.normal(0, 1, (T, E))
    bias = rng.uniform(-0.1, 0.1, E)
    r = O.route(logits, bias, G, g, k, 1.0)
    gs = E // G
    for t in range(T):
        b = r["b"][t]
        gsc = sorted((max(b[i] + b[j] for i, j in itertools.combinations(range(q * gs, (q + 1) * gs), 2))
                      for q in range(G)), reverse=True)
        assert abs(r["group_margin"][t] - (gsc[g - 1] - gsc[g])) < 1e-12
        kept = np.argsort(-np.array([max(b[i] + b[j] for i, j in
                                          itertools.combinations(range(q * gs, (q + 1) * gs), 2))
                                      for q in range(G)]), kind="stable")[:g]
        elig = sorted((b[e] for q in kept for e in range(q * gs, (q + 1) * gs)), reverse=True)
        assert abs(r["expert_margin"][t] - (elig[k - 1] - elig[k])) < 1e-12


def _read_golden(name):
    rows = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            key, val = line.split("=", 1)
            rows[key.strip()] = [float(v) for v in val.split()]
    return rows


def test_hand_worked_routing_example():
    """A routing example worked by hand (tests/golden/route_hand_example.txt)."""
    d = _read_golden("route_hand_example.txt")
    b = np.array(d["b"])
    E = len(b)
    G, g, k = int(d["n_group"][0]), int(d["topk_group"][0]), int(d["top_k"][0])
    # b = s + bias with bias = 0 -> logits = logit(b)
    logits = np.log(b / (1 - b))[None, :]
    r = O.route(logits, np.zeros(E), G, g, k, d["rsf"][0])
    assert r["idx"][0].tolist() == [int(v) for v in d["expected_idx"]]
    assert np.allclose(r["w"][0], d["expected_w"], atol=1e-12)
    assert np.allclose(r["group_score"][0], d["expected_group_score"], atol=1e-12)
