"""Pins of the oracle's permute maps (TransformerEngine PR "DeepSeekV3Layer",
Performance, "NCCL EP local permute": expert-major staging with zero-filled
padding; its reduce is the inverse map).  Checked against an independent
sort-based construction and against the invariants of a permutation."""

import numpy as np
import pytest

from oracle import moe_oracle as O


def _random_idx(rng, T, E, k):
    return np.stack([rng.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32)


def sort_based_maps(idx, E, P):
    """The same maps from a stable argsort of the flat expert ids."""
    T, k = idx.shape
    flat = idx.reshape(-1)
    order = np.argsort(flat, kind="stable")
    counts = np.bincount(flat, minlength=E)
    padded = -(-counts // P) * P
    offsets = np.concatenate([[0], np.cumsum(padded)])
    first = np.concatenate([[0], np.cumsum(counts)])[:-1]
    token_row = np.empty(T * k, dtype=np.int64)
    ranks = np.arange(T * k) - first[flat[order]]
    token_row[order] = offsets[flat[order]] + ranks
    row_token = np.full(offsets[-1], -1)
    row_token[token_row] = np.arange(T * k) // k
    return counts, offsets, row_token, token_row


@pytest.mark.parametrize("T,E,k,P", [(64, 16, 4, 8), (300, 64, 6, 128), (7, 8, 3, 1), (1, 4, 4, 16)])
def test_permute_matches_sort_construction(T, E, k, P):
    rng = np.random.default_rng(T * 13 + E)
    idx = _random_idx(rng, T, E, k)
    m = O.permute_maps(idx, E, P)
    c, off, rt, tr = sort_based_maps(idx, E, P)
    assert np.array_equal(m["counts"], c)
    assert np.array_equal(m["offsets"], off)
    assert np.array_equal(m["row_token"], rt)
    assert np.array_equal(m["token_row"], tr)


def test_permute_invariants():
    rng = np.random.default_rng(9)
    T, E, k, P = 500, 32, 6, 16
    idx = _random_idx(rng, T, E, k)
    m = O.permute_maps(idx, E, P)
    off, rt, tr, cnt = m["offsets"], m["row_token"], m["token_row"], m["counts"]
    assert cnt.sum() == T * k
    assert np.all(np.diff(off) >= 0) and np.all(off % P == 0)
    # unpermute(permute) is the identity on (t, j)
    assert np.array_equal(rt[tr], np.arange(T * k) // k)
    # every valid row is used exactly once
    assert np.array_equal(np.sort(tr), np.sort(np.nonzero(rt >= 0)[0]))
    for e in range(E):
        seg = rt[off[e]:off[e + 1]]
        toks = seg[:cnt[e]]
        assert np.all(seg[cnt[e]:] == -1)
        assert np.all(np.diff(toks) > 0)
        assert set(toks.tolist()) == set(np.nonzero((idx == e).any(axis=1))[0].tolist())
    x = rng.normal(size=(T, 8))
    rows = O.gather_rows(x, rt)
    assert np.all(rows[rt < 0] == 0)
    assert np.array_equal(rows[tr], np.repeat(x, k, axis=0))


def test_permute_empty_experts():
    idx = np.array([[0, 1], [0, 1], [1, 0]], dtype=np.int32)
    m = O.permute_maps(idx, 5, 4)
    assert m["counts"].tolist() == [3, 3, 0, 0, 0]
    assert m["offsets"].tolist() == [0, 4, 8, 8, 8, 8]
    assert m["row_token"].tolist() == [0, 1, 2, -1, 0, 1, 2, -1]
    assert m["token_row"].tolist() == [0, 4, 1, 5, 6, 2]
