"""Pins of the oracle's routing and permutation against hand-worked cases,
brute force and invariants (no GPU)."""
import itertools

import numpy as np
import pytest
import scipy.special

from oracle import moe_oracle as O


def test_route_golden(golden):
    g = golden("route_cases.json")
    for case in g["cases"]:
        L = np.array([case["logits"]], dtype=np.float32)
        idx, w, w64 = O.route(L, case["k"])
        assert idx[0].tolist() == case["idx"], case["name"]
        np.testing.assert_allclose(w[0], case["w"], rtol=1e-6, atol=0, err_msg=case["name"])


def _topk_by_definition(l, k):
    """The unique k-subset S with: every i in S beats every j outside S, where i
    beats j iff l_i > l_j or (l_i == l_j and i < j). Found by enumerating all subsets."""
    E = len(l)

    def beats(i, j):
        return l[i] > l[j] or (l[i] == l[j] and i < j)

    winners = [S for S in itertools.combinations(range(E), k)
               if all(beats(i, j) for i in S for j in range(E) if j not in S)]
    assert len(winners) == 1
    S = list(winners[0])
    # slots ordered so that each slot beats the next
    for a in range(len(S)):
        for b in range(a + 1, len(S)):
            if beats(S[b], S[a]):
                S[a], S[b] = S[b], S[a]
    return S


@pytest.mark.parametrize("E,k", [(3, 1), (4, 2), (5, 3), (6, 2), (7, 3), (6, 6)])
def test_route_brute_force_with_ties(E, k):
    rng = np.random.default_rng(E * 10 + k)
    L = rng.integers(0, 3, size=(200, E)).astype(np.float32)  # many ties
    idx, w, _ = O.route(L, k)
    for t in range(L.shape[0]):
        assert idx[t].tolist() == _topk_by_definition(L[t].tolist(), k)


def test_route_weights_properties():
    rng = np.random.default_rng(1)
    L = rng.standard_normal((500, 16), dtype=np.float32)
    for k in (1, 2, 4, 8, 16):
        idx, w, w64 = O.route(L, k)
        assert np.all(np.abs(w64.sum(axis=1) - 1.0) <= 1e-12)
        assert np.all(np.abs(w.astype(np.float64).sum(axis=1) - 1.0) <= 1e-6)
        assert np.all(np.diff(w64, axis=1) <= 0)  # slots in descending weight
        if k == 16:
            # k = E: the renormalised weights are the softmax itself
            ref = scipy.special.softmax(L.astype(np.float64), axis=1)
            np.testing.assert_allclose(np.take_along_axis(ref, idx.astype(np.int64), 1), w64,
                                       rtol=1e-12)
        else:
            # renormalised = softmax restricted to the chosen experts
            sel = np.take_along_axis(L.astype(np.float64), idx.astype(np.int64), 1)
            np.testing.assert_allclose(scipy.special.softmax(sel, axis=1), w64, rtol=1e-12)


def test_route_token_permutation_invariance():
    rng = np.random.default_rng(2)
    L = rng.standard_normal((300, 12), dtype=np.float32)
    perm = rng.permutation(300)
    i1, w1, _ = O.route(L, 3)
    i2, w2, _ = O.route(L[perm], 3)
    assert (i1[perm] == i2).all() and (w1[perm] == w2).all()


def test_permute_golden(golden):
    g = golden("permute_cases.json")
    for case in g["cases"]:
        p = O.permute(np.array(case["topk_idx"]), case["E"], case["BM"])
        assert p["cnt"].tolist() == case["cnt"], case["name"]
        assert p["off"].tolist() == case["off"], case["name"]
        assert p["row_src"].tolist() == case["row_src"], case["name"]
        assert p["slot_row"].tolist() == case["slot_row"], case["name"]


@pytest.mark.parametrize("T,E,k,BM", [(1, 4, 1, 128), (37, 8, 2, 8), (200, 16, 4, 16), (64, 60, 4, 1),
                                      (513, 128, 8, 128)])
def test_permute_invariants_and_brute_force(T, E, k, BM):
    rng = np.random.default_rng(T + E)
    L = rng.standard_normal((T, E), dtype=np.float32)
    idx, _, _ = O.route(L, k)
    p = O.permute(idx, E, BM)
    cnt, off, row_src, slot_row = p["cnt"], p["off"], p["row_src"], p["slot_row"]
    assert (cnt == np.bincount(idx.ravel(), minlength=E)).all()
    assert off[0] == 0 and (np.diff(off) % BM == 0).all()
    assert (np.diff(off) == -(-cnt // BM) * BM).all()
    valid = row_src >= 0
    assert valid.sum() == T * k
    # bijection between valid rows and assignments
    assert sorted(row_src[valid].tolist()) == list(range(T * k))
    assert (row_src[slot_row] == np.arange(T * k)).all()
    # brute force: a plain sort by (expert, token) gives the rows without padding
    order = sorted(range(T * k), key=lambda a: (idx.ravel()[a], a // k))
    assert row_src[valid].tolist() == order
    for e in range(E):
        blk = row_src[off[e]:off[e + 1]]
        assert (blk[:cnt[e]] >= 0).all() and (blk[cnt[e]:] == -1).all()
        assert (idx.ravel()[blk[:cnt[e]]] == e).all()
        assert (np.diff(blk[:cnt[e]] // k) > 0).all()  # ascending tokens


# ---------------------------------------------------------------------------
# router logits (the router GEMM ahead of the routing)
# ---------------------------------------------------------------------------

def test_router_logits_one_hot_rows_select_weight_columns():
    rng = np.random.default_rng(7)
    E, H = 5, 12
    w = rng.standard_normal((E, H))
    x = np.zeros((H, H))
    x[np.arange(H), np.arange(H)] = 1.0  # token h is the unit vector e_h
    np.testing.assert_array_equal(O.router_logits(x, w), w.T)


def test_router_logits_brute_force_and_linearity():
    rng = np.random.default_rng(8)
    T, E, H = 4, 3, 6
    x = rng.standard_normal((T, H))
    w = rng.standard_normal((E, H))
    L = O.router_logits(x, w)
    for t in range(T):
        for e in range(E):
            s = 0.0
            for h in range(H):
                s += x[t, h] * w[e, h]
            assert abs(L[t, e] - s) < 1e-12
    x2 = rng.standard_normal((T, H))
    np.testing.assert_allclose(O.router_logits(2.0 * x - 3.0 * x2, w), 2.0 * L - 3.0 * O.router_logits(x2, w),
                               rtol=1e-12, atol=1e-12)
    # a transposed weight matrix cannot be applied, and swapped operands give E x T
    assert O.router_logits(x, w).shape == (T, E)
