"""Pattern tools (IndexCache paper, Appendix Figure 4: pairwise top-k overlap
between layers; Table 5: a pattern searched from that similarity; Abstract:
greedy removal of indexers by a loss): the oracle pinned to closed forms, and
the library's host-side search functions checked against the oracle. No GPU
needed: ic_search_pattern and ic_greedy_pattern run on the host."""

import itertools

import numpy as np
import pytest

import oracle


# --------------------------------------------------------------------------- oracle pins
def test_oracle_overlap_closed_forms():
    rng = np.random.default_rng(0)
    n_k, topk = 97, 16
    a = np.stack([rng.permutation(n_k)[:topk] for _ in range(8)]).astype(np.int32)
    # identical rows: every valid entry
    assert np.array_equal(oracle.topk_overlap(a, a, n_k), np.full(8, topk))
    # the same sets in another order
    b = np.stack([rng.permutation(r) for r in a]).astype(np.int32)
    assert np.array_equal(oracle.topk_overlap(a, b, n_k), np.full(8, topk))
    # disjoint sets
    c = ((a + n_k // 2) % n_k).astype(np.int32)
    lo = np.where(a < n_k // 2, a, -1).astype(np.int32)
    hi = np.where(c >= n_k // 2, c, -1).astype(np.int32)
    assert np.array_equal(oracle.topk_overlap(lo, hi, n_k), np.zeros(8))
    # padding and out-of-range entries never count
    pad = np.full_like(a, -1)
    assert np.array_equal(oracle.topk_overlap(a, pad, n_k), np.zeros(8))
    assert np.array_equal(oracle.topk_overlap(a + n_k, a + n_k, n_k), np.zeros(8))
    # a hand-checked example: {1,2,3} & {3,2,9} = 2; {5..8} & {8..5} = 4
    x = np.array([[1, 2, 3, -1], [5, 6, 7, 8]], np.int32)
    y = np.array([[3, 2, 9, -1], [8, 7, 6, 5]], np.int32)
    assert list(oracle.topk_overlap(x, y, 10)) == [2, 4]


def _block_matrix(starts, n):
    """R[l][f] = 1 when l and f lie in the same block (blocks begin at `starts`)."""
    block = np.zeros(n, int)
    for i, s in enumerate(starts):
        block[s:] = i
    return (block[:, None] == block[None, :]).astype(np.float64)


def test_oracle_search_closed_forms():
    n = 10
    # with one Full layer per block, every layer reuses its own block: score n
    starts = [0, 3, 7]
    R = _block_matrix(starts, n)
    pat, score = oracle.search_pattern(R, len(starts))
    assert pat == "".join("F" if l in starts else "S" for l in range(n))
    assert score == n
    # all Full: score = trace
    rng = np.random.default_rng(1)
    M = rng.random((n, n))
    pat, score = oracle.search_pattern(M, n)
    assert pat == "F" * n and score == pytest.approx(np.trace(M), abs=1e-12)
    # one Full layer: every layer reuses layer 0
    pat, score = oracle.search_pattern(M, 1)
    assert pat == "F" + "S" * (n - 1) and score == pytest.approx(M[:, 0].sum(), abs=1e-12)


def test_oracle_pattern_score_definition():
    rng = np.random.default_rng(2)
    M = rng.random((5, 5))
    # FSFSS: layer sources 0,0,2,2,2
    want = M[0, 0] + M[1, 0] + M[2, 2] + M[3, 2] + M[4, 2]
    assert oracle.pattern_score(M, "FSFSS") == pytest.approx(want, abs=1e-12)
    assert oracle.pattern_score(M, "SFFSS") == -np.inf


def test_oracle_greedy_additive_objective():
    # objective = sum of per-layer costs of the Shared layers: the greedy
    # search removes the cheapest layers first (a closed form)
    cost = np.array([9.0, 4.0, 1.5, 7.0, 0.5, 3.0, 2.5, 8.0])
    obj = lambda p: sum(cost[l] for l, c in enumerate(p) if c == "S")
    pat, v = oracle.greedy_pattern(len(cost), 3, obj)
    removed = sorted(range(1, len(cost)), key=lambda l: cost[l])[: len(cost) - 3]
    assert pat == "".join("S" if l in removed else "F" for l in range(len(cost)))
    assert v == pytest.approx(cost[removed].sum())


# --------------------------------------------------------------------------- library vs oracle (host)
@pytest.fixture(scope="module")
def ic():
    import dsa_indexer_reuse_b200 as m
    return m


@pytest.mark.parametrize("n,n_full", [(1, 1), (4, 2), (9, 3), (12, 4), (12, 11), (16, 5)])
def test_search_pattern_matches_exhaustive(ic, n, n_full):
    rng = np.random.default_rng(10 + n + n_full)
    R = rng.random((n, n))
    np.fill_diagonal(R, 1.0)
    got, gs = ic.search_pattern(R, n_full)
    want, ws = oracle.search_pattern(R, n_full)
    assert got == want
    assert gs == pytest.approx(ws, rel=1e-12)
    assert oracle.pattern_score(R, got) == pytest.approx(gs, rel=1e-12)


def test_search_pattern_block_structure(ic):
    n = 47
    starts = [0, 5, 11, 12, 20, 33, 40]
    R = _block_matrix(starts, n) * 0.9 + 0.05
    pat, _ = ic.search_pattern(R, len(starts))
    assert pat == "".join("F" if l in starts else "S" for l in range(n))


@pytest.mark.parametrize("n,n_full", [(6, 2), (10, 3), (12, 6)])
def test_greedy_pattern_matches_oracle(ic, n, n_full):
    rng = np.random.default_rng(n * 7 + n_full)
    R = rng.random((n, n))
    np.fill_diagonal(R, 1.0)
    # a non-additive objective: minus the overlap score of the pattern
    obj = lambda p: -oracle.pattern_score(R, p)
    got, gv = ic.greedy_pattern(n, n_full, obj)
    want, wv = oracle.greedy_pattern(n, n_full, obj)
    assert got == want
    assert gv == pytest.approx(wv, rel=1e-12)
    assert got.count("F") == n_full and got[0] == "F"


def test_pattern_tools_reject_bad_arguments(ic):
    R = np.eye(4)
    with pytest.raises(ic.IcError):
        ic.search_pattern(R, 0)
    with pytest.raises(ic.IcError):
        ic.search_pattern(R, 5)
    bad = R.copy()
    bad[1, 2] = np.nan
    with pytest.raises(ic.IcError):
        ic.search_pattern(bad, 2)
    with pytest.raises(ic.IcError):
        ic.greedy_pattern(4, 2, lambda p: float("inf"))
    with pytest.raises(ZeroDivisionError):
        ic.greedy_pattern(4, 2, lambda p: 1 / 0)


@pytest.mark.parametrize("n", [1, 4, 9])
def test_pattern_score_matches_oracle(ic, n):
    rng = np.random.default_rng(n)
    R = rng.random((n, n))
    for bits in itertools.product("FS", repeat=n - 1):
        pat = "F" + "".join(bits)
        assert ic.pattern_score(R, pat) == pytest.approx(oracle.pattern_score(R, pat), rel=1e-15, abs=1e-15)
    with pytest.raises(ic.IcError) as e:
        ic.pattern_score(R, "S" * n)
    assert e.value.code == 2
    with pytest.raises(ic.IcError):
        ic.pattern_score(R, "F" * (n + 1))
