"""GPU parity of the fused indexer + top-k (ic_indexer_topk) against the oracle.

Criteria:
  * small-integer inputs (every score exact in fp32): index sets bit-exact;
  * Gaussian inputs: recall >= 0.999 over all checked rows, and every key in
    the symmetric difference scores within 1e-3 (relative) of the oracle's
    k-th score of that row;
  * the output lists each set once, -1 padding last; the entry order is
    deterministic but unspecified (the 4-head tiny workload's lists are
    ascending; the 64-head paths emit the keys grouped by the warp that
    scored them, ascending within a group).
"""

import numpy as np
import pytest
import torch

from dsa_indexer_reuse_b200 import workloads as W
from gpu_util import canon, check_topk_tolerant, host_indexer, oracle_scores, oracle_topk, to_dev

pytestmark = pytest.mark.gpu


def run_gpu(ind, wl, topk=None, q_pos0=None):
    import dsa_indexer_reuse_b200 as ic
    d = to_dev(ind)
    idx = ic.indexer_topk(d["q_I"], d["w"], d["k_I"], topk or wl.topk, q_scale=d["q_scale"],
                          k_scale=d["k_scale"], q_pos0=wl.q_pos0 if q_pos0 is None else q_pos0)
    torch.cuda.synchronize()
    return idx.cpu().numpy().reshape(-1, topk or wl.topk)


def assert_ascending_then_padding(idx):
    for row in idx:
        v = row[row >= 0]
        n = len(v)
        assert (row[n:] == -1).all(), "padding must come last"
        assert (np.diff(v) > 0).all(), "valid entries must be strictly ascending"


def assert_distinct_then_padding(idx):
    for row in idx:
        v = row[row >= 0]
        n = len(v)
        assert (row[n:] == -1).all(), "padding must come last"
        assert len(np.unique(v)) == n, "valid entries must be distinct"


def test_tiny_int_exact(cuda_ok):
    wl = W.TINY_INT
    ind = W.indexer_inputs(wl, 0)
    got = run_gpu(ind, wl)
    ref, _ = oracle_topk(host_indexer(ind), wl)
    assert_ascending_then_padding(got)
    assert (got == canon(ref)).all()


@pytest.mark.parametrize("L,topk", [(1, 128), (130, 128), (700, 64), (1000, 1), (2049, 100)])
def test_tiny_int_shapes_exact(cuda_ok, L, topk):
    wl = W.TINY_INT.with_(n_q=L, n_k=L)
    ind = W.indexer_inputs(wl, 1, seed=L)
    got = run_gpu(ind, wl, topk=topk)
    ref, _ = oracle_topk(host_indexer(ind), wl, topk=topk)
    assert (got == canon(ref)).all()


def test_tiny_int_all_ties_and_negative_zero(cuda_ok):
    # w <= 0 everywhere: every score is -0.0 or negative; zero-score ties must
    # go to the lowest indices regardless of the sign of zero
    wl = W.TINY_INT.with_(n_q=600, n_k=600)
    ind = W.indexer_inputs(wl, 2)
    ind["w"] = -ind["w"].abs()
    got = run_gpu(ind, wl)
    ref, _ = oracle_topk(host_indexer(ind), wl)
    assert (got == canon(ref)).all()


def gaussian(wl, layer=0, seed=0):
    ind = W.indexer_inputs(wl, layer, seed=seed)
    return ind, host_indexer(ind)


@pytest.mark.parametrize("fp8", [False, True])
def test_gaussian_ragged_exact_oracle(cuda_ok, fp8):
    base = W.PREFILL_8K if not fp8 else W.PREFILL_200K
    wl = base.with_(n_q=1500, n_k=1500, topk=300)
    ind, ind_np = gaussian(wl, seed=3)
    got = run_gpu(ind, wl)
    ref, kth = oracle_topk(ind_np, wl)
    assert_distinct_then_padding(got)
    rows = np.arange(wl.n_q)
    sc = oracle_scores(ind_np, wl, rows)
    check_topk_tolerant(got, ref, sc, kth)


@pytest.mark.parametrize("fp8", [False, True])
def test_gaussian_topk2048(cuda_ok, fp8):
    base = W.PREFILL_8K if not fp8 else W.PREFILL_200K
    wl = base.with_(n_q=3000, n_k=3000)
    ind, ind_np = gaussian(wl, seed=4)
    got = run_gpu(ind, wl)
    rows = np.r_[0:40, 2040:2060, 2900:3000]
    ref, kth = oracle_topk(ind_np, wl, rows=rows)
    sc = oracle_scores(ind_np, wl, rows)
    check_topk_tolerant(got[rows], ref, sc, kth)


def test_batched_chunked_prefill(cuda_ok):
    # two sequences, 700 new queries appended after 900 cached keys
    wl = W.PREFILL_8K.with_(batch=2, n_q=700, n_k=1600, q_pos0=900, topk=256)
    ind, ind_np = gaussian(wl, seed=5)
    got = run_gpu(ind, wl)
    rows = np.r_[0:30, 690:730, 1370:1400]
    ref, kth = oracle_topk(ind_np, wl, rows=rows)
    sc = oracle_scores(ind_np, wl, rows)
    check_topk_tolerant(got[rows], ref, sc, kth)


@pytest.mark.parametrize("fp8,n_k", [(True, 20000), (False, 9000), (True, 1500)])
def test_decode_split_path(cuda_ok, fp8, n_k):
    base = W.DECODE_32X32K if fp8 else W.DECODE_32X32K.with_(qk_dtype=W.BF16, w_dtype=W.BF16)
    wl = base.with_(batch=5, n_k=n_k, q_pos0=n_k - 1)
    ind, ind_np = gaussian(wl, seed=6)
    got = run_gpu(ind, wl)
    ref, kth = oracle_topk(ind_np, wl)
    assert_distinct_then_padding(got)
    sc = oracle_scores(ind_np, wl, np.arange(wl.batch))
    check_topk_tolerant(got, ref, sc, kth)


def test_deterministic(cuda_ok):
    wl = W.PREFILL_8K.with_(n_q=2000, n_k=2000, topk=512)
    ind, _ = gaussian(wl, seed=7)
    a = run_gpu(ind, wl)
    b = run_gpu(ind, wl)
    assert (a == b).all()


def test_full_size_prefill_8k_sampled_rows(cuda_ok):
    wl = W.PREFILL_8K
    ind, ind_np = gaussian(wl, seed=0)
    got = run_gpu(ind, wl)
    rows = np.r_[0:8, 2047:2050, 4000:4004, 8180:8192]
    ref, kth = oracle_topk(ind_np, wl, rows=rows)
    sc = oracle_scores(ind_np, wl, rows)
    check_topk_tolerant(got[rows], ref, sc, kth)
    assert_distinct_then_padding(got[::97])


def test_full_size_decode_sampled(cuda_ok):
    wl = W.DECODE_32X32K
    ind, ind_np = gaussian(wl, seed=0)
    got = run_gpu(ind, wl)
    rows = np.array([0, 7, 31])
    ref, kth = oracle_topk(ind_np, wl, rows=rows)
    sc = oracle_scores(ind_np, wl, rows)
    check_topk_tolerant(got[rows], ref, sc, kth)
