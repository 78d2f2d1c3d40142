"""The work counts behind bench.py's roofline fractions, checked against
counts taken from the oracle's own outputs: visible (query, key) pairs are
the finite entries of the oracle's score matrix, and selected keys are the
valid entries of the oracle's index rows."""

import numpy as np
import pytest

import bench
import oracle
from dsa_indexer_reuse_b200 import workloads as W


def _small(wl, **kw):
    return wl.with_(**kw)


@pytest.mark.parametrize("wl", [
    _small(W.TINY_INT, n_q=96, n_k=96, topk=40),
    _small(W.TINY_INT, n_q=1, n_k=150, q_pos0=149, topk=64, batch=3),
    _small(W.TINY_INT, n_q=50, n_k=80, q_pos0=30, topk=16),
])
def test_flop_counts_match_the_oracle(wl):
    ind = {k: W.raw_numpy(v) for k, v in W.indexer_inputs(wl, 0).items()}
    common = dict(qk_dtype=wl.qk_dtype, w_dtype=wl.w_dtype, batch=wl.batch, n_q=wl.n_q, n_k=wl.n_k,
                  q_pos0=wl.q_pos0, H_I=wl.H_I, d_I=wl.d_I)
    scores = oracle.indexer_scores(ind["q_I"], ind["q_scale"], ind["w"], ind["k_I"], ind["k_scale"],
                                   **common)
    pairs = int(np.isfinite(scores).sum())
    assert bench.indexer_flops(wl) == pairs * wl.H_I * wl.d_I * 2
    idx, _ = oracle.indexer_topk(ind["q_I"], ind["q_scale"], ind["w"], ind["k_I"], ind["k_scale"],
                                 topk=wl.topk, **common)
    keys = int((idx >= 0).sum())
    assert bench.attn_flops(wl) == keys * wl.H * (wl.d_qk + wl.d_v) * 2
    for n_served in (1, 3):
        assert bench.distill_flops(wl, n_served) == keys * (n_served * wl.H * wl.d_qk + wl.H_I * wl.d_I) * 2
    compulsory, gather = bench.attn_bytes(wl)
    assert gather == keys * wl.d_qk * 2
    rows = wl.batch * wl.n_q
    # distinct KV rows the attention must read: the union of each sequence's
    # index rows, bounded by min(n_k, that sequence's selected keys)
    sel = idx.reshape(wl.batch, wl.n_q * wl.topk)
    distinct = sum(len(np.unique(r[r >= 0])) for r in sel)
    bound = wl.batch * min(wl.n_k, keys // wl.batch)
    assert distinct <= bound
    assert compulsory == (rows * wl.H * wl.d_qk * 2 + bound * wl.d_qk * 2 + rows * wl.topk * 4
                          + rows * wl.H * wl.d_v * 2)
    if wl.n_q == 1:
        assert distinct == bound          # decode: every selected row is distinct
    else:
        # causal prefill: almost every visible key is some query's choice
        assert distinct >= 0.9 * min(wl.n_k, wl.q_pos0 + wl.n_q)


def test_fp32_peak_is_derived_from_unit_counts_and_clock():
    assert bench.FP32_FMA_TFLOPS == pytest.approx(148 * 128 * 2 * 1.965e9 / 1e12)
