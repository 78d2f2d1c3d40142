"""Exact parity of the decode path (one query per sequence, 64 heads,
d_I = 128: score rows + per-row select) on inputs whose scores are exact in
fp32, so indices must match the oracle bit for bit. Small-integer inputs give
many exactly equal scores (ties to the lower key), all-equal scores leave the
radix select no bit to fix, three distinct scores put the k-th key in a large
class of equal keys, and short contexts give fewer than k keys."""

import numpy as np
import pytest
import torch

import dsa_indexer_reuse_b200 as ic
import oracle

from gpu_util import canon

pytestmark = pytest.mark.gpu


def _int_inputs(B, n_k, seed, zero_keys=False):
    g = torch.Generator().manual_seed(seed)
    q = torch.randint(-3, 4, (B, 1, 64, 128), generator=g).to(torch.bfloat16)
    k = torch.randint(-3, 4, (B, n_k, 128), generator=g).to(torch.bfloat16)
    if zero_keys:
        k.zero_()
    w = torch.randint(-3, 4, (B, 1, 64), generator=g).to(torch.bfloat16)
    return q, w, k


def _oracle(q, w, k, topk, q_pos0):
    B, n_k = k.shape[0], k.shape[1]
    bits = lambda t: t.contiguous().view(torch.int16).numpy().view("uint16")
    idx, _ = oracle.indexer_topk(bits(q), None, bits(w), bits(k), None, qk_dtype=oracle.BF16,
                                 w_dtype=oracle.BF16, batch=B, n_q=1, n_k=n_k, q_pos0=q_pos0,
                                 H_I=64, d_I=128, topk=topk)
    return idx


@pytest.mark.parametrize("B,n_k,topk,q_pos0", [
    (3, 32768, 2048, 32767), (2, 5000, 2048, 4999), (2, 9000, 100, 8999), (4, 1500, 2048, 1499),
    (2, 32768, 2048, 20000),
])
def test_decode_rows_exact_on_integer_scores(cuda_ok, B, n_k, topk, q_pos0):
    q, w, k = _int_inputs(B, n_k, seed=n_k + topk)
    dev = torch.device("cuda")
    got = ic.indexer_topk(q.to(dev), w.to(dev), k.to(dev), topk, q_pos0=q_pos0).cpu().numpy()
    want = _oracle(q, w, k, topk, q_pos0)
    assert np.array_equal(canon(got.reshape(B, topk)), canon(want))
    # the GPU writes ascending key order, -1 last
    g = got.reshape(B, topk)
    for r in range(B):
        v = g[r][g[r] >= 0]
        assert np.all(np.diff(v) > 0)


def test_decode_rows_all_equal_scores(cuda_ok):
    # every score equal: the k lowest key indices, through the full-row fallback
    B, n_k, topk = 2, 32768, 2048
    q, w, k = _int_inputs(B, n_k, seed=5, zero_keys=True)
    dev = torch.device("cuda")
    got = ic.indexer_topk(q.to(dev), w.to(dev), k.to(dev), topk, q_pos0=n_k - 1).cpu().numpy()
    assert np.array_equal(got.reshape(B, topk), np.tile(np.arange(topk, dtype=np.int32), (B, 1)))


def test_decode_rows_three_distinct_scores(cuda_ok):
    # every key row is one of three patterns, so each sequence has three
    # distinct scores and the k-th largest sits in a class of ~11k equal keys:
    # the radix select fixes every bit of that score and takes the class's
    # lowest key indices (ties go to the lower key)
    B, n_k, topk = 2, 32768, 2048
    g = torch.Generator().manual_seed(9)
    q = torch.randint(-3, 4, (B, 1, 64, 128), generator=g).to(torch.bfloat16)
    w = torch.randint(-3, 4, (B, 1, 64), generator=g).to(torch.bfloat16)
    pats = torch.randint(-3, 4, (B, 3, 128), generator=g).to(torch.bfloat16)
    cls = torch.randint(0, 3, (B, n_k), generator=g)
    k = torch.stack([pats[b][cls[b]] for b in range(B)])
    dev = torch.device("cuda")
    got = ic.indexer_topk(q.to(dev), w.to(dev), k.to(dev), topk, q_pos0=n_k - 1).cpu().numpy()
    want = _oracle(q, w, k, topk, n_k - 1)
    assert np.array_equal(canon(got.reshape(B, topk)), canon(want))
