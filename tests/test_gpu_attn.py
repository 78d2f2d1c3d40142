"""GPU parity of the sparse attention (ic_sparse_attn) against the oracle.

Criterion: for every (query row, head) the output vector's max absolute error
is <= 1e-2 of the oracle vector's max magnitude (bf16 inputs, fp32
accumulation, bf16 output). Index lists come from a seeded generator (valid
causal keys in arbitrary order, -1 padding anywhere), so the test does not
depend on the indexer.
"""

import math

import numpy as np
import pytest
import torch

import oracle
from dsa_indexer_reuse_b200 import workloads as W
from gpu_util import attn_rel_err

pytestmark = pytest.mark.gpu
TOL = 1e-2


def random_idx(B, n_q, n_k, topk, q_pos0, seed, pad_frac=0.1):
    rng = np.random.default_rng(seed)
    idx = np.full((B, n_q, topk), -1, np.int32)
    for b in range(B):
        for t in range(n_q):
            vis = min(q_pos0 + t + 1, n_k)
            n = min(topk, vis)
            sel = rng.choice(vis, size=n, replace=False).astype(np.int32)
            row = np.full(topk, -1, np.int32)
            row[:n] = sel
            if pad_frac > 0:
                rng.shuffle(row)  # padding anywhere in the row
            idx[b, t] = row
    return idx


def run(wl, idx, seed=0, scale_q=1.0):
    import dsa_indexer_reuse_b200 as ic
    att = W.attention_inputs(wl, 0, seed=seed)
    if scale_q != 1.0:
        att["q"] = (att["q"].float() * scale_q).to(torch.bfloat16)
    q, kv = att["q"].cuda(), att["kv"].cuda()
    out = ic.sparse_attn(q, kv, torch.from_numpy(idx).cuda(), d_v=wl.d_v, sm_scale=wl.sm_scale)
    torch.cuda.synchronize()
    return out.float().cpu().numpy(), W.raw_numpy(att["q"]), W.raw_numpy(att["kv"])


def ref(wl, q, kv, idx, rows=None):
    return oracle.sparse_attn(q, kv, idx, batch=wl.batch, n_q=wl.n_q, n_k=wl.n_k, H=wl.H,
                              d_qk=wl.d_qk, d_v=wl.d_v, topk=idx.shape[-1], sm_scale=wl.sm_scale,
                              rows=rows)


def check(wl, out, q, kv, idx, rows=None):
    r = ref(wl, q, kv, idx, rows)
    o = out.reshape(-1, wl.H, wl.d_v)
    if rows is not None:
        o = o[rows]
    err = attn_rel_err(o, r)
    assert err.max() <= TOL, "max rel err %.3g" % err.max()
    return err.max()


def test_tiny_heads_d64(cuda_ok):
    wl = W.TINY_INT.with_(n_q=300, n_k=300)
    idx = random_idx(1, 300, 300, 128, 0, seed=1)
    out, q, kv = run(wl, idx)
    check(wl, out, q, kv, idx)


def test_latent_576_512_ragged(cuda_ok):
    wl = W.PREFILL_8K.with_(n_q=200, n_k=700, q_pos0=500, topk=300)
    idx = random_idx(1, 200, 700, 300, 500, seed=2)
    out, q, kv = run(wl, idx)
    check(wl, out, q, kv, idx)


def test_latent_topk2048_sampled(cuda_ok):
    wl = W.PREFILL_8K.with_(n_q=3000, n_k=3000)
    idx = random_idx(1, 3000, 3000, 2048, 0, seed=3, pad_frac=0)
    out, q, kv = run(wl, idx)
    rows = np.r_[0:5, 2046:2050, 2990:3000]
    check(wl, out, q, kv, idx, rows)


def test_decode_split(cuda_ok):
    wl = W.DECODE_32X32K.with_(batch=6, n_k=9000, q_pos0=8999)
    idx = random_idx(6, 1, 9000, 2048, 8999, seed=4, pad_frac=0)
    out, q, kv = run(wl, idx)
    check(wl, out, q, kv, idx)


def test_rows_without_keys_and_single_key(cuda_ok):
    wl = W.PREFILL_8K.with_(n_q=4, n_k=100, topk=64)
    idx = np.full((1, 4, 64), -1, np.int32)
    idx[0, 1, 17] = 5          # one key
    idx[0, 2, :3] = [99, 0, 50]
    idx[0, 3, 5] = 1000        # out of range only: skipped
    out, q, kv = run(wl, idx)
    o = out.reshape(4, wl.H, wl.d_v)
    assert (o[0] == 0).all() and (o[3] == 0).all()
    v5 = oracle.bf16_to_float64(kv.reshape(100, wl.d_qk)[5, : wl.d_v])
    assert (o[1] == v5[None, :]).all()  # softmax of one key is exactly 1
    check(wl, out, q, kv, idx, rows=np.array([2]))


def test_large_logit_spread_takes_rescale_path(cuda_ok):
    # first selected key of each row has a small logit, later keys have
    # logits far above it: the reference must be raised mid-row
    wl = W.PREFILL_8K.with_(n_q=8, n_k=600, q_pos0=592, topk=512)
    idx = random_idx(1, 8, 600, 512, 592, seed=5, pad_frac=0)
    out, q, kv = run(wl, idx, scale_q=24.0)  # logits ~ N(0, 24^2)
    check(wl, out, q, kv, idx)


def test_deterministic(cuda_ok):
    wl = W.PREFILL_8K.with_(n_q=64, n_k=1000, q_pos0=936, topk=512)
    idx = random_idx(1, 64, 1000, 512, 936, seed=6)
    a, _, _ = run(wl, idx)
    b, _, _ = run(wl, idx)
    assert (a == b).all()


def _decode_call(wl, idx, seed, workspace):
    import dsa_indexer_reuse_b200 as ic
    att = W.attention_inputs(wl, 0, seed=seed)
    q, kv = att["q"].cuda(), att["kv"].cuda()
    out = ic.sparse_attn(q, kv, torch.from_numpy(idx).cuda(), d_v=wl.d_v, sm_scale=wl.sm_scale,
                         workspace=workspace)
    torch.cuda.synchronize()
    return out.float().cpu().numpy(), W.raw_numpy(att["q"]), W.raw_numpy(att["kv"])


@pytest.mark.parametrize("shape", ["latent", "tiny_h40"])
def test_decode_split_dirty_shared_workspace(cuda_ok, shape):
    # Decode-style calls split each row's keys across CTAs and merge the
    # partials from the workspace. The workspace starts dirty (every byte
    # 0xFF), two calls in a row share it, and some rows have no key at all
    # (every split empty) or keys in the first split only; fewer than 64
    # heads leave the second softmax warpgroup's head half short.
    import dsa_indexer_reuse_b200 as ic
    if shape == "latent":
        wl = W.DECODE_32X32K.with_(batch=8, n_k=5000, q_pos0=4999)
    else:
        wl = W.TINY_INT.with_(batch=8, n_q=1, n_k=5000, q_pos0=4999, topk=1024, H=40)
    topk = wl.topk
    assert ic.sparse_attn_workspace_size(wl.batch, 1, wl.H, wl.d_v, topk) > 0  # the split path
    ws = torch.full((ic.sparse_attn_workspace_size(wl.batch, 1, wl.H, wl.d_v, topk),), 255,
                    dtype=torch.uint8, device="cuda")
    for call, seed in enumerate((11, 12)):
        idx = random_idx(wl.batch, 1, wl.n_k, topk, wl.q_pos0, seed=seed, pad_frac=0)
        idx[1] = -1                      # a row without keys
        idx[2, 0, 40:] = -1              # keys in the first split only
        out, q, kv = _decode_call(wl, idx, seed, ws)
        o = out.reshape(wl.batch, wl.H, wl.d_v)
        assert (o[1] == 0).all(), "call %d: a row without keys must give 0" % call
        check(wl, out, q, kv, idx, rows=np.array([r for r in range(wl.batch) if r != 1]))
