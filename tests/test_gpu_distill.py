"""GPU parity of the multi-layer distillation target (ic_distill_target)
against the oracle (IndexCache paper, Abstract; Table 3's "w/o cross-layer
loss" is the one-served-layer case).

Tolerances follow from fp32 arithmetic on the GPU side. A logit is a
d_qk-term fp32 dot product of bf16 values, with an error of order 1e-5 for the
Gaussian inputs here. Probabilities therefore carry ~1e-5 relative error, so
the target is checked to 1e-5 absolute + 1e-4 relative. The KL sums
P * (log P - log Q) terms whose logs carry the same relative error, so it is
checked to 1e-4 * max(1, KL)."""

import numpy as np
import pytest
import torch

import dsa_indexer_reuse_b200 as ic
import oracle
from dsa_indexer_reuse_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _inputs(wl, n_served, seed=0):
    dev = torch.device("cuda")
    ind = W.indexer_inputs(wl, 0, seed=seed, device=dev)
    served = []
    for l in range(n_served):
        att = W.attention_inputs(wl, l, seed=seed, device=dev)
        served.append((att["q"], att["kv"]))
    idx = ic.indexer_topk(ind["q_I"], ind["w"], ind["k_I"], wl.topk, q_scale=ind["q_scale"],
                          k_scale=ind["k_scale"], q_pos0=wl.q_pos0)
    return ind, served, idx


def _oracle(wl, ind, served, idx):
    raw = lambda t: None if t is None else W.raw_numpy(t.cpu())
    return oracle.distill_target([(raw(q), raw(kv)) for q, kv in served], raw(ind["q_I"]),
                                 raw(ind["q_scale"]), raw(ind["w"]), raw(ind["k_I"]), raw(ind["k_scale"]),
                                 idx.cpu().numpy().reshape(-1, wl.topk), qk_dtype=wl.qk_dtype,
                                 w_dtype=wl.w_dtype, batch=wl.batch, n_q=wl.n_q, n_k=wl.n_k,
                                 H_I=wl.H_I, d_I=wl.d_I, topk=wl.topk, H=wl.H, d_qk=wl.d_qk,
                                 sm_scale=wl.sm_scale)


def _check(wl, ind, served, idx):
    target, kl = ic.distill_target(served, ind["q_I"], ind["w"], ind["k_I"], idx, q_scale=ind["q_scale"],
                                   k_scale=ind["k_scale"], sm_scale=wl.sm_scale)
    torch.cuda.synchronize()
    want_t, want_kl = _oracle(wl, ind, served, idx)
    got_t = target.cpu().numpy().reshape(-1, wl.topk).astype(np.float64)
    got_kl = kl.cpu().numpy().reshape(-1).astype(np.float64)
    assert np.all(np.abs(got_t - want_t) <= 1e-5 + 1e-4 * np.abs(want_t))
    assert np.all(np.abs(got_kl - want_kl) <= 1e-4 * np.maximum(1.0, np.abs(want_kl)))
    return got_t, got_kl


def test_small_heads_bf16_two_served_layers(cuda_ok):
    # 4 heads of 64, bf16 indexer with 4 heads of 64; early rows see fewer
    # keys than topk (padded index rows)
    wl = W.TINY_INT.with_(n_q=384, n_k=384, topk=128, int_values=False)
    _check(wl, *_inputs(wl, 2))


def test_latent_fp8_three_served_layers(cuda_ok):
    # 64 heads, 576-wide latent rows, FP8 indexer with per-token scales
    wl = W.PREFILL_200K.with_(n_q=320, n_k=320, topk=256, n_layers=3)
    _check(wl, *_inputs(wl, 3, seed=2))


def test_latent_bf16_own_layer_only(cuda_ok):
    # "w/o cross-layer loss": the Full layer alone
    wl = W.PREFILL_8K.with_(n_q=256, n_k=256, topk=192, n_layers=1)
    _check(wl, *_inputs(wl, 1, seed=4))


def test_rows_without_keys_and_out_of_range_entries(cuda_ok):
    wl = W.TINY_INT.with_(n_q=128, n_k=128, topk=32, int_values=False)
    ind, served, idx = _inputs(wl, 2, seed=6)
    idx = idx.clone()
    idx[0, 5] = -1           # no valid entry
    idx[0, 9, :7] = 4096     # out of range: skipped
    t, kl = _check(wl, ind, served, idx)
    assert kl[5] == 0.0 and (t[5] == 0).all()
    assert (t[9, :7] == 0).all()


def test_decode_rows(cuda_ok):
    # one query per sequence over 2048 keys, the full topk
    wl = W.DECODE_32X32K.with_(batch=3, n_k=2048, q_pos0=2047, n_layers=2)
    _check(wl, *_inputs(wl, 2, seed=8))


def test_unsupported_shapes_are_refused(cuda_ok):
    wl = W.TINY_INT.with_(n_q=64, n_k=64, topk=16, int_values=False)
    ind, served, idx = _inputs(wl, 1)
    with pytest.raises(ic.IcError) as e:
        ic.distill_target(served * 65, ind["q_I"], ind["w"], ind["k_I"], idx)
    assert e.value.code == 3  # IC_ERR_UNSUPPORTED


def test_latent_rows_without_keys_and_out_of_range_entries(cuda_ok):
    # the tensor-core configuration (64 heads, 576-wide rows, 64-head indexer)
    wl = W.PREFILL_8K.with_(n_q=192, n_k=192, topk=128, n_layers=2)
    ind, served, idx = _inputs(wl, 2, seed=10)
    idx = idx.clone()
    idx[0, 5] = -1            # no valid entry
    idx[0, 9, :7] = 4096      # out of range: skipped
    idx[0, 150, ::3] = -1     # holes inside a row
    t, kl = _check(wl, ind, served, idx)
    assert kl[5] == 0.0 and (t[5] == 0).all()
    assert (t[9, :7] == 0).all() and (t[150, ::3] == 0).all()


def test_latent_long_rows_peaked_logits(cuda_ok):
    # rows of 1536 keys (12 tiles of 128: the first 4 are computed twice) and
    # logits with a standard deviation of ~32, so every head's softmax is
    # dominated by a few keys and the running maxima matter
    wl = W.DECODE_32X32K.with_(batch=2, n_k=1536, q_pos0=1535, n_layers=2)
    ind, served, idx = _inputs(wl, 2, seed=12)
    served = [(q * 32, kv) for q, kv in served]
    _check(wl, ind, served, idx)


def test_workspace_is_required_for_long_rows(cuda_ok):
    # topk 2048 on the tensor-core shapes spills logits: without a workspace
    # the call is refused before anything is enqueued
    import ctypes
    wl = W.DECODE_32X32K.with_(batch=1, n_k=1536, q_pos0=1535, n_layers=1)
    ind, served, idx = _inputs(wl, 1, seed=14)
    need = ic.distill_target_workspace_size(1, 1, wl.topk, wl.H, wl.d_qk, wl.H_I, wl.d_I)
    assert need > 0
    (q, kv), = served
    q_arr = (ctypes.c_void_p * 1)(q.data_ptr())
    kv_arr = (ctypes.c_void_p * 1)(kv.data_ptr())
    kl = torch.empty(1, dtype=torch.float32, device="cuda")
    small = torch.empty(need // 2, dtype=torch.uint8, device="cuda")
    for ws, n in ((None, 0), (small.data_ptr(), small.numel())):
        code = ic.lib.ic_distill_target(ctypes.cast(q_arr, ctypes.c_void_p), ctypes.cast(kv_arr, ctypes.c_void_p),
                                        1, ind["q_I"].data_ptr(), ind["q_scale"].data_ptr(), ind["w"].data_ptr(),
                                        2 if ind["w"].dtype == torch.float32 else 0, ind["k_I"].data_ptr(),
                                        ind["k_scale"].data_ptr(), 1, idx.data_ptr(), 1, 1, wl.n_k, wl.H_I, wl.d_I,
                                        wl.topk, wl.H, wl.d_qk, wl.sm_scale, None, kl.data_ptr(), ws, n, None)
        assert code == 6  # IC_ERR_WORKSPACE
