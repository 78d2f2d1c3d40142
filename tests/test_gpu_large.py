"""GPU parity at the large workloads' shapes and on the list-cut paths.

* FP8 prefill at topk 2048 past the candidate capacity (the sampled cut and
  its fallback run on every long row), bf16 prefill with a small k (the
  sampled branch of the 2816-entry lists);
* one layer of the 204800-token FP8 workload and of the 61440-token bf16
  workload: indexer rows sampled across t against the oracle, and the
  attention on the GPU's own index rows;
* the 47-layer, index_topk_freq=4 decode stack (ic_layer_stack) against the
  oracle's layer loop: exact on integer-valued FP8 indexer inputs (every
  score exact in fp32), recall / tolerance on the Gaussian recipe.

IndexCache paper, Abstract (per-query top-k over causal keys; sparse attention
over the selected keys) and Figure 2 caption (the F/S layer loop over one
index buffer). Inputs are generated on the device (same bytes on both sides);
only the sampled rows' query tensors travel to the host, in an otherwise
untouched zero array the oracle reads by row.
"""

import numpy as np
import pytest
import torch

import oracle
from dsa_indexer_reuse_b200 import workloads as W
from gpu_util import attn_rel_err, canon, check_topk_tolerant, oracle_scores, oracle_topk

pytestmark = pytest.mark.gpu


def raw(t):
    return W.raw_numpy(t)


def sparse_rows_host(t, rows):
    """Host storage array of device tensor t [B*n_q, ...] holding only `rows`
    (the rest is a lazily zeroed allocation the oracle never reads)."""
    dt = {torch.bfloat16: np.uint16, torch.uint8: np.uint8, torch.float32: np.float32}[t.dtype]
    flat = t.reshape(-1, *t.shape[2:]) if t.dim() > 2 else t.reshape(-1, 1)
    host = np.zeros(tuple(flat.shape), dt)
    sel = torch.as_tensor(np.asarray(rows), device=t.device)
    host[np.asarray(rows)] = raw(flat.index_select(0, sel))
    return host.reshape(t.shape)


def indexer_on_device(wl, layer=0, seed=0):
    d = W.indexer_inputs(wl, layer, seed=seed, device="cuda")
    return d


def host_indexer_rows(d, rows):
    """The oracle's view of device indexer tensors: keys and per-query scales
    and weights whole, q_I only at the sampled rows."""
    return {"q_I": sparse_rows_host(d["q_I"], rows), "w": raw(d["w"]),
            "q_scale": raw(d["q_scale"]), "k_I": raw(d["k_I"]), "k_scale": raw(d["k_scale"])}


def run_indexer(d, wl, topk=None):
    import dsa_indexer_reuse_b200 as ic
    k = topk or wl.topk
    idx = ic.indexer_topk(d["q_I"], d["w"], d["k_I"], k, q_scale=d["q_scale"],
                          k_scale=d["k_scale"], q_pos0=wl.q_pos0)
    torch.cuda.synchronize()
    return idx


def check_indexer_rows(idx, d, wl, rows, topk=None):
    k = topk or wl.topk
    got = idx.reshape(-1, k)[torch.as_tensor(rows, device=idx.device)].cpu().numpy()
    hst = host_indexer_rows(d, rows)
    ref, kth = oracle_topk(hst, wl, rows=rows, topk=k)
    sc = oracle_scores(hst, wl, rows)
    return check_topk_tolerant(got, ref, sc, kth)


def check_attention_rows(wl, idx, rows, layer=0, seed=0):
    """Attention on the GPU's own index rows against the oracle on the same
    rows (each row is independent: a compact problem of just those rows)."""
    import dsa_indexer_reuse_b200 as ic
    q = W.attention_query(wl, layer, seed=seed, device="cuda")
    kv = W.attention_kv(wl, layer, seed=seed, device="cuda")
    out = ic.sparse_attn(q, kv, idx, d_v=wl.d_v, sm_scale=wl.sm_scale)
    torch.cuda.synchronize()
    sel = torch.as_tensor(rows, device="cuda")
    q_rows = raw(q.reshape(-1, wl.H, wl.d_qk).index_select(0, sel))
    idx_rows = idx.reshape(-1, wl.topk).index_select(0, sel).cpu().numpy()
    out_rows = out.reshape(-1, wl.H, wl.d_v).index_select(0, sel).float().cpu().numpy()
    del q, out
    ref = oracle.sparse_attn(q_rows, raw(kv), idx_rows, batch=1, n_q=len(rows), n_k=wl.n_k, H=wl.H,
                             d_qk=wl.d_qk, d_v=wl.d_v, topk=wl.topk, sm_scale=wl.sm_scale)
    err = attn_rel_err(out_rows, ref).max()
    assert err <= 1e-2, "attention max rel err %.3g" % err


def spread_rows(n, count, tail=4):
    """`count` rows spread over [0, n) plus the last `tail` rows."""
    r = np.unique(np.r_[np.linspace(0, n - 1, count).astype(np.int64), np.arange(n - tail, n)])
    return r


def test_fp8_prefill_list_cut(cuda_ok):
    # capacity 4096 per query at topk 2048: every row past ~4k keys is cut by
    # the sampled threshold (or its exact fallback) several times
    wl = W.PREFILL_200K.with_(n_q=16384, n_k=16384)
    d = indexer_on_device(wl, seed=11)
    idx = run_indexer(d, wl)
    rows = np.unique(np.r_[spread_rows(wl.n_q, 16), 4095, 4096, 4097, 8191, 12000])
    check_indexer_rows(idx, d, wl, rows)


def test_bf16_prefill_sampled_cut_small_k(cuda_ok):
    # 2816-entry lists with topk 1024 leave 1792 >= 1536 slots: the sampled cut
    wl = W.PREFILL_8K.with_(n_q=6144, n_k=6144, topk=1024)
    d = indexer_on_device(wl, seed=12)
    idx = run_indexer(d, wl)
    rows = np.unique(np.r_[spread_rows(wl.n_q, 16), 1023, 1024, 2900, 2901])
    check_indexer_rows(idx, d, wl, rows)


def test_prefill_200k_one_layer_sampled_rows(cuda_ok):
    wl = W.PREFILL_200K
    d = indexer_on_device(wl, seed=0)
    idx = run_indexer(d, wl)
    rows = spread_rows(wl.n_q, 14, tail=2)
    check_indexer_rows(idx, d, wl, rows)
    del d
    torch.cuda.empty_cache()
    check_attention_rows(wl, idx, rows)


def test_prefill_60k_one_layer_sampled_rows(cuda_ok):
    wl = W.PREFILL_60K
    d = indexer_on_device(wl, seed=0)
    idx = run_indexer(d, wl)
    rows = spread_rows(wl.n_q, 14, tail=2)
    check_indexer_rows(idx, d, wl, rows)
    del d
    torch.cuda.empty_cache()
    check_attention_rows(wl, idx, rows)


# ----------------------------------------------------------------- decode stack
def fp8_int_codes(shape, gen, device):
    """E4M3 codes of integers in [-3, 3] (exact in the format)."""
    v = torch.randint(-3, 4, shape, generator=gen, device=device).float()
    return v.to(torch.float8_e4m3fn).view(torch.uint8).contiguous()


def decode_stack_layers(wl, int_indexer, seed=0):
    """Device layers of a decode stack and the oracle's host view. Shared
    layers carry no indexer tensors."""
    import dsa_indexer_reuse_b200 as ic
    is_full, _ = ic.resolve_pattern(wl.n_layers, wl.freq, wl.pattern)
    dev, host = [], []
    for l in range(wl.n_layers):
        L = {}
        if is_full[l]:
            if int_indexer:
                g = torch.Generator(device="cuda")
                g.manual_seed(seed * 1000 + l * 16 + 9)
                B = wl.batch
                L["q_I"] = fp8_int_codes((B, wl.n_q, wl.H_I, wl.d_I), g, "cuda")
                L["k_I"] = fp8_int_codes((B, wl.n_k, wl.d_I), g, "cuda")
                L["w"] = torch.randint(-3, 4, (B, wl.n_q, wl.H_I), generator=g, device="cuda").float()
                # power-of-two token scales keep every score exact
                L["q_scale"] = torch.pow(2.0, torch.randint(-2, 3, (B, wl.n_q), generator=g,
                                                            device="cuda").float()).contiguous()
                L["k_scale"] = torch.pow(2.0, torch.randint(-2, 3, (B, wl.n_k), generator=g,
                                                            device="cuda").float()).contiguous()
            else:
                L.update(W.indexer_inputs(wl, l, seed=seed, device="cuda"))
        else:
            L.update(q_I=None, q_scale=None, w=None, k_I=None, k_scale=None)
        L["q"] = W.attention_query(wl, l, seed=seed, device="cuda")
        L["kv"] = W.attention_kv(wl, l, seed=seed, device="cuda")
        L["out"] = torch.empty((wl.batch, wl.n_q, wl.H, wl.d_v), dtype=torch.bfloat16, device="cuda")
        dev.append(L)
        host.append({k: raw(v) for k, v in L.items() if k != "out"})
    return dev, host, is_full


def stack_shape(wl):
    return dict(batch=wl.batch, n_q=wl.n_q, n_k=wl.n_k, q_pos0=wl.q_pos0, H_I=wl.H_I, d_I=wl.d_I,
                topk=wl.topk, qk_dtype=wl.qk_dtype, w_dtype=wl.w_dtype, H=wl.H, d_qk=wl.d_qk,
                d_v=wl.d_v, sm_scale=wl.sm_scale)


def oracle_stack(wl, host):
    return oracle.layer_stack(host, freq=wl.freq, pattern=wl.pattern, qk_dtype=wl.qk_dtype,
                              w_dtype=wl.w_dtype, batch=wl.batch, n_q=wl.n_q, n_k=wl.n_k,
                              q_pos0=wl.q_pos0, H_I=wl.H_I, d_I=wl.d_I, topk=wl.topk, H=wl.H,
                              d_qk=wl.d_qk, d_v=wl.d_v, sm_scale=wl.sm_scale)


def test_decode_stack_47_layers_integer_exact(cuda_ok):
    import dsa_indexer_reuse_b200 as ic
    wl = W.DECODE_32X32K.with_(batch=4, n_k=8192, q_pos0=8191)
    dev, host, is_full = decode_stack_layers(wl, int_indexer=True, seed=3)
    idx = ic.layer_stack(dev, stack_shape(wl), freq=wl.freq)
    torch.cuda.synchronize()
    ref_idx, ref_out = oracle_stack(wl, host)
    last_full = int(np.nonzero(is_full)[0][-1])
    got = idx.cpu().numpy().reshape(wl.batch, wl.topk)
    assert (got == canon(ref_idx[last_full])).all()
    for l in range(wl.n_layers):
        out = dev[l]["out"].float().cpu().numpy().reshape(-1, wl.H, wl.d_v)
        err = attn_rel_err(out, ref_out[l]).max()
        assert err <= 1e-2, "layer %d: max rel err %.3g" % (l, err)


def test_decode_stack_47_layers_gaussian(cuda_ok):
    import dsa_indexer_reuse_b200 as ic
    wl = W.DECODE_32X32K.with_(batch=2)
    dev, host, is_full = decode_stack_layers(wl, int_indexer=False, seed=4)
    idx = ic.layer_stack(dev, stack_shape(wl), freq=wl.freq)
    torch.cuda.synchronize()
    stack_idx = idx.cpu().numpy().reshape(wl.batch, wl.topk)
    ref_idx, ref_out = oracle_stack(wl, host)
    _, src = ic.resolve_pattern(wl.n_layers, wl.freq, wl.pattern)
    # each Full layer's own indices (the same kernel as inside the stack)
    gpu_idx = {}
    for l in np.nonzero(is_full)[0]:
        L = dev[l]
        g = ic.indexer_topk(L["q_I"], L["w"], L["k_I"], wl.topk, q_scale=L["q_scale"],
                            k_scale=L["k_scale"], q_pos0=wl.q_pos0)
        torch.cuda.synchronize()
        gpu_idx[int(l)] = g.cpu().numpy().reshape(wl.batch, wl.topk)
        hst = {k: host[l][k] for k in ("q_I", "q_scale", "w", "k_I", "k_scale")}
        sc = oracle_scores(hst, wl, np.arange(wl.batch))
        kth = np.sort(np.nan_to_num(sc, nan=-np.inf), axis=1)[:, -wl.topk]
        check_topk_tolerant(gpu_idx[int(l)], ref_idx[l], sc, kth)
    last_full = int(np.nonzero(is_full)[0][-1])
    assert (stack_idx == gpu_idx[last_full]).all(), "the stack's buffer is the last Full layer's"
    matched = 0
    for l in range(wl.n_layers):
        out = dev[l]["out"].float().cpu().numpy().reshape(-1, wl.H, wl.d_v)
        same = (canon(gpu_idx[int(src[l])]) == canon(ref_idx[int(src[l])])).all(axis=1)
        matched += int(same.sum())
        if same.any():
            err = attn_rel_err(out[same], ref_out[l][same]).max()
            assert err <= 1e-2, "layer %d: max rel err %.3g" % (l, err)
    assert matched >= wl.n_layers * wl.batch * 3 // 4, "too few rows with identical index sets"
