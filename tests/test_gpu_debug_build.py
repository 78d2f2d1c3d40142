"""The IC_DEBUG build of the library (build.py --debug): the same kernels with
the by-construction index checks compiled in (list appends, select outputs,
compacted index rows, gathered rows). Small parity cases run through it in a
child process (IC_LIB_PATH selects the library at import) and must leave the
device status clean: no check fired, and the results match the oracle."""

import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r'''
import sys
sys.path.insert(0, ROOT)
sys.path.insert(0, ROOT + "/tests")
import numpy as np, torch
import dsa_indexer_reuse_b200 as ic
assert ic.LIB_PATH.endswith("libindexcache_debug.so"), ic.LIB_PATH
from dsa_indexer_reuse_b200 import workloads as W
from gpu_util import canon, check_topk_tolerant, host_indexer, oracle_scores, oracle_topk, attn_rel_err
import oracle
# tiny integer workload: exact indices (ascending lists, per-step barrier path)
wl = W.TINY_INT.with_(n_q=700, n_k=700)
ind = W.indexer_inputs(wl, 0)
d = {k: (None if v is None else v.cuda()) for k, v in ind.items()}
got = ic.indexer_topk(d["q_I"], d["w"], d["k_I"], wl.topk).cpu().numpy().reshape(-1, wl.topk)
ref, _ = oracle_topk(host_indexer(ind), wl)
assert (got == canon(ref)).all()
# 64-head FP8 prefill past the list capacity (cuts), bf16 prefill, decode split + merge
for wl, rows in ((W.PREFILL_200K.with_(n_q=6000, n_k=6000), np.r_[0:4, 2047:2050, 5990:6000]),
                 (W.PREFILL_8K.with_(n_q=3000, n_k=3000), np.r_[0:4, 2900:2910]),
                 (W.DECODE_32X32K.with_(batch=3, n_k=40000, q_pos0=39999), np.arange(3))):
    ind = W.indexer_inputs(wl, 0, seed=2)
    d = {k: (None if v is None else v.cuda()) for k, v in ind.items()}
    got = ic.indexer_topk(d["q_I"], d["w"], d["k_I"], wl.topk, q_scale=d["q_scale"], k_scale=d["k_scale"],
                          q_pos0=wl.q_pos0).cpu().numpy().reshape(-1, wl.topk)
    hst = host_indexer(ind)
    ref, kth = oracle_topk(hst, wl, rows=rows)
    check_topk_tolerant(got[rows], ref, oracle_scores(hst, wl, rows), kth)
# sparse attention on those decode indices (split + combine)
att = W.attention_inputs(wl, 0, seed=3)
q, kv = att["q"].cuda(), att["kv"].cuda()
idx = torch.as_tensor(got.reshape(wl.batch, 1, wl.topk)).cuda()
out = ic.sparse_attn(q, kv, idx, d_v=wl.d_v, sm_scale=wl.sm_scale).float().cpu().numpy().reshape(-1, wl.H, wl.d_v)
refa = oracle.sparse_attn(W.raw_numpy(att["q"]), W.raw_numpy(att["kv"]), got, batch=wl.batch, n_q=1, n_k=wl.n_k,
                          H=wl.H, d_qk=wl.d_qk, d_v=wl.d_v, topk=wl.topk, sm_scale=wl.sm_scale)
assert attn_rel_err(out, refa).max() <= 1e-2
st = ic.get_device_status()
assert st == 0, "device status %d" % st
print("DEBUG_BUILD_OK")
'''


def test_debug_build_parity_and_clean_status(cuda_ok):
    lib = os.path.join(ROOT, "dsa_indexer_reuse_b200", "libindexcache_debug.so")
    if not os.path.exists(lib):
        from dsa_indexer_reuse_b200 import build
        build.build(debug=True)
    env = dict(os.environ, IC_LIB_PATH=lib)
    p = subprocess.run([sys.executable, "-c", "ROOT = %r\n" % ROOT + CHILD], env=env, capture_output=True,
                       text=True, timeout=900)
    assert p.returncode == 0 and "DEBUG_BUILD_OK" in p.stdout, (p.stdout[-2000:], p.stderr[-4000:])
