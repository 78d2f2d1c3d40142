"""The allocation-free indexer entry point (ic_indexer_topk_noalloc) against
the regular one (ic_indexer_topk with a caller-provided workspace).

Some callers of this library cannot call cudaMalloc (their device memory
belongs to another allocator or a fixed arena, or they must not risk an
allocation's implicit synchronisation); the no-alloc entry point serves them
from a fixed array the library owns. This file sorts last so that a run that
stops at the first failure has run every other test first; it passes both
alone in a fresh process and after the rest of the suite.
"""

import ctypes

import numpy as np
import pytest
import torch

from dsa_indexer_reuse_b200 import workloads as W
from gpu_util import canon

pytestmark = pytest.mark.gpu


def _lib():
    import dsa_indexer_reuse_b200 as ic
    lib = ic.lib
    P, I = ctypes.c_void_p, ctypes.c_int
    lib.ic_indexer_topk_noalloc.argtypes = [P, P, P, I, P, P, I, I, I, I, I, I, I, I, P, P]
    lib.ic_indexer_topk_noalloc.restype = I
    lib.ic_indexer_noalloc_max_scratch.argtypes = []
    lib.ic_indexer_noalloc_max_scratch.restype = ctypes.c_size_t
    return ic, lib


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _call_noalloc(lib, ic, d, wl, out):
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return lib.ic_indexer_topk_noalloc(
        _p(d["q_I"]), _p(d["q_scale"]), _p(d["w"]), wl.w_dtype, _p(d["k_I"]), _p(d["k_scale"]),
        wl.qk_dtype, wl.batch, wl.n_q, wl.n_k, wl.q_pos0, wl.H_I, wl.d_I, wl.topk, _p(out), stream)


@pytest.mark.parametrize("wl", [
    W.DECODE_32X32K.with_(batch=8, n_k=20000, q_pos0=19999),                    # split path: scratch
    W.DECODE_32X32K.with_(batch=3, n_k=9000, q_pos0=8999, qk_dtype=W.BF16, w_dtype=W.BF16),
    W.PREFILL_8K.with_(n_q=1200, n_k=1200, topk=256),                           # no scratch needed
], ids=["decode-fp8", "decode-bf16", "prefill"])
def test_noalloc_matches_workspace_entry_point_twice(cuda_ok, wl):
    ic, lib = _lib()
    ind = W.indexer_inputs(wl, 0, seed=11)
    d = {k: (None if v is None else v.cuda()) for k, v in ind.items()}
    ref = ic.indexer_topk(d["q_I"], d["w"], d["k_I"], wl.topk, q_scale=d["q_scale"],
                          k_scale=d["k_scale"], q_pos0=wl.q_pos0)
    torch.cuda.synchronize()
    ref = ref.cpu().numpy()
    for _ in range(2):  # two calls in a row share the same scratch array
        out = torch.full((wl.batch, wl.n_q, wl.topk), -7, dtype=torch.int32, device="cuda")
        assert _call_noalloc(lib, ic, d, wl, out) == 0
        torch.cuda.synchronize()
        # index sets are exact: both paths score every key with the same
        # arithmetic; the order of a row's entries may differ between the
        # split lists and the score-row select, so rows compare as sets
        assert np.array_equal(canon(out.cpu().numpy().reshape(-1, wl.topk)), canon(ref.reshape(-1, wl.topk)))
    assert ic.get_device_status() == 0


def test_noalloc_array_covers_every_supported_decode_shape(cuda_ok):
    # the fixed array must hold the split scratch of every decode-style call
    # this GPU can be given (requests beyond it are refused with
    # IC_ERR_WORKSPACE before anything is enqueued)
    ic, lib = _lib()
    limit = lib.ic_indexer_noalloc_max_scratch()
    assert limit == 8 << 20
    lib.ic_indexer_noalloc_scratch_size.argtypes = [ctypes.c_int] * 7 + [ctypes.POINTER(ctypes.c_size_t)]
    lib.ic_indexer_noalloc_scratch_size.restype = ctypes.c_int

    def need(b, H_I, d_I, topk, dt, n_k=32768):
        out = ctypes.c_size_t(0)
        assert lib.ic_indexer_noalloc_scratch_size(b, 1, n_k, H_I, d_I, topk, dt,
                                                   ctypes.byref(out)) == 0
        return out.value

    # every compiled decode plan at its largest supported top-k
    for H_I, d_I, topk, dt in ((64, 128, 2048, ic.FP8_E4M3), (64, 128, 2048, ic.BF16),
                               (4, 64, 128, ic.BF16)):
        worst = max(need(b, H_I, d_I, topk, dt) for b in range(1, 600))
        assert 0 < worst <= limit, (H_I, d_I, topk, dt, worst)

    # a top-k the plan cannot serve is refused as unsupported, before sizing
    out = ctypes.c_size_t(0)
    assert lib.ic_indexer_noalloc_scratch_size(1, 1, 32768, 4, 64, 1024, ic.BF16,
                                               ctypes.byref(out)) == 3
