"""C-ABI checks that need no GPU: the library loads, exports every function
include/indexcache.h declares, resolves F/S patterns exactly as the oracle
does, and rejects invalid calls on the host before any device work."""

import ctypes
import os
import re

import numpy as np
import pytest

import oracle
from conftest import ROOT, read_golden_lines

HEADER = os.path.join(ROOT, "include", "indexcache.h")


@pytest.fixture(scope="module")
def ic():
    from dsa_indexer_reuse_b200 import build as b
    b.build()
    import dsa_indexer_reuse_b200 as m
    return m


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^(?:const\s+char\s*\*|ic_status|int|size_t)\s+(ic_\w+)\s*\(", text,
                                 flags=re.M)))


def test_header_declares_the_path():
    names = declared_functions()
    for n in ("ic_resolve_pattern", "ic_indexer_topk", "ic_sparse_attn", "ic_layer_stack"):
        assert n in names


def test_library_exports_every_declared_symbol(ic):
    lib = ctypes.CDLL(ic.LIB_PATH)
    for n in declared_functions():
        assert hasattr(lib, n), n


def test_status_strings(ic):
    for code, name in ic.STATUS.items():
        assert ic.lib.ic_status_string(code).decode() == name
    assert ic.version() >> 16 == 1


@pytest.mark.parametrize("n,freq,pattern", [
    (8, 2, None), (47, 4, None), (47, 1, None), (47, 0, None), (5, 9, None), (4, 0, "FSFS"),
    (4, 0, "FFSS"), (1, 0, "F"), (3, 3, None),
])
def test_resolve_pattern_matches_oracle(ic, n, freq, pattern):
    a = ic.resolve_pattern(n, freq, pattern)
    b = oracle.resolve_pattern(n, freq, pattern)
    assert (a[0] == b[0]).all() and (a[1] == b[1]).all()


def test_resolve_printed_glm5_pattern(ic):
    (s,) = read_golden_lines("glm5_pattern.txt")
    a = ic.resolve_pattern(len(s), 0, s)
    b = oracle.resolve_pattern(len(s), 0, s)
    assert (a[0] == b[0]).all() and (a[1] == b[1]).all()


@pytest.mark.parametrize("n,freq,pattern,code", [
    (4, 0, "FSF", 2), (4, 0, "FSXS", 2), (4, 0, "SFSF", 2), (4, 2, "FSFS", 1), (4, -1, None, 1),
    (0, 0, None, 1),
])
def test_resolve_pattern_errors_match_oracle(ic, n, freq, pattern, code):
    with pytest.raises(ic.IcError) as e:
        ic.resolve_pattern(n, freq, pattern)
    assert e.value.code == code
    with pytest.raises(oracle.PatternError) as e2:
        oracle.resolve_pattern(n, freq, pattern)
    assert e2.value.code == code


def test_invalid_calls_fail_on_host(ic):
    L = ic.lib
    P = ctypes.c_void_p
    fake = P(0x10000)  # never dereferenced: validation fails first
    # null q_I
    assert L.ic_indexer_topk(None, None, fake, 0, fake, None, 0, 1, 16, 16, 0, 64, 128, 8, fake,
                             None, 0, None) == 1
    # FP8 without scales
    assert L.ic_indexer_topk(fake, None, fake, 2, fake, None, 1, 1, 16, 16, 0, 64, 128, 8, fake,
                             None, 0, None) == 1
    # negative sizes, bad dtype
    assert L.ic_indexer_topk(fake, None, fake, 0, fake, None, 0, -1, 16, 16, 0, 64, 128, 8, fake,
                             None, 0, None) == 1
    assert L.ic_indexer_topk(fake, None, fake, 7, fake, None, 0, 1, 16, 16, 0, 64, 128, 8, fake,
                             None, 0, None) == 1
    # misaligned q_I (TMA needs 16-byte aligned bases)
    assert L.ic_indexer_topk(P(0x10002), None, fake, 0, fake, None, 0, 1, 16, 16, 0, 64, 128, 8,
                             fake, None, 0, None) == 1
    # attention: zero heads, null out
    assert L.ic_sparse_attn(fake, fake, fake, 1, 4, 16, 0, 576, 512, 8, ctypes.c_float(0.1), fake,
                            None, 0, None) == 1
    assert L.ic_sparse_attn(fake, fake, fake, 1, 4, 16, 8, 576, 512, 8, ctypes.c_float(0.1), None,
                            None, 0, None) == 1
    # a workspace that is not 256-byte aligned is refused before any device work
    assert L.ic_indexer_topk(fake, None, fake, 0, fake, None, 0, 1, 1, 16, 15, 64, 128, 8, fake,
                             P(0x10010), 1 << 20, None) == 6
    assert L.ic_sparse_attn(fake, fake, fake, 1, 1, 16, 8, 576, 512, 8, ctypes.c_float(0.1), fake,
                            P(0x10010), 1 << 20, None) == 6
    # empty problems are valid no-ops
    assert L.ic_indexer_topk(None, None, None, 0, None, None, 0, 0, 0, 0, 0, 64, 128, 8, None,
                             None, 0, None) == 0
    assert L.ic_debug_expire_wait(0, None) == 1


def test_layer_stack_rejects_bad_pattern_before_launching(ic):
    import torch  # noqa: F401  (ctypes structs only)
    from dsa_indexer_reuse_b200._binding import _LayerIO, _StackShape
    arr = (_LayerIO * 2)()
    shape = _StackShape(1, 16, 16, 0, 64, 128, 8, 0, 0, 64, 576, 512, 0.1)
    code = ic.lib.ic_layer_stack(arr, 2, 0, b"SF", ctypes.byref(shape), ctypes.c_void_p(0x10000),
                                 None, 0, None)
    assert code == 2
    code = ic.lib.ic_layer_stack(arr, 2, 1, b"FS", ctypes.byref(shape), ctypes.c_void_p(0x10000),
                                 None, 0, None)
    assert code == 1
    # Full layer with null indexer inputs is rejected before anything runs
    code = ic.lib.ic_layer_stack(arr, 2, 1, None, ctypes.byref(shape), ctypes.c_void_p(0x10000),
                                 None, 0, None)
    assert code == 1


def _host_stack_call(ic, alias_out_to_input):
    """ic_layer_stack_host on two host layers (pattern FS); layer 1's output
    either aliases layer 0's q buffer or has its own. No staging is passed,
    so a call that passes the host checks stops at the device query (no GPU)
    or at the staging check."""
    from dsa_indexer_reuse_b200 import _binding as B
    shape = dict(batch=1, n_q=64, n_k=64, q_pos0=0, H_I=4, d_I=64, topk=16, qk_dtype=B.BF16,
                 w_dtype=B.BF16, H=4, d_qk=64, d_v=64, sm_scale=0.125)
    buf = lambda n: np.zeros(n, np.uint16)
    keep = []
    def mk(**kw):
        vals = {}
        for k, a in kw.items():
            keep.append(a)
            vals[k] = None if a is None else a.ctypes.data
        return vals
    q0 = buf(64 * 4 * 64)
    l0 = mk(q_I=buf(64 * 4 * 64), q_scale=None, w=buf(64 * 4), k_I=buf(64 * 64), k_scale=None,
            q=q0, kv=buf(64 * 64), out=buf(64 * 4 * 64))
    out1 = q0 if alias_out_to_input else buf(64 * 4 * 64)
    l1 = mk(q_I=None, q_scale=None, w=None, k_I=None, k_scale=None, q=buf(64 * 4 * 64),
            kv=buf(64 * 64), out=out1)
    arr = (B._LayerIO * 2)(B._LayerIO(**l0), B._LayerIO(**l1))
    c_shape = B._stack_shape(shape)
    return ic.lib.ic_layer_stack_host(arr, 2, 0, b"FS", ctypes.byref(c_shape), None, None, 0, None,
                                      None, None)


def test_host_stack_refuses_an_output_that_overlaps_an_input(ic):
    assert _host_stack_call(ic, alias_out_to_input=True) == 1      # IC_ERR_INVALID_ARG
    assert _host_stack_call(ic, alias_out_to_input=False) in (4, 6)  # past the host checks


def test_distill_target_validates_on_the_host(ic):
    """Argument checks of ic_distill_target come before any device work."""
    lib = ic.lib
    q = np.zeros(16, np.uint16)
    arr = (ctypes.c_void_p * 2)(q.ctypes.data, q.ctypes.data)
    kl = np.zeros(4, np.float32)
    idx = np.zeros(64, np.int32)

    def call(n_served=1, d_qk=64, H=4, topk=16, H_I=4, d_I=64, batch=1, kl_ptr=kl.ctypes.data,
             qk=0, w=0):
        return lib.ic_distill_target(ctypes.cast(arr, ctypes.c_void_p), ctypes.cast(arr, ctypes.c_void_p),
                                     n_served, q.ctypes.data, None, q.ctypes.data, w, q.ctypes.data, None,
                                     qk, idx.ctypes.data, batch, 4, 64, H_I, d_I, topk, H, d_qk, 0.125,
                                     None, kl_ptr, None, 0, None)
    assert call(n_served=0) == 1                      # IC_ERR_INVALID_ARG
    assert call(kl_ptr=None) == 1
    assert call(qk=7) == 1 and call(w=1) == 1         # FP8 weights are not a w dtype
    assert call(qk=1) == 1                            # FP8 without scales
    assert call(n_served=65) == 3                     # IC_ERR_UNSUPPORTED
    assert call(d_qk=128) == 3 and call(H=65) == 3 and call(topk=4096) == 3
    assert call(H_I=8) == 3 and call(d_I=60) == 3
    assert call(batch=0) == 0                         # nothing to do


def test_distill_workspace_size_on_the_host(ic):
    """Shapes outside the tensor-core configuration need no workspace; the
    size query checks its arguments without touching a device."""
    lib = ic.lib
    out = ctypes.c_size_t(123)
    assert lib.ic_distill_target_workspace_size(1, 64, 2048, 4, 64, 4, 64, ctypes.byref(out)) == 0
    assert out.value == 0
    assert lib.ic_distill_target_workspace_size(1, 64, 2048, 4, 64, 4, 64, None) == 1
    assert lib.ic_distill_target_workspace_size(-1, 64, 2048, 64, 576, 64, 128, ctypes.byref(out)) == 1
    assert lib.ic_distill_target_workspace_size(1, 64, 0, 64, 576, 64, 128, ctypes.byref(out)) == 1
