"""ctypes marshalling for libindexcache.so (see include/indexcache.h).

Argument marshalling only: shapes and dtypes are read from the tensors, raw
device pointers and the current stream are handed to the C ABI, and a
non-zero status is raised as IcError.
"""

from __future__ import annotations

import ctypes
import math
import os

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# IC_LIB_PATH selects another build of the same C ABI (e.g. a debug build)
LIB_PATH = os.environ.get("IC_LIB_PATH") or os.path.join(_HERE, "libindexcache.so")

BF16, FP8_E4M3, F32 = 0, 1, 2
STATUS = {
    0: "IC_OK", 1: "IC_ERR_INVALID_ARG", 2: "IC_ERR_BAD_PATTERN", 3: "IC_ERR_UNSUPPORTED",
    4: "IC_ERR_CUDA", 5: "IC_ERR_TIMEOUT", 6: "IC_ERR_WORKSPACE", 7: "IC_ERR_INTERNAL",
}


class IcError(RuntimeError):
    def __init__(self, code, what="", detail=""):
        msg = "%s failed: %s" % (what, STATUS.get(code, str(code)))
        if detail:
            msg += " (%s)" % detail
        super().__init__(msg)
        self.code = code


if not os.path.exists(LIB_PATH):
    raise ImportError(
        "libindexcache.so is not built (run `python -m dsa_indexer_reuse_b200.build`); "
        "there is no fallback implementation")

lib = ctypes.CDLL(LIB_PATH)

_P = ctypes.c_void_p
_I = ctypes.c_int
_SZ = ctypes.c_size_t


class _LayerIO(ctypes.Structure):
    _fields_ = [("q_I", _P), ("q_scale", _P), ("w", _P), ("k_I", _P), ("k_scale", _P),
                ("q", _P), ("kv", _P), ("out", _P)]


class _StackShape(ctypes.Structure):
    _fields_ = [("batch", _I), ("n_q", _I), ("n_k", _I), ("q_pos0", _I), ("H_I", _I), ("d_I", _I),
                ("topk", _I), ("qk_dtype", _I), ("w_dtype", _I), ("H", _I), ("d_qk", _I),
                ("d_v", _I), ("sm_scale", ctypes.c_float)]


lib.ic_status_string.argtypes = [_I]
lib.ic_status_string.restype = ctypes.c_char_p
lib.ic_version.argtypes = []
lib.ic_version.restype = _I
lib.ic_resolve_pattern.argtypes = [_I, _I, ctypes.c_char_p, _P, _P]
lib.ic_resolve_pattern.restype = _I
lib.ic_indexer_workspace_size.argtypes = [_I, _I, _I, _I, _I, _I, _I, ctypes.POINTER(_SZ)]
lib.ic_indexer_workspace_size.restype = _I
lib.ic_indexer_topk.argtypes = [_P, _P, _P, _I, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _P, _P,
                                _SZ, _P]
lib.ic_indexer_topk.restype = _I
lib.ic_sparse_attn_workspace_size.argtypes = [_I, _I, _I, _I, _I, ctypes.POINTER(_SZ)]
lib.ic_sparse_attn_workspace_size.restype = _I
lib.ic_sparse_attn.argtypes = [_P, _P, _P, _I, _I, _I, _I, _I, _I, _I, ctypes.c_float, _P, _P,
                               _SZ, _P]
lib.ic_sparse_attn.restype = _I
lib.ic_layer_stack_workspace_size.argtypes = [ctypes.POINTER(_StackShape), ctypes.POINTER(_SZ)]
lib.ic_layer_stack_workspace_size.restype = _I
lib.ic_layer_stack.argtypes = [ctypes.POINTER(_LayerIO), _I, _I, ctypes.c_char_p,
                               ctypes.POINTER(_StackShape), _P, _P, _SZ, _P]
lib.ic_layer_stack.restype = _I
lib.ic_layer_stack_host_staging_size.argtypes = [ctypes.POINTER(_LayerIO), _I, ctypes.POINTER(_StackShape),
                                                 ctypes.POINTER(_SZ)]
lib.ic_layer_stack_host_staging_size.restype = _I
lib.ic_layer_stack_host.argtypes = [ctypes.POINTER(_LayerIO), _I, _I, ctypes.c_char_p,
                                    ctypes.POINTER(_StackShape), _P, _P, _SZ, _P,
                                    ctypes.POINTER(_SZ), ctypes.POINTER(_SZ)]
lib.ic_layer_stack_host.restype = _I
lib.ic_distill_target_workspace_size.argtypes = [_I, _I, _I, _I, _I, _I, _I, ctypes.POINTER(_SZ)]
lib.ic_distill_target_workspace_size.restype = _I
lib.ic_distill_target.argtypes = [_P, _P, _I, _P, _P, _P, _I, _P, _P, _I, _P, _I, _I, _I, _I, _I, _I,
                                  _I, _I, ctypes.c_float, _P, _P, _P, _SZ, _P]
lib.ic_distill_target.restype = _I
lib.ic_get_device_status.argtypes = [_I]
lib.ic_get_device_status.restype = _I
lib.ic_last_error_string.argtypes = []
lib.ic_last_error_string.restype = ctypes.c_char_p
lib.ic_debug_expire_wait.argtypes = [ctypes.c_longlong, _P]
lib.ic_debug_expire_wait.restype = _I
lib.ic_topk_overlap.argtypes = [_P, _P, _I, _I, _I, _P, _P]
lib.ic_topk_overlap.restype = _I
lib.ic_overlap_matrix_workspace_size.argtypes = [_I, ctypes.POINTER(_SZ)]
lib.ic_overlap_matrix_workspace_size.restype = _I
lib.ic_overlap_matrix.argtypes = [_P, _I, _I, _I, _I, _P, _SZ, _P, _P]
lib.ic_overlap_matrix.restype = _I
lib.ic_pattern_score.argtypes = [_P, _I, ctypes.c_char_p, ctypes.POINTER(ctypes.c_double)]
lib.ic_pattern_score.restype = _I
lib.ic_search_pattern.argtypes = [_P, _I, _I, ctypes.c_char_p, ctypes.POINTER(ctypes.c_double)]
lib.ic_search_pattern.restype = _I
_OBJECTIVE = ctypes.CFUNCTYPE(ctypes.c_double, ctypes.c_char_p, _P)
lib.ic_greedy_pattern.argtypes = [_I, _I, _OBJECTIVE, _P, ctypes.c_char_p, ctypes.POINTER(ctypes.c_double)]
lib.ic_greedy_pattern.restype = _I


def _check(code, what):
    if code != 0:
        detail = lib.ic_last_error_string().decode() if code == 4 else ""
        raise IcError(code, what, detail)


def version() -> int:
    return int(lib.ic_version())


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _qk_code(t):
    if t.dtype == torch.bfloat16:
        return BF16
    if t.dtype in (torch.uint8, torch.float8_e4m3fn):
        return FP8_E4M3
    raise TypeError("q_I/k_I must be bfloat16 or FP8 E4M3 (uint8 codes), got %s" % t.dtype)


def _w_code(t):
    if t.dtype == torch.bfloat16:
        return BF16
    if t.dtype == torch.float32:
        return F32
    raise TypeError("w must be bfloat16 or float32, got %s" % t.dtype)


def _dev(*ts):
    for t in ts:
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise ValueError("tensors must be contiguous CUDA tensors")


def resolve_pattern(n_layers: int, freq: int = 0, pattern: str | None = None):
    """Host-side F/S resolution; returns (is_full uint8[n], src int32[n])."""
    n = max(int(n_layers), 1)
    is_full = np.zeros(n, np.uint8)
    src = np.zeros(n, np.int32)
    code = lib.ic_resolve_pattern(int(n_layers), int(freq),
                                  None if pattern is None else pattern.encode(),
                                  is_full.ctypes.data, src.ctypes.data)
    _check(code, "ic_resolve_pattern")
    return is_full, src


def indexer_workspace_size(batch, n_q, n_k, H_I, d_I, topk, qk_dtype) -> int:
    out = _SZ(0)
    _check(lib.ic_indexer_workspace_size(batch, n_q, n_k, H_I, d_I, topk, qk_dtype,
                                         ctypes.byref(out)), "ic_indexer_workspace_size")
    return int(out.value)


def _workspace(nbytes, device, workspace):
    if nbytes == 0:
        return workspace, 0 if workspace is None else workspace.numel()
    if workspace is None or workspace.numel() < nbytes:
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=device)
    return workspace, workspace.numel()


def indexer_topk(q_I, w, k_I, topk, *, q_scale=None, k_scale=None, q_pos0=0, idx_out=None,
                 workspace=None, stream=None):
    """Fused lightning indexer + top-k. q_I [B, n_q, H_I, d_I], w [B, n_q, H_I],
    k_I [B, n_k, d_I] (bf16, or uint8 E4M3 codes with fp32 per-token scales).
    Returns idx [B, n_q, topk] int32 (ascending key order, -1 padded)."""
    _dev(q_I, w, k_I, q_scale, k_scale, idx_out)
    B, n_q, H_I, d_I = q_I.shape
    n_k = k_I.shape[1]
    qk = _qk_code(q_I)
    if idx_out is None:
        idx_out = torch.empty((B, n_q, topk), dtype=torch.int32, device=q_I.device)
    ws_bytes = indexer_workspace_size(B, n_q, n_k, H_I, d_I, topk, qk)
    workspace, ws_len = _workspace(ws_bytes, q_I.device, workspace)
    code = lib.ic_indexer_topk(_ptr(q_I), _ptr(q_scale), _ptr(w), _w_code(w), _ptr(k_I),
                               _ptr(k_scale), qk, B, n_q, n_k, int(q_pos0), H_I, d_I, int(topk),
                               _ptr(idx_out), _ptr(workspace), ws_len, _stream(stream))
    _check(code, "ic_indexer_topk")
    return idx_out


def sparse_attn_workspace_size(batch, n_q, H, d_v, topk) -> int:
    out = _SZ(0)
    _check(lib.ic_sparse_attn_workspace_size(batch, n_q, H, d_v, topk, ctypes.byref(out)),
           "ic_sparse_attn_workspace_size")
    return int(out.value)


def sparse_attn(q, kv, idx, *, d_v, sm_scale=None, out=None, workspace=None, stream=None):
    """Sparse attention. q [B, n_q, H, d_qk] bf16, kv [B, n_k, d_qk] bf16,
    idx [B, n_q, topk] int32. Returns out [B, n_q, H, d_v] bf16."""
    _dev(q, kv, idx, out)
    B, n_q, H, d_qk = q.shape
    n_k = kv.shape[1]
    topk = idx.shape[-1]
    if sm_scale is None:
        sm_scale = 1.0 / math.sqrt(d_qk)
    if out is None:
        out = torch.empty((B, n_q, H, d_v), dtype=torch.bfloat16, device=q.device)
    ws_bytes = sparse_attn_workspace_size(B, n_q, H, d_v, topk)
    workspace, ws_len = _workspace(ws_bytes, q.device, workspace)
    code = lib.ic_sparse_attn(_ptr(q), _ptr(kv), _ptr(idx), B, n_q, n_k, H, d_qk, d_v, topk,
                              float(sm_scale), _ptr(out), _ptr(workspace), ws_len, _stream(stream))
    _check(code, "ic_sparse_attn")
    return out


def _stack_shape(shape: dict):
    return _StackShape(shape["batch"], shape["n_q"], shape["n_k"], shape.get("q_pos0", 0),
                       shape["H_I"], shape["d_I"], shape["topk"], shape["qk_dtype"],
                       shape["w_dtype"], shape["H"], shape["d_qk"], shape["d_v"],
                       float(shape["sm_scale"]))


def layer_stack_workspace_size(shape: dict) -> int:
    out = _SZ(0)
    s = _stack_shape(shape)
    _check(lib.ic_layer_stack_workspace_size(ctypes.byref(s), ctypes.byref(out)),
           "ic_layer_stack_workspace_size")
    return int(out.value)


class StackCall:
    """A prepared ic_layer_stack call: marshalled once, launched many times
    (the pointer structs stay alive with this object)."""

    def __init__(self, layers, shape: dict, *, freq=0, pattern=None, idx_buffer=None,
                 workspace=None):
        self.shape = dict(shape)
        self.freq = int(freq)
        self.pattern = None if pattern is None else pattern.encode()
        dev = layers[0]["q"].device
        B, n_q, topk = shape["batch"], shape["n_q"], shape["topk"]
        if idx_buffer is None:
            idx_buffer = torch.empty((B, n_q, topk), dtype=torch.int32, device=dev)
        self.idx_buffer = idx_buffer
        ws_bytes = layer_stack_workspace_size(shape)
        self.workspace, self.ws_len = _workspace(ws_bytes, dev, workspace)
        self.arr = (_LayerIO * len(layers))()
        self.keep = []
        for i, L in enumerate(layers):
            vals = {}
            for k in ("q_I", "q_scale", "w", "k_I", "k_scale", "q", "kv", "out"):
                t = L.get(k)
                _dev(t)
                self.keep.append(t)
                vals[k] = None if t is None else t.data_ptr()
            self.arr[i] = _LayerIO(**vals)
        self.n = len(layers)
        self.c_shape = _stack_shape(shape)

    def __call__(self, stream=None):
        code = lib.ic_layer_stack(self.arr, self.n, self.freq, self.pattern,
                                  ctypes.byref(self.c_shape), _ptr(self.idx_buffer),
                                  _ptr(self.workspace), self.ws_len, _stream(stream))
        _check(code, "ic_layer_stack")
        return self.idx_buffer


def layer_stack(layers, shape: dict, *, freq=0, pattern=None, idx_buffer=None, workspace=None,
                stream=None):
    """Run the IndexCache layer loop. `layers`: list of dicts of CUDA tensors
    (q_I, q_scale, w, k_I, k_scale, q, kv, out; indexer entries may be None
    on Shared layers). Returns the index buffer (last Full layer's indices)."""
    call = StackCall(layers, shape, freq=freq, pattern=pattern, idx_buffer=idx_buffer,
                     workspace=workspace)
    return call(stream)


class StackHostCall:
    """A prepared ic_layer_stack_host call: the layers' tensors may be CPU
    tensors (page-locked ones let the copies overlap the kernels) or CUDA
    tensors (used in place, e.g. a resident KV cache); CPU `out` tensors
    receive each layer's output. The device staging area is allocated once
    here, on `device`."""

    def __init__(self, layers, shape: dict, *, freq=0, pattern=None, idx_out=None, device=None,
                 staging=None):
        self.shape = dict(shape)
        self.freq = int(freq)
        self.pattern = None if pattern is None else pattern.encode()
        self.arr = (_LayerIO * len(layers))()
        self.keep = []
        for i, L in enumerate(layers):
            vals = {}
            for k in ("q_I", "q_scale", "w", "k_I", "k_scale", "q", "kv", "out"):
                t = L.get(k)
                if t is not None and not t.is_contiguous():
                    raise ValueError("tensors must be contiguous")
                self.keep.append(t)
                vals[k] = None if t is None else t.data_ptr()
            self.arr[i] = _LayerIO(**vals)
        self.n = len(layers)
        self.c_shape = _stack_shape(shape)
        if idx_out is not None and not idx_out.is_contiguous():
            raise ValueError("idx_out must be contiguous")
        self.idx_out = idx_out
        size = _SZ(0)
        _check(lib.ic_layer_stack_host_staging_size(self.arr, self.n, ctypes.byref(self.c_shape),
                                                    ctypes.byref(size)), "ic_layer_stack_host_staging_size")
        device = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
        if staging is None or staging.numel() < size.value:
            staging = torch.empty(max(int(size.value), 1), dtype=torch.uint8, device=device)
        self.staging = staging

    def __call__(self, stream=None):
        h2d, d2h = _SZ(0), _SZ(0)
        code = lib.ic_layer_stack_host(self.arr, self.n, self.freq, self.pattern, ctypes.byref(self.c_shape),
                                       _ptr(self.idx_out), _ptr(self.staging), self.staging.numel(),
                                       _stream(stream), ctypes.byref(h2d), ctypes.byref(d2h))
        _check(code, "ic_layer_stack_host")
        self.h2d_bytes, self.d2h_bytes = int(h2d.value), int(d2h.value)  # bytes this call copies
        return self.idx_out


def layer_stack_host(layers, shape: dict, *, freq=0, pattern=None, idx_out=None, stream=None):
    """Run the IndexCache layer loop on tensors that may live in host memory
    (see StackHostCall). Asynchronous on `stream`: synchronise it before
    reading CPU outputs."""
    return StackHostCall(layers, shape, freq=freq, pattern=pattern, idx_out=idx_out)(stream)


def distill_target_workspace_size(batch, n_q, topk, H, d_qk, H_I, d_I) -> int:
    out = _SZ(0)
    _check(lib.ic_distill_target_workspace_size(batch, n_q, topk, H, d_qk, H_I, d_I, ctypes.byref(out)),
           "ic_distill_target_workspace_size")
    return int(out.value)


def distill_target(served, q_I, w, k_I, idx, *, q_scale=None, k_scale=None, sm_scale=None,
                   with_target=True, workspace=None, stream=None):
    """Multi-layer distillation target of one Full layer (ic_distill_target).
    `served`: list of (q [B, n_q, H, d_qk], kv [B, n_k, d_qk]) bf16 tensors of
    the layers it serves (itself first, by convention); q_I, w, k_I (and the
    FP8 scales) are its indexer tensors and idx [B, n_q, topk] its index rows.
    Returns (target [B, n_q, topk] fp32 or None, kl [B, n_q] fp32)."""
    _dev(q_I, w, k_I, idx, q_scale, k_scale)
    for q, kv in served:
        _dev(q, kv)
    B, n_q, H, d_qk = served[0][0].shape
    n_k = served[0][1].shape[1]
    H_I, d_I = q_I.shape[2], q_I.shape[3]
    topk = idx.shape[-1]
    if sm_scale is None:
        sm_scale = 1.0 / math.sqrt(d_qk)
    q_arr = (ctypes.c_void_p * len(served))(*[q.data_ptr() for q, _ in served])
    kv_arr = (ctypes.c_void_p * len(served))(*[kv.data_ptr() for _, kv in served])
    dev = idx.device
    target = torch.empty((B, n_q, topk), dtype=torch.float32, device=dev) if with_target else None
    kl = torch.empty((B, n_q), dtype=torch.float32, device=dev)
    ws_bytes = distill_target_workspace_size(B, n_q, topk, H, d_qk, H_I, d_I)
    workspace, ws_len = _workspace(ws_bytes, dev, workspace)
    code = lib.ic_distill_target(ctypes.cast(q_arr, ctypes.c_void_p), ctypes.cast(kv_arr, ctypes.c_void_p),
                                 len(served), _ptr(q_I), _ptr(q_scale), _ptr(w), _w_code(w), _ptr(k_I),
                                 _ptr(k_scale), _qk_code(q_I), _ptr(idx), B, n_q, n_k, H_I, d_I, topk, H,
                                 d_qk, float(sm_scale), _ptr(target), _ptr(kl), _ptr(workspace), ws_len,
                                 _stream(stream))
    _check(code, "ic_distill_target")
    return target, kl


def get_device_status(reset: bool = False) -> int:
    return int(lib.ic_get_device_status(1 if reset else 0))


def debug_expire_wait(timeout_ns: int, stream=None) -> None:
    _check(lib.ic_debug_expire_wait(int(timeout_ns), _stream(stream)), "ic_debug_expire_wait")


# --------------------------------------------------------------------------- pattern tools
def topk_overlap(idx_a, idx_b, n_k: int, *, counts_out=None, stream=None):
    """Per-row |valid(idx_a[r]) & valid(idx_b[r])| of two index tensors of the
    same shape [..., topk] (int32, as indexer_topk writes them). Returns an
    int32 tensor of the leading shape."""
    _dev(idx_a, idx_b, counts_out)
    if idx_a.shape != idx_b.shape or idx_a.dtype != torch.int32 or idx_b.dtype != torch.int32:
        raise ValueError("index tensors must be int32 of one shape")
    topk = idx_a.shape[-1]
    rows = idx_a.numel() // max(topk, 1)
    if counts_out is None:
        counts_out = torch.empty(idx_a.shape[:-1], dtype=torch.int32, device=idx_a.device)
    _check(lib.ic_topk_overlap(_ptr(idx_a), _ptr(idx_b), rows, topk, int(n_k), _ptr(counts_out),
                               _stream(stream)), "ic_topk_overlap")
    return counts_out


def overlap_matrix(idx_layers, n_k: int, stream=None) -> np.ndarray:
    """Layer x layer overlap ratios from each layer's own index tensor
    (ic_overlap_matrix): R[a][b] = sum_rows |T_a & T_b| / sum_rows |T_a|, the
    share of layer a's selections that layer b also selects. Synchronises
    the stream."""
    n = len(idx_layers)
    if n == 0:
        raise ValueError("no index tensors")
    _dev(*idx_layers)
    shape = idx_layers[0].shape
    if any(t.shape != shape or t.dtype != torch.int32 for t in idx_layers):
        raise ValueError("index tensors must be int32 of one shape")
    topk = shape[-1]
    rows = idx_layers[0].numel() // max(topk, 1)
    size = _SZ(0)
    _check(lib.ic_overlap_matrix_workspace_size(n, ctypes.byref(size)), "ic_overlap_matrix_workspace_size")
    ws = torch.empty(int(size.value), dtype=torch.uint8, device=idx_layers[0].device)
    ptrs = (ctypes.c_void_p * n)(*[t.data_ptr() for t in idx_layers])
    R = np.zeros((n, n), np.float64)
    _check(lib.ic_overlap_matrix(ptrs, n, rows, topk, int(n_k), _ptr(ws), ws.numel(), R.ctypes.data,
                                 _stream(stream)), "ic_overlap_matrix")
    return R


def pattern_score(overlap, pattern: str) -> float:
    """The pattern-search objective of one F/S pattern (ic_pattern_score):
    sum over layers of overlap[l][nearest Full layer at or before l]."""
    m = np.ascontiguousarray(overlap, dtype=np.float64)
    n = m.shape[0]
    if m.shape != (n, n):
        raise ValueError("overlap must be square")
    out = ctypes.c_double(0.0)
    _check(lib.ic_pattern_score(m.ctypes.data, n, pattern.encode(), ctypes.byref(out)), "ic_pattern_score")
    return float(out.value)


def search_pattern(overlap, n_full: int):
    """Best F/S pattern (layer 0 Full, n_full Full layers) under an overlap
    matrix (host, exact). Returns (pattern, score)."""
    m = np.ascontiguousarray(overlap, dtype=np.float64)
    n = m.shape[0]
    if m.shape != (n, n):
        raise ValueError("overlap must be square")
    out = ctypes.create_string_buffer(n + 1)
    score = ctypes.c_double(0.0)
    _check(lib.ic_search_pattern(m.ctypes.data, n, int(n_full), out, ctypes.byref(score)),
           "ic_search_pattern")
    return out.value.decode(), float(score.value)


def greedy_pattern(n_layers: int, n_full: int, objective):
    """Greedy indexer removal (host): objective(pattern: str) -> float, lower
    is better. Returns (pattern, objective value)."""
    err = []

    def cb(pat, _ctx):
        try:
            return float(objective(pat.decode()))
        except Exception as e:  # surfaced after the C call returns
            err.append(e)
            return float("nan")

    fn = _OBJECTIVE(cb)
    out = ctypes.create_string_buffer(int(n_layers) + 1)
    value = ctypes.c_double(0.0)
    code = lib.ic_greedy_pattern(int(n_layers), int(n_full), fn, None, out, ctypes.byref(value))
    if err:
        raise err[0]
    _check(code, "ic_greedy_pattern")
    return out.value.decode(), float(value.value)
