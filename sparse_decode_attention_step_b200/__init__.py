"""Python binding of the SAGA + Atop-N decode attention library (sm_100a).

A thin ctypes layer over ``include/saga.h``: the same entry points, the same
argument order, and argument marshalling only (device pointers from torch
tensors or plain integers, the CUDA stream handle). Every step of the
computation runs in the CUDA library ``_lib/libsaga_b200.so``; there is no
fallback, and every call fails loudly if the library is missing or returns an
error status.
"""
import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
# SAGA_CHECKED_BUILD=1 selects the bounds-checked build (build.py --check)
LIB_PATH = os.path.join(_HERE, "_lib", "libsaga_b200_check.so"
                        if os.environ.get("SAGA_CHECKED_BUILD") == "1" else "libsaga_b200.so")

SAGA_OK = 0
SAGA_ERR_INVALID_ARG = 1
SAGA_ERR_UNSUPPORTED = 2
SAGA_ERR_WORKSPACE = 3
SAGA_ERR_CUDA = 4
SAGA_ERR_DEVICE = 5
SAGA_F32 = 0
SAGA_BF16 = 1
DEVERR_LKV_NEGATIVE = 1
DEVERR_LKV_TOO_LONG = 2


class SagaError(RuntimeError):
    def __init__(self, status, where):
        self.status = status
        msg = f"{where}: {status_string(status)} (status {status})"
        if status == SAGA_ERR_CUDA:
            msg += f": {last_error()}"
        super().__init__(msg)


class saga_shape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("h_q", ctypes.c_int32), ("h_k", ctypes.c_int32),
                ("h_v", ctypes.c_int32), ("d", ctypes.c_int32), ("dtype", ctypes.c_int32),
                ("cap", ctypes.c_int64), ("max_l_kv", ctypes.c_int64),
                ("q_stride_b", ctypes.c_int64), ("q_stride_h", ctypes.c_int64),
                ("k_stride_b", ctypes.c_int64), ("k_stride_h", ctypes.c_int64),
                ("v_stride_b", ctypes.c_int64), ("v_stride_h", ctypes.c_int64)]


class saga_merge_shape(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int32), ("d_model", ctypes.c_int32), ("h_q", ctypes.c_int32),
                ("h_k", ctypes.c_int32), ("d", ctypes.c_int32)]


_lib = None
_P = ctypes.c_void_p
_SP = ctypes.POINTER(saga_shape)
_MP = ctypes.POINTER(saga_merge_shape)

_SIGS = {
    "saga_shape_contiguous": (None, [_SP, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                     ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                     ctypes.c_int64, ctypes.c_int64]),
    "saga_workspace_size": (ctypes.c_size_t, [_SP, ctypes.c_int32]),
    "saga_workspace_init": (ctypes.c_int, [_P, ctypes.c_size_t, _P]),
    "saga_decode_step": (ctypes.c_int, [_SP, _P, _P, _P, _P, _P, _P, _P, _P, _P,
                                        ctypes.c_size_t, _P]),
    "saga_refresh_threshold": (ctypes.c_int, [_SP, _P, _P, _P, _P, ctypes.c_int32, _P, _P,
                                              _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "gqa_dense_decode": (ctypes.c_int, [_SP, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "saga_dense_decode": (ctypes.c_int, [_SP, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "saga_append_kv": (ctypes.c_int, [_SP, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "saga_topn_step": (ctypes.c_int, [_SP, _P, _P, _P, _P, ctypes.c_int32, _P, _P, _P, _P, _P,
                                      ctypes.c_size_t, _P]),
    "saga_debug_scores": (ctypes.c_int, [_SP, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "saga_decode_step_noalloc": (ctypes.c_int, [_SP, _P, _P, _P, _P, _P, _P, _P, _P]),
    "saga_read_device_error": (ctypes.c_int, [_P, _P, ctypes.POINTER(ctypes.c_int32)]),
    "saga_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "saga_last_error": (ctypes.c_char_p, []),
    "saga_merge_workspace_size": (ctypes.c_size_t, [_MP]),
    "saga_merge_keys": (ctypes.c_int, [_MP, _P, _P, _P, ctypes.c_double, _P, _P, _P, _P, _P,
                                       ctypes.c_size_t, _P]),
}


def load():
    """Load the CUDA library (once). Raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise FileNotFoundError(
                f"{LIB_PATH} is missing: build it with "
                "`python sparse_decode_attention_step_b200/build.py`")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def _ptr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(s):
    if s is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _check(rc, where):
    if rc != SAGA_OK:
        raise SagaError(rc, where)


def status_string(status):
    return load().saga_status_string(status).decode()


def last_error():
    """The last CUDA failure a library call saw on this thread (or "")."""
    return load().saga_last_error().decode()


def shape(B, h_q, h_k, h_v, d, dtype, cap, max_l_kv=None):
    """A saga_shape for contiguous q [B][h_q][d], K [B][h_k][cap][d], V [B][h_v][cap][d]."""
    s = saga_shape()
    load().saga_shape_contiguous(ctypes.byref(s), B, h_q, h_k, h_v, d, dtype, cap,
                                 cap if max_l_kv is None else max_l_kv)
    return s


def workspace_size(shp, N=1):
    return int(load().saga_workspace_size(ctypes.byref(shp), N))


def workspace_init(ws, nbytes, stream=None):
    _check(load().saga_workspace_init(_ptr(ws), nbytes, _stream(stream)), "saga_workspace_init")


class Workspace:
    """Device workspace for one shape, allocated through torch and zeroed."""

    def __init__(self, shp, N=1, device="cuda", stream=None):
        import torch
        self.nbytes = workspace_size(shp, N)
        if self.nbytes == 0:
            raise SagaError(SAGA_ERR_INVALID_ARG, "saga_workspace_size")
        self.buf = torch.empty(self.nbytes, dtype=torch.uint8, device=device)
        workspace_init(self.buf, self.nbytes, stream)

    def data_ptr(self):
        return self.buf.data_ptr()


def _ws(ws):
    return _ptr(ws), ws.nbytes


def decode_step(shp, q, K, V, l_kv, tau, out, ws, sel_count=None, sel_mask=None, stream=None):
    p, n = _ws(ws)
    _check(load().saga_decode_step(ctypes.byref(shp), _ptr(q), _ptr(K), _ptr(V), _ptr(l_kv),
                                   _ptr(tau), _ptr(out), _ptr(sel_count), _ptr(sel_mask), p, n,
                                   _stream(stream)), "saga_decode_step")


def refresh_threshold(shp, q, K, l_kv, N, tau, ws, V=None, out=None, sel_count=None,
                      sel_mask=None, scores=None, stream=None):
    p, n = _ws(ws)
    _check(load().saga_refresh_threshold(ctypes.byref(shp), _ptr(q), _ptr(K), _ptr(V),
                                         _ptr(l_kv), N, _ptr(tau), _ptr(out), _ptr(sel_count),
                                         _ptr(sel_mask), _ptr(scores), p, n, _stream(stream)),
           "saga_refresh_threshold")


def gqa_dense_decode(shp, q, K, V, l_kv, out, ws, stream=None):
    p, n = _ws(ws)
    _check(load().gqa_dense_decode(ctypes.byref(shp), _ptr(q), _ptr(K), _ptr(V), _ptr(l_kv),
                                   _ptr(out), p, n, _stream(stream)), "gqa_dense_decode")


def dense_decode(shp, q, K, V, l_kv, out, ws, stream=None):
    """Full attention with the shape's key and value head maps (SAGA full
    attention when h_k < h_v, GQA full attention when h_k == h_v)."""
    p, n = _ws(ws)
    _check(load().saga_dense_decode(ctypes.byref(shp), _ptr(q), _ptr(K), _ptr(V), _ptr(l_kv),
                                    _ptr(out), p, n, _stream(stream)), "saga_dense_decode")


def topn_step(shp, q, K, V, l_kv, N, out, ws, sel_count=None, sel_mask=None, scores=None,
              stream=None):
    """Exact top-N attention (ties to the lower position) for this step."""
    p, n = _ws(ws)
    _check(load().saga_topn_step(ctypes.byref(shp), _ptr(q), _ptr(K), _ptr(V), _ptr(l_kv), N,
                                 _ptr(out), _ptr(sel_count), _ptr(sel_mask), _ptr(scores), p, n,
                                 _stream(stream)), "saga_topn_step")


def append_kv(shp, k_new, v_new, K, V, l_kv, ws, stream=None):
    """Write the token's key/value rows at position l_kv[b] and grow l_kv."""
    p, n = _ws(ws)
    _check(load().saga_append_kv(ctypes.byref(shp), _ptr(k_new), _ptr(v_new), _ptr(K), _ptr(V),
                                 _ptr(l_kv), p, n, _stream(stream)), "saga_append_kv")


NOALLOC_SCRATCH_BYTES = 160 << 20


def decode_step_noalloc(shp, q, K, V, l_kv, tau, out, sel_count=None, stream=None):
    """saga_decode_step with the library's fixed device scratch instead of a
    workspace, for callers that cannot allocate device memory."""
    _check(load().saga_decode_step_noalloc(ctypes.byref(shp), _ptr(q), _ptr(K), _ptr(V),
                                           _ptr(l_kv), _ptr(tau), _ptr(out), _ptr(sel_count),
                                           _stream(stream)), "saga_decode_step_noalloc")


def debug_scores(shp, q, K, l_kv, scores, ws, stream=None):
    p, n = _ws(ws)
    _check(load().saga_debug_scores(ctypes.byref(shp), _ptr(q), _ptr(K), _ptr(l_kv),
                                    _ptr(scores), p, n, _stream(stream)), "saga_debug_scores")


def read_device_error(ws, stream=None):
    """Synchronise, return and clear the device error word (0 = clean)."""
    flags = ctypes.c_int32(0)
    rc = load().saga_read_device_error(_ptr(ws), _stream(stream), ctypes.byref(flags))
    if rc not in (SAGA_OK, SAGA_ERR_DEVICE):
        raise SagaError(rc, "saga_read_device_error")
    return flags.value


# ---------------------------------------------------------------------------
# closed-form GQA-to-SAGA key-head merge (include/saga_merge.h)
# ---------------------------------------------------------------------------
def merge_shape(T, d_model, h_q, h_k, d):
    return saga_merge_shape(T, d_model, h_q, h_k, d)


def merge_workspace_size(mshape):
    return int(load().saga_merge_workspace_size(ctypes.byref(mshape)))


class MergeWorkspace:
    """Device workspace for saga_merge_keys, allocated through torch; its
    error word is zeroed."""

    def __init__(self, mshape, device="cuda", stream=None):
        import torch
        self.nbytes = merge_workspace_size(mshape)
        if self.nbytes == 0:
            raise SagaError(SAGA_ERR_INVALID_ARG, "saga_merge_workspace_size")
        self.buf = torch.empty(self.nbytes, dtype=torch.uint8, device=device)
        workspace_init(self.buf, self.nbytes, stream)

    def data_ptr(self):
        return self.buf.data_ptr()


def merge_keys(mshape, X, W_K, Q, rcond, w, pairs, W_S, ws, total=None, stream=None):
    """Pair weights w [h_k][h_k] (float64), the minimum-weight pairing
    pairs [h_k/2][2] (int32) and the student's key projection
    W_S [h_k/2*d][d_model] (float32) from bf16 X [T][d_model],
    W_K [h_k*d][d_model] and Q [T][h_q*d]."""
    p, n = _ws(ws)
    _check(load().saga_merge_keys(ctypes.byref(mshape), _ptr(X), _ptr(W_K), _ptr(Q),
                                  float(rcond), _ptr(w), _ptr(pairs), _ptr(total), _ptr(W_S),
                                  p, n, _stream(stream)), "saga_merge_keys")
