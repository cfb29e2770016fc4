"""Python binding of libnsa, the B200 Native Sparse Attention library.

Argument marshalling only: every function here forwards to the C entry point
of the same name (include/nsa.h) with raw device pointers taken from torch
tensors, and the current torch CUDA stream unless one is given.  All
arithmetic runs in the library's CUDA kernels; if ``libnsa.so`` has not been
built, importing the entry points raises instead of falling back to anything.
"""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libnsa.so")

NSA_OK, NSA_ERR_INVALID_ARG, NSA_ERR_UNSUPPORTED, NSA_ERR_WORKSPACE, NSA_ERR_CUDA, NSA_ERR_TIMEOUT = range(6)
NSA_CODE_CU_SEQLENS = 200   # status word: a variable-length call's cu_seqlens broke its rules
NSA_MODE_NSA, NSA_MODE_MOBA, NSA_MODE_DSA = 0, 1, 2
NSA_MAP_TOUCH, NSA_MAP_CONTAINED, NSA_MAP_OVERLAP = 0, 1, 2

EXPORTED = ("nsa_workspace_size", "nsa_compress", "nsa_compress_append", "nsa_compress_mlp",
            "nsa_compress_append_mlp", "nsa_forward", "nsa_forward_varlen",
            "nsa_dsa_forward", "nsa_backward", "nsa_backward_ex", "nsa_decode",
            "nsa_forward_noalloc", "nsa_device_status", "nsa_device_status_noalloc", "nsa_selftest_wait_timeout",
            "nsa_status_string")


class NsaGrads(ctypes.Structure):
    """Mirror of ``nsa_grads`` in include/nsa.h: the fp32 gradient outputs of nsa_backward_ex."""
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("dq", "dk", "dv", "dgates", "dw_k", "dw_v", "db_k", "db_v", "dw_k2", "dw_v2")]


class NsaConfig(ctypes.Structure):
    """Mirror of ``nsa_config`` in include/nsa.h (field order and types must match)."""
    _fields_ = [
        ("mode", ctypes.c_int32),
        ("batch", ctypes.c_int32), ("seqlen", ctypes.c_int32), ("h_q", ctypes.c_int32),
        ("h_kv", ctypes.c_int32), ("d_k", ctypes.c_int32), ("d_v", ctypes.c_int32),
        ("cmp_block", ctypes.c_int32), ("cmp_stride", ctypes.c_int32), ("sel_block", ctypes.c_int32),
        ("top_k", ctypes.c_int32), ("window", ctypes.c_int32),
        ("force_first", ctypes.c_int32), ("force_local", ctypes.c_int32),
        ("softmax_scale", ctypes.c_float),
        ("w_cmp_k", ctypes.c_void_p), ("w_cmp_v", ctypes.c_void_p),
        ("sel_idx_out", ctypes.c_void_p),
        ("kc_out", ctypes.c_void_p), ("vc_out", ctypes.c_void_p),
        ("workspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_size_t),
        ("stage_events", ctypes.POINTER(ctypes.c_void_p)), ("n_stage_events", ctypes.c_int32),
        ("score_map", ctypes.c_int32),
        ("phi_mlp", ctypes.c_int32),
        ("w_cmp_k2", ctypes.c_void_p), ("w_cmp_v2", ctypes.c_void_p),
        ("b_cmp_k", ctypes.c_void_p), ("b_cmp_v", ctypes.c_void_p),
    ]


class NsaError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {nsa_status_string(status)} ({status})")
        self.status = status


_lib = None


def load_library() -> ctypes.CDLL:
    """Load libnsa.so from the package directory (raises if it is missing)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is not built; run `python -m block_sparse_attention_compress_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
    cfgp = ctypes.POINTER(NsaConfig)
    lib.nsa_workspace_size.argtypes = [cfgp, ctypes.c_int]
    lib.nsa_workspace_size.restype = sz
    lib.nsa_compress.argtypes = [vp, vp, i32, i32, i32, i32, i32, i32, i32, vp, vp]
    lib.nsa_compress.restype = ctypes.c_int
    lib.nsa_compress_append.argtypes = [vp, vp, vp, i32, i32, i32, i32, i32, i32, i32, vp, i32, vp]
    lib.nsa_compress_append.restype = ctypes.c_int
    lib.nsa_compress_mlp.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, vp, vp, vp]
    lib.nsa_compress_mlp.restype = ctypes.c_int
    lib.nsa_compress_append_mlp.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, vp, vp, i32, vp]
    lib.nsa_compress_append_mlp.restype = ctypes.c_int
    lib.nsa_forward.argtypes = [vp, vp, vp, vp, cfgp, vp, vp]
    lib.nsa_backward.restype = ctypes.c_int
    lib.nsa_backward.argtypes = [vp, vp, vp, vp, vp, vp, cfgp, vp, vp, vp, vp, vp, vp, vp]
    lib.nsa_backward_ex.restype = ctypes.c_int
    lib.nsa_backward_ex.argtypes = [vp, vp, vp, vp, vp, vp, vp, i32, cfgp, ctypes.POINTER(NsaGrads), vp]
    lib.nsa_dsa_forward.restype = ctypes.c_int
    lib.nsa_dsa_forward.argtypes = [vp, vp, vp, vp, vp, vp, i32, i32, cfgp, vp, vp, vp]
    lib.nsa_forward_varlen.restype = ctypes.c_int
    lib.nsa_forward_varlen.argtypes = [vp, vp, vp, vp, vp, i32, cfgp, vp, vp]
    lib.nsa_forward.restype = ctypes.c_int
    lib.nsa_decode.argtypes = [vp, vp, vp, vp, vp, vp, i32, vp, cfgp, vp, vp]
    lib.nsa_decode.restype = ctypes.c_int
    lib.nsa_forward_noalloc.argtypes = [vp, vp, vp, vp, cfgp, vp, vp]
    lib.nsa_forward_noalloc.restype = ctypes.c_int
    lib.nsa_device_status.argtypes = [vp, ctypes.POINTER(i32), vp]
    lib.nsa_device_status.restype = ctypes.c_int
    lib.nsa_device_status_noalloc.argtypes = [ctypes.POINTER(i32), vp]
    lib.nsa_device_status_noalloc.restype = ctypes.c_int
    lib.nsa_selftest_wait_timeout.argtypes = [vp, sz, ctypes.c_uint32, vp]
    lib.nsa_selftest_wait_timeout.restype = ctypes.c_int
    lib.nsa_status_string.argtypes = [ctypes.c_int]
    lib.nsa_status_string.restype = ctypes.c_char_p
    _lib = lib
    return lib


def _ptr(x) -> int | None:
    if x is None:
        return None
    if isinstance(x, int):
        return x
    if not x.is_contiguous():
        raise ValueError("tensors passed to libnsa must be contiguous")
    return x.data_ptr()


def _stream(stream, *tensors) -> int | None:
    if stream is not None:
        return stream if isinstance(stream, int) else stream.cuda_stream
    import torch
    for t in tensors:
        if t is not None and not isinstance(t, int) and t.is_cuda:
            return torch.cuda.current_stream(t.device).cuda_stream
    return None


def make_config(**fields) -> NsaConfig:
    """Build an NsaConfig; tensors given for pointer fields are replaced by their addresses."""
    cfg = NsaConfig()
    defaults = dict(mode=NSA_MODE_NSA, cmp_block=32, cmp_stride=16, sel_block=64, top_k=16, window=512,
                    force_first=1, force_local=1, softmax_scale=0.0)
    defaults.update(fields)
    for name, val in defaults.items():
        if name in ("w_cmp_k", "w_cmp_v", "sel_idx_out", "kc_out", "vc_out", "workspace", "w_cmp_k2", "w_cmp_v2",
                    "b_cmp_k", "b_cmp_v"):
            val = _ptr(val)
        setattr(cfg, name, val)
    return cfg


def nsa_status_string(status: int) -> str:
    return load_library().nsa_status_string(int(status)).decode()


def nsa_workspace_size(cfg: NsaConfig, decode_batch: int = 0) -> int:
    return int(load_library().nsa_workspace_size(ctypes.byref(cfg), int(decode_batch)))


def _check(status: int, where: str) -> int:
    if status != NSA_OK:
        raise NsaError(status, where)
    return status


def nsa_compress(x, w, out, l: int = 32, s: int = 16, stream=None, check: bool = True) -> int:
    """phi over [B, T, H, d] -> out [B, N_c, H, d_out] (see include/nsa.h)."""
    B, T, H, d = x.shape
    st = load_library().nsa_compress(_ptr(x), _ptr(w), B, T, H, d, w.shape[1], l, s, _ptr(out),
                                     _stream(stream, x))
    return _check(st, "nsa_compress") if check else st


def nsa_compress_append(x_cache, w, seqlens, out_cache, l: int = 32, s: int = 16, stream=None,
                        check: bool = True) -> int:
    """Write the compressed block that each sequence's newest token completes (see include/nsa.h)."""
    B, Lmax, H, d = x_cache.shape
    st = load_library().nsa_compress_append(_ptr(x_cache), _ptr(w), _ptr(seqlens), B, Lmax, H, d, w.shape[1], l, s,
                                            _ptr(out_cache), out_cache.shape[1], _stream(stream, x_cache))
    return _check(st, "nsa_compress_append") if check else st


def nsa_compress_mlp(x, w1, b1, w2, hidden, out, l: int = 32, s: int = 16, stream=None, check: bool = True) -> int:
    """phi as the two-layer MLP over [B, T, H, d]; hidden and out [B, N_c, H, d] (see include/nsa.h)."""
    B, T, H, d = x.shape
    st = load_library().nsa_compress_mlp(_ptr(x), _ptr(w1), _ptr(b1), _ptr(w2), B, T, H, d, l, s, _ptr(hidden),
                                         _ptr(out), _stream(stream, x))
    return _check(st, "nsa_compress_mlp") if check else st


def nsa_compress_append_mlp(x_cache, w1, b1, w2, seqlens, hidden, out_cache, l: int = 32, s: int = 16, stream=None,
                            check: bool = True) -> int:
    """nsa_compress_append with phi as the two-layer MLP; hidden is scratch [B, H, d] (see include/nsa.h)."""
    B, Lmax, H, d = x_cache.shape
    st = load_library().nsa_compress_append_mlp(_ptr(x_cache), _ptr(w1), _ptr(b1), _ptr(w2), _ptr(seqlens), B, Lmax,
                                                H, d, l, s, _ptr(hidden), _ptr(out_cache), out_cache.shape[1],
                                                _stream(stream, x_cache))
    return _check(st, "nsa_compress_append_mlp") if check else st


def nsa_forward(q, k, v, gates, cfg: NsaConfig, out, stream=None, check: bool = True) -> int:
    st = load_library().nsa_forward(_ptr(q), _ptr(k), _ptr(v), _ptr(gates), ctypes.byref(cfg), _ptr(out),
                                    _stream(stream, q))
    return _check(st, "nsa_forward") if check else st


def nsa_forward_varlen(q, k, v, gates, cu_seqlens, cfg: NsaConfig, out, stream=None, check: bool = True) -> int:
    """Packed variable-length batch: q [total, H_q, d_k] etc., cu_seqlens int32 [B + 1] on the
    device (see include/nsa.h); total = q.shape[0]."""
    st = load_library().nsa_forward_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(gates), _ptr(cu_seqlens),
                                           int(q.shape[0]), ctypes.byref(cfg), _ptr(out), _stream(stream, q))
    return _check(st, "nsa_forward_varlen") if check else st


def nsa_backward(q, k, v, gates, sel_idx, dout, cfg: NsaConfig, dq, dk, dv, dgates, dw_k, dw_v, stream=None,
                 check: bool = True) -> int:
    """Gradients of the NSA forward (see include/nsa.h); every gradient buffer is fp32 and written."""
    st = load_library().nsa_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(gates), _ptr(sel_idx), _ptr(dout),
                                     ctypes.byref(cfg), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dgates), _ptr(dw_k),
                                     _ptr(dw_v), _stream(stream, q))
    return _check(st, "nsa_backward") if check else st


def nsa_backward_ex(q, k, v, gates, sel_idx, dout, cfg: NsaConfig, grads: dict, cu_seqlens=None, stream=None,
                    check: bool = True) -> int:
    """nsa_backward for the MLP phi and packed variable-length batches (see include/nsa.h).
    grads: dict of fp32 device tensors by nsa_grads field name (db_k, db_v, dw_k2, dw_v2 with the
    MLP only); cu_seqlens int32 [B + 1] on the device, or None."""
    g = NsaGrads(**{n: (_ptr(t) if t is not None else None) for n, t in grads.items()})
    total = int(q.shape[0]) if cu_seqlens is not None else 0
    st = load_library().nsa_backward_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(gates), _ptr(sel_idx), _ptr(dout),
                                        _ptr(cu_seqlens) if cu_seqlens is not None else None, total,
                                        ctypes.byref(cfg), ctypes.byref(g), _stream(stream, q))
    return _check(st, "nsa_backward_ex") if check else st


def nsa_dsa_forward(q, k, v, q_idx, k_idx, w_idx, cfg: NsaConfig, out, sel_out=None, stream=None,
                    check: bool = True) -> int:
    """DSA forward (cfg.mode = NSA_MODE_DSA): indexer heads and dim from q_idx's shape."""
    st = load_library().nsa_dsa_forward(_ptr(q), _ptr(k), _ptr(v), _ptr(q_idx), _ptr(k_idx), _ptr(w_idx),
                                        int(q_idx.shape[-2]), int(q_idx.shape[-1]), ctypes.byref(cfg), _ptr(out),
                                        _ptr(sel_out), _stream(stream, q))
    return _check(st, "nsa_dsa_forward") if check else st


def nsa_decode(q, k_cache, v_cache, kc_cache, vc_cache, seqlens, max_seqlen: int, gates, cfg: NsaConfig, out,
               stream=None, check: bool = True) -> int:
    st = load_library().nsa_decode(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(kc_cache), _ptr(vc_cache),
                                   _ptr(seqlens), int(max_seqlen), _ptr(gates), ctypes.byref(cfg), _ptr(out),
                                   _stream(stream, q))
    return _check(st, "nsa_decode") if check else st


def nsa_device_status(workspace, stream=None) -> tuple[int, int]:
    """(status, word) of the workspace's status word after synchronising the stream:
    NSA_OK with word 0, NSA_ERR_INVALID_ARG with NSA_CODE_CU_SEQLENS, or NSA_ERR_TIMEOUT with
    the code of the wait that gave up."""
    word = ctypes.c_int32(0)
    st = load_library().nsa_device_status(_ptr(workspace), ctypes.byref(word), _stream(stream, workspace))
    return st, int(word.value)


def nsa_selftest_wait_timeout(workspace, limit_us: int, stream=None, check: bool = True) -> int:
    """Launch the timeout self-test: one bounded wait that nothing releases (see include/nsa.h)."""
    st = load_library().nsa_selftest_wait_timeout(_ptr(workspace), workspace.numel() * workspace.element_size(),
                                                  int(limit_us), _stream(stream, workspace))
    return _check(st, "nsa_selftest_wait_timeout") if check else st


def nsa_forward_noalloc(q, k, v, gates, cfg: NsaConfig, out, stream=None, check: bool = True) -> int:
    """nsa_forward with the library's own fixed scratch array instead of cfg.workspace."""
    st = load_library().nsa_forward_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(gates), ctypes.byref(cfg), _ptr(out),
                                            _stream(stream, q))
    return _check(st, "nsa_forward_noalloc") if check else st


def nsa_device_status_noalloc(stream=None) -> tuple[int, int]:
    """(status, word) of the status word of the library's built-in scratch array (the one
    nsa_forward_noalloc uses on the current device), after synchronising the stream."""
    import torch
    word = ctypes.c_int32(0)
    s = _stream(stream) if stream is not None else torch.cuda.current_stream().cuda_stream
    st = load_library().nsa_device_status_noalloc(ctypes.byref(word), s)
    return st, int(word.value)
