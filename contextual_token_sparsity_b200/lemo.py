"""ctypes binding of liblemo.so (C ABI in include/lemo.h), same entry-point names.

Argument marshalling only: tensors become device pointers, the stream is the
current torch stream unless one is given, and a non-OK status raises
``LemoError``.  Every step of the path runs in the library's CUDA kernels;
there is no CPU fallback - if the library is missing, every call raises.
"""

from __future__ import annotations

import ctypes
import os

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "liblemo.so")

STATUS = {0: "LEMO_OK", 1: "LEMO_ERR_INVALID_ARG", 2: "LEMO_ERR_UNSUPPORTED", 3: "LEMO_ERR_CUDA",
          4: "LEMO_ERR_CAPACITY", 5: "LEMO_ERR_TIMEOUT"}
LEMO_OK = 0
LEMO_ERR_INVALID_ARG = 1
LEMO_ERR_UNSUPPORTED = 2
LEMO_ERR_CUDA = 3
LEMO_ERR_CAPACITY = 4
LEMO_ERR_TIMEOUT = 5


class LemoError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = int(status)
        super().__init__(f"{where}: {STATUS.get(self.status, self.status)}")


class lemo_shape(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int32),
        ("cu_seqlens", ctypes.c_void_p),
        ("total_L", ctypes.c_int32),
        ("max_seqlen", ctypes.c_int32),
        ("H", ctypes.c_int32),
        ("dh", ctypes.c_int32),
        ("block", ctypes.c_int32),
    ]


_P = ctypes.c_void_p
_I32 = ctypes.c_int32
_I64 = ctypes.c_int64
_SIGS = {
    "lemo_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "lemo_workspace_size": (ctypes.c_size_t, [ctypes.POINTER(lemo_shape)]),
    "lemo_block_max_elems": (_I64, [_I32, _P, _I32]),
    "lemo_score_blocks": (ctypes.c_int, [ctypes.POINTER(lemo_shape), _P, _P, ctypes.c_float, _P,
                                         _P, _P, ctypes.c_size_t, _P]),
    "lemo_score_blocks_shard": (ctypes.c_int, [ctypes.POINTER(lemo_shape), _P, _P, ctypes.c_float,
                                               _I32, _I32, _P, _P, _P, ctypes.c_size_t, _P]),
    "lemo_select": (ctypes.c_int, [ctypes.POINTER(lemo_shape), _P, ctypes.c_float, _P, _P, _P,
                                   _P, _P, ctypes.c_size_t, _P]),
    "lemo_select_static_ws": (ctypes.c_int, [ctypes.POINTER(lemo_shape), _P, ctypes.c_float, _P,
                                             _P, _P, _P, _P]),
    "lemo_gather_pad": (ctypes.c_int, [_P, _I64, _I64, _I32, _P, _P, _I32, _P, _I64, _I64, _P]),
    "lemo_scatter_residual": (ctypes.c_int, [_P, _I64, _I64, _I32, _P, _I64, _P, _P, _P]),
    "lemo_recompute_input": (ctypes.c_int, [_P, _I64, _I64, _I32, _P, _I64, _P, _P, _P]),
    "lemo_mlp_block_scores": (ctypes.c_int, [ctypes.POINTER(lemo_shape), _I32, _P, _P, _P, _I64,
                                             _P, _P, _P, ctypes.c_size_t, _P]),
    "lemo_predict_workspace_size": (ctypes.c_size_t, [ctypes.POINTER(lemo_shape), _I32, _I32]),
    "lemo_predict_scores": (ctypes.c_int, [ctypes.POINTER(lemo_shape), _I32, _P, _I64, _P, _P, _P,
                                           _P, _I32, _P, _P, ctypes.c_size_t, _P]),
    "lemo_attention_workspace_size": (ctypes.c_size_t, [_I32]),
    "lemo_attention_kept": (ctypes.c_int, [ctypes.POINTER(lemo_shape), _P, _P, _P, _I64, _P, _P,
                                           _P, ctypes.c_float, _P, _I64, _P, _I64, _P,
                                           ctypes.c_size_t, _P]),
    "lemo_segment_loss_workspace_size": (ctypes.c_size_t, [_I64, _I32, _I32]),
    "lemo_segment_loss": (ctypes.c_int, [_P, _I64, _I64, _I32, _P, _I64, _I32, _P, _I32, _I32, _P,
                                         _P, _P, _I64, _P, _I64, _P, ctypes.c_size_t, _P]),
    "lemo_get_error": (ctypes.c_int, [_P]),
    "lemo_set_test_hooks": (None, [_I32, _I64]),
    "lemo_set_predict_test_hook": (None, [_I32]),
}

_lib = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load liblemo.so (once) and declare its signatures.  Raises if absent."""
    global _lib
    if _lib is None:
        if not os.path.exists(path):
            raise RuntimeError(f"liblemo.so not found at {path}; build it with "
                               "`python -m contextual_token_sparsity_b200.build`")
        lib = ctypes.CDLL(path)
        for name, (res, args) in _SIGS.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(st: int, where: str):
    if st != LEMO_OK:
        raise LemoError(st, where)


def make_shape(cu_seqlens, total_L: int, max_seqlen: int, H: int = 1, dh: int = 64,
               block: int = 64) -> lemo_shape:
    """lemo_shape for a packed batch; ``cu_seqlens`` is a device int32 tensor."""
    return lemo_shape(int(cu_seqlens.numel()) - 1, _ptr(cu_seqlens), int(total_L),
                      int(max_seqlen), int(H), int(dh), int(block))


def lemo_workspace_size(shape: lemo_shape) -> int:
    return int(load().lemo_workspace_size(ctypes.byref(shape)))


def lemo_block_max_elems(lengths, block: int) -> int:
    arr = (ctypes.c_int32 * len(lengths))(*[int(v) for v in lengths])
    return int(load().lemo_block_max_elems(len(lengths), ctypes.cast(arr, ctypes.c_void_p), block))


def lemo_score_blocks(shape, q, k, scale, block_max, block_scores, ws, stream=None):
    _check(load().lemo_score_blocks(ctypes.byref(shape), _ptr(q), _ptr(k), float(scale),
                                    _ptr(block_max), _ptr(block_scores), _ptr(ws),
                                    ws.numel() * ws.element_size(), _stream(stream)),
           "lemo_score_blocks")


def lemo_score_blocks_shard(shape, q, k, scale, shard, nshards, block_max, block_scores, ws,
                            stream=None):
    _check(load().lemo_score_blocks_shard(ctypes.byref(shape), _ptr(q), _ptr(k), float(scale),
                                          int(shard), int(nshards), _ptr(block_max),
                                          _ptr(block_scores), _ptr(ws),
                                          ws.numel() * ws.element_size(), _stream(stream)),
           "lemo_score_blocks_shard")


def lemo_select(shape, block_scores, threshold, block_mask, kept_idx, cu_kept, kept_total, ws,
                stream=None):
    _check(load().lemo_select(ctypes.byref(shape), _ptr(block_scores), float(threshold),
                              _ptr(block_mask), _ptr(kept_idx), _ptr(cu_kept), _ptr(kept_total),
                              _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)),
           "lemo_select")


def lemo_select_static_ws(shape, block_scores, threshold, block_mask, kept_idx, cu_kept,
                          kept_total, stream=None):
    """lemo_select with the library's own device scratch (no workspace argument)."""
    _check(load().lemo_select_static_ws(ctypes.byref(shape), _ptr(block_scores), float(threshold),
                                        _ptr(block_mask), _ptr(kept_idx), _ptr(cu_kept),
                                        _ptr(kept_total), _stream(stream)),
           "lemo_select_static_ws")


def lemo_gather_pad(x, kept_idx, kept_total, pad_to, y, stream=None, d=None):
    """x [rows, ld_x] and y [capacity, ld_y] bf16/int16 2-D tensors (row-major)."""
    d = x.shape[1] if d is None else d
    _check(load().lemo_gather_pad(_ptr(x), x.stride(0), x.shape[0], int(d), _ptr(kept_idx),
                                  _ptr(kept_total), int(pad_to), _ptr(y), y.stride(0),
                                  y.shape[0], _stream(stream)),
           "lemo_gather_pad")


def lemo_scatter_residual(x, y, kept_idx, kept_total, stream=None, d=None):
    d = x.shape[1] if d is None else d
    _check(load().lemo_scatter_residual(_ptr(x), x.stride(0), x.shape[0], int(d), _ptr(y),
                                        y.stride(0), _ptr(kept_idx), _ptr(kept_total),
                                        _stream(stream)),
           "lemo_scatter_residual")


def lemo_recompute_input(x, y, kept_idx, kept_total, stream=None, d=None):
    """x [rows, ld_x] (in place), y [>= K, ld_y] bf16 2-D tensors."""
    d = x.shape[1] if d is None else d
    _check(load().lemo_recompute_input(_ptr(x), x.stride(0), x.shape[0], int(d), _ptr(y),
                                       y.stride(0), _ptr(kept_idx), _ptr(kept_total),
                                       _stream(stream)),
           "lemo_recompute_input")


def lemo_mlp_block_scores(shape, block_scores, ws, act=None, gate=None, up=None,
                          token_scores=None, stream=None):
    """act, or gate and up: bf16 [total_L, ld] tensors (d_ff = their width)."""
    ref = act if act is not None else gate
    _check(load().lemo_mlp_block_scores(ctypes.byref(shape), int(ref.shape[1]), _ptr(act),
                                        _ptr(gate), _ptr(up), ref.stride(0), _ptr(token_scores),
                                        _ptr(block_scores), _ptr(ws),
                                        ws.numel() * ws.element_size(), _stream(stream)),
           "lemo_mlp_block_scores")


def lemo_predict_workspace_size(shape: lemo_shape, d: int, rank: int) -> int:
    return int(load().lemo_predict_workspace_size(ctypes.byref(shape), int(d), int(rank)))


def lemo_predict_scores(shape, x, w1q, w2q, w1k, w2k, block_scores, ws, stream=None, d=None):
    """x [rows, ld_x] bf16; w1 [d, rank], w2 [rank, H*dh] bf16 row-major tensors."""
    d = x.shape[1] if d is None else d
    _check(load().lemo_predict_scores(ctypes.byref(shape), int(d), _ptr(x), x.stride(0),
                                      _ptr(w1q), _ptr(w2q), _ptr(w1k), _ptr(w2k),
                                      int(w1q.shape[1]), _ptr(block_scores), _ptr(ws),
                                      ws.numel() * ws.element_size(), _stream(stream)),
           "lemo_predict_scores")


def lemo_attention_workspace_size(batch: int) -> int:
    return int(load().lemo_attention_workspace_size(int(batch)))


def lemo_attention_kept(shape, q, k, v, kept_idx, cu_kept, kept_total, ws, x=None, o=None,
                        scale=None, stream=None):
    """q, k, v bf16 [total_L, ld] 2-D tensors (same stride); exactly one of x
    (residual, updated in place) or o (compact output) bf16 2-D tensors."""
    import math
    if scale is None:
        scale = 1.0 / math.sqrt(shape.dh)
    _check(load().lemo_attention_kept(
        ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), q.stride(0), _ptr(kept_idx),
        _ptr(cu_kept), _ptr(kept_total), float(scale), _ptr(x),
        x.stride(0) if x is not None else 0, _ptr(o), o.stride(0) if o is not None else 0,
        _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)),
        "lemo_attention_kept")


def lemo_segment_loss_workspace_size(T: int, V: int, seg_rows: int) -> int:
    return int(load().lemo_segment_loss_workspace_size(int(T), int(V), int(seg_rows)))


def lemo_segment_loss(h, w, targets, seg_rows, loss, ws, token_loss=None, dh=None, dw=None,
                      ignore_index=-100, stream=None):
    """h [T, ld_h] and w [V, ld_w] bf16 2-D tensors, targets int32 [T]; dh
    bf16 [T, ld_dh] and dw fp32 [V, ld_dw] optional (dw is accumulated)."""
    _check(load().lemo_segment_loss(
        _ptr(h), h.stride(0), h.shape[0], int(h.shape[1]), _ptr(w), w.stride(0), int(w.shape[0]),
        _ptr(targets), int(ignore_index), int(seg_rows), _ptr(loss), _ptr(token_loss), _ptr(dh),
        dh.stride(0) if dh is not None else 0, _ptr(dw), dw.stride(0) if dw is not None else 0,
        _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)),
        "lemo_segment_loss")


def lemo_get_error(stream=None) -> int:
    """Synchronise the stream; return (and clear) the device error status."""
    return int(load().lemo_get_error(_stream(stream)))


def lemo_set_test_hooks(select_skip_publish_tile: int = -1, spin_limit_ns: int = 0):
    load().lemo_set_test_hooks(int(select_skip_publish_tile), int(spin_limit_ns))


def lemo_set_predict_test_hook(skip_cta: int = -1):
    load().lemo_set_predict_test_hook(int(skip_cta))
