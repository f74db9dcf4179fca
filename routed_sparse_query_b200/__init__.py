"""Python binding of libgqe.so, the B200 (sm_100a) GQE prefill layer.

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels. Tensors are torch CUDA tensors (torch supplies device memory and
streams); each function has the name and argument order of the C entry point
it calls (see include/gqe.h) and raises ``GQEError`` on a non-OK status.

There is no CPU fallback: importing this module fails loudly when libgqe.so
is missing or cannot be loaded.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libgqe.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"libgqe.so not built ({LIB_PATH}); run python -m routed_sparse_query_b200.build")
_lib = ctypes.CDLL(LIB_PATH)

GQE_OK, GQE_ERR_INVALID, GQE_ERR_UNSUPPORTED, GQE_ERR_WORKSPACE = 0, 1, 2, 3
GQE_ERR_CUDA, GQE_ERR_TIMEOUT, GQE_ERR_DEVICE_CHECK = 4, 5, 6
GQE_WS_DISPATCH, GQE_WS_LAYER, GQE_WS_DENSE, GQE_WS_ATTENTION = 1, 2, 3, 4
GQE_WS_DECODE, GQE_WS_DENSE_DECODE, GQE_WS_BACKWARD = 5, 6, 7
GQE_FLAG_WS_CLEAN, GQE_FLAG_EXPERT_MAJOR = 1, 2
# Output constructions (at most one): see include/gqe.h.
GQE_FLAG_SLOT_GROUP_MEAN, GQE_FLAG_OUT_HARD, GQE_FLAG_OUT_WEIGHTED_CONCAT = 4, 8, 16
GQE_FLAG_NO_SHARED_HEAD = 32  # a shard of the layer split over KV groups (no shared head)
OUTPUT_MODE_FLAGS = {"gqe": 0, "group_mean": GQE_FLAG_SLOT_GROUP_MEAN, "hard": GQE_FLAG_OUT_HARD,
                     "weighted_concat": GQE_FLAG_OUT_WEIGHTED_CONCAT}
ITEMS = {"idx": 1, "r": 2, "omega": 3, "counts": 4, "offsets": 5, "tok": 6, "slot_pos": 7,
         "Qv": 8, "Qs": 9, "K": 10, "V": 11, "slots": 12, "dispatch_ws": 13, "attention_ws": 14,
         "dense_Q": 32, "dense_O": 33}

EXPORTED = ("gqe_workspace_bytes", "gqe_workspace_offset", "gqe_router_topk", "gqe_dispatch",
            "gqe_kv_proj", "gqe_attention_fwd", "gqe_output_proj", "gqe_layer_fwd",
            "gqa_dense_fwd", "gqe_read_status", "gqe_selftest_wait_timeout",
            "gqe_status_string", "gqe_version", "gqe_dispatch_noalloc", "gqe_attention_fwd_compact",
            "gqe_decode_step", "gqa_dense_decode_step", "gqe_layer_bwd")


class GQEConfig(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("T", ctypes.c_int32), ("d_model", ctypes.c_int32),
                ("G", ctypes.c_int32), ("M", ctypes.c_int32), ("k", ctypes.c_int32),
                ("d_head", ctypes.c_int32), ("flags", ctypes.c_uint32)]

    @classmethod
    def of(cls, shape, flags: int = 0) -> "GQEConfig":
        return cls(shape.B, shape.T, shape.d_model, shape.G, shape.M, shape.k, shape.d_head, flags)


class GQEError(RuntimeError):
    def __init__(self, status: int, where: str):
        msg = _lib.gqe_status_string(status).decode()
        super().__init__(f"{where}: {msg} (status {status})")
        self.status = status


_P = ctypes.c_void_p
_CFG = ctypes.POINTER(GQEConfig)
_sig = {
    "gqe_workspace_bytes": (ctypes.c_size_t, [_CFG, ctypes.c_int]),
    "gqe_workspace_offset": (ctypes.c_size_t, [_CFG, ctypes.c_int, ctypes.c_int]),
    "gqe_router_topk": (ctypes.c_int, [_CFG, _P, _P, _P, _P, _P, _P, _P]),
    "gqe_dispatch": (ctypes.c_int, [_CFG, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P,
                                    ctypes.c_size_t, _P]),
    "gqe_dispatch_noalloc": (ctypes.c_int, [_CFG, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P]),
    "gqe_kv_proj": (ctypes.c_int, [_CFG, _P, _P, _P, _P, _P, _P]),
    "gqe_attention_fwd": (ctypes.c_int, [_CFG, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "gqe_attention_fwd_compact": (ctypes.c_int, [_CFG, _P, _P, _P, _P, _P, _P, _P, _P, _P]),
    "gqe_output_proj": (ctypes.c_int, [_CFG, _P, _P, _P, _P, _P]),
    "gqe_layer_fwd": (ctypes.c_int, [_CFG, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P,
                                     ctypes.c_size_t, _P]),
    "gqa_dense_fwd": (ctypes.c_int, [_CFG, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "gqe_decode_step": (ctypes.c_int, [_CFG, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, ctypes.c_int32,
                                       _P, _P, ctypes.c_size_t, _P]),
    "gqa_dense_decode_step": (ctypes.c_int, [_CFG, _P, _P, _P, _P, _P, _P, _P, ctypes.c_int32, _P,
                                             _P, ctypes.c_size_t, _P]),
    "gqe_layer_bwd": (ctypes.c_int, [_CFG] + [_P] * 18 + [ctypes.c_size_t, _P]),
    "gqe_read_status": (ctypes.c_int, [ctypes.POINTER(ctypes.c_int32)]),
    "gqe_selftest_wait_timeout": (ctypes.c_int, [ctypes.c_uint64, _P]),
    "gqe_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "gqe_version": (ctypes.c_int, []),
}
for _name, (_res, _args) in _sig.items():
    _fn = getattr(_lib, _name)
    _fn.restype = _res
    _fn.argtypes = _args


def lib():
    return _lib


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda or not t.is_contiguous():
        raise ValueError("tensors must be contiguous CUDA tensors")
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check(status: int, where: str):
    if status != GQE_OK:
        raise GQEError(status, where)


def _cfg(cfg):
    return ctypes.byref(cfg if isinstance(cfg, GQEConfig) else GQEConfig.of(cfg))


def gqe_workspace_bytes(cfg, which: int) -> int:
    return int(_lib.gqe_workspace_bytes(_cfg(cfg), which))


def gqe_workspace_offset(cfg, which: int, item) -> int:
    item = ITEMS[item] if isinstance(item, str) else item
    return int(_lib.gqe_workspace_offset(_cfg(cfg), which, item))


def gqe_router_topk(cfg, x, W_r, b_r, idx, r, omega, stream=None):
    _check(_lib.gqe_router_topk(_cfg(cfg), _ptr(x), _ptr(W_r), _ptr(b_r), _ptr(idx), _ptr(r),
                                _ptr(omega), _stream(stream)), "gqe_router_topk")


def gqe_dispatch(cfg, idx, x, W_q, W_qs, counts, offsets, tok, slot_pos, Qv, Qs, ws, stream=None):
    _check(_lib.gqe_dispatch(_cfg(cfg), _ptr(idx), _ptr(x), _ptr(W_q), _ptr(W_qs), _ptr(counts),
                             _ptr(offsets), _ptr(tok), _ptr(slot_pos), _ptr(Qv), _ptr(Qs),
                             _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)),
           "gqe_dispatch")


def gqe_dispatch_noalloc(cfg, idx, x, W_q, W_qs, counts, offsets, tok, slot_pos, Qv, Qs,
                         stream=None):
    """gqe_dispatch for callers that cannot allocate a workspace: the scratch is
    a fixed device array of the library (see include/gqe.h)."""
    _check(_lib.gqe_dispatch_noalloc(_cfg(cfg), _ptr(idx), _ptr(x), _ptr(W_q), _ptr(W_qs),
                                     _ptr(counts), _ptr(offsets), _ptr(tok), _ptr(slot_pos),
                                     _ptr(Qv), _ptr(Qs), _stream(stream)), "gqe_dispatch_noalloc")


def gqe_kv_proj(cfg, x, W_k, W_v, K, V, stream=None):
    _check(_lib.gqe_kv_proj(_cfg(cfg), _ptr(x), _ptr(W_k), _ptr(W_v), _ptr(K), _ptr(V),
                            _stream(stream)), "gqe_kv_proj")


def gqe_attention_fwd(cfg, Qv, Qs, K, V, slots, ws, stream=None):
    _check(_lib.gqe_attention_fwd(_cfg(cfg), _ptr(Qv), _ptr(Qs), _ptr(K), _ptr(V), _ptr(slots),
                                  _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)),
           "gqe_attention_fwd")


def gqe_attention_fwd_compact(cfg, Qe, Qs, K, V, idx, offsets, tok, slots, stream=None):
    _check(_lib.gqe_attention_fwd_compact(_cfg(cfg), _ptr(Qe), _ptr(Qs), _ptr(K), _ptr(V), _ptr(idx),
                                          _ptr(offsets), _ptr(tok), _ptr(slots), _stream(stream)),
           "gqe_attention_fwd_compact")


def gqe_output_proj(cfg, slots, omega, W_o, y, stream=None):
    _check(_lib.gqe_output_proj(_cfg(cfg), _ptr(slots), _ptr(omega), _ptr(W_o), _ptr(y),
                                _stream(stream)), "gqe_output_proj")


def gqe_layer_fwd(cfg, x, W_r, b_r, W_q, W_qs, W_k, W_v, W_o, y, ws, stream=None):
    _check(_lib.gqe_layer_fwd(_cfg(cfg), _ptr(x), _ptr(W_r), _ptr(b_r), _ptr(W_q), _ptr(W_qs),
                              _ptr(W_k), _ptr(W_v), _ptr(W_o), _ptr(y), _ptr(ws),
                              ws.numel() * ws.element_size(), _stream(stream)), "gqe_layer_fwd")


def gqe_layer_bwd(cfg, x, W_r, b_r, W_q, W_qs, W_k, W_v, W_o, dy, dx, dW_r, db_r, dW_q, dW_qs, dW_k, dW_v,
                  dW_o, ws, stream=None):
    _check(_lib.gqe_layer_bwd(_cfg(cfg), _ptr(x), _ptr(W_r), _ptr(b_r), _ptr(W_q), _ptr(W_qs), _ptr(W_k),
                              _ptr(W_v), _ptr(W_o), _ptr(dy), _ptr(dx), _ptr(dW_r), _ptr(db_r), _ptr(dW_q),
                              _ptr(dW_qs), _ptr(dW_k), _ptr(dW_v), _ptr(dW_o), _ptr(ws),
                              ws.numel() * ws.element_size(), _stream(stream)), "gqe_layer_bwd")


def gqa_dense_fwd(cfg, x, W_q, W_k, W_v, W_o_dense, y, ws, stream=None):
    _check(_lib.gqa_dense_fwd(_cfg(cfg), _ptr(x), _ptr(W_q), _ptr(W_k), _ptr(W_v),
                              _ptr(W_o_dense), _ptr(y), _ptr(ws), ws.numel() * ws.element_size(),
                              _stream(stream)), "gqa_dense_fwd")


def gqe_decode_step(cfg, x, W_r, b_r, W_q, W_qs, W_k, W_v, W_o, K_cache, V_cache, y, ws,
                    stream=None):
    """cfg.T = keys after the step (the new token at T - 1); the cache capacity
    is K_cache.shape[2]."""
    _check(_lib.gqe_decode_step(_cfg(cfg), _ptr(x), _ptr(W_r), _ptr(b_r), _ptr(W_q), _ptr(W_qs),
                                _ptr(W_k), _ptr(W_v), _ptr(W_o), _ptr(K_cache), _ptr(V_cache),
                                int(K_cache.shape[2]), _ptr(y), _ptr(ws),
                                ws.numel() * ws.element_size(), _stream(stream)), "gqe_decode_step")


def gqa_dense_decode_step(cfg, x, W_q, W_k, W_v, W_o_dense, K_cache, V_cache, y, ws, stream=None):
    _check(_lib.gqa_dense_decode_step(_cfg(cfg), _ptr(x), _ptr(W_q), _ptr(W_k), _ptr(W_v),
                                      _ptr(W_o_dense), _ptr(K_cache), _ptr(V_cache),
                                      int(K_cache.shape[2]), _ptr(y), _ptr(ws),
                                      ws.numel() * ws.element_size(), _stream(stream)),
           "gqa_dense_decode_step")


def gqe_read_status() -> int:
    out = ctypes.c_int32(0)
    _check(_lib.gqe_read_status(ctypes.byref(out)), "gqe_read_status")
    return int(out.value)


def gqe_selftest_wait_timeout(limit_ns: int, stream=None):
    _check(_lib.gqe_selftest_wait_timeout(int(limit_ns), _stream(stream)),
           "gqe_selftest_wait_timeout")


def gqe_status_string(status: int) -> str:
    return _lib.gqe_status_string(status).decode()


def gqe_version() -> int:
    return int(_lib.gqe_version())


def workspace_view(ws: torch.Tensor, cfg, which: int, item, dtype, shape) -> torch.Tensor:
    """A typed view of one item of a layer / dense workspace (for inspection)."""
    off = gqe_workspace_offset(cfg, which, item)
    if off == 2 ** 64 - 1:
        raise ValueError(f"no item {item} in workspace {which}")
    n = 1
    for s in shape:
        n *= s
    nbytes = n * torch.empty((), dtype=dtype).element_size()
    return ws[off:off + nbytes].view(dtype).view(*shape)
