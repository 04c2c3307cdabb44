"""Thin ctypes binding of libqsa.so (include/qsa.h): argument marshalling only.

Every call takes torch tensors that already live on the GPU and passes their device
pointers and the stream handle to the C ABI; every step of the decode path runs in
the library's CUDA kernels. There is no fallback: if libqsa.so is missing or cannot be
loaded, importing the binding's library raises.
"""
from __future__ import annotations

import ctypes
import os
from ctypes import c_float, c_int32, c_size_t, c_void_p

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libqsa.so")

QSA_OK = 0
STATUS_NAMES = {0: "QSA_OK", 1: "QSA_ERR_INVALID_ARG", 2: "QSA_ERR_CAPACITY", 3: "QSA_ERR_STATE",
                4: "QSA_ERR_CUDA", 5: "QSA_ERR_UNSUPPORTED", 6: "QSA_ERR_BAD_INDEX",
                7: "QSA_ERR_TIMEOUT"}
(QSA_BUF_KV, QSA_BUF_IDX, QSA_BUF_POOLED, QSA_BUF_WORKSPACE, QSA_BUF_MAX_CELLS, QSA_BUF_SCORE_STRIDE,
 QSA_BUF_KV_SCALES, QSA_BUF_POOLED_SCALES) = range(8)
QSA_KV_F16, QSA_KV_FP8 = 0, 1
QSA_SCAN_TENSOR, QSA_SCAN_CUDA_CORES = 0, 1
QSA_POOLED_F16, QSA_POOLED_FP8 = 0, 1
QSA_INPUTS_ORDERED, QSA_INPUTS_EARLY = 0, 1
QSA_MAX_QUERIES = 4


class QsaError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


class QsaConfig(ctypes.Structure):
    _fields_ = [("n_layers", c_int32), ("max_ctx", c_int32), ("d_idx", c_int32),
                ("n_idx_heads", c_int32), ("top_k_tokens", c_int32), ("n_q_heads", c_int32),
                ("n_kv_heads", c_int32), ("head_dim", c_int32), ("rope_base", c_float),
                ("rms_eps", c_float), ("rope_dims", c_int32), ("rope_interleaved", c_int32),
                ("rope_pos_stride", c_int32), ("rope_pos_offset", c_int32), ("kv_format", c_int32),
                ("scan_kind", c_int32), ("pooled_format", c_int32), ("early_inputs", c_int32)]


class QsaLayerBuffers(ctypes.Structure):
    _fields_ = [("k_cache", c_void_p), ("v_cache", c_void_p), ("idx_cache", c_void_p),
                ("pooled_cache", c_void_p), ("rms_gain", c_void_p), ("workspace", c_void_p),
                ("kv_scales", c_void_p), ("pooled_scales", c_void_p)]


_P = c_void_p
_I = c_int32
# name -> (restype, argtypes); must list every function include/qsa.h declares
SIGNATURES = {
    "qsa_buffer_bytes": (c_size_t, [ctypes.POINTER(QsaConfig), _I]),
    "qsa_create": (_I, [ctypes.POINTER(QsaConfig), ctypes.POINTER(_P)]),
    "qsa_destroy": (None, [_P]),
    "qsa_last_error": (ctypes.c_char_p, [_P]),
    "qsa_bind_layer": (_I, [_P, _I, ctypes.POINTER(QsaLayerBuffers), _P]),
    "qsa_restore_layer": (_I, [_P, _I, _I, _I, _P]),
    "qsa_read_layer_state": (_I, [_P, _I, ctypes.POINTER(_I), ctypes.POINTER(_I), ctypes.POINTER(_I), _I, _P]),
    "qsa_append_token": (_I, [_P, _I, _P, _P, _P, _P]),
    "qsa_append_tokens": (_I, [_P, _I, _I, _P, _P, _P, _P]),
    "qsa_update_pooled_cache": (_I, [_P, _I, _P]),
    "qsa_decode_append": (_I, [_P, _I, _P, _P, _P, _P]),
    "qsa_invalidate_pooled_cache": (_I, [_P, _I, _I, _P]),
    "qsa_index_topk": (_I, [_P, _I, _P, _P, _P, _P, _P, _P]),
    "qsa_index_scores": (_I, [_P, _I, _P, _P, _P, _P]),
    "qsa_select_topk": (_I, [_P, _I, _P, _P, _P, _P]),
    "qsa_gather_kv": (_I, [_P, _I, _P, _P, _P, _P, _P, _P, _P]),
    "qsa_sparse_attend": (_I, [_P, _I, _P, _P, _P, _P, _P]),
    "qsa_sparse_attend_selected": (_I, [_P, _I, _P, _P, _P, _P, _P]),
    "qsa_sparse_attend_noalloc": (_I, [_P, _P, _P, _I, _P, _P, _P, _I, _I, _I, _I, _P]),
    "qsa_index_topk_multi": (_I, [_P, _I, _I, _P, _P, _P, _P, _P, _P]),
    "qsa_sparse_attend_selected_multi": (_I, [_P, _I, _I, _P, _P, _P, _P, _P]),
    "qsa_rollback": (_I, [_P, _I, _I, _P]),
    "qsa_layer_bytes": (c_size_t, [ctypes.POINTER(QsaConfig), _I]),
    "qsa_n_ctx": (_I, [_P, _I]),
    "qsa_get_device_status": (_I, [_P, ctypes.POINTER(_I)]),
    "qsa_decode_step": (_I, [_P, _I, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P]),
    "qsa_cp_index_candidates": (_I, [_P, _I, _P, _P, _I, _I, _P, _P, _P, _P]),
    "qsa_cp_select": (_I, [_P, _P, _I, _I, _P, _P, _P]),
    "qsa_cp_attend_partial": (_I, [_P, _I, _P, _P, _P, _I, _P, _P, _P]),
    "qsa_cp_merge": (_I, [_P, _P, _I, _I, _I, _P, _P]),
}

_lib = None


def load_library(path: str | None = None) -> ctypes.CDLL:
    """Load libqsa.so (or the library QSA_LIBRARY names, e.g. the checked build) and
    declare its signatures. Raises if it is missing."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or os.environ.get("QSA_LIBRARY") or LIB_PATH
    if not os.path.exists(p):
        raise ImportError(f"{p} is missing: build it with `python -m sparse_attention_decode_02_b200.build`")
    lib = ctypes.CDLL(p)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    if path is None:
        _lib = lib
    return lib


def _ptr(t):
    """Device pointer of a torch tensor (None -> NULL)."""
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensors passed to the QSA library must live on the GPU")
    if not t.is_contiguous():
        raise ValueError("tensors passed to the QSA library must be contiguous")
    return t.data_ptr()


def _stream(stream):
    import torch
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return getattr(stream, "cuda_stream", stream)


def make_config(n_layers, max_ctx, d_idx, n_idx_heads, top_k_tokens, n_q_heads, n_kv_heads, head_dim,
                rope_base=10000.0, rms_eps=1e-6, rope_dims=0, rope_interleaved=False, rope_pos_stride=4,
                rope_pos_offset=0, kv_format=QSA_KV_F16, scan_kind=QSA_SCAN_TENSOR,
                pooled_format=QSA_POOLED_F16, early_inputs=QSA_INPUTS_ORDERED) -> QsaConfig:
    return QsaConfig(n_layers, max_ctx, d_idx, n_idx_heads, top_k_tokens, n_q_heads, n_kv_heads, head_dim,
                     rope_base, rms_eps, rope_dims, int(bool(rope_interleaved)), rope_pos_stride, rope_pos_offset,
                     kv_format, scan_kind, pooled_format, early_inputs)


def buffer_bytes(cfg: QsaConfig, which: int) -> int:
    return int(load_library().qsa_buffer_bytes(ctypes.byref(cfg), which))


class Qsa:
    """One library context (qsa_ctx) on the current CUDA device. Method names follow the C ABI."""

    def __init__(self, cfg: QsaConfig):
        self.lib = load_library()
        self.cfg = cfg
        h = c_void_p()
        st = self.lib.qsa_create(ctypes.byref(cfg), ctypes.byref(h))
        if st != QSA_OK:
            raise QsaError(st, "qsa_create rejected the configuration")
        self.handle = h

    def close(self):
        if getattr(self, "handle", None):
            self.lib.qsa_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def _check(self, st):
        if st != QSA_OK:
            msg = self.lib.qsa_last_error(self.handle)
            raise QsaError(st, msg.decode() if msg else "")

    def buffer_bytes(self, which: int) -> int:
        return buffer_bytes(self.cfg, which)

    def bind_layer(self, layer, k_cache, v_cache, idx_cache, pooled_cache, workspace, rms_gain=None,
                   kv_scales=None, pooled_scales=None, stream=None):
        b = QsaLayerBuffers(_ptr(k_cache), _ptr(v_cache), _ptr(idx_cache), _ptr(pooled_cache),
                            _ptr(rms_gain), _ptr(workspace), _ptr(kv_scales), _ptr(pooled_scales))
        self._check(self.lib.qsa_bind_layer(self.handle, layer, ctypes.byref(b), _stream(stream)))

    def restore_layer(self, layer, n_ctx, n_pooled, stream=None):
        self._check(self.lib.qsa_restore_layer(self.handle, layer, n_ctx, n_pooled, _stream(stream)))

    def read_layer_state(self, layer, clear=False, stream=None):
        n, p, s = c_int32(), c_int32(), c_int32()
        self._check(self.lib.qsa_read_layer_state(self.handle, layer, ctypes.byref(n), ctypes.byref(p),
                                                  ctypes.byref(s), int(clear), _stream(stream)))
        return n.value, p.value, s.value

    def append_token(self, layer, k, v, idx_key, stream=None):
        self._check(self.lib.qsa_append_token(self.handle, layer, _ptr(k), _ptr(v), _ptr(idx_key),
                                              _stream(stream)))

    def append_tokens(self, layer, k, v, idx_key, stream=None):
        self._check(self.lib.qsa_append_tokens(self.handle, layer, int(k.shape[0]), _ptr(k), _ptr(v),
                                               _ptr(idx_key), _stream(stream)))

    def decode_append(self, layer, k, v, idx_key, stream=None):
        self._check(self.lib.qsa_decode_append(self.handle, layer, _ptr(k), _ptr(v), _ptr(idx_key), _stream(stream)))

    def update_pooled_cache(self, layer, stream=None):
        self._check(self.lib.qsa_update_pooled_cache(self.handle, layer, _stream(stream)))

    def invalidate_pooled_cache(self, layer, from_block, stream=None):
        self._check(self.lib.qsa_invalidate_pooled_cache(self.handle, layer, from_block, _stream(stream)))

    def index_topk(self, layer, q_idx, w, sel_blocks, n_sel, scores=None, stream=None):
        self._check(self.lib.qsa_index_topk(self.handle, layer, _ptr(q_idx), _ptr(w), _ptr(sel_blocks),
                                            _ptr(n_sel), _ptr(scores), _stream(stream)))

    def index_scores(self, layer, q_idx, w, scores, stream=None):
        self._check(self.lib.qsa_index_scores(self.handle, layer, _ptr(q_idx), _ptr(w), _ptr(scores),
                                              _stream(stream)))

    def select_topk(self, layer, scores, sel_blocks, n_sel, stream=None):
        self._check(self.lib.qsa_select_topk(self.handle, layer, _ptr(scores), _ptr(sel_blocks), _ptr(n_sel),
                                             _stream(stream)))

    def gather_kv(self, layer, sel_blocks, n_sel, cells, n_cells, k_compact=None, v_compact=None,
                  stream=None):
        self._check(self.lib.qsa_gather_kv(self.handle, layer, _ptr(sel_blocks), _ptr(n_sel), _ptr(cells),
                                           _ptr(n_cells), _ptr(k_compact), _ptr(v_compact), _stream(stream)))

    def sparse_attend_selected(self, layer, q, sel_blocks, n_sel, out, stream=None):
        self._check(self.lib.qsa_sparse_attend_selected(self.handle, layer, _ptr(q), _ptr(sel_blocks), _ptr(n_sel),
                                                        _ptr(out), _stream(stream)))

    def sparse_attend(self, layer, q, cells, n_cells, out, stream=None):
        self._check(self.lib.qsa_sparse_attend(self.handle, layer, _ptr(q), _ptr(cells), _ptr(n_cells),
                                               _ptr(out), _stream(stream)))

    def index_topk_multi(self, layer, q_idx, w, sel_blocks, n_sel, scores=None, stream=None):
        """T = q_idx.shape[0] queries (the last T tokens) in one scan and one selection."""
        self._check(self.lib.qsa_index_topk_multi(self.handle, layer, int(q_idx.shape[0]), _ptr(q_idx), _ptr(w),
                                                  _ptr(sel_blocks), _ptr(n_sel), _ptr(scores), _stream(stream)))

    def sparse_attend_selected_multi(self, layer, q, sel_blocks, n_sel, out, stream=None):
        self._check(self.lib.qsa_sparse_attend_selected_multi(self.handle, layer, int(q.shape[0]), _ptr(q),
                                                              _ptr(sel_blocks), _ptr(n_sel), _ptr(out),
                                                              _stream(stream)))

    def rollback(self, layer, n_keep, stream=None):
        self._check(self.lib.qsa_rollback(self.handle, layer, int(n_keep), _stream(stream)))

    def decode_step(self, layer, k, v, idx_key, q_idx, w, q, sel_blocks, n_sel, out, stream=None):
        """The whole hot path of one decode step of one layer in one ABI call."""
        self._check(self.lib.qsa_decode_step(self.handle, layer, _ptr(k), _ptr(v), _ptr(idx_key), _ptr(q_idx),
                                             _ptr(w), _ptr(q), _ptr(sel_blocks), _ptr(n_sel), _ptr(out),
                                             _stream(stream)))

    def cp_index_candidates(self, layer, q_idx, w, n_global, block_base, cand_scores, cand_blocks, n_cand,
                            stream=None):
        """A context-parallel shard's scan (query at global position n_global - 1) and its
        local top-K as fixed-size slots of scores and global block ids."""
        self._check(self.lib.qsa_cp_index_candidates(self.handle, layer, _ptr(q_idx), _ptr(w), int(n_global),
                                                     int(block_base), _ptr(cand_scores), _ptr(cand_blocks),
                                                     _ptr(n_cand), _stream(stream)))

    def cp_attend_partial(self, layer, q, sel_blocks, n_sel, block_base, out, lse, stream=None):
        """A context-parallel shard's attention over its part of the global selection:
        normalised output and per-head log-sum-exp."""
        self._check(self.lib.qsa_cp_attend_partial(self.handle, layer, _ptr(q), _ptr(sel_blocks), _ptr(n_sel),
                                                   int(block_base), _ptr(out), _ptr(lse), _stream(stream)))

    def n_ctx(self, layer) -> int:
        """Tokens in the layer's caches (synchronises the device)."""
        n = self.lib.qsa_n_ctx(self.handle, layer)
        if n < 0:
            raise QsaError(1, f"qsa_n_ctx failed for layer {layer}")
        return n

    def device_status(self) -> int:
        """First non-zero device status word over the bound layers (synchronises the device)."""
        st = c_int32()
        self._check(self.lib.qsa_get_device_status(self.handle, ctypes.byref(st)))
        return st.value


def cp_select(cand_scores, cand_blocks, n_shards, k_blocks, sel_blocks, n_sel, stream=None):
    """qsa_cp_select: the global top-K of every shard's candidate slots."""
    st = load_library().qsa_cp_select(_ptr(cand_scores), _ptr(cand_blocks), int(n_shards), int(k_blocks),
                                      _ptr(sel_blocks), _ptr(n_sel), _stream(stream))
    if st != QSA_OK:
        raise QsaError(st, "qsa_cp_select failed")


def cp_merge(o_parts, lse_parts, n_shards, n_q_heads, head_dim, out, stream=None):
    """qsa_cp_merge: the exact merge of the shards' attention partials."""
    st = load_library().qsa_cp_merge(_ptr(o_parts), _ptr(lse_parts), int(n_shards), int(n_q_heads), int(head_dim),
                                     _ptr(out), _stream(stream))
    if st != QSA_OK:
        raise QsaError(st, "qsa_cp_merge failed")


def sparse_attend_noalloc(q, k_cache, v_cache, n_ctx, cells, n_cells, out, n_q_heads, n_kv_heads, head_dim,
                          top_k_tokens, stream=None):
    """qsa_sparse_attend_noalloc: attention with the library's fixed scratch array (no
    context, no workspace). Raises QsaError with the returned status on failure."""
    st = load_library().qsa_sparse_attend_noalloc(_ptr(q), _ptr(k_cache), _ptr(v_cache), int(n_ctx), _ptr(cells),
                                                  _ptr(n_cells), _ptr(out), n_q_heads, n_kv_heads, head_dim,
                                                  top_k_tokens, _stream(stream))
    if st != QSA_OK:
        raise QsaError(st, "qsa_sparse_attend_noalloc failed")


def alloc_layer(cfg: QsaConfig, device="cuda"):
    """Allocate one layer's buffers with torch (the caller owns them). With QSA_KV_FP8 the
    K/V caches are uint8 e4m3 codes and `kv_scales` holds the per-row K and V scales."""
    import torch
    fp8 = cfg.kv_format == QSA_KV_FP8
    kv_dtype = torch.uint8 if fp8 else torch.float16
    shape = (cfg.max_ctx, cfg.n_kv_heads, cfg.head_dim)
    bufs = {
        "k_cache": torch.zeros(shape, dtype=kv_dtype, device=device),
        "v_cache": torch.zeros(shape, dtype=kv_dtype, device=device),
        "idx_cache": torch.zeros(cfg.max_ctx, cfg.d_idx, dtype=torch.float16, device=device),
        "pooled_cache": torch.zeros(cfg.max_ctx // 4, cfg.d_idx, device=device,
                                    dtype=torch.uint8 if cfg.pooled_format == QSA_POOLED_FP8 else torch.float16),
        "workspace": torch.zeros(buffer_bytes(cfg, QSA_BUF_WORKSPACE), dtype=torch.uint8, device=device),
    }
    assert bufs["k_cache"].numel() * bufs["k_cache"].element_size() == buffer_bytes(cfg, QSA_BUF_KV)
    if fp8:
        bufs["kv_scales"] = torch.zeros(cfg.max_ctx, cfg.n_kv_heads, 2, dtype=torch.float32, device=device)
    if cfg.pooled_format == QSA_POOLED_FP8:
        bufs["pooled_scales"] = torch.zeros(cfg.max_ctx // 4, dtype=torch.float32, device=device)
    assert bufs["pooled_cache"].numel() * bufs["pooled_cache"].element_size() == buffer_bytes(cfg, QSA_BUF_POOLED)
    return bufs


def alloc_multi_outputs(cfg: QsaConfig, n_queries: int, device="cuda"):
    """Outputs of a multi-query step: per-query selections, counts, scores and attention."""
    import torch
    k_blocks = cfg.top_k_tokens // 4
    return {
        "sel": torch.zeros(n_queries, k_blocks, dtype=torch.int32, device=device),
        "n_sel": torch.zeros(n_queries, dtype=torch.int32, device=device),
        "scores": torch.zeros(n_queries, buffer_bytes(cfg, QSA_BUF_SCORE_STRIDE), dtype=torch.float32,
                              device=device),
        "out": torch.zeros(n_queries, cfg.n_q_heads, cfg.head_dim, dtype=torch.float32, device=device),
    }


def alloc_step_outputs(cfg: QsaConfig, device="cuda"):
    """Per-step output buffers: selected blocks, cells, counts and the attention output."""
    import torch
    k_blocks = cfg.top_k_tokens // 4
    return {
        "sel": torch.zeros(k_blocks, dtype=torch.int32, device=device),
        "n_sel": torch.zeros(4, dtype=torch.int32, device=device),
        "cells": torch.zeros(4 * k_blocks + 3, dtype=torch.int32, device=device),
        "n_cells": torch.zeros(4, dtype=torch.int32, device=device),
        "out": torch.zeros(cfg.n_q_heads, cfg.head_dim, dtype=torch.float32, device=device),
    }
