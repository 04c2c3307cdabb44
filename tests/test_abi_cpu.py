"""C-ABI library checks that need no GPU: it loads, exports every declared symbol, and
validates configurations and sizes on the host."""
import ctypes
import os
import re

import pytest

import sparse_attention_decode_02_b200 as qsa_pkg
from sparse_attention_decode_02_b200 import build as qbuild
from sparse_attention_decode_02_b200 import qsa as Q

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = set()
    for h in os.listdir(os.path.join(ROOT, "include")):
        if h.endswith(".h"):
            txt = open(os.path.join(ROOT, "include", h)).read()
            txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
            names |= set(re.findall(r"\b(qsa_[a-z0-9_]+)\s*\(", txt))
    return names


@pytest.fixture(scope="module")
def lib():
    qbuild.build()
    return Q.load_library()


def test_library_exports_every_declared_function(lib):
    declared = _declared()
    assert len(declared) >= 14
    for name in sorted(declared):
        assert hasattr(lib, name), f"libqsa.so does not export {name}"
    # the binding declares a signature for every function of the header
    assert declared <= set(Q.SIGNATURES), declared - set(Q.SIGNATURES)


def test_buffer_sizes(lib):
    cfg = Q.make_config(12, 255184 + 512, 128, 16, 2048, 32, 4, 128)
    assert Q.buffer_bytes(cfg, Q.QSA_BUF_KV) == cfg.max_ctx * 4 * 128 * 2
    assert Q.buffer_bytes(cfg, Q.QSA_BUF_IDX) == cfg.max_ctx * 128 * 2
    assert Q.buffer_bytes(cfg, Q.QSA_BUF_POOLED) == cfg.max_ctx // 4 * 128 * 2
    assert Q.buffer_bytes(cfg, Q.QSA_BUF_MAX_CELLS) == 2051
    ws = Q.buffer_bytes(cfg, Q.QSA_BUF_WORKSPACE)
    assert ws % 256 == 0 and ws >= 256 + cfg.max_ctx // 4 * 4


@pytest.mark.parametrize("bad", [
    dict(d_idx=96), dict(n_idx_heads=3), dict(n_idx_heads=32), dict(top_k_tokens=2046),
    dict(head_dim=256), dict(n_q_heads=32, n_kv_heads=2), dict(max_ctx=1026), dict(max_ctx=4 << 20),
    dict(top_k_tokens=4096), dict(top_k_tokens=0),
    dict(n_layers=0),
    dict(rope_dims=33), dict(rope_dims=130), dict(rope_dims=-2), dict(rope_interleaved=2),
    dict(rope_pos_stride=17), dict(rope_pos_stride=-1), dict(rope_pos_offset=-1),
    dict(rope_pos_offset=(1 << 20) + 1),
])
def test_unsupported_configs_are_rejected(lib, bad):
    base = dict(n_layers=1, max_ctx=4096, d_idx=128, n_idx_heads=16, top_k_tokens=2048, n_q_heads=32,
                n_kv_heads=4, head_dim=128)
    cfg = Q.make_config(**{**base, **{k: v for k, v in bad.items() if k in base}})
    for k, v in bad.items():  # raw struct fields, past the binding's own conversions
        setattr(cfg, k, v)
    assert Q.buffer_bytes(cfg, Q.QSA_BUF_KV) == 0
    h = ctypes.c_void_p()
    assert lib.qsa_create(ctypes.byref(cfg), ctypes.byref(h)) == 5  # QSA_ERR_UNSUPPORTED
    assert not h.value


def test_config_struct_matches_header():
    import re
    with open(os.path.join(ROOT, "include", "qsa.h")) as f:
        text = f.read()
    body = re.search(r"typedef struct \{(.*?)\} qsa_config;", text, re.S).group(1)
    body = re.sub(r"/\*.*?\*/", "", body, flags=re.S)
    fields = re.findall(r"(int32_t|float)\s+(\w+);", body)
    ctype = {"int32_t": ctypes.c_int32, "float": ctypes.c_float}
    assert [(n, ctype[t]) for t, n in fields] == list(Q.QsaConfig._fields_)


def test_buffers_struct_matches_header():
    import re
    with open(os.path.join(ROOT, "include", "qsa.h")) as f:
        text = f.read()
    body = re.search(r"typedef struct \{([^{}]*?)\} qsa_layer_buffers;", text, re.S).group(1)
    body = re.sub(r"/\*.*?\*/", "", body, flags=re.S)
    names = re.findall(r"\*\s*(\w+);", body)
    assert names == [n for n, _ in Q.QsaLayerBuffers._fields_]
    assert all(t is ctypes.c_void_p for _, t in Q.QsaLayerBuffers._fields_)


def test_fp8_buffer_sizes(lib):
    cfg = Q.make_config(1, 4096, 128, 16, 2048, 32, 4, 128, kv_format=Q.QSA_KV_FP8)
    assert Q.buffer_bytes(cfg, Q.QSA_BUF_KV) == 4096 * 4 * 128
    assert Q.buffer_bytes(cfg, Q.QSA_BUF_KV_SCALES) == 4096 * 4 * 2 * 4
    f16 = Q.make_config(1, 4096, 128, 16, 2048, 32, 4, 128)
    assert Q.buffer_bytes(f16, Q.QSA_BUF_KV) == 2 * Q.buffer_bytes(cfg, Q.QSA_BUF_KV)
    assert Q.buffer_bytes(f16, Q.QSA_BUF_KV_SCALES) == 0
    assert Q.buffer_bytes(cfg, Q.QSA_BUF_SCORE_STRIDE) == 1024
    bad = Q.make_config(1, 4096, 128, 16, 2048, 32, 4, 128)
    bad.kv_format = 2
    assert Q.buffer_bytes(bad, Q.QSA_BUF_KV) == 0


def test_scan_kind_is_validated(lib):
    cfg = Q.make_config(1, 4096, 128, 16, 2048, 32, 4, 128, scan_kind=Q.QSA_SCAN_CUDA_CORES)
    assert Q.buffer_bytes(cfg, Q.QSA_BUF_KV) == 4096 * 4 * 128 * 2
    cfg.scan_kind = 2
    assert Q.buffer_bytes(cfg, Q.QSA_BUF_KV) == 0


def test_pooled_format_and_early_inputs_are_validated(lib):
    cfg = Q.make_config(1, 4096, 128, 16, 2048, 32, 4, 128, pooled_format=Q.QSA_POOLED_FP8,
                        early_inputs=Q.QSA_INPUTS_EARLY)
    assert Q.buffer_bytes(cfg, Q.QSA_BUF_POOLED) == 1024 * 128
    assert Q.buffer_bytes(cfg, Q.QSA_BUF_POOLED_SCALES) == 1024 * 4
    cfg.early_inputs = 2
    assert Q.buffer_bytes(cfg, Q.QSA_BUF_POOLED) == 0
    d64 = Q.make_config(1, 4096, 64, 16, 2048, 32, 4, 128, pooled_format=Q.QSA_POOLED_FP8)
    assert Q.buffer_bytes(d64, Q.QSA_BUF_POOLED) == 0  # 8-bit pooled keys need d_idx 128


def test_null_arguments_are_rejected(lib):
    assert lib.qsa_create(None, None) == 1
    lib.qsa_destroy(None)  # no-op
    assert lib.qsa_last_error(None) == b"null context"
    assert lib.qsa_n_ctx(None, 0) == -1
    st = ctypes.c_int32(7)
    assert lib.qsa_get_device_status(None, ctypes.byref(st)) == 1
    assert lib.qsa_decode_step(None, 0, *([None] * 9), None) == 1
    assert lib.qsa_rollback(None, 0, 0, None) == 1
    assert lib.qsa_index_topk_multi(None, 0, 1, *([None] * 5), None) == 1


def test_layer_bytes_is_buffer_bytes(lib):
    cfg = Q.make_config(12, 255184 + 512, 128, 16, 2048, 32, 4, 128)
    for which in range(8):
        assert lib.qsa_layer_bytes(ctypes.byref(cfg), which) == Q.buffer_bytes(cfg, which)


def test_binding_has_no_fallback(tmp_path):
    with pytest.raises(ImportError):
        Q.load_library(str(tmp_path / "missing.so"))
    assert qsa_pkg.Qsa is Q.Qsa


@pytest.mark.slow
def test_checked_build_compiles_and_exports(tmp_path):
    """The checked build (-DQSA_CHECKED bounds guards) compiles, links and exports the ABI."""
    lib_path = qbuild.build(checked=True)
    assert lib_path.endswith("libqsa_checked.so") and os.path.exists(lib_path)
    lib = Q.load_library(lib_path)
    for name in _declared():
        assert hasattr(lib, name), name
    cfg = Q.make_config(1, 4096, 128, 16, 2048, 32, 4, 128)
    assert lib.qsa_buffer_bytes(ctypes.byref(cfg), Q.QSA_BUF_MAX_CELLS) == 2051
