"""GPU parity of the FP8 (e4m3) K/V cache.

The Qwen3.8-Flash-Next parameter-tuning post on EVO-X2 (section "KV cacheをQ8_0にしてみる")
tried an 8-bit K/V cache. With kv_format = QSA_KV_FP8 the library stores each
(token, KV head) row as e4m3 codes of x * 448/amax with the f32 scale amax/448 and
attends over code * scale. The codes and scales must equal the oracle's byte for byte
(both sides round the same f32 values to nearest-even), and the attention must match the
oracle's attention over the dequantised rows.
"""
import numpy as np
import pytest
import torch

import synth
from oracle import qsa_oracle as O
from tests import gpu_harness as H

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    H.ensure_library()


def _pair(wl_name, n0, extra=16):
    import sparse_attention_decode_02_b200 as Q
    wl = synth.workload(wl_name)
    qsa = Q.Qsa(H.config_of(wl, max_ctx=(n0 + extra + 3) // 4 * 4, kv_format=Q.QSA_KV_FP8))
    g = H.GpuLayer(qsa)
    assert g.buf["k_cache"].dtype == torch.uint8 and "kv_scales" in g.buf
    ref = O.OracleLayer(O.QsaShape.of(wl), max_ctx=g.cfg.max_ctx, kv_fp8=True)
    pre = synth.prefill_tokens(wl, 0, n0)
    g.append(pre["k"], pre["v"], pre["idx"])          # bulk append: quantising append kernel
    g.update()
    ref.append_tokens(pre["k"], pre["v"], pre["idx"])
    ref.update_pooled_cache()
    return wl, qsa, g, ref


def _assert_cache_equal(g, ref, rows):
    torch.cuda.synchronize()
    np.testing.assert_array_equal(g.buf["k_cache"][rows].cpu().numpy(), ref.k_codes[rows])
    np.testing.assert_array_equal(g.buf["v_cache"][rows].cpu().numpy(), ref.v_codes[rows])
    np.testing.assert_array_equal(g.buf["kv_scales"][rows].cpu().numpy(), ref.kv_scales[rows])


@pytest.mark.parametrize("wl_name,n0", [("tiny", 1019), ("tiny", 1020)])
def test_fp8_codes_scales_and_attention_match_oracle(wl_name, n0):
    wl, qsa, g, ref = _pair(wl_name, n0)
    _assert_cache_equal(g, ref, slice(0, n0))
    for step in range(6):   # fused decode append (quantising) + index + attention
        st = synth.step_inputs(wl, 0, step)
        qsa.decode_append(0, H.to_dev(st["k"]), H.to_dev(st["v"]), H.to_dev(st["idx"]))
        g.index_topk(st["q_idx"], st["w"])
        g.gather()
        g.attend(st["q"])
        got = g.fetch()
        r = ref.decode_step(st["k"], st["v"], st["idx"], st["q_idx"], st["w"], st["q"])
        H.selection_mismatch(got["sel"], r["scores"], wl.k_blocks, H.CHAIN_GAP_REL)
        H.assert_attention_close(got["out"], O.sparse_attention(st["q"], ref.k, ref.v, got["cells"], ref.shape))
        # the selected-block form reads the same FP8 rows
        g.attend_selected(st["q"])
        torch.cuda.synchronize()
        np.testing.assert_allclose(g.outs["out"].cpu().numpy(), got["out"], rtol=0, atol=1e-6)
    _assert_cache_equal(g, ref, slice(0, n0 + 6))
    assert g.state()[2] == 0


def test_fp8_full_size_64k():
    wl, qsa, g, ref = _pair("ctx64k", 61789)
    rng = np.random.default_rng(5)
    _assert_cache_equal(g, ref, np.sort(rng.choice(61789, 4096, replace=False)))
    st = synth.step_inputs(wl, 0, 0)
    got = g.step(st)
    r = ref.decode_step(st["k"], st["v"], st["idx"], st["q_idx"], st["w"], st["q"])
    _assert_cache_equal(g, ref, slice(61789, 61790))
    H.selection_mismatch(got["sel"], r["scores"], wl.k_blocks, H.CHAIN_GAP_REL)
    H.assert_attention_close(got["out"], O.sparse_attention(st["q"], ref.k, ref.v, got["cells"], ref.shape))


def test_fp8_multi_query_step():
    import sparse_attention_decode_02_b200 as Q
    wl, qsa, g, ref = _pair("tiny", 1018)
    T = 3
    st = [synth.step_inputs(wl, 0, u) for u in range(T)]
    x = {k: np.stack([s[k] for s in st]) for k in st[0]}
    o = Q.alloc_multi_outputs(g.cfg, T)
    g.append(x["k"], x["v"], x["idx"])
    g.update()
    qsa.index_topk_multi(0, H.to_dev(x["q_idx"]), H.to_dev(x["w"].astype(np.float32)), o["sel"], o["n_sel"])
    qsa.sparse_attend_selected_multi(0, H.to_dev(x["q"]), o["sel"], o["n_sel"], o["out"])
    torch.cuda.synchronize()
    refs = ref.multi_query_step(x["k"], x["v"], x["idx"], x["q_idx"], x["w"], x["q"])
    _assert_cache_equal(g, ref, slice(0, 1018 + T))
    for u in range(T):
        n_u = 1018 + u + 1
        sel = o["sel"][u, : int(o["n_sel"][u])].cpu().numpy().astype(np.int64)
        H.selection_mismatch(sel, refs[u]["scores"], wl.k_blocks, H.CHAIN_GAP_REL)
        cells = O.expand_cells(sel, n_u)
        H.assert_attention_close(o["out"][u].cpu().numpy().astype(np.float64),
                                 O.sparse_attention(x["q"][u], ref.k, ref.v, cells, ref.shape))


def test_fp8_zero_rows_and_compact_gather_refused():
    import sparse_attention_decode_02_b200 as Q
    wl, qsa, g, ref = _pair("tiny", 8)
    z = {"k": np.zeros((1, wl.n_kv_heads, wl.head_dim), np.float16), "v": np.zeros((1, wl.n_kv_heads, wl.head_dim), np.float16),
         "idx": np.zeros((1, wl.d_idx), np.float16)}
    g.append(z["k"], z["v"], z["idx"])
    ref.append_tokens(z["k"], z["v"], z["idx"])
    _assert_cache_equal(g, ref, slice(0, 9))
    assert np.all(ref.kv_scales[8] == 1.0)
    kc = torch.zeros(g.cfg.top_k_tokens + 3, wl.n_kv_heads, wl.head_dim, dtype=torch.float16, device="cuda")
    with pytest.raises(Q.QsaError) as e:
        g.gather(k_compact=kc, v_compact=kc.clone())
    assert e.value.status == 5
