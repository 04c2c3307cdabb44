"""GPU parity of 8-bit pooled keys (pooled_format QSA_POOLED_FP8).

Each block's f16 summary is stored as d_idx e4m3 codes and one f32 scale (amax / 448,
codes of x * 448 / amax rounded to nearest even and saturated: the FP8 K/V rule), and the
indexer scores code * scale ("Part 10", section "QSA indexer": the indexer reads one
pooled key per block; storing it in 8 bits halves the bytes the scan streams). The scan
multiplies the codes on the tensor cores (kind::f8f6f4) with the query split into five
e4m3 terms.

The chain of checks, each against something other than the library:
  - the f16 summaries themselves are pinned elsewhere (pooled rows against the oracle);
  - the codes and scales must equal, bit for bit, the oracle's quantisation of the f16
    summaries the library computes for the same tokens (a second context in f16);
  - the scores must match the oracle scoring the library's codes * scales (f64) within
    SCORE_REL, the selection must be the oracle's on those scores up to TIE_GAP_REL
    near-ties, and the attention must match the oracle over the library's own cells;
  - the decode step (scan that appends and pools) must equal the separate calls bit for bit.
"""
import numpy as np
import pytest
import torch

import synth
from oracle import qsa_oracle as O
from tests import gpu_harness as H

pytestmark = pytest.mark.gpu

FP8 = 1  # QSA_POOLED_FP8


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    H.ensure_library()


def _wl(name, heads=None):
    if name == "tiny":  # the small layer at the 8-bit scan's width (d_idx 128)
        return synth.workload("tiny", d_idx=128, n_idx_heads=heads or 4)
    return synth.workload(name)


def _pair(wl, n0, extra=16, **kw):
    """An FP8-pooled context and an f16-pooled one over the same tokens."""
    import sparse_attention_decode_02_b200 as Q
    max_ctx = (n0 + extra + 3) // 4 * 4
    pre = synth.prefill_tokens(wl, 0, n0)
    out = []
    for fmt in (FP8, 0):
        qsa = Q.Qsa(H.config_of(wl, max_ctx=max_ctx, pooled_format=fmt, **kw))
        g = H.GpuLayer(qsa)
        g.append(pre["k"], pre["v"], pre["idx"])
        out.append((qsa, g))
    return out[0], out[1], pre


def _codes(g, nb):
    torch.cuda.synchronize()
    return (g.buf["pooled_cache"][:nb].cpu().numpy(), g.buf["pooled_scales"][:nb].cpu().numpy())


def _assert_codes_quantise(g8, g16, nb):
    codes, scales = _codes(g8, nb)
    want_c, want_s = O.pooled_fp8_rows(g16.pooled_rows(0, nb))
    np.testing.assert_array_equal(scales.view(np.uint32), want_s.astype(np.float32).view(np.uint32))
    np.testing.assert_array_equal(codes, want_c)
    return codes, scales


def _decode_step(qsa, g, st):
    d = {k: H.to_dev(x) for k, x in st.items()}
    qsa.decode_step(0, d["k"], d["v"], d["idx"], d["q_idx"], d["w"], d["q"], g.outs["sel"], g.outs["n_sel"],
                    g.outs["out"])


CASES = [("tiny", 1, 1027), ("tiny", 2, 1030), ("tiny", 4, 1025), ("tiny", 8, 1029), ("tiny", 16, 1031),
         ("ctx64k", None, 61789)]


@pytest.mark.parametrize("wl_name,heads,n", CASES, ids=[f"{c[0]}-H{c[1] or 16}-n{c[2]}" for c in CASES])
def test_fp8_pooled_codes_scores_and_selection(wl_name, heads, n):
    wl = _wl(wl_name, heads)
    (q8, g8), (q16, g16), pre = _pair(wl, n)
    g8.update()
    g16.update()
    nb = n // 4
    codes, scales = _assert_codes_quantise(g8, g16, nb)
    shape = O.QsaShape.of(wl)
    for step in range(3):
        st = synth.step_inputs(wl, 0, step)
        g8.index_topk(st["q_idx"], st["w"])
        got = g8.fetch()
        ref = O.block_scores(O.dequantize_kv_rows(codes, scales), st["q_idx"], st["w"], n, shape)
        err = np.abs(got["scores"][:nb] - ref).max()
        assert err <= H.SCORE_REL * np.abs(ref).max(), f"score err {err:.3e} vs max {np.abs(ref).max():.3e}"
        H.selection_mismatch(got["sel"], ref, wl.k_blocks, H.TIE_GAP_REL)
        g8.attend_selected(st["q"])
        out = g8.fetch()["out"]
        want = O.sparse_attention(st["q"], pre["k"], pre["v"], O.expand_cells(got["sel"], n), shape)
        H.assert_attention_close(out, want)


def test_fp8_pooled_zero_query_and_equal_rows():
    """A zero indexer query scores every block 0 (the selection is the first K blocks by the
    tie rule); rows that are all equal quantise to equal codes and tie the same way."""
    wl = _wl("tiny", 4)
    (q8, g8), (q16, g16), pre = _pair(wl, 4 * 600 + 1)
    g8.update()
    st = dict(synth.step_inputs(wl, 0, 0))
    st["q_idx"] = np.zeros_like(st["q_idx"])
    g8.index_topk(st["q_idx"], st["w"])
    got = g8.fetch()
    assert got["sel"].tolist() == list(range(wl.k_blocks))
    assert not got["scores"][:600].any()
    # every row equal: the oracle's codes of one row, written into the cache
    row = synth.random_pooled(wl, 0, 1, salt=5)
    c, s = O.pooled_fp8_rows(row)
    g8.buf["pooled_cache"][:600] = H.to_dev(np.repeat(c, 600, axis=0))
    g8.buf["pooled_scales"][:600] = float(s[0])
    st = synth.step_inputs(wl, 0, 1)
    g8.index_topk(st["q_idx"], st["w"])
    got = g8.fetch()
    assert got["sel"].tolist() == list(range(wl.k_blocks))
    assert np.unique(got["scores"][:600]).size == 1


@pytest.mark.parametrize("wl_name,kw", [("tiny", {}), ("tiny", dict(rope_interleaved=True)),
                                        ("tiny", dict(kv_format=1)), ("ctx64k", {})],
                         ids=["tiny", "tiny-interleaved", "tiny-kvfp8", "ctx64k"])
def test_fp8_pooled_decode_step_equals_separate_calls(wl_name, kw):
    """The three-launch decode step (the scan appends the token and pools and quantises the
    block it completes) against the separate calls, over three block completions; the live
    codes then equal a full rebuild and the oracle's quantisation of the f16 summaries."""
    wl = _wl(wl_name)
    n0 = 1017 if wl_name == "tiny" else 8193
    (qa, ga), (q16, g16), _ = _pair(wl, n0, **kw)
    (qb, gb), _, _ = _pair(wl, n0, **kw)
    for g in (ga, gb, g16):
        g.update()
    for step in range(11):
        st = synth.step_inputs(wl, 0, step)
        _decode_step(qa, ga, st)
        qb.decode_append(0, H.to_dev(st["k"]), H.to_dev(st["v"]), H.to_dev(st["idx"]))
        gb.index_topk(st["q_idx"], st["w"])
        gb.attend_selected(st["q"])
        q16.decode_append(0, H.to_dev(st["k"]), H.to_dev(st["v"]), H.to_dev(st["idx"]))
        torch.cuda.synchronize()
        na, nb_ = int(ga.outs["n_sel"][0]), int(gb.outs["n_sel"][0])
        assert na == nb_ == min(wl.k_blocks, (n0 + step + 1) // 4)
        assert torch.equal(ga.outs["sel"][:na], gb.outs["sel"][:nb_]), f"step {step}: selection"
        assert torch.equal(ga.outs["out"], gb.outs["out"]), f"step {step}: attention output"
        assert ga.state() == gb.state() == (n0 + step + 1, (n0 + step + 1) // 4, 0)
    n = n0 + 11
    for key in ("k_cache", "v_cache", "idx_cache", "pooled_cache", "pooled_scales"):
        assert torch.equal(ga.buf[key], gb.buf[key]), key
    codes, scales = _assert_codes_quantise(ga, g16, n // 4)
    qa.invalidate_pooled_cache(0, 0)
    ga.buf["pooled_cache"].zero_()
    ga.buf["pooled_scales"].zero_()
    ga.update()
    c2, s2 = _codes(ga, n // 4)
    np.testing.assert_array_equal(c2, codes)
    np.testing.assert_array_equal(s2, scales)


def test_fp8_pooled_decode_step_matches_oracle_every_step():
    """The fused step with 8-bit pooled keys against the oracle, step by step: codes and
    scales (exact quantisation of the f16 summaries), the selection on the oracle's scores
    of those codes (near-ties only), the attention over the library's cells."""
    wl = _wl("tiny", 8)
    n0 = 1017
    (q8, g8), (q16, g16), pre = _pair(wl, n0)
    g8.update()
    g16.update()
    shape = O.QsaShape.of(wl)
    ref = O.OracleLayer(shape, max_ctx=g8.cfg.max_ctx, pooled_fp8=True)
    ref.append_tokens(pre["k"], pre["v"], pre["idx"])
    ref.update_pooled_cache()
    for step in range(9):
        st = synth.step_inputs(wl, 0, step)
        _decode_step(q8, g8, st)
        q16.decode_append(0, H.to_dev(st["k"]), H.to_dev(st["v"]), H.to_dev(st["idx"]))
        got = g8.fetch()
        r = ref.decode_step(st["k"], st["v"], st["idx"], st["q_idx"], st["w"], st["q"])
        n = ref.n
        H.assert_pooled_close(g16.pooled_rows(0, n // 4), ref.pooled.rows[: n // 4])
        codes, scales = _assert_codes_quantise(g8, g16, n // 4)
        scores = O.block_scores(O.dequantize_kv_rows(codes, scales), st["q_idx"], st["w"], n, shape)
        H.selection_mismatch(got["sel"], scores, wl.k_blocks, H.TIE_GAP_REL)
        flips = len(set(got["sel"].tolist()) ^ set(r["sel"].tolist()))
        H.record_chain("tiny-fp8-pooled", step, flips)
        cells = O.expand_cells(got["sel"], n)
        H.assert_attention_close(got["out"], O.sparse_attention(st["q"], ref.k, ref.v, cells, shape))
    assert g8.state() == (n0 + 9, (n0 + 9) // 4, 0)


def test_fp8_pooled_refuses_multi_query_and_cuda_core_scan():
    import sparse_attention_decode_02_b200 as Q
    wl = _wl("tiny")
    with pytest.raises(Q.QsaError):
        Q.Qsa(H.config_of(wl, pooled_format=FP8, scan_kind=1))
    with pytest.raises(Q.QsaError):
        Q.Qsa(H.config_of(synth.workload("tiny"), pooled_format=FP8))  # d_idx 64
